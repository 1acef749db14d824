// gemm_pair_sm100.cu -- the down projection of the grouped expert GEMMs on CTA pairs
// (tcgen05 cta_group::2); the gate/up projection's pair kernel is gemm_gateup_pair_sm100.cu.
//
// Same contraction, groups and tile order as gemm_sm100.cu (DeepSeekMoE summary,
// shared-expert layer equation):   Y[r, n] = sum_k A1[r,k] W_down[e,n,k]
// but each tile is computed by a cluster of two CTAs on neighbouring SMs with one M=256
// MMA per K step (weights on M, tokens on N, N = the tile's token count rounded up to
// 16, at most 256). Each SM stages only its own 128 weight rows and half of the token
// rows, so per MAC it stages and reads half the operand bytes of a one-CTA M=128, N=128
// MMA. Its outputs are bit-identical to the one-CTA kernel's.
//
// Tile of a pair (even CTA = rank 0, odd = rank 1): 256 output rows, rank r holds rows
// 128r..128r+127; token rows: rank 0 stages row0.., rank 1 row0+N/2.. (the MMA's B
// columns N/2..N-1 come from the odd CTA).
//
// Roles (192 threads per CTA):
//   warp 0     TMA producer of this CTA's half of every stage (6 stages of 32 KB); all
//              copies complete on the even CTA's `landed` barrier, on which the even
//              producer alone expects the pair's bytes.
//   warp 1     allocates the pair's 512 TMEM columns (two 256-column accumulators); in
//              the even CTA one thread issues the MMAs and commits to the `empty` and
//              `acc_full` barriers of both CTAs.
//   warps 2-5  epilogue of this CTA's 128 accumulator rows; one lane per warp releases
//              the accumulator on the even CTA's `acc_empty` barrier.
// Every wait is bounded; a role that gives up raises the abort flag of both CTAs and a
// status bit. At the end the even CTA waits (at least one second) for every copy either
// CTA issued and for its MMAs, and only then may either CTA release TMEM and exit.
#include "grouped_tiles.cuh"
#include "sm100_pair_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kBK = 64;
constexpr int kMmaK = 16;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kTok = kGemmPairTokenTile;            // the MMA's largest N
constexpr int kRowsPerCta = 128;                    // weight rows and token rows per CTA
constexpr uint32_t kABytes = kRowsPerCta * kBK * 2;  // 16 KB
constexpr uint32_t kBBytes = kRowsPerCta * kBK * 2;  // 16 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kStages = 6;
constexpr int kBufs = 2;
constexpr uint32_t kAccCols = kTok;
constexpr uint32_t kStageRow = 33;

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffBars = kOffB + kStages * kBBytes;
// landed, empty, acc_full, acc_empty, drain
constexpr uint32_t kNumBars = 2 * kStages + 2 * kBufs + 1;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;      // tmem slot, abort, never, pad, issued[kStages]
constexpr uint32_t kOffTiles = (kOffMisc + 16 + kStages * 4 + 15) & ~15u;
constexpr uint32_t kOffEpi = (kOffTiles + (kGemmMaxGroups + 1) * 4 + 15) & ~15u;
constexpr uint32_t kSmemUsed = kOffEpi + 4 * 32 * kStageRow * 4;  // per warp a 32 x 33 fp32 transpose tile
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack to align the ring to 1024 bytes
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kBufs * kAccCols <= kTmemCols, "TMEM budget");

__global__ void __launch_bounds__(kThreads, 1) down_pair_kernel(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* sA = base + kOffA;
  uint8_t* sB = base + kOffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* landed = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + kBufs;
  uint64_t* drain = acc_empty + kBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 8);
  uint32_t* issued_n = reinterpret_cast<uint32_t*>(base + kOffMisc + 16);
  int32_t* tile_start = reinterpret_cast<int32_t*>(base + kOffTiles);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = pair::cta_rank();
  const bool even = rank == 0;
  const int G = a.n_shared_groups + a.n_routed;
  const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  tile_counts<kTok>(a, tile_start, G);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *never_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&landed[s], 1);
      mbar_init(&empty[s], 1);
      issued_n[s] = 0;
    }
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * 4);  // one lane of each epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    pair::tmem_alloc(tmem_slot, kTmemCols);
    pair::tmem_relinquish();
  }
  __syncthreads();
  if (warp == 0) tile_scan(tile_start, G, lane);
  tc_fence_before();
  __syncthreads();
  pair::cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[G];
  const uint32_t peer_abort = pair::map_to(smem_addr(const_cast<int*>(abort_flag)), rank ^ 1u);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&a.a_routed);
      tma_prefetch_desc(&a.b0_routed);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += n_pairs) {
        const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
        const int n_mma = (t.m_valid + 15) & ~15;
        const int brow = t.row0 + (even ? 0 : n_mma / 2);
        const CUtensorMap* tx = t.shared ? &a.a_shared : &a.a_routed;
        const CUtensorMap* tw0 = t.shared ? &a.b0_shared : &a.b0_routed;
        const int kb_per = t.shared ? a.kb_per_b_expert_shared : t.kb_n;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!pair::mbar_wait_bounded_cl(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = pair::map_to(smem_addr(&landed[stage]), 0);
          if (even) mbar_arrive_expect_tx(&landed[stage], 2 * kStageBytes);
          const int be = t.expert + kb / kb_per;
          const int bk = (kb % kb_per) * kBK;
          uint8_t* sa = sA + stage * kABytes;  // 128 consecutive output rows
          pair::tma_load_3d_pair(sa, tw0, bar, bk, t.n_blk * 2 * kRowsPerCta + static_cast<int>(rank) * kRowsPerCta, be);
          pair::tma_load_2d_pair(sB + stage * kBBytes, tx, bar, kb * kBK, brow);
          issued_n[stage] += 1;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        pair::st_cluster_u32(peer_abort, 1);
        atomicOr(a.status, kStatusTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    if (even && lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair_id; ok && tile < total; tile += n_pairs, ++it) {
        const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
        const int n_mma = (t.m_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(2 * kRowsPerCta, n_mma);
        const int acc = it % kBufs;
        if (!pair::mbar_wait_bounded_cl(&acc_empty[acc], ((it / kBufs) & 1) ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!pair::mbar_wait_bounded_cl(&landed[stage], phase, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_kmajor_sw128(smem_addr(sA + stage * kABytes));
          const uint64_t bd = smem_desc_kmajor_sw128(smem_addr(sB + stage * kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            const uint64_t dk = static_cast<uint64_t>(2 * k);
            pair::mma_bf16_ss(d0, ad + dk, bd + dk, idesc, (kb | k) ? 1u : 0u);
          }
          pair::mma_commit_both(&empty[stage], 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        pair::mma_commit_both(&acc_full[acc], 0x3);
      }
      if (!ok) {
        *abort_flag = 1;
        pair::st_cluster_u32(peer_abort, 1);
        atomicOr(a.status, kStatusTimeoutMma);
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    const int q = warp & 3;  // this warp may read TMEM lanes [32q, 32q+32)
    float* stg = reinterpret_cast<float*>(base + kOffEpi) + q * 32 * kStageRow;
    int it = 0;
    bool ok = true;
    for (int tile = pair_id; ok && tile < total; tile += n_pairs, ++it) {
      const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
      const int acc = it % kBufs;
      if (!pair::mbar_wait_warp_sleepy_cl(&acc_full[acc], (it / kBufs) & 1, a.wait_limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      const int n_valid = t.shared ? a.n_valid_shared : a.n_valid_routed;
      const int64_t ld = t.shared ? a.ld_shared : a.ld_routed;
      {
        // thread of TMEM lane l holds output row feat_base + l; per 32 tokens the warp
        // transposes its 32 rows x 32 tokens and lane L stores 8 consecutive outputs of
        // token L/4 + 8i (16 B of bf16, or 32 B of fp32 with the residual added)
        const bool f32_out = t.shared && a.out_shared_f32 != nullptr;
        const int rr = lane >> 2, cc = (lane & 3) * 8;
        const int feat = t.n_blk * 2 * kRowsPerCta + static_cast<int>(rank) * kRowsPerCta + q * 32 + cc;
        const bool ok_f = feat < n_valid;  // n_valid is a multiple of 64, feat of 8
#pragma unroll 1
        for (int c0 = 0; c0 < t.m_valid; c0 += 32) {
          uint32_t v[32];
          tmem_ld16(tb + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          tmem_ld16(tb + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[j * kStageRow + lane] = __uint_as_float(v[j]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = rr + 8 * i;
            if (ok_f && c0 + row < t.m_valid) {
              const float* src = stg + row * kStageRow + cc;
              const int64_t o = static_cast<int64_t>(t.row0 + c0 + row) * ld + feat;
              if (f32_out) {
                const uint4 rv = *reinterpret_cast<const uint4*>(a.residual + o);
                const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
                float out8[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 xr = unpack_bf16x2(rw[k]);
                  out8[2 * k] = src[2 * k] + xr.x;
                  out8[2 * k + 1] = src[2 * k + 1] + xr.y;
                }
                float4* dst = reinterpret_cast<float4*>(a.out_shared_f32 + o);
                dst[0] = make_float4(out8[0], out8[1], out8[2], out8[3]);
                dst[1] = make_float4(out8[4], out8[5], out8[6], out8[7]);
              } else {
                bf16* obase = t.shared ? a.out_shared + static_cast<int64_t>(t.group) * a.shared_col_stride
                                       : a.out_routed;
                *reinterpret_cast<uint4*>(obase + o) =
                    make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                               pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
              }
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::mbar_arrive_cluster(pair::map_to(smem_addr(&acc_empty[acc]), 0));
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      pair::st_cluster_u32(peer_abort, 1);
      atomicOr(a.status, kStatusTimeoutEpilogue);
    }
  }

  // ---------------------------------------------------------------------- teardown
  // Without an abort every copy was consumed by an MMA and every MMA was observed
  // complete by both epilogues, so only an abort needs the bounded drain.
  __syncthreads();
  pair::cluster_sync();  // every role of both CTAs has finished issuing
  if (even && *abort_flag) {  // (a role of either CTA gave up: both flags are set)
    if (warp == 0 && lane == 0) {
      // the last phase of each stage that either CTA loaded must have landed
      for (int s = 0; s < kStages; ++s) {
        const uint32_t n_peer = pair::ld_cluster_u32(pair::map_to(smem_addr(&issued_n[s]), 1));
        const uint32_t n = max(issued_n[s], n_peer);
        if (n > 0 &&
            !pair::mbar_wait_bounded_cl(&landed[s], (n - 1) & 1u, drain_wait_limit(a.wait_limit_ns), never_flag))
          atomicOr(a.status, kStatusTimeoutDrain);
      }
    }
    if (warp == 1 && lane == 0) {
      pair::mma_commit_local(drain);
      if (!pair::mbar_wait_bounded_cl(drain, 0, drain_wait_limit(a.wait_limit_ns), never_flag))
        atomicOr(a.status, kStatusTimeoutDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  pair::cluster_sync();  // copies into, and MMAs on, both CTAs' memories have completed
  if (warp == 1) {
    tc_fence_after();
    pair::tmem_dealloc(tmem_base, kTmemCols);
  }
}

cudaLaunchConfig_t pair_config(int clusters, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = 2;
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
}  // namespace

int down_pair_max_clusters() {
  if (cudaFuncSetAttribute(down_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes)) != cudaSuccess)
    return 0;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t cfg = pair_config(1, nullptr, &attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, down_pair_kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_down_pair(const GemmArgs& a, int clusters, cudaStream_t s) {
  if (a.n_shared_groups + a.n_routed > kGemmMaxGroups) return cudaErrorInvalidValue;
  if (clusters < 1) clusters = 1;
  cudaError_t e = cudaFuncSetAttribute(down_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t cfg = pair_config(clusters, s, &attr);
  return cudaLaunchKernelEx(&cfg, down_pair_kernel, a);
}

}  // namespace dsmoe
