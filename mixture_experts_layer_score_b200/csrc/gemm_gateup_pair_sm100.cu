// gemm_gateup_pair_sm100.cu -- the gate/up projection with SiLU(gate) * up on CTA pairs
// (tcgen05 cta_group::2), in the tile shape that moves the fewest operand bytes per MAC.
//
// Per routed expert (and per shared expert over all tokens; DeepSeekMoE summary,
// shared-expert layer equation; SwiGLU form on the "MoE: sparse activation" page):
//   A1[r, n] = SiLU(sum_k X[r,k] W_gate[e,n,k]) * (sum_k X[r,k] W_up[e,n,k])
// A tile is 256 features by up to 256 tokens, computed by a cluster of two CTAs with two
// M=256 MMA chains per K step, one for W_gate and one for W_up, that share the token
// operand. CTA rank r stages the gate rows and the up rows of features f0+128r ..
// f0+128r+127 (two 128-row TMA boxes) and token rows r*N/2 .. of the tile; the pair's MMA
// reads each CTA's weight rows from its own shared memory and the token columns from
// both. Its TMEM then holds, for its 128 features, the gate sums in columns [0, N) and
// the up sums in [256, 256 + N) of the same lane, so the epilogue combines them without
// any exchange between warps or CTAs.
//
// Bytes staged per SM per MAC: each SM loads 256 weight rows and 128 token rows per 64-wide
// K block for 128 x 256 x 64 x 2 MACs, half of the one-CTA kernel's (256 weight rows and
// 128 token rows for 128 x 128 x 64 x 2 MACs), so the 4-stage, 192 KB ring covers twice
// as much MMA time against the latency of the operand loads. The price is one accumulator
// (the tile's two chains take all 512 TMEM columns): the MMAs of the next tile wait for
// this tile's epilogue, which eight warps keep short while the producer refills the ring.
//
// Roles (320 threads per CTA):
//   warp 0     TMA producer of this CTA's part of every stage; all copies complete on the
//              even CTA's `landed` barrier, where the even producer alone expects the
//              pair's bytes.
//   warp 1     allocates the pair's 512 TMEM columns; in the even CTA one thread issues the
//              MMAs and commits to the `empty` and `acc_full` barriers of both CTAs.
//   warps 2-9  epilogue: warps 2+q and 6+q read TMEM lanes [32q, 32q+32) (features) for
//              alternate 32-token chunks, apply SiLU(g) * u in fp32, round to bf16, transpose
//              through shared memory and store 16-byte vectors along output rows; with
//              save_ab set they also store the pre-activations g and u (backward pass).
// Every wait is bounded; a role that gives up raises the abort flag of both CTAs and a
// status bit; the even CTA then waits (at least one second) for every copy either CTA
// issued and for its MMAs, and only then may either CTA release TMEM and exit.
#include "grouped_tiles.cuh"
#include "sm100_pair_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kBK = 64;
constexpr int kMmaK = 16;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr int kTok = kGemmPairTokenTile;             // 256: the MMA's largest N
constexpr int kRows = 128;                           // weight rows per chain per CTA, token rows per CTA
constexpr uint32_t kWBytes = 2 * kRows * kBK * 2;   // 32 KB: gate rows then up rows
constexpr uint32_t kXBytes = kRows * kBK * 2;       // 16 KB
constexpr uint32_t kStageBytes = kWBytes + kXBytes;
constexpr int kStages = 4;
constexpr uint32_t kUpCol = 256;                     // TMEM column of the up chain
constexpr uint32_t kStgRow = 40;                     // bf16 staging row: 32 features + 8 pad (80 B)
constexpr uint32_t kOffW = 0;
constexpr uint32_t kOffX = kOffW + kStages * kWBytes;
constexpr uint32_t kOffBars = kOffX + kStages * kXBytes;
constexpr uint32_t kNumBars = 2 * kStages + 2 + 1;  // landed, empty, acc_full, acc_empty, drain
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;  // tmem slot, abort, never, pad, issued[kStages]
constexpr uint32_t kOffTiles = (kOffMisc + 16 + kStages * 4 + 15) & ~15u;
constexpr uint32_t kOffEpi = (kOffTiles + (kGemmMaxGroups + 1) * 4 + 15) & ~15u;
constexpr uint32_t kSmemUsed = kOffEpi + kEpiWarps * 32 * kStgRow * 2;
constexpr size_t kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(2 * kUpCol <= kTmemCols && kTok <= 256, "TMEM budget");

__global__ void __launch_bounds__(kThreads, 1) gateup_pair_kernel(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* sW = base + kOffW;
  uint8_t* sX = base + kOffX;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* landed = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
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
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);  // one lane of each epilogue warp of both CTAs
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
      tma_prefetch_desc(&a.b1_routed);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += n_pairs) {
        const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
        const int n_mma = (t.m_valid + 15) & ~15;
        const int xrow = t.row0 + (even ? 0 : n_mma / 2);
        const int f0 = t.n_blk * 2 * kRows + static_cast<int>(rank) * kRows;
        const CUtensorMap* tx = t.shared ? &a.a_shared : &a.a_routed;
        const CUtensorMap* tg = t.shared ? &a.b0_shared : &a.b0_routed;
        const CUtensorMap* tu = t.shared ? &a.b1_shared : &a.b1_routed;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!pair::mbar_wait_bounded_cl(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = pair::map_to(smem_addr(&landed[stage]), 0);
          if (even) mbar_arrive_expect_tx(&landed[stage], 2 * kStageBytes);
          uint8_t* w = sW + stage * kWBytes;
          pair::tma_load_3d_pair(w, tg, bar, kb * kBK, f0, t.expert);
          pair::tma_load_3d_pair(w + kWBytes / 2, tu, bar, kb * kBK, f0, t.expert);
          pair::tma_load_2d_pair(sX + stage * kXBytes, tx, bar, kb * kBK, xrow);
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
        const uint32_t idesc = idesc_bf16_f32(2 * kRows, n_mma);
        if (!pair::mbar_wait_bounded_cl(acc_empty, (it & 1) ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!pair::mbar_wait_bounded_cl(&landed[stage], phase, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t gd = smem_desc_kmajor_sw128(smem_addr(sW + stage * kWBytes));
          const uint64_t ud = smem_desc_kmajor_sw128(smem_addr(sW + stage * kWBytes + kWBytes / 2));
          const uint64_t xd = smem_desc_kmajor_sw128(smem_addr(sX + stage * kXBytes));
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            const uint64_t dk = static_cast<uint64_t>(2 * k);
            const uint32_t accum = (kb | k) ? 1u : 0u;
            pair::mma_bf16_ss(tmem_base, gd + dk, xd + dk, idesc, accum);
            pair::mma_bf16_ss(tmem_base + kUpCol, ud + dk, xd + dk, idesc, accum);
          }
          pair::mma_commit_both(&empty[stage], 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        pair::mma_commit_both(acc_full, 0x3);
      }
      if (!ok) {
        *abort_flag = 1;
        pair::st_cluster_u32(peer_abort, 1);
        atomicOr(a.status, kStatusTimeoutMma);
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    // Warp w (2..9) reads TMEM lanes [32q, 32q+32) with q = w % 4, i.e. features
    // f0 + 32q + lane of this CTA's 128, and takes the 32-token chunks c with
    // c % 2 == (w - 2) / 4. Per chunk: SiLU(g) * u -> bf16 -> a 32 x 32 transpose in shared
    // memory -> lane L stores the 8 features cc.. of token row L/4 + 8i (16 bytes).
    const int q = warp & 3, half = (warp - 2) >> 2;
    uint16_t* stg = reinterpret_cast<uint16_t*>(base + kOffEpi) + (warp - 2) * 32 * kStgRow;
    const int rr = lane >> 2, cc = (lane & 3) * 8;
    int it = 0;
    bool ok = true;
    for (int tile = pair_id; ok && tile < total; tile += n_pairs, ++it) {
      const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
      if (!pair::mbar_wait_warp_sleepy_cl(acc_full, it & 1, a.wait_limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      const int n_valid = t.shared ? a.n_valid_shared : a.n_valid_routed;  // F or F_s
      const int64_t ld = t.shared ? a.ld_shared : a.ld_routed;
      bf16* obase = t.shared ? a.out_shared + static_cast<int64_t>(t.group) * a.shared_col_stride : a.out_routed;
      bf16* save = t.shared ? a.save_ab_shared : a.save_ab_routed;
      const int64_t lds = 2 * ld;
      const int64_t scol = t.shared ? static_cast<int64_t>(t.group) * 2 * n_valid : 0;
      const int feat = t.n_blk * 2 * kRows + static_cast<int>(rank) * kRows + q * 32 + cc;
      const bool ok_f = feat < n_valid;  // n_valid is a multiple of 64, feat of 8
#pragma unroll 1
      for (int c0 = 32 * half; c0 < t.m_valid; c0 += 64) {
        uint32_t g[32], u[32];
        tmem_ld16(tb + c0, *reinterpret_cast<uint32_t(*)[16]>(&g[0]));
        tmem_ld16(tb + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&g[16]));
        tmem_ld16(tb + kUpCol + c0, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
        tmem_ld16(tb + kUpCol + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
        tmem_wait_ld();
        const int n_out = save ? 3 : 1;  // A1, then (backward pass) a and b
#pragma unroll 1
        for (int o = 0; o < n_out; ++o) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
            const float v = o == 0 ? __fdividef(gv, 1.0f + __expf(-gv)) * uv : (o == 1 ? gv : uv);
            stg[j * kStgRow + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = rr + 8 * i;
            if (ok_f && c0 + row < t.m_valid) {
              const uint4 v = *reinterpret_cast<const uint4*>(stg + row * kStgRow + cc);
              const int64_t r = t.row0 + c0 + row;
              bf16* dst = o == 0 ? obase + r * ld + feat : save + r * lds + scol + (o - 1) * n_valid + feat;
              *reinterpret_cast<uint4*>(dst) = v;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::mbar_arrive_cluster(pair::map_to(smem_addr(acc_empty), 0));
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      pair::st_cluster_u32(peer_abort, 1);
      atomicOr(a.status, kStatusTimeoutEpilogue);
    }
  }

  // ---------------------------------------------------------------------- teardown
  __syncthreads();
  pair::cluster_sync();  // every role of both CTAs has finished issuing
  if (even && *abort_flag) {
    if (warp == 0 && lane == 0) {
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

cudaLaunchConfig_t config(int clusters, cudaStream_t s, cudaLaunchAttribute* attr) {
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

int gateup_pair_max_clusters() {
  if (cudaFuncSetAttribute(gateup_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes)) != cudaSuccess)
    return 0;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t cfg = config(1, nullptr, &attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gateup_pair_kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_gateup_pair(const GemmArgs& a, int clusters, cudaStream_t s) {
  if (a.n_shared_groups + a.n_routed > kGemmMaxGroups) return cudaErrorInvalidValue;
  if (clusters < 1) clusters = 1;
  cudaError_t e = cudaFuncSetAttribute(gateup_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t cfg = config(clusters, s, &attr);
  return cudaLaunchKernelEx(&cfg, gateup_pair_kernel, a);
}

}  // namespace dsmoe
