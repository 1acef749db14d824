// gemm_bwd_sm100.cu -- the grouped GEMMs of the experts' backward pass (data gradients)
// on the 5th-generation tensor cores, with the weights read in the layout the forward
// uses (nn.Linear [out, in], in contiguous), which for these contractions is MN-major.
//
// For an expert FFN y = W_down m, m = SiLU(a) * b, a = W_gate u, b = W_up u (DeepSeekMoE
// summary, shared-expert layer equation; SwiGLU form noted on the "MoE: sparse
// activation" page) and an output gradient dy (g * dh for a routed pick, dh for a shared
// expert):
//   dm = W_down^T dy,  da = dm * b * SiLU'(a),  db = dm * SiLU(a),
//   du = W_gate^T da + W_up^T db,   SiLU'(a) = sigma(a) (1 + a (1 - sigma(a))).
// Two kernels over the forward's tile schedule (grouped_tiles.cuh):
//   kDM: D^T[f, s] = sum_n W_down[e][n, f] dy[s, n]: A = W_down viewed [K = d rows,
//        M = F cols] (MN-major), B = dy rows (K-major). The epilogue reads the forward's
//        saved pre-activations a, b of the same (slot, f) and writes da | db side by side.
//   kDX: D^T[n, s] = sum_f W_gate[e][f, n] da[s, f] + sum_f W_up[e][f, n] db[s, f]: A =
//        W_gate then W_up viewed [K = F rows, M = d cols] (MN-major), B = the da | db rows
//        (K = 2F, K-major). Routed rows are written as bf16 per slot; the shared experts
//        form one group whose K loop runs over every shared expert's da | db and whose
//        fp32 rows sum all of them.
// Both: one CTA per SM, 320 threads (warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 2-9 epilogue: warps 2+q and 6+q read TMEM lanes [32q, 32q+32) for
// alternate 32-token chunks), tiles of 256 M rows (two M=128 chains) by at most 128
// tokens, a 4-stage ring of 48 KB, two TMEM accumulators of 2 x 128 columns. The A
// operand of a stage (256 M rows x 64 K rows) arrives in one TMA copy through a 4-D view
// (64 M, K, M / 64, experts) of the weights, which lands as four 64-row MN-major
// swizzle-128B atoms 8 KB apart.
// Every wait is bounded; a role that gives up raises the abort flag and a status bit, the
// CTA waits (at least one second) for its copies and MMAs in flight, frees TMEM, returns.
#include "grouped_tiles.cuh"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kBK = 64;
constexpr int kFeat = 128;
constexpr int kMmaK = 16;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr int kTok = 128;
constexpr int kStages = 4;
constexpr uint32_t kABytes = 2 * kFeat * kBK * 2;  // 32 KB: 256 M rows x 64 K rows
constexpr uint32_t kXBytes = kTok * kBK * 2;       // 16 KB
constexpr uint32_t kStageBytes = kABytes + kXBytes;
constexpr uint32_t kChainCols = kTok;
constexpr uint32_t kAccCols = 2 * kChainCols;
constexpr int kBufs = 2;
constexpr uint32_t kStageRow = 33;
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffX = kOffA + kStages * kABytes;
constexpr uint32_t kOffBars = kOffX + kStages * kXBytes;
constexpr uint32_t kNumBars = 2 * kStages + 2 * kBufs + 1;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kOffTiles = kOffMisc + 16;
constexpr uint32_t kOffEpi = (kOffTiles + (kGemmMaxGroups + 1) * 4 + 15) & ~15u;
constexpr uint32_t kStgFloats = 16 * kStageRow;  // per epilogue warp: 16 token rows of 32 (+1) floats
constexpr uint32_t kSmemUsed = kOffEpi + kEpiWarps * kStgFloats * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// MN-major, 128-byte swizzle: 64-element (128 B) M atoms of 8 K rows (1024 B); atoms
// along K follow at SBO = 1024 B, atoms along M at LBO = 8 KB (64 K rows per atom column).
__device__ __forceinline__ uint64_t smem_desc_mnmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((kBK * 128) >> 4) << 16;  // leading byte offset: next 64 M rows
  d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride byte offset: next 8 K rows
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0, int32_t c1,
                                            int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_bwd_kernel(const __grid_constant__ GemmBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* sA = base + kOffA;
  uint8_t* sX = base + kOffX;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + kBufs;
  uint64_t* drain = acc_empty + kBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 8);
  int32_t* tile_start = reinterpret_cast<int32_t*>(base + kOffTiles);

  const GemmArgs& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = g.n_shared_groups + g.n_routed;

  tile_counts<kTok>(g, tile_start, G);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *never_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);  // one lane of each epilogue warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 0) tile_scan(tile_start, G, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[G];

  uint32_t issued_mask = 0, issued_parity = 0;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile<kTok>(g, tile_start, G, tile);
        const CUtensorMap* tx = t.shared ? &g.a_shared : &g.a_routed;
        const int m_atom0 = t.n_blk * (2 * kFeat / 64);  // first 64-row M atom of the tile
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, g.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          // which weight matrix, expert and K rows this K block reads
          const CUtensorMap* tw;
          int we, krow;
          if (kMode == kBwdDM) {
            tw = t.shared ? &g.b0_shared : &g.b0_routed;
            we = t.expert;
            krow = kb * kBK;
          } else {
            const int per_half = t.shared ? a.kb_half_shared : a.kb_half_routed;  // F / 64 K blocks
            const int kk = t.shared ? kb % (2 * per_half) : kb;
            we = t.shared ? t.expert + kb / (2 * per_half) : t.expert;
            const bool up = kk >= per_half;
            tw = t.shared ? (up ? &g.b1_shared : &g.b0_shared) : (up ? &g.b1_routed : &g.b0_routed);
            krow = (kk % per_half) * kBK;
          }
          tma_load_4d(sA + stage * kABytes, tw, &full[stage], 0, krow, m_atom0, we);
          tma_load_2d(sX + stage * kXBytes, tx, &full[stage], kb * kBK, t.row0);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(g.status, kStatusTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        const Tile t = decode_tile<kTok>(g, tile_start, G, tile);
        const int n_mma = (t.m_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kFeat, n_mma) | (1u << 15);  // A is MN-major
        const int acc = it % kBufs;
        if (!mbar_wait_bounded(&acc_empty[acc], ((it / kBufs) & 1) ^ 1u, g.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, g.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // chain c covers M rows 128c .. 128c+127: the atoms 2c and 2c+1, 16 KB in
          const uint32_t abase = smem_addr(sA + stage * kABytes);
          const uint64_t xd = smem_desc_kmajor_sw128(smem_addr(sX + stage * kXBytes));
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            const uint32_t accum = (kb | k) ? 1u : 0u;
            const uint32_t koff = static_cast<uint32_t>(k) * kMmaK * 128;  // 16 K rows of 128 B
            mma_bf16_ss(d0, smem_desc_mnmajor_sw128(abase + koff), xd + static_cast<uint64_t>(2 * k), idesc, accum);
            mma_bf16_ss(d0 + kChainCols, smem_desc_mnmajor_sw128(abase + 2 * kBK * 128 + koff),
                        xd + static_cast<uint64_t>(2 * k), idesc, accum);
          }
          mma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(g.status, kStatusTimeoutMma);
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    // Thread f of TMEM lane f holds M row f of both chains. Per 32 tokens the warp
    // transposes its 32 rows x 32 tokens through shared memory in two 16-token halves,
    // then lane L handles 8 consecutive M rows of token row L/4 + 8i (16-byte vectors).
    const int q = warp & 3, half = (warp - 2) >> 2;
    float* stg = reinterpret_cast<float*>(base + kOffEpi) + (warp - 2) * kStgFloats;
    const int rr = lane >> 2, cc = (lane & 3) * 8;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const Tile t = decode_tile<kTok>(g, tile_start, G, tile);
      const int acc = it % kBufs;
      if (!mbar_wait_warp_sleepy(&acc_full[acc], (it / kBufs) & 1, g.wait_limit_ns, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(g.status, kStatusTimeoutEpilogue);
        }
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      const int n_valid = t.shared ? g.n_valid_shared : g.n_valid_routed;
#pragma unroll 1
      for (int c0 = 32 * half; c0 < t.m_valid; c0 += 64) {
        uint32_t v0[32], v1[32];
        tmem_ld16(tb + c0, *reinterpret_cast<uint32_t(*)[16]>(&v0[0]));
        tmem_ld16(tb + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v0[16]));
        tmem_ld16(tb + kChainCols + c0, *reinterpret_cast<uint32_t(*)[16]>(&v1[0]));
        tmem_ld16(tb + kChainCols + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v1[16]));
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int f = t.n_blk * 2 * kFeat + ch * kFeat + q * 32 + cc;  // first of this lane's 8 M rows
          const bool ok_f = f < n_valid;  // n_valid is a multiple of 64, f of 8
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              stg[j * kStageRow + lane] = __uint_as_float(ch == 0 ? v0[16 * hh + j] : v1[16 * hh + j]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int row = rr + 8 * i, tok = c0 + 16 * hh + row;
              if (!ok_f || tok >= t.m_valid) continue;
              const float* src = stg + row * kStageRow + cc;
              const int64_t r = t.row0 + tok;
              if (kMode == kBwdDM) {
                // saved pre-activations a | b of this row, and the da | db outputs, side by side
                const int64_t ld = t.shared ? a.ld_ab_shared : a.ld_ab_routed;
                const int64_t col = t.shared ? static_cast<int64_t>(t.group) * 2 * a.width_shared + f : f;
                const int64_t wh = t.shared ? a.width_shared : a.width_routed;
                const bf16* ab = t.shared ? a.ab_shared : a.ab_routed;
                bf16* dab = t.shared ? a.dab_shared : a.dab_routed;
                const uint4 av = *reinterpret_cast<const uint4*>(ab + r * ld + col);
                const uint4 bv = *reinterpret_cast<const uint4*>(ab + r * ld + col + wh);
                const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
                uint32_t da[4], db[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 x = unpack_bf16x2(aw[k]), y = unpack_bf16x2(bw[k]);
                  const float s0 = __fdividef(1.0f, 1.0f + __expf(-x.x)), s1 = __fdividef(1.0f, 1.0f + __expf(-x.y));
                  const float dm0 = src[2 * k], dm1 = src[2 * k + 1];
                  da[k] = pack_bf16x2(dm0 * y.x * s0 * (1.0f + x.x * (1.0f - s0)),
                                      dm1 * y.y * s1 * (1.0f + x.y * (1.0f - s1)));
                  db[k] = pack_bf16x2(dm0 * x.x * s0, dm1 * x.y * s1);
                }
                *reinterpret_cast<uint4*>(dab + r * ld + col) = make_uint4(da[0], da[1], da[2], da[3]);
                *reinterpret_cast<uint4*>(dab + r * ld + col + wh) = make_uint4(db[0], db[1], db[2], db[3]);
              } else if (t.shared) {  // fp32 sum over the shared experts, one row per token
                float4* dst = reinterpret_cast<float4*>(a.dx_shared + r * a.ld_dx + f);
                dst[0] = make_float4(src[0], src[1], src[2], src[3]);
                dst[1] = make_float4(src[4], src[5], src[6], src[7]);
              } else {
                *reinterpret_cast<uint4*>(a.dx_routed + r * a.ld_dx + f) =
                    make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                               pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
              }
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < kStages; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, drain_wait_limit(g.wait_limit_ns), never_flag))
            atomicOr(g.status, kStatusTimeoutDrain);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      if (!mbar_wait_bounded(drain, 0, drain_wait_limit(g.wait_limit_ns), never_flag))
        atomicOr(g.status, kStatusTimeoutDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}
}  // namespace

cudaError_t launch_grouped_gemm_bwd(int mode, const GemmBwdArgs& a, int grid, cudaStream_t s) {
  if (a.g.n_shared_groups + a.g.n_routed > kGemmMaxGroups) return cudaErrorInvalidValue;
  if (grid < 1) grid = 1;
  cudaError_t e;
  if (mode == kBwdDM) {
    e = cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kBwdDM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    grouped_gemm_bwd_kernel<kBwdDM><<<grid, kThreads, kSmemBytes, s>>>(a);
  } else if (mode == kBwdDX) {
    e = cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kBwdDX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    grouped_gemm_bwd_kernel<kBwdDX><<<grid, kThreads, kSmemBytes, s>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace dsmoe
