// gemm_sm100.cu -- persistent grouped GEMM for the expert FFNs on the 5th-generation
// tensor cores (tcgen05 + TMEM), operands staged by TMA.
//
// Each expert FFN of the DeepSeekMoE layer (DeepSeekMoE summary, shared-expert layer
// equation; SwiGLU form noted on the "MoE: sparse activation" page) is two dense
// contractions over the rows routed to that expert:
//   gate/up:  A1[r, n] = SiLU(sum_k X[r,k] W_gate[e,n,k]) * (sum_k X[r,k] W_up[e,n,k])
//   down:     Y[r, n]  = sum_k A1[r,k] W_down[e,n,k]
// The routed experts are groups of a variable number of rows (their segment of the
// expert-contiguous slot order, read from the device-side offsets), the shared
// experts are dense groups over all T tokens that run first.
//
// One CTA per SM, 192 threads in three roles:
//   warp 0     TMA producer: streams 128x64 A tiles and 256x64 B tiles through a
//              4-stage shared-memory ring (mbarrier full/empty pairs).
//   warp 1     allocates 512 TMEM columns (two 128x256 fp32 accumulators) and issues
//              tcgen05.mma (M=128, N=256, K=16) from one thread; commits free ring
//              stages and publish finished accumulators.
//   warps 2-5  epilogue: tcgen05.ld of the accumulator rows, SiLU(gate)*up (gate/up
//              GEMM) or a plain conversion (down GEMM), bf16 stores; the second TMEM
//              accumulator lets the next tile's MMAs overlap this epilogue.
// For the gate/up GEMM the 256-row B tile is [128 gate rows | 128 up rows] of the same
// output features, so one MMA chain yields both halves side by side in TMEM.
//
// Every wait is bounded (wait_limit_ns); a role that gives up raises a CTA-wide abort
// flag and a bit of the device status word, the CTA lets in-flight TMA loads and MMAs
// finish (again bounded), frees its TMEM and returns.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kBM = 128;        // output rows per tile (= TMEM lanes)
constexpr int kBK = 64;         // K per ring stage (one 128-byte swizzled row of bf16)
constexpr int kMmaN = 256;      // N of each tcgen05.mma
constexpr int kMmaK = 16;       // K of each bf16 tcgen05.mma
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 8 + 512;
constexpr uint32_t kABytes = kBM * kBK * 2;    // 16 KB
constexpr uint32_t kBBytes = kMmaN * kBK * 2;  // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffBars = kOffB + kStages * kBBytes;
constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kOffTiles = kOffMisc + 16;
constexpr uint32_t kSmemUsed = kOffTiles + (kMaxGroups + 1) * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack to align the ring to 1024 bytes
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Tile {
  int shared;   // 1: shared-expert group
  int group;    // group index (shared groups first)
  int expert;   // expert index inside its kind
  int row0;     // first A / output row of the tile
  int m_valid;  // valid rows in the tile
  int n_blk;    // output tile index along N
  int kb_n;     // K blocks
};

__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, const int32_t* tile_start, int G, int tile) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // last group whose first tile is <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  Tile t;
  t.group = lo;
  int M, base;
  if (lo < a.n_shared_groups) {
    t.shared = 1;
    t.expert = lo;
    M = a.m_shared;
    base = 0;
    t.kb_n = a.kb_shared;
  } else {
    t.shared = 0;
    t.expert = lo - a.n_shared_groups;
    base = a.offsets[t.expert];
    M = a.offsets[t.expert + 1] - base;
    t.kb_n = a.kb_routed;
  }
  const int mt = (M + kBM - 1) / kBM;
  const int local = tile - tile_start[lo];
  const int m_blk = local % mt;
  t.n_blk = local / mt;
  t.row0 = base + m_blk * kBM;
  t.m_valid = min(kBM, M - m_blk * kBM);
  return t;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* sA = base + kOffA;
  uint8_t* sB = base + kOffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 8);
  int32_t* tile_start = reinterpret_cast<int32_t*>(base + kOffTiles);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.n_shared_groups + a.n_routed;

  // tiles of each group, then an inclusive prefix -> first tile of each group
  for (int g = threadIdx.x; g < G; g += kThreads) {
    int M, nt;
    if (g < a.n_shared_groups) {
      M = a.m_shared;
      nt = a.n_tiles_shared;
    } else {
      const int e = g - a.n_shared_groups;
      M = a.offsets[e + 1] - a.offsets[e];
      nt = a.n_tiles_routed;
    }
    M = max(M, 0);
    tile_start[g + 1] = ((M + kBM - 1) / kBM) * nt;
  }
  if (threadIdx.x == 0) {
    tile_start[0] = 0;
    *abort_flag = 0;
    *never_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int b0 = 1; b0 <= G; b0 += 32) {
      const int i = b0 + lane;
      int v = (i <= G) ? tile_start[i] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (i <= G) tile_start[i] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[G];

  uint32_t issued_mask = 0, issued_parity = 0;  // producer bookkeeping for the abort drain

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&a.a_routed);
      tma_prefetch_desc(&a.b0_routed);
      if (kSwiGLU) tma_prefetch_desc(&a.b1_routed);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile(a, tile_start, G, tile);
        const CUtensorMap* ta = t.shared ? &a.a_shared : &a.a_routed;
        const CUtensorMap* tb0 = t.shared ? &a.b0_shared : &a.b0_routed;
        const CUtensorMap* tb1 = t.shared ? &a.b1_shared : &a.b1_routed;
        const int kb_per = t.shared ? a.kb_per_b_expert_shared : t.kb_n;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(sA + stage * kABytes, ta, &full[stage], kb * kBK, t.row0);
          const int be = t.expert + kb / kb_per;
          const int bk = (kb % kb_per) * kBK;
          if (kSwiGLU) {
            tma_load_3d(sB + stage * kBBytes, tb0, &full[stage], bk, t.n_blk * (kMmaN / 2), be);
            tma_load_3d(sB + stage * kBBytes + kBBytes / 2, tb1, &full[stage], bk, t.n_blk * (kMmaN / 2), be);
          } else {
            tma_load_3d(sB + stage * kBBytes, tb0, &full[stage], bk, t.n_blk * kMmaN, be);
          }
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
        atomicOr(a.status, kStatusTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kBM, kMmaN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        const Tile t = decode_tile(a, tile_start, G, tile);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait_bounded(&acc_empty[acc], acc_phase ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_kmajor_sw128(smem_addr(sA + stage * kABytes));
          const uint64_t bd = smem_desc_kmajor_sw128(smem_addr(sB + stage * kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k)
            mma_bf16_ss(d_tmem, ad + static_cast<uint64_t>(2 * k), bd + static_cast<uint64_t>(2 * k), idesc,
                        (kb | k) ? 1u : 0u);
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
        atomicOr(a.status, kStatusTimeoutMma);
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    const int q = warp & 3;  // this warp may read TMEM lanes [32q, 32q+32)
    const int r = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const Tile t = decode_tile(a, tile_start, G, tile);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const bool w = mbar_wait_bounded(&acc_full[acc], acc_phase, a.wait_limit_ns, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(a.status, kStatusTimeoutEpilogue);
        }
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      const bool row_ok = r < t.m_valid;
      bf16* out;
      int n_valid;
      if (t.shared) {
        out = a.out_shared + static_cast<int64_t>(t.row0 + r) * a.ld_shared +
              static_cast<int64_t>(t.group) * a.shared_col_stride;
        n_valid = a.n_valid_shared;
      } else {
        out = a.out_routed + static_cast<int64_t>(t.row0 + r) * a.ld_routed;
        n_valid = a.n_valid_routed;
      }
      if (kSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < kMmaN / 2; c += 16) {
          uint32_t gv[16], uv[16];
          tmem_ld16(tb + c, gv);
          tmem_ld16(tb + kMmaN / 2 + c, uv);
          tmem_wait_ld();
          const int col = t.n_blk * (kMmaN / 2) + c;
          if (row_ok && col < n_valid) {
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float g0 = __uint_as_float(gv[2 * j]), g1 = __uint_as_float(gv[2 * j + 1]);
              const float u0 = __uint_as_float(uv[2 * j]), u1 = __uint_as_float(uv[2 * j + 1]);
              pk[j] = pack_bf16x2(silu(g0) * u0, silu(g1) * u1);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else if (t.shared && a.out_shared_f32) {
        // shared experts of the down GEMM: fp32 row of (residual + sum of shared outputs)
        float* o32 = a.out_shared_f32 + static_cast<int64_t>(t.row0 + r) * a.ld_shared;
        const bf16* res = a.residual + static_cast<int64_t>(t.row0 + r) * a.ld_shared;
#pragma unroll 1
        for (int c = 0; c < kMmaN; c += 16) {
          uint32_t v[16];
          tmem_ld16(tb + c, v);
          tmem_wait_ld();
          const int col = t.n_blk * kMmaN + c;
          if (row_ok && col < n_valid) {
            const uint4* r4 = reinterpret_cast<const uint4*>(res + col);
            const uint4 q0 = r4[0], q1 = r4[1];
            const uint32_t rw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            float4* dst = reinterpret_cast<float4*>(o32 + col);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 a0 = unpack_bf16x2(rw[2 * j]), a1 = unpack_bf16x2(rw[2 * j + 1]);
              dst[j] = make_float4(__uint_as_float(v[4 * j]) + a0.x, __uint_as_float(v[4 * j + 1]) + a0.y,
                                   __uint_as_float(v[4 * j + 2]) + a1.x, __uint_as_float(v[4 * j + 3]) + a1.y);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kMmaN; c += 16) {
          uint32_t v[16];
          tmem_ld16(tb + c, v);
          tmem_wait_ld();
          const int col = t.n_blk * kMmaN + c;
          if (row_ok && col < n_valid) {
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // let every copy and MMA this CTA started finish before its memory is released
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < kStages; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, a.wait_limit_ns, never_flag))
            atomicOr(a.status, kStatusTimeoutDrain);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      if (!mbar_wait_bounded(drain, 0, a.wait_limit_ns, never_flag)) atomicOr(a.status, kStatusTimeoutDrain);
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

cudaError_t launch_grouped_gemm(bool swiglu, const GemmArgs& a, int grid, cudaStream_t s) {
  if (a.n_shared_groups + a.n_routed > kMaxGroups) return cudaErrorInvalidValue;
  if (grid < 1) grid = 1;
  cudaError_t e;
  if (swiglu) {
    e = cudaFuncSetAttribute(grouped_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(grouped_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dsmoe
