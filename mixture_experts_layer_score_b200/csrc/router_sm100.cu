// router_sm100.cu -- router affinities on the 5th-generation tensor cores, with the
// scoring, top-K' selection, gates and balance-statistics partials fused into the
// epilogue that reads the accumulator out of TMEM.
//
// Affinity l[t,i] = u_t . e_i ("MoE architecture: how DeepSeek achieves more",
// section 2); scores softmax / sigmoid / sqrt(softplus) (DeepSeek-V4 book ch. 2,
// section 2); selection key s + b with a selection-only bias (same chapter, section 3;
// "MoE: sparse activation", load-balancing section); top-K' ordered by key, ties to
// the lower index; gates g = s or s / sum_selected s; per-CTA partial sums of s for
// P_i (DeepSeekMoE summary, "Expert-level balance loss").
//
// A CTA owns 128 tokens at a time (persistent over token tiles). The affinities of
// the 128 tokens with all N' experts accumulate in TMEM (fp32), N' columns wide, as
// one or two chains of tcgen05.mma (M=128, N<=256, K=16) fed by a TMA ring of
// x tiles (128x64) and router tiles (N'x64). The epilogue thread of TMEM lane r owns
// token r: it streams its row of N' logits out of TMEM in 32-column groups, scores
// them, keeps its K' best in a sorted register list, and the warp sums every column
// of scores over its 32 tokens with a 31-shuffle transposed reduction.
#include <float.h>
#include <math.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMmaK = 16;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kMaxCols = 512;
constexpr int kKMax = 16;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr size_t kSmemLimit = 232448;

struct Layout {
  uint32_t b_bytes, stage_bytes, stages;
  uint32_t off_b, off_bars, off_misc, off_red, off_bias, used;
};

__host__ __device__ inline Layout router_layout(int n_chunks, int nc) {
  Layout L;
  L.b_bytes = static_cast<uint32_t>(n_chunks) * nc * kBK * 2;
  L.stage_bytes = kABytes + L.b_bytes;
  const uint32_t fixed = 1024 + 256 + 4 * kMaxCols * 4 + kMaxCols * 4;
  uint32_t st = static_cast<uint32_t>((kSmemLimit - fixed) / L.stage_bytes);
  L.stages = st > 4 ? 4 : st;
  L.off_b = L.stages * kABytes;
  L.off_bars = L.off_b + L.stages * L.b_bytes;
  L.off_misc = L.off_bars + (2 * 4 + 3) * 8;
  L.off_red = (L.off_misc + 16 + 15) & ~15u;
  L.off_bias = L.off_red + 4 * kMaxCols * 4;
  L.used = L.off_bias + kMaxCols * 4;
  return L;
}

__device__ __forceinline__ float score_of(int score, float l, float m, float inv_z) {
  if (score == 0) return expf(l - m) * inv_z;
  if (score == 1) return 1.f / (1.f + expf(-l));
  return sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
}

// 32 lanes each hold v[0..31] (one value per column); afterwards lane l holds in v[0]
// the sum over the 32 lanes of column l (recursive halving, 31 shuffles).
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kThreads, 1) router_tc_kernel(const __grid_constant__ RouterTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  const Layout L = router_layout(a.n_chunks, a.nc);
  const int stages = static_cast<int>(L.stages);
  uint8_t* sA = base;
  uint8_t* sB = base + L.off_b;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.off_bars);
  uint64_t* empty = full + 4;
  uint64_t* acc_full = empty + 4;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.off_misc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + L.off_misc + 8);
  float* red = reinterpret_cast<float*>(base + L.off_red);   // [4][kMaxCols] per-quarter column sums
  float* sbias = reinterpret_cast<float*>(base + L.off_bias);  // [kMaxCols]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N, K = a.K;
  const int n_tiles = (a.T + kBM - 1) / kBM;
  const int kb_n = a.d / kBK;

  for (int i = threadIdx.x; i < kMaxCols; i += kThreads) {
    sbias[i] = ((a.bias_select || a.bias_in_logits) && i < N) ? a.b[i] : 0.f;
    for (int q = 0; q < 4; ++q) red[q * kMaxCols + i] = 0.f;
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *never_flag = 0;
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiThreads);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  uint32_t issued_mask = 0, issued_parity = 0;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&a.tm_x);
      tma_prefetch_desc(&a.tm_w);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L.stage_bytes);
          tma_load_2d(sA + stage * kABytes, &a.tm_x, &full[stage], kb * kBK, tile * kBM);
          for (int c = 0; c < a.n_chunks; ++c)
            tma_load_2d(sB + stage * L.b_bytes + c * a.nc * kBK * 2, &a.tm_w, &full[stage], kb * kBK, c * a.nc);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == stages) {
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
      // -------------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kBM, a.nc);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
        if (!mbar_wait_bounded(acc_empty, (it & 1) ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_kmajor_sw128(smem_addr(sA + stage * kABytes));
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k)
            for (int c = 0; c < a.n_chunks; ++c) {
              const uint64_t bd = smem_desc_kmajor_sw128(smem_addr(sB + stage * L.b_bytes + c * a.nc * kBK * 2));
              mma_bf16_ss(tmem_base + c * a.nc, ad + static_cast<uint64_t>(2 * k), bd + static_cast<uint64_t>(2 * k),
                          idesc, (kb | k) ? 1u : 0u);
            }
          mma_commit(&empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(acc_full);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeoutMma);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int ngroups = (N + 31) / 32;
    // per-expert bias added to the logits (DSMOE_BIAS_IN_LOGITS), else 0
    auto lb = [&](int n) -> float { return a.bias_in_logits ? sbias[min(n, kMaxCols - 1)] : 0.f; };
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const bool w = mbar_wait_bounded(acc_full, it & 1, a.wait_limit_ns, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(a.status, kStatusTimeoutEpilogue);
        }
        break;
      }
      tc_fence_after();
      const int t = tile * kBM + r;
      const bool valid = t < a.T;
      float m = 0.f, inv_z = 1.f;
      if (a.score == 0) {  // softmax: the row maximum, then the normaliser
        m = -INFINITY;
        for (int g = 0; g < ngroups; ++g) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tb + g * 32, v0);
          tmem_ld16(tb + g * 32 + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (g * 32 + j < N) m = fmaxf(m, __uint_as_float(v0[j]) + lb(g * 32 + j));
            if (g * 32 + 16 + j < N) m = fmaxf(m, __uint_as_float(v1[j]) + lb(g * 32 + 16 + j));
          }
        }
        float z = 0.f;
        for (int g = 0; g < ngroups; ++g) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tb + g * 32, v0);
          tmem_ld16(tb + g * 32 + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (g * 32 + j < N) z += expf(__uint_as_float(v0[j]) + lb(g * 32 + j) - m);
            if (g * 32 + 16 + j < N) z += expf(__uint_as_float(v1[j]) + lb(g * 32 + 16 + j) - m);
          }
        }
        inv_z = 1.f / z;
      }
      float tk_key[kKMax], tk_s[kKMax];
      int tk_idx[kKMax];
#pragma unroll
      for (int j = 0; j < kKMax; ++j) {
        tk_key[j] = -INFINITY;
        tk_s[j] = 0.f;
        tk_idx[j] = 0;
      }
      float kth = -INFINITY;  // key of the K'-th entry
      for (int g = 0; g < ngroups; ++g) {
        float s[32];
        {
          uint32_t v0[16], v1[16];
          tmem_ld16(tb + g * 32, v0);
          tmem_ld16(tb + g * 32 + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            s[j] = __uint_as_float(v0[j]);
            s[16 + j] = __uint_as_float(v1[j]);
          }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int n = g * 32 + j;
          s[j] = (n < N) ? score_of(a.score, s[j] + lb(n), m, inv_z) : 0.f;
        }
        if (valid) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = g * 32 + j;
            float key = s[j] + (a.bias_select ? sbias[min(n, kMaxCols - 1)] : 0.f);
            if (isnan(key)) key = -INFINITY;
            if (n < N && key > kth) {  // sorted insert (descending key, earlier index first on ties)
              const float ns = s[j];
#pragma unroll
              for (int p = kKMax - 1; p >= 1; --p) {
                if (key > tk_key[p - 1]) {
                  tk_key[p] = tk_key[p - 1];
                  tk_s[p] = tk_s[p - 1];
                  tk_idx[p] = tk_idx[p - 1];
                } else if (key > tk_key[p]) {
                  tk_key[p] = key;
                  tk_s[p] = ns;
                  tk_idx[p] = n;
                }
              }
              if (key > tk_key[0]) {
                tk_key[0] = key;
                tk_s[0] = ns;
                tk_idx[0] = n;
              }
#pragma unroll
              for (int p = 0; p < kKMax; ++p)
                if (p == K - 1) kth = tk_key[p];
            }
          }
          if (a.scores_dbg) {
            float4* dst = reinterpret_cast<float4*>(a.scores_dbg + static_cast<int64_t>(t) * N + g * 32);
            if ((N & 3) == 0 && g * 32 + 32 <= N) {
#pragma unroll
              for (int j = 0; j < 8; ++j) dst[j] = make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
            } else {
              for (int j = 0; j < 32 && g * 32 + j < N; ++j) a.scores_dbg[static_cast<int64_t>(t) * N + g * 32 + j] = s[j];
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j] = 0.f;
        }
        const float colsum = transpose_reduce32(s, lane);
        if (g * 32 + lane < N) red[q * kMaxCols + g * 32 + lane] += colsum;
      }
      tc_fence_before();
      mbar_arrive(acc_empty);  // the accumulator may be overwritten by the next tile
      if (valid) {
        float zsel = 0.f;
#pragma unroll
        for (int p = 0; p < kKMax; ++p)
          if (p < K) zsel += tk_s[p];
        const float inv_sel = 1.f / fmaxf(zsel, FLT_MIN);
#pragma unroll
        for (int p = 0; p < kKMax; ++p) {
          if (p < K) {
            a.topk_idx[static_cast<int64_t>(t) * K + p] = tk_idx[p];
            a.gates[static_cast<int64_t>(t) * K + p] = a.renormalize ? tk_s[p] * inv_sel : tk_s[p];
            atomicAdd(&a.counts[tk_idx[p]], 1);
          }
        }
      }
    }
  }

  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < stages; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, a.wait_limit_ns, never_flag))
            atomicOr(a.status, kStatusTimeoutDrain);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      if (!mbar_wait_bounded(drain, 0, a.wait_limit_ns, never_flag)) atomicOr(a.status, kStatusTimeoutDrain);
    }
  }
  // this CTA's partial score sums: the four quarters added in a fixed order
  for (int i = threadIdx.x; i < N; i += kThreads)
    a.P_part[static_cast<int64_t>(blockIdx.x) * N + i] =
        ((red[i] + red[kMaxCols + i]) + red[2 * kMaxCols + i]) + red[3 * kMaxCols + i];
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
}
}  // namespace

void router_tc_shape(int N, int* n_chunks, int* nc, uint32_t* tmem_cols) {
  const int chunks = (N + 255) / 256;
  const int per = (N + chunks - 1) / chunks;
  const int c = (per + 15) / 16 * 16;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(chunks * c)) cols <<= 1;
  *n_chunks = chunks;
  *nc = c;
  *tmem_cols = cols;
}

size_t router_tc_smem_bytes(int n_chunks, int nc) { return router_layout(n_chunks, nc).used + 1024; }

cudaError_t launch_router_tc(const RouterTcArgs& a, int grid, cudaStream_t s) {
  const size_t smem = router_tc_smem_bytes(a.n_chunks, a.nc);
  if (smem > kSmemLimit || router_layout(a.n_chunks, a.nc).stages < 2) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  router_tc_kernel<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dsmoe
