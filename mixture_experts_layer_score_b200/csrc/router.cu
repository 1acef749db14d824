// router.cu -- router affinity, scoring, top-K' selection and gates.
//
// Affinity l[t,i] = u_t . e_i ("MoE architecture: how DeepSeek achieves more",
// section 2: G(x) = Softmax(W_g x)); scores softmax / sigmoid / sqrt(softplus)
// (DeepSeek-V4 book ch. 2, section 2); selection key s + b with the bias deciding
// selection only (same chapter, section 3); gates g = s or s / sum_selected s;
// hash routing expert = token_id * mult mod N (same chapter, section 5).
#include <float.h>
#include <math.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

// --------------------------------------------------------------------------------------
// router logits on CUDA cores: a 64 tokens x 64 experts tile per CTA, 4x4 per thread,
// fp32 FMA accumulation in ascending k.
// --------------------------------------------------------------------------------------
namespace {
constexpr int kRTM = 64, kRTN = 64, kRTK = 32;

// blockIdx.z selects a slice [z*kc, (z+1)*kc) of the reduction dimension; slice z
// writes its partial sums to logits + z*T*N. The select kernel adds the slices in order.
__global__ void __launch_bounds__(256) router_logits_kernel(const bf16* __restrict__ x,
                                                            const bf16* __restrict__ W, int T, int N, int d,
                                                            int kc, float* __restrict__ logits) {
  __shared__ __align__(16) float xs[kRTK][kRTM + 4];
  __shared__ __align__(16) float ws[kRTK][kRTN + 4];
  const int t0 = blockIdx.x * kRTM, n0 = blockIdx.y * kRTN;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 2, lc = (tid & 3) * 8;  // loader: row, first column of 8
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  const int k_begin = blockIdx.z * kc, k_end = min(d, k_begin + kc);
  logits += static_cast<int64_t>(blockIdx.z) * T * N;
  for (int k0 = k_begin; k0 < k_end; k0 += kRTK) {
    uint4 vx = make_uint4(0, 0, 0, 0), vw = make_uint4(0, 0, 0, 0);
    if (t0 + lr < T) vx = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t0 + lr) * d + k0 + lc);
    if (n0 + lr < N) vw = *reinterpret_cast<const uint4*>(W + static_cast<int64_t>(n0 + lr) * d + k0 + lc);
    const uint32_t ux[4] = {vx.x, vx.y, vx.z, vx.w}, uw[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fx = unpack_bf16x2(ux[j]), fw = unpack_bf16x2(uw[j]);
      xs[lc + 2 * j][lr] = fx.x;
      xs[lc + 2 * j + 1][lr] = fx.y;
      ws[lc + 2 * j][lr] = fw.x;
      ws[lc + 2 * j + 1][lr] = fw.y;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRTK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 w = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) logits[static_cast<int64_t>(t) * N + n] = acc[i][j];
    }
  }
}
}  // namespace

int router_logits_splits(int T, int N, int d, int num_sms) {
  const int tiles = ((T + kRTM - 1) / kRTM) * ((N + kRTN - 1) / kRTN);
  int splits = (2 * num_sms + tiles - 1) / tiles;  // about two CTAs per SM
  const int steps = d / kRTK;
  if (splits > steps) splits = steps;
  if (splits > kRouterMaxSplits) splits = kRouterMaxSplits;
  if (splits < 1) splits = 1;
  // the launch covers d with slices of ceil(steps/splits) k-steps: only that many slices
  // are non-empty, and the select kernel adds exactly the slices written
  const int per = (steps + splits - 1) / splits;
  return (steps + per - 1) / per;
}

cudaError_t launch_router_logits(const bf16* x, const bf16* W_router, int T, int N, int d, int splits,
                                 float* logits, cudaStream_t s) {
  // slice length: a multiple of the 32-wide k step covering d in `splits` slices (a
  // count from router_logits_splits, so that every slice is non-empty)
  const int kc = ((d / kRTK + splits - 1) / splits) * kRTK;
  if ((d + kc - 1) / kc != splits) return cudaErrorInvalidValue;
  dim3 grid((T + kRTM - 1) / kRTM, (N + kRTN - 1) / kRTN, splits);
  router_logits_kernel<<<grid, 256, 0, s>>>(x, W_router, T, N, d, kc, logits);
  return cudaGetLastError();
}

// --------------------------------------------------------------------------------------
// scores + top-K' + gates + statistics partials: one warp per token, lane j owns experts
// j, j+32, ... (kNPL per lane). Selection is rounds of a warp arg-max over the keys not
// yet taken; ties go to the lower expert index. The first mask_top rounds only mask
// their winner (the DeepSeekMoE summary's "disable the top routed experts" analysis);
// the next K' rounds select.
// --------------------------------------------------------------------------------------
namespace {
constexpr int kSelWarps = 8;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float score_sigmoid(float l) { return 1.f / (1.f + expf(-l)); }
// sqrt(log(1 + e^l)) through log(1+e^l) = max(l,0) + log1p(e^{-|l|}).
__device__ __forceinline__ float score_sqrt_softplus(float l) {
  return sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
}

template <int kNPL>
__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(const SelectArgs a) {
  // 4 KB at kNPL = 8, so that a block fits on an SM beside a grouped-GEMM CTA (the shared
  // experts' GEMMs run concurrently with this kernel)
  __shared__ float red[kSelWarps / 2][kNPL * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N, K = a.K;
  float pacc[kNPL];
  float bias[kNPL];
#pragma unroll
  for (int j = 0; j < kNPL; ++j) {
    pacc[j] = 0.f;
    const int i = lane + 32 * j;
    bias[j] = (a.bias_select && i < N) ? a.b[i] : 0.f;
  }
  const int gw = blockIdx.x * kSelWarps + warp, nw = gridDim.x * kSelWarps;
  for (int t = gw; t < a.T; t += nw) {
    const float* lrow = a.logits + static_cast<int64_t>(t) * N;
    const int64_t slice = static_cast<int64_t>(a.T) * N;
    float s[kNPL];
#pragma unroll
    for (int j = 0; j < kNPL; ++j) {
      const int i = lane + 32 * j;
      float v = -INFINITY;
      if (i < N) {
        v = lrow[i];
        for (int z = 1; z < a.splits; ++z) v += lrow[z * slice + i];
        if (a.bias_in_logits) v += a.b[i];
      }
      s[j] = v;
    }
    if (a.score == 0) {  // softmax over the routed experts
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < kNPL; ++j) m = fmaxf(m, s[j]);
      m = warp_max(m);
      float z = 0.f;
#pragma unroll
      for (int j = 0; j < kNPL; ++j) {
        s[j] = (lane + 32 * j < N) ? expf(s[j] - m) : 0.f;
        z += s[j];
      }
      z = warp_sum(z);
      const float inv = 1.f / z;
#pragma unroll
      for (int j = 0; j < kNPL; ++j) s[j] *= inv;
    } else if (a.score == 1) {
#pragma unroll
      for (int j = 0; j < kNPL; ++j) s[j] = (lane + 32 * j < N) ? score_sigmoid(s[j]) : 0.f;
    } else {
#pragma unroll
      for (int j = 0; j < kNPL; ++j) s[j] = (lane + 32 * j < N) ? score_sqrt_softplus(s[j]) : 0.f;
    }
    // selection keys; NaN keys rank last
    float key[kNPL];
#pragma unroll
    for (int j = 0; j < kNPL; ++j) {
      const float kv = s[j] + bias[j];
      key[j] = (lane + 32 * j < N && !isnan(kv)) ? kv : -INFINITY;
    }
    uint32_t taken = 0;
    int my_idx = 0;
    float my_s = 0.f;
    const int rounds = a.mask_top + K;
    for (int r = 0; r < rounds; ++r) {
      float bk = -INFINITY;
      int bi = 0x7fffffff;
      float bs = 0.f;
#pragma unroll
      for (int j = 0; j < kNPL; ++j) {
        const int i = lane + 32 * j;
        const bool cand = (i < N) && !((taken >> j) & 1u);
        if (cand && (key[j] > bk || (key[j] == bk && i < bi))) {
          bk = key[j];
          bi = i;
          bs = s[j];
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        if (ok > bk || (ok == bk && oi < bi)) {
          bk = ok;
          bi = oi;
          bs = os;
        }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == r - a.mask_top) {
        my_idx = bi;
        my_s = bs;
      }
    }
    float g = my_s;
    if (a.renormalize) {
      const float z = warp_sum(lane < K ? my_s : 0.f);
      g = my_s / fmaxf(z, FLT_MIN);
    }
    if (lane < K) {
      if (my_idx < 0 || my_idx >= N) {  // cannot happen for K <= N; recorded, never dereferenced
        atomicOr(a.status, kStatusBadIndex);
        my_idx = 0;
      }
      a.topk_idx[static_cast<int64_t>(t) * K + lane] = my_idx;
      a.gates[static_cast<int64_t>(t) * K + lane] = g;
      atomicAdd(&a.counts[my_idx], 1);
    }
#pragma unroll
    for (int j = 0; j < kNPL; ++j) pacc[j] += s[j];
    if (a.scores_dbg) {
      float* srow = a.scores_dbg + static_cast<int64_t>(t) * N;
#pragma unroll
      for (int j = 0; j < kNPL; ++j)
        if (lane + 32 * j < N) srow[lane + 32 * j] = s[j];
    }
  }
  // per-block partial sums of the scores, reduced over warps in a fixed order: warp w + 4
  // into row w, warp w adds its own, then the 4 rows in order
  constexpr int kHalf = kSelWarps / 2;
  if (warp >= kHalf) {
#pragma unroll
    for (int j = 0; j < kNPL; ++j) red[warp - kHalf][lane + 32 * j] = pacc[j];
  }
  __syncthreads();
  if (warp < kHalf) {
#pragma unroll
    for (int j = 0; j < kNPL; ++j) red[warp][lane + 32 * j] += pacc[j];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kHalf; ++w) v += red[w][i];
    a.P_part[static_cast<int64_t>(blockIdx.x) * N + i] = v;
  }
}
}  // namespace

int select_grid(int T, int num_sms) {
  int g = (T + kSelWarps - 1) / kSelWarps;
  const int cap = 4 * num_sms;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return g;
}

cudaError_t launch_select(const SelectArgs& a, int grid, cudaStream_t s) {
  const int npl = (a.N + 31) / 32;
  const dim3 blk(kSelWarps * 32);
  if (npl <= 1) select_kernel<1><<<grid, blk, 0, s>>>(a);
  else if (npl <= 2) select_kernel<2><<<grid, blk, 0, s>>>(a);
  else if (npl <= 4) select_kernel<4><<<grid, blk, 0, s>>>(a);
  else if (npl <= 8) select_kernel<8><<<grid, blk, 0, s>>>(a);
  else if (npl <= 12) select_kernel<12><<<grid, blk, 0, s>>>(a);
  else select_kernel<16><<<grid, blk, 0, s>>>(a);
  return cudaGetLastError();
}

// --------------------------------------------------------------------------------------
// hash routing: one expert per token, gate 1. The product is taken in 64 bits (no wrap).
// --------------------------------------------------------------------------------------
namespace {
__global__ void hash_route_kernel(const int32_t* __restrict__ ids, int T, int N, uint32_t mult, uint32_t mod,
                                  int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                                  int32_t* __restrict__ counts, uint32_t* status) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    const int32_t id = ids[t];
    int e = 0;
    if (id < 0) {
      atomicOr(status, kStatusBadIndex);
    } else {
      e = static_cast<int>((static_cast<uint64_t>(id) * mult) % mod);
    }
    if (e >= N) e = 0;
    topk_idx[t] = e;
    gates[t] = 1.f;
    atomicAdd(&counts[e], 1);
  }
}
}  // namespace

cudaError_t launch_hash_route(const int32_t* token_ids, int T, int N, uint32_t mult, uint32_t mod,
                              int32_t* topk_idx, float* gates, int32_t* counts, uint32_t* status,
                              cudaStream_t s) {
  const int blk = 256;
  int grid = (T + blk - 1) / blk;
  if (grid < 1) grid = 1;
  hash_route_kernel<<<grid, blk, 0, s>>>(token_ids, T, N, mult, mod, topk_idx, gates, counts, status);
  return cudaGetLastError();
}

}  // namespace dsmoe
