// backward.cu -- the first steps of the layer's backward pass: the gate gradients and the
// expert output gradients in slot order, and the router's backward with the expert-level
// balance term.
//
// For an upstream gradient dh = dL/dh of the layer output (DeepSeekMoE summary,
// shared-expert layer equation h_t = u_t + sum_shared FFN(u_t) + sum_k g_{t,k} y_{t,k}):
//   dg_{t,k} = <dh_t, y_{t,k}>                      (y = the forward's expert output row)
//   dY[slot(t,k)] = g_{t,k} dh_t                     (the routed experts' output gradient)
// The scores reach the loss through the gates and through P_i = (1/T) sum_t s_{t,i}
// in alpha * sum_i f_i P_i (same page, "Expert-level balance loss": f_i is built from the
// top-K' indicator and carries no gradient, P_i carries it to the router):
//   ds_{t,i} = alpha f_i / T + the gate terms at the kept experts: dg (g = s), or
//              (dg_k - sum_j dg_j g_j) / Z with Z = sum_kept s (g = s / Z)
//   dl = s (ds - <s, ds>) (softmax over the routed experts), s (1 - s) ds (sigmoid), or
//        sigma(l) / (2 s) ds for s = sqrt(softplus(l)) (DeepSeek-V4 book ch. 2 section 2),
//        where sigma(l) = 1 - exp(-s^2) follows from s alone.
//   du += dl W_router, dW_router = dl^T u        (the affinity l = u W_router^T)
// The selection itself is held fixed (the indicator has no gradient).
#include <cfloat>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kGateThreads = 128;

// One block per token: dh_t is read once; each k's expert row y is read once and dotted
// with it in fp32; g_k dh_t is written to the k-th slot as bf16. The K' dot products are
// reduced over the block in a fixed order (deterministic).
template <int KMAX>
__global__ void __launch_bounds__(kGateThreads) gate_grad_kernel(const GateGradArgs a) {
  __shared__ int32_t s_slot[16];
  __shared__ float s_gate[16];
  __shared__ float s_red[kGateThreads / 32][16];
  const int K = a.K, d8 = a.d >> 3, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* __restrict__ dh4 = reinterpret_cast<const uint4*>(a.dh);
  const uint4* __restrict__ y4 = reinterpret_cast<const uint4*>(a.Y);
  uint4* __restrict__ dy4 = reinterpret_cast<uint4*>(a.dY);
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < K) {
      s_slot[threadIdx.x] = a.slot_of[static_cast<int64_t>(t) * K + threadIdx.x];
      s_gate[threadIdx.x] = a.gates[static_cast<int64_t>(t) * K + threadIdx.x];
    }
    __syncthreads();
    float dot[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) dot[k] = 0.f;
    for (int c = threadIdx.x; c < d8; c += kGateThreads) {
      const uint4 hv = dh4[static_cast<int64_t>(t) * d8 + c];
      const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
      float hf[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(hw[j]);
        hf[2 * j] = f.x;
        hf[2 * j + 1] = f.y;
      }
      uint4 yv[KMAX];
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const int p = k < K ? s_slot[k] : -1;
        yv[k] = p >= 0 ? y4[static_cast<int64_t>(p) * d8 + c] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const int p = k < K ? s_slot[k] : -1;
        if (p < 0) continue;
        const uint32_t w[4] = {yv[k].x, yv[k].y, yv[k].z, yv[k].w};
        float acc = dot[k];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(w[j]);
          acc = fmaf(hf[2 * j], f.x, acc);
          acc = fmaf(hf[2 * j + 1], f.y, acc);
        }
        dot[k] = acc;
        const float g = s_gate[k];
        dy4[static_cast<int64_t>(p) * d8 + c] =
            make_uint4(pack_bf16x2(g * hf[0], g * hf[1]), pack_bf16x2(g * hf[2], g * hf[3]),
                       pack_bf16x2(g * hf[4], g * hf[5]), pack_bf16x2(g * hf[6], g * hf[7]));
      }
    }
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      float v = dot[k];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s_red[warp][k] = v;
    }
    __syncthreads();
    if (threadIdx.x < K) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kGateThreads / 32; ++w) v += s_red[w][threadIdx.x];
      a.dg[static_cast<int64_t>(t) * K + threadIdx.x] = v;
    }
  }
}

constexpr int kRbWarps = 8;

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per token; lane j holds experts j, j + 32, ... (kNPL of them).
template <int kNPL>
__global__ void __launch_bounds__(kRbWarps * 32) router_backward_kernel(const RouterBwdArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N, K = a.K;
  float bal[kNPL];
#pragma unroll
  for (int j = 0; j < kNPL; ++j) {
    const int i = lane + 32 * j;
    bal[j] = (a.f && i < N) ? a.alpha * a.f[i] / static_cast<float>(a.T) : 0.f;
  }
  for (int t = blockIdx.x * kRbWarps + warp; t < a.T; t += gridDim.x * kRbWarps) {
    const float* srow = a.scores + static_cast<int64_t>(t) * N;
    float s[kNPL], ds[kNPL];
#pragma unroll
    for (int j = 0; j < kNPL; ++j) {
      const int i = lane + 32 * j;
      s[j] = i < N ? srow[i] : 0.f;
      ds[j] = bal[j];
    }
    // the gate terms at the kept experts: lane k < K holds pick k
    int e = -1;
    float dgk = 0.f, gk = 0.f, sk = 0.f;
    if (lane < K) {
      e = a.topk_idx[static_cast<int64_t>(t) * K + lane];
      dgk = a.dg[static_cast<int64_t>(t) * K + lane];
      gk = a.gates[static_cast<int64_t>(t) * K + lane];
      if (e < 0 || e >= N) {  // recorded, never dereferenced
        atomicOr(a.status, kStatusBadIndex);
        e = -1;
      } else {
        sk = srow[e];
      }
    }
    float contrib = dgk;
    if (a.renormalize) {
      const float Z = warp_sum_f(lane < K ? sk : 0.f);
      const float dot = warp_sum_f(lane < K ? dgk * gk : 0.f);
      contrib = (dgk - dot) / fmaxf(Z, FLT_MIN);
    }
    for (int k = 0; k < K; ++k) {
      const int ek = __shfl_sync(0xffffffffu, e, k);
      const float ck = __shfl_sync(0xffffffffu, contrib, k);
      if (ek >= 0 && (ek & 31) == lane) {
#pragma unroll
        for (int j = 0; j < kNPL; ++j)
          if (j == (ek >> 5)) ds[j] += ck;
      }
    }
    float dl[kNPL];
    if (a.score == 0) {  // softmax over the routed experts
      float sd = 0.f;
#pragma unroll
      for (int j = 0; j < kNPL; ++j) sd += s[j] * ds[j];
      sd = warp_sum_f(sd);
#pragma unroll
      for (int j = 0; j < kNPL; ++j) dl[j] = s[j] * (ds[j] - sd);
    } else if (a.score == 1) {  // sigmoid
#pragma unroll
      for (int j = 0; j < kNPL; ++j) dl[j] = s[j] * (1.f - s[j]) * ds[j];
    } else {  // sqrt(softplus): ds/dl = sigma(l) / (2 s), sigma(l) = 1 - exp(-s^2)
#pragma unroll
      for (int j = 0; j < kNPL; ++j) {
        const float sq = s[j] * s[j];
        const float slope = sq > 1e-12f ? -expm1f(-sq) / (2.f * s[j]) : 0.5f * s[j];
        dl[j] = slope * ds[j];
      }
    }
    float* drow = a.dlogits + static_cast<int64_t>(t) * N;
#pragma unroll
    for (int j = 0; j < kNPL; ++j)
      if (lane + 32 * j < N) drow[lane + 32 * j] = dl[j];
  }
}

// dx = dh + (shared experts' fp32 rows) + (router part) + sum of the token's slot rows,
// accumulated in fp32 in that order; 8 elements (16 bytes of each bf16 source) per step.
template <int KMAX>
__global__ void __launch_bounds__(128) dx_combine_kernel(const bf16* __restrict__ dh, const float* __restrict__ dXs,
                                                          const float* __restrict__ dx_add,
                                                          const bf16* __restrict__ dXp,
                                                          const int32_t* __restrict__ slot_of, int T, int K, int d,
                                                          float* __restrict__ dx) {
  __shared__ int32_t s_slot[16];
  const int d8 = d >> 3;
  const uint4* dh4 = reinterpret_cast<const uint4*>(dh);
  const uint4* dp4 = reinterpret_cast<const uint4*>(dXp);
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < K) s_slot[threadIdx.x] = slot_of[static_cast<int64_t>(t) * K + threadIdx.x];
    __syncthreads();
    for (int c = threadIdx.x; c < d8; c += blockDim.x) {
      uint4 pv[KMAX];
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const int p = k < K ? s_slot[k] : -1;
        pv[k] = p >= 0 ? dp4[static_cast<int64_t>(p) * d8 + c] : make_uint4(0u, 0u, 0u, 0u);
      }
      float acc[8];
      const uint4 hv = dh4[static_cast<int64_t>(t) * d8 + c];
      const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(hw[j]);
        acc[2 * j] = f.x;
        acc[2 * j + 1] = f.y;
      }
      const int64_t o = static_cast<int64_t>(t) * d + 8 * c;
      if (dXs) {
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += dXs[o + j];
      }
      if (dx_add) {
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += dx_add[o + j];
      }
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        if (k >= K || s_slot[k] < 0) continue;
        const uint32_t w[4] = {pv[k].x, pv[k].y, pv[k].z, pv[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(w[j]);
          acc[2 * j] += f.x;
          acc[2 * j + 1] += f.y;
        }
      }
      float4* o4 = reinterpret_cast<float4*>(dx + o);
      o4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// C[m, n] = sum_k A(m, k) B[k, n] on the CUDA cores: A fp32 with element (m, k) at
// A[m * a_sm + k * a_sk], B bf16 row-major [K, ldb], C fp32 [M, ldc]. A block computes a
// 128 x 128 tile from 16-deep slices staged in shared memory (B converted to fp32 there);
// each thread owns 8 x 8 outputs, rows 4ty.. and 64 + 4ty.., columns 4tx.. and 64 + 4tx..,
// read as float4 from shared memory (fixed summation order: k ascending).
constexpr int kGm = 128, kGn = 128, kGk = 16, kGThreads = 256;

__global__ void __launch_bounds__(kGThreads, 2) gemm_f32_bf16_kernel(const GemmF32Args a) {
  __shared__ __align__(16) float sA[kGk][kGm];
  __shared__ __align__(16) float sB[kGk][kGn];
  const int m0 = blockIdx.y * kGm, n0 = blockIdx.x * kGn;
  // split z of the K range (split-K: each split writes its own partial C, summed later)
  const int kc = a.splits > 1 ? ((a.K + a.splits - 1) / a.splits + kGk - 1) / kGk * kGk : a.K;
  const int kz0 = blockIdx.z * kc, kz1 = min(a.K, kz0 + kc);
  float* C = a.splits > 1 ? a.partial + static_cast<int64_t>(blockIdx.z) * a.M * a.ldc : a.C;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;  // 16 x 16 threads
  const bool m_fast = a.a_sm == 1;  // A's contiguous dimension
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = kz0; k0 < kz1; k0 += kGk) {
    // consecutive threads walk A's contiguous dimension: m when a_sm == 1, else k
#pragma unroll
    for (int u = 0; u < kGm * kGk / kGThreads; ++u) {
      const int idx = threadIdx.x + u * kGThreads;
      const int mm = m_fast ? idx % kGm : idx / kGk, kk = m_fast ? idx / kGm : idx % kGk;
      const int m = m0 + mm, k = k0 + kk;
      sA[kk][mm] = (m < a.M && k < kz1) ? a.A[static_cast<int64_t>(m) * a.a_sm + static_cast<int64_t>(k) * a.a_sk]
                                         : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kGk * kGn / kGThreads; ++u) {
      const int idx = threadIdx.x + u * kGThreads;
      const int kk = idx / kGn, nn = idx % kGn;
      const int k = k0 + kk, n = n0 + nn;
      sB[kk][nn] = (k < kz1 && n < a.N) ? __bfloat162float(a.B[static_cast<int64_t>(k) * a.ldb + n]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGk; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&sA[kk][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sA[kk][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&sB[kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sB[kk][64 + 4 * tx]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? 4 * tx + j : 64 + 4 * tx + j - 4);
      if (n < a.N) C[static_cast<int64_t>(m) * a.ldc + n] = acc[i][j];
    }
  }
}

// C[m, n] = sum over z = 0.. in order of partial[z][m, n] (the split-K partial sums).
__global__ void split_sum_kernel(const float* __restrict__ partial, int splits, int M, int N, int64_t ldc,
                                 float* __restrict__ C) {
  const int64_t total = static_cast<int64_t>(M) * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i % N, o = m * ldc + n;
    float v = 0.f;
    for (int z = 0; z < splits; ++z) v += partial[z * static_cast<int64_t>(M) * ldc + o];
    C[o] = v;
  }
}
// dl = hi + lo with hi = bf16(dl) and lo = bf16(dl - hi) (what remains is below 2^-16 of
// |dl|), written as rows [hi | lo] of 2N bf16: the router's backward contractions then run
// on the tensor cores as bf16 products summed in fp32. Four consecutive values per thread.
__global__ void hilo_split_kernel(const float* __restrict__ src, bf16* __restrict__ dst, int T, int N) {
  const int64_t quads = static_cast<int64_t>(T) * N / 4;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < quads;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = 4 * i, t = e / N;
    const int j = static_cast<int>(e - t * N);
    const float4 v = *reinterpret_cast<const float4*>(src + e);
    const float x[4] = {v.x, v.y, v.z, v.w};
    __align__(8) bf16 hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      hi[k] = __float2bfloat16_rn(x[k]);
      lo[k] = __float2bfloat16_rn(x[k] - __bfloat162float(hi[k]));
    }
    bf16* row = dst + t * 2 * N;
    *reinterpret_cast<uint2*>(row + j) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(row + N + j) = *reinterpret_cast<const uint2*>(lo);
  }
}
}  // namespace

cudaError_t launch_hilo_split(const float* src, bf16* dst, int T, int N, int num_sms, cudaStream_t s) {
  if (N % 4) return cudaErrorInvalidValue;
  const int64_t quads = static_cast<int64_t>(T) * N / 4;
  if (quads <= 0) return cudaSuccess;
  int64_t grid = (quads + 255) / 256;
  if (grid > 8 * num_sms) grid = 8 * num_sms;
  hilo_split_kernel<<<static_cast<int>(grid), 256, 0, s>>>(src, dst, T, N);
  return cudaGetLastError();
}

cudaError_t launch_split_sum(const float* partial, int splits, int M, int N, int64_t ldc, float* C, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  split_sum_kernel<<<1024, 256, 0, s>>>(partial, splits, M, N, ldc, C);
  return cudaGetLastError();
}

cudaError_t launch_gate_grad(const GateGradArgs& a, int num_sms, cudaStream_t s) {
  int grid = a.T;
  if (grid > 16 * num_sms) grid = 16 * num_sms;
  if (grid < 1) grid = 1;
  if (a.K <= 2) gate_grad_kernel<2><<<grid, kGateThreads, 0, s>>>(a);
  else if (a.K <= 4) gate_grad_kernel<4><<<grid, kGateThreads, 0, s>>>(a);
  else if (a.K <= 8) gate_grad_kernel<8><<<grid, kGateThreads, 0, s>>>(a);
  else if (a.K <= 16) gate_grad_kernel<16><<<grid, kGateThreads, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_router_backward(const RouterBwdArgs& a, int num_sms, cudaStream_t s) {
  int grid = (a.T + kRbWarps - 1) / kRbWarps;
  if (grid > 8 * num_sms) grid = 8 * num_sms;
  if (grid < 1) grid = 1;
  const int npl = (a.N + 31) / 32;
  if (npl <= 1) router_backward_kernel<1><<<grid, kRbWarps * 32, 0, s>>>(a);
  else if (npl <= 2) router_backward_kernel<2><<<grid, kRbWarps * 32, 0, s>>>(a);
  else if (npl <= 4) router_backward_kernel<4><<<grid, kRbWarps * 32, 0, s>>>(a);
  else if (npl <= 8) router_backward_kernel<8><<<grid, kRbWarps * 32, 0, s>>>(a);
  else if (npl <= 12) router_backward_kernel<12><<<grid, kRbWarps * 32, 0, s>>>(a);
  else if (npl <= 16) router_backward_kernel<16><<<grid, kRbWarps * 32, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_dx_combine(const bf16* dh, const float* dXs, const float* dx_add, const bf16* dXp,
                              const int32_t* slot_of, int T, int K, int d, float* dx, int num_sms, cudaStream_t s) {
  int grid = T;
  if (grid > 16 * num_sms) grid = 16 * num_sms;
  if (grid < 1) grid = 1;
  if (K <= 2) dx_combine_kernel<2><<<grid, 128, 0, s>>>(dh, dXs, dx_add, dXp, slot_of, T, K, d, dx);
  else if (K <= 4) dx_combine_kernel<4><<<grid, 128, 0, s>>>(dh, dXs, dx_add, dXp, slot_of, T, K, d, dx);
  else if (K <= 8) dx_combine_kernel<8><<<grid, 128, 0, s>>>(dh, dXs, dx_add, dXp, slot_of, T, K, d, dx);
  else if (K <= 16) dx_combine_kernel<16><<<grid, 128, 0, s>>>(dh, dXs, dx_add, dXp, slot_of, T, K, d, dx);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_gemm_f32_bf16(const GemmF32Args& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  const int splits = a.splits > 1 ? a.splits : 1;
  if (splits > 1 && !a.partial) return cudaErrorInvalidValue;
  const dim3 grid((a.N + kGn - 1) / kGn, (a.M + kGm - 1) / kGm, splits);
  if (grid.y > 65535 || splits > 64) return cudaErrorInvalidValue;
  gemm_f32_bf16_kernel<<<grid, kGThreads, 0, s>>>(a);
  if (splits > 1) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    split_sum_kernel<<<1024, 256, 0, s>>>(a.partial, splits, a.M, a.N, a.ldc, a.C);
  }
  return cudaGetLastError();
}

}  // namespace dsmoe
