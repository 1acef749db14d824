// combine.cu -- gate-weighted combine with the residual (DeepSeekMoE summary,
// shared-expert layer equation):
//   h_t = u_t + sum_{shared} FFN_i(u_t) + sum_k g_{t,k} FFN_{e(t,k)}(u_t)
// accumulated in fp32 and rounded to bf16 once. The residual plus the shared experts'
// sum arrives as one fp32 row Hs[t] (written by the down-projection GEMM, which
// accumulates across the shared experts); the routed terms are gathered from the
// expert-contiguous rows Y[slot_of[t,k]].
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kCombineThreads = 128;

// KMAX >= K bounds the unrolled gather: every 16-byte load of a chunk's K expert rows
// is issued before the first FMA, so a thread keeps K loads in flight instead of one.
template <int KMAX>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const bf16* __restrict__ x,
                                                                  const float* __restrict__ Hs,
                                                                  const bf16* __restrict__ Y,
                                                                  const int32_t* __restrict__ slot_of,
                                                                  const float* __restrict__ gates, int T, int K,
                                                                  int d, bf16* __restrict__ h) {
  __shared__ int32_t s_slot[16];
  __shared__ float s_gate[16];
  const int d8 = d >> 3;
  const uint4* __restrict__ x4 = reinterpret_cast<const uint4*>(x);
  const uint4* __restrict__ y4 = reinterpret_cast<const uint4*>(Y);
  uint4* __restrict__ h4 = reinterpret_cast<uint4*>(h);
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < K) {
      s_slot[threadIdx.x] = slot_of[static_cast<int64_t>(t) * K + threadIdx.x];
      s_gate[threadIdx.x] = gates[static_cast<int64_t>(t) * K + threadIdx.x];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < d8; c += kCombineThreads) {
      uint4 yv[KMAX];
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const int p = k < K ? s_slot[k] : -1;
        yv[k] = p >= 0 ? y4[static_cast<int64_t>(p) * d8 + c] : make_uint4(0u, 0u, 0u, 0u);
      }
      float acc[8];
      if (Hs) {
        const float4* hs4 = reinterpret_cast<const float4*>(Hs + static_cast<int64_t>(t) * d) + 2 * c;
        const float4 a0 = hs4[0], a1 = hs4[1];
        acc[0] = a0.x; acc[1] = a0.y; acc[2] = a0.z; acc[3] = a0.w;
        acc[4] = a1.x; acc[5] = a1.y; acc[6] = a1.z; acc[7] = a1.w;
      } else {
        const uint4 v = x4[static_cast<int64_t>(t) * d8 + c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(w[j]);
          acc[2 * j] = f.x;
          acc[2 * j + 1] = f.y;
        }
      }
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        if (k >= K || s_slot[k] < 0) continue;
        const float g = s_gate[k];
        const uint32_t w[4] = {yv[k].x, yv[k].y, yv[k].z, yv[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(w[j]);
          acc[2 * j] = fmaf(g, f.x, acc[2 * j]);
          acc[2 * j + 1] = fmaf(g, f.y, acc[2 * j + 1]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      h4[static_cast<int64_t>(t) * d8 + c] = o;
    }
  }
}
}  // namespace

cudaError_t launch_combine(const bf16* x, const float* Hs, const bf16* Y, const int32_t* slot_of,
                           const float* gates, int T, int K, int d, bf16* h, int num_sms, cudaStream_t s) {
  int grid = T;
  if (grid > 16 * num_sms) grid = 16 * num_sms;
  if (grid < 1) grid = 1;
  if (K <= 2)
    combine_kernel<2><<<grid, kCombineThreads, 0, s>>>(x, Hs, Y, slot_of, gates, T, K, d, h);
  else if (K <= 4)
    combine_kernel<4><<<grid, kCombineThreads, 0, s>>>(x, Hs, Y, slot_of, gates, T, K, d, h);
  else if (K <= 8)
    combine_kernel<8><<<grid, kCombineThreads, 0, s>>>(x, Hs, Y, slot_of, gates, T, K, d, h);
  else if (K <= 16)
    combine_kernel<16><<<grid, kCombineThreads, 0, s>>>(x, Hs, Y, slot_of, gates, T, K, d, h);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace dsmoe
