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
// The base of each row is Hs (fp32 residual + shared experts), x, or zero; the routed
// terms of slots set to -1 (experts another rank applies) are left out. The result is
// rounded to bf16 once, or stored as fp32 when h32 is set (a partial sum that ranks add).
template <int KMAX>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineArgs a) {
  __shared__ int32_t s_slot[16];
  __shared__ float s_gate[16];
  const int K = a.K, d = a.d, d8 = d >> 3;
  const uint4* __restrict__ x4 = reinterpret_cast<const uint4*>(a.x);
  const uint4* __restrict__ y4 = reinterpret_cast<const uint4*>(a.Y);
  uint4* __restrict__ h4 = reinterpret_cast<uint4*>(a.h);
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < K) {
      s_slot[threadIdx.x] = a.slot_of[static_cast<int64_t>(t) * K + threadIdx.x];
      s_gate[threadIdx.x] = a.gates[static_cast<int64_t>(t) * K + threadIdx.x];
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
      if (a.Hs) {
        const float4* hs4 = reinterpret_cast<const float4*>(a.Hs + static_cast<int64_t>(t) * d) + 2 * c;
        const float4 a0 = hs4[0], a1 = hs4[1];
        acc[0] = a0.x; acc[1] = a0.y; acc[2] = a0.z; acc[3] = a0.w;
        acc[4] = a1.x; acc[5] = a1.y; acc[6] = a1.z; acc[7] = a1.w;
      } else if (a.add_x) {
        const uint4 v = x4[static_cast<int64_t>(t) * d8 + c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(w[j]);
          acc[2 * j] = f.x;
          acc[2 * j + 1] = f.y;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.f;
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
      if (a.h32) {
        float4* o4 = reinterpret_cast<float4*>(a.h32 + static_cast<int64_t>(t) * d) + 2 * c;
        o4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        o4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        h4[static_cast<int64_t>(t) * d8 + c] = o;
      }
    }
  }
}

// Eight fp32 values per thread and step -> one 16-byte bf16 store.
__global__ void round_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, int64_t n8) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = s4[2 * i], b = s4[2 * i + 1];
    d4[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                       pack_bf16x2(b.z, b.w));
  }
}
}  // namespace

cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s) {
  int grid = a.T;
  if (grid > 16 * num_sms) grid = 16 * num_sms;
  if (grid < 1) grid = 1;
  if (a.K <= 2)
    combine_kernel<2><<<grid, kCombineThreads, 0, s>>>(a);
  else if (a.K <= 4)
    combine_kernel<4><<<grid, kCombineThreads, 0, s>>>(a);
  else if (a.K <= 8)
    combine_kernel<8><<<grid, kCombineThreads, 0, s>>>(a);
  else if (a.K <= 16)
    combine_kernel<16><<<grid, kCombineThreads, 0, s>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_round_bf16(const float* src, bf16* dst, int64_t n, int num_sms, cudaStream_t s) {
  if (n % 8) return cudaErrorInvalidValue;
  const int64_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  int64_t grid = (n8 + 255) / 256;
  if (grid > 8 * num_sms) grid = 8 * num_sms;
  round_bf16_kernel<<<static_cast<int>(grid), 256, 0, s>>>(src, dst, n8);
  return cudaGetLastError();
}

}  // namespace dsmoe
