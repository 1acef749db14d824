// permute.cu -- expert histogram scan, balance statistics, and the token permutation that
// gathers each token's row once per selected expert into expert-contiguous order.
//
// Balance statistics (DeepSeekMoE summary, "Expert-level balance loss"):
//   f_i = N' / (K' T) * sum_t 1(token t selects expert i),  P_i = (1/T) sum_t s_{i,t}.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kScanThreads = 512;  // one thread per expert (N' <= 512)

__global__ void __launch_bounds__(kScanThreads) scan_stats_kernel(const ScanArgs a) {
  __shared__ int32_t warp_tot[kScanThreads / 32];
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const int32_t c = (i < a.N) ? a.counts_ws[i] : 0;
  // slots exist only for the experts in [e_begin, e_end); the statistics use every count
  const int32_t c_slots = (i >= a.e_begin && i < a.e_end) ? c : 0;
  if (i < a.N) {
    a.counts[i] = c;
    a.f[i] = (a.T > 0) ? static_cast<float>(static_cast<double>(a.N) * c / (static_cast<double>(a.K) * a.T)) : 0.f;
    double p = 0.0;
    if (a.P_part)
      for (int r = 0; r < a.n_part; ++r) p += a.P_part[static_cast<int64_t>(r) * a.N + i];
    if (a.P_sum) a.P_sum[i] = static_cast<float>(p);
    a.P[i] = (a.T > 0) ? static_cast<float>(p / static_cast<double>(a.T)) : 0.f;
    if (a.cursor) a.cursor[i] = 0;
  }
  if (!a.offsets) return;
  // exclusive scan of the slot counts -> slot offset of each expert's segment
  int32_t v = c_slots;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int32_t w = (lane < kScanThreads / 32) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < kScanThreads / 32) warp_tot[lane] = w;  // inclusive totals of warps
  }
  __syncthreads();
  const int32_t incl = v + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (i < a.N) a.offsets[i] = incl - c_slots;
  if (i == a.N - 1) a.offsets[a.N] = incl;
}

__global__ void balance_stats_kernel(const int32_t* __restrict__ counts, const float* __restrict__ P_sum,
                                     int64_t T, int N, int K, float* __restrict__ f, float* __restrict__ P) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    f[i] = (T > 0) ? static_cast<float>(static_cast<double>(N) * counts[i] / (static_cast<double>(K) * T)) : 0.f;
    P[i] = (T > 0 && P_sum) ? static_cast<float>(static_cast<double>(P_sum[i]) / static_cast<double>(T)) : 0.f;
  }
}

// One warp per token: lanes k < K' claim a slot in expert topk_idx[t,k]'s segment (experts
// in [e_begin, e_end) only; the others get slot -1), then the warp copies the token's row
// (16-byte vectors) to each claimed slot.
__global__ void __launch_bounds__(256) permute_gather_kernel(const bf16* __restrict__ x,
                                                             const int32_t* __restrict__ topk_idx,
                                                             const int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ cursor, int T, int K, int N,
                                                             int e_begin, int e_end, int d,
                                                             int32_t* __restrict__ slot_of,
                                                             bf16* __restrict__ Xp, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nw = (gridDim.x * blockDim.x) >> 5;
  const int d8 = d >> 3;
  const uint4* __restrict__ x4 = reinterpret_cast<const uint4*>(x);
  uint4* __restrict__ xp4 = reinterpret_cast<uint4*>(Xp);
  for (int t = gw; t < T; t += nw) {
    int pos = -1;
    if (lane < K) {
      const int e = topk_idx[static_cast<int64_t>(t) * K + lane];
      if (e < 0 || e >= N) {
        atomicOr(status, kStatusBadIndex);
      } else if (e >= e_begin && e < e_end) {
        pos = offsets[e] + atomicAdd(&cursor[e], 1);
      }
      slot_of[static_cast<int64_t>(t) * K + lane] = pos;
    }
    int pk[16];  // every lane learns all K' slots (uniform shuffles, K' <= 16)
#pragma unroll
    for (int k = 0; k < 16; ++k) pk[k] = __shfl_sync(0xffffffffu, pos, k);
    const uint4* src = x4 + static_cast<int64_t>(t) * d8;
    // four 16-byte chunks per lane per step: their loads are all in flight before the
    // first store
    for (int c0 = lane; c0 < d8; c0 += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < d8) v[u] = src[c];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < d8) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (k < K && pk[k] >= 0) xp4[static_cast<int64_t>(pk[k]) * d8 + c] = v[u];
        }
      }
    }
  }
}
__global__ void block_rows_kernel(const int32_t* __restrict__ offsets, int N, int world, int32_t* __restrict__ out) {
  for (int j = threadIdx.x; j < world; j += blockDim.x) {
    const int base = N / world, extra = N % world;
    const int e0 = j * base + min(j, extra), e1 = e0 + base + (j < extra ? 1 : 0);
    out[j] = offsets[e1] - offsets[e0];
  }
}

// One block of kScanThreads threads: an exclusive scan of up to kScanThreads counts.
__global__ void __launch_bounds__(kScanThreads) group_offsets_kernel(const int32_t* __restrict__ counts, int groups,
                                                                      int32_t* __restrict__ offsets,
                                                                      uint32_t* status) {
  __shared__ int32_t warp_tot[kScanThreads / 32];
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  int32_t c = (i < groups) ? counts[i] : 0;
  if (c < 0) {
    atomicOr(status, kStatusBadIndex);
    c = 0;
  }
  int32_t v = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int32_t w = (lane < kScanThreads / 32) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < kScanThreads / 32) warp_tot[lane] = w;
  }
  __syncthreads();
  const int32_t incl = v + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (i < groups) offsets[i] = incl - c;
  if (i == groups - 1) offsets[groups] = incl;
}
}  // namespace

cudaError_t launch_block_rows(const int32_t* offsets, int N, int world, int32_t* out, cudaStream_t s) {
  block_rows_kernel<<<1, 256, 0, s>>>(offsets, N, world, out);
  return cudaGetLastError();
}

cudaError_t launch_group_offsets(const int32_t* counts, int groups, int32_t* offsets, uint32_t* status,
                                 cudaStream_t s) {
  if (groups < 1 || groups > kScanThreads) return cudaErrorInvalidValue;
  group_offsets_kernel<<<1, kScanThreads, 0, s>>>(counts, groups, offsets, status);
  return cudaGetLastError();
}

cudaError_t launch_scan_stats(const ScanArgs& a, cudaStream_t s) {
  scan_stats_kernel<<<1, kScanThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_balance_stats(const int32_t* counts, const float* P_sum, int64_t T, int N, int K, float* f,
                                 float* P, cudaStream_t s) {
  balance_stats_kernel<<<(N + 255) / 256, 256, 0, s>>>(counts, P_sum, T, N, K, f, P);
  return cudaGetLastError();
}

cudaError_t launch_permute_gather(const bf16* x, const int32_t* topk_idx, const int32_t* offsets,
                                  int32_t* cursor, int T, int K, int N, int e_begin, int e_end, int d,
                                  int32_t* slot_of, bf16* Xp, uint32_t* status, int num_sms, cudaStream_t s) {
  const int warps_per_block = 8;
  int grid = (T + warps_per_block - 1) / warps_per_block;
  if (grid > 8 * num_sms) grid = 8 * num_sms;
  if (grid < 1) grid = 1;
  permute_gather_kernel<<<grid, warps_per_block * 32, 0, s>>>(x, topk_idx, offsets, cursor, T, K, N, e_begin,
                                                              e_end, d, slot_of, Xp, status);
  return cudaGetLastError();
}

}  // namespace dsmoe
