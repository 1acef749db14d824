// route_noalloc.cu -- the routing stage of the layer (router affinities, scores,
// top-K' selection, gates, expert counts, f_i and P_i) as one kernel that needs no
// allocation by anyone: its scratch is a fixed array in the library's own device
// memory image.
//
// Who this is for: code that runs where device memory cannot be requested at the
// time of the call -- a caller whose framework owns every byte of the GPU through
// a pre-reserved pool, a plugin that must not touch the allocator while its host
// is serving, or code that must not create a handle (dsmoe_create allocates the
// workspace). Such a caller passes its own input and output buffers and nothing
// else.
//
// Scratch: g_route_scratch below, a static __device__ array of kScratchBytes
// (about 514 KiB) that every GPU loading the library keeps until the process
// exits. It holds per-block partial score sums (at most kMaxBlocks blocks of at
// most kMaxExperts experts), the expert counters and a block-completion ticket.
// Host code cannot use the array's name as a device address; the entry point
// looks the address up with cudaGetSymbolAddress once per device (on its first
// call on that device, with that device current) and passes it to the kernel.
//
// Every call shares the array and it keeps the last call's contents; each call
// clears the counters and the ticket on its stream before its kernel starts.
// Calls whose work overlaps on the GPU (other streams, other host threads) race
// on the array and must be serialised by the caller.
//
// Each logit is one sequential fp32 fma chain over k in ascending order; scores,
// top-K' (ties to the lower index), gates and statistics follow the same definitions
// as dsmoe_forward. The two agree up to fp32 rounding: experts whose selection keys
// tie within rounding may be picked or ordered differently, and P differs in the
// order of its sums.
#include <float.h>
#include <math.h>

#include <mutex>

#include "dsmoe.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

#define DSMOE_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kThreads = 256;     // one token per block at a time
constexpr int kMaxBlocks = 256;   // rows of the partial-sum table
constexpr int kMaxExperts = 512;  // columns of the partial-sum table (N' limit)
constexpr int kMaxDevices = 64;
constexpr size_t kPartialBytes = sizeof(float) * kMaxBlocks * kMaxExperts;
constexpr size_t kCountsOff = kPartialBytes;
constexpr size_t kTicketOff = kCountsOff + sizeof(int32_t) * kMaxExperts;
constexpr size_t kScratchBytes = kTicketOff + 256;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

__device__ __forceinline__ float warp_max_(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct RouteArgs {
  const dsmoe::bf16* x;
  const dsmoe::bf16* W;
  const float* b;
  int T, N, K, d, score, bias_mode, renormalize;
  int32_t* topk_idx;
  float* gates;
  int32_t* counts;
  float* f;
  float* P;
  unsigned char* scratch;  // device address of g_route_scratch
};

template <int kNPL>
__global__ void __launch_bounds__(kThreads) route_noalloc_kernel(const RouteArgs a) {
  __shared__ float s_logit[kMaxExperts];
  __shared__ bool s_last;
  float* partial = reinterpret_cast<float*>(a.scratch);
  int32_t* cnt = reinterpret_cast<int32_t*>(a.scratch + kCountsOff);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(a.scratch + kTicketOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.N, K = a.K, d8 = a.d >> 3;
  const bool bias_in_logits = a.bias_mode == DSMOE_BIAS_IN_LOGITS;
  const bool bias_select = a.bias_mode == DSMOE_BIAS_SELECT_ONLY;
  float pacc[kNPL], bias[kNPL];
#pragma unroll
  for (int j = 0; j < kNPL; ++j) {
    pacc[j] = 0.f;
    const int i = lane + 32 * j;
    bias[j] = (bias_select && i < N) ? a.b[i] : 0.f;
  }
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
    // affinities: thread n owns experts n and n + 256, one sequential fma chain each
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<int64_t>(t) * a.d);
    for (int n = tid; n < N; n += kThreads) {
      const uint4* wr = reinterpret_cast<const uint4*>(a.W + static_cast<int64_t>(n) * a.d);
      float acc = 0.f;
      for (int c = 0; c < d8; ++c) {
        const uint4 xv = xr[c], wv = wr[c];
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 fx = dsmoe::unpack_bf16x2(xw[j]), fw = dsmoe::unpack_bf16x2(ww[j]);
          acc = fmaf(fx.x, fw.x, acc);
          acc = fmaf(fx.y, fw.y, acc);
        }
      }
      s_logit[n] = acc + (bias_in_logits ? a.b[n] : 0.f);
    }
    __syncthreads();
    if (warp == 0) {
      float s[kNPL];
#pragma unroll
      for (int j = 0; j < kNPL; ++j) {
        const int i = lane + 32 * j;
        s[j] = (i < N) ? s_logit[i] : -INFINITY;
      }
      if (a.score == DSMOE_SCORE_SOFTMAX) {
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < kNPL; ++j) m = fmaxf(m, s[j]);
        m = warp_max_(m);
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < kNPL; ++j) {
          s[j] = (lane + 32 * j < N) ? expf(s[j] - m) : 0.f;
          z += s[j];
        }
        z = warp_sum_(z);
        const float inv = 1.f / z;
#pragma unroll
        for (int j = 0; j < kNPL; ++j) s[j] *= inv;
      } else if (a.score == DSMOE_SCORE_SIGMOID) {
#pragma unroll
        for (int j = 0; j < kNPL; ++j) s[j] = (lane + 32 * j < N) ? 1.f / (1.f + expf(-s[j])) : 0.f;
      } else {
#pragma unroll
        for (int j = 0; j < kNPL; ++j)
          s[j] = (lane + 32 * j < N) ? sqrtf(fmaxf(s[j], 0.f) + log1pf(expf(-fabsf(s[j])))) : 0.f;
      }
      float key[kNPL];
#pragma unroll
      for (int j = 0; j < kNPL; ++j) {
        const float kv = s[j] + bias[j];
        key[j] = (lane + 32 * j < N && !isnan(kv)) ? kv : -INFINITY;
      }
      uint32_t taken = 0;
      int my_idx = 0;
      float my_s = 0.f;
      for (int r = 0; r < K; ++r) {
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
        if (lane == r) {
          my_idx = bi;
          my_s = bs;
        }
      }
      float g = my_s;
      if (a.renormalize) {
        const float z = warp_sum_(lane < K ? my_s : 0.f);
        g = my_s / fmaxf(z, FLT_MIN);
      }
      if (lane < K) {
        if (my_idx < 0 || my_idx >= N) my_idx = 0;  // unreachable for K' <= N'
        a.topk_idx[static_cast<int64_t>(t) * K + lane] = my_idx;
        a.gates[static_cast<int64_t>(t) * K + lane] = g;
        atomicAdd(&cnt[my_idx], 1);
      }
#pragma unroll
      for (int j = 0; j < kNPL; ++j) pacc[j] += s[j];
    }
    __syncthreads();  // s_logit is rewritten for the next token
  }
  // this block's partial score sums, then the last block to finish reduces them
  if (warp == 0) {
#pragma unroll
    for (int j = 0; j < kNPL; ++j)
      if (lane + 32 * j < N) partial[static_cast<int64_t>(blockIdx.x) * kMaxExperts + lane + 32 * j] = pacc[j];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int n = tid; n < N; n += kThreads) {
    const int32_t c = *reinterpret_cast<volatile int32_t*>(&cnt[n]);
    double p = 0.0;
    for (int r = 0; r < static_cast<int>(gridDim.x); ++r)
      p += *reinterpret_cast<volatile float*>(&partial[static_cast<int64_t>(r) * kMaxExperts + n]);
    a.counts[n] = c;
    a.f[n] = static_cast<float>(static_cast<double>(N) * c / (static_cast<double>(K) * a.T));
    a.P[n] = static_cast<float>(p / static_cast<double>(a.T));
  }
}

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

// The routing stage with no allocation; declared and documented in dsmoe.h.
DSMOE_EXPORT dsmoe_status dsmoe_route_noalloc(const dsmoe_cfg* cfg, int32_t T, const void* x, const void* W_router,
                                              const float* b, int32_t* topk_idx, float* gates, int32_t* counts,
                                              float* f, float* P, void* stream) {
  const dsmoe_status st = dsmoe_check_config(cfg);
  if (st != DSMOE_OK) return st;
  if (cfg->score == DSMOE_ROUTE_HASH) {
    dsmoe::note_error("dsmoe_route_noalloc: hash routing has no router to run");
    return DSMOE_ERR_UNSUPPORTED;
  }
  if (cfg->n_routed > kMaxExperts) {
    dsmoe::note_error("dsmoe_route_noalloc: n_routed %d exceeds the %d experts its fixed scratch holds",
                      cfg->n_routed, kMaxExperts);
    return DSMOE_ERR_UNSUPPORTED;
  }
  if (T < 0 || T > cfg->max_tokens) {
    dsmoe::note_error("dsmoe_route_noalloc: T = %d outside [0, max_tokens = %d]", T, cfg->max_tokens);
    return DSMOE_ERR_WORKSPACE;
  }
  if (!counts || !f || !P || (T > 0 && (!x || !W_router || !topk_idx || !gates)) ||
      (cfg->bias_mode != DSMOE_BIAS_NONE && !b)) {
    dsmoe::note_error("dsmoe_route_noalloc: a required pointer is NULL");
    return DSMOE_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(W_router)) & 15u) {
    dsmoe::note_error("dsmoe_route_noalloc: x and W_router must be 16-byte aligned");
    return DSMOE_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    dsmoe::note_error("dsmoe_route_noalloc: no usable current device");
    return DSMOE_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array's device address is looked up with the device current and kept per
  // device. A call whose stream is not being captured looks it up again, so that the
  // address stays right after cudaDeviceReset reloads the library's device image; a
  // call under capture uses the address an earlier call found.
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) {
    dsmoe::note_error("dsmoe_route_noalloc: cudaStreamIsCapturing failed on the given stream");
    return DSMOE_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_addr[dev] || capture == cudaStreamCaptureStatusNone) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
      if (e != cudaSuccess || !p) {
        dsmoe::note_error("dsmoe_route_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return DSMOE_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  const int N = cfg->n_routed;
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, N * sizeof(int32_t), s) != cudaSuccess ||
        cudaMemsetAsync(f, 0, N * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(P, 0, N * sizeof(float), s) != cudaSuccess)
      return DSMOE_ERR_CUDA;
    return DSMOE_OK;
  }
  // counters and the completion ticket start at zero for every call
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + kCountsOff, 0, kScratchBytes - kCountsOff, s) !=
      cudaSuccess)
    return DSMOE_ERR_CUDA;
  RouteArgs a{static_cast<const dsmoe::bf16*>(x), static_cast<const dsmoe::bf16*>(W_router), b, T, N, cfg->top_k,
              cfg->d_model, cfg->score, cfg->bias_mode, cfg->renormalize, topk_idx, gates, counts, f, P,
              static_cast<unsigned char*>(scratch)};
  const int grid = T < kMaxBlocks ? T : kMaxBlocks;
  const int npl = (N + 31) / 32;
  if (npl <= 1) route_noalloc_kernel<1><<<grid, kThreads, 0, s>>>(a);
  else if (npl <= 2) route_noalloc_kernel<2><<<grid, kThreads, 0, s>>>(a);
  else if (npl <= 4) route_noalloc_kernel<4><<<grid, kThreads, 0, s>>>(a);
  else if (npl <= 8) route_noalloc_kernel<8><<<grid, kThreads, 0, s>>>(a);
  else if (npl <= 12) route_noalloc_kernel<12><<<grid, kThreads, 0, s>>>(a);
  else route_noalloc_kernel<16><<<grid, kThreads, 0, s>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    dsmoe::note_error("dsmoe_route_noalloc: launch failed: %s", cudaGetErrorString(e));
    return DSMOE_ERR_CUDA;
  }
  return DSMOE_OK;
}
