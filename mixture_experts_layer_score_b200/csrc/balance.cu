// balance.cu -- load-balance control computed from a forward's routing statistics.
//
//   expert level   L_ExpBal = alpha_1 (1/N') sum_i f_i P_i
//   device level   f'_d = mean_{j in E_d} f_j,  P'_d = sum_{j in E_d} P_j,
//                  L_DevBal = alpha_2 sum_d f'_d P'_d
//                  (DeepSeekMoE summary, "Expert-level / Device-level balance loss")
//   sequence-wise  f_i^seq = share of a sequence's tokens that selected expert i,
//                  p_i^seq = mean score of expert i over the sequence,
//                  loss = beta * mean over sequences of sum_i f_i^seq p_i^seq
//   bias update    b_i <- b_i + alpha (K'/N' - counts_i / T)
//                  (DeepSeek-V4 book ch. 2, section 3)
// Every sum runs in a fixed order in double precision, so results are deterministic.
#include "kernels.h"

namespace dsmoe {

namespace {
constexpr int kThreads = 512;

__device__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
  return t;  // valid in thread 0
}

__global__ void __launch_bounds__(kThreads) balance_losses_kernel(const float* __restrict__ f,
                                                                  const float* __restrict__ P, int N, int G,
                                                                  const int32_t* __restrict__ group_of,
                                                                  float alpha1, float alpha2, float* f_dev,
                                                                  float* P_dev, float* losses) {
  __shared__ double red[kThreads / 32];
  __shared__ double dev_prod[kThreads];
  double e = 0.0;
  for (int i = threadIdx.x; i < N; i += kThreads) e += static_cast<double>(f[i]) * P[i];
  const double se = block_sum(e, red);
  // device groups: group g accumulates its experts in ascending index order
  for (int g = threadIdx.x; g < kThreads; g += kThreads) dev_prod[g] = 0.0;
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += kThreads) {
    double fs = 0.0, ps = 0.0;
    int n = 0;
    for (int i = 0; i < N; ++i)
      if (group_of[i] == g) {
        fs += f[i];
        ps += P[i];
        ++n;
      }
    const double fm = n ? fs / n : 0.0;
    f_dev[g] = static_cast<float>(fm);
    P_dev[g] = static_cast<float>(ps);
    dev_prod[g] = fm * ps;
  }
  __syncthreads();
  double d = 0.0;
  for (int g = threadIdx.x; g < G; g += kThreads) d += dev_prod[g];
  const double sd = block_sum(d, red);
  if (threadIdx.x == 0) {
    losses[0] = static_cast<float>(alpha1 * se / N);
    losses[1] = static_cast<float>(alpha2 * sd);
  }
}

// one CTA per sequence: token counts per expert (exact) and the mean score per expert,
// then the sequence's sum_i f_i p_i
__global__ void __launch_bounds__(kThreads) sequence_stats_kernel(const int32_t* __restrict__ topk_idx,
                                                                  const float* __restrict__ scores, int seq_len,
                                                                  int N, int K, float* __restrict__ f_seq,
                                                                  float* __restrict__ p_seq,
                                                                  float* __restrict__ seq_terms) {
  __shared__ int32_t cnt[512];
  __shared__ double red[kThreads / 32];
  const int q = blockIdx.x;
  for (int i = threadIdx.x; i < N; i += kThreads) cnt[i] = 0;
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(q) * seq_len;
  for (int64_t j = threadIdx.x; j < static_cast<int64_t>(seq_len) * K; j += kThreads) {
    const int e = topk_idx[t0 * K + j];
    if (e >= 0 && e < N) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  double term = 0.0;
  for (int i = threadIdx.x; i < N; i += kThreads) {
    double ps = 0.0;
    for (int t = 0; t < seq_len; ++t) ps += scores[(t0 + t) * N + i];
    const double pm = ps / seq_len;
    const double fm = static_cast<double>(cnt[i]) / seq_len;
    f_seq[static_cast<int64_t>(q) * N + i] = static_cast<float>(fm);
    p_seq[static_cast<int64_t>(q) * N + i] = static_cast<float>(pm);
    term += fm * pm;
  }
  const double s = block_sum(term, red);
  if (threadIdx.x == 0) seq_terms[q] = static_cast<float>(s);
}

__global__ void __launch_bounds__(kThreads) sequence_loss_kernel(const float* __restrict__ seq_terms, int S,
                                                                 float beta, float* loss) {
  __shared__ double red[kThreads / 32];
  double v = 0.0;
  for (int q = threadIdx.x; q < S; q += kThreads) v += seq_terms[q];
  const double s = block_sum(v, red);
  if (threadIdx.x == 0) loss[0] = S ? static_cast<float>(beta * s / S) : 0.f;
}

__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int64_t T, int N, int K, float alpha,
                                   float* __restrict__ b) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N && T > 0)
    b[i] = static_cast<float>(b[i] + static_cast<double>(alpha) *
                                          (static_cast<double>(K) / N - static_cast<double>(counts[i]) / T));
}
}  // namespace

cudaError_t launch_balance_losses(const float* f, const float* P, int N, int G, const int32_t* group_of,
                                  float alpha1, float alpha2, float* f_dev, float* P_dev, float* losses,
                                  cudaStream_t s) {
  balance_losses_kernel<<<1, kThreads, 0, s>>>(f, P, N, G, group_of, alpha1, alpha2, f_dev, P_dev, losses);
  return cudaGetLastError();
}

cudaError_t launch_sequence_balance(const int32_t* topk_idx, const float* scores, int S, int seq_len, int N,
                                    int K, float beta, float* f_seq, float* p_seq, float* seq_terms, float* loss,
                                    cudaStream_t s) {
  if (S > 0) {
    sequence_stats_kernel<<<S, kThreads, 0, s>>>(topk_idx, scores, seq_len, N, K, f_seq, p_seq, seq_terms);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sequence_loss_kernel<<<1, kThreads, 0, s>>>(seq_terms, S, beta, loss);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(const int32_t* counts, int64_t T, int N, int K, float alpha, float* b,
                               cudaStream_t s) {
  bias_update_kernel<<<(N + 255) / 256, 256, 0, s>>>(counts, T, N, K, alpha, b);
  return cudaGetLastError();
}

}  // namespace dsmoe
