// router_sm100.cu -- router affinities on the 5th-generation tensor cores.
//
// Affinity l[t,i] = u_t . e_i ("MoE architecture: how DeepSeek achieves more",
// section 2). The router is a skinny contraction (N' outputs per token, K = d), so
// the work is split over (128-token tile, slice of K) pairs to keep every SM streaming:
// each pair accumulates its partial affinities of 128 tokens with all N' experts in
// TMEM (fp32, one or two chains of tcgen05.mma with N <= 256), fed by a TMA ring of
// x tiles (128x64) and router tiles (N'x64), and writes them to partial[slice][t][i].
// The select kernel (router.cu) adds the slices in a fixed order, then scores,
// selects and gates; a bias that enters the logits is added there.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace dsmoe {

namespace {
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMmaK = 16;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kMaxStages = 6;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr size_t kSmemLimit = 232448;

struct Layout {
  uint32_t b_bytes, stage_bytes, stages;
  uint32_t off_b, off_bars, off_misc, used;
};

__host__ __device__ inline Layout router_layout(int n_chunks, int nc) {
  Layout L;
  L.b_bytes = static_cast<uint32_t>(n_chunks) * nc * kBK * 2;
  L.stage_bytes = kABytes + L.b_bytes;
  const uint32_t fixed = 1024 + 256;
  uint32_t st = static_cast<uint32_t>((kSmemLimit - fixed) / L.stage_bytes);
  L.stages = st > kMaxStages ? kMaxStages : st;
  L.off_b = L.stages * kABytes;
  L.off_bars = L.off_b + L.stages * L.b_bytes;
  L.off_misc = L.off_bars + (2 * kMaxStages + 3) * 8;
  L.used = L.off_misc + 16;
  return L;
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
  uint64_t* empty = full + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.off_misc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + L.off_misc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  const int n_tok_tiles = (a.T + kBM - 1) / kBM;
  const int kb_total = a.d / kBK;
  const int kb_per = (kb_total + a.splits - 1) / a.splits;
  const int n_work = n_tok_tiles * a.splits;

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
      for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
        const int tile = w / a.splits, z = w % a.splits;
        const int kb0 = z * kb_per, kb1 = min(kb_total, kb0 + kb_per);
        for (int kb = kb0; kb < kb1; ++kb) {
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
      for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x, ++it) {
        const int z = w % a.splits;
        const int kb0 = z * kb_per, kb1 = min(kb_total, kb0 + kb_per);
        if (!mbar_wait_bounded(acc_empty, (it & 1) ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb) {
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
                          idesc, (kb > kb0 || k) ? 1u : 0u);
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
    // the thread of TMEM lane r writes token r's N' partial affinities (16-byte stores)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int ngroups = (N + 15) / 16;
    int it = 0;
    for (int w = blockIdx.x; w < n_work; w += gridDim.x, ++it) {
      const int tile = w / a.splits, z = w % a.splits;
      if (!mbar_wait_warp_sleepy(acc_full, it & 1, a.wait_limit_ns, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(a.status, kStatusTimeoutEpilogue);
        }
        break;
      }
      tc_fence_after();
      const int t = tile * kBM + r;
      const bool row_ok = t < a.T;
      float* dst = a.partial + (static_cast<int64_t>(z) * a.T + (row_ok ? t : 0)) * N;
      for (int g = 0; g < ngroups; ++g) {
        uint32_t v[16];
        tmem_ld16(tb + g * 16, v);
        tmem_wait_ld();
        if (row_ok) {
          if ((N & 3) == 0 && g * 16 + 16 <= N) {
            float4* d4 = reinterpret_cast<float4*>(dst + g * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                  __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (g * 16 + j < N) dst[g * 16 + j] = __uint_as_float(v[j]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < stages; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, drain_wait_limit(a.wait_limit_ns), never_flag))
            atomicOr(a.status, kStatusTimeoutDrain);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      if (!mbar_wait_bounded(drain, 0, drain_wait_limit(a.wait_limit_ns), never_flag))
        atomicOr(a.status, kStatusTimeoutDrain);
    }
  }
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

int router_tc_splits(int T, int d, int num_sms) {
  const int tiles = (T + kBM - 1) / kBM;
  int s = (2 * num_sms + tiles - 1) / tiles;  // about two (tile, slice) pairs per SM
  const int kb = d / kBK;
  if (s > kb) s = kb;
  if (s > kRouterMaxSplits) s = kRouterMaxSplits;
  if (s < 1) s = 1;
  // every slice must hold at least one K block: with ceil(kb/s) blocks per slice, only
  // ceil(kb / ceil(kb/s)) slices are non-empty
  const int per = (kb + s - 1) / s;
  return (kb + per - 1) / per;
}

cudaError_t launch_router_tc(const RouterTcArgs& a, int grid, cudaStream_t s) {
  const Layout L = router_layout(a.n_chunks, a.nc);
  const size_t smem = L.used + 1024;
  if (smem > kSmemLimit || L.stages < 2) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  router_tc_kernel<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dsmoe
