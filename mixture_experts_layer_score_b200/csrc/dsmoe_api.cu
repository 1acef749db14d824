// dsmoe_api.cu -- the C ABI of libdsmoe.so: configuration checks, the handle and its
// workspace, TMA tensor maps, and the launch sequence of one layer forward:
//
//   router logits -> scores / top-K' / gates (+ statistics partials) -> counts scan,
//   f_i, P_i, segment offsets -> slot permutation + row gather -> gate/up grouped GEMM
//   with SiLU*up -> down grouped GEMM -> gate-weighted combine + residual.
//
// Nothing here synchronises the device inside dsmoe_forward, and nothing allocates
// outside dsmoe_create.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <functional>
#include <mutex>
#include <string>

#include "dsmoe.h"
#include "kernels.h"
#include "role_clock.cuh"

#define DSMOE_EXPORT extern "C" __attribute__((visibility("default")))

using dsmoe::bf16;

namespace {

// Stages 0-6 run one after another on the caller's stream (marks 0..7 bracket them);
// the shared experts' two GEMMs (stage 7) run on the handle's side stream, concurrently
// with the routing stages, between marks 8 and 9.
constexpr int kNumStages = 8;
constexpr int kChainStages = 7;
constexpr int kNumMarks = kChainStages + 3;
const char* const kStageNames[kNumStages] = {"router", "select", "scan", "permute", "gemm_gate_up", "gemm_down",
                                             "combine", "shared_experts"};
constexpr int kSelectMaxBlocks = 1024;  // rows of the statistics partials
constexpr int kTimingSlots = 64;        // forwards whose stage events are kept
constexpr int kTcRouterMinTokens = 256; // below this the CUDA-core router spreads over more SMs
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
constexpr int kEpMaxGroups = 512;       // (source rank, local expert) groups of dsmoe_ep_experts

thread_local std::string g_last_error;

dsmoe_status fail(dsmoe_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define CUDA_TRY(expr)                                                                              \
  do {                                                                                              \
    cudaError_t e_ = (expr);                                                                        \
    if (e_ != cudaSuccess) return fail(DSMOE_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D bf16 map [outer, inner] (inner contiguous), 128-byte swizzle, box (64, box_outer).
bool map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map [experts, rows, inner], 128-byte swizzle, box (64, box_rows, 1).
bool map_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t experts, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {inner, rows, experts};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4D bf16 view (64, rows, cols / 64, experts) of an [experts, rows, cols] tensor whose
// cols are contiguous, 128-byte swizzle, box (64, 64, 4, 1): one copy lands 256 cols x 64
// rows as four MN-major atoms (the backward GEMMs' A operand).
bool map_4d_mn(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t experts) {
  auto enc = tensor_map_encoder();
  if (!enc || cols % 64) return false;
  cuuint64_t dims[4] = {64, rows, cols / 64, experts};
  cuuint64_t strides[3] = {cols * 2, 128, rows * cols * 2};
  cuuint32_t box[4] = {64, 64, 4, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 view (64, rows, cols / 64) of a [rows, cols] buffer (cols contiguous), 128-byte
// swizzle, box (64, 64, atoms): one copy lands 64 rows x 64*atoms columns as MN-major
// atoms (the weight-gradient GEMMs' operands, reduced over rows).
bool map_view_mn(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t atoms) {
  auto enc = tensor_map_encoder();
  if (!enc || cols % 64 || rows == 0) return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, 64, atoms};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D fp32 map (cols, rows, groups) of a [groups, rows, cols] tensor, 64-byte swizzle,
// box (16, 32, 1): the weight-gradient GEMM's bulk stores of 32-row x 16-column halves.
bool map_out_f32(CUtensorMap* m, float* ptr, uint64_t rows, uint64_t cols, uint64_t groups) {
  auto enc = tensor_map_encoder();
  if (!enc || cols % 32 || rows % 32 || groups == 0) return false;
  cuuint64_t dims[3] = {cols, rows, groups};
  cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
  cuuint32_t box[3] = {16, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceGuard {
  int prev = -1, want;
  bool ok = false;
  explicit DeviceGuard(int d) : want(d) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    ok = (prev == d) || cudaSetDevice(d) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0 && prev != want) cudaSetDevice(prev);
  }
};

struct Layout {
  size_t logits, counts_ws, cursor, offsets, P_part, slot_of, Xp, A1, A1s, Y, Hs, status, seq_terms;
  size_t x_stage[2], ids_stage[2], h_stage[2], topk_stage[2], gates_stage[2], counts_stage[2], f_stage[2],
      P_stage[2];  // two staging slots for the host entry points
  size_t total;
};

size_t up256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

Layout plan(const dsmoe_cfg& c) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes > 0 ? bytes : 1);
    return o;
  };
  const size_t T = static_cast<size_t>(c.max_tokens), N = c.n_routed, K = c.top_k, d = c.d_model, F = c.d_ff;
  const size_t S = T * K, KsFs = static_cast<size_t>(c.n_shared) * c.d_ff_shared;
  const bool hash = c.score == DSMOE_ROUTE_HASH;
  // router logits as split-K partial sums: up to kRouterMaxSplits slices for small
  // batches (CUDA-core router), T + kRouterTcExtraRows rows for the tensor-core router
  const size_t small_T = T < static_cast<size_t>(kTcRouterMinTokens) ? T : kTcRouterMinTokens - 1;
  size_t logit_floats = dsmoe::kRouterMaxSplits * small_T * N;
  if (T >= static_cast<size_t>(kTcRouterMinTokens))
    logit_floats = std::max(logit_floats, (T + static_cast<size_t>(dsmoe::kRouterTcExtraRows)) * N);
  L.logits = take(hash ? 0 : logit_floats * 4);
  L.counts_ws = take(N * 4);
  L.cursor = take(N * 4);
  L.offsets = take((std::max<size_t>(N, kEpMaxGroups) + 1) * 4);  // also the expert-parallel groups
  L.P_part = take(hash ? 0 : static_cast<size_t>(kSelectMaxBlocks) * N * 4);
  L.slot_of = take(S * 4);
  L.Xp = take(S * d * 2);
  L.A1 = take(S * F * 2);
  L.A1s = take(T * KsFs * 2);
  L.Y = take(S * d * 2);
  L.Hs = take(c.n_shared > 0 ? T * d * 4 : 0);
  L.status = take(4);
  L.seq_terms = take(T * 4);
  for (int i = 0; i < 2; ++i) {
    L.x_stage[i] = take(T * d * 2);
    L.ids_stage[i] = take(hash ? T * 4 : 0);
    L.h_stage[i] = take(T * d * 2);
    L.topk_stage[i] = take(S * 4);
    L.gates_stage[i] = take(S * 4);
    L.counts_stage[i] = take(N * 4);
    L.f_stage[i] = take(N * 4);
    L.P_stage[i] = take(N * 4);
  }
  L.total = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

void dsmoe::note_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

struct dsmoe_handle {
  dsmoe_cfg cfg;
  int device = 0;
  int num_sms = 148;
  int pair_clusters[2] = {0, 0};  // co-resident CTA pairs of the pair GEMM (down, gate/up)
  int32_t gemm_kernel = DSMOE_GEMM_SINGLE;
  int32_t mask_top = 0;  // selection variant: top-ranked experts masked before the choice
  int32_t k_active = 0;  // selection variant: experts kept per token (cfg.top_k by default)
  // expert range: the routed experts whose weights this handle applies ([0, N') by
  // default), whether h is an fp32 partial sum, and whether the residual and the
  // shared experts are added
  int32_t e_begin = 0, e_end = 0;
  bool partial = false, add_shared = true;
  uint64_t wait_ns = kDefaultWaitNs;
  char* ws = nullptr;
  Layout L;
  float* logits;
  int32_t *counts_ws, *cursor, *offsets, *slot_of;
  float* P_part;
  bf16 *Xp, *A1, *A1s, *Y;
  float* Hs;
  uint32_t* status;
  float* seq_terms;
  struct Stage {
    bf16 *x, *h;
    int32_t *ids, *topk, *counts;
    float *gates, *f, *P;
  } stage[2];
  // the pipelined host entry point: its copy stream and, per staging slot, the events
  // that order input copy -> forward -> output copy -> reuse of the slot
  cudaStream_t copy_stream = nullptr;    // input copies
  cudaStream_t copy_stream_out = nullptr;  // output copies (both directions run at once)
  cudaEvent_t ev_in[2] = {}, ev_out[2] = {}, ev_d2h[2] = {};
  int64_t async_calls = 0;
  // the shared experts' GEMMs depend on x alone: they run on this stream, forked from and
  // joined back into the caller's stream, while the routing stages run
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  CUtensorMap tm_a1, tm_a1s;
  // weight maps, cached per pointer: W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, W_router
  // (the gate/up maps serve both GEMM kernels), then W_down and Ws_down for the pair down GEMM
  static constexpr int kMaps = 9;
  const void* wkey[kMaps] = {};
  int wkey_n[kMaps] = {};  // experts each cached routed map spans
  CUtensorMap tm_w[kMaps];
  int rt_chunks = 1, rt_nc = 16;
  uint32_t rt_cols = 32;
  bool timing = false;
  int timed_forwards = 0;               // forwards recorded since timing was enabled
  cudaEvent_t ev[kTimingSlots][kNumMarks] = {};
  int64_t launches = 0;
  int32_t ep_T = -1;  // tokens of the last dsmoe_ep_route (its slot table is in the workspace)
  // training buffers (dsmoe_set_training): the forward's saved pre-activations a | b, and
  // the backward's da | db and per-slot / shared input gradients
  char* tr = nullptr;
  bf16 *AB = nullptr, *ABs = nullptr, *dAB = nullptr, *dABs = nullptr, *dXp = nullptr;
  float* dXs = nullptr;
  int32_t saved_T = -1;  // tokens of the last forward that saved a | b
  bool dab_ready = false;  // da | db of that forward computed (dsmoe_backward_experts)
};

// ========================================================================================
// configuration
// ========================================================================================
DSMOE_EXPORT int32_t dsmoe_abi_version(void) { return DSMOE_ABI_VERSION; }

DSMOE_EXPORT const char* dsmoe_status_string(dsmoe_status s) {
  switch (s) {
    case DSMOE_OK: return "ok";
    case DSMOE_ERR_INVALID_ARG: return "invalid argument";
    case DSMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case DSMOE_ERR_WORKSPACE: return "workspace too small or allocation failed";
    case DSMOE_ERR_CUDA: return "CUDA error";
    case DSMOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

DSMOE_EXPORT const char* dsmoe_last_error(void) { return g_last_error.c_str(); }

DSMOE_EXPORT dsmoe_status dsmoe_check_config(const dsmoe_cfg* c) {
  if (!c) return fail(DSMOE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->score < DSMOE_SCORE_SOFTMAX || c->score > DSMOE_ROUTE_HASH)
    return fail(DSMOE_ERR_INVALID_ARG, "score %d is not a dsmoe_score", c->score);
  if (c->bias_mode < DSMOE_BIAS_NONE || c->bias_mode > DSMOE_BIAS_IN_LOGITS)
    return fail(DSMOE_ERR_INVALID_ARG, "bias_mode %d is not a dsmoe_bias_mode", c->bias_mode);
  if (c->renormalize != 0 && c->renormalize != 1) return fail(DSMOE_ERR_INVALID_ARG, "renormalize must be 0 or 1");
  if (c->d_model <= 0 || c->n_routed <= 0 || c->top_k <= 0 || c->d_ff <= 0 || c->max_tokens <= 0)
    return fail(DSMOE_ERR_INVALID_ARG, "d_model, n_routed, top_k, d_ff and max_tokens must be positive");
  if (c->n_shared < 0 || (c->n_shared > 0 && c->d_ff_shared <= 0))
    return fail(DSMOE_ERR_INVALID_ARG, "n_shared must be >= 0 and d_ff_shared > 0 when it is not");
  if (c->top_k > c->n_routed) return fail(DSMOE_ERR_INVALID_ARG, "top_k %d exceeds n_routed %d", c->top_k, c->n_routed);
  if (c->score == DSMOE_ROUTE_HASH) {
    if (c->top_k != 1) return fail(DSMOE_ERR_INVALID_ARG, "hash routing picks one expert per token (top_k=1)");
    if (c->bias_mode != DSMOE_BIAS_NONE) return fail(DSMOE_ERR_INVALID_ARG, "hash routing takes no bias");
    if (c->hash_mult == 0) return fail(DSMOE_ERR_INVALID_ARG, "hash_mult must be non-zero");
    if (c->hash_mod > static_cast<uint32_t>(c->n_routed))
      return fail(DSMOE_ERR_INVALID_ARG, "hash_mod %u exceeds n_routed %d", c->hash_mod, c->n_routed);
  }
  if (c->d_model % 64 || c->d_ff % 64 || (c->n_shared > 0 && c->d_ff_shared % 64))
    return fail(DSMOE_ERR_UNSUPPORTED, "d_model, d_ff and d_ff_shared must be multiples of 64");
  if (c->n_routed > 512) return fail(DSMOE_ERR_UNSUPPORTED, "n_routed %d > 512", c->n_routed);
  if (c->top_k > 16) return fail(DSMOE_ERR_UNSUPPORTED, "top_k %d > 16", c->top_k);
  if (c->n_shared > 8) return fail(DSMOE_ERR_UNSUPPORTED, "n_shared %d > 8", c->n_shared);
  if (c->d_model > 32768 || c->d_ff > 32768 || c->d_ff_shared > 32768)
    return fail(DSMOE_ERR_UNSUPPORTED, "d_model / d_ff above 32768");
  if (static_cast<int64_t>(c->max_tokens) * c->top_k > (int64_t{1} << 30))
    return fail(DSMOE_ERR_UNSUPPORTED, "max_tokens * top_k above 2^30");
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_workspace_bytes(const dsmoe_cfg* cfg, size_t* bytes) {
  if (!bytes) return fail(DSMOE_ERR_INVALID_ARG, "bytes is NULL");
  const dsmoe_status st = dsmoe_check_config(cfg);
  if (st != DSMOE_OK) return st;
  *bytes = plan(*cfg).total;
  return DSMOE_OK;
}

// ========================================================================================
// handle
// ========================================================================================
static void release(dsmoe_handle* h) {
  if (!h) return;
  DeviceGuard g(h->device);
  for (auto& set : h->ev)
    for (auto& e : set)
      if (e) cudaEventDestroy(e);
  for (int i = 0; i < 2; ++i)
    for (cudaEvent_t e : {h->ev_in[i], h->ev_out[i], h->ev_d2h[i]})
      if (e) cudaEventDestroy(e);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  if (h->copy_stream_out) cudaStreamDestroy(h->copy_stream_out);
  if (h->side) cudaStreamDestroy(h->side);
  if (h->tr) cudaFree(h->tr);
  if (h->ws) cudaFree(h->ws);
  delete h;
}

DSMOE_EXPORT dsmoe_status dsmoe_create(const dsmoe_cfg* cfg, int32_t device, dsmoe_handle** out) {
  if (!out) return fail(DSMOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  dsmoe_status st = dsmoe_check_config(cfg);
  if (st != DSMOE_OK) return st;
  int ndev = 0;
  CUDA_TRY(cudaGetDeviceCount(&ndev));
  if (device < 0 || device >= ndev) return fail(DSMOE_ERR_INVALID_ARG, "device %d of %d", device, ndev);
  DeviceGuard g(device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", device);
  cudaDeviceProp prop;
  CUDA_TRY(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10 || prop.minor != 0)
    return fail(DSMOE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", device, prop.major,
                prop.minor);
  if (!tensor_map_encoder()) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");

  dsmoe_handle* h = new dsmoe_handle();
  h->cfg = *cfg;
  if (h->cfg.score == DSMOE_ROUTE_HASH && h->cfg.hash_mod == 0) h->cfg.hash_mod = h->cfg.n_routed;
  h->device = device;
  h->k_active = h->cfg.top_k;
  h->e_end = h->cfg.n_routed;
  h->num_sms = prop.multiProcessorCount;
  h->pair_clusters[0] = dsmoe::down_pair_max_clusters();
  h->pair_clusters[1] = dsmoe::gateup_pair_max_clusters();
  dsmoe::router_tc_shape(cfg->n_routed, &h->rt_chunks, &h->rt_nc, &h->rt_cols);
  h->L = plan(h->cfg);
  cudaError_t e = cudaMalloc(&h->ws, h->L.total);
  if (e != cudaSuccess) {
    h->ws = nullptr;
    release(h);
    return fail(DSMOE_ERR_WORKSPACE, "cudaMalloc(%zu) failed: %s", h->L.total, cudaGetErrorString(e));
  }
  char* w = h->ws;
  const Layout& L = h->L;
  h->logits = reinterpret_cast<float*>(w + L.logits);
  h->counts_ws = reinterpret_cast<int32_t*>(w + L.counts_ws);
  h->cursor = reinterpret_cast<int32_t*>(w + L.cursor);
  h->offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  h->P_part = reinterpret_cast<float*>(w + L.P_part);
  h->slot_of = reinterpret_cast<int32_t*>(w + L.slot_of);
  h->Xp = reinterpret_cast<bf16*>(w + L.Xp);
  h->A1 = reinterpret_cast<bf16*>(w + L.A1);
  h->A1s = reinterpret_cast<bf16*>(w + L.A1s);
  h->Y = reinterpret_cast<bf16*>(w + L.Y);
  h->Hs = reinterpret_cast<float*>(w + L.Hs);
  h->status = reinterpret_cast<uint32_t*>(w + L.status);
  h->seq_terms = reinterpret_cast<float*>(w + L.seq_terms);
  for (int i = 0; i < 2; ++i) {
    h->stage[i].x = reinterpret_cast<bf16*>(w + L.x_stage[i]);
    h->stage[i].ids = reinterpret_cast<int32_t*>(w + L.ids_stage[i]);
    h->stage[i].h = reinterpret_cast<bf16*>(w + L.h_stage[i]);
    h->stage[i].topk = reinterpret_cast<int32_t*>(w + L.topk_stage[i]);
    h->stage[i].gates = reinterpret_cast<float*>(w + L.gates_stage[i]);
    h->stage[i].counts = reinterpret_cast<int32_t*>(w + L.counts_stage[i]);
    h->stage[i].f = reinterpret_cast<float*>(w + L.f_stage[i]);
    h->stage[i].P = reinterpret_cast<float*>(w + L.P_stage[i]);
  }
  e = cudaMemset(h->ws, 0, h->L.total);
  if (e != cudaSuccess) {
    release(h);
    return fail(DSMOE_ERR_CUDA, "cudaMemset failed: %s", cudaGetErrorString(e));
  }
  const dsmoe_cfg& c = h->cfg;
  const uint64_t S = static_cast<uint64_t>(c.max_tokens) * c.top_k;
  const uint32_t t2 = dsmoe::kGemmTokenTile;  // the down projection's token tile
  bool ok = map_2d(&h->tm_a1, h->A1, c.d_ff, S, t2);
  if (c.n_shared > 0)
    ok = ok && map_2d(&h->tm_a1s, h->A1s, static_cast<uint64_t>(c.n_shared) * c.d_ff_shared, c.max_tokens, t2);
  else
    h->tm_a1s = h->tm_a1;
  if (!ok) {
    release(h);
    return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a workspace tensor map");
  }
  for (auto& set : h->ev)
    for (auto& ev : set) {
      e = cudaEventCreate(&ev);
      if (e != cudaSuccess) {
        release(h);
        return fail(DSMOE_ERR_CUDA, "cudaEventCreate failed: %s", cudaGetErrorString(e));
      }
    }
  for (int i = 0; i < 2 && e == cudaSuccess; ++i)
    for (cudaEvent_t* ev : {&h->ev_in[i], &h->ev_out[i], &h->ev_d2h[i]})
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_stream_out, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    release(h);
    return fail(DSMOE_ERR_CUDA, "event or stream creation failed: %s", cudaGetErrorString(e));
  }
  *out = h;
  return DSMOE_OK;
}

DSMOE_EXPORT void dsmoe_destroy(dsmoe_handle* h) {
  if (!h) return;
  {
    DeviceGuard g(h->device);
    cudaDeviceSynchronize();
  }
  release(h);
}

// ========================================================================================
// forward
// ========================================================================================
namespace {

struct FwdArgs {
  int32_t T;
  const void *x, *W_router, *W_gate, *W_up, *W_down, *Ws_gate, *Ws_up, *Ws_down;
  const int32_t* token_ids;
  const float* b;
  void* h;
  int32_t* topk_idx;
  float* gates;
  int32_t* counts;
  float *f, *P, *P_sum, *scores_dbg;
};

// The routing half's arguments (router inputs and routing outputs).
dsmoe_status check_route(dsmoe_handle* h, const FwdArgs& a) {
  const dsmoe_cfg& c = h->cfg;
  if (a.T < 0) return fail(DSMOE_ERR_INVALID_ARG, "T = %d is negative", a.T);
  if (a.T > c.max_tokens) return fail(DSMOE_ERR_WORKSPACE, "T = %d exceeds max_tokens = %d", a.T, c.max_tokens);
  if (!a.counts || !a.f || !a.P) return fail(DSMOE_ERR_INVALID_ARG, "counts, f and P are required");
  if (a.T == 0) return DSMOE_OK;
  const bool hash = c.score == DSMOE_ROUTE_HASH;
  if (!a.x || !a.topk_idx || !a.gates) return fail(DSMOE_ERR_INVALID_ARG, "x, topk_idx and gates are required");
  if (hash && !a.token_ids) return fail(DSMOE_ERR_INVALID_ARG, "hash routing needs token_ids");
  if (!hash && !a.W_router) return fail(DSMOE_ERR_INVALID_ARG, "W_router is required");
  if (c.bias_mode != DSMOE_BIAS_NONE && !a.b) return fail(DSMOE_ERR_INVALID_ARG, "bias b is required by bias_mode");
  if (!aligned16(a.x) || (a.W_router && !aligned16(a.W_router)))
    return fail(DSMOE_ERR_INVALID_ARG, "x and W_router must be 16-byte aligned");
  return DSMOE_OK;
}

dsmoe_status check_forward(dsmoe_handle* h, const FwdArgs& a) {
  const dsmoe_cfg& c = h->cfg;
  if (a.T < 0) return fail(DSMOE_ERR_INVALID_ARG, "T = %d is negative", a.T);
  if (a.T > c.max_tokens) return fail(DSMOE_ERR_WORKSPACE, "T = %d exceeds max_tokens = %d", a.T, c.max_tokens);
  if (!a.counts || !a.f || !a.P) return fail(DSMOE_ERR_INVALID_ARG, "counts, f and P are required");
  if (a.T == 0) return DSMOE_OK;
  const bool hash = c.score == DSMOE_ROUTE_HASH;
  if (!a.x || !a.h || !a.topk_idx || !a.gates || !a.W_gate || !a.W_up || !a.W_down)
    return fail(DSMOE_ERR_INVALID_ARG, "x, h, topk_idx, gates and the routed weights are required");
  if (hash && !a.token_ids) return fail(DSMOE_ERR_INVALID_ARG, "hash routing needs token_ids");
  if (!hash && !a.W_router) return fail(DSMOE_ERR_INVALID_ARG, "W_router is required");
  if (c.bias_mode != DSMOE_BIAS_NONE && !a.b) return fail(DSMOE_ERR_INVALID_ARG, "bias b is required by bias_mode");
  if (h->add_shared && c.n_shared > 0 && (!a.Ws_gate || !a.Ws_up || !a.Ws_down))
    return fail(DSMOE_ERR_INVALID_ARG, "shared expert weights are required (n_shared = %d)", c.n_shared);
  const void* must_align[] = {a.x, a.W_router, a.W_gate, a.W_up, a.W_down, a.Ws_gate, a.Ws_up, a.Ws_down, a.h};
  for (const void* p : must_align)
    if (p && !aligned16(p)) return fail(DSMOE_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
  return DSMOE_OK;
}

// Tensor maps of the weights, cached per pointer and expert count. The routed maps
// (0-2, 7-9) span n_local experts: the handle's expert range unless the caller says.
const CUtensorMap* weight_map(dsmoe_handle* h, int which, const void* ptr, bool* ok, int n_local = -1) {
  if (n_local < 0) n_local = h->e_end - h->e_begin;
  if (h->wkey[which] != ptr || h->wkey_n[which] != n_local) {
    const dsmoe_cfg& c = h->cfg;
    h->wkey_n[which] = n_local;
    bool r = false;
    switch (which) {
      case 0:
      case 1: r = map_3d(&h->tm_w[which], ptr, c.d_model, c.d_ff, n_local, 128); break;
      case 2: r = map_3d(&h->tm_w[which], ptr, c.d_ff, c.d_model, n_local, 256); break;
      case 3:
      case 4: r = map_3d(&h->tm_w[which], ptr, c.d_model, c.d_ff_shared, c.n_shared, 128); break;
      case 5: r = map_3d(&h->tm_w[which], ptr, c.d_ff_shared, c.d_model, c.n_shared, 256); break;
      case 6: r = map_2d(&h->tm_w[which], ptr, c.d_model, c.n_routed, static_cast<uint32_t>(h->rt_nc)); break;
      case 7: r = map_3d(&h->tm_w[which], ptr, c.d_ff, c.d_model, n_local, 128); break;
      case 8: r = map_3d(&h->tm_w[which], ptr, c.d_ff_shared, c.d_model, c.n_shared, 128); break;
    }
    if (!r) {
      h->wkey[which] = nullptr;
      *ok = false;
      return &h->tm_w[which];
    }
    h->wkey[which] = ptr;
  }
  return &h->tm_w[which];
}

int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// ---- stages of the forward, shared by dsmoe_forward and the expert-parallel entry points

// Router affinities, scores, top-K', gates and statistics partials (or hash routing) for
// a.T > 0 tokens. Writes the routing outputs and h->counts_ws; *sel_grid = rows of score
// partials (0 for hash routing).
dsmoe_status route_stage(dsmoe_handle* h, const FwdArgs& a, cudaStream_t s, int* sel_grid,
                         const std::function<cudaError_t(int)>& mark) {
  const dsmoe_cfg& c = h->cfg;
  const int T = a.T, N = c.n_routed, K = h->k_active, d = c.d_model;
  const bool hash = c.score == DSMOE_ROUTE_HASH;
  bool ok = true;
  CUDA_TRY(cudaMemsetAsync(h->counts_ws, 0, N * sizeof(int32_t), s));
  *sel_grid = 0;
  if (hash) {
    CUDA_TRY(dsmoe::launch_hash_route(a.token_ids, T, N, c.hash_mult, c.hash_mod, a.topk_idx, a.gates, h->counts_ws,
                                      h->status, s));
    h->launches += 1;
    CUDA_TRY(mark(1));
    return DSMOE_OK;
  }
  // router affinities as split-K partial sums: tensor cores for larger batches,
  // CUDA cores below kTcRouterMinTokens tokens; then scores, top-K', gates, partials
  int splits;
  if (T >= kTcRouterMinTokens) {
    CUtensorMap m_x_router;  // token rows of x in the router's 128-token tiles
    if (!map_2d(&m_x_router, a.x, d, T, 128))
      return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected the router's token map");
    dsmoe::RouterTcArgs ra;
    memset(&ra, 0, sizeof(ra));
    const CUtensorMap* m_wr = weight_map(h, 6, a.W_router, &ok);
    if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected the router tensor map");
    splits = dsmoe::router_tc_splits(T, d, h->num_sms);
    ra.tm_x = m_x_router;
    ra.tm_w = *m_wr;
    ra.T = T;
    ra.N = N;
    ra.d = d;
    ra.splits = splits;
    ra.n_chunks = h->rt_chunks;
    ra.nc = h->rt_nc;
    ra.tmem_cols = h->rt_cols;
    ra.partial = h->logits;
    ra.status = h->status;
    ra.wait_limit_ns = h->wait_ns;
    const int work = cdiv(T, 128) * splits;
    CUDA_TRY(dsmoe::launch_router_tc(ra, work < h->num_sms ? work : h->num_sms, s));
  } else {
    splits = dsmoe::router_logits_splits(T, N, d, h->num_sms);
    CUDA_TRY(dsmoe::launch_router_logits(static_cast<const bf16*>(a.x), static_cast<const bf16*>(a.W_router), T, N,
                                         d, splits, h->logits, s));
  }
  CUDA_TRY(mark(1));
  dsmoe::SelectArgs sa;
  sa.logits = h->logits;
  sa.splits = splits;
  sa.b = a.b;
  sa.T = T;
  sa.N = N;
  sa.K = K;
  sa.mask_top = h->mask_top;
  sa.score = c.score;
  sa.bias_select = c.bias_mode == DSMOE_BIAS_SELECT_ONLY;
  sa.bias_in_logits = c.bias_mode == DSMOE_BIAS_IN_LOGITS;
  sa.renormalize = c.renormalize;
  sa.topk_idx = a.topk_idx;
  sa.gates = a.gates;
  sa.counts = h->counts_ws;
  sa.P_part = h->P_part;
  sa.scores_dbg = a.scores_dbg;
  sa.status = h->status;
  // two blocks per SM: enough warps for the tokens, few partial rows for the scan
  *sel_grid = dsmoe::select_grid(T, h->num_sms / 2 > 0 ? h->num_sms / 2 : 1);
  CUDA_TRY(dsmoe::launch_select(sa, *sel_grid, s));
  h->launches += 2;
  return DSMOE_OK;
}

// Counts, f, P (and P_sum), the slot offsets of the experts in [e0, e1), and the
// permutation + gather of the token rows into h->Xp.
dsmoe_status scan_permute_stage(dsmoe_handle* h, const FwdArgs& a, cudaStream_t s, int sel_grid, int e0, int e1,
                                const std::function<cudaError_t(int)>& mark) {
  const dsmoe_cfg& c = h->cfg;
  const int T = a.T, N = c.n_routed, K = h->k_active, d = c.d_model;
  dsmoe::ScanArgs sc;
  sc.counts_ws = h->counts_ws;
  sc.P_part = c.score == DSMOE_ROUTE_HASH ? nullptr : h->P_part;
  sc.n_part = sel_grid;
  sc.N = N;
  sc.K = K;
  sc.T = T;
  sc.counts = a.counts;
  sc.f = a.f;
  sc.P = a.P;
  sc.P_sum = a.P_sum;
  sc.offsets = h->offsets;
  sc.cursor = h->cursor;
  sc.e_begin = e0;
  sc.e_end = e1;
  CUDA_TRY(dsmoe::launch_scan_stats(sc, s));
  h->launches += 1;
  CUDA_TRY(mark(3));
  CUDA_TRY(dsmoe::launch_permute_gather(static_cast<const bf16*>(a.x), a.topk_idx, h->offsets, h->cursor, T, K, N,
                                        e0, e1, d, h->slot_of, h->Xp, h->status, h->num_sms, s));
  h->launches += 1;
  return DSMOE_OK;
}

// The grouped GEMMs of one projection pair over `n_groups` routed groups (device offsets
// [n_groups + 1], rows of `rows_map`, weights expert_mod-mapped) and Ks shared experts on
// the T token rows of `x_map` (gate/up) / h->A1s (down). Gate/up writes A1 (routed) and
// A1s (shared); down writes Y_out (routed) and Hs = residual + shared outputs (fp32).
struct GemmPlan {
  const void* rows;                 // routed token rows (Xp or received rows), gate/up operand
  uint64_t rows_extent;             // rows addressable at `rows` ([rows_extent, d])
  const void* x;                    // [T, d] x rows of the shared groups
  const int32_t* offsets;
  int n_groups, expert_mod;
  int64_t routed_rows;              // rows the routed groups cover (tile bound)
  int T, Ks;
  const CUtensorMap *wg, *wu, *wd, *swg, *swu, *swd;
  const bf16* residual;             // x, added to the shared rows of the down GEMM
  bf16* Y_out;                      // [routed_rows, d] routed expert outputs
  bool save_ab = false;             // also store the pre-activations a | b (training)
};

dsmoe_status gemm_stage(dsmoe_handle* h, const GemmPlan& p, cudaStream_t s,
                        const std::function<cudaError_t(int)>& mark) {
  const dsmoe_cfg& c = h->cfg;
  const int d = c.d_model, F = c.d_ff, Fs = c.d_ff_shared, Ks = p.Ks, T = p.T;
  const bool pair = h->gemm_kernel == DSMOE_GEMM_PAIR;
  // ---- gate/up GEMM with SiLU(gate) * up
  {
    // token tile of this launch (the pair kernel stages 128 of its 256 token rows per CTA)
    const int tok = pair ? dsmoe::kGemmTokenTile
                         : dsmoe::gateup_token_tile(d, p.routed_rows + static_cast<int64_t>(T) * Ks, p.n_groups + Ks);
    CUtensorMap m_rows, m_x;
    bool ok = true;
    if (p.n_groups > 0) ok = map_2d(&m_rows, p.rows, d, p.rows_extent, tok);
    if (Ks > 0) ok = ok && map_2d(&m_x, p.x, d, T, tok);
    if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a token tensor map of the gate/up GEMM");
    dsmoe::GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.a_routed = p.n_groups > 0 ? m_rows : m_x;  // (a kind with no groups is never read)
    g.a_shared = Ks > 0 ? m_x : m_rows;
    g.b0_routed = *p.wg;
    g.b1_routed = *p.wu;
    g.b0_shared = *p.swg;
    g.b1_shared = *p.swu;
    g.offsets = p.offsets;
    g.n_routed = p.n_groups;
    g.expert_mod = p.expert_mod;
    g.n_shared_groups = Ks;
    g.m_shared = T;
    const int ftile = pair ? 256 : 128;  // features per gate/up tile
    g.n_tiles_routed = p.n_groups ? cdiv(F, ftile) : 0;
    g.n_tiles_shared = Ks ? cdiv(Fs, ftile) : 0;
    g.kb_routed = d / 64;
    g.kb_shared = d / 64;
    g.kb_per_b_expert_shared = d / 64;
    g.n_valid_routed = F;
    g.n_valid_shared = Fs;
    g.out_routed = h->A1;
    g.ld_routed = F;
    g.out_shared = h->A1s;
    g.ld_shared = static_cast<int64_t>(Ks) * Fs;
    g.shared_col_stride = Fs;
    g.save_ab_routed = p.save_ab ? h->AB : nullptr;
    g.save_ab_shared = p.save_ab ? h->ABs : nullptr;
    g.status = h->status;
    g.wait_limit_ns = h->wait_ns;
    const int64_t tt = pair ? dsmoe::kGemmPairTokenTile : tok;
    const int64_t bound = (cdiv(p.routed_rows, tt) + p.n_groups) * static_cast<int64_t>(g.n_tiles_routed) +
                          static_cast<int64_t>(Ks) * cdiv(T, tt) * g.n_tiles_shared;
    if (bound > 0) {
      if (pair) {
        const int clusters = static_cast<int>(bound < h->pair_clusters[1] ? bound : h->pair_clusters[1]);
        CUDA_TRY(dsmoe::launch_gateup_pair(g, clusters, s));
      } else {
        const int grid = static_cast<int>(bound < h->num_sms ? bound : h->num_sms);
        CUDA_TRY(dsmoe::launch_grouped_gemm(true, tok, g, grid, s));
      }
      h->launches += 1;
    }
  }
  CUDA_TRY(mark(5));
  // ---- down GEMM; the shared experts accumulate into one output row per token
  {
    dsmoe::GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.a_routed = h->tm_a1;
    g.a_shared = h->tm_a1s;
    g.b0_routed = *p.wd;
    g.b1_routed = *p.wd;
    g.b0_shared = *p.swd;
    g.b1_shared = *p.swd;
    g.offsets = p.offsets;
    g.n_routed = p.n_groups;
    g.expert_mod = p.expert_mod;
    g.n_shared_groups = Ks ? 1 : 0;
    g.m_shared = T;
    g.n_tiles_routed = p.n_groups ? cdiv(d, 256) : 0;
    g.n_tiles_shared = Ks ? cdiv(d, 256) : 0;
    g.kb_routed = F / 64;
    g.kb_shared = Ks ? Ks * Fs / 64 : 0;
    g.kb_per_b_expert_shared = Ks ? Fs / 64 : 1;
    g.n_valid_routed = d;
    g.n_valid_shared = d;
    g.out_routed = p.Y_out;
    g.ld_routed = d;
    g.out_shared = nullptr;
    g.out_shared_f32 = h->Hs;
    g.residual = p.residual;
    g.ld_shared = d;
    g.shared_col_stride = 0;
    g.status = h->status;
    g.wait_limit_ns = h->wait_ns;
    const int64_t tt = pair ? dsmoe::kGemmPairTokenTile : dsmoe::kGemmTokenTile;
    const int64_t bound = (cdiv(p.routed_rows, tt) + p.n_groups) * static_cast<int64_t>(g.n_tiles_routed) +
                          static_cast<int64_t>(g.n_shared_groups) * cdiv(T, tt) * g.n_tiles_shared;
    if (bound > 0) {
      if (pair) {
        const int clusters = static_cast<int>(bound < h->pair_clusters[0] ? bound : h->pair_clusters[0]);
        CUDA_TRY(dsmoe::launch_down_pair(g, clusters, s));
      } else {
        const int grid = static_cast<int>(bound < h->num_sms ? bound : h->num_sms);
        CUDA_TRY(dsmoe::launch_grouped_gemm(false, dsmoe::kGemmTokenTile, g, grid, s));
      }
      h->launches += 1;
    }
  }
  CUDA_TRY(mark(6));
  return DSMOE_OK;
}

// h = base + sum_k g Y[slot_of], base = Hs (Ks > 0), x (add_x) or 0; bf16 or fp32 out.
dsmoe_status combine_stage(dsmoe_handle* h, const FwdArgs& a, const bf16* Y, int Ks, bool add_x, bool partial,
                           cudaStream_t s) {
  dsmoe::CombineArgs ca;
  ca.x = static_cast<const bf16*>(a.x);
  ca.Hs = Ks ? h->Hs : nullptr;
  ca.add_x = add_x ? 1 : 0;
  ca.Y = Y;
  ca.slot_of = h->slot_of;
  ca.gates = a.gates;
  ca.T = a.T;
  ca.K = h->k_active;
  ca.d = h->cfg.d_model;
  ca.h = partial ? nullptr : static_cast<bf16*>(a.h);
  ca.h32 = partial ? static_cast<float*>(a.h) : nullptr;
  CUDA_TRY(dsmoe::launch_combine(ca, h->num_sms, s));
  h->launches += 1;
  return DSMOE_OK;
}

dsmoe_status zero_stats(const FwdArgs& a, int N, cudaStream_t s) {
  CUDA_TRY(cudaMemsetAsync(a.counts, 0, N * sizeof(int32_t), s));
  CUDA_TRY(cudaMemsetAsync(a.f, 0, N * sizeof(float), s));
  CUDA_TRY(cudaMemsetAsync(a.P, 0, N * sizeof(float), s));
  if (a.P_sum) CUDA_TRY(cudaMemsetAsync(a.P_sum, 0, N * sizeof(float), s));
  return DSMOE_OK;
}

#define STAGE_TRY(expr)                        \
  do {                                         \
    const dsmoe_status st_ = (expr);           \
    if (st_ != DSMOE_OK) return st_;           \
  } while (0)

dsmoe_status run_forward(dsmoe_handle* h, const FwdArgs& a, cudaStream_t s) {
  const dsmoe_cfg& c = h->cfg;
  const int T = a.T, N = c.n_routed, K = h->k_active;
  // shared experts (and the residual) only where this handle adds them
  const int Ks = h->add_shared ? c.n_shared : 0;
  const int e0 = h->e_begin, NL = h->e_end - h->e_begin;  // routed experts applied here
  const bool timing = h->timing && T > 0;
  cudaEvent_t* evs = h->ev[h->timed_forwards % kTimingSlots];
  // under stream capture the stage events become graph nodes that record on every replay
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (timing) CUDA_TRY(cudaStreamIsCapturing(s, &cap));
  const unsigned rec_flags = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  const std::function<cudaError_t(int)> mark = [&](int i) -> cudaError_t {
    return timing ? cudaEventRecordWithFlags(evs[i], s, rec_flags) : cudaSuccess;
  };

  if (T == 0) return zero_stats(a, N, s);

  // tensor maps that depend on the call's pointers
  bool ok = true;
  const bool pair = h->gemm_kernel == DSMOE_GEMM_PAIR;  // the down projection's weight box differs
  GemmPlan p;
  p.wg = weight_map(h, 0, a.W_gate, &ok);
  p.wu = weight_map(h, 1, a.W_up, &ok);
  p.wd = weight_map(h, pair ? 7 : 2, a.W_down, &ok);
  p.swg = Ks ? weight_map(h, 3, a.Ws_gate, &ok) : p.wg;
  p.swu = Ks ? weight_map(h, 4, a.Ws_up, &ok) : p.wu;
  p.swd = Ks ? weight_map(h, pair ? 8 : 5, a.Ws_down, &ok) : p.wd;
  if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map of this call");

  CUDA_TRY(mark(0));
  if (Ks > 0) {  // the side stream starts after everything the caller queued before this call
    CUDA_TRY(cudaEventRecord(h->ev_fork, s));
    CUDA_TRY(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
  }
  int sel_grid = 0;
  STAGE_TRY(route_stage(h, a, s, &sel_grid, mark));
  p.x = a.x;
  p.T = T;
  p.residual = static_cast<const bf16*>(a.x);
  p.save_ab = h->tr != nullptr;
  p.offsets = h->offsets + e0;
  p.expert_mod = 0;
  const std::function<cudaError_t(int)> no_mark = [](int) { return cudaSuccess; };
  if (Ks > 0) {
    // shared experts (gate/up into A1s, down into Hs with the residual), queued after the
    // router so that its CTAs are placed first; the permute's CTAs fit beside these GEMMs'
    if (timing) CUDA_TRY(cudaEventRecordWithFlags(evs[kChainStages + 1], h->side, rec_flags));
    GemmPlan sp = p;
    sp.rows = a.x;
    sp.rows_extent = static_cast<uint64_t>(T);
    sp.n_groups = 0;
    sp.routed_rows = 0;
    sp.Ks = Ks;
    sp.Y_out = nullptr;
    STAGE_TRY(gemm_stage(h, sp, h->side, no_mark));
    if (timing) CUDA_TRY(cudaEventRecordWithFlags(evs[kChainStages + 2], h->side, rec_flags));
    CUDA_TRY(cudaEventRecord(h->ev_join, h->side));
  }
  CUDA_TRY(mark(2));
  STAGE_TRY(scan_permute_stage(h, a, s, sel_grid, e0, e0 + NL, mark));
  CUDA_TRY(mark(4));
  p.rows = h->Xp;
  p.rows_extent = static_cast<uint64_t>(c.max_tokens) * c.top_k;
  p.n_groups = NL;
  p.routed_rows = static_cast<int64_t>(T) * K;
  p.Ks = 0;
  p.Y_out = h->Y;
  STAGE_TRY(gemm_stage(h, p, s, mark));
  if (Ks > 0) CUDA_TRY(cudaStreamWaitEvent(s, h->ev_join, 0));
  if (h->tr) {
    h->saved_T = T;
    h->dab_ready = false;
  }
  STAGE_TRY(combine_stage(h, a, h->Y, Ks, h->add_shared, h->partial, s));
  CUDA_TRY(mark(7));
  if (timing && Ks == 0) {  // no shared-expert stage: an empty interval
    CUDA_TRY(cudaEventRecordWithFlags(evs[kChainStages + 1], s, rec_flags));
    CUDA_TRY(cudaEventRecordWithFlags(evs[kChainStages + 2], s, rec_flags));
  }
  if (timing) h->timed_forwards += 1;
  return DSMOE_OK;
}

}  // namespace

DSMOE_EXPORT dsmoe_status dsmoe_forward(dsmoe_handle* h, int32_t T, const void* x, const int32_t* token_ids,
                                        const void* W_router, const float* b, const void* W_gate, const void* W_up,
                                        const void* W_down, const void* Ws_gate, const void* Ws_up,
                                        const void* Ws_down, void* h_out, int32_t* topk_idx, float* gates,
                                        int32_t* counts, float* f, float* P, float* P_sum, float* scores_dbg,
                                        void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  FwdArgs a{T, x, W_router, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, token_ids, b, h_out, topk_idx, gates,
            counts, f, P, P_sum, scores_dbg};
  dsmoe_status st = check_forward(h, a);
  if (st != DSMOE_OK) return st;
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  return run_forward(h, a, static_cast<cudaStream_t>(stream));
}

namespace {
struct HostArgs {
  int32_t T;
  const void *x_host, *W_router, *W_gate, *W_up, *W_down, *Ws_gate, *Ws_up, *Ws_down;
  const int32_t* token_ids_host;
  const float* b;
  void* h_host;
  int32_t* topk_idx_host;
  float* gates_host;
  int32_t* counts_host;
  float *f_host, *P_host;
};

dsmoe_status check_host(dsmoe_handle* h, const HostArgs& a) {
  const dsmoe_cfg& c = h->cfg;
  if (h->partial) return fail(DSMOE_ERR_UNSUPPORTED, "the host entry points run the whole layer only");
  if (a.T < 0) return fail(DSMOE_ERR_INVALID_ARG, "T = %d is negative", a.T);
  if (a.T > c.max_tokens) return fail(DSMOE_ERR_WORKSPACE, "T = %d exceeds max_tokens = %d", a.T, c.max_tokens);
  if (!a.counts_host || !a.f_host || !a.P_host) return fail(DSMOE_ERR_INVALID_ARG, "counts, f and P are required");
  if (a.T > 0 && (!a.x_host || !a.h_host || !a.topk_idx_host || !a.gates_host))
    return fail(DSMOE_ERR_INVALID_ARG, "x, h, topk_idx and gates are required");
  if (a.T > 0 && c.score == DSMOE_ROUTE_HASH && !a.token_ids_host)
    return fail(DSMOE_ERR_INVALID_ARG, "hash routing needs token_ids");
  return DSMOE_OK;
}

// One host forward through staging slot `slot`: input copies on `cin`, the forward on
// `s`, output copies on `cout` (all three the same stream for the synchronous entry).
dsmoe_status host_forward(dsmoe_handle* h, const HostArgs& a, int slot, cudaStream_t cin, cudaStream_t s,
                          cudaStream_t cout, bool pipelined) {
  const dsmoe_cfg& c = h->cfg;
  const int T = a.T;
  const bool hash = c.score == DSMOE_ROUTE_HASH;
  dsmoe_handle::Stage& st = h->stage[slot];
  const size_t xb = static_cast<size_t>(T) * c.d_model * 2, sb = static_cast<size_t>(T) * h->k_active * 4,
               nb = static_cast<size_t>(c.n_routed) * 4;
  // the slot's input buffer is free once the forward that last read it has finished
  if (pipelined) CUDA_TRY(cudaStreamWaitEvent(cin, h->ev_out[slot], 0));
  if (T > 0) {
    CUDA_TRY(cudaMemcpyAsync(st.x, a.x_host, xb, cudaMemcpyHostToDevice, cin));
    if (hash) CUDA_TRY(cudaMemcpyAsync(st.ids, a.token_ids_host, static_cast<size_t>(T) * 4, cudaMemcpyHostToDevice, cin));
  }
  if (pipelined) {
    CUDA_TRY(cudaEventRecord(h->ev_in[slot], cin));
    CUDA_TRY(cudaStreamWaitEvent(s, h->ev_in[slot], 0));
    CUDA_TRY(cudaStreamWaitEvent(s, h->ev_d2h[slot], 0));  // the slot's previous outputs have left
  }
  FwdArgs f{T, st.x, a.W_router, a.W_gate, a.W_up, a.W_down, a.Ws_gate, a.Ws_up, a.Ws_down,
            hash ? st.ids : nullptr, a.b, st.h, st.topk, st.gates, st.counts, st.f, st.P, nullptr, nullptr};
  dsmoe_status r = check_forward(h, f);
  if (r != DSMOE_OK) return r;
  r = run_forward(h, f, s);
  if (r != DSMOE_OK) return r;
  if (pipelined) {
    CUDA_TRY(cudaEventRecord(h->ev_out[slot], s));
    CUDA_TRY(cudaStreamWaitEvent(cout, h->ev_out[slot], 0));
  }
  if (T > 0) {
    CUDA_TRY(cudaMemcpyAsync(a.h_host, st.h, xb, cudaMemcpyDeviceToHost, cout));
    CUDA_TRY(cudaMemcpyAsync(a.topk_idx_host, st.topk, sb, cudaMemcpyDeviceToHost, cout));
    CUDA_TRY(cudaMemcpyAsync(a.gates_host, st.gates, sb, cudaMemcpyDeviceToHost, cout));
  }
  CUDA_TRY(cudaMemcpyAsync(a.counts_host, st.counts, nb, cudaMemcpyDeviceToHost, cout));
  CUDA_TRY(cudaMemcpyAsync(a.f_host, st.f, nb, cudaMemcpyDeviceToHost, cout));
  CUDA_TRY(cudaMemcpyAsync(a.P_host, st.P, nb, cudaMemcpyDeviceToHost, cout));
  if (pipelined) CUDA_TRY(cudaEventRecord(h->ev_d2h[slot], cout));
  return DSMOE_OK;
}
}  // namespace

DSMOE_EXPORT dsmoe_status dsmoe_forward_host(dsmoe_handle* h, int32_t T, const void* x_host,
                                             const int32_t* token_ids_host, const void* W_router, const float* b,
                                             const void* W_gate, const void* W_up, const void* W_down,
                                             const void* Ws_gate, const void* Ws_up, const void* Ws_down,
                                             void* h_host, int32_t* topk_idx_host, float* gates_host,
                                             int32_t* counts_host, float* f_host, float* P_host, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  HostArgs a{T, x_host, W_router, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, token_ids_host, b, h_host,
             topk_idx_host, gates_host, counts_host, f_host, P_host};
  STAGE_TRY(check_host(h, a));
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(cudaStreamSynchronize(h->copy_stream));  // no pipelined call still uses the staging
  CUDA_TRY(cudaStreamSynchronize(h->copy_stream_out));
  STAGE_TRY(host_forward(h, a, 0, s, s, s, false));
  CUDA_TRY(cudaStreamSynchronize(s));
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_forward_host_async(dsmoe_handle* h, int32_t T, const void* x_host,
                                                   const int32_t* token_ids_host, const void* W_router,
                                                   const float* b, const void* W_gate, const void* W_up,
                                                   const void* W_down, const void* Ws_gate, const void* Ws_up,
                                                   const void* Ws_down, void* h_host, int32_t* topk_idx_host,
                                                   float* gates_host, int32_t* counts_host, float* f_host,
                                                   float* P_host, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  HostArgs a{T, x_host, W_router, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, token_ids_host, b, h_host,
             topk_idx_host, gates_host, counts_host, f_host, P_host};
  STAGE_TRY(check_host(h, a));
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  const int slot = static_cast<int>(h->async_calls & 1);
  STAGE_TRY(host_forward(h, a, slot, h->copy_stream, static_cast<cudaStream_t>(stream), h->copy_stream_out, true));
  h->async_calls += 1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_host_join(dsmoe_handle* h, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < 2; ++i) CUDA_TRY(cudaStreamWaitEvent(s, h->ev_d2h[i], 0));
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_host_sync(dsmoe_handle* h) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  CUDA_TRY(cudaStreamSynchronize(h->copy_stream));
  CUDA_TRY(cudaStreamSynchronize(h->copy_stream_out));
  return DSMOE_OK;
}

// ========================================================================================
// expert parallelism with token dispatch (route -> exchange rows -> owners' experts ->
// exchange back -> combine); the exchanges are the caller's collectives
// ========================================================================================
DSMOE_EXPORT dsmoe_status dsmoe_ep_route(dsmoe_handle* h, int32_t T, const void* x, const int32_t* token_ids,
                                         const void* W_router, const float* b, int32_t* topk_idx, float* gates,
                                         int32_t* counts, float* f, float* P, float* P_sum, float* scores_dbg,
                                         int32_t world, int32_t* send_rows, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (world < 1 || world > c.n_routed) return fail(DSMOE_ERR_INVALID_ARG, "world = %d outside [1, N']", world);
  if (!send_rows) return fail(DSMOE_ERR_INVALID_ARG, "send_rows is required");
  FwdArgs a{T, x, W_router, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, token_ids, b, nullptr, topk_idx,
            gates, counts, f, P, P_sum, scores_dbg};
  const dsmoe_status st = check_route(h, a);
  if (st != DSMOE_OK) return st;
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const std::function<cudaError_t(int)> mark = [](int) { return cudaSuccess; };
  if (T == 0) {
    STAGE_TRY(zero_stats(a, c.n_routed, s));
    CUDA_TRY(cudaMemsetAsync(send_rows, 0, world * sizeof(int32_t), s));
    return DSMOE_OK;
  }
  int sel_grid = 0;
  STAGE_TRY(route_stage(h, a, s, &sel_grid, mark));
  STAGE_TRY(scan_permute_stage(h, a, s, sel_grid, 0, c.n_routed, mark));
  CUDA_TRY(dsmoe::launch_block_rows(h->offsets, c.n_routed, world, send_rows, s));
  h->launches += 1;
  h->ep_T = T;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_ep_experts(dsmoe_handle* h, int32_t n_src, int32_t e_begin, int32_t e_end,
                                           const int32_t* recv_counts, int64_t n_rows, const void* rows,
                                           const void* W_gate, const void* W_up, const void* W_down, void* Y,
                                           void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  const int n_local = e_end - e_begin;
  if (e_begin < 0 || n_local < 1 || e_end > c.n_routed)
    return fail(DSMOE_ERR_INVALID_ARG, "expert block [%d, %d) is not a non-empty part of [0, %d)", e_begin, e_end,
                c.n_routed);
  if (n_src < 1 || static_cast<int64_t>(n_src) * n_local > kEpMaxGroups)
    return fail(DSMOE_ERR_UNSUPPORTED, "n_src * local experts = %lld outside [1, %d]",
                static_cast<long long>(n_src) * n_local, kEpMaxGroups);
  if (n_rows < 0 || n_rows > static_cast<int64_t>(c.max_tokens) * c.top_k)
    return fail(DSMOE_ERR_WORKSPACE, "n_rows = %lld outside [0, max_tokens * top_k = %lld]",
                static_cast<long long>(n_rows), static_cast<long long>(c.max_tokens) * c.top_k);
  if (!recv_counts || (n_rows > 0 && (!rows || !W_gate || !W_up || !W_down || !Y)))
    return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  const void* must_align[] = {rows, W_gate, W_up, W_down, Y};
  for (const void* p : must_align)
    if (p && !aligned16(p)) return fail(DSMOE_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_rows == 0) return DSMOE_OK;
  const int groups = n_src * n_local;
  CUDA_TRY(dsmoe::launch_group_offsets(recv_counts, groups, h->offsets, h->status, s));
  h->launches += 1;
  bool ok = true;
  const bool pair = h->gemm_kernel == DSMOE_GEMM_PAIR;
  GemmPlan p;
  p.wg = weight_map(h, 0, W_gate, &ok, n_local);
  p.wu = weight_map(h, 1, W_up, &ok, n_local);
  p.wd = weight_map(h, pair ? 7 : 2, W_down, &ok, n_local);
  p.swg = p.wg;
  p.swu = p.wu;
  p.swd = p.wd;
  if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map of this call");
  p.rows = rows;
  p.rows_extent = static_cast<uint64_t>(n_rows);
  p.x = rows;
  p.offsets = h->offsets;
  p.n_groups = groups;
  p.expert_mod = n_local;
  p.routed_rows = n_rows;
  p.T = 0;
  p.Ks = 0;
  p.residual = nullptr;
  p.Y_out = static_cast<bf16*>(Y);
  const std::function<cudaError_t(int)> mark = [](int) { return cudaSuccess; };
  return gemm_stage(h, p, s, mark);
}

DSMOE_EXPORT dsmoe_status dsmoe_ep_combine(dsmoe_handle* h, int32_t T, const void* x, const void* Ws_gate,
                                           const void* Ws_up, const void* Ws_down, const float* gates, const void* Y,
                                           void* h_out, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (T != h->ep_T) return fail(DSMOE_ERR_INVALID_ARG, "T = %d differs from the last dsmoe_ep_route (%d)", T, h->ep_T);
  if (T == 0) return DSMOE_OK;
  if (!x || !gates || !Y || !h_out) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  const int Ks = c.n_shared;
  if (Ks > 0 && (!Ws_gate || !Ws_up || !Ws_down))
    return fail(DSMOE_ERR_INVALID_ARG, "shared expert weights are required (n_shared = %d)", Ks);
  const void* must_align[] = {x, Ws_gate, Ws_up, Ws_down, Y, h_out};
  for (const void* p : must_align)
    if (p && !aligned16(p)) return fail(DSMOE_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const std::function<cudaError_t(int)> mark = [](int) { return cudaSuccess; };
  if (Ks > 0) {
    bool ok = true;
    const bool pair = h->gemm_kernel == DSMOE_GEMM_PAIR;
    GemmPlan p;
    p.swg = weight_map(h, 3, Ws_gate, &ok);
    p.swu = weight_map(h, 4, Ws_up, &ok);
    p.swd = weight_map(h, pair ? 8 : 5, Ws_down, &ok);
    p.wg = p.swg;
    p.wu = p.swu;
    p.wd = p.swd;
    if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map of this call");
    p.rows = x;
    p.rows_extent = static_cast<uint64_t>(T);
    p.x = x;
    p.offsets = h->offsets;
    p.n_groups = 0;
    p.expert_mod = 0;
    p.routed_rows = 0;
    p.T = T;
    p.Ks = Ks;
    p.residual = static_cast<const bf16*>(x);
    p.Y_out = nullptr;
    STAGE_TRY(gemm_stage(h, p, s, mark));
  }
  FwdArgs a{T, x, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, h_out, nullptr,
            const_cast<float*>(gates), nullptr, nullptr, nullptr, nullptr, nullptr};
  return combine_stage(h, a, static_cast<const bf16*>(Y), Ks, true, false, s);
}

DSMOE_EXPORT dsmoe_status dsmoe_balance_stats(dsmoe_handle* h, int64_t T_total, const int32_t* counts,
                                              const float* P_sum, float* f, float* P, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (T_total < 0) return fail(DSMOE_ERR_INVALID_ARG, "T_total is negative");
  if (!counts || !P_sum || !f || !P) return fail(DSMOE_ERR_INVALID_ARG, "counts, P_sum, f and P are required");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  CUDA_TRY(dsmoe::launch_balance_stats(counts, P_sum, T_total, h->cfg.n_routed, h->k_active, f, P,
                                       static_cast<cudaStream_t>(stream)));
  h->launches += 1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_get_status(dsmoe_handle* h) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard g(h->device);
  CUDA_TRY(cudaDeviceSynchronize());
  uint32_t v = 0;
  CUDA_TRY(cudaMemcpy(&v, h->status, 4, cudaMemcpyDeviceToHost));
  CUDA_TRY(cudaMemset(h->status, 0, 4));
  if (v & (dsmoe::kStatusTimeoutProducer | dsmoe::kStatusTimeoutMma | dsmoe::kStatusTimeoutEpilogue |
           dsmoe::kStatusTimeoutDrain))
    return fail(DSMOE_ERR_DEVICE_TIMEOUT, "device status word 0x%x", v);
  if (v) return fail(DSMOE_ERR_INVALID_ARG, "device status word 0x%x (out-of-range index)", v);
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_set_wait_limit(dsmoe_handle* h, uint64_t ns) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (ns == 0) return fail(DSMOE_ERR_INVALID_ARG, "the wait limit must be at least 1 ns");
  h->wait_ns = ns;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_set_gemm_kernel(dsmoe_handle* h, int32_t kind) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (kind != DSMOE_GEMM_PAIR && kind != DSMOE_GEMM_SINGLE)
    return fail(DSMOE_ERR_INVALID_ARG, "unknown GEMM kernel kind %d", kind);
  if (kind == DSMOE_GEMM_PAIR && (h->pair_clusters[0] < 1 || h->pair_clusters[1] < 1))
    return fail(DSMOE_ERR_UNSUPPORTED, "the CTA-pair GEMM cannot be launched on this device");
  h->gemm_kernel = kind;
  return DSMOE_OK;
}

DSMOE_EXPORT int32_t dsmoe_get_gemm_kernel(dsmoe_handle* h) { return h ? h->gemm_kernel : -1; }

DSMOE_EXPORT dsmoe_status dsmoe_set_selection(dsmoe_handle* h, int32_t mask_top, int32_t k_active) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (k_active < 1 || k_active > c.top_k)
    return fail(DSMOE_ERR_INVALID_ARG, "k_active = %d is outside [1, top_k = %d]", k_active, c.top_k);
  if (mask_top < 0 || mask_top + k_active > c.n_routed)
    return fail(DSMOE_ERR_INVALID_ARG, "mask_top = %d with k_active = %d exceeds n_routed = %d", mask_top, k_active,
                c.n_routed);
  if (c.score == DSMOE_ROUTE_HASH && (mask_top != 0 || k_active != c.top_k))
    return fail(DSMOE_ERR_UNSUPPORTED, "hash routing has no ranking to mask or shorten");
  h->mask_top = mask_top;
  h->k_active = k_active;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_get_selection(dsmoe_handle* h, int32_t* mask_top, int32_t* k_active) {
  if (!h || !mask_top || !k_active) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  *mask_top = h->mask_top;
  *k_active = h->k_active;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_set_expert_range(dsmoe_handle* h, int32_t e_begin, int32_t e_end, int32_t flags) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (e_begin < 0 || e_end <= e_begin || e_end > c.n_routed)
    return fail(DSMOE_ERR_INVALID_ARG, "expert range [%d, %d) is not a non-empty part of [0, %d)", e_begin, e_end,
                c.n_routed);
  if (flags & ~(DSMOE_RANGE_PARTIAL | DSMOE_RANGE_ADD_SHARED))
    return fail(DSMOE_ERR_INVALID_ARG, "unknown expert-range flags 0x%x", flags);
  const bool partial = (flags & DSMOE_RANGE_PARTIAL) != 0, add_shared = (flags & DSMOE_RANGE_ADD_SHARED) != 0;
  if (!partial && (e_begin != 0 || e_end != c.n_routed || !add_shared))
    return fail(DSMOE_ERR_INVALID_ARG, "a part of the layer (an expert sub-range, or no residual and shared "
                "experts) needs DSMOE_RANGE_PARTIAL: its output is an fp32 partial sum");
  h->e_begin = e_begin;
  h->e_end = e_end;
  h->partial = partial;
  h->add_shared = add_shared;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_get_expert_range(dsmoe_handle* h, int32_t* e_begin, int32_t* e_end, int32_t* flags) {
  if (!h || !e_begin || !e_end || !flags) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  *e_begin = h->e_begin;
  *e_end = h->e_end;
  *flags = (h->partial ? DSMOE_RANGE_PARTIAL : 0) | (h->add_shared ? DSMOE_RANGE_ADD_SHARED : 0);
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_round_bf16(dsmoe_handle* h, int64_t n, const float* src, void* dst, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (n < 0 || n % 8) return fail(DSMOE_ERR_INVALID_ARG, "n = %lld is not a non-negative multiple of 8",
                                  static_cast<long long>(n));
  if (n > 0 && (!src || !dst)) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(src) || !aligned16(dst)) return fail(DSMOE_ERR_INVALID_ARG, "src and dst must be 16-byte aligned");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  CUDA_TRY(dsmoe::launch_round_bf16(src, static_cast<bf16*>(dst), n, h->num_sms, static_cast<cudaStream_t>(stream)));
  if (n > 0) h->launches += 1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_backward_gates(dsmoe_handle* h, int32_t T, const void* dh, const float* gates,
                                               float* dg, void* dY, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (T < 0 || T > h->cfg.max_tokens) return fail(DSMOE_ERR_INVALID_ARG, "T = %d outside [0, max_tokens]", T);
  if (T == 0) return DSMOE_OK;
  if (!dh || !gates || !dg || !dY) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(dh) || !aligned16(dY)) return fail(DSMOE_ERR_INVALID_ARG, "dh and dY must be 16-byte aligned");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  dsmoe::GateGradArgs a;
  a.dh = static_cast<const bf16*>(dh);
  a.Y = h->Y;
  a.slot_of = h->slot_of;
  a.gates = gates;
  a.T = T;
  a.K = h->k_active;
  a.d = h->cfg.d_model;
  a.dg = dg;
  a.dY = static_cast<bf16*>(dY);
  CUDA_TRY(dsmoe::launch_gate_grad(a, h->num_sms, static_cast<cudaStream_t>(stream)));
  h->launches += 1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_backward_router(dsmoe_handle* h, int32_t T, const void* x, const void* W_router,
                                                const int32_t* topk_idx, const float* gates, const float* scores,
                                                const float* dg, const float* f, float alpha, float* dlogits,
                                                float* dx, float* dW_router, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (c.score == DSMOE_ROUTE_HASH) return fail(DSMOE_ERR_UNSUPPORTED, "hash routing has no router to differentiate");
  if (T < 0 || T > c.max_tokens) return fail(DSMOE_ERR_INVALID_ARG, "T = %d outside [0, max_tokens]", T);
  if (!dW_router) return fail(DSMOE_ERR_INVALID_ARG, "dW_router is required");
  if (T > 0 && (!x || !W_router || !topk_idx || !gates || !scores || !dg || !dlogits || !dx))
    return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  if (alpha != 0.f && !f) return fail(DSMOE_ERR_INVALID_ARG, "a balance term (alpha != 0) needs f");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = c.n_routed, d = c.d_model;
  if (T == 0) {
    CUDA_TRY(cudaMemsetAsync(dW_router, 0, static_cast<size_t>(N) * d * sizeof(float), st));
    return DSMOE_OK;
  }
  dsmoe::RouterBwdArgs r;
  r.scores = scores;
  r.topk_idx = topk_idx;
  r.gates = gates;
  r.dg = dg;
  r.f = alpha != 0.f ? f : nullptr;
  r.alpha = alpha;
  r.T = T;
  r.N = N;
  r.K = h->k_active;
  r.score = c.score;
  r.renormalize = c.renormalize;
  r.dlogits = dlogits;
  r.status = h->status;
  CUDA_TRY(dsmoe::launch_router_backward(r, h->num_sms, st));
  // The two contractions on the tensor cores where the shapes allow: dlogits split into
  // bf16 parts hi + lo (what remains is below 2^-16 of each value), every product exact in
  // the fp32 accumulation. [hi | lo] goes to the router-logits workspace, which the
  // forward alone uses.
  const size_t hilo_bytes = static_cast<size_t>(T) * N * 4;
  const bool on_tensor_cores = N % 64 == 0 && d % 64 == 0 && T >= kTcRouterMinTokens && T >= 2 * N &&
                               hilo_bytes <= h->L.counts_ws - h->L.logits && aligned16(dlogits) && aligned16(x) &&
                               aligned16(W_router) && aligned16(dx) && aligned16(dW_router);
  if (on_tensor_cores) {
    bf16* hilo = reinterpret_cast<bf16*>(h->logits);
    CUDA_TRY(dsmoe::launch_hilo_split(dlogits, hilo, T, N, h->num_sms, st));
    // dW_router = hi^T x + lo^T x: the weight-gradient GEMM over all T rows with the two
    // parts as two groups; their fp32 results go to dx's memory (T x d >= 2 x N' x d
    // floats), which the dx GEMM overwrites afterwards, and are added in that order
    dsmoe::GemmDwArgs w;
    memset(&w, 0, sizeof(w));
    CUtensorMap m_hilo, m_w;
    bool ok = map_view_mn(&w.a_shared, hilo, T, 2 * static_cast<uint64_t>(N), 2) &&
              map_view_mn(&w.b_shared, x, T, d, 4) && map_out_f32(&w.out_map_shared, dx, N, d, 2) &&
              map_2d(&m_hilo, hilo, 2 * static_cast<uint64_t>(N), T, 128) && map_4d_mn(&m_w, W_router, N, d, 1);
    if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map of the router backward");
    w.a_routed = w.a_shared;
    w.b_routed = w.b_shared;
    w.a_atom_step_shared = N / 64;
    w.offsets = h->offsets;
    w.n_routed = 0;
    w.n_shared = 2;
    w.T = T;
    w.m_tiles_shared = cdiv(N, 128);
    w.n_tiles_shared = cdiv(d, 256);
    w.m_shared = N;
    w.n_shared_cols = d;
    w.status = h->status;
    w.wait_limit_ns = h->wait_ns;
    CUDA_TRY(dsmoe::launch_grouped_dw(w, h->num_sms, st));
    CUDA_TRY(dsmoe::launch_split_sum(dx, 2, N, d, d, dW_router, st));
    // dx = dl W_router: the input-gradient GEMM (weights read MN-major) with W_router as
    // both halves of one dense group's K loop over [hi | lo], fp32 rows
    dsmoe::GemmBwdArgs b;
    memset(&b, 0, sizeof(b));
    dsmoe::GemmArgs& g = b.g;
    g.a_routed = g.a_shared = m_hilo;
    g.b0_routed = g.b1_routed = g.b0_shared = g.b1_shared = m_w;
    g.offsets = h->offsets;
    g.n_routed = 0;
    g.n_shared_groups = 1;
    g.m_shared = T;
    g.n_tiles_routed = cdiv(d, 256);
    g.n_tiles_shared = cdiv(d, 256);
    g.kb_routed = g.kb_shared = 2 * N / 64;
    g.n_valid_routed = g.n_valid_shared = d;
    g.status = h->status;
    g.wait_limit_ns = h->wait_ns;
    b.kb_half_routed = b.kb_half_shared = N / 64;
    b.dx_shared = dx;
    b.ld_dx = d;
    const int64_t tiles = cdiv(T, 128) * static_cast<int64_t>(g.n_tiles_shared);
    CUDA_TRY(dsmoe::launch_grouped_gemm_bwd(dsmoe::kBwdDX, b, static_cast<int>(std::min<int64_t>(tiles, h->num_sms)),
                                            st));
    h->launches += 5;
    return DSMOE_OK;
  }
  dsmoe::GemmF32Args a;
  memset(&a, 0, sizeof(a));
  // dW_router = dlogits^T x  (M = N', K = T, N = d). Few output tiles and a long K: the K
  // range is split so that about two blocks per SM work; the partial sums go to dx's
  // memory (T x d >= splits x N' x d floats), which the next GEMM then overwrites.
  a.A = dlogits;
  a.a_sm = 1;
  a.a_sk = N;
  a.B = static_cast<const bf16*>(x);
  a.ldb = d;
  a.C = dW_router;
  a.ldc = d;
  a.M = N;
  a.N = d;
  a.K = T;
  {
    const int64_t tiles = static_cast<int64_t>(cdiv(N, 128)) * cdiv(d, 128);  // 128 x 128 output tiles
    int64_t splits = (2 * h->num_sms + tiles - 1) / tiles;
    splits = std::min<int64_t>(splits, std::min<int64_t>(32, T / 256));  // slices of >= 256 tokens
    splits = std::min<int64_t>(splits, T / N);                           // partials fit in dx
    a.splits = static_cast<int>(std::max<int64_t>(splits, 1));
    a.partial = a.splits > 1 ? dx : nullptr;
  }
  CUDA_TRY(dsmoe::launch_gemm_f32_bf16(a, st));
  // dx = dlogits W_router  (M = T, K = N', N = d)
  memset(&a, 0, sizeof(a));
  a.A = dlogits;
  a.a_sm = N;
  a.a_sk = 1;
  a.B = static_cast<const bf16*>(W_router);
  a.ldb = d;
  a.C = dx;
  a.ldc = d;
  a.M = T;
  a.N = d;
  a.K = N;
  a.splits = 1;
  CUDA_TRY(dsmoe::launch_gemm_f32_bf16(a, st));
  h->launches += 3;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_set_training(dsmoe_handle* h, int32_t enable) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  if (!enable) {
    if (h->tr) {
      CUDA_TRY(cudaDeviceSynchronize());
      CUDA_TRY(cudaFree(h->tr));
    }
    h->tr = nullptr;
    h->AB = h->ABs = h->dAB = h->dABs = h->dXp = nullptr;
    h->dXs = nullptr;
    h->saved_T = -1;
    return DSMOE_OK;
  }
  if (h->tr) return DSMOE_OK;
  const dsmoe_cfg& c = h->cfg;
  const size_t T = c.max_tokens, S = T * c.top_k, F = c.d_ff, d = c.d_model;
  const size_t KsFs = static_cast<size_t>(c.n_shared) * c.d_ff_shared;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes > 0 ? bytes : 1);
    return o;
  };
  const size_t oAB = take(S * 2 * F * 2), oABs = take(T * 2 * KsFs * 2), odAB = take(S * 2 * F * 2),
               odABs = take(T * 2 * KsFs * 2), odXp = take(S * d * 2), odXs = take(c.n_shared ? T * d * 4 : 0);
  char* p = nullptr;
  const cudaError_t e = cudaMalloc(&p, off);
  if (e != cudaSuccess) return fail(DSMOE_ERR_WORKSPACE, "cudaMalloc(%zu) of the training buffers failed: %s", off,
                                    cudaGetErrorString(e));
  h->tr = p;
  h->AB = reinterpret_cast<bf16*>(p + oAB);
  h->ABs = reinterpret_cast<bf16*>(p + oABs);
  h->dAB = reinterpret_cast<bf16*>(p + odAB);
  h->dABs = reinterpret_cast<bf16*>(p + odABs);
  h->dXp = reinterpret_cast<bf16*>(p + odXp);
  h->dXs = reinterpret_cast<float*>(p + odXs);
  h->saved_T = -1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_backward_experts(dsmoe_handle* h, int32_t T, const void* dh, const void* dY,
                                                 const void* W_gate, const void* W_up, const void* W_down,
                                                 const void* Ws_gate, const void* Ws_up, const void* Ws_down,
                                                 const float* dx_add, float* dx, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (!h->tr) return fail(DSMOE_ERR_INVALID_ARG, "training buffers are not enabled (dsmoe_set_training)");
  if (T != h->saved_T || T <= 0)
    return fail(DSMOE_ERR_INVALID_ARG, "T = %d is not the token count of the last training forward (%d)", T,
                h->saved_T);
  const int Ks = h->add_shared ? c.n_shared : 0;
  if (!dh || !dY || !W_gate || !W_up || !W_down || !dx || (Ks && (!Ws_gate || !Ws_up || !Ws_down)))
    return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  const void* must_align[] = {dh, dY, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, dx, dx_add};
  for (const void* q : must_align)
    if (q && !aligned16(q)) return fail(DSMOE_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", q);
  DeviceGuard gd(h->device);
  if (!gd.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = c.d_model, F = c.d_ff, Fs = c.d_ff_shared, K = h->k_active;
  const int NL = h->e_end - h->e_begin;
  const int64_t S = static_cast<int64_t>(T) * K;
  CUtensorMap m_dY, m_dh, m_dAB, m_dABs, m_wd, m_wg, m_wu, m_swd, m_swg, m_swu;
  bool ok = map_2d(&m_dY, dY, d, S, 128) && map_2d(&m_dh, dh, d, T, 128) &&
            map_2d(&m_dAB, h->dAB, 2 * F, S, 128) && map_4d_mn(&m_wd, W_down, d, F, NL) &&
            map_4d_mn(&m_wg, W_gate, F, d, NL) && map_4d_mn(&m_wu, W_up, F, d, NL);
  if (Ks)
    ok = ok && map_2d(&m_dABs, h->dABs, 2 * static_cast<uint64_t>(Ks) * Fs, T, 128) &&
         map_4d_mn(&m_swd, Ws_down, d, Fs, Ks) && map_4d_mn(&m_swg, Ws_gate, Fs, d, Ks) &&
         map_4d_mn(&m_swu, Ws_up, Fs, d, Ks);
  else
    m_dABs = m_dAB, m_swd = m_wd, m_swg = m_wg, m_swu = m_wu;
  if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map of the backward");
  auto grid_for = [&](const dsmoe::GemmArgs& g) {
    const int64_t bound = (cdiv(S, 128) + NL) * static_cast<int64_t>(g.n_tiles_routed) +
                          static_cast<int64_t>(g.n_shared_groups) * cdiv(T, 128) * g.n_tiles_shared;
    return static_cast<int>(bound < h->num_sms ? bound : h->num_sms);
  };
  // da | db from dy (routed: dY per slot; shared: dh) and W_down
  {
    dsmoe::GemmBwdArgs b;
    memset(&b, 0, sizeof(b));
    dsmoe::GemmArgs& g = b.g;
    g.a_routed = m_dY;
    g.a_shared = m_dh;
    g.b0_routed = g.b1_routed = m_wd;
    g.b0_shared = g.b1_shared = m_swd;
    g.offsets = h->offsets + h->e_begin;
    g.n_routed = NL;
    g.n_shared_groups = Ks;
    g.m_shared = T;
    g.n_tiles_routed = cdiv(F, 256);
    g.n_tiles_shared = Ks ? cdiv(Fs, 256) : 0;
    g.kb_routed = d / 64;
    g.kb_shared = d / 64;
    g.n_valid_routed = F;
    g.n_valid_shared = Fs;
    g.status = h->status;
    g.wait_limit_ns = h->wait_ns;
    b.ab_routed = h->AB;
    b.ab_shared = h->ABs;
    b.dab_routed = h->dAB;
    b.dab_shared = h->dABs;
    b.ld_ab_routed = 2 * static_cast<int64_t>(F);
    b.ld_ab_shared = 2 * static_cast<int64_t>(Ks) * Fs;
    b.width_routed = F;
    b.width_shared = Fs;
    CUDA_TRY(dsmoe::launch_grouped_gemm_bwd(dsmoe::kBwdDM, b, grid_for(g), s));
  }
  // input gradients from da | db and W_gate, W_up (the shared experts summed in one group)
  {
    dsmoe::GemmBwdArgs b;
    memset(&b, 0, sizeof(b));
    dsmoe::GemmArgs& g = b.g;
    g.a_routed = m_dAB;
    g.a_shared = m_dABs;
    g.b0_routed = m_wg;
    g.b1_routed = m_wu;
    g.b0_shared = m_swg;
    g.b1_shared = m_swu;
    g.offsets = h->offsets + h->e_begin;
    g.n_routed = NL;
    g.n_shared_groups = Ks ? 1 : 0;
    g.m_shared = T;
    g.n_tiles_routed = cdiv(d, 256);
    g.n_tiles_shared = Ks ? cdiv(d, 256) : 0;
    g.kb_routed = 2 * F / 64;
    g.kb_shared = Ks ? 2 * Ks * Fs / 64 : 0;
    g.n_valid_routed = d;
    g.n_valid_shared = d;
    g.status = h->status;
    g.wait_limit_ns = h->wait_ns;
    b.kb_half_routed = F / 64;
    b.kb_half_shared = Fs / 64;
    b.dx_routed = h->dXp;
    b.dx_shared = h->dXs;
    b.ld_dx = d;
    CUDA_TRY(dsmoe::launch_grouped_gemm_bwd(dsmoe::kBwdDX, b, grid_for(g), s));
  }
  CUDA_TRY(dsmoe::launch_dx_combine(static_cast<const bf16*>(dh), Ks ? h->dXs : nullptr, dx_add, h->dXp, h->slot_of,
                                    T, K, d, dx, h->num_sms, s));
  h->launches += 3;
  h->dab_ready = true;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_backward_weights(dsmoe_handle* h, int32_t T, const void* dh, const void* dY,
                                                 const void* x, float* dW_gate, float* dW_up, float* dW_down,
                                                 float* dWs_gate, float* dWs_up, float* dWs_down, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  const dsmoe_cfg& c = h->cfg;
  if (!h->tr) return fail(DSMOE_ERR_INVALID_ARG, "training buffers are not enabled (dsmoe_set_training)");
  if (T != h->saved_T || T <= 0 || !h->dab_ready)
    return fail(DSMOE_ERR_INVALID_ARG,
                "call after dsmoe_backward_experts for the last training forward (T = %d, forward T = %d)", T,
                h->saved_T);
  const int Ks = h->add_shared ? c.n_shared : 0;
  if (!dh || !dY || !x || !dW_gate || !dW_up || !dW_down || (Ks && (!dWs_gate || !dWs_up || !dWs_down)))
    return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  const void* must_align[] = {dh, dY, x, dW_gate, dW_up, dW_down, dWs_gate, dWs_up, dWs_down};
  for (const void* q : must_align)
    if (q && !aligned16(q)) return fail(DSMOE_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", q);
  DeviceGuard gd(h->device);
  if (!gd.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = c.d_model, F = c.d_ff, Fs = c.d_ff_shared;
  const int NL = h->e_end - h->e_begin;
  // operand views: routed rows in slot order (the T K' rows this forward wrote; the
  // copies read zeros past them), shared rows = the T tokens
  const uint64_t S = static_cast<uint64_t>(T) * h->k_active, KsFs = static_cast<uint64_t>(Ks) * Fs;
  CUtensorMap v_dY, v_A1, v_dAB, v_Xp, v_dh, v_A1s, v_dABs, v_x;
  bool ok = map_view_mn(&v_dY, dY, S, d, 2) && map_view_mn(&v_A1, h->A1, S, F, 4) &&
            map_view_mn(&v_dAB, h->dAB, S, 2 * static_cast<uint64_t>(F), 2) && map_view_mn(&v_Xp, h->Xp, S, d, 4);
  if (Ks)
    ok = ok && map_view_mn(&v_dh, dh, T, d, 2) && map_view_mn(&v_A1s, h->A1s, T, KsFs, 4) &&
         map_view_mn(&v_dABs, h->dABs, T, 2 * KsFs, 2) && map_view_mn(&v_x, x, T, d, 4);
  if (!ok) return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map of the weight gradients");
  auto plan = [&](dsmoe::GemmDwArgs& g, int M, int N, int Ms, int Ns) {
    memset(&g, 0, sizeof(g));
    g.offsets = h->offsets + h->e_begin;
    g.n_routed = NL;
    g.n_shared = Ks;
    g.T = T;
    g.m_routed = M;
    g.n_routed_cols = N;
    g.m_shared = Ms;
    g.n_shared_cols = Ns;
    g.m_tiles_routed = cdiv(M, 128);
    g.n_tiles_routed = cdiv(N, 256);
    g.m_tiles_shared = Ks ? cdiv(Ms, 128) : 0;
    g.n_tiles_shared = Ks ? cdiv(Ns, 256) : 0;
    g.status = h->status;
    g.wait_limit_ns = h->wait_ns;
  };
  // outputs: routed [NL, M, N], shared [Ks, Ms, Ns]
  auto outputs = [&](dsmoe::GemmDwArgs& g, float* routed, float* shared) {
    bool m_ok = NL == 0 || map_out_f32(&g.out_map_routed, routed, g.m_routed, g.n_routed_cols, NL);
    if (Ks) m_ok = m_ok && map_out_f32(&g.out_map_shared, shared, g.m_shared, g.n_shared_cols, Ks);
    return m_ok;
  };
  // dW_down[e] = sum_r dy_r m_r^T: A = dY (d columns), B = A1 (F columns)
  dsmoe::GemmDwArgs g;
  plan(g, d, F, d, Fs);
  g.a_routed = v_dY;
  g.b_routed = v_A1;
  g.a_shared = Ks ? v_dh : v_dY;
  g.b_shared = Ks ? v_A1s : v_A1;
  g.b_atom_step_shared = Fs / 64;
  if (!outputs(g, dW_down, dWs_down))
    return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a weight-gradient output map");
  CUDA_TRY(dsmoe::launch_grouped_dw(g, h->num_sms, s));
  // dW_gate[e] = sum_r da_r u_r^T and dW_up[e] = sum_r db_r u_r^T: A = da | db, B = Xp (x)
  for (int up = 0; up < 2; ++up) {
    plan(g, F, d, Fs, d);
    g.a_routed = v_dAB;
    g.b_routed = v_Xp;
    g.a_shared = Ks ? v_dABs : v_dAB;
    g.b_shared = Ks ? v_x : v_Xp;
    g.a_atom0_routed = up ? F / 64 : 0;
    g.a_atom0_shared = up ? Fs / 64 : 0;
    g.a_atom_step_shared = 2 * Fs / 64;
    if (!outputs(g, up ? dW_up : dW_gate, up ? dWs_up : dWs_gate))
      return fail(DSMOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a weight-gradient output map");
    CUDA_TRY(dsmoe::launch_grouped_dw(g, h->num_sms, s));
  }
  h->launches += 3;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_set_timing(dsmoe_handle* h, int32_t enable) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  h->timing = enable != 0;
  h->timed_forwards = 0;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_stage_times(dsmoe_handle* h, float* ms, int32_t max_n, int32_t* n) {
  if (!h || !ms || !n) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  *n = 0;
  if (h->timed_forwards == 0) return fail(DSMOE_ERR_INVALID_ARG, "no timed forward recorded (enable timing first)");
  DeviceGuard g(h->device);
  const int kept = h->timed_forwards < kTimingSlots ? h->timed_forwards : kTimingSlots;
  const int cnt = max_n < kNumStages ? max_n : kNumStages;
  for (int i = 0; i < cnt; ++i) ms[i] = 0.f;
  for (int f = 0; f < kept; ++f) {
    cudaEvent_t* evs = h->ev[(h->timed_forwards - 1 - f) % kTimingSlots];
    CUDA_TRY(cudaEventSynchronize(evs[kChainStages]));
    CUDA_TRY(cudaEventSynchronize(evs[kChainStages + 2]));
    for (int i = 0; i < cnt; ++i) {
      // chain stages: consecutive marks; the shared experts: their own pair of marks
      const int m0 = i < kChainStages ? i : kChainStages + 1;
      float v = 0.f;
      CUDA_TRY(cudaEventElapsedTime(&v, evs[m0], evs[m0 + 1]));
      ms[i] += v / kept;
    }
  }
  *n = cnt;
  return DSMOE_OK;
}

DSMOE_EXPORT const char* dsmoe_stage_name(int32_t i) {
  return (i >= 0 && i < kNumStages) ? kStageNames[i] : nullptr;
}

DSMOE_EXPORT dsmoe_status dsmoe_gemm_role_cycles(uint64_t* out, int32_t n) {
  if (!out || n < dsmoe::kRoleCounters)
    return fail(DSMOE_ERR_INVALID_ARG, "a buffer of %d counters is required", dsmoe::kRoleCounters);
  cudaError_t e = cudaSuccess;
  if (!dsmoe::read_role_cycles(reinterpret_cast<unsigned long long*>(out), &e))
    return fail(DSMOE_ERR_UNSUPPORTED, "this library was built without the role cycle counters");
  if (e != cudaSuccess) return fail(DSMOE_ERR_CUDA, "reading the role counters failed: %s", cudaGetErrorString(e));
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_launch_count(dsmoe_handle* h, int64_t* n) {
  if (!h || !n) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  *n = h->launches;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_workspace_tensor(dsmoe_handle* h, const char* name, void** ptr, int64_t* rows,
                                                 int64_t* cols) {
  if (!h || !name || !ptr || !rows || !cols) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  const dsmoe_cfg& c = h->cfg;
  const int64_t T = c.max_tokens, S = T * c.top_k;
  const bool hash = c.score == DSMOE_ROUTE_HASH;
  struct Entry {
    const char* n;
    void* p;
    int64_t r, k;
    bool present;
  } table[] = {
      {"logits", h->logits, T, c.n_routed, !hash},
      {"offsets", h->offsets, 1, c.n_routed + 1, true},
      {"slot_of", h->slot_of, T, h->k_active, true},
      {"Xp", h->Xp, S, c.d_model, true},
      {"A1", h->A1, S, c.d_ff, true},
      {"A1s", h->A1s, T, static_cast<int64_t>(c.n_shared) * c.d_ff_shared, c.n_shared > 0},
      {"Y", h->Y, S, c.d_model, true},
      {"Hs", h->Hs, T, c.d_model, c.n_shared > 0},
      {"AB", h->AB, S, 2 * static_cast<int64_t>(c.d_ff), h->tr != nullptr},
      {"dAB", h->dAB, S, 2 * static_cast<int64_t>(c.d_ff), h->tr != nullptr},
      {"ABs", h->ABs, T, 2 * static_cast<int64_t>(c.n_shared) * c.d_ff_shared, h->tr != nullptr && c.n_shared > 0},
      {"dABs", h->dABs, T, 2 * static_cast<int64_t>(c.n_shared) * c.d_ff_shared, h->tr != nullptr && c.n_shared > 0},
      {"dXp", h->dXp, S, c.d_model, h->tr != nullptr},
      {"dXs", h->dXs, T, c.d_model, h->tr != nullptr && c.n_shared > 0},
  };
  for (const Entry& e : table) {
    if (strcmp(e.n, name) == 0) {
      if (!e.present) return fail(DSMOE_ERR_INVALID_ARG, "this configuration has no %s buffer", name);
      *ptr = e.p;
      *rows = e.r;
      *cols = e.k;
      return DSMOE_OK;
    }
  }
  return fail(DSMOE_ERR_INVALID_ARG, "unknown workspace buffer '%s'", name);
}

DSMOE_EXPORT dsmoe_status dsmoe_balance_losses(dsmoe_handle* h, const float* f, const float* P, int32_t n_groups,
                                               const int32_t* group_of, float alpha1, float alpha2, float* f_dev,
                                               float* P_dev, float* losses, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (!f || !P || !group_of || !f_dev || !P_dev || !losses) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  if (n_groups < 1 || n_groups > h->cfg.n_routed || n_groups > 512)
    return fail(DSMOE_ERR_INVALID_ARG, "n_groups = %d outside [1, min(N', 512)]", n_groups);
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  CUDA_TRY(dsmoe::launch_balance_losses(f, P, h->cfg.n_routed, n_groups, group_of, alpha1, alpha2, f_dev, P_dev,
                                        losses, static_cast<cudaStream_t>(stream)));
  h->launches += 1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_sequence_balance(dsmoe_handle* h, int32_t T, int32_t seq_len, const int32_t* topk_idx,
                                                 const float* scores, float beta, float* f_seq, float* p_seq,
                                                 float* loss, void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (h->cfg.score == DSMOE_ROUTE_HASH) return fail(DSMOE_ERR_UNSUPPORTED, "hash routing has no scores");
  if (seq_len <= 0 || T < 0 || T % seq_len) return fail(DSMOE_ERR_INVALID_ARG, "T = %d is not whole sequences of %d", T, seq_len);
  if (T > h->cfg.max_tokens) return fail(DSMOE_ERR_WORKSPACE, "T = %d exceeds max_tokens", T);
  if (!loss || (T > 0 && (!topk_idx || !scores || !f_seq || !p_seq))) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  const int S = T / seq_len;
  CUDA_TRY(dsmoe::launch_sequence_balance(topk_idx, scores, S, seq_len, h->cfg.n_routed, h->k_active, beta, f_seq,
                                          p_seq, h->seq_terms, loss, static_cast<cudaStream_t>(stream)));
  h->launches += S > 0 ? 2 : 1;
  return DSMOE_OK;
}

DSMOE_EXPORT dsmoe_status dsmoe_bias_update(dsmoe_handle* h, int64_t T, const int32_t* counts, float alpha, float* b,
                                            void* stream) {
  if (!h) return fail(DSMOE_ERR_INVALID_ARG, "handle is NULL");
  if (!counts || !b) return fail(DSMOE_ERR_INVALID_ARG, "NULL argument");
  if (T < 0) return fail(DSMOE_ERR_INVALID_ARG, "T is negative");
  DeviceGuard g(h->device);
  if (!g.ok) return fail(DSMOE_ERR_CUDA, "cannot select device %d", h->device);
  CUDA_TRY(dsmoe::launch_bias_update(counts, T, h->cfg.n_routed, h->k_active, alpha, b,
                                     static_cast<cudaStream_t>(stream)));
  h->launches += 1;
  return DSMOE_OK;
}
