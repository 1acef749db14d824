/*
 * dsmoe.h -- C ABI of libdsmoe.so, the forward pass of a DeepSeekMoE layer on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (DeepSeekMoE summary, heloowird.com, shared-expert layer equation):
 *
 *     h_t = u_t + sum_{i <= K_s} FFN_i(u_t) + sum_{routed i} g_{i,t} FFN_i(u_t)
 *
 * with router affinities l = u . e_i ("MoE architecture: how DeepSeek achieves
 * more", section 2, G(x) = Softmax(W_g x)), scores s = softmax(l) | sigmoid(l) |
 * sqrt(softplus(l)) (DeepSeek-V4 book ch. 2, section 2), top-K' selection on
 * s + b with a selection-only bias (same chapter, section 3), gates g = s or
 * s / sum_selected s, and SwiGLU experts FFN(u) = W_down (SiLU(W_gate u) * W_up u).
 * The expert-level balance statistics f_i and P_i (DeepSeekMoE summary,
 * "Expert-level balance loss") are produced alongside.
 *
 * Conventions shared by every entry point:
 *   - All tensors are row-major and caller-owned. bf16 tensors are passed as
 *     void* to raw IEEE bfloat16 words. Weights use the nn.Linear layout
 *     [out_features, in_features] (the reduction dimension is contiguous).
 *   - Device pointers must be 16-byte aligned; NULL is allowed only where
 *     stated.
 *   - No entry point allocates device memory except dsmoe_create, and no
 *     entry point synchronises the device except where it says so. Work is
 *     enqueued on the caller's stream (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream); a forward with shared experts also runs their
 *     GEMMs on the handle's own side stream, forked from the caller's stream at the
 *     start of the call and joined back into it before the call's last kernel, so
 *     the caller's stream still orders everything (a CUDA graph capture of the call
 *     captures both).
 *   - Errors are returned, never raised: no exit, abort or trap. A kernel that
 *     gives up a bounded wait records DSMOE_ERR_DEVICE_TIMEOUT in a device
 *     status word that dsmoe_get_status() reports.
 *   - A handle may be used by one host thread at a time. Its forwards share one
 *     workspace: enqueue them on one stream (or order the streams); two forwards of
 *     the same handle that overlap on the GPU race. Separate handles are independent.
 */
#ifndef DSMOE_H
#define DSMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSMOE_ABI_VERSION 1

typedef enum dsmoe_status {
  DSMOE_OK = 0,
  DSMOE_ERR_INVALID_ARG = 1,    /* bad pointer, size or enum value                     */
  DSMOE_ERR_UNSUPPORTED = 2,    /* valid request outside what the kernels implement    */
  DSMOE_ERR_WORKSPACE = 3,      /* T above the handle's max_tokens, or allocation fail */
  DSMOE_ERR_CUDA = 4,           /* a CUDA runtime call failed (see dsmoe_last_error)   */
  DSMOE_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up a bounded wait                     */
} dsmoe_status;

/* Score function (DeepSeek-V4 book ch. 2, sections 2 and 5). */
typedef enum dsmoe_score {
  DSMOE_SCORE_SOFTMAX = 0,        /* s = softmax over the routed experts            */
  DSMOE_SCORE_SIGMOID = 1,        /* s = 1 / (1 + exp(-l))                          */
  DSMOE_SCORE_SQRT_SOFTPLUS = 2,  /* s = sqrt(log(1 + exp(l)))                      */
  DSMOE_ROUTE_HASH = 3            /* expert = token_id * hash_mult mod hash_mod, g=1 */
} dsmoe_score;

/* Where the per-expert bias b enters. */
typedef enum dsmoe_bias_mode {
  DSMOE_BIAS_NONE = 0,
  DSMOE_BIAS_SELECT_ONLY = 1,  /* key s~ = s + b decides the top-K'; gates and P use s
                                  (V4 book ch. 2 section 3; "MoE: sparse activation",
                                  load-balancing section)                                 */
  DSMOE_BIAS_IN_LOGITS = 2     /* l + b is scored ("MoE architecture", section 6 form)    */
} dsmoe_bias_mode;

/* Layer configuration. Field names follow the pages' notation:
 * d = d_model, N' = n_routed, K' = top_k, F = d_ff, K_s = n_shared, F_s = d_ff_shared. */
typedef struct dsmoe_cfg {
  int32_t d_model;      /* d, multiple of 64, >= 64                                  */
  int32_t n_routed;     /* N', 1..512                                                */
  int32_t top_k;        /* K', 1..16 and <= N' (1 for hash routing)                  */
  int32_t d_ff;         /* F, multiple of 64                                         */
  int32_t n_shared;     /* K_s, 0..8                                                 */
  int32_t d_ff_shared;  /* F_s, multiple of 64 when K_s > 0                          */
  int32_t score;        /* dsmoe_score                                               */
  int32_t bias_mode;    /* dsmoe_bias_mode                                           */
  int32_t renormalize;  /* 0: g = s of the selected experts; 1: g = s / sum_sel s    */
  int32_t max_tokens;   /* largest T a forward call may pass (sizes the workspace)   */
  uint32_t hash_mult;   /* hash routing multiplier (2654435761 for the V4 layer)     */
  uint32_t hash_mod;    /* hash routing modulus, 0 means N'; must be <= N'           */
} dsmoe_cfg;

typedef struct dsmoe_handle dsmoe_handle;

/* Library ABI version (DSMOE_ABI_VERSION). Host only. */
int32_t dsmoe_abi_version(void);

/* Human-readable name of a status code. Host only; never NULL. */
const char* dsmoe_status_string(dsmoe_status s);

/* The message of the last error raised on the calling host thread ("" if none). */
const char* dsmoe_last_error(void);

/* Validate a configuration without touching a GPU. Host only.
 * Returns DSMOE_OK, DSMOE_ERR_INVALID_ARG or DSMOE_ERR_UNSUPPORTED. */
dsmoe_status dsmoe_check_config(const dsmoe_cfg* cfg);

/* Device workspace bytes a handle for cfg allocates. Host only. */
dsmoe_status dsmoe_workspace_bytes(const dsmoe_cfg* cfg, size_t* bytes);

/* Create a handle on CUDA device `device`: validates cfg, allocates the
 * workspace (expert-contiguous activations, intermediate activations, routing
 * tables, statistics partials and the status word) sized for cfg->max_tokens.
 * The caller's current device is restored before returning. On failure *out is
 * NULL and nothing stays allocated. */
dsmoe_status dsmoe_create(const dsmoe_cfg* cfg, int32_t device, dsmoe_handle** out);

/* Release a handle and its workspace (synchronises the handle's device). NULL is a no-op. */
void dsmoe_destroy(dsmoe_handle* h);

/*
 * One forward pass of the layer for T tokens (0 <= T <= max_tokens), enqueued
 * on `stream`. Device pointers, all caller-owned:
 *
 *   x          bf16 [T, d]        token activations u_t
 *   token_ids  int32 [T]          hash routing only (else NULL); values >= 0
 *   W_router   bf16 [N', d]       expert centroids e_i (NULL for hash routing)
 *   b          fp32 [N']          per-expert bias (NULL iff bias_mode == NONE)
 *   W_gate     bf16 [N', F, d]    routed experts, gate projection
 *   W_up       bf16 [N', F, d]    routed experts, up projection
 *   W_down     bf16 [N', d, F]    routed experts, down projection
 *   Ws_gate    bf16 [K_s, F_s, d] shared experts (all three NULL iff K_s == 0)
 *   Ws_up      bf16 [K_s, F_s, d]
 *   Ws_down    bf16 [K_s, d, F_s]
 *
 * Outputs (device, caller-owned, fully overwritten; K' here is the handle's k_active,
 * cfg.top_k unless dsmoe_set_selection changed it):
 *
 *   h          bf16 [T, d]        layer output, accumulated in fp32, rounded once
 *                                 (fp32 partial sums under dsmoe_set_expert_range PARTIAL)
 *   topk_idx   int32 [T, K']      selected experts, by descending selection key,
 *                                 ties to the lower index
 *   gates      fp32 [T, K']       g_{i,t} of the selected experts, same order
 *   counts     int32 [N']         sum_t 1(token t selects expert i)
 *   f          fp32 [N']          f_i = N' / (K' T) * counts_i
 *   P          fp32 [N']          P_i = (1/T) sum_t s_{i,t} (0 for hash routing)
 *   P_sum      fp32 [N'] or NULL  sum_t s_{i,t}, for reductions across token shards
 *   scores_dbg fp32 [T, N'] or NULL  the raw scores s (not for hash routing)
 *
 * T == 0 writes counts = f = P = P_sum = 0 and nothing else. Returns
 * DSMOE_ERR_WORKSPACE if T > max_tokens, DSMOE_ERR_INVALID_ARG for a NULL or
 * misaligned pointer, DSMOE_ERR_CUDA if a launch fails. The output h does not
 * depend on the order of slots inside an expert's segment.
 */
dsmoe_status dsmoe_forward(dsmoe_handle* h, int32_t T,
                           const void* x, const int32_t* token_ids,
                           const void* W_router, const float* b,
                           const void* W_gate, const void* W_up, const void* W_down,
                           const void* Ws_gate, const void* Ws_up, const void* Ws_down,
                           void* h_out, int32_t* topk_idx, float* gates,
                           int32_t* counts, float* f, float* P, float* P_sum,
                           float* scores_dbg, void* stream);

/*
 * The same forward with the per-call tensors in HOST memory: x, token_ids and
 * every output (h, topk_idx, gates, counts, f, P) are host pointers (pinned
 * memory gives asynchronous copies; pageable memory works but serialises).
 * The weights stay device-resident. The inputs are copied into the handle's
 * workspace, the forward runs on `stream`, the outputs are copied back, and
 * the call synchronises `stream` before returning.
 */
dsmoe_status dsmoe_forward_host(dsmoe_handle* h, int32_t T,
                                const void* x_host, const int32_t* token_ids_host,
                                const void* W_router, const float* b,
                                const void* W_gate, const void* W_up, const void* W_down,
                                const void* Ws_gate, const void* Ws_up, const void* Ws_down,
                                void* h_host, int32_t* topk_idx_host, float* gates_host,
                                int32_t* counts_host, float* f_host, float* P_host,
                                void* stream);

/*
 * The host forward pipelined for serving loops: the same arguments and results as
 * dsmoe_forward_host, but the call only enqueues work and returns. Input copies and
 * output copies run on a copy stream the handle owns, the forward on `stream`, through
 * two staging slots used in turn, so the copies of one call overlap the forward of the
 * next or previous one. The caller must keep each call's host buffers alive and
 * untouched until that call has finished: dsmoe_host_sync blocks until every enqueued
 * host call is done; dsmoe_host_join makes `stream` wait for them without blocking the
 * host. All host entry points of a handle share its workspace: issue them from one host
 * thread with one `stream`.
 */
dsmoe_status dsmoe_forward_host_async(dsmoe_handle* h, int32_t T,
                                      const void* x_host, const int32_t* token_ids_host,
                                      const void* W_router, const float* b,
                                      const void* W_gate, const void* W_up, const void* W_down,
                                      const void* Ws_gate, const void* Ws_up, const void* Ws_down,
                                      void* h_host, int32_t* topk_idx_host, float* gates_host,
                                      int32_t* counts_host, float* f_host, float* P_host, void* stream);
dsmoe_status dsmoe_host_join(dsmoe_handle* h, void* stream);
dsmoe_status dsmoe_host_sync(dsmoe_handle* h);

/*
 * Expert-level balance statistics from token counts and score sums gathered
 * over T_total tokens (e.g. summed across token shards on several GPUs):
 * f_i = N' / (K' T_total) * counts_i and P_i = P_sum_i / T_total
 * (DeepSeekMoE summary, "Expert-level balance loss"). Device pointers, [N'] each.
 * T_total == 0 writes zeros.
 */
dsmoe_status dsmoe_balance_stats(dsmoe_handle* h, int64_t T_total, const int32_t* counts,
                                 const float* P_sum, float* f, float* P, void* stream);

/*
 * Load-balance control from a forward's statistics (all device pointers, [N'] unless
 * stated; nothing is allocated, work is enqueued on `stream`):
 *
 * dsmoe_balance_losses -- expert-level loss L_ExpBal = alpha1 (1/N') sum_i f_i P_i and
 *   device-level loss over n_groups groups of experts (group_of[i] in [0, n_groups)):
 *   f_dev[d] = mean of f over group d, P_dev[d] = sum of P over group d,
 *   L_DevBal = alpha2 sum_d f_dev[d] P_dev[d]  (DeepSeekMoE summary, "Expert-level
 *   balance loss" and "Device-level balance loss"). losses[0] = L_ExpBal,
 *   losses[1] = L_DevBal. 1 <= n_groups <= min(N', 512).
 *
 * dsmoe_sequence_balance -- sequence-wise statistics for T tokens made of T / seq_len
 *   whole sequences (DeepSeek-V4 book ch. 2, section 3): f_seq[q,i] = share of sequence
 *   q's tokens that selected expert i, p_seq[q,i] = mean score of expert i over the
 *   sequence ([S, N'] each), loss[0] = beta * mean_q sum_i f_seq[q,i] p_seq[q,i].
 *   topk_idx [T, K'] and scores [T, N'] come from dsmoe_forward (scores_dbg).
 *   T must be a multiple of seq_len and T <= max_tokens.
 *
 * dsmoe_bias_update -- the auxiliary-loss-free bias step b_i += alpha (K'/N' - counts_i/T)
 *   for counts gathered over T tokens (same chapter, section 3): an over-loaded expert's
 *   bias falls, an under-loaded one's rises. b is updated in place.
 */
dsmoe_status dsmoe_balance_losses(dsmoe_handle* h, const float* f, const float* P, int32_t n_groups,
                                  const int32_t* group_of, float alpha1, float alpha2, float* f_dev,
                                  float* P_dev, float* losses, void* stream);
dsmoe_status dsmoe_sequence_balance(dsmoe_handle* h, int32_t T, int32_t seq_len, const int32_t* topk_idx,
                                    const float* scores, float beta, float* f_seq, float* p_seq, float* loss,
                                    void* stream);
dsmoe_status dsmoe_bias_update(dsmoe_handle* h, int64_t T, const int32_t* counts, float alpha, float* b,
                               void* stream);

/* Read and clear the device status word (synchronises the handle's device).
 * DSMOE_OK, or DSMOE_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait. */
dsmoe_status dsmoe_get_status(dsmoe_handle* h);

/* Bound on the in-kernel waits of later forwards, in nanoseconds (default 2e9): a kernel
 * role (TMA producer, MMA issuer, epilogue) that waits longer for its operands or its
 * accumulator gives up, the kernel records it in the status word (dsmoe_get_status then
 * returns DSMOE_ERR_DEVICE_TIMEOUT) and that forward's outputs are undefined. Before the
 * kernel exits it still waits for the copies and MMAs it already started, for at least
 * one second whatever this limit, so that no asynchronous write outlives its CTA.
 * ns = 0 returns DSMOE_ERR_INVALID_ARG and keeps the previous limit. */
dsmoe_status dsmoe_set_wait_limit(dsmoe_handle* h, uint64_t ns);

/* Which kernel computes the two grouped expert GEMMs of dsmoe_forward (the gate/up
 * projection with SiLU(gate) * up, and the down projection; DeepSeekMoE summary,
 * shared-expert layer equation). Both accumulate each output in fp32 over K in
 * 16-element MMA steps, in the same order, and share the epilogue arithmetic.
 *   DSMOE_GEMM_SINGLE (default) one CTA per tile, M=128 MMAs, tiles of up to 128 tokens.
 *   DSMOE_GEMM_PAIR   CTA pairs on neighbouring SMs with M=256 MMAs (tcgen05 cta_group::2)
 *                     and tiles of up to 256 tokens: gate/up as two chains (gate, up) of
 *                     256 features sharing the token operand, down as 256 output rows.
 * dsmoe_set_gemm_kernel returns DSMOE_ERR_UNSUPPORTED when the pair kernel cannot be
 * launched on the device (the handle keeps its kind), and DSMOE_ERR_INVALID_ARG for
 * another kind. dsmoe_get_gemm_kernel returns the kind in use (-1 for a NULL handle). */
enum { DSMOE_GEMM_PAIR = 0, DSMOE_GEMM_SINGLE = 1 };
dsmoe_status dsmoe_set_gemm_kernel(dsmoe_handle* h, int32_t kind);
int32_t dsmoe_get_gemm_kernel(dsmoe_handle* h);

/* Inference-time selection variants of the DeepSeekMoE summary's expert-specialisation
 * analysis, applied by later dsmoe_forward / dsmoe_forward_host calls on this handle:
 *   mask_top = r >= 0 -- per token, the r experts ranked first by the selection key
 *     (s + b with a selection-only bias, else s; ties to the lower index) are masked out
 *     before the top-K' choice ("disable the top routed experts");
 *   k_active in [1, cfg.top_k] -- the number of routed experts each token activates
 *     ("fewer activated routed experts"): topk_idx and gates are then [T, k_active]
 *     row-major, gates are renormalised over the kept experts when cfg.renormalize is
 *     set, and f_i = N'/(k_active T) counts_i (also in dsmoe_balance_stats,
 *     dsmoe_sequence_balance and dsmoe_bias_update).
 * Requires mask_top + k_active <= n_routed; hash routing accepts only (0, top_k)
 * (DSMOE_ERR_UNSUPPORTED otherwise). Defaults (0, cfg.top_k) give the trained router's
 * selection. P_i (the mean score) does not depend on the variant.
 * dsmoe_route_noalloc always uses the configuration's plain selection. */
dsmoe_status dsmoe_set_selection(dsmoe_handle* h, int32_t mask_top, int32_t k_active);
dsmoe_status dsmoe_get_selection(dsmoe_handle* h, int32_t* mask_top, int32_t* k_active);

/*
 * Expert range: the part of the layer this handle applies, for expert parallelism
 * (DeepSeek-MoE interview card, deep dive on engineering trade-offs, item 5: the shared
 * experts are dense and replicated on every GPU while the routed experts are sharded
 * across GPUs; "MoE architecture" page, memory section: with expert parallelism each GPU
 * stores only part of the experts). Later forwards route every token over all N'
 * experts exactly as before (topk_idx, gates, counts, f, P are the whole layer's), but
 * apply only the routed experts e_begin <= e < e_end:
 *   W_gate, W_up [e_end - e_begin, F, d] and W_down [e_end - e_begin, d, F] hold those
 *   experts only (expert e_begin first); W_router and b stay [N', d] and [N'].
 * flags:
 *   DSMOE_RANGE_PARTIAL     h is fp32 [T, d] (not bf16): the partial sum
 *                           sum_{k : e(t,k) in range} g_{t,k} FFN_{e(t,k)}(u_t), never rounded,
 *                           for the ranks of an expert-parallel group to add;
 *   DSMOE_RANGE_ADD_SHARED  add the residual u_t and the shared experts'
 *                           sum_{i<=K_s} FFN_i(u_t) (one rank of the group does this; Ws_*
 *                           may be NULL on the others).
 * The default, (0, N', DSMOE_RANGE_ADD_SHARED), is the whole layer with bf16 h. Any other
 * part needs DSMOE_RANGE_PARTIAL; a full range with PARTIAL | ADD_SHARED gives the whole
 * layer unrounded in fp32. Errors: an empty or out-of-bounds range, unknown flags, or a
 * part without DSMOE_RANGE_PARTIAL return DSMOE_ERR_INVALID_ARG and leave the handle as
 * it was. dsmoe_forward_host supports the default only (DSMOE_ERR_UNSUPPORTED otherwise).
 *
 * dsmoe_round_bf16: dst[i] = bf16(src[i]) (round to nearest even) for n fp32 values,
 * n a multiple of 8, both device pointers 16-byte aligned; for summed partials.
 */
enum { DSMOE_RANGE_PARTIAL = 1, DSMOE_RANGE_ADD_SHARED = 2 };
dsmoe_status dsmoe_set_expert_range(dsmoe_handle* h, int32_t e_begin, int32_t e_end, int32_t flags);
dsmoe_status dsmoe_get_expert_range(dsmoe_handle* h, int32_t* e_begin, int32_t* e_end, int32_t* flags);
dsmoe_status dsmoe_round_bf16(dsmoe_handle* h, int64_t n, const float* src, void* dst, void* stream);

/*
 * Expert parallelism with token dispatch: routed experts split over `world` ranks in
 * contiguous blocks (rank j holds experts [j*B + min(j, R), ...) with B = N' / world,
 * R = N' % world, the first R blocks one larger), the router and the shared experts
 * replicated on every rank (DeepSeek-MoE interview card, deep dive on engineering
 * trade-offs, item 5; "MoE: sparse activation" page, training-cost section: tokens travel
 * by all-to-all to the GPUs that hold their experts). Each rank calls, in order:
 *
 * dsmoe_ep_route -- route its T tokens (as dsmoe_forward: topk_idx, gates, counts, f, P,
 *   P_sum, scores_dbg over its own tokens) and gather their rows into the expert-
 *   contiguous slot order, which is also destination order: workspace "Xp" rows
 *   [0, T K') are what this rank sends. send_rows int32 [world] (device, out) = rows
 *   bound for each rank. The per-expert row counts to send are `counts` (rank j's block).
 * (the caller exchanges the per-expert counts and the rows, e.g. NCCL all-to-all)
 * dsmoe_ep_experts -- the owner's experts on the rows it received: rows bf16
 *   [n_rows, d] grouped by source rank, and within a source by expert; recv_counts int32
 *   [n_src, e_end - e_begin] (device) rows per (source, local expert); W_gate, W_up
 *   [e_end - e_begin, F, d] and W_down [e_end - e_begin, d, F] this rank's experts.
 *   Writes Y bf16 [n_rows, d], row for row. n_rows <= max_tokens * top_k and
 *   n_src * (e_end - e_begin) <= 512 (DSMOE_ERR_WORKSPACE / DSMOE_ERR_UNSUPPORTED).
 * (the caller sends Y back along the reverse exchange, so that it arrives in the order
 *  the rows left)
 * dsmoe_ep_combine -- the shared experts on the rank's own tokens and the combine
 *   h_t = u_t + sum_shared FFN(u_t) + sum_k g_{t,k} Y[slot(t,k)], Y bf16 [T K', d] in
 *   this rank's slot order (the returned rows); h bf16 [T, d]. Uses the slot table of the
 *   handle's last dsmoe_ep_route (T must match, else DSMOE_ERR_INVALID_ARG).
 * The three calls use the handle's workspace (dsmoe_ep_experts overwrites the expert
 * offsets and the A1 rows); a handle serves one rank, one layer call at a time.
 */
dsmoe_status dsmoe_ep_route(dsmoe_handle* h, int32_t T, const void* x, const int32_t* token_ids,
                            const void* W_router, const float* b, int32_t* topk_idx, float* gates,
                            int32_t* counts, float* f, float* P, float* P_sum, float* scores_dbg, int32_t world,
                            int32_t* send_rows, void* stream);
dsmoe_status dsmoe_ep_experts(dsmoe_handle* h, int32_t n_src, int32_t e_begin, int32_t e_end,
                              const int32_t* recv_counts, int64_t n_rows, const void* rows, const void* W_gate,
                              const void* W_up, const void* W_down, void* Y, void* stream);
dsmoe_status dsmoe_ep_combine(dsmoe_handle* h, int32_t T, const void* x, const void* Ws_gate, const void* Ws_up,
                              const void* Ws_down, const float* gates, const void* Y, void* h_out, void* stream);

/*
 * First steps of the backward pass, for an upstream gradient dh = dL/dh of the layer
 * output h_t = u_t + sum_shared FFN(u_t) + sum_k g_{t,k} y_{t,k} (DeepSeekMoE summary,
 * shared-expert layer equation), the top-K' selection held fixed (its indicator has no
 * gradient).
 *
 * dsmoe_backward_gates -- uses the expert outputs y and the slot table of this handle's
 *   last forward (call it after that forward, on the same stream, with the same T):
 *     dh     bf16 [T, d]        upstream gradient (device, 16-byte aligned)
 *     gates  fp32 [T, K']       the forward's gates
 *     dg     fp32 [T, K'] out   dg_{t,k} = <dh_t, y_{t,k}>, fp32 accumulation of bf16 terms
 *     dY     bf16 [T K', d] out the routed experts' output gradient g_{t,k} dh_t, in the
 *                               forward's slot order (expert-contiguous; workspace "slot_of"
 *                               maps (t, k) to its row)
 *   Under an expert range, picks of experts outside it get dg = 0 and no dY row.
 *
 * dsmoe_backward_router -- the router's backward with the expert-level balance term
 *   alpha sum_i f_i P_i (same page, "Expert-level balance loss": P_i carries the
 *   gradient to the router, f_i is a constant). Not for hash routing (UNSUPPORTED).
 *     x, W_router        the forward's bf16 inputs
 *     topk_idx, gates    the forward's picks and gates [T, K']
 *     scores             fp32 [T, N'], the forward's raw scores (its scores_dbg output)
 *     dg                 fp32 [T, K'] from dsmoe_backward_gates
 *     f, alpha           the balance term's f_i [N'] and factor (f may be NULL iff alpha = 0)
 *     dlogits fp32 [T, N'] out  dL/dl: ds = alpha f_i / T + the gate terms (dg at the kept
 *                               experts, or (dg_k - sum_j dg_j g_j) / sum_kept s when the
 *                               gates are renormalised), then the score function's
 *                               derivative (softmax, sigmoid, or sqrt(softplus), whose slope
 *                               sigma(l) / (2 s) uses sigma(l) = 1 - exp(-s^2))
 *     dx      fp32 [T, d] out   dlogits W_router (the router's part of dL/du)
 *     dW_router fp32 [N', d] out dlogits^T x
 *   With N' a multiple of 64, d a multiple of 64, T >= 256, T >= 2 N' and all pointers
 *   16-byte aligned, both products run on the tensor cores: dlogits is split into bf16
 *   parts hi + lo (what remains is below 2^-16 of each value of magnitude below 3.39e38,
 *   the largest finite bf16; the [hi | lo] rows overwrite
 *   the handle's "logits" workspace, which only the forward reads), dW_router = hi^T x +
 *   lo^T x on the weight-gradient GEMM (the two fp32 results held in dx's memory until
 *   they are added, hi first) and dx = [hi | lo] [W_router; W_router] on the input-
 *   gradient GEMM. Otherwise both run on the CUDA cores in fp32, dW_router (few outputs,
 *   K = T) split over T into slices whose partial sums are held in dx's memory until
 *   they are added, before dx itself is computed. dx must not alias another argument.
 *   All sums run in a fixed order (deterministic).
 */
dsmoe_status dsmoe_backward_gates(dsmoe_handle* h, int32_t T, const void* dh, const float* gates, float* dg,
                                  void* dY, void* stream);

/*
 * The experts' part of dL/du (the input gradient through the expert FFNs), for the same
 * upstream gradient:
 *   dm = W_down^T dy, da = dm * b * SiLU'(a), db = dm * SiLU(a), du = W_gate^T da + W_up^T db
 * with SiLU'(a) = sigma(a)(1 + a(1 - sigma(a))), dy = g dh for a routed pick (the dY of
 * dsmoe_backward_gates) and dy = dh for a shared expert.
 *
 * dsmoe_set_training(h, 1) allocates the training buffers (about (4 F + d) T K' bf16 plus
 * the shared experts' share, sized for max_tokens); from then on every forward of the
 * handle also stores its pre-activations a = u W_gate^T and b = u W_up^T (bf16). (h, 0)
 * frees them. Neither is called inside a forward.
 *
 * dsmoe_backward_experts -- after a training forward of T tokens on this handle (same T,
 * else DSMOE_ERR_INVALID_ARG):
 *     dh        bf16 [T, d]          upstream gradient
 *     dY        bf16 [T K', d]       the routed experts' output gradients in slot order
 *                                    (dsmoe_backward_gates)
 *     W_*, Ws_* the forward's weights (the handle's expert range, as for the forward)
 *     dx_add    fp32 [T, d] or NULL  added to the result (e.g. dsmoe_backward_router's dx)
 *     dx        fp32 [T, d] out      dh + sum_shared du + sum_k du_{t,k} (+ dx_add): the
 *                                    residual, shared-expert and routed-expert parts of dL/du
 *   Two grouped GEMMs on the tensor cores (the weights read MN-major, in the forward's
 *   layout) and one combine; fp32 accumulation, da | db and the per-slot du rows stored
 *   as bf16, the shared experts' du summed in fp32. The weight gradients are computed by
 *   dsmoe_backward_weights.
 */
/*
 * dsmoe_backward_weights -- the experts' weight gradients, after dsmoe_backward_experts
 * for the last training forward (same T, else DSMOE_ERR_INVALID_ARG):
 *   dW_down = sum_r dy_r m_r^T, dW_gate = sum_r da_r u_r^T, dW_up = sum_r db_r u_r^T
 * summed over the rows r each expert applied to (routed: its picks' slots, with
 * dy = g dh; shared: every token, dy = dh), from the forward's saved m (A1) and gathered
 * rows u, and the da | db of dsmoe_backward_experts:
 *     dh, dY, x          bf16, as given to the forward and dsmoe_backward_experts
 *     dW_gate, dW_up     fp32 [N_local, F, d] out   (N_local = the handle's expert range)
 *     dW_down            fp32 [N_local, d, F] out
 *     dWs_gate, dWs_up   fp32 [K_s, F_s, d] out, dWs_down fp32 [K_s, d, F_s] out
 *                        (all three NULL iff the handle adds no shared experts)
 *   Grouped GEMMs on the tensor cores reducing over token rows (both operands MN-major,
 *   each routed expert's rows a ragged K range), fp32 accumulation of bf16 products.
 *   An expert no token picked gets a zero gradient. All nine pointers must be 16-byte
 *   aligned (the gradients are written by bulk tensor copies of 32 x 16 fp32 blocks);
 *   else DSMOE_ERR_INVALID_ARG.
 */
dsmoe_status dsmoe_backward_weights(dsmoe_handle* h, int32_t T, const void* dh, const void* dY, const void* x,
                                    float* dW_gate, float* dW_up, float* dW_down, float* dWs_gate, float* dWs_up,
                                    float* dWs_down, void* stream);
dsmoe_status dsmoe_set_training(dsmoe_handle* h, int32_t enable);
dsmoe_status dsmoe_backward_experts(dsmoe_handle* h, int32_t T, const void* dh, const void* dY, const void* W_gate,
                                    const void* W_up, const void* W_down, const void* Ws_gate, const void* Ws_up,
                                    const void* Ws_down, const float* dx_add, float* dx, void* stream);
dsmoe_status dsmoe_backward_router(dsmoe_handle* h, int32_t T, const void* x, const void* W_router,
                                   const int32_t* topk_idx, const float* gates, const float* scores,
                                   const float* dg, const float* f, float alpha, float* dlogits, float* dx,
                                   float* dW_router, void* stream);

/* Per-stage timing: while enabled, each forward with T > 0 records CUDA events at every
 * stage boundary (no synchronisation): on its stream for the chain router -> select ->
 * scan -> permute -> routed gate/up GEMM -> routed down GEMM -> combine, and on the
 * handle's side stream around the shared experts' two GEMMs, which run concurrently with
 * the routing stages (an empty interval without shared experts). dsmoe_stage_times waits
 * for the recorded events and writes, per stage, the mean duration in ms over the last
 * min(64, forwards recorded since timing was enabled) forwards. Enabling (or disabling)
 * timing resets the record. */
dsmoe_status dsmoe_set_timing(dsmoe_handle* h, int32_t enable);
dsmoe_status dsmoe_stage_times(dsmoe_handle* h, float* ms, int32_t max_n, int32_t* n);
/* Name of stage i ("router", "select", "scan", "permute", "gemm_gate_up", "gemm_down",
 * "combine", "shared_experts"), or NULL past the last. */
const char* dsmoe_stage_name(int32_t i);

/* Number of kernels this handle has launched since creation. */
dsmoe_status dsmoe_launch_count(dsmoe_handle* h, int64_t* n);

/* Role cycle counters of the grouped GEMMs, for profiling (a library built with
 * DSMOE_ROLE_CYCLES defined: `build.py --role-cycles`). Copies the counters of the current
 * device, summed over every launch since the last call, to out[n], n >= 5 * 160 * 9 = 7200
 * (uint64, layout [launch kind][CTA 0..159][slot]; kinds: 0 down and 1 gate/up launches
 * with routed groups, 2 down and 3 gate/up launches of the shared experts alone, 4 the
 * weight-gradient GEMM of dsmoe_backward_weights), and clears them.
 * Slots: 0 clock64 cycles from CTA start to exit, 1 globaltimer ns over the same interval,
 * 2 producer cycles waiting for a free ring stage, 3 MMA-thread cycles waiting for a
 * landed stage, 4 MMA-thread cycles waiting for a free accumulator, 5 MMA-thread cycles
 * in its tile loop, 6 epilogue (first warp) cycles waiting for a finished accumulator,
 * 7 epilogue cycles in its tile loop, 8 tiles. Synchronous. Returns
 * DSMOE_ERR_UNSUPPORTED from a library built without the counters, DSMOE_ERR_INVALID_ARG
 * for a NULL or short buffer. */
dsmoe_status dsmoe_gemm_role_cycles(uint64_t* out, int32_t n);

/*
 * Device address and shape of one intermediate buffer of the handle's workspace, for
 * tests and debugging; contents are those of the last forward on this handle:
 *   "logits"  fp32 [T, N']        router affinities, written when the CUDA-core router
 *                                 runs (T < 256) as split-K partial sums: the first
 *                                 slice of [splits, T, N']; absent for hash routing
 *   "offsets" int32 [N'+1]        first slot of each expert's segment
 *   "slot_of" int32 [T, K']       slot holding token t's k-th expert row
 *   "Xp"      bf16 [T K', d]      token rows in expert-contiguous slot order
 *   "A1"      bf16 [T K', F]      SiLU(X W_gate^T) * (X W_up^T) per slot
 *   "A1s"     bf16 [T, K_s F_s]   the same for the shared experts, side by side
 *   "Y"       bf16 [T K', d]      routed expert outputs per slot
 *   "Hs"      fp32 [T, d]         u_t + sum of the shared experts' outputs
 *   training buffers (dsmoe_set_training), absent otherwise:
 *   "AB"      bf16 [T K', 2 F]    a | b pre-activations per slot (last training forward)
 *   "ABs"     bf16 [T, 2 K_s F_s] a | b of the shared experts, [a_s | b_s] per expert
 *   "dAB"     bf16 [T K', 2 F]    da | db per slot (last dsmoe_backward_experts)
 *   "dABs"    bf16 [T, 2 K_s F_s] da | db of the shared experts
 *   "dXp"     bf16 [T K', d]      du per slot (routed experts)
 *   "dXs"     fp32 [T, d]         du summed over the shared experts
 * Rows/cols are given for max_tokens; the first T (or T K') rows are meaningful.
 * Returns DSMOE_ERR_INVALID_ARG for an unknown name or a buffer this cfg lacks.
 */
dsmoe_status dsmoe_workspace_tensor(dsmoe_handle* h, const char* name, void** ptr, int64_t* rows,
                                    int64_t* cols);

/*
 * The routing stage with no allocation: router affinities, scores, top-K' experts,
 * gates, expert counts, f_i and P_i for T tokens -- the outputs dsmoe_forward gives,
 * up to fp32 rounding (experts whose keys tie within rounding may be picked or
 * ordered differently) -- without a handle and without any device allocation.
 *
 * The pages have no counterpart to this entry point. It is for callers that cannot
 * call cudaMalloc when they route a batch: code whose framework has already claimed
 * all device memory through its own pool, plugins that must not touch the allocator
 * while their host serves requests, or anything that cannot create a handle
 * (dsmoe_create allocates a workspace). The caller passes inputs and outputs only:
 *
 *   cfg        layer configuration (host); T must not exceed cfg->max_tokens
 *   x          bf16 [T, d], W_router bf16 [N', d], b fp32 [N'] (NULL iff no bias)
 *   topk_idx   int32 [T, K'], gates fp32 [T, K'], counts int32 [N'], f fp32 [N'],
 *              P fp32 [N'] -- device, caller-owned, fully overwritten
 *
 * Scratch: a fixed array of about 514 KiB inside the library's device image (each
 * GPU that loads the library holds it until the process exits); it bounds N' to at
 * most 512. Learned routing only: hash routing returns DSMOE_ERR_UNSUPPORTED, as
 * does N' > 512; T > cfg->max_tokens returns DSMOE_ERR_WORKSPACE (dsmoe_last_error
 * says which). The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before
 * any stream capture. Later calls whose stream is not capturing look it up again, so
 * the address stays valid after cudaDeviceReset; after a reset, make one such call
 * before capturing again. Work runs on `stream` of the current device. Every call
 * shares the array: each call clears the counters it needs on its stream first,
 * and calls that overlap on the GPU (other streams or threads) race and must be
 * serialised by the caller.
 */
dsmoe_status dsmoe_route_noalloc(const dsmoe_cfg* cfg, int32_t T, const void* x, const void* W_router,
                                 const float* b, int32_t* topk_idx, float* gates, int32_t* counts, float* f,
                                 float* P, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif /* DSMOE_H */
