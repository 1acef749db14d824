// kernels.h -- host-side launchers of the dsmoe kernels (internal to libdsmoe.so).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsmoe {

using bf16 = __nv_bfloat16;

// Bits of the device status word.
enum : uint32_t {
  kStatusTimeoutProducer = 1u << 0,
  kStatusTimeoutMma = 1u << 1,
  kStatusTimeoutEpilogue = 1u << 2,
  kStatusTimeoutDrain = 1u << 3,
  kStatusBadIndex = 1u << 4,
};


// ---------------------------------------------------------------- router (router.cu)
// logits[t, i] = sum_k x[t,k] W_router[i,k], fp32, as `splits` partial sums over
// slices of k (logits holds splits x T x N floats).
constexpr int kRouterMaxSplits = 64;
int router_logits_splits(int T, int N, int d, int num_sms);
cudaError_t launch_router_logits(const bf16* x, const bf16* W_router, int T, int N, int d, int splits,
                                 float* logits, cudaStream_t s);

struct SelectArgs {
  const float* logits;   // [splits, T, N] partial sums
  int splits;
  const float* b;        // [N] or nullptr
  int T, N, K;           // K: experts kept per token
  int mask_top;          // experts ranked first that are masked before the K are kept
  int score;             // dsmoe_score
  int bias_select;       // selection-only bias
  int bias_in_logits;    // b is added to the summed logits before scoring
  int renormalize;
  int32_t* topk_idx;     // [T, K]
  float* gates;          // [T, K]
  int32_t* counts;       // [N], accumulated with atomics (zeroed by the caller)
  float* P_part;         // [gridDim.x, N] per-block partial score sums
  float* scores_dbg;     // [T, N] or nullptr
  uint32_t* status;
};
// Scores, top-K' selection, gates and per-block statistics partials; returns the grid size used.
cudaError_t launch_select(const SelectArgs& a, int grid, cudaStream_t s);
int select_grid(int T, int num_sms);

// Router affinities on the tensor cores (router_sm100.cu): split-K partial sums,
// partial[slice][t][i] for `splits` slices of the reduction dimension. The B tile is
// n_chunks chunks of nc router rows (nc a multiple of 16, at most 256); the
// accumulator takes tmem_cols TMEM columns.
struct RouterTcArgs {
  CUtensorMap tm_x;  // 2D [T, d] bf16, box (64, 128)
  CUtensorMap tm_w;  // 2D [N', d] bf16, box (64, nc)
  int T, N, d, splits;
  int n_chunks, nc;
  uint32_t tmem_cols;
  float* partial;    // [splits, T, N']
  uint32_t* status;
  uint64_t wait_limit_ns;
};
void router_tc_shape(int N, int* n_chunks, int* nc, uint32_t* tmem_cols);
int router_tc_splits(int T, int d, int num_sms);
// Rows of partial sums the tensor-core router may write beyond T (for any GPU with at
// most 192 SMs): splits * T <= T + 2 * 192 * 128.
constexpr int64_t kRouterTcExtraRows = 2 * 192 * 128;
cudaError_t launch_router_tc(const RouterTcArgs& a, int grid, cudaStream_t s);

cudaError_t launch_hash_route(const int32_t* token_ids, int T, int N, uint32_t mult, uint32_t mod,
                              int32_t* topk_idx, float* gates, int32_t* counts, uint32_t* status,
                              cudaStream_t s);

// ---------------------------------------------------------------- routing tables (permute.cu)
struct ScanArgs {
  const int32_t* counts_ws;  // [N]
  const float* P_part;       // [n_part, N] or nullptr (hash routing)
  int n_part, N, K;
  int64_t T;                 // tokens the statistics are taken over
  int32_t* counts;           // [N] out
  float* f;                  // [N] out
  float* P;                  // [N] out
  float* P_sum;              // [N] out or nullptr
  int32_t* offsets;          // [N+1] out, or nullptr
  int32_t* cursor;           // [N] zeroed, or nullptr
  int32_t e_begin, e_end;    // experts that get slots; the others' segments are empty
};
cudaError_t launch_scan_stats(const ScanArgs& a, cudaStream_t s);

// Balance statistics from already-reduced counts and score sums.
cudaError_t launch_balance_stats(const int32_t* counts, const float* P_sum, int64_t T, int N, int K,
                                 float* f, float* P, cudaStream_t s);

// slot positions + gather of token rows into expert-contiguous order. Only experts in
// [e_begin, e_end) get slots; a (token, k) whose expert lies outside has slot -1.
cudaError_t launch_permute_gather(const bf16* x, const int32_t* topk_idx, const int32_t* offsets,
                                  int32_t* cursor, int T, int K, int N, int e_begin, int e_end, int d,
                                  int32_t* slot_of, bf16* Xp, uint32_t* status, int num_sms, cudaStream_t s);

// Expert parallelism. block_rows: out[j] = rows of the slot order that fall in rank j's
// contiguous block of experts (blocks of N / world, the first N % world one larger).
// group_offsets: offsets[0..groups] = exclusive scan of counts[groups] (negative counts
// are recorded in the status word and taken as 0).
cudaError_t launch_block_rows(const int32_t* offsets, int N, int world, int32_t* out, cudaStream_t s);
cudaError_t launch_group_offsets(const int32_t* counts, int groups, int32_t* offsets, uint32_t* status,
                                 cudaStream_t s);

// ---------------------------------------------------------------- balance control (balance.cu)
cudaError_t launch_balance_losses(const float* f, const float* P, int N, int G, const int32_t* group_of,
                                  float alpha1, float alpha2, float* f_dev, float* P_dev, float* losses,
                                  cudaStream_t s);
cudaError_t launch_sequence_balance(const int32_t* topk_idx, const float* scores, int S, int seq_len, int N,
                                    int K, float beta, float* f_seq, float* p_seq, float* seq_terms, float* loss,
                                    cudaStream_t s);
cudaError_t launch_bias_update(const int32_t* counts, int64_t T, int N, int K, float alpha, float* b,
                               cudaStream_t s);

// ---------------------------------------------------------------- combine (combine.cu)
// h = base + sum_k gates[t,k] Y[slot_of[t,k]] over the k whose slot is not -1, where base
// is Hs (fp32 x + shared experts) when Hs is not null, else x when add_x, else 0; written
// as bf16 h (rounded once) or, when h32 is not null, as fp32 h32.
struct CombineArgs {
  const bf16* x;
  const float* Hs;
  int add_x;
  const bf16* Y;
  const int32_t* slot_of;
  const float* gates;
  int T, K, d;
  bf16* h;
  float* h32;
};
cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s);
// dst[i] = bf16(src[i]) (round to nearest even), n a multiple of 8, both 16-byte aligned.
cudaError_t launch_round_bf16(const float* src, bf16* dst, int64_t n, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- backward (backward.cu)
// dg[t,k] = <dh_t, Y[slot_of[t,k]]> and dY[slot_of[t,k]] = bf16(gates[t,k] dh_t).
struct GateGradArgs {
  const bf16* dh;          // [T, d]
  const bf16* Y;           // [slots, d] the forward's expert outputs in slot order
  const int32_t* slot_of;  // [T, K]
  const float* gates;      // [T, K]
  int T, K, d;
  float* dg;               // [T, K]
  bf16* dY;                // [slots, d]
};
cudaError_t launch_gate_grad(const GateGradArgs& a, int num_sms, cudaStream_t s);

// dlogits [T, N] from the forward's scores, picks and gates, dg, and the balance term
// alpha f_i / T (f may be null: no balance term).
struct RouterBwdArgs {
  const float* scores;     // [T, N]
  const int32_t* topk_idx; // [T, K]
  const float* gates;      // [T, K]
  const float* dg;         // [T, K]
  const float* f;          // [N] or nullptr
  float alpha;
  int T, N, K, score, renormalize;
  float* dlogits;          // [T, N]
  uint32_t* status;
};
cudaError_t launch_router_backward(const RouterBwdArgs& a, int num_sms, cudaStream_t s);

// dx[t] = dh[t] + dXs[t] (if set) + dx_add[t] (if set) + sum_k dXp[slot_of[t,k]] (fp32 out;
// slots of -1 are skipped).
cudaError_t launch_dx_combine(const bf16* dh, const float* dXs, const float* dx_add, const bf16* dXp,
                              const int32_t* slot_of, int T, int K, int d, float* dx, int num_sms, cudaStream_t s);

// C[M, N] = A(M x K, fp32, element (m, k) at A[m a_sm + k a_sk]) * B (bf16 [K, ldb]), fp32 out.
struct GemmF32Args {
  const float* A;
  int64_t a_sm, a_sk;
  const bf16* B;
  int64_t ldb;
  float* C;
  int64_t ldc;
  int M, N, K;
  // split-K (splits > 1): the K range is cut into `splits` slices whose partial products go
  // to partial[splits][M][ldc] and are then summed in slice order into C (deterministic)
  int splits;
  float* partial;
};
cudaError_t launch_gemm_f32_bf16(const GemmF32Args& a, cudaStream_t s);
// dst [T, 2N] bf16 = rows [hi | lo] of src [T, N] fp32 (hi = bf16(v), lo = bf16(v - hi));
// N a multiple of 4, src 16-byte and dst 8-byte aligned.
cudaError_t launch_hilo_split(const float* src, bf16* dst, int T, int N, int num_sms, cudaStream_t s);
// C[m, n] = sum over z = 0 .. splits-1, in order, of partial[z][m, n] ([splits, M, ldc] floats).
cudaError_t launch_split_sum(const float* partial, int splits, int M, int N, int64_t ldc, float* C, cudaStream_t s);

// ---------------------------------------------------------------- grouped GEMM (gemm_sm100.cu)
constexpr int kGemmMaxGroups = 8 + 512;  // shared + routed groups of one grouped GEMM
// Tokens per grouped-GEMM tile (the row box of the token-side tensor maps): 128, or 256
// for the gate/up projection of layers with a K loop of at least 20 blocks of 64 and a
// few hundred rows per expert, where the larger N moves fewer shared-memory bytes per MAC
// and the one accumulator it leaves (the next tile waits for this tile's epilogue) costs
// less than that saves (measured: V3, d = 7168, gate/up -5%; the 2B-shaped layer,
// d = 1280, -3.5%; the GShard shapes, d = 1024, +2-5%, so they keep 128).
constexpr int kGemmTokenTile = 128;
constexpr int kGemmTokenTileLarge = 256;
// rows, groups: the token rows and the groups (routed and shared) of the launch
inline int gateup_token_tile(int d_model, int64_t rows, int groups) {
  return (d_model >= 1280 && groups > 0 && rows >= 192LL * groups) ? kGemmTokenTileLarge : kGemmTokenTile;
}
struct GemmArgs {
  CUtensorMap a_routed;   // 2D [rows, K] activations of routed slots, box (64, token tile)
  CUtensorMap a_shared;   // 2D [T, K_shared] activations of the shared groups, box (64, token tile)
  CUtensorMap b0_routed;  // 3D (K, rows, experts): gate (SwiGLU) or down (plain) weights
  CUtensorMap b1_routed;  // 3D up-projection weights (SwiGLU only)
  CUtensorMap b0_shared;
  CUtensorMap b1_shared;
  const int32_t* offsets;         // [n_routed + 1] slot offset of each routed group
  int32_t n_routed;               // routed groups
  int32_t expert_mod;             // 0: routed group g is expert g; n > 0: expert g mod n
  int32_t n_shared_groups;        // shared groups (tiles run before the routed ones)
  int32_t m_shared;               // rows of every shared group (T)
  int32_t n_tiles_routed, n_tiles_shared;  // output tiles along N
  int32_t kb_routed, kb_shared;            // 64-wide K blocks per tile
  int32_t kb_per_b_expert_shared;          // shared B switches expert every this many K blocks
  int32_t n_valid_routed, n_valid_shared;  // valid output columns
  bf16* out_routed;
  int64_t ld_routed;
  bf16* out_shared;               // bf16 output of the shared groups (gate/up GEMM)
  float* out_shared_f32;          // fp32 output of the shared group + residual (down GEMM)
  const bf16* residual;           // [m_shared, ld_shared] added to out_shared_f32
  int64_t ld_shared;
  int32_t shared_col_stride;      // shared group g writes at column g * shared_col_stride
  uint32_t* status;
  uint64_t wait_limit_ns;
  // gate/up only, for the backward pass: when set, the pre-activations a = X W_gate^T and
  // b = X W_up^T are also stored (bf16), a | b side by side: routed [rows, 2F]; shared
  // [T, K_s 2 F_s] with shared expert g at columns 2 g F_s
  bf16* save_ab_routed;
  bf16* save_ab_shared;
};
// tok: the token tile, kGemmTokenTile, or kGemmTokenTileLarge for the gate/up projection
// (the token maps' row box must equal it)
cudaError_t launch_grouped_gemm(bool swiglu, int tok, const GemmArgs& a, int grid, cudaStream_t s);
// Profiling builds (DSMOE_ROLE_CYCLES, role_clock.cuh): copy the one-CTA grouped GEMM's role
// counters to host[kRoleCounters] and clear them; false in any other build.
bool read_role_cycles(unsigned long long* host, cudaError_t* err);
// The weight-gradient GEMM's counters (one row set, kRoleCtas x kRsSlots), cleared likewise.
bool read_role_cycles_dw(unsigned long long* host, cudaError_t* err);

// The experts' backward GEMMs (gemm_bwd_sm100.cu). kBwdDM: da | db from dy and W_down;
// kBwdDX: dx rows from da | db and W_gate, W_up. The weight maps b0 / b1 of `g` are 4-D
// views (64 M, K, M / 64, experts) of the weights with box (64, 64, 4, 1), M contiguous.
enum { kBwdDM = 0, kBwdDX = 1 };
struct GemmBwdArgs {
  GemmArgs g;                              // schedule, token-row maps, weight views, status
  int32_t kb_half_routed, kb_half_shared;  // kBwdDX: F / 64 and F_s / 64 (K blocks per half)
  const bf16* ab_routed;                   // kBwdDM: the forward's saved a | b
  const bf16* ab_shared;
  bf16* dab_routed;                        // kBwdDM out: da | db, same layout
  bf16* dab_shared;
  int64_t ld_ab_routed, ld_ab_shared;
  int32_t width_routed, width_shared;      // F and F_s
  bf16* dx_routed;                         // kBwdDX out: [rows, d] bf16 per slot
  float* dx_shared;                        // kBwdDX out: [T, d] fp32, summed over shared experts
  int64_t ld_dx;
};
cudaError_t launch_grouped_gemm_bwd(int mode, const GemmBwdArgs& a, int grid, cudaStream_t s);

// The experts' weight gradients (gemm_dw_sm100.cu): per group g, out[g][i][j] =
// sum_r A[r, i] B[r, j] over the group's rows r (routed group g: rows offsets[g] ..
// offsets[g+1] of the slot order; shared group: rows 0 .. T). A and B are 3-D views
// (64, rows, cols / 64) of [rows, cols] bf16 buffers, A with box (64, 64, 2), B with box
// (64, 64, 4); an operand starts at atom column atom0 (+ g * step for shared group g).
struct GemmDwArgs {
  CUtensorMap a_routed, b_routed, a_shared, b_shared;
  int32_t a_atom0_routed, b_atom0_routed;
  int32_t a_atom0_shared, b_atom0_shared, a_atom_step_shared, b_atom_step_shared;
  const int32_t* offsets;  // [n_routed + 1]
  int32_t n_routed, n_shared, T;
  int32_t m_tiles_routed, n_tiles_routed, m_tiles_shared, n_tiles_shared;  // 128-row x 256-col tiles
  int32_t m_routed, n_routed_cols, m_shared, n_shared_cols;                // output [M, N] per group
  // fp32 outputs [groups, M, N] as 3-D maps (N, M, groups), box (16, 32, 1), 64-byte
  // swizzle: routed [n_routed, m_routed, n_routed_cols], shared [n_shared, m_shared, n_shared_cols]
  CUtensorMap out_map_routed, out_map_shared;
  uint32_t* status;
  uint64_t wait_limit_ns;
};
cudaError_t launch_grouped_dw(const GemmDwArgs& a, int num_sms, cudaStream_t s);

// The down projection on CTA pairs (gemm_pair_sm100.cu; clusters of two, tcgen05
// cta_group::2): a pair computes 256 output rows by up to kGemmPairTokenTile tokens; each
// CTA stages 128 weight rows and half of the tile's token rows. Weight maps: box
// (64, 128); token maps: box (64, 128).
constexpr int kGemmPairTokenTile = 256;
// Largest number of co-resident pairs (0 when the pair kernel cannot be launched).
int down_pair_max_clusters();
cudaError_t launch_down_pair(const GemmArgs& a, int clusters, cudaStream_t s);

// The gate/up projection on CTA pairs with two M=256 chains (gemm_gateup_pair_sm100.cu):
// tiles of 256 features by up to kGemmPairTokenTile tokens; weight maps box (64, 128)
// (the one-CTA kernel's), token maps box (64, 128); n_tiles_* count 256-feature tiles.
int gateup_pair_max_clusters();
cudaError_t launch_gateup_pair(const GemmArgs& a, int clusters, cudaStream_t s);

// ---------------------------------------------------------------- errors (dsmoe_api.cu)
// Record the calling thread's last-error message (read back by dsmoe_last_error).
void note_error(const char* fmt, ...);

}  // namespace dsmoe
