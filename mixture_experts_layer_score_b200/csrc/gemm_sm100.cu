// gemm_sm100.cu -- persistent grouped GEMM for the expert FFNs on the 5th-generation
// tensor cores (tcgen05 + TMEM), operands staged by TMA.
//
// Each expert FFN of the DeepSeekMoE layer (DeepSeekMoE summary, shared-expert layer
// equation; SwiGLU form noted on the "MoE: sparse activation" page) is two dense
// contractions over the rows routed to that expert:
//   gate/up:  A1[r, n] = SiLU(sum_k X[r,k] W_gate[e,n,k]) * (sum_k X[r,k] W_up[e,n,k])
//   down:     Y[r, n]  = sum_k A1[r,k] W_down[e,n,k]
// The routed experts are groups of a variable number of rows (their segment of the
// expert-contiguous slot order, read from the device-side offsets); the shared experts
// are dense groups over all T tokens that run first.
//
// Orientation: the MMA's M dimension is the weights' output features and its N
// dimension is the group's tokens, D^T[feature, token] = W[feature, :] . X[token, :]^T.
// A tile is 128 (gate/up: 128 gate + the same 128 up features; down: 2 x 128 output
// features) by at most kTok tokens, and N is the tile's token count rounded up to 16,
// so an expert's ragged last tile wastes at most 15 token columns of tensor work and
// an expert with a handful of decode tokens costs N=16, not a full tile.
//
// Token tile kTok = 128 or 256 (a template parameter chosen per launch). A 256-token
// tile stages the same weight bytes for twice the MMA work and runs the MMAs at N=256,
// where the tensor core reads fewer shared-memory bytes per MAC than at N=128; its two
// chains then fill all 512 TMEM columns, so the next tile's MMAs wait for this tile's
// epilogue. It pays where the K loop is long (d >= 4096) and experts hold a few hundred
// rows; elsewhere the 128-token tile with two accumulators is faster.
//
// One CTA per SM, 320 threads in three roles:
//   warp 0     TMA producer: per 64-wide K block a 256x64 weight tile (two 128-row
//              halves) and a kTok x 64 token tile through a ring of 48 KB (4 stages,
//              128-token tiles) or 64 KB (3 stages, 256-token tiles) stages.
//   warp 1     allocates 512 TMEM columns (accumulators of two chains of kTok columns)
//              and issues tcgen05.mma (M=128, N=16..kTok, K=16) from one thread, two
//              chains (one per weight half) sharing the token tile; commits free ring
//              stages and publish finished accumulators.
//   warps 2-9  epilogue: warps 2+q and 6+q read TMEM lanes [32q, 32q+32) (thread f of
//              lane f owns output feature f of both chains) for alternate 32-token
//              chunks. Per chunk: tcgen05.ld of both chains (the next chunk's loads are
//              issued before this one's last rows are stored), SiLU(gate)*up (or the
//              residual) in fp32,
//              a 32 x 32 transpose through shared memory (bf16; fp32 in 16-token halves
//              for the shared experts' fp32 sums) and 16-byte stores along output rows.
// Every wait is bounded (wait_limit_ns); a role that gives up raises a CTA-wide abort
// flag and a bit of the device status word, the CTA lets in-flight TMA loads and MMAs
// finish (a wait bounded by at least one second, whatever the caller's limit), frees its
// TMEM and returns.
#include "grouped_tiles.cuh"
#include "role_clock.cuh"
#include "sm100_ptx.cuh"

namespace dsmoe {

#ifdef DSMOE_ROLE_CYCLES
__device__ unsigned long long g_role_cycles[kRoleKindDw][kRoleCtas][kRsSlots];
#endif

namespace {
// Adds v to this CTA's counter `slot` of kernel `k` (profiling builds only).
__device__ __forceinline__ void role_add(int k, int slot, long long v) {
#ifdef DSMOE_ROLE_CYCLES
  if (blockIdx.x < kRoleCtas) atomicAdd(&g_role_cycles[k][blockIdx.x][slot], static_cast<unsigned long long>(v));
#else
  (void)k;
  (void)slot;
  (void)v;
#endif
}

constexpr int kBK = 64;         // K per ring stage (one 128-byte swizzled row of bf16)
constexpr int kFeat = 128;      // output features per MMA chain (the MMA's M, TMEM lanes)
constexpr int kMmaK = 16;       // K of each bf16 tcgen05.mma
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWBytes = 2 * kFeat * kBK * 2;  // 32 KB: two 128-row weight halves
constexpr uint32_t kStgRow = 40;                   // bf16 staging row: 32 values + 8 pad (80 B)
constexpr uint32_t kStgRowF = 33;                  // fp32 staging row: 32 values + 1 pad
constexpr uint32_t kStgBytes = 32 * kStgRow * 2;   // per epilogue warp: 32 bf16 rows or 16 fp32 rows
static_assert(16 * kStgRowF * 4 <= kStgBytes, "fp32 half-chunk staging fits the bf16 chunk's");

template <int kTok>
struct Geo {
  static constexpr uint32_t kChainCols = kTok;
  static constexpr uint32_t kAccCols = 2 * kChainCols;
  static constexpr int kBufs = static_cast<int>(kTmemCols / kAccCols);
  static constexpr int kStages = kTok == 256 ? 3 : 4;
  static constexpr uint32_t kXBytes = kTok * kBK * 2;
  static constexpr uint32_t kStageBytes = kWBytes + kXBytes;
  static constexpr uint32_t kOffW = 0;
  static constexpr uint32_t kOffX = kOffW + kStages * kWBytes;
  static constexpr uint32_t kOffBars = kOffX + kStages * kXBytes;
  static constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1;
  static constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
  static constexpr uint32_t kOffTiles = kOffMisc + 16;
  static constexpr uint32_t kOffEpi = (kOffTiles + (kGemmMaxGroups + 1) * 4 + 15) & ~15u;
  static constexpr uint32_t kSmemUsed = kOffEpi + kEpiWarps * kStgBytes;
  static constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack to align the ring to 1024 bytes
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kBufs >= 1 && kBufs <= 2 && kTok % 32 == 0 && kTok <= 256, "tile geometry");
};

template <bool kSwiGLU, int kTok>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs a) {
  using G_ = Geo<kTok>;
  RoleClock rc_kernel;
  rc_kernel.start();
  const unsigned long long rc_ns0 = role_ns();
  const int rk = (kSwiGLU ? 1 : 0) + (a.n_routed == 0 ? 2 : 0);  // role counter set
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* sW = base + G_::kOffW;
  uint8_t* sX = base + G_::kOffX;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + G_::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + G_::kStages;
  uint64_t* acc_full = bars + 2 * G_::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + G_::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + G_::kOffMisc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + G_::kOffMisc + 8);
  int32_t* tile_start = reinterpret_cast<int32_t*>(base + G_::kOffTiles);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.n_shared_groups + a.n_routed;

  tile_counts<kTok>(a, tile_start, G);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *never_flag = 0;
    for (int s = 0; s < G_::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);  // one lane of each epilogue warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 0) tile_scan(tile_start, G, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[G];

  uint32_t issued_mask = 0, issued_parity = 0;  // producer bookkeeping for the abort drain

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&a.a_routed);
      tma_prefetch_desc(&a.b0_routed);
      if (kSwiGLU) tma_prefetch_desc(&a.b1_routed);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      RoleClock rc_wait;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
        const CUtensorMap* tx = t.shared ? &a.a_shared : &a.a_routed;
        const CUtensorMap* tw0 = t.shared ? &a.b0_shared : &a.b0_routed;
        const CUtensorMap* tw1 = t.shared ? &a.b1_shared : &a.b1_routed;
        const int kb_per = t.shared ? a.kb_per_b_expert_shared : t.kb_n;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          rc_wait.start();
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          rc_wait.stop();
          mbar_arrive_expect_tx(&full[stage], G_::kStageBytes);
          const int be = t.expert + kb / kb_per;
          const int bk = (kb % kb_per) * kBK;
          uint8_t* w = sW + stage * kWBytes;
          if (kSwiGLU) {  // [128 gate rows | the same 128 up rows]
            tma_load_3d(w, tw0, &full[stage], bk, t.n_blk * kFeat, be);
            tma_load_3d(w + kWBytes / 2, tw1, &full[stage], bk, t.n_blk * kFeat, be);
          } else {        // 256 consecutive output rows
            tma_load_3d(w, tw0, &full[stage], bk, t.n_blk * 2 * kFeat, be);
          }
          tma_load_2d(sX + stage * G_::kXBytes, tx, &full[stage], kb * kBK, t.row0);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == G_::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeoutProducer);
      }
      role_add(rk, kRsProducerWaitStage, rc_wait.total);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      RoleClock rc_loop, rc_stage, rc_acc;
      rc_loop.start();
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
        const int n_mma = (t.m_valid + 15) & ~15;  // tokens, rounded up to the MMA's N step
        const uint32_t idesc = idesc_bf16_f32(kFeat, n_mma);
        const int acc = it % G_::kBufs;
        rc_acc.start();
        if (!mbar_wait_bounded(&acc_empty[acc], ((it / G_::kBufs) & 1) ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        rc_acc.stop();
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * G_::kAccCols;
        for (int kb = 0; kb < t.kb_n; ++kb) {
          rc_stage.start();
          if (!mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          rc_stage.stop();
          tc_fence_after();
          const uint64_t w0 = smem_desc_kmajor_sw128(smem_addr(sW + stage * kWBytes));
          const uint64_t w1 = smem_desc_kmajor_sw128(smem_addr(sW + stage * kWBytes + kWBytes / 2));
          const uint64_t xd = smem_desc_kmajor_sw128(smem_addr(sX + stage * G_::kXBytes));
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            const uint64_t dk = static_cast<uint64_t>(2 * k);
            const uint32_t accum = (kb | k) ? 1u : 0u;
            mma_bf16_ss(d0, w0 + dk, xd + dk, idesc, accum);
            mma_bf16_ss(d0 + G_::kChainCols, w1 + dk, xd + dk, idesc, accum);
          }
          mma_commit(&empty[stage]);
          if (++stage == G_::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeoutMma);
      }
      rc_loop.stop();
      role_add(rk, kRsMmaWaitStage, rc_stage.total);
      role_add(rk, kRsMmaWaitAcc, rc_acc.total);
      role_add(rk, kRsMmaLoop, rc_loop.total);
      role_add(rk, kRsTiles, it);
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes [32q, 32q+32), q = w % 4: thread f of lane f holds output
    // feature f of both chains. It takes the tile's 32-token chunks c with
    // c % 2 == (w - 2) / 4, transposes each 32 features x 32 tokens block through its
    // staging area, and lane L stores 8 consecutive features (16 B of bf16, 32 B of fp32)
    // of token row L/4 + 8i: four lanes cover the warp's 32-feature segment of a row.
    const int q = warp & 3, half = (warp - 2) >> 2;
    uint8_t* stg_raw = base + G_::kOffEpi + (warp - 2) * kStgBytes;
    uint16_t* stg = reinterpret_cast<uint16_t*>(stg_raw);  // [32 tokens][kStgRow] bf16
    float* stgf = reinterpret_cast<float*>(stg_raw);       // [16 tokens][kStgRowF] fp32
    const int rr = lane >> 2, cc = (lane & 3) * 8;  // read-out: row (plus 8i), first feature
    int it = 0;
    RoleClock rc_loop, rc_acc;
    rc_loop.start();
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const Tile t = decode_tile<kTok>(a, tile_start, G, tile);
      const int acc = it % G_::kBufs;
      rc_acc.start();
      if (!mbar_wait_warp_sleepy(&acc_full[acc], (it / G_::kBufs) & 1, a.wait_limit_ns, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(a.status, kStatusTimeoutEpilogue);
        }
        break;
      }
      rc_acc.stop();
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * G_::kAccCols;
      const int n_valid = t.shared ? a.n_valid_shared : a.n_valid_routed;
      const int64_t ld = t.shared ? a.ld_shared : a.ld_routed;
      const bool f32_out = !kSwiGLU && t.shared && a.out_shared_f32 != nullptr;
      // the backward pass's saved pre-activations: a (chain 0) and b (chain 1) as bf16
      bf16* save = kSwiGLU ? (t.shared ? a.save_ab_shared : a.save_ab_routed) : nullptr;
      // chains whose values leave this tile: gate/up gives one output chain, down two
      constexpr int kOut = kSwiGLU ? 1 : 2;
      const int n_chunks = (t.m_valid + 31) >> 5;
      uint32_t v0[32], v1[32];  // this chunk's accumulator columns of the two chains
      if (half < n_chunks) {
        tmem_ld16(tb + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(&v0[0]));
        tmem_ld16(tb + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(&v0[16]));
        tmem_ld16(tb + G_::kChainCols + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(&v1[0]));
        tmem_ld16(tb + G_::kChainCols + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(&v1[16]));
      }
      tmem_wait_ld();
#pragma unroll 1
      for (int ch_i = half; ch_i < n_chunks; ch_i += 2) {
        const int c0 = 32 * ch_i;
        // Once the last staging write has read v0 / v1, the next chunk's columns are
        // loaded into them while this chunk's rows are stored.
        const bool more = ch_i + 2 < n_chunks;
        auto load_next = [&]() {
          if (more) {
            const uint32_t cn = static_cast<uint32_t>(c0 + 64);
            tmem_ld16(tb + cn, *reinterpret_cast<uint32_t(*)[16]>(&v0[0]));
            tmem_ld16(tb + cn + 16, *reinterpret_cast<uint32_t(*)[16]>(&v0[16]));
            tmem_ld16(tb + G_::kChainCols + cn, *reinterpret_cast<uint32_t(*)[16]>(&v1[0]));
            tmem_ld16(tb + G_::kChainCols + cn + 16, *reinterpret_cast<uint32_t(*)[16]>(&v1[16]));
          }
        };
        if (kSwiGLU && save) {
          const int width = t.shared ? a.shared_col_stride : a.n_valid_routed;  // F_s or F
          const int64_t lds = 2 * (t.shared ? a.ld_shared : a.ld_routed);
          const int64_t col0 = t.shared ? static_cast<int64_t>(t.group) * 2 * width : 0;
          const int feat = t.n_blk * kFeat + q * 32 + cc;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              stg[j * kStgRow + lane] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(ch == 0 ? v0[j] : v1[j])));
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = rr + 8 * i;
              if (feat < width && c0 + row < t.m_valid)
                *reinterpret_cast<uint4*>(save + static_cast<int64_t>(t.row0 + c0 + row) * lds + col0 +
                                          ch * width + feat) =
                    *reinterpret_cast<const uint4*>(stg + row * kStgRow + cc);
            }
            __syncwarp();
          }
        }
#pragma unroll
        for (int ch = 0; ch < kOut; ++ch) {
          const int feat = (kSwiGLU ? t.n_blk * kFeat : t.n_blk * 2 * kFeat + ch * kFeat) + q * 32 + cc;
          const bool ok_f = feat < n_valid;  // n_valid is a multiple of 64, feat of 8
          if (f32_out) {
            // the shared experts' sum plus the residual x, in fp32: two 16-token halves
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                stgf[j * kStgRowF + lane] = __uint_as_float(ch == 0 ? v0[16 * hh + j] : v1[16 * hh + j]);
              __syncwarp();
              if (ch == kOut - 1 && hh == 1) load_next();
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const int row = rr + 8 * i, tok = c0 + 16 * hh + row;
                if (ok_f && tok < t.m_valid) {
                  const float* src = stgf + row * kStgRowF + cc;
                  const int64_t o = static_cast<int64_t>(t.row0 + tok) * ld + feat;
                  const uint4 rv = *reinterpret_cast<const uint4*>(a.residual + o);
                  const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
                  float out8[8];
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const float2 xr = unpack_bf16x2(rw[k]);
                    out8[2 * k] = src[2 * k] + xr.x;
                    out8[2 * k + 1] = src[2 * k + 1] + xr.y;
                  }
                  float4* dst = reinterpret_cast<float4*>(a.out_shared_f32 + o);
                  dst[0] = make_float4(out8[0], out8[1], out8[2], out8[3]);
                  dst[1] = make_float4(out8[4], out8[5], out8[6], out8[7]);
                }
              }
              __syncwarp();
            }
          } else {
            // stage: row = token (c0 + j), column = this lane's feature, rounded to bf16
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float val;
              if (kSwiGLU) {
                const float g = __uint_as_float(v0[j]);
                val = __fdividef(g, 1.0f + __expf(-g)) * __uint_as_float(v1[j]);  // SiLU(g) * u
              } else {
                val = __uint_as_float(ch == 0 ? v0[j] : v1[j]);
              }
              stg[j * kStgRow + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
            }
            __syncwarp();
            if (ch == kOut - 1) load_next();
            bf16* obase = t.shared ? a.out_shared + static_cast<int64_t>(t.group) * a.shared_col_stride
                                   : a.out_routed;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = rr + 8 * i;
              if (ok_f && c0 + row < t.m_valid)
                *reinterpret_cast<uint4*>(obase + static_cast<int64_t>(t.row0 + c0 + row) * ld + feat) =
                    *reinterpret_cast<const uint4*>(stg + row * kStgRow + cc);
            }
            __syncwarp();
          }
        }
        tmem_wait_ld();  // the next chunk's columns have landed in v0 / v1
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
    rc_loop.stop();
    if (warp == 2 && lane == 0) {
      role_add(rk, kRsEpiWaitAcc, rc_acc.total);
      role_add(rk, kRsEpiLoop, rc_loop.total);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // let every copy and MMA this CTA started finish before its memory is released
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < G_::kStages; ++s)
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
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {
    rc_kernel.stop();
    role_add(rk, kRsCycles, rc_kernel.total);
    role_add(rk, kRsNanoseconds, static_cast<long long>(role_ns() - rc_ns0));
  }
}
}  // namespace

namespace {
template <bool kSwiGLU, int kTok>
cudaError_t launch_one(const GemmArgs& a, int grid, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kSwiGLU, kTok>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Geo<kTok>::kSmemBytes));
  if (e != cudaSuccess) return e;
  grouped_gemm_kernel<kSwiGLU, kTok><<<grid, kThreads, Geo<kTok>::kSmemBytes, s>>>(a);
  return cudaGetLastError();
}
}  // namespace

bool read_role_cycles(unsigned long long* host, cudaError_t* err) {
#ifdef DSMOE_ROLE_CYCLES
  static unsigned long long zeros[kRoleCounters];
  *err = cudaMemcpyFromSymbol(host, g_role_cycles, sizeof(g_role_cycles));
  if (*err == cudaSuccess) *err = cudaMemcpyToSymbol(g_role_cycles, zeros, sizeof(g_role_cycles));
  if (*err == cudaSuccess) read_role_cycles_dw(host + kRoleKindDw * kRoleCtas * kRsSlots, err);
  return true;
#else
  (void)host;
  *err = cudaSuccess;
  return false;
#endif
}

cudaError_t launch_grouped_gemm(bool swiglu, int tok, const GemmArgs& a, int grid, cudaStream_t s) {
  if (a.n_shared_groups + a.n_routed > kGemmMaxGroups) return cudaErrorInvalidValue;
  if (grid < 1) grid = 1;
  if (tok == 256 && swiglu) return launch_one<true, 256>(a, grid, s);
  if (tok != kGemmTokenTile) return cudaErrorInvalidValue;
  return swiglu ? launch_one<true, kGemmTokenTile>(a, grid, s) : launch_one<false, kGemmTokenTile>(a, grid, s);
}

}  // namespace dsmoe
