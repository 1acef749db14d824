// gemm_dw_sm100.cu -- the experts' weight gradients on the 5th-generation tensor cores.
//
// For an expert FFN y = W_down m, m = SiLU(a) * b, a = W_gate u, b = W_up u (DeepSeekMoE
// summary, shared-expert layer equation; SwiGLU form noted on the "MoE: sparse
// activation" page), summed over the rows r the expert applies to:
//   dW_down = sum_r dy_r m_r^T,   dW_gate = sum_r da_r u_r^T,   dW_up = sum_r db_r u_r^T
// i.e. D[i, j] = sum_r A[r, i] B[r, j] with the reduction over token rows, which are
// contiguous in both operands' [rows, cols] layouts: both MMA operands are MN-major, and
// each routed expert's K range is its segment of the slot order (ragged), each shared
// expert's all T tokens.
//
// One CTA per SM, 320 threads: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// warps 2-9 epilogue (each stages 32-row x 16-column fp32 halves of the accumulator in two
// 2 KB buffers of its own shared memory and writes them to the output with bulk tensor
// stores of whole 64-byte row segments). A tile is 128 output rows by 256 output columns, one M=128, N=256 chain (per
// MAC it reads a quarter fewer shared-memory bytes than two M=128, N=128 chains, whose
// operand reads alone fill the shared memory's bandwidth); per 64-row K block the
// producer stages A (128 columns of the A buffer) and B (256 columns of the B buffer)
// through 3-D views (64, rows, cols / 64) that land as 64-element MN-major swizzle-128B
// atoms 8 KB apart. A K block that runs past the group's last row holds rows of the next
// group (or the buffer's zero fill): only its 16-row MMA steps that hold valid rows are
// issued, and the MMA warp zeroes the invalid rows of the last of them in the A
// operand's shared memory (making the stores visible to the tensor core) first.
// A group with no rows gets a zero tile. Output fp32, D row-major per group.
// Every wait is bounded; a role that gives up raises the abort flag and a status bit, the
// CTA waits (at least one second) for its copies and MMAs in flight, frees TMEM, returns.
#include "kernels.h"
#include "role_clock.cuh"
#include "sm100_ptx.cuh"

namespace dsmoe {

#ifdef DSMOE_ROLE_CYCLES
__device__ unsigned long long g_role_cycles_dw[kRoleCtas][kRsSlots];
#endif

namespace {
__device__ __forceinline__ void role_add_dw(int slot, long long v) {
#ifdef DSMOE_ROLE_CYCLES
  if (blockIdx.x < kRoleCtas) atomicAdd(&g_role_cycles_dw[blockIdx.x][slot], static_cast<unsigned long long>(v));
#else
  (void)slot;
  (void)v;
#endif
}

constexpr int kBK = 64;
constexpr int kFeat = 128;                          // output rows per tile (the MMA's M)
constexpr int kMmaK = 16;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr int kN = 256;                             // output columns per tile (the MMA's N)
constexpr int kStages = 4;
constexpr uint32_t kABytes = kFeat * kBK * 2;      // 16 KB: 128 output rows x 64 K rows
constexpr uint32_t kBBytes = kN * kBK * 2;         // 32 KB: 256 output columns x 64 K rows
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kAccCols = kN;
constexpr int kBufs = 2;
constexpr uint32_t kAtom = kBK * 128;              // one 64-element atom column of a stage: 8 KB
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kStgBytes = 32 * 32 * 4;        // one warp's two 32 x 16 fp32 staging buffers
constexpr uint32_t kOffStg = kOffB + kStages * kBBytes;
constexpr uint32_t kOffBars = kOffStg + kEpiWarps * kStgBytes;
constexpr uint32_t kNumBars = 2 * kStages + 2 * kBufs + 1;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr size_t kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(kAtom >> 4) << 16;  // leading byte offset: next 64 MN elements
  d |= static_cast<uint64_t>(1024 >> 4) << 32;   // stride byte offset: next 8 K rows
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void tma_load_3d_view(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t row,
                                                 int32_t atom) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(0), "r"(row), "r"(atom)
      : "memory");
}

// Bulk tensor store of one staged half: box (16 fp32 columns, 32 rows, 1 group) of a 3-D
// map (columns, rows, groups) with the 64-byte swizzle; rows past a group's end are not
// written (the map's row extent is the group's).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int32_t col, int32_t row,
                                             int32_t group) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(col), "r"(row), "r"(group)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed copy but the most recent one has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_but_last() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct DwTile {
  int group, shared, row0, rows, m_blk, n_blk;
};

__device__ __forceinline__ DwTile dw_decode(const GemmDwArgs& a, int tile) {
  DwTile t;
  const int tiles_s = a.m_tiles_shared * a.n_tiles_shared, tiles_r = a.m_tiles_routed * a.n_tiles_routed;
  int local, n_tiles;
  if (tile < a.n_shared * tiles_s) {
    t.shared = 1;
    t.group = tile / tiles_s;
    local = tile - t.group * tiles_s;
    n_tiles = a.n_tiles_shared;
    t.row0 = 0;
    t.rows = a.T;
  } else {
    t.shared = 0;
    const int r = tile - a.n_shared * tiles_s;
    t.group = r / tiles_r;
    local = r - t.group * tiles_r;
    n_tiles = a.n_tiles_routed;
    t.row0 = __ldg(a.offsets + t.group);
    t.rows = max(__ldg(a.offsets + t.group + 1) - t.row0, 0);
  }
  t.m_blk = local / n_tiles;
  t.n_blk = local % n_tiles;
  return t;
}

__global__ void __launch_bounds__(kThreads, 1) grouped_dw_kernel(const __grid_constant__ GemmDwArgs a) {
  RoleClock rc_kernel;
  rc_kernel.start();
  const unsigned long long rc_ns0 = role_ns();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* base = smem_raw + pad;
  uint8_t* sA = base + kOffA;
  uint8_t* sB = base + kOffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + kBufs;
  uint64_t* drain = acc_empty + kBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.n_shared * a.m_tiles_shared * a.n_tiles_shared +
                    a.n_routed * a.m_tiles_routed * a.n_tiles_routed;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *never_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kBufs; ++i) {
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  uint32_t issued_mask = 0, issued_parity = 0;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      RoleClock rc_wait;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const DwTile t = dw_decode(a, tile);
        const CUtensorMap* ta = t.shared ? &a.a_shared : &a.a_routed;
        const CUtensorMap* tb = t.shared ? &a.b_shared : &a.b_routed;
        const int a_atom = (t.shared ? a.a_atom0_shared + t.group * a.a_atom_step_shared : a.a_atom0_routed) +
                           t.m_blk * (kFeat / 64);
        const int b_atom = (t.shared ? a.b_atom0_shared + t.group * a.b_atom_step_shared : a.b_atom0_routed) +
                           t.n_blk * (kN / 64);
        const int kb_n = (t.rows + kBK - 1) / kBK;
        for (int kb = 0; kb < kb_n; ++kb) {
          rc_wait.start();
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          rc_wait.stop();
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_3d_view(sA + stage * kABytes, ta, &full[stage], t.row0 + kb * kBK, a_atom);
          tma_load_3d_view(sB + stage * kBBytes, tb, &full[stage], t.row0 + kb * kBK, b_atom);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeoutProducer);
      }
      role_add_dw(kRsProducerWaitStage, rc_wait.total);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------- MMA issuer
    // The whole warp follows the loop: on a K block that runs past the group's rows it
    // zeroes those rows of the A operand first; lane 0 issues the MMAs.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int it = 0;
    const uint32_t idesc = idesc_bf16_f32(kFeat, kN) | (1u << 15) | (1u << 16);  // A and B MN-major
    RoleClock rc_loop, rc_stage, rc_acc;
    rc_loop.start();
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
      const DwTile t = dw_decode(a, tile);
      const int kb_n = (t.rows + kBK - 1) / kBK;
      const int acc = it % kBufs;
      rc_acc.start();
      if (!mbar_wait_warp(&acc_empty[acc], ((it / kBufs) & 1) ^ 1u, a.wait_limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      rc_acc.stop();
      tc_fence_after();
      const uint32_t d0 = tmem_base + acc * kAccCols;
      for (int kb = 0; kb < kb_n; ++kb) {
        rc_stage.start();
        if (!mbar_wait_warp(&full[stage], phase, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        rc_stage.stop();
        tc_fence_after();
        const int valid = t.rows - kb * kBK;  // rows of this K block inside the group (> 0)
        // K steps of 16 rows that hold any of them; the rows of the last such step past the
        // group's end (fewer than 16) are zeroed in the A operand, whose 2 atom columns of
        // 128-byte rows cancel those rows' products (B's rows there are finite: the next
        // group's data or the copy's zero fill): lane l clears the 16-byte chunk l % 8 of
        // rows r + l / 8
        const int ksteps = valid >= kBK ? kBK / kMmaK : (valid + kMmaK - 1) / kMmaK;
        const int z1 = ksteps * kMmaK;
        if (valid < z1) {
          const int q = lane & 7;
          for (int col = 0; col < 2; ++col) {
            uint8_t* atom = sA + stage * kABytes + col * kAtom;
            for (int r = valid + (lane >> 3); r < z1; r += 4)
              *reinterpret_cast<uint4*>(atom + r * 128 + q * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t abase = smem_addr(sA + stage * kABytes), bbase = smem_addr(sB + stage * kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            if (k >= ksteps) break;
            const uint32_t accum = (kb | k) ? 1u : 0u;
            const uint32_t koff = static_cast<uint32_t>(k) * kMmaK * 128;
            mma_bf16_ss(d0, desc_mn_sw128(abase + koff), desc_mn_sw128(bbase + koff), idesc, accum);
          }
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(&acc_full[acc]);  // with no K block: arrives at once
      __syncwarp();
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(a.status, kStatusTimeoutMma);
    }
    rc_loop.stop();
    if (lane == 0) {
      role_add_dw(kRsMmaWaitStage, rc_stage.total);
      role_add_dw(kRsMmaWaitAcc, rc_acc.total);
      role_add_dw(kRsMmaLoop, rc_loop.total);
      role_add_dw(kRsTiles, it);
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes [32q, 32q+32), q = w % 4: thread l of lane l holds output row
    // 32q + l, 32 consecutive fp32 columns per chunk. Each 16-column half of the chunk goes
    // into one of the warp's two staging buffers (a quarter-warp's stores hit all 32 banks
    // once) and lane 0 stores it with one bulk tensor copy, alternating buffers, so a
    // buffer waits only for the copy before the last. Warps 2+q and 6+q take alternate
    // chunks of the tile's kN/32; the next chunk's TMEM reads are issued before this chunk
    // is staged. (One 4 KB buffer of whole 32-column chunks, each waiting for the previous
    // copy, ran the V3 weight gradients 1.5% slower.)
    const int q = warp & 3, half = (warp - 2) >> 2;
    constexpr int kChunks = kN / 32;
    const uint32_t stg = smem_addr(base + kOffStg + (warp - 2) * kStgBytes);
    uint32_t sc = 0;  // staged halves so far: the buffer of the next one is sc % 2
    int it = 0;
    RoleClock rc_loop, rc_acc;
    rc_loop.start();
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const DwTile t = dw_decode(a, tile);
      const int acc = it % kBufs;
      rc_acc.start();
      if (!mbar_wait_warp_sleepy(&acc_full[acc], (it / kBufs) & 1, a.wait_limit_ns, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(a.status, kStatusTimeoutEpilogue);
        }
        break;
      }
      rc_acc.stop();
      tc_fence_after();
      const bool empty_group = t.rows == 0;
      const int M = t.shared ? a.m_shared : a.m_routed, N = t.shared ? a.n_shared_cols : a.n_routed_cols;
      const CUtensorMap* omap = t.shared ? &a.out_map_shared : &a.out_map_routed;
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      uint32_t v[32];
      auto load = [&](int idx) {
        const uint32_t col = static_cast<uint32_t>(idx * 32);
        tmem_ld16(tb + col, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
        tmem_ld16(tb + col + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
      };
      load(half);
      tmem_wait_ld();
#pragma unroll 1
      for (int idx = half; idx < kChunks; idx += 2) {
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = empty_group ? 0u : v[j];
        if (idx + 2 < kChunks) load(idx + 2);  // lands while this chunk is stored
        const int row0 = t.m_blk * kFeat + q * 32;  // M and N are multiples of 64:
        const int n = t.n_blk * kN + idx * 32;      // a chunk is all inside or all out
        if (row0 < M && n < N) {
          // two 16-column halves, each staged in one of the warp's two 2 KB buffers (64-byte
          // rows, 64-byte swizzle: 16-byte unit c of row r at unit c ^ ((r / 2) % 4)) and
          // stored by its own copy; a buffer is rewritten once the copy before the last has
          // read it
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t buf = stg + (sc & 1u) * (kStgBytes / 2);
            ++sc;
            if (lane == 0) bulk_wait_read_but_last();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 4; ++c)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)),
                           "r"(r[16 * hf + 4 * c]), "r"(r[16 * hf + 4 * c + 1]), "r"(r[16 * hf + 4 * c + 2]),
                           "r"(r[16 * hf + 4 * c + 3])
                           : "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(omap, buf, n + 16 * hf, row0, t.group);
              bulk_commit();
            }
          }
        }
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
    if (lane == 0) bulk_wait_all();  // the CTA's shared memory outlives every copy from it
    __syncwarp();
    rc_loop.stop();
    if (warp == 2 && lane == 0) {
      role_add_dw(kRsEpiWaitAcc, rc_acc.total);
      role_add_dw(kRsEpiLoop, rc_loop.total);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < kStages; ++s)
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
    role_add_dw(kRsCycles, rc_kernel.total);
    role_add_dw(kRsNanoseconds, static_cast<long long>(role_ns() - rc_ns0));
  }
}
}  // namespace

bool read_role_cycles_dw(unsigned long long* host, cudaError_t* err) {
#ifdef DSMOE_ROLE_CYCLES
  static unsigned long long zeros[kRoleCtas * kRsSlots];
  *err = cudaMemcpyFromSymbol(host, g_role_cycles_dw, sizeof(zeros));
  if (*err == cudaSuccess) *err = cudaMemcpyToSymbol(g_role_cycles_dw, zeros, sizeof(zeros));
  return true;
#else
  (void)host;
  *err = cudaSuccess;
  return false;
#endif
}

cudaError_t launch_grouped_dw(const GemmDwArgs& a, int num_sms, cudaStream_t s) {
  if (a.n_routed > kGemmMaxGroups) return cudaErrorInvalidValue;
  const int64_t total = static_cast<int64_t>(a.n_shared) * a.m_tiles_shared * a.n_tiles_shared +
                        static_cast<int64_t>(a.n_routed) * a.m_tiles_routed * a.n_tiles_routed;
  if (total <= 0) return cudaSuccess;
  const int grid = static_cast<int>(total < num_sms ? total : num_sms);
  cudaError_t e = cudaFuncSetAttribute(grouped_dw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  grouped_dw_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dsmoe
