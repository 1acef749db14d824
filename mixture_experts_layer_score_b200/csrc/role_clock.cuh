// role_clock.cuh -- per-CTA cycle counters of the grouped GEMMs' roles (profiling).
//
// In a build with DSMOE_ROLE_CYCLES defined (build.py --role-cycles writes it to its own
// library file), every CTA of the one-CTA grouped GEMM adds to its row of counters, per
// launch: the clock64 cycles and globaltimer nanoseconds from its start to its exit (their
// ratio is the SM clock the launch ran at); the cycles its producer waited for a free ring
// stage; the cycles its MMA thread waited for a landed stage and for a free accumulator,
// and spent in its whole tile loop; the cycles its first epilogue warp waited for a
// finished accumulator and spent in its whole tile loop; and the tiles it ran.
// dsmoe_gemm_role_cycles copies the counters out and clears them. In any other build these
// helpers compile to nothing and the kernels are unchanged.
#pragma once

#include <cstdint>

namespace dsmoe {

enum RoleSlot : int {
  kRsCycles = 0,
  kRsNanoseconds,
  kRsProducerWaitStage,
  kRsMmaWaitStage,
  kRsMmaWaitAcc,
  kRsMmaLoop,
  kRsEpiWaitAcc,
  kRsEpiLoop,
  kRsTiles,
  kRsSlots
};
constexpr int kRoleCtas = 160;   // counter rows: CTAs with blockIdx.x < kRoleCtas
// launches: 0 down, 1 gate/up (with routed groups); 2 down, 3 gate/up (shared experts
// only) of the one-CTA grouped GEMM; 4 the weight-gradient GEMM (gemm_dw_sm100.cu)
constexpr int kRoleKernels = 5;
constexpr int kRoleKindDw = 4;
constexpr int kRoleCounters = kRoleKernels * kRoleCtas * kRsSlots;

#ifdef DSMOE_ROLE_CYCLES
// An interval accumulator of clock64 cycles.
struct RoleClock {
  long long total = 0, t0 = 0;
  __device__ __forceinline__ void start() { t0 = clock64(); }
  __device__ __forceinline__ void stop() { total += clock64() - t0; }
};
__device__ __forceinline__ unsigned long long role_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#else
struct RoleClock {
  static constexpr long long total = 0;
  __device__ __forceinline__ void start() {}
  __device__ __forceinline__ void stop() {}
};
__device__ __forceinline__ unsigned long long role_ns() { return 0; }
#endif

}  // namespace dsmoe
