// tc_common.cuh -- device helpers shared by the tensor-core kernels (one
// copy per translation unit): bounded warp-wide waits, the release of TMEM
// stores to the MMA issuer, psi = 1 + elu, and the optional cycle trace.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace rehyat {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Bounded warp-wide wait: every lane polls; the result is uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(kFull, ok);
}

// Bounded wait that ignores the abort word: used to drain in-flight async
// work (TMA copies, MMAs) before a CTA releases its shared / tensor memory.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  volatile int never = 0;
  (void)mbar_wait(bar, parity, &never);
}

__device__ __forceinline__ float psi1(float x) {  // 1 + elu(x)
  return x > 0.f ? x + 1.f : ex2(x * kLog2e);
}

// Make this warp's TMEM stores visible to the MMA issuer and arrive once on
// `bar` for the whole warp.
__device__ __forceinline__ void warp_release(uint32_t bar, int lane) {
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

}  // namespace
}  // namespace rehyat

// Optional cycle tracing (build with -DREHYAT_TRACE): CTAs 0..TRACE_CTAS-1
// record clock64() at each stage of the first TRACE_TILES key tiles into
// p.trace[cta][event][tile]; without the macro the hooks compile to nothing.
#ifdef REHYAT_TRACE
namespace rehyat {
constexpr int TRACE_CTAS = 4, TRACE_EVENTS = 16, TRACE_TILES = 64;
}
#define TRACE(ev, j)                                                                       \
  do {                                                                                    \
    if (p.trace != nullptr && blockIdx.x < ::rehyat::TRACE_CTAS && (j) < ::rehyat::TRACE_TILES) \
      p.trace[(blockIdx.x * ::rehyat::TRACE_EVENTS + (ev)) * ::rehyat::TRACE_TILES + (j)] =     \
          clock64();                                                                      \
  } while (0)
#else
#define TRACE(ev, j) \
  do {               \
  } while (0)
#endif
