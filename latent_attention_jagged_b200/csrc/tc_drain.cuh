// Abort-path drain of a producer's TMA ring (sm_100a).
#pragma once

#include "tc_common.cuh"

namespace llatte {
namespace tc {

// After an abort, a producer waits for the loads of its last min(stages,
// issued) ring issues: issue i went to stage i % stages and completes that
// stage's full barrier in the phase of parity (i / stages) & 1; the last
// issue of a stage has no later phase, so the parity is unambiguous.  Then
// no TMA write lands in shared memory after the CTA has exited.  The waits
// ignore the abort flag and are bounded by kDrainTimeoutNs each (a stage
// whose bytes the other CTA of a pair never sent ends its wait there).
constexpr uint64_t kDrainTimeoutNs = 100000000ull;   // 100 ms
__device__ __forceinline__ void drain_ring(uint64_t* full, uint32_t stages, uint32_t issued,
                                           int32_t* status) {
  for (uint32_t k = 0; k < stages && k < issued; ++k) {
    const uint32_t i = issued - 1 - k;
    int never = 0;
    mbar_wait(&full[i % stages], (i / stages) & 1, &never, status, kDrainTimeoutNs);
  }
}

}  // namespace tc
}  // namespace llatte
