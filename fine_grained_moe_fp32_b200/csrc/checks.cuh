// Device-side bounds checks of the MOE_CHECKS build.
//
// Built with -DMOE_CHECKS=1 (libmoe_b200_checks.so), MOE_CHECK(cond) tests an
// index against the buffer it addresses; a false condition records
// DEV_BOUNDS in the per-device status word (the host reads it as
// MOE_ERR_BOUNDS) and the caller skips the access, so the kernel neither
// faults nor traps and the context stays usable.  In the normal build the
// macro is the constant true and costs nothing.
//
// The status word lives in moe_api.cu.  Without relocatable device code a
// translation unit cannot name another unit's device variable, so every unit
// that includes this header holds its own copy of the pointer, set once per
// device by its MOE_CHECKS_UNIT(name) host function (called by the
// library's device set-up).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "moe_internal.h"

#ifdef MOE_CHECKS
namespace moe {
namespace checks {
static __device__ unsigned int* g_status = nullptr;
__device__ __forceinline__ bool ok(bool cond) {
  if (!cond && g_status != nullptr) atomicCAS(g_status, 0u, (unsigned)DEV_BOUNDS);
  return cond;
}
}  // namespace checks
}  // namespace moe
#define MOE_CHECK(cond) (::moe::checks::ok(cond))
#define MOE_CHECKS_UNIT(name)                                                 \
  namespace moe {                                                             \
  cudaError_t checks_init_##name(unsigned int* status) {                      \
    return cudaMemcpyToSymbol(checks::g_status, &status, sizeof(status));     \
  }                                                                           \
  }
#else
#define MOE_CHECK(cond) true
#define MOE_CHECKS_UNIT(name)
#endif
