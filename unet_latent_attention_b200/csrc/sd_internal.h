// Host-side helpers shared by the library's translation units (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sd_kernels.h"

namespace sd {

// Records a message for sd_last_error() on the calling thread and returns `st`.
sd_status fail(sd_status st, const char* fmt, ...);

// Converts a CUDA error into SD_ERR_CUDA (with the CUDA text); cudaSuccess gives SD_OK.
sd_status cuda_check(cudaError_t err, const char* where);

// Device address of the current device's status word (kernels atomicOr error bits into it).
// Returns nullptr and records the CUDA error if the symbol cannot be resolved.
unsigned int* device_status_word();

// Bits of the device status word.
enum : unsigned int { kDevErrTimeout = 1u };

// True if [a, a+na) and [b, b+nb) (bytes) intersect.
inline bool overlaps(const void* a, int64_t na, const void* b, int64_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return na > 0 && nb > 0 && pa < pb + static_cast<uintptr_t>(nb) && pb < pa + static_cast<uintptr_t>(na);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The calling thread's current CUDA context (as an opaque handle), so that per-device caches of
// device addresses can notice a context that was destroyed and created again.
sd_status current_context(void** ctx);

// Streaming-multiprocessor count of the current device (cached per device).
int sm_count();

// Clears the attention hand-off workspace of the current device on `s` (after a kernel gave up a
// bounded wait, its flags may be left set).
sd_status attention_clear_handoff(cudaStream_t s);

// Programmatic dependent launch. Every kernel of the library is launched so that its CTAs may start
// while the kernel before it on the stream is still finishing. Each kernel executes grid_dep_wait()
// before its first global-memory access: that returns once the previous kernel has completed and its
// memory operations are visible, so stream order is kept for all data. grid_dep_launch() lets the
// next kernel on the stream start its own launch early. Both are no-ops when the launch carries no
// programmatic dependency.
#ifndef SD_PDL
#define SD_PDL 1
#endif
#ifdef __CUDACC__
__device__ __forceinline__ void grid_dep_wait() {
  if (SD_PDL) asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  if (SD_PDL) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif
// Writes the programmatic-serialization launch attribute into `attr` (if enabled) and returns the
// number of attributes written.
inline unsigned int pdl_attr(cudaLaunchAttribute* attr) {
  if (!SD_PDL) return 0;
  attr->id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr->val.programmaticStreamSerializationAllowed = 1;
  return 1;
}

}  // namespace sd
