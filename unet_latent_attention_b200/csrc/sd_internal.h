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

// Streaming-multiprocessor count of the current device (cached per device).
int sm_count();

}  // namespace sd
