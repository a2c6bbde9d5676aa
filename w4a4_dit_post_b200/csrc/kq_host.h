// Host-side helpers shared by the C-ABI entry points: argument checks, the
// thread-local error message and cached per-device properties.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kq.h"

namespace kq {

// Record a failure message for kq_last_error() on this thread; returns status.
int fail(int status, const char* fmt, ...);

// Turn a CUDA error into KQ_ERR_CUDA with the CUDA message.
int cuda_fail(cudaError_t err, const char* what);

// Check the result of a kernel launch.
int check_launch(const char* what);

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Multiprocessor count of the current device (cached per device).
int sm_count(int* out);

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Device address of the per-device status word (defined in kq_stream.cu),
// for kernels compiled in other translation units; cached per device.
int device_status_address(unsigned int** out);

// Common checks of (M, d): M >= 0, d > 0, d % 32 == 0, d <= max_d,
// M * d / 32 < 2^31.
int check_shape(int64_t M, int64_t d, int64_t max_d, const char* fn);

}  // namespace kq
