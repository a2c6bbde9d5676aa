// Host-side helpers: status strings, the per-thread error message, argument
// checks and cached device properties.
#include "kq_host.h"

#include <cstdarg>
#include <cstdio>
#include <mutex>

namespace kq {

namespace {
thread_local char g_msg[512] = "";
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
std::mutex g_mu;
}  // namespace

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return status;
}

int cuda_fail(cudaError_t err, const char* what) {
  return fail(KQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(err), cudaGetErrorName(err));
}

int check_launch(const char* what) {
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return cuda_fail(err, what);
  return KQ_OK;
}

int sm_count(int* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_sm_count[dev] > 0) {
      *out = g_sm_count[dev];
      return KQ_OK;
    }
  }
  int n = 0;
  err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaDeviceGetAttribute");
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_sm_count[dev] = n;
  }
  *out = n;
  return KQ_OK;
}

int check_shape(int64_t M, int64_t d, int64_t max_d, const char* fn) {
  if (M < 0) return fail(KQ_ERR_INVALID_ARG, "%s: M = %lld < 0", fn, (long long)M);
  if (d <= 0 || d % 32 != 0)
    return fail(KQ_ERR_INVALID_ARG, "%s: d = %lld must be a positive multiple of 32", fn,
                (long long)d);
  if (max_d > 0 && d > max_d)
    return fail(KQ_ERR_UNSUPPORTED, "%s: d = %lld exceeds the limit %lld", fn, (long long)d,
                (long long)max_d);
  if (M > 0 && M > (((int64_t)1 << 31) - 1) / (d / 32))
    return fail(KQ_ERR_UNSUPPORTED, "%s: M * d / 32 = %lld blocks exceeds 2^31 - 1", fn,
                (long long)(M * (d / 32)));
  return KQ_OK;
}

}  // namespace kq

extern "C" {

const char* kq_status_string(int status) {
  switch (status) {
    case KQ_OK: return "KQ_OK: success";
    case KQ_ERR_INVALID_ARG: return "KQ_ERR_INVALID_ARG: invalid argument";
    case KQ_ERR_ALIGNMENT: return "KQ_ERR_ALIGNMENT: pointer not aligned as required";
    case KQ_ERR_DTYPE: return "KQ_ERR_DTYPE: unsupported input element type";
    case KQ_ERR_UNSUPPORTED: return "KQ_ERR_UNSUPPORTED: size beyond a documented limit";
    case KQ_ERR_CUDA: return "KQ_ERR_CUDA: a CUDA call failed";
    default: return "unknown KroQuant status";
  }
}

const char* kq_last_error(void) { return kq::g_msg; }

int kq_version(void) { return 10000; }

}  // extern "C"
