// Library-wide host plumbing: per-thread last-error text and the version.
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace rkv {

static thread_local char g_last_error[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

void clear_error() { g_last_error[0] = '\0'; }

rkv_status fail(rkv_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

rkv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(RKV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

}  // namespace rkv

extern "C" const char* rkv_last_error_string(void) { return rkv::g_last_error; }

extern "C" int32_t rkv_version(void) { return RKV_VERSION; }
