// Library-wide C ABI pieces: status strings, per-thread error messages,
// version, and the read-back of the kernels' sticky device error words.
#include <cuda_runtime.h>

#include <atomic>
#include <string>

#include "pa_host.h"
#include "pagedkv.h"

int pa_internal_take_errors_cacheops(unsigned int* bits);
int pa_internal_take_errors_decode(unsigned int* bits);
int pa_internal_take_errors_prefill(unsigned int* bits);
int pa_internal_take_errors_checked(unsigned int* bits);

namespace pa {

static thread_local std::string t_last_error;

int fail(int code, const std::string& msg) {
  t_last_error = msg;
  return code;
}

void clear_error() { t_last_error.clear(); }

static std::atomic<unsigned long long> g_launches{0};

void count_launches(int n) { g_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed); }

}  // namespace pa

extern "C" {

const char* pa_strerror(int code) {
  switch (code) {
    case PA_OK: return "ok";
    case PA_ERR_ARG: return "invalid argument";
    case PA_ERR_DTYPE: return "unsupported or mismatched dtype";
    case PA_ERR_OOM: return "free pool is empty";
    case PA_ERR_STATE: return "invalid allocator state transition";
    case PA_ERR_BOUNDS: return "device bounds check fired";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_TIMEOUT: return "bounded device wait ran out";
    default: return "unknown error";
  }
}

const char* pa_last_error(void) { return pa::t_last_error.c_str(); }

const char* pa_version(void) { return "1.0.0"; }

int pa_launch_count(uint64_t* count_out) {
  pa::clear_error();
  if (!count_out) return pa::fail(PA_ERR_ARG, "NULL output");
  *count_out = pa::g_launches.load(std::memory_order_relaxed);
  return PA_OK;
}

int pa_device_errors(pa_stream stream, uint32_t* bits_out) {
  pa::clear_error();
  if (!bits_out) return pa::fail(PA_ERR_ARG, "NULL output");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("stream sync: ") + cudaGetErrorString(e));
  unsigned int a = 0, b = 0, c = 0, d = 0;
  if (pa_internal_take_errors_cacheops(&a) != PA_OK || pa_internal_take_errors_decode(&b) != PA_OK ||
      pa_internal_take_errors_prefill(&c) != PA_OK || pa_internal_take_errors_checked(&d) != PA_OK)
    return pa::fail(PA_ERR_CUDA, "reading the device error words failed");
  *bits_out = a | b | c | d;
  return PA_OK;
}

}  // extern "C"
