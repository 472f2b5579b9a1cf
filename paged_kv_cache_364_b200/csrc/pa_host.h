// Host-side helpers shared by the C-ABI translation units: error reporting and
// pa_tensor checks.  No CUDA types here, so the allocator builds as plain C++.
#pragma once

#include <cstdint>
#include <string>

#include "pagedkv.h"

namespace pa {

// Record a detailed message for pa_last_error() and return `code`.
int fail(int code, const std::string& msg);
void clear_error();
// Count kernels this library has enqueued (reported by pa_launch_count).
void count_launches(int n);

// Checked mode (PA_OPT_CHECKED, csrc/checked.cu): device pre-passes that find
// aliasing writes; each synchronises `stream` (a cudaStream_t) and returns
// PA_ERR_BOUNDS when it found any.
bool checked_mode();
int check_slots(const int32_t* slots, int64_t stride, int64_t T, int64_t num_slots, void* stream);
int check_pairs(const int64_t* pairs, int64_t row, int64_t col, int64_t P, void* stream);
int check_append(const int32_t* tables, int64_t tab_s, int64_t tab_b, const int32_t* lens, int64_t len_s, int batch,
                 int block_size, int max_blocks, int max_tokens, void* stream);

inline int64_t dtype_size(int32_t dt) {
  switch (dt) {
    case PA_F32: return 4;
    case PA_F16: return 2;
    case PA_BF16: return 2;
    case PA_I32: return 4;
    case PA_I64: return 8;
    case PA_U8: return 1;
    default: return 0;
  }
}

inline bool is_float(int32_t dt) { return dt == PA_F32 || dt == PA_F16 || dt == PA_BF16; }

// Row-major contiguous (the standard strides for its shape).
inline bool is_contiguous(const pa_tensor& t) {
  int64_t expect = 1;
  for (int i = t.ndim - 1; i >= 0; --i) {
    if (t.shape[i] != 1 && t.stride[i] != expect) return false;
    expect *= t.shape[i];
  }
  return true;
}

inline int64_t numel(const pa_tensor& t) {
  int64_t n = 1;
  for (int i = 0; i < t.ndim; ++i) n *= t.shape[i];
  return n;
}

}  // namespace pa
