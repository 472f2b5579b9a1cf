// Tensor maps (TMA descriptors) over the paged KV cache, shared by the
// attention translation units.
#pragma once

#include <cuda.h>

#include "pagedkv.h"

namespace pa {

// 2-D view of a contiguous [num_blocks, Hkv, B, d] fp16/bf16 cache as
// (d, num_blocks * Hkv * B rows); box = 64 elements x B rows with 128-byte
// swizzling, so one (block, KV head) page is d/64 boxes.  Returns PA_OK or an
// error recorded for pa_last_error().
int encode_page_map(CUtensorMap* map, const pa_tensor& cache);

}  // namespace pa
