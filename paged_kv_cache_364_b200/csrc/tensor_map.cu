// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link dependency), and the page map of the paged KV cache.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "pa_host.h"
#include "pa_tmap.h"

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

namespace pa {

int encode_page_map(CUtensorMap* map, const pa_tensor& cache) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int64_t d = cache.shape[3];
  const int64_t rows = cache.shape[0] * cache.shape[1] * cache.shape[2];
  cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(d * 2)};
  cuuint32_t box[2] = {64, cuuint32_t(cache.shape[2])};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      cache.dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, dt, 2, cache.data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string(int(r)));
  return PA_OK;
}

}  // namespace pa
