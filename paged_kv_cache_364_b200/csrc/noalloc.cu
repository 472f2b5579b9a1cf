// pa_decode_noalloc: paged decode attention for callers that cannot allocate
// device memory.
//
// pa_decode needs a scratch buffer (the split-context plan and the partial
// softmax states of every partition), which its caller allocates.  Some
// callers cannot do that:
//   - a serving engine that hands nearly all of HBM to its KV block pool at
//     start-up and forbids any later device allocation (a late cudaMalloc can
//     fail once the pool is carved out, and may stall the device while the
//     decode loop is running);
//   - a plain C host that embeds this library without any device-memory
//     manager of its own and owns only the tensors it passes in.
// For them this entry point keeps its scratch in a fixed array compiled into
// the library, so the call itself allocates nothing.
//
// Rules of use
//   - The array holds kNoallocScratchBytes (32 MiB).  Every GPU that loads
//     this part of the library keeps that much device memory until the process
//     exits.  A call whose batch needs more scratch than that is rejected
//     with PA_ERR_ARG before anything is launched.
//   - Set-up: the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current, once per device.  Make
//     that first call outside any CUDA stream capture.
//   - All calls share the one array, which keeps the contents of the last
//     call.  Nothing in it needs to start at zero: every byte a call reads is
//     written earlier in that same call.  Two calls that can overlap on the GPU
//     (different streams, no ordering between them) race on the array; order
//     them on one stream or use pa_decode with separate workspaces.
#include <mutex>
#include <string>

#include "pa_device.cuh"
#include "pa_host.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return pa::fail(PA_ERR_ARG, "device index above the supported range");
  std::lock_guard<std::mutex> g(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return pa::fail(PA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_noalloc(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                                 const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                                 int32_t max_context, int32_t partition_tokens, const pa_tensor* out,
                                 pa_stream stream) {
  pa::clear_error();
  if (!q || q->ndim != 3) return pa::fail(PA_ERR_ARG, "q must be [batch, Hq, head_dim]");
  const int64_t batch = q->shape[0], hq = q->shape[1], d = q->shape[2];
  if (batch > INT32_MAX || hq > INT32_MAX || d > INT32_MAX) return pa::fail(PA_ERR_ARG, "q shape too large");
  const size_t need = pa_decode_workspace_size(int32_t(batch), int32_t(hq), int32_t(d), max_context,
                                               partition_tokens);
  if (batch > 0 && need == 0) return pa::fail(PA_ERR_ARG, "invalid max_context / partition_tokens / shape");
  if (need > kNoallocScratchBytes)
    return pa::fail(PA_ERR_ARG, "this batch needs " + std::to_string(need) +
                                    " bytes of decode scratch; the built-in scratch holds " +
                                    std::to_string(kNoallocScratchBytes) +
                                    " (use pa_decode with a caller-provided workspace)");
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != PA_OK) return rc;
  pa_tensor ws;
  ws.data = scratch;
  ws.dtype = PA_U8;
  ws.ndim = 1;
  ws.shape[0] = int64_t(kNoallocScratchBytes);
  ws.stride[0] = 1;
  for (int i = 1; i < PA_MAX_DIMS; ++i) ws.shape[i] = ws.stride[i] = 0;
  return pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, max_context, partition_tokens,
                   &ws, out, stream);
}
