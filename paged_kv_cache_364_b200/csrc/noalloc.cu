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
//   - When the 32 MiB is taken: the library links the CUDA runtime statically
//     and, with the runtime's default lazy module loading, a module's
//     __device__ arrays are allocated when the module is first used on a
//     device -- here, at the first call on that device (with
//     CUDA_MODULE_LOADING=EAGER, when the library's modules are loaded).  An
//     engine that hands nearly all HBM to its block pool must therefore make
//     one call per device BEFORE it reserves the pool; a call with an empty
//     batch (q of shape [0, Hq, head_dim]) does only this set-up.
//   - Set-up: the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current.  Make that first call
//     outside any CUDA stream capture.  The address is kept per device
//     together with the id of the CUDA context it belongs to; a call that
//     finds another context current (after cudaDeviceReset the primary
//     context, and with it the module and its array, is created anew) looks
//     the address up again, so that call too must come outside stream capture.
//   - All calls share the one array, which keeps the contents of the last
//     call.  Nothing in it needs to start at zero: every byte a call reads is
//     written earlier in that same call.  Two calls that can overlap on the GPU
//     (different streams, no ordering between them) race on the array; order
//     them on one stream or use pa_decode with separate workspaces.
#include <cudaTypedefs.h>

#include <mutex>
#include <string>

#include "pa_device.cuh"
#include "pa_host.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mu;
struct ScratchSlot {
  unsigned long long ctx_id;   // id of the CUDA context the address belongs to
  void* ptr;
};
ScratchSlot g_scratch[kMaxDevices] = {};

// Id of the current CUDA context (unique for the life of the process), through
// the runtime's driver entry points; 0 if it cannot be read.
unsigned long long current_context_id() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device: looked up on the
// first call on a device, and again whenever the current context is not the
// one the kept address belongs to.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return pa::fail(PA_ERR_ARG, "device index above the supported range");
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> g(g_setup_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.ptr || ctx == 0 || slot.ctx_id != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return pa::fail(PA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    slot.ptr = p;
    slot.ctx_id = ctx != 0 ? ctx : current_context_id();
  }
  *out = slot.ptr;
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
  if (batch < 0) return pa::fail(PA_ERR_ARG, "q: negative batch size");
  if (hq < 1 || d < 1) return pa::fail(PA_ERR_ARG, "q: need at least one query head and head_dim >= 1");
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
