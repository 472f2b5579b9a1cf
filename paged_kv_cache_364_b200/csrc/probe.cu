// Read-bandwidth probe (pa_read_probe): a measurement helper beside the
// method's kernels, not a step of it.  The decode kernel only reads K/V pages
// (its writes are a few MB of partial states and outputs), so besides the
// copy (read + write) ceiling it is compared with the rate at which this GPU
// streams a buffer it only reads.  The probe reads a device buffer once with
// 16-byte read-only loads, several in flight per thread, and folds every
// 32-bit word into one XOR so that no load can be dropped.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <string>

#include "pa_host.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;        // independent 16-byte loads per thread per round
constexpr int kCtasPerSm = 4;     // 1024 threads per SM: 64 KB of loads in flight per SM

__device__ __forceinline__ uint32_t fold(const uint4& v) { return v.x ^ v.y ^ v.z ^ v.w; }

// Grid-stride over n 16-byte vectors.  Round r of thread t reads vectors
// i, i + stride, ..., i + (kUnroll - 1) * stride, all below n; the remainder
// loop reads what is left one vector at a time.
__global__ void __launch_bounds__(kThreads) read_probe_kernel(const uint4* __restrict__ p, int64_t n,
                                                              uint32_t* sink) {
  uint32_t acc = 0;
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x;
  for (; i + (kUnroll - 1) * stride < n; i += kUnroll * stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = __ldg(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc ^= fold(v[u]);
  }
  for (; i < n; i += stride) acc ^= fold(__ldg(p + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

int probe_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return std::max(n, 1);
}

}  // namespace

extern "C" int pa_read_probe(const void* buf, uint64_t bytes, uint32_t* sink, pa_stream stream) {
  pa::clear_error();
  if (!sink || (bytes != 0 && !buf)) return pa::fail(PA_ERR_ARG, "pa_read_probe: NULL pointer");
  if (bytes % 16 != 0 || reinterpret_cast<uintptr_t>(buf) % 16 != 0)
    return pa::fail(PA_ERR_ARG, "pa_read_probe: the buffer must start on and span whole 16-byte units");
  if (reinterpret_cast<uintptr_t>(sink) % 4 != 0) return pa::fail(PA_ERR_ARG, "pa_read_probe: sink not 4-byte aligned");
  if (bytes == 0) return PA_OK;
  const int64_t n = static_cast<int64_t>(bytes / 16);
  const int64_t want = (n + kThreads - 1) / kThreads;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(want, int64_t(probe_sms()) * kCtasPerSm));
  read_probe_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(buf), n,
                                                                              sink);
  pa::count_launches(1);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("pa_read_probe launch: ") + cudaGetErrorString(e));
  return PA_OK;
}
