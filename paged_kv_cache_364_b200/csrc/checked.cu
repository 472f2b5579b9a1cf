// Checked mode (pa_set_option(PA_OPT_CHECKED, 1)): device pre-passes that
// find inputs whose writes would alias, before anything is written.
//
// The pages' sharing rule ("Stop Wasting GPU Memory: A Deep Dive Into vLLM's
// PagedAttention", "Copy-on-Write for Parallel Sampling"): a block shared by
// several sequences is copied before one of them writes into it.  An engine
// that gets this wrong -- or hands the cache operations aliasing arguments --
// corrupts a shared prefix silently, because the kernels only check that ids
// are inside the pool.  In checked mode:
//   pa_write_kv       two tokens of one call with the same live slot;
//   pa_copy_blocks    a destination block named twice, or also as a source;
//   pa_decode_append  a sequence's newest block (the one its new row is
//                     stored into) that another sequence of the batch also
//                     reads, or that its own table lists twice.
// Each check is one small kernel over the call's index arguments (all pairs,
// in shared-memory chunks; no scratch memory).  It sets PA_DEVERR_ALIAS in
// the sticky device error word, counts the violations and keeps the lowest
// offending index; the entry point synchronises its stream, reads that count
// and, if it is not zero, returns PA_ERR_BOUNDS without launching the write.
// Checked mode therefore blocks the host once per call and cannot run inside
// a stream capture (PA_ERR_STATE).  With the option off (the default) none of
// this runs.
#include <string>

#include "pa_device.cuh"
#include "pa_host.h"

PA_DEFINE_ERROR_WORD(checked)

namespace {

int g_checked = 0;

// violations found by the last check, and the lowest offending index
__device__ unsigned int g_check_hits;
__device__ long long g_check_first;

__device__ __forceinline__ void report(long long index) {
  atomicAdd(&g_check_hits, 1u);
  atomicMin(&g_check_first, index);
  checked_flag(PA_DEVERR_ALIAS);
}

constexpr int kThreads = 256;
constexpr int kChunk = 1024;   // entries of the compared list staged per round

// Token t has a live slot (in [0, num_slots)) equal to that of an earlier token.
__global__ void __launch_bounds__(kThreads) dup_slots_kernel(const int32_t* slots, int64_t stride, int64_t T,
                                                             int64_t num_slots) {
  __shared__ int32_t chunk[kChunk];
  const int64_t t = int64_t(blockIdx.x) * kThreads + threadIdx.x;
  const int32_t mine = t < T ? slots[t * stride] : -1;
  const bool live = mine >= 0 && mine < num_slots;
  bool hit = false;
  const int64_t last = min(T, (int64_t(blockIdx.x) + 1) * kThreads);   // earlier tokens of this CTA's last one
  for (int64_t c0 = 0; c0 < last; c0 += kChunk) {
    const int n = int(last - c0 < kChunk ? last - c0 : kChunk);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kThreads) chunk[i] = slots[(c0 + i) * stride];
    __syncthreads();
    if (live && !hit) {
      const int64_t before = t - c0;   // only tokens before t
      const int lim = int(before < n ? before : n);
      for (int i = 0; i < lim; ++i)
        if (chunk[i] == mine) {
          hit = true;
          break;
        }
    }
  }
  if (hit) report(t);
}

// Pair i's destination equals an earlier pair's destination or any pair's source.
__global__ void __launch_bounds__(kThreads) dup_pairs_kernel(const int64_t* pairs, int64_t row, int64_t col,
                                                             int64_t P) {
  __shared__ int64_t src[kChunk / 2], dst[kChunk / 2];
  const int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t my_dst = i < P ? pairs[i * row + col] : -1;
  bool hit = false;
  for (int64_t c0 = 0; c0 < P; c0 += kChunk / 2) {
    const int n = int(P - c0 < kChunk / 2 ? P - c0 : kChunk / 2);
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += kThreads) {
      src[j] = pairs[(c0 + j) * row];
      dst[j] = pairs[(c0 + j) * row + col];
    }
    __syncthreads();
    if (i < P && !hit)
      for (int j = 0; j < n; ++j)
        if (src[j] == my_dst || (c0 + j < i && dst[j] == my_dst)) {
          hit = true;
          break;
        }
  }
  if (hit) report(i);
}

// Every table entry (s', b) a sequence reads (b < ceil(n_s' / B)) is compared
// with every sequence's newest block: equal ids at another (sequence, logical
// block) mean the new row would be stored into a block read elsewhere.
__global__ void __launch_bounds__(kThreads) append_alias_kernel(const int32_t* tables, int64_t tab_s,
                                                                int64_t tab_b, const int32_t* lens, int64_t len_s,
                                                                int batch, int block_size, int max_blocks,
                                                                int max_tokens) {
  __shared__ int32_t newest[kChunk];
  __shared__ int32_t newest_b[kChunk];
  const int64_t e = int64_t(blockIdx.x) * kThreads + threadIdx.x;   // entry index s' * max_blocks + b
  const int64_t total = int64_t(batch) * max_blocks;
  int32_t id = -1;
  int s2 = -1, b2 = -1;
  if (e < total) {
    s2 = int(e / max_blocks);
    b2 = int(e % max_blocks);
    const int n = lens[s2 * len_s];
    if (n >= 1 && n <= max_tokens && b2 < (n + block_size - 1) / block_size) id = tables[s2 * tab_s + b2 * tab_b];
  }
  bool hit = false;
  for (int c0 = 0; c0 < batch; c0 += kChunk) {
    const int cnt = min(kChunk, batch - c0);
    __syncthreads();
    for (int j = threadIdx.x; j < cnt; j += kThreads) {
      const int s = c0 + j;
      const int n = lens[s * len_s];
      const bool ok = n >= 1 && n <= max_tokens;
      const int b = ok ? (n - 1) / block_size : -1;
      newest_b[j] = b;
      newest[j] = ok ? tables[s * tab_s + int64_t(b) * tab_b] : -1;
    }
    __syncthreads();
    if (id >= 0 && !hit)
      for (int j = 0; j < cnt; ++j)
        if (newest[j] == id && (c0 + j != s2 || newest_b[j] != b2)) {
          hit = true;
          break;
        }
  }
  if (hit) report(int64_t(s2));
}

// Reset the counters, run `launch` on `s`, wait, and turn violations into
// PA_ERR_BOUNDS.
template <typename F>
int run_check(cudaStream_t s, const char* what, F launch) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "checked mode: cudaStreamIsCapturing failed");
  if (cap != cudaStreamCaptureStatusNone)
    return pa::fail(PA_ERR_STATE, std::string(what) + ": checked mode synchronises and cannot run in a stream capture");
  const unsigned int zero = 0u;
  const long long big = 0x7fffffffffffffffLL;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_check_hits, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_check_first, &big, sizeof(big), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("checked mode reset: ") + cudaGetErrorString(e));
  launch();
  pa::count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("checked mode launch: ") + cudaGetErrorString(e));
  unsigned int hits = 0;
  long long first = 0;
  e = cudaMemcpyFromSymbolAsync(&hits, g_check_hits, sizeof(hits), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(&first, g_check_first, sizeof(first), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("checked mode read-back: ") + cudaGetErrorString(e));
  if (hits)
    return pa::fail(PA_ERR_BOUNDS, std::string(what) + ": " + std::to_string(hits) +
                                       " aliasing input(s), first at index " + std::to_string(first));
  return PA_OK;
}

unsigned grid_for(int64_t n) { return unsigned((n + kThreads - 1) / kThreads); }

}  // namespace

int pa_internal_take_errors_checked(unsigned int* bits) { return checked_take_errors(bits); }

int pa_internal_set_checked(int32_t v) {
  if (v < 0 || v > 1) return pa::fail(PA_ERR_ARG, "PA_OPT_CHECKED takes 0 or 1");
  g_checked = v;
  return PA_OK;
}

int pa_internal_get_checked() { return g_checked; }

namespace pa {

bool checked_mode() { return g_checked != 0; }

int check_slots(const int32_t* slots, int64_t stride, int64_t T, int64_t num_slots, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T <= 1) return PA_OK;
  if (T > int64_t(UINT32_MAX) * kThreads) return fail(PA_ERR_ARG, "checked mode: too many tokens");
  return run_check(s, "pa_write_kv", [&] {
    dup_slots_kernel<<<grid_for(T), kThreads, 0, s>>>(slots, stride, T, num_slots);
  });
}

int check_pairs(const int64_t* pairs, int64_t row, int64_t col, int64_t P, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (P < 1) return PA_OK;
  return run_check(s, "pa_copy_blocks", [&] { dup_pairs_kernel<<<grid_for(P), kThreads, 0, s>>>(pairs, row, col, P); });
}

int check_append(const int32_t* tables, int64_t tab_s, int64_t tab_b, const int32_t* lens, int64_t len_s, int batch,
                 int block_size, int max_blocks, int max_tokens, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (batch < 1 || max_blocks < 1) return PA_OK;
  return run_check(s, "pa_decode_append", [&] {
    append_alias_kernel<<<grid_for(int64_t(batch) * max_blocks), kThreads, 0, s>>>(
        tables, tab_s, tab_b, lens, len_s, batch, block_size, max_blocks, max_tokens);
  });
}

}  // namespace pa
