// Slot-mapping write (pa_write_kv) and copy-on-write block copy
// (pa_copy_blocks).  Both move bits only; both are bound by HBM traffic and
// launch latency, so each thread moves fixed-size vectors (16 bytes whenever
// alignment allows) with all loads issued before the stores.
//
// Write: "Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
// Technical Details, "Single Sequence Generation" -- a new token fills the
// next slot of its sequence's current physical block.
// Copy: same page, "Copy-on-Write for Parallel Sampling" -- on divergence the
// diverging block is copied to a new physical block.
#include <algorithm>
#include <string>

#include "pa_device.cuh"
#include "pa_host.h"

PA_DEFINE_ERROR_WORD(cacheops)

namespace {

// A vector of W bytes.
template <int W> struct Vec;
template <> struct Vec<16> { using type = uint4; };
template <> struct Vec<8> { using type = uint2; };
template <> struct Vec<4> { using type = uint32_t; };
template <> struct Vec<2> { using type = uint16_t; };
template <> struct Vec<1> { using type = uint8_t; };

struct WriteParams {
  const char* k;
  const char* v;
  int64_t k_tok, k_head;   // byte strides of k over tokens / heads
  int64_t v_tok, v_head;
  const int32_t* slots;
  int64_t slot_stride;     // elements
  char* k_cache;
  char* v_cache;
  int64_t T, H, row_bytes, block_size, num_slots;
};

// One thread per W-byte vector of one (token, head) row; rows are copied from
// the token's input row to its slot in both caches.
template <int W>
__global__ void __launch_bounds__(256) write_kv_kernel(WriteParams p) {
  // A following kernel launched as a programmatic dependent (the decode
  // planner) may start now; it waits for this grid before using its results.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using V = typename Vec<W>::type;
  const int64_t vec_per_row = p.row_bytes / W;
  const int64_t total = p.T * p.H * vec_per_row;
  for (int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; u < total;
       u += int64_t(gridDim.x) * blockDim.x) {
    const int64_t c = u % vec_per_row;
    const int64_t th = u / vec_per_row;
    const int64_t h = th % p.H;
    const int64_t t = th / p.H;
    const int64_t slot = p.slots[t * p.slot_stride];
    if (slot == -1) continue;
    if (slot < 0 || slot >= p.num_slots) {
      if (h == 0 && c == 0) cacheops_flag(PA_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = slot / p.block_size;
    const int64_t off = slot % p.block_size;
    const int64_t dst = ((blk * p.H + h) * p.block_size + off) * p.row_bytes + c * W;
    const V kv = *reinterpret_cast<const V*>(p.k + t * p.k_tok + h * p.k_head + c * W);
    const V vv = *reinterpret_cast<const V*>(p.v + t * p.v_tok + h * p.v_head + c * W);
    *reinterpret_cast<V*>(p.k_cache + dst) = kv;
    *reinterpret_cast<V*>(p.v_cache + dst) = vv;
  }
}

constexpr int kMaxCopyCaches = 64;

struct CopyParams {
  char* cache[kMaxCopyCaches];
  int n_caches;
  const int64_t* pairs;
  int64_t pair_row, pair_col;   // element strides of the [P, 2] pair tensor
  int64_t P, num_blocks, block_bytes;
};

constexpr int kCopyUnroll = 4;

// grid: x = chunks of a block, y = pairs (strided), z = caches.
template <int W>
__global__ void __launch_bounds__(256) copy_blocks_kernel(CopyParams p) {
  using V = typename Vec<W>::type;
  const int64_t vecs = p.block_bytes / W;
  char* base = p.cache[blockIdx.z];
  for (int64_t i = blockIdx.y; i < p.P; i += gridDim.y) {
    const int64_t src = p.pairs[i * p.pair_row];
    const int64_t dst = p.pairs[i * p.pair_row + p.pair_col];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
      if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) cacheops_flag(PA_DEVERR_COPY_PAIR);
      continue;
    }
    const V* s = reinterpret_cast<const V*>(base + src * p.block_bytes);
    V* d = reinterpret_cast<V*>(base + dst * p.block_bytes);
    const int64_t stride = int64_t(gridDim.x) * blockDim.x * kCopyUnroll;
    for (int64_t v0 = (int64_t(blockIdx.x) * blockDim.x * kCopyUnroll) + threadIdx.x; v0 < vecs;
         v0 += stride) {
      V buf[kCopyUnroll];
#pragma unroll
      for (int j = 0; j < kCopyUnroll; ++j) {
        const int64_t v = v0 + int64_t(j) * blockDim.x;
        if (v < vecs) buf[j] = s[v];
      }
#pragma unroll
      for (int j = 0; j < kCopyUnroll; ++j) {
        const int64_t v = v0 + int64_t(j) * blockDim.x;
        if (v < vecs) d[v] = buf[j];
      }
    }
  }
}

int vector_width(std::initializer_list<int64_t> values) {
  for (int w : {16, 8, 4, 2}) {
    bool ok = true;
    for (int64_t x : values) ok = ok && (x % w == 0);
    if (ok) return w;
  }
  return 1;
}

int cuda_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return PA_OK;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

int pa_internal_take_errors_cacheops(unsigned int* bits) { return cacheops_take_errors(bits); }

extern "C" int pa_write_kv(const pa_tensor* k, const pa_tensor* v, const pa_tensor* slot_mapping,
                           const pa_tensor* k_cache, const pa_tensor* v_cache, pa_stream stream) {
  pa::clear_error();
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return pa::fail(PA_ERR_ARG, "NULL tensor");
  if (k->ndim != 3 || v->ndim != 3) return pa::fail(PA_ERR_ARG, "k and v must be [T, Hkv, head_dim]");
  if (k_cache->ndim != 4 || v_cache->ndim != 4)
    return pa::fail(PA_ERR_ARG, "caches must be [num_blocks, Hkv, B, head_dim]");
  if (slot_mapping->ndim != 1 || slot_mapping->dtype != PA_I32)
    return pa::fail(PA_ERR_ARG, "slot_mapping must be int32 [T]");
  if (!pa::is_float(k->dtype) || v->dtype != k->dtype || k_cache->dtype != k->dtype ||
      v_cache->dtype != k->dtype)
    return pa::fail(PA_ERR_DTYPE, "k, v and both caches must share one float dtype");
  for (int i = 0; i < 4; ++i)
    if (k_cache->shape[i] != v_cache->shape[i]) return pa::fail(PA_ERR_ARG, "k_cache and v_cache shapes differ");
  if (!pa::is_contiguous(*k_cache) || !pa::is_contiguous(*v_cache))
    return pa::fail(PA_ERR_ARG, "caches must be contiguous");
  const int64_t T = k->shape[0], H = k->shape[1], D = k->shape[2];
  for (int i = 0; i < 3; ++i)
    if (v->shape[i] != k->shape[i]) return pa::fail(PA_ERR_ARG, "k and v shapes differ");
  if (slot_mapping->shape[0] != T) return pa::fail(PA_ERR_ARG, "slot_mapping length differs from T");
  if (k_cache->shape[1] != H || k_cache->shape[3] != D)
    return pa::fail(PA_ERR_ARG, "cache head count or head_dim differs from k");
  if ((k->stride[2] != 1 && D > 1) || (v->stride[2] != 1 && D > 1))
    return pa::fail(PA_ERR_ARG, "k and v need a contiguous last dimension");
  if (T == 0 || H == 0 || D == 0) return PA_OK;
  const int64_t elt = pa::dtype_size(k->dtype);
  WriteParams p;
  p.k = static_cast<const char*>(k->data);
  p.v = static_cast<const char*>(v->data);
  p.k_tok = k->stride[0] * elt;
  p.k_head = k->stride[1] * elt;
  p.v_tok = v->stride[0] * elt;
  p.v_head = v->stride[1] * elt;
  p.slots = static_cast<const int32_t*>(slot_mapping->data);
  p.slot_stride = slot_mapping->stride[0];
  p.k_cache = static_cast<char*>(k_cache->data);
  p.v_cache = static_cast<char*>(v_cache->data);
  p.T = T;
  p.H = H;
  p.row_bytes = D * elt;
  p.block_size = k_cache->shape[2];
  p.num_slots = k_cache->shape[0] * k_cache->shape[2];
  if (!p.k || !p.v || !p.slots || !p.k_cache || !p.v_cache) return pa::fail(PA_ERR_ARG, "NULL data pointer");
  const int W = vector_width({reinterpret_cast<int64_t>(p.k), reinterpret_cast<int64_t>(p.v),
                              reinterpret_cast<int64_t>(p.k_cache),
                              reinterpret_cast<int64_t>(p.v_cache), p.k_tok, p.k_head, p.v_tok,
                              p.v_head, p.row_bytes});
  const int64_t total = T * H * (p.row_bytes / W);
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((total + threads - 1) / threads, int64_t(num_sms()) * 16);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pa::checked_mode()) {
    const int rc = pa::check_slots(p.slots, p.slot_stride, T, p.num_slots, stream);
    if (rc != PA_OK) return rc;
  }
  switch (W) {
    case 16: write_kv_kernel<16><<<blocks, threads, 0, s>>>(p); break;
    case 8: write_kv_kernel<8><<<blocks, threads, 0, s>>>(p); break;
    case 4: write_kv_kernel<4><<<blocks, threads, 0, s>>>(p); break;
    case 2: write_kv_kernel<2><<<blocks, threads, 0, s>>>(p); break;
    default: write_kv_kernel<1><<<blocks, threads, 0, s>>>(p); break;
  }
  pa::count_launches(1);
  return cuda_status("pa_write_kv launch");
}

extern "C" int pa_copy_blocks(const pa_tensor* caches, int32_t n_caches, const pa_tensor* src_dst_pairs,
                              pa_stream stream) {
  pa::clear_error();
  if (!src_dst_pairs || n_caches < 0 || (n_caches > 0 && !caches)) return pa::fail(PA_ERR_ARG, "bad arguments");
  if (src_dst_pairs->ndim != 2 || src_dst_pairs->shape[1] != 2 || src_dst_pairs->dtype != PA_I64)
    return pa::fail(PA_ERR_ARG, "src_dst_pairs must be int64 [P, 2]");
  const int64_t P = src_dst_pairs->shape[0];
  if (n_caches == 0 || P == 0) return PA_OK;
  const pa_tensor& c0 = caches[0];
  if (c0.ndim < 1) return pa::fail(PA_ERR_ARG, "a cache must have a block dimension");
  for (int32_t i = 0; i < n_caches; ++i) {
    const pa_tensor& c = caches[i];
    if (c.ndim != c0.ndim || c.dtype != c0.dtype) return pa::fail(PA_ERR_ARG, "caches differ in rank or dtype");
    for (int d = 0; d < c.ndim; ++d)
      if (c.shape[d] != c0.shape[d]) return pa::fail(PA_ERR_ARG, "caches differ in shape");
    if (!pa::is_contiguous(c)) return pa::fail(PA_ERR_ARG, "caches must be contiguous");
    if (!c.data) return pa::fail(PA_ERR_ARG, "NULL cache pointer");
    if (pa::dtype_size(c.dtype) == 0) return pa::fail(PA_ERR_DTYPE, "unknown cache dtype");
  }
  if (!src_dst_pairs->data) return pa::fail(PA_ERR_ARG, "NULL pair pointer");
  const int64_t block_bytes = pa::numel(c0) / c0.shape[0] * pa::dtype_size(c0.dtype);
  if (block_bytes == 0) return PA_OK;
  CopyParams p;
  p.pairs = static_cast<const int64_t*>(src_dst_pairs->data);
  p.pair_row = src_dst_pairs->stride[0];
  p.pair_col = src_dst_pairs->stride[1];
  p.P = P;
  p.num_blocks = c0.shape[0];
  p.block_bytes = block_bytes;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pa::checked_mode()) {
    const int rc = pa::check_pairs(p.pairs, p.pair_row, p.pair_col, P, stream);
    if (rc != PA_OK) return rc;
  }
  for (int32_t first = 0; first < n_caches; first += kMaxCopyCaches) {
    const int n = std::min<int32_t>(kMaxCopyCaches, n_caches - first);
    int64_t align_probe = block_bytes;
    for (int i = 0; i < n; ++i) {
      p.cache[i] = static_cast<char*>(caches[first + i].data);
      align_probe |= reinterpret_cast<int64_t>(p.cache[i]);
    }
    p.n_caches = n;
    const int W = vector_width({align_probe});
    const int64_t vecs = block_bytes / W;
    const int threads = 256;
    const int64_t per_cta = int64_t(threads) * kCopyUnroll;
    const unsigned gx = static_cast<unsigned>(std::min<int64_t>((vecs + per_cta - 1) / per_cta, 1024));
    const unsigned gy = static_cast<unsigned>(std::min<int64_t>(P, 65535));
    dim3 grid(gx, gy, n);
    switch (W) {
      case 16: copy_blocks_kernel<16><<<grid, threads, 0, s>>>(p); break;
      case 8: copy_blocks_kernel<8><<<grid, threads, 0, s>>>(p); break;
      case 4: copy_blocks_kernel<4><<<grid, threads, 0, s>>>(p); break;
      case 2: copy_blocks_kernel<2><<<grid, threads, 0, s>>>(p); break;
      default: copy_blocks_kernel<1><<<grid, threads, 0, s>>>(p); break;
    }
    pa::count_launches(1);
    int rc = cuda_status("pa_copy_blocks launch");
    if (rc != PA_OK) return rc;
  }
  return PA_OK;
}
