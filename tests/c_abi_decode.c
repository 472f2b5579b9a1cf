/*
 * One decode step through the C ABI alone -- no Python, no torch -- for
 * tests/test_gpu_c_abi.py: device memory from cudaMalloc, pa_write_kv of each
 * sequence's new token, then pa_decode into an fp32 output.
 *
 * Usage: c_abi_decode IN OUT
 * IN  (little-endian): int32 batch, Hq, Hkv, head_dim, num_blocks, max_blocks,
 *     dtype (a pa_dtype), partition_tokens, max_context; float32 scale; then
 *     the raw elements of q [batch, Hq, d], k_new, v_new [batch, Hkv, d],
 *     k_cache, v_cache [num_blocks, Hkv, 16, d], block_tables int32
 *     [batch, max_blocks], context_lens int32 [batch], slots int32 [batch].
 * OUT: out float32 [batch, Hq, d], then k_cache and v_cache after the step,
 *     then the uint32 device error bits.
 * Exit status 0, or 1 with a message on stderr.
 */
#include <cuda_runtime_api.h>
#include <stdio.h>
#include <stdlib.h>

#include "pagedkv.h"

#define BLOCK 16

static void die(const char* what, const char* detail) {
  fprintf(stderr, "%s: %s\n", what, detail);
  exit(1);
}

static void check(int rc, const char* what) {
  if (rc != PA_OK) die(what, pa_last_error());
}

static void check_cuda(cudaError_t e, const char* what) {
  if (e != cudaSuccess) die(what, cudaGetErrorString(e));
}

/* A contiguous descriptor of `ndim` dimensions. */
static pa_tensor desc(void* data, int32_t dtype, int32_t ndim, const int64_t* shape) {
  pa_tensor t;
  t.data = data;
  t.dtype = dtype;
  t.ndim = ndim;
  int64_t stride = 1;
  for (int i = PA_MAX_DIMS - 1; i >= 0; --i) {
    t.shape[i] = i < ndim ? shape[i] : 1;
    t.stride[i] = 0;
  }
  for (int i = ndim - 1; i >= 0; --i) {
    t.stride[i] = stride;
    stride *= shape[i];
  }
  return t;
}

/* Read `bytes` from f into a fresh device buffer. */
static void* upload(FILE* f, size_t bytes, const char* what) {
  void* host = malloc(bytes ? bytes : 1);
  void* dev = NULL;
  if (!host) die(what, "out of host memory");
  if (fread(host, 1, bytes, f) != bytes) die(what, "input file too short");
  check_cuda(cudaMalloc(&dev, bytes ? bytes : 1), what);
  check_cuda(cudaMemcpy(dev, host, bytes, cudaMemcpyHostToDevice), what);
  free(host);
  return dev;
}

static void download(FILE* f, const void* dev, size_t bytes, const char* what) {
  void* host = malloc(bytes ? bytes : 1);
  if (!host) die(what, "out of host memory");
  check_cuda(cudaMemcpy(host, dev, bytes, cudaMemcpyDeviceToHost), what);
  if (fwrite(host, 1, bytes, f) != bytes) die(what, "short write");
  free(host);
}

int main(int argc, char** argv) {
  if (argc != 3) die("usage", "c_abi_decode IN OUT");
  FILE* in = fopen(argv[1], "rb");
  if (!in) die("open", argv[1]);
  int32_t h[9];
  float scale = 0.f;
  if (fread(h, sizeof(int32_t), 9, in) != 9 || fread(&scale, sizeof(float), 1, in) != 1) die("header", "short");
  const int64_t batch = h[0], hq = h[1], hkv = h[2], d = h[3], nb = h[4], max_blocks = h[5];
  const int32_t dtype = h[6], part = h[7], max_context = h[8];
  const size_t es = dtype == PA_F32 ? 4 : 2;
  if (batch < 1 || hq < 1 || hkv < 1 || d < 1 || nb < 1 || max_blocks < 1) die("header", "bad sizes");

  const int64_t q_shape[3] = {batch, hq, d}, kv_shape[3] = {batch, hkv, d};
  const int64_t cache_shape[4] = {nb, hkv, BLOCK, d}, table_shape[2] = {batch, max_blocks};
  const size_t q_bytes = (size_t)(batch * hq * d) * es, kv_bytes = (size_t)(batch * hkv * d) * es;
  const size_t cache_bytes = (size_t)(nb * hkv * BLOCK * d) * es;
  void* q = upload(in, q_bytes, "q");
  void* k_new = upload(in, kv_bytes, "k_new");
  void* v_new = upload(in, kv_bytes, "v_new");
  void* k_cache = upload(in, cache_bytes, "k_cache");
  void* v_cache = upload(in, cache_bytes, "v_cache");
  void* tables = upload(in, (size_t)(batch * max_blocks) * 4, "block_tables");
  void* lens = upload(in, (size_t)batch * 4, "context_lens");
  void* slots = upload(in, (size_t)batch * 4, "slots");
  fclose(in);

  const pa_tensor tq = desc(q, dtype, 3, q_shape), tk = desc(k_new, dtype, 3, kv_shape),
                  tv = desc(v_new, dtype, 3, kv_shape), tkc = desc(k_cache, dtype, 4, cache_shape),
                  tvc = desc(v_cache, dtype, 4, cache_shape), tt = desc(tables, PA_I32, 2, table_shape),
                  tl = desc(lens, PA_I32, 1, &batch), ts = desc(slots, PA_I32, 1, &batch);
  check(pa_write_kv(&tk, &tv, &ts, &tkc, &tvc, NULL), "pa_write_kv");

  const size_t ws_bytes = pa_decode_workspace_size((int32_t)batch, (int32_t)hq, (int32_t)d, max_context, part);
  if (ws_bytes == 0) die("pa_decode_workspace_size", "invalid arguments");
  void* ws = NULL;
  float* out = NULL;
  check_cuda(cudaMalloc(&ws, ws_bytes), "workspace");
  check_cuda(cudaMalloc((void**)&out, (size_t)(batch * hq * d) * 4), "out");
  const int64_t ws_shape[1] = {(int64_t)ws_bytes};
  const pa_tensor tws = desc(ws, PA_U8, 1, ws_shape), tout = desc(out, PA_F32, 3, q_shape);
  check(pa_decode(&tq, &tkc, &tvc, &tt, &tl, scale, max_context, part, &tws, &tout, NULL), "pa_decode");
  uint32_t errors = 0;
  check(pa_device_errors(NULL, &errors), "pa_device_errors");

  FILE* o = fopen(argv[2], "wb");
  if (!o) die("open", argv[2]);
  download(o, out, (size_t)(batch * hq * d) * 4, "out");
  download(o, k_cache, cache_bytes, "k_cache");
  download(o, v_cache, cache_bytes, "v_cache");
  if (fwrite(&errors, sizeof(errors), 1, o) != 1) die("write", "errors");
  fclose(o);

  void* bufs[] = {q, k_new, v_new, k_cache, v_cache, tables, lens, slots, ws, out};
  for (size_t i = 0; i < sizeof(bufs) / sizeof(bufs[0]); ++i) check_cuda(cudaFree(bufs[i]), "cudaFree");
  return 0;
}
