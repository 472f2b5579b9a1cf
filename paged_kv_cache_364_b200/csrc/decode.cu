// Paged decode attention (pa_decode) for sm_100a.
//
// What is computed: for query head h of sequence s,
//     out[s, h] = softmax(scale * K_s q[s, h]) V_s,
// where K_s / V_s are the sequence's first context_lens[s] token rows reached
// through its block table.  Paging leaves the attention math unchanged
// ("PagedAttention: How Virtual Memory Paging Solved LLM KV Cache Waste", Key
// points, "Engineering insight"); the kernel gathers the scattered blocks
// through the block table on the fly (same page, "Why it matters"; "49 vLLM /
// PagedAttention", "Questions worth asking": the attention kernel has to cope
// with non-contiguous memory).  Cache layout: [num_blocks, Hkv, B, d], so
// one (block, KV head) page is B*d contiguous elements.
//
// Kernels in this file
//   decode_plan_kernel     one CTA: lists the (sequence, partition) work items
//                          in the workspace -- the full partitions, then
//                          every partial or single partition by decreasing
//                          size.
//   decode_fast_kernel     persistent, 2 CTAs x 4 warps per SM, every warp an
//                          independent worker: it claims whole partitions of a
//                          (sequence, KV head) from a shared counter, streams
//                          their pages through its own ring of shared-memory
//                          stages with 2-D tensor copies (128-byte swizzle,
//                          mbarrier completion, bounded waits) and keeps an
//                          online softmax state.  A single partition's output
//                          is written directly; otherwise the partition's
//                          (m, l, acc) state, and the last warp of a (sequence,
//                          KV head) merges them (up to 32 partitions).  For
//                          pa_decode_append it also stores each sequence's new
//                          K/V row while it stages that token's page.
//                            MHA (one query head per KV head): fp32 FMAs on CUDA
//                            cores, warp-shuffle reductions for q.k and the max.
//                            GQA (2..8 or 16 query heads per KV head): q.k and p.V as
//                            m16n8k16 tensor-core MMAs with tokens as the M
//                            dimension; p is split into two 16-bit terms so the
//                            product keeps ~16 bits of p.
//   append_rows_kernel     the new K/V rows for pa_decode_append where the fast
//                          kernel cannot store them (generic path, rows not
//                          16-byte aligned).
//   decode_generic_kernel  CUDA-core fallback for every other shape and dtype
//                          (fp32, any head size, block size or group size).
//   decode_merge_kernel    log-sum-exp merge of the partition states of
//                          sequences the fast kernel does not merge itself
//                          (more than 32 partitions; every multi-partition
//                          sequence on the generic path):
//                          M = max m_p, L = sum l_p 2^(m_p-M),
//                          out = sum 2^(m_p-M) acc_p / L   (base-2 scores).
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <type_traits>
#include <utility>
#include <vector>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tmap.h"

PA_DEFINE_ERROR_WORD(decode)

// prefill path switch (prefill.cu), reached through pa_set_option / pa_get_option
int pa_internal_set_prefill_path(int32_t v);
int pa_internal_get_prefill_path();
// checked mode switch (checked.cu)
int pa_internal_set_checked(int32_t v);
int pa_internal_get_checked();

// Work order of the plan: 0 = the full partitions, then every other item by
// decreasing size (see decode_plan_kernel); 1 = single-partition sequences
// after all partial partitions of longer ones (measured slower: a 32-page
// single claimed late ends the run long after the rest).
#ifndef PA_SINGLES_LAST
#define PA_SINGLES_LAST 0
#endif
// Sort key of the partial last partition of a multi-partition sequence: its
// pages plus this bias (its merge comes after it), capped below a full one.
#ifndef PA_MERGE_BIAS
#define PA_MERGE_BIAS 0
#endif

namespace {

using pa::fast_exp2;
using pa::pack2_rn;
using pa::store4;

constexpr float kNegInf = -__builtin_huge_valf();

// ----------------------------------------------------------- workspace ----
// header (256 B: int n_pairs, int work) | records int4[batch*max_parts] |
// counters int[batch*Hq] | ml float2[batch*Hq*max_parts] |
// acc float[batch*Hq*max_parts*d]
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t pairs_off, cnt_off, ml_off, acc_off, total;
};

WsLayout ws_layout(int64_t batch, int64_t hq, int64_t d, int64_t max_parts) {
  WsLayout w;
  w.pairs_off = 256;
  w.cnt_off = w.pairs_off + align256(size_t(batch) * max_parts * sizeof(int4));
  w.ml_off = w.cnt_off + align256(size_t(batch) * hq * sizeof(int));
  w.acc_off = w.ml_off + align256(size_t(batch) * hq * max_parts * sizeof(float2));
  w.total = w.acc_off + align256(size_t(batch) * hq * max_parts * d * sizeof(float));
  return w;
}

__device__ __forceinline__ bool len_ok(int n, int max_tokens) { return n >= 1 && n <= max_tokens; }

// ---------------------------------------------------------- plan kernel ----
struct PlanParams {
  const int32_t* lens;
  int64_t len_stride;
  int batch;
  int max_tokens;      // min(max_blocks * B, max_context)
  int block_size;
  int part_blocks;     // partition length in blocks (<= kMaxPartBlocks)
  int4* pairs;         // work records {sequence, partition, length, blocks in partition}
  int* n_pairs;
  int* counters;       // per (sequence, KV head) partition-done counters, zeroed here
  int n_counters;
  int* work;           // dynamic work counter: items below n_workers are taken statically
  int n_workers;       // warps of the attention grid (worker w starts with item w)
};

// Bucket of the non-full item of a sequence of nb blocks (partitions of PB).
__device__ __forceinline__ int sort_key(int nb, int PB) {
  const int r = nb % PB;
  return nb > PB ? min(PB - 1, r + PA_MERGE_BIAS) : r;
}

constexpr int kPlanThreads = 1024;
constexpr int kPlanPer = 4;   // sequences per plan thread kept in registers
constexpr int kMaxPartBlocks = 128;

// Work order (the attention warps take the list front to back): (1) the full
// partitions, (2) every other item -- the partial last partition of a long
// sequence or the only partition of a short one -- by decreasing size.  Large
// items go first and the run ends with the smallest, so the warps finish
// close together.  (With PA_SINGLES_LAST the single partitions form a third
// list of their own after (2).)
__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(PlanParams p) {
  __shared__ int hist_multi[kMaxPartBlocks + 1];    // partial partitions by size
  __shared__ int hist_single[kMaxPartBlocks + 1];   // single partitions by size
  __shared__ int warp_sums[kPlanThreads / 32];
  __shared__ int total_full_s;
  __shared__ int thr_base[kPlanThreads];            // first full record of each thread (one sequence each)
  __shared__ int thr_len[kPlanThreads];
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // let the attention kernel launch now (it waits for this grid), then wait
  // until the previous kernel's results (lengths, cache writes) are visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  const int PB = p.part_blocks;
  for (int i = tid; i <= kMaxPartBlocks; i += blockDim.x) hist_multi[i] = hist_single[i] = 0;
  for (int i = tid; i < p.n_counters; i += blockDim.x) p.counters[i] = 0;
  if (tid == 0) *p.work = p.n_workers;
  __syncthreads();
  const int per = (p.batch + kPlanThreads - 1) / kPlanThreads;
  const int s0 = min(p.batch, tid * per), s1 = min(p.batch, s0 + per);
  // lengths of this thread's sequences, read once (-1 = invalid)
  int nreg[kPlanPer];
#pragma unroll
  for (int k = 0; k < kPlanPer; ++k) {
    const int s = s0 + k;
    nreg[k] = -1;
    if (s < s1) {
      const int n = p.lens[s * p.len_stride];
      if (len_ok(n, p.max_tokens)) nreg[k] = n;
      else decode_flag(PA_DEVERR_CONTEXT_LEN);
    }
  }
  auto len_of = [&](int s) {
    if (s - s0 < kPlanPer) {
      int v = -1;
#pragma unroll
      for (int k = 0; k < kPlanPer; ++k)
        if (k == s - s0) v = nreg[k];
      return v;
    }
    const int n = p.lens[s * p.len_stride];
    if (!len_ok(n, p.max_tokens)) {
      decode_flag(PA_DEVERR_CONTEXT_LEN);
      return -1;
    }
    return n;
  };
  int my_full = 0;
  for (int s = s0; s < s1; ++s) {
    const int n = len_of(s);
    if (n < 0) continue;
    const int nb = (n + p.block_size - 1) / p.block_size;
    if (nb <= PB && PA_SINGLES_LAST) {
      atomicAdd(&hist_single[nb], 1);
    } else {
      my_full += nb / PB;
      if (nb % PB) atomicAdd(&hist_multi[sort_key(nb, PB)], 1);
    }
  }
  // exclusive scan of my_full over the CTA
  const int lane = tid & 31, warp = tid >> 5;
  int x = my_full;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;   // inclusive
    if (lane == 31) total_full_s = w;
  }
  __syncthreads();
  int base = x - my_full + (warp ? warp_sums[warp - 1] : 0);
  if (per == 1) {
    // one sequence per thread: the full records are written by all threads
    // together below (a long sequence has hundreds of them)
    thr_base[tid] = base;
    thr_len[tid] = nreg[0];
  } else {
    for (int s = s0; s < s1; ++s) {
      const int n = len_of(s);
      if (n < 0) continue;
      const int nb = (n + p.block_size - 1) / p.block_size;
      if (nb <= PB && PA_SINGLES_LAST) continue;
      for (int q = 0; q < nb / PB; ++q) p.pairs[base++] = make_int4(s, q, n, PB);
    }
  }
  __syncthreads();
  if (per == 1) {
    const int nthr = p.batch;                        // threads owning a sequence
    for (int e = tid; e < total_full_s; e += kPlanThreads) {
      // owner: the last thread whose first record is at or before e
      int lo = 0, hi = nthr;                         // thr_base[lo] <= e < thr_base[hi] (hi = nthr: end)
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (thr_base[mid] <= e) lo = mid;
        else hi = mid;
      }
      p.pairs[e] = make_int4(lo, e - thr_base[lo], thr_len[lo], PB);
    }
  }
  // bucket offsets: partial partitions (sizes PB-1 .. 1), then singles (PB .. 1)
  if (PB <= 32 && !PA_SINGLES_LAST) {
    if (warp == 0) {
      // lane i: bucket PB-1-i; an exclusive scan in decreasing size order
      const int r = PB - 1 - lane;
      const int c = lane < PB - 1 ? hist_multi[r] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < PB - 1) hist_multi[r] = total_full_s + incl - c;
      if (lane == 31) *p.n_pairs = total_full_s + incl;
    }
  } else if (tid == 0) {
    int off = total_full_s;
    for (int r = PB - 1; r >= 1; --r) {
      const int c = hist_multi[r];
      hist_multi[r] = off;
      off += c;
    }
    for (int r = PB; r >= 1; --r) {
      const int c = hist_single[r];
      hist_single[r] = off;
      off += c;
    }
    *p.n_pairs = off;
  }
  __syncthreads();
  for (int s = s0; s < s1; ++s) {
    const int n = len_of(s);
    if (n < 0) continue;
    const int nb = (n + p.block_size - 1) / p.block_size;
    if (nb <= PB && PA_SINGLES_LAST) {
      p.pairs[atomicAdd(&hist_single[nb], 1)] = make_int4(s, 0, n, nb);
    } else if (nb % PB) {
      p.pairs[atomicAdd(&hist_multi[sort_key(nb, PB)], 1)] = make_int4(s, nb / PB, n, nb % PB);
    }
  }
}

// ------------------------------------------------------ fast decode -------
struct FastParams {
  const void* q;
  int64_t q_s, q_h;               // element strides
  const int32_t* tables;
  int64_t tab_s, tab_b;
  const int32_t* lens;
  int64_t len_s;
  void* out;
  int64_t out_s, out_h;
  float2* ml;
  float* acc;
  const int4* pairs;
  const int* n_pairs;
  int* counters;                  // per (sequence, KV head) finished-partition counters
  int* work;                      // next unclaimed work item
  int hq, hkv, group, num_blocks, max_tokens, part_tokens, part_blocks, max_parts;
  float scale_log2;               // scale * log2(e)
  // pa_decode_append: rows [batch, Hkv, d] of the token at position n - 1 of
  // each sequence, stored into the caches by the warp that attends that
  // token's page (null for pa_decode)
  const void* k_new;
  const void* v_new;
  int64_t kn_s, kn_h, vn_s, vn_h;  // element strides, 16-byte multiples
  void* k_cache;
  void* v_cache;
};

// Warps per CTA, stages per warp and the CTAs per SM the register budget is
// sized for; overridable at build time for tuning sweeps.
#ifndef PA_FAST_WARPS
#define PA_FAST_WARPS 4
#endif
#ifndef PA_FAST_MIN_CTAS
#define PA_FAST_MIN_CTAS 2
#endif
#ifndef PA_FAST_STAGES_D64
#define PA_FAST_STAGES_D64 5
#endif
#ifndef PA_FAST_STAGES_D128
#define PA_FAST_STAGES_D128 3
#endif
#ifndef PA_FAST_STAGES_D256
#define PA_FAST_STAGES_D256 2
#endif
#ifndef PA_FUSED_MERGE
#define PA_FUSED_MERGE 1
#endif
// Sequences with up to this many partitions are merged inside the attention
// kernel by the last warp to finish; longer ones by decode_merge_kernel.
constexpr int kFusedMergeMaxParts = 32;
constexpr int kWarps = PA_FAST_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kBlock = 16;        // tokens per block (page rows)

template <int D> struct FastCfg {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kPageBytes = kBlock * kRowBytes;
  static constexpr int kStages = D == 64 ? PA_FAST_STAGES_D64 : (D == 128 ? PA_FAST_STAGES_D128 : PA_FAST_STAGES_D256);
  static constexpr int kStageBytes = 2 * kPageBytes;          // K page + V page
};

// Byte offset of (row t, 16-byte unit u) in a staged page.  A page is staged
// as [d/64 chunks][16 rows][128 B] by one 2-D tensor copy per chunk with
// 128-byte swizzling: inside a chunk the 16-byte unit index is XORed with the
// row index mod 8, so the same unit of 8 consecutive rows lies in 8 distinct
// bank groups.
__device__ __forceinline__ uint32_t page_off(uint32_t t, uint32_t u) {
  return (u >> 3) * 2048u + t * 128u + (((u & 7u) ^ (t & 7u)) << 4);
}


// ---- MHA math: one query head, fp32 FMAs ---------------------------------
template <typename T, int D> struct MhaMath {
  static constexpr int U = D / 8;            // 16-byte units per row
  static constexpr int TPL = 32 / U;         // tokens per load round
  static constexpr int R = kBlock / TPL;     // load rounds per page
  float q[8];
  float m, lpart;
  float acc[8];
  int cu, tg, lane;

  __device__ __forceinline__ void init(int lane_) {
    lane = lane_;
    cu = lane % U;
    tg = lane / U;
  }
  __device__ __forceinline__ void load_q(const FastParams& p, int s, int hk) {
    const T* qp = static_cast<const T*>(p.q) + s * p.q_s + hk * p.q_h + cu * 8;
    const uint4 w = *reinterpret_cast<const uint4*>(qp);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = pa::unpack2<T>(ws[i]);
      q[2 * i] = f.x * p.scale_log2;
      q[2 * i + 1] = f.y * p.scale_log2;
    }
  }
  __device__ __forceinline__ void reset() {
    m = kNegInf;
    lpart = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  }
  __device__ __forceinline__ float dot8(uint4 w) const {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = pa::unpack2<T>(ws[i]);
      a = fmaf(q[2 * i], f.x, a);
      a = fmaf(q[2 * i + 1], f.y, a);
    }
    return a;
  }
  // kb / vb: shared addresses of the K and V pages.  pos0: position of page
  // row 0; rows at or past n (or all rows of an invalid block) are masked.
  __device__ __forceinline__ void block(uint32_t kb, uint32_t vb, int pos0, int n, bool valid) {
    float v[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int t = i * TPL + tg;
      v[i] = dot8(pa::lds128(kb + page_off(t, cu)));
    }
    // reduce-scatter over the U lanes of a token group
    int idx = 0;
    int cnt = R;
#pragma unroll
    for (int off = U / 2; off >= 1; off >>= 1) {
      const bool b = (lane & off) != 0;
      if (cnt > 1) {
        const int half = cnt / 2;
#pragma unroll
        for (int j = 0; j < half; ++j) {
          const float keep = b ? v[half + j] : v[j];
          const float send = b ? v[j] : v[half + j];
          v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
        idx += b ? half : 0;
        cnt = half;
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
      }
    }
    const int tok = idx * TPL + tg;
    const bool masked = !valid || (pos0 + tok >= n);
    const float sc = masked ? kNegInf : v[0];
    float bmax = sc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
    const float m_new = fmaxf(m, bmax);
    const float m_use = m_new == kNegInf ? 0.f : m_new;
    const float alpha = fast_exp2(m - m_use);
    const float pe = masked ? 0.f : fast_exp2(sc - m_use);
    lpart = lpart * alpha + ((lane & 1) ? 0.f : pe);
    if (alpha != 1.f) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= alpha;
    }
    const bool partial = !valid || (pos0 + kBlock > n);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int t = i * TPL + tg;
      const float pt = __shfl_sync(0xffffffffu, pe, (i << 1) | (tg * U));
      const uint4 w = pa::lds128(vb + page_off(t, cu));
      if (partial && (!valid || pos0 + t >= n)) continue;
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = pa::unpack2<T>(ws[k]);
        acc[2 * k] = fmaf(pt, f.x, acc[2 * k]);
        acc[2 * k + 1] = fmaf(pt, f.y, acc[2 * k + 1]);
      }
    }
    m = m_new;
  }
  float l;
  // Combine the lanes' token groups and the softmax sum.
  __device__ __forceinline__ void finalize() {
#pragma unroll
    for (int off = U; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    l = lpart;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  }
  template <typename TO>
  __device__ __forceinline__ void store_final(TO* row, int64_t /*head_stride*/, int /*heads*/) const {
    if (tg != 0) return;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    store4<TO>(row + cu * 8, make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv));
    store4<TO>(row + cu * 8 + 4, make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv));
  }
  __device__ __forceinline__ void store_partial(float* acc_row, float2* ml, int64_t /*slot_stride*/,
                                                int /*heads*/) const {
    if (tg == 0) {
      float4* dst = reinterpret_cast<float4*>(acc_row + cu * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    if (lane == 0) *ml = make_float2(m, l);
  }
};

// ---- GQA math: 2..8 or 16 query heads share a KV head; tensor-core MMAs ---
template <typename T, int D, int NT> struct GqaMath {
  // NT column tiles of 8 query heads each (NT = 1: up to 8 heads, 2: 16)
  static constexpr int KS = D / 16;   // k-steps of q.k, and d-tiles of p.V
  uint32_t qf[NT][KS][2];
  float m[NT][2], lpart[NT][2];
  // tile n, d-tile t: {O[8n+2c][16t+r], O[8n+2c+1][16t+r], O[8n+2c][16t+8+r], O[8n+2c+1][16t+8+r]}
  float acc[NT][KS][4];
  int r, c, lane;
  uint32_t krow, vrow;   // per-lane ldmatrix row addressing (see block())
  int kb1, vb1;

  __device__ __forceinline__ void init(int lane_) {
    lane = lane_;
    r = lane >> 2;
    c = lane & 3;
    const int mat = lane >> 3, j = lane & 7;
    // K (row-major A, rows = tokens): matrices (rows 0-7 | 8-15) x (d 0-7 | 8-15)
    krow = uint32_t(j + 8 * (mat & 1));
    kb1 = mat >> 1;
    // V (transposed load of V^T, k = tokens): k = 2i <-> token i, k = 2i+1 <->
    // token i+4 (i < 4), +8 for k >= 8; rows of every 8x8 matrix then sit in 8
    // distinct 16-byte bank groups of the swizzled page
    vrow = uint32_t((j >> 1) + 4 * (j & 1) + 8 * (mat >> 1));
    vb1 = mat & 1;
  }
  __device__ __forceinline__ void load_q(const FastParams& p, int s, int hk) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int h = 8 * n + r;
      const bool live = h < p.group;
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(static_cast<const T*>(p.q) + s * p.q_s +
                                                             (hk * p.group + (live ? h : 0)) * p.q_h);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qf[n][ks][0] = live ? qw[8 * ks + c] : 0u;
        qf[n][ks][1] = live ? qw[8 * ks + 4 + c] : 0u;
      }
    }
  }
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      m[n][0] = m[n][1] = kNegInf;
      lpart[n][0] = lpart[n][1] = 0.f;
#pragma unroll
      for (int t = 0; t < KS; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][t][e] = 0.f;
    }
  }
  __device__ __forceinline__ void block(uint32_t kb, uint32_t vb, int pos0, int n_tok, bool valid,
                                        float scale_log2) {
    // ---- S = K_page q^T : rows = tokens, cols = heads (8n + 2c, 8n + 2c + 1 on this lane)
    float sc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      pa::ldsm_x4(kb + page_off(krow, 2 * ks + kb1), a0, a1, a2, a3);
#pragma unroll
      for (int n = 0; n < NT; ++n) pa::mma16816<T>(sc[n], a0, a1, a2, a3, qf[n][ks][0], qf[n][ks][1]);
    }
    const bool mask_a = !valid || (pos0 + r >= n_tok);
    const bool mask_b = !valid || (pos0 + r + 8 >= n_tok);
    float al[NT][2];
    uint32_t b01h[NT], b23h[NT], b01l[NT], b23l[NT];
    bool rescale = false;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      sc[n][0] = mask_a ? kNegInf : sc[n][0] * scale_log2;
      sc[n][1] = mask_a ? kNegInf : sc[n][1] * scale_log2;
      sc[n][2] = mask_b ? kNegInf : sc[n][2] * scale_log2;
      sc[n][3] = mask_b ? kNegInf : sc[n][3] * scale_log2;
      // ---- online softmax per head
      float mx0 = fmaxf(sc[n][0], sc[n][2]), mx1 = fmaxf(sc[n][1], sc[n][3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m[n][0], mx0), mn1 = fmaxf(m[n][1], mx1);
      const float mu0 = mn0 == kNegInf ? 0.f : mn0, mu1 = mn1 == kNegInf ? 0.f : mn1;
      al[n][0] = fast_exp2(m[n][0] - mu0);
      al[n][1] = fast_exp2(m[n][1] - mu1);
      const float p0 = fast_exp2(sc[n][0] - mu0), p1 = fast_exp2(sc[n][1] - mu1);
      const float p2 = fast_exp2(sc[n][2] - mu0), p3 = fast_exp2(sc[n][3] - mu1);
      lpart[n][0] = lpart[n][0] * al[n][0] + p0 + p2;
      lpart[n][1] = lpart[n][1] * al[n][1] + p1 + p3;
      m[n][0] = mn0;
      m[n][1] = mn1;
      rescale = rescale || al[n][0] != 1.f || al[n][1] != 1.f;
      // ---- P as two 16-bit terms (hi + lo), moved from the S layout to the
      // B-operand layout of P^T: b01 = P[token c, c+4][h], b23 = P[token c+8, c+12][h]
      const uint32_t z0h = pack2_rn<T>(p0, p1), z1h = pack2_rn<T>(p2, p3);
      const float2 f0 = pa::unpack2<T>(z0h), f1 = pa::unpack2<T>(z1h);
      const uint32_t z0l = pack2_rn<T>(p0 - f0.x, p1 - f0.y), z1l = pack2_rn<T>(p2 - f1.x, p3 - f1.y);
      const int src0 = c * 4 + (r >> 1), src1 = (c + 4) * 4 + (r >> 1);
      const uint32_t sel = (r & 1) ? 0x7632u : 0x5410u;
      b01h[n] = pa::prmt(__shfl_sync(0xffffffffu, z0h, src0), __shfl_sync(0xffffffffu, z0h, src1), sel);
      b23h[n] = pa::prmt(__shfl_sync(0xffffffffu, z1h, src0), __shfl_sync(0xffffffffu, z1h, src1), sel);
      b01l[n] = pa::prmt(__shfl_sync(0xffffffffu, z0l, src0), __shfl_sync(0xffffffffu, z0l, src1), sel);
      b23l[n] = pa::prmt(__shfl_sync(0xffffffffu, z1l, src0), __shfl_sync(0xffffffffu, z1l, src1), sel);
    }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int t = 0; t < KS; ++t) {
          acc[n][t][0] *= al[n][0];
          acc[n][t][1] *= al[n][1];
          acc[n][t][2] *= al[n][0];
          acc[n][t][3] *= al[n][1];
        }
    }
    // ---- O^T += V^T P^T  (masked rows of V were zeroed in shared memory)
#pragma unroll
    for (int t = 0; t < KS; ++t) {
      uint32_t x0, x1, x2, x3;
      pa::ldsm_x4_trans(vb + page_off(vrow, 2 * t + vb1), x0, x1, x2, x3);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        pa::mma16816<T>(acc[n][t], x0, x1, x2, x3, b01h[n], b23h[n]);
        pa::mma16816<T>(acc[n][t], x0, x1, x2, x3, b01l[n], b23l[n]);
      }
    }
  }
  float l[NT][2];
  // Softmax sums over the lanes that share a head.
  __device__ __forceinline__ void finalize() {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      l[n][0] = lpart[n][0];
      l[n][1] = lpart[n][1];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l[n][0] += __shfl_xor_sync(0xffffffffu, l[n][0], off);
        l[n][1] += __shfl_xor_sync(0xffffffffu, l[n][1], off);
      }
    }
  }
  // Lane (r, c) holds heads 8n + 2c, 8n + 2c + 1 at d = 16t + r and 16t + 8 + r.
  template <typename TO>
  __device__ __forceinline__ void store_final(TO* row0, int64_t head_stride, int heads) const {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int head = 8 * n + 2 * c + e;
        if (head >= heads) continue;
        TO* row = row0 + head * head_stride;
        const float inv = l[n][e] > 0.f ? 1.f / l[n][e] : 0.f;
#pragma unroll
        for (int t = 0; t < KS; ++t) {
          row[16 * t + r] = pa::from_f32<TO>(acc[n][t][e] * inv);
          row[16 * t + 8 + r] = pa::from_f32<TO>(acc[n][t][2 + e] * inv);
        }
      }
  }
  __device__ __forceinline__ void store_partial(float* acc_row0, float2* ml0, int64_t slot_stride,
                                                int heads) const {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int head = 8 * n + 2 * c + e;
        if (head >= heads) continue;
        float* row = acc_row0 + head * slot_stride * D;
#pragma unroll
        for (int t = 0; t < KS; ++t) {
          row[16 * t + r] = acc[n][t][e];
          row[16 * t + 8 + r] = acc[n][t][2 + e];
        }
        if (r == 0) ml0[head * slot_stride] = make_float2(m[n][e], l[n][e]);
      }
  }
};

// Fused append: the new token (position n - 1, row r of the staged page whose
// physical block is blk) is stored into both caches and into the staged K and
// V pages, which the tensor copy filled with the row's previous contents.
// Nothing else reads that cache row in this launch: the block holding a
// sequence's newest token belongs to that sequence alone (a shared block is
// copied before it is written), and only this (sequence, KV head)'s last item
// stages the page.
template <typename T, int D>
__device__ __forceinline__ void append_row(const FastParams& p, int s, int hk, int blk, int r, uint32_t kb,
                                           int lane) {
  constexpr int kUnits = D / 8;   // 16-byte units per row
  const int64_t row = (int64_t(blk) * p.hkv + hk) * kBlock + r;
  for (int e = lane; e < 2 * kUnits; e += 32) {
    const bool is_v = e >= kUnits;
    const int u = is_v ? e - kUnits : e;
    const T* src = static_cast<const T*>(is_v ? p.v_new : p.k_new) + int64_t(s) * (is_v ? p.vn_s : p.kn_s) +
                   int64_t(hk) * (is_v ? p.vn_h : p.kn_h) + 8 * u;
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(src));
    *reinterpret_cast<uint4*>(static_cast<T*>(is_v ? p.v_cache : p.k_cache) + row * D + 8 * u) = x;
    pa::sts128(kb + (is_v ? FastCfg<D>::kPageBytes : 0) + page_off(r, u), x);
  }
  __syncwarp();
}

// Merge of the np (<= 32) partition states of query heads qh0 .. qh0+nh-1
// (nh <= HC) of sequence s:  M = max m_p, L = sum l_p 2^(m_p - M),
// out = sum 2^(m_p - M) acc_p / L  (scores in base 2).
// Latency-bound: the states were just written by other warps and sit in L2.
// Lane q loads partition q's (m, l) of every head of the chunk at once (one
// round trip); then each lane owns the same CPL float4 columns of every head
// and reads the accumulators of QB partitions x HC heads per round trip (8
// independent 16-byte loads), taking each weight's m_p from lane p by a
// shuffle.
template <typename TO, int D, int HC>
__device__ __forceinline__ void merge_chunk(const FastParams& p, int s, int qh0, int nh, int np, int lane) {
  constexpr int kCols = D / 4;                        // float4 columns of a row
  constexpr int CPL = kCols >= 32 ? kCols / 32 : 1;    // columns per lane
  constexpr int QB = (8 / (HC * CPL)) > 0 ? 8 / (HC * CPL) : 1;
  float mq[HC], M[HC], inv[HC];
#pragma unroll
  for (int h = 0; h < HC; ++h) {
    const int64_t base = (int64_t(s) * p.hq + qh0 + h) * p.max_parts;
    const float2 ml = lane < np && h < nh ? __ldcg(&p.ml[base + lane]) : make_float2(kNegInf, 0.f);
    mq[h] = ml.x;
    M[h] = ml.y;   // l for now
  }
#pragma unroll
  for (int h = 0; h < HC; ++h) {
    float mx = mq[h];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float mu = mx == kNegInf ? 0.f : mx;
    float l = lane < np ? M[h] * fast_exp2(mq[h] - mu) : 0.f;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    M[h] = mu;
    inv[h] = l > 0.f ? 1.f / l : 0.f;
  }
  float4 a[HC][CPL];
#pragma unroll
  for (int h = 0; h < HC; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c) a[h][c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
  for (int q0 = 0; q0 < np; q0 += QB) {
    float4 x[QB][HC][CPL];
#pragma unroll
    for (int u = 0; u < QB; ++u)
#pragma unroll
      for (int h = 0; h < HC; ++h)
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const int col = lane + 32 * c;
          const int64_t row = (int64_t(s) * p.hq + qh0 + h) * p.max_parts + q0 + u;
          x[u][h][c] = q0 + u < np && h < nh && col < kCols
                           ? __ldcg(reinterpret_cast<const float4*>(p.acc + row * D) + col)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
    for (int u = 0; u < QB; ++u)
#pragma unroll
      for (int h = 0; h < HC; ++h) {
        const float m = __shfl_sync(0xffffffffu, mq[h], (q0 + u) & 31);
        const float w = q0 + u < np ? fast_exp2(m - M[h]) : 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          a[h][c].x = fmaf(x[u][h][c].x, w, a[h][c].x);
          a[h][c].y = fmaf(x[u][h][c].y, w, a[h][c].y);
          a[h][c].z = fmaf(x[u][h][c].z, w, a[h][c].z);
          a[h][c].w = fmaf(x[u][h][c].w, w, a[h][c].w);
        }
      }
  }
#pragma unroll
  for (int h = 0; h < HC; ++h) {
    TO* dst = static_cast<TO*>(p.out) + s * p.out_s + (qh0 + h) * p.out_h;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int col = lane + 32 * c;
      if (col < kCols && h < nh)
        store4<TO>(dst + 4 * col, make_float4(a[h][c].x * inv[h], a[h][c].y * inv[h], a[h][c].z * inv[h],
                                              a[h][c].w * inv[h]));
    }
  }
}

// All `heads` heads of an item, HC at a time.
template <typename TO, int D, int HC>
__device__ __forceinline__ void merge_states(const FastParams& p, int s, int qh0, int heads, int np, int lane) {
#pragma unroll 1
  for (int h0 = 0; h0 < heads; h0 += HC) merge_chunk<TO, D, HC>(p, s, qh0 + h0, min(HC, heads - h0), np, lane);
}

// Work item = (sequence s, partition p, KV head hk); the plan lists (s, p).
struct Item {
  int s, hk, part, n, blk0, nblk;
};

__device__ __forceinline__ Item item_from_record(const FastParams& p, int4 rec, int idx) {
  Item it;
  it.s = rec.x;
  it.part = rec.y;
  it.n = rec.z;
  it.nblk = rec.w;
  it.hk = idx % p.hkv;
  it.blk0 = it.part * p.part_blocks;
  return it;
}

// Block ids of an item, one per lane (lane j holds logical block blk0 + j).
__device__ __forceinline__ int load_ids(const FastParams& p, const Item& it, int lane) {
  return lane < it.nblk ? p.tables[it.s * p.tab_s + int64_t(it.blk0 + lane) * p.tab_b] : -1;
}

constexpr int kItemRing = 8;   // items started by the producer ahead of the consumer, per warp
// ring entry: s, hk, part, n, blk0, nblk (ints 0..5), then the 32 block ids
constexpr int kRingIds = 8;
constexpr int kRingInts = kRingIds + 32;

// Persistent kernel; every warp is an independent worker.  A warp claims whole
// partitions (largest first) from a global counter, streams their pages
// through its own ring of shared-memory stages with tensor copies issued up to
// S pages ahead (across item boundaries), and writes each partition's output
// -- or its (m, l, acc) state, the last warp of a (sequence, KV head) then
// merging all partitions of it.  No CTA-wide synchronisation after set-up.
// NT = 0: one query head per KV head (MHA); NT = 1, 2: tensor-core GQA with
// NT tiles of 8 query heads (groups of 2..8, 16).
template <typename T, typename TO, int D, int NT>
__global__ void __launch_bounds__(kThreads, PA_FAST_MIN_CTAS)
    decode_fast_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const FastParams p) {
  using Cfg = FastCfg<D>;
  constexpr bool GQA = NT > 0;
  using Math = typename std::conditional<GQA, GqaMath<T, D, (NT > 0 ? NT : 1)>, MhaMath<T, D>>::type;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kWarps * S * Cfg::kStageBytes) + warp * S;
  int* ring = reinterpret_cast<int*>(smem + kWarps * S * Cfg::kStageBytes + kWarps * S * sizeof(uint64_t)) +
              warp * kItemRing * kRingInts;
  const uint32_t stage0 = pa::smem_addr(smem + warp * S * Cfg::kStageBytes);
  if (lane == 0) {
    for (int i = 0; i < S; ++i) pa::mbar_init(&full[i], 1);
    pa::fence_mbar_init();
    pa::fence_proxy_async_smem();
    pa::prefetch_tensormap(&kmap);
    pa::prefetch_tensormap(&vmap);
  }
  __syncwarp();

  // the plan kernel (a programmatic prerequisite) must be complete from here on
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int total = *p.n_pairs * p.hkv;
  const uint64_t policy = pa::l2_evict_first_policy();
  const int heads_item = GQA ? p.group : 1;

  // ---- producer side: claims items, issues page copies S pages ahead
  // The item after the one being issued goes through a short pipeline, one
  // step per issued page, so that no step waits on a load started in the same
  // step: stage 1 = its index is known (lane 0 claimed it from the shared
  // counter), 2 = its work record is being read, 3 = its block ids are being
  // read (and its q rows prefetched to L2).  The claim is made kClaimAhead
  // pages before the current item's pages run out: late enough to keep the
  // end of the run balanced, early enough that the loads have landed when the
  // item starts.  Each started item goes to the consumer through a ring in
  // shared memory (decoded fields + block ids), so the consumer reloads
  // nothing but q.
  constexpr int kClaimAhead = 2;
  int nx_stage = 1;
  int nx_claim = blockIdx.x * kWarps + warp;   // lane 0's copy is the index
  int nx_idx = 0, nx_ids = -1;
  int4 nx_rec = make_int4(0, 0, 0, 0);
  Item nx_it;
  nx_it.nblk = 0;
  int ring_w = 0;
  Item is_it;
  int is_ids = -1, is_j = 0;
  is_it.nblk = 0;
  bool is_done = false;
  int st_i = 0;
  uint32_t n_issued = 0;
  auto advance = [&]() {
    if (nx_stage == 0) {
      if (lane == 0) nx_claim = atomicAdd(p.work, 1);
      nx_stage = 1;
    } else if (nx_stage == 1) {
      nx_idx = __shfl_sync(0xffffffffu, nx_claim, 0);
      if (nx_idx < total) nx_rec = __ldg(&p.pairs[nx_idx / p.hkv]);
      nx_stage = 2;
    } else if (nx_stage == 2) {
      if (nx_idx < total) {
        nx_it = item_from_record(p, nx_rec, nx_idx);
        nx_ids = load_ids(p, nx_it, lane);
        if (lane < heads_item) {
          const T* qrow = static_cast<const T*>(p.q) + nx_it.s * p.q_s +
                          int64_t(GQA ? nx_it.hk * p.group + lane : nx_it.hk) * p.q_h;
          pa::prefetch_l2_bulk(qrow, D * int(sizeof(T)));
        }
      }
      nx_stage = 3;
    }
  };
  auto issue_next = [&]() {
    while (is_j >= is_it.nblk) {
      if (is_done) return;
      while (nx_stage < 3) advance();
      int* ent = ring + ring_w * kRingInts;
      ring_w = (ring_w + 1) & (kItemRing - 1);
      if (nx_idx >= total) {
        is_done = true;
        if (lane == 0) ent[0] = -1;
        return;
      }
      is_it = nx_it;
      is_ids = nx_ids;
      is_j = 0;
      if (lane == 0) {
        ent[0] = is_it.s;
        ent[1] = is_it.hk;
        ent[2] = is_it.part;
        ent[3] = is_it.n;
        ent[4] = is_it.blk0;
        ent[5] = is_it.nblk;
      }
      ent[kRingIds + lane] = is_ids;
      nx_stage = 0;
    }
    const int blk = __shfl_sync(0xffffffffu, is_ids, is_j);
    if (lane == 0) {
      uint64_t* bar = &full[st_i];
      if (blk >= 0 && blk < p.num_blocks) {
        pa::fence_proxy_async_smem();
        pa::mbar_arrive_expect_tx(bar, Cfg::kStageBytes);
        const int row = (blk * p.hkv + is_it.hk) * kBlock;
        const uint32_t dst = stage0 + st_i * Cfg::kStageBytes;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          pa::tma_load_2d(dst + ch * 2048, &kmap, bar, 64 * ch, row, policy);
          pa::tma_load_2d(dst + Cfg::kPageBytes + ch * 2048, &vmap, bar, 64 * ch, row, policy);
        }
      } else {
        decode_flag(PA_DEVERR_BLOCK_ID);
        pa::mbar_arrive(bar);
      }
    }
    ++n_issued;
    ++is_j;
    if (++st_i == S) st_i = 0;
    // claim the next item no earlier than kClaimAhead pages before it is
    // needed: earlier claims pin items to this warp and undo the balancing
    // at the end of the run
    if (nx_stage == 1 || nx_stage == 2 || (nx_stage == 0 && is_it.nblk - is_j <= kClaimAhead)) advance();
  };
#pragma unroll 1
  for (int i = 0; i < S; ++i) issue_next();

  // ---- finishing a partition of a multi-partition sequence: count it, and
  // the last warp of a (sequence, KV head) merges all its partitions:
  // M = max m_p, L = sum l_p 2^(m_p - M), out = sum 2^(m_p - M) acc_p / L
  auto release = [&](int s_, int hk_, int np) {
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence();
      last = atomicAdd(&p.counters[s_ * p.hkv + hk_], 1) == np - 1;
      if (last) __threadfence();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    const int qh0 = GQA ? hk_ * p.group : hk_;
    merge_states<TO, D, (GQA ? 4 : 1)>(p, s_, qh0, heads_item, np, lane);
  };
  int pend_s = 0, pend_hk = 0, pend_np = 0;

  // ---- consumer side
  Math math;
  math.init(lane);
  int ring_r = 0, st_c = 0;
  uint32_t ph_c = 0, n_used = 0;
  bool timed_out = false;
#pragma unroll 1
  while (!timed_out) {
    __syncwarp();
    const int* ent = ring + ring_r * kRingInts;
    Item it;
    it.s = ent[0];
    if (it.s < 0) break;
    it.hk = ent[1];
    it.part = ent[2];
    it.n = ent[3];
    it.blk0 = ent[4];
    it.nblk = ent[5];
    const int ids = ent[kRingIds + lane];
    ring_r = (ring_r + 1) & (kItemRing - 1);
    math.load_q(p, it.s, it.hk);
    math.reset();
#pragma unroll 1
    for (int j = 0; j < it.nblk; ++j) {
      if (!pa::mbar_wait_bounded(&full[st_c], ph_c)) {
        timed_out = true;
        if (lane == 0) decode_flag(PA_DEVERR_WAIT_TIMEOUT);
        break;
      }
      const int blk = __shfl_sync(0xffffffffu, ids, j);
      const bool valid = blk >= 0 && blk < p.num_blocks;
      const int pos0 = (it.blk0 + j) * kBlock;
      const uint32_t kb = stage0 + st_c * Cfg::kStageBytes;
      if constexpr (GQA) {
        if (!valid || pos0 + kBlock > it.n) {
          // rows past the sequence (or a whole skipped page) may hold anything:
          // zero them so the p.V product sees 0 * 0 there
          const int keep = valid ? it.n - pos0 : 0;
          for (int e = lane; e < (kBlock - keep) * (D / 8); e += 32)
            pa::sts128_zero(kb + Cfg::kPageBytes + page_off(keep + e / (D / 8), e % (D / 8)));
          __syncwarp();
        }
      }
      if (p.k_new != nullptr && valid && pos0 + kBlock >= it.n)
        append_row<T, D>(p, it.s, it.hk, blk, it.n - 1 - pos0, kb, lane);
      if constexpr (GQA) {
        math.block(kb, kb + Cfg::kPageBytes, pos0, it.n, valid, p.scale_log2);
      } else {
        math.block(kb, kb + Cfg::kPageBytes, pos0, it.n, valid);
      }
      __syncwarp();
      ++n_used;
      if (++st_c == S) {
        st_c = 0;
        ph_c ^= 1u;
      }
      issue_next();
    }
    if (timed_out) break;
    math.finalize();
    // publish the previous partition's partials now: their stores are long done
    if (pend_np) release(pend_s, pend_hk, pend_np);
    pend_np = 0;
    const int np = (it.n + p.part_tokens - 1) / p.part_tokens;
    const int qh0 = GQA ? it.hk * p.group : it.hk;
    if (np == 1) {
      math.store_final(static_cast<TO*>(p.out) + it.s * p.out_s + qh0 * p.out_h, p.out_h, heads_item);
      continue;
    }
    const int64_t slot0 = (int64_t(it.s) * p.hq + qh0) * p.max_parts + it.part;
    math.store_partial(p.acc + slot0 * D, p.ml + slot0, int64_t(p.max_parts), heads_item);
    if (PA_FUSED_MERGE && np <= kFusedMergeMaxParts) {
      pend_s = it.s;
      pend_hk = it.hk;
      pend_np = np;
    }
  }
  if (pend_np) release(pend_s, pend_hk, pend_np);
  // Drain this warp's copies still in flight before it exits (bounded waits).
  while (n_used < n_issued) {
    if (!pa::mbar_wait_bounded(&full[st_c], ph_c)) break;
    ++n_used;
    if (++st_c == S) {
      st_c = 0;
      ph_c ^= 1u;
    }
  }
}

// ------------------------------------------------------ append rows -------
// The new token's K/V rows for pa_decode_append when the attention kernel
// cannot store them itself (generic path, or rows not 16-byte aligned): the
// slot of position n - 1 of sequence s is table[s][(n-1) / B] * B + (n-1) % B.
struct AppendParams {
  const void* k_new;
  const void* v_new;
  int64_t kn_s, kn_h, vn_s, vn_h;   // element strides (last dimension contiguous)
  void* k_cache;
  void* v_cache;
  const int32_t* tables;
  int64_t tab_s, tab_b;
  const int32_t* lens;
  int64_t len_s;
  int hkv, d, block_size, num_blocks, max_tokens;
};

// One CTA per (sequence, KV head); E is the element's bit container.
template <typename E>
__global__ void __launch_bounds__(128) append_rows_kernel(const AppendParams p) {
  const int s = blockIdx.x / p.hkv, hk = blockIdx.x % p.hkv;
  const int n = p.lens[s * p.len_s];
  if (!len_ok(n, p.max_tokens)) return;   // flagged by the attention kernels
  const int pos = n - 1;
  const int blk = p.tables[s * p.tab_s + int64_t(pos / p.block_size) * p.tab_b];
  if (blk < 0 || blk >= p.num_blocks) {
    if (threadIdx.x == 0) decode_flag(PA_DEVERR_BLOCK_ID);
    return;
  }
  const int64_t row = ((int64_t(blk) * p.hkv + hk) * p.block_size + pos % p.block_size) * p.d;
  const E* kn = static_cast<const E*>(p.k_new) + int64_t(s) * p.kn_s + int64_t(hk) * p.kn_h;
  const E* vn = static_cast<const E*>(p.v_new) + int64_t(s) * p.vn_s + int64_t(hk) * p.vn_h;
  for (int e = threadIdx.x; e < p.d; e += blockDim.x) {
    static_cast<E*>(p.k_cache)[row + e] = kn[e];
    static_cast<E*>(p.v_cache)[row + e] = vn[e];
  }
}

// ------------------------------------------------------ generic decode ----
struct GenericParams {
  const void* q;
  int64_t q_s, q_h;
  const void* k_cache;
  const void* v_cache;
  const int32_t* tables;
  int64_t tab_s, tab_b;
  const int32_t* lens;
  int64_t len_s;
  void* out;
  int64_t out_s, out_h;
  float2* ml;
  float* acc;
  int hq, hkv, group, d, block_size, num_blocks, max_tokens, part_tokens, max_parts;
  float scale_log2;
};

constexpr int kGenericMaxD = 512;
constexpr int kGenericRegs = kGenericMaxD / 32;

// grid (partition, q head, sequence); kGenericWarps warps take tokens
// round-robin.  Latency-bound on short rows: each token costs a block-table
// load and then its K and V rows, so the next token's table entry is fetched
// while the current one is processed, K and V of a token are loaded together,
// and a CTA has 16 warps so that a short sequence takes few rounds.
constexpr int kGenericWarps = 16;

template <typename T, typename TO>
__global__ void __launch_bounds__(kGenericWarps * 32) decode_generic_kernel(const GenericParams p) {
  __shared__ float s_m[kGenericWarps], s_l[kGenericWarps];
  __shared__ float s_acc[kGenericWarps][kGenericMaxD];
  const int part = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = p.lens[s * p.len_s];
  if (!len_ok(n, p.max_tokens)) {
    if (part == 0 && h == 0 && threadIdx.x == 0) decode_flag(PA_DEVERR_CONTEXT_LEN);
    return;
  }
  const int np = (n + p.part_tokens - 1) / p.part_tokens;
  if (part >= np) return;
  const int hk = h / p.group;
  const int t0 = part * p.part_tokens, t1 = min(n, t0 + p.part_tokens);
  const T* qp = static_cast<const T*>(p.q) + s * p.q_s + h * p.q_h;
  float q[kGenericRegs], acc[kGenericRegs];
#pragma unroll
  for (int i = 0; i < kGenericRegs; ++i) {
    const int d = lane + 32 * i;
    q[i] = d < p.d ? pa::to_f32(qp[d]) * p.scale_log2 : 0.f;
    acc[i] = 0.f;
  }
  float m = kNegInf, l = 0.f;
  const T* kc = static_cast<const T*>(p.k_cache);
  const T* vc = static_cast<const T*>(p.v_cache);
  auto table_at = [&](int t) { return t < t1 ? p.tables[s * p.tab_s + int64_t(t / p.block_size) * p.tab_b] : -1; };
  int blk_next = table_at(t0 + warp);
  for (int t = t0 + warp; t < t1; t += kGenericWarps) {
    const int blk = blk_next;
    blk_next = table_at(t + kGenericWarps);
    if (blk < 0 || blk >= p.num_blocks) {
      if (lane == 0) decode_flag(PA_DEVERR_BLOCK_ID);
      continue;
    }
    const int64_t row = ((int64_t(blk) * p.hkv + hk) * p.block_size + t % p.block_size) * p.d;
    float kr[kGenericRegs], vr[kGenericRegs];
#pragma unroll
    for (int i = 0; i < kGenericRegs; ++i) {
      const int d = lane + 32 * i;
      kr[i] = d < p.d ? pa::to_f32(kc[row + d]) : 0.f;
      vr[i] = d < p.d ? pa::to_f32(vc[row + d]) : 0.f;
    }
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < kGenericRegs; ++i) dot = fmaf(q[i], kr[i], dot);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float m_new = fmaxf(m, dot);
    const float alpha = exp2f(m - m_new);
    const float pe = exp2f(dot - m_new);
    l = l * alpha + pe;
#pragma unroll
    for (int i = 0; i < kGenericRegs; ++i) acc[i] = fmaf(pe, vr[i], acc[i] * alpha);
    m = m_new;
  }
  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int i = 0; i < kGenericRegs; ++i) {
    const int d = lane + 32 * i;
    if (d < p.d) s_acc[warp][d] = acc[i];
  }
  __syncthreads();
  float M = kNegInf;
  for (int w = 0; w < kGenericWarps; ++w) M = fmaxf(M, s_m[w]);
  const float Mu = M == kNegInf ? 0.f : M;
  float wt[kGenericWarps], L = 0.f;
#pragma unroll
  for (int w = 0; w < kGenericWarps; ++w) {
    wt[w] = exp2f(s_m[w] - Mu);
    L += s_l[w] * wt[w];
  }
  for (int d = threadIdx.x; d < p.d; d += blockDim.x) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kGenericWarps; ++w) a += s_acc[w][d] * wt[w];
    if (np == 1) {
      TO* o = static_cast<TO*>(p.out) + s * p.out_s + h * p.out_h;
      o[d] = pa::from_f32<TO>(L > 0.f ? a / L : 0.f);
    } else {
      const int64_t slot = (int64_t(s) * p.hq + h) * p.max_parts + part;
      p.acc[slot * p.d + d] = a;
      if (d == 0) p.ml[slot] = make_float2(M, L);
    }
  }
}

// -------------------------------------------------------- merge kernel ----
struct MergeParams {
  const int32_t* lens;
  int64_t len_s;
  const float2* ml;
  const float* acc;
  void* out;
  int64_t out_s, out_h;
  int hq, d, max_tokens, part_tokens, max_parts;
  int min_parts;   // rows with fewer partitions were already merged
};

// One CTA of kMergeWarps warps per (query head, sequence).  Latency-bound (a
// few hundred partitions of one row at most): the maximum and the sum take one
// pass with the partitions spread over the threads; then each warp takes every
// kMergeWarps-th partition, each lane four columns, with kMergeUnroll
// independent loads in flight, and the warps' sums are added in shared memory.
constexpr int kMergeWarps = 8;
constexpr int kMergeUnroll = 4;

template <typename TO>
__global__ void __launch_bounds__(kMergeWarps * 32) decode_merge_kernel(const MergeParams p) {
  __shared__ float red[kMergeWarps];
  __shared__ float s_M, s_L;
  __shared__ __align__(16) float part[kMergeWarps][kGenericMaxD];
  // launched as a programmatic dependent of the attention kernel: its
  // partition states must be complete and visible from here on
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int h = blockIdx.x, s = blockIdx.y;
  const int n = p.lens[s * p.len_s];
  if (!len_ok(n, p.max_tokens)) return;
  const int np = (n + p.part_tokens - 1) / p.part_tokens;
  if (np <= 1 || np < p.min_parts) return;
  const int64_t base = (int64_t(s) * p.hq + h) * p.max_parts;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kT = kMergeWarps * 32;
  float mx = kNegInf;
  for (int i = tid; i < np; i += kT) mx = fmaxf(mx, p.ml[base + i].x);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (tid == 0) {
    float m = red[0];
    for (int w = 1; w < kMergeWarps; ++w) m = fmaxf(m, red[w]);
    s_M = m == kNegInf ? 0.f : m;
  }
  __syncthreads();
  const float M = s_M;
  float sum = 0.f;
  for (int i = tid; i < np; i += kT) {
    const float2 v = p.ml[base + i];
    sum += v.y * exp2f(v.x - M);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  __syncthreads();
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  if (tid == 0) {
    float l = 0.f;
    for (int w = 0; w < kMergeWarps; ++w) l += red[w];
    s_L = l;
  }
  // this warp's partitions, columns c = 4 * lane + 128 * k
  const bool vec = (p.d & 3) == 0;
  for (int c0 = 0; c0 < p.d; c0 += 128) {
    const int c = c0 + 4 * lane;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = warp; i0 < np; i0 += kMergeWarps * kMergeUnroll) {
      float4 x[kMergeUnroll];
      float w[kMergeUnroll];
#pragma unroll
      for (int u = 0; u < kMergeUnroll; ++u) {
        const int i = i0 + u * kMergeWarps;
        x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        w[u] = 0.f;
        if (i < np) {
          const float* row = p.acc + (base + i) * p.d;
          w[u] = p.ml[base + i].x;
          if (vec) {
            if (c < p.d) x[u] = *reinterpret_cast<const float4*>(row + c);
          } else {
            x[u].x = c < p.d ? row[c] : 0.f;
            x[u].y = c + 1 < p.d ? row[c + 1] : 0.f;
            x[u].z = c + 2 < p.d ? row[c + 2] : 0.f;
            x[u].w = c + 3 < p.d ? row[c + 3] : 0.f;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kMergeUnroll; ++u) {
        const float wt = i0 + u * kMergeWarps < np ? exp2f(w[u] - M) : 0.f;
        a.x = fmaf(x[u].x, wt, a.x);
        a.y = fmaf(x[u].y, wt, a.y);
        a.z = fmaf(x[u].z, wt, a.z);
        a.w = fmaf(x[u].w, wt, a.w);
      }
    }
    if (c < p.d) {
      part[warp][c] = a.x;
      if (c + 1 < p.d) part[warp][c + 1] = a.y;
      if (c + 2 < p.d) part[warp][c + 2] = a.z;
      if (c + 3 < p.d) part[warp][c + 3] = a.w;
    }
  }
  __syncthreads();
  const float inv = s_L > 0.f ? 1.f / s_L : 0.f;
  TO* o = static_cast<TO*>(p.out) + s * p.out_s + h * p.out_h;
  for (int d = tid; d < p.d; d += kT) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) t += part[w][d];
    o[d] = pa::from_f32<TO>(t * inv);
  }
}

// ----------------------------------------------------------- host side ----
int g_decode_path = 0;   // PA_OPT_DECODE_PATH

// Measurement hook: CUDA event pairs recorded around the main decode kernel.
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> spare;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending;
  cudaEvent_t get() {
    if (!spare.empty()) {
      cudaEvent_t e = spare.back();
      spare.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};
Profiler& profiler() {
  static Profiler p;
  return p;
}
struct ProfileScope {
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  explicit ProfileScope(cudaStream_t st) : s(st) {
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    if (!p.on) return;
    a = p.get();
    b = p.get();
    if (a && b) cudaEventRecord(a, s);
  }
  ~ProfileScope() {
    if (!a || !b) return;
    cudaEventRecord(b, s);
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    p.pending.emplace_back(a, b);
  }
};

int cuda_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return PA_OK;
}

struct DeviceInfo {
  int sms = 148;
};

DeviceInfo device_info() {
  DeviceInfo di;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
  return di;
}

// With grid_out set: report the persistent grid size only.  Otherwise launch
// it as a programmatic dependent of the plan kernel just enqueued on `s`.
template <typename T, typename TO, int D, int NT>
int launch_fast(const CUtensorMap* km, const CUtensorMap* vm, const FastParams* fp, cudaStream_t s,
                int* grid_out) {
  using Cfg = FastCfg<D>;
  const size_t smem = 1024 + size_t(kWarps) * Cfg::kStages * Cfg::kStageBytes +
                      size_t(kWarps) * Cfg::kStages * sizeof(uint64_t) +
                      size_t(kWarps) * kItemRing * kRingInts * sizeof(int);
  auto kern = decode_fast_kernel<T, TO, D, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("smem attribute: ") + cudaGetErrorString(e));
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess || per_sm < 1) per_sm = 1;
  const int grid = device_info().sms * per_sm;
  if (grid_out) {
    *grid_out = grid;
    return PA_OK;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, *km, *vm, *fp);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("decode fast kernel launch: ") + cudaGetErrorString(e));
  pa::count_launches(1);
  return cuda_status("decode fast kernel launch");
}

// nt: head tiles of the GQA math (0 = MHA); nt = 2 exists for d = 64, 128
template <typename T, typename TO>
int dispatch_fast(int d, int nt, const CUtensorMap* km, const CUtensorMap* vm, const FastParams* fp,
                  cudaStream_t s, int* grid_out) {
  if (nt == 2) {
    if (d == 64) return launch_fast<T, TO, 64, 2>(km, vm, fp, s, grid_out);
    return launch_fast<T, TO, 128, 2>(km, vm, fp, s, grid_out);
  }
  if (nt == 1) {
    if (d == 64) return launch_fast<T, TO, 64, 1>(km, vm, fp, s, grid_out);
    if (d == 128) return launch_fast<T, TO, 128, 1>(km, vm, fp, s, grid_out);
    return launch_fast<T, TO, 256, 1>(km, vm, fp, s, grid_out);
  }
  if (d == 64) return launch_fast<T, TO, 64, 0>(km, vm, fp, s, grid_out);
  if (d == 128) return launch_fast<T, TO, 128, 0>(km, vm, fp, s, grid_out);
  return launch_fast<T, TO, 256, 0>(km, vm, fp, s, grid_out);
}

int dispatch_fast_any(int q_dtype, int out_dtype, int d, int nt, const CUtensorMap* km, const CUtensorMap* vm,
                      const FastParams* fp, cudaStream_t s, int* grid_out) {
  if (q_dtype == PA_BF16)
    return out_dtype == PA_F32 ? dispatch_fast<__nv_bfloat16, float>(d, nt, km, vm, fp, s, grid_out)
                               : dispatch_fast<__nv_bfloat16, __nv_bfloat16>(d, nt, km, vm, fp, s, grid_out);
  return out_dtype == PA_F32 ? dispatch_fast<__half, float>(d, nt, km, vm, fp, s, grid_out)
                             : dispatch_fast<__half, __half>(d, nt, km, vm, fp, s, grid_out);
}

template <typename T, typename TO>
void launch_generic(const GenericParams& gp, int max_parts, int batch, cudaStream_t s) {
  dim3 grid(max_parts, gp.hq, batch);
  decode_generic_kernel<T, TO><<<grid, kGenericWarps * 32, 0, s>>>(gp);
  pa::count_launches(1);
}

// The merge is a programmatic dependent of the attention kernel before it on
// the stream: its CTAs launch as that kernel's CTAs retire and wait
// (griddepcontrol.wait) until all of its results are visible.
template <typename TO>
int launch_merge(const MergeParams& mp, int batch, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mp.hq, batch);
  cfg.blockDim = dim3(kMergeWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<TO>, mp);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("decode merge launch: ") + cudaGetErrorString(e));
  pa::count_launches(1);
  return PA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// ever completes, gives up after `polls` polls and records the timeout bit.
__global__ void bounded_wait_selftest_kernel(uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  pa::mbar_init(&bar, 1);
  pa::fence_mbar_init();
  bool done = false;
  for (uint32_t i = 0; i < polls && !done; ++i) done = pa::mbar_try_wait(&bar, 0);
  if (!done) decode_flag(PA_DEVERR_WAIT_TIMEOUT);
}

}  // namespace

int pa_internal_take_errors_decode(unsigned int* bits) { return decode_take_errors(bits); }

extern "C" int pa_selftest_bounded_wait(uint32_t polls, pa_stream stream) {
  pa::clear_error();
  if (polls == 0 || polls > pa::kWaitPolls) return pa::fail(PA_ERR_ARG, "polls must be in [1, 2^22]");
  bounded_wait_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(polls);
  pa::count_launches(1);
  return cuda_status("bounded wait self-test launch");
}

extern "C" size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                           int32_t max_context, int32_t partition_tokens) {
  if (batch < 0 || num_q_heads < 1 || head_dim < 1 || max_context < 1 || partition_tokens < 1) return 0;
  const int64_t max_parts = (int64_t(max_context) + partition_tokens - 1) / partition_tokens;
  return ws_layout(batch, num_q_heads, head_dim, max_parts).total;
}

extern "C" int pa_profile_enable(int32_t on) {
  pa::clear_error();
  Profiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = on != 0;
  return PA_OK;
}

extern "C" int pa_profile_take(float* total_ms_out, int32_t* count_out) {
  pa::clear_error();
  if (!total_ms_out || !count_out) return pa::fail(PA_ERR_ARG, "NULL output");
  Profiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  float total = 0.f;
  int rc = PA_OK;
  for (auto& ab : p.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(ab.second) != cudaSuccess || cudaEventElapsedTime(&ms, ab.first, ab.second) != cudaSuccess)
      rc = pa::fail(PA_ERR_CUDA, "reading profile events failed");
    total += ms;
    p.spare.push_back(ab.first);
    p.spare.push_back(ab.second);
  }
  *count_out = int32_t(p.pending.size());
  *total_ms_out = total;
  p.pending.clear();
  return rc;
}

extern "C" int pa_set_option(int32_t key, int32_t value) {
  pa::clear_error();
  if (key == PA_OPT_DECODE_PATH) {
    if (value < 0 || value > 1) return pa::fail(PA_ERR_ARG, "PA_OPT_DECODE_PATH takes 0 or 1");
    g_decode_path = value;
    return PA_OK;
  }
  if (key == PA_OPT_PREFILL_PATH) return pa_internal_set_prefill_path(value);
  if (key == PA_OPT_CHECKED) return pa_internal_set_checked(value);
  return pa::fail(PA_ERR_ARG, "unknown option");
}

extern "C" int pa_get_option(int32_t key, int32_t* value_out) {
  pa::clear_error();
  if (!value_out) return pa::fail(PA_ERR_ARG, "NULL output");
  if (key == PA_OPT_DECODE_PATH) {
    *value_out = g_decode_path;
    return PA_OK;
  }
  if (key == PA_OPT_PREFILL_PATH) {
    *value_out = pa_internal_get_prefill_path();
    return PA_OK;
  }
  if (key == PA_OPT_CHECKED) {
    *value_out = pa_internal_get_checked();
    return PA_OK;
  }
  return pa::fail(PA_ERR_ARG, "unknown option");
}

// pa_decode, and pa_decode_append when k_new / v_new are given.
static int decode_impl(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                       const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                       int32_t max_context, int32_t partition_tokens, const pa_tensor* workspace,
                       const pa_tensor* out, pa_stream stream, const pa_tensor* k_new,
                       const pa_tensor* v_new) {
  pa::clear_error();
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace || !out)
    return pa::fail(PA_ERR_ARG, "NULL tensor");
  if (q->ndim != 3) return pa::fail(PA_ERR_ARG, "q must be [batch, Hq, head_dim]");
  if (k_cache->ndim != 4 || v_cache->ndim != 4)
    return pa::fail(PA_ERR_ARG, "caches must be [num_blocks, Hkv, B, head_dim]");
  if (block_tables->ndim != 2 || block_tables->dtype != PA_I32)
    return pa::fail(PA_ERR_ARG, "block_tables must be int32 [batch, max_blocks]");
  if (context_lens->ndim != 1 || context_lens->dtype != PA_I32)
    return pa::fail(PA_ERR_ARG, "context_lens must be int32 [batch]");
  if (out->ndim != 3) return pa::fail(PA_ERR_ARG, "out must be [batch, Hq, head_dim]");
  if (workspace->ndim != 1 || workspace->dtype != PA_U8)
    return pa::fail(PA_ERR_ARG, "workspace must be a 1-D uint8 buffer");
  if (!pa::is_float(q->dtype) || k_cache->dtype != q->dtype || v_cache->dtype != q->dtype)
    return pa::fail(PA_ERR_DTYPE, "q and both caches must share one float dtype");
  if (out->dtype != PA_F32 && out->dtype != q->dtype)
    return pa::fail(PA_ERR_DTYPE, "out must be fp32 or the dtype of q");
  for (int i = 0; i < 4; ++i)
    if (k_cache->shape[i] != v_cache->shape[i]) return pa::fail(PA_ERR_ARG, "k_cache and v_cache shapes differ");
  if (!pa::is_contiguous(*k_cache) || !pa::is_contiguous(*v_cache))
    return pa::fail(PA_ERR_ARG, "caches must be contiguous");
  const int64_t batch = q->shape[0], hq = q->shape[1], d = q->shape[2];
  const int64_t nb = k_cache->shape[0], hkv = k_cache->shape[1], bs = k_cache->shape[2];
  if (k_cache->shape[3] != d) return pa::fail(PA_ERR_ARG, "cache head_dim differs from q");
  if (hkv < 1 || hq % hkv != 0) return pa::fail(PA_ERR_ARG, "Hq must be a positive multiple of Hkv");
  if (bs < 1) return pa::fail(PA_ERR_ARG, "block size must be positive");
  if (block_tables->shape[0] != batch || context_lens->shape[0] != batch)
    return pa::fail(PA_ERR_ARG, "block_tables / context_lens batch differs from q");
  for (int i = 0; i < 3; ++i)
    if (out->shape[i] != q->shape[i]) return pa::fail(PA_ERR_ARG, "out shape differs from q");
  if ((q->stride[2] != 1 || out->stride[2] != 1) && d > 1)
    return pa::fail(PA_ERR_ARG, "q and out need a contiguous last dimension");
  if (partition_tokens < 1 || partition_tokens % bs != 0)
    return pa::fail(PA_ERR_ARG, "partition_tokens must be a positive multiple of the block size");
  if (max_context < 1) return pa::fail(PA_ERR_ARG, "max_context must be >= 1");
  if (d > kGenericMaxD) return pa::fail(PA_ERR_ARG, "head_dim above 512 is not supported");
  if (nb * hkv * bs > INT32_MAX) return pa::fail(PA_ERR_ARG, "cache has more than 2^31 rows");
  if (batch > 65535 || hq > 65535) return pa::fail(PA_ERR_ARG, "batch and Hq must be <= 65535");
  const bool append = k_new != nullptr;
  if (append) {
    for (const pa_tensor* t : {k_new, v_new}) {
      if (t->ndim != 3 || t->shape[0] != batch || t->shape[1] != hkv || t->shape[2] != d)
        return pa::fail(PA_ERR_ARG, "k_new and v_new must be [batch, Hkv, head_dim]");
      if (t->dtype != k_cache->dtype) return pa::fail(PA_ERR_DTYPE, "k_new and v_new must have the cache dtype");
      if (t->stride[2] != 1 && d > 1) return pa::fail(PA_ERR_ARG, "k_new and v_new need a contiguous last dimension");
      if (batch > 0 && !t->data) return pa::fail(PA_ERR_ARG, "NULL data pointer");
    }
  }
  if (batch == 0) return PA_OK;
  const int64_t max_parts = (int64_t(max_context) + partition_tokens - 1) / partition_tokens;
  const WsLayout wl = ws_layout(batch, hq, d, max_parts);
  if (size_t(workspace->shape[0]) < wl.total)
    return pa::fail(PA_ERR_ARG, "workspace smaller than pa_decode_workspace_size()");
  if ((reinterpret_cast<uintptr_t>(workspace->data) & 255u) != 0)
    return pa::fail(PA_ERR_ARG, "workspace must be 256-byte aligned");
  if (!q->data || !k_cache->data || !v_cache->data || !block_tables->data || !context_lens->data ||
      !out->data || !workspace->data)
    return pa::fail(PA_ERR_ARG, "NULL data pointer");
  const int64_t max_tokens = std::min<int64_t>(block_tables->shape[1] * bs, max_context);
  char* ws = static_cast<char*>(workspace->data);
  int* n_pairs = reinterpret_cast<int*>(ws);
  int4* pairs = reinterpret_cast<int4*>(ws + wl.pairs_off);
  int* counters = reinterpret_cast<int*>(ws + wl.cnt_off);
  float2* ml = reinterpret_cast<float2*>(ws + wl.ml_off);
  float* accw = reinterpret_cast<float*>(ws + wl.acc_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int group = int(hq / hkv);
  const float scale_log2 = scale * pa::kLog2e;
  const int elt = int(pa::dtype_size(q->dtype));
  const int oelt = int(pa::dtype_size(out->dtype));

  const bool fast = g_decode_path == 0 && q->dtype != PA_F32 && bs == kBlock &&
                    (d == 64 || d == 128 || d == 256) && (group <= 8 || (group == 16 && d <= 128)) &&
                    partition_tokens / kBlock <= 32 && aligned16(q->data) &&
                    aligned16(out->data) && (q->stride[0] * elt) % 16 == 0 && (q->stride[1] * elt) % 16 == 0 &&
                    (out->stride[0] * oelt) % 16 == 0 && (out->stride[1] * oelt) % 16 == 0 &&
                    aligned16(k_cache->data) && aligned16(v_cache->data);
  // the attention kernel stores the new rows itself when they are 16-byte aligned
  const bool append_in_kernel =
      append && fast && aligned16(k_new->data) && aligned16(v_new->data) && (k_new->stride[0] * elt) % 16 == 0 &&
      (k_new->stride[1] * elt) % 16 == 0 && (v_new->stride[0] * elt) % 16 == 0 && (v_new->stride[1] * elt) % 16 == 0;
  int rc = PA_OK;
  if (append && pa::checked_mode()) {
    rc = pa::check_append(static_cast<const int32_t*>(block_tables->data), block_tables->stride[0],
                          block_tables->stride[1], static_cast<const int32_t*>(context_lens->data),
                          context_lens->stride[0], int(batch), int(bs), int(block_tables->shape[1]),
                          int(max_tokens), stream);
    if (rc != PA_OK) return rc;
  }
  if (append && !append_in_kernel) {
    AppendParams ap;
    ap.k_new = k_new->data;
    ap.v_new = v_new->data;
    ap.kn_s = k_new->stride[0];
    ap.kn_h = k_new->stride[1];
    ap.vn_s = v_new->stride[0];
    ap.vn_h = v_new->stride[1];
    ap.k_cache = k_cache->data;
    ap.v_cache = v_cache->data;
    ap.tables = static_cast<const int32_t*>(block_tables->data);
    ap.tab_s = block_tables->stride[0];
    ap.tab_b = block_tables->stride[1];
    ap.lens = static_cast<const int32_t*>(context_lens->data);
    ap.len_s = context_lens->stride[0];
    ap.hkv = int(hkv);
    ap.d = int(d);
    ap.block_size = int(bs);
    ap.num_blocks = int(nb);
    ap.max_tokens = int(max_tokens);
    const unsigned grid = unsigned(batch * hkv);
    if (elt == 4) append_rows_kernel<uint32_t><<<grid, 128, 0, s>>>(ap);
    else append_rows_kernel<uint16_t><<<grid, 128, 0, s>>>(ap);
    pa::count_launches(1);
    rc = cuda_status("append rows kernel launch");
    if (rc != PA_OK) return rc;
  }
  if (fast) {
    const int nt = group == 1 ? 0 : (group <= 8 ? 1 : 2);
    int grid = 0;
    rc = dispatch_fast_any(q->dtype, out->dtype, int(d), nt, nullptr, nullptr, nullptr, s, &grid);
    if (rc != PA_OK) return rc;
    PlanParams pp;
    pp.lens = static_cast<const int32_t*>(context_lens->data);
    pp.len_stride = context_lens->stride[0];
    pp.batch = int(batch);
    pp.max_tokens = int(max_tokens);
    pp.block_size = int(bs);
    pp.part_blocks = partition_tokens / kBlock;
    pp.pairs = pairs;
    pp.n_pairs = n_pairs;
    pp.counters = counters;
    pp.n_counters = int(batch * hkv);
    pp.work = n_pairs + 1;
    pp.n_workers = grid * kWarps;
    {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1);
      cfg.blockDim = dim3(kPlanThreads);
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cudaError_t e = cudaLaunchKernelEx(&cfg, decode_plan_kernel, pp);
      if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("decode plan launch: ") + cudaGetErrorString(e));
    }
    pa::count_launches(1);
    rc = cuda_status("decode plan kernel launch");
    if (rc != PA_OK) return rc;
    CUtensorMap km, vm;
    rc = pa::encode_page_map(&km, *k_cache);
    if (rc == PA_OK) rc = pa::encode_page_map(&vm, *v_cache);
    if (rc != PA_OK) return rc;
    FastParams fp;
    fp.q = q->data;
    fp.q_s = q->stride[0];
    fp.q_h = q->stride[1];
    fp.tables = static_cast<const int32_t*>(block_tables->data);
    fp.tab_s = block_tables->stride[0];
    fp.tab_b = block_tables->stride[1];
    fp.lens = pp.lens;
    fp.len_s = pp.len_stride;
    fp.out = out->data;
    fp.out_s = out->stride[0];
    fp.out_h = out->stride[1];
    fp.ml = ml;
    fp.acc = accw;
    fp.pairs = pairs;
    fp.n_pairs = n_pairs;
    fp.counters = counters;
    fp.work = n_pairs + 1;
    fp.hq = int(hq);
    fp.hkv = int(hkv);
    fp.group = group;
    fp.num_blocks = int(nb);
    fp.max_tokens = int(max_tokens);
    fp.part_tokens = partition_tokens;
    fp.part_blocks = partition_tokens / kBlock;
    fp.max_parts = int(max_parts);
    fp.scale_log2 = scale_log2;
    fp.k_new = append_in_kernel ? k_new->data : nullptr;
    fp.v_new = append_in_kernel ? v_new->data : nullptr;
    fp.kn_s = append ? k_new->stride[0] : 0;
    fp.kn_h = append ? k_new->stride[1] : 0;
    fp.vn_s = append ? v_new->stride[0] : 0;
    fp.vn_h = append ? v_new->stride[1] : 0;
    fp.k_cache = k_cache->data;
    fp.v_cache = v_cache->data;
    ProfileScope prof(s);
    rc = dispatch_fast_any(q->dtype, out->dtype, int(d), nt, &km, &vm, &fp, s, nullptr);
    if (rc != PA_OK) return rc;
  } else {
    if (max_parts > 65535) return pa::fail(PA_ERR_ARG, "too many partitions for the generic kernel");
    GenericParams gp;
    gp.q = q->data;
    gp.q_s = q->stride[0];
    gp.q_h = q->stride[1];
    gp.k_cache = k_cache->data;
    gp.v_cache = v_cache->data;
    gp.tables = static_cast<const int32_t*>(block_tables->data);
    gp.tab_s = block_tables->stride[0];
    gp.tab_b = block_tables->stride[1];
    gp.lens = static_cast<const int32_t*>(context_lens->data);
    gp.len_s = context_lens->stride[0];
    gp.out = out->data;
    gp.out_s = out->stride[0];
    gp.out_h = out->stride[1];
    gp.ml = ml;
    gp.acc = accw;
    gp.hq = int(hq);
    gp.hkv = int(hkv);
    gp.group = group;
    gp.d = int(d);
    gp.block_size = int(bs);
    gp.num_blocks = int(nb);
    gp.max_tokens = int(max_tokens);
    gp.part_tokens = partition_tokens;
    gp.max_parts = int(max_parts);
    gp.scale_log2 = scale_log2;
    const int mp = int(max_parts);
    ProfileScope prof(s);
    switch (q->dtype) {
      case PA_F32: launch_generic<float, float>(gp, mp, int(batch), s); break;
      case PA_F16:
        if (out->dtype == PA_F32) launch_generic<__half, float>(gp, mp, int(batch), s);
        else launch_generic<__half, __half>(gp, mp, int(batch), s);
        break;
      default:
        if (out->dtype == PA_F32) launch_generic<__nv_bfloat16, float>(gp, mp, int(batch), s);
        else launch_generic<__nv_bfloat16, __nv_bfloat16>(gp, mp, int(batch), s);
        break;
    }
    rc = cuda_status("decode generic kernel launch");
    if (rc != PA_OK) return rc;
  }
  const bool fused_all = fast && PA_FUSED_MERGE && max_parts <= kFusedMergeMaxParts;
  if (max_parts > 1 && !fused_all) {
    MergeParams mp;
    mp.lens = static_cast<const int32_t*>(context_lens->data);
    mp.len_s = context_lens->stride[0];
    mp.ml = ml;
    mp.acc = accw;
    mp.out = out->data;
    mp.out_s = out->stride[0];
    mp.out_h = out->stride[1];
    mp.hq = int(hq);
    mp.d = int(d);
    mp.max_tokens = int(max_tokens);
    mp.part_tokens = partition_tokens;
    mp.max_parts = int(max_parts);
    mp.min_parts = (fast && PA_FUSED_MERGE) ? kFusedMergeMaxParts + 1 : 2;
    switch (out->dtype) {
      case PA_F32: rc = launch_merge<float>(mp, int(batch), s); break;
      case PA_F16: rc = launch_merge<__half>(mp, int(batch), s); break;
      default: rc = launch_merge<__nv_bfloat16>(mp, int(batch), s); break;
    }
    if (rc != PA_OK) return rc;
    rc = cuda_status("decode merge kernel launch");
  }
  return rc;
}

extern "C" int pa_decode(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                         const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                         int32_t max_context, int32_t partition_tokens, const pa_tensor* workspace,
                         const pa_tensor* out, pa_stream stream) {
  return decode_impl(q, k_cache, v_cache, block_tables, context_lens, scale, max_context, partition_tokens,
                     workspace, out, stream, nullptr, nullptr);
}

extern "C" int pa_decode_append(const pa_tensor* q, const pa_tensor* k_new, const pa_tensor* v_new,
                                const pa_tensor* k_cache, const pa_tensor* v_cache,
                                const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                                int32_t max_context, int32_t partition_tokens, const pa_tensor* workspace,
                                const pa_tensor* out, pa_stream stream) {
  if (!k_new || !v_new) {
    pa::clear_error();
    return pa::fail(PA_ERR_ARG, "NULL tensor");
  }
  return decode_impl(q, k_cache, v_cache, block_tables, context_lens, scale, max_context, partition_tokens,
                     workspace, out, stream, k_new, v_new);
}
