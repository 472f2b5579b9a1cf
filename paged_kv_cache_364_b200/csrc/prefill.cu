// Paged prefill attention (pa_prefill) for sm_100a.
//
// What is computed: each sequence s brings q_len_s new tokens, the last q_len_s
// of its n_s = context_lens[s] positions, whose K/V are already in the cache.
// The new token at position p attends keys 0..p of its sequence:
//     out[row, h] = softmax(scale * K_s[0..p] q[row, h]) V_s[0..p],
// K_s / V_s reached through the block table.  Prompt tokens live in logical
// blocks mapped to arbitrary physical blocks ("Stop Wasting GPU Memory: A Deep
// Dive Into vLLM's PagedAttention", Technical Details, "Single Sequence
// Generation"); a cached prefix -- for instance a system prompt whose blocks
// many requests share -- is attended, not recomputed ("49 vLLM /
// PagedAttention", "Questions worth asking").  Query rows of all sequences
// are packed: sequence s owns rows query_start[s] .. query_start[s+1]-1.
//
// Kernels in this file
//   prefill_tc_kernel       one CTA per (128-row query tile, KV head,
//                           sequence).  A query tile is floor(128/G) consecutive
//                           new tokens x the G query heads of one KV head
//                           (G = 1..8 or 16; leftover rows stay empty).
//                           Warps 4 and 6 stream K and V pages (tensor copies,
//                           64 keys per slot, one ring each).  Warp 5 owns the
//                           tensor memory and issues S = Q K^T into one of two
//                           S buffers; warp 7 issues O += P V with P read from
//                           tensor memory.  Each issuing warp has its own
//                           tcgen05.mma issue rate, so two issuers per CTA keep
//                           the tensor core fed where one could not, and S of
//                           the next key tile is computed while the softmax
//                           works on this one.  Each thread of warps 0-3 owns one query
//                           row: it reads S from tensor memory, applies the
//                           causal mask (diagonal tiles only), keeps the
//                           running max / sum, rescales O in tensor memory when
//                           the max grows by more than 2^8, and writes P back
//                           over S as two 16-bit terms (P = hi + lo) so the
//                           product keeps ~16 bits of each weight.  Two CTAs
//                           share an SM (one for head_dim 256), so one CTA's
//                           softmax overlaps the other's MMAs.
//   prefill_generic_kernel  CUDA-core fallback for every other dtype and shape
//                           (one warp per (row, head), online softmax).
#include <cudaTypedefs.h>

#include <algorithm>
#include <string>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tc.cuh"
#include "pa_tmap.h"

PA_DEFINE_ERROR_WORD(prefill)

namespace {

constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBlock = 16;          // tokens per cache block on the tensor-core path
constexpr int kBM = 128;            // query rows per tile = tensor-memory lanes
constexpr int kBN = 64;             // keys per K/V stage
constexpr int kStagePages = kBN / kBlock;
constexpr int kSoftWarps = 4;
constexpr int kProducerWarp = 4;    // K pages
constexpr int kMmaWarp = 5;
constexpr int kVProducerWarp = 6;   // V pages
constexpr int kPvWarp = 7;          // issues O += P V
constexpr int kThreads = 256;
// The running max used for the exponentials lags the true max by at most
// this much (base 2), so weights stay <= 2^8 and O is rescaled only when the
// max grows past it.  The final division uses the same max: no change in value.
constexpr float kRescaleLog2 = 8.f;

template <int D> struct TcCfg {
  static constexpr int kChunks = D / 64;              // 128-byte swizzle columns of a row
  static constexpr int kQChunk = kBM * 128;
  static constexpr int kQBytes = kChunks * kQChunk;
  static constexpr int kKvChunk = kBN * 128;
  static constexpr int kKBytes = kChunks * kKvChunk;
  // separate K and V rings: a K slot is free once its S = Q K^T is done, a V
  // slot once its O += P V is done
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kKOff = kQBytes;
  static constexpr int kVOff = kKOff + kStages * kKBytes;
  static constexpr int kBarOff = kVOff + kStages * kKBytes;
  // k_full[], k_empty[], v_full[], v_empty[], s_full[2], p_full[2], pv_done, pv_buf[2], o_done
  static constexpr int kNumBars = 4 * kStages + 8;
  static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;   // + tensor-memory slot + alignment
  // tensor-memory columns: two S buffers [0, 64) and [64, 128) -- tile j uses
  // buffer j % 2, and its P (hi in the first 32 columns, lo in the next 32)
  // overwrites its S once read -- and O [128, 128 + D)
  static constexpr uint32_t kOCol = 128;
  // head_dim 64 / 128: two CTAs per SM share the 512 columns; head_dim 256
  // (O takes 256 columns): one CTA per SM with all of them
  static constexpr uint32_t kTmemCols = D == 256 ? 512 : 256;
  static constexpr int kMinCtas = D == 256 ? 1 : 2;
  // shared memory keeps more CTAs than that off an SM, so tensor memory is
  // never requested beyond its 512 columns
  static_assert((512 / kTmemCols + 1) * (kSmem + 1024) > 228 * 1024, "tensor memory oversubscribed");
};

struct PrefillParams {
  const void* q;
  int64_t q_t, q_h;                 // element strides (row, head)
  const int32_t* tables;
  int64_t tab_s, tab_b;
  const int32_t* lens;
  int64_t len_s;
  const int32_t* qstart;
  int64_t qs_s;
  void* out;
  int64_t out_t, out_h;
  const void* k_cache;              // generic path only (the tensor-core path reads through tensor maps)
  const void* v_cache;
  int batch, hq, hkv, group, d, block_size, num_blocks, max_tokens, total_rows, tiles_per_seq;
  float scale_log2;
  // split over the keys (n_splits > 1): CTA split covers keys
  // [split * split_keys, (split + 1) * split_keys) and leaves its unnormalised
  // state in the workspace for prefill_merge_kernel
  int n_splits, split_keys;
  float* ws_acc;                    // [n_splits][rows][Hq][d]
  float2* ws_ml;                    // [n_splits][rows][Hq]: (running max, base 2; sum)
};

struct SeqGeom {
  int r0, qlen, n;
  bool ok;
};

// Sequence s: first query row, new tokens, context length, and whether they
// are consistent (0 <= q_len <= n <= max_tokens, rows inside q).
__device__ __forceinline__ SeqGeom seq_geom(const PrefillParams& p, int s) {
  SeqGeom g;
  g.r0 = p.qstart[int64_t(s) * p.qs_s];
  const int r1 = p.qstart[int64_t(s + 1) * p.qs_s];
  g.n = p.lens[int64_t(s) * p.len_s];
  g.qlen = r1 - g.r0;
  g.ok = g.r0 >= 0 && r1 >= g.r0 && r1 <= p.total_rows &&
         (g.qlen == 0 || (g.n >= 1 && g.n <= p.max_tokens && g.qlen <= g.n));
  return g;
}


// two-lane fp32 arithmetic (one instruction for a pair of floats)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <typename T> constexpr bool is_bf16() { return std::is_same<T, __nv_bfloat16>::value; }

// ------------------------------------------------------ tensor-core path ---
template <typename T, typename TO, int D, int G>
__global__ void __launch_bounds__(kThreads, TcCfg<D>::kMinCtas)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const PrefillParams p) {
  using C = TcCfg<D>;
  constexpr int TT = kBM / G;                       // new tokens per query tile
  // the tiles of one (sequence, KV head) are adjacent in launch order, so the
  // K/V they all stream stays in L2; within it the last tiles (the most keys
  // under the causal mask) come first
  const int split = int(blockIdx.x % p.n_splits);
  const int rest = int(blockIdx.x / p.n_splits);
  const int pair = rest / p.tiles_per_seq;
  const int tile = p.tiles_per_seq - 1 - rest % p.tiles_per_seq;
  const int s = pair / p.hkv;
  const int hk = pair % p.hkv;
  const SeqGeom g = seq_geom(p, s);
  if (!g.ok) {
    if (tile == 0 && hk == 0 && split == 0 && threadIdx.x == 0) prefill_flag(PA_DEVERR_CONTEXT_LEN);
    return;
  }
  if (tile == p.tiles_per_seq - 1 && hk == 0 && split == 0 && threadIdx.x == 0 && g.qlen > p.tiles_per_seq * TT)
    prefill_flag(PA_DEVERR_CONTEXT_LEN);            // q_len above max_query_len: rows past it are skipped
  const int t0 = tile * TT;
  if (t0 >= g.qlen) return;
  const int tcount = min(TT, g.qlen - t0);           // new tokens in this tile
  const int pos0 = g.n - g.qlen + t0;                // position of the tile's first token
  const int n_kv = pos0 + tcount;                    // keys 0 .. n_kv-1 are seen by some row
  const int kbase = split * p.split_keys;            // this CTA's keys: [kbase, kend), kbase % kBN == 0
  if (kbase >= n_kv) return;
  const int kend = min(n_kv, kbase + p.split_keys);
  const int ntiles = (kend - kbase + kBN - 1) / kBN;
  const int npages = (kend + kBlock - 1) / kBlock;  // pages 0 .. npages-1 hold keys below kend

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = pa::smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + C::kStages;
  uint64_t* v_full = bars + 2 * C::kStages;
  uint64_t* v_empty = bars + 3 * C::kStages;
  uint64_t* s_full = bars + 4 * C::kStages;           // [2]
  uint64_t* p_full = s_full + 2;                      // [2]: P_j written, by tile parity
  uint64_t* pv_done = s_full + 4;                     // each PV_j done (waited only before a rescale of O)
  uint64_t* pv_buf = s_full + 5;                      // [2]: PV_j done with S buffer j % 2
  uint64_t* o_done = s_full + 7;                      // the last PV done: O is final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == kMmaWarp) {
    pa::tc::tmem_alloc(pa::smem_addr(tmem_slot), C::kTmemCols);
    pa::tc::tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    for (int i = 0; i < 4 * C::kStages + 2; ++i) pa::mbar_init(&bars[i], 1);   // rings, s_full[2]
    pa::mbar_init(&p_full[0], kSoftWarps);
    pa::mbar_init(&p_full[1], kSoftWarps);
    pa::mbar_init(pv_done, 1);
    pa::mbar_init(&pv_buf[0], 1);
    pa::mbar_init(&pv_buf[1], 1);
    pa::mbar_init(o_done, 1);
    pa::fence_mbar_init();
    pa::prefetch_tensormap(&kmap);
    pa::prefetch_tensormap(&vmap);
  }
  // query tile -> shared memory as [D/64][128 rows][128 B], 128-byte swizzle;
  // row r = (token r / G, query head hk*G + r % G); rows past the tile are zero
  const int r = threadIdx.x;
  const int tok = r / G;
  const bool row_valid = warp < kSoftWarps && tok < tcount;
  if (warp < kSoftWarps) {
    const T* src = static_cast<const T*>(p.q) + int64_t(g.r0 + t0 + (row_valid ? tok : 0)) * p.q_t +
                   int64_t(hk * G + r % G) * p.q_h;
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
      const uint4 x = row_valid ? __ldg(reinterpret_cast<const uint4*>(src) + u) : make_uint4(0, 0, 0, 0);
      pa::sts128(sb + (u >> 3) * C::kQChunk + r * 128 + (((u & 7) ^ (r & 7)) << 4), x);
    }
    pa::fence_proxy_async_smem();
  }
  pa::tc::fence_before_sync();
  __syncthreads();
  pa::tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp || warp == kVProducerWarp) {
    // ---- K and V pages of the keys this tile needs, kBN keys per slot.
    // One warp streams K, another V, each at its own pace: a K slot frees
    // when its S = Q K^T is done, long before the V slot of the same tile,
    // so the next K copies start about a tile earlier than if one thread
    // issued K and V in turn.
    // The whole warp takes part: lane (page q, chunk ch) issues that copy, so
    // one warp instruction issues a tile's kStagePages x kChunks copies
    // instead of one thread issuing them one after another (about 125 cycles
    // each), and each lane reads its page's block id one tile ahead, while
    // the slot is still awaited.
    {
      const int which = warp == kVProducerWarp;      // 0 = K, 1 = V
      uint64_t policy;
      asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(policy));
      const CUtensorMap* map = which ? &vmap : &kmap;
      uint64_t* full_ring = which ? v_full : k_full;
      uint64_t* empty_ring = which ? v_empty : k_empty;
      const uint32_t ring = sb + (which ? C::kVOff : C::kKOff);
      const int my_q = lane / C::kChunks, my_ch = lane % C::kChunks;
      const bool copier = lane < kStagePages * C::kChunks;
      int issued = 0;                                // tiles whose copies were issued
      bool ok = true;
      int nxt = -1;                                  // this lane's block id of the next tile
      auto read_id = [&](int j) {
        const int pg = kbase / kBlock + j * kStagePages + my_q;
        nxt = copier && pg < npages ? p.tables[int64_t(s) * p.tab_s + int64_t(pg) * p.tab_b] : -1;
      };
      read_id(0);
      for (int j = 0; j < ntiles; ++j) {
        const int slot = j % C::kStages, use = j / C::kStages;
        const int blk = nxt;
        const bool in_tile = copier && kbase / kBlock + j * kStagePages + my_q < npages;
        if (j + 1 < ntiles) read_id(j + 1);
        if (use > 0 && !__all_sync(0xffffffffu, pa::mbar_wait_bounded(&empty_ring[slot], (use - 1) & 1))) {
          ok = false;
          break;
        }
        const bool valid = in_tile && blk >= 0 && blk < p.num_blocks;
        if (in_tile && !valid && which == 0 && my_ch == 0) prefill_flag(PA_DEVERR_BLOCK_ID);
        const uint32_t pages = __popc(__ballot_sync(0xffffffffu, valid && my_ch == 0));
        if (lane == 0) {
          if (pages) pa::mbar_arrive_expect_tx(&full_ring[slot], pages * uint32_t(kBlock) * D * 2u);
          else pa::mbar_arrive(&full_ring[slot]);
        }
        __syncwarp();
        if (valid) {
          const uint32_t dst = ring + slot * C::kKBytes + my_ch * C::kKvChunk + my_q * kBlock * 128;
          pa::tma_load_2d(dst, map, &full_ring[slot], 64 * my_ch, (blk * p.hkv + hk) * kBlock, policy);
        }
        issued = j + 1;
      }
      if (!ok && lane == 0) prefill_flag(PA_DEVERR_WAIT_TIMEOUT);
      // copies still in flight must land before the CTA's shared memory goes
      // away (only reachable after a lost wait): wait for each slot's last use
      if (lane == 0)
        for (int slot = 0; slot < C::kStages && slot < issued; ++slot) {
          const int last = slot + ((issued - 1 - slot) / C::kStages) * C::kStages;
          pa::mbar_wait_bounded(&full_ring[slot], (last / C::kStages) & 1);
        }
    }
  } else if (warp == kMmaWarp) {
    // ---- S = Q K^T into S buffer j % 2 (K-major A and B).  Buffer j % 2
    // is free again once PV_{j-2}, issued by the PV warp, has read P_{j-2}.
    constexpr uint32_t kIdS = pa::tc::idesc_f16(is_bf16<T>(), kBM, kBN, false);
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int slot = j % C::kStages;
      ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(&k_full[slot], (j / C::kStages) & 1));
      if (ok && j >= 2) ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(&pv_buf[j & 1], ((j - 2) >> 1) & 1));
      if (!ok) break;
      pa::tc::fence_after_sync();
      if (lane == 0) {
        const uint32_t kst = sb + C::kKOff + slot * C::kKBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          pa::tc::mma_ss(tmem + (j & 1) * 64,
                         pa::tc::smem_desc_sw128(sb + (kk >> 2) * C::kQChunk + (kk & 3) * 32, 16, 1024),
                         pa::tc::smem_desc_sw128(kst + (kk >> 2) * C::kKvChunk + (kk & 3) * 32, 16, 1024), kIdS,
                         kk > 0);
        pa::tc::commit(&k_empty[slot]);
        pa::tc::commit(&s_full[j & 1]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) prefill_flag(PA_DEVERR_WAIT_TIMEOUT);
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ---- O += P V with P read from S buffer j % 2 and V an MN-major B
    // operand (head_dim contiguous)
    constexpr uint32_t kIdPV = pa::tc::idesc_f16(is_bf16<T>(), kBM, D, true);
    const uint32_t tO = tmem + C::kOCol;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int slot = j % C::kStages;
      const uint32_t vst = sb + C::kVOff + slot * C::kKBytes;
      ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(&v_full[slot], (j / C::kStages) & 1));
      if (!ok) break;
      if (j == ntiles - 1 && kend < kbase + (j + 1) * kBN) {
        // V rows of keys at or past kend (unloaded pages, rows past the
        // context) may hold anything: zero them so their zero weights meet 0
        const int keep = kend - kbase - j * kBN;
        for (int e = lane; e < (kBN - keep) * (D / 8); e += 32) {
          const int row = keep + e / (D / 8), u = e % (D / 8);
          pa::sts128_zero(vst + (u >> 3) * C::kKvChunk + row * 128 + (((u & 7) ^ (row & 7)) << 4));
        }
        pa::fence_proxy_async_smem();
        __syncwarp();
      }
      ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(&p_full[j & 1], (j >> 1) & 1));
      if (!ok) break;
      pa::tc::fence_after_sync();
      if (lane == 0) {
        // a K-step of 16 keys is 8 tensor-memory columns of P
        const uint32_t pcol = tmem + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          pa::tc::mma_ts(tO, pcol + kk * 8, pa::tc::smem_desc_sw128(vst + kk * 16 * 128, C::kKvChunk, 1024), kIdPV,
                         j > 0 || kk > 0);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          pa::tc::mma_ts(tO, pcol + 32 + kk * 8, pa::tc::smem_desc_sw128(vst + kk * 16 * 128, C::kKvChunk, 1024),
                         kIdPV, 1);
        pa::tc::commit(&v_empty[slot]);
        pa::tc::commit(pv_done);
        pa::tc::commit(&pv_buf[j & 1]);
        if (j == ntiles - 1) pa::tc::commit(o_done);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      prefill_flag(PA_DEVERR_WAIT_TIMEOUT);
      pa::tc::commit(o_done);                        // lets the epilogue's wait end
    }
    __syncwarp();
  } else {
    // ---- softmax: thread r owns query row r (tensor-memory lane r)
    const int pos = pos0 + tok;                      // this row sees keys 0 .. pos
    const uint32_t trow = tmem + (uint32_t(warp * 32) << 16);
    float m_use = kNegInf, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(&s_full[j & 1], (j >> 1) & 1));
      if (!ok) break;
      pa::tc::fence_after_sync();
      const uint32_t sbuf = trow + (j & 1) * 64;
      float sv[kBN];
      {
        float a[32], b[32];
        pa::tc::ld_x32(sbuf, a);
        pa::tc::ld_x32(sbuf + 32, b);
        pa::tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sv[c] = a[c];
          sv[32 + c] = b[c];
        }
      }
      const int lim = row_valid ? pos - kbase - j * kBN : -1;   // keys c <= lim are visible
      // max of the raw visible scores; the (positive) scale enters in the
      // exponent.  Below the diagonal every key of the tile is visible to
      // every row and the mask is skipped.
      float mr = kNegInf;
      if (__all_sync(0xffffffffu, lim >= kBN - 1)) {
#pragma unroll
        for (int c = 0; c < kBN; c += 2) mr = max3(mr, sv[c], sv[c + 1]);
      } else {
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          sv[c] = c <= lim ? sv[c] : kNegInf;
          mr = fmaxf(mr, sv[c]);
        }
      }
      const float mt = mr * p.scale_log2;
      const bool grow = mt > m_use + kRescaleLog2;
      float alpha = 1.f;
      if (grow) {
        alpha = pa::fast_exp2(m_use - mt);           // 0 on the first visible tile
        m_use = mt;
        l *= alpha;
      }
      const float mu = m_use == kNegInf ? 0.f : m_use;
      // P row -> tensor memory over this tile's S: keys (2i, 2i+1) in column i,
      // hi in the first 32 columns, lo in the next 32
      uint32_t pk[kBN / 2];
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-mu, -mu);
      float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < kBN / 2; ++i) {
        const float2 e = fma2(make_float2(sv[2 * i], sv[2 * i + 1]), sc2, nm2);
        const float a = pa::fast_exp2(e.x), b = pa::fast_exp2(e.y);
        l2 = add2(l2, make_float2(a, b));
        sv[2 * i] = a;
        sv[2 * i + 1] = b;
        pk[i] = pa::pack2_rn<T>(a, b);
      }
      l += l2.x + l2.y;
      pa::tc::st_x32(sbuf, pk);
      const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
      for (int i = 0; i < kBN / 2; ++i) {
        const float2 r = fma2(pa::unpack2<T>(pk[i]), m1, make_float2(sv[2 * i], sv[2 * i + 1]));
        pk[i] = pa::pack2_rn<T>(r.x, r.y);
      }
      pa::tc::st_x32(sbuf + 32, pk);
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O is rescaled only after PV_{j-1} is done; PV_j waits for this
        // warp's arrival below.  Holding S_j means PV_{j-2} is done (S_j
        // reused its buffer) and PV_j cannot have started, so pv_done has
        // completed j-1 or j times and a parity wait for the (j-1)-th
        // completion is unambiguous.
        ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(pv_done, (j - 1) & 1));
        if (!ok) break;
        {
          pa::tc::fence_after_sync();
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            float o[32];
            pa::tc::ld_x32(trow + C::kOCol + cc * 32, o);
            pa::tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            pa::tc::st_x32(trow + C::kOCol + cc * 32, o);
          }
        }
      }
      pa::tc::wait_st();
      pa::tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) pa::mbar_arrive(&p_full[j & 1]);
    }
    if (!ok && lane == 0) prefill_flag(PA_DEVERR_WAIT_TIMEOUT);
    ok = __all_sync(0xffffffffu, pa::mbar_wait_bounded(o_done, 0));
    if (ok) {
      pa::tc::fence_after_sync();
      const bool partial = p.n_splits > 1;
      const float inv = partial ? 1.f : (l > 0.f ? 1.f / l : 0.f);
      const int64_t row = g.r0 + t0 + (row_valid ? tok : 0), head = hk * G + r % G;
      const int64_t wslot = (int64_t(split) * p.total_rows + row) * p.hq + head;
      TO* dst = static_cast<TO*>(p.out) + row * p.out_t + head * p.out_h;
      float* wdst = p.ws_acc + wslot * D;
      if (partial && row_valid) p.ws_ml[wslot] = make_float2(l > 0.f ? m_use : kNegInf, l);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        pa::tc::ld_x32(trow + C::kOCol + cc * 32, o);
        pa::tc::wait_ld();
        if (row_valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 v4 = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
            if (partial) *reinterpret_cast<float4*>(wdst + cc * 32 + i) = v4;
            else pa::store4<TO>(dst + cc * 32 + i, v4);
          }
        }
      }
    } else if (lane == 0) {
      prefill_flag(PA_DEVERR_WAIT_TIMEOUT);
    }
  }
  pa::tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    pa::tc::fence_after_sync();
    pa::tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------- generic path -----
constexpr int kGenericMaxD = 512;

// One warp per (query row, query head); each lane holds d/32 elements.
template <typename T, typename TO>
__global__ void __launch_bounds__(128) prefill_generic_kernel(const PrefillParams p) {
  constexpr int kRegs = kGenericMaxD / 32;
  const int lane = threadIdx.x & 31;
  const int64_t gw = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (gw >= int64_t(p.total_rows) * p.hq) return;
  const int row = int(gw / p.hq), h = int(gw % p.hq);
  // the sequence owning this row: last s with query_start[s] <= row
  int lo = 0, hi = p.batch;                          // invariant: qstart[lo] <= row < qstart[hi]
  if (!(p.qstart[0] <= row && row < p.qstart[int64_t(p.batch) * p.qs_s])) return;   // no sequence owns it
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.qstart[int64_t(mid) * p.qs_s] <= row) lo = mid;
    else hi = mid;
  }
  const int s = lo;
  const SeqGeom g = seq_geom(p, s);
  if (!g.ok) {
    if (lane == 0) prefill_flag(PA_DEVERR_CONTEXT_LEN);
    return;
  }
  const int pos = g.n - g.qlen + (row - g.r0);
  const int hk = h / p.group;
  float qv[kRegs], acc[kRegs];
  const T* qrow = static_cast<const T*>(p.q) + int64_t(row) * p.q_t + int64_t(h) * p.q_h;
#pragma unroll
  for (int i = 0; i < kRegs; ++i) {
    const int c = lane + 32 * i;
    qv[i] = c < p.d ? pa::to_f32(qrow[c]) : 0.f;
    acc[i] = 0.f;
  }
  float m = kNegInf, l = 0.f;
  for (int j = 0; j <= pos; ++j) {
    const int blk = p.tables[int64_t(s) * p.tab_s + int64_t(j / p.block_size) * p.tab_b];
    if (blk < 0 || blk >= p.num_blocks) {
      if (lane == 0) prefill_flag(PA_DEVERR_BLOCK_ID);
      continue;
    }
    const int64_t base = ((int64_t(blk) * p.hkv + hk) * p.block_size + j % p.block_size) * p.d;
    const T* krow = static_cast<const T*>(p.k_cache) + base;
    const T* vrow = static_cast<const T*>(p.v_cache) + base;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < kRegs; ++i) {
      const int c = lane + 32 * i;
      if (c < p.d) dot += qv[i] * pa::to_f32(krow[c]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float sc = dot * p.scale_log2;
    const float m_new = fmaxf(m, sc);
    const float corr = exp2f(m - m_new);            // 0 on the first key (m = -inf)
    const float w = exp2f(sc - m_new);
    l = l * corr + w;
#pragma unroll
    for (int i = 0; i < kRegs; ++i) {
      const int c = lane + 32 * i;
      acc[i] = acc[i] * corr + (c < p.d ? w * pa::to_f32(vrow[c]) : 0.f);
    }
    m = m_new;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  TO* orow = static_cast<TO*>(p.out) + int64_t(row) * p.out_t + int64_t(h) * p.out_h;
#pragma unroll
  for (int i = 0; i < kRegs; ++i) {
    const int c = lane + 32 * i;
    if (c < p.d) orow[c] = pa::from_f32<TO>(acc[i] * inv);
  }
}

// ------------------------------------------------------------ key splits ---
// Partitions of the keys when a launch would leave most SMs idle (few rows,
// long cached prefixes): each (query tile, KV head) is cut into partitions
// of split_keys keys, and this kernel merges a row's partition states:
// M = max m_p, L = sum l_p 2^(m_p - M), out = sum 2^(m_p - M) acc_p / L.
// One warp per (row, query head); partitions past the row's position hold
// no key it sees and are skipped.
template <typename TO>
__global__ void __launch_bounds__(128) prefill_merge_kernel(const PrefillParams p) {
  constexpr int kRegs = 256 / 32;
  const int lane = threadIdx.x & 31;
  const int64_t gw = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (gw >= int64_t(p.total_rows) * p.hq) return;
  const int row = int(gw / p.hq), h = int(gw % p.hq);
  if (!(p.qstart[0] <= row && row < p.qstart[int64_t(p.batch) * p.qs_s])) return;   // no sequence owns it
  int lo = 0, hi = p.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.qstart[int64_t(mid) * p.qs_s] <= row) lo = mid;
    else hi = mid;
  }
  const SeqGeom g = seq_geom(p, lo);
  const int tt = kBM / p.group;
  if (!g.ok || row - g.r0 >= p.tiles_per_seq * tt) return;   // rows the attention kernel skipped
  const int pos = g.n - g.qlen + (row - g.r0);
  const int nsp = min(p.n_splits, pos / p.split_keys + 1);
  float M = kNegInf;
  for (int q = 0; q < nsp; ++q)
    M = fmaxf(M, p.ws_ml[(int64_t(q) * p.total_rows + row) * p.hq + h].x);
  const float Mu = M == kNegInf ? 0.f : M;
  float L = 0.f, acc[kRegs];
#pragma unroll
  for (int i = 0; i < kRegs; ++i) acc[i] = 0.f;
  for (int q = 0; q < nsp; ++q) {
    const int64_t slot = (int64_t(q) * p.total_rows + row) * p.hq + h;
    const float2 ml = p.ws_ml[slot];
    const float w = exp2f(ml.x - Mu);              // 0 for a partition with no visible key
    L += ml.y * w;
    const float* a = p.ws_acc + slot * p.d;
#pragma unroll
    for (int i = 0; i < kRegs; ++i) {
      const int c = lane + 32 * i;
      if (c < p.d) acc[i] += a[c] * w;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  TO* orow = static_cast<TO*>(p.out) + int64_t(row) * p.out_t + int64_t(h) * p.out_h;
#pragma unroll
  for (int i = 0; i < kRegs; ++i) {
    const int c = lane + 32 * i;
    if (c < p.d) orow[c] = pa::from_f32<TO>(acc[i] * inv);
  }
}

// Key partitions for a tensor-core launch: split when the (query tile, KV
// head) grid is under four CTAs per SM (two waves at two CTAs per SM), into
// partitions of at least kSplitMinKeys keys (a multiple of kBN), at most
// kMaxSplits of them.  Such CTAs are long (thousands of keys each), so a
// grid of barely one wave would leave most SMs idle in its second.
constexpr int kSplitMinKeys = 1024;
constexpr int kMaxSplits = 64;

int prefill_splits(int64_t tiles_per_seq, int64_t batch, int64_t hkv, int64_t max_tokens, int sms,
                   int* split_keys) {
  const int64_t base = std::max<int64_t>(1, tiles_per_seq * batch * hkv);
  const int64_t target = 4 * int64_t(sms);
  int64_t n = base < target ? (target + base - 1) / base : 1;
  n = std::min<int64_t>(n, std::max<int64_t>(1, max_tokens / kSplitMinKeys));
  n = std::min<int64_t>(n, kMaxSplits);
  int64_t keys = (max_tokens + n - 1) / n;
  keys = (keys + kBN - 1) / kBN * kBN;
  n = (max_tokens + keys - 1) / keys;
  *split_keys = int(std::min<int64_t>(keys, INT32_MAX));
  return int(std::max<int64_t>(n, 1));
}

size_t split_workspace_bytes(int64_t n_splits, int64_t rows, int64_t hq, int64_t d) {
  if (n_splits <= 1) return 0;
  const size_t acc = size_t(n_splits) * rows * hq * d * sizeof(float);
  return ((acc + 255) & ~size_t(255)) + size_t(n_splits) * rows * hq * sizeof(float2);
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace


// ------------------------------------------------------------ host side ----
namespace {

int g_prefill_path = 0;   // 0 = tensor-core kernel where it applies, 1 = generic kernel only

int cuda_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return PA_OK;
}

template <typename T, typename TO, int D, int G>
int launch_tc(const CUtensorMap& km, const CUtensorMap& vm, const PrefillParams& p, unsigned grid, cudaStream_t s) {
  auto kern = prefill_tc_kernel<T, TO, D, G>;
  const int smem = TcCfg<D>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, std::string("prefill smem attribute: ") + cudaGetErrorString(e));
  kern<<<grid, kThreads, smem, s>>>(km, vm, p);
  pa::count_launches(1);
  return cuda_status("prefill tensor-core kernel launch");
}

template <typename T, typename TO, int D>
int launch_tc_group(int group, const CUtensorMap& km, const CUtensorMap& vm, const PrefillParams& p, unsigned grid,
                    cudaStream_t s) {
  switch (group) {
    case 1: return launch_tc<T, TO, D, 1>(km, vm, p, grid, s);
    case 2: return launch_tc<T, TO, D, 2>(km, vm, p, grid, s);
    case 3: return launch_tc<T, TO, D, 3>(km, vm, p, grid, s);
    case 4: return launch_tc<T, TO, D, 4>(km, vm, p, grid, s);
    case 5: return launch_tc<T, TO, D, 5>(km, vm, p, grid, s);
    case 6: return launch_tc<T, TO, D, 6>(km, vm, p, grid, s);
    case 7: return launch_tc<T, TO, D, 7>(km, vm, p, grid, s);
    case 8: return launch_tc<T, TO, D, 8>(km, vm, p, grid, s);
    default: return launch_tc<T, TO, D, 16>(km, vm, p, grid, s);
  }
}

template <typename T, typename TO>
int launch_tc_any(int d, int group, const CUtensorMap& km, const CUtensorMap& vm, const PrefillParams& p,
                  unsigned grid, cudaStream_t s) {
  if (d == 64) return launch_tc_group<T, TO, 64>(group, km, vm, p, grid, s);
  if (d == 128) return launch_tc_group<T, TO, 128>(group, km, vm, p, grid, s);
  return launch_tc_group<T, TO, 256>(group, km, vm, p, grid, s);
}

template <typename T, typename TO>
int launch_generic(const PrefillParams& p, cudaStream_t s) {
  const int64_t warps = int64_t(p.total_rows) * p.hq;
  const int64_t blocks = (warps + 3) / 4;
  if (blocks > INT32_MAX) return pa::fail(PA_ERR_ARG, "too many query rows x heads");
  prefill_generic_kernel<T, TO><<<unsigned(blocks), 128, 0, s>>>(p);
  pa::count_launches(1);
  return cuda_status("prefill generic kernel launch");
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

int pa_internal_take_errors_prefill(unsigned int* bits) { return prefill_take_errors(bits); }

int pa_internal_set_prefill_path(int32_t v) {
  if (v != 0 && v != 1) return pa::fail(PA_ERR_ARG, "prefill path must be 0 (auto) or 1 (generic)");
  g_prefill_path = v;
  return PA_OK;
}
int pa_internal_get_prefill_path() { return g_prefill_path; }

extern "C" size_t pa_prefill_workspace_size(int32_t rows, int32_t num_q_heads, int32_t num_kv_heads,
                                           int32_t head_dim, int32_t batch, int32_t max_query_len,
                                           int32_t max_tokens) {
  if (rows < 1 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads || head_dim < 1 ||
      batch < 1 || max_query_len < 1 || max_tokens < 1)
    return 0;
  const int group = num_q_heads / num_kv_heads;
  if (group > kBM) return 0;
  const int tt = kBM / group;
  int keys = 0;
  const int n = prefill_splits((max_query_len + tt - 1) / tt, batch, num_kv_heads, max_tokens, device_sms(), &keys);
  return split_workspace_bytes(n, rows, num_q_heads, head_dim);
}

extern "C" int pa_prefill(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                          const pa_tensor* block_tables, const pa_tensor* context_lens,
                          const pa_tensor* query_start, float scale, int32_t max_query_len,
                          const pa_tensor* workspace, const pa_tensor* out, pa_stream stream) {
  pa::clear_error();
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start || !out)
    return pa::fail(PA_ERR_ARG, "NULL tensor");
  if (q->ndim != 3) return pa::fail(PA_ERR_ARG, "q must be [rows, Hq, head_dim]");
  if (k_cache->ndim != 4 || v_cache->ndim != 4)
    return pa::fail(PA_ERR_ARG, "caches must be [num_blocks, Hkv, B, head_dim]");
  if (block_tables->ndim != 2 || block_tables->dtype != PA_I32)
    return pa::fail(PA_ERR_ARG, "block_tables must be int32 [batch, max_blocks]");
  if (context_lens->ndim != 1 || context_lens->dtype != PA_I32)
    return pa::fail(PA_ERR_ARG, "context_lens must be int32 [batch]");
  if (query_start->ndim != 1 || query_start->dtype != PA_I32)
    return pa::fail(PA_ERR_ARG, "query_start must be int32 [batch + 1]");
  if (out->ndim != 3) return pa::fail(PA_ERR_ARG, "out must be [rows, Hq, head_dim]");
  if (workspace && (workspace->ndim != 1 || workspace->dtype != PA_U8))
    return pa::fail(PA_ERR_ARG, "workspace must be a 1-D uint8 buffer");
  if (workspace && workspace->shape[0] > 0 && (reinterpret_cast<uintptr_t>(workspace->data) & 255u) != 0)
    return pa::fail(PA_ERR_ARG, "workspace must be 256-byte aligned");
  if (!pa::is_float(q->dtype) || k_cache->dtype != q->dtype || v_cache->dtype != q->dtype)
    return pa::fail(PA_ERR_DTYPE, "q and both caches must share one float dtype");
  if (out->dtype != PA_F32 && out->dtype != q->dtype)
    return pa::fail(PA_ERR_DTYPE, "out must be fp32 or the dtype of q");
  for (int i = 0; i < 4; ++i)
    if (k_cache->shape[i] != v_cache->shape[i]) return pa::fail(PA_ERR_ARG, "k_cache and v_cache shapes differ");
  if (!pa::is_contiguous(*k_cache) || !pa::is_contiguous(*v_cache))
    return pa::fail(PA_ERR_ARG, "caches must be contiguous");
  const int64_t rows = q->shape[0], hq = q->shape[1], d = q->shape[2];
  const int64_t nb = k_cache->shape[0], hkv = k_cache->shape[1], bs = k_cache->shape[2];
  const int64_t batch = context_lens->shape[0];
  if (k_cache->shape[3] != d) return pa::fail(PA_ERR_ARG, "cache head_dim differs from q");
  if (hkv < 1 || hq % hkv != 0) return pa::fail(PA_ERR_ARG, "Hq must be a positive multiple of Hkv");
  if (bs < 1) return pa::fail(PA_ERR_ARG, "block size must be positive");
  if (block_tables->shape[0] != batch) return pa::fail(PA_ERR_ARG, "block_tables batch differs from context_lens");
  if (query_start->shape[0] != batch + 1) return pa::fail(PA_ERR_ARG, "query_start must have batch + 1 entries");
  for (int i = 0; i < 3; ++i)
    if (out->shape[i] != q->shape[i]) return pa::fail(PA_ERR_ARG, "out shape differs from q");
  if ((q->stride[2] != 1 || out->stride[2] != 1) && d > 1)
    return pa::fail(PA_ERR_ARG, "q and out need a contiguous last dimension");
  if (max_query_len < 0) return pa::fail(PA_ERR_ARG, "max_query_len must be >= 0");
  if (d > kGenericMaxD) return pa::fail(PA_ERR_ARG, "head_dim above 512 is not supported");
  if (nb * hkv * bs > INT32_MAX) return pa::fail(PA_ERR_ARG, "cache has more than 2^31 rows");
  if (rows > INT32_MAX / 2 || batch > INT32_MAX / 2) return pa::fail(PA_ERR_ARG, "too many rows or sequences");
  if (batch == 0 || rows == 0 || max_query_len == 0) return PA_OK;
  if (!q->data || !k_cache->data || !v_cache->data || !block_tables->data || !context_lens->data ||
      !query_start->data || !out->data)
    return pa::fail(PA_ERR_ARG, "NULL data pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int group = int(hq / hkv);
  const int elt = int(pa::dtype_size(q->dtype));
  const int oelt = int(pa::dtype_size(out->dtype));

  PrefillParams p;
  p.q = q->data;
  p.q_t = q->stride[0];
  p.q_h = q->stride[1];
  p.tables = static_cast<const int32_t*>(block_tables->data);
  p.tab_s = block_tables->stride[0];
  p.tab_b = block_tables->stride[1];
  p.lens = static_cast<const int32_t*>(context_lens->data);
  p.len_s = context_lens->stride[0];
  p.qstart = static_cast<const int32_t*>(query_start->data);
  p.qs_s = query_start->stride[0];
  p.out = out->data;
  p.out_t = out->stride[0];
  p.out_h = out->stride[1];
  p.k_cache = k_cache->data;
  p.v_cache = v_cache->data;
  p.batch = int(batch);
  p.hq = int(hq);
  p.hkv = int(hkv);
  p.group = group;
  p.d = int(d);
  p.block_size = int(bs);
  p.num_blocks = int(nb);
  p.max_tokens = int(std::min<int64_t>(block_tables->shape[1] * bs, INT32_MAX));
  p.total_rows = int(rows);
  p.scale_log2 = scale * kLog2e;
  p.n_splits = 1;
  p.split_keys = int(std::min<int64_t>((int64_t(p.max_tokens) + kBN - 1) / kBN * kBN, INT32_MAX - kBN));
  p.ws_acc = nullptr;
  p.ws_ml = nullptr;

  // the tensor-core kernel takes the maximum of raw scores, so it needs scale > 0
  const bool fast = g_prefill_path == 0 && scale > 0.f && q->dtype != PA_F32 && bs == kBlock &&
                    (d == 64 || d == 128 || d == 256) &&
                    ((group >= 1 && group <= 8) || group == 16) && aligned16(q->data) &&
                    aligned16(out->data) && (q->stride[0] * elt) % 16 == 0 && (q->stride[1] * elt) % 16 == 0 &&
                    (out->stride[0] * oelt) % 16 == 0 && (out->stride[1] * oelt) % 16 == 0 &&
                    aligned16(k_cache->data) && aligned16(v_cache->data);
  if (fast) {
    const int tt = kBM / group;
    p.tiles_per_seq = (max_query_len + tt - 1) / tt;
    // key partitions when the (query tile, KV head) grid would leave SMs idle
    // and the caller gave room for the partial states
    int keys = 0;
    const int n = prefill_splits(p.tiles_per_seq, batch, hkv, p.max_tokens, device_sms(), &keys);
    const size_t need = split_workspace_bytes(n, rows, hq, d);
    if (n > 1 && workspace && workspace->data && size_t(workspace->shape[0]) >= need) {
      p.n_splits = n;
      p.split_keys = keys;
      char* ws = static_cast<char*>(workspace->data);
      p.ws_acc = reinterpret_cast<float*>(ws);
      p.ws_ml = reinterpret_cast<float2*>(ws + ((size_t(n) * rows * hq * d * sizeof(float) + 255) & ~size_t(255)));
    }
    const int64_t grid = int64_t(p.tiles_per_seq) * batch * hkv * p.n_splits;
    if (grid > INT32_MAX) return pa::fail(PA_ERR_ARG, "too many query tiles");
    CUtensorMap km, vm;
    int rc = pa::encode_page_map(&km, *k_cache);
    if (rc == PA_OK) rc = pa::encode_page_map(&vm, *v_cache);
    if (rc != PA_OK) return rc;
    const unsigned g = unsigned(grid);
    const bool o32 = out->dtype == PA_F32;
    if (q->dtype == PA_BF16)
      rc = o32 ? launch_tc_any<__nv_bfloat16, float>(int(d), group, km, vm, p, g, s)
               : launch_tc_any<__nv_bfloat16, __nv_bfloat16>(int(d), group, km, vm, p, g, s);
    else
      rc = o32 ? launch_tc_any<__half, float>(int(d), group, km, vm, p, g, s)
               : launch_tc_any<__half, __half>(int(d), group, km, vm, p, g, s);
    if (rc != PA_OK || p.n_splits == 1) return rc;
    const int64_t blocks = (rows * hq + 3) / 4;
    if (o32) prefill_merge_kernel<float><<<unsigned(blocks), 128, 0, s>>>(p);
    else if (q->dtype == PA_BF16) prefill_merge_kernel<__nv_bfloat16><<<unsigned(blocks), 128, 0, s>>>(p);
    else prefill_merge_kernel<__half><<<unsigned(blocks), 128, 0, s>>>(p);
    pa::count_launches(1);
    return cuda_status("prefill merge kernel launch");
  }
  p.tiles_per_seq = 0;
  switch (q->dtype) {
    case PA_F32: return launch_generic<float, float>(p, s);
    case PA_F16:
      return out->dtype == PA_F32 ? launch_generic<__half, float>(p, s) : launch_generic<__half, __half>(p, s);
    default:
      return out->dtype == PA_F32 ? launch_generic<__nv_bfloat16, float>(p, s)
                                  : launch_generic<__nv_bfloat16, __nv_bfloat16>(p, s);
  }
}
