/*
 * pagedkv.h -- C ABI of the B200 paged KV cache library (libpagedkv.so).
 *
 * The library implements the data-parallel hot path of PagedAttention:
 *   - the KV cache is cut into fixed-size physical blocks of B token slots
 *     ("Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
 *     Technical Details, "Core Architecture": fixed-size KV blocks, default
 *     B = 16, reached through a block table that maps contiguous logical
 *     blocks to scattered physical blocks);
 *   - pa_write_kv appends new tokens' K/V into their physical slots;
 *   - pa_decode computes single-query attention per sequence by walking its
 *     block table ("PagedAttention: How Virtual Memory Paging Solved LLM KV
 *     Cache Waste", Why it matters: the attention kernel gathers scattered
 *     blocks on the fly; Key points: the transformer math is unchanged);
 *   - pa_decode_append does both in one call (the attention kernel stores
 *     each sequence's new token while it stages that token's page);
 *   - pa_prefill computes causal attention of several new tokens per
 *     sequence over its paged context (a prompt, a chunk of one, or tokens
 *     after a cached or shared prefix) on the tensor cores;
 *   - pa_copy_blocks performs the block copies of copy-on-write ("Stop
 *     Wasting GPU Memory ...", Technical Details, "Copy-on-Write for Parallel
 *     Sampling");
 *   - pa_alloc_* / pa_seqs_* are the host-side block allocator: a free pool,
 *     a reference count per physical block, per-sequence block tables
 *     ("Stop Wasting GPU Memory ...", Technical Details, "Copy-on-Write ..."
 *     and "Beam Search Optimization"; "49 vLLM / PagedAttention", "The block
 *     table (the paging idea)").
 *
 * Conventions
 *   - Every function returns an int: PA_OK (0) or a negative PA_ERR_* code.
 *     pa_strerror() names a code; pa_last_error() gives the calling thread's
 *     most recent detailed message.
 *   - The library never allocates device memory (pa_decode_noalloc's scratch
 *     is a fixed array inside the library).  All tensors are owned by
 *     the caller (normally allocated by PyTorch) and passed as pa_tensor
 *     descriptors: a data pointer, a dtype, a rank and shape/stride arrays
 *     (strides in elements).  Device tensors are CUDA device pointers.
 *   - Kernel entry points take a CUDA stream (cudaStream_t passed as void*;
 *     NULL is the legacy default stream), validate every argument on the host
 *     before launching, enqueue their work and return without synchronising.
 *     An argument error returns before anything is enqueued.
 *   - Device kernels never fault on bad table contents: an out-of-range block
 *     id, slot, length or copy pair is skipped and recorded in a sticky device
 *     error word, read (and cleared) with pa_device_errors().
 *   - Cache layout: k_cache and v_cache are [num_blocks, num_kv_heads, B,
 *     head_dim], contiguous, so one (block, KV head) page is one contiguous
 *     run of B * head_dim elements.
 *   - Allocator objects are host-only, not thread-safe, and never touch the
 *     GPU; a caller serialises its own access.
 *   - List getters (pa_alloc_free_list, pa_seqs_table, pa_seqs_live) write the
 *     length to *n_out; called with out = NULL and cap = 0 they only report it.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status -- */
enum {
  PA_OK = 0,
  PA_ERR_ARG = -1,     /* a shape, stride, size or scalar argument is invalid */
  PA_ERR_DTYPE = -2,   /* unsupported dtype, or dtypes that must match do not */
  PA_ERR_OOM = -3,     /* the free pool is empty (allocator state unchanged) */
  PA_ERR_STATE = -4,   /* a reference count would become invalid, unknown id */
  PA_ERR_BOUNDS = -5,  /* a device-side bounds check fired (pa_device_errors) */
  PA_ERR_CUDA = -6,    /* a CUDA runtime call failed (message in pa_last_error) */
  PA_ERR_TIMEOUT = -7  /* a bounded device-side wait ran out */
};

/* Device error bits reported by pa_device_errors(). */
enum {
  PA_DEVERR_BLOCK_ID = 1,      /* block table entry outside [0, num_blocks) */
  PA_DEVERR_SLOT = 2,          /* slot outside [0, num_blocks * B) and not -1 */
  PA_DEVERR_CONTEXT_LEN = 4,   /* context_len < 1 or > max_blocks * B or > max_context */
  PA_DEVERR_COPY_PAIR = 8,     /* copy pair block id outside the pool */
  PA_DEVERR_WAIT_TIMEOUT = 16, /* a bounded wait on a copy completion ran out */
  PA_DEVERR_ALIAS = 32         /* checked mode: aliasing writes found (see PA_OPT_CHECKED) */
};

typedef enum {
  PA_F32 = 0,
  PA_F16 = 1,
  PA_BF16 = 2,
  PA_I32 = 3,
  PA_I64 = 4,
  PA_U8 = 5
} pa_dtype;

#define PA_MAX_DIMS 5

typedef struct {
  void* data;                 /* device pointer (first element) */
  int32_t dtype;              /* a pa_dtype */
  int32_t ndim;               /* 0 .. PA_MAX_DIMS */
  int64_t shape[PA_MAX_DIMS];
  int64_t stride[PA_MAX_DIMS];/* in elements */
} pa_tensor;

typedef void* pa_stream;      /* a cudaStream_t */

const char* pa_strerror(int code);
/* Detailed message of the calling thread's last failing call ("" if none). */
const char* pa_last_error(void);
/* Library version, e.g. "1.0.0". */
const char* pa_version(void);
/* Number of CUDA kernels this library has enqueued since it was loaded. */
int pa_launch_count(uint64_t* count_out);

/* Synchronise `stream`, then return and clear the sticky device error bits
 * (PA_DEVERR_*) that kernels on the current device have set.  For tests and
 * checked runs; it blocks the host. */
int pa_device_errors(pa_stream stream, uint32_t* bits_out);

/* Self-test of the kernels' bounded waits: a one-thread kernel waits on a
 * shared-memory barrier that nothing completes, gives up after `polls` polls
 * (1 .. 2^22) and sets PA_DEVERR_WAIT_TIMEOUT, which pa_device_errors() then
 * reports.  It ends on its own; no GPU state is left behind. */
int pa_selftest_bounded_wait(uint32_t polls, pa_stream stream);

/* ------------------------------------------------------------ slot write -- */
/*
 * pa_write_kv -- store each new token's K and V rows into its physical slot.
 * ("Stop Wasting GPU Memory ...", Technical Details, "Single Sequence
 * Generation": new tokens fill the remaining slots of the current physical
 * block; "49 vLLM / PagedAttention", "The block table (the paging idea)".)
 *
 *   k, v          [T, Hkv, head_dim]  fp32 | fp16 | bf16, last dim contiguous
 *   slot_mapping  [T] int32: slot = block * B + offset, or -1 to skip token
 *   k_cache,      [num_blocks, Hkv, B, head_dim], contiguous, same dtype as k
 *   v_cache
 *
 * For each t with slot_mapping[t] = s != -1:
 *   k_cache[s / B, h, s % B, :] = k[t, h, :] (all h), likewise v.
 * The copy is bitwise.  Slots must be distinct (two tokens writing one slot
 * race).  A slot outside the pool is skipped and sets PA_DEVERR_SLOT.
 * T = 0 is a no-op.
 */
int pa_write_kv(const pa_tensor* k, const pa_tensor* v, const pa_tensor* slot_mapping,
                const pa_tensor* k_cache, const pa_tensor* v_cache, pa_stream stream);

/* ---------------------------------------------------------- decode ------- */
/*
 * Bytes of scratch that pa_decode needs for a batch whose longest context is
 * max_context tokens, split into partitions of partition_tokens tokens.
 * Returns 0 for invalid arguments.
 */
size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context, int32_t partition_tokens);

/*
 * pa_decode -- single-query decode attention over the paged cache.
 * ("PagedAttention: How Virtual Memory Paging Solved LLM KV Cache Waste",
 * Key points: paging leaves the attention math unchanged; Why it matters:
 * the kernel gathers the scattered blocks through the block table.)
 *
 *   q             [batch, Hq, head_dim]  fp32 | fp16 | bf16, last dim contiguous
 *   k_cache,      [num_blocks, Hkv, B, head_dim], contiguous, dtype of q;
 *   v_cache       Hq must be a multiple of Hkv
 *   block_tables  [batch, max_blocks] int32, row s lists the physical blocks of
 *                 sequence s in logical order (entries past its last block
 *                 are not read)
 *   context_lens  [batch] int32, tokens attended by sequence s, in
 *                 [1, min(max_blocks * B, max_context)]
 *   scale         softmax scale applied to q . k (commonly 1/sqrt(head_dim))
 *   max_context   host-side upper bound of context_lens (sizes the split)
 *   partition_tokens  split-context partition length, a positive multiple of B
 *   workspace     uint8 device buffer of >= pa_decode_workspace_size() bytes,
 *                 256-byte aligned; its contents are scratch and need no
 *                 initialisation; concurrent calls need distinct workspaces
 *   out           [batch, Hq, head_dim], fp32 or the dtype of q, last dim
 *                 contiguous
 *
 * For query head h of sequence s, with g = Hq / Hkv and KV head h / g:
 *   out[s, h] = softmax(scale * K_s q[s, h]) V_s
 * where K_s, V_s are the first context_lens[s] token rows reached through the
 * block table.  Computed with fp32 accumulation and a streaming softmax;
 * contexts longer than one partition are split and their partial states are
 * merged by log-sum-exp.  A narrow `out` is rounded to nearest even.
 * Rows with an invalid context length are left unwritten and set
 * PA_DEVERR_CONTEXT_LEN; invalid block ids are skipped (PA_DEVERR_BLOCK_ID).
 * batch = 0 is a no-op.
 */
int pa_decode(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
              const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
              int32_t max_context, int32_t partition_tokens, const pa_tensor* workspace,
              const pa_tensor* out, pa_stream stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  The pages describe no such variant; it has no counterpart there.
 *
 * Same arguments and result as pa_decode, without the workspace: its scratch
 * lives in a 32 MiB array built into the library (every GPU that loads it
 * keeps that memory until the process exits).  Meant for callers that must
 * not allocate after start-up -- e.g. a serving engine that gives nearly all
 * HBM to its block pool up front -- or that have no device allocator at all
 * (a plain C host that only owns the tensors it passes in).  The call issues
 * no cudaMalloc/cudaFree and calls no allocating routine.
 *   - A batch whose scratch (pa_decode_workspace_size) exceeds 32 MiB is
 *     rejected with PA_ERR_ARG before anything is launched; so is a q with a
 *     negative batch, no query head or head_dim < 1.
 *   - When the 32 MiB is taken: with the CUDA runtime's default lazy module
 *     loading the array is allocated when its module is first used on a
 *     device, i.e. by the first call on that device (with
 *     CUDA_MODULE_LOADING=EAGER, when the library's modules load).  A caller
 *     that reserves nearly all HBM for its block pool must make one call per
 *     device BEFORE reserving it; a call with an empty batch (q of shape
 *     [0, Hq, head_dim]) does only this set-up.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call outside any stream capture.
 *     The address is kept with the id of its CUDA context, and looked up
 *     again by a call that finds another context current (after
 *     cudaDeviceReset): make that call outside stream capture too.
 *   - All calls share the array and it keeps the last call's contents;
 *     nothing in it needs to start at zero.  Calls that can overlap on the
 *     GPU (unordered streams) race on it: order them on one stream.
 */
int pa_decode_noalloc(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
                      const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                      int32_t max_context, int32_t partition_tokens, const pa_tensor* out,
                      pa_stream stream);

/*
 * pa_decode_append -- store each sequence's new token and attend over the
 * context that includes it, in one call.
 * ("Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
 * Technical Details, "Single Sequence Generation": each new token's K/V fills
 * the next slot of the sequence's current block; "49 vLLM / PagedAttention",
 * "The block table (the paging idea)": the append writes into the last block.)
 *
 *   k_new, v_new  [batch, Hkv, head_dim], dtype of the caches, last dim
 *                 contiguous: the K and V rows of the token at position
 *                 context_lens[s] - 1 of sequence s
 *   all other arguments as for pa_decode (same workspace size)
 *
 * Result: the caches as after pa_write_kv with
 *   slot[s] = block_tables[s][(n_s - 1) / B] * B + (n_s - 1) % B,  n_s = context_lens[s],
 * followed by pa_decode -- the same output bits and cache bits.  The block
 * holding position n_s - 1 must belong to sequence s alone (the allocator's
 * copy-on-write gives a writer a private block), so no other sequence of the
 * batch reads the slot being written.
 * On the fast path (fp16/bf16, B = 16, head_dim 64/128/256, Hq/Hkv <= 8 or
 * Hq/Hkv = 16 at head_dim <= 128, 16-byte aligned k_new / v_new rows) the
 * attention kernel stores the rows
 * itself, as it stages the token's page, and the step has no separate write
 * launch; otherwise one small kernel stores them first.  A sequence with an
 * invalid context length gets no write and no output (PA_DEVERR_CONTEXT_LEN);
 * an invalid block id skips the write (PA_DEVERR_BLOCK_ID).
 */
int pa_decode_append(const pa_tensor* q, const pa_tensor* k_new, const pa_tensor* v_new,
                     const pa_tensor* k_cache, const pa_tensor* v_cache, const pa_tensor* block_tables,
                     const pa_tensor* context_lens, float scale, int32_t max_context,
                     int32_t partition_tokens, const pa_tensor* workspace, const pa_tensor* out,
                     pa_stream stream);

/* ---------------------------------------------------------- prefill ------ */
/*
 * pa_prefill -- attention of each sequence's new tokens (a prompt, a chunk of
 * one, or several speculative tokens) over its paged context.
 * ("Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
 * Technical Details, "Single Sequence Generation": prompt tokens go into
 * logical blocks mapped to arbitrary physical blocks; "49 vLLM /
 * PagedAttention", "Questions worth asking": a shared prompt prefix is stored
 * once and attended, not prefilled again.)
 *
 *   q             [rows, Hq, head_dim] fp32 | fp16 | bf16, last dim
 *                 contiguous: the query rows of all sequences, packed
 *   k_cache,      [num_blocks, Hkv, B, head_dim], contiguous, dtype of q,
 *   v_cache       already holding the new tokens' K/V (pa_write_kv first)
 *   block_tables  [batch, max_blocks] int32
 *   context_lens  [batch] int32: n_s, tokens of sequence s in the cache,
 *                 its new tokens included, n_s <= max_blocks * B
 *   query_start   [batch + 1] int32, nondecreasing, query_start[0] = 0,
 *                 query_start[batch] <= rows: sequence s owns query rows
 *                 query_start[s] .. query_start[s+1]-1, which are its last
 *                 q_len_s = query_start[s+1] - query_start[s] positions
 *                 (q_len_s <= n_s; 0 = nothing to do)
 *   scale         softmax scale applied to q . k
 *   max_query_len host-side upper bound of q_len_s (sizes the launch)
 *   workspace     NULL, or a uint8 device buffer (256-byte aligned) of
 *                 pa_prefill_workspace_size() bytes: when the launch would
 *                 leave SMs idle, the keys of each query tile are split into
 *                 partitions whose partial softmax states are kept there and
 *                 merged by log-sum-exp; with NULL (or too small) no split
 *   out           [rows, Hq, head_dim], fp32 or the dtype of q, last dim
 *                 contiguous
 *
 * Query row i of sequence s sits at position p = n_s - q_len_s + i and gets
 *   out[row, h] = softmax(scale * K_s[0..p] q[row, h]) V_s[0..p]
 * with KV head h / (Hq / Hkv): causal over the new tokens, the whole cached
 * prefix visible.  fp32 accumulation; a narrow `out` is rounded to nearest
 * even.  fp16/bf16 with B = 16, head_dim 64, 128 or 256, Hq / Hkv in
 * 1..8 or 16 and scale > 0 run on the tensor cores (tcgen05, accumulators in
 * tensor memory); everything else on a CUDA-core kernel.  Rows of a sequence with
 * inconsistent lengths or starts, and rows past max_query_len, are left
 * unwritten and set PA_DEVERR_CONTEXT_LEN; invalid block ids set
 * PA_DEVERR_BLOCK_ID.  No device memory is allocated; rows not owned by any
 * sequence are not written.  batch = 0, rows = 0 or max_query_len = 0 is a
 * no-op.
 */
int pa_prefill(const pa_tensor* q, const pa_tensor* k_cache, const pa_tensor* v_cache,
               const pa_tensor* block_tables, const pa_tensor* context_lens, const pa_tensor* query_start,
               float scale, int32_t max_query_len, const pa_tensor* workspace, const pa_tensor* out,
               pa_stream stream);

/*
 * Bytes of scratch pa_prefill can use to split the keys of a launch that
 * would otherwise leave SMs idle (few new tokens over long contexts); 0 when
 * such a launch would not be split.  max_tokens = max_blocks * B of the
 * block table.  Returns 0 for invalid arguments.
 */
size_t pa_prefill_workspace_size(int32_t rows, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t batch, int32_t max_query_len, int32_t max_tokens);

/* Process-wide options.
 *   PA_OPT_DECODE_PATH: 0 = automatic (default), 1 = always the generic
 *   CUDA-core kernel (any dtype, head size, group size and block size).
 *   PA_OPT_PREFILL_PATH: the same choice for pa_prefill.
 *   PA_OPT_CHECKED: 0 = off (default), 1 = checked mode.  Writes whose
 *   targets alias corrupt the cache silently (a shared block must be copied
 *   before a sequence writes into it: "Stop Wasting GPU Memory ...",
 *   "Copy-on-Write for Parallel Sampling"), so in checked mode a device
 *   pre-pass over the call's index arguments runs first:
 *     pa_write_kv       two tokens with the same live slot;
 *     pa_copy_blocks    a destination named twice, or also as a source;
 *     pa_decode_append  a sequence's newest block (where its new row goes)
 *                       that another sequence of the batch also reads, or
 *                       that its own table lists at another position.
 *   On a finding the call sets PA_DEVERR_ALIAS, writes and launches nothing
 *   else, and returns PA_ERR_BOUNDS (pa_last_error() names the count and the
 *   first offending token, pair or sequence).  The pre-pass synchronises the
 *   call's stream, so checked calls block the host and return PA_ERR_STATE
 *   inside a stream capture.  Off, nothing of it runs. */
enum { PA_OPT_DECODE_PATH = 1, PA_OPT_PREFILL_PATH = 2, PA_OPT_CHECKED = 3 };
int pa_set_option(int32_t key, int32_t value);
int pa_get_option(int32_t key, int32_t* value_out);

/* Measurement hook.  While enabled, every pa_decode call records a CUDA event
 * pair on its stream around its main attention kernel (not around the small
 * planning and merge kernels).  pa_profile_take() waits for the recorded
 * pairs, returns their summed duration in milliseconds and their count, and
 * forgets them.  Events are created on first use and reused; no device memory
 * is allocated. */
int pa_profile_enable(int32_t on);
int pa_profile_take(float* total_ms_out, int32_t* count_out);

/* Read-bandwidth probe, a measurement helper (no step of the method).  The
 * decode kernel is a pure reader of K/V pages, so it is compared with the
 * rate at which the GPU streams a buffer it only reads, as well as with a
 * copy's.
 *   buf    device pointer, 16-byte aligned; bytes a multiple of 16 (0 = no-op)
 *   sink   device pointer to one uint32: the XOR of every 32-bit word of buf
 *          is XORed into *sink (so a zeroed sink ends holding that XOR)
 * One asynchronous kernel on `stream`: 16-byte read-only loads, four in
 * flight per thread, 1024 threads per SM.  Time it with CUDA events on
 * `stream` over a buffer well above the 126 MB L2.  PA_ERR_ARG for a NULL
 * or misaligned pointer or a size that is not a multiple of 16. */
int pa_read_probe(const void* buf, uint64_t bytes, uint32_t* sink, pa_stream stream);

/* ------------------------------------------------------------ block copy -- */
/*
 * pa_copy_blocks -- copy-on-write block copies.
 * ("Stop Wasting GPU Memory ...", Technical Details, "Copy-on-Write for
 * Parallel Sampling": on divergence only the diverging block is copied to a
 * new physical location.)
 *
 *   caches        array of n_caches descriptors, each [num_blocks, ...]
 *                 contiguous, all with the same shape and dtype (normally the
 *                 K and V cache of every layer)
 *   src_dst_pairs [P, 2] int64 on the device: row i copies block pairs[i][0]
 *                 onto block pairs[i][1] in every cache
 *
 * Destinations must be distinct and must not be sources (the allocator's
 * fresh blocks are).  A pair with an id outside the pool is skipped and sets
 * PA_DEVERR_COPY_PAIR.  The copy is bitwise.  P = 0 is a no-op.
 */
int pa_copy_blocks(const pa_tensor* caches, int32_t n_caches, const pa_tensor* src_dst_pairs,
                   pa_stream stream);

/* ------------------------------------------------------- block allocator -- */
/*
 * Free pool + reference counts.  The pool is a LIFO stack seeded from
 * init_free_order (its last element is handed out first); NULL seeds it with
 * num_blocks-1 .. 0, so blocks come out as 0, 1, 2, ...
 * Every failing call leaves the allocator unchanged.
 */
typedef struct pa_alloc pa_alloc;

int pa_alloc_create(int32_t num_blocks, const int32_t* init_free_order, pa_alloc** out);
int pa_alloc_destroy(pa_alloc* a);
/* Pop a block (count becomes 1).  PA_ERR_OOM when the pool is empty. */
int pa_alloc_block(pa_alloc* a, int32_t* block_out);
/* Add `by` (>= 0) to the count of each listed block; every block must be in use. */
int pa_alloc_incref(pa_alloc* a, const int32_t* blocks, int32_t n, int32_t by);
/* Subtract one per listed occurrence; blocks reaching zero are pushed onto
 * the pool in list order.  PA_ERR_STATE if any count would go below zero. */
int pa_alloc_decref(pa_alloc* a, const int32_t* blocks, int32_t n);
/* Copy-on-write test for a block about to be written: if its count is above
 * one, pop a fresh block into *target_out, drop the old block's count by one
 * and set *copied_out = 1; else *target_out = block, *copied_out = 0. */
int pa_alloc_cow(pa_alloc* a, int32_t block, int32_t* target_out, int32_t* copied_out);
int pa_alloc_refcount(const pa_alloc* a, int32_t block, int32_t* rc_out);
int pa_alloc_num_free(const pa_alloc* a, int32_t* n_out);
int pa_alloc_num_blocks(const pa_alloc* a, int32_t* n_out);
/* Free pool contents bottom..top (the next block handed out is last). */
int pa_alloc_free_list(const pa_alloc* a, int32_t* out, int32_t cap, int32_t* n_out);
/* All reference counts, out[num_blocks]. */
int pa_alloc_refcounts(const pa_alloc* a, int32_t* out, int32_t cap);

/* Pool occupancy, for memory-utilisation accounting ("Stop Wasting GPU
 * Memory ...", "Copy-on-Write for Parallel Sampling": shared blocks carry a
 * reference count).  free_blocks + used_blocks = num_blocks. */
typedef struct {
  int32_t num_blocks;
  int32_t free_blocks;     /* in the free pool (count 0) */
  int32_t used_blocks;     /* count >= 1 */
  int32_t shared_blocks;   /* count >= 2: referenced by more than one holder */
  int64_t references;      /* sum of all counts */
} pa_alloc_stats_t;
int pa_alloc_stats(const pa_alloc* a, pa_alloc_stats_t* out);

/* --------------------------------------------------- sequence block tables -- */
/*
 * Per-sequence block tables on top of a pool (which must outlive them).
 * Sequence ids are handed out 0, 1, 2, ... and never reused.
 */
typedef struct pa_seqs pa_seqs;

int pa_seqs_create(pa_alloc* pool, int32_t block_size, pa_seqs** out);
int pa_seqs_destroy(pa_seqs* s);
int pa_seqs_add(pa_seqs* s, int32_t* seq_out);
/*
 * Place one new token for each listed sequence, in list order ("49 vLLM /
 * PagedAttention", "The block table (the paging idea)": a sequence holding n
 * tokens gets a new block when len(blocks) * B <= n; "Stop Wasting GPU Memory
 * ...", "Copy-on-Write for Parallel Sampling": a write into a shared block
 * first copies it).  For each: slots_out[i] = block * B + offset; when the
 * write needed a copy, the pair (old, new) is appended to cow_pairs_out
 * (int64 [n][2], room for n pairs).  On PA_ERR_OOM, *n_done_out sequences were
 * placed and the failing one is unchanged.
 */
int pa_seqs_append(pa_seqs* s, const int32_t* seq_ids, int32_t n, int32_t* slots_out,
                   int64_t* cow_pairs_out, int32_t* n_cow_out, int32_t* n_done_out);
/* Append `n_tokens` tokens to one sequence (a prompt); slots_out[n_tokens],
 * cow_pairs_out room for n_tokens pairs.  Tokens are placed one by one as by
 * pa_seqs_append; on PA_ERR_OOM the tokens placed before the failing one stay
 * (their slots and copies are in the outputs, *n_cow_out counts the copies). */
int pa_seqs_append_n(pa_seqs* s, int32_t seq, int32_t n_tokens, int32_t* slots_out,
                     int64_t* cow_pairs_out, int32_t* n_cow_out);
/* A child sharing every block of `parent` (each count grows by one). */
int pa_seqs_fork(pa_seqs* s, int32_t parent, int32_t* child_out);
/* Release a sequence: decrement its blocks in table order. */
int pa_seqs_free(pa_seqs* s, int32_t seq);
int pa_seqs_len(const pa_seqs* s, int32_t seq, int32_t* len_out);
int pa_seqs_table(const pa_seqs* s, int32_t seq, int32_t* out, int32_t cap, int32_t* n_out);
/* Number of live sequences and their ids (ascending). */
int pa_seqs_live(const pa_seqs* s, int32_t* out, int32_t cap, int32_t* n_out);
/* Rows for a decode batch: tables_out[n][max_blocks] (unused entries = pad)
 * and lens_out[n].  PA_ERR_ARG if a table is longer than max_blocks. */
int pa_seqs_block_tables(const pa_seqs* s, const int32_t* seq_ids, int32_t n,
                         int32_t max_blocks, int32_t pad, int32_t* tables_out,
                         int32_t* lens_out);

/*
 * Checkpoint / resume of the host-side state (the caches themselves are
 * caller-owned device tensors and are saved by the caller).
 *
 * pa_seqs_snapshot writes the pool and every live table into buf (cap bytes)
 * and the byte count to *n_out; buf = NULL with cap = 0 only reports the
 * size.  Layout, 32-bit integers in native byte order:
 *   magic 0x564B4150, version 1,
 *   num_blocks, block_size, next_id, n_free, n_seqs,
 *   free pool [n_free] (bottom .. top), counts [num_blocks],
 *   per live sequence in ascending id: id, len, n_blocks, blocks [n_blocks].
 * pa_seqs_restore builds a new pool and table set from such a buffer (the
 * caller destroys both, the tables first).  It checks the buffer before
 * building anything: exact size; every id in range; the free pool holds each
 * block of count 0 exactly once and no other; each table has
 * ceil(len / block_size) blocks, all in use; no block is referenced by more
 * tables than its count; ids ascending and below next_id.  PA_ERR_ARG
 * otherwise, with nothing created.  Restored state continues exactly as the
 * saved one would (same ids, same next blocks).
 */
int pa_seqs_snapshot(const pa_seqs* s, void* buf, uint64_t cap, uint64_t* n_out);
int pa_seqs_restore(const void* buf, uint64_t n, pa_alloc** pool_out, pa_seqs** seqs_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
