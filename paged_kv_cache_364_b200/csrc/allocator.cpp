// Host-side block allocator: free pool, reference counts, per-sequence block
// tables, append (slot mapping), fork, copy-on-write and free.
//
// Procedures follow the PagedAttention pages:
//  - "Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
//    Technical Details: "Single Sequence Generation" (a new physical block once
//    the current one is full; waste bounded by the last block), "Copy-on-Write
//    for Parallel Sampling" (shared blocks carry a reference count; on
//    divergence only the diverging block is copied and counts are adjusted),
//    "Beam Search Optimization" (a block whose count reaches zero returns to
//    the free pool);
//  - "49 vLLM / PagedAttention", "The block table (the paging idea)": the
//    allocation test len(blocks) * B <= tokens-stored-before-the-append.
// Readings: the free pool is a LIFO stack; a writer copies iff the block it
// writes into is shared at that moment; freeing walks the table in order.
// Every failing call leaves the state unchanged.
#include <algorithm>
#include <cstring>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"
#include "pa_host.h"

struct pa_alloc {
  int32_t num_blocks = 0;
  std::vector<int32_t> free_stack;   // back() is handed out next
  std::vector<int32_t> refcount;
};

struct pa_seqs {
  pa_alloc* pool = nullptr;
  int32_t block_size = 0;
  int32_t next_id = 0;
  struct Seq {
    std::vector<int32_t> blocks;
    int32_t len = 0;
  };
  std::unordered_map<int32_t, Seq> seqs;
};

namespace {

bool in_pool(const pa_alloc* a, int32_t b) { return b >= 0 && b < a->num_blocks; }

int pop_block(pa_alloc* a, int32_t* out) {
  if (a->free_stack.empty()) return pa::fail(PA_ERR_OOM, "free pool is empty");
  int32_t b = a->free_stack.back();
  a->free_stack.pop_back();
  a->refcount[b] = 1;
  *out = b;
  return PA_OK;
}

// Copy-on-write test without argument checks (caller validated `block`).
int cow_block(pa_alloc* a, int32_t block, int32_t* target, bool* copied) {
  if (a->refcount[block] > 1) {
    int32_t fresh;
    int rc = pop_block(a, &fresh);
    if (rc != PA_OK) return rc;
    a->refcount[block] -= 1;
    *target = fresh;
    *copied = true;
  } else {
    *target = block;
    *copied = false;
  }
  return PA_OK;
}

// One token for one sequence.  State is unchanged on error.
int append_one(pa_seqs* s, pa_seqs::Seq& q, int32_t* slot, int64_t* pair, bool* has_pair) {
  const int32_t B = s->block_size;
  const int32_t n = q.len;
  *has_pair = false;
  if (static_cast<int64_t>(q.blocks.size()) * B <= n) {
    int32_t b;
    int rc = pop_block(s->pool, &b);
    if (rc != PA_OK) return rc;
    q.blocks.push_back(b);
  } else {
    int32_t last = q.blocks.back();
    int32_t target;
    bool copied;
    int rc = cow_block(s->pool, last, &target, &copied);
    if (rc != PA_OK) return rc;
    if (copied) {
      q.blocks.back() = target;
      pair[0] = last;
      pair[1] = target;
      *has_pair = true;
    }
  }
  *slot = q.blocks[n / B] * B + n % B;
  q.len = n + 1;
  return PA_OK;
}

}  // namespace

extern "C" {

int pa_alloc_create(int32_t num_blocks, const int32_t* init_free_order, pa_alloc** out) {
  pa::clear_error();
  if (!out) return pa::fail(PA_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (num_blocks < 0) return pa::fail(PA_ERR_ARG, "num_blocks < 0");
  auto* a = new pa_alloc;
  a->num_blocks = num_blocks;
  a->refcount.assign(num_blocks, 0);
  a->free_stack.resize(num_blocks);
  if (init_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      int32_t b = init_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return pa::fail(PA_ERR_ARG, "init_free_order is not a permutation of 0..num_blocks-1");
      }
      seen[b] = 1;
      a->free_stack[i] = b;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->free_stack[i] = num_blocks - 1 - i;
  }
  *out = a;
  return PA_OK;
}

int pa_alloc_destroy(pa_alloc* a) {
  pa::clear_error();
  delete a;
  return PA_OK;
}

int pa_alloc_block(pa_alloc* a, int32_t* block_out) {
  pa::clear_error();
  if (!a || !block_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  return pop_block(a, block_out);
}

int pa_alloc_incref(pa_alloc* a, const int32_t* blocks, int32_t n, int32_t by) {
  pa::clear_error();
  if (!a || (n > 0 && !blocks) || n < 0) return pa::fail(PA_ERR_ARG, "bad arguments");
  if (by < 0) return pa::fail(PA_ERR_STATE, "negative increment");
  for (int32_t i = 0; i < n; ++i)
    if (!in_pool(a, blocks[i]) || a->refcount[blocks[i]] <= 0)
      return pa::fail(PA_ERR_STATE, "incref of a block that is not in use");
  for (int32_t i = 0; i < n; ++i) a->refcount[blocks[i]] += by;
  return PA_OK;
}

int pa_alloc_decref(pa_alloc* a, const int32_t* blocks, int32_t n) {
  pa::clear_error();
  if (!a || (n > 0 && !blocks) || n < 0) return pa::fail(PA_ERR_ARG, "bad arguments");
  std::unordered_map<int32_t, int32_t> need;
  for (int32_t i = 0; i < n; ++i) {
    if (!in_pool(a, blocks[i])) return pa::fail(PA_ERR_STATE, "decref of a block outside the pool");
    need[blocks[i]] += 1;
  }
  for (const auto& kv : need)
    if (a->refcount[kv.first] < kv.second)
      return pa::fail(PA_ERR_STATE, "reference count would go below zero");
  for (int32_t i = 0; i < n; ++i) {
    int32_t b = blocks[i];
    if (--a->refcount[b] == 0) a->free_stack.push_back(b);
  }
  return PA_OK;
}

int pa_alloc_cow(pa_alloc* a, int32_t block, int32_t* target_out, int32_t* copied_out) {
  pa::clear_error();
  if (!a || !target_out || !copied_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  if (!in_pool(a, block) || a->refcount[block] <= 0)
    return pa::fail(PA_ERR_STATE, "copy-on-write of a block that is not in use");
  bool copied;
  int rc = cow_block(a, block, target_out, &copied);
  if (rc == PA_OK) *copied_out = copied ? 1 : 0;
  return rc;
}

int pa_alloc_refcount(const pa_alloc* a, int32_t block, int32_t* rc_out) {
  pa::clear_error();
  if (!a || !rc_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  if (!in_pool(a, block)) return pa::fail(PA_ERR_ARG, "block outside the pool");
  *rc_out = a->refcount[block];
  return PA_OK;
}

int pa_alloc_num_free(const pa_alloc* a, int32_t* n_out) {
  pa::clear_error();
  if (!a || !n_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  *n_out = static_cast<int32_t>(a->free_stack.size());
  return PA_OK;
}

int pa_alloc_num_blocks(const pa_alloc* a, int32_t* n_out) {
  pa::clear_error();
  if (!a || !n_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  *n_out = a->num_blocks;
  return PA_OK;
}

int pa_alloc_free_list(const pa_alloc* a, int32_t* out, int32_t cap, int32_t* n_out) {
  pa::clear_error();
  if (!a || !n_out || (cap > 0 && !out)) return pa::fail(PA_ERR_ARG, "NULL argument");
  int32_t n = static_cast<int32_t>(a->free_stack.size());
  *n_out = n;
  if (!out && cap == 0) return PA_OK;   // size query
  if (cap < n) return pa::fail(PA_ERR_ARG, "output capacity too small");
  if (n) std::memcpy(out, a->free_stack.data(), sizeof(int32_t) * n);
  return PA_OK;
}

int pa_alloc_refcounts(const pa_alloc* a, int32_t* out, int32_t cap) {
  pa::clear_error();
  if (!a || (cap > 0 && !out)) return pa::fail(PA_ERR_ARG, "NULL argument");
  if (cap < a->num_blocks) return pa::fail(PA_ERR_ARG, "output capacity too small");
  if (a->num_blocks) std::memcpy(out, a->refcount.data(), sizeof(int32_t) * a->num_blocks);
  return PA_OK;
}

int pa_seqs_create(pa_alloc* pool, int32_t block_size, pa_seqs** out) {
  pa::clear_error();
  if (!out) return pa::fail(PA_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (!pool) return pa::fail(PA_ERR_ARG, "pool is NULL");
  if (block_size < 1) return pa::fail(PA_ERR_ARG, "block_size < 1");
  auto* s = new pa_seqs;
  s->pool = pool;
  s->block_size = block_size;
  *out = s;
  return PA_OK;
}

int pa_seqs_destroy(pa_seqs* s) {
  pa::clear_error();
  delete s;
  return PA_OK;
}

int pa_seqs_add(pa_seqs* s, int32_t* seq_out) {
  pa::clear_error();
  if (!s || !seq_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  int32_t id = s->next_id++;
  s->seqs.emplace(id, pa_seqs::Seq{});
  *seq_out = id;
  return PA_OK;
}

int pa_seqs_append(pa_seqs* s, const int32_t* seq_ids, int32_t n, int32_t* slots_out,
                   int64_t* cow_pairs_out, int32_t* n_cow_out, int32_t* n_done_out) {
  pa::clear_error();
  if (!s || n < 0 || (n > 0 && (!seq_ids || !slots_out || !cow_pairs_out)) || !n_cow_out)
    return pa::fail(PA_ERR_ARG, "bad arguments");
  int32_t n_cow = 0;
  if (n_done_out) *n_done_out = 0;
  *n_cow_out = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = s->seqs.find(seq_ids[i]);
    if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
    bool has_pair;
    int rc = append_one(s, it->second, &slots_out[i], &cow_pairs_out[2 * n_cow], &has_pair);
    if (rc != PA_OK) return rc;
    if (has_pair) ++n_cow;
    *n_cow_out = n_cow;
    if (n_done_out) *n_done_out = i + 1;
  }
  return PA_OK;
}

int pa_seqs_append_n(pa_seqs* s, int32_t seq, int32_t n_tokens, int32_t* slots_out,
                     int64_t* cow_pairs_out, int32_t* n_cow_out) {
  pa::clear_error();
  if (!s || n_tokens < 0 || (n_tokens > 0 && (!slots_out || !cow_pairs_out)) || !n_cow_out)
    return pa::fail(PA_ERR_ARG, "bad arguments");
  auto it = s->seqs.find(seq);
  if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
  int32_t n_cow = 0;
  *n_cow_out = 0;
  for (int32_t i = 0; i < n_tokens; ++i) {
    bool has_pair;
    int rc = append_one(s, it->second, &slots_out[i], &cow_pairs_out[2 * n_cow], &has_pair);
    if (rc != PA_OK) return rc;
    if (has_pair) ++n_cow;
    *n_cow_out = n_cow;
  }
  return PA_OK;
}

int pa_seqs_fork(pa_seqs* s, int32_t parent, int32_t* child_out) {
  pa::clear_error();
  if (!s || !child_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  auto it = s->seqs.find(parent);
  if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
  const auto& blocks = it->second.blocks;
  int rc = pa_alloc_incref(s->pool, blocks.data(), static_cast<int32_t>(blocks.size()), 1);
  if (rc != PA_OK) return rc;
  pa_seqs::Seq child = it->second;   // copy before emplace (rehash)
  int32_t id = s->next_id++;
  s->seqs.emplace(id, std::move(child));
  *child_out = id;
  return PA_OK;
}

int pa_seqs_free(pa_seqs* s, int32_t seq) {
  pa::clear_error();
  if (!s) return pa::fail(PA_ERR_ARG, "NULL argument");
  auto it = s->seqs.find(seq);
  if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
  const auto& blocks = it->second.blocks;
  int rc = pa_alloc_decref(s->pool, blocks.data(), static_cast<int32_t>(blocks.size()));
  if (rc != PA_OK) return rc;
  s->seqs.erase(it);
  return PA_OK;
}

int pa_seqs_len(const pa_seqs* s, int32_t seq, int32_t* len_out) {
  pa::clear_error();
  if (!s || !len_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  auto it = s->seqs.find(seq);
  if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
  *len_out = it->second.len;
  return PA_OK;
}

int pa_seqs_table(const pa_seqs* s, int32_t seq, int32_t* out, int32_t cap, int32_t* n_out) {
  pa::clear_error();
  if (!s || !n_out || (cap > 0 && !out)) return pa::fail(PA_ERR_ARG, "NULL argument");
  auto it = s->seqs.find(seq);
  if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
  const auto& b = it->second.blocks;
  int32_t n = static_cast<int32_t>(b.size());
  *n_out = n;
  if (!out && cap == 0) return PA_OK;   // size query
  if (cap < n) return pa::fail(PA_ERR_ARG, "output capacity too small");
  if (n) std::memcpy(out, b.data(), sizeof(int32_t) * n);
  return PA_OK;
}

int pa_seqs_live(const pa_seqs* s, int32_t* out, int32_t cap, int32_t* n_out) {
  pa::clear_error();
  if (!s || !n_out || (cap > 0 && !out)) return pa::fail(PA_ERR_ARG, "NULL argument");
  std::vector<int32_t> ids;
  ids.reserve(s->seqs.size());
  for (const auto& kv : s->seqs) ids.push_back(kv.first);
  std::sort(ids.begin(), ids.end());
  int32_t n = static_cast<int32_t>(ids.size());
  *n_out = n;
  if (!out && cap == 0) return PA_OK;   // size query
  if (cap < n) return pa::fail(PA_ERR_ARG, "output capacity too small");
  if (n) std::memcpy(out, ids.data(), sizeof(int32_t) * n);
  return PA_OK;
}

int pa_seqs_block_tables(const pa_seqs* s, const int32_t* seq_ids, int32_t n,
                         int32_t max_blocks, int32_t pad, int32_t* tables_out,
                         int32_t* lens_out) {
  pa::clear_error();
  if (!s || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !tables_out || !lens_out)))
    return pa::fail(PA_ERR_ARG, "bad arguments");
  for (int32_t i = 0; i < n; ++i) {
    auto it = s->seqs.find(seq_ids[i]);
    if (it == s->seqs.end()) return pa::fail(PA_ERR_STATE, "unknown sequence id");
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks)
      return pa::fail(PA_ERR_ARG, "a block table is longer than max_blocks");
  }
  for (int32_t i = 0; i < n; ++i) {
    const auto& q = s->seqs.find(seq_ids[i])->second;
    int32_t* row = tables_out + static_cast<int64_t>(i) * max_blocks;
    int32_t nb = static_cast<int32_t>(q.blocks.size());
    if (nb) std::memcpy(row, q.blocks.data(), sizeof(int32_t) * nb);
    for (int32_t j = nb; j < max_blocks; ++j) row[j] = pad;
    lens_out[i] = q.len;
  }
  return PA_OK;
}

}  // extern "C"
