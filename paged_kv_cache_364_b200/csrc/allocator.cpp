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
// Every failing call leaves the state unchanged.  Beyond the pages: pool
// statistics (pa_alloc_stats) and a checkpoint of the pool and tables
// (pa_seqs_snapshot / pa_seqs_restore) that restore validates in full.
#include <algorithm>
#include <cstring>
#include <string>
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

// Snapshot header: "PAKV" read as a little-endian 32-bit word, and the layout version.
constexpr uint32_t kSnapMagic = 0x564B4150u;
constexpr int32_t kSnapVersion = 1;

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


int pa_alloc_stats(const pa_alloc* a, pa_alloc_stats_t* out) {
  pa::clear_error();
  if (!a || !out) return pa::fail(PA_ERR_ARG, "NULL argument");
  pa_alloc_stats_t st{};
  st.num_blocks = a->num_blocks;
  st.free_blocks = static_cast<int32_t>(a->free_stack.size());
  for (int32_t c : a->refcount) {
    st.used_blocks += c > 0;
    st.shared_blocks += c > 1;
    st.references += c;
  }
  *out = st;
  return PA_OK;
}

int pa_seqs_snapshot(const pa_seqs* s, void* buf, uint64_t cap, uint64_t* n_out) {
  pa::clear_error();
  if (!s || !n_out || (cap > 0 && !buf)) return pa::fail(PA_ERR_ARG, "NULL argument");
  const pa_alloc* a = s->pool;
  std::vector<int32_t> ids;
  ids.reserve(s->seqs.size());
  for (const auto& kv : s->seqs) ids.push_back(kv.first);
  std::sort(ids.begin(), ids.end());
  std::vector<int32_t> w;
  w.reserve(9 + a->free_stack.size() + a->refcount.size() + 3 * ids.size());
  w.push_back(static_cast<int32_t>(kSnapMagic));
  w.push_back(kSnapVersion);
  w.push_back(a->num_blocks);
  w.push_back(s->block_size);
  w.push_back(s->next_id);
  w.push_back(static_cast<int32_t>(a->free_stack.size()));
  w.push_back(static_cast<int32_t>(ids.size()));
  w.insert(w.end(), a->free_stack.begin(), a->free_stack.end());
  w.insert(w.end(), a->refcount.begin(), a->refcount.end());
  for (int32_t id : ids) {
    const auto& q = s->seqs.at(id);
    w.push_back(id);
    w.push_back(q.len);
    w.push_back(static_cast<int32_t>(q.blocks.size()));
    w.insert(w.end(), q.blocks.begin(), q.blocks.end());
  }
  const uint64_t bytes = w.size() * sizeof(int32_t);
  *n_out = bytes;
  if (!buf && cap == 0) return PA_OK;   // size query
  if (cap < bytes) return pa::fail(PA_ERR_ARG, "output capacity too small");
  std::memcpy(buf, w.data(), bytes);
  return PA_OK;
}

int pa_seqs_restore(const void* buf, uint64_t n, pa_alloc** pool_out, pa_seqs** seqs_out) {
  pa::clear_error();
  if (!pool_out || !seqs_out) return pa::fail(PA_ERR_ARG, "NULL argument");
  *pool_out = nullptr;
  *seqs_out = nullptr;
  if (!buf || n % sizeof(int32_t) != 0) return pa::fail(PA_ERR_ARG, "snapshot: not a whole number of words");
  const uint64_t words = n / sizeof(int32_t);
  std::vector<int32_t> w(words);
  if (words) std::memcpy(w.data(), buf, n);
  uint64_t at = 0;
  auto take = [&](int32_t* v) {
    if (at >= words) return false;
    *v = w[at++];
    return true;
  };
  auto bad = [](const char* why) { return pa::fail(PA_ERR_ARG, std::string("snapshot: ") + why); };
  int32_t magic, version, nb, bs, next_id, n_free, n_seqs;
  if (!take(&magic) || !take(&version) || static_cast<uint32_t>(magic) != kSnapMagic || version != kSnapVersion)
    return bad("not a snapshot of this version");
  if (!take(&nb) || !take(&bs) || !take(&next_id) || !take(&n_free) || !take(&n_seqs)) return bad("truncated header");
  if (nb < 0 || bs < 1 || next_id < 0 || n_free < 0 || n_free > nb || n_seqs < 0 || n_seqs > next_id)
    return bad("header out of range");
  if (words - at < static_cast<uint64_t>(n_free) + static_cast<uint64_t>(nb)) return bad("truncated pool");
  std::vector<int32_t> free_stack(w.begin() + at, w.begin() + at + n_free);
  at += n_free;
  std::vector<int32_t> refcount(w.begin() + at, w.begin() + at + nb);
  at += nb;
  // the free pool holds each block of count 0 exactly once, and no other
  std::vector<char> in_free(nb, 0);
  for (int32_t b : free_stack) {
    if (b < 0 || b >= nb || in_free[b]) return bad("free pool entry out of range or repeated");
    in_free[b] = 1;
  }
  for (int32_t b = 0; b < nb; ++b) {
    if (refcount[b] < 0) return bad("negative count");
    if ((refcount[b] == 0) != (in_free[b] != 0)) return bad("free pool and counts disagree");
  }
  std::vector<int64_t> table_refs(nb, 0);
  std::vector<std::pair<int32_t, pa_seqs::Seq>> seqs;
  seqs.reserve(n_seqs);
  int32_t prev_id = -1;
  for (int32_t i = 0; i < n_seqs; ++i) {
    int32_t id, len, n_blocks;
    if (!take(&id) || !take(&len) || !take(&n_blocks)) return bad("truncated table");
    if (id <= prev_id || id >= next_id) return bad("sequence ids not ascending below next_id");
    if (len < 0 || n_blocks < 0 || int64_t(n_blocks) != (int64_t(len) + bs - 1) / bs)
      return bad("table length does not match the token count");
    if (words - at < static_cast<uint64_t>(n_blocks)) return bad("truncated table");
    pa_seqs::Seq q;
    q.len = len;
    q.blocks.assign(w.begin() + at, w.begin() + at + n_blocks);
    at += n_blocks;
    for (int32_t b : q.blocks) {
      if (b < 0 || b >= nb || refcount[b] < 1) return bad("table entry not a block in use");
      if (++table_refs[b] > refcount[b]) return bad("block referenced by more tables than its count");
    }
    seqs.emplace_back(id, std::move(q));
    prev_id = id;
  }
  if (at != words) return bad("trailing data");

  auto* a = new pa_alloc;
  a->num_blocks = nb;
  a->free_stack = std::move(free_stack);
  a->refcount = std::move(refcount);
  auto* s = new pa_seqs;
  s->pool = a;
  s->block_size = bs;
  s->next_id = next_id;
  for (auto& kv : seqs) s->seqs.emplace(kv.first, std::move(kv.second));
  *pool_out = a;
  *seqs_out = s;
  return PA_OK;
}

}  // extern "C"
