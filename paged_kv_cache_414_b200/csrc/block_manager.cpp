// Host KV block manager: free list, reference counts, fork, copy-on-write.
//
// Follows "Why OS Virtual Memory Paging Saved LLM Inference: The vLLM
// Breakthrough", section 2 (physical blocks handed out one at a time as new
// tokens arrive; a block table per sequence) and section 3 (branches of
// parallel sampling or beam search share the prompt's physical blocks; the
// branch that writes gets a private block), and "Can OS paging techniques
// reduce LLM serving memory waste?", second paragraph (a KV cache manager
// tracking one block table per request; sharing within and across a batch).
//
// Policy where the pages are silent: a first-in-first-out free list
// (allocate from the front, release to the back); a write into a shared
// partial last block copies it unless the writer is the last holder.
//
// Prefix caching across requests (the same pages: blocks shared across the
// requests of a batch; block tables make KV memory reusable): a block that a
// prompt fills completely is identified by the whole token prefix up to its
// end.  Prefixes are nodes of a trie keyed by (parent node, the block's
// tokens), compared exactly, so two different prefixes can never alias.  A
// cached block whose last holder frees it keeps its node while it waits in
// the free list and leaves the cache when the free list hands it out again.
// That hand-out is applied when a call commits, so a batch of appends that
// fails part-way is rolled back exactly.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int64_t len = 0;
};

// Undo record of one append, so a batch can be rolled back exactly.
struct AppendUndo {
  int64_t seq;
  int kind;       // 0 in place, 1 new block at a boundary, 2 copy-on-write
  int32_t old_b;  // kind 2: the shared block the table pointed at
  int32_t new_b;  // kind 1, 2: the block taken from the free list
};

// A token prefix ending at a block boundary.
struct PrefixNode {
  int64_t parent = -1;          // the prefix one block shorter, -1 for the first block
  std::vector<int32_t> toks;    // the tokens of this block
  int32_t block = -1;           // the block holding this prefix's K/V, or -1
  int32_t children = 0;         // nodes whose parent this is
};

uint64_t mix64(uint64_t x) {  // splitmix64 finaliser
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

}  // namespace

struct pa_bm {
  int num_blocks = 0;
  int block_size = 0;
  // free list: doubly linked through the block ids, so a cached block can
  // leave it from the middle when a prompt reuses it
  std::vector<int32_t> nxt, prv;
  std::vector<char> is_free;
  int32_t head = -1, tail = -1;
  int64_t nfree = 0;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  // prefix cache
  std::unordered_map<int64_t, PrefixNode> nodes;
  std::unordered_map<uint64_t, std::vector<int64_t>> index;  // hash -> nodes
  std::vector<int64_t> node_of;                              // block -> node or -1
  int64_t next_node = 0;
  int64_t cached = 0;

  void push_back(int32_t b) {
    nxt[b] = -1;
    prv[b] = tail;
    if (tail >= 0) nxt[tail] = b; else head = b;
    tail = b;
    is_free[b] = 1;
    ++nfree;
  }
  void push_front(int32_t b) {
    prv[b] = -1;
    nxt[b] = head;
    if (head >= 0) prv[head] = b; else tail = b;
    head = b;
    is_free[b] = 1;
    ++nfree;
  }
  void unlink(int32_t b) {
    if (prv[b] >= 0) nxt[prv[b]] = nxt[b]; else head = nxt[b];
    if (nxt[b] >= 0) prv[nxt[b]] = prv[b]; else tail = prv[b];
    is_free[b] = 0;
    --nfree;
  }
  // Take the front block.  A cached prefix it may hold stays entered until
  // the caller commits and calls evict().
  int32_t take() {
    int32_t b = head;
    unlink(b);
    ref[b] = 1;
    return b;
  }
  void untake(int32_t b) {  // exact inverse of take()
    ref[b] = 0;
    push_front(b);
  }

  static uint64_t key_hash(int64_t parent, const int32_t *toks, int n) {
    uint64_t h = mix64((uint64_t)parent);
    for (int i = 0; i < n; ++i) h = mix64(h ^ (uint32_t)toks[i]);
    return h;
  }
  int64_t find_node(int64_t parent, const int32_t *toks) const {
    auto it = index.find(key_hash(parent, toks, block_size));
    if (it == index.end()) return -1;
    for (int64_t id : it->second) {
      const PrefixNode &nd = nodes.at(id);
      if (nd.parent == parent &&
          std::memcmp(nd.toks.data(), toks, sizeof(int32_t) * block_size) == 0)
        return id;
    }
    return -1;
  }
  int64_t get_or_create(int64_t parent, const int32_t *toks) {
    int64_t id = find_node(parent, toks);
    if (id >= 0) return id;
    id = next_node++;
    PrefixNode nd;
    nd.parent = parent;
    nd.toks.assign(toks, toks + block_size);
    nodes.emplace(id, std::move(nd));
    index[key_hash(parent, toks, block_size)].push_back(id);
    if (parent >= 0) nodes.at(parent).children += 1;
    return id;
  }
  // Drop nodes that hold no block and have no children, walking up.
  void collect(int64_t id) {
    while (id >= 0) {
      PrefixNode &nd = nodes.at(id);
      if (nd.block >= 0 || nd.children > 0) return;
      const int64_t parent = nd.parent;
      auto &bucket = index.at(key_hash(parent, nd.toks.data(), block_size));
      bucket.erase(std::find(bucket.begin(), bucket.end(), id));
      if (bucket.empty()) index.erase(key_hash(parent, nd.toks.data(), block_size));
      nodes.erase(id);
      if (parent >= 0) nodes.at(parent).children -= 1;
      id = parent;
    }
  }
  // Block b has been handed out for new content: it leaves the cache.
  void evict(int32_t b) {
    const int64_t id = node_of[b];
    if (id < 0) return;
    node_of[b] = -1;
    nodes.at(id).block = -1;
    --cached;
    collect(id);
  }
  // Enter block b under prefix node id (replacing an older block there).
  void enter(int64_t id, int32_t b) {
    PrefixNode &nd = nodes.at(id);
    if (nd.block >= 0) node_of[nd.block] = -1; else ++cached;
    nd.block = b;
    node_of[b] = id;
  }
  int64_t slot_of(const Seq &s, int64_t t) const {
    return (int64_t)s.table[t / block_size] * block_size + t % block_size;
  }

  // One append; fills undo on success.
  int append(int64_t seq, int64_t *slot, int32_t *cs, int32_t *cd, AppendUndo *undo) {
    auto it = seqs.find(seq);
    if (it == seqs.end()) return PA_ERR_SEQ;
    Seq &s = it->second;
    const int64_t t = s.len;
    int cow = 0;
    undo->seq = seq;
    undo->kind = 0;
    if (t % block_size == 0) {
      if (nfree == 0) return PA_ERR_NO_BLOCKS;
      int32_t b = take();
      s.table.push_back(b);
      undo->kind = 1;
      undo->new_b = b;
    } else if (ref[s.table.back()] > 1) {
      if (nfree == 0) return PA_ERR_NO_BLOCKS;
      int32_t old_b = s.table.back();
      int32_t new_b = take();
      ref[old_b] -= 1;
      s.table.back() = new_b;
      *cs = old_b;
      *cd = new_b;
      cow = 1;
      undo->kind = 2;
      undo->old_b = old_b;
      undo->new_b = new_b;
    }
    s.len = t + 1;
    *slot = slot_of(s, t);
    return cow;
  }

  void undo_append(const AppendUndo &u) {
    Seq &s = seqs.at(u.seq);
    s.len -= 1;
    if (u.kind == 1) {
      s.table.pop_back();
      untake(u.new_b);
    } else if (u.kind == 2) {
      s.table.back() = u.old_b;
      ref[u.old_b] += 1;
      untake(u.new_b);
    }
  }
};

extern "C" {

pa_bm *pa_bm_create(int num_blocks, int block_size, const int32_t *free_order) {
  if (num_blocks < 0 || block_size <= 0) return nullptr;
  pa_bm *bm = new (std::nothrow) pa_bm();
  if (!bm) return nullptr;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  bm->nxt.assign(num_blocks, -1);
  bm->prv.assign(num_blocks, -1);
  bm->is_free.assign(num_blocks, 0);
  bm->node_of.assign(num_blocks, -1);
  if (free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return nullptr;
      }
      seen[b] = 1;
      bm->push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->push_back(i);
  }
  return bm;
}

void pa_bm_destroy(pa_bm *bm) { delete bm; }

int pa_bm_allocate(pa_bm *bm, int64_t seq, int num_tokens, int64_t *slots_out) {
  if (!bm || num_tokens < 0) return PA_ERR_ARG;
  if (bm->seqs.count(seq)) return PA_ERR_SEQ;
  const int64_t need = ((int64_t)num_tokens + bm->block_size - 1) / bm->block_size;
  if (need > bm->nfree) return PA_ERR_NO_BLOCKS;
  Seq s;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(bm->take());
  for (int32_t b : s.table) bm->evict(b);
  s.len = num_tokens;
  if (slots_out)
    for (int64_t t = 0; t < num_tokens; ++t) slots_out[t] = bm->slot_of(s, t);
  bm->seqs.emplace(seq, std::move(s));
  return PA_OK;
}

int pa_bm_fork(pa_bm *bm, int64_t parent, int64_t child) {
  if (!bm) return PA_ERR_ARG;
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end() || bm->seqs.count(child)) return PA_ERR_SEQ;
  Seq c = it->second;
  for (int32_t b : c.table) bm->ref[b] += 1;
  bm->seqs.emplace(child, std::move(c));
  return PA_OK;
}

int pa_bm_append_slot(pa_bm *bm, int64_t seq, int64_t *slot_out, int32_t *cow_src,
                      int32_t *cow_dst) {
  if (!bm || !slot_out) return PA_ERR_ARG;
  int32_t cs = -1, cd = -1;
  AppendUndo u;
  int r = bm->append(seq, slot_out, &cs, &cd, &u);
  if (r >= 0 && u.kind != 0) bm->evict(u.new_b);
  if (r == 1) {
    if (cow_src) *cow_src = cs;
    if (cow_dst) *cow_dst = cd;
  }
  return r;
}

int pa_bm_append_slots(pa_bm *bm, const int64_t *seqs, int n, int64_t *slots_out,
                       int64_t *cow_pairs_out, int *num_cow_out) {
  if (!bm || n < 0 || (n > 0 && (!seqs || !slots_out))) return PA_ERR_ARG;
  std::vector<AppendUndo> log;
  log.reserve(n);
  int ncow = 0;
  for (int i = 0; i < n; ++i) {
    int32_t cs, cd;
    AppendUndo u;
    int r = bm->append(seqs[i], &slots_out[i], &cs, &cd, &u);
    if (r < 0) {
      for (auto it = log.rbegin(); it != log.rend(); ++it) bm->undo_append(*it);
      return r;
    }
    log.push_back(u);
    if (r == 1) {
      if (cow_pairs_out) {
        cow_pairs_out[2 * ncow] = cs;
        cow_pairs_out[2 * ncow + 1] = cd;
      }
      ++ncow;
    }
  }
  for (const AppendUndo &u : log)
    if (u.kind != 0) bm->evict(u.new_b);
  if (num_cow_out) *num_cow_out = ncow;
  return PA_OK;
}

int pa_bm_allocate_prefix(pa_bm *bm, int64_t seq, const int32_t *tokens, int num_tokens,
                          int64_t *slots_out, int *num_cached_out) {
  if (!bm || num_tokens < 0 || (num_tokens > 0 && !tokens)) return PA_ERR_ARG;
  if (bm->seqs.count(seq)) return PA_ERR_SEQ;
  const int B = bm->block_size;
  const int64_t need = ((int64_t)num_tokens + B - 1) / B;
  const int64_t full = num_tokens / B;
  // longest run of cached full blocks, prefix by prefix
  std::vector<int32_t> hits;
  int64_t parent = -1, revived = 0;
  for (int64_t j = 0; j < full; ++j) {
    const int64_t id = bm->find_node(parent, tokens + j * B);
    if (id < 0 || bm->nodes.at(id).block < 0) break;
    const int32_t b = bm->nodes.at(id).block;
    hits.push_back(b);
    if (bm->ref[b] == 0) ++revived;
    parent = id;
  }
  const int64_t fresh = need - (int64_t)hits.size();
  if (fresh > bm->nfree - revived) return PA_ERR_NO_BLOCKS;
  Seq s;
  s.table.reserve(need);
  for (int32_t b : hits) {
    if (bm->ref[b] == 0) bm->unlink(b);
    bm->ref[b] += 1;
    s.table.push_back(b);
  }
  for (int64_t i = 0; i < fresh; ++i) s.table.push_back(bm->take());
  for (size_t j = hits.size(); j < s.table.size(); ++j) bm->evict(s.table[j]);
  // enter the new full blocks under their prefixes
  for (int64_t j = (int64_t)hits.size(); j < full; ++j) {
    const int64_t id = bm->get_or_create(parent, tokens + j * B);
    bm->enter(id, s.table[j]);
    parent = id;
  }
  s.len = num_tokens;
  const int64_t ncached = (int64_t)hits.size() * B;
  if (slots_out)
    for (int64_t t = 0; t < num_tokens; ++t) slots_out[t] = t < ncached ? -1 : bm->slot_of(s, t);
  if (num_cached_out) *num_cached_out = (int)ncached;
  bm->seqs.emplace(seq, std::move(s));
  return PA_OK;
}

int pa_bm_num_cached(const pa_bm *bm) { return bm ? (int)bm->cached : PA_ERR_ARG; }

int pa_bm_free(pa_bm *bm, int64_t seq) {
  if (!bm) return PA_ERR_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_SEQ;
  for (int32_t b : it->second.table) {
    bm->ref[b] -= 1;
    if (bm->ref[b] == 0) bm->push_back(b);
  }
  bm->seqs.erase(it);
  return PA_OK;
}

int pa_bm_block_table(const pa_bm *bm, int64_t seq, int32_t *out, int cap, int *n_out) {
  if (!bm) return PA_ERR_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_SEQ;
  const auto &t = it->second.table;
  if (n_out) *n_out = (int)t.size();
  if ((int)t.size() > cap || (!out && !t.empty())) return PA_ERR_ARG;
  std::copy(t.begin(), t.end(), out);
  return PA_OK;
}

int pa_bm_block_tables(const pa_bm *bm, const int64_t *seqs, int n, int32_t *out, int cap,
                       int32_t *lens_out) {
  if (!bm || n < 0 || cap < 0 || (n > 0 && (!seqs || (!out && cap > 0)))) return PA_ERR_ARG;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PA_ERR_SEQ;
    if ((int)it->second.table.size() > cap) return PA_ERR_ARG;
  }
  for (int i = 0; i < n; ++i) {
    const Seq &s = bm->seqs.find(seqs[i])->second;
    int32_t *row = out + (int64_t)i * cap;
    std::copy(s.table.begin(), s.table.end(), row);
    std::fill(row + s.table.size(), row + cap, -1);
    if (lens_out) lens_out[i] = (int32_t)s.len;
  }
  return PA_OK;
}

int pa_bm_seq_len(const pa_bm *bm, int64_t seq) {
  if (!bm) return PA_ERR_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_SEQ;
  return (int)it->second.len;
}

int pa_bm_num_free(const pa_bm *bm) { return bm ? (int)bm->nfree : PA_ERR_ARG; }

int pa_bm_ref_count(const pa_bm *bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return PA_ERR_ARG;
  return bm->ref[block];
}

int pa_bm_num_seqs(const pa_bm *bm) { return bm ? (int)bm->seqs.size() : PA_ERR_ARG; }

int pa_bm_stats(const pa_bm *bm, pa_bm_stats_t *out) {
  if (!bm || !out) return PA_ERR_ARG;
  // filled slots of each block in use: the largest fill any holder gives it
  std::unordered_map<int32_t, int> fill;
  int64_t logical = 0;
  for (const auto &kv : bm->seqs) {
    const Seq &s = kv.second;
    logical += s.len;
    for (size_t j = 0; j < s.table.size(); ++j) {
      const int64_t n = std::min<int64_t>(bm->block_size, s.len - (int64_t)j * bm->block_size);
      int &f = fill[s.table[j]];
      f = std::max<int>(f, (int)n);
    }
  }
  int64_t filled = 0, shared = 0;
  for (const auto &kv : fill) {
    filled += kv.second;
    if (bm->ref[kv.first] > 1) ++shared;
  }
  out->num_blocks = bm->num_blocks;
  out->free_blocks = bm->nfree;
  out->used_blocks = (int64_t)fill.size();
  out->shared_blocks = shared;
  out->num_seqs = (int64_t)bm->seqs.size();
  out->logical_tokens = logical;
  out->filled_slots = filled;
  out->block_size = bm->block_size;
  return PA_OK;
}

}  // extern "C"
