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
#include <algorithm>
#include <cstdint>
#include <deque>
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

}  // namespace

struct pa_bm {
  int num_blocks = 0;
  int block_size = 0;
  std::deque<int32_t> free_list;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;

  int32_t take() {
    int32_t b = free_list.front();
    free_list.pop_front();
    ref[b] = 1;
    return b;
  }
  void untake(int32_t b) {  // exact inverse of take()
    ref[b] = 0;
    free_list.push_front(b);
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
      if (free_list.empty()) return PA_ERR_NO_BLOCKS;
      int32_t b = take();
      s.table.push_back(b);
      undo->kind = 1;
      undo->new_b = b;
    } else if (ref[s.table.back()] > 1) {
      if (free_list.empty()) return PA_ERR_NO_BLOCKS;
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
  if (free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return nullptr;
      }
      seen[b] = 1;
      bm->free_list.push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
  }
  return bm;
}

void pa_bm_destroy(pa_bm *bm) { delete bm; }

int pa_bm_allocate(pa_bm *bm, int64_t seq, int num_tokens, int64_t *slots_out) {
  if (!bm || num_tokens < 0) return PA_ERR_ARG;
  if (bm->seqs.count(seq)) return PA_ERR_SEQ;
  const int64_t need = ((int64_t)num_tokens + bm->block_size - 1) / bm->block_size;
  if (need > (int64_t)bm->free_list.size()) return PA_ERR_NO_BLOCKS;
  Seq s;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(bm->take());
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
  if (num_cow_out) *num_cow_out = ncow;
  return PA_OK;
}

int pa_bm_free(pa_bm *bm, int64_t seq) {
  if (!bm) return PA_ERR_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_SEQ;
  for (int32_t b : it->second.table) {
    bm->ref[b] -= 1;
    if (bm->ref[b] == 0) bm->free_list.push_back(b);
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

int pa_bm_num_free(const pa_bm *bm) { return bm ? (int)bm->free_list.size() : PA_ERR_ARG; }

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
  out->free_blocks = (int64_t)bm->free_list.size();
  out->used_blocks = (int64_t)fill.size();
  out->shared_blocks = shared;
  out->num_seqs = (int64_t)bm->seqs.size();
  out->logical_tokens = logical;
  out->filled_slots = filled;
  out->block_size = bm->block_size;
  return PA_OK;
}

}  // extern "C"
