// Host block allocator behind the pkv_alloc_* / pkv_seq_* calls of pagedkv.h.
//
// Semantics of "Hands-On Implementation: Building a PagedAttention Block
// Allocator in Python" and "How Block Paging Operates During Generation"
// ("PagedAttention and KV Cache Management"): a FIFO free list (take from the
// head, return to the tail), reference counts per block, ceil(n / B) blocks
// per n-token sequence, zero-copy fork, copy-on-write of a shared block that
// a sequence is about to write into. Every call validates first and then
// mutates, so a failing call changes nothing.
//
// The structure is a ring buffer of free block ids (the free list never holds
// more than num_blocks ids), a refcount array and a hash map from sequence id
// to (table, token count).

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pagedkv.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int64_t tokens = 0;
};

class Pool {
 public:
  Pool(int32_t n, int32_t bs) : n_(n), bs_(bs), ring_(n), ref_(n, 0) {}

  int init_order(const int32_t* order) {
    std::vector<char> seen(n_, 0);
    for (int32_t i = 0; i < n_; ++i) {
      int32_t b = order ? order[i] : i;
      if (b < 0 || b >= n_ || seen[b]) return PKV_ERR_INVALID_ARG;
      seen[b] = 1;
      ring_[i] = b;
    }
    head_ = 0;
    count_ = n_;
    return PKV_OK;
  }

  int allocate(int64_t id, int32_t ntok) {
    if (ntok < 0) return PKV_ERR_INVALID_ARG;
    if (seqs_.count(id)) return PKV_ERR_EXISTS;
    int64_t need = (static_cast<int64_t>(ntok) + bs_ - 1) / bs_;
    if (need > count_) return PKV_ERR_OOM;
    Seq s;
    s.table.reserve(need);
    for (int64_t i = 0; i < need; ++i) s.table.push_back(take());
    s.tokens = ntok;
    seqs_.emplace(id, std::move(s));
    return PKV_OK;
  }

  int append_slot(int64_t id, int64_t* slot, int32_t* cow_src, int32_t* cow_dst) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    Seq& s = it->second;
    int64_t room = static_cast<int64_t>(s.table.size()) * bs_ - s.tokens;
    int32_t src = -1, dst = -1, blk;
    int64_t offset;
    if (room == 0) {  // boundary: the token starts a new block
      if (count_ < 1) return PKV_ERR_OOM;
      blk = take();
      s.table.push_back(blk);
      offset = 0;
    } else {
      blk = s.table.back();
      offset = bs_ - room;
      if (ref_[blk] > 1) {  // the slot lies in a shared block: copy it first
        if (count_ < 1) return PKV_ERR_OOM;
        int32_t fresh = take();
        ref_[blk] -= 1;
        s.table.back() = fresh;
        src = blk;
        dst = fresh;
        blk = fresh;
      }
    }
    s.tokens += 1;
    if (slot) *slot = static_cast<int64_t>(blk) * bs_ + offset;
    if (cow_src) *cow_src = src;
    if (cow_dst) *cow_dst = dst;
    return PKV_OK;
  }

  int fork(int64_t src, int64_t dst) {
    auto it = seqs_.find(src);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    if (seqs_.count(dst)) return PKV_ERR_EXISTS;
    Seq copy = it->second;
    for (int32_t b : copy.table) ref_[b] += 1;
    seqs_.emplace(dst, std::move(copy));
    return PKV_OK;
  }

  int free_seq(int64_t id) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PKV_OK;
    for (int32_t b : it->second.table)
      if (ref_[b] <= 0) return PKV_ERR_DOUBLE_FREE;  // cannot happen through this API
    for (int32_t b : it->second.table) {
      ref_[b] -= 1;
      if (ref_[b] == 0) give(b);
    }
    seqs_.erase(it);
    return PKV_OK;
  }

  int64_t num_tokens(int64_t id) const {
    auto it = seqs_.find(id);
    return it == seqs_.end() ? PKV_ERR_UNKNOWN_SEQ : it->second.tokens;
  }

  const Seq* find(int64_t id) const {
    auto it = seqs_.find(id);
    return it == seqs_.end() ? nullptr : &it->second;
  }

  void stats(int32_t* fr, int32_t* used, int32_t* shared, int64_t* tokens) const {
    int32_t u = 0, sh = 0;
    for (int32_t r : ref_) {
      u += r > 0;
      sh += r > 1;
    }
    if (fr) *fr = count_;
    if (used) *used = u;
    if (shared) *shared = sh;
    if (tokens) {
      // each physical slot once: a block's fill is the largest fill any
      // sequence referencing it sees
      std::vector<int32_t> fill(n_, 0);
      for (const auto& kv : seqs_) {
        const Seq& s = kv.second;
        for (size_t i = 0; i < s.table.size(); ++i) {
          int64_t f = s.tokens - static_cast<int64_t>(i) * bs_;
          f = f < 0 ? 0 : (f > bs_ ? bs_ : f);
          if (f > fill[s.table[i]]) fill[s.table[i]] = static_cast<int32_t>(f);
        }
      }
      int64_t t = 0;
      for (int32_t f : fill) t += f;
      *tokens = t;
    }
  }

  int refcount(int32_t b) const { return (b < 0 || b >= n_) ? PKV_ERR_INVALID_ARG : ref_[b]; }
  int32_t block_size() const { return bs_; }

 private:
  int32_t take() {
    int32_t b = ring_[head_];
    head_ = (head_ + 1) % n_;
    count_ -= 1;
    ref_[b] = 1;
    return b;
  }
  void give(int32_t b) {
    ring_[(head_ + count_) % n_] = b;
    count_ += 1;
  }

  int32_t n_, bs_;
  std::vector<int32_t> ring_;  // free list, FIFO, head_ .. head_+count_-1 (mod n_)
  int32_t head_ = 0, count_ = 0;
  std::vector<int32_t> ref_;
  std::unordered_map<int64_t, Seq> seqs_;
};

Pool* as_pool(void* h) { return static_cast<Pool*>(h); }

}  // namespace

extern "C" {

int pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                     void** handle) {
  if (!handle || num_blocks <= 0 || block_size <= 0) return PKV_ERR_INVALID_ARG;
  *handle = nullptr;
  Pool* p = new (std::nothrow) Pool(num_blocks, block_size);
  if (!p) return PKV_ERR_OOM;
  int st = p->init_order(initial_free_order);
  if (st != PKV_OK) {
    delete p;
    return st;
  }
  *handle = p;
  return PKV_OK;
}

void pkv_alloc_destroy(void* handle) { delete as_pool(handle); }

int pkv_seq_allocate(void* handle, int64_t seq, int32_t num_tokens) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  return as_pool(handle)->allocate(seq, num_tokens);
}

int pkv_seq_append_slot(void* handle, int64_t seq, int64_t* slot, int32_t* cow_src,
                        int32_t* cow_dst) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  return as_pool(handle)->append_slot(seq, slot, cow_src, cow_dst);
}

int pkv_seq_fork(void* handle, int64_t src, int64_t dst) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  return as_pool(handle)->fork(src, dst);
}

int pkv_seq_free(void* handle, int64_t seq) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  return as_pool(handle)->free_seq(seq);
}

int64_t pkv_seq_num_tokens(void* handle, int64_t seq) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  return as_pool(handle)->num_tokens(seq);
}

int pkv_seq_block_table(void* handle, int64_t seq, int32_t* table, int32_t cap) {
  if (!handle || cap < 0 || (cap > 0 && !table)) return PKV_ERR_INVALID_ARG;
  const Seq* s = as_pool(handle)->find(seq);
  if (!s) return PKV_ERR_UNKNOWN_SEQ;
  int32_t n = static_cast<int32_t>(s->table.size());
  int32_t m = n < cap ? n : cap;
  if (m > 0) std::memcpy(table, s->table.data(), sizeof(int32_t) * m);
  return n;
}

int pkv_build_block_tables(void* handle, const int64_t* seqs, int32_t n, int32_t* table,
                           int32_t max_blocks, int32_t* lens) {
  if (!handle || n < 0 || max_blocks < 0 || (n > 0 && (!seqs || !table || !lens)))
    return PKV_ERR_INVALID_ARG;
  Pool* p = as_pool(handle);
  for (int32_t i = 0; i < n; ++i) {  // validate everything before writing
    const Seq* s = p->find(seqs[i]);
    if (!s) return PKV_ERR_UNKNOWN_SEQ;
    if (static_cast<int64_t>(s->table.size()) > max_blocks) return PKV_ERR_INVALID_ARG;
    if (s->tokens > INT32_MAX) return PKV_ERR_INVALID_ARG;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq* s = p->find(seqs[i]);
    int32_t* row = table + static_cast<int64_t>(i) * max_blocks;
    int32_t k = static_cast<int32_t>(s->table.size());
    if (k > 0) std::memcpy(row, s->table.data(), sizeof(int32_t) * k);
    for (int32_t j = k; j < max_blocks; ++j) row[j] = -1;
    lens[i] = static_cast<int32_t>(s->tokens);
  }
  return PKV_OK;
}

int pkv_alloc_stats(void* handle, int32_t* free_blocks, int32_t* used_blocks,
                    int32_t* shared_blocks, int64_t* tokens) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  as_pool(handle)->stats(free_blocks, used_blocks, shared_blocks, tokens);
  return PKV_OK;
}

int pkv_block_refcount(void* handle, int32_t block) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  return as_pool(handle)->refcount(block);
}

// Shared-prefix groups of a decode batch (prefix sharing: "PagedAttention:
// treat the cache like virtual memory", "Shared System Prompts & Prefix
// Caching"): rows whose first block is full are bucketed by that block id in
// order of first appearance; a bucket of at least min_members rows is a group
// whose prefix is the longest run of leading columns holding the same block,
// full, in every member.
int pkv_prefix_groups(const int32_t* tables, int32_t S, int32_t width, const int32_t* lens,
                      int32_t block_size, int32_t min_members, int32_t* group_start,
                      int32_t* members, int32_t* prefix_blocks, int32_t* num_groups,
                      int32_t* num_members) {
  if (S < 0 || width < 1 || block_size < 1 || min_members < 1 || !group_start || !members ||
      !prefix_blocks || !num_groups || !num_members || (S > 0 && (!tables || !lens)))
    return PKV_ERR_INVALID_ARG;
  try {
    std::unordered_map<int32_t, int32_t> bucket_of;  // first block -> bucket
    std::vector<std::vector<int32_t>> buckets;
    for (int32_t r = 0; r < S; ++r) {
      prefix_blocks[r] = 0;
      if (lens[r] < block_size) continue;
      const int32_t key = tables[static_cast<int64_t>(r) * width];
      auto it = bucket_of.find(key);
      if (it == bucket_of.end()) {
        bucket_of.emplace(key, static_cast<int32_t>(buckets.size()));
        buckets.emplace_back(1, r);
      } else {
        buckets[it->second].push_back(r);
      }
    }
    int32_t g = 0, m = 0;
    group_start[0] = 0;
    for (const auto& rows : buckets) {
      if (static_cast<int32_t>(rows.size()) < min_members) continue;
      int32_t min_len = lens[rows[0]];
      for (int32_t r : rows) min_len = lens[r] < min_len ? lens[r] : min_len;
      const int32_t lim = std::min<int64_t>(width, min_len / block_size);  // columns full in all
      const int32_t* first = tables + static_cast<int64_t>(rows[0]) * width;
      int32_t n = 0;
      for (; n < lim; ++n) {
        bool same = true;
        for (int32_t r : rows)
          if (tables[static_cast<int64_t>(r) * width + n] != first[n]) {
            same = false;
            break;
          }
        if (!same) break;
      }
      for (int32_t r : rows) {
        members[m++] = r;
        prefix_blocks[r] = n;
      }
      group_start[++g] = m;
    }
    *num_groups = g;
    *num_members = m;
  } catch (const std::bad_alloc&) {
    return PKV_ERR_OOM;
  }
  return PKV_OK;
}

}  // extern "C"
