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
// Preemption by swapping ("Preemption and eviction", "Preemption & GPU
// Swapping"): a swapped-out sequence gives up one reference on each of its
// blocks (the caller copies them to host memory first, swap_out_blocks) and
// keeps its token count; swapping it in takes fresh blocks in table order
// (filled by swap_in_blocks). A swapped-out id is unknown to every other call
// but free and swap-in, and stays taken.
//
// The structure is a ring buffer of free block ids (the free list never holds
// more than num_blocks ids), a refcount array, a hash map from sequence id to
// (table, token count) and one from swapped-out id to token count.

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

class PrefixCache;

class Pool {
 public:
  Pool(int32_t n, int32_t bs) : n_(n), bs_(bs), ring_(n), ref_(n, 0) {}
  ~Pool();

  // Prefix caches attached to this pool (detached if the pool goes first).
  std::vector<PrefixCache*> caches;

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
    if (seqs_.count(id) || swapped_.count(id)) return PKV_ERR_EXISTS;
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
    if (seqs_.count(dst) || swapped_.count(dst)) return PKV_ERR_EXISTS;
    Seq copy = it->second;
    for (int32_t b : copy.table) ref_[b] += 1;
    seqs_.emplace(dst, std::move(copy));
    return PKV_OK;
  }

  int free_seq(int64_t id) {
    swapped_.erase(id);
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

  // Blocks of `id` in table order into out[0..n) (cap entries), then drop
  // this sequence's reference on each; the sequence becomes swapped out.
  int swap_out(int64_t id, int32_t* out, int32_t cap, int32_t* n) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    const std::vector<int32_t>& t = it->second.table;
    if (static_cast<int64_t>(t.size()) > cap || (!out && !t.empty())) return PKV_ERR_INVALID_ARG;
    for (int32_t b : t)
      if (ref_[b] <= 0) return PKV_ERR_DOUBLE_FREE;  // cannot happen through this API
    swapped_.emplace(id, it->second.tokens);  // may throw: before any change
    for (size_t i = 0; i < t.size(); ++i) {
      out[i] = t[i];
      ref_[t[i]] -= 1;
      if (ref_[t[i]] == 0) give(t[i]);
    }
    *n = static_cast<int32_t>(t.size());
    seqs_.erase(it);
    return PKV_OK;
  }

  // Fresh blocks for swapped-out `id`, in table order, into out[0..n).
  int swap_in(int64_t id, int32_t* out, int32_t cap, int32_t* n) {
    auto it = swapped_.find(id);
    if (it == swapped_.end()) return PKV_ERR_UNKNOWN_SEQ;
    const int64_t need = (it->second + bs_ - 1) / bs_;
    if (need > cap || (!out && need > 0)) return PKV_ERR_INVALID_ARG;
    if (need > count_) return PKV_ERR_OOM;
    Seq& s = seqs_[id];  // may throw: before any change
    s.table.reserve(need);  // likewise (an empty entry is removed again)
    for (int64_t i = 0; i < need; ++i) {
      s.table.push_back(take());
      out[i] = s.table.back();
    }
    s.tokens = it->second;
    *n = static_cast<int32_t>(need);
    swapped_.erase(it);
    return PKV_OK;
  }

  // Undo a table entry that swap_in created but could not fill.
  void drop_empty(int64_t id) {
    auto it = seqs_.find(id);
    if (it != seqs_.end() && it->second.table.empty() && swapped_.count(id)) seqs_.erase(it);
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
  int32_t num_blocks() const { return n_; }

  // A new sequence whose first nb table entries are the given blocks (in
  // use: one more reference each), the rest of ceil(ntok / B) fresh.
  int allocate_prefix(int64_t id, const int32_t* blocks, int32_t nb, int32_t ntok) {
    if (ntok < 0 || nb < 0 || (nb > 0 && !blocks) || static_cast<int64_t>(nb) * bs_ > ntok)
      return PKV_ERR_INVALID_ARG;
    if (seqs_.count(id) || swapped_.count(id)) return PKV_ERR_EXISTS;
    for (int32_t i = 0; i < nb; ++i)
      if (blocks[i] < 0 || blocks[i] >= n_ || ref_[blocks[i]] <= 0) return PKV_ERR_INVALID_ARG;
    const int64_t need = (static_cast<int64_t>(ntok) + bs_ - 1) / bs_;
    if (need - nb > count_) return PKV_ERR_OOM;
    Seq s;
    s.table.reserve(need);  // may throw: before any change
    auto ins = seqs_.emplace(id, Seq());
    for (int32_t i = 0; i < nb; ++i) {
      ref_[blocks[i]] += 1;
      s.table.push_back(blocks[i]);
    }
    for (int64_t i = nb; i < need; ++i) s.table.push_back(take());
    s.tokens = ntok;
    ins.first->second = std::move(s);
    return PKV_OK;
  }

  // One more / one fewer reference held by a prefix cache (release frees the
  // block when the count reaches 0).
  void retain(int32_t b) { ref_[b] += 1; }
  void release(int32_t b) {
    ref_[b] -= 1;
    if (ref_[b] == 0) give(b);
  }

  void utilisation(int64_t* table_blocks, int32_t* sequences) const {
    int64_t tb = 0;
    for (const auto& kv : seqs_) tb += static_cast<int64_t>(kv.second.table.size());
    if (table_blocks) *table_blocks = tb;
    if (sequences) *sequences = static_cast<int32_t>(seqs_.size());
  }

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
  std::unordered_map<int64_t, int64_t> swapped_;  // swapped-out id -> tokens
};

Pool* as_pool(void* h) { return static_cast<Pool*>(h); }

// Prefix cache ("RadixAttention — reuse a shared prefix"; "Shared System
// Prompts & Prefix Caching"): a radix tree whose nodes are full blocks (their
// B token ids and physical block); the cache holds one reference on each
// node's block. insert walks a sequence's full blocks and adds the missing
// ones; match returns the blocks of the longest cached run of leading full
// blocks; evict releases least-recently-used leaves that only the cache
// references (ties: the older node first). The clock advances once per
// insert or match.
class PrefixCache {
 public:
  explicit PrefixCache(Pool* a) : a_(a), bs_(a->block_size()) {
    nodes_.push_back(Node{});
    a_->caches.push_back(this);
  }
  ~PrefixCache() {
    if (!a_) return;
    for (size_t i = 1; i < nodes_.size(); ++i)
      if (nodes_[i].live) a_->release(nodes_[i].block);
    auto& v = a_->caches;
    v.erase(std::find(v.begin(), v.end(), this));
  }
  // The pool is being destroyed: nothing to release any more.
  void detach() { a_ = nullptr; }
  bool attached() const { return a_ != nullptr; }

  int insert(int64_t seq, const int32_t* tok, int32_t n, int32_t* added) {
    const Seq* s = a_->find(seq);
    if (!s) return PKV_ERR_UNKNOWN_SEQ;
    if (n < 0 || (n > 0 && !tok) || n > s->tokens) return PKV_ERR_INVALID_ARG;
    const int32_t nb = n / bs_;
    // reserve first so that nothing below can fail half-way
    nodes_.reserve(nodes_.size() + nb);
    ++clock_;
    int32_t cur = 0, add = 0;
    for (int32_t i = 0; i < nb; ++i) {
      const int32_t* key = tok + static_cast<int64_t>(i) * bs_;
      int32_t ch = find_child(cur, key);
      if (ch < 0) {
        ch = new_node(cur, key, s->table[i]);
        a_->retain(s->table[i]);
        ++add;
      }
      nodes_[ch].last = clock_;
      cur = ch;
    }
    if (added) *added = add;
    return PKV_OK;
  }

  int match(const int32_t* tok, int32_t n, int32_t* blocks, int32_t cap, int32_t* matched) {
    if (n < 0 || (n > 0 && !tok) || cap < 0 || (cap > 0 && !blocks)) return PKV_ERR_INVALID_ARG;
    ++clock_;
    int32_t cur = 0, m = 0;
    for (int32_t i = 0; i < n / bs_ && m < cap; ++i) {
      const int32_t ch = find_child(cur, tok + static_cast<int64_t>(i) * bs_);
      if (ch < 0) break;
      nodes_[ch].last = clock_;
      blocks[m++] = nodes_[ch].block;
      cur = ch;
    }
    *matched = m;
    return PKV_OK;
  }

  int evict(int32_t n, int32_t* freed, int32_t* nfreed) {
    if (n < 0 || (n > 0 && !freed)) return PKV_ERR_INVALID_ARG;
    int32_t k = 0;
    while (k < n) {
      int32_t best = -1;
      for (size_t i = 1; i < nodes_.size(); ++i) {
        const Node& x = nodes_[i];
        if (!x.live || x.nchild > 0 || a_->refcount(x.block) != 1) continue;
        if (best < 0 || x.last < nodes_[best].last ||
            (x.last == nodes_[best].last && x.born < nodes_[best].born))
          best = static_cast<int32_t>(i);
      }
      if (best < 0) break;
      Node& v = nodes_[best];
      unlink(best);
      a_->release(v.block);
      freed[k++] = v.block;
    }
    *nfreed = k;
    return PKV_OK;
  }

  int32_t live_nodes() const { return live_; }

 private:
  struct Node {
    std::vector<int32_t> key;
    int32_t block = -1, parent = -1, nchild = 0;
    int64_t last = 0, born = 0;
    bool live = false;
    std::unordered_map<uint64_t, std::vector<int32_t>> kids;  // key hash -> nodes
  };

  uint64_t hash(const int32_t* key) const {
    uint64_t h = 1469598103934665603ull;  // FNV-1a over the token ids' bytes
    for (int32_t i = 0; i < bs_; ++i) {
      uint32_t v = static_cast<uint32_t>(key[i]);
      for (int b = 0; b < 4; ++b) {
        h ^= (v >> (8 * b)) & 0xffu;
        h *= 1099511628211ull;
      }
    }
    return h;
  }

  int32_t find_child(int32_t parent, const int32_t* key) const {
    const auto& kids = nodes_[parent].kids;
    auto it = kids.find(hash(key));
    if (it == kids.end()) return -1;
    for (int32_t c : it->second)
      if (std::equal(key, key + bs_, nodes_[c].key.begin())) return c;
    return -1;
  }

  int32_t new_node(int32_t parent, const int32_t* key, int32_t block) {
    Node x;
    x.key.assign(key, key + bs_);
    x.block = block;
    x.parent = parent;
    x.born = ++born_;
    x.live = true;
    nodes_.push_back(std::move(x));
    const int32_t id = static_cast<int32_t>(nodes_.size() - 1);
    nodes_[parent].kids[hash(key)].push_back(id);
    nodes_[parent].nchild += 1;
    ++live_;
    return id;
  }

  void unlink(int32_t id) {
    Node& x = nodes_[id];
    auto& bucket = nodes_[x.parent].kids[hash(x.key.data())];
    bucket.erase(std::find(bucket.begin(), bucket.end(), id));
    if (bucket.empty()) nodes_[x.parent].kids.erase(hash(x.key.data()));
    nodes_[x.parent].nchild -= 1;
    x.live = false;
    --live_;
  }

  Pool* a_;  // null once the pool is gone
  int32_t bs_;
  std::vector<Node> nodes_;  // [0] is the root
  int64_t clock_ = 0, born_ = 0;
  int32_t live_ = 0;
};

Pool::~Pool() {
  for (PrefixCache* c : caches) c->detach();
}

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

int pkv_seq_allocate_prefix(void* handle, int64_t seq, const int32_t* blocks, int32_t num_blocks,
                            int32_t num_tokens) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  try {
    return as_pool(handle)->allocate_prefix(seq, blocks, num_blocks, num_tokens);
  } catch (const std::bad_alloc&) {
    return PKV_ERR_OOM;
  }
}

int pkv_alloc_utilisation(void* handle, int64_t* table_blocks, int32_t* sequences) {
  if (!handle) return PKV_ERR_INVALID_ARG;
  as_pool(handle)->utilisation(table_blocks, sequences);
  return PKV_OK;
}

int pkv_cache_create(void* alloc, void** cache) {
  if (!alloc || !cache) return PKV_ERR_INVALID_ARG;
  try {
    as_pool(alloc)->caches.reserve(as_pool(alloc)->caches.size() + 1);
    *cache = new PrefixCache(as_pool(alloc));
  } catch (const std::bad_alloc&) {
    return PKV_ERR_OOM;
  }
  return PKV_OK;
}

void pkv_cache_destroy(void* cache) { delete static_cast<PrefixCache*>(cache); }

int pkv_cache_insert(void* cache, int64_t seq, const int32_t* tokens, int32_t n, int32_t* added) {
  if (!cache || !static_cast<PrefixCache*>(cache)->attached()) return PKV_ERR_INVALID_ARG;
  try {
    return static_cast<PrefixCache*>(cache)->insert(seq, tokens, n, added);
  } catch (const std::bad_alloc&) {
    return PKV_ERR_OOM;
  }
}

int pkv_cache_match(void* cache, const int32_t* tokens, int32_t n, int32_t* blocks, int32_t cap,
                    int32_t* matched) {
  if (!cache || !matched || !static_cast<PrefixCache*>(cache)->attached()) return PKV_ERR_INVALID_ARG;
  return static_cast<PrefixCache*>(cache)->match(tokens, n, blocks, cap, matched);
}

int pkv_cache_evict(void* cache, int32_t n, int32_t* freed, int32_t* num_freed) {
  if (!cache || !num_freed || !static_cast<PrefixCache*>(cache)->attached()) return PKV_ERR_INVALID_ARG;
  return static_cast<PrefixCache*>(cache)->evict(n, freed, num_freed);
}

int pkv_cache_nodes(void* cache) {
  return cache ? static_cast<PrefixCache*>(cache)->live_nodes() : PKV_ERR_INVALID_ARG;
}

int pkv_seq_swap_out(void* handle, int64_t seq, int32_t* blocks, int32_t cap, int32_t* n) {
  if (!handle || !n) return PKV_ERR_INVALID_ARG;
  try {
    return as_pool(handle)->swap_out(seq, blocks, cap, n);
  } catch (const std::bad_alloc&) {
    return PKV_ERR_OOM;
  }
}

int pkv_seq_swap_in(void* handle, int64_t seq, int32_t* blocks, int32_t cap, int32_t* n) {
  if (!handle || !n) return PKV_ERR_INVALID_ARG;
  try {
    return as_pool(handle)->swap_in(seq, blocks, cap, n);
  } catch (const std::bad_alloc&) {
    as_pool(handle)->drop_empty(seq);
    return PKV_ERR_OOM;
  }
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
