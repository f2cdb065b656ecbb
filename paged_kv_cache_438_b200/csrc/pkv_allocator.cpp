// Host-side paged KV block manager (CPU only, no device memory).
//
// "大模型推理的KV Cache管理从内存碎片到前缀缓存的优化实战" (wmrh.cn), §二:
//   * BlockTable: free list initialised to 0..n-1, allocate() pops its end and
//     reports failure when empty, free() pushes a block back;
//   * PagedKVCache.append_slot: token `pos` belongs to logical block pos / 16,
//     a physical block is taken when that logical block is not mapped yet;
//   * copy_prefix: a child maps its first ceil(prefix / 16) logical blocks to
//     the parent's physical blocks and their reference counts go up by one.
// Copy-on-write (ascendai.csdn.net article §二 写时复制; "LLM 推理优化深度解析"
// §意外的收获：prefix sharing): a shared block stays shared until a token is
// written into it; the writer then takes a fresh block, reports (old, new)
// for a block copy and the old count drops.  A fresh block starts at count 1;
// the last holder (count 1) writes in place.
//
// Every mutating call is transactional: an undo log restores the exact prior
// state (free-list order included) when a block allocation fails.
//
// Automatic prefix caching (same page, §三 AutomaticPrefixCache and
// PrefixRadixTree): the longest cached prefix of a request's token ids is
// found in a radix tree and rounded down to whole blocks; the key is a
// 16-byte BLAKE2b digest of the token ids as little-endian int32; least
// recently used entries are evicted.  Here every full block of a cached
// sequence is one tree node (its edge: that block's 16 token ids), since the
// KV of a sequence covers all of its prefixes.  The cache holds a reference
// on each cached block; only blocks no sequence holds, with no cached block
// below them, can be evicted (least recently used first, by a logical clock
// that ticks once per cache call, ties to the older node).  An allocation
// that finds the free list empty evicts one such block.
#include <algorithm>
#include <array>
#include <cstdint>
#include <cstring>
#include <new>
#include <set>
#include <tuple>
#include <unordered_map>
#include <vector>

#include "pkv_blake2b.h"
#include "pkv_error.h"

namespace pkv {

char* error_buffer() {
  static thread_local char buf[512];
  return buf;
}

namespace {

struct Sequence {
  std::vector<int32_t> table;
  int64_t len = 0;
};

using Chunk = std::array<int32_t, 16>;

struct ChildKey {
  int parent;
  Chunk chunk;
  bool operator==(const ChildKey& o) const { return parent == o.parent && chunk == o.chunk; }
};

struct ChildKeyHash {
  size_t operator()(const ChildKey& k) const {
    uint64_t h = 1469598103934665603ull ^ static_cast<uint64_t>(k.parent);
    for (int32_t t : k.chunk) h = (h ^ static_cast<uint32_t>(t)) * 1099511628211ull;
    return static_cast<size_t>(h);
  }
};

// One cached block of the prefix tree (node 0 is the root, which has none).
struct Node {
  int parent = -1;
  Chunk chunk{};
  int32_t block = -1;
  uint8_t key[16] = {};
  int64_t last = 0;   // logical time of the last use
  int64_t order = 0;  // creation order (LRU tie-break)
  int children = 0;
  bool alive = false;
};

class BlockManager {
 public:
  BlockManager(int num_blocks, int block_size, const int32_t* order)
      : block_size_(block_size), rc_(num_blocks, 0) {
    free_.reserve(num_blocks);
    if (order) {
      free_.assign(order, order + num_blocks);
    } else {
      for (int b = 0; b < num_blocks; ++b) free_.push_back(b);
    }
    nodes_.emplace_back();  // root
    nodes_[0].alive = true;
  }

  // ---- prefix cache --------------------------------------------------------
  // Nodes of the longest cached whole-block prefix of tokens[0, n).
  void walk(const int32_t* tokens, int n, std::vector<int>* path) const {
    path->clear();
    int cur = 0;
    for (int i = 0; i + 16 <= n; i += 16) {
      ChildKey k{cur, {}};
      std::copy(tokens + i, tokens + i + 16, k.chunk.begin());
      auto it = children_.find(k);
      if (it == children_.end()) break;
      cur = it->second;
      path->push_back(cur);
    }
  }

  void touch(int id) {
    Node& nd = nodes_[id];
    lru_.erase(std::make_tuple(nd.last, nd.order, id));
    nd.last = clock_;
    lru_.insert(std::make_tuple(nd.last, nd.order, id));
  }

  int match(const int32_t* tokens, int n, int* hit, uint8_t* key) {
    ++clock_;
    walk(tokens, n, &path_);
    for (int id : path_) touch(id);
    ++lookups_;
    if (!path_.empty()) ++hits_;
    if (hit) *hit = static_cast<int>(path_.size()) * block_size_;
    if (key) {
      if (path_.empty()) std::memset(key, 0, 16);
      else std::memcpy(key, nodes_[path_.back()].key, 16);
    }
    return ok();
  }

  int add_cached(int64_t id, const int32_t* tokens, int n, int* hit_out) {
    if (seqs_.count(id)) return fail(PKV_ERR_EXISTS, "sequence %lld already exists", (long long)id);
    int hit = 0;
    match(tokens, n, &hit, nullptr);
    Sequence s;
    for (int nd : path_) {
      s.table.push_back(nodes_[nd].block);
      ++rc_[nodes_[nd].block];
    }
    s.len = hit;
    seqs_.emplace(id, std::move(s));
    if (hit_out) *hit_out = hit;
    return ok();
  }

  int insert(int64_t id, const int32_t* tokens, int n, int* newly) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return fail(PKV_ERR_NOT_FOUND, "sequence %lld not found", (long long)id);
    const Sequence& s = it->second;
    const int nblk = static_cast<int>(std::min<int64_t>(n, s.len) / block_size_);
    ++clock_;
    Blake2b128 st;
    int cur = 0, added = 0;
    for (int i = 0; i < nblk; ++i) {
      const int32_t* c = tokens + static_cast<size_t>(i) * 16;
      blake2b_tokens(&st, c, 16);
      ChildKey k{cur, {}};
      std::copy(c, c + 16, k.chunk.begin());
      auto f = children_.find(k);
      if (f != children_.end()) {
        cur = f->second;
        touch(cur);
        continue;
      }
      const int nid = new_node();
      Node& nd = nodes_[nid];
      nd.parent = cur;
      nd.chunk = k.chunk;
      nd.block = s.table[static_cast<size_t>(i)];
      st.digest(nd.key);
      nd.last = clock_;
      nd.order = next_order_++;
      nd.children = 0;
      nd.alive = true;
      children_.emplace(k, nid);
      ++nodes_[cur].children;
      lru_.insert(std::make_tuple(nd.last, nd.order, nid));
      ++rc_[nd.block];
      ++cached_;
      ++added;
      cur = nid;
    }
    if (newly) *newly = added;
    return ok();
  }

  int evict_to(int max_cached, int* evicted) {
    int k = 0;
    while (cached_ > max_cached && evict_one(false)) ++k;
    if (evicted) *evicted = k;
    return ok();
  }

  void cache_stats(int* cached, int* evictable, int64_t* lookups, int64_t* hits, int64_t* evictions) const {
    int ev = 0;
    for (size_t i = 1; i < nodes_.size(); ++i) {
      const Node& nd = nodes_[i];
      if (nd.alive && nd.children == 0 && rc_[nd.block] == 1) ++ev;
    }
    if (cached) *cached = cached_;
    if (evictable) *evictable = ev;
    if (lookups) *lookups = lookups_;
    if (hits) *hits = hits_;
    if (evictions) *evictions = evictions_;
  }

  int num_blocks() const { return static_cast<int>(rc_.size()); }

  int add(int64_t id) {
    if (seqs_.count(id)) return fail(PKV_ERR_EXISTS, "sequence %lld already exists", (long long)id);
    seqs_.emplace(id, Sequence{});
    return ok();
  }

  int fork(int64_t parent, int64_t child, int prefix_len) {
    auto it = seqs_.find(parent);
    if (it == seqs_.end()) return fail(PKV_ERR_NOT_FOUND, "parent %lld not found", (long long)parent);
    if (seqs_.count(child)) return fail(PKV_ERR_EXISTS, "child %lld already exists", (long long)child);
    const Sequence& p = it->second;
    int64_t plen = prefix_len < 0 ? p.len : prefix_len;
    if (plen > p.len) return fail(PKV_ERR_INVALID_ARG, "prefix_len %d exceeds parent length %lld", prefix_len, (long long)p.len);
    size_t nb = static_cast<size_t>((plen + block_size_ - 1) / block_size_);
    Sequence c;
    c.table.assign(p.table.begin(), p.table.begin() + nb);
    c.len = plen;
    for (int32_t b : c.table) ++rc_[b];
    seqs_.emplace(child, std::move(c));
    return ok();
  }

  // Appends n tokens to each listed sequence in order.  Writes slots (one per
  // token, sequence-major) and CoW pairs.  On failure restores everything.
  int append(const int64_t* ids, int n_seqs, int n_tokens, int64_t* slots, int32_t* pairs,
             int cow_cap, int* n_pairs) {
    for (int i = 0; i < n_seqs; ++i)
      if (!seqs_.count(ids[i])) return fail(PKV_ERR_NOT_FOUND, "sequence %lld not found", (long long)ids[i]);
    undo_.clear();
    int np = 0;
    size_t k = 0;
    for (int i = 0; i < n_seqs; ++i) {
      Sequence& s = seqs_[ids[i]];
      for (int t = 0; t < n_tokens; ++t) {
        const int64_t pos = s.len;
        const size_t lb = static_cast<size_t>(pos / block_size_);
        if (pos % block_size_ == 0) {
          int32_t b;
          if (!pop(&b)) return rollback(PKV_ERR_NO_BLOCKS, "out of free blocks");
          undo_.push_back({Op::kPush, ids[i], b, 0});
          s.table.push_back(b);
        } else {
          const int32_t old = s.table[lb];
          if (rc_[old] > 1) {
            if (np >= cow_cap) return rollback(PKV_ERR_INVALID_ARG, "cow_pairs_out capacity %d exceeded", cow_cap);
            int32_t b;
            if (!pop(&b)) return rollback(PKV_ERR_NO_BLOCKS, "out of free blocks");
            --rc_[old];
            undo_.push_back({Op::kCow, ids[i], b, old, static_cast<int64_t>(lb)});
            s.table[lb] = b;
            pairs[2 * np] = old;
            pairs[2 * np + 1] = b;
            ++np;
          }
        }
        undo_.push_back({Op::kLen, ids[i], 0, 0, pos});
        s.len = pos + 1;
        slots[k++] = static_cast<int64_t>(s.table[lb]) * block_size_ + pos % block_size_;
      }
    }
    if (n_pairs) *n_pairs = np;
    for (const Undo& u : undo_)  // committed: evicted nodes' slots can be reused
      if (u.op == Op::kEvict) dead_.push_back(static_cast<int>(u.aux));
    undo_.clear();
    return ok();
  }

  int release(int64_t id) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return fail(PKV_ERR_NOT_FOUND, "sequence %lld not found", (long long)id);
    for (int32_t b : it->second.table) {
      if (--rc_[b] == 0) free_.push_back(b);
    }
    seqs_.erase(it);
    return ok();
  }

  const Sequence* find(int64_t id) const {
    auto it = seqs_.find(id);
    return it == seqs_.end() ? nullptr : &it->second;
  }

  int refcount(int32_t b) const { return rc_[b]; }

  void stats(int* nfree, int* nshared, int* run) const {
    std::vector<char> is_free(rc_.size(), 0);
    for (int32_t b : free_) is_free[b] = 1;
    int best = 0, cur = 0, shared = 0;
    for (size_t b = 0; b < rc_.size(); ++b) {
      cur = is_free[b] ? cur + 1 : 0;
      best = std::max(best, cur);
      if (rc_[b] > 1) ++shared;
    }
    if (nfree) *nfree = static_cast<int>(free_.size());
    if (nshared) *nshared = shared;
    if (run) *run = best;
  }

 private:
  enum class Op { kPush, kCow, kLen, kEvict };
  struct Undo {
    Op op;
    int64_t seq;
    int32_t block;   // block taken from the free list
    int32_t old;     // kCow: the shared block that was replaced
    int64_t aux = 0; // kCow: logical index; kLen: previous length; kEvict: node id
  };

  int new_node() {
    if (!dead_.empty()) {
      const int id = dead_.back();
      dead_.pop_back();
      return id;
    }
    nodes_.emplace_back();
    return static_cast<int>(nodes_.size()) - 1;
  }

  // Evicts the least recently used cached block that no sequence holds and
  // that has no cached child; its block returns to the free list.
  bool evict_one(bool log) {
    for (auto it = lru_.begin(); it != lru_.end(); ++it) {
      const int id = std::get<2>(*it);
      Node& nd = nodes_[id];
      if (nd.children != 0 || rc_[nd.block] != 1) continue;
      lru_.erase(it);
      children_.erase(ChildKey{nd.parent, nd.chunk});
      --nodes_[nd.parent].children;
      nd.alive = false;
      rc_[nd.block] = 0;
      free_.push_back(nd.block);
      --cached_;
      ++evictions_;
      if (log) {
        undo_.push_back({Op::kEvict, 0, nd.block, 0, id});
      } else {
        dead_.push_back(id);
      }
      return true;
    }
    return false;
  }

  bool pop(int32_t* b) {
    if (free_.empty() && !evict_one(true)) return false;
    *b = free_.back();
    free_.pop_back();
    rc_[*b] = 1;
    return true;
  }

  int rollback(int code, const char* fmt, ...) {
    for (auto it = undo_.rbegin(); it != undo_.rend(); ++it) {
      if (it->op == Op::kEvict) {
        // the evicted block went to the back of the free list; take it back
        const int id = static_cast<int>(it->aux);
        Node& nd = nodes_[id];
        free_.pop_back();
        rc_[nd.block] = 1;
        nd.alive = true;
        children_.emplace(ChildKey{nd.parent, nd.chunk}, id);
        ++nodes_[nd.parent].children;
        lru_.insert(std::make_tuple(nd.last, nd.order, id));
        ++cached_;
        --evictions_;
        continue;
      }
      Sequence& s = seqs_[it->seq];
      switch (it->op) {
        case Op::kLen:
          s.len = it->aux;
          break;
        case Op::kPush:
          s.table.pop_back();
          rc_[it->block] = 0;
          free_.push_back(it->block);
          break;
        case Op::kCow:
          s.table[static_cast<size_t>(it->aux)] = it->old;
          ++rc_[it->old];
          rc_[it->block] = 0;
          free_.push_back(it->block);
          break;
        case Op::kEvict:
          break;
      }
    }
    undo_.clear();
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(error_buffer(), 512, fmt, ap);
    va_end(ap);
    return code;
  }

  int block_size_;
  std::vector<int32_t> free_;
  std::vector<int32_t> rc_;
  std::unordered_map<int64_t, Sequence> seqs_;
  std::vector<Undo> undo_;
  // prefix cache
  std::vector<Node> nodes_;
  std::vector<int> dead_;  // reusable node slots
  std::unordered_map<ChildKey, int, ChildKeyHash> children_;
  std::set<std::tuple<int64_t, int64_t, int>> lru_;
  std::vector<int> path_;
  int64_t clock_ = 0;
  int64_t next_order_ = 1;
  int cached_ = 0;
  int64_t lookups_ = 0, hits_ = 0, evictions_ = 0;
};

BlockManager* as_mgr(void* h) { return static_cast<BlockManager*>(h); }

}  // namespace
}  // namespace pkv

using pkv::fail;
using pkv::ok;

extern "C" {

const char* pkv_last_error(void) { return pkv::error_buffer(); }

int pkv_version(void) { return 10000; }

int pkv_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order, void** handle_out) {
  if (!handle_out) return fail(PKV_ERR_INVALID_ARG, "handle_out is NULL");
  *handle_out = nullptr;
  if (num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "num_blocks must be positive (got %d)", num_blocks);
  if (block_size != 16) return fail(PKV_ERR_UNSUPPORTED, "block_size must be 16 (got %d)", block_size);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b])
        return fail(PKV_ERR_INVALID_ARG, "initial_free_order is not a permutation of 0..%d", num_blocks - 1);
      seen[b] = 1;
    }
  }
  auto* m = new (std::nothrow) pkv::BlockManager(num_blocks, block_size, initial_free_order);
  if (!m) return fail(PKV_ERR_INVALID_ARG, "out of host memory");
  *handle_out = m;
  return ok();
}

int pkv_alloc_destroy(void* handle) {
  delete pkv::as_mgr(handle);
  return ok();
}

int pkv_seq_add(void* h, int64_t seq_id) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  return pkv::as_mgr(h)->add(seq_id);
}

int pkv_seq_fork(void* h, int64_t parent, int64_t child, int prefix_len) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  return pkv::as_mgr(h)->fork(parent, child, prefix_len);
}

int pkv_seq_append(void* h, int64_t seq_id, int n_tokens, int64_t* slots_out, int32_t* cow_pairs_out,
                   int cow_cap, int* num_cow_out) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (n_tokens < 0) return fail(PKV_ERR_INVALID_ARG, "n_tokens < 0");
  if (n_tokens > 0 && !slots_out) return fail(PKV_ERR_INVALID_ARG, "slots_out is NULL");
  if (cow_cap > 0 && !cow_pairs_out) return fail(PKV_ERR_INVALID_ARG, "cow_pairs_out is NULL");
  if (num_cow_out) *num_cow_out = 0;
  return pkv::as_mgr(h)->append(&seq_id, 1, n_tokens, slots_out, cow_pairs_out, cow_cap < 0 ? 0 : cow_cap,
                                num_cow_out);
}

int pkv_batch_append(void* h, const int64_t* seq_ids, int n, int64_t* slots_out, int32_t* cow_pairs_out,
                     int cow_cap, int* num_cow_out) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (n < 0 || (n > 0 && (!seq_ids || !slots_out))) return fail(PKV_ERR_INVALID_ARG, "bad batch arguments");
  if (cow_cap > 0 && !cow_pairs_out) return fail(PKV_ERR_INVALID_ARG, "cow_pairs_out is NULL");
  if (num_cow_out) *num_cow_out = 0;
  return pkv::as_mgr(h)->append(seq_ids, n, 1, slots_out, cow_pairs_out, cow_cap < 0 ? 0 : cow_cap, num_cow_out);
}

int pkv_batch_tables(void* h, const int64_t* seq_ids, int n, int32_t* bt, int max_blocks, int32_t* ctx) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (n < 0 || (n > 0 && (!seq_ids || !bt || !ctx)) || max_blocks <= 0)
    return fail(PKV_ERR_INVALID_ARG, "bad table export arguments");
  auto* m = pkv::as_mgr(h);
  for (int i = 0; i < n; ++i) {
    const pkv::Sequence* s = m->find(seq_ids[i]);
    if (!s) return fail(PKV_ERR_NOT_FOUND, "sequence %lld not found", (long long)seq_ids[i]);
    if (s->table.size() > static_cast<size_t>(max_blocks))
      return fail(PKV_ERR_INVALID_ARG, "sequence %lld has %zu blocks > max_blocks %d", (long long)seq_ids[i],
                  s->table.size(), max_blocks);
  }
  for (int i = 0; i < n; ++i) {
    const pkv::Sequence* s = m->find(seq_ids[i]);
    int32_t* row = bt + static_cast<size_t>(i) * max_blocks;
    std::memcpy(row, s->table.data(), s->table.size() * sizeof(int32_t));
    std::fill(row + s->table.size(), row + max_blocks, 0);
    ctx[i] = static_cast<int32_t>(s->len);
  }
  return ok();
}

int pkv_seq_free(void* h, int64_t seq_id) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  return pkv::as_mgr(h)->release(seq_id);
}

int pkv_seq_block_table(void* h, int64_t seq_id, int32_t* out, int cap, int* n_out) {
  if (!h || !n_out) return fail(PKV_ERR_INVALID_ARG, "NULL argument");
  const pkv::Sequence* s = pkv::as_mgr(h)->find(seq_id);
  if (!s) return fail(PKV_ERR_NOT_FOUND, "sequence %lld not found", (long long)seq_id);
  *n_out = static_cast<int>(s->table.size());
  if (s->table.size() > static_cast<size_t>(cap < 0 ? 0 : cap) || (!out && !s->table.empty()))
    return fail(PKV_ERR_INVALID_ARG, "table has %zu blocks, capacity %d", s->table.size(), cap);
  if (!s->table.empty()) std::memcpy(out, s->table.data(), s->table.size() * sizeof(int32_t));
  return ok();
}

int pkv_seq_len(void* h, int64_t seq_id, int* len_out) {
  if (!h || !len_out) return fail(PKV_ERR_INVALID_ARG, "NULL argument");
  const pkv::Sequence* s = pkv::as_mgr(h)->find(seq_id);
  if (!s) return fail(PKV_ERR_NOT_FOUND, "sequence %lld not found", (long long)seq_id);
  *len_out = static_cast<int>(s->len);
  return ok();
}

int pkv_block_refcount(void* h, int32_t block, int* rc_out) {
  if (!h || !rc_out) return fail(PKV_ERR_INVALID_ARG, "NULL argument");
  auto* m = pkv::as_mgr(h);
  if (block < 0 || block >= m->num_blocks()) return fail(PKV_ERR_INVALID_ARG, "block %d out of range", block);
  *rc_out = m->refcount(block);
  return ok();
}

int pkv_alloc_stats(void* h, int* num_free, int* num_shared, int* largest_free_run) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  pkv::as_mgr(h)->stats(num_free, num_shared, largest_free_run);
  return ok();
}

int pkv_prefix_key(const int32_t* token_ids, int n_tokens, uint8_t* key_out) {
  if (n_tokens < 0 || (n_tokens > 0 && !token_ids) || !key_out) return fail(PKV_ERR_INVALID_ARG, "bad arguments");
  pkv::Blake2b128 st;
  pkv::blake2b_tokens(&st, token_ids, n_tokens);
  st.digest(key_out);
  return ok();
}

int pkv_prefix_cache_insert(void* h, int64_t seq_id, const int32_t* token_ids, int n_tokens, int* newly_cached_out) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (n_tokens < 0 || (n_tokens > 0 && !token_ids)) return fail(PKV_ERR_INVALID_ARG, "bad token arguments");
  return pkv::as_mgr(h)->insert(seq_id, token_ids, n_tokens, newly_cached_out);
}

int pkv_prefix_cache_match(void* h, const int32_t* token_ids, int n_tokens, int* hit_tokens_out, uint8_t* key_out) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (n_tokens < 0 || (n_tokens > 0 && !token_ids)) return fail(PKV_ERR_INVALID_ARG, "bad token arguments");
  return pkv::as_mgr(h)->match(token_ids, n_tokens, hit_tokens_out, key_out);
}

int pkv_seq_add_cached(void* h, int64_t seq_id, const int32_t* token_ids, int n_tokens, int* hit_tokens_out) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (n_tokens < 0 || (n_tokens > 0 && !token_ids)) return fail(PKV_ERR_INVALID_ARG, "bad token arguments");
  return pkv::as_mgr(h)->add_cached(seq_id, token_ids, n_tokens, hit_tokens_out);
}

int pkv_prefix_cache_evict(void* h, int max_cached_blocks, int* evicted_out) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  if (max_cached_blocks < 0) return fail(PKV_ERR_INVALID_ARG, "max_cached_blocks < 0");
  return pkv::as_mgr(h)->evict_to(max_cached_blocks, evicted_out);
}

int pkv_prefix_cache_stats(void* h, int* cached_blocks, int* evictable_blocks, int64_t* lookups, int64_t* hits,
                           int64_t* evictions) {
  if (!h) return fail(PKV_ERR_INVALID_ARG, "NULL handle");
  pkv::as_mgr(h)->cache_stats(cached_blocks, evictable_blocks, lookups, hits, evictions);
  return ok();
}

}  // extern "C"
