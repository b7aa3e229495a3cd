// block_allocator.cpp — host-side page (block) allocator for the paged KV cache.
//
// Pages are handed out on demand and a sequence gains pages as it grows
// ([csdn] "分页式KV缓存" benefit list; [betteryeah] §2.2); a finished
// sequence's pages return to the free list ([csdn] "典型工作流程拆解" step 7);
// samples of one prompt share its pages through their block tables, pages are
// reference-counted, and a page that several holders must modify is copied on
// write ([cortexgrid] FAQ answer on parallel sampling).
//
// Policy where the pages are silent: a FIFO free queue (front out, back in)
// with a caller-given initial order; copy-on-write only on an append into a
// partly filled last block whose refcount exceeds one; the last holder writes
// in place.  Every failing call leaves the state unchanged.
//
// Prefix caching ([csdn] API example `enable_prefix_caching` and its
// `cache_hit_rate` metric): a full prompt block is known by its whole token
// prefix.  Here that prefix is represented by a chain hash,
// h_k = mix(h_{k-1}, tokens of block k), with splitmix64 as the mixer
// (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
// 2014); a candidate block must also carry the same parent hash and the same
// block tokens, so two prefixes are confused only on a 64-bit collision of the
// parent chain.  Cached blocks whose refcount drops to zero stay cached on an
// LRU list and are evicted only when the free queue is empty.
#include <algorithm>
#include <climits>
#include <deque>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

struct pkv_alloc {
  struct Seq {
    std::vector<int> blocks;
    int64_t tokens = 0;
  };
  struct CacheEntry {
    bool cached = false;
    uint64_t hash = 0;         // chain hash of the block's prefix
    uint64_t parent_hash = 0;  // chain hash of the prefix before it
    std::vector<int32_t> tokens;
    std::list<int>::iterator lru;  // valid while the block is evictable
    bool evictable = false;
  };
  int num_blocks = 0;
  int block_size = 0;
  std::deque<int> free_q;
  std::vector<int> refcount;
  std::unordered_map<int64_t, Seq> seqs;
  std::vector<CacheEntry> entry;                 // per physical block
  std::unordered_map<uint64_t, int> cache;       // chain hash -> block
  std::list<int> evictable;                      // refcount-0 cached blocks, oldest first
  int64_t queried = 0, hits = 0, evicted = 0;

  int available() const { return static_cast<int>(free_q.size() + evictable.size()); }

  // A block with refcount 1: the free queue first, else the oldest evictable
  // cached block (its cache entry is dropped).  The caller checked available().
  int take() {
    int b;
    if (!free_q.empty()) {
      b = free_q.front();
      free_q.pop_front();
    } else {
      b = evictable.front();
      evictable.pop_front();
      CacheEntry& e = entry[b];
      cache.erase(e.hash);
      e.cached = false;
      e.evictable = false;
      e.tokens.clear();
      ++evicted;
    }
    refcount[b] = 1;
    return b;
  }

  void release(int b) {
    if (--refcount[b] == 0) {
      CacheEntry& e = entry[b];
      if (e.cached) {
        e.lru = evictable.insert(evictable.end(), b);
        e.evictable = true;
      } else {
        free_q.push_back(b);
      }
    }
  }
};

namespace {

int64_t blocks_for(int64_t tokens, int bs) { return (tokens + bs - 1) / bs; }

uint64_t splitmix64(uint64_t x) {
  x += 0x9e3779b97f4a7c15ull;
  x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
  x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}

constexpr uint64_t kRootHash = 0x243f6a8885a308d3ull;  // chain hash of the empty prefix

uint64_t chain_hash(uint64_t parent, const int32_t* tokens, int n) {
  uint64_t h = splitmix64(parent);
  for (int i = 0; i < n; ++i) h = splitmix64(h ^ static_cast<uint32_t>(tokens[i]));
  return h;
}

}  // namespace

extern "C" pkv_alloc* pkv_alloc_create(int num_blocks, int block_size,
                                       const int32_t* free_order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pkv_alloc* a = new (std::nothrow) pkv_alloc();
  if (a == nullptr) return nullptr;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->refcount.assign(num_blocks, 0);
  a->entry.resize(num_blocks);
  if (free_order == nullptr) {
    for (int b = 0; b < num_blocks; ++b) a->free_q.push_back(b);
  } else {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return nullptr;
      }
      seen[b] = 1;
      a->free_q.push_back(b);
    }
  }
  return a;
}

extern "C" void pkv_alloc_destroy(pkv_alloc* a) { delete a; }

extern "C" pkv_status pkv_alloc_add_seq(pkv_alloc* a, int64_t seq_id, int64_t num_tokens) {
  if (a == nullptr || num_tokens < 0 || a->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
  const int64_t need = blocks_for(num_tokens, a->block_size);
  if (need > a->available()) return PKV_ERR_OUT_OF_BLOCKS;
  pkv_alloc::Seq s;
  s.tokens = num_tokens;
  s.blocks.reserve(static_cast<size_t>(need));
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->take());
  a->seqs.emplace(seq_id, std::move(s));
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_fork(pkv_alloc* a, int64_t parent, int64_t child) {
  if (a == nullptr) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child)) return PKV_ERR_INVALID_ARG;
  pkv_alloc::Seq c = it->second;  // copy before emplace may rehash
  for (int b : c.blocks) a->refcount[b] += 1;
  a->seqs.emplace(child, std::move(c));
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_append_slot(pkv_alloc* a, int64_t seq_id, int64_t* slot,
                                            int64_t* cow_src, int64_t* cow_dst) {
  if (a == nullptr || slot == nullptr) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
  pkv_alloc::Seq& s = it->second;
  const int64_t pos = s.tokens;
  const int offset = static_cast<int>(pos % a->block_size);
  int64_t src = -1, dst = -1;
  if (offset == 0) {
    if (a->available() == 0) return PKV_ERR_OUT_OF_BLOCKS;
    s.blocks.push_back(a->take());
  } else {
    const int last = s.blocks.back();
    if (a->refcount[last] > 1) {
      if (a->available() == 0) return PKV_ERR_OUT_OF_BLOCKS;
      const int fresh = a->take();
      a->refcount[last] -= 1;
      s.blocks.back() = fresh;
      src = last;
      dst = fresh;
    }
  }
  s.tokens = pos + 1;
  *slot = static_cast<int64_t>(s.blocks.back()) * a->block_size + offset;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_append_slots(pkv_alloc* a, const int64_t* seq_ids, int n,
                                             int64_t* slots, int64_t* cow_pairs, int* num_cow,
                                             int* num_done) {
  if (num_done) *num_done = 0;
  if (num_cow) *num_cow = 0;
  if (a == nullptr || n < 0 || (n > 0 && (seq_ids == nullptr || slots == nullptr)))
    return PKV_ERR_INVALID_ARG;
  int ncow = 0;
  for (int i = 0; i < n; ++i) {
    int64_t src = -1, dst = -1;
    const pkv_status st = pkv_alloc_append_slot(a, seq_ids[i], &slots[i], &src, &dst);
    if (st != PKV_OK) return st;
    if (src >= 0) {
      if (cow_pairs) {
        cow_pairs[2 * ncow] = src;
        cow_pairs[2 * ncow + 1] = dst;
      }
      ++ncow;
      if (num_cow) *num_cow = ncow;
    }
    if (num_done) *num_done = i + 1;
  }
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_free_seq(pkv_alloc* a, int64_t seq_id) {
  if (a == nullptr) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
  for (int b : it->second.blocks) a->release(b);
  a->seqs.erase(it);
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_add_seq_cached(pkv_alloc* a, int64_t seq_id,
                                               const int32_t* token_ids, int64_t num_tokens,
                                               int64_t* num_cached_tokens) {
  if (a == nullptr || num_tokens < 0 || a->seqs.count(seq_id) ||
      (num_tokens > 0 && token_ids == nullptr))
    return PKV_ERR_INVALID_ARG;
  const int bs = a->block_size;
  const int64_t nfull = num_tokens / bs;
  const int64_t need = blocks_for(num_tokens, bs);
  // look the full blocks up in order, up to the first miss
  std::vector<int> hit;
  std::vector<uint64_t> hashes;
  uint64_t parent = kRootHash;
  for (int64_t k = 0; k < nfull; ++k) {
    const int32_t* tok = token_ids + k * bs;
    const uint64_t h = chain_hash(parent, tok, bs);
    hashes.push_back(h);
    if (static_cast<int64_t>(hit.size()) == k) {
      auto f = a->cache.find(h);
      if (f != a->cache.end()) {
        const pkv_alloc::CacheEntry& e = a->entry[f->second];
        if (e.parent_hash == parent && std::equal(e.tokens.begin(), e.tokens.end(), tok))
          hit.push_back(f->second);
      }
    }
    parent = h;
  }
  int reclaimed = 0;
  for (int b : hit) reclaimed += a->refcount[b] == 0 ? 1 : 0;
  if (need - static_cast<int64_t>(hit.size()) > a->available() - reclaimed)
    return PKV_ERR_OUT_OF_BLOCKS;
  a->queried += nfull;
  a->hits += static_cast<int64_t>(hit.size());
  pkv_alloc::Seq s;
  s.tokens = num_tokens;
  s.blocks.reserve(static_cast<size_t>(need));
  for (int b : hit) {
    pkv_alloc::CacheEntry& e = a->entry[b];
    if (a->refcount[b] == 0) {
      a->evictable.erase(e.lru);
      e.evictable = false;
    }
    a->refcount[b] += 1;
    s.blocks.push_back(b);
  }
  for (int64_t k = static_cast<int64_t>(hit.size()); k < need; ++k) {
    const int b = a->take();
    if (k < nfull && a->cache.find(hashes[k]) == a->cache.end()) {
      pkv_alloc::CacheEntry& e = a->entry[b];
      e.cached = true;
      e.hash = hashes[k];
      e.parent_hash = k == 0 ? kRootHash : hashes[k - 1];
      e.tokens.assign(token_ids + k * bs, token_ids + (k + 1) * bs);
      a->cache.emplace(hashes[k], b);
    }
    s.blocks.push_back(b);
  }
  a->seqs.emplace(seq_id, std::move(s));
  if (num_cached_tokens) *num_cached_tokens = static_cast<int64_t>(hit.size()) * bs;
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_cache_stats(const pkv_alloc* a, int64_t* queried_blocks,
                                            int64_t* hit_blocks, int64_t* cached_blocks,
                                            int64_t* evicted_blocks) {
  if (a == nullptr) return PKV_ERR_INVALID_ARG;
  if (queried_blocks) *queried_blocks = a->queried;
  if (hit_blocks) *hit_blocks = a->hits;
  if (cached_blocks) *cached_blocks = static_cast<int64_t>(a->cache.size());
  if (evicted_blocks) *evicted_blocks = a->evicted;
  return PKV_OK;
}

extern "C" int pkv_alloc_num_evictable(const pkv_alloc* a) {
  return a ? static_cast<int>(a->evictable.size()) : -1;
}

extern "C" pkv_status pkv_alloc_block_table(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                            int max_blocks, int32_t* table_out) {
  if (a == nullptr || n < 0 || max_blocks <= 0 || (n > 0 && (!seq_ids || !table_out)))
    return PKV_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end() || static_cast<int>(it->second.blocks.size()) > max_blocks)
      return PKV_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n; ++i) {
    const auto& blocks = a->seqs.find(seq_ids[i])->second.blocks;
    int32_t* row = table_out + static_cast<size_t>(i) * max_blocks;
    int j = 0;
    for (; j < static_cast<int>(blocks.size()); ++j) row[j] = blocks[j];
    for (; j < max_blocks; ++j) row[j] = -1;
  }
  return PKV_OK;
}

extern "C" pkv_status pkv_alloc_context_lens(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                             int32_t* lens_out) {
  if (a == nullptr || n < 0 || (n > 0 && (!seq_ids || !lens_out))) return PKV_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end() || it->second.tokens > INT32_MAX) return PKV_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n; ++i)
    lens_out[i] = static_cast<int32_t>(a->seqs.find(seq_ids[i])->second.tokens);
  return PKV_OK;
}

extern "C" int pkv_alloc_num_free(const pkv_alloc* a) {
  return a ? static_cast<int>(a->free_q.size()) : -1;
}

extern "C" int pkv_alloc_refcount(const pkv_alloc* a, int block) {
  if (a == nullptr || block < 0 || block >= a->num_blocks) return -1;
  return a->refcount[block];
}

extern "C" int64_t pkv_alloc_seq_len(const pkv_alloc* a, int64_t seq_id) {
  if (a == nullptr) return -1;
  auto it = a->seqs.find(seq_id);
  return it == a->seqs.end() ? -1 : it->second.tokens;
}

extern "C" int pkv_alloc_seq_num_blocks(const pkv_alloc* a, int64_t seq_id) {
  if (a == nullptr) return -1;
  auto it = a->seqs.find(seq_id);
  return it == a->seqs.end() ? -1 : static_cast<int>(it->second.blocks.size());
}

extern "C" pkv_status pkv_alloc_usage(const pkv_alloc* a, int64_t* cached_tokens,
                                      int64_t* used_blocks) {
  if (a == nullptr || cached_tokens == nullptr || used_blocks == nullptr)
    return PKV_ERR_INVALID_ARG;
  std::vector<int> fill(a->num_blocks, -1);
  for (const auto& kv : a->seqs) {
    const auto& s = kv.second;
    for (size_t k = 0; k < s.blocks.size(); ++k) {
      const int64_t f = std::min<int64_t>(a->block_size, s.tokens - static_cast<int64_t>(k) * a->block_size);
      const int b = s.blocks[k];
      if (f > fill[b]) fill[b] = static_cast<int>(f);
    }
  }
  int64_t tokens = 0, used = 0;
  for (int f : fill) {
    if (f >= 0) {
      tokens += f;
      ++used;
    }
  }
  *cached_tokens = tokens;
  *used_blocks = used;
  return PKV_OK;
}
