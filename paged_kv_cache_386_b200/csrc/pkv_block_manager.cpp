// pkv_block_manager.cpp -- host-side block manager of the paged KV cache
// (declared in include/pagedkv.h, pkv_bm_*).
//
// It keeps the physical block pool and the per-sequence block tables that the
// kernels read ("Transformer anatomy" ch. 15 §15.5: fixed blocks of 16 tokens,
// a per-sequence block table, append into the current block and take a new
// block from the free pool when it is full, return the blocks when the
// sequence ends; "LLM Primer VI" ch. 8 §8.1: a flat physical pool, refcounted
// block sharing for parallel sampling).  Prefix caching ("Transformer anatomy"
// §15.6, hash-keyed blocks with LRU eviction; "LLM Primer VI" §8.3: hash the
// prompt per block, point the table at cached blocks and skip their prefill)
// keys full prompt blocks by a caller-supplied chained hash.
//
// Determinism (so that a reference model can be compared operation by
// operation): a new block is the lowest free block id; when no block is free,
// the least recently released cached block is evicted.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <map>
#include <memory>
#include <iterator>
#include <new>
#include <set>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

namespace {

struct Sequence {
  std::vector<int32_t> blocks;
  int64_t tokens = 0;
};

struct CachedInfo {
  uint64_t hash;
  bool in_lru;
  std::list<int32_t>::iterator lru_it;
};

}  // namespace

struct pkv_block_manager {
  int32_t num_blocks;
  int32_t block_size;
  bool prefix_cache;
  std::vector<int32_t> refcount;                     // per block
  std::set<int32_t> free_blocks;                     // refcount 0, not cached
  std::unordered_map<uint64_t, int32_t> hash_to_block;
  std::unordered_map<int32_t, CachedInfo> cached;    // registered blocks
  std::list<int32_t> lru;                            // cached blocks with refcount 0, oldest first
  std::map<int64_t, Sequence> seqs;

  // Blocks that can be handed out now (free or evictable).
  int64_t available() const { return static_cast<int64_t>(free_blocks.size()) + static_cast<int64_t>(lru.size()); }

  int32_t take_block() {
    int32_t b;
    if (!free_blocks.empty()) {
      b = *free_blocks.begin();
      free_blocks.erase(free_blocks.begin());
    } else {
      b = lru.front();  // callers check available() first
      lru.pop_front();
      auto it = cached.find(b);
      hash_to_block.erase(it->second.hash);
      cached.erase(it);
    }
    refcount[b] = 1;
    return b;
  }

  void release(int32_t b) {
    if (--refcount[b] > 0) return;
    auto it = cached.find(b);
    if (it != cached.end()) {
      lru.push_back(b);
      it->second.in_lru = true;
      it->second.lru_it = std::prev(lru.end());
    } else {
      free_blocks.insert(b);
    }
  }

  void acquire_cached(int32_t b) {
    if (refcount[b]++ == 0) {
      auto& ci = cached.find(b)->second;
      if (ci.in_lru) {
        lru.erase(ci.lru_it);
        ci.in_lru = false;
      }
    }
  }
};

// The C entry points must not let an exception escape; host allocation
// failure inside the containers is reported as PKV_ERR_HOST_MEMORY.
template <class F>
static pkv_status guarded(F&& f) noexcept {
  try {
    return f();
  } catch (...) {
    return PKV_ERR_HOST_MEMORY;
  }
}

// FNV-1a, 64-bit (offset basis 0xcbf29ce484222325, prime 0x100000001b3).
static uint64_t fnv1a_update(uint64_t h, const uint8_t* p, size_t n) {
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 0x100000001b3ull;
  }
  return h;
}

extern "C" {

pkv_status pkv_bm_create(int32_t num_blocks, int32_t block_size, int32_t enable_prefix_cache,
                         pkv_block_manager** out) {
  if (!out || num_blocks <= 0 || block_size <= 0) return PKV_ERR_INVALID_ARG;
  return guarded([&] {
    std::unique_ptr<pkv_block_manager> bm(new pkv_block_manager());
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->prefix_cache = enable_prefix_cache != 0;
    bm->refcount.assign(num_blocks, 0);
    for (int32_t b = 0; b < num_blocks; ++b) bm->free_blocks.insert(bm->free_blocks.end(), b);
    *out = bm.release();
    return PKV_OK;
  });
}

pkv_status pkv_bm_hash_blocks(const int32_t* tokens, int64_t n_tokens, int32_t block_size, uint64_t seed,
                              uint64_t* hashes) {
  if (n_tokens < 0 || block_size <= 0 || (n_tokens >= block_size && (!tokens || !hashes)))
    return PKV_ERR_INVALID_ARG;
  uint64_t prev = seed;
  for (int64_t i = 0; i < n_tokens / block_size; ++i) {
    uint8_t bytes[8];
    for (int j = 0; j < 8; ++j) bytes[j] = static_cast<uint8_t>(prev >> (8 * j));
    uint64_t h = fnv1a_update(0xcbf29ce484222325ull, bytes, 8);
    for (int32_t t = 0; t < block_size; ++t) {
      const uint32_t v = static_cast<uint32_t>(tokens[i * block_size + t]);
      uint8_t tb[4] = {static_cast<uint8_t>(v), static_cast<uint8_t>(v >> 8), static_cast<uint8_t>(v >> 16),
                       static_cast<uint8_t>(v >> 24)};
      h = fnv1a_update(h, tb, 4);
    }
    hashes[i] = h;
    prev = h;
  }
  return PKV_OK;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, int64_t n_prompt_tokens,
                               const uint64_t* block_hashes, int64_t* n_cached_tokens) {
  if (!bm || n_prompt_tokens < 0 || bm->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
  const int64_t bs = bm->block_size;
  const int64_t n_blocks = (n_prompt_tokens + bs - 1) / bs;
  const int64_t n_full = n_prompt_tokens / bs;
  // Leading full blocks found in the prefix cache are shared.
  int64_t hits = 0;
  if (bm->prefix_cache && block_hashes) {
    while (hits < n_full && bm->hash_to_block.count(block_hashes[hits])) ++hits;
  }
  // Capacity: cached hits that sit in the LRU list leave it, new blocks are taken.
  int64_t hits_from_lru = 0;
  for (int64_t i = 0; i < hits; ++i)
    if (bm->refcount[bm->hash_to_block.at(block_hashes[i])] == 0) ++hits_from_lru;
  if (bm->available() - hits_from_lru < n_blocks - hits) return PKV_ERR_NO_BLOCKS;
  return guarded([&] {
  Sequence s;
  s.tokens = n_prompt_tokens;
  for (int64_t i = 0; i < hits; ++i) {
    const int32_t b = bm->hash_to_block.at(block_hashes[i]);
    bm->acquire_cached(b);
    s.blocks.push_back(b);
  }
  for (int64_t i = hits; i < n_blocks; ++i) {
    const int32_t b = bm->take_block();
    s.blocks.push_back(b);
    if (bm->prefix_cache && block_hashes && i < n_full && !bm->hash_to_block.count(block_hashes[i])) {
      bm->hash_to_block[block_hashes[i]] = b;
      bm->cached[b] = CachedInfo{block_hashes[i], false, {}};
    }
  }
  bm->seqs.emplace(seq_id, std::move(s));
  if (n_cached_tokens) *n_cached_tokens = hits * bs;
  return PKV_OK;
  });
}

pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child) {
  if (!bm || !bm->seqs.count(parent) || bm->seqs.count(child)) return PKV_ERR_INVALID_ARG;
  return guarded([&] {
    Sequence s = bm->seqs.at(parent);
    bm->seqs.emplace(child, s);
    for (int32_t b : s.blocks) ++bm->refcount[b];
    return PKV_OK;
  });
}

pkv_status pkv_bm_append(pkv_block_manager* bm, const int64_t* seq_ids, int32_t n, int64_t* slot_mapping,
                         int32_t* cow_src, int32_t* cow_dst, int32_t* n_cow) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !slot_mapping || !cow_src || !cow_dst)) || !n_cow)
    return PKV_ERR_INVALID_ARG;
  const int64_t bs = bm->block_size;
  // Validate and count the blocks needed before changing anything.
  int64_t need = 0;
  std::vector<int64_t> sorted;
  if (guarded([&] { sorted.assign(seq_ids, seq_ids + n); return PKV_OK; }) != PKV_OK) return PKV_ERR_HOST_MEMORY;
  std::sort(sorted.begin(), sorted.end());
  if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end()) return PKV_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
    const Sequence& s = it->second;
    if (s.tokens % bs == 0) ++need;                                   // a new block
    else if (bm->refcount[s.blocks.back()] > 1) ++need;               // copy-on-write of a shared tail
  }
  if (bm->available() < need) return PKV_ERR_NO_BLOCKS;
  return guarded([&] {
  int32_t copies = 0;
  for (int32_t i = 0; i < n; ++i) {
    Sequence& s = bm->seqs.find(seq_ids[i])->second;
    const int64_t off = s.tokens % bs;
    if (off == 0) {
      s.blocks.push_back(bm->take_block());
    } else if (bm->refcount[s.blocks.back()] > 1) {
      const int32_t old = s.blocks.back();
      const int32_t fresh = bm->take_block();
      bm->release(old);
      s.blocks.back() = fresh;
      cow_src[copies] = old;
      cow_dst[copies] = fresh;
      ++copies;
    }
    slot_mapping[i] = static_cast<int64_t>(s.blocks.back()) * bs + off;
    ++s.tokens;
  }
  *n_cow = copies;
  return PKV_OK;
  });
}

pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
  if (!bm) return PKV_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
  // Release from the tail so that earlier (prefix) blocks stay cached longer.
  return guarded([&] {
    for (auto b = it->second.blocks.rbegin(); b != it->second.blocks.rend(); ++b) bm->release(*b);
    bm->seqs.erase(it);
    return PKV_OK;
  });
}

pkv_status pkv_bm_get_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int32_t n, int32_t width,
                             int32_t* block_tables, int32_t* context_lens) {
  if (!bm || n < 0 || width <= 0 || (n > 0 && (!seq_ids || !block_tables || !context_lens)))
    return PKV_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
    const Sequence& s = it->second;
    if (static_cast<int64_t>(s.blocks.size()) > width || s.tokens > INT32_MAX) return PKV_ERR_INVALID_ARG;
    int32_t* row = block_tables + static_cast<size_t>(i) * width;
    for (int32_t j = 0; j < width; ++j) row[j] = j < static_cast<int32_t>(s.blocks.size()) ? s.blocks[j] : -1;
    context_lens[i] = static_cast<int32_t>(s.tokens);
  }
  return PKV_OK;
}

pkv_status pkv_bm_stats(const pkv_block_manager* bm, pkv_bm_stats_t* out) {
  if (!bm || !out) return PKV_ERR_INVALID_ARG;
  out->num_blocks = bm->num_blocks;
  out->free_blocks = static_cast<int32_t>(bm->free_blocks.size());
  out->cached_idle_blocks = static_cast<int32_t>(bm->lru.size());
  out->used_blocks = bm->num_blocks - out->free_blocks - out->cached_idle_blocks;
  out->cached_blocks = static_cast<int32_t>(bm->cached.size());
  out->sequences = static_cast<int32_t>(bm->seqs.size());
  int64_t tokens = 0, slots = 0;
  for (const auto& kv : bm->seqs) {
    tokens += kv.second.tokens;
    slots += static_cast<int64_t>(kv.second.blocks.size()) * bm->block_size;
  }
  out->tokens = tokens;
  out->allocated_slots = slots;
  return PKV_OK;
}

pkv_status pkv_bm_refcount(const pkv_block_manager* bm, int32_t block, int32_t* refcount) {
  if (!bm || !refcount || block < 0 || block >= bm->num_blocks) return PKV_ERR_INVALID_ARG;
  *refcount = bm->refcount[block];
  return PKV_OK;
}

}  // extern "C"
