// Host block manager (include/block_manager.h): on-demand block allocation,
// reference counts, fork, copy-on-write of a shared partial last block and a
// prefix cache of full blocks keyed by their token ids.  Plain C++17 on the
// host; it never touches device memory (the copy-on-write copies are the
// caller's pa_copy_blocks launch).
#include "../../include/block_manager.h"

#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

namespace {

constexpr uint64_t kNoHash = 0;

// 64-bit hash of one full block: FNV-1a over the parent block's hash and the
// block's token ids (8 bytes each, little-endian), never 0 (0 marks "none").
uint64_t block_hash(uint64_t parent, const int64_t* tokens, int32_t n) {
  uint64_t h = 1469598103934665603ull;
  auto mix = [&h](uint64_t v) {
    for (int i = 0; i < 8; ++i) {
      h ^= (v >> (8 * i)) & 0xffu;
      h *= 1099511628211ull;
    }
  };
  mix(parent);
  for (int32_t i = 0; i < n; ++i) mix(static_cast<uint64_t>(tokens[i]));
  return h == kNoHash ? 1 : h;
}

struct Block {
  int32_t ref = 0;
  uint64_t hash = kNoHash;  // registered in the prefix cache under this hash (full blocks only)
  uint64_t parent = kNoHash;
  std::vector<int64_t> tokens;  // the token ids of a registered block
};

struct Seq {
  std::vector<int32_t> blocks;
  int32_t len = 0;
  // Prefix-cache chaining: the hash of the last full block, whether every
  // token so far is known, and the token ids of the partly filled last block.
  uint64_t last_full_hash = kNoHash;
  bool tokens_known = true;
  std::vector<int64_t> tail_tokens;
};

}  // namespace

struct pa_block_manager {
  int32_t num_blocks = 0, block_size = 0;
  std::vector<Block> blocks;
  std::deque<int32_t> free_list;  // blocks with count 0, in the order they were freed (stale entries skipped)
  std::vector<char> in_free;      // block is in free_list
  int32_t n_free = 0;
  std::unordered_map<uint64_t, int32_t> cache;  // hash -> registered block
  std::unordered_map<int64_t, Seq> seqs;

  // A registered block for (parent, tokens), or -1.
  int32_t lookup(uint64_t parent, const int64_t* tokens) const {
    const uint64_t h = block_hash(parent, tokens, block_size);
    auto it = cache.find(h);
    if (it == cache.end()) return -1;
    const Block& blk = blocks[it->second];
    if (blk.parent != parent || std::memcmp(blk.tokens.data(), tokens, sizeof(int64_t) * block_size) != 0)
      return -1;  // a hash collision: not the same prefix
    return it->second;
  }

  void unregister(int32_t id) {
    Block& blk = blocks[id];
    if (blk.hash != kNoHash) {
      auto it = cache.find(blk.hash);
      if (it != cache.end() && it->second == id) cache.erase(it);
      blk.hash = kNoHash;
      blk.parent = kNoHash;
      blk.tokens.clear();
    }
  }

  void register_full(int32_t id, uint64_t parent, const int64_t* tokens, uint64_t h) {
    if (cache.count(h)) return;  // an equal block is already registered: keep that one
    Block& blk = blocks[id];
    blk.hash = h;
    blk.parent = parent;
    blk.tokens.assign(tokens, tokens + block_size);
    cache[h] = id;
  }

  // Take a free block (count 0 -> 1); the caller has checked n_free > 0.
  int32_t allocate() {
    while (!free_list.empty()) {
      const int32_t id = free_list.front();
      free_list.pop_front();
      in_free[id] = 0;
      if (blocks[id].ref != 0) continue;  // revived from the prefix cache since it was freed
      unregister(id);
      blocks[id].ref = 1;
      --n_free;
      return id;
    }
    return -1;
  }

  // Count + 1 on a block that may be free (a prefix-cache hit).
  void acquire(int32_t id) {
    if (blocks[id].ref++ == 0) --n_free;  // its free-list entry becomes stale
  }

  void release(int32_t id) {
    if (--blocks[id].ref == 0) {
      ++n_free;
      if (!in_free[id]) {
        free_list.push_back(id);
        in_free[id] = 1;
      }
    }
  }

  // Blocks a new sequence of n tokens takes, with prefix-cache hits (a chain of
  // full blocks from the start) not counted.
  int32_t needed(const int64_t* tokens, int32_t n, int32_t* hits_out) const {
    int32_t hits = 0;
    if (tokens) {
      uint64_t parent = kNoHash;
      for (int32_t i = 0; (i + 1) * block_size <= n; ++i) {
        const int32_t id = lookup(parent, tokens + (size_t)i * block_size);
        if (id < 0) break;
        parent = blocks[id].hash;
        ++hits;
      }
    }
    if (hits_out) *hits_out = hits;
    const int32_t total = (n + block_size - 1) / block_size;
    return total - hits;
  }

  // Free blocks that allocation may use for a new sequence: the hits that are
  // free themselves (count 0) do not come from the free list, so they reduce
  // what is available.
  int32_t free_hits(const int64_t* tokens, int32_t hits) const {
    int32_t n = 0;
    uint64_t parent = kNoHash;
    for (int32_t i = 0; i < hits; ++i) {
      const int32_t id = lookup(parent, tokens + (size_t)i * block_size);
      if (blocks[id].ref == 0) ++n;
      parent = blocks[id].hash;
    }
    return n;
  }
};

extern "C" {

pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pa_block_manager* bm = new (std::nothrow) pa_block_manager();
  if (!bm) return nullptr;
  try {
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->blocks.resize(num_blocks);
    bm->in_free.assign(num_blocks, 1);
    for (int32_t i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
    bm->n_free = num_blocks;
  } catch (...) {
    delete bm;
    return nullptr;
  }
  return bm;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

int32_t pa_bm_num_free(const pa_block_manager* bm) { return bm ? bm->n_free : -1; }

int32_t pa_bm_blocks_needed(const pa_block_manager* bm, const int64_t* token_ids, int32_t num_tokens) {
  if (!bm || num_tokens < 0) return -1;
  return bm->needed(token_ids, num_tokens, nullptr);
}

pa_status_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int64_t* token_ids, int32_t num_tokens,
                               int32_t* cached_tokens) {
  if (!bm || num_tokens < 0 || bm->seqs.count(seq_id)) return PA_ERR_INVALID;
  int32_t hits = 0;
  const int32_t fresh = bm->needed(token_ids, num_tokens, &hits);
  const int32_t avail = bm->n_free - (token_ids ? bm->free_hits(token_ids, hits) : 0);
  if (fresh > avail) return PA_ERR_WORKSPACE;
  try {
    Seq s;
    const int32_t bs = bm->block_size;
    const int32_t nblk = (num_tokens + bs - 1) / bs;
    s.blocks.reserve(nblk);
    uint64_t parent = kNoHash;
    for (int32_t i = 0; i < nblk; ++i) {
      const bool full = (i + 1) * bs <= num_tokens;
      const int64_t* tk = token_ids ? token_ids + (size_t)i * bs : nullptr;
      int32_t id = -1;
      if (i < hits) {
        id = bm->lookup(parent, tk);
        bm->acquire(id);
      } else {
        id = bm->allocate();
        if (full && tk) bm->register_full(id, parent, tk, block_hash(parent, tk, bs));
      }
      if (full && tk) parent = block_hash(parent, tk, bs);
      s.blocks.push_back(id);
    }
    s.len = num_tokens;
    s.tokens_known = token_ids != nullptr;
    s.last_full_hash = parent;
    if (token_ids && num_tokens % bs) {
      const int32_t start = (num_tokens / bs) * bs;
      s.tail_tokens.assign(token_ids + start, token_ids + num_tokens);
    }
    bm->seqs.emplace(seq_id, std::move(s));
  } catch (...) {
    return PA_ERR_INVALID;  // out of host memory
  }
  if (cached_tokens) *cached_tokens = hits * bm->block_size;
  return PA_OK;
}

pa_status_t pa_bm_append_slots(pa_block_manager* bm, const int64_t* seq_ids, const int64_t* token_ids, int32_t n,
                               int64_t* slots_out, int32_t* cow_out, int32_t* num_cow) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !slots_out || !cow_out || !num_cow))) return PA_ERR_INVALID;
  const int32_t bs = bm->block_size;
  // Check everything first: ids known and distinct, and enough free blocks
  // for the new blocks and copies the step needs.
  int32_t need = 0;
  std::unordered_set<int64_t> seen;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || !seen.insert(seq_ids[i]).second) return PA_ERR_INVALID;
    const Seq& s = it->second;
    if (s.len % bs == 0) {
      ++need;  // a new block
    } else if (bm->blocks[s.blocks.back()].ref > 1) {
      ++need;  // copy-on-write of the shared partial last block
    }
  }
  if (need > bm->n_free) return PA_ERR_WORKSPACE;
  int32_t ncow = 0;
  for (int32_t i = 0; i < n; ++i) {
    Seq& s = bm->seqs[seq_ids[i]];
    const int32_t pos = s.len;
    if (pos % bs == 0) {
      s.blocks.push_back(bm->allocate());
    } else {
      const int32_t last = s.blocks.back();
      if (bm->blocks[last].ref > 1) {
        const int32_t fresh = bm->allocate();
        bm->release(last);
        s.blocks.back() = fresh;
        cow_out[2 * ncow] = last;
        cow_out[2 * ncow + 1] = fresh;
        ++ncow;
      }
    }
    slots_out[i] = (int64_t)s.blocks[pos / bs] * bs + pos % bs;
    s.len = pos + 1;
    // Prefix cache: a block the step fills, with every token known, is registered.
    if (token_ids && s.tokens_known) {
      s.tail_tokens.push_back(token_ids[i]);
      if (s.len % bs == 0) {
        const uint64_t h = block_hash(s.last_full_hash, s.tail_tokens.data(), bs);
        bm->register_full(s.blocks.back(), s.last_full_hash, s.tail_tokens.data(), h);
        s.last_full_hash = h;
        s.tail_tokens.clear();
      }
    } else {
      s.tokens_known = false;
    }
  }
  *num_cow = ncow;
  return PA_OK;
}

pa_status_t pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id) {
  if (!bm || parent_id == child_id || bm->seqs.count(child_id)) return PA_ERR_INVALID;
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID;
  try {
    Seq child = it->second;
    for (int32_t id : child.blocks) bm->acquire(id);
    bm->seqs.emplace(child_id, std::move(child));
  } catch (...) {
    return PA_ERR_INVALID;
  }
  return PA_OK;
}

pa_status_t pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id) {
  if (!bm) return PA_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID;
  for (int32_t id : it->second.blocks) bm->release(id);
  bm->seqs.erase(it);
  return PA_OK;
}

int32_t pa_bm_length(const pa_block_manager* bm, int64_t seq_id) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : it->second.len;
}

pa_status_t pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n, int32_t max_blocks,
                               int32_t* tables_out, int32_t* lens_out) {
  if (!bm || n < 0 || max_blocks <= 0 || (n > 0 && (!seq_ids || !tables_out || !lens_out))) return PA_ERR_INVALID;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || (int64_t)it->second.blocks.size() > max_blocks) return PA_ERR_INVALID;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq& s = bm->seqs.find(seq_ids[i])->second;
    int32_t* row = tables_out + (size_t)i * max_blocks;
    const int32_t k = (int32_t)s.blocks.size();
    for (int32_t j = 0; j < max_blocks; ++j) row[j] = j < k ? s.blocks[j] : -1;
    lens_out[i] = s.len;
  }
  return PA_OK;
}

pa_status_t pa_bm_slots(const pa_block_manager* bm, int64_t seq_id, int32_t start, int32_t count,
                        int64_t* slots_out) {
  if (!bm || start < 0 || count < 0 || (count > 0 && !slots_out)) return PA_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end() || (int64_t)start + count > it->second.len) return PA_ERR_INVALID;
  const int32_t bs = bm->block_size;
  for (int32_t i = 0; i < count; ++i) {
    const int32_t t = start + i;
    slots_out[i] = (int64_t)it->second.blocks[t / bs] * bs + t % bs;
  }
  return PA_OK;
}

int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->blocks[block].ref;
}

}  // extern "C"
