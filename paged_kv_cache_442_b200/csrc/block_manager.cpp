// Host-side block manager: which physical block of the KV pool each block of a request
// lives in, and which blocks requests share.
//
// Follows the nano vllm KV-cache practice page: a Block has an id, a reference count,
// a content hash (-1 while unset) and the token ids it holds (section 3.2.1); allocation
// walks a request's blocks, and a full block whose chained hash is already registered
// (and whose tokens match) is reused with its reference count raised, otherwise a free
// block is taken and registered (section 3.2.2); the hash of a block is the rolling
// hash h = h * 31 + token (mod 2^32) seeded with the previous block's hash (section 4.2);
// finishing a request drops one reference per block and returns blocks that reach zero
// to the free list (section 3.2.1). The mini-vllm page plans this BlockAllocator in C++
// (section 1): it hands out blocks for prefill and decode and takes them back.
//
// Readings where the pages are silent (the same as the test fixture's):
//  * a hash hit is confirmed by comparing token ids (guards 32-bit collisions);
//  * a trailing partial block whose whole prefix chain matched, and whose tokens begin
//    an already cached full block chained on the same prefix, reuses that block;
//  * free blocks are taken in a caller-given order (a permutation of the pool);
//  * a freed block forgets its hash (it is not found again once its count is zero);
//  * decode append: a position that starts a block takes a fresh block; a block other
//    sequences also hold is replaced by a private copy first (copy-on-write; the copy is
//    reported for pa_copy_blocks); a private block still registered under a hash leaves
//    the hash map before it is written. Blocks filled by appends are not hashed.
#include <algorithm>
#include <cstdint>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_block_manager {
  struct Block {
    int32_t ref = 0;
    int64_t hash = -1;    // -1: unset, else a 32-bit hash
    int64_t parent = -1;  // hash this block was chained on (-1: none)
    std::vector<int32_t> tokens;
  };

  int32_t bs = 0;
  std::vector<Block> blocks;
  std::vector<int32_t> free_list;  // consumed from free_pos; freed blocks go to the end
  size_t free_pos = 0;
  std::unordered_map<uint32_t, int32_t> hash_to_id;
  std::unordered_map<uint32_t, std::vector<int32_t>> children;  // parent hash -> cached full blocks

  static uint32_t chain(const int32_t* t, int32_t n, uint32_t h) {
    for (int32_t i = 0; i < n; ++i) h = h * 31u + static_cast<uint32_t>(t[i]);
    return h;
  }

  void forget(int32_t id) {
    Block& b = blocks[id];
    if (b.hash >= 0) {
      auto it = hash_to_id.find(static_cast<uint32_t>(b.hash));
      if (it != hash_to_id.end() && it->second == id) hash_to_id.erase(it);
    }
    if (b.parent >= 0) {
      auto it = children.find(static_cast<uint32_t>(b.parent));
      if (it != children.end()) {
        auto& v = it->second;
        auto pos = std::find(v.begin(), v.end(), id);
        if (pos != v.end()) v.erase(pos);
      }
    }
    b.hash = -1;
    b.parent = -1;
    b.tokens.clear();
  }

  // next free block (reference count 0) in free-list order, or -1 when none is left
  int32_t take_free() {
    while (free_pos < free_list.size()) {
      const int32_t id = free_list[free_pos++];
      Block& b = blocks[id];
      if (b.ref == 0) {
        if (b.hash != -1) forget(id);
        if (free_pos > 4096 && free_pos * 2 > free_list.size()) {  // drop the consumed prefix
          free_list.erase(free_list.begin(), free_list.begin() + static_cast<long>(free_pos));
          free_pos = 0;
        }
        return id;
      }
    }
    return -1;
  }

  void release(const int32_t* table, int32_t n) {
    for (int32_t i = 0; i < n; ++i) {
      Block& b = blocks[table[i]];
      b.ref -= 1;
      if (b.ref == 0) {
        forget(table[i]);
        free_list.push_back(table[i]);
      }
    }
  }
};

extern "C" {

pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t* free_order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pa_block_manager* m = new (std::nothrow) pa_block_manager();
  if (!m) return nullptr;
  m->bs = block_size;
  m->blocks.resize(static_cast<size_t>(num_blocks));
  m->free_list.resize(static_cast<size_t>(num_blocks));
  if (free_order) {
    std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      const int32_t id = free_order[i];
      if (id < 0 || id >= num_blocks || seen[id]) {
        delete m;
        return nullptr;  // not a permutation of the pool
      }
      seen[id] = 1;
      m->free_list[i] = id;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) m->free_list[i] = i;
  }
  return m;
}

void pa_bm_destroy(pa_block_manager* m) { delete m; }

pa_status pa_bm_allocate(pa_block_manager* m, const int32_t* token_ids, int32_t num_tokens,
                         const uint32_t* block_hashes, int32_t* table_out) {
  if (!m || num_tokens < 0 || (num_tokens > 0 && (!token_ids || !table_out)))
    return PA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < num_tokens; ++i)
    if (token_ids[i] < 0) return PA_ERR_INVALID_ARG;
  const int32_t bs = m->bs;
  uint32_t h = 0;
  bool chain_ok = true;
  int32_t nt = 0;
  for (int32_t start = 0; start < num_tokens; start += bs) {
    const int32_t* chunk = token_ids + start;
    const int32_t len = std::min(bs, num_tokens - start);
    int32_t id = -1;
    if (len == bs) {
      const uint32_t parent = h;
      h = block_hashes ? block_hashes[start / bs] : pa_block_manager::chain(chunk, len, h);
      if (chain_ok) {
        auto it = m->hash_to_id.find(h);
        if (it != m->hash_to_id.end()) {
          const auto& t = m->blocks[it->second].tokens;
          if (static_cast<int32_t>(t.size()) == len && std::equal(t.begin(), t.end(), chunk))
            id = it->second;
        }
      }
      if (id >= 0) {
        m->blocks[id].ref += 1;
      } else {
        chain_ok = false;
        id = m->take_free();
        if (id < 0) {
          m->release(table_out, nt);  // the request holds nothing after a failure
          return PA_ERR_NO_BLOCKS;
        }
        auto& b = m->blocks[id];
        b.ref = 1;
        b.hash = h;
        b.parent = parent;
        b.tokens.assign(chunk, chunk + len);
        m->hash_to_id[h] = id;
        m->children[parent].push_back(id);
      }
    } else {
      if (chain_ok) {
        auto it = m->children.find(h);
        if (it != m->children.end()) {
          for (int32_t cand : it->second) {
            const auto& t = m->blocks[cand].tokens;
            if (static_cast<int32_t>(t.size()) >= len && std::equal(chunk, chunk + len, t.begin())) {
              id = cand;
              break;
            }
          }
        }
      }
      if (id >= 0) {
        m->blocks[id].ref += 1;
      } else {
        id = m->take_free();
        if (id < 0) {
          m->release(table_out, nt);
          return PA_ERR_NO_BLOCKS;
        }
        auto& b = m->blocks[id];
        b.ref = 1;
        b.hash = -1;
        b.tokens.assign(chunk, chunk + len);
      }
    }
    table_out[nt++] = id;
  }
  return PA_OK;
}

pa_status pa_bm_allocate_batch(pa_block_manager* m, const int32_t* token_ids,
                               const int32_t* cu_tokens, int32_t num_seqs,
                               const uint32_t* block_hashes, const int32_t* cu_blocks,
                               int32_t* tables_out, int32_t* num_done) {
  if (!m || num_seqs < 0 || !num_done || (num_seqs > 0 && (!cu_tokens || !tables_out)))
    return PA_ERR_INVALID_ARG;
  *num_done = 0;
  if (num_seqs == 0) return PA_OK;
  if (cu_tokens[0] != 0) return PA_ERR_INVALID_ARG;
  if (block_hashes && (!cu_blocks || cu_blocks[0] != 0)) return PA_ERR_INVALID_ARG;
  const int32_t bs = m->bs;
  // validate every request before taking any block
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int32_t len = cu_tokens[s + 1] - cu_tokens[s];
    if (len < 0) return PA_ERR_INVALID_ARG;
    if (len > 0 && !token_ids) return PA_ERR_INVALID_ARG;
    if (block_hashes && cu_blocks[s + 1] - cu_blocks[s] != len / bs) return PA_ERR_INVALID_ARG;
    // token ids are checked here too, so that every PA_ERR_INVALID_ARG comes before
    // any block is taken (pa_bm_allocate would reject a negative id only once the
    // requests before this one hold their blocks)
    for (int32_t i = cu_tokens[s]; i < cu_tokens[s + 1]; ++i)
      if (token_ids[i] < 0) return PA_ERR_INVALID_ARG;
  }
  int64_t off = 0;
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int32_t len = cu_tokens[s + 1] - cu_tokens[s];
    const pa_status st = pa_bm_allocate(m, token_ids ? token_ids + cu_tokens[s] : nullptr, len,
                                        block_hashes ? block_hashes + cu_blocks[s] : nullptr,
                                        tables_out + off);
    if (st != PA_OK) return st;  // requests before s stay allocated; s holds nothing
    off += (len + bs - 1) / bs;
    *num_done = s + 1;
  }
  return PA_OK;
}

pa_status pa_bm_free(pa_block_manager* m, const int32_t* table, int32_t num_entries) {
  if (!m || num_entries < 0 || (num_entries > 0 && !table)) return PA_ERR_INVALID_ARG;
  // validate first: every id in the pool and held at least as often as it is listed
  std::unordered_map<int32_t, int32_t> count;
  for (int32_t i = 0; i < num_entries; ++i) {
    const int32_t id = table[i];
    if (id < 0 || id >= static_cast<int32_t>(m->blocks.size())) return PA_ERR_INVALID_ARG;
    if (++count[id] > m->blocks[id].ref) return PA_ERR_INVALID_ARG;  // double free
  }
  m->release(table, num_entries);
  return PA_OK;
}

pa_status pa_bm_append(pa_block_manager* m, int32_t* table, int32_t* num_entries, int32_t capacity,
                       int32_t pos, int32_t token_id, int32_t* slot_out, int32_t* copy_src,
                       int32_t* copy_dst) {
  if (!m || !table || !num_entries || !slot_out || !copy_src || !copy_dst || pos < 0 ||
      token_id < 0)
    return PA_ERR_INVALID_ARG;
  const int32_t bs = m->bs;
  const int32_t bi = pos / bs, off = pos % bs;
  const int32_t n = *num_entries;
  *copy_src = *copy_dst = -1;
  if (bi == n) {
    if (off != 0 || n >= capacity) return PA_ERR_INVALID_ARG;
    const int32_t id = m->take_free();
    if (id < 0) return PA_ERR_NO_BLOCKS;
    auto& b = m->blocks[id];
    b.ref = 1;
    b.hash = -1;
    b.tokens.assign(1, token_id);
    table[n] = id;
    *num_entries = n + 1;
    *slot_out = id * bs;
    return PA_OK;
  }
  if (bi > n) return PA_ERR_INVALID_ARG;
  int32_t id = table[bi];
  if (id < 0 || id >= static_cast<int32_t>(m->blocks.size()) || m->blocks[id].ref <= 0)
    return PA_ERR_INVALID_ARG;
  if (m->blocks[id].ref > 1) {
    const int32_t nid = m->take_free();
    if (nid < 0) return PA_ERR_NO_BLOCKS;
    auto& src = m->blocks[id];
    auto& dst = m->blocks[nid];
    dst.ref = 1;
    dst.hash = -1;
    dst.tokens.assign(src.tokens.begin(),
                      src.tokens.begin() + std::min<size_t>(src.tokens.size(), static_cast<size_t>(off)));
    src.ref -= 1;
    *copy_src = id;
    *copy_dst = nid;
    table[bi] = nid;
    id = nid;
  } else if (m->blocks[id].hash != -1) {
    std::vector<int32_t> keep(m->blocks[id].tokens.begin(),
                              m->blocks[id].tokens.begin() +
                                  std::min<size_t>(m->blocks[id].tokens.size(), static_cast<size_t>(off)));
    m->forget(id);
    m->blocks[id].tokens = std::move(keep);
  }
  auto& t = m->blocks[id].tokens;
  if (t.size() > static_cast<size_t>(off)) t.resize(static_cast<size_t>(off));
  t.push_back(token_id);
  *slot_out = id * bs + off;
  return PA_OK;
}

int32_t pa_bm_num_used(const pa_block_manager* m) {
  if (!m) return -1;
  int32_t n = 0;
  for (const auto& b : m->blocks) n += b.ref > 0;
  return n;
}

pa_status pa_bm_ref_counts(const pa_block_manager* m, int32_t* out) {
  if (!m || !out) return PA_ERR_INVALID_ARG;
  for (size_t i = 0; i < m->blocks.size(); ++i) out[i] = m->blocks[i].ref;
  return PA_OK;
}

}  // extern "C"
