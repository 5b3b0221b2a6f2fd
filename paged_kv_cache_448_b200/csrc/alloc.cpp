// alloc.cpp — host block allocator and integer-table builders.
//
// The free list of "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.2
// (Block管理器实现): allocate(n) hands out the first n free ids or fails with
// out-of-memory leaving the list untouched; free appends released ids to the
// back. Blocks of a shared prompt prefix carry a reference count
// ("大模型推理KV Cache内存管理与PagedAttention分页显存实战": several sampling
// requests of one prompt share the prefix blocks, their lifetime managed by a
// reference count). Host memory only; no device calls.
//
// Prefix caching ("大模型推理KV Cache内存管理与PagedAttention分页显存实战",
// Prefix Caching: prefix blocks are reused across requests, found by hash
// matching): a full block may carry the content hash of prefix_hash.cpp. A
// block keeps its hash after its last reference is freed, so a later request
// with the same prefix can take it back from the free list; the hash is
// dropped only when the block is handed out for other content (it reaches
// the head of the free list), i.e. cached blocks are evicted oldest-freed first.
#include <array>
#include <cstring>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "paged.h"
#include "status.h"

namespace {
using Hash = std::array<uint8_t, 32>;
struct HashKey {
  size_t operator()(const Hash& h) const {
    size_t v;
    std::memcpy(&v, h.data(), sizeof(v));
    return v;
  }
};
Hash to_hash(const uint8_t* p) {
  Hash h;
  std::memcpy(h.data(), p, 32);
  return h;
}
}  // namespace

struct pa_alloc {
  std::list<int32_t> free_list;
  std::vector<std::list<int32_t>::iterator> where;  // position in free_list when free
  std::vector<int32_t> refcount;
  std::vector<char> hashed;
  std::vector<Hash> hash_of;
  std::unordered_map<Hash, int32_t, HashKey> by_hash;

  void push_free(int32_t id) { where[id] = free_list.insert(free_list.end(), id); }
  void drop_hash(int32_t id) {
    if (!hashed[id]) return;
    by_hash.erase(hash_of[id]);
    hashed[id] = 0;
  }
  // The head of the free list, for new content: its cached hash goes.
  int32_t pop_free() {
    const int32_t id = free_list.front();
    free_list.pop_front();
    drop_hash(id);
    refcount[id] = 1;
    return id;
  }
};

using paged::clear_error;
using paged::fail;

extern "C" {

PA_API pa_status pa_alloc_create(int64_t num_blocks, const int32_t* initial_free_order,
                                 pa_alloc** out) {
  clear_error();
  if (!out) return fail(PA_ERR_INVALID_ARG, "alloc_create: null output");
  *out = nullptr;
  if (num_blocks <= 0 || num_blocks > INT32_MAX)
    return fail(PA_ERR_INVALID_ARG, "alloc_create: num_blocks out of range");
  pa_alloc* a = new (std::nothrow) pa_alloc;
  if (!a) return fail(PA_ERR_OOM, "alloc_create: host allocation failed");
  a->refcount.assign(static_cast<size_t>(num_blocks), 0);
  a->where.resize(static_cast<size_t>(num_blocks));
  a->hashed.assign(static_cast<size_t>(num_blocks), 0);
  a->hash_of.resize(static_cast<size_t>(num_blocks));
  if (initial_free_order) {
    std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
    for (int64_t i = 0; i < num_blocks; ++i) {
      const int32_t id = initial_free_order[i];
      if (id < 0 || id >= num_blocks || seen[id]) {
        delete a;
        return fail(PA_ERR_INVALID_ARG, "alloc_create: initial order is not a permutation");
      }
      seen[id] = 1;
      a->push_free(id);
    }
  } else {
    for (int64_t i = 0; i < num_blocks; ++i) a->push_free(static_cast<int32_t>(i));
  }
  *out = a;
  return PA_OK;
}

PA_API void pa_alloc_destroy(pa_alloc* a) { delete a; }

PA_API pa_status pa_alloc_allocate(pa_alloc* a, int32_t n, int32_t* ids_out) {
  clear_error();
  if (!a || n < 0 || (n > 0 && !ids_out)) return fail(PA_ERR_INVALID_ARG, "alloc_allocate: bad args");
  if (static_cast<size_t>(n) > a->free_list.size())
    return fail(PA_ERR_OOM, "Need %d blocks, only %zu available", n, a->free_list.size());
  for (int32_t i = 0; i < n; ++i) ids_out[i] = a->pop_free();
  return PA_OK;
}

PA_API pa_status pa_alloc_share(pa_alloc* a, int32_t id) {
  clear_error();
  if (!a || id < 0 || static_cast<size_t>(id) >= a->refcount.size() || a->refcount[id] == 0)
    return fail(PA_ERR_INVALID_ARG, "alloc_share: block %d is not allocated", id);
  if (a->refcount[id] == INT32_MAX) return fail(PA_ERR_INVALID_ARG, "alloc_share: refcount overflow");
  ++a->refcount[id];
  return PA_OK;
}

PA_API pa_status pa_alloc_free(pa_alloc* a, const int32_t* ids, int32_t n) {
  clear_error();
  if (!a || n < 0 || (n > 0 && !ids)) return fail(PA_ERR_INVALID_ARG, "alloc_free: bad args");
  std::unordered_map<int32_t, int32_t> drops;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = ids[i];
    if (id < 0 || static_cast<size_t>(id) >= a->refcount.size())
      return fail(PA_ERR_INVALID_ARG, "alloc_free: unknown block %d", id);
    if (++drops[id] > a->refcount[id])
      return fail(PA_ERR_INVALID_ARG, "alloc_free: block %d freed more often than referenced", id);
  }
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = ids[i];
    if (--a->refcount[id] == 0) a->push_free(id);
  }
  return PA_OK;
}

// A holder about to write into a block with refcount > 1 moves its reference
// to a fresh block (the head of the free list) and copies the contents there;
// with refcount 1 it writes in place. The pages give refcounted sharing but no
// write rule: this is the plainest reading that keeps other holders intact.
PA_API pa_status pa_alloc_copy_on_write(pa_alloc* a, int32_t id, int32_t* id_out,
                                        int32_t* must_copy) {
  clear_error();
  if (!a || !id_out || !must_copy) return fail(PA_ERR_INVALID_ARG, "alloc_copy_on_write: bad args");
  if (id < 0 || static_cast<size_t>(id) >= a->refcount.size() || a->refcount[id] == 0)
    return fail(PA_ERR_INVALID_ARG, "alloc_copy_on_write: block %d is not allocated", id);
  if (a->refcount[id] == 1) {
    *id_out = id;
    *must_copy = 0;
    return PA_OK;
  }
  if (a->free_list.empty()) return fail(PA_ERR_OOM, "Need 1 block, only 0 available");
  const int32_t fresh = a->pop_free();
  --a->refcount[id];
  *id_out = fresh;
  *must_copy = 1;
  return PA_OK;
}

PA_API pa_status pa_alloc_acquire_prefix(pa_alloc* a, const uint8_t* hashes, int32_t n,
                                         int32_t* ids_out, int32_t* num_hits) {
  clear_error();
  if (!a || n < 0 || (n > 0 && (!hashes || !ids_out)) || !num_hits)
    return fail(PA_ERR_INVALID_ARG, "alloc_acquire_prefix: bad args");
  // Feasibility first (nothing changes on PA_ERR_OOM): cached blocks that sit
  // in the free list leave it, and every other hash needs a fresh block.
  int64_t free_hits = 0, misses = 0;
  std::unordered_map<Hash, int32_t, HashKey> fresh;  // hashes first seen in this request
  for (int32_t i = 0; i < n; ++i) {
    const Hash h = to_hash(hashes + 32 * static_cast<int64_t>(i));
    auto it = a->by_hash.find(h);
    if (it != a->by_hash.end()) {
      if (a->refcount[it->second] == 0 && !fresh.count(h)) {
        fresh.emplace(h, -1);  // revived once
        ++free_hits;
      }
    } else if (fresh.emplace(h, -1).second) {
      ++misses;
    }
  }
  if (misses > static_cast<int64_t>(a->free_list.size()) - free_hits)
    return fail(PA_ERR_OOM, "Need %lld new blocks, only %lld available",
                static_cast<long long>(misses),
                static_cast<long long>(a->free_list.size()) - free_hits);
  // Cached blocks first, so that no fresh allocation evicts one of them.
  int32_t hits = 0;
  std::vector<char> done(static_cast<size_t>(n), 0);
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->by_hash.find(to_hash(hashes + 32 * static_cast<int64_t>(i)));
    if (it == a->by_hash.end()) continue;
    const int32_t id = it->second;
    if (a->refcount[id] == 0) {
      a->free_list.erase(a->where[id]);
      a->refcount[id] = 1;
    } else {
      ++a->refcount[id];
    }
    ids_out[i] = id;
    done[i] = 1;
    ++hits;
  }
  for (int32_t i = 0; i < n; ++i) {
    if (done[i]) continue;
    const Hash h = to_hash(hashes + 32 * static_cast<int64_t>(i));
    auto it = a->by_hash.find(h);
    if (it != a->by_hash.end()) {  // registered by an earlier block of this request
      ++a->refcount[it->second];
      ids_out[i] = it->second;
      ++hits;
      continue;
    }
    const int32_t id = a->pop_free();
    a->hashed[id] = 1;
    a->hash_of[id] = h;
    a->by_hash.emplace(h, id);
    ids_out[i] = id;
  }
  *num_hits = hits;
  return PA_OK;
}

PA_API pa_status pa_alloc_register_hash(pa_alloc* a, int32_t id, const uint8_t* hash) {
  clear_error();
  if (!a || !hash || id < 0 || static_cast<size_t>(id) >= a->refcount.size() ||
      a->refcount[id] == 0)
    return fail(PA_ERR_INVALID_ARG, "alloc_register_hash: block %d is not allocated", id);
  const Hash h = to_hash(hash);
  auto it = a->by_hash.find(h);
  if (it != a->by_hash.end()) return PA_OK;  // that content is cached already (maybe here)
  a->drop_hash(id);
  a->hashed[id] = 1;
  a->hash_of[id] = h;
  a->by_hash.emplace(h, id);
  return PA_OK;
}

PA_API int32_t pa_alloc_lookup(const pa_alloc* a, const uint8_t* hash) {
  if (!a || !hash) return -1;
  auto it = a->by_hash.find(to_hash(hash));
  return it == a->by_hash.end() ? -1 : it->second;
}

PA_API int64_t pa_alloc_num_free(const pa_alloc* a) {
  return a ? static_cast<int64_t>(a->free_list.size()) : -1;
}

PA_API int64_t pa_alloc_num_blocks(const pa_alloc* a) {
  return a ? static_cast<int64_t>(a->refcount.size()) : -1;
}

PA_API int32_t pa_alloc_refcount(const pa_alloc* a, int32_t id) {
  if (!a || id < 0 || static_cast<size_t>(id) >= a->refcount.size()) return -1;
  return a->refcount[id];
}

PA_API int64_t pa_alloc_free_list(const pa_alloc* a, int32_t* ids_out, int64_t cap) {
  if (!a) return -1;
  int64_t i = 0;
  for (int32_t id : a->free_list) {
    if (i >= cap) break;
    ids_out[i++] = id;
  }
  return static_cast<int64_t>(a->free_list.size());
}

PA_API pa_status pa_build_block_table(const int32_t* const* seq_block_ids,
                                      const int32_t* num_blocks_per_seq, int32_t num_seqs,
                                      int32_t max_blocks_per_seq, int32_t* table_out) {
  clear_error();
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || (num_seqs > 0 && (!seq_block_ids ||
      !num_blocks_per_seq || !table_out)))
    return fail(PA_ERR_INVALID_ARG, "build_block_table: bad args");
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int32_t n = num_blocks_per_seq[s];
    if (n < 0 || n > max_blocks_per_seq || (n > 0 && !seq_block_ids[s]))
      return fail(PA_ERR_INVALID_ARG, "build_block_table: sequence %d has %d blocks (max %d)", s,
                  n, max_blocks_per_seq);
  }
  for (int32_t s = 0; s < num_seqs; ++s) {
    int32_t* row = table_out + static_cast<int64_t>(s) * max_blocks_per_seq;
    const int32_t n = num_blocks_per_seq[s];
    for (int32_t j = 0; j < max_blocks_per_seq; ++j) row[j] = j < n ? seq_block_ids[s][j] : -1;
  }
  return PA_OK;
}

PA_API pa_status pa_build_slot_mapping(const int32_t* block_tables, int32_t num_seqs,
                                       int32_t max_blocks_per_seq, const int32_t* seq_ids,
                                       const int32_t* positions, int32_t num_tokens,
                                       int32_t block_size, int32_t* slots_out) {
  clear_error();
  if (num_tokens < 0 || num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 ||
      (num_tokens > 0 && (!block_tables || !positions || !slots_out)))
    return fail(PA_ERR_INVALID_ARG, "build_slot_mapping: bad args");
  for (int32_t i = 0; i < num_tokens; ++i) {
    const int32_t seq = seq_ids ? seq_ids[i] : i;
    const int32_t pos = positions[i];
    if (pos < 0) {
      slots_out[i] = -1;
      continue;
    }
    if (seq < 0 || seq >= num_seqs)
      return fail(PA_ERR_INVALID_ARG, "build_slot_mapping: token %d names sequence %d", i, seq);
    const int32_t logical = pos / block_size;
    if (logical >= max_blocks_per_seq)
      return fail(PA_ERR_BAD_TABLE, "build_slot_mapping: position %d past the table", pos);
    const int64_t phys = block_tables[static_cast<int64_t>(seq) * max_blocks_per_seq + logical];
    if (phys < 0)
      return fail(PA_ERR_BAD_TABLE, "build_slot_mapping: no block for position %d", pos);
    const int64_t slot = phys * block_size + pos % block_size;
    if (slot > INT32_MAX) return fail(PA_ERR_BAD_TABLE, "build_slot_mapping: slot overflows int32");
    slots_out[i] = static_cast<int32_t>(slot);
  }
  return PA_OK;
}

}  // extern "C"
