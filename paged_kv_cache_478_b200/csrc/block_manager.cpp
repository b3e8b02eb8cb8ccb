// Host block manager: free list and per-block reference counts.
//
// "Atención paginada en modelos de lenguaje grandes (LLM)" (7minutos.es),
// section 2: a flat pool of equal pages with a free list and a reference
// count per page; a page whose count reaches zero is free again at once, and
// a request claims a new page only when its token count crosses a page
// boundary.  Section 3: share() adds a holder without allocating; cow_copy()
// gives one holder a private page and drops its reference to the original.
//
// The free list is a min-heap, so the lowest free id is handed out first (a
// fresh pool gives 0, 1, 2, ...).  The device never sees this structure; it
// only receives the block tables, slots and copy pairs built here.
#include <algorithm>
#include <cstdint>
#include <functional>
#include <new>
#include <queue>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"
#include "status.h"

struct pa_allocator {
  std::vector<int32_t> refcount;
  std::priority_queue<int32_t, std::vector<int32_t>, std::greater<int32_t>> free_ids;
};

namespace {

bool live(const pa_allocator* a, int32_t id) {
  return id >= 0 && static_cast<size_t>(id) < a->refcount.size() && a->refcount[id] > 0;
}

pa_status take(pa_allocator* a, int32_t* id) {
  if (a->free_ids.empty()) return pa::fail(PA_ERR_NO_FREE_BLOCKS, "block pool exhausted");
  *id = a->free_ids.top();
  a->free_ids.pop();
  a->refcount[*id] = 1;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_alloc_create(int64_t num_blocks, pa_allocator** out) {
  if (!out) return pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_create: out is null");
  *out = nullptr;
  if (num_blocks <= 0 || num_blocks > INT32_MAX)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_create: num_blocks must be in [1, 2^31)");
  pa_allocator* a = new (std::nothrow) pa_allocator;
  if (!a) return pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_create: out of host memory");
  a->refcount.assign(static_cast<size_t>(num_blocks), 0);
  std::vector<int32_t> ids(static_cast<size_t>(num_blocks));
  for (int32_t i = 0; i < static_cast<int32_t>(num_blocks); ++i) ids[i] = i;
  a->free_ids = decltype(a->free_ids)(std::greater<int32_t>(), std::move(ids));
  *out = a;
  return PA_OK;
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

pa_status pa_alloc_block(pa_allocator* a, int32_t* block_id) {
  if (!a || !block_id) return pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_block: null argument");
  return take(a, block_id);
}

pa_status pa_share_block(pa_allocator* a, int32_t block_id) {
  if (!a) return pa::fail(PA_ERR_INVALID_ARG, "pa_share_block: null allocator");
  if (!live(a, block_id)) return pa::fail(PA_ERR_INVALID_ARG, "pa_share_block: block not allocated");
  a->refcount[block_id] += 1;
  return PA_OK;
}

pa_status pa_free_block(pa_allocator* a, int32_t block_id) {
  if (!a) return pa::fail(PA_ERR_INVALID_ARG, "pa_free_block: null allocator");
  if (!live(a, block_id)) return pa::fail(PA_ERR_INVALID_ARG, "pa_free_block: block not allocated");
  if (--a->refcount[block_id] == 0) a->free_ids.push(block_id);
  return PA_OK;
}

pa_status pa_cow_block(pa_allocator* a, int32_t block_id, int32_t* new_block_id) {
  if (!a || !new_block_id) return pa::fail(PA_ERR_INVALID_ARG, "pa_cow_block: null argument");
  if (!live(a, block_id)) return pa::fail(PA_ERR_INVALID_ARG, "pa_cow_block: block not allocated");
  pa_status st = take(a, new_block_id);
  if (st != PA_OK) return st;
  // the holder leaves the original; with refcount 1 this frees it
  if (--a->refcount[block_id] == 0) a->free_ids.push(block_id);
  return PA_OK;
}

pa_status pa_refcount(const pa_allocator* a, int32_t block_id, int32_t* refcount) {
  if (!a || !refcount) return pa::fail(PA_ERR_INVALID_ARG, "pa_refcount: null argument");
  if (block_id < 0 || static_cast<size_t>(block_id) >= a->refcount.size())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_refcount: block id outside the pool");
  *refcount = a->refcount[block_id];
  return PA_OK;
}

int64_t pa_num_free(const pa_allocator* a) {
  return a ? static_cast<int64_t>(a->free_ids.size()) : -1;
}

pa_status pa_append_tokens(pa_allocator* a, int32_t block_size, int32_t* block_table,
                           int32_t max_blocks, int32_t* context_len, int32_t num_new,
                           int32_t* slots, int32_t* cow_pairs, int32_t* num_cow) {
  if (!a || !block_table || !context_len || (num_new > 0 && !slots) || !num_cow)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_append_tokens: null argument");
  if (block_size <= 0 || max_blocks < 0 || num_new < 0 || *context_len < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_append_tokens: negative size");
  *num_cow = 0;
  for (int32_t i = 0; i < num_new; ++i) {
    const int64_t pos = *context_len;
    const int64_t logical = pos / block_size;
    if (pos % block_size == 0) {
      if (logical >= max_blocks)
        return pa::fail(PA_ERR_INVALID_ARG, "pa_append_tokens: block table is full");
      int32_t id = -1;
      pa_status st = take(a, &id);
      if (st != PA_OK) return st;
      block_table[logical] = id;
    } else {
      const int32_t tail = block_table[logical];
      if (!live(a, tail))
        return pa::fail(PA_ERR_INVALID_ARG, "pa_append_tokens: tail block is not allocated");
      if (a->refcount[tail] > 1) {
        if (!cow_pairs)
          return pa::fail(PA_ERR_INVALID_ARG, "pa_append_tokens: shared tail needs cow_pairs");
        int32_t fresh;
        pa_status st = pa_cow_block(a, tail, &fresh);
        if (st != PA_OK) return st;
        block_table[logical] = fresh;
        cow_pairs[2 * *num_cow] = tail;
        cow_pairs[2 * *num_cow + 1] = fresh;
        *num_cow += 1;
      }
    }
    const int64_t slot = static_cast<int64_t>(block_table[logical]) * block_size + pos % block_size;
    if (slot > INT32_MAX) return pa::fail(PA_ERR_INVALID_ARG, "pa_append_tokens: slot overflows int32");
    slots[i] = static_cast<int32_t>(slot);
    *context_len += 1;
  }
  return PA_OK;
}

pa_status pa_fork_table(pa_allocator* a, const int32_t* src_table, int32_t num_blocks,
                        int32_t* dst_table) {
  if (!a || (num_blocks > 0 && (!src_table || !dst_table)) || num_blocks < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_fork_table: bad argument");
  for (int32_t i = 0; i < num_blocks; ++i)
    if (!live(a, src_table[i])) return pa::fail(PA_ERR_INVALID_ARG, "pa_fork_table: block not allocated");
  for (int32_t i = 0; i < num_blocks; ++i) {
    a->refcount[src_table[i]] += 1;
    dst_table[i] = src_table[i];
  }
  return PA_OK;
}

pa_status pa_release_table(pa_allocator* a, const int32_t* block_table, int32_t num_blocks) {
  if (!a || (num_blocks > 0 && !block_table) || num_blocks < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_release_table: bad argument");
  for (int32_t i = 0; i < num_blocks; ++i)
    if (!live(a, block_table[i]))
      return pa::fail(PA_ERR_INVALID_ARG, "pa_release_table: block not allocated");
  for (int32_t i = 0; i < num_blocks; ++i) pa_free_block(a, block_table[i]);
  return PA_OK;
}

pa_status pa_find_shared_prefixes(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t num_seqs,
                                  int32_t block_size, int32_t min_shared_blocks,
                                  int32_t* group_offsets, int32_t* group_members,
                                  int32_t* group_blocks, int32_t* num_groups,
                                  int32_t* max_group_size, int32_t* max_shared_blocks) {
  if (num_seqs < 0 || block_size <= 0 || max_blocks_per_seq <= 0 || min_shared_blocks < 1)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_find_shared_prefixes: bad size");
  if (!group_offsets || !num_groups || !max_group_size || !max_shared_blocks ||
      (num_seqs > 0 && (!block_tables || !context_lens || !group_members || !group_blocks)))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_find_shared_prefixes: null argument");
  auto row = [&](int32_t s) { return block_tables + static_cast<int64_t>(s) * max_blocks_per_seq; };
  auto full_blocks = [&](int32_t s) {
    return std::min<int64_t>(max_blocks_per_seq, std::max(0, context_lens[s]) / block_size);
  };
  // candidates keyed by their first block, in order of first appearance
  std::unordered_map<int32_t, size_t> slot_of_key;
  std::vector<std::vector<int32_t>> cand;
  for (int32_t s = 0; s < num_seqs; ++s) {
    if (full_blocks(s) < min_shared_blocks) continue;
    const int32_t key = row(s)[0];
    auto it = slot_of_key.find(key);
    if (it == slot_of_key.end()) {
      slot_of_key.emplace(key, cand.size());
      cand.push_back({s});
    } else {
      cand[it->second].push_back(s);
    }
  }
  int32_t ng = 0, members = 0, max_size = 0, max_blocks = 0;
  group_offsets[0] = 0;
  for (const auto& c : cand) {
    if (c.size() < 2) continue;
    int64_t lcp = full_blocks(c[0]);
    const int32_t* r0 = row(c[0]);
    for (size_t i = 1; i < c.size(); ++i) {
      const int32_t* r = row(c[i]);
      const int64_t lim = std::min<int64_t>(lcp, full_blocks(c[i]));
      int64_t k = 0;
      while (k < lim && r[k] == r0[k]) ++k;
      lcp = k;
    }
    if (lcp < min_shared_blocks) continue;
    for (int32_t s : c) group_members[members++] = s;
    group_blocks[ng] = static_cast<int32_t>(lcp);
    group_offsets[ng + 1] = members;
    max_size = std::max<int32_t>(max_size, static_cast<int32_t>(c.size()));
    max_blocks = std::max<int32_t>(max_blocks, static_cast<int32_t>(lcp));
    ++ng;
  }
  *num_groups = ng;
  *max_group_size = max_size;
  *max_shared_blocks = max_blocks;
  return PA_OK;
}

pa_status pa_decode_slots(const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t num_seqs, int32_t block_size,
                          int32_t* slots) {
  if (num_seqs < 0 || block_size <= 0 || max_blocks_per_seq < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_slots: bad size");
  if (num_seqs > 0 && (!block_tables || !context_lens || !slots))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_slots: null argument");
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int64_t L = context_lens[s];
    if (L == 0) {
      slots[s] = -1;
      continue;
    }
    const int64_t pos = L - 1;
    if (L < 0 || pos / block_size >= max_blocks_per_seq)
      return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_slots: context length outside the table");
    const int64_t slot =
        static_cast<int64_t>(block_tables[static_cast<int64_t>(s) * max_blocks_per_seq + pos / block_size]) *
            block_size + pos % block_size;
    if (slot < 0 || slot > INT32_MAX)
      return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_slots: slot outside int32");
    slots[s] = static_cast<int32_t>(slot);
  }
  return PA_OK;
}

}  // extern "C"
