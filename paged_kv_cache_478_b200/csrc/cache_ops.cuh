// Cache maintenance kernels: write new tokens into their slots, and copy
// whole blocks for copy-on-write.  Both are bit copies in 16-byte chunks.
//
// "Atención paginada en modelos de lenguaje grandes (LLM)" (7minutos.es),
// section 2: a new token's K/V goes into the tail page of its request;
// section 3: cow_copy() gives a writer a private copy of a shared page.
#pragma once

#include <stdint.h>

#include "pagedattn.h"

namespace pa {

// One CTA per new token.  row_chunks = head_dim * elem_bytes / 16.
// k_new/v_new: [T][H][row_chunks] chunks; pools: [NB][H][16][row_chunks].
__global__ void __launch_bounds__(128)
    reshape_and_cache_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                             const int32_t* __restrict__ slot_mapping, uint4* __restrict__ k_pool,
                             uint4* __restrict__ v_pool, int heads, int row_chunks,
                             int64_t num_slots, uint32_t* err) {
  const int t = blockIdx.x;
  const int32_t slot = slot_mapping[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (threadIdx.x == 0) atomicOr(err, PA_DEVERR_SLOT);
    return;
  }
  const int64_t blk = slot / 16, off = slot % 16;
  const int n = heads * row_chunks;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int h = i / row_chunks, c = i % row_chunks;
    const int64_t dst = ((blk * heads + h) * 16 + off) * row_chunks + c;
    const int64_t src = (int64_t)t * n + i;
    k_pool[dst] = k_new[src];
    v_pool[dst] = v_new[src];
  }
}

// grid (num_pairs, split): CTA y of pair x copies its 1/split share of the
// block (block_chunks 16-byte chunks) for K and for V.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                       const int32_t* __restrict__ pairs, int64_t num_blocks,
                       int64_t block_chunks, uint32_t* err) {
  const int32_t src = pairs[2 * blockIdx.x], dst = pairs[2 * blockIdx.x + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, PA_DEVERR_PAIR);
    return;
  }
  const int64_t per = (block_chunks + gridDim.y - 1) / gridDim.y;
  const int64_t lo = blockIdx.y * per;
  const int64_t hi = min(block_chunks, lo + per);
  const uint4* ks = k_pool + (int64_t)src * block_chunks;
  const uint4* vs = v_pool + (int64_t)src * block_chunks;
  uint4* kd = k_pool + (int64_t)dst * block_chunks;
  uint4* vd = v_pool + (int64_t)dst * block_chunks;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    kd[i] = ks[i];
    vd[i] = vs[i];
  }
}

}  // namespace pa
