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

// One thread per 16-byte chunk of every new row (K and V), grid-stride, so a
// small batch of tokens still puts enough copies in flight.
// row_chunks = head_dim * elem_bytes / 16.  k_new/v_new: [T][H][row_chunks]
// chunks; pools: [NB][H][16][row_chunks].
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                             const int32_t* __restrict__ slot_mapping, uint4* __restrict__ k_pool,
                             uint4* __restrict__ v_pool, int heads, int row_chunks,
                             int64_t num_tokens, int64_t num_slots, uint32_t* err) {
  const int64_t per_token = (int64_t)heads * row_chunks;
  const int64_t total = num_tokens * per_token;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t rem = i - t * per_token;
    const int32_t slot = slot_mapping[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (rem == 0) atomicOr(err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t h = rem / row_chunks, c = rem - h * row_chunks;
    const int64_t blk = slot / 16, off = slot % 16;
    const int64_t dst = ((blk * heads + h) * 16 + off) * row_chunks + c;
    k_pool[dst] = k_new[i];
    v_pool[dst] = v_new[i];
  }
}

// One thread per 16-byte chunk of every (src, dst) block pair, grid-stride.
// block_chunks = heads * 16 * head_dim * elem_bytes / 16.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                       const int32_t* __restrict__ pairs, int64_t num_pairs, int64_t num_blocks,
                       int64_t block_chunks, uint32_t* err) {
  const int64_t total = num_pairs * block_chunks;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t pr = i / block_chunks;
    const int64_t c = i - pr * block_chunks;
    const int32_t src = pairs[2 * pr], dst = pairs[2 * pr + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (c == 0) atomicOr(err, PA_DEVERR_PAIR);
      continue;
    }
    k_pool[(int64_t)dst * block_chunks + c] = k_pool[(int64_t)src * block_chunks + c];
    v_pool[(int64_t)dst * block_chunks + c] = v_pool[(int64_t)src * block_chunks + c];
  }
}

}  // namespace pa
