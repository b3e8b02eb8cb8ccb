// Tiled tensor copies (TMA with a tensor map) and the 128-byte swizzle they
// write, shared by the kernels that stage K/V tiles for the tensor cores.
// No multicast: every copy reads this GPU's memory into this CTA.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace pa {

// 2-D tiled tensor copy global -> shared, completing its bytes on `bar`.  x is
// the innermost coordinate (elements; x * element size must be a multiple of
// 16 bytes), y the row.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile whose
// rows are 128 bytes (64 fp16/bf16 elements).  TMA copies with 128-byte
// swizzle produce this placement for boxes that start 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

}  // namespace pa
