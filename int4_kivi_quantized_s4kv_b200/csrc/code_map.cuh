// Where a (token, channel) code sits in a page block, for every code width:
// the position the int4 layout gives it as (32-bit word, nibble) of the
// MMA-fragment order, and the byte (8-bit) or bit pair (2-bit) that holds the
// same fragment place in the wider or narrower block.  Used by the batched
// dequantization and the prefill operand tiles of 8- and 2-bit caches.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace s4kv {

// The code at 4-bit position (word, nibble): that nibble, or with 8-bit
// codes the byte holding the same fragment place (tile 4*(word/128) +
// word%4, lane (word/4)%32, register reg_of_nibble(nibble), half
// half_of_nibble(nibble)), or with 2-bit codes the bit pair holding it.
__device__ __forceinline__ uint32_t code_at(const uint8_t *region, int word, int nibble, int bits) {
  const int r = reg_of_nibble(nibble), e = half_of_nibble(nibble);
  if (bits == 8) {
    const int tile = 4 * (word >> 7) + (word & 3), lane = (word >> 2) & 31;
    return region[((tile >> 1) * 32 + lane) * 16 + (tile & 1) * 8 + 2 * r + e];
  }
  if (bits == 2) {
    const int tile = 4 * (word >> 7) + (word & 3), lane = (word >> 2) & 31;
    const uint32_t w = reinterpret_cast<const uint32_t *>(region)[4 * lane + (tile >> 1)];
    return (w >> (16 * e + 2 * (4 * (tile & 1) + r))) & 3u;
  }
  const uint32_t w = reinterpret_cast<const uint32_t *>(region)[word];
  return (w >> (4 * nibble)) & 0xFu;
}

// (word, nibble) of key (token t, channel c) and of value (token t, channel
// c) in the int4 fragment order.
__device__ __forceinline__ void key_position(int t, int c, int &word, int &nibble) {
  const int ki = c >> 5, kt = (c & 31) >> 2, ke = c & 3;
  word = 128 * (kt >> 2) + 4 * (4 * (t & 7) + ki) + (kt & 3);
  nibble = nibble_of((t >> 3) + 2 * (ke >> 1), ke & 1);
}
__device__ __forceinline__ void value_position(int t, int c, int &word, int &nibble) {
  const int vn = (c & 31) >> 2, ve = c & 3, vm = 2 * (c >> 5) + (ve >> 1);
  word = 128 * (vm >> 2) + 4 * (4 * vn + ((t & 7) >> 1)) + (vm & 3);
  nibble = nibble_of((ve & 1) + 2 * (t >> 3), t & 1);
}

// Slot of channel c's key zero point (stored in MMA k order).
__host__ __device__ __forceinline__ int key_zero_slot(int c) {
  return 16 * ((c & 31) >> 2) + 2 * (c >> 5) + (c & 1) + 8 * ((c & 3) >> 1);
}

}  // namespace s4kv
