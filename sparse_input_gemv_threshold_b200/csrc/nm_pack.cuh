// One thread's share of the packed 2:4 operand: 16 consecutive entries of a
// row (four blocks of four), packed to their kept values and the 16-bit
// metadata field they form.  N = 2 keeps the two largest |x| of every block
// of four (ties by lower position, NaN last); N = 1 keeps the largest and
// pads the second slot with +0 at the block's smallest other position.  The
// two slots are written in ascending position order (values, then positions
// as the metadata nibble p0 | p1 << 2, block q at bits 4 q).
//
// Metadata layout of a 128-row x 128-entry block (the order a 128x128b
// tensor-memory copy hands it to the sparse MMA): lane L = r % 8 + 8 h +
// 16 (r / 16) holds, for K group j (entries 32 j .. 32 j + 31), the 16 bits
// of row r's half h (entries 32 j + 16 h .. + 15) at bytes 4 j, 4 j + 1 when
// r % 16 < 8, else at bytes 4 j + 2, 4 j + 3.  Rows 32 c .. 32 c + 31 own
// lanes 32 c .. 32 c + 31, one contiguous 512-byte quarter of the block's
// 2048 bytes.
#pragma once

#include "common.cuh"
#include "nm_select.cuh"

namespace sig {

// Entries 16 part .. 16 part + 15 of a row (v0: the first eight, v1: the
// next eight) packed: `vals` receives the eight kept values, the return value
// the 16-bit metadata field.
template <int N>
__device__ __forceinline__ uint32_t pack_piece(const uint4& v0, const uint4& v1, uint4& vals) {
  uint32_t out[4];
  uint32_t nib = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // the block's four entries, entry j at bits 16 j
    const uint4& w = q < 2 ? v0 : v1;
    const uint64_t ev = (q & 1) ? ((uint64_t)w.w << 32 | w.z) : ((uint64_t)w.y << 32 | w.x);
    uint32_t comp[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)    // unique composites: position breaks ties
      comp[j] = (mag_key((uint16_t)(ev >> (16 * j))) << 2) | (uint32_t)(3 - j);
    const uint32_t top = select_top_n<4>(comp, N);            // the kept positions
    // N = 1: the second slot is the smallest position not kept
    const uint32_t slots = N == 2 ? top : top | ((top & 1u) ? 2u : 1u);
    const uint32_t p0 = (uint32_t)(__ffs(slots) - 1);
    const uint32_t p1 = (uint32_t)(31 - __clz(slots));
    const uint32_t lo = ((top >> p0) & 1u) ? (uint32_t)(ev >> (16 * p0)) & 0xffffu : 0u;  // padding: +0
    const uint32_t hi = ((top >> p1) & 1u) ? (uint32_t)(ev >> (16 * p1)) & 0xffffu : 0u;
    out[q] = lo | (hi << 16);
    nib |= (p0 | (p1 << 2)) << (4 * q);
  }
  vals = make_uint4(out[0], out[1], out[2], out[3]);
  return nib;
}

// Byte offset, inside the 512-byte metadata quarter of rows 32 c .. 32 c + 31
// of a 128-row block (c = (r / 32) % 4), of the field of row r's entries
// 16 part .. 16 part + 15 of a 128-entry block.
__device__ __forceinline__ uint32_t meta_quarter_offset(int r, int part) {
  const int j = part >> 1, h = part & 1;
  const int r128 = r & 127;                                   // row inside the 128-row block
  const int L = (r128 & 7) + 8 * h + 16 * (r128 >> 4);        // in [32 c, 32 c + 32)
  return (uint32_t)((L & 31) * 16 + 4 * j + 2 * ((r128 >> 3) & 1));
}

}  // namespace sig
