// Base-3 decode shared by the decode GEMV and the transposed product.
#pragma once

#include <cstdint>

namespace tern {

// Base-3 word (bytes b0..b3, each sum_i c_i 3^i with c = t + 1) -> 10 registers: o[5h + i] holds the
// two's-complement field of t for digit 4 - i of byte h at bits 14..15 and for the same digit of byte
// 2 + h at bits 30..31, every other bit zero (so each half is the fp16 value 2t, and o & 0xC0000000 or
// o << 16 is the fp32 value 2t). Bytes (0, 2) and (1, 3) sit in 16-bit lanes V; with k0 =
// 130 | 130 << 16 + 0xC000C000, R = V * 202 + k0 maps each byte v to r = floor(R / 64) in
// [256 v / 81, 256 (v + 1) / 81), so bits 14..15 hold the leading digit and bits 6..13 a scaled
// remainder; "times three" steps give the following digits the same way, and the 0xC000 per lane
// turns digit c into the field of t = c - 1. Checked exhaustively over all byte pairs (the carry one
// lane passes to the other only touches bits that are masked or already garbage); an invalid byte
// (> 242) gives unspecified fields.
__device__ __forceinline__ void dec_t3_word(uint32_t w, uint32_t k0, uint32_t (&o)[10]) {
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const uint32_t V = h ? __byte_perm(w, 0u, 0x4341) : (w & 0x00FF00FFu);
    uint32_t R = V * 202u + k0;
    o[5 * h] = R & 0xC000C000u;
    R = (R & 0x3FC03FC0u) * 3u + 0xC000C000u;
    o[5 * h + 1] = R & 0xC000C000u;
#pragma unroll
    for (int i = 2; i < 5; i++) {
      R = (R - o[5 * h + i - 1]) * 3u + 0xC000C000u;
      o[5 * h + i] = R & 0xC000C000u;
    }
  }
}

}  // namespace tern
