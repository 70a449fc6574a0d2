// Counter-based random bytes for attention dropout.
//
// Generator: Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011): ten rounds over a 128-bit counter
// with a 64-bit key; a round multiplies words 0 and 2 by 0xD2511F53 and
// 0xCD9E8D57 (full 64-bit products) and returns
//     (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0),
// and the key is bumped by (0x9E3779B9, 0xBB67AE85) between rounds.
//
// Dropout scheme of this library: the random byte of element (b, h, query i,
// key j) is byte (j mod 4) (least significant first) of output word (i mod 4)
// of Philox4x32-10 with counter (j / 4, i / 4, h, b) and key (seed low,
// seed high).  The element is kept iff its byte is >= t = round(256 p), and
// kept probabilities are scaled by 256 / (256 - t).  A query row therefore
// gets four keys per generator call and a key row four queries.
#pragma once

#include <cstdint>

namespace fa2 {

struct DropoutParams {
  uint32_t seed_lo, seed_hi;
  uint32_t threshold;   // t in [0, 255]
  float keep_scale;     // 256 / (256 - t)
};

struct Philox4 {
  uint32_t w[4];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  Philox4 out;
  out.w[0] = c0;
  out.w[1] = c1;
  out.w[2] = c2;
  out.w[3] = c3;
  return out;
}

// Four random bytes (keys 4*j4 .. 4*j4+3) of query row i, packed in a word.
__device__ __forceinline__ uint32_t dropout_word_row(const DropoutParams& dp, int b, int h, int i, int j4) {
  const Philox4 o = philox4x32_10(uint32_t(j4), uint32_t(i >> 2), uint32_t(h), uint32_t(b), dp.seed_lo,
                                  dp.seed_hi);
  const int s = i & 3;
  return s == 0 ? o.w[0] : s == 1 ? o.w[1] : s == 2 ? o.w[2] : o.w[3];
}

// Byte e (0..3) of a packed word kept?
__device__ __forceinline__ bool dropout_keep(uint32_t word, int e, uint32_t threshold) {
  return ((word >> (8 * e)) & 0xFFu) >= threshold;
}

}  // namespace fa2
