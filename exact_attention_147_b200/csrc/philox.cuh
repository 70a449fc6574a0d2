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
// kept probabilities are scaled by 256 / (256 - t).  One generator call
// covers a 4 x 4 block of (query, key) pairs; the tensor-core kernels, whose
// threads each own one row, share every call across the four lanes that own
// the block's four rows (quad_transpose below), so each byte drawn is used.
#pragma once

#include <cstdint>

namespace fa2 {

constexpr int kPhiloxRounds = 10;

struct DropoutParams {
  uint32_t seed_lo, seed_hi;
  uint32_t threshold;   // t in [0, 255]
  float keep_scale;     // 256 / (256 - t)
  // The key of round r, (seed_lo + r 0x9E3779B9, seed_hi + r 0xBB67AE85) mod
  // 2^32: the same for every generator call of a launch, so it is formed
  // once on the host, and the rounds read it from the kernel's parameters.
  uint32_t rk0[kPhiloxRounds], rk1[kPhiloxRounds];
};

struct Philox4 {
  uint32_t w[4];
};

// One 32 x 32 -> 64-bit product gives both halves a round needs.
__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 const DropoutParams& dp) {
#pragma unroll
  for (int r = 0; r < kPhiloxRounds; ++r) {
    const uint64_t p0 = uint64_t(0xD2511F53u) * c0, p1 = uint64_t(0xCD9E8D57u) * c2;
    const uint32_t lo0 = uint32_t(p0), hi0 = uint32_t(p0 >> 32);
    const uint32_t lo1 = uint32_t(p1), hi1 = uint32_t(p1 >> 32);
    const uint32_t n0 = hi1 ^ c1 ^ dp.rk0[r], n2 = hi0 ^ c3 ^ dp.rk1[r];
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
  const Philox4 o = philox4x32_10(uint32_t(j4), uint32_t(i >> 2), uint32_t(h), uint32_t(b), dp);
  const int s = i & 3;
  return s == 0 ? o.w[0] : s == 1 ? o.w[1] : s == 2 ? o.w[2] : o.w[3];
}

// The four lanes 4q .. 4q+3 of a warp (a "quad") hold four consecutive query
// rows (or key rows) whose counters coincide, so one generator call serves
// the whole quad: each lane computes one call of four and the quad trades the
// results, instead of every lane computing all four and keeping a quarter.
//
// quad_transpose: lane s of the quad holds x[w] = the word it prepared for
// lane w; afterwards lane r holds z[c] = the word lane c prepared for lane r.
// Round u sends x[(s - u) mod 4] to the lane (s - u) mod 4, which reads it
// from lane (r + u) mod 4; z is the received words rotated into place.
// All 32 lanes of the warp must be active.
__device__ __forceinline__ uint32_t pick4(const uint32_t (&x)[4], int k) {
  const uint32_t lo = (k & 1) ? x[1] : x[0];
  const uint32_t hi = (k & 1) ? x[3] : x[2];
  return (k & 2) ? hi : lo;
}

__device__ __forceinline__ void quad_transpose(const uint32_t (&x)[4], uint32_t (&z)[4]) {
  const int lane = int(threadIdx.x & 31u);
  const int s = lane & 3, base = lane & ~3;
  uint32_t y[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t v = pick4(x, (s - u) & 3);
    y[u] = u == 0 ? v : __shfl_sync(0xffffffffu, v, base | ((s + u) & 3));
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) z[c] = pick4(y, (c - s) & 3);
}

// Random words of this lane's query row i for key groups j4_0 + c, c = 0..3
// (16 consecutive keys starting at 4 j4_0; z[c] holds keys 4(j4_0+c) ..
// 4(j4_0+c)+3 as bytes, least significant first).  j4_0 must be a multiple
// of 4 and the quad must hold rows i with i mod 4 = lane mod 4.
__device__ __forceinline__ void dropout_words_row16(const DropoutParams& dp, int b, int h, int i, int j4_0,
                                                    uint32_t (&z)[4]) {
  const int s = int(threadIdx.x & 3u);
  const Philox4 o = philox4x32_10(uint32_t(j4_0 + s), uint32_t(i >> 2), uint32_t(h), uint32_t(b), dp);
  // word w of call (j4_0 + s) belongs to row 4 (i / 4) + w, i.e. quad lane w
  quad_transpose(o.w, z);
}

// Random bytes of this lane's key row j for query groups i4_0 + c, c = 0..3
// (16 consecutive queries starting at 4 i4_0; z[c] holds queries
// 4(i4_0+c) .. 4(i4_0+c)+3 as bytes, least significant first).  i4_0 must be
// a multiple of 4 and the quad must hold keys j with j mod 4 = lane mod 4.
__device__ __forceinline__ void dropout_words_col16(const DropoutParams& dp, int b, int h, int j, int i4_0,
                                                    uint32_t (&z)[4]) {
  const int s = int(threadIdx.x & 3u);
  const Philox4 o = philox4x32_10(uint32_t(j >> 2), uint32_t(i4_0 + s), uint32_t(h), uint32_t(b), dp);
  // byte r of every word belongs to key 4 (j / 4) + r, i.e. quad lane r:
  // transpose the 4 x 4 bytes so that x[r] gathers byte r of words 0..3
  const uint32_t lo01 = __byte_perm(o.w[0], o.w[1], 0x5140), hi01 = __byte_perm(o.w[0], o.w[1], 0x7362);
  const uint32_t lo23 = __byte_perm(o.w[2], o.w[3], 0x5140), hi23 = __byte_perm(o.w[2], o.w[3], 0x7362);
  const uint32_t x[4] = {__byte_perm(lo01, lo23, 0x5410), __byte_perm(lo01, lo23, 0x7632),
                         __byte_perm(hi01, hi23, 0x5410), __byte_perm(hi01, hi23, 0x7632)};
  quad_transpose(x, z);
}

// 0x80 in every byte of `word` that is kept (byte >= threshold t), else 0x00,
// in three integer operations: d = (word | 0x80808080) - (t mod 128) * 0x01010101
// cannot borrow across bytes, and bit 7 of a byte of d says whether that
// byte's low seven bits are >= those of t; so the byte is >= t iff its bit 7
// or d's is set (t < 128), or both are (t >= 128).
__device__ __forceinline__ uint32_t dropout_keep_msb4(uint32_t word, uint32_t threshold) {
  const uint32_t d = (word | 0x80808080u) - (threshold & 0x7Fu) * 0x01010101u;
  return (threshold < 128u ? (word | d) : (word & d)) & 0x80808080u;
}

// Byte e (0..3) of a packed word kept?
__device__ __forceinline__ bool dropout_keep(uint32_t word, int e, uint32_t threshold) {
  return ((word >> (8 * e)) & 0xFFu) >= threshold;
}

}  // namespace fa2
