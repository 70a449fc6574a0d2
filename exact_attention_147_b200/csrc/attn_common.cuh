// Argument block and mask helpers shared by the attention kernels.
#pragma once

#include <cstdint>

#include "philox.cuh"

namespace fa2 {

struct Strides {
  int64_t b, n, h;  // element strides of a [B, N, H, d] tensor (d stride 1)
};

// Everything a kernel needs about one call.  Masks are normalised on the
// host: `wl` / `wr` are the inclusive window bounds (negative = unbounded)
// with `causal` folded in as wr = 0.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  void* o;
  void* dq;
  void* dk;
  void* dv;
  float* lse;         // [B, H, N]
  const float* dvec;  // D = rowsum(dO o O), [B, H, N]
  const float* alibi; // [H] or null
  float* dq_accum;    // fp32 [B, H, N, d] workspace (bf16 backward)
  Strides sq, sk, sv, so, sdo, sdq, sdk, sdv;
  int B, N, H, d;
  float scale;        // softmax scale
  int wl, wr;         // window bounds, negative = unbounded
  int dropout;        // nonzero: apply the dropout mask described in philox.cuh
  DropoutParams drop;
};

// Keys visible to query i lie in [visible_lo, visible_hi] ("FlashAttention
// v2" article, §5.1: causal and window_size=(left, right); inclusive bounds
// are the reading taken).
__host__ __device__ __forceinline__ int visible_lo(const AttnArgs& a, int i) {
  return a.wl >= 0 ? (i - a.wl > 0 ? i - a.wl : 0) : 0;
}
__host__ __device__ __forceinline__ int visible_hi(const AttnArgs& a, int i) {
  return a.wr >= 0 ? (i + a.wr < a.N - 1 ? i + a.wr : a.N - 1) : a.N - 1;
}
// Queries that see key j lie in [queries_lo, queries_hi].
__host__ __device__ __forceinline__ int queries_lo(const AttnArgs& a, int j) {
  return a.wr >= 0 ? (j - a.wr > 0 ? j - a.wr : 0) : 0;
}
__host__ __device__ __forceinline__ int queries_hi(const AttnArgs& a, int j) {
  return a.wl >= 0 ? (j + a.wl < a.N - 1 ? j + a.wl : a.N - 1) : a.N - 1;
}

}  // namespace fa2
