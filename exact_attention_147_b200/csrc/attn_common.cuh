// Argument block, sequence views and mask helpers shared by the attention
// kernels.
#pragma once

#include <cstdint>

#include "philox.cuh"
#include "status.cuh"

namespace fa2 {

// Layout modes of the tensor-core kernels (template argument MODE).
constexpr int kLayoutPadded = 0;   // [B, N, H, d]
constexpr int kLayoutPacked = 1;   // [total, H, d] with cu_seqlens
constexpr int kLayoutSparse = 2;   // [B, N, H, d] with a 128 x 128 block mask

struct Strides {
  int64_t b, n, h;  // element strides of a [B, N, H, d] tensor (d stride 1)
};

// Everything a kernel needs about one call.  Masks are normalised on the
// host: `wl` / `wr` are the inclusive window bounds (negative = unbounded)
// with `causal` folded in as wr = 0.
//
// Two layouts share these fields:
//   padded    : B sequences of N rows each, tensors [B, N, H, d], row
//               statistics (LSE, D) [B, H, N];  cu_seqlens == nullptr.
//   packed    : B sequences of different lengths stored back to back,
//               tensors [total, H, d] (the b strides are unused), row
//               statistics [H, total]; sequence b owns rows
//               [cu_seqlens[b], cu_seqlens[b+1]) and N is the longest
//               length (it sizes the grids).
// Rows are addressed through a SeqView (below), which hides the difference.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  void* o;
  void* dq;
  void* dk;
  void* dv;
  float* lse;         // row statistics, layout above
  const float* dvec;  // D = rowsum(dO o O), same layout as lse
  const float* alibi; // [H] or null
  float* dq_accum;    // fp32 [B*H, N, d] (padded) or [H, total, d] (packed) workspace
  const int* cu_seqlens;  // [B + 1] device offsets (packed) or null (padded)
  int total;          // packed: rows of the tensors; padded: unused
  const uint8_t* block_mask;  // [B, H, nb, nb] 128 x 128 block mask (padded only) or null
  int64_t bm_sb, bm_sh;       // its batch and head strides in elements; rows hold nb bytes
  Strides sq, sk, sv, so, sdo, sdq, sdk, sdv;
  int B, N, H, d;
  float scale;        // softmax scale
  int wl, wr;         // window bounds, negative = unbounded
  int dropout;        // nonzero: apply the dropout mask described in philox.cuh
  DropoutParams drop;
  float descale_qk;   // e4m3 inputs: q_descale * k_descale (else 1)
  float descale_v;    // e4m3 inputs: v_descale (else 1)
};

// One sequence of a call: batch coordinate `bt` and first row `row0` of its
// rows in the tensors, and its length.  Row i (0 <= i < len) of sequence b is
// tensor row (bt, row0 + i); its statistics live at
//   (bt * H + h) * stat_rows + row0 + i,   stat_rows = N (padded) or total.
// Masks, ALiBi distances and dropout counters all use the local index i, so a
// sequence of a packed call computes exactly what a padded call with that
// sequence alone at batch index b computes.
struct SeqView {
  int bt, row0, len;
};

// Offsets are clamped into [0, total] and the length to N before any use, so
// a malformed cu_seqlens cannot move an access outside the tensors; such an
// input is recorded in the device status word.
__device__ __forceinline__ SeqView seq_view(const int* cu, int b, int N, int total) {
  SeqView s;
  if (cu == nullptr) {
    s.bt = b;
    s.row0 = 0;
    s.len = N;
    return s;
  }
  const int c0 = __ldg(cu + b), c1 = __ldg(cu + b + 1);
  const int r0 = min(max(c0, 0), total);
  const int r1 = min(max(c1, r0), total);
  int len = r1 - r0;
  if (len > N) len = N;
  if (r0 != c0 || r1 != c1 || len != r1 - r0) atomicCAS(&g_fa2_device_status, 0, SITE_BAD_SEQLENS);
  s.bt = 0;
  s.row0 = r0;
  s.len = len;
  return s;
}

// Counter-scheduled calls (work items taken from a shared counter pair
// {next item, finished CTAs}): each CTA calls this once, from one thread,
// when it takes no further item -- including a CTA that stops before taking
// any -- and the call's last CTA returns the pair to zero.
__device__ __forceinline__ void sched_cta_done(unsigned int* sched) {
  __threadfence();
  if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
    sched[0] = 0u;
    sched[1] = 0u;
    __threadfence();
  }
}

// Element pointer of row i, head h of a [B, N, H, d] / [total, H, d] tensor.
template <typename T, typename P>
__device__ __forceinline__ T* row_ptr(P* base, const Strides& s, const SeqView& v, int i, int h) {
  return static_cast<T*>(base) + v.bt * s.b + int64_t(v.row0 + i) * s.n + h * s.h;
}

// Index of row i, head h in the row-statistics vectors (LSE, D).
__device__ __forceinline__ size_t stat_index(const AttnArgs& a, const SeqView& v, int h, int i) {
  const int rows = a.cu_seqlens ? a.total : a.N;
  return (size_t(v.bt) * a.H + h) * size_t(rows) + size_t(v.row0 + i);
}

// Block mask: may query i see key j at all?  (nb = ceil(N / 128).)
__device__ __forceinline__ bool block_kept(const AttnArgs& a, int b, int h, int i, int j) {
  if (a.block_mask == nullptr) return true;
  const int64_t nb = (a.N + 127) / 128;
  return a.block_mask[b * a.bm_sb + h * a.bm_sh + (i >> 7) * nb + (j >> 7)] != 0;
}

// Keys visible to query i of a sequence of n rows lie in [visible_lo,
// visible_hi] ("FlashAttention v2" article, §5.1: causal and
// window_size=(left, right); inclusive bounds are the reading taken).
__host__ __device__ __forceinline__ int visible_lo(const AttnArgs& a, int i) {
  return a.wl >= 0 ? (i - a.wl > 0 ? i - a.wl : 0) : 0;
}
__host__ __device__ __forceinline__ int visible_hi(const AttnArgs& a, int i, int n) {
  return a.wr >= 0 ? (i + a.wr < n - 1 ? i + a.wr : n - 1) : n - 1;
}
// Queries that see key j lie in [queries_lo, queries_hi].
__host__ __device__ __forceinline__ int queries_lo(const AttnArgs& a, int j) {
  return a.wr >= 0 ? (j - a.wr > 0 ? j - a.wr : 0) : 0;
}
__host__ __device__ __forceinline__ int queries_hi(const AttnArgs& a, int j, int n) {
  return a.wl >= 0 ? (j + a.wl < n - 1 ? j + a.wl : n - 1) : n - 1;
}

}  // namespace fa2
