// CUDA-core (SIMT) attention kernels, one warp per row, full fp32
// arithmetic.  They serve the fp32 data type, whose 1e-4 error budget the
// bf16 tensor-core path cannot meet, and they compute the same quantities as
// the tensor-core kernels:
//   forward  : online softmax over the visible keys of one query row
//              (running max, running sum, running output, rescaled when
//              the max grows -- the explainer "AI基础 | Flash Attention",
//              "Online softmax" section), O normalised once at the end;
//   backward : probabilities recomputed from q, k and the saved LSE
//              ("Backward pass" section of the same page), then the
//              softmax/matmul gradients, with dK/dV owned by a key-row warp
//              and dQ by a query-row warp, so no atomics are needed.
// Lane l owns head-dimension elements c = l + 32 e, e < d / 32.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "attn_common.cuh"

namespace fa2 {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Forward: grid (ceil(N / 4), H, B), 128 threads; warp w handles query row
// 4 * blockIdx.x + w.
template <typename T, int HD>
__global__ void __launch_bounds__(128) simt_fwd_kernel(const AttnArgs a) {
  constexpr int E = HD / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const SeqView sv = seq_view(a.cu_seqlens, b, a.N, a.total);
  if (i >= sv.len) return;
  const T* q = row_ptr<const T>(a.q, a.sq, sv, i, h);
  const T* kb = row_ptr<const T>(a.k, a.sk, sv, 0, h);
  const T* vb = row_ptr<const T>(a.v, a.sv, sv, 0, h);
  float qr[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qr[e] = to_f(q[lane + 32 * e]);
    acc[e] = 0.f;
  }
  const int lo = visible_lo(a, i), hi = visible_hi(a, i, sv.len);
  const float slope = a.alibi ? a.alibi[h] : 0.f;
  float m = -CUDART_INF_F, l = 0.f;
  for (int j = lo; j <= hi; ++j) {
    if (!block_kept(a, b, h, i, j)) continue;
    const T* kr = kb + j * a.sk.n;
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) part = fmaf(qr[e], to_f(kr[lane + 32 * e]), part);
    float s = warp_sum(part) * a.scale;
    if (a.alibi) s -= slope * fabsf(float(i - j));
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);   // 0 on the first visible key
    const float p = expf(s - m_new);
    l = l * alpha + p;                      // the un-dropped sum
    float pk = p;
    if (a.dropout) {
      const uint32_t word = dropout_word_row(a.drop, b, h, i, j >> 2);
      pk = dropout_keep(word, j & 3, a.drop.threshold) ? p * a.drop.keep_scale : 0.f;
    }
    const T* vr = vb + j * a.sv.n;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(pk, to_f(vr[lane + 32 * e]), acc[e] * alpha);
    m = m_new;
  }
  T* o = row_ptr<T>(a.o, a.so, sv, i, h);
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) o[lane + 32 * e] = from_f<T>(acc[e] * inv);
  if (lane == 0) a.lse[stat_index(a, sv, h, i)] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
}

// dK, dV: warp per key row j; loops over the queries that see key j.
template <typename T, int HD>
__global__ void __launch_bounds__(128) simt_bwd_dkdv_kernel(const AttnArgs a) {
  constexpr int E = HD / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int j = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const SeqView sv = seq_view(a.cu_seqlens, b, a.N, a.total);
  if (j >= sv.len) return;
  const T* kr = row_ptr<const T>(a.k, a.sk, sv, j, h);
  const T* vr = row_ptr<const T>(a.v, a.sv, sv, j, h);
  const T* qb = row_ptr<const T>(a.q, a.sq, sv, 0, h);
  const T* dob = row_ptr<const T>(a.dout, a.sdo, sv, 0, h);
  const float* lse = a.lse + stat_index(a, sv, h, 0);
  const float* dvec = a.dvec + stat_index(a, sv, h, 0);
  float kf[E], vf[E], dk[E], dv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kf[e] = to_f(kr[lane + 32 * e]);
    vf[e] = to_f(vr[lane + 32 * e]);
    dk[e] = dv[e] = 0.f;
  }
  const float slope = a.alibi ? a.alibi[h] : 0.f;
  // queries i that see key j: lo(i) <= j <= hi(i)
  const int i_lo = queries_lo(a, j), i_hi = queries_hi(a, j, sv.len);
  for (int i = i_lo; i <= i_hi; ++i) {
    if (!block_kept(a, b, h, i, j)) continue;
    const T* qr = qb + i * a.sq.n;
    const T* dor = dob + i * a.sdo.n;
    float qf[E], df[E], ps = 0.f, pd = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qf[e] = to_f(qr[lane + 32 * e]);
      df[e] = to_f(dor[lane + 32 * e]);
      ps = fmaf(qf[e], kf[e], ps);
      pd = fmaf(df[e], vf[e], pd);
    }
    float s = warp_sum(ps) * a.scale;
    if (a.alibi) s -= slope * fabsf(float(i - j));
    float dp = warp_sum(pd);
    const float p = expf(s - lse[i]);
    float pk = p;
    if (a.dropout) {
      const uint32_t word = dropout_word_row(a.drop, b, h, i, j >> 2);
      const float km = dropout_keep(word, j & 3, a.drop.threshold) ? a.drop.keep_scale : 0.f;
      pk = p * km;
      dp *= km;
    }
    const float ds = p * (dp - dvec[i]);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dv[e] = fmaf(pk, df[e], dv[e]);
      dk[e] = fmaf(ds, qf[e], dk[e]);
    }
  }
  T* dkr = row_ptr<T>(a.dk, a.sdk, sv, j, h);
  T* dvr = row_ptr<T>(a.dv, a.sdv, sv, j, h);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    dkr[lane + 32 * e] = from_f<T>(dk[e] * a.scale);
    dvr[lane + 32 * e] = from_f<T>(dv[e]);
  }
}

// dQ: warp per query row i; loops over the keys row i sees.
template <typename T, int HD>
__global__ void __launch_bounds__(128) simt_bwd_dq_kernel(const AttnArgs a) {
  constexpr int E = HD / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const SeqView sv = seq_view(a.cu_seqlens, b, a.N, a.total);
  if (i >= sv.len) return;
  const T* qr = row_ptr<const T>(a.q, a.sq, sv, i, h);
  const T* dor = row_ptr<const T>(a.dout, a.sdo, sv, i, h);
  const T* kb = row_ptr<const T>(a.k, a.sk, sv, 0, h);
  const T* vb = row_ptr<const T>(a.v, a.sv, sv, 0, h);
  const float lse_i = a.lse[stat_index(a, sv, h, i)];
  const float d_i = a.dvec[stat_index(a, sv, h, i)];
  float qf[E], df[E], dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qf[e] = to_f(qr[lane + 32 * e]);
    df[e] = to_f(dor[lane + 32 * e]);
    dq[e] = 0.f;
  }
  const float slope = a.alibi ? a.alibi[h] : 0.f;
  const int lo = visible_lo(a, i), hi = visible_hi(a, i, sv.len);
  for (int j = lo; j <= hi; ++j) {
    if (!block_kept(a, b, h, i, j)) continue;
    const T* kr = kb + j * a.sk.n;
    const T* vr = vb + j * a.sv.n;
    float kf[E], ps = 0.f, pd = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kf[e] = to_f(kr[lane + 32 * e]);
      ps = fmaf(qf[e], kf[e], ps);
      pd = fmaf(df[e], to_f(vr[lane + 32 * e]), pd);
    }
    float s = warp_sum(ps) * a.scale;
    if (a.alibi) s -= slope * fabsf(float(i - j));
    float dp = warp_sum(pd);
    const float p = expf(s - lse_i);
    if (a.dropout) {
      const uint32_t word = dropout_word_row(a.drop, b, h, i, j >> 2);
      dp *= dropout_keep(word, j & 3, a.drop.threshold) ? a.drop.keep_scale : 0.f;
    }
    const float ds = p * (dp - d_i);
#pragma unroll
    for (int e = 0; e < E; ++e) dq[e] = fmaf(ds, kf[e], dq[e]);
  }
  T* dqr = row_ptr<T>(a.dq, a.sdq, sv, i, h);
#pragma unroll
  for (int e = 0; e < E; ++e) dqr[lane + 32 * e] = from_f<T>(dq[e] * a.scale);
}

}  // namespace fa2
