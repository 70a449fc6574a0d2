// Memory-bound row kernels of the backward pass:
//   bwd_preprocess : D[b,h,i] = sum_c dO[b,i,h,c] * O[b,i,h,c]   (fp32)
//   dq_convert     : dQ[b,i,h,:] = scale * dQaccum[b,h,i,:] cast to bf16 (or
//                    the sum of two accumulators, in a fixed order)
// Each row of d elements is read by a group of lanes with 16-byte vector
// loads (d * element size / 16 lanes per row), so every warp touches whole
// 32-byte sectors; rows are ordered with i fastest so the fp32 [B,H,N]
// vectors are written contiguously.
#pragma once

#include <cuda_bf16.h>

#include "attn_common.cuh"

namespace fa2 {

template <int L>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float dot16(const uint4& a, const uint4& b, __nv_bfloat16) {
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 fx = __bfloat1622float2(x[e]);
    const float2 fy = __bfloat1622float2(y[e]);
    s = fmaf(fx.x, fy.x, s);
    s = fmaf(fx.y, fy.y, s);
  }
  return s;
}

__device__ __forceinline__ float dot16(const uint4& a, const uint4& b, float) {
  return __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
         __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
}

// 256 threads; L lanes per row; grid = ceil(B*H*N / (256 / L)).
template <typename T, int HD>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const AttnArgs a) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int L = HD / VEC;          // lanes per row (<= 32)
  static_assert(L >= 1 && L <= 32 && (32 % L) == 0, "row split");
  const long long rows = (long long)a.B * a.H * a.N;
  const long long R = (long long)blockIdx.x * (256 / L) + threadIdx.x / L;
  const int li = threadIdx.x % L;
  float s = 0.f;
  if (R < rows) {
    const int n = int(R % a.N);
    const long long bh = R / a.N;
    const int h = int(bh % a.H), b = int(bh / a.H);
    const T* o = static_cast<const T*>(a.o) + b * a.so.b + (long long)n * a.so.n + h * a.so.h;
    const T* g = static_cast<const T*>(a.dout) + b * a.sdo.b + (long long)n * a.sdo.n + h * a.sdo.h;
    const uint4 vo = *reinterpret_cast<const uint4*>(o + li * VEC);
    const uint4 vg = *reinterpret_cast<const uint4*>(g + li * VEC);
    s = dot16(vo, vg, T());
  }
  s = group_sum<L>(s);
  if (R < rows && li == 0) const_cast<float*>(a.dvec)[R] = s;
}

// dQaccum (fp32, [B,H,N,d] dense) -> dQ (bf16, strided [B,N,H,d]).  With
// NACC = 2 the workspace holds two such accumulators back to back (the
// ordered deterministic backward's even and odd key blocks), added here in
// that fixed order.
template <int HD, int NACC = 1>
__global__ void __launch_bounds__(256) dq_convert_kernel(const AttnArgs a) {
  constexpr int L = HD / 4;  // lanes per row, 4 floats each
  const long long rows = (long long)a.B * a.H * a.N;
  const long long R = (long long)blockIdx.x * (256 / L) + threadIdx.x / L;
  const int li = threadIdx.x % L;
  if (R >= rows) return;
  const int n = int(R % a.N);
  const long long bh = R / a.N;
  const int h = int(bh % a.H), b = int(bh / a.H);
  float4 v = *reinterpret_cast<const float4*>(a.dq_accum + R * HD + li * 4);
  if (NACC == 2) {
    const float4 w2 = *reinterpret_cast<const float4*>(a.dq_accum + (rows + R) * HD + li * 4);
    v = make_float4(v.x + w2.x, v.y + w2.y, v.z + w2.z, v.w + w2.w);
  }
  __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(a.dq) + b * a.sdq.b + (long long)n * a.sdq.n +
                      h * a.sdq.h + li * 4;
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * a.scale, v.y * a.scale);
  __nv_bfloat162 hi = __floats2bfloat162_rn(v.z * a.scale, v.w * a.scale);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dq) = w;
}

}  // namespace fa2
