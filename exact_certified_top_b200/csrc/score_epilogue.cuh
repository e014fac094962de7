// The head reduction of the indexer score, shared by every kernel that
// produces a final score (dense scorer, survivor rescoring, repair) so that
// they agree bit for bit: the same FMA sequence in the same order.
#pragma once

#include <cuda_runtime.h>

namespace dosa {

// sum_h w[h] * ReLU(x[h]) over 64 heads: four interleaved fp32 FMA chains
// (head h goes to chain h mod 4), combined as (c0 + c1) + (c2 + c3).
// w: 16-byte aligned, read through the read-only path (every lane of a warp
// reads the same address, so each load is a broadcast).  Measured faster on
// B200 than a packed fma.rn.f32x2 form or an 8-chain form.  The reduction may
// be fed in two halves of 32 heads (head_accumulate32 on heads 0-31, then on
// heads 32-63): each chain sees the same FMAs in the same order, so the result
// is bit-identical to head_reduce64.
struct HeadAcc {
  float c0, c1, c2, c3;
};

__device__ __forceinline__ void head_accumulate32(HeadAcc& a, const float* x,
                                                  const float* __restrict__ w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 ww = __ldg(w4 + i);
    a.c0 = fmaf(ww.x, fmaxf(x[4 * i + 0], 0.f), a.c0);
    a.c1 = fmaf(ww.y, fmaxf(x[4 * i + 1], 0.f), a.c1);
    a.c2 = fmaf(ww.z, fmaxf(x[4 * i + 2], 0.f), a.c2);
    a.c3 = fmaf(ww.w, fmaxf(x[4 * i + 3], 0.f), a.c3);
  }
}

__device__ __forceinline__ float head_total(const HeadAcc& a) {
  return (a.c0 + a.c1) + (a.c2 + a.c3);
}

__device__ __forceinline__ float head_reduce64(const float* x, const float* __restrict__ w) {
  HeadAcc a = {0.f, 0.f, 0.f, 0.f};
  head_accumulate32(a, x, w);
  head_accumulate32(a, x + 32, w + 32);
  return head_total(a);
}

// The same reduction with two heads per packed add and FMA (add.rn.f32x2,
// fma.rn.f32x2).  y = x + |x| is exactly 2 ReLU(x), and doubling commutes with
// round-to-nearest (no overflow or subnormals at these magnitudes), so each
// chain holds exactly twice the chain of head_accumulate32 after every step
// and the halved total is bit-identical to head_total.  Fewer instructions, and no max on the ALU
// pipe: measured faster in the filter and certified scorers, slower in the
// dense scorer, which keeps the form above.
struct HeadAcc2 {
  float2 c01, c23;   // chains 0,1 and 2,3
};

__device__ __forceinline__ void head_accumulate32(HeadAcc2& a, const float* x,
                                                  const float* __restrict__ w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 ww = __ldg(w4 + i);
    const float2 y01 = __fadd2_rn(make_float2(x[4 * i + 0], x[4 * i + 1]),
                                  make_float2(fabsf(x[4 * i + 0]), fabsf(x[4 * i + 1])));
    const float2 y23 = __fadd2_rn(make_float2(x[4 * i + 2], x[4 * i + 3]),
                                  make_float2(fabsf(x[4 * i + 2]), fabsf(x[4 * i + 3])));
    a.c01 = __ffma2_rn(make_float2(ww.x, ww.y), y01, a.c01);
    a.c23 = __ffma2_rn(make_float2(ww.z, ww.w), y23, a.c23);
  }
}

// The same packed reduction with the weights in shared memory (broadcast
// reads; identical FMA sequence).
__device__ __forceinline__ void head_accumulate32_smem(HeadAcc2& a, const float* x,
                                                       const float* w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 ww = w4[i];
    const float2 y01 = __fadd2_rn(make_float2(x[4 * i + 0], x[4 * i + 1]),
                                  make_float2(fabsf(x[4 * i + 0]), fabsf(x[4 * i + 1])));
    const float2 y23 = __fadd2_rn(make_float2(x[4 * i + 2], x[4 * i + 3]),
                                  make_float2(fabsf(x[4 * i + 2]), fabsf(x[4 * i + 3])));
    a.c01 = __ffma2_rn(make_float2(ww.x, ww.y), y01, a.c01);
    a.c23 = __ffma2_rn(make_float2(ww.z, ww.w), y23, a.c23);
  }
}

// The packed reduction over 16 heads with their weights already in
// registers (same FMA sequence, chain by chain, as head_accumulate32 above).
__device__ __forceinline__ void load_w16(float4 (&w4)[4], const float* __restrict__ w) {
  const float4* p = reinterpret_cast<const float4*>(w);
#pragma unroll
  for (int i = 0; i < 4; ++i) w4[i] = __ldg(p + i);
}

__device__ __forceinline__ void head_accumulate16w(HeadAcc2& a, const float* x,
                                                   const float4 (&w4)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 ww = w4[i];
    const float2 y01 = __fadd2_rn(make_float2(x[4 * i + 0], x[4 * i + 1]),
                                  make_float2(fabsf(x[4 * i + 0]), fabsf(x[4 * i + 1])));
    const float2 y23 = __fadd2_rn(make_float2(x[4 * i + 2], x[4 * i + 3]),
                                  make_float2(fabsf(x[4 * i + 2]), fabsf(x[4 * i + 3])));
    a.c01 = __ffma2_rn(make_float2(ww.x, ww.y), y01, a.c01);
    a.c23 = __ffma2_rn(make_float2(ww.z, ww.w), y23, a.c23);
  }
}

__device__ __forceinline__ float head_total(const HeadAcc2& a) {
  return 0.5f * ((a.c01.x + a.c01.y) + (a.c23.x + a.c23.y));
}

__device__ __forceinline__ float head_reduce32_packed(const float* x, const float* __restrict__ w) {
  HeadAcc2 a = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  head_accumulate32(a, x, w);
  return head_total(a);
}

__device__ __forceinline__ float head_reduce64_packed(const float* x, const float* __restrict__ w) {
  HeadAcc2 a = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  head_accumulate32(a, x, w);
  head_accumulate32(a, x + 32, w + 32);
  return head_total(a);
}

}  // namespace dosa
