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

}  // namespace dosa
