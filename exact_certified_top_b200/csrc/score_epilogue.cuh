// The head reduction of the indexer score, shared by every kernel that
// produces a final score (dense scorer, survivor rescoring, repair) so that
// they agree bit for bit: the same FMA sequence in the same order.
#pragma once

#include <cuda_runtime.h>

namespace dosa {

// Two independent fp32 FMAs in one instruction (fma.rn.f32x2, sm_100a): each
// lane is a correctly rounded fp32 FMA, identical to fmaf.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// sum_h w[h] * ReLU(x[h]) over 64 heads: four fp32 FMA chains (head h goes to
// chain h mod 4), combined as (c0 + c1) + (c2 + c3).  Chains (0,1) and (2,3)
// advance together as packed pairs.  x: 64 consecutive values (registers after
// inlining); w: 16-byte aligned, read through the read-only path (all lanes
// of a warp read the same address, so each load is a broadcast).
__device__ __forceinline__ float head_reduce64(const float* x, const float* __restrict__ w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
  float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 ww = __ldg(w4 + i);
    a = ffma2(make_float2(ww.x, ww.y),
              make_float2(fmaxf(x[4 * i + 0], 0.f), fmaxf(x[4 * i + 1], 0.f)), a);
    b = ffma2(make_float2(ww.z, ww.w),
              make_float2(fmaxf(x[4 * i + 2], 0.f), fmaxf(x[4 * i + 3], 0.f)), b);
  }
  return (a.x + a.y) + (b.x + b.y);
}

}  // namespace dosa
