// The head reduction of the indexer score, shared by every kernel that
// produces a final score (dense scorer, survivor rescoring, repair) so that
// they agree bit for bit: the same FMA sequence in the same order.
#pragma once

#include <cuda_runtime.h>

namespace dosa {

// sum_h w[h] * ReLU(x[h]) over 64 heads: four interleaved fp32 FMA chains
// (head h goes to chain h mod 4), combined as (c0 + c1) + (c2 + c3).
// x: 64 consecutive values (registers after inlining); w: 16-byte aligned,
// read through the read-only path (every lane of a warp reads the same
// address, so each load is a broadcast).  Measured faster on B200 than a
// packed fma.rn.f32x2 form or an 8-chain form.
__device__ __forceinline__ float head_reduce64(const float* x, const float* __restrict__ w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
  float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 ww = __ldg(w4 + i);
    c0 = fmaf(ww.x, fmaxf(x[4 * i + 0], 0.f), c0);
    c1 = fmaf(ww.y, fmaxf(x[4 * i + 1], 0.f), c1);
    c2 = fmaf(ww.z, fmaxf(x[4 * i + 2], 0.f), c2);
    c3 = fmaf(ww.w, fmaxf(x[4 * i + 3], 0.f), c3);
  }
  return (c0 + c1) + (c2 + c3);
}

}  // namespace dosa
