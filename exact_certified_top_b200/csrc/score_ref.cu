// CUDA-core reference scorer: the indexer score with plain fp32 FMAs, one
// thread per key, no tensor cores.  It exists to cross-check the tensor-core
// path on the device; it is not on any timed path.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dosa_internal.h"

namespace dosa {

template <bool kFp8>
__device__ __forceinline__ float load_code(const void* base, int64_t idx) {
  if constexpr (kFp8) {
    __nv_fp8_e4m3 v;
    v.__x = reinterpret_cast<const uint8_t*>(base)[idx];
    return float(v);
  } else {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  }
}

// grid (rows, key blocks of 128); block 128 threads.
template <bool kFp8>
__global__ void __launch_bounds__(128) score_ref_kernel(const void* q, const float* q_scale,
                                                         const float* w, const void* k,
                                                         const float* k_scale, int64_t row0,
                                                         int64_t pos0, int H, float* scores,
                                                         int64_t ld) {
  __shared__ float sq[64 * kHeadDim];
  const int64_t i = blockIdx.x;
  const int64_t t = row0 + i;
  const int64_t pos = pos0 + i;
  const int64_t s0 = (int64_t)blockIdx.y * 128;
  if (s0 > pos) return;
  for (int e = threadIdx.x; e < H * kHeadDim; e += blockDim.x)
    sq[e] = load_code<kFp8>(q, t * H * kHeadDim + e);
  __syncthreads();
  const int64_t s = s0 + threadIdx.x;
  if (s > pos) return;
  float kr[kHeadDim];
#pragma unroll
  for (int e = 0; e < kHeadDim; ++e) kr[e] = load_code<kFp8>(k, s * kHeadDim + e);
  float acc = 0.f;
  for (int h = 0; h < H; ++h) {
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < kHeadDim; ++e) dot = fmaf(sq[h * kHeadDim + e], kr[e], dot);
    acc = fmaf(w[t * H + h], fmaxf(dot, 0.f), acc);
  }
  if constexpr (kFp8) acc *= q_scale[t] * k_scale[s];
  scores[i * ld + s] = acc;
}

cudaError_t launch_scores_ref(const Handle& h, const SeqView& v, float* scores, int64_t ld,
                              cudaStream_t stream) {
  if (v.rows == 0) return cudaSuccess;
  const int64_t max_pos = v.pos0 + v.rows - 1;
  dim3 grid((unsigned)v.rows, (unsigned)((max_pos + 128) / 128));
  profile_before(DOSA_KERNEL_REFERENCE, stream);
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    score_ref_kernel<true><<<grid, 128, 0, stream>>>(v.q, v.q_scale, v.w, v.k, v.k_scale, v.row0,
                                                     v.pos0, h.cfg.H, scores, ld);
  else
    score_ref_kernel<false><<<grid, 128, 0, stream>>>(v.q, v.q_scale, v.w, v.k, v.k_scale,
                                                      v.row0, v.pos0, h.cfg.H, scores, ld);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_REFERENCE, stream);
  return e;
}

}  // namespace dosa
