// Exact per-row Top-K by radix select ("DOSA: Dots Sparse Attention", Daily
// Paper Cast transcript, Related Work: radix selection narrows the Top-K
// candidates without fully sorting the scores).
//
// One CTA per row.  Scores are mapped to order-preserving 32-bit keys (-0.0
// mapped like +0.0).  Four 8-bit digit passes, most significant first, find
// the exact key of the K-th largest score; a final pass compacts, in index
// order, every element above it plus the first (smallest-index) elements equal
// to it until K are taken.  The output is therefore ascending by index and
// ties go to the smaller index.
#include "dosa_device.cuh"
#include "dosa_internal.h"

namespace dosa {

constexpr int kTopkThreads = 1024;

// Exclusive prefix count of `flag` over the CTA in thread order; returns the
// CTA total through *total.  Uses `scratch` (32 ints of shared memory).
__device__ __forceinline__ int block_exclusive_count(bool flag, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned ballot = __ballot_sync(0xFFFFFFFFu, flag);
  const int in_warp = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) scratch[warp] = __popc(ballot);
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int v = lane < nw ? scratch[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane < nw) scratch[lane] = incl - v;     // exclusive per-warp offsets
    if (lane == 31) scratch[32] = incl;          // total
  }
  __syncthreads();
  const int r = scratch[warp] + in_warp;
  *total = scratch[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(
    const float* __restrict__ scores, int64_t ld, const int64_t* __restrict__ row_len, int64_t len0,
    int64_t max_len, int K, int32_t* __restrict__ out, int64_t out_ld,
    const int* __restrict__ row_list, const int* __restrict__ row_count) {
  __shared__ unsigned hist[256];
  __shared__ int scan_scratch[33];
  __shared__ unsigned s_digit, s_above;
  // Row-list mode: block i handles scores row i for output row row_list[i].
  int64_t row = blockIdx.x, orow = blockIdx.x;
  if (row_list) {
    if ((int)blockIdx.x >= *row_count) return;
    orow = row_list[blockIdx.x];
  }
  int64_t n = row_len ? row_len[row] : len0 + orow;
  if (n > max_len) n = max_len;
  if (n < 0) n = 0;
  const float* x = scores + row * ld;
  int32_t* o = out + orow * out_ld;
  if (n <= K) {
    for (int i = threadIdx.x; i < K; i += blockDim.x) o[i] = i < n ? i : -1;
    return;
  }
  unsigned prefix = 0, mask = 0, remaining = (unsigned)K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned u = ordered_key(x[i]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l down to 248-8l (descending order)
      const int lane = threadIdx.x;
      unsigned c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      unsigned incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned nb = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += nb;
      }
      const unsigned excl = incl - sum;   // count of digits above this lane's block
      if (excl < remaining && remaining <= incl) {
        unsigned acc = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc < remaining && remaining <= acc + c[j]) {
            s_digit = 255 - 8 * lane - j;
            s_above = acc;
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    remaining -= s_above;
    __syncthreads();
  }
  // prefix = key of the K-th largest; take `remaining` (>= 1) of the equal keys.
  int taken = 0, ties_seen = 0;
  for (int64_t base = 0; base < n; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    const unsigned u = i < n ? ordered_key(x[i]) : 0u;
    const bool gt = i < n && u > prefix;
    const bool eq = i < n && u == prefix;
    int eq_total;
    const int tie_rank = ties_seen + block_exclusive_count(eq, scan_scratch, &eq_total);
    const bool sel = gt || (eq && tie_rank < (int)remaining);
    int sel_total;
    const int pos = taken + block_exclusive_count(sel, scan_scratch, &sel_total);
    if (sel && pos < K) o[pos] = (int32_t)i;
    taken += sel_total;
    ties_seen += eq_total;
  }
}

__global__ void fill_kernel(float* __restrict__ p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

cudaError_t launch_fill(float* p, int64_t n, float v, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = (n + 255) / 256;
  profile_before(DOSA_KERNEL_FILL, stream);
  fill_kernel<<<(unsigned)(blocks < 8LL * sms ? blocks : 8LL * sms), 256, 0, stream>>>(p, n, v);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_FILL, stream);
  return e;
}

cudaError_t launch_topk_rows(const float* scores, int64_t ld, const int64_t* row_len, int64_t len0,
                             int64_t max_len, int64_t rows, int K, int32_t* out, int64_t out_ld,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  profile_before(DOSA_KERNEL_TOPK, stream);
  topk_rows_kernel<<<(unsigned)rows, kTopkThreads, 0, stream>>>(scores, ld, row_len, len0,
                                                                 max_len, K, out, out_ld, nullptr,
                                                                 nullptr);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_TOPK, stream);
  return e;
}

cudaError_t launch_topk_list(const float* scores, int64_t ld, const int* row_list,
                             const int* row_count, int list_cap, int64_t len0, int64_t max_len,
                             int K, int32_t* out, int64_t out_ld, cudaStream_t stream) {
  if (list_cap <= 0) return cudaSuccess;
  profile_before(DOSA_KERNEL_TOPK, stream);
  topk_rows_kernel<<<(unsigned)list_cap, kTopkThreads, 0, stream>>>(
      scores, ld, nullptr, len0, max_len, K, out, out_ld, row_list, row_count);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_TOPK, stream);
  return e;
}

}  // namespace dosa
