// Final selection of the certified indexer: per query row, the exact Top-K of
// its packed (score, key) candidates ("DOSA: Dots Sparse Attention", Daily
// Paper Cast transcript, Related Work: radix selection narrows the Top-K
// without a full sort; Method section: packed scores for selection).
//
// Every candidate was written with a score >= the row's threshold at the
// time, and the row's final threshold tau is <= its K-th score, so the Top-K
// are exactly the K best of the candidates with score >= tau.  Those are
// gathered into shared memory, the K-th score is found by 4 radix passes over
// order-preserving keys, ties at the K-th score go to the smallest key
// indices, and the K indices are written in ascending order.
#include "dosa_device.cuh"
#include "dosa_internal.h"

namespace dosa {

constexpr int kSelThreads = 512;
constexpr int kSelList = 6144;        // candidates >= tau held in shared memory
constexpr int kSelOut = 4096;         // >= max K, power of two

struct CandView {
  float score;
  int key;
};

// Bitonic sort (ascending) of n_pow2 uint32 values in shared memory.
__device__ void block_bitonic_sort(uint32_t* a, int n_pow2) {
  for (int k = 2; k <= n_pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & k) == 0;
          const uint32_t x = a[i], y = a[ixj];
          if ((x > y) == up) {
            a[i] = y;
            a[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Radix select over n keys read through `get(i)`: returns the key of the K-th
// largest and writes how many elements equal to it must be taken.
template <typename Get>
__device__ uint32_t radix_kth(Get get, int n, int K, uint32_t* hist, uint32_t* s_digit,
                              uint32_t* s_above, uint32_t* take) {
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t u = get(i);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nb = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += nb;
      }
      const uint32_t excl = incl - sum;
      if (excl < remaining && remaining <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc < remaining && remaining <= acc + c[j]) {
            *s_digit = 255 - 8 * lane - j;
            *s_above = acc;
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= *s_digit << shift;
    mask |= 255u << shift;
    remaining -= *s_above;
    __syncthreads();
  }
  *take = remaining;
  return prefix;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const CandView* __restrict__ cand, int cap, const int* __restrict__ cand_count,
    const float* __restrict__ tau, int64_t pos0, int K, int32_t* __restrict__ out) {
  extern __shared__ uint32_t sel_smem[];
  uint32_t* lkey = sel_smem;                  // [kSelList]
  int32_t* lidx = reinterpret_cast<int32_t*>(lkey + kSelList);   // [kSelList]
  uint32_t* outv = reinterpret_cast<uint32_t*>(lidx + kSelList); // [kSelOut]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_above, s_take, s_n, s_nout, s_nties;
  const int64_t row = blockIdx.x;
  const int64_t nvis = pos0 + row + 1;
  int32_t* o = out + row * K;
  const int cnt = cand_count[row];
  if (cnt < 0) return;                        // overflowed: written by the repair pass
  const CandView* cl = cand + row * (int64_t)cap;
  if (nvis <= K) {
    // every visible key is a candidate; the answer is all of them
    for (int i = threadIdx.x; i < K; i += blockDim.x) o[i] = i < nvis ? i : -1;
    return;
  }
  const float th = tau[row];
  if (threadIdx.x == 0) s_n = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    const CandView c = cl[i];
    if (c.score >= th) {
      const uint32_t slot = atomicAdd(&s_n, 1u);
      if (slot < (uint32_t)kSelList) {
        lkey[slot] = ordered_key(c.score);
        lidx[slot] = c.key;
      }
    }
  }
  __syncthreads();
  const int n = (int)s_n;
  const bool in_smem = n <= kSelList;
  auto key_at = [&](int i) -> uint32_t {
    return in_smem ? lkey[i] : ordered_key(cl[i].score);
  };
  auto idx_at = [&](int i) -> int32_t { return in_smem ? lidx[i] : cl[i].key; };
  const int m = in_smem ? n : cnt;            // the global path scans every candidate
  const uint32_t kth = radix_kth([&](int i) { return key_at(i); }, m, K, hist, &s_digit,
                                 &s_above, &s_take);
  const uint32_t take = s_take;
  // gather: keys above the K-th go straight to the output list; ties are
  // collected (ascending index order is decided by sorting them)
  if (threadIdx.x == 0) {
    s_nout = 0;
    s_nties = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const uint32_t u = key_at(i);
    if (u > kth) {
      const uint32_t p = atomicAdd(&s_nout, 1u);
      outv[p] = (uint32_t)idx_at(i);
    }
  }
  __syncthreads();
  const uint32_t n_above = s_nout;            // == K - take
  // ties: reuse the tail of the output buffer region as scratch when they fit
  uint32_t* ties = outv + n_above;
  const uint32_t tie_room = kSelOut - n_above;
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    if (key_at(i) == kth) {
      const uint32_t p = atomicAdd(&s_nties, 1u);
      if (p < tie_room) ties[p] = (uint32_t)idx_at(i);
    }
  }
  __syncthreads();
  const uint32_t n_ties = s_nties;
  if (n_ties <= tie_room) {
    // sort the ties, keep the `take` smallest indices
    uint32_t pw = 1;
    while (pw < n_ties) pw <<= 1;
    if (pw > tie_room) {
      // not enough room to pad: fall back to repeated minimum extraction
      for (uint32_t r = 0; r < take; ++r) {
        __shared__ uint32_t best;
        if (threadIdx.x == 0) best = 0xFFFFFFFFu;
        __syncthreads();
        for (uint32_t i = threadIdx.x + r; i < n_ties; i += blockDim.x) atomicMin(&best, ties[i]);
        __syncthreads();
        if (threadIdx.x == 0) {
          for (uint32_t i = r; i < n_ties; ++i)
            if (ties[i] == best) {
              ties[i] = ties[r];
              ties[r] = best;
              break;
            }
        }
        __syncthreads();
      }
    } else {
      for (uint32_t i = n_ties + threadIdx.x; i < pw; i += blockDim.x) ties[i] = 0xFFFFFFFFu;
      __syncthreads();
      block_bitonic_sort(ties, (int)pw);
    }
  } else {
    // more ties than room: take the `take` smallest tie indices by repeated
    // selection over the candidates (rare; many exactly equal scores)
    uint32_t floor_idx = 0;
    for (uint32_t r = 0; r < take; ++r) {
      __shared__ uint32_t best;
      if (threadIdx.x == 0) best = 0xFFFFFFFFu;
      __syncthreads();
      for (int i = threadIdx.x; i < m; i += blockDim.x)
        if (key_at(i) == kth && (uint32_t)idx_at(i) >= floor_idx) atomicMin(&best, (uint32_t)idx_at(i));
      __syncthreads();
      if (threadIdx.x == 0) ties[r] = best;
      floor_idx = best + 1;
      __syncthreads();
    }
  }
  __syncthreads();
  // the K selected indices: n_above + take == K; pad to a power of two and sort
  uint32_t pw = 1;
  while (pw < (uint32_t)K) pw <<= 1;
  for (uint32_t i = K + threadIdx.x; i < pw; i += blockDim.x) outv[i] = 0xFFFFFFFFu;
  __syncthreads();
  block_bitonic_sort(outv, (int)pw);
  for (int i = threadIdx.x; i < K; i += blockDim.x) o[i] = (int32_t)outv[i];
}

constexpr int kSelSmem = (2 * kSelList + kSelOut) * 4;

cudaError_t launch_select(const CertBuffers& b, int64_t rows, int64_t pos0, int K, int32_t* out,
                          cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSelSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  profile_before(DOSA_KERNEL_SELECT, stream);
  select_kernel<<<(unsigned)rows, kSelThreads, kSelSmem, stream>>>(
      reinterpret_cast<const CandView*>(b.cand), b.cap, b.cand_count, b.tau, pos0, K, out);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_SELECT, stream);
  return e;
}

}  // namespace dosa
