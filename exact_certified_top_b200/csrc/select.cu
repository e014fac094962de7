// Final selection of the certified indexer: per query row, the exact Top-K of
// its packed (score, key) candidates ("DOSA: Dots Sparse Attention", Daily
// Paper Cast transcript, Related Work: radix selection narrows the Top-K
// without a full sort; Method section: packed scores for selection).
//
// Every candidate was written with a score >= the row's threshold at the
// time, and the row's final threshold tau is <= its K-th score, so the Top-K
// are exactly the K best candidates with score >= tau.  Those are gathered
// into shared memory (when they fit; otherwise the passes read the whole list
// from global memory).  The K-th (score, index) is found in one pass when
// the list fits: a 2048-bin histogram of the order-preserving keys above tau,
// a suffix scan for the bin of the K-th key, and a direct rank of that bin's
// few entries (score descending, index ascending).  A bin of more than 128
// entries that all hold one score is a tie at the K-th score: only the index
// cut among them is left.  Otherwise (the list is in global memory, or a
// crowded bin holds several scores) 4 radix passes find the K-th score, and
// when more entries tie with it than are needed, a second radix select over
// the complemented key indices of the tied entries finds the smallest
// indices (skipped when every tied entry is needed).  The
// K indices are put in ascending order through a bitmap over the row's keys
// (one bit per key, then a block-wide prefix count), or by a bitonic sort for
// rows longer than the bitmap.  Every step is a parallel pass; nothing is
// serial in the number of ties.
#include "dosa_device.cuh"
#include "dosa_internal.h"

namespace dosa {

constexpr int kSelThreads = 512;
constexpr int kSelList = 4096;        // candidates >= tau held in shared memory
constexpr int kSelOut = 4096;         // >= max K, power of two
constexpr int kBitmapWords = 32768;   // rows of up to 1,048,576 keys use the bitmap

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

// Warp-aggregated slot reservation: one atomic per warp; returns this lane's
// slot (meaningful only for active lanes).
__device__ __forceinline__ uint32_t agg_slot(uint32_t* counter, bool active) {
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, active);
  const int lane = threadIdx.x & 31;
  uint32_t base = 0;
  const int leader = m ? __ffs(m) - 1 : 0;
  if (m && lane == leader) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(0xFFFFFFFFu, base, leader);
  return base + __popc(m & ((1u << lane) - 1u));
}

// Radix select over n elements: `get(i, &key)` returns false to skip element i.
// Returns the key of the K-th largest selected element; *take = how many
// elements equal to it belong to the K largest, *eq = how many equal it.
// hist: 2 x 256 words, both zero on entry and left zero on return; each pass
// counts into one while the other is being cleared, two barriers per pass.
template <typename Get>
__device__ uint32_t radix_kth(Get get, int n, uint32_t K, uint32_t* hist, uint32_t* s_res,
                              uint32_t* take, uint32_t* eq) {
  uint32_t prefix = 0, mask = 0, remaining = K, eq_count = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* h = hist + (pass & 1) * 256;
    const int nn = (n + 31) & ~31;             // whole warps for the aggregated adds
    for (int i = threadIdx.x; i < nn; i += blockDim.x) {
      uint32_t u = 0;
      const bool in = i < n && get(i, &u) && (u & mask) == prefix;
      const uint32_t bin = (u >> shift) & 255u;
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
      if (in) {
        const uint32_t peers = __match_any_sync(m, bin);
        if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = h[255 - 8 * lane - j];
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
            s_res[(pass & 1) * 4 + 0] = 255 - 8 * lane - j;
            s_res[(pass & 1) * 4 + 1] = acc;
            s_res[(pass & 1) * 4 + 2] = c[j];
          }
          acc += c[j];
        }
      }
    } else if (threadIdx.x < 64) {
      // clear the other histogram for the next pass (and on return)
      uint32_t* o = hist + ((pass + 1) & 1) * 256;
      for (int j = threadIdx.x - 32; j < 256; j += 32) o[j] = 0u;
    }
    __syncthreads();
    const uint32_t* r = s_res + (pass & 1) * 4;
    prefix |= r[0] << shift;
    mask |= 255u << shift;
    remaining -= r[1];
    eq_count = r[2];
  }
  // the last pass's histogram is still counted: clear it (the caller
  // synchronises before the next use)
  for (int j = threadIdx.x; j < 256; j += blockDim.x) hist[256 + j] = 0u;
  *take = remaining;
  *eq = eq_count;       // elements whose key equals the result (last digit's bin)
  return prefix;
}

// Exclusive prefix sum of v over the CTA in thread order (scratch: 32 words).
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    const uint32_t t = lane < nw ? scratch[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, ti, o);
      if (lane >= o) ti += n;
    }
    if (lane < nw) scratch[lane] = ti - t;
  }
  __syncthreads();
  return scratch[warp] + incl - v;
}

constexpr int kFineBins = 2048;       // one histogram pass over keys above tau
constexpr int kBoundaryCap = 128;     // entries of the K-th key's bin ranked directly
                                      // (quadratic: larger bins take the tie or radix path)

// The K-th largest (key, index) pair of the n entries lkey/lidx (key
// descending, index ascending), as the pair (*kth, *cut): the winners are the
// entries with key > kth, or key == kth and index <= cut.  Every key is >=
// lo.  scratch: kFineBins + 2 kBoundaryCap words; red: 32 words.  Returns
//   kFineDone   *kth and *cut set;
//   kFineTies   the bin of the K-th key holds more than kBoundaryCap entries,
//               all with one key: *kth set, and the winners among them are
//               the *take with the smallest indices (the caller cuts them);
//   kFineRadix  neither: the caller runs the radix passes.
// Called by the whole CTA.
constexpr int kFineRadix = 0, kFineDone = 1, kFineTies = 2;
__device__ int fine_bin_kth(const uint32_t* lkey, const int32_t* lidx, int n, uint32_t K,
                            uint32_t lo, uint32_t* scratch, uint32_t* red, uint32_t* kth,
                            uint32_t* cut, uint32_t* take) {
  __shared__ uint32_t s_shift, s_bin, s_need, s_cnt, s_kth, s_cut, s_nb, s_kmin, s_kmax;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* h = scratch;                                   // [kFineBins]
  uint32_t* bk = scratch + kFineBins;                      // [kBoundaryCap] keys
  uint32_t* bi = bk + kBoundaryCap;                        // [kBoundaryCap] indices
  if (n < (int)K) return kFineRadix;
  // the largest key, then the shift that maps [lo, max] into kFineBins bins
  uint32_t mx = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) mx = max(mx, lkey[i]);
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if (lane == 0) red[warp] = mx;
  for (int j = threadIdx.x; j < kFineBins; j += blockDim.x) h[j] = 0u;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t m2 = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m2 = max(m2, red[w]);
    const uint32_t range = m2 - lo;
    uint32_t sh = 0;
    while ((range >> sh) >= (uint32_t)kFineBins) ++sh;
    s_shift = sh;
    s_nb = 0;
  }
  __syncthreads();
  const uint32_t sh = s_shift;
  for (int i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&h[(lkey[i] - lo) >> sh], 1u);
  __syncthreads();
  // bins in descending order: thread t holds bins kFineBins-1-4t .. -4t-3
  uint32_t c[4], local = 0;
  const int per = kFineBins / kSelThreads;
#pragma unroll
  for (int j = 0; j < per; ++j) {
    c[j] = h[kFineBins - 1 - per * threadIdx.x - j];
    local += c[j];
  }
  const uint32_t above = block_exclusive_sum(local, red);
  if (above < K && K <= above + local) {
    uint32_t acc = above;
#pragma unroll
    for (int j = 0; j < per; ++j) {
      if (acc < K && K <= acc + c[j]) {
        s_bin = kFineBins - 1 - per * threadIdx.x - j;
        s_need = K - acc;                 // entries of the bin that win
        s_cnt = c[j];
      }
      acc += c[j];
    }
  }
  __syncthreads();
  const uint32_t bin = s_bin, need = s_need, cnt = s_cnt;
  if (cnt > (uint32_t)kBoundaryCap) {
    // a crowded bin: when it holds a single key (a tie at the K-th score)
    // only the index cut among the tied entries is left
    if (threadIdx.x == 0) {
      s_kmin = 0xFFFFFFFFu;
      s_kmax = 0u;
    }
    __syncthreads();
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t u = lkey[i];
      if (((u - lo) >> sh) == bin) {
        kmin = min(kmin, u);
        kmax = max(kmax, u);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xFFFFFFFFu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    }
    if (lane == 0) {
      atomicMin(&s_kmin, kmin);
      atomicMax(&s_kmax, kmax);
    }
    __syncthreads();
    if (s_kmin != s_kmax) return kFineRadix;
    *kth = s_kmin;
    *take = need;
    return kFineTies;
  }
  // the bin's entries, then each one's rank among them
  for (int i = threadIdx.x; i < ((n + 31) & ~31); i += blockDim.x) {
    const bool in = i < n && ((lkey[i] - lo) >> sh) == bin;
    const uint32_t slot = agg_slot(&s_nb, in);
    if (in) {
      bk[slot] = lkey[i];
      bi[slot] = (uint32_t)lidx[i];
    }
  }
  __syncthreads();
  for (uint32_t e = threadIdx.x; e < cnt; e += blockDim.x) {
    const uint32_t ke = bk[e], ie = bi[e];
    uint32_t rank = 0;
    for (uint32_t f = 0; f < cnt; ++f) {
      const uint32_t kf = bk[f];
      rank += (kf > ke || (kf == ke && bi[f] < ie)) ? 1u : 0u;
    }
    if (rank == need - 1) {
      s_kth = ke;
      s_cut = ie;
    }
  }
  __syncthreads();
  *kth = s_kth;
  *cut = s_cut;
  return kFineDone;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const CandView* __restrict__ cand, int seg_cap, const int* __restrict__ cand_count,
    const float* __restrict__ tau, int64_t pos0, int K, int32_t* __restrict__ out) {
  extern __shared__ uint32_t sel_smem[];
  uint32_t* lkey = sel_smem;                                        // [kSelList]
  int32_t* lidx = reinterpret_cast<int32_t*>(lkey + kSelList);     // [kSelList]
  uint32_t* bm = reinterpret_cast<uint32_t*>(lidx + kSelList);     // [kBitmapWords] or sort area
  __shared__ uint32_t hist[2 * 256];
  __shared__ uint32_t scan[32];
  __shared__ uint32_t s_res[8];
  __shared__ uint32_t s_n, s_nout;
  const int64_t row = blockIdx.x;
  const int64_t nvis = pos0 + row + 1;
  int32_t* o = out + row * K;
  // the row's list: kSegs segments of seg_cap entries, counts c0..c3
  const int4 cc = *reinterpret_cast<const int4*>(cand_count + row * 4);
  if (cc.x < 0) return;                       // overflowed: written by the repair pass
  const CandView* cl = cand + row * 4 * (int64_t)seg_cap;
  const int e1 = cc.x, e2 = e1 + cc.y, e3 = e2 + cc.z, cnt = e3 + cc.w;
  // i-th entry of the concatenated segments
  auto entry = [&](int i) -> const CandView& {
    const int j = (i >= e1) + (i >= e2) + (i >= e3);
    const int off = i - (j == 0 ? 0 : j == 1 ? e1 : j == 2 ? e2 : e3);
    return cl[j * (int64_t)seg_cap + off];
  };
  if (nvis <= K) {
    // every visible key is a candidate; the answer is all of them
    for (int i = threadIdx.x; i < K; i += blockDim.x) o[i] = i < nvis ? i : -1;
    return;
  }
  const float th = tau[row];
  if (threadIdx.x == 0) {
    s_n = 0;
    s_nout = 0;
  }
  for (int j = threadIdx.x; j < 2 * 256; j += blockDim.x) hist[j] = 0u;
  __syncthreads();
  // gather the candidates >= tau, segment by segment, eight per thread per
  // pass: four 16-byte loads issued before any is used (segments start
  // 512-byte aligned)
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    const int cj = j == 0 ? cc.x : j == 1 ? cc.y : j == 2 ? cc.z : cc.w;
    const CandView* sp = cl + j * (int64_t)seg_cap;
    for (int b0 = 0; b0 < cj; b0 += blockDim.x * 8) {
      const int b = b0 + threadIdx.x * 4;
      const int bh = b + blockDim.x * 4;
      CandView c[8];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int bb = hh ? bh : b;
        if (bb + 3 < cj) {
          const int4 v0 = *reinterpret_cast<const int4*>(sp + bb);
          const int4 v1 = *reinterpret_cast<const int4*>(sp + bb + 2);
          c[hh * 4 + 0] = CandView{__int_as_float(v0.x), v0.y};
          c[hh * 4 + 1] = CandView{__int_as_float(v0.z), v0.w};
          c[hh * 4 + 2] = CandView{__int_as_float(v1.x), v1.y};
          c[hh * 4 + 3] = CandView{__int_as_float(v1.z), v1.w};
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            c[hh * 4 + e] = bb + e < cj ? sp[bb + e] : CandView{-INFINITY, 0};
        }
      }
      // one slot reservation per warp and pass: a warp scan of the
      // per-thread counts, one shared atomic by the last lane
      uint32_t mine = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int at = (e < 4 ? b : bh) + (e & 3);
        if (at < cj && c[e].score >= th) mine |= 1u << e;
      }
      const int lane = threadIdx.x & 31;
      const uint32_t cm = __popc(mine);
      uint32_t incl = cm;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      uint32_t base = 0;
      if (lane == 31 && incl) base = atomicAdd(&s_n, incl);
      uint32_t slot = __shfl_sync(0xFFFFFFFFu, base, 31) + incl - cm;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((mine >> e) & 1u) {
          if (slot < (uint32_t)kSelList) {
            lkey[slot] = ordered_key(c[e].score);
            lidx[slot] = c[e].key;
          }
          ++slot;
        }
      }
    }
  }
  __syncthreads();
  const int n = (int)s_n;
  const bool in_smem = n <= kSelList;
  const int m = in_smem ? n : cnt;            // the global path scans every candidate
  auto key_at = [&](int i) -> uint32_t { return in_smem ? lkey[i] : ordered_key(entry(i).score); };
  auto idx_at = [&](int i) -> uint32_t { return (uint32_t)(in_smem ? lidx[i] : entry(i).key); };
  uint32_t kth = 0, cut = 0xFFFFFFFFu;
  // Fast path (the list is in shared memory): one histogram of the keys above
  // the threshold in kFineBins bins, the bin that holds the K-th key from a
  // block suffix scan, and the exact rank (key descending, index ascending)
  // of the few entries of that bin.  Falls back to the radix passes when that
  // bin holds more than kBoundaryCap entries (heavy ties).
  uint32_t tie_take = 0;
  const int fine = in_smem ? fine_bin_kth(lkey, lidx, n, (uint32_t)K, ordered_key(th), bm, scan,
                                          &kth, &cut, &tie_take)
                           : kFineRadix;
  __syncthreads();
  if (fine == kFineTies) {
    // the K-th key is known; keep the tie_take smallest indices among its
    // entries (the tie_take-th largest complemented index is the cut)
    uint32_t t2, e2;
    cut = ~radix_kth(
        [&](int i, uint32_t* u) {
          if (key_at(i) != kth) return false;
          *u = ~idx_at(i);
          return true;
        },
        m, tie_take, hist, s_res, &t2, &e2);
  } else if (fine == kFineRadix) {
    uint32_t take = 0, eq = 0;
    kth = radix_kth(
        [&](int i, uint32_t* u) {
          *u = key_at(i);
          return true;
        },
        m, (uint32_t)K, hist, s_res, &take, &eq);
    // Among entries equal to the K-th key, keep those with the `take` smallest
    // indices: the take-th largest complemented index is the cut.  When all of
    // them are needed there is nothing to cut.
    if (take < eq) {
      uint32_t t2, e2;
      __syncthreads();
      cut = ~radix_kth(
          [&](int i, uint32_t* u) {
            if (key_at(i) != kth) return false;
            *u = ~idx_at(i);
            return true;
          },
          m, take, hist, s_res, &t2, &e2);
    }
  }
  auto winner = [&](int i, uint32_t* id) -> bool {
    const uint32_t u = key_at(i);
    *id = idx_at(i);
    return u > kth || (u == kth && *id <= cut);
  };
  if (nvis <= (int64_t)kBitmapWords * 32) {
    // ascending order through a bitmap over the row's keys
    const int nwords = (int)((nvis + 31) >> 5);
    for (int w = threadIdx.x; w < nwords; w += blockDim.x) bm[w] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
      uint32_t id;
      if (winner(i, &id) && id < (uint32_t)nvis) atomicOr(&bm[id >> 5], 1u << (id & 31));
    }
    __syncthreads();
    // each warp owns a contiguous run of words, its lanes four consecutive
    // words at a time (16-byte loads, no bank conflicts); a warp scan orders
    // the bits within a run
    const int lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int per = ((nwords + nwarps - 1) / nwarps + 127) & ~127;
    const int w0 = (threadIdx.x >> 5) * per, w1 = min(w0 + per, nwords);
    auto quad_at = [&](int w) -> uint4 {
      if (w + 3 < w1) return *reinterpret_cast<const uint4*>(bm + w);
      return make_uint4(w < w1 ? bm[w] : 0u, w + 1 < w1 ? bm[w + 1] : 0u,
                        w + 2 < w1 ? bm[w + 2] : 0u, 0u);
    };
    uint32_t c = 0;
    for (int w = w0 + 4 * lane; w < w1; w += 128) {
      const uint4 q = quad_at(w);
      c += __popc(q.x) + __popc(q.y) + __popc(q.z) + __popc(q.w);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, off);
    uint32_t base = block_exclusive_sum(lane == 0 ? c : 0u, scan);
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
    for (int wb = w0; wb < w1; wb += 128) {
      const int w = wb + 4 * lane;
      const uint4 q = w < w1 ? quad_at(w) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t pc = __popc(q.x) + __popc(q.y) + __popc(q.z) + __popc(q.w);
      uint32_t inc = pc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, inc, off);
        if (lane >= off) inc += n;
      }
      uint32_t at = base + inc - pc;
      const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t bits = words[e];
        while (bits) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1u;
          if (at < (uint32_t)K) o[at] = (int32_t)((w + e) * 32 + b);
          ++at;
        }
      }
      base += __shfl_sync(0xFFFFFFFFu, inc, 31);
    }
    return;
  }
  // long rows: gather the K winners (distinct indices: exactly K), sort, write
  uint32_t* outv = bm;
  const int mw = (m + 31) & ~31;
  for (int i = threadIdx.x; i < mw; i += blockDim.x) {
    uint32_t id = 0;
    const bool in = i < m && winner(i, &id);
    const uint32_t slot = agg_slot(&s_nout, in);
    if (in && slot < (uint32_t)kSelOut) outv[slot] = id;
  }
  __syncthreads();
  uint32_t pw = 1;
  while (pw < (uint32_t)K) pw <<= 1;
  for (uint32_t i = K + threadIdx.x; i < pw; i += blockDim.x) outv[i] = 0xFFFFFFFFu;
  __syncthreads();
  block_bitonic_sort(outv, (int)pw);
  for (int i = threadIdx.x; i < K; i += blockDim.x) o[i] = (int32_t)outv[i];
}

// Dynamic shared memory: the candidate key and index lists, then the bitmap
// (one bit per key of the longest row, at most kBitmapWords words) or the sort
// area of the long-row path (kSelOut words), whichever is larger.
static int select_smem_bytes(int64_t max_nvis) {
  int64_t words = (max_nvis + 31) / 32;
  if (words > kBitmapWords) words = kBitmapWords;
  if (words < kSelOut) words = kSelOut;
  return (int)((2 * kSelList + words) * 4);
}

cudaError_t launch_select(const CertBuffers& b, int64_t rows, int64_t pos0, int K, int32_t* out,
                          cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         select_smem_bytes((int64_t)kBitmapWords * 32));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int smem = select_smem_bytes(pos0 + rows);
  profile_before(DOSA_KERNEL_SELECT, stream);
  select_kernel<<<(unsigned)rows, kSelThreads, smem, stream>>>(
      reinterpret_cast<const CandView*>(b.cand), b.seg_cap, b.cand_count, b.tau, pos0, K, out);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_SELECT, stream);
  return e;
}

}  // namespace dosa
