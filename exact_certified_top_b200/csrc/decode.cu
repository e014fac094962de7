// Decode-step indexer for sm_100a: a few query rows (one decode token per
// sequence, or a handful of multi-token-prediction rows) against a long key
// cache, seeded by the previous step's selection ("DOSA: Dots Sparse
// Attention", Daily Paper Cast transcript, Experiments: the decode-time gain
// comes mostly from less selection work, the scores of keys selected at the
// previous step giving the threshold; Method section: a threshold from the
// K-th largest exact score of a subset of visible keys).
//
//   decode_seed   scores the K keys the previous step selected for each row
//                 (CUDA cores, fp32) and keeps the smallest of
//                 score - rounding margin.  When the row has K distinct
//                 visible seeds, that minimum is a sound lower bound tau0 of
//                 the row's K-th largest score as the scan computes it: at
//                 least K scores (the seeds') are >= it.  The largest seed
//                 score is kept too: it spans the row's histogram.
//   decode_scan   every visible key, split over all SMs by key range: the
//                 tensor-core scorer of the filter kernel (one MMA tile per 4
//                 query rows; two epilogue teams drain the two accumulators,
//                 alternate key tiles), scores >= tau counted in the row's
//                 256-bin histogram over [tau0, max seed score] and appended
//                 to the row's list eight tiles later.  Each CTA counts into shared
//                 memory; a threshold warp per CTA keeps moving those counts
//                 into the row's global histogram (shared by all CTAs) and
//                 raises the CTA's threshold to the lower edge of the highest
//                 global bin whose suffix count reaches K.  Counted keys are
//                 real scores >= their bin's edge, so the threshold stays a
//                 sound lower bound however the CTAs interleave.
//   decode_finish per-row counts and the final threshold (from the complete
//                 histogram) for the shared selection kernel (select.cu).
//                 A row's list has room for all its visible keys, so no row
//                 needs a repair pass.
//
// The margin covers the difference between the two fp32 evaluations of the
// same score (sequential CUDA-core FMAs here, tensor-core accumulation in the
// scan): every dot product of 128 exact products errs by at most 2^-17 of
// ||q_h|| ||k|| per evaluation, ReLU is 1-Lipschitz, and the head sum adds
// 2^-18 of sum_h |w_h| ||q_h|| ||k||; the margin 2^-13 (sum_h |w_h| ||q_h||)
// ||k|| leaves at least 4x headroom for the tensor core's accumulation.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "cand_state.cuh"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "score_epilogue.cuh"
#include "work_items.cuh"

namespace dosa {

constexpr float kSeedMargin = 0x1p-13f;
constexpr int kSeedKeys = 64;          // seeds per CTA of decode_seed
constexpr int kSeedSmem = (64 + kSeedKeys) * (kHeadDim + 1) * 4;

// The codes of 16 bytes as floats: 16 e4m3 values or 8 bf16 values.
template <bool kFp8>
__device__ __forceinline__ void codes16(const uint4& u, float* out) {
  const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (kFp8) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        __nv_fp8_e4m3 v;
        v.__x = (uint8_t)(wd[i] >> (8 * b));
        out[4 * i + b] = float(v);
      }
    } else {
      out[2 * i] = __uint_as_float(wd[i] << 16);
      out[2 * i + 1] = __uint_as_float(wd[i] & 0xFFFF0000u);
    }
  }
}

struct SeedParams {
  const void* q;            // absolute rows
  const float* q_scale;
  const float* w;
  const void* k;            // the sequence's first key
  const float* k_scale;
  const int32_t* seed;      // [rows, K] previous selection (sequence-relative, -1 padded)
  int64_t row0, rows, pos0, S;
  int K;
  int H;                    // heads per query row (32: slots 32..63 are zero)
  uint32_t* bitmap;         // [rows][words], zero on entry
  int64_t words;
  uint32_t* tau_key;        // [rows] ordered keys, 0xFFFFFFFF on entry
  uint32_t* smax_key;       // [rows] ordered keys, zero on entry
  int* seed_count;          // [rows] zero on entry
  int* dup;                 // [rows] zero on entry
};

// One CTA per (row, 64 seeds), 256 threads.  Thread (kg = tid / 16,
// hg = tid % 16) forms the dot products of keys kg + 16i with heads hg + 16j
// (i, j < 4): eight shared-memory loads feed sixteen FMAs.  Every dot product
// is one FMA chain over the 128 dimensions in order; the 16 threads of a key
// group add their head partial sums by shuffles.
template <bool kFp8>
__global__ void __launch_bounds__(256) decode_seed_kernel(const SeedParams p) {
  constexpr int H = 64, D = kHeadDim, P = D + 1;   // head slots; p.H of them are real
  extern __shared__ float seed_dyn[];
  float(*qf)[P] = reinterpret_cast<float(*)[P]>(seed_dyn);
  float(*kf)[P] = reinterpret_cast<float(*)[P]>(seed_dyn + H * P);
  __shared__ float wv[H], qn[H], kn[kSeedKeys];
  __shared__ int sidx[kSeedKeys];
  __shared__ float s_scale;
  const int row = blockIdx.x;
  const int64_t t = p.row0 + row;
  const int64_t pos = p.pos0 + row;
  const int j0 = blockIdx.y * kSeedKeys;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 16-byte loads, all issued before any is converted
  constexpr int EB = kFp8 ? 1 : 2;           // bytes per code
  constexpr int PER = 16 / EB;               // codes per 16 bytes
  constexpr int QV = H * D * EB / 16 / 256;  // 16-byte loads per thread (q row)
  constexpr int KC = D * EB / 16;            // 16-byte chunks per key
  constexpr int KV = kSeedKeys * KC / 256;   // 16-byte loads per thread (seed keys)
  {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                                      t * (int64_t)(p.H * D * EB));
    const int nvec = p.H * D * EB / 16;
    uint4 u[QV];
#pragma unroll
    for (int i = 0; i < QV; ++i) {
      const int e16 = threadIdx.x + i * 256;
      u[i] = e16 < nvec ? __ldg(src + e16) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < QV; ++i) {
      float f[PER];
      codes16<kFp8>(u[i], f);
      const int e = (threadIdx.x + i * 256) * PER;
#pragma unroll
      for (int c = 0; c < PER; ++c) qf[(e + c) / D][(e + c) % D] = f[c];
    }
  }
  if (threadIdx.x < H) wv[threadIdx.x] = threadIdx.x < p.H ? p.w[t * p.H + threadIdx.x] : 0.f;
  if (threadIdx.x < kSeedKeys) {
    const int j = j0 + threadIdx.x;
    int idx = j < p.K ? p.seed[row * (int64_t)p.K + j] : -1;
    if (idx < 0 || idx > pos || idx >= p.S) idx = -1;
    if (idx >= 0) {
      const uint32_t bit = 1u << (idx & 31);
      const uint32_t old = atomicOr(&p.bitmap[row * p.words + (idx >> 5)], bit);
      if (old & bit) atomicExch(&p.dup[row], 1);
    }
    sidx[threadIdx.x] = idx;
  }
  __syncthreads();
  {
    uint4 u[KV];
#pragma unroll
    for (int i = 0; i < KV; ++i) {
      const int e = threadIdx.x + i * 256, jj = e / KC, ch = e % KC;
      const int idx = sidx[jj];
      u[i] = idx >= 0 ? __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.k) +
                                                              (int64_t)idx * (D * EB)) + ch)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < KV; ++i) {
      float f[PER];
      codes16<kFp8>(u[i], f);
      const int e = threadIdx.x + i * 256, jj = e / KC, c0 = (e % KC) * PER;
#pragma unroll
      for (int c = 0; c < PER; ++c) kf[jj][c0 + c] = f[c];
    }
  }
  // ||q_h|| (one warp per 8 heads) for the margin, code domain, rounded up
  for (int h = warp; h < H; h += 8) {
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) ss = fmaf(qf[h][c], qf[h][c], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) qn[h] = sqrtf(ss) * (1.f + 0x1p-16f);
  }
  __syncthreads();
  {
    // ||k|| of every seed: 4 threads per key, 32 dimensions each
    const int key = threadIdx.x >> 2, part = threadIdx.x & 3;
    float ss = 0.f;
#pragma unroll 8
    for (int c = part * (D / 4); c < (part + 1) * (D / 4); ++c) ss = fmaf(kf[key][c], kf[key][c], ss);
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 1);
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 2);
    if (part == 0) kn[key] = sqrtf(ss) * (1.f + 0x1p-16f);
    // sum_h |w_h| ||q_h||
    if (warp == 0) {
      float sc = fmaf(fabsf(wv[lane]), qn[lane], fabsf(wv[lane + 32]) * qn[lane + 32]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(0xFFFFFFFFu, sc, o);
      if (lane == 0) s_scale = sc * (1.f + 0x1p-16f);
    }
  }
  const int kg = threadIdx.x >> 4, hg = threadIdx.x & 15;
  float x[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) x[i][j] = 0.f;
#pragma unroll 4
  for (int c = 0; c < D; ++c) {
    float a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = kf[kg + 16 * i][c];
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = qf[hg + 16 * j][c];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) x[i][j] = fmaf(b[j], a[i], x[i][j]);
  }
  float acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i] = fmaf(wv[hg + 16 * j], fmaxf(x[i][j], 0.f), acc[i]);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
  }
  __syncthreads();                       // kn and s_scale
  if (hg < 4) {
    const int jj = kg + 16 * hg;
    const int idx = sidx[jj];
    float sc = hg == 0 ? acc[0] : hg == 1 ? acc[1] : hg == 2 ? acc[2] : acc[3];
    if (idx >= 0) {
      float margin = kSeedMargin * s_scale * kn[jj];
      if constexpr (kFp8) {
        const float s2 = p.q_scale[t] * p.k_scale[idx];
        sc *= s2;
        margin = margin * s2 * (1.f + 0x1p-20f);
      }
      atomicMin(&p.tau_key[row], ordered_key(sc - margin));
      atomicMax(&p.smax_key[row], ordered_key(sc));
      atomicAdd(&p.seed_count[row], 1);
    }
  }
}

// ---- split-S scan -------------------------------------------------------------------

// Rows per work item: one MMA tile (N = 4 rows x 64 heads = 256) per key tile.
constexpr int kDecRows = 4;

template <bool kFp8>
struct ScanCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  // deep key pipeline: the scan streams the whole cache once and nothing else
  // needs the shared memory (fp8: 10 x 16 KB, bf16: 4 x 32 KB in flight)
  static constexpr int kKeyStages = kFp8 ? 10 : 4;
  static constexpr int kH = 64;
  static constexpr int kQRows = kDecRows * kH;         // 256 = MMA N
  static constexpr uint32_t kKeySubBytes = kKeyTile * 128;
  static constexpr uint32_t kKeyStageBytes = kKeySubBytes * kSub;
  static constexpr uint32_t kQSubBytes = kQRows * 128;
  static constexpr uint32_t kQBytes = kQSubBytes * kSub;
  static constexpr int kEpiWarps = 16;
  // producer, MMA issuer, 16 epilogue warps, the threshold warp
  static constexpr int kThreads = 64 + kEpiWarps * 32 + 32;
  static constexpr int kTauWarp = 2 + kEpiWarps;
  static constexpr int kUnitThreads = (kEpiWarps + 1) * 32;   // named barrier: epilogue + threshold
  static constexpr uint32_t kTmemCols = 512;           // two accumulators of 256 columns
  static constexpr uint32_t kSmemBytes = 1024 + kQBytes + kKeyStages * kKeyStageBytes + 256;
  // appends trail the scores by 2 kHoldT - 2 tiles (kHoldT - 1 of a team's
  // tiles): long enough for the counts of a tile to reach the global
  // histogram from every CTA and come back as a higher threshold (a few
  // passes of the threshold warps)
  static constexpr int kHoldT = 5;
};

struct ScanParams {
  const float* w;            // absolute rows
  const float* q_scale;
  const float* k_scale;      // the sequence's first key
  int64_t row0, rows, pos0, S;
  int n_items, parts, K;
  int H;                     // heads per query row: 32 or 64 (the MMA always sees 64)
  const uint32_t* tau_key;   // [rows] from decode_seed
  const uint32_t* smax_key;  // [rows] from decode_seed
  const int* seed_count;
  const int* dup;
  unsigned* hist;            // [rows][kBins], zero on entry
  uint32_t* tau_run;         // [rows] ordered shared threshold, zero on entry
  Cand* cand;                // [rows][cap]
  int cap;
  int* count;                // [rows] candidates reserved (may exceed cap)
  unsigned long long* counters;
  int* err;
};

// The row's starting threshold: the seeds' bound when the row has K distinct
// visible seeds, else -inf.
__device__ __forceinline__ float seed_tau(const ScanParams& p, int64_t r) {
  return (p.seed_count[r] == p.K && !p.dup[r]) ? key_to_float(p.tau_key[r]) : -INFINITY;
}

// The row's histogram: kBins bins of width w from tau0 up to the largest seed
// score (rows without a seed bound keep no histogram).
struct RowBins {
  float lo, w, inv_w;
  bool on;
  float t0;           // the seed bound (or -inf)
};

__device__ __forceinline__ RowBins row_bins(const ScanParams& p, int64_t r) {
  RowBins b;
  const float t0 = seed_tau(p, r);
  b.on = t0 > -INFINITY;
  b.lo = b.on ? t0 : 0.f;
  const float span = b.on ? key_to_float(p.smax_key[r]) - b.lo : 0.f;
  b.w = span > 0.f ? span * (1.f / kBins) : 0.f;
  b.inv_w = span > 0.f ? (float)kBins / span : 0.f;
  b.t0 = t0;
  return b;
}

__device__ __forceinline__ uint32_t load_tau_run(const ScanParams& p, int64_t r) {
  return *reinterpret_cast<const volatile uint32_t*>(p.tau_run + r);
}

// Current threshold of row r: the seed bound or the shared histogram's, the
// larger (an untouched shared key reads as NaN, which fmaxf ignores).
__device__ __forceinline__ float row_tau(float t0, uint32_t run_key) {
  return fmaxf(t0, key_to_float(run_key));
}

// Barrier `id` over `nthreads` threads that returns whether any of them passed
// pred = true (every participant gets the same answer).
__device__ __forceinline__ bool bar_any(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Work unit u: item u / parts (kDecRows consecutive rows), key tiles
// [n_tiles * part / parts, n_tiles * (part + 1) / parts) of it.
struct Unit {
  int64_t local0, t0, pos_first;
  int nq, tile_lo, tile_hi;
};

__device__ __forceinline__ Unit scan_unit(const ScanParams& p, int u) {
  Unit x;
  const int item = u / p.parts, part = u % p.parts;
  x.local0 = (int64_t)item * kDecRows;
  x.t0 = p.row0 + x.local0;
  const int64_t left = p.rows - x.local0;
  x.nq = (int)(left < kDecRows ? left : kDecRows);
  x.pos_first = p.pos0 + x.local0;
  const int nt = (int)((x.pos_first + x.nq - 1) / kKeyTile) + 1;
  x.tile_lo = (int)((int64_t)nt * part / p.parts);
  x.tile_hi = (int)((int64_t)nt * (part + 1) / p.parts);
  return x;
}

// kHeads: heads per query row (32 or 64); the MMA always sees 64 head slots.
template <bool kFp8, int kHeads>
__global__ void __launch_bounds__(ScanCfg<kFp8>::kThreads, 1)
    decode_scan_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap, const ScanParams p) {
  using C = ScanCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + C::kKeyStages * C::kKeyStageBytes);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* acc_full = bars + 2;     // [2]
  uint64_t* acc_empty = bars + 4;    // [2]
  uint64_t* done_bar = bars + 6;
  uint64_t* k_full = bars + 7;                   // [kKeyStages]
  uint64_t* k_empty = k_full + C::kKeyStages;    // [kKeyStages]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(k_empty + C::kKeyStages);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = p.n_items * p.parts;
  __shared__ float s_hold[C::kEpiWarps][2][C::kHoldT][32];   // [warp][row][team tile mod kHoldT][lane]
  __shared__ unsigned s_hist[kDecRows][kBins];            // this CTA's counts not yet moved
  __shared__ float s_tau[kDecRows];                       // the CTA's view of the shared threshold
  __shared__ unsigned s_done;                             // epilogue warps done, over all units
  __shared__ float4 s_w[kDecRows][16];                    // the unit's head weights (64 per row)
  for (int i = threadIdx.x; i < kDecRows * kBins; i += blockDim.x) (&s_hist[0][0])[i] = 0u;
  if (threadIdx.x < kDecRows) s_tau[threadIdx.x] = -INFINITY;
  if (threadIdx.x == 0) s_done = 0u;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps / 2);   // one team per accumulator
    }
    mbar_init(done_bar, 1);
    for (int i = 0; i < C::kKeyStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    *s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t kc = 0;
      int it = 0;
      bool ok = true;
      uint32_t inflight_q = 0xFFFFFFFFu;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit x = scan_unit(p, u);
        if (x.tile_hi <= x.tile_lo) continue;
        if (!mbar_wait(q_empty, (it & 1) ^ 1, s_abort, p.err)) break;
        mbar_arrive_expect_tx(q_full, C::kQBytes);
        for (int sub = 0; sub < C::kSub; ++sub)
          tma_load_3d(sQ + sub * C::kQSubBytes, &qmap, q_full, sub * 64, 0, (int32_t)x.t0);
        inflight_q = it & 1;
        ++it;
        for (int j = x.tile_lo; j < x.tile_hi; ++j, ++kc) {
          const int s_ = kc % C::kKeyStages;
          if (!mbar_wait(&k_empty[s_], ((kc / C::kKeyStages) & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s_], C::kKeyStageBytes);
          for (int sub = 0; sub < C::kSub; ++sub)
            tma_load_2d(sK + s_ * C::kKeyStageBytes + sub * C::kKeySubBytes, &kmap, &k_full[s_],
                        sub * 64, j * kKeyTile);
        }
      }
      if (*s_abort) {
        if (inflight_q != 0xFFFFFFFFu) mbar_wait_drain(q_full, inflight_q);
        for (uint32_t c = (kc > (uint32_t)C::kKeyStages ? kc - C::kKeyStages : 0); c < kc; ++c)
          mbar_wait_drain(&k_full[c % C::kKeyStages], (c / C::kKeyStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: one 128 x 256 tile per key tile ----------------
      constexpr uint32_t idesc = make_idesc<kFp8>(kKeyTile, C::kQRows);
      uint32_t kc = 0;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit x = scan_unit(p, u);
        if (x.tile_hi <= x.tile_lo) continue;
        if (!mbar_wait(q_full, it & 1, s_abort, p.err)) break;
        ++it;
        tc_fence_after();
        const uint32_t b_base = smem_u32(sQ);
        for (int j = x.tile_lo; j < x.tile_hi; ++j, ++kc) {
          const int s_ = kc % C::kKeyStages;
          const uint32_t buf = kc & 1;
          if (!mbar_wait(&k_full[s_], (kc / C::kKeyStages) & 1, s_abort, p.err) ||
              !mbar_wait(&acc_empty[buf], ((kc >> 1) & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + s_ * C::kKeyStageBytes);
          const uint32_t d = tmem_base + buf * C::kQRows;
#pragma unroll
          for (int step = 0; step < C::kKSteps; ++step) {
            const uint32_t sub = step >> 2, off = (step & 3) * 32;
            tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                         smem_desc_sw128(b_base + sub * C::kQSubBytes + off), idesc,
                         step > 0 ? 1u : 0u);
          }
          tc_commit(&acc_full[buf]);
          tc_commit(&k_empty[s_]);
        }
        tc_commit(q_empty);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else if (warp < C::kTauWarp) {
    // ---------------- epilogue: two teams of 8 warps ----------------
    // Team t drains accumulator t, i.e. the key tiles the CTA takes at even
    // or odd counts, so the two teams' TMEM loads and arithmetic interleave.
    // Warp (2 + ew) reads TMEM lane quadrant (warp & 3) for rows 2 rp and
    // 2 rp + 1 of the item (rp = ew >> 3): two reductions per wait.
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int team = (ew >> 2) & 1;
    const int rp = ew >> 3;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t kc = 0;
    unsigned long long n_exact = 0, n_cand = 0;
    bool ok = true;
    float(*hold)[C::kHoldT][32] = s_hold[ew];
    const volatile float* vtau = s_tau;
    constexpr bool h64 = kHeads == 64;
    constexpr int D = C::kHoldT - 1;          // team tiles an append trails by
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit x = scan_unit(p, u);
      if (x.tile_hi <= x.tile_lo) {
        continue;
      }
      bool valid[2];
      int64_t rr[2], pos[2];
      RowBins bins[2];
      const float* wq[2];
      float qs[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int sub = 2 * rp + k;
        valid[k] = sub < x.nq;
        rr[k] = x.local0 + (valid[k] ? sub : 0);
        pos[k] = x.pos_first + sub;
        bins[k] = row_bins(p, rr[k]);
        wq[k] = p.w + (x.t0 + (valid[k] ? sub : 0)) * kHeads;
        qs[k] = 1.f;
        if constexpr (kFp8) qs[k] = __ldg(p.q_scale + x.t0 + (valid[k] ? sub : 0));
      }
      // Appends trail the scores by D of this team's tiles (2 D tiles): a
      // tile's kept scores wait in shared memory until then, by which time
      // the threshold reflects the counts of that tile from every CTA, so the
      // first tiles are filtered by the K-th largest of everything scored so
      // far rather than by the seed bound alone.
      // Appends are staged in registers, one pending entry per lane and row
      // (lanes 0 .. pend - 1), and written 32 at a time: one reservation on
      // the row's shared count per 32 entries instead of one per append (all
      // CTAs update the same few counts), and an exact one at the unit's end.
      float ps[2] = {0.f, 0.f};
      int pk[2] = {0, 0}, pend[2] = {0, 0};
      auto flush = [&](int k, int cnt) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&p.count[rr[k]], cnt);
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        if (lane < cnt && base + lane < p.cap) p.cand[rr[k] * p.cap + base + lane] = Cand{ps[k], pk[k]};
        n_cand += cnt;
      };
      // new entries (lanes of am, in lane order) into the pending lanes from
      // `first`: entry j goes to lane first + j, for j < count
      auto stage = [&](int k, unsigned am, float sc, int key0, int first, int from, int count) {
        const int j = lane - first;
        const bool mine = j >= 0 && j < count;
        const int src = mine ? (int)__fns(am, 0, from + j + 1) : 0;
        const float v = __shfl_sync(0xFFFFFFFFu, sc, src);
        if (mine) {
          ps[k] = v;
          pk[k] = key0 + src;
        }
      };
      auto append_held = [&](int k, int slot, int key0, float tau) {
        const float sc = hold[k][slot][lane];
        const unsigned am = __ballot_sync(0xFFFFFFFFu, sc >= tau);
        if (!am) return;
        const int n = __popc(am);
        const int fill = n < 32 - pend[k] ? n : 32 - pend[k];
        stage(k, am, sc, key0, pend[k], 0, fill);
        pend[k] += fill;
        if (pend[k] == 32) {
          flush(k, 32);
          pend[k] = n - fill;
          if (pend[k] > 0) stage(k, am, sc, key0, 0, fill, pend[k]);
        }
      };
      // the unit's weights into shared memory, once per unit (warps 0 and 8
      // of the epilogue write their two rows; the previous unit's readers are
      // past the barrier that ended it)
      if ((ew & 7) == 0) {
        float* sw = reinterpret_cast<float*>(s_w[2 * rp]);
#pragma unroll
        for (int k = 0; k < 2; ++k)
          for (int hh = lane; hh < 64; hh += 32) sw[k * 64 + hh] = hh < kHeads ? __ldg(wq[k] + hh) : 0.f;
      }
      asm volatile("bar.sync 2, %0;" ::"n"(C::kEpiWarps * 32) : "memory");
      // this team's first tile of the unit (tiles alternate between teams)
      const int j_first = x.tile_lo + (int)(((uint32_t)team - kc) & 1u);
      float sk_next = 1.f;
      if constexpr (kFp8) {
        const int s0 = j_first * kKeyTile + quad * 32 + lane;
        sk_next = (j_first < x.tile_hi && s0 < p.S) ? __ldg(p.k_scale + s0) : 0.f;
      }
      int m = 0;                                  // this team's tiles of the unit so far
      int j_last = -1;
      for (int j = j_first; j < x.tile_hi && ok; j += 2, ++m) {
        const uint32_t kt = kc + (uint32_t)(j - x.tile_lo);   // the CTA's count of this tile
        const int s = j * kKeyTile + quad * 32 + lane;
        const float sk = sk_next;
        if constexpr (kFp8) {
          const int sn = s + 2 * kKeyTile;
          sk_next = (j + 2 < x.tile_hi && sn < p.S) ? __ldg(p.k_scale + sn) : 0.f;
        }
        if (!mbar_wait(&acc_full[team], (kt >> 1) & 1, s_abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col = tmem_base + lane_off + team * C::kQRows + (2 * rp) * 64;
        HeadAcc2 acc[2] = {{make_float2(0.f, 0.f), make_float2(0.f, 0.f)},
                           {make_float2(0.f, 0.f), make_float2(0.f, 0.f)}};
        constexpr int kQuarters = h64 ? 4 : 2;
#pragma unroll
        for (int hq = 0; hq < kQuarters; ++hq) {
          float xa[16], xb[16];
          float4 w4[4];
          tmem_ld16_async(col + 16 * hq, xa);
          tmem_ld16_async(col + 64 + 16 * hq, xb);
          tmem_wait_ld16(xa);
          tmem_wait_ld16(xb);
          if (hq == kQuarters - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[team]);
          }
#pragma unroll
          for (int m4 = 0; m4 < 4; ++m4) w4[m4] = s_w[2 * rp][4 * hq + m4];
          head_accumulate16w(acc[0], xa, w4);
#pragma unroll
          for (int m4 = 0; m4 < 4; ++m4) w4[m4] = s_w[2 * rp + 1][4 * hq + m4];
          head_accumulate16w(acc[1], xb, w4);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (!valid[k]) continue;
          float sc = head_total(acc[k]);
          if constexpr (kFp8) sc *= qs[k] * sk;
          const int sub = 2 * rp + k;
          const float tau = fmaxf(bins[k].t0, vtau[sub]);
          const bool vis = s <= pos[k];
          n_exact += __popc(__ballot_sync(0xFFFFFFFFu, vis));
          const bool keep = vis && sc >= tau;
          if (bins[k].on && __any_sync(0xFFFFFFFFu, keep)) {
            // count the kept scores in the CTA's histogram, one shared-memory
            // atomic per distinct bin of the warp
            const int bin = keep ? bin_index(bins[k].lo, bins[k].inv_w, sc) : -1;
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
            if (keep && lane == __ffs(peers) - 1)
              atomicAdd(&s_hist[sub][bin], (unsigned)__popc(peers));
          }
          hold[k][m % C::kHoldT][lane] = keep ? sc : -INFINITY;
          if (m >= D) append_held(k, (m - D) % C::kHoldT, s - 2 * D * kKeyTile - lane, tau);
        }
        j_last = j;
      }
      // this team's last D tiles of the unit, then what is still pending
      if (ok && m > 0) {
        for (int k = 0; k < 2; ++k) {
          if (!valid[k]) continue;
          const float tau = fmaxf(bins[k].t0, vtau[2 * rp + k]);
          for (int mm = (m > D ? m - D : 0); mm < m; ++mm)
            append_held(k, mm % C::kHoldT, (j_last - 2 * (m - 1 - mm)) * kKeyTile + quad * 32, tau);
        }
      }
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (pend[k] > 0) flush(k, pend[k]);
      kc += (uint32_t)(x.tile_hi - x.tile_lo);
      __syncwarp();
      __threadfence_block();
      if (lane == 0) atomicAdd(&s_done, 1u);
      if (bar_any(1, C::kUnitThreads, !ok || *s_abort)) break;
    }
    if (lane == 0) {
      atomicAdd(&p.counters[kCntExact], n_exact);
      atomicAdd(&p.counters[kCntFiltered], n_exact);
      atomicAdd(&p.counters[kCntCandidates], n_cand);
    }
  } else {
    // ---------------- threshold warp ----------------
    // Moves the CTA's counts into the rows' global histograms (exchange with
    // zero, then add) and sets the CTA's threshold to the best of its own
    // reading of the global histogram and the shared threshold, until the
    // epilogue warps finish the unit; then a last move, and the next unit.
    volatile float* vtau = s_tau;
    const volatile unsigned* vdone = &s_done;
    unsigned target = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit x = scan_unit(p, u);
      if (x.tile_hi <= x.tile_lo) continue;
      target += C::kEpiWarps;
      const unsigned long long t_start = global_ns();
      RowBins rb[kDecRows];
#pragma unroll
      for (int q = 0; q < kDecRows; ++q) {
        rb[q] = row_bins(p, x.local0 + (q < x.nq ? q : 0));
        rb[q].on = rb[q].on && q < x.nq;
      }
      for (;;) {
        const bool last = *vdone >= target || *s_abort;
        __threadfence_block();
        // all rows at once: one round trip to L2 per pass
        unsigned c[kDecRows][8];
        uint32_t run[kDecRows];
#pragma unroll
        for (int q = 0; q < kDecRows; ++q) {
          if (!rb[q].on) continue;
          const int64_t r = x.local0 + q;
          // bins i * 32 + lane: consecutive lanes, no bank conflicts
#pragma unroll
          for (int i = 0; i < 8; ++i) c[q][i] = atomicExch(&s_hist[q][i * 32 + lane], 0u);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (c[q][i]) atomicAdd(&p.hist[r * kBins + i * 32 + lane], c[q][i]);
        }
#pragma unroll
        for (int q = 0; q < kDecRows; ++q) {
          if (!rb[q].on) continue;
          const int64_t r = x.local0 + q;
          load_bins(p.hist + r * kBins, lane, c[q]);
          run[q] = load_tau_run(p, r);
        }
#pragma unroll
        for (int q = 0; q < kDecRows; ++q) {
          if (!rb[q].on) continue;
          const int best = suffix_bin_of(c[q], p.K, lane);
          const uint32_t mine = best >= 0 ? ordered_key(bin_edge_at(rb[q].lo, rb[q].w, best)) : 0u;
          const uint32_t cur = run[q] > mine ? run[q] : mine;
          if (lane == 0) {
            if (mine > run[q]) atomicMax(&p.tau_run[x.local0 + q], mine);
            if (cur) vtau[q] = fmaxf(vtau[q], key_to_float(cur));
          }
        }
        __syncwarp();
        if (last) break;
        if (global_ns() - t_start > kWaitLimitNs) {
          record_error(p.err, kDevTimeout);
          *s_abort = 1;
        }
      }
      if (lane < kDecRows) vtau[lane] = -INFINITY;     // the next unit's rows
      if (bar_any(1, C::kUnitThreads, *s_abort != 0)) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Per row (one warp): the count for the selection kernel (one segment) and
// the final threshold, from the complete histogram.
__global__ void decode_finish_kernel(const ScanParams p, int* cand_count, float* tau_out) {
  const int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= p.rows) return;
  const RowBins b = row_bins(p, r);
  float tau = row_tau(seed_tau(p, r), load_tau_run(p, r));
  if (b.on) {
    const int best = suffix_bin(p.hist + r * kBins, p.K, lane);
    if (best >= 0) tau = fmaxf(tau, bin_edge_at(b.lo, b.w, best));
  }
  if (lane == 0) {
    const int cnt = p.count[r];
    int* cc = cand_count + r * 4;
    if (cnt > p.cap) record_error(p.err, kDevBounds);     // never: a list holds every key
    cc[0] = cnt > p.cap ? p.cap : cnt;
    cc[1] = 0;
    cc[2] = 0;
    cc[3] = 0;
    tau_out[r] = tau;
  }
}

// ---- host side ---------------------------------------------------------------------

template <bool kFp8>
static cudaError_t launch_decode_impl(const Handle& h, const SeqView& v, const DecodeBuffers& b,
                                      int K, const int32_t* seed, cudaStream_t stream) {
  using C = ScanCfg<kFp8>;
  if (v.rows <= 0) return cudaSuccess;
  // seeds
  SeedParams sp;
  sp.q = v.q;
  sp.q_scale = v.q_scale;
  sp.w = v.w;
  sp.k = v.k;
  sp.k_scale = v.k_scale;
  sp.seed = seed;
  sp.row0 = v.row0;
  sp.rows = v.rows;
  sp.pos0 = v.pos0;
  sp.S = v.S;
  sp.K = K;
  sp.H = v.H;
  sp.bitmap = b.bitmap;
  sp.words = b.words;
  sp.tau_key = b.tau_key;
  sp.smax_key = b.smax_key;
  sp.seed_count = b.seed_count;
  sp.dup = b.dup;
  static bool seed_attr = false;
  cudaError_t e;
  if (!seed_attr) {
    e = cudaFuncSetAttribute(decode_seed_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSeedSmem);
    if (e != cudaSuccess) return e;
    seed_attr = true;
  }
  profile_before(DOSA_KERNEL_DECODE, stream);
  decode_seed_kernel<kFp8><<<dim3((unsigned)v.rows, (unsigned)((K + kSeedKeys - 1) / kSeedKeys)),
                             256, kSeedSmem, stream>>>(sp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // scan
  CUtensorMap qmap, kmap;
  if (!encode_q_map(&qmap, v.q, kFp8, (uint64_t)(v.row0 + v.rows), v.H) ||
      !encode_rows_map(&kmap, v.k, kFp8, (uint64_t)v.S, kKeyTile))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(decode_scan_kernel<kFp8, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_scan_kernel<kFp8, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  ScanParams p;
  p.w = v.w;
  p.q_scale = v.q_scale;
  p.k_scale = v.k_scale;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.H = v.H;
  p.n_items = (int)((v.rows + kDecRows - 1) / kDecRows);
  // about one unit per SM (the key pipeline restarts at each unit), at least
  // 16 key tiles per unit
  const int64_t tiles = (v.pos0 + v.rows - 1) / kKeyTile + 1;
  int64_t parts = ((int64_t)sms + p.n_items - 1) / p.n_items;
  if (parts > tiles / 16) parts = tiles / 16;
  if (parts < 1) parts = 1;
  p.parts = (int)parts;
  p.K = K;
  p.tau_key = b.tau_key;
  p.smax_key = b.smax_key;
  p.seed_count = b.seed_count;
  p.dup = b.dup;
  p.hist = b.hist;
  p.tau_run = b.tau_run;
  p.cand = reinterpret_cast<Cand*>(b.cand);
  p.cap = b.cap;
  p.count = b.count;
  p.counters = b.counters;
  p.err = b.err;
  const int units = p.n_items * p.parts;
  const int grid = units < sms ? units : sms;
  if (v.H == 64)
    decode_scan_kernel<kFp8, 64><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, kmap, p);
  else
    decode_scan_kernel<kFp8, 32><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, kmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_finish_kernel<<<(unsigned)((v.rows + 3) / 4), 128, 0, stream>>>(p, b.cand_count, b.tau);
  e = cudaGetLastError();
  profile_after(DOSA_KERNEL_DECODE, stream);
  return e;
}

cudaError_t launch_decode(const Handle& h, const SeqView& v, const DecodeBuffers& b, int K,
                          const int32_t* seed, cudaStream_t stream) {
  if (h.cfg.dtype == DOSA_FP8_E4M3) return launch_decode_impl<true>(h, v, b, K, seed, stream);
  return launch_decode_impl<false>(h, v, b, K, seed, stream);
}

}  // namespace dosa
