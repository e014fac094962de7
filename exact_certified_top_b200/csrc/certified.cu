// Certified indexer scorer for sm_100a: screening, rescoring and sparse
// writeback fused in one persistent tcgen05 kernel ("DOSA: Dots Sparse
// Attention", Daily Paper Cast transcript, Method section: candidate
// refinement = screening dot products, bound evaluation, pruning and score
// compaction, repeated for every tile of visible keys and query tiles; GPU
// kernel design: fixed-width query tiles on tensor cores, survivor masks
// compacted into shared streams so key loads are not repeated, full-score
// computation fused with threshold filtering and packed writeback).
//
// Work item = 8 consecutive query rows.  Resident in shared memory: their
// 8 x 64 head rows and their 8 x 8 bound rows (4 retained heads, u_1 hi/lo,
// u_2 hi/lo, from cert_setup).  For each key tile of 128 keys (tile 0 first,
// which holds the first seed keys, then from the diagonal downwards):
//   1. bound MMA   D_b[128 keys x 64] = keys x bound rows            (N = 64)
//   2. bound epilogue: UB(t,s) per (key, query); a key survives when it is a
//      seed, when the query is still warming up (fewer than K exact scores),
//      or when UB + margin >= tau_t.  Survivor masks go to shared memory.
//   3. exact MMA for each pair of queries with at least one survivor
//      D_e[128 keys x 128] = keys x (2 queries x 64 heads)           (N = 128)
//   4. exact epilogue on survivors only: the same head reduction as the
//      dense scorer (bit-identical scores); scores >= tau_t are appended as
//      packed (score, key) pairs to the query's candidate list.
//   5. tile barrier; the warp that owns each query refreshes tau_t.
// tau_t is a lower bound on the K-th largest exact score so far: during
// warm-up it is -inf; once K candidates exist the owner bins them into a
// 256-bin histogram over [min, max] and from then on tau_t is the (rounded
// down) lower edge of the highest bin whose suffix count reaches K.  Every
// candidate counted there has a score >= that edge, so at least K exact scores
// are >= tau_t: rejecting UB + margin < tau_t never drops a Top-K key, and a
// key tied with the K-th score is never rejected.
#include "cert_layout.h"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "score_epilogue.cuh"

namespace dosa {

constexpr int kBins = 256;
// Adaptive screening: decided once per work item, after at least this many
// screened pairs; screening stops when fewer than 1 in kAdaptiveRejectRatio
// screened pairs were rejected.
constexpr unsigned long long kAdaptiveMinScreened = 4096;
constexpr unsigned long long kAdaptiveRejectRatio = 32;
// Epilogue warps meet (threshold refresh, adaptive decision) every this many
// key tiles and at the last tile of a work item.
constexpr int kCkptTiles = 4;

struct QState {
  float tau;
  int phase;          // 0 = unused slot, 1 = warm-up, 2 = screening
  int count;          // candidates reserved (may exceed the capacity)
  int overflow;
  float lo, inv_w, w;
  float omega[4];
  float beta, margin;
  float scale[4];
  float sq;
  long long pos;      // position of the query among the sequence's keys
  long long row;      // chunk-local row
  unsigned hist[kBins];
};

template <bool kFp8>
struct CertCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kKeyStages = kFp8 ? 4 : 2;
  static constexpr int kH = 64;
  static constexpr int kQT = 8;
  static constexpr int kQRows = kQT * kH;
  static constexpr int kBRows = kQT * kBoundRows;      // 64
  static constexpr int kGroupN = 2 * kH;               // 128 columns = 2 queries
  static constexpr int kGroups = kQT / 2;
  static constexpr uint32_t kKeySubBytes = kKeyTile * 128;
  static constexpr uint32_t kKeyStageBytes = kKeySubBytes * kSub;
  static constexpr uint32_t kQSubBytes = kQRows * 128;
  static constexpr uint32_t kQBytes = kQSubBytes * kSub;
  static constexpr uint32_t kBSubBytes = kBRows * 128;
  static constexpr uint32_t kBBytes = kBSubBytes * kSub;
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 64 + kEpiWarps * 32;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kAccBufs = 3;
  static constexpr uint32_t kAccCol = 0;       // three 128-column exact accumulators
  static constexpr uint32_t kBndCol = 384;     // two 64-column bound accumulators
  static constexpr uint32_t kStateBytes = sizeof(QState) * kQT;
  static constexpr uint32_t kMiscBytes = 1024;  // barriers, masks, flags
  static constexpr uint32_t kSmemBytes =
      1024 + kQBytes + kBBytes + kKeyStages * kKeyStageBytes + kStateBytes + kMiscBytes;
};

struct Cand {
  float score;
  int key;
};

struct CertParams {
  const float* w;          // [rows_total, 64] absolute rows
  const float* q_scale;    // absolute rows (fp8)
  const float* k_scale;    // sequence base (fp8)
  const float* key_norm;   // [S] code-domain ||k||, rounded up
  const float* cert;       // [chunk rows, kCertFloats]
  Cand* cand;              // [chunk rows, cap]
  int* cand_count;         // [chunk rows]
  float* tau_out;          // [chunk rows]
  int* repair_list;        // [repair_cap] chunk-local rows whose list overflowed
  int* repair_count;
  int repair_cap;
  unsigned long long* counters;
  int* err;
  int64_t row0, rows, pos0, S;   // chunk: absolute first row, rows, first position
  int n_items, K, cap, seed_first, seed_last, screening;
};

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

struct Geom {
  int64_t t0;        // absolute first row
  int64_t local0;    // chunk-local first row
  int nq;
  int64_t pos_first;
  int n_tiles;       // key tiles 0..n_tiles-1
};

__device__ __forceinline__ Geom cert_geom(const CertParams& p, int item) {
  Geom g;
  const int tile = p.n_items - 1 - item;       // longest rows first
  g.local0 = (int64_t)tile * 8;
  g.t0 = p.row0 + g.local0;
  const int64_t left = p.rows - g.local0;
  g.nq = (int)(left < 8 ? left : 8);
  g.pos_first = p.pos0 + g.local0;
  g.n_tiles = (int)((g.pos_first + g.nq - 1) / kKeyTile) + 1;
  return g;
}

// Processing order of key tiles: tile 0 (the first seed keys), then from the
// diagonal tile downwards.
__device__ __forceinline__ int tile_at(int ti, int n_tiles) {
  return ti == 0 ? 0 : n_tiles - ti;
}

// Sound lower edge of bin i: every score binned at >= i is >= the result.
__device__ __forceinline__ float bin_edge(const QState& s, int i) {
  const float iw = (float)i * s.w;
  return fmaf((float)i, s.w, s.lo) - (fabsf(s.lo) + iw) * 0x1p-20f;
}

__device__ __forceinline__ int bin_of(const QState& s, float score) {
  float b = floorf((score - s.lo) * s.inv_w);
  b = fminf(fmaxf(b, 0.f), (float)(kBins - 1));
  return (int)b;
}

// Owner warp: highest bin whose suffix count reaches K -> its sound edge
// (or -inf when fewer than K are counted).
__device__ float hist_threshold(const QState& s, int K, int lane) {
  unsigned c[8], local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = *reinterpret_cast<const volatile unsigned*>(&s.hist[lane * 8 + j]);
    local += c[j];
  }
  unsigned suf = local;   // sum over lanes >= this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned n = __shfl_down_sync(0xFFFFFFFFu, suf, o);
    if (lane + o < 32) suf += n;
  }
  const unsigned above = suf - local;
  int best = -1;
  if (above < (unsigned)K && suf >= (unsigned)K) {
    unsigned acc = above;
    for (int j = 7; j >= 0; --j) {
      acc += c[j];
      if (acc >= (unsigned)K) {
        best = lane * 8 + j;
        break;
      }
    }
  }
  // exactly one lane can hold the answer
  const unsigned who = __ballot_sync(0xFFFFFFFFu, best >= 0);
  if (!who) return -INFINITY;
  const int src = __ffs(who) - 1;
  best = __shfl_sync(0xFFFFFFFFu, best, src);
  return bin_edge(s, best);
}

template <bool kFp8>
__global__ void __launch_bounds__(CertCfg<kFp8>::kThreads, 1)
    certified_kernel(const __grid_constant__ CUtensorMap qmap,
                     const __grid_constant__ CUtensorMap bmap,
                     const __grid_constant__ CUtensorMap kmap, const CertParams p) {
  using C = CertCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sB = sQ + C::kQBytes;
  uint8_t* sK = sB + C::kBBytes;
  QState* st = reinterpret_cast<QState*>(sK + C::kKeyStages * C::kKeyStageBytes);
  uint8_t* misc = reinterpret_cast<uint8_t*>(st + C::kQT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* bnd_full = bars + 2;     // [2]
  uint64_t* bnd_empty = bars + 4;    // [2]
  uint64_t* acc_full = bars + 6;     // [3]
  uint64_t* acc_empty = bars + 9;    // [3]
  // mask_ready is double-buffered by tile parity: with one barrier, a tile
  // without survivors lets the epilogue complete the next tile's phase before
  // the MMA thread polls for this one, and a parity wait would then block.
  uint64_t* mask_ready = bars + 12;  // [2]
  uint64_t* tile_done = bars + 14;
  uint64_t* item_ready = bars + 15;
  uint64_t* done_bar = bars + 16;
  uint64_t* k_full = bars + 17;                    // [kKeyStages]
  uint64_t* k_empty = k_full + C::kKeyStages;      // [kKeyStages]
  // Survivor masks and query-pair flags of a screened tile, three slots: a
  // slot is rewritten (bound evaluation of tile b+3) only after every warp has
  // passed the bound evaluation of tile b+2, which follows its exact stage of b.
  uint32_t* masks = reinterpret_cast<uint32_t*>(k_empty + C::kKeyStages);  // [3][8][4]
  uint32_t* gflag = masks + 3 * 8 * 4;                                      // [3][8]
  uint32_t* s_tmem = gflag + 3 * 8;
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* stop_word = reinterpret_cast<int*>(s_tmem + 2);             // first unscreened tile
  unsigned long long* snap = reinterpret_cast<unsigned long long*>(s_tmem + 4);  // [2][8][2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bnd_full[i], 1);
      mbar_init(&bnd_empty[i], C::kEpiWarps);
    }
    for (int i = 0; i < C::kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(&mask_ready[0], C::kEpiWarps);
    mbar_init(&mask_ready[1], C::kEpiWarps);
    mbar_init(tile_done, C::kEpiWarps);
    mbar_init(item_ready, C::kEpiWarps);
    mbar_init(done_bar, 1);
    for (int i = 0; i < C::kKeyStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    *s_abort = 0;
    *stop_word = 0x7FFFFFFF;
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&bmap);
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
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
        const Geom g = cert_geom(p, item);
        if (!mbar_wait(q_empty, (it & 1) ^ 1, s_abort, p.err)) break;
        mbar_arrive_expect_tx(q_full, C::kQBytes + C::kBBytes);
        for (int sub = 0; sub < C::kSub; ++sub) {
          for (int b = 0; b < C::kQRows / 256; ++b)
            tma_load_2d(sQ + sub * C::kQSubBytes + b * 256 * 128, &qmap, q_full, sub * 64,
                        (int32_t)(g.t0 * C::kH + b * 256));
          tma_load_2d(sB + sub * C::kBSubBytes, &bmap, q_full, sub * 64,
                      (int32_t)(g.local0 * kBoundRows));
        }
        inflight_q = it & 1;
        for (int ti = 0; ti < g.n_tiles; ++ti, ++kc) {
          const int s_ = kc % C::kKeyStages;
          const uint32_t rnd = kc / C::kKeyStages;
          if (!mbar_wait(&k_empty[s_], (rnd & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s_], C::kKeyStageBytes);
          const int j = tile_at(ti, g.n_tiles);
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
      // ---------------- MMA issuer ----------------
      // Order per item: bound(0); then for each tile t: bound(t+1), [wait for
      // tile t's survivor masks], exact(t).  The epilogue screens one tile
      // ahead, so tile t's exact MMAs run while tile t+1's bounds are
      // evaluated.  Screened tiles form a prefix of the processing order: all
      // of them (screening = 1), none (0), or those before the item's stop
      // tile (2, adaptive), which the epilogue publishes in *stop_word before
      // its mask arrival for the tile that precedes this thread's last use.
      constexpr uint32_t idesc_b = make_idesc<kFp8>(kKeyTile, C::kBRows);
      constexpr uint32_t idesc_e = make_idesc<kFp8>(kKeyTile, C::kGroupN);
      uint32_t kc = 0, nb = 0, u = 0;
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
        const Geom g = cert_geom(p, item);
        if (!mbar_wait(q_full, it & 1, s_abort, p.err)) break;
        tc_fence_after();
        const uint32_t b_bound = smem_u32(sB);
        // (a decision never stops before tile 4, so tiles 0-3 need no read)
        auto screened = [&](int t) -> bool {
          if (p.screening == 0) return false;
          if (p.screening == 1) return true;
          return t < 4 || t < *reinterpret_cast<volatile int*>(stop_word);
        };
        auto issue_bound = [&](int t) -> bool {
          const uint32_t c = kc + t, s_ = c % C::kKeyStages, b = nb + t;
          if (!mbar_wait(&k_full[s_], (c / C::kKeyStages) & 1, s_abort, p.err) ||
              !mbar_wait(&bnd_empty[b & 1], ((b >> 1) & 1) ^ 1, s_abort, p.err))
            return false;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + s_ * C::kKeyStageBytes);
          const uint32_t d = tmem_base + C::kBndCol + (b & 1) * C::kBRows;
#pragma unroll
          for (int step = 0; step < C::kKSteps; ++step) {
            const uint32_t sub = step >> 2, off = (step & 3) * 32;
            tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                         smem_desc_sw128(b_bound + sub * C::kBSubBytes + off), idesc_b,
                         step > 0 ? 1u : 0u);
          }
          tc_commit(&bnd_full[b & 1]);
          return true;
        };
        bool scr_cur = screened(0);
        if (scr_cur && !issue_bound(0)) break;
        int n_scr = scr_cur ? 1 : 0;
        for (int ti = 0; ti < g.n_tiles && ok; ++ti) {
          bool scr_next = false;
          if (ti + 1 < g.n_tiles) {
            scr_next = scr_cur && screened(ti + 1);
            if (scr_next) {
              if (!issue_bound(ti + 1)) {
                ok = false;
                break;
              }
              ++n_scr;
            }
          }
          // exact MMAs of tile ti
          const uint32_t c = kc + ti, s_ = c % C::kKeyStages;
          uint32_t groups;
          if (scr_cur) {
            const uint32_t b = nb + ti;
            if (!mbar_wait(&mask_ready[b & 1], (b >> 1) & 1, s_abort, p.err)) {
              ok = false;
              break;
            }
            groups = 0;
            for (int w = 0; w < C::kEpiWarps; ++w)
              groups |= reinterpret_cast<volatile uint32_t*>(gflag)[(b % 3) * 8 + w];
          } else {
            if (!mbar_wait(&k_full[s_], (c / C::kKeyStages) & 1, s_abort, p.err)) {
              ok = false;
              break;
            }
            groups = (1u << ((g.nq + 1) / 2)) - 1u;   // every pair with a valid query
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + s_ * C::kKeyStageBytes);
          for (int grp = 0; grp < C::kGroups && ok; ++grp) {
            if (!(groups >> grp & 1)) continue;
            const uint32_t ab = u % C::kAccBufs;
            if (!mbar_wait(&acc_empty[ab], ((u / C::kAccBufs) & 1) ^ 1, s_abort, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t b_base = smem_u32(sQ + grp * C::kGroupN * 128);
            const uint32_t d = tmem_base + C::kAccCol + ab * C::kGroupN;
#pragma unroll
            for (int step = 0; step < C::kKSteps; ++step) {
              const uint32_t sub = step >> 2, off = (step & 3) * 32;
              tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                           smem_desc_sw128(b_base + sub * C::kQSubBytes + off), idesc_e,
                           step > 0 ? 1u : 0u);
            }
            tc_commit(&acc_full[ab]);
            ++u;
          }
          tc_commit(&k_empty[s_]);
          scr_cur = scr_next;
        }
        kc += g.n_tiles;
        nb += n_scr;
        tc_commit(q_empty);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    // Order per item: bound(0); then for each tile t: bound(t+1), exact(t),
    // tile barrier, threshold refresh by each query's owner warp.
    const int ew = warp - 2;                 // owner of query slot ew
    const int quad = warp & 3;
    const int half = ew >> 2;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t nb = 0, u = 0, nbar = 0;
    int it = 0;
    unsigned long long n_seed = 0, n_screened = 0, n_rejected = 0, n_exact = 0, n_cand = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
      const Geom g = cert_geom(p, item);
      // owner: load this item's state of query slot ew
      {
        QState& s = st[ew];
        if (lane == 0) {
          const bool valid = ew < g.nq;
          s.tau = -INFINITY;
          s.phase = valid ? 1 : 0;
          s.count = 0;
          s.overflow = 0;
          s.lo = 0.f;
          s.inv_w = 0.f;
          s.w = 0.f;
          s.row = g.local0 + ew;
          s.pos = valid ? g.pos_first + ew : -1;
          const float* cf = p.cert + (valid ? s.row : 0) * kCertFloats;
          for (int j = 0; j < 4; ++j) {
            s.omega[j] = valid ? cf[kCertOmega + j] : 0.f;
            s.scale[j] = valid ? cf[kCertScale + j] : 0.f;
          }
          s.beta = valid ? cf[kCertBeta] : 0.f;
          s.margin = valid ? cf[kCertMargin] : 0.f;
          s.sq = (kFp8 && valid) ? __ldg(p.q_scale + g.t0 + ew) : 1.f;
          if (ew == 0) *reinterpret_cast<volatile int*>(stop_word) = 0x7FFFFFFF;
        }
        for (int b = lane; b < kBins; b += 32) s.hist[b] = 0;
        __syncwarp();
        __threadfence_block();
        if (lane == 0) mbar_arrive(item_ready);
        if (!mbar_wait(item_ready, it & 1, s_abort, p.err)) break;
      }
      int stop = 0x7FFFFFFF;                 // first unscreened tile (adaptive mode)
      bool decided = p.screening != 2;
      unsigned long long it_scr = 0, it_rej = 0;   // this warp's screened/rejected, this item
      auto screened = [&](int t) -> bool {
        return p.screening == 1 || (p.screening == 2 && t < stop);
      };
      // key of this lane in tile ti
      auto key_of = [&](int ti) -> int64_t {
        return (int64_t)tile_at(ti, g.n_tiles) * kKeyTile + quad * 32 + lane;
      };
      // ---- bound evaluation of tile t (a screened tile) ----
      auto bound_eval = [&](int t) -> bool {
        const uint32_t b = nb + t;
        const int64_t s = key_of(t);
        const bool key_ok = s < p.S;
        const float nk = key_ok ? __ldg(p.key_norm + s) : 0.f;
        float sk = 1.f;
        if constexpr (kFp8) sk = key_ok ? __ldg(p.k_scale + s) : 0.f;
        if (!mbar_wait(&bnd_full[b & 1], (b >> 1) & 1, s_abort, p.err)) return false;
        tc_fence_after();
        float v[32];
        tmem_ld32(tmem_base + lane_off + C::kBndCol + (b & 1) * C::kBRows + half * 32, v);
        uint32_t gbits = 0;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int ql = half * 4 + qq;
          const QState& q = st[ql];
          const int phase = *reinterpret_cast<const volatile int*>(&q.phase);
          const bool vis = phase != 0 && key_ok && s <= q.pos;
          const bool seed = s < p.seed_first || s > q.pos - p.seed_last;
          const bool screen = vis && !seed && phase == 2;
          bool rej = false;
          if (screen) {
            const float* x = v + qq * 8;
            float ub = q.omega[0] * fmaxf(x[0], 0.f);
            ub = fmaf(q.omega[1], fmaxf(x[1], 0.f), ub);
            ub = fmaf(q.omega[2], fmaxf(x[2], 0.f), ub);
            ub = fmaf(q.omega[3], fmaxf(x[3], 0.f), ub);
            ub = fmaf(q.beta + q.margin, nk, ub);
            ub -= fmaxf(fmaf(q.scale[0], x[4], q.scale[1] * x[5]), 0.f);
            ub -= fmaxf(fmaf(q.scale[2], x[6], q.scale[3] * x[7]), 0.f);
            float sqk = 1.f;
            if constexpr (kFp8) sqk = q.sq * sk;
            const float tau = *reinterpret_cast<const volatile float*>(&q.tau);
            rej = ub * sqk < tau;
          }
          const bool surv = vis && !rej;
          const uint32_t mk = __ballot_sync(0xFFFFFFFFu, surv);
          const uint32_t scr = __popc(__ballot_sync(0xFFFFFFFFu, screen));
          const uint32_t rjm = __popc(__ballot_sync(0xFFFFFFFFu, rej));
          n_seed += __popc(__ballot_sync(0xFFFFFFFFu, vis && seed));
          n_screened += scr;
          n_rejected += rjm;
          it_scr += scr;
          it_rej += rjm;
          if (lane == 0) masks[((b % 3) * 8 + ql) * 4 + quad] = mk;
          if (mk) gbits |= 1u << (ql >> 1);
        }
        if (lane == 0) gflag[(b % 3) * 8 + ew] = gbits;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bnd_empty[b & 1]);
          mbar_arrive(&mask_ready[b & 1]);
        }
        return mbar_wait(&mask_ready[b & 1], (b >> 1) & 1, s_abort, p.err);
      };
      bool scr_cur = screened(0);
      int n_scr = scr_cur ? 1 : 0;
      if (scr_cur && !bound_eval(0)) break;
      for (int ti = 0; ti < g.n_tiles && ok; ++ti) {
        bool scr_next = false;
        if (ti + 1 < g.n_tiles) {
          scr_next = scr_cur && screened(ti + 1);
          if (scr_next) {
            if (!bound_eval(ti + 1)) {
              ok = false;
              break;
            }
            ++n_scr;
          }
        }
        // ---- exact scoring of tile ti's survivors, filter, packed writeback ----
        const int64_t s = key_of(ti);
        const bool key_ok = s < p.S;
        float sk = 1.f;
        if constexpr (kFp8) sk = key_ok ? __ldg(p.k_scale + s) : 0.f;
        uint32_t groups;
        const uint32_t b = nb + ti;
        if (scr_cur) {
          groups = 0;
          for (int w = 0; w < C::kEpiWarps; ++w)
            groups |= reinterpret_cast<volatile uint32_t*>(gflag)[(b % 3) * 8 + w];
        } else {
          groups = (1u << ((g.nq + 1) / 2)) - 1u;
        }
        for (int grp = 0; grp < C::kGroups; ++grp) {
          if (!(groups >> grp & 1)) continue;
          const uint32_t ab = u % C::kAccBufs;
          if (!mbar_wait(&acc_full[ab], (u / C::kAccBufs) & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int ql = grp * 2 + half;
          QState& q = st[ql];
          uint32_t mk;
          if (scr_cur) {
            mk = reinterpret_cast<volatile uint32_t*>(masks)[((b % 3) * 8 + ql) * 4 + quad];
          } else {
            const int phase = *reinterpret_cast<const volatile int*>(&q.phase);
            mk = __ballot_sync(0xFFFFFFFFu, phase != 0 && key_ok && s <= q.pos);
            if (p.screening == 2) {
              // pairs no longer screened still count as seeds when they are
              const bool seed = s < p.seed_first || s > q.pos - p.seed_last;
              n_seed += __popc(mk & __ballot_sync(0xFFFFFFFFu, seed));
            } else {
              const bool seed = s < p.seed_first || s > q.pos - p.seed_last;
              n_seed += __popc(mk & __ballot_sync(0xFFFFFFFFu, seed));
            }
          }
          if (mk) {
            float x[64];
            tmem_ld64(tmem_base + lane_off + C::kAccCol + ab * C::kGroupN + half * 64, x);
            const bool mine = (mk >> lane) & 1;
            float sc = 0.f;
            if (mine) {
              const int64_t t = g.t0 + ql;
              sc = head_reduce64(x, p.w + t * C::kH);
              if constexpr (kFp8) sc *= __ldg(p.q_scale + t) * sk;
            }
            n_exact += __popc(mk);
            const float tau = *reinterpret_cast<const volatile float*>(&q.tau);
            const bool app = mine && sc >= tau;
            const uint32_t am = __ballot_sync(0xFFFFFFFFu, app);
            if (am) {
              int base = 0;
              if (lane == 0) base = atomicAdd(&q.count, __popc(am));
              base = __shfl_sync(0xFFFFFFFFu, base, 0);
              const int slot = base + __popc(am & ((1u << lane) - 1u));
              const int phase = *reinterpret_cast<const volatile int*>(&q.phase);
              if (app) {
                if (slot < p.cap) {
                  Cand cd;
                  cd.score = sc;
                  cd.key = (int)s;
                  p.cand[q.row * (int64_t)p.cap + slot] = cd;
                  if (phase == 2) atomicAdd(&q.hist[bin_of(q, sc)], 1u);
                } else {
                  q.overflow = 1;
                }
              }
              n_cand += __popc(am);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          ++u;
        }
        if (!ok) break;
        // ---- checkpoint (every kCkptTiles tiles, and at the item's last tile) ----
        // All epilogue warps meet; each owner then refreshes its query's
        // threshold.  Between checkpoints the warps are coupled only through
        // the accumulator and mask barriers.
        const bool ckpt = ((ti + 1) % kCkptTiles) == 0 || ti + 1 == g.n_tiles;
        if (ckpt) {
          // The owner's own count, read before it arrives: every slot below it
          // was reserved in a tile <= ti and written before its writer arrived,
          // and none of those writers saw the screening phase, so the warm-up
          // scan below neither misses a written entry nor counts one twice.
          int snap_cnt = 0;
          if (lane == 0 && ew < g.nq) snap_cnt = *reinterpret_cast<volatile int*>(&st[ew].count);
          snap_cnt = __shfl_sync(0xFFFFFFFFu, snap_cnt, 0);
          if (lane == 0) {
            snap[(nbar & 1) * 16 + ew * 2 + 0] = it_scr;
            snap[(nbar & 1) * 16 + ew * 2 + 1] = it_rej;
          }
          __threadfence_block();
          if (lane == 0) mbar_arrive(tile_done);
          if (!mbar_wait(tile_done, nbar & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          const uint32_t slot = nbar & 1;
          ++nbar;
          // adaptive screening: every warp reads the same snapshot and takes
          // the same decision; screening ends at tile ti + 4 (the MMA thread
          // learns it from *stop_word before it would issue that tile's bound)
          if (!decided) {
            unsigned long long tot_s = 0, tot_r = 0;
            for (int w = 0; w < C::kEpiWarps; ++w) {
              tot_s += reinterpret_cast<volatile unsigned long long*>(snap)[slot * 16 + w * 2];
              tot_r += reinterpret_cast<volatile unsigned long long*>(snap)[slot * 16 + w * 2 + 1];
            }
            if (tot_s >= kAdaptiveMinScreened) {
              decided = true;
              if (tot_r * kAdaptiveRejectRatio < tot_s) {
                stop = ti + 4;
                if (ew == 0 && lane == 0) *reinterpret_cast<volatile int*>(stop_word) = stop;
              }
            }
          }
          // the owner refreshes its query's threshold
          if (ti + 1 < g.n_tiles && ew < g.nq) {
            QState& q = st[ew];
            const int phase = q.phase;
            const int cnt = snap_cnt;
            if (phase == 1 && cnt >= p.K && cnt <= p.cap) {
              // warm-up complete: bin the candidates so far over [min, max]
              const Cand* cl = p.cand + q.row * (int64_t)p.cap;
              float mn = INFINITY, mx = -INFINITY;
              for (int i = lane; i < cnt; i += 32) {
                const float x = cl[i].score;
                mn = fminf(mn, x);
                mx = fmaxf(mx, x);
              }
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
              }
              float w = (mx - mn) / (float)kBins;
              if (!(w > 0.f) || !isfinite(w)) w = fmaxf(fabsf(mn), 1e-30f) * 0x1p-8f;
              if (lane == 0) {
                q.lo = mn;
                q.w = w;
                q.inv_w = 1.f / w;
              }
              __syncwarp();
              for (int i = lane; i < cnt; i += 32) atomicAdd(&q.hist[bin_of(q, cl[i].score)], 1u);
              __syncwarp();
              const float tn = hist_threshold(q, p.K, lane);
              if (lane == 0) {
                q.tau = fmaxf(q.tau, tn);
                __threadfence_block();
                *reinterpret_cast<volatile int*>(&q.phase) = 2;
              }
            } else if (phase == 2) {
              const float tn = hist_threshold(q, p.K, lane);
              if (lane == 0 && tn > q.tau) *reinterpret_cast<volatile float*>(&q.tau) = tn;
            }
            __syncwarp();
          }
        }
        scr_cur = scr_next;
      }
      nb += n_scr;
      // ---- item end: the owner publishes its query ----
      if (ok && ew < g.nq && lane == 0) {
        QState& q = st[ew];
        const int cnt = *reinterpret_cast<volatile int*>(&q.count);
        const bool over = q.overflow || cnt > p.cap;
        p.cand_count[q.row] = over ? -1 : cnt;
        p.tau_out[q.row] = q.tau;
        if (over) {
          const int r = atomicAdd(p.repair_count, 1);
          if (r < p.repair_cap) p.repair_list[r] = (int)q.row;
          else record_error(p.err, kDevBounds);
        }
      }
    }
    if (lane == 0) {
      atomicAdd(&p.counters[kCntSeedPairs], n_seed);
      atomicAdd(&p.counters[kCntScreened], n_screened);
      atomicAdd(&p.counters[kCntRejected], n_rejected);
      atomicAdd(&p.counters[kCntExact], n_exact);
      atomicAdd(&p.counters[kCntCandidates], n_cand);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---- host side ---------------------------------------------------------------------

static bool encode_map(CUtensorMap* map, const void* base, bool fp8, uint64_t rows,
                       uint32_t box_rows) {
  auto enc = get_tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {(cuuint32_t)(fp8 ? 128 : 64), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kFp8>
static cudaError_t launch_cert_impl(const Handle& h, const SeqView& v, const CertBuffers& b,
                                    int K, cudaStream_t stream) {
  using C = CertCfg<kFp8>;
  CUtensorMap qmap, bmap, kmap;
  if (!encode_map(&qmap, v.q, kFp8, (uint64_t)(v.row0 + v.rows) * C::kH, 256) ||
      !encode_map(&bmap, b.bdir, kFp8, (uint64_t)v.rows * kBoundRows, C::kBRows) ||
      !encode_map(&kmap, v.k, kFp8, (uint64_t)v.S, kKeyTile))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(certified_kernel<kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  CertParams p;
  p.w = v.w;
  p.q_scale = v.q_scale;
  p.k_scale = v.k_scale;
  p.key_norm = b.key_norm;
  p.cert = b.cert;
  p.cand = reinterpret_cast<Cand*>(b.cand);
  p.cand_count = b.cand_count;
  p.tau_out = b.tau;
  p.repair_list = b.repair_list;
  p.repair_count = b.repair_count;
  p.repair_cap = b.repair_cap;
  p.counters = b.counters;
  p.err = b.err;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.n_items = (int)((v.rows + 7) / 8);
  p.K = K;
  p.cap = b.cap;
  p.seed_first = h.cfg.seed_first;
  p.seed_last = h.cfg.seed_last;
  p.screening = h.cfg.screening;
  if (p.n_items == 0) return cudaSuccess;
  const int grid = p.n_items < sms ? p.n_items : sms;
  profile_before(DOSA_KERNEL_CERTIFIED, stream);
  certified_kernel<kFp8><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, bmap, kmap, p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_CERTIFIED, stream);
  return e;
}

cudaError_t launch_certified(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                             cudaStream_t stream) {
  if (h.cfg.dtype == DOSA_FP8_E4M3) return launch_cert_impl<true>(h, v, b, K, stream);
  return launch_cert_impl<false>(h, v, b, K, stream);
}

size_t certified_smem_bytes(bool fp8) {
  return fp8 ? CertCfg<true>::kSmemBytes : CertCfg<false>::kSmemBytes;
}

}  // namespace dosa
