// Ranked screening of the certified indexer for sm_100a: the bound kernel of
// the ranked threshold schedule ("DOSA: Dots Sparse Attention", Daily Paper
// Cast transcript, Method section: screening dot products and bound
// evaluation on the tensor cores, pruning, survivor masks; the pages do not
// fix the order in which the keys are screened).
//
// Every non-warm-up key of a row is screened against a band of the bound:
// pass 1 keeps the keys whose v = (UB + margin) * q_scale * k_scale is at least
// an estimate U_1 of a score a little below the row's K-th (rank_prep, from
// the exact warm-up scores); a later pass j keeps the keys with
// lo_j <= v < hi_j, the band the rescoring pass chose after it checked the
// previous estimate against the K-th it reached (rescore.cu).
//
// A unit is 32 query rows (four 8-row work items) x up to 64 key tiles, so
// the bound rows of 32 queries (N = 32 x 8 = 256) share every key tile the TMA
// brings in.  Per key tile: one M = 128 x N = 256 MMA into one of two TMEM
// accumulators, then 16 epilogue warps (4 per TMEM lane quadrant, 8 rows each)
// evaluate the bound, ballot the survivors and store one 32-bit survivor word
// per (row, 32 keys).  Words are written by exactly one warp, so no atomics
// sit on the data path; per-row maxima of the rejected bounds (which decide
// whether another pass is needed) are merged once per unit.
#include "cand_state.cuh"
#include "cert_layout.h"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "work_items.cuh"

namespace dosa {

struct RankParams {
  const float* key_norm;   // [S] code-domain ||k|| (rounded up)
  const float* k_scale;    // [S] (fp8)
  const float* cert;       // [chunk rows][kCertFloats]
  const float* q_scale;    // absolute rows (fp8)
  float* band_lo;          // [chunk rows] kept band lo <= v < hi
  float* band_hi;
  uint32_t* maxrej;        // [chunk rows] ordered largest rejected bound
  int* row_next;           // [chunk rows] pass a row waits for
  int* pass_any;           // this pass has rows (the launch is a no-op otherwise)
  const int* item_sel;     // [n_items] or null
  int want;
  uint32_t* bits;          // [chunk rows][words]
  int64_t words;
  unsigned long long* item_cnt;   // [n_items][2] probe counts, or null
  unsigned long long* counters;
  int* err;
  int64_t row0, rows, pos0, S;
  int n_items, W, K, seed_first, seed_last;
  int pass, lo_off, hi_off;
  int n_groups, parts, span;
};

template <bool kFp8>
struct RankCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kKeyStages = kFp8 ? 6 : 3;
  static constexpr int kRows = kRankRows;              // 32 query rows per unit
  static constexpr int kBRows = kRows * kBoundRows;    // 256: the MMA N
  static constexpr uint32_t kKeySubBytes = kKeyTile * 128;
  static constexpr uint32_t kKeyStageBytes = kKeySubBytes * kSub;
  static constexpr uint32_t kBSubBytes = kBRows * 128;
  static constexpr uint32_t kBBytes = kBSubBytes * kSub;
  static constexpr int kEpiWarps = 16;                 // 4 per lane quadrant, 8 rows each
  static constexpr int kThreads = 64 + kEpiWarps * 32;
  static constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
  static constexpr uint32_t kSmemBytes =
      1024 + kBBytes + kKeyStages * kKeyStageBytes + kEpiWarps * 8 * 80 + 256;
};

// One row of a unit, as an epilogue warp reads it (five 16-byte vectors).
struct RankRow {
  float4 om;          // folded retained-head weights x q_scale
  float4 sc;          // negative-aggregate row scales x q_scale
  float4 blh;         // (beta + margin) x q_scale (coefficient of ||k||), band lo, hi
  int jlo;            // screened key tiles [jlo, jhi)
  int jhi;
  int jplain;         // tiles below it hold no seed key and only visible keys
  int pad;
  long long pos;      // position of the row among the keys
  long long pad2;
};
static_assert(sizeof(RankRow) == 80, "RankRow is five 16-byte vectors");

// Units: groups of 32 chunk rows (longest first) x `parts` key-tile ranges.
struct RankUnit {
  int group;          // chunk-local rows [32 group, 32 group + 32)
  int j0, j1;         // key tiles of this unit
  bool active;
};

__device__ __forceinline__ int rank_item_of_row(const RankParams& p, int64_t r) {
  return p.n_items - 1 - (int)(r / kItemQueries);
}

// Screened key tiles of the work item holding chunk row r: [jlo, jhi).
__device__ __forceinline__ void rank_tiles_of_row(const RankParams& p, int64_t r, int& jlo,
                                                  int& jhi) {
  const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, rank_item_of_row(p, r));
  const int L = g.n_tiles - p.W + 1;   // tiles 0 and L.. were scored in the warm-up
  jhi = L - p.lo_off;
  jlo = p.hi_off > 0 ? L - p.hi_off : 1;
  if (jlo < 1) jlo = 1;
  if (jhi < jlo) jhi = jlo;
}

__device__ __forceinline__ bool rank_row_selected(const RankParams& p, int64_t r) {
  if (r >= p.rows) return false;
  if (p.item_sel && p.item_sel[rank_item_of_row(p, r)] != p.want) return false;
  if (p.row_next && p.row_next[r] != p.pass) return false;
  return true;
}

// Every role computes the same unit description (read-only inputs).
__device__ __forceinline__ RankUnit rank_unit(const RankParams& p, int u) {
  RankUnit U;
  U.group = p.n_groups - 1 - u / p.parts;
  const int part = u % p.parts;
  const int64_t r0 = (int64_t)U.group * kRankRows;
  int64_t r1 = r0 + kRankRows;
  if (r1 > p.rows) r1 = p.rows;
  int lo_first, hi_first, lo_last, hi_last;
  rank_tiles_of_row(p, r0, lo_first, hi_first);
  rank_tiles_of_row(p, r1 - 1, lo_last, hi_last);
  const int jmin = lo_first < lo_last ? lo_first : lo_last;
  const int jmax = hi_first > hi_last ? hi_first : hi_last;
  U.j0 = 1 + part * p.span;
  U.j1 = U.j0 + p.span;
  if (U.j0 < jmin) U.j0 = jmin;
  if (U.j1 > jmax) U.j1 = jmax;
  U.active = U.j1 > U.j0;
  if (U.active && (p.item_sel || p.row_next)) {
    bool any = false;
    for (int64_t r = r0; r < r1 && !any; ++r) any = rank_row_selected(p, r);
    U.active = any;
  }
  return U;
}

// kFirst: pass 1 (keep v >= lo; count screened and kept pairs), or a later
// pass (keep lo <= v < hi; count the band's pairs).
template <bool kFp8, bool kFirst>
__global__ void __launch_bounds__(RankCfg<kFp8>::kThreads, 1)
    rank_screen_kernel(const __grid_constant__ CUtensorMap bmap,
                       const __grid_constant__ CUtensorMap kmap, const RankParams p) {
  using C = RankCfg<kFp8>;
  if (p.pass_any && *p.pass_any == 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;
  uint8_t* sK = sB + C::kBBytes;
  RankRow* prm_all = reinterpret_cast<RankRow*>(sK + C::kKeyStages * C::kKeyStageBytes);
  static_assert((RankCfg<kFp8>::kKeyStages * RankCfg<kFp8>::kKeyStageBytes) % 16 == 0, "");
  uint64_t* bars = reinterpret_cast<uint64_t*>(prm_all + C::kEpiWarps * 8);
  uint64_t* b_full = bars + 0;
  uint64_t* b_empty = bars + 1;
  uint64_t* acc_full = bars + 2;                   // [2]
  uint64_t* acc_empty = bars + 4;                  // [2]
  uint64_t* done_bar = bars + 6;
  uint64_t* k_full = bars + 7;                     // [kKeyStages]
  uint64_t* k_empty = k_full + C::kKeyStages;      // [kKeyStages]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(k_empty + C::kKeyStages);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = p.n_groups * p.parts;

  if (threadIdx.x == 0) {
    mbar_init(b_full, 1);
    mbar_init(b_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(done_bar, 1);
    for (int i = 0; i < C::kKeyStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    *s_abort = 0;
    fence_barrier_init();
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
      uint32_t kc = 0, uc = 0;
      bool ok = true;
      bool b_inflight = false;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const RankUnit U = rank_unit(p, u);
        if (!U.active) continue;
        if (!mbar_wait(b_empty, (uc & 1) ^ 1, s_abort, p.err)) break;
        mbar_arrive_expect_tx(b_full, C::kBBytes);
        for (int sub = 0; sub < C::kSub; ++sub)
          tma_load_2d(sB + sub * C::kBSubBytes, &bmap, b_full, sub * 64,
                      U.group * C::kBRows);
        b_inflight = true;
        ++uc;
        for (int j = U.j0; j < U.j1; ++j, ++kc) {
          const int s_ = kc % C::kKeyStages;
          if (!mbar_wait(&k_empty[s_], ((kc / C::kKeyStages) & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s_], C::kKeyStageBytes);
          for (int sub = 0; sub < C::kSub; ++sub)
            tma_load_2d(sK + s_ * C::kKeyStageBytes + sub * C::kKeySubBytes, &kmap,
                        &k_full[s_], sub * 64, j * kKeyTile);
        }
      }
      if (*s_abort) {
        if (b_inflight) mbar_wait_drain(b_full, (uc - 1) & 1);
        for (uint32_t c = (kc > (uint32_t)C::kKeyStages ? kc - C::kKeyStages : 0); c < kc; ++c)
          mbar_wait_drain(&k_full[c % C::kKeyStages], (c / C::kKeyStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = make_idesc<kFp8>(kKeyTile, C::kBRows);
      uint32_t kc = 0, uc = 0, tc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const RankUnit U = rank_unit(p, u);
        if (!U.active) continue;
        if (!mbar_wait(b_full, uc & 1, s_abort, p.err)) break;
        ++uc;
        tc_fence_after();
        const uint32_t b_base = smem_u32(sB);
        for (int j = U.j0; j < U.j1; ++j, ++kc, ++tc) {
          const uint32_t s_ = kc % C::kKeyStages, buf = tc & 1;
          if (!mbar_wait(&k_full[s_], (kc / C::kKeyStages) & 1, s_abort, p.err) ||
              !mbar_wait(&acc_empty[buf], ((tc >> 1) & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + s_ * C::kKeyStageBytes);
          const uint32_t d = tmem_base + buf * C::kBRows;
#pragma unroll
          for (int step = 0; step < C::kKSteps; ++step) {
            const uint32_t sub = step >> 2, off = (step & 3) * 32;
            tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                         smem_desc_sw128(b_base + sub * C::kBSubBytes + off), idesc,
                         step > 0 ? 1u : 0u);
          }
          tc_commit(&acc_full[buf]);
          tc_commit(&k_empty[s_]);
        }
        tc_commit(b_empty);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue: bound evaluation ----------------
    const int ew = warp - 2;
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int qset = ew >> 2;                  // rows qset * 8 .. + 8 of the unit
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    RankRow* prm = prm_all + ew * 8;
    uint32_t tc = 0;
    unsigned long long n_seed = 0, n_scr = 0, n_rej = 0, n_band = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const RankUnit U = rank_unit(p, u);
      if (!U.active) continue;
      const int64_t row_base = (int64_t)U.group * kRankRows + qset * 8;
      // this warp's 8 rows (one work item): parameters into shared memory
      if (lane < 8) {
        const int64_t r = row_base + lane;
        RankRow R;
        const bool sel = rank_row_selected(p, r);
        int jlo = 0, jhi = 0;
        if (sel) rank_tiles_of_row(p, r, jlo, jhi);
        const float* cf = p.cert + (sel ? r : 0) * kCertFloats;
        const float sq = (kFp8 && sel) ? __ldg(p.q_scale + p.row0 + r) : 1.f;
        auto f = [&](int at) { return sel ? cf[at] * sq : 0.f; };
        R.om = make_float4(f(kCertOmega), f(kCertOmega + 1), f(kCertOmega + 2), f(kCertOmega + 3));
        R.sc = make_float4(f(kCertScale), f(kCertScale + 1), f(kCertScale + 2), f(kCertScale + 3));
        R.blh = make_float4(sel ? (cf[kCertBeta] + cf[kCertMargin]) * sq : 0.f,
                            sel ? p.band_lo[r] : INFINITY, sel ? p.band_hi[r] : INFINITY, 0.f);
        R.jlo = sel ? jlo : 0;
        R.jhi = sel ? jhi : 0;
        // seed-free, fully visible tiles: past the first seed keys and ending
        // before the last seed_last keys (which end at the row's position)
        const long long last_free = p.pos0 + r - p.seed_last;   // keys <= it are not seeds
        const int jp = last_free >= kKeyTile - 1 ? (int)((last_free + 1) / kKeyTile) : 0;
        R.jplain = p.seed_first <= jlo * kKeyTile ? jp : 0;
        R.pad = 0;
        R.pos = p.pos0 + r;
        R.pad2 = 0;
        prm[lane] = R;
      }
      __syncwarp();
      // rows of this warp that take part, and whether every one of them is
      // seed-free and fully visible over the whole unit (the fast loop)
      uint32_t live = 0;
      bool fast = true;
      if (lane < 8) {
        const RankRow& R = prm[lane];
        const bool in = R.jhi > R.jlo && U.j0 < R.jhi && U.j1 > R.jlo;
        const bool whole = R.jlo <= U.j0 && U.j1 <= R.jhi && U.j1 <= R.jplain;
        live = in ? 1u : 0u;
        fast = !in || whole;
      }
      live = __ballot_sync(0xFFFFFFFFu, live != 0) & 0xFFu;
      fast = __all_sync(0xFFFFFFFFu, fast);
      const int item = rank_item_of_row(p, row_base);
      // this unit's counts (32 bits suffice: at most 64 tiles x 32 keys x 8 rows)
      uint32_t u_seed = 0, u_scr = 0, u_kept = 0, u_band = 0;
      float mr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mr[i] = -INFINITY;
      for (int j = U.j0; j < U.j1 && ok; ++j, ++tc) {
        const uint32_t buf = tc & 1;
        const int64_t s = (int64_t)j * kKeyTile + quad * 32 + lane;
        const bool key_ok = s < p.S;
        const float nk = key_ok ? __ldg(p.key_norm + s) : 0.f;
        float sk = 1.f;
        if constexpr (kFp8) sk = key_ok ? __ldg(p.k_scale + s) : 0.f;
        if (!mbar_wait(&acc_full[buf], (tc >> 1) & 1, s_abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the warp's 64 columns in two halves of 4 rows; the accumulator is
        // released once both halves are in registers
        const uint32_t col = tmem_base + lane_off + buf * C::kBRows + qset * 64;
        uint32_t word = 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float x32[32];
          tmem_ld32_async(col + half * 32, x32);
          tmem_wait_ld(x32);
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
          }
          if (fast && ((live >> (half * 4)) & 0xFu) == 0xFu) {
            // four seed-free, fully visible rows: four independent chains
            float v[4], lo[4], hi[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float4* R4 = reinterpret_cast<const float4*>(prm + half * 4 + qq);
              const float4 om = R4[0], sc = R4[1], blh = R4[2];
              const float* x = x32 + qq * 8;
              float ub = om.x * fmaxf(x[0], 0.f);
              ub = fmaf(om.y, fmaxf(x[1], 0.f), ub);
              ub = fmaf(om.z, fmaxf(x[2], 0.f), ub);
              ub = fmaf(om.w, fmaxf(x[3], 0.f), ub);
              ub = fmaf(blh.x, nk, ub);
              ub -= fmaxf(fmaf(sc.x, x[4], sc.y * x[5]), 0.f);
              ub -= fmaxf(fmaf(sc.z, x[6], sc.w * x[7]), 0.f);
              v[qq] = ub * sk;
              lo[qq] = blh.y;
              hi[qq] = blh.z;
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const int i = half * 4 + qq;
              const bool rej = v[qq] < lo[qq];
              mr[i] = fmaxf(mr[i], rej ? v[qq] : -INFINITY);
              const uint32_t mask =
                  __ballot_sync(0xFFFFFFFFu, kFirst ? !rej : (!rej && v[qq] < hi[qq]));
              if constexpr (kFirst) {
                u_scr += 32;
                u_kept += __popc(mask);
              } else {
                u_band += __popc(mask);
              }
              if (lane == i) word = mask;
            }
            continue;
          }
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int i = half * 4 + qq;
            if (!(live >> i & 1)) continue;                   // uniform over the warp
            const float4* R4 = reinterpret_cast<const float4*>(prm + i);
            const float4 om = R4[0], sc = R4[1], blh = R4[2];
            const float* x = x32 + qq * 8;
            float ub = om.x * fmaxf(x[0], 0.f);
            ub = fmaf(om.y, fmaxf(x[1], 0.f), ub);
            ub = fmaf(om.z, fmaxf(x[2], 0.f), ub);
            ub = fmaf(om.w, fmaxf(x[3], 0.f), ub);
            ub = fmaf(blh.x, nk, ub);
            ub -= fmaxf(fmaf(sc.x, x[4], sc.y * x[5]), 0.f);
            ub -= fmaxf(fmaf(sc.z, x[6], sc.w * x[7]), 0.f);
            const float v = ub * sk;
            uint32_t mask;
            if (fast || (j >= prm[i].jlo && j < prm[i].jhi && j < prm[i].jplain)) {
              // no seed, every key visible
              const bool rej = v < blh.y;
              mr[i] = fmaxf(mr[i], rej ? v : -INFINITY);
              mask = __ballot_sync(0xFFFFFFFFu, kFirst ? !rej : (!rej && v < blh.z));
              if constexpr (kFirst) {
                u_scr += 32;
                u_kept += __popc(mask);
              } else {
                u_band += __popc(mask);
              }
            } else {
              if (j < prm[i].jlo || j >= prm[i].jhi) continue;   // uniform over the warp
              const long long pos = prm[i].pos;
              const bool vis = key_ok && s <= pos;
              const bool seed = s < p.seed_first || s > pos - p.seed_last;
              bool surv;
              if constexpr (kFirst) surv = vis && (seed || v >= blh.y);
              else surv = vis && !seed && v >= blh.y && v < blh.z;
              const bool rej = vis && !seed && v < blh.y;
              mr[i] = fmaxf(mr[i], rej ? v : -INFINITY);
              mask = __ballot_sync(0xFFFFFFFFu, surv);
              if constexpr (kFirst) {
                const uint32_t sm = __ballot_sync(0xFFFFFFFFu, vis && seed);
                const uint32_t vm = __ballot_sync(0xFFFFFFFFu, vis);
                u_seed += __popc(sm);
                u_scr += __popc(vm & ~sm);
                u_kept += __popc(mask & ~sm);
              } else {
                u_band += __popc(mask);
              }
            }
            if (lane == i) word = mask;
          }
        }
        if (lane < 8 && j >= prm[lane].jlo && j < prm[lane].jhi)
          p.bits[(row_base + lane) * p.words + (int64_t)j * 4 + quad] = word;
      }
      // per-row largest rejected bound of this unit, and the item's counts
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float m = mr[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0 && m > -INFINITY && prm[i].jhi > prm[i].jlo)
          atomicMax(p.maxrej + row_base + i, ordered_key(m));
      }
      if (lane == 0 && p.item_cnt && u_scr) {
        atomicAdd(&p.item_cnt[item * 2 + 0], (unsigned long long)u_scr);
        atomicAdd(&p.item_cnt[item * 2 + 1], (unsigned long long)u_kept);
      }
      n_seed += u_seed;
      n_scr += u_scr;
      n_rej += u_scr - u_kept;
      n_band += u_band;
      __syncwarp();
    }
    if (lane == 0 && !p.item_cnt) {     // a probe's counts go through rank_decide
      if (kFirst) {
        atomicAdd(&p.counters[kCntSeedPairs], n_seed);
        atomicAdd(&p.counters[kCntScreened], n_scr);
        atomicAdd(&p.counters[kCntRejected], n_rej);
      } else {
        atomicAdd(&p.counters[kCntBandPairs], n_band);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---- per-row estimates of the threshold ---------------------------------------

// One warp per chunk row of the selected items: the descending estimates U_j
// (the m_j-th largest warm-up score, m_1 = ceil(1.5 K n_e / n), m_{j+1} = 8 m_j,
// the last with m = K) from the row's warm-up histogram, the pass-1 band
// [U_1, inf), and the row's pass bookkeeping.  A histogram lower edge is at or
// below the score it stands for, so every estimate is at or below the exact
// m-th largest warm-up score; the last one equals the warm-up threshold.
__global__ void rank_prep_kernel(const RankParams p, const QStateG* qstate, float* est) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= p.rows) return;
  if (p.item_sel && p.item_sel[rank_item_of_row(p, r)] != p.want) return;
  const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, rank_item_of_row(p, r));
  const int64_t pos = p.pos0 + r, n = pos + 1;
  // exact warm-up keys: tile 0 and the tiles from L on (the item's last W - 1);
  // a row with no tile in between was finished (and published) by the warm-up
  const int64_t L = g.n_tiles - p.W + 1;
  if (L <= 1) return;
  const int64_t first = (L > 1 ? L : 1) * kKeyTile;
  const int64_t n_e = (n < kKeyTile ? n : kKeyTile) + (n > first ? n - first : 0);
  const QStateG& q = qstate[r];
  const bool have = q.phase == 2;
  int64_t m = (3 * (int64_t)p.K * n_e + 2 * n - 1) / (2 * n);   // ceil(1.5 K n_e / n)
  if (m < 1) m = 1;
  if (m > p.K) m = p.K;
  float prev = INFINITY;
  for (int e = 0; e < kRankEst; ++e) {
    float u = -INFINITY;
    if (have) {
      const int b = suffix_bin(q.hist, (int)m, lane);
      if (b >= 0) u = bin_edge_at(q.lo, q.w, b);
    }
    u = fminf(u, prev);
    prev = u;
    if (lane == 0) est[r * kRankEst + e] = u;
    m = m * 8 > p.K ? p.K : m * 8;
  }
  if (lane == 0) {
    p.band_lo[r] = est[r * kRankEst + 0];
    p.band_hi[r] = INFINITY;
    p.maxrej[r] = 0u;
    p.row_next[r] = 1;
    *p.pass_any = 1;
  }
}

// One thread per work item: after a probe pass, an item whose probe kept at
// most 1 in kRankKeepRatio of its screened pairs goes on with ranked
// screening (kItemRank, and the gate is raised); any other item is finished
// by the filter scorer (kItemFilter).  The probe's pair counts enter the
// call's counters here, for the ranked items only.
__global__ void rank_decide_kernel(int* item_flag, const unsigned long long* item_cnt,
                                   int n_items, int want, int* gate,
                                   unsigned long long* counters) {
  const int it = blockIdx.x * blockDim.x + threadIdx.x;
  if (it >= n_items || item_flag[it] != want) return;
  const unsigned long long scr = item_cnt[it * 2], surv = item_cnt[it * 2 + 1];
  const bool rank = scr >= kRankMinScreened && surv * kRankKeepRatio <= scr;
  item_flag[it] = rank ? kItemRank : kItemFilter;
  if (rank) {
    *reinterpret_cast<volatile int*>(gate) = 1;
    // the probe's pairs count for the items that keep its result (the filter
    // scorer scores the others' pairs again)
    atomicAdd(&counters[kCntScreened], scr);
    atomicAdd(&counters[kCntRejected], scr - surv);
  }
}

// ---- host side --------------------------------------------------------------------

static RankParams rank_params(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                              int W, const RankPass& rp) {
  RankParams p;
  p.key_norm = b.key_norm;
  p.k_scale = v.k_scale;
  p.cert = b.cert;
  p.q_scale = v.q_scale;
  p.band_lo = b.band_lo;
  p.band_hi = b.band_hi;
  p.maxrej = b.maxrej;
  p.row_next = b.row_next;
  p.pass_any = b.pass_any + rp.pass;
  p.item_sel = rp.item_sel;
  p.want = rp.want;
  p.bits = b.bits;
  p.words = b.words;
  p.item_cnt = rp.item_cnt;
  p.counters = b.counters;
  p.err = b.err;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.n_items = (int)((v.rows + kItemQueries - 1) / kItemQueries);
  p.W = W;
  p.K = K;
  p.seed_first = h.cfg.seed_first;
  p.seed_last = h.cfg.seed_last;
  p.pass = rp.pass;
  p.lo_off = rp.lo_off;
  p.hi_off = rp.hi_off;
  p.n_groups = (int)((v.rows + kRankRows - 1) / kRankRows);
  p.parts = 0;
  p.span = 0;
  return p;
}

template <bool kFp8>
static cudaError_t launch_rank_impl(const SeqView& v, const RankParams& p, const void* bdir,
                                    cudaStream_t stream) {
  using C = RankCfg<kFp8>;
  CUtensorMap bmap, kmap;
  if (!encode_rows_map(&bmap, bdir, kFp8, (uint64_t)v.rows * kBoundRows, C::kBRows) ||
      !encode_rows_map(&kmap, v.k, kFp8, (uint64_t)v.S, kKeyTile))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(rank_screen_kernel<kFp8, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(rank_screen_kernel<kFp8, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int units = p.n_groups * p.parts;
  const int grid = units < sms ? units : sms;
  profile_before(DOSA_KERNEL_RANK, stream);
  if (p.pass == 1)
    rank_screen_kernel<kFp8, true><<<grid, C::kThreads, C::kSmemBytes, stream>>>(bmap, kmap, p);
  else
    rank_screen_kernel<kFp8, false><<<grid, C::kThreads, C::kSmemBytes, stream>>>(bmap, kmap, p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_RANK, stream);
  return e;
}

cudaError_t launch_rank_screen(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                               int W, const RankPass& rp, cudaStream_t stream) {
  RankParams p = rank_params(h, v, b, K, W, rp);
  // units: 32-row groups x key-tile parts of about kRankUnitTiles tiles (one
  // part for the probe, whose tiles per item are few)
  const int64_t n_tiles_max = (v.pos0 + v.rows - 1) / kKeyTile + 1;
  const int64_t L = n_tiles_max - W + 1 - rp.lo_off;   // tiles [1, L) at most
  if (L <= 1 || p.n_groups == 0) return cudaSuccess;
  const int64_t span_all = L - 1;
  p.parts = rp.hi_off > 0 ? 1 : (int)((span_all + kRankUnitTiles - 1) / kRankUnitTiles);
  p.span = (int)((span_all + p.parts - 1) / p.parts);
  if (h.cfg.dtype == DOSA_FP8_E4M3) return launch_rank_impl<true>(v, p, b.bdir, stream);
  return launch_rank_impl<false>(v, p, b.bdir, stream);
}

cudaError_t launch_rank_prep(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                             int W, const int* item_sel, int want, cudaStream_t stream) {
  if (v.rows <= 0) return cudaSuccess;
  RankPass rp{1, 0, 0, item_sel, want, nullptr};
  const RankParams p = rank_params(h, v, b, K, W, rp);
  constexpr int kWarps = 8;
  const int grid = (int)((v.rows + kWarps - 1) / kWarps);
  profile_before(DOSA_KERNEL_RANK, stream);
  rank_prep_kernel<<<grid, kWarps * 32, 0, stream>>>(
      p, reinterpret_cast<const QStateG*>(b.qstate), b.est);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_RANK, stream);
  return e;
}

cudaError_t launch_rank_decide(int* item_flag, const unsigned long long* item_cnt, int n_items,
                               int want, int* gate, unsigned long long* counters,
                               cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  rank_decide_kernel<<<(n_items + 255) / 256, 256, 0, stream>>>(item_flag, item_cnt, n_items,
                                                                want, gate, counters);
  return cudaGetLastError();
}

}  // namespace dosa
