// Certified indexer scorer for sm_100a: screening, rescoring and sparse
// writeback fused in one persistent tcgen05 kernel ("DOSA: Dots Sparse
// Attention", Daily Paper Cast transcript, Method section: every tile of
// visible keys goes through the screening products, the bound, the pruning
// and the compaction of what survives; GPU kernel design: query tiles of a
// fixed width on the tensor cores, the survivors of a key tile packed so the
// tile is loaded once, exact scoring fused with the threshold test and the
// packed writeback).
//
// Work item = 8 consecutive query rows (work_items.cuh).  Resident in shared
// memory: their 8 x 64 head rows and their 8 x 8 bound rows (4 retained heads,
// u_1 hi/lo, u_2 hi/lo, from cert_setup).  For each key tile of 128 keys of
// the item's range, in processing order:
//   1. bound MMA   D_b[128 keys x 64] = keys x bound rows            (N = 64)
//   2. bound epilogue: UB(t,s) per (key, query); a key survives when it is a
//      seed, when the query is still warming up (fewer than K exact scores),
//      or when (UB + margin) * scales >= tau_t.  Masks go to shared memory.
//   3. exact MMA for each pair of queries with at least one survivor
//      D_e[128 keys x 128] = keys x (2 queries x 64 heads)           (N = 128)
//   4. exact epilogue on survivors only: the head reduction shared with the
//      dense scorer (bit-identical scores); scores >= tau_t are appended as
//      packed (score, key) pairs (cand_state.cuh keeps tau_t sound).
// The epilogue screens one tile ahead of the exact MMAs (bound(t+1) before
// exact(t)), so screening overlaps the tensor core.  Every 4 tiles, and at the
// end of a range, the epilogue warps meet and each query's owner warp
// refreshes its threshold.
//
// A launch processes a range of steps of every item (work_items.cuh).  This
// kernel runs the pages' own schedule (screening = 1: every tile after the
// warm-up is screened, the threshold rising as tiles are scored); the ranked
// schedule of the other screening modes is rank_screen.cu + rescore.cu.
#include "cand_state.cuh"
#include "cert_layout.h"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "score_epilogue.cuh"
#include "work_items.cuh"

namespace dosa {

template <bool kFp8>
struct CertCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kKeyStages = kFp8 ? 4 : 2;
  static constexpr int kH = 64;
  static constexpr int kQT = kItemQueries;
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

struct CertParams {
  const float* w;          // [rows_total, H] absolute rows
  const float* q_scale;    // absolute rows (fp8)
  const float* k_scale;    // sequence base (fp8)
  const float* key_norm;   // [S] code-domain ||k||, rounded up
  const float* cert;       // [chunk rows, kCertFloats]
  Cand* cand;              // [chunk rows][kSegs][seg_cap]
  QStateG* qstate;         // [chunk rows] state carried between passes
  int* item_flag;          // [n_items] decision of the probe pass
  PublishOut out;
  unsigned long long* counters;
  int* err;
  int64_t row0, rows, pos0, S;   // chunk: absolute first row, rows, first position
  int n_items, K, seg_cap, seed_first, seed_last;
  int H;                   // heads per query row: 32 or 64 (the MMA always sees 64)
  float* dense;            // dense writeback (ablation): [chunk rows, dense_ld], or null
  int64_t dense_ld;
  const int* step_list;    // per item, the steps left by block screening, or null
  const int* step_count;
  int step_cap;
  StepRange steps;         // what this launch processes
};

// The steps an item processes in this launch: its range, or the list block
// screening left of it (never empty when the range is not).
__device__ __forceinline__ int steps_of(const CertParams& p, const Range& rg, int item) {
  return p.step_list ? p.step_count[item] : rg.end - rg.begin;
}
__device__ __forceinline__ int step_at(const CertParams& p, const Range& rg, int item, int i) {
  return p.step_list ? p.step_list[(int64_t)item * p.step_cap + i] : rg.begin + i;
}


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

// kHeads: heads per query row (32 or 64); the MMA always sees 64 head slots.
template <bool kFp8, int kHeads>
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
  // Survivor masks and query-pair flags of a tile, three slots: a slot is
  // rewritten (bound evaluation of tile b+3) only after every warp has passed
  // the bound evaluation of tile b+2, which follows its exact stage of b.
  uint32_t* masks = reinterpret_cast<uint32_t*>(k_empty + C::kKeyStages);  // [3][8][4]
  uint32_t* gflag = masks + 3 * 8 * 4;                                      // [3][8]
  uint32_t* s_tmem = gflag + 3 * 8;
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bnd_full[i], 1);
      mbar_init(&bnd_empty[i], C::kEpiWarps);
      mbar_init(&mask_ready[i], C::kEpiWarps);
    }
    for (int i = 0; i < C::kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(tile_done, C::kEpiWarps);
    mbar_init(item_ready, C::kEpiWarps);
    mbar_init(done_bar, 1);
    for (int i = 0; i < C::kKeyStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    *s_abort = 0;
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
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
        const Range rg = item_steps(p.steps, p.item_flag, g, item);
        if (rg.end <= rg.begin) continue;
        if (!mbar_wait(q_empty, (it & 1) ^ 1, s_abort, p.err)) break;
        mbar_arrive_expect_tx(q_full, C::kQBytes + C::kBBytes);
        for (int sub = 0; sub < C::kSub; ++sub) {
          for (int b = 0; b < C::kQRows / 256; ++b)
            tma_load_3d(sQ + sub * C::kQSubBytes + b * 256 * 128, &qmap, q_full, sub * 64, 0,
                        (int32_t)(g.t0 + b * 4));
          tma_load_2d(sB + sub * C::kBSubBytes, &bmap, q_full, sub * 64,
                      (int32_t)(g.local0 * kBoundRows));
        }
        inflight_q = it & 1;
        ++it;
        const int n_steps = steps_of(p, rg, item);
        for (int i = 0; i < n_steps; ++i, ++kc) {
          const int s_ = kc % C::kKeyStages;
          const uint32_t rnd = kc / C::kKeyStages;
          if (!mbar_wait(&k_empty[s_], (rnd & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s_], C::kKeyStageBytes);
          const int j = tile_at(step_at(p, rg, item, i), g.n_tiles);
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
      // Per item: bound(first); then for each step i: bound(i+1), [wait for
      // step i's survivor masks], exact MMAs of step i.
      constexpr uint32_t idesc_b = make_idesc<kFp8>(kKeyTile, C::kBRows);
      constexpr uint32_t idesc_e = make_idesc<kFp8>(kKeyTile, C::kGroupN);
      uint32_t kc = 0, u = 0;
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
        const Range rg = item_steps(p.steps, p.item_flag, g, item);
        if (rg.end <= rg.begin) continue;
        if (!mbar_wait(q_full, it & 1, s_abort, p.err)) break;
        ++it;
        tc_fence_after();
        const uint32_t b_bound = smem_u32(sB);
        const int n = steps_of(p, rg, item);
        // bound tiles use the same running index as key stages (kc)
        auto issue_bound = [&](int i) -> bool {
          const uint32_t c = kc + i, s_ = c % C::kKeyStages;
          if (!mbar_wait(&k_full[s_], (c / C::kKeyStages) & 1, s_abort, p.err) ||
              !mbar_wait(&bnd_empty[c & 1], ((c >> 1) & 1) ^ 1, s_abort, p.err))
            return false;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + s_ * C::kKeyStageBytes);
          const uint32_t d = tmem_base + C::kBndCol + (c & 1) * C::kBRows;
#pragma unroll
          for (int step = 0; step < C::kKSteps; ++step) {
            const uint32_t sub = step >> 2, off = (step & 3) * 32;
            tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                         smem_desc_sw128(b_bound + sub * C::kBSubBytes + off), idesc_b,
                         step > 0 ? 1u : 0u);
          }
          tc_commit(&bnd_full[c & 1]);
          return true;
        };
        if (!issue_bound(0)) break;
        for (int i = 0; i < n && ok; ++i) {
          if (i + 1 < n && !issue_bound(i + 1)) {
            ok = false;
            break;
          }
          const uint32_t c = kc + i, s_ = c % C::kKeyStages;
          if (!mbar_wait(&mask_ready[c & 1], (c >> 1) & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          uint32_t groups = 0;
          for (int w = 0; w < C::kEpiWarps; ++w)
            groups |= reinterpret_cast<volatile uint32_t*>(gflag)[(c % 3) * 8 + w];
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
        }
        kc += n;
        tc_commit(q_empty);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    // Per item: bound(first); then for each step i: bound(i+1), exact(i), and
    // at checkpoints the threshold refresh by each query's owner warp.
    const int ew = warp - 2;                 // owner of query slot ew
    const int quad = warp & 3;
    const int half = ew >> 2;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t kc = 0, u = 0, nbar = 0;
    int it = 0;
    unsigned long long n_seed = 0, n_screened = 0, n_rejected = 0, n_exact = 0, n_cand = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
      const Range rg = item_steps(p.steps, p.item_flag, g, item);
      if (rg.end <= rg.begin) continue;
      const int n = steps_of(p, rg, item);
      // owner: this item's state of query slot ew (fresh, or carried over)
      {
        QState& s = st[ew];
        const bool valid = ew < g.nq;
        const int64_t row = g.local0 + ew;
        if (lane == 0) {
          s.row = row;
          s.pos = valid ? g.pos_first + ew : -1;
          const float* cf = p.cert + (valid ? row : 0) * kCertFloats;
          for (int j = 0; j < 4; ++j) {
            s.omega[j] = valid ? cf[kCertOmega + j] : 0.f;
            s.scale[j] = valid ? cf[kCertScale + j] : 0.f;
          }
          s.beta = valid ? cf[kCertBeta] : 0.f;
          s.margin = valid ? cf[kCertMargin] : 0.f;
          s.sq = (kFp8 && valid) ? __ldg(p.q_scale + g.t0 + ew) : 1.f;
        }
        if (valid && rg.begin > 0) state_load(s, p.qstate + row, lane);
        else state_fresh(s, valid, lane);
        __syncwarp();
        __threadfence_block();
        if (lane == 0) mbar_arrive(item_ready);
        if (!mbar_wait(item_ready, it & 1, s_abort, p.err)) break;
        ++it;
      }
      // this warp's segment counts of its queries grp * 2 + half (grp = 0..3)
      int cnt[C::kGroups];
#pragma unroll
      for (int grp = 0; grp < C::kGroups; ++grp)
        cnt[grp] = *reinterpret_cast<volatile int*>(&st[grp * 2 + half].seg[quad]);
      auto key_of = [&](int i) -> int64_t {
        return (int64_t)tile_at(step_at(p, rg, item, i), g.n_tiles) * kKeyTile + quad * 32 + lane;
      };
      // ---- bound evaluation of step i ----
      auto bound_eval = [&](int i) -> bool {
        const uint32_t c = kc + i;
        const int64_t s = key_of(i);
        const bool key_ok = s < p.S;
        const float nk = key_ok ? __ldg(p.key_norm + s) : 0.f;
        float sk = 1.f;
        if constexpr (kFp8) sk = key_ok ? __ldg(p.k_scale + s) : 0.f;
        if (!mbar_wait(&bnd_full[c & 1], (c >> 1) & 1, s_abort, p.err)) return false;
        tc_fence_after();
        float v[32];
        tmem_ld32(tmem_base + lane_off + C::kBndCol + (c & 1) * C::kBRows + half * 32, v);
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
          n_seed += __popc(__ballot_sync(0xFFFFFFFFu, vis && seed));
          n_screened += __popc(__ballot_sync(0xFFFFFFFFu, screen));
          n_rejected += __popc(__ballot_sync(0xFFFFFFFFu, rej));
          if (lane == 0) masks[((c % 3) * 8 + ql) * 4 + quad] = mk;
          if (mk) gbits |= 1u << (ql >> 1);
        }
        if (lane == 0) gflag[(c % 3) * 8 + ew] = gbits;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bnd_empty[c & 1]);
          mbar_arrive(&mask_ready[c & 1]);
        }
        return mbar_wait(&mask_ready[c & 1], (c >> 1) & 1, s_abort, p.err);
      };
      if (!bound_eval(0)) break;
      for (int i = 0; i < n && ok; ++i) {
        if (i + 1 < n && !bound_eval(i + 1)) {
          ok = false;
          break;
        }
        // ---- exact scoring of step i's survivors, filter, packed writeback ----
        const int64_t s = key_of(i);
        const bool key_ok = s < p.S;
        float sk = 1.f;
        if constexpr (kFp8) sk = key_ok ? __ldg(p.k_scale + s) : 0.f;
        const uint32_t c = kc + i;
        uint32_t groups = 0;
        for (int w = 0; w < C::kEpiWarps; ++w)
          groups |= reinterpret_cast<volatile uint32_t*>(gflag)[(c % 3) * 8 + w];
#pragma unroll
        for (int grp = 0; grp < C::kGroups; ++grp) {
          if (!(groups >> grp & 1) || !ok) continue;
          const uint32_t ab = u % C::kAccBufs;
          if (!mbar_wait(&acc_full[ab], (u / C::kAccBufs) & 1, s_abort, p.err)) {
            ok = false;
            continue;
          }
          tc_fence_after();
          const int ql = grp * 2 + half;
          QState& q = st[ql];
          const uint32_t mk =
              reinterpret_cast<volatile uint32_t*>(masks)[((c % 3) * 8 + ql) * 4 + quad];
          if (mk) {
            float x[64];
            tmem_ld64(tmem_base + lane_off + C::kAccCol + ab * C::kGroupN + half * 64, x);
            const bool mine = (mk >> lane) & 1;
            float sc = 0.f;
            if (mine) {
              const int64_t t = g.t0 + ql;
              sc = kHeads == 64 ? head_reduce64_packed(x, p.w + t * 64)
                                : head_reduce32_packed(x, p.w + t * 32);
              if constexpr (kFp8) sc *= __ldg(p.q_scale + t) * sk;
              if (p.dense && s <= q.pos) p.dense[q.row * p.dense_ld + s] = sc;
            }
            n_exact += __popc(mk);
            const float tau = *reinterpret_cast<const volatile float*>(&q.tau);
            n_cand += append_candidates(
                q, p.cand + (q.row * kSegs + quad) * (int64_t)p.seg_cap, p.seg_cap, cnt[grp],
                mine && sc >= tau, sc, (int)s, lane);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          ++u;
        }
        if (!ok) break;
        // ---- checkpoint: every kCkptTiles steps and at the range's last ----
        const bool last = i + 1 == n;
        if (((i + 1) % kCkptTiles) == 0 || last) {
          // Publish this warp's segment counts: every entry below them is
          // written, so the owner's warm-up scan after the barrier neither
          // misses a written entry nor counts one twice.
          if (lane == 0) {
#pragma unroll
            for (int grp = 0; grp < C::kGroups; ++grp) st[grp * 2 + half].seg[quad] = cnt[grp];
          }
          __threadfence_block();
          if (lane == 0) mbar_arrive(tile_done);
          if (!mbar_wait(tile_done, nbar & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          ++nbar;
          if (ew < g.nq)
            refresh_threshold(st[ew], p.cand + st[ew].row * kSegs * (int64_t)p.seg_cap, p.seg_cap,
                              p.K, lane);
        }
      }
      kc += n;
      // ---- range end: carry the query's state over, or publish it ----
      if (ok && ew < g.nq) {
        if (rg.end < g.n_tiles) state_save(st[ew], p.qstate + st[ew].row, lane);
        else if (lane == 0) publish_query(st[ew], p.out);
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

template <bool kFp8>
static cudaError_t launch_cert_impl(const Handle& h, const SeqView& v, const CertBuffers& b,
                                    int K, StepRange steps, cudaStream_t stream, int use_list) {
  using C = CertCfg<kFp8>;
  CUtensorMap qmap, bmap, kmap;
  if (!encode_q_map(&qmap, v.q, kFp8, (uint64_t)(v.row0 + v.rows), v.H) ||
      !encode_rows_map(&bmap, b.bdir, kFp8, (uint64_t)v.rows * kBoundRows, C::kBRows) ||
      !encode_rows_map(&kmap, v.k, kFp8, (uint64_t)v.S, kKeyTile))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    for (auto fn : {certified_kernel<kFp8, 64>, certified_kernel<kFp8, 32>})
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  p.qstate = reinterpret_cast<QStateG*>(b.qstate);
  p.item_flag = b.item_flag;
  p.out.cand_count = b.cand_count;
  p.out.tau = b.tau;
  p.out.repair_list = b.repair_list;
  p.out.repair_count = b.repair_count;
  p.out.repair_cap = b.repair_cap;
  p.out.n_repair = b.counters + kCntOverflow;
  p.out.dense = b.dense != nullptr;
  p.out.err = b.err;
  p.dense = b.dense;
  p.dense_ld = b.dense_ld;
  p.counters = b.counters;
  p.err = b.err;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.H = v.H;
  p.n_items = (int)((v.rows + kItemQueries - 1) / kItemQueries);
  p.K = K;
  p.seg_cap = b.seg_cap;
  p.seed_first = h.cfg.seed_first;
  p.seed_last = h.cfg.seed_last;
  p.steps = steps;
  p.step_list = use_list == 1 ? b.step_list : nullptr;
  p.step_count = use_list == 1 ? b.step_count : nullptr;
  p.step_cap = b.step_cap;
  if (p.n_items == 0) return cudaSuccess;
  const int grid = p.n_items < sms ? p.n_items : sms;
  profile_before(DOSA_KERNEL_CERTIFIED, stream);
  auto fn = v.H == 64 ? certified_kernel<kFp8, 64> : certified_kernel<kFp8, 32>;
  fn<<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, bmap, kmap, p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_CERTIFIED, stream);
  return e;
}

cudaError_t launch_certified(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                             StepRange steps, cudaStream_t stream, int use_list) {
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    return launch_cert_impl<true>(h, v, b, K, steps, stream, use_list);
  return launch_cert_impl<false>(h, v, b, K, steps, stream, use_list);
}

size_t certified_smem_bytes(bool fp8) {
  return fp8 ? CertCfg<true>::kSmemBytes : CertCfg<false>::kSmemBytes;
}

}  // namespace dosa
