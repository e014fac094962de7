// Filter scorer of the certified indexer for sm_100a: exact scores of every
// visible pair of a work item, filtered against the running threshold and
// written back packed ("DOSA: Dots Sparse Attention", Daily Paper Cast
// transcript, Method section: exact scoring fused with the threshold test and
// the packed writeback; GPU kernel design: query tiles of a fixed width as
// dense tensor-core products).
//
// Tiles: A = 128 keys x d, B = 2 queries x 64 heads (N = 128).  Key tiles
// are taken two at a time: each of the two 256-column TMEM accumulators holds
// one query pair against both tiles (tile 0 in columns 0-127, tile 1 in
// 128-255), so an epilogue thread reduces two keys of the same query per
// accumulator wait, with the query's weights loaded once for both.  One
// persistent CTA per SM runs a TMA producer warp, an MMA warp and 16 epilogue
// warps in two teams of 8 (team t drains accumulator t: query pairs t and
// t + 2).  The epilogue keeps the candidate state of the item's 8 queries in
// shared memory (cand_state.cuh) and appends only scores >= tau_t,
// refreshing tau_t every 8 key tiles.
//
// A launch processes a range of steps of every item (work_items.cuh): the
// warm-up tiles before screening starts, the rest of the items that the
// certified kernel's probe found screening does not pay for (resuming their
// state), or every tile when screening is switched off.
#include <type_traits>

#include "cand_state.cuh"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "score_epilogue.cuh"
#include "work_items.cuh"

namespace dosa {

template <bool kFp8>
struct FilterCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kKeyStages = kFp8 ? 4 : 2;
  static constexpr int kH = 64;
  static constexpr int kQT = kItemQueries;
  static constexpr int kQRows = kQT * kH;
  static constexpr int kGroupRows = 128;               // MMA N: 2 queries
  static constexpr int kGroups = kQRows / kGroupRows;  // 4 query pairs
  static constexpr int kBufCols = 256;                 // a query pair over two key tiles
  static constexpr uint32_t kKeySubBytes = kKeyTile * 128;
  static constexpr uint32_t kKeyStageBytes = kKeySubBytes * kSub;
  static constexpr uint32_t kQSubBytes = kQRows * 128;
  static constexpr uint32_t kQBytes = kQSubBytes * kSub;
  static constexpr int kEpiWarps = 16;                 // 4 per TMEM lane quadrant
  static constexpr int kThreads = 64 + kEpiWarps * 32;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kStateBytes = sizeof(QState) * kQT;
  static constexpr uint32_t kSmemBytes =
      1024 + kQBytes + kKeyStages * kKeyStageBytes + kStateBytes + 256;
};

template <bool kFp8>
struct FilterTileCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kKeyStages = kFp8 ? 4 : 2;
  static constexpr int kH = 64;
  static constexpr int kQT = kItemQueries;
  static constexpr int kQRows = kQT * kH;
  static constexpr int kGroupRows = 256;               // MMA N: 4 queries
  static constexpr int kGroups = kQRows / kGroupRows;
  static constexpr int kQPerGroup = kGroupRows / kH;
  static constexpr uint32_t kKeySubBytes = kKeyTile * 128;
  static constexpr uint32_t kKeyStageBytes = kKeySubBytes * kSub;
  static constexpr uint32_t kQSubBytes = kQRows * 128;
  static constexpr uint32_t kQBytes = kQSubBytes * kSub;
  static constexpr int kEpiWarps = 16;                 // 4 per TMEM lane quadrant
  static constexpr int kThreads = 64 + kEpiWarps * 32;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kStateBytes = sizeof(QState) * kQT;
  static constexpr uint32_t kSmemBytes =
      1024 + kQBytes + kKeyStages * kKeyStageBytes + kStateBytes + 256;
};

struct FilterParams {
  const float* w;          // [rows_total, 64] absolute rows
  const float* q_scale;    // absolute rows (fp8)
  const float* k_scale;    // sequence base (fp8)
  Cand* cand;              // [chunk rows][kSegs][seg_cap]
  QStateG* qstate;         // [chunk rows] state handed over by the probe pass
  const int* item_flag;    // [n_items] decisions of the probe pass
  PublishOut out;
  unsigned long long* counters;
  int* err;
  int64_t row0, rows, pos0, S;
  int n_items, K, seg_cap, seed_first, seed_last;
  int H;                   // heads per query row: 32 or 64 (the MMA always sees 64)
  float* dense;            // dense writeback (ablation): [chunk rows, dense_ld], or null
  int64_t dense_ld;
  StepRange steps;         // what this launch processes
};

// One key tile per accumulator wait (B = 4 queries x 64 heads, N = 256, two
// 256-column accumulators; 16 epilogue warps, each reducing one key of a
// query per wait).  Used for bf16, whose two-stage key pipeline (the 8-query
// bf16 Q tile takes 128 KB of shared memory) cannot hold a second key tile
// ahead of a pair of tiles.
// kHeads: heads per query row (32 or 64); the MMA always sees 64 head slots.
// kDense: also write every exact score to p.dense (the dense-writeback ablation).
template <bool kFp8, int kHeads, bool kDense>
__global__ void __launch_bounds__(FilterTileCfg<kFp8>::kThreads, 1)
    filter_tile_kernel(const __grid_constant__ CUtensorMap qmap,
                  const __grid_constant__ CUtensorMap kmap, const FilterParams p) {
  using C = FilterTileCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kQBytes;
  QState* st = reinterpret_cast<QState*>(sK + C::kKeyStages * C::kKeyStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(st + C::kQT);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* acc_full = bars + 2;     // [2]
  uint64_t* acc_empty = bars + 4;    // [2]
  uint64_t* tile_done = bars + 6;
  uint64_t* item_ready = bars + 7;
  uint64_t* done_bar = bars + 8;
  uint64_t* k_full = bars + 9;                   // [kKeyStages]
  uint64_t* k_empty = k_full + C::kKeyStages;    // [kKeyStages]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(k_empty + C::kKeyStages);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
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
        mbar_arrive_expect_tx(q_full, C::kQBytes);
        for (int sub = 0; sub < C::kSub; ++sub)
          for (int b = 0; b < C::kQRows / 256; ++b)
            tma_load_3d(sQ + sub * C::kQSubBytes + b * 256 * 128, &qmap, q_full, sub * 64, 0,
                        (int32_t)(g.t0 + b * 4));
        inflight_q = it & 1;
        ++it;
        for (int ti = rg.begin; ti < rg.end; ++ti, ++kc) {
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
      constexpr uint32_t idesc = make_idesc<kFp8>(kKeyTile, C::kGroupRows);
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
        for (int ti = rg.begin; ti < rg.end && ok; ++ti, ++kc) {
          const int s_ = kc % C::kKeyStages;
          if (!mbar_wait(&k_full[s_], (kc / C::kKeyStages) & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + s_ * C::kKeyStageBytes);
          for (int grp = 0; grp < C::kGroups; ++grp, ++u) {
            const uint32_t buf = u & 1;
            if (!mbar_wait(&acc_empty[buf], ((u >> 1) & 1) ^ 1, s_abort, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t b_base = smem_u32(sQ + grp * C::kGroupRows * 128);
            const uint32_t d = tmem_base + buf * C::kGroupRows;
#pragma unroll
            for (int step = 0; step < C::kKSteps; ++step) {
              const uint32_t sub = step >> 2, off = (step & 3) * 32;
              tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                           smem_desc_sw128(b_base + sub * C::kQSubBytes + off), idesc,
                           step > 0 ? 1u : 0u);
            }
            tc_commit(&acc_full[buf]);
          }
          tc_commit(&k_empty[s_]);
        }
        tc_commit(q_empty);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    // 16 warps: warp (2 + ew) reads TMEM lane quadrant (warp & 3), i.e. 32
    // keys, and query (ew >> 2) of each 4-query MMA tile.  Warps 0-7 of the
    // epilogue also own query slot ew (state set-up, threshold refresh,
    // publication).
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int sub = ew >> 2;
    const bool owner = ew < C::kQT;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t u = 0, nbar = 0;
    int it = 0;
    unsigned long long n_seed = 0, n_exact = 0, n_cand = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
      const Range rg = item_steps(p.steps, p.item_flag, g, item);
      if (rg.end <= rg.begin) continue;
      const int n = rg.end - rg.begin;
      if (owner) {
        QState& s = st[ew];
        const bool valid = ew < g.nq;
        const int64_t row = g.local0 + ew;
        if (lane == 0) {
          s.row = row;
          s.pos = valid ? g.pos_first + ew : -1;
        }
        if (valid && rg.begin > 0) state_load(s, p.qstate + row, lane);
        else state_fresh(s, valid, lane);
        __syncwarp();
        __threadfence_block();
        if (valid && lane == 0) {
          // Visible and seed pairs of this query in the item's range: step 0
          // is key tile 0, steps ti >= 1 are key tiles n_tiles - ti.
          const int64_t pos = g.pos_first + ew;
          const int64_t nonseed_lo = p.seed_first, nonseed_hi = pos - p.seed_last;
          long long vis = 0, nonseed = 0;
          if (rg.begin == 0) {
            vis += overlap_count(0, kKeyTile - 1, 0, pos);
            nonseed += overlap_count(0, (kKeyTile - 1 < pos ? kKeyTile - 1 : pos), nonseed_lo,
                                     nonseed_hi);
          }
          const int t_first = rg.begin > 1 ? rg.begin : 1;
          if (t_first < rg.end) {
            const int64_t k_lo = (int64_t)(g.n_tiles - (rg.end - 1)) * kKeyTile;
            const int64_t k_hi = (int64_t)(g.n_tiles - t_first) * kKeyTile + kKeyTile - 1;
            vis += overlap_count(k_lo, k_hi, 0, pos);
            nonseed += overlap_count(k_lo, (k_hi < pos ? k_hi : pos), nonseed_lo, nonseed_hi);
          }
          n_exact += vis;
          n_seed += vis - nonseed;
        }
      }
      if (lane == 0) mbar_arrive(item_ready);
      if (!mbar_wait(item_ready, it & 1, s_abort, p.err)) break;
      ++it;
      // Per item: this warp's queries sub (MMA tile 0) and 4 + sub (tile 1),
      // their positions, weight rows, scales, list segments and counts.
      const int qa = sub, qb = C::kQPerGroup + sub;
      const bool va = qa < g.nq, vb = qb < g.nq;
      const int pos_a = (int)(g.pos_first + qa), pos_b = (int)(g.pos_first + qb);
      const float* wa = p.w + (g.t0 + (va ? qa : g.nq - 1)) * kHeads;
      const float* wb = p.w + (g.t0 + (vb ? qb : g.nq - 1)) * kHeads;
      constexpr bool h64 = kHeads == 64;
      float qsa = 1.f, qsb = 1.f;
      if constexpr (kFp8) {
        qsa = __ldg(p.q_scale + g.t0 + (va ? qa : 0));
        qsb = __ldg(p.q_scale + g.t0 + (vb ? qb : 0));
      }
      Cand* la = p.cand + ((g.local0 + qa) * kSegs + quad) * (int64_t)p.seg_cap;
      Cand* lb = p.cand + ((g.local0 + qb) * kSegs + quad) * (int64_t)p.seg_cap;
      int cnt_a = *reinterpret_cast<volatile int*>(&st[qa].seg[quad]);
      int cnt_b = *reinterpret_cast<volatile int*>(&st[qb].seg[quad]);
      const uint32_t col0 = tmem_base + lane_off + sub * 64;
      for (int i = 0; i < n && ok; ++i) {
        const int s = tile_at(rg.begin + i, g.n_tiles) * kKeyTile + quad * 32 + lane;
        float sk = 1.f;
        if constexpr (kFp8) sk = s < p.S ? __ldg(p.k_scale + s) : 0.f;
#pragma unroll
        for (int grp = 0; grp < C::kGroups; ++grp) {
          if (!ok) continue;
          const uint32_t buf = u & 1;
          if (!mbar_wait(&acc_full[buf], (u >> 1) & 1, s_abort, p.err)) {
            ok = false;
            continue;
          }
          ++u;
          tc_fence_after();
          // 32 heads at a time (the register budget of 18 warps is 96 per thread)
          const uint32_t col = col0 + buf * C::kGroupRows;
          const float* wq = grp ? wb : wa;
          float x[32];
          HeadAcc2 acc = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          tmem_ld32_async(col, x);
          tmem_wait_ld(x);
          if (h64) {
            head_accumulate32(acc, x, wq);
            tmem_ld32_async(col + 32, x);
            tmem_wait_ld(x);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
          head_accumulate32(acc, x, wq + (h64 ? 32 : 0));   // H = 32: heads 0-31 only
          if (grp ? vb : va) {
            QState& q = st[grp ? qb : qa];
            float sc = head_total(acc);
            if constexpr (kFp8) sc *= (grp ? qsb : qsa) * sk;
            const float tau = *reinterpret_cast<const volatile float*>(&q.tau);
            int& cnt = grp ? cnt_b : cnt_a;
            n_cand += append_candidates(q, grp ? lb : la, p.seg_cap, cnt,
                                        s <= (grp ? pos_b : pos_a) && sc >= tau, sc, s, lane);
            if constexpr (kDense)
              if (s <= (grp ? pos_b : pos_a))
                p.dense[(g.local0 + (grp ? qb : qa)) * p.dense_ld + s] = sc;
          }
        }
        if (!ok) break;
        // ---- checkpoint: every kCkptTiles steps and at the item's last ----
        if (((i + 1) % kCkptTiles) == 0 || i + 1 == n) {
          // publish this warp's segment counts (see certified.cu)
          if (lane == 0) {
            st[qa].seg[quad] = cnt_a;
            st[qb].seg[quad] = cnt_b;
          }
          __threadfence_block();
          if (lane == 0) mbar_arrive(tile_done);
          if (!mbar_wait(tile_done, nbar & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          ++nbar;
          if (owner && ew < g.nq)
            refresh_threshold(st[ew], p.cand + st[ew].row * kSegs * (int64_t)p.seg_cap, p.seg_cap,
                              p.K, lane);
        }
      }
      if (ok && owner && ew < g.nq) {
        if (rg.end < g.n_tiles) state_save(st[ew], p.qstate + st[ew].row, lane);
        else if (lane == 0) publish_query(st[ew], p.out);
      }
    }
    if (lane == 0) {
      atomicAdd(&p.counters[kCntSeedPairs], n_seed);
      atomicAdd(&p.counters[kCntExact], n_exact);
      atomicAdd(&p.counters[kCntCandidates], n_cand);
      atomicAdd(&p.counters[kCntFiltered], n_exact);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// kHeads: heads per query row (32 or 64); the MMA always sees 64 head slots.
// kDense: also write every exact score to p.dense (the dense-writeback ablation).
template <bool kFp8, int kHeads, bool kDense>
__global__ void __launch_bounds__(FilterCfg<kFp8>::kThreads, 1)
    filter_kernel(const __grid_constant__ CUtensorMap qmap,
                  const __grid_constant__ CUtensorMap kmap, const FilterParams p) {
  using C = FilterCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kQBytes;
  QState* st = reinterpret_cast<QState*>(sK + C::kKeyStages * C::kKeyStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(st + C::kQT);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* acc_full = bars + 2;     // [2]
  uint64_t* acc_empty = bars + 4;    // [2]
  uint64_t* tile_done = bars + 6;
  uint64_t* item_ready = bars + 7;
  uint64_t* done_bar = bars + 8;
  uint64_t* k_full = bars + 9;                   // [kKeyStages]
  uint64_t* k_empty = k_full + C::kKeyStages;    // [kKeyStages]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(k_empty + C::kKeyStages);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps / 2);   // one team of 8 warps per buffer
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
        mbar_arrive_expect_tx(q_full, C::kQBytes);
        for (int sub = 0; sub < C::kSub; ++sub)
          for (int b = 0; b < C::kQRows / 256; ++b)
            tma_load_3d(sQ + sub * C::kQSubBytes + b * 256 * 128, &qmap, q_full, sub * 64, 0,
                        (int32_t)(g.t0 + b * 4));
        inflight_q = it & 1;
        ++it;
        for (int ti = rg.begin; ti < rg.end; ++ti, ++kc) {
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
      constexpr uint32_t idesc = make_idesc<kFp8>(kKeyTile, C::kGroupRows);
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
        for (int ti = rg.begin; ti < rg.end && ok; ti += 2) {
          const bool two = ti + 1 < rg.end;
          const int sa = kc % C::kKeyStages, sb = (kc + 1) % C::kKeyStages;
          if (!mbar_wait(&k_full[sa], (kc / C::kKeyStages) & 1, s_abort, p.err) ||
              (two && !mbar_wait(&k_full[sb], ((kc + 1) / C::kKeyStages) & 1, s_abort, p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sK + sa * C::kKeyStageBytes);
          const uint32_t a1 = smem_u32(sK + sb * C::kKeyStageBytes);
          for (int grp = 0; grp < C::kGroups; ++grp, ++u) {
            const uint32_t buf = u & 1;
            if (!mbar_wait(&acc_empty[buf], ((u >> 1) & 1) ^ 1, s_abort, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t b_base = smem_u32(sQ + grp * C::kGroupRows * 128);
            for (int t = 0; t < (two ? 2 : 1); ++t) {
              const uint32_t a_base = t ? a1 : a0;
              const uint32_t d = tmem_base + buf * C::kBufCols + t * C::kGroupRows;
#pragma unroll
              for (int step = 0; step < C::kKSteps; ++step) {
                const uint32_t sub = step >> 2, off = (step & 3) * 32;
                tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kKeySubBytes + off),
                             smem_desc_sw128(b_base + sub * C::kQSubBytes + off), idesc,
                             step > 0 ? 1u : 0u);
              }
            }
            tc_commit(&acc_full[buf]);
          }
          if (!ok) break;
          tc_commit(&k_empty[sa]);
          if (two) tc_commit(&k_empty[sb]);
          kc += two ? 2 : 1;
        }
        tc_commit(q_empty);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    // 16 warps: warp (2 + ew) reads TMEM lane quadrant (warp & 3), i.e. 32
    // keys of each key tile, in team (ew >> 2) & 1, for query (ew >> 3) of
    // each query pair.  Warps 0-7 of the epilogue also own query slot ew
    // (state set-up, threshold refresh, publication).
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int sub = ew >> 2;
    const int team = sub & 1, qsel = sub >> 1;   // buffer and query within the pair
    const bool owner = ew < C::kQT;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t uu = 0, nbar = 0;
    int it = 0;
    unsigned long long n_seed = 0, n_exact = 0, n_cand = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
      const Range rg = item_steps(p.steps, p.item_flag, g, item);
      if (rg.end <= rg.begin) continue;
      const int n = rg.end - rg.begin;
      if (owner) {
        QState& s = st[ew];
        const bool valid = ew < g.nq;
        const int64_t row = g.local0 + ew;
        if (lane == 0) {
          s.row = row;
          s.pos = valid ? g.pos_first + ew : -1;
        }
        if (valid && rg.begin > 0) state_load(s, p.qstate + row, lane);
        else state_fresh(s, valid, lane);
        __syncwarp();
        __threadfence_block();
        if (valid && lane == 0) {
          // Visible and seed pairs of this query in the item's range: step 0
          // is key tile 0, steps ti >= 1 are key tiles n_tiles - ti.
          const int64_t pos = g.pos_first + ew;
          const int64_t nonseed_lo = p.seed_first, nonseed_hi = pos - p.seed_last;
          long long vis = 0, nonseed = 0;
          if (rg.begin == 0) {
            vis += overlap_count(0, kKeyTile - 1, 0, pos);
            nonseed += overlap_count(0, (kKeyTile - 1 < pos ? kKeyTile - 1 : pos), nonseed_lo,
                                     nonseed_hi);
          }
          const int t_first = rg.begin > 1 ? rg.begin : 1;
          if (t_first < rg.end) {
            const int64_t k_lo = (int64_t)(g.n_tiles - (rg.end - 1)) * kKeyTile;
            const int64_t k_hi = (int64_t)(g.n_tiles - t_first) * kKeyTile + kKeyTile - 1;
            vis += overlap_count(k_lo, k_hi, 0, pos);
            nonseed += overlap_count(k_lo, (k_hi < pos ? k_hi : pos), nonseed_lo, nonseed_hi);
          }
          n_exact += vis;
          n_seed += vis - nonseed;
        }
      }
      if (lane == 0) mbar_arrive(item_ready);
      if (!mbar_wait(item_ready, it & 1, s_abort, p.err)) break;
      ++it;
      // Per item: this warp's two queries, qa (query pair `team`) and qb = qa + 4
      // (query pair team + 2), their positions, weight rows, scales, list
      // segments and counts.  Per pair of key tiles the warp takes 2 keys of
      // qa, then 2 keys of qb, from buffer `team`.
      const int qa = 2 * team + qsel, qb = qa + 4;
      const bool va = qa < g.nq, vb = qb < g.nq;
      const int pos_a = va ? (int)(g.pos_first + qa) : -1;
      const int pos_b = vb ? (int)(g.pos_first + qb) : -1;
      const float* wa = p.w + (g.t0 + (va ? qa : g.nq - 1)) * kHeads;
      const float* wb = p.w + (g.t0 + (vb ? qb : g.nq - 1)) * kHeads;
      constexpr bool h64 = kHeads == 64;
      float qsa = 1.f, qsb = 1.f;
      if constexpr (kFp8) {
        qsa = __ldg(p.q_scale + g.t0 + (va ? qa : 0));
        qsb = __ldg(p.q_scale + g.t0 + (vb ? qb : 0));
      }
      Cand* la = p.cand + ((g.local0 + qa) * kSegs + quad) * (int64_t)p.seg_cap;
      Cand* lb = p.cand + ((g.local0 + qb) * kSegs + quad) * (int64_t)p.seg_cap;
      int cnt_a = *reinterpret_cast<volatile int*>(&st[qa].seg[quad]);
      int cnt_b = *reinterpret_cast<volatile int*>(&st[qb].seg[quad]);
      const uint32_t col0 = tmem_base + lane_off + team * C::kBufCols + qsel * C::kH;
      for (int i = 0; i < n && ok; i += 2) {
        const bool two = i + 1 < n;
        const int s0 = tile_at(rg.begin + i, g.n_tiles) * kKeyTile + quad * 32 + lane;
        const int s1 = two ? tile_at(rg.begin + i + 1, g.n_tiles) * kKeyTile + quad * 32 + lane
                           : 0x7FFFFFFF;
        float sk0 = 1.f, sk1 = 1.f;
        if constexpr (kFp8) {
          sk0 = s0 < p.S ? __ldg(p.k_scale + s0) : 0.f;
          sk1 = s1 < p.S ? __ldg(p.k_scale + s1) : 0.f;
        }
        // the body specialised on whether the second key tile exists (every
        // pair but an odd item's last tile): no per-quarter branch on it
        auto uses = [&](auto two_c) {
          constexpr bool two = decltype(two_c)::value;
#pragma unroll
          for (int use = 0; use < 2; ++use) {
            if (!ok) continue;
            if (!mbar_wait(&acc_full[team], uu & 1, s_abort, p.err)) {
              ok = false;
              continue;
            }
            ++uu;
            tc_fence_after();
            const float* wq = use ? wb : wa;
            HeadAcc2 acc0 = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            HeadAcc2 acc1 = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float x[16];
            float4 w4[4];
            constexpr int kQuarters = h64 ? 4 : 2;
#pragma unroll
            for (int hh = 0; hh < kQuarters; ++hh) {
              load_w16(w4, wq + 16 * hh);
              tmem_ld16_async(col0 + 16 * hh, x);
              tmem_wait_ld16(x);
              head_accumulate16w(acc0, x, w4);
              if constexpr (two) {
                tmem_ld16_async(col0 + C::kGroupRows + 16 * hh, x);
                tmem_wait_ld16(x);
              }
              if (hh == kQuarters - 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[team]);
              }
              if constexpr (two) head_accumulate16w(acc1, x, w4);
            }
            // an invalid query slot (past the item's last row) never appends:
            // its position is -1
            QState& q = st[use ? qb : qa];
            const float qs = use ? qsb : qsa;
            const int pos = use ? pos_b : pos_a;
            float sc0 = head_total(acc0), sc1 = head_total(acc1);
            if constexpr (kFp8) {
              sc0 *= qs * sk0;
              sc1 *= qs * sk1;
            }
            int& cnt = use ? cnt_b : cnt_a;
            Cand* lst = use ? lb : la;
            float tau = *reinterpret_cast<const volatile float*>(&q.tau);
            n_cand += append_candidates(q, lst, p.seg_cap, cnt, s0 <= pos && sc0 >= tau, sc0, s0,
                                        lane);
            if constexpr (two) {
              tau = *reinterpret_cast<const volatile float*>(&q.tau);
              n_cand += append_candidates(q, lst, p.seg_cap, cnt, s1 <= pos && sc1 >= tau, sc1,
                                          s1, lane);
            }
            if constexpr (kDense) {
              if (use ? vb : va) {
                float* drow = p.dense + (g.local0 + (use ? qb : qa)) * p.dense_ld;
                if (s0 <= pos) drow[s0] = sc0;
                if (two && s1 <= pos) drow[s1] = sc1;
              }
            }
          }
        };
        if (two) uses(std::true_type{});
        else uses(std::false_type{});
        if (!ok) break;
        // ---- checkpoint: every kCkptTiles steps and at the item's last ----
        if (((i + 2) % kCkptTiles) == 0 || i + 2 >= n) {
          // publish this warp's segment counts (see certified.cu)
          if (lane == 0) {
            st[qa].seg[quad] = cnt_a;
            st[qb].seg[quad] = cnt_b;
          }
          __threadfence_block();
          if (lane == 0) mbar_arrive(tile_done);
          if (!mbar_wait(tile_done, nbar & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          ++nbar;
          if (owner && ew < g.nq)
            refresh_threshold(st[ew], p.cand + st[ew].row * kSegs * (int64_t)p.seg_cap, p.seg_cap,
                              p.K, lane);
        }
      }
      if (ok && owner && ew < g.nq) {
        if (rg.end < g.n_tiles) state_save(st[ew], p.qstate + st[ew].row, lane);
        else if (lane == 0) publish_query(st[ew], p.out);
      }
    }
    if (lane == 0) {
      atomicAdd(&p.counters[kCntSeedPairs], n_seed);
      atomicAdd(&p.counters[kCntExact], n_exact);
      atomicAdd(&p.counters[kCntCandidates], n_cand);
      atomicAdd(&p.counters[kCntFiltered], n_exact);
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

// fp8: the pair kernel (two key tiles per accumulator wait); bf16: the
// one-tile kernel (see filter_tile_kernel).
template <bool kFp8, int kHeads, bool kDense>
constexpr auto filter_fn() {
  if constexpr (kFp8) return filter_kernel<kFp8, kHeads, kDense>;
  else return filter_tile_kernel<kFp8, kHeads, kDense>;
}

template <bool kFp8>
static cudaError_t launch_filter_impl(const Handle& h, const SeqView& v, const CertBuffers& b,
                                      int K, StepRange steps, cudaStream_t stream) {
  using C = std::conditional_t<kFp8, FilterCfg<kFp8>, FilterTileCfg<kFp8>>;
  CUtensorMap qmap, kmap;
  if (!encode_q_map(&qmap, v.q, kFp8, (uint64_t)(v.row0 + v.rows), v.H) ||
      !encode_rows_map(&kmap, v.k, kFp8, (uint64_t)v.S, kKeyTile))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    for (auto fn : {filter_fn<kFp8, 64, false>(), filter_fn<kFp8, 32, false>(),
                    filter_fn<kFp8, 64, true>(), filter_fn<kFp8, 32, true>()})
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  FilterParams p;
  p.w = v.w;
  p.q_scale = v.q_scale;
  p.k_scale = v.k_scale;
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
  p.dense = b.dense;
  p.dense_ld = b.dense_ld;
  p.out.err = b.err;
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
  if (p.n_items == 0) return cudaSuccess;
  const int grid = p.n_items < sms ? p.n_items : sms;
  profile_before(DOSA_KERNEL_FILTER, stream);
  auto fn = v.H == 64 ? (b.dense ? filter_fn<kFp8, 64, true>() : filter_fn<kFp8, 64, false>())
                      : (b.dense ? filter_fn<kFp8, 32, true>() : filter_fn<kFp8, 32, false>());
  fn<<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, kmap, p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_FILTER, stream);
  return e;
}

size_t qstate_bytes() { return sizeof(QStateG); }

cudaError_t launch_filter(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                          StepRange steps, cudaStream_t stream) {
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    return launch_filter_impl<true>(h, v, b, K, steps, stream);
  return launch_filter_impl<false>(h, v, b, K, steps, stream);
}

}  // namespace dosa
