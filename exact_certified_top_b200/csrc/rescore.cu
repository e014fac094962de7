// Survivor rescoring of the certified indexer for sm_100a ("DOSA: Dots Sparse
// Attention", Daily Paper Cast transcript, Method section, GPU kernel design:
// the keys that survive screening are packed into a separate stream per
// query and scored exactly with every head; only scores at or above the
// threshold are written back, packed).
//
// A pass of rank_screen leaves, per query row, one survivor bit per screened
// key.  One CTA takes a row at a time:
//   warp 0      compaction: reads the row's survivor words (bulk copies into
//               shared memory, 64 words per step, prefix sums of the popcounts
//               from bit-sliced ballots) into a ring of key indices and cuts
//               it into tiles of 128 keys; it also TMA-loads the row's 64
//               head slots
//   warp 1      MMA: M = 128 gathered keys x N = 64 heads, fp32 in TMEM
//   warps 2-5   epilogue, one TMEM lane quadrant each: the head reduction
//               shared with every other scorer (bit-identical scores), the
//               threshold filter and the packed append; the threshold is
//               refreshed from the histogram every 8 tiles and at the row end
//   warps 6-7   gather, alternate tiles: 16-byte cp.async into the 128-byte
//               swizzled layout the MMA reads, eight lanes per key row so
//               that one instruction moves four whole rows; a tile is handed
//               to the MMA once it has landed
// At the row end the owner warp checks the pass: if a key the pass rejected
// has a bound at or above the threshold now reached, the row gets the next
// band [max(tau, next estimate), this pass's lower limit) and its state is
// saved; otherwise the row is published for the selection.
#include "cand_state.cuh"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "score_epilogue.cuh"
#include "work_items.cuh"

namespace dosa {

template <bool kFp8>
struct RsCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kStages = 4;                        // gathered key tiles
  static constexpr int kGatherWarps = 2;                   // copy issuers, alternate tiles
  static constexpr int kBufs = 4;                          // TMEM accumulators of 64 columns
  static constexpr int kChunk = 128;                       // keys per MMA tile
  static constexpr int kHeadsN = 64;                       // MMA N: one row's head slots
  static constexpr int kKeySlots = 8;                      // tiles' key lists
  static constexpr int kScanWords = 64;                    // survivor words per scan half-step
  static constexpr int kRing = 4096;                       // survivor keys staged by warp 0
  static constexpr int kBitsWords = 512;                   // survivor words per bulk copy
  static_assert(kRing >= kScanWords * 32 + kChunk, "a half-step must fit in the ring");
  static_assert((kRing & (kRing - 1)) == 0, "ring positions wrap by mask");
  static_assert(kBitsWords % kScanWords == 0, "a scan step stays inside one piece");
  static_assert(kKeySlots % kGatherWarps == 0, "a gather warp keeps its key slots");
  static constexpr int kCtasPerSm = kFp8 ? 2 : 1;
  static constexpr uint32_t kASubBytes = kChunk * 128;
  static constexpr uint32_t kAStageBytes = kASubBytes * kSub;
  static constexpr uint32_t kBSubBytes = kHeadsN * 128;
  static constexpr uint32_t kBBytes = kBSubBytes * kSub;
  static constexpr int kEpiWarps = 4;
  static constexpr int kGatherWarp0 = 2 + kEpiWarps;
  static constexpr int kThreads = 32 * (kGatherWarp0 + kGatherWarps);
  static constexpr uint32_t kTmemCols = kBufs * kHeadsN;
  static constexpr int kCkptChunks = 8;
  static constexpr uint32_t kSmemBytes = 1024 + 2 * kBBytes + kStages * kAStageBytes +
                                         kKeySlots * (kChunk * 8 + 16) + kRing * 4 +
                                         2 * kBitsWords * 4 + 256 + (uint32_t)sizeof(QState) + 1024;
};

struct RescoreParams {
  const void* k;             // the sequence's first key (codes)
  const float* k_scale;      // the sequence's first key scale (fp8)
  const float* w;            // [rows_total, H] absolute rows
  const float* q_scale;      // absolute rows (fp8)
  const uint32_t* bits;      // [chunk rows][words] survivor bits of this pass
  int64_t words;
  Cand* cand;                // [chunk rows][kSegs][seg_cap]
  QStateG* qstate;           // [chunk rows] carried candidate state
  const int* item_sel;       // [n_items] or null
  int want;
  int pass;
  int* row_next;             // [chunk rows] pass a row waits for
  float* band_lo;            // [chunk rows] this pass's band; the next one on exit
  float* band_hi;
  uint32_t* maxrej;          // [chunk rows] ordered largest bound this pass rejected
  const float* est;          // [chunk rows][kRankEst] threshold estimates
  int* pass_any;             // this pass has rows
  int* pass_any_next;        // set when a row needs the next pass
  PublishOut out;
  float* dense;              // dense writeback (ablation): [chunk rows, dense_ld], or null
  int64_t dense_ld;
  unsigned long long* counters;
  int* err;
  int64_t row0, rows, pos0, S;
  int n_items, W, K, seg_cap;
};

struct StageMeta {
  int count;    // valid keys in the tile; -1: no more tiles (gather warps stop)
  int end;      // last tile of its row
  int pad[2];
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Chunk row handled at flat index f (work items longest first, 8 rows each),
// or -1 when it is not part of this pass.
__device__ __forceinline__ int64_t rescore_row_at(const RescoreParams& p, int f) {
  const int item = f / kItemQueries;
  const int64_t r = (int64_t)(p.n_items - 1 - item) * kItemQueries + f % kItemQueries;
  if (r >= p.rows) return -1;
  if (p.item_sel && p.item_sel[item] != p.want) return -1;
  if (p.row_next[r] != p.pass) return -1;
  return r;
}

// Warp-wide exclusive prefix sum and total of per-lane counts below 128, from
// one ballot per bit of the count (independent ballots instead of a chain of
// dependent shuffles).
__device__ __forceinline__ uint32_t warp_excl_sum7(uint32_t cnt, int lane, uint32_t& total) {
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t excl = 0, tot = 0;
#pragma unroll
  for (int b = 0; b < 7; ++b) {
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, (cnt >> b) & 1u);
    excl += (uint32_t)__popc(m & lt) << b;
    tot += (uint32_t)__popc(m) << b;
  }
  total = tot;
  return excl;
}

template <bool kFp8, int kHeads>
__global__ void __launch_bounds__(RsCfg<kFp8>::kThreads, RsCfg<kFp8>::kCtasPerSm)
    rescore_kernel(const __grid_constant__ CUtensorMap qmap, const RescoreParams p) {
  using C = RsCfg<kFp8>;
  if (*p.pass_any == 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                            // [2] query head tiles
  uint8_t* sA = sQ + 2 * C::kBBytes;                             // [kStages] key tiles
  int* skeys = reinterpret_cast<int*>(sA + C::kStages * C::kAStageBytes);   // [kKeySlots][128]
  float* sscale = reinterpret_cast<float*>(skeys + C::kKeySlots * C::kChunk);  // [kKeySlots][128]
  StageMeta* meta = reinterpret_cast<StageMeta*>(sscale + C::kKeySlots * C::kChunk);
  int* ring = reinterpret_cast<int*>(meta + C::kKeySlots);
  uint32_t* sbits = reinterpret_cast<uint32_t*>(ring + C::kRing);     // [2][kBitsWords]
  float* sw = reinterpret_cast<float*>(sbits + 2 * C::kBitsWords);   // [64] the row's weights
  QState* st = reinterpret_cast<QState*>(sw + 64);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(st + 1) + 7) & ~uintptr_t(7));
  uint64_t* q_full = bars;                          // [2]
  uint64_t* q_empty = bars + 2;                     // [2]
  uint64_t* a_full = bars + 4;                      // [kStages] a tile's codes landed
  uint64_t* a_empty = a_full + C::kStages;          // [kStages] ... and were read by the MMA
  uint64_t* acc_full = a_empty + C::kStages;        // [kBufs]
  uint64_t* acc_empty = acc_full + C::kBufs;        // [kBufs]
  uint64_t* k_full = acc_empty + C::kBufs;          // [kKeySlots] a tile's key list is cut
  uint64_t* sc_full = k_full + C::kKeySlots;        // [kKeySlots] ... its scales landed
  uint64_t* ks_empty = sc_full + C::kKeySlots;      // [kKeySlots] ... read by the epilogue
  uint64_t* bits_full = ks_empty + C::kKeySlots;    // [2] a piece of survivor words landed
  uint64_t* done_bar = bits_full + 2;
  uint64_t* ep_bar = done_bar + 1;                  // epilogue meeting point
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(ep_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_flat = p.n_items * kItemQueries;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);                  // the MMA's commit
    }
    for (int i = 0; i < C::kKeySlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&sc_full[i], 1);
      mbar_init(&ks_empty[i], C::kEpiWarps);
    }
    mbar_init(&bits_full[0], 1);
    mbar_init(&bits_full[1], 1);
    for (int i = 0; i < C::kBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(done_bar, 1);
    mbar_init(ep_bar, C::kEpiWarps);
    *s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
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
    // ---------------- compaction: survivor words -> key tiles ----------------
    uint32_t ac = 0, qc = 0, bc = 0;             // bc: survivor-word pieces of earlier rows
    int fetched = 0, waited = 0;                 // pieces of the current row in flight / landed
    bool ok = true;
    for (int f = blockIdx.x; f < n_flat && ok; f += gridDim.x) {
      const int64_t r = rescore_row_at(p, f);
      if (r < 0) continue;
      // the head tile buffer is free once the MMA finished the row before the
      // last one (the gather warps hand every tile over without waiting here)
      if (lane == 0) {
        if (!mbar_wait(&q_empty[qc & 1], ((qc >> 1) & 1) ^ 1, s_abort, p.err)) ok = false;
        if (ok) {
          mbar_arrive_expect_tx(&q_full[qc & 1], C::kBBytes);
          for (int sub = 0; sub < C::kSub; ++sub)
            tma_load_3d(sQ + (qc & 1) * C::kBBytes + sub * C::kBSubBytes, &qmap, &q_full[qc & 1],
                        sub * 64, 0, (int32_t)(p.row0 + r));
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++qc;
      const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items,
                                   p.n_items - 1 - (int)(r / kItemQueries));
      const int64_t L = g.n_tiles - p.W + 1;                   // screened tiles [1, L)
      const int64_t wlo = 4, whi = L > 1 ? 4 * L : 4;
      // the row's survivor words come into shared memory in pieces of
      // kBitsWords (bulk copies, double-buffered: the next piece is in flight
      // while this one is scanned)
      const uint32_t* gwords = p.bits + r * p.words;
      const int64_t n_words = whi - wlo;
      const int n_pieces = (int)((n_words + C::kBitsWords - 1) / C::kBitsWords);
      auto fetch_piece = [&](int piece) {
        if (lane == 0 && piece < n_pieces) {
          const int64_t w0 = wlo + (int64_t)piece * C::kBitsWords;
          const int64_t nw = whi - w0 < C::kBitsWords ? whi - w0 : C::kBitsWords;
          const uint32_t b = (bc + piece) & 1;
          mbar_arrive_expect_tx(&bits_full[b], (uint32_t)nw * 4);
          bulk_copy_g2s(sbits + b * C::kBitsWords, gwords + w0, (uint32_t)nw * 4, &bits_full[b]);
        }
      };
      fetch_piece(0);
      fetch_piece(1);
      fetched = n_pieces < 2 ? n_pieces : 2;
      int piece = 0;                   // piece being scanned
      int pw = 0;                      // next word of it
      bool have = false;               // the piece has landed
      int64_t wpos = wlo;
      uint32_t n_avail = 0, rd = 0;
      while (ok) {
        // refill the ring until a full tile of survivors is staged; a step
        // takes two words per lane (keys in any order: the selection orders
        // candidates by score and index)
        while (n_avail - rd < (uint32_t)C::kChunk && wpos < whi) {
          const uint32_t b = (bc + piece) & 1;
          if (!have) {
            bool w_ok = true;
            if (lane == 0) w_ok = mbar_wait(&bits_full[b], ((bc + piece) >> 1) & 1, s_abort, p.err);
            if (!__shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0)) {
              ok = false;
              break;
            }
            have = true;
            waited = piece + 1;
            __syncwarp();
          }
          // two independent halves of 64 words (A, then B when the piece has
          // room for it), two adjacent words per lane in each: their prefix
          // sums and expansions interleave, so one step's dependency chain
          // covers 128 words.  B waits for the next step when both halves
          // together could overrun the ring (only at survivor densities
          // near one).
          const uint32_t* sb = sbits + b * C::kBitsWords + pw;
          const int64_t wa = wpos + 2 * lane, wb = wa + C::kScanWords;
          uint64_t ma = 0, mb = 0;
          if (wa < whi) {
            const uint2 v = *reinterpret_cast<const uint2*>(sb + 2 * lane);
            ma = ((uint64_t)v.y << 32) | v.x;
          }
          const bool half_b = pw + 2 * C::kScanWords <= C::kBitsWords;
          if (half_b && wb < whi) {
            const uint2 v = *reinterpret_cast<const uint2*>(sb + C::kScanWords + 2 * lane);
            mb = ((uint64_t)v.y << 32) | v.x;
          }
          uint32_t tot_a, tot_b;
          const uint32_t ex_a = warp_excl_sum7((uint32_t)__popcll(ma), lane, tot_a);
          const uint32_t ex_b = warp_excl_sum7((uint32_t)__popcll(mb), lane, tot_b);
          const bool take_b = half_b && (n_avail - rd) + tot_a + tot_b <= (uint32_t)C::kRing;
          if (!take_b) mb = 0;
          uint32_t at_a = n_avail + ex_a, at_b = n_avail + tot_a + ex_b;
          const int kb_a = (int)(wa * 32), kb_b = (int)(wb * 32);
          while (ma | mb) {
            if (ma) {
              ring[at_a & (C::kRing - 1)] = kb_a + __ffsll(ma) - 1;
              ++at_a;
              ma &= ma - 1;
            }
            if (mb) {
              ring[at_b & (C::kRing - 1)] = kb_b + __ffsll(mb) - 1;
              ++at_b;
              mb &= mb - 1;
            }
          }
          n_avail += tot_a + (take_b ? tot_b : 0u);
          const int adv = take_b ? 2 * C::kScanWords : C::kScanWords;
          wpos += adv;
          pw += adv;
          if (pw >= C::kBitsWords) {
            // piece done (every lane has used its words): its buffer takes
            // the piece after next
            fence_proxy_async_smem();
            __syncwarp();
            fetch_piece(piece + 2);
            if (piece + 2 < n_pieces) fetched = piece + 3;
            ++piece;
            pw = 0;
            have = false;
          }
        }
        if (!ok) break;
        __syncwarp();
        const uint32_t left = n_avail - rd;
        const int cnt = (int)(left < (uint32_t)C::kChunk ? left : (uint32_t)C::kChunk);
        const int end = (wpos >= whi && left <= (uint32_t)C::kChunk) ? 1 : 0;
        const int ks = (int)(ac % C::kKeySlots);
        bool w_ok = true;
        if (lane == 0)
          w_ok = mbar_wait(&ks_empty[ks], ((ac / C::kKeySlots) & 1) ^ 1, s_abort, p.err);
        if (!__shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int i = 0; i < C::kChunk / 32; ++i) {
          const int row = lane + 32 * i;
          skeys[ks * C::kChunk + row] = row < cnt ? ring[(rd + row) & (C::kRing - 1)] : -1;
        }
        if (lane == 0) {
          meta[ks].count = cnt;
          meta[ks].end = end;
        }
        __threadfence_block();
        __syncwarp();
        if (lane == 0) mbar_arrive(&k_full[ks]);
        rd += (uint32_t)cnt;
        ++ac;
        if (end) break;
      }
      // every piece of the row was fetched and waited for (a row's scan reads
      // all of its words before its last tile), so the buffers are free
      if (ok) {
        bc += (uint32_t)n_pieces;
        fetched = waited = 0;
      }
    }
    // one stop mark per gather warp, in the key slots they would read next
    for (int g = 0; g < C::kGatherWarps && ok; ++g, ++ac) {
      const int ks = (int)(ac % C::kKeySlots);
      bool w_ok = true;
      if (lane == 0) {
        w_ok = mbar_wait(&ks_empty[ks], ((ac / C::kKeySlots) & 1) ^ 1, s_abort, p.err);
        if (w_ok) {
          meta[ks].count = -1;
          meta[ks].end = 1;
          __threadfence_block();
          mbar_arrive(&k_full[ks]);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && *s_abort && qc > 0) mbar_wait_drain(&q_full[(qc - 1) & 1], ((qc - 1) >> 1) & 1);
    // survivor-word copies still in flight after an abort
    if (lane == 0 && *s_abort)
      for (int k = waited; k < fetched; ++k)
        mbar_wait_drain(&bits_full[(bc + k) & 1], ((bc + k) >> 1) & 1);
  } else if (warp >= C::kGatherWarp0) {
    // ---------------- gather: key codes into the swizzled tiles ----------------
    const int g = warp - C::kGatherWarp0;
    const int piece = lane & 7;        // 16-byte piece of a 128-byte row
    const int r4 = lane >> 3;          // row within each group of four
    // swizzled offsets of this lane's piece in rows r4 + 8m and r4 + 4 + 8m
    const uint32_t off0 = (uint32_t)(r4 * 128 + ((piece ^ r4) << 4));
    const uint32_t off1 = (uint32_t)((r4 + 4) * 128 + ((piece ^ (r4 + 4)) << 4));
    const char* kbase = static_cast<const char*>(p.k);
    constexpr int kRowBytes = kHeadDim * (kFp8 ? 1 : 2);
    bool held = false;                 // a tile issued and not yet handed over
    uint32_t held_c = 0;
    auto hand_over = [&]() {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a_full[held_c % C::kStages]);
        mbar_arrive(&sc_full[held_c % C::kKeySlots]);
      }
      held = false;
    };
    for (uint32_t c = (uint32_t)g;; c += C::kGatherWarps) {
      const int ks = (int)(c % C::kKeySlots), s_ = (int)(c % C::kStages);
      // never block with a tile held back: the MMA (and through it the
      // compaction warp) may be waiting for it
      bool ready = true;
      if (lane == 0) ready = mbar_try_wait(smem_u32(&k_full[ks]), (c / C::kKeySlots) & 1);
      if (!__shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) && held) {
        cp_async_wait<0>();
        hand_over();
      }
      bool w_ok = true;
      if (lane == 0) w_ok = mbar_wait(&k_full[ks], (c / C::kKeySlots) & 1, s_abort, p.err);
      if (!__shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0)) break;
      __syncwarp();                    // lane 0's acquire covers the whole warp
      const int count = reinterpret_cast<volatile int*>(&meta[ks].count)[0];
      if (count < 0) break;
      if (lane == 0) w_ok = mbar_wait(&a_empty[s_], ((c / C::kStages) & 1) ^ 1, s_abort, p.err);
      if (!__shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0)) break;
      const uint32_t stage = smem_u32(sA + s_ * C::kAStageBytes);
      const int* keys = skeys + ks * C::kChunk;
#pragma unroll 4
      for (int i = 0; i < C::kChunk / 4; ++i) {
        const int row = r4 + 4 * i;
        if (row < count) {
          const char* src = kbase + (int64_t)keys[row] * kRowBytes + piece * 16;
          const uint32_t dst = stage + (uint32_t)(i >> 1) * 1024u + ((i & 1) ? off1 : off0);
#pragma unroll
          for (int sub = 0; sub < C::kSub; ++sub)
            cp_async16(dst + sub * C::kASubBytes, src + sub * 128);
        }
      }
      if constexpr (kFp8) {
#pragma unroll
        for (int i = 0; i < C::kChunk / 32; ++i) {
          const int row = lane + 32 * i;
          if (row < count)
            cp_async4(smem_u32(sscale + ks * C::kChunk + row), p.k_scale + keys[row]);
        }
      }
      cp_async_commit();
      // the previous tile of this warp has landed once only the newest group
      // is pending
      if (held) {
        cp_async_wait<1>();
        hand_over();
      }
      held = true;
      held_c = c;
    }
    cp_async_wait<0>();
    if (held && !*s_abort) hand_over();
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc<kFp8>(C::kChunk, C::kHeadsN);
      uint32_t ac = 0, qc = 0;
      bool ok = true;
      for (int f = blockIdx.x; f < n_flat && ok; f += gridDim.x) {
        const int64_t r = rescore_row_at(p, f);
        if (r < 0) continue;
        const uint32_t qb = qc & 1;
        if (!mbar_wait(&q_full[qb], (qc >> 1) & 1, s_abort, p.err)) break;
        ++qc;
        tc_fence_after();
        const uint32_t b_base = smem_u32(sQ + qb * C::kBBytes);
        while (true) {
          const uint32_t s_ = ac % C::kStages, buf = ac % C::kBufs;
          if (!mbar_wait(&a_full[s_], (ac / C::kStages) & 1, s_abort, p.err) ||
              !mbar_wait(&acc_empty[buf], ((ac / C::kBufs) & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          const int end = reinterpret_cast<volatile int*>(&meta[ac % C::kKeySlots].end)[0];
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s_ * C::kAStageBytes);
          const uint32_t d = tmem_base + buf * C::kHeadsN;
#pragma unroll
          for (int step = 0; step < C::kKSteps; ++step) {
            const uint32_t sub = step >> 2, off = (step & 3) * 32;
            tc_mma<kFp8>(d, smem_desc_sw128(a_base + sub * C::kASubBytes + off),
                         smem_desc_sw128(b_base + sub * C::kBSubBytes + off), idesc,
                         step > 0 ? 1u : 0u);
          }
          tc_commit(&acc_full[buf]);
          tc_commit(&a_empty[s_]);
          ++ac;
          if (end) break;
        }
        tc_commit(&q_empty[qb]);
      }
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue: one TMEM lane quadrant per warp ----------------
    const int ew = warp - 2;
    const int quad = warp & 3;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    QState& q = *st;
    uint32_t ac = 0, nb = 0;
    unsigned long long n_exact = 0, n_cand = 0;
    bool ok = true;
    // the four epilogue warps meet on an mbarrier with bounded waits: after
    // an abort every wait returns at once, so no warp can be left behind
    auto meet = [&]() {
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(ep_bar);
      if (!mbar_wait(ep_bar, nb & 1, s_abort, p.err)) ok = false;
      ++nb;
    };
    for (int f = blockIdx.x; f < n_flat && ok; f += gridDim.x) {
      const int64_t r = rescore_row_at(p, f);
      if (r < 0) continue;
      if (ew == 0) {
        if (lane == 0) {
          q.row = r;
          q.pos = p.pos0 + r;
        }
        state_load(q, p.qstate + r, lane);
        // the row's head weights, read by every key of every tile
        const float* wq = p.w + (p.row0 + r) * kHeads;
        for (int h = lane; h < kHeads; h += 32) sw[h] = __ldg(wq + h);
      }
      meet();
      int cnt = *reinterpret_cast<volatile int*>(&q.seg[quad]);
      // a row whose threshold comes from the histogram alone (past warm-up)
      // refreshes it without meeting: counts only grow, so any snapshot of
      // the histogram gives a sound threshold
      const bool settled = *reinterpret_cast<volatile int*>(&q.phase) == 2;
      Cand* seg = p.cand + (r * kSegs + quad) * (int64_t)p.seg_cap;
      float qs = 1.f;
      if constexpr (kFp8) qs = __ldg(p.q_scale + p.row0 + r);
      for (int nc = 0; ok; ++nc) {
        const uint32_t ks = ac % C::kKeySlots, buf = ac % C::kBufs;
        if (!mbar_wait(&sc_full[ks], (ac / C::kKeySlots) & 1, s_abort, p.err) ||
            !mbar_wait(&acc_full[buf], (ac / C::kBufs) & 1, s_abort, p.err)) {
          ok = false;
          break;
        }
        const int end = reinterpret_cast<volatile int*>(&meta[ks].end)[0];
        const int tile_cnt = reinterpret_cast<volatile int*>(&meta[ks].count)[0];
        const int at = quad * 32 + lane;
        const bool valid = at < tile_cnt;
        const int key = valid ? skeys[ks * C::kChunk + at] : 0;
        float sk = 1.f;
        if constexpr (kFp8) sk = valid ? sscale[ks * C::kChunk + at] : 0.f;
        tc_fence_after();
        const uint32_t col = tmem_base + lane_off + buf * C::kHeadsN;
        float x0[32], x1[32];
        tmem_ld32_async(col, x0);
        if constexpr (kHeads == 64) tmem_ld32_async(col + 32, x1);
        const float tau = *reinterpret_cast<const volatile float*>(&q.tau);
        tmem_wait_ld(x0);
        if constexpr (kHeads == 64) tmem_wait_ld(x1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_empty[buf]);
          mbar_arrive(&ks_empty[ks]);
        }
        HeadAcc2 acc = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        head_accumulate32_smem(acc, x0, sw);
        if constexpr (kHeads == 64) head_accumulate32_smem(acc, x1, sw + 32);
        float sc = head_total(acc);
        if constexpr (kFp8) sc *= qs * sk;
        if (p.dense && valid) p.dense[r * p.dense_ld + key] = sc;
        n_exact += __popc(__ballot_sync(0xFFFFFFFFu, valid));
        n_cand += append_candidates(q, seg, p.seg_cap, cnt, valid && sc >= tau, sc, key, lane);
        ++ac;
        if (end || (!settled && (nc + 1) % C::kCkptChunks == 0)) {
          if (lane == 0) q.seg[quad] = cnt;
          meet();
          if (ew == 0 && ok)
            refresh_threshold(q, p.cand + r * kSegs * (int64_t)p.seg_cap, p.seg_cap, p.K, lane);
          meet();
        } else if (settled && ew == 0 && (nc + 1) % C::kCkptChunks == 0) {
          const float tn = hist_threshold(q, p.K, lane);
          if (lane == 0 && tn > q.tau) *reinterpret_cast<volatile float*>(&q.tau) = tn;
          __syncwarp();
        }
        if (end) break;
      }
      if (ew == 0 && ok) {
        // another band when a key this pass rejected bounds at or above tau
        const float tau = q.tau;
        const uint32_t mk = p.maxrej[r];
        const bool over = *reinterpret_cast<const volatile int*>(&q.overflow) != 0;
        const bool again = !over && mk != 0u && mk >= ordered_key(tau);
        if (again) {
          const float nxt = p.pass < kRankEst ? p.est[r * kRankEst + p.pass] : -INFINITY;
          state_save(q, p.qstate + r, lane);
          if (lane == 0) {
            p.band_hi[r] = p.band_lo[r];
            p.band_lo[r] = fmaxf(tau, nxt);
            p.maxrej[r] = 0u;
            p.row_next[r] = p.pass + 1;
            *reinterpret_cast<volatile int*>(p.pass_any_next) = 1;
          }
        } else if (lane == 0) {
          publish_query(q, p.out);
          p.row_next[r] = 0;
        }
      }
      meet();
    }
    if (lane == 0) {
      atomicAdd(&p.counters[kCntExact], n_exact);
      atomicAdd(&p.counters[kCntRescored], n_exact);
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

template <bool kFp8>
static cudaError_t launch_rescore_impl(const SeqView& v, const RescoreParams& p,
                                       cudaStream_t stream) {
  using C = RsCfg<kFp8>;
  CUtensorMap qmap;
  if (!encode_q_map(&qmap, v.q, kFp8, (uint64_t)(v.row0 + v.rows), v.H, 1))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(rescore_kernel<kFp8, 64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(rescore_kernel<kFp8, 32>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows8 = p.n_items * kItemQueries;
  const int grid = rows8 < C::kCtasPerSm * sms ? rows8 : C::kCtasPerSm * sms;
  profile_before(DOSA_KERNEL_RESCORE, stream);
  if (v.H == 64)
    rescore_kernel<kFp8, 64><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, p);
  else
    rescore_kernel<kFp8, 32><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_RESCORE, stream);
  return e;
}

cudaError_t launch_rescore(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                           int W, const RankPass& rp, cudaStream_t stream) {
  if (v.rows <= 0) return cudaSuccess;
  RescoreParams p;
  p.k = v.k;
  p.k_scale = v.k_scale;
  p.w = v.w;
  p.q_scale = v.q_scale;
  p.bits = b.bits;
  p.words = b.words;
  p.cand = reinterpret_cast<Cand*>(b.cand);
  p.qstate = reinterpret_cast<QStateG*>(b.qstate);
  p.item_sel = rp.item_sel;
  p.want = rp.want;
  p.pass = rp.pass;
  p.row_next = b.row_next;
  p.band_lo = b.band_lo;
  p.band_hi = b.band_hi;
  p.maxrej = b.maxrej;
  p.est = b.est;
  p.pass_any = b.pass_any + rp.pass;
  p.pass_any_next = b.pass_any + rp.pass + 1;
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
  p.n_items = (int)((v.rows + kItemQueries - 1) / kItemQueries);
  p.W = W;
  p.K = K;
  p.seg_cap = b.seg_cap;
  if (h.cfg.dtype == DOSA_FP8_E4M3) return launch_rescore_impl<true>(v, p, stream);
  return launch_rescore_impl<false>(v, p, stream);
}

}  // namespace dosa
