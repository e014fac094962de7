// Per-query candidate state shared by the certified scorer and the filter
// scorer: the running threshold tau, the candidate lists, and the 256-bin
// score histogram that keeps tau a sound lower bound on the K-th largest exact
// score seen so far ("DOSA: Dots Sparse Attention", Daily Paper Cast
// transcript, Method section: a threshold from the K-th largest exact score of
// a subset of visible keys, refined tile by tile).
//
// tau is -inf during warm-up (fewer than K exact scores).  Once K candidates
// exist, their scores are binned over [min, max]; from then on tau is the
// rounded-down lower edge of the highest bin whose suffix count reaches K.
// Every counted candidate in those bins has a score >= that edge, so at least
// K exact scores are >= tau.
//
// Candidate lists are split into kSegs segments per query, one per TMEM lane
// quadrant: key s of a tile is scored by a warp of quadrant (s mod 128) / 32
// in every kernel, and for a given query exactly one warp of each quadrant
// does so.  That warp is the only writer of its segment and keeps the
// segment's count in a register; counts are published to shared memory at the
// threshold checkpoints, where all epilogue warps meet.
#pragma once

#include <cuda_runtime.h>
#include <math.h>

#include "dosa_device.cuh"

namespace dosa {

constexpr int kBins = 256;
constexpr int kSegs = 4;

// Shared-memory state of one query of a work item.
struct QState {
  float tau;
  int phase;          // 0 = unused slot, 1 = warm-up, 2 = screening/filtering
  int overflow;       // a segment ran out of room
  float lo, inv_w, w;
  int seg[kSegs];     // candidates per segment, as of the last checkpoint
  float omega[4];
  float beta, margin;
  float scale[4];
  float sq;
  long long pos;      // position of the query among the sequence's keys
  long long row;      // chunk-local row
  unsigned hist[kBins];
};

// The part of QState that survives from one kernel to the next (global memory,
// one record per chunk-local query row).
struct QStateG {
  float tau;
  int phase;
  int overflow;
  float lo, inv_w, w;
  int seg[kSegs];
  int pad[2];
  unsigned hist[kBins];
};

struct Cand {
  float score;
  int key;
};

// Bins of width w from lo: sound lower edge of bin i (every score binned at
// >= i is >= the result), and the bin of a score (clamped to [0, kBins)).
__device__ __forceinline__ float bin_edge_at(float lo, float w, int i) {
  const float iw = (float)i * w;
  return fmaf((float)i, w, lo) - (fabsf(lo) + iw) * 0x1p-20f;
}

__device__ __forceinline__ int bin_index(float lo, float inv_w, float score) {
  float b = floorf((score - lo) * inv_w);
  b = fminf(fmaxf(b, 0.f), (float)(kBins - 1));
  return (int)b;
}

__device__ __forceinline__ float bin_edge(const QState& s, int i) { return bin_edge_at(s.lo, s.w, i); }

__device__ __forceinline__ int bin_of(const QState& s, float score) {
  return bin_index(s.lo, s.inv_w, score);
}

// One warp: the highest bin whose suffix count (bins >= it) reaches K, or -1
// when fewer than K are counted.  h points at kBins counts that other warps
// may still be incrementing; any snapshot gives a sound answer because
// counts only grow.
// Counts c[0..7] are bins lane * 8 .. lane * 8 + 7.
__device__ __forceinline__ int suffix_bin_of(const unsigned (&c)[8], int K, int lane) {
  unsigned local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) local += c[j];
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
  const unsigned who = __ballot_sync(0xFFFFFFFFu, best >= 0);
  if (!who) return -1;
  return __shfl_sync(0xFFFFFFFFu, best, __ffs(who) - 1);
}

// This lane's 8 counts of a histogram other warps may still be incrementing.
__device__ __forceinline__ void load_bins(const unsigned* h, int lane, unsigned (&c)[8]) {
  const volatile unsigned* v = h + lane * 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) c[j] = v[j];
}

__device__ __forceinline__ int suffix_bin(const unsigned* h, int K, int lane) {
  unsigned c[8];
  load_bins(h, lane, c);
  return suffix_bin_of(c, K, lane);
}

// Owner warp: highest bin whose suffix count reaches K -> its sound edge
// (or -inf when fewer than K are counted).
__device__ __forceinline__ float hist_threshold(const QState& s, int K, int lane) {
  const int best = suffix_bin(s.hist, K, lane);
  return best < 0 ? -INFINITY : bin_edge(s, best);
}

// Owner warp, after a checkpoint barrier: finish warm-up (bin every candidate
// so far: the segment counts published at this barrier cover only entries
// whose writes are complete, and their writers saw the warm-up phase, so
// none of them is in the histogram yet) or refresh tau from the histogram.
// Segment j of the query's list starts at list + j * seg_cap.
__device__ __forceinline__ void refresh_threshold(QState& q, const Cand* list, int seg_cap, int K,
                                                  int lane) {
  const int phase = q.phase;
  if (phase == 1) {
    int cnt[kSegs], total = 0;
#pragma unroll
    for (int j = 0; j < kSegs; ++j) {
      const int c = q.seg[j];
      cnt[j] = c < seg_cap ? c : seg_cap;
      total += cnt[j];
    }
    if (total < K || *reinterpret_cast<const volatile int*>(&q.overflow)) return;
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kSegs; ++j)
      for (int i = lane; i < cnt[j]; i += 32) {
        const float x = list[j * seg_cap + i].score;
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
#pragma unroll
    for (int j = 0; j < kSegs; ++j)
      for (int i = lane; i < cnt[j]; i += 32)
        atomicAdd(&q.hist[bin_of(q, list[j * seg_cap + i].score)], 1u);
    __syncwarp();
    const float tn = hist_threshold(q, K, lane);
    if (lane == 0) {
      q.tau = fmaxf(q.tau, tn);
      __threadfence_block();
      *reinterpret_cast<volatile int*>(&q.phase) = 2;
    }
  } else if (phase == 2) {
    const float tn = hist_threshold(q, K, lane);
    if (lane == 0 && tn > q.tau) *reinterpret_cast<volatile float*>(&q.tau) = tn;
  }
  __syncwarp();
}

// Append the warp's candidates (lanes with app set) to the warp's segment of
// query q, whose count the warp holds in `cnt`.  Returns the number appended.
// No atomic on the count: the warp is the segment's only writer.
__device__ __forceinline__ unsigned append_candidates(QState& q, Cand* seg, int seg_cap, int& cnt,
                                                      bool app, float sc, int key, int lane) {
  const unsigned am = __ballot_sync(0xFFFFFFFFu, app);
  if (!am) return 0;
  const int slot = cnt + __popc(am & ((1u << lane) - 1u));
  cnt += __popc(am);
  if (app) {
    if (slot < seg_cap) {
      Cand cd;
      cd.score = sc;
      cd.key = key;
      seg[slot] = cd;
      if (*reinterpret_cast<const volatile int*>(&q.phase) == 2)
        atomicAdd(&q.hist[bin_of(q, sc)], 1u);
    } else {
      q.overflow = 1;
    }
  }
  return __popc(am);
}

// Owner warp: copy the carried part of a query's state between shared and
// global memory.
__device__ __forceinline__ void state_save(const QState& q, QStateG* g, int lane) {
  if (lane == 0) {
    g->tau = q.tau;
    g->phase = q.phase;
    g->overflow = q.overflow;
    g->lo = q.lo;
    g->inv_w = q.inv_w;
    g->w = q.w;
#pragma unroll
    for (int j = 0; j < kSegs; ++j) g->seg[j] = q.seg[j];
  }
  for (int b = lane; b < kBins; b += 32) g->hist[b] = q.hist[b];
}

__device__ __forceinline__ void state_load(QState& q, const QStateG* g, int lane) {
  if (lane == 0) {
    q.tau = g->tau;
    q.phase = g->phase;
    q.overflow = g->overflow;
    q.lo = g->lo;
    q.inv_w = g->inv_w;
    q.w = g->w;
#pragma unroll
    for (int j = 0; j < kSegs; ++j) q.seg[j] = g->seg[j];
  }
  for (int b = lane; b < kBins; b += 32) q.hist[b] = g->hist[b];
}

// Owner warp: a fresh state (warm-up) for a valid query slot, or an unused one.
__device__ __forceinline__ void state_fresh(QState& q, bool valid, int lane) {
  if (lane == 0) {
    q.tau = -INFINITY;
    q.phase = valid ? 1 : 0;
    q.overflow = 0;
    q.lo = 0.f;
    q.inv_w = 0.f;
    q.w = 0.f;
#pragma unroll
    for (int j = 0; j < kSegs; ++j) q.seg[j] = 0;
  }
  for (int b = lane; b < kBins; b += 32) q.hist[b] = 0;
}

// Where a finished query's result goes.
struct PublishOut {
  int* cand_count;     // [rows][kSegs]: per-segment counts; all -1 on overflow
  float* tau;          // [rows]: final threshold
  int* repair_list;    // rows whose list overflowed (rescored densely)
  int* repair_count;
  int repair_cap;
  int dense;           // the selection reads a dense score matrix: no repair needed
  int* err;
  unsigned long long* n_repair;   // rows registered for the repair, all chunks
};

// Owner lane 0: publish a finished query (segment counts as of the last
// checkpoint, which every range ends with).
__device__ __forceinline__ void publish_query(const QState& q, const PublishOut& o) {
  const bool over = *reinterpret_cast<const volatile int*>(&q.overflow) != 0;
  int* cc = o.cand_count + q.row * kSegs;
#pragma unroll
  for (int j = 0; j < kSegs; ++j) cc[j] = over ? -1 : q.seg[j];
  o.tau[q.row] = q.tau;
  if (over && !o.dense) {
    atomicAdd(o.n_repair, 1ull);
    const int r = atomicAdd(o.repair_count, 1);
    if (r < o.repair_cap) o.repair_list[r] = (int)q.row;
    else record_error(o.err, kDevBounds);
  }
}

// Integers in [a, b] that also lie in [c, d].
__device__ __forceinline__ long long overlap_count(long long a, long long b, long long c,
                                                  long long d) {
  const long long lo = a > c ? a : c, hi = b < d ? b : d;
  return hi >= lo ? hi - lo + 1 : 0;
}

}  // namespace dosa
