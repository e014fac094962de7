// Key-block certificate ("DOSA: Dots Sparse Attention", Daily Paper Cast
// transcript, future work: extending the certificate from single keys to key
// blocks, which cuts key accesses as well as scoring).
//
// block_prep: every key tile of 128 keys becomes a ball in the real domain:
//   center c = the mean key, radius r >= max_s ||k_s - c||, n >= max_s ||k_s||
//   (rounded up to cover the fp32 arithmetic that formed them).
// block_screen: for each work item (8 query rows) and each step of a range,
//   the per-key certificate UB(s) = sum_j omega_j ReLU(q_j.k) + beta ||k||
//   - sum_g ReLU(u_g.k) is bounded over the whole ball, since v.k lies in
//   [v.c - ||v|| r, v.c + ||v|| r] for every key of it:
//     UB_B = sum_j omega_j ReLU(q_j.c + ||q_j|| r) + (beta + margin) n
//            - sum_g ReLU(u_g.c - ||u_g|| r).
//   A step is dropped when, for every query of the item that sees any of its
//   keys, the tile holds none of the query's seed keys, the query's threshold
//   is active and UB_B (times the query scale) plus a rounding slack is below
//   the threshold carried from the previous launch.  Thresholds only rise, so
//   the decision stays sound for the rest of the scan.  The surviving steps
//   are written in order as the item's step list (its last step is always
//   kept, so no list is empty); the visible pairs of dropped steps are
//   counted as screened, rejected and block-skipped.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "cand_state.cuh"
#include "cert_layout.h"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "work_items.cuh"

namespace dosa {

template <bool kFp8>
__device__ __forceinline__ float blk_code(const void* base, int64_t i) {
  if constexpr (kFp8) {
    __nv_fp8_e4m3 v;
    v.__x = static_cast<const uint8_t*>(base)[i];
    return float(v);
  } else {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
  }
}

// ---- block prep: one CTA of 128 threads per key tile ----------------------------
constexpr int kPrepSmem = kKeyTile * (kHeadDim + 1) * 4;   // the tile's real keys

template <bool kFp8>
__global__ void __launch_bounds__(128) block_prep_kernel(const void* k, const float* k_scale,
                                                         int64_t S, float* blk) {
  constexpr int D = kHeadDim;
  extern __shared__ float prep_dyn[];
  float(*kt)[D + 1] = reinterpret_cast<float(*)[D + 1]>(prep_dyn);
  __shared__ float cen[D];
  __shared__ float red[2][4];
  const int64_t s0 = (int64_t)blockIdx.x * kKeyTile;
  const int n = (int)(S - s0 < kKeyTile ? S - s0 : kKeyTile);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < kKeyTile * D; e += blockDim.x) {
    const int row = e / D, c = e % D;
    float v = 0.f;
    if (row < n) {
      v = blk_code<kFp8>(k, (s0 + row) * D + c);
      if constexpr (kFp8) v *= k_scale[s0 + row];
    }
    kt[row][c] = v;
  }
  __syncthreads();
  {
    const int c = threadIdx.x;          // one dimension per thread
    float sum = 0.f;
    for (int r = 0; r < n; ++r) sum += kt[r][c];
    cen[c] = sum / (float)n;
  }
  __syncthreads();
  float d2 = 0.f, n2 = 0.f;
  if (threadIdx.x < n) {
    const int r = threadIdx.x;          // one key per thread
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float x = kt[r][c], df = x - cen[c];
      d2 = fmaf(df, df, d2);
      n2 = fmaf(x, x, n2);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    d2 = fmaxf(d2, __shfl_xor_sync(0xFFFFFFFFu, d2, o));
    n2 = fmaxf(n2, __shfl_xor_sync(0xFFFFFFFFu, n2, o));
  }
  if (lane == 0) {
    red[0][warp] = d2;
    red[1][warp] = n2;
  }
  __syncthreads();
  float* out = blk + (int64_t)blockIdx.x * kBlkFloats;
  out[threadIdx.x] = cen[threadIdx.x];
  if (threadIdx.x == 0) {
    const float md = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
    const float mn = fmaxf(fmaxf(red[1][0], red[1][1]), fmaxf(red[1][2], red[1][3]));
    const float nmax = sqrtf(mn) * (1.f + 0x1p-14f);
    // the keys themselves were rounded to fp32 (k code x scale): their error
    // is at most 2^-24 of ||k|| per element, covered by the last term
    out[D] = sqrtf(md) * (1.f + 0x1p-14f) + 0x1p-20f * nmax;
    out[D + 1] = nmax;
    out[D + 2] = 0.f;
    out[D + 3] = 0.f;
  }
}

cudaError_t launch_block_prep(const Handle& h, const void* k, const float* k_scale, int64_t S,
                              float* blk, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  const unsigned tiles = (unsigned)((S + kKeyTile - 1) / kKeyTile);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(block_prep_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(block_prep_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  profile_before(DOSA_KERNEL_BLOCK, stream);
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    block_prep_kernel<true><<<tiles, 128, kPrepSmem, stream>>>(k, k_scale, S, blk);
  else
    block_prep_kernel<false><<<tiles, 128, kPrepSmem, stream>>>(k, k_scale, S, blk);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_BLOCK, stream);
  return e;
}

// ---- block screening: one CTA of 256 threads per work item ----------------------
struct BlockParams {
  const void* bdir;          // [chunk rows][kBoundRows][d] codes
  const float* cert;         // [chunk rows][kCertFloats]
  const QStateG* qstate;     // [chunk rows] carried threshold and phase
  const float* q_scale;      // absolute rows (fp8) or null
  const float* blk;          // [tiles][kBlkFloats]
  const int* item_flag;
  int* step_list;            // [items][cap]
  int* step_count;           // [items]
  int cap;
  unsigned long long* counters;
  int64_t row0, rows, pos0, S;
  int n_items, seed_first, seed_last;
  StepRange steps;
};

constexpr int kBlkThreads = 256;
constexpr int kBlkMaxSteps = 8192;   // key tiles of the longest sequence screened (1M keys)

template <bool kFp8>
__global__ void __launch_bounds__(kBlkThreads) block_screen_kernel(const BlockParams p) {
  constexpr int D = kHeadDim, Q = kItemQueries;
  __shared__ float rowsf[Q][kBoundRows][D];      // bound rows of the item's queries (codes)
  __shared__ float rnorm[Q][kBoundRows];
  __shared__ float qc[Q][12];                    // omega[4], beta + margin, scale[4], qs, tau, live
  __shared__ long long qpos[Q];
  __shared__ uint8_t keep[kBlkMaxSteps];
  __shared__ uint32_t scan[32];
  __shared__ unsigned long long s_skip;
  const int item = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
  const Range rg = item_steps(p.steps, p.item_flag, g, item);
  if (rg.end <= rg.begin) {
    if (threadIdx.x == 0) p.step_count[item] = 0;
    return;
  }
  const int n = rg.end - rg.begin;
  // queries: bound rows as floats, their norms, certificate constants
  for (int e = threadIdx.x; e < Q * kBoundRows * D; e += blockDim.x) {
    const int ql = e / (kBoundRows * D), rem = e % (kBoundRows * D);
    const int64_t row = g.local0 + (ql < g.nq ? ql : 0);
    rowsf[ql][rem / D][rem % D] = blk_code<kFp8>(p.bdir, row * kBoundRows * D + rem);
  }
  if (threadIdx.x == 0) s_skip = 0ull;
  __syncthreads();
  for (int t = warp; t < Q * kBoundRows; t += kBlkThreads / 32) {
    const int ql = t / kBoundRows, j = t % kBoundRows;
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) ss = fmaf(rowsf[ql][j][c], rowsf[ql][j][c], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) rnorm[ql][j] = sqrtf(ss) * (1.f + 0x1p-14f);
  }
  if (threadIdx.x < Q) {
    const int ql = threadIdx.x;
    const bool valid = ql < g.nq;
    const int64_t row = g.local0 + (valid ? ql : 0);
    const float* cf = p.cert + row * kCertFloats;
    const QStateG& st = p.qstate[row];
    for (int j = 0; j < 4; ++j) qc[ql][j] = cf[kCertOmega + j];
    qc[ql][4] = cf[kCertBeta] + cf[kCertMargin];
    for (int j = 0; j < 4; ++j) qc[ql][5 + j] = cf[kCertScale + j];
    qc[ql][9] = kFp8 ? p.q_scale[g.t0 + (valid ? ql : 0)] : 1.f;
    qc[ql][10] = st.tau;
    qc[ql][11] = (valid && st.phase == 2) ? 1.f : 0.f;
    qpos[ql] = valid ? g.pos_first + ql : -1;
  }
  __syncthreads();
  // one warp per step; lanes split the 128 dimensions (4 each)
  unsigned long long skipped = 0;
  for (int i = warp; i < n; i += kBlkThreads / 32) {
    const int ti = rg.begin + i;
    const int j = tile_at(ti, g.n_tiles);
    const int64_t lo = (int64_t)j * kKeyTile;
    const int64_t hi = (lo + kKeyTile - 1 < p.S - 1) ? lo + kKeyTile - 1 : p.S - 1;
    const float* b = p.blk + (int64_t)j * kBlkFloats;
    float cv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) cv[e] = b[lane * 4 + e];
    const float rad = b[D], nmax = b[D + 1];
    float cn = 0.f;                                   // ||c||
#pragma unroll
    for (int e = 0; e < 4; ++e) cn = fmaf(cv[e], cv[e], cn);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cn += __shfl_xor_sync(0xFFFFFFFFu, cn, o);
    cn = sqrtf(cn) * (1.f + 0x1p-14f);
    bool drop = i + 1 < n;                            // the range's last step is kept
    long long vis_pairs = 0;
    for (int ql = 0; ql < Q && drop; ++ql) {
      const long long pos = qpos[ql];
      if (pos < 0 || lo > pos) continue;              // nothing of the tile is visible
      const bool seeds = lo < p.seed_first || hi > pos - p.seed_last;
      if (seeds || qc[ql][11] == 0.f) {
        drop = false;
        break;
      }
      // rows . c: 4 retained heads, u_1 hi/lo, u_2 hi/lo
      float dot[kBoundRows];
#pragma unroll
      for (int r = 0; r < kBoundRows; ++r) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) a = fmaf(rowsf[ql][r][lane * 4 + e], cv[e], a);
        dot[r] = a;
      }
#pragma unroll
      for (int r = 0; r < kBoundRows; ++r)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot[r] += __shfl_xor_sync(0xFFFFFFFFu, dot[r], o);
      float ub = 0.f, mag = 0.f;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        ub = fmaf(qc[ql][r], fmaxf(fmaf(rnorm[ql][r], rad, dot[r]), 0.f), ub);
        mag = fmaf(qc[ql][r], rnorm[ql][r] * (cn + rad), mag);
      }
      ub = fmaf(qc[ql][4], nmax, ub);
      mag = fmaf(qc[ql][4], nmax, mag);
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const float sa = qc[ql][5 + 2 * gi], sb = qc[ql][6 + 2 * gi];
        const float uc = fmaf(sa, dot[4 + 2 * gi], sb * dot[5 + 2 * gi]);
        const float un = fabsf(sa) * rnorm[ql][4 + 2 * gi] + fabsf(sb) * rnorm[ql][5 + 2 * gi];
        ub -= fmaxf(uc - un * rad, 0.f);
        mag = fmaf(un, cn + rad, mag);
      }
      const float bound = (ub + 0x1p-14f * mag) * qc[ql][9];
      if (!(bound < qc[ql][10])) {
        drop = false;
        break;
      }
      vis_pairs += (hi < pos ? hi : pos) - lo + 1;
    }
    if (lane == 0) keep[i] = drop ? 0 : 1;
    if (drop) skipped += (unsigned long long)vis_pairs;
  }
  if (lane == 0 && skipped) atomicAdd(&s_skip, skipped);
  __syncthreads();
  // the kept steps in order: a contiguous run of steps per thread
  const int per = (n + kBlkThreads - 1) / kBlkThreads;
  const int i0 = threadIdx.x * per, i1 = i0 + per < n ? i0 + per : n;
  uint32_t c = 0;
  for (int i = i0; i < i1; ++i) c += keep[i];
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = lane < kBlkThreads / 32 ? scan[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, ti, o);
      if (lane >= o) ti += v;
    }
    if (lane < kBlkThreads / 32) scan[lane] = ti - t;
  }
  __syncthreads();
  uint32_t at = scan[warp] + incl - c;
  int* list = p.step_list + (int64_t)item * p.cap;
  for (int i = i0; i < i1; ++i)
    if (keep[i]) list[at++] = rg.begin + i;
  if (threadIdx.x == kBlkThreads - 1) p.step_count[item] = (int)at;
  if (threadIdx.x == 0 && s_skip) {
    atomicAdd(&p.counters[kCntScreened], s_skip);
    atomicAdd(&p.counters[kCntRejected], s_skip);
    atomicAdd(&p.counters[kCntBlockSkipped], s_skip);
  }
}

cudaError_t launch_block_screen(const Handle& h, const SeqView& v, const CertBuffers& b,
                                StepRange steps, cudaStream_t stream) {
  if (v.rows <= 0) return cudaSuccess;
  const int64_t n_tiles = (v.pos0 + v.rows - 1) / kKeyTile + 1;
  if (n_tiles > kBlkMaxSteps || n_tiles > b.step_cap) return cudaErrorInvalidValue;
  BlockParams p;
  p.bdir = b.bdir;
  p.cert = b.cert;
  p.qstate = reinterpret_cast<const QStateG*>(b.qstate);
  p.q_scale = v.q_scale;
  p.blk = b.blk;
  p.item_flag = b.item_flag;
  p.step_list = b.step_list;
  p.step_count = b.step_count;
  p.cap = b.step_cap;
  p.counters = b.counters;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.n_items = (int)((v.rows + kItemQueries - 1) / kItemQueries);
  p.seed_first = h.cfg.seed_first;
  p.seed_last = h.cfg.seed_last;
  p.steps = steps;
  profile_before(DOSA_KERNEL_BLOCK, stream);
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    block_screen_kernel<true><<<(unsigned)p.n_items, kBlkThreads, 0, stream>>>(p);
  else
    block_screen_kernel<false><<<(unsigned)p.n_items, kBlkThreads, 0, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_BLOCK, stream);
  return e;
}

}  // namespace dosa
