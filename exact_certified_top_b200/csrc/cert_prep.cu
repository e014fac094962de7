// Certificate preparation for the certified indexer ("DOSA: Dots Sparse
// Attention", Daily Paper Cast transcript, Method section: the certificate's
// three stages; "arXiv Releases DoSA ...", Technical Mechanism Analysis,
// point 2: nonnegative head projections and joint residual bounds limit the
// positive contributions, activation-informed aggregation bounds what the
// negative heads subtract).
//
// key_prep: per key ||k|| (code domain, rounded up) and the per-sequence key
//   sum (real domain) whose mean decides which negative heads are active.
// cert_setup: per query, in the code domain (the fp8 per-token scales are
//   positive and factor out of every ReLU):
//   R   = the r positive heads with the largest w_h ||q_h|| (ties: smaller h)
//   a_h = NNLS projection of each omitted positive head onto the heads in R,
//         exact by trying every support (r <= 4), solved in fp64
//   rho_h = q_h - sum_j a_hj q_j,  omega_j = w_j + sum_h w_h a_hj
//   beta  = min( sum_h w_h ||rho_h|| , sqrt(W_O * lambda) )  where lambda is a
//           Collatz-Wielandt upper bound on the spectral radius of
//           |[sqrt(w_h w_h') rho_h . rho_h']| (>= lambda_max of the weighted
//           residual Gram matrix), plus the slack terms below
//   u_g   = sum_{h in A_g} |w_h| q_h over A_1 = {negative h : q_h . k_mean > 0}
//           and A_2 = the other negative heads; each u_g is stored as two rows
//           in the MMA input type (hi + lo, each with an fp32 scale) and the
//           split error ||u_g - s_hi u_hi - s_lo u_lo|| is added to beta.
//   Slack: every fp32 rounding of the quantities above is covered by adding
//   2^-16 * sum_h |w_h| ||q_h|| to beta (each individual error is at most
//   2^-18 of that scale).  The candidate margin is
//   c = 2^margin_log2 * sum_h |w_h| ||q_h||, rounded up.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "cert_layout.h"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "work_items.cuh"

namespace dosa {

template <bool kFp8>
__device__ __forceinline__ float decode_code(const void* base, int64_t i) {
  if constexpr (kFp8) {
    __nv_fp8_e4m3 v;
    v.__x = static_cast<const uint8_t*>(base)[i];
    return float(v);
  } else {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
  }
}

// ---- key prep --------------------------------------------------------------------
// One warp per key: ||k_code|| rounded up; real-domain key sum into key_sum[d]
// (block-level partial sums, then one atomicAdd per element per block).
template <bool kFp8>
__global__ void __launch_bounds__(256) key_prep_kernel(const void* k, const float* k_scale,
                                                       int64_t S, float* key_norm,
                                                       float* key_sum) {
  __shared__ float part[8][kHeadDim];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t s = (int64_t)blockIdx.x * 8 + warp; s < S; s += (int64_t)gridDim.x * 8) {
    float v[4], ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[e] = decode_code<kFp8>(k, s * kHeadDim + lane * 4 + e);
      ss = fmaf(v[e], v[e], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    const float sc = kFp8 ? k_scale[s] : 1.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = fmaf(v[e], sc, acc[e]);
    if (lane == 0) key_norm[s] = sqrtf(ss) * (1.f + 0x1p-20f);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) part[warp][lane * 4 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += part[w][threadIdx.x];
    atomicAdd(&key_sum[threadIdx.x], t);
  }
}

// ---- certificate setup ------------------------------------------------------------
// One CTA of 256 threads per query.  Every phase spreads its work over all
// warps: dot products are split 8 ways (fp64 partial sums for the NNLS
// inputs), the NNLS tries its supports on 16 lanes per omitted head at once,
// and the power iteration runs in warp 0 while warps 4-7 aggregate the
// negative heads.
constexpr int kSetupThreads = 256;
constexpr int kQPad = kHeadDim + 1;
constexpr int kSetupSmem = (64 * kQPad + 64 * 65) * 4;
constexpr int kPowerIters = 12;

// Least squares on the support `mask` (bits over the 4 retained slots) of
// G a = b, in fp64: inactive slots get an identity row and column and a zero
// right-hand side, so their coefficient is exactly 0 and the active block is
// solved as if alone (Cholesky, one reciprocal per pivot).  False when a pivot
// shows the support (numerically) rank deficient.
__device__ __forceinline__ bool ls_support(const double (&G)[4][4], const double (&b)[4],
                                           int mask, double (&a)[4]) {
  double M[4][4], rhs[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool ai = (mask >> i) & 1;
    rhs[i] = ai ? b[i] : 0.0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool aj = (mask >> j) & 1;
      M[i][j] = (ai && aj) ? G[i][j] : (i == j ? 1.0 : 0.0);
    }
  }
  double L[4][4], inv[4];
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j <= i; ++j) {
      double v = M[i][j];
#pragma unroll
      for (int k = 0; k < j; ++k) v -= L[i][k] * L[j][k];
      if (i == j) {
        ok = ok && (v > 1e-12 * (M[i][i] + 1e-300));
        const double d = sqrt(v > 0.0 ? v : 1.0);
        L[i][i] = d;
        inv[i] = 1.0 / d;
      } else {
        L[i][j] = v * inv[j];
      }
    }
  }
  double y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    double v = rhs[i];
#pragma unroll
    for (int k = 0; k < i; ++k) v -= L[i][k] * y[k];
    y[i] = v * inv[i];
  }
#pragma unroll
  for (int i = 3; i >= 0; --i) {
    double v = y[i];
#pragma unroll
    for (int k = i + 1; k < 4; ++k) v -= L[k][i] * a[k];
    a[i] = v * inv[i];
  }
  return ok;
}

template <bool kFp8>
__device__ __forceinline__ void store_code(void* base, int64_t i, float x) {
  if constexpr (kFp8) {
    static_cast<uint8_t*>(base)[i] =
        (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
  } else {
    static_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
  }
}

template <bool kFp8>
__device__ __forceinline__ float roundtrip(float x) {
  if constexpr (kFp8) {
    __nv_fp8_e4m3 v;
    v.__x = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
    return float(v);
  } else {
    return __bfloat162float(__float2bfloat16_rn(x));
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Decode 16 consecutive input codes starting at element e into dst[0..15].
template <bool kFp8>
__device__ __forceinline__ void decode16(const void* q, int64_t e, float* dst) {
  if constexpr (kFp8) {
    const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(q) + e);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      __nv_fp8_e4m3 c;
      c.__x = (uint8_t)(w[i >> 2] >> (8 * (i & 3)));
      dst[i] = float(c);
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(q) + e);
    const uint4 v0 = p[0], v1 = p[1];
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t bits = (i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16);
      dst[i] = __uint_as_float(bits);
    }
  }
}

struct SetupParams {
  const void* q;          // [rows, nh, d] codes (absolute rows)
  const float* w;         // [rows, nh]
  int nh;                 // heads per row: 32 or 64 (slots nh..63 are zero heads)
  const float* key_sum;   // [d] real-domain key sum of the sequence
  float inv_nkeys;        // 1 / number of keys of the sequence
  int64_t row0;           // first row of the chunk
  int64_t rows;
  int r, G, margin_log2;
  void* bdir;             // [rows, 8, d] codes (chunk-local rows)
  float* cert;            // [rows, kCertFloats]
  int32_t* retained;      // [rows, 4]
  int sample;             // which rows (see launch_cert_setup)
  int stride;             // every stride-th item is sampled (probe_stride)
  int n_items;
  int* item_flag;
  const int* gate;
};

// upper-triangle pairs of the 4 retained slots
__constant__ int8_t kPairA[10] = {0, 0, 0, 0, 1, 1, 1, 2, 2, 3};
__constant__ int8_t kPairB[10] = {0, 1, 2, 3, 1, 2, 3, 2, 3, 3};

template <bool kFp8>
__global__ void __launch_bounds__(kSetupThreads) cert_setup_kernel(const SetupParams p) {
  constexpr int H = 64, D = kHeadDim;   // head slots; p.nh of them are real
  extern __shared__ float setup_dyn[];
  // code-domain heads, then residuals in place (padded rows); weighted residual Gram
  float(*qs)[kQPad] = reinterpret_cast<float(*)[kQPad]>(setup_dyn);
  float(*gt)[65] = reinterpret_cast<float(*)[65]>(setup_dyn + H * kQPad);
  // The NNLS inputs and coefficients live in the Gram's space: they are dead
  // (omega already written) before the Gram is computed.
  double(*Bm)[4] = reinterpret_cast<double(*)[4]>(setup_dyn + H * kQPad);
  double* QQ = reinterpret_cast<double*>(Bm + H);
  double(*alpha_s)[4] = reinterpret_cast<double(*)[4]>(QQ + H);
  static_assert(H * 4 * 8 * 2 + H * 8 <= H * 65 * 4, "NNLS arrays fit in the Gram's space");
  __shared__ float wv[H], qn[H], act[H], rn[H];
  __shared__ float kbar[D];
  __shared__ float vec[64];
  __shared__ double Gr[4][4];
  __shared__ int R[4], O[64], A1[64], A2[64];
  __shared__ int nR, nO, nA1, nA2;
  __shared__ float red[8];
  __shared__ float uv[2][D], rv[2][D];
  __shared__ float s_lam;
  int64_t i = blockIdx.x;
  if (p.sample == 1) {
    // the rows of sampled item stride * (blockIdx.x / 8); items run longest
    // rows first, so item j holds the rows of group n_items-1-j
    const int item = p.stride * (int)(blockIdx.x / kItemQueries);
    i = (int64_t)(p.n_items - 1 - item) * kItemQueries + blockIdx.x % kItemQueries;
    if (i >= p.rows) return;
    if (threadIdx.x == 0 && blockIdx.x % kItemQueries == 0) p.item_flag[item] = kItemSample;
  } else if (p.sample == 2) {
    const int item = p.n_items - 1 - (int)(i / kItemQueries);
    if (item % p.stride == 0 || *reinterpret_cast<const volatile int*>(p.gate) == 0)
      return;
  }
  const int64_t t = p.row0 + i;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- A: decode q (16 codes per load), weights, mean key.  Slots past the
  // row's heads hold zero heads with zero weight: neither positive nor
  // negative, they join no list and add nothing. ----
  for (int e = threadIdx.x * 16; e < H * D; e += blockDim.x * 16) {
    float v[16];
    const int h = e / D, c = e % D;
    if (h < p.nh) {
      decode16<kFp8>(p.q, t * p.nh * D + e, v);
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) qs[h][c + k] = v[k];
  }
  if (threadIdx.x < H) wv[threadIdx.x] = threadIdx.x < p.nh ? p.w[t * p.nh + threadIdx.x] : 0.f;
  if (threadIdx.x < D) kbar[threadIdx.x] = p.key_sum[threadIdx.x] * p.inv_nkeys;
  __syncthreads();
  // ---- B: ||q_h|| and q_h . k_mean, 4 threads per head ----
  {
    const int h = threadIdx.x >> 2, part = threadIdx.x & 3;
    float ss = 0.f, ka = 0.f;
#pragma unroll 8
    for (int k = 0; k < D / 4; ++k) {
      const int c = part + 4 * k;
      const float x = qs[h][c];
      ss = fmaf(x, x, ss);
      ka = fmaf(x, kbar[c], ka);
    }
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 1);
    ka += __shfl_xor_sync(0xFFFFFFFFu, ka, 1);
    ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 2);
    ka += __shfl_xor_sync(0xFFFFFFFFu, ka, 2);
    if (part == 0) {
      qn[h] = sqrtf(ss);
      act[h] = ka;
    }
  }
  __syncthreads();
  // ---- C: retained heads and head lists (warp 0) ----
  if (warp == 0) {
    // the r positive heads with the largest w_h ||q_h||, ties to the smaller
    // head; lane l holds heads l and l + 32
    const int ha = lane, hb = lane + 32;
    bool ta = false, tb = false;
    for (int k = 0; k < p.r; ++k) {
      const float va = (wv[ha] > 0.f && !ta) ? wv[ha] * qn[ha] : -1.f;
      const float vb = (wv[hb] > 0.f && !tb) ? wv[hb] * qn[hb] : -1.f;
      float bv = va >= vb ? va : vb;                 // prefer the smaller head on a tie
      int bh = va >= vb ? ha : hb;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
        const int oh = __shfl_xor_sync(0xFFFFFFFFu, bh, o);
        if (ov > bv || (ov == bv && oh < bh)) {
          bv = ov;
          bh = oh;
        }
      }
      if (bv < 0.f) break;                           // no positive head left
      ta |= bh == ha;
      tb |= bh == hb;
    }
    // lists in ascending head order via ballots (heads 0..31 then 32..63)
    const bool pa = wv[ha] > 0.f, pb = wv[hb] > 0.f, na = wv[ha] < 0.f, nb = wv[hb] < 0.f;
    const unsigned below = (1u << lane) - 1u;
    auto compact = [&](bool ca, bool cb, int* list, int* count) {
      const unsigned ma = __ballot_sync(0xFFFFFFFFu, ca), mb = __ballot_sync(0xFFFFFFFFu, cb);
      if (ca) list[__popc(ma & below)] = ha;
      if (cb) list[__popc(ma) + __popc(mb & below)] = hb;
      if (lane == 0) *count = __popc(ma) + __popc(mb);
    };
    compact(ta, tb, R, &nR);
    compact(pa && !ta, pb && !tb, O, &nO);
    compact(na && p.G >= 1 && act[ha] > 0.f, nb && p.G >= 1 && act[hb] > 0.f, A1, &nA1);
    compact(na && p.G >= 2 && !(act[ha] > 0.f), nb && p.G >= 2 && !(act[hb] > 0.f), A2, &nA2);
  }
  __syncthreads();
  const int r = nR, no = nO;
  // ---- D: NNLS inputs in fp64 (exact products of fp32 values): q_h . q_Rj
  // and ||q_h||^2 for every omitted head, and the retained heads' Gram.
  // Eight threads per dot product. ----
  {
    const int nd = no * 5 + 10;
    const int part = threadIdx.x & 7;
    for (int base = 0; base < nd; base += kSetupThreads / 8) {
      const int task = base + (threadIdx.x >> 3);
      int ha = -1, hb = -1;
      if (task < no * 5) {
        const int k = task / 5, j = task % 5;
        ha = O[k];
        hb = j == 4 ? ha : (j < r ? R[j] : -1);
      } else if (task < nd) {
        const int a = kPairA[task - no * 5], b = kPairB[task - no * 5];
        if (a < r && b < r) {
          ha = R[a];
          hb = R[b];
        }
      }
      double v = 0.0;
      if (ha >= 0 && hb >= 0) {
#pragma unroll
        for (int k = 0; k < D / 8; ++k) {
          const int c = part + 8 * k;
          v = fma((double)qs[ha][c], (double)qs[hb][c], v);
        }
      }
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
      if (part == 0 && task < nd) {
        if (task < no * 5) {
          const int k = task / 5, j = task % 5;
          if (j == 4) QQ[k] = v;
          else Bm[k][j] = v;
        } else {
          const int a = kPairA[task - no * 5], b = kPairB[task - no * 5];
          Gr[a][b] = v;
          Gr[b][a] = v;
        }
      }
    }
  }
  __syncthreads();
  // ---- E: NNLS for every omitted head, one support per lane (16 lanes per
  // head: support masks 0..15 over the retained slots), best feasible
  // support by a half-warp reduction.  The empty support (alpha = 0) is
  // always feasible with residual ||q_h||^2. ----
  {
    const int m = lane & 15;
    double G[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) G[a][b] = Gr[a][b];
    for (int base = 0; base < no; base += kSetupThreads / 16) {
      const int k = base + (threadIdx.x >> 4);
      double res = INFINITY, a[4] = {0.0, 0.0, 0.0, 0.0};
      if (k < no && (m >> r) == 0) {
        const double qq = QQ[k];
        if (m == 0) {
          res = qq;
        } else {
          double b[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) b[j] = Bm[k][j];
          bool ok = ls_support(G, b, m, a);
          double ab = 0.0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if ((m >> j) & 1) ok = ok && a[j] > 0.0;
            ab += a[j] * b[j];
          }
          if (ok) res = qq - ab;   // residual^2 at the least-squares point
        }
      }
      // min residual over the 16 lanes, ties to the smaller mask
      double best = res;
      int who = m;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int ow = __shfl_xor_sync(0xFFFFFFFFu, who, o);
        if (ob < best || (ob == best && ow < who)) {
          best = ob;
          who = ow;
        }
      }
      if (k < no && who == m) {
        const int h = O[k];
#pragma unroll
        for (int j = 0; j < 4; ++j) alpha_s[h][j] = m == 0 ? 0.0 : a[j];
      }
    }
  }
  __syncthreads();
  float* cf = p.cert + i * kCertFloats;
  if (warp == 1 && lane < 4) {
    // omega_j = w_j + sum_h w_h alpha_hj (fp64)
    const int j = lane;
    float om = 0.f;
    if (j < r) {
      double o = wv[R[j]];
      for (int k = 0; k < no; ++k) o += (double)wv[O[k]] * alpha_s[O[k]][j];
      om = (float)o;
    }
    cf[kCertOmega + j] = om;
    p.retained[i * 4 + j] = j < r ? R[j] : -1;
  }
  // ---- F: residuals in place of the omitted heads.  Thread c of each half
  // of the CTA owns column c of every other omitted head; the retained heads'
  // values of that column stay in registers (the coefficients are read before
  // the barrier that precedes the Gram, which reuses their space). ----
  {
    const int c = threadIdx.x & (D - 1);
    float qr[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) qr[j] = j < r ? qs[R[j]][c] : 0.f;
    for (int k = threadIdx.x >> 7; k < no; k += kSetupThreads / D) {
      const int h = O[k];
      float x = qs[h][c];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j < r) x = fmaf(-(float)alpha_s[h][j], qr[j], x);
      qs[h][c] = x;
    }
  }
  __syncthreads();
  // ---- G: weighted residual Gram |[sqrt(w w') rho . rho']| and ||rho_h||:
  // 4 x 4 blocks of the lower triangle, 8 threads per block (16 columns each)
  // ----
  {
    const int nb = (no + 3) / 4, nblk = nb * (nb + 1) / 2;
    const int part = threadIdx.x & 7;
    for (int base = 0; base < nblk; base += kSetupThreads / 8) {
      const int task = base + (threadIdx.x >> 3);
      int A = 0;
      while ((A + 1) * (A + 2) / 2 <= task) ++A;
      const int Bb = task - A * (A + 1) / 2;       // block (A, Bb), Bb <= A
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      if (task < nblk) {
        int ha[4], hb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ha[i] = O[min(4 * A + i, no - 1)];
          hb[i] = O[min(4 * Bb + i, no - 1)];
        }
#pragma unroll 4
        for (int k = 0; k < D / 8; ++k) {
          const int c = part + 8 * k;
          float xa[4], xb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            xa[i] = qs[ha[i]][c];
            xb[i] = qs[hb[i]][c];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], xb[j], acc[i][j]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v = acc[i][j];
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
          acc[i][j] = v;
        }
      if (part == 0 && task < nblk) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int ra = 4 * A + i, cb = 4 * Bb + j;
            if (ra < no && cb < no && cb <= ra) {
              const int h1 = O[ra], h2 = O[cb];
              // sqrt(w) sqrt(w'), not sqrt(w w'): the product of two small
              // weights can underflow fp32 where each root does not
              const float g = fabsf(sqrtf(wv[h1]) * sqrtf(wv[h2]) * acc[i][j]);
              gt[ra][cb] = g;
              gt[cb][ra] = g;
              if (ra == cb) rn[h1] = sqrtf(acc[i][j]);
            }
          }
      }
    }
  }
  __syncthreads();
  // ---- H: power iterations on |Gram| from the all-ones vector, then the
  // Collatz-Wielandt bound max_a (|Gram| v)_a / v_a.  Four threads per row
  // (columns q * 16 + k), block-wide maximum through shared memory. ----
  {
    const int a = threadIdx.x >> 2, q = threadIdx.x & 3;
    const bool row = a < no;
    if (threadIdx.x < 64) vec[threadIdx.x] = 1.f;
    __syncthreads();
    float sa = 0.f, lam = 0.f;
    for (int it = 0; it <= kPowerIters; ++it) {
      float p0 = 0.f, p1 = 0.f;
      if (row) {
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const int b0 = q * 16 + k, b1 = b0 + 1;
          if (b0 < no) p0 = fmaf(gt[a][b0], vec[b0], p0);
          if (b1 < no) p1 = fmaf(gt[a][b1], vec[b1], p1);
        }
      }
      sa = p0 + p1;
      sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 1);
      sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 2);
      if (it == kPowerIters) break;
      const float m = warp_max(row ? sa : 0.f);
      if (lane == 0) red[warp] = m;
      __syncthreads();
      const float mm = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])),
                             fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
      if (row && q == 0) vec[a] = mm > 0.f ? sa / mm : 1.f;
      __syncthreads();
    }
    // Collatz-Wielandt needs v_a > 0; an entry that underflowed makes the
    // joint bound unusable (beta falls back to the per-head sum)
    lam = row ? (vec[a] > 0x1p-100f ? sa / vec[a] : INFINITY) : 0.f;
    lam = warp_max(lam);
    __syncthreads();
    if (lane == 0) red[warp] = lam;
    __syncthreads();
    if (threadIdx.x == 0)
      s_lam = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])),
                    fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
  }
  // ---- I: negative aggregates, thread c < 128 owns element c of u_1, thread
  // 128 + c element c of u_2 ----
  {
    const int c = threadIdx.x & (D - 1);
    const int* list = threadIdx.x < D ? A1 : A2;
    const int cnt = threadIdx.x < D ? nA1 : nA2;
    float u = 0.f;
    for (int k = 0; k < cnt; ++k) {
      const int h = list[k];
      u = fmaf(fabsf(wv[h]), qs[h][c], u);
    }
    uv[threadIdx.x < D ? 0 : 1][c] = u;
  }
  __syncthreads();
  // ---- J: each aggregate as a hi row and a lo row in the input type, with
  // fp32 scales; the split error is added to beta ----
  float beta_add = 0.f;   // (thread 0)
  const size_t esz = kFp8 ? 1 : 2;
  uint8_t* rows_out = static_cast<uint8_t*>(p.bdir) + (size_t)i * 8 * D * esz;
  float s_hi[2], s_lo[2];
  for (int g = 0; g < 2; ++g) {
    // hi part: scale then round; lo part: the remainder, scaled and rounded
    float m = threadIdx.x < D ? fabsf(uv[g][threadIdx.x]) : 0.f;
    m = warp_max(m);
    if (lane == 0 && warp < 4) red[warp] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    s_hi[g] = kFp8 ? (m > 0.f ? m / 448.f : 0.f) : 1.f;
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      const float x = s_hi[g] > 0.f ? uv[g][c] / s_hi[g] : 0.f;
      store_code<kFp8>(rows_out, (4 + 2 * g) * D + c, x);
      rv[g][c] = uv[g][c] - s_hi[g] * roundtrip<kFp8>(x);
    }
    __syncthreads();
    float m2 = threadIdx.x < D ? fabsf(rv[g][threadIdx.x]) : 0.f;
    m2 = warp_max(m2);
    if (lane == 0 && warp < 4) red[4 + warp] = m2;
    __syncthreads();
    m2 = fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]));
    s_lo[g] = kFp8 ? (m2 > 0.f ? m2 / 448.f : 0.f) : 1.f;
    float e2 = 0.f;
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      const float x = s_lo[g] > 0.f ? rv[g][c] / s_lo[g] : 0.f;
      store_code<kFp8>(rows_out, (5 + 2 * g) * D + c, x);
      const float err = rv[g][c] - s_lo[g] * roundtrip<kFp8>(x);
      e2 = err * err;
    }
    e2 = warp_sum(e2);
    __syncthreads();
    if (lane == 0 && warp < 4) red[warp] = e2;
    __syncthreads();
    if (threadIdx.x == 0) beta_add += sqrtf(red[0] + red[1] + red[2] + red[3]) * (1.f + 0x1p-10f);
    __syncthreads();
  }
  // bound rows 0..3: the retained heads' own codes
  const uint8_t* qrow = static_cast<const uint8_t*>(p.q) + (size_t)t * p.nh * D * esz;
  for (int e = threadIdx.x; e < 4 * D * (int)esz; e += blockDim.x) {
    const int j = e / (D * esz), b = e % (D * esz);
    rows_out[e] = j < r ? qrow[(size_t)R[j] * D * esz + b] : 0;
  }
  if (warp == 0) {
    float wO = 0.f, bsum = 0.f, z2 = 0.f, scale = 0.f;
    for (int k = lane; k < no; k += 32) {
      const int h = O[k];
      wO += wv[h];
      bsum = fmaf(wv[h], rn[h], bsum);
      z2 = fmaf(wv[h], rn[h] * rn[h], z2);
    }
    for (int h = lane; h < H; h += 32) scale = fmaf(fabsf(wv[h]), qn[h], scale);
    wO = warp_sum(wO);
    bsum = warp_sum(bsum);
    z2 = warp_sum(z2);
    scale = warp_sum(scale);
    if (lane == 0) {
      // lambda bound: CW value with rounding headroom plus the Gram entry errors
      const float lam_b = s_lam * (1.f + 0x1p-16f) + 0x1p-16f * z2;
      const float bjoint = sqrtf(wO) * sqrtf(lam_b) * (1.f + 0x1p-20f);
      const float bs = bsum * (1.f + 0x1p-20f);
      float beta = no > 0 ? fminf(bs, bjoint) : 0.f;
      beta += 0x1p-16f * scale + beta_add;
      cf[kCertBeta] = beta;
      cf[kCertMargin] = ldexpf(scale, p.margin_log2) * (1.f + 0x1p-20f);
      cf[kCertScale + 0] = s_hi[0];
      cf[kCertScale + 1] = s_lo[0];
      cf[kCertScale + 2] = s_hi[1];
      cf[kCertScale + 3] = s_lo[1];
      cf[kCertBetaSum] = bs;
      cf[kCertBetaJoint] = bjoint;
      cf[kCertNA1] = (float)nA1;
      cf[kCertNA2] = (float)nA2;
      cf[kCertNO] = (float)no;
    }
  }
}

cudaError_t launch_key_prep(const Handle& h, const void* k, const float* k_scale, int64_t S,
                            float* key_norm, float* key_sum, cudaStream_t stream) {
  if (S <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(key_sum, 0, kHeadDim * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  int blocks = (int)((S + 7) / 8);
  if (blocks > 4096) blocks = 4096;
  profile_before(DOSA_KERNEL_KEY_PREP, stream);
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    key_prep_kernel<true><<<blocks, 256, 0, stream>>>(k, k_scale, S, key_norm, key_sum);
  else
    key_prep_kernel<false><<<blocks, 256, 0, stream>>>(k, k_scale, S, key_norm, key_sum);
  e = cudaGetLastError();
  profile_after(DOSA_KERNEL_KEY_PREP, stream);
  return e;
}

__global__ void probe_resolve_kernel(int* item_flag, int n_items, const int* gate) {
  const bool probe = *gate != 0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_items; i += gridDim.x * blockDim.x)
    if (item_flag[i] == 0) item_flag[i] = probe ? kItemProbe : kItemUnprobed;
}

cudaError_t launch_probe_resolve(int* item_flag, int n_items, const int* gate,
                                 cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  const int grid = (n_items + 255) / 256 < 1024 ? (n_items + 255) / 256 : 1024;
  profile_before(DOSA_KERNEL_CERT_SETUP, stream);
  probe_resolve_kernel<<<grid, 256, 0, stream>>>(item_flag, n_items, gate);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_CERT_SETUP, stream);
  return e;
}

cudaError_t launch_cert_setup(const Handle& h, const SeqView& v, const float* key_sum,
                              void* bdir, float* cert, int32_t* retained, cudaStream_t stream,
                              int sample, int* item_flag, const int* gate) {
  if (v.rows <= 0) return cudaSuccess;
  SetupParams p;
  p.q = v.q;
  p.w = v.w;
  p.nh = v.H;
  p.key_sum = key_sum;
  p.inv_nkeys = 1.f / (float)v.S;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.r = h.cfg.r;
  p.G = h.cfg.G;
  p.margin_log2 = h.cfg.margin_log2;
  p.bdir = bdir;
  p.cert = cert;
  p.retained = retained;
  p.sample = sample;
  p.n_items = (int)((v.rows + kItemQueries - 1) / kItemQueries);
  p.stride = probe_stride(p.n_items);
  p.item_flag = item_flag;
  p.gate = gate;
  unsigned grid = (unsigned)v.rows;
  if (sample == 1) grid = (unsigned)((p.n_items + p.stride - 1) / p.stride) * kItemQueries;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(cert_setup_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kSetupSmem);
    cudaFuncSetAttribute(cert_setup_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kSetupSmem);
    attr = true;
  }
  profile_before(DOSA_KERNEL_CERT_SETUP, stream);
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    cert_setup_kernel<true><<<grid, kSetupThreads, kSetupSmem, stream>>>(p);
  else
    cert_setup_kernel<false><<<grid, kSetupThreads, kSetupSmem, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_CERT_SETUP, stream);
  return e;
}

}  // namespace dosa
