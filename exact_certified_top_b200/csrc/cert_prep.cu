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
constexpr int kSetupThreads = 256;
constexpr int kSetupSmem = (64 * (kHeadDim + 1) + 60 * 61) * 4;
constexpr int kPowerIters = 12;

// Solve the r x r symmetric positive definite system G a = b (Cholesky, fp64).
// Returns false when G is not numerically positive definite.
__device__ bool chol_solve(const double* G, const double* b, int n, double* a) {
  double L[4][4] = {};
  for (int i = 0; i < n; ++i) {
    for (int j = 0; j <= i; ++j) {
      double s = G[i * 4 + j];
      for (int k = 0; k < j; ++k) s -= L[i][k] * L[j][k];
      if (i == j) {
        if (!(s > 1e-12 * (G[i * 4 + i] + 1e-300))) return false;
        L[i][i] = sqrt(s);
      } else {
        L[i][j] = s / L[j][j];
      }
    }
  }
  double y[4];
  for (int i = 0; i < n; ++i) {
    double s = b[i];
    for (int k = 0; k < i; ++k) s -= L[i][k] * y[k];
    y[i] = s / L[i][i];
  }
  for (int i = n - 1; i >= 0; --i) {
    double s = y[i];
    for (int k = i + 1; k < n; ++k) s -= L[k][i] * a[k];
    a[i] = s / L[i][i];
  }
  return true;
}

// NNLS over supports of the r retained heads.  Gram: r x r (row stride 4),
// bh: r, qq = ||q_h||^2.  Writes alpha (>= 0, zeros off the support).
__device__ void nnls_enum(const double* Gram, const double* bh, double qq, int r, double* alpha) {
  double best = qq;
  for (int j = 0; j < 4; ++j) alpha[j] = 0.0;
  for (int mask = 1; mask < (1 << r); ++mask) {
    int idx[4], n = 0;
    for (int j = 0; j < r; ++j)
      if (mask >> j & 1) idx[n++] = j;
    double G[16], b[4], a[4];
    for (int i = 0; i < n; ++i) {
      b[i] = bh[idx[i]];
      for (int j = 0; j < n; ++j) G[i * 4 + j] = Gram[idx[i] * 4 + idx[j]];
    }
    if (!chol_solve(G, b, n, a)) continue;
    bool feasible = true;
    for (int i = 0; i < n; ++i) feasible &= a[i] > 0.0;
    if (!feasible) continue;
    // residual^2 = qq - 2 a.b + a^T G a = qq - a.b at the least-squares point
    double ab = 0.0;
    for (int i = 0; i < n; ++i) ab += a[i] * b[i];
    const double res = qq - ab;
    if (res < best) {
      best = res;
      for (int j = 0; j < 4; ++j) alpha[j] = 0.0;
      for (int i = 0; i < n; ++i) alpha[idx[i]] = a[i];
    }
  }
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

struct SetupParams {
  const void* q;          // [rows, 64, d] codes (absolute rows)
  const float* w;         // [rows, 64]
  const float* key_sum;   // [d] real-domain key sum of the sequence
  float inv_nkeys;        // 1 / number of keys of the sequence
  int64_t row0;           // first row of the chunk
  int64_t rows;
  int r, G, margin_log2;
  void* bdir;             // [rows, 8, d] codes (chunk-local rows)
  float* cert;            // [rows, kCertFloats]
  int32_t* retained;      // [rows, 4]
};

template <bool kFp8>
__global__ void __launch_bounds__(kSetupThreads) cert_setup_kernel(const SetupParams p) {
  constexpr int H = 64, D = kHeadDim;
  extern __shared__ float setup_dyn[];
  // code-domain heads, then residuals in place (padded rows); weighted residual Gram
  float(*qs)[D + 1] = reinterpret_cast<float(*)[D + 1]>(setup_dyn);
  float(*gt)[61] = reinterpret_cast<float(*)[61]>(setup_dyn + H * (D + 1));
  __shared__ float wv[H], qn[H], act[H], rn[H];
  __shared__ float kbar[D];
  __shared__ float vec[2][60];
  __shared__ double gram_r[16];
  __shared__ double alpha_s[H][4];
  __shared__ int R[4], O[64], A1[64], A2[64];
  __shared__ int nR, nO, nA1, nA2;
  __shared__ float red[kSetupThreads / 32];
  const int64_t i = blockIdx.x;
  const int64_t t = p.row0 + i;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = kSetupThreads / 32;

  for (int e = threadIdx.x; e < H * D; e += blockDim.x)
    qs[e / D][e % D] = decode_code<kFp8>(p.q, t * H * D + e);
  if (threadIdx.x < H) wv[threadIdx.x] = p.w[t * H + threadIdx.x];
  if (threadIdx.x < D) kbar[threadIdx.x] = p.key_sum[threadIdx.x] * p.inv_nkeys;
  __syncthreads();
  for (int h = warp; h < H; h += NW) {
    float ss = 0.f, ka = 0.f;
    for (int e = lane; e < D; e += 32) {
      ss = fmaf(qs[h][e], qs[h][e], ss);
      ka = fmaf(qs[h][e], kbar[e], ka);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      ka += __shfl_xor_sync(0xFFFFFFFFu, ka, o);
    }
    if (lane == 0) {
      qn[h] = sqrtf(ss);
      act[h] = ka;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // retained heads: top-r positive heads by w_h ||q_h||, ties to the smaller head
    int n = 0;
    bool taken[64] = {};
    for (int k = 0; k < p.r; ++k) {
      int best = -1;
      for (int h = 0; h < H; ++h) {
        if (wv[h] > 0.f && !taken[h] &&
            (best < 0 || wv[h] * qn[h] > wv[best] * qn[best]))
          best = h;
      }
      if (best < 0) break;
      taken[best] = true;
      ++n;
    }
    nR = 0;
    for (int h = 0; h < H; ++h)
      if (taken[h]) R[nR++] = h;     // ascending head order
    nO = nA1 = nA2 = 0;
    for (int h = 0; h < H; ++h) {
      if (wv[h] > 0.f && !taken[h]) O[nO++] = h;
      if (wv[h] < 0.f) {
        if (p.G >= 1 && act[h] > 0.f) A1[nA1++] = h;
        else if (p.G >= 2) A2[nA2++] = h;
      }
    }
  }
  __syncthreads();
  const int r = nR, no = nO;
  // Gram of the retained heads (fp64 from fp32 products summed in fp64)
  if (threadIdx.x < 16) {
    const int a = threadIdx.x >> 2, b = threadIdx.x & 3;
    double s = 0.0;
    if (a < r && b < r)
      for (int e = 0; e < D; ++e) s += (double)qs[R[a]][e] * (double)qs[R[b]][e];
    gram_r[threadIdx.x] = s;
  }
  __syncthreads();
  // NNLS for every omitted positive head: one thread per head
  if (threadIdx.x < no) {
    const int h = O[threadIdx.x];
    double bh[4] = {0, 0, 0, 0}, qq = 0.0;
    for (int e = 0; e < D; ++e) {
      const double x = qs[h][e];
      qq += x * x;
      for (int j = 0; j < r; ++j) bh[j] += (double)qs[R[j]][e] * x;
    }
    double a[4];
    nnls_enum(gram_r, bh, qq, r, a);
    for (int j = 0; j < 4; ++j) alpha_s[h][j] = a[j];
  }
  __syncthreads();
  // residuals in place of the omitted heads (retained rows are not modified)
  for (int e = threadIdx.x; e < no * D; e += blockDim.x) {
    const int h = O[e / D], c = e % D;
    float x = qs[h][c];
    for (int j = 0; j < r; ++j) x = fmaf(-(float)alpha_s[h][j], qs[R[j]][c], x);
    qs[h][c] = x;
  }
  __syncthreads();
  for (int k = warp; k < no; k += NW) {
    const int h = O[k];
    float ss = 0.f;
    for (int e = lane; e < D; e += 32) ss = fmaf(qs[h][e], qs[h][e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) rn[h] = sqrtf(ss);
  }
  // weighted residual Gram |[sqrt(w w') rho . rho']|
  for (int e = warp; e < no * no; e += NW) {
    const int a = e / no, b = e % no;
    if (b < a) continue;
    const int ha = O[a], hb = O[b];
    float s = 0.f;
    for (int c = lane; c < D; c += 32) s = fmaf(qs[ha][c], qs[hb][c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) {
      const float g = fabsf(sqrtf(wv[ha] * wv[hb]) * s);
      gt[a][b] = g;
      gt[b][a] = g;
    }
  }
  __syncthreads();
  // power iterations on |Gram| from the all-ones vector, then the
  // Collatz-Wielandt bound max_i (|Gram| v)_i / v_i
  if (threadIdx.x < 60) vec[0][threadIdx.x] = 1.f;
  __syncthreads();
  int cur = 0;
  for (int it = 0; it < kPowerIters; ++it) {
    if (threadIdx.x < no) {
      float s = 0.f;
      for (int b = 0; b < no; ++b) s = fmaf(gt[threadIdx.x][b], vec[cur][b], s);
      vec[cur ^ 1][threadIdx.x] = s;
    }
    __syncthreads();
    // normalise by the max entry
    float m = 0.f;
    for (int b = 0; b < no; ++b) m = fmaxf(m, vec[cur ^ 1][b]);
    __syncthreads();
    if (threadIdx.x < no) vec[cur ^ 1][threadIdx.x] = m > 0.f ? vec[cur ^ 1][threadIdx.x] / m : 1.f;
    __syncthreads();
    cur ^= 1;
  }
  float lam_part = 0.f;
  if (threadIdx.x < no) {
    float s = 0.f;
    for (int b = 0; b < no; ++b) s = fmaf(gt[threadIdx.x][b], vec[cur][b], s);
    const float v = fmaxf(vec[cur][threadIdx.x], 1e-30f);
    lam_part = s / v;
  }
  // block max of lam_part
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lam_part = fmaxf(lam_part, __shfl_xor_sync(0xFFFFFFFFu, lam_part, o));
  if (lane == 0) red[warp] = lam_part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float lam = 0.f;
    for (int w = 0; w < NW; ++w) lam = fmaxf(lam, red[w]);
    float wO = 0.f, bsum = 0.f, z2 = 0.f, scale = 0.f;
    for (int k = 0; k < no; ++k) {
      const int h = O[k];
      wO += wv[h];
      bsum = fmaf(wv[h], rn[h], bsum);
      z2 = fmaf(wv[h], rn[h] * rn[h], z2);
    }
    for (int h = 0; h < H; ++h) scale = fmaf(fabsf(wv[h]), qn[h], scale);
    // lambda bound: CW value with rounding headroom plus the Gram entry errors
    const float lam_b = lam * (1.f + 0x1p-16f) + 0x1p-16f * z2;
    const float bjoint = sqrtf(wO * lam_b) * (1.f + 0x1p-20f);
    const float bs = bsum * (1.f + 0x1p-20f);
    float beta = no > 0 ? fminf(bs, bjoint) : 0.f;
    beta += 0x1p-16f * scale;
    float* cf = p.cert + i * kCertFloats;
    for (int j = 0; j < 4; ++j) {
      float om = 0.f;
      if (j < r) {
        double o = wv[R[j]];
        for (int k = 0; k < no; ++k) o += (double)wv[O[k]] * alpha_s[O[k]][j];
        om = (float)o;
      }
      cf[kCertOmega + j] = om;
      p.retained[i * 4 + j] = j < r ? R[j] : -1;
    }
    cf[kCertBeta] = beta;   // the split errors of u_g are added below
    cf[kCertMargin] = ldexpf(scale, p.margin_log2) * (1.f + 0x1p-20f);
    cf[kCertBetaSum] = bs;
    cf[kCertBetaJoint] = bjoint;
    cf[kCertNA1] = (float)nA1;
    cf[kCertNA2] = (float)nA2;
    cf[kCertNO] = (float)no;
  }
  __syncthreads();
  // bound rows 0..3: the retained heads' own codes; 4..7: u_1 hi/lo, u_2 hi/lo
  const size_t esz = kFp8 ? 1 : 2;
  uint8_t* rows_out = static_cast<uint8_t*>(p.bdir) + (size_t)i * 8 * D * esz;
  const uint8_t* qrow = static_cast<const uint8_t*>(p.q) + (size_t)t * H * D * esz;
  for (int e = threadIdx.x; e < 4 * D * (int)esz; e += blockDim.x) {
    const int j = e / (D * esz), b = e % (D * esz);
    rows_out[e] = j < r ? qrow[(size_t)R[j] * D * esz + b] : 0;
  }
  // negative aggregates: thread c < D owns element c of u_1 and u_2
  __shared__ float uv[2][D], rv[2][D], red2[2][4];
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float u1 = 0.f, u2 = 0.f;
    for (int k = 0; k < nA1; ++k) u1 = fmaf(fabsf(wv[A1[k]]), qs[A1[k]][c], u1);
    for (int k = 0; k < nA2; ++k) u2 = fmaf(fabsf(wv[A2[k]]), qs[A2[k]][c], u2);
    uv[0][c] = u1;
    uv[1][c] = u2;
  }
  __syncthreads();
  for (int g = 0; g < 2; ++g) {
    // hi part: scale then round; lo part: the remainder, scaled and rounded
    float m = 0.f;
    for (int c = 0; c < D; ++c) m = fmaxf(m, fabsf(uv[g][c]));
    const float s_hi = kFp8 ? (m > 0.f ? m / 448.f : 0.f) : 1.f;
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      const float x = s_hi > 0.f ? uv[g][c] / s_hi : 0.f;
      const float hi = roundtrip<kFp8>(x);
      store_code<kFp8>(rows_out, (4 + 2 * g) * D + c, x);
      rv[g][c] = uv[g][c] - s_hi * hi;
    }
    __syncthreads();
    float m2 = 0.f;
    for (int c = 0; c < D; ++c) m2 = fmaxf(m2, fabsf(rv[g][c]));
    const float s_lo = kFp8 ? (m2 > 0.f ? m2 / 448.f : 0.f) : 1.f;
    float e2 = 0.f;
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      const float x = s_lo > 0.f ? rv[g][c] / s_lo : 0.f;
      const float lo = roundtrip<kFp8>(x);
      store_code<kFp8>(rows_out, (5 + 2 * g) * D + c, x);
      const float err = rv[g][c] - s_lo * lo;
      e2 = err * err;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e2 += __shfl_xor_sync(0xFFFFFFFFu, e2, o);
    if (lane == 0 && warp < 4) red2[g][warp] = e2;
    __syncthreads();
    if (threadIdx.x == 0) {
      const float err = sqrtf(red2[g][0] + red2[g][1] + red2[g][2] + red2[g][3]);
      float* cf = p.cert + i * kCertFloats;
      cf[kCertScale + 2 * g] = s_hi;
      cf[kCertScale + 2 * g + 1] = s_lo;
      cf[kCertBeta] += err * (1.f + 0x1p-10f);
    }
    __syncthreads();
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

cudaError_t launch_cert_setup(const Handle& h, const SeqView& v, const float* key_sum,
                              void* bdir, float* cert, int32_t* retained, cudaStream_t stream) {
  if (v.rows <= 0) return cudaSuccess;
  SetupParams p;
  p.q = v.q;
  p.w = v.w;
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
    cert_setup_kernel<true><<<(unsigned)v.rows, kSetupThreads, kSetupSmem, stream>>>(p);
  else
    cert_setup_kernel<false><<<(unsigned)v.rows, kSetupThreads, kSetupSmem, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_CERT_SETUP, stream);
  return e;
}

}  // namespace dosa
