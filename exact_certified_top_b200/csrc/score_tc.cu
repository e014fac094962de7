// Tensor-core dense indexer scorer for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]) for every visible pair
// of a block of query rows ("DOSA: Dots Sparse Attention", Daily Paper Cast
// transcript, Method section, problem formulation; and GPU kernel design:
// queries grouped into fixed-width tiles so dense tensor-core matrix
// operations can be used).
//
// One persistent CTA per SM.  A work item is a tile of kQueryTile (8)
// consecutive query rows; its 8 x 64 head vectors stay resident in shared
// memory while every key tile it can see streams through a ring of stages.
//   warp 0      TMA producer (one elected thread)
//   warp 1      TMEM owner and MMA issuer (one elected thread)
//   warps 2-17  epilogue: TMEM -> registers, w * ReLU, head sum, store
// MMA tile: A = 128 keys x d (K-major), B = 256 head rows (4 queries x 64
// heads) x d (K-major), D = 128 x 256 fp32 in TMEM.  Two D buffers (512 TMEM
// columns) let the epilogue of one tile overlap the MMA of the next.  TMEM lane
// = key, column = (query, head), so the head reduction runs down one thread's
// registers with no cross-thread traffic.  Every wait is bounded (dosa_device.cuh).
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "score_epilogue.cuh"

namespace dosa {

template <bool kFp8>
struct ScoreCfg {
  static constexpr int kSub = kFp8 ? 1 : 2;            // 128-byte K sub-tiles per d row
  static constexpr int kKSteps = kFp8 ? 4 : 8;         // 32-byte MMA K steps per d row
  static constexpr int kKeyStages = kFp8 ? 4 : 2;
  static constexpr int kH = 64;
  static constexpr int kQT = kQueryTile;
  static constexpr int kQRows = kQT * kH;              // 512 head rows per work item
  static constexpr int kGroupRows = 256;               // MMA N
  static constexpr int kGroups = kQRows / kGroupRows;  // 2 MMA tiles per key tile
  static constexpr int kQPerGroup = kGroupRows / kH;   // 4 queries per MMA tile
  static constexpr uint32_t kKeySubBytes = kKeyTile * 128;
  static constexpr uint32_t kKeyStageBytes = kKeySubBytes * kSub;
  static constexpr uint32_t kQSubBytes = kQRows * 128;
  static constexpr uint32_t kQBytes = kQSubBytes * kSub;
  static constexpr int kEpiWarps = 16;                 // 4 per TMEM lane quadrant
  static constexpr int kThreads = 64 + kEpiWarps * 32;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSmemBytes =
      1024 + kQBytes + kKeyStages * kKeyStageBytes + 256;
};

struct ScoreParams {
  const float* w;        // [rows_total, H], absolute rows
  const float* q_scale;  // [rows_total] (fp8) or null
  const float* k_scale;  // [S] (fp8) or null
  float* scores;         // row (t - row0), column s
  int64_t ld;
  int64_t row0, rows, pos0, S;
  int n_items;
  int H;                 // heads per query row: 32 or 64 (the MMA always sees 64)
  int* err;
  // Row-list mode (rows repaired after a candidate-list overflow): item i
  // scores part i % parts of the key tiles of the single row
  // row0 + row_list[i / parts] into output row i / parts; the number of rows is
  // min(*row_count, list_cap), read on the device.
  const int* row_list;
  const int* row_count;
  int list_cap;
  int parts;
};

struct ItemGeom {
  int64_t t0;     // first query row (absolute)
  int nq;         // valid queries in the tile
  int64_t pos_first;
  int64_t out0;   // output row of query t0
  int nkt;        // key tiles 0..nkt-1 cover keys 0..pos_last
  int j0, j1;     // the key tiles this item scores (empty item when j1 <= j0)
};

__device__ __forceinline__ ItemGeom item_geom(const ScoreParams& p, int item) {
  ItemGeom g;
  if (p.row_list) {
    const int64_t r = p.row_list[item / p.parts];
    g.t0 = p.row0 + r;
    g.nq = 1;
    g.pos_first = p.pos0 + r;
    g.out0 = item / p.parts;
  } else {
    const int tile = p.n_items - 1 - item;  // longest rows first
    g.t0 = p.row0 + (int64_t)tile * kQueryTile;
    const int64_t left = p.row0 + p.rows - g.t0;
    g.nq = (int)(left < kQueryTile ? left : kQueryTile);
    g.pos_first = p.pos0 + (int64_t)tile * kQueryTile;
    g.out0 = g.t0 - p.row0;
  }
  const int64_t pos_last = g.pos_first + g.nq - 1;
  g.nkt = (int)(pos_last / kKeyTile) + 1;
  g.j0 = 0;
  g.j1 = g.nkt;
  if (p.row_list) {
    const int part = item % p.parts;
    g.j0 = (int)((int64_t)g.nkt * part / p.parts);
    g.j1 = (int)((int64_t)g.nkt * (part + 1) / p.parts);
  }
  return g;
}

// kHeads: heads per query row (32 or 64); the MMA always sees 64 head slots.
template <bool kFp8, int kHeads>
__global__ void __launch_bounds__(ScoreCfg<kFp8>::kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap kmap, ScoreParams p) {
  using C = ScoreCfg<kFp8>;
  if (p.row_list) {
    const int n = *p.row_count;
    p.n_items = (n < p.list_cap ? n : p.list_cap) * p.parts;
    if (p.n_items <= 0) return;
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + C::kKeyStages * C::kKeyStageBytes);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::kKeyStages;
  uint64_t* acc_full = k_empty + C::kKeyStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done_bar = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::kKeyStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(done_bar, 1);
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
      uint32_t inflight_q = 0xFFFFFFFFu;   // item parity of the last Q load
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const ItemGeom g = item_geom(p, item);
        if (g.j1 <= g.j0) continue;
        if (!mbar_wait(q_empty, (it & 1) ^ 1, s_abort, p.err)) break;
        mbar_arrive_expect_tx(q_full, C::kQBytes);
        for (int sub = 0; sub < C::kSub; ++sub)
          for (int b = 0; b < C::kQRows / 256; ++b)
            tma_load_3d(sQ + sub * C::kQSubBytes + b * 256 * 128, &qmap, q_full, sub * 64, 0,
                        (int32_t)(g.t0 + b * 4));
        inflight_q = it & 1;
        ++it;
        for (int j = g.j0; j < g.j1; ++j, ++kc) {
          const int st = kc % C::kKeyStages;
          const uint32_t rnd = kc / C::kKeyStages;
          if (!mbar_wait(&k_empty[st], (rnd & 1) ^ 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[st], C::kKeyStageBytes);
          for (int sub = 0; sub < C::kSub; ++sub)
            tma_load_2d(sK + st * C::kKeyStageBytes + sub * C::kKeySubBytes, &kmap, &k_full[st],
                        sub * 64, j * kKeyTile);
        }
      }
      if (*s_abort) {
        // Let copies already issued land before the CTA can exit.
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
        const ItemGeom g = item_geom(p, item);
        if (g.j1 <= g.j0) continue;
        if (!mbar_wait(q_full, it & 1, s_abort, p.err)) break;
        ++it;
        tc_fence_after();
        for (int j = g.j0; j < g.j1 && ok; ++j, ++kc) {
          const int st = kc % C::kKeyStages;
          const uint32_t rnd = kc / C::kKeyStages;
          if (!mbar_wait(&k_full[st], rnd & 1, s_abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sK + st * C::kKeyStageBytes);
          for (int grp = 0; grp < C::kGroups; ++grp, ++u) {
            const uint32_t buf = u & 1;
            if (!mbar_wait(&acc_empty[buf], ((u >> 1) & 1) ^ 1, s_abort, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t b_base = smem_u32(sQ + grp * C::kGroupRows * 128);
            const uint32_t d_tmem = tmem_base + buf * C::kGroupRows;
#pragma unroll
            for (int step = 0; step < C::kKSteps; ++step) {
              const uint32_t sub = step >> 2, off = (step & 3) * 32;
              const uint64_t a = smem_desc_sw128(a_base + sub * C::kKeySubBytes + off);
              const uint64_t b = smem_desc_sw128(b_base + sub * C::kQSubBytes + off);
              tc_mma<kFp8>(d_tmem, a, b, idesc, step > 0 ? 1u : 0u);
            }
            tc_commit(&acc_full[buf]);
          }
          tc_commit(&k_empty[st]);
        }
        tc_commit(q_empty);
      }
      // Every MMA this thread issued has completed once done_bar flips.
      tc_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    // 16 warps: warp (2 + ew) reads TMEM lane quadrant (warp & 3), i.e. 32
    // keys, and query (ew >> 2) of each 4-query MMA tile.
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int sub = ew >> 2;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t u = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const ItemGeom g = item_geom(p, item);
      if (g.j1 <= g.j0) continue;
      // this warp's queries sub (MMA tile 0) and 4 + sub (MMA tile 1)
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
      float* ra = p.scores + (g.out0 + (va ? qa : 0)) * p.ld;
      float* rb = p.scores + (g.out0 + (vb ? qb : 0)) * p.ld;
      const uint32_t col0 = tmem_base + lane_off + sub * 64;
      for (int j = g.j0; j < g.j1 && ok; ++j) {
        const int s = j * kKeyTile + quad * 32 + lane;
        float sk = 1.0f;
        if constexpr (kFp8) sk = (s < p.S) ? __ldg(p.k_scale + s) : 0.0f;
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
          if (!(grp ? vb : va)) {
            // a query slot the item does not have (partial tiles, row lists)
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
            continue;
          }
          float v[32];
          HeadAcc acc = {0.f, 0.f, 0.f, 0.f};
          tmem_ld32_async(col, v);
          tmem_wait_ld(v);
          if (h64) {
            head_accumulate32(acc, v, wq);
            tmem_ld32_async(col + 32, v);
            tmem_wait_ld(v);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
          head_accumulate32(acc, v, wq + (h64 ? 32 : 0));   // H = 32: heads 0-31 only
          {
            float sc = head_total(acc);
            if constexpr (kFp8) sc *= (grp ? qsb : qsa) * sk;
            if (s <= (grp ? pos_b : pos_a)) (grp ? rb : ra)[s] = sc;
          }
        }
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

// ---- host side ------------------------------------------------------------------

bool encode_rows_map(CUtensorMap* map, const void* base, bool fp8, uint64_t rows,
                     uint32_t box_rows) {
  auto enc = get_tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {(cuuint32_t)(fp8 ? 128 : 64), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_q_map(CUtensorMap* map, const void* q, bool fp8, uint64_t rows, int H,
                  int box_rows) {
  auto enc = get_tensor_map_encoder();
  if (!enc || (H != 32 && H != 64)) return false;
  const uint64_t esz = fp8 ? 1 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * esz, (cuuint64_t)H * kHeadDim * esz};
  const cuuint32_t box[3] = {(cuuint32_t)(fp8 ? 128 : 64), 64, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         3, const_cast<void*>(q), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kFp8>
static cudaError_t launch_impl(const SeqView& v, float* scores, int64_t ld, int* err,
                               cudaStream_t stream, const int* row_list = nullptr,
                               const int* row_count = nullptr, int list_cap = 0) {
  using C = ScoreCfg<kFp8>;
  CUtensorMap qmap, kmap;
  if (!encode_q_map(&qmap, v.q, kFp8, (uint64_t)(v.row0 + v.rows), v.H) ||
      !encode_rows_map(&kmap, v.k, kFp8, (uint64_t)v.S, kKeyTile))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<kFp8, 64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(score_tc_kernel<kFp8, 32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  ScoreParams p;
  p.w = v.w;
  p.q_scale = v.q_scale;
  p.k_scale = v.k_scale;
  p.scores = scores;
  p.ld = ld;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.H = v.H;
  p.n_items = (int)((v.rows + kQueryTile - 1) / kQueryTile);
  p.err = err;
  p.row_list = row_list;
  p.row_count = row_count;
  p.list_cap = list_cap;
  // row lists: each row's key tiles split into parts of at least 64 tiles,
  // so that a few long rows still spread over every SM
  p.parts = 1;
  if (row_list) {
    const int64_t nkt = (v.pos0 + v.rows - 1) / kKeyTile + 1;
    int64_t parts = nkt / 64;
    if (parts > 2 * sms) parts = 2 * sms;
    p.parts = parts < 1 ? 1 : (int)parts;
    p.n_items = list_cap * p.parts;
  }
  if (p.n_items == 0) return cudaSuccess;
  const int grid = p.n_items < sms ? p.n_items : sms;
  profile_before(DOSA_KERNEL_SCORE, stream);
  if (v.H == 64)
    score_tc_kernel<kFp8, 64><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, kmap, p);
  else
    score_tc_kernel<kFp8, 32><<<grid, C::kThreads, C::kSmemBytes, stream>>>(qmap, kmap, p);
  const cudaError_t e = cudaGetLastError();
  profile_after(DOSA_KERNEL_SCORE, stream);
  return e;
}

cudaError_t launch_scores_tc(const Handle& h, const SeqView& v, float* scores, int64_t ld,
                             int* err, cudaStream_t stream) {
  if (h.cfg.dtype == DOSA_FP8_E4M3) return launch_impl<true>(v, scores, ld, err, stream);
  return launch_impl<false>(v, scores, ld, err, stream);
}

cudaError_t launch_scores_tc_rows(const Handle& h, const SeqView& v, const int* row_list,
                                  const int* row_count, int list_cap, float* scores, int64_t ld,
                                  int* err, cudaStream_t stream) {
  if (h.cfg.dtype == DOSA_FP8_E4M3)
    return launch_impl<true>(v, scores, ld, err, stream, row_list, row_count, list_cap);
  return launch_impl<false>(v, scores, ld, err, stream, row_list, row_count, list_cap);
}

}  // namespace dosa
