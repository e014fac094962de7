// Survivor rescoring of the certified indexer for sm_100a ("DOSA: Dots Sparse
// Attention", Daily Paper Cast transcript, Method section: survivor masks
// compacted into per-query refinement streams, rescored with all heads on
// dense tensor-core tiles; scores at or above the threshold written back
// packed).
//
// A screening pass of the certified scorer leaves, per query row, the list of
// keys its certificate did not reject (survivor lists).  Here one CTA takes a
// work item (8 query rows) at a time and, per row, gathers its survivors 128
// at a time into shared memory in the 128-byte swizzled layout the MMA
// descriptors expect (a producer warp: 16-byte global loads, swizzled
// 16-byte shared stores, then a proxy fence), multiplies them with the row's
// 64 head slots on the tensor cores (M = 128 keys, N = 64, fp32 in TMEM),
// and reduces the heads in four epilogue warps (one per TMEM lane quadrant)
// with the same arithmetic as every other scorer, so the scores are bit-equal
// to the dense path's.  Scores >= the row's running threshold are appended to
// its candidate lists; the threshold is refreshed from the histogram every 8
// chunks and once more at the row's end.
//
// A launch covers one step range of the items flagged want_flag (all items
// when want_flag < 0): rows are published when the range reaches their
// item's last step, otherwise their state is saved for the next range.  An
// item with a row whose survivors did not fit its list is not rescored:
// ovf[item] is set and the filter scorer redoes the range for it from the
// state the screening pass saved.
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
  static constexpr int kStages = 4;                       // gathered key tiles in flight
  static constexpr int kBufs = 4;                         // TMEM accumulators of 64 columns
  static constexpr int kChunk = 128;                      // keys per MMA tile
  static constexpr int kHeadsN = 64;                      // MMA N: one row's 64 head slots
  static constexpr uint32_t kASubBytes = kChunk * 128;
  static constexpr uint32_t kAStageBytes = kASubBytes * kSub;
  static constexpr uint32_t kBSubBytes = kHeadsN * 128;
  static constexpr uint32_t kBBytes = kBSubBytes * kSub;
  static constexpr int kEpiWarps = 4;
  static constexpr int kThreads = 64 + kEpiWarps * 32;    // gather warp, MMA warp, epilogue
  static constexpr uint32_t kTmemCols = kBufs * kHeadsN;
  static constexpr int kCkptChunks = 8;
  static constexpr uint32_t kSmemBytes = 1024 + kBBytes + kStages * kAStageBytes +
                                         (uint32_t)sizeof(QState) + 512;
};

struct RescoreParams {
  const void* k;             // the sequence's first key (codes)
  const float* k_scale;      // the sequence's first key scale (fp8)
  const float* w;            // [rows_total, H] absolute rows
  const float* q_scale;      // absolute rows (fp8)
  const int* surv;           // [chunk rows][surv_cap] survivor keys (sequence-relative)
  const int* surv_count;     // [chunk rows]
  int surv_cap;
  Cand* cand;                // [chunk rows][kSegs][seg_cap]
  QStateG* qstate;           // [chunk rows] state saved by the screening pass
  const int* item_flag;
  int want_flag;
  StepRange range;           // the steps the screening pass covered
  int* ovf;                  // [items] set for items whose lists overflowed
  const unsigned long long* item_cnt;   // [items][3] the screening pass's held-back counts
  PublishOut out;
  unsigned long long* counters;
  int* err;
  int64_t row0, rows, pos0, S;
  int n_items, K, seg_cap;
};

template <bool kFp8, int kHeads>
__global__ void __launch_bounds__(RsCfg<kFp8>::kThreads, 1)
    rescore_kernel(const __grid_constant__ CUtensorMap qmap, const RescoreParams p) {
  using C = RsCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;
  uint8_t* sA = sB + C::kBBytes;
  QState* st = reinterpret_cast<QState*>(sA + C::kStages * C::kAStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(st + 1) + 7) & ~uintptr_t(7));
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* a_full = bars + 2;                      // [kStages]
  uint64_t* a_empty = a_full + C::kStages;          // [kStages]
  uint64_t* acc_full = a_empty + C::kStages;        // [kBufs]
  uint64_t* acc_empty = acc_full + C::kBufs;        // [kBufs]
  uint64_t* done_bar = acc_empty + C::kBufs;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  volatile int* s_go = s_abort + 1;                 // current item rescored (1) or skipped (0)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < C::kBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWarps);
    }
    mbar_init(done_bar, 1);
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

  // Items in CTA order; every role walks the same rows and chunk counts.
  // go: every row's survivors fit its list (decided by thread 0, shared by a
  // block barrier at each item).
  uint32_t a_cnt = 0, acc_cnt = 0, q_cnt = 0;
  unsigned long long n_exact = 0, n_cand = 0;
  bool ok = true;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    const Geom g = item_geometry(p.row0, p.rows, p.pos0, p.n_items, item);
    // thread 0 alone reads (and may rewrite) the item's flag; every thread
    // takes its decision from shared memory, so all reach the same barriers
    if (threadIdx.x == 0) {
      const Range rg = item_steps(p.range, p.item_flag, g, item);
      int go = rg.end > rg.begin ? (rg.end < g.n_tiles ? 1 : 2) : 0;   // 2: publish at the end
      if (go) {
        for (int ql = 0; ql < g.nq; ++ql)
          if (p.surv_count[g.local0 + ql] > p.surv_cap) go = 0;
        if (!go) {
          p.ovf[item] = 1;                       // the filter redoes (and counts) the range
        } else {
          atomicAdd(&p.counters[kCntSeedPairs], p.item_cnt[item * 3 + 0]);
          atomicAdd(&p.counters[kCntScreened], p.item_cnt[item * 3 + 1]);
          atomicAdd(&p.counters[kCntRejected], p.item_cnt[item * 3 + 2]);
        }
      }
      *s_go = go;
    }
    __syncthreads();
    const int go_v = *s_go;
    const bool go = go_v != 0, publish = go_v == 2;
    __syncthreads();
    if (!go) continue;
    for (int ql = 0; ql < g.nq; ++ql) {
      const int64_t r = g.local0 + ql;
      const int n = p.surv_count[r];
      const int n_chunks = (n + C::kChunk - 1) / C::kChunk;
      const int* list = p.surv + r * (int64_t)p.surv_cap;
      if (warp == 0) {
        // ---------------- gather producer ----------------
        if (lane == 0 && ok) {
          if (!mbar_wait(q_empty, (q_cnt & 1) ^ 1, s_abort, p.err)) ok = false;
          if (ok) {
            mbar_arrive_expect_tx(q_full, C::kBBytes);
            for (int sub = 0; sub < C::kSub; ++sub)
              tma_load_3d(sB + sub * C::kBSubBytes, &qmap, q_full, sub * 64, 0,
                          (int32_t)(g.t0 + ql));
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        for (int c = 0; c < n_chunks && ok; ++c, ++a_cnt) {
          const int s_ = a_cnt % C::kStages;
          bool w_ok = true;
          if (lane == 0) w_ok = mbar_wait(&a_empty[s_], ((a_cnt / C::kStages) & 1) ^ 1, s_abort, p.err);
          if (!__shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0)) {
            ok = false;
            break;
          }
          uint8_t* stage = sA + s_ * C::kAStageBytes;
          // 4 rows per lane, kSub x 8 chunks of 16 bytes per row
#pragma unroll
          for (int i = 0; i < C::kChunk / 32; ++i) {
            const int row = lane + 32 * i;
            const int at = c * C::kChunk + row;
            const int key = at < n ? list[at] : list[n - 1];
            const uint4* src = reinterpret_cast<const uint4*>(
                static_cast<const uint8_t*>(p.k) + (int64_t)key * kHeadDim * (kFp8 ? 1 : 2));
            uint4 v[8 * C::kSub];
#pragma unroll
            for (int j = 0; j < 8 * C::kSub; ++j) v[j] = __ldg(src + j);
#pragma unroll
            for (int sub = 0; sub < C::kSub; ++sub)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(stage + sub * C::kASubBytes + row * 128 +
                                          ((j ^ (row & 7)) << 4)) = v[sub * 8 + j];
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[s_]);
        }
      } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && ok) {
          constexpr uint32_t idesc = make_idesc<kFp8>(C::kChunk, C::kHeadsN);
          if (!mbar_wait(q_full, q_cnt & 1, s_abort, p.err)) ok = false;
          tc_fence_after();
          const uint32_t b_base = smem_u32(sB);
          for (int c = 0; c < n_chunks && ok; ++c) {
            const uint32_t s_ = (a_cnt + c) % C::kStages, buf = (acc_cnt + c) % C::kBufs;
            if (!mbar_wait(&a_full[s_], ((a_cnt + c) / C::kStages) & 1, s_abort, p.err) ||
                !mbar_wait(&acc_empty[buf], (((acc_cnt + c) / C::kBufs) & 1) ^ 1, s_abort, p.err)) {
              ok = false;
              break;
            }
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
          }
          tc_commit(q_empty);
        }
        a_cnt += n_chunks;
        acc_cnt += n_chunks;
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      } else {
        // ---------------- epilogue: one TMEM lane quadrant per warp ----------------
        const int ew = warp - 2;
        const int quad = warp & 3;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        QState& q = *st;
        if (ew == 0) {
          if (lane == 0) {
            q.row = r;
            q.pos = g.pos_first + ql;
          }
          state_load(q, p.qstate + r, lane);
          __syncwarp();
          __threadfence_block();
        }
        asm volatile("bar.sync 1, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
        int cnt = *reinterpret_cast<volatile int*>(&q.seg[quad]);
        Cand* seg = p.cand + (r * kSegs + quad) * (int64_t)p.seg_cap;
        const float* wq = p.w + (g.t0 + ql) * kHeads;
        float qs = 1.f;
        if constexpr (kFp8) qs = __ldg(p.q_scale + g.t0 + ql);
        // every epilogue warp runs all n_chunks iterations and every named
        // barrier, whatever happens, so none can wait on a warp that left
        for (int c = 0; c < n_chunks; ++c) {
          const int at = c * C::kChunk + quad * 32 + lane;
          const bool valid = at < n;
          const int key = valid ? list[at] : 0;
          float sk = 1.f;
          if constexpr (kFp8) sk = valid ? __ldg(p.k_scale + key) : 0.f;
          const uint32_t buf = (acc_cnt + c) % C::kBufs;
          if (ok && !mbar_wait(&acc_full[buf], ((acc_cnt + c) / C::kBufs) & 1, s_abort, p.err))
            ok = false;
          if (ok) {
          tc_fence_after();
          const uint32_t col = tmem_base + lane_off + buf * C::kHeadsN;
          float x[32];
          HeadAcc2 acc = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          tmem_ld32_async(col, x);
          tmem_wait_ld(x);
          if constexpr (kHeads == 64) {
            head_accumulate32(acc, x, wq);
            tmem_ld32_async(col + 32, x);
            tmem_wait_ld(x);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
          head_accumulate32(acc, x, wq + (kHeads == 64 ? 32 : 0));
          float sc = head_total(acc);
          if constexpr (kFp8) sc *= qs * sk;
          n_exact += __popc(__ballot_sync(0xFFFFFFFFu, valid));
          const float tau = *reinterpret_cast<const volatile float*>(&q.tau);
          n_cand += append_candidates(q, seg, p.seg_cap, cnt, valid && sc >= tau, sc, key, lane);
          }
          if ((c + 1) % C::kCkptChunks == 0 || c + 1 == n_chunks) {
            if (lane == 0) q.seg[quad] = cnt;
            __threadfence_block();
            asm volatile("bar.sync 1, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
            if (ew == 0 && ok)
              refresh_threshold(q, p.cand + r * kSegs * (int64_t)p.seg_cap, p.seg_cap, p.K, lane);
            asm volatile("bar.sync 1, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
          }
        }
        if (n_chunks == 0) {
          // no survivors: the state as saved is final
          asm volatile("bar.sync 1, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
        }
        if (ew == 0 && ok) {
          if (publish) {
            if (lane == 0) publish_query(q, p.out);
          } else {
            state_save(q, p.qstate + r, lane);
          }
        }
        acc_cnt += n_chunks;
        asm volatile("bar.sync 1, %0;" ::"r"(C::kEpiWarps * 32) : "memory");
      }
      if (warp == 0) q_cnt += 1;
      else if (warp == 1) q_cnt += 1;
    }
  }
  if (warp >= 2 && lane == 0) {
    atomicAdd(&p.counters[kCntExact], n_exact);
    atomicAdd(&p.counters[kCntRescored], n_exact);
    atomicAdd(&p.counters[kCntCandidates], n_cand);
  }
  if (warp == 1 && lane == 0) {
    tc_commit(done_bar);
    mbar_wait_drain(done_bar, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <bool kFp8>
static cudaError_t launch_rescore_impl(const Handle& h, const SeqView& v, const CertBuffers& b,
                                       int K, StepRange range, cudaStream_t stream) {
  using C = RsCfg<kFp8>;
  if (v.rows <= 0) return cudaSuccess;
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
  RescoreParams p;
  p.k = v.k;
  p.k_scale = v.k_scale;
  p.w = v.w;
  p.q_scale = v.q_scale;
  p.surv = b.surv;
  p.surv_count = b.surv_count;
  p.surv_cap = b.surv_cap;
  p.cand = reinterpret_cast<Cand*>(b.cand);
  p.qstate = reinterpret_cast<QStateG*>(b.qstate);
  p.item_flag = b.item_flag;
  p.want_flag = range.want_flag;
  p.range = range;
  p.ovf = b.ovf;
  p.item_cnt = b.item_cnt;
  p.out.cand_count = b.cand_count;
  p.out.tau = b.tau;
  p.out.repair_list = b.repair_list;
  p.out.repair_count = b.repair_count;
  p.out.repair_cap = b.repair_cap;
  p.out.n_repair = b.counters + kCntOverflow;
  p.out.dense = 0;
  p.out.err = b.err;
  p.counters = b.counters;
  p.err = b.err;
  p.row0 = v.row0;
  p.rows = v.rows;
  p.pos0 = v.pos0;
  p.S = v.S;
  p.n_items = (int)((v.rows + kItemQueries - 1) / kItemQueries);
  p.K = K;
  p.seg_cap = b.seg_cap;
  const int grid = p.n_items < 2 * sms ? p.n_items : 2 * sms;
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
                           StepRange range, cudaStream_t stream) {
  if (h.cfg.dtype == DOSA_FP8_E4M3) return launch_rescore_impl<true>(h, v, b, K, range, stream);
  return launch_rescore_impl<false>(h, v, b, K, range, stream);
}

}  // namespace dosa
