// C-ABI layer of libdosa: argument validation, workspace layout, launch
// orchestration.  No device memory is allocated here; every kernel runs on the
// caller's stream.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>
#include <algorithm>

#include "cert_layout.h"
#include "dosa_device.cuh"
#include "dosa_internal.h"
#include "work_items.cuh"

namespace dosa {

PFN_cuTensorMapEncodeTiled_v12000 get_tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace dosa

using namespace dosa;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct SeqInfo {
  int64_t q_start, q_end, k_start, k_end, q_pos0;
};

// Validate the pointers and the packed varlen batch shared by the Top-K calls.
dosa_status check_common(const Handle* h, const void* q, const float* q_scale, const float* w,
                         const void* k, const float* k_scale, const int64_t* seq_offsets, int B,
                         int K, const int32_t* out_idx) {
  if (!h || !q || !w || !k || !seq_offsets || !out_idx || B < 1) return DOSA_ERR_INVALID_ARG;
  if (K < 1 || K > h->cfg.max_K) return DOSA_ERR_INVALID_ARG;
  const bool fp8 = h->cfg.dtype == DOSA_FP8_E4M3;
  if (fp8 && (!q_scale || !k_scale)) return DOSA_ERR_INVALID_ARG;
  if (!fp8 && (q_scale || k_scale)) return DOSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(w)) return DOSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    const int64_t* r = seq_offsets + 3 * b;
    const int64_t* n = seq_offsets + 3 * (b + 1);
    const int64_t nq = n[0] - r[0], nk = n[1] - r[1];
    if (r[0] < 0 || r[1] < 0 || nq < 0 || nk < 0 || r[2] < 0) return DOSA_ERR_INVALID_ARG;
    if (nq > 0 && r[2] + nq > nk) return DOSA_ERR_INVALID_ARG;
    if (nk > (int64_t)1 << 31) return DOSA_ERR_UNSUPPORTED;
    if (b == 0 && (r[0] != 0 || r[1] != 0)) return DOSA_ERR_INVALID_ARG;
  }
  return DOSA_OK;
}

SeqInfo seq_info(const int64_t* so, int b) {
  SeqInfo s;
  s.q_start = so[3 * b];
  s.q_end = so[3 * (b + 1)];
  s.k_start = so[3 * b + 1];
  s.k_end = so[3 * (b + 1) + 1];
  s.q_pos0 = so[3 * b + 2];
  return s;
}

int64_t max_keys(const int64_t* so, int B) {
  int64_t m = 0;
  for (int b = 0; b < B; ++b) {
    const SeqInfo s = seq_info(so, b);
    if (s.k_end - s.k_start > m) m = s.k_end - s.k_start;
  }
  return m;
}

size_t elem_bytes(const Handle* h) { return h->cfg.dtype == DOSA_FP8_E4M3 ? 1 : 2; }

SeqView make_view(const Handle* h, const void* q, const float* q_scale, const float* w,
                  const void* k, const float* k_scale, const SeqInfo& s) {
  SeqView v;
  v.q = q;
  v.q_scale = q_scale;
  v.w = w;
  v.k = static_cast<const uint8_t*>(k) + s.k_start * kHeadDim * elem_bytes(h);
  v.k_scale = k_scale ? k_scale + s.k_start : nullptr;
  v.row0 = s.q_start;
  v.rows = s.q_end - s.q_start;
  v.pos0 = s.q_pos0;
  v.S = s.k_end - s.k_start;
  v.H = h->cfg.H;
  return v;
}

constexpr int64_t kDefaultChunkBytes = (int64_t)4 << 30;   // dense score chunk budget
constexpr int64_t kDefaultCertChunkBytes = (int64_t)8 << 30;   // certified per-row arrays
// Rows per chunk whose candidate list may overflow and be rescored densely:
// as many fp32 score rows of S_max keys as fit in 1 GiB, at least 64 and at
// most 512 (a row overflows when a tie at its K-th score spans more keys than
// its list holds).
int64_t repair_rows(int64_t S_max) {
  const int64_t n = ((int64_t)1 << 30) / (4 * (S_max > 1 ? S_max : 1));
  return n < 64 ? 64 : n > 512 ? 512 : n;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Candidate capacity per query row and segment.  A row's list has 4
// segments, one per 32-key quarter of every key tile.  A row with n keys
// appends about K (1 + ln(n / K)) candidates (a key is appended when it
// enters the running Top-K, with probability about K / its rank in the
// processing order).  The histogram threshold's coarseness adds more on rows
// where a few very large scores stretch its range: measured tails reach 1.75x
// the mean at 128K keys and more at 1M.  A segment holds 0.9 K (1 + ln(S_max /
// K)) entries (3.6x the mean per segment; at least 1024, rounded up to 64),
// and never more than the keys it can see: 32 per key tile.  A row that
// overflows is rescored densely.
int seg_capacity(int K, int64_t S_max) {
  const double ratio = S_max > K ? (double)S_max / K : 1.0;
  int64_t cap = (int64_t)ceil(0.9 * K * (1.0 + log(ratio)));
  cap = (cap + 63) / 64 * 64;
  if (cap < 1024) cap = 1024;
  const int64_t most = (S_max + kKeyTile - 1) / kKeyTile * 32;
  if (cap > most) cap = most;
  if (cap < 1) cap = 1;
  return (int)cap;
}

// Workspace of the certified path: a fixed part (header, key norms, key sum,
// repair area) and Tc rows of per-query state.
struct CertLayout {
  size_t key_norm, key_sum, repair_list, repair_count, repair_scores, blk, pass_any, fixed;
  int64_t repair_rows;
  int step_cap;     // block screening: steps per item list (key tiles of S_max), or 0
  int64_t words;    // ranked screening: survivor words per row (4 per key tile), or 0
  size_t per_row;   // bytes per chunk row (bound rows, record, retained, list, count, tau)
  int seg_cap;
  int64_t dense_ld; // dense writeback: the score matrix's row length (0 when sparse)
};

CertLayout cert_layout(const Handle* h, int64_t S_max, int K) {
  CertLayout L;
  size_t off = kWsHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += (size_t)round_up((int64_t)bytes, 256);
    return at;
  };
  L.seg_cap = seg_capacity(K, S_max);
  L.key_norm = take((size_t)S_max * 4);
  L.key_sum = take(kHeadDim * 4);
  L.repair_rows = repair_rows(S_max);
  L.repair_list = take((size_t)L.repair_rows * 4);
  L.repair_count = take(4);
  L.repair_scores = take((size_t)L.repair_rows * S_max * 4);
  // block screening covers sequences of up to 8192 key tiles (1M keys)
  L.step_cap = h->cfg.block_bound ? (int)((S_max + kKeyTile - 1) / kKeyTile) : 0;
  if (L.step_cap > 8192) L.step_cap = 0;
  L.blk = take((size_t)L.step_cap * kBlkFloats * 4);
  L.pass_any = take((kRankEst + 2) * 4);
  L.fixed = off;
  // bound rows, record, retained, list, count, tau, carried state, item flag
  L.per_row = (size_t)kBoundRows * kHeadDim * elem_bytes(h) + kCertFloats * 4 + 4 * 4 +
              (size_t)L.seg_cap * 4 * 8 + 4 * 4 + 4 + qstate_bytes() + 1;
  L.dense_ld = h->cfg.sparse_writeback ? 0 : round_up(S_max > 1 ? S_max : 1, 64);
  L.per_row += (size_t)L.dense_ld * 4;
  // step lists: one per work item of 8 rows (plus the count)
  L.per_row += ((size_t)L.step_cap * 4 + 4 + 7) / 8;
  // ranked screening: survivor bits, threshold estimates, band, largest
  // rejected bound and pass of each row, probe counts of each item
  const bool ranked = h->cfg.screening >= 2;
  L.words = ranked ? (S_max + kKeyTile - 1) / kKeyTile * 4 : 0;
  if (ranked) L.per_row += (size_t)L.words * 4 + kRankEst * 4 + 4 * 4 + 2;
  return L;
}

// Carve the per-row arrays of a chunk of Tc rows after the fixed part.
CertBuffers cert_buffers(const Handle* h, const CertLayout& L, uint8_t* ws, int64_t Tc) {
  CertBuffers b;
  size_t off = L.fixed;
  auto take = [&](size_t bytes) {
    uint8_t* p = ws + off;
    off += (size_t)round_up((int64_t)bytes, 256);
    return p;
  };
  b.key_norm = reinterpret_cast<float*>(ws + L.key_norm);
  b.key_sum = reinterpret_cast<float*>(ws + L.key_sum);
  b.repair_list = reinterpret_cast<int*>(ws + L.repair_list);
  b.repair_count = reinterpret_cast<int*>(ws + L.repair_count);
  b.repair_scores = reinterpret_cast<float*>(ws + L.repair_scores);
  b.repair_cap = (int)L.repair_rows;
  b.seg_cap = L.seg_cap;
  b.bdir = take((size_t)Tc * kBoundRows * kHeadDim * elem_bytes(h));
  b.cert = reinterpret_cast<float*>(take((size_t)Tc * kCertFloats * 4));
  b.retained = reinterpret_cast<int32_t*>(take((size_t)Tc * 16));
  b.cand = take((size_t)Tc * 4 * L.seg_cap * 8);
  b.cand_count = reinterpret_cast<int*>(take((size_t)Tc * 4 * 4));
  b.tau = reinterpret_cast<float*>(take((size_t)Tc * 4));
  b.qstate = take((size_t)Tc * qstate_bytes());
  b.item_flag = reinterpret_cast<int*>(take((size_t)(Tc / 8 + 1) * 4));
  b.dense = L.dense_ld ? reinterpret_cast<float*>(take((size_t)Tc * L.dense_ld * 4)) : nullptr;
  b.dense_ld = L.dense_ld;
  b.blk = L.step_cap ? reinterpret_cast<float*>(ws + L.blk) : nullptr;
  b.step_cap = L.step_cap;
  b.step_list = L.step_cap ? reinterpret_cast<int*>(take((size_t)(Tc / 8 + 1) * L.step_cap * 4))
                           : nullptr;
  b.step_count = L.step_cap ? reinterpret_cast<int*>(take((size_t)(Tc / 8 + 1) * 4)) : nullptr;
  b.words = L.words;
  const bool ranked = L.words > 0;
  b.bits = ranked ? reinterpret_cast<uint32_t*>(take((size_t)Tc * L.words * 4)) : nullptr;
  b.est = ranked ? reinterpret_cast<float*>(take((size_t)Tc * kRankEst * 4)) : nullptr;
  b.band_lo = ranked ? reinterpret_cast<float*>(take((size_t)Tc * 4)) : nullptr;
  b.band_hi = ranked ? reinterpret_cast<float*>(take((size_t)Tc * 4)) : nullptr;
  b.maxrej = ranked ? reinterpret_cast<uint32_t*>(take((size_t)Tc * 4)) : nullptr;
  b.row_next = ranked ? reinterpret_cast<int*>(take((size_t)Tc * 4)) : nullptr;
  b.rank_cnt = ranked ? reinterpret_cast<unsigned long long*>(take((size_t)(Tc / 8 + 1) * 16))
                      : nullptr;
  b.pass_any = reinterpret_cast<int*>(ws + L.pass_any);
  b.gate = &reinterpret_cast<WsHeader*>(ws)->probe_gate;
  b.probe_sample = 0;
  b.counters = reinterpret_cast<WsHeader*>(ws)->counters;
  b.err = &reinterpret_cast<WsHeader*>(ws)->error;
  return b;
}

// Padding the per-row arrays of a chunk may need (each starts 256-aligned),
// plus the item-flag array's extra entry.
constexpr size_t kCertPad = 20 * 256 + 16 + 16 * 1024 * 4;

// Rows per certified chunk that fit in ws_bytes (a multiple of 8, or 0).
int64_t cert_chunk_rows(const CertLayout& L, size_t ws_bytes) {
  if (ws_bytes <= L.fixed + kCertPad) return 0;
  int64_t rows = (int64_t)((ws_bytes - L.fixed - kCertPad) / L.per_row);
  return rows / 8 * 8;
}

// Steps of the warm-up (enough key tiles for K exact scores, whichever tile
// is partial), rounded up to the threshold checkpoint interval, and the
// steps the probe screens after it.
int warmup_steps(int K) { return ((K + kKeyTile - 1) / kKeyTile + 1 + 3) / 4 * 4; }
// Screening every tile with the key-block certificate: the certified scorer
// runs this many steps after the warm-up before the first block pass.
constexpr int kProbeSteps = 4;

int64_t total_visible(const int64_t* so, int B) {
  int64_t v = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t nq = so[3 * (b + 1)] - so[3 * b], p0 = so[3 * b + 2];
    v += nq * (2 * p0 + nq + 1) / 2;
  }
  return v;
}

}  // namespace

extern "C" {

const char* dosa_status_string(dosa_status s) {
  switch (s) {
    case DOSA_OK: return "ok";
    case DOSA_ERR_INVALID_ARG: return "invalid argument";
    case DOSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case DOSA_ERR_WORKSPACE: return "workspace too small";
    case DOSA_ERR_CUDA: return "CUDA error";
    case DOSA_ERR_TIMEOUT: return "device wait timed out";
    case DOSA_ERR_DEVICE_CHECK: return "device bounds check failed";
  }
  return "unknown status";
}

void dosa_index_config_default(dosa_index_config* cfg) {
  if (!cfg) return;
  cfg->H = 64;
  cfg->d = 128;
  cfg->dtype = DOSA_BF16;
  cfg->max_K = 2048;
  cfg->seed_first = 64;
  cfg->seed_last = 512;
  cfg->r = 4;
  cfg->G = 2;
  cfg->margin_log2 = -12;
  cfg->screening = 2;
  cfg->sparse_writeback = 1;
  cfg->block_bound = 1;
  cfg->probe_sample = 1;
  cfg->short_dense_keys = 16384;
}

dosa_status dosa_index_create(const dosa_index_config* cfg, dosa_index_t* out) {
  if (!cfg || !out) return DOSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg->dtype != DOSA_BF16 && cfg->dtype != DOSA_FP8_E4M3) return DOSA_ERR_INVALID_ARG;
  if (cfg->max_K < 1 || cfg->max_K > 4096) return DOSA_ERR_INVALID_ARG;
  if (cfg->seed_first < 0 || cfg->seed_last < 0 || cfg->r < 0 || cfg->r > 4 || cfg->G < 0 ||
      cfg->G > 2 || cfg->margin_log2 > -4 || cfg->margin_log2 < -24 || cfg->screening < 0 ||
      cfg->screening > 3 || cfg->sparse_writeback < 0 || cfg->sparse_writeback > 1 ||
      cfg->block_bound < 0 || cfg->block_bound > 1 || cfg->probe_sample < 0 ||
      cfg->probe_sample > 1 || cfg->short_dense_keys < 0)
    return DOSA_ERR_INVALID_ARG;
  if (cfg->d != kHeadDim || (cfg->H != 32 && cfg->H != 64)) return DOSA_ERR_UNSUPPORTED;
  Handle* h = new (std::nothrow) Handle;
  if (!h) return DOSA_ERR_INVALID_ARG;
  h->cfg = *cfg;
  *out = reinterpret_cast<dosa_index_t>(h);
  return DOSA_OK;
}

void dosa_index_destroy(dosa_index_t hh) {
  Handle* h = reinterpret_cast<Handle*>(hh);
  if (!h) return;
  if (h->copy_stream) {
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(h->copy_device);
    cudaStreamDestroy(h->copy_stream);
    for (cudaEvent_t e : {h->ev_loaded[0], h->ev_loaded[1], h->ev_done[0], h->ev_done[1],
                          h->ev_keys, h->ev_out})
      if (e) cudaEventDestroy(e);
    cudaSetDevice(cur);
  }
  delete h;
}

dosa_status dosa_index_workspace_size(dosa_index_t hh, int64_t Tq, int64_t S_max, int K,
                                      int certified, int64_t chunk_rows, size_t* bytes) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  if (!h || !bytes || Tq < 0 || S_max < 0 || K < 1 || K > h->cfg.max_K || chunk_rows < 0)
    return DOSA_ERR_INVALID_ARG;
  if (certified) {
    const CertLayout L = cert_layout(h, S_max, K);
    int64_t rows = chunk_rows;
    if (rows == 0) {
      rows = kDefaultCertChunkBytes / (int64_t)L.per_row;
      rows = rows / 8 * 8;
      if (rows < 8) rows = 8;
    }
    rows = round_up(rows, 8);
    if (rows > round_up(Tq, 8)) rows = round_up(Tq, 8);
    if (rows < 8) rows = 8;
    *bytes = L.fixed + (size_t)rows * L.per_row + kCertPad;
    return DOSA_OK;
  }
  int64_t rows = chunk_rows;
  if (rows == 0) {
    rows = S_max > 0 ? kDefaultChunkBytes / (S_max * 4) : Tq;
    rows = rows / kQueryTile * kQueryTile;
    if (rows < kQueryTile) rows = kQueryTile;
  }
  if (rows > round_up(Tq, kQueryTile)) rows = round_up(Tq, kQueryTile);
  if (rows < 1) rows = 1;
  *bytes = (size_t)(kWsHeaderBytes + round_up(rows * S_max * 4, 256));
  return DOSA_OK;
}

dosa_status dosa_index_dense_topk(dosa_index_t hh, const void* q, const float* q_scale,
                                  const float* w, const void* k, const float* k_scale,
                                  const int64_t* seq_offsets, int B, int K, int32_t* out_idx,
                                  void* workspace, size_t ws_bytes, void* stream_) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  dosa_status st = check_common(h, q, q_scale, w, k, k_scale, seq_offsets, B, K, out_idx);
  if (st != DOSA_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DOSA_ERR_INVALID_ARG;
  const int64_t S_max = max_keys(seq_offsets, B);
  if (ws_bytes < kWsHeaderBytes + (size_t)S_max * 4) return DOSA_ERR_WORKSPACE;
  int64_t chunk = S_max > 0 ? (int64_t)((ws_bytes - kWsHeaderBytes) / ((size_t)S_max * 4)) : 1;
  if (chunk >= kQueryTile) chunk = chunk / kQueryTile * kQueryTile;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int* err = static_cast<int*>(workspace);
  float* scores = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeaderBytes);
  for (int b = 0; b < B; ++b) {
    const SeqInfo s = seq_info(seq_offsets, b);
    SeqView v = make_view(h, q, q_scale, w, k, k_scale, s);
    const int64_t rows = v.rows;
    for (int64_t r = 0; r < rows; r += chunk) {
      SeqView c = v;
      c.row0 = v.row0 + r;
      c.rows = rows - r < chunk ? rows - r : chunk;
      c.pos0 = v.pos0 + r;
      if (launch_scores_tc(*h, c, scores, v.S, err, stream) != cudaSuccess) return DOSA_ERR_CUDA;
      if (launch_topk_rows(scores, v.S, nullptr, c.pos0 + 1, v.S, c.rows, K, out_idx + c.row0 * K,
                           K, stream) != cudaSuccess)
        return DOSA_ERR_CUDA;
    }
  }
  return DOSA_OK;
}

}  // extern "C"

// Whether a chunk whose longest row has max_tiles key tiles is screened at
// all: never with screening off; with ranked screening only when some row
// has key tiles past the warm-up (past the probe too, in the adaptive mode):
// before them every pair is scored exactly, so the chunk goes to the filter
// scorer alone.
static bool screening_can_act(const Handle* h, int64_t max_tiles, int K) {
  if (h->cfg.screening == 2) return max_tiles > warmup_steps(K) + kRankProbeTiles;
  if (h->cfg.screening == 3) return max_tiles > warmup_steps(K);
  return h->cfg.screening != 0;
}

// The certificate set-up of a chunk.  With every row's record wanted (or
// screening on every item) all rows are set up; with screening off none; in
// the adaptive mode only the rows of the sampled items, the others after the
// sampled probe, if it found an item worth screening (cert_chunk).
static dosa_status setup_chunk(const Handle* h, const SeqView& c, CertBuffers& cb, bool records,
                               int K, cudaStream_t stream) {
  const int mode = h->cfg.screening;
  cb.probe_sample = 0;
  if (!records && !screening_can_act(h, (c.pos0 + c.rows - 1) / kKeyTile + 1, K)) return DOSA_OK;
  if (!records && mode == 2 && h->cfg.probe_sample) {
    const int64_t n_items = (c.rows + 7) / 8;
    if (cudaMemsetAsync(cb.item_flag, 0, (size_t)n_items * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(cb.gate, 0, sizeof(int), stream) != cudaSuccess ||
        launch_cert_setup(*h, c, cb.key_sum, cb.bdir, cb.cert, cb.retained, stream, 1,
                          cb.item_flag, cb.gate) != cudaSuccess)
      return DOSA_ERR_CUDA;
    cb.probe_sample = 1;
    return DOSA_OK;
  }
  return launch_cert_setup(*h, c, cb.key_sum, cb.bdir, cb.cert, cb.retained, stream) ==
                 cudaSuccess
             ? DOSA_OK
             : DOSA_ERR_CUDA;
}

// Runs key prep and certificate setup for one sequence chunk by chunk, calling
// `body(chunk view, buffers)` after each setup.
template <typename Body>
static dosa_status for_each_cert_chunk(const Handle* h, const void* q, const float* q_scale,
                                       const float* w, const void* k, const float* k_scale,
                                       const int64_t* seq_offsets, int B, int K, void* workspace,
                                       size_t ws_bytes, cudaStream_t stream, float* cert_out,
                                       int32_t* retained_out, Body body) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DOSA_ERR_INVALID_ARG;
  const int64_t S_max = max_keys(seq_offsets, B);
  const CertLayout L = cert_layout(h, S_max, K);
  const int64_t Tc = cert_chunk_rows(L, ws_bytes);
  if (Tc < 8) return DOSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, kWsHeaderBytes, stream) != cudaSuccess) return DOSA_ERR_CUDA;
  CertBuffers buf = cert_buffers(h, L, ws, Tc);
  for (int b = 0; b < B; ++b) {
    const SeqInfo s = seq_info(seq_offsets, b);
    const SeqView v = make_view(h, q, q_scale, w, k, k_scale, s);
    if (v.rows == 0) continue;
    if (launch_key_prep(*h, v.k, v.k_scale, v.S, buf.key_norm, buf.key_sum, stream) !=
            cudaSuccess ||
        (buf.blk && screening_can_act(h, (v.S + kKeyTile - 1) / kKeyTile, K) &&
         launch_block_prep(*h, v.k, v.k_scale, v.S, buf.blk, stream) != cudaSuccess))
      return DOSA_ERR_CUDA;
    for (int64_t r = 0; r < v.rows; r += Tc) {
      SeqView c = v;
      c.row0 = v.row0 + r;
      c.rows = v.rows - r < Tc ? v.rows - r : Tc;
      c.pos0 = v.pos0 + r;
      CertBuffers cb = buf;
      if (cert_out) cb.cert = cert_out + c.row0 * kCertFloats;
      if (retained_out) cb.retained = retained_out + c.row0 * 4;
      dosa_status st = setup_chunk(h, c, cb, cert_out != nullptr, K, stream);
      if (st != DOSA_OK) return st;
      st = body(c, cb);
      if (st != DOSA_OK) return st;
    }
  }
  return DOSA_OK;
}

// The certified Top-K of one chunk of rows whose certificate is set up:
// scoring passes, selection, repair of overflowed rows.  out: row 0 of the
// chunk's indices.
static dosa_status cert_chunk(const Handle* h, const SeqView& c, const CertBuffers& b, int K,
                              int32_t* out, cudaStream_t stream) {
  if (cudaMemsetAsync(b.repair_count, 0, sizeof(int), stream) != cudaSuccess)
    return DOSA_ERR_CUDA;
  // dense writeback (ablation): pairs the scorers never write (rejected) stay -inf
  if (b.dense && launch_fill(b.dense, c.rows * b.dense_ld, -INFINITY, stream) != cudaSuccess)
    return DOSA_ERR_CUDA;
  // screening 0: the filter scorer alone; 1: the certified scorer alone (the
  // pages' streaming schedule); 3: warm-up by the filter scorer, then ranked
  // screening of every item; 2: warm-up, a ranked probe of kRankProbeTiles
  // key tiles per item, then each item finished by ranked screening or by the
  // filter scorer, as its probe chose
  constexpr int kAll = 0x3FFFFFFF;
  const int mode =
      screening_can_act(h, (c.pos0 + c.rows - 1) / kKeyTile + 1, K) ? h->cfg.screening : 0;
  // With the key-block certificate, the certified scorer's last range is
  // first screened tile by tile as a whole (block_screen) and then processes
  // the steps left.
  const bool blk = b.blk != nullptr;
  const int W = warmup_steps(K), P = W + kProbeSteps;
  const int n_items = (int)((c.rows + 7) / 8);
  // The certified scorer from step `from` on.  With the key-block certificate
  // the rest runs in passes [r0, 2 r0): each pass first drops the tiles that
  // the threshold reached so far rules out.
  auto certified_rest = [&](int from) -> bool {
    if (!blk)
      return launch_certified(*h, c, b, K, StepRange{from, kAll, -1}, stream) == cudaSuccess;
    const int max_steps = (int)((c.pos0 + c.rows - 1) / kKeyTile + 1);
    for (int r0 = from; r0 < max_steps; r0 *= 2) {
      const int r1 = 2 * r0 >= max_steps ? kAll : 2 * r0;
      if (launch_block_screen(*h, c, b, StepRange{r0, r1, -1}, stream) != cudaSuccess ||
          launch_certified(*h, c, b, K, StepRange{r0, r1, -1}, stream, 1) != cudaSuccess)
        return false;
    }
    return true;
  };
  // Ranked passes of the rows waiting for pass 1 (of the items flagged `want`
  // when sel is set): pass 1 screens the tiles the probe left (lo_off), every
  // later pass the whole range for the rows the rescoring sent back.
  auto ranked = [&](const int* sel, int want, int lo_off) -> bool {
    for (int pass = 1; pass <= kRankEst; ++pass) {
      const RankPass rp{pass, pass == 1 ? lo_off : 0, 0, pass == 1 ? sel : nullptr, want,
                        nullptr};
      if (launch_rank_screen(*h, c, b, K, W, rp, stream) != cudaSuccess ||
          launch_rescore(*h, c, b, K, W, rp, stream) != cudaSuccess)
        return false;
    }
    return true;
  };
  // The probe of the items flagged `want`: estimates, kRankProbeTiles screened
  // tiles per item, and the decision (kItemRank or kItemFilter).
  auto probe = [&](int want) -> bool {
    const RankPass rp{1, 0, kRankProbeTiles, b.item_flag, want, b.rank_cnt};
    return cudaMemsetAsync(b.rank_cnt, 0, (size_t)n_items * 16, stream) == cudaSuccess &&
           launch_rank_prep(*h, c, b, K, W, b.item_flag, want, stream) == cudaSuccess &&
           launch_rank_screen(*h, c, b, K, W, rp, stream) == cudaSuccess &&
           launch_rank_decide(b.item_flag, b.rank_cnt, n_items, want, b.gate, b.counters,
                              stream) == cudaSuccess;
  };
  if (mode >= 2 && (cudaMemsetAsync(b.row_next, 0, (size_t)c.rows * 4, stream) != cudaSuccess ||
                    cudaMemsetAsync(b.pass_any, 0, (kRankEst + 2) * 4, stream) != cudaSuccess))
    return DOSA_ERR_CUDA;
  if (mode == 0) {
    if (launch_filter(*h, c, b, K, StepRange{0, kAll, -1}, stream) != cudaSuccess)
      return DOSA_ERR_CUDA;
  } else if (mode == 1) {
    if (launch_certified(*h, c, b, K, StepRange{0, blk ? P : kAll, -1}, stream) != cudaSuccess ||
        (blk && !certified_rest(P)))
      return DOSA_ERR_CUDA;
  } else if (mode == 3) {
    if (launch_filter(*h, c, b, K, StepRange{0, W, -1}, stream) != cudaSuccess ||
        launch_rank_prep(*h, c, b, K, W, nullptr, 0, stream) != cudaSuccess ||
        !ranked(nullptr, 0, 0))
      return DOSA_ERR_CUDA;
  } else {
    // The probe: all items, or the sampled items first and the others only
    // when some sampled item chose ranked screening (else they go to the
    // filter scorer unprobed, from the warm-up's end).
    auto probes = [&]() -> bool {
      if (!b.probe_sample)
        return cudaMemsetAsync(b.item_flag, 0, (size_t)n_items * 4, stream) == cudaSuccess &&
               probe(0);
      return probe(kItemSample) &&
             launch_probe_resolve(b.item_flag, n_items, b.gate, stream) == cudaSuccess &&
             launch_cert_setup(*h, c, b.key_sum, b.bdir, b.cert, b.retained, stream, 2,
                               b.item_flag, b.gate) == cudaSuccess &&
             probe(kItemProbe);
    };
    // the filter scorer finishes the items whose probe chose it, and the
    // unprobed items, from the warm-up's end, in one launch
    if (launch_filter(*h, c, b, K, StepRange{0, W, -1}, stream) != cudaSuccess || !probes() ||
        launch_filter(*h, c, b, K, StepRange{W, kAll, kItemFilter, kItemUnprobed, W}, stream) !=
            cudaSuccess ||
        !ranked(b.item_flag, kItemRank, kRankProbeTiles))
      return DOSA_ERR_CUDA;
  }
  if (b.dense) {
    // the dense Top-K of every exact score; no list can need a repair
    return launch_topk_rows(b.dense, b.dense_ld, nullptr, c.pos0 + 1, b.dense_ld, c.rows, K, out,
                            K, stream) == cudaSuccess
               ? DOSA_OK
               : DOSA_ERR_CUDA;
  }
  if (launch_select(b, c.rows, c.pos0, K, out, stream) != cudaSuccess) return DOSA_ERR_CUDA;
  // rows whose candidate list overflowed: dense rescoring of just those rows
  if (launch_scores_tc_rows(*h, c, b.repair_list, b.repair_count, b.repair_cap, b.repair_scores,
                            c.S, b.err, stream) != cudaSuccess)
    return DOSA_ERR_CUDA;
  if (launch_topk_list(b.repair_scores, c.S, b.repair_list, b.repair_count, b.repair_cap,
                       c.pos0 + 1, c.S, K, out, K, stream) != cudaSuccess)
    return DOSA_ERR_CUDA;
  return DOSA_OK;
}

// Counters of the workspace header into *stats (synchronises the stream).
static dosa_status read_stats(const void* workspace, const int64_t* seq_offsets, int B,
                              cudaStream_t stream, dosa_stats* stats) {
  WsHeader hdr;
  if (cudaMemcpyAsync(&hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return DOSA_ERR_CUDA;
  stats->visible_pairs = total_visible(seq_offsets, B);
  stats->seed_pairs = (int64_t)hdr.counters[kCntSeedPairs];
  stats->screened_pairs = (int64_t)hdr.counters[kCntScreened];
  // pairs rejected by the first ranked pass and scored by a later one are not
  // rejected in the end
  stats->rejected_pairs =
      (int64_t)hdr.counters[kCntRejected] - (int64_t)hdr.counters[kCntBandPairs];
  stats->exact_pairs = (int64_t)hdr.counters[kCntExact];
  stats->candidates = (int64_t)hdr.counters[kCntCandidates];
  stats->filtered_pairs = (int64_t)hdr.counters[kCntFiltered];
  stats->block_skipped_pairs = (int64_t)hdr.counters[kCntBlockSkipped];
  stats->rescored_pairs = (int64_t)hdr.counters[kCntRescored];
  stats->repaired_rows = (int64_t)hdr.counters[kCntOverflow];
  stats->rescreened_pairs = (int64_t)hdr.counters[kCntBandPairs];
  if (hdr.error) return hdr.error == kDevTimeout ? DOSA_ERR_TIMEOUT : DOSA_ERR_DEVICE_CHECK;
  return DOSA_OK;
}

// ---- host-staged certified calls ---------------------------------------------------

namespace {

// Device workspace of a host-staged call: the certified workspace for Tc rows,
// the keys (and key scales) of every sequence, and two staging slots of Tc
// query rows (q, q_scale, w in; indices out).
struct HostLayout {
  CertLayout L;
  int64_t Tc;
  size_t keys, kscale, slot[2], slot_q, slot_qs, slot_w, slot_out, total;
};

constexpr int64_t kHostChunkRows = 16384;

HostLayout host_layout(const Handle* h, int64_t Tq, int64_t S_total, int64_t S_max, int K,
                       int64_t chunk_rows) {
  HostLayout H;
  H.L = cert_layout(h, S_max, K);
  int64_t rows = chunk_rows > 0 ? chunk_rows : kHostChunkRows;
  rows = round_up(rows, 8);
  if (rows > round_up(Tq, 8)) rows = round_up(Tq, 8);
  if (rows < 8) rows = 8;
  H.Tc = rows;
  const size_t esz = elem_bytes(h);
  const bool fp8 = h->cfg.dtype == DOSA_FP8_E4M3;
  size_t off = (size_t)round_up((int64_t)(H.L.fixed + (size_t)rows * H.L.per_row + kCertPad), 256);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += (size_t)round_up((int64_t)bytes, 256);
    return at;
  };
  H.keys = take((size_t)S_total * kHeadDim * esz);
  H.kscale = take(fp8 ? (size_t)S_total * 4 : 0);
  size_t so = 0;
  auto take_slot = [&](size_t bytes) {
    const size_t at = so;
    so += (size_t)round_up((int64_t)bytes, 256);
    return at;
  };
  H.slot_q = take_slot((size_t)rows * h->cfg.H * kHeadDim * esz);
  H.slot_qs = take_slot(fp8 ? (size_t)rows * 4 : 0);
  H.slot_w = take_slot((size_t)rows * h->cfg.H * 4);
  H.slot_out = take_slot((size_t)rows * K * 4);
  H.slot[0] = take(so);
  H.slot[1] = take(so);
  H.total = off;
  return H;
}

// The handle's copy stream and events on the current device (created on
// first use, recreated when the device changes).
dosa_status ensure_copy_stream(Handle* h) {
  std::lock_guard<std::mutex> lock(h->copy_mutex);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DOSA_ERR_CUDA;
  if (h->copy_stream && h->copy_device == dev) return DOSA_OK;
  if (h->copy_stream) {
    cudaSetDevice(h->copy_device);
    cudaStreamDestroy(h->copy_stream);
    for (cudaEvent_t* e : {&h->ev_loaded[0], &h->ev_loaded[1], &h->ev_done[0], &h->ev_done[1],
                           &h->ev_keys, &h->ev_out})
      if (*e) cudaEventDestroy(*e), *e = nullptr;
    h->copy_stream = nullptr;
    cudaSetDevice(dev);
  }
  if (cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking) != cudaSuccess)
    return DOSA_ERR_CUDA;
  for (cudaEvent_t* e : {&h->ev_loaded[0], &h->ev_loaded[1], &h->ev_done[0], &h->ev_done[1],
                         &h->ev_keys, &h->ev_out})
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return DOSA_ERR_CUDA;
  h->copy_device = dev;
  return DOSA_OK;
}

}  // namespace

// Whether a certified call takes the dense path: the adaptive mode, every
// sequence within short_dense_keys keys, and room in the workspace for at
// least one query tile of scores.
static bool short_dense(const Handle* h, const int64_t* seq_offsets, int B, size_t ws_bytes) {
  if (h->cfg.screening != 2 || h->cfg.short_dense_keys <= 0) return false;
  const int64_t S_max = max_keys(seq_offsets, B);
  if (S_max > h->cfg.short_dense_keys) return false;
  return ws_bytes >= kWsHeaderBytes + (size_t)kQueryTile * (size_t)(S_max > 0 ? S_max : 1) * 4;
}

extern "C" {

dosa_status dosa_index_topk(dosa_index_t hh, const void* q, const float* q_scale, const float* w,
                            const void* k, const float* k_scale, const int64_t* seq_offsets,
                            int B, int K, int32_t* out_idx, void* workspace, size_t ws_bytes,
                            void* stream_, dosa_stats* stats) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  dosa_status st = check_common(h, q, q_scale, w, k, k_scale, seq_offsets, B, K, out_idx);
  if (st != DOSA_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (short_dense(h, seq_offsets, B, ws_bytes)) {
    // short rows: the dense scorer and radix Top-K, the same selection
    if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, stream) != cudaSuccess) return DOSA_ERR_CUDA;
    st = dosa_index_dense_topk(hh, q, q_scale, w, k, k_scale, seq_offsets, B, K, out_idx,
                               workspace, ws_bytes, stream_);
    if (st != DOSA_OK) return st;
    if (stats) {
      st = read_stats(workspace, seq_offsets, B, stream, stats);
      stats->exact_pairs = stats->visible_pairs;
      return st;
    }
    return DOSA_OK;
  }
  st = for_each_cert_chunk(
      h, q, q_scale, w, k, k_scale, seq_offsets, B, K, workspace, ws_bytes, stream, nullptr,
      nullptr, [&](const SeqView& c, const CertBuffers& b) -> dosa_status {
        return cert_chunk(h, c, b, K, out_idx + c.row0 * K, stream);
      });
  if (st != DOSA_OK) return st;
  if (stats) return read_stats(workspace, seq_offsets, B, stream, stats);
  return DOSA_OK;
}

dosa_status dosa_index_host_workspace_size(dosa_index_t hh, int64_t Tq, int64_t S_total,
                                           int64_t S_max, int K, int64_t chunk_rows,
                                           size_t* bytes) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  if (!h || !bytes || Tq < 0 || S_total < 0 || S_max < 0 || S_max > S_total || K < 1 ||
      K > h->cfg.max_K || chunk_rows < 0)
    return DOSA_ERR_INVALID_ARG;
  *bytes = host_layout(h, Tq, S_total, S_max, K, chunk_rows).total;
  return DOSA_OK;
}

dosa_status dosa_index_topk_host(dosa_index_t hh, const void* q, const float* q_scale,
                                 const float* w, const void* k, const float* k_scale,
                                 const int64_t* seq_offsets, int B, int K, int32_t* out_idx,
                                 void* workspace, size_t ws_bytes, void* stream_,
                                 dosa_stats* stats) {
  Handle* h = reinterpret_cast<Handle*>(hh);
  dosa_status st = check_common(h, q, q_scale, w, k, k_scale, seq_offsets, B, K, out_idx);
  if (st != DOSA_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DOSA_ERR_INVALID_ARG;
  const int64_t Tq = seq_offsets[3 * B], S_total = seq_offsets[3 * B + 1];
  const int64_t S_max = max_keys(seq_offsets, B);
  // the most rows per staging slot (up to the default) that fit the workspace
  HostLayout H = host_layout(h, Tq, S_total, S_max, K, 0);
  if (ws_bytes < H.total) {
    int64_t lo = 8, hi = H.Tc;            // largest multiple of 8 in [lo, hi) that fits
    if (host_layout(h, Tq, S_total, S_max, K, lo).total > ws_bytes) return DOSA_ERR_WORKSPACE;
    while (hi - lo > 8) {
      const int64_t mid = (lo + hi) / 2 / 8 * 8;
      if (host_layout(h, Tq, S_total, S_max, K, mid).total <= ws_bytes) lo = mid;
      else hi = mid;
    }
    H = host_layout(h, Tq, S_total, S_max, K, lo);
  }
  st = ensure_copy_stream(h);
  if (st != DOSA_OK) return st;
  cudaStream_t main = static_cast<cudaStream_t>(stream_), cpy = h->copy_stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool fp8 = h->cfg.dtype == DOSA_FP8_E4M3;
  const size_t esz = elem_bytes(h), qrow = (size_t)h->cfg.H * kHeadDim * esz;
  const CertBuffers buf = cert_buffers(h, H.L, ws, H.Tc);
  uint8_t* dk = ws + H.keys;
  float* dks = fp8 ? reinterpret_cast<float*>(ws + H.kscale) : nullptr;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // keys first (on the caller's stream, ordered after its earlier work); the
  // copy stream starts after that point, so it never overwrites a slot that
  // an earlier call on this stream still reads
  if (!ok(cudaMemsetAsync(ws, 0, kWsHeaderBytes, main)) ||
      !ok(cudaMemcpyAsync(dk, k, (size_t)S_total * kHeadDim * esz, cudaMemcpyHostToDevice, main)) ||
      (fp8 && !ok(cudaMemcpyAsync(dks, k_scale, (size_t)S_total * 4, cudaMemcpyHostToDevice,
                                  main))) ||
      !ok(cudaEventRecord(h->ev_keys, main)) || !ok(cudaStreamWaitEvent(cpy, h->ev_keys, 0)))
    return DOSA_ERR_CUDA;
  struct Chunk {
    int b;
    int64_t r0, rows;
  };
  std::vector<Chunk> chunks;
  for (int b = 0; b < B; ++b) {
    const SeqInfo si = seq_info(seq_offsets, b);
    for (int64_t r = 0; r < si.q_end - si.q_start; r += H.Tc)
      chunks.push_back({b, r, std::min<int64_t>(H.Tc, si.q_end - si.q_start - r)});
  }
  const uint8_t* qh = static_cast<const uint8_t*>(q);
  // stage chunk ci's query rows into slot ci % 2 (after the compute that last
  // read that slot)
  auto load = [&](size_t ci) -> bool {
    const Chunk& ch = chunks[ci];
    const int slot = (int)(ci & 1);
    const int64_t t0 = seq_info(seq_offsets, ch.b).q_start + ch.r0;
    uint8_t* sb = ws + H.slot[slot];
    return ok(cudaStreamWaitEvent(cpy, h->ev_done[slot], 0)) &&
           ok(cudaMemcpyAsync(sb + H.slot_q, qh + (size_t)t0 * qrow, (size_t)ch.rows * qrow,
                              cudaMemcpyHostToDevice, cpy)) &&
           (!fp8 || ok(cudaMemcpyAsync(sb + H.slot_qs, q_scale + t0, (size_t)ch.rows * 4,
                                       cudaMemcpyHostToDevice, cpy))) &&
           ok(cudaMemcpyAsync(sb + H.slot_w, w + t0 * h->cfg.H, (size_t)ch.rows * h->cfg.H * 4,
                              cudaMemcpyHostToDevice, cpy)) &&
           ok(cudaEventRecord(h->ev_loaded[slot], cpy));
  };
  if (!chunks.empty() && !load(0)) return DOSA_ERR_CUDA;
  int prev_b = -1;
  for (size_t ci = 0; ci < chunks.size(); ++ci) {
    if (ci + 1 < chunks.size() && !load(ci + 1)) return DOSA_ERR_CUDA;
    const Chunk& ch = chunks[ci];
    const int slot = (int)(ci & 1);
    const SeqInfo si = seq_info(seq_offsets, ch.b);
    uint8_t* sb = ws + H.slot[slot];
    SeqView c;
    c.q = sb + H.slot_q;
    c.q_scale = fp8 ? reinterpret_cast<const float*>(sb + H.slot_qs) : nullptr;
    c.w = reinterpret_cast<const float*>(sb + H.slot_w);
    c.k = dk + (size_t)si.k_start * kHeadDim * esz;
    c.k_scale = fp8 ? dks + si.k_start : nullptr;
    c.row0 = 0;
    c.rows = ch.rows;
    c.pos0 = si.q_pos0 + ch.r0;
    c.S = si.k_end - si.k_start;
    c.H = h->cfg.H;
    int32_t* dout = reinterpret_cast<int32_t*>(sb + H.slot_out);
    if (ch.b != prev_b) {
      if (launch_key_prep(*h, c.k, c.k_scale, c.S, buf.key_norm, buf.key_sum, main) !=
              cudaSuccess ||
          (buf.blk && screening_can_act(h, (c.S + kKeyTile - 1) / kKeyTile, K) &&
           launch_block_prep(*h, c.k, c.k_scale, c.S, buf.blk, main) != cudaSuccess))
        return DOSA_ERR_CUDA;
      prev_b = ch.b;
    }
    if (!ok(cudaStreamWaitEvent(main, h->ev_loaded[slot], 0))) return DOSA_ERR_CUDA;
    CertBuffers cb = buf;
    st = setup_chunk(h, c, cb, false, K, main);
    if (st != DOSA_OK) return st;
    st = cert_chunk(h, c, cb, K, dout, main);
    if (st != DOSA_OK) return st;
    if (!ok(cudaEventRecord(h->ev_done[slot], main)) ||
        !ok(cudaStreamWaitEvent(cpy, h->ev_done[slot], 0)) ||
        !ok(cudaMemcpyAsync(out_idx + (si.q_start + ch.r0) * K, dout, (size_t)ch.rows * K * 4,
                            cudaMemcpyDeviceToHost, cpy)))
      return DOSA_ERR_CUDA;
  }
  // the caller's stream completes after the last copy out
  if (!ok(cudaEventRecord(h->ev_out, cpy)) || !ok(cudaStreamWaitEvent(main, h->ev_out, 0)))
    return DOSA_ERR_CUDA;
  if (stats) return read_stats(workspace, seq_offsets, B, main, stats);
  return DOSA_OK;
}

// ---- decode step ----------------------------------------------------------------
}  // extern "C"

namespace {

// Decode workspace: the header, then per query row the seed bitmap, the seed
// bounds, counts, the shared histogram and threshold (all zeroed per call),
// the selection inputs and the candidate list.  A row's list holds all its
// visible keys, so it cannot overflow.
struct DecodeLayout {
  size_t bitmap, tau_key, smax_key, seed_count, dup, count, hist, tau_run, zero_end;
  size_t cand_count, tau, cand, total;
  int64_t words;
  int64_t cap;
};

DecodeLayout decode_layout(int64_t Tq, int64_t S_max, int K) {
  (void)K;
  DecodeLayout L;
  size_t off = kWsHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += (size_t)round_up((int64_t)bytes, 256);
    return at;
  };
  L.cap = round_up(S_max > 64 ? S_max : 64, 64);
  L.words = (S_max + 31) / 32;
  // zeroed per call: bitmap .. tau_run (tau_key is then set to all ones)
  L.bitmap = take((size_t)Tq * L.words * 4);
  L.tau_key = take((size_t)Tq * 4);
  L.smax_key = take((size_t)Tq * 4);
  L.seed_count = take((size_t)Tq * 4);
  L.dup = take((size_t)Tq * 4);
  L.count = take((size_t)Tq * 4);
  L.hist = take((size_t)Tq * 256 * 4);
  L.tau_run = take((size_t)Tq * 4);
  L.zero_end = off;
  L.cand_count = take((size_t)Tq * 16);
  L.tau = take((size_t)Tq * 4);
  L.cand = take((size_t)Tq * L.cap * 8);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

dosa_status dosa_index_decode_workspace_size(dosa_index_t hh, int64_t Tq, int64_t S_max, int K,
                                             size_t* bytes) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  if (!h || !bytes || Tq < 0 || S_max < 0 || K < 1 || K > h->cfg.max_K)
    return DOSA_ERR_INVALID_ARG;
  *bytes = decode_layout(Tq, S_max, K).total;
  return DOSA_OK;
}

dosa_status dosa_index_decode_topk(dosa_index_t hh, const void* q, const float* q_scale,
                                   const float* w, const void* k, const float* k_scale,
                                   const int64_t* seq_offsets, int B, int K,
                                   const int32_t* seed_idx, int32_t* out_idx, void* workspace,
                                   size_t ws_bytes, void* stream_, dosa_stats* stats) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  dosa_status st = check_common(h, q, q_scale, w, k, k_scale, seq_offsets, B, K, out_idx);
  if (st != DOSA_OK) return st;
  if (!seed_idx) return DOSA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DOSA_ERR_INVALID_ARG;
  const int64_t Tq = seq_offsets[3 * B], S_max = max_keys(seq_offsets, B);
  const DecodeLayout L = decode_layout(Tq, S_max, K);
  if (ws_bytes < L.total) return DOSA_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, kWsHeaderBytes, stream) != cudaSuccess ||
      cudaMemsetAsync(ws + L.bitmap, 0, L.zero_end - L.bitmap, stream) != cudaSuccess ||
      cudaMemsetAsync(ws + L.tau_key, 0xFF, (size_t)Tq * 4, stream) != cudaSuccess)
    return DOSA_ERR_CUDA;
  for (int b = 0; b < B; ++b) {
    const SeqInfo s = seq_info(seq_offsets, b);
    const SeqView v = make_view(h, q, q_scale, w, k, k_scale, s);
    if (v.rows == 0) continue;
    const int64_t r0 = s.q_start;
    DecodeBuffers d;
    d.words = L.words;
    d.bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap) + r0 * L.words;
    d.tau_key = reinterpret_cast<uint32_t*>(ws + L.tau_key) + r0;
    d.smax_key = reinterpret_cast<uint32_t*>(ws + L.smax_key) + r0;
    d.seed_count = reinterpret_cast<int*>(ws + L.seed_count) + r0;
    d.dup = reinterpret_cast<int*>(ws + L.dup) + r0;
    d.count = reinterpret_cast<int*>(ws + L.count) + r0;
    d.hist = reinterpret_cast<unsigned*>(ws + L.hist) + r0 * 256;
    d.tau_run = reinterpret_cast<uint32_t*>(ws + L.tau_run) + r0;
    d.cand_count = reinterpret_cast<int*>(ws + L.cand_count) + r0 * 4;
    d.tau = reinterpret_cast<float*>(ws + L.tau) + r0;
    d.cand = ws + L.cand + (size_t)r0 * L.cap * 8;
    d.cap = (int)L.cap;
    d.counters = reinterpret_cast<WsHeader*>(ws)->counters;
    d.err = &reinterpret_cast<WsHeader*>(ws)->error;
    int32_t* out = out_idx + r0 * K;
    if (launch_decode(*h, v, d, K, seed_idx + r0 * K, stream) != cudaSuccess)
      return DOSA_ERR_CUDA;
    // selection over the candidate lists (one segment of cap entries per row)
    CertBuffers sb;
    std::memset(&sb, 0, sizeof(sb));
    sb.cand = d.cand;
    sb.seg_cap = d.cap / 4;                 // rows are 4 * seg_cap apart; one segment used
    sb.cand_count = d.cand_count;
    sb.tau = d.tau;
    if (launch_select(sb, v.rows, v.pos0, K, out, stream) != cudaSuccess) return DOSA_ERR_CUDA;
  }
  if (stats) return read_stats(workspace, seq_offsets, B, stream, stats);
  return DOSA_OK;
}

dosa_status dosa_index_certificate(dosa_index_t hh, const void* q, const float* q_scale,
                                   const float* w, const void* k, const float* k_scale,
                                   const int64_t* seq_offsets, int B, float* cert_out,
                                   int32_t* retained_out, void* bound_out, void* workspace,
                                   size_t ws_bytes, void* stream_) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  if (!cert_out || !retained_out) return DOSA_ERR_INVALID_ARG;
  dosa_status st = check_common(h, q, q_scale, w, k, k_scale, seq_offsets, B, 1, retained_out);
  if (st != DOSA_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const size_t row_bytes = (size_t)kBoundRows * kHeadDim * elem_bytes(h);
  return for_each_cert_chunk(
      h, q, q_scale, w, k, k_scale, seq_offsets, B, 1, workspace, ws_bytes, stream, cert_out,
      retained_out, [&](const SeqView& c, const CertBuffers& b) -> dosa_status {
        if (!bound_out || c.rows == 0) return DOSA_OK;
        return cudaMemcpyAsync(static_cast<uint8_t*>(bound_out) + (size_t)c.row0 * row_bytes,
                               b.bdir, (size_t)c.rows * row_bytes, cudaMemcpyDeviceToDevice,
                               stream) == cudaSuccess
                   ? DOSA_OK
                   : DOSA_ERR_CUDA;
      });
}

static dosa_status scores_common(dosa_index_t hh, const void* q, const float* q_scale,
                                 const float* w, const void* k, const float* k_scale, int64_t row0,
                                 int64_t rows, int64_t pos0, int64_t S, float* scores, int64_t ld,
                                 SeqView* v) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  if (!h || !q || !w || !k || !scores || row0 < 0 || rows < 0 || pos0 < 0 || S < 1)
    return DOSA_ERR_INVALID_ARG;
  if (rows > 0 && (pos0 + rows > S || ld < pos0 + rows)) return DOSA_ERR_INVALID_ARG;
  const bool fp8 = h->cfg.dtype == DOSA_FP8_E4M3;
  if (fp8 != (q_scale != nullptr) || fp8 != (k_scale != nullptr)) return DOSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(w)) return DOSA_ERR_INVALID_ARG;
  v->q = q;
  v->q_scale = q_scale;
  v->w = w;
  v->k = k;
  v->k_scale = k_scale;
  v->row0 = row0;
  v->rows = rows;
  v->pos0 = pos0;
  v->S = S;
  v->H = h->cfg.H;
  return DOSA_OK;
}

dosa_status dosa_index_scores(dosa_index_t hh, const void* q, const float* q_scale, const float* w,
                              const void* k, const float* k_scale, int64_t row0, int64_t rows,
                              int64_t pos0, int64_t S, float* scores, int64_t ld, void* scratch,
                              void* stream) {
  SeqView v;
  dosa_status st = scores_common(hh, q, q_scale, w, k, k_scale, row0, rows, pos0, S, scores, ld, &v);
  if (st != DOSA_OK) return st;
  if (!scratch) return DOSA_ERR_INVALID_ARG;
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  return launch_scores_tc(*h, v, scores, ld, static_cast<int*>(scratch),
                          static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DOSA_OK
             : DOSA_ERR_CUDA;
}

dosa_status dosa_reference_scores(dosa_index_t hh, const void* q, const float* q_scale,
                                  const float* w, const void* k, const float* k_scale,
                                  int64_t row0, int64_t rows, int64_t pos0, int64_t S,
                                  float* scores, int64_t ld, void* stream) {
  SeqView v;
  dosa_status st = scores_common(hh, q, q_scale, w, k, k_scale, row0, rows, pos0, S, scores, ld, &v);
  if (st != DOSA_OK) return st;
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  return launch_scores_ref(*h, v, scores, ld, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DOSA_OK
             : DOSA_ERR_CUDA;
}

dosa_status dosa_topk_rows(const float* scores, int64_t ld, const int64_t* row_len, int64_t rows,
                           int K, int32_t* out, void* stream) {
  if (!scores || !row_len || !out || rows < 0 || K < 1 || ld < 0) return DOSA_ERR_INVALID_ARG;
  return launch_topk_rows(scores, ld, row_len, 0, ld, rows, K, out, K,
                          static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DOSA_OK
             : DOSA_ERR_CUDA;
}

dosa_status dosa_check_device(void* workspace, void* stream) {
  // NULL: the error word of dosa_index_dense_topk_static, which lives in the
  // header of the library's fixed scratch array on the current device
  if (!workspace) workspace = static_scratch_address();
  if (!workspace) return DOSA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DOSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DOSA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(int), s) != cudaSuccess) return DOSA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DOSA_ERR_CUDA;
    return word == kDevTimeout ? DOSA_ERR_TIMEOUT : DOSA_ERR_DEVICE_CHECK;
  }
  return DOSA_OK;
}

}  // extern "C"
