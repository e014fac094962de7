// C-ABI layer of libdosa: argument validation, workspace layout, launch
// orchestration.  No device memory is allocated here; every kernel runs on the
// caller's stream.
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "dosa_device.cuh"
#include "dosa_internal.h"

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
  return v;
}

constexpr int64_t kDefaultChunkBytes = (int64_t)4 << 30;   // dense score chunk budget

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

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
  cfg->screening = 1;
}

dosa_status dosa_index_create(const dosa_index_config* cfg, dosa_index_t* out) {
  if (!cfg || !out) return DOSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg->dtype != DOSA_BF16 && cfg->dtype != DOSA_FP8_E4M3) return DOSA_ERR_INVALID_ARG;
  if (cfg->max_K < 1 || cfg->max_K > 4096) return DOSA_ERR_INVALID_ARG;
  if (cfg->seed_first < 0 || cfg->seed_last < 0 || cfg->r < 0 || cfg->r > 4 || cfg->G < 0 ||
      cfg->G > 2 || cfg->margin_log2 > -4 || cfg->margin_log2 < -24)
    return DOSA_ERR_INVALID_ARG;
  if (cfg->d != kHeadDim || cfg->H != 64) return DOSA_ERR_UNSUPPORTED;
  Handle* h = new (std::nothrow) Handle;
  if (!h) return DOSA_ERR_INVALID_ARG;
  h->cfg = *cfg;
  *out = reinterpret_cast<dosa_index_t>(h);
  return DOSA_OK;
}

void dosa_index_destroy(dosa_index_t h) { delete reinterpret_cast<Handle*>(h); }

dosa_status dosa_index_workspace_size(dosa_index_t hh, int64_t Tq, int64_t S_max, int K,
                                      int certified, int64_t chunk_rows, size_t* bytes) {
  const Handle* h = reinterpret_cast<const Handle*>(hh);
  if (!h || !bytes || Tq < 0 || S_max < 0 || K < 1 || K > h->cfg.max_K || chunk_rows < 0)
    return DOSA_ERR_INVALID_ARG;
  if (certified) return DOSA_ERR_UNSUPPORTED;
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

dosa_status dosa_index_topk(dosa_index_t hh, const void* q, const float* q_scale, const float* w,
                            const void* k, const float* k_scale, const int64_t* seq_offsets,
                            int B, int K, int32_t* out_idx, void* workspace, size_t ws_bytes,
                            void* stream, dosa_stats* stats) {
  (void)hh; (void)q; (void)q_scale; (void)w; (void)k; (void)k_scale; (void)seq_offsets;
  (void)B; (void)K; (void)out_idx; (void)workspace; (void)ws_bytes; (void)stream; (void)stats;
  return DOSA_ERR_UNSUPPORTED;
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
  if (!workspace) return DOSA_ERR_INVALID_ARG;
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
