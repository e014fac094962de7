// Internal interfaces between the C-ABI layer (dosa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "dosa.h"

namespace dosa {

constexpr int kHeadDim = 128;     // d
constexpr int kKeyTile = 128;     // keys per MMA tile (M)
constexpr int kQueryTile = 8;     // queries resident per scorer work item

// Workspace header: word 0 = device error word, then counters.
struct WsHeader {
  int error;
  int probe_gate;        // the sampled probe found an item worth screening
  unsigned long long counters[15];   // see CounterId
};
enum CounterId : int {
  kCntSeedPairs = 0,
  kCntScreened = 1,
  kCntRejected = 2,
  kCntExact = 3,
  kCntCandidates = 4,
  kCntOverflow = 5,
  kCntFiltered = 6,
  kCntBlockSkipped = 7,
  kCntRescored = 8,
  kCntBandPairs = 9,       // survivors of the later ranked passes (rejected by pass 1)
};
constexpr size_t kWsHeaderBytes = 256;

// One sequence's slice of a call.
struct SeqView {
  const void* q;          // q rows of the whole call (row index = absolute row)
  const float* q_scale;
  const float* w;
  const void* k;          // the sequence's first key
  const float* k_scale;   // the sequence's first key scale
  int64_t row0;           // first query row handled
  int64_t rows;           // number of rows
  int64_t pos0;           // position of row0 among the sequence's keys
  int64_t S;              // keys of the sequence
  int H;                  // heads per query row: 32 or 64
};

struct Handle {
  dosa_index_config cfg;
  // Host-staged calls: a copy stream and staging events, created on first use
  // on the device current at that time (per device).
  int copy_device = -1;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ev_loaded[2] = {nullptr, nullptr};
  cudaEvent_t ev_done[2] = {nullptr, nullptr};
  cudaEvent_t ev_keys = nullptr, ev_out = nullptr;
  std::mutex copy_mutex;
};

// Device address of the allocation-free entry point's fixed scratch array on
// the current device (static_scratch.cu), or nullptr.
void* static_scratch_address();

// Kernel timing hooks (profile.cu): bracket one launch with events when enabled.
void profile_before(int kind, cudaStream_t stream);
void profile_after(int kind, cudaStream_t stream);

// Tensor-map encoder from the driver (fetched once through the runtime).
PFN_cuTensorMapEncodeTiled_v12000 get_tensor_map_encoder();
// 2-D map over `rows` rows of d = 128 elements (bf16 or fp8 codes), 128-byte
// swizzle, boxes of one 128-byte row segment x box_rows rows (score_tc.cu).
// Queries as a 3-D tensor [rows][H][d] read in boxes of 4 rows x 64 head
// slots x one 128-byte row: with H = 32 the slots 32..63 lie outside the
// tensor and arrive as zeros, so every kernel sees 64 heads per row.
bool encode_q_map(CUtensorMap* map, const void* q, bool fp8, uint64_t rows, int H,
                  int box_rows = 4);
bool encode_rows_map(CUtensorMap* map, const void* base, bool fp8, uint64_t rows,
                     uint32_t box_rows);

// Device buffers of one certified chunk (all inside the caller's workspace).
struct CertBuffers {
  float* key_norm;       // [S] code-domain ||k|| (rounded up)
  float* key_sum;        // [d] real-domain key sum
  void* bdir;            // [rows, 8, d] bound rows in the input type
  float* cert;           // [rows, kCertFloats]
  int32_t* retained;     // [rows, 4]
  void* cand;            // [rows][4][seg_cap] packed (score, key), 4 segments per row
  int* cand_count;       // [rows][4] per-segment counts; -1 marks a row repaired densely
  float* tau;            // [rows] final threshold
  void* qstate;          // [rows] candidate state carried from the probe pass
  int* item_flag;        // [rows / 8] what the probe pass decided per work item
  int* repair_list;      // [repair_cap]
  int* repair_count;
  int repair_cap;
  float* repair_scores;  // [repair_cap, S]
  int seg_cap;           // entries per candidate segment
  float* dense;          // [rows, dense_ld] every exact score (dense writeback), or null
  int64_t dense_ld;
  float* blk;            // [key tiles][kBlkFloats] key-block balls, or null (no block bound)
  int* step_list;        // [rows / 8 + 1][step_cap] steps left after block screening
  int* step_count;       // [rows / 8 + 1]
  int step_cap;
  // ranked screening (rank_screen.cu, rescore.cu)
  uint32_t* bits;        // [rows][words] survivor bits of the current pass
  int64_t words;         // 32-bit words per row: 4 per key tile of S_max
  float* est;            // [rows][kRankEst] descending threshold estimates
  float* band_lo;        // [rows] the current pass keeps lo <= v < hi
  float* band_hi;
  uint32_t* maxrej;      // [rows] ordered largest bound the current pass rejected
  int* row_next;         // [rows] the pass a row waits for (0: done or not ranked)
  int* pass_any;         // [kRankEst + 2] some row waits for pass j
  unsigned long long* rank_cnt;   // [rows / 8 + 1][2] probe: screened, kept pairs per item
  int* gate;             // set by the probe when a sampled item chose screening
  int probe_sample;      // the chunk's set-up covered only the sampled items
  unsigned long long* counters;
  int* err;
};

// Device buffers of a decode call (all inside the caller's workspace; per-row
// arrays start at the sequence's first row).
struct DecodeBuffers {
  uint32_t* bitmap;      // [rows][words] seed de-duplication, zero on entry
  int64_t words;
  uint32_t* tau_key;     // [rows] ordered seed bound, 0xFFFFFFFF on entry
  uint32_t* smax_key;    // [rows] ordered largest seed score, zero on entry
  int* seed_count;       // [rows] zero on entry
  int* dup;              // [rows] zero on entry
  int* count;            // [rows] candidates appended, zero on entry
  unsigned* hist;        // [rows][256] shared score histogram, zero on entry
  uint32_t* tau_run;     // [rows] ordered shared threshold, zero on entry
  int* cand_count;       // [rows][4] for the selection kernel
  float* tau;            // [rows]
  void* cand;            // [rows][cap] packed (score, key)
  int cap;               // >= every row's visible keys, a multiple of 64
  unsigned long long* counters;
  int* err;
};

// ---- launches (each returns the cudaError_t of its launch) --------------------
// Tensor-core scorer writing every visible score of rows [row0, row0+rows).
cudaError_t launch_scores_tc(const Handle& h, const SeqView& v, float* scores, int64_t ld,
                             int* err, cudaStream_t stream);
// Same scorer over a device list of rows (row0 + row_list[i] -> output row i).
cudaError_t launch_scores_tc_rows(const Handle& h, const SeqView& v, const int* row_list,
                                  const int* row_count, int list_cap, float* scores, int64_t ld,
                                  int* err, cudaStream_t stream);
// Certified pipeline pieces.
cudaError_t launch_key_prep(const Handle& h, const void* k, const float* k_scale, int64_t S,
                            float* key_norm, float* key_sum, cudaStream_t stream);
// sample 0: every row of the chunk; 1: the rows of the sampled work items
// (every probe_stride(n_items)-th), whose item_flag becomes kItemSample; 2: the
// other rows, only when *gate is set (a no-op launch otherwise).
cudaError_t launch_cert_setup(const Handle& h, const SeqView& v, const float* key_sum,
                              void* bdir, float* cert, int32_t* retained, cudaStream_t stream,
                              int sample = 0, int* item_flag = nullptr,
                              const int* gate = nullptr);
// After the sampled probe: items still unflagged become kItemProbe when *gate
// is set (they are set up and probed next), kItemUnprobed otherwise.
cudaError_t launch_probe_resolve(int* item_flag, int n_items, const int* gate,
                                 cudaStream_t stream);
// Key-block balls of a sequence: per key tile of 128 keys the real-domain
// center, radius and largest norm (kBlkFloats floats per tile).
constexpr int kBlkFloats = 132;
cudaError_t launch_block_prep(const Handle& h, const void* k, const float* k_scale, int64_t S,
                              float* blk, cudaStream_t stream);
// The steps of every work item one launch processes: [begin, min(end,
// n_tiles)) for the items whose probe flag equals want_flag (every item when
// want_flag < 0).  Step 0 is key tile 0, step i >= 1 is key tile n_tiles - i.
// A range that starts after step 0 resumes the state the previous launch
// saved; a range that ends before the item's last step saves it again.  When
// alt_flag > 0, the items flagged alt_flag are processed too, from alt_begin.
struct StepRange {
  int begin, end, want_flag;
  int alt_flag, alt_begin;
};
// Key-block screening of a range: per work item, the steps of `steps` whose key
// tile cannot hold a Top-K key of any of the item's queries (block bound +
// margin below the carried threshold) are dropped; the rest go to
// b.step_list / b.step_count (the range's last step is always kept).
cudaError_t launch_block_screen(const Handle& h, const SeqView& v, const CertBuffers& b,
                                StepRange steps, cudaStream_t stream);
// Certified scorer (the streaming schedule) over a range of steps.  use_list
// = 1: each item processes b.step_list instead of the whole range.
cudaError_t launch_certified(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                             StepRange steps, cudaStream_t stream, int use_list = 0);

// ---- ranked screening (rank_screen.cu, rescore.cu) ----------------------------
constexpr int kRankRows = 32;          // query rows per bound unit (N = 32 x 8 = 256)
constexpr int kRankUnitTiles = 64;     // key tiles per bound unit, at most
constexpr int kRankEst = 5;            // threshold estimates per row (m, 8m, ..., K)
constexpr int kRankProbeTiles = 4;     // key tiles per item the probe screens
// The probe keeps an item on ranked screening when it screened at least
// kRankMinScreened pairs and kept at most 1 in kRankKeepRatio of them.
constexpr unsigned long long kRankMinScreened = 1024;
constexpr unsigned long long kRankKeepRatio = 4;
// One pass of ranked screening: pass 1 keeps v >= the row's first estimate,
// pass j > 1 the band the previous rescoring chose.  Key tiles [jlo, jhi) of
// an item with L = n_tiles - W + 1 screened tiles [1, L): jhi = L - lo_off,
// jlo = hi_off > 0 ? L - hi_off : 1 (the probe: hi_off = kRankProbeTiles; the
// rest after it: lo_off = kRankProbeTiles).  Rows: those with
// row_next == pass, of the items whose flag equals `want` (all when
// item_sel is null).
struct RankPass {
  int pass;
  int lo_off, hi_off;
  const int* item_sel;
  int want;
  unsigned long long* item_cnt;   // probe counts per item, or null
};
// Threshold estimates from each selected row's warm-up histogram; the rows
// then wait for pass 1.
cudaError_t launch_rank_prep(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                             int W, const int* item_sel, int want, cudaStream_t stream);
// The bound pass: survivor bits, per-row largest rejected bound, counters.
cudaError_t launch_rank_screen(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                               int W, const RankPass& rp, cudaStream_t stream);
// Rescoring of the pass's survivors; rows are published or given the next band.
cudaError_t launch_rescore(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                           int W, const RankPass& rp, cudaStream_t stream);
// After the probe: items flagged `want` become kItemRank (raising *gate and
// adding their probe counts to the call's counters) or kItemFilter.
cudaError_t launch_rank_decide(int* item_flag, const unsigned long long* item_cnt, int n_items,
                               int want, int* gate, unsigned long long* counters,
                               cudaStream_t stream);
// Filter scorer (exact scores, threshold filter, no bounds) over a range.
cudaError_t launch_filter(const Handle& h, const SeqView& v, const CertBuffers& b, int K,
                          StepRange steps, cudaStream_t stream);
// Decode step: seed bound, split-S scan, per-row counts and repair list.
cudaError_t launch_decode(const Handle& h, const SeqView& v, const DecodeBuffers& b, int K,
                          const int32_t* seed, cudaStream_t stream);
// Bytes of carried candidate state per query row.
size_t qstate_bytes();
cudaError_t launch_select(const CertBuffers& b, int64_t rows, int64_t pos0, int K, int32_t* out,
                          cudaStream_t stream);
cudaError_t launch_topk_list(const float* scores, int64_t ld, const int* row_list,
                             const int* row_count, int list_cap, int64_t len0, int64_t max_len,
                             int K, int32_t* out, int64_t out_ld, cudaStream_t stream);
size_t certified_smem_bytes(bool fp8);
// CUDA-core reference scorer, same contract.
cudaError_t launch_scores_ref(const Handle& h, const SeqView& v, float* scores, int64_t ld,
                              cudaStream_t stream);
// p[0..n) = v.
cudaError_t launch_fill(float* p, int64_t n, float v, cudaStream_t stream);
// Per-row radix Top-K.  Row i has n_i = row_len ? row_len[i] : (len0 + i) entries
// (clipped to max_len).
cudaError_t launch_topk_rows(const float* scores, int64_t ld, const int64_t* row_len,
                             int64_t len0, int64_t max_len, int64_t rows, int K, int32_t* out,
                             int64_t out_ld, cudaStream_t stream);

}  // namespace dosa
