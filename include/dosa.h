/*
 * dosa.h -- C ABI of libdosa, the B200 (sm_100a) DoSA certified indexer Top-K.
 *
 * The operation.  For a query row t with H indexer heads q[t,h] (head dim d),
 * signed head weights w[t,h] and keys k[s] shared by all heads, the indexer
 * score is
 *     I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]),     causal: s <= pos(t),
 * and the result is the K keys with the largest I (ties to the smaller key
 * index).  Source: "DOSA: Dots Sparse Attention", Daily Paper Cast transcript,
 * Method section (problem formulation: one query with several indexer heads,
 * each with its own query vector and weight, scored against shared keys; the
 * top K keys by score) and Experiments section (the dense baseline scores
 * every visible key and then selects the Top-K, K = 2048).  The certified
 * entry point returns
 * the same selection while scoring only the keys a certificate cannot reject
 * (same transcript, Method section: seed threshold, three bound stages,
 * candidate refinement per key tile; "Xiaohongshu DoSA sparse attention cuts
 * TTFT by up to 48% via score bounds", section 02: the original scoring
 * function is kept and every unrejected candidate is scored with all heads).
 *
 * Conventions shared by every entry point
 *  - Device pointers unless stated otherwise; the caller owns every buffer.
 *    The library allocates no device memory during a call: scratch space is
 *    the caller's workspace (size from dosa_index_workspace_size).
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = the
 *    legacy default stream) and is asynchronous unless a `stats` pointer is
 *    given, in which case the call synchronises `stream` to read counters.
 *  - Arguments are validated on the host before anything is launched.  A
 *    device-side bounded wait that expires, or a device bounds check that
 *    fires, is reported as DOSA_ERR_TIMEOUT / DOSA_ERR_DEVICE_CHECK by the
 *    call that reads it back (any call given `stats`, or dosa_check_device).
 *
 * Bit-identical selections.  Every scorer computes a score with the same
 * tensor-core dot products and the same fp32 head sum in the same order.  The
 * dense scorer sums w * ReLU(x) head by head; the other scorers sum
 * w * (x + |x|), which is exactly twice as much at every step, and halve the
 * total.  Doubling commutes with fp32 rounding as long as no partial sum is
 * subnormal (below 2^-126 in magnitude, zero excepted) or overflows, so the
 * certified, decode and dense selections are identical for weights and keys
 * of ordinary magnitude; a head sum whose partial sums reach the subnormal
 * range (for instance weights below about 2^-100) can round differently by
 * one unit in the last place and flip an exact tie at the K-th score.
 *
 * Layouts
 *  - q:       [Tq, H, d] row-major codes: bf16 (2 bytes) or OCP FP8 E4M3
 *             (1 byte).  Base 16-byte aligned.
 *  - q_scale: [Tq] fp32 per-token scales (E4M3 only; NULL for bf16).  The real
 *             query is q_scale[t] * decode(q[t,h,:]).
 *  - w:       [Tq, H] fp32.
 *  - k:       [S, d] row-major codes, same dtype as q.  Base 16-byte aligned.
 *  - k_scale: [S] fp32 per-token scales (E4M3 only; NULL for bf16).
 *  - seq_offsets: HOST array of (B+1) x 3 int64, a packed varlen batch.  Row b
 *             = {q_row_start[b], k_start[b], q_pos0[b]}; row B = {Tq, S, 0}.
 *             Sequence b owns query rows [q_row_start[b], q_row_start[b+1]) and
 *             keys [k_start[b], k_start[b+1]).  Its query row i sits at position
 *             q_pos0[b] + (i - q_row_start[b]) among its own keys and sees keys
 *             0..position (causal).  Requires position < number of its keys.
 *             (Chunked prefill: queries at an offset against a cached key
 *             prefix -- same transcript, Experiments section, chunks of 4K-32K.)
 *  - out_idx: [Tq, K] int32.  Per row: the selected key indices, relative to
 *             the sequence's first key, in ascending order; rows with fewer
 *             than K visible keys list all of them and pad with -1.
 */
#ifndef DOSA_H_
#define DOSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DOSA_OK = 0,
  DOSA_ERR_INVALID_ARG = 1,   /* a pointer, size, layout or alignment is wrong */
  DOSA_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. d != 128)           */
  DOSA_ERR_WORKSPACE = 3,     /* workspace smaller than dosa_index_workspace_size */
  DOSA_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, sync, ...) */
  DOSA_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired             */
  DOSA_ERR_DEVICE_CHECK = 6   /* a device-side bounds check fired               */
} dosa_status;

typedef enum { DOSA_BF16 = 0, DOSA_FP8_E4M3 = 1 } dosa_dtype;

/* Fixed at create time.  Defaults (dosa_index_config_default): H = 64, d = 128,
 * bf16, max_K = 2048, seed_first = 64, seed_last = 512, r = 4, G = 2,
 * margin_log2 = -12, screening = 2, sparse_writeback = 1, block_bound = 1,
 * probe_sample = 1. */
typedef struct {
  int H;            /* indexer heads per query: 64 or 32.  With 32 the kernels
                       read each query row into 64 head slots (the other 32
                       arrive as zeros) and reduce only the 32 real heads.   */
  int d;            /* head dimension (128 in this library)                     */
  dosa_dtype dtype; /* storage type of q and k                                  */
  int max_K;        /* largest K the handle will be called with (<= 4096)      */
  int seed_first;   /* seed subset: the first seed_first keys ...               */
  int seed_last;    /* ... and the last seed_last keys ending at the query      */
  int r;            /* retained positive heads evaluated exactly (0..4)         */
  int G;            /* negative-head groups (0 = no negative aggregate, 1, 2)   */
  int margin_log2;  /* soundness margin 2^margin_log2 * sum|w|||q|| * ||k||     */
  int screening;    /* How keys are screened after the warm-up (key tile 0 and
                       the tiles at the diagonal, scored exactly until K exact
                       scores exist).  3: ranked -- every remaining key of a
                       row is screened once against an estimate of a score a
                       little below its K-th (from the warm-up scores); the
                       survivors are gathered and scored with all heads, and
                       the estimate is then checked against the K-th reached:
                       a row where a rejected key's bound is not below it is
                       screened again over the band of bounds between them
                       (lower estimates, down to the warm-up threshold).
                       2 (default): adaptive -- each work item of 8 queries
                       is screened over 4 key tiles first and goes on with
                       ranked screening where that kept at most 1 in 4 of
                       1024 or more screened pairs; the others are scored
                       exactly without bounds.  1: the streaming schedule --
                       every tile is screened against the threshold reached
                       so far, tile after tile.  0: never (ablation).  The
                       selection is exact in every mode.                      */
  int sparse_writeback; /* 1 (default): only scores >= the running threshold
                       are written, as packed (score, key) candidates, and the
                       selection reads those; 0 (ablation): every exact score
                       is also written into a dense [rows, keys] matrix of the
                       chunk (rejected pairs as -inf) and the selection is the
                       dense Top-K of that matrix.  Same result either way.   */
  int block_bound;  /* screening = 1 only.  1 (default): before the certified
                       scorer resumes an item after its warm-up, every key
                       tile is bounded as a whole (a ball around the tile's
                       mean key) and tiles that can hold no Top-K key of the
                       item's queries are skipped without loading their keys;
                       0: off (ablation).                                     */
  int probe_sample;  /* screening = 2 only.  1 (default): every 7th work item
                       (on chunks of more than 1,792 items a larger prime
                       stride, about 256 items; longest rows first) is set
                       up and probed first; the
                       other items are set up and probed only if one of those
                       chose screening, and otherwise go to the filter scorer
                       straight after their warm-up.  0: every item is set up
                       and probed (ablation).  Same result either way.        */
  int short_dense_keys; /* screening = 2 only.  A dosa_index_topk call whose
                       sequences all have at most this many keys runs the dense
                       scorer and radix Top-K instead (the same selection:
                       every pair scored exactly, ties to the smaller index;
                       on short rows the certified path's set-up, warm-up and
                       probe launches cost more than they save).  Default
                       16384; 0: never.  Its stats count every visible pair as
                       exact and nothing as screened or filtered.               */
} dosa_index_config;

/* Counters of the last certified call (filled when `stats` is non-NULL). */
typedef struct {
  int64_t visible_pairs;   /* sum over rows of (position + 1)                        */
  int64_t seed_pairs;      /* pairs scored exactly as seeds                          */
  int64_t screened_pairs;  /* non-seed pairs whose bound was evaluated               */
  int64_t rejected_pairs;  /* screened pairs rejected (bound + margin < threshold)   */
  int64_t exact_pairs;     /* pairs scored with all heads (seeds + survivors)        */
  int64_t candidates;      /* (score, index) pairs written for the final selection   */
  int64_t filtered_pairs;  /* exact pairs scored by the filter scorer (no bounds)    */
  int64_t block_skipped_pairs; /* rejected pairs of key tiles skipped whole by the
                                  key-block certificate (keys never loaded)      */
  int64_t rescored_pairs;  /* exact pairs scored from gathered survivors (ranked)   */
  int64_t repaired_rows;   /* rows whose candidate list overflowed and were scored
                              again densely (a tie at the K-th score spanning
                              more keys than the list holds; at most 64 to 512
                              rows per chunk of rows, depending on S_max)       */
  int64_t rescreened_pairs; /* ranked screening: pairs the first pass rejected and
                               a later pass (a lower band of bounds) scored      */
} dosa_stats;

typedef struct dosa_index* dosa_index_t;

/* Fill *cfg with the defaults listed above. */
void dosa_index_config_default(dosa_index_config* cfg);

/* Validate cfg and create a handle (host memory only; it holds the config and
 * per-device kernel attributes).  Errors: INVALID_ARG for NULL or out-of-range
 * fields, UNSUPPORTED for d != 128 or H other than 32 or 64. */
dosa_status dosa_index_create(const dosa_index_config* cfg, dosa_index_t* out);

/* Free a handle (NULL is accepted). */
void dosa_index_destroy(dosa_index_t h);

/* Bytes of device workspace a call needs for a batch of Tq query rows, at most
 * S_max keys in one sequence, and K.  `certified` selects dosa_index_topk (1)
 * or dosa_index_dense_topk (0).  The dense path's workspace holds one chunk of
 * fp32 score rows; `chunk_rows` (0 = library choice) sets its height. */
dosa_status dosa_index_workspace_size(dosa_index_t h, int64_t Tq, int64_t S_max, int K,
                                      int certified, int64_t chunk_rows, size_t* bytes);

/* Certified Top-K (the DoSA pipeline): key prep, certificate setup, seed
 * scoring, bound screening, survivor rescoring with all heads, threshold
 * filtering with packed writeback, radix selection.  Returns exactly the
 * selection of dosa_index_dense_topk.  Workspace: dosa_index_workspace_size
 * with certified = 1. */
dosa_status dosa_index_topk(dosa_index_t h, const void* q, const float* q_scale, const float* w,
                            const void* k, const float* k_scale, const int64_t* seq_offsets,
                            int B, int K, int32_t* out_idx, void* workspace, size_t ws_bytes,
                            void* stream, dosa_stats* stats);

/* Certified Top-K with the inputs and the output in HOST memory (page-locked
 * for the copies to overlap the kernels; pageable memory works, serialised).
 * q, q_scale, w, k, k_scale, out_idx are host pointers with the layouts of
 * dosa_index_topk; seq_offsets as there.  The keys (and key scales) of every
 * sequence are copied first; then the query rows stream through two device
 * staging slots: while the kernels run on one chunk of rows, the next chunk's
 * q, q_scale and w are copied in and the previous chunk's indices copied out,
 * on a copy stream the handle creates on first use (per device).  The call is
 * asynchronous on `stream` like the others: out_idx is complete when `stream`
 * is; the host buffers must stay valid until then.  Same selection as
 * dosa_index_topk.  Workspace (device): dosa_index_host_workspace_size.
 * Errors as dosa_index_topk; DOSA_ERR_CUDA also when the copy stream cannot
 * be created. */
dosa_status dosa_index_topk_host(dosa_index_t h, const void* q, const float* q_scale,
                                 const float* w, const void* k, const float* k_scale,
                                 const int64_t* seq_offsets, int B, int K, int32_t* out_idx,
                                 void* workspace, size_t ws_bytes, void* stream,
                                 dosa_stats* stats);

/* Device workspace of dosa_index_topk_host for Tq query rows, S_total keys
 * over all sequences, at most S_max keys in one, and K; chunk_rows (0 =
 * library choice, 16384) is the number of query rows per staging slot.  A
 * call given less workspace than the default uses the most rows per slot
 * that fit (at least 8). */
dosa_status dosa_index_host_workspace_size(dosa_index_t h, int64_t Tq, int64_t S_total,
                                           int64_t S_max, int K, int64_t chunk_rows,
                                           size_t* bytes);

/* Decode-step Top-K: a few query rows per sequence (e.g. the next token, or a
 * handful of multi-token-prediction rows) against the sequence's cached keys,
 * seeded by the previous step's selection.  seed_idx: device [Tq, K] int32,
 * indices relative to each sequence's first key (the previous step's out_idx
 * for the same rows; -1 entries are ignored).  For each row the exact scores
 * of its seed keys, lowered by a rounding margin, give a lower bound tau0 of
 * its K-th largest score when the row has K distinct visible seeds; every
 * visible key is then scored on the tensor cores with the key range split
 * over all SMs, and only scores >= tau0 enter the selection.  Rows without K
 * distinct visible seeds, or whose candidates exceed the list capacity
 * (4 K, at least 4096), are rescored densely; at most 64 rows per sequence
 * can be (more: DOSA_ERR_DEVICE_CHECK).  Returns exactly the selection of
 * dosa_index_dense_topk.  Workspace: dosa_index_decode_workspace_size.
 * Errors: INVALID_ARG also for a NULL seed_idx. */
dosa_status dosa_index_decode_topk(dosa_index_t h, const void* q, const float* q_scale,
                                   const float* w, const void* k, const float* k_scale,
                                   const int64_t* seq_offsets, int B, int K,
                                   const int32_t* seed_idx, int32_t* out_idx, void* workspace,
                                   size_t ws_bytes, void* stream, dosa_stats* stats);

/* Device workspace of dosa_index_decode_topk for Tq query rows (all
 * sequences), at most S_max keys in one sequence, and K. */
dosa_status dosa_index_decode_workspace_size(dosa_index_t h, int64_t Tq, int64_t S_max, int K,
                                             size_t* bytes);

/* The per-query certificate the certified path screens with (for inspection
 * and tests; the Top-K calls compute it internally).  cert_out: [Tq, 16] fp32,
 * code domain (for E4M3 the real-valued bound is q_scale[t] * k_scale[s] times
 * the code-domain one): [0..3] folded weights omega of the retained heads,
 * [4] beta (coefficient of ||k||, including rounding slack and the hi/lo split
 * error of the negative aggregates), [5] c (the candidate margin is c * ||k||),
 * [6..9] scales of the negative-aggregate rows (u_1 hi, u_1 lo, u_2 hi, u_2 lo),
 * [10] the per-head residual sum, [11] the joint (spectral) residual bound,
 * [12] |A_1|, [13] |A_2|, [14] number of omitted positive heads, [15] unused.
 * retained_out: [Tq, 4] int32 retained head indices, ascending, -1 padded.
 * bound_out (nullable): [Tq, 8, d] codes in the input type, the bound rows the
 * screening multiplies with the keys: rows 0..3 the retained heads' query codes
 * (zero rows when fewer are retained), rows 4..7 the negative aggregates u_1
 * and u_2, each as a hi row and a lo row (u_g = scale[6+2g] * hi + scale[7+2g]
 * * lo, code domain).  With them and cert_out, the bound of every pair can be
 * rebuilt: UB = sum_j omega_j ReLU(row_j . k) + (beta + c) ||k|| -
 * sum_g ReLU(scale_hi row_hi . k + scale_lo row_lo . k).
 * Workspace: as dosa_index_topk (certified = 1, K = 1 is enough). */
dosa_status dosa_index_certificate(dosa_index_t h, const void* q, const float* q_scale,
                                   const float* w, const void* k, const float* k_scale,
                                   const int64_t* seq_offsets, int B, float* cert_out,
                                   int32_t* retained_out, void* bound_out, void* workspace,
                                   size_t ws_bytes, void* stream);

/* Dense Top-K: every visible key is scored with all heads (tensor-core scorer),
 * score rows are materialised chunk by chunk in the workspace, then a per-row
 * radix select picks the K largest.  The reference the certified path must
 * match bit for bit.  Workspace: certified = 0. */
dosa_status dosa_index_dense_topk(dosa_index_t h, const void* q, const float* q_scale,
                                  const float* w, const void* k, const float* k_scale,
                                  const int64_t* seq_offsets, int B, int K, int32_t* out_idx,
                                  void* workspace, size_t ws_bytes, void* stream);

/* Dense Top-K that allocates nothing and takes no workspace.  For callers
 * that cannot allocate device memory themselves -- for example code running
 * inside a host framework whose memory pool must not be bypassed, or a
 * latency-critical path where an allocation could block or fail.  The paper
 * has no counterpart; it is a deployment convenience.  Scratch space is a
 * fixed 16 MiB array compiled into the library (every GPU that loads the
 * library holds it until the process exits).  The first call on each device
 * looks up that array's device address; make the first call on a device
 * before any stream capture.  All calls share the array and it keeps the last
 * call's contents (the call clears the part that must start at zero), so calls
 * whose work overlaps on the GPU race on it: serialise them.  Sizes: returns
 * DOSA_ERR_WORKSPACE when 256 + 32 * S_max bytes exceed 16 MiB (S_max = the
 * largest key count of a sequence, so up to 524280 keys), before any CUDA
 * call.  Otherwise as dosa_index_dense_topk, with identical results.  A
 * device-side failure of the call (an expired bounded wait, a bounds check)
 * is recorded in the array's header, not returned: read it back with
 * dosa_check_device(NULL, stream) after the call, before the next static call
 * clears it. */
dosa_status dosa_index_dense_topk_static(dosa_index_t h, const void* q, const float* q_scale,
                                         const float* w, const void* k, const float* k_scale,
                                         const int64_t* seq_offsets, int B, int K,
                                         int32_t* out_idx, void* stream);

/* Dense scorer alone, for one sequence: scores[i * ld + s] = I(row0 + i, s) for
 * rows row0..row0+rows-1 of q (positions pos0 + i) and s = 0..position; other
 * entries are left untouched.  k points at the sequence's first key, S is its
 * key count.  `scratch` is 16 bytes of zeroed device memory (error word). */
dosa_status dosa_index_scores(dosa_index_t h, const void* q, const float* q_scale, const float* w,
                              const void* k, const float* k_scale, int64_t row0, int64_t rows,
                              int64_t pos0, int64_t S, float* scores, int64_t ld, void* scratch,
                              void* stream);

/* Plain CUDA-core scorer with the same contract as dosa_index_scores (fp32
 * FMAs, no tensor cores): a cross-check for the tensor-core path. */
dosa_status dosa_reference_scores(dosa_index_t h, const void* q, const float* q_scale,
                                  const float* w, const void* k, const float* k_scale,
                                  int64_t row0, int64_t rows, int64_t pos0, int64_t S,
                                  float* scores, int64_t ld, void* stream);

/* Per-row exact Top-K of fp32 score rows (radix select; ties to the smaller
 * index; -0.0 equals +0.0): row i has n_i = row_len[i] (device int64 array)
 * scores at scores + i * ld; out[i * K ...] as for out_idx.  NaN scores are
 * not allowed. */
dosa_status dosa_topk_rows(const float* scores, int64_t ld, const int64_t* row_len, int64_t rows,
                           int K, int32_t* out, void* stream);

/* Read back and clear the device error word of the last calls on `stream`
 * that used `workspace` (synchronises it).  workspace = NULL reads the error
 * word of dosa_index_dense_topk_static on the current device (the header of
 * the library's fixed scratch array).  Returns DOSA_ERR_TIMEOUT or
 * DOSA_ERR_DEVICE_CHECK for a recorded failure, DOSA_ERR_CUDA when the copy
 * fails, DOSA_OK otherwise. */
dosa_status dosa_check_device(void* workspace, void* stream);

/* Kernel kinds reported by the profiling counters. */
typedef enum {
  DOSA_KERNEL_SCORE = 0,       /* tensor-core scorer (dense scores)            */
  DOSA_KERNEL_TOPK = 1,        /* per-row radix select                         */
  DOSA_KERNEL_REFERENCE = 2,   /* CUDA-core reference scorer                   */
  DOSA_KERNEL_KEY_PREP = 3,    /* key norms and key mean                       */
  DOSA_KERNEL_CERT_SETUP = 4,  /* per-query certificate                        */
  DOSA_KERNEL_CERTIFIED = 5,   /* seed scoring, screening, rescoring, writeback */
  DOSA_KERNEL_SELECT = 6,      /* selection over the packed candidates         */
  DOSA_KERNEL_FILTER = 7,      /* exact scoring + threshold filter, no bounds  */
  DOSA_KERNEL_DECODE = 8,      /* decode step: seed bound, split-S scan        */
  DOSA_KERNEL_FILL = 9,        /* dense-writeback ablation: matrix set to -inf */
  DOSA_KERNEL_BLOCK = 10,      /* key-block certificate: block statistics and  */
                               /* per-item block screening                      */
  DOSA_KERNEL_RESCORE = 11,    /* rescoring of gathered survivors               */
  DOSA_KERNEL_RANK = 12,       /* ranked screening: estimates and bound passes  */
  DOSA_KERNEL_KINDS = 13
} dosa_kernel;

/* Kernel timing.  While enabled, every kernel a call launches is bracketed by
 * CUDA events recorded on the call's stream (host-side cost: two event records
 * per launch; the events are created once and reused).  dosa_profile_read
 * synchronises on the recorded events and returns, for one kernel kind, the
 * number of launches and their summed device time in milliseconds since the
 * last reset.  Enabling or resetting discards earlier records.  Not
 * thread-safe: profile from one host thread. */
dosa_status dosa_profile_enable(int on);
dosa_status dosa_profile_reset(void);
dosa_status dosa_profile_read(int kind, int64_t* launches, double* ms);

/* Static description of a status code. */
const char* dosa_status_string(dosa_status s);

#ifdef __cplusplus
}
#endif
#endif /* DOSA_H_ */
