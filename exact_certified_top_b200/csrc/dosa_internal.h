// Internal interfaces between the C-ABI layer (dosa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dosa.h"

namespace dosa {

constexpr int kHeadDim = 128;     // d
constexpr int kKeyTile = 128;     // keys per MMA tile (M)
constexpr int kQueryTile = 8;     // queries resident per scorer work item

// Workspace header: word 0 = device error word, then counters.
struct WsHeader {
  int error;
  int pad0;
  unsigned long long counters[15];   // see CounterId
};
enum CounterId : int {
  kCntSeedPairs = 0,
  kCntScreened = 1,
  kCntRejected = 2,
  kCntExact = 3,
  kCntCandidates = 4,
  kCntOverflow = 5,
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
};

struct Handle {
  dosa_index_config cfg;
};

// Kernel timing hooks (profile.cu): bracket one launch with events when enabled.
void profile_before(int kind, cudaStream_t stream);
void profile_after(int kind, cudaStream_t stream);

// Tensor-map encoder from the driver (fetched once through the runtime).
PFN_cuTensorMapEncodeTiled_v12000 get_tensor_map_encoder();

// ---- launches (each returns the cudaError_t of its launch) --------------------
// Tensor-core scorer writing every visible score of rows [row0, row0+rows).
cudaError_t launch_scores_tc(const Handle& h, const SeqView& v, float* scores, int64_t ld,
                             int* err, cudaStream_t stream);
// CUDA-core reference scorer, same contract.
cudaError_t launch_scores_ref(const Handle& h, const SeqView& v, float* scores, int64_t ld,
                              cudaStream_t stream);
// Per-row radix Top-K.  Row i has n_i = row_len ? row_len[i] : (len0 + i) entries
// (clipped to max_len).
cudaError_t launch_topk_rows(const float* scores, int64_t ld, const int64_t* row_len,
                             int64_t len0, int64_t max_len, int64_t rows, int K, int32_t* out,
                             int64_t out_ld, cudaStream_t stream);

}  // namespace dosa
