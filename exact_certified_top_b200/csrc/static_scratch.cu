// Dense Top-K with no device allocation anywhere: the scratch space is a
// fixed array compiled into the library instead of a caller workspace.
//
// Every GPU that loads the library holds kStaticScratchBytes for this array
// until the process exits.  In host code `g_static_scratch` is only a
// host-side stand-in for the device symbol; its device address is looked up
// once per device with cudaGetSymbolAddress (with that device current) and
// cached.  All calls share the one array, so calls whose work overlaps on the
// GPU (different streams, or different host threads) race on it.
#include <mutex>

#include "dosa_internal.h"

namespace dosa {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)16 << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_lock;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr when the runtime cannot provide it.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> g(g_lock);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    g_addr[dev] = p;
  }
  return g_addr[dev];
}

}  // namespace

// The static array's address on the current device (its header holds the
// device error word of the static calls), or nullptr.
void* static_scratch_address() { return scratch_address(); }

}  // namespace dosa

using namespace dosa;

extern "C" dosa_status dosa_index_dense_topk_static(dosa_index_t h, const void* q,
                                                    const float* q_scale, const float* w,
                                                    const void* k, const float* k_scale,
                                                    const int64_t* seq_offsets, int B, int K,
                                                    int32_t* out_idx, void* stream) {
  if (!h || !seq_offsets || B < 1) return DOSA_ERR_INVALID_ARG;
  // The dense path needs the header plus at least one row of fp32 scores per
  // key of the longest sequence (in practice a multiple of 8 rows).
  int64_t S_max = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t nk = seq_offsets[3 * (b + 1) + 1] - seq_offsets[3 * b + 1];
    if (nk > S_max) S_max = nk;
  }
  if (S_max < 0) return DOSA_ERR_INVALID_ARG;
  if ((size_t)kWsHeaderBytes + (size_t)S_max * 4 * kQueryTile > kStaticScratchBytes)
    return DOSA_ERR_WORKSPACE;
  void* ws = scratch_address();
  if (!ws) return DOSA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The header holds the device error word, which must start at zero; the
  // score rows are fully rewritten by every call.
  if (cudaMemsetAsync(ws, 0, kWsHeaderBytes, s) != cudaSuccess) return DOSA_ERR_CUDA;
  return dosa_index_dense_topk(h, q, q_scale, w, k, k_scale, seq_offsets, B, K, out_idx, ws,
                               kStaticScratchBytes, stream);
}
