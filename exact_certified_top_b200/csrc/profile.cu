// Opt-in kernel timing: CUDA events around each launch, summed per kernel kind.
#include <vector>

#include "dosa_internal.h"

namespace dosa {
namespace {

struct Record {
  int kind;
  cudaEvent_t start, stop;
};

bool g_enabled = false;
std::vector<Record> g_records;        // in launch order
std::vector<cudaEvent_t> g_pool;      // reusable events
cudaEvent_t g_pending = nullptr;      // start event of the launch in progress
int g_pending_kind = -1;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void recycle_all() {
  for (const Record& r : g_records) {
    g_pool.push_back(r.start);
    g_pool.push_back(r.stop);
  }
  g_records.clear();
  if (g_pending) g_pool.push_back(g_pending);
  g_pending = nullptr;
}

}  // namespace

void profile_before(int kind, cudaStream_t stream) {
  if (!g_enabled) return;
  g_pending = take_event();
  g_pending_kind = kind;
  if (g_pending) cudaEventRecord(g_pending, stream);
}

void profile_after(int kind, cudaStream_t stream) {
  if (!g_enabled || !g_pending || g_pending_kind != kind) return;
  cudaEvent_t stop = take_event();
  if (!stop) return;
  cudaEventRecord(stop, stream);
  g_records.push_back({kind, g_pending, stop});
  g_pending = nullptr;
}

}  // namespace dosa

using namespace dosa;

extern "C" {

dosa_status dosa_profile_enable(int on) {
  recycle_all();
  g_enabled = on != 0;
  return DOSA_OK;
}

dosa_status dosa_profile_reset(void) {
  recycle_all();
  return DOSA_OK;
}

dosa_status dosa_profile_read(int kind, int64_t* launches, double* ms) {
  if (kind < 0 || kind >= DOSA_KERNEL_KINDS || !launches || !ms) return DOSA_ERR_INVALID_ARG;
  int64_t n = 0;
  double total = 0.0;
  for (const Record& r : g_records) {
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return DOSA_ERR_CUDA;
    float e = 0.f;
    if (cudaEventElapsedTime(&e, r.start, r.stop) != cudaSuccess) return DOSA_ERR_CUDA;
    ++n;
    total += e;
  }
  *launches = n;
  *ms = total;
  return DOSA_OK;
}

}  // extern "C"
