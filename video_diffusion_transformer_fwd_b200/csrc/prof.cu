// Launch instrumentation: while enabled, every kernel launch of the library
// is bracketed by a pair of CUDA events recorded on the launching stream, so
// the caller can read per-kernel-class device time of a region of work.
#include "common.cuh"

#include <mutex>
#include <vector>

namespace wan {

namespace {
struct Entry {
  cudaEvent_t a, b;
  int cls;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Entry> g_pool;
size_t g_used = 0;
constexpr size_t MAX_ENTRIES = 1 << 16;
}  // namespace

ProfScope::ProfScope(int cls, cudaStream_t s) : idx(-1), stream(s) {
  if (!g_on) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_used >= MAX_ENTRIES) return;
  if (g_used == g_pool.size()) {
    Entry e{nullptr, nullptr, cls};
    if (cudaEventCreate(&e.a) != cudaSuccess || cudaEventCreate(&e.b) != cudaSuccess) return;
    g_pool.push_back(e);
  }
  g_pool[g_used].cls = cls;
  if (cudaEventRecord(g_pool[g_used].a, s) != cudaSuccess) return;
  idx = (int)g_used++;
}

ProfScope::~ProfScope() {
  if (idx < 0) return;
  cudaEventRecord(g_pool[idx].b, stream);
}

}  // namespace wan

using namespace wan;

extern "C" {

int wan_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = on != 0;
  g_used = 0;
  return WAN_OK;
}

int wan_profile_read(int kernel_class, int *launches, double *total_ms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (kernel_class < 0 || kernel_class >= WAN_K_COUNT || !launches || !total_ms)
    return set_error(WAN_EINVAL, "wan_profile_read: bad arguments");
  int n = 0;
  double ms = 0.0;
  for (size_t i = 0; i < g_used; ++i) {
    if (g_pool[i].cls != kernel_class) continue;
    WAN_TRY_CUDA(cudaEventSynchronize(g_pool[i].b), "profile event synchronize");
    float t = 0.f;
    WAN_TRY_CUDA(cudaEventElapsedTime(&t, g_pool[i].a, g_pool[i].b), "profile elapsed time");
    ms += t;
    ++n;
  }
  *launches = n;
  *total_ms = ms;
  return WAN_OK;
}

}  // extern "C"
