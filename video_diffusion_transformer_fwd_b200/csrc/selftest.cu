// Self-test of the bounded-wait path: a kernel waits on an mbarrier that no
// one arrives on; the wait gives up after its time limit, records a code in
// the watchdog word and the kernel returns normally (no trap), so the host
// can observe WAN_ETIMEOUT through wan_device_status with the context intact.
#include "common.cuh"
#include "sm100.cuh"

namespace wan {
namespace {

__global__ void watchdog_probe_kernel(int *watchdog) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: nothing arrives on this barrier
    sm100::mbar_wait(sm100::smem_u32(&bar), 0, &abort_flag, watchdog, 0x7e57);
  }
  __syncthreads();
}

}  // namespace
}  // namespace wan

using namespace wan;

extern "C" int wan_selftest_watchdog(wan_stream_t stream) {
  int *wd = watchdog_ptr();
  if (!wd) return set_error(WAN_ECUDA, "watchdog symbol unavailable");
  watchdog_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(wd);
  WAN_CHECK_LAUNCH("watchdog_probe");
  return WAN_OK;
}
