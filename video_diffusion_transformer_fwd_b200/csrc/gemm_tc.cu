// placeholder, replaced by the tcgen05 GEMM
#include "common.cuh"
namespace wan {
bool gemm_tc_supported(const GemmArgs &) { return false; }
int gemm_tc(const GemmArgs &, cudaStream_t) { return set_error(WAN_EUNSUPPORTED, "gemm_tc"); }
}
