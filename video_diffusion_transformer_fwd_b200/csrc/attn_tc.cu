// placeholder, replaced by the tcgen05 flash attention
#include "common.cuh"
namespace wan {
bool attention_tc_supported(const AttnArgs &) { return false; }
int attention_tc(const AttnArgs &, cudaStream_t) { return set_error(WAN_EUNSUPPORTED, "attention_tc"); }
}
