// wan_block_forward_noalloc: the block forward for callers that cannot hand
// the library a device workspace. The workspace lives in a fixed-size array
// in the library's own device memory, so neither the caller nor the library
// allocates anything per call.
//
// Facts a caller should know:
//  - The array has WAN_NOALLOC_WORKSPACE_BYTES bytes on every GPU that loads
//    the library, held until the process exits. Problems whose workspace
//    (wan_block_workspace_bytes) is larger are rejected with WAN_EINVAL.
//  - Its device address is looked up on every call made while the stream is
//    not capturing (a device reset moves the array, so a remembered address
//    could go stale); the first call with a given device current must come
//    before any stream capture, since a call made during a capture can only
//    use the address found by an earlier call.
//  - Every call on a device uses the same array and it keeps the previous
//    call's contents. The block forward writes every workspace byte it later
//    reads, so nothing needs clearing between calls, but two calls that can
//    overlap on the GPU (different streams without ordering) race on it.
#include "common.cuh"

#include <mutex>

namespace wan {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_workspace[WAN_NOALLOC_WORKSPACE_BYTES];

// Device address of g_noalloc_workspace for the current device. In host code
// the array's name is only a host-side stand-in; the address a kernel can use
// comes from cudaGetSymbolAddress, asked again on every call outside a stream
// capture and remembered per device for calls made during one.
int noalloc_workspace(cudaStream_t stream, void **out) {
  static void *addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  WAN_TRY_CUDA(cudaGetDevice(&dev), "wan_block_forward_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 64) return set_error(WAN_EUNSUPPORTED, "wan_block_forward_noalloc: device %d", dev);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    cs = cudaStreamCaptureStatusActive;      // cannot tell: do not call into the runtime's module state
  }
  std::lock_guard<std::mutex> lk(mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
    if (e != cudaSuccess) return cuda_error(e, "wan_block_forward_noalloc: cudaGetSymbolAddress");
    addr[dev] = p;
  } else if (!addr[dev]) {
    return set_error(WAN_EINVAL, "wan_block_forward_noalloc: the first call on device %d was made during a "
                                 "stream capture; make one call before capturing", dev);
  }
  *out = addr[dev];
  return WAN_OK;
}

}  // namespace
}  // namespace wan

using namespace wan;

extern "C" int wan_block_forward_noalloc(const wan_dims *dims, int B, float *x, const void *ctx,
                                         const int *ctx_lens, const float *e0,
                                         const wan_block_weights *w, const float *rope,
                                         int rope_max_pos, wan_stream_t stream) {
  const size_t need = dims && B > 0 ? wan_block_workspace_bytes(dims, B) : 0;
  // an empty call or invalid dims: the workspace entry point validates them
  // and returns the same status and message (it launches nothing)
  if (need == 0) return wan_block_forward(dims, B, x, ctx, ctx_lens, e0, w, rope, rope_max_pos, nullptr, 0, stream);
  if (need > (size_t)WAN_NOALLOC_WORKSPACE_BYTES)
    return set_error(WAN_EINVAL,
                     "wan_block_forward_noalloc: this problem needs %zu bytes of workspace, more than "
                     "the built-in %zu-byte array; call wan_block_forward with a workspace instead",
                     need, (size_t)WAN_NOALLOC_WORKSPACE_BYTES);
  void *ws = nullptr;
  const int rc = noalloc_workspace((cudaStream_t)stream, &ws);
  if (rc) return rc;
  return wan_block_forward(dims, B, x, ctx, ctx_lens, e0, w, rope, rope_max_pos, ws,
                           (size_t)WAN_NOALLOC_WORKSPACE_BYTES, stream);
}
