// gdn_frame_fwd_noalloc: gdn_frame_fwd for callers that cannot allocate device
// memory (no cudaMalloc, no allocator of their own to carve a workspace from).
//
// Such callers exist: a plugin or custom operator loaded into a host program
// that owns every device allocation and hands the plugin only its input and
// output buffers, or a runtime with a static, pre-planned memory layout that
// forbids any allocation after start-up.  They can pass q, k, v, gates, states
// and o, but not the scratch that the frame chain needs (ticket counter, frame
// flags, published frame states).  This entry point supplies that scratch from
// a fixed-size array in the library's own device memory instead.
//
// The array lives for as long as the library is loaded, on every GPU that
// loads it (GDN_NOALLOC_SCRATCH_BYTES of device memory each).  All calls share
// it: calls whose executions overlap on the GPU (different streams, or
// different host threads without ordering) race on it and must not be made.
// The part that has to start at zero (counter and flags) is cleared by every
// call, on the call's stream, before the kernel runs.
#include <atomic>

#include "launch.h"

namespace gdn {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
std::atomic<void *> g_scratch_addr[kMaxDev];

// Device address of g_noalloc_scratch on the current device.  The host-side
// name is only a stand-in, so kernels must be given this address, never
// &g_noalloc_scratch.  The address is looked up with the device current on
// every call made outside stream capture (after a device reset the runtime
// loads the module again, possibly elsewhere, so a cached address could be
// stale) and remembered per device for calls made while `st` is being
// captured, which do not look it up; so the first call on a device must come
// before any capture.
int scratch_address(cudaStream_t st, void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return GDN_ERR_NO_DEVICE;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return GDN_ERR_CUDA;
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (cs == cudaStreamCaptureStatusNone) {
    void *fresh = nullptr;
    if (cudaGetSymbolAddress(&fresh, g_noalloc_scratch) != cudaSuccess || fresh == nullptr) return GDN_ERR_CUDA;
    if (fresh != p) g_scratch_addr[dev].store(fresh, std::memory_order_release);
    p = fresh;
  } else if (p == nullptr) {
    return GDN_ERR_INVALID_ARG;  // first call on this device inside a capture: not supported
  }
  *out = p;
  return GDN_OK;
}

}  // namespace
}  // namespace gdn

extern "C" int gdn_frame_fwd_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                                     const float *beta, const float *state_in, float *state_out, float *o, int B,
                                     int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_workspace_bytes(GDN_OP_GDN, B, H, F, L, dk, dv, opts);
  if (need > (size_t)GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  const int rc = gdn::scratch_address((cudaStream_t)opts->stream, &scratch);
  if (rc != GDN_OK) return rc;
  gdn_opts_t o2 = *opts;
  o2.workspace = scratch;
  o2.workspace_bytes = (size_t)GDN_NOALLOC_SCRATCH_BYTES;
  return gdn_frame_fwd(q, k, v, alpha, beta, state_in, state_out, o, B, H, F, L, dk, dv, &o2);
}
