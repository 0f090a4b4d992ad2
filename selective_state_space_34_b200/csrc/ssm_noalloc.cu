// ssm_noalloc.cu -- ssm_scan_bwd_noalloc: the backward pass with its scratch memory built into the
// library instead of supplied by the caller.
//
// Who this is for: callers that cannot allocate device memory themselves -- a plain C or plugin
// host program that is only ever handed device pointers and has no allocator of its own, or code
// running where allocating is not allowed or not safe (for example while another framework's
// caching allocator owns the device's free memory). ssm_scan_bwd asks such callers for a
// workspace they have no way to provide; this entry point needs nothing beyond the inputs and the
// gradient outputs.
//
// How: the scratch is one file-scope __device__ array of SSM_NOALLOC_SCRATCH_BYTES. Every GPU on
// which the library is loaded holds that array until the process exits. Host code cannot pass the
// array's name to a kernel (on the host it only names a stand-in symbol, not a device address), so
// the first call on each device looks up the array's device address with cudaGetSymbolAddress
// while that device is current, checks the result, and caches it per device; later calls reuse it.
// That first-call set-up makes a runtime API call, so make the first call on a device before any
// stream capture. All calls on a device share the one array and it keeps whatever the previous
// call left in it: the backward overwrites every scratch byte it later reads, so nothing needs
// clearing, but two calls whose work overlaps on the GPU (different streams, no ordering between
// them) race on the array and give wrong gradients. Order them on one stream or with events.
#include <mutex>

#include "ssm_internal.h"

namespace {

__device__ __align__(256) unsigned char g_bwd_scratch[SSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

}  // namespace

extern "C" {

ssm_status ssm_scan_bwd_noalloc(const ssm_bwd_args *args, void *stream) {
  if (!args) return SSM_ERR_NULL;
  // The smallest thread-block cluster whose scratch fits the array: clusters of 4 or 8 CTAs add
  // their dB / dC partial sums on chip, dividing that (largest) part of the scratch by 4 or 8 for
  // a slightly slower kernel. Problems that fit with none of them are rejected before anything
  // touches the device.
  int cluster = 0;
  for (int c : {1, 4, 8})
    if (ssm::bwd_workspace_for(args, c) <= (size_t)SSM_NOALLOC_SCRATCH_BYTES) {
      cluster = c;
      break;
    }
  if (!cluster) return SSM_ERR_WORKSPACE;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (ssm_status)ssm::record_cuda_error_code(e);
  if (dev < 0 || dev >= kMaxDevices) return SSM_ERR_UNSUPPORTED;  // beyond the address cache
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_bwd_scratch);
      if (e == cudaSuccess && p == nullptr) e = cudaErrorInvalidSymbol;
      if (e != cudaSuccess) return (ssm_status)ssm::record_cuda_error_code(e);
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  ssm_bwd_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = (size_t)SSM_NOALLOC_SCRATCH_BYTES;
  return ssm::scan_bwd_clustered(&a, stream, cluster);
}

}  // extern "C"
