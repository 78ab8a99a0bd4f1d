// noalloc.cu -- moe_forward_noalloc: the forward on scratch memory the library
// owns, for callers that cannot allocate device memory themselves.
//
// Some callers have no way to obtain device memory for a workspace: plugins
// running inside a host runtime that reserves all device memory up front and
// hands out no allocator, and request paths that must not call cudaMalloc
// because it can synchronise the device and take unbounded time.  For them
// this entry point runs the same forward on a fixed-size scratch array that is
// part of the library's device image.
//
// The array is a file-scope __device__ variable: every GPU that loads this code
// holds MOE_NOALLOC_WORKSPACE_BYTES of it until the process exits.  Its
// device address is looked up once per device with cudaGetSymbolAddress (host
// code must not pass the variable's name itself to a kernel: on the host that
// name is only a stand-in).  Every call shares the one array, and it keeps
// the last call's contents; the forward clears its status word on every call
// and writes every other region before reading it, so nothing else needs
// clearing.  Two calls that overlap on the GPU (different streams, or
// different host threads) race on the array.
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up on the
// first call made with that device current.
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return set_error(MOE_ERR_UNSUPPORTED, "device ordinal beyond 63");
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(MOE_ERR_CUDA, "cudaGetSymbolAddress of the static scratch array failed");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" int moe_forward_noalloc(const moe_shape* s, const moe_options* o, const moe_tensors* t,
                                   void* stream) {
  const size_t need = moe_workspace_size(s, o);
  if (need == 0)  // invalid arguments: report the validation error, launch nothing
    return moe::forward_on_workspace(s, o, t, nullptr, 0, stream);
  if (need > (size_t)MOE_NOALLOC_WORKSPACE_BYTES) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "moe_forward_noalloc: this problem needs %zu bytes of scratch, the static array holds %zu; "
             "use moe_forward with a caller workspace",
             need, (size_t)MOE_NOALLOC_WORKSPACE_BYTES);
    return moe::set_error(MOE_ERR_WORKSPACE, msg);
  }
  void* ws = nullptr;
  const int rc = moe::scratch_address(&ws);
  if (rc != MOE_OK) return rc;
  return moe::forward_on_workspace(s, o, t, ws, (size_t)MOE_NOALLOC_WORKSPACE_BYTES, stream);
}
