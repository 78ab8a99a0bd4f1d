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
// holds MOE_NOALLOC_WORKSPACE_BYTES of it until the process exits.  Host code
// must not pass the variable's name to a kernel (on the host that name is only
// a stand-in); its device address is looked up with cudaGetSymbolAddress, with
// the device current, the first time a call runs in a CUDA context, and cached
// per context (keyed by the driver's unique context id, so that a caller's own
// context, or the primary context re-created after cudaDeviceReset, gets its
// own lookup).  Every call shares the one array, and it keeps the last call's
// contents; the forward clears its status word on every call and writes every
// other region before reading it, so nothing else needs clearing.  Two calls
// that overlap on the GPU (different streams, or different host threads) race
// on the array.
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_WORKSPACE_BYTES];

struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return f;
}

// Unique id of the calling thread's current CUDA context (0 if there is none
// yet, or the driver cannot say).
unsigned long long current_context_id() {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

constexpr int kCacheEntries = 64;
std::mutex g_mu;
struct Entry {
  unsigned long long ctx_id;
  void* ptr;
};
Entry g_cache[kCacheEntries] = {};
int g_next = 0;

int lookup_symbol(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr)
    return set_error(MOE_ERR_CUDA, "cudaGetSymbolAddress of the static scratch array failed");
  *out = p;
  return MOE_OK;
}

// Device address of g_noalloc_scratch in the calling thread's current context.
int scratch_address(void** out) {
  const unsigned long long id = current_context_id();
  if (id == 0) return lookup_symbol(out);  // no context id to key on: look it up every time
  std::lock_guard<std::mutex> lock(g_mu);
  for (const Entry& en : g_cache)
    if (en.ctx_id == id) {
      *out = en.ptr;
      return MOE_OK;
    }
  void* p = nullptr;
  const int rc = lookup_symbol(&p);
  if (rc != MOE_OK) return rc;
  g_cache[g_next] = Entry{id, p};
  g_next = (g_next + 1) % kCacheEntries;
  *out = p;
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

extern "C" int moe_noalloc_debug_status(void* stream) {
  void* ws = nullptr;
  const int rc = moe::scratch_address(&ws);
  if (rc != MOE_OK) return rc;
  return moe_debug_status(ws, stream);
}

extern "C" size_t moe_noalloc_workspace_bytes(void) { return (size_t)MOE_NOALLOC_WORKSPACE_BYTES; }
