// route.cu -- routing kernel: one warp per token picks k of E experts and their
// weights ("Struct MoeSpec" score, selection_bias, groups, renormalize, scale; the
// per-token steps and their definitions are in route.cuh).
#include "route.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

template <int EPL>
__global__ void __launch_bounds__(kWarps * 32) route_kernel(RouteArgs a) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= a.T) return;
  routing::route_token<EPL>(a, t, lane);
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const dim3 grid((a.T + kWarps - 1) / kWarps), block(kWarps * 32);
  const int epl = (a.E + 31) / 32;
  if (epl <= 1) return launch_pdl(route_kernel<1>, grid, block, 0, st, a);
  if (epl <= 2) return launch_pdl(route_kernel<2>, grid, block, 0, st, a);
  if (epl <= 4) return launch_pdl(route_kernel<4>, grid, block, 0, st, a);
  if (epl <= 8) return launch_pdl(route_kernel<8>, grid, block, 0, st, a);
  if (epl <= 16) return launch_pdl(route_kernel<16>, grid, block, 0, st, a);
  return launch_pdl(route_kernel<32>, grid, block, 0, st, a);
}

}  // namespace moe
