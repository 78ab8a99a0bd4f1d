// ep.cu -- the expert of each routed row, for the expert-parallel exchange: rows in
// expert order travel to the rank that holds their expert together with its index
// there (experts split over devices; given the routing, each expert's rows are
// independent of the others').
#include "ep.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) row_expert_kernel(const int32_t* off, int E, int R, int per_rank,
                                                           int32_t* out) {
  pdl_enter();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  int lo = 0, hi = E - 1;  // last expert e with off[e] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  out[r] = per_rank > 0 ? lo % per_rank : lo;
}

}  // namespace

cudaError_t launch_row_expert(const int32_t* off, int E, int R, int experts_per_rank, int32_t* row_expert,
                              cudaStream_t st) {
  if (R == 0) return cudaSuccess;
  return launch_pdl(row_expert_kernel, dim3((R + 255) / 256), dim3(256), 0, st, off, E, R, experts_per_rank,
                    row_expert);
}

}  // namespace moe
