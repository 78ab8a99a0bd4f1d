// ep.cuh -- device pieces of the expert-parallel building blocks (moe_permute):
// kept out of the headers the grouped GEMMs include.
#pragma once

#include "common.cuh"

namespace moe {

// row_expert[r] = the expert of routed row r (rows of expert e are off[e] .. off[e+1]-1),
// taken modulo experts_per_rank when that is positive (the expert's index on the rank
// that holds it).
cudaError_t launch_row_expert(const int32_t* off, int E, int R, int experts_per_rank, int32_t* row_expert,
                              cudaStream_t st);

}  // namespace moe
