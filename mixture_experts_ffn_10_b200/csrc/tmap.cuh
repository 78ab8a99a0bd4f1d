// tmap.cuh -- host-side TMA tensor-map encoding and the device-side tile walk
// shared by the grouped GEMM kernels.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point.
// dims[0] is the innermost extent (elements), strides are in bytes for dims 1..rank-1.
bool encode_tiled(CUtensorMap* m, CUtensorMapDataType dtype, int rank, const void* base,
                  const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                  CUtensorMapSwizzle swizzle);

// One tile of a grouped GEMM: segment, first row inside the segment, N block,
// and the segment's row count.  Tiles are numbered segment-major, then N block,
// then M block (fastest), from the device-side prefix `tiles` [NS + 1] over the
// segments' visiting positions (segment order, or GemmCommon::order).
struct Tile {
  int seg, m0, n_blk, rows;
};

template <int BM>
__device__ __forceinline__ Tile decode_tile(const GemmCommon& c, int tile) {
  int lo = 0, hi = c.NS - 1;  // last visiting position p with tiles[p] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.tiles[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  Tile t;
  t.seg = c.order ? c.order[lo] : lo;
  t.rows = c.cnt[t.seg];
  const int mt = (t.rows + BM - 1) / BM;
  const int local = tile - c.tiles[lo];
  t.n_blk = local / mt;
  t.m0 = (local % mt) * BM;
  return t;
}

}  // namespace moe
