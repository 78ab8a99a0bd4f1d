// sort.cuh -- block-level pieces of the expert sort used by the sort kernels: a
// block-wide exclusive scan, the segment scan (offsets and per-GEMM tile
// prefixes), and the stable in-order scatter of one chunk of (token, slot) entries.
#pragma once

#include "common.cuh"

namespace moe {
namespace sorting {

// Block-wide exclusive scan of up to 1024 * kItems values held in shared memory.
template <int kItems>
__device__ void block_exclusive_scan(int32_t* v, int n, int32_t* total, int32_t* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  int32_t loc[kItems];
  int32_t run = 0;
#pragma unroll
  for (int i = 0; i < kItems; i++) {
    const int idx = tid * kItems + i;
    loc[i] = idx < n ? v[idx] : 0;
    run += loc[i];
  }
  int32_t incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int nw = blockDim.x >> 5;
    int32_t wv = lane < nw ? warp_tot[lane] : 0, wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < nw) warp_tot[lane] = wi - wv;
    if (lane == nw - 1) *total = wi;
  }
  __syncthreads();
  int32_t base = warp_tot[wid] + incl - run;
#pragma unroll
  for (int i = 0; i < kItems; i++) {
    const int idx = tid * kItems + i;
    if (idx < n) v[idx] = base;
    base += loc[i];
  }
  __syncthreads();
}

// Segment offsets and per-GEMM tile prefixes from the per-expert row counts in
// cnt[0..E) (shared memory; one block).  Leaves the segments'
// first rows (exclusive prefix) in cnt.
//
// With a.order set, the GEMMs visit the segments in an interleaved order: by rows,
// the largest first, each followed by the smallest one left (order[p] = segment at
// position p; the tile prefixes follow the positions).  Tiles of experts with few
// rows stream their weights from memory while those of large experts keep the
// tensor cores busy, so that SMs working at the same time mix the two.
template <int kItems>  // blockDim.x * kItems >= NS
__device__ void segment_scan(const SortArgs& a, int32_t* cnt, int32_t* tg, int32_t* td, int32_t* warp_tot,
                             int32_t* tot, int32_t* ord) {
  if (threadIdx.x == 0 && a.NS > a.E) cnt[a.E] = a.shared_rows;
  __syncthreads();
  for (int s = threadIdx.x; s < a.NS; s += blockDim.x) {
    const bool sh = s >= a.E;
    const int32_t mt = (cnt[s] + a.bm - 1) / a.bm;
    a.cnt[s] = cnt[s];
    tg[s] = mt * (sh ? a.nt_gu_shared : a.nt_gu_routed);
    td[s] = mt * (sh ? a.nt_dn_shared : a.nt_dn_routed);
  }
  __syncthreads();
  if (a.order) {
    // rank by rows (descending, ties to the lower segment), then interleave the ranks
    for (int s = threadIdx.x; s < a.NS; s += blockDim.x) {
      const int32_t cs = cnt[s];
      int rank = 0;
      for (int q = 0; q < a.NS; q++) {
        const int32_t cq = cnt[q];
        rank += (cq > cs || (cq == cs && q < s)) ? 1 : 0;
      }
      const int h = (a.NS + 1) / 2;
      const int pos = rank < h ? 2 * rank : 2 * (a.NS - 1 - rank) + 1;
      ord[pos] = s;
      a.order[pos] = s;
    }
    __syncthreads();
    int32_t g[kItems], dd[kItems];
#pragma unroll
    for (int i = 0; i < kItems; i++) {
      const int pos = threadIdx.x + i * blockDim.x;
      g[i] = pos < a.NS ? tg[ord[pos]] : 0;
      dd[i] = pos < a.NS ? td[ord[pos]] : 0;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kItems; i++) {
      const int pos = threadIdx.x + i * blockDim.x;
      if (pos < a.NS) {
        tg[pos] = g[i];
        td[pos] = dd[i];
      }
    }
    __syncthreads();
  }
  block_exclusive_scan<kItems>(cnt, a.NS, tot, warp_tot);
  for (int s = threadIdx.x; s < a.NS; s += blockDim.x) a.off[s] = cnt[s];
  if (threadIdx.x == 0) {
    a.off[a.NS] = *tot;
    if (*tot != a.R + a.shared_rows) set_status(a.status, MOE_ERR_SHAPE);
  }
  __syncthreads();
  block_exclusive_scan<kItems>(tg, a.NS, tot, warp_tot);
  for (int s = threadIdx.x; s < a.NS; s += blockDim.x) a.tile_gu[s] = tg[s];
  if (threadIdx.x == 0) a.tile_gu[a.NS] = *tot;
  __syncthreads();
  block_exclusive_scan<kItems>(td, a.NS, tot, warp_tot);
  for (int s = threadIdx.x; s < a.NS; s += blockDim.x) a.tile_dn[s] = td[s];
  if (threadIdx.x == 0) a.tile_dn[a.NS] = *tot;
}

// Stable in-order placement of the (t, j) entries n0 .. n0 + n_ent - 1 of one chunk by
// one warp: row = first row of the expert + `before` (rows of earlier chunks, or null)
// + run (earlier entries of this chunk; run[] zeroed, in shared memory).
__device__ inline void scatter_chunk(const SortArgs& a, int t0, int n_ent, const int32_t* first_row,
                              const int32_t* before, int32_t* run) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < n_ent; base += 32) {
    const int n = base + lane;
    const bool valid = n < n_ent;
    const int64_t slot = (int64_t)t0 * a.k + n;
    int e = valid ? a.idx[slot] : -1;
    if (e < 0 || e >= a.E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    if (e >= 0) {
      const int32_t row = first_row[e] + (before ? before[e] : 0) + run[e] + rank;
      if (row >= 0 && row < a.R) {
        const int t = t0 + n / a.k;
        a.pos[slot] = row;
        a.perm[row] = t;
        a.roww[row] = a.w[slot];
      } else {
        set_status(a.status, MOE_ERR_SHAPE);
      }
    }
    __syncwarp();
    if (e >= 0 && rank == 0) run[e] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace sorting
}  // namespace moe
