// sort.cu -- expert histogram, exclusive scans and the stable token permutation
// that turns the routing [T, k] into expert-contiguous rows, and the gather of
// the input rows into that order.
//
// Rows of expert e are offsets[e] .. offsets[e+1]-1, token-ascending; the shared
// expert (when present) is segment E with one row per token at R + t.  The same
// pass computes, per GEMM, the prefix of tiles per segment that the grouped
// GEMMs walk on the device (no host round trip).
#include "sort.cuh"

namespace moe {
namespace {

using namespace sorting;

// Per-chunk expert histogram: hist[b][e] = #(t in chunk b, j) with idx[t][j] == e.
// Also clears the GEMMs' counters (SortArgs::sync).
__global__ void __launch_bounds__(256) hist_kernel(SortArgs a) {
  pdl_enter();
  extern __shared__ int32_t sh[];
  const int b = blockIdx.x;
  for (int i = b * blockDim.x + threadIdx.x; i < a.n_sync; i += gridDim.x * blockDim.x) a.sync[i] = 0;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) sh[e] = 0;
  __syncthreads();
  const int t0 = b * kChunkTokens;
  const int t1 = min(a.T, t0 + kChunkTokens);
  for (int n = threadIdx.x; n < (t1 - t0) * a.k; n += blockDim.x) {
    const int e = a.idx[(int64_t)t0 * a.k + n];
    if (e >= 0 && e < a.E) atomicAdd(&sh[e], 1);
    else set_status(a.status, MOE_ERR_SHAPE);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.hist[(int64_t)b * a.E + e] = sh[e];
}

// One block of 1024 threads: per-expert chunk prefixes, segment offsets, tile prefixes.
__global__ void __launch_bounds__(1024) scan_kernel(SortArgs a) {
  __shared__ int32_t cnt[kMaxE + 1];
  __shared__ int32_t tg[kMaxE + 1];
  __shared__ int32_t td[kMaxE + 1];
  __shared__ int32_t ord[kMaxE + 1];
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t tot;
  pdl_enter();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int32_t run = 0;
    for (int b = 0; b < a.nchunks; b++) {
      int32_t* p = &a.hist[(int64_t)b * a.E + e];
      const int32_t h = *p;
      *p = run;
      run += h;
    }
    cnt[e] = run;
  }
  segment_scan<2>(a, cnt, tg, td, warp_tot, &tot, ord);
}

// The whole sort for a single chunk of tokens (T <= kChunkTokens) in one block:
// histogram in shared memory, the segment scan, and the in-order scatter (and the
// GEMMs' counters cleared).
__global__ void __launch_bounds__(1024) sort_one_chunk_kernel(SortArgs a) {
  __shared__ int32_t cnt[kMaxE + 1];
  __shared__ int32_t tg[kMaxE + 1];
  __shared__ int32_t td[kMaxE + 1];
  __shared__ int32_t run[kMaxE];
  __shared__ int32_t ord[kMaxE + 1];
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t tot;
  pdl_enter();
  for (int i = threadIdx.x; i < a.n_sync; i += blockDim.x) a.sync[i] = 0;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    cnt[e] = 0;
    run[e] = 0;
  }
  __syncthreads();
  const int n_ent = a.T * a.k;
  for (int n = threadIdx.x; n < n_ent; n += blockDim.x) {
    const int e = a.idx[n];
    if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
    else set_status(a.status, MOE_ERR_SHAPE);
  }
  __syncthreads();
  segment_scan<2>(a, cnt, tg, td, warp_tot, &tot, ord);
  __syncthreads();
  if (threadIdx.x < 32) scatter_chunk(a, 0, n_ent, cnt, nullptr, run);
}

// One warp per chunk walks its (t, j) entries in order, so rows inside an expert
// stay token-ascending: row = off[e] + (earlier chunks) + (earlier in this chunk).
constexpr int kScatterWarps = 4;
__global__ void __launch_bounds__(kScatterWarps * 32) scatter_kernel(SortArgs a) {
  extern __shared__ int32_t run_all[];  // [kScatterWarps][E]
  pdl_enter();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int b = blockIdx.x * kScatterWarps + wid;
  int32_t* run = run_all + wid * a.E;
  for (int e = lane; e < a.E; e += 32) run[e] = 0;
  __syncwarp();
  if (b >= a.nchunks) return;
  const int t0 = b * kChunkTokens;
  scatter_chunk(a, t0, (min(a.T, t0 + kChunkTokens) - t0) * a.k, a.off, a.hist + (int64_t)b * a.E, run);
}

// xg[pos[t, j]] = x[t] (times the row's routing weight for weigh-inputs), token
// by token, so that x is read once and written k times: one warp per token and
// slice of its row (slice blockIdx.y of gridDim.y; more than one only when there
// are too few tokens to fill the GPU), 16-byte vectors.
template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= a.T) return;
  constexpr int kVec = 16 / sizeof(T);
  const int nv = a.d / kVec;
  const int per = (nv + gridDim.y - 1) / gridDim.y;
  const int v0 = blockIdx.y * per, v1 = min(nv, v0 + per);
  const uint4* src = reinterpret_cast<const uint4*>((const T*)a.x + t * a.d);
  // each lane holds the row and weight of slot (lane mod k); shuffled to every lane
  int my_row = 0;
  float my_w = 1.f;
  if (lane < a.k) {
    my_row = a.pos[t * a.k + lane];
    if (my_row < 0 || my_row >= a.R) {
      set_status(a.status, MOE_ERR_SHAPE);
      my_row = -1;
    } else if (a.weigh_inputs) {
      my_w = a.roww[my_row];
    }
  }
  if (__any_sync(0xffffffffu, my_row < 0)) return;
  // four vectors per lane in flight: loads first, then the k (scaled) stores of each;
  // every lane runs every iteration (the shuffles below need the whole warp)
  constexpr int kBatch = 4;
  for (int vb = v0; vb < v1; vb += 32 * kBatch) {
    const int v = vb + lane;
    uint4 q[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; b++)
      if (v + 32 * b < v1) q[b] = __ldg(src + v + 32 * b);
    for (int j = 0; j < a.k; j++) {
      const int row = __shfl_sync(0xffffffffu, my_row, j);
      const float w = __shfl_sync(0xffffffffu, my_w, j);
      uint4* dst = reinterpret_cast<uint4*>((T*)a.xg + (int64_t)row * a.d);
#pragma unroll
      for (int b = 0; b < kBatch; b++) {
        if (v + 32 * b >= v1) break;
        uint4 o = q[b];
        if (a.weigh_inputs) {
          if constexpr (sizeof(T) == 2) {
            uint32_t* u = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int i = 0; i < 4; i++) {
              const float lo = bf16_to_f32(u[i] & 0xffff) * w, hi = bf16_to_f32(u[i] >> 16) * w;
              u[i] = pack_bf16x2(lo, hi);
            }
          } else {
            float* f = reinterpret_cast<float*>(&o);
#pragma unroll
            for (int i = 0; i < 4; i++) f[i] *= w;
          }
        }
        dst[v + 32 * b] = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_sort(const SortArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (a.nchunks == 1) {  // small batches: one launch instead of three
    // as few threads as the segment scan needs (two segments per thread): its block
    // barriers are the kernel's latency
    int threads = ((a.NS + 1) / 2 + 31) / 32 * 32;
    threads = threads < 128 ? 128 : (threads > 1024 ? 1024 : threads);
    return launch_pdl(sort_one_chunk_kernel, 1, threads, 0, st, a);
  }
  cudaError_t e = launch_pdl(hist_kernel, (unsigned)a.nchunks, 256, a.E * sizeof(int32_t), st, a);
  if (e == cudaSuccess) e = launch_pdl(scan_kernel, 1, 1024, 0, st, a);
  const int blocks = (a.nchunks + kScatterWarps - 1) / kScatterWarps;
  if (e == cudaSuccess)
    e = launch_pdl(scatter_kernel, (unsigned)blocks, kScatterWarps * 32, kScatterWarps * a.E * sizeof(int32_t), st, a);
  return e;
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t st) {
  if (a.R == 0) return cudaSuccess;
  const int blocks = (a.T + 7) / 8;
  // few tokens: split each row into slices of at least 32 vectors until ~512 blocks
  const int nv = a.d / (a.bf16 ? 8 : 4);
  int slices = 1;
  while (blocks * slices * 2 <= 512 && nv / (slices * 2) >= 32) slices *= 2;
  const dim3 grid(blocks, slices);
  if (a.bf16) return launch_pdl(gather_kernel<uint16_t>, grid, 256, 0, st, a);
  return launch_pdl(gather_kernel<float>, grid, 256, 0, st, a);
}

}  // namespace moe
