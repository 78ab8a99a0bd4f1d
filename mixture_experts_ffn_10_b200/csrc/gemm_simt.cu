// gemm_simt.cu -- fp32 grouped GEMMs on CUDA cores (FFMA), for fp32 problems.
//
// TF32 tensor cores keep 10 mantissa bits, too few for a 1e-4 relative bound,
// so fp32 problems run here.  Same segment/tile walk as the tensor-core path:
//   gate_up: h[row, f] = gated(W_gate[e] . z_row + b_gate, W_up[e] . z_row + b_up)
//   down:    Y[row, o] = (W_down[e] . h_row + b_down[o]) * w_row
// (graph-op page: fc1 [E, 2*inter, hidden], fc2 [E, hidden, inter]; "Struct
// MoeSpec" biases, act, weigh_inputs).  Rows of segment s are off[s].., the
// shared expert (segment E) reads x directly and has weight 1.
#include "common.cuh"

namespace moe {
namespace {

constexpr int BM = kSimtBM;  // 64 rows
constexpr int BK = 16;
constexpr int kGuFeat = 32;  // gate_up: 32 features -> 64 weight rows per tile
constexpr int kDnFeat = 64;  // down: 64 output features per tile

struct TileInfo {
  int seg, m0, n_blk, rows;
};

__device__ __forceinline__ bool find_tile(const GemmCommon& c, int tile, TileInfo* ti) {
  const int total = tile_total(c);
  if (tile >= total) return false;
  int lo = 0, hi = c.NS - 1;  // last s with tiles[s] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.tiles[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  const int rows = c.cnt[lo];
  const int mt = (rows + BM - 1) / BM;
  const int local = tile - c.tiles[lo];
  ti->seg = lo;
  ti->rows = rows;
  ti->n_blk = local / mt;
  ti->m0 = (local % mt) * BM;
  return true;
}

__global__ void __launch_bounds__(256) simt_gate_up_kernel(SimtArgs a) {
  pdl_enter();
  const GemmCommon& c = a.c;
  TileInfo ti;
  if (!find_tile(c, blockIdx.x, &ti)) return;
  const bool shared = ti.seg >= c.E;
  const int K = c.d;
  const int F = shared ? c.Fs : c.F;
  // plain FFN: the 64 weight rows of a tile are 64 features of fc1 (columns of accg
  // are features f0 + 2tx + j, of accu features f0 + 32 + 2tx + j); gated: 32 gate
  // rows and their 32 up rows
  const bool plain = c.ffn == MOE_FFN_PLAIN;
  const bool unfused = !shared && !plain && c.gu_layout == MOE_GU_UNFUSED;
  const int layout = (shared && c.gu_layout == MOE_GU_UNFUSED) ? MOE_GU_CONCAT : c.gu_layout;
  const GuRows gr = gu_rows(layout, F);
  const int64_t stack_rows = (plain || unfused) ? F : 2 * F;   // rows of one expert's gate_up stack
  const float* W = shared ? a.sh_gate_up : a.gate_up + (int64_t)ti.seg * stack_rows * c.d;
  const float* WG = unfused ? a.gate + (int64_t)ti.seg * F * c.d : W;   // the gate rows' stack
  const float* bias = (!shared && a.gate_up_bias) ? a.gate_up_bias + (int64_t)ti.seg * stack_rows : nullptr;
  const float* gbias = unfused ? (a.gate_bias ? a.gate_bias + (int64_t)ti.seg * F : nullptr) : bias;
  const int row_base = c.off[ti.seg];
  const int f0 = ti.n_blk * kGuFeat * (plain ? 2 : 1);

  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][2 * kGuFeat + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float accg[4][2], accu[4][2];
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 2; j++) accg[i][j] = accu[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int q = threadIdx.x; q < BM * BK; q += 256) {
      const int r = q / BK, kk = q % BK;
      const int row = ti.m0 + r, k = k0 + kk;
      float v = 0.f;
      if (row < ti.rows && k < K)
        v = shared ? a.x[(int64_t)row * K + k] : a.xg[(int64_t)(row_base + row) * K + k];
      As[kk][r] = v;
    }
    for (int q = threadIdx.x; q < 2 * kGuFeat * BK; q += 256) {
      const int r = q / BK, kk = q % BK;  // r < 32: gate feature r; else up feature r - 32
      const int f = plain ? f0 + r : f0 + (r & (kGuFeat - 1));
      const int k = k0 + kk;
      float v = 0.f;
      if (f < F && k < K) {
        if (plain) v = W[(int64_t)f * K + k];
        else if (r < kGuFeat) v = WG[(gr.gate0 + (int64_t)gr.stride * f) * K + k];
        else v = W[(gr.up0 + (int64_t)gr.stride * f) * K + k];
      }
      Bs[kk][r] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; kk++) {
      float av[4];
#pragma unroll
      for (int i = 0; i < 4; i++) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 2; j++) {
        const float bg = Bs[kk][tx * 2 + j], bu = Bs[kk][kGuFeat + tx * 2 + j];
#pragma unroll
        for (int i = 0; i < 4; i++) {
          accg[i][j] = fmaf(av[i], bg, accg[i][j]);
          accu[i][j] = fmaf(av[i], bu, accu[i][j]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int row = ti.m0 + ty * 4 + i;
    if (row >= ti.rows) continue;
#pragma unroll
    for (int j = 0; j < 2; j++) {
      float* hrow = a.h + (int64_t)(row_base + row) * c.Fmax;
      if (plain) {
        const int fa = f0 + tx * 2 + j, fb = fa + kGuFeat;
        if (fa < F) hrow[fa] = plain_act(c.act, accg[i][j] + (bias ? bias[fa] : 0.f));
        if (fb < F) hrow[fb] = plain_act(c.act, accu[i][j] + (bias ? bias[fb] : 0.f));
        continue;
      }
      const int f = f0 + tx * 2 + j;
      if (f >= F) continue;
      float g = accg[i][j], u = accu[i][j];
      if (gbias) g += gbias[gr.gate0 + (int64_t)gr.stride * f];
      if (bias) u += bias[gr.up0 + (int64_t)gr.stride * f];
      hrow[f] = gated_act(c.act, g, u);
    }
  }
}

__global__ void __launch_bounds__(256) simt_down_kernel(SimtArgs a) {
  pdl_enter();
  const GemmCommon& c = a.c;
  TileInfo ti;
  if (!find_tile(c, blockIdx.x, &ti)) return;
  const bool shared = ti.seg >= c.E;
  const int K = shared ? c.Fs : c.F;
  const int N = c.d;
  const float* W = shared ? a.sh_down : a.down + (int64_t)ti.seg * c.d * c.F;
  const float* bias = (!shared && a.down_bias) ? a.down_bias + (int64_t)ti.seg * c.d : nullptr;
  const int row_base = c.off[ti.seg];
  const int n0 = ti.n_blk * kDnFeat;

  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][kDnFeat + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 4; j++) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int q = threadIdx.x; q < BM * BK; q += 256) {
      const int r = q / BK, kk = q % BK;
      const int row = ti.m0 + r, k = k0 + kk;
      As[kk][r] = (row < ti.rows && k < K) ? a.h[(int64_t)(row_base + row) * c.Fmax + k] : 0.f;
    }
    for (int q = threadIdx.x; q < kDnFeat * BK; q += 256) {
      const int r = q / BK, kk = q % BK;
      const int o = n0 + r, k = k0 + kk;
      Bs[kk][r] = (o < N && k < K) ? W[(int64_t)o * K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; kk++) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; i++) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; j++) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int row = ti.m0 + ty * 4 + i;
    if (row >= ti.rows) continue;
    const int64_t grow = row_base + row;
    const float w = (!shared && !c.weigh_inputs) ? a.roww[grow] : 1.f;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int o = n0 + tx * 4 + j;
      if (o >= N) continue;
      float v = acc[i][j];
      if (bias) v += bias[o];
      a.Y[grow * N + o] = v * w;
    }
  }
}

}  // namespace

cudaError_t launch_simt_gate_up(const SimtArgs& a, cudaStream_t st) {
  if (a.c.max_tiles == 0) return cudaSuccess;
  return launch_pdl(simt_gate_up_kernel, (unsigned)a.c.max_tiles, 256, 0, st, a);
}

cudaError_t launch_simt_down(const SimtArgs& a, cudaStream_t st) {
  if (a.c.max_tiles == 0) return cudaSuccess;
  return launch_pdl(simt_down_kernel, (unsigned)a.c.max_tiles, 256, 0, st, a);
}

}  // namespace moe
