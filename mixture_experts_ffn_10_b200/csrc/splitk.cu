// splitk.cu -- split-K for the bf16 tensor-core GEMMs when they have fewer tiles
// than SMs (small token counts: every SM should stream weights).
//
// The GEMM writes each split's fp32 partial accumulators; these kernels add the
// splits in split order (so the result does not depend on timing) and apply the
// same epilogues as the unsplit GEMM: bias + gated activation -> h (gate_up), or
// (bias + sum) x routing weight -> Y (down).
#include "epilogue.cuh"

namespace moe {
namespace {

__device__ __forceinline__ int segment_of(const GemmCommon& c, int row) {
  int lo = 0, hi = c.NS - 1;  // last segment whose first row is <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.off[mid] <= row) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// One block per (row, 128 features); thread = feature.
__global__ void __launch_bounds__(128) reduce_gate_up_kernel(TcArgs a) {
  pdl_enter();
  const GemmCommon& c = a.c;
  const int row = blockIdx.x;
  const int f = blockIdx.y * 128 + threadIdx.x;
  const int seg = segment_of(c, row);
  const bool sh = seg >= c.E;
  const int F = sh ? c.Fs : c.F;
  if (f >= F) return;
  const int rows = c.R + (c.Fs > 0 ? c.T : 0);
  uint16_t* out = reinterpret_cast<uint16_t*>(a.h) + (int64_t)row * c.Fmax + f;
  // weigh-inputs on x read in place (direct_x): W (w x) = w (W x)
  const float wi = (!sh && c.direct_x && c.weigh_inputs) ? a.roww[row] : 1.f;
  if (c.ffn == MOE_FFN_PLAIN) {  // tile columns are features: column f
    float v = 0.f;
    for (int sp = 0; sp < c.splits; sp++) v += c.partial[((int64_t)sp * rows + row) * c.partial_pitch + f];
    v *= wi;
    if (!sh && a.gate_up_bias) v += bf16_to_f32(((const uint16_t*)a.gate_up_bias)[(int64_t)seg * c.F + f]);
    *out = f32_to_bf16_rn(plain_act_bf16(c.act, v));
    return;
  }
  // gated: a tile of 128 features holds the gate values in columns 0..127 and the
  // up values in 128..255
  const int64_t col = (int64_t)(f / 128) * 256 + (f % 128);
  float g = 0.f, u = 0.f;
  for (int sp = 0; sp < c.splits; sp++) {
    const float* pr = c.partial + ((int64_t)sp * rows + row) * c.partial_pitch;
    g += pr[col];
    u += pr[col + 128];
  }
  g *= wi;
  u *= wi;
  if (!sh) {
    const GuBias gb = gu_bias(c.gu_layout, c.F, seg, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias);
    if (gb.g) g += bf16_to_f32(gb.g[(int64_t)gb.stride * f]);
    if (gb.u) u += bf16_to_f32(gb.u[(int64_t)gb.stride * f]);
  }
  *out = f32_to_bf16_rn(gated_act_bf16(c.act, g, u));
}

// One block per (row, 256 outputs); thread = output feature.
__global__ void __launch_bounds__(256) reduce_down_kernel(TcArgs a) {
  pdl_enter();
  const GemmCommon& c = a.c;
  const int row = blockIdx.x;
  const int o = blockIdx.y * 256 + threadIdx.x;
  if (o >= c.d) return;
  const int seg = segment_of(c, row);
  const bool sh = seg >= c.E;
  const int rows = c.R + (c.Fs > 0 ? c.T : 0);
  float v = 0.f;
  for (int sp = 0; sp < c.splits; sp++) v += c.partial[((int64_t)sp * rows + row) * c.partial_pitch + o];
  const uint16_t* bias = (!sh && a.down_bias) ? (const uint16_t*)a.down_bias + (int64_t)seg * c.d : nullptr;
  if (bias) v += bf16_to_f32(bias[o]);
  const float w = (sh || c.weigh_inputs) ? 1.f : a.roww[row];
  reinterpret_cast<uint16_t*>(a.Y)[(int64_t)row * c.d + o] = f32_to_bf16_rn(v * w);
}

}  // namespace

// Cost of a split factor in 64-deep K steps per CTA: the waves of work units
// times (K steps per unit + kUnitOverhead for a unit's pipeline fill and
// epilogue), plus kReduceCost for the reduction kernel when S > 1.
constexpr int64_t kUnitOverhead = 2;
constexpr int64_t kReduceCost = 4;

int choose_splits(int64_t tiles, int nkb, int sms) {
  if (tiles <= 0 || tiles >= sms) return 1;
  int best = 1;
  int64_t best_cost = ((tiles + sms - 1) / sms) * (nkb + kUnitOverhead);
  for (int s = 2; s <= 8 && 2 * s <= nkb; s++) {
    const int64_t cost = ((tiles * s + sms - 1) / sms) * ((nkb + s - 1) / s + kUnitOverhead) + kReduceCost;
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_splitk_gate_up_reduce(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  const int rows = c.R + (c.Fs > 0 ? c.T : 0);
  if (rows == 0) return cudaSuccess;
  const dim3 grid(rows, (c.Fmax + 127) / 128);
  return launch_pdl(reduce_gate_up_kernel, grid, 128, 0, st, a);
}

cudaError_t launch_splitk_down_reduce(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  const int rows = c.R + (c.Fs > 0 ? c.T : 0);
  if (rows == 0) return cudaSuccess;
  const dim3 grid(rows, (c.d + 255) / 256);
  return launch_pdl(reduce_down_kernel, grid, 256, 0, st, a);
}

}  // namespace moe
