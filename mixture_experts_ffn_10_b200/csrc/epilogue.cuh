// epilogue.cuh -- per-chunk epilogues of the tensor-core grouped GEMMs: 16
// accumulator columns of one row -> bias, gated activation or routing weight ->
// 16 bf16 outputs.  Shared by the bf16 and the MXFP4 kernels.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Gated activation for bf16 outputs.  sigmoid(x) = 0.5 + 0.5 tanh(x / 2) with the
// hardware tanh (relative error ~5e-4, well under the 2^-8 of the bf16 result);
// GELU-tanh uses the same instruction, GELU-erf the library erff.
__device__ __forceinline__ float gated_act_bf16(const ActParams& a, float g, float u) {
  float v;
  switch (a.act) {
    case MOE_ACT_SILU:
      if (a.limit > 0.f) {
        g = fminf(g, a.limit);
        u = fminf(fmaxf(u, -a.limit), a.limit);
      }
      v = g * fmaf(0.5f, tanh_fast(0.5f * a.alpha * g), 0.5f);
      break;
    case MOE_ACT_GELU_ERF: v = 0.5f * g * (1.f + erff(g * 0.70710678118654752f)); break;
    case MOE_ACT_GELU_TANH: {
      const float c = 0.79788456080286536f;  // sqrt(2/pi)
      v = 0.5f * g * (1.f + tanh_fast(c * fmaf(0.044715f * g, g * g, g)));
      break;
    }
    case MOE_ACT_RELU: v = fmaxf(g, 0.f); break;
    default: v = g; break;
  }
  return v * (u + a.beta);
}

// Non-gated activation for bf16 outputs (same instructions as gated_act_bf16).
__device__ __forceinline__ float plain_act_bf16(const ActParams& a, float g) {
  switch (a.act) {
    case MOE_ACT_SILU: return g * fmaf(0.5f, tanh_fast(0.5f * a.alpha * g), 0.5f);
    case MOE_ACT_GELU_ERF: return 0.5f * g * (1.f + erff(g * 0.70710678118654752f));
    case MOE_ACT_GELU_TANH: {
      const float c = 0.79788456080286536f;  // sqrt(2/pi)
      return 0.5f * g * (1.f + tanh_fast(c * fmaf(0.044715f * g, g * g, g)));
    }
    case MOE_ACT_RELU: return fmaxf(g, 0.f);
    default: return g;
  }
}

// 16 consecutive bf16 values p[0..15] (p 16-byte aligned) -> floats.
__device__ __forceinline__ void load_bf16x16(const uint16_t* p, float (&f)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int v = 0; v < 2; v++) {
    const uint4 w = __ldg(q + v);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      f[8 * v + 2 * i] = bf16_to_f32(u[i] & 0xffff);
      f[8 * v + 2 * i + 1] = bf16_to_f32(u[i] >> 16);
    }
  }
}

__device__ __forceinline__ void store_bf16x16(uint16_t* out, int n_valid, const float (&h)[16]) {
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; i++) packed[i] = pack_bf16x2(h[2 * i], h[2 * i + 1]);
  if (n_valid >= 16) {
    uint4* dst = reinterpret_cast<uint4*>(out);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  } else {
    for (int i = 0; i < n_valid; i++) out[i] = (uint16_t)(packed[i / 2] >> (16 * (i & 1)));
  }
}

// gate_up chunk: gate features fb..fb+15 in g[], their up partners in u[].  The
// bias of feature f is gbias[stride * f] (gate) and ubias[stride * f] (up), either
// null (see gu_rows: concat, interleaved or unfused bias rows); out = this row's h
// at column fb.
__device__ __forceinline__ void gate_up_chunk(const uint32_t (&g)[16], const uint32_t (&u)[16],
                                              const uint16_t* gbias, const uint16_t* ubias, int stride,
                                              int fb, int F, const ActParams& act, float wi, uint16_t* out) {
  float gb[16], ub[16];
#pragma unroll
  for (int i = 0; i < 16; i++) gb[i] = ub[i] = 0.f;
  const int nv = F - fb;
  const auto al16 = [](const uint16_t* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (gbias && ubias) {
    if (nv >= 16 && stride == 2 && ubias == gbias + 1 && al16(gbias + 2 * fb)) {
      float both[2][16];  // bias[2fb .. 2fb+31] = g0, u0, g1, u1, ...
      load_bf16x16(gbias + 2 * fb, both[0]);
      load_bf16x16(gbias + 2 * fb + 16, both[1]);
#pragma unroll
      for (int i = 0; i < 16; i++) {
        gb[i] = both[i / 8][2 * (i % 8)];
        ub[i] = both[i / 8][2 * (i % 8) + 1];
      }
    } else if (nv >= 16 && stride == 1 && al16(gbias + fb) && al16(ubias + fb)) {
      load_bf16x16(gbias + fb, gb);
      load_bf16x16(ubias + fb, ub);
    } else {
      for (int i = 0; i < 16 && i < nv; i++) {
        gb[i] = bf16_to_f32(gbias[stride * (fb + i)]);
        ub[i] = bf16_to_f32(ubias[stride * (fb + i)]);
      }
    }
  } else if (gbias || ubias) {  // unfused with only one of the two biases
    const uint16_t* b = gbias ? gbias : ubias;
    float* dst = gbias ? gb : ub;
    for (int i = 0; i < 16 && i < nv; i++) dst[i] = bf16_to_f32(b[stride * (fb + i)]);
  }
  float h[16];
#pragma unroll
  for (int i = 0; i < 16; i++)
    h[i] = gated_act_bf16(act, fmaf(wi, __uint_as_float(g[i]), gb[i]), fmaf(wi, __uint_as_float(u[i]), ub[i]));
  store_bf16x16(out + fb, nv, h);
}

// Bias row pointers of a gated expert's gate and up values (see gu_rows):
// fused stacks have one [2F] bias row per expert, the unfused layout two [F] rows.
struct GuBias {
  const uint16_t *g, *u;
  int stride;
};
__device__ __forceinline__ GuBias gu_bias(int layout, int64_t F, int e, const uint16_t* gate_up_bias,
                                          const uint16_t* gate_bias) {
  const GuRows r = gu_rows(layout, F);
  if (layout == MOE_GU_UNFUSED)
    return GuBias{gate_bias ? gate_bias + (int64_t)e * F : nullptr,
                  gate_up_bias ? gate_up_bias + (int64_t)e * F : nullptr, 1};
  if (!gate_up_bias) return GuBias{nullptr, nullptr, r.stride};
  const uint16_t* row = gate_up_bias + (int64_t)e * 2 * F;
  return GuBias{row + r.gate0, row + r.up0, r.stride};
}

// Plain (non-gated) chunk: features fb..fb+15 of fc1 in v[] -> h = act(wi acc + b1)
// (wi: the weigh-inputs scale, else 1).
__device__ __forceinline__ void plain_chunk(const uint32_t (&v)[16], const uint16_t* bias_e, int fb, int F,
                                            const ActParams& act, float wi, uint16_t* out) {
  float b[16];
#pragma unroll
  for (int i = 0; i < 16; i++) b[i] = 0.f;
  const int nv = F - fb;
  if (bias_e) {
    if (nv >= 16 && (reinterpret_cast<uintptr_t>(bias_e + fb) & 15u) == 0) {
      load_bf16x16(bias_e + fb, b);
    } else {
      for (int i = 0; i < 16 && i < nv; i++) b[i] = bf16_to_f32(bias_e[fb + i]);
    }
  }
  float h[16];
#pragma unroll
  for (int i = 0; i < 16; i++) h[i] = plain_act_bf16(act, fmaf(wi, __uint_as_float(v[i]), b[i]));
  store_bf16x16(out + fb, nv, h);
}

// down chunk: output features ob..ob+15; Y = (acc + bias) * w.
__device__ __forceinline__ void down_chunk(const uint32_t (&v)[16], const uint16_t* bias_e, int ob, int N,
                                           float w, uint16_t* out) {
  float b[16];
#pragma unroll
  for (int i = 0; i < 16; i++) b[i] = 0.f;
  const int nv = N - ob;
  if (bias_e) {
    if (nv >= 16 && (reinterpret_cast<uintptr_t>(bias_e) & 15u) == 0) {
      load_bf16x16(bias_e + ob, b);
    } else {
      for (int i = 0; i < 16 && i < nv; i++) b[i] = bf16_to_f32(bias_e[ob + i]);
    }
  }
  float o[16];
#pragma unroll
  for (int i = 0; i < 16; i++) o[i] = (__uint_as_float(v[i]) + b[i]) * w;
  store_bf16x16(out + ob, nv, o);
}

}  // namespace moe
