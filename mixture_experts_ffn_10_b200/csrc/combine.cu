// combine.cu -- deterministic gather-reduce of the expert outputs.
//
// y[t] = sum_{j=0..k-1} Y[pos[t, j]]  (each row already carries its routing
//        weight, or none for weigh-inputs)
//      + gate_t * Y[R + t]            (shared expert row; gate_t = sigmoid(x_t . g) or 1)
//      + shared_output[t]             (caller's precomputed shared branch)
// summed in fp32 in exactly this order, then rounded once to y's dtype
// ("ClikaRT::nn::QMoEWoQ" forward: shared_output folds into the routed combine;
// "Struct MoeSpec" weigh_inputs; "Struct Moe" shared_gate).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 128;
constexpr int kBatch = 4;  // expert rows whose loads are issued together

template <typename T>
__device__ __forceinline__ void load8(const T* p, float* f) {
  if constexpr (sizeof(T) == 2) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      f[2 * i] = bf16_to_f32(u[i] & 0xffff);
      f[2 * i + 1] = bf16_to_f32(u[i] >> 16);
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
  pdl_enter();
  const int t = blockIdx.x;
  const int c = (blockIdx.y * kThreads + threadIdx.x) * 8;
  if (c >= a.d) return;
  const T* Y = (const T*)a.Y;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; i++) acc[i] = 0.f;
  float v[8];
  // batches of kBatch rows: all loads first, then the adds in slot order
  for (int j0 = 0; j0 < a.k; j0 += kBatch) {
    float b[kBatch][8];
#pragma unroll
    for (int u = 0; u < kBatch; u++) {
#pragma unroll
      for (int i = 0; i < 8; i++) b[u][i] = 0.f;
      const int j = j0 + u;
      if (j < a.k) {
        const int64_t row = a.pos[(int64_t)t * a.k + j];
        if (row < 0 || row >= a.R) set_status(a.status, MOE_ERR_SHAPE);
        else load8<T>(Y + row * a.d + c, b[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; u++) {
      if (j0 + u < a.k) {
#pragma unroll
        for (int i = 0; i < 8; i++) acc[i] += b[u][i];
      }
    }
  }
  if (a.has_shared) {
    const float g = a.sgate ? a.sgate[t] : 1.f;
    load8<T>(Y + ((int64_t)a.R + t) * a.d + c, v);
#pragma unroll
    for (int i = 0; i < 8; i++) acc[i] += g * v[i];
  }
  if (a.shared_output) {
    load8<T>((const T*)a.shared_output + (int64_t)t * a.d + c, v);
#pragma unroll
    for (int i = 0; i < 8; i++) acc[i] += v[i];
  }
  T* y = (T*)a.y + (int64_t)t * a.d + c;
  if constexpr (sizeof(T) == 2) {
    uint4 q;
    q.x = pack_bf16x2(acc[0], acc[1]);
    q.y = pack_bf16x2(acc[2], acc[3]);
    q.z = pack_bf16x2(acc[4], acc[5]);
    q.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y) = q;
  } else {
    reinterpret_cast<float4*>(y)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(y)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const dim3 grid(a.T, (a.d / 8 + kThreads - 1) / kThreads);
  if (a.bf16) return launch_pdl(combine_kernel<uint16_t>, grid, kThreads, 0, st, a);
  return launch_pdl(combine_kernel<float>, grid, kThreads, 0, st, a);
}

}  // namespace moe
