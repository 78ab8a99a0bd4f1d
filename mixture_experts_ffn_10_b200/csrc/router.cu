// router.cu -- the router in front of the routing: logits = x Wr ("Struct MoeSpec"
// wr, indexed wr[(i-1)E + e], so Wr is [d, E] with the expert index fastest; "the
// router's bias, added to each logit before the softmax (router Wr plus Br)"),
// fused with the per-token routing of route.cuh so the logits never go to memory
// (unless the caller asks for them).
//
// A block owns 32 tokens.  Its threads accumulate the 32 x E logits in double,
// each (token, expert) serially over i = 0 .. d-1: every product of two bf16 (or
// fp32) values is exact in double, so each partial sum is rounded exactly as a
// plain serial double loop rounds it, and the fp32 logit is that sum rounded once.
// The choice of k experts -- an integer decided by floating point -- therefore
// sees the same logits as a plain double evaluation of x Wr.  Cost: 2 T d E
// floating-point operations at the FP64 rate, on top of reading x and Wr.
// Then each of the 8 warps routes 4 of the block's tokens from shared memory.
#include "route.cuh"

namespace moe {
namespace {

constexpr int kTok = 32;    // tokens per block
constexpr int kKc = 32;     // K elements per shared-memory chunk
constexpr int kEpass = 128; // experts per accumulation pass (32 lanes x 4)
constexpr int kXp = kTok + 4; // x chunk row pitch (floats): 16-byte rows, fewer bank conflicts

template <typename T>
__device__ __forceinline__ float ldx(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ldx<uint16_t>(const uint16_t* p, int64_t i) { return bf16_to_f32(p[i]); }
template <>
__device__ __forceinline__ float ldx<float>(const float* p, int64_t i) { return p[i]; }

template <int EPL, typename T>
__global__ void __launch_bounds__(256) router_kernel(RouteArgs a) {
  extern __shared__ float sm[];
  float* xs = sm;                      // [kKc][kXp]
  float* ws = xs + kKc * kXp;          // [kKc][kEpass]
  float* lg = ws + kKc * kEpass;       // [kTok][E]: the block's logits
  pdl_enter();
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // expert lane, token group of 4
  const int t0 = blockIdx.x * kTok;
  const int E = a.E, d = a.d;
  const T* x = static_cast<const T*>(a.x);
  const T* wr = static_cast<const T*>(a.router_weight);

  for (int e0 = 0; e0 < E; e0 += kEpass) {
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
      for (int j = 0; j < 4; j++) acc[i][j] = 0.0;
    for (int k0 = 0; k0 < d; k0 += kKc) {
      __syncthreads();
      for (int q = threadIdx.x; q < kKc * kTok; q += 256) {  // x chunk, token-fastest in smem
        const int tt = q / kKc, kk = q % kKc;
        const int t = t0 + tt, k = k0 + kk;
        xs[kk * kXp + tt] = (t < a.T && k < d) ? ldx<T>(x, (int64_t)t * d + k) : 0.f;
      }
      for (int q = threadIdx.x; q < kKc * kEpass; q += 256) {  // Wr chunk, expert-fastest
        const int kk = q / kEpass, ee = q % kEpass;
        const int k = k0 + kk, e = e0 + ee;
        ws[kk * kEpass + ee] = (k < d && e < E) ? ldx<T>(wr, (int64_t)k * E + e) : 0.f;
      }
      __syncthreads();
      const int kn = min(kKc, d - k0);
      for (int kk = 0; kk < kn; kk++) {  // index order: the sums round as a serial loop's
        const float4 xv = *reinterpret_cast<const float4*>(&xs[kk * kXp + ty * 4]);
        const float xt[4] = {xv.x, xv.y, xv.z, xv.w};
        float wv[4];
#pragma unroll
        for (int j = 0; j < 4; j++) wv[j] = ws[kk * kEpass + tx + 32 * j];
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
          for (int j = 0; j < 4; j++) acc[i][j] = fma((double)xt[i], (double)wv[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int tt = ty * 4 + i, e = e0 + tx + 32 * j;
        if (e < E) {
          const float l = (float)acc[i][j];
          lg[tt * E + e] = l;
          if (a.logits_out && t0 + tt < a.T) a.logits_out[(int64_t)(t0 + tt) * E + e] = l;
        }
      }
  }
  __syncthreads();
  for (int i = 0; i < kTok / 8; i++) {  // warp ty routes tokens ty, ty + 8, ...
    const int tt = ty + 8 * i;
    if (t0 + tt < a.T) routing::route_token<EPL>(a, t0 + tt, tx, lg + tt * E);
  }
}

template <int EPL>
cudaError_t launch_epl(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)(kKc * kXp + kKc * kEpass + kTok * a.E) * sizeof(float);
  const dim3 grid((a.T + kTok - 1) / kTok);
  if (a.act_bf16) {
    cudaError_t e = cudaFuncSetAttribute(router_kernel<EPL, uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(router_kernel<EPL, uint16_t>, grid, dim3(256), smem, st, a);
  }
  cudaError_t e = cudaFuncSetAttribute(router_kernel<EPL, float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(router_kernel<EPL, float>, grid, dim3(256), smem, st, a);
}

}  // namespace

cudaError_t launch_router(const RouteArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int epl = (a.E + 31) / 32;
  if (epl <= 1) return launch_epl<1>(a, st);
  if (epl <= 2) return launch_epl<2>(a, st);
  if (epl <= 4) return launch_epl<4>(a, st);
  if (epl <= 8) return launch_epl<8>(a, st);
  if (epl <= 16) return launch_epl<16>(a, st);
  return launch_epl<32>(a, st);
}

}  // namespace moe
