// route.cuh -- routing of one token by one warp: picks k of E experts and their weights.
//
// Definitions ("Struct MoeSpec" field docs; graph-op page attributes k and
// normalize_routing_weights; "Struct Moe" groups):
//   l'_e = fp32(l_e) + fp32(router_bias_e)                      (router_bias)
//   s_e  = softmax_e(l') over every expert, or sigmoid(l'_e)     (score)
//   key_e = l'_e for an unbiased softmax (monotone in s_e), else s_e + B_e,
//           formed in double                                     (selection_bias)
//   groups: E/n_group contiguous experts per group, group score = the sum of
//           its two best keys; only the best topk_group groups are eligible
//   top-k by key, larger first, ties to the lower index, NaN keys last
//   w_j = s_{e_j}; renormalize: w_j / max(sum_j w_j, 2^-14); then w_j * S
// Scores and weights are computed in double, then rounded once to fp32.
#pragma once

#include "common.cuh"

namespace moe {
namespace routing {

// Order-preserving 64-bit image of a key: larger keys map to larger integers, NaN to
// 0 (below every number), -0 to the image of +0.  Experts (and groups) rank by image,
// larger first, equal images to the lower index (ahead()): the order the oracle
// defines on the keys themselves.
__device__ __forceinline__ uint64_t ord_key(double k) {
  if (isnan(k)) return 0ull;
  if (k == 0.0) k = 0.0;
  const uint64_t b = (uint64_t)__double_as_longlong(k);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// (key image, expert) candidates: larger image first, then the lower index; the
// empty candidate (0, kNone) ranks below every expert, NaN keys included.
constexpr int kNone = 0x7fffffff;
__device__ __forceinline__ bool ahead(uint64_t ka, int ia, uint64_t kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

__device__ __forceinline__ float load_logit(const void* p, int bf16, int64_t i) {
  return bf16 ? bf16_to_f32(((const uint16_t*)p)[i]) : ((const float*)p)[i];
}

// The key whose image is k (ord_key inverted; NaN comes back as a NaN, -0 as +0).
__device__ __forceinline__ double key_of_image(uint64_t k) {
  const uint64_t b = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double((long long)b);
}

// Warp arg-best over (image, expert) candidates, one per lane (kNone = none): the
// largest image, then the lowest index, in three single-instruction warp reductions.
// Returns the best image; *winner = its index (kNone if every lane offered none).
__device__ __forceinline__ uint64_t warp_argbest(uint64_t k, int idx, int* winner) {
  const uint32_t hi = (uint32_t)(k >> 32), lo = (uint32_t)k;
  const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
  const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
  const uint32_t cand = (hi == mhi && lo == mlo) ? (uint32_t)idx : (uint32_t)kNone;
  *winner = (int)__reduce_min_sync(0xffffffffu, cand);
  return ((uint64_t)mhi << 32) | mlo;
}

// Routes token t with the calling warp (lane = this thread's lane).  The token's
// logits are read from a.logits, or from lrow (fp32, E values) when it is given.
template <int EPL>  // experts per lane: E <= 32 * EPL, expert e = lane + 32 * i
__device__ __forceinline__ void route_token(const RouteArgs& a, int t, int lane, const float* lrow = nullptr) {
  const int E = a.E;

  float lp[EPL];
#pragma unroll
  for (int i = 0; i < EPL; i++) {
    const int e = lane + 32 * i;
    float l = 0.f;
    if (e < E) {
      l = lrow ? lrow[e] : load_logit(a.logits, a.logit_bf16, (int64_t)t * E + e);
      if (a.router_bias) l = l + load_logit(a.router_bias, a.logit_bf16, e);
    }
    lp[i] = l;
  }

  // ---- scores (double)
  double s[EPL];
  if (a.score == MOE_SCORE_SOFTMAX) {
    float m = -INFINITY;  // NaN logits never compare greater, so they never become the max
#pragma unroll
    for (int i = 0; i < EPL; i++)
      if (lane + 32 * i < E && lp[i] > m) m = lp[i];
    {  // warp max on the order-preserving image of the (non-NaN) fp32 values
      uint32_t u = __float_as_uint(m);
      u = (u >> 31) ? ~u : (u | 0x80000000u);
      u = __reduce_max_sync(0xffffffffu, u);
      m = __uint_as_float((u >> 31) ? (u & 0x7fffffffu) : ~u);
    }
    double den = 0.0;
#pragma unroll
    for (int i = 0; i < EPL; i++) {
      s[i] = (lane + 32 * i < E) ? exp((double)lp[i] - (double)m) : 0.0;
      den += s[i];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
#pragma unroll
    for (int i = 0; i < EPL; i++) s[i] = s[i] / den;
  } else {
#pragma unroll
    for (int i = 0; i < EPL; i++) s[i] = 1.0 / (1.0 + exp(-(double)lp[i]));
  }

  // ---- keys
  double key[EPL];
  const bool plain_softmax = a.score == MOE_SCORE_SOFTMAX && a.sel_bias == nullptr;
#pragma unroll
  for (int i = 0; i < EPL; i++) {
    const int e = lane + 32 * i;
    if (plain_softmax)
      key[i] = (double)lp[i];
    else
      key[i] = s[i] + ((a.sel_bias && e < E) ? (double)a.sel_bias[e] : 0.0);
  }

  // ---- group limit -> eligibility mask over groups
  uint32_t kept_groups = 0xffffffffu;
  int per = E;
  if (a.n_group > 0) {
    per = E / a.n_group;
    double my_gscore = 0.0;
    for (int g = 0; g < a.n_group; g++) {
      // lane-local best two of group g on the key images, then the warp's best and
      // second best by single-instruction warp reductions
      uint64_t k1 = 0ull, k2 = 0ull;
      int i1 = kNone, i2 = kNone;
#pragma unroll
      for (int i = 0; i < EPL; i++) {
        const int e = lane + 32 * i;
        if (e < E && e / per == g) {
          const uint64_t ke = ord_key(key[i]);
          if (ahead(ke, e, k1, i1)) {
            k2 = k1;
            i2 = i1;
            k1 = ke;
            i1 = e;
          } else if (ahead(ke, e, k2, i2)) {
            k2 = ke;
            i2 = e;
          }
        }
      }
      int w1;
      const uint64_t best = warp_argbest(k1, i1, &w1);
      double gs = key_of_image(best);
      if (per >= 2) {
        // the lane that held the winner offers its second best instead
        const bool had = i1 == w1;
        int w2;
        const uint64_t second = warp_argbest(had ? k2 : k1, had ? i2 : i1, &w2);
        gs = gs + key_of_image(second);
      }
      if (lane == g) my_gscore = gs;
    }
    kept_groups = 0;
    bool gtaken = false;
    const uint64_t gk = ord_key(my_gscore);
    for (int r = 0; r < a.topk_group; r++) {
      // lane g offers group g until it is kept; other lanes offer the empty candidate
      const bool offer = lane < a.n_group && !gtaken;
      int wg;
      warp_argbest(offer ? gk : 0ull, offer ? lane : kNone, &wg);
      if (wg != kNone) kept_groups |= 1u << wg;
      if (lane == wg) gtaken = true;
    }
  }

  // ---- top-k: k rounds of a warp arg-best over the eligible, untaken experts,
  // on the keys' order-preserving integer images
  uint64_t okey[EPL];
  bool avail[EPL];  // eligible and not yet taken
#pragma unroll
  for (int i = 0; i < EPL; i++) {
    const int e = lane + 32 * i;
    avail[i] = e < E && ((kept_groups >> (e / per)) & 1u);
    okey[i] = ord_key(key[i]);
  }
  double my_s = 0.0;
  int my_idx = -1;
  for (int j = 0; j < a.k; j++) {
    uint64_t bk = 0ull;
    int bi = kNone;
#pragma unroll
    for (int i = 0; i < EPL; i++) {
      const int e = lane + 32 * i;
      if (avail[i] && ahead(okey[i], e, bk, bi)) {
        bk = okey[i];
        bi = e;
      }
    }
    // warp arg-best in three single-instruction warp reductions (same order as ahead())
    warp_argbest(bk, bi, &bi);
    // the winner's owner lane marks it taken and hands its score to lane j
    double sv = 0.0;
    const int slot = bi >> 5;
#pragma unroll
    for (int i = 0; i < EPL; i++) {
      if (i == slot) sv = s[i];
    }
    const double got = __shfl_sync(0xffffffffu, sv, bi & 31);
    if ((bi & 31) == lane) {
#pragma unroll
      for (int i = 0; i < EPL; i++)
        if (i == slot) avail[i] = false;
    }
    if (lane == j) {
      my_s = got;
      my_idx = bi == kNone ? -1 : bi;
    }
  }

  // ---- weights: renormalize (sum in slot order) with the 2^-14 clamp, then the scale
  double sum = 0.0;
  for (int j = 0; j < a.k; j++) sum += __shfl_sync(0xffffffffu, my_s, j);
  if (lane < a.k) {
    double w = my_s;
    if (a.renorm) {
      const double den = sum > 0x1p-14 ? sum : 0x1p-14;
      w = w / den;
    }
    w = w * (double)a.scale;
    const int64_t o = (int64_t)t * a.k + lane;
    a.idx[o] = my_idx;
    a.w[o] = (float)w;
    if (a.idx_user) a.idx_user[o] = my_idx;
    if (a.w_user) a.w_user[o] = (float)w;
  }

  // ---- shared expert gate sigma(x_t . g)
  if (a.sgate) {
    float acc = 0.f;
    for (int i = lane; i < a.d; i += 32) {
      const int64_t xi = (int64_t)t * a.d + i;
      const float xv = a.act_bf16 ? bf16_to_f32(((const uint16_t*)a.x)[xi]) : ((const float*)a.x)[xi];
      const float gv = a.act_bf16 ? bf16_to_f32(((const uint16_t*)a.gvec)[i]) : ((const float*)a.gvec)[i];
      acc = fmaf(xv, gv, acc);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) a.sgate[t] = 1.f / (1.f + expf(-acc));
  }
}

}  // namespace routing
}  // namespace moe
