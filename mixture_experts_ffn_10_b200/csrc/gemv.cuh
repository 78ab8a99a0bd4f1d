// gemv.cuh -- declarations of the one-launch forward for a few tokens (gemv.cu),
// kept out of the headers the grouped GEMMs include.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace moe {

// ---------------------------------------------------------------- few-token forward
// Batches of at most kGemvMaxTokens tokens with bf16 weights: the whole forward in one
// cooperative launch (gemv.cu).  Every CTA routes the tokens itself (or reads the
// routing kernel's result); then each warp streams its share of the chosen experts'
// weights, tiles of 16 rows x kGemvKS, through its own shared-memory slots (TMA loads
// it issues itself) and multiplies them by the tokens' rows with warp-level
// mma.sync (the tokens are the 8 columns): gate_up (activation fused) first, then,
// once every CTA has published its h features, down with the combine.
constexpr int kGemvMaxTokens = 4;
constexpr int kGemvDefaultTokens = 0;  // off unless MOE_B200_GEMV=N asks (measured slower)
constexpr int kGemvMaxWarps = 16;
constexpr int kGemvSlotsPerWarp = 2;
constexpr int kGemvKB = 4;             // 64-element k-blocks per stage
constexpr int kGemvKS = 64 * kGemvKB;  // K per stage
constexpr int kGemvSlotBytes = 16 * kGemvKS * 2;  // 16 weight rows of one stage: 8 KiB
constexpr int kGemvRowBlock = 16;      // output features per down unit
constexpr int kGemvMaxEnt = kGemvMaxTokens * kMaxK + 1;  // distinct experts + the shared one
constexpr int kGemvDoneOffset = 64;   // its CTA counter: workspace bytes after the status word
constexpr int kGemvRbOffset = 128;    // its per-row-block counters [ceil(d / 16)]
struct GemvArgs {
  RouteArgs ra;             // in-kernel routing (router_logits given): idx, w, sgate unused
  int pre_routed;           // 1: read idx, w (and sgate) that the routing kernel wrote
  const int32_t* idx;       // [T, k] (pre_routed)
  const float* w;           // [T, k] (pre_routed)
  const float* sgate;       // [T] or null (pre_routed with a shared gate)
  int has_sgate;            // shared expert output times sigmoid(x . g)
  const uint16_t* x;        // [T, d]
  const uint16_t* gate_up;  // as TcArgs
  const uint16_t* gate_up_bias;
  const uint16_t* gate;
  const uint16_t* gate_bias;
  const uint16_t* down;
  const uint16_t* down_bias;
  const uint16_t* sh_gate_up;
  const uint16_t* sh_down;
  const uint16_t* shared_output;  // [T, d] or null
  uint16_t* h;              // [rows, Fmax] workspace
  uint16_t* Y;              // [rows, d] workspace: each routed slot's (and shared) expert output
  uint16_t* y;              // [T, d]
  int32_t* done;            // CTAs that have published their h features (zero before the launch)
  int32_t* rb_done;         // [ceil(d / 16)] down units finished per row block (zero before)
  int T, d, F, Fs, E, k, R, Fmax;
  int gu_layout, ffn, weigh_inputs;
  ActParams act;
  int* status;
  int warps, xh_bytes, smem_bytes;  // geometry (make_plan)
};
// The few-token kernel's routing result and its list of distinct experts (static
// shared memory): entry u is expert e[u] (-1: the shared expert) with cnt[u] token
// slots; slot c is token tok[u][c], row row[u][c] of h and Y (t k + j, or R + t for
// the shared expert), routing weight wt[u][c] (1 for the shared expert).
struct GemvMeta {
  int32_t idx[kGemvMaxTokens * kMaxK];
  float w[kGemvMaxTokens * kMaxK];
  float sgate[kGemvMaxTokens];
  int n_ent;
  int abort;
  int e[kGemvMaxEnt], cnt[kGemvMaxEnt];
  int tok[kGemvMaxEnt][kGemvMaxTokens], row[kGemvMaxEnt][kGemvMaxTokens];
  float wt[kGemvMaxEnt][kGemvMaxTokens];
};
// Dynamic shared-memory bytes of the few-token kernel: alignment slack, the warps'
// slots and the x / h staging area of xh bytes.
__host__ __device__ constexpr int gemv_smem(int warps, int xh) {
  return 1024 + warps * kGemvSlotsPerWarp * kGemvSlotBytes + xh;
}
cudaError_t launch_gemv_ffn(const GemvArgs& a, int num_sms, cudaStream_t st);

// Its geometry for one problem (api.cu: plan_gemv): off, or the warps per CTA, the x / h
// staging bytes and the dynamic shared memory of the launch.
struct GemvPlan {
  bool on = false;
  int warps = 0, xh = 0, smem = 0;
};
GemvPlan gemv_plan(const moe_shape* s, const Plan& p);  // (api.cu)
// Workspace bytes of the status block: the status word, the CTA counter and the
// per-row-block counters of a d-wide output.
inline size_t gemv_status_bytes(int64_t d) {
  return (size_t)kGemvRbOffset + (size_t)((d + kGemvRowBlock - 1) / kGemvRowBlock) * 4;
}

namespace sm100 {
__device__ __forceinline__ void tma_load_5d(const CUtensorMap* m, uint64_t* bar, void* dst, int c0,
                                            int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
}  // namespace sm100

}  // namespace moe
