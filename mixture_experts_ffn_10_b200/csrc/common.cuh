// common.cuh -- internal declarations shared by the CUDA translation units of
// libmoe_b200: the workspace plan, kernel argument blocks, small device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- sizes and limits
constexpr int kMaxE = 1024;       // experts handled by one routing warp (32 per lane)
constexpr int kMaxK = 32;         // chosen experts per token (one lane each)
constexpr int kMaxGroups = 32;    // groups (one lane each)
constexpr int kChunkTokens = 64;  // tokens per histogram / scatter chunk
constexpr int kSimtBM = 64;       // rows per SIMT GEMM tile
constexpr int kTcBM = 128;        // rows per tensor-core GEMM tile (UMMA M)
constexpr int kPairBM = 256;      // rows per CTA-pair tile (UMMA M over two SMs)
constexpr int kPairMinRows = 512; // CTA pairs when routed rows per expert average at least this
constexpr int kTcGuBN = 128;      // h features per gate_up tile (gate rows + up rows = 256)
constexpr int kTcDnBN = 256;      // output features per down tile
constexpr int kTcBK = 64;         // K elements per pipeline stage of the bf16 tensor-core GEMMs
constexpr int kFixRegions = 8;      // split-K arrival counters per tile (one per epilogue warp, at most 8)
constexpr int kSplitMaxRows = 4096;  // split-K only for problems with at most this many routed rows
constexpr int kDirectMaxTokens = 64; // batches whose gate_up reads x in place (one 64-row A tile)

// ---------------------------------------------------------------- workspace plan
// Segments: experts 0..E-1 (routed rows, sorted by expert, token-ascending
// inside each expert), then segment E = the shared expert (one row per token)
// when Fs > 0.  Row r of X (gathered inputs), H (gated activations) and Y (the
// expert outputs) belongs to segment s for seg_off[s] <= r < seg_off[s+1];
// routed rows occupy [0, R), R = T*k, and shared rows [R, R+T).
struct Plan {
  int64_t T, d, F, E, k, Fs;
  int64_t R;          // routed rows T*k
  int64_t NS;         // segments E (+1 with a shared expert)
  int64_t rows;       // R (+T)
  int64_t Fmax;       // max(F, Fs): pitch of H in elements
  int64_t nchunks;    // ceil(T / kChunkTokens)
  int act_dtype, w_dtype, logit_dtype;
  bool tc;            // tensor-core path (bf16 activations) vs SIMT fp32 path
  bool pair;          // bf16 GEMMs on CTA pairs (256 x 256 tiles over two SMs)
  bool direct_x;      // gate_up reads x in place (small batches, single-CTA bf16 GEMMs)
  bool pair_fp4;      // MXFP4 GEMMs on CTA pairs (256 weight rows over two SMs)
  bool swap;          // bf16 GEMMs on CTA pairs with the weights as M (256 weight rows x <= 256 tokens)
  bool interleave;    // bf16 GEMMs visit the experts in interleaved order (sort.cuh: segment_scan)
  bool fused_ffn;     // direct_x: gate_up and down in one launch (launch_tc_ffn)
  int bm;             // GEMM tile rows
  int nt_gu_routed, nt_gu_shared, nt_dn_routed, nt_dn_shared;  // N tiles per segment
  int splits_gu, splits_dn;  // split-K factors of the two GEMMs (1 = none)
  int64_t partial_pitch;     // floats per row of the split-K partial buffer
  int64_t max_tiles_gu, max_tiles_dn;  // upper bounds of the GEMMs' tile counts
  int64_t n_sync;            // GEMM counters the sort clears (GemmCommon::fix, ready)
  // byte offsets into the workspace
  size_t o_status, o_idx, o_w, o_hist, o_cnt, o_off, o_tgu, o_tdn, o_ord, o_pos, o_perm, o_roww,
      o_sgate, o_x, o_h, o_y, o_part, o_sync, total;
};

// Fills `p` from validated arguments; returns the workspace size.
size_t make_plan(const moe_shape* s, const moe_options* o, Plan* p);

// The whole forward on a given device workspace (the body of moe_forward).
int forward_on_workspace(const moe_shape* s, const moe_options* o, const moe_tensors* t, void* ws,
                         size_t ws_bytes, void* stream);
// Records a message for moe_last_error() and returns `code`.
int set_error(int code, const char* msg);

// ---------------------------------------------------------------- device status
// First word of the workspace: 0 = OK, else a moe_status a kernel recorded.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float((uint32_t)b << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16_rn(lo) | ((uint32_t)f32_to_bf16_rn(hi) << 16);
}

// Gated activation h = act(g) * (u + beta); SiLU uses alpha and the limit clamp.
struct ActParams {
  int act;
  float alpha, beta, limit;
};
__device__ __forceinline__ float gated_act(const ActParams& a, float g, float u) {
  float v;
  switch (a.act) {
    case MOE_ACT_SILU:
      if (a.limit > 0.f) {
        g = fminf(g, a.limit);
        u = fminf(fmaxf(u, -a.limit), a.limit);
      }
      v = g / (1.f + __expf(-a.alpha * g));
      break;
    case MOE_ACT_GELU_ERF: v = 0.5f * g * (1.f + erff(g * 0.70710678118654752f)); break;
    case MOE_ACT_GELU_TANH: {
      const float c = 0.79788456080286536f;  // sqrt(2/pi)
      v = 0.5f * g * (1.f + tanhf(c * (g + 0.044715f * g * g * g)));
      break;
    }
    case MOE_ACT_RELU: v = fmaxf(g, 0.f); break;
    default: v = g; break;
  }
  return v * (u + a.beta);
}

// Activation of a non-gated expert ("MoE" graph-op activation_type with fusion_size 1):
// the gated forms without an up value; alpha for SiLU, no limit, no beta.
__device__ __forceinline__ float plain_act(const ActParams& a, float g) {
  switch (a.act) {
    case MOE_ACT_SILU: return g / (1.f + __expf(-a.alpha * g));
    case MOE_ACT_GELU_ERF: return 0.5f * g * (1.f + erff(g * 0.70710678118654752f));
    case MOE_ACT_GELU_TANH: {
      const float c = 0.79788456080286536f;  // sqrt(2/pi)
      return 0.5f * g * (1.f + tanhf(c * (g + 0.044715f * g * g * g)));
    }
    case MOE_ACT_RELU: return fmaxf(g, 0.f);
    default: return g;
  }
}

// Where the gate and up values of feature f of a gated expert come from: weight /
// bias rows gate_base + stride * f and up_base + stride * f of the expert's stacks.
//   concat:      one stack [2F]: gate rows 0..F-1, up rows F..2F-1 (stride 1)
//   interleaved: one stack [2F]: gate rows 2f, up rows 2f + 1 (stride 2)
//   unfused:     gate stack [F] and up stack [F] (stride 1)
struct GuRows {
  int64_t gate0, up0;  // row of feature 0 (in its own stack for unfused)
  int stride;
};
__host__ __device__ __forceinline__ GuRows gu_rows(int layout, int64_t F) {
  if (layout == MOE_GU_INTERLEAVED) return GuRows{0, 1, 2};
  if (layout == MOE_GU_UNFUSED) return GuRows{0, 0, 1};
  return GuRows{0, F, 1};
}

// ---------------------------------------------------------------- launchers
struct RouteArgs {
  const void* logits;
  const void* router_bias;
  const float* sel_bias;
  int T, E, k, logit_bf16;
  int score, renorm;
  float scale;
  int n_group, topk_group;
  int32_t* idx;     // [T, k] workspace
  float* w;         // [T, k] workspace
  int32_t* idx_user;
  float* w_user;
  // shared gate sigma(x . g)
  const void* x;
  const void* gvec;
  int d, act_bf16;
  float* sgate;     // [T] or null
  // router weight Wr [d, E] (act dtype): with logits null the logits are x Wr,
  // accumulated in double in index order and rounded once to fp32
  const void* router_weight;
  float* logits_out;  // [T, E] or null
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);
cudaError_t launch_router(const RouteArgs& a, cudaStream_t st);  // logits x Wr, then the routing

struct SortArgs {
  const int32_t* idx;   // [T, k]
  const float* w;       // [T, k]
  int T, k, E, NS, nchunks;
  int R;
  int shared_rows;      // T when a shared expert exists, else 0
  int32_t* hist;        // [nchunks, E]
  int32_t* cnt;         // [NS]
  int32_t* off;         // [NS + 1]
  int32_t* tile_gu;     // [NS + 1] (by visiting position when order is set)
  int32_t* tile_dn;     // [NS + 1]
  int32_t* order;       // [NS] segment visited at each position, or null (segment order)
  int bm, nt_gu_routed, nt_gu_shared, nt_dn_routed, nt_dn_shared;
  int32_t* pos;         // [T, k] -> row
  int32_t* perm;        // [R] row -> token
  float* roww;          // [R] row -> routing weight
  int32_t* sync;        // [n_sync] counters of the GEMMs (split-K arrivals, finished h
  int n_sync;           // regions), set to zero here, before the GEMMs run
  int* status;
};
cudaError_t launch_sort(const SortArgs& a, cudaStream_t st);

struct GatherArgs {
  const void* x;        // [T, d]
  const int32_t* pos;   // [T, k] token slot -> row
  const float* roww;    // [R]
  void* xg;             // [R, d]
  int R, d, T, k, bf16, weigh_inputs;
  int* status;
};
cudaError_t launch_gather(const GatherArgs& a, cudaStream_t st);

struct CombineArgs {
  const void* Y;        // [rows, d] expert outputs (bf16 or f32)
  const int32_t* pos;   // [T, k]
  const float* sgate;   // [T] or null
  const void* shared_output;  // [T, d] or null
  void* y;              // [T, d]
  int T, d, k, R, has_shared, bf16;
  int* status;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);

// Grouped GEMM arguments common to the SIMT and tensor-core paths.
struct GemmCommon {
  int NS, E, R, T;
  const int32_t* cnt;       // [NS]
  const int32_t* off;       // [NS + 1]
  const int32_t* tiles;     // [NS + 1] tile prefix for this GEMM (by visiting position)
  const int32_t* order;     // [NS] segment at each visiting position, or null (identity)
  int max_tiles;            // host upper bound of tiles[NS] - tiles[seg_begin]
  int seg_begin;            // CTA-pair bf16 kernel: walk segments seg_begin .. NS-1 only (else 0)
  int d, F, Fs, Fmax;
  int gu_layout;             // MOE_GU_* of the routed experts (the shared expert: concat if unfused)
  int ffn;                   // MOE_FFN_GATED or MOE_FFN_PLAIN
  ActParams act;
  int weigh_inputs;
  // Small batches (the single-CTA bf16 gate_up with T <= 64): the activation tile of
  // every routed segment is x itself, rows 0 .. T-1, and accumulator row i belongs to
  // token i; its output row is pos[i][j] for the slot j with topk_idx[i][j] == e (if
  // any).  No copy of the rows in expert order is made.  Weigh-inputs then scales the
  // accumulators (W (w x) = w (W x)) before the bias and the activation.
  int direct_x;
  int k;
  const int32_t* topk_idx;  // [T, k]
  const int32_t* pos;       // [T, k]
  int* status;
  // split-K: each tile's K range is cut into `splits` parts whose fp32 partial
  // accumulators go to partial[split][row][n_blk * 256 + col] (pitch floats per
  // row).  Each epilogue warp of a tile owns one region of it (its TMEM lane
  // quadrant, its column chunks) and counts its split done in fix[tile * kFixRegions
  // + region]; the last of the splits to arrive sums the region's partials in split
  // order and runs the epilogue.  The counters start at zero (the sort clears them).
  int splits;
  float* partial;
  int partial_pitch;
  int32_t* fix;
};

// The GEMM's tile count from the device-side prefix, at most the host's bound
// max_tiles past tiles[seg_begin]: a larger count means the workspace was changed
// under the call (MOE_ERR_SHAPE recorded, the walk clamped to the bound).
__device__ __forceinline__ int tile_total(const GemmCommon& c) {
  const int first = c.tiles[c.seg_begin];
  const int total = c.tiles[c.NS];
  if (total >= first && total - first <= c.max_tiles) return total;
  set_status(c.status, MOE_ERR_SHAPE);
  return total < first ? first : first + c.max_tiles;
}

struct SimtArgs {
  GemmCommon c;
  const float* x;           // [T, d] (shared rows read x directly)
  const float* xg;          // [R, d]
  const float* gate_up;     // [E, 2F, d]; unfused: up rows [E, F, d]; plain: fc1 [E, F, d]
  const float* gate_up_bias;// [E, 2F] ([E, F] unfused / plain) or null
  const float* gate;        // unfused: gate rows [E, F, d]
  const float* gate_bias;   // unfused: [E, F] or null
  const float* down;        // [E, d, F]
  const float* down_bias;   // [E, d] or null
  const float* sh_gate_up;  // [2Fs, d]
  const float* sh_down;     // [d, Fs]
  const float* roww;        // [R]
  float* h;                 // [rows, Fmax]
  float* Y;                 // [rows, d]
};
cudaError_t launch_simt_gate_up(const SimtArgs& a, cudaStream_t st);
cudaError_t launch_simt_down(const SimtArgs& a, cudaStream_t st);

struct TcArgs {
  GemmCommon c;
  const void* x;            // [T, d] bf16
  const void* xg;           // [R, d] bf16
  const void* gate_up;      // [E, 2F, d] bf16; unfused: up rows [E, F, d]; plain: fc1 [E, F, d]
  const void* gate_up_bias; // [E, 2F] ([E, F] unfused / plain) bf16 or null
  const void* gate;         // unfused: gate rows [E, F, d] (MXFP4: codes [E, F, d/2])
  const void* gate_bias;    // unfused: [E, F] bf16 or null
  const uint8_t* gate_scales;  // unfused MXFP4: e8m0 [E, F, d/32]
  const void* down;         // [E, d, F] bf16
  const void* down_bias;    // [E, d] bf16 or null
  const void* sh_gate_up;   // [2Fs, d] bf16
  const void* sh_down;      // [d, Fs] bf16
  const float* roww;        // [R]
  void* h;                  // [rows, Fmax] bf16
  void* Y;                  // [rows, d] bf16
  int num_sms;
  const uint8_t* gate_up_scales;  // MXFP4 only: e8m0 [E, 2F, d/32]
  const uint8_t* down_scales;     // MXFP4 only: e8m0 [E, d, F/32]
};
cudaError_t launch_tc_gate_up(const TcArgs& a, cudaStream_t st);
cudaError_t launch_tc_down(const TcArgs& a, cudaStream_t st);
cudaError_t launch_tcs_gate_up(const TcArgs& a, cudaStream_t st);  // CTA pairs, weights as M
cudaError_t launch_tcs_down(const TcArgs& a, cudaStream_t st);
constexpr int kSwapBM = 256;      // token rows per swapped-operand pair tile (the MMA's N, trimmed)
cudaError_t launch_tc2_gate_up(const TcArgs& a, cudaStream_t st);  // CTA-pair variants
cudaError_t launch_tc2_down(const TcArgs& a, cudaStream_t st);
// Small batches with x read in place (direct_x): gate_up and down in one launch of the
// single-CTA kernel.  a.c is the gate_up GEMM, dn the down GEMM; ready [NS] counts the
// finished h regions of each segment (zero before the launch).
cudaError_t launch_tc_ffn(const TcArgs& a, const GemmCommon& dn, int32_t* ready, cudaStream_t st);
// Split count for a GEMM of at most `tiles` tiles of `nkb` k-blocks on `sms` SMs.
int choose_splits(int64_t tiles, int nkb, int sms);
// MXFP4 expert stacks (gate_up / down are e2m1 codes), routed segments only (a shared
// expert runs on the CTA-pair bf16 kernel, GemmCommon::seg_begin = E).
cudaError_t launch_fp4_gate_up(const TcArgs& a, cudaStream_t st);
cudaError_t launch_fp4_down(const TcArgs& a, cudaStream_t st);
cudaError_t launch_fp4p_gate_up(const TcArgs& a, cudaStream_t st);  // CTA-pair variants
cudaError_t launch_fp4p_down(const TcArgs& a, cudaStream_t st);
constexpr int kFp4BM = 256;       // activation rows per MXFP4 tile (the MMA's N, trimmed to the live rows)
constexpr int kFp4PairBN = 256;   // weight rows per CTA-pair MXFP4 tile (128 decoded by each CTA)
constexpr int kFp4PairMinRows = 128;  // CTA pairs when routed rows per expert average at least this
constexpr int kFp4GuBN = 64;      // h features per MXFP4 gate_up tile (64 gate + 64 up rows)
constexpr int kFp4DnBN = 128;     // output features per MXFP4 down tile

// ---------------------------------------------------------------- programmatic dependent launch
// Every kernel of the forward is launched with programmatic stream serialization:
// it may be scheduled, and run a prologue that touches only shared memory, TMEM
// and its parameters, while the kernel before it in the stream still runs.
// pdl_enter() must come before the kernel's first global-memory access: it
// returns once the preceding kernel has completed with its writes visible, then
// lets the next kernel be scheduled.  Without the launch attribute (or with
// MOE_B200_PDL=0) the wait returns at once and launches serialize as usual.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
bool pdl_enabled();  // false when the environment sets MOE_B200_PDL=0

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// launch_pdl for a kernel whose CTAs wait on one another: a cooperative launch too,
// which fails instead of starting when the grid cannot be resident all at once.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_coop_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                   Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe
