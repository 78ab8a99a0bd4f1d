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
constexpr int kSplitMaxRows = 4096;  // split-K only for problems with at most this many routed rows

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
  int bm;             // GEMM tile rows
  int nt_gu_routed, nt_gu_shared, nt_dn_routed, nt_dn_shared;  // N tiles per segment
  int splits_gu, splits_dn;  // split-K factors of the two GEMMs (1 = none)
  int64_t partial_pitch;     // floats per row of the split-K partial buffer
  // byte offsets into the workspace
  size_t o_status, o_idx, o_w, o_hist, o_cnt, o_off, o_tgu, o_tdn, o_pos, o_perm, o_roww,
      o_sgate, o_x, o_h, o_y, o_part, total;
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
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);

struct SortArgs {
  const int32_t* idx;   // [T, k]
  const float* w;       // [T, k]
  int T, k, E, NS, nchunks;
  int R;
  int shared_rows;      // T when a shared expert exists, else 0
  int32_t* hist;        // [nchunks, E]
  int32_t* cnt;         // [NS]
  int32_t* off;         // [NS + 1]
  int32_t* tile_gu;     // [NS + 1]
  int32_t* tile_dn;     // [NS + 1]
  int bm, nt_gu_routed, nt_gu_shared, nt_dn_routed, nt_dn_shared;
  int32_t* pos;         // [T, k] -> row
  int32_t* perm;        // [R] row -> token
  float* roww;          // [R] row -> routing weight
  int* status;
};
cudaError_t launch_sort(const SortArgs& a, cudaStream_t st);

struct GatherArgs {
  const void* x;        // [T, d]
  const int32_t* perm;  // [R]
  const float* roww;    // [R]
  void* xg;             // [R, d]
  int R, d, T, bf16, weigh_inputs;
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
  const int32_t* tiles;     // [NS + 1] tile prefix for this GEMM
  int max_tiles;            // host upper bound of tiles[NS]
  int d, F, Fs, Fmax;
  int gu_layout;
  ActParams act;
  int weigh_inputs;
  int* status;
  // split-K: each tile's K range is cut into `splits` parts whose fp32 partial
  // accumulators go to partial[split][row][n_blk * 256 + col] (pitch floats per
  // row); a reduce kernel then sums them in split order and runs the epilogue.
  int splits;
  float* partial;
  int partial_pitch;
};

struct SimtArgs {
  GemmCommon c;
  const float* x;           // [T, d] (shared rows read x directly)
  const float* xg;          // [R, d]
  const float* gate_up;     // [E, 2F, d]
  const float* gate_up_bias;// [E, 2F] or null
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
  const void* gate_up;      // [E, 2F, d] bf16
  const void* gate_up_bias; // [E, 2F] bf16 or null
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
cudaError_t launch_tc2_gate_up(const TcArgs& a, cudaStream_t st);  // CTA-pair variants
cudaError_t launch_tc2_down(const TcArgs& a, cudaStream_t st);
// Split-K reductions (partials -> epilogue) for the bf16 tensor-core GEMMs.
cudaError_t launch_splitk_gate_up_reduce(const TcArgs& a, cudaStream_t st);
cudaError_t launch_splitk_down_reduce(const TcArgs& a, cudaStream_t st);
// Split count for a GEMM of at most `tiles` tiles of `nkb` k-blocks on `sms` SMs.
int choose_splits(int64_t tiles, int nkb, int sms);
// MXFP4 expert stacks (gate_up / down are e2m1 codes); no shared expert.
cudaError_t launch_fp4_gate_up(const TcArgs& a, cudaStream_t st);
cudaError_t launch_fp4_down(const TcArgs& a, cudaStream_t st);
constexpr int kFp4BM = 256;       // activation rows per MXFP4 tile (the MMA's N, trimmed to the live rows)
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

}  // namespace moe
