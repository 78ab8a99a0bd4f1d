// gemm_tc.cu -- bf16 grouped GEMMs on the sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
//   gate_up (MODE 0): per expert e and row r of its segment,
//       g = W_gate[e] . x_r + b_gate,  u = W_up[e] . x_r + b_up,  h = gated(g, u) -> bf16
//   down    (MODE 1): Y_r = (W_down[e] . h_r + b_down) * w_r -> bf16
// (graph-op page "MoE": fc1 [E, 2*inter, hidden] fused gate||up, swiglu_fusion
// interleaved or not; fc2 [E, hidden, inter]; "Struct MoeSpec" biases, act,
// weigh_inputs).  The shared expert is one more segment whose rows are x itself.
//
// One persistent CTA per SM walks the device-computed tile list (segment-major,
// then N block, then M block, so CTAs working at the same time share a weight
// tile through L2).  Warp roles:
//   warp 0     TMA producer: A tile 128 x 64 (32 or 64 rows for batches of at most
//              that many tokens) and B tile 256 x 64 (bf16, 128-byte swizzle) per
//              stage into a 4-stage (5, 6 with the smaller A tiles) shared-memory ring;
//   warp 1     TMEM allocator and MMA issuer: tcgen05.mma M=128 N=256 K=16,
//              fp32 accumulators in TMEM, two accumulator buffers of 256 columns;
//   warps 2-5  epilogue: tcgen05.ld the accumulator rows, bias + activation (or
//              bias x routing weight), bf16 stores; overlaps the next tile's MMAs.
// For gate_up the B tile is 128 gate rows followed by the 128 matching up rows,
// fetched through a 4-D tensor map view of the stack that hides the layout:
// concat [E][2][F][d] or interleaved [E][F][2][d].  So accumulator column j
// (< 128) is gate feature f0 + j and column 128 + j its up partner.
#include "epilogue.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = kTcBM;            // 128 rows per tile (the MMA's M)
constexpr int BK = 64;               // K per stage: 128-byte swizzled rows
constexpr int BNB = 256;             // B rows per tile
constexpr int B_BYTES = BNB * BK * 2;
// Stage layout for ABOX loaded activation rows (128, or 64 / 32 when no segment
// can have more rows, i.e. small batches): [ABOX x 64 bf16][256 x 64 bf16].  The
// MMA always reads 128 A rows; rows past ABOX alias the stage's B tile and only
// feed accumulator rows that are never stored (row i of D depends on row i of
// A alone).  Smaller A tiles leave room for more stages of weights in flight.
template <int ABOX>
struct Stage {
  static constexpr int A_BYTES = ABOX * BK * 2;
  static constexpr int BYTES = A_BYTES + B_BYTES;  // 48, 40 or 36 KiB (1024-aligned)
  static constexpr int COUNT = ABOX == 128 ? 4 : ABOX == 64 ? 5 : 6;
  static constexpr int SMEM = COUNT * BYTES + 1024 /*align*/ + 256 /*barriers*/;
};
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
#ifndef MOE_TC_EPI_WARPS
#define MOE_TC_EPI_WARPS 4
#endif
constexpr int kEpiWarps = MOE_TC_EPI_WARPS;  // 4, or 8 = two per TMEM lane quadrant splitting the chunks
constexpr int kEpiGroups = kEpiWarps / 4;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BNB);

struct TcParams {
  GemmCommon c;
  const uint16_t* gate_up_bias;  // [E, 2F] ([E, F] unfused / plain) or null
  const uint16_t* gate_bias;     // unfused: [E, F] or null
  const uint16_t* down_bias;     // [E, d] or null
  const float* roww;             // [R]
  uint16_t* out;                 // h [rows, Fmax] or Y [rows, d]
};

template <int MODE>
__device__ __forceinline__ int k_extent(const GemmCommon& c, bool shared) {
  return MODE == 0 ? c.d : (shared ? c.Fs : c.F);
}

template <int MODE, int ABOX>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBs,
                   const __grid_constant__ CUtensorMap tmG, const TcParams p) {
  constexpr int STAGES = Stage<ABOX>::COUNT, STAGE_BYTES = Stage<ABOX>::BYTES, A_BYTES = Stage<ABOX>::A_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const GemmCommon& c = p.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmAs);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmBs);
    if (MODE == 0 && c.gu_layout == MOE_GU_UNFUSED) prefetch_tmap(&tmG);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_enter();
  const uint32_t tmem_base = *tmem_slot;
  // Work units: (tile, split).  Split sp of a tile covers k-blocks
  // [sp * nkb / S, (sp + 1) * nkb / S) of the tile's K range.
  const int S = c.splits;
  const int total = c.tiles[c.NS] * S;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      auto issue = [&](const Tile& t, int kb, uint64_t* bar, uint8_t* sa) {
        const bool sh = t.seg >= c.E;
        const int arow = (sh || (MODE == 0 && c.direct_x)) ? t.m0 : c.off[t.seg] + t.m0;
        const CUtensorMap* mA = sh ? &tmAs : &tmA;
        const CUtensorMap* mB = sh ? &tmBs : &tmB;
        const int e = sh ? 0 : t.seg;
        const int k0 = kb * BK;
        tma_load_2d(mA, bar, sa, k0, arow);
        if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
          tma_load_3d(mB, bar, sa + A_BYTES, k0, t.n_blk * BNB, e);  // 256 rows of fc1 [E][F][d]
        } else if (MODE == 0 && c.gu_layout == MOE_GU_UNFUSED && !sh) {
          const int f0 = t.n_blk * (BNB / 2);  // 128 gate rows, then the 128 up rows
          tma_load_3d(&tmG, bar, sa + A_BYTES, k0, f0, e);
          tma_load_3d(mB, bar, sa + A_BYTES + B_BYTES / 2, k0, f0, e);
        } else if (MODE == 0) {
          const int f0 = t.n_blk * (BNB / 2);
          const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
          for (int half = 0; half < 2; half++) {
            const int c1 = il ? half : f0, c2 = il ? f0 : half;
            tma_load_4d(mB, bar, sa + A_BYTES + half * (B_BYTES / 2), k0, c1, c2, e);
          }
        } else {
          tma_load_3d(mB, bar, sa + A_BYTES, k0, t.n_blk * BNB, e);
        }
      };
      uint32_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; ok && unit < total; unit += gridDim.x) {
        const Tile t = decode_tile<BM>(c, unit / S);
        const int nkb = (k_extent<MODE>(c, t.seg >= c.E) + BK - 1) / BK;
        const int sp = unit % S, kb1 = (sp + 1) * nkb / S;
        for (int kb = sp * nkb / S; kb < kb1; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          issue(t, kb, &full[s], smem + s * STAGE_BYTES);
        }
      }
      // every load issued into a stage has landed before the CTA may exit
      for (uint32_t j = (it > (uint32_t)STAGES ? it - STAGES : 0); j < it; j++) {
        const uint64_t t0 = global_timer();
        while (!mbar_try_wait(&full[j % STAGES], (j / STAGES) & 1) && global_timer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int unit = blockIdx.x; ok && unit < total; unit += gridDim.x, tcount++) {
        const Tile t = decode_tile<BM>(c, unit / S);
        const bool sh = t.seg >= c.E;
        const int nkb = (k_extent<MODE>(c, sh) + BK - 1) / BK;
        const int sp = unit % S, kb0 = sp * nkb / S, kb1 = (sp + 1) * nkb / S;
        const int acc = tcount & 1;
        if (!mbar_wait(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, c.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + acc * ACC_COLS;
        for (int kb = kb0; kb < kb1; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t ad = sdesc_k_sw128(sa), bd = sdesc_k_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++)
            mma_bf16(dt, ad + 2 * kk, bd + 2 * kk, IDESC, (kb > kb0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      // all issued MMAs complete before TMEM is released
      mma_commit(drain);
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(drain, 0) && global_timer() - t0 < kTimeoutNs) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // this warp may read TMEM lanes 32q .. 32q+31
    const int part = (warp - 2) / 4;   // which alternate column chunks this warp drains
    const int r_in_tile = q * 32 + lane;
    uint32_t tcount = 0;
    for (int unit = blockIdx.x; unit < total; unit += gridDim.x, tcount++) {
      const Tile t = decode_tile<BM>(c, unit / S);
      const bool sh = t.seg >= c.E;
      const int acc = tcount & 1;
      if (!mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      const int row = t.m0 + r_in_tile;
      bool valid = row < t.rows;
      int64_t grow = (int64_t)c.off[t.seg] + row;
      float wi = 1.f;  // weigh-inputs scale of the accumulators (direct_x only)
      if (MODE == 0 && c.direct_x && !sh) {
        // accumulator row = token r_in_tile: its row of this expert, if it chose it
        valid = false;
        if (r_in_tile < c.T) {
          for (int j = 0; j < c.k; j++)
            if (c.topk_idx[(int64_t)r_in_tile * c.k + j] == t.seg) {
              grow = c.pos[(int64_t)r_in_tile * c.k + j];
              valid = true;
            }
        }
        if (valid && c.weigh_inputs) wi = p.roww[grow];
      }
      if (S > 1) {
        // split-K: this unit's fp32 partial accumulator row goes to the partial buffer
        if (__any_sync(0xffffffffu, valid)) {
          float* prow = c.partial + ((int64_t)(unit % S) * (c.R + (c.Fs > 0 ? c.T : 0)) + grow) * c.partial_pitch +
                        t.n_blk * ACC_COLS;
#pragma unroll 1
          for (int ch = part; ch < ACC_COLS / 16; ch += kEpiGroups) {
            uint32_t v[16];
            tmem_ld16(tb + ch * 16, v);
            tmem_ld_wait();
            if (valid) {
              float4* dst = reinterpret_cast<float4*>(prow + ch * 16);
#pragma unroll
              for (int i = 0; i < 4; i++)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          }
        }
      } else if (__any_sync(0xffffffffu, valid)) {
        if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
          const int F = sh ? c.Fs : c.F;
          const int f0 = t.n_blk * BNB;
          const uint16_t* bias = (!sh && p.gate_up_bias) ? p.gate_up_bias + (int64_t)t.seg * c.F : nullptr;
          uint16_t* out = p.out + grow * c.Fmax;
#pragma unroll 1
          for (int ch = part; ch < BNB / 16; ch += kEpiGroups) {
            uint32_t v[16];
            tmem_ld16(tb + ch * 16, v);
            tmem_ld_wait();
            const int fb = f0 + ch * 16;
            if (valid && fb < F) plain_chunk(v, bias, fb, F, c.act, wi, out);
          }
        } else if (MODE == 0) {
          const int F = sh ? c.Fs : c.F;
          const int f0 = t.n_blk * (BNB / 2);
          const GuBias gb = sh ? GuBias{nullptr, nullptr, 1}
                               : gu_bias(c.gu_layout, c.F, t.seg, p.gate_up_bias, p.gate_bias);
          uint16_t* out = p.out + grow * c.Fmax;
#pragma unroll 1
          for (int ch = part; ch < (BNB / 2) / 16; ch += kEpiGroups) {
            uint32_t g[16], u[16];
            tmem_ld16(tb + ch * 16, g);
            tmem_ld16(tb + BNB / 2 + ch * 16, u);
            tmem_ld_wait();
            const int fb = f0 + ch * 16;
            if (valid && fb < F) gate_up_chunk(g, u, gb.g, gb.u, gb.stride, fb, F, c.act, wi, out);
          }
        } else {
          const int n0 = t.n_blk * BNB;
          const uint16_t* bias = (!sh && p.down_bias) ? p.down_bias + (int64_t)t.seg * c.d : nullptr;
          const float w = (sh || c.weigh_inputs || !valid) ? 1.f : p.roww[grow];
          uint16_t* out = p.out + grow * c.d;
#pragma unroll 1
          for (int ch = part; ch < BNB / 16; ch += kEpiGroups) {
            uint32_t v[16];
            tmem_ld16(tb + ch * 16, v);
            tmem_ld_wait();
            const int ob = n0 + ch * 16;
            if (valid && ob < c.d) down_chunk(v, bias, ob, c.d, w, out);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

// bf16 tensor map with the swizzle the UMMA descriptors expect.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// rows x K matrix with row pitch `pitch` elements; box 64 x box_rows.
bool map_rows(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t pitch, uint32_t box_rows) {
  const uint64_t dims[2] = {K, rows > 0 ? rows : 1};
  const uint64_t strides[1] = {pitch * 2};
  const uint32_t box[2] = {BK, box_rows};
  return make_map(m, base, 2, dims, strides, box);
}

// Fused gate||up stack [E][2F][d] seen as 4-D so that one box is 128 gate (or up) rows.
bool map_gate_up(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int layout) {
  if (layout == MOE_GU_INTERLEAVED) {  // [E][F][2][d]: dims {d, 2, F, E}
    const uint64_t dims[4] = {d, 2, F, E};
    const uint64_t strides[3] = {d * 2, 2 * d * 2, 2 * F * d * 2};
    const uint32_t box[4] = {BK, 1, BNB / 2, 1};
    return make_map(m, base, 4, dims, strides, box);
  }
  const uint64_t dims[4] = {d, F, 2, E};  // [E][2][F][d]
  const uint64_t strides[3] = {d * 2, F * d * 2, 2 * F * d * 2};
  const uint32_t box[4] = {BK, BNB / 2, 1, 1};
  return make_map(m, base, 4, dims, strides, box);
}

// Down stack [E][d][F]: dims {F, d, E}, box 64 x 256 x 1.
bool map_down(CUtensorMap* m, const void* base, uint64_t F, uint64_t d, uint64_t E) {
  const uint64_t dims[3] = {F, d, E};
  const uint64_t strides[2] = {F * 2, d * F * 2};
  const uint32_t box[3] = {BK, BNB, 1};
  return make_map(m, base, 3, dims, strides, box);
}

template <int MODE, int ABOX>
cudaError_t launch_box(const CUtensorMap& a, const CUtensorMap& as, const CUtensorMap& b, const CUtensorMap& bs,
                       const CUtensorMap& g, const TcParams& p, int num_sms, cudaStream_t st) {
  constexpr int smem = Stage<ABOX>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<MODE, ABOX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int units = p.c.max_tiles * p.c.splits;
  const int grid = units < num_sms ? units : num_sms;
  return launch_pdl(tc_gemm_kernel<MODE, ABOX>, (unsigned)grid, kThreads, smem, st, a, as, b, bs, g, p);
}

// Activation rows each stage loads: no segment has more rows than there are tokens.
int a_box_rows(const GemmCommon& c) { return c.T <= 32 ? 32 : c.T <= 64 ? 64 : BM; }

template <int MODE>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& as, const CUtensorMap& b, const CUtensorMap& bs,
                   const CUtensorMap& g, const TcParams& p, int abox, int num_sms, cudaStream_t st) {
  if (abox == 32) return launch_box<MODE, 32>(a, as, b, bs, g, p, num_sms, st);
  if (abox == 64) return launch_box<MODE, 64>(a, as, b, bs, g, p, num_sms, st);
  return launch_box<MODE, BM>(a, as, b, bs, g, p, num_sms, st);
}

// Maps of one gate_up weight stack (E experts of F features): a plain fc1 [E][F][d]
// in boxes of 256 rows; an unfused gate or up stack [E][F][d] in boxes of 128 rows;
// a fused stack [E][2F][d] through the 4-D view.
bool map_fc1(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int ffn, int layout) {
  if (ffn == MOE_FFN_PLAIN) return map_down(m, base, d, F, E);  // same shape: {d, F, E}, box 64 x 256
  if (layout == MOE_GU_UNFUSED) {
    const uint64_t dims[3] = {d, F, E};
    const uint64_t strides[2] = {d * 2, F * d * 2};
    const uint32_t box[3] = {BK, BNB / 2, 1};
    return make_map(m, base, 3, dims, strides, box);
  }
  return map_gate_up(m, base, d, F, E, layout);
}

}  // namespace

cudaError_t launch_tc_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mAs, mB, mBs, mG;
  const int abox = a_box_rows(c);
  // small batches read the activation rows from x itself (direct_x), else the rows
  // gathered into expert order
  bool ok = c.direct_x ? map_rows(&mA, a.x, c.d, c.T, c.d, abox) : map_rows(&mA, a.xg, c.d, c.R, c.d, abox);
  ok = ok && map_fc1(&mB, a.gate_up, c.d, c.F, c.E, c.ffn, c.gu_layout);
  if (c.gu_layout == MOE_GU_UNFUSED) ok = ok && map_fc1(&mG, a.gate, c.d, c.F, c.E, c.ffn, c.gu_layout);
  else mG = mB;
  if (c.Fs > 0) {
    // the shared expert keeps one stack (gate rows first when the routed experts are unfused)
    const int sh_layout = c.gu_layout == MOE_GU_UNFUSED ? MOE_GU_CONCAT : c.gu_layout;
    ok = ok && map_rows(&mAs, a.x, c.d, c.T, c.d, abox);
    ok = ok && map_fc1(&mBs, a.sh_gate_up, c.d, c.Fs, 1, c.ffn, sh_layout);
  } else {
    mAs = mA;
    mBs = mB;
  }
  if (!ok) return cudaErrorInvalidValue;
  TcParams p{c, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias, nullptr, a.roww, (uint16_t*)a.h};
  return launch<0>(mA, mAs, mB, mBs, mG, p, abox, a.num_sms, st);
}

cudaError_t launch_tc_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mAs, mB, mBs;
  const int abox = a_box_rows(c);
  bool ok = map_rows(&mA, a.h, c.F, c.R, c.Fmax, abox);
  ok = ok && map_down(&mB, a.down, c.F, c.d, c.E);
  if (c.Fs > 0) {
    ok = ok && map_rows(&mAs, (const uint16_t*)a.h + (int64_t)c.R * c.Fmax, c.Fs, c.T, c.Fmax, abox);
    ok = ok && map_down(&mBs, a.sh_down, c.Fs, c.d, 1);
  } else {
    mAs = mA;
    mBs = mB;
  }
  if (!ok) return cudaErrorInvalidValue;
  TcParams p{c, nullptr, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(mA, mAs, mB, mBs, mB, p, abox, a.num_sms, st);
}

}  // namespace moe
