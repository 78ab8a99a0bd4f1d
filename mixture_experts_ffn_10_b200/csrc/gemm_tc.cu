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
  GemmCommon c;                  // gate_up (MODE 0 and 2) or down (MODE 1)
  const uint16_t* gate_up_bias;  // [E, 2F] ([E, F] unfused / plain) or null
  const uint16_t* gate_bias;     // unfused: [E, F] or null
  const uint16_t* down_bias;     // [E, d] or null
  const float* roww;             // [R]
  uint16_t* out;                 // h [rows, Fmax] (MODE 0 and 2) or Y [rows, d] (MODE 1)
  GemmCommon c2;                 // MODE 2: the down GEMM of the same forward
  uint16_t* out2;                // MODE 2: Y [rows, d]
  int32_t* ready;                // MODE 2: [NS] finished h regions per segment
};

// A work unit: split sp (of S) of tile `tile` of the gate_up GEMM or (dn) of the down
// GEMM, K blocks kb0 .. kb1-1.  MODE 2 numbers the gate_up units first, then the
// down units (u1 = the number of gate_up units).
struct Unit {
  Tile t;
  int tile, sp, S, kb0, kb1;
  bool dn;
};

template <int MODE>
__device__ __forceinline__ Unit unit_of(const TcParams& p, int unit, int u1) {
  Unit u;
  u.dn = MODE == 1 || (MODE == 2 && unit >= u1);
  const GemmCommon& c = (MODE == 2 && u.dn) ? p.c2 : p.c;
  const int local = (MODE == 2 && u.dn) ? unit - u1 : unit;
  u.S = c.splits;
  u.tile = local / u.S;
  u.sp = local % u.S;
  u.t = decode_tile<BM>(c, u.tile);
  const bool sh = u.t.seg >= c.E;
  const int K = u.dn ? (sh ? c.Fs : c.F) : c.d;
  const int nkb = (K + BK - 1) / BK;
  u.kb0 = u.sp * nkb / u.S;
  u.kb1 = (u.sp + 1) * nkb / u.S;
  return u;
}

// h regions (one per epilogue warp and gate_up tile) of segment `seg` that the MODE 2
// down tiles of the segment wait for (the segment's tiles are visited in segment order).
__device__ __forceinline__ int h_regions(const GemmCommon& gu, int seg) {
  return (gu.tiles[seg + 1] - gu.tiles[seg]) * kEpiWarps;
}

// Bounded wait until *ctr >= need.  On a timeout it records MOE_ERR_TIMEOUT and sets
// the CTA's abort flag (later waits then return at once, and the other roles stop);
// the h rows then read are not final, and the forward reports the error.
__device__ __forceinline__ void wait_count(const int32_t* ctr, int need, volatile int* abort, int* status) {
  if (ld_acquire_gpu(ctr) >= need || *abort) return;
  const uint64_t t0 = global_timer();
  while (ld_acquire_gpu(ctr) < need) {
    if (*abort) return;
    if (global_timer() - t0 > kTimeoutNs) {
      *abort = 1;
      set_status(status, MOE_ERR_TIMEOUT);
      return;
    }
    __nanosleep(64);
  }
}

// Whole warp: counts this warp's split of a region done (after its partial stores);
// true in every lane for the last of the S splits, which then sees all partials.
__device__ __forceinline__ bool split_arrive(int32_t* ctr, int S, int lane) {
  __threadfence();
  __syncwarp();
  int old = 0;
  if (lane == 0) old = atomicAdd(ctr, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old != S - 1) return false;
  __threadfence();
  return true;
}

// Whole warp: publishes this warp's finished h region (after its stores) to the
// MODE 2 down tiles, whose h loads go through the async proxy.
__device__ __forceinline__ void signal_region(int32_t* ctr, int lane) {
  __threadfence();
  fence_proxy_async_global();
  __syncwarp();
  if (lane == 0) atomicAdd(ctr, 1);
}

// 16 accumulator columns of one row summed over the S (<= 8) split partials in split
// order, as fp32 bits; the loads of four splits at a time are issued before their sums
// (not inlined: the gate and up sums of a chunk then do not hold their loads at once).
__device__ __noinline__ void sum_splits(const float* row, int64_t split_stride, int S, uint32_t (&v)[16]) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; i++) a[i] = 0.f;
#pragma unroll 1
  for (int s0 = 0; s0 < S; s0 += 4) {
    float4 q[4][4];
#pragma unroll
    for (int j = 0; j < 4; j++)
      if (s0 + j < S) {
#pragma unroll
        for (int i = 0; i < 4; i++)
          q[j][i] = __ldcg(reinterpret_cast<const float4*>(row + (s0 + j) * split_stride) + i);
      }
#pragma unroll
    for (int j = 0; j < 4; j++)
      if (s0 + j < S) {
#pragma unroll
        for (int i = 0; i < 4; i++) {
          a[4 * i] += q[j][i].x;
          a[4 * i + 1] += q[j][i].y;
          a[4 * i + 2] += q[j][i].z;
          a[4 * i + 3] += q[j][i].w;
        }
      }
  }
#pragma unroll
  for (int i = 0; i < 16; i++) v[i] = __float_as_uint(a[i]);
}

// The same for two 16-column groups of the row at once (a gate chunk and its up
// partner): the loads of three slots of both at a time are issued before their sums.
__device__ __noinline__ void sum_splits_pair(const float* ra, const float* rb, int64_t split_stride, int S,
                                             uint32_t (&va)[16], uint32_t (&vb)[16]) {
  float a[16], b[16];
#pragma unroll
  for (int i = 0; i < 16; i++) a[i] = b[i] = 0.f;
#pragma unroll 1
  for (int s0 = 0; s0 < S; s0 += 3) {
    float4 qa[3][4], qb[3][4];
#pragma unroll
    for (int j = 0; j < 3; j++)
      if (s0 + j < S) {
#pragma unroll
        for (int i = 0; i < 4; i++) {
          qa[j][i] = __ldcg(reinterpret_cast<const float4*>(ra + (s0 + j) * split_stride) + i);
          qb[j][i] = __ldcg(reinterpret_cast<const float4*>(rb + (s0 + j) * split_stride) + i);
        }
      }
#pragma unroll
    for (int j = 0; j < 3; j++)
      if (s0 + j < S) {
#pragma unroll
        for (int i = 0; i < 4; i++) {
          a[4 * i] += qa[j][i].x;
          a[4 * i + 1] += qa[j][i].y;
          a[4 * i + 2] += qa[j][i].z;
          a[4 * i + 3] += qa[j][i].w;
          b[4 * i] += qb[j][i].x;
          b[4 * i + 1] += qb[j][i].y;
          b[4 * i + 2] += qb[j][i].z;
          b[4 * i + 3] += qb[j][i].w;
        }
      }
  }
#pragma unroll
  for (int i = 0; i < 16; i++) {
    va[i] = __float_as_uint(a[i]);
    vb[i] = __float_as_uint(b[i]);
  }
}

// Column chunks of a tile's accumulator row: a gated gate_up chunk ch is gate columns
// 16ch .. 16ch+15 with their up partners 128 columns on (8 chunks); plain gate_up and
// down chunks are 16 columns each (16 chunks).
__device__ __forceinline__ int chunks_of(const GemmCommon& c, bool dn) {
  return (!dn && c.ffn != MOE_FFN_PLAIN) ? (BNB / 2) / 16 : BNB / 16;
}

// The epilogue of chunk ch of one accumulator row (output row grow, weigh-inputs
// scale wi), stored if `store`; fetch(col, v) yields columns col .. col+15 of the row,
// fetch2(c1, c2, v1, v2) two such groups (called whether or not the chunk is stored:
// TMEM loads are whole-warp).
template <typename Fetch, typename Fetch2>
__device__ __forceinline__ void emit_chunk(const TcParams& p, const GemmCommon& c, bool dn, uint16_t* out,
                                           const Tile& t, bool store, int64_t grow, float wi, int ch,
                                           Fetch&& fetch, Fetch2&& fetch2) {
  const bool sh = t.seg >= c.E;
  if (!dn && c.ffn == MOE_FFN_PLAIN) {
    const int F = sh ? c.Fs : c.F;
    const uint16_t* bias = (!sh && p.gate_up_bias) ? p.gate_up_bias + (int64_t)t.seg * c.F : nullptr;
    uint32_t v[16];
    fetch(ch * 16, v);
    const int fb = t.n_blk * BNB + ch * 16;
    if (store && fb < F) plain_chunk(v, bias, fb, F, c.act, wi, out + grow * c.Fmax);
  } else if (!dn) {
    const int F = sh ? c.Fs : c.F;
    const GuBias gb = sh ? GuBias{nullptr, nullptr, 1} : gu_bias(c.gu_layout, c.F, t.seg, p.gate_up_bias, p.gate_bias);
    uint32_t g[16], u[16];
    fetch2(ch * 16, BNB / 2 + ch * 16, g, u);
    const int fb = t.n_blk * (BNB / 2) + ch * 16;
    if (store && fb < F) gate_up_chunk(g, u, gb.g, gb.u, gb.stride, fb, F, c.act, wi, out + grow * c.Fmax);
  } else {
    const uint16_t* bias = (!sh && p.down_bias) ? p.down_bias + (int64_t)t.seg * c.d : nullptr;
    uint32_t v[16];
    fetch(ch * 16, v);
    const int ob = t.n_blk * BNB + ch * 16;
    if (store && ob < c.d) {
      const float w = (sh || c.weigh_inputs) ? 1.f : p.roww[grow];
      down_chunk(v, bias, ob, c.d, w, out + grow * c.d);
    }
  }
}

// MODE 0: gate_up; 1: down; 2: gate_up then down in one launch (small batches with x
// read in place).  In MODE 2 a CTA's producer, reaching a down tile of a segment
// whose h rows are not all written yet, loads the weights of the tile's first stages
// and waits for the segment's count of finished h regions before loading the h rows.
// Every CTA takes its gate_up units before its down units, and a gate_up unit waits
// on no other CTA, so the waits end once every CTA runs (one per SM, a cooperative
// launch).
template <int MODE, int ABOX>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBs,
                   const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmA2,
                   const __grid_constant__ CUtensorMap tmAs2, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmBs2, const TcParams p) {
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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* const status = p.c.status;

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
    if (MODE != 1 && p.c.gu_layout == MOE_GU_UNFUSED) prefetch_tmap(&tmG);
    if (MODE == 2) {
      prefetch_tmap(&tmA2);
      prefetch_tmap(&tmAs2);
      prefetch_tmap(&tmB2);
      prefetch_tmap(&tmBs2);
    }
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
  // Work units: (tile, split) of the GEMM (MODE 2: of gate_up, then of down).  Split
  // sp of a tile covers k-blocks [sp * nkb / S, (sp + 1) * nkb / S) of its K range.
  const int u1 = tile_total(p.c) * p.c.splits;
  const int total = u1 + (MODE == 2 ? tile_total(p.c2) * p.c2.splits : 0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // the activation rows of k-block kb (x, gathered rows, or h)
      auto issue_a = [&](const Unit& u, int kb, uint64_t* bar, uint8_t* sa) {
        const GemmCommon& c = (MODE == 2 && u.dn) ? p.c2 : p.c;
        const bool sh = u.t.seg >= c.E;
        const int arow = (sh || (!u.dn && c.direct_x)) ? u.t.m0 : c.off[u.t.seg] + u.t.m0;
        const CUtensorMap* m = (MODE == 2 && u.dn) ? (sh ? &tmAs2 : &tmA2) : (sh ? &tmAs : &tmA);
        tma_load_2d(m, bar, sa, kb * BK, arow);
      };
      // the 256 weight rows of k-block kb
      auto issue_b = [&](const Unit& u, int kb, uint64_t* bar, uint8_t* sb) {
        const GemmCommon& c = (MODE == 2 && u.dn) ? p.c2 : p.c;
        const bool sh = u.t.seg >= c.E;
        const int e = sh ? 0 : u.t.seg;
        const int k0 = kb * BK;
        if (u.dn) {
          const CUtensorMap* m = MODE == 2 ? (sh ? &tmBs2 : &tmB2) : (sh ? &tmBs : &tmB);
          tma_load_3d(m, bar, sb, k0, u.t.n_blk * BNB, e);  // 256 rows of down [E][d][F]
        } else if (c.ffn == MOE_FFN_PLAIN) {
          tma_load_3d(sh ? &tmBs : &tmB, bar, sb, k0, u.t.n_blk * BNB, e);  // 256 rows of fc1 [E][F][d]
        } else if (c.gu_layout == MOE_GU_UNFUSED && !sh) {
          const int f0 = u.t.n_blk * (BNB / 2);  // 128 gate rows, then the 128 up rows
          tma_load_3d(&tmG, bar, sb, k0, f0, e);
          tma_load_3d(&tmB, bar, sb + B_BYTES / 2, k0, f0, e);
        } else {
          const int f0 = u.t.n_blk * (BNB / 2);
          const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
          for (int half = 0; half < 2; half++) {
            const int c1 = il ? half : f0, c2 = il ? f0 : half;
            tma_load_4d(sh ? &tmBs : &tmB, bar, sb + half * (B_BYTES / 2), k0, c1, c2, e);
          }
        }
      };
      uint32_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; ok && unit < total; unit += gridDim.x) {
        const Unit u = unit_of<MODE>(p, unit, u1);
        // MODE 2 down unit whose h rows are not complete: the first `pre` stages get
        // their weights now and their h tiles once the rows are ready
        int pre = 0, need = 0;
        if (MODE == 2 && u.dn && u.t.seg < p.c.NS) {
          need = h_regions(p.c, u.t.seg);
          if (ld_acquire_gpu(p.ready + u.t.seg) < need) pre = min(u.kb1 - u.kb0, STAGES);
        }
        for (int kb = u.kb0; kb < u.kb1; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, status)) {
            // stages that hold weights without their h tile get it, so that every
            // issued stage completes before the CTA exits
            const int held = kb - u.kb0 < pre ? kb - u.kb0 : 0;
            for (int j = 0; j < held; j++) {
              const uint32_t i2 = it - held + j;
              issue_a(u, u.kb0 + j, &full[i2 % STAGES], smem + (i2 % STAGES) * STAGE_BYTES);
            }
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          uint8_t* sa = smem + s * STAGE_BYTES;
          issue_b(u, kb, &full[s], sa + A_BYTES);
          if (kb - u.kb0 >= pre) {
            issue_a(u, kb, &full[s], sa);
          } else if (kb - u.kb0 == pre - 1) {
            wait_count(p.ready + u.t.seg, need, abort_flag, status);
            fence_proxy_async_global();
            for (int j = 0; j < pre; j++) {
              const uint32_t i2 = it - (pre - 1) + j;
              issue_a(u, u.kb0 + j, &full[i2 % STAGES], smem + (i2 % STAGES) * STAGE_BYTES);
            }
          }
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
        const Unit u = unit_of<MODE>(p, unit, u1);
        const int acc = tcount & 1;
        if (!mbar_wait(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + acc * ACC_COLS;
        for (int kb = u.kb0; kb < u.kb1; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t ad = sdesc_k_sw128(sa), bd = sdesc_k_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++)
            mma_bf16(dt, ad + 2 * kk, bd + 2 * kk, IDESC, (kb > u.kb0 || kk > 0) ? 1u : 0u);
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
    const int region = warp - 2;       // this warp's region of a tile (split-K, h readiness)
    const int r_in_tile = q * 32 + lane;
    uint32_t tcount = 0;
    for (int unit = blockIdx.x; unit < total; unit += gridDim.x, tcount++) {
      const Unit u = unit_of<MODE>(p, unit, u1);
      const GemmCommon& c = (MODE == 2 && u.dn) ? p.c2 : p.c;
      uint16_t* out = (MODE == 2 && u.dn) ? p.out2 : p.out;
      const Tile& t = u.t;
      const bool sh = t.seg >= c.E;
      const int acc = tcount & 1;
      if (!mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      const int row = t.m0 + r_in_tile;
      bool valid = row < t.rows;
      int64_t grow = (int64_t)c.off[t.seg] + row;
      float wi = 1.f;  // weigh-inputs scale of the accumulators (direct_x only)
      if (!u.dn && c.direct_x && !sh) {
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
      const bool any = __any_sync(0xffffffffu, valid);
      auto from_tmem = [&](int col, uint32_t (&v)[16]) {
        tmem_ld16(tb + col, v);
        tmem_ld_wait();
      };
      auto from_tmem2 = [&](int c1, int c2, uint32_t (&v1)[16], uint32_t (&v2)[16]) {
        tmem_ld16(tb + c1, v1);
        tmem_ld16(tb + c2, v2);
        tmem_ld_wait();
      };
      bool final_region = true;  // this warp's region of the tile holds its final output
      if (u.S > 1) {
        // split-K: this split's fp32 partial accumulators, then the last split of
        // the region to arrive sums them all and runs the epilogue
        const int64_t split_stride = (int64_t)(c.R + (c.Fs > 0 ? c.T : 0)) * c.partial_pitch;
        float* prow = c.partial + (int64_t)u.sp * split_stride + grow * c.partial_pitch + t.n_blk * ACC_COLS;
        if (any) {
          // two chunks per TMEM wait
          constexpr int kGroup = 2;
#pragma unroll 1
          for (int c0 = part; c0 < ACC_COLS / 16; c0 += kGroup * kEpiGroups) {
            uint32_t v[kGroup][16];
#pragma unroll
            for (int j = 0; j < kGroup; j++)
              if (c0 + j * kEpiGroups < ACC_COLS / 16) tmem_ld16(tb + (c0 + j * kEpiGroups) * 16, v[j]);
            tmem_ld_wait();
            if (valid) {
#pragma unroll
              for (int j = 0; j < kGroup; j++) {
                const int ch = c0 + j * kEpiGroups;
                if (ch >= ACC_COLS / 16) break;
                float4* dst = reinterpret_cast<float4*>(prow + ch * 16);
#pragma unroll
                for (int i = 0; i < 4; i++)
                  dst[i] = make_float4(__uint_as_float(v[j][4 * i]), __uint_as_float(v[j][4 * i + 1]),
                                       __uint_as_float(v[j][4 * i + 2]), __uint_as_float(v[j][4 * i + 3]));
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        final_region = split_arrive(c.fix + (int64_t)u.tile * kFixRegions + region, u.S, lane);
        if (final_region && any) {
          // (row, chunk) items of the region spread over the lanes, so that the
          // partials of up to 32 chunks are in flight at once
          const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
          const int nch = (chunks_of(c, u.dn) - part + kEpiGroups - 1) / kEpiGroups;
          const int items = __popc(vmask) * nch;
          for (int base = 0; base < items; base += 32) {
            const int item = base + lane;
            const int ri = item < items ? item / nch : 0;
            uint32_t m = vmask;  // the lane holding the ri-th valid row
            for (int i = 0; i < ri; i++) m &= m - 1;
            const int src = __ffs(m) - 1;
            const int64_t g_row = __shfl_sync(0xffffffffu, grow, src);
            const float w_row = __shfl_sync(0xffffffffu, wi, src);
            if (item < items) {
              const float* row0 = c.partial + g_row * c.partial_pitch + t.n_blk * ACC_COLS;
              emit_chunk(p, c, u.dn, out, t, true, g_row, w_row, part + (item % nch) * kEpiGroups,
                         [&](int col, uint32_t (&v)[16]) { sum_splits(row0 + col, split_stride, u.S, v); },
                         [&](int c1, int c2, uint32_t (&v1)[16], uint32_t (&v2)[16]) {
                           sum_splits_pair(row0 + c1, row0 + c2, split_stride, u.S, v1, v2);
                         });
            }
          }
        }
      } else {
        if (any) {
#pragma unroll 1
          for (int ch = part; ch < chunks_of(c, u.dn); ch += kEpiGroups)
            emit_chunk(p, c, u.dn, out, t, valid, grow, wi, ch, from_tmem, from_tmem2);
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      }
      if (MODE == 2 && !u.dn && final_region) signal_region(p.ready + t.seg, lane);
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

// The kernel's tensor maps: gate_up (a, as, b, bs, g) and, for MODE 2, down (a2 .. bs2).
// Maps a mode does not read are copies of a used one.
struct Maps {
  CUtensorMap a, as, b, bs, g, a2, as2, b2, bs2;
};

template <int MODE, int ABOX>
cudaError_t launch_box(const Maps& m, const TcParams& p, int num_sms, cudaStream_t st) {
  constexpr int smem = Stage<ABOX>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<MODE, ABOX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int units = p.c.max_tiles * p.c.splits + (MODE == 2 ? p.c2.max_tiles * p.c2.splits : 0);
  const int grid = units < num_sms ? units : num_sms;
  if (MODE == 2)  // CTAs wait for h regions that other CTAs write: all must be resident
    return launch_coop_pdl(tc_gemm_kernel<MODE, ABOX>, (unsigned)grid, kThreads, smem, st, m.a, m.as, m.b, m.bs,
                           m.g, m.a2, m.as2, m.b2, m.bs2, p);
  return launch_pdl(tc_gemm_kernel<MODE, ABOX>, (unsigned)grid, kThreads, smem, st, m.a, m.as, m.b, m.bs, m.g, m.a2,
                    m.as2, m.b2, m.bs2, p);
}

// Activation rows each stage loads: no segment has more rows than there are tokens.
int a_box_rows(const GemmCommon& c) { return c.T <= 32 ? 32 : c.T <= 64 ? 64 : BM; }

template <int MODE>
cudaError_t launch(const Maps& m, const TcParams& p, int abox, int num_sms, cudaStream_t st) {
  if (abox == 32) return launch_box<MODE, 32>(m, p, num_sms, st);
  if (abox == 64) return launch_box<MODE, 64>(m, p, num_sms, st);
  if (MODE == 2) return cudaErrorInvalidValue;  // only batches of at most 64 tokens
  return launch_box<MODE == 2 ? 0 : MODE, BM>(m, p, num_sms, st);
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

namespace {

// gate_up maps: activation rows (x itself for direct_x, else the gathered rows), the
// weight stack, the shared expert's rows and stack, the unfused gate stack.
bool gate_up_maps(const TcArgs& a, int abox, Maps* m) {
  const GemmCommon& c = a.c;
  bool ok = c.direct_x ? map_rows(&m->a, a.x, c.d, c.T, c.d, abox) : map_rows(&m->a, a.xg, c.d, c.R, c.d, abox);
  ok = ok && map_fc1(&m->b, a.gate_up, c.d, c.F, c.E, c.ffn, c.gu_layout);
  if (c.gu_layout == MOE_GU_UNFUSED) ok = ok && map_fc1(&m->g, a.gate, c.d, c.F, c.E, c.ffn, c.gu_layout);
  else m->g = m->b;
  if (c.Fs > 0) {
    // the shared expert keeps one stack (gate rows first when the routed experts are unfused)
    const int sh_layout = c.gu_layout == MOE_GU_UNFUSED ? MOE_GU_CONCAT : c.gu_layout;
    ok = ok && map_rows(&m->as, a.x, c.d, c.T, c.d, abox);
    ok = ok && map_fc1(&m->bs, a.sh_gate_up, c.d, c.Fs, 1, c.ffn, sh_layout);
  } else {
    m->as = m->a;
    m->bs = m->b;
  }
  return ok;
}

// down maps: h rows (routed, then the shared expert's at R), the down stacks.
bool down_maps(const TcArgs& a, const GemmCommon& c, int abox, CUtensorMap* mA, CUtensorMap* mAs, CUtensorMap* mB,
               CUtensorMap* mBs) {
  bool ok = map_rows(mA, a.h, c.F, c.R, c.Fmax, abox);
  ok = ok && map_down(mB, a.down, c.F, c.d, c.E);
  if (c.Fs > 0) {
    ok = ok && map_rows(mAs, (const uint16_t*)a.h + (int64_t)c.R * c.Fmax, c.Fs, c.T, c.Fmax, abox);
    ok = ok && map_down(mBs, a.sh_down, c.Fs, c.d, 1);
  } else {
    *mAs = *mA;
    *mBs = *mB;
  }
  return ok;
}

}  // namespace

cudaError_t launch_tc_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  Maps m;
  const int abox = a_box_rows(c);
  if (!gate_up_maps(a, abox, &m)) return cudaErrorInvalidValue;
  m.a2 = m.as2 = m.b2 = m.bs2 = m.b;
  TcParams p{c, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias, nullptr, a.roww, (uint16_t*)a.h};
  return launch<0>(m, p, abox, a.num_sms, st);
}

cudaError_t launch_tc_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  Maps m;
  const int abox = a_box_rows(c);
  if (!down_maps(a, c, abox, &m.a, &m.as, &m.b, &m.bs)) return cudaErrorInvalidValue;
  m.g = m.a2 = m.as2 = m.b2 = m.bs2 = m.b;
  TcParams p{c, nullptr, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(m, p, abox, a.num_sms, st);
}

cudaError_t launch_tc_ffn(const TcArgs& a, const GemmCommon& dn, int32_t* ready, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  Maps m;
  const int abox = a_box_rows(c);
  if (!c.direct_x || c.order || !ready || abox > 64) return cudaErrorInvalidValue;
  if (!gate_up_maps(a, abox, &m) || !down_maps(a, dn, abox, &m.a2, &m.as2, &m.b2, &m.bs2))
    return cudaErrorInvalidValue;
  TcParams p{c, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias, (const uint16_t*)a.down_bias,
             a.roww, (uint16_t*)a.h, dn, (uint16_t*)a.Y, ready};
  return launch<2>(m, p, abox, a.num_sms, st);
}

}  // namespace moe
