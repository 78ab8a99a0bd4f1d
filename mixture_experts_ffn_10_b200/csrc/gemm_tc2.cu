// gemm_tc2.cu -- the bf16 grouped GEMMs of gemm_tc.cu on CTA pairs (tcgen05 cta_group::2),
// for prefill-sized batches where every expert has hundreds of rows.
//
// Same operations as gemm_tc.cu (graph-op page "MoE": fc1 fused gate||up, fc2 down;
// "Struct MoeSpec" biases, activation, weigh_inputs):
//   gate_up (MODE 0): h = gated(W_gate[e] . x_r + b_gate, W_up[e] . x_r + b_up) -> bf16
//   down    (MODE 1): Y_r = (W_down[e] . h_r + b_down) * w_r -> bf16
//
// A cluster of two CTAs on neighbouring SMs owns one 256 x 256 output tile.  CTA r
// (r = 0, 1) stages A rows m0 + 128 r .. + 127 and B rows 128 r .. 128 r + 127 of
// the tile in its own shared memory; the even CTA issues one tcgen05.mma M=256
// N=256 K=16 per step, which reads both CTAs' operands and leaves rows
// 128 r .. 128 r + 127 of the fp32 accumulator in CTA r's tensor memory.  Per SM
// and per output element this moves two thirds of the bytes of the single-CTA
// 128 x 256 tile through TMA (32 KiB instead of 48 KiB per 64-deep K step), which
// is what limits the single-CTA kernel at large batch.
//
// For gate_up the B tile is 128 gate rows (staged by CTA 0) and the matching 128
// up rows (CTA 1), so accumulator column j < 128 is gate feature f0 + j and
// column 128 + j its up partner, exactly as in the single-CTA kernel.
//
// Warp roles in each CTA:
//   warp 0     TMA producer for this CTA's half of every stage; the loads complete
//              on the even CTA's `full` barrier, which the even CTA arms for the
//              bytes of both (no multicast loads);
//   warp 1     TMEM allocation for the pair; in the even CTA also the MMA issuer,
//              whose commits arrive on both CTAs' `empty` / `tfull` barriers;
//   warps 2-5  epilogue of this CTA's 128 accumulator rows; each warp signals the
//              even CTA's `tempty` barrier when it has read an accumulator buffer.
// Every wait is bounded (2 s) and reports MOE_ERR_TIMEOUT through the status word.
#include <atomic>

#include "epilogue.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM2 = kPairBM;          // 256 rows per cluster tile
constexpr int BMC = BM2 / 2;          // 128 rows per CTA
constexpr int BK = 64;                // K per stage (128-byte swizzled rows)
constexpr int BNB = 256;              // accumulator columns per tile
constexpr int BNC = BNB / 2;          // B rows staged per CTA
constexpr int STAGES = 6;
constexpr int A_BYTES = BMC * BK * 2;  // 16 KiB
constexpr int B_BYTES = BNC * BK * 2;  // 16 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int ACC_COLS = BNB;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t IDESC = idesc_bf16_f32(BM2, BNB);
constexpr uint16_t kBothCtas = 0x3;
constexpr uint16_t kEvenCta = 0x1;

struct Tc2Params {
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

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc2_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBs,
                    const __grid_constant__ CUtensorMap tmG, const Tc2Params p) {
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
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    // full / tempty are used in the even CTA only; empty / tfull in both.
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&full[s], 1);  // the even CTA's expect_tx covers both CTAs' loads
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmAs);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmBs);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barrier init and the TMEM address visible to both CTAs
  tc_fence_after();
  pdl_enter();
  const uint32_t tmem_base = *tmem_slot;
  const int S = 1;  // the plan never splits K for pair tiles (launch rejects it)
  const int total = tile_total(c);
  const int first = c.tiles[c.seg_begin];  // tiles of segments seg_begin .. NS-1 only

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int unit = first + cluster; ok && unit < total; unit += nclusters) {
        const Tile t = decode_tile<BM2>(c, unit / S);
        const bool sh = t.seg >= c.E;
        const int nkb = (k_extent<MODE>(c, sh) + BK - 1) / BK;
        const int sp = unit % S, kb1 = (sp + 1) * nkb / S;
        const int arow = (sh ? t.m0 : c.off[t.seg] + t.m0) + BMC * (int)rank;
        const CUtensorMap* mA = sh ? &tmAs : &tmA;
        const CUtensorMap* mB = sh ? &tmBs : &tmB;
        const int e = sh ? 0 : t.seg;
        for (int kb = sp * nkb / S; kb < kb1; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          // Only the even CTA arms the stage, for the bytes of both CTAs (every
          // box lands in full, zero-filled past the tensor's edge).  The odd
          // CTA's bytes may land first: the transaction count goes negative but
          // the phase cannot complete before the even CTA's arrival.  (A remote
          // arrival per stage from the odd CTA measured 2x slower.)
          const uint32_t fb = mapa_shared(&full[s], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
          uint8_t* sa = smem + s * STAGE_BYTES;
          const int k0 = kb * BK;
          tma_load_2d_pair(mA, fb, sa, k0, arow);
          if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
            // CTA r: fc1 rows n_blk * 256 + 128 r .. + 127
            tma_load_3d_pair(mB, fb, sa + A_BYTES, k0, t.n_blk * BNB + BNC * (int)rank, e);
          } else if (MODE == 0 && c.gu_layout == MOE_GU_UNFUSED && !sh) {
            // CTA 0: 128 rows of the gate stack, CTA 1: the matching up rows
            tma_load_3d_pair(rank == 0 ? &tmG : mB, fb, sa + A_BYTES, k0, t.n_blk * BNC, e);
          } else if (MODE == 0) {
            const int f0 = t.n_blk * BNC;
            const int half = (int)rank;  // CTA 0: gate rows, CTA 1: up rows
            const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
            tma_load_4d_pair(mB, fb, sa + A_BYTES, k0, il ? half : f0, il ? f0 : half, e);
          } else {
            tma_load_3d_pair(mB, fb, sa + A_BYTES, k0, t.n_blk * BNB + BNC * (int)rank, e);
          }
        }
      }
      // Every stage this CTA loaded has been consumed by the MMAs (so its bytes
      // have landed) before the CTA may exit.  The empty barriers see the same
      // commits in both CTAs.
      const uint64_t t0 = global_timer();
      for (uint32_t j = (it > (uint32_t)STAGES ? it - STAGES : 0); j < it; j++) {
        while (!mbar_try_wait(&empty[j % STAGES], (j / STAGES) & 1) && global_timer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int unit = first + cluster; ok && unit < total; unit += nclusters, tcount++) {
        const Tile t = decode_tile<BM2>(c, unit / S);
        const int nkb = (k_extent<MODE>(c, t.seg >= c.E) + BK - 1) / BK;
        const int sp = unit % S, kb0 = sp * nkb / S, kb1 = (sp + 1) * nkb / S;
        const int acc = tcount & 1;
        // the odd CTA's epilogue warps arrive here with cluster-scope release
        if (!mbar_wait_cluster(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, c.status)) break;
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
            mma_bf16_pair(dt, ad + 2 * kk, bd + 2 * kk, IDESC, (kb > kb0 || kk > 0) ? 1u : 0u);
          mma_commit_pair(&empty[s], kBothCtas);
        }
        if (ok) mma_commit_pair(&tfull[acc], kBothCtas);
      }
      // all issued MMAs complete before either CTA releases its tensor memory
      mma_commit_pair(drain, kEvenCta);
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(drain, 0) && global_timer() - t0 < kTimeoutNs) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;  // this warp may read TMEM lanes 32q .. 32q+31
    const int r_in_tile = BMC * (int)rank + q * 32 + lane;
    const uint32_t tempty_even0 = mapa_shared(&tempty[0], 0), tempty_even1 = mapa_shared(&tempty[1], 0);
    uint32_t tcount = 0;
    for (int unit = first + cluster; unit < total; unit += nclusters, tcount++) {
      const Tile t = decode_tile<BM2>(c, unit / S);
      const bool sh = t.seg >= c.E;
      const int acc = tcount & 1;
      // warp-uniform: the TMEM loads below need every lane of the warp
      const bool got = mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      const int row = t.m0 + r_in_tile;
      const bool valid = row < t.rows;
      const int64_t grow = (int64_t)c.off[t.seg] + row;
      if (__any_sync(0xffffffffu, valid)) {
        if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
          const int F = sh ? c.Fs : c.F;
          const int f0 = t.n_blk * BNB;
          const uint16_t* bias = (!sh && p.gate_up_bias) ? p.gate_up_bias + (int64_t)t.seg * c.F : nullptr;
          uint16_t* out = p.out + grow * c.Fmax;
#pragma unroll 1
          for (int ch = 0; ch < BNB / 16; ch++) {
            uint32_t v[16];
            tmem_ld16(tb + ch * 16, v);
            tmem_ld_wait();
            const int fb = f0 + ch * 16;
            if (valid && fb < F) plain_chunk(v, bias, fb, F, c.act, 1.f, out);
          }
        } else if (MODE == 0) {
          const int F = sh ? c.Fs : c.F;
          const int f0 = t.n_blk * BNC;
          const GuBias gb = sh ? GuBias{nullptr, nullptr, 1}
                               : gu_bias(c.gu_layout, c.F, t.seg, p.gate_up_bias, p.gate_bias);
          uint16_t* out = p.out + grow * c.Fmax;
#pragma unroll 1
          for (int ch = 0; ch < BNC / 16; ch++) {
            uint32_t g[16], u[16];
            tmem_ld16(tb + ch * 16, g);
            tmem_ld16(tb + BNC + ch * 16, u);
            tmem_ld_wait();
            const int fb = f0 + ch * 16;
            if (valid && fb < F) gate_up_chunk(g, u, gb.g, gb.u, gb.stride, fb, F, c.act, 1.f, out);
          }
        } else {
          const int n0 = t.n_blk * BNB;
          const uint16_t* bias = (!sh && p.down_bias) ? p.down_bias + (int64_t)t.seg * c.d : nullptr;
          const float w = (sh || c.weigh_inputs || !valid) ? 1.f : p.roww[grow];
          uint16_t* out = p.out + grow * c.d;
#pragma unroll 1
          for (int ch = 0; ch < BNB / 16; ch++) {
            uint32_t v[16];
            tmem_ld16(tb + ch * 16, v);
            tmem_ld_wait();
            const int ob = n0 + ch * 16;
            if (valid && ob < c.d) down_chunk(v, bias, ob, c.d, w, out);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_even1 : tempty_even0);
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // both CTAs done: MMAs drained, loads consumed, remote arrivals made
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// rows x K matrix with row pitch `pitch` elements; box 64 x 128.
bool map_rows(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t pitch) {
  const uint64_t dims[2] = {K, rows > 0 ? rows : 1};
  const uint64_t strides[1] = {pitch * 2};
  const uint32_t box[2] = {BK, BMC};
  return make_map(m, base, 2, dims, strides, box);
}

// Fused gate||up stack [E][2F][d] as 4-D so that one box is 128 gate (or up) rows.
bool map_gate_up(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int layout) {
  if (layout == MOE_GU_INTERLEAVED) {  // [E][F][2][d]: dims {d, 2, F, E}
    const uint64_t dims[4] = {d, 2, F, E};
    const uint64_t strides[3] = {d * 2, 2 * d * 2, 2 * F * d * 2};
    const uint32_t box[4] = {BK, 1, BNC, 1};
    return make_map(m, base, 4, dims, strides, box);
  }
  const uint64_t dims[4] = {d, F, 2, E};  // [E][2][F][d]
  const uint64_t strides[3] = {d * 2, F * d * 2, 2 * F * d * 2};
  const uint32_t box[4] = {BK, BNC, 1, 1};
  return make_map(m, base, 4, dims, strides, box);
}

// Down stack [E][d][F]: dims {F, d, E}, box 64 x 128 x 1.
bool map_down(CUtensorMap* m, const void* base, uint64_t F, uint64_t d, uint64_t E) {
  const uint64_t dims[3] = {F, d, E};
  const uint64_t strides[2] = {F * 2, d * F * 2};
  const uint32_t box[3] = {BK, BNC, 1};
  return make_map(m, base, 3, dims, strides, box);
}

// One CTA's half of a gate_up weight stack (E experts of F features), box 128 rows:
// a plain fc1 or an unfused gate or up stack [E][F][d] as 3-D; a fused stack
// [E][2F][d] through the 4-D view.
bool map_fc1(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int ffn, int layout) {
  if (ffn == MOE_FFN_PLAIN || layout == MOE_GU_UNFUSED) return map_down(m, base, d, F, E);
  return map_gate_up(m, base, d, F, E, layout);
}

// Co-resident clusters of the kernel on the current device (cached per device and mode).
template <int MODE>
int max_clusters(int num_sms) {
  static std::atomic<int> cache[64] = {};  // callers may race: each writes the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / 2;
  const int cached = cache[dev].load(std::memory_order_relaxed);
  if (cached > 0) return cached;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (unsigned)(num_sms / 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc2_gemm_kernel<MODE>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms / 2;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int MODE>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& as, const CUtensorMap& b, const CUtensorMap& bs,
                   const CUtensorMap& g, const Tc2Params& p, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc2_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (p.c.splits != 1) return cudaErrorInvalidValue;
  const int units = p.c.max_tiles;
  const int mc = max_clusters<MODE>(num_sms);
  const int clusters = units < mc ? units : mc;
  return launch_pdl(tc2_gemm_kernel<MODE>, (unsigned)(2 * clusters), kThreads, SMEM_BYTES, st, a, as, b, bs, g, p);
}

}  // namespace

cudaError_t launch_tc2_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mAs, mB, mBs, mG;
  // the shared expert alone (beside MXFP4 experts) needs no maps of the routed stacks
  const bool shared_only = c.seg_begin >= c.E;
  bool ok = true;
  if (!shared_only) {
    ok = map_rows(&mA, a.xg, c.d, c.R, c.d);
    ok = ok && map_fc1(&mB, a.gate_up, c.d, c.F, c.E, c.ffn, c.gu_layout);
    if (c.gu_layout == MOE_GU_UNFUSED) ok = ok && map_fc1(&mG, a.gate, c.d, c.F, c.E, c.ffn, c.gu_layout);
    else mG = mB;
  }
  if (c.Fs > 0) {
    // the shared expert keeps one stack (gate rows first when the routed experts are unfused)
    const int sh_layout = c.gu_layout == MOE_GU_UNFUSED ? MOE_GU_CONCAT : c.gu_layout;
    ok = ok && map_rows(&mAs, a.x, c.d, c.T, c.d);
    ok = ok && map_fc1(&mBs, a.sh_gate_up, c.d, c.Fs, 1, c.ffn, sh_layout);
  } else {
    mAs = mA;
    mBs = mB;
  }
  if (shared_only) {
    mA = mAs;
    mB = mG = mBs;
  }
  if (!ok) return cudaErrorInvalidValue;
  Tc2Params p{c, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias, nullptr, a.roww, (uint16_t*)a.h};
  return launch<0>(mA, mAs, mB, mBs, mG, p, a.num_sms, st);
}

cudaError_t launch_tc2_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mAs, mB, mBs;
  const bool shared_only = c.seg_begin >= c.E;  // beside MXFP4 experts
  bool ok = true;
  if (!shared_only) {
    ok = map_rows(&mA, a.h, c.F, c.R, c.Fmax);
    ok = ok && map_down(&mB, a.down, c.F, c.d, c.E);
  }
  if (c.Fs > 0) {
    ok = ok && map_rows(&mAs, (const uint16_t*)a.h + (int64_t)c.R * c.Fmax, c.Fs, c.T, c.Fmax);
    ok = ok && map_down(&mBs, a.sh_down, c.Fs, c.d, 1);
  } else {
    mAs = mA;
    mBs = mB;
  }
  if (shared_only) {
    mA = mAs;
    mB = mBs;
  }
  if (!ok) return cudaErrorInvalidValue;
  Tc2Params p{c, nullptr, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(mA, mAs, mB, mBs, mB, p, a.num_sms, st);
}

}  // namespace moe
