// gemm_tcs.cu -- the bf16 grouped GEMMs with the operands swapped, on CTA pairs
// (tcgen05 cta_group::2): the weight rows are the MMA's M = 256 (128 per CTA), the
// token rows its N (the tile's rows rounded up to 16, at most 256, split evenly
// across the pair).  Same operations as gemm_tc.cu ("MoE" graph-op page: fc1 fused
// gate||up or plain, fc2 down; "Struct MoeSpec" biases, activation, weigh_inputs):
//   gate_up (MODE 0): h = gated(W_gate[e] x + b_gate, W_up[e] x + b_up) or act(W_1 x + b_1)
//   down    (MODE 1): Y = (W_down[e] h + b_down) * w
//
// Why swapped: with many experts each holds few rows (a DeepSeek-V3-shaped batch
// has a median of ~100 rows per expert), so 128- or 256-row token tiles are mostly
// padding; here a tile pads its token rows to a multiple of 16 only.  Why a pair:
// per SM and K step the pair stages 16 KiB of weights and at most 16 KiB of token
// rows, and the MMA reads each CTA's operands once for both SMs -- the shared-
// memory traffic that bounds a single-CTA tile.
//
// Gate and up rows of one feature sit in neighbouring TMEM lanes: the weight box of
// a gated gate_up tile is 64 features x (gate, up) through a 4-D view of the stack
// whose feature dimension is outer to the gate/up one, for both fused layouts
// (concat: [E][2][F][d] read as {d, 2, F, E}; interleaved: [E][F][2][d]).
//
// Warp roles in each CTA: warp 0 TMA producer (this CTA's 128 weight rows and its
// token rows, completing on the even CTA's barrier, which the even CTA arms for the
// bytes of both; no multicast); warp 1 TMEM allocation for the pair and, in the even
// CTA, the MMA issuer; warps 2-9 epilogue of this CTA's 128 accumulator lanes.
// Every wait is bounded (2 s) and reports MOE_ERR_TIMEOUT through the status word.
#include <atomic>

#include "epilogue.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = kSwapBM;             // 256 token rows per tile (the MMA's N, trimmed)
constexpr int BMC = BM / 2;             // token rows staged per CTA (at most)
constexpr int BK = 64;                  // K elements per stage
constexpr int BNW = 256;                // weight rows per pair tile (the MMA's M)
constexpr int BNC = BNW / 2;            // 128 weight rows per CTA
constexpr int STAGES = 6;
constexpr int W_BYTES = BNC * BK * 2;   // 16 KiB
constexpr int A_BYTES = BMC * BK * 2;   // 16 KiB
constexpr int STAGE_BYTES = W_BYTES + A_BYTES;
constexpr int ACC_COLS = BM;            // one column per token row
constexpr int TMEM_COLS = 2 * ACC_COLS; // double-buffered
constexpr int kEpiWarps = 8;            // two per TMEM lane quadrant, alternate token chunks
constexpr int kEpiGroups = kEpiWarps / 4;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint16_t kBothCtas = 0x3;
constexpr uint16_t kEvenCta = 0x1;

struct TcsParams {
  GemmCommon c;
  const uint16_t* gate_up_bias;  // [E, 2F] ([E, F] plain) or null
  const uint16_t* down_bias;     // [E, d] or null
  const float* roww;             // [R]
  uint16_t* out;                 // h [rows, Fmax] or Y [rows, d]
};

template <int MODE>
__device__ __forceinline__ int k_extent(const GemmCommon& c, bool shared) {
  return MODE == 0 ? c.d : (shared ? c.Fs : c.F);
}

__device__ __forceinline__ int tile_live(const Tile& t) { return t.rows - t.m0 < BM ? t.rows - t.m0 : BM; }
__device__ __forceinline__ int tile_n(const Tile& t) { return (tile_live(t) + 15) & ~15; }

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tcs_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWs,
                    const TcsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [128 weight rows x 64][128 token rows x 64], both bf16 128B-swizzled K-major
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);  // even CTA only
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;  // even CTA only
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const GemmCommon& c = p.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
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
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmWs);
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
  const int total = tile_total(c);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        const Tile t = decode_tile<BM>(c, tile);
        const bool sh = t.seg >= c.E;
        const int nkb = (k_extent<MODE>(c, sh) + BK - 1) / BK;
        // CTA r stages token rows m0 + r N/2 .. (128 rows; those past N/2 are not read)
        const int arow = (sh ? 0 : c.off[t.seg]) + t.m0 + rank * (tile_n(t) / 2);
        const CUtensorMap* mA = sh ? &tmAs : &tmA;
        const CUtensorMap* mW = sh ? &tmWs : &tmW;
        const int e = sh ? 0 : t.seg;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          // only the even CTA arms the stage, for both CTAs' bytes; the odd CTA's bytes
          // may land first (the transaction count goes negative, the phase cannot
          // complete before the even CTA's arrival)
          const uint32_t fb = mapa_shared(&full[s], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
          uint8_t* sw = smem + s * STAGE_BYTES;
          const int k0 = kb * BK;
          if (MODE == 0 && c.ffn == MOE_FFN_GATED) {
            // 64 features x (gate, up) through the feature-outer 4-D view
            tma_load_4d_pair(mW, fb, sw, k0, 0, t.n_blk * (BNW / 2) + (BNC / 2) * rank, e);
          } else {
            tma_load_3d_pair(mW, fb, sw, k0, t.n_blk * BNW + BNC * rank, e);
          }
          tma_load_2d_pair(mA, fb, sw + W_BYTES, k0, arow);
        }
      }
      // every stage this CTA loaded has been consumed by the MMAs (so its bytes have
      // landed) before the CTA may exit; the empty barriers see the same commits in
      // both CTAs
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
      for (int tile = cluster; ok && tile < total; tile += nclusters, tcount++) {
        const Tile t = decode_tile<BM>(c, tile);
        const int nkb = (k_extent<MODE>(c, t.seg >= c.E) + BK - 1) / BK;
        const uint32_t idesc = idesc_bf16_f32(BNW, tile_n(t));
        const int acc = tcount & 1;
        // both CTAs' epilogue warps arrive here with cluster-scope release
        if (!mbar_wait_cluster(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, c.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + acc * ACC_COLS;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t wd = sdesc_k_sw128(sa), xd = sdesc_k_sw128(sa + W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++)
            mma_bf16_pair(dt, wd + 2 * kk, xd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
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
    // Lane r of this CTA's accumulator is its weight row r (32q + lane), column j
    // token m0 + j of the tile.
    const int q = warp & 3;                 // TMEM lane quadrant this warp may read
    const int part = (warp - 2) / 4;        // which alternate 16-token chunks it drains
    const int r = q * 32 + lane;
    const uint32_t tempty_even0 = mapa_shared(&tempty[0], 0), tempty_even1 = mapa_shared(&tempty[1], 0);
    uint32_t tcount = 0;
    for (int tile = cluster; tile < total; tile += nclusters, tcount++) {
      const Tile t = decode_tile<BM>(c, tile);
      const bool sh = t.seg >= c.E;
      const int acc = tcount & 1;
      // warp-uniform: the TMEM loads below need every lane of the warp
      const bool got = mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      const int live = tile_live(t);
      const int64_t grow0 = (int64_t)c.off[t.seg] + t.m0;
      if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
        const int F = sh ? c.Fs : c.F;
        const int f = t.n_blk * BNW + BNC * rank + r;
        const float b = (!sh && p.gate_up_bias && f < F) ? bf16_to_f32(p.gate_up_bias[(int64_t)t.seg * c.F + f]) : 0.f;
#pragma unroll 1
        for (int ch = part; ch < BM / 16 && ch * 16 < live; ch += kEpiGroups) {
          uint32_t v[16];
          tmem_ld16(tb + ch * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i++) {
            const int tok = ch * 16 + i;
            if (tok < live && f < F)
              p.out[(grow0 + tok) * c.Fmax + f] = f32_to_bf16_rn(plain_act_bf16(c.act, __uint_as_float(v[i]) + b));
          }
        }
      } else if (MODE == 0) {
        // lanes 2j / 2j+1 hold the gate / up row of feature f; the even lane
        // finishes the chunk's first 8 tokens, the odd lane the last 8
        const int F = sh ? c.Fs : c.F;
        const int f = t.n_blk * (BNW / 2) + (BNC / 2) * rank + (r >> 1);
        const bool odd = lane & 1;
        float bg = 0.f, bu = 0.f;
        if (!sh && f < F) {
          const GuBias gb = gu_bias(c.gu_layout, c.F, t.seg, p.gate_up_bias, nullptr);
          if (gb.g) bg = bf16_to_f32(gb.g[(int64_t)gb.stride * f]);
          if (gb.u) bu = bf16_to_f32(gb.u[(int64_t)gb.stride * f]);
        }
#pragma unroll 1
        for (int ch = part; ch < BM / 16 && ch * 16 < live; ch += kEpiGroups) {
          uint32_t v[16];
          tmem_ld16(tb + ch * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; i++) {
            const uint32_t give = odd ? v[i] : v[8 + i];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, give, 1);
            const float g = __uint_as_float(odd ? recv : v[i]);
            const float u = __uint_as_float(odd ? v[8 + i] : recv);
            const int tok = ch * 16 + (odd ? 8 : 0) + i;
            if (tok < live && f < F)
              p.out[(grow0 + tok) * c.Fmax + f] = f32_to_bf16_rn(gated_act_bf16(c.act, g + bg, u + bu));
          }
        }
      } else {
        const int o = t.n_blk * BNW + BNC * rank + r;
        const float b = (!sh && p.down_bias && o < c.d) ? bf16_to_f32(p.down_bias[(int64_t)t.seg * c.d + o]) : 0.f;
#pragma unroll 1
        for (int ch = part; ch < BM / 16 && ch * 16 < live; ch += kEpiGroups) {
          uint32_t v[16];
          tmem_ld16(tb + ch * 16, v);
          tmem_ld_wait();
          // routing weights of the chunk's 16 tokens: lane i (and i + 16) loads token i's
          const int my_tok = ch * 16 + (lane & 15);
          const float my_w = (sh || c.weigh_inputs || my_tok >= live) ? 1.f : p.roww[grow0 + my_tok];
#pragma unroll
          for (int i = 0; i < 16; i++) {
            const float w = __shfl_sync(0xffffffffu, my_w, i);
            const int tok = ch * 16 + i;
            if (tok < live && o < c.d)
              p.out[(grow0 + tok) * c.d + o] = f32_to_bf16_rn((__uint_as_float(v[i]) + b) * w);
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

// rows x K matrix with row pitch `pitch` elements; box 64 x 128 rows.
bool map_rows(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t pitch) {
  const uint64_t dims[2] = {K, rows > 0 ? rows : 1};
  const uint64_t strides[1] = {pitch * 2};
  const uint32_t box[2] = {BK, BMC};
  return make_map(m, base, 2, dims, strides, box);
}

// A gated gate||up stack [E][2F][d] seen as {d, 2 (gate, up), F, E} with the
// feature dimension outer to the gate/up one: one box = 64 features x (gate, up)
// = 128 rows, gate and up of a feature adjacent, for both fused layouts.
bool map_gate_up_pairs(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int layout) {
  const uint64_t dims[4] = {d, 2, F, E};
  const bool il = layout == MOE_GU_INTERLEAVED;
  const uint64_t strides[3] = {il ? d * 2 : F * d * 2, il ? 2 * d * 2 : d * 2, 2 * F * d * 2};
  const uint32_t box[4] = {BK, 2, BNC / 2, 1};
  return make_map(m, base, 4, dims, strides, box);
}

// An [E][rows][K] stack (plain fc1 [E][F][d], down [E][d][F]) with boxes of 128 rows.
bool map_stack(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t E) {
  const uint64_t dims[3] = {K, rows, E};
  const uint64_t strides[2] = {K * 2, rows * K * 2};
  const uint32_t box[3] = {BK, BNC, 1};
  return make_map(m, base, 3, dims, strides, box);
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
  if (cudaOccupancyMaxActiveClusters(&n, tcs_gemm_kernel<MODE>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int MODE>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& as, const CUtensorMap& w, const CUtensorMap& ws,
                   const TcsParams& p, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tcs_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (p.c.splits != 1) return cudaErrorInvalidValue;
  const int mc = max_clusters<MODE>(num_sms);
  const int clusters = p.c.max_tiles < mc ? p.c.max_tiles : mc;
  return launch_pdl(tcs_gemm_kernel<MODE>, (unsigned)(2 * clusters), kThreads, SMEM_BYTES, st, a, as, w, ws, p);
}

bool map_fc1(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int ffn, int layout) {
  if (ffn == MOE_FFN_PLAIN) return map_stack(m, base, d, F, E);
  return map_gate_up_pairs(m, base, d, F, E, layout);
}

}  // namespace

cudaError_t launch_tcs_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  if (c.gu_layout == MOE_GU_UNFUSED) return cudaErrorInvalidValue;  // the plan never picks it then
  CUtensorMap mA, mAs, mW, mWs;
  bool ok = map_rows(&mA, a.xg, c.d, c.R, c.d);
  ok = ok && map_fc1(&mW, a.gate_up, c.d, c.F, c.E, c.ffn, c.gu_layout);
  if (c.Fs > 0) {
    ok = ok && map_rows(&mAs, a.x, c.d, c.T, c.d);
    ok = ok && map_fc1(&mWs, a.sh_gate_up, c.d, c.Fs, 1, c.ffn, c.gu_layout);
  } else {
    mAs = mA;
    mWs = mW;
  }
  if (!ok) return cudaErrorInvalidValue;
  TcsParams p{c, (const uint16_t*)a.gate_up_bias, nullptr, a.roww, (uint16_t*)a.h};
  return launch<0>(mA, mAs, mW, mWs, p, a.num_sms, st);
}

cudaError_t launch_tcs_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mAs, mW, mWs;
  bool ok = map_rows(&mA, a.h, c.F, c.R, c.Fmax);
  ok = ok && map_stack(&mW, a.down, c.F, c.d, c.E);
  if (c.Fs > 0) {
    ok = ok && map_rows(&mAs, (const uint16_t*)a.h + (int64_t)c.R * c.Fmax, c.Fs, c.T, c.Fmax);
    ok = ok && map_stack(&mWs, a.sh_down, c.Fs, c.d, 1);
  } else {
    mAs = mA;
    mWs = mW;
  }
  if (!ok) return cudaErrorInvalidValue;
  TcsParams p{c, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(mA, mAs, mW, mWs, p, a.num_sms, st);
}

}  // namespace moe
