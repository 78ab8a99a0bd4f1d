// gemm_fp4p.cu -- the MXFP4 grouped GEMMs of gemm_fp4.cu on CTA pairs (tcgen05
// cta_group::2), for batches whose experts hold on average at least 128 rows
// ("ClikaRT::nn::QMoEWoQ": weight-only quantized experts, each weight block
// decoded inside the GEMM dot, never as a dense copy).
//
//   gate_up (MODE 0): h = gated(W_gate[e] x + b_gate, W_up[e] x + b_up) (or, plain,
//                     h = act(W_1[e] x + b_1)) -> bf16
//   down    (MODE 1): Y = (W_down[e] h + b_down) * w -> bf16
//
// A cluster of two CTAs owns a tile of 256 weight rows x up to 256 token rows,
// computed transposed like the single-CTA kernel: the decoded weights are the
// MMA's A operand (M = 256, CTA r decodes weight rows 128 r .. 128 r + 127 into
// its own shared memory) and the token rows its B operand (N = the tile's rows
// rounded up to 16; the instruction takes columns 0 .. N/2 - 1 from the even CTA
// and N/2 .. N - 1 from the odd one, so CTA r stages token rows m0 + r N/2 ..).
// Per SM and K step this halves the activation bytes staged and read against
// the single-CTA kernel (the B tile is shared by the pair) -- the shared-memory
// traffic that bounds that kernel.
//
// Warp roles in each CTA (the even CTA also issues the MMAs):
//   warp 0      TMA producer of this CTA's activation rows (128 x 64 bf16), loads
//               completing on the even CTA's barrier, which the even CTA arms for
//               the bytes of both (no multicast);
//   warp 1      TMEM allocation for the pair; in the even CTA the MMA issuer
//               (M=256 N<=256 K=16 over both CTAs), whose commits arrive on both
//               CTAs' barriers;
//   warps 2-9   epilogue of this CTA's 128 accumulator lanes (its weight rows);
//   warps 10-25 converters (four groups of four warps): codes + scales -> bf16 in
//               the 128B-swizzled K-major layout, a proxy fence for this CTA's
//               shared memory, a local barrier of
//               the group's warps, then one arrival per group and stage on the even
//               CTA's decoded-slot barrier (remote, with release at cluster scope,
//               from the odd CTA);
//   warp 26     TMA producer of this CTA's codes (128 weight rows x 32 bytes).
// Every wait is bounded (2 s) and reports MOE_ERR_TIMEOUT through the status word.
#include <atomic>

#include "epilogue.cuh"
#include "mxfp4.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace mxfp4;

constexpr int BM = kFp4BM;              // 256 token rows per tile (the MMA's N, trimmed)
constexpr int BMC = BM / 2;             // token rows staged per CTA (at most)
constexpr int BK = 64;                  // K elements per stage
constexpr int BNW = kFp4PairBN;         // 256 weight rows per pair tile (the MMA's M)
constexpr int BNC = BNW / 2;            // 128 weight rows decoded per CTA
constexpr int AST = 4;                  // activation stages, freed by the MMA
constexpr int QST = 6;                  // code stages, freed once converted
constexpr int WST = 8;                  // decoded weight stages, freed by the MMA (two per group)
constexpr int A_BYTES = BMC * BK * 2;   // 16 KiB
constexpr int Q_BYTES = BNC * BK / 2;   // 4 KiB
constexpr int W_BYTES = BNC * BK * 2;   // 16 KiB
constexpr int RING_BYTES = AST * A_BYTES + WST * W_BYTES + QST * Q_BYTES;
constexpr int ACC_COLS = BM;            // one column per token row
constexpr int TMEM_COLS = 2 * ACC_COLS; // double-buffered
constexpr int kEpiWarps = 8;            // two per TMEM lane quadrant, alternate token chunks
constexpr int kEpiGroups = kEpiWarps / 4;
constexpr int kCvtWarps = 16;
constexpr int kCvtGroups = 4;
constexpr int kCvtGroupWarps = kCvtWarps / kCvtGroups;
constexpr int kThreads = 64 + (kEpiWarps + kCvtWarps + 1) * 32;
constexpr int SMEM_BYTES = RING_BYTES + 1024 + 512;
constexpr uint16_t kBothCtas = 0x3;
constexpr uint16_t kEvenCta = 0x1;
static_assert(kCvtGroupWarps * 32 == BNC, "one converter thread per weight row in a group");
static_assert(WST % kCvtGroups == 0, "a group's stages map to its own decoded-weight slots");

struct Fp4pParams {
  GemmCommon c;
  const uint8_t* scales;        // e8m0 [E, rows, K/32] (unfused gate_up: the up rows' scales)
  const uint8_t* gate_scales;   // unfused gate_up: the gate rows' scales [E, F, d/32]
  const uint16_t* gate_up_bias; // [E, 2F] ([E, F] unfused / plain) or null
  const uint16_t* gate_bias;    // unfused: [E, F] or null
  const uint16_t* down_bias;    // [E, d] or null
  const float* roww;            // [R]
  uint16_t* out;                // h [rows, Fmax] or Y [rows, d]
};

template <int MODE>
__device__ __forceinline__ int k_extent(const GemmCommon& c) {
  return MODE == 0 ? c.d : c.F;
}

// Row of the scale / code stack (inside expert e) that weight row r of CTA `rank`'s
// half reads.  Gated gate_up: rows 2j, 2j+1 of the half = gate and up rows of feature
// n_blk * 128 + 64 rank + j (for the unfused layout each in its own stack, *gate set
// for the gate row); plain gate_up: feature n_blk * 256 + 128 rank + r; down: output
// n_blk * 256 + 128 rank + r.
template <int MODE>
__device__ __forceinline__ int weight_row(const GemmCommon& c, int n_blk, int rank, int r, bool* valid,
                                          bool* gate) {
  *gate = false;
  if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
    const int f = n_blk * BNW + BNC * rank + r;
    *valid = f < c.F;
    return f;
  }
  if (MODE == 0) {
    const int half = r & 1;
    const int f = n_blk * (BNW / 2) + (BNC / 2) * rank + (r >> 1);
    *valid = f < c.F;
    if (c.gu_layout == MOE_GU_UNFUSED) {
      *gate = half == 0;
      return f;
    }
    if (c.gu_layout == MOE_GU_INTERLEAVED) return 2 * f + half;
    return half ? c.F + f : f;
  }
  const int o = n_blk * BNW + BNC * rank + r;
  *valid = o < c.d;
  return o;
}

// Token rows of a tile and the MMA's N (rows rounded up to 16, at most 256).
__device__ __forceinline__ int tile_live(const Tile& t) { return t.rows - t.m0 < BM ? t.rows - t.m0 : BM; }
__device__ __forceinline__ int tile_n(const Tile& t) { return (tile_live(t) + 15) & ~15; }

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fp4p_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmG, const Fp4pParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ringA = smem;                                   // AST x 16 KiB (1024-aligned)
  uint8_t* ringW = ringA + AST * A_BYTES;                  // WST x 16 KiB (1024-aligned)
  uint8_t* ringQ = ringW + WST * W_BYTES;                  // QST x 4 KiB
  uint64_t* fullA = reinterpret_cast<uint64_t*>(smem + RING_BYTES);  // even CTA only
  uint64_t* emptyA = fullA + AST;
  uint64_t* fullW = emptyA + AST;                          // even CTA only
  uint64_t* emptyW = fullW + WST;
  uint64_t* fullQ = emptyW + WST;
  uint64_t* emptyQ = fullQ + QST;
  uint64_t* tfull = emptyQ + QST;
  uint64_t* tempty = tfull + 2;                            // even CTA only
  uint64_t* drain = tempty + 2;
  uint64_t* wdone = drain + 1;                             // [WST] the converter group's warps done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wdone + WST);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const GemmCommon& c = p.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  constexpr int kCodesWarp = 2 + kEpiWarps + kCvtWarps;

  if (threadIdx.x == 0) {
    for (int s = 0; s < AST; s++) {
      mbar_init(&fullA[s], 1);  // the even CTA's expect_tx covers both CTAs' loads
      mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < WST; s++) {
      mbar_init(&fullW[s], 2);  // one arrival per converter group of both CTAs
      mbar_init(&emptyW[s], 1);
    }
    for (int s = 0; s < QST; s++) {
      mbar_init(&fullQ[s], 1);
      mbar_init(&emptyQ[s], kCvtGroupWarps);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int s = 0; s < WST; s++) mbar_init(&wdone[s], kCvtGroupWarps);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmQ);
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
  const int K = k_extent<MODE>(c);
  const int nkb = (K + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ activation producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        const Tile t = decode_tile<BM>(c, tile);
        // CTA r stages token rows m0 + r N/2 .. (128 rows; those past N/2 are not read)
        const int row0 = c.off[t.seg] + t.m0 + rank * (tile_n(t) / 2);
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % AST;
          if (!mbar_wait(&emptyA[s], ((it / AST) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          // only the even CTA arms the stage, for both CTAs' bytes; the odd CTA's bytes
          // may land first (the transaction count goes negative, the phase cannot
          // complete before the even CTA's arrival)
          const uint32_t fb = mapa_shared(&fullA[s], 0);
          if (rank == 0) mbar_arrive_expect_tx(&fullA[s], 2 * A_BYTES);
          tma_load_2d_pair(&tmA, fb, ringA + s * A_BYTES, kb * BK, row0);
        }
      }
      // every stage this CTA loaded has been consumed by the MMAs (so its bytes have
      // landed) before the CTA may exit; the empty barriers see the same commits in
      // both CTAs
      const uint64_t t0 = global_timer();
      for (uint32_t j = (it > (uint32_t)AST ? it - AST : 0); j < it; j++) {
        while (!mbar_try_wait(&emptyA[j % AST], (j / AST) & 1) && global_timer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else if (warp == kCodesWarp) {
    // ------------------------------------------------------------ code producer (both CTAs, local)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        const Tile t = decode_tile<BM>(c, tile);
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % QST;
          if (!mbar_wait(&emptyQ[s], ((it / QST) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          uint8_t* sq = ringQ + s * Q_BYTES;
          mbar_arrive_expect_tx(&fullQ[s], Q_BYTES);
          const int kq = kb * (BK / 2);
          if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
            tma_load_3d(&tmQ, &fullQ[s], sq, kq, t.n_blk * BNW + BNC * rank, t.seg);
          } else if (MODE == 0 && c.gu_layout == MOE_GU_UNFUSED) {
            const int f0 = t.n_blk * (BNW / 2) + (BNC / 2) * rank;  // 64 gate rows, then the 64 up rows
            tma_load_3d(&tmG, &fullQ[s], sq, kq, f0, t.seg);
            tma_load_3d(&tmQ, &fullQ[s], sq + Q_BYTES / 2, kq, f0, t.seg);
          } else if (MODE == 0) {
            const int f0 = t.n_blk * (BNW / 2) + (BNC / 2) * rank;
            const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
            for (int half = 0; half < 2; half++)
              tma_load_4d(&tmQ, &fullQ[s], sq + half * (Q_BYTES / 2), kq, il ? half : f0, il ? f0 : half, t.seg);
          } else {
            tma_load_3d(&tmQ, &fullQ[s], sq, kq, t.n_blk * BNW + BNC * rank, t.seg);
          }
        }
      }
      for (uint32_t j = (it > (uint32_t)QST ? it - QST : 0); j < it; j++) {
        const uint64_t t0 = global_timer();
        while (!mbar_try_wait(&fullQ[j % QST], (j / QST) & 1) && global_timer() - t0 < kTimeoutNs) {
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
        const uint32_t idesc = idesc_bf16_f32(BNW, tile_n(t));
        const int acc = tcount & 1;
        // both CTAs' epilogue warps arrive here with cluster-scope release
        if (!mbar_wait_cluster(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, c.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + acc * ACC_COLS;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int sa = it % AST, sw = it % WST;
          if (!mbar_wait(&fullA[sa], (it / AST) & 1, abort_flag, c.status) ||
              !mbar_wait_cluster(&fullW[sw], (it / WST) & 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t wd = sdesc_k_sw128(smem_u32(ringW + sw * W_BYTES));  // A: decoded weights
          const uint64_t xd = sdesc_k_sw128(smem_u32(ringA + sa * A_BYTES));  // B: token rows
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++)
            mma_bf16_pair(dt, wd + 2 * kk, xd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit_pair(&emptyA[sa], kBothCtas);
          mma_commit_pair(&emptyW[sw], kBothCtas);
        }
        if (ok) mma_commit_pair(&tfull[acc], kBothCtas);
      }
      // all issued MMAs complete before either CTA releases its tensor memory
      mma_commit_pair(drain, kEvenCta);
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(drain, 0) && global_timer() - t0 < kTimeoutNs) {
      }
    }
  } else if (warp < 2 + kEpiWarps) {
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
      const int acc = tcount & 1;
      // warp-uniform: the TMEM loads below need every lane of the warp
      const bool got = mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      const int live = tile_live(t);
      const int64_t grow0 = (int64_t)c.off[t.seg] + t.m0;
      if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
        const int f = t.n_blk * BNW + BNC * rank + r;
        const float b = (p.gate_up_bias && f < c.F) ? bf16_to_f32(p.gate_up_bias[(int64_t)t.seg * c.F + f]) : 0.f;
#pragma unroll 1
        for (int ch = part; ch < BM / 16 && ch * 16 < live; ch += kEpiGroups) {
          uint32_t v[16];
          tmem_ld16(tb + ch * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i++) {
            const int tok = ch * 16 + i;
            if (tok < live && f < c.F)
              p.out[(grow0 + tok) * c.Fmax + f] = f32_to_bf16_rn(plain_act_bf16(c.act, __uint_as_float(v[i]) + b));
          }
        }
      } else if (MODE == 0) {
        // lanes 2j / 2j+1 hold the gate / up row of feature f; the even lane
        // finishes the chunk's first 8 tokens, the odd lane the last 8
        const int f = t.n_blk * (BNW / 2) + (BNC / 2) * rank + (r >> 1);
        const bool odd = lane & 1;
        float bg = 0.f, bu = 0.f;
        if (f < c.F) {
          const GuBias gb = gu_bias(c.gu_layout, c.F, t.seg, p.gate_up_bias, p.gate_bias);
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
            if (tok < live && f < c.F)
              p.out[(grow0 + tok) * c.Fmax + f] = f32_to_bf16_rn(gated_act_bf16(c.act, g + bg, u + bu));
          }
        }
      } else {
        const int o = t.n_blk * BNW + BNC * rank + r;
        const float b = (p.down_bias && o < c.d) ? bf16_to_f32(p.down_bias[(int64_t)t.seg * c.d + o]) : 0.f;
#pragma unroll 1
        for (int ch = part; ch < BM / 16 && ch * 16 < live; ch += kEpiGroups) {
          uint32_t v[16];
          tmem_ld16(tb + ch * 16, v);
          tmem_ld_wait();
          // routing weights of the chunk's 16 tokens: lane i (and i + 16) loads token i's
          const int my_tok = ch * 16 + (lane & 15);
          const float my_w = (c.weigh_inputs || my_tok >= live) ? 1.f : p.roww[grow0 + my_tok];
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
  } else if (warp < kCodesWarp) {
    // ------------------------------------------------------------ converters (both CTAs)
    // Four groups of four warps; group g converts the stages it with it % 4 == g.  In
    // a group, thread = weight row of this CTA's half: it loads the row's 32 code
    // bytes, decodes 64 elements with the row's two block scales and writes the
    // 128-byte row in the swizzled layout; then one arrival per warp on the even
    // CTA's barrier of the slot, after a proxy fence that makes the generic-proxy
    // writes visible to the tensor cores of both SMs.
    const int cw = warp - 2 - kEpiWarps;
    const int group = cw / kCvtGroupWarps;
    const int r = (cw % kCvtGroupWarps) * 32 + lane;
    const int kblocks = K / 32;
    const int rows_per_e = MODE == 1 ? c.d : (c.ffn == MOE_FFN_PLAIN || c.gu_layout == MOE_GU_UNFUSED) ? c.F : 2 * c.F;
    const uint32_t fullW_even = mapa_shared(&fullW[0], 0);
    uint32_t it = 0;
    for (int tile = cluster; tile < total; tile += nclusters, it += nkb) {
      const Tile t = decode_tile<BM>(c, tile);
      bool rvalid, gate_row;
      const int wr = weight_row<MODE>(c, t.n_blk, rank, r, &rvalid, &gate_row);
      const uint8_t* srow = (gate_row ? p.gate_scales : p.scales) + ((int64_t)t.seg * rows_per_e + wr) * kblocks;
      auto load_scales = [&](int kb) -> uint32_t {  // the row's two block scales of k-block kb
        if (!rvalid || kb >= nkb) return 127u | (127u << 8);
        const int col = kb * 2;
        const uint32_t lo = col < kblocks ? __ldg(srow + col) : 127u;
        const uint32_t hi = col + 1 < kblocks ? __ldg(srow + col + 1) : 127u;
        return lo | (hi << 8);
      };
      int kb = (int)((group - (int)(it % kCvtGroups) + kCvtGroups) % kCvtGroups);
      uint32_t sc = load_scales(kb);
      bool ok = true;
      for (; kb < nkb; kb += kCvtGroups) {
        const uint32_t next = load_scales(kb + kCvtGroups);
        const uint32_t st = it + kb;
        const int sq = st % QST, sw = st % WST;
        if (!mbar_wait(&fullQ[sq], (st / QST) & 1, abort_flag, c.status)) {
          ok = false;
          break;
        }
        // code rows in the slot: gated gate_up 64 gate rows then their 64 up rows; else in order
        const int qr = (MODE == 0 && c.ffn == MOE_FFN_GATED) ? (r & 1) * (BNC / 2) + (r >> 1) : r;
        const uint4* qrow = reinterpret_cast<const uint4*>(ringQ + sq * Q_BYTES + qr * (BK / 2));
        const uint4 q0 = qrow[0], q1 = qrow[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyQ[sq]);  // codes are in registers: the slot may refill
        // the slot is free once the pair MMAs that read it committed to this CTA
        if (!mbar_wait(&emptyW[sw], ((st / WST) & 1) ^ 1, abort_flag, c.status)) {
          ok = false;
          break;
        }
        decode_row_sw128(q0, q1, sc, ringW + sw * W_BYTES + r * (BK * 2), r);
        // this CTA's shared memory, which the pair MMAs read through the async proxy
        // (the all-state-space fence cost ~1200 cycles per stage here)
        fence_proxy_async_smem();
        __syncwarp();
        // the group's four warps meet on a local barrier, then its first warp signals
        // the slot to the MMA issuer (one remote arrival per stage from the odd CTA)
        if (lane == 0) mbar_arrive(&wdone[sw]);
        if (cw % kCvtGroupWarps == 0 && lane == 0) {
          if (!mbar_wait(&wdone[sw], (st / WST) & 1, abort_flag, c.status)) {
            ok = false;
          } else if (rank == 0) {
            mbar_arrive(&fullW[sw]);
          } else {
            mbar_arrive_cluster(fullW_even + sw * (uint32_t)sizeof(uint64_t));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        sc = next;
      }
      if (!ok) break;
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

// Token rows x K (bf16, 128B swizzle), box 64 x 128 rows (one CTA's half of a tile).
bool map_act(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t pitch) {
  const uint64_t dims[2] = {K, rows > 0 ? rows : 1};
  const uint64_t strides[1] = {pitch * 2};
  const uint32_t box[2] = {BK, BMC};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// e2m1 code stack [E][2F][d/2] as 4-D: one box = 64 gate (or up) rows x 32 bytes.
bool map_codes_gate_up(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int layout) {
  const uint64_t kb = d / 2;
  if (layout == MOE_GU_INTERLEAVED) {
    const uint64_t dims[4] = {kb, 2, F, E};
    const uint64_t strides[3] = {kb, 2 * kb, 2 * F * kb};
    const uint32_t box[4] = {BK / 2, 1, BNC / 2, 1};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  const uint64_t dims[4] = {kb, F, 2, E};
  const uint64_t strides[3] = {kb, F * kb, 2 * F * kb};
  const uint32_t box[4] = {BK / 2, BNC / 2, 1, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// An [E][rows][K/2] code stack (plain fc1, an unfused gate or up stack, or the down
// stack) with boxes of `box_rows` rows x 32 bytes.
bool map_codes_rows(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t E, uint32_t box_rows) {
  const uint64_t kb = K / 2;
  const uint64_t dims[3] = {kb, rows, E};
  const uint64_t strides[2] = {kb, rows * kb};
  const uint32_t box[3] = {BK / 2, box_rows, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
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
  if (cudaOccupancyMaxActiveClusters(&n, fp4p_gemm_kernel<MODE>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int MODE>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& q, const CUtensorMap& g, const Fp4pParams& p,
                   int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(fp4p_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int mc = max_clusters<MODE>(num_sms);
  const int clusters = p.c.max_tiles < mc ? p.c.max_tiles : mc;
  return launch_pdl(fp4p_gemm_kernel<MODE>, (unsigned)(2 * clusters), kThreads, SMEM_BYTES, st, a, q, g, p);
}

}  // namespace

cudaError_t launch_fp4p_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mQ, mG;
  bool ok = map_act(&mA, a.xg, c.d, c.R, c.d);
  if (c.ffn == MOE_FFN_PLAIN) {
    ok = ok && map_codes_rows(&mQ, a.gate_up, c.d, c.F, c.E, BNC);
    mG = mQ;
  } else if (c.gu_layout == MOE_GU_UNFUSED) {
    ok = ok && map_codes_rows(&mQ, a.gate_up, c.d, c.F, c.E, BNC / 2);
    ok = ok && map_codes_rows(&mG, a.gate, c.d, c.F, c.E, BNC / 2);
  } else {
    ok = ok && map_codes_gate_up(&mQ, a.gate_up, c.d, c.F, c.E, c.gu_layout);
    mG = mQ;
  }
  if (!ok) return cudaErrorInvalidValue;
  Fp4pParams p{c,       a.gate_up_scales, a.gate_scales, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias,
               nullptr, a.roww,           (uint16_t*)a.h};
  return launch<0>(mA, mQ, mG, p, a.num_sms, st);
}

cudaError_t launch_fp4p_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mQ;
  bool ok = map_act(&mA, a.h, c.F, c.R, c.Fmax);
  ok = ok && map_codes_rows(&mQ, a.down, c.F, c.d, c.E, BNC);
  if (!ok) return cudaErrorInvalidValue;
  Fp4pParams p{c, a.down_scales, nullptr, nullptr, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(mA, mQ, mQ, p, a.num_sms, st);
}

}  // namespace moe
