// gemm_fp4.cu -- grouped GEMMs over weight-only MXFP4 expert stacks, decoded to
// bf16 block by block inside the GEMM pipeline ("ClikaRT::nn::QMoEWoQ": the
// activations stay floating point, each expert weight decodes one block at a
// time inside the GEMM dot, never a dense copy).
//
//   gate_up (MODE 0): g, u = W_gate[e] x + b_gate, W_up[e] x + b_up; h = gated(g, u) -> bf16
//   down    (MODE 1): Y = (W_down[e] h + b_down) * w -> bf16
// with W[e][r][k] = e2m1(code[e][r][k]) * 2^(scale[e][r][k/32] - 127) (OCP MX v1.0:
// e2m1 two per byte, even k in the low nibble; e8m0 scale per 32 elements of K).
//
// Tile: 256 activation rows x 128 weight rows x K, computed transposed: the
// decoded weights are the MMA's A operand (M = 128 weight rows) and the
// activation rows its B operand (N = the tile's token rows rounded up to 16, at
// most 256), so one M=128 N<=256 instruction per K step reads 4 KiB of weights
// and at most 8 KiB of activations.  The tensor pipe's shared-memory operand
// reads, not the data movement, bound this kernel, and an M=128 N=256 step needs
// a quarter less of them per FLOP than two M=128 N=128 halves sharing the
// weights.  TMEM: 128 lanes (weight rows) x 256 columns (tokens), double-buffered.
// Warp roles:
//   warp 0      TMA producer of activations 256 x 64 (bf16, 128B swizzle)
//   warp 1      TMEM owner and MMA issuer (M=128 N<=256 K=16)
//   warp 13     TMA producer of the codes, 128 x 32 bytes, running up to 6 stages ahead
//   warps 2-9   epilogue: two warps per TMEM lane quadrant, alternate 16-token chunks;
//               for gate_up, weight rows 2j and 2j+1 are the gate and up rows of one
//               feature, so neighbouring lanes pair up with one shuffle
//   warps 10-30 except 13, 17, 21, 25, 29: converters in four groups of four, group
//               g owning stages it % 4 == g: codes + scale -> bf16 in the
//               128B-swizzled K-major layout the MMA descriptor reads (mxfp4.cuh),
//               then a proxy fence and one arrive per warp.  None shares the MMA
//               issuer's scheduler (warp w issues on scheduler w % 4); warps 17, 21,
//               25 and 29 idle.
#include "epilogue.cuh"
#include "mxfp4.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace mxfp4;

constexpr int BM = kFp4BM;              // 256 activation rows per tile (MMA N)
constexpr int BK = 64;                  // K elements per stage
constexpr int BNB = 128;                // weight rows per tile
// Three rings, so that decoding never holds an activation slot:
constexpr int AST = 4;                  // activations: 256 x 64 bf16, freed by the MMA
constexpr int QST = 6;                  // e2m1 codes: 128 x 32 bytes, freed once converted
constexpr int WST = 4;                  // decoded bf16 weights: 128 x 64, freed by the MMA
constexpr int A_BYTES = BM * BK * 2;    // 32 KiB
constexpr int Q_BYTES = BNB * BK / 2;   // 4 KiB
constexpr int W_BYTES = BNB * BK * 2;   // 16 KiB
constexpr int RING_BYTES = AST * A_BYTES + WST * W_BYTES + QST * Q_BYTES;
constexpr int ACC_COLS = BM;            // one column per activation row
constexpr int TMEM_COLS = 2 * ACC_COLS; // double-buffered
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant, alternate token chunks
constexpr int kEpiGroups = kEpiWarps / 4;
constexpr int kCvtWarps = 16;
constexpr int kCvtGroups = 4;                // converter groups, each owning every 4th stage
constexpr int kCvtGroupWarps = kCvtWarps / kCvtGroups;
// Warps 0 .. 30.  Warp w runs on the SM's scheduler w % 4; the MMA issuer (warp 1)
// shares its scheduler only with warps that issue few instructions (two epilogue
// warps and the code producer), never with a converter, so that its MMAs issue on
// time: converters are the warps 10 .. 30 other than 13, 17, 21, 25 and 29.  Four
// groups with a decoded slot each: a group's slot comes free three stages of MMAs
// after it was filled (with three groups the converters waited ~400 cycles per stage
// for it: 0.545 -> 0.527 ms per gpt-oss layer).
constexpr int kWarps = 31;
constexpr int kThreads = kWarps * 32;
constexpr int kCodesWarp = 13;
__host__ __device__ constexpr int converter_index(int w) {  // -1: not a converter
  return (w < 10 || w >= kWarps || w % 4 == 1) ? -1
                                               : w - 10 - (w > 13) - (w > 17) - (w > 21) - (w > 25) - (w > 29);
}
constexpr int SMEM_BYTES = RING_BYTES + 1024 + 512;
static_assert(kCvtGroupWarps * 32 == BNB, "one converter thread per weight row in a group");
static_assert(WST % kCvtGroups == 0, "a group's stages map to its own decoded-weight slots");
static_assert(converter_index(30) == kCvtWarps - 1, "sixteen converter warps");

struct Fp4Params {
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

// Row of the scale / code stack (inside expert e) that weight row r of the tile
// (the MMA's M index) reads.  Gated gate_up: rows 2j, 2j+1 = gate and up rows of
// feature n_blk * 64 + j (for the unfused layout each in its own stack, *gate
// set for the gate row); plain gate_up: feature n_blk * 128 + r of fc1.
template <int MODE>
__device__ __forceinline__ int weight_row(const GemmCommon& c, int n_blk, int r, bool* valid, bool* gate) {
  *gate = false;
  if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
    const int f = n_blk * BNB + r;
    *valid = f < c.F;
    return f;
  }
  if (MODE == 0) {
    const int half = r & 1;
    const int f = n_blk * (BNB / 2) + (r >> 1);
    *valid = f < c.F;
    if (c.gu_layout == MOE_GU_UNFUSED) {
      *gate = half == 0;
      return f;
    }
    if (c.gu_layout == MOE_GU_INTERLEAVED) return 2 * f + half;
    return half ? c.F + f : f;
  }
  const int o = n_blk * BNB + r;
  *valid = o < c.d;
  return o;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmG, const Fp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ringA = smem;                                   // AST x 32 KiB (1024-aligned)
  uint8_t* ringW = ringA + AST * A_BYTES;                  // WST x 16 KiB (1024-aligned)
  uint8_t* ringQ = ringW + WST * W_BYTES;                  // QST x 4 KiB
  uint64_t* fullA = reinterpret_cast<uint64_t*>(smem + RING_BYTES);
  uint64_t* emptyA = fullA + AST;
  uint64_t* fullW = emptyA + AST;
  uint64_t* emptyW = fullW + WST;
  uint64_t* fullQ = emptyW + WST;
  uint64_t* emptyQ = fullQ + QST;
  uint64_t* tfull = emptyQ + QST;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const GemmCommon& c = p.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < AST; s++) {
      mbar_init(&fullA[s], 1);
      mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < WST; s++) {
      mbar_init(&fullW[s], kCvtGroupWarps);
      mbar_init(&emptyW[s], 1);
    }
    for (int s = 0; s < QST; s++) {
      mbar_init(&fullQ[s], 1);
      mbar_init(&emptyQ[s], kCvtGroupWarps);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmQ);
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
  const int total = tile_total(c);
  const int K = k_extent<MODE>(c);
  const int nkb = (K + BK - 1) / BK;

  if (warp == 0 || warp == kCodesWarp) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool codes = warp == kCodesWarp;
      const int depth = codes ? QST : AST;
      uint64_t* full = codes ? fullQ : fullA;
      uint64_t* empty = codes ? emptyQ : emptyA;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile<BM>(c, tile);
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % depth;
          if (!mbar_wait(&empty[s], ((it / depth) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          if (!codes) {
            mbar_arrive_expect_tx(&full[s], A_BYTES);
            tma_load_2d(&tmA, &full[s], ringA + s * A_BYTES, kb * BK, c.off[t.seg] + t.m0);
          } else {
            uint8_t* sq = ringQ + s * Q_BYTES;
            mbar_arrive_expect_tx(&full[s], Q_BYTES);
            const int kq = kb * (BK / 2);
            if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
              tma_load_3d(&tmQ, &full[s], sq, kq, t.n_blk * BNB, t.seg);  // 128 rows of fc1 codes
            } else if (MODE == 0 && c.gu_layout == MOE_GU_UNFUSED) {
              const int f0 = t.n_blk * (BNB / 2);  // 64 gate rows, then the 64 up rows
              tma_load_3d(&tmG, &full[s], sq, kq, f0, t.seg);
              tma_load_3d(&tmQ, &full[s], sq + Q_BYTES / 2, kq, f0, t.seg);
            } else if (MODE == 0) {
              const int f0 = t.n_blk * (BNB / 2);
              const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
              for (int half = 0; half < 2; half++)
                tma_load_4d(&tmQ, &full[s], sq + half * (Q_BYTES / 2), kq, il ? half : f0, il ? f0 : half, t.seg);
            } else {
              tma_load_3d(&tmQ, &full[s], sq, kq, t.n_blk * BNB, t.seg);
            }
          }
        }
      }
      // every load issued into a slot has landed before the CTA may exit
      for (uint32_t j = (it > (uint32_t)depth ? it - depth : 0); j < it; j++) {
        const uint64_t t0 = global_timer();
        while (!mbar_try_wait(&full[j % depth], (j / depth) & 1) && global_timer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, tcount++) {
        const Tile t = decode_tile<BM>(c, tile);
        const int live = t.rows - t.m0 < BM ? t.rows - t.m0 : BM;  // token rows of this tile
        const uint32_t idesc = idesc_bf16_f32(BNB, (live + 15) & ~15);
        const int acc = tcount & 1;
        if (!mbar_wait(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, c.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + acc * ACC_COLS;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int sa = it % AST, sw = it % WST;
          if (!mbar_wait(&fullA[sa], (it / AST) & 1, abort_flag, c.status) ||
              !mbar_wait(&fullW[sw], (it / WST) & 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t wd = sdesc_k_sw128(smem_u32(ringW + sw * W_BYTES));  // A: decoded weights
          const uint64_t xd = sdesc_k_sw128(smem_u32(ringA + sa * A_BYTES));  // B: activations
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++)
            mma_bf16(dt, wd + 2 * kk, xd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(&emptyA[sa]);
          mma_commit(&emptyW[sw]);
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      mma_commit(drain);
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(drain, 0) && global_timer() - t0 < kTimeoutNs) {
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    // Lane r of the accumulator is weight row r (32q + lane), column j token m0 + j.
    const int q = warp & 3;                 // TMEM lane quadrant this warp may read
    const int part = (warp - 2) / 4;        // which alternate 16-token chunks it drains
    const int r = q * 32 + lane;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, tcount++) {
      const Tile t = decode_tile<BM>(c, tile);
      const int acc = tcount & 1;
      // warp-uniform: the TMEM loads below need every lane of the warp
      const bool got = mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      const int live = t.rows - t.m0;      // token rows of the tile (may exceed BM)
      const int64_t grow0 = (int64_t)c.off[t.seg] + t.m0;
      if (MODE == 0 && c.ffn == MOE_FFN_PLAIN) {
        // lane r holds fc1 feature f for the tile's tokens
        const int f = t.n_blk * BNB + r;
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
        const int f = t.n_blk * (BNB / 2) + (r >> 1);
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
            // the even lane keeps its gate values of tokens 0..7 and receives the
            // up values; the odd lane keeps up 8..15 and receives gate 8..15
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
        const int o = t.n_blk * BNB + r;
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
      mbar_arrive(&tempty[acc]);
    }
  } else if (converter_index(warp) >= 0) {
    // ------------------------------------------------------------ converters
    // Four groups of four warps; group g converts the stages it with it % 4 == g,
    // so four stages are in conversion at once.  In a group, thread = weight row:
    // it loads the row's 32 code bytes, decodes 64 elements with the row's two
    // block scales and writes the 128-byte row in the swizzled layout (the 8
    // consecutive rows of a quarter-warp hit distinct banks).
    const int cw = converter_index(warp);        // 0 .. kCvtWarps-1
    const int group = cw / kCvtGroupWarps;       // 0 .. kCvtGroups-1
    const int r = (cw % kCvtGroupWarps) * 32 + lane;  // weight row inside the tile
    const int kblocks = K / 32;                  // scale bytes per weight row
    const int rows_per_e = MODE == 1 ? c.d : (c.ffn == MOE_FFN_PLAIN || c.gu_layout == MOE_GU_UNFUSED) ? c.F : 2 * c.F;
    uint32_t it = 0;  // stage index of the tile's first k-block
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, it += nkb) {
      const Tile t = decode_tile<BM>(c, tile);
      bool rvalid;
      bool gate_row;
      const int wr = weight_row<MODE>(c, t.n_blk, r, &rvalid, &gate_row);
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
        // code rows in the slot: gate_up 64 gate rows then their 64 up rows; down in order
        const int qr = (MODE == 0 && c.ffn == MOE_FFN_GATED) ? (r & 1) * (BNB / 2) + (r >> 1) : r;
        const uint4* qrow = reinterpret_cast<const uint4*>(ringQ + sq * Q_BYTES + qr * (BK / 2));
        const uint4 q0 = qrow[0], q1 = qrow[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyQ[sq]);  // codes are in registers: the slot may refill
        if (!mbar_wait(&emptyW[sw], ((st / WST) & 1) ^ 1, abort_flag, c.status)) {
          ok = false;
          break;
        }
        decode_row_sw128(q0, q1, sc, ringW + sw * W_BYTES + r * (BK * 2), r);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&fullW[sw]);
        sc = next;
      }
      if (!ok) break;
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

bool map_act(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t pitch) {
  const uint64_t dims[2] = {K, rows > 0 ? rows : 1};
  const uint64_t strides[1] = {pitch * 2};
  const uint32_t box[2] = {BK, BM};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// e2m1 code stack [E][2F][d/2] bytes seen as 4-D: one box = 64 gate (or up) rows x 32 bytes.
bool map_codes_gate_up(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, int layout) {
  const uint64_t kb = d / 2;
  if (layout == MOE_GU_INTERLEAVED) {
    const uint64_t dims[4] = {kb, 2, F, E};
    const uint64_t strides[3] = {kb, 2 * kb, 2 * F * kb};
    const uint32_t box[4] = {BK / 2, 1, BNB / 2, 1};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  const uint64_t dims[4] = {kb, F, 2, E};
  const uint64_t strides[3] = {kb, F * kb, 2 * F * kb};
  const uint32_t box[4] = {BK / 2, BNB / 2, 1, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Down code stack [E][d][F/2] bytes: dims {F/2, d, E}, box 32 x 128 x 1.
bool map_codes_down(CUtensorMap* m, const void* base, uint64_t F, uint64_t d, uint64_t E) {
  const uint64_t kb = F / 2;
  const uint64_t dims[3] = {kb, d, E};
  const uint64_t strides[2] = {kb, d * kb};
  const uint32_t box[3] = {BK / 2, BNB, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// An [E][F][d/2] code stack (plain fc1, or an unfused gate or up stack) with
// boxes of `rows` rows x 32 bytes.
bool map_codes_rows(CUtensorMap* m, const void* base, uint64_t d, uint64_t F, uint64_t E, uint32_t rows) {
  const uint64_t kb = d / 2;
  const uint64_t dims[3] = {kb, F, E};
  const uint64_t strides[2] = {kb, F * kb};
  const uint32_t box[3] = {BK / 2, rows, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int MODE>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& q, const CUtensorMap& g, const Fp4Params& p,
                   int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(fp4_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = p.c.max_tiles < num_sms ? p.c.max_tiles : num_sms;
  return launch_pdl(fp4_gemm_kernel<MODE>, (unsigned)grid, kThreads, SMEM_BYTES, st, a, q, g, p);
}

}  // namespace

cudaError_t launch_fp4_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mQ, mG;
  bool ok = map_act(&mA, a.xg, c.d, c.R, c.d);
  if (c.ffn == MOE_FFN_PLAIN) {
    ok = ok && map_codes_rows(&mQ, a.gate_up, c.d, c.F, c.E, BNB);
    mG = mQ;
  } else if (c.gu_layout == MOE_GU_UNFUSED) {
    ok = ok && map_codes_rows(&mQ, a.gate_up, c.d, c.F, c.E, BNB / 2);
    ok = ok && map_codes_rows(&mG, a.gate, c.d, c.F, c.E, BNB / 2);
  } else {
    ok = ok && map_codes_gate_up(&mQ, a.gate_up, c.d, c.F, c.E, c.gu_layout);
    mG = mQ;
  }
  if (!ok) return cudaErrorInvalidValue;
  Fp4Params p{c,       a.gate_up_scales, a.gate_scales, (const uint16_t*)a.gate_up_bias, (const uint16_t*)a.gate_bias,
              nullptr, a.roww,           (uint16_t*)a.h};
  return launch<0>(mA, mQ, mG, p, a.num_sms, st);
}

cudaError_t launch_fp4_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mQ;
  bool ok = map_act(&mA, a.h, c.F, c.R, c.Fmax);
  ok = ok && map_codes_down(&mQ, a.down, c.F, c.d, c.E);
  if (!ok) return cudaErrorInvalidValue;
  Fp4Params p{c, a.down_scales, nullptr, nullptr, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(mA, mQ, mQ, p, a.num_sms, st);
}

}  // namespace moe
