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
// Tile: 256 activation rows (two M=128 halves) x 128 weight rows x K, fp32 in TMEM
// (2 halves x 128 columns, double-buffered).  Both halves share each decoded
// weight stage, halving the decode work per FLOP.  Warp roles:
//   warp 0      TMA producer of activations 256 x 64 (bf16, 128B swizzle)
//   warp 1      TMEM owner and MMA issuer (M=128 N=128 K=16 per half)
//   warp 26     TMA producer of the codes, 128 x 32 bytes, running up to 6 stages ahead
//   warps 2-9   epilogue (bias + activation, or bias x routing weight; bf16 stores);
//               warps 2-5 drain the first M half, warps 6-9 the second
//   warps 10-25 converters in four groups, group g owning stages it % 4 == g:
//               codes + scale -> bf16 in the 128B-swizzled K-major layout the MMA
//               descriptor reads, then a proxy fence and one arrive per warp.
// Decode: the hardware conversion cvt.rn.f16x2.e2m1x2 turns each code byte into two
// exact f16 values; shifting an f16's exponent and mantissa right by 3 bits (sign
// kept) gives a bf16 of the same value times 2^-112, and one bf16x2 multiply by
// 2^(s-15) applies the block scale and undoes the bias.  Exact (both factors have
// at most two significant bits, the product stays normal) for scale bytes 2..142;
// larger scale bytes take a second multiply.
#include <cuda_bf16.h>

#include "epilogue.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = kFp4BM;              // 256 = 2 x 128
constexpr int HALF = 128;
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
constexpr int ACC_COLS = 2 * BNB;       // two halves
constexpr int TMEM_COLS = 2 * ACC_COLS; // double-buffered
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant: one per M half
constexpr int kCvtWarps = 16;
constexpr int kCvtGroups = 4;                // converter groups, each owning every 4th stage
constexpr int kCvtGroupWarps = kCvtWarps / kCvtGroups;
constexpr int kThreads = 64 + (kEpiWarps + kCvtWarps + 1) * 32;  // + the codes producer warp
constexpr int SMEM_BYTES = RING_BYTES + 1024 + 512;
constexpr uint32_t IDESC = idesc_bf16_f32(HALF, BNB);
static_assert(kCvtGroupWarps * 32 == BNB, "one converter thread per weight row in a group");
static_assert(WST % kCvtGroups == 0, "a group's stages map to its own decoded-weight slots");

struct Fp4Params {
  GemmCommon c;
  const uint8_t* scales;        // e8m0 [E, rows, K/32]
  const uint16_t* gate_up_bias; // [E, 2F] or null
  const uint16_t* down_bias;    // [E, d] or null
  const float* roww;            // [R]
  uint16_t* out;                // h [rows, Fmax] or Y [rows, d]
};

template <int MODE>
__device__ __forceinline__ int k_extent(const GemmCommon& c) {
  return MODE == 0 ? c.d : c.F;
}

// Row of the scale / code stack (inside expert e) that tile row r reads.
template <int MODE>
__device__ __forceinline__ int weight_row(const GemmCommon& c, int n_blk, int r, bool* valid) {
  if (MODE == 0) {
    const int half = r / (BNB / 2);
    const int f = n_blk * (BNB / 2) + r % (BNB / 2);
    *valid = f < c.F;
    if (c.gu_layout == MOE_GU_INTERLEAVED) return 2 * f + half;
    return half ? c.F + f : f;
  }
  const int o = n_blk * BNB + r;
  *valid = o < c.d;
  return o;
}

// 8 e2m1 codes (one 32-bit word, element j in bits 4j..4j+3) -> 4 f16x2 words
// (element 2i in the low half of word i), exact.
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

// f16x2 of e2m1 values -> bf16x2 of the same values times 2^-112 (exponent and
// mantissa bits moved down by 3, signs kept; the low 3 mantissa bits are zero).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2_biased(uint32_t h) {
  return ((h >> 3) & 0x0FFF0FFFu) | (h & 0x80008000u);
}

// bf16x2 multiplier that applies 2^(s-127) to a value biased by 2^-112: 2^(s-15).
// For s > 142 that factor is not a bf16; `extra` then holds the remaining 2^(s-142).
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t s, uint32_t* extra) {
  uint32_t e = s + 112;   // bf16 exponent field of 2^(s-15)
  *extra = 0;
  if (s == 255) e = 255;  // NaN scale propagates
  else if (e > 254) {
    *extra = (s - 142 + 127) << 7;  // 2^(s-142)
    *extra |= *extra << 16;
    e = 254;                          // 2^127
  }
  const uint32_t b = (e << 7) | (s == 255 ? 0x40u : 0u);
  return b | (b << 16);
}

__device__ __forceinline__ uint32_t bmul(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  x = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&x);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                    const Fp4Params p) {
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
  constexpr int kCodesWarp = 2 + kEpiWarps + kCvtWarps;

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
  const uint32_t tmem_base = *tmem_slot;
  const int total = c.tiles[c.NS];
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
            if (MODE == 0) {
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
        const bool two = t.rows - t.m0 > HALF;  // second half holds rows of this segment
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
          const uint64_t bd = sdesc_k_sw128(smem_u32(ringW + sw * W_BYTES));
#pragma unroll
          for (int h = 0; h < 2; h++) {
            if (h == 1 && !two) break;
            const uint64_t ad = sdesc_k_sw128(smem_u32(ringA + sa * A_BYTES + h * (HALF * BK * 2)));
#pragma unroll
            for (int kk = 0; kk < BK / 16; kk++)
              mma_bf16(dt + h * BNB, ad + 2 * kk, bd + 2 * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
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
    const int q = warp & 3;                 // TMEM lane quadrant this warp may read
    const int h = (warp - 2) / 4;           // M half this warp drains
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, tcount++) {
      const Tile t = decode_tile<BM>(c, tile);
      const int acc = tcount & 1;
      if (!mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS + h * BNB;
      const int row = t.m0 + h * HALF + q * 32 + lane;
      const bool valid = row < t.rows;
      if (__any_sync(0xffffffffu, valid)) {
        const int64_t grow = (int64_t)c.off[t.seg] + row;
        if (MODE == 0) {
          const int f0 = t.n_blk * (BNB / 2);
          const uint16_t* bias = p.gate_up_bias ? p.gate_up_bias + (int64_t)t.seg * 2 * c.F : nullptr;
          const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
          uint16_t* out = p.out + grow * c.Fmax;
#pragma unroll 1
          for (int ch = 0; ch < (BNB / 2) / 16; ch++) {
            uint32_t g[16], u[16];
            tmem_ld16(tb + ch * 16, g);
            tmem_ld16(tb + BNB / 2 + ch * 16, u);
            tmem_ld_wait();
            const int fb = f0 + ch * 16;
            if (valid && fb < c.F) gate_up_chunk(g, u, bias, fb, c.F, il, c.act, out);
          }
        } else {
          const int n0 = t.n_blk * BNB;
          const uint16_t* bias = p.down_bias ? p.down_bias + (int64_t)t.seg * c.d : nullptr;
          const float w = (c.weigh_inputs || !valid) ? 1.f : p.roww[grow];
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
      mbar_arrive(&tempty[acc]);
    }
  } else if (warp < kCodesWarp) {
    // ------------------------------------------------------------ converters
    // Four groups of four warps; group g converts the stages it with it % 4 == g,
    // so four stages are in conversion at once.  In a group, thread = weight row:
    // it loads the row's 32 code bytes, decodes 64 elements with the row's two
    // block scales and writes the 128-byte row in the swizzled layout (the 8
    // consecutive rows of a quarter-warp hit distinct banks).
    const int cw = warp - 2 - kEpiWarps;         // 0 .. kCvtWarps-1
    const int group = cw / kCvtGroupWarps;       // 0 .. kCvtGroups-1
    const int r = (cw % kCvtGroupWarps) * 32 + lane;  // weight row inside the tile
    const int kblocks = K / 32;                  // scale bytes per weight row
    const int rows_per_e = MODE == 0 ? 2 * c.F : c.d;
    uint32_t it = 0;  // stage index of the tile's first k-block
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, it += nkb) {
      const Tile t = decode_tile<BM>(c, tile);
      bool rvalid;
      const int wr = weight_row<MODE>(c, t.n_blk, r, &rvalid);
      const uint8_t* srow = p.scales + ((int64_t)t.seg * rows_per_e + wr) * kblocks;
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
        const uint4* qrow = reinterpret_cast<const uint4*>(ringQ + sq * Q_BYTES + r * (BK / 2));
        const uint4 q0 = qrow[0], q1 = qrow[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyQ[sq]);  // codes are in registers: the slot may refill
        if (!mbar_wait(&emptyW[sw], ((st / WST) & 1) ^ 1, abort_flag, c.status)) {
          ok = false;
          break;
        }
        uint8_t* wrow = ringW + sw * W_BYTES + r * (BK * 2);
        const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int blk = 0; blk < 2; blk++) {
          uint32_t extra;
          const uint32_t scale = scale_bf16x2((sc >> (8 * blk)) & 0xFF, &extra);
#pragma unroll
          for (int wi = 0; wi < 4; wi++) {
            uint32_t h[4], o[4];
            e2m1x8_to_f16x8(words[blk * 4 + wi], h);
#pragma unroll
            for (int i = 0; i < 4; i++) {
              o[i] = bmul(f16x2_to_bf16x2_biased(h[i]), scale);
              if (extra) o[i] = bmul(o[i], extra);
            }
            const int chunk = blk * 4 + wi;  // 16-byte chunk (8 elements) of the 128-byte row
            *reinterpret_cast<uint4*>(wrow + ((chunk ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
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

template <int MODE>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& q, const Fp4Params& p, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(fp4_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = p.c.max_tiles < num_sms ? p.c.max_tiles : num_sms;
  fp4_gemm_kernel<MODE><<<grid, kThreads, SMEM_BYTES, st>>>(a, q, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fp4_gate_up(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mQ;
  bool ok = map_act(&mA, a.xg, c.d, c.R, c.d);
  ok = ok && map_codes_gate_up(&mQ, a.gate_up, c.d, c.F, c.E, c.gu_layout);
  if (!ok) return cudaErrorInvalidValue;
  Fp4Params p{c, a.gate_up_scales, (const uint16_t*)a.gate_up_bias, nullptr, a.roww, (uint16_t*)a.h};
  return launch<0>(mA, mQ, p, a.num_sms, st);
}

cudaError_t launch_fp4_down(const TcArgs& a, cudaStream_t st) {
  const GemmCommon& c = a.c;
  if (c.max_tiles == 0) return cudaSuccess;
  CUtensorMap mA, mQ;
  bool ok = map_act(&mA, a.h, c.F, c.R, c.Fmax);
  ok = ok && map_codes_down(&mQ, a.down, c.F, c.d, c.E);
  if (!ok) return cudaErrorInvalidValue;
  Fp4Params p{c, a.down_scales, nullptr, (const uint16_t*)a.down_bias, a.roww, (uint16_t*)a.Y};
  return launch<1>(mA, mQ, p, a.num_sms, st);
}

}  // namespace moe
