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
//   warp 0      TMA: activations 256 x 64 (bf16, 128B swizzle) and codes 128 x 32 B
//   warp 1      TMEM owner and MMA issuer (M=128 N=128 K=16 per half)
//   warps 2-5   epilogue (bias + activation, or bias x routing weight; bf16 stores)
//   warps 6-13  converters: codes + scale -> bf16 in the 128B-swizzled K-major layout
//               the MMA descriptor reads, then a proxy fence and a barrier arrive.
// Decode: a code's 3 magnitude bits select the two bytes of its unscaled bf16 value
// through byte permutes of two 8-entry byte tables, the sign bit is moved to bit 15,
// and one bf16x2 multiply by 2^(s-127) applies the block scale.  Exact (both factors
// have at most two significant bits) for scale bytes 8..252.
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = kFp4BM;              // 256 = 2 x 128
constexpr int HALF = 128;
constexpr int BK = 64;                  // K elements per stage
constexpr int BNB = 128;                // weight rows per tile
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;    // 32 KiB
constexpr int Q_BYTES = BNB * BK / 2;   // 4 KiB of codes
constexpr int W_BYTES = BNB * BK * 2;   // 16 KiB decoded bf16
constexpr int STAGE_BYTES = A_BYTES + Q_BYTES + W_BYTES;
constexpr int ACC_COLS = 2 * BNB;       // two halves
constexpr int TMEM_COLS = 2 * ACC_COLS; // double-buffered
constexpr int kEpiWarps = 4;
constexpr int kCvtWarps = 8;
constexpr int kCvtThreads = kCvtWarps * 32;  // one (row, 32-element block) per thread and stage
constexpr int kThreads = 64 + (kEpiWarps + kCvtWarps) * 32;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint32_t IDESC = idesc_bf16_f32(HALF, BNB);
static_assert(kCvtThreads == BNB * (BK / 32), "one converter thread per (row, block)");

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

// 8 e2m1 codes (one 32-bit word, element j in bits 4j..4j+3) -> 4 bf16x2 words, scaled.
__device__ __forceinline__ void decode8(uint32_t w, __nv_bfloat162 scale2, uint32_t (&out)[4]) {
  // unscaled bf16 of magnitude code 0..7: {0, .5, 1, 1.5, 2, 3, 4, 6}
  constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;  // high bytes, codes 0-3 / 4-7
  constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;  // low bytes
  const uint32_t m = w & 0x77777777u;
  const uint32_t sel_a = m, sel_b = m >> 16;
  const uint32_t hi_a = __byte_perm(kHi0, kHi1, sel_a), lo_a = __byte_perm(kLo0, kLo1, sel_a);
  const uint32_t hi_b = __byte_perm(kHi0, kHi1, sel_b), lo_b = __byte_perm(kLo0, kLo1, sel_b);
  uint32_t p[4];
  p[0] = __byte_perm(lo_a, hi_a, 0x5140);
  p[1] = __byte_perm(lo_a, hi_a, 0x7362);
  p[2] = __byte_perm(lo_b, hi_b, 0x5140);
  p[3] = __byte_perm(lo_b, hi_b, 0x7362);
  // sign of element j (bit 4j+3) -> bit 15 (even j) or bit 31 (odd j) of its pair
  p[0] |= ((w << 12) & 0x8000u) | ((w << 24) & 0x80000000u);
  p[1] |= ((w << 4) & 0x8000u) | ((w << 16) & 0x80000000u);
  p[2] |= ((w >> 4) & 0x8000u) | ((w << 8) & 0x80000000u);
  p[3] |= ((w >> 12) & 0x8000u) | (w & 0x80000000u);
#pragma unroll
  for (int i = 0; i < 4; i++) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&p[i]);
    v = __hmul2(v, scale2);
    out[i] = *reinterpret_cast<uint32_t*>(&v);
  }
}

// bf16x2 holding 2^(s-127) twice (s = 0 is the subnormal 2^-127, 255 is NaN).
__device__ __forceinline__ __nv_bfloat162 scale_pair(uint32_t s) {
  const uint32_t b = s == 0 ? 0x0040u : (s == 255 ? 0x7FC0u : (s << 7));
  const uint32_t pr = b | (b << 16);
  return *reinterpret_cast<const __nv_bfloat162*>(&pr);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                    const Fp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* conv = full + STAGES;
  uint64_t* empty = conv + STAGES;
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
      mbar_init(&conv[s], kCvtThreads);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile<BM>(c, tile);
        const int arow = c.off[t.seg] + t.m0;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sq = sa + A_BYTES;
          mbar_arrive_expect_tx(&full[s], A_BYTES + Q_BYTES);
          tma_load_2d(&tmA, &full[s], sa, kb * BK, arow);
          if (MODE == 0) {
            const int f0 = t.n_blk * (BNB / 2);
            if (c.gu_layout == MOE_GU_INTERLEAVED) {
              tma_load_4d(&tmQ, &full[s], sq, kb * (BK / 2), 0, f0, t.seg);
              tma_load_4d(&tmQ, &full[s], sq + Q_BYTES / 2, kb * (BK / 2), 1, f0, t.seg);
            } else {
              tma_load_4d(&tmQ, &full[s], sq, kb * (BK / 2), f0, 0, t.seg);
              tma_load_4d(&tmQ, &full[s], sq + Q_BYTES / 2, kb * (BK / 2), f0, 1, t.seg);
            }
          } else {
            tma_load_3d(&tmQ, &full[s], sq, kb * (BK / 2), t.n_blk * BNB, t.seg);
          }
        }
      }
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
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, tcount++) {
        const Tile t = decode_tile<BM>(c, tile);
        const bool two = t.rows - t.m0 > HALF;  // second half holds rows of this segment
        const int acc = tcount & 1;
        if (!mbar_wait(&tempty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, c.status)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + acc * ACC_COLS;
        for (int kb = 0; kb < nkb; kb++, it++) {
          const int s = it % STAGES;
          if (!mbar_wait(&conv[s], (it / STAGES) & 1, abort_flag, c.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t bd = sdesc_k_sw128(sa + A_BYTES + Q_BYTES);
#pragma unroll
          for (int h = 0; h < 2; h++) {
            if (h == 1 && !two) break;
            const uint64_t ad = sdesc_k_sw128(sa + h * (HALF * BK * 2));
#pragma unroll
            for (int kk = 0; kk < BK / 16; kk++)
              mma_bf16(dt + h * BNB, ad + 2 * kk, bd + 2 * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
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
    const int q = warp & 3;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, tcount++) {
      const Tile t = decode_tile<BM>(c, tile);
      const int acc = tcount & 1;
      if (!mbar_wait(&tfull[acc], (tcount >> 1) & 1, abort_flag, c.status)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; h++) {
        const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS + h * BNB;
        const int row = t.m0 + h * HALF + q * 32 + lane;
        const bool valid = row < t.rows;
        if (!__any_sync(0xffffffffu, valid)) continue;
        const int64_t grow = (int64_t)c.off[t.seg] + row;
        if (MODE == 0) {
          const int F = c.F;
          const int f0 = t.n_blk * (BNB / 2);
          const uint16_t* bias = p.gate_up_bias ? p.gate_up_bias + (int64_t)t.seg * 2 * F : nullptr;
          const bool il = c.gu_layout == MOE_GU_INTERLEAVED;
          uint16_t* out = p.out + grow * c.Fmax;
#pragma unroll 1
          for (int ch = 0; ch < (BNB / 2) / 16; ch++) {
            uint32_t g[16], u[16];
            tmem_ld16(tb + ch * 16, g);
            tmem_ld16(tb + BNB / 2 + ch * 16, u);
            tmem_ld_wait();
            const int fb = f0 + ch * 16;
            if (valid && fb < F) {
              uint32_t packed[8];
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                float hv[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; h2++) {
                  const int f = fb + i + h2;
                  float gv = __uint_as_float(g[i + h2]), uv = __uint_as_float(u[i + h2]);
                  if (bias && f < F) {
                    gv += bf16_to_f32(bias[il ? 2 * f : f]);
                    uv += bf16_to_f32(bias[il ? 2 * f + 1 : F + f]);
                  }
                  hv[h2] = gated_act(c.act, gv, uv);
                }
                packed[i / 2] = pack_bf16x2(hv[0], hv[1]);
              }
              if (fb + 16 <= F) {
                uint4* dst = reinterpret_cast<uint4*>(out + fb);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
              } else {
                for (int i = 0; i < 16 && fb + i < F; i++)
                  out[fb + i] = (uint16_t)(packed[i / 2] >> (16 * (i & 1)));
              }
            }
          }
        } else {
          const int N = c.d;
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
            if (valid && ob < N) {
              uint32_t packed[8];
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                float o[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; h2++) {
                  float a = __uint_as_float(v[i + h2]);
                  if (bias && ob + i + h2 < N) a += bf16_to_f32(bias[ob + i + h2]);
                  o[h2] = a * w;
                }
                packed[i / 2] = pack_bf16x2(o[0], o[1]);
              }
              if (ob + 16 <= N) {
                uint4* dst = reinterpret_cast<uint4*>(out + ob);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
              } else {
                for (int i = 0; i < 16 && ob + i < N; i++)
                  out[ob + i] = (uint16_t)(packed[i / 2] >> (16 * (i & 1)));
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  } else {
    // ------------------------------------------------------------ converters
    const int u = threadIdx.x - 64 - kEpiWarps * 32;  // 0 .. kCvtThreads-1
    const int r = u % BNB;                           // weight row inside the tile
    const int b = u / BNB;                           // 32-element block inside the stage
    const int kblocks = K / 32;                      // scale bytes per weight row
    const int rows_per_e = MODE == 0 ? 2 * c.F : c.d;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const Tile t = decode_tile<BM>(c, tile);
      bool rvalid;
      const int wr = weight_row<MODE>(c, t.n_blk, r, &rvalid);
      const uint8_t* srow = p.scales + ((int64_t)t.seg * rows_per_e + wr) * kblocks;
      // scale bytes of this thread's block for k-blocks kb .. kb+3, loaded ahead
      auto load_scale = [&](int kb) -> uint32_t {
        const int col = kb * 2 + b;
        return (rvalid && kb < nkb && col < kblocks) ? (uint32_t)__ldg(srow + col) : 127u;
      };
      uint32_t s0 = load_scale(0), s1 = load_scale(1), s2 = load_scale(2), s3 = load_scale(3);
      bool ok = true;
      for (int kb = 0; kb < nkb; kb++, it++) {
        const uint32_t s4 = load_scale(kb + 4);
        const int st = it % STAGES;
        if (!mbar_wait(&full[st], (it / STAGES) & 1, abort_flag, c.status)) {
          ok = false;
          break;
        }
        uint8_t* base = smem + st * STAGE_BYTES;
        const uint4 q = *reinterpret_cast<const uint4*>(base + A_BYTES + r * (BK / 2) + b * 16);
        uint8_t* wrow = base + A_BYTES + Q_BYTES + r * (BK * 2);
        const __nv_bfloat162 sc = scale_pair(s0);
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int wi = 0; wi < 4; wi++) {
          uint32_t o[4];
          decode8(words[wi], sc, o);
          const int chunk = b * 4 + wi;  // 16-byte chunk of the 128-byte row
          *reinterpret_cast<uint4*>(wrow + ((chunk ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&conv[st]);
        s0 = s1;
        s1 = s2;
        s2 = s3;
        s3 = s4;
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
