// mxfp4.cuh -- decoding OCP MX v1.0 MXFP4 weights (e2m1 codes, two per byte with
// the even element in the low nibble; one e8m0 scale byte per 32 elements) to
// bf16 in registers.  Shared by the MXFP4 grouped GEMMs.
//
// The hardware conversion cvt.rn.f16x2.e2m1x2 turns each code byte into two exact
// f16 values; shifting an f16's exponent and mantissa right by 3 bits (sign kept)
// gives a bf16 of the same value times 2^-112, and one bf16x2 multiply by
// 2^(s-15) applies the block scale and undoes the bias.  Exact (both factors have
// at most two significant bits, the product stays normal) for scale bytes 2..142;
// larger scale bytes take a second multiply.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {
namespace mxfp4 {

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

// One weight row of a 64-deep K step: 32 code bytes (q0, q1) and the two block
// scale bytes (sc: low byte first) -> 64 bf16 values written as the 128-byte row
// `r` of a K-major tile in the 128-byte-swizzled layout the UMMA descriptors
// read (16-byte chunk j stored at chunk j ^ (r % 8); the 8 consecutive rows of a
// quarter-warp hit distinct banks).
__device__ __forceinline__ void decode_row_sw128(const uint4& q0, const uint4& q1, uint32_t sc, uint8_t* wrow,
                                                 int r) {
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
}

}  // namespace mxfp4
}  // namespace moe
