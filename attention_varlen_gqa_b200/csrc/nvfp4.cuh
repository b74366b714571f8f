// nvfp4.cuh -- NVFP4 quantise-dequantise pieces for the decode's P and V
// (NVIDIA/Model-Optimizer PR 1941, "Add split-k decode kernel for skip
// softmax", What does this PR do?, third bullet, and Usage: p_qdq / v_qdq =
// "nvfp4" with an amax each).
//
// Per block of 16 values x along the key axis, with the tensor constants
// k = 448 / amax and g = 2688 / amax (fp32):
//   s = E4M3(b * k), b = max |x_i|   (round to nearest even, saturating)
//   r = g / s (0 when s = 0)
//   q_i = E2M1(x_i * r)               (round to nearest even, saturating at 6)
// and the kernel multiplies q_i * s (exact in f16 and bf16: at most 6
// significant bits), leaving the factor 1 / g for the output.  The fp32
// products are taken with explicit round-to-nearest multiplies; the two
// format conversions are the sm_100a cvt instructions.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace attn {

// (lo, hi) fp32 -> E2M1 pair -> f16x2 (lo in bits 0-15).
ATTN_DEVICE uint32_t e2m1x2_as_f16x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// (lo, hi) fp32 -> E4M3 pair -> f16x2 (lo in bits 0-15).
ATTN_DEVICE uint32_t e4m3x2_as_f16x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

ATTN_DEVICE float f16_lo(uint32_t x) { return __half2float(__ushort_as_half((unsigned short)(x & 0xffffu))); }
ATTN_DEVICE float f16_hi(uint32_t x) { return __half2float(__ushort_as_half((unsigned short)(x >> 16))); }

// Two floats -> packed f16 (round to nearest even); `lo` lands in bits 0..15.
ATTN_DEVICE uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

ATTN_DEVICE uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// f16x2 -> bf16x2 of the same values (exact for the dequantised products,
// which have at most 6 significant bits and lie inside both ranges).
ATTN_DEVICE uint32_t f16x2_to_bf16x2(uint32_t x) { return pack_bf16x2(f16_lo(x), f16_hi(x)); }

// Both halves of an f16x2 set to its low (hi = false) or high half.
ATTN_DEVICE uint32_t f16x2_bcast(uint32_t x, bool hi) {
  return hi ? ((x & 0xffff0000u) | (x >> 16)) : ((x & 0xffffu) | (x << 16));
}

// g / s for a block scale s (an E4M3 value as fp32, so at most 3 mantissa
// bits: s = (1 + m / 8) 2^E), from the tensor's table held across the warp
// (lane j: g / (1 + (j & 7) / 8), fp32 round to nearest): g / s is that
// entry times 2^-E exactly, so it equals the correctly rounded quotient.
// Every lane of the warp calls it.  0 for s = 0.
ATTN_DEVICE float ratio_from_table(float s, float tab) {
  const uint32_t b = __float_as_uint(s);
  const float t = __shfl_sync(0xffffffffu, tab, (int)((b >> 20) & 7u));
  const uint32_t e = b & 0x7f800000u;
  return s > 0.f ? __uint_as_float(__float_as_uint(t) - (e - 0x3f800000u)) : 0.f;
}

// Largest |.| over the halves of four bf16x2 words, as a bf16x2 pair:
// low half from (a, b), high half from (c, d).
ATTN_DEVICE uint32_t absmax_pairs_bf16(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  uint32_t x, y, lo, hi, r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(x) : "r"(a & 0x7fff7fffu), "r"(b & 0x7fff7fffu));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(c & 0x7fff7fffu), "r"(d & 0x7fff7fffu));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(lo) : "r"(x), "r"(y));   // (x.lo, y.lo)
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(hi) : "r"(x), "r"(y));   // (x.hi, y.hi)
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(lo), "r"(hi));
  return r;
}

ATTN_DEVICE uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// The dequantised pair (times g) of a bf16x2 pair of one block: its E2M1
// codes at ratio r (r2 = the pair (r, r)), times the block scale (f16x2 with
// both halves s).  The two products are one packed fp32 multiply, each lane
// rounded to nearest as a scalar product would be.
ATTN_DEVICE uint32_t qdq_bf16_pair(uint32_t x, uint64_t r2, uint32_t s2) {
  uint64_t y;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(f2_pack(bf16_lo(x), bf16_hi(x))), "l"(r2));
  float y0, y1;
  f2_unpack(y, y0, y1);
  return hmul2_u32(e2m1x2_as_f16x2(y0, y1), s2);
}

// m16n8k16 MMA with f16 operands (fp32 accumulate).
ATTN_DEVICE void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace attn
