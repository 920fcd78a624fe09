// nvfp4.cuh -- NVFP4 block quantiser (device side).
//
// Format (the 4-bit precision listed for Blackwell / B200 in chaosnode.de
// "Nunchaku Lite: 4-Bit Diffusion-Inferenz direkt in Diffusers", section
// "Hardware-Support"): E2M1 element codes {0,.5,1,1.5,2,3,4,6} x sign, one
// E4M3 scale per 16 consecutive elements along K.  For a block v[0..15]:
//     a = max|v_i|,  s = E4M3_rn_satfinite(f32(a / 6)),
//     q_i = E2M1_rn_satfinite(f32(v_i / s))   (q_i = +-0 when s == 0),
// with IEEE float32 division, round-to-nearest-even conversions, and the sign
// bit of E2M1 kept (a negative value that rounds to zero is code 0x8).
// Codes are packed two per byte, element 2j in the low nibble of byte j.
#pragma once

#include <stdint.h>

namespace svdq {

// E4M3 code (0x00..0x7E) of a non-negative float, RNE, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float x) {
  uint16_t out;
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
      "mov.b16 %0, t;\n\t}\n"
      : "=h"(out)
      : "f"(0.0f), "f"(x));
  return static_cast<uint32_t>(out) & 0xFFu;
}

// Exact float value of a non-negative E4M3 code.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0x1p-9f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight E2M1 magnitude codes of |q0..q7| (RNE, satfinite), packed with q0 in
// the lowest nibble; sign bits are added by the caller.
__device__ __forceinline__ uint32_t e2m1x8_magnitudes(const float (&a)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}\n"
      : "=r"(out)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]),
        "f"(a[7]));
  return out;
}

// E2M1 magnitude codes of 8 non-negative float32 bit patterns.
__device__ __forceinline__ uint32_t e2m1x8_of_bits(const uint32_t (&b)[8]) {
  const float a[8] = {__uint_as_float(b[0]), __uint_as_float(b[1]), __uint_as_float(b[2]),
                      __uint_as_float(b[3]), __uint_as_float(b[4]), __uint_as_float(b[5]),
                      __uint_as_float(b[6]), __uint_as_float(b[7])};
  return e2m1x8_magnitudes(a);
}

// Quantise 8 consecutive values forming one half of a 16-element block; the
// other half lives on lane (laneid ^ 1).  Must be called by all 32 lanes of
// the warp.  Returns the 8 packed codes; `scale_code` receives the block's
// E4M3 code (identical on both lanes of the pair).
//
// The codes are E2M1_rn(RN(v_i / s)) exactly, without one IEEE division per
// element: q_i = RN(v_i * RN(1/s)) differs from v_i / s by at most
// (2^-23 + 2^-48) |v_i / s|, i.e. by less than 2 ulps of q_i, and RN(v_i / s)
// lies within half an ulp of v_i / s; so RN(v_i / s) is inside [lo, hi], the
// float32 values 4 representable steps below and above |q_i| (4 steps span at
// least 2 ulps even across a binade boundary).  E2M1 rounding is monotone, so
// when lo and hi get the same code every value in between does too, and that
// code is the answer.  Otherwise (|q_i| within a few ulps of a rounding
// threshold, exact ties included) the block takes the IEEE division.
__device__ __forceinline__ uint32_t nvfp4_quant_half_block(const float (&v)[8],
                                                          uint32_t& scale_code) {
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
  const uint32_t sc = e4m3_rn_satfinite(__fdiv_rn(am, 6.0f));
  const float s = e4m3_to_f32(sc);
  scale_code = sc;
  uint32_t signs = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) signs |= (__float_as_uint(v[i]) >> 31) << (4 * i + 3);
  if (s == 0.0f) return signs;                 // every |v_i| / s taken as +-0
  const float inv_s = __frcp_rn(s);
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t m = __float_as_uint(fabsf(__fmul_rn(v[i], inv_s)));
    lo[i] = (m > 4u ? m : 4u) - 4u;
    hi[i] = m + 4u;
  }
  const uint32_t clo = e2m1x8_of_bits(lo);
  const uint32_t chi = e2m1x8_of_bits(hi);
  if (clo == chi) return clo | signs;
  float mag[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mag[i] = fabsf(__fdiv_rn(v[i], s));
  return e2m1x8_magnitudes(mag) | signs;
}

// Packed float32 pairs (Blackwell f32x2 arithmetic, each half an ordinary
// IEEE round-to-nearest-even operation).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t d, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Entry c of the E4M3 table: (s, RN(1/s)) for s = E4M3 value of code c, and
// (0, 0) for c == 0.
__device__ __forceinline__ float2 e4m3_table_entry(uint32_t c) {
  const float s = e4m3_to_f32(c);
  return make_float2(s, s == 0.0f ? 0.0f : __frcp_rn(s));
}

// Correctly rounded quotients v / s of a pair, without a division, by the
// quotient-correction step of Markstein (IBM J. Res. Dev. 34(1), 1990, "Computation
// of elementary functions on the IBM RISC System/6000 processor"): with
// y = RN(1/s) and q0 = RN(v y) (faithful), the remainder v - s q0 is exact in
// one FMA and RN(q0 + (v - s q0) y) = RN(v / s).
// The input is u = -v (the pair negated) and the constants are s2 = (s, s) and
// neg_y2 = (-y, -y): then q0 = u (-y), rn = s q0 + u = -(v - s q0) and the
// result is q0 + rn (-y).  Every step is the textbook one up to exact
// negations, and a zero v gives a zero quotient with v's sign (-0 / s = -0):
// the plain ordering would return +0 for v = -0, since the exact remainder
// +0 + (-0) rounds to +0.  With s = y = 0 the result is a zero with v's sign.
__device__ __forceinline__ uint64_t quotient_f32x2(uint64_t u, uint64_t s2, uint64_t neg_y2) {
  const uint64_t q0 = f32x2_mul(u, neg_y2);
  const uint64_t rn = f32x2_fma(s2, q0, u);
  return f32x2_fma(rn, neg_y2, q0);
}

// E2M1 codes (RNE, satfinite, sign kept) of the 8 signed floats q0..q7, q0 in
// the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8_signed(const uint64_t (&q)[4]) {
  float a[8];
#pragma unroll
  for (int u = 0; u < 4; ++u) f32x2_unpack(q[u], a[2 * u], a[2 * u + 1]);
  return e2m1x8_magnitudes(a);
}

// Same result as nvfp4_quant_half_block for the 8 values v, given NEGATED and
// packed in pairs (nv[u] = (-v[2u], -v[2u+1])), taking s and RN(1/s) from
// `tab` (128 entries of e4m3_table_entry, in shared memory) and every
// quotient -- amax / 6 as well as the element quotients -- from
// quotient_f32x2 (six = (6, 6), neg_y6 = (-RN(1/6), -RN(1/6))).  Called by
// all 32 lanes; the other half of the block lives on lane (laneid ^ 1).
__device__ __forceinline__ uint32_t nvfp4_quant_half_block_x2(const uint64_t (&nv)[4], const float2* tab,
                                                             uint64_t six, uint64_t neg_y6,
                                                             uint32_t& scale_code) {
  float am = 0.0f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float lo, hi;
    f32x2_unpack(nv[u], lo, hi);
    am = fmaxf(am, fmaxf(fabsf(lo), fabsf(hi)));
  }
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
  float a6, a6b;
  f32x2_unpack(quotient_f32x2(f32x2_pack(-am, -am), six, neg_y6), a6, a6b);   // RN(amax / 6)
  const uint32_t sc = e4m3_rn_satfinite(a6);
  scale_code = sc;
  const float2 sy = tab[sc];
  const uint64_t s2 = f32x2_pack(sy.x, sy.x), neg_y2 = f32x2_pack(-sy.y, -sy.y);
  uint64_t q[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) q[u] = quotient_f32x2(nv[u], s2, neg_y2);
  return e2m1x8_signed(q);
}

// One whole 16-element block in one thread: the same result as
// nvfp4_quant_half_block_x2 for the pair of lanes holding its halves, for the
// 16 values given NEGATED and packed in pairs (nv[u] = (-v[2u], -v[2u+1])),
// with s and RN(1/s) read from `tab` (the 128 entries of e4m3_table_entry,
// in shared memory).  The block maximum is taken as a tree (max is exact, so
// the order does not matter).  Returns the 16 codes, element 0 in the lowest
// nibble.
__device__ __forceinline__ uint64_t nvfp4_quant_block16_x2(const uint64_t (&nv)[8], const float2* tab, uint64_t six,
                                                          uint64_t neg_y6, uint32_t& scale_code) {
  float m[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    float lo, hi;
    f32x2_unpack(nv[u], lo, hi);
    m[u] = fmaxf(fabsf(lo), fabsf(hi));
  }
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int u = 0; u < w; ++u) m[u] = fmaxf(m[u], m[u + w]);
  const float am = m[0];
  float a6, a6b;
  f32x2_unpack(quotient_f32x2(f32x2_pack(-am, -am), six, neg_y6), a6, a6b);   // RN(amax / 6)
  const uint32_t sc = e4m3_rn_satfinite(a6);
  scale_code = sc;
  const float2 sy = tab[sc];
  const uint64_t s2 = f32x2_pack(sy.x, sy.x), neg_y2 = f32x2_pack(-sy.y, -sy.y);
  uint64_t q0[4], q1[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    q0[u] = quotient_f32x2(nv[u], s2, neg_y2);
    q1[u] = quotient_f32x2(nv[u + 4], s2, neg_y2);
  }
  return static_cast<uint64_t>(e2m1x8_signed(q0)) | (static_cast<uint64_t>(e2m1x8_signed(q1)) << 32);
}

// Byte offset of scale (row, kb16) in the scale-factor tile layout:
// 512-byte tiles of 128 rows x 4 scales, tile (row/128, kb16/4) at
// ((row/128) * (K/64) + kb16/4) * 512, inside it (row%32)*16 + ((row/32)%4)*4 + kb16%4.
__host__ __device__ __forceinline__ uint64_t sf_offset(uint32_t row, uint32_t kb16, uint32_t K) {
  const uint64_t tile = static_cast<uint64_t>(row >> 7) * (K >> 6) + (kb16 >> 2);
  return tile * 512u + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u + (kb16 & 3u);
}

// Round float64 to bf16 (RNE, single rounding); returns the bit pattern.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  if (fabs(x) < 0x1p-126) {
    // bf16 subnormal range: multiples of 2^-133, ties to even (rint).
    const float f = static_cast<float>(rint(x * 0x1p133) * 0x1p-133);
    return static_cast<uint16_t>(__float_as_uint(f) >> 16);
  }
  unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  const unsigned long long lsb = (u >> 45) & 1ull;
  u = (u + ((1ull << 44) - 1ull) + lsb) & ~((1ull << 45) - 1ull);
  const float f = static_cast<float>(__longlong_as_double(static_cast<long long>(u)));
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Two floats -> packed bf16x2 (RNE), first argument in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
  return out;
}

}  // namespace svdq
