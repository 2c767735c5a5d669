// NVFP4 group arithmetic (device): a 16-element group's UE4M3 factor, its decoded scale and
// its E2M1 codes, every step the correctly rounded FP32 operation that the format's
// definition names:
//   s_t = RN(amax_t / 2688)                            tensor scale (2688 = 6 * 448)
//   e   = E4M3_RNE_sat(RN(RN(amax_g / 6) / s_t))       the group's factor byte
//   S   = RN(dec(e) * s_t)                             its decoded scale
//   q   = E2M1_RNE_sat(RN(x / S)), a signed zero when S == 0
// The divisions run as Markstein's FMA correction of a product with a correctly rounded
// reciprocal (P. Markstein, IBM J. Res. Develop. 34(1), 1990): q = RN(a * y),
// q' = RN(q + RN(a - q * b) * y) with y = RN(1 / b). Where that sequence could leave the
// normal range (s_t or S below 2^-90, amax_g below 2^-100) the exact path uses IEEE division.
// The fast path is checked against IEEE division over its whole domain by a GPU test.
#pragma once

#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"
#include "quant_math.cuh"

namespace puro {

constexpr float kNvTensorDiv = 2688.0f;  // 6 * 448: E2M1 max times E4M3 max
constexpr float kNvInv6 = 1.0f / 6.0f;    // RN(1/6), folded at compile time

// two E2M1 codes in one byte: `lo` in bits 0..3, `hi` in bits 4..7 (RN, satfinite)
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t v;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(v)
      : "f"(hi), "f"(lo));
  return v & 0xFFu;
}

// value of a non-negative E4M3 byte (exact): subnormal m * 2^-9, normal (8 + m) * 2^(e - 10)
__device__ __forceinline__ float ue4m3_value(uint32_t b) {
  const uint32_t ex = (b >> 3) & 0xFu, m = b & 7u;
  return ex == 0 ? static_cast<float>(m) * 0.001953125f  // 2^-9
                 : __uint_as_float(((ex + 120u) << 23) | (m << 20));
}

// The tensor's constants: s_t, and RN(1 / s_t) when the fast path applies. `all_fast`: s_t >=
// 2^-81, so that every group of the tensor takes the fast path: a group maximum below 2^-100
// gives a quotient by s_t below 2^-21 (factor 0, whatever its last bits), and every non-zero
// factor's S = dec(e) * s_t is at least 2^-9 * 2^-81 = 2^-90.
struct NvTensor {
  float s_t;
  float r_t;
  bool fast;
  bool all_fast;
};

__device__ __forceinline__ NvTensor nv_tensor(float amax_t) {
  NvTensor t;
  t.s_t = __fdiv_rn(amax_t, kNvTensorDiv);
  t.fast = t.s_t >= 0x1p-90f;  // s_t <= 2^128 / 2688 < 2^120 always
  t.all_fast = t.s_t >= 0x1p-81f;
  t.r_t = t.fast ? rcp_rn_fast(t.s_t) : 0.0f;
  return t;
}

// The group's factor byte and decoded scale S, with IEEE division throughout (out of line:
// only groups and tensors far below the normal range take it). Returns (e, bits of S).
__device__ __noinline__ uint2 nv_factor_exact(float amax_g, float s_t) {
  if (s_t > 0.0f) {
    const uint32_t e = e4m3x2(__fdiv_rn(__fdiv_rn(amax_g, 6.0f), s_t), 0.0f) & 0xFFu;
    return make_uint2(e, __float_as_uint(__fmul_rn(ue4m3_value(e), s_t)));
  }
  return make_uint2(0u, 0u);
}

// The same, by Markstein's correction when the tensor and the group allow it (amax_g = 0, or
// amax_g >= 2^-100 so that amax_g / 6 is a normal number; the quotient by s_t is at most
// about 448, and where it is below the normal range its factor is zero either way).
// ALL_FAST: the caller has checked t.all_fast, and no group needs the exact path.
template <bool ALL_FAST = false>
__device__ __forceinline__ uint32_t nv_factor(float amax_g, const NvTensor &t, float &S) {
  if (ALL_FAST || (t.fast && (amax_g == 0.0f || amax_g >= 0x1p-100f))) {
    const float q = __fmul_rn(amax_g, kNvInv6);
    const float d = __fmaf_rn(__fmaf_rn(-q, 6.0f, amax_g), kNvInv6, q);
    const float q2 = __fmul_rn(d, t.r_t);
    const float v = __fmaf_rn(__fmaf_rn(-q2, t.s_t, d), t.r_t, q2);
    const uint32_t e = e4m3x2(v, 0.0f) & 0xFFu;
    S = __fmul_rn(ue4m3_value(e), t.s_t);
    return e;
  }
  const uint2 r = nv_factor_exact(amax_g, t.s_t);
  S = __uint_as_float(r.y);
  return r.x;
}

// The divider of a group with decoded scale S: RN(1 / S) packed for the fast path, which
// applies when S == 0 (every quotient a signed zero: r = 0, s = 1) or S >= 2^-90.
struct NvDivider {
  uint64_t nr2;  // (-r, -r)
  uint64_t s2;   // (s, s)
  bool fast;
};

template <bool ALL_FAST = false>
__device__ __forceinline__ NvDivider nv_divider(float S) {
  NvDivider d;
  d.fast = ALL_FAST || S == 0.0f || S >= 0x1p-90f;
  const float s = S == 0.0f ? 1.0f : S;
  const float r = S == 0.0f ? 0.0f : (d.fast ? rcp_rn_fast(S) : 0.0f);
  d.nr2 = pack2(-r, -r);
  d.s2 = pack2(s, s);
  return d;
}

// Eight E2M1 codes in one word, x0 in bits 0..3 (RN, satfinite).
__device__ __forceinline__ uint32_t e2m1x8(float x0, float x1, float x2, float x3, float x4, float x5, float x6,
                                           float x7) {
  uint32_t r;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
  return r;
}

// Two quotients of values given negated (nx = (-x0, -x1)), by the packed form of Markstein's
// correction with both signs flipped (round to nearest is symmetric): q = RN(-x * -r),
// t = RN(q * s - x), q' = RN(t * -r + q). A zero x keeps its sign (x = -0: q = -0, t = +0,
// q' = -0).
__device__ __forceinline__ uint64_t nv_quot2_fast(uint64_t nx, const NvDivider &d) {
  const uint64_t q = fmul2(nx, d.nr2);
  return ffma2(ffma2(q, d.s2, nx), d.nr2, q);
}

// Eight codes from four negated pairs on the fast path.
__device__ __forceinline__ uint32_t nv_codes8_fast(uint64_t n0, uint64_t n1, uint64_t n2, uint64_t n3,
                                                   const NvDivider &d) {
  float a[8];
  unpack2(nv_quot2_fast(n0, d), a[0], a[1]);
  unpack2(nv_quot2_fast(n1, d), a[2], a[3]);
  unpack2(nv_quot2_fast(n2, d), a[4], a[5]);
  unpack2(nv_quot2_fast(n3, d), a[6], a[7]);
  return e2m1x8(a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7]);
}

// Codes by IEEE division for 0 < S < 2^-90 (out of line: only tensors far below the normal
// range meet it). Eight values held as the low (hi = false) or high halves of the words
// w[0..7] when `pairs` is false, or as both halves of w[0..3] when `pairs` is true.
__device__ __noinline__ uint32_t nv_codes8_exact(uint4 a, uint4 b, bool pairs, bool hi, float S) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    x[i] = pairs ? ((i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1])) : (hi ? bf16_hi(w[i]) : bf16_lo(w[i]));
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __fdiv_rn(x[i], S);
  return e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
}

// A 16-element group held in two 16-byte words (element 2i in the low half of word i): its
// factor byte, and its eight bytes of codes in out0 (elements 0..7) and out1.
template <bool ALL_FAST = false>
__device__ __forceinline__ uint32_t nv_row_group(const uint4 &v0, const uint4 &v1, const NvTensor &t, uint32_t &out0,
                                                 uint32_t &out1) {
  uint32_t m = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(v0.x, v0.y), bf16x2_absmax(v0.z, v0.w)),
                             bf16x2_absmax(bf16x2_absmax(v1.x, v1.y), bf16x2_absmax(v1.z, v1.w)));
  m &= 0x7FFF7FFFu;
  m = max(m & 0xFFFFu, m >> 16);
  float S;
  const uint32_t e = nv_factor<ALL_FAST>(__uint_as_float(m << 16), t, S);
  const NvDivider d = nv_divider<ALL_FAST>(S);
  if (ALL_FAST || d.fast) {
    out0 = nv_codes8_fast(pack2(neg_bf16_lo(v0.x), neg_bf16_hi(v0.x)), pack2(neg_bf16_lo(v0.y), neg_bf16_hi(v0.y)),
                          pack2(neg_bf16_lo(v0.z), neg_bf16_hi(v0.z)), pack2(neg_bf16_lo(v0.w), neg_bf16_hi(v0.w)), d);
    out1 = nv_codes8_fast(pack2(neg_bf16_lo(v1.x), neg_bf16_hi(v1.x)), pack2(neg_bf16_lo(v1.y), neg_bf16_hi(v1.y)),
                          pack2(neg_bf16_lo(v1.z), neg_bf16_hi(v1.z)), pack2(neg_bf16_lo(v1.w), neg_bf16_hi(v1.w)), d);
  } else {
    out0 = nv_codes8_exact(v0, make_uint4(0, 0, 0, 0), true, false, S);
    out1 = nv_codes8_exact(v1, make_uint4(0, 0, 0, 0), true, false, S);
  }
  return e;
}

// The per-half magnitude maximum of 16 words (both columns of a column pair at once).
__device__ __forceinline__ uint32_t nv_absmax16(const uint32_t *w) {
  uint32_t m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = bf16x2_absmax(w[2 * i], w[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = bf16x2_absmax(m[i], m[i + 4]);
  return bf16x2_absmax(bf16x2_absmax(m[0], m[1]), bf16x2_absmax(m[2], m[3])) & 0x7FFF7FFFu;
}

// A 16-element group down one column: w[i] holds row i of two adjacent columns (the left one
// in the low half), HI picks the right one; `m2` is nv_absmax16(w). Returns the factor byte;
// codes in out0/out1.
template <bool HI, bool ALL_FAST = false>
__device__ __forceinline__ uint32_t nv_col_group(const uint32_t *w, uint32_t m2, const NvTensor &t, uint32_t &out0,
                                                 uint32_t &out1) {
  const uint32_t m = HI ? (m2 >> 16) : (m2 & 0xFFFFu);
  float S;
  const uint32_t e = nv_factor<ALL_FAST>(__uint_as_float(m << 16), t, S);
  const NvDivider d = nv_divider<ALL_FAST>(S);
  if (ALL_FAST || d.fast) {
    uint64_t n[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      n[i] = HI ? pack2(neg_bf16_hi(w[2 * i]), neg_bf16_hi(w[2 * i + 1]))
                : pack2(neg_bf16_lo(w[2 * i]), neg_bf16_lo(w[2 * i + 1]));
    out0 = nv_codes8_fast(n[0], n[1], n[2], n[3], d);
    out1 = nv_codes8_fast(n[4], n[5], n[6], n[7], d);
  } else {
    out0 = nv_codes8_exact(make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]), false, HI, S);
    out1 = nv_codes8_exact(make_uint4(w[8], w[9], w[10], w[11]), make_uint4(w[12], w[13], w[14], w[15]), false, HI,
                           S);
  }
  return e;
}

}  // namespace puro
