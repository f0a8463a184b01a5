// Exact format decisions for the quantising kernels: block scales and element codes
// that equal the round-to-nearest-even of the exact quotients (amax / (6 s_g),
// y / (s_b s_g), amax / 7, y / s) of the kernel's fp32 values.
//
// The fast path multiplies by a reciprocal, which is within a few fp32 ulps of the
// exact quotient.  Each value is quantised twice, against reciprocals nudged down
// and up by 2^-20 relative, which brackets the exact quotient.  When the two
// results agree (all but values within about 1e-6 relative of a boundary), that is
// the exact decision, since rounding onto a grid is monotone.  Otherwise exactly
// one boundary lies inside the bracket, and an exact comparison of the value
// against that boundary times the scale settles it: the boundary times the scale
// has few significant bits (an FMA gives the sign of the difference exactly when
// the product needs more than 24), and an exact tie goes to the even code.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace wush {

constexpr float kBracketLo = 0.99999904632568359375f;   // 1 - 2^-20
constexpr float kBracketHi = 1.00000095367431640625f;   // 1 + 2^-20

__device__ __forceinline__ float exp2i(int k) {  // exact 2^k for k in [-149, 127]
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

__device__ __forceinline__ int floor_log2(float a) {  // a > 0, finite
  const uint32_t b = __float_as_uint(a);
  const int e = (b >> 23) & 0xFF;
  return e ? e - 127 : (31 - __clz(b & 0x7FFFFFu)) - 149;
}

// E2M1 magnitude of a 3-bit code: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_magnitude(uint32_t c) {
  return c < 4u ? 0.5f * static_cast<float>(c) : static_cast<float>(c == 7u ? 6u : c - 2u);
}

// UE4M3 byte of t >= 0: round to nearest even, saturating at 448 (hardware
// conversion with .satfinite; the sign bit of a non-negative input is 0).
__device__ __forceinline__ uint32_t ue4m3_rn(float t) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(t));
  return h & 0xFFu;
}

// Value of a UE4M3 byte (exact through fp16).
__device__ __forceinline__ float ue4m3_val(uint32_t c) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(c)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// (a, b) * s as one packed f32x2 multiply, each lane rounded to nearest like FMUL.
__device__ __forceinline__ void mul2_rn(float a, float b, float s, float& pa, float& pb) {
  unsigned long long x, y, z;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(y) : "f"(s));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(pa), "=f"(pb) : "l"(z));
}

// Eight values -> eight E2M1 codes, element 0 in the low nibble (RNE, satfinite;
// the sign bit follows the value, also when the magnitude rounds to 0).
__device__ __forceinline__ uint32_t e2m1x8_cvt(const float (&p)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(p[0]), "f"(p[1]), "f"(p[2]), "f"(p[3]), "f"(p[4]), "f"(p[5]), "f"(p[6]), "f"(p[7]));
  return out;
}

// Eight values times s -> eight E2M1 codes (packed multiply, then conversion).
__device__ __forceinline__ uint32_t e2m1x8_times(const float* v, float s) {
  float p[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) mul2_rn(v[i], v[i + 1], s, p[i], p[i + 1]);
  return e2m1x8_cvt(p);
}

// NVFP4 block scale s_b = UE4M3_RNE(amax / (6 s_g)), decided exactly; inv_den is
// fp32(1 / fp32(6 s_g)).
__device__ __forceinline__ uint32_t nvfp4_scale_byte(float amax, float sg, float inv_den) {
  const float t = __fmul_rn(amax, inv_den);          // within 2^-22 of amax / (6 s_g)
  const uint32_t lo = ue4m3_rn(__fmul_rn(t, kBracketLo)), hi = ue4m3_rn(__fmul_rn(t, kBracketHi));
  if (lo == hi) return lo;
  // the UE4M3 midpoint m between the two codes: compare amax with 6 m s_g exactly
  const float m6 = 3.0f * (ue4m3_val(lo) + ue4m3_val(hi));   // 6 m: at most 7 significant bits
  const float e = fmaf(-m6, sg, amax);
  return e > 0.f ? hi : (e < 0.f ? lo : ((lo & 1u) ? hi : lo));
}

// Eight NVFP4 codes of v[0..7] with block scale value sbv and per-tensor scale sg;
// r = fp32(1 / fp32(sbv * sg)).  Exact: equal to E2M1_RNE_sat(v / (sbv sg)).
__device__ __forceinline__ uint32_t nvfp4_codes8(const float* v, float r, float sbv, float sg) {
  const uint32_t a = e2m1x8_times(v, __fmul_rn(r, kBracketLo));
  const uint32_t b = e2m1x8_times(v, __fmul_rn(r, kBracketHi));
  if (a == b) return a;
  uint32_t w = a;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t ca = (a >> (4 * i)) & 15u, cb = (b >> (4 * i)) & 15u;
    if (ca == cb) continue;
    const uint32_t lo = min(ca & 7u, cb & 7u), hi = max(ca & 7u, cb & 7u);
    const float m = 0.5f * (e2m1_magnitude(lo) + e2m1_magnitude(hi));   // at most 3 significant bits
    const float e = fmaf(-(m * sbv), sg, fabsf(v[i]));                  // m * sbv is exact
    const uint32_t mag = e > 0.f ? hi : (e < 0.f ? lo : ((lo & 1u) ? hi : lo));
    const uint32_t c = mag | ((__float_as_uint(v[i]) >> 28) & 8u);
    w = (w & ~(15u << (4 * i))) | (c << (4 * i));
  }
  return w;
}

// INT4 group scale s = fp16_RNE(amax / 7) (saturating at 65504), decided exactly.
__device__ __forceinline__ __half int4_scale(float amax) {
  const float pre = __fmul_rn(amax, 0.142857149243354797363f);   // fp32(1/7); within 2^-23 of amax / 7
  const __half lo = __float2half_rn(fminf(__fmul_rn(pre, kBracketLo), 65504.0f));
  const __half hi = __float2half_rn(fminf(__fmul_rn(pre, kBracketHi), 65504.0f));
  if (__half_as_ushort(lo) == __half_as_ushort(hi)) return lo;
  // the fp16 midpoint m between the two: 7 m has at most 15 significant bits
  const float m7 = 3.5f * (__half2float(lo) + __half2float(hi));
  return amax > m7 ? hi : (amax < m7 ? lo : ((__half_as_ushort(lo) & 1u) ? hi : lo));
}

// RNE(v) of |v| < 2^22 without a float-to-integer conversion: adding 1.5 * 2^23
// rounds to an integer (the ulp there is 1) held in the low mantissa bits, whose
// low four bits are the two's-complement nibble of the result.
__device__ __forceinline__ uint32_t rne_bits(float v) { return __float_as_uint(__fadd_rn(v, 12582912.0f)); }

// Insert the low four bits of src into w at bit position pos.
__device__ __forceinline__ uint32_t put_nibble(uint32_t w, uint32_t src, uint32_t pos) {
  uint32_t out;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(out) : "r"(src), "r"(w), "r"(pos));
  return out;
}

__device__ __forceinline__ int int4_from_nibble(uint32_t n) {
  return static_cast<int>(n << 28) >> 28;
}

// (a0, a1) + (b0, b1) and (a0, a1) * (b0, b1) + (c0, c1) as packed f32x2 operations,
// each lane rounded to nearest like FADD / FFMA.
__device__ __forceinline__ void pk_add(float a0, float a1, float b0, float b1, float& o0, float& o1) {
  unsigned long long x, y, z;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(o0), "=f"(o1) : "l"(z));
}
__device__ __forceinline__ void pk_fma(float a0, float a1, float b0, float b1, float& c0, float& c1) {
  unsigned long long x, y, z;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b0), "f"(b1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(z) : "f"(c0), "f"(c1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(z) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(c0), "=f"(c1) : "l"(z));
}

// Eight INT4 codes (two's-complement nibbles) of v[0..7] with scale s > 0 and
// r = fp32(1 / s).  Exact: equal to clamp(RNE(v / s), -7, 7).
// When s is a normal fp16 below 65504 (s = fp16_RNE(amax / 7) within 2^-11), no
// |v / s| exceeds 7 (1 + 2^-10) < 7.5, so no value needs the clamp.
// Both brackets are rounded with packed adds of 1.5 * 2^23; only the low one is
// packed into nibbles.  The two agree everywhere exactly when the sum of the squared
// differences of their rounded values (each 0 or 1, all exact) is zero.
__device__ __forceinline__ uint32_t int4_codes8(const float* v, float r, float s) {
  constexpr float kBias = 12582912.0f;                         // 1.5 * 2^23
  const float ra = __fmul_rn(r, kBracketLo), rb = __fmul_rn(r, kBracketHi);
  const bool in_range = s >= 6.103515625e-05f && s < 65504.0f;
  uint32_t wa = 0;
  float dd0 = 0.f, dd1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float a0, a1, b0, b1;
    mul2_rn(v[i], v[i + 1], ra, a0, a1);
    mul2_rn(v[i], v[i + 1], rb, b0, b1);
    if (!in_range) {
      a0 = fminf(fmaxf(a0, -7.0f), 7.0f);
      a1 = fminf(fmaxf(a1, -7.0f), 7.0f);
      b0 = fminf(fmaxf(b0, -7.0f), 7.0f);
      b1 = fminf(fmaxf(b1, -7.0f), 7.0f);
    }
    pk_add(a0, a1, kBias, kBias, a0, a1);
    pk_add(b0, b1, kBias, kBias, b0, b1);
    wa = put_nibble(put_nibble(wa, __float_as_uint(a0), 4 * i), __float_as_uint(a1), 4 * i + 4);
    pk_add(b0, b1, -a0, -a1, b0, b1);                           // 0 or +-1, exact
    pk_fma(b0, b1, b0, b1, dd0, dd1);
  }
  if (dd0 + dd1 == 0.f) return wa;
  uint32_t w = wa;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float b = __fmul_rn(v[i], rb);
    if (!in_range) b = fminf(fmaxf(b, -7.0f), 7.0f);
    const int qa = int4_from_nibble((wa >> (4 * i)) & 15u), qb = int4_from_nibble(rne_bits(b) & 15u);
    if (qa == qb) continue;
    const int lo = min(qa, qb), hi = max(qa, qb);
    const float p = (static_cast<float>(lo) + 0.5f) * s;     // at most 15 significant bits: exact
    const int q = v[i] > p ? hi : (v[i] < p ? lo : ((lo & 1) ? hi : lo));
    w = put_nibble(w, static_cast<uint32_t>(q), 4 * i);
  }
  return w;
}

}  // namespace wush
