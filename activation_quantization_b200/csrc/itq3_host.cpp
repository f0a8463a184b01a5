// Host-side ITQ3_S-style weight quantisation: 256-wide Walsh-Hadamard rotation
// followed by a uniform 3-bit code (offline, not on the timed path).
//
// ITQ3_S article, section "核心技术：FWHT预旋转与TurboQuant的完美融合": every
// 256-dimensional weight vector is rotated with the fast Walsh-Hadamard
// transform before the 3-bit quantiser, so that outlier energy is spread over
// the vector.  Per block (256 consecutive d_in weights of one row), in fp64:
//   r = H_256 w / 16 (butterflies, exact for fp16 inputs),
//   s = fp16 RNE(max|r| / 3.5),  c = clamp(rint(r / s + 3.5), 0, 7), c = 0 if s = 0.
// Codes are packed 3 bits each, little-endian, element e of a block at bits
// 3e .. 3e + 2 of the block's 96 bytes (see itq3_quantize_weights in wush.h).
#include <cmath>
#include <cstdint>
#include <cstring>

#include "wush.h"

namespace {

float half_bits_to_float(uint16_t h) {
  const uint32_t sign = (h >> 15) & 1u, exp = (h >> 10) & 0x1Fu, man = h & 0x3FFu;
  double v;
  if (exp == 0) v = std::ldexp(static_cast<double>(man), -24);
  else if (exp == 31) v = man ? NAN : INFINITY;
  else v = std::ldexp(static_cast<double>(man | 0x400u), static_cast<int>(exp) - 25);
  return static_cast<float>(sign ? -v : v);
}

// fp64 -> fp16 bits, one rounding (nearest, ties to even).  Returns false on overflow.
bool double_to_half_rne(double v, uint16_t* out) {
  const uint16_t sign = std::signbit(v) ? 0x8000u : 0u;
  const double a = std::fabs(v);
  if (a == 0.0) { *out = sign; return true; }
  if (!(a < 65520.0)) return false;                // 65504 + half an ulp rounds to inf
  int e;
  std::frexp(a, &e);                                // a = m 2^e, m in [0.5, 1)
  if (e - 1 >= -14) {                               // normal range
    double r = std::nearbyint(std::ldexp(a, 11 - e));   // significand scaled to [1024, 2048)
    int ee = e - 1;
    if (r >= 2048.0) { r = 1024.0; ++ee; }
    if (ee > 15) return false;
    *out = static_cast<uint16_t>(sign | ((ee + 15) << 10) | (static_cast<uint32_t>(r) - 1024u));
    return true;
  }
  const double r = std::nearbyint(std::ldexp(a, 24));   // subnormal units of 2^-24
  *out = static_cast<uint16_t>(sign | static_cast<uint32_t>(r));  // 1024 becomes the min normal
  return true;
}

void fwht256(double* x) {
  for (int h = 1; h < 256; h <<= 1)
    for (int i = 0; i < 256; i += 2 * h)
      for (int k = i; k < i + h; ++k) {
        const double a = x[k], b = x[k + h];
        x[k] = a + b;
        x[k + h] = a - b;
      }
}

}  // namespace

extern "C" int itq3_quantize_weights(const uint16_t* w_fp16, int64_t d_out, int64_t d_in, uint8_t* codes,
                                     uint16_t* scales_fp16) {
  if (!w_fp16 || !codes || !scales_fp16 || d_out <= 0 || d_in <= 0 || d_in % 256) return WUSH_ERR_INVALID_ARG;
  // an fp16 with all exponent bits set is an infinity or NaN: no scale exists for its block
  bool finite = true;
#pragma omp parallel for reduction(&& : finite) schedule(static)
  for (int64_t i = 0; i < d_out * d_in; ++i) finite = finite && (w_fp16[i] & 0x7C00u) != 0x7C00u;
  if (!finite) return WUSH_ERR_INVALID_ARG;
  const int64_t nb = d_in / 256;
  int status = WUSH_OK;
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < d_out; ++o) {
    double r[256];
    uint8_t c[256];
    for (int64_t blk = 0; blk < nb; ++blk) {
      const uint16_t* src = w_fp16 + o * d_in + blk * 256;
      for (int i = 0; i < 256; ++i) r[i] = half_bits_to_float(src[i]);
      fwht256(r);
      double amax = 0.0;
      for (int i = 0; i < 256; ++i) {
        r[i] /= 16.0;
        amax = std::fmax(amax, std::fabs(r[i]));
      }
      uint16_t sbits;
      if (!double_to_half_rne(amax / 3.5, &sbits)) {
#pragma omp critical
        status = WUSH_ERR_INVALID_ARG;
        sbits = 0;
      }
      const double s = half_bits_to_float(sbits);
      for (int i = 0; i < 256; ++i) {
        if (s == 0.0) { c[i] = 0; continue; }
        double q = std::nearbyint(r[i] / s + 3.5);
        q = q < 0.0 ? 0.0 : (q > 7.0 ? 7.0 : q);
        c[i] = static_cast<uint8_t>(q);
      }
      scales_fp16[o * nb + blk] = sbits;
      uint8_t packed[96];
      std::memset(packed, 0, sizeof(packed));
      for (int i = 0; i < 256; ++i)
        for (int p = 0; p < 3; ++p)
          if ((c[i] >> p) & 1) {
            const int bit = 3 * i + p;
            packed[bit >> 3] |= static_cast<uint8_t>(1u << (bit & 7));
          }
      std::memcpy(codes + (o * nb + blk) * 96, packed, sizeof(packed));
    }
  }
  return status;
}
