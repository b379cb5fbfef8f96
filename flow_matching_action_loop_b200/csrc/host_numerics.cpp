// Host number-format utilities of the weight packer (no GPU involved).
//
// bf16: the top half of a float32, rounded to nearest even.
// e4m3: the OCP 8-bit floating point "E4M3" format (exponent bias 7, three
// fraction bits, subnormal quantum 2^-9, largest finite 448, no infinities,
// NaN = S.1111.111); quantisation saturates to +-448 and rounds to nearest even.
// RoPE tables: rotate-half pairing, frequency theta^(-2j/dh) (FlashRT
// walkthrough, component 8: QKV split + RoPE is one of the hand-written ops).
// 4-bit group weights (PhyAI page, optimisation paragraph: W4A16): per row, groups of
// 128 consecutive inputs share one bf16 scale s = bf16(max|w| / 7); codes are
// round-half-even(w / s) clamped to [-7, 7].
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "fr.h"

namespace {

inline uint16_t bf16_bits_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) {
    return static_cast<uint16_t>((u >> 16) | 0x0040u);   // quiet NaN, sign kept
  }
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

inline uint8_t e4m3_code(double x) {
  if (std::isnan(x)) return 0x7F;
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double ax = std::fabs(x);
  if (ax > 448.0) ax = 448.0;
  if (ax < 0.015625) {                               // below 2^-6: subnormal grid 2^-9
    const double q = std::nearbyint(ax * 512.0);     // 0..8; 8 is the smallest normal
    return static_cast<uint8_t>(sign | static_cast<uint8_t>(q));
  }
  int e2 = 0;
  std::frexp(ax, &e2);                               // ax in [2^(e2-1), 2^e2)
  int lead = e2 - 1;
  double q = std::nearbyint(std::ldexp(ax, 3 - lead));   // 8..16
  if (q >= 16.0) { q = 8.0; ++lead; }
  const int code = ((lead + 7) << 3) | (static_cast<int>(q) - 8);
  return static_cast<uint8_t>(sign | code);
}

// double -> bf16 bits with one rounding (nearest even) from the double itself; finite values in
// the bf16 normal range (weight scales), zero kept exact.
inline uint16_t bf16_bits_rne_double(double x) {
  const uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
  if (x == 0.0) return sign;
  int e = 0;
  const double m = std::frexp(std::fabs(x), &e);   // |x| = m * 2^e, m in [0.5, 1)
  double q = std::nearbyint(std::ldexp(m, 8));     // 128..256, ties to even
  if (q == 256.0) {
    q = 128.0;
    ++e;
  }
  // |x| ~ q * 2^(e - 8) = (q / 128) * 2^(e - 1): biased exponent e - 1 + 127, 7 fraction bits q - 128
  return static_cast<uint16_t>(sign | (static_cast<uint32_t>(e + 126) << 7) | (static_cast<uint32_t>(q) - 128u));
}

inline double bf16_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

}  // namespace

extern "C" {

int fr_quantize_w4(const float* w, int rows, int cols, int8_t* q, uint16_t* scale_bits) {
  if (!w || !q || !scale_bits || rows < 0 || cols < 0) return FR_ERR_ARG;
  const int ng = (cols + FR_W4_GROUP - 1) / FR_W4_GROUP;
  for (int r = 0; r < rows; ++r) {
    const float* wr = w + static_cast<size_t>(r) * cols;
    int8_t* qr = q + static_cast<size_t>(r) * cols;
    for (int g = 0; g < ng; ++g) {
      const int c0 = g * FR_W4_GROUP, c1 = std::min(cols, c0 + FR_W4_GROUP);
      double amax = 0.0;
      for (int c = c0; c < c1; ++c) amax = std::max(amax, std::fabs(static_cast<double>(wr[c])));
      const uint16_t sb = bf16_bits_rne_double(amax / 7.0);
      scale_bits[static_cast<size_t>(r) * ng + g] = sb;
      const double sv = bf16_value(sb);
      for (int c = c0; c < c1; ++c) {
        double v = sv > 0.0 ? std::nearbyint(static_cast<double>(wr[c]) / sv) : 0.0;
        v = std::min(7.0, std::max(-7.0, v));
        qr[c] = static_cast<int8_t>(v);
      }
    }
  }
  return FR_OK;
}

int fr_rope_tables(int n_pos, int dh, double theta, float* cos_out, float* sin_out) {
  if (n_pos < 0 || dh <= 0 || (dh & 1) || !cos_out || !sin_out) return FR_ERR_ARG;
  const int half = dh / 2;
  for (int j = 0; j < half; ++j) {
    const double inv = std::pow(theta, -2.0 * j / dh);
    for (int p = 0; p < n_pos; ++p) {
      const double a = p * inv;
      cos_out[static_cast<size_t>(p) * half + j] = static_cast<float>(std::cos(a));
      sin_out[static_cast<size_t>(p) * half + j] = static_cast<float>(std::sin(a));
    }
  }
  return FR_OK;
}

void fr_round_bf16(const float* in, uint16_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = bf16_bits_rne(in[i]);
}

void fr_quantize_e4m3(const float* in, uint8_t* out, size_t n, double scale) {
  for (size_t i = 0; i < n; ++i) out[i] = e4m3_code(static_cast<double>(in[i]) / scale);
}

}  // extern "C"
