// Host number-format utilities of the weight packer (no GPU involved).
//
// bf16: the top half of a float32, rounded to nearest even.
// e4m3: the OCP 8-bit floating point "E4M3" format (exponent bias 7, three
// fraction bits, subnormal quantum 2^-9, largest finite 448, no infinities,
// NaN = S.1111.111); quantisation saturates to +-448 and rounds to nearest even.
// RoPE tables: rotate-half pairing, frequency theta^(-2j/dh) (FlashRT
// walkthrough, component 8: QKV split + RoPE is one of the hand-written ops).
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

}  // namespace

extern "C" {

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
