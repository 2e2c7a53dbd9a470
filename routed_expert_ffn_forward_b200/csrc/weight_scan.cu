// Host-side scan of Q4_K weights at registration: the power-of-two scale of
// each weight row for the fp16 dequantisation of the prefill GEMMs.
//
// A Q4_K weight is d*sc*q - dmin*m with 6-bit sc, m and 4-bit q, so every
// intermediate of its fp16 dequantisation (d*2^k, d*2^k*sc, dmin*2^k*m and
// q*(d*2^k*sc) - dmin*2^k*m) is bounded by 2^k * (|d|*63*15 + |dmin|*63).
// The row's exponent k is the largest k <= 8 for which that bound stays
// below 60000 on every block of the row; the GEMM epilogue multiplies by
// 2^-k, so the scale costs nothing in accuracy.
#include <cmath>
#include <cstring>

#include "moe_internal.h"

namespace moe {
namespace {

// IEEE binary16 bit pattern -> float (exact).
float half_bits_to_float(uint16_t h) {
  const int sign = (h >> 15) & 1, ex = (h >> 10) & 31, man = h & 1023;
  float v;
  if (ex == 0)
    v = std::ldexp((float)man, -24);
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = std::ldexp((float)(man | 1024), ex - 25);
  return sign ? -v : v;
}

constexpr int kMaxExp = 8, kMinExp = -14;
constexpr double kLimit = 60000.0;

}  // namespace

void q4k_row_exponents(const uint8_t* q4k, int rows, int nb, int8_t* out) {
  for (int r = 0; r < rows; ++r) {
    const uint8_t* row = q4k + (size_t)r * nb * kQBytes;
    double bound = 0.0;
    for (int b = 0; b < nb; ++b) {
      uint16_t dh, mh;
      std::memcpy(&dh, row + (size_t)b * kQBytes, 2);
      std::memcpy(&mh, row + (size_t)b * kQBytes + 2, 2);
      const double v = std::fabs((double)half_bits_to_float(dh)) * 945.0 +
                       std::fabs((double)half_bits_to_float(mh)) * 63.0;
      if (!(v <= bound)) bound = v;  // also takes a NaN
    }
    int k = kMaxExp;
    if (!std::isfinite(bound))
      k = kMinExp;  // inf or NaN scales give non-finite outputs on every path
    else
      while (k > kMinExp && std::ldexp(bound, k) >= kLimit) --k;
    out[r] = (int8_t)k;
  }
}

}  // namespace moe
