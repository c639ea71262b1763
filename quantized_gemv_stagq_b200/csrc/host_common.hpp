// Host-side helpers shared by the encoder, the packer and the API.
#pragma once
#include <cmath>
#include <cstdint>
#include <cstring>
#include <string>

#include "stagq.h"

namespace stagq {

// Thread-local detail message for stagq_last_error().
void set_error(const std::string& msg);

inline int fail(int status, const std::string& msg) {
  set_error(msg);
  return status;
}

// IEEE binary16 -> binary64 (exact).
inline double half_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int exp = (h >> 10) & 31;
  const int man = h & 1023;
  double v;
  if (exp == 0) {
    v = std::ldexp((double)man, -24);
  } else if (exp == 31) {
    v = man ? NAN : INFINITY;
  } else {
    v = std::ldexp((double)(man | 1024), exp - 25);
  }
  return sign ? -v : v;
}

// binary64 -> binary16, round to nearest even, directly from the double
// (no intermediate float rounding).
inline uint16_t double_to_half(double d) {
  uint16_t sign = std::signbit(d) ? 0x8000 : 0;
  if (std::isnan(d)) return sign | 0x7E00;
  const double a = std::fabs(d);
  if (a >= 65520.0) return sign | 0x7C00;
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);                 // a in [2^(ex-1), 2^ex)
  const int E = ex - 1;
  const int qexp = (E < -14) ? -24 : E - 10;  // exponent of one unit in the last place
  const double r = std::nearbyint(std::ldexp(a, -qexp));  // exact scaling, then RNE
  if (E < -14) return sign | (uint16_t)r;    // subnormal (r == 1024 becomes the smallest normal)
  return sign | (uint16_t)(((E + 15) << 10) + ((int)r - 1024));
}

}  // namespace stagq
