// Host stand-in for the bf16 types the decode kernels use (CPU emulation
// only): storage as the upper 16 bits of an IEEE float, conversion to float
// by a shift, and from float by round-to-nearest-even on the bit pattern
// (NaN kept quiet).
#pragma once

#include <cstdint>
#include <cstring>

struct alignas(2) __nv_bfloat16 {
  uint16_t bits;
};
struct alignas(4) __nv_bfloat162 {
  __nv_bfloat16 x, y;
};

inline float __bfloat162float(__nv_bfloat16 h) {
  const uint32_t u = static_cast<uint32_t>(h.bits) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

inline float2 __bfloat1622float2(__nv_bfloat162 h) {
  return float2{__bfloat162float(h.x), __bfloat162float(h.y)};
}

inline __nv_bfloat16 __float2bfloat16_rn(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
    return __nv_bfloat16{static_cast<uint16_t>((u >> 16) | 0x0040u)};
  const uint32_t round = 0x7fffu + ((u >> 16) & 1u);
  return __nv_bfloat16{static_cast<uint16_t>((u + round) >> 16)};
}
