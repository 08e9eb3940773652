// BF16 field merge and 4-bit palette lookup shared by the library's kernels.
#pragma once

#include <cstdint>

namespace uw {

// Four sign+mantissa bytes (s) and four exponent bytes (e) -> four BF16 values:
// bf16 = sign << 15 | exponent << 7 | mantissa, with s = sign << 7 | mantissa.
__device__ __forceinline__ uint2 merge4(uint32_t s, uint32_t e) {
  const uint32_t hi = (s & 0x80808080u) | ((e >> 1) & 0x7F7F7F7Fu);  // sign | E[7:1]
  const uint32_t lo = ((e << 7) & 0x80808080u) | (s & 0x7F7F7F7Fu);  // E[0] | mantissa
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

// Exponent bytes of four 4-bit palette indices (nibble i of v16 -> byte i);
// p0..p3 hold palette entries 0..15 in byte order.
__device__ __forceinline__ uint32_t palette4(uint32_t v16, uint32_t p0, uint32_t p1, uint32_t p2,
                                             uint32_t p3) {
  const uint32_t sel = v16 & 0x7777u;          // index mod 8 per nibble
  const uint32_t lo = __byte_perm(p0, p1, sel);  // entries 0..7
  const uint32_t hi = __byte_perm(p2, p3, sel);  // entries 8..15
  const uint32_t pick = ((v16 >> 1) & 0x4444u) | 0x3210u;  // byte i of lo or of hi
  return __byte_perm(lo, hi, pick);
}

// Exponent bytes of eight 4-bit palette indices (nibble i of v -> byte i of
// the pair, low word first).
__device__ __forceinline__ uint2 palette8(uint32_t v, uint32_t p0, uint32_t p1, uint32_t p2,
                                          uint32_t p3) {
  const uint32_t sel = v & 0x77777777u;                        // index mod 8 per nibble
  const uint32_t pick = ((v >> 1) & 0x44444444u) | 0x32103210u;  // byte of lo or of hi
  const uint32_t lo0 = __byte_perm(p0, p1, sel), hi0 = __byte_perm(p2, p3, sel);
  const uint32_t lo1 = __byte_perm(p0, p1, sel >> 16), hi1 = __byte_perm(p2, p3, sel >> 16);
  return make_uint2(__byte_perm(lo0, hi0, pick), __byte_perm(lo1, hi1, pick >> 16));
}

}  // namespace uw
