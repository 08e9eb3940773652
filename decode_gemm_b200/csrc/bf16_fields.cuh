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

// Exponent bytes of eight ranks in element order (nibble t of v = element t)
// for a palette that is the run b..b+15 (b4 = b in every byte): b + rank,
// element order restored by two byte permutes.
__device__ __forceinline__ uint2 run8(uint32_t v, uint32_t b4) {
  const uint32_t ev = (v & 0x0F0F0F0Fu) + b4;         // elements 0 2 4 6
  const uint32_t od = ((v >> 4) & 0x0F0F0F0Fu) + b4;  // elements 1 3 5 7
  return make_uint2(__byte_perm(ev, od, 0x5140), __byte_perm(ev, od, 0x7362));
}

// PTX prmt in its default mode: a selector nibble with bit 3 set fills the
// byte with the sign bit of the byte it selects (the CUDA intrinsic
// __byte_perm ignores that bit).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Packed-index word order.  The decoder's stage holds 8 indices per word in
// element order (nibble t = element t); the stored form interleaves them:
// element 2t at bits 4t, element 2t+1 at bits 16+4t, so each 16-bit half holds
// one index of every BF16 pair, in the pair's own lane.
__device__ __forceinline__ uint32_t nibbles_interleave(uint32_t v) {
  // swap nibbles 1 <-> 2 and 5 <-> 6 (a delta swap): the bytes become
  // (0 2) (1 3) (4 6) (5 7); then bytes 1 and 2 trade places
  const uint32_t t = (v ^ (v >> 4)) & 0x00F000F0u;
  return __byte_perm(v ^ t ^ (t << 4), 0u, 0x3120);
}

// Eight BF16 weights (four pair words, element order) from one interleaved
// index word v and their sign+mantissa bytes (s0: elements 0-3, s1: 4-7),
// for a palette that is the run base..base+15: the exponent is base + index,
// so a pair's exponent fields are (index << 7) + bias, bias = base * 128 in
// both halves.  The sign moves from bit 7 to bit 15 of each half by prmt's
// sign replication.
__device__ __forceinline__ uint4 rebuild8_run(uint32_t v, uint32_t s0, uint32_t s1,
                                              uint32_t bias) {
  const uint32_t m = 0x807F807Fu;  // sign and mantissa bits of a pair
  const uint32_t x0 = (v & 0x000F000Fu) * 128u + bias;
  const uint32_t x1 = (v & 0x00F000F0u) * 8u + bias;
  const uint32_t x2 = __umulhi(v & 0x0F000F00u, 0x80000000u) + bias;  // >> 1
  const uint32_t x3 = __umulhi(v & 0xF000F000u, 0x08000000u) + bias;  // >> 5
  return make_uint4(x0 | (prmt(s0, 0u, 0x9180u) & m), x1 | (prmt(s0, 0u, 0xB3A2u) & m),
                    x2 | (prmt(s1, 0u, 0x9180u) & m), x3 | (prmt(s1, 0u, 0xB3A2u) & m));
}

// The same for any palette (p0..p3: entries 0..15 in byte order): exponents
// by lookup, put back in element order, then merged.
__device__ __forceinline__ uint4 rebuild8_lut(uint32_t v, uint32_t s0, uint32_t s1, uint32_t p0,
                                              uint32_t p1, uint32_t p2, uint32_t p3) {
  const uint2 e = palette8(v, p0, p1, p2, p3);  // exponents of elements 0 2 4 6 | 1 3 5 7
  const uint2 lo = merge4(s0, __byte_perm(e.x, e.y, 0x5140));
  const uint2 hi = merge4(s1, __byte_perm(e.x, e.y, 0x7362));
  return make_uint4(lo.x, lo.y, hi.x, hi.y);
}

}  // namespace uw
