// Test helper (host only): prints the decode tables the library builds for a
// code-length vector and a palette, so the CPU tests can check every entry
// against the canonical code.  Input on stdin: 256 code lengths, then the 16
// palette values.  Output: 1 or 0 (tables built), then the kLutSize entries,
// then the kCanonWords words of the canonical tables, one number per line.
#include <cstdio>

#include "uw_internal.h"

int main() {
  uint8_t len[256], pal[16];
  for (int i = 0; i < 256; ++i) {
    unsigned v = 0;
    if (std::scanf("%u", &v) != 1) return 2;
    len[i] = (uint8_t)v;
  }
  for (int i = 0; i < 16; ++i) {
    unsigned v = 0;
    if (std::scanf("%u", &v) != 1) return 2;
    pal[i] = (uint8_t)v;
  }
  uw::DecodeTables t;
  const bool ok = uw::build_decode_tables(len, pal, &t);
  std::printf("%d\n", ok ? 1 : 0);
  if (!ok) return 0;
  for (int i = 0; i < uw::kLutSize; ++i) std::printf("%u\n", t.lut[i]);
  for (int i = 0; i < uw::kCanonWords; ++i) std::printf("%u\n", t.canon[i]);
  return 0;
}
