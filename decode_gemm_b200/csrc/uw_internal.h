// Internal declarations shared by the host encoder, the C ABI and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "unweight.h"

namespace uw {

constexpr int kRow = 64;            // weights per escape row
constexpr int kEscGroupRows = 128;  // rows per escape-row group (one GEMM row tile)
constexpr int kLutBits = 12;        // decode-table index width (= largest code length)
constexpr int kLutSize = 1 << kLutBits;

// Decode-table entry (one u32 per 12-bit window of the stream):
//   bits  0..23  decoded values, first one in the lowest bits
//                (exponent table: 8-bit exponents, up to 3;
//                 palette table: 4-bit palette indices, up to 6)
//   bits 24..26  number of values decoded from this window (0 = invalid code)
//   bits 28..31  number of stream bits those values consume
constexpr int kExpCap = 3;
constexpr int kPalCap = 6;

struct DecodeTables {
  std::vector<uint32_t> exp_lut;   // kLutSize entries
  std::vector<uint32_t> pal_lut;   // kLutSize entries
  // limit[l] (l = 1..12): first 12-bit window value whose first code is longer
  // than l; a window's first code length is the least l with window < limit[l].
  uint32_t limit[16];
};

// Build the decode tables for canonical codes with the given lengths.
// Returns false when the lengths are not a valid prefix code.
bool build_decode_tables(const uint8_t code_len[256], const uint8_t palette[16],
                         DecodeTables* out);

// Host encoder outputs (owned vectors).
struct HostEncoded {
  int64_t N = 0, K = 0;
  int32_t max_code_len = 12, chunk_syms = 1024;
  uint8_t code_len[256] = {0};
  uint8_t palette[16] = {0};
  std::vector<uint32_t> words, chunk_off, esc_bits, esc_off;
  std::vector<uint8_t> sm, esc_exp;
  std::vector<int64_t> hist;  // 256
  uint64_t total_bits = 0;
};

uw_status encode_host(const uint16_t* w, int64_t N, int64_t K, const uw_encode_opts& o,
                      HostEncoded* out);
void package_merge(const int64_t freq[256], int max_len, uint8_t lengths[256]);
void canonical_codes(const uint8_t lengths[256], uint32_t codes[256]);
void fill_stats(const uw_format& f, const int64_t* hist, uw_stats_t* s);

}  // namespace uw

struct uw_host_s {
  uw::HostEncoded enc;
};
