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
// Largest stream: the kernels count the stream's bits, padding words included, in 32 bits
constexpr int64_t kMaxStreamWords = (int64_t(1) << 27) - 4;

// Decode-table entry (one u32 per 12-bit window of the stream).  The table
// decodes to 4-bit palette ranks; all three preprocessing outputs derive from
// them (exponent = palette[rank]).
//   bits  0..3   stream bits the entry consumes (1..12)
//   bits  4..8   4 x the number of ranks it yields (4..4*kPalCap)
//   bit   9      special: the window starts with the code of an exponent outside
//                the palette ("raw"), or with no code at all (bit 10 set too);
//                the entry then yields a single rank 0 placeholder and consumes
//                the raw code's length (1 bit for a window with no code)
//   bit   10     no code starts the window (corrupt stream)
//   bits 12..31  the ranks of the codes that fit in the window, first one
//                lowest, at most kPalCap of them, stopping before any exponent
//                that is not in the palette
constexpr int kPalCap = 5;
constexpr uint32_t kLutSpecial = 1u << 9;
constexpr uint32_t kLutInvalid = 1u << 10;

// Canonical-code tables for one-symbol-at-a-time decoding (chunk tails, slow
// path): limit[l] = first 12-bit window whose first code is longer than l;
// first[l] = first code of length l; offset[l] = index in `symbols` of the
// first symbol of length l; symbols = exponents ordered by (length, value).
constexpr int kCanonLimit = 0, kCanonFirst = 16, kCanonOffset = 32, kCanonSymbols = 48;
constexpr int kCanonWords = 48 + 64;

struct DecodeTables {
  std::vector<uint32_t> lut;      // kLutSize entries
  uint32_t canon[kCanonWords];
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
