// Distribution bundle: one encoded matrix in a file.
//
// *Unweight* (format vs execution, untitled passage): the Huffman package is what is
// distributed; at load it is transcoded to the form inference runs on.  uw_host_save
// writes a host encoding to a file, uw_host_load reads it back (validated and
// checksummed), uw_load reads and uploads it (with the load-time palette transcode
// of pipeline 4 when opts->prepare_direct is set).
//
// File layout (little-endian), all sections starting at 16-byte offsets:
//   header     Header (below, 2416 bytes)
//   words      u32 [n_words]
//   chunk_off  u32 [n_chunk_off]
//   sm         u8  [n_sm]
//   esc_bits   u32 [n_esc_bits]
//   esc_off    u32 [n_esc_off]
//   esc_exp    u8  [n_esc_exp]
//   trailer    u64 FNV-1a (64-bit) of every byte before it, then the end tag
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "handle.h"
#include "uw_internal.h"

namespace {

constexpr char kMagic[8] = {'U', 'W', 'B', 'U', 'N', 'D', 'L', 'E'};
constexpr char kEndTag[8] = {'U', 'W', 'B', 'E', 'N', 'D', '0', '1'};
constexpr uint32_t kVersion = 1;

struct Header {
  char magic[8];
  uint32_t version, header_bytes;
  int64_t N, K;
  int32_t max_code_len, chunk_syms;
  uint8_t code_len[256];
  uint8_t palette[16];
  uint64_t total_bits;
  int64_t hist[256];  // exponent histogram (for uw_host_stats after a load)
  int64_t n_words, n_chunk_off, n_sm, n_esc_bits, n_esc_off, n_esc_exp;
};
static_assert(sizeof(Header) % 16 == 0, "sections start at 16-byte offsets");

uint64_t fnv1a(uint64_t h, const void* p, size_t n) {
  const uint8_t* b = static_cast<const uint8_t*>(p);
  for (size_t i = 0; i < n; ++i) {
    h ^= b[i];
    h *= 1099511628211ull;
  }
  return h;
}
constexpr uint64_t kFnvBasis = 14695981039346656037ull;

size_t pad16(size_t n) { return (16 - n % 16) % 16; }

struct Writer {
  FILE* f;
  uint64_t h = kFnvBasis;
  bool ok = true;
  void put(const void* p, size_t n) {
    if (!ok || n == 0) return;
    h = fnv1a(h, p, n);
    ok = std::fwrite(p, 1, n, f) == n;
  }
  size_t pos = 0;
  void section(const void* p, size_t n) {
    put(p, n);
    pos += n;
    const size_t z = pad16(pos);
    static const uint8_t zeros[16] = {0};
    put(zeros, z);
    pos += z;
  }
};

struct Reader {
  const std::vector<uint8_t>& buf;
  size_t pos = 0;
  bool take(void* dst, size_t n) {
    if (n > buf.size() - pos) return false;
    std::memcpy(dst, buf.data() + pos, n);
    pos += n;
    pos += pad16(pos);
    return pos <= buf.size();
  }
};

}  // namespace

uw_status uw_host_save(uw_host_t h, const char* path) {
  if (!h || !path) return UW_ERR_ARG;
  const uw::HostEncoded& e = h->enc;
  Header hd;
  std::memset(&hd, 0, sizeof(hd));
  std::memcpy(hd.magic, kMagic, 8);
  hd.version = kVersion;
  hd.header_bytes = (uint32_t)sizeof(Header);
  hd.N = e.N;
  hd.K = e.K;
  hd.max_code_len = e.max_code_len;
  hd.chunk_syms = e.chunk_syms;
  std::memcpy(hd.code_len, e.code_len, 256);
  std::memcpy(hd.palette, e.palette, 16);
  hd.total_bits = e.total_bits;
  for (int s = 0; s < 256 && s < (int)e.hist.size(); ++s) hd.hist[s] = e.hist[s];
  hd.n_words = (int64_t)e.words.size();
  hd.n_chunk_off = (int64_t)e.chunk_off.size();
  hd.n_sm = (int64_t)e.sm.size();
  hd.n_esc_bits = (int64_t)e.esc_bits.size();
  hd.n_esc_off = (int64_t)e.esc_off.size();
  hd.n_esc_exp = (int64_t)e.esc_exp.size();
  FILE* f = std::fopen(path, "wb");
  if (!f) return UW_ERR_IO;
  Writer w{f};
  w.section(&hd, sizeof(hd));
  w.section(e.words.data(), e.words.size() * 4);
  w.section(e.chunk_off.data(), e.chunk_off.size() * 4);
  w.section(e.sm.data(), e.sm.size());
  w.section(e.esc_bits.data(), e.esc_bits.size() * 4);
  w.section(e.esc_off.data(), e.esc_off.size() * 4);
  w.section(e.esc_exp.data(), e.esc_exp.size());
  const uint64_t sum = w.h;
  bool ok = w.ok && std::fwrite(&sum, 1, 8, f) == 8 && std::fwrite(kEndTag, 1, 8, f) == 8;
  ok = (std::fclose(f) == 0) && ok;
  return ok ? UW_OK : UW_ERR_IO;
}

uw_status uw_host_load(const char* path, uw_host_t* out) {
  if (!path || !out) return UW_ERR_ARG;
  *out = nullptr;
  FILE* f = std::fopen(path, "rb");
  if (!f) return UW_ERR_IO;
  std::vector<uint8_t> buf;
  uw_status st = UW_OK;
  try {
    uint8_t chunk[1 << 16];
    size_t n;
    while ((n = std::fread(chunk, 1, sizeof(chunk), f)) > 0) buf.insert(buf.end(), chunk, chunk + n);
    if (std::ferror(f)) st = UW_ERR_IO;
  } catch (const std::bad_alloc&) {
    st = UW_ERR_OOM;
  }
  std::fclose(f);
  if (st != UW_OK) return st;
  // trailer: checksum of everything before it, then the end tag
  if (buf.size() < sizeof(Header) + 16) return UW_ERR_FORMAT;
  const size_t body = buf.size() - 16;
  uint64_t sum;
  std::memcpy(&sum, buf.data() + body, 8);
  if (std::memcmp(buf.data() + body + 8, kEndTag, 8) != 0) return UW_ERR_FORMAT;
  if (fnv1a(kFnvBasis, buf.data(), body) != sum) return UW_ERR_FORMAT;
  Header hd;
  std::memcpy(&hd, buf.data(), sizeof(hd));
  if (std::memcmp(hd.magic, kMagic, 8) != 0 || hd.version != kVersion ||
      hd.header_bytes != sizeof(Header))
    return UW_ERR_FORMAT;
  const int64_t counts[6] = {hd.n_words, hd.n_chunk_off, hd.n_sm,
                             hd.n_esc_bits, hd.n_esc_off, hd.n_esc_exp};
  for (int64_t c : counts)
    if (c < 0 || c > (int64_t)body) return UW_ERR_FORMAT;
  uw_host_s* h = new (std::nothrow) uw_host_s;
  if (!h) return UW_ERR_OOM;
  uw::HostEncoded& e = h->enc;
  e.N = hd.N;
  e.K = hd.K;
  e.max_code_len = hd.max_code_len;
  e.chunk_syms = hd.chunk_syms;
  std::memcpy(e.code_len, hd.code_len, 256);
  std::memcpy(e.palette, hd.palette, 16);
  e.total_bits = hd.total_bits;
  Reader r{buf, sizeof(Header) + pad16(sizeof(Header))};
  bool ok = true;
  try {
    e.hist.assign(hd.hist, hd.hist + 256);
    e.words.resize((size_t)hd.n_words);
    e.chunk_off.resize((size_t)hd.n_chunk_off);
    e.sm.resize((size_t)hd.n_sm);
    e.esc_bits.resize((size_t)hd.n_esc_bits);
    e.esc_off.resize((size_t)hd.n_esc_off);
    e.esc_exp.resize((size_t)hd.n_esc_exp);
    ok = r.take(e.words.data(), e.words.size() * 4) &&
         r.take(e.chunk_off.data(), e.chunk_off.size() * 4) &&
         r.take(e.sm.data(), e.sm.size()) && r.take(e.esc_bits.data(), e.esc_bits.size() * 4) &&
         r.take(e.esc_off.data(), e.esc_off.size() * 4) &&
         r.take(e.esc_exp.data(), e.esc_exp.size()) && r.pos == body;
  } catch (const std::bad_alloc&) {
    delete h;
    return UW_ERR_OOM;
  }
  if (!ok) {
    delete h;
    return UW_ERR_FORMAT;
  }
  // the arrays must describe one encoded matrix, as an upload would check
  uw_format v;
  uw_host_view(h, &v);
  st = uw_validate_format(&v);
  if (st == UW_OK && (int64_t)e.sm.size() != e.N * e.K) st = UW_ERR_FORMAT;
  // the stored histogram (statistics only) must count the N*K exponents, every
  // counted exponent having a code
  if (st == UW_OK) {
    int64_t total = 0;
    for (int s = 0; s < 256 && st == UW_OK; ++s) {
      const int64_t c = e.hist[s];
      if (c < 0 || c > e.N * e.K || (c > 0 && e.code_len[s] == 0)) st = UW_ERR_FORMAT;
      total += c;
    }
    if (st == UW_OK && total != e.N * e.K) st = UW_ERR_FORMAT;
  }
  if (st != UW_OK) {
    delete h;
    return st;
  }
  *out = h;
  return UW_OK;
}

uw_status uw_load(const char* path, const uw_encode_opts* opts, void* stream, uw_handle_t* out) {
  if (!out) return UW_ERR_ARG;
  *out = nullptr;
  uw_host_t hh = nullptr;
  uw_status st = uw_host_load(path, &hh);
  if (st != UW_OK) return st;
  uw_format f;
  uw_host_view(hh, &f);
  st = uw_upload(&f, opts, stream, out);
  if (st == UW_OK) (*out)->hist = hh->enc.hist;  // (statistics after the load)
  uw_host_free(hh);
  return st;
}
