// Host-side encoder, format validation, decode-table construction and statistics.
//
// Method: *Unweight* (Cloudflare, "Unweight: how we compressed an LLM 22%
// without sacrificing quality"), section "Exponents are surprisingly
// predictable": keep sign+mantissa verbatim, Huffman-code the exponent byte,
// keep a 16-exponent palette, store 64-weight rows with an exponent outside the
// palette verbatim.  Section "Sharing the GPU between decode and compute": the
// decoder's table is ~16 KB (here 2^12 entries of 4 bytes).
//
// Choices where the post is silent (the same ones the test oracle makes, so the
// two encoders must agree byte for byte):
//   * optimal length-limited code lengths by package-merge (Larmore &
//     Hirschberg 1990), leaves ordered by (count, symbol), an item before a
//     package of equal weight, a lone symbol gets length 1;
//   * canonical codes as in RFC 1951 section 3.2.2;
//   * stream = codes of E in row-major order, MSB first, bit p in bit 31-p%32 of
//     32-bit word p/32, zero padded to 16 bytes; chunk c starts at chunk_off[c];
//   * palette = top 16 by (count desc, value asc), padded with the smallest
//     absent byte values, then sorted ascending (a run b..b+15 then has index
//     e - b); escape rows grouped by (n/128, kb);
//   * packed indices: 8 per little-endian 32-bit word, element 2t at bits 4t,
//     element 2t+1 at bits 16+4t (each half-word feeds one lane of a BF16 pair).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <new>
#include <thread>

#include "uw_internal.h"

namespace uw {

// ------------------------------------------------------------ code lengths --

void package_merge(const int64_t freq[256], int max_len, uint8_t lengths[256]) {
  std::memset(lengths, 0, 256);
  struct Entry {
    int64_t w;
    int32_t sym;   // >= 0: leaf; -1: package
    int32_t a, b;  // children (indices into the previous level's list)
  };
  std::vector<Entry> leaves;
  for (int s = 0; s < 256; ++s)
    if (freq[s] > 0) leaves.push_back({freq[s], s, -1, -1});
  const int n = static_cast<int>(leaves.size());
  if (n == 0) return;
  if (n == 1) {
    lengths[leaves[0].sym] = 1;
    return;
  }
  std::stable_sort(leaves.begin(), leaves.end(), [](const Entry& x, const Entry& y) {
    return x.w != y.w ? x.w < y.w : x.sym < y.sym;
  });
  std::vector<std::vector<Entry>> level;
  level.push_back(leaves);
  for (int r = 1; r < max_len; ++r) {
    const std::vector<Entry>& prev = level.back();
    std::vector<Entry> packages;
    for (size_t i = 0; i + 1 < prev.size(); i += 2)
      packages.push_back({prev[i].w + prev[i + 1].w, -1, (int32_t)i, (int32_t)(i + 1)});
    std::vector<Entry> merged;
    merged.reserve(leaves.size() + packages.size());
    size_t i = 0, j = 0;
    while (i < leaves.size() || j < packages.size()) {
      // an item precedes a package of equal weight
      if (j == packages.size() || (i < leaves.size() && leaves[i].w <= packages[j].w))
        merged.push_back(leaves[i++]);
      else
        merged.push_back(packages[j++]);
    }
    level.push_back(std::move(merged));
  }
  // Keep the 2n-2 lightest entries of the last level; each leaf found inside
  // them (recursively through packages) adds one bit to its symbol.
  int counts[256] = {0};
  std::vector<std::pair<int, int>> stack;  // (level, index)
  const int top = static_cast<int>(level.size()) - 1;
  for (int k = 0; k < 2 * n - 2; ++k) stack.push_back({top, k});
  while (!stack.empty()) {
    auto [lv, idx] = stack.back();
    stack.pop_back();
    const Entry& e = level[lv][idx];
    if (e.sym >= 0) {
      counts[e.sym] += 1;
    } else {
      stack.push_back({lv - 1, e.a});
      stack.push_back({lv - 1, e.b});
    }
  }
  for (int s = 0; s < 256; ++s) lengths[s] = static_cast<uint8_t>(counts[s]);
}

void canonical_codes(const uint8_t lengths[256], uint32_t codes[256]) {
  int bl_count[33] = {0};
  for (int s = 0; s < 256; ++s)
    if (lengths[s]) bl_count[lengths[s]]++;
  uint32_t next_code[34] = {0};
  uint32_t code = 0;
  for (int bits = 1; bits <= 32; ++bits) {
    code = (code + bl_count[bits - 1]) << 1;
    next_code[bits] = code;
  }
  for (int s = 0; s < 256; ++s) {
    codes[s] = 0;
    if (lengths[s]) codes[s] = next_code[lengths[s]]++;
  }
}

// ----------------------------------------------------------- decode tables --

bool build_decode_tables(const uint8_t code_len[256], const uint8_t palette[16],
                         DecodeTables* out) {
  uint64_t kraft = 0;
  int nsym = 0;
  for (int s = 0; s < 256; ++s) {
    if (code_len[s] > kLutBits) return false;
    if (code_len[s]) {
      kraft += 1ull << (kLutBits - code_len[s]);
      nsym++;
    }
  }
  if (nsym == 0 || kraft > (uint64_t)kLutSize) return false;
  uint32_t codes[256];
  canonical_codes(code_len, codes);
  // single-code table: which code a 12-bit window starts with
  std::vector<int16_t> first_sym(kLutSize, -1);
  std::vector<uint8_t> first_len(kLutSize, 0);
  for (int s = 0; s < 256; ++s) {
    const int l = code_len[s];
    if (!l) continue;
    const uint32_t lo = codes[s] << (kLutBits - l), hi = (codes[s] + 1) << (kLutBits - l);
    for (uint32_t v = lo; v < hi; ++v) {
      first_sym[v] = (int16_t)s;
      first_len[v] = (uint8_t)l;
    }
  }
  int rank[256];
  for (int v = 0; v < 256; ++v) rank[v] = -1;
  for (int i = 0; i < 16; ++i) rank[palette[i]] = i;
  out->lut.assign(kLutSize, 0);
  for (int v = 0; v < kLutSize; ++v) {
    const int s0 = first_sym[v];
    if (s0 < 0) {  // no code starts this window: one placeholder, one bit
      out->lut[v] = 1u | (4u << 4) | kLutSpecial | kLutInvalid;
      continue;
    }
    if (rank[s0] < 0) {  // an exponent outside the palette: one placeholder
      out->lut[v] = (uint32_t)first_len[v] | (4u << 4) | kLutSpecial;
      continue;
    }
    uint32_t vals = 0, cnt = 0, pos = 0;
    while ((int)cnt < kPalCap && pos < (uint32_t)kLutBits) {
      const uint32_t w = ((uint32_t)v << pos) & (kLutSize - 1);
      const int s = first_sym[w];
      const int l = first_len[w];
      if (s < 0 || rank[s] < 0 || pos + l > (uint32_t)kLutBits) break;
      vals |= (uint32_t)rank[s] << (4 * cnt);
      cnt++;
      pos += l;
    }
    out->lut[v] = pos | ((4 * cnt) << 4) | (vals << 12);
  }
  // canonical tables
  int count[kLutBits + 2] = {0};
  for (int s = 0; s < 256; ++s)
    if (code_len[s]) count[code_len[s]]++;
  uint32_t* lim = out->canon + kCanonLimit;
  uint32_t* fst = out->canon + kCanonFirst;
  uint32_t* ofs = out->canon + kCanonOffset;
  uint8_t* syms = reinterpret_cast<uint8_t*>(out->canon + kCanonSymbols);
  for (int i = 0; i < kCanonWords; ++i) out->canon[i] = 0;
  uint32_t first = 0, index = 0;
  for (int l = 1; l <= kLutBits; ++l) {
    first = (first + (uint32_t)count[l - 1]) << 1;
    fst[l] = first;
    ofs[l] = index;
    index += (uint32_t)count[l];
    lim[l] = (first + (uint32_t)count[l]) << (kLutBits - l);
  }
  for (int l = kLutBits + 1; l < 16; ++l) lim[l] = kLutSize;
  int k = 0;
  for (int l = 1; l <= kLutBits; ++l)
    for (int s = 0; s < 256; ++s)
      if (code_len[s] == l) syms[k++] = (uint8_t)s;
  return true;
}

// ----------------------------------------------------------------- encoder --

namespace {

int worker_count() {
  unsigned hc = std::thread::hardware_concurrency();
  return (int)std::max(1u, std::min(hc, 32u));
}

template <class F>
void parallel_for(int64_t n, F f) {
  const int nt = (int)std::min<int64_t>(worker_count(), std::max<int64_t>(1, n));
  if (nt <= 1) {
    f(0, n);
    return;
  }
  std::vector<std::thread> th;
  for (int t = 0; t < nt; ++t) {
    const int64_t lo = n * t / nt, hi = n * (t + 1) / nt;
    th.emplace_back([=] { f(lo, hi); });
  }
  for (auto& x : th) x.join();
}

inline void or_word(uint32_t* p, uint32_t v) { __atomic_fetch_or(p, v, __ATOMIC_RELAXED); }

}  // namespace

uw_status encode_host(const uint16_t* w, int64_t N, int64_t K, const uw_encode_opts& o,
                      HostEncoded* out) {
  if (!w || !out) return UW_ERR_ARG;
  if (N < 1 || K < kRow || K % kRow) return UW_ERR_SHAPE;
  if (o.max_code_len < 1 || o.max_code_len > kLutBits) return UW_ERR_ARG;
  if (o.chunk_syms <= 0 || o.chunk_syms % kRow) return UW_ERR_ARG;
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return UW_ERR_SHAPE;
  HostEncoded& e = *out;
  e = HostEncoded();
  e.N = N;
  e.K = K;
  e.max_code_len = o.max_code_len;
  e.chunk_syms = o.chunk_syms;
  const int64_t T = N * K;
  try {
    e.sm.resize(T);
    std::vector<uint8_t> E(T);
    // field split + per-thread histograms
    const int nt = worker_count();
    std::vector<std::vector<int64_t>> hists(nt, std::vector<int64_t>(256, 0));
    std::atomic<int> slot{0};
    parallel_for(T, [&](int64_t lo, int64_t hi) {
      std::vector<int64_t>& h = hists[slot.fetch_add(1)];
      for (int64_t i = lo; i < hi; ++i) {
        const uint16_t b = w[i];
        const uint8_t ex = (uint8_t)((b >> 7) & 0xFF);
        E[i] = ex;
        e.sm[i] = (uint8_t)(((b >> 8) & 0x80) | (b & 0x7F));
        h[ex]++;
      }
    });
    e.hist.assign(256, 0);
    for (auto& h : hists)
      for (int s = 0; s < 256; ++s) e.hist[s] += h[s];

    // code lengths and canonical codes
    package_merge(e.hist.data(), o.max_code_len, e.code_len);
    uint32_t codes[256];
    canonical_codes(e.code_len, codes);

    // chunk bit counts -> offsets
    const int64_t CS = o.chunk_syms;
    const int64_t C = (T + CS - 1) / CS;
    std::vector<uint64_t> cbits(C, 0);
    parallel_for(C, [&](int64_t lo, int64_t hi) {
      for (int64_t c = lo; c < hi; ++c) {
        uint64_t b = 0;
        const int64_t s1 = std::min(T, (c + 1) * CS);
        for (int64_t i = c * CS; i < s1; ++i) b += e.code_len[E[i]];
        cbits[c] = b;
      }
    });
    e.chunk_off.resize(C + 1);
    uint64_t acc = 0;
    for (int64_t c = 0; c < C; ++c) {
      e.chunk_off[c] = (uint32_t)acc;
      acc += cbits[c];
      if (acc > (uint64_t)kMaxStreamWords * 32) return UW_ERR_UNSUPPORTED;
    }
    e.chunk_off[C] = (uint32_t)acc;
    e.total_bits = acc;
    const int64_t n_words = (int64_t)((acc + 31) / 32);
    e.words.assign((size_t)((n_words + 3) / 4 * 4), 0u);

    // bit packing, parallel over chunk ranges; words shared by two ranges are OR-ed
    uint32_t* words = e.words.data();
    parallel_for(C, [&](int64_t c0, int64_t c1) {
      if (c0 >= c1) return;
      uint64_t pos = e.chunk_off[c0];
      int64_t wi = (int64_t)(pos >> 5);
      const int64_t first_wi = wi;
      uint64_t buf = 0;
      int nb = (int)(pos & 31);  // leading bits of the first word belong to the previous range
      const int64_t s1 = std::min(T, c1 * CS);
      for (int64_t i = c0 * CS; i < s1; ++i) {
        const int l = e.code_len[E[i]];
        buf = (buf << l) | codes[E[i]];
        nb += l;
        if (nb >= 32) {
          const uint32_t word = (uint32_t)(buf >> (nb - 32));
          if (wi == first_wi) or_word(&words[wi], word); else words[wi] = word;
          ++wi;
          nb -= 32;
          buf &= (nb ? ((uint64_t(1) << nb) - 1) : 0);
        }
      }
      if (nb > 0) or_word(&words[wi], (uint32_t)(buf << (32 - nb)));
    });

    // palette: the first 16 by count descending, value ascending; pad with the
    // smallest absent values; stored ascending
    std::vector<int> order;
    for (int s = 0; s < 256; ++s)
      if (e.hist[s] > 0) order.push_back(s);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
      return e.hist[a] != e.hist[b] ? e.hist[a] > e.hist[b] : a < b;
    });
    if (order.size() > 16) order.resize(16);
    bool used[256] = {false};
    for (int s : order) used[s] = true;
    for (int v = 0; (int)order.size() < 16 && v < 256; ++v)
      if (!used[v]) {
        order.push_back(v);
        used[v] = true;
      }
    std::sort(order.begin(), order.end());
    for (int i = 0; i < 16; ++i) e.palette[i] = (uint8_t)order[i];
    bool in_pal[256] = {false};
    for (int i = 0; i < 16; ++i) in_pal[e.palette[i]] = true;

    // escape rows
    const int64_t KB = K / kRow;
    const int64_t NW = 4 * ((N + kEscGroupRows - 1) / kEscGroupRows);  // 16 B per 128 rows
    std::vector<uint8_t> esc((size_t)(N * KB), 0);
    parallel_for(N, [&](int64_t n0, int64_t n1) {
      for (int64_t n = n0; n < n1; ++n)
        for (int64_t kb = 0; kb < KB; ++kb) {
          const uint8_t* r = &E[n * K + kb * kRow];
          uint8_t any = 0;
          for (int j = 0; j < kRow; ++j) any |= !in_pal[r[j]];
          esc[n * KB + kb] = any;
        }
    });
    e.esc_bits.assign((size_t)(KB * NW), 0u);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t kb = 0; kb < KB; ++kb)
        if (esc[n * KB + kb]) e.esc_bits[kb * NW + n / 32] |= 1u << (n % 32);
    const int64_t NG = (N + kEscGroupRows - 1) / kEscGroupRows;
    e.esc_off.assign((size_t)(NG * KB + 1), 0u);
    int64_t g = 0, rows = 0;
    for (int64_t nb = 0; nb < NG; ++nb)
      for (int64_t kb = 0; kb < KB; ++kb) {
        const int64_t n1 = std::min(N, (nb + 1) * kEscGroupRows);
        for (int64_t n = nb * kEscGroupRows; n < n1; ++n)
          if (esc[n * KB + kb]) {
            const uint8_t* r = &E[n * K + kb * kRow];
            e.esc_exp.insert(e.esc_exp.end(), r, r + kRow);
            ++rows;
          }
        e.esc_off[++g] = (uint32_t)rows;
      }
  } catch (const std::bad_alloc&) {
    return UW_ERR_OOM;
  }
  return UW_OK;
}

// -------------------------------------------------------------- statistics --

void fill_stats(const uw_format& f, const int64_t* hist, uw_stats_t* s) {
  std::memset(s, 0, sizeof(*s));
  s->N = f.N;
  s->K = f.K;
  const double T = (double)f.N * (double)f.K;
  const uint64_t total_bits = f.n_chunks > 0 ? f.chunk_off[f.n_chunks] : 0;
  s->bits_per_exponent = T > 0 ? (double)total_bits / T : 0.0;
  int maxl = 0, nsym = 0;
  for (int v = 0; v < 256; ++v)
    if (f.code_len[v]) {
      maxl = std::max<int>(maxl, f.code_len[v]);
      nsym++;
    }
  s->max_len_used = maxl;
  s->n_symbols = nsym;
  if (hist) {
    double H = 0, cov = 0;
    for (int v = 0; v < 256; ++v)
      if (hist[v] > 0) {
        const double p = (double)hist[v] / T;
        H -= p * std::log2(p);
      }
    for (int i = 0; i < 16; ++i) cov += (double)hist[f.palette[i]];
    s->entropy_bits = H;
    s->top16_coverage = cov / T;
  } else {
    s->entropy_bits = -1.0;
    s->top16_coverage = -1.0;
  }
  s->n_rows = f.N * (f.K / kRow);
  s->n_escape_rows = f.n_esc_rows;
  s->bytes_stream = (int64_t)((total_bits + 7) / 8);
  s->bytes_offsets = (f.n_chunks + 1) * 4;
  s->bytes_sm = f.N * f.K;
  s->bytes_escape = f.n_esc_rows * kRow + f.n_esc_words * 4 + (f.n_esc_groups + 1) * 4;
  s->bytes_palette_idx = f.N * f.K / 2;
  s->bytes_huffman_bundle = s->bytes_stream + s->bytes_offsets + s->bytes_sm + 256;
  s->bytes_palette_bundle = s->bytes_palette_idx + s->bytes_sm + s->bytes_escape + 16;
}

}  // namespace uw

// ================================================================ C ABI ====

using namespace uw;

extern "C" {

const char* uw_status_str(uw_status s) {
  switch (s) {
    case UW_OK: return "ok";
    case UW_ERR_ARG: return "invalid argument";
    case UW_ERR_SHAPE: return "invalid shape";
    case UW_ERR_FORMAT: return "invalid encoded format";
    case UW_ERR_UNSUPPORTED: return "unsupported";
    case UW_ERR_OOM: return "out of memory";
    case UW_ERR_CUDA: return "CUDA runtime error";
    case UW_ERR_DEVICE: return "device reported corrupt input";
    case UW_ERR_TIMEOUT: return "device wait timed out";
    case UW_ERR_WORKSPACE: return "workspace missing or too small";
    case UW_ERR_IO: return "file input/output failed";
  }
  return "unknown status";
}

int uw_abi_version(void) { return UW_ABI_VERSION; }

void uw_default_encode_opts(uw_encode_opts* o) {
  if (!o) return;
  o->max_code_len = 12;
  o->chunk_syms = 256;
  o->prepare_direct = 1;
  o->reserved = 0;
}

uw_status uw_encode_host(const uint16_t* w_host, int64_t N, int64_t K,
                         const uw_encode_opts* opts, uw_host_t* out) {
  if (!w_host || !out) return UW_ERR_ARG;
  *out = nullptr;
  uw_encode_opts o;
  uw_default_encode_opts(&o);
  if (opts) o = *opts;
  uw_host_s* h = new (std::nothrow) uw_host_s();
  if (!h) return UW_ERR_OOM;
  const uw_status st = encode_host(w_host, N, K, o, &h->enc);
  if (st != UW_OK) {
    delete h;
    return st;
  }
  *out = h;
  return UW_OK;
}

uw_status uw_host_view(uw_host_t h, uw_format* v) {
  if (!h || !v) return UW_ERR_ARG;
  const HostEncoded& e = h->enc;
  std::memset(v, 0, sizeof(*v));
  v->N = e.N;
  v->K = e.K;
  v->max_code_len = e.max_code_len;
  v->chunk_syms = e.chunk_syms;
  std::memcpy(v->code_len, e.code_len, 256);
  std::memcpy(v->palette, e.palette, 16);
  v->n_words = (int64_t)e.words.size();
  v->words = e.words.data();
  v->n_chunks = (int64_t)e.chunk_off.size() - 1;
  v->chunk_off = e.chunk_off.data();
  v->sm = e.sm.data();
  v->n_esc_words = (int64_t)e.esc_bits.size();
  v->esc_bits = e.esc_bits.data();
  v->n_esc_groups = (int64_t)e.esc_off.size() - 1;
  v->esc_off = e.esc_off.data();
  v->n_esc_rows = (int64_t)e.esc_exp.size() / kRow;
  v->esc_exp = e.esc_exp.data();
  return UW_OK;
}

void uw_host_free(uw_host_t h) { delete h; }

uw_status uw_host_stats(uw_host_t h, uw_stats_t* out) {
  if (!h || !out) return UW_ERR_ARG;
  uw_format f;
  uw_host_view(h, &f);
  fill_stats(f, h->enc.hist.data(), out);
  return UW_OK;
}

uw_status uw_validate_format(const uw_format* f) {
  if (!f) return UW_ERR_ARG;
  if (f->N < 1 || f->K < kRow || f->K % kRow) return UW_ERR_SHAPE;
  if (f->N > (int64_t(1) << 31) || f->K > (int64_t(1) << 31)) return UW_ERR_SHAPE;
  if (f->max_code_len < 1 || f->max_code_len > kLutBits) return UW_ERR_FORMAT;
  if (f->chunk_syms <= 0 || f->chunk_syms % kRow) return UW_ERR_FORMAT;
  if (!f->words || !f->chunk_off || !f->sm || !f->esc_bits || !f->esc_off) return UW_ERR_ARG;
  if (f->n_esc_rows > 0 && !f->esc_exp) return UW_ERR_ARG;
  // code lengths: within the cap, Kraft sum <= 1, at least one symbol
  uint64_t kraft = 0;
  int nsym = 0, minl = 99, maxl = 0;
  for (int s = 0; s < 256; ++s) {
    const int l = f->code_len[s];
    if (!l) continue;
    if (l > f->max_code_len) return UW_ERR_FORMAT;
    kraft += 1ull << (kLutBits - l);
    nsym++;
    minl = std::min(minl, l);
    maxl = std::max(maxl, l);
  }
  if (nsym == 0 || kraft > (uint64_t)kLutSize) return UW_ERR_FORMAT;
  // chunk offsets: count, monotone, inside the stream, bit counts plausible
  const int64_t T = f->N * f->K;
  const int64_t C = (T + f->chunk_syms - 1) / f->chunk_syms;
  if (f->n_chunks != C) return UW_ERR_FORMAT;
  if (f->n_words < 0 || f->n_words % 4) return UW_ERR_FORMAT;
  if (f->n_words > kMaxStreamWords) return UW_ERR_UNSUPPORTED;
  if (f->chunk_off[0] != 0) return UW_ERR_FORMAT;
  if ((uint64_t)f->chunk_off[C] > (uint64_t)f->n_words * 32) return UW_ERR_FORMAT;
  for (int64_t c = 0; c < C; ++c) {
    const int64_t syms = std::min<int64_t>(f->chunk_syms, T - c * f->chunk_syms);
    if (f->chunk_off[c + 1] < f->chunk_off[c]) return UW_ERR_FORMAT;
    const uint64_t bits = (uint64_t)f->chunk_off[c + 1] - f->chunk_off[c];
    if (bits < (uint64_t)(syms * minl) || bits > (uint64_t)(syms * maxl)) return UW_ERR_FORMAT;
  }
  // palette entries distinct
  bool seen[256] = {false};
  bool in_pal[256] = {false};
  for (int i = 0; i < 16; ++i) {
    if (seen[f->palette[i]]) return UW_ERR_FORMAT;
    seen[f->palette[i]] = in_pal[f->palette[i]] = true;
  }
  // escape bitmap vs group offsets vs verbatim rows
  const int64_t KB = f->K / kRow;
  const int64_t NG = (f->N + kEscGroupRows - 1) / kEscGroupRows;
  const int64_t NW = 4 * NG;  // words per K block, padded to 16 bytes per 128 rows
  if (f->n_esc_words != KB * NW) return UW_ERR_FORMAT;
  if (f->n_esc_groups != NG * KB) return UW_ERR_FORMAT;
  if (f->esc_off[0] != 0 || (int64_t)f->esc_off[NG * KB] != f->n_esc_rows) return UW_ERR_FORMAT;
  for (int64_t kb = 0; kb < KB; ++kb)  // bits past row N-1 must be clear
    for (int64_t wd = f->N / 32; wd < NW; ++wd) {
      const int64_t first = wd * 32;
      const uint32_t keep = first >= f->N ? 0u : ((1u << (f->N - first)) - 1u);
      if (f->esc_bits[kb * NW + wd] & ~keep) return UW_ERR_FORMAT;
    }
  for (int64_t nb = 0; nb < NG; ++nb)
    for (int64_t kb = 0; kb < KB; ++kb) {
      const int64_t g = nb * KB + kb;
      if (f->esc_off[g + 1] < f->esc_off[g]) return UW_ERR_FORMAT;
      int64_t cnt = 0;
      const int64_t n1 = std::min(f->N, (nb + 1) * kEscGroupRows);
      for (int64_t n = nb * kEscGroupRows; n < n1; ++n)
        cnt += (f->esc_bits[kb * NW + n / 32] >> (n % 32)) & 1u;
      if (cnt != (int64_t)(f->esc_off[g + 1] - f->esc_off[g])) return UW_ERR_FORMAT;
    }
  for (int64_t r = 0; r < f->n_esc_rows; ++r) {
    bool outside = false;
    for (int j = 0; j < kRow; ++j) outside |= !in_pal[f->esc_exp[r * kRow + j]];
    if (!outside) return UW_ERR_FORMAT;  // an escape row must need escaping
  }
  return UW_OK;
}

}  // extern "C"
