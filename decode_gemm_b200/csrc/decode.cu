// Chunk-parallel Huffman decoder and palette transcoder for sm_100a.
//
// *Unweight*, "Four ways to use compressed weights": the preprocessing kernels
// of pipelines 1-3 (full decode to BF16, exponent-only decode, transcode to
// 4-bit palette indices).  "Sharing the GPU between decode and compute": the
// decoder works from a ~16 KB lookup table in shared memory.
//
// Design (B200):
//   * One lane decodes one chunk (its start bit is stored, so chunks are
//     independent); a warp owns 32 consecutive chunks; one CTA per SM, whose
//     16-32 warps share the table in shared memory, strides over the chunk
//     groups (the warp count is picked so the last pass is nearly full).
//   * The 4096-entry table maps the next 12 stream bits to up to 5 palette
//     ranks, the number of stream bits they use and 4x their count.  Every
//     output derives from ranks: the transcode writes them, the exponent and
//     full decodes expand them through the 16-entry palette with byte
//     permutes.  A window that starts with the code of an exponent outside the
//     palette (rare; only inside escape rows) yields a rank-0 placeholder and
//     is flagged: the transcode ignores it (the row is zeroed anyway); the
//     other modes record the exponent as a per-lane exception and patch it
//     after the coalesced write, or, when a lane's exception list overflows,
//     replay the whole chunk one symbol at a time.
//   * Bit reader: a window of four stream words and a bit offset q < 32 into
//     the first; a lookup reads the 12 bits at q with one funnel shift, and the
//     window slides by a word (one predicated load, no branch) once q passes
//     32.  Lookups go in pairs with one slide per pair.
//   * While at least 2 x 5 symbols of the chunk are left every lookup takes
//     its whole entry with no per-lookup checks; the last few symbols go one
//     code at a time where an entry holds more than are left, so a lane stops
//     exactly at its chunk's last symbol, and its end bit is checked against
//     the stored offset.
//   * Ranks are packed into words (8 per word) in registers and each completed
//     word goes to a per-lane shared-memory row (stride 17 words: lanes that
//     store their k-th word at the same time hit distinct banks).  After a
//     128-symbol round the warp writes its 32 chunks' outputs with 128-bit
//     stores, each warp-wide store covering contiguous, fully used lines.
//     Shared memory stays small so L1 can hold every lane's stream lines.
//   * The Huffman-direct product (kDecodeDot; *Unweight*, "How the
//     reconstructive matmul works": decoding inside the matmul) keeps the
//     decode and replaces the write-out: a warp's 32 chunks are one chunk
//     position of 32 rows, and each decoded round is multiplied with X in
//     warp-level BF16 MMAs (FP32 accumulation) while the weights are still
//     in registers; only Y leaves the chip.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "bf16_fields.cuh"
#include "pdl.cuh"
#include "uw_internal.h"
#include "uw_kernels.h"

namespace uw {

namespace {

constexpr int kMaxWarps = 32;                   // one CTA per SM, up to 1024 threads
constexpr int kMinWarps = 16;
constexpr int kRoundSyms = 128;                 // symbols per lane per staging round
constexpr int kRoundWords = kRoundSyms / 8;     // 16 words of 4-bit ranks
constexpr int kStageStride = kRoundWords + 1;   // 17: lanes spread over banks
constexpr int kExcCap = 4;                      // exceptions held per lane
constexpr int kFullPair = 2 * 4 * kPalCap;      // 4x symbols two whole lookups may yield
constexpr int kFullOne = 4 * kPalCap;
constexpr int kNoRound = 1 << 30;
// The product runs at most 25 warps per CTA: 72 registers a thread instead of
// 64 (fewer spills; measured 3 % faster than a 32-warp bound).
constexpr int kDotMaxWarps = 25;


// Shared memory: the tables, then per warp its ranks stage (32 lanes x 17
// words) and exception lists.  At most ~104 KB, so L1 keeps over 120 KB for the
// lanes' stream lines (each lane streams its own).
struct __align__(16) SmemHead {
  uint32_t lut[kLutSize];
  uint32_t canon[kCanonWords];
};
constexpr int kWarpSmemWords = 32 * kStageStride + 32 * kExcCap;
// The product's running sums between rounds: 8 per lane (see below).
constexpr int kDotAccWords = 32 * 16;  // and its corrections: 8 more per lane

size_t smem_bytes(int warps, int mode) {
  return sizeof(SmemHead) + (size_t)warps * (kWarpSmemWords + (mode == kDecodeDot ? kDotAccWords : 0)) * 4;
}


// Four consecutive stream words; bit q (MSB first) of w0 is the next bit.
struct Bits {
  uint32_t w0, w1, w2, w3;
  uint32_t q;
  uint32_t nxt;  // index of the word after w3
};

__device__ __forceinline__ void bits_init(Bits& b, const uint32_t* words, uint32_t start) {
  const uint32_t i = start >> 5;
  b.w0 = __ldg(words + i);
  b.w1 = __ldg(words + i + 1);
  b.w2 = __ldg(words + i + 2);
  b.w3 = __ldg(words + i + 3);
  b.q = start & 31u;
  b.nxt = i + 4;
}

// The 32 stream bits starting at the next bit (q < 32).
__device__ __forceinline__ uint32_t bits_peek(const Bits& b) {
  return __funnelshift_l(b.w1, b.w0, b.q);
}

// Slide the window by one word once q has passed 32 (q < 64): predicated
// moves and load, no branch.  Reads stay in the padded stream buffer: a lane
// never reads more than 12 bits per symbol past its chunk's start, plus the
// window.
__device__ __forceinline__ void bits_slide(Bits& b, const uint32_t* words) {
  const uint32_t* p = words + b.nxt;
  asm("{\n\t.reg .pred s;\n\t"
      "setp.gt.u32 s, %4, 31;\n\t"
      "@s mov.b32 %0, %1;\n\t"
      "@s mov.b32 %1, %2;\n\t"
      "@s mov.b32 %2, %3;\n\t"
      "@s ld.global.nc.u32 %3, [%6];\n\t"
      "@s add.u32 %5, %5, 1;\n\t"
      "and.b32 %4, %4, 31;\n\t}"
      : "+r"(b.w0), "+r"(b.w1), "+r"(b.w2), "+r"(b.w3), "+r"(b.q), "+r"(b.nxt)
      : "l"(p));
}

// Predicated global accesses: the write-out computes every piece and only
// stores (or, for inputs that may lie past the arrays, loads) under the
// predicate, so its loops carry no branch and their iterations interleave.
__device__ __forceinline__ void st_v4_if(void* p, uint4 v, bool pred) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %5, 0;\n\t"
               "@q st.global.v4.u32 [%0], {%1, %2, %3, %4};\n\t}"
               ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"((uint32_t)pred)
               : "memory");
}

__device__ __forceinline__ uint2 ld_v2_if(const void* p, bool pred) {
  uint2 v = make_uint2(0u, 0u);
  asm("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %3, 0;\n\t"
      "@q ld.global.nc.v2.u32 {%0, %1}, [%2];\n\t}"
      : "+r"(v.x), "+r"(v.y)
      : "l"(p), "r"((uint32_t)pred));
  return v;
}

__device__ __forceinline__ uint32_t ld_u32_if(const uint32_t* p, bool pred) {
  uint32_t v = 0u;
  asm("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q ld.global.nc.u32 %0, [%1];\n\t}"
      : "+r"(v)
      : "l"(p), "r"((uint32_t)pred));
  return v;
}

// D += A B for one m16n8k16 tile (BF16 operands, FP32 accumulation).  Lane
// (g, t) = (lane / 4, lane % 4) holds a0..a3 = A[g][2t..2t+1], A[g+8][2t..2t+1],
// A[g][2t+8..2t+9], A[g+8][2t+8..2t+9], b0 / b1 = B[2t..2t+1][g] /
// B[2t+8..2t+9][g], and d = D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1].
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The caller's X, read after the dependency wait with coherent loads (the
// kernel ahead of this one may have written it).
__device__ __forceinline__ uint4 ld_x4(const void* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ uint16_t ld_x1(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.u16 %0, [%1];" : "=h"(v) : "l"(p) : "memory");
  return v;
}

// 16 sign+mantissa bytes (the handle's own, never written by a kernel), or
// zeros where pred is false.
__device__ __forceinline__ uint4 ld_v4_if(const void* p, bool pred) {
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  asm("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %5, 0;\n\t"
      "@q ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "l"(p), "r"((uint32_t)pred));
  return v;
}


// Stream bit position of the next bit.
__device__ __forceinline__ uint32_t bits_pos(const Bits& b) { return (b.nxt - 4u) * 32u + b.q; }

// Length of the code that starts the 12-bit window (canonical limits).
__device__ __forceinline__ uint32_t first_code_len(const uint32_t* canon, uint32_t idx) {
  uint32_t len = 1;
  while (len < 12 && idx >= canon[kCanonLimit + len]) ++len;
  return len;
}

// Exponent whose code starts the 12-bit window, and that code's length.
__device__ __forceinline__ uint32_t canon_symbol(const uint32_t* canon, uint32_t idx,
                                                 uint32_t* len_out) {
  const uint32_t len = first_code_len(canon, idx);
  const uint32_t code = idx >> (12 - len);
  const uint32_t k = canon[kCanonOffset + len] + code - canon[kCanonFirst + len];
  *len_out = len;
  return reinterpret_cast<const uint8_t*>(canon + kCanonSymbols)[k & 255];
}

// Ranks are appended to a_lo (ab valid bits, < 32 between appends); each
// completed word is stored at shared address sp, which then moves on.
struct Packer {
  uint32_t a_lo, ab;
  uint32_t sp;
};

// Append the entry's ranks (c4 = 4 x their count); a completed word is stored
// with a predicated shared store.
__device__ __forceinline__ void pack(Packer& pk, uint32_t e, uint32_t c4) {
  asm("{\n\t.reg .pred f;\n\t.reg .b32 v, lo, hi;\n\t"
      "shr.b32 v, %3, 12;\n\t"
      "shl.b32 lo, v, %1;\n\t"
      "or.b32 lo, lo, %0;\n\t"
      "shf.l.wrap.b32 hi, v, 0, %1;\n\t"
      "add.u32 %1, %1, %4;\n\t"
      "setp.gt.u32 f, %1, 31;\n\t"
      "@f st.shared.u32 [%2], lo;\n\t"
      "@f add.u32 %2, %2, 4;\n\t"
      "selp.b32 %0, hi, lo, f;\n\t"
      "and.b32 %1, %1, 31;\n\t}"
      : "+r"(pk.a_lo), "+r"(pk.ab), "+r"(pk.sp)
      : "r"(e), "r"(c4)
      : "memory");
}

// GATHER (full decode only): the launch's chunks are the chunks of the rows
// a.rows[] (see DecodeArgs); a lane reads its chunk's stream and S at the real
// chunk and writes its output at the launch's (virtual) chunk.
//
// DOT (the Huffman-direct product): the write-out becomes a matrix product of
// the rebuilt weights with X; nothing but Y leaves the chip.
template <int MODE, bool GATHER>
__global__ void __launch_bounds__(32 * (MODE == kDecodeDot ? kDotMaxWarps : kMaxWarps), 1)
    decode_kernel(const DecodeArgs a, void* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SmemHead& sm = *reinterpret_cast<SmemHead*>(smem_raw);
  for (int i = threadIdx.x; i < kLutSize / 4; i += blockDim.x)
    reinterpret_cast<uint4*>(sm.lut)[i] = __ldg(reinterpret_cast<const uint4*>(a.lut) + i);
  for (int i = threadIdx.x; i < kCanonWords; i += blockDim.x) sm.canon[i] = __ldg(a.canon + i);
  __syncthreads();
  // the tables, the stream and S are the handle's own (never written by a
  // kernel); the output may still be read by the kernel before this one, so a
  // warp waits for that kernel before its first write (its first round is
  // decoded meanwhile)
  if (threadIdx.x == 0) pdl_release();
  bool waited = false;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int n_warps = blockDim.x >> 5;
  uint32_t* const stage =
      reinterpret_cast<uint32_t*>(smem_raw + sizeof(SmemHead)) + warp * kWarpSmemWords;
  const uint32_t st_addr = (uint32_t)__cvta_generic_to_shared(stage + lane * kStageStride);
  uint32_t* const exc = stage + 32 * kStageStride + lane * kExcCap;
  // (product) this lane's 8 running sums and 8 corrections (one per token),
  // behind all warps' areas
  float* const dsum_w = reinterpret_cast<float*>(smem_raw + sizeof(SmemHead)) +
                        (size_t)n_warps * kWarpSmemWords + (size_t)warp * 32 * 16;
  float* const dsum = dsum_w + lane * 16;
  float* const dcorr = dsum + 8;
  const uint32_t* const lut = sm.lut;
  // the product's groups are 32 rows at one chunk position (one column range)
  const int64_t groups =
      MODE == kDecodeDot ? (a.matrix_rows + 31) / 32 * a.cpr : (a.n_chunks + 31) / 32;
  const uint32_t* const words = a.words;
  const uint32_t stream_bits = (uint32_t)(a.n_words * 32);
  const int64_t cs = a.chunk_syms;
  const int rows_per_chunk = (int)(cs / 64);
  const uint32_t p0 = a.palette[0], p1 = a.palette[1], p2 = a.palette[2], p3 = a.palette[3];
  const bool pal_run = a.pal_run_b4 != 0xFFFFFFFFu;  // ranks are exponent - b
  const uint32_t b4 = a.pal_run_b4;
  const int64_t grid_warps = (int64_t)gridDim.x * n_warps;

  // A warp takes runs of G consecutive groups (the product: G chunk positions
  // of the same 32 rows, whose sums carry over; every other mode: G = 1).
  const int G = MODE == kDecodeDot ? a.run : 1;
  const int64_t n_runs = (groups + G - 1) / G;
  bool fixed = false;  // (product) a correction was made in this run
  for (int64_t run = (int64_t)blockIdx.x * n_warps + warp; run < n_runs; run += grid_warps)
  for (int64_t grp = run * G; grp < (run + 1) * G && grp < groups; ++grp) {
    const bool run_first = grp == run * G;
    const bool run_last = grp + 1 == (run + 1) * G || grp + 1 == groups;
    const int64_t c0 = grp * 32;
    const int64_t c = c0 + lane;
    // product: rows rb*32 .. rb*32+31 (lane = row), chunk position cc
    const int64_t rb = MODE == kDecodeDot ? grp / a.cpr : 0;
    const int cc = MODE == kDecodeDot ? (int)(grp - rb * a.cpr) : 0;
    const bool live = MODE == kDecodeDot ? rb * 32 + lane < a.matrix_rows : c < a.n_chunks;
    uint32_t start = 0, end = 0;
    int nsyms = 0;
    bool bad = false;
    // the chunk of the matrix this lane decodes
    int64_t cr = MODE == kDecodeDot ? (rb * 32 + lane) * a.cpr + cc : c;
    if (GATHER && !waited) {  // the row ids are the caller's: after the kernel before
      pdl_wait();
      waited = true;
    }
    if (GATHER && live) {
      const int64_t v = c / a.cpr;
      const int64_t row = a.rows[v];
      if (row < 0 || row >= a.matrix_rows) {  // not a row of the matrix: nothing is read
        bad = true;
        cr = -1;
      } else {
        cr = row * a.cpr + (c - v * a.cpr);
      }
    }
    if (live && cr >= 0) {
      start = __ldg(a.chunk_off + cr);
      end = __ldg(a.chunk_off + cr + 1);
      const int64_t left = (GATHER || MODE == kDecodeDot) ? cs : a.total_syms - c * cs;
      nsyms = (int)(left < cs ? left : cs);
      if (start > stream_bits) {  // corrupt offset: nothing is read
        bad = true;
        start = 0;
        nsyms = 0;
      }
    }
    if (cr < 0 || (MODE == kDecodeDot && !live)) cr = 0;  // (a rejected row or a row
                                                          // past N reads nothing)
    // the stream of this warp's next group: into L2 while this one decodes
    if (!GATHER) {
      int64_t cn = c + grid_warps * 32;
      bool next = cn < a.n_chunks;
      if (MODE == kDecodeDot) {
        const int64_t g2 = run_last ? (run + grid_warps) * G : grp + 1, rb2 = g2 / a.cpr;
        cn = (rb2 * 32 + lane) * a.cpr + (g2 - rb2 * a.cpr);
        next = g2 < groups && rb2 * 32 + lane < a.matrix_rows;
      }
      if (next) {
        const uint32_t nb = __ldg(a.chunk_off + cn) >> 3;
        if (nb < stream_bits / 8) {
          const char* p = reinterpret_cast<const char*>(words) + nb;
          asm volatile("prefetch.global.L2 [%0];" :: "l"(p));
          asm volatile("prefetch.global.L2 [%0];" :: "l"(p + 128));
        }
      }
    }
    const int my_rounds = (nsyms + kRoundSyms - 1) / kRoundSyms;
    const int warp_rounds = __reduce_max_sync(0xffffffffu, my_rounds);
    // symbols from the group's first one to the end of the matrix
    const int64_t grp_syms_left = a.total_syms - c0 * cs;

    // (row, K block) of the 64-weight row where this lane's round starts
    int row_n = 0, row_kb = 0;
    if (MODE == kDecodePalette && live) {
      const int64_t row0 = c * rows_per_chunk;
      row_n = (int)(row0 / a.kb_per_row);
      row_kb = (int)(row0 - (int64_t)row_n * a.kb_per_row);
    }

    Bits b;
    bits_init(b, words, start);
    Packer pk{0u, 0u, st_addr};
    int left4 = 4 * nsyms;  // 4 x symbols of the chunk not yet decoded
    int nx = 0;
    bool overflow = false;

    // Product state: the first round after which this lane's chunk is left to
    // the replay (its exception list overflowed).  The running sums (dsum)
    // and the lane's corrections (dcorr: the true weights' products at its
    // chunk's exceptions, per token) live in shared memory.
    int dirty_from = kNoRound;
    if (MODE == kDecodeDot) {
#pragma unroll
      for (int q = 0; q < kExcCap; ++q) exc[q] = 0xFFFFFFFFu;
      if (run_first) {
#pragma unroll
        for (int v = 0; v < 4; ++v) reinterpret_cast<float4*>(dsum)[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        fixed = false;
      }
    }
    // BF16 weight w times X[t, column col] into this lane's correction
    // (the product of two BF16 is exact in FP32)
    auto add_corr = [&](uint32_t w, int64_t col) {
      const int64_t K = (int64_t)a.kb_per_row * kRow;
      fixed = true;
      for (int t = 0; t < a.m; ++t)
        dcorr[t] += __uint_as_float(w << 16) * __uint_as_float((uint32_t)ld_x1(a.x + t * K + col) << 16);
    };

    // A flagged entry: record the exception (position = symbols decoded so far).
    auto special = [&](uint32_t e, uint32_t win, int left4_before) {
      if (e & kLutInvalid) {
        bad = true;
      } else if (MODE != kDecodePalette) {
        uint32_t len;
        const uint32_t ex = canon_symbol(sm.canon, win >> 20, &len);
        const uint32_t pos = (uint32_t)((4 * nsyms - left4_before) >> 2);
        if (nx < kExcCap)
          exc[nx++] = (pos << 8) | ex;
        else
          overflow = true;
      }
    };
    // Two whole lookups (at least 2 x kPalCap symbols left, q < 32).
    auto lookup_pair = [&]() {
      const uint32_t win1 = bits_peek(b);
      const uint32_t e1 = lut[win1 >> 20];
      const uint32_t q1 = b.q + (e1 & 15u);
      const bool up = q1 >= 32u;
      const uint32_t x0 = up ? b.w1 : b.w0, x1 = up ? b.w2 : b.w1;
      const uint32_t win2 = __funnelshift_l(x1, x0, q1);
      const uint32_t e2 = lut[win2 >> 20];
      if ((e1 | e2) & kLutSpecial) {
        if (e1 & kLutSpecial) special(e1, win1, left4);
        if (e2 & kLutSpecial) special(e2, win2, left4 - (int)((e1 >> 4) & 31u));
      }
      b.q = q1 + (e2 & 15u);
      const uint32_t c1 = (e1 >> 4) & 31u, c2 = (e2 >> 4) & 31u;
      left4 -= (int)(c1 + c2);
      pack(pk, e1, c1);
      pack(pk, e2, c2);
      bits_slide(b, words);
    };
    // One lookup; TAIL: fewer than kPalCap symbols may be left, so an entry
    // holding more than are left gives way to its first code alone.
    auto lookup_one = [&](auto tail_tag) {
      constexpr bool TAIL = decltype(tail_tag)::value;
      const uint32_t win = bits_peek(b);
      uint32_t e = lut[win >> 20];
      if (TAIL && (int)((e >> 4) & 31u) > left4)
        e = (e & 0xF000u) | (4u << 4) | first_code_len(sm.canon, win >> 20);
      if (e & kLutSpecial) special(e, win, left4);
      b.q += e & 15u;
      const uint32_t c = (e >> 4) & 31u;
      left4 -= (int)c;
      pack(pk, e, c);
      bits_slide(b, words);
    };

    for (int r = 0; r < warp_rounds; ++r) {
      pk.sp = st_addr;
      if ((MODE == kDecodeFull || MODE == kDecodeDot) && r < my_rounds) {
        // this round's sign+mantissa bytes into L2 (the product: into L1, its
        // reads follow this lane's own chunk) while the round decodes
        const uint8_t* sp8 = a.sm + cr * cs + (int64_t)r * kRoundSyms;
        if (MODE == kDecodeDot)
          asm volatile("prefetch.global.L1 [%0];" :: "l"(sp8));
        else
          asm volatile("prefetch.global.L2 [%0];" :: "l"(sp8));
      }
      if (r < my_rounds - 1) {
        // a round that ends inside the chunk: fill exactly kRoundWords words,
        // the ranks past them (fewer than 32 bits) carry into the next round
        while (pk.sp < st_addr + 4 * (kRoundWords - 1)) lookup_pair();
        while (pk.sp < st_addr + 4 * kRoundWords) lookup_one(std::false_type());
      } else if (r == my_rounds - 1) {
        while (left4 >= kFullPair) lookup_pair();
        while (left4 >= kFullOne) lookup_one(std::false_type());
        while (left4 > 0) lookup_one(std::true_type());
      }
      __syncwarp();
      if (!waited) {
        pdl_wait();
        waited = true;
      }

      // ---- coalesced write-out of round r for the warp's 32 chunks ----
      // rel0: this round's first symbol inside each chunk; a lane's part of
      // chunk j is written when it lies inside the chunk and the matrix
      const int64_t rel0 = (int64_t)r * kRoundSyms;
      if (MODE == kDecodeExp) {
        // 8 lanes per chunk, 16 symbols (two rank words) per lane
        const int m = lane & 7, jq = lane >> 3;
        const bool in_chunk = rel0 + 16 * m < cs;
        uint8_t* base = static_cast<uint8_t*>(out) + c0 * cs + rel0 + 16 * m;
        auto write = [&](auto expo) {
#pragma unroll 4
          for (int i = 0; i < 8; ++i) {
            const int j = 4 * i + jq;
            const int64_t o = (int64_t)j * cs;
            const uint32_t* sw = stage + j * kStageStride + 2 * m;
            const uint2 lo = expo(sw[0]);
            const uint2 hi = expo(sw[1]);
            st_v4_if(base + o, make_uint4(lo.x, lo.y, hi.x, hi.y),
                     in_chunk && o + rel0 + 16 * m < grp_syms_left);
          }
        };
        // (the palette form is uniform: one loop per form)
        if (pal_run)
          write([&](uint32_t v) { return run8(v, b4); });
        else
          write([&](uint32_t v) { return palette8(v, p0, p1, p2, p3); });
      } else if (MODE == kDecodeFull) {
        // 16 lanes per chunk, 8 symbols (one rank word) per lane
        const int m = lane & 15, jh = lane >> 4;
        const bool in_chunk = rel0 + 8 * m < cs;
        const int64_t sym0 = c0 * cs + rel0 + 8 * m;
        const uint8_t* sbase = a.sm + sym0;
        uint16_t* obase = static_cast<uint16_t*>(out) + sym0;
        auto write = [&](auto expo) {
          // eight loads in flight before their first use
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint2 sv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int j = 16 * h + 2 * i + jh;
              const int64_t o = (int64_t)j * cs;
              // S of chunk j: consecutive in the matrix, or (gather) at its real chunk
              const uint8_t* sp =
                  GATHER ? a.sm + (int64_t)(uint32_t)__shfl_sync(0xffffffffu, (uint32_t)cr, j) * cs +
                               rel0 + 8 * m
                         : sbase + o;
              sv[i] = ld_v2_if(sp, in_chunk && o + rel0 + 8 * m < grp_syms_left);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int j = 16 * h + 2 * i + jh;
              const int64_t o = (int64_t)j * cs;
              const uint2 e = expo(stage[j * kStageStride + m]);
              const uint2 lo = merge4(sv[i].x, e.x), hi = merge4(sv[i].y, e.y);
              st_v4_if(obase + o, make_uint4(lo.x, lo.y, hi.x, hi.y),
                       in_chunk && o + rel0 + 8 * m < grp_syms_left);
            }
          }
        };
        if (pal_run)
          write([&](uint32_t v) { return run8(v, b4); });
        else
          write([&](uint32_t v) { return palette8(v, p0, p1, p2, p3); });
      } else if (MODE == kDecodeDot) {
        // The group's 32 chunks hold the same columns of 32 rows, so the
        // round's product is a small matrix product: for each block of 16
        // rows and each 16 of the round's 128 columns, one mma.sync m16n8k16
        // with A = the rebuilt BF16 weights, straight from the field merge,
        // and B = X transposed (tokens as columns, zero past M), FP32
        // accumulation.  The 16 k slots of MMA q are columns 32t + 4q + {0..3}
        // of lane group t = lane % 4 (any column order works when A and B
        // share it), so lane (g, t) = (lane / 4, lane % 4) rebuilds rows g and
        // g + 8 of each block at columns 32t .. 32t+31 and holds X[g] at the
        // same columns.  A lane whose exception list overflowed leaves its
        // chunk to the replay from this round on; at recorded exceptions the
        // weight is zeroed here and the owner lane adds the true product to
        // its correction.
        if (overflow && dirty_from == kNoRound) dirty_from = r;
        const uint32_t dirty = __ballot_sync(0xffffffffu, dirty_from <= r);
        const uint32_t excm = __ballot_sync(0xffffffffu, nx > 0);
        const int g = lane >> 2, tq = lane & 3;
        const int p32 = (int)rel0 + 32 * tq;  // this lane's first symbol in each chunk
        const bool in_chunk = p32 < cs;
        const int64_t K = (int64_t)a.kb_per_row * kRow;
        const int64_t col0 = (int64_t)cc * cs + p32;  // its first column
        // X[g] at this lane's 32 columns (zero past M or past the chunk), in
        // registers for the round (measured: 13 % faster at M = 8 than four
        // columns loaded per MMA)
        const bool have_x = in_chunk && g < a.m;
        const uint16_t* xp = a.x + (have_x ? g * K + col0 : 0);
        uint32_t xr[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x4 = have_x ? ld_x4(xp + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
          xr[4 * v] = x4.x;
          xr[4 * v + 1] = x4.y;
          xr[4 * v + 2] = x4.z;
          xr[4 * v + 3] = x4.w;
        }
        // this lane's rows j (g, then g + 8, of block bk): rebuild rule and
        // exceptions to zero (bit i: symbol p32 + i)
        auto row_setup = [&](int j, bool& valid, uint32_t& kill) {
          valid = in_chunk && rb * 32 + j < a.matrix_rows && !((dirty >> j) & 1u);
          kill = 0;
          if ((excm >> j) & 1u) {
            const uint32_t* ej = stage + 32 * kStageStride + j * kExcCap;
#pragma unroll
            for (int qq = 0; qq < kExcCap; ++qq) {
              const uint32_t d = (ej[qq] >> 8) - (uint32_t)p32;
              if (d < 32u) kill |= 1u << d;
            }
          }
        };
        auto killed = [&](uint2 b, uint32_t kill, int q) {
          const uint32_t k4 = kill >> (4 * q);
          b.x &= ((k4 & 1u) ? 0u : 0xFFFFu) | ((k4 & 2u) ? 0u : 0xFFFF0000u);
          b.y &= ((k4 & 4u) ? 0u : 0xFFFFu) | ((k4 & 8u) ? 0u : 0xFFFF0000u);
          return b;
        };
        auto dot = [&](auto expo) {
#pragma unroll 1
          for (int bk = 0; bk < 2; ++bk) {
            const int ja = 16 * bk + g, jb = ja + 8;
            bool va, vb;
            uint32_t ka, kb;
            row_setup(ja, va, ka);
            row_setup(jb, vb, kb);
            const bool any_kill = __any_sync(0xffffffffu, (ka | kb) != 0u);
            float4 d4 = reinterpret_cast<const float4*>(dsum)[bk];  // the block's sums
            float dacc[4] = {d4.x, d4.y, d4.z, d4.w};
            __syncwarp();  // converged for the warp-wide MMAs below
            const uint8_t* spa = a.sm + (rb * 32 + ja) * K + col0;
            const uint8_t* spb = a.sm + (rb * 32 + jb) * K + col0;
#pragma unroll
            for (int u = 0; u < 4; ++u) {  // symbols 8u .. 8u+7 of the lane's 32
              const uint2 sa = ld_v2_if(spa + 8 * u, va), sb = ld_v2_if(spb + 8 * u, vb);
              uint2 ea = expo(stage[ja * kStageStride + 4 * tq + u]);
              uint2 eb = expo(stage[jb * kStageStride + 4 * tq + u]);
              ea = va ? ea : make_uint2(0u, 0u);  // (S reads as zero there too: +0)
              eb = vb ? eb : make_uint2(0u, 0u);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int q = 2 * u + h;
                uint2 wa = merge4(h ? sa.y : sa.x, h ? ea.y : ea.x);
                uint2 wb = merge4(h ? sb.y : sb.x, h ? eb.y : eb.x);
                if (any_kill) {  // (uniform; lanes without exceptions keep all)
                  wa = killed(wa, ka, q);
                  wb = killed(wb, kb, q);
                }
                mma_16816(dacc, wa.x, wb.x, wa.y, wb.y, xr[2 * q], xr[2 * q + 1]);
              }
            }
            reinterpret_cast<float4*>(dsum)[bk] = make_float4(dacc[0], dacc[1], dacc[2], dacc[3]);
          }
        };
        if (pal_run)
          dot([&](uint32_t v) { return run8(v, b4); });
        else
          dot([&](uint32_t v) { return palette8(v, p0, p1, p2, p3); });
      } else {
        // 4 lanes per chunk, 32 symbols (four rank words, half a 64-weight
        // row) per lane; escape rows are written as zeros
        const int m = lane & 3, jr = lane >> 2;
        const bool in_chunk = rel0 + 32 * m < cs;
        const int n_me = row_n, kb_me = row_kb;
        uint8_t* base = static_cast<uint8_t*>(out) + (c0 * cs + rel0) / 2 + 16 * m;
#pragma unroll 2
        for (int i = 0; i < 4; ++i) {
          const int j = 8 * i + jr;
          const int n_j = __shfl_sync(0xffffffffu, n_me, j);
          const int kb_j = __shfl_sync(0xffffffffu, kb_me, j);
          const int64_t o = (int64_t)j * cs;
          const bool valid = in_chunk && o + rel0 + 32 * m < grp_syms_left;
          int n = n_j, kb = kb_j + (m >> 1);
          while (kb >= a.kb_per_row) {  // a row of 64 weights past the end of row n
            kb -= a.kb_per_row;
            ++n;
          }
          const bool esc =
              (ld_u32_if(a.esc_bits + (int64_t)kb * a.esc_nw + (n >> 5), valid) >> (n & 31)) & 1u;
          const uint32_t* sw = stage + j * kStageStride + 4 * m;
          // stored word order: element 2t at bits 4t, 2t+1 at bits 16+4t
          const uint4 v = esc ? make_uint4(0u, 0u, 0u, 0u)
                              : make_uint4(nibbles_interleave(sw[0]), nibbles_interleave(sw[1]),
                                           nibbles_interleave(sw[2]), nibbles_interleave(sw[3]));
          st_v4_if(base + o / 2, v, valid);
        }
      }
      __syncwarp();
      if (MODE == kDecodePalette) {  // the next round's first row
        row_kb += kRoundSyms / 64;
        while (row_kb >= a.kb_per_row) {
          row_kb -= a.kb_per_row;
          ++row_n;
        }
      }

      // exceptions of this round overwrite the placeholder the bulk write left
      if (MODE != kDecodePalette && nx > 0) {
        const int64_t base = c * cs;
        const uint32_t lo = (uint32_t)(r * kRoundSyms), hi = lo + kRoundSyms;
        int keep = 0;
        for (int i = 0; i < nx; ++i) {
          const uint32_t x = exc[i];
          const uint32_t pos = x >> 8;
          if (pos >= lo && pos < hi) {
            const int64_t o = base + pos;
            if (MODE == kDecodeExp) {
              static_cast<uint8_t*>(out)[o] = (uint8_t)(x & 0xFFu);
            } else if (MODE == kDecodeFull) {
              const uint32_t s = a.sm[cr * cs + pos];
              static_cast<uint16_t*>(out)[o] =
                  (uint16_t)(((s & 0x80u) << 8) | ((x & 0xFFu) << 7) | (s & 0x7Fu));
            } else if (dirty_from > r) {  // the product: the true weight's terms
              const uint32_t s = a.sm[cr * cs + pos];
              add_corr(((s & 0x80u) << 8) | ((x & 0xFFu) << 7) | (s & 0x7Fu),
                       (int64_t)cc * cs + pos);
            }
          } else {
            exc[keep++] = x;
          }
        }
        if (MODE == kDecodeDot)  // freed entries match no position
          for (int q = keep; q < nx; ++q) exc[q] = 0xFFFFFFFFu;
        nx = keep;
      }
      __syncwarp();
    }

    // a lane whose exception list overflowed replays its chunk symbol by symbol
    if (MODE == kDecodeDot && overflow) {  // the product: from its first dirty round on
      Bits sb;
      bits_init(sb, words, start);
      for (int i = 0; i < nsyms; ++i) {
        uint32_t len;
        const uint32_t ex = canon_symbol(sm.canon, bits_peek(sb) >> 20, &len);
        sb.q += len;
        bits_slide(sb, words);
        if (i >= dirty_from * kRoundSyms) {
          const uint32_t s = a.sm[cr * cs + i];
          add_corr(((s & 0x80u) << 8) | (ex << 7) | (s & 0x7Fu), (int64_t)cc * cs + i);
        }
      }
    }
    if (MODE != kDecodePalette && MODE != kDecodeDot && overflow) {
      Bits sb;
      bits_init(sb, words, start);
      const int64_t base = c * cs;
      for (int i = 0; i < nsyms; ++i) {
        uint32_t len;
        const uint32_t ex = canon_symbol(sm.canon, bits_peek(sb) >> 20, &len);
        sb.q += len;
        bits_slide(sb, words);
        if (MODE == kDecodeExp) {
          static_cast<uint8_t*>(out)[base + i] = (uint8_t)ex;
        } else {
          const uint32_t s = a.sm[cr * cs + i];
          static_cast<uint16_t*>(out)[base + i] =
              (uint16_t)(((s & 0x80u) << 8) | (ex << 7) | (s & 0x7Fu));
        }
      }
    }
    if (live && (bad || bits_pos(b) != end)) atomicOr(a.status, kStatusBadChunk);
    __syncwarp();

    if (MODE == kDecodeDot && run_last) {
      // Lane (g, t) holds the sums of rows 16 bk + g + 8 h (dsum[4 bk + 2 h +
      // e]) for tokens 2t + e; with the owners' corrections added they are
      // the run's partial sums, stored at part[(row * kDotMaxM + token) * S +
      // segment] (S = cpr / G segments per row, this run's is cc / G).  The
      // run that brings a row's S-th partial adds them in segment order and
      // writes Y.
      const int g = lane >> 2, tq = lane & 3;
      const int nseg = a.cpr / G;
      const bool any_corr = __any_sync(0xffffffffu, fixed);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int bk = k >> 2, h = (k >> 1) & 1, e = k & 1;
        const int j = 16 * bk + g + 8 * h, t = 2 * tq + e;
        float v = dsum[k];
        if (any_corr && t < a.m) v += dsum_w[j * 16 + 8 + t];  // row j's owner's correction
        const int64_t row = rb * 32 + j;
        if (t < a.m && row < a.matrix_rows) a.part[(row * kDotMaxM + t) * nseg + cc / G] = v;
      }
      __threadfence();
      __syncwarp();
      const int64_t row = rb * 32 + lane;  // lane l: row l of the group
      if (row < a.matrix_rows && atomicAdd(a.row_cnt + row, 1u) == (uint32_t)(nseg - 1)) {
        __threadfence();
        for (int t = 0; t < a.m; ++t) {
          // the row's partials for token t are contiguous: loaded four at a
          // time when they can be, added in chunk order
          const float* pt = a.part + (row * kDotMaxM + t) * nseg;
          float y = 0.f;
          int q = 0;
          if ((nseg & 3) == 0)
            for (; q < nseg; q += 4) {
              const float4 v = __ldcg(reinterpret_cast<const float4*>(pt + q));
              y = y + v.x + v.y + v.z + v.w;
            }
          for (; q < nseg; ++q) y += __ldcg(pt + q);
          const int64_t o = (int64_t)t * a.matrix_rows + row;
          if (a.out_f32)
            static_cast<float*>(a.y)[o] = y;
          else
            static_cast<uint16_t*>(a.y)[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
        }
        a.row_cnt[row] = 0u;
      }
      __syncwarp();
    }
  }
}

template <typename F>
cudaError_t set_attrs(F* f, size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  // the smallest shared-memory split that holds the CTA leaves L1 the rest
  const int pct = (int)((100 * (smem + 1024) + 228 * 1024 - 1) / (228 * 1024));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, pct);
  return e;
}

}  // namespace

// The longest run (a divisor of cpr) that still leaves about 24 runs per SM,
// so a launch keeps its warps busy in one pass.
int dot_run_length(int64_t N, int64_t cpr, int sms) {
  const int64_t groups = (N + 31) / 32 * cpr;
  int best = 1;
  for (int G = 2; G <= 8 && G <= cpr; ++G)
    if (cpr % G == 0 && groups / G >= (int64_t)sms * 24) best = G;
  return best;
}

bool dot_supported(int64_t K, int64_t chunk_syms, int64_t M) {
  return chunk_syms > 0 && K % chunk_syms == 0 && M >= 1 && M <= kDotMaxM;
}

// Launch shape: one CTA per SM (capped at `sms`) with W warps, a warp decoding
// 32 chunks per pass.  A pass takes about as long as the SM's warps share its
// issue slots, so W is chosen in [16, 32] to minimise passes x W (the last
// pass nearly full); a problem too small to give every SM 16 warps spreads
// over more SMs with fewer warps instead.
void decode_launch_shape(int64_t n_chunks, int sms, int* ctas, int* warps, int max_w) {
  const int64_t groups = (n_chunks + 31) / 32;
  if (sms < 1) sms = 1;
  if (groups <= (int64_t)sms * kMinWarps) {
    const int64_t w = groups <= sms ? 1 : (groups + sms - 1) / sms;
    *warps = (int)w;
    *ctas = (int)((groups + w - 1) / w);
    return;
  }
  int best_w = max_w;
  int64_t best_cost = -1;
  for (int w = max_w; w >= kMinWarps; --w) {
    const int64_t per = (int64_t)sms * w;
    const int64_t cost = (groups + per - 1) / per * w;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_w = w;
    }
  }
  *warps = best_w;
  *ctas = sms;
}

int decode_ctas_needed(int64_t n_chunks) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int ctas = 0, warps = 0;
  decode_launch_shape(n_chunks, sms, &ctas, &warps);
  return ctas;
}

cudaError_t launch_decode(int mode, const DecodeArgs& a, void* out, int ctas, cudaStream_t s) {
  if (a.n_chunks <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (ctas > 0 && ctas < sms) sms = ctas;  // an SM budget (decoder/GEMM split)
  int grid = 0, warps = 0;
  // (the product's work items are its runs)
  decode_launch_shape(mode == kDecodeDot ? (a.matrix_rows + 31) / 32 * a.cpr / a.run * 32 : a.n_chunks,
                      sms, &grid, &warps, mode == kDecodeDot ? kDotMaxWarps : kMaxWarps);
  const size_t smem = smem_bytes(warps, mode);
  const dim3 block(32 * warps);
  switch (mode) {
    case kDecodeDot: {
      if (a.rows || !a.x || !a.y || !a.part || !a.row_cnt || a.m < 1 || a.m > kDotMaxM ||
          a.run < 1 || a.cpr % a.run)
        return cudaErrorInvalidValue;
      e = set_attrs(decode_kernel<kDecodeDot, false>, smem);
      if (e == cudaSuccess)
        e = launch_pdl(decode_kernel<kDecodeDot, false>, grid, block, smem, s, a, out);
      break;
    }
    case kDecodeExp:
      if (a.rows) return cudaErrorInvalidValue;
      e = set_attrs(decode_kernel<kDecodeExp, false>, smem);
      if (e == cudaSuccess) e = launch_pdl(decode_kernel<kDecodeExp, false>, grid, block, smem, s, a, out);
      break;
    case kDecodeFull:
      if (a.rows) {
        e = set_attrs(decode_kernel<kDecodeFull, true>, smem);
        if (e == cudaSuccess)
          e = launch_pdl(decode_kernel<kDecodeFull, true>, grid, block, smem, s, a, out);
      } else {
        e = set_attrs(decode_kernel<kDecodeFull, false>, smem);
        if (e == cudaSuccess)
          e = launch_pdl(decode_kernel<kDecodeFull, false>, grid, block, smem, s, a, out);
      }
      break;
    case kDecodePalette:
      if (a.rows) return cudaErrorInvalidValue;
      e = set_attrs(decode_kernel<kDecodePalette, false>, smem);
      if (e == cudaSuccess) e = launch_pdl(decode_kernel<kDecodePalette, false>, grid, block, smem, s, a, out);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace uw
