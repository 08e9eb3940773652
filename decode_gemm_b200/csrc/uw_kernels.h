// Kernel launch interfaces (device code lives in decode.cu and gemm.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

namespace uw {

// Limit of every bounded wait inside a kernel (UW_WAIT_LIMIT_MS, default 2 s);
// a wait that runs out sets the timeout status and the kernel returns.
inline uint64_t wait_limit_ns() {
  static const uint64_t ns = [] {
    const char* s = std::getenv("UW_WAIT_LIMIT_MS");
    const long long ms = s ? std::atoll(s) : 2000;
    return (uint64_t)(ms > 0 ? ms : 2000) * 1000000ull;
  }();
  return ns;
}

// kDecodeDot: the Huffman-direct matrix-vector product (no decoded weights
// leave the chip; see DecodeArgs' product fields).
enum DecodeMode { kDecodeExp = 0, kDecodeFull = 1, kDecodePalette = 2, kDecodeDot = 3 };

// Zero words that follow the Huffman stream in device memory: a lane decoding
// a chunk reads at most 12 bits per symbol past the chunk's start plus a
// four-word window, so every read of a chunk whose start lies inside the
// stream stays inside the padded buffer.
inline int64_t stream_pad_words(int64_t chunk_syms) { return 3 * chunk_syms / 8 + 8; }

// Everything a decode/transcode launch reads, as device pointers.
struct DecodeArgs {
  const uint32_t* words;      // Huffman stream: n_words (a multiple of 4) words,
                              // then stream_pad_words(chunk_syms) zero words
  const uint32_t* chunk_off;  // n_chunks + 1 bit offsets
  const uint32_t* lut;        // 4096-entry rank table (see DecodeTables)
  const uint32_t* canon;      // canonical-code tables (kCanonWords words)
  uint32_t palette[4];        // the 16 palette exponents, byte i = rank i
  uint32_t pal_run_b4;        // palette = the run b..b+15: b in every byte, else 0xFFFFFFFF
  const uint8_t* sm;          // sign+mantissa bytes (full decode and product)
  const uint32_t* esc_bits;   // escape bitmap (palette transcode only)
  uint32_t* status;           // device status word (bit 0: bad chunk)
  int64_t n_words;
  int64_t n_chunks;
  int64_t total_syms;         // N*K
  int32_t chunk_syms;
  int32_t kb_per_row;         // K / 64
  int32_t esc_nw;             // escape-bitmap words per K block: 4*ceil(N/128)
  // Row gather (full decode only): decode the rows rows[0 .. gather_rows-1] of
  // the matrix into consecutive output rows.  Chunk v of the launch (n_chunks =
  // gather_rows * cpr, total_syms = gather_rows * K) is chunk v % cpr of row
  // rows[v / cpr]; needs K % chunk_syms == 0 (cpr = K / chunk_syms).
  const int64_t* rows = nullptr;
  int64_t gather_rows = 0;
  int64_t matrix_rows = 0;    // N
  int32_t cpr = 0;
  // Huffman-direct product (kDecodeDot): Y[t, n] = sum_k X[t, k] W[n, k] for
  // t < m, computed while the stream decodes; needs K % chunk_syms == 0 and
  // cpr = K / chunk_syms.  A warp's group is 32 rows at one chunk position
  // (one column range); a warp takes runs of `run` groups (consecutive
  // positions of the same rows, run divides cpr), and each (row, run) leaves
  // m FP32 partial sums at part[(row * kDotMaxM + t) * (cpr / run) + segment];
  // the run that brings a row's last partial (row_cnt, zero between
  // launches) adds them in segment order and writes Y (BF16 or FP32, [m, N]).
  const uint16_t* x = nullptr;  // X [m, K] BF16, rows 16-byte aligned
  void* y = nullptr;
  int32_t m = 0;
  int32_t out_f32 = 0;
  float* part = nullptr;
  uint32_t* row_cnt = nullptr;
  int32_t run = 1;
};

constexpr int kDotMaxM = 8;
// Whether the product serves (K, chunk_syms, M): rows are whole chunks and
// 1 <= M <= kDotMaxM.
bool dot_supported(int64_t K, int64_t chunk_syms, int64_t M);
// Chunk positions per run of the product for an N x (cpr chunks) matrix on
// `sms` SMs (decode.cu).
int dot_run_length(int64_t N, int64_t cpr, int sms);
// Partial-sum floats of a Huffman-direct launch over n_chunks chunks.
inline int64_t dot_part_floats(int64_t n_chunks) { return n_chunks * kDotMaxM; }

// Decode/transcode every chunk into `out` (layout per mode: BF16 [N*K],
// exponent bytes [N*K], packed nibbles [N*K/2]).  ctas > 0 caps the SMs the
// launch may use (one CTA per SM); ctas <= 0: all of them.  Returns the
// launch error.
cudaError_t launch_decode(int mode, const DecodeArgs& a, void* out, int ctas, cudaStream_t s);
int decode_ctas_needed(int64_t n_chunks);
// CTAs and warps per CTA (at most max_w) of a decode over n_chunks chunks on
// `sms` SMs.
void decode_launch_shape(int64_t n_chunks, int sms, int* ctas, int* warps, int max_w = 32);

// Device status bits.
constexpr uint32_t kStatusBadChunk = 1u;
constexpr uint32_t kStatusTimeout = 2u;

}  // namespace uw

namespace uw {

// Reconstructive / plain GEMM: Y[M, N] = X[M, K] * W^T.
enum GemmMode { kGemmBf16 = 0, kGemmExp = 1, kGemmPalette = 2 };

// Most persistent CTAs a GEMM launch may use, and the words of the per-handle
// split-K hand-off block: [0] launch epoch, [1] CTAs that have exited, then
// one ready flag per CTA (see launch_gemm).  The block starts zeroed.
constexpr int kGemmMaxCtas = 1024;
constexpr int kGemmSyncWords = 2 + kGemmMaxCtas;

struct GemmArgs {
  int mode = kGemmBf16;
  int64_t M = 0, N = 0, K = 0;
  const uint16_t* X = nullptr;   // [M, K] bf16
  const uint16_t* W = nullptr;   // [N, K] bf16 (kGemmBf16)
  const uint8_t* S = nullptr;    // [N, K] sign+mantissa (kGemmExp, kGemmPalette)
  const uint8_t* E = nullptr;    // [N, K] exponents (kGemmExp)
  const uint8_t* I = nullptr;    // [N, K/2] packed palette indices (kGemmPalette)
  int w1_resident = 0;           // I is the handle's resident array (not a kernel's output)
  const uint32_t* esc_bits = nullptr;
  const uint32_t* esc_off = nullptr;
  const uint8_t* esc_exp = nullptr;
  const uint8_t* esc_pack = nullptr;   // per group: bitmap then rows (see handle)
  int32_t esc_nw = 0;
  uint8_t palette[16] = {0};
  void* Y = nullptr;             // [M, N] bf16 or f32
  int out_f32 = 0;
  float* partials = nullptr;     // workspace for split partial sums
  size_t partials_bytes = 0;
  uint32_t* sync = nullptr;      // kGemmSyncWords words, zeroed before first use
  int tile_n = 0;                // tokens per tile (0 = auto)
  int halves = 0;                // W rows per unit / 128: 1, 2 (wide), 0 = auto by M
  int stages = 0;                // load ring depth (0 = auto)
  int wslots = 0;                // rebuilt-W ring depth (0 = auto)
  int ks = 0;                    // resolved: 64-wide K blocks per unit (stage)
  int xstages = 0;               // resolved: X ring depth
  int y_tma = 0;                 // resolved: BF16 Y through TMA stores
  int tmem_w = 0;                // resolved: W rebuilt into TMEM (else shared memory)
  int pair = 0;                  // CTA pairs with two-SM MMAs: 1 on, -1 off, 0 automatic;
                                 // resolved to 1 or 0
  int ctas = 0;                  // persistent CTAs (0 = SM count)
  int sm_count = 148;
  uint32_t* status = nullptr;
};

// Optional launch hooks (kernel tracing): begin(ctx, kind) returns a slot that
// end(ctx, slot) closes; kinds follow uw_kernel_kind.
struct LaunchHooks {
  void* ctx = nullptr;
  int (*begin)(void* ctx, int kind) = nullptr;
  void (*end)(void* ctx, int slot) = nullptr;
};

// Matrix-vector kernel on the CUDA cores for M <= kGemvMaxM tokens (gemv.cu):
// the same arguments as the GEMM (mode, M, N, K, X, the weight arrays of the
// mode, escape data, palette, Y, out_f32, w1_resident); no partial sums, no
// workspace of its own.  Traced as kinds 7 (BF16), 8 (exponent), 9 (palette).
constexpr int kGemvMaxM = 2;
bool gemv_supported(const GemmArgs& a);
cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t s, const LaunchHooks* hooks = nullptr);

// Fill in automatic tile_n / stages / ctas; returns false for unsupported shapes.
bool gemm_resolve(GemmArgs* a);
size_t gemm_partials_bytes(const GemmArgs& a);  // after gemm_resolve
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, const LaunchHooks* hooks = nullptr);

}  // namespace uw
