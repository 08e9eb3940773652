// Chunk-parallel Huffman decoder and palette transcoder for sm_100a.
//
// *Unweight*, "Four ways to use compressed weights": the preprocessing kernels
// of pipelines 1-3 (full decode to BF16, exponent-only decode, transcode to
// 4-bit palette indices).  "Sharing the GPU between decode and compute": the
// decoder works from a ~16 KB lookup table in shared memory.
//
// Design (B200):
//   * One lane decodes one chunk (its start bit is stored, so chunks are
//     independent); a warp owns 32 consecutive chunks; 16 warps share the
//     table in shared memory.
//   * The 4096-entry table maps the next 12 stream bits to up to 6 palette
//     ranks and the bits they use.  Every output derives from ranks: the
//     transcode writes them, the exponent and full decodes expand them through
//     the 16-entry palette with byte permutes.  A code for an exponent outside
//     the palette (rare; only inside escape rows) is a one-symbol "raw" entry:
//     the transcode writes rank 0 (the row is zeroed anyway); the other modes
//     record the exponent as a per-lane exception and patch it after the
//     coalesced write, or, when a lane's exception list overflows, replay the
//     whole chunk one symbol at a time.
//   * Bit buffer in two registers with funnel shifts; it is topped up 32 bits
//     at a time from 8-byte loads (next pair prefetched), once per two lookups.
//   * In the last few symbols of a chunk the lane decodes one symbol per lookup
//     (first-code length from the canonical limits) so it stops exactly at the
//     chunk's end bit, which is checked against the stored offset.
//   * Each lane stages 256 decoded symbols (4 rows of 64) in shared memory;
//     the warp then writes its 32 lanes' rows so each row is one contiguous,
//     fully used run of 32-byte sectors (full decode merges the sign+mantissa
//     bytes on the way out).
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "bf16_fields.cuh"
#include "uw_internal.h"
#include "uw_kernels.h"

namespace uw {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRoundSyms = 256;                 // symbols per lane per staging round
constexpr int kRoundWords = kRoundSyms / 8;     // 32 words of 4-bit ranks
constexpr int kStageStride = kRoundWords + 1;   // lanes spread over banks
constexpr int kExcCap = 8;                      // exceptions held per lane

struct __align__(16) Smem {
  uint32_t lut[kLutSize];
  uint32_t canon[kCanonWords];
  uint32_t stage[kWarps][32 * kStageStride];
  uint32_t exc[kWarps][32 * kExcCap];  // (chunk symbol index << 8) | exponent
};

struct Reader {
  uint32_t hi, lo;  // next stream bits, most significant first
  int nb;           // valid bits in hi:lo
  uint2 c, cn;      // current and next 8-byte stream words
  int ci;           // next word of c to use
  int64_t gi;       // index of the 8-byte group after cn
  int fed;          // 32-bit words fed into the buffer after the first
};

__device__ __forceinline__ uint2 ld_pair(const uint2* p, int64_t i, int64_t n) {
  return i < n ? __ldg(p + i) : make_uint2(0u, 0u);
}

__device__ __forceinline__ void reader_init(Reader& r, const uint2* src, int64_t ng,
                                            uint32_t start) {
  const int64_t g = start >> 6;
  r.c = ld_pair(src, g, ng);
  r.cn = ld_pair(src, g + 1, ng);
  r.gi = g + 2;
  r.ci = (int)((start >> 5) & 1);
  const uint32_t w = r.ci ? r.c.y : r.c.x;
  r.hi = w << (start & 31);
  r.lo = 0;
  r.nb = 32 - (int)(start & 31);
  r.fed = 0;
  if (r.ci) {
    r.c = r.cn;
    r.cn = ld_pair(src, r.gi++, ng);
    r.ci = 0;
  } else {
    r.ci = 1;
  }
}

// Top the buffer up with one 32-bit word when it holds 32 bits or fewer.
__device__ __forceinline__ void reader_refill(Reader& r, const uint2* src, int64_t ng) {
  if (r.nb <= 32) {
    const uint32_t w = r.ci ? r.c.y : r.c.x;
    r.hi |= __funnelshift_rc(w, 0u, (uint32_t)r.nb);          // w >> nb
    r.lo |= __funnelshift_lc(0u, w, (uint32_t)(32 - r.nb));   // w << (32 - nb)
    r.nb += 32;
    r.fed += 1;
    if (r.ci) {
      r.c = r.cn;
      r.cn = ld_pair(src, r.gi++, ng);
      r.ci = 0;
    } else {
      r.ci = 1;
    }
  }
}

// Stream bits consumed since reader_init(start).
__device__ __forceinline__ uint32_t reader_consumed(const Reader& r, uint32_t start) {
  return (uint32_t)(32 - (int)(start & 31) + 32 * r.fed - r.nb);
}

__device__ __forceinline__ void reader_consume(Reader& r, uint32_t len) {
  r.hi = __funnelshift_l(r.lo, r.hi, len);
  r.lo = __funnelshift_l(0u, r.lo, len);
  r.nb -= (int)len;
}

// Length of the code that starts the 12-bit window (canonical limits).
__device__ __forceinline__ uint32_t first_code_len(const uint32_t* canon, uint32_t idx) {
  uint32_t len = 1;
  while (len < 12 && idx >= canon[kCanonLimit + len]) ++len;
  return len;
}

// One symbol, one lookup at a time (slow path): returns the exponent.
__device__ __forceinline__ uint32_t slow_symbol(Reader& r, const uint2* src, int64_t ng,
                                                const uint32_t* canon) {
  reader_refill(r, src, ng);
  const uint32_t idx = r.hi >> 20;
  const uint32_t len = first_code_len(canon, idx);
  const uint32_t code = idx >> (12 - len);
  const uint32_t k = canon[kCanonOffset + len] + code - canon[kCanonFirst + len];
  const uint8_t* syms = reinterpret_cast<const uint8_t*>(canon + kCanonSymbols);
  reader_consume(r, len);
  return syms[k & 255];
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const DecodeArgs a, void* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  for (int i = threadIdx.x; i < kLutSize / 4; i += kThreads)
    reinterpret_cast<uint4*>(sm.lut)[i] = __ldg(reinterpret_cast<const uint4*>(a.lut) + i);
  for (int i = threadIdx.x; i < kCanonWords; i += kThreads) sm.canon[i] = __ldg(a.canon + i);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint32_t* stage = sm.stage[warp];
  uint32_t* exc = sm.exc[warp] + lane * kExcCap;
  const int64_t groups = (a.n_chunks + 31) / 32;
  const uint2* src = reinterpret_cast<const uint2*>(a.words);
  const int64_t ng = a.n_words / 2;
  const int64_t cs = a.chunk_syms;
  const int rows_per_chunk = (int)(cs / 64);
  const uint32_t p0 = a.palette[0], p1 = a.palette[1], p2 = a.palette[2], p3 = a.palette[3];

  for (int64_t grp = (int64_t)blockIdx.x * kWarps + warp; grp < groups;
       grp += (int64_t)gridDim.x * kWarps) {
    const int64_t c0 = grp * 32;
    const int64_t c = c0 + lane;
    const bool live = c < a.n_chunks;
    uint32_t start = 0, end = 0;
    int nsyms = 0;
    if (live) {
      start = a.chunk_off[c];
      end = a.chunk_off[c + 1];
      const int64_t left = a.total_syms - c * cs;
      nsyms = (int)(left < cs ? left : cs);
    }
    // (output row n, K block kb) of this chunk's first 64-symbol row
    int n0 = 0, kb0 = 0;
    if (MODE == kDecodePalette && live) {
      const int64_t row0 = c * rows_per_chunk;
      n0 = (int)(row0 / a.kb_per_row);
      kb0 = (int)(row0 - (int64_t)n0 * a.kb_per_row);
    }
    const int my_rounds = (nsyms + kRoundSyms - 1) / kRoundSyms;
    const int warp_rounds = __reduce_max_sync(0xffffffffu, my_rounds);

    Reader rd;
    reader_init(rd, src, live ? ng : 0, start);
    uint32_t a_lo = 0, a_hi = 0;  // ranks waiting to be staged (ab bits)
    int ab = 0;
    int nx = 0;
    bool bad = false, overflow = false;
    uint32_t* st = stage + lane * kStageStride;
    // rounds before every lane's last one cannot reach a chunk's end
    const int fast_rounds = __reduce_min_sync(0xffffffffu, my_rounds) - 1;

    for (int r = 0; r < warp_rounds; ++r) {
      const int rsyms = min(kRoundSyms, max(0, nsyms - r * kRoundSyms));
      const int rwords = rsyms / 8;
      int filled = 0;  // fewer than 32 bits (whole ranks) carry over between rounds
      // One lookup: decodes up to kPalCap ranks; TAIL selects the careful
      // variant that stops exactly at the chunk's last symbol.
      auto lookup = [&](auto tail_tag) {
        constexpr bool TAIL = decltype(tail_tag)::value;
        const uint32_t idx = rd.hi >> 20;
        uint32_t e = sm.lut[idx];
        uint32_t cnt = (e >> 24) & 7u;
        uint32_t len = e >> 28;
        int rem = kPalCap;
        if (TAIL) rem = nsyms - r * kRoundSyms - filled * 8 - (ab >> 2);
        if (cnt == 0u || (TAIL && rem < kPalCap)) {
          if (TAIL && rem <= 0) {  // chunk done (second lookup of a pair)
            cnt = 0;
            len = 0;
            e = 0;
          } else if (e & kLutRaw) {  // exponent outside the palette
            if (MODE != kDecodePalette) {
              const uint32_t pos = (uint32_t)(r * kRoundSyms + filled * 8 + (ab >> 2));
              if (nx < kExcCap)
                exc[nx++] = (pos << 8) | (e & 0xFFu);
              else
                overflow = true;
            }
            cnt = 1;
            e = 0;
          } else if (len == 0u) {  // no code starts here: corrupt stream
            bad = true;
            cnt = 1;
            len = 1;
            e = 0;
          } else {  // last symbols of the chunk: one at a time
            len = first_code_len(sm.canon, idx);
            cnt = 1;
            e &= 0xFu;
          }
        }
        reader_consume(rd, len);
        const uint32_t v = e & 0xFFFFFFu;
        a_lo |= v << ab;
        a_hi |= __funnelshift_l(v, 0u, (uint32_t)ab);
        ab += 4 * (int)cnt;
        if (ab >= 32 && filled < rwords) {
          st[filled++] = a_lo;
          a_lo = a_hi;
          a_hi = 0;
          ab -= 32;
        }
      };
      if (r < fast_rounds) {
        while (filled < rwords) {
          reader_refill(rd, src, ng);
          lookup(std::false_type());
          // a pair's second lookup only while the round still needs words, so
          // fewer than 32 bits are pending whenever ranks are appended
          if (filled < rwords) lookup(std::false_type());
        }
      } else {
        while (filled < rwords) {
          reader_refill(rd, src, ng);
          lookup(std::true_type());
          if (filled < rwords) lookup(std::true_type());
        }
      }
      __syncwarp();

      // coalesced write-out: row slot rs of each of the 32 lanes
#pragma unroll 1
      for (int rs = 0; rs < kRoundSyms / 64; ++rs) {
        // operands fetched for all 8 passes first so their latencies overlap
        uint2 pre[8];
        uint32_t okmask = 0;
        const int w = lane & 7;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int j = 4 * p + (lane >> 3);
          const int nj = __shfl_sync(0xffffffffu, nsyms, j);
          const bool ok = (c0 + j < a.n_chunks) && (r * kRoundSyms + rs * 64 < nj);
          okmask |= ok ? (1u << p) : 0u;
          const int64_t row = (c0 + j) * rows_per_chunk + r * (kRoundSyms / 64) + rs;
          pre[p] = make_uint2(0u, 0u);
          int n_j = 0, kb_j = 0;
          if (MODE == kDecodePalette) {
            n_j = __shfl_sync(0xffffffffu, n0, j);
            kb_j = __shfl_sync(0xffffffffu, kb0, j);
          }
          if (ok) {
            if (MODE == kDecodeFull) {
              pre[p] = __ldg(reinterpret_cast<const uint2*>(a.sm + row * 64) + w);
            } else if (MODE == kDecodePalette) {
              // (n, kb) of the row from lane j's chunk start, no division
              int n = n_j;
              int kb = kb_j + r * (kRoundSyms / 64) + rs;
              while (kb >= a.kb_per_row) {
                kb -= a.kb_per_row;
                ++n;
              }
              pre[p].x = (__ldg(a.esc_bits + (int64_t)kb * a.esc_nw + (n >> 5)) >> (n & 31)) & 1u;
            }
          }
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int j = 4 * p + (lane >> 3);
          if (!((okmask >> p) & 1u)) continue;
          const int64_t row = (c0 + j) * rows_per_chunk + r * (kRoundSyms / 64) + rs;
          const uint32_t word = stage[j * kStageStride + rs * 8 + w];
          if (MODE == kDecodePalette) {
            reinterpret_cast<uint32_t*>(out)[row * 8 + w] = pre[p].x ? 0u : word;
          } else {
            const uint32_t e0 = palette4(word & 0xFFFFu, p0, p1, p2, p3);
            const uint32_t e1 = palette4(word >> 16, p0, p1, p2, p3);
            if (MODE == kDecodeExp) {
              reinterpret_cast<uint2*>(out)[row * 8 + w] = make_uint2(e0, e1);
            } else {
              const uint2 lo = merge4(pre[p].x, e0), hi = merge4(pre[p].y, e1);
              reinterpret_cast<uint4*>(out)[row * 8 + w] = make_uint4(lo.x, lo.y, hi.x, hi.y);
            }
          }
        }
      }
      __syncwarp();

      // exceptions of this round overwrite the placeholder the bulk write left
      if (MODE != kDecodePalette && nx > 0) {
        const int64_t base = c * cs;
        const uint32_t lim = (uint32_t)((r + 1) * kRoundSyms);
        int keep = 0;
        for (int i = 0; i < nx; ++i) {
          const uint32_t x = exc[i];
          const uint32_t pos = x >> 8;
          if (pos < lim) {
            const int64_t o = base + pos;
            if (MODE == kDecodeExp) {
              static_cast<uint8_t*>(out)[o] = (uint8_t)(x & 0xFFu);
            } else {
              const uint32_t s = a.sm[o];
              const uint32_t ex = x & 0xFFu;
              static_cast<uint16_t*>(out)[o] =
                  (uint16_t)(((s & 0x80u) << 8) | (ex << 7) | (s & 0x7Fu));
            }
          } else {
            exc[keep++] = x;
          }
        }
        nx = keep;
      }
      __syncwarp();
    }

    // a lane whose exception list overflowed replays its chunk symbol by symbol
    if (MODE != kDecodePalette && overflow) {
      Reader sr;
      reader_init(sr, src, ng, start);
      const int64_t base = c * cs;
      for (int i = 0; i < nsyms; ++i) {
        const uint32_t ex = slow_symbol(sr, src, ng, sm.canon);
        if (MODE == kDecodeExp) {
          static_cast<uint8_t*>(out)[base + i] = (uint8_t)ex;
        } else {
          const uint32_t s = a.sm[base + i];
          static_cast<uint16_t*>(out)[base + i] =
              (uint16_t)(((s & 0x80u) << 8) | (ex << 7) | (s & 0x7Fu));
        }
      }
    }
    if (live && (bad || reader_consumed(rd, start) != end - start))
      atomicOr(a.status, kStatusBadChunk);
    __syncwarp();
  }
}

}  // namespace

int decode_ctas_needed(int64_t n_chunks) {
  const int64_t groups = (n_chunks + 31) / 32;
  return (int)((groups + kWarps - 1) / kWarps);
}

cudaError_t launch_decode(int mode, const DecodeArgs& a, void* out, int ctas, cudaStream_t s) {
  const int need = decode_ctas_needed(a.n_chunks);
  const int grid = (ctas > 0 && ctas < need) ? ctas : need;
  if (grid <= 0) return cudaSuccess;
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaSuccess;
  switch (mode) {
    case kDecodeExp:
      e = cudaFuncSetAttribute(decode_kernel<kDecodeExp>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) decode_kernel<kDecodeExp><<<grid, kThreads, smem, s>>>(a, out);
      break;
    case kDecodeFull:
      e = cudaFuncSetAttribute(decode_kernel<kDecodeFull>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) decode_kernel<kDecodeFull><<<grid, kThreads, smem, s>>>(a, out);
      break;
    case kDecodePalette:
      e = cudaFuncSetAttribute(decode_kernel<kDecodePalette>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) decode_kernel<kDecodePalette><<<grid, kThreads, smem, s>>>(a, out);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace uw
