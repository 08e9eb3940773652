// Chunk-parallel Huffman decoder and palette transcoder for sm_100a.
//
// *Unweight*, "Four ways to use compressed weights": the preprocessing kernels
// of pipelines 1-3 (full decode to BF16, exponent-only decode, transcode to
// 4-bit palette indices).  "Sharing the GPU between decode and compute": the
// decoder works from a ~16 KB lookup table in shared memory.
//
// Design (B200):
//   * One lane decodes one chunk (chunk_syms symbols; chunks are independent
//     because their start bits are stored).  A warp owns 32 consecutive chunks.
//   * The 4096-entry table in shared memory maps the next 12 stream bits to up
//     to 3 exponents (or 6 palette indices) at once plus the bits they use, so
//     one lookup usually retires several symbols.  In the last few symbols of a
//     chunk the lane decodes one symbol per lookup (first-code length from the
//     canonical limits), so it stops exactly at the chunk's end bit, which is
//     checked against the stored offset.
//   * Each lane reads its stream with 16-byte loads, double buffered.
//   * Decoded rows of 64 symbols are staged per warp in shared memory and
//     written out so each 64-symbol row is one contiguous, fully used run of
//     32-byte sectors (full decode: sign+mantissa merged on the way out).
#include <cuda_runtime.h>

#include <cstdint>

#include "uw_kernels.h"

namespace uw {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kLut = 4096;

__device__ __forceinline__ uint4 ldg_u4(const uint4* p) { return __ldg(p); }

__device__ __forceinline__ uint32_t pick(const uint4& q, int i) {
  return i == 0 ? q.x : (i == 1 ? q.y : (i == 2 ? q.z : q.w));
}

// Merge 4 sign+mantissa bytes with 4 exponent bytes into 4 BF16 values.
__device__ __forceinline__ uint2 merge4(uint32_t s, uint32_t e) {
  const uint32_t hi = (s & 0x80808080u) | ((e >> 1) & 0x7F7F7F7Fu);  // sign | E[7:1]
  const uint32_t lo = ((e << 7) & 0x80808080u) | (s & 0x7F7F7F7Fu);  // E[0] | mantissa
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

template <int MODE>
struct ModeTraits;
template <>
struct ModeTraits<kDecodeExp> {
  static constexpr int kCap = 3, kValBits = 8, kRowWords = 16;
};
template <>
struct ModeTraits<kDecodeFull> {
  static constexpr int kCap = 3, kValBits = 8, kRowWords = 16;
};
template <>
struct ModeTraits<kDecodePalette> {
  static constexpr int kCap = 6, kValBits = 4, kRowWords = 8;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeArgs a, void* __restrict__ out) {
  using T = ModeTraits<MODE>;
  constexpr int kStride = T::kRowWords + 1;  // padded staging row (bank spread)
  extern __shared__ __align__(16) uint32_t smem[];
  uint32_t* lut = smem;
  uint32_t* limit = smem + kLut;
  uint32_t* stage_base = smem + kLut + 16;

  for (int i = threadIdx.x; i < kLut / 4; i += kThreads)
    reinterpret_cast<uint4*>(lut)[i] = ldg_u4(reinterpret_cast<const uint4*>(a.lut) + i);
  if (threadIdx.x < 16) limit[threadIdx.x] = a.limit[threadIdx.x];
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint32_t* stage = stage_base + warp * 32 * kStride;
  const int64_t groups = (a.n_chunks + 31) / 32;
  const int64_t n_words4 = a.n_words / 4;
  const uint4* words4 = reinterpret_cast<const uint4*>(a.words);
  const int cs = a.chunk_syms;

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
      const int64_t left = a.total_syms - c * (int64_t)cs;
      nsyms = (int)(left < cs ? left : cs);
    }
    const int my_rounds = nsyms / 64;
    const int warp_rounds = __reduce_max_sync(0xffffffffu, my_rounds);

    // bit reader: bb holds nb valid bits, most significant first
    int64_t g4 = (int64_t)(start >> 7);  // 16-byte group of the first word
    int qi = (int)((start >> 5) & 3);
    uint4 q = make_uint4(0, 0, 0, 0), qn = make_uint4(0, 0, 0, 0);
    if (live) {
      q = g4 < n_words4 ? ldg_u4(words4 + g4) : q;
      qn = g4 + 1 < n_words4 ? ldg_u4(words4 + g4 + 1) : qn;
    }
    const int drop = (int)(start & 31);
    uint64_t bb = (uint64_t)pick(q, qi) << (32 + drop);
    int nb = 32 - drop;
    if (++qi == 4) {
      qi = 0;
      ++g4;
      q = qn;
      qn = (live && g4 + 1 < n_words4) ? ldg_u4(words4 + g4 + 1) : make_uint4(0, 0, 0, 0);
    }

    uint64_t acc = 0;
    int acc_bits = 0;
    int remaining = nsyms;
    uint32_t consumed = 0;
    bool bad = false;

    for (int r = 0; r < warp_rounds; ++r) {
      // write-out operands fetched early so their latency hides behind decoding
      uint32_t pre[T::kRowWords];
      if constexpr (MODE == kDecodeFull) {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const int j = 2 * p + (lane >> 4), w = lane & 15;
          const int64_t cj = c0 + j;
          const int rj = __shfl_sync(0xffffffffu, my_rounds, j);
          pre[p] = (cj < a.n_chunks && r < rj)
                       ? __ldg(reinterpret_cast<const uint32_t*>(a.sm + cj * cs + r * 64) + w)
                       : 0u;
        }
      } else if constexpr (MODE == kDecodePalette) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int j = 4 * p + (lane >> 3);
          const int64_t cj = c0 + j;
          const int rj = __shfl_sync(0xffffffffu, my_rounds, j);
          uint32_t esc = 0;
          if (cj < a.n_chunks && r < rj) {
            const int64_t row = cj * (cs / 64) + r;
            const int64_t n = row / a.kb_per_row, kb = row % a.kb_per_row;
            esc = (__ldg(a.esc_bits + kb * a.esc_nw + (n >> 5)) >> (n & 31)) & 1u;
          }
          pre[p] = esc;
        }
      }

      if (r < my_rounds) {
        int filled = 0;
        while (filled < T::kRowWords) {
          if (nb <= 32) {
            bb |= (uint64_t)pick(q, qi) << (32 - nb);
            nb += 32;
            if (++qi == 4) {
              qi = 0;
              ++g4;
              q = qn;
              qn = g4 + 1 < n_words4 ? ldg_u4(words4 + g4 + 1) : make_uint4(0, 0, 0, 0);
            }
          }
          const uint32_t idx = (uint32_t)(bb >> 52);
          uint32_t e = lut[idx];
          uint32_t cnt = (e >> 24) & 7u;
          uint32_t len = e >> 28;
          if (cnt == 0) {  // not a code word: corrupt stream; keep going, report
            bad = true;
            cnt = 1;
            len = 1;
            e = 0;
          } else if (remaining < T::kCap) {
            // last symbols of the chunk: exactly one per lookup
            len = 1;
            while (len < 12 && idx >= limit[len]) ++len;
            cnt = 1;
            e &= (1u << T::kValBits) - 1u;
          }
          bb <<= len;
          nb -= (int)len;
          consumed += len;
          remaining -= (int)cnt;
          acc |= (uint64_t)(e & 0xFFFFFFu) << acc_bits;
          acc_bits += (int)cnt * T::kValBits;
          if (acc_bits >= 32) {
            stage[lane * kStride + filled] = (uint32_t)acc;
            acc >>= 32;
            acc_bits -= 32;
            ++filled;
          }
        }
      }
      __syncwarp();

      // coalesced write-out of the warp's 32 rows of 64 symbols
      if constexpr (MODE == kDecodeExp) {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const int j = 2 * p + (lane >> 4), w = lane & 15;
          const int64_t cj = c0 + j;
          const int rj = __shfl_sync(0xffffffffu, my_rounds, j);
          if (cj < a.n_chunks && r < rj)
            reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + cj * cs + r * 64)[w] =
                stage[j * kStride + w];
        }
      } else if constexpr (MODE == kDecodeFull) {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const int j = 2 * p + (lane >> 4), w = lane & 15;
          const int64_t cj = c0 + j;
          const int rj = __shfl_sync(0xffffffffu, my_rounds, j);
          if (cj < a.n_chunks && r < rj)
            reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + cj * cs + r * 64)[w] =
                merge4(pre[p], stage[j * kStride + w]);
        }
      } else {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int j = 4 * p + (lane >> 3), w = lane & 7;
          const int64_t cj = c0 + j;
          const int rj = __shfl_sync(0xffffffffu, my_rounds, j);
          if (cj < a.n_chunks && r < rj) {
            const int64_t row = cj * (cs / 64) + r;
            reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + row * 32)[w] =
                pre[p] ? 0u : stage[j * kStride + w];
          }
        }
      }
      __syncwarp();
    }
    if (live && (bad || consumed != end - start)) atomicOr(a.status, kStatusBadChunk);
  }
}

template <int MODE>
size_t decode_smem_bytes() {
  return (size_t)(kLut + 16 + kWarps * 32 * (ModeTraits<MODE>::kRowWords + 1)) * 4;
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
  switch (mode) {
    case kDecodeExp:
      decode_kernel<kDecodeExp><<<grid, kThreads, decode_smem_bytes<kDecodeExp>(), s>>>(a, out);
      break;
    case kDecodeFull:
      decode_kernel<kDecodeFull><<<grid, kThreads, decode_smem_bytes<kDecodeFull>(), s>>>(a, out);
      break;
    case kDecodePalette:
      decode_kernel<kDecodePalette>
          <<<grid, kThreads, decode_smem_bytes<kDecodePalette>(), s>>>(a, out);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace uw
