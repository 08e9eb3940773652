// Plain and reconstructive BF16 GEMM for sm_100a (tcgen05 + TMA + TMEM).
//
// *Unweight*, "How the reconstructive matmul works": a producer stages the
// compressed inputs (sign+mantissa bytes, exponent bytes or palette indices,
// and the verbatim exponent rows of escape rows) into a ring buffer in shared
// memory with the TMA; consumers rebuild BF16 weights in shared memory and feed
// them straight to the tensor cores, so rebuilt weights never reach HBM.
// "Four ways to use compressed weights": the same kernel with the weight tile
// loaded as BF16 is the plain GEMM of pipeline 1.
//
// B200 design (the post's kernel targets H100 WGMMA; this one is new):
//   * Swap-AB: the MMA's M side is 128 rows of W, its N side is a tile of
//     tile_n tokens (16..256), so a batch of 1 wastes no weight bandwidth.
//   * tcgen05.mma (kind::f16, BF16 x BF16 -> FP32) issued by one thread,
//     accumulating in TMEM; two accumulators so the epilogue of one output
//     tile overlaps the main loop of the next.
//   * Warp roles: warp 0 TMA producer, warp 1 MMA issuer (and TMEM owner),
//     warps 2-5 epilogue (TMEM -> registers -> global), warps 6-13 rebuild
//     (reconstructive modes only).
//   * Rebuild: 8 weights per 16-byte store into the 128-byte-swizzled K-major
//     layout the MMA descriptor expects; palette lookup is three byte permutes
//     per 4 weights; the escape decision is taken once per 64-weight row from a
//     16-byte bitmap staged with the tile.
//   * Persistent CTAs split the flattened (output tile, K block) space evenly
//     (stream-K); tiles shared by two CTAs are finished by a small fix-up kernel
//     that adds the partial sums in K order, so results are deterministic.
//   * Every mbarrier wait is bounded in wall time; on expiry the kernel records
//     a timeout in the status word, drains its MMAs and copies, frees TMEM and
//     returns.
//   * No cluster multicast anywhere.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bf16_fields.cuh"
#include "gemm_sm100.cuh"
#include "uw_kernels.h"

namespace uw {

namespace {

using namespace sm100;

constexpr int kBM = 128;           // W rows per tile (MMA M)
constexpr int kBK = 64;            // K per stage: one 128-byte swizzle row of BF16
constexpr int kWTileBytes = kBM * kBK * 2;
constexpr int kEscCap = 32;        // escape rows staged per stage (more: read from global)
constexpr int kWSlots = 2;         // rebuilt-W ring depth
constexpr int kNumEpiWarps = 4;
constexpr int kNumRebuildWarps = 8;
constexpr int kEpiWarp0 = 2;
constexpr int kRebuildWarp0 = kEpiWarp0 + kNumEpiWarps;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block

__host__ __device__ constexpr int threads_for(int mode) {
  return (mode == kGemmBf16 ? kRebuildWarp0 : kRebuildWarp0 + kNumRebuildWarps) * 32;
}

struct GemmParams {
  CUtensorMap tm_x;   // X [M, K] bf16, box {64, tile_n}, 128B swizzle
  CUtensorMap tm_w0;  // bf16 mode: W [N, K] box {64, 128} 128B swizzle; else S [N, K] u8 box {64,128}
  CUtensorMap tm_w1;  // exp mode: E [N, K] u8 box {64, 128}; palette mode: I [N, K/2] u8 box {32, 128}
  const uint32_t* esc_bits;
  const uint32_t* esc_off;
  const uint8_t* esc_exp;
  void* Y;
  float* partials;
  uint32_t* status;
  int64_t M, N, K;
  int64_t units;      // output tiles * K blocks
  int32_t tile_n, stages, NT, MT, KB, esc_nwp, out_f32, tmem_cols;
  uint32_t palette[4];
  uint32_t stage_bytes, x_bytes;
  uint64_t wait_ns;
};

// Per-stage shared-memory layout, offsets from the stage base.
struct StageLayout {
  uint32_t x, w0, w1, ebits, erows, bytes;
};

__host__ __device__ inline StageLayout stage_layout(int mode, int tile_n) {
  StageLayout L;
  L.x = 0;
  const uint32_t xb = (uint32_t)tile_n * kBK * 2;  // multiple of 2048 for tile_n % 16 == 0
  L.w0 = xb;
  if (mode == kGemmBf16) {
    L.w1 = L.ebits = L.erows = xb + kWTileBytes;
    L.bytes = xb + kWTileBytes;
  } else if (mode == kGemmExp) {
    L.w1 = xb + 8192;
    L.ebits = L.erows = xb + 16384;
    L.bytes = xb + 16384;
  } else {
    L.w1 = xb + 8192;
    L.ebits = xb + 12288;
    L.erows = xb + 12288 + 128;
    L.bytes = xb + 12288 + 128 + kEscCap * 64;
  }
  L.bytes = (L.bytes + 1023) / 1024 * 1024;
  return L;
}

// Segment of the flattened (tile, K block) space owned by one CTA.
__device__ __forceinline__ int64_t unit_begin(int64_t cta, int64_t units, int64_t G) {
  return cta * units / G;
}
__device__ __forceinline__ int64_t unit_owner(int64_t u, int64_t units, int64_t G) {
  return ((u + 1) * G - 1) / units;
}

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ void set_abort(volatile int* abort, uint32_t* status) {
  if (!*abort) {
    *abort = 1;
    atomicOr(status, kStatusTimeout);
  }
}

template <int MODE>
__global__ void __launch_bounds__(threads_for(MODE), 1)
    gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const StageLayout L = stage_layout(MODE, p.tile_n);
  const int S = p.stages;
  uint8_t* ring = smem;
  uint8_t* wring = ring + (size_t)S * L.bytes;  // rebuilt W tiles (reconstructive modes)
  uint8_t* tail = wring + (MODE == kGemmBf16 ? 0 : kWSlots * kWTileBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  // barrier indices
  const int b_full = 0, b_empty = S, b_wfull = 2 * S, b_wfree = 2 * S + kWSlots,
            b_tfull = 2 * S + 2 * kWSlots, b_tempty = b_tfull + 2, b_drain = b_tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + b_drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(b_full + s), 1);
      mbar_init(bar(b_empty + s), 1 + (MODE == kGemmBf16 ? 0 : kNumRebuildWarps));
    }
    for (int w = 0; w < kWSlots; ++w) {
      mbar_init(bar(b_wfull + w), kNumRebuildWarps);
      mbar_init(bar(b_wfree + w), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(b_tfull + a), 1);
      mbar_init(bar(b_tempty + a), kNumEpiWarps);
    }
    mbar_init(bar(b_drain), 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.tm_x);
    prefetch_tensormap(&p.tm_w0);
    if (MODE != kGemmBf16) prefetch_tensormap(&p.tm_w1);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t G = gridDim.x;
  const int64_t u0 = unit_begin(blockIdx.x, p.units, G);
  const int64_t u1 = unit_begin(blockIdx.x + 1, p.units, G);
  const int KB = p.KB;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok;) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const int64_t nt = t / p.MT, mt = t - nt * p.MT;
      const int32_t n0 = (int32_t)(nt * kBM), m0 = (int32_t)(mt * p.tile_n);
      // escape-row offsets of this tile's groups, 31 at a time in lanes
      int win0 = kb0;
      uint32_t eoff = 0;
      if (MODE == kGemmPalette) {
        const int64_t gi = nt * KB + win0 + lane;
        eoff = gi <= (int64_t)p.NT * KB ? __ldg(p.esc_off + gi) : 0u;
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        uint32_t c0 = 0, c1 = 0;
        if (MODE == kGemmPalette) {
          if (kb - win0 + 1 > 31) {
            win0 = kb;
            const int64_t gi = nt * KB + win0 + lane;
            eoff = gi <= (int64_t)p.NT * KB ? __ldg(p.esc_off + gi) : 0u;
          }
          c0 = __shfl_sync(0xffffffffu, eoff, kb - win0);
          c1 = __shfl_sync(0xffffffffu, eoff, kb - win0 + 1);
        }
        if (lane == 0) {
          if (!mbar_wait_bounded(bar(b_empty + stage), phase ^ 1u, abort, p.wait_ns)) {
            set_abort(abort, p.status);
            ok = false;
          } else {
            uint8_t* st = ring + (size_t)stage * L.bytes;
            const uint32_t fb = bar(b_full + stage);
            uint32_t bytes = p.x_bytes;
            uint32_t nesc = 0;
            if (MODE == kGemmBf16) bytes += kWTileBytes;
            if (MODE == kGemmExp) bytes += 16384;
            if (MODE == kGemmPalette) {
              nesc = min(c1 - c0, (uint32_t)kEscCap);
              bytes += 8192 + 4096 + 16 + nesc * 64;
            }
            mbar_expect_tx(fb, bytes);
            tma_load_2d(smem_u32(st + L.x), &p.tm_x, fb, kb * kBK, m0);
            tma_load_2d(smem_u32(st + L.w0), &p.tm_w0, fb, kb * kBK, n0);
            if (MODE == kGemmExp) tma_load_2d(smem_u32(st + L.w1), &p.tm_w1, fb, kb * kBK, n0);
            if (MODE == kGemmPalette) {
              tma_load_2d(smem_u32(st + L.w1), &p.tm_w1, fb, kb * (kBK / 2), n0);
              bulk_load(smem_u32(st + L.ebits), p.esc_bits + (int64_t)kb * p.esc_nwp + nt * 4, 16,
                        fb);
              if (nesc)
                bulk_load(smem_u32(st + L.erows), p.esc_exp + (int64_t)c0 * 64, nesc * 64, fb);
            }
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      u += kb1 - kb0;
    }
    // in-flight copies must land before the CTA exits
    if (lane == 0 && *abort) {
      const int64_t outstanding = issued < S ? issued : S;
      int s = stage;
      uint32_t ph = phase;
      for (int64_t i = 0; i < outstanding; ++i) {
        if (--s < 0) {
          s = S - 1;
          ph ^= 1u;
        }
        volatile int no_abort = 0;
        mbar_wait_bounded(bar(b_full + s), ph, &no_abort, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    const uint32_t idesc = idesc_bf16(kBM, p.tile_n);
    int stage = 0, wslot = 0;
    uint32_t phase = 0, wphase = 0;
    int seg = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++seg) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const int acc = seg & 1;
      const uint32_t acc_phase = (uint32_t)(seg >> 1) & 1u;
      if (lane == 0 &&
          !mbar_wait_bounded(bar(b_tempty + acc), acc_phase ^ 1u, abort, p.wait_ns)) {
        set_abort(abort, p.status);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.tile_n);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (lane == 0) {
          bool got = mbar_wait_bounded(bar(b_full + stage), phase, abort, p.wait_ns);
          if (got && MODE != kGemmBf16)
            got = mbar_wait_bounded(bar(b_wfull + wslot), wphase, abort, p.wait_ns);
          if (!got) {
            set_abort(abort, p.status);
            ok = false;
          } else {
            tc_fence_after();
            uint8_t* st = ring + (size_t)stage * L.bytes;
            const uint32_t a_addr =
                MODE == kGemmBf16 ? smem_u32(st + L.w0) : smem_u32(wring + wslot * kWTileBytes);
            const uint64_t a_desc = smem_desc_sw128(a_addr);
            const uint64_t b_desc = smem_desc_sw128(smem_u32(st + L.x));
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              mma_bf16(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc,
                       (kb > kb0 || k > 0) ? 1u : 0u);
            mma_commit(bar(b_empty + stage));
            if (MODE != kGemmBf16) mma_commit(bar(b_wfree + wslot));
            if (kb == kb1 - 1) mma_commit(bar(b_tfull + acc));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
        if (MODE != kGemmBf16 && ++wslot == kWSlots) {
          wslot = 0;
          wphase ^= 1u;
        }
      }
      u += kb1 - kb0;
    }
    // every issued MMA completes before TMEM is released
    if (lane == 0) {
      mma_commit(bar(b_drain));
      volatile int no_abort = 0;
      mbar_wait_bounded(bar(b_drain), 0, &no_abort, p.wait_ns);
    }
    __syncwarp();
  } else if (warp < kRebuildWarp0) {
    // ------------------------------------------------------------ epilogue --
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    int seg = 0;
    for (int64_t u = u0; u < u1; ++seg) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const bool full = kb0 == 0 && kb1 == KB;
      const int slot = (u == u0) ? 0 : 1;
      const int acc = seg & 1;
      const uint32_t acc_phase = (uint32_t)(seg >> 1) & 1u;
      // every lane observes the accumulator barrier before reading TMEM
      const bool got = mbar_wait_bounded(bar(b_tfull + acc), acc_phase, abort, p.wait_ns);
      if (!got) set_abort(abort, p.status);
      if (__any_sync(0xffffffffu, !got)) break;
      tc_fence_after();
      const int64_t nt = t / p.MT, mt = t - nt * p.MT;
      const int64_t n = nt * kBM + row;
      const int64_t m0 = mt * p.tile_n;
      const int cols = (int)imin64(p.tile_n, p.M - m0);
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * p.tile_n);
      float* part = p.partials + ((int64_t)blockIdx.x * 2 + slot) * (int64_t)p.tile_n * kBM;
      for (int c = 0; c < cols; c += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + (uint32_t)c, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (c + j < cols) {
            const float v = __uint_as_float(r[j]);
            if (full) {
              if (n < p.N) {
                const int64_t o = (m0 + c + j) * p.N + n;
                if (p.out_f32)
                  static_cast<float*>(p.Y)[o] = v;
                else
                  static_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(v);
              }
            } else {
              part[(int64_t)(c + j) * kBM + row] = v;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(b_tempty + acc));
      u += kb1 - kb0;
    }
  } else {
    // ------------------------------------------------------------- rebuild --
    const int rt = threadIdx.x - kRebuildWarp0 * 32;  // 0..255
    int stage = 0, wslot = 0;
    uint32_t phase = 0, wphase = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok;) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const int64_t nt = t / p.MT;
      for (int kb = kb0; kb < kb1; ++kb) {
        // every thread observes the stage's TMA completion before reading it
        const bool got = mbar_wait_bounded(bar(b_full + stage), phase, abort, p.wait_ns) &&
                         mbar_wait_bounded(bar(b_wfree + wslot), wphase ^ 1u, abort, p.wait_ns);
        if (!got) set_abort(abort, p.status);
        ok = !__any_sync(0xffffffffu, !got);
        if (!ok) break;
        const uint8_t* st = ring + (size_t)stage * L.bytes;
        uint8_t* wt = wring + wslot * kWTileBytes;
        const uint32_t* ebits = reinterpret_cast<const uint32_t*>(st + L.ebits);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q = rt + 256 * i;
          const int r = q >> 3, c = q & 7;
          const uint2 s8 = *reinterpret_cast<const uint2*>(st + L.w0 + r * 64 + c * 8);
          uint2 e8;
          if (MODE == kGemmExp) {
            e8 = *reinterpret_cast<const uint2*>(st + L.w1 + r * 64 + c * 8);
          } else {
            const uint32_t word = ebits[r >> 5];
            if ((word >> (r & 31)) & 1u) {
              // escape row: verbatim exponents, decided once for the row
              uint32_t slot = (uint32_t)__popc(word & ((1u << (r & 31)) - 1u));
              for (int w = 0; w < (r >> 5); ++w) slot += (uint32_t)__popc(ebits[w]);
              if (slot < (uint32_t)kEscCap) {
                e8 = *reinterpret_cast<const uint2*>(st + L.erows + slot * 64 + c * 8);
              } else {
                const uint32_t first = __ldg(p.esc_off + nt * KB + kb);
                e8 = __ldg(reinterpret_cast<const uint2*>(p.esc_exp + (int64_t)(first + slot) * 64 +
                                                          c * 8));
              }
            } else {
              const uint32_t v = *reinterpret_cast<const uint32_t*>(st + L.w1 + r * 32 + c * 4);
              e8.x = palette4(v & 0xFFFFu, p.palette[0], p.palette[1], p.palette[2], p.palette[3]);
              e8.y = palette4(v >> 16, p.palette[0], p.palette[1], p.palette[2], p.palette[3]);
            }
          }
          const uint2 lo = merge4(s8.x, e8.x);
          const uint2 hi = merge4(s8.y, e8.y);
          *reinterpret_cast<uint4*>(wt + r * 128 + ((c ^ (r & 7)) << 4)) =
              make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(b_wfull + wslot));
          mbar_arrive(bar(b_empty + stage));
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
        if (++wslot == kWSlots) {
          wslot = 0;
          wphase ^= 1u;
        }
      }
      u += kb1 - kb0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
  }
}

// Finish tiles whose K range was split between CTAs: add the partial sums in
// K order (CTA order) and write Y.
__global__ void __launch_bounds__(128) splitk_fixup_kernel(const __grid_constant__ GemmParams p,
                                                           int64_t G) {
  const int64_t t = blockIdx.x;
  const int64_t ua = t * p.KB, ub = ua + p.KB - 1;
  const int64_t i0 = unit_owner(ua, p.units, G), i1 = unit_owner(ub, p.units, G);
  if (i0 == i1) return;  // written by the GEMM itself
  const int row = threadIdx.x;
  const int64_t nt = t / p.MT, mt = t - nt * p.MT;
  const int64_t n = nt * kBM + row;
  const int64_t m0 = mt * p.tile_n;
  const int cols = (int)imin64(p.tile_n, p.M - m0);
  if (n >= p.N) return;
  for (int j = 0; j < cols; ++j) {
    float acc = 0.f;
    for (int64_t i = i0; i <= i1; ++i) {
      const int64_t s = unit_begin(i, p.units, G), e = unit_begin(i + 1, p.units, G);
      if (s == e) continue;
      const int slot = (s / p.KB == t) ? 0 : 1;  // first segment of CTA i, or its last
      acc += p.partials[((i * 2 + slot) * p.tile_n + j) * kBM + row];
    }
    const int64_t o = (m0 + j) * p.N + n;
    if (p.out_f32)
      static_cast<float*>(p.Y)[o] = acc;
    else
      static_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(acc);
  }
}

// ----------------------------------------------------------------- host ----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base,
                 uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                 bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint64_t wait_limit_ns() {
  static uint64_t ns = [] {
    const char* s = std::getenv("UW_WAIT_LIMIT_MS");
    const long long ms = s ? std::atoll(s) : 2000;
    return (uint64_t)(ms > 0 ? ms : 2000) * 1000000ull;
  }();
  return ns;
}

int tmem_cols_for(int tile_n) {
  int c = 32;
  while (c < 2 * tile_n) c *= 2;
  return c;
}

size_t smem_bytes(int mode, int tile_n, int stages) {
  const StageLayout L = stage_layout(mode, tile_n);
  size_t b = 1024 /* alignment slack */ + (size_t)stages * L.bytes;
  if (mode != kGemmBf16) b += kWSlots * kWTileBytes;
  b += (size_t)(2 * stages + 2 * kWSlots + 5) * 8 + 16;
  return b;
}

template <int MODE>
cudaError_t set_smem_attr() {
  static cudaError_t e = cudaFuncSetAttribute(
      gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  return e;
}

}  // namespace

bool gemm_resolve(GemmArgs* a) {
  if (a->M <= 0 || a->N <= 0 || a->K <= 0 || a->K % kBK) return false;
  if (a->tile_n == 0) {
    const int64_t mt = (a->M + 255) / 256;
    const int64_t per = (a->M + mt - 1) / mt;
    a->tile_n = (int)((per + 15) / 16 * 16);
  }
  if (a->tile_n < 16 || a->tile_n > 256 || a->tile_n % 16) return false;
  const int max_stages = 8;
  if (a->stages == 0) {
    int s = max_stages;
    while (s > 2 && smem_bytes(a->mode, a->tile_n, s) > (size_t)kSmemLimit) --s;
    a->stages = s;
  }
  if (a->stages < 2 || smem_bytes(a->mode, a->tile_n, a->stages) > (size_t)kSmemLimit)
    return false;
  const int64_t NT = (a->N + kBM - 1) / kBM;
  const int64_t MT = (a->M + a->tile_n - 1) / a->tile_n;
  const int64_t units = NT * MT * (a->K / kBK);
  int ctas = a->ctas > 0 ? a->ctas : a->sm_count;
  if ((int64_t)ctas > units) ctas = (int)units;
  a->ctas = ctas;
  return true;
}

size_t gemm_partials_bytes(const GemmArgs& a) {
  return (size_t)a.ctas * 2 * (size_t)a.tile_n * kBM * sizeof(float);
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, const LaunchHooks* hooks) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int64_t KB = a.K / kBK;
  if (!make_map_2d(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.X, (uint64_t)a.K,
                   (uint64_t)a.M, kBK, (uint32_t)a.tile_n, true))
    return cudaErrorInvalidValue;
  bool ok = true;
  if (a.mode == kGemmBf16) {
    ok = make_map_2d(&p.tm_w0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.W, (uint64_t)a.K,
                     (uint64_t)a.N, kBK, kBM, true);
  } else {
    ok = make_map_2d(&p.tm_w0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.S, (uint64_t)a.K,
                     (uint64_t)a.N, kBK, kBM, false);
    if (ok && a.mode == kGemmExp)
      ok = make_map_2d(&p.tm_w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.E, (uint64_t)a.K,
                       (uint64_t)a.N, kBK, kBM, false);
    if (ok && a.mode == kGemmPalette)
      ok = make_map_2d(&p.tm_w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.I, (uint64_t)a.K / 2,
                       (uint64_t)a.N, kBK / 2, kBM, false);
  }
  if (!ok) return cudaErrorInvalidValue;
  p.esc_bits = a.esc_bits;
  p.esc_off = a.esc_off;
  p.esc_exp = a.esc_exp;
  p.Y = a.Y;
  p.partials = a.partials;
  p.status = a.status;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.tile_n = a.tile_n;
  p.stages = a.stages;
  p.NT = (int32_t)((a.N + kBM - 1) / kBM);
  p.MT = (int32_t)((a.M + a.tile_n - 1) / a.tile_n);
  p.KB = (int32_t)KB;
  p.units = (int64_t)p.NT * p.MT * KB;
  p.esc_nwp = a.esc_nw;
  p.out_f32 = a.out_f32;
  p.tmem_cols = tmem_cols_for(a.tile_n);
  std::memcpy(p.palette, a.palette, 16);
  p.x_bytes = (uint32_t)a.tile_n * kBK * 2;
  p.stage_bytes = stage_layout(a.mode, a.tile_n).bytes;
  p.wait_ns = wait_limit_ns();
  const size_t smem = smem_bytes(a.mode, a.tile_n, a.stages);
  const int G = a.ctas;
  cudaError_t e = cudaSuccess;
  auto begin = [&](int kind) { return hooks && hooks->begin ? hooks->begin(hooks->ctx, kind) : -1; };
  auto end = [&](int slot) {
    if (hooks && hooks->end) hooks->end(hooks->ctx, slot);
  };
  // kinds: 3 bf16, 4 exponent, 5 palette GEMM; 6 fix-up
  const int slot = begin(3 + a.mode);
  switch (a.mode) {
    case kGemmBf16:
      if ((e = set_smem_attr<kGemmBf16>()) != cudaSuccess) return e;
      gemm_kernel<kGemmBf16><<<G, threads_for(kGemmBf16), smem, s>>>(p);
      break;
    case kGemmExp:
      if ((e = set_smem_attr<kGemmExp>()) != cudaSuccess) return e;
      gemm_kernel<kGemmExp><<<G, threads_for(kGemmExp), smem, s>>>(p);
      break;
    case kGemmPalette:
      if ((e = set_smem_attr<kGemmPalette>()) != cudaSuccess) return e;
      gemm_kernel<kGemmPalette><<<G, threads_for(kGemmPalette), smem, s>>>(p);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  end(slot);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // tiles split between CTAs get their sum here (only when some tile is split)
  if (p.units % G != 0 || (p.units / G) % KB != 0) {
    const int fs = begin(6);
    splitk_fixup_kernel<<<(unsigned)(p.NT * p.MT), kBM, 0, s>>>(p, G);
    end(fs);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace uw
