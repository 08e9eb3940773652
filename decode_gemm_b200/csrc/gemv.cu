// Matrix-vector products (M <= 2 tokens) on the CUDA cores, for all four
// pipelines' weight forms: BF16 (pipeline 1), sign+mantissa and exponent bytes
// (pipeline 2), sign+mantissa bytes and 4-bit palette indices with escape rows
// (pipelines 3 and 4).
//
// *Unweight*, "How the reconstructive matmul works": the weights are rebuilt
// from their compressed form on chip and never reach main memory in BF16.
// "The GPU memory bottleneck": at batch 1 the matmul is bound by the bytes of
// the weights.  At one or two tokens every weight takes part in one or two
// multiply-adds, so the tensor cores have nothing to gain and the MMA path's
// fixed costs (TMEM, rebuilt tiles in shared memory, 16-wide MMAs of which
// 15/16 are padding) only slow it down; here each weight is rebuilt in
// registers and multiplied on the CUDA cores, and the kernel streams the
// compressed bytes once, with 128-bit loads that do not allocate in L1.
//
// Layout of the work: a CTA owns a run of rows; a work item is one row and one
// segment of 1024 weights along K (32 consecutive weights per lane); 16 warps
// take items in turn.  Each warp streams its items' compressed bytes through a
// ring of slots in shared memory with bulk copies (6-8 items ahead, about
// 190 KB in flight per SM, enough to keep HBM busy), keeps the segment's X
// values in registers while it walks down the rows, rebuilds each weight in
// registers and multiply-adds two FP32 lanes per instruction (fma.rn.f32x2).
// Every wait for a copy is bounded in time (timeout status, no hang).  Each item's lane sums are reduced across the
// warp, stored per (row, segment) in shared memory, and the segments of a row
// are added in K order at the end (deterministic).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bf16_fields.cuh"
#include "pdl.cuh"
#include "uw_internal.h"
#include "uw_kernels.h"

namespace uw {

namespace {

constexpr int kGvWarps = 16;
constexpr int kGvThreads = 32 * kGvWarps;
constexpr int kSeg = 1024;    // weights of a row per work item (32 per lane)

// Per-warp ring of item slots in shared memory, each filled by one or two bulk
// copies (cp.async.bulk, completion counted on the slot's mbarrier) issued by
// lane 0: an item's sign+mantissa bytes (1 KB) and its indices (512 B) or
// exponent bytes (1 KB) are each contiguous in memory, as are its BF16
// weights (2 KB).  Lane l then reads its 32 weights' bytes from the slot.
template <int MODE>
struct Ring {
  static constexpr int kBytesA = MODE == kGemmBf16 ? 2048 : 1024;  // W, or S
  static constexpr int kBytesB = MODE == kGemmBf16 ? 0 : (MODE == kGemmExp ? 1024 : 512);
  static constexpr int kSlotBytes = kBytesA + kBytesB;
  static constexpr int kSlots = MODE == kGemmPalette ? 8 : 6;
};

struct GvParams {
  const uint16_t* X;   // [M, K] bf16
  const uint16_t* W;   // [N, K] bf16 (pipeline 1)
  const uint8_t* S;    // [N, K] sign+mantissa
  const uint8_t* E;    // [N, K] exponents (pipeline 2)
  const uint8_t* I;    // [N, K/2] packed palette indices (pipelines 3, 4)
  const uint32_t* esc_bits;
  const uint32_t* esc_off;
  const uint8_t* esc_pack;
  void* Y;
  uint32_t* status;
  uint64_t wait_ns;
  int64_t N, K;
  int32_t M, out_f32, esc_nw, kbk, segs, rows_per_cta, esc_words;  // esc_words per K block
  int32_t pal_run, w_early;  // w_early: the weights are the handle's own (read before the wait)
  uint32_t pal_bias;
  uint32_t palette[4];
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t par) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(par)
      : "memory");
  return ok != 0;
}

// Wait for the slot's copies (phase parity `par`), giving up after limit_ns.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t par, uint64_t limit_ns) {
  if (bar_try(bar, par)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t i = 1;; ++i) {
    if (bar_try(bar, par)) return true;
    if ((i & 63) == 0 && gtimer() - t0 > limit_ns) return false;
  }
}

// 1-D bulk copy global -> shared (both 16-byte aligned, bytes % 16 == 0); the
// copy reads L2, coherent with the kernel this one may overlap once the
// dependency wait is passed.
__device__ __forceinline__ void bulk(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// The handle's escape data (never written by a kernel).
__device__ __forceinline__ uint4 ld_cached(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The caller's X, read after the dependency wait with coherent loads (the
// kernel ahead of this one may have written it).
__device__ __forceinline__ uint4 ld_x(const void* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// Two BF16 (a pair word, element order) as the two FP32 of a 64-bit pair.
__device__ __forceinline__ uint64_t pair_f32(uint32_t w) {
  return ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint64_t)(w << 16);
}

// acc.lo += a.lo * b.lo, acc.hi += a.hi * b.hi (two FP32 lanes, one instruction).
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// The lane's 32 BF16 weights of one item as 16 pair words, element order;
// `sa` / `sb`: the slot's two regions, `esc`: whether the lane's 64-weight
// row is an escape row.
template <int MODE>
__device__ __forceinline__ void rebuild_item(const GvParams& p, const uint8_t* sa, const uint8_t* sb,
                                             int lane, int64_t n, int k0, bool esc,
                                             uint32_t (&w)[16]) {
  if (MODE == kGemmBf16) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = *reinterpret_cast<const uint4*>(sa + 64 * lane + 16 * q);
      w[4 * q] = v.x;
      w[4 * q + 1] = v.y;
      w[4 * q + 2] = v.z;
      w[4 * q + 3] = v.w;
    }
    return;
  }
  const uint4 a = *reinterpret_cast<const uint4*>(sa + 32 * lane);
  const uint4 b = *reinterpret_cast<const uint4*>(sa + 32 * lane + 16);
  const uint32_t sv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  if (MODE == kGemmExp) {
    const uint4 c = *reinterpret_cast<const uint4*>(sb + 32 * lane);
    const uint4 d = *reinterpret_cast<const uint4*>(sb + 32 * lane + 16);
    const uint32_t e[8] = {c.x, c.y, c.z, c.w, d.x, d.y, d.z, d.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint2 q = merge4(sv[j], e[j]);
      w[2 * j] = q.x;
      w[2 * j + 1] = q.y;
    }
    return;
  }
  if (esc) {
    // escape row (the 64 weights of row n in K block k0/64 are stored
    // verbatim): the exponents come from the escape data
    const int kb = k0 >> 6;
    const int64_t g = (n >> 7) * p.kbk + kb;
    const uint8_t* base = p.esc_pack + 16 * g + 64 * (int64_t)__ldg(p.esc_off + g);
    const uint4 bm = ld_cached(base);
    const uint32_t bw[4] = {bm.x, bm.y, bm.z, bm.w};
    const int r = (int)(n & 127);
    int rank = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int lo = i * 32;
      if (r >= lo + 32)
        rank += __popc(bw[i]);
      else if (r > lo)
        rank += __popc(bw[i] & ((1u << (r - lo)) - 1u));
    }
    const uint8_t* ex = base + 16 + 64 * rank + (k0 & 63);
    const uint4 e0 = ld_cached(ex), e1 = ld_cached(ex + 16);
    const uint32_t e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint2 q = merge4(sv[j], e[j]);
      w[2 * j] = q.x;
      w[2 * j + 1] = q.y;
    }
    return;
  }
  const uint4 c = *reinterpret_cast<const uint4*>(sb + 16 * lane);
  const uint32_t v[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 q = p.pal_run ? rebuild8_run(v[j], sv[2 * j], sv[2 * j + 1], p.pal_bias)
                              : rebuild8_lut(v[j], sv[2 * j], sv[2 * j + 1], p.palette[0],
                                             p.palette[1], p.palette[2], p.palette[3]);
    w[4 * j] = q.x;
    w[4 * j + 1] = q.y;
    w[4 * j + 2] = q.z;
    w[4 * j + 3] = q.w;
  }
}

// Work items of a CTA, segment-major (item i: segment i / R, row i % R of the
// CTA's R rows), so a warp's items (i, i + 16, ...) stay in one segment for
// several rows and its X values are loaded once per segment.
template <int MODE, int MM>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_kernel(const GvParams p) {
  using RG = Ring<MODE>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t r0 = (int64_t)blockIdx.x * p.rows_per_cta;
  const int64_t r1 = r0 + p.rows_per_cta < p.N ? r0 + p.rows_per_cta : p.N;
  const int R = (int)(r1 - r0);
  const int items = R * p.segs;
  // shared memory: the rings, the slots' barriers, the escape bitmap words of
  // the CTA's rows (palette modes), the partial sums
  uint8_t* ring = smem + (size_t)warp * RG::kSlots * RG::kSlotBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kGvWarps * RG::kSlots * RG::kSlotBytes);
  uint32_t* escw = reinterpret_cast<uint32_t*>(bars + kGvWarps * RG::kSlots);
  const int w0 = (int)(r0 >> 5);
  float* part = reinterpret_cast<float*>(escw + (MODE == kGemmPalette ? p.kbk * p.esc_words : 0));
  const uint32_t bar0 = smem_addr(bars + warp * RG::kSlots);
  const uint32_t ring_s = smem_addr(ring);
  const int my_items = items > warp ? (items - warp + kGvWarps - 1) / kGvWarps : 0;

  if (lane == 0) {
    for (int sl = 0; sl < RG::kSlots; ++sl)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8u * sl));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (MODE == kGemmPalette) {  // (the handle's own data)
    for (int t = threadIdx.x; t < p.kbk * p.esc_words; t += kGvThreads) {
      const int kb = t / p.esc_words, wi = w0 + (t - kb * p.esc_words);
      escw[t] = wi < p.esc_nw ? __ldg(p.esc_bits + (int64_t)kb * p.esc_nw + wi) : 0u;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // item cursors (segment, row within the CTA): one for the copies, kSlots
  // items ahead, one for the arithmetic; a warp's items are 16 apart
  auto advance = [&](int& sg, int& rl) {
    rl += kGvWarps;
    while (rl >= R) {
      rl -= R;
      ++sg;
    }
  };
  int sg_i = R > 0 ? warp / R : 0, rl_i = R > 0 ? warp - sg_i * R : 0;
  // lane 0 issues item t's copies into slot t % kSlots (t in order)
  auto issue = [&](int t) {
    if (t >= my_items) return;
    if (lane == 0) {
      const int kw = p.K - (int64_t)sg_i * kSeg < kSeg ? (int)(p.K - (int64_t)sg_i * kSeg) : kSeg;
      const uint32_t bytes_a = MODE == kGemmBf16 ? 2u * kw : (uint32_t)kw;
      const uint32_t bytes_b =
          MODE == kGemmBf16 ? 0u : (MODE == kGemmExp ? (uint32_t)kw : (uint32_t)kw / 2u);
      const int sl = t % RG::kSlots;
      const uint32_t bar = bar0 + 8u * sl, dst = ring_s + (uint32_t)sl * RG::kSlotBytes;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                   "r"(bytes_a + bytes_b)
                   : "memory");
      const int64_t o = (r0 + rl_i) * p.K + (int64_t)sg_i * kSeg;
      if (MODE == kGemmBf16) {
        bulk(dst, p.W + o, bytes_a, bar);
      } else {
        bulk(dst, p.S + o, bytes_a, bar);
        if (MODE == kGemmExp)
          bulk(dst + RG::kBytesA, p.E + o, bytes_b, bar);
        else
          bulk(dst + RG::kBytesA, p.I + o / 2, bytes_b, bar);
      }
    }
    advance(sg_i, rl_i);
  };

  // the handle's own weights may be read before the kernel ahead of this one
  // has finished; a workspace, X and Y only after
  if (!p.w_early) asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int t = 0; t < RG::kSlots; ++t) issue(t);
  if (p.w_early) asm volatile("griddepcontrol.wait;" ::: "memory");

  uint64_t x[MM][16];  // this segment's X values, as FP32 pairs
  int cur_sg = -1;
  int t_dead = -1;  // the item whose wait ran out
  int sg = R > 0 ? warp / R : 0, rl = R > 0 ? warp - sg * R : 0;
#pragma unroll 1
  for (int t = 0; t < my_items; ++t, advance(sg, rl)) {
    const int sl = t % RG::kSlots;
    const bool ok = __all_sync(0xffffffffu,
                               bar_wait(bar0 + 8u * sl, (uint32_t)((t / RG::kSlots) & 1), p.wait_ns));
    if (!ok) {
      if (lane == 0) atomicOr(p.status, kStatusTimeout);
      t_dead = t;
      break;
    }
    const int64_t n = r0 + rl;
    const int k0 = sg * kSeg + 32 * lane;
    const bool on = k0 < p.K;
    if (sg != cur_sg) {  // (uniform over the warp) this segment's X values
      cur_sg = sg;
#pragma unroll
      for (int m = 0; m < MM; ++m) {
        if (on) {
          const uint16_t* xr = p.X + (int64_t)m * p.K + k0;
          const uint4 x0 = ld_x(xr), x1 = ld_x(xr + 8), x2 = ld_x(xr + 16), x3 = ld_x(xr + 24);
          const uint32_t xv[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                   x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
#pragma unroll
          for (int j = 0; j < 16; ++j) x[m][j] = pair_f32(xv[j]);
        }
      }
    }
    uint64_t acc[MM][2];
#pragma unroll
    for (int m = 0; m < MM; ++m) acc[m][0] = acc[m][1] = 0ull;
    if (on) {
      bool esc = false;
      if (MODE == kGemmPalette) {
        const int kb = k0 >> 6;
        const int wi = (int)(n >> 5) - w0;
        esc = (escw[kb * p.esc_words + wi] >> (n & 31)) & 1u;
      }
      const uint8_t* sa = ring + (size_t)sl * RG::kSlotBytes;
      uint32_t w[16];
      rebuild_item<MODE>(p, sa, sa + RG::kBytesA, lane, n, k0, esc, w);
#pragma unroll
      for (int m = 0; m < MM; ++m) {
#pragma unroll
        for (int j = 0; j < 16; ++j) ffma2(acc[m][j & 1], pair_f32(w[j]), x[m][j]);
      }
    }
    __syncwarp();
    issue(t + RG::kSlots);  // the slot is read: refill it
#pragma unroll
    for (int m = 0; m < MM; ++m) {
      float v = (__uint_as_float((uint32_t)acc[m][0]) + __uint_as_float((uint32_t)(acc[m][0] >> 32))) +
                (__uint_as_float((uint32_t)acc[m][1]) + __uint_as_float((uint32_t)(acc[m][1] >> 32)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      // part[row][segment][m]
      if (lane == 0) part[(rl * p.segs + sg) * MM + m] = v;
    }
  }
  if (t_dead >= 0) {  // copies still in flight (items t_dead ..) must land before the CTA exits
    for (int u = t_dead; u < t_dead + RG::kSlots && u < my_items; ++u)
      bar_wait(bar0 + 8u * (u % RG::kSlots), (uint32_t)((u / RG::kSlots) & 1), p.wait_ns);
  }
  __syncthreads();
  // each row: its segments in K order
  for (int t = threadIdx.x; t < R * p.M; t += kGvThreads) {
    const int rl = t / p.M, m = t - rl * p.M;
    float y = 0.f;
    for (int sg = 0; sg < p.segs; ++sg) y += part[(rl * p.segs + sg) * MM + m];
    const int64_t o = (int64_t)m * p.N + r0 + rl;
    if (p.out_f32)
      static_cast<float*>(p.Y)[o] = y;
    else
      static_cast<uint16_t*>(p.Y)[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
  }
}

// Escape-bitmap words of a CTA's rows per K block (rows_per_cta rows starting
// at any row: one more word than they fill when they straddle a boundary).
int esc_words_for(int rows_per_cta) { return (rows_per_cta + 31) / 32 + 1; }

template <int MODE>
size_t gemv_smem(int rows_per_cta, int segs, int mm, int kbk) {
  using RG = Ring<MODE>;
  return (size_t)kGvWarps * RG::kSlots * RG::kSlotBytes + (size_t)kGvWarps * RG::kSlots * 8 +
         (MODE == kGemmPalette ? (size_t)kbk * esc_words_for(rows_per_cta) * 4 : 0) +
         (size_t)rows_per_cta * segs * mm * 4;
}

}  // namespace

size_t gemv_smem_for(int mode, int rows, int segs, int mm, int kbk) {
  return mode == kGemmBf16 ? gemv_smem<kGemmBf16>(rows, segs, mm, kbk)
         : mode == kGemmExp ? gemv_smem<kGemmExp>(rows, segs, mm, kbk)
                            : gemv_smem<kGemmPalette>(rows, segs, mm, kbk);
}

bool gemv_supported(const GemmArgs& a) {
  if (a.M < 1 || a.M > kGemvMaxM || a.N < 1 || a.K < 64 || a.K % 64) return false;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t segs = (a.K + kSeg - 1) / kSeg;
  const int64_t rows = (a.N + sms - 1) / sms;
  if (rows * segs >= (int64_t)1 << 30) return false;
  return gemv_smem_for(a.mode, (int)rows, (int)segs, kGemvMaxM, (int)(a.K / 64)) <= 227 * 1024;
}

cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t s, const LaunchHooks* hooks) {
  if (!gemv_supported(a)) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  GvParams p;
  p.X = a.X;
  p.W = a.W;
  p.S = a.S;
  p.E = a.E;
  p.I = a.I;
  p.esc_bits = a.esc_bits;
  p.esc_off = a.esc_off;
  p.esc_pack = a.esc_pack;
  p.Y = a.Y;
  p.N = a.N;
  p.K = a.K;
  p.M = (int32_t)a.M;
  p.out_f32 = a.out_f32;
  p.esc_nw = a.esc_nw;
  p.kbk = (int32_t)(a.K / 64);
  p.segs = (int32_t)((a.K + kSeg - 1) / kSeg);
  const int64_t grid = a.N < sms ? a.N : sms;
  p.rows_per_cta = (int32_t)((a.N + grid - 1) / grid);
  const int64_t blocks = (a.N + p.rows_per_cta - 1) / p.rows_per_cta;
  bool run = true;
  for (int i = 1; i < 16; ++i)
    if (a.palette[i] != a.palette[0] + i) run = false;
  p.pal_run = run ? 1 : 0;
  p.pal_bias = (uint32_t)a.palette[0] * 128u * 0x00010001u;
  for (int i = 0; i < 4; ++i)
    p.palette[i] = (uint32_t)a.palette[4 * i] | ((uint32_t)a.palette[4 * i + 1] << 8) |
                   ((uint32_t)a.palette[4 * i + 2] << 16) | ((uint32_t)a.palette[4 * i + 3] << 24);
  p.w_early = a.mode == kGemmPalette && a.w1_resident ? 1 : 0;
  p.status = a.status;
  p.wait_ns = wait_limit_ns();
  p.esc_words = esc_words_for(p.rows_per_cta);
  const int mm = a.M <= 1 ? 1 : 2;
  const size_t smem = gemv_smem_for(a.mode, p.rows_per_cta, p.segs, mm, p.kbk);
  const int kind = a.mode == kGemmBf16 ? 7 : (a.mode == kGemmExp ? 8 : 9);
  const int slot = hooks && hooks->begin ? hooks->begin(hooks->ctx, kind) : -1;
  auto go = [&](auto kernel) {
    cudaError_t r = cudaSuccess;
    if (smem > 48 * 1024)
      r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (r == cudaSuccess) r = launch_pdl(kernel, dim3((unsigned)blocks), dim3(kGvThreads), smem, s, p);
    return r;
  };
  switch (a.mode * 2 + (mm - 1)) {
    case kGemmBf16 * 2: e = go(gemv_kernel<kGemmBf16, 1>); break;
    case kGemmBf16 * 2 + 1: e = go(gemv_kernel<kGemmBf16, 2>); break;
    case kGemmExp * 2: e = go(gemv_kernel<kGemmExp, 1>); break;
    case kGemmExp * 2 + 1: e = go(gemv_kernel<kGemmExp, 2>); break;
    case kGemmPalette * 2: e = go(gemv_kernel<kGemmPalette, 1>); break;
    default: e = go(gemv_kernel<kGemmPalette, 2>); break;
  }
  if (hooks && hooks->end) hooks->end(hooks->ctx, slot);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace uw
