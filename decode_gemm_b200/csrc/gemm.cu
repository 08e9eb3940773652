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
//   * Warp roles: warp 0 weight producer (TMA), warps 1-2 MMA issuers (units
//     alternate between them by parity, each with its own accumulators; warp
//     1 owns TMEM), warps 3-6 epilogue (TMEM -> registers -> global), warps
//     7-14 rebuild in two groups of 4 taking alternate units (reconstructive
//     modes only), and the last warp the X producer (X tiles on a ring of
//     their own, so the weight ring's depth goes to HBM traffic).
//   * Rebuild: for token tiles up to 96, each thread rebuilds one W row of
//     the unit's K blocks and writes it to TMEM (tcgen05.st); the MMA reads A
//     from TMEM.  Larger tiles rebuild into the 128-byte-swizzled K-major
//     shared layout the MMA descriptor expects.  A palette that is one run
//     of exponents rebuilds with a multiply-add per BF16 pair, any other with
//     byte-permute lookups; the escape decision is taken once per 64-weight
//     row from a 16-byte bitmap staged with the tile.
//   * Persistent CTAs split the flattened (output tile, K block) space evenly
//     (stream-K).  A tile shared by several CTAs is finished inside the kernel
//     by the CTA holding its first K block: that tile is the last it works on,
//     so by then the others have usually handed over their partial sums
//     (written to the workspace, then a ready flag tagged with the launch's
//     epoch); it adds them in K order, so results are deterministic.  The
//     epoch lives on the device (the last CTA to exit advances it), so stale
//     flags from earlier launches, aborted ones or graph replays never match.
//   * CTA pairs (BF16 mode, on request): two-SM MMAs of 256 W rows over a
//     cluster of two CTAs, the same stream-K split per pair.
//   * Every mbarrier wait is bounded in wall time; on expiry the kernel records
//     a timeout in the status word, drains its MMAs and copies, frees TMEM and
//     returns.
//   * No TMA load with cluster multicast anywhere (CTA pairs load their own
//     halves; only MMA commits arrive on both CTAs' barriers).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bf16_fields.cuh"
#include "gemm_sm100.cuh"
#include "pdl.cuh"
#include "uw_kernels.h"

namespace uw {

namespace {

using namespace sm100;

constexpr int kBM = 128;           // W rows per tile (MMA M)
constexpr int kBK = 64;            // K per stage: one 128-byte swizzle row of BF16
constexpr int kWTileBytes = kBM * kBK * 2;
constexpr int kEscCap = 15;        // escape rows staged per stage (more: read from global);
                                   // 15 keeps a 16-token palette stage at 15 KB
constexpr int kMaxWSlots = 8;      // rebuilt-W ring depth (runtime, <= this)
constexpr int kMaxStages = 16;     // load ring depth (runtime, <= this)
constexpr int64_t kWideMinM = 512;  // tokens from which the BF16 GEMM uses 256-token tiles
constexpr int kNumEpiWarps = 4;
constexpr int kNumRebuildWarps = 8;  // two groups of 4, alternating stages
constexpr int kGroupWarps = kNumRebuildWarps / 2;
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kRebuildItems = kBM * kBK / 8 / kGroupThreads;  // 8-weight items per thread
static_assert(kRebuildItems == 8, "escape-bit mapping assumes rows gt/8 + 16 i");
constexpr int kMmaWarp0 = 1;         // MMA issuers: warps 1 and 2
constexpr int kNumMmaWarps = 2;
constexpr int kEpiWarp0 = kMmaWarp0 + kNumMmaWarps;  // warps 3..6 (quadrants 3,0,1,2)
constexpr int kRebuildWarp0 = kEpiWarp0 + kNumEpiWarps;
constexpr uint32_t kEpiSleepNs = 200;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block

// The X producer is the last warp.
__host__ __device__ constexpr int x_warp_for(int mode) {
  return mode == kGemmBf16 ? kRebuildWarp0 : kRebuildWarp0 + kNumRebuildWarps;
}
__host__ __device__ constexpr int threads_for(int mode) { return (x_warp_for(mode) + 1) * 32; }

struct GemmParams {
  CUtensorMap tm_x;   // X [M, K] bf16, box {64, tile_n}, 128B swizzle
  CUtensorMap tm_w0;  // bf16 mode: W [N, K] box {64, 128} 128B swizzle; else S [N, K] u8 box {64,128}
  CUtensorMap tm_w1;  // exp mode: E [N, K] u8 box {64, 128}; palette mode: I [N, K/2] u8 box {32, 128}
  CUtensorMap tm_y;   // Y [M, N] bf16, box {128, 16} (when y_tma)
  const uint32_t* esc_bits;
  const uint32_t* esc_off;
  const uint8_t* esc_exp;
  const uint8_t* esc_pack;  // per group (tile, K block): 16-byte bitmap, then its escape rows
  void* Y;
  float* partials;
  uint32_t* status;
  uint32_t* sync;     // [0] epoch, [1] exited CTAs, [2 + cta] ready flags
  int64_t M, N, K;
  int64_t units;      // output tiles * K blocks
  int32_t tile_n, stages, wslots, n_mma, NT, MT, esc_nwp, out_f32, tmem_cols;
  int32_t KB;        // units along K (K blocks / ks)
  int32_t KBK;       // 64-wide K blocks
  int32_t ks;        // K blocks per unit (stage): 1, or 2 on the TMEM path
  int32_t halves;    // 128-row halves per unit: 1, or 2 for the wide (large-M) shape
  int32_t acc_bufs;  // TMEM accumulator sets (2: epilogue overlaps the next tile)
  int32_t NG;        // 128-row groups of W (escape groups per K block)
  int32_t xstages;   // X ring depth (the units' X tiles ride their own ring)
  int32_t y_tma;     // BF16 Y written by TMA stores of 16-token blocks
  int32_t tmem_w;    // W slots in TMEM (MMA A from TMEM) rather than shared memory
  uint32_t wcol0;    // first TMEM column of the W slots
  const uint8_t* pf_s;   // the handle's sign+mantissa array, for early L2 prefetch
  const uint8_t* pf_i;   // resident index array (pipeline 4), or null
  int32_t pal_run;   // palette is the run base..base+15 (index = exponent - base)
  uint32_t pal_bias; // base * 128 in both 16-bit halves
  uint32_t palette[4];
  uint32_t stage_bytes, x_bytes;
  uint64_t wait_ns;
  int32_t withhold;  // failure-detection tests: contributors never publish (see launch)
};

// Per-stage shared-memory layout, offsets from the stage base.
struct StageLayout {
  uint32_t x, w0, w1, ebits, erows, bytes;
};

// A load stage holds the unit's W data: the TMA boxes cover all H*128 rows
// and ks K blocks at once (row-major inside a box, 64*ks sign+mantissa or
// exponent bytes, 32*ks index bytes per row).  Palette escape data has one
// area per (half, K block) part (H * ks <= 2): a 16-byte bitmap, then up to
// kEscCap rows (kEscArea bytes).  The units' X tiles (ks per unit) ride a
// separate, shallower ring: they come from L2, while W needs a deep ring to
// keep HBM busy.
constexpr uint32_t kEscArea = 16 + kEscCap * 64;
// One epilogue block of Y staged for a TMA store: 16 tokens x 128 rows, BF16.
constexpr uint32_t kYBlockBytes = 16 * kBM * 2;

__host__ __device__ inline StageLayout stage_layout(int mode, int tile_n, int halves, int ks) {
  StageLayout L;
  (void)tile_n;
  L.x = 0;  // (X has its own ring)
  const uint32_t HK = (uint32_t)(halves * ks);  // 128x64 W blocks per stage
  L.w0 = 0;
  if (mode == kGemmBf16) {
    L.w1 = L.ebits = L.erows = L.w0 + HK * kWTileBytes;
    L.bytes = L.w0 + HK * kWTileBytes;
  } else if (mode == kGemmExp) {
    L.w1 = L.w0 + HK * 8192;
    L.ebits = L.erows = L.w0 + HK * 16384;
    L.bytes = L.w0 + HK * 16384;
  } else {
    L.w1 = L.w0 + HK * 8192;
    L.ebits = L.w0 + HK * 12288;  // part p: bitmap at ebits + p*kEscArea, rows 16 bytes on
    L.erows = L.ebits + 16;
    L.bytes = L.ebits + HK * kEscArea;
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

// The four epilogue warps synchronise among themselves on named barrier 1;
// the OR-reduction gives all 128 threads the same decision.
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void epi_sync() {
  asm volatile("barrier.cta.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait until *flag == tag, giving up after limit_ns or when *abort is raised.
__device__ __forceinline__ bool wait_flag(const uint32_t* flag, uint32_t tag, volatile int* abort,
                                          uint64_t limit_ns) {
  if (ld_acquire(flag) == tag) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire(flag) == tag) return true;
    if (*abort || globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// KS_: K blocks per unit (compile time, so the per-block loops unroll); it
// equals p.ks.
template <int MODE, int KS_, bool PAIR = false>
__global__ void __launch_bounds__(threads_for(MODE), 1)
    gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned, by an offset into the shared array (the accesses stay
  // shared-window loads and stores)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const StageLayout L = stage_layout(MODE, p.tile_n, p.halves, p.ks);
  const int S = p.stages;
  const int WS = MODE == kGemmBf16 ? 0 : p.wslots;
  // MMA-issuing warps: with one half per unit they split the units by parity
  // (NM = 2) or one takes all (NM = 1); in the wide shape warp h takes half h
  // of every unit, and rebuild group h rebuilds it
  const int NM = p.n_mma;
  const int H = p.halves;
  const bool wide = H == 2;
  const int RU = kBM * H;  // W rows per unit
  // CTA pairs (two-SM MMA): the CTA's rank in its pair; the rank-0 CTA
  // issues the MMAs
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  const bool lead = crank == 0;
  // first W row of this CTA in row tile nt (a pair's tile has 256 rows, rank r
  // holds rows 128 r ..)
  auto row0_of = [&](int64_t nt) -> int64_t {
    return PAIR ? nt * (2 * kBM) + (int64_t)crank * kBM : nt * RU;
  };
  const int SX = p.xstages;
  const uint32_t xst_bytes = (uint32_t)KS_ * p.x_bytes;  // one unit's X tiles
  uint8_t* ring = smem;
  uint8_t* xring = ring + (size_t)S * L.bytes;       // X tiles
  // rebuilt W tiles (shared-memory path); a pair keeps a spare X tile's room
  // after its X ring, so no operand read of the MMA can pass the block's end
  uint8_t* wring = xring + (size_t)SX * xst_bytes + (PAIR ? xst_bytes : 0);
  uint8_t* ystage = wring + (size_t)(p.tmem_w ? 0 : WS) * kWTileBytes;  // 2 x [16][128] BF16
  uint8_t* tail = ystage + (p.y_tma ? 2 * kYBlockBytes : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  // barrier indices
  const int b_full = 0, b_empty = S, b_xfull = 2 * S, b_xempty = 2 * S + SX,
            b_wfull = 2 * S + 2 * SX, b_wfree = b_wfull + WS, b_tfull = b_wfree + WS,
            b_tempty = b_tfull + 2, b_drain = b_tempty + 2, b_part = b_drain + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + b_part + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(b_full + s), 1);
      // released by each half's reader: its MMA commit (BF16 tiles) or its
      // rebuild group's warps (compressed tiles)
      mbar_init(bar(b_empty + s), (uint32_t)H * (MODE == kGemmBf16 ? 1 : kGroupWarps));
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(bar(b_xfull + s), 1);
      mbar_init(bar(b_xempty + s), (uint32_t)H);  // each half's MMA commit
    }
    for (int w = 0; w < WS; ++w) {
      mbar_init(bar(b_wfull + w), kGroupWarps);
      mbar_init(bar(b_wfree + w), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(b_tfull + a), (uint32_t)NM);
      mbar_init(bar(b_tempty + a), PAIR ? 2 * kNumEpiWarps : kNumEpiWarps);
      mbar_init(bar(b_drain + a), 1);
    }
    mbar_init(bar(b_part), 1);
    *abort = 0;
    fence_mbar_init();
  }
  // CTA pairs: both CTAs of a pair take the pair's units; partitions, their
  // count and owners are per pair, while partial sums and ready flags stay
  // per CTA (slot 2 pid + rank)
  const int64_t G = PAIR ? gridDim.x / 2 : gridDim.x;
  const int64_t pid = PAIR ? blockIdx.x / 2 : blockIdx.x;
  auto slot_of = [&](int64_t q) { return PAIR ? 2 * q + crank : q; };
  const int64_t u0 = unit_begin(pid, p.units, G);
  const int64_t u1 = unit_begin(pid + 1, p.units, G);
  const int KB = p.KB;    // units along K
  constexpr int KS = KS_;  // K blocks per unit
  const int NP = H * KS;  // escape parts per stage: (half, K block) pairs, at most 2
  // Palette escape offsets (first and end row of each part's escape run) of 32
  // units, one unit per lane, loaded together: a load per stage would put its
  // latency on the issue path.  The first batch is loaded during setup, later
  // ones half a batch ahead.
  uint32_t lc0[2] = {0u, 0u}, lc1[2] = {0u, 0u}, nc0[2] = {0u, 0u}, nc1[2] = {0u, 0u};
  auto esc_batch = [&](int64_t qfirst, uint32_t (&o0)[2], uint32_t (&o1)[2]) {
    const int64_t uu = u0 + qfirst + lane;
    o0[0] = o0[1] = o1[0] = o1[1] = 0u;
    if (uu < u1) {
      const int64_t tt = uu / KB;
      const int64_t kk = uu - tt * KB;
      const int64_t g0 = (tt / p.MT) * H;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (q >= NP) break;
        // part q: half q / KS, K block kk * KS + q % KS
        const int64_t g = g0 + q / KS;
        if (g < p.NG) {
          const int64_t gi = g * p.KBK + kk * KS + q % KS;
          o0[q] = __ldg(p.esc_off + gi);
          o1[q] = __ldg(p.esc_off + gi + 1);
        }
      }
    }
  };
  if (MODE == kGemmPalette && warp == 0) esc_batch(0, lc0, lc1);
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.tm_x);
    prefetch_tensormap(&p.tm_w0);
    if (p.y_tma) prefetch_tensormap(&p.tm_y);
    if (MODE != kGemmBf16) prefetch_tensormap(&p.tm_w1);
  }
  if (warp == kMmaWarp0) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair's barriers are all initialised before either CTA signals the other's
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up above touched only the handle's immutable arrays; from here on X,
  // the preprocessed weights, the workspace and the hand-off flags may belong
  // to the kernel before this one.  Meanwhile the rebuild warps (idle until
  // the first stage lands) pull the first ring's immutable weight rows into
  // L2, so the first loads after the wait hit L2.
  if (threadIdx.x == 0) pdl_release();
  if (MODE != kGemmBf16 && warp >= kRebuildWarp0 && warp < kRebuildWarp0 + kNumRebuildWarps &&
      H == 1) {
    const int64_t n_pf = imin64(u1 - u0, S);
    const int rt = threadIdx.x - kRebuildWarp0 * 32;
    for (int64_t i = rt; i < n_pf * kBM; i += kNumRebuildWarps * 32) {
      const int64_t u = u0 + i / kBM;
      const int64_t t = u / p.KB;
      const int64_t nt = t / p.MT;
      const int64_t n = nt * kBM + i % kBM;
      const int64_t kbk = (u - t * p.KB) * KS;
      if (n < p.N) {
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p.pf_s + n * p.K + kbk * kBK));
        if (p.pf_i) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.pf_i + n * (p.K / 2) + kbk * (kBK / 2)));
      }
    }
  }
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    int qi = 0;  // index of the unit among this CTA's units
    for (int64_t u = u0; u < u1 && ok;) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const int64_t nt = t / p.MT;
      const int32_t n0 = (int32_t)row0_of(nt);
      for (int kb = kb0; kb < kb1; ++kb, ++qi) {
        uint32_t c0[2] = {0u, 0u}, c1[2] = {0u, 0u};
        if (MODE == kGemmPalette) {
          if ((qi & 31) == 16) esc_batch(qi + 16, nc0, nc1);
          if ((qi & 31) == 0 && qi > 0) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              lc0[q] = nc0[q];
              lc1[q] = nc1[q];
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            c0[h] = __shfl_sync(0xffffffffu, lc0[h], qi & 31);
            c1[h] = __shfl_sync(0xffffffffu, lc1[h], qi & 31);
          }
        }
        if (lane == 0) {
          if (!mbar_wait_bounded(bar(b_empty + stage), phase ^ 1u, abort, p.wait_ns)) {
            set_abort(abort, p.status);
            ok = false;
          } else {
            uint8_t* st = ring + (size_t)stage * L.bytes;
            const uint32_t fb = bar(b_full + stage);
            uint32_t bytes = 0;
            if (MODE == kGemmBf16) bytes += NP * kWTileBytes;
            if (MODE == kGemmExp) bytes += NP * 16384;
            // escape rows of each part's 128-row group and K block: one copy of
            // its bitmap and first rows, or none and a zero bitmap
            uint32_t nesc[2] = {0u, 0u};
            bool has[2] = {false, false};
            if (MODE == kGemmPalette) {
              bytes += NP * 12288;
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                if (q >= NP) break;
                // (past the last group: no escapes)
                has[q] = c1[q] > c0[q];
                nesc[q] = min(c1[q] - c0[q], (uint32_t)kEscCap);
                if (has[q]) {
                  bytes += 16 + nesc[q] * 64;
                } else {
                  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                                   smem_u32(st + L.ebits + q * kEscArea)),
                               "r"(0u)
                               : "memory");
                }
              }
            }
            const int kbk = kb * KS;  // first K block of the unit
            if constexpr (PAIR) {
              // both CTAs' tiles count on the leader's barrier, which expects both
              if (lead) mbar_expect_tx(fb, 2 * bytes);
              tma_load_2d_pair(smem_u32(st + L.w0), &p.tm_w0, mapa_shared(fb, 0), kbk * kBK, n0);
            } else {
              mbar_expect_tx(fb, bytes);
              tma_load_2d(smem_u32(st + L.w0), &p.tm_w0, fb, kbk * kBK, n0);
            }
            if (MODE == kGemmExp) tma_load_2d(smem_u32(st + L.w1), &p.tm_w1, fb, kbk * kBK, n0);
            if (MODE == kGemmPalette) {
              tma_load_2d(smem_u32(st + L.w1), &p.tm_w1, fb, kbk * (kBK / 2), n0);
#pragma unroll
              for (int q = 0; q < 2; ++q)
                if (q < NP && has[q])
                  bulk_load(smem_u32(st + L.ebits + q * kEscArea),
                            p.esc_pack + 16 * ((nt * H + q / KS) * p.KBK + kbk + q % KS) +
                                (int64_t)c0[q] * 64,
                            16 + nesc[q] * 64, fb);
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
    // in-flight copies must land before the CTA exits (a pair's copies count
    // on the leader's barriers: the leader drains them, and the pair leaves
    // together)
    if (lane == 0 && *abort && (!PAIR || lead)) {
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
  } else if (warp < kMmaWarp0 + kNumMmaWarps) {
    // ---------------------------------------------------------- MMA issuers --
    // One half per unit: warp kMmaWarp0 + par takes the CTA's units q with
    // q % 2 == par (all of them when NM == 1) and accumulates into its own
    // TMEM columns.  The ring depths are then even, so a stage or W slot is
    // always consumed by the same warp, in order: a parity wait can never see
    // a stale phase.  (With an odd depth a stage would alternate between the
    // warps, and a parity wait cannot tell the fill before last, still
    // pending, from its own completed fill.)  Wide shape: warp par takes half
    // par of every unit (W slots go in pairs, slot 2 j + par for pair j) into
    // its own columns.
    const int par = warp - kMmaWarp0;
    // (a pair's MMAs are the rank-0 CTA's: they fill both CTAs' TMEM)
    if (par < NM && (!PAIR || lead)) {
      const uint32_t idesc = idesc_bf16(PAIR ? 2 * kBM : kBM, p.tile_n);
      auto commit = [&](uint32_t b) {
        if constexpr (PAIR)
          mma_commit_pair(b, 0x3);  // the barrier at this offset in both CTAs
        else
          mma_commit(b);
      };
      const int WP = wide ? WS / 2 : WS;  // W slot positions this warp cycles through
      // ring positions of the current unit, advanced for every unit of the CTA
      int stage = 0, wpos = 0, xs = 0;
      uint32_t phase = 0, wphase = 0, xph = 0;
      int q = 0;  // index of the unit among this CTA's units
      int seg = 0;
      bool ok = true;
      for (int64_t u = u0; u < u1 && ok; ++seg) {
        const int64_t t = u / KB;
        const int kb0 = (int)(u - t * KB);
        const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
        const int acc = p.acc_bufs == 2 ? (seg & 1) : 0;
        const uint32_t acc_phase = (uint32_t)(p.acc_bufs == 2 ? (seg >> 1) : seg) & 1u;
        if (lane == 0 &&
            !mbar_wait_bounded(bar(b_tempty + acc), acc_phase ^ 1u, abort, p.wait_ns)) {
          set_abort(abort, p.status);
          ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)((acc * NM + par) * p.tile_n);
        bool first = true;
        for (int kb = kb0; kb < kb1; ++kb, ++q) {
          const bool mine = wide || NM == 1 || (q & 1) == par;
          const int wslot = wide ? 2 * wpos + par : wpos;
          if (mine && lane == 0) {
            // A: BF16 tiles from the load stage, rebuilt tiles from their slot;
            // B: the unit's X tiles from the X ring
            bool got = true;
            if (MODE == kGemmBf16) got = mbar_wait_bounded(bar(b_full + stage), phase, abort, p.wait_ns);
            if (got) got = mbar_wait_bounded(bar(b_xfull + xs), xph, abort, p.wait_ns);
            if (got && MODE != kGemmBf16)
              got = mbar_wait_bounded(bar(b_wfull + wslot), wphase, abort, p.wait_ns);
            if (!got) {
              set_abort(abort, p.status);
              ok = false;
            } else {
              tc_fence_after();
              uint8_t* st = ring + (size_t)stage * L.bytes;
              uint8_t* xt = xring + (size_t)xs * xst_bytes;
              const uint64_t b_desc = smem_desc_sw128(smem_u32(xt));
              if (MODE != kGemmBf16 && p.tmem_w) {
                // A: 32 columns of the slot per K block, 8 per 16-wide K step;
                // B: the K block's X tile
                const uint32_t a_tmem = tmem_base + p.wcol0 + (uint32_t)(wslot * 32 * KS);
#pragma unroll
                for (int j = 0; j < KS; ++j) {
                  const uint64_t bj = smem_desc_sw128(smem_u32(xt + j * p.x_bytes));
#pragma unroll
                  for (int k = 0; k < kBK / 16; ++k)
                    mma_bf16_tmem_a(d_tmem, a_tmem + 32 * j + 8 * k, bj + 2 * k, idesc,
                                    (!first || j > 0 || k > 0) ? 1u : 0u);
                }
              } else {
                const uint32_t a_addr =
                    MODE == kGemmBf16 ? smem_u32(st + L.w0 + (wide ? par * kWTileBytes : 0))
                                      : smem_u32(wring + (size_t)wslot * kWTileBytes);
                const uint64_t a_desc = smem_desc_sw128(a_addr);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k) {
                  if constexpr (PAIR)
                    mma_bf16_pair(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc,
                                  (!first || k > 0) ? 1u : 0u);
                  else
                    mma_bf16(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc,
                             (!first || k > 0) ? 1u : 0u);
                }
              }
              if (MODE == kGemmBf16) commit(bar(b_empty + stage));
              commit(bar(b_xempty + xs));
              if (MODE != kGemmBf16) commit(bar(b_wfree + wslot));
            }
          }
          if (mine) first = false;
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
          if (++xs == SX) {
            xs = 0;
            xph ^= 1u;
          }
          if (WP && ++wpos == WP) {
            wpos = 0;
            wphase ^= 1u;
          }
        }
        // the segment's accumulator is complete once this warp's MMAs finish
        if (ok && lane == 0) commit(bar(b_tfull + acc));
        u += kb1 - kb0;
      }
      // every issued MMA completes before TMEM is released
      if (lane == 0) {
        commit(bar(b_drain + par));
        volatile int no_abort = 0;
        mbar_wait_bounded(bar(b_drain + par), 0, &no_abort, p.wait_ns);
      }
      __syncwarp();
    }
  } else if (warp < kRebuildWarp0) {
    // ------------------------------------------------------------ epilogue --
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    const bool leader = warp == kEpiWarp0 && lane == 0;
    // this launch's hand-off tag: the epoch (advanced by the previous launch's
    // last CTA, constant while this launch runs) plus one
    const uint32_t tag = __ldcg(p.sync) + 1u;
    const int64_t part_stride = (int64_t)p.tile_n * RU;  // a CTA's partial-sum tile
    int yblk = 0;  // Y blocks stored through the staging buffers
    int seg = 0;
    int64_t qa = 0;  // index (among this CTA's units) of the segment's first unit
    for (int64_t u = u0; u < u1; ++seg) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const bool split = !(kb0 == 0 && kb1 == KB);
      const int acc = p.acc_bufs == 2 ? (seg & 1) : 0;
      const uint32_t acc_phase = (uint32_t)(p.acc_bufs == 2 ? (seg >> 1) : seg) & 1u;
      // every lane observes the accumulator barrier before reading TMEM; the
      // wait is long (a whole segment), so it sleeps between polls
      const bool got =
          mbar_wait_bounded(bar(b_tfull + acc), acc_phase, abort, p.wait_ns, kEpiSleepNs);
      if (!got) set_abort(abort, p.status);
      if (epi_any(!got)) break;
      tc_fence_after();
      // a split tile's owner (the CTA, or pair, with its first K block)
      // collects the partial sums of partitions pid+1 .. last
      const int64_t nt = t / p.MT, mt = t - nt * p.MT;
      const int64_t m0 = mt * p.tile_n;
      const int cols = (int)imin64(p.tile_n, p.M - m0);
      bool owner = false, staged = false;
      int64_t last = 0;
      if (split) {
        const int64_t ua = t * KB;
        owner = unit_owner(ua, p.units, G) == pid;
        last = unit_owner(ua + KB - 1, p.units, G);
        if (owner) {
          // The owner's split segment is its CTA's last (the CTA's range ends
          // inside the tile), so the load ring is idle: the contributors' sums
          // (adjacent in the workspace) can come over in one bulk copy instead
          // of one L2 round trip per 16 columns.  Measured on 14336x4096 and
          // 4096x14336: a gain for 32..64 columns; for 16 or fewer the copy
          // moves mostly unused columns, for 128..256 its latency does not pay.
          const int64_t sbytes = (last - pid) * part_stride * 4;
          // (a pair's contributors' slots are not adjacent)
          staged = !PAIR && cols >= 32 && cols <= 64 && sbytes <= (int64_t)S * L.bytes;
          bool ok = true;
          if (leader) {
            for (int64_t q = pid + 1; q <= last && ok; ++q)
              ok = wait_flag(p.sync + 2 + slot_of(q), tag, abort, p.wait_ns);
            if (!ok) {
              set_abort(abort, p.status);
            } else if (staged) {
              fence_proxy_async_global();
              mbar_expect_tx(bar(b_part), (uint32_t)sbytes);
              bulk_load(smem_u32(ring), p.partials + (pid + 1) * part_stride,
                        (uint32_t)sbytes, bar(b_part));
            }
          }
          if (epi_any(!ok)) break;
          if (staged) {
            const bool in = mbar_wait_bounded(bar(b_part), 0, abort, p.wait_ns);
            if (!in) set_abort(abort, p.status);
            if (epi_any(!in)) break;
          }
        }
      }
      // which parity accumulators received MMAs in this segment (one half
      // per unit; in the wide shape each half has its own accumulator)
      const bool has0 = NM == 1 || (kb1 - kb0 >= 2) || ((qa & 1) == 0);
      const bool has1 = NM == 2 && ((kb1 - kb0 >= 2) || ((qa & 1) == 1));
      const uint32_t lanebase = (uint32_t)(quad * 32) << 16;
      for (int h = 0; h < H; ++h) {
        const bool use0 = wide || has0, use1 = !wide && has1;
        const uint32_t t0 =
            tmem_base + lanebase + (uint32_t)((acc * NM + (wide ? h : 0)) * p.tile_n);
        const uint32_t t1 = tmem_base + lanebase + (uint32_t)((acc * NM + 1) * p.tile_n);
        const int64_t n = row0_of(nt) + h * kBM + row;
        const int64_t hoff = (int64_t)h * kBM * p.tile_n;  // the half's place in a partial tile
        float* part = p.partials + slot_of(pid) * part_stride + hoff;
        // an owner reads the first contributor's sums one column block ahead,
        // so their latency overlaps the TMEM reads and the stores
        const bool gather = split && owner;
        const float* part1 = p.partials + slot_of(pid + 1) * part_stride + hoff + row;
        float pn[16];
        if (gather && !staged) {
#pragma unroll
          for (int j = 0; j < 16; ++j) pn[j] = j < cols ? __ldcg(part1 + j * kBM) : 0.f;
        }
        for (int c = 0; c < cols; c += 16) {
          uint32_t r0[16], r1[16];
          if (use0) tmem_ld16(t0 + (uint32_t)c, r0);
          if (use1) tmem_ld16(t1 + (uint32_t)c, r1);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = use0 ? __uint_as_float(r0[j]) : 0.f;
            if (use1) v[j] += __uint_as_float(r1[j]);
          }
          if (split && !owner) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c + j < cols) part[(int64_t)(c + j) * kBM + row] = v[j];
            continue;
          }
          if (gather && staged) {
            // the other CTAs' sums, in K order, from the staged copies
            const float* sp = reinterpret_cast<const float*>(ring) + hoff + (int64_t)c * kBM + row;
            for (int64_t q = 0; q < last - pid; ++q) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (c + j < cols) v[j] += sp[q * part_stride + j * kBM];
            }
          } else if (gather) {
            // the other CTAs' sums, in K order; a contributor's 16 loads are all
            // in flight before the first add
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += pn[j];
            if (c + 16 < cols) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                pn[j] = c + 16 + j < cols ? __ldcg(part1 + (int64_t)(c + 16 + j) * kBM) : 0.f;
            }
            for (int64_t q = pid + 2; q <= last; ++q) {
              const float* src = p.partials + slot_of(q) * part_stride + hoff + (int64_t)c * kBM + row;
              float pv[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) pv[j] = c + j < cols ? __ldcg(src + j * kBM) : 0.f;
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] += pv[j];
            }
          }
          if (KS_ == 1 && p.y_tma) {
            // (128+-token tiles always run with one K block per unit)
            // the block as [token][row] BF16 in shared memory, then one TMA
            // store of 16 token rows of 128 outputs each (parts past M or N are
            // not written); two buffers, so a store overlaps the next block
            uint16_t* yb = reinterpret_cast<uint16_t*>(ystage + (yblk & 1) * kYBlockBytes);
            if (leader) bulk_wait_read<1>();  // this buffer's previous store has read it
            epi_sync();
#pragma unroll
            for (int j = 0; j < 16; ++j) yb[j * kBM + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
            fence_proxy_async_smem();
            epi_sync();
            if (leader && row0_of(nt) + h * kBM < p.N) {  // (a box wholly past N writes nothing)
              tma_store_2d(&p.tm_y, smem_u32(yb), (int32_t)(row0_of(nt) + h * kBM), (int32_t)(m0 + c));
              bulk_commit();
            }
            ++yblk;
          } else if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (c + j < cols) {
                const int64_t o = (m0 + c + j) * p.N + n;
                if (p.out_f32)
                  static_cast<float*>(p.Y)[o] = v[j];
                else
                  static_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(v[j]);
              }
            }
          }
        }
      }
      if (split && !owner) {  // hand the partial sum over
        __threadfence();
        epi_sync();
        if (leader && !p.withhold) st_release(p.sync + 2 + slot_of(pid), tag);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(bar(b_tempty + acc), 0));  // the leader's barrier
        else
          mbar_arrive(bar(b_tempty + acc));
      }
      u += kb1 - kb0;
      qa += kb1 - kb0;
    }
    // the stores must have read the staging buffers (and landed) before exit
    if (KS_ == 1 && leader && p.y_tma) bulk_wait_all();
  } else if (warp == x_warp_for(MODE)) {
    // ---------------------------------------------------------- X producer --
    // The units' X tiles (K blocks of the token tile), in unit order, into
    // their own ring: X comes from L2 and needs few stages in flight, so the
    // load ring's depth goes to W.
    int xs = 0;
    uint32_t xph = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok;) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      // (a pair's CTA loads its half of the token tile: rank r tokens
      // tile_n / 2 * r ..)
      const int32_t m0 = (int32_t)((t - (t / p.MT) * p.MT) * p.tile_n +
                                   (PAIR ? (int64_t)crank * (p.tile_n / 2) : 0));
      for (int kb = kb0; kb < kb1; ++kb) {
        if (lane == 0) {
          if (!mbar_wait_bounded(bar(b_xempty + xs), xph ^ 1u, abort, p.wait_ns)) {
            set_abort(abort, p.status);
            ok = false;
          } else {
            const uint32_t fb = bar(b_xfull + xs);
            uint8_t* xt = xring + (size_t)xs * xst_bytes;
            if constexpr (PAIR) {
              if (lead) mbar_expect_tx(fb, 2 * xst_bytes);
              const uint32_t fbl = mapa_shared(fb, 0);
#pragma unroll
              for (int j = 0; j < KS; ++j)
                tma_load_2d_pair(smem_u32(xt + j * p.x_bytes), &p.tm_x, fbl, (kb * KS + j) * kBK, m0);
            } else {
              mbar_expect_tx(fb, xst_bytes);
#pragma unroll
              for (int j = 0; j < KS; ++j)
                tma_load_2d(smem_u32(xt + j * p.x_bytes), &p.tm_x, fb, (kb * KS + j) * kBK, m0);
            }
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (++xs == SX) {
          xs = 0;
          xph ^= 1u;
        }
      }
      u += kb1 - kb0;
    }
    // in-flight copies must land before the CTA exits (a pair's: see the
    // weight producer)
    if (lane == 0 && *abort && (!PAIR || lead)) {
      const int64_t outstanding = issued < SX ? issued : SX;
      int s = xs;
      uint32_t ph = xph;
      for (int64_t i = 0; i < outstanding; ++i) {
        if (--s < 0) {
          s = SX - 1;
          ph ^= 1u;
        }
        volatile int no_abort = 0;
        mbar_wait_bounded(bar(b_xfull + s), ph, &no_abort, p.wait_ns);
      }
    }
  } else if constexpr (MODE != kGemmBf16) {
    // ------------------------------------------------------------- rebuild --
    // Two groups of 4 warps take alternate stages (unit q of this CTA goes to
    // group q % 2), so two tiles are rebuilt while the tensor core consumes.
    // Wide shape: group h rebuilds half h of every unit (W slot 2 j + h).
    const int rt = threadIdx.x - kRebuildWarp0 * 32;  // 0..255
    const int grp = rt >> 7;                           // 0 or 1
    const int gt = rt & 127;                           // thread within the group
    const int WP = wide ? WS / 2 : WS;
    bool ok = true;
    int q = 0;  // index of the unit among this CTA's units
    // ring positions of unit q, advanced for every unit of the CTA
    int stage = 0, wpos = 0;
    uint32_t phase = 0, wphase = 0;
    for (int64_t u = u0; u < u1 && ok;) {
      const int64_t t = u / KB;
      const int kb0 = (int)(u - t * KB);
      const int kb1 = (int)imin64(KB, kb0 + (u1 - u));
      const int64_t nt = t / p.MT;
      for (int kb = kb0; kb < kb1; ++kb, ++q) {
        const int cur_stage = stage, cur_wslot = wide ? 2 * wpos + grp : wpos;
        const uint32_t cur_phase = phase, cur_wphase = wphase;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
        if (++wpos == WP) {
          wpos = 0;
          wphase ^= 1u;
        }
        if (!wide && (q & 1) != grp) continue;
        // every thread observes the stage's TMA completion before reading it
        const bool got = mbar_wait_bounded(bar(b_full + cur_stage), cur_phase, abort, p.wait_ns) &&
                         mbar_wait_bounded(bar(b_wfree + cur_wslot), cur_wphase ^ 1u, abort, p.wait_ns);
        if (!got) set_abort(abort, p.status);
        ok = !__any_sync(0xffffffffu, !got);
        if (!ok) break;
        const uint8_t* st = ring + (size_t)cur_stage * L.bytes;
        // this group's half of the stage: sign+mantissa, exponents or indices,
        // escape bitmap and rows; its 128-row escape group
        const int hh = wide ? grp : 0;
        const uint8_t* sS = st + L.w0 + hh * 8192;
        const uint8_t* sW1 = st + L.w1 + hh * (MODE == kGemmExp ? 8192 : 4096);
        const uint8_t* sEsc = st + L.ebits + hh * kEscArea;
        const int64_t grow = nt * H + hh;
        if (p.tmem_w) {
          // One W row per thread: row r (TMEM lane r, the warp's quadrant) gets
          // K block j's 64 weights in columns 32 j .. 32 j + 31 of the slot.
          // Rows were staged with the TMA swizzle of their width (128, 64 or 32
          // bytes: 16-byte chunk c of row r sits at chunk c ^ (bits 7.. of the
          // row's offset)), so a quarter-warp's 16-byte reads hit distinct banks.
          const int r = 32 * (warp & 3) + lane;
          const int wq = warp & 3;
          const uint32_t sw_rb = 64u * KS;                  // S / E row bytes
          const uint32_t sw_m = sw_rb / 16u - 1u;           // chunk-index swizzle mask
          const uint32_t sw_x = ((uint32_t)r * sw_rb >> 7) & sw_m;
          const uint32_t iw_rb = 32u * KS;                  // index row bytes
          const uint32_t iw_x = ((uint32_t)r * iw_rb >> 7) & (iw_rb / 16u - 1u);
          const uint32_t tcol = tmem_base + ((uint32_t)(32 * wq) << 16) + p.wcol0 +
                                (uint32_t)(cur_wslot * 32 * KS);
          // after the slot's previous MMAs (observed through its free barrier)
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < KS; ++j) {
            uint4 sv[4], ev[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              sv[k] = *reinterpret_cast<const uint4*>(sS + r * sw_rb +
                                                      (((uint32_t)(4 * j + k) ^ sw_x) << 4));
            const uint32_t* s32 = reinterpret_cast<const uint32_t*>(sv);
            uint32_t wv[32];
            bool verbatim = MODE == kGemmExp;  // exponents in ev[] (else W built from indices)
            if (MODE == kGemmExp) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ev[k] = *reinterpret_cast<const uint4*>(sW1 + r * sw_rb +
                                                        (((uint32_t)(4 * j + k) ^ sw_x) << 4));
            } else {
              const uint4 i0 = *reinterpret_cast<const uint4*>(
                  sW1 + r * iw_rb + (((uint32_t)(2 * j) ^ iw_x) << 4));
              const uint4 i1 = *reinterpret_cast<const uint4*>(
                  sW1 + r * iw_rb + (((uint32_t)(2 * j + 1) ^ iw_x) << 4));
              const uint32_t iw[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
              // W straight from the index words (weights 8 m .. 8 m + 7 per word);
              // the choice of form is uniform, so it stays outside the loops
              if (p.pal_run) {
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                  const uint4 w4 = rebuild8_run(iw[m], s32[2 * m], s32[2 * m + 1], p.pal_bias);
                  wv[4 * m] = w4.x;
                  wv[4 * m + 1] = w4.y;
                  wv[4 * m + 2] = w4.z;
                  wv[4 * m + 3] = w4.w;
                }
              } else {
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                  const uint4 w4 = rebuild8_lut(iw[m], s32[2 * m], s32[2 * m + 1], p.palette[0],
                                                p.palette[1], p.palette[2], p.palette[3]);
                  wv[4 * m] = w4.x;
                  wv[4 * m + 1] = w4.y;
                  wv[4 * m + 2] = w4.z;
                  wv[4 * m + 3] = w4.w;
                }
              }
              // escape rows take their verbatim exponents (slot = escape rows
              // before the row in the 128-row group); the warp's 32 rows are one
              // word of the K block's bitmap
              const uint8_t* sEj = sEsc + j * kEscArea;
              const uint4 eb4 = *reinterpret_cast<const uint4*>(sEj);
              const uint32_t word = wq == 0 ? eb4.x : wq == 1 ? eb4.y : wq == 2 ? eb4.z : eb4.w;
              if ((word >> lane) & 1u) {
                verbatim = true;
                const uint32_t before = (wq > 0 ? __popc(eb4.x) : 0) +
                                        (wq > 1 ? __popc(eb4.y) : 0) + (wq > 2 ? __popc(eb4.z) : 0);
                const uint32_t slot = before + (uint32_t)__popc(word & ((1u << lane) - 1u));
                const uint4* src;
                if (slot < (uint32_t)kEscCap) {
                  src = reinterpret_cast<const uint4*>(sEj + 16 + slot * 64);
                } else {
                  const uint32_t first = __ldg(p.esc_off + grow * p.KBK + kb * KS + j);
                  src = reinterpret_cast<const uint4*>(p.esc_exp + (int64_t)(first + slot) * 64);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) ev[k] = src[k];
              }
            }
            if (verbatim) {
              const uint32_t* e32 = reinterpret_cast<const uint32_t*>(ev);
#pragma unroll
              for (int m = 0; m < 16; ++m) {
                const uint2 w2 = merge4(s32[m], e32[m]);
                wv[2 * m] = w2.x;
                wv[2 * m + 1] = w2.y;
              }
            }
            // (the store reads its registers at issue: the next K block may
            // reuse them without waiting for the store to land)
            tmem_st32(tcol + (uint32_t)(32 * j), wv);
          }
          // the stage's inputs are consumed: release it; once the unit's
          // stores have landed, hand the slot over
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(b_empty + cur_stage));
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(b_wfull + cur_wslot));
          continue;
        }
        uint8_t* wt = wring + (size_t)cur_wslot * kWTileBytes;
        // all inputs first (the stores below may alias nothing they read, but
        // the compiler cannot know that), then rebuild and store
        uint2 s8[8];
        uint2 e8[8];
        uint32_t v4[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c8 = gt + 128 * i;
          const int r = c8 >> 3, c = c8 & 7;
          s8[i] = *reinterpret_cast<const uint2*>(sS + r * 64 + c * 8);
          if (MODE == kGemmExp)
            e8[i] = *reinterpret_cast<const uint2*>(sW1 + r * 64 + c * 8);
          else
            v4[i] = *reinterpret_cast<const uint32_t*>(sW1 + r * 32 + c * 4);
        }
        // every item as if no row were an escape row (no branch in the loop, so
        // the items' dependency chains interleave) ...
        // (the palette form is uniform: one loop per form)
        auto store_item = [&](int i, uint4 w4) {
          const int c8 = gt + kGroupThreads * i;
          const int r = c8 >> 3, c = c8 & 7;
          *reinterpret_cast<uint4*>(wt + r * 128 + ((c ^ (r & 7)) << 4)) = w4;
        };
        if (MODE == kGemmExp) {
#pragma unroll
          for (int i = 0; i < kRebuildItems; ++i) {
            const uint2 lo = merge4(s8[i].x, e8[i].x);
            const uint2 hi = merge4(s8[i].y, e8[i].y);
            store_item(i, make_uint4(lo.x, lo.y, hi.x, hi.y));
          }
        } else if (p.pal_run) {
#pragma unroll
          for (int i = 0; i < kRebuildItems; ++i)
            store_item(i, rebuild8_run(v4[i], s8[i].x, s8[i].y, p.pal_bias));
        } else {
#pragma unroll
          for (int i = 0; i < kRebuildItems; ++i)
            store_item(i, rebuild8_lut(v4[i], s8[i].x, s8[i].y, p.palette[0], p.palette[1],
                                       p.palette[2], p.palette[3]));
        }
        // ... then the escape rows.  Thread rows r_i = gt/8 + 16 i, so a warp's
        // 32 rows are bits 4w..4w+3 and 16+4w..16+4w+3 (w = warp in the group) of
        // each 32-row bitmap word: one masked OR tells the whole warp whether
        // any of its rows is an escape row.  Those rows' verbatim exponents (slot
        // = escape rows before the row in the tile) overwrite the 16-byte pieces
        // just written.
        uint4 eb4 = make_uint4(0u, 0u, 0u, 0u);
        if (MODE == kGemmPalette) eb4 = *reinterpret_cast<const uint4*>(sEsc);
        const uint32_t warp_rows = 0x000F000Fu << (4 * (gt >> 5));
        if (MODE == kGemmPalette && ((eb4.x | eb4.y | eb4.z | eb4.w) & warp_rows)) {
          const uint32_t eb[4] = {eb4.x, eb4.y, eb4.z, eb4.w};
          const uint32_t sh = (uint32_t)gt >> 3;
          uint32_t emask = 0;
#pragma unroll
          for (int i = 0; i < kRebuildItems; ++i)
            emask |= ((eb[i >> 1] >> (sh + 16 * (i & 1))) & 1u) << i;
          const uint32_t pc1 = __popc(eb[0]), pc2 = pc1 + __popc(eb[1]),
                         pc3 = pc2 + __popc(eb[2]);
#pragma unroll
          for (int i = 0; i < kRebuildItems; ++i) {
            if (!((emask >> i) & 1u)) continue;
            const int c8 = gt + kGroupThreads * i;
            const int r = c8 >> 3, c = c8 & 7;
            const int w = r >> 5;
            const uint32_t word = w == 0 ? eb[0] : w == 1 ? eb[1] : w == 2 ? eb[2] : eb[3];
            const uint32_t before = w == 0 ? 0u : w == 1 ? pc1 : w == 2 ? pc2 : pc3;
            const uint32_t slot = before + (uint32_t)__popc(word & ((1u << (r & 31)) - 1u));
            uint2 ex;
            if (slot < (uint32_t)kEscCap) {
              ex = *reinterpret_cast<const uint2*>(sEsc + 16 + slot * 64 + c * 8);
            } else {
              const uint32_t first = __ldg(p.esc_off + grow * p.KBK + kb);
              ex = __ldg(reinterpret_cast<const uint2*>(p.esc_exp + (int64_t)(first + slot) * 64 +
                                                        c * 8));
            }
            const uint2 lo = merge4(s8[i].x, ex.x);
            const uint2 hi = merge4(s8[i].y, ex.y);
            *reinterpret_cast<uint4*>(wt + r * 128 + ((c ^ (r & 7)) << 4)) =
                make_uint4(lo.x, lo.y, hi.x, hi.y);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(b_wfull + cur_wslot));
          mbar_arrive(bar(b_empty + cur_stage));
        }
      }
      u += kb1 - kb0;
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair leaves together: the peer's MMAs read this CTA's shared memory
  if constexpr (PAIR) cluster_sync();
  if (warp == kMmaWarp0) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, (uint32_t)p.tmem_cols);
    else
      tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
  }
  // the last CTA to leave advances the epoch for the next launch
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sync + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sync + 1, 0u);
      __threadfence();
      atomicAdd(p.sync, 1u);
    }
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
                 CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int mma_warps_for(int tile_n) { return tile_n <= 128 ? 2 : 1; }

// TMEM columns: two accumulator sets, then (TMEM path) the W slots.
int tmem_cols_for(int tile_n, int w_cols) {
  int c = 32;
  while (c < 2 * mma_warps_for(tile_n) * tile_n + w_cols) c *= 2;
  return c;
}

// K blocks per unit when the reconstructive modes rebuild W into TMEM (the MMA
// then reads A from there, and the shared-memory W ring becomes load stages);
// 0 when W goes through shared memory.  Needs one half per unit and the slots
// (32 columns per K block) beside the accumulators.  Two K blocks per unit
// when K allows: the ring then holds twice the bytes in flight in the same
// number of stages (pure load streams of the 14336x4096 palette form: 35 us
// with one K block per stage, 26 us with two; with 64 KB or more in flight per
// SM every box shape and layout measured the same).
int tmem_ks_for(const GemmArgs& a) {
  if (a.mode == kGemmBf16 || a.halves != 1) return 0;
  const int acc = 2 * mma_warps_for(a.tile_n) * a.tile_n;
  if ((a.K / kBK) % 2 == 0 && acc + 64 * a.wslots <= 512) return 2;
  if (acc + 32 * a.wslots <= 512) return 1;
  return 0;
}

size_t smem_bytes(int mode, int tile_n, int stages, int wslots, int halves, bool tmem_w, int ks,
                  int xstages, bool y_tma, bool pair) {
  const StageLayout L = stage_layout(mode, tile_n, halves, ks);
  const int ws = mode == kGemmBf16 ? 0 : wslots;  // W slots (their barriers exist either way)
  size_t b = 1024 /* alignment slack */ + (size_t)stages * L.bytes;
  b += (size_t)(xstages + (pair ? 1 : 0)) * ks * (pair ? tile_n / 2 : tile_n) * kBK * 2;  // X ring
                                                     // (a pair: half tiles and a spare)
  if (!tmem_w) b += (size_t)ws * kWTileBytes;       // (TMEM path: the slots live in TMEM)
  if (y_tma) b += 2 * kYBlockBytes;                 // Y staging
  b += (size_t)(2 * stages + 2 * xstages + 2 * ws + 7) * 8 + 16;
  return b;
}

template <int MODE, int KS, bool PAIR = false>
cudaError_t set_smem_attr() {
  static cudaError_t e = cudaFuncSetAttribute(
      gemm_kernel<MODE, KS, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  return e;
}

}  // namespace

bool gemm_resolve(GemmArgs* a) {
  if (a->M <= 0 || a->N <= 0 || a->K <= 0 || a->K % kBK) return false;
  // Defaults (measured with X on its own ring, 14336x4096, 4096x14336 and
  // 28672x8192): 128-row units (the wide 256-row shape only on request: it
  // halves the X reads per W row but, with X off the load stage, one
  // 256-token tile that rebuilds W once per 256 tokens wins, e.g. palette
  // M = 1024 on 14336x4096: 171 us against 218).  Token tiles: all of M up
  // to 128 tokens; the reconstructive modes use one tile up to 256 tokens
  // when the matrix has enough 128-row tiles to keep the K splits short
  // (otherwise, 4096x14336 at M = 256: 90 us with 128-token tiles against 102),
  // and 256-token tiles above; the BF16 GEMM keeps 128-token tiles below
  // M = 512 and 256 from there.
  if (a->halves == 0) a->halves = 1;
  if (a->halves != 1 && a->halves != 2) return false;
  const bool wide = a->halves == 2;
  if (a->tile_n == 0) {
    const int64_t row_tiles = (a->N + kBM - 1) / kBM;
    if (a->M <= 128)
      a->tile_n = (int)((a->M + 15) / 16 * 16);
    else if (a->mode == kGemmBf16)
      a->tile_n = a->M >= kWideMinM ? 256 : 128;
    else if (a->M <= 256)
      a->tile_n = 3 * row_tiles >= 2 * (int64_t)a->sm_count ? (int)((a->M + 15) / 16 * 16) : 128;
    else
      a->tile_n = 256;
  }
  if (a->tile_n < 16 || a->tile_n > 256 || a->tile_n % 16) return false;
  // CTA pairs (BF16, one half per unit): one MMA of 256 W rows x 256 tokens
  // over an SM pair, each CTA loading its 128 W rows and half of the tokens
  {
    const bool want = a->pair > 0;  // (on request only)
    if (want && (a->mode != kGemmBf16 || wide)) return false;
    a->pair = want ? 1 : 0;
    if (a->pair) a->tile_n = 256;
  }
  // One half per unit: ring depths are even, consumers alternate units, so an
  // even depth keeps every slot with one consumer (see the MMA issuers).  Wide:
  // every consumer takes every stage, any depth works; W slots go in pairs.
  // As many load stages as fit (up to kMaxStages) beside four rebuilt-W slots
  // (two per rebuild group: with one, a group's next rebuild waits for its
  // last tile's MMA).
  const int max_stages = a->mode == kGemmBf16 ? 12 : kMaxStages;
  const int step = wide ? 1 : 2;
  if (a->wslots == 0) a->wslots = a->mode == kGemmBf16 ? 0 : 4;
  if (a->mode != kGemmBf16 &&
      (a->wslots < 2 || a->wslots > kMaxWSlots || (a->wslots & 1)))
    return false;
  // BF16 Y by TMA stores of 16-token blocks, for token tiles of 128 and more
  // (per-thread 2-byte stores of 256-token tiles cost 20 us at M = 1024;
  // for small tiles the store's completion at the end costs more than it
  // saves), when a tensor map can describe Y (row pitch a multiple of 16 B)
  // and the staging leaves the load ring at least 4 stages (checked below)
  a->y_tma = !a->out_f32 && a->N % 8 == 0 && a->tile_n >= 128;
  const int tks = tmem_ks_for(*a);
  a->tmem_w = tks > 0;
  a->ks = tks > 0 ? tks : 1;
  // X ring: X tiles come from L2; about 48 KB in flight where a rebuild paces
  // the units (96 KB for 256-token tiles: 4096x14336 palette M = 1024 198 ->
  // 170 us), 96 KB (128 KB for 256-token tiles) for the BF16 GEMM whose MMAs
  // take units as fast as they land (32 KB starved it at M = 256); 2..8
  // units, an even number when two MMA warps alternate units
  {
    const int xunit = a->ks * (a->pair ? a->tile_n / 2 : a->tile_n) * kBK * 2;
    // (a pair's CTA: 64 KB, so the W ring keeps 8 stages)
    const int x_target = a->pair ? 65536
                         : a->mode == kGemmBf16 ? (a->tile_n > 128 ? 131072 : 98304)
                                              : (a->tile_n > 128 ? 98304 : 49152);
    int sx = x_target / xunit;
    sx = sx < 2 ? 2 : (sx > 8 ? 8 : sx);
    if (!wide && mma_warps_for(a->tile_n) == 2) sx &= ~1;
    a->xstages = sx;
  }
  if (a->stages == 0) {
    const int wslots0 = a->wslots;
    for (;;) {
      int s = max_stages;
      while (s > 2 && smem_bytes(a->mode, a->tile_n, s, a->wslots, a->halves, a->tmem_w, a->ks, a->xstages, a->y_tma, a->pair != 0) > (size_t)kSmemLimit)
        s -= step;
      if (smem_bytes(a->mode, a->tile_n, s, a->wslots, a->halves, a->tmem_w, a->ks, a->xstages, a->y_tma, a->pair != 0) <= (size_t)kSmemLimit ||
          a->wslots <= 2 || wide) {
        a->stages = s;
        if (a->y_tma && s < 4) {  // the staging would cost too much of the load ring
          a->y_tma = 0;
          a->wslots = wslots0;
          continue;
        }
        break;
      }
      a->wslots -= 2;
    }
  }
  if (a->stages < 2 || (!wide && (a->stages & 1)) ||
      smem_bytes(a->mode, a->tile_n, a->stages, a->wslots, a->halves, a->tmem_w, a->ks, a->xstages, a->y_tma, a->pair != 0) > (size_t)kSmemLimit)
    return false;
  const int64_t RU = (int64_t)kBM * (a->pair ? 2 : a->halves);
  const int64_t NT = (a->N + RU - 1) / RU;
  const int64_t MT = (a->M + a->tile_n - 1) / a->tile_n;
  const int64_t units = NT * MT * (a->K / kBK / a->ks);
  int ctas = a->ctas > 0 ? a->ctas : a->sm_count;
  if (ctas > kGemmMaxCtas) ctas = kGemmMaxCtas;
  if (a->pair) {  // whole pairs, at most one per unit
    const int64_t pairs = imin64(ctas / 2, units);
    if (pairs < 1) return false;
    ctas = (int)(2 * pairs);
  } else if ((int64_t)ctas > units) {
    ctas = (int)units;
  }
  a->ctas = ctas;
  return true;
}

// One partial-sum tile per CTA: a CTA hands over at most one (the split tile
// its range starts in, when it does not hold that tile's first K block).
size_t gemm_partials_bytes(const GemmArgs& a) {
  return (size_t)a.ctas * (size_t)a.tile_n * kBM * (a.halves == 2 ? 2 : 1) * sizeof(float);
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, const LaunchHooks* hooks) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  if (a.ks < 1 || a.ks > 2 || (a.K / kBK) % a.ks) return cudaErrorInvalidValue;  // unresolved
  const int KS = a.ks;
  const int64_t KBK = a.K / kBK;
  const bool wide = a.halves == 2;
  const uint32_t RU = (uint32_t)kBM * (wide ? 2 : 1);
  const bool tw = a.tmem_w != 0;
  if (KS > 1 && (!tw || a.mode == kGemmBf16)) return cudaErrorInvalidValue;
  const bool pair = a.pair != 0;
  if (pair && (a.mode != kGemmBf16 || wide || KS != 1 || a.tile_n % 32)) return cudaErrorInvalidValue;
  // (a pair's CTA loads half of the token tile)
  if (!make_map_2d(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.X, (uint64_t)a.K,
                   (uint64_t)a.M, kBK, (uint32_t)(pair ? a.tile_n / 2 : a.tile_n),
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool ok = true;
  if (a.mode == kGemmBf16) {
    ok = make_map_2d(&p.tm_w0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.W, (uint64_t)a.K,
                     (uint64_t)a.N, kBK, RU, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    // rows rebuilt one per thread (TMEM path) are read 16 bytes at a time
    // along the row: the swizzle of the row's width (KS K blocks: 64 KS bytes of
    // S or E, 32 KS of indices) spreads a warp's rows over the banks
    auto sw_for = [&](int row_bytes) {
      if (!tw) return CU_TENSOR_MAP_SWIZZLE_NONE;
      return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
             : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                               : CU_TENSOR_MAP_SWIZZLE_32B;
    };
    ok = make_map_2d(&p.tm_w0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.S, (uint64_t)a.K,
                     (uint64_t)a.N, kBK * KS, RU, sw_for(kBK * KS));
    if (ok && a.mode == kGemmExp)
      ok = make_map_2d(&p.tm_w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.E, (uint64_t)a.K,
                       (uint64_t)a.N, kBK * KS, RU, sw_for(kBK * KS));
    if (ok && a.mode == kGemmPalette)
      ok = make_map_2d(&p.tm_w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.I, (uint64_t)a.K / 2,
                       (uint64_t)a.N, kBK / 2 * KS, RU, sw_for(kBK / 2 * KS));
  }
  if (!ok) return cudaErrorInvalidValue;
  p.esc_bits = a.esc_bits;
  p.esc_off = a.esc_off;
  p.esc_exp = a.esc_exp;
  p.esc_pack = a.esc_pack;
  p.Y = a.Y;
  p.partials = a.partials;
  p.status = a.status;
  p.sync = a.sync;
  if (!p.sync) return cudaErrorInvalidValue;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.tile_n = a.tile_n;
  p.stages = a.stages;
  p.xstages = a.xstages;
  p.y_tma = 0;
  if (a.y_tma && KS == 1) {
    if (!make_map_2d(&p.tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.Y, (uint64_t)a.N,
                     (uint64_t)a.M, kBM, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    p.y_tma = 1;
  }
  if (p.xstages < 2 || (!wide && mma_warps_for(a.tile_n) == 2 && (p.xstages & 1)))
    return cudaErrorInvalidValue;  // unresolved
  p.wslots = a.wslots;
  p.NT = (int32_t)((a.N + (pair ? 2 * kBM : RU) - 1) / (pair ? 2 * kBM : RU));
  p.NG = (int32_t)((a.N + kBM - 1) / kBM);
  p.halves = wide ? 2 : 1;
  p.MT = (int32_t)((a.M + a.tile_n - 1) / a.tile_n);
  p.KBK = (int32_t)KBK;
  p.ks = KS;
  p.KB = (int32_t)(KBK / KS);
  p.units = (int64_t)p.NT * p.MT * p.KB;
  p.esc_nwp = a.esc_nw;
  p.out_f32 = a.out_f32;
  p.n_mma = wide ? 2 : mma_warps_for(a.tile_n);
  p.tmem_cols = wide ? 512 : tmem_cols_for(a.tile_n, tw ? 32 * KS * a.wslots : 0);
  p.tmem_w = tw ? 1 : 0;
  p.wcol0 = (uint32_t)(2 * mma_warps_for(a.tile_n) * a.tile_n);
  p.acc_bufs = (!wide || 4 * a.tile_n <= 512) ? 2 : 1;  // TMEM: bufs x NM x tile_n columns
  std::memcpy(p.palette, a.palette, 16);
  p.pf_s = a.S;
  p.pf_i = a.w1_resident ? a.I : nullptr;
  p.pal_run = 1;
  for (int i = 1; i < 16; ++i)
    if (a.palette[i] != a.palette[0] + i) p.pal_run = 0;
  p.pal_bias = (uint32_t)a.palette[0] * 128u * 65537u;
  p.x_bytes = (uint32_t)(pair ? a.tile_n / 2 : a.tile_n) * kBK * 2;
  p.stage_bytes = stage_layout(a.mode, a.tile_n, p.halves, KS).bytes;
  p.wait_ns = wait_limit_ns();
  // Failure-detection tests (UW_TEST_WITHHOLD_HANDOFF set in the environment,
  // read once per process): split-tile contributors keep their ready flags
  // back, so every owner's bounded wait runs out and the launch reports a
  // timeout through the status word instead of hanging.
  static const int withhold = std::getenv("UW_TEST_WITHHOLD_HANDOFF") ? 1 : 0;
  p.withhold = withhold;
  const size_t smem =
      smem_bytes(a.mode, a.tile_n, a.stages, a.wslots, p.halves, tw, KS, a.xstages, a.y_tma != 0,
                 a.pair != 0);
  const int G = a.ctas;
  cudaError_t e = cudaSuccess;
  auto begin = [&](int kind) { return hooks && hooks->begin ? hooks->begin(hooks->ctx, kind) : -1; };
  auto end = [&](int slot) {
    if (hooks && hooks->end) hooks->end(hooks->ctx, slot);
  };
  // kinds: 3 bf16, 4 exponent, 5 palette GEMM
  const int slot = begin(3 + a.mode);
  switch (a.mode) {
    case kGemmBf16:
      if (pair) {
        if ((e = set_smem_attr<kGemmBf16, 1, true>()) != cudaSuccess) return e;
        // every pair must be resident at once (owners wait for later pairs'
        // partial sums): at most as many pairs as the GPU holds
        int G2 = G;
        {
          cudaLaunchConfig_t q = {};
          q.gridDim = dim3(G2);
          q.blockDim = dim3(threads_for(kGemmBf16));
          q.dynamicSmemBytes = smem;
          cudaLaunchAttribute ca[1];
          ca[0].id = cudaLaunchAttributeClusterDimension;
          ca[0].val.clusterDim.x = 2;
          ca[0].val.clusterDim.y = 1;
          ca[0].val.clusterDim.z = 1;
          q.attrs = ca;
          q.numAttrs = 1;
          int clusters = 0;
          if ((e = cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel<kGemmBf16, 1, true>, &q)) !=
              cudaSuccess)
            return e;
          if (clusters < 1) return cudaErrorInvalidConfiguration;
          if (G2 > 2 * clusters) G2 = 2 * clusters;
        }
        e = launch_pdl_pair(gemm_kernel<kGemmBf16, 1, true>, G2, threads_for(kGemmBf16), smem, s, p);
      } else {
        if ((e = set_smem_attr<kGemmBf16, 1>()) != cudaSuccess) return e;
        e = launch_pdl(gemm_kernel<kGemmBf16, 1>, G, threads_for(kGemmBf16), smem, s, p);
      }
      break;
    case kGemmExp:
      if (KS == 2) {
        if ((e = set_smem_attr<kGemmExp, 2>()) != cudaSuccess) return e;
        e = launch_pdl(gemm_kernel<kGemmExp, 2>, G, threads_for(kGemmExp), smem, s, p);
      } else {
        if ((e = set_smem_attr<kGemmExp, 1>()) != cudaSuccess) return e;
        e = launch_pdl(gemm_kernel<kGemmExp, 1>, G, threads_for(kGemmExp), smem, s, p);
      }
      break;
    case kGemmPalette:
      if (KS == 2) {
        if ((e = set_smem_attr<kGemmPalette, 2>()) != cudaSuccess) return e;
        e = launch_pdl(gemm_kernel<kGemmPalette, 2>, G, threads_for(kGemmPalette), smem, s, p);
      } else {
        if ((e = set_smem_attr<kGemmPalette, 1>()) != cudaSuccess) return e;
        e = launch_pdl(gemm_kernel<kGemmPalette, 1>, G, threads_for(kGemmPalette), smem, s, p);
      }
      break;
    default:
      return cudaErrorInvalidValue;
  }
  end(slot);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace uw
