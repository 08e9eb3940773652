// Allocation-free GEMM entry point (palette indices prepared at load).
//
// Some callers cannot allocate device memory at the moment they run a matmul:
// code running under an allocator that is locked or exhausted, inference
// loops whose memory was planned once up front, or hosts that forbid
// cudaMalloc on the hot path.  uw_gemm needs a workspace for the split-K
// partial sums; this entry point instead keeps that scratch in a fixed-size
// array compiled into the library, so a call allocates nothing.
//
// Cost of the convenience: every GPU on which the library's device code is
// loaded holds the array (kScratchFloats floats, 5 MiB) until the process
// exits, and all calls share it.
//
// When the array comes into being: the CUDA driver allocates it when it loads
// this file's device module, and with lazy module loading that happens at the
// first lookup of its address.  uw_upload with prepare_direct (the only kind
// of handle this entry point serves) does that lookup, so the allocation
// happens at load time, when the caller can still allocate, not at the first
// matmul.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "handle.h"

namespace {

// Split-K partial sums: up to kMaxCtas CTAs x 64 tokens x 128 rows.
constexpr int kMaxCtas = 160;
constexpr int kMaxM = 64;
constexpr size_t kScratchFloats = (size_t)kMaxCtas * kMaxM * 128;

static __device__ __align__(256) float g_gemm_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {nullptr};

// Look up the scratch array's device address on the current device `dev` and
// remember it (the host-side symbol itself is not a device address).
uw_status lookup_scratch(int dev) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_gemm_scratch) != cudaSuccess || !p) return UW_ERR_CUDA;
  g_scratch_ptr[dev] = static_cast<float*>(p);
  return UW_OK;
}

// The remembered address for the current device `dev`; looked up here only if
// no handle was uploaded with prepare_direct on this device before.
uw_status scratch_for_device(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return UW_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    const uw_status st = lookup_scratch(dev);
    if (st != UW_OK) return st;
  }
  *out = g_scratch_ptr[dev];
  return UW_OK;
}

}  // namespace

namespace uw {
// Called by uw_upload (prepare_direct) with the handle's device current: loads
// the module that holds the array, so the driver allocates it now, and looks
// its address up again.  Looking it up at every such upload also replaces an
// address left over from a context that was destroyed (cudaDeviceReset) and
// recreated since: every handle of the new context passes through here.
void noalloc_prepare_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_mu);
  lookup_scratch(dev);  // a failure here resurfaces as UW_ERR_CUDA at the call
}
}  // namespace uw

extern "C" {

uw_status uw_gemm_palette_noalloc(uw_handle_t h, const uint16_t* X_dev, void* Y_dev, int64_t M,
                                  int32_t out_f32) {
  if (!h || !X_dev || !Y_dev) return UW_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(X_dev) & 15) || (reinterpret_cast<uintptr_t>(Y_dev) & 15))
    return UW_ERR_ARG;
  if (M < 0) return UW_ERR_SHAPE;
  if (M == 0) return UW_OK;
  if (M > kMaxM) return UW_ERR_SHAPE;  // more than the static scratch holds
  if (!h->d_pal_idx) return UW_ERR_UNSUPPORTED;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return UW_ERR_CUDA;
  if (cur != h->device) return UW_ERR_ARG;  // the handle's device must be current
  float* scratch = nullptr;
  uw_status st = scratch_for_device(cur, &scratch);
  if (st != UW_OK) return st;

  uw::GemmArgs a;
  a.mode = uw::kGemmPalette;
  a.M = M;
  a.N = h->N;
  a.K = h->K;
  a.X = X_dev;
  a.S = h->d_sm;
  a.I = h->d_pal_idx;
  a.w1_resident = 1;
  a.esc_bits = h->d_esc_bits;
  a.esc_off = h->d_esc_off;
  a.esc_exp = h->d_esc_exp;
  a.esc_pack = h->d_esc_pack;
  a.esc_nw = (int32_t)(4 * ((h->N + uw::kEscGroupRows - 1) / uw::kEscGroupRows));
  std::memcpy(a.palette, h->palette, 16);
  a.Y = Y_dev;
  a.out_f32 = out_f32 ? 1 : 0;
  a.sm_count = h->sm_count < kMaxCtas ? h->sm_count : kMaxCtas;
  a.status = h->d_status;
  a.sync = h->d_sync;
  if (!uw::gemm_resolve(&a)) return UW_ERR_UNSUPPORTED;
  a.partials_bytes = uw::gemm_partials_bytes(a);
  if (a.partials_bytes > kScratchFloats * sizeof(float)) return UW_ERR_SHAPE;
  // Nothing in the scratch has to start at zero: every partial sum a tile's
  // owner reads is written earlier in the same call (the hand-off flags live
  // in the handle's own zeroed block).
  a.partials = scratch;
  const cudaError_t e = uw::launch_gemm(a, h->stream, nullptr);
  return e == cudaSuccess ? UW_OK : UW_ERR_CUDA;
}

}  // extern "C"
