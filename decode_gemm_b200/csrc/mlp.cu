// MLP stack driver: SwiGLU blocks whose projections run through the
// compressed-weight pipelines, with the preprocessing of "hard" projections
// overlapped on a side stream.
//
// *Unweight*, "Sharing the GPU between decode and compute": layers whose
// projections need Huffman preprocessing ("hard") alternate with layers that
// use palette data prepared at load ("easy"); while the GPU computes, a
// separate CUDA stream decodes the next hard projection's weights, into
// double-buffered preprocessing slots so a slot is not overwritten while it is
// still being read; down_proj, consumed last in the block, gains the most.
// The decoder/GEMM SM split caps both launches so they can run side by side.
//
// Block (per layer l):  g = x W_gate^T,  u = x W_up^T,
//                       h = SiLU(g) * u  (g, u BF16; SiLU and product in FP32,
//                                         result rounded to BF16),
//                       x_{l+1} = h W_down^T.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "handle.h"

using namespace uw;

namespace {

__global__ void swiglu_kernel(const uint16_t* __restrict__ g, const uint16_t* __restrict__ u,
                              uint16_t* __restrict__ h, int64_t n) {
  // 8 elements per thread with 16-byte accesses; a scalar tail
  const int64_t i8 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i8 + 8 <= n) {
    const uint4 gv = *reinterpret_cast<const uint4*>(g + i8);
    const uint4 uv = *reinterpret_cast<const uint4*>(u + i8);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    const uint32_t uw4[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t o = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float gf = __uint_as_float(((gw[j] >> (16 * k)) & 0xFFFFu) << 16);
        const float uf = __uint_as_float(((uw4[j] >> (16 * k)) & 0xFFFFu) << 16);
        const float hf = gf / (1.0f + expf(-gf)) * uf;
        o |= (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hf)) << (16 * k);
      }
      out[j] = o;
    }
    *reinterpret_cast<uint4*>(h + i8) = make_uint4(out[0], out[1], out[2], out[3]);
  } else {
    for (int64_t i = i8; i < n; ++i) {
      const float gf = __uint_as_float((uint32_t)g[i] << 16);
      const float uf = __uint_as_float((uint32_t)u[i] << 16);
      h[i] = __bfloat16_as_ushort(__float2bfloat16_rn(gf / (1.0f + expf(-gf)) * uf));
    }
  }
}

cudaError_t launch_swiglu(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n,
                          cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t threads = (n + 7) / 8;
  const int block = 256;
  const int64_t grid = (threads + block - 1) / block;
  swiglu_kernel<<<(unsigned)grid, block, 0, s>>>(g, u, h, n);
  return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct Plan {
  int64_t D = 0, F = 0;
  size_t off_x0, off_x1, off_g, off_u, off_part, off_slot0, off_slot1, total;
  size_t part_bytes = 0, slot_bytes = 0;
};

struct Proj {
  uw_handle_s* h;
  int which;  // 0 gate, 1 up, 2 down
  uw_gemm_config cfg;
  bool hard;
};

uw_status make_plan(const uw_mlp_layer* layers, int32_t n, int64_t M, const uw_mlp_opts& o,
                    Plan* pl, std::vector<Proj>* projs) {
  if (!layers || n <= 0) return UW_ERR_ARG;
  if (M <= 0 || M > (int64_t(1) << 24)) return UW_ERR_SHAPE;
  Plan p;
  p.D = layers[0].gate ? layers[0].gate->K : 0;
  p.F = layers[0].gate ? layers[0].gate->N : 0;
  projs->clear();
  for (int l = 0; l < n; ++l) {
    uw_handle_s* hh[3] = {layers[l].gate, layers[l].up, layers[l].down};
    for (int j = 0; j < 3; ++j) {
      if (!hh[j]) return UW_ERR_ARG;
      if (hh[j]->device != hh[0]->device) return UW_ERR_ARG;
    }
    if (hh[0]->N != p.F || hh[0]->K != p.D || hh[1]->N != p.F || hh[1]->K != p.D ||
        hh[2]->N != p.D || hh[2]->K != p.F)
      return UW_ERR_SHAPE;
    for (int j = 0; j < 3; ++j) {
      Proj pr;
      pr.h = hh[j];
      pr.which = j;
      pr.cfg = choose_variant(hh[j], M);
      if (o.gemm_ctas > 0 && pr.cfg.gemm_ctas == 0) pr.cfg.gemm_ctas = o.gemm_ctas;
      const uw_status st = check_config(hh[j], pr.cfg);
      if (st != UW_OK) return st;
      pr.hard = needs_preprocess(pr.cfg.pipeline);
      GemmArgs a;
      size_t need = 0, pre = 0;
      const uw_status ps = plan_gemm(hh[j], nullptr, nullptr, M, pr.cfg, 0, &a, &need, &pre);
      if (ps != UW_OK) return ps;
      p.part_bytes = std::max(p.part_bytes, a.partials_bytes);
      if (pr.hard) p.slot_bytes = std::max(p.slot_bytes, preprocessed_bytes(hh[j], pr.cfg.pipeline));
      projs->push_back(pr);
    }
  }
  size_t off = 0;
  auto place = [&](size_t b) {
    const size_t at = off;
    off = align256(off + b);
    return at;
  };
  p.off_x0 = place((size_t)M * p.D * 2);
  p.off_x1 = place((size_t)M * p.D * 2);
  p.off_g = place((size_t)M * p.F * 2);
  p.off_u = place((size_t)M * p.F * 2);
  p.off_part = place(std::max<size_t>(p.part_bytes, 256));
  p.off_slot0 = place(std::max<size_t>(p.slot_bytes, 256));
  p.off_slot1 = o.overlap ? place(std::max<size_t>(p.slot_bytes, 256)) : p.off_slot0;
  p.total = off;
  *pl = p;
  return UW_OK;
}

uw_mlp_opts opts_or_default(const uw_mlp_opts* o) {
  uw_mlp_opts d;
  std::memset(&d, 0, sizeof(d));
  if (o) d = *o;
  return d;
}

}  // namespace

extern "C" {

uw_status uw_swiglu(const uint16_t* g_dev, const uint16_t* u_dev, uint16_t* h_dev, int64_t n,
                    void* stream) {
  if (n < 0) return UW_ERR_SHAPE;
  if (n == 0) return UW_OK;
  if (!g_dev || !u_dev || !h_dev) return UW_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(g_dev) | reinterpret_cast<uintptr_t>(u_dev) |
       reinterpret_cast<uintptr_t>(h_dev)) & 15)
    return UW_ERR_ARG;
  return launch_swiglu(g_dev, u_dev, h_dev, n, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? UW_OK
             : UW_ERR_CUDA;
}

uw_status uw_mlp_workspace_bytes(const uw_mlp_layer* layers, int32_t n_layers, int64_t M,
                                 const uw_mlp_opts* opts, size_t* bytes) {
  if (!bytes) return UW_ERR_ARG;
  Plan pl;
  std::vector<Proj> projs;
  const uw_status st = make_plan(layers, n_layers, M, opts_or_default(opts), &pl, &projs);
  if (st != UW_OK) return st;
  *bytes = pl.total;
  return UW_OK;
}

}  // extern "C"

namespace {

// The stacked forward; when act is not null, each layer's g, u, h and output
// are also copied there (main stream, right after they are produced).
uw_status mlp_forward(const uw_mlp_layer* layers, int32_t n_layers, const uint16_t* X_dev,
                      uint16_t* Y_dev, int64_t M, void* ws_dev, size_t ws_bytes, void* stream,
                      void* side_stream, const uw_mlp_opts* opts, uint16_t* act) {
  const uw_mlp_opts o = opts_or_default(opts);
  if (o.decode_ctas < 0 || o.gemm_ctas < 0) return UW_ERR_ARG;
  Plan pl;
  std::vector<Proj> projs;
  uw_status st = make_plan(layers, n_layers, M, o, &pl, &projs);
  if (st != UW_OK) return st;
  if (!X_dev || !Y_dev || !ws_dev) return UW_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(X_dev) | reinterpret_cast<uintptr_t>(Y_dev)) & 15)
    return UW_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(ws_dev) & 255) return UW_ERR_ARG;
  if (ws_bytes < pl.total) return UW_ERR_WORKSPACE;
  if (o.overlap && !side_stream) return UW_ERR_ARG;
  DeviceGuard g(projs[0].h->device);
  cudaStream_t ms = static_cast<cudaStream_t>(stream);
  cudaStream_t ss = o.overlap ? static_cast<cudaStream_t>(side_stream) : ms;
  uint8_t* ws = static_cast<uint8_t*>(ws_dev);
  uint16_t* xb[2] = {reinterpret_cast<uint16_t*>(ws + pl.off_x0),
                     reinterpret_cast<uint16_t*>(ws + pl.off_x1)};
  uint16_t* gbuf = reinterpret_cast<uint16_t*>(ws + pl.off_g);
  uint16_t* ubuf = reinterpret_cast<uint16_t*>(ws + pl.off_u);
  float* part = reinterpret_cast<float*>(ws + pl.off_part);
  uint8_t* slot[2] = {ws + pl.off_slot0, ws + pl.off_slot1};

  // hard projections in order of use
  std::vector<int> hard;
  for (size_t i = 0; i < projs.size(); ++i)
    if (projs[i].hard) hard.push_back((int)i);
  cudaEvent_t ready[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
  if (o.overlap) {
    for (int i = 0; i < 2; ++i) {
      if (cudaEventCreateWithFlags(&ready[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&freed[i], cudaEventDisableTiming) != cudaSuccess)
        return UW_ERR_CUDA;
    }
  }
  auto cleanup = [&]() {
    for (int i = 0; i < 2; ++i) {
      if (ready[i]) cudaEventDestroy(ready[i]);
      if (freed[i]) cudaEventDestroy(freed[i]);
    }
  };
  // side stream: preprocess hard projection k into slot k % 2
  std::vector<bool> freed_recorded(2, false);
  auto enqueue_pre = [&](size_t k) -> uw_status {
    const Proj& pr = projs[hard[k]];
    const int sl = (int)(k & 1);
    if (o.overlap && freed_recorded[sl] &&
        cudaStreamWaitEvent(ss, freed[sl], 0) != cudaSuccess)
      return UW_ERR_CUDA;
    const uw_status r = run_preprocess(pr.h, pr.cfg.pipeline, slot[sl],
                                       o.overlap ? o.decode_ctas : pr.cfg.decode_ctas, ss);
    if (r != UW_OK) return r;
    if (o.overlap && cudaEventRecord(ready[sl], ss) != cudaSuccess) return UW_ERR_CUDA;
    return UW_OK;
  };
  if (o.overlap && !hard.empty()) {
    // the side stream writes a slot only after all main-stream work enqueued
    // so far (an earlier call may still be reading either slot)
    for (int i = 0; i < 2; ++i) {
      if (cudaEventRecord(freed[i], ms) != cudaSuccess) {
        cleanup();
        return UW_ERR_CUDA;
      }
      freed_recorded[i] = true;
    }
    st = enqueue_pre(0);
  }
  const size_t xbytes = (size_t)M * pl.D * 2;
  const size_t fbytes = (size_t)M * pl.F * 2;
  // act layout per layer: g [M, F], u [M, F], h [M, F], output [M, D]
  const size_t act_layer = (size_t)M * (3 * pl.F + pl.D);
  auto record = [&](int layer, int part, const uint16_t* src, size_t bytes) -> uw_status {
    if (!act) return UW_OK;
    uint16_t* dst = act + (size_t)layer * act_layer + (size_t)part * M * pl.F;
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, ms) == cudaSuccess
               ? UW_OK
               : UW_ERR_CUDA;
  };
  if (st == UW_OK && cudaMemcpyAsync(xb[0], X_dev, xbytes, cudaMemcpyDeviceToDevice, ms) != cudaSuccess)
    st = UW_ERR_CUDA;
  size_t hk = 0;  // index into `hard` of the next hard projection
  int cur = 0;
  for (size_t i = 0; i < projs.size() && st == UW_OK; ++i) {
    const Proj& pr = projs[i];
    const uint16_t* in = pr.which == 2 ? gbuf : xb[cur];
    uint16_t* out = pr.which == 0 ? gbuf : (pr.which == 1 ? ubuf : xb[cur ^ 1]);
    const void* pre = nullptr;
    if (pr.hard) {
      const int sl = (int)(hk & 1);
      if (o.overlap) {
        if (hk + 1 < hard.size()) st = enqueue_pre(hk + 1);  // look one hard projection ahead
        if (st == UW_OK && cudaStreamWaitEvent(ms, ready[sl], 0) != cudaSuccess) st = UW_ERR_CUDA;
      } else {
        st = enqueue_pre(hk);
      }
      pre = slot[sl];
    }
    if (st == UW_OK)
      st = run_gemm_on(pr.h, in, out, M, pr.cfg, 0, pre, part, pl.part_bytes, ms);
    if (st == UW_OK && pr.hard) {
      if (o.overlap) {
        if (cudaEventRecord(freed[hk & 1], ms) != cudaSuccess) st = UW_ERR_CUDA;
        freed_recorded[hk & 1] = true;
      }
      ++hk;
    }
    const int layer = (int)(i / 3);
    if (st == UW_OK && pr.which == 0) st = record(layer, 0, gbuf, fbytes);
    if (st == UW_OK && pr.which == 1) st = record(layer, 1, ubuf, fbytes);
    if (st == UW_OK && pr.which == 1) {  // h = SiLU(g) * u, in place over g
      if (launch_swiglu(gbuf, ubuf, gbuf, M * pl.F, ms) != cudaSuccess) st = UW_ERR_CUDA;
      if (st == UW_OK) st = record(layer, 2, gbuf, fbytes);
    }
    if (st == UW_OK && pr.which == 2) st = record(layer, 3, xb[cur ^ 1], xbytes);
    if (pr.which == 2) cur ^= 1;
  }
  if (st == UW_OK &&
      cudaMemcpyAsync(Y_dev, xb[cur], xbytes, cudaMemcpyDeviceToDevice, ms) != cudaSuccess)
    st = UW_ERR_CUDA;
  cleanup();
  return st;
}

}  // namespace

extern "C" {

uw_status uw_mlp_forward(const uw_mlp_layer* layers, int32_t n_layers, const uint16_t* X_dev,
                         uint16_t* Y_dev, int64_t M, void* ws_dev, size_t ws_bytes,
                         void* stream, void* side_stream, const uw_mlp_opts* opts) {
  return mlp_forward(layers, n_layers, X_dev, Y_dev, M, ws_dev, ws_bytes, stream, side_stream,
                     opts, nullptr);
}

uw_status uw_mlp_forward_record(const uw_mlp_layer* layers, int32_t n_layers,
                                const uint16_t* X_dev, uint16_t* Y_dev, int64_t M, void* ws_dev,
                                size_t ws_bytes, void* stream, void* side_stream,
                                const uw_mlp_opts* opts, uint16_t* act_dev) {
  if (!act_dev || (reinterpret_cast<uintptr_t>(act_dev) & 15)) return UW_ERR_ARG;
  return mlp_forward(layers, n_layers, X_dev, Y_dev, M, ws_dev, ws_bytes, stream, side_stream,
                     opts, act_dev);
}

uw_status uw_mlp_tune_split(const uw_mlp_layer* layers, int32_t n_layers, const uint16_t* X_dev,
                            uint16_t* Y_dev, int64_t M, void* ws_dev, size_t ws_bytes,
                            void* stream, void* side_stream, uw_mlp_opts* best) {
  if (!best || !side_stream) return UW_ERR_ARG;
  if (!layers || n_layers <= 0 || !layers[0].gate) return UW_ERR_ARG;
  const int sms = layers[0].gate->sm_count;
  // (decoder CTAs, GEMM CTAs): no split, then the decoder on a few SMs
  std::vector<std::pair<int, int>> splits = {{0, 0}};
  for (int d : {4, 8, 16, 24})
    if (d < sms) splits.push_back({d, sms - d});  // one decoder CTA per SM
  cudaStream_t ms = static_cast<cudaStream_t>(stream);
  cudaEvent_t a = nullptr, b = nullptr;
  if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return UW_ERR_CUDA;
  float best_ms = 1e30f;
  uw_mlp_opts best_o;
  std::memset(&best_o, 0, sizeof(best_o));
  uw_status st = UW_OK;
  for (const auto& sp : splits) {
    uw_mlp_opts o;
    std::memset(&o, 0, sizeof(o));
    o.overlap = 1;
    o.decode_ctas = sp.first;
    o.gemm_ctas = sp.second;
    float t_best = 1e30f;
    for (int r = 0; r < 4 && st == UW_OK; ++r) {
      cudaEventRecord(a, ms);
      st = uw_mlp_forward(layers, n_layers, X_dev, Y_dev, M, ws_dev, ws_bytes, stream, side_stream,
                          &o);
      cudaEventRecord(b, ms);
      if (st != UW_OK) break;
      if (cudaEventSynchronize(b) != cudaSuccess) {
        st = UW_ERR_CUDA;
        break;
      }
      float t = 0.f;
      cudaEventElapsedTime(&t, a, b);
      if (r > 0) t_best = std::min(t_best, t);  // first run warms up
    }
    if (st != UW_OK) break;
    if (t_best < best_ms) {
      best_ms = t_best;
      best_o = o;
    }
  }
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (st != UW_OK) return st;
  *best = best_o;
  return UW_OK;
}

}  // extern "C"
