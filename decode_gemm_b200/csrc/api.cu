// C ABI, device side: upload, preprocessing entry points, GEMM dispatch over
// the four pipelines and the Huffman-direct product, workspace and status
// handling.
//
// *Unweight*, "Four ways to use compressed weights": pipeline 1 decodes to
// BF16 in HBM and runs a plain GEMM; pipeline 2 decodes exponent bytes only,
// pipeline 3 transcodes to 4-bit palette indices at run time, pipeline 4 uses
// indices transcoded once at load; 2-4 run the reconstructive GEMM.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <new>

#include "handle.h"

using namespace uw;

namespace {

uw_status map_cuda(cudaError_t e) {
  if (e == cudaSuccess) return UW_OK;
  if (e == cudaErrorMemoryAllocation) return UW_ERR_OOM;
  return UW_ERR_CUDA;
}

#define UW_CK(x)                                  \
  do {                                            \
    cudaError_t e_ = (x);                         \
    if (e_ != cudaSuccess) return map_cuda(e_);   \
  } while (0)


size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

void free_handle(uw_handle_s* h) {
  if (!h) return;
  DeviceGuard g(h->device);
  for (cudaEvent_t ev : h->trace_events) cudaEventDestroy(ev);
  if (h->d_block) cudaFree(h->d_block);
  if (h->ws_owned && h->ws) cudaFree(h->ws);
  delete h;
}

// bytes of preprocessed weights a pipeline writes to the workspace
size_t preprocess_bytes(const uw_handle_s* h, int pipeline) {
  const size_t T = (size_t)h->N * (size_t)h->K;
  switch (pipeline) {
    case UW_PIPE_FULL: return 2 * T;
    case UW_PIPE_EXP: return T;
    case UW_PIPE_PALETTE_RT: return T / 2;
    default: return 0;
  }
}

GemmArgs base_gemm_args(const uw_handle_s* h) {
  GemmArgs a;
  a.N = h->N;
  a.K = h->K;
  a.S = h->d_sm;
  a.esc_bits = h->d_esc_bits;
  a.esc_off = h->d_esc_off;
  a.esc_exp = h->d_esc_exp;
  a.esc_pack = h->d_esc_pack;
  a.esc_nw = (int32_t)(4 * ((h->N + kEscGroupRows - 1) / kEscGroupRows));
  std::memcpy(a.palette, h->palette, 16);
  a.sm_count = h->sm_count;
  a.status = h->d_status;
  a.sync = h->d_sync;
  return a;
}

bool valid_pipeline(int p) { return p >= UW_PIPE_FULL && p <= UW_PIPE_HUFFMAN_DIRECT; }

// Workspace bytes of the Huffman-direct product's partial sums.
size_t dot_part_bytes(const uw_handle_s* h) {
  return align_up((size_t)dot_part_floats(h->n_chunks) * 4, 256);
}

}  // namespace

namespace uw {
// Make the handle's device current for the scope of a call.
DeviceGuard::DeviceGuard(int dev) {
  if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) changed = cudaSetDevice(dev) == cudaSuccess;
}
DeviceGuard::~DeviceGuard() {
  if (changed) cudaSetDevice(prev);
}

DecodeArgs decode_args(const uw_handle_s* h) {
  DecodeArgs a;
  a.words = h->d_words;
  a.chunk_off = h->d_chunk_off;
  a.lut = h->d_lut;
  a.canon = h->d_canon;
  std::memcpy(a.palette, h->palette, 16);
  bool run = true;
  for (int i = 1; i < 16; ++i)
    if (h->palette[i] != h->palette[0] + i) run = false;
  a.pal_run_b4 = run ? (uint32_t)h->palette[0] * 0x01010101u : 0xFFFFFFFFu;
  a.sm = h->d_sm;
  a.esc_bits = h->d_esc_bits;
  a.status = h->d_status;
  a.n_words = h->n_words;
  a.n_chunks = h->n_chunks;
  a.total_syms = h->N * h->K;
  a.chunk_syms = h->chunk_syms;
  a.kb_per_row = (int32_t)(h->K / kRow);
  a.esc_nw = (int32_t)(4 * ((h->N + kEscGroupRows - 1) / kEscGroupRows));
  return a;
}

// Choose the variant for (handle, M): the profile entry for the smallest tuned
// M at or above the request (else the largest), otherwise a static default.
uw_gemm_config choose_variant(const uw_handle_s* h, int64_t M) {
  uw_gemm_config c;
  std::memset(&c, 0, sizeof(c));
  if (!h->profile.empty()) {
    auto it = h->profile.lower_bound(M);
    if (it == h->profile.end()) --it;
    c = it->second;
    if (c.pipeline == UW_PIPE_PALETTE_DIRECT && !h->d_pal_idx) c.pipeline = UW_PIPE_PALETTE_RT;
    // an entry tuned for fewer tokens may name a kernel that does not serve M:
    // the tensor-core GEMM of its pipeline, or the default pipeline, instead
    if (c.gemv > 0 && M > kGemvMaxM) c.gemv = 0;
    if (c.pipeline == UW_PIPE_HUFFMAN_DIRECT && !dot_for(h, M)) {
      std::memset(&c, 0, sizeof(c));
      c.pipeline = h->d_pal_idx ? UW_PIPE_PALETTE_DIRECT : UW_PIPE_PALETTE_RT;
    }
    return c;
  }
  c.pipeline = h->d_pal_idx ? UW_PIPE_PALETTE_DIRECT : UW_PIPE_PALETTE_RT;
  return c;
}

constexpr int kTraceCap = 16384;

int trace_begin(uw_handle_s* h, int kind) {
  if (!h->trace || (int)h->trace_kinds.size() >= kTraceCap) return -1;
  const int slot = (int)h->trace_kinds.size();
  while ((int)h->trace_events.size() < 2 * (slot + 1)) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return -1;
    h->trace_events.push_back(ev);
  }
  if (cudaEventRecord(h->trace_events[2 * slot], h->stream) != cudaSuccess) return -1;
  h->trace_kinds.push_back(kind);
  return slot;
}

void trace_end(uw_handle_s* h, int slot) {
  if (slot >= 0) cudaEventRecord(h->trace_events[2 * slot + 1], h->stream);
}

static int hook_begin(void* ctx, int kind) { return trace_begin(static_cast<uw_handle_s*>(ctx), kind); }
static void hook_end(void* ctx, int slot) { trace_end(static_cast<uw_handle_s*>(ctx), slot); }

bool dot_for(const uw_handle_s* h, int64_t M) {
  return dot_supported(h->K, h->chunk_syms, M);
}

// The Huffman-direct product Y = X W^T (pipeline 5), partial sums in `part`.
uw_status run_dot_on(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M, int out_f32,
                     int ctas, float* part, size_t part_bytes, cudaStream_t s) {
  if (!dot_for(h, M)) return UW_ERR_UNSUPPORTED;
  if (!part || part_bytes < (size_t)dot_part_floats(h->n_chunks) * 4) return UW_ERR_WORKSPACE;
  DecodeArgs a = decode_args(h);
  a.cpr = (int32_t)(h->K / h->chunk_syms);
  a.matrix_rows = h->N;
  a.x = X;
  a.y = Y;
  a.m = (int32_t)M;
  a.out_f32 = out_f32;
  a.part = part;
  a.row_cnt = h->d_row_cnt;
  // (from the device's SM count, not the launch's: the summation order, and so
  // the result, does not depend on an SM budget)
  a.run = dot_run_length(h->N, a.cpr, h->sm_count);
  const int slot = trace_begin(h, UW_KERNEL_DECODE_DOT);
  const cudaError_t e = launch_decode(kDecodeDot, a, nullptr, ctas, s);
  trace_end(h, slot);
  return map_cuda(e);
}

uw_status run_decode(uw_handle_s* h, int mode, void* out, int ctas, cudaStream_t s) {
  DecodeArgs a = decode_args(h);
  // kinds: 0 full, 1 exponent, 2 transcode
  const int kind = mode == kDecodeFull ? 0 : (mode == kDecodeExp ? 1 : 2);
  const int slot = trace_begin(h, kind);
  const cudaError_t e = launch_decode(mode, a, out, ctas, s);
  trace_end(h, slot);
  return map_cuda(e);
}

// Resolve a GEMM request into kernel arguments and the workspace it needs.
uw_status plan_gemm(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M,
                    const uw_gemm_config& cfg, int out_f32, GemmArgs* ga, size_t* ws_need,
                    size_t* pre_bytes) {
  GemmArgs a = base_gemm_args(h);
  a.M = M;
  a.X = X;
  a.Y = Y;
  a.out_f32 = out_f32;
  if (cfg.pipeline == UW_PIPE_HUFFMAN_DIRECT) {  // one kernel: partial sums only
    if (!dot_for(h, M)) return UW_ERR_UNSUPPORTED;
    a.partials_bytes = dot_part_bytes(h);
    *pre_bytes = 0;
    *ws_need = a.partials_bytes;
    *ga = a;
    return UW_OK;
  }
  a.tile_n = cfg.tile_n;
  a.stages = cfg.stages;
  a.halves = cfg.halves;
  a.pair = cfg.pair ? 1 : -1;
  a.ctas = cfg.gemm_ctas;
  switch (cfg.pipeline) {
    case UW_PIPE_FULL: a.mode = kGemmBf16; break;
    case UW_PIPE_EXP: a.mode = kGemmExp; break;
    default: a.mode = kGemmPalette; break;
  }
  if (!gemm_resolve(&a)) return UW_ERR_UNSUPPORTED;
  const size_t pre = align_up(preprocess_bytes(h, cfg.pipeline), 256);
  a.partials_bytes = gemm_partials_bytes(a);
  *pre_bytes = pre;
  *ws_need = pre + a.partials_bytes;
  *ga = a;
  return UW_OK;
}

// Whether a request runs on the matrix-vector kernel (uw_gemm_config.gemv = 1;
// the autotuner tries it at M <= 2 and keeps it where it measures faster).
bool use_gemv(const uw_gemm_config& c, int64_t M) { return c.gemv > 0 && M <= kGemvMaxM; }

uw_status check_config(const uw_handle_s* h, const uw_gemm_config& cfg) {
  if (!valid_pipeline(cfg.pipeline)) return UW_ERR_ARG;
  if (cfg.gemv < 0 || cfg.gemv > 1) return UW_ERR_ARG;
  if (cfg.pipeline == UW_PIPE_PALETTE_DIRECT && !h->d_pal_idx) return UW_ERR_UNSUPPORTED;
  if (cfg.tile_n < 0 || cfg.tile_n > 256 || cfg.tile_n % 16) return UW_ERR_ARG;
  if (cfg.halves < 0 || cfg.halves > 2) return UW_ERR_ARG;
  if (cfg.pair < 0 || cfg.pair > 1 || (cfg.pair && cfg.halves == 2)) return UW_ERR_ARG;
  if (cfg.pair && cfg.pipeline != UW_PIPE_FULL) return UW_ERR_UNSUPPORTED;
  if (cfg.gemv && cfg.pipeline == UW_PIPE_HUFFMAN_DIRECT) return UW_ERR_ARG;
  if (cfg.stages < 0 || cfg.stages > 16 || (cfg.halves != 2 && (cfg.stages & 1)))
    return UW_ERR_ARG;
  if (cfg.gemm_ctas < 0 || cfg.decode_ctas < 0) return UW_ERR_ARG;
  return UW_OK;
}

size_t preprocessed_bytes(const uw_handle_s* h, int pipeline) {
  return preprocess_bytes(h, pipeline);
}

uw_status run_preprocess(uw_handle_s* h, int pipeline, void* out, int ctas, cudaStream_t s) {
  switch (pipeline) {
    case UW_PIPE_FULL: return run_decode(h, kDecodeFull, out, ctas, s);
    case UW_PIPE_EXP: return run_decode(h, kDecodeExp, out, ctas, s);
    case UW_PIPE_PALETTE_RT: return run_decode(h, kDecodePalette, out, ctas, s);
    default: return UW_OK;
  }
}

// The GEMM of a pipeline on weights already preprocessed into `pre` (ignored
// for pipeline 4), partial sums in `partials` (gemm_partials_bytes of the plan).
// The matrix-vector kernel for (handle, pipeline) on weights already
// preprocessed into `pre` (ignored for pipeline 4).
uw_status run_gemv_on(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M, int pipeline,
                      int out_f32, const void* pre, cudaStream_t s) {
  if (M > kGemvMaxM) return UW_ERR_UNSUPPORTED;
  GemmArgs a = base_gemm_args(h);
  a.M = M;
  a.X = X;
  a.Y = Y;
  a.out_f32 = out_f32;
  switch (pipeline) {
    case UW_PIPE_FULL:
      a.mode = kGemmBf16;
      a.W = static_cast<const uint16_t*>(pre);
      break;
    case UW_PIPE_EXP:
      a.mode = kGemmExp;
      a.E = static_cast<const uint8_t*>(pre);
      break;
    case UW_PIPE_PALETTE_RT:
      a.mode = kGemmPalette;
      a.I = static_cast<const uint8_t*>(pre);
      break;
    default:
      a.mode = kGemmPalette;
      a.I = h->d_pal_idx;
      a.w1_resident = 1;
      break;
  }
  if (!gemv_supported(a)) return UW_ERR_UNSUPPORTED;
  LaunchHooks hooks;
  hooks.ctx = h;
  hooks.begin = hook_begin;
  hooks.end = hook_end;
  return map_cuda(launch_gemv(a, s, &hooks));
}

// The matrix-vector kernel serves (handle, M, variant).
bool gemv_for(const uw_handle_s* h, const uw_gemm_config& cfg, int64_t M) {
  (void)h;
  return use_gemv(cfg, M);
}

uw_status run_gemm_on(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M,
                      const uw_gemm_config& cfg, int out_f32, const void* pre, float* partials,
                      size_t partials_bytes, cudaStream_t s) {
  if (cfg.pipeline == UW_PIPE_HUFFMAN_DIRECT)
    return run_dot_on(h, X, Y, M, out_f32, cfg.gemm_ctas, partials, partials_bytes, s);
  if (gemv_for(h, cfg, M)) return run_gemv_on(h, X, Y, M, cfg.pipeline, out_f32, pre, s);
  GemmArgs a;
  size_t need = 0, pre_b = 0;
  uw_status st = plan_gemm(h, X, Y, M, cfg, out_f32, &a, &need, &pre_b);
  if (st != UW_OK) return st;
  if (a.partials_bytes > partials_bytes) return UW_ERR_WORKSPACE;
  a.partials = a.partials_bytes ? partials : nullptr;
  switch (cfg.pipeline) {
    case UW_PIPE_FULL: a.W = static_cast<const uint16_t*>(pre); break;
    case UW_PIPE_EXP: a.E = static_cast<const uint8_t*>(pre); break;
    case UW_PIPE_PALETTE_RT: a.I = static_cast<const uint8_t*>(pre); break;
    default:
      a.I = h->d_pal_idx;
      a.w1_resident = 1;
      break;
  }
  LaunchHooks hooks;
  hooks.ctx = h;
  hooks.begin = hook_begin;
  hooks.end = hook_end;
  return map_cuda(launch_gemm(a, s, &hooks));
}

uw_status run_gemm(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M,
                   const uw_gemm_config& cfg_in, int out_f32) {
  uw_gemm_config cfg = cfg_in;
  if (cfg.pipeline == UW_PIPE_AUTO) {
    const uw_gemm_config c = choose_variant(h, M);
    cfg = c;
  }
  uw_status st = check_config(h, cfg);
  if (st != UW_OK) return st;
  if (cfg.gemv > 0 && M > kGemvMaxM) return UW_ERR_UNSUPPORTED;
  if (cfg.pipeline == UW_PIPE_HUFFMAN_DIRECT) {
    if (!dot_for(h, M)) return UW_ERR_UNSUPPORTED;
    return run_dot_on(h, X, Y, M, out_f32, cfg.gemm_ctas, static_cast<float*>(h->ws),
                      h->ws_bytes, h->stream);
  }
  if (gemv_for(h, cfg, M)) {
    // preprocessed weights (pipelines 1-3) in the workspace; no partial sums
    const size_t pre_b = align_up(preprocess_bytes(h, cfg.pipeline), 256);
    if (pre_b > 0 && (!h->ws || h->ws_bytes < pre_b)) return UW_ERR_WORKSPACE;
    if (cfg.pipeline != UW_PIPE_PALETTE_DIRECT) {
      const int mode = cfg.pipeline == UW_PIPE_FULL
                           ? kDecodeFull
                           : (cfg.pipeline == UW_PIPE_EXP ? kDecodeExp : kDecodePalette);
      st = run_decode(h, mode, h->ws, cfg.decode_ctas, h->stream);
      if (st != UW_OK) return st;
    }
    return run_gemv_on(h, X, Y, M, cfg.pipeline, out_f32, h->ws, h->stream);
  }
  GemmArgs a;
  size_t need = 0, pre = 0;
  st = plan_gemm(h, X, Y, M, cfg, out_f32, &a, &need, &pre);
  if (st != UW_OK) return st;
  if (need > 0 && (!h->ws || h->ws_bytes < need)) return UW_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(h->ws);
  a.partials = a.partials_bytes ? reinterpret_cast<float*>(ws + pre) : nullptr;
  cudaStream_t s = h->stream;
  switch (cfg.pipeline) {
    case UW_PIPE_FULL:
      st = run_decode(h, kDecodeFull, ws, cfg.decode_ctas, s);
      a.W = reinterpret_cast<const uint16_t*>(ws);
      break;
    case UW_PIPE_EXP:
      st = run_decode(h, kDecodeExp, ws, cfg.decode_ctas, s);
      a.E = ws;
      break;
    case UW_PIPE_PALETTE_RT:
      st = run_decode(h, kDecodePalette, ws, cfg.decode_ctas, s);
      a.I = ws;
      break;
    default:
      a.I = h->d_pal_idx;
      break;
  }
  if (st != UW_OK) return st;
  LaunchHooks hooks;
  hooks.ctx = h;
  hooks.begin = hook_begin;
  hooks.end = hook_end;
  return map_cuda(launch_gemm(a, s, &hooks));
}
}  // namespace uw

extern "C" {

uw_status uw_upload(const uw_format* f, const uw_encode_opts* opts, void* stream,
                    uw_handle_t* out) {
  if (!out) return UW_ERR_ARG;
  *out = nullptr;
  const uw_status vs = uw_validate_format(f);
  if (vs != UW_OK) return vs;
  uw_encode_opts o;
  uw_default_encode_opts(&o);
  if (opts) o = *opts;
  uw_handle_s* h = new (std::nothrow) uw_handle_s();
  if (!h) return UW_ERR_OOM;
  if (!build_decode_tables(f->code_len, f->palette, &h->tables)) {
    delete h;
    return UW_ERR_FORMAT;
  }
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return UW_ERR_CUDA;
  }
  cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, h->device);
  h->stream = static_cast<cudaStream_t>(stream);
  h->N = f->N;
  h->K = f->K;
  h->chunk_syms = f->chunk_syms;
  h->max_code_len = f->max_code_len;
  std::memcpy(h->code_len, f->code_len, 256);
  std::memcpy(h->palette, f->palette, 16);
  h->n_words = f->n_words;
  h->n_chunks = f->n_chunks;
  h->n_esc_words = f->n_esc_words;
  h->n_esc_groups = f->n_esc_groups;
  h->n_esc_rows = f->n_esc_rows;

  const size_t T = (size_t)f->N * (size_t)f->K;
  struct Part { void** dst; const void* src; size_t bytes; };
  size_t off = 0;
  auto place = [&](size_t bytes) { size_t at = off; off = align_up(off + bytes, 256); return at; };
  // the stream is followed by zero words: the decoder reads past a chunk's end
  const int64_t pad_words = stream_pad_words(f->chunk_syms);
  const size_t o_words = place((size_t)(f->n_words + pad_words) * 4);
  const size_t o_coff = place((size_t)(f->n_chunks + 1) * 4);
  const size_t o_lut = place(kLutSize * 4);
  const size_t o_canon = place(kCanonWords * 4);
  const size_t o_sm = place(T);
  const size_t o_ebits = place((size_t)std::max<int64_t>(f->n_esc_words, 1) * 4);
  const size_t o_eoff = place((size_t)(f->n_esc_groups + 1) * 4);
  const size_t o_eexp = place((size_t)std::max<int64_t>(f->n_esc_rows, 1) * kRow);
  const size_t pack_bytes = (size_t)f->n_esc_groups * 16 + (size_t)f->n_esc_rows * kRow;
  const size_t o_epack = place(std::max<size_t>(pack_bytes, 16));
  const size_t o_stat = place(256);
  const size_t o_sync = place(kGemmSyncWords * 4);
  const size_t o_pidx = o.prepare_direct ? place(T / 2) : 0;
  const size_t o_rcnt = place((size_t)f->N * 4);
  cudaError_t e = cudaMalloc(&h->d_block, off);
  if (e != cudaSuccess) {
    delete h;
    return map_cuda(e);
  }
  uint8_t* base = static_cast<uint8_t*>(h->d_block);
  h->d_words = reinterpret_cast<uint32_t*>(base + o_words);
  h->d_chunk_off = reinterpret_cast<uint32_t*>(base + o_coff);
  h->d_lut = reinterpret_cast<uint32_t*>(base + o_lut);
  h->d_canon = reinterpret_cast<uint32_t*>(base + o_canon);
  h->d_sm = base + o_sm;
  h->d_esc_bits = reinterpret_cast<uint32_t*>(base + o_ebits);
  h->d_esc_off = reinterpret_cast<uint32_t*>(base + o_eoff);
  h->d_esc_exp = base + o_eexp;
  h->d_esc_pack = base + o_epack;
  // escape groups packed for the GEMM: bitmap of the group's 128 rows, then its rows
  std::vector<uint8_t> pack(pack_bytes);
  {
    const int64_t KB = f->K / kRow, nwp = 4 * ((f->N + kEscGroupRows - 1) / kEscGroupRows);
    for (int64_t g = 0; g < f->n_esc_groups; ++g) {
      const int64_t nt = g / KB, kb = g % KB;
      uint8_t* dst = pack.data() + 16 * g + (size_t)f->esc_off[g] * kRow;
      std::memcpy(dst, f->esc_bits + kb * nwp + nt * 4, 16);
      std::memcpy(dst + 16, f->esc_exp + (size_t)f->esc_off[g] * kRow,
                  (size_t)(f->esc_off[g + 1] - f->esc_off[g]) * kRow);
    }
  }
  h->d_status = reinterpret_cast<uint32_t*>(base + o_stat);
  h->d_sync = reinterpret_cast<uint32_t*>(base + o_sync);
  h->d_pal_idx = o.prepare_direct ? base + o_pidx : nullptr;
  h->d_row_cnt = reinterpret_cast<uint32_t*>(base + o_rcnt);
  cudaStream_t s = h->stream;
  const Part parts[] = {
      {(void**)&h->d_words, f->words, (size_t)f->n_words * 4},
      {(void**)&h->d_chunk_off, f->chunk_off, (size_t)(f->n_chunks + 1) * 4},
      {(void**)&h->d_lut, h->tables.lut.data(), kLutSize * 4},
      {(void**)&h->d_canon, h->tables.canon, kCanonWords * 4},
      {(void**)&h->d_sm, f->sm, T},
      {(void**)&h->d_esc_bits, f->esc_bits, (size_t)f->n_esc_words * 4},
      {(void**)&h->d_esc_off, f->esc_off, (size_t)(f->n_esc_groups + 1) * 4},
      {(void**)&h->d_esc_exp, f->esc_exp, (size_t)f->n_esc_rows * kRow},
      {(void**)&h->d_esc_pack, pack.data(), pack_bytes},
  };
  for (const Part& p : parts) {
    if (p.bytes == 0) continue;
    e = cudaMemcpyAsync(*p.dst, p.src, p.bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) break;
  }
  if (e == cudaSuccess)
    e = cudaMemsetAsync(h->d_words + f->n_words, 0, (size_t)pad_words * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->d_status, 0, 256, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->d_sync, 0, kGemmSyncWords * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->d_row_cnt, 0, (size_t)f->N * 4, s);
  if (e == cudaSuccess && h->d_pal_idx) {
    // load-time transcode: the resident palette form of pipeline 4
    DecodeArgs a = decode_args(h);
    e = launch_decode(kDecodePalette, a, h->d_pal_idx, 0, s);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    free_handle(h);
    return map_cuda(e);
  }
  // the allocation-free matmul serves handles with resident indices: its
  // scratch array is brought into being now, while allocating is allowed
  if (h->d_pal_idx) noalloc_prepare_device(h->device);
  *out = h;
  return UW_OK;
}

uw_status uw_encode(const uint16_t* w_host, int64_t N, int64_t K, const uw_encode_opts* opts,
                    void* stream, uw_handle_t* out) {
  if (!out) return UW_ERR_ARG;
  *out = nullptr;
  uw_host_t hh = nullptr;
  uw_status st = uw_encode_host(w_host, N, K, opts, &hh);
  if (st != UW_OK) return st;
  uw_format f;
  uw_host_view(hh, &f);
  st = uw_upload(&f, opts, stream, out);
  if (st == UW_OK) (*out)->hist = hh->enc.hist;
  uw_host_free(hh);
  return st;
}

uw_status uw_free(uw_handle_t h) {
  if (!h) return UW_ERR_ARG;
  free_handle(h);
  return UW_OK;
}

uw_status uw_set_stream(uw_handle_t h, void* stream) {
  if (!h) return UW_ERR_ARG;
  h->stream = static_cast<cudaStream_t>(stream);
  return UW_OK;
}

uw_status uw_stats(uw_handle_t h, uw_stats_t* out) {
  if (!h || !out) return UW_ERR_ARG;
  uw_format f;
  std::memset(&f, 0, sizeof(f));
  f.N = h->N;
  f.K = h->K;
  std::memcpy(f.code_len, h->code_len, 256);
  std::memcpy(f.palette, h->palette, 16);
  f.n_chunks = h->n_chunks;
  f.n_words = h->n_words;
  f.n_esc_words = h->n_esc_words;
  f.n_esc_groups = h->n_esc_groups;
  f.n_esc_rows = h->n_esc_rows;
  // total bits = last chunk offset (read back from the device)
  uint32_t last = 0;
  DeviceGuard g(h->device);
  UW_CK(cudaMemcpy(&last, h->d_chunk_off + h->n_chunks, 4, cudaMemcpyDeviceToHost));
  std::vector<uint32_t> coff((size_t)h->n_chunks + 1, 0);
  coff.back() = last;
  f.chunk_off = coff.data();
  fill_stats(f, h->hist.empty() ? nullptr : h->hist.data(), out);
  return UW_OK;
}

uw_status uw_workspace_bytes(uw_handle_t h, int32_t pipeline, int64_t M, size_t* bytes) {
  if (!h || !bytes) return UW_ERR_ARG;
  if (M < 0) return UW_ERR_SHAPE;
  uw_gemm_config c;
  std::memset(&c, 0, sizeof(c));
  c.pipeline = pipeline;
  if (pipeline == UW_PIPE_AUTO) c = choose_variant(h, M);
  if (!valid_pipeline(c.pipeline)) return UW_ERR_ARG;
  if (M == 0) {
    *bytes = 0;
    return UW_OK;
  }
  // enough for any variant: every token tile (16..256), both unit shapes and
  // up to one CTA per SM
  size_t worst = 0;
  for (int hv = 1; hv <= 2; ++hv)
    for (int tn = 16; tn <= 256; tn += 16) {
      uw_gemm_config v = c;
      v.tile_n = tn;
      v.stages = 2;
      v.halves = hv;
      v.gemm_ctas = h->sm_count;
      GemmArgs a;
      size_t need = 0, pre = 0;
      if (plan_gemm(h, nullptr, nullptr, M, v, 1, &a, &need, &pre) == UW_OK)
        worst = std::max(worst, need);
    }
  if (!worst) return UW_ERR_UNSUPPORTED;
  *bytes = worst;
  return UW_OK;
}

uw_status uw_set_workspace(uw_handle_t h, void* ws_dev, size_t bytes) {
  if (!h) return UW_ERR_ARG;
  if (ws_dev && (reinterpret_cast<uintptr_t>(ws_dev) & 255)) return UW_ERR_ARG;
  DeviceGuard g(h->device);
  if (h->ws_owned && h->ws) cudaFree(h->ws);
  h->ws = ws_dev;
  h->ws_bytes = ws_dev ? bytes : 0;
  h->ws_owned = false;
  return UW_OK;
}

uw_status uw_alloc_workspace(uw_handle_t h, size_t bytes) {
  if (!h) return UW_ERR_ARG;
  DeviceGuard g(h->device);
  void* p = nullptr;
  if (bytes) UW_CK(cudaMalloc(&p, bytes));
  if (h->ws_owned && h->ws) cudaFree(h->ws);
  h->ws = p;
  h->ws_bytes = bytes;
  h->ws_owned = bytes != 0;
  return UW_OK;
}

static uw_status check_out_ptr(const void* p) {
  if (!p) return UW_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(p) & 15) return UW_ERR_ARG;
  return UW_OK;
}

uw_status uw_decode_full(uw_handle_t h, uint16_t* w_dev) {
  if (!h) return UW_ERR_ARG;
  uw_status st = check_out_ptr(w_dev);
  if (st != UW_OK) return st;
  DeviceGuard g(h->device);
  return run_decode(h, kDecodeFull, w_dev, 0, h->stream);
}

uw_status uw_decode_exp(uw_handle_t h, uint8_t* e_dev) {
  if (!h) return UW_ERR_ARG;
  uw_status st = check_out_ptr(e_dev);
  if (st != UW_OK) return st;
  DeviceGuard g(h->device);
  return run_decode(h, kDecodeExp, e_dev, 0, h->stream);
}

uw_status uw_transcode_palette(uw_handle_t h, uint8_t* idx_dev) {
  if (!h) return UW_ERR_ARG;
  uw_status st = check_out_ptr(idx_dev);
  if (st != UW_OK) return st;
  DeviceGuard g(h->device);
  return run_decode(h, kDecodePalette, idx_dev, 0, h->stream);
}

uw_status uw_decode_rows(uw_handle_t h, const int64_t* rows_dev, int64_t n_rows,
                         uint16_t* w_dev) {
  if (!h) return UW_ERR_ARG;
  if (n_rows < 0) return UW_ERR_SHAPE;
  if (n_rows == 0) return UW_OK;
  if (!rows_dev || (reinterpret_cast<uintptr_t>(rows_dev) & 7)) return UW_ERR_ARG;
  uw_status st = check_out_ptr(w_dev);
  if (st != UW_OK) return st;
  if (h->K % h->chunk_syms) return UW_ERR_UNSUPPORTED;  // rows must be whole chunks
  DeviceGuard g(h->device);
  DecodeArgs a = decode_args(h);
  a.cpr = (int32_t)(h->K / h->chunk_syms);
  a.rows = rows_dev;
  a.gather_rows = n_rows;
  a.matrix_rows = h->N;
  a.n_chunks = n_rows * a.cpr;
  a.total_syms = n_rows * h->K;
  const int slot = trace_begin(h, UW_KERNEL_DECODE_FULL);
  const cudaError_t e = launch_decode(kDecodeFull, a, w_dev, 0, h->stream);
  trace_end(h, slot);
  return map_cuda(e);
}

uw_status uw_gemm_ex(uw_handle_t h, const uint16_t* X_dev, void* Y_dev, int64_t M,
                     const uw_gemm_config* cfg, int32_t out_f32) {
  if (!h || !cfg) return UW_ERR_ARG;
  if (M < 0 || M > (int64_t(1) << 24)) return UW_ERR_SHAPE;
  if (M == 0) return UW_OK;
  if (check_out_ptr(X_dev) != UW_OK || check_out_ptr(Y_dev) != UW_OK) return UW_ERR_ARG;
  DeviceGuard g(h->device);
  return run_gemm(h, X_dev, Y_dev, M, *cfg, out_f32 ? 1 : 0);
}

uw_status uw_gemm(uw_handle_t h, const uint16_t* X_dev, uint16_t* Y_dev, int64_t M,
                  uw_pipeline pipeline) {
  uw_gemm_config c;
  std::memset(&c, 0, sizeof(c));
  c.pipeline = pipeline;
  if (pipeline != UW_PIPE_AUTO && !valid_pipeline(pipeline)) return UW_ERR_ARG;
  return uw_gemm_ex(h, X_dev, Y_dev, M, &c, 0);
}

uw_status uw_gemm_f32(uw_handle_t h, const uint16_t* X_dev, float* Y_dev, int64_t M,
                      uw_pipeline pipeline) {
  uw_gemm_config c;
  std::memset(&c, 0, sizeof(c));
  c.pipeline = pipeline;
  if (pipeline != UW_PIPE_AUTO && !valid_pipeline(pipeline)) return UW_ERR_ARG;
  return uw_gemm_ex(h, X_dev, Y_dev, M, &c, 1);
}

uw_status uw_trace_enable(uw_handle_t h, int32_t enable) {
  if (!h) return UW_ERR_ARG;
  h->trace = enable != 0;
  return UW_OK;
}

uw_status uw_trace_read(uw_handle_t h, int32_t* kinds, float* ms, int32_t capacity,
                        int32_t* count) {
  if (!h || !count || capacity < 0 || (capacity > 0 && (!kinds || !ms))) return UW_ERR_ARG;
  DeviceGuard g(h->device);
  UW_CK(cudaStreamSynchronize(h->stream));
  const int n = (int)h->trace_kinds.size();
  *count = n;
  for (int i = 0; i < n && i < capacity; ++i) {
    kinds[i] = h->trace_kinds[i];
    float t = 0.f;
    if (cudaEventElapsedTime(&t, h->trace_events[2 * i], h->trace_events[2 * i + 1]) != cudaSuccess)
      t = -1.f;
    ms[i] = t;
  }
  h->trace_kinds.clear();
  return UW_OK;
}

uw_status uw_last_device_status(uw_handle_t h) {
  if (!h) return UW_ERR_ARG;
  DeviceGuard g(h->device);
  UW_CK(cudaStreamSynchronize(h->stream));
  uint32_t st = 0;
  UW_CK(cudaMemcpy(&st, h->d_status, 4, cudaMemcpyDeviceToHost));
  // cleared on the handle's own stream (which need not synchronise with the
  // legacy default stream) and waited for, so no later launch can race it
  UW_CK(cudaMemsetAsync(h->d_status, 0, 4, h->stream));
  UW_CK(cudaStreamSynchronize(h->stream));
  if (st & kStatusTimeout) return UW_ERR_TIMEOUT;
  if (st & kStatusBadChunk) return UW_ERR_DEVICE;
  return UW_OK;
}

}  // extern "C"
