// Device-resident encoded matrix (the object behind uw_handle_t).
#pragma once

#include <cuda_runtime.h>

#include <map>
#include <vector>

#include "uw_internal.h"
#include "uw_kernels.h"

struct uw_handle_s {
  int device = 0;
  int sm_count = 148;
  cudaStream_t stream = nullptr;

  int64_t N = 0, K = 0;
  int32_t chunk_syms = 1024, max_code_len = 12;
  uint8_t code_len[256] = {0};
  uint8_t palette[16] = {0};
  uw::DecodeTables tables;
  int64_t n_words = 0, n_chunks = 0, n_esc_words = 0, n_esc_groups = 0, n_esc_rows = 0;
  std::vector<int64_t> hist;  // exponent histogram when known (for statistics)

  // one device allocation holding every array below
  void* d_block = nullptr;
  uint32_t* d_words = nullptr;
  uint32_t* d_chunk_off = nullptr;
  uint32_t* d_lut = nullptr;
  uint32_t* d_canon = nullptr;
  uint8_t* d_sm = nullptr;
  uint32_t* d_esc_bits = nullptr;
  uint32_t* d_esc_off = nullptr;
  uint8_t* d_esc_exp = nullptr;
  // per escape group g = (n/128, kb): its 16-byte row bitmap, then its escape
  // rows (64 bytes each), at byte 16 g + 64 esc_off[g] (one copy per GEMM unit)
  uint8_t* d_esc_pack = nullptr;
  uint32_t* d_status = nullptr;
  uint32_t* d_sync = nullptr;    // GEMM split-K hand-off (kGemmSyncWords, zeroed at upload)
  uint8_t* d_pal_idx = nullptr;  // resident palette indices (pipeline 4), may be null
  uint32_t* d_row_cnt = nullptr; // Huffman-direct product: N row arrival counters (zeroed)

  // workspace for pipelines 1-3 and split-K partial sums
  void* ws = nullptr;
  size_t ws_bytes = 0;
  bool ws_owned = false;

  // autotuned choices: M -> variant (nearest M at or above is used)
  std::map<int64_t, uw_gemm_config> profile;

  // kernel tracing (uw_trace_enable): event pairs around each launch
  bool trace = false;
  std::vector<cudaEvent_t> trace_events;  // pool, 2 per launch
  std::vector<int32_t> trace_kinds;
};

namespace uw {
DecodeArgs decode_args(const uw_handle_s* h);
// Shared by the C ABI, the autotuner and the MLP driver (api.cu).
uw_gemm_config choose_variant(const uw_handle_s* h, int64_t M);
uw_status check_config(const uw_handle_s* h, const uw_gemm_config& cfg);
bool use_gemv(const uw_gemm_config& c, int64_t M);
bool gemv_for(const uw_handle_s* h, const uw_gemm_config& cfg, int64_t M);
// The Huffman-direct product (pipeline 5) serves (handle, M).
bool dot_for(const uw_handle_s* h, int64_t M);
// Does the pipeline need a preprocessing pass (pipelines 1-3)?
inline bool needs_preprocess(int pipeline) { return pipeline >= 1 && pipeline <= 3; }
size_t preprocessed_bytes(const uw_handle_s* h, int pipeline);
uw_status plan_gemm(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M,
                    const uw_gemm_config& cfg, int out_f32, GemmArgs* ga, size_t* ws_need,
                    size_t* pre_bytes);
uw_status run_preprocess(uw_handle_s* h, int pipeline, void* out, int ctas, cudaStream_t s);
uw_status run_gemm_on(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M,
                      const uw_gemm_config& cfg, int out_f32, const void* pre, float* partials,
                      size_t partials_bytes, cudaStream_t s);
uw_status run_gemm(uw_handle_s* h, const uint16_t* X, void* Y, int64_t M,
                   const uw_gemm_config& cfg, int out_f32);
struct DeviceGuard {
  int prev = -1;
  bool changed = false;
  explicit DeviceGuard(int dev);
  ~DeviceGuard();
};
// Record the start event of a traced launch (no-op unless tracing); returns the
// slot to pass to trace_end, or -1.
int trace_begin(uw_handle_s* h, int kind);
void trace_end(uw_handle_s* h, int slot);
// Allocation-free matmul (noalloc.cu): make the scratch array of device `dev`
// (current) exist and remember its address; called when a handle is uploaded
// with the load-time palette transcode.
void noalloc_prepare_device(int dev);
}
