// Autotuner and per-model profile I/O.
//
// *Unweight*, "Sharing the GPU between decode and compute" (closing
// paragraphs): the configuration space (pipeline, matmul variant, decoder/GEMM
// SM split) is too large to hard-code, so the runtime measures real
// throughput on the target GPU: it sweeps the candidates of the gate
// projection with up and down fixed, then up, then down, repeating until no
// change improves the result, and records the winner per projection and per
// batch size in a per-model profile.
//
// Here: for every M, every handle in turn tries each candidate variant while
// the others keep theirs; a candidate is scored by the device time (CUDA
// events, best of several runs) of the whole sequence of the handles'
// matmuls, so interactions between projections (L2 reuse, launch gaps) count.
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <cctype>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "handle.h"

using namespace uw;

namespace {

struct Timer {
  cudaEvent_t a = nullptr, b = nullptr;
  Timer() {
    cudaEventCreate(&a);
    cudaEventCreate(&b);
  }
  ~Timer() {
    if (a) cudaEventDestroy(a);
    if (b) cudaEventDestroy(b);
  }
};

// Candidate variants for (handle, M).
std::vector<uw_gemm_config> candidates(const uw_handle_s* h, int64_t M) {
  std::vector<int> tiles = {0};
  const int m16 = (int)std::min<int64_t>(256, (M + 15) / 16 * 16);
  for (int t : {16, 32, 64, 128, 256})
    if (t <= std::max(16, 2 * m16) && (M <= 256 || t >= 128)) tiles.push_back(t);
  std::vector<uw_gemm_config> out;
  if (dot_for(h, M)) {  // the Huffman-direct product: one kernel, no preprocessing
    uw_gemm_config c;
    std::memset(&c, 0, sizeof(c));
    c.pipeline = UW_PIPE_HUFFMAN_DIRECT;
    out.push_back(c);
  }
  for (int p = UW_PIPE_FULL; p <= UW_PIPE_PALETTE_DIRECT; ++p) {
    if (p == UW_PIPE_PALETTE_DIRECT && !h->d_pal_idx) continue;
    if (M <= kGemvMaxM) {  // the matrix-vector kernel on the CUDA cores, if it fits
      uw_gemm_config c;
      std::memset(&c, 0, sizeof(c));
      c.pipeline = p;
      c.gemv = 1;
      GemmArgs a;
      a.M = M;
      a.N = h->N;
      a.K = h->K;
      a.mode = p == UW_PIPE_FULL ? kGemmBf16 : (p == UW_PIPE_EXP ? kGemmExp : kGemmPalette);
      if (gemv_supported(a)) out.push_back(c);
    }
    for (int t : tiles)
      for (int st : {0, 4})
        for (int hv : {0, 1, 2}) {
          // the wide shape (on request only) could pay from a few token
          // tiles on; one half per unit is the automatic choice
          if (hv == 2 && M < 256) continue;
          if (hv == 1) continue;
          uw_gemm_config c;
          std::memset(&c, 0, sizeof(c));
          c.pipeline = p;
          c.tile_n = t;
          c.stages = st;
          c.halves = hv;
          out.push_back(c);
          // the BF16 GEMM on CTA pairs (256-token tiles)
          if (p == UW_PIPE_FULL && M >= 256 && hv != 2 && (t == 0 || t == 256)) {
            c.pair = 1;
            c.tile_n = 256;
            out.push_back(c);
          }
        }
  }
  return out;
}

bool fits(uw_handle_s* h, int64_t M, const uw_gemm_config& c) {
  if (check_config(h, c) != UW_OK) return false;
  if (gemv_for(h, c, M)) {  // preprocessed weights only
    const size_t need = preprocessed_bytes(h, c.pipeline);
    return need == 0 || (h->ws && h->ws_bytes >= need);
  }
  GemmArgs a;
  size_t need = 0, pre = 0;
  if (plan_gemm(h, nullptr, nullptr, M, c, 0, &a, &need, &pre) != UW_OK) return false;
  return need == 0 || (h->ws && h->ws_bytes >= need);
}

// Device milliseconds of one pass over all handles (best of `reps`).
uw_status time_sequence(const std::vector<uw_handle_s*>& hs, const std::vector<uw_gemm_config>& cfg,
                        int64_t M, const uint16_t* X, uint16_t* Y, cudaStream_t s, Timer& tm,
                        int reps, float* best_ms) {
  float best = 1e30f;
  for (int r = 0; r < reps + 1; ++r) {
    if (cudaEventRecord(tm.a, s) != cudaSuccess) return UW_ERR_CUDA;
    for (size_t i = 0; i < hs.size(); ++i) {
      const uw_status st = run_gemm(hs[i], X, Y, M, cfg[i], 0);
      if (st != UW_OK) return st;
    }
    if (cudaEventRecord(tm.b, s) != cudaSuccess) return UW_ERR_CUDA;
    if (cudaEventSynchronize(tm.b) != cudaSuccess) return UW_ERR_CUDA;
    float ms = 0.f;
    cudaEventElapsedTime(&ms, tm.a, tm.b);
    if (r > 0) best = std::min(best, ms);  // the first pass warms up
  }
  *best_ms = best;
  return UW_OK;
}

// ------------------------------------------------------------- tiny JSON ----

struct JVal {
  enum Kind { Null, Num, Str, Arr, Obj } kind = Null;
  double num = 0;
  std::string str;
  std::vector<JVal> arr;
  std::vector<std::pair<std::string, JVal>> obj;
  const JVal* get(const char* k) const {
    for (const auto& kv : obj)
      if (kv.first == k) return &kv.second;
    return nullptr;
  }
};

struct JParser {
  const char* p;
  const char* end;
  bool ok = true;
  void ws() {
    while (p < end && std::isspace((unsigned char)*p)) ++p;
  }
  bool lit(const char* s) {
    const size_t n = std::strlen(s);
    if ((size_t)(end - p) >= n && std::strncmp(p, s, n) == 0) {
      p += n;
      return true;
    }
    return false;
  }
  JVal value(int depth = 0) {
    JVal v;
    ws();
    if (p >= end || depth > 32) {
      ok = false;
      return v;
    }
    if (*p == '{') {
      ++p;
      v.kind = JVal::Obj;
      ws();
      if (p < end && *p == '}') {
        ++p;
        return v;
      }
      while (ok) {
        ws();
        JVal k = value(depth + 1);
        if (k.kind != JVal::Str) {
          ok = false;
          break;
        }
        ws();
        if (p >= end || *p != ':') {
          ok = false;
          break;
        }
        ++p;
        v.obj.emplace_back(k.str, value(depth + 1));
        ws();
        if (p < end && *p == ',') {
          ++p;
          continue;
        }
        if (p < end && *p == '}') {
          ++p;
          break;
        }
        ok = false;
      }
    } else if (*p == '[') {
      ++p;
      v.kind = JVal::Arr;
      ws();
      if (p < end && *p == ']') {
        ++p;
        return v;
      }
      while (ok) {
        v.arr.push_back(value(depth + 1));
        ws();
        if (p < end && *p == ',') {
          ++p;
          continue;
        }
        if (p < end && *p == ']') {
          ++p;
          break;
        }
        ok = false;
      }
    } else if (*p == '"') {
      ++p;
      v.kind = JVal::Str;
      while (p < end && *p != '"') v.str.push_back(*p++);
      if (p >= end) ok = false;
      else ++p;
    } else if (lit("null") || lit("true") || lit("false")) {
      v.kind = JVal::Null;
    } else {
      char* e = nullptr;
      v.num = std::strtod(p, &e);
      if (e == p) ok = false;
      p = e;
      v.kind = JVal::Num;
    }
    return v;
  }
};

bool num_field(const JVal& o, const char* k, int64_t* out) {
  const JVal* v = o.get(k);
  // (a number outside the int64 range, or not finite, is not a field value)
  if (!v || v->kind != JVal::Num || !(std::fabs(v->num) < 9.0e18)) return false;
  *out = (int64_t)v->num;
  return true;
}

}  // namespace

extern "C" {

uw_status uw_autotune(uw_handle_t* hs_in, int32_t n_handles, const int64_t* Ms, int32_t n_M,
                      const char* profile_out_json) {
  if (!hs_in || n_handles <= 0 || !Ms || n_M <= 0) return UW_ERR_ARG;
  std::vector<uw_handle_s*> hs(hs_in, hs_in + n_handles);
  for (auto* h : hs)
    if (!h || h->device != hs[0]->device) return UW_ERR_ARG;
  for (int i = 0; i < n_M; ++i)
    if (Ms[i] <= 0) return UW_ERR_SHAPE;
  DeviceGuard g(hs[0]->device);
  const cudaStream_t s = hs[0]->stream;
  int64_t kmax = 0, nmax = 0, mmax = 0;
  for (auto* h : hs) {
    kmax = std::max(kmax, h->K);
    nmax = std::max(nmax, h->N);
  }
  for (int i = 0; i < n_M; ++i) mmax = std::max(mmax, Ms[i]);
  // Measurement buffers: the tuner runs at set-up time and allocates them.
  uint16_t *X = nullptr, *Y = nullptr;
  if (cudaMalloc(&X, (size_t)mmax * kmax * 2) != cudaSuccess) return UW_ERR_OOM;
  if (cudaMalloc(&Y, (size_t)mmax * nmax * 2) != cudaSuccess) {
    cudaFree(X);
    return UW_ERR_OOM;
  }
  cudaMemsetAsync(X, 0x3C, (size_t)mmax * kmax * 2, s);  // BF16 0x3C3C (~0.0115)
  std::vector<cudaStream_t> saved;
  for (auto* h : hs) {
    saved.push_back(h->stream);
    h->stream = s;  // one stream: the sequence is timed end to end
  }
  uw_status st = UW_OK;
  std::vector<std::vector<std::pair<int64_t, uw_gemm_config>>> chosen(hs.size());
  std::vector<std::vector<float>> chosen_ms(hs.size());
  {
    Timer tm;
    for (int mi = 0; mi < n_M && st == UW_OK; ++mi) {
      const int64_t M = Ms[mi];
      std::vector<uw_gemm_config> cfg(hs.size());
      for (size_t i = 0; i < hs.size(); ++i) {
        // start from the library default that fits the registered workspace
        cfg[i] = choose_variant(hs[i], M);
        if (!fits(hs[i], M, cfg[i])) {
          bool found = false;
          for (const auto& c : candidates(hs[i], M))
            if (fits(hs[i], M, c)) {
              cfg[i] = c;
              found = true;
              break;
            }
          if (!found) {
            st = UW_ERR_WORKSPACE;
            break;
          }
        }
      }
      if (st != UW_OK) break;
      float best = 0.f;
      st = time_sequence(hs, cfg, M, X, Y, s, tm, 3, &best);
      for (int sweep = 0; sweep < 3 && st == UW_OK; ++sweep) {
        bool improved = false;
        for (size_t i = 0; i < hs.size() && st == UW_OK; ++i) {
          uw_gemm_config best_c = cfg[i];  // the others stay fixed while handle i is swept
          for (const auto& c : candidates(hs[i], M)) {
            if (!fits(hs[i], M, c)) continue;
            cfg[i] = c;
            float t = 0.f;
            st = time_sequence(hs, cfg, M, X, Y, s, tm, 3, &t);
            if (st != UW_OK) break;
            if (t < best * 0.99f) {  // a 1 % gain, not noise
              best = t;
              best_c = c;
              improved = true;
            }
          }
          cfg[i] = best_c;
        }
        if (!improved) break;
      }
      if (st != UW_OK) break;
      // record the winners, with each handle's own time at the winning choice
      for (size_t i = 0; i < hs.size(); ++i) {
        std::vector<uw_handle_s*> one = {hs[i]};
        std::vector<uw_gemm_config> oc = {cfg[i]};
        float t = 0.f;
        st = time_sequence(one, oc, M, X, Y, s, tm, 3, &t);
        if (st != UW_OK) break;
        chosen[i].push_back({M, cfg[i]});
        chosen_ms[i].push_back(t);
      }
    }
  }
  for (size_t i = 0; i < hs.size(); ++i) hs[i]->stream = saved[i];
  cudaFree(X);
  cudaFree(Y);
  if (st != UW_OK) return st;
  for (size_t i = 0; i < hs.size(); ++i) {
    hs[i]->profile.clear();
    for (const auto& mc : chosen[i]) hs[i]->profile[mc.first] = mc.second;
  }
  if (profile_out_json) {
    FILE* f = std::fopen(profile_out_json, "w");
    if (!f) return UW_ERR_ARG;
    std::fprintf(f, "{\n  \"version\": 1,\n  \"handles\": [\n");
    for (size_t i = 0; i < hs.size(); ++i) {
      std::fprintf(f, "    {\"N\": %lld, \"K\": %lld, \"choices\": [\n", (long long)hs[i]->N,
                   (long long)hs[i]->K);
      for (size_t j = 0; j < chosen[i].size(); ++j) {
        const auto& c = chosen[i][j].second;
        std::fprintf(f,
                     "      {\"M\": %lld, \"pipeline\": %d, \"tile_n\": %d, \"stages\": %d, "
                     "\"gemm_ctas\": %d, \"decode_ctas\": %d, \"halves\": %d, \"pair\": %d, "
                     "\"gemv\": %d, \"us\": %.2f}%s\n",
                     (long long)chosen[i][j].first, c.pipeline, c.tile_n, c.stages, c.gemm_ctas,
                     c.decode_ctas, c.halves, c.pair, c.gemv, 1e3 * chosen_ms[i][j],
                     j + 1 < chosen[i].size() ? "," : "");
      }
      std::fprintf(f, "    ]}%s\n", i + 1 < hs.size() ? "," : "");
    }
    std::fprintf(f, "  ]\n}\n");
    std::fclose(f);
  }
  return UW_OK;
}

uw_status uw_load_profile(uw_handle_t* hs, int32_t n_handles, const char* profile_json) {
  if (!hs || n_handles <= 0 || !profile_json) return UW_ERR_ARG;
  FILE* f = std::fopen(profile_json, "rb");
  if (!f) return UW_ERR_ARG;
  std::string text;
  char buf[4096];
  size_t n;
  while ((n = std::fread(buf, 1, sizeof(buf), f)) > 0) text.append(buf, n);
  std::fclose(f);
  JParser jp{text.data(), text.data() + text.size()};
  const JVal root = jp.value();
  if (!jp.ok || root.kind != JVal::Obj) return UW_ERR_FORMAT;
  const JVal* handles = root.get("handles");
  if (!handles || handles->kind != JVal::Arr || (int)handles->arr.size() != n_handles)
    return UW_ERR_FORMAT;
  std::vector<std::map<int64_t, uw_gemm_config>> parsed(n_handles);
  for (int i = 0; i < n_handles; ++i) {
    if (!hs[i]) return UW_ERR_ARG;
    const JVal& hv = handles->arr[i];
    int64_t N = 0, K = 0;
    if (hv.kind != JVal::Obj || !num_field(hv, "N", &N) || !num_field(hv, "K", &K))
      return UW_ERR_FORMAT;
    if (N != hs[i]->N || K != hs[i]->K) return UW_ERR_FORMAT;
    const JVal* ch = hv.get("choices");
    if (!ch || ch->kind != JVal::Arr) return UW_ERR_FORMAT;
    for (const JVal& c : ch->arr) {
      int64_t M = 0, pl = 0, tn = 0, sg = 0, gc = 0, dc = 0, hv2 = 0, pr = 0, gv = 0;
      if (c.kind != JVal::Obj || !num_field(c, "M", &M) || !num_field(c, "pipeline", &pl))
        return UW_ERR_FORMAT;
      num_field(c, "tile_n", &tn);
      num_field(c, "stages", &sg);
      num_field(c, "gemm_ctas", &gc);
      num_field(c, "decode_ctas", &dc);
      num_field(c, "halves", &hv2);
      num_field(c, "pair", &pr);
      num_field(c, "gemv", &gv);
      uw_gemm_config cfg;
      std::memset(&cfg, 0, sizeof(cfg));
      cfg.pipeline = (int32_t)pl;
      cfg.tile_n = (int32_t)tn;
      cfg.stages = (int32_t)sg;
      cfg.gemm_ctas = (int32_t)gc;
      cfg.decode_ctas = (int32_t)dc;
      cfg.halves = (int32_t)hv2;
      cfg.pair = (int32_t)pr;
      cfg.gemv = (int32_t)gv;
      if (M <= 0 || check_config(hs[i], cfg) != UW_OK) return UW_ERR_FORMAT;
      parsed[i][M] = cfg;
    }
  }
  for (int i = 0; i < n_handles; ++i) hs[i]->profile = parsed[i];
  return UW_OK;
}

uw_status uw_get_choice(uw_handle_t h, int64_t M, uw_gemm_config* cfg) {
  if (!h || !cfg) return UW_ERR_ARG;
  if (M < 0) return UW_ERR_SHAPE;
  *cfg = choose_variant(h, M);
  return UW_OK;
}

}  // extern "C"
