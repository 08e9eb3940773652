// Autotuner and profile I/O (placeholder).
#include <cstring>

#include "handle.h"

extern "C" {
uw_status uw_autotune(uw_handle_t*, int32_t, const int64_t*, int32_t, const char*) {
  return UW_ERR_UNSUPPORTED;
}
uw_status uw_load_profile(uw_handle_t*, int32_t, const char*) { return UW_ERR_UNSUPPORTED; }
uw_status uw_get_choice(uw_handle_t, int64_t, uw_gemm_config*) { return UW_ERR_UNSUPPORTED; }
}
