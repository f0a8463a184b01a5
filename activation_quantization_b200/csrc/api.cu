// Status strings, the device error word and the diagnostics entry points.
#include "common.cuh"

namespace wush {
// Poll limit for bounded mbarrier waits in the GEMM (0 = default); see wush.h.
int64_t g_wait_limit_override = 0;
// ITQ3 mode-1 kernel: 0 tensor cores where the shape allows, 1 CUDA cores; see wush.h.
int g_itq3_variant = 0;
}  // namespace wush

extern "C" const char* wush_status_string(int status) {
  switch (status) {
    case WUSH_OK: return "ok";
    case WUSH_ERR_INVALID_ARG: return "invalid argument";
    case WUSH_ERR_UNSUPPORTED: return "unsupported format, transform or size";
    case WUSH_ERR_NOT_SPD: return "weight second moment is not positive definite";
    case WUSH_ERR_CUDA: return "CUDA error";
    case WUSH_ERR_TIMEOUT: return "a bounded device wait gave up";
    case WUSH_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    case WUSH_ERR_IO: return "file could not be opened, read or written";
    default: return "unknown status";
  }
}

extern "C" int wush_check_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WUSH_ERR_CUDA;
  int word = 0, word_tq = 0, word_i4 = 0, word_it = 0, word_itc = 0;
  if (wush::read_and_clear_error_word(&word) != cudaSuccess) return WUSH_ERR_CUDA;
  if (wush::read_and_clear_tq_error(&word_tq) != cudaSuccess) return WUSH_ERR_CUDA;
  if (wush::read_and_clear_int4_error(&word_i4) != cudaSuccess) return WUSH_ERR_CUDA;
  if (wush::read_and_clear_itq3_error(&word_it) != cudaSuccess) return WUSH_ERR_CUDA;
  if (wush::read_and_clear_itq3_tc_error(&word_itc) != cudaSuccess) return WUSH_ERR_CUDA;
  return (word | word_tq | word_i4 | word_it | word_itc) == 0 ? WUSH_OK : WUSH_ERR_TIMEOUT;
}

extern "C" int wush_debug_set_gemm_variant(int variant) {
  if (variant < 0 || variant > 2) return WUSH_ERR_INVALID_ARG;
  wush::g_gemm_variant = variant;
  return WUSH_OK;
}

extern "C" int wush_debug_set_wait_limit(int64_t max_polls) {
  if (max_polls < 0) return WUSH_ERR_INVALID_ARG;
  wush::g_wait_limit_override = max_polls;
  return WUSH_OK;
}

extern "C" int wush_debug_set_itq3_variant(int variant) {
  if (variant < 0 || variant > 3) return WUSH_ERR_INVALID_ARG;
  wush::g_itq3_variant = variant;
  return WUSH_OK;
}
