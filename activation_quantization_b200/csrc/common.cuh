// Shared device helpers of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "wush.h"

namespace wush {

// Bits of the device error word that kernels with bounded waits set when a wait
// gives up (see wush_check_device_status).  The word lives in qgemm.cu.
enum : int { kErrTimeoutBarrier = 1, kErrTimeoutTmem = 2 };

// Reads the device error word of the GEMM translation unit into *word and clears
// it; returns a cudaError_t as int.
int read_and_clear_error_word(int* word);

// The same for the tensor-core transform+quant kernel's and the INT4 GEMM's words.
int read_and_clear_tq_error(int* word);
int read_and_clear_int4_error(int* word);
int read_and_clear_itq3_error(int* word);
int read_and_clear_itq3_tc_error(int* word);

// Tensor-core form of wush_transform_quant (bf16 inputs); WUSH_ERR_UNSUPPORTED
// for shapes it does not take.
// gs_amax (device, optional): NVFP4 takes its per-tensor scale from this amax
// (nvfp4_dynamic_scale) instead of gscale, and CTA 0 writes it to gs_out if given.
int transform_amax_tc(const void* x, int64_t rows, int64_t d_in, const float* t, int kind, int block,
                      float* amax_out, cudaStream_t st);
// t_index (device int32 [d_in/b], optional): block j uses transform t[t_index[j]],
// clamped to [0, n_t), instead of t[j].
int transform_quant_tc(const void* x, int64_t rows, int64_t d_in, const float* t, const int* t_index, int n_t,
                       int kind, int fmt, float gscale, const float* gs_amax, float* gs_out, uint8_t* codes,
                       void* scales, float* ydbg, cudaStream_t st);

// GEMM kernel choice (see wush_debug_set_gemm_variant).
extern int g_gemm_variant;

// Tensor-core form of the ITQ3 activation-side GEMV on rotated fp32 x (device
// [tokens, d_in]); WUSH_ERR_UNSUPPORTED, before any launch, for shapes it does not take.
int itq3_gemv_tc(const uint8_t* codes, const void* scales_fp16, const float* x_rot, int tokens, int d_out, int d_in,
                 float* y, cudaStream_t st);

// ITQ3 mode-1 kernel choice (see wush_debug_set_itq3_variant).
extern int g_itq3_variant;

// Poll limit for bounded mbarrier waits (0 = the built-in default).
extern int64_t g_wait_limit_override;

inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? WUSH_OK : WUSH_ERR_CUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raises a kernel's dynamic shared-memory limit to ``bytes`` once per device;
// ``done`` holds one bit per device (devices 64 and up are set on every call).
// Safe to call from several host threads: setting the attribute twice is harmless.
template <typename Kernel>
inline int set_smem_once(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WUSH_ERR_CUDA;
  const uint64_t bit = dev >= 0 && dev < 64 ? uint64_t(1) << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return WUSH_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return WUSH_ERR_CUDA;
  if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return WUSH_OK;
}

// Dynamic NVFP4 per-tensor scale from the device amax of the transformed tensor:
// s_g = fp32(amax / 2688), 2688 = 6 * 448 (largest E2M1 magnitude times largest
// UE4M3 block scale); 1 when that is below 1e-30 (an all-zero or denormal tensor,
// whose codes are zero whatever the scale).
__device__ __forceinline__ float nvfp4_dynamic_scale(float amax) {
  const float g = __fdiv_rn(amax, 2688.0f);
  return g >= 1e-30f ? g : 1.0f;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of scale (r, c) in the block-scaled MMA scale-factor tile layout:
// 128-row x 4-column atoms of 512 bytes, (r, c) at (r%32)*16 + (r/32)*4 + c inside
// an atom, atoms ordered row-block-major.
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t n_atom_cols) {
  return ((r >> 7) * n_atom_cols + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

}  // namespace wush
