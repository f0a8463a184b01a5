// ITQ3_S-style 3-bit weight GEMV / small-batch matmul with the 256-wide inverse
// Walsh-Hadamard transform.
//
// ITQ3_S article, section "核心技术：FWHT预旋转与TurboQuant的完美融合": weights are
// stored as uniform 3-bit codes of their FWHT-rotated 256-element blocks, and
// the exact inverse transform is applied as the weights are loaded for the
// matmul.  Here one warp owns one output row; lane l holds elements 32*i + l
// (i = 0..7) of each 256-block, which is exactly the bit-plane word layout of
// the packed codes (word p*8 + i, bit l), so every lane unpacks its own eight
// codes from six broadcast 16-byte loads.
//
// mode 0 (the article's design): the 256-point inverse FWHT of each weight
//   block runs in registers -- index bits 5..7 inside the lane, bits 0..4 across
//   lanes with xor-shuffles -- and the restored weights meet x.
// mode 1 (algebraically identical, cheaper per weight on B200): H/16 is
//   symmetric and orthogonal, so w_hat . x = ((c - 3.5) s) . (H x / 16).  A
//   first kernel rotates each 256-block of x once into the caller's fp32
//   workspace; the GEMV then uses the levels (c - 3.5) s with no transform.
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"

namespace wush {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ void unpack_levels(const uint32_t* __restrict__ words, int lane, float s,
                                              float (&v)[8]) {
  const uint4* w4 = reinterpret_cast<const uint4*>(words);
  uint32_t w[24];
#pragma unroll
  for (int q = 0; q < 6; ++q) {
    const uint4 t = __ldg(w4 + q);
    w[4 * q] = t.x; w[4 * q + 1] = t.y; w[4 * q + 2] = t.z; w[4 * q + 3] = t.w;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = ((w[i] >> lane) & 1u) | (((w[8 + i] >> lane) & 1u) << 1) | (((w[16 + i] >> lane) & 1u) << 2);
    v[i] = (static_cast<float>(c) - 3.5f) * s;
  }
}

// In-place unnormalised 256-point FWHT of the warp-distributed vector (element
// 32*i + lane in v[i]).
__device__ __forceinline__ void warp_fwht256(float (&v)[8], int lane) {
#pragma unroll
  for (int b = 0; b < 5; ++b) {
    const bool hi = (lane >> b) & 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, v[i], 1 << b);
      v[i] = hi ? other - v[i] : v[i] + other;
    }
  }
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & h) continue;
      const float a = v[i], c = v[i + h];
      v[i] = a + c;
      v[i + h] = a - c;
    }
  }
}

template <int T>
__global__ void __launch_bounds__(kWarps * 32) itq3_fused_kernel(const uint32_t* __restrict__ codes,
                                                                  const __half* __restrict__ scales,
                                                                  const __half* __restrict__ x, int tokens,
                                                                  int d_out, int d_in, float* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int o = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (o >= d_out) return;
  const int nb = d_in / 256;
  float acc[T];
#pragma unroll
  for (int t = 0; t < T; ++t) acc[t] = 0.f;
  for (int blk = 0; blk < nb; ++blk) {
    float v[8];
    unpack_levels(codes + (static_cast<int64_t>(o) * nb + blk) * 24, lane,
                  __half2float(scales[static_cast<int64_t>(o) * nb + blk]), v);
    warp_fwht256(v, lane);
#pragma unroll
    for (int t = 0; t < T; ++t) {
      if (t >= tokens) break;
      const __half* xr = x + static_cast<int64_t>(t) * d_in + blk * 256 + lane;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[t] = fmaf(v[i] * 0.0625f, __half2float(xr[32 * i]), acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < T; ++t) {
    if (t >= tokens) break;
    float a = acc[t];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane == 0) y[static_cast<int64_t>(t) * d_out + o] = a;
  }
}

// x_rot[t, blk*256 + e] = (H_256 x[t, blk*256 : +256])[e] / 16; one warp per (t, blk).
__global__ void __launch_bounds__(kWarps * 32) itq3_rotate_x_kernel(const __half* __restrict__ x, int tokens,
                                                                     int d_in, float* __restrict__ x_rot) {
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int nb = d_in / 256;
  if (item >= tokens * nb) return;
  const int t = item / nb, blk = item % nb;
  const __half* xr = x + static_cast<int64_t>(t) * d_in + blk * 256 + lane;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __half2float(xr[32 * i]);
  warp_fwht256(v, lane);
  float* out = x_rot + static_cast<int64_t>(t) * d_in + blk * 256 + lane;
#pragma unroll
  for (int i = 0; i < 8; ++i) out[32 * i] = v[i] * 0.0625f;
}

template <int T>
__global__ void __launch_bounds__(kWarps * 32) itq3_rotated_kernel(const uint32_t* __restrict__ codes,
                                                                    const __half* __restrict__ scales,
                                                                    const float* __restrict__ x_rot, int tokens,
                                                                    int d_out, int d_in, float* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int o = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (o >= d_out) return;
  const int nb = d_in / 256;
  float acc[T];
#pragma unroll
  for (int t = 0; t < T; ++t) acc[t] = 0.f;
  for (int blk = 0; blk < nb; ++blk) {
    float v[8];
    unpack_levels(codes + (static_cast<int64_t>(o) * nb + blk) * 24, lane,
                  __half2float(scales[static_cast<int64_t>(o) * nb + blk]), v);
#pragma unroll
    for (int t = 0; t < T; ++t) {
      if (t >= tokens) break;
      const float* xr = x_rot + static_cast<int64_t>(t) * d_in + blk * 256 + lane;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[t] = fmaf(v[i], __ldg(xr + 32 * i), acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < T; ++t) {
    if (t >= tokens) break;
    float a = acc[t];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane == 0) y[static_cast<int64_t>(t) * d_out + o] = a;
  }
}

}  // namespace
}  // namespace wush

using namespace wush;

extern "C" int itq3_dequant_gemv(const uint8_t* codes, const void* scales_fp16, const void* x_fp16,
                                 int64_t tokens, int64_t d_out, int64_t d_in, int mode, float* workspace,
                                 float* y, void* stream) {
  if (tokens < 1 || tokens > 16 || d_out <= 0 || d_in <= 0 || d_in % 256 || d_out % 8) return WUSH_ERR_INVALID_ARG;
  if (d_out > (int64_t(1) << 30) || d_in > (int64_t(1) << 30)) return WUSH_ERR_UNSUPPORTED;
  if (mode != 0 && mode != 1) return WUSH_ERR_UNSUPPORTED;
  if (!codes || !scales_fp16 || !x_fp16 || !y || !aligned16(codes)) return WUSH_ERR_INVALID_ARG;
  if (mode == 1 && (!workspace || !aligned16(workspace))) return WUSH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* c32 = reinterpret_cast<const uint32_t*>(codes);
  const auto* sc = static_cast<const __half*>(scales_fp16);
  const auto* xh = static_cast<const __half*>(x_fp16);
  const int t = static_cast<int>(tokens), n = static_cast<int>(d_out), k = static_cast<int>(d_in);
  const dim3 grid(static_cast<unsigned>((d_out + kWarps - 1) / kWarps)), block(kWarps * 32);
  if (mode == 0) {
    if (t == 1) itq3_fused_kernel<1><<<grid, block, 0, st>>>(c32, sc, xh, t, n, k, y);
    else if (t <= 4) itq3_fused_kernel<4><<<grid, block, 0, st>>>(c32, sc, xh, t, n, k, y);
    else itq3_fused_kernel<16><<<grid, block, 0, st>>>(c32, sc, xh, t, n, k, y);
    return launch_status();
  }
  const int items = t * (k / 256);
  itq3_rotate_x_kernel<<<(items + kWarps - 1) / kWarps, block, 0, st>>>(xh, t, k, workspace);
  if (t == 1) itq3_rotated_kernel<1><<<grid, block, 0, st>>>(c32, sc, workspace, t, n, k, y);
  else if (t <= 4) itq3_rotated_kernel<4><<<grid, block, 0, st>>>(c32, sc, workspace, t, n, k, y);
  else itq3_rotated_kernel<16><<<grid, block, 0, st>>>(c32, sc, workspace, t, n, k, y);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Allocation-free variant of mode 1.
//
// Some callers cannot call cudaMalloc at the point where they run this GEMV: an
// inference engine that carves all device memory out of its own pool at start-up
// and forbids further allocations, a real-time loop that cannot afford the
// latency or the possible failure of an allocation, or a plugin whose host owns
// the device memory.  For them the rotated activations live in one fixed array
// inside this library instead of a caller-provided workspace.
namespace wush {
namespace {

// Capacity of the fixed scratch: tokens * d_in fp32 values (1 MiB).  Every device
// that loads the library holds this array until the process exits.
constexpr int64_t kNoAllocScratchFloats = int64_t(1) << 18;

}  // namespace

static __device__ __align__(256) float g_itq3_noalloc_scratch[kNoAllocScratchFloats];

namespace {

constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device, looked up once per
// device.  (In host code the array's name is only a host-side stand-in, so the
// kernels must be handed this address, never the name.)
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WUSH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_itq3_noalloc_scratch) != cudaSuccess || !p) return WUSH_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return WUSH_OK;
}

}  // namespace
}  // namespace wush

extern "C" int itq3_dequant_gemv_noalloc(const uint8_t* codes, const void* scales_fp16, const void* x_fp16,
                                         int64_t tokens, int64_t d_out, int64_t d_in, float* y, void* stream) {
  if (tokens < 1 || tokens > 16 || d_out <= 0 || d_in <= 0 || d_in % 256 || d_out % 8) return WUSH_ERR_INVALID_ARG;
  if (tokens * d_in > kNoAllocScratchFloats) return WUSH_ERR_BUFFER_TOO_SMALL;
  if (d_out > (int64_t(1) << 30)) return WUSH_ERR_UNSUPPORTED;
  if (!codes || !scales_fp16 || !x_fp16 || !y || !aligned16(codes)) return WUSH_ERR_INVALID_ARG;
  float* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != WUSH_OK) return st;
  // The rotation kernel writes every scratch element the GEMV then reads, so
  // nothing left there by an earlier call needs clearing.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const auto* c32 = reinterpret_cast<const uint32_t*>(codes);
  const auto* sc = static_cast<const __half*>(scales_fp16);
  const auto* xh = static_cast<const __half*>(x_fp16);
  const int t = static_cast<int>(tokens), n = static_cast<int>(d_out), k = static_cast<int>(d_in);
  const dim3 grid(static_cast<unsigned>((d_out + kWarps - 1) / kWarps)), block(kWarps * 32);
  const int items = t * (k / 256);
  itq3_rotate_x_kernel<<<(items + kWarps - 1) / kWarps, block, 0, s>>>(xh, t, k, scratch);
  if (t == 1) itq3_rotated_kernel<1><<<grid, block, 0, s>>>(c32, sc, scratch, t, n, k, y);
  else if (t <= 4) itq3_rotated_kernel<4><<<grid, block, 0, s>>>(c32, sc, scratch, t, n, k, y);
  else itq3_rotated_kernel<16><<<grid, block, 0, s>>>(c32, sc, scratch, t, n, k, y);
  return launch_status();
}
