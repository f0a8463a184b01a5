// ITQ3_S-style 3-bit weight GEMV / small-batch matmul with the 256-wide inverse
// Walsh-Hadamard transform.
//
// ITQ3_S article, section "核心技术：FWHT预旋转与TurboQuant的完美融合": weights are
// stored as uniform 3-bit codes of their FWHT-rotated 256-element blocks, and
// the exact inverse transform is applied as the weights are loaded for the
// matmul.  Here one warp owns one output row; lane l holds elements 8*l .. 8*l + 7
// of each 256-block, whose codes are the 24 contiguous bits at bit 24*l of the
// block's packed 96 bytes, so a lane decodes its eight weights with one funnel
// shift and one bit-field extract and one FMA each, and reads its x values with
// 16-byte shared loads.
//
// mode 0 (the article's design): the 256-point inverse FWHT of each weight
//   block runs in registers -- index bits 0..2 inside the lane, bits 3..7 across
//   lanes with xor-shuffles -- and the restored weights meet x.
// mode 1 (algebraically identical, cheaper per weight on B200): H/16 is
//   symmetric and orthogonal, so w_hat . x = ((c - 3.5) s) . (H x / 16).  A
//   first kernel rotates each 256-block of x once into the caller's fp32
//   workspace; the GEMV then uses the levels (c - 3.5) s with no transform.
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace wush {

static __device__ int g_itq3_error = 0;

int read_and_clear_itq3_error(int* word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_itq3_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (*word) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_itq3_error, &zero, sizeof(int));
  }
  return e;
}

namespace {

constexpr int kWarps = 8;

// Levels (c - 3.5) s of the eight elements 8 lane .. 8 lane + 7 of one 256-block,
// from the CTA's shared copy of its 24 code words: 3-bit codes packed
// little-endian, element e at bits 3e .. 3e + 2 of the block.
__device__ __forceinline__ void unpack_levels_smem(const uint32_t* words, int lane, float s, float (&v)[8]) {
  const int bit = 24 * lane;
  const int w0 = bit >> 5;
  const uint32_t lo = words[w0], hi = words[w0 + 1 < 24 ? w0 + 1 : 23];
  const uint32_t bits = __funnelshift_r(lo, hi, bit & 31);
  const float m = -3.5f * s;
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = fmaf(static_cast<float>((bits >> (3 * i)) & 7u), s, m);
}

// In-place unnormalised 256-point FWHT of a warp-distributed vector whose index
// bits are split between the lane (five bits) and the register index (three
// bits); the butterflies run over all eight bits, so either split gives the
// Sylvester-ordered H_256 times the vector.
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

// One CTA owns kWarps consecutive output rows (one per warp).  Thread 0 fetches
// the CTA's packed codes and scales (contiguous, kWarps * nb * 96 and
// kWarps * nb * 2 bytes) with two bulk async copies; meanwhile all threads stage
// the activations of the current 256-block for every token as fp32 in a double
// buffer, so each warp reads its x values and code words from shared memory.
// MODE 0: x is fp16 and the inverse FWHT runs on every weight block (the
// article's fused design).  MODE 1: x is the fp32 rotated activation (H x / 16)
// and the weights are used as their levels (c - 3.5) s.
template <int T, int MODE>
__global__ void __launch_bounds__(kWarps * 32) itq3_gemv_kernel(const uint8_t* __restrict__ codes,
                                                                const __half* __restrict__ scales,
                                                                const void* __restrict__ xin, int tokens,
                                                                int d_out, int d_in, float* __restrict__ y) {
  extern __shared__ __align__(16) uint8_t itq3_smem[];
  const int nb = d_in / 256;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int o0 = blockIdx.x * kWarps;
  const int codes_bytes = kWarps * nb * 96;
  const int scale_bytes = ((kWarps * nb * 2 + 15) / 16) * 16;
  uint8_t* scodes = itq3_smem;
  const __half* sscales = reinterpret_cast<const __half*>(itq3_smem + codes_bytes);
  float* sx = reinterpret_cast<float*>(itq3_smem + codes_bytes + scale_bytes);   // [2][T][256]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sx + 2 * T * 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 1);

  if (threadIdx.x == 0) {
    sm100::mbar_init(bar, 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
    sm100::mbar_arrive_expect_tx(bar, static_cast<uint32_t>(codes_bytes + kWarps * nb * 2));
    sm100::bulk_load(scodes, codes + static_cast<int64_t>(o0) * nb * 96, static_cast<uint32_t>(codes_bytes), bar);
    sm100::bulk_load(itq3_smem + codes_bytes, scales + static_cast<int64_t>(o0) * nb,
                     static_cast<uint32_t>(kWarps * nb * 2), bar);
  }
  auto stage_x = [&](int blk, int buf) {
    float* dst = sx + buf * T * 256;
    for (int i = threadIdx.x; i < tokens * 256; i += kWarps * 32) {
      const int tt = i >> 8, e = i & 255;
      const int64_t src = static_cast<int64_t>(tt) * d_in + blk * 256 + e;
      dst[tt * 256 + e] = MODE == 0 ? __half2float(static_cast<const __half*>(xin)[src])
                                    : static_cast<const float*>(xin)[src];
    }
  };
  stage_x(0, 0);
  __syncthreads();                                   // barrier initialised, block 0 of x staged
  const bool have_codes = sm100::mbar_wait_bounded(bar, 0, int64_t(1) << 40, 4000000000ull, abort_flag);
  if (!have_codes && threadIdx.x == 0) atomicOr(&g_itq3_error, 1 << kErrTimeoutBarrier);

  float acc[T];
#pragma unroll
  for (int t = 0; t < T; ++t) acc[t] = 0.f;
  const int row = warp;
  for (int blk = 0; blk < nb; ++blk) {
    if (blk + 1 < nb) stage_x(blk + 1, (blk + 1) & 1);
    float v[8];
    unpack_levels_smem(reinterpret_cast<const uint32_t*>(scodes + (row * nb + blk) * 96), lane,
                       __half2float(sscales[row * nb + blk]), v);
    if constexpr (MODE == 0) {
      warp_fwht256(v, lane);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] *= 0.0625f;
    }
    const float* xb = sx + (blk & 1) * T * 256 + 8 * lane;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      if (t >= tokens) break;
      const float4 xa = *reinterpret_cast<const float4*>(xb + t * 256);
      const float4 xc = *reinterpret_cast<const float4*>(xb + t * 256 + 4);
      acc[t] = fmaf(v[0], xa.x, acc[t]); acc[t] = fmaf(v[1], xa.y, acc[t]);
      acc[t] = fmaf(v[2], xa.z, acc[t]); acc[t] = fmaf(v[3], xa.w, acc[t]);
      acc[t] = fmaf(v[4], xc.x, acc[t]); acc[t] = fmaf(v[5], xc.y, acc[t]);
      acc[t] = fmaf(v[6], xc.z, acc[t]); acc[t] = fmaf(v[7], xc.w, acc[t]);
    }
    __syncthreads();                                 // x block blk + 1 staged; block blk no longer read
  }
  if (!have_codes) return;
#pragma unroll
  for (int t = 0; t < T; ++t) {
    if (t >= tokens) break;
    float a = acc[t];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane == 0) y[static_cast<int64_t>(t) * d_out + o0 + row] = a;
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

size_t itq3_smem_bytes(int tmax, int64_t d_in) {
  const int64_t nb = d_in / 256;
  return static_cast<size_t>(kWarps * nb * 96 + ((kWarps * nb * 2 + 15) / 16) * 16 + 2 * tmax * 256 * 4 + 16);
}

template <int MODE>
int launch_gemv(const uint32_t* c32, const __half* sc, const void* x, int t, int n, int k, float* y,
                cudaStream_t st) {
  const int tmax = t == 1 ? 1 : (t <= 4 ? 4 : 16);
  const size_t smem = itq3_smem_bytes(tmax, k);
  if (smem > 200 * 1024) return WUSH_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(n / kWarps)), block(kWarps * 32);
  const uint8_t* cb = reinterpret_cast<const uint8_t*>(c32);
#define WUSH_ITQ3(TT)                                                                                          \
  do {                                                                                                         \
    if (smem > 48 * 1024 &&                                                                                    \
        cudaFuncSetAttribute(itq3_gemv_kernel<TT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,          \
                             static_cast<int>(smem)) != cudaSuccess)                                           \
      return WUSH_ERR_CUDA;                                                                                    \
    itq3_gemv_kernel<TT, MODE><<<grid, block, smem, st>>>(cb, sc, x, t, n, k, y);                              \
  } while (0)
  if (tmax == 1) WUSH_ITQ3(1);
  else if (tmax == 4) WUSH_ITQ3(4);
  else WUSH_ITQ3(16);
#undef WUSH_ITQ3
  return launch_status();
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
  if (!codes || !scales_fp16 || !x_fp16 || !y || !aligned16(codes) || !aligned16(scales_fp16))
    return WUSH_ERR_INVALID_ARG;
  if (mode == 1 && (!workspace || !aligned16(workspace))) return WUSH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* c32 = reinterpret_cast<const uint32_t*>(codes);
  const auto* sc = static_cast<const __half*>(scales_fp16);
  const auto* xh = static_cast<const __half*>(x_fp16);
  const int t = static_cast<int>(tokens), n = static_cast<int>(d_out), k = static_cast<int>(d_in);
  if (mode == 0) return launch_gemv<0>(c32, sc, xh, t, n, k, y, st);
  const dim3 block(kWarps * 32);
  const int items = t * (k / 256);
  itq3_rotate_x_kernel<<<(items + kWarps - 1) / kWarps, block, 0, st>>>(xh, t, k, workspace);
  if (launch_status() != WUSH_OK) return WUSH_ERR_CUDA;
  return launch_gemv<1>(c32, sc, workspace, t, n, k, y, st);
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
  if (!codes || !scales_fp16 || !x_fp16 || !y || !aligned16(codes) || !aligned16(scales_fp16))
    return WUSH_ERR_INVALID_ARG;
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
  const dim3 block(kWarps * 32);
  const int items = t * (k / 256);
  itq3_rotate_x_kernel<<<(items + kWarps - 1) / kWarps, block, 0, s>>>(xh, t, k, scratch);
  if (launch_status() != WUSH_OK) return WUSH_ERR_CUDA;
  return launch_gemv<1>(c32, sc, scratch, t, n, k, y, s);
}
