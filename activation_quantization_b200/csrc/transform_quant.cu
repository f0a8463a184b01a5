// Fused per-block transform + microscaled quantisation (MXFP4 / NVFP4 / INT4).
//
// WUSH news article, paragraph 6 (at inference only the input activations are
// transformed; the transform is block-diagonal so blocks are independent) and
// AI Radio episode, "The gist" (a fused GPU implementation of transform and
// quantisation).  The format rules are stated in wush.h.
//
// Work split: one thread owns one row (token) and walks kBlocksPerCta
// consecutive b-blocks of it, so the b transformed values of a block, its
// absmax, its scale and its packed codes never leave the thread's registers (no
// shuffles, no shared-memory reductions).  A CTA covers 128 rows x 4 blocks:
// exactly one 512-byte atom of the MMA scale-factor layout, which it stages in
// shared memory and stores with 16-byte writes.  For the dense (WUS/WUSH)
// transform the CTA's four b x b matrices sit in shared memory and every lane
// reads the same word at the same time (broadcast).
#include <cuda_fp16.h>

#include "common.cuh"
#include "quant_decide.cuh"

namespace wush {
namespace {

constexpr int kRowsPerCta = 128;
constexpr int kBlocksPerCta = 4;

enum Kind : int { kIdentity = 0, kHadamard = 1, kDense = 2 };
enum Fmt : int { kMx = 0, kNv = 1, kI4 = 2, kAmax = 3 };

template <int B, bool XF32>
__device__ __forceinline__ void load_block(const void* x, int64_t off, float (&v)[B]) {
  if constexpr (XF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + off);
#pragma unroll
    for (int w = 0; w < B / 4; ++w) {
      const float4 q = __ldg(p + w);
      v[4 * w] = q.x; v[4 * w + 1] = q.y; v[4 * w + 2] = q.z; v[4 * w + 3] = q.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + off);
#pragma unroll
    for (int w = 0; w < B / 8; ++w) {
      const uint4 q = __ldg(p + w);
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[8 * w + 2 * h] = bf16_lo(u[h]);
        v[8 * w + 2 * h + 1] = bf16_hi(u[h]);
      }
    }
  }
}

template <int B>
__device__ __forceinline__ void fwht_normalized(float (&y)[B]) {
#pragma unroll
  for (int h = 1; h < B; h <<= 1) {
#pragma unroll
    for (int i = 0; i < B; i += 2 * h) {
#pragma unroll
      for (int k = i; k < i + h; ++k) {
        const float a = y[k], b = y[k + h];
        y[k] = a + b;
        y[k + h] = a - b;
      }
    }
  }
  const float s = B == 32 ? 0.17677669529663688f : (B == 16 ? 0.25f : rsqrtf(static_cast<float>(B)));
#pragma unroll
  for (int i = 0; i < B; ++i) y[i] *= s;
}

// y = T x with T [B][B] in shared memory; four interleaved FMA chains of B/4 terms,
// combined pairwise, keep the fp32 error near (B/4 + 2) ulp of sum |T x|.
template <int B>
__device__ __forceinline__ void dense_apply(const float* __restrict__ tj, const float (&x)[B], float (&y)[B]) {
#pragma unroll
  for (int i = 0; i < B; ++i) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int k = 0; k < B; k += 4) {
      const float4 t4 = *reinterpret_cast<const float4*>(tj + i * B + k);
      a0 = fmaf(t4.x, x[k], a0);
      a1 = fmaf(t4.y, x[k + 1], a1);
      a2 = fmaf(t4.z, x[k + 2], a2);
      a3 = fmaf(t4.w, x[k + 3], a3);
    }
    y[i] = (a0 + a1) + (a2 + a3);
  }
}

template <int B, int KIND, int FMT, bool XF32, bool DBG>
__global__ void __launch_bounds__(kRowsPerCta) transform_quant_kernel(
    const void* __restrict__ x, int64_t rows, int64_t d_in, const float* __restrict__ t,
    const int* __restrict__ t_index, int n_t, float gscale_arg,
    const float* __restrict__ gs_amax, float* __restrict__ gs_out, uint8_t* __restrict__ codes,
    void* __restrict__ scales, float* __restrict__ ydbg, float* __restrict__ amax_out) {
  // NVFP4 per-tensor scale: the caller's, or derived from a device amax
  float gscale = gscale_arg;
  if (FMT == kNv && gs_amax) {
    gscale = nvfp4_dynamic_scale(__ldg(gs_amax));
    if (gs_out && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *gs_out = gscale;
  }
  constexpr int CH = kBlocksPerCta;
  __shared__ __align__(16) float s_t[KIND == kDense ? CH * B * B : 4];
  __shared__ __align__(16) uint8_t s_sf[512];
  __shared__ float s_red[kRowsPerCta / 32];

  const int64_t nb = d_in / B;
  const int64_t j0 = static_cast<int64_t>(blockIdx.y) * CH;
  const int nblk = static_cast<int>(nb - j0 < CH ? nb - j0 : CH);
  const int tid = threadIdx.x;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + tid;

  if constexpr (KIND == kDense) {
    // block j's T is t[j], or t[t_index[j]] (clamped to the n_t transforms)
    constexpr int kQuads = B * B / 4;
    float4* dst = reinterpret_cast<float4*>(s_t);
    for (int i = tid; i < nblk * kQuads; i += kRowsPerCta) {
      const int k = i / kQuads;
      int64_t jt = j0 + k;
      if (t_index) {
        const int v = __ldg(t_index + j0 + k);
        jt = v < 0 ? 0 : (v >= n_t ? n_t - 1 : v);
      }
      dst[i] = __ldg(reinterpret_cast<const float4*>(t + jt * B * B) + (i - k * kQuads));
    }
  }
  if constexpr (FMT == kMx || FMT == kNv) reinterpret_cast<uint32_t*>(s_sf)[tid] = 0u;
  __syncthreads();

  float amax_all = 0.f;
  if (r < rows) {
    for (int jj = 0; jj < nblk; ++jj) {
      const int64_t j = j0 + jj;
      float xv[B], y[B];
      load_block<B, XF32>(x, r * d_in + j * B, xv);
      if constexpr (KIND == kDense) {
        dense_apply<B>(s_t + jj * B * B, xv, y);
      } else {
#pragma unroll
        for (int i = 0; i < B; ++i) y[i] = xv[i];
        if constexpr (KIND == kHadamard) fwht_normalized<B>(y);
      }
      if constexpr (DBG) {
        float4* dp = reinterpret_cast<float4*>(ydbg + r * d_in + j * B);
#pragma unroll
        for (int w = 0; w < B / 4; ++w) dp[w] = make_float4(y[4 * w], y[4 * w + 1], y[4 * w + 2], y[4 * w + 3]);
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < B; ++i) amax = fmaxf(amax, fabsf(y[i]));
      if constexpr (FMT == kAmax) {
        amax_all = fmaxf(amax_all, amax);
        continue;
      }

      // every decision is the round-to-nearest-even of the exact quotient (quant_decide.cuh)
      uint32_t wv[B / 8];
      if constexpr (FMT == kMx) {
        int e = amax > 0.f ? floor_log2(amax) - 2 : -127;
        e = e < -127 ? -127 : (e > 127 ? 127 : e);
        const float inv = exp2i(-e);  // y * 2^-e is exact
#pragma unroll
        for (int w = 0; w < B / 8; ++w) wv[w] = amax > 0.f ? e2m1x8_times(y + 8 * w, inv) : 0u;
        s_sf[(tid & 31) * 16 + (tid >> 5) * 4 + jj] = static_cast<uint8_t>(e + 127);
      } else if constexpr (FMT == kNv) {
        const uint32_t sb = nvfp4_scale_byte(amax, gscale, __frcp_rn(__fmul_rn(6.0f, gscale)));
        const float sbv = ue4m3_val(sb);
        const bool live = sb != 0u && amax > 0.f;
        const float rd = live ? __frcp_rn(__fmul_rn(sbv, gscale)) : 0.f;
#pragma unroll
        for (int w = 0; w < B / 8; ++w) wv[w] = live ? nvfp4_codes8(y + 8 * w, rd, sbv, gscale) : 0u;
        s_sf[(tid & 31) * 16 + (tid >> 5) * 4 + jj] = static_cast<uint8_t>(sb);
      } else {  // INT4
        const __half s16 = int4_scale(amax);
        const float s = __half2float(s16);
        const float rs = s > 0.f ? __frcp_rn(s) : 0.f;
#pragma unroll
        for (int w = 0; w < B / 8; ++w) wv[w] = s > 0.f ? int4_codes8(y + 8 * w, rs, s) : 0u;
        reinterpret_cast<__half*>(scales)[r * nb + j] = s16;
      }
      uint8_t* cp = codes + r * (d_in / 2) + j * (B / 2);
      if constexpr (B == 32) {
        *reinterpret_cast<uint4*>(cp) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      } else {
        *reinterpret_cast<uint2*>(cp) = make_uint2(wv[0], wv[1]);
      }
    }
  }

  if constexpr (FMT == kMx || FMT == kNv) {
    __syncthreads();
    if (tid < 32) {
      const int64_t atom = static_cast<int64_t>(blockIdx.x) * gridDim.y + blockIdx.y;
      reinterpret_cast<uint4*>(static_cast<uint8_t*>(scales) + atom * 512)[tid] =
          reinterpret_cast<const uint4*>(s_sf)[tid];
    }
  }
  if constexpr (FMT == kAmax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax_all = fmaxf(amax_all, __shfl_xor_sync(0xffffffffu, amax_all, o));
    if ((tid & 31) == 0) s_red[tid >> 5] = amax_all;
    __syncthreads();
    if (tid == 0) {
      float m = s_red[0];
      for (int w = 1; w < kRowsPerCta / 32; ++w) m = fmaxf(m, s_red[w]);
      atomicMax(reinterpret_cast<unsigned int*>(amax_out), __float_as_uint(m));
    }
  }
}

template <int B, int FMT>
int launch_fmt(const void* x, bool xf32, int64_t rows, int64_t d_in, const float* t, int kind, float gscale,
               uint8_t* codes, void* scales, float* ydbg, float* amax_out, cudaStream_t st,
               const float* gs_amax = nullptr, float* gs_out = nullptr, const int* t_index = nullptr, int n_t = 0) {
  const dim3 grid(static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta),
                  static_cast<unsigned>((d_in / B + kBlocksPerCta - 1) / kBlocksPerCta));
  const dim3 block(kRowsPerCta);
  const int k = kind == WUSH_T_IDENTITY ? kIdentity : (kind == WUSH_T_HADAMARD ? kHadamard : kDense);
#define WUSH_TQ_LAUNCH(KK, XF, DB)                                                                \
  transform_quant_kernel<B, KK, FMT, XF, DB><<<grid, block, 0, st>>>(x, rows, d_in, t, t_index, n_t, gscale, \
                                                                     gs_amax, gs_out, codes, scales, ydbg, amax_out)
#define WUSH_TQ_KIND(XF, DB)                       \
  do {                                             \
    if (k == kIdentity) WUSH_TQ_LAUNCH(kIdentity, XF, DB); \
    else if (k == kHadamard) WUSH_TQ_LAUNCH(kHadamard, XF, DB); \
    else WUSH_TQ_LAUNCH(kDense, XF, DB);            \
  } while (0)
  if constexpr (FMT == kAmax) {
    if (xf32) WUSH_TQ_KIND(true, false); else WUSH_TQ_KIND(false, false);
  } else {
    if (xf32) {
      if (ydbg) WUSH_TQ_KIND(true, true); else WUSH_TQ_KIND(true, false);
    } else {
      if (ydbg) WUSH_TQ_KIND(false, true); else WUSH_TQ_KIND(false, false);
    }
  }
#undef WUSH_TQ_KIND
#undef WUSH_TQ_LAUNCH
  return launch_status();
}

int check_common(const void* x, int x_dtype, int64_t rows, int64_t d_in, const float* t, int kind, int b) {
  if (rows < 0 || d_in <= 0 || d_in % b) return WUSH_ERR_INVALID_ARG;
  if (x_dtype != WUSH_IN_BF16 && x_dtype != WUSH_IN_FP32) return WUSH_ERR_UNSUPPORTED;
  if (kind < WUSH_T_IDENTITY || kind > WUSH_T_WUSH_DIAG) return WUSH_ERR_UNSUPPORTED;
  if (rows > 0 && (!x || !aligned16(x))) return WUSH_ERR_INVALID_ARG;
  // WUS, WUSH and WUSH-diag are applied as dense per-block matrices
  if (kind >= WUSH_T_WUS && (!t || !aligned16(t))) return WUSH_ERR_INVALID_ARG;
  if ((d_in / b + kBlocksPerCta - 1) / kBlocksPerCta > 65535) return WUSH_ERR_UNSUPPORTED;
  if ((rows + kRowsPerCta - 1) / kRowsPerCta > 0x7FFFFFFF) return WUSH_ERR_UNSUPPORTED;
  return WUSH_OK;
}

}  // namespace
}  // namespace wush

using namespace wush;

extern "C" int wush_block_size(int fmt) {
  return fmt == WUSH_FMT_MXFP4 ? 32 : fmt == WUSH_FMT_NVFP4 ? 16 : fmt == WUSH_FMT_INT4 ? 32 : 0;
}

extern "C" size_t wush_codes_bytes(int64_t rows, int64_t d_in, int fmt) {
  if (rows < 0 || d_in <= 0 || wush_block_size(fmt) == 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(d_in) / 2;
}

extern "C" size_t wush_scales_bytes(int64_t rows, int64_t d_in, int fmt) {
  const int b = wush_block_size(fmt);
  if (rows < 0 || d_in <= 0 || b == 0) return 0;
  const int64_t nb = (d_in + b - 1) / b;
  if (fmt == WUSH_FMT_INT4) return static_cast<size_t>(rows * nb) * 2;
  return static_cast<size_t>(((rows + 127) / 128) * ((nb + 3) / 4)) * 512;
}

extern "C" int wush_transform_quant(const void* x, int x_dtype, int64_t rows, int64_t d_in, const float* t,
                                    int kind, int fmt, float global_scale, uint8_t* codes, void* scales,
                                    float* y_debug, void* stream) {
  const int b = wush_block_size(fmt);
  if (b == 0) return WUSH_ERR_UNSUPPORTED;
  int st = check_common(x, x_dtype, rows, d_in, t, kind, b);
  if (st != WUSH_OK) return st;
  if (rows == 0) return WUSH_OK;
  if (!codes || !scales || !aligned16(codes) || !aligned16(scales)) return WUSH_ERR_INVALID_ARG;
  if (y_debug && !aligned16(y_debug)) return WUSH_ERR_INVALID_ARG;
  if (fmt == WUSH_FMT_NVFP4 && !(global_scale >= 1e-30f && global_scale < 1e30f)) return WUSH_ERR_INVALID_ARG;
  const bool xf32 = x_dtype == WUSH_IN_FP32;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!xf32) {
    const int tc = transform_quant_tc(x, rows, d_in, t, nullptr, 0, kind, fmt, global_scale, nullptr, nullptr, codes,
                                      scales, y_debug, s);
    if (tc != WUSH_ERR_UNSUPPORTED) return tc;
  }
  if (fmt == WUSH_FMT_MXFP4)
    return launch_fmt<32, kMx>(x, xf32, rows, d_in, t, kind, 0.f, codes, scales, y_debug, nullptr, s);
  if (fmt == WUSH_FMT_NVFP4)
    return launch_fmt<16, kNv>(x, xf32, rows, d_in, t, kind, global_scale, codes, scales, y_debug, nullptr, s);
  return launch_fmt<32, kI4>(x, xf32, rows, d_in, t, kind, 0.f, codes, scales, y_debug, nullptr, s);
}

extern "C" int wush_transform_quant_indexed(const void* x, int x_dtype, int64_t rows, int64_t d_in, const float* t,
                                            const int32_t* t_index, int n_t, int kind, int fmt, float global_scale,
                                            uint8_t* codes, void* scales, float* y_debug, void* stream) {
  const int b = wush_block_size(fmt);
  if (b == 0) return WUSH_ERR_UNSUPPORTED;
  if (kind < WUSH_T_WUS) return WUSH_ERR_INVALID_ARG;   // only dense transforms are shared
  int st = check_common(x, x_dtype, rows, d_in, t, kind, b);
  if (st != WUSH_OK) return st;
  if (!t_index || (reinterpret_cast<uintptr_t>(t_index) & 3u) || n_t < 1) return WUSH_ERR_INVALID_ARG;
  if (rows == 0) return WUSH_OK;
  if (!codes || !scales || !aligned16(codes) || !aligned16(scales)) return WUSH_ERR_INVALID_ARG;
  if (y_debug && !aligned16(y_debug)) return WUSH_ERR_INVALID_ARG;
  if (fmt == WUSH_FMT_NVFP4 && !(global_scale >= 1e-30f && global_scale < 1e30f)) return WUSH_ERR_INVALID_ARG;
  const bool xf32 = x_dtype == WUSH_IN_FP32;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!xf32) {
    const int tc = transform_quant_tc(x, rows, d_in, t, t_index, n_t, kind, fmt, global_scale, nullptr, nullptr,
                                      codes, scales, y_debug, s);
    if (tc != WUSH_ERR_UNSUPPORTED) return tc;
  }
  if (fmt == WUSH_FMT_MXFP4)
    return launch_fmt<32, kMx>(x, xf32, rows, d_in, t, kind, 0.f, codes, scales, y_debug, nullptr, s, nullptr,
                               nullptr, t_index, n_t);
  if (fmt == WUSH_FMT_NVFP4)
    return launch_fmt<16, kNv>(x, xf32, rows, d_in, t, kind, global_scale, codes, scales, y_debug, nullptr, s,
                               nullptr, nullptr, t_index, n_t);
  return launch_fmt<32, kI4>(x, xf32, rows, d_in, t, kind, 0.f, codes, scales, y_debug, nullptr, s, nullptr, nullptr,
                             t_index, n_t);
}

extern "C" int wush_transform_quant_nvfp4_dynamic(const void* x, int x_dtype, int64_t rows, int64_t d_in,
                                                  const float* t, int kind, const float* amax,
                                                  float* global_scale_out, uint8_t* codes, void* scales,
                                                  float* y_debug, void* stream) {
  int st = check_common(x, x_dtype, rows, d_in, t, kind, 16);
  if (st != WUSH_OK) return st;
  if (!amax || (reinterpret_cast<uintptr_t>(amax) & 3u)) return WUSH_ERR_INVALID_ARG;
  if (global_scale_out && (reinterpret_cast<uintptr_t>(global_scale_out) & 3u)) return WUSH_ERR_INVALID_ARG;
  if (rows == 0) return WUSH_OK;
  if (!codes || !scales || !aligned16(codes) || !aligned16(scales)) return WUSH_ERR_INVALID_ARG;
  if (y_debug && !aligned16(y_debug)) return WUSH_ERR_INVALID_ARG;
  const bool xf32 = x_dtype == WUSH_IN_FP32;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!xf32) {
    // the placeholder scale 1 is never used: the kernel reads the amax
    const int tc = transform_quant_tc(x, rows, d_in, t, nullptr, 0, kind, WUSH_FMT_NVFP4, 1.0f, amax,
                                      global_scale_out, codes, scales, y_debug, s);
    if (tc != WUSH_ERR_UNSUPPORTED) return tc;
  }
  return launch_fmt<16, kNv>(x, xf32, rows, d_in, t, kind, 1.0f, codes, scales, y_debug, nullptr, s, amax,
                             global_scale_out);
}

extern "C" int wush_transform_amax(const void* x, int x_dtype, int64_t rows, int64_t d_in, const float* t,
                                   int kind, int block, float* amax_out, void* stream) {
  if (block != 16 && block != 32) return WUSH_ERR_UNSUPPORTED;
  int st = check_common(x, x_dtype, rows, d_in, t, kind, block);
  if (st != WUSH_OK) return st;
  if (!amax_out || (reinterpret_cast<uintptr_t>(amax_out) & 3u)) return WUSH_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess) return WUSH_ERR_CUDA;
  if (rows == 0) return WUSH_OK;
  const bool xf32 = x_dtype == WUSH_IN_FP32;
  if (!xf32) {
    const int tc = transform_amax_tc(x, rows, d_in, t, kind, block, amax_out, s);
    if (tc != WUSH_ERR_UNSUPPORTED) return tc;
  }
  if (block == 32)
    return launch_fmt<32, kAmax>(x, xf32, rows, d_in, t, kind, 0.f, nullptr, nullptr, nullptr, amax_out, s);
  return launch_fmt<16, kAmax>(x, xf32, rows, d_in, t, kind, 0.f, nullptr, nullptr, nullptr, amax_out, s);
}
