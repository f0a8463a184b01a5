// ITQ3_S-style 3-bit weight GEMV / small-batch matmul with the 256-wide inverse
// Walsh-Hadamard transform.
//
// ITQ3_S article, section "核心技术：FWHT预旋转与TurboQuant的完美融合": weights are
// stored as uniform 3-bit codes of their FWHT-rotated 256-element blocks, and
// the exact inverse transform is applied as the weights are loaded for the
// matmul.  Here one warp owns one to four output rows; lane l holds elements
// 8*l .. 8*l + 7 of each 256-block, whose codes are the 24 contiguous bits at bit
// 24*l of the block's packed 96 bytes, so a lane gathers its bits with one funnel
// shift, decodes each weight with an integer multiply, a mask and one FMA, and
// reads its x values with 16-byte loads.
//
// mode 0 (the article's design): the 256-point inverse FWHT of each weight
//   block runs in registers -- index bits 0..2 inside the lane, bits 3..7 across
//   lanes with xor-shuffles -- and the restored weights meet x.
// mode 1 (algebraically identical, cheaper per weight on B200): H/16 is
//   symmetric and orthogonal, so w_hat . x = ((c - 3.5) s) . (H x / 16).  A
//   first kernel rotates each 256-block of x once into the caller's fp32
//   workspace; the GEMV then uses the levels (c - 3.5) s with no transform.  For
//   one or two tokens the call is a single kernel instead (itq3_gemv_rot_kernel):
//   every CTA rotates the tokens of x into its shared memory.
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

// Programmatic dependent launch, so that the launch latency of each kernel hides
// under the previous one:
//  * the rotation kernel waits for the kernel before it before it reads x, and only
//    then lets the GEMV that follows it start;
//  * the GEMV issues its code-word loads at once (no kernel still running can be
//    writing them: the rotation has passed its wait), and waits for the rotation's
//    results only where it first reads them;
//  * every GEMV lets the next call's first kernel start early (mode 1 at entry,
//    mode 0 once its work is done); that kernel waits for the GEMV to finish
//    before it touches memory.
// Both instructions are no-ops in a kernel launched without the attribute.
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_for_prerequisite_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Levels (c - 3.5) s of the eight elements 8 lane .. 8 lane + 7 of one 256-block.
// Lane j < 24 holds word j of the block's 96 packed bytes (3-bit codes,
// little-endian, element e at bits 3e .. 3e + 2); this lane's 24 bits start at bit
// 24 lane, inside words (24 lane) / 32 and the one after it.  Code i goes into
// mantissa bits 20 .. 22 of 1.0f (see levels8 below), giving f = 1 + c / 8 exactly,
// and (c - 3.5) s = f (8 s) - 11.5 s: 8 s and 11.5 s are exact, and so is the FMA,
// since (c - 3.5) s needs at most 15 significant bits.
__device__ __forceinline__ void decode_levels(uint32_t word, int lane, float s, float (&v)[8]) {
  const int bit = 24 * lane;
  const int w0 = bit >> 5;
  const uint32_t lo = __shfl_sync(0xffffffffu, word, w0);
  const uint32_t hi = __shfl_sync(0xffffffffu, word, w0 + 1 < 24 ? w0 + 1 : 23);
  const uint32_t bits = __funnelshift_r(lo, hi, bit & 31);
  const float s8 = 8.0f * s, m = -11.5f * s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t t;
    if (i < 7)
      asm("mul.lo.u32 %0, %1, %2;" : "=r"(t) : "r"(bits), "r"((1u << (20 - 3 * (i < 7 ? i : 0))) | 0x80000000u));
    else
      t = bits >> 1;
    v[i] = fmaf(__uint_as_float((t & 0x00700000u) | 0x3F800000u), s8, m);
  }
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

// One warp owns R consecutive output rows and walks the 256-blocks of d_in in
// windows of W blocks: it first issues every code-word and scale load of the
// window (lanes 0..23 take the 24 words of a block, one each), then decodes each
// block (two shuffles and a funnel shift per lane) and multiplies it into the
// accumulators of TC tokens at a time; each x load is shared by the R rows.  With
// STAGE the CTA first copies the chunk's TC tokens of x into shared memory as fp32,
// so the block loop waits on shared-memory latency rather than L2.
// MODE 0: x is fp16 and the inverse FWHT runs on every weight block (the
// article's fused design).  MODE 1: x is the fp32 rotated activation (H x / 16)
// and the weights are used as their levels (c - 3.5) s.
template <int R, int W, int TC, int MODE, bool STAGE>
__global__ void __launch_bounds__(kWarps * 32) itq3_gemv_kernel(const uint32_t* __restrict__ codes,
                                                                const __half* __restrict__ scales,
                                                                const void* __restrict__ xin, int tokens,
                                                                int d_out, int d_in, float* __restrict__ y) {
  extern __shared__ __align__(16) float sx[];      // STAGE: [TC][d_in] fp32
  // Mode 1 (memory-bound) lets the next kernel launch at once.  Mode 0 is bound by
  // its arithmetic, and a next kernel whose CTAs wait beside it on the same SMs
  // measured up to 1.6x slower, so it lets the next kernel launch only once its
  // own work is done; as the call's only kernel it reads nothing global before the
  // kernel launched before it has finished.
  if constexpr (MODE == 1) allow_dependent_launch();
  if constexpr (MODE == 0) wait_for_prerequisite_grid();
  const int lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kWarps + (threadIdx.x >> 5)) * R;
  if (!STAGE && row0 >= d_out) return;             // with STAGE every warp joins the barriers
  const int nb = d_in / 256;
  // Copies tokens tc0 .. tc0 + TC - 1 of x into shared memory as fp32 (zeros past
  // the last token); every warp of the CTA takes part.
  auto stage_x = [&](int tc0) {
    __syncthreads();                               // the previous chunk is no longer read
    for (int i = threadIdx.x * 4; i < TC * d_in; i += kWarps * 32 * 4) {
      const int tt = i / d_in, e = i - tt * d_in, t = tc0 + tt;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < tokens) {
        const int64_t xo = static_cast<int64_t>(t) * d_in + e;
        if constexpr (MODE == 0) {
          const uint2 h = __ldg(reinterpret_cast<const uint2*>(static_cast<const __half*>(xin) + xo));
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
          v = make_float4(a.x, a.y, b.x, b.y);
        } else {
          v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(xin) + xo));
        }
      }
      *reinterpret_cast<float4*>(sx + i) = v;
    }
    __syncthreads();
  };
  for (int tc0 = 0; tc0 < tokens; tc0 += TC) {
    float acc[R][TC];
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
#pragma unroll
      for (int tt = 0; tt < TC; ++tt) acc[rr][tt] = 0.f;
    for (int b0 = 0; b0 < nb; b0 += W) {
      uint32_t word[R][W];
      float sc[R][W];
#pragma unroll
      for (int rr = 0; rr < R; ++rr)
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const int row = row0 + rr, blk = b0 + w;
          const bool live = row < d_out && blk < nb;
          const int64_t cb = (static_cast<int64_t>(row) * nb + blk);
          word[rr][w] = (live && lane < 24) ? __ldg(codes + cb * 24 + lane) : 0u;
          sc[rr][w] = live ? __half2float(scales[cb]) : 0.f;
        }
      // x_rot comes from the rotation kernel launched just before (mode 1)
      if constexpr (MODE == 1) {
        if (b0 == 0 && tc0 == 0) wait_for_prerequisite_grid();
      }
      // the first window's loads are in flight while the CTA stages x; warps past
      // the last row (only in the last CTA) run on zero codes and store nothing
      if constexpr (STAGE) {
        if (b0 == 0) stage_x(tc0);
      }
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const int blk = b0 + w;
        if (blk >= nb) break;
        float v[R][8];
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
          decode_levels(word[rr][w], lane, sc[rr][w], v[rr]);
          if constexpr (MODE == 0) {
            warp_fwht256(v[rr], lane);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[rr][i] *= 0.0625f;
          }
        }
#pragma unroll
        for (int tt = 0; tt < TC; ++tt) {
          const int t = tc0 + tt;
          if (t >= tokens) break;
          const int64_t xo = static_cast<int64_t>(t) * d_in + blk * 256 + 8 * lane;
          float x8[8];
          if constexpr (STAGE) {
            const float* xs = sx + tt * d_in + blk * 256 + 8 * lane;
            const float4 xa = *reinterpret_cast<const float4*>(xs);
            const float4 xb = *reinterpret_cast<const float4*>(xs + 4);
            x8[0] = xa.x; x8[1] = xa.y; x8[2] = xa.z; x8[3] = xa.w;
            x8[4] = xb.x; x8[5] = xb.y; x8[6] = xb.z; x8[7] = xb.w;
          } else if constexpr (MODE == 0) {
            const uint4 h = __ldg(reinterpret_cast<const uint4*>(static_cast<const __half*>(xin) + xo));
            const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
              x8[2 * i] = f.x;
              x8[2 * i + 1] = f.y;
            }
          } else {
            const float4 xa = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(xin) + xo));
            const float4 xb = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(xin) + xo + 4));
            x8[0] = xa.x; x8[1] = xa.y; x8[2] = xa.z; x8[3] = xa.w;
            x8[4] = xb.x; x8[5] = xb.y; x8[6] = xb.z; x8[7] = xb.w;
          }
#pragma unroll
          for (int rr = 0; rr < R; ++rr)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[rr][tt] = fmaf(v[rr][i], x8[i], acc[rr][tt]);
        }
      }
    }
    if constexpr (MODE == 0) {
      if (tc0 + TC >= tokens) allow_dependent_launch();
    }
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
#pragma unroll
      for (int tt = 0; tt < TC; ++tt) {
        const int t = tc0 + tt, row = row0 + rr;
        float a = acc[rr][tt];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (lane == 0 && t < tokens && row < d_out) y[static_cast<int64_t>(t) * d_out + row] = a;
      }
  }
}

// Levels c - 3.5 of the lane's eight elements, as four packed f32x2 pairs.  Code i
// (bits 3i .. 3i + 2 of the lane's 24 bits) is moved to mantissa bits 20 .. 22 of
// 1.0f, giving exactly f = 1 + c / 8, and 8 f - 11.5 = c - 3.5 exactly (one packed
// FMA per pair).  The move is an integer multiply by 2^(20 - 3i) + 2^31 (the 2^31
// term only reaches bit 31, which the mask drops; it keeps the multiply off the
// shift unit, which the masks already keep busy), and a right shift by one for
// i = 7.  Bits past the lane's 24 are masked off.
__device__ __forceinline__ void levels8(uint32_t word, int lane, uint64_t (&lv)[4]) {
  const int bit = 24 * lane;
  const int w0 = bit >> 5;
  const uint32_t lo = __shfl_sync(0xffffffffu, word, w0);
  const uint32_t hi = __shfl_sync(0xffffffffu, word, w0 + 1 < 24 ? w0 + 1 : 23);
  const uint32_t bits = __funnelshift_r(lo, hi, bit & 31);
  const uint64_t eight = (static_cast<uint64_t>(__float_as_uint(8.0f)) << 32) | __float_as_uint(8.0f);
  const uint64_t off = (static_cast<uint64_t>(__float_as_uint(-11.5f)) << 32) | __float_as_uint(-11.5f);
  uint32_t e[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) {
    uint32_t t;
    asm("mul.lo.u32 %0, %1, %2;" : "=r"(t) : "r"(bits), "r"((1u << (20 - 3 * i)) | 0x80000000u));
    e[i] = (t & 0x00700000u) | 0x3F800000u;
  }
  e[7] = ((bits >> 1) & 0x00700000u) | 0x3F800000u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    asm("mov.b64 %0, {%1, %2};" : "=l"(lv[i]) : "r"(e[2 * i]), "r"(e[2 * i + 1]));
    asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(lv[i]) : "l"(eight), "l"(off));
  }
}

// Sum of the eight products level * x, in two packed partial sums.
__device__ __forceinline__ float dot8(const uint64_t (&lv)[4], const float4& xa, const float4& xb) {
  const float x8[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
  uint64_t acc = 0;                                                 // (+0, +0)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint64_t xx;
    asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x8[2 * i]), "f"(x8[2 * i + 1]));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(lv[i]), "l"(xx));
  }
  float a0, a1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
  return a0 + a1;
}

// Mode 1 for up to T tokens in one launch.  A call of two dependent kernels pays two
// launch-to-launch hand-overs for about 1 us of memory traffic; here each CTA
// rotates the tokens of x itself (a warp per 256-block and token, x read from L2)
// into shared memory, so the call is one kernel and needs no workspace.
//  * Before it waits for the kernel launched before it, every thread asks L2 for one
//    128-byte line of the CTA's code words and scales.  A prefetch writes no
//    register, so a kernel still writing them is no hazard: the loads after the wait
//    read what it wrote, now from L2 instead of DRAM.
//  * After the wait each warp rotates its blocks of x, the CTA meets at a barrier,
//    and each warp then loads its code words from L2 for the dot products.
//  * Each warp owns R rows; the CTA's WARPS * R rows share the rotated x.  A row's
//    levels are decoded once per block and meet every token.
template <int WARPS, int R, int W, int T>
__global__ void __launch_bounds__(WARPS * 32) itq3_gemv_rot_kernel(const uint32_t* __restrict__ codes,
                                                                    const __half* __restrict__ scales,
                                                                    const __half* __restrict__ x, int tokens,
                                                                    int d_out, int d_in, float* __restrict__ y) {
  extern __shared__ __align__(16) float sx[];      // H x / 16, [tokens][d_in] fp32
  allow_dependent_launch();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nb = d_in / 256;
  const int row_cta = blockIdx.x * WARPS * R;
  {
    const int rows = min(WARPS * R, d_out - row_cta);
    const char* cb = reinterpret_cast<const char*>(codes) + static_cast<int64_t>(row_cta) * nb * 96;
    const int64_t c_bytes = static_cast<int64_t>(rows) * nb * 96;
    for (int64_t off = static_cast<int64_t>(threadIdx.x) * 128; off < c_bytes; off += WARPS * 32 * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(cb + off));
    const char* sb = reinterpret_cast<const char*>(scales + static_cast<int64_t>(row_cta) * nb);
    const int64_t s_bytes = static_cast<int64_t>(rows) * nb * 2;
    for (int64_t off = static_cast<int64_t>(threadIdx.x) * 128; off < s_bytes; off += WARPS * 32 * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(sb + off));
  }
  wait_for_prerequisite_grid();
  // x first: it is small and stays in L2; the code words (prefetched into L2 above)
  // are loaded once x is rotated, so that no x load queues behind them
  for (int item = warp; item < tokens * nb; item += WARPS) {
    const int64_t base = (T == 1 ? item * 256 : static_cast<int64_t>(item / nb) * d_in + (item % nb) * 256) + lane;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __half2float(x[base + 32 * i]);
    warp_fwht256(v, lane);
#pragma unroll
    for (int i = 0; i < 8; ++i) sx[base + 32 * i] = v[i] * 0.0625f;
  }
  __syncthreads();
  const int row0 = row_cta + warp * R;
  // the scales stay fp16 in registers until they are used
  uint32_t word[R][W];
  __half sc[R][W];
  // a full window of a row's scales is W * 2 contiguous bytes, 16-byte aligned when
  // nb % 8 == 0: then it is read with W / 8 vector loads
  const bool vec_scales = (nb & 7) == 0 && (W & 7) == 0;
  float acc[R][T];
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
#pragma unroll
    for (int tt = 0; tt < T; ++tt) acc[rr][tt] = 0.f;
  for (int b0 = 0; b0 < nb; b0 += W) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      const int row = row0 + rr;
      const uint32_t* crow = codes + (static_cast<int64_t>(row) * nb + b0) * 24 + lane;
      const __half* srow = scales + static_cast<int64_t>(row) * nb + b0;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const bool live = row < d_out && b0 + w < nb;
        word[rr][w] = (live && lane < 24) ? __ldg(crow + 24 * w) : 0u;
      }
      if (vec_scales && row < d_out && b0 + W <= nb) {
#pragma unroll
        for (int w = 0; w < W; w += 8) {
          const uint4 q = __ldg(reinterpret_cast<const uint4*>(srow + w));
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int h = 0; h < 8; ++h)
            sc[rr][w + h] = __ushort_as_half(static_cast<unsigned short>(qw[h / 2] >> (16 * (h & 1))));
        }
      } else {
#pragma unroll
        for (int w = 0; w < W; ++w)
          sc[rr][w] = (row < d_out && b0 + w < nb) ? srow[w] : __ushort_as_half(0);
      }
    }
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int blk = b0 + w;
      if (blk >= nb) break;
      if constexpr (T == 1) {
        // one token: each row's levels go straight into its products
        const float* xs = sx + blk * 256 + 8 * lane;
        const float4 xa = *reinterpret_cast<const float4*>(xs);
        const float4 xb = *reinterpret_cast<const float4*>(xs + 4);
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
          uint64_t lv[4];
          levels8(word[rr][w], lane, lv);
          acc[rr][0] = fmaf(__half2float(sc[rr][w]), dot8(lv, xa, xb), acc[rr][0]);
        }
        continue;
      }
      uint64_t lv[R][4];
#pragma unroll
      for (int rr = 0; rr < R; ++rr) levels8(word[rr][w], lane, lv[rr]);
#pragma unroll
      for (int tt = 0; tt < T; ++tt) {
        if (tt >= tokens) break;
        const float* xs = sx + static_cast<int64_t>(tt) * d_in + blk * 256 + 8 * lane;
        const float4 xa = *reinterpret_cast<const float4*>(xs);
        const float4 xb = *reinterpret_cast<const float4*>(xs + 4);
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
          acc[rr][tt] = fmaf(__half2float(sc[rr][w]), dot8(lv[rr], xa, xb), acc[rr][tt]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
#pragma unroll
    for (int tt = 0; tt < T; ++tt) {
      const int row = row0 + rr;
      float a = acc[rr][tt];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0 && row < d_out && tt < tokens) y[static_cast<int64_t>(tt) * d_out + row] = a;
    }
}

// Largest token-chunk of rotated x (tokens * d_in fp32) the one-launch kernel keeps in
// shared memory.
constexpr int64_t kRotSmemFloats = 40960;

template <int T>
int launch_rot_t(const uint32_t* c32, const __half* sc, const __half* x, int t, int n, int k, float* y,
                 cudaStream_t st) {
  constexpr int kW = 16, kR = 2, kWin = 16;
  auto kern = itq3_gemv_rot_kernel<kW, kR, kWin, T>;
  const size_t smem = static_cast<size_t>(t) * k * 4;
  if (smem > 48 * 1024) {
    static std::atomic<uint64_t> attr_done{0};
    if (set_smem_once(kern, kRotSmemFloats * 4, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((n + kW * kR - 1) / (kW * kR)));
  cfg.blockDim = dim3(kW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, c32, sc, x, t, n, k, y) != cudaSuccess) return WUSH_ERR_CUDA;
  return launch_status();
}

int launch_rot(const uint32_t* c32, const __half* sc, const __half* x, int t, int n, int k, float* y,
               cudaStream_t st) {
  if (t == 1) return launch_rot_t<1>(c32, sc, x, t, n, k, y, st);
  if (t == 2) return launch_rot_t<2>(c32, sc, x, t, n, k, y, st);
  if (t <= 4) return launch_rot_t<4>(c32, sc, x, t, n, k, y, st);
  return launch_rot_t<8>(c32, sc, x, t, n, k, y, st);
}

// Whether a mode-1 call runs as the one-launch kernel (see wush_debug_set_itq3_variant):
// by default for one and two tokens, whose rotated x fits shared memory.
bool use_rot(int t, int k) {
  if (static_cast<int64_t>(t) * k > kRotSmemFloats || t > 8) return false;
  if (g_itq3_variant == 3) return true;
  return t <= 2 && g_itq3_variant != 2;
}

// x_rot[t, blk*256 + e] = (H_256 x[t, blk*256 : +256])[e] / 16; one warp per (t, blk).
__global__ void __launch_bounds__(kWarps * 32) itq3_rotate_x_kernel(const __half* __restrict__ x, int tokens,
                                                                     int d_in, float* __restrict__ x_rot) {
  wait_for_prerequisite_grid();
  allow_dependent_launch();
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

// Rotation of every 256-block of x into x_rot, launched with programmatic stream
// serialization (see above).
int launch_rotation(const __half* x, int t, int k, float* x_rot, cudaStream_t st) {
  const int items = t * (k / 256);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((items + kWarps - 1) / kWarps));
  cfg.blockDim = dim3(kWarps * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, itq3_rotate_x_kernel, x, t, k, x_rot) != cudaSuccess) return WUSH_ERR_CUDA;
  return launch_status();
}

// Rows per warp, blocks per load window and tokens per pass by token count: one
// row and all 16 blocks of a 4096-wide row in flight per warp for a single token
// (memory-bound), more rows sharing each x load as the token count grows.
template <int R, int W, int TC, int MODE>
int launch_one(const uint32_t* c32, const __half* sc, const void* x, int t, int n, int k, float* y, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(TC) * k * 4;
  // a single token's x is read through L1 well enough; staging pays off once a
  // chunk of several tokens is reused by every row of the CTA
  const bool stage = TC > 1 && smem <= 160 * 1024;
  auto kern = stage ? itq3_gemv_kernel<R, W, TC, MODE, true> : itq3_gemv_kernel<R, W, TC, MODE, false>;
  if (stage) {
    static std::atomic<uint64_t> attr_done{0};     // the limit is raised to the 160 KB cap once
    if (smem > 48 * 1024 && set_smem_once(kern, 160 * 1024, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((n + kWarps * R - 1) / (kWarps * R)));
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = stage ? smem : 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, c32, sc, x, t, n, k, y) != cudaSuccess) return WUSH_ERR_CUDA;
  return launch_status();
}

// Rows per warp, blocks per load window and tokens per pass by token count: one
// row and all 16 blocks of a 4096-wide row in flight per warp for a single token,
// four rows sharing each decoded x load once there are several tokens (measured
// best on B200).  For several tokens x is staged in shared memory when a token
// chunk of it fits.
template <int MODE>
int launch_gemv(const uint32_t* c32, const __half* sc, const void* x, int t, int n, int k, float* y,
                cudaStream_t st) {
  if (t == 1) return launch_one<1, 16, 1, MODE>(c32, sc, x, t, n, k, y, st);
  if (t <= 4) return launch_one<4, 4, 4, MODE>(c32, sc, x, t, n, k, y, st);
  return launch_one<4, 4, 8, MODE>(c32, sc, x, t, n, k, y, st);
}

// Mode 1 after the rotation: the tensor-core kernel (itq3_tc.cu) where the shape
// allows it and the CUDA-core kernel above otherwise.
int gemv_rotated(const uint8_t* codes, const void* scales_fp16, const float* x_rot, int t, int n, int k, float* y,
                 cudaStream_t st) {
  if (g_itq3_variant == 0) {
    const int r = itq3_gemv_tc(codes, scales_fp16, x_rot, t, n, k, y, st);
    if (r != WUSH_ERR_UNSUPPORTED) return r;
  }
  return launch_gemv<1>(reinterpret_cast<const uint32_t*>(codes), static_cast<const __half*>(scales_fp16), x_rot, t,
                        n, k, y, st);
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
  if (!codes || !scales_fp16 || !x_fp16 || !y || !aligned16(codes) || !aligned16(scales_fp16) || !aligned16(x_fp16))
    return WUSH_ERR_INVALID_ARG;
  if (mode == 1 && (!workspace || !aligned16(workspace))) return WUSH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* c32 = reinterpret_cast<const uint32_t*>(codes);
  const auto* sc = static_cast<const __half*>(scales_fp16);
  const auto* xh = static_cast<const __half*>(x_fp16);
  const int t = static_cast<int>(tokens), n = static_cast<int>(d_out), k = static_cast<int>(d_in);
  if (mode == 0) return launch_gemv<0>(c32, sc, xh, t, n, k, y, st);
  if (use_rot(t, k)) return launch_rot(c32, sc, xh, t, n, k, y, st);
  if (launch_rotation(xh, t, k, workspace, st) != WUSH_OK) return WUSH_ERR_CUDA;
  return gemv_rotated(codes, scales_fp16, workspace, t, n, k, y, st);
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

// Per device: the context the address was looked up in, and the address.
struct ScratchEntry {
  unsigned long long ctx_id;
  float* addr;
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context (ids are never reused within a process,
// also when a context is destroyed and a new one made at the same handle); 0 when
// it cannot be had.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array in the current device's context, looked up
// once per device and context: a device reset makes a new context and module, so
// the next call looks the address up again.  (In host code the array's name is
// only a host-side stand-in, so the kernels must be handed this address, never the
// name.)
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WUSH_ERR_CUDA;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& e = g_scratch[dev];
  // (no current context yet: id 0, looked up again until a context is current)
  if (!e.addr || id == 0 || e.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_itq3_noalloc_scratch) != cudaSuccess || !p) return WUSH_ERR_CUDA;
    e.addr = static_cast<float*>(p);
    e.ctx_id = id;
  }
  *out = e.addr;
  return WUSH_OK;
}

}  // namespace
}  // namespace wush

extern "C" int itq3_dequant_gemv_noalloc(const uint8_t* codes, const void* scales_fp16, const void* x_fp16,
                                         int64_t tokens, int64_t d_out, int64_t d_in, float* y, void* stream) {
  if (tokens < 1 || tokens > 16 || d_out <= 0 || d_in <= 0 || d_in % 256 || d_out % 8) return WUSH_ERR_INVALID_ARG;
  if (tokens * d_in > kNoAllocScratchFloats) return WUSH_ERR_BUFFER_TOO_SMALL;
  if (d_out > (int64_t(1) << 30)) return WUSH_ERR_UNSUPPORTED;
  if (!codes || !scales_fp16 || !x_fp16 || !y || !aligned16(codes) || !aligned16(scales_fp16) || !aligned16(x_fp16))
    return WUSH_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const auto* xh = static_cast<const __half*>(x_fp16);
  const int t = static_cast<int>(tokens), n = static_cast<int>(d_out), k = static_cast<int>(d_in);
  if (use_rot(t, k))
    return launch_rot(reinterpret_cast<const uint32_t*>(codes), static_cast<const __half*>(scales_fp16), xh, t, n, k,
                      y, s);
  float* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != WUSH_OK) return st;
  // The rotation kernel writes every scratch element the GEMV then reads, so
  // nothing left there by an earlier call needs clearing.
  if (launch_rotation(xh, t, k, scratch, s) != WUSH_OK) return WUSH_ERR_CUDA;
  return gemv_rotated(codes, scales_fp16, scratch, t, n, k, y, s);
}
