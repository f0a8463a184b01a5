// Fused per-block transform + microscaled quantisation on tcgen05 tensor cores
// (bf16 activations).
//
// WUSH news article, paragraph 6 (only the activations are transformed at
// inference; blocks are independent) and AI Radio episode, "The gist" (a fused
// GPU implementation).  The format rules are stated in wush.h.
//
// A persistent CTA walks a contiguous range of 128-row x 128-column tiles of X in
// column-major order (so a CTA meets at most a few columns of T), with three roles:
//   warp 0     TMA producer: each tile is two 128-byte-swizzled boxes of 64 bf16
//              columns, landing in a 5-stage shared-memory ring;
//   warp 1     MMA issuer (WUS/WUSH): y = x T^T per b-block as kind::f16 MMAs,
//              M = 128 rows, K = 16 per instruction.  T is split exactly into three
//              bf16 parts (hi + mid + lo = the fp32 T).  Quarter q (32 columns)
//              of every tile goes to TMEM slot q of an accumulator set; the
//              epilogue frees a set as soon as its TMEM loads are done, so the
//              next tile's MMAs overlap this tile's quantisation.
//                b = 16: per K-step one MMA, N = 3b, against [T_hi; T_mid; T_lo]
//                stacked along N: three partial products side by side, one
//                384-column set (8 MMAs per tile).
//                b = 32: per K-step one MMA, N = 2b, against [T_hi; T_mid] and a
//                second, N = b, adding x T_lo^T onto the T_hi columns: two partial
//                products, two 256-column sets alternating by tile (16 MMAs per
//                tile).  Measured side by side, each form is the faster one for
//                its block size;
//   warps 2-17 epilogue, four warpgroups, warpgroup q owning quarter q of every
//              tile: one thread per row reads the partial products of its row out
//              of TMEM (tcgen05.ld 32x32b) and adds them -- y = hi + (mid + lo),
//              or (hi + lo) + mid for b = 32 --
//              or, for identity and Hadamard, reads X out of the swizzled
//              shared-memory tile -- and computes absmax, scale and codes in
//              registers (hardware cvt.rn.satfinite e2m1x2 / e4m3x2), storing
//              packed codes and scale bytes.  The same warps convert each new
//              column's fp32 T into the stacked bf16 operand in shared memory
//              (two column buffers).
// Every mbarrier wait is bounded (see sm100.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "quant_decide.cuh"
#include "sm100.cuh"

namespace wush {
namespace {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kTileCols = 128;                       // bf16 elements
constexpr int kQuarterCols = 32;                     // columns of a tile owned by one epilogue warpgroup
constexpr int kBoxCols = 64;                         // 128 bytes
constexpr int kStages = 5;
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kEpiGroups = kTileCols / kQuarterCols; // epilogue warpgroups, one quarter each
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kStageBytes = kTileRows * kTileCols * 2;  // 32 KB
constexpr int kBoxBytes = kTileRows * kBoxCols * 2;     // 16 KB
constexpr int kTBufBytes = 24 * 1024;
constexpr uint32_t kTmemCols = 512;                // allocation: the power of two >= kSets * kSetCols
constexpr int64_t kDefaultPolls = int64_t(1) << 40;
constexpr uint64_t kDeadlineNs = 4000000000ull;
constexpr int kSmemBytes = kStages * kStageBytes + 2 * kTBufBytes + 1024 + 256;
static_assert(kEpiGroups * 4 == kEpiWarps, "four warps per epilogue warpgroup");
static_assert(kTmemCols == 512, "TMEM allocation is a power of two of at most 512 columns");

// TMEM accumulator layout per block size (see the file comment).
template <int B>
struct AccLayout {
  static constexpr bool kThree = B == 16;                   // one N = 3b MMA per K-step
  static constexpr int kParts = kThree ? 3 : 2;             // partial products per block in TMEM
  static constexpr int kSlotCols = (kQuarterCols / B) * kParts * B;  // one quarter: 96 or 64 columns
  static constexpr int kSets = kThree ? 1 : 2;              // accumulator sets (whole tiles)
  static constexpr int kSetCols = kEpiGroups * kSlotCols;   // 384 or 256
  static_assert(kSets * kSetCols <= static_cast<int>(kTmemCols), "TMEM holds 512 columns");
};

enum Kind : int { kIdentity = 0, kHadamard = 1, kDense = 2 };
// kAm: no quantisation; the kernel's only output is max |T x| over the tensor
enum Fmt : int { kMx = 0, kNv = 1, kI4 = 2, kAm = 3 };

__device__ int g_tq_error = 0;

// max |y_i| as a pairwise tree (max is exact, so the order is free): depth log2 B
// instead of a B-long dependent chain.
template <int B>
__device__ __forceinline__ float block_amax(const float (&y)[B]) {
  float m[B / 2];
#pragma unroll
  for (int i = 0; i < B / 2; ++i) m[i] = fmaxf(fabsf(y[2 * i]), fabsf(y[2 * i + 1]));
#pragma unroll
  for (int w = B / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

// Quantise one block of B fp32 values held by this thread.  Writes B/8 code
// words and returns the scale (byte for MXFP4/NVFP4, fp16 bits for INT4).  Every
// decision is the round-to-nearest-even of the exact quotient (quant_decide.cuh).
template <int B, int FMT>
__device__ __forceinline__ uint32_t quantize_block(const float (&y)[B], float gscale, float inv_den,
                                                  uint32_t (&w)[B / 8]) {
  const float amax = block_amax<B>(y);
  if constexpr (FMT == kMx) {
    int e = amax > 0.f ? floor_log2(amax) - 2 : -127;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    const float inv = exp2i(-e);                 // y * 2^-e is exact
#pragma unroll
    for (int q = 0; q < B / 8; ++q) w[q] = amax > 0.f ? e2m1x8_times(y + 8 * q, inv) : 0u;
    return static_cast<uint32_t>(e + 127);
  } else if constexpr (FMT == kNv) {
    const uint32_t sb = nvfp4_scale_byte(amax, gscale, inv_den);
    const float sbv = ue4m3_val(sb);
    const bool live = sb != 0u && amax > 0.f;
    const float r = live ? __frcp_rn(__fmul_rn(sbv, gscale)) : 0.f;
#pragma unroll
    for (int q = 0; q < B / 8; ++q) w[q] = live ? nvfp4_codes8(y + 8 * q, r, sbv, gscale) : 0u;
    return sb;
  } else {
    const __half s16 = int4_scale(amax);
    const float s = __half2float(s16);
    const float r = s > 0.f ? __frcp_rn(s) : 0.f;
#pragma unroll
    for (int q = 0; q < B / 8; ++q) w[q] = s > 0.f ? int4_codes8(y + 8 * q, r, s) : 0u;
    return static_cast<uint32_t>(__half_as_ushort(s16));
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
  const float s = B == 32 ? 0.17677669529663688f : 0.25f;
#pragma unroll
  for (int i = 0; i < B; ++i) y[i] *= s;
}

// (a0, a1) + (b0, b1) as one packed f32x2 add, each lane rounded to nearest like FADD.
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  unsigned long long x, y, z;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(z));
}

template <int B>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[B]) {
  if constexpr (B == 32) tmem_ld_32x32b_x32(taddr, r);
  else tmem_ld_32x32b_x16(taddr, r);
}

// Ties loaded registers to the preceding tcgen05.wait::ld: the empty asm statements
// are ordered after it, so no use of a value is scheduled before the load landed.
template <int B>
__device__ __forceinline__ void tmem_tie(uint32_t (&r)[B]) {
#pragma unroll
  for (int i = 0; i < B; ++i) asm volatile("" : "+r"(r[i]));
}

// y = hi + (mid + lo) for one b-block of this thread's row (b = 16): the MMA
// leaves x T_hi^T, x T_mid^T and x T_lo^T in TMEM columns taddr + [0, B),
// [B, 2B) and [2B, 3B).  The two small parts are added first.
template <int B>
__device__ __forceinline__ void tmem_sum3(uint32_t taddr, float (&y)[B]) {
  uint32_t h[B], m[B], l[B];
  tmem_ld_cols<B>(taddr, h);
  tmem_ld_cols<B>(taddr + B, m);
  tmem_ld_cols<B>(taddr + 2 * B, l);
  tmem_ld_wait();
  tmem_tie<B>(h);
  tmem_tie<B>(m);
  tmem_tie<B>(l);
#pragma unroll
  for (int i = 0; i < B; i += 2) {
    float s0 = __uint_as_float(m[i]), s1 = __uint_as_float(m[i + 1]);
    add2(s0, s1, __uint_as_float(l[i]), __uint_as_float(l[i + 1]));
    y[i] = __uint_as_float(h[i]);
    y[i + 1] = __uint_as_float(h[i + 1]);
    add2(y[i], y[i + 1], s0, s1);
  }
}

// tmem_sum3 for both b = 16 blocks of a quarter: columns [0, 48) hold block 0's
// hi, mid and lo, [48, 96) block 1's.  Block 1's loads are issued before block 0's
// sums are formed, so their latency overlaps that arithmetic.
__device__ __forceinline__ void tmem_sum3_pair16(uint32_t taddr, float (&y0)[16], float (&y1)[16]) {
  uint32_t h[16], m[16], l[16];
  tmem_ld_cols<16>(taddr, h);
  tmem_ld_cols<16>(taddr + 16, m);
  tmem_ld_cols<16>(taddr + 32, l);
  tmem_ld_wait();
  tmem_tie<16>(h);
  tmem_tie<16>(m);
  tmem_tie<16>(l);
  uint32_t h1[16], m1[16], l1[16];
  tmem_ld_cols<16>(taddr + 48, h1);
  tmem_ld_cols<16>(taddr + 64, m1);
  tmem_ld_cols<16>(taddr + 80, l1);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    float s0 = __uint_as_float(m[i]), s1 = __uint_as_float(m[i + 1]);
    add2(s0, s1, __uint_as_float(l[i]), __uint_as_float(l[i + 1]));
    y0[i] = __uint_as_float(h[i]);
    y0[i + 1] = __uint_as_float(h[i + 1]);
    add2(y0[i], y0[i + 1], s0, s1);
  }
  tmem_ld_wait();
  tmem_tie<16>(h1);
  tmem_tie<16>(m1);
  tmem_tie<16>(l1);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    float s0 = __uint_as_float(m1[i]), s1 = __uint_as_float(m1[i + 1]);
    add2(s0, s1, __uint_as_float(l1[i]), __uint_as_float(l1[i + 1]));
    y1[i] = __uint_as_float(h1[i]);
    y1[i + 1] = __uint_as_float(h1[i + 1]);
    add2(y1[i], y1[i + 1], s0, s1);
  }
}

// y = (hi + lo) + mid for one b-block of this thread's row (b = 32): the MMAs
// leave x (T_hi + T_lo)^T in TMEM columns taddr + [0, B) and x T_mid^T in [B, 2B).
template <int B>
__device__ __forceinline__ void tmem_sum2(uint32_t taddr, float (&y)[B]) {
  uint32_t a[B], c[B];
  tmem_ld_cols<B>(taddr, a);
  tmem_ld_cols<B>(taddr + B, c);
  tmem_ld_wait();
  tmem_tie<B>(a);
  tmem_tie<B>(c);
#pragma unroll
  for (int i = 0; i < B; i += 2) {
    y[i] = __uint_as_float(a[i]);
    y[i + 1] = __uint_as_float(a[i + 1]);
    add2(y[i], y[i + 1], __uint_as_float(c[i]), __uint_as_float(c[i + 1]));
  }
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t m, uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int B, int FMT, int KIND, bool DBG>
__global__ void __launch_bounds__(kThreads, 1)
    tq_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const float* __restrict__ t,
                 const int* __restrict__ t_index, int n_t, float gscale_arg,
                 const float* __restrict__ gs_amax, float* __restrict__ gs_out, uint8_t* __restrict__ codes, void* __restrict__ scales, float* __restrict__ ydbg, int rows,
                 int d_in, int n_row_tiles, int n_tiles, int64_t max_polls) {
  constexpr int kBlocks = kTileCols / B;           // b-blocks per tile: 4 or 8
  constexpr int kQBlocks = kQuarterCols / B;       // b-blocks per quarter: 1 or 2
  constexpr int kKSteps = B / 16;                  // K = 16 per MMA
  using L = AccLayout<B>;
  constexpr int kN = L::kParts * B;                // N of the stacked MMA: [T_hi; T_mid(; T_lo)]
  constexpr int kSlotCols = L::kSlotCols, kSets = L::kSets, kSetCols = L::kSetCols;
  constexpr int kChunk = B * 32;                   // bytes of one [B n x 16 k] bf16 operand chunk
  constexpr bool kMma = KIND == kDense;
  static_assert(kQBlocks * kN <= kSlotCols, "a quarter's partial products must fit its TMEM slot");
  static_assert(kSets * kSetCols <= 512, "TMEM holds 512 columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tbuf = smem + kStages * kStageBytes;
  uint64_t* x_full = reinterpret_cast<uint64_t*>(tbuf + 2 * kTBufBytes);
  uint64_t* x_empty = x_full + kStages;
  uint64_t* acc_full = x_empty + kStages;
  uint64_t* acc_empty = acc_full + kSets;
  uint64_t* t_full = acc_empty + kSets;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(t_full + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nb = d_in / B;
  const int tile_lo = static_cast<int>(static_cast<int64_t>(blockIdx.x) * n_tiles / gridDim.x);
  const int tile_hi = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * n_tiles / gridDim.x);
  const int col_lo = tile_lo / n_row_tiles;

  // Every ring and slot below has consumers that each take its phases in order,
  // so the parity waits are unambiguous for any ring depth: the MMA warp (or all
  // sixteen epilogue warps) for the X stages, all epilogue warps for the TMEM
  // accumulator set(s).  Epilogue warps poll with lane 0 and
  // release with one arrival per warp.
  const int n_mine = tile_hi - tile_lo;
  const int n_cols = n_mine > 0 ? (tile_hi - 1) / n_row_tiles - col_lo + 1 : 0;
  // Right after the launch wait, thread 0 sends the first X loads and the epilogue
  // threads then fetch the fp32 T of this CTA's first two columns, ahead of the rest
  // of the X tiles.
  constexpr int kTGroups = kBlocks * B * B / 4;    // float4 groups of T per column
  constexpr int kTPer = kTGroups / kEpiThreads;    // per epilogue thread: 2 or 1
  static_assert(kTPer * kEpiThreads == kTGroups, "T column splits evenly over the epilogue threads");
  // T of block j: t[j], or t[t_index[j]] (clamped to the n_t transforms) when
  // blocks share transforms
  auto t_block = [&](int j) -> const float* {
    int jt = j;
    if (t_index) {
      const int v = __ldg(t_index + j);
      jt = v < 0 ? 0 : (v >= n_t ? n_t - 1 : v);
    }
    return t + static_cast<int64_t>(jt) * B * B;
  };
  auto issue_load = [&](int n) {
    const int i = tile_lo + n, s = n % kStages;
    const int row0 = (i % n_row_tiles) * kTileRows, col0 = (i / n_row_tiles) * kTileCols;
    uint8_t* st = smem + s * kStageBytes;
    mbar_arrive_expect_tx(&x_full[s], kStageBytes);
    tma_load_2d(st, &tmap_x, col0, row0, &x_full[s]);
    tma_load_2d(st + kBoxBytes, &tmap_x, col0 + kBoxCols, row0, &x_full[s]);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], kMma ? 1 : kEpiWarps);
    }
    for (int p = 0; p < kSets; ++p) {
      mbar_init(&acc_full[p], 1);
      mbar_init(&acc_empty[p], kEpiWarps);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&t_full[b], 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmap_x);
  }
  if (warp == 1 && kMma) tmem_alloc(tmem_slot, kTmemCols);
  // Launched after another kernel with programmatic stream serialization, the set-up
  // above overlaps that kernel's tail; no global input is read and no output written
  // before the wait.
  pdl_launch_dependents();
  pdl_wait();
  // the ring starts empty: the first loads go out before the rest of the set-up
  if (threadIdx.x == 0)
    for (int n = 0; n < kStages && n < n_mine; ++n) issue_load(n);
  float4 t_pre[2][kTPer];
  if (kMma && threadIdx.x >= 64) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int p = 0; p < kTPer; ++p) {
        const int e0 = 4 * (static_cast<int>(threadIdx.x) - 64 + p * kEpiThreads);
        const int j = (col_lo + c) * kBlocks + e0 / (B * B);
        t_pre[c][p] = (c < n_cols && j < nb) ? __ldg(reinterpret_cast<const float4*>(t_block(j) + e0 % (B * B)))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = kMma ? *tmem_slot : 0u;

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      atomicOr(&g_tq_error, 1 << kErrTimeoutBarrier);
    }
  };

  if (warp == 0) {
    if (threadIdx.x == 0) {
      for (int n = kStages; n < n_mine; ++n) {
        if (!mbar_wait_bounded(&x_empty[n % kStages], ((n / kStages) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
          give_up();
          break;
        }
        issue_load(n);
      }
    }
  } else if (warp == 1) {
    if (kMma && elect_one()) {
      // Tile n goes to accumulator set n % kSets; quarter q of it to columns
      // kSetCols (n % kSets) + kSlotCols q.  Per b-block and K-step one MMA against
      // the stacked parts (N = 3b, or N = 2b plus one N = b MMA for T_lo onto the
      // T_hi columns).  Descriptors are a per-tile base plus constant offsets.
      constexpr uint32_t idesc_n = idesc_bf16_f32(kTileRows, kN);
      constexpr uint32_t idesc_lo = idesc_bf16_f32(kTileRows, B);
      bool ok = true;
      int col = col_lo, row_tile = tile_lo % n_row_tiles, k_ready = -1;
      for (int n = 0; n < n_mine; ++n) {
        const int s = n % kStages, p = n % kSets, k = col - col_lo;
        if (k != k_ready) {
          if (!mbar_wait_bounded(&t_full[k & 1], (k >> 1) & 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
          k_ready = k;
        }
        if (!mbar_wait_bounded(&x_full[s], (n / kStages) & 1, max_polls, kDeadlineNs, abort_flag) ||
            !mbar_wait_bounded(&acc_empty[p], ((n / kSets) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = desc_kmajor_sw128(smem_u32(smem + s * kStageBytes));
        const uint64_t b0 = smem_desc(smem_u32(tbuf + (k & 1) * kTBufBytes), 128, 256, kLayoutNone);
        const uint32_t d0 = tmem + p * kSetCols;
#pragma unroll
        for (int jj = 0; jj < kBlocks; ++jj) {
          const int col_bytes = jj * B * 2;                      // b-block jj within the tile
          const uint32_t a_off = (col_bytes / 128) * kBoxBytes + (col_bytes % 128);
          const uint32_t d = d0 + (jj / kQBlocks) * kSlotCols + (jj % kQBlocks) * kN;
#pragma unroll
          for (int kk = 0; kk < kKSteps; ++kk) {
            const uint64_t ad = a0 + ((a_off + kk * 32) >> 4);
            const uint32_t b_off = (jj * kKSteps + kk) * 3 * kChunk;
            mma_bf16(d, ad, b0 + (b_off >> 4), idesc_n, kk ? 1u : 0u);
            if constexpr (!L::kThree) mma_bf16(d, ad, b0 + ((b_off + 2 * kChunk) >> 4), idesc_lo, 1u);
          }
        }
        tc_commit(&acc_full[p]);
        tc_commit(&x_empty[s]);
        if (++row_tile == n_row_tiles) { row_tile = 0; ++col; }
      }
      if (!ok) give_up();
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // Four warpgroups of 4 warps; warpgroup g owns columns [32 g, 32 g + 32) of
    // every tile (TMEM columns kSlotCols g .. of the tile's accumulator set).  Warp w may read only TMEM lane quarter w % 4, i.e.
    // rows 32 (w % 4) .. + 31, and each thread handles one row of the quarter.
    const int et = threadIdx.x - 64;            // 0..511
    const int g = et / 128;                     // warpgroup = quarter
    const int q = warp & 3;
    const int rloc = q * 32 + lane;             // row within the tile
    // NVFP4 per-tensor scale: the caller's, or derived from a device amax
    float gscale = gscale_arg;
    if (FMT == kNv && gs_amax) {
      gscale = nvfp4_dynamic_scale(__ldg(gs_amax));
      if (gs_out && blockIdx.x == 0 && et == 0) *gs_out = gscale;
    }
    const float inv_den = __frcp_rn(__fmul_rn(6.0f, gscale));   // 1 / (6 s_g), for the scale bracket
    const int n_atom_cols = (nb + 3) / 4;

    // Four fp32 values of T (group gi of a column: block jj, output row nrow,
    // inputs kcol .. kcol + 3) -> the three bf16 parts in T buffer dst.  Chunk
    // (block jj, K-step kk) holds the parts hi, mid, lo one after another, i.e. a
    // [3b n x 16 k] K-major operand whose row n = part * b + output index.
    auto t_store_group = [&](uint8_t* dst, int gi, float4 v) {
      const int e0 = 4 * gi;
      const int jj = e0 / (B * B), nrow = (e0 / B) % B, kcol = e0 % B;
      const int kk = kcol / 16, kin = kcol % 16;
      const int off = (nrow / 8) * 256 + (kin / 8) * 128 + (nrow % 8) * 16 + (kin % 8) * 2;
      const float x4[4] = {v.x, v.y, v.z, v.w};
      uint32_t h[3][4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        h[0][c] = bf16_bits_rn(x4[c]);
        const float r1 = x4[c] - __uint_as_float(h[0][c] << 16);
        h[1][c] = bf16_bits_rn(r1);
        const float r2 = r1 - __uint_as_float(h[1][c] << 16);
        h[2][c] = bf16_bits_rn(r2);
      }
#pragma unroll
      for (int sp = 0; sp < 3; ++sp)
        *reinterpret_cast<uint2*>(dst + ((jj * kKSteps + kk) * 3 + sp) * kChunk + off) =
            make_uint2(h[sp][0] | (h[sp][1] << 16), h[sp][2] | (h[sp][3] << 16));
    };
    // fp32 T of column col_lo + k -> buffer k & 1, by nthr threads (id tid); all
    // float4 loads of a thread are issued first.
    auto convert_t = [&](int k, int tid, int nthr, int bar_id) {
      uint8_t* dst = tbuf + (k & 1) * kTBufBytes;
      const int j0 = (col_lo + k) * kBlocks;
      for (int base = 0; base < kTGroups; base += 8 * nthr) {
        float4 v[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int gi = base + tid + p * nthr;
          const int e0 = 4 * gi;
          v[p] = (gi < kTGroups && j0 + e0 / (B * B) < nb)
                     ? __ldg(reinterpret_cast<const float4*>(t_block(j0 + e0 / (B * B)) + e0 % (B * B)))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int gi = base + tid + p * nthr;
          if (gi < kTGroups) t_store_group(dst, gi, v[p]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthr) : "memory");
      if (tid == 0) mbar_arrive(&t_full[k & 1]);
    };
    if constexpr (kMma) {
      // columns 0 and 1 from the values fetched at kernel entry
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int p = 0; p < kTPer; ++p) t_store_group(tbuf + c * kTBufBytes, et + p * kEpiThreads, t_pre[c][p]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.sync %0, %1;" ::"r"(1), "r"(kEpiThreads) : "memory");
      if (et == 0) {
        mbar_arrive(&t_full[0]);
        mbar_arrive(&t_full[1]);
      }
    }

    float run_max = 0.f;                        // kAm: this thread's max |y|
    // tile i = (column col, row tile row_tile), advanced incrementally: no division
    // by the runtime row-tile count inside the loop
    int col = col_lo, row_tile = tile_lo - col_lo * n_row_tiles;
    for (int i = tile_lo; i < tile_hi; ++i) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int n = i - tile_lo, s = n % kStages;
      const int row0 = row_tile * kTileRows, col0 = col * kTileCols;
      const int r = row0 + rloc;
      const bool row_ok = r < rows;
      const int p = n % kSets;
      uint64_t* full = kMma ? &acc_full[p] : &x_full[s];
      const uint32_t parity = kMma ? (n / kSets) & 1 : (n / kStages) & 1;
      // lane 0 polls; once it has seen the phase complete, every lane's own
      // try_wait succeeds at once and gives that lane its acquire
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(full, parity, max_polls, kDeadlineNs, abort_flag);
      __syncwarp();
      if (!__shfl_sync(0xffffffffu, ok, 0)) { give_up(); break; }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(full, parity, max_polls, kDeadlineNs, abort_flag))) {
        give_up();
        break;
      }

      float y[kQBlocks][B];
      if constexpr (kMma) {
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + p * kSetCols + g * kSlotCols;
        if constexpr (L::kThree && kQBlocks == 2 && B == 16) {
          // both blocks' three partial products (96 contiguous columns) in one round
          // trip: three loads, one wait
          tmem_sum3_pair16(taddr, y[0], y[1]);
        } else {
#pragma unroll
          for (int u = 0; u < kQBlocks; ++u) {
            if constexpr (L::kThree) tmem_sum3<B>(taddr + u * kN, y[u]);
            else tmem_sum2<B>(taddr + u * kN, y[u]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[p]);
      } else {
        const uint8_t* sx = smem + s * kStageBytes;
#pragma unroll
        for (int u = 0; u < kQBlocks; ++u) {
          const int col_bytes = (g * kQBlocks + u) * B * 2;
          const uint8_t* rowp = sx + (col_bytes / 128) * kBoxBytes + rloc * 128;
#pragma unroll
          for (int c = 0; c < B / 8; ++c) {
            const int chunk = (col_bytes % 128) / 16 + c;
            const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((chunk ^ (rloc & 7)) * 16));
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              y[u][8 * c + 2 * h] = bf16_lo(wd[h]);
              y[u][8 * c + 2 * h + 1] = bf16_hi(wd[h]);
            }
          }
          if constexpr (KIND == kHadamard) fwht_normalized<B>(y[u]);
        }
        // The next writer of this stage is the TMA engine (async proxy): order
        // this thread's shared-memory reads of it before that write.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_empty[s]);
      }

#pragma unroll
      for (int u = 0; u < kQBlocks; ++u) {
        const int j = col0 / B + g * kQBlocks + u;
        const bool blk_ok = row_ok && j < nb;
        if constexpr (DBG) {
          if (blk_ok) {
            float4* dp =
                reinterpret_cast<float4*>(ydbg + static_cast<int64_t>(r) * d_in + static_cast<int64_t>(j) * B);
#pragma unroll
            for (int w = 0; w < B / 4; ++w)
              dp[w] = make_float4(y[u][4 * w], y[u][4 * w + 1], y[u][4 * w + 2], y[u][4 * w + 3]);
          }
        }
        if constexpr (FMT == kAm) {
          if (blk_ok) {
#pragma unroll
            for (int e = 0; e < B; ++e) run_max = fmaxf(run_max, fabsf(y[u][e]));
          }
        } else {
          uint32_t cw[B / 8];
          const uint32_t sc = quantize_block<B, FMT>(y[u], gscale, inv_den, cw);
          if (blk_ok) {
            uint8_t* cp = codes + static_cast<int64_t>(r) * (d_in / 2) + static_cast<int64_t>(j) * (B / 2);
            if constexpr (B == 32) *reinterpret_cast<uint4*>(cp) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            else *reinterpret_cast<uint2*>(cp) = make_uint2(cw[0], cw[1]);
          }
          if constexpr (FMT == kI4) {
            if (blk_ok)
              reinterpret_cast<uint16_t*>(scales)[static_cast<int64_t>(r) * nb + j] = static_cast<uint16_t>(sc);
          } else if (j < n_atom_cols * 4) {
            // padding rows and columns of an existing atom are written as zero
            static_cast<uint8_t*>(scales)[sf_offset(r, j, n_atom_cols)] = static_cast<uint8_t>(blk_ok ? sc : 0u);
          }
        }
      }

      if constexpr (kMma) {
        // Warpgroup kEpiGroups - 1 sees its slot's commit last in each tile, and a
        // commit covers every MMA issued before it: after the last tile of column k,
        // no MMA reads that column's T buffer any more, so it refills it with k + 2.
        if (g == kEpiGroups - 1) {
          const int k = col - col_lo;
          const bool last_of_col = (i + 1 == tile_hi) || (row_tile + 1 == n_row_tiles);
          if (last_of_col && k + 2 < n_cols) convert_t(k + 2, et - g * 128, 128, 2 + g);
        }
      }
      if (++row_tile == n_row_tiles) {
        row_tile = 0;
        ++col;
      }
    }
    if constexpr (FMT == kAm) {
      // non-negative floats order like their bit patterns; gs_out holds the
      // tensor's running amax (zeroed by the caller)
      const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(run_max));
      if (lane == 0 && m) atomicMax(reinterpret_cast<unsigned int*>(gs_out), m);
    }
  }

  __syncwarp();
  if (*abort_flag) {
    const uint64_t until = globaltimer_ns() + 200000ull;
    while (globaltimer_ns() < until) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1 && kMma) tmem_dealloc(tmem, kTmemCols);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

int num_sms() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int B, int FMT, int KIND, bool DBG>
int launch_tc(const void* x, int64_t rows, int64_t d_in, const float* t, const int* t_index, int n_t, float gscale,
              const float* gs_amax, float* gs_out, uint8_t* codes, void* scales, float* ydbg, cudaStream_t st) {
  EncodeFn enc = get_encode();
  if (!enc) return WUSH_ERR_CUDA;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d_in), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d_in) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBoxCols), static_cast<cuuint32_t>(kTileRows)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return WUSH_ERR_CUDA;
  auto kern = tq_tc_kernel<B, FMT, KIND, DBG>;
  static std::atomic<uint64_t> attr_done{0};
  if (set_smem_once(kern, kSmemBytes, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  const int n_row_tiles = static_cast<int>((rows + kTileRows - 1) / kTileRows);
  const int n_col_tiles = static_cast<int>((d_in + kTileCols - 1) / kTileCols);
  const int n_tiles = n_row_tiles * n_col_tiles;
  const int sms = num_sms();
  if (sms <= 0) return WUSH_ERR_CUDA;
  const int grid = n_tiles < sms ? n_tiles : sms;
  const int64_t polls = g_wait_limit_override > 0 ? g_wait_limit_override : kDefaultPolls;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, map, t, t_index, n_t, gscale, gs_amax, gs_out, codes, scales, ydbg,
                         static_cast<int>(rows), static_cast<int>(d_in), n_row_tiles, n_tiles, polls) != cudaSuccess)
    return WUSH_ERR_CUDA;
  return launch_status();
}

template <int B, int FMT>
int dispatch_kind(int kind, const void* x, int64_t rows, int64_t d_in, const float* t, const int* t_index, int n_t,
                  float gscale, const float* gs_amax, float* gs_out, uint8_t* codes, void* scales, float* ydbg,
                  cudaStream_t st) {
  const int k = kind == WUSH_T_IDENTITY ? kIdentity : (kind == WUSH_T_HADAMARD ? kHadamard : kDense);
#define WUSH_TC(KK)                                                                                             \
  return ydbg ? launch_tc<B, FMT, KK, true>(x, rows, d_in, t, t_index, n_t, gscale, gs_amax, gs_out, codes, scales, \
                                            ydbg, st)                                                             \
              : launch_tc<B, FMT, KK, false>(x, rows, d_in, t, t_index, n_t, gscale, gs_amax, gs_out, codes, scales, \
                                             ydbg, st)
  if (k == kIdentity) { WUSH_TC(kIdentity); }
  if (k == kHadamard) { WUSH_TC(kHadamard); }
  WUSH_TC(kDense);
#undef WUSH_TC
}

}  // namespace

int read_and_clear_tq_error(int* word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_tq_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (*word) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_tq_error, &zero, sizeof(int));
  }
  return e;
}

// Tensor-core form of wush_transform_quant for bf16 inputs whose rows are 16-byte
// aligned and whose sizes fit int32 indexing.  Returns WUSH_ERR_UNSUPPORTED when the
// shape is outside that, so the caller can use the one-row-per-thread kernel.
// max |T x| of a bf16 tensor into *amax_out (atomicMax on its bits; the caller
// zeroes it first) by the tensor-core kernel; WUSH_ERR_UNSUPPORTED for shapes it
// does not take.
int transform_amax_tc(const void* x, int64_t rows, int64_t d_in, const float* t, int kind, int block,
                      float* amax_out, cudaStream_t st) {
  if (d_in % 8 || rows > (int64_t(1) << 30) || d_in > (int64_t(1) << 30)) return WUSH_ERR_UNSUPPORTED;
  if (block == 32)
    return dispatch_kind<32, kAm>(kind, x, rows, d_in, t, nullptr, 0, 1.0f, nullptr, amax_out, nullptr, nullptr,
                                  nullptr, st);
  if (block == 16)
    return dispatch_kind<16, kAm>(kind, x, rows, d_in, t, nullptr, 0, 1.0f, nullptr, amax_out, nullptr, nullptr,
                                  nullptr, st);
  return WUSH_ERR_UNSUPPORTED;
}

int transform_quant_tc(const void* x, int64_t rows, int64_t d_in, const float* t, const int* t_index, int n_t,
                       int kind, int fmt, float gscale, const float* gs_amax, float* gs_out, uint8_t* codes,
                       void* scales, float* ydbg, cudaStream_t st) {
  if (d_in % 8 || rows > (int64_t(1) << 30) || d_in > (int64_t(1) << 30) || rows * (d_in / 2) > (int64_t(1) << 62))
    return WUSH_ERR_UNSUPPORTED;
  if (fmt == WUSH_FMT_MXFP4)
    return dispatch_kind<32, kMx>(kind, x, rows, d_in, t, t_index, n_t, gscale, nullptr, nullptr, codes, scales,
                                  ydbg, st);
  if (fmt == WUSH_FMT_NVFP4)
    return dispatch_kind<16, kNv>(kind, x, rows, d_in, t, t_index, n_t, gscale, gs_amax, gs_out, codes, scales,
                                  ydbg, st);
  return dispatch_kind<32, kI4>(kind, x, rows, d_in, t, t_index, n_t, gscale, nullptr, nullptr, codes, scales, ydbg,
                                st);
}

}  // namespace wush
