// Tensor-core form of the ITQ3_S activation-side GEMV (mode 1):
//   y[t, o] = sum_blk s[o, blk] * sum_e (c[o, blk, e] - 3.5) * x_rot[t, blk * 256 + e],
// x_rot = H_256 x / 16 per 256-block (ITQ3_S article, section
// "核心技术：FWHT预旋转与TurboQuant的完美融合"; its performance section names
// tensor cores as the way to speed the dequantising matmul up).
//
// The levels c - 3.5 are exact in fp16, so the 3-bit codes become the A operand
// of kind::f16 MMAs with no rounding.  x_rot is fp32; each (token, block) slice is
// scaled by a power of two 2^-e that brings its largest magnitude into
// [2^14, 2^15) and split into two fp16 parts hi + lo (|error| <= 2^-22 of the
// value), which sit side by side as the B operand: MMA column 2t holds token t's
// hi part, column 2t + 1 its lo part.  A block's products are therefore exact and
// only the fp32 accumulation rounds.  The block scale s and 2^e are applied when
// the per-block accumulator is read back:
//   y[t, o] += s[o, blk] * 2^e * (D[o, 2t] + D[o, 2t + 1]).
//
// Work split: one CTA per 128 output rows and 256-block range.  The C CTAs of a
// thread-block cluster share a 128-row tile and split its blocks; their partial
// sums meet in distributed shared memory and are added in rank order, so the
// result does not depend on timing.  Per block, all sixteen warps
//   * decode this row's codes into TMEM as fp16 levels (A operand, M = 128
//     rows = TMEM lanes, two fp16 per 32-bit column; four warps per lane
//     quarter split the 256 codes of a row),
//   * build the hi/lo B operand (K-major, 128-byte swizzle) from x_rot,
// then a seventeenth warp issues the block's 16 MMAs (K = 16 each) and commits
// them, so that no decode warp waits on MMA issue; the next block's decode
// overlaps them (two A buffers, two B stages).  Accumulators rotate over three
// TMEM slots and are read two blocks later, when their MMAs are long done.  An
// eighteenth warp streams code tiles and x_rot rows by TMA into a four-block ring,
// codes and x on separate barriers so that decoding can start before x exists.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace wush {

static __device__ int g_itq3_tc_error = 0;

int read_and_clear_itq3_tc_error(int* word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_itq3_tc_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (*word) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_itq3_tc_error, &zero, sizeof(int));
  }
  return e;
}

namespace {
using namespace sm100;

constexpr int kDecThreads = 512;               // 16 decode warps, four per TMEM lane quarter
constexpr int kThreads = kDecThreads + 64;     // + the MMA warp and the TMA producer warp
constexpr int kRows = 128;                     // output rows per CTA = MMA M (2^7)
constexpr int kStages = 4;                     // TMA ring of blocks
constexpr int kCodeBytes = kRows * 128;        // one block's code tile: 128 rows x 128 bytes (96 used)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACols = 128;               // 256 fp16 levels of a row per block
constexpr uint32_t kDCol0 = 2 * kACols;        // accumulators after the two A buffers
constexpr uint32_t kDCols = 32;
constexpr int kDBufs = 3;                      // accumulators: block b in b % 3, read two blocks later
constexpr int kMinSmem = 120 * 1024;           // > half an SM's shared memory: one CTA per SM
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMaxLocalBlocks = 64;
constexpr int kMinTokens = 3;
constexpr int64_t kDefaultPolls = int64_t(1) << 40;
constexpr uint64_t kDeadlineNs = 4000000000ull;

// NT = MMA N = 2 x token slots (16 for up to 8 tokens, 32 for up to 16).
template <int NT>
struct Cfg {
  static constexpr int kSlots = NT / 2;
  static constexpr int kXBytes = kSlots * 1024;                 // fp32 x_rot of one block, all slots (TMA box)
  static constexpr int kStageBytes = kCodeBytes + kXBytes;
  static constexpr int kBBoxBytes = NT * 128;                   // 64 k x NT rows
  static constexpr int kBStageBytes = 4 * kBBoxBytes;           // 256 k
  static_assert(kBBoxBytes % 1024 == 0, "swizzle atoms are 1024-byte aligned");
  static_assert(kStageBytes % 1024 == 0, "stages keep the alignment");

  static int smem_bytes(int nbl_max) {
    const int b = 1024 + 2 * kBStageBytes + kStages * kStageBytes + kSlots * kRows * 4 +
                  nbl_max * (kRows + kSlots) * 4 + 8 * (3 * kStages + kDBufs + 2) + 16;
    return b < kMinSmem ? kMinSmem : b;
  }
};

__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// D (TMEM) += A (TMEM, M x 16 fp16) * B (shared, N x 16 fp16, K-major)^T
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane <- r (32x32b shape).
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// tcgen05.wait::ld that also names the loaded registers, so that no use of them
// is scheduled before the wait.
template <int N>
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
  } else {
    static_assert(N == 4, "4 or 8 registers");
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]) : : "memory");
  }
}

// Waits until the grid this one depends on programmatically (the rotation kernel)
// has completed and its writes are visible; a no-op without that dependency.
__device__ __forceinline__ void wait_for_prerequisite_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void st_shared_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// fp16x2 levels (c0 - 3.5, c1 - 3.5) of the two 3-bit codes in the low six bits
// of p: 0x4800 | c << 7 is the fp16 value 8 + c, so one multiply places c0 at
// bits 7..9 and c1 at bits 23..25, and subtracting 11.5 is exact.
__device__ __forceinline__ uint32_t levels_pair(uint32_t p) {
  const uint32_t v = ((p * 0x100080u) & 0x03800380u) | 0x48004800u;
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&v), __floats2half2_rn(11.5f, 11.5f));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 32 codes packed 3 bits each in w[0..2] (code i at bit 3i) -> 16 fp16x2 levels.
__device__ __forceinline__ void decode32(const uint32_t* w, uint32_t (&out)[16]) {
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int pos = 6 * m, wi = pos >> 5, sh = pos & 31;
    const uint32_t lo = w[wi], hi = w[wi + 1 < 3 ? wi + 1 : 2];
    out[m] = levels_pair(__funnelshift_r(lo, hi, sh) & 0x3Fu);
  }
}

// 32 codes (3 bits each, code i at bit 3i of w[0..2]) -> 16 fp16x2 levels, for
// the code words of one thread picked out of a 32-byte chunk pair.
__device__ __forceinline__ void decode64(const uint32_t* w, uint32_t (&lo)[16], uint32_t (&hi)[16]) {
  decode32(w, lo);
  decode32(w + 3, hi);
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    itq3_tc_kernel(const __grid_constant__ CUtensorMap tmap_codes, const __grid_constant__ CUtensorMap tmap_x,
                   const __half* __restrict__ scales, int tokens, int d_out, int nb, int nbl_max, int lg_ncl,
                   float* __restrict__ y, int64_t max_polls) {
  using C_ = Cfg<NT>;
  constexpr int kSlots = C_::kSlots;
  // the next call's first kernel may start early; it waits for this one to finish
  // before it touches memory
  allow_dependent_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bst = smem;                                              // two B stages
  uint8_t* ring = bst + 2 * C_::kBStageBytes;                       // TMA ring: code tile, then x_rot rows
  float* red = reinterpret_cast<float*>(ring + kStages * C_::kStageBytes);   // [ranks][kSlots][rows / ranks]
  float* s_tab = red + kSlots * kRows;                              // [nbl_max][128] block scales
  float* inv_tab = s_tab + nbl_max * kRows;                         // [nbl_max][kSlots] 2^e
  uint64_t* codes_full = reinterpret_cast<uint64_t*>(inv_tab + nbl_max * kSlots);
  uint64_t* x_full = codes_full + kStages;
  uint64_t* empty = x_full + kStages;
  uint64_t* mma_done = empty + kStages;
  uint64_t* a_full = mma_done + kDBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a_full + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, g = warp >> 2;                      // lane quarter, quarter of the row's codes
  const int r = quarter * 32 + lane;                                // row within the tile = TMEM lane
  // The cluster (1, 2, 4 or 8 consecutive CTAs) shares one row tile; its rank is
  // blockIdx.x mod the width.  Shifts instead of the width register and divisions
  // save about a quarter of a microsecond at kernel entry.
  const int ncl = 1 << lg_ncl;
  const int q = static_cast<int>(blockIdx.x) & (ncl - 1);
  const int tile = static_cast<int>(blockIdx.x) >> lg_ncl;
  const int grow = tile * kRows + r;
  const int b_lo = (q * nb) >> lg_ncl, nbl = (((q + 1) * nb) >> lg_ncl) - b_lo;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  constexpr int kMmaWarp = kDecThreads / 32, kProducerWarp = kMmaWarp + 1;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&codes_full[i], 1);
      mbar_init(&x_full[i], 1);
      mbar_init(&empty[i], kDecThreads / 32);
    }
    for (int i = 0; i < kDBufs; ++i) mbar_init(&mma_done[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&a_full[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    // The first ring's code tiles need nothing else: request them before the
    // TMEM allocation and the CTA-wide barrier.
    const int first = nbl < kStages ? nbl : kStages;
    for (int b = 0; b < first; ++b) {
      mbar_arrive_expect_tx(&codes_full[b], kCodeBytes);
      tma_load_2d(ring + b * C_::kStageBytes, &tmap_codes, (b_lo + b) * 96, tile * kRows, &codes_full[b]);
    }
    prefetch_tmap(&tmap_x);
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      atomicOr(&g_itq3_tc_error, 1 << kErrTimeoutBarrier);
    }
  };

  if (warp == kProducerWarp) {
    // Block b -> ring stage b % kStages: the 128-row code tile (128-byte rows,
    // 128-byte swizzle; bytes 96.. belong to the next block or are zero fill) and
    // the kSlots x 256 x_rot rows (rows past the last token are zero fill), each
    // with its own barrier.  Thread 0 has requested the first ring's code tiles;
    // x_rot is written by the rotation kernel launched just before this one.
    if (lane == 0) {
      const int first = nbl < kStages ? nbl : kStages;
      wait_for_prerequisite_grid();
      for (int b = 0; b < first; ++b) {
        mbar_arrive_expect_tx(&x_full[b], C_::kXBytes);
        tma_load_2d(ring + b * C_::kStageBytes + kCodeBytes, &tmap_x, (b_lo + b) * 256, 0, &x_full[b]);
      }
      for (int b = first; b < nbl; ++b) {
        const int s = b % kStages;
        if (!mbar_wait_bounded(&empty[s], ((b / kStages) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
          give_up();
          break;
        }
        uint8_t* st = ring + s * C_::kStageBytes;
        mbar_arrive_expect_tx(&codes_full[s], kCodeBytes);
        tma_load_2d(st, &tmap_codes, (b_lo + b) * 96, tile * kRows, &codes_full[s]);
        mbar_arrive_expect_tx(&x_full[s], C_::kXBytes);
        tma_load_2d(st + kCodeBytes, &tmap_x, (b_lo + b) * 256, 0, &x_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // Block b's operands are complete once the decode warps' barrier phase for it
    // has passed: 16 MMAs (K = 16) into accumulator b % 3, then a commit.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kRows, NT);
      for (int b = 0; b < nbl; ++b) {
        const int st = b & 1;
        if (!mbar_wait_bounded(&a_full[st], (b >> 1) & 1, max_polls, kDeadlineNs, abort_flag)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t a0 = tmem + st * kACols;
        const uint32_t d = tmem + kDCol0 + (b % kDBufs) * kDCols;
        const uint64_t b0 = desc_kmajor_sw128(smem_u32(bst + st * C_::kBStageBytes));
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          mma_f16_tmem_a(d, a0 + 8 * kk, b0 + (kk >> 2) * (C_::kBBoxBytes >> 4) + 2 * (kk & 3), idesc,
                         kk ? 1u : 0u);
        tc_commit(&mma_done[b % kDBufs]);
      }
    }
    __syncwarp();
  } else {
    const int slot = warp;                        // token slot whose B rows this warp builds
    constexpr int kQ = kSlots / 4;                // token slots this thread sums
    float acc[kQ];
#pragma unroll
    for (int j = 0; j < kQ; ++j) acc[j] = 0.f;

    if (g == 0) {
      // this row's block scales, loaded together; first used two blocks from now
      for (int b0 = 0; b0 < nbl; b0 += 8) {
        __half hv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          hv[i] = b0 + i < nbl ? scales[static_cast<int64_t>(grow) * nb + b_lo + b0 + i] : __float2half(0.f);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (b0 + i < nbl) s_tab[(b0 + i) * kRows + r] = __half2float(hv[i]);
      }
    }

    // Accumulator of block b: wait for its MMAs and start the TMEM load of this
    // thread's row and quarter of the token slots; add() finishes it.
    uint32_t dv[2 * kQ];
    auto start_drain = [&](int b) {
      if (!mbar_wait_bounded(&mma_done[b % kDBufs], (b / kDBufs) & 1, max_polls, kDeadlineNs, abort_flag))
        give_up();
      tc_fence_after();
      const uint32_t dcol = tmem + lane_base + kDCol0 + (b % kDBufs) * kDCols + g * 2 * kQ;
      if constexpr (kQ == 4) tmem_ld_x8(dcol, *reinterpret_cast<uint32_t(*)[8]>(dv));
      else tmem_ld_x4(dcol, *reinterpret_cast<uint32_t(*)[4]>(dv));
    };
    auto add = [&](int b) {
      const float s = s_tab[b * kRows + r];
#pragma unroll
      for (int j = 0; j < kQ; ++j)
        acc[j] = fmaf(s * inv_tab[b * kSlots + g * kQ + j], __uint_as_float(dv[2 * j]) + __uint_as_float(dv[2 * j + 1]),
                      acc[j]);
    };

    // This thread's 24 code bytes start at byte 24g of its 96-byte row block: in
    // 16-byte chunks c0 = (24g) / 16 and c0 + 1, at word (24g % 16) / 4 of the pair.
    const int c0 = (24 * g) >> 4, wofs = ((24 * g) & 15) >> 2;
    uint32_t w[6];
    auto load_codes = [&](int b) {
      const int s = b % kStages;
      const bool ok = mbar_wait_bounded(&codes_full[s], (b / kStages) & 1, max_polls, kDeadlineNs, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) give_up();
      const uint8_t* row = ring + s * C_::kStageBytes + r * 128;
      const uint4 u0 = *reinterpret_cast<const uint4*>(row + ((c0 ^ (r & 7)) << 4));
      const uint4 u1 = *reinterpret_cast<const uint4*>(row + (((c0 + 1) ^ (r & 7)) << 4));
      const uint32_t W[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int i = 0; i < 6; ++i) w[i] = wofs == 0 ? W[i] : (wofs == 2 ? W[i + 2] : W[i + 4]);
    };

    if (nbl > 0) load_codes(0);
    for (int b = 0; b < nbl; ++b) {
      const int st = b & 1, s = b % kStages;
      // Block b - 2's MMAs, the last readers of A buffer and B stage st, are done
      // once its accumulator is; its TMEM load overlaps the decode below.
      if (b >= 2) start_drain(b - 2);

      // A: this row's codes 64g .. 64g + 63 -> levels in TMEM buffer st, columns 32g ..
      const uint32_t acol = tmem + lane_base + st * kACols + 32 * g;
      {
        uint32_t lv0[16], lv1[16];
        decode64(w, lv0, lv1);
        tmem_st_x16(acol, lv0);
        tmem_st_x16(acol + 16, lv1);
      }

      // B: token slot t -> rows 2t (hi) and 2t + 1 (lo); lane l holds k-group l
      // (elements 8l .. 8l + 7): 128-byte box l / 8, 16-byte chunk l % 8 of the row.
      if (slot < kSlots) {
        const bool ok = mbar_wait_bounded(&x_full[s], (b / kStages) & 1, max_polls, kDeadlineNs, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) give_up();
        const uint8_t* xs = ring + s * C_::kStageBytes + kCodeBytes + slot * 1024 + lane * 32;
        const float4 xa = *reinterpret_cast<const float4*>(xs);
        const float4 xb = *reinterpret_cast<const float4*>(xs + 16);
        const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(xv[i]));
        // non-negative floats order like their bit patterns
        m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
        // m = 2^E * 1.f (normal: x_rot of fp16 inputs is 0 or >= 2^-28 in magnitude);
        // scale by 2^(14 - E), undo with 2^(E - 14).
        const uint32_t e = (__float_as_uint(m) >> 23) & 0xFFu;
        const float sc = m > 0.f ? __uint_as_float((268u - e) << 23) : 1.f;
        const float inv = m > 0.f ? __uint_as_float((e - 14u) << 23) : 0.f;
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 u = make_float2(xv[2 * i] * sc, xv[2 * i + 1] * sc);
          const __half2 h = __float22half2_rn(u);
          const float2 hf = __half22float2(h);
          const __half2 l = __float22half2_rn(make_float2(u.x - hf.x, u.y - hf.y));
          hw[i] = *reinterpret_cast<const uint32_t*>(&h);
          lw[i] = *reinterpret_cast<const uint32_t*>(&l);
        }
        uint8_t* box = bst + st * C_::kBStageBytes + (lane >> 3) * C_::kBBoxBytes;
        const int n0 = 2 * slot, n1 = 2 * slot + 1;
        *reinterpret_cast<uint4*>(box + n0 * 128 + (((lane & 7) ^ (n0 & 7)) * 16)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(box + n1 * 128 + (((lane & 7) ^ (n1 & 7)) * 16)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        if (lane == 0) inv_tab[b * kSlots + slot] = inv;
      }
      // This warp's reads of stage s are done (the TMA engine writes it next) and
      // its B rows are written (the tensor cores read them): one proxy fence for both.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      if (b + 1 < nbl) load_codes(b + 1);
      if (b >= 2) {
        tmem_ld_wait_regs(dv);
        add(b - 2);
      }
      tmem_st_wait();
      tc_fence_before();
      asm volatile("bar.sync 1, %0;" ::"n"(kDecThreads) : "memory");   // decode warps only
      if (tid == 0) mbar_arrive(&a_full[st]);
    }
    for (int b = nbl >= 2 ? nbl - 2 : 0; b < nbl; ++b) {
      start_drain(b);
      tmem_ld_wait_regs(dv);
      add(b);
    }

    // Rank k of the cluster owns rows [k * 128 / C, (k + 1) * 128 / C): this CTA's
    // partial sums go straight into the owner's reduction buffer, slot [q][t][row].
    const int lg_rows = 7 - lg_ncl, rows_per = 1 << lg_rows, owner = r >> lg_rows;
    const uint32_t dst = mapa_shared(smem_u32(red + (q * kSlots) * rows_per + (r & (rows_per - 1))), owner);
#pragma unroll
    for (int j = 0; j < kQ; ++j) st_shared_cluster_f32(dst + ((g * kQ + j) * rows_per) * 4, acc[j]);
  }

  cluster_sync();                                 // every rank's partials have landed
  {
    const int lg_rows = 7 - lg_ncl, rows_per = 1 << lg_rows;
    for (int i = tid; i < kSlots * rows_per; i += kThreads) {
      const int t = i >> lg_rows, rr = i & (rows_per - 1);
      if (t >= tokens) continue;
      float sum = 0.f;
      for (int k = 0; k < ncl; ++k) sum += red[(k * kSlots + t) * rows_per + rr];
      y[static_cast<int64_t>(t) * d_out + tile * kRows + q * rows_per + rr] = sum;
    }
  }

  __syncwarp();
  if (*abort_flag) {                              // MMAs may still be in flight: let them drain
    const uint64_t until = globaltimer_ns() + 200000ull;
    while (globaltimer_ns() < until) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

int num_sms_cached() {
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

template <int NT>
int launch_tc(const uint8_t* codes, const __half* scales, const float* xrot, int t, int d_out, int nb, float* y,
              cudaStream_t st) {
  const int tiles = d_out / kRows, sms = num_sms_cached();
  if (sms <= 0) return WUSH_ERR_CUDA;
  // Widest cluster (<= 8 CTAs, <= one block each) whose grid still fits in one
  // wave of one CTA per SM.
  int ncl = 1;
  while (ncl < 8 && 2 * ncl <= nb && tiles * 2 * ncl <= sms) ncl *= 2;
  const int nbl_max = (nb + ncl - 1) / ncl;
  const int lg_ncl = ncl == 1 ? 0 : ncl == 2 ? 1 : ncl == 4 ? 2 : 3;
  if (nbl_max > kMaxLocalBlocks) return WUSH_ERR_UNSUPPORTED;
  const int smem = Cfg<NT>::smem_bytes(nbl_max);
  if (smem > kMaxSmem) return WUSH_ERR_UNSUPPORTED;
  EncodeFn enc = get_encode();
  if (!enc) return WUSH_ERR_CUDA;
  // codes: [d_out, nb * 96] bytes, boxes of 128 rows x 128 bytes, 128-byte swizzle;
  // x_rot: fp32 [t, nb * 256], boxes of kSlots rows x 256 (rows >= t read as zero)
  CUtensorMap mc, mx;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(nb) * 96, static_cast<cuuint64_t>(d_out)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(nb) * 96};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kRows)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return WUSH_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(nb) * 256, static_cast<cuuint64_t>(t)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(nb) * 256 * 4};
    const cuuint32_t box[2] = {256, static_cast<cuuint32_t>(Cfg<NT>::kSlots)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(xrot), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return WUSH_ERR_CUDA;
  }
  auto kern = itq3_tc_kernel<NT>;
  static std::atomic<uint64_t> attr_done{0};
  if (set_smem_once(kern, kMaxSmem, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * ncl));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ncl);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlaps the rotation kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const int64_t polls = g_wait_limit_override > 0 ? g_wait_limit_override : kDefaultPolls;
  if (cudaLaunchKernelEx(&cfg, kern, mc, mx, scales, t, d_out, nb, nbl_max, lg_ncl, y, polls) != cudaSuccess)
    return WUSH_ERR_CUDA;
  return launch_status();
}

}  // namespace

int itq3_gemv_tc(const uint8_t* codes, const void* scales_fp16, const float* x_rot, int tokens, int d_out, int d_in,
                 float* y, cudaStream_t st) {
  // One or two tokens: the decode, not the multiply, is the work, and the CUDA-core
  // kernel (no TMEM round trip, no cluster reduction) is faster on B200.
  if (tokens < kMinTokens || tokens > 16 || d_out <= 0 || d_out % kRows || d_in <= 0 || d_in % 256)
    return WUSH_ERR_UNSUPPORTED;
  const auto* sc = static_cast<const __half*>(scales_fp16);
  const int nb = d_in / 256;
  if (tokens <= 8) return launch_tc<16>(codes, sc, x_rot, tokens, d_out, nb, y, st);
  return launch_tc<32>(codes, sc, x_rot, tokens, d_out, nb, y, st);
}

}  // namespace wush
