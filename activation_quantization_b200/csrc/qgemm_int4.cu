// INT4 x INT4 GEMM with per-32-group fp16 scales on tcgen05 tensor cores.
//
// WUSH news article, experiments paragraph: INT4 is the format where WUSH cuts
// the layer loss most.  y[m, n] = sum_g s_a[m, g] s_b[n, g] sum_{k in g} q_a q_b,
// with q in [-7, 7] (two's-complement nibbles, low nibble = lower k) and fp16 s.
// sm_100 tensor cores have no 4-bit integer kind and no per-group integer
// scaling, so each operand element is dequantised to fp16(q * s) -- one rounding,
// relative error <= 2^-11 -- and multiplied with kind::f16 MMAs (fp16 x fp16,
// fp32 accumulation in TMEM).
//
// A persistent CTA per SM walks 128 x 256 output tiles round-robin (M fastest):
//   warps 0-7   dequantisers: per 64-wide k-step, thread t turns row t of the B
//               tile (and, for t < 128, row t of the A tile) from 32 code bytes
//               and two fp16 scales into 128 bytes of fp16 written in the 128-byte
//               swizzled K-major operand layout of a 4-stage shared ring;
//   warp 8      allocates TMEM; one thread issues four M=128 N=256 K=16 MMAs per
//               k-step and commits the stage back to the dequantisers;
//   warps 9-16  epilogue: TMEM -> registers -> 128-byte-swizzled shared chunk ->
//               TMA store of y (fp32), releasing the accumulator once it is read.
// Every wait is bounded; a wait that gives up sets the device error word.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace wush {

static __device__ int g_int4_error = 0;

int read_and_clear_int4_error(int* word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_int4_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (*word) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_int4_error, &zero, sizeof(int));
  }
  return e;
}

namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;          // fp16 elements: 128-byte operand rows
constexpr int kStages = 4;
constexpr int kDqWarps = 8, kDqThreads = kDqWarps * 32;
constexpr int kMmaWarp = kDqWarps;
constexpr int kEpiWarp0 = kDqWarps + 1, kEpiWarps = 8, kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;  // 544
constexpr int kABytes = kBM * kBK * 2;                   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;                   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiChunkBytes = 32 * 32 * 4;
constexpr int kSmemBytes = kStages * kStageBytes + kEpiWarps * kEpiChunkBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 256;
constexpr int64_t kDefaultPolls = int64_t(1) << 40;
constexpr uint64_t kDeadlineNs = 4000000000ull;

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight two's-complement nibbles (element 2i in the low nibble of byte i) times the
// fp16 scale s2 = (s, s): four half2 words holding elements (0,1) (2,3) (4,5) (6,7).
// Each nibble is biased to q + 8, placed in the mantissa of 1024.0 (0x6400 | n =
// 1024 + n exactly), 1032 is subtracted (exact), then one fp16 multiply by s.
__device__ __forceinline__ void dequant8(uint32_t w, __half2 s2, uint32_t (&out)[4]) {
  const uint32_t b = w ^ 0x88888888u;
  const uint32_t kMagic = 0x64006400u;
  const __half2 bias = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1032
  uint32_t h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = ((b >> (4 * i)) & 0x000F000Fu) | kMagic;  // (e_i, e_{i+4})
  __half2 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 x = *reinterpret_cast<const __half2*>(&h[i]);
    v[i] = __hmul2(__hsub2(x, bias), s2);
  }
  const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
  out[0] = prmt(u[0], u[1], 0x5410);   // e0, e1
  out[1] = prmt(u[2], u[3], 0x5410);   // e2, e3
  out[2] = prmt(u[0], u[1], 0x7632);   // e4, e5
  out[3] = prmt(u[2], u[3], 0x7632);   // e6, e7
}

// Raw inputs of one operand row for one 64-wide k-step: 32 code bytes and the two
// group scales.
struct RawRow {
  uint4 c0, c1;
  __half2 sc;
};

__device__ __forceinline__ RawRow load_row(const uint8_t* __restrict__ codes, const __half* __restrict__ scales) {
  RawRow r;
  r.c0 = __ldg(reinterpret_cast<const uint4*>(codes));
  r.c1 = __ldg(reinterpret_cast<const uint4*>(codes + 16));
  r.sc = __ldg(reinterpret_cast<const __half2*>(scales));
  return r;
}

// 128 bytes of fp16 at row ``r`` of a 128-byte-swizzled tile.
__device__ __forceinline__ void dequant_row(const RawRow& raw, uint8_t* tile, int r) {
  const __half2 s0 = __low2half2(raw.sc), s1 = __high2half2(raw.sc);
  const uint32_t w[8] = {raw.c0.x, raw.c0.y, raw.c0.z, raw.c0.w, raw.c1.x, raw.c1.y, raw.c1.z, raw.c1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {           // j: 8 elements = one 16-byte chunk of the fp16 row
    uint32_t o[4];
    dequant8(w[j], j < 4 ? s0 : s1, o);
    *reinterpret_cast<uint4*>(tile + r * 128 + ((j ^ (r & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    qgemm_int4_kernel(const uint8_t* __restrict__ a_codes, const __half* __restrict__ a_scales,
                      const uint8_t* __restrict__ b_codes, const __half* __restrict__ b_scales,
                      const __grid_constant__ CUtensorMap tmap_y, int M, int N, int K, int64_t max_polls) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + kEpiWarps * kEpiChunkBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int mt = M / kBM, n_tiles = mt * (N / kBN), k_steps = K / kBK;
  const int64_t row_bytes = K / 2, n_groups = K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], kDqThreads);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiThreads);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmap_y);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      atomicOr(&g_int4_error, 1 << kErrTimeoutBarrier);
    }
  };

  if (warp < kDqWarps) {
    // The raw codes and scales of the next k-step are loaded before waiting for
    // a free stage, so their L2 latency overlaps the wait and the current step.
    const int t = threadIdx.x;                       // B row t of the tile; A row t for t < 128
    const bool has_a = t < kBM;
    int it = 0;
    const int first = blockIdx.x;
    auto row_ptrs = [&](int tile, const uint8_t*& br, const __half*& bs, const uint8_t*& ar, const __half*& as) {
      const int m0 = (tile % mt) * kBM, n0 = (tile / mt) * kBN;
      br = b_codes + static_cast<int64_t>(n0 + t) * row_bytes;
      bs = b_scales + static_cast<int64_t>(n0 + t) * n_groups;
      ar = a_codes + static_cast<int64_t>(m0 + (t & (kBM - 1))) * row_bytes;
      as = a_scales + static_cast<int64_t>(m0 + (t & (kBM - 1))) * n_groups;
    };
    const uint8_t *br, *ar;
    const __half *bs, *as;
    RawRow nb{}, na{};
    if (first < n_tiles) {
      row_ptrs(first, br, bs, ar, as);
      nb = load_row(br, bs);
      if (has_a) na = load_row(ar, as);
    }
    for (int tile = first; tile < n_tiles; tile += gridDim.x) {
      bool ok = true;
      for (int ks = 0; ks < k_steps; ++ks, ++it) {
        const RawRow cb = nb, ca = na;
        // prefetch the next k-step (of this tile, or the first of the next tile)
        if (ks + 1 < k_steps) {
          nb = load_row(br + (ks + 1) * 32, bs + (ks + 1) * 2);
          if (has_a) na = load_row(ar + (ks + 1) * 32, as + (ks + 1) * 2);
        } else if (tile + static_cast<int>(gridDim.x) < n_tiles) {
          row_ptrs(tile + gridDim.x, br, bs, ar, as);
          nb = load_row(br, bs);
          if (has_a) na = load_row(ar, as);
        }
        const int s = it % kStages;
        ok = mbar_wait_bounded(&empty[s], ((it / kStages) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { give_up(); ok = false; break; }
        uint8_t* sa = smem + s * kStageBytes;
        uint8_t* sb = sa + kABytes;
        dequant_row(cb, sb, t);
        if (has_a) dequant_row(ca, sa, t);
        fence_proxy_async_smem();                    // generic writes -> tensor-core reads
        mbar_arrive(&full[s]);
      }
      if (!ok) break;
    }
  } else if (warp == kMmaWarp) {
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_f16_f32(kBM, kBN);
      bool ok = true;
      int it = 0, tcount = 0;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++tcount) {
        if (!mbar_wait_bounded(acc_empty, (tcount & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait_bounded(&full[s], (it / kStages) & 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_f16(tmem, desc_kmajor_sw128(sa + kk * 32), desc_kmajor_sw128(sb + kk * 32), idesc, (ks | kk) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) give_up();
    }
  } else {
    const int ew = warp - kEpiWarp0, q = warp & 3, half = ew / 4;
    uint8_t* sbuf = epi_smem + ew * kEpiChunkBytes;
    int tcount = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tcount) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int m0 = (tile % mt) * kBM, n0 = (tile / mt) * kBN;
      bool ok = mbar_wait_bounded(acc_full, tcount & 1, max_polls, kDeadlineNs, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { give_up(); break; }
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + half * 128;
#pragma unroll
      for (int p = 0; p < 2; ++p) {              // two rounds of 64 columns keep the registers in budget
        uint32_t r[2][32];
        tmem_ld_32x32b_x32(tbase + 64 * p, r[0]);
        tmem_ld_32x32b_x32(tbase + 64 * p + 32, r[1]);
        tmem_ld_wait();
        if (p == 1) {
          tc_fence_before();
          mbar_arrive(acc_empty);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(sbuf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                make_uint4(r[c][4 * j], r[c][4 * j + 1], r[c][4 * j + 2], r[c][4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmap_y, sbuf, n0 + half * 128 + 64 * p + 32 * c, m0 + q * 32);
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }
  __syncwarp();
  if (*abort_flag) {
    const uint64_t until = globaltimer_ns() + 200000ull;
    while (globaltimer_ns() < until) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Two-pass form.
//
// Dequantising inside the GEMM repeats the conversion for every output tile that
// reads an operand row (N / 256 times for a row of A, M / 128 times for a row of
// B); at the sizes of a transformer layer that conversion, not the tensor cores,
// bounds the fused kernel.  The two-pass form converts each operand element once,
// into a caller workspace (a memory-bound pass), and multiplies the fp16 operands
// with a CTA-pair GEMM.  With no scale factors in TMEM, two 256-column fp32
// accumulators fit, so the epilogue of one tile overlaps the main loop of the next.

// out[g] = the eight fp16(q * s) of INT4 code word g (elements 8g .. 8g + 7 of the
// row-major [rows, K] matrix), one thread per word; scales are fp16 [rows, K / 32].
__global__ void __launch_bounds__(256) int4_dequant_kernel(const uint32_t* __restrict__ codes,
                                                           const __half* __restrict__ scales, int64_t words,
                                                           int words_per_row, uint4* __restrict__ out) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= words) return;
  const int64_t r = g / words_per_row;
  const int c = static_cast<int>(g - r * words_per_row);
  const __half s = scales[r * (words_per_row / 4) + c / 4];
  uint32_t o[4];
  dequant8(__ldg(codes + g), __halves2half2(s, s), o);
  out[g] = make_uint4(o[0], o[1], o[2], o[3]);
}

namespace hp {
constexpr int kRowBytes = 128;                       // 64 fp16 of an operand row per k-tile
constexpr int kKTile = 64;
constexpr int kABytes = 128 * kRowBytes;             // this CTA's 128 rows of A
constexpr int kBBytes = 128 * kRowBytes;             // this CTA's 128-row half of the 256 B rows
constexpr int kStageBytes = kABytes + kBBytes;       // 32 KB, a multiple of 1024
constexpr int kStages = 6;
constexpr int kAccs = 2;
constexpr int kEpiWarps = 8;                         // two per TMEM lane quarter
constexpr int kThreads = 64 + kEpiWarps * 32;        // producer warp, MMA warp, epilogue
constexpr int kEpiChunk = 32 * 32 * 4;               // one warp's 32 x 32 fp32 output chunk
constexpr int kSmemBytes = kStages * kStageBytes + kEpiWarps * kEpiChunk + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kTmemCols = 512;                  // two 256-column accumulators
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
}  // namespace hp

// Tile order of the fp16 pair GEMM: groups of ``group`` 256-row blocks of A, the
// row blocks fastest inside a group, so the tiles in flight at once share one or
// two 256-row blocks of B while the group's rows of A stay in L2 (their loads are
// marked evict-last, y's stores evict-first) for the whole sweep over N: each
// group reads its rows of A once and B once.  The host sizes the group so its rows
// of A fill at most about a third of L2.
__device__ __forceinline__ void pair_tile_coords(int pt, int mt, int nt, int group, int& pm, int& pn) {
  const int g = pt / (group * nt);
  const int rows = min(group, mt - g * group);
  const int w = pt - g * group * nt;
  pm = g * group + w % rows;
  pn = w / rows;
}

__device__ __forceinline__ void mma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// y = A B^T for fp16 A [M, K] and B [N, K] (K-major), fp32 y [M, N]; CTA pairs own
// 256 x 256 output tiles (in pair_tile_coords order), each CTA loading its 128
// rows of A and its 128-row half of B per 64-wide k-tile into a 6-stage ring:
//   warp 0      TMA producer (both CTAs; transaction bytes counted on the leader);
//   warp 1      leader only: four M = 256, N = 256, K = 16 MMAs per k-tile into
//               accumulator (tile & 1), committing stages and tiles to both CTAs;
//   warps 2-9   epilogue (both CTAs): TMEM -> registers, release the accumulator,
//               then 128-byte-swizzled shared chunks -> TMA stores of y.
__global__ void __launch_bounds__(hp::kThreads, 1)
    hgemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_y, int M, int N, int K, int group,
                      int64_t max_polls) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + hp::kStages * hp::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + hp::kEpiWarps * hp::kEpiChunk);
  uint64_t* empty = full + hp::kStages;
  uint64_t* acc_full = empty + hp::kStages;
  uint64_t* acc_empty = acc_full + hp::kAccs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + hp::kAccs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;
  const int mt = M / 256, nt = N / 256, n_ptiles = mt * nt;
  const int k_tiles = K / hp::kKTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < hp::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < hp::kAccs; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * hp::kEpiWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_y);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, hp::kTmemCols);
  tc_fence_before();
  cluster_sync();                       // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      const uint32_t peer = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
      asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
      atomicOr(&g_int4_error, 1 << kErrTimeoutBarrier);
    }
  };

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t keep_a = l2_policy_evict_last();
      int it = 0;
      bool ok = true;
      for (int pt = pair; ok && pt < n_ptiles; pt += n_pairs) {
        int pm, pn;
        pair_tile_coords(pt, mt, nt, group, pm, pn);
        const int arow = pm * 256 + static_cast<int>(rank) * 128;   // this CTA's A rows
        const int brow = pn * 256 + static_cast<int>(rank) * 128;   // this CTA's half of the B rows
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % hp::kStages;
          if (!mbar_wait_bounded(&empty[s], ((it / hp::kStages) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * hp::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * hp::kStageBytes);
          tma_load_2d_pair_hint(sa, &tmap_a, kt * hp::kRowBytes, arow, &full[s], keep_a);
          tma_load_2d_pair(sa + hp::kABytes, &tmap_b, kt * hp::kRowBytes, brow, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (leader && elect_one()) {
      constexpr uint32_t idesc = idesc_f16_f32(256, 256);
      bool ok = true;
      int it = 0, tcount = 0;
      for (int pt = pair; ok && pt < n_ptiles; pt += n_pairs, ++tcount) {
        const int a = tcount & 1;
        if (!mbar_wait_bounded(&acc_empty[a], ((tcount >> 1) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + a * 256;
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % hp::kStages;
          if (!mbar_wait_bounded(&full[s], (it / hp::kStages) & 1, max_polls, kDeadlineNs, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc_kmajor_sw128(smem_u32(smem + s * hp::kStageBytes));
          const uint64_t b0 = desc_kmajor_sw128(smem_u32(smem + s * hp::kStageBytes + hp::kABytes));
#pragma unroll
          for (int kk = 0; kk < hp::kKTile / 16; ++kk)       // 32-byte steps inside the 128-byte rows
            mma_f16_pair(d, a0 + 2 * kk, b0 + 2 * kk, idesc, (kt | kk) ? 1u : 0u);
          tc_commit_pair(&empty[s], 0x3);
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[a], 0x3);
      }
      if (!ok) give_up();
    }
  } else {
    const int ew = warp - 2, q = warp & 3, half = ew / 4;
    uint8_t* buf = epi_smem + ew * hp::kEpiChunk;
    const uint64_t stream_y = l2_policy_evict_first();
    int tcount = 0;
    for (int pt = pair; pt < n_ptiles; pt += n_pairs, ++tcount) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      int pm, pn;
      pair_tile_coords(pt, mt, nt, group, pm, pn);
      const int a = tcount & 1;
      bool ok = mbar_wait_bounded(&acc_full[a], (tcount >> 1) & 1, max_polls, kDeadlineNs, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { give_up(); break; }
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + a * 256 + half * 128;
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tbase + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[a]), 0));
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (lane == 0) bulk_wait_group_read<0>();       // the previous store has read the chunk
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
              make_uint4(r[c][4 * j], r[c][4 * j + 1], r[c][4 * j + 2], r[c][4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d_hint(&tmap_y, buf, pn * 256 + half * 128 + 32 * c, pm * 256 + static_cast<int>(rank) * 128 + q * 32,
                            stream_y);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }
  __syncwarp();
  if (*abort_flag) {
    const uint64_t until = globaltimer_ns() + 200000ull;
    while (globaltimer_ns() < until) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                       // no CTA frees TMEM or exits while its pair still works
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, hp::kTmemCols);
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


// Map over a row-major matrix viewed as bytes: rows x row_bytes, boxes of
// box_rows x 128 bytes with the 128-byte swizzle (the K-major operand layout).
bool make_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 y [rows, cols]: 32 x 32 boxes with the 128-byte swizzle (TMA stores).
bool make_y_map32(CUtensorMap* map, float* y, int64_t rows, int64_t cols) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int launch_dequant(const uint8_t* codes, const void* scales, int64_t rows, int64_t K, __half* out, cudaStream_t st) {
  const int64_t words = rows * (K / 8);
  const int64_t blocks = (words + 255) / 256;
  if (blocks > 0x7FFFFFFF) return WUSH_ERR_UNSUPPORTED;
  int4_dequant_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      reinterpret_cast<const uint32_t*>(codes), static_cast<const __half*>(scales), words, static_cast<int>(K / 8),
      reinterpret_cast<uint4*>(out));
  return launch_status();
}

int launch_hgemm_pair(const __half* a, const __half* b, int64_t M, int64_t N, int64_t K, float* y, cudaStream_t st) {
  CUtensorMap ma, mb, my;
  if (!make_operand_map(&ma, a, M, K * 2, 128) || !make_operand_map(&mb, b, N, K * 2, 128) ||
      !make_y_map32(&my, y, M, N))
    return WUSH_ERR_CUDA;
  static std::atomic<uint64_t> attr_done{0};
  if (set_smem_once(hgemm_pair_kernel, hp::kSmemBytes, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WUSH_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
    return WUSH_ERR_CUDA;
  const int64_t n_ptiles = (M / 256) * (N / 256);
  const int pairs = static_cast<int>(n_ptiles < sms / 2 ? n_ptiles : sms / 2);
  // row blocks of A per group: as many 256-row blocks as fit in a third of L2 (fp16,
  // K wide), at least 8.  (Measured at 8192 x 17408 x 5120: a group holding all of A,
  // 84 MB, did not stay in L2 and read 2.4 GB from DRAM per launch; 16 row blocks,
  // 42 MB, ran fastest.)
  int l2 = 0;
  if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0) return WUSH_ERR_CUDA;
  const int64_t fit = (static_cast<int64_t>(l2) / 3) / (256 * K * 2);
  const int group = static_cast<int>(fit < 8 ? 8 : (fit > M / 256 ? M / 256 : fit));
  const int64_t polls = g_wait_limit_override > 0 ? g_wait_limit_override : kDefaultPolls;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(hp::kThreads);
  cfg.dynamicSmemBytes = hp::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, hgemm_pair_kernel, ma, mb, my, static_cast<int>(M), static_cast<int>(N),
                         static_cast<int>(K), group, polls) != cudaSuccess)
    return WUSH_ERR_CUDA;
  return launch_status();
}
}  // namespace
}  // namespace wush

using namespace wush;

extern "C" int wush_qgemm_int4(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                               const void* b_scales, int64_t M, int64_t N, int64_t K, float* y, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 256 || K % 64) return WUSH_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return WUSH_ERR_UNSUPPORTED;
  if (!a_codes || !a_scales || !b_codes || !b_scales || !y) return WUSH_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(a_scales) & 3u) || (reinterpret_cast<uintptr_t>(b_scales) & 3u))
    return WUSH_ERR_INVALID_ARG;
  EncodeFn enc = get_encode();
  if (!enc) return WUSH_ERR_CUDA;
  CUtensorMap my;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return WUSH_ERR_CUDA;
  static std::atomic<uint64_t> attr_done{0};
  if (set_smem_once(qgemm_int4_kernel, kSmemBytes, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WUSH_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return WUSH_ERR_CUDA;
  const int64_t n_tiles = (M / kBM) * (N / kBN);
  const int grid = static_cast<int>(n_tiles < sms ? n_tiles : sms);
  const int64_t polls = g_wait_limit_override > 0 ? g_wait_limit_override : kDefaultPolls;
  qgemm_int4_kernel<<<grid, kThreads, kSmemBytes, static_cast<cudaStream_t>(stream)>>>(
      a_codes, static_cast<const __half*>(a_scales), b_codes, static_cast<const __half*>(b_scales), my,
      static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), polls);
  return launch_status();
}

extern "C" size_t wush_qgemm_int4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return static_cast<size_t>(M + N) * static_cast<size_t>(K) * 2;
}

extern "C" int wush_qgemm_int4_ws(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                                  const void* b_scales, int64_t M, int64_t N, int64_t K, void* workspace,
                                  size_t workspace_bytes, float* y, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || M % 256 || N % 256 || K % 64) return WUSH_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return WUSH_ERR_UNSUPPORTED;
  if (!a_codes || !a_scales || !b_codes || !b_scales || !workspace || !y) return WUSH_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(workspace) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(a_scales) & 1u) || (reinterpret_cast<uintptr_t>(b_scales) & 1u))
    return WUSH_ERR_INVALID_ARG;
  if (workspace_bytes < wush_qgemm_int4_workspace_bytes(M, N, K)) return WUSH_ERR_BUFFER_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  __half* wa = static_cast<__half*>(workspace);
  __half* wb = wa + M * K;
  // B first: A's fp16 copy, which the GEMM keeps in L2, is then the most recently written
  int status = launch_dequant(b_codes, b_scales, N, K, wb, st);
  if (status == WUSH_OK) status = launch_dequant(a_codes, a_scales, M, K, wa, st);
  if (status == WUSH_OK) status = launch_hgemm_pair(wa, wb, M, N, K, y, st);
  return status;
}
