// Block-scaled FP4 GEMM on tcgen05 tensor cores: y = alpha * dq(A) dq(B)^T.
//
// AI Radio episode "WUSH: Near-Optimal Adaptive Transforms for LLM Quantization",
// "Conclusion": the W4A4 layer runs an FP4 MatMul (up to 5.8x per layer over
// BF16).  A holds the quantised activations [M = tokens, K = d_in], B the
// quantised weights [N = d_out, K]; both are packed E2M1 codes, K contiguous, with
// block scales in the MMA scale-factor tile layout written by
// wush_transform_quant: UE8M0 per 32 (MXFP4, kind::mxf4, block32) or UE4M3 per 16
// (NVFP4, kind::mxf4nvf4, block16).  Products of codes and scales are exact;
// accumulation is fp32 in TMEM.
//
// Two kernels.  When M and N are multiples of 256, persistent CTA pairs
// (qgemm_pair_kernel, described above its configuration below) own 256 x 256
// tiles.  Otherwise a persistent CTA per SM (qgemm_kernel) walks 128 x BN output
// tiles (BN = 256, or 128 when N % 256 != 0) round-robin, with three roles:
//   warp 0     TMA producer: per 256-wide k-tile, one 2D TMA load of the A tile
//              (128 rows x 128 bytes, 128-byte swizzle), one of the B tile, and
//              untiled bulk copies of the matching 512-byte scale atoms, all
//              completing on the stage's "full" mbarrier; the 3-stage (BN 256)
//              or 4-stage (BN 128) ring runs on across tile boundaries;
//   warp 1     allocates TMEM; one elected thread copies the stage's scale atoms
//              into TMEM (tcgen05.cp 32x128b.warpx4) and issues the four K=64
//              block-scaled MMAs, then commits the stage back to the producer;
//   warps 2-9  epilogue: tcgen05.ld of the fp32 accumulator (two warps per TMEM
//              lane quarter, half the columns each), release of the accumulator
//              as soon as it is in registers, then times alpha and stored to y
//              while the next tile's MMAs already run.
// Every mbarrier wait is bounded (poll count, wall time, and a shared abort
// flag); a wait that gives up records a device error word and the CTA drains
// and frees its TMEM before returning.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace wush {

static __device__ int g_error_word = 0;

// Kernel choice for shapes several forms accept (set through
// wush_debug_set_gemm_variant): 0 = CTA pairs where possible, 1 = single-CTA
// 128 x 256 tiles where possible, 2 = single-CTA 128 x 128 tiles.
int g_gemm_variant = 0;

int read_and_clear_error_word(int* word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_error_word, sizeof(int));
  if (e != cudaSuccess) return e;
  if (*word) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int));
  }
  return e;
}

namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 256;             // fp4 elements per k-tile = 128 bytes per row
constexpr int kBKBytes = kBK / 2;
constexpr int kEpiChunkBytes = 32 * 32 * 4;       // one warp's 32 x 32 fp32 output chunk
constexpr int kEpiWarps = 8;                      // two per TMEM lane quarter
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;         // producer warp, MMA warp, epilogue
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = 256;    // TMEM column of the A scale factors
constexpr uint32_t kSfbCol = 288;    // TMEM column of the B scale factors
constexpr int64_t kDefaultPolls = int64_t(1) << 40;
constexpr uint64_t kDeadlineNs = 4000000000ull;  // 4 s of wall time per wait, from its start

template <int BN, bool NV>
struct Cfg {
  static constexpr int kAtomsK = NV ? 4 : 2;             // 512-byte scale atoms per row block per k-tile
  static constexpr int kRowAtomsB = BN / 128;
  static constexpr int kABytes = kBM * kBKBytes;         // 16 KB
  static constexpr int kBBytes = BN * kBKBytes;          // 32 KB or 16 KB
  static constexpr int kSfaBytes = kAtomsK * 512;
  static constexpr int kSfbBytes = kRowAtomsB * kAtomsK * 512;
  static constexpr int kStageBytes = ((kABytes + kBBytes + kSfaBytes + kSfbBytes + 1023) / 1024) * 1024;
  static constexpr int kTxBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kStages = BN == 256 ? 3 : 4;
  static constexpr int kEpiBufs = (BN == 256 && NV) ? 1 : 2;   // staging buffers per epilogue warp
  static constexpr int kEpiBytes = kEpiWarps * kEpiBufs * kEpiChunkBytes;
  static constexpr int kSmemBytes = kStages * kStageBytes + kEpiBytes + 1024 /*align*/ + 256 /*barriers*/;
};

template <int BN, bool NV>
__global__ void __launch_bounds__(kThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
                 const __grid_constant__ CUtensorMap tmap_y, int M, int N, int K, float alpha,
                 const float* __restrict__ alpha_scale, int64_t max_polls, int debug_never) {
  using C = Cfg<BN, NV>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + C::kEpiBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* never = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int n_tiles_n = N / BN;
  const int n_tiles = (M / kBM) * n_tiles_n;
  const int k_tiles = K / kBK;
  const int n_acols = (K / (NV ? 16 : 32) + 3) / 4;     // scale atoms per 128-row block

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiThreads);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_y);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      atomicOr(&g_error_word, 1 << kErrTimeoutBarrier);
    }
  };

  // Tiles are taken round-robin, walking down M inside each BN-wide column of
  // output so that concurrently running CTAs share their B (weight) tiles in L2.
  if (warp == 0) {
    if (elect_one()) {
      int it = 0;  // k-tile counter over all of this CTA's tiles: drives the ring
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int m_blk = tile % (M / kBM), n_blk = tile / (M / kBM);
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % kStages;
          if (!mbar_wait_bounded(&empty[s], ((it / kStages) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          uint8_t* ssfa = sb + C::kBBytes;
          uint8_t* ssfb = ssfa + C::kSfaBytes;
          mbar_arrive_expect_tx(&full[s], C::kTxBytes);
          tma_load_2d(sa, &tmap_a, kt * kBKBytes, m_blk * kBM, &full[s]);
          tma_load_2d(sb, &tmap_b, kt * kBKBytes, n_blk * BN, &full[s]);
          bulk_load(ssfa, sfa + (static_cast<int64_t>(m_blk) * n_acols + kt * C::kAtomsK) * 512, C::kSfaBytes,
                    &full[s]);
#pragma unroll
          for (int h = 0; h < C::kRowAtomsB; ++h)
            bulk_load(ssfb + h * C::kAtomsK * 512,
                      sfb + (static_cast<int64_t>(n_blk * C::kRowAtomsB + h) * n_acols + kt * C::kAtomsK) * 512,
                      C::kAtomsK * 512, &full[s]);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      bool ok = true;
      if (debug_never) {
        // test hook: wait on a barrier nothing arrives on, to exercise the give-up path
        ok = mbar_wait_bounded(never, 0, max_polls, kDeadlineNs, abort_flag);
      }
      const uint32_t tsfa = tmem + kSfaCol;
      const uint32_t tsfb = tmem + kSfbCol;
      int it = 0, tcount = 0;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++tcount) {
        // the epilogue must have drained the accumulator of the previous tile
        if (!mbar_wait_bounded(acc_empty, (tcount & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % kStages;
          if (!mbar_wait_bounded(&full[s], (it / kStages) & 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
          const uint32_t ssfa = sb + C::kBBytes;
          const uint32_t ssfb = ssfa + C::kSfaBytes;
#pragma unroll
          for (int a = 0; a < C::kAtomsK; ++a) {
            tc_cp_32x128b_warpx4(tsfa + 4 * a, desc_sf_atom(ssfa + a * 512));
#pragma unroll
            for (int h = 0; h < C::kRowAtomsB; ++h)
              tc_cp_32x128b_warpx4(tsfb + 4 * (C::kRowAtomsB * a + h), desc_sf_atom(ssfb + (h * C::kAtomsK + a) * 512));
          }
#pragma unroll
          for (int kk = 0; kk < kBK / 64; ++kk) {
            const int atom = NV ? kk : kk / 2;
            const uint32_t sf_id = NV ? 0u : 2u * (kk & 1);
            const uint32_t idesc = idesc_block_scaled_e2m1(kBM, BN, NV ? 0u : 1u, sf_id, sf_id);
            const uint64_t ad = desc_kmajor_sw128(sa + kk * 32);
            const uint64_t bd = desc_kmajor_sw128(sb + kk * 32);
            mma_block_scaled<NV>(tmem, ad, bd, idesc, (kt | kk) ? 1u : 0u, (tsfa + 4 * atom) | (sf_id << 30),
                                 (tsfb + 4 * C::kRowAtomsB * atom) | (sf_id << 30));
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) give_up();
    }
  } else {
    // epilogue: warp w drains TMEM lane quarter w % 4 (rows 32*(w%4) ..), columns
    // [half * BN/2, (half + 1) * BN/2), 32 columns at a time.  Each 32 x 32 chunk
    // goes through a 128-byte-swizzled shared buffer and out with one TMA store,
    // so y is written in whole 128-byte lines.  The accumulator is released as
    // soon as its values are in registers: the next tile's MMAs overlap the stores.
    const int ew = warp - 2;
    const int q = warp & 3;
    const int half = ew / 4;
    // alpha times the device factor (a per-tensor scale computed on the device)
    const float alpha_eff = alpha_scale ? __fmul_rn(__ldg(alpha_scale), alpha) : alpha;
    uint8_t* bufs = epi_smem + ew * C::kEpiBufs * kEpiChunkBytes;
    int buf = 0, tcount = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tcount) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int m_blk = tile % (M / kBM), n_blk = tile / (M / kBM);
      bool ok = mbar_wait_bounded(acc_full, tcount & 1, max_polls, kDeadlineNs, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { give_up(); break; }
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + half * (BN / 2);
      // the whole accumulator slice goes to registers first, so TMEM is handed
      // back to the MMA thread after one round of TMEM loads
      constexpr int kChunks = BN / 64;
      uint32_t r[kChunks][32];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(tbase + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(acc_empty);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        if (lane == 0) bulk_wait_group_read<C::kEpiBufs - 1>();   // this buffer's previous store has read it
        __syncwarp();
        uint8_t* sb = bufs + buf * kEpiChunkBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(sb + lane * 128 + ((j ^ (lane & 7)) * 16)) =
              make_float4(alpha_eff * __uint_as_float(r[c][4 * j]), alpha_eff * __uint_as_float(r[c][4 * j + 1]),
                          alpha_eff * __uint_as_float(r[c][4 * j + 2]), alpha_eff * __uint_as_float(r[c][4 * j + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmap_y, sb, n_blk * BN + half * (BN / 2) + 32 * c, m_blk * kBM + q * 32);
          bulk_commit_group();
        }
        buf = (buf + 1) % C::kEpiBufs;
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }
  __syncwarp();

  if (*abort_flag) {
    // let loads and MMAs already issued by this CTA land before its shared memory
    // and TMEM are released
    const uint64_t until = globaltimer_ns() + 200000ull;
    while (globaltimer_ns() < until) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
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

// ---------------------------------------------------------------------------
// CTA-pair form (tcgen05 cta_group::2) for M % 256 == 0 and N % 256 == 0.
//
// Two CTAs of a cluster compute one 256 x 256 output tile with one MMA stream:
// each CTA TMA-loads its own 128 rows of A, its own 128 rows (half) of B and
// the scale factors its TMEM needs (its rows of SFA, all 256 rows of SFB), all
// counted on the even (leader) CTA's stage barrier; the leader's MMA thread
// copies the scales into both CTAs' TMEM and issues M = 256, N = 256 MMAs whose
// accumulator rows land in the two CTAs' TMEM, and its commits arrive on both
// CTAs' barriers.  Per SM this halves the B bytes fetched from L2 for the same
// FLOPs as the single-CTA 128 x 256 tile.  No load uses cluster multicast.
template <bool NV>
struct Cfg2 {
  static constexpr int kAtomsK = NV ? 4 : 2;
  static constexpr int kABytes = kBM * kBKBytes;                // own 128 rows of A
  static constexpr int kBBytes = kBM * kBKBytes;                // own 128 rows of B
  static constexpr int kSfaBytes = kAtomsK * 512;
  static constexpr int kSfbBytes = 2 * kAtomsK * 512;           // both 128-row halves of the N tile
  static constexpr int kCtaBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kStageBytes = ((kCtaBytes + 1023) / 1024) * 1024;
  // MXFP4 stages are small enough for a sixth if the epilogue stages y in 1 KB
  // chunks (32 rows x 8 fp32); NVFP4's scale tiles leave room for five with 4 KB
  // chunks (32 rows x 32 fp32, 128-byte swizzle).
  static constexpr int kStages = NV ? 5 : 6;
  static constexpr int kTxBytesPair = 2 * kCtaBytes;
  static constexpr int kEpiCols = NV ? 32 : 8;                  // fp32 columns per staged chunk
  static constexpr int kEpiBytes = kEpiWarps * 32 * kEpiCols * 4;
  static constexpr int kSmemBytes = kStages * kStageBytes + kEpiBytes + 1024 + 256;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

template <bool NV>
__global__ void __launch_bounds__(kThreads, 1)
    qgemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                      const __grid_constant__ CUtensorMap tmap_y, int M, int N, int K, float alpha,
                      const float* __restrict__ alpha_scale, int64_t max_polls, int debug_never) {
  using C = Cfg2<NV>;
  constexpr int kSt = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + kSt * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + C::kEpiBytes);
  uint64_t* empty = full + kSt;
  uint64_t* acc_full = empty + kSt;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* never = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;
  const int mt = M / 256, n_ptiles = mt * (N / 256);
  const int k_tiles = K / kBK;
  const int n_acols = (K / (NV ? 16 : 32) + 3) / 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
    prefetch_tmap(&tmap_y);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tc_fence_before();
  cluster_sync();                       // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched after another kernel with programmatic stream serialization, the set-up
  // above overlaps that kernel's tail; no operand is read and no output written
  // before the wait.
  pdl_launch_dependents();
  pdl_wait();

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      const uint32_t peer = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
      asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
      atomicOr(&g_error_word, 1 << kErrTimeoutBarrier);
    }
  };

  if (warp == 0) {
    if (elect_one()) {
      int it = 0;
      for (int pt = pair; pt < n_ptiles; pt += n_pairs) {
        const int pm = pt % mt, pn = pt / mt;
        const int arow = pm * 256 + static_cast<int>(rank) * 128;   // this CTA's A rows
        const int brow = pn * 256 + static_cast<int>(rank) * 128;   // this CTA's half of the B rows
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % kSt;
          if (!mbar_wait_bounded(&empty[s], ((it / kSt) & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) {
            give_up();
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          uint8_t* ssfa = sb + C::kBBytes;
          uint8_t* ssfb = ssfa + C::kSfaBytes;
          if (leader) mbar_arrive_expect_tx(&full[s], C::kTxBytesPair);
          tma_load_2d_pair(sa, &tmap_a, kt * kBKBytes, arow, &full[s]);
          tma_load_2d_pair(sb, &tmap_b, kt * kBKBytes, brow, &full[s]);
          // scale atoms: the maps view the scale buffers as rows of 256 bytes, two per atom
          tma_load_2d_pair(ssfa, &tmap_sfa, 0, ((pm * 2 + static_cast<int>(rank)) * n_acols + kt * C::kAtomsK) * 2,
                           &full[s]);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_2d_pair(ssfb + h * C::kAtomsK * 512, &tmap_sfb, 0,
                             ((pn * 2 + h) * n_acols + kt * C::kAtomsK) * 2, &full[s]);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (leader && elect_one()) {
      bool ok = true;
      if (debug_never) ok = mbar_wait_bounded(never, 0, max_polls, kDeadlineNs, abort_flag);
      const uint32_t tsfa = tmem + kSfaCol;
      const uint32_t tsfb = tmem + kSfbCol;
      int it = 0, tcount = 0;
      for (int pt = pair; ok && pt < n_ptiles; pt += n_pairs, ++tcount) {
        if (!mbar_wait_bounded(acc_empty, (tcount & 1) ^ 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int kt = 0; kt < k_tiles; ++kt, ++it) {
          const int s = it % kSt;
          if (!mbar_wait_bounded(&full[s], (it / kSt) & 1, max_polls, kDeadlineNs, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
          const uint32_t ssfa = sb + C::kBBytes;
          const uint32_t ssfb = ssfa + C::kSfaBytes;
#pragma unroll
          for (int a = 0; a < C::kAtomsK; ++a) {
            tc_cp_32x128b_warpx4_pair(tsfa + 4 * a, desc_sf_atom(ssfa + a * 512));
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tc_cp_32x128b_warpx4_pair(tsfb + 4 * (2 * a + h), desc_sf_atom(ssfb + (h * C::kAtomsK + a) * 512));
          }
#pragma unroll
          for (int kk = 0; kk < kBK / 64; ++kk) {
            const int atom = NV ? kk : kk / 2;
            const uint32_t sf_id = NV ? 0u : 2u * (kk & 1);
            const uint32_t idesc = idesc_block_scaled_e2m1(256, 256, NV ? 0u : 1u, sf_id, sf_id);
            mma_block_scaled_pair<NV>(tmem, desc_kmajor_sw128(sa + kk * 32), desc_kmajor_sw128(sb + kk * 32), idesc,
                                      (kt | kk) ? 1u : 0u, (tsfa + 4 * atom) | (sf_id << 30),
                                      (tsfb + 8 * atom) | (sf_id << 30));
          }
          tc_commit_pair(&empty[s], 0x3);
        }
        if (!ok) break;
        tc_commit_pair(acc_full, 0x3);
      }
      if (!ok) give_up();
    }
  } else {
    const int ew = warp - 2, q = warp & 3, half = ew / 4;
    // alpha times the device factor (a per-tensor scale computed on the device)
    const float alpha_eff = alpha_scale ? __fmul_rn(__ldg(alpha_scale), alpha) : alpha;
    const uint32_t leader_acc_empty = mapa_shared(smem_u32(acc_empty), 0);
    uint8_t* sbuf = epi_smem + ew * 32 * C::kEpiCols * 4;
    int tcount = 0;
    for (int pt = pair; pt < n_ptiles; pt += n_pairs, ++tcount) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int pm = pt % mt, pn = pt / mt;
      bool ok = mbar_wait_bounded(acc_full, tcount & 1, max_polls, kDeadlineNs, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { give_up(); break; }
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + half * 128;
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tbase + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int sc = 0; sc < 32 / C::kEpiCols; ++sc) {
          if (lane == 0) bulk_wait_group_read<0>();   // the previous store has read the chunk
          __syncwarp();
          if constexpr (C::kEpiCols == 32) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4*>(sbuf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_float4(alpha_eff * __uint_as_float(r[c][4 * j]), alpha_eff * __uint_as_float(r[c][4 * j + 1]),
                              alpha_eff * __uint_as_float(r[c][4 * j + 2]), alpha_eff * __uint_as_float(r[c][4 * j + 3]));
          } else {
            // 32-byte rows, one per lane: the warp writes one contiguous kilobyte
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int e = sc * 8 + 4 * j;
              *reinterpret_cast<float4*>(sbuf + lane * 32 + j * 16) =
                  make_float4(alpha_eff * __uint_as_float(r[c][e]), alpha_eff * __uint_as_float(r[c][e + 1]),
                              alpha_eff * __uint_as_float(r[c][e + 2]), alpha_eff * __uint_as_float(r[c][e + 3]));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmap_y, sbuf, pn * 256 + half * 128 + 32 * c + sc * C::kEpiCols,
                         pm * 256 + static_cast<int>(rank) * 128 + q * 32);
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
  cluster_sync();                       // no CTA frees TMEM or exits while its pair still works
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
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

// 2D map over a [rows, row_bytes] uint8 matrix, box = box_rows x 128 bytes, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKBytes), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over fp32 y [rows, cols] for TMA stores: boxes of 32 rows x box_cols; 32
// columns (128-byte rows) use the 128-byte swizzle, 8 columns (32-byte rows) none.
bool make_y_map(CUtensorMap* map, float* y, int64_t rows, int64_t cols, int box_cols) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over a scale buffer viewed as rows of 256 bytes (two rows per 512-byte atom).
bool make_sf_map(CUtensorMap* map, const void* base, int64_t bytes, int box_rows) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {256, static_cast<cuuint64_t>(bytes / 256)};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool NV>
int launch_pair(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, int64_t M, int64_t N,
                int64_t K, float alpha, const float* alpha_scale, float* y, cudaStream_t st) {
  using C = Cfg2<NV>;
  const int64_t n_acols = (K / (NV ? 16 : 32) + 3) / 4;
  CUtensorMap ma, mb, msa, msb, my;
  if (!make_map(&ma, a, M, K / 2, kBM) || !make_map(&mb, b, N, K / 2, kBM) ||
      !make_y_map(&my, y, M, N, C::kEpiCols) ||
      !make_sf_map(&msa, sfa, (M / 128) * n_acols * 512, 2 * C::kAtomsK) ||
      !make_sf_map(&msb, sfb, (N / 128) * n_acols * 512, 2 * C::kAtomsK))
    return WUSH_ERR_CUDA;
  auto kern = qgemm_pair_kernel<NV>;
  static std::atomic<uint64_t> attr_done{0};
  if (set_smem_once(kern, C::kSmemBytes, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  const int n_ptiles = static_cast<int>((M / 256) * (N / 256));
  const int sms = num_sms();
  if (sms < 2) return WUSH_ERR_CUDA;
  const int pairs = n_ptiles < sms / 2 ? n_ptiles : sms / 2;
  const int64_t polls = g_wait_limit_override > 0 ? g_wait_limit_override : kDefaultPolls;
  const int debug_never = g_wait_limit_override > 0 ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, ma, mb, msa, msb, my, static_cast<int>(M), static_cast<int>(N),
                         static_cast<int>(K), alpha, alpha_scale, polls, debug_never) != cudaSuccess)
    return WUSH_ERR_CUDA;
  return launch_status();
}

template <int BN, bool NV>
int launch(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, int64_t M, int64_t N,
           int64_t K, float alpha, const float* alpha_scale, float* y, cudaStream_t st) {
  using C = Cfg<BN, NV>;
  CUtensorMap ma, mb, my;
  if (!make_map(&ma, a, M, K / 2, kBM) || !make_map(&mb, b, N, K / 2, BN) || !make_y_map(&my, y, M, N, 32))
    return WUSH_ERR_CUDA;
  auto kern = qgemm_kernel<BN, NV>;
  static std::atomic<uint64_t> attr_done{0};
  if (set_smem_once(kern, C::kSmemBytes, attr_done) != WUSH_OK) return WUSH_ERR_CUDA;
  const int64_t polls = g_wait_limit_override > 0 ? g_wait_limit_override : kDefaultPolls;
  const int debug_never = g_wait_limit_override > 0 ? 1 : 0;
  const int n_tiles = static_cast<int>((M / kBM) * (N / BN));
  const int sms = num_sms();
  if (sms <= 0) return WUSH_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>(n_tiles < sms ? n_tiles : sms));
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(ma, mb, sfa, sfb, my, static_cast<int>(M), static_cast<int>(N),
                                              static_cast<int>(K), alpha, alpha_scale, polls, debug_never);
  return launch_status();
}

}  // namespace
}  // namespace wush

using namespace wush;

namespace {

int qgemm_impl(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes, const void* b_scales, int64_t M,
               int64_t N, int64_t K, int fmt, float alpha, const float* alpha_scale, float* y, void* stream) {
  if (fmt != WUSH_FMT_MXFP4 && fmt != WUSH_FMT_NVFP4) return WUSH_ERR_UNSUPPORTED;
  if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 256) return WUSH_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30) || N / 128 > 65535 * 128)
    return WUSH_ERR_UNSUPPORTED;
  if (!a_codes || !a_scales || !b_codes || !b_scales || !y) return WUSH_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) || !aligned16(y))
    return WUSH_ERR_INVALID_ARG;
  if (M / 128 > 65535) return WUSH_ERR_UNSUPPORTED;
  const auto* sa = static_cast<const uint8_t*>(a_scales);
  const auto* sb = static_cast<const uint8_t*>(b_scales);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool nv = fmt == WUSH_FMT_NVFP4;
  const float* as = alpha_scale;
  if (M % 256 == 0 && N % 256 == 0 && g_gemm_variant == 0) {
    return nv ? launch_pair<true>(a_codes, sa, b_codes, sb, M, N, K, alpha, as, y, st)
              : launch_pair<false>(a_codes, sa, b_codes, sb, M, N, K, alpha, as, y, st);
  }
  if (N % 256 == 0 && g_gemm_variant != 2) {
    return nv ? launch<256, true>(a_codes, sa, b_codes, sb, M, N, K, alpha, as, y, st)
              : launch<256, false>(a_codes, sa, b_codes, sb, M, N, K, alpha, as, y, st);
  }
  return nv ? launch<128, true>(a_codes, sa, b_codes, sb, M, N, K, alpha, as, y, st)
            : launch<128, false>(a_codes, sa, b_codes, sb, M, N, K, alpha, as, y, st);
}

}  // namespace

extern "C" int wush_qgemm(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                          const void* b_scales, int64_t M, int64_t N, int64_t K, int fmt, float alpha, float* y,
                          void* stream) {
  return qgemm_impl(a_codes, a_scales, b_codes, b_scales, M, N, K, fmt, alpha, nullptr, y, stream);
}

extern "C" int wush_qgemm_nvfp4_dynamic(const uint8_t* a_codes, const void* a_scales, const uint8_t* b_codes,
                                        const void* b_scales, int64_t M, int64_t N, int64_t K,
                                        const float* a_global_scale, float b_global_scale, float* y, void* stream) {
  if (!a_global_scale || (reinterpret_cast<uintptr_t>(a_global_scale) & 3u)) return WUSH_ERR_INVALID_ARG;
  return qgemm_impl(a_codes, a_scales, b_codes, b_scales, M, N, K, WUSH_FMT_NVFP4, b_global_scale, a_global_scale,
                    y, stream);
}
