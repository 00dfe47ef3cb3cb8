// gemm_sm100.cuh - persistent, warp-specialised tcgen05 GEMM with a pluggable
// epilogue.  D[M, N] = A[M, K] . B[N, K]^T, BF16 operands, FP32 accumulator
// in tensor memory.
//
// One CTA per SM (192 threads):
//   warp 0      one lane issues TMA tile loads into a STAGES-deep ring;
//   warp 1      allocates 512 TMEM columns, one lane issues tcgen05.mma;
//   warps 2..5  epilogue: each thread owns one accumulator row (TMEM lane)
//               and runs Epi::tile() on its 256 columns.
// The accumulator is double-buffered in TMEM (2 x 256 columns) so the
// epilogue of tile t overlaps the main loop of tile t+1.  Every wait is
// bounded: on timeout the CTA records FLCE_DEVERR_TIMEOUT, drains its own
// copies and MMAs (again bounded), frees TMEM and returns.
#pragma once

#include "ptx_sm100.cuh"

namespace flce {

constexpr int kBM = 128;      // tile rows (TMEM lanes)
constexpr int kBN = 256;      // tile columns (TMEM columns per accumulator)
constexpr int kBK = 64;       // K per stage: one 128-byte swizzle row of BF16
constexpr int kUmmaK = 16;    // K per tcgen05.mma (kind::f16)
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kTmemCols = 512;
constexpr uint32_t kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBTileBytes = kBN * kBK * 2;  // 32 KB
constexpr uint32_t kStageBytes = kATileBytes + kBTileBytes;
constexpr uint32_t kMnBlockBytes = 64 * kBK * 2;  // one 64-wide MN block x 64 K rows = 8 KB
constexpr size_t kGemmSmemBytes = 1024 + kStages * kStageBytes + 256;

constexpr unsigned kDevErrBadLabel = 1u;
constexpr unsigned kDevErrTimeout = 2u;

// Linear tile index -> (m tile, n tile).  Tiles are taken in groups of
// `group_m` m-tiles; within a group the m index runs fastest, so the CTAs
// working at the same time share a few B tiles (hit in L2) while the group's
// A panel stays resident in L2.
struct TileRaster {
  int m_tiles;
  int n_tiles;
  int group_m;
  __device__ __forceinline__ void coords(int64_t t, int& mt, int& nt) const {
    const int64_t per_group = static_cast<int64_t>(group_m) * n_tiles;
    const int64_t g = t / per_group;
    const int64_t r = t - g * per_group;
    const int m0 = static_cast<int>(g) * group_m;
    const int gm = min(group_m, m_tiles - m0);
    mt = m0 + static_cast<int>(r % gm);
    nt = static_cast<int>(r / gm);
  }
};

struct GemmShape {
  int64_t m, n, k;       // problem sizes (D is m x n, contraction over k)
  int a_mn_off, a_k_off;  // coordinate offsets added to A's (MN, K) tile coordinates
  int b_mn_off, b_k_off;  // coordinate offsets added to B's (MN, K) tile coordinates
  TileRaster raster;
  int64_t tiles;
  unsigned* err;          // device error word
  uint64_t timeout_ns;
};

struct PipeCtl {
  volatile int abort;
};

// Bounded wait: true once the phase completed; false on abort or timeout.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, PipeCtl* ctl,
                                           const GemmShape& g) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (ctl->abort) return false;
    if (global_timer_ns() - t0 > g.timeout_ns) {
      ctl->abort = 1;
      atomicOr(g.err, kDevErrTimeout);
      return false;
    }
  }
  return true;
}

// Wait used while draining after an abort: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

template <class Epi, bool kAMn, bool kBMn>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                   const __grid_constant__ CUtensorMap tm_b, const GemmShape g,
                   const typename Epi::Params ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  // bars[0..S) full, [S..2S) empty, [2S..2S+2) tmem_full, [2S+2..2S+4) tmem_empty, [2S+4] drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  PipeCtl* ctl = reinterpret_cast<PipeCtl*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
  auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * kStages + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * kStages + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * kStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiThreads);
    }
    mbar_init(drain_bar, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  const int num_kb = static_cast<int>((g.k + kBK - 1) / kBK);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage bit masks, for draining
      bool ok = true;
      for (int64_t t = blockIdx.x; t < g.tiles && ok; t += gridDim.x) {
        int mt, nt;
        g.raster.coords(t, mt, nt);
        const int am = mt * kBM + g.a_mn_off;
        const int bm = nt * kBN + g.b_mn_off;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_phase(empty_bar(stage), phase ^ 1u, ctl, g)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, kStageBytes);
          const uint32_t sa = smem_base + stage * kStageBytes;
          const uint32_t sb = sa + kATileBytes;
          const int kc = kb * kBK;
          if (!kAMn) {
            tma_load_2d(sa, &tm_a, fb, kc + g.a_k_off, am);
          } else {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d(sa + j * kMnBlockBytes, &tm_a, fb, am + 64 * j, kc + g.a_k_off);
          }
          if (!kBMn) {
            tma_load_2d(sb, &tm_b, fb, kc + g.b_k_off, bm);
          } else {
#pragma unroll
            for (int j = 0; j < kBN / 64; ++j)
              tma_load_2d(sb + j * kMnBlockBytes, &tm_b, fb, bm + 64 * j, kc + g.b_k_off);
          }
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let every copy this thread started land before the CTA exits.
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) drain_wait(full_bar(s), (issued_parity >> s) & 1u, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = mma_idesc_bf16(kBM, kBN, kAMn, kBMn);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < g.tiles && ok; t += gridDim.x) {
        if (!wait_phase(tempty_bar(acc), acc_phase ^ 1u, ctl, g)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_phase(full_bar(stage), phase, ctl, g)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_base + stage * kStageBytes;
          const uint32_t sb = sa + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t adesc =
                kAMn ? smem_desc_sw128(sa + kk * (kUmmaK * 128), kMnBlockBytes, 1024)
                     : smem_desc_sw128(sa + kk * (kUmmaK * 2), 16, 1024);
            const uint64_t bdesc =
                kBMn ? smem_desc_sw128(sb + kk * (kUmmaK * 128), kMnBlockBytes, 1024)
                     : smem_desc_sw128(sb + kk * (kUmmaK * 2), 16, 1024);
            tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));  // frees the smem stage once these MMAs finish
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));  // accumulator ready for the epilogue
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Every MMA issued above has completed once this barrier flips.
      tc_commit(drain_bar);
      drain_wait(drain_bar, 0, ok ? g.timeout_ns : 100000000ull);
    }
  } else {
    // -------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t t = blockIdx.x; t < g.tiles; t += gridDim.x) {
      int mt, nt;
      g.raster.coords(t, mt, nt);
      if (!wait_phase(tfull_bar(acc), acc_phase, ctl, g)) break;
      tc_fence_after_sync();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      Epi::tile(ep, taddr, mt, nt, row);
      tc_fence_before_sync();
      mbar_arrive(tempty_bar(acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace flce
