// gemm_sm100.cuh - persistent, warp-specialised tcgen05 GEMM over a group of
// up to kMaxProblems problems in one launch, each with its own operands,
// operand major-ness and epilogue:  D[M, N] = A[M, K] . B[N, K]^T, BF16
// operands, FP32 accumulator in tensor memory.
//
// One CTA per SM (192 threads):
//   warp 0      one lane takes tiles (static round robin, or dynamically from
//               a global counter so CTAs that start late or draw long tiles
//               take fewer), broadcasts each tile index to the other roles
//               through a small shared-memory ring, and issues the TMA tile
//               loads into a kStages-deep ring of operand stages;
//   warp 1      allocates 512 TMEM columns, one lane issues tcgen05.mma;
//   warps 2..5  epilogue: each thread owns one accumulator row (TMEM lane)
//               and runs the problem's epilogue on its 256 columns.
// The accumulator is double-buffered in TMEM (2 x 256 columns) so the
// epilogue of tile t overlaps the main loop of tile t+1.  Every wait is
// bounded: on timeout the CTA records kDevErrTimeout, drains its own copies
// and MMAs (again bounded), frees TMEM and returns.
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
constexpr int kEpiWarps = 4;
constexpr int kTmemCols = 512;
constexpr int kSchedSlots = 4;
constexpr int kMaxProblems = 3;
constexpr uint32_t kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBTileBytes = kBN * kBK * 2;  // 32 KB
constexpr uint32_t kStageBytes = kATileBytes + kBTileBytes;
constexpr uint32_t kMnBlockBytes = 64 * kBK * 2;  // one 64-wide MN block x 64 K rows = 8 KB
constexpr size_t kGemmSmemBytes = 1024 + kStages * kStageBytes + 512;

constexpr unsigned kDevErrBadLabel = 1u;
constexpr unsigned kDevErrTimeout = 2u;

// Linear tile index -> (m tile, n tile).  Tiles are taken in groups of `group`
// m-tiles (n_fast == 0) or n-tiles (n_fast == 1); inside a group the grouped
// index runs fastest, so CTAs working at the same time share the other
// operand's tiles in L2 while the group's panels stay resident.
struct TileRaster {
  int m_tiles;
  int n_tiles;
  int group;
  int n_fast;
  __device__ __forceinline__ void coords(int64_t t, int& mt, int& nt) const {
    if (!n_fast) {
      const int64_t per_group = static_cast<int64_t>(group) * n_tiles;
      const int64_t g = t / per_group;
      const int64_t r = t - g * per_group;
      const int m0 = static_cast<int>(g) * group;
      const int gm = min(group, m_tiles - m0);
      mt = m0 + static_cast<int>(r % gm);
      nt = static_cast<int>(r / gm);
    } else {
      const int64_t per_group = static_cast<int64_t>(group) * m_tiles;
      const int64_t g = t / per_group;
      const int64_t r = t - g * per_group;
      const int n0 = static_cast<int>(g) * group;
      const int gn = min(group, n_tiles - n0);
      nt = n0 + static_cast<int>(r % gn);
      mt = static_cast<int>(r / gn);
    }
  }
};

enum EpiKind : int { kEpiForward = 0, kEpiGrad = 1, kEpiStoreRows = 2, kEpiAccumRows = 3 };

struct GemmProblem {
  int64_t m, n, k;        // D is m x n, contraction over k
  int a_mn, b_mn;         // 1: operand stored MN-contiguous (else K-contiguous)
  int a_mn_off, a_k_off;  // offsets added to A's (MN, K) tile coordinates
  int b_mn_off, b_k_off;  // offsets added to B's (MN, K) tile coordinates
  int epi;                // EpiKind
  int num_kb;             // ceil(k / kBK)
  TileRaster raster;
  int64_t tiles;
  int64_t tile_begin;     // first group-wide tile index of this problem
};

struct __align__(64) GemmMaps {
  CUtensorMap a[kMaxProblems];
  CUtensorMap b[kMaxProblems];
};

struct GemmGroup {
  int num_problems;
  GemmProblem prob[kMaxProblems];
  int64_t total_tiles;
  unsigned* tile_counter;  // zero before the launch; nullptr = static round robin
  unsigned* err;           // device error word
  uint64_t timeout_ns;
};

struct PipeCtl {
  volatile int abort;
};

// Bounded wait: true once the phase completed; false on abort or timeout.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, PipeCtl* ctl,
                                           unsigned* err, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (ctl->abort) return false;
    if (global_timer_ns() - t0 > timeout_ns) {
      ctl->abort = 1;
      atomicOr(err, kDevErrTimeout);
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

// Compile-time configuration of one problem slot of a grouped launch.
template <bool kAMnMajor, bool kBMnMajor, int kEpiKind>
struct ProblemCfg {
  static constexpr bool kAMn = kAMnMajor;
  static constexpr bool kBMn = kBMnMajor;
  static constexpr int kEpi = kEpiKind;
  static constexpr bool kValid = true;
};
struct NoProblem {
  static constexpr bool kAMn = false;
  static constexpr bool kBMn = false;
  static constexpr int kEpi = -1;
  static constexpr bool kValid = false;
};

// Upper bits of a 128-byte-swizzle descriptor (everything but the start
// address); the start address field is added per stage / k-step: smem
// addresses are below 256 KB, so the 14-bit field never carries.
__host__ __device__ constexpr uint64_t desc_hi_sw128(uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) |
         (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ int problem_of(const GemmGroup& g, int64_t t) {
  int p = 0;
#pragma unroll
  for (int i = 1; i < kMaxProblems; ++i)
    if (i < g.num_problems && t >= g.prob[i].tile_begin) p = i;
  return p;
}

// Producer: issue the TMA loads of one tile's k-blocks.
template <class C>
__device__ __forceinline__ bool produce_tile(const GemmProblem& pr, const CUtensorMap* ma,
                                             const CUtensorMap* mb, int mt, int nt,
                                             uint32_t smem_base, uint32_t bar_base, int& stage,
                                             uint32_t& phase, uint32_t& issued,
                                             uint32_t& issued_parity, PipeCtl* ctl,
                                             const GemmGroup& g) {
  const int am = mt * kBM + pr.a_mn_off;
  const int bm = nt * kBN + pr.b_mn_off;
  const int num_kb = pr.num_kb;
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!wait_phase(bar_base + 8u * (kStages + stage), phase ^ 1u, ctl, g.err, g.timeout_ns))
      return false;
    const uint32_t fb = bar_base + 8u * stage;
    mbar_arrive_expect_tx(fb, kStageBytes);
    const uint32_t sa = smem_base + stage * kStageBytes;
    const uint32_t sb = sa + kATileBytes;
    const int kc = kb * kBK;
    if constexpr (!C::kAMn) {
      tma_load_2d(sa, ma, fb, kc + pr.a_k_off, am);
    } else {
#pragma unroll
      for (int j = 0; j < kBM / 64; ++j)
        tma_load_2d(sa + j * kMnBlockBytes, ma, fb, am + 64 * j, kc + pr.a_k_off);
    }
    if constexpr (!C::kBMn) {
      tma_load_2d(sb, mb, fb, kc + pr.b_k_off, bm);
    } else {
#pragma unroll
      for (int j = 0; j < kBN / 64; ++j)
        tma_load_2d(sb + j * kMnBlockBytes, mb, fb, bm + 64 * j, kc + pr.b_k_off);
    }
    issued |= 1u << stage;
    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

// MMA issuer: all k-blocks of one tile into the TMEM accumulator d_tmem.
template <class C>
__device__ __forceinline__ bool mma_tile(int num_kb, uint32_t d_tmem, uint32_t smem_base,
                                         uint32_t bar_base, int& stage, uint32_t& phase,
                                         PipeCtl* ctl, const GemmGroup& g) {
  constexpr uint32_t idesc = mma_idesc_bf16(kBM, kBN, C::kAMn, C::kBMn);
  constexpr uint64_t a_hi = desc_hi_sw128(C::kAMn ? kMnBlockBytes : 16u, 1024u);
  constexpr uint64_t b_hi = desc_hi_sw128(C::kBMn ? kMnBlockBytes : 16u, 1024u);
  constexpr uint32_t a_kstep16 = (C::kAMn ? kUmmaK * 128u : kUmmaK * 2u) >> 4;
  constexpr uint32_t b_kstep16 = (C::kBMn ? kUmmaK * 128u : kUmmaK * 2u) >> 4;
  const uint64_t a_desc0 = a_hi | static_cast<uint64_t>((smem_base & 0x3FFFFu) >> 4);
  const uint64_t b_desc0 = b_hi | static_cast<uint64_t>(((smem_base + kATileBytes) & 0x3FFFFu) >> 4);
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!wait_phase(bar_base + 8u * stage, phase, ctl, g.err, g.timeout_ns)) return false;
    const uint64_t soff = static_cast<uint64_t>((stage * kStageBytes) >> 4);
#pragma unroll
    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
      tc_mma_bf16(d_tmem, a_desc0 + soff + kk * a_kstep16, b_desc0 + soff + kk * b_kstep16, idesc,
                  (kb | kk) != 0 ? 1u : 0u);
    tc_commit(bar_base + 8u * (kStages + stage));  // frees the smem stage once these MMAs finish
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

// EpiSet: the epilogues' Params and a static dispatch(kind, params, taddr, mt,
// nt, row) (epilogues.cuh).  C0..C2: compile-time configuration of the
// problem slots (operand major-ness, epilogue kind).
template <class EpiSet, class C0, class C1 = NoProblem, class C2 = NoProblem>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_group_kernel(const __grid_constant__ GemmMaps maps, const GemmGroup g,
                         const EpiSet ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  // bars: [0,S) full, [S,2S) empty, 2S+{0,1} tmem_full, 2S+{2,3} tmem_empty, 2S+4 drain,
  //       2S+5.. sched_full[kSchedSlots], then sched_empty[kSchedSlots]
  int64_t* sched_tile = reinterpret_cast<int64_t*>(bars + 2 * kStages + 5 + 2 * kSchedSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_tile + kSchedSlots);
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
  auto sfull_bar = [&](int s) { return bar_base + 8u * (2 * kStages + 5 + s); };
  auto sempty_bar = [&](int s) { return bar_base + 8u * (2 * kStages + 5 + kSchedSlots + s); };

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
    for (int s = 0; s < kSchedSlots; ++s) {
      mbar_init(sfull_bar(s), 1);
      mbar_init(sempty_bar(s), 1 + kEpiWarps);  // MMA thread + one lane per epilogue warp
    }
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < g.num_problems; ++p) {
      tma_prefetch_desc(&maps.a[p]);
      tma_prefetch_desc(&maps.b[p]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ scheduler + TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      uint32_t sphase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage bit masks, for draining
      bool ok = true;
      int64_t next_static = blockIdx.x;
      while (ok) {
        int64_t t;
        if (g.tile_counter != nullptr)
          t = static_cast<int64_t>(atomicAdd(g.tile_counter, 1u));
        else {
          t = next_static;
          next_static += gridDim.x;
        }
        if (t >= g.total_tiles) t = -1;
        if (!wait_phase(sempty_bar(slot), sphase ^ 1u, ctl, g.err, g.timeout_ns)) {
          ok = false;
          break;
        }
        sched_tile[slot] = t;
        mbar_arrive(sfull_bar(slot));
        if (++slot == kSchedSlots) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        const int p = problem_of(g, t);
        const GemmProblem& pr = g.prob[p];
        int mt, nt;
        pr.raster.coords(t - pr.tile_begin, mt, nt);
        if (p == 0)
          ok = produce_tile<C0>(pr, &maps.a[0], &maps.b[0], mt, nt, smem_base, bar_base, stage,
                                phase, issued, issued_parity, ctl, g);
        else if constexpr (C1::kValid) {
          if (p == 1)
            ok = produce_tile<C1>(pr, &maps.a[1], &maps.b[1], mt, nt, smem_base, bar_base,
                                  stage, phase, issued, issued_parity, ctl, g);
          else if constexpr (C2::kValid)
            ok = produce_tile<C2>(pr, &maps.a[2], &maps.b[2], mt, nt, smem_base, bar_base,
                                  stage, phase, issued, issued_parity, ctl, g);
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
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      while (ok) {
        if (!wait_phase(sfull_bar(slot), sphase, ctl, g.err, g.timeout_ns)) break;
        const int64_t t = sched_tile[slot];
        mbar_arrive(sempty_bar(slot));
        if (++slot == kSchedSlots) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        const int p = problem_of(g, t);
        const int num_kb = g.prob[p].num_kb;
        if (!wait_phase(tempty_bar(acc), acc_phase ^ 1u, ctl, g.err, g.timeout_ns)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        if (p == 0)
          ok = mma_tile<C0>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
        else if constexpr (C1::kValid) {
          if (p == 1)
            ok = mma_tile<C1>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
          else if constexpr (C2::kValid)
            ok = mma_tile<C2>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
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
    int slot = 0;
    uint32_t sphase = 0;
    while (true) {
      if (!wait_phase(sfull_bar(slot), sphase, ctl, g.err, g.timeout_ns)) break;
      const int64_t t = sched_tile[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty_bar(slot));
      if (++slot == kSchedSlots) {
        slot = 0;
        sphase ^= 1u;
      }
      if (t < 0) break;
      const int p = problem_of(g, t);
      const GemmProblem& pr = g.prob[p];
      int mt, nt;
      pr.raster.coords(t - pr.tile_begin, mt, nt);
      if (!wait_phase(tfull_bar(acc), acc_phase, ctl, g.err, g.timeout_ns)) break;
      tc_fence_after_sync();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      if (p == 0)
        EpiSet::dispatch(C0::kEpi, ep, taddr, mt, nt, row);
      else if constexpr (C1::kValid) {
        if (p == 1)
          EpiSet::dispatch(C1::kEpi, ep, taddr, mt, nt, row);
        else if constexpr (C2::kValid)
          EpiSet::dispatch(C2::kEpi, ep, taddr, mt, nt, row);
      }
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
