// gemm_sm100.cuh - definitions shared by the tensor-core GEMM of this
// library (gemm_sm100_pair.cuh): tile shape constants, the tile raster, the
// description of a grouped launch (up to kMaxProblems problems D[M, N] =
// A[M, K] . B[N, K]^T per launch, each with its own operands, operand
// major-ness and epilogue), and the bounded pipeline waits.
//
// Every wait is bounded: on timeout the waiting thread records kDevErrTimeout
// in the device error word and raises the CTA's abort flag, so the other roles
// stop, drain their own copies and MMAs (again bounded), free tensor memory
// and return.
#pragma once

#include "ptx_sm100.cuh"

namespace flce {

constexpr int kBM = 128;      // accumulator rows per CTA (TMEM lanes)
constexpr int kBN = 256;      // tile columns (TMEM columns per accumulator)
constexpr int kBK = 64;       // K per stage: one 128-byte swizzle row of BF16
constexpr int kUmmaK = 16;    // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192; // warp 0 scheduler/loads, warp 1 MMA, warps 2..5 epilogue
constexpr int kEpiWarps = 4;
constexpr int kConvWarps = 8; // warps 6..13 of kernels with an FP32 B operand: the converter
constexpr int kTmemCols = 512;
constexpr int kSchedSlots = 4;
constexpr int kMaxProblems = 3;
constexpr uint32_t kMnBlockBytes = 64 * kBK * 2;  // one 64-wide MN block x 64 K rows = 8 KB

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
  int a_keep, b_keep;     // 1: the raster keeps all of this operand in L2 and every tile
                          // row / column re-reads it: load it with evict_last priority
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
// kCluster: acquire at cluster scope (the arrivals publish the peer CTA's
// shared-memory stores).
template <bool kCluster = false>
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, PipeCtl* ctl,
                                           unsigned* err, uint64_t timeout_ns) {
  auto test = [&]() {
    return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (test()) return true;
  const uint64_t t0 = global_timer_ns();
  while (!test()) {
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
// kBF32: B is FP32 in global memory and is rounded to BF16 (nearest even) on
// its way into shared memory by the kernel's converter warps.
template <bool kAMnMajor, bool kBMnMajor, int kEpiKind, bool kBFp32 = false>
struct ProblemCfg {
  static constexpr bool kAMn = kAMnMajor;
  static constexpr bool kBMn = kBMnMajor;
  static constexpr int kEpi = kEpiKind;
  static constexpr bool kBF32 = kBFp32;
  static constexpr bool kValid = true;
};
struct NoProblem {
  static constexpr bool kAMn = false;
  static constexpr bool kBMn = false;
  static constexpr int kEpi = -1;
  static constexpr bool kBF32 = false;
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

}  // namespace flce
