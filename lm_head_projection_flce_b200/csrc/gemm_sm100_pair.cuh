// gemm_sm100_pair.cuh - the grouped persistent GEMM on CTA pairs: a cluster
// of two CTAs on neighbouring SMs computes 256 x 256 tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16).
//
// CTA r of the pair loads A rows [128 r, 128 r + 128) and B rows
// [128 r, 128 r + 128) of the tile into its own shared memory (32 KB per
// 64-deep k-block, 7 stages: 224 KB) and receives D rows [128 r, 128 r + 128) in its
// own tensor memory.  Per SM this moves two thirds of the operand bytes of a
// 128 x 256 single-CTA tile for the same FLOPs.
//
//   leader (rank 0): warp 0 lane 0 takes tiles (static or from a global
//     counter) and broadcasts them to both CTAs through their shared-memory
//     rings, then loads its halves; warp 1 lane 0 issues the pair MMAs and
//     commits to the stage / accumulator barriers of both CTAs;
//   peer (rank 1): warp 0 lane 0 loads its halves onto the leader's stage
//     barrier; its warp 1 only allocates / frees tensor memory;
//   both: warps 2..5 run the epilogue on the CTA's 128 accumulator rows and
//     hand the accumulator back on the leader's barrier.
//
// A problem may take B as FP32 (an FP32 LM head used without a BF16 copy):
// the producer then loads this CTA's FP32 B rows into a staging ring
// (2 stages of 32 KB, beside 5 BF16 stages), and warps 6..13 of both CTAs
// (the converter) round them to BF16 (nearest even, as a cast would) into
// the stage's B slot in the swizzled layout the MMA reads, fence the stores
// for the async proxy and arrive on the leader's stage barrier, which then
// waits for both CTAs' converters besides the A bytes.
// Every wait is bounded (see gemm_sm100.cuh).  No tile load uses multicast:
// each CTA fetches its own halves.
#pragma once

#include <cuda_bf16.h>

#include "gemm_sm100.cuh"

namespace flce {

constexpr int kPairBM = 256;  // rows of a pair tile (128 per CTA)
constexpr uint32_t kPairATileBytes = 128 * kBK * 2;  // this CTA's 128 A rows x 64 K
constexpr uint32_t kPairBTileBytes = 128 * kBK * 2;  // this CTA's 128 of B's 256 rows x 64 K
constexpr uint32_t kPairStageBytes = kPairATileBytes + kPairBTileBytes;  // 32 KB

// Launch shape and shared-memory plan of one kernel instantiation; kConv:
// some problem has an FP32 B operand (converter warps and a staging ring).
template <bool kConv>
struct PairLayout {
  static constexpr int kStages = kConv ? 5 : 7;     // BF16 operand stages (A, B)
  static constexpr int kF32Stages = kConv ? 2 : 0;  // FP32 B staging stages
  static constexpr int kF32Ring = kConv ? kF32Stages : 1;  // (a ring type needs >= 1)
  static constexpr int kBlockThreads = kThreads + (kConv ? 32 * kConvWarps : 0);
  // Arrivals a stage's full barrier takes besides the bytes: the leader's
  // arm, plus one per converter warp of both CTAs.
  static constexpr uint32_t kFullArrivals = kConv ? 1 + 2 * kConvWarps : 1;
  // Readers of the tile ring: leader MMA, both CTAs' epilogue (and
  // converter) warps, the peer's producer.
  static constexpr int kSchedConsumers =
      1 + kEpiWarps + 1 + kEpiWarps + (kConv ? 2 * kConvWarps : 0);
  static constexpr size_t kSmemBytes =
      1024 + static_cast<size_t>(kStages + kF32Stages) * kPairStageBytes + 512;
  // Barrier indices (8 bytes each) after the stages.
  static constexpr int kBarEmpty = kStages;
  static constexpr int kBarF32Full = 2 * kStages;
  static constexpr int kBarF32Empty = 2 * kStages + kF32Stages;
  static constexpr int kBarTmem = 2 * kStages + 2 * kF32Stages;  // full 0,1; empty 2,3; drain 4
  static constexpr int kBarSched = kBarTmem + 5;  // full[kSchedSlots], then empty[kSchedSlots]
  static constexpr int kNumBars = kBarSched + 2 * kSchedSlots;
};
static_assert(PairLayout<true>::kSmemBytes == PairLayout<false>::kSmemBytes,
              "both layouts use 224 KB of stages");

// Position in a ring of kN stages (index and the parity of its barriers).
template <int kN>
struct Ring {
  int i = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++i == kN) {
      i = 0;
      phase ^= 1u;
    }
  }
  __device__ __forceinline__ void skip(int n) {
    const int j = i + n;
    i = j % kN;
    phase ^= static_cast<uint32_t>((j / kN) & 1);
  }
};

template <class C, class L>
__device__ __forceinline__ bool pair_produce_tile(const GemmProblem& pr, const CUtensorMap* ma,
                                                  const CUtensorMap* mb, int mt, int nt,
                                                  uint32_t rank, uint32_t smem_base,
                                                  uint32_t bar_base, uint32_t leader_bar_base,
                                                  Ring<L::kStages>& ring,
                                                  Ring<L::kF32Ring>& fring, PipeCtl* ctl,
                                                  const GemmGroup& g, uint64_t pol_keep,
                                                  uint64_t pol_normal, bool reverse_k) {
  const int am = mt * kPairBM + 128 * static_cast<int>(rank) + pr.a_mn_off;
  const int bm = nt * kBN + 128 * static_cast<int>(rank) + pr.b_mn_off;
  const int num_kb = pr.num_kb;
  const uint64_t pol_a = pr.a_keep ? pol_keep : pol_normal;
  const uint64_t pol_b = pr.b_keep ? pol_keep : pol_normal;
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!wait_phase(bar_base + 8u * (L::kBarEmpty + ring.i), ring.phase ^ 1u, ctl, g.err,
                    g.timeout_ns))
      return false;
    if constexpr (C::kBF32) {
      if (!wait_phase(bar_base + 8u * (L::kBarF32Empty + fring.i), fring.phase ^ 1u, ctl, g.err,
                      g.timeout_ns))
        return false;
    }
    // The leader's full barrier counts both CTAs' bytes; only the leader arms it.
    if (rank == 0)
      mbar_arrive_expect_tx(bar_base + 8u * ring.i,
                            C::kBF32 ? 2 * kPairATileBytes : 2 * kPairStageBytes);
    const uint32_t fb = leader_bar_base + 8u * ring.i;
    const uint32_t sa = smem_base + ring.i * kPairStageBytes;
    const uint32_t sb = sa + kPairATileBytes;
    // Serpentine: odd waves of tiles walk K downwards, so they start on the
    // k-blocks the previous wave read last, which are still in L2.  The MMA
    // side is unchanged: it consumes stages in order and zero-initialises the
    // accumulator on the first one, whichever k-block that holds.
    const int kc = (reverse_k ? num_kb - 1 - kb : kb) * kBK;
    if constexpr (!C::kAMn) {
      tma_load_2d_pair_hint(sa, ma, fb, kc + pr.a_k_off, am, pol_a);
    } else {
#pragma unroll
      for (int j = 0; j < 2; ++j)
        tma_load_2d_pair_hint(sa + j * kMnBlockBytes, ma, fb, am + 64 * j, kc + pr.a_k_off, pol_a);
    }
    if constexpr (C::kBF32) {
      // FP32 B rows into this CTA's staging stage, counted on its own barrier:
      // K-major as two boxes of 128 rows x 32 K, MN-major as four boxes of
      // 32 MN x 64 K rows (128-byte rows, swizzled).
      const uint32_t ffb = bar_base + 8u * (L::kBarF32Full + fring.i);
      const uint32_t sf = smem_base + (L::kStages + fring.i) * kPairStageBytes;
      mbar_arrive_expect_tx(ffb, kPairStageBytes);
      if constexpr (!C::kBMn) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          tma_load_2d_hint(sf + j * kPairBTileBytes, mb, ffb, kc + pr.b_k_off + 32 * j, bm, pol_b);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_2d_hint(sf + j * kMnBlockBytes, mb, ffb, bm + 32 * j, kc + pr.b_k_off, pol_b);
      }
      fring.advance();
    } else {
      if constexpr (!C::kBMn) {
        tma_load_2d_pair_hint(sb, mb, fb, kc + pr.b_k_off, bm, pol_b);
      } else {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          tma_load_2d_pair_hint(sb + j * kMnBlockBytes, mb, fb, bm + 64 * j, kc + pr.b_k_off,
                                pol_b);
      }
      // Nothing to convert in this k-block: the leader stands in for the
      // converter warps' arrivals.
      if constexpr (L::kFullArrivals > 1) {
        if (rank == 0) mbar_arrive_count(bar_base + 8u * ring.i, L::kFullArrivals - 1);
      }
    }
    ring.advance();
  }
  return true;
}

__device__ __forceinline__ uint32_t bf16x2_rne(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Converter: rounds one staged k-block of this CTA's FP32 B rows (at sf) to
// BF16 into the stage's B slot (at sb).  Both sides use the 128-byte swizzle:
// 16-byte chunk q of a 128-byte row r sits at chunk q ^ (r mod 8).  Thread ct
// (0..255) writes 4 of the slot's 1024 chunks; the 8 threads of a quarter warp
// take 8 consecutive rows, so their chunks fall in distinct banks.
template <bool kMn>
__device__ __forceinline__ void convert_b_kblock(uint32_t sf, uint32_t sb, int ct) {
  // K-major: row r of the slot holds 64 K values of B row r; FP32 box j holds K
  // values [32 j, 32 j + 32).  MN-major: K row r of 64-wide MN block jb; FP32
  // box i holds MN values [32 i, 32 i + 32) of 64 K rows.  Thread ct takes row
  // r and the chunks [4 h, 4 h + 4) of it, h = ct / 128.
  const int r = kMn ? (ct & 63) : (ct & 127);
  const uint32_t jb = static_cast<uint32_t>((ct >> 6) & 1);
  const uint32_t sw = static_cast<uint32_t>(r & 7);
  const uint32_t dst_row = sb + (kMn ? jb * kMnBlockBytes : 0u) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
  for (uint32_t c4 = 0; c4 < 4; ++c4) {
    const uint32_t c = c4 + 4u * static_cast<uint32_t>(ct >> 7);
    const uint32_t box = kMn ? 2u * jb + (c >> 2) : (c >> 2);
    const uint32_t src_row =
        sf + box * (kMn ? kMnBlockBytes : kPairBTileBytes) + static_cast<uint32_t>(r) * 128u;
    const uint32_t q0 = 2u * (c & 3u);
    const float4 x = ld_shared_f4(src_row + ((q0 ^ sw) << 4));
    const float4 y = ld_shared_f4(src_row + (((q0 + 1u) ^ sw) << 4));
    uint4 w;
    w.x = bf16x2_rne(x.x, x.y);
    w.y = bf16x2_rne(x.z, x.w);
    w.z = bf16x2_rne(y.x, y.y);
    w.w = bf16x2_rne(y.z, y.w);
    st_shared_u4(dst_row + ((c ^ sw) << 4), w);
  }
}

template <class C, class L>
__device__ __forceinline__ bool pair_mma_tile(int num_kb, uint32_t d_tmem, uint32_t smem_base,
                                              uint32_t bar_base, int& stage, uint32_t& phase,
                                              PipeCtl* ctl, const GemmGroup& g) {
  constexpr uint32_t idesc = mma_idesc_bf16(kPairBM, kBN, C::kAMn, C::kBMn);
  constexpr uint64_t a_hi = desc_hi_sw128(C::kAMn ? kMnBlockBytes : 16u, 1024u);
  constexpr uint64_t b_hi = desc_hi_sw128(C::kBMn ? kMnBlockBytes : 16u, 1024u);
  constexpr uint32_t a_kstep16 = (C::kAMn ? kUmmaK * 128u : kUmmaK * 2u) >> 4;
  constexpr uint32_t b_kstep16 = (C::kBMn ? kUmmaK * 128u : kUmmaK * 2u) >> 4;
  const uint64_t a_desc0 = a_hi | static_cast<uint64_t>((smem_base & 0x3FFFFu) >> 4);
  const uint64_t b_desc0 =
      b_hi | static_cast<uint64_t>(((smem_base + kPairATileBytes) & 0x3FFFFu) >> 4);
  for (int kb = 0; kb < num_kb; ++kb) {
    // With converters, the arrivals publish the peer's stores to its B half.
    if (!wait_phase<(L::kFullArrivals > 1)>(bar_base + 8u * stage, phase, ctl, g.err,
                                             g.timeout_ns))
      return false;
    const uint64_t soff = static_cast<uint64_t>((stage * kPairStageBytes) >> 4);
#pragma unroll
    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
      tc_mma_bf16_pair(d_tmem, a_desc0 + soff + kk * a_kstep16, b_desc0 + soff + kk * b_kstep16,
                       idesc, (kb | kk) != 0 ? 1u : 0u);
    // Frees this stage in both CTAs once these MMAs have read it.
    tc_commit_pair_mc(bar_base + 8u * (L::kBarEmpty + stage), 0x3);
    if (++stage == L::kStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

template <class C0, class C1, class C2>
using PairLayoutOf = PairLayout<C0::kBF32 || C1::kBF32 || C2::kBF32>;

template <class EpiSet, class C0, class C1 = NoProblem, class C2 = NoProblem>
__global__ void __launch_bounds__(PairLayoutOf<C0, C1, C2>::kBlockThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ GemmMaps maps, const GemmGroup g,
                        const EpiSet ep) {
  using L = PairLayoutOf<C0, C1, C2>;
  constexpr bool kConv = L::kFullArrivals > 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + static_cast<size_t>(L::kStages + L::kF32Stages) * kPairStageBytes);
  // bars: stage full / empty, FP32 staging full / empty, tmem full {0,1} / empty {2,3},
  //       drain, sched_full[kSchedSlots], sched_empty[kSchedSlots] (PairLayout's indices)
  int64_t* sched_tile = reinterpret_cast<int64_t*>(bars + L::kNumBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_tile + kSchedSlots);
  PipeCtl* ctl = reinterpret_cast<PipeCtl*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  const uint32_t leader_bar_base = map_shared_to_rank(bar_base, 0);
  const uint32_t peer_bar_base = map_shared_to_rank(bar_base, 1);
  auto tfull_bar = [&](int a) { return bar_base + 8u * (L::kBarTmem + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (L::kBarTmem + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (L::kBarTmem + 4);
  auto sfull_off = [&](int s) { return 8u * (L::kBarSched + s); };
  auto sempty_off = [&](int s) { return 8u * (L::kBarSched + kSchedSlots + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar_base + 8u * s, L::kFullArrivals);
      mbar_init(bar_base + 8u * (L::kBarEmpty + s), 1);
    }
    for (int s = 0; s < L::kF32Stages; ++s) {
      mbar_init(bar_base + 8u * (L::kBarF32Full + s), 1);
      mbar_init(bar_base + 8u * (L::kBarF32Empty + s), kConvWarps);  // this CTA's converter
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);  // one lane per epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    for (int s = 0; s < kSchedSlots; ++s) {
      mbar_init(bar_base + sfull_off(s), 1);
      mbar_init(bar_base + sempty_off(s), L::kSchedConsumers);
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
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after_sync();
  // The set-up above (barriers, tensor-map prefetch, TMEM) touches nothing the
  // previous launch writes, so with a programmatic dependent launch it overlaps
  // that launch's tail; everything below may read its results.  The next launch
  // may be scheduled right away: its CTAs take SMs as ours exit and wait too.
  grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t pair_id = blockIdx.x >> 1;
  const int64_t num_pairs = gridDim.x >> 1;

  // Tile ring: the leader's producer writes each tile index into both CTAs'
  // slots; the slot is free again once the leader's MMA thread, both CTAs'
  // epilogue warps and the peer's producer have read it.
  auto read_slot = [&](int slot, uint32_t sphase, int64_t& t) -> bool {
    if (!wait_phase(bar_base + sfull_off(slot), sphase, ctl, g.err, g.timeout_ns)) return false;
    t = sched_tile[slot];
    return true;
  };
  auto release_slot = [&](int slot) { mbar_arrive_cluster(leader_bar_base + sempty_off(slot)); };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ scheduler (leader) + loads (both)
      Ring<L::kStages> ring;
      Ring<L::kF32Ring> fring;
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      int64_t next_static = pair_id;
      const uint32_t sched_addr = smem_u32(sched_tile);
      const uint32_t peer_sched_addr = map_shared_to_rank(sched_addr, 1);
      // The leader claims one tile ahead, so the counter's round trip overlaps
      // the current tile's loads.
      auto claim = [&]() -> int64_t {
        int64_t c;
        if (g.tile_counter != nullptr)
          c = static_cast<int64_t>(atomicAdd(g.tile_counter, 1u));
        else {
          c = next_static;
          next_static += num_pairs;
        }
        return c >= g.total_tiles ? -1 : c;
      };
      const uint64_t pol_keep = l2_policy_evict_last();
      const uint64_t pol_normal = l2_policy_evict_normal();
      int64_t claimed = rank == 0 ? claim() : -1;
      while (ok) {
        int64_t t;
        if (rank == 0) {
          t = claimed;
          if (!wait_phase(bar_base + sempty_off(slot), sphase ^ 1u, ctl, g.err, g.timeout_ns)) {
            ok = false;
            break;
          }
          sched_tile[slot] = t;
          st_shared_cluster_s64(peer_sched_addr + 8u * slot, t);
          mbar_arrive(bar_base + sfull_off(slot));
          mbar_arrive_cluster(peer_bar_base + sfull_off(slot));
        } else {
          if (!read_slot(slot, sphase, t)) {
            ok = false;
            break;
          }
          release_slot(slot);
        }
        if (++slot == kSchedSlots) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        if (rank == 0) claimed = claim();
        const int p = problem_of(g, t);
        const GemmProblem& pr = g.prob[p];
        int mt, nt;
        pr.raster.coords(t - pr.tile_begin, mt, nt);
        const bool rev = ((t / num_pairs) & 1) != 0;  // a function of the tile index only
        if (p == 0)
          ok = pair_produce_tile<C0, L>(pr, &maps.a[0], &maps.b[0], mt, nt, rank, smem_base,
                                        bar_base, leader_bar_base, ring, fring, ctl, g, pol_keep,
                                        pol_normal, rev);
        else if constexpr (C1::kValid) {
          if (p == 1)
            ok = pair_produce_tile<C1, L>(pr, &maps.a[1], &maps.b[1], mt, nt, rank, smem_base,
                                          bar_base, leader_bar_base, ring, fring, ctl, g,
                                          pol_keep, pol_normal, rev);
          else if constexpr (C2::kValid)
            ok = pair_produce_tile<C2, L>(pr, &maps.a[2], &maps.b[2], mt, nt, rank, smem_base,
                                          bar_base, leader_bar_base, ring, fring, ctl, g,
                                          pol_keep, pol_normal, rev);
        }
      }
      if (!ok) {
        // Copies this thread started signal the leader's barriers; give them
        // time to land before the CTA can exit.
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (leader only)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      while (ok) {
        int64_t t;
        if (!read_slot(slot, sphase, t)) break;
        release_slot(slot);
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
          ok = pair_mma_tile<C0, L>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
        else if constexpr (C1::kValid) {
          if (p == 1)
            ok = pair_mma_tile<C1, L>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
          else if constexpr (C2::kValid)
            ok = pair_mma_tile<C2, L>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
        }
        if (!ok) break;
        tc_commit_pair_mc(tfull_bar(acc), 0x3);  // accumulator ready in both CTAs
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Every MMA issued above has completed once this barrier flips.
      tc_commit_pair_mc(drain_bar, 0x1);
      drain_wait(drain_bar, 0, ok ? g.timeout_ns : 100000000ull);
    }
  } else if (warp < 2 + kEpiWarps) {
    // -------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    int slot = 0;
    uint32_t sphase = 0;
    while (true) {
      int64_t t;
      if (!read_slot(slot, sphase, t)) break;
      __syncwarp();
      if (lane == 0) release_slot(slot);
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
      const int mt128 = 2 * mt + static_cast<int>(rank);  // this CTA's 128-row block
      if (p == 0)
        EpiSet::dispatch(C0::kEpi, ep, taddr, mt128, nt, row);
      else if constexpr (C1::kValid) {
        if (p == 1)
          EpiSet::dispatch(C1::kEpi, ep, taddr, mt128, nt, row);
        else if constexpr (C2::kValid)
          EpiSet::dispatch(C2::kEpi, ep, taddr, mt128, nt, row);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_shared_to_rank(tempty_bar(acc), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  } else if constexpr (kConv) {
    // -------------------------------------------------- converter (both CTAs)
    // Follows the producer through both rings: per k-block of a problem with
    // an FP32 B it waits for the staged rows, rounds them into the stage's B
    // slot and arrives on the staging stage's empty barrier and on the
    // leader's stage barrier; k-blocks of other problems it only counts.
    const int ct = static_cast<int>(threadIdx.x) - 32 * (2 + kEpiWarps);  // 0..255
    Ring<L::kStages> ring;
    Ring<L::kF32Ring> fring;
    int slot = 0;
    uint32_t sphase = 0;
    bool ok = true;
    while (ok) {
      int64_t t;
      if (!read_slot(slot, sphase, t)) break;
      __syncwarp();
      if (lane == 0) release_slot(slot);
      if (++slot == kSchedSlots) {
        slot = 0;
        sphase ^= 1u;
      }
      if (t < 0) break;
      const int p = problem_of(g, t);
      const int num_kb = g.prob[p].num_kb;
      const bool conv = p == 0 ? C0::kBF32 : (p == 1 ? C1::kBF32 : C2::kBF32);
      const bool b_mn = p == 0 ? C0::kBMn : (p == 1 ? C1::kBMn : C2::kBMn);
      if (!conv) {
        ring.skip(num_kb);
        continue;
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!wait_phase(bar_base + 8u * (L::kBarF32Full + fring.i), fring.phase, ctl, g.err,
                        g.timeout_ns)) {
          ok = false;
          break;
        }
        const uint32_t sf = smem_base + (L::kStages + fring.i) * kPairStageBytes;
        const uint32_t sb = smem_base + ring.i * kPairStageBytes + kPairATileBytes;
        if (b_mn)
          convert_b_kblock<true>(sf, sb, ct);
        else
          convert_b_kblock<false>(sf, sb, ct);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar_base + 8u * (L::kBarF32Empty + fring.i));
          mbar_arrive_cluster(leader_bar_base + 8u * ring.i);
        }
        fring.advance();
        ring.advance();
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs into this CTA's tensor memory are done
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace flce
