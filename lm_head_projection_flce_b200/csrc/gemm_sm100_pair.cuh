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
// Every wait is bounded (see gemm_sm100.cuh).  No tile load uses multicast:
// each CTA fetches its own halves.
#pragma once

#include "gemm_sm100.cuh"

namespace flce {

constexpr int kPairBM = 256;  // rows of a pair tile (128 per CTA)
constexpr int kPairStages = 7;
constexpr uint32_t kPairATileBytes = 128 * kBK * 2;  // this CTA's 128 A rows x 64 K
constexpr uint32_t kPairBTileBytes = 128 * kBK * 2;  // this CTA's 128 of B's 256 rows x 64 K
constexpr uint32_t kPairStageBytes = kPairATileBytes + kPairBTileBytes;  // 32 KB
constexpr size_t kPairSmemBytes = 1024 + kPairStages * kPairStageBytes + 512;
constexpr int kPairSchedConsumers = 1 + kEpiWarps + 1 + kEpiWarps;  // see the ring below

template <class C>
__device__ __forceinline__ bool pair_produce_tile(const GemmProblem& pr, const CUtensorMap* ma,
                                                  const CUtensorMap* mb, int mt, int nt,
                                                  uint32_t rank, uint32_t smem_base,
                                                  uint32_t bar_base, uint32_t leader_bar_base,
                                                  int& stage, uint32_t& phase, PipeCtl* ctl,
                                                  const GemmGroup& g, uint64_t pol_keep,
                                                  uint64_t pol_normal, bool reverse_k) {
  const int am = mt * kPairBM + 128 * static_cast<int>(rank) + pr.a_mn_off;
  const int bm = nt * kBN + 128 * static_cast<int>(rank) + pr.b_mn_off;
  const int num_kb = pr.num_kb;
  const uint64_t pol_a = pr.a_keep ? pol_keep : pol_normal;
  const uint64_t pol_b = pr.b_keep ? pol_keep : pol_normal;
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!wait_phase(bar_base + 8u * (kPairStages + stage), phase ^ 1u, ctl, g.err, g.timeout_ns))
      return false;
    // The leader's full barrier counts both CTAs' bytes; only the leader arms it.
    if (rank == 0) mbar_arrive_expect_tx(bar_base + 8u * stage, 2 * kPairStageBytes);
    const uint32_t fb = leader_bar_base + 8u * stage;
    const uint32_t sa = smem_base + stage * kPairStageBytes;
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
    if constexpr (!C::kBMn) {
      tma_load_2d_pair_hint(sb, mb, fb, kc + pr.b_k_off, bm, pol_b);
    } else {
#pragma unroll
      for (int j = 0; j < 2; ++j)
        tma_load_2d_pair_hint(sb + j * kMnBlockBytes, mb, fb, bm + 64 * j, kc + pr.b_k_off, pol_b);
    }
    if (++stage == kPairStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

template <class C>
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
    if (!wait_phase(bar_base + 8u * stage, phase, ctl, g.err, g.timeout_ns)) return false;
    const uint64_t soff = static_cast<uint64_t>((stage * kPairStageBytes) >> 4);
#pragma unroll
    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
      tc_mma_bf16_pair(d_tmem, a_desc0 + soff + kk * a_kstep16, b_desc0 + soff + kk * b_kstep16,
                       idesc, (kb | kk) != 0 ? 1u : 0u);
    // Frees this stage in both CTAs once these MMAs have read it.
    tc_commit_pair_mc(bar_base + 8u * (kPairStages + stage), 0x3);
    if (++stage == kPairStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

template <class EpiSet, class C0, class C1 = NoProblem, class C2 = NoProblem>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ GemmMaps maps, const GemmGroup g,
                        const EpiSet ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  // bars: [0,S) full, [S,2S) empty, 2S+{0,1} tmem_full, 2S+{2,3} tmem_empty, 2S+4 drain,
  //       2S+5.. sched_full[kSchedSlots], then sched_empty[kSchedSlots]
  int64_t* sched_tile = reinterpret_cast<int64_t*>(bars + 2 * kPairStages + 5 + 2 * kSchedSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_tile + kSchedSlots);
  PipeCtl* ctl = reinterpret_cast<PipeCtl*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  const uint32_t leader_bar_base = map_shared_to_rank(bar_base, 0);
  const uint32_t peer_bar_base = map_shared_to_rank(bar_base, 1);
  auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * kPairStages + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * kPairStages + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * kPairStages + 4);
  auto sfull_off = [&](int s) { return 8u * (2 * kPairStages + 5 + s); };
  auto sempty_off = [&](int s) { return 8u * (2 * kPairStages + 5 + kSchedSlots + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(bar_base + 8u * s, 1);
      mbar_init(bar_base + 8u * (kPairStages + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);  // one lane per epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    for (int s = 0; s < kSchedSlots; ++s) {
      mbar_init(bar_base + sfull_off(s), 1);
      mbar_init(bar_base + sempty_off(s), kPairSchedConsumers);
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
      int stage = 0;
      uint32_t phase = 0;
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
          ok = pair_produce_tile<C0>(pr, &maps.a[0], &maps.b[0], mt, nt, rank, smem_base, bar_base,
                                     leader_bar_base, stage, phase, ctl, g, pol_keep,
                                     pol_normal, rev);
        else if constexpr (C1::kValid) {
          if (p == 1)
            ok = pair_produce_tile<C1>(pr, &maps.a[1], &maps.b[1], mt, nt, rank, smem_base,
                                       bar_base, leader_bar_base, stage, phase, ctl, g,
                                       pol_keep, pol_normal, rev);
          else if constexpr (C2::kValid)
            ok = pair_produce_tile<C2>(pr, &maps.a[2], &maps.b[2], mt, nt, rank, smem_base,
                                       bar_base, leader_bar_base, stage, phase, ctl, g,
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
          ok = pair_mma_tile<C0>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
        else if constexpr (C1::kValid) {
          if (p == 1)
            ok = pair_mma_tile<C1>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
          else if constexpr (C2::kValid)
            ok = pair_mma_tile<C2>(num_kb, d_tmem, smem_base, bar_base, stage, phase, ctl, g);
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
  } else {
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
