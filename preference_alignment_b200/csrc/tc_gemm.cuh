// Persistent, warp-specialised bf16 GEMMs on the 5th-generation tensor cores with a
// pluggable per-row epilogue: k_tc_gemm (one CTA per tile, tcgen05.mma cta_group::1)
// and k_tc_gemm_pair (two CTAs of a cluster per tile, cta_group::2; the default).
//
//   D[M x N] = A[M x K] . B[N x K]^T     (fp32 accumulation in tensor memory)
//
// A and B are fed from global memory by TMA into a STAGES-deep ring of
// 128-byte-swizzled shared-memory tiles. Each operand can be K-major (rows of K
// contiguous) or MN-major (rows of M or N contiguous, i.e. the transposed
// storage); the shared-memory descriptor and the TMA boxes follow.
//
// Roles of the single-CTA kernel (192 threads, one CTA per SM, persistent over a
// static tile schedule; the pair kernel below splits them across the pair):
//   warp 0     one thread issues the TMA loads,
//   warp 1     allocates 512 TMEM columns; one thread issues the MMAs,
//   warps 2-5  epilogue: each thread owns one accumulator row (TMEM lane) and
//              reads its 256 fp32 columns in 8 chunks of 32 (tcgen05.ld).
// The accumulator is double-buffered (2 x 256 columns) so the epilogue of tile
// i overlaps the main loop of tile i+1.
#pragma once

#include "ptx_sm100.cuh"
#include "tile_config.h"

namespace dpo {

constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KiB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kGemmThreads = 192;
constexpr int kTmemCols = 512;
// Per epilogue warp: two 32 x 32 bf16 staging buffers for TMA stores.
constexpr int kEpiWarpBytes = 2 * 32 * 32 * 2;
constexpr int kEpiSmemBytes = 4 * kEpiWarpBytes;      // 16 KiB
constexpr int kGemmSmemBytes =
    kStages * kStageBytes + kEpiSmemBytes + 1024 /*align*/ + 256 /*barriers*/;

// What an epilogue thread may use besides its accumulator row: the store tensor
// map and its warp's shared-memory staging buffers.
struct EpiCtx {
  const CUtensorMap* map;
  uint32_t stage;     // shared address of this warp's kEpiWarpBytes
  int lane;
};

// Tile schedule: linear tile index -> (m tile, n tile).
//   order 0: m fastest (all M tiles of one N tile run together: B tile shared via L2)
//   order 1: n fastest (all N tiles of one M tile run together: A tile shared via L2)
//   order 2: grouped along M: `group` consecutive M tiles are swept across every N
//            tile (N outer, M inner) before the next group starts, so the group's
//            A rows stay in L2 while B streams past them once per group
//   order 3: grouped along N, the same with the roles of M and N exchanged
struct GemmGeom {
  int m_tiles, n_tiles, k_blocks;
  int order;
  int group;
  // Split-K: the K blocks are cut into k_parts parts of kb_part blocks (the last may be
  // shorter, none empty); a work unit is (part, m tile, n tile), parts outermost, and
  // the epilogue learns its part. k_parts = 1: one unit per output tile.
  int k_parts, kb_part;
  // Tile claim counter of the CTA-pair kernel (zeroed before the launch), or nullptr
  // for the static schedule (pair p takes tiles p, p + n_pairs, ...). With the counter
  // each pair claims its next tile in raster order when it starts loading it, so the
  // tiles in flight stay one contiguous window of the raster even when pairs run at
  // different speeds, and share their operand tiles in L2.
  int* counter;
};

__device__ __forceinline__ void tile_coords(const GemmGeom& g, int tile, int& mt, int& nt) {
  if (g.order == 0) {
    mt = tile % g.m_tiles;
    nt = tile / g.m_tiles;
  } else if (g.order == 1) {
    mt = tile / g.n_tiles;
    nt = tile % g.n_tiles;
  } else if (g.order == 2) {
    const int per_group = g.group * g.n_tiles;
    const int grp = tile / per_group;
    const int first_m = grp * g.group;
    const int rem = g.m_tiles - first_m;
    const int gm = rem < g.group ? rem : g.group;
    const int local = tile - grp * per_group;
    nt = local / gm;
    mt = first_m + local % gm;
  } else {
    const int per_group = g.group * g.m_tiles;
    const int grp = tile / per_group;
    const int first_n = grp * g.group;
    const int rem = g.n_tiles - first_n;
    const int gn = rem < g.group ? rem : g.group;
    const int local = tile - grp * per_group;
    mt = local / gn;
    nt = first_n + local % gn;
  }
}

// Work unit -> K part ks, tile (mt, nt) and the unit's K blocks [kb0, kb1).
__device__ __forceinline__ void unit_coords(const GemmGeom& g, int unit, int& ks, int& mt, int& nt,
                                            int& kb0, int& kb1) {
  const int per_part = g.m_tiles * g.n_tiles;
  ks = unit / per_part;
  tile_coords(g, unit - ks * per_part, mt, nt);
  kb0 = ks * g.kb_part;
  kb1 = min(g.k_blocks, kb0 + g.kb_part);
}

// Epilogue interface (one object per epilogue thread, per unit; every thread of the
// warp calls each method, in step):
//   __device__ void begin(const Params&, int m_row, int nt, int ks, const EpiCtx&);
//       m_row: row of D; nt: column tile; ks: K part of the unit (0 without split-K)
//   __device__ void chunk(const Params&, int c, const uint32_t (&v)[32]);   // columns c*32..+31
//   __device__ void end(const Params&);
template <bool A_MN, bool B_MN, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmC, GemmGeom g, typename Epi::Params ep,
              DevCtl ctl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                                  // kStages x 16 KiB
  uint8_t* sB = smem + kStages * kABytes;              // kStages x 32 KiB
  uint8_t* sE = smem + kStages * kStageBytes;          // epilogue staging, 16 KiB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + kEpiSmemBytes);
  // bars[0..S)   full      (TMA -> MMA)
  // bars[S..2S)  empty     (MMA -> TMA)
  // bars[2S..2S+2) acc_full  (MMA -> epilogue)
  // bars[2S+2..2S+4) acc_empty (epilogue -> MMA)
  // bars[2S+4]   drain     (MMA teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + kStages);
  const uint32_t accf0 = smem_u32(bars + 2 * kStages);
  const uint32_t acce0 = smem_u32(bars + 2 * kStages + 2);
  const uint32_t drain = smem_u32(bars + 2 * kStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_tiles_total = g.m_tiles * g.n_tiles * g.k_parts;   // work units
  // Producer bookkeeping kept for the teardown: which stages have a load issued
  // and the parity of the `full` phase that load completes.
  uint32_t issued_mask = 0, issued_par = 0;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
      int ks, mt, nt, kb0, kb1;
      unit_coords(g, tile, ks, mt, nt, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, ctl, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t fb = full0 + 8 * stage;
        mbar_arrive_expect_tx(fb, kStageBytes);
        const uint32_t a_dst = smem_u32(sA + stage * kABytes);
        const uint32_t b_dst = smem_u32(sB + stage * kBBytes);
        if (!A_MN) {
          tma_load_2d(a_dst, &tmA, fb, kb * kBK, mt * kBM);
        } else {
#pragma unroll
          for (int j = 0; j < kBM / 64; ++j)
            tma_load_2d(a_dst + j * 8192, &tmA, fb, mt * kBM + j * 64, kb * kBK);
        }
        if (!B_MN) {
          // two 128-row boxes: the same tensor map serves the CTA-pair kernel
          tma_load_2d(b_dst, &tmB, fb, kb * kBK, nt * kBN);
          tma_load_2d(b_dst + 128 * 128, &tmB, fb, kb * kBK, nt * kBN + 128);
        } else {
#pragma unroll
          for (int j = 0; j < kBN / 64; ++j)
            tma_load_2d(b_dst + j * 8192, &tmB, fb, nt * kBN + j * 64, kb * kBK);
        }
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      record_status(ctl, kStatusTimeout);
      *abort_flag = 1;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, A_MN, B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(acce0 + 8 * acc, acc_phase ^ 1, ctl, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * kBN;
      int ks, mt, nt, kb0, kb1;
      unit_coords(g, tile, ks, mt, nt, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full0 + 8 * stage, phase, ctl, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * kABytes);
        const uint32_t b0 = smem_u32(sB + stage * kBBytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          // K-major: the 16-wide K slice sits 32 bytes further along the swizzled row.
          // MN-major: it is the next 16 rows of K, 16 * 128 bytes further.
          const uint64_t ad = A_MN ? sw128_desc(a0 + k * 2048, 8192, 1024)
                                   : sw128_desc(a0 + k * 32, 16, 1024);
          const uint64_t bd = B_MN ? sw128_desc(b0 + k * 2048, 8192, 1024)
                                   : sw128_desc(b0 + k * 32, 16, 1024);
          tc_mma_f16(d_tmem, ad, bd, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
        }
        tc_commit(empty0 + 8 * stage);   // frees this stage once its MMAs are done
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      tc_commit(accf0 + 8 * acc);        // accumulator ready for the epilogue
    }
    if (!ok) {
      record_status(ctl, kStatusTimeout);
      *abort_flag = 1;
    }
    // Drain: wait (bounded) until every MMA issued by this thread has completed,
    // so TMEM is not freed under an MMA in flight.
    tc_commit(drain);
    DevCtl c2 = ctl;
    volatile int never = 0;
    if (!mbar_wait(drain, 0, c2, &never)) record_status(ctl, kStatusTimeout);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int lg = warp & 3;                 // TMEM lane group this warp may access
    const int row = lg * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(lg * 32) << 16);
    const EpiCtx ectx{&tmC, smem_u32(sE + (warp - 2) * kEpiWarpBytes), lane};
    int local = 0;
    for (int tile = blockIdx.x; tile < n_tiles_total; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(accf0 + 8 * acc, acc_phase, ctl, abort_flag)) {
        record_status(ctl, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int ks, mt, nt, kb0, kb1;
      unit_coords(g, tile, ks, mt, nt, kb0, kb1);
      Epi epi;
      epi.begin(ep, mt * kBM + row, nt, ks, ectx);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_addr + acc * kBN + c * 32, v);
        tmem_wait_ld();
        epi.chunk(ep, c, v);
      }
      tc_fence_before();
      mbar_arrive(acce0 + 8 * acc);
      epi.end(ep);
    }
  }

  // Bulk stores an epilogue issued must finish before the CTA (and its shared
  // memory) goes away; warps that issued none return at once. An epilogue whose stores
  // go to another process's memory (Epi::kSystemFence) fences them at system scope.
  if (warp >= 2 && lane == 0) bulk_wait_group<0>();
  if constexpr (Epi::kSystemFence) {
    if (warp >= 2) __threadfence_system();
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // After an abort, loads may still be in flight into shared memory: wait
    // (bounded) for the phase each stage's last load completes before the CTA
    // exits. A phase that already completed returns at once.
    volatile int never = 0;
    DevCtl c2 = ctl;
    c2.budget_ns = ctl.budget_ns / 4 + 1000000ull;
    for (int s = 0; s < kStages; ++s)
      if (issued_mask & (1u << s))
        (void)mbar_wait(full0 + 8 * s, (issued_par >> s) & 1u, c2, &never);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}


// =====================================================================================
// Pair variant: two CTAs of a cluster compute a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256 across the pair). Each CTA loads its own 128
// rows of A and its own 128 rows (N half) of B, so a CTA moves 32 KiB per K step
// instead of 48 KiB; the freed shared memory buys a 6-deep pipeline.
//   leader (cluster rank 0): owns the `full` and `acc_empty` barriers and issues
//     the MMAs; its commits are multicast to both CTAs' `empty` / `acc_full`.
//   both CTAs: TMA producer, epilogue over their own 128 TMEM lanes (rows
//     rank * 128 ... + 127 of the 256-row tile), arriving on the leader's
//     `acc_empty` through its shared::cluster address.
// No TMA load uses cluster multicast: each CTA reads only its own operand rows.
// =====================================================================================
constexpr int kPairM = 256;                        // rows of D per CTA pair
constexpr int kPABytes = 128 * kBK * 2;            // 16 KiB: this CTA's 128 rows of A
constexpr int kPBBytes = (kBN / 2) * kBK * 2;      // 16 KiB: this CTA's half of B
constexpr int kPStageBytes = kPABytes + kPBBytes;
// Pipeline depth: 6 stages of 32 KiB for every epilogue (an epilogue that stores
// through TMA, Epi::kStaging, adds 16 KiB of staging buffers). A 7th stage fits the
// epilogues without staging and made the serialised GEMMs ~1 % faster under ncu, but
// inside the power-capped step (same box, alternating runs at the Llama-3.1-8B head)
// 6 stages were 0.2-2.3 % faster.
template <class Epi>
constexpr int pair_stages() { return 6; }
// Schedule ring of the dynamic tile schedule: slots of claimed tile indices, written
// by the leader's producer into both CTAs and read by every role.
constexpr int kSchedSlots = 4;
// Readers of a slot, each arriving once on the leader's `sched_empty`: the follower's
// producer, the leader's MMA issuer and the 4 epilogue warps of each CTA.
constexpr int kSchedReaders = 1 + 1 + 2 * 4;
template <class Epi>
constexpr int pair_smem_bytes() {
  return pair_stages<Epi>() * kPStageBytes + (Epi::kStaging ? kEpiSmemBytes : 0) + 1024 + 512;
}

// The schedule ring as one role sees it: slot i holds the pair's i-th tile (-1 = none
// left). `full` barriers live in each CTA (one release-arrive from the leader's
// producer per phase); `empty` barriers are the leader's.
struct SchedRing {
  uint32_t full0, empty_leader0, tile0;   // shared addresses (empty: shared::cluster)

  // A reader takes slot i: wait (bounded, cluster-scope acquire) until it is published,
  // read the tile, release the slot to the leader. False when the wait gave up.
  __device__ __forceinline__ bool take(int i, int& tile, const DevCtl& ctl,
                                       volatile int* abort_flag) const {
    const int slot = i % kSchedSlots;
    const uint32_t ph = static_cast<uint32_t>(i / kSchedSlots) & 1u;
    if (!mbar_wait_cluster(full0 + 8 * slot, ph, ctl, abort_flag)) return false;
    tile = static_cast<int>(ld_shared_u32(tile0 + 4 * slot));
    mbar_arrive_cluster(empty_leader0 + 8 * slot);
    return true;
  }
};

template <bool A_MN, bool B_MN, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    k_tc_gemm_pair(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, GemmGeom g,
                   typename Epi::Params ep, DevCtl ctl) {
  constexpr int kPStages = pair_stages<Epi>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPStages * kPABytes;
  uint8_t* sE = smem + kPStages * kPStageBytes;        // epilogue staging (Epi::kStaging)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + (Epi::kStaging ? kEpiSmemBytes : 0));
  // bars: [0, S) full, [S, 2S) empty, 2S + {0,1} acc_full, 2S + {2,3} acc_empty,
  // 2S + 4 drain, then kSchedSlots sched_full and kSchedSlots sched_empty
  int* sched_tile = reinterpret_cast<int*>(bars + 2 * kPStages + 5 + 2 * kSchedSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_tile + kSchedSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + kPStages);
  const uint32_t accf0 = smem_u32(bars + 2 * kPStages);
  const uint32_t acce0 = smem_u32(bars + 2 * kPStages + 2);
  const uint32_t drain = smem_u32(bars + 2 * kPStages + 4);
  const uint32_t sfull0 = smem_u32(bars + 2 * kPStages + 5);
  const uint32_t sempty0 = smem_u32(bars + 2 * kPStages + 5 + kSchedSlots);
  const SchedRing ring{sfull0, mapa_shared(sempty0, 0), smem_u32(sched_tile)};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(full0 + 8 * s, 1);          // leader: its arrive.expect_tx (both CTAs' bytes)
      mbar_init(empty0 + 8 * s, 1);         // one multicast commit per phase
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 2 * 128);    // leader: every epilogue thread of both CTAs
    }
    mbar_init(drain, 1);
    for (int s = 0; s < kSchedSlots; ++s) {
      mbar_init(sfull0 + 8 * s, 1);         // the leader producer's release-arrive
      mbar_init(sempty0 + 8 * s, kSchedReaders);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();                       // barriers initialised in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int n_tiles_total = g.m_tiles * g.n_tiles * g.k_parts;   // work units (256-row tiles)
  const bool dyn = g.counter != nullptr;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    // The leader's producer also claims the pair's tiles and publishes them in the ring,
    // one tile ahead: the claim of tile i + 1 is issued when tile i's loads start and
    // published when they have all been issued, so the atomic's round trip overlaps the
    // loads instead of stalling them at every tile boundary.
    const uint32_t full_leader = mapa_shared(full0, 0);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    // Leader: wait (bounded) for slot i to be free, then write `tile` into both CTAs'
    // copies of it and release-arrive on both CTAs' `full` barrier. The wait acquires at
    // cluster scope: readers in the other CTA release the slot with a release-arrive.
    auto publish = [&](int i, int tile) -> bool {
      const int slot = i % kSchedSlots;
      const uint32_t ph = static_cast<uint32_t>(i / kSchedSlots) & 1u;
      if (!mbar_wait_cluster(sempty0 + 8 * slot, ph ^ 1u, ctl, abort_flag)) return false;
      for (uint32_t r = 0; r < 2; ++r) {
        st_shared_cluster_u32(mapa_shared(ring.tile0 + 4 * slot, r), static_cast<uint32_t>(tile));
        mbar_arrive_cluster(mapa_shared(sfull0 + 8 * slot, r));
      }
      return true;
    };
    int claimed = -1;                       // leader: the tile published in slot i
    if (dyn && leader) {
      claimed = atomicAdd(g.counter, 1);
      if (claimed >= n_tiles_total) claimed = -1;
      ok = publish(0, claimed);
    }
    for (int i = 0; ok; ++i) {
      int tile = pair + i * n_pairs;
      int next = -1;
      if (dyn) {
        if (leader) {
          tile = claimed;
          if (tile >= 0) next = atomicAdd(g.counter, 1);   // the result is used after the loads
        } else if (!ring.take(i, tile, ctl, abort_flag)) {
          ok = false;
          break;
        }
        if (tile < 0) break;
      } else if (tile >= n_tiles_total) {
        break;
      }
      int ks, mt, nt, kb0, kb1;
      unit_coords(g, tile, ks, mt, nt, kb0, kb1);
      const int arow = mt * kPairM + static_cast<int>(rank) * 128;
      const int brow = nt * kBN + static_cast<int>(rank) * (kBN / 2);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, ctl, abort_flag)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * kPStageBytes);
        const uint32_t fb = full_leader + 8 * stage;
        const uint32_t a_dst = smem_u32(sA + stage * kPABytes);
        const uint32_t b_dst = smem_u32(sB + stage * kPBBytes);
        if (!A_MN) {
          tma_load_2d_pair(a_dst, &tmA, fb, kb * kBK, arow);
        } else {
          tma_load_2d_pair(a_dst, &tmA, fb, arow, kb * kBK);
          tma_load_2d_pair(a_dst + 8192, &tmA, fb, arow + 64, kb * kBK);
        }
        if (!B_MN) {
          tma_load_2d_pair(b_dst, &tmB, fb, kb * kBK, brow);
        } else {
          tma_load_2d_pair(b_dst, &tmB, fb, brow, kb * kBK);
          tma_load_2d_pair(b_dst + 8192, &tmB, fb, brow + 64, kb * kBK);
        }
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (ok && dyn && leader) {
        claimed = next < n_tiles_total ? next : -1;
        ok = publish(i + 1, claimed);
      }
    }
    if (!ok) {
      record_status(ctl, kStatusTimeout);
      *abort_flag = 1;
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    constexpr uint32_t idesc = idesc_bf16_f32(kPairM, kBN, A_MN, B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    for (int i = 0; ok; ++i, ++local) {
      int tile = pair + i * n_pairs;
      if (dyn) {
        if (!ring.take(i, tile, ctl, abort_flag)) {
          ok = false;
          break;
        }
        if (tile < 0) break;
      } else if (tile >= n_tiles_total) {
        break;
      }
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(acce0 + 8 * acc, acc_phase ^ 1, ctl, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * kBN;
      int ks, mt, nt, kb0, kb1;
      unit_coords(g, tile, ks, mt, nt, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full0 + 8 * stage, phase, ctl, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * kPABytes);
        const uint32_t b0 = smem_u32(sB + stage * kPBBytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t ad = A_MN ? sw128_desc(a0 + k * 2048, 8192, 1024)
                                   : sw128_desc(a0 + k * 32, 16, 1024);
          const uint64_t bd = B_MN ? sw128_desc(b0 + k * 2048, 8192, 1024)
                                   : sw128_desc(b0 + k * 32, 16, 1024);
          tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
        }
        tc_commit_pair_mc(empty0 + 8 * stage, 0x3);
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      tc_commit_pair_mc(accf0 + 8 * acc, 0x3);
    }
    if (!ok) {
      record_status(ctl, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_commit_pair(drain);
    volatile int never = 0;
    if (!mbar_wait(drain, 0, ctl, &never)) record_status(ctl, kStatusTimeout);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int lg = warp & 3;
    const int row = static_cast<int>(rank) * 128 + lg * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(lg * 32) << 16);
    const uint32_t acce_leader = mapa_shared(acce0, 0);
    const EpiCtx ectx{&tmC, smem_u32(sE + (warp - 2) * kEpiWarpBytes), lane};
    int local = 0;
    for (int i = 0;; ++i, ++local) {
      int tile = pair + i * n_pairs;
      if (dyn) {
        // lane 0 takes the slot for the warp (one release per warp) and shares the tile
        int ok = 1;
        if (lane == 0) ok = ring.take(i, tile, ctl, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        tile = __shfl_sync(0xffffffffu, tile, 0);
        if (!ok) {
          if (lane == 0) {
            record_status(ctl, kStatusTimeout);
            *abort_flag = 1;
          }
          break;
        }
        if (tile < 0) break;
      } else if (tile >= n_tiles_total) {
        break;
      }
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(accf0 + 8 * acc, acc_phase, ctl, abort_flag)) {
        record_status(ctl, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int ks, mt, nt, kb0, kb1;
      unit_coords(g, tile, ks, mt, nt, kb0, kb1);
      Epi epi;
      epi.begin(ep, mt * kPairM + row, nt, ks, ectx);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_addr + acc * kBN + c * 32, v);
        tmem_wait_ld();
        epi.chunk(ep, c, v);
      }
      tc_fence_before();
      mbar_arrive_cluster(acce_leader + 8 * acc);
      epi.end(ep);
    }
  }

  // Bulk stores an epilogue issued must finish before the CTA (and its shared
  // memory) goes away; warps that issued none return at once. An epilogue whose stores
  // go to another process's memory (Epi::kSystemFence) fences them at system scope.
  if (warp >= 2 && lane == 0) bulk_wait_group<0>();
  if constexpr (Epi::kSystemFence) {
    if (warp >= 2) __threadfence_system();
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // After an abort a load issued just before may still be landing in this CTA's
    // shared memory: give it a bounded 2 ms before the pair leaves.
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  tc_fence_before();
  cluster_sync_all();                       // neither CTA leaves while the pair is in use
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace dpo
