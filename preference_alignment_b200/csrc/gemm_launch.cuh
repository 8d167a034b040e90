// Host-side launch of the tcgen05 GEMM kernels (included by the .cu files that
// instantiate them). The CTA-pair kernel is the default; the single-CTA kernel
// is used when the device cannot co-schedule CTA pairs, when its 128-row tiles
// fill the waves clearly better, or when the diagnostic variant mask asks for it.
#pragma once

#include "internal.h"
#include "tc_gemm.cuh"

namespace dpo {

// Token tiles (256 rows of packed H, K = d) per group of the forward raster: as
// many as fit DPO_L2_GROUP_BYTES, at least one.
inline int token_group(int d) {
  const long long per_tile = 256ll * d * 2;
  const long long g = DPO_L2_GROUP_BYTES / per_tile;
  return g < 1 ? 1 : static_cast<int>(g);
}

// Clusters of two that can be resident at once for a pair-kernel instantiation
// on the current device (cached per device).
template <class Kern>
int max_pair_clusters(Kern kern, int smem_bytes) {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] != 0) return cache[dev] > 0 ? cache[dev] : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[dev] = n > 0 ? n : -1;
  return n;
}

// Fraction of a launch's row slots that hold real rows: M rows in tiles of tile_m,
// times n_tiles, spread over `slots` concurrent tiles in whole waves (the ragged
// last row tile and the partly idle last wave are the waste).
inline double tile_fill(int M, int tile_m, int n_tiles, int slots) {
  const long long tiles = static_cast<long long>((M + tile_m - 1) / tile_m) * n_tiles;
  const long long waves = (tiles + slots - 1) / slots;
  return static_cast<double>(M) * n_tiles / (static_cast<double>(waves) * slots * tile_m);
}

// Number of K parts of kb_part blocks each (the last may be shorter, none is empty).
inline int split_k_parts(int k_blocks, int kb_part) { return (k_blocks + kb_part - 1) / kb_part; }

// A CTA pair does a 256-row tile ~3 % faster than two single CTAs do its halves
// (measured under the power cap); the single-CTA kernel is chosen only when its
// finer tiles fill the GPU's waves better by more than this margin.
constexpr double kPairMargin = 1.05;

// D[M x N] = A[M x K] . B[N x K]^T with the epilogue Epi; `sms` is the device's SM
// count (or the SM budget of this launch).
// Raster: `order` as in GemmGeom (0: M fastest, 1: N fastest, 2/3 grouped along M/N
// with `group` 256-wide tiles per group; a group of 0 falls back to order 0).
// `kind` (a GemmKind) selects this GEMM's bits of the dpo_set_gemm_variant mask:
//   bit kind      set: the single-CTA kernel; clear: CTA pairs unless 128-row tiles
//                 fill the waves clearly better (tile_fill), e.g. 4,648 rows x 8 column
//                 tiles: 152 pair tiles are 2.05 waves of 74 pairs (3 launched, 68 %
//                 full), 296 single tiles exactly 2 waves of 148 CTAs;
//   bit 4 + kind  set: the pair kernel's static tile schedule; clear: tiles claimed in
//                 raster order from `counter` (one int of workspace, zeroed here).
// mapC is the epilogue's store tensor map (epilogues that do not store through TMA
// ignore it; pass any valid map).
// kb_part > 0 splits K into parts of kb_part K blocks (split_k_parts gives their
// count); each part of a tile is its own work unit and the epilogue learns its part.
template <bool A_MN, bool B_MN, class Epi>
cudaError_t launch_gemm(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapC,
                        int M, int N, int K, int order, const typename Epi::Params& p, int sms,
                        const DevCtl& ctl, cudaStream_t st, int kind, int group, int* counter,
                        int kb_part = 0) {
  if (order >= 2 && group <= 0) order = 0;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int k_blocks = (K + kBK - 1) / kBK;
  if (kb_part <= 0 || kb_part > k_blocks) kb_part = k_blocks;
  const int k_parts = split_k_parts(k_blocks, kb_part);
  const int variant = gemm_variant();
  if (((variant >> kind) & 1) == 0) {
    auto kern = k_tc_gemm_pair<A_MN, B_MN, Epi>;
    constexpr int smem = pair_smem_bytes<Epi>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int clusters = max_pair_clusters(kern, smem);
    if (clusters > 0) {
      GemmGeom g{(M + kPairM - 1) / kPairM, n_tiles, k_blocks, order, group > 0 ? group : 1,
                 k_parts, kb_part, nullptr};
      const int tiles = g.m_tiles * g.n_tiles * k_parts;
      int pairs = clusters < sms / 2 ? clusters : sms / 2;
      if (pairs > tiles) pairs = tiles;
      if (pairs < 1) pairs = 1;
      const bool single_fills_better =
          tile_fill(M, kBM, n_tiles * k_parts, sms) >
          kPairMargin * tile_fill(M, kPairM, n_tiles * k_parts, pairs);
      if (!single_fills_better) {
        // Claiming tiles in raster order pays where the static round-robin's drift
        // spreads the tiles in flight over more than they can share in L2: across the
        // group boundaries of a grouped raster (the forward and dz GEMMs at the
        // Llama-3.1-8B head: 2 token groups, DRAM reads halved) and over the long K loops
        // of dH and dW. A grouped raster with a single group (every token tile in one
        // group: `small`, `long`) streams each weight tile past all its token tiles at
        // once either way, and there the static schedule measured ~2 % faster per call.
        const bool one_group = order == 2 && g.m_tiles <= g.group;
        if (((variant >> (4 + kind)) & 1) == 0 && counter != nullptr && !one_group) {
          e = cudaMemsetAsync(counter, 0, sizeof(int), st);
          if (e != cudaSuccess) return e;
          g.counter = counter;
        }
        kern<<<2 * pairs, kGemmThreads, smem, st>>>(mapA, mapB, mapC, g, p, ctl);
        return cudaGetLastError();
      }
    }
  }
  auto kern = k_tc_gemm<A_MN, B_MN, Epi>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGemmSmemBytes);
  if (e != cudaSuccess) return e;
  GemmGeom g{(M + kBM - 1) / kBM, n_tiles, k_blocks, order,
             group > 0 ? (order == 2 ? 2 * group : group) : 1, k_parts, kb_part, nullptr};
  const int tiles = g.m_tiles * g.n_tiles * k_parts;
  kern<<<sms < tiles ? sms : tiles, kGemmThreads, kGemmSmemBytes, st>>>(mapA, mapB, mapC, g, p,
                                                                        ctl);
  return cudaGetLastError();
}

}  // namespace dpo
