// Tile shape of the tcgen05 GEMMs, shared by the kernels and the host-side
// tensor-map set-up (TMA boxes must match the shared-memory tiles).
#pragma once

namespace dpo {

constexpr int kBM = 128;   // accumulator rows (TMEM lanes) per tile
constexpr int kBN = 256;   // accumulator columns per tile
constexpr int kBK = 64;    // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kBoxRows = 128;  // rows of a K-major TMA box (a CTA's share of a tile)
constexpr int kBoxMN = 64;     // columns of an MN-major TMA box (one 128-byte swizzle row)

// Raster of each GEMM. The forward and the dz recompute sweep groups of token
// tiles over the vocabulary; a group's packed rows take at most DPO_L2_GROUP_BYTES
// of L2 (the rest holds the streamed weight tiles). At the Llama-3.1-8B head this
// cut the forward's DRAM reads per launch from 13-15 GB to ~4.6 GB (ncu), and
// claiming tiles in raster order to 2.3 GB. dH and dW: 0 keeps N fastest, > 0
// groups that many 256-column tiles of d. With tiles claimed in raster order, dH's
// 74 tiles in flight then span ~9 token tiles x 8 column tiles instead of ~5 x 16,
// which cut its DRAM reads by a third (12.0 -> 8.0 GB on a 2-pair Llama-8B case) and
// its time by 4 %; the same grouping raised dW's reads (1.9 -> 2.6 GB), so dW keeps
// N fastest. L2 eviction-priority hints on the TMA loads were measured too and
// raised traffic.
#ifndef DPO_L2_GROUP_BYTES
#define DPO_L2_GROUP_BYTES (40ll << 20)
#endif
#ifndef DPO_GROUP_DH
#define DPO_GROUP_DH 8
#endif
#ifndef DPO_GROUP_DW
#define DPO_GROUP_DW 0
#endif
// Ints of the workspace's counter area (the pair kernels' tile claim counter is the
// first; each GEMM launch zeroes it before it starts).
constexpr int kSyncInts = 64;

}  // namespace dpo
