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
// cut the forward's DRAM reads per launch from 13-15 GB to ~4.6 GB (ncu). dH and
// dW: 0 keeps N fastest, > 0 groups that many 256-column tiles of d (measured: no
// gain, their re-reads come from tiles drifting apart over long K loops). L2
// eviction-priority hints on the TMA loads were measured too and raised traffic.
#ifndef DPO_L2_GROUP_BYTES
#define DPO_L2_GROUP_BYTES (40ll << 20)
#endif
#ifndef DPO_GROUP_DH
#define DPO_GROUP_DH 0
#endif
#ifndef DPO_GROUP_DW
#define DPO_GROUP_DW 0
#endif
// Ints of the workspace's counter area (the pair kernels' tile claim counter is the
// first; each GEMM launch zeroes it before it starts).
constexpr int kSyncInts = 64;

}  // namespace dpo
