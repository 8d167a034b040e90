// Tile shape of the tcgen05 GEMMs, shared by the kernels and the host-side
// tensor-map set-up (TMA boxes must match the shared-memory tiles).
#pragma once

namespace dpo {

constexpr int kBM = 128;   // accumulator rows (TMEM lanes) per tile
constexpr int kBN = 256;   // accumulator columns per tile
constexpr int kBK = 64;    // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kBoxRows = 128;  // rows of a K-major TMA box (a CTA's share of a tile)
constexpr int kBoxMN = 64;     // columns of an MN-major TMA box (one 128-byte swizzle row)

}  // namespace dpo
