// Logits-mean metrics: the mean of the logits z = h_t . W^T over every position of
// the chosen rows, and of the rejected rows, over the whole vocabulary (the
// torchtune DPO loop of "Run Distributed Full-Model DPO with PyTorch FSDP" logs
// them; Step 4 splits the logits of all positions into the two halves).
//
// The logits are never formed: by bilinearity
//   sum_{t, v} z_tv = sum_k (sum_t h_tk) (sum_v W_vk),
// so each side needs the column sums of its H rows and of W, and one dot product.
// The work is two HBM-bound column reductions (W read once, H once) and a tiny
// finishing kernel. Each lane adds groups of 8 (bf16) or 4 (fp32) rows in fp32 and
// the group sums in fp64; every reduction has a fixed order, so the result is the
// same for every run.
#include "internal.h"

namespace dpo {

namespace {

// Which rows of a [n, d] matrix a column sum covers: row i of the sum is flat row
//   i                                     (identity: W)
//   (side * B + i / L) * L + i % L        (halves: rows [0, B) chosen, [B, 2B) rejected)
//   (2 * (i / L) + side) * L + i % L      (adjacent: even rows chosen, odd rejected)
// Row indices fit 32 bits (R * L < 2^31 and V <= 2^24); halves and W need no
// division, adjacent pairs one 32-bit division per row.
struct RowMap {
  int identity, adjacent, side, B, L;
  __device__ __forceinline__ long long operator()(int i) const {
    if (identity) return i;
    if (!adjacent) return static_cast<long long>(side) * B * L + i;
    const unsigned p = static_cast<unsigned>(i) / static_cast<unsigned>(L);
    return static_cast<long long>(i) + static_cast<long long>(p + side) * L;  // (2p + side) L + t
  }
};

// One row's 8 columns, loaded raw (loads of several rows are issued before any is
// converted, to keep enough bytes in flight); a group of rows is added in fp32, the
// group sums and the tail rows in fp64.
template <typename T>
struct Raw8;

template <>
struct Raw8<uint16_t> {
  static constexpr int kUnroll = 8;   // rows in flight per warp: 8 x 16 B per lane
  uint4 v;
  __device__ __forceinline__ void load(const uint16_t* p) {
    v = __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ void add_f32(float (&f)[8]) const {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] += __uint_as_float(w[j] << 16);
      f[2 * j + 1] += __uint_as_float(w[j] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ void add_to(double (&acc)[8]) const {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {     // bf16 -> fp32 is exact: the bits move up 16 places
      acc[2 * j] += static_cast<double>(__uint_as_float(w[j] << 16));
      acc[2 * j + 1] += static_cast<double>(__uint_as_float(w[j] & 0xffff0000u));
    }
  }
};

template <>
struct Raw8<float> {
  static constexpr int kUnroll = 4;   // 4 x 32 B per lane
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void add_f32(float (&f)[8]) const {
    f[0] += a.x; f[1] += a.y; f[2] += a.z; f[3] += a.w;
    f[4] += b.x; f[5] += b.y; f[6] += b.z; f[7] += b.w;
  }
  __device__ __forceinline__ void add_to(double (&acc)[8]) const {
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
};

constexpr int kSlab = 256;          // columns per block: 32 lanes x 8 columns
constexpr int kWarps = 8;

// Column sums of W and of both sides' H rows in one launch. Grid: (column slabs,
// S_W + 2 S_H). blockIdx.y < S_W: rows [s V / S_W, (s + 1) V / S_W) of W into
// pW[s * d + k]; otherwise side = (y - S_W) / S_H, split s = (y - S_W) % S_H of that
// side's B L rows into pH[(side * S_H + s) * d + k]. The splits are chosen so every
// block reads about the same number of rows. Warp w of a block takes rows w, w + 8,
// ... of its range, in that order; the 8 warps' sums are then added in warp order.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32, 3)
    k_colsum(const T* __restrict__ W, const T* __restrict__ H, int d, int nW, int nH, int S_W,
             int S_H, RowMap hmap, double* __restrict__ pW, double* __restrict__ pH) {
  constexpr int U = Raw8<T>::kUnroll;
  __shared__ double red[kWarps][kSlab];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * kSlab + lane * 8;
  const T* X;
  RowMap map;
  int n, S, s;
  double* partial;
  if (static_cast<int>(blockIdx.y) < S_W) {
    X = W;
    map = RowMap{1, 0, 0, 0, 0};
    n = nW;
    S = S_W;
    s = blockIdx.y;
    partial = pW;
  } else {
    const int k = blockIdx.y - S_W;
    X = H;
    map = hmap;
    map.side = k / S_H;
    n = nH;
    S = S_H;
    s = k - map.side * S_H;
    partial = pH + static_cast<long long>(map.side) * S_H * d;
  }
  const int r0 = static_cast<int>(static_cast<long long>(n) * s / S);
  const int r1 = static_cast<int>(static_cast<long long>(n) * (s + 1) / S);
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (col < d) {                    // d is a multiple of 8: a lane's 8 columns are all in or all out
    int i = r0 + warp;
    for (; i + (U - 1) * kWarps < r1; i += U * kWarps) {
      Raw8<T> x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) x[u].load(X + map(i + u * kWarps) * d + col);
      // the U rows are added in fp32 first (one fp64 conversion per U values: the
      // conversion, not HBM, limits the kernel at power-capped clocks otherwise)
      float f[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) x[u].add_f32(f);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += static_cast<double>(f[j]);
    }
    for (; i < r1; i += kWarps) {
      Raw8<T> x;
      x.load(X + map(i) * d + col);
      x.add_to(acc);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = acc[j];
  __syncthreads();
  const int c = blockIdx.x * kSlab + threadIdx.x;
  if (c < d) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w][threadIdx.x];
    partial[static_cast<long long>(s) * d + c] = t;
  }
}

constexpr int kDotCols = 32;        // columns per k_mean_dot block (one per lane)

// Per group of 32 columns: u_side[k] = sum_s pH[side][s][k], w[k] = sum_s pW[s][k]
// (warp w adds the splits s = w, w + 8, ... of each; the 8 warps' sums are then added in
// warp order), and dots[side][group] = sum over the group's columns of u_side[k] w[k]
// (lane order).
__global__ void __launch_bounds__(kWarps * 32) k_mean_dot(const double* __restrict__ pW,
                                                          const double* __restrict__ pH, int S_W,
                                                          int S_H, int d,
                                                          double* __restrict__ dots) {
  __shared__ double red[3][kWarps][kDotCols];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * kDotCols + lane;
  double w = 0.0, u0 = 0.0, u1 = 0.0;
  if (k < d) {
    const long long sd = static_cast<long long>(S_H) * d;
    for (int s = warp; s < S_W; s += kWarps) w += pW[static_cast<long long>(s) * d + k];
    for (int s = warp; s < S_H; s += kWarps) {
      const long long o = static_cast<long long>(s) * d + k;
      u0 += pH[o];
      u1 += pH[sd + o];
    }
  }
  red[0][warp][lane] = w;
  red[1][warp][lane] = u0;
  red[2][warp][lane] = u1;
  __syncthreads();
  if (warp == 0) {
    double tw = 0.0, t0 = 0.0, t1 = 0.0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) {
      tw += red[0][i][lane];
      t0 += red[1][i][lane];
      t1 += red[2][i][lane];
    }
    red[1][0][lane] = t0 * tw;
    red[2][0][lane] = t1 * tw;
    __syncwarp();
    if (lane == 0) {
      double a = 0.0, b = 0.0;
      for (int i = 0; i < kDotCols; ++i) {
        a += red[1][0][i];
        b += red[2][0][i];
      }
      dots[blockIdx.x] = a;
      dots[gridDim.x + blockIdx.x] = b;
    }
  }
}

constexpr int kMaxGroups = 65536 / kDotCols;   // d <= 65536

// means[side] = (sum over column groups of dots[side][group], in group order) / count.
// The block stages the dot products in shared memory, then one thread per side adds.
__global__ void __launch_bounds__(256) k_mean_finish(const double* __restrict__ dots, int groups,
                                                     double inv_count, float* __restrict__ means) {
  __shared__ double sd[2 * kMaxGroups];
  for (int i = threadIdx.x; i < 2 * groups; i += blockDim.x) sd[i] = dots[i];
  __syncthreads();
  const int side = threadIdx.x;
  if (side < 2) {
    double t = 0.0;
    for (int b = 0; b < groups; ++b) t += sd[side * groups + b];
    means[side] = static_cast<float>(t * inv_count);
  }
}

template <typename T>
cudaError_t run(const T* H, const T* W, int R, int L, int d, int V, int adjacent, int S_W,
                int S_H, double* pW, double* pH, double* dots, float* means, cudaStream_t st) {
  const int slabs = (d + kSlab - 1) / kSlab;
  const int B = R / 2;
  k_colsum<T><<<dim3(slabs, S_W + 2 * S_H), kWarps * 32, 0, st>>>(
      W, H, d, V, B * L, S_W, S_H, RowMap{0, adjacent, 0, B, L}, pW, pH);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int groups = (d + kDotCols - 1) / kDotCols;
  k_mean_dot<<<groups, kWarps * 32, 0, st>>>(pW, pH, S_W, S_H, d, dots);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const double inv_count = 1.0 / (static_cast<double>(B) * L * V);
  k_mean_finish<<<1, 256, 0, st>>>(dots, groups, inv_count, means);
  return cudaGetLastError();
}

// Resident k_colsum blocks per SM (cached per device).
template <typename T>
int colsum_blocks_per_sm() {
  static int cache[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 1;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_colsum<T>, kWarps * 32, 0) !=
            cudaSuccess ||
        n < 1)
      n = 1;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace

// Largest number of row splits of a column sum for hidden size d (bounds the
// workspace): at most 64, and at most 1024 blocks per sum.
int logits_mean_splits(int d) {
  const int slabs = (d + kSlab - 1) / kSlab;
  const int s = 1024 / slabs;
  return s < 1 ? 1 : (s > 64 ? 64 : s);
}

// Workspace of launch_logits_mean: W's and both sides' partial column sums, then
// the per-group dot products.
size_t logits_mean_bytes(int d) {
  const size_t groups = (d + kDotCols - 1) / kDotCols;
  return (3ull * logits_mean_splits(d) * static_cast<size_t>(d) + 2 * groups) * sizeof(double);
}

// The splits actually used: one wave of resident blocks over the column slabs,
// shared between W (V rows) and the two sides (B L rows each) in proportion to
// their rows, at least one split each and at most logits_mean_splits(d).
cudaError_t launch_logits_mean(const void* H, const void* W, bool bf16, int R, int L, int d, int V,
                               int adjacent, void* ws, float* means, int sms, cudaStream_t st) {
  const int slabs = (d + kSlab - 1) / kSlab;
  const int per_sm = bf16 ? colsum_blocks_per_sm<uint16_t>() : colsum_blocks_per_sm<float>();
  const int cap = logits_mean_splits(d);
  const double nW = V, nH = static_cast<double>(R / 2) * L;
  const int total = sms * per_sm / slabs;                 // blocks per slab in one wave
  int S_H = static_cast<int>(total * nH / (nW + 2 * nH) + 0.5);
  S_H = S_H < 1 ? 1 : (S_H > cap ? cap : S_H);
  int S_W = total - 2 * S_H;
  S_W = S_W < 1 ? 1 : (S_W > cap ? cap : S_W);
  double* pW = static_cast<double*>(ws);
  double* pH = pW + static_cast<size_t>(cap) * d;
  double* dots = pH + 2ull * cap * d;
  if (bf16)
    return run(static_cast<const uint16_t*>(H), static_cast<const uint16_t*>(W), R, L, d, V,
               adjacent, S_W, S_H, pW, pH, dots, means, st);
  return run(static_cast<const float*>(H), static_cast<const float*>(W), R, L, d, V, adjacent,
             S_W, S_H, pW, pH, dots, means, st);
}

}  // namespace dpo
