// Backward kernels of the DPO head path (bf16 tensor-core route).
//
// The objective is sum_r coef_r * S_r with S_r the row's completion log-prob sum,
// so for a scored position t of row r the logit gradient is
//   dz[t, v] = coef_r * (1[v = y_t] - softmax(z_t)[v])
// and dH[t] = dz[t] . W, dW = sum_t dz[t]^T h_t (chain rule through log-softmax;
// the pages run this as loss.backward() on the chunked, checkpointed loss of
// "DPO Training on GPU, in depth", "A training configuration that fits", which
// recomputes each chunk's log-softmax in the backward: here the logits are
// recomputed tile by tile).
//
// Three persistent tcgen05 GEMMs per token chunk:
//   k_tc_gemm<K,K,EpiGrad>  z tile = Hp . W^T, epilogue forms dz in bf16 (never z)
//   k_tc_gemm<K,MN,EpiRows> dH chunk = dz . W        (K = V)
//   k_tc_gemm<MN,MN,EpiDW>  dW (+)= dz^T . Hp        (K = tokens)
#include <cmath>

#include "internal.h"
#include "gemm_launch.cuh"

namespace dpo {

constexpr float kLog2eB = 1.4426950408889634f;

// ------------------------------------------------------------------ dz epilogue
// Each thread forms its row's 32 bf16 values of a chunk; the warp stages its 32 x 32
// block in shared memory (64-byte swizzled, matching the store map) and one lane
// stores it with a TMA bulk tensor store (rows beyond the chunk and columns beyond V
// fall outside the tensor map and are skipped).
// Two staging buffers per warp: a buffer is refilled only after the store issued
// from it two chunks earlier has finished reading it.
struct EpiGrad {
  static constexpr bool kStaging = true;   // stores through TMA staging buffers
  static constexpr bool kSystemFence = false;
  struct Params {
    const int* y;
    const float* lse;
    const float* coef;     // [R] per-row coefficient
    const int* rowid;
    int Mc, V, tok0;
  };
  int vbase, yl, row0;
  float nl2, cf;
  EpiCtx ctx;

  __device__ __forceinline__ void begin(const Params& p, int m_row, int nt, int,
                                        const EpiCtx& c) {
    const int tok = m_row;
    ctx = c;
    row0 = tok - c.lane;                 // first row of this warp's 32-row block
    vbase = nt * kBN;
    yl = -1;
    nl2 = 0.f;
    cf = 0.f;                            // rows past the chunk compute zeros (not stored)
    if (tok < p.Mc) {
      const int gt = p.tok0 + tok;
      const int y = __ldg(p.y + gt);
      yl = y - vbase;
      nl2 = -__ldg(p.lse + gt) * kLog2eB;
      // bad target: no gradient; a target in another vocabulary shard keeps the
      // softmax term (yl never matches a column of this call)
      cf = y != kTargetBad ? __ldg(p.coef + __ldg(p.rowid + gt)) : 0.f;
    }
  }

  __device__ __forceinline__ void chunk(const Params&, int c, const uint32_t (&v)[32]) {
    uint32_t packed[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const int col = c * 32 + j;
      const float g0 = cf * ((col == yl ? 1.f : 0.f) -
                             ex2_approx(fmaf(__uint_as_float(v[j]), kLog2eB, nl2)));
      const float g1 = cf * ((col + 1 == yl ? 1.f : 0.f) -
                             ex2_approx(fmaf(__uint_as_float(v[j + 1]), kLog2eB, nl2)));
      packed[j / 2] = pack_bf16x2(g0, g1);
    }
    const uint32_t buf = ctx.stage + (c & 1) * (kEpiWarpBytes / 2);
    if (ctx.lane == 0) bulk_wait_group_read<1>();   // the store from this buffer is done
    __syncwarp();
    // row `lane`: 32 bf16 = 64 bytes, its four 16-byte pieces placed by the store
    // map's 64-byte swizzle (piece q at q ^ ((row >> 1) & 3)), so the 32 lanes' stores
    // spread over all 32 banks; the TMA store writes the rows back unswizzled
    const uint32_t dst = buf + ctx.lane * 64;
    const uint32_t sw = (ctx.lane >> 1) & 3;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16 * (q ^ sw)),
                   "r"(packed[4 * q]), "r"(packed[4 * q + 1]), "r"(packed[4 * q + 2]),
                   "r"(packed[4 * q + 3])
                   : "memory");
    fence_proxy_async_smem();
    __syncwarp();
    if (ctx.lane == 0 && row0 >= 0) {
      tma_store_2d(ctx.map, buf, vbase + c * 32, row0);
      bulk_commit_group();
    }
  }

  __device__ __forceinline__ void end(const Params&) {}
};

// ------------------------------------------------------------------ dH rows epilogue
// K part 0 of a unit writes (or adds to) the dH rows of its positions; with split-K
// the later parts write their partial sums to fp32 scratch, which k_dh_reduce adds
// to the rows in part order.
struct EpiRows {
  static constexpr bool kStaging = false;   // stores go straight to global memory
  static constexpr bool kSystemFence = false;
  struct Params {
    const int* dst;        // packed position -> flat row r * L + t
    float* out;            // dH [R * L, d]
    float* part;           // split-K scratch [k_parts - 1, Mc, d] of parts 1.. (or null)
    int Mc, d, tok0;
    int accumulate;        // part 0 adds to the rows (a later vocabulary chunk of K)
  };
  float* o;
  int nbase;
  bool valid, acc;

  __device__ __forceinline__ void begin(const Params& p, int m_row, int nt, int ks,
                                        const EpiCtx&) {
    const int tok = m_row;
    valid = tok < p.Mc;
    nbase = nt * kBN;
    o = nullptr;
    acc = false;
    if (!valid) return;
    if (ks == 0) {
      o = p.out + static_cast<long long>(__ldg(p.dst + p.tok0 + tok)) * p.d;
      acc = p.accumulate != 0;
    } else {
      o = p.part + (static_cast<long long>(ks - 1) * p.Mc + tok) * p.d;
    }
  }

  __device__ __forceinline__ void chunk(const Params& p, int c, const uint32_t (&v)[32]) {
    if (!valid) return;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int col = nbase + c * 32 + q * 4;
      if (col < p.d) {
        float4 r = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                               __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        float4* dst = reinterpret_cast<float4*>(o + col);
        if (acc) {
          const float4 old = *dst;
          r.x += old.x;
          r.y += old.y;
          r.z += old.z;
          r.w += old.w;
        }
        *dst = r;
      }
    }
  }

  __device__ __forceinline__ void end(const Params&) {}
};

// dH[dst[tok0 + i]] += part[0][i] + part[1][i] + ... (parts in order, one thread per 4
// columns): the split-K partial sums of K parts 1.., after part 0 wrote the rows.
__global__ void __launch_bounds__(256) k_dh_reduce(float* __restrict__ dH,
                                                   const float* __restrict__ part,
                                                   const int* __restrict__ dst, int tok0, int Mc,
                                                   int d, int n_extra) {
  const int d4 = d / 4;
  const long long q = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (q >= static_cast<long long>(Mc) * d4) return;
  const int i = static_cast<int>(q / d4);
  const int c = static_cast<int>(q - static_cast<long long>(i) * d4);
  float4* o = reinterpret_cast<float4*>(dH + static_cast<long long>(__ldg(dst + tok0 + i)) * d) + c;
  float4 a = *o;
  const long long stride = static_cast<long long>(Mc) * d4;
  const float4* src = reinterpret_cast<const float4*>(part) + q;
  for (int s = 0; s < n_extra; ++s) {
    const float4 b = __ldg(src + s * stride);
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
  }
  *o = a;
}

// ------------------------------------------------------------------ dW epilogue
struct EpiDW {
  static constexpr bool kStaging = false;   // stores go straight to global memory
  static constexpr bool kSystemFence = false;
  struct Params {
    float* out;            // dW [V, d]
    int V, d, accumulate;
  };
  float* o;
  int nbase;
  bool valid;

  __device__ __forceinline__ void begin(const Params& p, int m_row, int nt, int,
                                        const EpiCtx&) {
    const int v = m_row;
    valid = v < p.V;
    nbase = nt * kBN;
    o = valid ? p.out + static_cast<long long>(v) * p.d : nullptr;
  }

  __device__ __forceinline__ void chunk(const Params& p, int c, const uint32_t (&v)[32]) {
    if (!valid) return;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int col = nbase + c * 32 + q * 4;
      if (col < p.d) {
        float4 r = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                               __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        float4* dst = reinterpret_cast<float4*>(o + col);
        if (p.accumulate) {
          const float4 old = *dst;
          r.x += old.x;
          r.y += old.y;
          r.z += old.z;
          r.w += old.w;
        }
        *dst = r;
      }
    }
  }

  __device__ __forceinline__ void end(const Params&) {}
};

// ------------------------------------------------------------------ dW scatter epilogue
// The data-parallel exchange fused into the dW GEMM, as a reduce-scatter: the vocabulary
// rows are owned by ranks in blocks (rank q owns rows [q * rows_per_rank, ...), the last
// rank the rest), and each finished row of this rank's contribution dz_r^T . Hp_r is
// stored straight into its owner's receive buffer, in this rank's slot. The owner's
// buffer is another process's memory mapped into this one (peer memory over NVLink when
// that process runs on another GPU), so the transfer happens tile by tile while the GEMM
// runs; the epilogue threads fence at system scope before the kernel ends, so a barrier
// after the kernel (on every rank) makes every rank's rows visible to their owners,
// who then add the slots in rank order (k_dw_reduce_slots).
struct EpiDWScatter {
  static constexpr bool kStaging = false;   // plain stores to (peer) global memory
  static constexpr bool kSystemFence = true;
  struct Params {
    float* recv[kMaxScatterRanks];   // recv[q]: rank q's buffer [n_ranks, rows_q, d]
    int V, d, n_ranks, rank, rows_per_rank;
  };
  float* o;
  int nbase;
  bool valid;

  __device__ __forceinline__ void begin(const Params& p, int m_row, int nt, int,
                                        const EpiCtx&) {
    const int v = m_row;
    valid = v < p.V;
    nbase = nt * kBN;
    o = nullptr;
    if (!valid) return;
    const int q = min(v / p.rows_per_rank, p.n_ranks - 1);
    const int first = q * p.rows_per_rank;
    const int rows_q = q == p.n_ranks - 1 ? p.V - first : p.rows_per_rank;
    o = p.recv[q] + (static_cast<long long>(p.rank) * rows_q + (v - first)) * p.d;
  }

  __device__ __forceinline__ void chunk(const Params& p, int c, const uint32_t (&v)[32]) {
    if (!valid) return;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int col = nbase + c * 32 + q * 4;
      if (col < p.d)
        *reinterpret_cast<float4*>(o + col) =
            make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                        __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
    }
  }

  __device__ __forceinline__ void end(const Params&) {}
};

// out[row] (+)= slot 0[row] + slot 1[row] + ... (slots in rank order, fp32, one thread per
// 4 columns): the owner's side of the reduce-scatter, over its [n_slots, rows, d] buffer.
__global__ void __launch_bounds__(256) k_dw_reduce_slots(const float* __restrict__ recv,
                                                         int n_slots, long long rows_x_d4,
                                                         float* __restrict__ out,
                                                         int accumulate) {
  const long long q = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (q >= rows_x_d4) return;
  const float4* src = reinterpret_cast<const float4*>(recv) + q;
  float4 a = __ldg(src);
  for (int s = 1; s < n_slots; ++s) {
    const float4 b = __ldg(src + s * rows_x_d4);
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
  }
  float4* o = reinterpret_cast<float4*>(out) + q;
  if (accumulate) {
    const float4 old = *o;
    a.x += old.x;
    a.y += old.y;
    a.z += old.z;
    a.w += old.w;
  }
  *o = a;
}

cudaError_t launch_bwd_dw_scatter(const CUtensorMap& mapA, const CUtensorMap& mapB, int Mc, int V,
                                  int d, float* const* recv, int n_ranks, int rank,
                                  int rows_per_rank, int grid, int* sync, const DevCtl& ctl,
                                  cudaStream_t st) {
  if (n_ranks < 1 || n_ranks > kMaxScatterRanks) return cudaErrorInvalidValue;
  EpiDWScatter::Params p{};
  for (int q = 0; q < n_ranks; ++q) p.recv[q] = recv[q];
  p.V = V;
  p.d = d;
  p.n_ranks = n_ranks;
  p.rank = rank;
  p.rows_per_rank = rows_per_rank;
  return launch_gemm<true, true, EpiDWScatter>(mapA, mapB, mapA, V, d, Mc,
                                               DPO_GROUP_DW > 0 ? 3 : 1, p, grid, ctl, st,
                                               kGemmDW, DPO_GROUP_DW, sync);
}

cudaError_t launch_dw_reduce_slots(const float* recv, int n_slots, int rows, int d, float* out,
                                   int accumulate, cudaStream_t st) {
  const long long n4 = static_cast<long long>(rows) * (d / 4);
  if (n4 == 0) return cudaSuccess;
  k_dw_reduce_slots<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(recv, n_slots, n4,
                                                                            out, accumulate);
  return cudaGetLastError();
}

cudaError_t launch_bwd_grad(const CUtensorMap& mapA, const CUtensorMap& mapB,
                            const CUtensorMap& mapG, int Mc, int V, int d, int tok0, const int* y,
                            const float* lse, const float* coef, const int* rowid, int grid,
                            int* sync, const DevCtl& ctl, cudaStream_t st) {
  EpiGrad::Params p{y, lse, coef, rowid, Mc, V, tok0};
  return launch_gemm<false, false, EpiGrad>(mapA, mapB, mapG, Mc, V, d, 2, p, grid, ctl, st,
                                            kGemmGrad, token_group(d), sync);
}

cudaError_t launch_bwd_dh(const CUtensorMap& mapA, const CUtensorMap& mapB, int Mc, int V, int d,
                          int tok0, const int* dst, float* dH, int accumulate, float* part,
                          int kb_part, int grid, int* sync, const DevCtl& ctl, cudaStream_t st) {
  const int k_blocks = (V + kBK - 1) / kBK;
  if (kb_part <= 0 || kb_part > k_blocks) kb_part = k_blocks;
  const int n_extra = split_k_parts(k_blocks, kb_part) - 1;
  if (n_extra > 0 && (part == nullptr || accumulate)) return cudaErrorInvalidValue;
  EpiRows::Params p{dst, dH, part, Mc, d, tok0, accumulate};
  cudaError_t e = launch_gemm<false, true, EpiRows>(mapA, mapB, mapA, Mc, d, V,
                                                    DPO_GROUP_DH > 0 ? 3 : 1, p, grid, ctl, st,
                                                    kGemmDH, DPO_GROUP_DH, sync, kb_part);
  if (e != cudaSuccess || n_extra == 0) return e;
  const long long n4 = static_cast<long long>(Mc) * (d / 4);
  k_dh_reduce<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(dH, part, dst, tok0, Mc, d,
                                                                       n_extra);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dw(const CUtensorMap& mapA, const CUtensorMap& mapB, int Mc, int V, int d,
                          float* dW, int accumulate, int grid, int* sync, const DevCtl& ctl,
                          cudaStream_t st) {
  EpiDW::Params p{dW, V, d, accumulate};
  return launch_gemm<true, true, EpiDW>(mapA, mapB, mapA, V, d, Mc, DPO_GROUP_DW > 0 ? 3 : 1, p, grid,
                                         ctl, st, kGemmDW, DPO_GROUP_DW, sync);
}

}  // namespace dpo
