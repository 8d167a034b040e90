// Forward kernels of the DPO head path:
//   k_upload_rows   row table (packed offsets, prompt lengths) into the workspace
//   k_prep          scored-position tables + packed bf16 copy of the scored H rows
//   k_tc_gemm<EpiLSE>  z = Hp . W^T on tcgen05, fp32 online log-sum-exp per vocab
//                   tile and the target logit pick, in the epilogue; logits never
//                   leave the SM
//   k_combine       per position: lse over vocab tiles (fixed order), lp = z_y - lse
//   k_rowsum        per row: fp64 sum of lp over the completion (fixed order)
//
// The step being computed is the pages' sequence log-prob: log-softmax over the
// full vocabulary, gather of the next token, completion mask, sum per row
// ("DPO Training on GPU, in depth", sequence_logps / _chunk_logps in "A
// training configuration that fits"; sums kept in fp32 or wider as its section
// "A worked example of the numbers" asks).
#include <cfloat>
#include <cmath>

#include "internal.h"
#include "gemm_launch.cuh"

namespace dpo {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ row table upload
__global__ void k_upload_rows(const __grid_constant__ RowChunk rc, int* row_start, int* prompt) {
  for (int i = threadIdx.x; i < rc.n; i += blockDim.x) {
    row_start[rc.row0 + i] = rc.rs[i];
    prompt[rc.row0 + i] = rc.P[i];
  }
  if (threadIdx.x == 0 && rc.row0 + rc.n == rc.R) row_start[rc.R] = rc.total;
}

cudaError_t launch_upload_rows(const RowChunk& rc, int* row_start, int* prompt,
                               cudaStream_t st) {
  k_upload_rows<<<1, 256, 0, st>>>(rc, row_start, prompt);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ prep
// One warp per scored position i: find its row (last r with row_start[r] <= i),
// its position t = P_r - 1 + (i - row_start[r]) and target tokens[r, t + 1].
__global__ void __launch_bounds__(256) k_prep(const uint16_t* __restrict__ H,
                                              const int* __restrict__ tokens, Sched s, int R,
                                              int L, int d, int V, int v0, int Vtot, int Nc,
                                              uint16_t* __restrict__ Hp, DevCtl ctl) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp;
  if (i >= Nc) return;
  int lo = 0, hi = R;                       // invariant: row_start[lo] <= i < row_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(s.row_start + mid) <= i) lo = mid; else hi = mid;
  }
  const int r = lo;
  const int t = __ldg(s.prompt + r) - 1 + (i - __ldg(s.row_start + r));
  const long long src = static_cast<long long>(r) * L + t;
  if (lane == 0) {
    const int tgt = __ldg(tokens + src + 1);
    const bool ok = tgt >= 0 && tgt < Vtot;
    if (!ok) record_status(ctl, kStatusBadTarget);
    const int yl = tgt - v0;            // column in this call's vocabulary rows [v0, v0 + V)
    s.y[i] = !ok ? kTargetBad : (yl >= 0 && yl < V ? yl : kTargetElsewhere);
    s.dst[i] = static_cast<int>(src);
    s.rowid[i] = r;
  }
  if (Hp != nullptr) {
    const uint4* a = reinterpret_cast<const uint4*>(H + src * d);
    uint4* b = reinterpret_cast<uint4*>(Hp + static_cast<long long>(i) * d);
    for (int k = lane; k < d / 8; k += 32) b[k] = __ldg(a + k);
  }
}

cudaError_t launch_prep(const uint16_t* H, const int* tokens, const Sched& s, int R, int L, int d,
                        int V, int v0, int Vtot, int Nc, uint16_t* Hp, const DevCtl& ctl,
                        cudaStream_t st) {
  if (Nc == 0) return cudaSuccess;
  k_prep<<<(Nc + 7) / 8, 256, 0, st>>>(H, tokens, s, R, L, d, V, v0, Vtot, Nc, Hp, ctl);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ GEMM epilogue: online LSE
// One thread = one packed position (accumulator row), 256 vocab columns per tile.
struct EpiLSE {
  static constexpr bool kStaging = false;   // stores go straight to global memory
  static constexpr bool kSystemFence = false;
  struct Params {
    const int* y;
    float2* part;
    float* zy;
    int Nc, V, ldp;
  };
  int tok, nt, yl, vlim;
  bool valid;
  float mx, s, zyv;

  __device__ __forceinline__ void begin(const Params& p, int m_row, int nt_, int,
                                        const EpiCtx&) {
    nt = nt_;
    tok = m_row;
    valid = tok < p.Nc;
    const int vbase = nt * kBN;
    yl = valid ? __ldg(p.y + tok) - vbase : -1;   // negative targets never match
    vlim = p.V - vbase;
    mx = -INFINITY;
    s = 0.f;
    zyv = 0.f;
  }

  __device__ __forceinline__ void chunk(const Params& p, int c, const uint32_t (&v)[32]) {
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(v[j]);
    if (vlim < kBN) {                      // last vocab tile: columns >= V are padding
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c * 32 + j >= vlim) x[j] = -INFINITY;
    }
    float cm = x[0];
#pragma unroll
    for (int j = 1; j < 32; ++j) cm = fmaxf(cm, x[j]);
    const float nm = fmaxf(mx, cm);
    const float nm2 = nm * kLog2e;
    float acc = s * ex2_approx(fmaf(mx, kLog2e, -nm2));
#pragma unroll
    for (int j = 0; j < 32; ++j) acc += ex2_approx(fmaf(x[j], kLog2e, -nm2));
    s = acc;
    mx = nm;
    const int jj = yl - c * 32;
    if (static_cast<unsigned>(jj) < 32u) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j == jj) zyv = x[j];
    }
  }

  __device__ __forceinline__ void end(const Params& p) {
    if (!valid) return;
    p.part[static_cast<long long>(nt) * p.ldp + tok] = make_float2(mx, s);
    if (yl >= 0 && yl < kBN && yl < vlim) p.zy[tok] = zyv;
  }
};

cudaError_t launch_fwd_lse(const CUtensorMap& mapA, const CUtensorMap& mapB, int Nc, int V,
                           int d, const int* y, float2* part, int ldp, float* zy, int grid,
                           int* sync, const DevCtl& ctl, cudaStream_t st) {
  if (Nc == 0) return cudaSuccess;
  EpiLSE::Params p{y, part, zy, Nc, V, ldp};
  // order 0: all token tiles of one vocab tile run together, so each W tile is
  // read from HBM once and served to the other CTAs from L2
  return launch_gemm<false, false, EpiLSE>(mapA, mapB, mapA, Nc, V, d, 2, p, grid, ctl, st,
                                           kGemmForward, token_group(d), sync);
}

// ------------------------------------------------------------------ combine
// lse_i = M + log(sum_s s_s * exp(m_s - M)) over the vocab-tile partials of
// position i, then lp_i = z_y - lse_i. A block covers 32 positions; its 8 warps
// take the partials s = g, g + 8, ... (warp g), reading 32 consecutive positions
// per partial (coalesced), and the 8 running (max, sum) pairs are merged in warp
// order. The assignment and the merge order are fixed, so the result is
// bit-identical from run to run.
__device__ __forceinline__ void lse_merge(float& M, float& S, float m, float s) {
  if (m == -INFINITY) return;
  if (m > M) {
    S = S * expf(M - m) + s;
    M = m;
  } else {
    S += s * expf(m - M);
  }
}

__global__ void __launch_bounds__(256) k_combine(const float2* __restrict__ part, int ldp, int S,
                                                 const float* __restrict__ zy,
                                                 const int* __restrict__ y, int Nc,
                                                 float* __restrict__ lp,
                                                 float* __restrict__ lse_out,
                                                 float* __restrict__ zy_out) {
  __shared__ float sm[8][32], ss[8][32];
  const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 32 + lane;
  float M = -INFINITY, sum = 0.f;
  if (i < Nc) {
    int s = g;
    for (; s + 24 < S; s += 32) {          // four independent loads in flight
      const float2 q0 = __ldg(part + static_cast<long long>(s) * ldp + i);
      const float2 q1 = __ldg(part + static_cast<long long>(s + 8) * ldp + i);
      const float2 q2 = __ldg(part + static_cast<long long>(s + 16) * ldp + i);
      const float2 q3 = __ldg(part + static_cast<long long>(s + 24) * ldp + i);
      lse_merge(M, sum, q0.x, q0.y);
      lse_merge(M, sum, q1.x, q1.y);
      lse_merge(M, sum, q2.x, q2.y);
      lse_merge(M, sum, q3.x, q3.y);
    }
    for (; s < S; s += 8) {
      const float2 q = __ldg(part + static_cast<long long>(s) * ldp + i);
      lse_merge(M, sum, q.x, q.y);
    }
  }
  sm[g][lane] = M;
  ss[g][lane] = sum;
  __syncthreads();
  if (g == 0 && i < Nc) {
    float Mt = sm[0][lane], St = ss[0][lane];
    for (int h = 1; h < 8; ++h) lse_merge(Mt, St, sm[h][lane], ss[h][lane]);
    const float lse = Mt + logf(St);
    const bool here = __ldg(y + i) >= 0;
    lp[i] = here ? __ldg(zy + i) - lse : 0.f;
    if (lse_out != nullptr) lse_out[i] = lse;
    if (zy_out != nullptr) zy_out[i] = here ? __ldg(zy + i) : -INFINITY;
  }
}

cudaError_t launch_combine(const float2* part, int ldp, int S, const float* zy, const int* y,
                           int Nc, float* lp, float* lse_out, float* zy_out, cudaStream_t st) {
  if (Nc == 0) return cudaSuccess;
  k_combine<<<(Nc + 31) / 32, 256, 0, st>>>(part, ldp, S, zy, y, Nc, lp, lse_out, zy_out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ vocabulary shards
// Merge the per-shard results of each position (shards in index order, fp64):
//   lse = M + log(sum_k exp(lse_k - M)),  M = max_k lse_k
//   z_y = the one finite shard value (the shard that holds the target)
//   lp  = z_y - lse, or 0 for a bad target (y = kTargetBad)
// One thread per position; the shard order is fixed, so every rank that merges the
// same gathered values gets the same bits.
__global__ void __launch_bounds__(256) k_shard_combine(const float* __restrict__ lse_parts,
                                                       const float* __restrict__ zy_parts,
                                                       int n_shards, int Nc,
                                                       const int* __restrict__ y,
                                                       float* __restrict__ lp,
                                                       float* __restrict__ lse_out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= Nc) return;
  double M = -INFINITY;
  float zyv = -INFINITY;
  for (int k = 0; k < n_shards; ++k) {
    M = fmax(M, static_cast<double>(__ldg(lse_parts + static_cast<long long>(k) * Nc + i)));
    zyv = fmaxf(zyv, __ldg(zy_parts + static_cast<long long>(k) * Nc + i));
  }
  double S = 0.0;
  for (int k = 0; k < n_shards; ++k) {
    const double l = __ldg(lse_parts + static_cast<long long>(k) * Nc + i);
    if (l != -INFINITY) S += exp(l - M);
  }
  const float lse = static_cast<float>(M + log(S));
  lp[i] = __ldg(y + i) == kTargetBad ? 0.f : zyv - lse;
  if (lse_out != nullptr) lse_out[i] = lse;
}

cudaError_t launch_shard_combine(const float* lse_parts, const float* zy_parts, int n_shards,
                                 int Nc, const int* y, float* lp, float* lse_out,
                                 cudaStream_t st) {
  if (Nc == 0) return cudaSuccess;
  k_shard_combine<<<(Nc + 255) / 256, 256, 0, st>>>(lse_parts, zy_parts, n_shards, Nc, y, lp,
                                                    lse_out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ row sums
// One block per row; each thread sums a fixed stride of the row in fp64, then a
// fixed-shape tree combines the 256 partials: the result does not depend on timing.
__global__ void __launch_bounds__(256) k_rowsum(const float* __restrict__ lp,
                                                const int* __restrict__ row_start,
                                                const int* __restrict__ prompt, int L,
                                                float* __restrict__ seq,
                                                float* __restrict__ tok_logp) {
  __shared__ double red[256];
  const int r = blockIdx.x;
  const int a = row_start[r], b = row_start[r + 1];
  double acc = 0.0;
  for (int i = a + threadIdx.x; i < b; i += blockDim.x) acc += static_cast<double>(lp[i]);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) seq[r] = static_cast<float>(red[0]);
  if (tok_logp != nullptr) {
    const int t0 = prompt[r] - 1, n = b - a;
    float* out = tok_logp + static_cast<long long>(r) * L;
    for (int t = threadIdx.x; t < L; t += blockDim.x)
      out[t] = (t >= t0 && t < t0 + n) ? lp[a + t - t0] : 0.f;
  }
}

cudaError_t launch_rowsum(const float* lp, const int* row_start, const int* prompt, int R, int L,
                          float* seq, float* tok_logp, cudaStream_t st) {
  k_rowsum<<<R, 256, 0, st>>>(lp, row_start, prompt, L, seq, tok_logp);
  return cudaGetLastError();
}

}  // namespace dpo
