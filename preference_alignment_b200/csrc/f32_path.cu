// SIMT route for DPO_F32 inputs (small problems; no tensor cores): fp32 inputs and
// products, fp64 accumulation of the long reductions (over the vocabulary and over
// the scored positions). Same quantities as the bf16 route: per scored position the
// log-sum-exp over the full vocabulary and the target logit, then
// dz = coef * (onehot - softmax) and its products with W and H. Each reduction runs
// in a fixed order.
#include <cmath>

#include "internal.h"

namespace dpo {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// z_v = h . W[v] for one vocab row, by one warp (lanes stride over d).
__device__ __forceinline__ float warp_dot(const float* __restrict__ h,
                                          const float* __restrict__ w, int d, int lane) {
  float a = 0.f;
  for (int k = lane; k < d; k += 32) a = fmaf(__ldg(h + k), __ldg(w + k), a);
  return warp_sum(a);
}

// One block per scored position; warp w handles vocab rows w, w + 8, ...
__global__ void __launch_bounds__(256) k_f32_fwd(const float* __restrict__ H,
                                                 const float* __restrict__ W, Sched s, int d,
                                                 int V, float2* __restrict__ part,
                                                 float* __restrict__ zy) {
  __shared__ float sm[8];
  __shared__ double ss[8];
  const int i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* h = H + static_cast<long long>(s.dst[i]) * d;
  const int y = s.y[i];
  // running (max, sum of exp) in fp64: a vocabulary of millions of terms would
  // swamp an fp32 running sum
  float m = -INFINITY;
  double sum = 0.0;
  for (int v = warp; v < V; v += 8) {
    const float z = warp_dot(h, W + static_cast<long long>(v) * d, d, lane);
    if (z > m) {
      sum = sum * exp(static_cast<double>(m) - z) + 1.0;
      m = z;
    } else {
      sum += exp(static_cast<double>(z) - m);
    }
    if (v == y && lane == 0) zy[i] = z;
  }
  if (lane == 0) {
    sm[warp] = m;
    ss[warp] = sum;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    double S = 0.0;
    for (int w = 0; w < 8; ++w) {
      if (sm[w] == -INFINITY) continue;            // warp saw no vocab row (V < 8)
      if (sm[w] > M) {
        S = S * exp(static_cast<double>(M) - sm[w]) + ss[w];
        M = sm[w];
      } else {
        S += ss[w] * exp(static_cast<double>(sm[w]) - M);
      }
    }
    // the combine stage takes (max, sum) in fp32; fold the sum's magnitude into the
    // max so the fp32 value stays near 1 and loses nothing
    const double ls = log(S);
    part[i] = make_float2(static_cast<float>(M + ls), 1.f);
  }
}

cudaError_t launch_f32_fwd(const float* H, const float* W, const Sched& s, int Nc, int d, int V,
                           float2* part, float* zy, cudaStream_t st) {
  if (Nc == 0) return cudaSuccess;
  k_f32_fwd<<<Nc, 256, 0, st>>>(H, W, s, d, V, part, zy);
  return cudaGetLastError();
}

// G[i, v] = coef_r * (1[v = y] - exp(z_v - lse)) for positions tok0 + i, i < Mc.
__global__ void __launch_bounds__(256) k_f32_grad(const float* __restrict__ H,
                                                  const float* __restrict__ W, Sched s, int tok0,
                                                  int d, int V, const float* __restrict__ lse,
                                                  const float* __restrict__ coef,
                                                  float* __restrict__ G) {
  const int i = blockIdx.x, gt = tok0 + i;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* h = H + static_cast<long long>(s.dst[gt]) * d;
  const int y = s.y[gt];
  const float cf = y != kTargetBad ? coef[s.rowid[gt]] : 0.f;
  const float l = lse[gt];
  float* g = G + static_cast<long long>(i) * V;
  for (int v = warp; v < V; v += 8) {
    const float z = warp_dot(h, W + static_cast<long long>(v) * d, d, lane);
    if (lane == 0) g[v] = cf * ((v == y ? 1.f : 0.f) - expf(z - l));
  }
}

cudaError_t launch_f32_grad(const float* H, const float* W, const Sched& s, int tok0, int Mc,
                            int d, int V, const float* lse, const float* coef, float* G,
                            cudaStream_t st) {
  if (Mc == 0) return cudaSuccess;
  k_f32_grad<<<Mc, 256, 0, st>>>(H, W, s, tok0, d, V, lse, coef, G);
  return cudaGetLastError();
}

// dH[dst[tok0 + i], k] = sum_v G[i, v] W[v, k]; one block per position.
__global__ void __launch_bounds__(256) k_f32_dh(const float* __restrict__ G,
                                                const float* __restrict__ W, Sched s, int tok0,
                                                int d, int V, float* __restrict__ dH) {
  const int i = blockIdx.x;
  const float* g = G + static_cast<long long>(i) * V;
  float* o = dH + static_cast<long long>(s.dst[tok0 + i]) * d;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    double a = 0.0;     // fp64: V products per element
    for (int v = 0; v < V; ++v)
      a = fma(static_cast<double>(__ldg(g + v)), static_cast<double>(__ldg(W + static_cast<long long>(v) * d + k)), a);
    o[k] = static_cast<float>(a);
  }
}

cudaError_t launch_f32_dh(const float* G, const float* W, const Sched& s, int tok0, int Mc, int d,
                          int V, float* dH, cudaStream_t st) {
  if (Mc == 0) return cudaSuccess;
  k_f32_dh<<<Mc, 256, 0, st>>>(G, W, s, tok0, d, V, dH);
  return cudaGetLastError();
}

// dW[v, k] (+)= sum_i G[i, v] H[dst[tok0 + i], k] for v in [v0, v0 + gridDim.x);
// one block per vocab row.
__global__ void __launch_bounds__(256) k_f32_dw(const float* __restrict__ G,
                                                const float* __restrict__ H, Sched s, int tok0,
                                                int Mc, int d, int V, int v0,
                                                float* __restrict__ dW, int accumulate) {
  const int v = v0 + blockIdx.x;
  float* o = dW + static_cast<long long>(v) * d;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    double a = 0.0;     // fp64: Mc products per element
    for (int i = 0; i < Mc; ++i)
      a = fma(static_cast<double>(__ldg(G + static_cast<long long>(i) * V + v)),
              static_cast<double>(__ldg(H + static_cast<long long>(s.dst[tok0 + i]) * d + k)), a);
    o[k] = accumulate ? o[k] + static_cast<float>(a) : static_cast<float>(a);
  }
}

cudaError_t launch_f32_dw(const float* G, const float* H, const Sched& s, int tok0, int Mc, int d,
                          int V, int v0, int v1, float* dW, int accumulate, cudaStream_t st) {
  if (v1 <= v0) return cudaSuccess;
  k_f32_dw<<<v1 - v0, 256, 0, st>>>(G, H, s, tok0, Mc, d, V, v0, dW, accumulate);
  return cudaGetLastError();
}

}  // namespace dpo
