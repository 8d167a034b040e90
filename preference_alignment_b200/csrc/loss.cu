// Sigmoid DPO loss over B pairs, fp64 inside, fp32 out.
//
// Per pair: rho_c = pi_c - ref_c, rho_r = pi_r - ref_r (log-ratios first),
// rewards beta * rho, margin m = beta * (rho_c - rho_r), loss term
// -log sigmoid(m) = softplus(-m), gradient weight sigmoid(-m); the batch loss is
// the mean over pairs and the accuracy the fraction with m > 0.
// ("DPO Training on GPU, in depth": the loss formula in "What one DPO step
// computes", rewards/margin/weight in "A worked example of the numbers", the
// mean and reward accuracy of dpo_step in "A training configuration that fits".)
// row_coef[row] = d(grad_scale * loss)/d pi_row = -/+ grad_scale * beta * w / B.
#include <cmath>

#include "internal.h"

namespace dpo {

__device__ __forceinline__ double softplus_d(double x) {   // log(1 + e^x), no overflow
  return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

__device__ __forceinline__ double sigmoid_d(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  const double e = exp(x);
  return e / (1.0 + e);
}

__global__ void __launch_bounds__(256) k_dpo_loss(int B, int layout, const float* __restrict__ pol,
                                                  const float* __restrict__ ref, double beta,
                                                  double gscale, float* loss, float* accuracy,
                                                  float* margins, float* chosen_rewards,
                                                  float* rejected_rewards, float* weights,
                                                  float* row_coef) {
  __shared__ double s_loss[256];
  __shared__ double s_acc[256];
  double lsum = 0.0, asum = 0.0;
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const int c = layout == 0 ? i : 2 * i;
    const int r = layout == 0 ? B + i : 2 * i + 1;
    const double rho_c = static_cast<double>(pol[c]) - static_cast<double>(ref[c]);
    const double rho_r = static_cast<double>(pol[r]) - static_cast<double>(ref[r]);
    const double m = beta * (rho_c - rho_r);
    const double w = sigmoid_d(-m);
    lsum += softplus_d(-m);
    asum += m > 0.0 ? 1.0 : 0.0;
    if (margins) margins[i] = static_cast<float>(m);
    if (chosen_rewards) chosen_rewards[i] = static_cast<float>(beta * rho_c);
    if (rejected_rewards) rejected_rewards[i] = static_cast<float>(beta * rho_r);
    if (weights) weights[i] = static_cast<float>(w);
    if (row_coef) {
      const double k = gscale * beta * w / B;
      row_coef[c] = static_cast<float>(-k);
      row_coef[r] = static_cast<float>(k);
    }
  }
  s_loss[threadIdx.x] = lsum;
  s_acc[threadIdx.x] = asum;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      s_loss[threadIdx.x] += s_loss[threadIdx.x + w];
      s_acc[threadIdx.x] += s_acc[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *loss = static_cast<float>(s_loss[0] / B);
    if (accuracy) *accuracy = static_cast<float>(s_acc[0] / B);
  }
}

cudaError_t launch_loss(int B, int layout, const float* pol, const float* ref, double beta,
                        double grad_scale, float* loss, float* accuracy, float* margins,
                        float* chosen_rewards, float* rejected_rewards, float* weights,
                        float* row_coef, cudaStream_t st) {
  k_dpo_loss<<<1, 256, 0, st>>>(B, layout, pol, ref, beta, grad_scale, loss, accuracy, margins,
                                chosen_rewards, rejected_rewards, weights, row_coef);
  return cudaGetLastError();
}

}  // namespace dpo
