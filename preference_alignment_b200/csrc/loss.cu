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
//
// Data-parallel shares: with pairs_total = B_g (the pairs of the whole batch over
// every rank) the batch means divide by B_g instead of this call's B, and with
// nll_tokens_total = N_g the NLL term divides by the whole batch's chosen tokens, so
// loss, accuracy, nll and row_coef are this rank's share of the global values: their
// sum over ranks equals the single-process result on the whole batch.
//
// Reference-free objective ("Run Distributed Full-Model DPO with PyTorch FSDP",
// "Where to Go Next"; no formula there): ref == NULL reads every reference sum as 0.
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
                                                  double gscale, int normalize, double nll_w,
                                                  const int* __restrict__ clen, double pairs_div,
                                                  double ntok_total, float* loss,
                                                  float* accuracy, float* margins,
                                                  float* chosen_rewards, float* rejected_rewards,
                                                  float* weights, float* row_coef, float* nll_out) {
  __shared__ double s_loss[256];
  __shared__ double s_acc[256];
  __shared__ double s_num[256];
  __shared__ double s_den[256];
  double lsum = 0.0, asum = 0.0, num = 0.0, den = 0.0;
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const int c = layout == 0 ? i : 2 * i;
    const int r = layout == 0 ? B + i : 2 * i + 1;
    // length normalisation: the loss sees S / C (0 for an empty row) instead of S
    double sc = 1.0, sr = 1.0;
    if (normalize) {
      sc = clen[c] > 0 ? 1.0 / clen[c] : 0.0;
      sr = clen[r] > 0 ? 1.0 / clen[r] : 0.0;
    }
    const double ref_c = ref != nullptr ? static_cast<double>(ref[c]) : 0.0;
    const double ref_r = ref != nullptr ? static_cast<double>(ref[r]) : 0.0;
    const double rho_c = static_cast<double>(pol[c]) * sc - ref_c * sc;
    const double rho_r = static_cast<double>(pol[r]) * sr - ref_r * sr;
    const double m = beta * (rho_c - rho_r);
    const double w = sigmoid_d(-m);
    lsum += softplus_d(-m);
    asum += m > 0.0 ? 1.0 : 0.0;
    if (nll_w != 0.0) {
      num += static_cast<double>(pol[c]);
      den += static_cast<double>(clen[c]);
    }
    if (margins) margins[i] = static_cast<float>(m);
    if (chosen_rewards) chosen_rewards[i] = static_cast<float>(beta * rho_c);
    if (rejected_rewards) rejected_rewards[i] = static_cast<float>(beta * rho_r);
    if (weights) weights[i] = static_cast<float>(w);
    if (row_coef) {
      const double k = gscale * beta * w / pairs_div;
      row_coef[c] = static_cast<float>(-k * sc);
      row_coef[r] = static_cast<float>(k * sr);
    }
  }
  s_loss[threadIdx.x] = lsum;
  s_acc[threadIdx.x] = asum;
  s_num[threadIdx.x] = num;
  s_den[threadIdx.x] = den;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      s_loss[threadIdx.x] += s_loss[threadIdx.x + w];
      s_acc[threadIdx.x] += s_acc[threadIdx.x + w];
      s_num[threadIdx.x] += s_num[threadIdx.x + w];
      s_den[threadIdx.x] += s_den[threadIdx.x + w];
    }
    __syncthreads();
  }
  // NLL of the chosen completions: mean over all their tokens, from the raw sums
  // (over the whole batch's chosen tokens when ntok_total > 0)
  const double ntok = ntok_total > 0.0 ? ntok_total : s_den[0];
  const double nll = (nll_w != 0.0 && ntok > 0.0) ? -s_num[0] / ntok : 0.0;
  if (threadIdx.x == 0) {
    *loss = static_cast<float>(s_loss[0] / pairs_div + nll_w * nll);
    if (accuracy) *accuracy = static_cast<float>(s_acc[0] / pairs_div);
    if (nll_out) *nll_out = static_cast<float>(nll);
  }
  if (row_coef && nll_w != 0.0 && ntok > 0.0) {
    // d(lambda * NLL)/d S_c = -lambda / ntok for every chosen row (same thread owns row c)
    const double k = gscale * nll_w / ntok;
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
      const int c = layout == 0 ? i : 2 * i;
      row_coef[c] = static_cast<float>(static_cast<double>(row_coef[c]) - k);
    }
  }
}

cudaError_t launch_loss(int B, int layout, const float* pol, const float* ref, double beta,
                        double grad_scale, int normalize, double nll_weight, const int* clen,
                        long long pairs_total, long long nll_tokens_total, float* loss,
                        float* accuracy, float* margins, float* chosen_rewards,
                        float* rejected_rewards, float* weights, float* row_coef, float* nll,
                        cudaStream_t st) {
  const double pairs_div = static_cast<double>(pairs_total > 0 ? pairs_total : B);
  k_dpo_loss<<<1, 256, 0, st>>>(B, layout, pol, ref, beta, grad_scale, normalize, nll_weight, clen,
                                pairs_div, static_cast<double>(nll_tokens_total), loss, accuracy,
                                margins, chosen_rewards, rejected_rewards, weights, row_coef, nll);
  return cudaGetLastError();
}

}  // namespace dpo
