// Host-side launchers shared between the library's translation units.
// Device code lives in the .cu files; this header only declares what the C ABI
// (api.cu) calls.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx_sm100.cuh"
#include "tile_config.h"

namespace dpo {

constexpr int kRowChunk = 1024;   // rows uploaded per k_upload_rows launch (kernel parameter)

// Longest reduction one tensor-core accumulator takes: the fp32 accumulation of a
// tcgen05 MMA chain rounds with a small bias per step, which grows linearly with K
// (measured: ~2% of dH at K = 2^24, negligible at 2^17). Longer reductions (dH over
// a vocabulary beyond it, dW over more scored positions) are split into chunks
// added together in fp32 by the epilogue.
constexpr int kMaxAccumK = 1 << 20;

// dH = dz . W runs over the whole vocabulary in one launch (or split over it into K parts,
// see the backward's plan), in chunks of kMaxAccumK columns only beyond that bound. With
// the static tile schedule, sequential launches of 16,384 columns had been ~0.5 % faster at
// the Llama-3.1-8B head (short K loops kept concurrent pairs close in K); with tiles claimed
// in raster order and dH's squarer raster, one launch won 5 of 6 alternating runs (0.2-0.4 %)
// and skips re-reading and re-writing dH per chunk (2.3 GB per step).

// Row table slice passed by value to k_upload_rows.
struct RowChunk {
  int row0;                       // first row of the slice
  int n;                          // rows in the slice
  int R;                          // total rows (row_start has R + 1 entries)
  int total;                      // Nc, written to row_start[R] by the last slice
  int rs[kRowChunk];              // packed offset of each row's first scored position
  int P[kRowChunk];               // prompt length of each row
};

// Target of a scored position, as k_prep stores it: the column in the call's
// vocabulary rows, or one of these (neither matches a vocabulary column).
constexpr int kTargetBad = -1;         // token outside [0, total vocabulary): scored 0, no gradient
constexpr int kTargetElsewhere = -2;   // valid token held by another vocabulary shard

// Device views of the per-call schedule held in the workspace.
struct Sched {
  const int* row_start;   // [R + 1] packed offset of row r's first scored position
  const int* prompt;      // [R]
  int* y;                 // [Nc] target token of each scored position (-1 = out of range)
  int* dst;               // [Nc] flat index r * L + t of each scored position
  int* rowid;             // [Nc] row of each scored position
  int* sync;              // [kSyncInts] the GEMM launches' tile claim counter
};

cudaError_t launch_upload_rows(const RowChunk& rc, int* row_start, int* prompt,
                               cudaStream_t st);

// Scored-position tables (y, dst, rowid) and, when Hp != nullptr, the packed
// bf16 copy of the scored H rows. The call's W holds vocabulary rows [v0, v0 + V) of
// a head of Vtot rows (v0 = 0, Vtot = V for the whole head).
cudaError_t launch_prep(const uint16_t* H, const int* tokens, const Sched& s, int R, int L, int d,
                        int V, int v0, int Vtot, int Nc, uint16_t* Hp, const DevCtl& ctl,
                        cudaStream_t st);

// Forward GEMM with the online log-sum-exp epilogue (bf16, tcgen05).
//   part[nt * ldp + i] = (max, sum exp(z - max)) of vocab tile nt for packed position i
//   zy[i] = z at the target column (written by the tile that holds it)
cudaError_t launch_fwd_lse(const CUtensorMap& mapA, const CUtensorMap& mapB, int Nc, int V,
                           int d, const int* y, float2* part, int ldp, float* zy, int grid,
                           int* sync, const DevCtl& ctl, cudaStream_t st);

// Combine the vocab-tile partials of each position into lse and lp = zy - lse;
// optionally the target logit, -inf when the target is not in the call's rows.
cudaError_t launch_combine(const float2* part, int ldp, int S, const float* zy, const int* y,
                           int Nc, float* lp, float* lse_out, float* zy_out, cudaStream_t st);

// Merge [n_shards, Nc] per-shard (lse, z_y) into lp and lse (shards in index order).
cudaError_t launch_shard_combine(const float* lse_parts, const float* zy_parts, int n_shards,
                                 int Nc, const int* y, float* lp, float* lse_out,
                                 cudaStream_t st);

// Per-row fp64 sum of lp over the row's scored positions; optional [R, L] token output.
cudaError_t launch_rowsum(const float* lp, const int* row_start, const int* prompt, int R, int L,
                          float* seq, float* tok_logp, cudaStream_t st);

// Backward (bf16): G = coef * (onehot - softmax) for packed positions [tok0, tok0 + Mc),
// stored through mapG (a [Mc, V] bf16 view of the dz chunk, 32 x 32 boxes, no swizzle).
cudaError_t launch_bwd_grad(const CUtensorMap& mapA, const CUtensorMap& mapB,
                            const CUtensorMap& mapG, int Mc, int V, int d, int tok0, const int* y,
                            const float* lse, const float* coef, const int* rowid, int grid,
                            int* sync, const DevCtl& ctl, cudaStream_t st);

// dH rows: out[dst[tok0 + i]] (+)= (G . W)[i]   (A = G K-major, B = W MN-major)
// kb_part > 0 splits K (the vocabulary) into parts of kb_part 64-column blocks run as
// separate work units of one launch; parts 1.. write fp32 partial sums to `part`
// ([parts - 1, Mc, d]) and a reduce kernel adds them to the rows in part order
// (split-K needs accumulate == 0).
cudaError_t launch_bwd_dh(const CUtensorMap& mapA, const CUtensorMap& mapB, int Mc, int V, int d,
                          int tok0, const int* dst, float* dH, int accumulate, float* part,
                          int kb_part, int grid, int* sync, const DevCtl& ctl, cudaStream_t st);

// dW (+)= G^T . Hp   (A = G MN-major, B = Hp MN-major)
cudaError_t launch_bwd_dw(const CUtensorMap& mapA, const CUtensorMap& mapB, int Mc, int V, int d,
                          float* dW, int accumulate, int grid, int* sync, const DevCtl& ctl,
                          cudaStream_t st);

// Data-parallel reduce-scatter fused into the dW GEMM (at most kMaxScatterRanks ranks):
// row v of this rank's dW contribution goes to recv[q] (rank q's buffer [n_ranks, rows_q,
// d], q = the owner of v) at slot `rank`; rank q owns rows [q * rows_per_rank, ...), the
// last rank the rest.
constexpr int kMaxScatterRanks = 8;   // DPO_MAX_SCATTER_RANKS
cudaError_t launch_bwd_dw_scatter(const CUtensorMap& mapA, const CUtensorMap& mapB, int Mc, int V,
                                  int d, float* const* recv, int n_ranks, int rank,
                                  int rows_per_rank, int grid, int* sync, const DevCtl& ctl,
                                  cudaStream_t st);
// out (+)= sum over the n_slots slots of recv ([n_slots, rows, d]), slots in order.
cudaError_t launch_dw_reduce_slots(const float* recv, int n_slots, int rows, int d, float* out,
                                   int accumulate, cudaStream_t st);

// Loss kernel (fp64 inside). pairs_total / nll_tokens_total: the whole data-parallel
// batch's pair count and chosen-token count (0: this call's own).
cudaError_t launch_loss(int B, int layout, const float* pol, const float* ref, double beta,
                        double grad_scale, int normalize, double nll_weight, const int* clen,
                        long long pairs_total, long long nll_tokens_total, float* loss, float* accuracy, float* margins, float* chosen_rewards,
                        float* rejected_rewards, float* weights, float* row_coef, float* nll,
                        cudaStream_t st);

// fp32 SIMT path.
cudaError_t launch_f32_fwd(const float* H, const float* W, const Sched& s, int Nc, int d, int V,
                           float2* part, float* zy, cudaStream_t st);
cudaError_t launch_f32_grad(const float* H, const float* W, const Sched& s, int tok0, int Mc,
                            int d, int V, const float* lse, const float* coef, float* G,
                            cudaStream_t st);
cudaError_t launch_f32_dh(const float* G, const float* W, const Sched& s, int tok0, int Mc, int d,
                          int V, float* dH, cudaStream_t st);
// dW rows [v0, v1) (dW points at the whole [V, d] array).
cudaError_t launch_f32_dw(const float* G, const float* H, const Sched& s, int tok0, int Mc, int d,
                          int V, int v0, int v1, float* dW, int accumulate, cudaStream_t st);

// 64-bit order-independent fingerprint of a device buffer into out (device).
cudaError_t launch_fingerprint(const void* data, unsigned long long bytes,
                               unsigned long long* out, int sms, cudaStream_t st);

// GEMM kernel selection (dpo_set_gemm_variant), two bits per GEMM kind: bit `kind` set
// runs that GEMM on the single-CTA kernel (clear: CTA pairs when the device can
// co-schedule them); bit 4 + kind set gives the pair kernel the static tile schedule
// (clear: tiles claimed in raster order).
enum GemmKind : int { kGemmForward = 0, kGemmGrad = 1, kGemmDH = 2, kGemmDW = 3 };
int gemm_variant();

// The CUDA context current on this thread (false if none or the driver call failed).
// Device addresses of the library's file-scope arrays are cached per context: a
// context that is destroyed and rebuilt reloads the module at new addresses.
bool current_context(void** ctx);

// Bounded-wait self-test: one CTA waits on an mbarrier nothing arrives on.
cudaError_t launch_wait_selftest(const DevCtl& ctl, cudaStream_t st);

// Logits-mean metrics (fp64 column sums of W and of each side's H rows, then their
// dot products): means[0] chosen, means[1] rejected. ws: logits_mean_bytes(d).
int logits_mean_splits(int d);
size_t logits_mean_bytes(int d);
cudaError_t launch_logits_mean(const void* H, const void* W, bool bf16, int R, int L, int d, int V,
                               int adjacent, void* ws, float* means, int sms, cudaStream_t st);

}  // namespace dpo
