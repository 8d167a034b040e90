/*
 * libdpo: the data-parallel hot path of Direct Preference Optimization (DPO) on
 * NVIDIA B200 (sm_100a), as a C ABI.
 *
 * The path, for a batch of 2B rows (chosen and rejected completions of B
 * prompts), each row = prompt | completion | pad:
 *   1. LM-head logits z = h . W^T for every scored position (never stored),
 *   2. log-softmax over the full vocabulary and the target-token pick,
 *   3. per-row sum of the completion tokens' log-probabilities, in fp32,
 *   4. the sigmoid DPO loss from policy and reference sums,
 *   5. the backward of (4) through (1)-(3) to dH and dW.
 * ("DPO Training on GPU, in depth", sections "What one DPO step computes",
 *  "A worked example of the numbers" and the hand-written sequence_logps /
 *  dpo_step in "A training configuration that fits".)
 *
 * Conventions shared by every call
 *   - Every buffer is owned by the caller. The library makes no device-memory
 *     allocation calls; each call that needs scratch takes a caller-provided
 *     workspace whose size dpo_workspace_size() returns (the one exception,
 *     dpo_seq_logprobs_noalloc, uses a scratch array compiled into the library).
 *   - Device pointers must point to device memory of the current CUDA device.
 *     "host" marks the few arguments read from host memory during the call.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). All device
 *     work is enqueued on it; calls return without waiting for the GPU, except
 *     dpo_check(), which synchronises the stream.
 *   - Errors the host can see (bad sizes, null pointers, misalignment, too
 *     small a workspace, unsupported dtype) are returned before any launch and
 *     leave every output untouched.
 *   - Errors only the GPU can see (a target token outside [0, V), a pipeline
 *     wait that exceeded its time budget) are recorded in a per-device status
 *     word that dpo_check() reads and clears. A bad target is scored as 0.
 *   - The forward is deterministic: the same inputs give bit-identical outputs.
 *
 * Row model (all calls that take a dpo_batch)
 *   Row r has prompt length P_r = prompt_len[r] >= 1 and completion length
 *   C_r = completion_len[r] >= 0 with P_r + C_r <= L. Completion tokens are
 *   tokens[r, P_r .. P_r + C_r - 1]; token j is predicted by position j - 1, so
 *   the scored positions are t in [P_r - 1, P_r + C_r - 1) and position t
 *   scores tokens[r, t + 1] ("DPO Training on GPU, in depth", sequence_logps:
 *   logits[:, :-1] pair with labels[:, 1:] and mask[:, 1:]). Positions outside
 *   that range (prompt, pad, the last position) contribute nothing.
 *   Nc = sum_r C_r is the number of scored positions.
 */
#ifndef LIBDPO_DPO_H
#define LIBDPO_DPO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DPO_OK = 0,
  DPO_ERR_INVALID_ARG = 1,  /* null pointer, size out of range, P_r/C_r do not fit L   */
  DPO_ERR_UNSUPPORTED = 2,  /* dtype (fp16 is refused), d not a multiple of 8, ...      */
  DPO_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                        */
  DPO_ERR_TIMEOUT = 4,      /* device: a pipeline wait ran out of its time budget       */
  DPO_ERR_BAD_TARGET = 5,   /* device: a scored target token was outside [0, V)         */
  DPO_ERR_WORKSPACE = 6     /* workspace null, too small or not 256-byte aligned        */
} dpo_status;

/* Element type of H and W. fp16 is refused: the pages' recipe raises on full
 * fp16 training because log-prob ratios leave fp16's range ("Run Distributed
 * Full-Model DPO with PyTorch FSDP", "What to Watch Out For"). DPO_BF16 runs on
 * the tcgen05 tensor cores with fp32 accumulation; DPO_F32 runs an exact-fp32
 * SIMT path meant for small problems. */
typedef enum { DPO_BF16 = 0, DPO_F32 = 1, DPO_F16 = 2 } dpo_dtype;

/* Which rows form pair i. HALVES: chosen row i, rejected row B + i (the
 * concatenated [2B, L] batch, "Run Distributed Full-Model DPO with PyTorch
 * FSDP", Step 4). ADJACENT: chosen row 2i, rejected row 2i + 1 (pairs next to
 * each other in the micro batch, Megatron-Bridge PR 6092 changelog). */
typedef enum { DPO_PAIRS_HALVES = 0, DPO_PAIRS_ADJACENT = 1 } dpo_layout;

typedef struct {
  int32_t R;                     /* rows (2B for a preference batch), 1 <= R <= 65535  */
  int32_t L;                     /* positions per row, 2 <= L                           */
  int32_t d;                     /* hidden size; a multiple of 8, 8 <= d <= 65536       */
  int32_t V;                     /* vocabulary size, 1 <= V <= 2^24                     */
  int32_t dtype;                 /* dpo_dtype of H and W                                */
  const void* H;                 /* device [R, L, d] row-major hidden states (LM-head
                                    input); 16-byte aligned                             */
  const void* W;                 /* device [V, d] row-major LM-head weight (policy or
                                    reference), logits = H . W^T; 16-byte aligned       */
  const int32_t* tokens;         /* device [R, L] token ids                             */
  const int32_t* prompt_len;     /* host [R], P_r >= 1                                  */
  const int32_t* completion_len; /* host [R], C_r >= 0, P_r + C_r <= L                  */
} dpo_batch;

/* Workspace bytes that dpo_seq_logprobs (fwd_bytes) and dpo_backward
 * (bwd_bytes) need for this batch. Either output pointer may be NULL.
 * bwd_bytes is the size that lets the backward run in one token chunk; a
 * smaller workspace of at least *bwd_min_bytes (may be NULL) makes it run in
 * several chunks. Pure host function. */
dpo_status dpo_workspace_size(const dpo_batch* batch, size_t* fwd_bytes, size_t* bwd_bytes,
                              size_t* bwd_min_bytes);

/* Per-row completion log-prob sums (steps 1-3), for the policy or the
 * reference, with or without what the backward needs.
 *   seq_logp  device [R] fp32, out: S_r = sum over scored t of log p(tokens[r,t+1])
 *   tok_logp  device [R, L] fp32 or NULL, out: log p at scored positions, 0 elsewhere
 *   lse_state device [Nc] fp32, out: log-sum-exp of each scored position in row
 *             order; required when want_grad != 0 (dpo_backward reads it), else
 *             may be NULL
 *   ws        device workspace of ws_bytes >= fwd_bytes, 256-byte aligned
 * Sums carry no beta, so one scoring pass serves every beta (offline reference
 * scoring: Megatron-Bridge PR 6092, "Why the reference is scored offline"); rows
 * keep their order so stored sums can be joined back by row index. */
dpo_status dpo_seq_logprobs(const dpo_batch* batch, int want_grad, float* seq_logp,
                            float* tok_logp, float* lse_state, void* ws, size_t ws_bytes,
                            void* stream);

/* Sigmoid DPO loss and its metrics (step 4), for B pairs.
 *   pol, ref        device [2B] fp32 sequence sums of policy and reference, in `layout`
 *   beta            the DPO temperature (> 0)
 *   grad_scale      factor folded into row_coef (e.g. 1/accumulation steps)
 *   loss            device [1]: mean over pairs of -log sigmoid(margin)
 *   accuracy        device [1]: fraction of pairs with margin > 0 (strict)
 *   margins         device [B]: beta * ((pol_c - ref_c) - (pol_r - ref_r))
 *   chosen_rewards  device [B]: beta * (pol_c - ref_c)
 *   rejected_rewards device [B]: beta * (pol_r - ref_r)
 *   weights         device [B]: sigmoid(-margin), the per-pair gradient weight
 *   row_coef        device [2B] or NULL: d(grad_scale * loss) / d pol[row]
 * ("DPO Training on GPU, in depth": the loss formula, the worked example's
 *  rewards, margin and sigmoid(-margin) weight, and dpo_step's mean loss and
 *  reward accuracy.) Computed in fp64 on the device, stored as fp32. Any of the
 * outputs except loss may be NULL. */
dpo_status dpo_loss(int32_t B, int32_t layout, const float* pol, const float* ref, float beta,
                    float grad_scale, float* loss, float* accuracy, float* margins,
                    float* chosen_rewards, float* rejected_rewards, float* weights,
                    float* row_coef, void* stream);

/* Loss variants on the same per-row sums ("Run Distributed Full-Model DPO with
 * PyTorch FSDP", Step 4: un-averaged sums let the loss use length-normalised or
 * sum-based rewards; "DPO Training on GPU, in depth", failure modes: length-
 * normalised variants and an added SFT term; the video transcript: total loss =
 * DPO loss + lambda * a standard language-modelling NLL on the chosen responses).
 *   normalize       1: the loss, rewards and margins use S_r / C_r (the average
 *                   completion log-prob; 0 for C_r = 0) for policy and reference
 *   nll_weight      lambda >= 0: add lambda * NLL, NLL = -(sum of the chosen rows'
 *                   policy sums) / (their total completion length), i.e. the mean
 *                   over all chosen completion tokens
 *   completion_len  device [2B] int32 C_r in the row layout; required when
 *                   normalize != 0 or nll_weight > 0, else may be NULL
 *   pairs_total     data parallelism: when > 0 the batch means (loss, accuracy,
 *                   row_coef) divide by B_g = pairs_total, the pair count summed over
 *                   every rank, instead of this call's B (B_g < B is refused)
 *   nll_tokens_total  when > 0 the NLL divides by N_g, the chosen completion tokens
 *                   summed over every rank, instead of this call's own count
 * With both set, loss, accuracy, nll and row_coef are this rank's share of the
 * whole batch's values: summing them over the ranks (one all-reduce) gives the
 * single-process result on the whole batch, for unequal shards too ("Run
 * Distributed Full-Model DPO with PyTorch FSDP", Step 1: every rank holds part of
 * the global batch). Margins, rewards and weights are per pair and unchanged.
 *   reference_free  1: the reference-free objective ("Run Distributed Full-Model DPO
 *                   with PyTorch FSDP", "Where to Go Next": it skips the frozen
 *                   reference model; the pages give no formula): the reference sums
 *                   are read as 0, so rewards are beta * pi (normalised when asked)
 *                   and the margin beta * (pi_c - pi_r); ref is not read and may be
 *                   NULL. Composes with the options above.
 * Zero-initialise the struct (dpo_loss_options o = {0};) and set the fields wanted: zero
 * is "off" for every field. The struct grew with reference_free (library version 0.3.0);
 * a caller built against an older header passes a shorter struct, so check
 * dpo_version() >= 300 before relying on this layout. */
typedef struct {
  int32_t normalize;
  float nll_weight;
  const int32_t* completion_len;
  int32_t pairs_total;      /* 0, or B_g >= B: the pairs of the whole data-parallel batch */
  int64_t nll_tokens_total; /* 0, or N_g >= 0: the whole batch's chosen completion tokens */
  int32_t reference_free;   /* 0, or 1: no reference model (ref may be NULL) */
} dpo_loss_options;

/* dpo_loss with the variants above (opt may be NULL: then it equals dpo_loss).
 * ref is required (DPO_ERR_INVALID_ARG when NULL) unless opt->reference_free is set.
 * row_coef stays d(grad_scale * loss)/d pol[row] and feeds dpo_backward as is.
 *   nll   device [1] or NULL: the NLL value (0 when nll_weight is 0) */
dpo_status dpo_loss_ex(int32_t B, int32_t layout, const float* pol, const float* ref, float beta,
                       float grad_scale, const dpo_loss_options* opt, float* loss,
                       float* accuracy, float* margins, float* chosen_rewards,
                       float* rejected_rewards, float* weights, float* row_coef, float* nll,
                       void* stream);

/* Backward of sum_r row_coef[r] * seq_logp[r] (step 5) to H and W.
 *   lse_state   device [Nc] fp32 from dpo_seq_logprobs(want_grad=1) on the same batch
 *   row_coef    device [R] fp32, d(objective)/d seq_logp[r] (dpo_loss writes it)
 *   dH          device [R, L, d] fp32, 16-byte aligned, out: fully written; 0 at
 *               unscored positions
 *   dW          device [V, d] fp32, 16-byte aligned, out: dW = sum_t dz_t^T h_t, or
 *               dW += that when accumulate_dW != 0 (gradient accumulation over
 *               micro-batches)
 *   ws          device workspace, >= bwd_min_bytes, 256-byte aligned
 * with dz[t, v] = row_coef[r(t)] * (1[v = tokens[r, t+1]] - softmax(z_t)[v]). The
 * logits are recomputed tile by tile. dH may be NULL (only dW is formed).
 * dW may be NULL too: then the whole batch must fit one workspace chunk (ws_bytes >=
 * bwd_bytes and Nc <= 2^20, else DPO_ERR_WORKSPACE) and the logit gradient dz stays
 * in the workspace, where dpo_backward_dw and dpo_backward_dh read it. */
dpo_status dpo_backward(const dpo_batch* batch, const float* lse_state, const float* row_coef,
                        float* dH, float* dW, int accumulate_dW, void* ws, size_t ws_bytes,
                        void* stream);

/* Rows [v_begin, v_end) of dW from the dz that a preceding dpo_backward(dW = NULL) on
 * the same batch left in ws (ws unchanged since). Splitting dW by vocabulary rows
 * lets a data-parallel caller start the all-reduce of each finished block of rows
 * while the next block is computed ("Run Distributed Full-Model DPO with PyTorch
 * FSDP", Step 1: the ranks' gradients are summed).
 *   v_begin, v_end  0 <= v_begin <= v_end <= V; v_begin a multiple of 8, v_end a
 *                   multiple of 8 or V
 *   dW              device [V, d] fp32, the whole array: only the range's rows are
 *                   written (or accumulated when accumulate_dW != 0)
 *   max_sms         0: use every SM; > 0: at most that many, leaving the others free
 *                   for kernels of other streams (a collective) to run beside it
 * Every row is computed with the same order of operations as in dpo_backward, so the
 * result does not depend on the split or on max_sms. Errors: DPO_ERR_INVALID_ARG for
 * a bad range, NULL dW or max_sms < 0; DPO_ERR_WORKSPACE when ws cannot hold the whole
 * batch's dz. */
dpo_status dpo_backward_dw(const dpo_batch* batch, int32_t v_begin, int32_t v_end, float* dW,
                           int accumulate_dW, int32_t max_sms, void* ws, size_t ws_bytes,
                           void* stream);

/* dH (device [R, L, d] fp32, fully written, 0 at unscored positions) from the dz a
 * preceding dpo_backward(dW = NULL) left in ws; max_sms and errors as for
 * dpo_backward_dw. The same values as dpo_backward's dH. */
dpo_status dpo_backward_dh(const dpo_batch* batch, float* dH, int32_t max_sms, void* ws,
                           size_t ws_bytes, void* stream);

/* ---- Data-parallel exchange fused into the dW GEMM ---------------------------
 * With the pairs split across ranks (each rank its own pairs, the same W), dW is the
 * sum over ranks of each rank's dz_r^T . Hp_r. As a reduce-scatter fused into the dW
 * GEMM: rank q owns a block of W's rows; every rank forms its whole contribution and
 * its GEMM epilogue stores each finished row straight into the owner's receive buffer,
 * in this rank's slot (another process's buffer, mapped with dpo_ipc_import: peer
 * memory over NVLink when the ranks run on different GPUs), so the transfer proceeds
 * tile by tile while the GEMM runs. After a barrier on every rank (an all-reduce of one
 * number on the same stream is one), each owner adds its slots in rank order
 * (dpo_dw_reduce_slots) and holds its block of the summed dW, as a sharded optimiser
 * needs ("Run Distributed Full-Model DPO with PyTorch FSDP", Step 1). Deterministic:
 * the sum is taken in rank order. */
#define DPO_MAX_SCATTER_RANKS 8
typedef struct {
  int32_t n_ranks;          /* 1 .. DPO_MAX_SCATTER_RANKS                                 */
  int32_t rank;             /* this rank, 0 .. n_ranks - 1                                */
  int32_t rows_per_rank;    /* rank q < n_ranks - 1 owns W rows [q * rows_per_rank, +rows_per_rank);
                               the last rank owns the rest (at least one row)             */
  float* recv[DPO_MAX_SCATTER_RANKS];  /* recv[q]: rank q's receive buffer [n_ranks, rows_q,
                               d] fp32, 16-byte aligned, as this process addresses it     */
} dpo_dw_scatter;

/* This rank's contribution to dW (the dz that a preceding dpo_backward(dW = NULL) left in
 * ws, times the batch's packed H), each row stored into its owner's buffer at slot
 * `rank` (recv[q] + (rank * rows_q + row - q * rows_per_rank) * d). bf16 batches only
 * (DPO_ERR_UNSUPPORTED otherwise). The epilogue fences its stores at system scope before
 * the kernel ends. max_sms and workspace errors as for dpo_backward_dw; a bad scatter
 * description is DPO_ERR_INVALID_ARG. A batch with no scored position zeroes its slots. */
dpo_status dpo_backward_dw_scatter(const dpo_batch* batch, const dpo_dw_scatter* scatter,
                                   int32_t max_sms, void* ws, size_t ws_bytes, void* stream);

/* The owner's side: dW_shard (+)= slot 0 + slot 1 + ... in slot order, over a receive
 * buffer recv [n_slots, rows, d] fp32 (both 16-byte aligned; d a multiple of 8). Call it
 * after every rank's dpo_backward_dw_scatter has completed (a barrier). */
dpo_status dpo_dw_reduce_slots(const float* recv, int32_t n_slots, int32_t rows, int32_t d,
                               float* dW_shard, int accumulate, void* stream);

/* CUDA IPC of a device buffer between processes (the receive buffers above).
 * dpo_ipc_export: the handle of the allocation that holds ptr (this process's device
 * memory from cudaMalloc, as PyTorch's default allocator makes it; memory mapped through
 * the virtual-memory API, such as PyTorch's expandable segments, is refused with
 * DPO_ERR_CUDA), and ptr's byte offset in it; DPO_ERR_INVALID_ARG when ptr is not device
 * memory of this process. dpo_ipc_import (in another process): map that allocation, peer
 * access enabled; the buffer is at *base + offset. dpo_ipc_close: unmap. */
typedef struct {
  unsigned char bytes[64];
} dpo_ipc_handle;
dpo_status dpo_ipc_export(const void* ptr, dpo_ipc_handle* handle, size_t* offset);
dpo_status dpo_ipc_import(const dpo_ipc_handle* handle, void** base);
dpo_status dpo_ipc_close(void* base);

/* ---- Vocabulary-parallel head ----------------------------------------------
 * W split by vocabulary rows across ranks, every rank holding the same batch (the
 * vocabulary-parallel alternative to data parallelism for a head too large to
 * replicate; [V, d] rows stay where they are). Per step, on every rank:
 *   1. dpo_shard_logprob_parts on its rows -> per-position (lse_k, z_y,k);
 *   2. all-gather those [Nc] vectors across the ranks, in shard order;
 *   3. dpo_shard_combine -> the full-vocabulary sums, log-probs and lse_state,
 *      identical on every rank;
 *   4. (policy) dpo_shard_backward with the global lse_state -> this rank's dW
 *      rows and a partial dH; all-reduce (sum) the partial dH across the ranks.
 * The library makes no collective call: the caller moves the buffers (NCCL).
 * Shard k's W is rows [offset, offset + V) of the full [total, d] head; shards
 * must not overlap and must cover [0, total). */
typedef struct {
  int32_t offset;   /* first vocabulary row of this shard in the full head */
  int32_t total;    /* vocabulary size of the full head (<= 2^24) */
} dpo_vocab_shard;

/* Step 1: the forward of dpo_seq_logprobs over this shard's rows only.
 *   batch      the shard: W = its [V, d] rows, V = its row count; tokens are ids in
 *              the full vocabulary (a token outside [0, total) is a bad target)
 *   shard_lse  device [Nc] fp32, out: log sum_{v in shard} exp(z_v) per scored position
 *   shard_zy   device [Nc] fp32, out: z of the target if this shard holds it, else -inf
 *   ws         device workspace, >= fwd_bytes of dpo_workspace_size(batch)
 * Nc = sum of completion_len. Errors: those of dpo_seq_logprobs, and
 * DPO_ERR_INVALID_ARG for a shard outside [0, total). */
dpo_status dpo_shard_logprob_parts(const dpo_batch* batch, const dpo_vocab_shard* shard,
                                   float* shard_lse, float* shard_zy, void* ws, size_t ws_bytes,
                                   void* stream);

/* Step 3: merge the gathered parts of n_shards shards (row k = shard k):
 *   shard_lse, shard_zy  device [n_shards, Nc] fp32 (all-gather of step 1's outputs)
 *   seq_logp, tok_logp, lse_state  as dpo_seq_logprobs (tok_logp, lse_state may be NULL)
 *   ws   device workspace, >= fwd_bytes of dpo_workspace_size(batch)
 * lse = M + log sum_k exp(lse_k - M) in fp64, shards in index order, so every rank
 * that merges the same gathered values gets the same bits; a bad target scores 0.
 * batch is any shard's batch (its rows and tokens are used; W is not read). */
dpo_status dpo_shard_combine(const dpo_batch* batch, int32_t vocab_total, int32_t n_shards,
                             const float* shard_lse, const float* shard_zy, float* seq_logp,
                             float* tok_logp, float* lse_state, void* ws, size_t ws_bytes,
                             void* stream);

/* Step 4: dpo_backward over this shard's rows, with lse_state from step 3:
 * dz = row_coef (onehot - softmax) on the shard's columns (the softmax uses the
 * full-vocabulary lse), dH_part = dz . W_shard (device [R, L, d] fp32, fully
 * written; the sum over shards is dH), dW_shard (device [V, d] fp32, written or
 * accumulated) = this shard's rows of dW. ws: >= bwd_min_bytes of
 * dpo_workspace_size(batch). dH_part may be NULL. */
dpo_status dpo_shard_backward(const dpo_batch* batch, const dpo_vocab_shard* shard,
                              const float* lse_state, const float* row_coef, float* dH_part,
                              float* dW_shard, int accumulate_dW, void* ws, size_t ws_bytes,
                              void* stream);

/* Logits-mean metrics: the mean of the logits z = h_t . W^T over every position
 * (prompt, completion and padding) of the chosen rows, and separately of the
 * rejected rows, over the whole vocabulary -- the policy_chosen_logits_mean and
 * policy_rejected_logits_mean the torchtune DPO loop logs ("Run Distributed
 * Full-Model DPO with PyTorch FSDP", Step 4 splits the logits of every position
 * into the two halves; "What to Watch Out For" names the metrics).
 *   batch    as for dpo_seq_logprobs; every position of every row counts, so
 *            prompt_len / completion_len are checked but do not change the result;
 *            R must be even
 *   layout   which rows are chosen: DPO_PAIRS_HALVES (rows [0, R/2)) or
 *            DPO_PAIRS_ADJACENT (even rows)
 *   means    device [2] fp32, out: {chosen mean, rejected mean}
 *   ws       device workspace, >= fwd_bytes of dpo_workspace_size, 256-byte aligned
 * The logits are not formed: sum_{t,v} z_tv = (sum_t h_t) . (sum_v W[v]), so the
 * call reads W and H once (column sums in fp64, fixed order: the same result on
 * every run). Errors: DPO_ERR_INVALID_ARG (odd R, bad layout, NULL means, or any
 * batch check of dpo_seq_logprobs), DPO_ERR_WORKSPACE, DPO_ERR_CUDA. */
dpo_status dpo_logits_mean(const dpo_batch* batch, int32_t layout, float* means, void* ws,
                           size_t ws_bytes, void* stream);

/* Size of the scratch array built into the library for dpo_seq_logprobs_noalloc. */
#define DPO_NOALLOC_SCRATCH_BYTES (32u << 20)

/* dpo_seq_logprobs without a workspace argument, for callers that may not
 * allocate device memory (for example code running inside a framework that owns
 * the device-memory budget and forbids allocation from its plugins, or code that
 * cannot accept the device-wide synchronisation cudaMalloc/cudaFree may cause).
 * The pages have no counterpart: this is a deployment convenience of the library.
 *   Arguments, outputs and errors are those of dpo_seq_logprobs.
 *   Scratch: a DPO_NOALLOC_SCRATCH_BYTES (32 MiB) array compiled into the
 *   library, held by every device that loads it until the process exits. A batch
 *   whose forward workspace (dpo_workspace_size's fwd_bytes) exceeds that size is
 *   refused with DPO_ERR_WORKSPACE before any device work.
 *   Set-up: the first call on a device, made with that device current, looks the
 *   array's address up (cudaGetSymbolAddress), as does the first call after that
 *   device's context was destroyed and rebuilt; make that first call before any
 *   stream capture.
 *   Sharing: all calls on a device use the same array and it keeps the last
 *   call's contents (every byte a call reads is written by that call first).
 *   Calls whose work overlaps on the GPU (different streams, or different host
 *   threads without ordering) race on the array: serialise them.
 *   The call allocates no device memory. */
dpo_status dpo_seq_logprobs_noalloc(const dpo_batch* batch, int want_grad, float* seq_logp,
                                    float* tok_logp, float* lse_state, void* stream);

/* Synchronise `stream`, then return and clear the current device's status word
 * (DPO_OK, DPO_ERR_TIMEOUT or DPO_ERR_BAD_TARGET), or DPO_ERR_CUDA if the
 * synchronisation itself failed. */
dpo_status dpo_check(void* stream);

/* Time budget, in milliseconds, of every bounded wait inside the kernels
 * launched afterwards by this process (default 4000). A wait that exceeds it
 * makes the kernel record DPO_ERR_TIMEOUT, drain its in-flight copies and MMAs
 * (again bounded) and exit. Returns the previous value. */
uint32_t dpo_set_wait_budget_ms(uint32_t ms);

/* 64-bit fingerprint of a device buffer, for tagging offline reference scores with
 * the weights they were computed from (Megatron-Bridge PR 6092: the scorer writes a
 * metadata record next to the stored sums and the trainer refuses a mismatch).
 *   data  device, 16-byte aligned, `bytes` long (bytes may be 0)
 *   out   device [1] uint64, 8-byte aligned: written asynchronously on `stream`
 * Each 16-byte word is hashed with its index through the splitmix64 finaliser
 * (Steele, Lea and Flood, OOPSLA 2014) and the hashes are summed mod 2^64, so the
 * value is the same for every launch configuration and run. Not cryptographic. */
dpo_status dpo_fingerprint(const void* data, size_t bytes, uint64_t* out, void* stream);

/* Self-test of the kernels' bounded waits: launches one CTA that waits, with the
 * same bounded wait the GEMM pipelines use, on a barrier nothing ever arrives on.
 * After budget_ms the wait gives up and records DPO_ERR_TIMEOUT in the status
 * word, which the next dpo_check(stream) returns; the kernel exits normally and
 * the context stays usable. No counterpart on the pages: a diagnostic of this
 * library's failure handling. */
dpo_status dpo_selftest_wait_timeout(uint32_t budget_ms, void* stream);

/* Which tensor-core GEMM kernel later calls of this process use, as a mask with
 * two bits per GEMM k: k = 0 the forward (logits + log-sum-exp), 1 the backward's
 * logit recompute (dz), 2 dH = dz.W, 3 dW = dz^T.H.
 *   bit k      clear: the GEMM runs on pairs of CTAs (tcgen05.mma.cta_group::2,
 *              256 x 256 tiles) when the device can co-schedule CTA pairs, unless one
 *              CTA per 128 x 256 tile fills the GPU's waves more than 5 % better for
 *              that launch's shape; set: always on one CTA per tile.
 *   bit 4 + k  clear: the CTA pairs claim tiles in raster order from a counter in the
 *              workspace (the tiles in flight stay one contiguous window of the
 *              raster); set: static round-robin (pair p takes tiles p, p + pairs, ...).
 *   bit 8      set: dH = dz.W is never split over the vocabulary (K) into parts of one
 *              launch (clear: split when that fills the GPU's waves better); this bit
 *              changes the backward workspace size, so set it before sizing.
 * Every choice gives the same results within rounding (bits 4-7 bit for bit: each tile
 * is computed the same way). Default 0. Returns the previous mask, or -1 for a value
 * outside 0..511. A diagnostic for measurements; the default is the fastest measured. */
int32_t dpo_set_gemm_variant(int32_t variant);

/* Static description of a status code. */
const char* dpo_status_string(dpo_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t dpo_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBDPO_DPO_H */
