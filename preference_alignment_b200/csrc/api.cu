// C ABI of libdpo: argument checks, the per-call schedule (packed scored
// positions), workspace layout, TMA tensor maps and the launch sequence of each
// entry point. See include/dpo.h for the contract of every call.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include "dpo.h"
#include "internal.h"

// Per-device status word: kernels record DPO_ERR_TIMEOUT / DPO_ERR_BAD_TARGET
// here; dpo_check() reads and clears it.
__device__ int g_dpo_status_word = 0;

namespace {

using namespace dpo;

// NVTX range around an entry point (names the call on profiler timelines; with no
// tool attached the push/pop cost a few nanoseconds).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr size_t kAlign = 256;
constexpr int kMinChunk = 128;   // smallest backward token chunk

std::atomic<uint32_t> g_budget_ms{4000};
std::atomic<int> g_gemm_variant{0};

struct DevInfo {
  bool ready = false;
  void* ctx = nullptr;     // the context the cached addresses belong to
  int* status = nullptr;
  int sms = 0;
};
std::mutex g_mu;
DevInfo g_dev[256];

dpo_status device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return DPO_ERR_CUDA;
  void* ctx = nullptr;
  if (!dpo::current_context(&ctx)) return DPO_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& di = g_dev[dev];
  if (!di.ready || di.ctx != ctx) {     // first call, or the context was rebuilt
    di.ready = false;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dpo_status_word) != cudaSuccess) return DPO_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DPO_ERR_CUDA;
    di.status = static_cast<int*>(p);
    di.sms = sms;
    di.ctx = ctx;
    di.ready = true;
  }
  *out = di;
  return DPO_OK;
}

DevCtl make_ctl(const DevInfo& di) {
  DevCtl c;
  c.status = di.status;
  c.budget_ns = static_cast<unsigned long long>(g_budget_ms.load()) * 1000000ull;
  return c;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [outer, inner] array; 128-byte swizzle for
// the GEMM operand tiles, 64-byte swizzle for the dz epilogue's 32 x 32 store boxes
// (64-byte rows).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Plan {
  int R = 0, L = 0, d = 0, V = 0, dtype = 0;
  int v0 = 0, Vtot = 0;                // W holds vocabulary rows [v0, v0 + V) of Vtot
  int Nc = 0;
  std::vector<int> row_start;          // [R + 1]
  // common prefix of both workspaces
  size_t off_rs = 0, off_P = 0, off_y = 0, off_dst = 0, off_rowid = 0, off_sync = 0, off_hp = 0,
         prefix = 0;
  // forward suffix
  int S = 0, ldp = 0;
  size_t off_part = 0, off_zy = 0, off_lp = 0, fwd_total = 0;
  // backward suffix: per position one dz row (g_row_bytes) and, with split-K dH, the
  // fp32 partial sums of K parts 1.. (part_row_bytes)
  size_t off_G = 0, g_row_bytes = 0, part_row_bytes = 0, bwd_total = 0, bwd_min = 0;
  long long ldG = 0;
  // dH = dz . W over the vocabulary: sequential launches of dh_chunk columns, each adding
  // to dH (dh_kb_part == 0), or one launch split into dh_parts K parts of dh_kb_part
  // 64-column blocks
  int dh_chunk = 0, dh_kb_part = 0, dh_parts = 1;
};

// CTA pairs a launch plans for: a B200 has 148 SMs (the dH split is chosen with it; on
// another SM count the choice is only less well tuned).
constexpr int kPlanPairs = 74;
constexpr int kMaxDhParts = 16;
// A unit's epilogue (a 256 x 256 fp32 tile written out) takes about as long as this many
// K blocks of MMAs; it overlaps the next unit's main loop, so a unit costs at least this.
// It is also the shortest K part the split uses.
constexpr int kEpilogueKb = 8;

// Estimated duration of a launch of `units` work units of `kb` K blocks each, in units
// of one K block on every pair: whole rounds of kPlanPairs units.
double rounds_x_k(long long units, long long kb) {
  const long long per_unit = kb > kEpilogueKb ? kb : kEpilogueKb;
  return static_cast<double>((units + kPlanPairs - 1) / kPlanPairs) *
         static_cast<double>(per_unit);
}

// dH = dz . W has few output tiles (token tiles x column tiles of d), so one launch can
// leave most of its last wave idle (e.g. 96 tiles on 74 pairs: 2 rounds for 1.3 waves of
// work). Cutting the vocabulary (K) into parts that run as separate work units of one
// launch fills the rounds; each part beyond the first costs an fp32 partial sum of the
// rows (written, then added in part order by a small kernel).
void plan_dh_split(Plan* p) {
  const long long kb = (p->V + kBK - 1) / kBK;
  const long long tiles = static_cast<long long>((p->Nc + 255) / 256) * ((p->d + kBN - 1) / kBN);
  p->dh_chunk = kMaxAccumK;                     // one launch unless the vocabulary exceeds it
  p->dh_kb_part = 0;
  p->dh_parts = 1;
  if (p->dtype != DPO_BF16 || tiles == 0 || ((gemm_variant() >> 8) & 1)) return;
  const double seq = rounds_x_k(tiles, kb);
  // the split with the fewest estimated K-block rounds, each extra part charged 2 %
  const long long max_kbp = kMaxAccumK / kBK;   // K blocks one accumulation may take
  double best = seq;
  for (int q = 2; q <= kMaxDhParts; ++q) {
    long long kbp = (kb + q - 1) / q;
    if (kbp > max_kbp) continue;
    if (kbp < kEpilogueKb) break;
    const int parts = static_cast<int>((kb + kbp - 1) / kbp);
    const double est = rounds_x_k(tiles * parts, kbp) * (1.0 + 0.02 * (parts - 1));
    if (est < best * 0.97) {
      best = est;
      p->dh_kb_part = static_cast<int>(kbp);
      p->dh_parts = parts;
    }
  }
  if (p->dh_parts > 1) {
    p->dh_chunk = p->V;
    p->part_row_bytes = static_cast<size_t>(p->dh_parts - 1) * p->d * sizeof(float);
  }
}

dpo_status make_plan(const dpo_batch* b, Plan* p) {
  if (b == nullptr) return DPO_ERR_INVALID_ARG;
  if (b->dtype == DPO_F16) return DPO_ERR_UNSUPPORTED;
  if (b->dtype != DPO_BF16 && b->dtype != DPO_F32) return DPO_ERR_INVALID_ARG;
  if (b->R < 1 || b->R > 65535 || b->L < 2 || b->V < 1 || b->V > (1 << 24) || b->d < 1 ||
      b->d > 65536)
    return DPO_ERR_INVALID_ARG;
  if (b->d % 8 != 0) return DPO_ERR_UNSUPPORTED;
  if (b->H == nullptr || b->W == nullptr || b->tokens == nullptr || b->prompt_len == nullptr ||
      b->completion_len == nullptr)
    return DPO_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(b->H) | reinterpret_cast<uintptr_t>(b->W)) % 16 != 0)
    return DPO_ERR_INVALID_ARG;
  if (static_cast<long long>(b->R) * b->L > (1ll << 31) - 2) return DPO_ERR_INVALID_ARG;
  p->R = b->R;
  p->L = b->L;
  p->d = b->d;
  p->V = b->V;
  p->v0 = 0;
  p->Vtot = b->V;
  p->dtype = b->dtype;
  p->row_start.assign(b->R + 1, 0);
  long long nc = 0;
  for (int r = 0; r < b->R; ++r) {
    const int P = b->prompt_len[r], C = b->completion_len[r];
    if (P < 1 || C < 0 || static_cast<long long>(P) + C > b->L) return DPO_ERR_INVALID_ARG;
    p->row_start[r] = static_cast<int>(nc);
    nc += C;
  }
  if (nc > (1ll << 30)) return DPO_ERR_INVALID_ARG;
  p->row_start[b->R] = static_cast<int>(nc);
  p->Nc = static_cast<int>(nc);
  const size_t Nc = p->Nc;
  const bool bf16 = b->dtype == DPO_BF16;

  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, kAlign);
    return at;
  };
  p->off_rs = take(sizeof(int) * (b->R + 1));
  p->off_P = take(sizeof(int) * b->R);
  p->off_y = take(sizeof(int) * Nc);
  p->off_dst = take(sizeof(int) * Nc);
  p->off_rowid = take(sizeof(int) * Nc);
  p->off_sync = take(sizeof(int) * kSyncInts);
  p->off_hp = take(bf16 ? Nc * b->d * 2 : 0);
  p->prefix = o;

  p->S = bf16 ? (b->V + kBN - 1) / kBN : 1;
  p->ldp = static_cast<int>(align_up(Nc > 0 ? Nc : 1, 64));
  p->off_part = take(sizeof(float2) * static_cast<size_t>(p->S) * p->ldp);
  p->off_zy = take(sizeof(float) * p->ldp);
  p->off_lp = take(sizeof(float) * p->ldp);
  // the forward workspace also serves dpo_logits_mean
  p->fwd_total = std::max(o, align_up(logits_mean_bytes(b->d), kAlign));

  o = p->prefix;
  p->ldG = bf16 ? static_cast<long long>(align_up(b->V, 8)) : b->V;
  p->g_row_bytes = static_cast<size_t>(p->ldG) * (bf16 ? 2 : 4);
  p->off_G = o;
  plan_dh_split(p);
  const size_t full_rows = Nc > 0 ? Nc : 1;
  const size_t min_rows = full_rows < static_cast<size_t>(kMinChunk) ? full_rows : kMinChunk;
  const size_t row_bytes = p->g_row_bytes + p->part_row_bytes;
  p->bwd_total = align_up(o + full_rows * row_bytes + kAlign, kAlign);
  p->bwd_min = align_up(o + min_rows * row_bytes + kAlign, kAlign);
  return DPO_OK;
}

// The batch's W is vocabulary rows [offset, offset + V) of a head of `total` rows.
dpo_status apply_shard(const dpo_vocab_shard* sh, Plan* p) {
  if (sh == nullptr || sh->offset < 0 || sh->total < 1 || sh->total > (1 << 24) ||
      static_cast<long long>(sh->offset) + p->V > sh->total)
    return DPO_ERR_INVALID_ARG;
  p->v0 = sh->offset;
  p->Vtot = sh->total;
  return DPO_OK;
}

Sched sched_of(const Plan& p, void* ws) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  Sched s;
  s.row_start = reinterpret_cast<const int*>(w + p.off_rs);
  s.prompt = reinterpret_cast<const int*>(w + p.off_P);
  s.y = reinterpret_cast<int*>(w + p.off_y);
  s.dst = reinterpret_cast<int*>(w + p.off_dst);
  s.rowid = reinterpret_cast<int*>(w + p.off_rowid);
  s.sync = reinterpret_cast<int*>(w + p.off_sync);
  return s;
}

dpo_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DPO_OK : DPO_ERR_CUDA; }

// Upload the row table and build the scored-position tables (+ packed H for bf16).
dpo_status stage_schedule(const Plan& p, const dpo_batch* b, void* ws, const DevCtl& ctl,
                          cudaStream_t st, bool pack = true) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  std::vector<RowChunk> chunks((p.R + kRowChunk - 1) / kRowChunk);
  for (size_t c = 0; c < chunks.size(); ++c) {
    RowChunk& rc = chunks[c];
    rc.row0 = static_cast<int>(c) * kRowChunk;
    rc.n = std::min(kRowChunk, p.R - rc.row0);
    rc.R = p.R;
    rc.total = p.Nc;
    for (int i = 0; i < rc.n; ++i) {
      rc.rs[i] = p.row_start[rc.row0 + i];
      rc.P[i] = b->prompt_len[rc.row0 + i];
    }
    cudaError_t e = launch_upload_rows(rc, reinterpret_cast<int*>(w + p.off_rs),
                                       reinterpret_cast<int*>(w + p.off_P), st);
    if (e != cudaSuccess) return DPO_ERR_CUDA;
  }
  uint16_t* Hp = pack && p.dtype == DPO_BF16 ? reinterpret_cast<uint16_t*>(w + p.off_hp) : nullptr;
  return cuda_status(launch_prep(static_cast<const uint16_t*>(b->H), b->tokens, sched_of(p, ws),
                                 p.R, p.L, p.d, p.V, p.v0, p.Vtot, p.Nc, Hp, ctl, st));
}

// Gradient outputs are written 16 bytes at a time (NULL passes: it means "not wanted").
bool aligned16(const void* ptr) { return reinterpret_cast<uintptr_t>(ptr) % 16 == 0; }

bool ws_ok(const void* ws, size_t have, size_t need) {
  return ws != nullptr && have >= need && reinterpret_cast<uintptr_t>(ws) % kAlign == 0;
}

// Schedule, LM-head GEMM with the online log-sum-exp, and the combine over the
// vocabulary tiles: lp in the workspace; lse and the target logit (-inf when the
// target is not in this call's rows) when asked.
dpo_status forward_core(const Plan& p, const dpo_batch* batch, void* ws, float* lse_out,
                        float* zy_out, const DevInfo& di, const DevCtl& ctl, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  dpo_status s = stage_schedule(p, batch, ws, ctl, st);
  if (s != DPO_OK) return s;
  const Sched sc = sched_of(p, ws);
  float2* part = reinterpret_cast<float2*>(w + p.off_part);
  float* zy = reinterpret_cast<float*>(w + p.off_zy);
  float* lp = reinterpret_cast<float*>(w + p.off_lp);
  if (p.Nc == 0) return DPO_OK;
  if (p.dtype == DPO_BF16) {
    CUtensorMap mA, mB;
    if (!make_map(&mA, w + p.off_hp, p.d, p.Nc, 2ull * p.d, kBK, kBoxRows) ||
        !make_map(&mB, batch->W, p.d, p.V, 2ull * p.d, kBK, kBoxRows))
      return DPO_ERR_CUDA;
    if (launch_fwd_lse(mA, mB, p.Nc, p.V, p.d, sc.y, part, p.ldp, zy, di.sms, sc.sync, ctl, st) !=
        cudaSuccess)
      return DPO_ERR_CUDA;
  } else {
    if (launch_f32_fwd(static_cast<const float*>(batch->H), static_cast<const float*>(batch->W),
                       sc, p.Nc, p.d, p.V, part, zy, st) != cudaSuccess)
      return DPO_ERR_CUDA;
  }
  return cuda_status(launch_combine(part, p.ldp, p.S, zy, sc.y, p.Nc, lp, lse_out, zy_out, st));
}

// SMs a launch may use: all of them, or at most max_sms (> 0) to leave the rest to
// kernels that run beside it (a collective on another stream).
int sm_budget(const DevInfo& di, int max_sms) {
  return max_sms > 0 && max_sms < di.sms ? max_sms : di.sms;
}

// Token chunk of the backward that fits the workspace (a multiple of 128 unless it
// covers every scored position; never more than kMaxAccumK, dW's K per chunk).
int backward_chunk(const Plan& p, size_t ws_bytes) {
  const size_t row_bytes = p.g_row_bytes + p.part_row_bytes;
  const size_t rows_fit =
      ws_bytes > p.off_G + kAlign ? (ws_bytes - p.off_G - kAlign) / row_bytes : 0;
  int Mc = static_cast<int>(std::min<size_t>(rows_fit, static_cast<size_t>(p.Nc)));
  Mc = std::min(Mc, kMaxAccumK);
  if (Mc < p.Nc) Mc = Mc / kMinChunk * kMinChunk;
  return Mc;
}

// Split-K partial sums of a token chunk of mc positions: after its dz rows.
float* dh_part_scratch(const Plan& p, uint8_t* w, int mc) {
  if (p.dh_parts < 2) return nullptr;
  return reinterpret_cast<float*>(w + align_up(p.off_G + static_cast<size_t>(mc) * p.g_row_bytes,
                                               kAlign));
}

// dH rows of the packed positions [tok0, tok0 + mc) from the dz chunk in the workspace:
// dH = dz . W, reduced over the vocabulary in one launch (split into K parts when that
// fills the GPU's waves better, see plan_dh_split); a vocabulary beyond kMaxAccumK
// columns runs in chunks of that many, the later chunks added to the rows by the
// epilogue. No accumulation runs longer than kMaxAccumK products.
dpo_status run_dh(const Plan& p, const dpo_batch* batch, uint8_t* w, const Sched& sc, int tok0,
                  int mc, float* dH, int sms, const DevCtl& ctl, cudaStream_t st) {
  if (p.dtype != DPO_BF16) {
    const float* G = reinterpret_cast<const float*>(w + p.off_G);
    return cuda_status(launch_f32_dh(G, static_cast<const float*>(batch->W), sc, tok0, mc, p.d,
                                     p.V, dH, st));
  }
  const uint16_t* G = reinterpret_cast<const uint16_t*>(w + p.off_G);
  float* part = dh_part_scratch(p, w, mc);
  for (int v0 = 0; v0 < p.V; v0 += p.dh_chunk) {
    const int vc = std::min(p.dh_chunk, p.V - v0);
    CUtensorMap mGk, mWmn;
    if (!make_map(&mGk, G + v0, vc, mc, 2ull * p.ldG, kBK, kBoxRows) ||
        !make_map(&mWmn, static_cast<const uint16_t*>(batch->W) + static_cast<size_t>(v0) * p.d,
                  p.d, vc, 2ull * p.d, kBoxMN, kBK))
      return DPO_ERR_CUDA;
    if (launch_bwd_dh(mGk, mWmn, mc, vc, p.d, tok0, sc.dst, dH, v0 > 0 ? 1 : 0, part,
                      p.dh_kb_part, sms, sc.sync, ctl, st) != cudaSuccess)
      return DPO_ERR_CUDA;
  }
  return DPO_OK;
}

// dW rows [v0, v1) (+)= dz^T . Hp for the packed positions [tok0, tok0 + mc) of the dz
// chunk in the workspace; dW points at the whole [V, d] array.
dpo_status run_dw(const Plan& p, const dpo_batch* batch, uint8_t* w, const Sched& sc, int tok0,
                  int mc, int v0, int v1, float* dW, int acc, int sms, const DevCtl& ctl,
                  cudaStream_t st) {
  if (v1 <= v0) return DPO_OK;
  if (p.dtype != DPO_BF16) {
    const float* G = reinterpret_cast<const float*>(w + p.off_G);
    return cuda_status(launch_f32_dw(G, static_cast<const float*>(batch->H), sc, tok0, mc, p.d,
                                     p.V, v0, v1, dW, acc, st));
  }
  const uint16_t* G = reinterpret_cast<const uint16_t*>(w + p.off_G);
  const uint16_t* hp0 = reinterpret_cast<const uint16_t*>(w + p.off_hp) +
                        static_cast<size_t>(tok0) * p.d;
  CUtensorMap mGmn, mHmn;
  if (!make_map(&mGmn, G + v0, v1 - v0, mc, 2ull * p.ldG, kBoxMN, kBK) ||
      !make_map(&mHmn, hp0, p.d, mc, 2ull * p.d, kBoxMN, kBK))
    return DPO_ERR_CUDA;
  return cuda_status(launch_bwd_dw(mGmn, mHmn, mc, v1 - v0, p.d,
                                   dW + static_cast<size_t>(v0) * p.d, acc, sms, sc.sync, ctl,
                                   st));
}

// Backward of sum_r row_coef[r] S_r for this call's vocabulary rows: dz chunks,
// dH (fully written, when dH != NULL) and dW (written or accumulated, when dW != NULL).
// With dW == NULL the whole batch must fit one chunk: its dz then stays in the
// workspace for dpo_backward_dw / dpo_backward_dh.
dpo_status backward_core(const Plan& p, const dpo_batch* batch, const float* lse_state,
                         const float* row_coef, float* dH, float* dW, int accumulate_dW, void* ws,
                         size_t ws_bytes, void* stream) {
  dpo_status s = DPO_OK;
  if ((p.Nc > 0 && lse_state == nullptr) || row_coef == nullptr) return DPO_ERR_INVALID_ARG;
  if (!aligned16(dH) || !aligned16(dW)) return DPO_ERR_INVALID_ARG;   // 16-byte row stores
  if (!ws_ok(ws, ws_bytes, p.bwd_min)) return DPO_ERR_WORKSPACE;
  const int Mc = backward_chunk(p, ws_bytes);
  if (p.Nc > 0 && Mc < 1) return DPO_ERR_WORKSPACE;
  if (dW == nullptr && Mc < p.Nc) return DPO_ERR_WORKSPACE;   // dz must stay whole
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  const DevCtl ctl = make_ctl(di);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);

  if ((s = stage_schedule(p, batch, ws, ctl, st)) != DPO_OK) return s;
  const Sched sc = sched_of(p, ws);
  if (dH != nullptr &&
      cudaMemsetAsync(dH, 0, sizeof(float) * static_cast<size_t>(p.R) * p.L * p.d, st) !=
          cudaSuccess)
    return DPO_ERR_CUDA;
  if (p.Nc == 0) {
    if (dW != nullptr && !accumulate_dW &&
        cudaMemsetAsync(dW, 0, sizeof(float) * static_cast<size_t>(p.V) * p.d, st) != cudaSuccess)
      return DPO_ERR_CUDA;
    return DPO_OK;
  }
  const bool bf16 = p.dtype == DPO_BF16;
  for (int tok0 = 0; tok0 < p.Nc; tok0 += Mc) {
    const int mc = std::min(Mc, p.Nc - tok0);
    const int acc = (accumulate_dW || tok0 > 0) ? 1 : 0;
    if (bf16) {
      uint16_t* G = reinterpret_cast<uint16_t*>(w + p.off_G);
      const uint16_t* hp0 = reinterpret_cast<const uint16_t*>(w + p.off_hp) +
                            static_cast<size_t>(tok0) * p.d;
      CUtensorMap mHk, mWk, mGst;
      if (!make_map(&mGst, G, p.V, mc, 2ull * p.ldG, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B) ||
          !make_map(&mHk, hp0, p.d, mc, 2ull * p.d, kBK, kBoxRows) ||
          !make_map(&mWk, batch->W, p.d, p.V, 2ull * p.d, kBK, kBoxRows))
        return DPO_ERR_CUDA;
      if (launch_bwd_grad(mHk, mWk, mGst, mc, p.V, p.d, tok0, sc.y, lse_state, row_coef,
                          sc.rowid, di.sms, sc.sync, ctl, st) != cudaSuccess)
        return DPO_ERR_CUDA;
    } else {
      if (launch_f32_grad(static_cast<const float*>(batch->H),
                          static_cast<const float*>(batch->W), sc, tok0, mc, p.d, p.V, lse_state,
                          row_coef, reinterpret_cast<float*>(w + p.off_G), st) != cudaSuccess)
        return DPO_ERR_CUDA;
    }
    if (dH != nullptr && (s = run_dh(p, batch, w, sc, tok0, mc, dH, di.sms, ctl, st)) != DPO_OK)
      return s;
    if (dW != nullptr &&
        (s = run_dw(p, batch, w, sc, tok0, mc, 0, p.V, dW, acc, di.sms, ctl, st)) != DPO_OK)
      return s;
  }
  return DPO_OK;
}

// Checks shared by the calls that continue from the dz a dpo_backward(dW = NULL) left
// in the workspace: the whole batch in one chunk.
dpo_status dz_resident(const Plan& p, const void* ws, size_t ws_bytes, int max_sms) {
  if (max_sms < 0) return DPO_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, p.bwd_min)) return DPO_ERR_WORKSPACE;
  if (backward_chunk(p, ws_bytes) < p.Nc) return DPO_ERR_WORKSPACE;
  return DPO_OK;
}

}  // namespace

int dpo::gemm_variant() { return g_gemm_variant.load(); }

bool dpo::current_context(void** ctx) {
  // The runtime's calls above made the device's primary context current; the driver's
  // cuCtxGetCurrent (reached without linking libcuda) names it.
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  if (fn == nullptr) return false;
  CUcontext c = nullptr;
  if (fn(&c) != CUDA_SUCCESS || c == nullptr) return false;
  *ctx = c;
  return true;
}

extern "C" {

dpo_status dpo_workspace_size(const dpo_batch* batch, size_t* fwd_bytes, size_t* bwd_bytes,
                              size_t* bwd_min_bytes) {
  Plan p;
  const dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (fwd_bytes) *fwd_bytes = p.fwd_total;
  if (bwd_bytes) *bwd_bytes = p.bwd_total;
  if (bwd_min_bytes) *bwd_min_bytes = p.bwd_min;
  return DPO_OK;
}

dpo_status dpo_seq_logprobs(const dpo_batch* batch, int want_grad, float* seq_logp,
                            float* tok_logp, float* lse_state, void* ws, size_t ws_bytes,
                            void* stream) {
  NvtxRange nvtx_range("dpo_seq_logprobs");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (seq_logp == nullptr || (want_grad && lse_state == nullptr)) return DPO_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, p.fwd_total)) return DPO_ERR_WORKSPACE;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  const DevCtl ctl = make_ctl(di);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);

  if ((s = forward_core(p, batch, ws, want_grad ? lse_state : nullptr, nullptr, di, ctl, st)) !=
      DPO_OK)
    return s;
  const Sched sc = sched_of(p, ws);
  float* lp = reinterpret_cast<float*>(w + p.off_lp);
  return cuda_status(launch_rowsum(lp, sc.row_start, sc.prompt, p.R, p.L, seq_logp, tok_logp, st));
}

dpo_status dpo_shard_logprob_parts(const dpo_batch* batch, const dpo_vocab_shard* shard,
                                   float* shard_lse, float* shard_zy, void* ws, size_t ws_bytes,
                                   void* stream) {
  NvtxRange nvtx_range("dpo_shard_logprob_parts");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if ((s = apply_shard(shard, &p)) != DPO_OK) return s;
  if (shard_lse == nullptr || shard_zy == nullptr) return DPO_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, p.fwd_total)) return DPO_ERR_WORKSPACE;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  return forward_core(p, batch, ws, shard_lse, shard_zy, di, make_ctl(di),
                      static_cast<cudaStream_t>(stream));
}

dpo_status dpo_shard_combine(const dpo_batch* batch, int32_t vocab_total, int32_t n_shards,
                             const float* shard_lse, const float* shard_zy, float* seq_logp,
                             float* tok_logp, float* lse_state, void* ws, size_t ws_bytes,
                             void* stream) {
  NvtxRange nvtx_range("dpo_shard_combine");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (vocab_total < p.V || vocab_total > (1 << 24) || n_shards < 1 || n_shards > vocab_total ||
      seq_logp == nullptr || (p.Nc > 0 && (shard_lse == nullptr || shard_zy == nullptr)))
    return DPO_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, p.fwd_total)) return DPO_ERR_WORKSPACE;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  const DevCtl ctl = make_ctl(di);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // targets classified against the whole head: valid or bad, never "elsewhere"
  Plan q = p;
  q.v0 = 0;
  q.V = vocab_total;
  q.Vtot = vocab_total;
  if ((s = stage_schedule(q, batch, ws, ctl, st, false)) != DPO_OK) return s;
  const Sched sc = sched_of(p, ws);
  float* lp = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + p.off_lp);
  if (launch_shard_combine(shard_lse, shard_zy, n_shards, p.Nc, sc.y, lp, lse_state, st) !=
      cudaSuccess)
    return DPO_ERR_CUDA;
  return cuda_status(launch_rowsum(lp, sc.row_start, sc.prompt, p.R, p.L, seq_logp, tok_logp, st));
}

dpo_status dpo_loss(int32_t B, int32_t layout, const float* pol, const float* ref, float beta,
                    float grad_scale, float* loss, float* accuracy, float* margins,
                    float* chosen_rewards, float* rejected_rewards, float* weights,
                    float* row_coef, void* stream) {
  NvtxRange nvtx_range("dpo_loss");
  if (B < 1 || B > (1 << 28) || (layout != DPO_PAIRS_HALVES && layout != DPO_PAIRS_ADJACENT))
    return DPO_ERR_INVALID_ARG;
  if (pol == nullptr || ref == nullptr || loss == nullptr) return DPO_ERR_INVALID_ARG;
  if (!(beta > 0.f) || !std::isfinite(beta) || !std::isfinite(grad_scale))
    return DPO_ERR_INVALID_ARG;
  return cuda_status(launch_loss(B, layout, pol, ref, beta, grad_scale, 0, 0.0, nullptr, 0, 0,
                                 loss, accuracy, margins, chosen_rewards, rejected_rewards, weights,
                                 row_coef, nullptr, static_cast<cudaStream_t>(stream)));
}

dpo_status dpo_loss_ex(int32_t B, int32_t layout, const float* pol, const float* ref, float beta,
                       float grad_scale, const dpo_loss_options* opt, float* loss, float* accuracy,
                       float* margins, float* chosen_rewards, float* rejected_rewards,
                       float* weights, float* row_coef, float* nll, void* stream) {
  NvtxRange nvtx_range("dpo_loss_ex");
  if (B < 1 || B > (1 << 28) || (layout != DPO_PAIRS_HALVES && layout != DPO_PAIRS_ADJACENT))
    return DPO_ERR_INVALID_ARG;
  const bool reference_free = opt != nullptr && opt->reference_free != 0;
  if (reference_free) ref = nullptr;   // the kernel reads a NULL reference as zeros
  if (pol == nullptr || (ref == nullptr && !reference_free) || loss == nullptr)
    return DPO_ERR_INVALID_ARG;
  if (!(beta > 0.f) || !std::isfinite(beta) || !std::isfinite(grad_scale))
    return DPO_ERR_INVALID_ARG;
  int normalize = 0;
  float nll_weight = 0.f;
  const int32_t* clen = nullptr;
  long long pairs_total = 0, ntok_total = 0;
  if (opt != nullptr) {
    normalize = opt->normalize ? 1 : 0;
    nll_weight = opt->nll_weight;
    clen = opt->completion_len;
    pairs_total = opt->pairs_total;
    ntok_total = opt->nll_tokens_total;
    if (!std::isfinite(nll_weight) || nll_weight < 0.f) return DPO_ERR_INVALID_ARG;
    if ((normalize || nll_weight > 0.f) && clen == nullptr) return DPO_ERR_INVALID_ARG;
    if (pairs_total != 0 && pairs_total < B) return DPO_ERR_INVALID_ARG;
    if (ntok_total < 0) return DPO_ERR_INVALID_ARG;
    if (opt->reference_free != 0 && opt->reference_free != 1) return DPO_ERR_INVALID_ARG;
  }
  return cuda_status(launch_loss(B, layout, pol, ref, beta, grad_scale, normalize, nll_weight,
                                 clen, pairs_total, ntok_total, loss, accuracy, margins,
                                 chosen_rewards, rejected_rewards, weights, row_coef, nll,
                                 static_cast<cudaStream_t>(stream)));
}

dpo_status dpo_backward(const dpo_batch* batch, const float* lse_state, const float* row_coef,
                        float* dH, float* dW, int accumulate_dW, void* ws, size_t ws_bytes,
                        void* stream) {
  NvtxRange nvtx_range("dpo_backward");
  Plan p;
  const dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  return backward_core(p, batch, lse_state, row_coef, dH, dW, accumulate_dW, ws, ws_bytes, stream);
}

dpo_status dpo_backward_dw(const dpo_batch* batch, int32_t v_begin, int32_t v_end, float* dW,
                           int accumulate_dW, int32_t max_sms, void* ws, size_t ws_bytes,
                           void* stream) {
  NvtxRange nvtx_range("dpo_backward_dw");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (dW == nullptr || !aligned16(dW) || v_begin < 0 || v_end > p.V || v_begin > v_end ||
      v_begin % 8 != 0 || (v_end % 8 != 0 && v_end != p.V))
    return DPO_ERR_INVALID_ARG;
  if ((s = dz_resident(p, ws, ws_bytes, max_sms)) != DPO_OK) return s;
  if (v_begin == v_end) return DPO_OK;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p.Nc == 0) {
    if (!accumulate_dW &&
        cudaMemsetAsync(dW + static_cast<size_t>(v_begin) * p.d, 0,
                        sizeof(float) * static_cast<size_t>(v_end - v_begin) * p.d,
                        st) != cudaSuccess)
      return DPO_ERR_CUDA;
    return DPO_OK;
  }
  return run_dw(p, batch, static_cast<uint8_t*>(ws), sched_of(p, ws), 0, p.Nc, v_begin, v_end, dW,
                accumulate_dW ? 1 : 0, sm_budget(di, max_sms), make_ctl(di), st);
}

static_assert(DPO_MAX_SCATTER_RANKS == dpo::kMaxScatterRanks, "one limit of scatter ranks");

dpo_status dpo_backward_dw_scatter(const dpo_batch* batch, const dpo_dw_scatter* sc_arg,
                                   int32_t max_sms, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("dpo_backward_dw_scatter");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (p.dtype != DPO_BF16) return DPO_ERR_UNSUPPORTED;
  if (sc_arg == nullptr) return DPO_ERR_INVALID_ARG;
  const dpo_dw_scatter& x = *sc_arg;
  if (x.n_ranks < 1 || x.n_ranks > kMaxScatterRanks || x.rank < 0 || x.rank >= x.n_ranks ||
      x.rows_per_rank < 1 || static_cast<long long>(x.rows_per_rank) * (x.n_ranks - 1) >= p.V)
    return DPO_ERR_INVALID_ARG;
  for (int q = 0; q < x.n_ranks; ++q)
    if (x.recv[q] == nullptr || !aligned16(x.recv[q])) return DPO_ERR_INVALID_ARG;
  if ((s = dz_resident(p, ws, ws_bytes, max_sms)) != DPO_OK) return s;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p.Nc == 0) {                      // no scored position: this rank's slots are zero
    for (int q = 0; q < x.n_ranks; ++q) {
      const long long first = static_cast<long long>(q) * x.rows_per_rank;
      const long long rows_q = q == x.n_ranks - 1 ? p.V - first : x.rows_per_rank;
      if (cudaMemsetAsync(x.recv[q] + static_cast<size_t>(x.rank) * rows_q * p.d, 0,
                          sizeof(float) * static_cast<size_t>(rows_q) * p.d, st) != cudaSuccess)
        return DPO_ERR_CUDA;
    }
    return DPO_OK;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  const uint16_t* G = reinterpret_cast<const uint16_t*>(w + p.off_G);
  const uint16_t* Hp = reinterpret_cast<const uint16_t*>(w + p.off_hp);
  CUtensorMap mGmn, mHmn;
  if (!make_map(&mGmn, G, p.V, p.Nc, 2ull * p.ldG, kBoxMN, kBK) ||
      !make_map(&mHmn, Hp, p.d, p.Nc, 2ull * p.d, kBoxMN, kBK))
    return DPO_ERR_CUDA;
  const Sched sc = sched_of(p, ws);
  return cuda_status(launch_bwd_dw_scatter(mGmn, mHmn, p.Nc, p.V, p.d, x.recv, x.n_ranks, x.rank,
                                           x.rows_per_rank, sm_budget(di, max_sms), sc.sync,
                                           make_ctl(di), st));
}

dpo_status dpo_dw_reduce_slots(const float* recv, int32_t n_slots, int32_t rows, int32_t d,
                               float* dW_shard, int accumulate, void* stream) {
  NvtxRange nvtx_range("dpo_dw_reduce_slots");
  if (recv == nullptr || dW_shard == nullptr || !aligned16(recv) || !aligned16(dW_shard) ||
      n_slots < 1 || n_slots > kMaxScatterRanks || rows < 0 || d < 8 || d % 8 != 0)
    return DPO_ERR_INVALID_ARG;
  return cuda_status(launch_dw_reduce_slots(recv, n_slots, rows, d, dW_shard, accumulate ? 1 : 0,
                                            static_cast<cudaStream_t>(stream)));
}

dpo_status dpo_backward_dh(const dpo_batch* batch, float* dH, int32_t max_sms, void* ws,
                           size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("dpo_backward_dh");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (dH == nullptr || !aligned16(dH)) return DPO_ERR_INVALID_ARG;
  if ((s = dz_resident(p, ws, ws_bytes, max_sms)) != DPO_OK) return s;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(dH, 0, sizeof(float) * static_cast<size_t>(p.R) * p.L * p.d, st) !=
      cudaSuccess)
    return DPO_ERR_CUDA;
  if (p.Nc == 0) return DPO_OK;
  return run_dh(p, batch, static_cast<uint8_t*>(ws), sched_of(p, ws), 0, p.Nc, dH,
                sm_budget(di, max_sms), make_ctl(di), st);
}

dpo_status dpo_shard_backward(const dpo_batch* batch, const dpo_vocab_shard* shard,
                              const float* lse_state, const float* row_coef, float* dH_part,
                              float* dW_shard, int accumulate_dW, void* ws, size_t ws_bytes,
                              void* stream) {
  NvtxRange nvtx_range("dpo_shard_backward");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if ((s = apply_shard(shard, &p)) != DPO_OK) return s;
  return backward_core(p, batch, lse_state, row_coef, dH_part, dW_shard, accumulate_dW, ws,
                       ws_bytes, stream);
}

dpo_status dpo_logits_mean(const dpo_batch* batch, int32_t layout, float* means, void* ws,
                           size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("dpo_logits_mean");
  Plan p;
  dpo_status s = make_plan(batch, &p);
  if (s != DPO_OK) return s;
  if (p.R % 2 != 0 || means == nullptr ||
      (layout != DPO_PAIRS_HALVES && layout != DPO_PAIRS_ADJACENT))
    return DPO_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, align_up(logits_mean_bytes(p.d), kAlign))) return DPO_ERR_WORKSPACE;
  DevInfo di;
  if ((s = device_info(&di)) != DPO_OK) return s;
  return cuda_status(launch_logits_mean(batch->H, batch->W, p.dtype == DPO_BF16, p.R, p.L, p.d,
                                        p.V, layout == DPO_PAIRS_ADJACENT ? 1 : 0, ws, means,
                                        di.sms, static_cast<cudaStream_t>(stream)));
}

dpo_status dpo_check(void* stream) {
  NvtxRange nvtx_range("dpo_check");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevInfo di;
  dpo_status s = device_info(&di);
  if (s != DPO_OK) return s;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DPO_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyAsync(&v, di.status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(di.status, 0, sizeof(int), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return DPO_ERR_CUDA;
  return static_cast<dpo_status>(v);
}

dpo_status dpo_fingerprint(const void* data, size_t bytes, uint64_t* out, void* stream) {
  NvtxRange nvtx_range("dpo_fingerprint");
  if (out == nullptr || reinterpret_cast<uintptr_t>(out) % 8 != 0) return DPO_ERR_INVALID_ARG;
  if (bytes > 0 && (data == nullptr || reinterpret_cast<uintptr_t>(data) % 16 != 0))
    return DPO_ERR_INVALID_ARG;
  DevInfo di;
  dpo_status s = device_info(&di);
  if (s != DPO_OK) return s;
  return cuda_status(launch_fingerprint(data, bytes, reinterpret_cast<unsigned long long*>(out),
                                        di.sms, static_cast<cudaStream_t>(stream)));
}

dpo_status dpo_selftest_wait_timeout(uint32_t budget_ms, void* stream) {
  DevInfo di;
  dpo_status s = device_info(&di);
  if (s != DPO_OK) return s;
  DevCtl ctl = make_ctl(di);
  ctl.budget_ns = static_cast<unsigned long long>(budget_ms < 1 ? 1 : budget_ms) * 1000000ull;
  return cuda_status(launch_wait_selftest(ctl, static_cast<cudaStream_t>(stream)));
}

int32_t dpo_set_gemm_variant(int32_t variant) {
  if (variant < 0 || variant > 511) return -1;
  return g_gemm_variant.exchange(variant);
}

uint32_t dpo_set_wait_budget_ms(uint32_t ms) { return g_budget_ms.exchange(ms < 1 ? 1 : ms); }

const char* dpo_status_string(dpo_status s) {
  switch (s) {
    case DPO_OK: return "ok";
    case DPO_ERR_INVALID_ARG: return "invalid argument";
    case DPO_ERR_UNSUPPORTED: return "unsupported (dtype or shape)";
    case DPO_ERR_CUDA: return "CUDA error";
    case DPO_ERR_TIMEOUT: return "device wait exceeded its time budget";
    case DPO_ERR_BAD_TARGET: return "target token outside [0, V)";
    case DPO_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
  }
  return "unknown status";
}

int32_t dpo_version(void) { return 300; }

}  // extern "C"
