// dpo_seq_logprobs_noalloc: the per-row log-prob forward for callers that may
// not allocate device memory.
//
// Some callers cannot call cudaMalloc: code that runs inside a host framework
// which owns the whole device-memory budget and forbids its plugins from
// allocating (an inference engine's enqueue callback, for instance), or code
// that cannot afford the device-wide synchronisation that cudaMalloc and
// cudaFree may imply while other streams are busy. Those callers cannot provide
// the workspace that dpo_seq_logprobs takes. This entry point uses a scratch
// array compiled into the library instead, so the caller passes only inputs and
// outputs.
//
// The scratch lives in the file-scope array below: every device that loads the
// library holds it until the process exits. In host code the array's name is not
// a device address, so its address is looked up with cudaGetSymbolAddress on the
// first call made while that device is current (and again if the device's context
// has been destroyed and rebuilt since, which moves the array) and then handed to
// the kernels like any caller-provided workspace.
#include <mutex>

#include "dpo.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DPO_NOALLOC_SCRATCH_BYTES];

struct ScratchAddr {
  void* ctx = nullptr;
  void* ptr = nullptr;
};
std::mutex g_noalloc_mu;
ScratchAddr g_noalloc[256];

// Device address of the scratch array on the current device, cached per context.
dpo_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return DPO_ERR_CUDA;
  void* ctx = nullptr;
  if (!dpo::current_context(&ctx)) return DPO_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  ScratchAddr& a = g_noalloc[dev];
  if (a.ptr == nullptr || a.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return DPO_ERR_CUDA;
    a.ptr = p;
    a.ctx = ctx;
  }
  *out = a.ptr;
  return DPO_OK;
}

}  // namespace

extern "C" dpo_status dpo_seq_logprobs_noalloc(const dpo_batch* batch, int want_grad,
                                               float* seq_logp, float* tok_logp,
                                               float* lse_state, void* stream) {
  size_t need = 0;
  dpo_status s = dpo_workspace_size(batch, &need, nullptr, nullptr);
  if (s != DPO_OK) return s;
  // Batches whose scratch does not fit the built-in array are refused before
  // any device work; the caller should use dpo_seq_logprobs with a workspace.
  if (need > static_cast<size_t>(DPO_NOALLOC_SCRATCH_BYTES)) return DPO_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != DPO_OK) return s;
  // The forward writes every scratch byte it later reads (row tables, position
  // tables, packed rows, per-tile partials, per-position values), so the
  // previous call's contents need no clearing.
  return dpo_seq_logprobs(batch, want_grad, seq_logp, tok_logp, lse_state, scratch,
                          static_cast<size_t>(DPO_NOALLOC_SCRATCH_BYTES), stream);
}
