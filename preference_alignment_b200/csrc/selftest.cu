// Self-test of the bounded waits: a one-CTA kernel waits, with the same
// mbar_wait every GEMM role uses, on an mbarrier that nothing ever arrives on.
// The wait must give up after the budget, record DPO_ERR_TIMEOUT in the status
// word and let the kernel exit normally, leaving the context usable.
#include "internal.h"

namespace dpo {

__global__ void k_wait_selftest(DevCtl ctl) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(smem_u32(&bar), 0, ctl, &abort_flag)) record_status(ctl, kStatusTimeout);
  }
  __syncthreads();
}

cudaError_t launch_wait_selftest(const DevCtl& ctl, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(ctl);
  return cudaGetLastError();
}

}  // namespace dpo

