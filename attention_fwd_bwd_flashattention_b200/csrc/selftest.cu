// Self-test of the bounded device waits that every tensor-core kernel relies on.
//
// One warp waits on an mbarrier that nothing arrives at, through the same wait
// routine the kernels use (with a caller-chosen limit instead of their 2 s).  The
// wait must give up after the limit, raise the CTA's abort flag, write
// RELPOS_ERR_TIMEOUT to the status word, and the kernel must return, leaving the
// context usable.  The time the wait took is reported as well.
#include "common.cuh"
#include "relpos_attn.h"
#include "tc_ptx.cuh"

namespace rp {
namespace tc {

__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(int32_t *status, unsigned long long *elapsed_ns,
                                                              uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);  // one arrival expected; none ever comes
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    const bool done = mbar_wait_for(b, 0, &abort_flag, status, RELPOS_ERR_TIMEOUT_DEV, limit_ns);
    *elapsed_ns = (unsigned long long)(globaltimer() - t0);
    if (done) *status = RELPOS_OK;  // not reachable: the phase never completes
  }
}

}  // namespace tc
}  // namespace rp

extern "C" int relpos_selftest_wait(uint64_t limit_ns, int32_t *dev_status, unsigned long long *dev_elapsed_ns,
                                    void *stream) {
  cudaGetLastError();  // an error left by an earlier, unrelated call in this thread is not ours
  if (!dev_status || !dev_elapsed_ns || limit_ns < 1000000ull || limit_ns > 10000000000ull) return RELPOS_ERR_INVALID_ARG;
  cudaPointerAttributes a1, a2;
  if (cudaPointerGetAttributes(&a1, dev_status) != cudaSuccess || cudaPointerGetAttributes(&a2, dev_elapsed_ns) != cudaSuccess) {
    cudaGetLastError();
    return RELPOS_ERR_INVALID_ARG;
  }
  if ((a1.type != cudaMemoryTypeDevice && a1.type != cudaMemoryTypeManaged) ||
      (a2.type != cudaMemoryTypeDevice && a2.type != cudaMemoryTypeManaged))
    return RELPOS_ERR_INVALID_ARG;
  rp::tc::wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dev_status, dev_elapsed_ns, limit_ns);
  return cudaGetLastError() == cudaSuccess ? RELPOS_OK : RELPOS_ERR_LAUNCH;
}
