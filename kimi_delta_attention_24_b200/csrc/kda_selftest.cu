// Self-test of the device time-out path: one CTA waits, through the same bounded wait and the
// same uniform abort decision as the forward kernels, on an mbarrier phase that nothing ever
// completes.  The wait runs out after `limit_ns`, records KDA_ERR_DEVICE_TIMEOUT in the status
// word and every thread leaves; nothing faults, traps or hangs, and the context stays usable.
#include "kda_device.cuh"

namespace kda {
namespace {

__global__ void __launch_bounds__(128) wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);  // one arrival completes the phase; none ever comes
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) bounded_wait(&bar, 0, &abort_flag, status, limit_ns);
  // every thread learns of the expiry at one barrier, as the kernels' roles do before leaving
  if (__syncthreads_or(abort_flag)) return;
}

}  // namespace

cudaError_t launch_wait_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 128, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace kda
