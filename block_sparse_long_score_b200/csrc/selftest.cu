// selftest.cu -- exercises the failure-detection path of the library without
// a GPU fault: a kernel waits, with the library's bounded wait, on an
// mbarrier that nothing ever arrives on. The wait gives up after its time
// limit, the kernel records XATTN_ERR_TIMEOUT in the device status word and
// returns normally, and the context stays usable. This is the same path every
// pipeline wait of the scoring and attention kernels takes on a time-out.
#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace {

__global__ void __launch_bounds__(32) selftest_timeout_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  volatile int* abort = &abort_flag;
  // phase 0 never completes: nothing arrives on the barrier
  const bool ok = warp_wait(&bar, 0, abort);
  if (threadIdx.x == 0 && !ok && *abort) atomicExch(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_selftest_timeout(int* status, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(status);
  return cudaGetLastError();
}

}  // namespace xattn
