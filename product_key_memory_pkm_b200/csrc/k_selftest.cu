// Self-test of the bounded-wait path: one warp waits on an mbarrier that nothing
// arrives on, with a short clock budget.  The wait gives up, records
// PKM_ERR_DEVICE_TIMEOUT in the device status word and the kernel returns; the
// context stays usable.  This exercises exactly the code every tcgen05 kernel uses
// for its waits, without faulting, trapping or hanging the GPU.
#include "tc_common.cuh"

namespace pkm {
namespace {

__global__ void wait_timeout_probe(long long budget_cycles, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: no thread arrives
    (void)tc::mbar_wait(&bar, 0, &abort_flag, status, budget_cycles);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_probe(long long budget_cycles, int* status, cudaStream_t st) {
  wait_timeout_probe<<<1, 32, 0, st>>>(budget_cycles, status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace pkm
