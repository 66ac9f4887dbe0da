// selftest.cu -- a kernel whose bounded wait is meant to run out, so that the
// timeout path of the library's waits (record the error and the site, give up,
// return) can be checked on a GPU without breaking a real kernel.
//
// One thread waits, with the caller's limit, through the same helpers the
// library's kernels use, on a condition nothing in the kernel satisfies:
//   which 0: an mbarrier phase no thread arrives on (mbar_wait, site 0x70);
//   which 1: a counter no thread increments (counter_wait, site 0x71).
// Nothing is in flight while it waits (no copy, no MMA, no TMEM), so giving
// up needs no draining: the thread records the timeout and the CTA returns.
#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

__global__ void selftest_wait_kernel(int which, long long limit, unsigned int *err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ unsigned int ctr;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    ctr = 0u;
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (which == 0)
      (void)mbar_wait(&bar, 0, &abort_flag, err, 0x70u, limit);
    else
      (void)counter_wait(&ctr, 1u, err, 0x71u, limit);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_wait(int which, long long limit_cycles, unsigned int *err, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(which, limit_cycles, err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace nsa
