// Self-test of the bounded device waits.  Every wait in the library's kernels
// (mbarrier phases inside a CTA, completion counters between CTAs) gives up
// after a clock budget of about a second, reports MOE_ERR_TIMEOUT through the
// workspace status word and lets the kernel return, so a lost arrival never
// hangs the GPU.  This kernel makes both kinds of wait run out on purpose:
// it waits on an mbarrier that nothing arrives on and on a counter that
// nothing increments, with the same helpers the kernels use.
//
// A second self-test kernel occupies some of the SMs for a fixed time while
// the layer runs on another stream: the layer must then finish on the SMs
// that are left, which checks that no wait inside it depends on CTAs that are
// not resident.
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

__device__ int g_never_incremented = 0;  // no code ever writes it

__global__ void bounded_wait_selftest_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool got_phase = ptx::mbar_wait(&bar, 0, &abort);  // no arrival will come
    abort = 0;
    const bool got_count = ptx::counter_wait(&g_never_incremented, 1, &abort);
    if (!got_phase && !got_count && status) atomicOr(status, kStTimeout);
  }
}

// Holds the SM it runs on for `cycles` SM clock cycles, then returns; it
// waits on nothing but its own clock.  Its dynamic shared memory is sized so
// that no CTA of the expert FFN (over 200 KB each) fits beside it.
__global__ void occupy_kernel(long long cycles) {
  extern __shared__ uint8_t hold[];
  const long long t0 = clock64();
  while (clock64() - t0 < cycles) __nanosleep(1000);
  if (threadIdx.x == 0) hold[0] = 0;
}

}  // namespace

cudaError_t launch_occupy_selftest(int nctas, long long cycles, cudaStream_t st) {
  constexpr int kHoldBytes = 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(occupy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kHoldBytes);
  if (e != cudaSuccess) return e;
  occupy_kernel<<<nctas, 32, kHoldBytes, st>>>(cycles);
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_selftest(int* status, cudaStream_t st) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(status);
  return cudaGetLastError();
}

}  // namespace moe
