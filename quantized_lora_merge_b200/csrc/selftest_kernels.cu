// Self-test of the bounded device waits and of their report to the host.
//
// Every tensor-core kernel of the library waits on mbarriers through
// mbar_wait (tcgen05_util.cuh): a wait that does not complete within its
// limit is counted in a device word, the CTA is told to stop and the kernel
// returns, so a broken pipeline yields an error status on the host instead of
// a hung GPU. This kernel exercises that path on purpose without any TMA copy
// or tensor-core product in flight: one thread initialises an mbarrier that
// expects one arrival, nobody arrives, and the thread waits on it with a
// short limit. The wait gives up, the count moves, the kernel returns, and
// intlora_device_status() reports INTLORA_ERR_TIMEOUT.
#include <cuda_runtime.h>

#include <cstdint>

#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

__device__ unsigned int g_selftest_timeouts;

__global__ void selftest_wait_kernel(uint64_t limit_ns, int* completed) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  tc::mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const bool ok = tc::mbar_wait_for(&bar, 0u, &abort_flag, &g_selftest_timeouts, limit_ns);
  if (completed != nullptr) *completed = ok ? 1 : 0;
}

}  // namespace

cudaError_t launch_selftest_wait(uint64_t limit_ns, int* completed, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, completed);
  return counted(cudaGetLastError());
}

unsigned int selftest_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_selftest_timeouts, sizeof v);
  return v;
}

}  // namespace intlora
