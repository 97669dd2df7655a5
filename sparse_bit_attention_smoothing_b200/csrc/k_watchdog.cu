// k_watchdog.cu -- a deliberate bounded-wait expiry, to exercise the
// failure-detection path of the library on the GPU without faulting it.
//
// Every device-side wait of the library is bounded; when one gives up the
// kernel records it in the per-device watchdog word, which
// sagesla_sync_status() reports (and clears).  This kernel waits on an
// mbarrier that nothing will ever arrive on, for a given number of probes,
// then records the expiry exactly as the pipeline kernels do and returns.
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

__global__ void watchdog_selftest_kernel(int probes, int* wd) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none is ever made
    mbar_fence_init();
    bool done = false;
    for (int i = 0; i < probes && !done; ++i) done = mbar_try(&bar, 0);
    if (!done) atomicExch(wd, 1);
  }
}

cudaError_t launch_watchdog_selftest(int probes, int* wd, cudaStream_t st) {
  watchdog_selftest_kernel<<<1, 32, 0, st>>>(probes, wd);
  return cudaGetLastError();
}

}  // namespace sagesla
