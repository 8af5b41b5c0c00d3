// Self-test of the bounded waits every kernel of the library relies on.
//
// The split-K and phase rendezvous, the grid barriers and the pipeline
// mbarriers all wait with a time limit (%globaltimer): when it expires the
// kernel records SPEC_DEVERR_TIMEOUT in an error word and returns, so that a
// lost arrival ends as an error the host reads instead of a hung GPU.  This
// entry point runs the same two primitives against a counter that nothing
// increments and an mbarrier that nothing arrives on, with a short limit, and
// reports what the host sees.  No fault, trap or endless loop is involved: the
// waits end by themselves and the context stays usable.
#include <cuda_runtime.h>

#include "../../include/spec.h"
#include "common.cuh"

namespace spec {
namespace {

// scratch: [0] a counter nothing increments, [1] error word, [2..3] the waits' results
__global__ void wait_selftest_kernel(int* scratch, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  uint32_t* err = reinterpret_cast<uint32_t*>(scratch + 1);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    scratch[2] = spin_until_geq(scratch, 1, err, limit_ns) ? 1 : 0;
    scratch[3] = mbar_wait(&bar, 0, err, nullptr, limit_ns) ? 1 : 0;
  }
}

}  // namespace
}  // namespace spec

extern "C" {

SPEC_API int spec_wait_selftest(void* device_scratch, uint32_t limit_us, int32_t* expired) {
  if (!device_scratch || !expired || limit_us == 0 || limit_us > 1000000u ||
      (reinterpret_cast<uintptr_t>(device_scratch) & 3u))
    return SPEC_ERR_ARG;
  int* s = static_cast<int*>(device_scratch);
  if (cudaMemset(s, 0, 16) != cudaSuccess) return SPEC_ERR_CUDA;
  spec::wait_selftest_kernel<<<1, 32>>>(s, (uint64_t)limit_us * 1000ull);
  if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return SPEC_ERR_CUDA;
  int h[4];
  if (cudaMemcpy(h, s, 16, cudaMemcpyDeviceToHost) != cudaSuccess) return SPEC_ERR_CUDA;
  // both waits must have given up, and the error word must say so
  *expired = (h[2] == 0 ? 1 : 0) + (h[3] == 0 ? 1 : 0);
  return (static_cast<uint32_t>(h[1]) & spec::SPEC_DEVERR_TIMEOUT) ? SPEC_ERR_TIMEOUT : SPEC_OK;
}

}  // extern "C"
