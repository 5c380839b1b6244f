// Failure-path probe: one bounded wait, through the same mbarrier helper the
// kernels use, on a barrier phase that can never complete (it needs two
// arrivals and gets one).  The wait must give up after its cycle limit, record
// MOE_ERR_TIMEOUT in the workspace's status word and return, leaving the
// context usable -- the behaviour every wait in the library relies on instead
// of a trap or an endless spin.
#include "moe_internal.cuh"

namespace {

__global__ void wait_probe_kernel(int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    moe::mbar_init(&bar, 2);
    moe::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    moe::mbar_arrive(&bar);                       // one of the two arrivals the phase needs
    if (!moe::mbar_wait(&bar, 0, nullptr)) moe::report_error(status, MOE_ERR_TIMEOUT, 77);
  }
}

}  // namespace

extern "C" int moe_debug_wait_probe(void* workspace, void* stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0) return MOE_ERR_INVALID_ARG;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(workspace));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
