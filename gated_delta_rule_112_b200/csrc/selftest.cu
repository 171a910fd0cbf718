// gdn_selftest_wait_timeout: checks, on the device, that a bounded wait that
// can never complete gives up instead of hanging, records the timeout in the
// workspace error word, and leaves the context usable. It runs the same
// bounded mbarrier wait the chunked-forward kernels use (about 1 s of SM
// clock), on a barrier that nothing arrives on.
#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

__global__ void __launch_bounds__(32) gdn_wait_selftest_kernel(uint32_t *ctrl) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);      // expects one arrival; none will come
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, ctrl, &abort_flag);
}

}  // namespace
}  // namespace gdn

extern "C" int gdn_selftest_wait_timeout(void *workspace, void *stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) return GDN_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 256, s) != cudaSuccess) return GDN_ERR_CUDA;
  gdn::gdn_wait_selftest_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t *>(workspace));
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
