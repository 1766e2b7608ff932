// stem_selftest.cu — self-test of the device-side failure detection.
//
// Every pipeline wait in the Stem kernels is bounded (mbar_wait: 2 s of
// %globaltimer); on expiry the kernel records STEM_ERR_TIMEOUT in the
// workspace status word and returns instead of hanging.  This kernel waits,
// through that same function, on an mbarrier that nothing ever arrives on, so
// a caller (or a test) can check on a real GPU that the bound fires, that the
// status word reports it, and that the context stays usable afterwards.
#include "stem.h"
#include "stem_device.cuh"

namespace stem {
namespace {

__global__ void wait_timeout_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort, status);  // no thread ever arrives on `bar`
}

}  // namespace
}  // namespace stem

extern "C" stem_status_t stem_selftest_wait_timeout(void* ws, stem_stream_t stream) {
  if (!ws) return STEM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return STEM_ERR_CUDA;
  stem::wait_timeout_kernel<<<1, 32, 0, s>>>(static_cast<int*>(ws));
  return cudaGetLastError() == cudaSuccess ? STEM_OK : STEM_ERR_CUDA;
}
