// Self-test of the failure detection shared by every pipelined kernel: a bounded mbarrier
// wait on a barrier that nothing ever completes must give up, record TIMEOUT in the
// workspace's status header and raise the CTA's abort flag, and a second warp waiting on
// the same barrier must then give up through the abort flag (without recording anything).
// The kernel ends by itself within the given limit; the CUDA context stays usable.
#include "bsa_kernels.cuh"

namespace bsa {

__global__ void __launch_bounds__(64) selftest_wait_kernel(uint32_t* status, uint64_t limit_ns,
                                                           uint32_t* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none ever comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* ab = &abort_flag;
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait_for(&bar, 0, ab, status, DETAIL_SELFTEST, limit_ns);
    result[0] = ok ? 1u : 0u;  // expected 0: the wait gave up
  } else if (threadIdx.x == 32) {
    // waits far longer than thread 0's limit; leaves through the abort flag
    const bool ok = mbar_wait_for(&bar, 0, ab, status, DETAIL_SELFTEST + 1, 8 * limit_ns);
    result[1] = ok ? 1u : 0u;  // expected 0
    result[2] = static_cast<uint32_t>(*ab);  // expected 1
  }
}

cudaError_t launch_selftest_wait(void* ws, uint64_t limit_ns, cudaStream_t stream) {
  uint32_t* status = static_cast<uint32_t*>(ws);
  // results after the status words the header defines (word 0 flags, 1 detail, 2-3 place)
  uint32_t* result = status + 8;
  selftest_wait_kernel<<<1, 64, 0, stream>>>(status, limit_ns, result);
  return cudaGetLastError();
}

// The compute capability the library's device code was built for (major * 10 + minor), as
// the runtime reports it for a kernel of this library: 100 for sm_100a.
cudaError_t kernel_binary_version(int* version) {
  cudaFuncAttributes attr;
  const cudaError_t e = cudaFuncGetAttributes(&attr, selftest_wait_kernel);
  if (e == cudaSuccess) *version = attr.binaryVersion;
  return e;
}

}  // namespace bsa
