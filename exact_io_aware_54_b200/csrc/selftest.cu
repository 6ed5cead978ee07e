// selftest.cu -- exercises the bounded-wait failure path on the GPU.
//
// Every wait of the library's kernels is bounded: when a phase does not complete
// within the limit, the kernel records FA_ERR_TIMEOUT in the workspace status
// word and returns, so the context stays usable and fa_check reports it.  This
// kernel runs that path on purpose and nothing else: one thread initialises an
// mbarrier in shared memory that nothing ever arrives on, waits on it with the
// same bounded wait the kernels use, and records the expiry.  It issues no
// memory copy and touches no tensor memory.
#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

__global__ void wait_timeout_selftest_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0, timeout_ns)) atomicCAS(status, 0, kStatusTimeout);
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" FA_API fa_status fa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, unsigned timeout_us,
                                                     cudaStream_t stream) {
  if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return FA_ERR_WORKSPACE;
  if (timeout_us == 0 || timeout_us > 1000000u) return FA_ERR_INVALID_ARG;  // at most one second
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<int*>(workspace), 1000ull * timeout_us);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
