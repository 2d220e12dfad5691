// Diagnostic: make one bounded barrier wait run out on purpose.
//
// Every wait of the library's kernels is an mbarrier wait bounded in time:
// when it runs out, the kernel records the wait's site in the device error
// word, raises its CTA's abort flag and returns, and rib_device_error()
// reports RIB_ERR_TIMEOUT. This kernel exercises exactly that path with a
// short limit: one warp waits on a barrier that nothing ever arrives on, so
// the GPU never faults or hangs and the context stays usable afterwards.
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kSelftestSite = 901;

__global__ void selftest_wait_kernel(unsigned long long limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // nothing arrives: phase 0 never completes
    abort_flag = 0u;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, err};
  if (!mbar_try_wait(&bar, 0)) mbar_wait_slow(&bar, 0, wc, kSelftestSite, limit_ns);
  __syncthreads();
}

}  // namespace

}  // namespace rib

using namespace rib;

extern "C" rib_status rib_selftest_wait_timeout(int limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 1000000)
    return fail(RIB_ERR_INVALID_ARG, "rib_selftest_wait_timeout: limit_us must be in 1..1000000");
  int* err = device_error_word();
  if (!err) return fail(RIB_ERR_CUDA, "rib_selftest_wait_timeout: no device error word");
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_us) * 1000ull, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rib_selftest_wait_timeout launch");
  return RIB_OK;
}
