// Failure-detection self-test: a device wait on a barrier that nothing
// completes must give up after its bounded limit, record MLRA_ERR_TIMEOUT in
// the caller's error record and return, leaving the context usable.  It runs
// the same bounded-wait helper every kernel of the library uses, with a short
// limit instead of the ~2 s one.
#include "../../include/mlra.h"
#include "launch.h"
#include "ptx.cuh"

namespace mlra {
namespace {

using namespace ptx;

constexpr int kSiteSelfTest = 99;

__global__ void wait_timeout_kernel(int* err, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);  // one arrival expected, none ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, err, kSiteSelfTest, limit);
}

}  // namespace
}  // namespace mlra

extern "C" MLRA_API mlra_status mlra_selftest_wait_timeout(void* workspace, long long limit_cycles,
                                                            cudaStream_t stream) {
  if (!workspace) return mlra::internal_fail(MLRA_ERR_INVALID_ARG, "workspace is NULL");
  if (limit_cycles < 1 || limit_cycles > 4000000000LL)
    return mlra::internal_fail(MLRA_ERR_INVALID_ARG, "limit_cycles must be in [1, 4e9]");
  mlra::wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<int*>(workspace), limit_cycles);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return mlra::internal_fail(MLRA_ERR_CUDA, cudaGetErrorString(e));
  return MLRA_OK;
}
