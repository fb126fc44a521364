// Self-test of the kernels' bounded waits: one warp waits, with the same bounded mbarrier
// wait the attention kernel uses, on a barrier that nothing arrives on. The wait gives up
// after `limit` SM cycles, sets the time-out bit of the error word and returns, so a lost
// arrival surfaces to the caller while the CUDA context stays usable.
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace bsa {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(long long limit, uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) ptx::mbar_wait(ptx::smem_u32(&bar), 0, &abort_flag, err, limit);
}

}  // namespace

cudaError_t launch_wait_selftest(long long limit_cycles, uint32_t* err, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(limit_cycles, err);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bsa
