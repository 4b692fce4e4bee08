// Self-test of the bounded-wait path that every tensor-core kernel relies on: one thread waits,
// through the same mbarrier wait, on a barrier that nothing ever arrives at.  The wait gives up
// after the given number of SM cycles, raises the CTA's abort flag and the kernel reports
// BHA_ERR_TIMEOUT through dev_err, exactly as a stalled pipeline would; no TMA copy, MMA or
// TMEM allocation is involved, so nothing is left in flight.
#include <cuda_runtime.h>

#include "../../include/bha.h"
#include "common.cuh"
#include "tc_util.cuh"

namespace bha {
namespace {

__global__ void bounded_wait_selftest_kernel(long long limit_cycles, int32_t* dev_err) {
  __shared__ uint64_t never_arrives;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&never_arrives, 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* flag = &abort_flag;
    const bool ok = tc::mbar_wait(&never_arrives, 0, flag, limit_cycles);
    if (!ok && abort_flag) set_error(dev_err, BHA_ERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace bha

extern "C" int bha_selftest_bounded_wait(int64_t limit_cycles, int32_t* dev_err, void* stream) {
  if (dev_err == nullptr || limit_cycles < 1 || limit_cycles > 4000000000ll) return BHA_ERR_INVALID;
  bha::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (long long)limit_cycles, dev_err);
  return cudaGetLastError() == cudaSuccess ? BHA_OK : BHA_ERR_CUDA;
}
