// moe_selftest_bounded_wait: a check of the bounded waits that every
// stage-ring kernel of this library uses (mbar_wait for a producer draining
// its copies, wait_or_abort for a consumer waiting for a stage), made on a
// stage whose bytes never arrive.
//
// One CTA of two warps. Warp 0 plays the producer: it arms an mbarrier for a
// 512-byte stage (arrive.expect_tx) and, when `deliver` is set, issues the
// bulk copy that fills it; otherwise nothing ever delivers those bytes. Warp 1
// plays a consumer and waits for the stage with wait_or_abort and a short
// limit; on a timeout it raises the CTA's abort flag, exactly as a ring
// kernel's consumer does. The producer then waits for its own stage with
// mbar_wait (the drain every ring kernel runs before it exits after an
// abort), also with a short limit. Thread 0 finally ORs kStatusWaitTimeout
// into the status word when the abort flag is up, the same last step as the
// ring kernels. No copy is ever in flight when a wait gives up (the stage
// that times out was never requested), so the CTA exits cleanly and the
// context stays usable.
#include <cuda_runtime.h>

#include "../../include/moe_mxfp4.h"
#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace moe {
namespace {

constexpr uint32_t kStageBytes = 512;

__global__ void __launch_bounds__(64) k_selftest_wait(int32_t* status, const uint8_t* src,
                                                      int deliver, uint32_t limit) {
  __shared__ __align__(128) uint8_t stage[kStageBytes];
  __shared__ __align__(8) uint64_t full;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&full, 1);
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(&full, kStageBytes);
      if (deliver) bulk_g2s(stage, src, kStageBytes, &full);
      // the drain before exit: wait for this stage's bytes (bounded)
      if (!mbar_wait(&full, 0, limit)) *abort = 1;
    }
  } else {
    if (!tc::wait_or_abort(&full, 0, abort, limit)) {
      if (lane == 0) *abort = 1;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(status, kStatusWaitTimeout);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_bounded_wait(int32_t* status, const void* src, int deliver,
                                                uint32_t limit, void* stream) {
  if (!status) return moe::record_error(MOE_ERR_INVALID_ARG, "status is NULL");
  if (deliver && (!src || (reinterpret_cast<uintptr_t>(src) & 15u)))
    return moe::record_error(MOE_ERR_ALIGNMENT, "src must be a 16-byte aligned device pointer");
  if (limit < 1 || limit > 4096)
    return moe::record_error(MOE_ERR_INVALID_ARG, "limit must be in [1, 4096] tries");
  moe::k_selftest_wait<<<1, 64, 0, (cudaStream_t)stream>>>(
      status, static_cast<const uint8_t*>(src), deliver ? 1 : 0, limit);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return moe::record_error(MOE_ERR_CUDA, cudaGetErrorString(e));
  return MOE_OK;
}
