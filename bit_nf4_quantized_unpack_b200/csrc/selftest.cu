// selftest.cu -- a hook that exercises the failure path shared by every kernel of the
// library: a bounded mbarrier wait that runs out records an error for the host and the
// kernel exits, leaving the context usable. Not part of the method.
#include "internal.h"
#include "sm100.cuh"

namespace qlora {
namespace {

// One CTA waits on phase 0 of an mbarrier that nothing arrives at, with the library's
// bounded wait (mbar_wait: %globaltimer, kWaitTimeoutNs). The wait gives up, the thread
// records kErrTimeoutSelfTest in the device error word, and the CTA exits.
__global__ void k_wait_selftest(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag))
    record_error(err, &abort_flag, kErrTimeoutSelfTest);
}

}  // namespace

cudaError_t launch_wait_selftest(cudaStream_t st) {
  int* err = device_error_word();
  if (!err) return cudaErrorInvalidDevice;
  note_launches(1);
  k_wait_selftest<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

}  // namespace qlora
