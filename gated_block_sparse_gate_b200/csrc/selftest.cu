// selftest.cu — exercises the expiry branch of the bounded mbarrier wait.
//
// Every pipeline wait of the tensor-core kernels goes through sm100::mbar_wait,
// which gives up after a time limit, records GBS_ERR_TIMEOUT in the device
// error word and lets the kernel drain and return instead of hanging. In a
// correct run that branch never executes. This kernel makes it execute: one
// thread waits, through the same helper, on a shared-memory mbarrier that
// nothing arrives at, so the wait expires after `limit_ns` and the status lands
// in the caller's error word. Nothing faults or traps; the context stays usable.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace {

__global__ void wait_expiry_kernel(unsigned int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  gbs::sm100::mbar_init(&bar, 1);  // one arrival expected; none will come
  abort_flag = 0;
  gbs::sm100::fence_barrier_init();
  gbs::sm100::mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
}

}  // namespace

extern "C" gbs_status gbs_selftest_wait_timeout(void* ws, unsigned int limit_us, void* stream) {
  gbs::set_last_error("");
  if (!ws || ((uintptr_t)ws & 255u)) {
    gbs::set_last_error("gbs_selftest_wait_timeout: workspace is NULL or not 256-byte aligned");
    return GBS_ERR_WORKSPACE;
  }
  if (limit_us == 0 || limit_us > 1000000u) {
    gbs::set_last_error("gbs_selftest_wait_timeout: limit_us must be in [1, 1000000]");
    return GBS_ERR_INVALID_ARG;
  }
  wait_expiry_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(static_cast<unsigned int*>(ws),
                                                       (uint64_t)limit_us * 1000ull);
  gbs::note_launch();
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    gbs::set_last_error(cudaGetErrorString(e));
    return GBS_ERR_CUDA;
  }
  return GBS_OK;
}
