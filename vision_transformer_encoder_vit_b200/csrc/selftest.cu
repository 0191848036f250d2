// Self-test of the library's failure detection: every wait in the kernels is bounded,
// and a wait that runs out must leave an error the host can read, with the CUDA
// context still usable.  The test kernel waits on an mbarrier that nothing ever
// arrives on; the bounded wait gives up after VT_WAIT_LIMIT_NS and records
// VT_DEVERR_TIMEOUT, which vt_check() reports as VT_ERR_TIMEOUT.  No fault, trap or
// endless loop is involved.
#include "../../include/vt.h"
#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

__device__ unsigned int g_selftest_err;

__global__ void wait_that_runs_out_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing arrives on `bar`, so phase 0 never completes: the wait must give up.
    mbar_wait(&bar, 0, &abort_flag, &g_selftest_err);
  }
}

}  // namespace

unsigned int selftest_read_clear_error(cudaStream_t stream) {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_selftest_err, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return 0;
  cudaStreamSynchronize(stream);
  if (v) {
    cudaMemcpyToSymbolAsync(g_selftest_err, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    cudaStreamSynchronize(stream);
  }
  return v;
}

}  // namespace vt

extern "C" vt_status vt_selftest_wait_timeout(void* stream) {
  vt::wait_that_runs_out_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  if (cudaGetLastError() != cudaSuccess) {
    vt::set_error_message("vt_selftest_wait_timeout: launch failed");
    return VT_ERR_CUDA;
  }
  return VT_OK;
}
