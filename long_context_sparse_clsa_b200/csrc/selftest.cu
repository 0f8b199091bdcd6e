// Failure-detection self-test: a wait that nothing will satisfy, to show that the
// library's bounded waits end with a status the host can read instead of hanging.
//   which = 0: the inter-CTA count barrier (count_barrier) of the fused decode step,
//              for two CTAs, launched with one: the second arrival never comes.
//   which = 1: an mbarrier phase (mbar_wait) of the tensor-core pipelines that expects
//              one arrival, and none is made.
// Either wait runs out after kWaitLimitNs of globaltimer, records CLSA_ERR_TIMEOUT (detail
// 900 + which) in the workspace error word and returns; the CTA then exits normally, so
// the context stays usable.  Nothing faults or traps.
#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

__global__ void __launch_bounds__(32) selftest_timeout_kernel(int which, uint32_t* word, void* ws_header) {
  if (which == 0) {
    (void)count_barrier(word, 2u, ws_header, 900);
  } else {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
      mbar_init(&bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0)) record_error(ws_header, CLSA_ERR_TIMEOUT, 901);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_selftest_timeout(int which, void* ws_header, void* ws_body, cudaStream_t s) {
  uint32_t* word = static_cast<uint32_t*>(ws_body);
  cudaError_t e = cudaMemsetAsync(word, 0, sizeof(uint32_t), s);  // a fresh barrier word
  if (e != cudaSuccess) return e;
  selftest_timeout_kernel<<<1, 32, 0, s>>>(which, word, ws_header);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace clsa
