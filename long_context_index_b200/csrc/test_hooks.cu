// test_hooks.cu -- hooks that let the tests exercise failure handling without
// faulting or hanging a GPU (declared in include/msa_testing.h).
#include <cstdint>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

// One thread waits on an mbarrier that nothing ever arrives on, with the
// given deadline; the bounded wait gives up, records the timeout in the
// status word and the kernel returns normally.
__global__ void never_ready_kernel(int* status, unsigned long long deadline_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx wc{&abort_flag, status};
    wc.deadline_ns = deadline_ns;
    mbar_wait(&bar, 0, wc);   // phase 0 never completes
  }
  __syncthreads();
}

}  // namespace
}  // namespace msa

extern "C" MSA_API int msa_test_never_ready_wait(void* ws, size_t ws_bytes, long long deadline_ns, void* stream) {
  if (!ws || ws_bytes < msa::kWsHeader || deadline_ns <= 0 || deadline_ns > 2000000000ll) return MSA_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return MSA_ERR_CUDA;
  msa::never_ready_kernel<<<1, 32, 0, st>>>(static_cast<int*>(ws), static_cast<unsigned long long>(deadline_ns));
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
