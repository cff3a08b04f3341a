// squad_wait_selftest: exercises the bounded device-side wait used by every kernel of this library on a
// barrier that nothing completes, so that the timeout path (record the status, give up, return) can be
// tested without faulting or hanging a GPU.
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "squad_attn.h"

namespace squad {
namespace {

__global__ void wait_selftest_kernel(uint32_t* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival would complete phase 0; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  WaitCtl ctl{&abort_flag, status, timeout_ns};
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ctl);   // gives up after timeout_ns, records kStatusTimeout
  __syncthreads();
}

}  // namespace
}  // namespace squad

extern "C" squad_status_t squad_wait_selftest(uint32_t* status, unsigned long long timeout_ns, squad_stream_t stream) {
  if (status == nullptr || (reinterpret_cast<uintptr_t>(status) & 3u) != 0) return SQUAD_ERR_INVALID_ARG;
  if (timeout_ns == 0 || timeout_ns > 1000000000ull) return SQUAD_ERR_INVALID_ARG;
  squad::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
}
