// Self-test of the bounded device-side wait (mbar_wait) that every kernel of
// the library uses: a wait that nobody completes must give up after its limit
// and leave SKV_ETIMEOUT in the workspace status word, without a fault and
// with the context still usable.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace skv {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int* status, unsigned long long limit_ns, int arrive) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(&bar);
    mbar_wait(&bar, 0, status, limit_ns);  // records kStatusTimeout when it gives up
  }
}

}  // namespace
}  // namespace skv

extern "C" int skv_wait_selftest(void* ws, uint64_t limit_ns, int arrive, skv_stream_t stream_) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return SKV_EINVAL;
  if (limit_ns < 1 || limit_ns > 10000000000ull) return SKV_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int), stream);
  if (e == cudaSuccess) {
    skv::wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<int*>(ws), limit_ns, arrive);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? SKV_OK : skv::skv_record_cuda_error(static_cast<int>(e));
}
