// gptq_selftest_wait_timeout: exercises the bounded-wait path every kernel
// of this library relies on.  One thread waits on an mbarrier that nothing
// ever arrives on; the wait gives up after limit_ns of %globaltimer and
// raises the timeout flag in a status word, which the host then reads.  No
// fault, trap or unbounded spin is involved, and the context stays usable.
#include "internal.cuh"

namespace gptq {
namespace {

__device__ uint32_t g_selftest_status;

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    g_selftest_status = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    bool done = false;
    while (!done) {
      if (mbar_try_wait(&bar, 0)) break;  // never completes: no arrival
      done = globaltimer() - t0 > limit_ns;
    }
    if (done) atomicOr(&g_selftest_status, ST_TIMEOUT);
  }
}

}  // namespace
}  // namespace gptq

extern "C" gptq_status_t gptq_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  using namespace gptq;
  clear_error();
  if (limit_ns == 0 || limit_ns > (uint64_t)kWaitLimitNs)
    return fail(GPTQ_ERR_INVALID_ARG, "limit_ns must be in [1, %llu]", (unsigned long long)kWaitLimitNs);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GPTQ_ERR_CUDA, "no CUDA device is available");
  const cudaStream_t st = (cudaStream_t)stream;
  selftest_wait_kernel<<<1, 32, 0, st>>>(limit_ns);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  uint32_t status = 0;
  CUDA_TRY(cudaMemcpyFromSymbolAsync(&status, g_selftest_status, sizeof(status), 0, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (status & ST_TIMEOUT) return fail(GPTQ_ERR_TIMEOUT, "the bounded wait gave up after %llu ns, as intended",
                                       (unsigned long long)limit_ns);
  return fail(GPTQ_ERR_CUDA, "the bounded wait did not report its timeout");
}
