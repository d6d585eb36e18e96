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

__device__ unsigned long long g_quot_count[2];  // pairs checked, mismatches

// splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): one 64-bit draw per counter value.
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// quot_rn against the IEEE division on n pseudo-random pairs (x, s): s with
// a random exponent in [-40, 20] and significand; x with a random exponent
// in [-40, 30] (a quarter of the pairs) or within 8 units in the last place
// of (m + 1/2) s for a random integer m in [-260, 260] (the rest: quotients
// next to a half-integer, where a wrong last bit would change a code).
__global__ void selftest_quot_kernel(uint64_t n, uint64_t seed) {
  unsigned long long checked = 0, bad = 0;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t h1 = mix64(seed ^ (2 * i)), h2 = mix64(seed ^ (2 * i + 1));
    const int es = (int)(h1 % 61) - 40;
    const float s = __uint_as_float((uint32_t)(es + 127) << 23 | (uint32_t)(h1 >> 40) & 0x7FFFFFu);
    float x;
    if ((h2 & 3) == 0) {
      const int ex = (int)((h2 >> 2) % 71) - 40;
      x = __uint_as_float((uint32_t)(h2 >> 63) << 31 | (uint32_t)(ex + 127) << 23 | (uint32_t)(h2 >> 20) & 0x7FFFFFu);
    } else {
      const int m = (int)((h2 >> 2) % 521) - 260;
      const float c = __fmul_rn((float)m + 0.5f, s);
      const int d = (int)((h2 >> 12) % 17) - 8;
      x = __uint_as_float(__float_as_uint(c) + (uint32_t)d);  // c is never 0: m + 1/2 != 0
    }
    if (!quot_in_range(x, s)) continue;
    ++checked;
    const float q = quot_rn(x, s, __frcp_rn(s));
    const float r = __fdiv_rn(x, s);
    if (__float_as_uint(q) != __float_as_uint(r)) ++bad;
  }
  atomicAdd(&g_quot_count[0], checked);
  atomicAdd(&g_quot_count[1], bad);
}

}  // namespace
}  // namespace gptq

extern "C" gptq_status_t gptq_selftest_quotient(uint64_t n, uint64_t seed, uint64_t* checked, uint64_t* mismatches,
                                                void* stream) {
  using namespace gptq;
  clear_error();
  if (!checked || !mismatches) return fail(GPTQ_ERR_INVALID_ARG, "checked and mismatches must not be NULL");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GPTQ_ERR_CUDA, "no CUDA device is available");
  const cudaStream_t st = (cudaStream_t)stream;
  unsigned long long c[2] = {0, 0};
  CUDA_TRY(cudaMemcpyToSymbolAsync(g_quot_count, c, sizeof(c), 0, cudaMemcpyHostToDevice, st));
  const DeviceInfo& di = device_info();
  selftest_quot_kernel<<<(unsigned)(di.sms * 8), 256, 0, st>>>(n, seed);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  CUDA_TRY(cudaMemcpyFromSymbolAsync(c, g_quot_count, sizeof(c), 0, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  *checked = c[0];
  *mismatches = c[1];
  return GPTQ_OK;
}

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
