// gptq_quantize_layer_noalloc: the quantize sweep on a fixed device scratch,
// for callers that cannot allocate device memory.  The scratch is a static
// device array; its address is looked up once per device and cached.  The
// work itself is gptq_quantize_layer's, called with that scratch as the
// workspace.
#include <mutex>

#include "internal.cuh"

namespace gptq {
namespace {

__device__ __align__(256) unsigned char g_static_scratch[GPTQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
void* g_scratch_addr[kMaxScratchDevices];
std::mutex g_scratch_mu;

// Address of this device's copy of g_static_scratch (the current device's).
gptq_status_t static_scratch(void** addr) {
  int d = -1;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return fail(GPTQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (d < 0 || d >= kMaxScratchDevices)
    return fail(GPTQ_ERR_UNSUPPORTED, "device %d: the static scratch is kept for devices 0..%d only", d,
                kMaxScratchDevices - 1);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[d]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_static_scratch);
    if (e != cudaSuccess)
      return fail(GPTQ_ERR_CUDA, "cudaGetSymbolAddress of the static scratch on device %d: %s", d,
                  cudaGetErrorString(e));
    g_scratch_addr[d] = ptr;
  }
  *addr = g_scratch_addr[d];
  return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

extern "C" gptq_status_t gptq_quantize_layer_noalloc(const void* W, gptq_dtype_t wt, int64_t out, int64_t in,
                                                     int64_t ldw, const float* U, const int32_t* perm,
                                                     const uint8_t* dead, const gptq_config_t* cfg, int32_t* codes,
                                                     uint32_t* qweight, float* scales, int32_t* zeros,
                                                     int32_t* g_idx, float* loss, void* stream) {
  using namespace gptq;
  gptq_status_t s = gptq_validate_config(cfg, out, in);
  if (s != GPTQ_OK) return s;
  if (out == 0)  // a no-op, as for gptq_quantize_layer: no scratch needed
    return gptq_quantize_layer(W, wt, out, in, ldw, U, perm, dead, cfg, codes, qweight, scales, zeros, g_idx,
                               loss, nullptr, 0, stream);
  const size_t need = quantize_ws_bytes(out, in, cfg);
  if (need > GPTQ_STATIC_SCRATCH_BYTES)
    return fail(GPTQ_ERR_WORKSPACE,
                "layer %lld x %lld (block_size %d) needs %zu bytes of scratch; the static scratch holds %zu: "
                "use gptq_quantize_layer with a caller workspace",
                (long long)out, (long long)in, cfg->block_size, need, (size_t)GPTQ_STATIC_SCRATCH_BYTES);
  void* ws = nullptr;
  s = static_scratch(&ws);
  if (s != GPTQ_OK) return s;
  return gptq_quantize_layer(W, wt, out, in, ldw, U, perm, dead, cfg, codes, qweight, scales, zeros, g_idx, loss,
                             ws, GPTQ_STATIC_SCRATCH_BYTES, stream);
}
