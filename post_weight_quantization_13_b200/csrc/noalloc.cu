// gptq_quantize_layer_noalloc: the quantize sweep on a fixed device scratch,
// for callers that cannot allocate device memory.  The scratch is a static
// device array.  Its address is looked up once per device context (set-up)
// and cached together with the context's id, so a context created after a
// device reset gets its own look-up.  The work itself is
// gptq_quantize_layer's, called with that scratch as the workspace.
#include <map>
#include <mutex>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {
namespace {

__device__ __align__(256) unsigned char g_static_scratch[GPTQ_STATIC_SCRATCH_BYTES];

typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

CtxGetIdFn ctx_get_id_fn() {
  static CtxGetIdFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetIdFn)p;
  });
  return fn;
}

struct ScratchEntry {
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};
std::map<int, ScratchEntry> g_scratch;  // device ordinal -> set-up of its current context
std::mutex g_scratch_mu;

// Id of the calling thread's current context (false if there is none yet).
bool current_ctx_id(unsigned long long* id) {
  CtxGetIdFn fn = ctx_get_id_fn();
  return fn && fn(nullptr, id) == CUDA_SUCCESS;
}

// Address of the current device's copy of g_static_scratch.  Set-up, once per
// device context, with that device current: cudaGetSymbolAddress (which
// creates the primary context if this thread has none yet), then every kernel
// the quantize call can launch is loaded on the device, so that later calls
// neither resolve symbols nor load device code.
gptq_status_t static_scratch(void** addr) {
  int d = -1;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return fail(GPTQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  unsigned long long id = 0;
  const bool have_ctx = current_ctx_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& ent = g_scratch[d];
  if (have_ctx && ent.addr && ent.ctx_id == id) {
    *addr = ent.addr;
    return GPTQ_OK;
  }
  void* ptr = nullptr;
  e = cudaGetSymbolAddress((void**)&ptr, g_static_scratch);
  if (e != cudaSuccess)
    return fail(GPTQ_ERR_CUDA, "cudaGetSymbolAddress of the static scratch on device %d: %s", d,
                cudaGetErrorString(e));
  if (!current_ctx_id(&id)) return fail(GPTQ_ERR_CUDA, "no current CUDA context on device %d", d);
  e = preload_quantize_kernels();
  if (e == cudaSuccess) e = preload_gemm_kernels();
  if (e == cudaSuccess) e = preload_simt_kernels();
  if (e != cudaSuccess)
    return fail(GPTQ_ERR_CUDA, "loading the quantize kernels on device %d: %s", d, cudaGetErrorString(e));
  ent.ctx_id = id;
  ent.addr = ptr;
  *addr = ptr;
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

extern "C" gptq_status_t gptq_quantize_layer_noalloc_status(void* stream) {
  using namespace gptq;
  clear_error();
  void* ws = nullptr;
  gptq_status_t s = static_scratch(&ws);
  if (s != GPTQ_OK) return s;
  return gptq_workspace_status(ws, GPTQ_STATIC_SCRATCH_BYTES, stream);
}
