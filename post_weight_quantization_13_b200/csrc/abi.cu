// extern "C" entry points of libgptq.so (declared in include/gptq.h):
// argument validation (the pages' config validator, AutoGPTQ artifact page),
// workspace checks, error messages, device checks, and dispatch to the
// kernels.  No entry point allocates device memory.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <map>
#include <mutex>
#include <string>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {

namespace {
thread_local std::string g_last_error;
constexpr int64_t kMaxIn = 32768;
constexpr int64_t kMaxOut = 65535;
}  // namespace

gptq_status_t fail(gptq_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

void clear_error() { g_last_error.clear(); }

gptq_status_t read_device_status(const PrepHeader* hdr, cudaStream_t st) {
  uint32_t status = 0;
  CUDA_TRY(cudaMemcpyAsync(&status, &hdr->status, sizeof(status), cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (status & ST_TIMEOUT) return fail(GPTQ_ERR_TIMEOUT, "a bounded device-side wait gave up");
  if (status & ST_NONFINITE) return fail(GPTQ_ERR_NONFINITE, "S holds NaN or Inf");
  if (status & ST_NOT_PD) return fail(GPTQ_ERR_NOT_PD, "the damped Hessian is not positive definite");
  return GPTQ_OK;
}

namespace {
std::atomic<uint64_t> g_launches{0};
}
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool force_simt() {
  static const bool on = [] {
    const char* v = getenv("GPTQ_FORCE_SIMT");
    return v && atoi(v) != 0;
  }();
  return on;
}

cudaError_t ensure_smem_limit(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;  // (kernel, device) -> bytes
  int d = 0;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int& cur = done[{func, d}];
  if (cur >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
}

const DeviceInfo& device_info() {
  // one entry per device ordinal, created on first use; entries are never
  // moved or freed, so the returned reference stays valid
  static std::map<int, DeviceInfo> infos;
  static std::mutex mu;
  static const DeviceInfo none;
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0) return none;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& di = infos[d];
  if (di.id != d) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, d) != cudaSuccess) return none;
    di.sms = prop.multiProcessorCount;
    di.major = prop.major;
    di.minor = prop.minor;
    di.id = d;
  }
  return di;
}

gptq_status_t hessian_accumulate(float* S, int64_t in, const void* X, gptq_dtype_t xt, int64_t tokens, int64_t ldx,
                                 cudaStream_t st) {
  const DeviceInfo& dev = device_info();
  GemmArgs g;
  g.op = xt == GPTQ_F16 ? OP_F16 : xt == GPTQ_BF16 ? OP_BF16 : OP_TF32X3;
  g.P = {X, nullptr, in, tokens, ldx};
  g.Q = g.P;
  g.R = in;
  g.Cn = in;
  g.K = tokens;
  g.C = S;
  g.ldc = in;
  g.alpha = 1.f;
  g.beta = 1.f;
  g.mask = 1;
  g.tri = 1;
  cudaError_t e;
  if (xt != GPTQ_F32 && !force_simt() && tc_gemm_supported(g))
    e = tc_gemm(g, st, dev.sms);
  else
    e = simt_gemm(g, st);
  CUDA_TRY(e);
  return GPTQ_OK;
}

namespace {

gptq_status_t check_device() {
  const DeviceInfo& d = device_info();
  if (d.id < 0) return fail(GPTQ_ERR_CUDA, "no CUDA device is available");
  if (d.major != 10 || d.minor != 0)
    return fail(GPTQ_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device is sm_%d%d", d.major,
                d.minor);
  return GPTQ_OK;
}

gptq_status_t check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(GPTQ_ERR_WORKSPACE, "workspace pointer is NULL");
  if (((uintptr_t)ws & 255u) != 0) return fail(GPTQ_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (ws_bytes < need)
    return fail(GPTQ_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  return GPTQ_OK;
}

bool dtype_ok(gptq_dtype_t t) { return t == GPTQ_F16 || t == GPTQ_BF16 || t == GPTQ_F32; }

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" {

int gptq_abi_version(void) { return GPTQ_ABI_VERSION; }

uint64_t gptq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gptq_last_error(void) { return g_last_error.c_str(); }

gptq_status_t gptq_validate_config(const gptq_config_t* cfg, int64_t out, int64_t in) {
  clear_error();
  if (!cfg) return fail(GPTQ_ERR_INVALID_ARG, "config is NULL");
  if (in < 1) return fail(GPTQ_ERR_INVALID_ARG, "in must be >= 1 (got %lld)", (long long)in);
  if (out < 0) return fail(GPTQ_ERR_INVALID_ARG, "out must be >= 0 (got %lld)", (long long)out);
  const int b = cfg->bits;
  if (b != 2 && b != 3 && b != 4 && b != 8) return fail(GPTQ_ERR_INVALID_ARG, "bits must be 2, 3, 4 or 8 (got %d)", b);
  const int gs = cfg->group_size;
  if (gs != -1 && (gs <= 0 || in % gs != 0))
    return fail(GPTQ_ERR_INVALID_ARG, "group_size must be -1 or a positive divisor of in=%lld (got %d)",
                (long long)in, gs);
  if (cfg->block_size <= 0) return fail(GPTQ_ERR_INVALID_ARG, "block_size must be positive (got %d)", cfg->block_size);
  if (gs != -1 && cfg->block_size % gs != 0 && gs % cfg->block_size != 0)
    return fail(GPTQ_ERR_INVALID_ARG, "block_size (%d) must divide group_size (%d) or be a multiple of it",
                cfg->block_size, gs);
  if (!std::isfinite(cfg->damp_percent) || cfg->damp_percent < 0.f)
    return fail(GPTQ_ERR_INVALID_ARG, "damp_percent must be finite and >= 0");
  if (cfg->sym != 0 && cfg->sym != 1) return fail(GPTQ_ERR_INVALID_ARG, "sym must be 0 or 1");
  if (cfg->desc_act != 0 && cfg->desc_act != 1) return fail(GPTQ_ERR_INVALID_ARG, "desc_act must be 0 or 1");
  if (gs != -1 && ((gs % 128 != 0 && 128 % gs != 0) || gs < 8))
    return fail(GPTQ_ERR_UNSUPPORTED,
                "group_size %d: this build needs group_size >= 8 with group_size | 128 or 128 | group_size", gs);
  if (in > kMaxIn || out > kMaxOut)
    return fail(GPTQ_ERR_UNSUPPORTED, "layer %lld x %lld exceeds this build's limits (in <= %lld, out <= %lld)",
                (long long)out, (long long)in, (long long)kMaxIn, (long long)kMaxOut);
  return GPTQ_OK;
}

size_t gptq_workspace_bytes(int64_t out, int64_t in, const gptq_config_t* cfg) {
  if (!cfg || in < 1 || out < 0 || in > kMaxIn || out > kMaxOut) return 0;
  size_t need = prepare_ws_bytes(in);
  if (out > 0) {
    const size_t q = quantize_ws_bytes(out, in, cfg);
    if (q > need) need = q;
  }
  return need;
}

gptq_status_t gptq_hessian_accumulate(float* S, int64_t in, const void* X, gptq_dtype_t xt, int64_t tokens,
                                      int64_t ldx, int64_t* n_accum, void* stream) {
  clear_error();
  if (in < 1 || in > kMaxIn) return fail(GPTQ_ERR_INVALID_ARG, "in must be in [1, %lld]", (long long)kMaxIn);
  if (tokens < 0) return fail(GPTQ_ERR_INVALID_ARG, "tokens must be >= 0");
  if (!dtype_ok(xt)) return fail(GPTQ_ERR_INVALID_ARG, "unknown X dtype %d", (int)xt);
  if (tokens > 0 && ldx < tokens) return fail(GPTQ_ERR_INVALID_ARG, "ldx (%lld) < tokens (%lld)", (long long)ldx,
                                              (long long)tokens);
  if (!S) return fail(GPTQ_ERR_INVALID_ARG, "S is NULL");
  if (tokens > 0 && !X) return fail(GPTQ_ERR_INVALID_ARG, "X is NULL");
  gptq_status_t s = check_device();
  if (s != GPTQ_OK) return s;
  if (tokens > 0) {
    s = hessian_accumulate(S, in, X, xt, tokens, ldx, (cudaStream_t)stream);
    if (s != GPTQ_OK) return s;
  }
  if (n_accum) *n_accum += tokens;
  return GPTQ_OK;
}

gptq_status_t gptq_prepare_hinv(const float* S, int64_t n, int64_t in, const gptq_config_t* cfg, float* U,
                                int32_t* perm, uint8_t* dead, void* ws, size_t ws_bytes, void* stream) {
  gptq_status_t s = gptq_validate_config(cfg, 0, in);
  if (s != GPTQ_OK) return s;
  if (n <= 0) return fail(GPTQ_ERR_INVALID_ARG, "n (tokens accumulated) must be positive");
  if (!S || !U || !perm || !dead) return fail(GPTQ_ERR_INVALID_ARG, "S, U, perm and dead must be non-NULL");
  s = check_device();
  if (s != GPTQ_OK) return s;
  s = check_ws(ws, ws_bytes, prepare_ws_bytes(in));
  if (s != GPTQ_OK) return s;
  return prepare_hinv(S, n, in, cfg, U, perm, dead, ws, ws_bytes, (cudaStream_t)stream);
}

gptq_status_t gptq_quantize_layer(const void* W, gptq_dtype_t wt, int64_t out, int64_t in, int64_t ldw,
                                  const float* U, const int32_t* perm, const uint8_t* dead,
                                  const gptq_config_t* cfg, int32_t* codes, uint32_t* qweight, float* scales,
                                  int32_t* zeros, int32_t* g_idx, float* loss, void* ws, size_t ws_bytes,
                                  void* stream) {
  gptq_status_t s = gptq_validate_config(cfg, out, in);
  if (s != GPTQ_OK) return s;
  if (!dtype_ok(wt)) return fail(GPTQ_ERR_INVALID_ARG, "unknown W dtype %d", (int)wt);
  if (out == 0) return GPTQ_OK;
  if (ldw < in) return fail(GPTQ_ERR_INVALID_ARG, "ldw (%lld) < in (%lld)", (long long)ldw, (long long)in);
  if (!W || !U || !perm || !dead || !scales || !zeros || !g_idx)
    return fail(GPTQ_ERR_INVALID_ARG, "W, U, perm, dead, scales, zeros and g_idx must be non-NULL");
  if (qweight && (in * cfg->bits) % 32 != 0)
    return fail(GPTQ_ERR_INVALID_ARG, "qweight needs in*bits to be a multiple of 32 (in=%lld, bits=%d)",
                (long long)in, cfg->bits);
  s = check_device();
  if (s != GPTQ_OK) return s;
  s = check_ws(ws, ws_bytes, quantize_ws_bytes(out, in, cfg));
  if (s != GPTQ_OK) return s;
  return quantize_layer(W, wt, out, in, ldw, U, perm, dead, cfg, codes, qweight, scales, zeros, g_idx, loss, ws,
                        ws_bytes, (cudaStream_t)stream);
}

gptq_status_t gptq_workspace_status(const void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (!ws) return fail(GPTQ_ERR_WORKSPACE, "workspace pointer is NULL");
  if (((uintptr_t)ws & 255u) != 0) return fail(GPTQ_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (ws_bytes < (size_t)kHeaderBytes)
    return fail(GPTQ_ERR_WORKSPACE, "workspace too small: %zu bytes given, %lld needed", ws_bytes,
                (long long)kHeaderBytes);
  gptq_status_t s = check_device();
  if (s != GPTQ_OK) return s;
  return read_device_status((const PrepHeader*)ws, (cudaStream_t)stream);
}

gptq_status_t gptq_dequantize_layer(const uint32_t* qweight, const float* scales, const int32_t* zeros,
                                    const int32_t* g_idx, int64_t out, int64_t in, int bits, int ngroups,
                                    void* Wq, gptq_dtype_t wt, int64_t ldw, void* stream) {
  clear_error();
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8)
    return fail(GPTQ_ERR_INVALID_ARG, "bits must be 2, 3, 4 or 8 (got %d)", bits);
  if (out < 0 || in < 1 || in > kMaxIn || out > kMaxOut)
    return fail(GPTQ_ERR_INVALID_ARG, "layer %lld x %lld is outside this build's limits", (long long)out,
                (long long)in);
  if (in % 8 != 0 || (in * bits) % 32 != 0)
    return fail(GPTQ_ERR_UNSUPPORTED, "dequantize needs in %% 8 == 0 and in*bits %% 32 == 0 (in=%lld, bits=%d)",
                (long long)in, bits);
  if (ngroups < 1 || ngroups > in) return fail(GPTQ_ERR_INVALID_ARG, "ngroups must be in [1, in] (got %d)", ngroups);
  if (!dtype_ok(wt)) return fail(GPTQ_ERR_INVALID_ARG, "unknown output dtype %d", (int)wt);
  if (ldw < in) return fail(GPTQ_ERR_INVALID_ARG, "ldw (%lld) < in (%lld)", (long long)ldw, (long long)in);
  if (out == 0) return GPTQ_OK;
  if (!qweight || !scales || !zeros || !g_idx || !Wq)
    return fail(GPTQ_ERR_INVALID_ARG, "qweight, scales, zeros, g_idx and Wq must be non-NULL");
  if (((uintptr_t)g_idx & 15u) != 0) return fail(GPTQ_ERR_INVALID_ARG, "g_idx must be 16-byte aligned");
  gptq_status_t s = check_device();
  if (s != GPTQ_OK) return s;
  return dequantize_layer(qweight, scales, zeros, g_idx, out, in, bits, ngroups, Wq, wt, ldw, (cudaStream_t)stream);
}

gptq_status_t gptq_export_checkpoint(const uint32_t* qweight, const float* scales, const int32_t* zeros, int64_t out,
                                     int64_t in, int bits, int ngroups, int zero_offset, uint32_t* qweight_t,
                                     uint32_t* qzeros, uint16_t* scales_h, void* stream) {
  clear_error();
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8)
    return fail(GPTQ_ERR_INVALID_ARG, "bits must be 2, 3, 4 or 8 (got %d)", bits);
  if (out < 0 || in < 1 || in > kMaxIn || out > kMaxOut)
    return fail(GPTQ_ERR_INVALID_ARG, "layer %lld x %lld is outside this build's limits", (long long)out,
                (long long)in);
  if (ngroups < 1 || ngroups > in) return fail(GPTQ_ERR_INVALID_ARG, "ngroups must be in [1, in] (got %d)", ngroups);
  if (zero_offset != 0 && zero_offset != 1)
    return fail(GPTQ_ERR_INVALID_ARG, "zero_offset must be 0 or 1 (got %d)", zero_offset);
  if (qweight_t && (in * bits) % 32 != 0)
    return fail(GPTQ_ERR_UNSUPPORTED, "qweight_t needs in*bits %% 32 == 0 (in=%lld, bits=%d)", (long long)in, bits);
  if (qzeros && (out * bits) % 32 != 0)
    return fail(GPTQ_ERR_UNSUPPORTED, "qzeros needs out*bits %% 32 == 0 (out=%lld, bits=%d)", (long long)out, bits);
  if ((qweight_t && !qweight) || (qzeros && !zeros) || (scales_h && !scales))
    return fail(GPTQ_ERR_INVALID_ARG, "each requested output needs its input (qweight, zeros, scales)");
  if (out == 0 || (!qweight_t && !qzeros && !scales_h)) return GPTQ_OK;
  gptq_status_t s = check_device();
  if (s != GPTQ_OK) return s;
  return export_checkpoint(qweight, scales, zeros, out, in, bits, ngroups, zero_offset, qweight_t, qzeros, scales_h,
                           (cudaStream_t)stream);
}

}  // extern "C"
