// Host-side internals shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstdint>

#include "common.cuh"

namespace gptq {

// First 256 bytes of every workspace.
struct PrepHeader {
  uint32_t status;  // ST_* flags OR-ed by kernels
  uint32_t pad0;
  double lambda;    // damping added to the diagonal
  uint32_t pad[60];
};
constexpr int64_t kHeaderBytes = 256;
static_assert(sizeof(PrepHeader) == kHeaderBytes, "header size");

inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

struct DeviceInfo {
  int id = -1;
  int sms = 0;
  int major = 0, minor = 0;
};
// Properties of the current device (cached per device).
const DeviceInfo& device_info();

// Process-wide count of kernels this library has launched (diagnostic).
void note_launch();

// True when the environment variable GPTQ_FORCE_SIMT was set to a non-zero
// integer at the library's first call: every GEMM then runs on the CUDA-core
// kernel (a cross-check of the tensor-core path).  Read once per process.
bool force_simt();

// Record a message for gptq_last_error() and return s.
gptq_status_t fail(gptq_status_t s, const char* fmt, ...);
void clear_error();

// Wait for st, read the status word of the workspace header hdr (device
// memory) and map its flags to a status code: GPTQ_ERR_TIMEOUT before
// GPTQ_ERR_NONFINITE before GPTQ_ERR_NOT_PD, GPTQ_OK when none is set.
gptq_status_t read_device_status(const PrepHeader* hdr, cudaStream_t st);

#define CUDA_TRY(x)                                                                           \
  do {                                                                                        \
    cudaError_t e_ = (x);                                                                     \
    if (e_ != cudaSuccess) return ::gptq::fail(GPTQ_ERR_CUDA, "%s: %s", #x, cudaGetErrorString(e_)); \
  } while (0)

// Workspace needs of the two workspace-using calls.
size_t prepare_ws_bytes(int64_t in);
size_t quantize_ws_bytes(int64_t out, int64_t in, const gptq_config_t* cfg);

gptq_status_t prepare_hinv(const float* S, int64_t n, int64_t in, const gptq_config_t* cfg, float* U,
                           int32_t* perm, uint8_t* dead, void* ws, size_t ws_bytes, cudaStream_t st);
gptq_status_t dequantize_layer(const uint32_t* qweight, const float* scales, const int32_t* zeros,
                               const int32_t* g_idx, int64_t out, int64_t in, int bits, int ngroups, void* Wq,
                               gptq_dtype_t wt, int64_t ldw, cudaStream_t st);
gptq_status_t quantize_layer(const void* W, gptq_dtype_t wt, int64_t out, int64_t in, int64_t ldw, const float* U,
                             const int32_t* perm, const uint8_t* dead, const gptq_config_t* cfg, int32_t* codes,
                             uint32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx, float* loss, void* ws,
                             size_t ws_bytes, cudaStream_t st);
gptq_status_t export_checkpoint(const uint32_t* qweight, const float* scales, const int32_t* zeros, int64_t out,
                                int64_t in, int bits, int ngroups, int zero_offset, uint32_t* qweight_t,
                                uint32_t* qzeros, uint16_t* scales_h, cudaStream_t st);
gptq_status_t hessian_accumulate(float* S, int64_t in, const void* X, gptq_dtype_t xt, int64_t tokens, int64_t ldx,
                                 cudaStream_t st);

// Blocked Cholesky R = L L^T of the np x np matrix R (lower triangle, np a
// multiple of 128) and the inverse M = L^-1, in one cooperative launch
// (chol.cu).  Outputs, split (tf32 hi + exact remainder): the panel tiles of L
// below the 64 x 64 diagonal blocks in Lh/Ll, the diagonal blocks of M in
// Mh/Ml, and all of M transposed in Mth/Mtl (Mt[c][r] = M[r][c]).  R and Gt
// (np x np scratch) are overwritten; Mth, Mtl and Gt must hold zeros on
// entry.  sync: chol_sync_bytes(np) bytes of scratch.  Device-side failures
// are raised in *status.
size_t chol_sync_bytes(int64_t np_);
cudaError_t chol_factor(float* R, int64_t np_, float* Lh, float* Ll, float* Mh, float* Ml, float* Mth, float* Mtl,
                        float* Gt, unsigned* sync, uint32_t* status, int sms, cudaStream_t st);

// A 2-D tensor map over a row-major fp32 matrix (cols x rows, row stride ld
// elements) with boxes of box_x columns by box_y rows; swizzle128 selects the
// 128-byte swizzle (the tensor core's K-major operand layout).
bool encode_f32_2d(CUtensorMap* m, const float* base, int64_t cols, int64_t rows, int64_t ld, uint32_t box_x,
                   uint32_t box_y, bool swizzle128);

// Make the driver load every kernel gptq_quantize_layer can launch on the
// current device now, instead of at their first launch.
cudaError_t preload_quantize_kernels();

// The sweep and its updates (solve.cu).  Wp (out x np, processing order) is
// updated in place; Uh/Ul = split U^T (np x np); Ud = solve_pack_ud's
// diagonal blocks; Eh/El (out x np) receive the split -E; sync:
// solve_sync_bytes scratch.  Writes codes_p (out x np, processing order),
// scales, zeros and loss (zeroed by the caller).
size_t solve_ud_bytes(int64_t np_);
size_t solve_sync_bytes(int64_t out, int64_t np_);
cudaError_t solve_pack_ud(const float* U, int64_t in, int64_t np_, float* Ud, cudaStream_t st);
cudaError_t solve_quantize(float* Wp, int64_t out, int64_t in, int64_t np_, const float* Uh, const float* Ul,
                           const float* Ud, float* Eh, float* El, const gptq_config_t* cfg, float* scales,
                           int32_t* zeros, uint8_t* codes_p, float* loss, void* sync, uint32_t* status, int sms,
                           cudaStream_t st);
cudaError_t preload_solve_kernels();

}  // namespace gptq
