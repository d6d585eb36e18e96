// Internal GEMM interface of the GPTQ solver library.
//
//   C[r][c] = beta * C[r][c] + alpha * sum_k P[r][k] * Q[c][k]
//
// P (rows r) and Q (rows c) are both stored row-major with k contiguous
// ("K-major"), which is how every product in the solver can be phrased:
//   Hessian         S  += X X^T           P = Q = X (fp16/bf16)
//   trailing update W  -= E U_blk         P = E, Q = U column-major
//   factorisation   panel / Schur / inverse products on split-fp32 blocks.
// Two implementations share these semantics: the tcgen05 tensor-core kernel
// (tc_gemm.cu) and a CUDA-core fp32 kernel (simt.cu) used for fp32 inputs,
// unaligned layouts and cross-checks.
#pragma once

#include "common.cuh"

namespace gptq {

enum GemmOp : int { OP_F16 = 0, OP_BF16 = 1, OP_TF32X3 = 2 };

// An fp32 matrix may be stored "split": value = hi + lo with hi rounded to
// tf32 and lo the exact remainder (split_tf32).  The tensor-core kernel then
// forms hi*hi + hi*lo + lo*hi, which is accurate to about 2^-22 relative.
struct Operand {
  const void* hi = nullptr;  // fp16/bf16/fp32 data (the hi part when split)
  const void* lo = nullptr;  // fp32 remainder, or null
  int64_t rows = 0;          // rows of the stored matrix (TMA bound)
  int64_t cols = 0;          // k extent of the stored matrix (TMA bound)
  int64_t ld = 0;            // row stride in elements
};

struct GemmArgs {
  int op = OP_TF32X3;
  Operand P, Q;
  int64_t R = 0, Cn = 0, K = 0;                 // sizes of one product
  int64_t p_row0 = 0, p_k0 = 0, q_row0 = 0, q_k0 = 0;
  float* C = nullptr;                           // output (hi part when split)
  float* C_lo = nullptr;                        // split output remainder or null
  int64_t ldc = 0, c_row0 = 0, c_col0 = 0;
  float alpha = 1.f, beta = 1.f;                // beta == 0: C is not read
  int mask = 0;                                 // 0 all, 1 keep c-r >= off, 2 keep c-r <= off
  int64_t mask_off = 0;
  int transpose = 0;                            // 1: write C[c][r] (row c0+c, col r0+r)
  // batches of identical products at strided offsets
  int batch = 1;
  int64_t bs_p_row = 0, bs_p_k = 0, bs_q_row = 0, bs_q_k = 0, bs_c_row = 0, bs_c_col = 0;
  int tri = 0;                                  // upper-triangle SYRK schedule (P == Q)
  int p_tile = 256;                             // grid schedule: P rows per output tile (256 or 128)
  int pdl = 0;                                  // 1: programmatic dependent launch (prologue overlaps
                                                //    the previous kernel of the stream)
  uint32_t* status = nullptr;                   // device status word (may be null)
};

void note_launch();

// Raise the dynamic shared-memory limit of kernel `func` to `bytes` on the
// current device, once per (kernel, device, size); thread-safe.
cudaError_t ensure_smem_limit(const void* func, int bytes);

// Returns cudaSuccess or the launch error.  Asynchronous.
cudaError_t tc_gemm(const GemmArgs& a, cudaStream_t stream, int num_sms);
cudaError_t simt_gemm(const GemmArgs& a, cudaStream_t stream);

// Make the driver load the GEMM kernels on the current device now (as their
// first launch would); cudaFuncGetAttributes on each.
cudaError_t preload_gemm_kernels();
cudaError_t preload_simt_kernels();

// Whether the tensor-core path can take this product (alignment of bases
// and strides for TMA, K extents compatible with the k-tile).
bool tc_gemm_supported(const GemmArgs& a);

}  // namespace gptq
