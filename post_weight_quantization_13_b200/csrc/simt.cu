// CUDA-core fp32 implementation of C (+)= alpha * P Q^T (semantics in
// gemm.cuh).  Used for fp32 calibration activations, for layouts the TMA
// path cannot address, and as an independent on-device check of the
// tensor-core kernel.  64 x 64 output tile per 256-thread block, 4 x 4 per
// thread, k-tiles of 16 staged in shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "gemm.cuh"

namespace gptq {
namespace {

struct SimtParams {
  const void* p_hi;
  const float* p_lo;
  const void* q_hi;
  const float* q_lo;
  int64_t ldp, ldq;
  int64_t R, Cn, K;
  int64_t p_row0, p_k0, q_row0, q_k0;
  int64_t bs_p_row, bs_p_k, bs_q_row, bs_q_k, bs_c_row, bs_c_col;
  float* C;
  float* C_lo;
  int64_t ldc, c_row0, c_col0;
  float alpha, beta;
  int mask;
  int64_t mask_off;
  int transpose;
  int tri;
};

template <typename T>
__device__ __forceinline__ float ld_elem(const void* p, int64_t i) {
  return static_cast<float>(static_cast<const T*>(p)[i]);
}
template <>
__device__ __forceinline__ float ld_elem<__half>(const void* p, int64_t i) {
  return __half2float(static_cast<const __half*>(p)[i]);
}
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const void* p, int64_t i) {
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

template <typename T>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtParams sp) {
  const int b = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.y * 64;
  const int64_t c0 = (int64_t)blockIdx.x * 64;
  if (sp.tri && c0 + 63 < r0) return;  // tile entirely below the diagonal
  __shared__ float Ps[16][65];
  __shared__ float Qs[16][65];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  const int64_t prow = sp.p_row0 + b * sp.bs_p_row, pk = sp.p_k0 + b * sp.bs_p_k;
  const int64_t qrow = sp.q_row0 + b * sp.bs_q_row, qk = sp.q_k0 + b * sp.bs_q_k;
  for (int64_t k0 = 0; k0 < sp.K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int rr = e >> 4, kk = e & 15;
      const int64_t r = r0 + rr, c = c0 + rr, k = k0 + kk;
      float pv = 0.f, qv = 0.f;
      if (r < sp.R && k < sp.K) {
        const int64_t i = (prow + r) * sp.ldp + pk + k;
        pv = ld_elem<T>(sp.p_hi, i);
        if (sp.p_lo) pv += sp.p_lo[i];
      }
      if (c < sp.Cn && k < sp.K) {
        const int64_t i = (qrow + c) * sp.ldq + qk + k;
        qv = ld_elem<T>(sp.q_hi, i);
        if (sp.q_lo) qv += sp.q_lo[i];
      }
      Ps[kk][rr] = pv;
      Qs[kk][rr] = qv;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = Ps[kk][ty * 4 + i];
        q[i] = Qs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], q[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int64_t cr = sp.c_row0 + b * sp.bs_c_row, cc = sp.c_col0 + b * sp.bs_c_col;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty * 4 + i;
    if (r >= sp.R) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = c0 + tx * 4 + j;
      if (c >= sp.Cn) continue;
      if (sp.mask == 1 && c - r < sp.mask_off) continue;
      if (sp.mask == 2 && c - r > sp.mask_off) continue;
      const int64_t idx = sp.transpose ? (cr + c) * sp.ldc + (cc + r) : (cr + r) * sp.ldc + (cc + c);
      float val = sp.alpha * acc[i][j];
      if (sp.beta != 0.f) {
        float old = sp.C[idx];
        if (sp.C_lo) old += sp.C_lo[idx];
        val = fmaf(sp.beta, old, val);
      }
      if (sp.C_lo) {
        float hi, lo;
        split_tf32(val, hi, lo);
        sp.C[idx] = hi;
        sp.C_lo[idx] = lo;
      } else {
        sp.C[idx] = val;
      }
    }
  }
}

}  // namespace

cudaError_t preload_simt_kernels() {
  const void* fns[] = {(const void*)simt_gemm_kernel<__half>, (const void*)simt_gemm_kernel<__nv_bfloat16>,
                       (const void*)simt_gemm_kernel<float>};
  for (const void* f : fns) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, f);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t simt_gemm(const GemmArgs& a, cudaStream_t st) {
  if (a.R <= 0 || a.Cn <= 0 || a.K <= 0 || a.batch <= 0) return cudaSuccess;
  SimtParams sp;
  sp.p_hi = a.P.hi;
  sp.p_lo = (const float*)a.P.lo;
  sp.q_hi = a.Q.hi;
  sp.q_lo = (const float*)a.Q.lo;
  sp.ldp = a.P.ld;
  sp.ldq = a.Q.ld;
  sp.R = a.R;
  sp.Cn = a.Cn;
  sp.K = a.K;
  sp.p_row0 = a.p_row0;
  sp.p_k0 = a.p_k0;
  sp.q_row0 = a.q_row0;
  sp.q_k0 = a.q_k0;
  sp.bs_p_row = a.bs_p_row;
  sp.bs_p_k = a.bs_p_k;
  sp.bs_q_row = a.bs_q_row;
  sp.bs_q_k = a.bs_q_k;
  sp.bs_c_row = a.bs_c_row;
  sp.bs_c_col = a.bs_c_col;
  sp.C = a.C;
  sp.C_lo = a.C_lo;
  sp.ldc = a.ldc;
  sp.c_row0 = a.c_row0;
  sp.c_col0 = a.c_col0;
  sp.alpha = a.alpha;
  sp.beta = a.beta;
  sp.mask = a.mask;
  sp.mask_off = a.mask_off;
  sp.transpose = a.transpose;
  sp.tri = a.tri;
  dim3 grid((unsigned)((a.Cn + 63) / 64), (unsigned)((a.R + 63) / 64), (unsigned)a.batch);
  switch (a.op) {
    case OP_F16:
      simt_gemm_kernel<__half><<<grid, 256, 0, st>>>(sp);
      note_launch();
      break;
    case OP_BF16:
      simt_gemm_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(sp);
      note_launch();
      break;
    default:
      simt_gemm_kernel<float><<<grid, 256, 0, st>>>(sp);
      note_launch();
      break;
  }
  return cudaGetLastError();
}

}  // namespace gptq
