// gptq_prepare_hinv: from the accumulated S and token count n to
//   H = 2 S / n, dead-channel fix, act-order permutation, dampening
//   ("Using AutoGPTQ in Practice", Key Parameters: desc_act, damp_percent),
//   and U, the upper Cholesky factor of H_perm^-1 ("Using AutoGPTQ in
//   Practice": Cholesky factorization).
//
// U is obtained through the reversal identity: with J the index reversal,
// factor R = J H_perm J = L L^T (lower Cholesky), invert M = L^-1; then
// U = J M J is upper triangular with positive diagonal and U^T U = H_perm^-1,
// hence it is the unique upper Cholesky factor of H_perm^-1.  That costs one
// Cholesky and one triangular inverse (2/3 n^3 flops) instead of
// factor -> invert -> factor again.
//
// The matrix is padded to a multiple of 128 with identity (block-diagonal,
// so the padding never mixes with the real channels).
//   Cholesky and inverse: right-looking with 64-wide blocks in one
//              cooperative launch (chol.cu): one CTA factors and inverts each
//              diagonal block while the others form, as 3xTF32 tensor-core
//              tiles on split operands (hi rounded to tf32 plus the exact
//              fp32 remainder), the panel L_ik = R_ik M_kk^T, the trailing
//              update R -= L_ik L_jk^T and, block row by block row, the
//              inverse M = L^-1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>

#include "internal.cuh"

namespace gptq {
namespace {

constexpr int NB = 128;

// ------------------------------------------------------------------ diag
// One CTA: hd[i] = fixed diagonal of H in double, hd = c * S_ii with
// c = 2 / n rounded to double (the same two roundings as forming H = (2/n) S
// in float64), dead channels (S_ii == 0) get 1; dead flags; and
// lambda = damp * mean(hd).  Deterministic tree reduction in double.
__global__ void __launch_bounds__(1024) diag_kernel(const float* __restrict__ S, int64_t in, double c,
                                                    float damp, double* __restrict__ hd, uint8_t* __restrict__ dead,
                                                    PrepHeader* hdr) {
  __shared__ double red[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < in; i += blockDim.x) {
    const float s = S[i * in + i];
    if (!isfinite(s)) raise_status(&hdr->status, ST_NONFINITE);
    const bool d = (s == 0.f);
    const double h = d ? 1.0 : __dmul_rn(c, (double)s);
    hd[i] = h;
    dead[i] = d ? 1 : 0;
    acc += h;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) hdr->lambda = (double)damp * (red[0] / (double)in);
}

// ------------------------------------------------------------------ act order
// perm[rank(i)] = i, rank = #{j : hd_j > hd_i} + #{j < i : hd_j == hd_i}:
// the stable descending order of the diagonal, compared in double on the
// values diag_kernel formed (so two channels tie exactly when their H_ii
// tie in float64).
__global__ void __launch_bounds__(256) rank_kernel(const double* __restrict__ hd, int64_t in, int desc_act,
                                                   int32_t* __restrict__ perm) {
  __shared__ double tile[1024];
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (!desc_act) {
    if (i < in) perm[i] = (int32_t)i;
    return;
  }
  const double key = i < in ? hd[i] : 0.0;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < in; j0 += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x) tile[t] = (j0 + t < in) ? hd[j0 + t] : 0.0;
    __syncthreads();
    const int m = (int)((in - j0) < 1024 ? (in - j0) : 1024);
    for (int t = 0; t < m; ++t) {
      const double v = tile[t];
      rank += (v > key) || (v == key && j0 + t < i);
    }
  }
  if (i < in) perm[rank] = (int32_t)i;
}

// ------------------------------------------------------------------ gather
// Lower triangle (b <= a) of R[a][b] = H_perm_damped[in-1-a][in-1-b], with
// the identity in the padding.  Only the lower triangle is ever read: the
// factorisation's leaf ignores what lies above the diagonal and the trailing
// updates add into lower tiles only.  With the natural order (i <= j for
// b <= a) the S reads run along rows of the stored upper triangle, so they
// coalesce; each block takes whole rows, four columns per thread.
__global__ void __launch_bounds__(256) gather_kernel(const float* __restrict__ S, int64_t in, int64_t np_,
                                                     float scale, const int32_t* __restrict__ perm,
                                                     const double* __restrict__ hd, PrepHeader* hdr,
                                                     float* __restrict__ R) {
  const double lam = hdr->lambda;
  // in <= 32768, so in * in fits 32-bit index arithmetic
  const int n = (int)in, np = (int)np_;
  for (int a = blockIdx.x; a < np; a += gridDim.x) {
    const int i = a < n ? __ldg(perm + n - 1 - a) : -1;
    for (int b0 = threadIdx.x * 4; b0 <= a; b0 += blockDim.x * 4) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u;
        float x = 0.f;
        if (a < n && b < n) {
          const int j = __ldg(perm + n - 1 - b);
          const unsigned lo = (unsigned)min(i, j), hi = (unsigned)max(i, j);
          const float sv = __ldg(S + (lo * (unsigned)n + hi));
          if (!isfinite(sv)) raise_status(&hdr->status, ST_NONFINITE);
          // the diagonal from diag_kernel's fixed values (dead channels
          // there hold 1), damped in double and rounded once
          x = (i == j) ? (float)(__ldg(hd + i) + lam) : sv * scale;
        } else if (a == b) {
          x = 1.f;
        }
        v[u] = x;
      }
      *reinterpret_cast<float4*>(R + (int64_t)a * np_ + b0) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

// U (column-major, in x in): U_cm[x][y] = Mt[in-1-x][in-1-y] for y <= x, 0 above.
// U[x][y] = M[in-1-y][in-1-x] = Mt[in-1-x][in-1-y] for y <= x (U = J M J with
// J the reversal), 0 above.  Rows of Mt are read backwards; with in % 4 == 0
// four consecutive y map to one aligned float4 of Mt.
__global__ void __launch_bounds__(256) write_u_kernel(const float* __restrict__ Mth, const float* __restrict__ Mtl,
                                                      int64_t np_, int64_t in, float* __restrict__ U) {
  const bool vec = (in & 3) == 0;
  for (int64_t x = blockIdx.x; x < in; x += gridDim.x) {
    const int64_t src = (in - 1 - x) * np_;
    if (vec) {
      for (int64_t y = (int64_t)threadIdx.x * 4; y < in; y += (int64_t)blockDim.x * 4) {
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        if (y <= x) {
          const int64_t q = in - 4 - y;  // Mt[.., q .. q+3] holds y+3 .. y
          const float4 h = *reinterpret_cast<const float4*>(Mth + src + q);
          const float4 l = *reinterpret_cast<const float4*>(Mtl + src + q);
          o.x = h.w + l.w;
          o.y = (y + 1 <= x) ? h.z + l.z : 0.f;
          o.z = (y + 2 <= x) ? h.y + l.y : 0.f;
          o.w = (y + 3 <= x) ? h.x + l.x : 0.f;
        }
        *reinterpret_cast<float4*>(U + x * in + y) = o;
      }
    } else {
      for (int64_t y = threadIdx.x; y < in; y += blockDim.x) {
        float v = 0.f;
        if (y <= x) {
          const int64_t q = in - 1 - y;
          v = Mth[src + q] + Mtl[src + q];
        }
        U[x * in + y] = v;
      }
    }
  }
}

}  // namespace

size_t prepare_ws_bytes(int64_t in) {
  const int64_t np_ = round_up(in, NB);
  size_t b = kHeaderBytes;
  b += round_up((int64_t)sizeof(double) * in, 256);              // hd
  b += 8 * round_up((int64_t)sizeof(float) * np_ * np_, 256);    // R; L, M, Mt (hi, lo); G^T
  b += round_up((int64_t)chol_sync_bytes(np_), 256);             // barrier and panel counters
  return b;
}

gptq_status_t prepare_hinv(const float* S, int64_t n, int64_t in, const gptq_config_t* cfg, float* U,
                           int32_t* perm, uint8_t* dead, void* ws, size_t ws_bytes, cudaStream_t st) {
  const DeviceInfo& dev = device_info();
  const int64_t np_ = round_up(in, NB);
  uint8_t* p = (uint8_t*)ws;
  PrepHeader* hdr = (PrepHeader*)p;
  p += kHeaderBytes;
  double* hd = (double*)p;
  p += round_up((int64_t)sizeof(double) * in, 256);
  const size_t mat = round_up((int64_t)sizeof(float) * np_ * np_, 256);
  float* R = (float*)p; p += mat;      // reversed, damped Hessian; Schur complements in place
  float* Lh = (float*)p; p += mat;     // L's panels (split), for the inverse
  float* Ll = (float*)p; p += mat;
  float* Mh = (float*)p; p += mat;
  float* Ml = (float*)p; p += mat;
  float* Mth = (float*)p; p += mat;
  float* Mtl = (float*)p; p += mat;
  float* Gt = (float*)p; p += mat;     // the inverse's accumulator, transposed
  unsigned* sync = (unsigned*)p;  // barrier, then the panel counters

  CUDA_TRY(cudaMemsetAsync(hdr, 0, kHeaderBytes, st));
  CUDA_TRY(cudaMemsetAsync(Mth, 0, 3 * mat, st));  // Mt (hi, lo): zeros above the diagonal; G^T starts at 0
  const double c = 2.0 / (double)n;
  const float scale = (float)c;
  diag_kernel<<<1, 1024, 0, st>>>(S, in, c, cfg->damp_percent, hd, dead, hdr);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  rank_kernel<<<(unsigned)((in + 255) / 256), 256, 0, st>>>(hd, in, cfg->desc_act, perm);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  {
    const unsigned grid = (unsigned)std::min<int64_t>(np_, (int64_t)dev.sms * 8);
    gather_kernel<<<grid, 256, 0, st>>>(S, in, np_, scale, perm, hd, hdr, R);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  // blocked Cholesky of R and the inverse M = L^-1 (transposed in Mth/Mtl)
  CUDA_TRY(chol_factor(R, np_, Lh, Ll, Mh, Ml, Mth, Mtl, Gt, sync, &hdr->status, dev.sms, st));
  {
    const unsigned grid = (unsigned)std::min<int64_t>(in, (int64_t)dev.sms * 8);
    write_u_kernel<<<grid, 256, 0, st>>>(Mth, Mtl, np_, in, U);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  return read_device_status(hdr, st);
}

}  // namespace gptq
