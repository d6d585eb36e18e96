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
// Working matrices are kept "split" (hi rounded to tf32 plus exact fp32
// remainder) so every block product runs on the tensor cores with 3xTF32
// accuracy.  The matrix is padded to a multiple of 128 with identity
// (block-diagonal, so the padding never mixes with the real channels).
//   Cholesky:  right-looking, 128-wide panels; the diagonal block is
//              factored and inverted in one CTA (leaf_kernel), the panel is
//              R_ik M_kk^T and the trailing update R -= L_ik L_jk^T.
//   Inverse:   pairs of already inverted diagonal groups are merged,
//              M21 = -M22 (L21 M11), doubling the group size each level; all
//              merges of one level are one batched launch.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>
#include <vector>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {
namespace {

constexpr int NB = 128;

// ------------------------------------------------------------------ diag
// One CTA: hd[i] = fixed diagonal of H (dead -> 1), dead flags, and
// lambda = damp * mean(hd).  Deterministic tree reduction in double.
__global__ void __launch_bounds__(1024) diag_kernel(const float* __restrict__ S, int64_t in, float scale,
                                                    float damp, float* __restrict__ hd, uint8_t* __restrict__ dead,
                                                    PrepHeader* hdr) {
  __shared__ double red[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < in; i += blockDim.x) {
    const float s = S[i * in + i];
    if (!isfinite(s)) raise_status(&hdr->status, ST_NONFINITE);
    const float h = s * scale;
    const bool d = (h == 0.f);
    const float hf = d ? 1.f : h;
    hd[i] = hf;
    dead[i] = d ? 1 : 0;
    acc += (double)hf;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) hdr->lambda = (float)((double)damp * (red[0] / (double)in));
}

// ------------------------------------------------------------------ act order
// perm[rank(i)] = i, rank = #{j : hd_j > hd_i} + #{j < i : hd_j == hd_i}:
// the stable descending order.
__global__ void __launch_bounds__(256) rank_kernel(const float* __restrict__ hd, int64_t in, int desc_act,
                                                   int32_t* __restrict__ perm) {
  __shared__ float tile[1024];
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (!desc_act) {
    if (i < in) perm[i] = (int32_t)i;
    return;
  }
  const float key = i < in ? hd[i] : 0.f;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < in; j0 += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x) tile[t] = (j0 + t < in) ? hd[j0 + t] : 0.f;
    __syncthreads();
    const int m = (int)((in - j0) < 1024 ? (in - j0) : 1024);
    for (int t = 0; t < m; ++t) {
      const float v = tile[t];
      rank += (v > key) || (v == key && j0 + t < i);
    }
  }
  if (i < in) perm[rank] = (int32_t)i;
}

// ------------------------------------------------------------------ gather
// R[a][b] = H_perm_damped[in-1-a][in-1-b] (split), identity in the padding.
__global__ void __launch_bounds__(256) gather_kernel(const float* __restrict__ S, int64_t in, int64_t np_,
                                                     float scale, const int32_t* __restrict__ perm,
                                                     const uint8_t* __restrict__ dead, PrepHeader* hdr,
                                                     float* __restrict__ R) {
  const int64_t a = blockIdx.y;
  const float lam = hdr->lambda;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < np_; b += (int64_t)gridDim.x * blockDim.x) {
    float v;
    if (a < in && b < in) {
      const int64_t i = perm[in - 1 - a], j = perm[in - 1 - b];
      const int64_t lo = min(i, j), hi = max(i, j);
      const float s = S[lo * in + hi];
      if (!isfinite(s)) raise_status(&hdr->status, ST_NONFINITE);
      v = s * scale;
      if (i == j) v = (dead[i] ? 1.f : v) + lam;
    } else {
      v = (a == b) ? 1.f : 0.f;
    }
    R[a * np_ + b] = v;
  }
}

// Pk[r][c] = split(R[r0 + r][kB + c]): the panel below diagonal block k as a
// 3xTF32 operand (rows x 128, row stride 128).
__global__ void __launch_bounds__(256) split_panel_kernel(const float* __restrict__ R, int64_t np_, int64_t r0,
                                                          int64_t kB, int64_t rows, float* __restrict__ Ph,
                                                          float* __restrict__ Pl) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * 32;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e >> 5, c4 = (e & 31) << 2;
    const float4 v = *reinterpret_cast<const float4*>(R + (r0 + r) * np_ + kB + c4);
    float4 h, l;
    split_tf32(v.x, h.x, l.x);
    split_tf32(v.y, h.y, l.y);
    split_tf32(v.z, h.z, l.z);
    split_tf32(v.w, h.w, l.w);
    *reinterpret_cast<float4*>(Ph + r * 128 + c4) = h;
    *reinterpret_cast<float4*>(Pl + r * 128 + c4) = l;
  }
}

// ------------------------------------------------------------------ leaf
// Factor the 128 x 128 diagonal block k of R (lower Cholesky) and invert the
// factor: L_kk into R, M_kk = L_kk^-1 into M and M_kk^T into Mt (all split).
// One CTA of 512 threads; thread (ty, tx) keeps the 8 x 4 block rows
// [8ty, 8ty+8) x columns [4tx, 4tx+4) in registers.
//   Cholesky, right-looking and unnormalised: at pivot j the owners of
//   column j publish it to shared memory (double-buffered), the pivot's owner
//   publishes 1/d_j, one barrier, then every thread applies
//   A[r][c] -= A[r][j] A[c][j] / d_j to its elements with j < c <= r.
//   Afterwards L[r][c] = A[r][c] / sqrt(d_c).
//   Inverse, right-looking on B = I: at step j row j of B becomes row j of
//   M (times 1/L_jj), is published, and rows r > j subtract L[r][j] M[j][:].
// A pivot that is not positive raises ST_NOT_PD and is replaced by 1 so the
// block stays finite.
constexpr int LD = NB + 1;

__global__ void __launch_bounds__(512) leaf_kernel(const float* R, float* Mh, float* Ml, float* Mth, float* Mtl,
                                                   int64_t np_, int k, PrepHeader* hdr) {
  extern __shared__ float Ls[];            // [NB][LD]: L, then staging for M^T
  __shared__ __align__(16) float colb[2][NB];  // published column (Cholesky) / row (inverse)
  __shared__ float pinv[NB];               // 1 / d_j
  __shared__ float rsq[NB];                // 1 / sqrt(d_j) = 1 / L_jj
  __shared__ float dpiv[NB];               // d_j
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  const int r0 = 8 * ty, c0 = 4 * tx;
  const int64_t o = (int64_t)k * NB;
  float a[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t g = (o + r0 + i) * np_ + o + c0;
    const float4 h = *reinterpret_cast<const float4*>(R + g);
    a[i][0] = h.x;
    a[i][1] = h.y;
    a[i][2] = h.z;
    a[i][3] = h.w;
  }
  // ---------------------------------------------------------- Cholesky
  for (int jj = 0; jj < NB / 4; ++jj) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int j = 4 * jj + kk;
      float* cb = colb[j & 1];
      if (tx == jj) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (r0 + i >= j) cb[r0 + i] = a[i][kk];
        if (ty == (j >> 3)) {
          float d = (jj & 1) ? a[4 + kk][kk] : a[kk][kk];
          if (!(d > 0.f) || !isfinite(d)) {
            raise_status(&hdr->status, ST_NOT_PD);
            d = 1.f;
          }
          dpiv[j] = d;
          pinv[j] = 1.f / d;
        }
      }
      __syncthreads();
      // this block has elements with j < c <= r
      if (r0 + 7 > j && c0 + 3 > j && c0 <= r0 + 7) {
        const float dinv = pinv[j];
        float cr[8], cc[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) cr[i] = cb[r0 + i] * dinv;
        const float4 c4 = *reinterpret_cast<const float4*>(cb + c0);
        cc[0] = c4.x;
        cc[1] = c4.y;
        cc[2] = c4.z;
        cc[3] = c4.w;
        if (c0 > j && c0 + 3 <= r0) {  // whole block strictly inside the update
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) a[i][q] = fmaf(-cr[i], cc[q], a[i][q]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int r = r0 + i, c = c0 + q;
              if (r > j && c > j && c <= r) a[i][q] = fmaf(-cr[i], cc[q], a[i][q]);
            }
        }
      }
    }
  }
  if (tid < NB) rsq[tid] = 1.f / sqrtf(dpiv[tid]);
  __syncthreads();
  // L[r][c] = A[r][c] / sqrt(d_c) below the diagonal, sqrt(d_r) on it
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = r0 + i, c = c0 + q;
      float v = 0.f;
      if (c < r) v = a[i][q] * rsq[c];
      if (c == r) v = sqrtf(dpiv[r]);
      a[i][q] = v;
      Ls[r * LD + c] = v;
    }
  __syncthreads();
  // ---------------------------------------------------------- inverse
  float b[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) b[i][q] = (r0 + i == c0 + q) ? 1.f : 0.f;
  for (int jj = 0; jj < NB / 4; ++jj) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int j = 4 * jj + kk;
      float* rb = colb[j & 1];
      if (ty == (j >> 3)) {
        const float s = rsq[j];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float m;
          if (jj & 1) {
            m = b[4 + kk][q] * s;
            b[4 + kk][q] = m;
          } else {
            m = b[kk][q] * s;
            b[kk][q] = m;
          }
          rb[c0 + q] = m;
        }
      }
      __syncthreads();
      // rows r > j take row j of M, which is zero past column j
      if (r0 + 7 > j && c0 <= j) {
        float lr[8], mr[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) lr[i] = Ls[(r0 + i) * LD + j];
        const float4 m4 = *reinterpret_cast<const float4*>(rb + c0);
        mr[0] = m4.x;
        mr[1] = m4.y;
        mr[2] = m4.z;
        mr[3] = m4.w;
        if (r0 > j) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) b[i][q] = fmaf(-lr[i], mr[q], b[i][q]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (r0 + i > j)
#pragma unroll
              for (int q = 0; q < 4; ++q) b[i][q] = fmaf(-lr[i], mr[q], b[i][q]);
        }
      }
    }
  }
  // ---------------------------------------------------------- write out
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t g = (o + r0 + i) * np_ + o + c0;
    float4 h, l;
    split_tf32(b[i][0], h.x, l.x);
    split_tf32(b[i][1], h.y, l.y);
    split_tf32(b[i][2], h.z, l.z);
    split_tf32(b[i][3], h.w, l.w);
    *reinterpret_cast<float4*>(Mh + g) = h;
    *reinterpret_cast<float4*>(Ml + g) = l;
  }
  __syncthreads();  // Ls is reused for M
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) Ls[(r0 + i) * LD + c0 + q] = b[i][q];
  __syncthreads();
  // Mt[r][c] = M[c][r]
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t g = (o + r0 + i) * np_ + o + c0;
    float4 h, l;
    split_tf32(Ls[(c0 + 0) * LD + r0 + i], h.x, l.x);
    split_tf32(Ls[(c0 + 1) * LD + r0 + i], h.y, l.y);
    split_tf32(Ls[(c0 + 2) * LD + r0 + i], h.z, l.z);
    split_tf32(Ls[(c0 + 3) * LD + r0 + i], h.w, l.w);
    *reinterpret_cast<float4*>(Mth + g) = h;
    *reinterpret_cast<float4*>(Mtl + g) = l;
  }
}

// Mt[o1 + c][o2 + r] = M[o2 + r][o1 + c] for the merged blocks of one level.
__global__ void __launch_bounds__(256) transpose_blocks_kernel(const float* __restrict__ Mh,
                                                               const float* __restrict__ Ml, float* __restrict__ Th,
                                                               float* __restrict__ Tl, int64_t np_, int64_t o1,
                                                               int64_t o2, int64_t s1, int64_t s2,
                                                               int64_t stride) {
  __shared__ float th[32][33], tl[32][33];
  const int64_t b = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int64_t O1 = o1 + b * stride, O2 = o2 + b * stride;
  for (int y = ty; y < 32; y += 8) {
    const int64_t r = r0 + y, c = c0 + tx;
    if (r < s2 && c < s1) {
      th[y][tx] = Mh[(O2 + r) * np_ + O1 + c];
      tl[y][tx] = Ml[(O2 + r) * np_ + O1 + c];
    }
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int64_t c = c0 + y, r = r0 + tx;
    if (r < s2 && c < s1) {
      Th[(O1 + c) * np_ + O2 + r] = th[tx][y];
      Tl[(O1 + c) * np_ + O2 + r] = tl[tx][y];
    }
  }
}

// U (column-major, in x in): U_cm[x][y] = Mt[in-1-x][in-1-y] for y <= x, 0 above.
__global__ void __launch_bounds__(256) write_u_kernel(const float* __restrict__ Mth, const float* __restrict__ Mtl,
                                                      int64_t np_, int64_t in, float* __restrict__ U) {
  const int64_t x = blockIdx.y;
  const int64_t src = (in - 1 - x) * np_;
  for (int64_t y = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; y < in; y += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    if (y <= x) {
      const int64_t q = in - 1 - y;
      v = Mth[src + q] + Mtl[src + q];
    }
    U[x * in + y] = v;
  }
}

cudaError_t run_gemm(GemmArgs& g, cudaStream_t st, int sms, bool force_simt) {
  if (!force_simt && tc_gemm_supported(g)) return tc_gemm(g, st, sms);
  return simt_gemm(g, st);
}

}  // namespace

size_t prepare_ws_bytes(int64_t in) {
  const int64_t np_ = round_up(in, NB);
  size_t b = kHeaderBytes;
  b += round_up((int64_t)sizeof(float) * in, 256);               // hd
  b += 9 * round_up((int64_t)sizeof(float) * np_ * np_, 256);    // R; L, M, Mt, X^T (hi, lo)
  b += 2 * round_up((int64_t)sizeof(float) * np_ * NB, 256);     // split panel
  return b;
}

gptq_status_t prepare_hinv(const float* S, int64_t n, int64_t in, const gptq_config_t* cfg, float* U,
                           int32_t* perm, uint8_t* dead, void* ws, size_t ws_bytes, cudaStream_t st) {
  const DeviceInfo& dev = device_info();
  const int64_t np_ = round_up(in, NB);
  uint8_t* p = (uint8_t*)ws;
  PrepHeader* hdr = (PrepHeader*)p;
  p += kHeaderBytes;
  float* hd = (float*)p;
  p += round_up((int64_t)sizeof(float) * in, 256);
  const size_t mat = round_up((int64_t)sizeof(float) * np_ * np_, 256);
  float* R = (float*)p; p += mat;      // reversed, damped Hessian; Schur complements in place
  float* Lh = (float*)p; p += mat;     // L's panels (split), for the inverse
  float* Ll = (float*)p; p += mat;
  float* Mh = (float*)p; p += mat;
  float* Ml = (float*)p; p += mat;
  float* Mth = (float*)p; p += mat;
  float* Mtl = (float*)p; p += mat;
  float* Xh = (float*)p; p += mat;
  float* Xl = (float*)p; p += mat;
  float* Pkh = (float*)p; p += round_up((int64_t)sizeof(float) * np_ * NB, 256);
  float* Pkl = (float*)p;
  const bool force_simt = getenv("GPTQ_FORCE_SIMT") && atoi(getenv("GPTQ_FORCE_SIMT")) != 0;

  CUDA_TRY(cudaMemsetAsync(hdr, 0, kHeaderBytes, st));
  CUDA_TRY(cudaMemsetAsync(Mh, 0, 4 * mat, st));  // M, Mt (hi, lo): strictly-off-triangle blocks stay 0
  const float scale = (float)(2.0 / (double)n);
  diag_kernel<<<1, 1024, 0, st>>>(S, in, scale, cfg->damp_percent, hd, dead, hdr);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  rank_kernel<<<(unsigned)((in + 255) / 256), 256, 0, st>>>(hd, in, cfg->desc_act, perm);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  {
    dim3 grid((unsigned)std::min<int64_t>((np_ + 255) / 256, 16), (unsigned)np_);
    gather_kernel<<<grid, 256, 0, st>>>(S, in, np_, scale, perm, dead, hdr, R);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  static bool leaf_cfg = false;
  const size_t leaf_smem = NB * LD * sizeof(float);
  if (!leaf_cfg) {
    CUDA_TRY(cudaFuncSetAttribute(leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)leaf_smem));
    leaf_cfg = true;
  }
  const int KB = (int)(np_ / NB);
  for (int k = 0; k < KB; ++k) {
    leaf_kernel<<<1, 512, leaf_smem, st>>>(R, Mh, Ml, Mth, Mtl, np_, k, hdr);
    note_launch();
    CUDA_TRY(cudaGetLastError());
    const int64_t kB = (int64_t)k * NB;
    const int64_t r0 = kB + NB;
    const int64_t m = np_ - r0;
    if (m <= 0) break;
    split_panel_kernel<<<(unsigned)std::min<int64_t>((m * 32 + 255) / 256, 1024), 256, 0, st>>>(R, np_, r0, kB, m,
                                                                                                 Pkh, Pkl);
    note_launch();
    CUDA_TRY(cudaGetLastError());
    // panel: L[r0:, k] = R[r0:, k] M_kk^T   -> L's panel (split)
    GemmArgs pg;
    pg.op = OP_TF32X3;
    pg.P = {Pkh, Pkl, m, NB, NB};
    pg.Q = {Mh, Ml, np_, np_, np_};
    pg.R = m;
    pg.Cn = NB;
    pg.K = NB;
    pg.p_row0 = 0;
    pg.p_k0 = 0;
    pg.q_row0 = kB;
    pg.q_k0 = kB;
    pg.C = Lh;
    pg.C_lo = Ll;
    pg.ldc = np_;
    pg.c_row0 = r0;
    pg.c_col0 = kB;
    pg.alpha = 1.f;
    pg.beta = 0.f;
    pg.status = &hdr->status;
    CUDA_TRY(run_gemm(pg, st, dev.sms, force_simt));
    // trailing: R[r0:, r0:] -= L[r0:, k] L[r0:, k]^T   (lower triangle)
    GemmArgs tg;
    tg.op = OP_TF32X3;
    tg.P = {Lh, Ll, np_, np_, np_};
    tg.Q = tg.P;
    tg.R = m;
    tg.Cn = m;
    tg.K = NB;
    tg.p_row0 = r0;
    tg.p_k0 = kB;
    tg.q_row0 = r0;
    tg.q_k0 = kB;
    tg.C = R;
    tg.ldc = np_;
    tg.c_row0 = r0;
    tg.c_col0 = r0;
    tg.alpha = -1.f;
    tg.beta = 1.f;
    tg.mask = 2;
    tg.status = &hdr->status;
    CUDA_TRY(run_gemm(tg, st, dev.sms, force_simt));
  }
  // triangular inverse: merge groups pairwise, M21 = -M22 (L21 M11)
  std::vector<std::pair<int64_t, int64_t>> groups;  // (offset, size)
  for (int k = 0; k < KB; ++k) groups.push_back({(int64_t)k * NB, NB});
  while (groups.size() > 1) {
    std::vector<std::pair<int64_t, int64_t>> next;
    size_t i = 0;
    while (i + 1 < groups.size()) {
      // batch consecutive pairs with identical sizes
      const int64_t s1 = groups[i].second, s2 = groups[i + 1].second;
      size_t j = i;
      int nb = 0;
      while (j + 1 < groups.size() && groups[j].second == s1 && groups[j + 1].second == s2 &&
             (nb == 0 || groups[j].first == groups[i].first + (int64_t)nb * (s1 + s2))) {
        next.push_back({groups[j].first, s1 + s2});
        j += 2;
        ++nb;
      }
      const int64_t o1 = groups[i].first, o2 = o1 + s1, stride = s1 + s2;
      // X^T[o1+c][o2+r] = (L21 M11)[r][c] = sum_t L[o2+r][o1+t] Mt[o1+c][o1+t]
      GemmArgs a;
      a.op = OP_TF32X3;
      a.P = {Lh, Ll, np_, np_, np_};
      a.Q = {Mth, Mtl, np_, np_, np_};
      a.R = s2;
      a.Cn = s1;
      a.K = s1;
      a.p_row0 = o2;
      a.p_k0 = o1;
      a.q_row0 = o1;
      a.q_k0 = o1;
      a.C = Xh;
      a.C_lo = Xl;
      a.ldc = np_;
      a.c_row0 = o1;  // transposed store: row o1 + c, col o2 + r
      a.c_col0 = o2;
      a.alpha = 1.f;
      a.beta = 0.f;
      a.transpose = 1;
      a.batch = nb;
      a.bs_p_row = stride;
      a.bs_p_k = stride;
      a.bs_q_row = stride;
      a.bs_q_k = stride;
      a.bs_c_row = stride;
      a.bs_c_col = stride;
      a.status = &hdr->status;
      CUDA_TRY(run_gemm(a, st, dev.sms, force_simt));
      // M21[r][c] = -sum_t M[o2+r][o2+t] X^T[o1+c][o2+t]
      GemmArgs b = a;
      b.P = {Mh, Ml, np_, np_, np_};
      b.Q = {Xh, Xl, np_, np_, np_};
      b.R = s2;
      b.Cn = s1;
      b.K = s2;
      b.p_row0 = o2;
      b.p_k0 = o2;
      b.q_row0 = o1;
      b.q_k0 = o2;
      b.C = Mh;
      b.C_lo = Ml;
      b.c_row0 = o2;
      b.c_col0 = o1;
      b.alpha = -1.f;
      b.transpose = 0;
      CUDA_TRY(run_gemm(b, st, dev.sms, force_simt));
      dim3 tg((unsigned)((s1 + 31) / 32), (unsigned)((s2 + 31) / 32), (unsigned)nb);
      transpose_blocks_kernel<<<tg, 256, 0, st>>>(Mh, Ml, Mth, Mtl, np_, o1, o2, s1, s2, stride);
      note_launch();
      CUDA_TRY(cudaGetLastError());
      i = j;
    }
    if (i < groups.size()) next.push_back(groups[i]);
    groups.swap(next);
  }
  {
    dim3 grid((unsigned)std::min<int64_t>((in + 255) / 256, 16), (unsigned)in);
    write_u_kernel<<<grid, 256, 0, st>>>(Mth, Mtl, np_, in, U);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  uint32_t status = 0;
  CUDA_TRY(cudaMemcpyAsync(&status, &hdr->status, sizeof(status), cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (status & ST_TIMEOUT) return fail(GPTQ_ERR_TIMEOUT, "a bounded device-side wait gave up");
  if (status & ST_NONFINITE) return fail(GPTQ_ERR_NONFINITE, "S holds NaN or Inf");
  if (status & ST_NOT_PD) return fail(GPTQ_ERR_NOT_PD, "the damped Hessian is not positive definite");
  return GPTQ_OK;
}

}  // namespace gptq
