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
// Lower triangle (b <= a) of R[a][b] = H_perm_damped[in-1-a][in-1-b], with
// the identity in the padding.  Only the lower triangle is ever read: the
// factorisation's leaf ignores what lies above the diagonal and the trailing
// updates add into lower tiles only.  With the natural order (i <= j for
// b <= a) the S reads run along rows of the stored upper triangle, so they
// coalesce; each block takes whole rows, four columns per thread.
__global__ void __launch_bounds__(256) gather_kernel(const float* __restrict__ S, int64_t in, int64_t np_,
                                                     float scale, const int32_t* __restrict__ perm,
                                                     const uint8_t* __restrict__ dead, PrepHeader* hdr,
                                                     float* __restrict__ R) {
  const float lam = hdr->lambda;
  for (int64_t a = blockIdx.x; a < np_; a += gridDim.x) {
    const int64_t i = a < in ? perm[in - 1 - a] : -1;
    for (int64_t b0 = (int64_t)threadIdx.x * 4; b0 <= a; b0 += (int64_t)blockDim.x * 4) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t b = b0 + u;
        float x = 0.f;
        if (a < in && b < in) {
          const int64_t j = perm[in - 1 - b];
          const int64_t lo = min(i, j), hi = max(i, j);
          const float sv = S[lo * in + hi];
          if (!isfinite(sv)) raise_status(&hdr->status, ST_NONFINITE);
          x = sv * scale;
          if (i == j) x = (dead[i] ? 1.f : x) + lam;
        } else if (a == b) {
          x = 1.f;
        }
        v[u] = x;
      }
      *reinterpret_cast<float4*>(R + a * np_ + b0) = make_float4(v[0], v[1], v[2], v[3]);
    }
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
// factor: M_kk = L_kk^-1 into M and M_kk^T into Mt (both split).  One CTA of
// 512 threads with A (the block, then L) and M in shared memory, recursively:
//   f(o, h): f(o, h/2); L21 = A21 M11^T; A22 -= L21 L21^T; f(o + h/2, h/2);
//            M21 = -M22 (L21 M11)
// down to 32 x 32 blocks, which one warp factors and inverts in registers
// with shuffles (no block-wide barrier per pivot).  The products between
// levels are small shared-memory GEMMs over all 512 threads.
// A pivot that is not positive raises ST_NOT_PD and is replaced by 1 so the
// block stays finite.
constexpr int LD = NB + 1;

// Warp 0: A[o:o+32, o:o+32] -> L (lower, in place) and M[o:, o:] = L^-1.
// Lane i keeps row i (Cholesky) or column i of M (inverse) in registers as a
// window w[t] = element j + t that slides by one column per pivot, so each
// loop is rolled and small: code size, not arithmetic, sets the cost of a
// routine that runs once per launch.  Column j of L goes through the shared
// scratch Lt from the diagonal down (Lt[j][t] = L[j + t][j]) and is read back
// with vector loads; window entries past the block's edge read stale scratch
// and are never used.
__device__ __noinline__ void leaf32(float* A, float* M, float* Lt, float* rdiag, int o, PrepHeader* hdr) {
  const int i = threadIdx.x & 31;
  float w[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) w[c] = A[(o + i) * LD + o + c];
#pragma unroll 1
  for (int j = 0; j < 32; ++j) {
    float d = __shfl_sync(0xffffffffu, w[0], j);
    if (!(d > 0.f) || !isfinite(d)) {
      if (i == 0) raise_status(&hdr->status, ST_NOT_PD);
      d = 1.f;
    }
    const float rs = rsqrtf(d);
    const float lj = (i == j) ? d * rs : w[0] * rs;  // L[i][j] for i >= j
    A[(o + i) * LD + o + j] = (i >= j) ? lj : 0.f;
    if (i >= j) Lt[j * 32 + (i - j)] = lj;
    if (i == j) rdiag[j] = rs;  // 1 / L[j][j]
    __syncwarp();
    const float* cj = Lt + j * 32;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 c4 = *reinterpret_cast<const float4*>(cj + 4 * q);
      if (q > 0) w[4 * q + 0] = fmaf(-lj, c4.x, w[4 * q + 0]);
      w[4 * q + 1] = fmaf(-lj, c4.y, w[4 * q + 1]);
      w[4 * q + 2] = fmaf(-lj, c4.z, w[4 * q + 2]);
      w[4 * q + 3] = fmaf(-lj, c4.w, w[4 * q + 3]);
    }
#pragma unroll
    for (int t = 0; t < 31; ++t) w[t] = w[t + 1];
    w[31] = 0.f;
  }
  __syncwarp();
  // lane i: column i of M = L^-1 by forward substitution on the identity
  // column, w[t] = b_{r+t}: M[r][i] = b_r / L[r][r]; b_k -= L[k][r] M[r][i]
#pragma unroll
  for (int t = 0; t < 32; ++t) w[t] = (t == i) ? 1.f : 0.f;
#pragma unroll 1
  for (int r = 0; r < 32; ++r) {
    const float m = w[0] * rdiag[r];
    M[(o + r) * LD + o + i] = m;
    const float* cr = Lt + r * 32;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 c4 = *reinterpret_cast<const float4*>(cr + 4 * q);
      if (q > 0) w[4 * q + 0] = fmaf(-c4.x, m, w[4 * q + 0]);
      w[4 * q + 1] = fmaf(-c4.y, m, w[4 * q + 1]);
      w[4 * q + 2] = fmaf(-c4.z, m, w[4 * q + 2]);
      w[4 * q + 3] = fmaf(-c4.w, m, w[4 * q + 3]);
    }
#pragma unroll
    for (int t = 0; t < 31; ++t) w[t] = w[t + 1];
    w[31] = 0.f;
  }
  __syncwarp();
}

// C = sign * X op(Y) over H x H outputs in shared memory, all 512 threads,
// each computing a 2 x 4 (H = 64) or 1 x 2 (H = 32) block; results are
// written after every thread has read its operands.
//   NT: C[r][c] = sum_t X[r][t] Y[c][t]      NN: C[r][c] = sum_t X[r][t] Y[t][c]
// lower: keep only c <= r; accumulate: C += instead of C =.
template <int H, bool NT>
__device__ __forceinline__ void smem_gemm(const float* X, const float* Y, float* C, float sign, bool lower,
                                          bool accumulate) {
  constexpr int RB = H == 64 ? 2 : 1;           // rows per thread
  constexpr int CB = H == 64 ? 4 : 2;           // columns per thread
  constexpr int TPR = H / CB;                   // threads per row group
  const int t = threadIdx.x;
  const int r0 = (t / TPR) * RB, c0 = (t % TPR) * CB;
  float acc[RB][CB] = {};
#pragma unroll 4
  for (int k = 0; k < H; ++k) {
    float xv[RB], yv[CB];
#pragma unroll
    for (int u = 0; u < RB; ++u) xv[u] = X[(r0 + u) * LD + k];
#pragma unroll
    for (int v = 0; v < CB; ++v) yv[v] = NT ? Y[(c0 + v) * LD + k] : Y[k * LD + c0 + v];
#pragma unroll
    for (int u = 0; u < RB; ++u)
#pragma unroll
      for (int v = 0; v < CB; ++v) acc[u][v] = fmaf(xv[u], yv[v], acc[u][v]);
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < RB; ++u)
#pragma unroll
    for (int v = 0; v < CB; ++v) {
      const int r = r0 + u, c = c0 + v;
      if (lower && c > r) continue;
      const float x = sign * acc[u][v];
      C[r * LD + c] = accumulate ? C[r * LD + c] + x : x;
    }
  __syncthreads();
}

// One level of the recursion for a block of size 2H at offset o.
template <int H>
__device__ __forceinline__ void leaf_merge_first(float* A, float* M, int o) {
  float* A21 = A + (o + H) * LD + o;
  float* A22 = A + (o + H) * LD + o + H;
  const float* M11 = M + o * LD + o;
  smem_gemm<H, true>(A21, M11, A21, 1.f, false, false);  // L21 = A21 M11^T
  smem_gemm<H, true>(A21, A21, A22, -1.f, true, true);   // A22 -= L21 L21^T (lower)
}
template <int H>
__device__ __forceinline__ void leaf_merge_second(float* A, float* M, int o) {
  const float* L21 = A + (o + H) * LD + o;
  const float* M11 = M + o * LD + o;
  const float* M22 = M + (o + H) * LD + o + H;
  float* X = A + o * LD + o + H;  // upper block of A: free space
  smem_gemm<H, false>(L21, M11, X, 1.f, false, false);                  // X = L21 M11
  smem_gemm<H, false>(M22, X, M + (o + H) * LD + o, -1.f, false, false);  // M21 = -M22 X
}

__global__ void __launch_bounds__(512) leaf_kernel(const float* R, float* Mh, float* Ml, float* Mth, float* Mtl,
                                                   int64_t np_, int k, PrepHeader* hdr) {
  extern __shared__ float sm[];
  float* A = sm;             // [NB][LD]
  float* M = sm + NB * LD;   // [NB][LD]
  __shared__ __align__(16) float Lt[32 * 32 + 32];   // leaf32 scratch (+ window overrun)
  __shared__ float rdiag[32];
  const int64_t o = (int64_t)k * NB;
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e / (NB / 4), c4 = (e % (NB / 4)) * 4;
    const float4 v = *reinterpret_cast<const float4*>(R + (o + r) * np_ + o + c4);
    A[r * LD + c4 + 0] = v.x;
    A[r * LD + c4 + 1] = v.y;
    A[r * LD + c4 + 2] = v.z;
    A[r * LD + c4 + 3] = v.w;
  }
  for (int e = threadIdx.x; e < NB * LD; e += blockDim.x) M[e] = 0.f;
  __syncthreads();
  const bool w0 = threadIdx.x < 32;
  // first half (64)
  if (w0) leaf32(A, M, Lt, rdiag, 0, hdr);
  __syncthreads();
  leaf_merge_first<32>(A, M, 0);
  if (w0) leaf32(A, M, Lt, rdiag, 32, hdr);
  __syncthreads();
  leaf_merge_second<32>(A, M, 0);
  // 128 level, first part
  leaf_merge_first<64>(A, M, 0);
  // second half (64)
  if (w0) leaf32(A, M, Lt, rdiag, 64, hdr);
  __syncthreads();
  leaf_merge_first<32>(A, M, 64);
  if (w0) leaf32(A, M, Lt, rdiag, 96, hdr);
  __syncthreads();
  leaf_merge_second<32>(A, M, 64);
  // 128 level, second part
  leaf_merge_second<64>(A, M, 0);
  // write M and M^T (split)
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e / (NB / 4), c4 = (e % (NB / 4)) * 4;
    const int64_t g = (o + r) * np_ + o + c4;
    float4 h, l;
    split_tf32(M[r * LD + c4 + 0], h.x, l.x);
    split_tf32(M[r * LD + c4 + 1], h.y, l.y);
    split_tf32(M[r * LD + c4 + 2], h.z, l.z);
    split_tf32(M[r * LD + c4 + 3], h.w, l.w);
    *reinterpret_cast<float4*>(Mh + g) = h;
    *reinterpret_cast<float4*>(Ml + g) = l;
    split_tf32(M[(c4 + 0) * LD + r], h.x, l.x);
    split_tf32(M[(c4 + 1) * LD + r], h.y, l.y);
    split_tf32(M[(c4 + 2) * LD + r], h.z, l.z);
    split_tf32(M[(c4 + 3) * LD + r], h.w, l.w);
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
    const unsigned grid = (unsigned)std::min<int64_t>(np_, (int64_t)dev.sms * 8);
    gather_kernel<<<grid, 256, 0, st>>>(S, in, np_, scale, perm, dead, hdr, R);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  static bool leaf_cfg = false;
  const size_t leaf_smem = 2 * NB * LD * sizeof(float);
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
    const unsigned grid = (unsigned)std::min<int64_t>(in, (int64_t)dev.sms * 8);
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
