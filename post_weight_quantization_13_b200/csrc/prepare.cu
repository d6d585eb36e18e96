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
//   Cholesky:  right-looking with 64-wide blocks in one cooperative launch
//              (factor_kernel): one CTA factors and inverts each diagonal
//              block while the others form the panel L_ik = R_ik M_kk^T and
//              the trailing update R -= L_ik L_jk^T, in fp32.
//   Inverse:   pairs of already inverted diagonal groups are merged,
//              M21 = -M22 (L21 M11), doubling the group size each level; all
//              merges of one level are one batched tensor-core launch on
//              "split" operands (hi rounded to tf32 plus the exact fp32
//              remainder, 3xTF32 accuracy).
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
// Larger matrices are factored in super-blocks of this size: one cooperative
// launch per diagonal super-block, the panel below it and the trailing
// update of the rest as tensor-core GEMMs (their work grows as np^3).
constexpr int64_t kSuperBlock = 4096;

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

// Ph/Pl[r][c] = split(R[r0 + r][c0 + c]) for c < width: a panel of R as a
// 3xTF32 operand (rows x width, row stride width).
__global__ void __launch_bounds__(256) split_panel_kernel(const float* __restrict__ R, int64_t np_, int64_t r0,
                                                          int64_t c0, int64_t rows, int64_t width,
                                                          float* __restrict__ Ph, float* __restrict__ Pl) {
  const int64_t q = width / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * q;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / q, c4 = (e % q) * 4;
    const float4 v = *reinterpret_cast<const float4*>(R + (r0 + r) * np_ + c0 + c4);
    float4 h, l;
    split_tf32(v.x, h.x, l.x);
    split_tf32(v.y, h.y, l.y);
    split_tf32(v.z, h.z, l.z);
    split_tf32(v.w, h.w, l.w);
    *reinterpret_cast<float4*>(Ph + r * width + c4) = h;
    *reinterpret_cast<float4*>(Pl + r * width + c4) = l;
  }
}

// ------------------------------------------------------------------ factor
// Blocked right-looking Cholesky of R = L L^T in one cooperative launch (all
// CTAs resident), with FB x FB blocks.  Step k (after a grid barrier):
//   CTA 0      panel tile (k+1, k): L = A M_kk^T; then A_{k+1,k+1} -= L L^T
//              and the leaf: L_{k+1,k+1} and its inverse M_{k+1,k+1};
//   CTAs 1..   the other panel tiles L_ik = A_ik M_kk^T (i > k + 1), then
//              the trailing tiles A_ij -= L_ik L_jk^T (i >= j > k, except
//              (k+1, k+1)) once every panel tile of the step is done (a
//              per-step counter).
// So the factorisation of the next diagonal block overlaps the trailing
// update of this step.  Tile products are fp32 FMA on register blocks.
// Tiles that other CTAs write during the launch are read with L2-only loads
// (the L1 caches are not coherent), after a flag or barrier with fences.
// Outputs: L's tiles below the diagonal (fp32 in R, split hi/lo in Lh/Ll)
// and the diagonal blocks of M = L^-1 (fp32 in MD; split in Mh/Ml and
// transposed in Mth/Mtl), which the blocked inverse then merges.
constexpr int FB = 64;          // block size
constexpr int FNT = 256;        // threads per CTA
constexpr int FP = FB + 1;      // pitch of the leaf's A and M tiles
constexpr int TP = FB + 4;      // pitch of transposed operand tiles (float4 rows)

// Warp 0: A[o:o+32, o:o+32] -> L (lower, in place) and M[o:, o:] = L^-1
// (pitch P).  Lane i keeps row i (Cholesky) or column i of M (inverse) in
// registers as a window w[t] = element j + t that slides by one column per
// pivot, so each loop is rolled and small.  Column j of L goes through the
// shared scratch Lt from the diagonal down (Lt[j][t] = L[j + t][j]) and is
// read back with vector loads; window entries past the block's edge read
// stale scratch and are never used.
template <int P>
__device__ __noinline__ void leaf32(float* A, float* M, float* Lt, float* rdiag, int o, PrepHeader* hdr) {
  const int i = threadIdx.x & 31;
  float w[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) w[c] = A[(o + i) * P + o + c];
#pragma unroll 1
  for (int j = 0; j < 32; ++j) {
    float d = __shfl_sync(0xffffffffu, w[0], j);
    if (!(d > 0.f) || !isfinite(d)) {
      if (i == 0) raise_status(&hdr->status, ST_NOT_PD);
      d = 1.f;
    }
    const float rs = rsqrtf(d);
    const float lj = (i == j) ? d * rs : w[0] * rs;  // L[i][j] for i >= j
    A[(o + i) * P + o + j] = (i >= j) ? lj : 0.f;
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
    M[(o + r) * P + o + i] = m;
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

// 32 x 32 products inside the leaf (FNT threads, 2 x 2 outputs each), pitch FP:
//   NT: C[r][c] = sign * sum_t X[r][t] Y[c][t]     NN: ... X[r][t] Y[t][c]
// lower: keep only c <= r; accumulate: C += instead of C =.  Results are
// written after every thread has read its operands.
template <bool NT>
__device__ __forceinline__ void gemm32(const float* X, const float* Y, float* C, float sign, bool lower,
                                       bool accumulate) {
  const int t = threadIdx.x;
  const int r0 = (t / 16) * 2, c0 = (t % 16) * 2;
  float acc[2][2] = {};
#pragma unroll 4
  for (int k = 0; k < 32; ++k) {
    const float x0 = X[r0 * FP + k], x1 = X[(r0 + 1) * FP + k];
    const float y0 = NT ? Y[c0 * FP + k] : Y[k * FP + c0];
    const float y1 = NT ? Y[(c0 + 1) * FP + k] : Y[k * FP + c0 + 1];
    acc[0][0] = fmaf(x0, y0, acc[0][0]);
    acc[0][1] = fmaf(x0, y1, acc[0][1]);
    acc[1][0] = fmaf(x1, y0, acc[1][0]);
    acc[1][1] = fmaf(x1, y1, acc[1][1]);
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int r = r0 + u, c = c0 + v;
      if (lower && c > r) continue;
      const float x = sign * acc[u][v];
      C[r * FP + c] = accumulate ? C[r * FP + c] + x : x;
    }
  __syncthreads();
}

// The FB x FB leaf on A (lower triangle read) and M (zeroed by the caller):
// two 32-blocks and their merge.  Leaves L in A's lower triangle, M = L^-1.
__device__ void leaf64(float* A, float* M, float* Lt, float* rdiag, PrepHeader* hdr) {
  const bool w0 = threadIdx.x < 32;
  if (w0) leaf32<FP>(A, M, Lt, rdiag, 0, hdr);
  __syncthreads();
  float* A21 = A + 32 * FP;
  float* A22 = A + 32 * FP + 32;
  gemm32<true>(A21, M, A21, 1.f, false, false);   // L21 = A21 M11^T
  gemm32<true>(A21, A21, A22, -1.f, true, true);  // A22 -= L21 L21^T (lower)
  if (w0) leaf32<FP>(A, M, Lt, rdiag, 32, hdr);
  __syncthreads();
  float* X = A + 32;                                            // A's upper block: free space
  gemm32<false>(A21, M, X, 1.f, false, false);                  // X = L21 M11
  gemm32<false>(M + 32 * FP + 32, X, M + 32 * FP, -1.f, false, false);  // M21 = -M22 X
}

// 16-byte global -> shared copy through L2 only (cp.async.cg): tiles that
// other CTAs write during the launch must not come from a stale L1 line.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// S[r][t] (pitch TP) <- G[r][t] for an FB x FB tile (row stride ld), async.
__device__ __forceinline__ void prefetch_tile(float* S, const float* G, int64_t ld) {
  for (int e = threadIdx.x; e < FB * FB / 4; e += FNT) {
    const int r = e / (FB / 4), t4 = (e % (FB / 4)) * 4;
    cp_async16(S + r * TP + t4, G + (int64_t)r * ld + t4);
  }
}

// acc[u][v] = sum_t X[tr + 16u][t] Y[tc + 16v][t]   (tr = tid / 16, tc = tid % 16)
// X, Y row-major tiles of pitch TP.  Output rows and columns are strided by
// 16 so that the 16 column groups of a warp read 16 consecutive rows of Y
// (two conflict-free wavefronts per vector load).
__device__ __forceinline__ void tile_product(const float* X, const float* Y, float acc[4][4]) {
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
#pragma unroll 2
  for (int t = 0; t < FB; t += 4) {
    float4 x[4], y[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = *reinterpret_cast<const float4*>(X + (tr + 16 * u) * TP + t);
#pragma unroll
    for (int v = 0; v < 4; ++v) y[v] = *reinterpret_cast<const float4*>(Y + (tc + 16 * v) * TP + t);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        acc[u][v] = fmaf(x[u].x, y[v].x, acc[u][v]);
        acc[u][v] = fmaf(x[u].y, y[v].y, acc[u][v]);
        acc[u][v] = fmaf(x[u].z, y[v].z, acc[u][v]);
        acc[u][v] = fmaf(x[u].w, y[v].w, acc[u][v]);
      }
  }
}

struct FactorParams {
  float* R;
  int64_t np_;
  int T;          // blocks per side
  float* MD;      // [T][FB][FB] diagonal blocks of M (fp32)
  float *Lh, *Ll, *Mh, *Ml, *Mth, *Mtl;
  unsigned* sync;  // [0] arrivals, [1] generation, [2] abort
  int* pdone;      // [T]: panel tiles finished in step k
  PrepHeader* hdr;
};

// Grid-wide barrier for a cooperative launch, bounded by kWaitLimitNs.
// Returns false once any CTA has given up (all CTAs then leave the loop).
__device__ bool grid_barrier(const FactorParams& fp) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* vs = fp.sync;
    const unsigned gen = vs[1];
    __threadfence();
    bool ok = true;
    if (atomicAdd(&fp.sync[0], 1u) == gridDim.x - 1) {
      atomicExch(&fp.sync[0], 0u);
      __threadfence();
      atomicAdd(&fp.sync[1], 1u);
    } else {
      const uint64_t t0 = globaltimer();
      while (vs[1] == gen) {
        if (vs[2]) break;
        if (globaltimer() - t0 > kWaitLimitNs) {
          raise_status(&fp.hdr->status, ST_TIMEOUT);
          atomicExch(&fp.sync[2], 1u);
          break;
        }
      }
    }
    __threadfence();
    ok_s = ok && vs[2] == 0;
  }
  __syncthreads();
  return ok_s != 0;
}

// Wait until pdone[k] (panel tiles finished in step k) reaches target
// (bounded); false on timeout or abort.
__device__ bool wait_panels(const FactorParams& fp, int k, int target) {
  __shared__ int ok_s;
  if (threadIdx.x == 0) {
    volatile int* vf = fp.pdone;
    volatile unsigned* vs = fp.sync;
    bool ok = true;
    const uint64_t t0 = globaltimer();
    while (vf[k] < target) {
      if (vs[2]) {
        ok = false;
        break;
      }
      if (globaltimer() - t0 > kWaitLimitNs) {
        raise_status(&fp.hdr->status, ST_TIMEOUT);
        atomicExch(&fp.sync[2], 1u);
        ok = false;
        break;
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// Write the leaf's M (pitch FP) as diagonal block b: fp32 to MD, split to
// Mh/Ml and, transposed, to Mth/Mtl.
__device__ void store_diag_m(const FactorParams& fp, const float* M, int b) {
  const int64_t o = (int64_t)b * FB;
  float* md = fp.MD + (int64_t)b * FB * FB;
  for (int e = threadIdx.x; e < FB * FB; e += FNT) {
    const int r = e / FB, c = e % FB;
    const float v = M[r * FP + c], vt = M[c * FP + r];
    md[e] = v;
    float h, l;
    split_tf32(v, h, l);
    fp.Mh[(o + r) * fp.np_ + o + c] = h;
    fp.Ml[(o + r) * fp.np_ + o + c] = l;
    split_tf32(vt, h, l);
    fp.Mth[(o + r) * fp.np_ + o + c] = h;
    fp.Mtl[(o + r) * fp.np_ + o + c] = l;
  }
}

// Store the panel tile L (acc, strided layout) at block (i, k): fp32 to R,
// split to Lh/Ll.
__device__ __forceinline__ void store_panel(const FactorParams& fp, int i, int k, const float acc[4][4]) {
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  const int64_t base = (int64_t)i * FB * fp.np_ + (int64_t)k * FB;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t g = base + (int64_t)(tr + 16 * u) * fp.np_ + tc + 16 * v;
      float h, l;
      split_tf32(acc[u][v], h, l);
      fp.R[g] = acc[u][v];
      fp.Lh[g] = h;
      fp.Ll[g] = l;
    }
}

__global__ void __launch_bounds__(FNT, 1) factor_kernel(const FactorParams fp) {
  extern __shared__ __align__(16) float fsm[];
  // double-buffered operand tiles [FB][TP]: X at buffers 0-1, Y at 2-3,
  // the target C at 4-5
  auto Xb = [&](int b) { return fsm + (0 + b) * FB * TP; };
  auto Yb = [&](int b) { return fsm + (2 + b) * FB * TP; };
  auto Cb = [&](int b) { return fsm + (4 + b) * FB * TP; };
  float* LT = fsm + 6 * FB * TP;     // [FB][TP]: L_{k+1,k} (CTA 0)
  float* A = LT + FB * TP;           // [FB][FP]
  float* M = A + FB * FP;            // [FB][FP]
  float* Lt = M + FB * FP;           // [32 * 32 + 32]
  float* rdiag = Lt + 32 * 32 + 32;  // [32]
  const int64_t np_ = fp.np_;
  const int T = fp.T;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  auto tile = [&](int i, int j) { return fp.R + (int64_t)i * FB * np_ + (int64_t)j * FB; };

  if (cta == 0) {  // the first diagonal block
    for (int e = threadIdx.x; e < FB * FB; e += FNT) {
      const int r = e / FB, c = e % FB;
      A[r * FP + c] = __ldcg(fp.R + (int64_t)r * np_ + c);
    }
    for (int e = threadIdx.x; e < FB * FP; e += FNT) M[e] = 0.f;
    __syncthreads();
    leaf64(A, M, Lt, rdiag, fp.hdr);
    store_diag_m(fp, M, 0);
  }
  if (!grid_barrier(fp)) return;

  for (int k = 0; k + 1 < T; ++k) {
    float acc[4][4];
    if (cta == 0) {
      // panel tile (k+1, k) = A M_kk^T with M_kk still in shared memory,
      // then A_{k+1,k+1} -= L L^T and the leaf on it
      prefetch_tile(Xb(0), tile(k + 1, k), np_);
      prefetch_tile(Cb(0), tile(k + 1, k + 1), np_);
      cp_async_commit();
      for (int e = threadIdx.x; e < FB * FB; e += FNT) {
        const int r = e / FB, c = e % FB;
        Yb(0)[r * TP + c] = M[r * FP + c];
      }
      cp_async_wait<0>();
      __syncthreads();
      tile_product(Xb(0), Yb(0), acc);
      store_panel(fp, k + 1, k, acc);
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) LT[(tr + 16 * u) * TP + tc + 16 * v] = acc[u][v];
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(&fp.pdone[k], 1);
      }
      tile_product(LT, LT, acc);  // L L^T
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int r = tr + 16 * u, c = tc + 16 * v;
          A[r * FP + c] = Cb(0)[r * TP + c] - acc[u][v];
        }
      for (int e = threadIdx.x; e < FB * FP; e += FNT) M[e] = 0.f;
      __syncthreads();
      leaf64(A, M, Lt, rdiag, fp.hdr);
      store_diag_m(fp, M, k + 1);
    } else {
      // tasks of this step, dealt round-robin to CTAs 1..G-1: first the
      // panel tiles i = k + 2 .. T - 1, then the trailing tiles column by
      // column (j = k + 1 .. T - 1, i = j .. T - 1, without (k+1, k+1))
      const int W = G - 1, slot = cta - 1;
      const int npanel = T - k - 2;
      const int m = T - k - 1;  // trailing tiles span m x m blocks
      const int total = npanel + m * (m + 1) / 2 - 1;
      int q = slot;
      for (; q < npanel; q += W) {
        const int i = k + 2 + q;
        prefetch_tile(Xb(0), tile(i, k), np_);
        prefetch_tile(Yb(0), fp.MD + (int64_t)k * FB * FB, FB);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        tile_product(Xb(0), Yb(0), acc);
        store_panel(fp, i, k, acc);
        __syncthreads();
        if (threadIdx.x == 0) {
          __threadfence();
          atomicAdd(&fp.pdone[k], 1);
        }
      }
      // every panel tile of the step (CTA 0 adds the first one)
      if (q < total && !wait_panels(fp, k, npanel + 1)) return;
      int jj = 0, base = 0;  // column walk: tiles before column jj
      auto locate = [&](int qq, int& i, int& j) {
        const int t = qq - npanel;
        while (t >= base + (m - jj - (jj == 0 ? 1 : 0))) {
          base += m - jj - (jj == 0 ? 1 : 0);
          ++jj;
        }
        j = k + 1 + jj;
        i = k + 1 + (jj == 0 ? 1 : jj) + (t - base);
      };
      auto prefetch = [&](int b, int i, int j) {
        prefetch_tile(Xb(b), tile(i, k), np_);
        if (i != j) prefetch_tile(Yb(b), tile(j, k), np_);
        prefetch_tile(Cb(b), tile(i, j), np_);
      };
      int ic = 0, jc = 0;
      if (q < total) {
        locate(q, ic, jc);
        prefetch(0, ic, jc);
        cp_async_commit();
      }
      int b = 0;
      for (; q < total; q += W) {
        int in_ = 0, jn = 0;
        const bool more = q + W < total;
        if (more) {
          locate(q + W, in_, jn);
          prefetch(b ^ 1, in_, jn);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        tile_product(Xb(b), ic != jc ? Yb(b) : Xb(b), acc);
        float* Ct = tile(ic, jc);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int r = tr + 16 * u, c = tc + 16 * v;
            Ct[(int64_t)r * np_ + c] = Cb(b)[r * TP + c] - acc[u][v];
          }
        __syncthreads();
        b ^= 1;
        ic = in_;
        jc = jn;
      }
      cp_async_wait<0>();
    }
    if (!grid_barrier(fp)) return;
  }
}

size_t factor_smem_bytes() { return sizeof(float) * (7 * FB * TP + 2 * FB * FP + 32 * 32 + 32 + 32); }

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

cudaError_t run_gemm(GemmArgs& g, cudaStream_t st, int sms) {
  if (!force_simt() && tc_gemm_supported(g)) return tc_gemm(g, st, sms);
  return simt_gemm(g, st);
}

}  // namespace

size_t prepare_ws_bytes(int64_t in) {
  const int64_t np_ = round_up(in, NB);
  size_t b = kHeaderBytes;
  b += round_up((int64_t)sizeof(double) * in, 256);              // hd
  b += 9 * round_up((int64_t)sizeof(float) * np_ * np_, 256);    // R; L, M, Mt, X^T (hi, lo)
  b += round_up((int64_t)sizeof(float) * np_ * FB, 256);         // diagonal blocks of M
  b += round_up((int64_t)sizeof(int) * (np_ / FB + 4), 256);      // barrier and panel flags
  if (np_ > kSuperBlock)                                          // split panel below a super-block
    b += 2 * round_up((int64_t)sizeof(float) * (np_ - kSuperBlock) * kSuperBlock, 256);
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
  float* Xh = (float*)p; p += mat;
  float* Xl = (float*)p; p += mat;
  float* MD = (float*)p; p += round_up((int64_t)sizeof(float) * np_ * FB, 256);
  unsigned* sync = (unsigned*)p;  // [0..2] barrier, then panel flags
  p += round_up((int64_t)sizeof(int) * (np_ / FB + 4), 256);
  float* Pkh = nullptr;
  float* Pkl = nullptr;
  if (np_ > kSuperBlock) {
    Pkh = (float*)p;
    p += round_up((int64_t)sizeof(float) * (np_ - kSuperBlock) * kSuperBlock, 256);
    Pkl = (float*)p;
  }

  CUDA_TRY(cudaMemsetAsync(hdr, 0, kHeaderBytes, st));
  CUDA_TRY(cudaMemsetAsync(Mh, 0, 4 * mat, st));  // M, Mt (hi, lo): strictly-off-triangle blocks stay 0
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
  // blocked Cholesky of R, one cooperative launch per diagonal super-block
  const size_t fsmem = factor_smem_bytes();
  CUDA_TRY(ensure_smem_limit((const void*)factor_kernel, (int)fsmem));
  int per_sm = 0;
  CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, factor_kernel, FNT, fsmem));
  if (per_sm < 1) return fail(GPTQ_ERR_CUDA, "factor_kernel does not fit on an SM");
  // triangular inverse: merge groups pairwise, M21 = -M22 (L21 M11)
  auto merge = [&](std::vector<std::pair<int64_t, int64_t>> groups) -> gptq_status_t {  // (offset, size)
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
      CUDA_TRY(run_gemm(a, st, dev.sms));
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
      CUDA_TRY(run_gemm(b, st, dev.sms));
      dim3 tg((unsigned)((s1 + 31) / 32), (unsigned)((s2 + 31) / 32), (unsigned)nb);
      transpose_blocks_kernel<<<tg, 256, 0, st>>>(Mh, Ml, Mth, Mtl, np_, o1, o2, s1, s2, stride);
      note_launch();
      CUDA_TRY(cudaGetLastError());
      i = j;
    }
    if (i < groups.size()) next.push_back(groups[i]);
    groups.swap(next);
  }
  return GPTQ_OK;
  };
  std::vector<std::pair<int64_t, int64_t>> supers;
  for (int64_t o = 0; o < np_; o += kSuperBlock) {
    const int64_t B = std::min<int64_t>(kSuperBlock, np_ - o);
    const int T = (int)(B / FB);
    supers.push_back({o, B});
    CUDA_TRY(cudaMemsetAsync(sync, 0, sizeof(int) * (T + 4), st));
    const int64_t off = o * np_ + o;
    FactorParams fp;
    fp.R = R + off;
    fp.np_ = np_;
    fp.T = T;
    fp.MD = MD;
    fp.Lh = Lh + off;
    fp.Ll = Ll + off;
    fp.Mh = Mh + off;
    fp.Ml = Ml + off;
    fp.Mth = Mth + off;
    fp.Mtl = Mtl + off;
    fp.sync = sync;
    fp.pdone = (int*)(sync + 4);
    fp.hdr = hdr;
    const int grid = std::max(2, std::min(dev.sms, T * T));
    void* args[] = {&fp};
    CUDA_TRY(cudaLaunchCooperativeKernel((const void*)factor_kernel, dim3(grid), dim3(FNT), args, fsmem, st));
    note_launch();
    // the inverse of this super-block's L (merging its 64-blocks)
    std::vector<std::pair<int64_t, int64_t>> groups;
    for (int k = 0; k < T; ++k) groups.push_back({o + (int64_t)k * FB, FB});
    gptq_status_t ms = merge(groups);
    if (ms != GPTQ_OK) return ms;
    const int64_t r0 = o + B, m = np_ - r0;
    if (m <= 0) break;
    // panel below the super-block, L21 = R21 M_sb^T (split), then the
    // trailing update R22 -= L21 L21^T (lower tiles), both on tensor cores
    split_panel_kernel<<<(unsigned)std::min<int64_t>((m * (B / 4) + 255) / 256, (int64_t)dev.sms * 8), 256, 0,
                         st>>>(R, np_, r0, o, m, B, Pkh, Pkl);
    note_launch();
    CUDA_TRY(cudaGetLastError());
    GemmArgs pg;
    pg.op = OP_TF32X3;
    pg.P = {Pkh, Pkl, m, B, B};
    pg.Q = {Mh, Ml, np_, np_, np_};
    pg.R = m;
    pg.Cn = B;
    pg.K = B;
    pg.q_row0 = o;
    pg.q_k0 = o;
    pg.C = Lh;
    pg.C_lo = Ll;
    pg.ldc = np_;
    pg.c_row0 = r0;
    pg.c_col0 = o;
    pg.alpha = 1.f;
    pg.beta = 0.f;
    pg.status = &hdr->status;
    CUDA_TRY(run_gemm(pg, st, dev.sms));
    GemmArgs tg;
    tg.op = OP_TF32X3;
    tg.P = {Lh, Ll, np_, np_, np_};
    tg.Q = tg.P;
    tg.R = m;
    tg.Cn = m;
    tg.K = B;
    tg.p_row0 = r0;
    tg.p_k0 = o;
    tg.q_row0 = r0;
    tg.q_k0 = o;
    tg.C = R;
    tg.ldc = np_;
    tg.c_row0 = r0;
    tg.c_col0 = r0;
    tg.alpha = -1.f;
    tg.beta = 1.f;
    tg.mask = 2;
    tg.status = &hdr->status;
    CUDA_TRY(run_gemm(tg, st, dev.sms));
  }
  if (supers.size() > 1) {
    gptq_status_t ms = merge(supers);
    if (ms != GPTQ_OK) return ms;
  }
  {
    const unsigned grid = (unsigned)std::min<int64_t>(in, (int64_t)dev.sms * 8);
    write_u_kernel<<<grid, 256, 0, st>>>(Mth, Mtl, np_, in, U);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  return read_device_status(hdr, st);
}

}  // namespace gptq
