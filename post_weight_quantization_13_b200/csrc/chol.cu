// Blocked Cholesky factorisation R = L L^T ("Using AutoGPTQ in Practice":
// the Hessian's Cholesky factorization) and the inverse M = L^-1, in one
// cooperative launch.  R is the reversed, damped Hessian of gptq_prepare_hinv
// (lower triangle, np x np, np a multiple of 128); U = J M J is read from M^T
// afterwards.
//
// Right-looking with 64-wide blocks and a look-ahead of one block.  Step k:
//   CTA 0 (the chain)   L_{k+1,k} = R_{k+1,k} M_kk^T and R_{k+1,k+1} - L L^T
//                       as 3xTF32 tcgen05 MMAs (M = 128 with zero rows), then
//                       the leaf of block k+1: its Cholesky factor in
//                       registers (one pivot chain per 32 rows) and the
//                       factor's inverse M_{k+1,k+1}, pipelined through shared
//                       memory.  Three warps with little leaf work meanwhile
//                       fetch the next step's two tiles once the workers have
//                       updated them.  The leaf's off-diagonal inverse block
//                       is a forward substitution that follows the second
//                       half's pivots, so the leaf ends with its last pivot
//                       chain.
//   CTAs 1.. (workers)  3xTF32 tcgen05 tile tasks (128 x 128 or 128 x 64,
//                       K = 64):
//                         M row tiles   M_kj = -M_kk G_kj   (j < k)
//                         panel tiles   L_ik = R_ik M_kk^T  (i >= k+2)
//                         trailing      R_ij -= L_ik L_jk^T (lower, block k+1 on)
//                         accumulation  G_ij += L_ik M_kj   (i > k, j <= k)
//                       where G accumulates sum_t L_it M_tj, so block row k of
//                       M is final once step k - 1's accumulation has landed.
// The CTAs never meet at a grid barrier: counters in global memory publish
// the diagonal blocks, panel tiles, M row tiles, and the trailing and
// accumulation tiles that have landed, and each task waits for exactly the
// counters its operands depend on (the reduce-adds of consecutive steps reach
// each element in step order).
//
// Worker CTAs: warps 0-3 stage a task's split operands (tf32 hi plus the exact
// fp32 remainder) in a two-stage ring of 128-byte-swizzled K chunks, by TMA
// tensor copies (L, M^T) or by splitting fp32 tiles on the way (R, G^T); one
// thread issues the MMAs chunk by chunk; warps 4-7 read the tensor-memory
// accumulator and write the result: trailing and accumulation tiles by TMA
// reduce-add into R and G^T in L2, panel and M row tiles by TMA tensor stores.
// Two tensor-memory accumulators let a task's epilogue overlap the next
// task's MMAs.
//
// Every wait is bounded by %globaltimer; a wait that gives up raises
// ST_TIMEOUT, sets the launch-wide abort flag and unwinds.
#include <algorithm>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {
namespace {

constexpr int FB = 64;        // block size of the factorisation
constexpr int FNT = 256;      // threads per CTA
constexpr int FP = FB + 1;    // pitch of the leaf's A and M tiles
constexpr int TP = FB + 4;    // pitch of the chain's operand tiles (float4 rows)

// worker shared-memory plan: four regions (A hi/lo, B hi/lo), each 128 rows x
// two 128-byte K chunks (K = 64 tf32)
constexpr uint32_t kChunkBytes = 128 * 128;         // 128 rows x 128 bytes
constexpr uint32_t kRegionBytes = 2 * kChunkBytes;  // K = 64
constexpr uint32_t kStageBytes = 32 * 128 * 4;      // one epilogue pass: 32 rows x 128 columns fp32
constexpr int kStages = 4;                           // epilogue staging buffers (one per 32-row pass)
constexpr uint32_t kWorkerSmem = 4 * kRegionBytes + kStages * kStageBytes;  // 192 KB
constexpr uint32_t kTmemCols = 256;                 // two 128-column accumulators
// chain CTA: fp32 tiles, then (1024-aligned) the tensor-core operand regions
constexpr uint32_t kChainFloats = 4 * FB * TP + 2 * FB * FP + FB * 64 + FB + 4;
constexpr uint32_t kChainOpOffset = (kChainFloats * 4 + 1023) / 1024 * 1024;
constexpr uint32_t kChainOpABytes = 2 * 2 * 128 * 128;  // 128 rows x K 64, hi and lo
constexpr uint32_t kChainOpBBytes = 2 * 2 * 64 * 128;   // 64 rows x K 64, hi and lo

struct CholParams {
  float* R;        // np x np (lower triangle used), updated in place
  int64_t np_;
  int T;           // np / 64
  float *Lh, *Ll;  // split L: panel tiles below the diagonal blocks
  float *Mh, *Ml;  // split diagonal blocks of M = L^-1
  float *Mth, *Mtl;
  unsigned* sync;  // [2] abort, [3] diagonal blocks published (M_kk for k < count)
  int* pdone;      // [T]: panel tiles written in step k (CTA 0 adds one)
  int* tdone;      // [T]: trailing tiles of step k whose reduce-adds have landed
  int* t0done;     // [T]: 1 once trailing tile (0, 0) of step k has landed
  int* mrdone;     // [T]: tiles of block row k of M written
  int* gdone;      // [T]: inverse-accumulator tiles of step k whose reduce-adds have landed
  int* p0done;     // [T]: 1 once panel tile 0 of step k (rows of block k + 2) is written
  int* lcdone;     // [T]: 1 once CTA 0 has written L_{k+1,k}
  float* Gt;       // np x np: G^T, G_ij = sum over t < (current step) of L_it M_tj
  uint32_t* status;
};

// ------------------------------------------------------------------ sync
__device__ __forceinline__ bool aborted(const CholParams& p) {
  return *(volatile unsigned*)(p.sync + 2) != 0;
}

__device__ __forceinline__ void give_up(const CholParams& p) {
  raise_status(p.status, ST_TIMEOUT);
  atomicExch(p.sync + 2, 1u);
}

// Wait until *f >= target (another CTA raises it), bounded by kWaitLimitNs;
// false once any CTA has given up.  One thread; a __threadfence follows a
// successful wait, so data published before the counter is then visible.
__device__ bool wait_ge(const CholParams& p, const int* f, int target) {
  volatile const int* vf = f;
  if (vf[0] < target) {
    const uint64_t t0 = globaltimer();
    for (;;) {
      // both loads are in flight together: one L2 round trip a poll
      const int v = vf[0];
      const bool ab = aborted(p);
      if (v >= target) break;
      if (ab) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        give_up(p);
        return false;
      }
      __nanosleep(64);
    }
  }
  __threadfence();
  return true;
}

// ------------------------------------------------------------------ copies
// 16-byte global -> shared copy through L2 only (cp.async.cg): data other
// CTAs write during the launch must not come from a stale L1 line.  With
// valid == false the 16 bytes are zero-filled and nothing is read.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid = true) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}


// Shared-memory flag between two warps of one CTA (release / acquire).
__device__ __forceinline__ void st_release_cta(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// ------------------------------------------------------------------ chain CTA
// The leaf: A (FB x FB, pitch FP, lower triangle read) -> M = L^-1 (pitch FP,
// zeros above the diagonal), where A = L L^T.  Five warps run chains of
// pivots over registers, fed through shared memory:
//   warp 0  factors rows 0..31 (pivots 0..31); lane i keeps row i; then
//           forms M10 = L11^-1 Y with Y = -L10 M00: Y once L10 and M00 are
//           complete (lane = column), then forward substitution with L11
//           behind warp 6;
//   warp 1  rows 32..63, columns 0..31: forms L[32+i][j] for pivots 0..31
//           from the pivots warp 0 publishes;
//   warp 6  rows 32..63, columns 32..63: applies the first 32 pivots' updates
//           to the trailing block, then factors it (pivots 32..63);
//   warp 7  inverts L00 (M00 = L00^-1 by forward substitution, lane =
//           column), trailing warp 0 by a pivot or more;
//   warp 3  inverts L11 (M11) behind warp 6;
//   warp 4  zeroes the upper block of M;
//   warps 1 (once L10 is done), 2 and 5 fetch the next step's tiles.
// Warp w issues on scheduler w % 4: warp 6's pivots share theirs with a
// warp that mostly sleeps (2, fetching the next tiles), and warps 0, 1, 3 and
// 7 do not run their pivot chains on the same scheduler at the same time.
// Column j of L goes to Lc[j][.] and 1/L_jj to rdiag[j]; fl[0..2] count the
// pivots published by warps 0, 1 and 6 (release / acquire, once per pass of
// four pivots) and fl[3] the rows of M00 (once, at the end).  Each lane keeps
// a 32-entry window of its row (or column) that slides by four pivots per
// pass, so every register index is a compile-time constant and the code of
// one pass serves all passes.  A non-positive or non-finite pivot raises
// ST_NOT_PD (it is replaced by 1 so the leaf finishes).  False if a wait gave
// up.
constexpr int LCP = 64;  // pitch of Lc (one column of L per row)

__device__ __forceinline__ bool wait_count(const int* f, int j) {
  if (ld_acquire_cta(f) > j) return true;
  const uint64_t t0 = globaltimer();
  while (ld_acquire_cta(f) <= j) {
    __nanosleep(32);  // leave the issue slots to the warp being waited for
    if (globaltimer() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// w[t] -= s * col[t] for t in (u, 32), col 16-byte aligned (8 vector loads).
template <int U>
__device__ __forceinline__ void axpy_window(float (&w)[32], float s, const float* col) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 c4 = *reinterpret_cast<const float4*>(col + 4 * q);
    if (4 * q + 0 > U) w[4 * q + 0] = fmaf(-s, c4.x, w[4 * q + 0]);
    if (4 * q + 1 > U) w[4 * q + 1] = fmaf(-s, c4.y, w[4 * q + 1]);
    if (4 * q + 2 > U) w[4 * q + 2] = fmaf(-s, c4.z, w[4 * q + 2]);
    if (4 * q + 3 > U) w[4 * q + 3] = fmaf(-s, c4.w, w[4 * q + 3]);
  }
}

__device__ __forceinline__ void shift4(float (&w)[32]) {
#pragma unroll
  for (int t = 0; t < 28; ++t) w[t] = w[t + 4];
#pragma unroll
  for (int t = 28; t < 32; ++t) w[t] = 0.f;
}

// One factor pivot on a window whose slot U holds column j of the lane's row
// (row j itself sits on lane jl): publish column j (rows row0 + lane) and
// 1/L_jj, then update the window with the column's rows col0 .. col0 + 31.
// The chain from one pivot to the next runs through registers only: dn is,
// on the lane of the pivot row, the fully updated diagonal entry.  Row j + 1's
// lane forms its next diagonal entry from its own L[j+1][j] (w - l l), and the
// column j + 1 entries of every lane take L[j+1][j] by shuffle; the other
// columns are updated from shared memory, two or more pivots ahead of use.
template <int U>
__device__ __forceinline__ bool factor_pivot(float (&w)[32], float& dn, int j, int jl, int row0, float* Lc,
                                             float* rdiag, const float* col) {
  const int lane = threadIdx.x & 31;
  float d = __shfl_sync(0xffffffffu, dn, jl);
  bool bad = false;
  if (!(d > 0.f) || !isfinite(d)) {
    bad = true;
    d = 1.f;
  }
  const float rs = rsqrtf(d);
  const float l = w[U] * rs;
  dn = fmaf(-l, l, w[U + 1]);                               // lane jl + 1: next pivot
  const float c1 = __shfl_sync(0xffffffffu, l, (jl + 1) & 31);  // L[j+1][j]
  w[U + 1] = fmaf(-l, c1, w[U + 1]);
  Lc[j * LCP + row0 + lane] = l;
  if (lane == 0) rdiag[j] = rs;
  __syncwarp();
  axpy_window<U + 1>(w, l, col);
  return bad;
}

// Publish pivots up to j (inclusive) to the warps that wait on flag: once per
// pass of four pivots, after the pass's columns are in shared memory.
__device__ __forceinline__ void publish(int* flag, int j) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) st_release_cta(flag, j + 1);
}

// Forward substitution with L on the pivots o .. o + 31, lane = one column of
// the right-hand side: x holds that column's rows o + 4m .. o + 4m + 31 at
// pass m (the window slides by four rows a pass; the rows past o + 31 are
// never read), and row j of the solution goes to M[j][oc + lane].  Follows
// the pivots as flag f publishes them.  False if a wait gave up.
__device__ __forceinline__ bool forward_subst(float (&x)[32], int o, int oc, const int* f, float* M, const float* Lc,
                                              const float* rdiag) {
  const int lane = threadIdx.x & 31;
  bool ok = true;
#pragma unroll 1
  for (int m = 0; m < 8 && ok; ++m) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = o + 4 * m + u;
      if (!wait_count(f, j)) ok = false;
      const float mj = x[u] * rdiag[j];
      M[j * FP + oc + lane] = mj;
      const float* col = Lc + j * LCP + o + 4 * m;
      switch (u) {
        case 0: axpy_window<0>(x, mj, col); break;
        case 1: axpy_window<1>(x, mj, col); break;
        case 2: axpy_window<2>(x, mj, col); break;
        default: axpy_window<3>(x, mj, col); break;
      }
    }
    shift4(x);
  }
  return ok;
}

// Tiles of the chain's next step, fetched by warps 1, 2 and 5 (a third each)
// while the leaf runs, once the workers have applied every update to them.
struct NextTiles {
  bool active;
  float *X, *C;               // shared destinations (pitch TP)
  const float *gX, *gC;       // R tiles (k+2, k+1) and (k+2, k+2)
  int k;                      // the step whose trailing tile (0, 0) must have landed
};

__device__ void fetch_next_tiles(const NextTiles& nt, int64_t np, const CholParams& p, int part, int nparts) {
  const int lane = threadIdx.x & 31;
  int go = 0;
  if (lane == 0) {
    bool ok = true;
    // trailing tile (0, 0) of step k brings the last update that the chain's
    // next step needs in both tiles: the worker that wrote it waited, before
    // its step, for every trailing tile of step k - 1 to land, and those
    // workers for step k - 2's, and so on
    if (nt.k >= 0) ok = wait_ge(p, &p.t0done[nt.k], 1);
    go = ok;
  }
  go = __shfl_sync(0xffffffffu, go, 0);
  if (!go) return;
  // this warp's share of the two tiles' 16-byte pieces
  for (int e = part * 32 + lane; e < 2 * FB * FB / 4; e += 32 * nparts) {
    const int which = e / (FB * FB / 4), q = e % (FB * FB / 4);
    const int r = q / (FB / 4), t4 = (q % (FB / 4)) * 4;
    cp_async16((which ? nt.C : nt.X) + r * TP + t4, (which ? nt.gC : nt.gX) + (int64_t)r * np + t4);
  }
  cp_async_commit();
  cp_async_wait<0>();
}

__device__ bool leaf64(const float* A, float* M, float* Lc, float* rdiag, int* fl, const CholParams& p,
                       const NextTiles& nt) {
  __shared__ int ok_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 4) fl[threadIdx.x] = 0;
  if (threadIdx.x == 0) ok_s = 1;
  __syncthreads();
  bool ok = true, bad = false;
  if (warp == 0) {
    float w[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) w[t] = t <= lane ? A[lane * FP + t] : 0.f;
    float dn = w[0];
#pragma unroll 1
    for (int m = 0; m < 8; ++m) {
      const float* col = Lc + 4 * m;
      bad |= factor_pivot<0>(w, dn, 4 * m + 0, 4 * m + 0, 0, Lc, rdiag, col + (4 * m + 0) * LCP);
      bad |= factor_pivot<1>(w, dn, 4 * m + 1, 4 * m + 1, 0, Lc, rdiag, col + (4 * m + 1) * LCP);
      bad |= factor_pivot<2>(w, dn, 4 * m + 2, 4 * m + 2, 0, Lc, rdiag, col + (4 * m + 2) * LCP);
      bad |= factor_pivot<3>(w, dn, 4 * m + 3, 4 * m + 3, 0, Lc, rdiag, col + (4 * m + 3) * LCP);
      publish(&fl[0], 4 * m + 3);
      shift4(w);
    }
    // M10: Y = -L10 M00 (x[r] = Y[r][lane]), then L11 M10 = Y
    float x[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) x[t] = 0.f;
    ok = wait_count(&fl[1], 31) && wait_count(&fl[3], 31);
    if (ok) {
#pragma unroll 1
      for (int t = 0; t < 32; ++t) axpy_window<-1>(x, M[t * FP + lane], Lc + t * LCP + 32);
      ok = forward_subst(x, 32, 0, &fl[2], M, Lc, rdiag);
    }
  } else if (warp == 1) {
    // rows 32..63, columns 0..31: L[32+i][j] = A'[32+i][j] / L_jj
    float v[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) v[t] = A[(32 + lane) * FP + t];
#pragma unroll 1
    for (int m = 0; m < 8 && ok; ++m) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = 4 * m + u;
        if (!wait_count(&fl[0], j)) ok = false;
        const float l = v[u] * rdiag[j];
        Lc[j * LCP + 32 + lane] = l;
        __syncwarp();
        const float* col = Lc + j * LCP + 4 * m;
        switch (u) {
          case 0: axpy_window<0>(v, l, col); break;
          case 1: axpy_window<1>(v, l, col); break;
          case 2: axpy_window<2>(v, l, col); break;
          default: axpy_window<3>(v, l, col); break;
        }
      }
      publish(&fl[1], 4 * m + 3);
      shift4(v);
    }
    if (ok && nt.active) fetch_next_tiles(nt, p.np_, p, 0, 3);
  } else if (warp == 6) {
    float z[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) z[t] = t <= lane ? A[(32 + lane) * FP + 32 + t] : 0.f;
    // the first 32 pivots' updates of the trailing block
#pragma unroll 1
    for (int j = 0; j < 32 && ok; ++j) {
      if (!wait_count(&fl[1], j)) ok = false;
      const float li = Lc[j * LCP + 32 + lane];
      axpy_window<-1>(z, li, Lc + j * LCP + 32);
    }
    // then its own factorisation, pivots 32..63
    float dn = z[0];
#pragma unroll 1
    for (int m = 0; m < 8; ++m) {
      const float* col = Lc + 32 + 4 * m;
      bad |= factor_pivot<0>(z, dn, 32 + 4 * m + 0, 4 * m + 0, 32, Lc, rdiag, col + (32 + 4 * m + 0) * LCP);
      bad |= factor_pivot<1>(z, dn, 32 + 4 * m + 1, 4 * m + 1, 32, Lc, rdiag, col + (32 + 4 * m + 1) * LCP);
      bad |= factor_pivot<2>(z, dn, 32 + 4 * m + 2, 4 * m + 2, 32, Lc, rdiag, col + (32 + 4 * m + 2) * LCP);
      bad |= factor_pivot<3>(z, dn, 32 + 4 * m + 3, 4 * m + 3, 32, Lc, rdiag, col + (32 + 4 * m + 3) * LCP);
      publish(&fl[2], 32 + 4 * m + 3);
      shift4(z);
    }
  } else if (warp == 7 || warp == 3) {
    // M00 = L00^-1 (warp 7) and M11 = L11^-1 (warp 3): right-hand side I
    float x[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) x[t] = t == lane ? 1.f : 0.f;
    if (warp == 7) {
      ok = forward_subst(x, 0, 0, &fl[0], M, Lc, rdiag);
      publish(&fl[3], 31);
    } else {
      ok = forward_subst(x, 32, 32, &fl[2], M, Lc, rdiag);
    }
  } else if (warp == 4) {
    for (int e = lane; e < 32 * 32; e += 32) M[(e >> 5) * FP + 32 + (e & 31)] = 0.f;
  } else if ((warp == 2 || warp == 5) && nt.active) {
    fetch_next_tiles(nt, p.np_, p, warp == 2 ? 1 : 2, 3);
  }
  if (bad && lane == 0) raise_status(p.status, ST_NOT_PD);
  if (!ok && lane == 0) ok_s = 0;
  __syncthreads();
  return ok_s != 0;
}

// Diagonal block b of M (pitch FP) -> split Mh/Ml and, transposed, Mth/Mtl.
__device__ void store_diag_m(const CholParams& p, const float* M, int b) {
  const int64_t o = (int64_t)b * FB;
  for (int e = threadIdx.x; e < FB * FB; e += FNT) {
    const int r = e / FB, c = e % FB;
    const float v = M[r * FP + c], vt = M[c * FP + r];
    float h, l;
    split_tf32(v, h, l);
    p.Mh[(o + r) * p.np_ + o + c] = h;
    p.Ml[(o + r) * p.np_ + o + c] = l;
    split_tf32(vt, h, l);
    p.Mth[(o + r) * p.np_ + o + c] = h;
    p.Mtl[(o + r) * p.np_ + o + c] = l;
  }
}

// ------------------------------------------------------------------ workers

// Stage rows [row0, row0 + nrows) x columns [col0, col0 + 64) of a split
// matrix (hi, lo; row stride ld) into regions Shi, Slo: 128-byte swizzled,
// two K chunks of 32.  Rows at or past rmax are zero-filled.  Loader threads
// only (128).
__device__ __forceinline__ void stage_split(uint8_t* Shi, uint8_t* Slo, const float* hi, const float* lo,
                                            int64_t ld, int64_t row0, int nrows, int64_t col0, int64_t rmax) {
  const int lt = threadIdx.x;  // 0..127
  for (int e = lt; e < nrows * 16; e += 128) {
    const int r = e >> 4, g = e & 15;  // g: 16-byte unit along K (0..15)
    const int ch = g >> 3, u = g & 7;
    const int64_t gr = row0 + r;
    const bool valid = gr < rmax;
    const int64_t off = (valid ? gr : 0) * ld + col0 + 4 * g;
    const uint32_t so = ch * kChunkBytes + sw128(r, u);
    cp_async16(Shi + so, hi + off, valid);
    cp_async16(Slo + so, lo + off, valid);
  }
}

// The same from an unsplit fp32 matrix (split while staging), 128 rows: all
// sixteen 16-byte loads of a thread are in flight before the first store.
__device__ __forceinline__ void stage_fp32(uint8_t* Shi, uint8_t* Slo, const float* src, int64_t ld,
                                           int64_t row0, int64_t col0, int64_t rmax) {
  const int lt = threadIdx.x;
  float4 v[16];
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int e = lt + 128 * it;
    const int r = e >> 4, g = e & 15;
    const int64_t gr = row0 + r;
    v[it] = gr < rmax ? __ldcg(reinterpret_cast<const float4*>(src + gr * ld + col0 + 4 * g))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int e = lt + 128 * it;
    const int r = e >> 4, g = e & 15;
    const int ch = g >> 3, u = g & 7;
    float4 h, l;
    split_tf32(v[it].x, h.x, l.x);
    split_tf32(v[it].y, h.y, l.y);
    split_tf32(v[it].z, h.z, l.z);
    split_tf32(v[it].w, h.w, l.w);
    const uint32_t so = ch * kChunkBytes + sw128(r, u);
    *reinterpret_cast<float4*>(Shi + so) = h;
    *reinterpret_cast<float4*>(Slo + so) = l;
  }
}

// 24 MMAs: D (+)= A B^T over K = 64 with split operands (hi hi + hi lo + lo hi);
// the operands' two K chunks are a_chunk / b_chunk bytes apart.
__device__ __forceinline__ void issue_mma_strided(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t a_chunk,
                                                  uint32_t b_hi, uint32_t b_lo, uint32_t b_chunk, uint32_t idesc) {
#pragma unroll
  for (int ch = 0; ch < 2; ++ch)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t ah = smem_desc_k_sw128(a_hi + ch * a_chunk + kk * 32);
      const uint64_t al = smem_desc_k_sw128(a_lo + ch * a_chunk + kk * 32);
      const uint64_t bh = smem_desc_k_sw128(b_hi + ch * b_chunk + kk * 32);
      const uint64_t bl = smem_desc_k_sw128(b_lo + ch * b_chunk + kk * 32);
      umma_tf32(d, ah, bh, idesc, (ch | kk) ? 1u : 0u);
      umma_tf32(d, ah, bl, idesc, 1u);
      umma_tf32(d, al, bh, idesc, 1u);
    }
}


// The tile tasks of step k, in this order:
//   kind 2  M row tiles: M_kj = -M_kk G_kj for the columns before block k
//           (128 columns each; G_kj is final once step k - 1's accumulation
//           has landed);
//   kind 0  panel tiles L_ik = R_ik M_kk^T, i >= k + 2 (128 rows each);
//   kind 1  trailing tiles R_ij -= L_ik L_jk^T, lower triangle from block
//           k + 1 on (128 x 128, block (k+1, k+1) excluded);
//   kind 3  inverse accumulation G_ij += L_ik M_kj for the rows after block k
//           and the columns up to block k (128 x 128).
// So M = L^-1 is complete, block row by block row, when the factorisation
// is; step T - 1 has only its M row tiles.
struct Task {
  int kind;
  int64_t r0;   // first row of the output tile
  int64_t c0;   // first column of the output tile
  int diag;     // trailing tile on the diagonal (both operands the same rows)
};

struct StepTasks {
  int nmrow, npan, ntrail, ngupd;
  int mg;  // row tiles of the inverse accumulation
  __host__ __device__ __forceinline__ int total() const { return nmrow + npan + ntrail + ngupd; }
};

__host__ __device__ __forceinline__ StepTasks step_tasks(int64_t np, int k) {
  StepTasks st;
  const int T = (int)(np / FB);
  st.nmrow = (k + 1) / 2;  // columns [0, 64k) in 128-column tiles
  const int64_t pr0 = (int64_t)FB * (k + 2);
  st.npan = (k + 1 < T && pr0 < np) ? (int)((np - pr0 + 127) / 128) : 0;
  const int64_t s = (int64_t)FB * (k + 1);
  const int64_t rem = np - s;
  const int m = (k + 1 < T && rem > FB) ? (int)((rem + 127) / 128) : 0;
  st.ntrail = m * (m + 1) / 2;
  st.mg = (k + 1 < T) ? (int)((rem + 127) / 128) : 0;
  st.ngupd = st.mg * ((k + 2) / 2);  // columns [0, 64(k+1)) in 128-column tiles
  return st;
}

// Position t of a worker's step list -> index in the kind order above.  The
// two tasks the chain's next step waits for come first: panel tile 0 (the
// rows of block k + 2) and trailing tile (0, 0), which holds the chain's
// next two tiles; the rest keep the kind order.
__host__ __device__ __forceinline__ int task_slot(int t, const StepTasks& st) {
  if (st.npan == 0 || st.ntrail == 0) return t;
  const int p0 = st.nmrow, t0 = st.nmrow + st.npan;
  if (t == 0) return p0;
  if (t == 1) return t0;
  t -= 2;
  if (t < p0) return t;
  if (t < t0 - 1) return t + 1;
  return t + 2;
}

__device__ __forceinline__ Task task_of(int64_t np, int k, int t, const StepTasks& st) {
  t = task_slot(t, st);
  Task x;
  x.diag = 0;
  if (t < st.nmrow) {
    x.kind = 2;
    x.r0 = (int64_t)FB * k;
    x.c0 = 128 * (int64_t)t;
    return x;
  }
  t -= st.nmrow;
  if (t < st.npan) {
    x.kind = 0;
    x.r0 = (int64_t)FB * (k + 2) + 128 * (int64_t)t;
    x.c0 = (int64_t)FB * k;
    return x;
  }
  t -= st.npan;
  const int64_t s = (int64_t)FB * (k + 1);
  if (t < st.ntrail) {
    // lower-triangular tile (a, b), b <= a, numbered row by row
    int a = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((a + 1) * (a + 2) / 2 <= t) ++a;
    while (a * (a + 1) / 2 > t) --a;
    const int b = t - a * (a + 1) / 2;
    x.kind = 1;
    x.r0 = s + 128 * (int64_t)a;
    x.c0 = s + 128 * (int64_t)b;
    x.diag = a == b;
    return x;
  }
  t -= st.ntrail;
  x.kind = 3;
  x.r0 = s + 128 * (int64_t)(t % st.mg);
  x.c0 = 128 * (int64_t)(t / st.mg);
  return x;
}

// Operand loads by TMA: the split panel columns of L and of M^T, boxes of 32
// columns (one 128-byte swizzled K chunk) by 128 rows.
struct OpMaps {
  CUtensorMap lh, ll, mth, mtl;
  CUtensorMap mth64, mtl64;  // the same with 64-row boxes (a half tile of M^T rows)
};

__global__ void __launch_bounds__(FNT, 1) chol_kernel(const __grid_constant__ CUtensorMap rmap,
                                                      const __grid_constant__ CUtensorMap gmap,
                                                      const __grid_constant__ OpMaps om, const CholParams p) {
  extern __shared__ __align__(1024) uint8_t csm_raw[];
  uint8_t* csm = (uint8_t*)(((uintptr_t)csm_raw + 1023) & ~(uintptr_t)1023);
  const int64_t np = p.np_;
  const int T = p.T;
  const int cta = blockIdx.x;
  const int G = gridDim.x;

  if (cta == 0) {
    // ---------------------------------------------------------------- chain
    float* fsm = reinterpret_cast<float*>(csm);
    float* Xb2 = fsm;                // [2][FB][TP] R_{k+1,k} (double-buffered across steps)
    float* Cb2 = Xb2 + 2 * FB * TP;  // [2][FB][TP] R_{k+1,k+1}
    float* A = Cb2 + 2 * FB * TP;    // [FB][FP]
    float* M = A + FB * FP;          // [FB][FP]
    float* Lc = M + FB * FP;         // [FB][LCP] columns of L (leaf), 16-byte aligned
    float* rdiag = Lc + FB * LCP;    // [FB]
    int* fl = reinterpret_cast<int*>(rdiag + FB);
    // tensor-core operands of the chain's two products (split, 128-byte
    // swizzled, K = 64 in two chunks): OPA 128 rows (rows 64..127 stay zero,
    // the MMA's M is 128), OPB 64 rows
    uint8_t* OPA = csm + kChainOpOffset;
    uint8_t* OPB = OPA + kChainOpABytes;
    constexpr uint32_t kAChunk = 128 * 128, kBChunk = 64 * 128;
    __shared__ uint64_t cbar;
    __shared__ uint32_t ctmem;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
      mbar_init(&cbar, 1);
      fence_mbar_init();
    }
    if (warp == 0) {
      tmem_alloc(&ctmem, 128);
      tmem_relinquish();
    }
    for (int e = threadIdx.x; e < (int)(kChainOpABytes / 16); e += FNT) {
      // zero OPA (rows 64..127 are never written again)
      reinterpret_cast<float4*>(OPA)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t ctb = ctmem;
    const uint32_t oah = smem_u32(OPA), oal = oah + 2 * kAChunk;
    const uint32_t obh = smem_u32(OPB), obl = obh + 2 * kBChunk;
    uint32_t cphase = 0;
    auto tile = [&](int i, int j) { return p.R + (int64_t)i * FB * np + (int64_t)j * FB; };
    // one 64-row operand into a region: element (r, t) of a row-major source
    // with pitch ld, split, at row r of the swizzled K-major layout
    auto stage_op = [&](uint8_t* dst, uint32_t chunk, const float* src, int ld) {
      for (int e = threadIdx.x; e < FB * 16; e += FNT) {
        const int r = e >> 4, g = e & 15;
        const float* q = src + r * ld + 4 * g;
        float4 h, l;
        split_tf32(q[0], h.x, l.x);
        split_tf32(q[1], h.y, l.y);
        split_tf32(q[2], h.z, l.z);
        split_tf32(q[3], h.w, l.w);
        const uint32_t so = (g >> 3) * chunk + sw128(r, g & 7);
        *reinterpret_cast<float4*>(dst + so) = h;
        *reinterpret_cast<float4*>(dst + 2 * chunk + so) = l;
      }
    };
    auto publish_m = [&](int count) {
      fence_proxy_async_global();  // workers read M_kk^T by TMA
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        atomicExch((int*)&p.sync[3], count);
      }
    };
    auto mma_wait = [&]() {
      if (!mbar_wait(&cbar, cphase)) give_up(p);
      cphase ^= 1;
      tc_fence_after();
    };
    // the next step's tiles, for warps 1, 2 and 5 during the leaf of step k (k = -1:
    // the first diagonal block's leaf, whose next tiles no one updates)
    auto next_tiles = [&](int k) {
      NextTiles nt;
      nt.active = k + 2 < T;
      const int b = (k + 1) & 1;
      nt.X = Xb2 + b * FB * TP;
      nt.C = Cb2 + b * FB * TP;
      nt.gX = tile(k + 2, k + 1);
      nt.gC = tile(k + 2, k + 2);
      nt.k = k;
      return nt;
    };
    // the first diagonal block
    for (int e = threadIdx.x; e < FB * FB; e += FNT) {
      const int r = e / FB, c = e % FB;
      A[r * FP + c] = __ldcg(p.R + (int64_t)r * np + c);
    }
    __syncthreads();
    if (!leaf64(A, M, Lc, rdiag, fl, p, next_tiles(-1))) give_up(p);
    store_diag_m(p, M, 0);
    publish_m(1);
    const uint32_t idesc = make_idesc(2, 128, 64);
    for (int k = 0; k + 1 < T && !aborted(p); ++k) {
      const float* Xb = Xb2 + (k & 1) * FB * TP;
      const float* Cb = Cb2 + (k & 1) * FB * TP;
      // L_{k+1,k} = R_{k+1,k} M_kk^T on the tensor cores: D1[r][c] =
      // sum_t X[r][t] M[c][t], lanes = rows of X (this step's tiles arrived
      // during the previous leaf: its fetching warps waited for their copies before the
      // leaf's closing barrier)
      stage_op(OPA, kAChunk, Xb, TP);
      stage_op(OPB, kBChunk, M, FP);
      fence_proxy_async_smem();
      __syncthreads();
      if (threadIdx.x == 0) {
        tc_fence_after();
        issue_mma_strided(ctb, oah, oal, kAChunk, obh, obl, kBChunk, idesc);
        umma_commit(&cbar);
      }
      mma_wait();
      // warps 0, 1, 4 and 5 read the accumulator: rows 32 (w % 4) .. + 31,
      // columns 32 (w / 4) .. + 31 (a warp reaches the lanes of its quarter)
      const bool reader = (warp & 3) < 2;
      const int rr = 32 * (warp & 3) + (threadIdx.x & 31);
      const int c0 = 32 * (warp >> 2);
      if (reader) {
        // row rr of L (columns c0 .. c0 + 31), published split for the
        // workers and staged as the operand of L L^T
        float v[32];
        tmem_ld32(ctb + (uint32_t)c0 + ((uint32_t)(32 * (warp & 3)) << 16), v);
        float* gh = p.Lh + (int64_t)((k + 1) * FB + rr) * np + (int64_t)k * FB + c0;
        float* gl = p.Ll + (int64_t)((k + 1) * FB + rr) * np + (int64_t)k * FB + c0;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 h, l;
          split_tf32(v[j + 0], h.x, l.x);
          split_tf32(v[j + 1], h.y, l.y);
          split_tf32(v[j + 2], h.z, l.z);
          split_tf32(v[j + 3], h.w, l.w);
          *reinterpret_cast<float4*>(gh + j) = h;
          *reinterpret_cast<float4*>(gl + j) = l;
          const int g = (c0 + j) >> 2;
          const uint32_t so = (g >> 3) * kAChunk + sw128(rr, g & 7);
          *reinterpret_cast<float4*>(OPA + so) = h;
          *reinterpret_cast<float4*>(OPA + 2 * kAChunk + so) = l;
        }
        fence_proxy_async_smem();
        fence_proxy_async_global();  // workers read L_{k+1,k} by TMA
      }
      tc_fence_before();
      __syncthreads();
      if (threadIdx.x == 0) {
        // L L^T: both operands are L (the first 64 rows of OPA)
        tc_fence_after();
        issue_mma_strided(ctb + 64, oah, oal, kAChunk, oah, oal, kAChunk, idesc);
        umma_commit(&cbar);
      } else if (threadIdx.x == 32) {
        __threadfence();
        atomicAdd(&p.pdone[k], 1);
        atomicExch(&p.lcdone[k], 1);
      }
      mma_wait();
      if (reader) {
        float v[32];
        tmem_ld32(ctb + 64 + (uint32_t)c0 + ((uint32_t)(32 * (warp & 3)) << 16), v);
#pragma unroll
        for (int j = 0; j < 32; ++j) A[rr * FP + c0 + j] = Cb[rr * TP + c0 + j] - v[j];
      }
      tc_fence_before();
      __syncthreads();
      if (!leaf64(A, M, Lc, rdiag, fl, p, next_tiles(k))) give_up(p);
      store_diag_m(p, M, k + 1);
      publish_m(k + 2);
    }
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(ctb, 128);
    }
    return;
  }

  // ------------------------------------------------------------------ workers
  uint8_t* SAh = csm;
  uint8_t* SAl = SAh + kRegionBytes;
  uint8_t* SBh = SAl + kRegionBytes;
  uint8_t* SBl = SBh + kRegionBytes;
  float* stg = reinterpret_cast<float*>(SBl + kRegionBytes);  // [kStages][32][128] epilogue staging
  __shared__ uint64_t st_full[2], st_empty[2], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int local_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st_full[b], 1);
      mbar_init(&st_empty[b], 1);
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain, 1);
    local_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
    if (lane == 0) {
      tma_prefetch_desc(&rmap);
      tma_prefetch_desc(&gmap);
      tma_prefetch_desc(&om.lh);
      tma_prefetch_desc(&om.ll);
      tma_prefetch_desc(&om.mth);
      tma_prefetch_desc(&om.mtl);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  const int W = G - 1, slot = cta - 1;
  const uint32_t aH = smem_u32(SAh), aL = smem_u32(SAl), bH = smem_u32(SBh), bL = smem_u32(SBl);
  int tcount = 0;    // tasks of this CTA so far (all steps): drives the barrier phases
  int epi_pass = 0;  // epilogue staging passes (selects the staging buffer)
  bool ok = true;
  for (int k = 0; ok && k < T; ++k) {
    const StepTasks st = step_tasks(np, k);
    const int ntask = st.total();
    if (warp < 4) {
      // ------------------------------------------------ staging and MMA issue
      // the step's inputs: M_kk published, and every trailing and inverse-
      // accumulation tile of the previous step landed (so column block k of R
      // and block row k of G are final, and the reduce-adds of consecutive
      // steps reach each element in order)
      if (threadIdx.x == 0) {
        bool w = wait_ge(p, (const int*)&p.sync[3], k + 1);
        if (w && k > 0) {
          const StepTasks pv = step_tasks(np, k - 1);
          w = wait_ge(p, &p.tdone[k - 1], pv.ntrail) && wait_ge(p, &p.gdone[k - 1], pv.ngupd);
        }
        if (!w) local_abort = 1;
        // operands written by other CTAs' generic stores are read by TMA below
        fence_proxy_async_global();
      }
      named_bar_sync(1, 128);
      bool panels_seen = false, mrows_seen = false;
      int tl = tcount;
      for (int t = slot; t < ntask && !local_abort; t += W, ++tl) {
        const Task x = task_of(np, k, t, st);
        const bool t00 = x.kind == 1 && x.r0 == (int64_t)FB * (k + 1) && x.c0 == (int64_t)FB * (k + 1);
        if (t00 && !panels_seen) {
          // trailing tile (0, 0) reads only L_{k+1,k} and panel tile 0
          if (threadIdx.x == 0) {
            if (!wait_ge(p, &p.lcdone[k], 1) || !wait_ge(p, &p.p0done[k], 1)) local_abort = 1;
            fence_proxy_async_global();
          }
          named_bar_sync(1, 128);
          if (local_abort) break;
        } else if ((x.kind == 1 || x.kind == 3) && !panels_seen) {
          // every panel tile of the step (by the workers, and one by CTA 0)
          if (threadIdx.x == 0) {
            if (!wait_ge(p, &p.pdone[k], st.npan + 1)) local_abort = 1;
            fence_proxy_async_global();
          }
          named_bar_sync(1, 128);
          panels_seen = true;
          if (local_abort) break;
        }
        if (x.kind == 3 && !mrows_seen) {
          // block row k of M
          if (threadIdx.x == 0) {
            if (!wait_ge(p, &p.mrdone[k], st.nmrow)) local_abort = 1;
            fence_proxy_async_global();
          }
          named_bar_sync(1, 128);
          mrows_seen = true;
          if (local_abort) break;
        }
        // The operands go through a ring of two stages, one K chunk (32 of
        // the 64) each: the MMAs of a chunk start once it has landed, and a
        // stage is refilled (for the next task) once its MMAs are done.
        const int64_t kc = (int64_t)FB * k;  // k range of every product: block column k
        const bool by_tma = x.kind == 1 || x.kind == 3;
        if (!by_tma) {
          // kinds 0 and 2 split an fp32 operand while staging it: all four
          // warps write both stages, then thread 0 marks them full
          bool w = true;
          if (tl > 0) w = mbar_wait(&st_empty[0], (tl - 1) & 1) && mbar_wait(&st_empty[1], (tl - 1) & 1);
          if (!w) {
            give_up(p);
            local_abort = 1;
            break;
          }
          if (x.kind == 0) {  // L_ik = R_ik M_kk^T
            stage_fp32(SAh, SAl, p.R, np, x.r0, kc, np);
          } else {  // (M_kk G_kj)[r][c] as D[c][r] = sum_t Gt[c][t] M_kk[r][t]
            stage_fp32(SAh, SAl, p.Gt, np, x.c0, kc, np);
          }
          stage_split(SBh, SBl, p.Mh, p.Ml, np, kc, FB, kc, np);
          cp_async_commit();
          cp_async_wait<0>();
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (threadIdx.x == 0) {
            mbar_arrive(&st_full[0]);
            mbar_arrive(&st_full[1]);
          }
        } else if (threadIdx.x == 0) {
          // kind 1: (L L^T)[c][r], A = L rows c, B = L rows r;
          // kind 3: (L_ik M_kj)[i][c] = sum_t L[i][t] Mt[c][t], A = L rows i,
          // B = Mt rows c.  Rows past the matrix arrive as zeros.
          const bool two = !(x.kind == 1 && x.diag);
          const int32_t ya = (int32_t)(x.kind == 1 ? x.c0 : x.r0);
          const int32_t yb = (int32_t)(x.kind == 1 ? x.r0 : x.c0);
          const CUtensorMap* bhm = x.kind == 1 ? &om.lh : &om.mth;
          const CUtensorMap* blm = x.kind == 1 ? &om.ll : &om.mtl;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            if (tl > 0 && !mbar_wait(&st_empty[ch], (tl - 1) & 1)) {
              give_up(p);
              local_abort = 1;
              break;
            }
            const int32_t xk = (int32_t)(kc + 32 * ch);
            mbar_arrive_expect_tx(&st_full[ch], (two ? 4u : 2u) * kChunkBytes);
            tma_load_2d(SAh + ch * kChunkBytes, &om.lh, &st_full[ch], xk, ya);
            tma_load_2d(SAl + ch * kChunkBytes, &om.ll, &st_full[ch], xk, ya);
            if (two) {
              tma_load_2d(SBh + ch * kChunkBytes, bhm, &st_full[ch], xk, yb);
              tma_load_2d(SBl + ch * kChunkBytes, blm, &st_full[ch], xk, yb);
            }
          }
        }
        if (threadIdx.x == 96) {
          // the MMA issuer: chunk by chunk, as the stages land
          const int buf = tl & 1;
          const int use = tl >> 1;
          bool w = !(use > 0 && !mbar_wait(&acc_empty[buf], (use - 1) & 1));
          const bool same = x.kind == 1 && x.diag;
          const uint32_t idesc = make_idesc(2, 128, (x.kind == 0 || x.kind == 2) ? 64u : 128u);
          const uint32_t d = tbase + (uint32_t)buf * 128;
#pragma unroll
          for (int ch = 0; ch < 2 && w; ++ch) {
            if (!mbar_wait(&st_full[ch], tl & 1)) {
              w = false;
              break;
            }
            tc_fence_after();
            const uint32_t off = ch * kChunkBytes;
            issue_mma_chunk(d, aH + off, aL + off, same ? aH + off : bH + off, same ? aL + off : bL + off, idesc,
                            ch > 0);
            umma_commit(&st_empty[ch]);
          }
          if (w) {
            umma_commit(&acc_full[buf]);
          } else {
            give_up(p);
            local_abort = 1;
          }
        }
      }
    } else {
      // ------------------------------------------------ epilogue (warps 4-7)
      const int quarter = warp & 3;
      const int cl = quarter * 32 + lane;
      int tl = tcount;
      for (int t = slot; t < ntask; t += W, ++tl) {
        const Task x = task_of(np, k, t, st);
        const int buf = tl & 1;
        if (!mbar_wait_sleep(&acc_full[buf], (tl >> 1) & 1)) {
          give_up(p);
          local_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tbase + (uint32_t)buf * 128 + ((uint32_t)(quarter * 32) << 16);
        if (x.kind == 0 || x.kind == 2) {
          // 64 accumulator columns per lane, split and staged in the 128-byte
          // swizzled layout (lane = row of the stored tile), then written by
          // TMA tensor stores:
          //   kind 0  rows of L: Lh/Ll[r][64k .. 64k + 63];
          //   kind 2  rows of M^T: Mth/Mtl[c][64k ..] = -D.  With k odd the
          //           tile's last 64 rows are block k, whose M_kk^T is
          //           already in place: only the first 64 rows are stored.
          const float sg = x.kind == 0 ? 1.f : -1.f;
          uint8_t* sbase = reinterpret_cast<uint8_t*>(stg);  // hi: 2 chunks, then lo: 2 chunks
          if (threadIdx.x == 128) bulk_wait_read<0>();  // earlier bulk copies are done reading stg
          named_bar_sync(2, 128);
#pragma unroll
          for (int n0 = 0; n0 < FB; n0 += 32) {
            float v[32];
            tmem_ld32(taddr + (uint32_t)n0, v);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 h, l;
              split_tf32(sg * v[j + 0], h.x, l.x);
              split_tf32(sg * v[j + 1], h.y, l.y);
              split_tf32(sg * v[j + 2], h.z, l.z);
              split_tf32(sg * v[j + 3], h.w, l.w);
              const int g = (n0 + j) >> 2;
              const uint32_t so = (g >> 3) * kChunkBytes + sw128(cl, g & 7);
              *reinterpret_cast<float4*>(sbase + so) = h;
              *reinterpret_cast<float4*>(sbase + 2 * kChunkBytes + so) = l;
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
          named_bar_sync(2, 128);
          if (threadIdx.x == 128) {
            const int64_t row0 = x.kind == 0 ? x.r0 : x.c0;
            const bool half = x.kind == 2 && row0 + 128 > (int64_t)FB * k;
            const CUtensorMap* mh = x.kind == 0 ? &om.lh : (half ? &om.mth64 : &om.mth);
            const CUtensorMap* ml = x.kind == 0 ? &om.ll : (half ? &om.mtl64 : &om.mtl);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              const int32_t xc = (int32_t)((int64_t)FB * k + 32 * ch);
              tma_store_2d(mh, sbase + ch * kChunkBytes, xc, (int32_t)row0);
              tma_store_2d(ml, sbase + (2 + ch) * kChunkBytes, xc, (int32_t)row0);
            }
            bulk_commit();
            // published once written: other CTAs read these tiles by TMA
            bulk_wait_all();
            fence_proxy_async_global();
            __threadfence();
            atomicAdd(x.kind == 0 ? &p.pdone[k] : &p.mrdone[k], 1);
            if (x.kind == 0 && x.r0 == (int64_t)FB * (k + 2)) atomicExch(&p.p0done[k], 1);
          }
        } else {
          // TMA reduce-add in L2, 32 accumulator columns per pass through one
          // of kStages staging tiles; elements outside the update add zero:
          //   kind 1  R[r][c] -= D[c][r] (lane = column c): above the diagonal,
          //           block (k+1, k+1) and past the matrix excluded;
          //   kind 3  Gt[c][i] += D[i][c] (lane = row i of G): columns from
          //           block k + 1 on and rows past the matrix excluded.
          const int64_t s = (int64_t)FB * (k + 1);
          const int64_t lane_idx = (x.kind == 1 ? x.c0 : x.r0) + cl;
#pragma unroll 1
          for (int pz = 0; pz < 4; ++pz) {
            float v[32];
            tmem_ld32(taddr + (uint32_t)(32 * pz), v);
            const int64_t nb = (x.kind == 1 ? x.r0 : x.c0) + 32 * pz;
            float* sb = stg + (epi_pass % kStages) * (32 * 128);
            if (threadIdx.x == 128) bulk_wait_read<kStages - 1>();  // the reduce that last read sb is done
            named_bar_sync(2, 128);
            // the kept entries of a pass are a range of j, [lo, hi)
            int lo, hi;
            float sg;
            if (x.kind == 1) {
              // r = nb + j < np, c <= r, and not both r and c in block k + 1
              const int64_t c = lane_idx;
              int64_t l = c - nb;
              if (c < s + FB) l = l > s + FB - nb ? l : s + FB - nb;
              lo = (int)(l < 0 ? 0 : (l > 32 ? 32 : l));
              const int64_t h = np - nb;
              hi = (int)(h < 0 ? 0 : (h > 32 ? 32 : h));
              sg = -1.f;
            } else {
              // column c = nb + j < s, row i < np
              const int64_t h = lane_idx < np ? s - nb : 0;
              lo = 0;
              hi = (int)(h < 0 ? 0 : (h > 32 ? 32 : h));
              sg = 1.f;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) sb[j * 128 + cl] = (j >= lo && j < hi) ? sg * v[j] : 0.f;
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            if (threadIdx.x == 128) {
              if (x.kind == 1)
                tma_reduce_add_2d(&rmap, sb, (int32_t)x.c0, (int32_t)nb);
              else
                tma_reduce_add_2d(&gmap, sb, (int32_t)x.r0, (int32_t)nb);
              bulk_commit();
            }
            ++epi_pass;
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
          if (x.kind == 1 && x.r0 == (int64_t)FB * (k + 1) && x.c0 == (int64_t)FB * (k + 1) && threadIdx.x == 128) {
            // trailing tile (0, 0) holds the chain's next two tiles
            bulk_wait_all();
            fence_proxy_async_global();
            __threadfence();
            atomicExch(&p.t0done[k], 1);
          }
        }
      }
    }
    if (threadIdx.x == 128) {
      // this CTA's reduce-adds of the step have landed: count them
      int mine_t = 0, mine_g = 0;
      for (int t = slot; t < ntask; t += W) {
        const int kd = task_of(np, k, t, st).kind;
        mine_t += kd == 1;
        mine_g += kd == 3;
      }
      bulk_wait_all();
      fence_proxy_async_global();
      __threadfence();
      if (mine_t) atomicAdd(&p.tdone[k], mine_t);
      if (mine_g) atomicAdd(&p.gdone[k], mine_g);
    }
    // both groups walked the same task list
    for (int t = slot; t < ntask; t += W) ++tcount;
    ok = !local_abort && !aborted(p);
  }
  if (threadIdx.x == 128) bulk_wait_all();
  __syncthreads();
  if (local_abort || aborted(p)) {
    // let MMAs already issued (by thread 96) finish before the tensor memory
    // goes away; copies in flight land on barriers that are never reused
    if (threadIdx.x == 96) {
      umma_commit(&drain);
      mbar_wait(&drain, 0);
    }
    __syncthreads();
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

size_t chain_smem_bytes() { return kChainOpOffset + kChainOpABytes + kChainOpBBytes; }

}  // namespace

size_t chol_smem_bytes() { return 1024 + std::max<size_t>(kWorkerSmem, chain_smem_bytes()); }

size_t chol_sync_bytes(int64_t np_) { return sizeof(int) * (size_t)(7 * (np_ / FB) + 4); }

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
}  // namespace

bool encode_f32_2d(CUtensorMap* m, const float* base, int64_t cols, int64_t rows, int64_t ld, uint32_t box_x,
                   uint32_t box_y, bool swizzle128) {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return (EncodeTiledFn)f;
  }();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)(ld * 4)};
  cuuint32_t box[2] = {box_x, box_y};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
// An np x np fp32 row-major matrix as a 2-D tensor: 128-column x 32-row boxes
// without swizzle for the reduce-add epilogues (R, G^T), 32-column x 128-row
// boxes with 128-byte swizzle for the operand loads (L, M^T; the tensor
// core's K-major layout).
bool make_r_map(CUtensorMap* m, float* R, int64_t np_, uint32_t box_x = 128, uint32_t box_y = 32,
                bool swz = false) {
  return encode_f32_2d(m, R, np_, np_, np_, box_x, box_y, swz);
}
}  // namespace

cudaError_t chol_factor(float* R, int64_t np_, float* Lh, float* Ll, float* Mh, float* Ml, float* Mth, float* Mtl,
                        float* Gt, unsigned* sync, uint32_t* status, int sms, cudaStream_t st) {
  const size_t smem = chol_smem_bytes();
  cudaError_t e = ensure_smem_limit((const void*)chol_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chol_kernel, FNT, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int T = (int)(np_ / FB);
  e = cudaMemsetAsync(sync, 0, chol_sync_bytes(np_), st);
  if (e != cudaSuccess) return e;
  // workers: enough for the first step's tasks (at most one CTA per SM)
  // workers: enough for the busiest step's tasks (at most one CTA per SM)
  int most = 1;
  for (int k = 0; k < T; ++k) most = std::max(most, step_tasks(np_, k).total());
  const int grid = std::max(2, std::min(sms, 1 + most));
  CholParams p;
  p.R = R;
  p.np_ = np_;
  p.T = T;
  p.Lh = Lh;
  p.Ll = Ll;
  p.Mh = Mh;
  p.Ml = Ml;
  p.Mth = Mth;
  p.Mtl = Mtl;
  p.sync = sync;
  p.pdone = (int*)(sync + 4);
  p.tdone = p.pdone + T;
  p.t0done = p.tdone + T;
  p.mrdone = p.t0done + T;
  p.gdone = p.mrdone + T;
  p.p0done = p.gdone + T;
  p.lcdone = p.p0done + T;
  p.Gt = Gt;
  p.status = status;
  CUtensorMap rmap, gmap;
  if (!make_r_map(&rmap, R, np_) || !make_r_map(&gmap, Gt, np_)) return cudaErrorInvalidValue;
  OpMaps om;
  const bool sw = true;
  if (!make_r_map(&om.lh, Lh, np_, 32, 128, sw) || !make_r_map(&om.ll, Ll, np_, 32, 128, sw) ||
      !make_r_map(&om.mth, Mth, np_, 32, 128, sw) || !make_r_map(&om.mtl, Mtl, np_, 32, 128, sw) ||
      !make_r_map(&om.mth64, Mth, np_, 32, 64, sw) || !make_r_map(&om.mtl64, Mtl, np_, 32, 64, sw))
    return cudaErrorInvalidValue;
  void* args[] = {&rmap, &gmap, &om, &p};
  e = cudaLaunchCooperativeKernel((const void*)chol_kernel, dim3(grid), dim3(FNT), args, smem, st);
  note_launch();
  return e;
}

}  // namespace gptq
