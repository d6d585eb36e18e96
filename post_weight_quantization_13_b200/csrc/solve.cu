// The column sweep with error compensation and its lazy updates, in one
// cooperative launch ("gptq" glossary page, Algorithm (2): quantize a column,
// then compensate the weights not yet quantized; Key innovation: lazy batch
// updates), with group parameters taken at each group's first column ("gptq"
// agent-skill page, Group-wise quantization).
//
// Rows of W never interact: a row's sweep reads only U (shared, read-only)
// and that row's own weights.  The launch splits W into slabs of 128 rows
// and 128-column blocks and runs two kinds of CTA side by side:
//
//   chain CTAs   own slabs.  For block k of a slab the block's columns go
//                through the sweep in four 32-column sub-blocks.  Inside a
//                sub-block each of 128 lanes owns one row and updates the
//                sub-block's later columns at once (fp32 FMA, U from shared
//                memory).  The sub-block's errors then update the block's
//                later columns on the tensor cores: 3xTF32 tcgen05 MMAs into
//                a tensor-memory accumulator D, so the next sub-block reads
//                W_block + D.  The sub-block's -E, split into tf32 hi and the
//                exact remainder, is the MMA's operand and goes to global
//                memory by TMA; once all of block k's -E has landed the slab
//                publishes it.
//   worker CTAs  apply a finished block's errors to the later blocks, one
//                column block of two slabs per task: W[slab, c] += (-E[slab,
//                k]) U[k, c] (3xTF32, 128 x 256 x 128), added in L2 by TMA
//                reduce-adds.  The tasks are taken in order of k, nearest
//                column block first, and each tile receives its
//                contributions in order of k, so the result does not depend
//                on timing.
//
// A chain starts block k of a slab once all k earlier contributions have
// landed in that block; the slabs of one chain alternate, so the tile tasks a
// slab waits for run while the chain sweeps its other slabs.  Counters in
// global memory carry every dependency (release: wait for the bulk copies,
// proxy fence, __threadfence, atomic store; acquire: bounded spin,
// __threadfence, proxy fence).  Every wait is bounded by %globaltimer; a wait
// that gives up raises ST_TIMEOUT and sets a launch-wide abort flag, and every
// CTA then unwinds.
#include <algorithm>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {
namespace {

constexpr int QB = 128;                        // block width (columns) and slab height (rows)
constexpr int SB = 32;                         // sub-block width
constexpr int QNT = 256;                       // threads per CTA
constexpr uint32_t kQChunk = 128 * 128;        // 128 rows x 32 fp32, 128-byte swizzled K-major
constexpr uint32_t kUdFloats = SB * SB + SB;   // a sub-block's U (row j: U[j][j']) and 1 / U_jj
constexpr uint32_t kUdBytes = kUdFloats * 4;

// chain CTA shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kCWb = 0;                   // 4 chunks: W of the slab's block
constexpr uint32_t kCUb = kCWb + 4 * kQChunk;  // 2 slots x (hi, lo): U rows of the block, one K chunk
constexpr uint32_t kCUn = kCUb + 4 * kQChunk;  // (hi, lo): U rows of the next block, the same K chunk
constexpr uint32_t kCA = kCUn + 2 * kQChunk;   // (hi, lo): -E of the sub-block
constexpr uint32_t kCX = kCA + 2 * kQChunk;    // each row's values at the sub-block's start
constexpr uint32_t kCUd = kCX + kQChunk;       // 2 slots of kUdBytes
constexpr uint32_t kChainSmem = kCUd + 2 * kUdBytes;
// worker CTA
constexpr int kWSlots = 2;                     // operand ring: K chunks of (U hi, U lo, E hi, E lo)
constexpr uint32_t kWRing = 0;
constexpr uint32_t kWStageBytes = 6 * kQChunk; // U 128 rows + E 256 rows, hi and lo
constexpr int kWStages = 2;                    // epilogue staging tiles, 32 rows x 128 columns fp32
constexpr uint32_t kWStg = kWRing + kWSlots * kWStageBytes;
constexpr uint32_t kWorkerSmem = kWStg + kWStages * 32 * 128 * 4;
constexpr uint32_t kSolveSmem = 1024 + (kChainSmem > kWorkerSmem ? kChainSmem : kWorkerSmem);
static_assert(kSolveSmem <= 232448, "shared memory per CTA");

struct SolveParams {
  float* Wp;        // out x np, row stride np: W in processing order, updated in place
  int64_t np_, out, in;
  const float* Ud;  // per 32-column sub-block: U[j][j'] (32 x 32, row-major) then 1 / U_jj
  int T;            // column blocks (np / 128)
  int nslab;        // row slabs (ceil(out / 128))
  int nchain;       // chain CTAs (CTAs 0 .. nchain - 1); slab i belongs to chain i % nchain
  int chain_next;   // the chains apply each block's errors to the slab's next block themselves
  int maxq, sym, gs, ngroups;
  float* scales;
  int32_t* zeros;
  uint8_t* codes_p;  // out x np codes in processing order
  float* loss;       // per row, may be null
  int* sdone;        // [nslab] blocks of the slab whose -E has landed
  int* cnt;          // [nslab][T] contributions landed in each block of each slab
  unsigned* abort_flag;
  uint32_t* status;
};

// Tensor maps, all fp32 2-D row-major: the chain's W loads (32-column x
// 128-row boxes, 128-byte swizzle), the workers' reduce-adds into W (128 x 32,
// no swizzle), split U^T (Uh/Ul[c][j] = U[j][c]) and split -E (32 x 128, 128-byte
// swizzle: the tensor core's K-major operand layout; eh2/el2 with 256-row
// boxes, a pair of slabs).
struct SolveMaps {
  CUtensorMap wld, wred, uh, ul, eh, el, eh2, el2;
};

__device__ __forceinline__ bool q_aborted(const SolveParams& p) { return *(volatile unsigned*)p.abort_flag != 0; }

__device__ __forceinline__ void q_give_up(const SolveParams& p) {
  raise_status(p.status, ST_TIMEOUT);
  atomicExch(p.abort_flag, 1u);
}

// One thread: wait until *f >= target, bounded; false once any CTA gave up.
__device__ bool q_wait_ge(const SolveParams& p, const int* f, int target) {
  volatile const int* vf = f;
  if (vf[0] < target) {
    const uint64_t t0 = globaltimer();
    for (;;) {
      // both loads are in flight together: one L2 round trip a poll
      const int v = vf[0];
      const bool ab = q_aborted(p);
      if (v >= target) break;
      if (ab) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        q_give_up(p);
        return false;
      }
      __nanosleep(64);
    }
  }
  __threadfence();
  return true;
}

// Bounded mbarrier phase wait that also stops once any CTA gave up.
__device__ bool q_mbar_wait(const SolveParams& p, uint64_t* bar, uint32_t parity, bool sleep = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (sleep) __nanosleep(64);
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63) == 0) {
      if (q_aborted(p)) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        q_give_up(p);
        return false;
      }
    }
  }
}

// Scale and zero of a group from its current values ("gptq" agent-skill
// page, Group-wise quantization): asymmetric over [min(0, lo), max(0, hi)]
// (both zero: [-1, 1]), symmetric over max |w| (zero: 1).
__device__ __forceinline__ void group_params(float lo, float hi, float amax, int sym, float fmaxq, float& s,
                                             float& z) {
  if (sym) {
    const float a = amax == 0.f ? 1.f : amax;
    s = __fdiv_rn(2.f * a, fmaxq);
    z = (fmaxq + 1.f) * 0.5f;
  } else {
    lo = fminf(lo, 0.f);
    hi = fmaxf(hi, 0.f);
    if (lo == 0.f && hi == 0.f) {
      lo = -1.f;
      hi = 1.f;
    }
    s = __fdiv_rn(hi - lo, fmaxq);
    z = rintf(__fdiv_rn(-lo, s));
  }
}

// rint(x / s) with x / s an IEEE division, from the product with the
// rounded reciprocal: the product is within 3 units in the last place of the
// quotient, so its rounding gives the same integer unless the quotient lies
// within a few units of a half-integer; there (and for non-finite products)
// the exact quotient is rounded instead.
__device__ __forceinline__ float round_div(float x, float s, float inv_s) {
  const float y = x * inv_s;
  const float fr = y - floorf(y);
  if (fabsf(fr - 0.5f) > fmaf(fabsf(y), 0x1p-20f, 0x1p-24f)) return rintf(y);
  return rintf(__fdiv_rn(x, s));
}

__device__ __forceinline__ void minmax(float v, float& lo, float& hi, float& am) {
  lo = fminf(lo, v);
  hi = fmaxf(hi, v);
  am = fmaxf(am, fabsf(v));
}

// Row r's 32 values of a 128-byte swizzled chunk (8 conflict-free vector loads
// per quarter warp: the rows of 8 consecutive lanes hit 8 different units).
__device__ __forceinline__ void load_row(const uint8_t* chunk, int r, float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 t = *reinterpret_cast<const float4*>(chunk + sw128(r, u));
    v[4 * u + 0] = t.x;
    v[4 * u + 1] = t.y;
    v[4 * u + 2] = t.z;
    v[4 * u + 3] = t.w;
  }
}

__device__ __forceinline__ void store_row(uint8_t* chunk, int r, const float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<float4*>(chunk + sw128(r, u)) = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
}

__device__ __forceinline__ void add_tmem(uint32_t taddr, float (&v)[32]) {
  float d[32];
  tmem_ld32(taddr, d);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] += d[i];
}

// A 16-byte shared-memory load the compiler keeps where it is written (it
// would otherwise hoist the U rows of many columns at once and run out of
// registers).
__device__ __forceinline__ float4 lds128(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ float lds32(const float* p) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ float elem(const float4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
// Zero, in a way the compiler cannot see through: an address plus
// after(v) is only formed once v is, which keeps a load behind v.
__device__ __forceinline__ uint32_t after(float v) {
  uint32_t z;
  asm volatile("and.b32 %0, %1, 0;" : "=r"(z) : "r"(__float_as_uint(v)));
  return z;
}

// One row's 32 columns of a sub-block (x: their current values; ud: the
// sub-block's U and 1 / U_jj).  For each column: the group's scale and zero
// at a group start inside the sub-block, the code clamp(rint(x / s) + z, 0,
// maxq), the error e = (x - s (code - z)) / U_jj (zero past the layer's
// columns), and x[j'] -= e U[j][j'] for the sub-block's later columns.  On
// return x holds -e, cw the codes (one byte each).
//
// kFast: x / s from the divide-free quotient, with no branch in the column
// loop; false if any quotient was outside its range (the results are then to
// be discarded).  U's row j + 1 is read while column j is quantized, so the
// loads never wait in front of the column's updates.  Otherwise x / s from
// round_div.
//
// kRagged: some of the 32 columns lie past the layer's (the last block of a
// layer whose width is not a multiple of 128); their errors are forced to
// zero.  A per-column bound check costs a quarter of the loop, so the other
// sub-blocks run without it.
template <int GSB, bool kFast, bool kRagged>
__device__ __forceinline__ bool sweep32(float (&x)[32], const float* ud, int64_t c0, const SolveParams& p,
                                        int64_t row, bool live, float fmaxq, float& s_, float& z_, float& inv_s,
                                        float& lsum, uint32_t (&cw)[8]) {
  const int nvalid = kRagged ? (int)(p.in - c0 < SB ? p.in - c0 : SB) : SB;
  bool in_range = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) cw[i] = 0u;
  float4 ucur[8], unext[8];
  float rcur = 0.f, rnext = 0.f;
  if (kFast) {
#pragma unroll
    for (int a = 0; a < 8; ++a) ucur[a] = lds128(ud + 4 * a);
    rcur = lds32(ud + SB * SB);
  }
#pragma unroll
  for (int j = 0; j < SB; ++j) {
    if (kFast && j + 1 < SB) {
      // U's row j + 1, once column j is final (not earlier: registers)
      const float* un = ud + after(x[j]);
#pragma unroll
      for (int a = (j + 2) >> 2; a < 8; ++a) unext[a] = lds128(un + (j + 1) * SB + 4 * a);
      rnext = lds32(un + SB * SB + j + 1);
    }
    if (GSB <= SB && j % GSB == 0 && (!kRagged || j < nvalid)) {
      float lo = INFINITY, hi = -INFINITY, am = 0.f;
#pragma unroll
      for (int i = j; i < j + (GSB <= SB ? GSB : 1); ++i) minmax(x[i], lo, hi, am);
      group_params(lo, hi, am, p.sym, fmaxq, s_, z_);
      inv_s = __frcp_rn(s_);
      if (live) {
        p.scales[row * p.ngroups + (c0 + j) / GSB] = s_;
        p.zeros[row * p.ngroups + (c0 + j) / GSB] = (int32_t)z_;
      }
    }
    const float xv = x[j];
    float qf;
    if (kFast) {
      qf = rintf(quot_rn(xv, s_, inv_s)) + z_;
      in_range &= quot_in_range(xv, s_);
    } else {
      qf = round_div(xv, s_, inv_s) + z_;
    }
    qf = fminf(fmaxf(qf, 0.f), fmaxq);
    const float deq = s_ * (qf - z_);
    float e = (xv - deq) * (kFast ? rcur : ud[SB * SB + j]);
    if (kRagged) e = j < nvalid ? e : 0.f;
    lsum = fmaf(e, e, lsum);
    cw[j >> 2] |= (uint32_t)qf << (8 * (j & 3));
    x[j] = -e;
    // the sub-block's later columns: x[j'] -= e U[j][j'], the next one first
    if (kFast) {
#pragma unroll
      for (int jp = j + 1; jp < SB; ++jp) x[jp] = fmaf(-e, elem(ucur[jp >> 2], jp & 3), x[jp]);
#pragma unroll
      for (int a = 0; a < 8; ++a) ucur[a] = unext[a];
      rcur = rnext;
    } else {
      const float* ur = ud + j * SB;
#pragma unroll
      for (int a = (j + 1) >> 2; a < 8; ++a) {
        const float4 u = *reinterpret_cast<const float4*>(ur + 4 * a);
        if (4 * a + 0 > j) x[4 * a + 0] = fmaf(-e, u.x, x[4 * a + 0]);
        if (4 * a + 1 > j) x[4 * a + 1] = fmaf(-e, u.y, x[4 * a + 1]);
        if (4 * a + 2 > j) x[4 * a + 2] = fmaf(-e, u.z, x[4 * a + 2]);
        if (4 * a + 3 > j) x[4 * a + 3] = fmaf(-e, u.w, x[4 * a + 3]);
      }
    }
  }
  return in_range;
}

// A row's 32 codes of a sub-block (one byte each, 16-byte aligned).
__device__ __forceinline__ void store_codes(const SolveParams& p, int64_t row, int64_t c0, bool live,
                                            const uint32_t (&cw)[8]) {
  if (!live) return;
  uint4* dst = reinterpret_cast<uint4*>(p.codes_p + row * p.np_ + c0);
  dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
}

struct RowState {
  float s, z, inv_s, lsum;
};

// The sub-block again with round_div, from the row's values at its start
// (in Xs, where the results, -e, go back too).  Kept out of line: it runs
// only for quotients outside quot_in_range, and inlined it would take
// registers from the main loop.
template <int GSB>
__device__ __noinline__ RowState replay32(uint8_t* Xs, int rl, const float* ud, int64_t c0, const SolveParams& p,
                                          int64_t row, bool live, float fmaxq, RowState st) {
  float x[32];
  uint32_t cw[8];
  load_row(Xs, rl, x);
  sweep32<GSB, false, true>(x, ud, c0, p, row, live, fmaxq, st.s, st.z, st.inv_s, st.lsum, cw);
  store_row(Xs, rl, x);
  store_codes(p, row, c0, live, cw);
  return st;
}

// ------------------------------------------------------------------ chain CTA
// Threads 0-127: one row each (warp w reads tensor-memory lanes 32w..32w+31,
// its own quarter).  Thread 128: loads, MMAs, the -E stores and the
// publication.  Threads 129-255 have nothing to do.
//
// With p.chain_next (at most two slabs per chain) the chain also applies a
// block's errors to the slab's next block: each slab keeps two 128-column
// accumulators, D_cur for the block being swept and D_next for the one after
// it, and every sub-block's MMAs add to both.  Block k + 1 then starts from
// W (with the workers' contributions of blocks up to k - 1) plus D_next, and
// the workers take only the blocks two and more ahead.  Without it the
// workers take every later block and the chain's one accumulator starts
// afresh with each block.
template <int GSB>
__device__ __forceinline__ void chain_cta(const SolveMaps& mp, const SolveParams& p, uint8_t* sm) {
  uint8_t* Wb = sm + kCWb;
  uint8_t* Ub = sm + kCUb;
  uint8_t* Un = sm + kCUn;
  uint8_t* Ab = sm + kCA;
  uint8_t* Xs = sm + kCX;
  float* Udb = reinterpret_cast<float*>(sm + kCUd);
  __shared__ uint64_t wb_full[4], wb_empty[4], ub_full[2], un_full, ud_full[2], ud_empty[2];
  __shared__ uint64_t a_full, a_empty, mma_next, mma_done, drain;
  __shared__ uint32_t tslot;
  const int warp = threadIdx.x >> 5;
  const int64_t np = p.np_;
  const int T = p.T;
  const bool cn = p.chain_next != 0;
  // items: (block k, slab) for k = 0 .. T - 1, this chain's slabs in turn
  const int spc = (p.nslab - (int)blockIdx.x + p.nchain - 1) / p.nchain;
  const int nitems = T * spc;
  const uint32_t tcols = cn ? (spc > 1 ? 512u : 256u) : 128u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&wb_full[i], 1);
      mbar_init(&wb_empty[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ub_full[i], 1);
      mbar_init(&ud_full[i], 1);
      mbar_init(&ud_empty[i], 128);
    }
    mbar_init(&un_full, 1);
    mbar_init(&a_full, 128);
    mbar_init(&a_empty, 1);
    mbar_init(&mma_next, 1);
    mbar_init(&mma_done, 1);
    mbar_init(&drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tslot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  auto item_k = [&](int it) { return it / spc; };
  auto item_slab = [&](int it) { return (int)blockIdx.x + (it % spc) * p.nchain; };
  // accumulator of item it's block (cur = 0) or of the block after it (cur = 1)
  auto acc = [&](int it, int nxt) -> uint32_t {
    return cn ? tbase + 256u * (uint32_t)(it % spc) + 128u * (uint32_t)((item_k(it) + nxt) & 1) : tbase;
  };
  // contributions to a slab's block k the workers make (the rest come from D)
  auto worker_count = [&](int k) { return cn ? (k > 0 ? k - 1 : 0) : k; };
  // sub-block g of the launch's sequence has a next-block product
  auto has_next = [&](int g) { return cn && g < 4 * nitems && item_k(g >> 2) + 1 < T; };
  bool ok = true;

  if (threadIdx.x == 128) {
    // ------------------------------------------------------------ control
    tma_prefetch_desc(&mp.wld);
    tma_prefetch_desc(&mp.uh);
    tma_prefetch_desc(&mp.ul);
    tma_prefetch_desc(&mp.eh);
    tma_prefetch_desc(&mp.el);
    // U rows of block k, K chunk s (use u = 3 it + s: the sub-blocks with
    // products inside the block), into slot u & 1
    auto load_ub = [&](int u) {
      const int it = u / 3, s = u % 3;
      const int k = item_k(it);
      uint8_t* dst = Ub + 2 * (u & 1) * kQChunk;
      mbar_arrive_expect_tx(&ub_full[u & 1], 2 * kQChunk);
      tma_load_2d(dst, &mp.uh, &ub_full[u & 1], QB * k + SB * s, QB * k);
      tma_load_2d(dst + kQChunk, &mp.ul, &ub_full[u & 1], QB * k + SB * s, QB * k);
    };
    // U rows of block k + 1, K chunk s of block k, for sub-block g
    auto load_un = [&](int g) {
      const int it = g >> 2, s = g & 3;
      const int k = item_k(it);
      mbar_arrive_expect_tx(&un_full, 2 * kQChunk);
      tma_load_2d(Un, &mp.uh, &un_full, QB * k + SB * s, QB * (k + 1));
      tma_load_2d(Un + kQChunk, &mp.ul, &un_full, QB * k + SB * s, QB * (k + 1));
    };
    // U of sub-block g (4 per item) into slot g & 1
    auto load_ud = [&](int g) {
      const int it = g >> 2, s = g & 3;
      const int k = item_k(it);
      mbar_arrive_expect_tx(&ud_full[g & 1], kUdBytes);
      bulk_load(Udb + (g & 1) * kUdFloats, p.Ud + (int64_t)(4 * k + s) * kUdFloats, kUdBytes, &ud_full[g & 1]);
    };
    // chunk c of item it's W, once the workers' contributions have landed
    // (wait: block until they have; else give up at once if they have not)
    auto wb_ready = [&](int it, bool wait) {
      const int* f = &p.cnt[(int64_t)item_slab(it) * T + item_k(it)];
      const int need = worker_count(item_k(it));
      if (wait) return q_wait_ge(p, f, need);
      if (*(volatile const int*)f < need) return false;
      __threadfence();
      return true;
    };
    auto load_wb = [&](int it, int c) {
      const int k = item_k(it), slab = item_slab(it);
      mbar_arrive_expect_tx(&wb_full[c], kQChunk);
      tma_load_2d(Wb + c * kQChunk, &mp.wld, &wb_full[c], QB * k + SB * c, QB * slab);
    };
    load_ud(0);
    if (4 * nitems > 1) load_ud(1);
    load_ub(0);
    if (3 * nitems > 1) load_ub(1);
    if (has_next(0)) load_un(0);
    int un_used = 0;
    ok = wb_ready(0, true);
    if (ok) {
      fence_proxy_async_global();
      for (int c = 0; c < 4; ++c) load_wb(0, c);
    }
    const uint32_t ah = smem_u32(Ab), al = ah + kQChunk;
    for (int it = 0; ok && it < nitems; ++it) {
      const int k = item_k(it), slab = item_slab(it);
      const uint32_t dcur = acc(it, 0), dnext = acc(it, 1);
      // in-block products add to what D_cur holds unless it starts afresh
      const bool fresh = !(cn && k > 0);
      int wb_next = 0;  // chunks of item it + 1's W already requested
      for (int s = 0; s < 4; ++s) {
        const int g = 4 * it + s;
        // item it + 1's W, chunk by chunk as the rows take this item's chunk
        // (they do at the start of sub-block s), once the next item's earlier
        // contributions are in: then the chunk lands during this sub-block
        if (it + 1 < nitems && wb_next <= s && wb_ready(it + 1, false)) {
          fence_proxy_async_global();
          for (; wb_next <= s; ++wb_next) {
            if (!q_mbar_wait(p, &wb_empty[wb_next], it & 1)) {
              ok = false;
              break;
            }
            load_wb(it + 1, wb_next);
          }
          if (!ok) break;
        }
        if (!q_mbar_wait(p, &a_full, g & 1)) {
          ok = false;
          break;
        }
        if (s < 3) {
          const int u = 3 * it + s;
          if (!q_mbar_wait(p, &ub_full[u & 1], (u >> 1) & 1)) {
            ok = false;
            break;
          }
        }
        const bool nx = has_next(g);
        if (nx) {
          if (!q_mbar_wait(p, &un_full, un_used & 1)) {
            ok = false;
            break;
          }
          ++un_used;
        }
        tc_fence_after();
        // D_cur[r][c] += sum_j A[r][j] U[j][c] for the block's columns after
        // this sub-block (first the next sub-block's 32, which the rows wait
        // for, then the rest), and D_next for all of the next block
        const bool accum = s > 0 || !fresh;
        if (s < 3) {
          const int u = 3 * it + s;
          const uint32_t bh = smem_u32(Ub) + 2 * (u & 1) * kQChunk, bl = bh + kQChunk;
          const uint32_t c1 = SB * (s + 1), c2 = SB * (s + 2);
          issue_mma_chunk(dcur + c1, ah, al, bh + c1 * 128, bl + c1 * 128, make_idesc(2, 128, SB), accum);
          umma_commit(&mma_next);
          if (c2 < QB)
            issue_mma_chunk(dcur + c2, ah, al, bh + c2 * 128, bl + c2 * 128, make_idesc(2, 128, QB - c2), accum);
        } else {
          umma_commit(&mma_next);
        }
        if (nx) {
          const uint32_t nh = smem_u32(Un);
          issue_mma_chunk(dnext, ah, al, nh, nh + kQChunk, make_idesc(2, 128, QB), s > 0);
        }
        umma_commit(&mma_done);
        // the sub-block's -E (hi, lo) for the workers
        tma_store_2d(&mp.eh, Ab, QB * k + SB * s, QB * slab);
        tma_store_2d(&mp.el, Ab + kQChunk, QB * k + SB * s, QB * slab);
        bulk_commit();
        if (!q_mbar_wait(p, &mma_done, g & 1)) {
          ok = false;
          break;
        }
        if (s < 3 && 3 * it + s + 2 < 3 * nitems) load_ub(3 * it + s + 2);
        // (the items without a next block are the last ones of the launch)
        if (has_next(g + 1)) load_un(g + 1);
        bulk_wait_read<0>();
        mbar_arrive(&a_empty);
        if (g + 2 < 4 * nitems) {
          if (!q_mbar_wait(p, &ud_empty[g & 1], (g >> 1) & 1)) {
            ok = false;
            break;
          }
          load_ud(g + 2);
        }
      }
      if (!ok) break;
      // block k of the slab: its -E has landed
      bulk_wait_all();
      fence_proxy_async_global();
      __threadfence();
      atomicExch(&p.sdone[slab], k + 1);
      if (it + 1 < nitems && wb_next < 4) {
        if (!wb_ready(it + 1, true)) {
          ok = false;
          break;
        }
        fence_proxy_async_global();
        for (; wb_next < 4; ++wb_next) {
          if (!q_mbar_wait(p, &wb_empty[wb_next], it & 1)) {
            ok = false;
            break;
          }
          load_wb(it + 1, wb_next);
        }
      }
    }
    if (!ok) q_give_up(p);
  } else if (threadIdx.x < 128) {
    // ------------------------------------------------------------ the rows
    const int rl = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float fmaxq = (float)p.maxq;
    for (int it = 0; ok && it < nitems; ++it) {
      const int k = item_k(it), slab = item_slab(it);
      const int64_t row = (int64_t)slab * QB + rl;
      const bool live = row < p.out;
      const int64_t kB = (int64_t)QB * k;
      const uint32_t dcur = acc(it, 0) + lane_off;
      const bool dprev = cn && k > 0;  // D_cur already holds the previous block's product
      float s_ = 1.f, z_ = 0.f, lsum = 0.f;
      const bool gstart0 = GSB == QB && (p.gs == -1 ? k == 0 : kB % p.gs == 0);
      if (GSB == QB && !gstart0 && live) {
        // a group that started in an earlier block keeps its scale and zero
        const int64_t gi = p.gs == -1 ? 0 : kB / p.gs;
        s_ = p.scales[row * p.ngroups + gi];
        z_ = (float)p.zeros[row * p.ngroups + gi];
      }
      float inv_s = __frcp_rn(s_);
#pragma unroll 1
      for (int s = 0; s < 4; ++s) {
        const int g = 4 * it + s;
        const int64_t c0 = kB + SB * s;  // first column of the sub-block
        float x[32];
        if (!q_mbar_wait(p, &wb_full[s], it & 1)) {
          ok = false;
          break;
        }
        // every product into this sub-block's columns has completed: the
        // previous sub-block's (s > 0) or all of the previous item's (s = 0)
        if (g > 0 && !q_mbar_wait(p, s > 0 ? &mma_next : &mma_done, (g - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        load_row(Wb + s * kQChunk, rl, x);
        if (s > 0 || dprev) add_tmem(dcur + SB * s, x);
        mbar_arrive(&wb_empty[s]);
        // group starts whose group reaches past this sub-block
        if (GSB == 64 && (s & 1) == 0 && c0 < p.in) {
          if (!q_mbar_wait(p, &wb_full[s + 1], it & 1) || (s > 0 && !q_mbar_wait(p, &mma_done, (g - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          float y[32];
          load_row(Wb + (s + 1) * kQChunk, rl, y);
          if (s > 0 || dprev) add_tmem(dcur + SB * (s + 1), y);
          float lo = INFINITY, hi = -INFINITY, am = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            minmax(x[i], lo, hi, am);
            minmax(y[i], lo, hi, am);
          }
          group_params(lo, hi, am, p.sym, fmaxq, s_, z_);
          inv_s = __frcp_rn(s_);
          if (live) {
            p.scales[row * p.ngroups + c0 / 64] = s_;
            p.zeros[row * p.ngroups + c0 / 64] = (int32_t)z_;
          }
        }
        if (GSB == QB && s == 0 && gstart0) {
          // the whole block as it stands, and the group's columns past it:
          // those need every earlier block's contribution, as this block has
          float lo = INFINITY, hi = -INFINITY, am = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) minmax(x[i], lo, hi, am);
          for (int c = 1; c < 4 && ok; ++c) {
            if (!q_mbar_wait(p, &wb_full[c], it & 1)) {
              ok = false;
              break;
            }
            float y[32];
            load_row(Wb + c * kQChunk, rl, y);
            if (dprev) add_tmem(dcur + SB * c, y);
#pragma unroll
            for (int i = 0; i < 32; ++i) minmax(y[i], lo, hi, am);
          }
          if (!ok) break;
          const int64_t gend = p.gs == -1 ? p.in : std::min<int64_t>(p.in, kB + p.gs);
          if (gend > kB + QB) {
            const int kl = (int)((gend - 1) / QB);
            for (int kb = k + 1; kb <= kl && ok; ++kb) ok = q_wait_ge(p, &p.cnt[(int64_t)slab * T + kb], k);
            if (!ok) break;
            if (live) {
              const float* src = p.Wp + row * np;
              for (int64_t c = kB + QB; c < gend; ++c) minmax(__ldcg(src + c), lo, hi, am);
            }
          }
          group_params(lo, hi, am, p.sym, fmaxq, s_, z_);
          inv_s = __frcp_rn(s_);
          if (live) {
            const int64_t gi = p.gs == -1 ? 0 : kB / p.gs;
            p.scales[row * p.ngroups + gi] = s_;
            p.zeros[row * p.ngroups + gi] = (int32_t)z_;
          }
        }
        if (!q_mbar_wait(p, &ud_full[g & 1], (g >> 1) & 1)) {
          ok = false;
          break;
        }
        const float* ud = Udb + (g & 1) * kUdFloats;
        uint32_t cw[8];
        {
          // the sub-block's columns with the divide-free quotient; a row
          // that met a quotient outside its range replays them with the
          // divide (its values at the sub-block's start wait in Xs for that)
          store_row(Xs, rl, x);
          RowState st{s_, z_, inv_s, lsum};
          const bool fast = c0 + SB <= p.in
                                ? sweep32<GSB, true, false>(x, ud, c0, p, row, live, fmaxq, s_, z_, inv_s, lsum, cw)
                                : sweep32<GSB, true, true>(x, ud, c0, p, row, live, fmaxq, s_, z_, inv_s, lsum, cw);
          if (fast) {
            store_codes(p, row, c0, live, cw);
          } else {
            st = replay32<GSB>(Xs, rl, ud, c0, p, row, live, fmaxq, st);
            s_ = st.s, z_ = st.z, inv_s = st.inv_s, lsum = st.lsum;
            load_row(Xs, rl, x);
          }
        }
        mbar_arrive(&ud_empty[g & 1]);
        // -E of the sub-block, split, as the MMA operand (row rl, K-major)
        if (g > 0 && !q_mbar_wait(p, &a_empty, (g - 1) & 1)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float4 h, l;
          split_tf32(x[4 * u + 0], h.x, l.x);
          split_tf32(x[4 * u + 1], h.y, l.y);
          split_tf32(x[4 * u + 2], h.z, l.z);
          split_tf32(x[4 * u + 3], h.w, l.w);
          *reinterpret_cast<float4*>(Ab + sw128(rl, u)) = h;
          *reinterpret_cast<float4*>(Ab + kQChunk + sw128(rl, u)) = l;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&a_full);
      }
      if (!ok) break;
      if (live && p.loss) p.loss[row] += lsum;
    }
    if (!ok) q_give_up(p);
  }
  __syncthreads();
  if (threadIdx.x == 128) {
    bulk_wait_all();
    if (q_aborted(p)) {
      // MMAs already issued finish before the tensor memory goes away
      umma_commit(&drain);
      mbar_wait(&drain, 0);
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, tcols);
  }
}

// ------------------------------------------------------------------ workers
// A task is one column block c of two slabs (rows 256 pair .. + 255, the
// second slab absent past the last): W[slab, c] += (-E[slab, k]) U[k, c]^T
// for both, as one 128 x 256 x 128 product, so one U tile serves two output
// tiles.  c runs from k + 1 on (k + 2 on when the chains take the next
// block); tasks go in order of k, then c (nearest first), then pair.  The
// split operands (U^T: 128 rows, -E: 256 rows; hi and lo) stream through a
// ring of kWSlots K chunks of 32 (96 KB each); the epilogue stages eight
// 32-row passes through kWStages buffers.  Thread 0 loads, thread 96 issues
// the MMAs, threads 128-255 run the epilogue; two tensor-memory accumulators
// (256 columns each) let a task's epilogue overlap the next task's MMAs.
struct QTask {
  int k, c, pair;
};

__host__ __device__ __forceinline__ int pairs_of(int nslab) { return (nslab + 1) / 2; }

__host__ __device__ __forceinline__ int64_t tasks_of_block(int64_t npair, int T, int k, int first) {
  const int later = T - k - first;  // column blocks k + first .. T - 1
  return later > 0 ? npair * later : 0;
}

__host__ __device__ __forceinline__ int64_t total_tasks(int64_t npair, int T, int first) {
  const int64_t m = T - first;  // sum over k of (T - k - first)
  return m > 0 ? npair * m * (m + 1) / 2 : 0;
}

struct TaskWalk {
  int k, first, npair;
  int64_t base, count;
  __device__ explicit TaskWalk(const SolveParams& p)
      : k(0), first(1 + p.chain_next), npair(pairs_of(p.nslab)), base(0),
        count(tasks_of_block(pairs_of(p.nslab), p.T, 0, 1 + p.chain_next)) {}
  __device__ QTask at(int64_t t, const SolveParams& p) {
    while (t >= base + count) {
      base += count;
      ++k;
      count = tasks_of_block(npair, p.T, k, first);
    }
    const int64_t idx = t - base;
    QTask q;
    q.k = k;
    q.c = k + first + (int)(idx / npair);
    q.pair = (int)(idx % npair);
    return q;
  }
};

__device__ __forceinline__ void worker_cta(const SolveMaps& mp, const SolveParams& p, uint8_t* sm) {
  uint8_t* ring = sm + kWRing;
  float* stg = reinterpret_cast<float*>(sm + kWStg);
  __shared__ uint64_t st_full[kWSlots], st_empty[kWSlots], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tslot;
  __shared__ int epi_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < kWSlots; ++b) {
      mbar_init(&st_full[b], 1);
      mbar_init(&st_empty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain, 1);
    epi_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  const int T = p.T;
  const int W = (int)gridDim.x - p.nchain, slot = (int)blockIdx.x - p.nchain;
  const int64_t total = total_tasks(pairs_of(p.nslab), T, 1 + p.chain_next);
  const uint32_t idesc = make_idesc(2, 128, 256);
  // a stage: U hi, U lo (128 rows each), then -E hi, -E lo (256 rows each)
  constexpr uint32_t kEOff = 2 * kQChunk, kEChunk = 2 * kQChunk, kStage = kEOff + 2 * kEChunk;
  if (threadIdx.x == 0) {
    // ------------------------------------------------------------ loader
    tma_prefetch_desc(&mp.uh);
    tma_prefetch_desc(&mp.ul);
    tma_prefetch_desc(&mp.eh2);
    tma_prefetch_desc(&mp.el2);
    TaskWalk tw(p);
    bool ok = true;
    int g = 0;  // K chunks loaded so far
    for (int64_t t = slot; ok && t < total; t += W) {
      const QTask q = tw.at(t, p);
      const int s0 = 2 * q.pair, s1 = s0 + 1;
      for (int ch = 0; ch < 4; ++ch, ++g) {
        const int rs = g % kWSlots, use = g / kWSlots;
        if (use > 0 && !q_mbar_wait(p, &st_empty[rs], (use - 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* dst = ring + rs * kStage;
        const int32_t xk = QB * q.k + SB * ch;
        mbar_arrive_expect_tx(&st_full[rs], kStage);
        tma_load_2d(dst, &mp.uh, &st_full[rs], xk, QB * q.c);
        tma_load_2d(dst + kQChunk, &mp.ul, &st_full[rs], xk, QB * q.c);
        if (ch == 0) {
          // both slabs' block k: -E published by their chains
          if (!q_wait_ge(p, &p.sdone[s0], q.k + 1) || (s1 < p.nslab && !q_wait_ge(p, &p.sdone[s1], q.k + 1))) {
            ok = false;
            break;
          }
          fence_proxy_async_global();
        }
        tma_load_2d(dst + kEOff, &mp.eh2, &st_full[rs], xk, QB * s0);
        tma_load_2d(dst + kEOff + kEChunk, &mp.el2, &st_full[rs], xk, QB * s0);
      }
    }
    if (!ok) q_give_up(p);
  } else if (threadIdx.x == 96) {
    // ------------------------------------------------------------ MMA issue
    bool ok = true;
    int tl = 0, g = 0;
    for (int64_t t = slot; ok && t < total; t += W, ++tl) {
      const int buf = tl & 1, use = tl >> 1;
      if (use > 0 && !q_mbar_wait(p, &acc_empty[buf], (use - 1) & 1)) {
        ok = false;
        break;
      }
      const uint32_t d = tbase + (uint32_t)buf * 256;
      for (int ch = 0; ch < 4; ++ch, ++g) {
        const int rs = g % kWSlots;
        if (!q_mbar_wait(p, &st_full[rs], (g / kWSlots) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(ring) + rs * kStage;
        // D[c][r] (+)= sum_j U^T[c][j] (-E)[r][j]: lanes are W's columns,
        // tensor-memory columns the pair's 256 rows
        issue_mma_chunk(d, base, base + kQChunk, base + kEOff, base + kEOff + kEChunk, idesc, ch > 0);
        umma_commit(&st_empty[rs]);
      }
      if (ok) umma_commit(&acc_full[buf]);
    }
    if (!ok) q_give_up(p);
  } else if (threadIdx.x >= 128) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int cl = quarter * 32 + lane;
    TaskWalk tw(p);
    int tl = 0, epi_pass = 0;
    for (int64_t t = slot; t < total; t += W, ++tl) {
      const QTask q = tw.at(t, p);
      const int s0 = 2 * q.pair, s1 = s0 + 1;
      const int buf = tl & 1;
      bool ok = q_mbar_wait(p, &acc_full[buf], (tl >> 1) & 1, true);
      if (threadIdx.x == 128 && ok) {
        // contributions reach a tile in order of k
        ok = q_wait_ge(p, &p.cnt[(int64_t)s0 * T + q.c], q.k) &&
             (s1 >= p.nslab || q_wait_ge(p, &p.cnt[(int64_t)s1 * T + q.c], q.k));
        fence_proxy_async_global();
      }
      if (!ok) epi_abort = 1;
      named_bar_sync(2, 128);
      if (epi_abort) break;  // the same decision in all 128 threads
      tc_fence_after();
      const uint32_t taddr = tbase + (uint32_t)buf * 256 + ((uint32_t)(quarter * 32) << 16);
      const int npass = s1 < p.nslab ? 8 : 4;
#pragma unroll 1
      for (int pz = 0; pz < npass; ++pz) {
        float v[32];
        tmem_ld32(taddr + (uint32_t)(32 * pz), v);
        float* sb = stg + (epi_pass % kWStages) * (32 * 128);
        if (threadIdx.x == 128) bulk_wait_read<kWStages - 1>();  // the reduce that last read sb is done
        named_bar_sync(2, 128);
#pragma unroll
        for (int j = 0; j < 32; ++j) sb[j * 128 + cl] = v[j];
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (threadIdx.x == 128) {
          tma_reduce_add_2d(&mp.wred, sb, QB * q.c, QB * s0 + 32 * pz);
          bulk_commit();
        }
        ++epi_pass;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      if (threadIdx.x == 128) {
        bulk_wait_all();
        fence_proxy_async_global();
        __threadfence();
        atomicExch(&p.cnt[(int64_t)s0 * T + q.c], q.k + 1);
        if (s1 < p.nslab) atomicExch(&p.cnt[(int64_t)s1 * T + q.c], q.k + 1);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 128) bulk_wait_all();
  if (q_aborted(p) && threadIdx.x == 96) {
    umma_commit(&drain);
    mbar_wait(&drain, 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int GSB>
__global__ void __launch_bounds__(QNT, 1) solve_kernel(const __grid_constant__ SolveMaps mp, const SolveParams p) {
  extern __shared__ __align__(1024) uint8_t qsm_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)qsm_raw + 1023) & ~(uintptr_t)1023);
  if ((int)blockIdx.x < p.nchain)
    chain_cta<GSB>(mp, p, sm);
  else
    worker_cta(mp, p, sm);
}

// Ud[b] for each 32-column sub-block b: U[c0 + j][c0 + j'] at [j][j'] for
// j < j' (the rest zero), then 1 / U_jj; columns past `in` are zero.  U is
// stored by columns: Ucm[c][j] = U[j][c].
__global__ void __launch_bounds__(256) pack_ud_kernel(const float* __restrict__ U, int64_t in,
                                                      float* __restrict__ Ud) {
  const int64_t c0 = (int64_t)SB * blockIdx.x;
  float* dst = Ud + (int64_t)blockIdx.x * kUdFloats;
  for (int e = threadIdx.x; e < SB * SB; e += blockDim.x) {
    const int jp = e / SB, j = e % SB;  // consecutive threads read consecutive j of column jp
    float v = 0.f;
    if (j < jp && c0 + jp < in) v = U[(c0 + jp) * in + c0 + j];
    dst[j * SB + jp] = v;
  }
  for (int j = threadIdx.x; j < SB; j += blockDim.x) dst[SB * SB + j] = c0 + j < in ? 1.f / U[(c0 + j) * in + c0 + j] : 0.f;
}

template <int GSB>
cudaError_t launch_solve(const SolveMaps& mp, const SolveParams& p, int grid, cudaStream_t st) {
  cudaError_t e = ensure_smem_limit((const void*)solve_kernel<GSB>, (int)kSolveSmem);
  if (e != cudaSuccess) return e;
  void* args[] = {(void*)&mp, (void*)&p};
  e = cudaLaunchCooperativeKernel((const void*)solve_kernel<GSB>, dim3(grid), dim3(QNT), args, kSolveSmem, st);
  note_launch();
  return e;
}

}  // namespace

size_t solve_ud_bytes(int64_t np_) { return (size_t)(np_ / SB) * kUdBytes; }

size_t solve_sync_bytes(int64_t out, int64_t np_) {
  const int64_t nslab = (out + QB - 1) / QB;
  return sizeof(int) * (size_t)(nslab + nslab * (np_ / QB) + 4);
}

cudaError_t solve_pack_ud(const float* U, int64_t in, int64_t np_, float* Ud, cudaStream_t st) {
  pack_ud_kernel<<<(unsigned)(np_ / SB), 256, 0, st>>>(U, in, Ud);
  note_launch();
  return cudaGetLastError();
}

cudaError_t solve_quantize(float* Wp, int64_t out, int64_t in, int64_t np_, const float* Uh, const float* Ul,
                           const float* Ud, float* Eh, float* El, const gptq_config_t* cfg, float* scales,
                           int32_t* zeros, uint8_t* codes_p, float* loss, void* sync, uint32_t* status, int sms,
                           cudaStream_t st) {
  if (out == 0) return cudaSuccess;
  const int gs = cfg->group_size;
  const int gsb = (gs == -1 || gs >= QB) ? QB : gs;
  const void* fn = nullptr;
  switch (gsb) {
    case 8: fn = (const void*)solve_kernel<8>; break;
    case 16: fn = (const void*)solve_kernel<16>; break;
    case 32: fn = (const void*)solve_kernel<32>; break;
    case 64: fn = (const void*)solve_kernel<64>; break;
    case 128: fn = (const void*)solve_kernel<128>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_limit(fn, (int)kSolveSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, QNT, kSolveSmem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int gmax = sms * per_sm;
  const int T = (int)(np_ / QB);
  const int nslab = (int)((out + QB - 1) / QB);
  // chains: at most a quarter of the CTAs, the slabs spread evenly over them
  const int cap = std::max(1, gmax / 4);
  const int spc = (nslab + cap - 1) / cap;
  const int nchain = (nslab + spc - 1) / spc;
  // up to two slabs per chain, the chains also take each slab's next block
  const int chain_next = spc <= 2 ? 1 : 0;
  const int64_t ntask = total_tasks(pairs_of(nslab), T, 1 + chain_next);
  const int nworker = ntask > 0 ? (int)std::min<int64_t>(gmax - nchain, ntask) : 0;
  if (ntask > 0 && nworker < 1) return cudaErrorInvalidConfiguration;
  e = cudaMemsetAsync(sync, 0, solve_sync_bytes(out, np_), st);
  if (e != cudaSuccess) return e;
  SolveParams p;
  p.Wp = Wp;
  p.np_ = np_;
  p.out = out;
  p.in = in;
  p.Ud = Ud;
  p.T = T;
  p.nslab = nslab;
  p.nchain = nchain;
  p.chain_next = chain_next;
  p.maxq = (1 << cfg->bits) - 1;
  p.sym = cfg->sym;
  p.gs = gs;
  p.ngroups = gs == -1 ? 1 : (int)(in / gs);
  p.scales = scales;
  p.zeros = zeros;
  p.codes_p = codes_p;
  p.loss = loss;
  p.sdone = (int*)sync;
  p.cnt = p.sdone + nslab;
  p.abort_flag = (unsigned*)(p.cnt + (int64_t)nslab * T);
  p.status = status;
  SolveMaps mp;
  if (!encode_f32_2d(&mp.wld, Wp, np_, out, np_, SB, QB, true) ||
      !encode_f32_2d(&mp.wred, Wp, np_, out, np_, QB, 32, false) ||
      !encode_f32_2d(&mp.uh, Uh, np_, np_, np_, SB, QB, true) ||
      !encode_f32_2d(&mp.ul, Ul, np_, np_, np_, SB, QB, true) ||
      !encode_f32_2d(&mp.eh, Eh, np_, out, np_, SB, QB, true) ||
      !encode_f32_2d(&mp.el, El, np_, out, np_, SB, QB, true) ||
      !encode_f32_2d(&mp.eh2, Eh, np_, out, np_, SB, 2 * QB, true) ||
      !encode_f32_2d(&mp.el2, El, np_, out, np_, SB, 2 * QB, true))
    return cudaErrorInvalidValue;
  const int grid = nchain + nworker;
  switch (gsb) {
    case 8: return launch_solve<8>(mp, p, grid, st);
    case 16: return launch_solve<16>(mp, p, grid, st);
    case 32: return launch_solve<32>(mp, p, grid, st);
    case 64: return launch_solve<64>(mp, p, grid, st);
    default: return launch_solve<128>(mp, p, grid, st);
  }
}

cudaError_t preload_solve_kernels() {
  const void* fns[] = {(const void*)solve_kernel<8>, (const void*)solve_kernel<16>, (const void*)solve_kernel<32>,
                       (const void*)solve_kernel<64>, (const void*)solve_kernel<128>, (const void*)pack_ud_kernel};
  for (const void* f : fns) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, f);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace gptq
