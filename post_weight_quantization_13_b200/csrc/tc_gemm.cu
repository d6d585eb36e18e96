// tcgen05 tensor-core kernel for C (+)= alpha * P Q^T (see gemm.cuh).
//
// One persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: fills a ring of shared-memory stages with
//               K-major operand tiles (128-byte rows, 128-byte swizzle: 64
//               16-bit or 32 tf32 elements of k per row).  Row ranges are
//               cut into power-of-two boxes (256/128/64/32/16 rows), so a
//               stage needs only a handful of copies.
//   warp 1      owns the tensor memory (all 512 columns) and issues
//               tcgen05.mma from one thread; completion is signalled back to
//               the producer (stage free) and to the epilogue (accumulator
//               ready) through tcgen05.commit on mbarriers.
//   warps 2-5   epilogue: tcgen05.ld of the fp32 accumulators, then a
//               coalesced read-modify-write of C (lane = column of C), with
//               32 loads in flight per thread.  They sleep while they wait,
//               so they do not take issue slots from warps 0 and 1.
//
// One MMA is M = 128 (C columns = tensor-memory lanes) by N <= 256 (C rows =
// tensor-memory columns).  A "piece" is a row range of up to 256 rows of C
// against one or two 128-column Q tiles (two accumulators that share the P
// tile: a 256 x N output from 256 + N operand rows per k).  Schedules:
//   tri   the upper triangle of a symmetric S = X X^T, in 256-column
//         super-strips; super-strip s needs rows [0, 256(s+1)), i.e. s + 1
//         pieces of 256 rows.  One piece per CTA and round; all CTAs stream
//         the same k-window of X together, which keeps X L2-resident.  With
//         one 256 x 256 piece per round a stage is 64 KB, so three stages
//         fit in shared memory.
//   grid  regular tiles of 128 C columns by 256 (or, on request, 128) C
//         rows (optionally batched), one per round, with two tensor-memory
//         buffers so a tile's epilogue overlaps the next tile's main loop.
//         128-row tiles halve a stage, so a 3xTF32 product keeps three
//         stages in flight instead of two.
// Long k ranges are cut into chunks; after each chunk the accumulators are
// drained into C with round-to-nearest adds, which bounds the error of the
// tensor core's in-place fp32 accumulation.
// Every wait is bounded: a wait that gives up records ST_TIMEOUT in the
// status word, stops the CTA's work, lets in-flight copies and MMAs drain
// (bounded again), frees the tensor memory and returns.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gemm.cuh"

namespace gptq {

namespace {

constexpr int kThreads = 192;
constexpr int kMaxPieces = 2;
constexpr uint32_t kRowBytes = 128;                // one K-major row per stage (128-byte swizzle)
constexpr uint32_t kQTileBytes = 128 * kRowBytes;  // 16 KB per component
constexpr int kNumBoxes = 5;                       // P boxes of 256, 128, 64, 32, 16 rows

struct Piece {
  int q0;     // first C column (Q row)
  int nh;     // 128-column halves: 1 or 2
  int p0;     // first C row (P row)
  int np;     // rows, multiple of 16, <= 256
  int qslot;  // Q slot of the stage
  int prow;   // first row inside the stage's P region
  int tcol;   // first tensor-memory column (half h at tcol + h * np)
  int batch;
};

struct KParams {
  int tri;
  int kbc;                       // k-tiles per round
  int kchunk, nchunks;           // k-tiles per accumulator drain, drains per round
  int p_row0, p_k0, q_row0, q_k0;
  int R, Cn;
  // grid schedule
  int nq, npt, ntiles;
  int ptile;  // P rows per output tile: 256, or 128 for more and smaller pipeline stages
  int64_t bs_p_row, bs_p_k, bs_q_row, bs_q_k, bs_c_row, bs_c_col;
  // tri schedule
  int n_in, nss;
  int grid, rounds;
  // epilogue
  float* C;
  float* C_lo;
  int64_t ldc, c_row0, c_col0;
  float alpha, beta;
  int mask;
  int64_t mask_off;
  int transpose;
  uint32_t* status;
  // TMA epilogue: accumulators staged in shared memory, written by a bulk
  // tensor store (beta == 0) or reduce-add (beta == 1)
  int epi_tma;
  int epi_split;  // also store the tf32 remainder (through map clo)
  int lower;      // grid schedule over tiles that hold elements with c - r <= mask_off only
  // shared-memory plan
  int stages, stage_bytes, qslots, slot_bytes, p_rows_max;
};

struct TmaMaps {
  CUtensorMap p[kNumBoxes];    // P (hi) with box heights 256, 128, 64, 32, 16
  CUtensorMap plo[kNumBoxes];  // P remainder (3xTF32 only)
  CUtensorMap q;               // Q (hi), 128-row boxes
  CUtensorMap qlo;
  CUtensorMap c;               // output (TMA epilogue): 32 x 128 tiles, 3-D (batch)
  CUtensorMap clo;             // output remainder (split outputs)
};
constexpr uint32_t kStageTileBytes = 32 * 128 * 4;  // one epilogue pass: 32 rows x 128 columns fp32

// Column tiles of row tile pt that hold an element with c - r <= mask_off.
__host__ __device__ __forceinline__ int lower_tiles(const KParams& kp, int pt) {
  const int64_t last = ((int64_t)pt * 256 + 255 + kp.mask_off) / 128 + 1;
  return (int)(last < 0 ? 0 : (last > kp.nq ? kp.nq : last));
}

__host__ __device__ int round_pieces(const KParams& kp, int cta, int round, Piece* pc) {
  if (kp.tri) {
    // piece index t -> (super-strip s, 256-row piece within it); super-strip
    // s has s + 1 pieces (the last super-strip may have fewer rows)
    const int t = round * kp.grid + cta;
    if (t >= kp.ntiles) return 0;
    int s = (int)((sqrtf(1.0f + 8.0f * (float)t) - 1.0f) * 0.5f);
    if (s < 0) s = 0;
    while (s + 1 < kp.nss && (s + 1) * (s + 2) / 2 <= t) ++s;
    while (s > 0 && s * (s + 1) / 2 > t) --s;
    const int piece = t - s * (s + 1) / 2;
    Piece& p = pc[0];
    p.q0 = 256 * s;
    p.nh = (256 * s + 128 < kp.n_in) ? 2 : 1;
    p.p0 = 256 * piece;
    const int rows = min(256, kp.n_in - p.p0);
    p.np = (rows + 15) & ~15;
    p.qslot = 0;
    p.prow = 0;
    p.tcol = 0;
    p.batch = 0;
    return 1;
  }
  if (kp.lower) {
    int t = round * kp.grid + cta;
    if (t >= kp.ntiles) return 0;
    for (int pt = 0; pt < kp.npt; ++pt) {
      const int cnt = lower_tiles(kp, pt);
      if (t < cnt) {
        Piece& p = pc[0];
        p.q0 = t * 128;
        p.nh = 1;
        p.p0 = pt * 256;
        const int rows = min(256, kp.R - p.p0);
        p.np = (rows + 15) & ~15;
        p.qslot = 0;
        p.prow = 0;
        p.tcol = 0;
        p.batch = 0;
        return 1;
      }
      t -= cnt;
    }
    return 0;
  }
  const int t = round * kp.grid + cta;
  if (t >= kp.ntiles) return 0;
  const int per = kp.nq * kp.npt;
  const int batch = t / per;
  const int rem = t - batch * per;
  const int pt = rem / kp.nq;
  const int qt = rem - pt * kp.nq;
  Piece& p = pc[0];
  p.q0 = qt * 128;
  p.nh = 1;
  p.p0 = pt * kp.ptile;
  const int rows = min(kp.ptile, kp.R - p.p0);
  p.np = (rows + 15) & ~15;
  p.qslot = 0;
  p.prow = 0;
  p.tcol = 0;
  p.batch = batch;
  return 1;
}

template <int OP>
struct OpTraits;
template <>
struct OpTraits<OP_F16> {
  static constexpr int kSplit = 1, kBK = 64, kFmt = 0;
};
template <>
struct OpTraits<OP_BF16> {
  static constexpr int kSplit = 1, kBK = 64, kFmt = 1;
};
template <>
struct OpTraits<OP_TF32X3> {
  static constexpr int kSplit = 2, kBK = 32, kFmt = 2;
};

__device__ __forceinline__ void abort_cta(const KParams& kp, volatile int* abort_flag) {
  raise_status(kp.status, ST_TIMEOUT);
  *abort_flag = 1;
}

template <int OP>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ TmaMaps maps, const __grid_constant__ KParams kp) {
  constexpr int SPLIT = OpTraits<OP>::kSplit;
  constexpr int BK = OpTraits<OP>::kBK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + (size_t)kp.stages * kp.stage_bytes + (kp.epi_tma ? 2 * kStageTileBytes : 0));
  uint64_t* empty = full + kp.stages;
  uint64_t* acc_full = empty + kp.stages;  // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;         // [1]
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nbuf = kp.tri ? 1 : 2;
  const uint32_t buf_cols = 512u / nbuf;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kp.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int b = 0; b < kNumBoxes; ++b) tma_prefetch_desc(&maps.p[b]);
    tma_prefetch_desc(&maps.q);
    if (SPLIT == 2) {
      for (int b = 0; b < kNumBoxes; ++b) tma_prefetch_desc(&maps.plo[b]);
      tma_prefetch_desc(&maps.qlo);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // everything above touches only this CTA's shared and tensor memory and the
  // kernel parameters: under a dependent launch (the 3xTF32 lazy updates of
  // the sweep) it overlaps the previous kernel, and the operand loads and
  // output writes below wait for it
  if constexpr (OP == OP_TF32X3) grid_dependency_wait();

  const uint32_t q_region = (uint32_t)(kp.qslots * kp.slot_bytes);
  const uint32_t p_comp = (uint32_t)kp.p_rows_max * kRowBytes;  // one component of the P region

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      // Parameters the loops use live in registers: the inline asm below
      // clobbers memory, which would otherwise force reloads of the
      // parameter block on every iteration.
      const int rounds = kp.rounds, kbc = kp.kbc, stages = kp.stages, stage_bytes = kp.stage_bytes;
      const int slot_bytes = kp.slot_bytes;
      const int q_k0 = kp.q_k0, q_row0 = kp.q_row0, p_k0 = kp.p_k0, p_row0 = kp.p_row0;
      const int64_t bs_q_k = kp.bs_q_k, bs_q_row = kp.bs_q_row, bs_p_k = kp.bs_p_k, bs_p_row = kp.bs_p_row;
      int stage = 0;
      uint32_t phase = 0;
      for (int round = 0; round < rounds && !*abort_flag; ++round) {
        Piece pl[kMaxPieces];
        const int npc = round_pieces(kp, blockIdx.x, round, pl);
        if (npc <= 0) break;
        Piece pc[kMaxPieces];
        uint32_t bytes = 0;
#pragma unroll
        for (int i = 0; i < kMaxPieces; ++i) {
          pc[i] = pl[i];
          if (i < npc) bytes += (uint32_t)(pc[i].nh * kQTileBytes + pc[i].np * kRowBytes) * SPLIT;
        }
        for (int kb = 0; kb < kbc; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            abort_cta(kp, abort_flag);
            break;
          }
          if (*abort_flag) break;
          uint8_t* sb = smem + (size_t)stage * stage_bytes;
          uint64_t* bar = &full[stage];
          mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
          for (int i = 0; i < kMaxPieces; ++i) {
            if (i >= npc) break;
            const Piece& p = pc[i];
            const int bq = p.batch;
            const int xq = (int)(q_k0 + bq * bs_q_k) + kb * BK;
            const int yq = (int)(q_row0 + bq * bs_q_row) + p.q0;
            uint8_t* dq = sb + p.qslot * slot_bytes;
            for (int h = 0; h < p.nh; ++h) {
              uint8_t* d = dq + h * kQTileBytes * SPLIT;
              tma_load_2d(d, &maps.q, bar, xq, yq + 128 * h);
              if (SPLIT == 2) tma_load_2d(d + kQTileBytes, &maps.qlo, bar, xq, yq + 128 * h);
            }
            const int xp = (int)(p_k0 + bq * bs_p_k) + kb * BK;
            const int yp = (int)(p_row0 + bq * bs_p_row) + p.p0;
            int off = 0;
#pragma unroll
            for (int b = 0; b < kNumBoxes; ++b) {
              const int rows = 256 >> b;
              if (p.np & rows) {
                uint8_t* d = sb + q_region + (uint32_t)(p.prow + off) * kRowBytes;
                tma_load_2d(d, &maps.p[b], bar, xp, yp + off);
                if (SPLIT == 2) tma_load_2d(d + p_comp, &maps.plo[b], bar, xp, yp + off);
                off += rows;
              }
            }
          }
          if (++stage == stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const int rounds = kp.rounds, nchunks = kp.nchunks, kchunk = kp.kchunk, kbc = kp.kbc;
      const int stages = kp.stages, stage_bytes = kp.stage_bytes, slot_bytes = kp.slot_bytes;
      int stage = 0;
      uint32_t phase = 0;
      int step = 0;  // (round, chunk) counter: selects the accumulator buffer
      bool ok = true;
      for (int round = 0; round < rounds && ok && !*abort_flag; ++round) {
        Piece pl[kMaxPieces];
        const int npc = round_pieces(kp, blockIdx.x, round, pl);
        if (npc <= 0) break;
        Piece pc[kMaxPieces];
        uint32_t idesc[kMaxPieces];
#pragma unroll
        for (int i = 0; i < kMaxPieces; ++i) {
          pc[i] = pl[i];
          idesc[i] = make_idesc(OpTraits<OP>::kFmt, 128, (uint32_t)pc[i].np);
        }
        for (int ch = 0; ch < nchunks && ok; ++ch, ++step) {
          const int buf = step % nbuf;
          const int use = step / nbuf;
          if (use > 0 && !mbar_wait(&acc_empty[buf], (use - 1) & 1)) {
            abort_cta(kp, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tacc = tbase + buf * buf_cols;
          const int kb0 = ch * kchunk;
          const int kb1 = min(kbc, kb0 + kchunk);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&full[stage], phase)) {
              abort_cta(kp, abort_flag);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sb = smem_u32(smem + (size_t)stage * stage_bytes);
#pragma unroll
            for (int i = 0; i < kMaxPieces; ++i) {
              if (i >= npc) break;
              const Piece& p = pc[i];
              const uint32_t pb = sb + q_region + (uint32_t)p.prow * kRowBytes;
              for (int h = 0; h < p.nh; ++h) {
                const uint32_t qa = sb + p.qslot * slot_bytes + h * kQTileBytes * SPLIT;
                const uint32_t d = tacc + (uint32_t)(p.tcol + h * p.np);
#pragma unroll
                for (int kk = 0; kk < (int)(kRowBytes / 32); ++kk) {
                  const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
                  const uint64_t ad = smem_desc_k_sw128(qa + kk * 32);
                  const uint64_t bd = smem_desc_k_sw128(pb + kk * 32);
                  if (SPLIT == 1) {
                    umma_f16(d, ad, bd, idesc[i], acc);
                  } else {
                    const uint64_t ad_lo = smem_desc_k_sw128(qa + kQTileBytes + kk * 32);
                    const uint64_t bd_lo = smem_desc_k_sw128(pb + p_comp + kk * 32);
                    umma_tf32(d, ad, bd, idesc[i], acc);
                    umma_tf32(d, ad, bd_lo, idesc[i], 1u);
                    umma_tf32(d, ad_lo, bd, idesc[i], 1u);
                  }
                }
              }
            }
            umma_commit(&empty[stage]);
            if (++stage == stages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          umma_commit(&acc_full[buf]);
        }
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2-5)
    const int quarter = warp & 3;  // tensor-memory lanes 32*quarter .. +31
    const int rounds = kp.rounds, nchunks = kp.nchunks;
    const int R = kp.R, Cn = kp.Cn, mask = kp.mask, transpose = kp.transpose;
    const int64_t mask_off = kp.mask_off, ldc = kp.ldc, c_row0 = kp.c_row0, c_col0 = kp.c_col0;
    const int64_t bs_c_row = kp.bs_c_row, bs_c_col = kp.bs_c_col;
    const float alpha = kp.alpha, beta0 = kp.beta;
    float* const Cbase = kp.C;
    float* const Clbase = kp.C_lo;
    const int epi_tma = kp.epi_tma, epi_split = kp.epi_split;
    uint8_t* const stage_out = smem + (size_t)kp.stages * kp.stage_bytes;  // 2 x 16 KB
    int epi_pass = 0;
    int step = 0;
    bool ok = true;
    for (int round = 0; round < rounds && ok; ++round) {
      Piece pc[kMaxPieces];
      const int npc = round_pieces(kp, blockIdx.x, round, pc);
      if (npc <= 0) break;
      for (int ch = 0; ch < nchunks; ++ch, ++step) {
        const int buf = step % nbuf;
        const int use = step / nbuf;
        if (!mbar_wait_sleep(&acc_full[buf], use & 1)) {
          abort_cta(kp, abort_flag);
          ok = false;
          break;
        }
        if (*abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the first chunk applies beta, later chunks accumulate onto C
        const float beta = ch == 0 ? beta0 : 1.f;
        for (int i = 0; i < npc; ++i) {
          const Piece& p = pc[i];
          const int64_t cr = c_row0 + (int64_t)p.batch * bs_c_row;
          const int64_t cc = c_col0 + (int64_t)p.batch * bs_c_col;
          for (int h = 0; h < p.nh; ++h) {
            const int c = p.q0 + 128 * h + quarter * 32 + lane;
            const uint32_t taddr = tbase + buf * buf_cols + (uint32_t)(p.tcol + h * p.np) +
                                   ((uint32_t)(quarter * 32) << 16);
            if (epi_tma) {
              const int cl = quarter * 32 + lane;  // column inside the 128-column tile
              const bool reduce = beta != 0.f;     // beta is 0 (store) or 1 (reduce-add)
              for (int n0 = 0; n0 < p.np; n0 += 32) {
                float v[32];
                if (p.np - n0 >= 32) {
                  tmem_ld32(taddr + (uint32_t)n0, v);
                } else {
                  float t16[16];
                  tmem_ld16(taddr + (uint32_t)n0, t16);
#pragma unroll
                  for (int j = 0; j < 16; ++j) v[j] = t16[j];
#pragma unroll
                  for (int j = 16; j < 32; ++j) v[j] = 0.f;
                }
                const int r0 = p.p0 + n0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  float x = alpha * v[j];
                  if (mask == 1 && (int64_t)c - (r0 + j) < mask_off) x = 0.f;
                  if (mask == 2 && (int64_t)c - (r0 + j) > mask_off) x = 0.f;
                  v[j] = x;
                }
                // the staging buffer is free once the bulk copy that last read it is done
                uint8_t* sb0 = stage_out + (epi_split ? 0 : (epi_pass & 1) * kStageTileBytes);
                if (threadIdx.x == 64) {
                  if (epi_split)
                    bulk_wait_read<0>();
                  else
                    bulk_wait_read<1>();
                }
                named_bar_sync(1, 128);
                float* sh = reinterpret_cast<float*>(sb0);
                float* sl = reinterpret_cast<float*>(sb0 + kStageTileBytes);
                if (!transpose) {
                  // tile [32 rows][128 columns]
#pragma unroll
                  for (int j = 0; j < 32; ++j) {
                    if (epi_split) {
                      float hi, lo;
                      split_tf32(v[j], hi, lo);
                      sh[j * 128 + cl] = hi;
                      sl[j * 128 + cl] = lo;
                    } else {
                      sh[j * 128 + cl] = v[j];
                    }
                  }
                } else {
                  // tile [128 columns of C = rows of the output][32], 128-byte swizzle
#pragma unroll
                  for (int m = 0; m < 8; ++m) {
                    const int off = cl * 32 + ((m ^ (cl & 7)) * 4);
                    if (epi_split) {
                      float4 h4, l4;
                      split_tf32(v[4 * m + 0], h4.x, l4.x);
                      split_tf32(v[4 * m + 1], h4.y, l4.y);
                      split_tf32(v[4 * m + 2], h4.z, l4.z);
                      split_tf32(v[4 * m + 3], h4.w, l4.w);
                      *reinterpret_cast<float4*>(sh + off) = h4;
                      *reinterpret_cast<float4*>(sl + off) = l4;
                    } else {
                      *reinterpret_cast<float4*>(sh + off) =
                          make_float4(v[4 * m + 0], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
                    }
                  }
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (threadIdx.x == 64) {
                  const int tc = p.q0 + 128 * h, tr = r0;
                  const int x = transpose ? tr : tc, y = transpose ? tc : tr;
                  if (reduce)
                    tma_reduce_add_3d(&maps.c, sh, x, y, p.batch);
                  else
                    tma_store_3d(&maps.c, sh, x, y, p.batch);
                  if (epi_split) tma_store_3d(&maps.clo, sl, x, y, p.batch);
                  bulk_commit();
                }
                ++epi_pass;
              }
              continue;
            }
            for (int n0 = 0; n0 < p.np; n0 += 32) {
              // 32 accumulator columns (C rows) per pass: every load of C is
              // issued before any store so they overlap in flight.
              float v[32];
              if (p.np - n0 >= 32) {
                tmem_ld32(taddr + (uint32_t)n0, v);
              } else {
                float t16[16];
                tmem_ld16(taddr + (uint32_t)n0, t16);
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = t16[j];
#pragma unroll
                for (int j = 16; j < 32; ++j) v[j] = 0.f;
              }
              if (c >= Cn) continue;
              const int nn = min(32, p.np - n0);
              const int r0 = p.p0 + n0;
              const int64_t base =
                  transpose ? (cr + c) * ldc + (cc + r0) : (cr + r0) * ldc + (cc + c);
              const int64_t stp = transpose ? 1 : ldc;
              uint32_t keep = 0;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int r = r0 + j;
                bool k = j < nn && r < R;
                if (mask == 1) k = k && ((int64_t)c - r >= mask_off);
                if (mask == 2) k = k && ((int64_t)c - r <= mask_off);
                keep |= (uint32_t)k << j;
              }
              float* __restrict__ Cp = Cbase + base;
              float* __restrict__ Cl = Clbase ? Clbase + base : nullptr;
              if (beta != 0.f) {
                float old[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) old[j] = ((keep >> j) & 1u) ? Cp[j * stp] : 0.f;
                if (Cl) {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if ((keep >> j) & 1u) old[j] += Cl[j * stp];
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = fmaf(beta, old[j], alpha * v[j]);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = alpha * v[j];
              }
              if (Cl) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (!((keep >> j) & 1u)) continue;
                  float hi, lo;
                  split_tf32(v[j], hi, lo);
                  Cp[j * stp] = hi;
                  Cl[j * stp] = lo;
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if ((keep >> j) & 1u) Cp[j * stp] = v[j];
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
      }
    }
    if (epi_tma && threadIdx.x == 64) bulk_wait_all();
  }

  __syncthreads();
  if (*abort_flag) {
    // Let copies and MMAs that were already issued finish before the shared
    // and tensor memory go away (both bounded).
    if (threadIdx.x == 32) {
      umma_commit(drain);
      mbar_wait(drain, 0);
    }
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 1000000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int esize, int op,
              int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  CUtensorMapDataType dt = op == OP_F16    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                           : op == OP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)(ld * esize)};
  cuuint32_t box[2] = {(cuuint32_t)(kRowBytes / esize), (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D output map (columns, rows, batch) for the TMA epilogue.  box_x x box_y
// fp32 tiles, no swizzle (box_x = 128) or 128-byte swizzle (box_x = 32).
bool make_out_map(CUtensorMap* m, const float* base, int64_t xdim, int64_t ydim, int64_t ld, int64_t batch,
                  int64_t bstride, int box_x, int box_y) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t gdim[3] = {(cuuint64_t)xdim, (cuuint64_t)ydim, (cuuint64_t)batch};
  cuuint64_t gstride[2] = {(cuuint64_t)(ld * 4), (cuuint64_t)(bstride * 4)};
  cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box_x == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int esize_of(int op) { return op == OP_TF32X3 ? 4 : 2; }
int bk_of(int op) { return op == OP_TF32X3 ? 32 : 64; }  // elements per 128-byte row

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

template <int OP>
cudaError_t launch(const TmaMaps& maps, const KParams& kp, int grid, size_t smem, cudaStream_t st, bool pdl) {
  cudaError_t ce = ensure_smem_limit((const void*)tc_gemm_kernel<OP>, 232448);
  if (ce != cudaSuccess) return ce;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  ce = cudaLaunchKernelEx(&cfg, tc_gemm_kernel<OP>, maps, kp);
  note_launch();
  return ce != cudaSuccess ? ce : cudaGetLastError();
}

}  // namespace

cudaError_t preload_gemm_kernels() {
  const void* fns[] = {(const void*)tc_gemm_kernel<OP_F16>, (const void*)tc_gemm_kernel<OP_BF16>,
                       (const void*)tc_gemm_kernel<OP_TF32X3>};
  for (const void* f : fns) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, f);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool tc_gemm_supported(const GemmArgs& a) {
  const int es = esize_of(a.op);
  const Operand* ops[2] = {&a.P, &a.Q};
  for (const Operand* o : ops) {
    if (!o->hi || !aligned16(o->hi) || (o->ld * es) % 16) return false;
    if (a.op == OP_TF32X3 && (!o->lo || !aligned16(o->lo))) return false;
    if (o->rows <= 0 || o->cols <= 0) return false;
  }
  if (a.tri) return a.batch == 1 && a.P.hi == a.Q.hi && a.R == a.Cn;
  // the k range of each product must end on a k-tile or at the stored edge
  const int bk = bk_of(a.op);
  if (a.K % bk) {
    for (int b = 0; b < a.batch; ++b) {
      if (a.p_k0 + b * a.bs_p_k + a.K != a.P.cols) return false;
      if (a.q_k0 + b * a.bs_q_k + a.K != a.Q.cols) return false;
    }
  }
  return true;
}

cudaError_t tc_gemm(const GemmArgs& a, cudaStream_t st, int num_sms) {
  if (a.R <= 0 || a.Cn <= 0 || a.K <= 0 || a.batch <= 0) return cudaSuccess;
  const int es = esize_of(a.op);
  const int split = a.op == OP_TF32X3 ? 2 : 1;
  TmaMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  for (int b = 0; b < kNumBoxes; ++b) {
    if (!make_map(&maps.p[b], a.P.hi, a.P.rows, a.P.cols, a.P.ld, es, a.op, 256 >> b)) return cudaErrorInvalidValue;
    if (split == 2 && !make_map(&maps.plo[b], a.P.lo, a.P.rows, a.P.cols, a.P.ld, es, a.op, 256 >> b))
      return cudaErrorInvalidValue;
  }
  if (!make_map(&maps.q, a.Q.hi, a.Q.rows, a.Q.cols, a.Q.ld, es, a.op, 128)) return cudaErrorInvalidValue;
  if (split == 2 && !make_map(&maps.qlo, a.Q.lo, a.Q.rows, a.Q.cols, a.Q.ld, es, a.op, 128))
    return cudaErrorInvalidValue;
  KParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.tri = a.tri;
  kp.kbc = (int)((a.K + bk_of(a.op) - 1) / bk_of(a.op));
  // Drain the fp32 accumulators into C every chunk of k-tiles: the tensor
  // core's in-place fp32 accumulation error grows with the number of MMAs
  // summed in one accumulator, while C gets round-to-nearest adds.  32768
  // elements of k per drain for 16-bit inputs, 4096 for 3xTF32.
  const int chunk_tiles = (split == 1 ? 32768 : 4096) / bk_of(a.op);
  kp.kchunk = std::min(kp.kbc, chunk_tiles);
  kp.nchunks = (kp.kbc + kp.kchunk - 1) / kp.kchunk;
  kp.p_row0 = (int)a.p_row0;
  kp.p_k0 = (int)a.p_k0;
  kp.q_row0 = (int)a.q_row0;
  kp.q_k0 = (int)a.q_k0;
  kp.R = (int)a.R;
  kp.Cn = (int)a.Cn;
  kp.C = a.C;
  kp.C_lo = a.C_lo;
  kp.ldc = a.ldc;
  kp.c_row0 = a.c_row0;
  kp.c_col0 = a.c_col0;
  kp.alpha = a.alpha;
  kp.beta = a.beta;
  kp.mask = a.mask;
  kp.mask_off = a.mask_off;
  kp.transpose = a.transpose;
  kp.status = a.status;
  int grid;
  if (a.tri) {
    // one CTA round = one 256-column super-strip x up to 256 rows; the
    // upper triangle needs pieces 0..s of super-strip s
    const int n = (int)a.R;
    kp.n_in = n;
    kp.nss = (n + 255) / 256;
    kp.ntiles = 0;
    for (int s = 0; s < kp.nss; ++s) kp.ntiles += (std::min(256 * (s + 1), n) + 255) / 256;
    grid = std::min(num_sms, kp.ntiles);
    kp.grid = grid;
    kp.rounds = (kp.ntiles + grid - 1) / grid;
    kp.qslots = 1;
    kp.slot_bytes = 2 * kQTileBytes * split;
    kp.p_rows_max = 256;
  } else {
    // 128-row tiles halve a stage (three stages fit instead of two for
    // 3xTF32); the banded schedule below keeps 256-row tiles
    const bool lower = a.mask == 2 && a.batch == 1;
    kp.ptile = (!lower && a.p_tile == 128) ? 128 : 256;
    kp.nq = (int)((a.Cn + 127) / 128);
    kp.npt = (int)((a.R + kp.ptile - 1) / kp.ptile);
    kp.ntiles = kp.nq * kp.npt * a.batch;
    if (lower) {  // skip tiles entirely above the kept band
      kp.lower = 1;
      kp.mask_off = a.mask_off;
      kp.ntiles = 0;
      for (int pt = 0; pt < kp.npt; ++pt) kp.ntiles += lower_tiles(kp, pt);
      if (kp.ntiles == 0) return cudaSuccess;
    }
    kp.bs_p_row = a.bs_p_row;
    kp.bs_p_k = a.bs_p_k;
    kp.bs_q_row = a.bs_q_row;
    kp.bs_q_k = a.bs_q_k;
    kp.bs_c_row = a.bs_c_row;
    kp.bs_c_col = a.bs_c_col;
    grid = std::min(num_sms, kp.ntiles);
    kp.grid = grid;
    kp.rounds = (kp.ntiles + grid - 1) / grid;
    kp.qslots = 1;
    kp.slot_bytes = kQTileBytes * split;
    kp.p_rows_max = kp.ptile;
  }
  // TMA epilogue when the output allows it: beta 0 (store) or 1 (reduce-add),
  // 16-byte aligned rows, and masks only where masked elements can add 0.
  {
    const int64_t bstride = a.batch > 1 ? a.bs_c_row * a.ldc + a.bs_c_col : a.ldc * (a.transpose ? a.Cn : a.R);
    const float* cbase = a.C + a.c_row0 * a.ldc + a.c_col0;
    bool ok = (a.beta == 0.f || a.beta == 1.f) && ((uintptr_t)cbase & 15u) == 0 && (a.ldc % 4) == 0 &&
              (bstride % 4) == 0 && !(a.mask != 0 && a.beta == 0.f);
    if (a.C_lo) {
      const float* lbase = a.C_lo + a.c_row0 * a.ldc + a.c_col0;
      ok = ok && a.beta == 0.f && kp.nchunks == 1 && ((uintptr_t)lbase & 15u) == 0;
    }
    if (ok) {
      const int bx = a.transpose ? 32 : 128, by = a.transpose ? 128 : 32;
      const int64_t xd = a.transpose ? a.R : a.Cn, yd = a.transpose ? a.Cn : a.R;
      ok = make_out_map(&maps.c, cbase, xd, yd, a.ldc, a.batch, bstride, bx, by);
      if (ok && a.C_lo)
        ok = make_out_map(&maps.clo, a.C_lo + a.c_row0 * a.ldc + a.c_col0, xd, yd, a.ldc, a.batch, bstride, bx,
                          by);
    }
    kp.epi_tma = ok ? 1 : 0;
    kp.epi_split = (ok && a.C_lo) ? 1 : 0;
  }
  kp.stage_bytes = kp.qslots * kp.slot_bytes + kp.p_rows_max * (int)kRowBytes * split;
  kp.stage_bytes = (kp.stage_bytes + 1023) & ~1023;
  const int budget = 232448 - 1024 - 256 - (kp.epi_tma ? 2 * (int)kStageTileBytes : 0);
  kp.stages = std::min(8, budget / kp.stage_bytes);
  if (kp.stages < 2) return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)kp.stages * kp.stage_bytes + (kp.epi_tma ? 2 * kStageTileBytes : 0) + 256;
  switch (a.op) {
    case OP_F16:
      return launch<OP_F16>(maps, kp, grid, smem, st, false);
    case OP_BF16:
      return launch<OP_BF16>(maps, kp, grid, smem, st, false);
    default:  // only this instantiation waits on the previous kernel
      return launch<OP_TF32X3>(maps, kp, grid, smem, st, a.pdl != 0);
  }
}

}  // namespace gptq
