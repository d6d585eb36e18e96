// gptq_quantize_layer: the column sweep with error compensation ("gptq"
// glossary page, Algorithm (2) and Key innovation) and group quantization
// ("gptq" agent-skill page, Group-wise quantization), then unpermute and
// bit-packing.
//
// Data flow on the device (all in the caller's workspace):
//   Wp   fp32 working copy of W in processing order (dead columns zeroed).
//   U    split into tf32 hi + fp32 remainder for the tensor-core updates.
//   for each 128-column block k:
//     sweep_kernel   rows in parallel; the block's columns in registers
//                    (4 lanes per row, interleaved columns), U's diagonal
//                    block in shared memory.  For each column: group
//                    parameters at a group start, code, error
//                    e = (w - deq) / U_jj, eager update of the block's later
//                    columns.  Writes codes, scales, zeros, and E (split).
//     tc_gemm        lazy update of later columns, W -= E U_blk (3xTF32).
//   pack_kernel      codes back to original column order, g_idx, LSB-first
//                    bit packing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {
namespace {

constexpr int BW = 128;          // columns per sweep block
constexpr int ROWS = 16;         // rows per sweep CTA (4 lanes per row)
constexpr int NT = ROWS * 4;     // threads per sweep CTA
constexpr int UPITCH = 36;       // floats per (j, lane) slice of U in smem
constexpr int EPITCH = BW + 1;
constexpr int CPITCH = BW + 4;   // bytes per row of staged codes (no bank conflicts)
// interleaved diagonal block of U (BW x 4 x UPITCH floats) followed by 1/U_jj
constexpr uint32_t kDiagBlockFloats = BW * 4 * UPITCH + BW;
constexpr uint32_t kDiagBlockBytes = kDiagBlockFloats * 4;

struct SweepParams {
  const float* Wp;
  int64_t ldw;  // = np_
  int64_t out, in;
  int64_t kB;    // first processing column of this block
  int ncols;     // columns of this block that exist (<= 128)
  const float* Uh;
  const float* Ul;
  int64_t ldu;
  int maxq;
  int sym;
  int gs;         // group size (-1: one group per row)
  int ngroups;
  int gstart0;    // GSB == 128: a group starts at column 0 of this block
  int gbeyond;    // GSB == 128: group columns past this block (read from Wp)
  float* scales;
  int32_t* zeros;
  uint8_t* codes_p;
  float* Eh;
  float* El;
  int64_t lde;
  int64_t e_col0;
  float* loss;
  const float* Ud;   // this block's interleaved U tile and 1/U_jj (pack_diag_kernel)
  uint32_t* status;
};

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

// One sweep block of BW = 128 processed columns.  Each row is handled by 4
// lanes; lane q of a row holds the block's columns 4m + q (m = 0..31) in
// registers w[].  The 128 columns are processed in 8 passes of 16; after a
// pass the register window slides by 4 (w[k] <- w[k+4]), so the code of one
// pass serves all passes (compact code, and the element being quantized is
// always at a compile-time register index).
template <int GSB>
__global__ void __launch_bounds__(NT) sweep_kernel(const SweepParams sp) {
  extern __shared__ __align__(16) float smf[];
  float* Us = smf;                                 // [128 j][4 q][UPITCH]: U[kB+j][kB+4m+q] at m
  float* rd = Us + BW * 4 * UPITCH;                // [128] 1 / U_jj
  float* Esh = rd + BW;                            // [ROWS][EPITCH]
  float* Esl = Esh + ROWS * EPITCH;                // [ROWS][EPITCH]
  uint8_t* Cs = reinterpret_cast<uint8_t*>(Esl + ROWS * EPITCH);  // [ROWS][CPITCH]
  const int tid = threadIdx.x;
  __shared__ uint64_t ubar;
  // U's diagonal block, already laid out for this kernel by pack_diag_kernel:
  // one bulk copy of the interleaved block and the reciprocal diagonal.
  if (tid == 0) {
    mbar_init(&ubar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&ubar, kDiagBlockBytes);
    bulk_load(Us, sp.Ud, kDiagBlockBytes, &ubar);
  }
  for (int e = tid; e < ROWS * EPITCH; e += NT) {
    Esh[e] = 0.f;
    Esl[e] = 0.f;
  }
  // U's diagonal blocks were written before the first sweep of the layer,
  // which is an ordinary launch; W, the scales and E come from the kernels
  // just before this one, so a dependent launch waits here for them
  grid_dependency_wait();
  const int warp = tid >> 5, lane = tid & 31;
  const int rl = warp * 8 + (lane >> 2);
  const int q = lane & 3;
  const int64_t row = (int64_t)blockIdx.x * ROWS + rl;
  const bool live = row < sp.out;
  float w[32];
  {
    const float* src = sp.Wp + row * sp.ldw + sp.kB;
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = live ? src[4 * i + q] : 0.f;
  }
  const float fmaxq = (float)sp.maxq;
  float s = 1.f, z = 0.f, inv_s = 1.f, lsum = 0.f;
  if (!mbar_wait(&ubar, 0)) raise_status(sp.status, ST_TIMEOUT);
  // a group that started in an earlier block keeps that block's scale/zero
  if (GSB == BW && !sp.gstart0 && live) {
    const int64_t g = sp.gs == -1 ? 0 : sp.kB / sp.gs;
    s = sp.scales[row * sp.ngroups + g];
    z = (float)sp.zeros[row * sp.ngroups + g];
  }
  inv_s = __frcp_rn(s);
  __syncthreads();
  for (int mo = 0; mo < 32; mo += 4) {  // pass: columns 4*mo .. 4*mo + 15
    if (4 * mo >= sp.ncols) break;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
      const int cbase = 4 * (mo + mi);
      if (cbase >= sp.ncols) break;
      const bool gstart = (GSB < BW) ? (cbase % GSB == 0) : (cbase == 0 && sp.gstart0);
      if (gstart) {
        float lo = INFINITY, hi = -INFINITY, am = 0.f;
#pragma unroll
        for (int k = mi; k < 32; ++k) {
          bool in_group;
          if (GSB < BW)
            in_group = k < mi + GSB / 4;
          else
            in_group = 4 * k + q < sp.ncols;  // pass 0: element k is column 4k + q
          if (in_group) {
            lo = fminf(lo, w[k]);
            hi = fmaxf(hi, w[k]);
            am = fmaxf(am, fabsf(w[k]));
          }
        }
        if (GSB == BW && sp.gbeyond > 0 && live) {
          const float* src = sp.Wp + row * sp.ldw + sp.kB + BW;
          for (int ci = q; ci < sp.gbeyond; ci += 4) {
            const float v = src[ci];
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
            am = fmaxf(am, fabsf(v));
          }
        }
#pragma unroll
        for (int m = 1; m <= 2; m <<= 1) {
          lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, m));
          hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, m));
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, m));
        }
        group_params(lo, hi, am, sp.sym, fmaxq, s, z);
        inv_s = __frcp_rn(s);
        if (q == 0 && live) {
          const int64_t g = sp.gs == -1 ? 0 : (sp.kB + cbase) / sp.gs;
          sp.scales[row * sp.ngroups + g] = s;
          sp.zeros[row * sp.ngroups + g] = (int32_t)z;
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int j = cbase + t;
        if (j >= sp.ncols) break;
        float e = 0.f;
        if (q == t) {
          const float x = w[mi];
          float qf = round_div(x, s, inv_s) + z;
          qf = fminf(fmaxf(qf, 0.f), fmaxq);
          const float deq = s * (qf - z);
          e = (x - deq) * rd[j];
          lsum = fmaf(e, e, lsum);
          Cs[rl * CPITCH + j] = (uint8_t)qf;
          float eh, el;
          split_tf32(e, eh, el);
          Esh[rl * EPITCH + j] = eh;
          Esl[rl * EPITCH + j] = el;
        }
        e = __shfl_sync(0xffffffffu, e, (lane & ~3) | t);
        // w[k] is column 4(mo + k) + q; its U entry is Us[j][q][mo + k]
        const float* urow = Us + (j * 4 + q) * UPITCH + mo;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const float4 u = *reinterpret_cast<const float4*>(urow + 4 * a);
          if (4 * a + 0 >= mi) w[4 * a + 0] = fmaf(-e, u.x, w[4 * a + 0]);
          if (4 * a + 1 >= mi) w[4 * a + 1] = fmaf(-e, u.y, w[4 * a + 1]);
          if (4 * a + 2 >= mi) w[4 * a + 2] = fmaf(-e, u.z, w[4 * a + 2]);
          if (4 * a + 3 >= mi) w[4 * a + 3] = fmaf(-e, u.w, w[4 * a + 3]);
        }
      }
    }
    // slide the register window by one pass
#pragma unroll
    for (int k = 0; k < 28; ++k) w[k] = w[k + 4];
#pragma unroll
    for (int k = 28; k < 32; ++k) w[k] = 0.f;
  }
  float l = lsum;
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (q == 0 && live && sp.loss) sp.loss[row] += l;
  __syncthreads();
  for (int e = tid; e < ROWS * BW; e += NT) {
    const int r = e / BW, c = e % BW;
    const int64_t gr = (int64_t)blockIdx.x * ROWS + r;
    if (gr >= sp.out) continue;
    sp.Eh[gr * sp.lde + sp.e_col0 + c] = Esh[r * EPITCH + c];
    sp.El[gr * sp.lde + sp.e_col0 + c] = Esl[r * EPITCH + c];
    if (c < sp.ncols) sp.codes_p[gr * sp.ldw + sp.kB + c] = Cs[r * CPITCH + c];
  }
}

// For every 128-column block k: Ud[k] = U's diagonal block in the sweep
// kernel's layout, Us[j][c % 4][c / 4] = U[kB+j][kB+c] (= Ucm[kB+c][kB+j]),
// then 1/U_jj.  One CTA per block.
__global__ void __launch_bounds__(256) pack_diag_kernel(const float* __restrict__ U, int64_t in,
                                                        float* __restrict__ Ud) {
  // blockIdx.x = diagonal block, blockIdx.y = which 16 of its 128 rows (c)
  const int64_t kB = (int64_t)blockIdx.x * BW;
  const int ncols = (int)((in - kB) < BW ? (in - kB) : BW);
  float* dst = Ud + (int64_t)blockIdx.x * kDiagBlockFloats;
  const int c0 = blockIdx.y * 16;
  if (blockIdx.y == 0)  // the pitch padding of every (j, q) slice
    for (int e = threadIdx.x; e < BW * 4 * (UPITCH - BW / 4); e += blockDim.x)
      dst[(e / (UPITCH - BW / 4)) * UPITCH + BW / 4 + e % (UPITCH - BW / 4)] = 0.f;
  for (int e = threadIdx.x; e < 16 * BW; e += blockDim.x) {
    const int c = c0 + e / BW, j = e % BW;
    float v = 0.f;
    if (c < ncols && j < ncols) v = U[(kB + c) * in + kB + j];
    dst[(j * 4 + (c & 3)) * UPITCH + (c >> 2)] = v;
    if (c == j) dst[BW * 4 * UPITCH + j] = (c < ncols) ? 1.f / v : 0.f;
  }
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Wp[r][p] = W[r][perm[p]] in fp32 (0 for dead columns and the padding):
// whole rows per block, four processed columns per thread.
template <typename T>
__global__ void __launch_bounds__(256) gather_w_kernel(const T* __restrict__ W, int64_t ldw_in, int64_t out,
                                                       int64_t in, int64_t np_, const int32_t* __restrict__ perm,
                                                       const uint8_t* __restrict__ dead, float* __restrict__ Wp) {
  const int n = (int)in, np = (int)np_;
  for (int64_t r = blockIdx.x; r < out; r += gridDim.x) {
    const T* Wr = W + r * ldw_in;
    float* dst = Wp + r * np_;
    for (int p = threadIdx.x * 4; p < np; p += blockDim.x * 4) {
      float v[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[t] = 0.f;
        if (p + t < n) {
          const int c = __ldg(perm + p + t);
          if (!__ldg(dead + c)) v[t] = to_f32(Wr[c]);
        }
      }
      *reinterpret_cast<float4*>(dst + p) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

// Uh/Ul[c][j] = split(Ucm[c][j]) with the padding zero.
__global__ void __launch_bounds__(256) split_u_kernel(const float* __restrict__ U, int64_t in, int64_t np_,
                                                      float* __restrict__ Uh, float* __restrict__ Ul) {
  // four columns per thread; U rows are float4-aligned when in % 4 == 0
  const bool vec = (in & 3) == 0;
  for (int64_t c = blockIdx.x; c < np_; c += gridDim.x) {
    for (int64_t j = (int64_t)threadIdx.x * 4; j < np_; j += (int64_t)blockDim.x * 4) {
      float v[4];
      if (vec && c < in && j + 3 < in) {
        const float4 u = *reinterpret_cast<const float4*>(U + c * in + j);
        v[0] = u.x, v[1] = u.y, v[2] = u.z, v[3] = u.w;
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) v[t] = (c < in && j + t < in) ? U[c * in + j + t] : 0.f;
      }
      float4 h, l;
      split_tf32(v[0], h.x, l.x);
      split_tf32(v[1], h.y, l.y);
      split_tf32(v[2], h.z, l.z);
      split_tf32(v[3], h.w, l.w);
      *reinterpret_cast<float4*>(Uh + c * np_ + j) = h;
      *reinterpret_cast<float4*>(Ul + c * np_ + j) = l;
    }
  }
}

__global__ void invperm_kernel(const int32_t* __restrict__ perm, int64_t in, int gs, int32_t* __restrict__ inv,
                               int32_t* __restrict__ g_idx) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p < in) {
    const int32_t c = perm[p];
    inv[c] = (int32_t)p;
    g_idx[c] = gs == -1 ? 0 : (int32_t)(p / gs);
  }
}

// One thread per packed word: gathers the (at most 32/bits + 1) codes whose
// fields overlap it, in original column order.  Also writes the unpacked
// int32 codes when requested (each column exactly once, by the word holding
// its first bit).
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t* __restrict__ codes_p, int64_t ldc_p, int64_t out,
                                                   int64_t in, int bits, const int32_t* __restrict__ inv,
                                                   uint32_t* __restrict__ qweight, int32_t* __restrict__ codes) {
  // one row at a time per block: the row's codes (processing order) are
  // staged in shared memory with 16-byte loads, then gathered into original
  // column order through inv (read-only, shared by all rows)
  extern __shared__ __align__(16) uint8_t srow[];
  const int64_t nwords = (in * bits + 31) / 32;
  for (int64_t r = blockIdx.x; r < out; r += gridDim.x) {
    __syncthreads();
    for (int64_t e = (int64_t)threadIdx.x * 16; e < ldc_p; e += (int64_t)blockDim.x * 16)
      *reinterpret_cast<uint4*>(srow + e) = *reinterpret_cast<const uint4*>(codes_p + r * ldc_p + e);
    __syncthreads();
    if (qweight) {
      const int nw = (int)nwords, n_in = (int)in;
      uint32_t* qrow = qweight + r * nwords;
      if (32 % bits == 0) {
        // 2, 4 and 8 bits: each word holds 32 / bits whole fields
        const int per = 32 / bits;
        for (int w = threadIdx.x; w < nw; w += blockDim.x) {
          uint32_t acc = 0;
          for (int u = 0; u < per; ++u) acc |= (uint32_t)srow[__ldg(inv + w * per + u)] << (u * bits);
          qrow[w] = acc;
        }
      } else {
        // 3 bits: fields may straddle words
        for (int w = threadIdx.x; w < nw; w += blockDim.x) {
          const int bit0 = w * 32;
          uint64_t acc = 0;
          for (int c = bit0 / bits; c < n_in && c * bits < bit0 + 32; ++c) {
            const uint32_t v = srow[__ldg(inv + c)];
            const int off = c * bits - bit0;  // negative for the field straddling in
            acc |= off >= 0 ? (uint64_t)v << off : (uint64_t)v >> (-off);
          }
          qrow[w] = (uint32_t)acc;
        }
      }
    }
    if (codes)
      for (int64_t c = threadIdx.x; c < in; c += blockDim.x) codes[r * in + c] = (int32_t)srow[__ldg(inv + c)];
  }
}

cudaError_t run_gemm(GemmArgs& g, cudaStream_t st, int sms) {
  if (!force_simt() && tc_gemm_supported(g)) return tc_gemm(g, st, sms);
  return simt_gemm(g, st);
}

// pdl: programmatic dependent launch.  Only for a sweep that follows a
// kernel of the same layer's sweep chain (a lazy update): its bulk copy of
// U's diagonal block is issued before it waits on that kernel.
template <int GSB>
cudaError_t launch_sweep(const SweepParams& sp, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)(BW * 4 * UPITCH + BW + 2 * ROWS * EPITCH) * sizeof(float) + ROWS * CPITCH;
  cudaError_t ce = ensure_smem_limit((const void*)sweep_kernel<GSB>, (int)smem);
  if (ce != cudaSuccess) return ce;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((sp.out + ROWS - 1) / ROWS));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  ce = cudaLaunchKernelEx(&cfg, sweep_kernel<GSB>, sp);
  note_launch();
  return ce != cudaSuccess ? ce : cudaGetLastError();
}

}  // namespace

cudaError_t preload_quantize_kernels() {
  const void* fns[] = {
      (const void*)sweep_kernel<8>,   (const void*)sweep_kernel<16>, (const void*)sweep_kernel<32>,
      (const void*)sweep_kernel<64>,  (const void*)sweep_kernel<128>, (const void*)pack_diag_kernel,
      (const void*)gather_w_kernel<__half>, (const void*)gather_w_kernel<__nv_bfloat16>,
      (const void*)gather_w_kernel<float>,  (const void*)split_u_kernel, (const void*)invperm_kernel,
      (const void*)pack_kernel};
  for (const void* f : fns) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, f);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int64_t outer_block(const gptq_config_t* cfg) {
  const int64_t gs = cfg->group_size;
  int64_t bo = std::min<int64_t>(cfg->block_size, 1024) / 128 * 128;
  for (; bo > 128; bo -= 128) {
    if (gs == -1 || gs % bo == 0 || bo % gs == 0) break;
  }
  return std::max<int64_t>(bo, 128);
}

size_t quantize_ws_bytes(int64_t out, int64_t in, const gptq_config_t* cfg) {
  const int64_t np_ = round_up(in, BW);
  const int64_t bo = outer_block(cfg);
  size_t b = kHeaderBytes;
  b += round_up(4 * out * np_, 256);       // Wp
  b += 2 * round_up(4 * np_ * np_, 256);   // Uh, Ul
  b += 2 * round_up(4 * out * bo, 256);    // Eh, El
  b += round_up(out * np_, 256);           // codes_p
  b += round_up(4 * (int64_t)kDiagBlockFloats * (np_ / BW), 256);  // interleaved diagonal blocks
  b += round_up(4 * in, 256);              // inverse permutation
  return b;
}

gptq_status_t quantize_layer(const void* W, gptq_dtype_t wt, int64_t out, int64_t in, int64_t ldw, const float* U,
                             const int32_t* perm, const uint8_t* dead, const gptq_config_t* cfg, int32_t* codes,
                             uint32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx, float* loss, void* ws,
                             size_t ws_bytes, cudaStream_t st) {
  const DeviceInfo& dev = device_info();
  const int64_t np_ = round_up(in, BW);
  const int64_t bo = outer_block(cfg);
  uint8_t* p = (uint8_t*)ws;
  PrepHeader* hdr = (PrepHeader*)p;
  p += kHeaderBytes;
  float* Wp = (float*)p;
  p += round_up(4 * out * np_, 256);
  float* Uh = (float*)p;
  p += round_up(4 * np_ * np_, 256);
  float* Ul = (float*)p;
  p += round_up(4 * np_ * np_, 256);
  float* Eh = (float*)p;
  p += round_up(4 * out * bo, 256);
  float* El = (float*)p;
  p += round_up(4 * out * bo, 256);
  uint8_t* codes_p = p;
  p += round_up(out * np_, 256);
  float* Ud = (float*)p;
  p += round_up(4 * (int64_t)kDiagBlockFloats * (np_ / BW), 256);
  int32_t* inv = (int32_t*)p;

  CUDA_TRY(cudaMemsetAsync(hdr, 0, kHeaderBytes, st));
  if (loss) CUDA_TRY(cudaMemsetAsync(loss, 0, sizeof(float) * out, st));
  {
    const unsigned grid = (unsigned)std::min<int64_t>(out, (int64_t)dev.sms * 8);
    switch (wt) {
      case GPTQ_F16:
        gather_w_kernel<__half><<<grid, 256, 0, st>>>((const __half*)W, ldw, out, in, np_, perm, dead, Wp);
        note_launch();
        break;
      case GPTQ_BF16:
        gather_w_kernel<__nv_bfloat16>
            <<<grid, 256, 0, st>>>((const __nv_bfloat16*)W, ldw, out, in, np_, perm, dead, Wp);
            note_launch();
        break;
      default:
        gather_w_kernel<float><<<grid, 256, 0, st>>>((const float*)W, ldw, out, in, np_, perm, dead, Wp);
        note_launch();
        break;
    }
    CUDA_TRY(cudaGetLastError());
  }
  {
    const unsigned grid = (unsigned)std::min<int64_t>(np_, (int64_t)dev.sms * 8);
    split_u_kernel<<<grid, 256, 0, st>>>(U, in, np_, Uh, Ul);
    note_launch();
    CUDA_TRY(cudaGetLastError());
    pack_diag_kernel<<<dim3((unsigned)(np_ / BW), BW / 16), 256, 0, st>>>(U, in, Ud);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  const int gs = cfg->group_size;
  const int ngroups = gs == -1 ? 1 : (int)(in / gs);
  const int gsb = (gs == -1 || gs >= BW) ? BW : gs;
  for (int64_t o0 = 0; o0 < in; o0 += bo) {
    const int64_t o1 = std::min(in, o0 + bo);
    for (int64_t k = o0; k < o1; k += BW) {
      SweepParams sp;
      sp.Wp = Wp;
      sp.ldw = np_;
      sp.out = out;
      sp.in = in;
      sp.kB = k;
      sp.ncols = (int)std::min<int64_t>(BW, in - k);
      sp.Uh = Uh;
      sp.Ul = Ul;
      sp.ldu = np_;
      sp.maxq = (1 << cfg->bits) - 1;
      sp.sym = cfg->sym;
      sp.gs = gs;
      sp.ngroups = ngroups;
      if (gsb == BW) {
        sp.gstart0 = (gs == -1) ? (k == 0) : (k % gs == 0);
        const int64_t gend = (gs == -1) ? in : k + gs;
        sp.gbeyond = sp.gstart0 ? (int)std::max<int64_t>(0, gend - (k + BW)) : 0;
      } else {
        sp.gstart0 = 0;
        sp.gbeyond = 0;
      }
      sp.scales = scales;
      sp.zeros = zeros;
      sp.codes_p = codes_p;
      sp.Eh = Eh;
      sp.El = El;
      sp.lde = bo;
      sp.e_col0 = k - o0;
      sp.loss = loss;
      sp.Ud = Ud + (k / BW) * (int64_t)kDiagBlockFloats;
      sp.status = &hdr->status;
      cudaError_t e;
      switch (gsb) {
        case 8:
          e = launch_sweep<8>(sp, st, k > 0);
          break;
        case 16:
          e = launch_sweep<16>(sp, st, k > 0);
          break;
        case 32:
          e = launch_sweep<32>(sp, st, k > 0);
          break;
        case 64:
          e = launch_sweep<64>(sp, st, k > 0);
          break;
        case 128:
          e = launch_sweep<128>(sp, st, k > 0);
          break;
        default:
          return fail(GPTQ_ERR_UNSUPPORTED, "group_size %d is not supported by the sweep kernel", gs);
      }
      CUDA_TRY(e);
      // inner lazy update: the rest of this outer block
      const int64_t c0 = k + BW;
      if (c0 < o1) {
        GemmArgs g;
        g.op = OP_TF32X3;
        g.P = {Eh, El, out, bo, bo};
        g.Q = {Uh, Ul, np_, np_, np_};
        g.R = out;
        g.Cn = o1 - c0;
        g.K = BW;
        g.p_tile = 128;
        g.pdl = 1;
        g.p_row0 = 0;
        g.p_k0 = k - o0;
        g.q_row0 = c0;
        g.q_k0 = k;
        g.C = Wp;
        g.ldc = np_;
        g.c_row0 = 0;
        g.c_col0 = c0;
        g.alpha = -1.f;
        g.beta = 1.f;
        g.status = &hdr->status;
        CUDA_TRY(run_gemm(g, st, dev.sms));
      }
    }
    // outer lazy update: every later column
    if (o1 < in) {
      GemmArgs g;
      g.op = OP_TF32X3;
      g.P = {Eh, El, out, bo, bo};
      g.Q = {Uh, Ul, np_, np_, np_};
      g.R = out;
      g.Cn = in - o1;
      g.K = o1 - o0;
      g.p_tile = 128;
      g.pdl = 1;
      g.p_row0 = 0;
      g.p_k0 = 0;
      g.q_row0 = o1;
      g.q_k0 = o0;
      g.C = Wp;
      g.ldc = np_;
      g.c_row0 = 0;
      g.c_col0 = o1;
      g.alpha = -1.f;
      g.beta = 1.f;
      g.status = &hdr->status;
      CUDA_TRY(run_gemm(g, st, dev.sms));
    }
  }
  invperm_kernel<<<(unsigned)((in + 255) / 256), 256, 0, st>>>(perm, in, gs, inv, g_idx);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  if (qweight || codes) {
    const unsigned grid = (unsigned)std::min<int64_t>(out, (int64_t)dev.sms * 8);
    pack_kernel<<<grid, 256, (size_t)np_, st>>>(codes_p, np_, out, in, cfg->bits, inv, qweight, codes);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  return GPTQ_OK;
}

}  // namespace gptq
