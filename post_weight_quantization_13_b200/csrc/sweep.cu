// gptq_quantize_layer: the column sweep with error compensation ("gptq"
// glossary page, Algorithm (2) and Key innovation) and group quantization
// ("gptq" agent-skill page, Group-wise quantization), then unpermute and
// bit-packing.
//
// Data flow on the device (all in the caller's workspace):
//   gather_w_kernel  Wp = fp32 working copy of W in processing order (dead
//                    columns zeroed).
//   split_u_kernel   U^T split into tf32 hi + exact fp32 remainder (the
//                    tensor-core operands of the updates).
//   pack_ud_kernel   each 32-column diagonal block of U and 1 / U_jj.
//   solve_kernel     the sweep and all its updates in one cooperative launch
//                    (solve.cu): codes, scales, zeros, loss.
//   pack_kernel      codes back to original column order, g_idx, LSB-first
//                    bit packing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>

#include "internal.cuh"

namespace gptq {
namespace {

constexpr int BW = 128;  // column blocks of the sweep (np is a multiple)

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

}  // namespace

cudaError_t preload_quantize_kernels() {
  const void* fns[] = {(const void*)gather_w_kernel<__half>, (const void*)gather_w_kernel<__nv_bfloat16>,
                       (const void*)gather_w_kernel<float>, (const void*)split_u_kernel,
                       (const void*)invperm_kernel, (const void*)pack_kernel};
  for (const void* f : fns) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, f);
    if (e != cudaSuccess) return e;
  }
  return preload_solve_kernels();
}

namespace {
// The workspace of gptq_quantize_layer, in order.
struct QuantizeWs {
  PrepHeader* hdr;
  float *Wp, *Uh, *Ul, *Eh, *El, *Ud;
  uint8_t* codes_p;
  void* sync;
  int32_t* inv;
  size_t bytes;
};

QuantizeWs quantize_ws(void* ws, int64_t out, int64_t in) {
  const int64_t np_ = round_up(in, BW);
  QuantizeWs w;
  uint8_t* p = (uint8_t*)ws;
  auto take = [&](int64_t bytes) {
    uint8_t* q = p;
    p += round_up(bytes, 256);
    return q;
  };
  w.hdr = (PrepHeader*)take(kHeaderBytes);
  w.Wp = (float*)take(4 * out * np_);
  w.Uh = (float*)take(4 * np_ * np_);
  w.Ul = (float*)take(4 * np_ * np_);
  w.Eh = (float*)take(4 * out * np_);
  w.El = (float*)take(4 * out * np_);
  w.codes_p = take(out * np_);
  w.Ud = (float*)take((int64_t)solve_ud_bytes(np_));
  w.sync = take((int64_t)solve_sync_bytes(out, np_));
  w.inv = (int32_t*)take(4 * in);
  w.bytes = (size_t)(p - (uint8_t*)ws);
  return w;
}
}  // namespace

size_t quantize_ws_bytes(int64_t out, int64_t in, const gptq_config_t*) { return quantize_ws(nullptr, out, in).bytes; }

gptq_status_t quantize_layer(const void* W, gptq_dtype_t wt, int64_t out, int64_t in, int64_t ldw, const float* U,
                             const int32_t* perm, const uint8_t* dead, const gptq_config_t* cfg, int32_t* codes,
                             uint32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx, float* loss, void* ws,
                             size_t ws_bytes, cudaStream_t st) {
  const DeviceInfo& dev = device_info();
  const int64_t np_ = round_up(in, BW);
  const QuantizeWs w = quantize_ws(ws, out, in);
  (void)ws_bytes;
  CUDA_TRY(cudaMemsetAsync(w.hdr, 0, kHeaderBytes, st));
  if (loss) CUDA_TRY(cudaMemsetAsync(loss, 0, sizeof(float) * out, st));
  {
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(out, (int64_t)dev.sms * 8));
    switch (wt) {
      case GPTQ_F16:
        gather_w_kernel<__half><<<grid, 256, 0, st>>>((const __half*)W, ldw, out, in, np_, perm, dead, w.Wp);
        break;
      case GPTQ_BF16:
        gather_w_kernel<__nv_bfloat16>
            <<<grid, 256, 0, st>>>((const __nv_bfloat16*)W, ldw, out, in, np_, perm, dead, w.Wp);
        break;
      default:
        gather_w_kernel<float><<<grid, 256, 0, st>>>((const float*)W, ldw, out, in, np_, perm, dead, w.Wp);
        break;
    }
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  {
    const unsigned grid = (unsigned)std::min<int64_t>(np_, (int64_t)dev.sms * 8);
    split_u_kernel<<<grid, 256, 0, st>>>(U, in, np_, w.Uh, w.Ul);
    note_launch();
    CUDA_TRY(cudaGetLastError());
    CUDA_TRY(solve_pack_ud(U, in, np_, w.Ud, st));
  }
  CUDA_TRY(solve_quantize(w.Wp, out, in, np_, w.Uh, w.Ul, w.Ud, w.Eh, w.El, cfg, scales, zeros, w.codes_p, loss,
                          w.sync, &w.hdr->status, dev.sms, st));
  invperm_kernel<<<(unsigned)((in + 255) / 256), 256, 0, st>>>(perm, in, cfg->group_size, w.inv, g_idx);
  note_launch();
  CUDA_TRY(cudaGetLastError());
  if (qweight || codes) {
    const unsigned grid = (unsigned)std::min<int64_t>(out, (int64_t)dev.sms * 8);
    pack_kernel<<<grid, 256, (size_t)np_, st>>>(w.codes_p, np_, out, in, cfg->bits, w.inv, qweight, codes);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  return GPTQ_OK;
}

}  // namespace gptq
