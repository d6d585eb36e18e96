// gptq_dequantize_layer: packed codes back to floating-point weights,
// deq[r][c] = scale[r][g] (code[r][c] - zero[r][g]) with g = g_idx[c] (the
// group quantizer's inverse, "gptq" agent-skill page, Group-wise
// quantization).  Memory-bound: each thread turns eight consecutive codes of
// one row into eight output values (one 16-byte store for 16-bit outputs).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "gemm.cuh"
#include "internal.cuh"

namespace gptq {
namespace {

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T>
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ qweight, const float* __restrict__ scales,
                                                      const int32_t* __restrict__ zeros, const int32_t* __restrict__ g_idx,
                                                      int64_t out, int64_t in, int bits, int ngroups, T* __restrict__ Wq,
                                                      int64_t ldw, bool vec) {
  const int64_t words = in * bits / 32;  // per row
  const int64_t oct = in / 8;            // groups of eight columns per row
  const uint32_t mask = (1u << bits) - 1u;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < out * oct;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / oct, c0 = (e % oct) * 8;
    const uint32_t* q = qweight + r * words;
    const int64_t bit0 = c0 * bits;
    const int64_t w0 = bit0 >> 5;
    const int sh = (int)(bit0 & 31);
    // eight fields start at a multiple of 8 * bits, so they lie within the
    // 64 bits from word w0 (shift <= 24 for 3-bit fields, 0 otherwise)
    uint64_t v = __ldg(q + w0);
    if (w0 + 1 < words) v |= (uint64_t)__ldg(q + w0 + 1) << 32;
    v >>= sh;
    // the group map is shared by every row and a row's scales and zeros by
    // its columns: read-only loads that stay in L1
    const int4 ga = __ldg(reinterpret_cast<const int4*>(g_idx + c0));
    const int4 gb = __ldg(reinterpret_cast<const int4*>(g_idx + c0 + 4));
    const int gs[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const float* srow = scales + r * ngroups;
    const int32_t* zrow = zeros + r * ngroups;
    T o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int code = (int)((v >> (u * bits)) & mask);
      const float s = __ldg(srow + gs[u]);
      const float z = (float)__ldg(zrow + gs[u]);
      o[u] = from_f32<T>(s * ((float)code - z));
    }
    T* dst = Wq + r * ldw + c0;
    if (vec) {
      if (sizeof(T) == 2) {
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(o);
      } else {
        reinterpret_cast<float4*>(dst)[0] = *reinterpret_cast<const float4*>(o);
        reinterpret_cast<float4*>(dst)[1] = *reinterpret_cast<const float4*>(o + 4);
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[u] = o[u];
    }
  }
}

}  // namespace

gptq_status_t dequantize_layer(const uint32_t* qweight, const float* scales, const int32_t* zeros,
                               const int32_t* g_idx, int64_t out, int64_t in, int bits, int ngroups, void* Wq,
                               gptq_dtype_t wt, int64_t ldw, cudaStream_t st) {
  const DeviceInfo& dev = device_info();
  const int es = wt == GPTQ_F32 ? 4 : 2;
  const bool vec = ((uintptr_t)Wq % 16 == 0) && ((ldw * es) % 16 == 0);
  const int64_t work = out * (in / 8);
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, (int64_t)dev.sms * 16));
  switch (wt) {
    case GPTQ_F16:
      dequant_kernel<__half><<<grid, 256, 0, st>>>(qweight, scales, zeros, g_idx, out, in, bits, ngroups,
                                                   (__half*)Wq, ldw, vec);
      break;
    case GPTQ_BF16:
      dequant_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(qweight, scales, zeros, g_idx, out, in, bits, ngroups,
                                                          (__nv_bfloat16*)Wq, ldw, vec);
      break;
    default:
      dequant_kernel<float><<<grid, 256, 0, st>>>(qweight, scales, zeros, g_idx, out, in, bits, ngroups,
                                                  (float*)Wq, ldw, vec);
      break;
  }
  note_launch();
  CUDA_TRY(cudaGetLastError());
  return GPTQ_OK;
}

}  // namespace gptq
