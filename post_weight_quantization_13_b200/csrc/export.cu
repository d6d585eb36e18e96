// gptq_export_checkpoint: the solver's row-major outputs rewritten in the
// input-dimension-major checkpoint layout that the GPTQ loaders read (the
// format the "AutoGPTQ" artifact page, "Why AutoGPTQ Matters", says
// ExLlamaV2 and vLLM load; the pages print no bit layout, so the layout is
// the reading stated in gptq.h):
//
//   qweight_t [in*bits/32][out]  the transpose of qweight: both hold each
//                                row's codes as one LSB-first stream along
//                                the input dimension, so word (j, o) of the
//                                checkpoint is word (o, j) of the solver.
//   qzeros    [ngroups][out*bits/32]  (zeros[o][g] - zero_offset) mod
//                                2^bits as an LSB-first stream along o.
//   scales_h  [ngroups][out]     scales^T rounded to float16.
//
// All three are memory-bound rewrites: 32 x 32 tiles through shared memory
// (coalesced reads and writes) for the two transposes, one output word per
// thread for the zeros.
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.cuh"

namespace gptq {
namespace {

constexpr int TT = 32;  // transpose tile edge; blocks of 32 x 8 threads

struct KeepWord {
  __device__ __forceinline__ uint32_t operator()(uint32_t v) const { return v; }
};
struct ToHalfBits {
  __device__ __forceinline__ uint16_t operator()(float v) const { return __half_as_ushort(__float2half_rn(v)); }
};

// dst[c][r] = cvt(src[r][c]) for a rows x cols row-major source.  Block
// (bx, by) moves the tile of rows [32 bx, 32 bx + 32) and columns
// [32 by, 32 by + 32); the shared tile is padded to 33 columns so that the
// column-wise reads of the write phase hit 32 different banks.
template <typename Tin, typename Tout, typename Cvt>
__global__ void __launch_bounds__(256) transpose_kernel(const Tin* __restrict__ src, int64_t rows, int64_t cols,
                                                        Tout* __restrict__ dst, Cvt cvt) {
  __shared__ Tin tile[TT][TT + 1];
  const int64_t r0 = (int64_t)blockIdx.x * TT, c0 = (int64_t)blockIdx.y * TT;
  const int tx = threadIdx.x;
  for (int i = threadIdx.y; i < TT; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + tx;
    if (r < rows && c < cols) tile[i][tx] = __ldg(src + r * cols + c);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < TT; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + tx;
    if (c < cols && r < rows) dst[c * rows + r] = cvt(tile[tx][i]);
  }
}

// qzeros[g][w] = word w of the LSB-first stream, along the output dimension,
// of the fields (zeros[o][g] - off) & (2^bits - 1).  The fields that touch
// word w start at o = 32 w / bits; the first may begin below bit 32 w (a
// 3-bit field straddling two words), hence the signed shift.
__global__ void __launch_bounds__(256) pack_zeros_kernel(const int32_t* __restrict__ zeros, int64_t out, int ngroups,
                                                         int bits, int off, uint32_t* __restrict__ qzeros) {
  const int64_t nw = out * bits / 32;
  const uint32_t mask = (1u << bits) - 1u;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)ngroups * nw;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = e / nw, w = e % nw;
    const int64_t bit0 = w * 32;
    uint64_t acc = 0;
    for (int64_t o = bit0 / bits; o < out && o * bits < bit0 + 32; ++o) {
      const uint64_t v = (uint32_t)(__ldg(zeros + o * ngroups + g) - off) & mask;
      const int sh = (int)(o * bits - bit0);
      acc |= sh >= 0 ? v << sh : v >> (-sh);
    }
    qzeros[e] = (uint32_t)acc;
  }
}

template <typename Tin, typename Tout, typename Cvt>
cudaError_t launch_transpose(const Tin* src, int64_t rows, int64_t cols, Tout* dst, Cvt cvt, cudaStream_t st) {
  const dim3 grid((unsigned)((rows + TT - 1) / TT), (unsigned)((cols + TT - 1) / TT));
  transpose_kernel<<<grid, dim3(TT, 8), 0, st>>>(src, rows, cols, dst, cvt);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

gptq_status_t export_checkpoint(const uint32_t* qweight, const float* scales, const int32_t* zeros, int64_t out,
                                int64_t in, int bits, int ngroups, int zero_offset, uint32_t* qweight_t,
                                uint32_t* qzeros, uint16_t* scales_h, cudaStream_t st) {
  if (qweight_t) CUDA_TRY(launch_transpose(qweight, out, in * bits / 32, qweight_t, KeepWord(), st));
  if (scales_h) CUDA_TRY(launch_transpose(scales, out, (int64_t)ngroups, scales_h, ToHalfBits(), st));
  if (qzeros) {
    const DeviceInfo& dev = device_info();
    const int64_t words = (int64_t)ngroups * (out * bits / 32);
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((words + 255) / 256, (int64_t)dev.sms * 8));
    pack_zeros_kernel<<<grid, 256, 0, st>>>(zeros, out, ngroups, bits, zero_offset, qzeros);
    note_launch();
    CUDA_TRY(cudaGetLastError());
  }
  return GPTQ_OK;
}

}  // namespace gptq
