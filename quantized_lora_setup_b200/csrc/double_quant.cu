// double_quant.cu -- standalone double quantization of an absmax array (aqnf4_double_quant).
//
// "QLoRA", "How It Works": the per-block scales get an 8-bit encoding of their own, worth
// about 0.37 bits per weight; "QLoRA Explained", "Double Quantization".  Each block of
// 256 constants keeps one binary32 scale s = max a and one byte per constant,
// code8 = round_half_even(fl(fl(a / s) * 255)).  The fused pass in quant_score.cu applies
// the same dq_code to the same constants, so both give identical bytes.
//
// HBM-bound and tiny (1/64 of the weights' element count): one CTA of 256 threads per DQ
// block, grid-stride, one coalesced 4-byte load and one byte store per thread.
#include <cfloat>

#include "device.cuh"

namespace aqnf4 {
namespace {

__global__ void __launch_bounds__(256) k_double_quant(const float* __restrict__ absmax, int64_t nb,
                                                      uint8_t* __restrict__ codes8,
                                                      float* __restrict__ scales, int32_t* flag) {
  __shared__ float red[2][8];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t nd = (nb + kDqBlock - 1) / kDqBlock;
  int buf = 0;
  for (int64_t d = blockIdx.x; d < nd; d += gridDim.x, buf ^= 1) {
    const int64_t i = d * kDqBlock + t;
    const bool valid = i < nb;
    const float a = valid ? __ldg(absmax + i) : 0.0f;
    float m = a;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax_nan(m, __shfl_xor_sync(kFull, m, off));
    if (lane == 0) red[buf][warp] = m;
    __syncthreads();  // red[buf] is rewritten two iterations later, after the next barrier
    float s = red[buf][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) s = fmax_nan(s, red[buf][w]);
    if (valid) codes8[i] = dq_code(a, s);
    if (t == 0) {
      scales[d] = s;
      if (!(s <= FLT_MAX) && flag) *flag = AQNF4_ERR_NONFINITE;
    }
  }
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

extern "C" aqnf4_status aqnf4_double_quant(const float* absmax, int64_t nb, uint8_t* codes8,
                                           float* scales, int32_t* dev_flag, cudaStream_t stream) {
  if (!absmax || !codes8 || !scales || nb < 1) return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(absmax, 4) || !is_aligned(scales, 4) || !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  const int64_t nd = (nb + kDqBlock - 1) / kDqBlock;
  const int sms = current_sm_count();
  int64_t grid = static_cast<int64_t>(sms > 0 ? sms : 1) * 8;
  if (grid > nd) grid = nd;
  k_double_quant<<<static_cast<unsigned>(grid), 256, 0, stream>>>(absmax, nb, codes8, scales,
                                                                  dev_flag);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}
