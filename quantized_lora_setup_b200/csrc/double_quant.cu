// double_quant.cu -- standalone double quantization of an absmax array (aqnf4_double_quant).
//
// "QLoRA", "How It Works": the per-block scales get an 8-bit encoding of their own, worth
// about 0.37 bits per weight; "QLoRA Explained", "Double Quantization".  Each block of
// 256 constants keeps one binary32 scale s = max a and one byte per constant,
// code8 = round_half_even(fl(fl(a / s) * 255)).  The fused pass in quant_score.cu applies
// the same dq_code to the same constants, so both give identical bytes.
//
// HBM-bound and tiny (1/64 of the weights' element count): one CTA of 256 threads per DQ
// block, grid-stride, one coalesced 4-byte load and one byte store per thread.  The
// mean-centred variant below takes one warp per DQ block.
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

// Mean-centred double quantization (aqnf4_double_quant_centered), a second format that
// the pages do not define (they give only the 0.37-bit saving): per block of 256 constants
// the mean mu, h = max |a - mu|, and code8 = rint(fl(fl((a - mu) / h) * 127)) + 128.  The
// mean is fl32(fl64(S / len)) with S the binary64 sum over a balanced binary tree of the
// 256 slots in index order (missing slots of a short last block hold +0).  One warp per
// block: lane l holds slots 8l .. 8l + 7 and adds them as the tree's three lowest levels;
// the xor butterfly over lanes 1, 2, 4, 8, 16 then forms the remaining five levels, each
// pair sum being the same in both lanes since binary64 addition is commutative.
__global__ void __launch_bounds__(256) k_double_quant_centered(const float* __restrict__ absmax,
                                                               int64_t nb,
                                                               uint8_t* __restrict__ codes8,
                                                               float* __restrict__ scales,
                                                               float* __restrict__ means,
                                                               int32_t* flag) {
  const int lane = threadIdx.x & 31;
  const int64_t nd = (nb + kDqBlock - 1) / kDqBlock;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t d = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; d < nd;
       d += nwarps) {
    const int64_t i0 = d * kDqBlock + 8 * lane;
    float a[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = i0 + j < nb ? __ldg(absmax + i0 + j) : 0.0f;
    double s = ((static_cast<double>(a[0]) + a[1]) + (static_cast<double>(a[2]) + a[3])) +
               ((static_cast<double>(a[4]) + a[5]) + (static_cast<double>(a[6]) + a[7]));
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) s = __dadd_rn(s, __shfl_xor_sync(kFull, s, off));
    const int64_t rem = nb - d * kDqBlock;
    const int len = rem < kDqBlock ? static_cast<int>(rem) : kDqBlock;
    const float mu = __double2float_rn(__ddiv_rn(s, static_cast<double>(len)));
    float h = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i0 + j < nb) h = fmax_nan(h, fabsf(__fsub_rn(a[j], mu)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) h = fmax_nan(h, __shfl_xor_sync(kFull, h, off));
    const bool finite = (fabsf(mu) <= FLT_MAX) && (h <= FLT_MAX);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (i0 + j >= nb) break;
      uint8_t c = 0;
      if (finite) {
        c = 128;
        if (h != 0.0f) {
          const float t = __fdiv_rn(__fsub_rn(a[j], mu), h);
          c = static_cast<uint8_t>(__float2int_rn(__fmul_rn(t, 127.0f)) + 128);
        }
      }
      codes8[i0 + j] = c;
    }
    if (lane == 0) {
      scales[d] = h;
      means[d] = mu;
      if (!finite && flag) *flag = AQNF4_ERR_NONFINITE;
    }
  }
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

extern "C" aqnf4_status aqnf4_double_quant_centered(const float* absmax, int64_t nb,
                                                    uint8_t* codes8, float* scales, float* means,
                                                    int32_t* dev_flag, cudaStream_t stream) {
  if (!absmax || !codes8 || !scales || !means || nb < 1) return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(absmax, 4) || !is_aligned(scales, 4) || !is_aligned(means, 4) ||
      !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  const int64_t nd = (nb + kDqBlock - 1) / kDqBlock;
  const int sms = current_sm_count();
  int64_t grid = static_cast<int64_t>(sms > 0 ? sms : 1) * 8;  // 8 warps (blocks) per CTA
  const int64_t need = (nd + 7) / 8;
  if (grid > need) grid = need;
  k_double_quant_centered<<<static_cast<unsigned>(grid), 256, 0, stream>>>(absmax, nb, codes8,
                                                                           scales, means, dev_flag);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}

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
