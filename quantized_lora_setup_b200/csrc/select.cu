// select.cu -- top-K layers under a byte budget (aqnf4_select_topk).
//
// arxivdaily 2608.23816, "English abstract": the pass ranks layers by NF4 reconstruction
// error and keeps the top-K in fp16 under a memory budget; "AQLoRA: A Zero-Search Recipe
// for Fast Quantized LoRA Fine-Tuning", "Technical Details": the budget is configurable.
//
// Ranking: score descending, equal scores by lower layer index, NaN scores last.  A model
// has a few hundred layers, so one CTA of 1024 threads computes every layer's rank by
// counting the layers that precede it (O(L^2 / 1024), no sort network, no tie ambiguity),
// scatters the ranking into sel_idx, then runs a block-wide int64 prefix sum of the costs
// in rank order and keeps the ranks before the first one whose prefix exceeds the budget
// or the cap.
#include "device.cuh"

namespace aqnf4 {
namespace {

constexpr int kSelThreads = 1024;

__device__ __forceinline__ bool ranks_before(float ej, int j, float ei, int i) {
  const bool nj = ej != ej, ni = ei != ei;
  if (nj != ni) return ni;  // the number comes first
  if (!nj && ej != ei) return ej > ei;
  return j < i;
}

__device__ __forceinline__ int64_t shfl_up_i64(int64_t v, int d) {
  const uint32_t lo = __shfl_up_sync(kFull, static_cast<uint32_t>(v), d);
  const uint32_t hi = __shfl_up_sync(kFull, static_cast<uint32_t>(static_cast<uint64_t>(v) >> 32), d);
  return static_cast<int64_t>((static_cast<uint64_t>(hi) << 32) | lo);
}

__global__ void __launch_bounds__(kSelThreads) k_select_topk(const float* __restrict__ e,
                                                             const int64_t* __restrict__ cost,
                                                             int L, int64_t budget, int k_cap,
                                                             int32_t* sel, int32_t* k_out) {
  __shared__ int64_t warp_sum[32];
  __shared__ int64_t carry;
  __shared__ int first_out;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  for (int i = t; i < L; i += kSelThreads) {
    const float ei = __ldg(e + i);
    int rank = 0;
    for (int j = 0; j < L; ++j) rank += ranks_before(__ldg(e + j), j, ei, i) ? 1 : 0;
    sel[rank] = i;
  }
  if (t == 0) {
    carry = 0;
    first_out = (k_cap >= 0 && k_cap < L) ? k_cap : L;
  }
  __syncthreads();

  for (int base = 0; base < L; base += kSelThreads) {
    const int r = base + t;
    int64_t v = r < L ? __ldcg(cost + sel[r]) : 0;
    // inclusive warp scan, then across warps
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int64_t u = shfl_up_i64(v, d);
      if (lane >= d) v += u;
    }
    if (lane == 31) warp_sum[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int64_t s = warp_sum[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int64_t u = shfl_up_i64(s, d);
        if (lane >= d) s += u;
      }
      warp_sum[lane] = s;  // inclusive prefix of warp totals
    }
    __syncthreads();
    const int64_t prefix = carry + v + (warp > 0 ? warp_sum[warp - 1] : 0);
    if (r < L && prefix > budget) atomicMin(&first_out, r);
    __syncthreads();
    if (t == 0) carry += warp_sum[31];
    __syncthreads();
  }
  if (t == 0) *k_out = first_out;
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

extern "C" aqnf4_status aqnf4_select_topk(const float* rel_err, const int64_t* cost_bytes,
                                          int32_t L, int64_t budget_bytes, int32_t k_cap,
                                          int32_t* sel_idx, int32_t* k_out, cudaStream_t stream) {
  if (!rel_err || !cost_bytes || !sel_idx || !k_out || L < 1 || budget_bytes < 0)
    return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(rel_err, 4) || !is_aligned(cost_bytes, 8) || !is_aligned(sel_idx, 4) ||
      !is_aligned(k_out, 4))
    return AQNF4_ERR_ALIGNMENT;
  k_select_topk<<<1, kSelThreads, 0, stream>>>(rel_err, cost_bytes, L, budget_bytes, k_cap,
                                               sel_idx, k_out);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}
