// select.cu -- top-K layers under a byte budget (aqnf4_select_topk) and the block-level
// selection of the speed setting (aqnf4_select_blocks).
//
// arxivdaily 2608.23816, "English abstract": the layers are ordered by their NF4 error and
// the highest-error ones stay in 16 bits while a byte budget allows; "AQLoRA: A Zero-Search
// Recipe for Fast Quantized LoRA Fine-Tuning", "Technical Details": the budget is a setting.
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

// Block-level selection ("English abstract": a speed setting adapts only the top blocks, so
// the backward pass stops early).  One CTA: each thread owns blocks b = t, t + 1024, ... and
// sums its layers in layer order in binary64 (the same order as any other caller, so the
// scores are reproducible to the bit); the ranking is the count of blocks ranked before
// each block; one thread then walks the ranking against the budget.
constexpr int kMaxBlocks = 2048;

__global__ void __launch_bounds__(kSelThreads) k_select_blocks(
    const double* __restrict__ sq_err, const double* __restrict__ sq_w,
    const int32_t* __restrict__ block_of, const int64_t* __restrict__ cost, int L, int B,
    int64_t budget, int order, int32_t* block_rank, float* block_err, int32_t* k_out,
    int32_t* flag) {
  __shared__ float s_err[kMaxBlocks];
  __shared__ int64_t s_cost[kMaxBlocks];
  __shared__ int bad;
  const int t = threadIdx.x;
  if (t == 0) bad = 0;
  __syncthreads();
  for (int b = t; b < B; b += kSelThreads) {
    double se = 0.0, sw = 0.0;
    int64_t c = 0;
    for (int l = 0; l < L; ++l) {
      const int32_t bl = __ldg(block_of + l);
      if (bl < 0 || bl >= B) bad = 1;
      if (bl != b) continue;
      se += __ldg(sq_err + l);
      sw += __ldg(sq_w + l);
      c += __ldg(cost + l);
    }
    double e = sw == 0.0 ? 0.0 : sqrt(se / sw);
    if (se != se || sw != sw) e = __longlong_as_double(0x7ff8000000000000ll);
    s_err[b] = __double2float_rn(e);
    s_cost[b] = c;
    if (block_err) block_err[b] = s_err[b];
  }
  __syncthreads();
  for (int b = t; b < B; b += kSelThreads) {
    int rank = B - 1 - b;  // by depth: the last block first
    if (order == 1) {
      rank = 0;
      for (int j = 0; j < B; ++j) rank += ranks_before(s_err[j], j, s_err[b], b) ? 1 : 0;
    }
    block_rank[rank] = b;
  }
  __syncthreads();
  if (t == 0) {
    int64_t used = 0;
    int k = 0;
    while (k < B && used + s_cost[__ldcg(block_rank + k)] <= budget)
      used += s_cost[__ldcg(block_rank + k++)];
    *k_out = bad ? -1 : k;
    if (bad && flag) *flag = AQNF4_ERR_INVALID_ARG;
  }
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

extern "C" aqnf4_status aqnf4_select_blocks(const double* sq_err, const double* sq_w,
                                            const int32_t* block_of, const int64_t* cost_bytes,
                                            int32_t num_layers, int32_t num_blocks,
                                            int64_t budget_bytes, int32_t order,
                                            int32_t* block_rank, float* block_err,
                                            int32_t* k_out, int32_t* dev_flag,
                                            cudaStream_t stream) {
  if (!sq_err || !sq_w || !block_of || !cost_bytes || !block_rank || !k_out ||
      num_layers < 1 || num_blocks < 1 || num_blocks > kMaxBlocks || budget_bytes < 0 ||
      (order != AQNF4_BLOCKS_BY_DEPTH && order != AQNF4_BLOCKS_BY_ERROR))
    return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(sq_err, 8) || !is_aligned(sq_w, 8) || !is_aligned(block_of, 4) ||
      !is_aligned(cost_bytes, 8) || !is_aligned(block_rank, 4) || !is_aligned(block_err, 4) ||
      !is_aligned(k_out, 4) || !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  k_select_blocks<<<1, kSelThreads, 0, stream>>>(sq_err, sq_w, block_of, cost_bytes, num_layers,
                                                 num_blocks, budget_bytes, order, block_rank,
                                                 block_err, k_out, dev_flag);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}
