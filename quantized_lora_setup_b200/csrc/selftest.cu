// selftest.cu -- diagnostics.  aqnf4_selftest_wait_timeout exercises the bounded mbarrier
// wait that every bulk-copy consumer in this library uses, on a barrier that nothing ever
// completes, so the give-up path (status AQNF4_ERR_TIMEOUT, kernel returns, context stays
// usable) can be tested without a fault or a hang.  aqnf4_selftest_division evaluates the
// fused pass's short reciprocal and quotient beside CUDA's correctly rounded ones.
#include "device.cuh"

namespace aqnf4 {
namespace {

__global__ void k_selftest_wait(uint64_t timeout_ns, int32_t* flag, int64_t* waited_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);  // one arrival expected; none will come
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t t0 = global_timer_ns();
  const bool ok = mbar_wait_bounded(smem_addr(&bar), 0, timeout_ns);
  if (threadIdx.x == 0) {
    if (!ok && flag) *flag = AQNF4_ERR_TIMEOUT;
    if (waited_ns) *waited_ns = static_cast<int64_t>(global_timer_ns() - t0);
  }
}

__global__ void k_selftest_division(const float* a, const float* s, int64_t n, float* out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float ai = a[i], si = s[i];
    float4 o;
    o.x = rcp16_rn(ai);
    o.y = __frcp_rn(ai);
    o.z = quot16_rn(ai, si, rcp16_rn(si));
    o.w = __fdiv_rn(ai, si);
    reinterpret_cast<float4*>(out)[i] = o;
  }
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

extern "C" aqnf4_status aqnf4_selftest_wait_timeout(int64_t timeout_ns, int32_t* dev_flag,
                                                    int64_t* waited_ns, cudaStream_t stream) {
  if (timeout_ns < 1 || timeout_ns > 2000000000ll || !dev_flag) return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(dev_flag, 4) || !is_aligned(waited_ns, 8)) return AQNF4_ERR_ALIGNMENT;
  k_selftest_wait<<<1, 32, 0, stream>>>(static_cast<uint64_t>(timeout_ns), dev_flag, waited_ns);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}

extern "C" aqnf4_status aqnf4_selftest_division(const float* a, const float* s, int64_t n,
                                                float* out, cudaStream_t stream) {
  if (!a || !s || !out || n < 1) return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(a, 4) || !is_aligned(s, 4) || !is_aligned(out, 16)) return AQNF4_ERR_ALIGNMENT;
  const int64_t blocks = (n + 255) / 256;
  k_selftest_division<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(
      a, s, n, out);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}
