// nf4_gemm.cu -- the forward product of a layer stored in NF4 + DQ on the tensor cores
// (aqnf4_nf4_linear): y = x w_hat^T.
//
// "QLoRA", "How It Works": the 4-bit weights are dequantized to 16 bits on the fly for the
// forward and backward pass.  Here that dequantization happens inside the GEMM: w_hat never
// exists in HBM.  For element (n, k) of the N x K layer (block b = (n K + k) / 64):
//   a'_b = fl(fl(code8_b / 255) * scales[b / 256]),  w_hat = dtype_rn(fl(level[code] * a'_b)),
// bit for bit what aqnf4_dequantize writes; then y = x w_hat^T with binary32 accumulation.
//
// Blackwell structure.  One CTA computes a 128 x 128 tile of y over K in steps of 64:
//   - x (M x K, K contiguous) arrives by TMA in 128-byte-swizzled 128 x 64 tiles;
//   - the 128 threads dequantize the matching 128 x 64 slice of w_hat -- thread t takes row
//     n0 + t, which is exactly one NF4 block per step (K is a multiple of 64) -- and store it
//     in the same swizzled K-major layout, 16 bytes at a time;
//   - one thread issues four tcgen05.mma (M 128, N 128, K 16, bf16/f16 in, f32 out) per step
//     into a TMEM accumulator, and tcgen05.commit frees the stage when they finish;
//   - three stages let the dequantization and the x copy of the next steps overlap the
//     tensor cores; the epilogue reads TMEM with tcgen05.ld (warp w owns lanes 32w..32w+31).
// Every wait is bounded: a wait that gives up records AQNF4_ERR_TIMEOUT, lets the copies and
// MMAs in flight finish (bounded too) and still frees the TMEM before the CTA exits.
#include <cuda.h>

#include <mutex>

#include "device.cuh"

namespace aqnf4 {
namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64, kStages = 3, kGThreads = 128;
constexpr int kTileBytesA = kBM * kBK * 2;  // 16 KB
constexpr int kTileBytesB = kBN * kBK * 2;  // 16 KB
constexpr int kStageBytes = kTileBytesA + kTileBytesB;
constexpr int kBarBase = kStages * kStageBytes;                // after the stages
constexpr int kGSmemBytes = kBarBase + 256 + 1024;             // barriers + alignment slack
constexpr uint32_t kTmemCols = 128;                            // f32 accumulator, 128 columns

struct GParams {
  const uint8_t* packed;
  const uint8_t* codes8;
  const float* scales;
  void* y;
  int64_t M, N, K;
  int32_t out_f32;
  int32_t* flag;
  float level[16];
};

// UMMA shared-memory descriptor of a K-major operand tile in the 128-byte swizzled layout:
// rows 128 bytes apart, 8-row groups 1024 bytes apart (SBO), version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;           // leading byte offset (unused here), 16 B
  d |= static_cast<uint64_t>(1024 >> 4) << 32;   // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;           // descriptor version
  d |= static_cast<uint64_t>(2) << 61;           // SWIZZLE_128B
  return d;
}

// Instruction descriptor: f32 accumulator, both operands DT (f16 = 0, bf16 = 1), K-major,
// N = 128, M = 128.
template <int DT>
__host__ __device__ constexpr uint32_t idesc() {
  return (1u << 4) | (static_cast<uint32_t>(DT) << 7) | (static_cast<uint32_t>(DT) << 10) |
         (static_cast<uint32_t>(kBN >> 3) << 17) | (static_cast<uint32_t>(kBM >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t tmem, uint64_t da, uint64_t db, uint32_t id,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
      "l"(da), "l"(db), "r"(id), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <int DT>
__global__ void __launch_bounds__(kGThreads) k_nf4_gemm(const __grid_constant__ CUtensorMap tmap_x,
                                                        const __grid_constant__ GParams p) {
  using F = Fmt<DT>;
  extern __shared__ uint8_t smem_raw[];
  // the swizzled tiles need 1024-byte alignment
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarBase);
  uint64_t* empty = full + kStages;
  uint64_t* accum = empty + kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kBN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
  const float tab_level = p.level[lane & 15];  // lanes 16..31 mirror 0..15

  if (t == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), 1);
    }
    mbar_init(smem_addr(accum), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int64_t kb = p.K / kBK;  // NF4 blocks per row of w = k steps
  const int64_t n = n0 + t;      // this thread's row of w_hat
  const bool row_ok = n < p.N;
  int pend_stage = -1;           // thread 0: a copy whose completion it did not see
  uint32_t pend_parity = 0;

  for (int64_t kt = 0; kt < kb; ++kt) {
    const int s = static_cast<int>(kt % kStages);
    const uint32_t use = static_cast<uint32_t>(kt / kStages);
    uint8_t* sa = smem + s * kStageBytes;
    uint8_t* sb = sa + kTileBytesA;
    if (kt >= kStages && !mbar_wait_bounded(smem_addr(empty + s), (use - 1) & 1)) *abort_flag = 1;
    __syncthreads();
    if (*abort_flag) break;
    if (t == 0) {
      mbar_arrive_expect_tx(smem_addr(full + s), kTileBytesA);
      tma_load_2d(smem_addr(sa), &tmap_x, static_cast<int>(kt * kBK), static_cast<int>(m0),
                  smem_addr(full + s));
    }
    // ---- dequantize row n, k = kt*64 .. kt*64+63 (one NF4 block) into the swizzled tile
    uint4 pk0 = make_uint4(0, 0, 0, 0), pk1 = pk0;
    float ap = 0.0f;
    if (row_ok) {
      const int64_t b = n * kb + kt;
      const uint4* src = reinterpret_cast<const uint4*>(p.packed + b * 32);
      pk0 = __ldg(src);
      pk1 = __ldg(src + 1);
      ap = __fmul_rn(__fdiv_rn(static_cast<float>(__ldg(p.codes8 + b)), 255.0f),
                     __ldg(p.scales + (b >> 8)));
    }
    const f32x2 a2 = pair(ap, ap);
    const uint32_t words[8] = {pk0.x, pk0.y, pk0.z, pk0.w, pk1.x, pk1.y, pk1.z, pk1.w};
    const int r = t;  // row within the tile
    uint8_t* rowp = sb + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t w = words[j];
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        // byte h: element 2h in the high nibble, 2h + 1 in the low nibble
        const float q0 = __shfl_sync(kFull, tab_level, static_cast<int>(w >> (8 * h + 4)));
        const float q1 = __shfl_sync(kFull, tab_level, static_cast<int>(w >> (8 * h)));
        const f32x2 v = pmul_rn(pair(q0, q1), a2);
        o[h] = row_ok ? F::pack_rn(pair_lo(v), pair_hi(v)) : 0u;
      }
      *reinterpret_cast<uint4*>(rowp + ((j ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    fence_proxy_async_smem();  // the tensor cores read this tile through the async proxy
    __syncthreads();
    if (t == 0) {
      if (!mbar_wait_bounded(smem_addr(full + s), use & 1)) {
        *abort_flag = 1;
        pend_stage = s;
        pend_parity = use & 1;
      } else {
        tc_fence_after();
        const uint32_t a0 = smem_addr(sa), b0 = smem_addr(sb);
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j)  // K = 16 per MMA: 32 bytes along the swizzled row
          umma_f16(tmem, sw128_desc(a0 + 32 * j), sw128_desc(b0 + 32 * j), idesc<DT>(),
                   (kt > 0 || j > 0) ? 1u : 0u);
        umma_commit(smem_addr(empty + s));
      }
    }
  }

  // ---- all MMAs done -> accumulator ready (the decision is made uniformly: tcgen05.ld is a
  // warp-collective instruction)
  if (t == 0) umma_commit(smem_addr(accum));
  const bool ready = mbar_wait_bounded(smem_addr(accum), 0);
  const int failed = __syncthreads_or(!ready || *abort_flag);
  tc_fence_after();
  if (failed) {
    if (t == 0 && p.flag) *p.flag = AQNF4_ERR_TIMEOUT;
  } else {
    // ---- epilogue: warp w reads TMEM lanes 32w..32w+31 = rows m0 + 32w + lane
    const int64_t m = m0 + 32 * warp + lane;
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * c, v);
      const int64_t col = n0 + 32 * c;
      if (m < p.M && col < p.N) {
        const bool whole = col + 32 <= p.N;
        if (p.out_f32) {
          float* dst = static_cast<float*>(p.y) + m * p.N + col;
          if (whole && (p.N & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else {
            for (int i = 0; i < 32 && col + i < p.N; ++i) dst[i] = v[i];
          }
        } else {
          uint16_t* dst = static_cast<uint16_t*>(p.y) + m * p.N + col;
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = F::pack_rn(v[2 * i], v[2 * i + 1]);
          if (whole && (p.N & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(h[i], h[i + 1], h[i + 2], h[i + 3]);
          } else {
            for (int i = 0; i < 32 && col + i < p.N; ++i)
              dst[i] = static_cast<uint16_t>(h[i >> 1] >> (16 * (i & 1)));
          }
        }
      }
    }
  }
  if (t == 0 && pend_stage >= 0) {
    // let the copy that timed out land before the shared memory goes away
    mbar_wait_bounded(smem_addr(full + pend_stage), pend_parity);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

template <int DT>
cudaError_t launch_gemm(const CUtensorMap& map, const GParams& p, cudaStream_t stream) {
  auto kern = k_nf4_gemm<DT>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemBytes);
  if (err != cudaSuccess) return err;
  const dim3 grid(static_cast<unsigned>((p.N + kBN - 1) / kBN),
                  static_cast<unsigned>((p.M + kBM - 1) / kBM));
  kern<<<grid, kGThreads, kGSmemBytes, stream>>>(map, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

extern "C" aqnf4_status aqnf4_nf4_linear(const void* x, int32_t dtype, int64_t M, int64_t K,
                                         const uint8_t* packed, const uint8_t* codes8,
                                         const float* scales, int64_t N, void* y,
                                         int32_t out_f32, int32_t* dev_flag,
                                         cudaStream_t stream) {
  if (!x || !packed || !codes8 || !scales || !y || M < 1 || N < 1 || K < kBK || K % kBK != 0)
    return AQNF4_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - kBM || N > (int64_t(1) << 31) - kBN || K > (int64_t(1) << 31))
    return AQNF4_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return AQNF4_ERR_DTYPE;
  if (!is_aligned(x, 16) || !is_aligned(packed, 16) || !is_aligned(scales, 4) ||
      !is_aligned(y, out_f32 ? 4 : 2) || !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  const Tables* tb = default_tables();
  const EncodeTiledFn encode = encode_tiled();
  if (!tb || !encode) return AQNF4_ERR_CUDA;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {kBK, kBM};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&map,
             dtype == AQNF4_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
             2, const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return AQNF4_ERR_INVALID_ARG;
  GParams p;
  p.packed = packed;
  p.codes8 = codes8;
  p.scales = scales;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.out_f32 = out_f32 ? 1 : 0;
  p.flag = dev_flag;
  for (int i = 0; i < 16; ++i) p.level[i] = tb->level[i];
  const cudaError_t err = dtype == AQNF4_BF16 ? launch_gemm<AQNF4_BF16>(map, p, stream)
                                              : launch_gemm<AQNF4_F16>(map, p, stream);
  return err == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}
