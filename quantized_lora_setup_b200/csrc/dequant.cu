// dequant.cu -- NF4 -> 16-bit dequantization (aqnf4_dequantize).
//
// "QLoRA", "How It Works": training computes with 16-bit values rebuilt from the 4-bit
// storage each time a pass needs them.  For element i of block b = i / 64:
//   a' = fl(fl(code8[b] / 255) * scales[b / 256])   (double-quantized constants), or
//   a' = absmax[b]                                  (plain constants);
//   out[i] = dtype_rn(fl(level[code_i] * a')).
//
// HBM-bound (0.516 B/element in, 2 B/element out).  A lane handles chunks of 16 elements
// (one 8-byte load of packed codes, one 32-byte store) when the output is 32-byte aligned,
// else chunks of 8 (a 4-byte load, a 16-byte store).  The 32 lanes of a warp take 32
// consecutive chunks, so loads and stores are fully coalesced; a warp-iteration covers 64
// elements per lane for memory-level parallelism.  The level lookup is a warp shuffle whose
// source lane is the nibble itself (lanes 16..31 mirror 0..15, so the shifted word needs
// no mask).  fl(c / 255) for the 256 possible bytes is tabulated in shared memory (the
// short exact quotient of device.cuh).  Stores are streaming (evict-first), which the write-heavy
// traffic favours.
#include "device.cuh"

namespace aqnf4 {
namespace {

// 16 chunks per lane cost occupancy (108 registers); 2 or 4 measured slower from 16 MB up
constexpr int kChunksPerLane = 8;

struct DqParams {
  float level[16];
};

// 32-byte streaming store (sm_100): eight 32-bit words
__device__ __forceinline__ void st_cs_v8(void* p, const uint32_t (&o)[8]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
               "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]),
               "r"(o[7])
               : "memory");
}

// CENTERED: the constants come from mean-centred DQ storage, a' = fl(fl(fl(q/127) * h) + mu)
// with q = code8 - 128, h = scales[b / 256] and mu = means[b / 256] (`absmax` carries the
// means); otherwise a' = fl(fl(code8/255) * s), or the plain absmax when codes8 is NULL.
// W: 32-bit words of packed codes per lane and chunk -- 1 (8 elements: a 4-byte load and a
// 16-byte store) or 2 (16 elements: an 8-byte load and a 32-byte store, for a 32-byte
// aligned output).  A lane takes 64 elements per iteration either way.
template <int DT, bool CENTERED, int W>
__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ packed,
                                                 const uint8_t* __restrict__ codes8,
                                                 const float* __restrict__ scales,
                                                 const float* __restrict__ absmax, int64_t n,
                                                 uint16_t* __restrict__ out,
                                                 const __grid_constant__ DqParams p) {
  using F = Fmt<DT>;
  static_assert(W == 1 || W == 2, "a chunk is one or two packed words");
  constexpr int kE = 8 * W;                        // elements per chunk
  constexpr int kCpl = kChunksPerLane / W;         // chunks per lane and iteration
  constexpr int kBlockShift = W == 1 ? 3 : 2;      // chunks per 64-element block: 8 or 4
  __shared__ float frac[256];
  const int t = threadIdx.x, lane = t & 31;
  if (CENTERED)
    frac[t] = __fdiv_rn(static_cast<float>(t - 128), 127.0f);
  else  // t and 255 are 16-bit values, t <= 255: the short quotient is exactly fl(t / 255)
    frac[t] = quot16_rn(static_cast<float>(t), 255.0f, rcp16_rn(255.0f));
  __syncthreads();
  const float tab_level = p.level[lane & 15];

  const int64_t nchunk = (n + kE - 1) / kE;
  const int64_t full_chunks = n / kE;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + t) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  constexpr int64_t kGroup = 32 * kCpl;

  for (int64_t g = warp_id; g * kGroup < nchunk; g += nwarps) {
    uint32_t wd[kCpl][W];
    float ap[kCpl];
#pragma unroll
    for (int j = 0; j < kCpl; ++j) {
      const int64_t c = g * kGroup + j * 32 + lane;
#pragma unroll
      for (int k = 0; k < W; ++k) wd[j][k] = 0;
      ap[j] = 0.0f;
      if (c < full_chunks) {
        if constexpr (W == 1) {
          wd[j][0] = __ldg(reinterpret_cast<const uint32_t*>(packed) + c);
        } else {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(packed) + c);
          wd[j][0] = v.x;
          wd[j][W - 1] = v.y;
        }
      } else if (c < nchunk) {  // last, partial chunk: read only the bytes that exist
        const int64_t nbytes = (n + 1) >> 1;
        if constexpr (W == 1) {
          for (int64_t byte = c * 4; byte < nbytes; ++byte)
            wd[j][0] |= static_cast<uint32_t>(packed[byte]) << (8 * (byte - c * 4));
        } else {
          uint32_t lo = 0, hi = 0;
          for (int64_t byte = c * 8; byte < nbytes; ++byte) {
            const int64_t o = byte - c * 8;
            const uint32_t v = static_cast<uint32_t>(packed[byte]) << (8 * (o & 3));
            if (o < 4)
              lo |= v;
            else
              hi |= v;
          }
          wd[j][0] = lo;
          wd[j][W - 1] = hi;
        }
      }
      if (c < nchunk) {
        const int64_t b = c >> kBlockShift;  // the chunk's 64-element block
        if (CENTERED)
          ap[j] = __fadd_rn(__fmul_rn(frac[__ldg(codes8 + b)], __ldg(scales + (b >> 8))),
                            __ldg(absmax + (b >> 8)));
        else
          ap[j] = codes8 ? __fmul_rn(frac[__ldg(codes8 + b)], __ldg(scales + (b >> 8)))
                         : __ldg(absmax + b);
      }
    }
#pragma unroll
    for (int j = 0; j < kCpl; ++j) {
      const f32x2 a2 = pair(ap[j], ap[j]);
      uint32_t o[4 * W];
#pragma unroll
      for (int k = 0; k < W; ++k) {
        const uint32_t w = wd[j][k];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          // byte h holds element 2h in its high nibble and element 2h+1 in its low nibble
          const float q0 = __shfl_sync(kFull, tab_level, static_cast<int>(w >> (8 * h + 4)));
          const float q1 = __shfl_sync(kFull, tab_level, static_cast<int>(w >> (8 * h)));
          const f32x2 v = pmul_rn(pair(q0, q1), a2);
          o[4 * k + h] = F::pack_rn(pair_lo(v), pair_hi(v));
        }
      }
      const int64_t c = g * kGroup + j * 32 + lane;
      if (c < full_chunks) {
        // streaming store: the output is not read again by this kernel
        if constexpr (W == 1)
          __stcs(reinterpret_cast<uint4*>(out + kE * c), make_uint4(o[0], o[1], o[2], o[3]));
        else
          st_cs_v8(out + kE * c, o);
      } else if (c < nchunk) {
        for (int e = 0; e < kE && kE * c + e < n; ++e)
          out[kE * c + e] = static_cast<uint16_t>(o[e >> 1] >> ((e & 1) * 16));
      }
    }
  }
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

namespace {

aqnf4_status launch_dequant(const uint8_t* packed, const uint8_t* codes8, const float* scales,
                            const float* absmax, int64_t n, int32_t out_dtype, void* out,
                            bool centered, cudaStream_t stream) {
  const Tables* tb = default_tables();
  if (!tb) return AQNF4_ERR_CUDA;
  DqParams p;
  for (int i = 0; i < 16; ++i) p.level[i] = tb->level[i];
  // 64 elements per lane and iteration, in either chunk width
  const int64_t groups = (n + 32 * 8 * kChunksPerLane - 1) / (32 * 8 * kChunksPerLane);
  const int sms = current_sm_count();
  int64_t grid = static_cast<int64_t>(sms > 0 ? sms : 1) * 8;  // 8 warps per CTA
  const int64_t need = (groups + 7) / 8;
  if (grid > need) grid = need;
  uint16_t* o = static_cast<uint16_t*>(out);
  const unsigned g = static_cast<unsigned>(grid);
  const bool wide = is_aligned(out, 32);  // 32-byte stores
#define AQNF4_DQ_LAUNCH(DTV, CEN)                                                        \
  do {                                                                                   \
    if (wide)                                                                            \
      k_dequant<DTV, CEN, 2><<<g, 256, 0, stream>>>(packed, codes8, scales, absmax, n, o, p); \
    else                                                                                 \
      k_dequant<DTV, CEN, 1><<<g, 256, 0, stream>>>(packed, codes8, scales, absmax, n, o, p); \
  } while (0)
  if (out_dtype == AQNF4_BF16) {
    if (centered)
      AQNF4_DQ_LAUNCH(AQNF4_BF16, true);
    else
      AQNF4_DQ_LAUNCH(AQNF4_BF16, false);
  } else {
    if (centered)
      AQNF4_DQ_LAUNCH(AQNF4_F16, true);
    else
      AQNF4_DQ_LAUNCH(AQNF4_F16, false);
  }
#undef AQNF4_DQ_LAUNCH
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}

}  // namespace

extern "C" aqnf4_status aqnf4_dequantize(const uint8_t* packed, const uint8_t* codes8,
                                         const float* scales, const float* absmax, int64_t n,
                                         int32_t out_dtype, void* out, cudaStream_t stream) {
  if (!packed || !out || n < 1) return AQNF4_ERR_INVALID_ARG;
  if (codes8 ? !scales : !absmax) return AQNF4_ERR_INVALID_ARG;
  if (!valid_dtype(out_dtype)) return AQNF4_ERR_DTYPE;
  if (!is_aligned(packed, 16) || !is_aligned(out, 16) || !is_aligned(scales, 4) ||
      !is_aligned(absmax, 4))
    return AQNF4_ERR_ALIGNMENT;
  return launch_dequant(packed, codes8, scales, absmax, n, out_dtype, out, false, stream);
}

extern "C" aqnf4_status aqnf4_dequantize_centered(const uint8_t* packed, const uint8_t* codes8,
                                                  const float* scales, const float* means,
                                                  int64_t n, int32_t out_dtype, void* out,
                                                  cudaStream_t stream) {
  if (!packed || !codes8 || !scales || !means || !out || n < 1) return AQNF4_ERR_INVALID_ARG;
  if (!valid_dtype(out_dtype)) return AQNF4_ERR_DTYPE;
  if (!is_aligned(packed, 16) || !is_aligned(out, 16) || !is_aligned(scales, 4) ||
      !is_aligned(means, 4))
    return AQNF4_ERR_ALIGNMENT;
  return launch_dequant(packed, codes8, scales, means, n, out_dtype, out, true, stream);
}
