// quant_score.cu -- the fused NF4 pass: blockwise absmax, NF4 codes, nibble packing, double
// quantization of the absmax constants and the per-layer reconstruction-error sums, in one
// read of the weights.  Entry points aqnf4_quantize, aqnf4_layer_error,
// aqnf4_workspace_size.
//
// What is computed ("QLoRA", "How It Works"; arxivdaily 2608.23816, "English abstract"):
//   per 64-element block b of a layer: a_b = max |x|; v = fl(x * fl(1/a_b));
//   code = #{ j : v > mid_j }; packed byte i = code[2i] << 4 | code[2i+1];
//   per 256 blocks: s = max a_b, code8_b = rint(fl(fl(a_b / s) * 255));
//   per layer: sum (x - w_hat)^2 and sum x^2 with w_hat = dtype_rn(fl(level[code] * a_b)).
//
// Each thread sums its block's (x - w_hat)^2 and x^2 in binary32 -- directly when
// 2^-40 <= a_b <= 2^40, where no term can overflow or underflow; otherwise in the
// normalised domain ((x - w_hat) r)^2 and v^2, scaled back by a_b^2 -- and the 256 block
// sums of a tile are added in binary64 in a fixed order.
//
// Work decomposition (B200): a tile is 16384 consecutive elements of one layer (one DQ
// block, 256 NF4 blocks).  A persistent CTA of 128 threads walks tiles with a grid stride;
// thread t owns NF4 blocks t and t + 128.  A 1-D bulk copy (TMA engine) brings each 32 KB
// tile into shared memory; five CTAs share an SM, so one CTA's copy overlaps the others'
// arithmetic.  Each thread reads its blocks twice with conflict-free 16-byte loads (chunk
// order rotated per thread): once for the absmax (packed bf16x2/f16x2 max), once to code,
// the two blocks' work interleaved.  A code does not count midpoints: an odd cubic
// k = round(a v + b v^3 + 8) (three packed FMA-pipe instructions per two elements) puts
// every midpoint in a slot of its own, so one warp-shuffle lookup of that slot's midpoint
// and the sign of one subtract give code = k - 1 + (v > slot_mid[k]); the code then
// indexes the level shuffle.  The tables and the proof that this equals the midpoint count
// for every normalised v are built on the host (codebook.cpp).  Arithmetic on pairs uses
// Blackwell's packed f32x2 instructions, and w_hat - x comes from the packed 16-bit w_hat
// with one mixed-precision subtract.  Packed codes are staged in shared memory and leave with
// coalesced 16-byte stores.  fl(1/a) and the DQ quotient fl(a/s) come from a one-step
// Newton-Raphson form on the fused multiply-add (rcp16_rn, quot16_rn), exact for the 16-bit
// values met here, instead of a full divide per block.  The per-tile extra work (the next
// bulk copy, the binary64 reduction) rotates over the warps so no warp is always last at a
// barrier.
#include <cfloat>
#include <mutex>

#include "device.cuh"

namespace aqnf4 {
namespace {

// Two NF4 blocks per thread (t and t + 128): their dependency chains interleave, which the
// shuffle latency needs, and per-tile costs are shared by 128 elements.
constexpr int kBpt = 2;
constexpr int kThreads = kDqBlock / kBpt;  // a CTA covers one tile (= one DQ block)
constexpr int kWarps = kThreads / 32;
static_assert(kWarps == 4, "the centred score's tree takes slot bits 5..6 from 4 warps");
// chunk loop of the coding pass unrolled by 2: smaller code, slightly faster than full unroll
constexpr int kP2Unroll = 2;
constexpr int kCtasPerSm = 5;  // 44 KB of shared memory and <= 102 registers per thread, no spills
constexpr int kMaxLayersPerLaunch = 384;

// The coding loop keeps each code as c = bits(2^23 + slot) + (v > mid) = kCodeBias + code,
// so that c's low 5 bits index the level table directly.  The byte (c0 << 4) + c1 and the
// packed word sum_j byte_j << 8j then carry data-independent constants, removed once per word.
constexpr uint32_t kCodeBias = 0x4B000001u;
constexpr uint32_t kByteBias = (kCodeBias << 4) + kCodeBias;
constexpr uint32_t kPackBias = kByteBias + (kByteBias << 8) + (kByteBias << 16) + (kByteBias << 24);

// shared memory layout (bytes): one input stage, the packed-output stage, the per-block
// (err, w^2, scale) floats, the per-warp absmax, the mbarrier and abort word.  The output
// and reduction buffers are single: a second barrier at the end of each tile separates
// their readers from the next tile's writers (double buffers cost registers that spill).
constexpr size_t kOutOff = kTileBytes;
constexpr size_t kRedOff = kOutOff + kPackedTileBytes;
constexpr size_t kRedBytes = 3 * kDqBlock * sizeof(float);
constexpr size_t kMaxOff = kRedOff + kRedBytes;
constexpr size_t kPreOff = kMaxOff + 16 * sizeof(float);  // per-warp max for a DQ score
constexpr size_t kCenOff = kPreOff + 16 * sizeof(float);  // per-warp sums for a centred score
constexpr size_t kBarOff = kCenOff + 2 * kWarps * sizeof(double);
constexpr size_t kSmemBytes = kBarOff + 16;

struct LayerRec {
  const void* w;
  uint8_t* packed;
  float* absmax;
  uint8_t* codes8;
  float* scales;
  int64_t numel;
  int32_t flags;  // AQNF4_SCORE_* bits
  int32_t pad;
};

struct QParams {
  int32_t num_layers;  // layers in this launch
  int32_t pad0;
  int64_t num_tiles;   // tiles in this launch
  int64_t tile_base;   // index of this launch's first tile in the partials array
  double2* partials;   // per tile (sum (x - w_hat)^2, sum x^2); score only
  int32_t* flag;       // optional device status word
  float curve_a, curve_b;
  float slot_mid[32];
  float slot_level[32];
  float level[16];
  float mid[15];
  int32_t tile_begin[kMaxLayersPerLaunch + 1];  // first tile of each layer (launch-local)
  LayerRec layers[kMaxLayersPerLaunch];
};

struct FParams {
  int32_t num_layers;
  int32_t layer_base;  // global index of this launch's first layer (outputs)
  int64_t tile_base;
  const double2* partials;
  double* sq_err;
  double* sq_w;
  float* rel_err;
  int32_t tile_begin[kMaxLayersPerLaunch + 1];
};

__device__ __forceinline__ int find_layer(const QParams& p, int64_t tile) {
  int lo = 0, hi = p.num_layers - 1;  // tile_begin[lo] <= tile < tile_begin[hi + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.tile_begin[mid] <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

struct TileGeom {
  int layer;
  int64_t tin;  // tile index inside the layer
  int cnt;      // elements in this tile (16384 except a layer's last tile)
};

// `cursor` caches the layer of the previous call: a CTA's tiles only move forward.
__device__ __forceinline__ TileGeom tile_geom(const QParams& p, int64_t tile, int& cursor) {
  TileGeom g;
  if (tile < p.tile_begin[cursor]) cursor = find_layer(p, tile);
  while (tile >= p.tile_begin[cursor + 1]) ++cursor;
  g.layer = cursor;
  g.tin = tile - p.tile_begin[g.layer];
  const int64_t rem = p.layers[g.layer].numel - g.tin * kTile;
  g.cnt = rem < kTile ? static_cast<int>(rem) : kTile;
  return g;
}

// Start the bulk copy of `tile` into the stage.  A short last tile copies its
// 16-byte-aligned prefix; its remaining < 8 elements are read from global memory later.
__device__ __forceinline__ void issue_tile(const QParams& p, int64_t tile, uint8_t* stage,
                                          uint32_t bar, uint64_t policy, int& cursor) {
  const TileGeom g = tile_geom(p, tile, cursor);
  const uint32_t bytes = static_cast<uint32_t>(g.cnt * 2) & ~15u;
  mbar_arrive_expect_tx(bar, bytes);
  if (bytes) {
    const uint8_t* src = static_cast<const uint8_t*>(p.layers[g.layer].w) + g.tin * kTileBytes;
    bulk_load(smem_addr(stage), src, bytes, bar, policy);
  }
}

// Generic per-element path for a block whose absmax lies outside [2^-40, 2^40] (zero,
// subnormal, huge or not finite), or whose rebuild constant does.  Re-reads the block
// (natural element order) from shared memory, rewrites this thread's packed words and
// returns the sums (err, w^2) normalised by sb = max(a, |ar|) -- scaled by sb^2 later.  ar
// is the constant w_hat is rebuilt from: a, or a double-quantized constant; normalising by
// the larger of the two keeps every term at most about 4 whatever ar is.
template <int DT, bool SCORE>
__device__ __noinline__ float2 block_generic(const uint8_t* my, float a, float ar,
                                             const QParams& p,
                                             uint8_t* ost) {  // ost: this block's 32 bytes
  using F = Fmt<DT>;
  const bool zero = (a == 0.0f);
  const bool finite = (a <= FLT_MAX);
  float scale = 1.0f, as = a;
  if (!zero && a < 0x1p-126f) {  // exact rescale keeps 1/a finite
    scale = 0x1p64f;
    as = __fmul_rn(a, scale);
  }
  const float r = zero ? 0.0f : __frcp_rn(as);
  // normalisation of the error terms: by sb = max(a, |ar|) (= a unless ar exceeds it)
  const float sb = fmaxf(a, fabsf(ar));
  float escale = scale, er = r;
  if (sb != a) {
    escale = 1.0f;
    float sbs = sb;
    if (sb < 0x1p-126f) {
      escale = 0x1p64f;
      sbs = __fmul_rn(sb, escale);
    }
    er = __frcp_rn(sbs);
  }
  const uint16_t* x16 = reinterpret_cast<const uint16_t*>(my);
  float se = 0.0f, sw = 0.0f;
  for (int c = 0; c < 8; ++c) {
    uint32_t pk = 0;
    for (int i = 0; i < 8; ++i) {
      const uint32_t h = x16[8 * c + i];
      const float x = F::lo(h);
      int code = 7;
      float v = 0.0f;
      if (!zero) {
        v = __fmul_rn(__fmul_rn(x, scale), r);
        code = 0;
        for (int j = 0; j < 15; ++j) code += (v > p.mid[j]) ? 1 : 0;
      }
      pk |= static_cast<uint32_t>(code) << ((i >> 1) * 8 + ((i & 1) ? 0 : 4));
      if (SCORE && !(zero && ar == 0.0f)) {
        const float wh = F::round_trip(__fmul_rn(p.level[code], ar));
        const float d = __fmul_rn(__fsub_rn(__fmul_rn(x, escale), __fmul_rn(wh, escale)), er);
        const float ve = sb == a ? v : __fmul_rn(__fmul_rn(x, escale), er);
        se = __fmaf_rn(d, d, se);
        sw = __fmaf_rn(ve, ve, sw);
      }
    }
    *reinterpret_cast<uint32_t*>(ost + c * 4) = pk;
  }
  if (!finite) {
    se = sw = __int_as_float(0x7fffffff);
    if (p.flag) *p.flag = AQNF4_ERR_NONFINITE;
  }
  return make_float2(se, sw);
}

template <int DT, bool SCORE>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_quant_score(const __grid_constant__ QParams p) {
  using F = Fmt<DT>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stage = smem;
  float* red = reinterpret_cast<float*>(smem + kRedOff);   // [3 = err, w2, scale][256]
  float* wmax = reinterpret_cast<float*>(smem + kMaxOff);  // [kWarps]
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smem + kPreOff);  // [kWarps]
  double* wcen = reinterpret_cast<double*>(smem + kCenOff);       // [2][kWarps]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBarOff);
  int* abort_flag = reinterpret_cast<int*>(smem + kBarOff + 8);
  const uint32_t bar_a = smem_addr(bar);

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // this lane's entries of the shuffle lookup tables
  const float tab_mid = p.slot_mid[lane];
  const float tab_level = p.slot_level[lane];

  if (t == 0) {
    mbar_init(bar_a, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t T = p.num_tiles;
  const int64_t stride = gridDim.x;
  const uint64_t policy = l2_evict_first_policy();
  int cursor = 0, issue_cursor = 0;
  if (t == 0 && blockIdx.x < T) issue_tile(p, blockIdx.x, stage, bar_a, policy, issue_cursor);

  const int rot = (t + (t >> 3)) & 7;  // conflict-free 16-byte reads and 4-byte writes
  int64_t k = 0;
  bool aborted = false;
  for (int64_t tile = blockIdx.x; tile < T; tile += stride, ++k) {
    if (!mbar_wait_bounded(bar_a, static_cast<uint32_t>(k & 1))) {
      *abort_flag = 1;
      if (p.flag) *p.flag = AQNF4_ERR_TIMEOUT;
    }
    const TileGeom g = tile_geom(p, tile, cursor);
    const LayerRec& L = p.layers[g.layer];
    const int nblk = (g.cnt + kBlock - 1) / kBlock;
    if (g.cnt < kTile) {
      // a layer's short last tile: finish it in shared memory (tail from global, then zeros)
      const int pre = static_cast<int>((static_cast<uint32_t>(g.cnt * 2) & ~15u) >> 1);
      uint16_t* s16 = reinterpret_cast<uint16_t*>(stage);
      const uint16_t* gw = static_cast<const uint16_t*>(L.w) + g.tin * kTile;
      for (int e = pre + t; e < kTile; e += kThreads) s16[e] = e < g.cnt ? gw[e] : 0;
      fence_proxy_async_smem();
      __syncthreads();
    }

    // ---- pass 1: absmax of this thread's blocks (NaN propagates)
    float a[kBpt], r[kBpt];
    bool fast[kBpt];
#pragma unroll
    for (int b = 0; b < kBpt; ++b) {
      const uint8_t* my = stage + (t + b * kThreads) * 128;
      uint32_t m0 = 0, m1 = 0;
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) {
        const uint4 v = lds128(my + ((k2 + rot) & 7) * 16);
        m0 = F::absmax2(m0, F::absmax2(v.x, v.y));
        m1 = F::absmax2(m1, F::absmax2(v.z, v.w));
      }
      m0 = F::absmax2(m0, m1);
      m0 = F::absmax2(m0, __byte_perm(m0, 0, 0x1032));
      a[b] = F::abs_lo(m0);
      // 2^-40 <= a <= 2^40: (w_hat - x)^2 and x^2 cannot overflow or flush in binary32
      fast[b] = (a[b] >= 0x1p-40f) && (a[b] <= 0x1p40f);
      r[b] = fast[b] ? rcp16_rn(a[b]) : 0.0f;
    }

    // ---- the constant w_hat is rebuilt from: a, or for a DQ score the double-quantized
    // a' = fl(fl(code8/255) s) with s the tile's (DQ block's) maximum.  a' <= ~2a (code8 > 0
    // needs a >= s/510), so the fast path's range argument still holds.  The branch is
    // uniform over the CTA (one layer per tile).
    float ar[kBpt];
#pragma unroll
    for (int b = 0; b < kBpt; ++b) ar[b] = a[b];
    if (SCORE && (L.flags & AQNF4_SCORE_DQ_ABSMAX)) {
      uint32_t m = 0;
#pragma unroll
      for (int b = 0; b < kBpt; ++b)
        if (t + b * kThreads < nblk) m = max(m, __float_as_uint(a[b]));
      m = __reduce_max_sync(kFull, m);
      if (lane == 0) wpre[warp] = m;
      __syncthreads();
      uint32_t sb = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sb = max(sb, wpre[w]);
      const float s = __uint_as_float(sb);
#pragma unroll
      for (int b = 0; b < kBpt; ++b) ar[b] = dq_constant(dq_code(a[b], s), s);
    } else if (SCORE && (L.flags & AQNF4_SCORE_DQ_CENTERED)) {
      // mean-centred DQ constants of this tile (one DQ block): the binary64 sum over the
      // balanced tree of its 256 slots, slot t + 128 b held by thread t.  Slot bits 0..4
      // are the lane (xor butterfly), bits 5..6 the warp, bit 7 the half b; each pair sum
      // is the same in both partners since binary64 addition is commutative.  Slots past
      // the layer's end hold the padding's absmax, +0.
      double v0 = static_cast<double>(a[0]), v1 = static_cast<double>(a[1]);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        v0 = __dadd_rn(v0, __shfl_xor_sync(kFull, v0, off));
        v1 = __dadd_rn(v1, __shfl_xor_sync(kFull, v1, off));
      }
      if (lane == 0) {
        wcen[warp] = v0;
        wcen[kWarps + warp] = v1;
      }
      __syncthreads();
      const double S = __dadd_rn(__dadd_rn(__dadd_rn(wcen[0], wcen[1]), __dadd_rn(wcen[2], wcen[3])),
                                 __dadd_rn(__dadd_rn(wcen[4], wcen[5]), __dadd_rn(wcen[6], wcen[7])));
      const float mu = __double2float_rn(__ddiv_rn(S, static_cast<double>(nblk)));
      float c[kBpt];
      uint32_t m = 0;
#pragma unroll
      for (int b = 0; b < kBpt; ++b) {
        c[b] = __fsub_rn(a[b], mu);
        // |c| >= 0 or NaN: as unsigned integers the patterns order like the values, NaN top
        if (t + b * kThreads < nblk) m = max(m, __float_as_uint(fabsf(c[b])));
      }
      m = __reduce_max_sync(kFull, m);
      if (lane == 0) wpre[warp] = m;
      __syncthreads();
      uint32_t hb = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) hb = max(hb, wpre[w]);
      const float h = __uint_as_float(hb);
      const bool finite = (fabsf(mu) <= FLT_MAX) && (h <= FLT_MAX);
#pragma unroll
      for (int b = 0; b < kBpt; ++b) {
        int q = -128;  // a non-finite block stores code 0
        if (finite) q = h == 0.0f ? 0 : __float2int_rn(__fmul_rn(__fdiv_rn(c[b], h), 127.0f));
        ar[b] = __fadd_rn(__fmul_rn(__fdiv_rn(static_cast<float>(q), 127.0f), h), mu);
        // a centred constant need not stay near a (a tile mixing tiny and huge blocks):
        // the binary32 fast path's range argument needs |ar| <= 2^40 as well
        if (!(fabsf(ar[b]) <= 0x1p40f)) fast[b] = false;
      }
    }

    // ---- pass 2: codes, packing, error; the blocks' chains interleave (all lanes run this
    // so the shuffles stay converged)
    f32x2 es2[kBpt], ws2[kBpt], r2[kBpt], a2[kBpt];
#pragma unroll
    for (int b = 0; b < kBpt; ++b) {
      es2[b] = ws2[b] = pair(0.0f, 0.0f);
      r2[b] = pair(r[b], r[b]);
      a2[b] = pair(ar[b], ar[b]);
    }
    const f32x2 ca2 = pair(p.curve_a, p.curve_a), cb2 = pair(p.curve_b, p.curve_b);
    const f32x2 off2 = pair(8388616.0f, 8388616.0f);  // 2^23 + 8
    uint8_t* ost = smem + kOutOff;
#pragma unroll kP2Unroll
    for (int k2 = 0; k2 < 8; ++k2) {
      const int c = (k2 + rot) & 7;
#pragma unroll
      for (int b = 0; b < kBpt; ++b) {
        const int blk = t + b * kThreads;
        const uint4 v4 = lds128(stage + blk * 128 + c * 16);
        const uint32_t w4[4] = {v4.x, v4.y, v4.z, v4.w};
        uint32_t pk = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t wd = w4[j];
          const f32x2 x = pair(F::lo(wd), F::hi(wd));
          const f32x2 v = pmul_rn(x, r2[b]);
          // slot k = round(a v + b v^3 + 8) lands in the low 5 bits of kk = 2^23 + k
          const f32x2 kk = pfma_rn(v, pfma_rn(pmul_rn(v, v), cb2, ca2), off2);
          const uint32_t k0 = __float_as_uint(pair_lo(kk)), k1 = __float_as_uint(pair_hi(kk));
          const f32x2 mid =
              pair(__shfl_sync(kFull, tab_mid, static_cast<int>(k0)),
                   __shfl_sync(kFull, tab_mid, static_cast<int>(k1)));
          // v > mid exactly when fl(mid - v) is negative (a difference is exact in sign).
          // This needs the rounded v: were the multiply fused into the subtract (x r - mid,
          // which ptxas does for a product with no other use, despite .rn), ties v == mid
          // would follow the exact product.  Here v also feeds the slot curve, and the GPU
          // parity tests include blocks of exact ties.
          const f32x2 dm = psub_rn(mid, v);
          // c = bits(kk) + (v > mid) = kCodeBias + code: code + 1 in the low 5 bits
          const uint32_t c0 = k0 + (__float_as_uint(pair_lo(dm)) >> 31);
          const uint32_t c1 = k1 + (__float_as_uint(pair_hi(dm)) >> 31);
          const uint32_t byte = (c0 << 4) + c1;  // code0 << 4 | code1, plus kByteBias
          pk = j == 0 ? byte : pk + (byte << (8 * j));
          if (SCORE) {
            const float q0 = __shfl_sync(kFull, tab_level, static_cast<int>(c0));
            const float q1 = __shfl_sync(kFull, tab_level, static_cast<int>(c1));
            const f32x2 wq = pmul_rn(pair(q0, q1), a2[b]);
            const uint32_t hb = F::pack_rn(pair_lo(wq), pair_hi(wq));
            // w_hat - x straight from the packed 16-bit w_hat (the sign does not matter)
            const f32x2 d = pair(F::sub_lo(hb, pair_lo(x)), F::sub_hi(hb, pair_hi(x)));
            es2[b] = pfma_rn(d, d, es2[b]);
            ws2[b] = pfma_rn(x, x, ws2[b]);
          }
        }
        *reinterpret_cast<uint32_t*>(ost + blk * 32 + c * 4) = pk - kPackBias;
      }
    }

    // ---- per block: sums (generic path where needed) into the reduction buffers
    float* r_err = red;
    float* r_w2 = red + kDqBlock;
    float* r_a = red + 2 * kDqBlock;
    uint32_t amax = 0;
#pragma unroll
    for (int b = 0; b < kBpt; ++b) {
      const int blk = t + b * kThreads;
      float2 sums = make_float2(pair_lo(es2[b]) + pair_hi(es2[b]),
                                pair_lo(ws2[b]) + pair_hi(ws2[b]));
      // factor that turns this block's sums into weight units once squared
      float sum_scale = 1.0f;
      if (!fast[b]) {
        sums = block_generic<DT, SCORE>(stage + blk * 128, a[b], ar[b], p, ost + blk * 32);
        sum_scale = fmaxf(a[b], fabsf(ar[b]));  // block_generic's normalisation
      }
      if (SCORE) {
        r_err[blk] = sums.x;
        r_w2[blk] = sums.y;
        r_a[blk] = sum_scale;
      }
      // a >= 0 or NaN: as unsigned integers the binary32 patterns order like the values,
      // with every NaN above +inf, so an integer max is the NaN-propagating float max
      if (blk < nblk) amax = max(amax, __float_as_uint(a[b]));
    }
    amax = __reduce_max_sync(kFull, amax);
    if (lane == 0) wmax[warp] = __uint_as_float(amax);
    __syncthreads();
    if (*abort_flag) {
      aborted = true;
      break;
    }
    const int lead = static_cast<int>(k & (kWarps - 1));  // warp doing this tile's extra work
    if (warp == lead && lane == 0 && tile + stride < T) {
      fence_proxy_async_smem();
      issue_tile(p, tile + stride, stage, bar_a, policy, issue_cursor);
    }

    // ---- outputs
    uint32_t sdq_bits = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sdq_bits = max(sdq_bits, __float_as_uint(wmax[w]));
    const float sdq = __uint_as_float(sdq_bits);
    const int64_t blk0 = g.tin * kDqBlock;
    // the short exact quotient needs the scale in [2^-40, 2^40]; otherwise (zero, subnormal,
    // huge or non-finite scale) the plain correctly rounded divide
    const bool sfast = sdq >= 0x1p-40f && sdq <= 0x1p40f;
    const float ys = sfast ? rcp16_rn(sdq) : 0.0f;
#pragma unroll
    for (int b = 0; b < kBpt; ++b) {
      const int blk = t + b * kThreads;
      if (blk < nblk) {
        if (L.absmax) __stcs(L.absmax + blk0 + blk, a[b]);
        if (L.codes8) __stcs(reinterpret_cast<char*>(L.codes8) + blk0 + blk,
                             static_cast<char>(sfast ? dq_code_fast(a[b], sdq, ys)
                                                     : dq_code(a[b], sdq)));
      }
    }
    if (t == 0 && L.codes8) {
      L.scales[g.tin] = sdq;
      if (!(sdq <= FLT_MAX) && p.flag) *p.flag = AQNF4_ERR_NONFINITE;
    }
    if (SCORE && warp == lead) {
      double se = 0.0, sw = 0.0;
#pragma unroll
      for (int j = 0; j < kDqBlock / 32; ++j) {
        const int i = lane + 32 * j;
        const double aa = static_cast<double>(r_a[i]) * static_cast<double>(r_a[i]);
        se += static_cast<double>(r_err[i]) * aa;
        sw += static_cast<double>(r_w2[i]) * aa;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        se += __shfl_xor_sync(kFull, se, off);
        sw += __shfl_xor_sync(kFull, sw, off);
      }
      if (lane == 0) p.partials[p.tile_base + tile] = make_double2(se, sw);
    }
    if (L.packed) {
      const uint8_t* os = smem + kOutOff;
      uint8_t* gp = L.packed + g.tin * kPackedTileBytes;
      if (g.cnt == kTile) {
#pragma unroll
        for (int i = t; i < kPackedTileBytes / 16; i += kThreads)
          __stcs(reinterpret_cast<uint4*>(gp + 16 * i), lds128(os + 16 * i));
      } else {
        const int nbytes = (g.cnt + 1) >> 1;
        for (int i = t; i < nbytes; i += kThreads) {
          uint8_t b = os[i];
          if ((g.cnt & 1) && i == nbytes - 1) b &= 0xF0;  // odd length: low nibble stays 0
          gp[i] = b;
        }
      }
    }
    __syncthreads();  // the single output and reduction buffers are free again
  }

  if (aborted && t == 0) {
    // let the bulk copy that timed out land before the CTA (and its shared memory) goes away
    mbar_wait_bounded(bar_a, static_cast<uint32_t>(k & 1));
  }
}

__global__ void __launch_bounds__(256) k_finalize(const __grid_constant__ FParams p) {
  __shared__ double s_e[256], s_w[256];
  const int l = blockIdx.x, t = threadIdx.x;
  const int64_t b = p.tile_begin[l], e = p.tile_begin[l + 1];
  double se = 0.0, sw = 0.0;
  for (int64_t i = b + t; i < e; i += 256) {
    const double2 v = p.partials[p.tile_base + i];
    se += v.x;
    sw += v.y;
  }
  s_e[t] = se;
  s_w[t] = sw;
  __syncthreads();
  for (int h = 128; h > 0; h >>= 1) {
    if (t < h) {
      s_e[t] += s_e[t + h];
      s_w[t] += s_w[t + h];
    }
    __syncthreads();
  }
  if (t == 0) {
    const double E = s_e[0], W = s_w[0];
    const int gl = p.layer_base + l;
    if (p.sq_err) p.sq_err[gl] = E;
    if (p.sq_w) p.sq_w[gl] = W;
    if (p.rel_err) {
      float rel;
      if (E != E || W != W)
        rel = __int_as_float(0x7fffffff);
      else
        rel = W == 0.0 ? 0.0f : static_cast<float>(sqrt(E / W));
      p.rel_err[gl] = rel;
    }
  }
}

int64_t tiles_of(int64_t numel) { return (numel + kTile - 1) / kTile; }

template <int DT, bool SCORE>
cudaError_t launch_main(const QParams& p, cudaStream_t stream) {
  auto kern = k_quant_score<DT, SCORE>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (err != cudaSuccess) return err;
  int occ = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, kSmemBytes);
  if (err != cudaSuccess) return err;
  if (occ < 1) occ = 1;
  const int sms = current_sm_count();
  int64_t grid = static_cast<int64_t>(sms > 0 ? sms : 1) * occ;
  if (grid > p.num_tiles) grid = p.num_tiles;
  kern<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_main_dt(int dt, bool score, const QParams& p, cudaStream_t stream) {
  if (dt == AQNF4_BF16)
    return score ? launch_main<AQNF4_BF16, true>(p, stream)
                 : launch_main<AQNF4_BF16, false>(p, stream);
  return score ? launch_main<AQNF4_F16, true>(p, stream) : launch_main<AQNF4_F16, false>(p, stream);
}

void fill_tables(QParams& p, const Tables& tb) {
  p.curve_a = tb.curve_a;
  p.curve_b = tb.curve_b;
  for (int i = 0; i < 32; ++i) {
    p.slot_mid[i] = tb.slot_mid[i];
    p.slot_level[i] = tb.slot_level[i];
  }
  for (int i = 0; i < 16; ++i) p.level[i] = tb.level[i];
  for (int i = 0; i < 15; ++i) p.mid[i] = tb.mid[i];
}

aqnf4_status check_layer(const aqnf4_layer& L) {
  const int32_t score_bits = AQNF4_SCORE_DQ_ABSMAX | AQNF4_SCORE_DQ_CENTERED;
  if (!L.w || L.numel < 1 || (L.flags & ~score_bits) != 0 || L.flags == score_bits)
    return AQNF4_ERR_INVALID_ARG;
  if (!valid_dtype(L.dtype)) return AQNF4_ERR_DTYPE;
  if (L.codes8 && !L.scales) return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(L.w, 16) || !is_aligned(L.packed, 16) || !is_aligned(L.absmax, 4) ||
      (L.codes8 && !is_aligned(L.scales, 4)))
    return AQNF4_ERR_ALIGNMENT;
  return AQNF4_OK;
}

}  // namespace

// Built-in scratch for aqnf4_layer_error_noalloc: one (err, w^2) double pair per
// 16384-element tile, enough for 2^19 tiles (8.6e9 weights) in one call.  Every GPU that
// loads this library holds these 8 MiB until the process exits.
constexpr int64_t kNoallocTiles = int64_t(1) << 19;
static __device__ __align__(256) double2 g_noalloc_scratch[kNoallocTiles];

}  // namespace aqnf4

using namespace aqnf4;

namespace {
// Device address of g_noalloc_scratch, looked up once per device.  On the host the array's
// name is only a stand-in for the device copy and must never reach a kernel.
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

extern "C" {

size_t aqnf4_workspace_size(const aqnf4_layer* layers, int32_t num_layers) {
  if (!layers || num_layers < 1) return 0;
  int64_t tiles = 0;
  for (int32_t i = 0; i < num_layers; ++i) {
    if (layers[i].numel < 1) return 0;
    tiles += tiles_of(layers[i].numel);
  }
  const size_t bytes = static_cast<size_t>(tiles) * sizeof(double2);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

aqnf4_status aqnf4_quantize(const void* w, int32_t dtype, int64_t n, uint8_t* packed,
                            float* absmax, int32_t* dev_flag, cudaStream_t stream) {
  if (!w || n < 1) return AQNF4_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return AQNF4_ERR_DTYPE;
  if (!is_aligned(w, 16) || !is_aligned(packed, 16) || !is_aligned(absmax, 4) ||
      !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  const Tables* tb = default_tables();
  if (!tb) return AQNF4_ERR_CUDA;
  static thread_local QParams p;  // ~20 KB: keep it off the stack
  p.num_layers = 1;
  p.num_tiles = tiles_of(n);
  p.tile_base = 0;
  p.partials = nullptr;
  p.flag = dev_flag;
  fill_tables(p, *tb);
  p.tile_begin[0] = 0;
  p.tile_begin[1] = static_cast<int32_t>(p.num_tiles);
  p.layers[0] = LayerRec{w, packed, absmax, nullptr, nullptr, n, 0, 0};
  if (p.num_tiles > INT32_MAX) return AQNF4_ERR_INVALID_ARG;
  return launch_main_dt(dtype, false, p, stream) == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}

aqnf4_status aqnf4_layer_error(const aqnf4_layer* layers, int32_t num_layers, void* workspace,
                               size_t ws_bytes, double* sq_err, double* sq_w, float* rel_err,
                               int32_t* dev_flag, cudaStream_t stream) {
  if (!layers || num_layers < 1) return AQNF4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < num_layers; ++i) {
    const aqnf4_status st = check_layer(layers[i]);
    if (st != AQNF4_OK) return st;
  }
  if (!is_aligned(sq_err, 8) || !is_aligned(sq_w, 8) || !is_aligned(rel_err, 4) ||
      !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  const size_t need = aqnf4_workspace_size(layers, num_layers);
  if (!workspace || !is_aligned(workspace, 256) || ws_bytes < need) return AQNF4_ERR_WORKSPACE;
  const Tables* tb = default_tables();
  if (!tb) return AQNF4_ERR_CUDA;

  static thread_local QParams p;
  static thread_local FParams f;
  fill_tables(p, *tb);
  p.partials = static_cast<double2*>(workspace);
  p.flag = dev_flag;
  f.partials = static_cast<const double2*>(workspace);
  f.sq_err = sq_err;
  f.sq_w = sq_w;
  f.rel_err = rel_err;

  int64_t tile_base = 0;
  int32_t i = 0;
  while (i < num_layers) {
    const int32_t dt = layers[i].dtype;
    int32_t n = 0;
    int64_t tiles = 0;
    while (i + n < num_layers && n < kMaxLayersPerLaunch && layers[i + n].dtype == dt) {
      const aqnf4_layer& L = layers[i + n];
      const int64_t lt = tiles_of(L.numel);
      if (tiles + lt > INT32_MAX) break;
      p.tile_begin[n] = static_cast<int32_t>(tiles);
      f.tile_begin[n] = static_cast<int32_t>(tiles);
      p.layers[n] = LayerRec{L.w, L.packed, L.absmax, L.codes8, L.scales, L.numel, L.flags, 0};
      tiles += lt;
      ++n;
    }
    if (n == 0) return AQNF4_ERR_INVALID_ARG;  // a single layer above 2^31 tiles
    p.tile_begin[n] = static_cast<int32_t>(tiles);
    f.tile_begin[n] = static_cast<int32_t>(tiles);
    p.num_layers = n;
    p.num_tiles = tiles;
    p.tile_base = tile_base;
    f.num_layers = n;
    f.layer_base = i;
    f.tile_base = tile_base;
    if (launch_main_dt(dt, true, p, stream) != cudaSuccess) return AQNF4_ERR_CUDA;
    k_finalize<<<n, 256, 0, stream>>>(f);
    count_launches(1);
    if (cudaGetLastError() != cudaSuccess) return AQNF4_ERR_CUDA;
    tile_base += tiles;
    i += n;
  }
  return AQNF4_OK;
}

// Same pass as aqnf4_layer_error, for callers that cannot hand over device memory: the
// per-tile partial sums go to the library's own fixed scratch array instead of a workspace.
// The first call on each device looks the array's device address up (with that device
// current); make that first call before any stream capture on the device.  Nothing in the
// array needs clearing between calls: every tile slot a call reads was written earlier in
// the same call.  All calls on a device share the one array, so calls whose kernels
// overlap on the GPU (for example on two streams) race and must be serialised by the caller.
aqnf4_status aqnf4_layer_error_noalloc(const aqnf4_layer* layers, int32_t num_layers,
                                       double* sq_err, double* sq_w, float* rel_err,
                                       int32_t* dev_flag, cudaStream_t stream) {
  if (!layers || num_layers < 1) return AQNF4_ERR_INVALID_ARG;
  const size_t need = aqnf4_workspace_size(layers, num_layers);
  if (need == 0) return AQNF4_ERR_INVALID_ARG;
  const size_t have = sizeof(g_noalloc_scratch);
  if (need > have) return AQNF4_ERR_WORKSPACE;  // more than 2^19 tiles: split the call
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AQNF4_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
        return AQNF4_ERR_CUDA;
      g_noalloc_ptr[dev] = ptr;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return aqnf4_layer_error(layers, num_layers, scratch, have, sq_err, sq_w, rel_err, dev_flag,
                           stream);
}

}  // extern "C"
