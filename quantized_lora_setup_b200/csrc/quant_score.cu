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
// The sums are taken per block in the normalised domain, sum ((x - w_hat) r)^2 and
// sum v^2 in binary32 (each term <= 1, so nothing overflows or underflows for any finite
// input), then scaled by a_b^2 and summed in binary64 in a fixed order.
//
// Work decomposition (B200): a tile is 16384 consecutive elements of one layer (one DQ
// block).  A persistent CTA of 256 threads walks tiles with a grid stride; one thread owns
// one 64-element block.  A 1-D bulk copy (TMA engine) streams each 32 KB tile into a
// 2-stage shared-memory ring (two CTAs per SM), so the only global-load instructions are
// the copies issued by one thread.  Each thread reads its own 128 bytes back with conflict-free 16-byte loads
// (chunk order rotated per thread), takes the absmax with packed bf16x2/f16x2 max, one
// correctly rounded reciprocal, and finds each code with one round-toward-minus-infinity
// FMA (bucket index) plus two warp-shuffle table lookups and one compare.  Packed codes are
// staged in shared memory and written out with coalesced 16-byte stores.
#include <cfloat>

#include "device.cuh"

namespace aqnf4 {
namespace {

constexpr int kThreads = 256;  // = kDqBlock: one thread per NF4 block of a tile
constexpr int kStages = 2;
constexpr int kMaxLayersPerLaunch = 384;
constexpr int kWarps = kThreads / 32;

struct LayerRec {
  const void* w;
  uint8_t* packed;
  float* absmax;
  uint8_t* codes8;
  float* scales;
  int64_t numel;
};

struct QParams {
  int32_t num_layers;  // layers in this launch
  int32_t pad0;
  int64_t num_tiles;   // tiles in this launch
  int64_t tile_base;   // index of this launch's first tile in the partials array
  double2* partials;   // per tile (sum (x - w_hat)^2, sum x^2); score only
  int32_t* flag;       // optional device status word
  float bucket_mid[32];
  uint32_t bucket_code[32];
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

constexpr size_t kStageBytes = static_cast<size_t>(kStages) * kTileBytes;
constexpr size_t kOutBytes = 2 * kPackedTileBytes;
// per tile: one (sum err, sum w^2) double pair per thread and one absmax per warp, twice
constexpr size_t kRedBytes = 2 * (kThreads * sizeof(double2) + kWarps * sizeof(float));
constexpr size_t kSmemBytes = kStageBytes + kOutBytes + kRedBytes + kStages * 8 + 16;

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

// Thread 0: start the bulk copy of `tile` into stage `s`.  A short last tile copies its
// 16-byte-aligned prefix; the remaining < 8 elements are read from global memory later.
__device__ __forceinline__ void issue_tile(const QParams& p, int64_t tile, int s, uint8_t* stage,
                                          uint64_t* bars, uint64_t policy, int& cursor) {
  const TileGeom g = tile_geom(p, tile, cursor);
  const uint32_t bytes = static_cast<uint32_t>(g.cnt * 2) & ~15u;
  const uint32_t bar = smem_addr(bars + s);
  mbar_arrive_expect_tx(bar, bytes);
  if (bytes) {
    const uint8_t* src = static_cast<const uint8_t*>(p.layers[g.layer].w) + g.tin * kTileBytes;
    bulk_load(smem_addr(stage + static_cast<size_t>(s) * kTileBytes), src, bytes, bar, policy);
  }
}

// Generic per-element path for a block whose absmax is 0, below the binary32 normal range,
// or not finite.  Recomputes this thread's packed words and error sums.
template <int DT, bool SCORE>
__device__ __noinline__ void block_generic(const uint32_t* wl, int rot, float a,
                                           const QParams& p, uint8_t* ost, int t, double* se_out,
                                           double* sw_out) {
  using F = Fmt<DT>;
  const bool zero = (a == 0.0f);
  const bool finite = (a <= FLT_MAX);
  float scale = 1.0f, as = a;
  if (!zero && a < 0x1p-126f) {  // exact rescale keeps 1/a finite
    scale = 0x1p64f;
    as = __fmul_rn(a, scale);
  }
  const float r = zero ? 0.0f : __frcp_rn(as);
  float se = 0.0f, sw = 0.0f;
  for (int c = 0; c < 8; ++c) {
    const int k2 = (c - rot) & 7;
    uint32_t pk = 0;
    for (int i = 0; i < 8; ++i) {
      const uint32_t wd = wl[4 * k2 + (i >> 1)];
      const float x = (i & 1) ? F::hi(wd) : F::lo(wd);
      int code = 7;
      float v = 0.0f;
      if (!zero) {
        v = __fmul_rn(__fmul_rn(x, scale), r);
        code = 0;
        for (int j = 0; j < 15; ++j) code += (v > p.mid[j]) ? 1 : 0;
      }
      pk |= static_cast<uint32_t>(code) << ((i >> 1) * 8 + ((i & 1) ? 0 : 4));
      if (SCORE && !zero) {
        const float wh = F::round_trip(__fmul_rn(p.level[code], a));
        const float d = __fmul_rn(__fsub_rn(__fmul_rn(x, scale), __fmul_rn(wh, scale)), r);
        se = __fmaf_rn(d, d, se);
        sw = __fmaf_rn(v, v, sw);
      }
    }
    *reinterpret_cast<uint32_t*>(ost + t * 32 + c * 4) = pk;
  }
  // back to the weights' scale: (a * scale)^2 / scale^2
  const double as2 = static_cast<double>(as) * static_cast<double>(as);
  const double inv_s2 = 1.0 / (static_cast<double>(scale) * static_cast<double>(scale));
  double E = static_cast<double>(se) * as2 * inv_s2;
  double W = static_cast<double>(sw) * as2 * inv_s2;
  if (zero) E = W = 0.0;
  if (!finite) {
    E = W = __longlong_as_double(0x7ff8000000000000ll);
    if (p.flag) *p.flag = AQNF4_ERR_NONFINITE;
  }
  *se_out = E;
  *sw_out = W;
}

template <int DT, bool SCORE>
__global__ void __launch_bounds__(kThreads, 2) k_quant_score(const __grid_constant__ QParams p) {
  using F = Fmt<DT>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stage = smem;
  uint8_t* out_stage = smem + kStageBytes;
  double2* red_sum = reinterpret_cast<double2*>(out_stage + kOutBytes);        // [2][256]
  float* red_max = reinterpret_cast<float*>(red_sum + 2 * kThreads);           // [2][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStageBytes + kOutBytes + kRedBytes);
  int* abort_flag = reinterpret_cast<int*>(bars + kStages);

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // this lane's entries of the shuffle lookup tables
  const float tab_mid = p.bucket_mid[lane];
  const uint32_t tab_code = p.bucket_code[lane];
  const float tab_level = p.level[lane & 15];

  if (t == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(smem_addr(bars + s), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t T = p.num_tiles;
  const int64_t stride = gridDim.x;
  uint64_t policy = 0;
  int issue_cursor = 0, cursor = 0;
  if (t == 0) {
    policy = l2_evict_first_policy();
    for (int s = 0; s < kStages; ++s) {
      const int64_t tile = blockIdx.x + s * stride;
      if (tile < T) issue_tile(p, tile, s, stage, bars, policy, issue_cursor);
    }
  }

  int64_t k = 0;
  bool aborted = false;
  for (int64_t tile = blockIdx.x; tile < T; tile += stride, ++k) {
    const int s = static_cast<int>(k % kStages);
    const uint32_t parity = static_cast<uint32_t>((k / kStages) & 1);
    if (!mbar_wait_bounded(smem_addr(bars + s), parity)) {
      *abort_flag = 1;
      if (p.flag) *p.flag = AQNF4_ERR_TIMEOUT;
    }

    const TileGeom g = tile_geom(p, tile, cursor);
    const LayerRec& L = p.layers[g.layer];
    const int nblk = (g.cnt + kBlock - 1) / kBlock;
    const uint8_t* st = stage + static_cast<size_t>(s) * kTileBytes;

    // ---- this thread's 64 elements into registers
    uint32_t words[32];
    int rot;
    if (g.cnt == kTile) {
      rot = (t + (t >> 3)) & 7;  // conflict-free for the 16-byte reads and 4-byte writes
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) {
        const int c = (k2 + rot) & 7;
        const uint4 v = *reinterpret_cast<const uint4*>(st + t * 128 + c * 16);
        words[4 * k2 + 0] = v.x;
        words[4 * k2 + 1] = v.y;
        words[4 * k2 + 2] = v.z;
        words[4 * k2 + 3] = v.w;
      }
    } else {
      rot = 0;
      const int pre = static_cast<int>((static_cast<uint32_t>(g.cnt * 2) & ~15u) >> 1);
      const uint16_t* gw = static_cast<const uint16_t*>(L.w) + g.tin * kTile;
      const uint16_t* sw = reinterpret_cast<const uint16_t*>(st);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = t * 64 + 2 * j;
        const uint32_t lo = e < g.cnt ? (e < pre ? sw[e] : gw[e]) : 0u;
        const uint32_t hi = e + 1 < g.cnt ? (e + 1 < pre ? sw[e + 1] : gw[e + 1]) : 0u;
        words[j] = lo | (hi << 16);
      }
    }

    // ---- block absmax (NaN propagates)
    uint32_t m16[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) m16[i] = F::absmax2(words[2 * i], words[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 8; ++i) m16[i] = F::absmax2(m16[2 * i], m16[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) m16[i] = F::absmax2(m16[2 * i], m16[2 * i + 1]);
    m16[0] = F::absmax2(m16[0], m16[1]);
    m16[1] = F::absmax2(m16[2], m16[3]);
    m16[0] = F::absmax2(m16[0], m16[1]);
    m16[0] = F::absmax2(m16[0], __byte_perm(m16[0], 0, 0x1032));
    const float a = F::abs_lo(m16[0]);
    const bool fast = (a >= 0x1p-126f) && (a <= FLT_MAX);
    const float r = fast ? __frcp_rn(a) : 0.0f;

    // ---- codes, packing, error (all lanes run this so the shuffles stay converged)
    uint8_t* ost = out_stage + (k & 1) * kPackedTileBytes;
    float2 err2 = make_float2(0.0f, 0.0f), sw2 = make_float2(0.0f, 0.0f);
    const float2 r2 = make_float2(r, r), a2 = make_float2(a, a);
    const float2 scale2 = make_float2(15.5f, 15.5f), off2 = make_float2(8388624.0f, 8388624.0f);
#pragma unroll
    for (int k2 = 0; k2 < 8; ++k2) {
      const int c = (k2 + rot) & 7;
      uint32_t pk = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t wd = words[4 * k2 + j];
        const float2 x = make_float2(F::lo(wd), F::hi(wd));
        const float2 v = mul2_rn(x, r2);
        // floor(15.5 v + 16) lands in the low 5 bits of tt (2^23 <= tt < 2^23 + 32)
        const float2 tt = fma2_rm(v, scale2, off2);
        const int i0 = __float_as_int(tt.x), i1 = __float_as_int(tt.y);
        const float m0 = __shfl_sync(kFull, tab_mid, i0);
        const float m1 = __shfl_sync(kFull, tab_mid, i1);
        const uint32_t c0 = __shfl_sync(kFull, tab_code, i0) + (v.x > m0 ? 1u : 0u);
        const uint32_t c1 = __shfl_sync(kFull, tab_code, i1) + (v.y > m1 ? 1u : 0u);
        pk |= ((c0 << 4) | c1) << (8 * j);
        if (SCORE) {
          const float q0 = __shfl_sync(kFull, tab_level, static_cast<int>(c0));
          const float q1 = __shfl_sync(kFull, tab_level, static_cast<int>(c1));
          const float2 wq = mul2_rn(make_float2(q0, q1), a2);
          const uint32_t hb = F::pack_rn(wq.x, wq.y);
          const float2 d = mul2_rn(sub2_rn(x, make_float2(F::lo(hb), F::hi(hb))), r2);
          err2 = fma2_rn(d, d, err2);
          sw2 = fma2_rn(v, v, sw2);
        }
      }
      *reinterpret_cast<uint32_t*>(ost + t * 32 + c * 4) = pk;
    }
    const double a2d = static_cast<double>(a) * static_cast<double>(a);
    double e_t = static_cast<double>(err2.x + err2.y) * a2d;
    double w_t = static_cast<double>(sw2.x + sw2.y) * a2d;
    if (!fast) {
      uint32_t wl[32];  // stack copy: keeps `words` itself in registers
#pragma unroll
      for (int j = 0; j < 32; ++j) wl[j] = words[j];
      block_generic<DT, SCORE>(wl, rot, a, p, ost, t, &e_t, &w_t);
    }

    // ---- tile reductions: DQ scale (max a over the tile's blocks) and error sums
    float am = t < nblk ? a : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) am = fmax_nan(am, __shfl_xor_sync(kFull, am, off));
    double2* rs = red_sum + (k & 1) * kThreads;
    float* rm = red_max + (k & 1) * kWarps;
    if (SCORE) rs[t] = make_double2(e_t, w_t);
    if (lane == 0) rm[warp] = am;
    __syncthreads();
    if (*abort_flag) {
      aborted = true;
      break;
    }
    if (t == 0) {
      const int64_t next = tile + kStages * stride;
      if (next < T) {
        fence_proxy_async_smem();
        issue_tile(p, next, s, stage, bars, policy, issue_cursor);
      }
    }

    // ---- outputs
    const int64_t blk0 = g.tin * kDqBlock;
    float sdq = rm[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) sdq = fmax_nan(sdq, rm[w]);
    if (t < nblk) {
      if (L.absmax) L.absmax[blk0 + t] = a;
      if (L.codes8) L.codes8[blk0 + t] = dq_code(a, sdq);
    }
    if (t == 0 && L.codes8) {
      L.scales[g.tin] = sdq;
      if (!(sdq <= FLT_MAX) && p.flag) *p.flag = AQNF4_ERR_NONFINITE;
    }
    if (SCORE && warp == 0) {
      double se = 0.0, sw = 0.0;
#pragma unroll
      for (int j = 0; j < kThreads / 32; ++j) {
        const double2 v = rs[lane + 32 * j];
        se += v.x;
        sw += v.y;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        se += __shfl_xor_sync(kFull, se, off);
        sw += __shfl_xor_sync(kFull, sw, off);
      }
      if (lane == 0) p.partials[p.tile_base + tile] = make_double2(se, sw);
    }
    if (L.packed) {
      uint8_t* gp = L.packed + g.tin * kPackedTileBytes;
      if (g.cnt == kTile) {
#pragma unroll
        for (int i = t; i < kPackedTileBytes / 16; i += kThreads)
          *reinterpret_cast<uint4*>(gp + 16 * i) = *reinterpret_cast<const uint4*>(ost + 16 * i);
      } else {
        const int nbytes = (g.cnt + 1) >> 1;
        for (int i = t; i < nbytes; i += kThreads) {
          uint8_t b = ost[i];
          if ((g.cnt & 1) && i == nbytes - 1) b &= 0xF0;  // odd length: low nibble stays 0
          gp[i] = b;
        }
      }
    }
  }

  if (aborted && t == 0) {
    // let every bulk copy this CTA still has in flight land before the CTA exits
    for (int64_t kk = k; kk < k + kStages; ++kk) {
      const int64_t tile = blockIdx.x + kk * stride;
      if (tile >= T) break;
      mbar_wait_bounded(smem_addr(bars + (kk % kStages)), static_cast<uint32_t>((kk / kStages) & 1));
    }
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
  for (int i = 0; i < 32; ++i) {
    p.bucket_mid[i] = tb.bucket_mid[i];
    p.bucket_code[i] = tb.bucket_code[i];
  }
  for (int i = 0; i < 16; ++i) p.level[i] = tb.level[i];
  for (int i = 0; i < 15; ++i) p.mid[i] = tb.mid[i];
}

aqnf4_status check_layer(const aqnf4_layer& L) {
  if (!L.w || L.numel < 1 || L.reserved != 0) return AQNF4_ERR_INVALID_ARG;
  if (!valid_dtype(L.dtype)) return AQNF4_ERR_DTYPE;
  if (L.codes8 && !L.scales) return AQNF4_ERR_INVALID_ARG;
  if (!is_aligned(L.w, 16) || !is_aligned(L.packed, 16) || !is_aligned(L.absmax, 4) ||
      (L.codes8 && !is_aligned(L.scales, 4)))
    return AQNF4_ERR_ALIGNMENT;
  return AQNF4_OK;
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

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
  p.layers[0] = LayerRec{w, packed, absmax, nullptr, nullptr, n};
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
      p.layers[n] = LayerRec{L.w, L.packed, L.absmax, L.codes8, L.scales, L.numel};
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

}  // extern "C"
