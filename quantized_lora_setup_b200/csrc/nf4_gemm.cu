// nf4_gemm.cu -- the forward product of a layer stored in NF4 + DQ on the tensor cores
// (aqnf4_nf4_linear): y = x w_hat^T.
//
// "QLoRA", "How It Works": a training pass computes with 16-bit values rebuilt from the
// 4-bit storage.  Here that rebuilding happens inside the GEMM: w_hat never
// exists in HBM.  For element (n, k) of the N x K layer (block b = (n K + k) / 64):
//   a'_b = fl(fl(code8_b / 255) * scales[b / 256]),  w_hat = dtype_rn(fl(level[code] * a'_b)),
// bit for bit what aqnf4_dequantize writes; then y = x w_hat^T with binary32 accumulation.
//
// Blackwell structure.  One CTA (18 warps, one per SM) computes a 256 x 256 tile of y over
// K in steps of 64, its roles specialised and coupled only through mbarriers:
//   - warp 16 streams, by TMA and up to kStagesA steps ahead, the step's x tile (M x K, K
//     contiguous; 128-byte-swizzled 256 x 64);
//   - warps 0-15 dequantize the step's 256-row slice of the layer into a 256 x 64 w_hat tile
//     (one of kStagesB) -- threads 2r and 2r + 1 take the two halves of row n0 + r, one NF4
//     block per row and step (K is a multiple of 64) -- in the same swizzled K-major layout,
//     16 bytes at a time, and arrive on the tile's barrier.  Each thread loads its packed
//     codes, the block's 8-bit constant and its DQ scale from global memory kStagesB steps
//     ahead into registers, so a w_hat tile can be rebuilt as soon as the tensor cores
//     release it, without waiting for a copy;
//   - warp 17 issues eight tcgen05.mma per step (M 128, N 256, K 16, bf16/f16 in, f32 out):
//     each x row half against the same w_hat tile, into two TMEM accumulators that fill all
//     512 columns, so every dequantized element feeds 256 rows of x; tcgen05.commit frees
//     the stage when they finish;
//   - warps 0-15 then read the accumulators with tcgen05.ld, stage each 128-row accumulator
//     in the idle rings and write y in whole rows.
// When the output has too few tiles to fill the GPU, K is split over up to 8 CTAs that form
// one thread-block cluster per tile; they add their partial sums through distributed shared
// memory instead of a trip through HBM and a second kernel.  With two or more row tiles and
// no split, two row tiles run on a CTA pair with two-CTA MMAs (tcgen05.mma.cta_group::2,
// M = 256 of which 128 rows from each CTA, N = 256 of which each CTA holds and dequantizes
// 128 w_hat rows): each CTA rebuilds half the w_hat tile, and the tensor cores read a
// w_hat row from shared memory once per 512 rows of x instead of once per 128.  A pair's
// dequantizing warps work in four groups that take the steps in turn, one thread per row.
// Every wait is bounded: a wait that gives up records AQNF4_ERR_TIMEOUT and makes every role
// stop; copies in flight are allowed to land and the TMEM is always freed before exit.
#include <cuda.h>

#include <mutex>

#include "device.cuh"

namespace aqnf4 {
namespace {

constexpr int kBM = 256, kBN = 256, kBK = 64;  // two 128-row accumulators
// ring depths: x tiles (TMA) and w_hat tiles (dequantized); the dequantizing loop is unrolled
// by kStagesB, so each of its steps works on a fixed tile and a fixed register set.  A fourth
// x tile measured slower: the 231 KB of shared memory it takes leave too little of the SM's
// on-chip memory to the L1 that serves the dequantizing warps' global loads.
constexpr int kStagesA = 3, kStagesB = 3;
constexpr int kDeqWarps = 16, kProducerWarp = 16, kMmaWarp = 17;
// A CTA pair's dequantizing warps take the steps in four groups of four warps, in turn: a
// thread rebuilds a whole 64-element row of its half of the w_hat tile every fourth step,
// so the per-step costs (waits, loads, the arrival) are paid once per 64 elements.
constexpr int kPairGroups = 4;
constexpr int kGThreads = 32 * (kDeqWarps + 2);            // 576
constexpr int kTileBytesA = kBM * kBK * 2;                  // 32 KB of x
constexpr int kTileBytesB = kBN * kBK * 2;                  // 32 KB of w_hat
constexpr int kRingB = kStagesA * kTileBytesA;              // the w_hat ring follows the x ring
constexpr int kBarBase = kRingB + kStagesB * kTileBytesB;   // after the rings
constexpr int kFracOff = kBarBase + 256;                     // fl(c / 255) for c = 0..255
constexpr int kGSmemBytes = kFracOff + 1024 + 1024;         // + alignment slack
constexpr uint32_t kTmemCols = 512;  // two f32 accumulators of 256 columns: all of TMEM
// split K: the splits of one output tile form a thread-block cluster (portable size <= 8);
// each stages a 128 x 256 binary32 accumulator in its (then idle) rings for the others
constexpr int kMaxSplits = 8;
constexpr int kStageBytes = 128 * kBN * 4;
static_assert(kStageBytes <= kBarBase, "the staged accumulator fits in the rings");

// Ring geometry of each form.  A CTA pair's w_hat tile is half as large (128 rows), which
// leaves room for a fourth x tile and a fourth w_hat tile in the same shared memory.
template <bool PAIR>
struct Ring {
  static constexpr int SA = PAIR ? 4 : kStagesA;                     // x tiles
  static constexpr int SB = PAIR ? 4 : kStagesB;                     // w_hat tiles
  static constexpr int TB = (PAIR ? kBN / 2 : kBN) * kBK * 2;        // bytes of a w_hat tile
  static constexpr int RingB = SA * kTileBytesA;                     // w_hat ring offset
  static constexpr int BarBase = RingB + SB * TB;                    // barriers
  static constexpr int FracOff = BarBase + 256;                      // fl(c / 255) table
  static_assert(FracOff + 1024 + 1024 <= kGSmemBytes, "both forms fit the same allocation");
  static_assert(2 * (SA + SB) * 8 + 8 + 16 <= 256, "the barriers fit their region");
};
static_assert(kDeqWarps * 16 == kBN, "two dequantizing threads per row of the w_hat tile");

struct GParams {
  const uint8_t* packed;
  const uint8_t* codes8;
  const float* scales;
  void* y;
  int64_t M, N, K;
  int32_t out_f32;
  int32_t splits;     // K is split over the gridDim.z CTAs of one cluster (<= kMaxSplits)
  int32_t* flag;
  int32_t a_rows;     // rows of x one copy brings: 128 when M <= 128 (the rest unused)
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
// N = 256, M = 128 (one of the two row halves of the tile; a CTA pair's MMA: M = 256, 128
// rows from each CTA).
template <int DT, int M = 128>
__host__ __device__ constexpr uint32_t idesc() {
  return (1u << 4) | (static_cast<uint32_t>(DT) << 7) | (static_cast<uint32_t>(DT) << 10) |
         (static_cast<uint32_t>(kBN >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
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

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// Thread-block cluster: a barrier over all threads of the cluster (release / acquire: the
// shared-memory writes before it are visible to every CTA of the cluster after it), the
// address of the same shared-memory location in CTA `rank`, and loads from there.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 ld_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// ---- CTA pair (two row tiles of y over one w_hat tile, one 1 x 2 x 1 cluster): the even
// CTA (the leader) issues tcgen05.mma.cta_group::2 with M = 256 (128 rows of x from each
// CTA) and N = 256, where each CTA holds 128 of the 256 w_hat rows; each CTA's TMEM receives
// its own rows.  Both CTAs' x copies and dequantizing warps complete on the leader's
// barriers; the leader's commits arrive on both CTAs' barriers.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x,
                                                 int y, uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t tmem, uint64_t da, uint64_t db,
                                              uint32_t id, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
      "l"(da), "l"(db), "r"(id), "r"(accumulate)
      : "memory");
}

// arrives on the barrier at this offset in both CTAs of the pair once the MMAs have finished
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// barrier over the dequantizing warps alone (named barrier 1)
__device__ __forceinline__ void deq_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDeqWarps) : "memory");
}

// arrival on a barrier of another CTA of the cluster
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

template <int DT, bool PAIR>
__global__ void __launch_bounds__(kGThreads, 1) k_nf4_gemm(const __grid_constant__ CUtensorMap tmap_x,
                                                           const __grid_constant__ GParams p) {
  using F = Fmt<DT>;
  using G = Ring<PAIR>;
  constexpr int kStagesA = G::SA, kStagesB = G::SB, kTileBytesB = G::TB, kRingB = G::RingB,
                kBarBase = G::BarBase, kFracOff = G::FracOff;
  extern __shared__ uint8_t smem_raw[];
  // the swizzled tiles need 1024-byte alignment
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + kBarBase);  // x tile landed
  uint64_t* empty_a = full_a + kStagesA;                            // x tile consumed
  uint64_t* full_b = empty_a + kStagesA;                            // w_hat tile written
  uint64_t* empty_b = full_b + kStagesB;                            // w_hat tile consumed
  uint64_t* accum = empty_b + kStagesB;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* fail_word = const_cast<int*>(abort_flag) + 1;  // split K: read by the cluster's CTAs
  float* frac = reinterpret_cast<float*>(smem + kFracOff);

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t < 256) frac[t] = __fdiv_rn(static_cast<float>(t), 255.0f);  // correctly rounded
  // tiles: column tile on grid x and row tile on y.  A pair's two CTAs are neighbours along
  // grid x (the cluster's x, as a two-CTA MMA needs): cluster k = blockIdx.x / 2 takes column
  // tile k mod (column tiles) of row tiles 2 (k / column tiles) + {0, 1}, so the clusters
  // resident at once share their rows of x through L2, as the unpaired grid order does.
  const int64_t col_tiles = (p.N + kBN - 1) / kBN;
  const int64_t pair_k = static_cast<int64_t>(blockIdx.x >> 1);
  const int64_t n0 = (PAIR ? pair_k % col_tiles : static_cast<int64_t>(blockIdx.x)) * kBN;
  const int64_t m0 =
      (PAIR ? 2 * (pair_k / col_tiles) + (blockIdx.x & 1) : static_cast<int64_t>(blockIdx.y)) *
      kBM;
  const int64_t kb = p.K / kBK;  // NF4 blocks per row of w = k steps
  // this CTA's steps [kt0, kt1): split z of p.splits (the pipeline counts i = kt - kt0)
  const int64_t kt0 = kb * blockIdx.z / p.splits, kt1 = kb * (blockIdx.z + 1) / p.splits;
  const int64_t nk = kt1 - kt0;
  const bool lower_half = m0 + 128 < p.M;  // the tile's second 128 rows hold any of x
  // CTA pair: rank q = blockIdx.x mod 2 (a 2 x 1 x 1 cluster); the leader (q = 0) issues the
  // MMAs.  Its lower_half covers the partner's too (the partner's rows lie further down).
  const uint32_t q_rank = PAIR ? (blockIdx.x & 1u) : 0u;
  const bool mma_cta = !PAIR || q_rank == 0;

  if (t == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(smem_addr(full_a + s), 1);
      mbar_init(smem_addr(empty_a + s), 1);
    }
    for (int s = 0; s < kStagesB; ++s) {
      // pair: one arrival per dequantizing warp of the tile's group in either CTA, on the
      // leader's barrier
      mbar_init(smem_addr(full_b + s), PAIR ? 2 * kDeqWarps / kPairGroups : 32 * kDeqWarps);
      mbar_init(smem_addr(empty_b + s), 1);
    }
    mbar_init(smem_addr(accum), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (PAIR) {
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before either arrives on the other's
  }
  if (warp == kMmaWarp) {
    if (PAIR) {  // the same warp of both CTAs allocates the pair's TMEM together
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_addr(tmem_holder)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_addr(tmem_holder)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  int64_t issued = 0;  // producer: x copies issued (step i went to tile i mod kStagesA)

  if (warp == kProducerWarp) {
    if (lane == 0) {
      for (int64_t i = 0; i < nk && !*abort_flag; ++i) {
        const int s = static_cast<int>(i % kStagesA);
        const uint32_t use = static_cast<uint32_t>(i / kStagesA);
        if (i >= kStagesA &&
            !(PAIR ? mbar_wait_bounded(smem_addr(empty_a + s), (use - 1) & 1)
                   : mbar_wait_bounded(smem_addr(empty_a + s), (use - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        if (PAIR) {  // both CTAs' copies complete on the leader's barrier
          if (q_rank == 0) mbar_arrive_expect_tx(smem_addr(full_a + s), 2u * kTileBytesA);
          tma_load_2d_pair(smem_addr(smem + s * kTileBytesA), &tmap_x,
                           static_cast<int>((kt0 + i) * kBK), static_cast<int>(m0),
                           cluster_map(smem_addr(full_a + s), 0u));
        } else {
          mbar_arrive_expect_tx(smem_addr(full_a + s), static_cast<uint32_t>(p.a_rows) * kBK * 2);
          tma_load_2d(smem_addr(smem + s * kTileBytesA), &tmap_x,
                      static_cast<int>((kt0 + i) * kBK), static_cast<int>(m0),
                      smem_addr(full_a + s));
        }
        issued = i + 1;
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && mma_cta) {
      for (int64_t i = 0; i < nk && !*abort_flag; ++i) {
        const int sa = static_cast<int>(i % kStagesA), sb = static_cast<int>(i % kStagesB);
        const uint32_t pa = static_cast<uint32_t>(i / kStagesA) & 1;
        const uint32_t pb = static_cast<uint32_t>(i / kStagesB) & 1;
        const bool ok = PAIR ? mbar_wait_bounded(smem_addr(full_a + sa), pa) &&
                                   mbar_wait_bounded(smem_addr(full_b + sb), pb)
                             : mbar_wait_bounded(smem_addr(full_a + sa), pa) &&
                                   mbar_wait_bounded(smem_addr(full_b + sb), pb);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_addr(smem + sa * kTileBytesA);
        const uint32_t b0 = smem_addr(smem + kRingB + sb * kTileBytesB);
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j) {  // K = 16 per MMA: 32 bytes along the swizzled row
          // rows 0..127 of x into columns 0..255 of TMEM, rows 128..255 into 256..511; both
          // use the same dequantized w_hat tile (pair: the same rows of both CTAs' x, and
          // the w_hat rows 0..127 held by the leader and 128..255 by the partner)
          const uint32_t acc = (i > 0 || j > 0) ? 1u : 0u;
          if (PAIR)
            umma_f16_pair(tmem, sw128_desc(a0 + 32 * j), sw128_desc(b0 + 32 * j),
                          idesc<DT, 256>(), acc);
          else
            umma_f16(tmem, sw128_desc(a0 + 32 * j), sw128_desc(b0 + 32 * j), idesc<DT>(), acc);
          if (lower_half) {  // uniform: skipped when those 128 rows lie past M
            if (PAIR)
              umma_f16_pair(tmem + kBN, sw128_desc(a0 + 128 * 128 + 32 * j),
                            sw128_desc(b0 + 32 * j), idesc<DT, 256>(), acc);
            else
              umma_f16(tmem + kBN, sw128_desc(a0 + 128 * 128 + 32 * j), sw128_desc(b0 + 32 * j),
                       idesc<DT>(), acc);
          }
        }
        // each arrives once the MMAs above have finished (pair: in both CTAs)
        if (PAIR) {
          umma_commit_pair(smem_addr(empty_a + sa));
          umma_commit_pair(smem_addr(empty_b + sb));
        } else {
          umma_commit(smem_addr(empty_a + sa));
          umma_commit(smem_addr(empty_b + sb));
        }
      }
      // arrives once every MMA issued above has finished
      if (PAIR)
        umma_commit_pair(smem_addr(accum));
      else
        umma_commit(smem_addr(accum));
    }
  } else {
    // ---- dequantizing warps: threads 2r and 2r + 1 own the two halves of row n0 + r of the
    // w_hat tile.  A pair's CTA q holds rows n0 + 128 q + r (r < 128) at tile row r, and its
    // dequantizing warps form kPairGroups groups that take the steps in turn (group g: steps
    // i = g mod kPairGroups); thread r of a group rebuilds all of row r.  Step i's packed
    // codes, 8-bit constant and DQ scale are loaded from global memory kStagesB steps ahead;
    // the loop is unrolled over the group's register sets, one per w_hat tile it uses.
    constexpr int kGroups = PAIR ? kPairGroups : 1;
    constexpr int kSets = kStagesB / kGroups;
    static_assert(kSets * kGroups == kStagesB, "each group owns whole w_hat tiles");
    constexpr int kTpr = PAIR && kGroups == 4 ? 1 : 2;  // threads per w_hat row
    constexpr int kVec = 2 / kTpr;                      // 16-byte code loads per thread and step
    const int grp = warp / (kDeqWarps / kGroups);
    const int tg = t - grp * (32 * kDeqWarps / kGroups);  // thread within its group
    const float tab_level = p.level[lane & 15];  // lanes 16..31 mirror 0..15
    const int r = tg / kTpr, hf = tg % kTpr;
    const int64_t n = n0 + 128 * static_cast<int64_t>(q_rank) + r;
    const bool row_ok = n < p.N;
    const uint8_t* prow = p.packed + n * (p.K / 2) + hf * 16;
    struct Codes {
      uint4 v[kVec];
    };
    auto fetch = [&](int64_t kt, Codes& pk, uint32_t& c, float& s8) {
      if (row_ok && kt < kt1) {
        const int64_t b = n * kb + kt;
#pragma unroll
        for (int k = 0; k < kVec; ++k)
          pk.v[k] = __ldg(reinterpret_cast<const uint4*>(prow + kt * (kBK / 2) + 16 * k));
        c = __ldg(p.codes8 + b);
        s8 = __ldg(p.scales + (b >> 8));
      }
    };
    // one step into w_hat tile u; false when the pipeline has been aborted
    auto dequant = [&](int64_t i, int u, const Codes& pk, uint32_t c8, float sc) -> bool {
      const uint32_t par = static_cast<uint32_t>(i / kStagesB - 1) & 1;
      bool ok = i < kStagesB || mbar_wait_bounded(smem_addr(empty_b + u), par);
      if (!ok) *abort_flag = 1;
      if (__any_sync(kFull, *abort_flag != 0)) return false;  // warp-uniform (shuffles below)
      // a zero constant (also for rows past N) gives 0
      const float ap = row_ok ? __fmul_rn(frac[c8], sc) : 0.0f;
      const f32x2 a2 = pair(ap, ap);
      uint32_t words[4 * kVec];
#pragma unroll
      for (int k = 0; k < kVec; ++k) {
        words[4 * k] = pk.v[k].x;
        words[4 * k + 1] = pk.v[k].y;
        words[4 * k + 2] = pk.v[k].z;
        words[4 * k + 3] = pk.v[k].w;
      }
      uint8_t* rowb = smem + kRingB + u * kTileBytesB + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int jj = 0; jj < 4 * kVec; ++jj) {
        const uint32_t w = words[jj];
        uint32_t o[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          // byte h: element 2h in the high nibble, 2h + 1 in the low nibble
          const float q0 = __shfl_sync(kFull, tab_level, static_cast<int>(w >> (8 * h + 4)));
          const float q1 = __shfl_sync(kFull, tab_level, static_cast<int>(w >> (8 * h)));
          const f32x2 v = pmul_rn(pair(q0, q1), a2);
          o[h] = F::pack_rn(pair_lo(v), pair_hi(v));
        }
        const int j = 4 * hf + jj;  // 16-byte chunk of the 128-byte row
        *reinterpret_cast<uint4*>(rowb + ((j ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();  // the tensor cores read this tile through the async proxy
      if (PAIR) {  // one arrival per warp, on the leader's barrier
        __syncwarp();
        if (lane == 0) {
          if (q_rank == 0)
            mbar_arrive(smem_addr(full_b + u));
          else
            mbar_arrive_remote(cluster_map(smem_addr(full_b + u), 0u));
        }
      } else {
        mbar_arrive(smem_addr(full_b + u));
      }
      return true;
    };
    // register set v (fully unrolled, so it stays in registers) holds the inputs of the
    // group's step that uses w_hat tile u = v kGroups + grp
    Codes pkr[kSets];
    uint32_t cr[kSets];
    float sr[kSets];
#pragma unroll
    for (int v = 0; v < kSets; ++v) {
#pragma unroll
      for (int k = 0; k < kVec; ++k) pkr[v].v[k] = make_uint4(0, 0, 0, 0);
      cr[v] = 0;
      sr[v] = 0.0f;
      fetch(kt0 + v * kGroups + grp, pkr[v], cr[v], sr[v]);
    }
    bool going = true;
    for (int64_t i0 = 0; i0 < nk && going; i0 += kStagesB) {
#pragma unroll
      for (int v = 0; v < kSets; ++v) {
        const int u = v * kGroups + grp;
        const int64_t i = i0 + u;
        if (going) {
          if (i >= nk || !dequant(i, u, pkr[v], cr[v], sr[v])) {
            going = false;
          } else {
            fetch(kt0 + i + kStagesB, pkr[v], cr[v], sr[v]);
          }
        }
      }
    }
  }

  // ---- accumulator ready?  (decided uniformly: tcgen05.ld is warp-collective)
  const bool ready =
      warp < kDeqWarps
          ? (PAIR ? mbar_wait_bounded(smem_addr(accum), 0) : mbar_wait_bounded(smem_addr(accum), 0))
          : true;
  const int failed = __syncthreads_or(!ready || *abort_flag);
  tc_fence_after();
  if (failed && t == 0 && p.flag) *p.flag = AQNF4_ERR_TIMEOUT;
  if (p.splits == 1 && !failed && warp < kDeqWarps) {
    // y, one 128-row accumulator at a time, through the (now idle) rings: warp w reads TMEM
    // lanes 32 (w mod 4).. (rows) and columns 64 (w / 4).., converts to y's format and stages
    // the rows in shared memory (16-byte chunk j of row r at j ^ (r mod 8): neither these
    // stores nor the reads below conflict on banks); then each warp writes whole rows of the
    // tile, 512 or 1024 contiguous bytes per row, rows w, w + 16, ..  The dequantizing warps
    // alone take part (named barrier 1); the staging needs 128 x 256 x 4 bytes at most.
    static_assert(128 * kBN * 4 <= Ring<PAIR>::BarBase, "a staged accumulator fits in the rings");
    const bool f32o = p.out_f32 != 0;
    const int esz = f32o ? 4 : 2;
    const int row_bytes = kBN * esz;    // 1024 or 512
    const int per = 16 / esz;           // elements per 16-byte chunk
    const int chunks = row_bytes / 16;  // 64 or 32 per row
    const bool vec = f32o ? (p.N & 3) == 0 : (p.N & 7) == 0;  // 16-byte aligned rows of y
    const int q = warp & 3, cq = warp >> 2;
    const int rr = 32 * q + lane;
    for (int hh = 0; hh < (lower_half ? 2 : 1); ++hh) {
      if (hh > 0) deq_bar_sync();  // the first half's rows have been read out
      uint8_t* srow = smem + rr * row_bytes;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v[32];
        const int cbase = 64 * cq + 32 * c;
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + kBN * hh + cbase, v);
        if (f32o) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int j = cbase / 4 + i;
            *reinterpret_cast<float4*>(srow + ((j ^ (rr & 7)) << 4)) =
                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = cbase / 8 + i;
            *reinterpret_cast<uint4*>(srow + ((j ^ (rr & 7)) << 4)) = make_uint4(
                F::pack_rn(v[8 * i], v[8 * i + 1]), F::pack_rn(v[8 * i + 2], v[8 * i + 3]),
                F::pack_rn(v[8 * i + 4], v[8 * i + 5]), F::pack_rn(v[8 * i + 6], v[8 * i + 7]));
          }
        }
      }
      deq_bar_sync();  // the half is staged
#pragma unroll 1
      for (int k = 0; k < 128 / kDeqWarps; ++k) {
        const int r2 = warp + kDeqWarps * k;
        const int64_t m = m0 + 128 * hh + r2;
        if (m >= p.M) break;  // warp-uniform; later rows lie further down
        for (int j = lane; j < chunks; j += 32) {
          const uint4 val = lds128(smem + r2 * row_bytes + ((j ^ (r2 & 7)) << 4));
          const int64_t col = n0 + static_cast<int64_t>(j) * per;
          if (col >= p.N) continue;
          uint8_t* dst = static_cast<uint8_t*>(p.y) + (m * p.N + col) * esz;
          if (vec && col + per <= p.N) {
            *reinterpret_cast<uint4*>(dst) = val;
          } else {
            for (int e = 0; e < per && col + e < p.N; ++e) {
              const int k = f32o ? e : e >> 1;  // the 32-bit word holding element e
              const uint32_t w = k == 0 ? val.x : k == 1 ? val.y : k == 2 ? val.z : val.w;
              if (f32o)
                reinterpret_cast<uint32_t*>(dst)[e] = w;
              else
                reinterpret_cast<uint16_t*>(dst)[e] = static_cast<uint16_t>(w >> (16 * (e & 1)));
            }
          }
        }
      }
    }
  }
  if (p.splits > 1) {
    // Split K over the cluster's CTAs (cluster rank = blockIdx.z = split).  For each
    // 128-row accumulator: every CTA stages its binary32 partial in its own rings (row-major,
    // 16-byte chunk j of row r at position j ^ (r mod 8), so that neither the staging stores
    // nor the reads below conflict on banks); after a cluster barrier, CTA z adds, for rows
    // [z rows / S, (z + 1) rows / S), the S partials in split order (the bits do not depend
    // on scheduling) through distributed shared memory and stores y; a second barrier keeps
    // every CTA's rings alive until the others have read them.  Every thread of the cluster
    // takes the same barriers; if any CTA of the cluster timed out, no CTA writes y.
    const int S = p.splits, z = static_cast<int>(blockIdx.z);
    if (t == 0) *fail_word = failed;
    const int cols = static_cast<int>(p.N - n0 < kBN ? p.N - n0 : kBN);
    const bool vec = (p.N & 3) == 0;
    const uint32_t stage = smem_addr(smem);
    int any_failed = 0;
    for (int hh = 0; hh < (lower_half ? 2 : 1); ++hh) {
      const int64_t r0 = m0 + 128 * hh;  // first row of y in this accumulator
      const int rows = static_cast<int>(p.M - r0 < 128 ? p.M - r0 : 128);
      if (!failed && warp < kDeqWarps && 32 * (warp & 3) < rows) {
        // warp w: TMEM lanes 32 (w mod 4).. = rows; columns 64 (w / 4)..
        const int q = warp & 3, cq = warp >> 2;
        const int r = 32 * q + lane;
        uint8_t* row = smem + r * (kBN * 4);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float v[32];
          const int cbase = 64 * cq + 32 * c;
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + kBN * hh + cbase, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int j = cbase / 4 + i;
            *reinterpret_cast<float4*>(row + ((j ^ (r & 7)) << 4)) =
                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
      cluster_sync();
      if (hh == 0)
        for (int s2 = 0; s2 < S; ++s2)
          any_failed |= ld_cluster_s32(cluster_map(smem_addr(fail_word), static_cast<uint32_t>(s2)));
      if (!any_failed) {
        const int lo = rows * z / S, hi = rows * (z + 1) / S;
        uint32_t peer[kMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2)
          peer[s2] = s2 < S ? cluster_map(stage, static_cast<uint32_t>(s2)) : 0u;
        const int nchunk = (cols + 3) >> 2;
        for (int e = t; e < (hi - lo) * nchunk; e += kGThreads) {
          const int r = lo + e / nchunk, j = e % nchunk;
          const uint32_t off = static_cast<uint32_t>(r * (kBN * 4) + ((j ^ (r & 7)) << 4));
          float4 u[kMaxSplits];
#pragma unroll
          for (int s2 = 0; s2 < kMaxSplits; ++s2)
            if (s2 < S) u[s2] = ld_cluster_v4(peer[s2] + off);
          float4 acc = u[0];
#pragma unroll
          for (int s2 = 1; s2 < kMaxSplits; ++s2)
            if (s2 < S)
              acc = make_float4(__fadd_rn(acc.x, u[s2].x), __fadd_rn(acc.y, u[s2].y),
                                __fadd_rn(acc.z, u[s2].z), __fadd_rn(acc.w, u[s2].w));
          const int64_t i = (r0 + r) * p.N + n0 + 4 * j;
          if (vec) {  // N, hence cols, a multiple of 4: whole 16- (8-) byte stores
            if (p.out_f32)
              *reinterpret_cast<float4*>(static_cast<float*>(p.y) + i) = acc;
            else
              *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.y) + i) =
                  make_uint2(F::pack_rn(acc.x, acc.y), F::pack_rn(acc.z, acc.w));
          } else {
            const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
            for (int k = 0; k < 4 && 4 * j + k < cols; ++k) {
              if (p.out_f32)
                static_cast<float*>(p.y)[i + k] = a4[k];
              else
                static_cast<uint16_t*>(p.y)[i + k] =
                    static_cast<uint16_t>(F::pack_rn(a4[k], 0.0f) & 0xffffu);
            }
          }
        }
      }
      cluster_sync();
    }
  }
  if (warp == kProducerWarp && lane == 0 && failed && mma_cta) {
    // let every copy issued land before the shared memory goes away: tile s last received
    // step s + kStagesA * ((issued - 1 - s) / kStagesA).  (A pair's partner counts its copies
    // on the leader's barriers, which it cannot wait on.  Its producer issues a copy only
    // after the leader's MMAs released the tile, and the leader gives up only after a
    // bounded wait of seconds on the missing copy, so nothing it issued is still in flight
    // when the pair passes the barrier below.)
    for (int s = 0; s < kStagesA && s < issued; ++s)
      mbar_wait_bounded(smem_addr(full_a + s),
                        static_cast<uint32_t>((issued - 1 - s) / kStagesA) & 1);
  }
  tc_fence_before();
  __syncthreads();
  // pair: neither CTA frees the TMEM or leaves while the other may still use its barriers
  if (PAIR) cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
  }
}

// Splits of K for a grid too small to fill the GPU: enough CTAs for one wave, at least 8
// steps of 64 per split, at most kMaxSplits (one cluster per output tile).
int choose_splits(int64_t M, int64_t N, int64_t K) {
  const int sms = current_sm_count() > 0 ? current_sm_count() : 148;
  const int64_t tiles = ((N + kBN - 1) / kBN) * ((M + kBM - 1) / kBM);
  if (tiles >= sms) return 1;
  int64_t s = sms / tiles;
  s = s < (K / kBK) / 8 ? s : (K / kBK) / 8;
  s = s < kMaxSplits ? s : kMaxSplits;
  return s >= 2 ? static_cast<int>(s) : 1;
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

// Whether a cluster of cx x cz CTAs of this kernel (cz = splits of K, or cx = 2 for a pair)
// can be resident at once (one CTA per SM: it needs that many SMs of one GPC); asked once per
// device, kernel and shape.
bool cluster_fits(const void* kern, int which, int cx, int cz) {
  static std::mutex mu;
  static int known[16][4][kMaxSplits + 1];  // 0 unknown, 1 fits, 2 does not
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return false;
  std::lock_guard<std::mutex> lock(mu);
  int& k = known[dev][which][cx * cz];
  if (k == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cx), 1, static_cast<unsigned>(cz));
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = kGSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cx);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = static_cast<unsigned>(cz);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    k = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters >= 1 ? 1 : 2;
    cudaGetLastError();  // a refused query leaves no error behind
  }
  return k == 1;
}

template <int DT, bool PAIR>
cudaError_t launch_cluster(const CUtensorMap& map, const GParams& q, unsigned row_tiles,
                           cudaStream_t stream) {
  auto kern = k_nf4_gemm<DT, PAIR>;
  const unsigned col_tiles = static_cast<unsigned>((q.N + kBN - 1) / kBN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = PAIR ? dim3(row_tiles * col_tiles, 1, 1)  // row_tiles even
                     : dim3(col_tiles, row_tiles, static_cast<unsigned>(q.splits));
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kGSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2u : 1u;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(q.splits);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, map, q);
  count_launches(1);
  return err;
}

// Three launch forms: K split over a cluster of the tile's CTAs (few tiles); two row tiles
// on a CTA pair with two-CTA MMAs (several row tiles, no split); or one CTA per tile.
template <int DT>
cudaError_t launch_gemm(const CUtensorMap& map, const GParams& p, cudaStream_t stream) {
  auto single = k_nf4_gemm<DT, false>;
  auto paired = k_nf4_gemm<DT, true>;
  cudaError_t err =
      cudaFuncSetAttribute(single, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemBytes);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(paired, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemBytes);
  if (err != cudaSuccess) return err;
  const int wd = DT == AQNF4_BF16 ? 0 : 1;
  GParams q = p;
  const int64_t row_tiles = (p.M + kBM - 1) / kBM;
  if (q.splits > 1 && !cluster_fits(reinterpret_cast<const void*>(single), wd, 1, q.splits))
    q.splits = 1;
  // a pair needs two row tiles (an odd count is rounded up: the last partner's rows are
  // past M, its x copies read the fill value and its epilogue stores nothing)
  const int64_t pair_ctas = (row_tiles + (row_tiles & 1)) * ((p.N + kBN - 1) / kBN);
  if (q.splits == 1 && row_tiles >= 2 && pair_ctas <= INT32_MAX &&
      cluster_fits(reinterpret_cast<const void*>(paired), 2 + wd, 2, 1))
    return launch_cluster<DT, true>(map, q, static_cast<unsigned>(row_tiles + (row_tiles & 1)),
                                    stream);
  return launch_cluster<DT, false>(map, q, static_cast<unsigned>(row_tiles), stream);
}

}  // namespace
}  // namespace aqnf4

using namespace aqnf4;

extern "C" int32_t aqnf4_nf4_linear_splits(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < kBK || K % kBK != 0) return 0;
  return choose_splits(M, N, K);
}

extern "C" aqnf4_status aqnf4_nf4_linear(const void* x, int32_t dtype, int64_t M, int64_t K,
                                         const uint8_t* packed, const uint8_t* codes8,
                                         const float* scales, int64_t N, void* y,
                                         int32_t out_f32, int32_t* dev_flag,
                                         cudaStream_t stream) {
  if (!x || !packed || !codes8 || !scales || !y || M < 1 || N < 1 || K < kBK || K % kBK != 0)
    return AQNF4_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - kBM || N > (int64_t(1) << 31) - kBN || K > (int64_t(1) << 31))
    return AQNF4_ERR_INVALID_ARG;
  if ((M + kBM - 1) / kBM > 65535) return AQNF4_ERR_INVALID_ARG;  // row tiles go on grid y
  if (!valid_dtype(dtype)) return AQNF4_ERR_DTYPE;
  // y: the epilogue stores whole 16-byte vectors of a row when N allows it
  if (!is_aligned(x, 16) || !is_aligned(packed, 16) || !is_aligned(scales, 4) ||
      !is_aligned(y, 16) || !is_aligned(dev_flag, 4))
    return AQNF4_ERR_ALIGNMENT;
  const Tables* tb = default_tables();
  const EncodeTiledFn encode = encode_tiled();
  if (!tb || !encode) return AQNF4_ERR_CUDA;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  // a layer product of at most 128 tokens copies only the x rows it has
  const cuuint32_t box[2] = {kBK, static_cast<cuuint32_t>(M <= 128 ? 128 : kBM)};
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
  p.splits = choose_splits(M, N, K);
  p.flag = dev_flag;
  p.a_rows = M <= 128 ? 128 : kBM;
  for (int i = 0; i < 16; ++i) p.level[i] = tb->level[i];
  const cudaError_t err = dtype == AQNF4_BF16 ? launch_gemm<AQNF4_BF16>(map, p, stream)
                                              : launch_gemm<AQNF4_F16>(map, p, stream);
  return err == cudaSuccess ? AQNF4_OK : AQNF4_ERR_CUDA;
}
