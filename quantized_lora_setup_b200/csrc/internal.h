// internal.h -- declarations shared by the translation units of libaqnf4 (not installed).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "aqnf4.h"

namespace aqnf4 {

constexpr int kBlock = 64;                 // NF4 block: elements per absmax constant
constexpr int kDqBlock = 256;              // double-quantization block: constants per scale
constexpr int kTile = kBlock * kDqBlock;   // 16384 elements: one DQ block of weights
constexpr int kTileBytes = kTile * 2;      // 16-bit weights of one tile
constexpr int kPackedTileBytes = kTile / 2;

// Lookup tables the kernels use, derived from the default codebook (codebook.cpp).
//   level[c], mid[j] : the codebook (16 levels, 15 midpoints).
//   curve_a, curve_b : the slot of a normalised value v is k(v) = round(a v + b v^3 + 8),
//                      an odd cubic fitted so that every midpoint sits in a slot of its own:
//                      for mid_{j-1} < v <= mid_j, k(v) is j or j + 1 (checked when the
//                      tables are built, with a margin far above binary32 rounding).
//   slot_mid[k]      : mid_{k-1} for k = 1..15; -inf at k = 0; +inf at k >= 16.
//   slot_level[k]    : level[k-1] for k = 1..16 (lane k of a shuffle table); the unused
//                      lanes repeat the end levels.
// With these, #{ j : v > mid_j } = k(v) - 1 + (v > slot_mid[k(v)]) for every |v| <= 1 + 2^-20,
// which covers every normalised value.  The code then indexes slot_level at k + 1.
struct Tables {
  float level[16];
  float mid[15];
  float curve_a, curve_b;
  float slot_mid[32];
  float slot_level[32];
};

// Builds (once) and returns the tables of the default codebook.  Returns nullptr if the
// codebook violates a table invariant (never for the default p_max).
const Tables* default_tables();

// Host-side launch accounting (aqnf4_launch_count).
void count_launches(uint64_t n);

// Number of SMs of the current device (queried per call; cheap).
int current_sm_count();

inline bool is_aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline bool valid_dtype(int32_t dt) { return dt == AQNF4_F16 || dt == AQNF4_BF16; }

}  // namespace aqnf4
