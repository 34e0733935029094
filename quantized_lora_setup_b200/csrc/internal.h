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
//   level[c]    : NF4 level of code c (16 entries).
//   bucket_mid  : for the bucket b = floor(15.5 v + 16) in [0, 32): the one midpoint that
//                 falls in bucket b, or +inf when none does.
//   bucket_code : number of midpoints below bucket b.
// With these, #{ j : v > mid_j } = bucket_code[b] + (v > bucket_mid[b]) for every finite v
// with |v| < 1 + 1/31 (every normalised value lies well inside that).
struct Tables {
  float level[16];
  float mid[15];
  float bucket_mid[32];
  uint32_t bucket_code[32];
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
