// Operand tiles of the 16-bit tcgen05 GEMMs: how a tile of R rows (M or N) by BK
// elements (K) is brought into shared memory by TMA with the 128-byte swizzle, and the
// UMMA descriptor of its i-th 16-element K slice.
//
//  - K-major operand (K contiguous in global memory): boxes of {64 (K), R}, BK/64 of
//    them along K, R*128 bytes apart; rows of 128 bytes, 8-row swizzle atoms of 1 KB.
//  - MN-major operand (M or N contiguous): boxes of {64 (rows), BK (K)}, R/64 of them,
//    BK*128 bytes apart; each k is one 128-byte row of 64 consecutive M/N elements.
#pragma once

#include "sm100.cuh"

namespace smg {

template <int R, int BK>
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                             int mn_major, int r0, int k0) {
  if (!mn_major) {
    // K-major: boxes of {64 (K), R (rows)}, BK/64 of them along K, R*128 bytes apart.
#pragma unroll
    for (int j = 0; j < BK / 64; ++j) tma_load_2d(dst + j * R * 128, map, bar, k0 + 64 * j, r0);
  } else {
    // MN-major: boxes of {64 (rows), BK (K)}, R/64 of them along the rows, BK*128 bytes apart.
#pragma unroll
    for (int j = 0; j < R / 64; ++j) tma_load_2d(dst + j * BK * 128, map, bar, r0 + 64 * j, k0);
  }
}

// The same tile loads for a CTA of a pair: the byte count completes on `bar_cluster`,
// an mbarrier of the rank-0 CTA (shared::cluster address).
template <int R, int BK>
__device__ __forceinline__ void load_operand_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                  int mn_major, int r0, int k0) {
  if (!mn_major) {
#pragma unroll
    for (int j = 0; j < BK / 64; ++j) tma_load_2d_pair(dst + j * R * 128, map, bar_cluster, k0 + 64 * j, r0);
  } else {
#pragma unroll
    for (int j = 0; j < R / 64; ++j) tma_load_2d_pair(dst + j * BK * 128, map, bar_cluster, r0 + 64 * j, k0);
  }
}

// The same tile from a map whose K-major box is {64 (K), 64 (rows)}: R/64 boxes per
// 64-element K slice, stacked 64 * 128 bytes apart (the layout of one R-row box, since
// each box starts on a 1 KB swizzle atom). The MN-major box is 64 rows wide already.
template <int R, int BK>
__device__ __forceinline__ void load_operand_pair_r64(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                      int mn_major, int r0, int k0) {
  static_assert(R % 64 == 0, "whole 64-row boxes");
  if (!mn_major) {
#pragma unroll
    for (int j = 0; j < BK / 64; ++j)
#pragma unroll
      for (int h = 0; h < R / 64; ++h)
        tma_load_2d_pair(dst + j * R * 128 + h * 64 * 128, map, bar_cluster, k0 + 64 * j, r0 + 64 * h);
  } else {
#pragma unroll
    for (int j = 0; j < R / 64; ++j) tma_load_2d_pair(dst + j * BK * 128, map, bar_cluster, r0 + 64 * j, k0);
  }
}

// Descriptor of the i-th 16-element K slice of an operand tile laid out by load_operand.
template <int R, int BK>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int mn_major, int i) {
  if (!mn_major) return sdesc_sw128(base + (i >> 2) * (R * 128) + (i & 3) * 32, 16, 1024);
  return sdesc_sw128(base + i * 2048, BK * 128, 1024);
}

template <int MMA_N>
struct TmemCols {
  static constexpr int v = (2 * MMA_N <= 32) ? 32 : (2 * MMA_N <= 64) ? 64 : (2 * MMA_N <= 128) ? 128
                          : (2 * MMA_N <= 256) ? 256 : 512;
};


}  // namespace smg
