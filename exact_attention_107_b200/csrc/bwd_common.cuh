// bwd_common.cuh -- pieces shared by the backward kernels (fa_bwd_sm100.cu for head dims
// up to 128, fa_bwd_d256_sm100.cu for 256): thread layout, exponent split, staging of
// 64-column boxes in the TMA 128-byte-swizzled layout, and UMMA operand descriptors.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "sm100_ptx.cuh"

namespace fa {
namespace {

// 640 threads: warp 0 loads, warp 1 issues MMAs, warps 4-19 are four warpgroups that
// share the element-wise work (no row reduction is needed in the backward, so the
// columns of a tile can be split across warpgroups to hide more latency).
constexpr int kThreads = 640;
constexpr float kLog2e = 1.44269504088896340736f;
// Of every 8 pairs of exponentials, this many go to the FMA-pipe polynomial
// (exp2_poly2) and the rest to the MUFU unit (1/8 to 3/8 measure within 1% of each other).
constexpr int kPolyPer8 = 2;
__device__ __forceinline__ bool poly_pair(int c2) { return (c2 & 7) >= 8 - kPolyPer8; }

// A tile of `rows` rows x D 16-bit values in shared memory, stored as D/64 boxes of rows x 128 bytes
// in the TMA 128-byte-swizzled layout.
template <int D, int ROWS>
struct Tile {
  static constexpr int kBox = ROWS * 128;
  static constexpr int kNBox = D / 64;
  static constexpr int kBytes = kBox * kNBox;
};

// Copies 64 columns (box `box`) of this thread's fp32 accumulator row in tensor memory,
// times `mul`, as bf16 (fp16 when F16) into row r of that box of a 128-row staging tile in the TMA
// 128-byte-swizzled layout.
template <int D, bool F16>
__device__ __forceinline__ void stage_box_16(uint32_t tacc, int box, float mul, uint8_t* stage, int r) {
#pragma unroll
  for (int cc = 2 * box; cc < 2 * box + 2; ++cc) {
    uint32_t o[32];
    tmem_ld32(tacc + cc * 32, o);
    tmem_ld_wait();
    reg_fence(o);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int chunk = (cc & 1) * 4 + q4;
      uint4 v;
      v.x = pack16<F16>(__uint_as_float(o[8 * q4 + 0]) * mul, __uint_as_float(o[8 * q4 + 1]) * mul);
      v.y = pack16<F16>(__uint_as_float(o[8 * q4 + 2]) * mul, __uint_as_float(o[8 * q4 + 3]) * mul);
      v.z = pack16<F16>(__uint_as_float(o[8 * q4 + 4]) * mul, __uint_as_float(o[8 * q4 + 5]) * mul);
      v.w = pack16<F16>(__uint_as_float(o[8 * q4 + 6]) * mul, __uint_as_float(o[8 * q4 + 7]) * mul);
      *reinterpret_cast<uint4*>(stage + box * Tile<D, 128>::kBox + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
    }
  }
}

// One warp stores its 32 staged rows of staging box `box` with the TMA (tensor map box:
// 64 x 32 x 1) at columns [64 xbox, 64 xbox + 64); rows at or past n_rows are skipped (or
// clipped by the hardware).
__device__ __forceinline__ void store_warp_box_x(const CUtensorMap* tm, uint32_t stage_s, int box, int xbox, int wrow,
                                                 int row0, int bh, int lane, int n_rows) {
  fence_async_smem();
  __syncwarp();
  if (lane == 0 && row0 + wrow < n_rows) {
    tma_store_3d(tm, stage_s + box * Tile<64, 128>::kBox + wrow * 128, xbox * 64, row0 + wrow, bh);
    bulk_commit();
    bulk_wait_read0();
  }
  __syncwarp();
}
template <int D>
__device__ __forceinline__ void store_warp_box(const CUtensorMap* tm, uint32_t stage_s, int box, int wrow, int row0,
                                               int bh, int lane, int n_rows) {
  store_warp_box_x(tm, stage_s, box, box, wrow, row0, bh, lane, n_rows);
}

// K-major operand slice for K-step kk (16 values = 32 bytes) of a swizzled tile with box size `box`.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk, int box) {
  return sdesc_sw128(tile + (kk >> 2) * box + (kk & 3) * 32, 16, 1024);
}
// MN-major operand slice for K-step kk (16 rows of 128 bytes) of a swizzled tile whose
// 64-column boxes are `box` bytes apart.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int kk, int box) {
  return sdesc_sw128(tile + kk * 2048, box, 1024);
}

// Tensor-memory column of the packed 16-bit pairs for K-step kk (16 queries) of the
// P^T (base 0) or dS^T (base 128) operand (and likewise for the dS operand of dQ): queries [32g, 32g+32) are packed into
// columns base + [32g, 32g+16).
__device__ __forceinline__ uint32_t packed_col(uint32_t base, int kk) {
  return base + 32 * (kk >> 1) + 8 * (kk & 1);
}

}  // namespace
}  // namespace fa
