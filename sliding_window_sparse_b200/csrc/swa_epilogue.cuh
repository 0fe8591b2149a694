// swa_epilogue.cuh -- writing a TMEM accumulator tile to global memory.
//
// A 32x32b TMEM load gives each thread one row (its TMEM lane), so stores
// straight from registers touch 32 rows per warp instruction.  The helpers
// here regroup 16-byte pieces inside each 8-lane group with warp shuffles,
// after which one store instruction writes four whole 128-byte row segments.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace swa {

// Transpose, within each group of 8 lanes, an 8 x 8 matrix of 16-byte pieces:
// on entry lane j of a group holds pieces 0..7 of its own row j (piece i in
// e[4i..4i+3]); on exit it holds piece j of rows 0..7 of the group (row i's in
// e[4i..4i+3]).  Stage s swaps bit s of the row index with bit s of the piece
// index: the lane whose bit s is 0 keeps the pieces whose bit s is 0 and trades
// the others with lane ^ (1 << s).  All 32 lanes must take part.
__device__ __forceinline__ void transpose8_pieces(uint32_t (&e)[32], int lane) {
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int m = 1 << s;
    const bool hi = (lane >> s) & 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & m) continue;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t send = hi ? e[4 * i + w] : e[4 * (i | m) + w];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
        if (hi)
          e[4 * i + w] = recv;
        else
          e[4 * (i | m) + w] = recv;
      }
    }
  }
}

// Store D fp32 TMEM columns of this warp's 32 rows, times `mul`, as bf16 rows
// of a row-major [rows, D] array.  `taddr` is this warp's TMEM address of
// column 0 (lane quadrant included); `grp0` points at column 0 of the first
// row of this lane's 8-lane group, `row_stride` is the distance between rows
// in elements; only the group's first `n_valid` rows are written.  Called by
// all 32 lanes.
template <int D>
__device__ __forceinline__ void store_tile_rows(__nv_bfloat16 *grp0, int64_t row_stride,
                                                int n_valid, uint32_t taddr, float mul,
                                                int lane) {
  __nv_bfloat16 *g = grp0 + 8 * (lane & 7);
#pragma unroll 1
  for (int h2 = 0; h2 < D / 64; ++h2) {
    uint32_t e[32];
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      uint32_t o32[32];
      tmem_ld32(taddr + h2 * 64 + c2 * 32, o32);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        e[c2 * 16 + i] =
            pack_bf16(__uint_as_float(o32[2 * i]) * mul, __uint_as_float(o32[2 * i + 1]) * mul);
    }
    transpose8_pieces(e, lane);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < n_valid)
        *reinterpret_cast<uint4 *>(g + i * row_stride + h2 * 64) =
            make_uint4(e[4 * i], e[4 * i + 1], e[4 * i + 2], e[4 * i + 3]);
  }
}

}  // namespace swa
