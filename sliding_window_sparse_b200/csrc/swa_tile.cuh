// swa_tile.cuh -- key tiles, their logical positions and their classes.
//
// Visibility rule (M003 note section 03; Chapter 10 section 10.1): a query at
// logical position i may read key position j iff i - W + 1 <= j <= i.
//
// A key tile is up to BK consecutive columns of one key source (the linear
// key tensor, the ring buffer, or the new chunk).  Its in-range columns are
// split into at most two segments; inside a segment, column c holds logical
// position base + c (positions are relative to a per-call origin).  Columns of
// a ring tile that hold nothing (ring not yet full) belong to no segment.
//
// Ring layout (blog "Dense attention vs sparse SWA" section 3.2 write order,
// so slot = position mod W once full): with L positions already written,
// slot s holds the largest p < L with p mod W == s.  For L >= W and
// w = L mod W, slots s < w hold p = L - w + s and slots s >= w hold
// p = L - W - w + s; for L < W, slots s < L hold p = s and the rest are empty.
#pragma once
#include <cstdint>

namespace swa {

struct Seg {
  int lo, hi;    // columns lo..hi (inclusive); empty if lo > hi
  int64_t base;  // logical position of column c is base + c
};

struct KeyTile {
  int src;     // 0 = main key tensor (linear keys, or the new chunk), 1 = ring
  int y0;      // first row of the tile in its source tensor
  int ncols;   // in-range columns (<= BK)
  Seg seg[2];  // segments with positions (second may be empty)
};

// Tile class from in-range query positions q_lo..q_hi (consecutive).
// 0 = no allowed pair (skip), 1 = every in-range pair allowed (no mask),
// 2 = some allowed (compute and mask).  Exact, not conservative.
__host__ __device__ inline int tile_class(const KeyTile &t, int64_t q_lo, int64_t q_hi,
                                          int64_t W) {
  bool any = false;
  int64_t all_cols = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const Seg &s = t.seg[i];
    if (s.lo > s.hi) continue;
    const int64_t p_lo = s.base + s.lo, p_hi = s.base + s.hi;
    // some query q in [q_lo, q_hi] and key j in [p_lo, p_hi] with q-W+1 <= j <= q
    if (p_lo <= q_hi && p_hi + W - 1 >= q_lo) any = true;
    // every pair allowed: j <= q for the smallest q and j >= q-W+1 for the largest
    if (p_hi <= q_lo && p_lo >= q_hi - W + 1) all_cols += s.hi - s.lo + 1;
  }
  if (!any) return 0;
  return all_cols == t.ncols ? 1 : 2;
}

// Linear key axis: tile kt of n_k keys at positions 0..n_k-1.
__host__ __device__ inline KeyTile linear_tile(int kt, int BK, int64_t n_k) {
  KeyTile t;
  t.src = 0;
  t.y0 = kt * BK;
  const int64_t rem = n_k - static_cast<int64_t>(kt) * BK;
  t.ncols = static_cast<int>(rem < BK ? rem : BK);
  t.seg[0] = Seg{0, t.ncols - 1, static_cast<int64_t>(kt) * BK};
  t.seg[1] = Seg{1, 0, 0};
  return t;
}

// Ring tile kt (slots kt*BK ..) of a W-slot ring after L writes; positions
// relative to `origin` (the caller's chosen zero).
__host__ __device__ inline KeyTile ring_tile(int kt, int BK, int64_t W, int64_t L,
                                             int64_t origin) {
  KeyTile t;
  t.src = 1;
  const int64_t s0 = static_cast<int64_t>(kt) * BK;
  t.y0 = static_cast<int>(s0);
  const int64_t rem = W - s0;
  t.ncols = static_cast<int>(rem < BK ? rem : BK);
  const int64_t s1 = s0 + t.ncols - 1;
  t.seg[0] = Seg{1, 0, 0};
  t.seg[1] = Seg{1, 0, 0};
  if (L <= 0) return t;
  if (L < W) {
    // slots 0..L-1 hold positions 0..L-1
    const int64_t hi = (L - 1 < s1 ? L - 1 : s1) - s0;
    if (hi >= 0) t.seg[0] = Seg{0, static_cast<int>(hi), s0 - origin};
    return t;
  }
  const int64_t w = L % W;
  // slots s < w: position L - w + s
  if (s0 <= w - 1) {
    const int64_t hi = (w - 1 < s1 ? w - 1 : s1) - s0;
    t.seg[0] = Seg{0, static_cast<int>(hi), L - w + s0 - origin};
  }
  // slots s >= w: position L - W - w + s
  if (s1 >= w) {
    const int64_t lo = (w > s0 ? w : s0) - s0;
    t.seg[1] = Seg{static_cast<int>(lo), t.ncols - 1, L - W - w + s0 - origin};
  }
  return t;
}

// Chunk tile kt of the Tq new keys at positions start + t (relative to origin).
__host__ __device__ inline KeyTile chunk_tile(int kt, int BK, int64_t Tq, int64_t start,
                                              int64_t origin) {
  KeyTile t = linear_tile(kt, BK, Tq);
  t.seg[0].base = static_cast<int64_t>(kt) * BK + start - origin;
  return t;
}

// Key tile number kt of a ring+chunk key axis (ring tiles first, physical order).
__host__ __device__ inline KeyTile ring_chunk_tile(int kt, int BK, int64_t W, int64_t Tq,
                                                   int64_t q_start, int64_t origin) {
  const int nrt = static_cast<int>((W + BK - 1) / BK);
  if (kt < nrt) return ring_tile(kt, BK, W, q_start, origin);
  return chunk_tile(kt - nrt, BK, Tq, q_start, origin);
}

}  // namespace swa
