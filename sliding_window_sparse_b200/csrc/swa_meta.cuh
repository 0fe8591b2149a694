// swa_meta.cuh -- device-built tile metadata and ring-buffer bookkeeping.
//
//  * block_meta_kernel: per (sequence, query tile) the class of every key tile
//    (M003 note section 04: skip / full / partial) and the summary
//    {live, full, first live, last live}.
//  * ring_positions_kernel: logical position held by each ring slot
//    (M003 note section 06; blog section 3.2).
//  * ring_write_kernel: append a chunk's last min(T, W) rows at slot
//    position mod W (Chapter 10 section 10.2: the persistent cache keeps the
//    last W positions).
#pragma once
#include <cstdint>

#include "sm100.cuh"
#include "swa_tile.cuh"

namespace swa {

struct MetaParams {
  int key_mode;  // 0 linear, 1 ring + chunk
  int B;
  int64_t n_q, n_k, W;
  int tile_q, tile_k;
  int nqt, nkt;
  const int64_t *q_pos0;  // [B] or nullptr (mode 0 only)
  int8_t *classes;        // [B, nqt, nkt] or nullptr
  int32_t *ranges;        // [B, nqt, 4] or nullptr
};

// One CTA per (b, query tile); threads stride over the key tiles.
__global__ void __launch_bounds__(256) block_meta_kernel(const MetaParams p) {
  const int qt = blockIdx.x;
  const int b = blockIdx.y;
  __shared__ int s_live, s_full, s_first, s_last;
  if (threadIdx.x == 0) {
    s_live = 0;
    s_full = 0;
    s_first = INT32_MAX;
    s_last = -1;
  }
  __syncthreads();
  int64_t p0 = 0;
  if (p.q_pos0) p0 = p.q_pos0[b];
  bool bad = p.key_mode == 1 && p0 < 0;
  const int64_t r_begin = static_cast<int64_t>(qt) * p.tile_q;
  const int64_t r_end = (r_begin + p.tile_q < p.n_q ? r_begin + p.tile_q : p.n_q) - 1;
  // mode 0: absolute positions; mode 1: positions relative to the chunk start
  const int64_t q_lo = (p.key_mode == 0 ? p0 : 0) + r_begin;
  const int64_t q_hi = (p.key_mode == 0 ? p0 : 0) + r_end;
  int live = 0, full = 0, first = INT32_MAX, last = -1;
  for (int kt = threadIdx.x; kt < p.nkt; kt += blockDim.x) {
    int cls = 0;
    if (!bad) {
      const KeyTile t = p.key_mode == 0
                            ? linear_tile(kt, p.tile_k, p.n_k)
                            : ring_chunk_tile(kt, p.tile_k, p.W, p.n_q, p0, p0);
      cls = tile_class(t, q_lo, q_hi, p.W);
    }
    if (p.classes) p.classes[(static_cast<int64_t>(b) * p.nqt + qt) * p.nkt + kt] =
        static_cast<int8_t>(cls);
    if (cls) {
      ++live;
      first = kt < first ? kt : first;
      last = kt > last ? kt : last;
    }
    if (cls == 1) ++full;
  }
  if (bad && threadIdx.x == 0) atomicOr(&g_swa_status, SWA_DEV_BADARG);
  atomicAdd(&s_live, live);
  atomicAdd(&s_full, full);
  atomicMin(&s_first, first);
  atomicMax(&s_last, last);
  __syncthreads();
  if (threadIdx.x == 0 && p.ranges) {
    int32_t *r = p.ranges + (static_cast<int64_t>(b) * p.nqt + qt) * 4;
    r[0] = s_live;
    r[1] = s_full;
    r[2] = s_live ? s_first : -1;
    r[3] = s_live ? s_last : -1;
  }
}

// slot_pos[b, s] = largest p < L_b with p mod W == s, else -1.
__global__ void ring_positions_kernel(int B, const int64_t *__restrict__ n_written, int64_t W,
                                      int64_t *__restrict__ slot_pos) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(B) * W) return;
  const int64_t b = idx / W, s = idx % W;
  const int64_t L = n_written[b];
  if (L < 0) {
    atomicOr(&g_swa_status, SWA_DEV_BADARG);
    slot_pos[idx] = -1;
    return;
  }
  slot_pos[idx] = s <= L - 1 ? (L - 1) - ((L - 1 - s) % W) : -1;
}

// Copy chunk rows t >= T_b - W (positions start + t among the last W) to slot
// (start + t) mod W, where T_b = lens[b] (or T when lens is null) is the
// number of valid rows of sequence b.  One thread moves 16 bytes;
// d * 2 / 16 threads per row.
__global__ void ring_write_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                  uint4 *__restrict__ k_ring, uint4 *__restrict__ v_ring,
                                  const int64_t *__restrict__ q_start,
                                  const int64_t *__restrict__ lens, int B, int Hkv, int64_t T,
                                  int vec_per_row, int64_t W) {
  const int64_t rows = T < W ? T : W;  // row slots per (b, kvh)
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(B) * Hkv * rows * vec_per_row;
  if (idx >= total) return;
  const int64_t c = idx % vec_per_row;
  const int64_t r = (idx / vec_per_row) % rows;
  const int64_t bh = idx / (static_cast<int64_t>(vec_per_row) * rows);
  const int64_t b = bh / Hkv;
  const int64_t start = q_start[b];
  const int64_t tb = lens ? lens[b] : T;
  if (start < 0 || tb < 0 || tb > T) {
    if (c == 0 && r == 0) atomicOr(&g_swa_status, SWA_DEV_BADARG);
    return;
  }
  const int64_t rows_b = tb < W ? tb : W;
  if (r >= rows_b) return;
  const int64_t t = tb - rows_b + r;  // chunk row
  const int64_t slot = (start + t) % W;
  const uint4 kv = k_new[(bh * T + t) * vec_per_row + c];
  const uint4 vv = v_new[(bh * T + t) * vec_per_row + c];
  k_ring[(bh * W + slot) * vec_per_row + c] = kv;
  v_ring[(bh * W + slot) * vec_per_row + c] = vv;
}

}  // namespace swa
