// swa_split.cuh -- splitting the key ranges of chunk-ring units across CTAs.
//
// The chunk-ring forward (fwd2_kernel MODE 1) runs one CTA per SM over
// two-query-tile units of about equal length (every query tile of a chunk
// sees a whole window).  When the number of live units L (units whose query
// tiles hold valid rows of their chunk) leaves the last round of units part
// empty, that round is the tail of the whole call.  With a caller workspace
// the call instead:
//   1. chunk_split_schedule_kernel lists, per CTA and round, the units it
//      runs: the first floor(L / P) * P live units whole, one per CTA and
//      round; each of the remaining L mod P units cut into R = P / (L mod P)
//      parts (contiguous pieces of its live key tiles), one part per CTA;
//   2. the attention kernel runs its list; a part writes its unnormalised O
//      rows with their running max and sum to the workspace (a whole unit
//      writes its output as usual);
//   3. chunk_split_merge_kernel merges each split unit's parts, as a softmax
//      over the union of their keys (the same merge as the decode path's),
//      into the bf16 output rows and the log-sum-exp.
// Chapter 10 section 10.2: each query of a chunk attends to its own window
// over ring and chunk keys; a split only partitions that key set.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "swa_fwd2.cuh"

namespace swa {

constexpr int kSplitThreads = 1024;
constexpr int kMaxSplitParts = 16;

// The workspace: a header {L, full rounds, split units, parts}, the item list
// int4 {unit, part, parts, slot} indexed [round * P + cta] (unit < 0 ends a
// CTA's list), then per part slot the partial rows of both query tiles:
// running max and sum [slot][2][kQT][2] and O [slot][2][kQT][D], fp32.
struct SplitLayout {
  static constexpr int kHeaderInts = 4;
  __host__ __device__ static int64_t items_len(int64_t n_units, int P) {
    return (n_units / P + 2) * static_cast<int64_t>(P);
  }
  __host__ __device__ static int64_t ml_offset(int64_t n_units, int P) {  // floats
    return ((kHeaderInts + 4 * items_len(n_units, P)) + 63) / 64 * 64;
  }
  __host__ __device__ static int64_t o_offset(int64_t n_units, int P) {  // floats
    return ml_offset(n_units, P) + static_cast<int64_t>(P) * 2 * kQT * 2;
  }
  __host__ __device__ static int64_t bytes(int64_t n_units, int P, int D) {
    return (o_offset(n_units, P) + static_cast<int64_t>(P) * 2 * kQT * D) * 4;
  }
};

// Live units in the attention kernel's unit order; one CTA.
template <int D>
__global__ void __launch_bounds__(kSplitThreads)
    chunk_split_schedule_kernel(const Fwd2Params p, int P, int *ws) {
  __shared__ int s_scan[kSplitThreads];
  __shared__ int s_total;
  int *hdr = ws;
  int4 *items = reinterpret_cast<int4 *>(ws + SplitLayout::kHeaderInts);
  const int tid = threadIdx.x;
  // the attention kernel's own test (a unit of a sequence with an invalid
  // start or length is skipped and flagged there; here it is flagged too)
  auto live = [&](int u) -> bool {
    Unit U = decode_unit(u, p);
    const int64_t qs = p.q_start[U.b];
    int len = p.n_q;
    bool bad = qs < 0;
    if (p.chunk_len) {
      const int64_t l = p.chunk_len[U.b];
      bad = bad || l < 0 || l > p.n_q;
      len = static_cast<int>(l);
    }
    if (bad) {
      atomicOr(&g_swa_status, SWA_DEV_BADARG);
      return false;
    }
    return U.t[0] * kQT < len;
  };
  // pass 1: L
  int cnt = 0;
  for (int u = tid; u < p.n_units; u += kSplitThreads) cnt += live(u) ? 1 : 0;
  s_scan[tid] = cnt;
  __syncthreads();
  for (int half = kSplitThreads / 2; half > 0; half >>= 1) {  // tree sum
    if (tid < half) s_scan[tid] += s_scan[tid + half];
    __syncthreads();
  }
  if (tid == 0) s_total = s_scan[0];
  __syncthreads();
  const int L = s_total;
  const int F = L / P, L_full = F * P, L_rem = L - L_full;
  int R = L_rem > 0 ? P / L_rem : 1;
  R = R < 1 ? 1 : (R > kMaxSplitParts ? kMaxSplitParts : R);
  const int64_t n_items = SplitLayout::items_len(p.n_units, P);
  for (int64_t i = tid; i < n_items; i += kSplitThreads) items[i] = make_int4(-1, 0, 1, -1);
  if (tid == 0) {
    hdr[0] = L;
    hdr[1] = F;
    hdr[2] = R > 1 ? L_rem : 0;
    hdr[3] = R;
  }
  __syncthreads();
  // pass 2: the rank of each live unit, in chunks of kSplitThreads units
  int base = 0;
  for (int u0 = 0; u0 < p.n_units; u0 += kSplitThreads) {
    const int u = u0 + tid;
    const int f = (u < p.n_units && live(u)) ? 1 : 0;
    s_scan[tid] = f;
    __syncthreads();
    for (int off = 1; off < kSplitThreads; off <<= 1) {  // inclusive scan
      const int v = tid >= off ? s_scan[tid - off] : 0;
      __syncthreads();
      s_scan[tid] += v;
      __syncthreads();
    }
    if (f) {
      const int k = base + s_scan[tid] - 1;
      if (k < L_full) {
        items[static_cast<int64_t>(k / P) * P + k % P] = make_int4(u, 0, 1, -1);
      } else if (R == 1) {
        items[static_cast<int64_t>(F) * P + (k - L_full)] = make_int4(u, 0, 1, -1);
      } else {
        for (int r = 0; r < R; ++r) {
          const int j = (k - L_full) * R + r;
          items[static_cast<int64_t>(F) * P + j] = make_int4(u, r, R, j);
        }
      }
    }
    const int chunk_total = s_scan[kSplitThreads - 1];
    __syncthreads();
    base += chunk_total;
  }
}

constexpr int kMergeRowsPerCta = 8;  // one warp per row

// Grid (split units, 2 query tiles, kQT / kMergeRowsPerCta): one warp per row,
// each lane D / 32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(32 * kMergeRowsPerCta)
    chunk_split_merge_kernel(const Fwd2Params p, int P, const int *ws) {
  constexpr int CPL = D / 32;  // columns per lane
  const int s = blockIdx.x, x = blockIdx.y;
  const int n_split = ws[2], R = ws[3], F = ws[1];
  if (s >= n_split) return;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.z * kMergeRowsPerCta + (threadIdx.x >> 5);
  const int4 *items = reinterpret_cast<const int4 *>(ws + SplitLayout::kHeaderInts);
  const int u = items[static_cast<int64_t>(F) * P + s * R].x;
  Unit U = decode_unit(u, p);
  int len = p.n_q;
  if (p.chunk_len) len = static_cast<int>(p.chunk_len[U.b]);
  if (U.has_b && U.t[1] * kQT >= len) U.has_b = false;
  if (x == 1 && !U.has_b) return;
  const int row = U.t[x] * kQT + r;
  if (row >= len) return;
  const float *ml = reinterpret_cast<const float *>(ws) + SplitLayout::ml_offset(p.n_units, P);
  const float *po = reinterpret_cast<const float *>(ws) + SplitLayout::o_offset(p.n_units, P);
  // lane j < R holds part j's running max and sum of this row
  float mj = -INFINITY, lj = 0.f;
  if (lane < R) {
    const int64_t mi = ((static_cast<int64_t>(s * R + lane) * 2 + x) * kQT + r) * 2;
    lj = ml[mi + 1];
    if (lj > 0.f) mj = ml[mi];  // a part that saw no key of this row has sum 0
  }
  float M = mj;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float wj = lj > 0.f ? exp2f(mj - M) : 0.f;
  float Lsum = lj * wj;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
  float acc[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
  for (int j = 0; j < R; ++j) {
    const float w = __shfl_sync(0xffffffffu, wj, j);
    if (w == 0.f) continue;
    const float *src = po + ((static_cast<int64_t>(s * R + j) * 2 + x) * kQT + r) * D + lane * CPL;
#pragma unroll
    for (int i = 0; i < CPL; i += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + i);
      acc[i] += v.x * w;
      acc[i + 1] += v.y * w;
      acc[i + 2] += v.z * w;
      acc[i + 3] += v.w * w;
    }
  }
  const float inv = 1.f / Lsum;
  __nv_bfloat16 *dst = p.out + ((static_cast<int64_t>(U.b) * p.H + U.h[x]) * p.n_q + row) * D +
                       lane * CPL;
#pragma unroll
  for (int i = 0; i < CPL; i += 2)
    *reinterpret_cast<__nv_bfloat162 *>(dst + i) =
        __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
  if (p.lse && lane == 0)
    p.lse[(static_cast<int64_t>(U.b) * p.H + U.h[x]) * p.n_q + row] =
        (M + __log2f(Lsum)) * 0.6931471805599453f;
}

}  // namespace swa
