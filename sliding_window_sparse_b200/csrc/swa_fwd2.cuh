// swa_fwd2.cuh -- persistent, two-query-tile sliding-window attention forward
// for sm_100a (tcgen05 MMAs, tensor-memory accumulators, TMA staging).
//
// Work unit: two 128-row query tiles A and B that read the same key/value
// tiles.  With G = H / Hkv even they are two query heads of one key/value
// group at the same query rows (identical tile lists); otherwise they are
// query tiles 2p and 2p+1 of one head (the key stream is the union of both
// windows and each tile uses its own part).  CTAs are persistent and walk the
// heavy-first unit order in a serpentine (see unit_of).
//
// Roles (384 threads, three warpgroups):
//   warp 0      TMA producer: Q_A, Q_B once per unit, then K and V tiles into
//               separate shared-memory rings (3 K and 2 V stages at d = 128;
//               128-byte swizzle, one box per 64 head-dim columns).  Only live
//               key tiles are loaded (M003 note section 04).
//   warp 1      one thread issues every tcgen05.mma:
//                 S_X = Q_X K^T        (A, B from shared memory)
//                 O_X += P_X V         (P from tensor memory, V from shared memory)
//               in the order PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the
//               softmax of one tile overlaps the MMAs of the other.  On the
//               linear and packed layouts the softmax hands P over in two
//               halves of 64 keys, and the PV of the first half runs while the
//               exponentials of the second are computed.
//   warps 2-3   idle (they complete warpgroup 0).
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: one row per
//               thread, one tensor-memory lane quadrant per warp.  Mask only
//               partial or ragged tiles, base-2 exponentials with
//               scale * log2(e) folded in, running max and sum in fp32, P
//               packed to bf16 into the tile's S columns, O rescaled in tensor
//               memory only when the running max grows by more than 2^8.
//               After the unit's last tile: O / l to bf16 rows, and the
//               log-sum-exp.
//
// Registers: 384 threads get 168 registers each at launch (three warps per
// SM sub-partition).  Warpgroup 0 then gives registers back (setmaxnreg.dec to
// kRegsControl) and the two softmax warpgroups take them (setmaxnreg.inc to
// kRegsSoftmax), so the softmax holds a whole 128-column score row without
// spilling.  The split must add up to the launch total exactly, or the
// increase would wait for registers that never come: the host checks the
// kernel's launch register count before the first launch.
//
// Tensor memory (512 columns): S_A/P_A [0,128), S_B/P_B [128,256),
// O_A [256, 256+D), O_B [256+D, 256+2D).  P_X overwrites the first 64 columns
// of S_X; the next S_X is issued after PV_X, and tcgen05 MMAs issued by one
// thread execute in order.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "swa_epilogue.cuh"
#include "swa_tile.cuh"

namespace swa {

constexpr int kQT = 128;  // query rows per tile (MMA M, tensor-memory lanes)
constexpr int kKT = 128;  // keys per tile
constexpr int kFwd2Threads = 384;
constexpr int kFwd2LaunchRegs = 168;  // registers per thread at launch (checked by the host)
constexpr int kRegsControl = 88;      // warpgroup 0: producer, MMA issuer, two idle warps
constexpr int kRegsSoftmax = 208;     // warpgroups 1 and 2: softmax + epilogue
static_assert(4 * kRegsControl + 8 * kRegsSoftmax == (kFwd2Threads / 32) * kFwd2LaunchRegs,
              "the register split must hand over exactly the launch allocation");
static_assert(kRegsControl % 8 == 0 && kRegsSoftmax % 8 == 0 && kRegsSoftmax <= 256,
              "setmaxnreg counts are multiples of 8, at most 256");
constexpr float kLazyRescaleLog2 = 8.0f;

// MODE 0: linear [B, heads, N, D] layout.  MODE 1: chunk [B, heads, Tq, D] over
// a ring [B, Hkv, W, D].  MODE 2: packed token-major [total, heads, D], sequence b
// on tokens cu_seqlens[b] .. cu_seqlens[b + 1] - 1 (positions from 0 in each).
struct Fwd2Params {
  __nv_bfloat16 *out = nullptr;        // [B, H, n_q, D]; MODE 2: [total, H, D]
  float *lse = nullptr;                // [B, H, n_q]; MODE 2: [H, total]; or nullptr
  const int64_t *q_start = nullptr;    // MODE 1: [B]
  const int64_t *chunk_len = nullptr;  // MODE 1: [B] valid chunk rows, or nullptr = n_q
  const int64_t *cu_seqlens = nullptr; // MODE 2: [B + 1]
  int64_t total = 0;                   // MODE 2: packed tokens
  int B = 0, H = 0, Hkv = 0, G = 0;
  int n_q = 0;             // query rows per (b, h); MODE 2: longest sequence
  int n_k = 0;             // rows of the main key source (N, or Tq for a chunk)
  int64_t W = 0;           // window (MODE 0 / 2: clamped to n_q + kQT)
  int n_sink = 0;          // keys 0 .. n_sink-1 stay visible to later queries (MODE 1: from
                           // their own rows, the tensor maps tm_ks / tm_vs)
  float scale_log2 = 0.f;  // scale * log2(e)
  int nqt = 0;             // query tiles per (b, h)
  int n_ring_tiles = 0;    // MODE 1: ceil(W / kKT)
  int pair_heads = 0;      // 1: A/B are heads 2p, 2p+1 of a group; 0: q tiles 2p, 2p+1
  int n_units = 0;
  // MODE 1 with split key ranges (swa_split.cuh): the per-CTA unit list
  // [round * gridDim.x + cta] = {unit, part, parts, slot} (unit < 0 ends it),
  // and the partial rows of the parts: running max and sum [slot][2][kQT][2],
  // unnormalised O [slot][2][kQT][D].
  const int4 *items = nullptr;
  float *ws_ml = nullptr;
  float *ws_o = nullptr;
};

template <int D>
struct Fwd2Layout {
  static constexpr int PANELS = D / 64;
  // K and V have rings of their own: a K tile is free once both S MMAs have
  // read it, a V tile once both PV MMAs have, so K is released one step early.
  static constexpr int NK = D == 64 ? 4 : 3;  // K stages
  static constexpr int NV = D == 64 ? 4 : 2;  // V stages
  static constexpr uint32_t Q_BYTES = kQT * D * 2;
  static constexpr uint32_t KV_BYTES = kKT * D * 2;
  static constexpr uint32_t OFF_QA = 0;
  static constexpr uint32_t OFF_QB = Q_BYTES;
  static constexpr uint32_t OFF_K = 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NV * KV_BYTES;
  // q_full, q_empty, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2], p_full[2],
  // o_full[2], mma_drain, p2_full[2]
  static constexpr int NBAR = 2 + 2 * NK + 2 * NV + 9;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t BYTES = OFF_MISC + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
};

struct Unit {
  int b, kvh, h[2], t[2];
  bool has_b;
};

// Unit order: query tile t from the last down (heavy first).  Head pairs on
// the linear and ring layouts run t-major over every (sequence, pair), so
// the units in flight share their key tiles across all sequences.  On the
// packed layout they run sequence-major (t-major within each sequence): the
// windows of many sequences at once would not stay in L2, and a unit whose
// query tile lies past its sequence's end is skipped at no cost.
template <int MODE = 0>
__device__ __forceinline__ Unit decode_unit(int u, const Fwd2Params &p) {
  Unit U;
  if (p.pair_heads) {
    const int half = p.G >> 1;
    int t, r, bk;
    if (MODE == 2) {
      const int per_t = p.Hkv * half, per_b = per_t * p.nqt;
      const int rb = u % per_b;
      t = p.nqt - 1 - rb / per_t;
      r = rb % per_t;
      bk = (u / per_b) * p.Hkv + r / half;
    } else {
      const int per_t = p.B * p.Hkv * half;
      t = p.nqt - 1 - u / per_t;
      r = u % per_t;
      bk = r / half;
    }
    const int pair = r % half;
    U.b = bk / p.Hkv;
    U.kvh = bk % p.Hkv;
    U.h[0] = U.kvh * p.G + 2 * pair;
    U.h[1] = U.h[0] + 1;
    U.t[0] = U.t[1] = t;
    U.has_b = true;
  } else {
    const int npairs = (p.nqt + 1) >> 1;
    const int pr = npairs - 1 - u % npairs;
    const int bh = u / npairs;
    U.b = bh / p.H;
    U.h[0] = U.h[1] = bh % p.H;
    U.kvh = U.h[0] / p.G;
    U.t[0] = 2 * pr;
    U.t[1] = 2 * pr + 1;
    U.has_b = U.t[1] < p.nqt;
  }
  return U;
}

// Live key tiles of a unit in stream order, with the class for each query
// tile.  Positions are int32: MODE 0 uses absolute positions (< 2^30),
// MODE 1 positions relative to the chunk start (ring slots hold -W .. -1),
// MODE 2 positions within the unit's sequence.  The segment bases follow the
// ring layout of swa_tile.cuh.  With sinks (SINK, MODE 0 / 2), key tile 0
// comes first when the window does not reach it.
template <int MODE, bool SINK>
struct Walker2 {
  int kt, kt_end;
  int qlo[2], qhi[2];
  int W;         // MODE 0: clamped window; MODE 1: ring slots
  int n_k;       // MODE 0 key rows; MODE 1 chunk rows
  int nrt;       // MODE 1 ring tiles
  int wrap;      // MODE 1: ring full ? L mod W : number of filled slots
  bool full_ring;
  bool has_b;
  int live_a_end, live_b_begin;  // MODE 0: A is live on [kt, live_a_end], B on [live_b_begin, kt_end)
  int n_sink;        // sink keys 0 .. n_sink-1
  bool sink_pending;  // the sink tile (MODE 0 / 2: key tile 0; MODE 1: the sink rows, k = -1)
                      // still to be yielded ahead of kt
  int sink_vis[2];    // MODE 1: sinks before the window of the tile's last row
  int idx, t_lo, t_hi;  // MODE 1: stream index of the next live tile; the part's range

  // len: valid query rows of this unit's sequence (MODE 1: also its chunk keys)
  __device__ __forceinline__ void init(const Unit &U, const Fwd2Params &p, int64_t qs, int len) {
    idx = 0;
    t_lo = 0;
    t_hi = 0x7FFFFFFF;
    has_b = U.has_b;
    n_k = MODE == 0 ? p.n_k : len;
    W = static_cast<int>(p.W);
    n_sink = SINK ? p.n_sink : 0;
    sink_pending = false;
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      qlo[x] = U.t[x] * kQT;
      qhi[x] = min(qlo[x] + kQT, len) - 1;
    }
    if (MODE != 1) {
      kt = max(qlo[0] - (W - 1), 0) / kKT;
      sink_pending = SINK && n_sink > 0 && kt > 0;
      kt_end = (has_b ? qhi[1] : qhi[0]) / kKT + 1;
      // the windows of consecutive rows overlap, so each tile's live key tiles are
      // one contiguous range: [first key of its first row, its last row] in tiles
      live_a_end = qhi[0] / kKT;
      live_b_begin = max(qlo[1] - (W - 1), 0) / kKT;
      nrt = 0;
      wrap = 0;
      full_ring = false;
    } else {
      nrt = p.n_ring_tiles;
      kt = 0;
      kt_end = nrt + (len + kKT - 1) / kKT;
      full_ring = qs >= p.W;
      wrap = static_cast<int>(full_ring ? qs % p.W : qs);
      if (SINK) {
        // query row r sees sink j iff j < n_sink and j < qs + r - W + 1
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int64_t v = qs + qhi[x] - p.W + 1;
          sink_vis[x] = static_cast<int>(v < 0 ? 0 : (v > n_sink ? n_sink : v));
        }
        sink_pending = n_sink > 0 && (sink_vis[0] > 0 || (has_b && sink_vis[1] > 0));
      }
    }
  }

  // Segments of tile kt: columns [lo_g, hi_g] hold positions base_g + c.
  __device__ __forceinline__ int segments(int k, int (&lo)[2], int (&hi)[2], int (&base)[2],
                                          int &src, int &y0) const {
    lo[1] = 1;
    hi[1] = 0;
    base[1] = 0;
    if (MODE != 1 || k >= nrt) {
      const int c0 = (k - nrt) * kKT;
      const int nc = min(kKT, n_k - c0);
      src = 0;
      y0 = c0;
      lo[0] = 0;
      hi[0] = nc - 1;
      base[0] = c0;
      return nc;
    }
    const int s0 = k * kKT;
    const int nc = min(kKT, W - s0);
    src = 1;
    y0 = s0;
    if (!full_ring) {  // slots 0 .. wrap-1 hold positions 0 .. wrap-1 (relative: s - wrap)
      lo[0] = 0;
      hi[0] = min(nc - 1, wrap - 1 - s0);
      base[0] = s0 - wrap;
    } else {  // slots < wrap: position s - wrap; slots >= wrap: s - wrap - W
      lo[0] = 0;
      hi[0] = min(nc - 1, wrap - 1 - s0);
      base[0] = s0 - wrap;
      lo[1] = max(0, wrap - s0);
      hi[1] = nc - 1;
      base[1] = s0 - wrap - W;
    }
    return nc;
  }

  __device__ __forceinline__ int klass(int x, int nc, const int (&lo)[2], const int (&hi)[2],
                                       const int (&base)[2]) const {
    bool any = false;
    int all_cols = 0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      if (lo[g] > hi[g]) continue;
      const int p_lo = base[g] + lo[g], p_hi = base[g] + hi[g];
      if (p_lo <= qhi[x] && p_hi + W - 1 >= qlo[x]) any = true;
      if (p_hi <= qlo[x] && p_lo >= qhi[x] - W + 1) all_cols += hi[g] - lo[g] + 1;
    }
    // A ragged tile (nc < kKT) is masked even when every in-range pair is allowed:
    // its out-of-range columns read as zero and must not enter the softmax.
    return !any ? 0 : (all_cols == nc && nc == kKT ? 1 : 2);
  }

  // Advance to the next live tile, reporting only which query tiles use it
  // (ca, cb nonzero) -- what the producer and the MMA issuer need.  MODE 0 / 2
  // reduce to two comparisons per tile; MODE 1 runs the full classification.
  // Every query row sees key 0, so with sinks tile 0 is live for both tiles.
  __device__ __forceinline__ bool next_live(int &k, int &src, int &y0, int &ca, int &cb) {
    if (MODE != 1) {
      src = 0;
      if (SINK && sink_pending) {
        sink_pending = false;
        k = 0;
        y0 = 0;
        ca = 1;
        cb = has_b;
        return true;
      }
      if (kt >= kt_end) return false;
      k = kt++;
      y0 = k * kKT;
      ca = k <= live_a_end;
      cb = has_b && (k >= live_b_begin || (SINK && k == 0 && n_sink > 0));
      return true;
    }
    return next(k, src, y0, ca, cb);
  }

  // MODE 1, part `part` of `parts`: keep only the part's contiguous piece of
  // the live tiles (by count), for a unit whose key range is split.
  __device__ __forceinline__ void set_part(int part, int parts) {
    if (parts <= 1) return;
    Walker2 w = *this;
    int n = 0, k, src, y0, ca, cb;
    while (w.next_all(k, src, y0, ca, cb)) ++n;
    t_lo = part * n / parts;
    t_hi = (part + 1) * n / parts;
  }

  // Advance to the next live tile: its index, source, first row and classes.
  // MODE 1 skips the tiles outside the part's range (set_part).
  __device__ __forceinline__ bool next(int &k, int &src, int &y0, int &ca, int &cb) {
    if (MODE != 1) return next_all(k, src, y0, ca, cb);
    while (next_all(k, src, y0, ca, cb)) {
      const int i = idx++;
      if (i < t_lo) continue;
      return i < t_hi;
    }
    return false;
  }

  // Every live tile in stream order.  Tile 0 under sinks is partial unless
  // the window alone covers it.
  __device__ __forceinline__ bool next_all(int &k, int &src, int &y0, int &ca, int &cb) {
    int lo[2], hi[2], base[2];
    if (SINK && MODE == 1 && sink_pending) {
      sink_pending = false;
      k = -1;
      src = 2;
      y0 = 0;
      ca = sink_vis[0] > 0 ? 2 : 0;
      cb = (has_b && sink_vis[1] > 0) ? 2 : 0;
      return true;
    }
    if (SINK && MODE != 1 && sink_pending) {
      sink_pending = false;
      k = 0;
      segments(0, lo, hi, base, src, y0);
      ca = 2;
      cb = has_b ? 2 : 0;
      return true;
    }
    while (kt < kt_end) {
      k = kt++;
      const int nc = segments(k, lo, hi, base, src, y0);
      ca = klass(0, nc, lo, hi, base);
      cb = has_b ? klass(1, nc, lo, hi, base) : 0;
      if (SINK && MODE != 1 && k == 0 && n_sink > 0) {
        if (ca != 1) ca = 2;
        if (has_b && cb != 1) cb = 2;
      }
      if (ca | cb) return true;
    }
    return false;
  }
};

// Per-warpgroup register budget (all four warps of the warpgroup execute it).
template <int N>
__device__ __forceinline__ void warpgroup_regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void warpgroup_regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <int D, int MODE, bool SINK>
__global__ void __launch_bounds__(kFwd2Threads, 1)
    fwd2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kr,
                const __grid_constant__ CUtensorMap tm_vr,
                const __grid_constant__ CUtensorMap tm_ks,
                const __grid_constant__ CUtensorMap tm_vs, const Fwd2Params p) {
  using L = Fwd2Layout<D>;
  constexpr int NK = L::NK, NV = L::NV;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw);
  const uint32_t sQ[2] = {base + L::OFF_QA, base + L::OFF_QB};
  const uint32_t sK = base + L::OFF_K, sV = base + L::OFF_V, bar = base + L::OFF_BAR;
  const uint32_t BAR_QF = bar, BAR_QE = bar + 8;
  const uint32_t BAR_KF = bar + 16;                 // + 8 * K stage
  const uint32_t BAR_KE = BAR_KF + 8 * NK;          // + 8 * K stage
  const uint32_t BAR_VF = BAR_KE + 8 * NK;          // + 8 * V stage
  const uint32_t BAR_VE = BAR_VF + 8 * NV;          // + 8 * V stage
  const uint32_t BAR_S = BAR_VE + 8 * NV;           // + 8 * tile
  const uint32_t BAR_P = BAR_S + 16;                // + 8 * tile
  const uint32_t BAR_O = BAR_P + 16;                // + 8 * tile
  const uint32_t BAR_DRAIN = BAR_O + 16;            // the MMA thread's teardown
  const uint32_t BAR_P2 = BAR_DRAIN + 8;            // + 8 * tile: second half of P stored
  // P is handed to the PV MMA in two halves of 64 keys (the first half's PV
  // runs while the softmax computes the second), except on the ring layout,
  // whose MMA thread already does more per tile (there the split measured
  // 2% slower; on the linear and packed layouts 3-6% faster).
  constexpr bool kSplitP = MODE != 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + L::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR_QF, 1);
    mbar_init(BAR_QE, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(BAR_KF + 8 * s, 1);
      mbar_init(BAR_KE + 8 * s, 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(BAR_VF + 8 * s, 1);
      mbar_init(BAR_VE + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(BAR_S + 8 * x, 1);
      mbar_init(BAR_P + 8 * x, 4 * 32);
      mbar_init(BAR_P2 + 8 * x, 4 * 32);
      mbar_init(BAR_O + 8 * x, 1);
    }
    mbar_init(BAR_DRAIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (MODE == 1) {
      tma_prefetch_desc(&tm_kr);
      tma_prefetch_desc(&tm_vr);
    }
    if (MODE == 1 && SINK) {
      tma_prefetch_desc(&tm_ks);
      tma_prefetch_desc(&tm_vs);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Serpentine static schedule over the heavy-first unit order: in round r
  // CTA c takes unit r * P + c (r even) or r * P + P - 1 - c (r odd), which
  // pairs heavy with light units.
  auto unit_of = [&](int i) -> int {
    const int P = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return i * P + ((i & 1) ? P - 1 - c : c);
  };
  // The i-th unit of this CTA and which part of it (of `parts`; slot: the
  // part's partial rows): from the split schedule's list when there is one.
  auto item_of = [&](int i, int &u, int &part, int &parts, int &slot) -> bool {
    if (MODE == 1 && p.items) {
      const int4 v = p.items[static_cast<int64_t>(i) * gridDim.x + blockIdx.x];
      u = v.x;
      part = v.y;
      parts = v.z;
      slot = v.w;
      return u >= 0;
    }
    u = unit_of(i);
    part = 0;
    parts = 1;
    slot = -1;
    return u < p.n_units;
  };

  // 0: run the unit; 1: invalid start position, chunk length or sequence
  // offsets (skip, flag); 2: the unit's query rows are all padding of a
  // shorter chunk or sequence (skip).  qs: MODE 1 the chunk's first position,
  // MODE 2 the sequence's first token.
  // Every role evaluates it identically, so they skip the same units.
  auto unit_start = [&](Unit &U, int64_t &qs, int &len) -> int {
    qs = 0;
    len = p.n_q;
    if (MODE == 1) {
      qs = p.q_start[U.b];
      if (qs < 0) return 1;
      if (p.chunk_len) {
        const int64_t l = p.chunk_len[U.b];
        if (l < 0 || l > p.n_q) return 1;
        len = static_cast<int>(l);
      }
    } else if (MODE == 2) {
      const int64_t a = p.cu_seqlens[U.b], e = p.cu_seqlens[U.b + 1];
      if (a < 0 || e < a || e - a > p.n_q || e > p.total) return 1;
      qs = a;  // first token of the sequence
      len = static_cast<int>(e - a);
    }
    if (MODE != 0) {
      if (U.t[0] * kQT >= len) return 2;
      if (U.has_b && U.t[1] * kQT >= len) U.has_b = false;
    }
    return 0;
  };

  if (warp < 4) {
  warpgroup_regs_dec<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int kv_iter = 0, q_iter = 0;
      bool k_ahead = false;  // K of iteration kv_iter issued, its V not (abort between them)
      int u, part, parts, slot;
      for (int it = 0; item_of(it, u, part, parts, slot); ++it) {
        Unit U = decode_unit<MODE>(u, p);
        int64_t qs;
        int len;
        const int ust = unit_start(U, qs, len);
        if (ust) {
          if (ust == 1) atomicOr(&g_swa_status, SWA_DEV_BADARG);
          continue;
        }
        if (q_iter > 0 && !mbar_wait(BAR_QE, (q_iter - 1) & 1, abort_flag)) break;
        mbar_expect_tx(BAR_QF, (U.has_b ? 2u : 1u) * L::Q_BYTES);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x == 1 && !U.has_b) break;
#pragma unroll
          for (int pn = 0; pn < L::PANELS; ++pn)
            if (MODE == 2)
              tma_load_3d(sQ[x] + pn * (kQT * 128), &tm_q, BAR_QF, pn * 64, U.h[x],
                          static_cast<int>(qs) + U.t[x] * kQT);
            else
              tma_load_3d(sQ[x] + pn * (kQT * 128), &tm_q, BAR_QF, pn * 64, U.t[x] * kQT,
                          U.b * p.H + U.h[x]);
        }
        ++q_iter;
        Walker2<MODE, SINK> wk;
        wk.init(U, p, qs, len);
        wk.set_part(part, parts);
        int k, src, y0, ca, cb;
        // MODE 2 maps are {D, heads, tokens}: (head, token) replace (row, plane)
        const int z = MODE == 2 ? static_cast<int>(qs) : U.b * p.Hkv + U.kvh;
        while (wk.next_live(k, src, y0, ca, cb)) {
          const int sk = kv_iter % NK, sv = kv_iter % NV;
          const CUtensorMap *mk = src == 1 ? &tm_kr : (src == 2 ? &tm_ks : &tm_k);
          const CUtensorMap *mv = src == 1 ? &tm_vr : (src == 2 ? &tm_vs : &tm_v);
          if (kv_iter >= NK && !mbar_wait(BAR_KE + 8 * sk, ((kv_iter / NK) - 1) & 1, abort_flag))
            break;
          mbar_expect_tx(BAR_KF + 8 * sk, L::KV_BYTES);
#pragma unroll
          for (int pn = 0; pn < L::PANELS; ++pn)
            tma_load_3d(sK + sk * L::KV_BYTES + pn * (kKT * 128), mk, BAR_KF + 8 * sk, pn * 64,
                        MODE == 2 ? U.kvh : y0, MODE == 2 ? z + y0 : z);
          if (kv_iter >= NV &&
              !mbar_wait(BAR_VE + 8 * sv, ((kv_iter / NV) - 1) & 1, abort_flag)) {
            k_ahead = true;
            break;
          }
          mbar_expect_tx(BAR_VF + 8 * sv, L::KV_BYTES);
#pragma unroll
          for (int pn = 0; pn < L::PANELS; ++pn)
            tma_load_3d(sV + sv * L::KV_BYTES + pn * (kKT * 128), mv, BAR_VF + 8 * sv, pn * 64,
                        MODE == 2 ? U.kvh : y0, MODE == 2 ? z + y0 : z);
          ++kv_iter;
        }
        if (*abort_flag) break;
      }
      // every copy issued must land before the CTA ends: wait for the last
      // phase of each barrier that a copy was issued on
      if (q_iter > 0) mbar_drain(BAR_QF, (q_iter - 1) & 1);
      const int k_issued = kv_iter + (k_ahead ? 1 : 0);
      for (int i = max(0, k_issued - NK); i < k_issued; ++i)
        mbar_drain(BAR_KF + 8 * (i % NK), (i / NK) & 1);
      for (int i = max(0, kv_iter - NV); i < kv_iter; ++i)
        mbar_drain(BAR_VF + 8 * (i % NV), (i / NV) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kQT, kKT, false);
      constexpr uint32_t idO = idesc_bf16_f32(kQT, D, true);
      int kv_iter = 0, q_iter = 0;
      uint32_t p_cnt[2] = {0u, 0u};
      // Shared-memory descriptors as (low word + offset >> 4, constant high
      // word): one 32-bit add per MMA.  The empty asm keeps the compiler from
      // precomputing every MMA's words for the whole loop, which would spill.
      constexpr uint32_t kDescHi = sdesc_sw128_hi(1024);
      const uint32_t q_lo[2] = {sdesc_sw128_lo(sQ[0], 16), sdesc_sw128_lo(sQ[1], 16)};
      const uint32_t k_lo = sdesc_sw128_lo(sK, 16), v_lo = sdesc_sw128_lo(sV, kKT * 128);
      auto issue_s = [&](int x, int st) {
        uint32_t qb = q_lo[x], kb = k_lo + st * (L::KV_BYTES >> 4), dS = tmem + x * 128;
        asm volatile("" : "+r"(qb), "+r"(kb), "+r"(dS));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = (kk >> 2) * (kQT * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kKT * 128) + (kk & 3) * 32;
          mma_ss_w(dS, qb + (offq >> 4), kb + (offk >> 4), kDescHi, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(BAR_S + 8 * x);
      };
      // PV over keys k_begin .. k_begin + n_keys - 1 of the tile
      auto issue_pv = [&](int x, int st, bool acc, int k_begin, int n_keys) {
        uint32_t dO = tmem + 256 + x * D, aP = tmem + x * 128, vb = v_lo + st * (L::KV_BYTES >> 4);
        asm volatile("" : "+r"(vb), "+r"(dO), "+r"(aP));
#pragma unroll
        for (int k16 = 0; k16 < n_keys / 16; ++k16) {
          const int kk = k_begin / 16 + k16;
          mma_ts_w(dO, aP + kk * 8, vb + ((kk * 16 * 128) >> 4), kDescHi, idO,
                   (acc || kk > 0) ? 1u : 0u);
        }
      };
      // P_X of one tile: in two halves (kSplitP), or whole; false if a wait gave up
      auto pv_tile = [&](int x, int st, bool acc) -> bool {
        if (kSplitP) {
          issue_pv(x, st, acc, 0, kKT / 2);
          if (!mbar_wait(BAR_P2 + 8 * x, p_cnt[x] & 1, abort_flag)) return false;
          tc_fence_after();
          issue_pv(x, st, true, kKT / 2, kKT / 2);
        } else {
          issue_pv(x, st, acc, 0, kKT);
        }
        return true;
      };
      int u, part, parts, slot;
      for (int it = 0; item_of(it, u, part, parts, slot); ++it) {
        Unit U = decode_unit<MODE>(u, p);
        int64_t qs;
        int len;
        if (unit_start(U, qs, len)) continue;
        if (!mbar_wait(BAR_QF, q_iter & 1, abort_flag)) break;
        tc_fence_after();
        Walker2<MODE, SINK> wk;
        wk.init(U, p, qs, len);
        wk.set_part(part, parts);
        int k, src, y0, ca, cb, na = 0, nb = 0;
        bool have = wk.next_live(k, src, y0, ca, cb);
        bool first[2] = {true, true};
        if (!have) {  // no live tile: keep the Q barriers' phase counts in step
          tc_commit(BAR_QE);
          ++q_iter;
          continue;
        }
        bool has_next = wk.next_live(k, src, y0, na, nb);
        {
          const int sk = kv_iter % NK;
          if (!mbar_wait(BAR_KF + 8 * sk, (kv_iter / NK) & 1, abort_flag)) break;
          tc_fence_after();
          if (ca) issue_s(0, sk);
          if (cb) issue_s(1, sk);
        }
        // tile B starting one tile after A (query tiles 2p, 2p+1): issue its first
        // S now instead of behind A's first softmax
        bool b_ahead = false;
        if (MODE != 1 && has_next && nb && !cb) {
          const int sk1 = (kv_iter + 1) % NK;
          if (!mbar_wait(BAR_KF + 8 * sk1, ((kv_iter + 1) / NK) & 1, abort_flag)) break;
          tc_fence_after();
          issue_s(1, sk1);
          b_ahead = true;
        }
        tc_commit(BAR_KE + 8 * (kv_iter % NK));  // K(first) is read by both S MMAs
        bool o_done[2] = {false, false};
        const bool b_contig = MODE != 1 && (!SINK || p.n_sink == 0 || p.pair_heads);
        bool stop = false;  // a wait gave up: issue nothing more
        while (have) {
          if (!has_next) tc_commit(BAR_QE);  // every S of this unit is issued
          const int sv = kv_iter % NV;
          const int skn = (kv_iter + 1) % NK;
          if (!mbar_wait(BAR_VF + 8 * sv, (kv_iter / NV) & 1, abort_flag)) {
            stop = true;
            break;
          }
          if (ca) {
            if (!mbar_wait(BAR_P, p_cnt[0] & 1, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            if (!pv_tile(0, sv, !first[0])) {
              stop = true;
              break;
            }
            ++p_cnt[0];
            first[0] = false;
            // linear keys: a query tile's live tiles are contiguous, so it is done
            // (tile A's stay so with the sink tile in front; B's need not)
            if (MODE != 1 && !(has_next && na)) {
              tc_commit(BAR_O);
              o_done[0] = true;
            }
          }
          if (has_next) {
            if (!mbar_wait(BAR_KF + 8 * skn, ((kv_iter + 1) / NK) & 1, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            if (na) issue_s(0, skn);
          }
          if (cb) {
            if (!mbar_wait(BAR_P + 8, p_cnt[1] & 1, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            if (!pv_tile(1, sv, !first[1])) {
              stop = true;
              break;
            }
            ++p_cnt[1];
            first[1] = false;
            if (b_contig && !(has_next && nb)) {
              tc_commit(BAR_O + 8);
              o_done[1] = true;
            }
          }
          tc_commit(BAR_VE + 8 * sv);  // V(j) is read by both PV MMAs
          if (has_next) {
            if (nb && !b_ahead) issue_s(1, skn);
            b_ahead = false;
            tc_commit(BAR_KE + 8 * skn);
          }
          ++kv_iter;
          ca = na;
          cb = nb;
          have = has_next;
          if (have) has_next = wk.next_live(k, src, y0, na, nb);
        }
        if (stop) break;
        // o_final completes once per unit in which the tile had work; its next
        // completion needs that tile's softmax to hand over its next P, so it
        // can never run two phases ahead of the waiting softmax warps
        if (!first[0] && !o_done[0]) tc_commit(BAR_O);
        if (!first[1] && !o_done[1]) tc_commit(BAR_O + 8);
        ++q_iter;
      }
      // every MMA issued must complete before the tensor memory is freed
      tc_commit(BAR_DRAIN);
      mbar_drain(BAR_DRAIN, 0);
    }
  }  // warps 2 and 3 have no role
  } else {
    warpgroup_regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax + epilogue
    const int x = warp < 8 ? 0 : 1;  // query tile of this warp group
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + x * 128 + lane_off;
    const uint32_t tO = tmem + 256 + x * D + lane_off;
    uint32_t s_cnt = 0, u_iter = 0;
    bool stop = false;  // a wait gave up (the whole warp): no more TMEM work or stores
    int u, part, parts, slot;
    for (int it = 0; item_of(it, u, part, parts, slot); ++it) {
      Unit U = decode_unit<MODE>(u, p);
      int64_t qs;
      int len;
      if (unit_start(U, qs, len)) continue;
      Walker2<MODE, SINK> wk;
      wk.init(U, p, qs, len);
      wk.set_part(part, parts);
      // MODE 0 absolute, MODE 1 relative to q_start, MODE 2 within the sequence
      const int qrow = U.t[x] * kQT + row;
      float m_run = -INFINITY, l_run = 0.f;
      int nt = 0;
      int k, src, y0, ca, cb;
      while (wk.next(k, src, y0, ca, cb)) {
        const int cls = x == 0 ? ca : cb;
        if (!cls) continue;
        if (!mbar_wait_warp(BAR_S + 8 * x, s_cnt & 1, abort_flag)) {
          stop = true;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128(tS, sr);
        float *s = reinterpret_cast<float *>(sr);
        if (cls == 2) {
          // allowed columns of this row: c in a segment with base + c in [q - W + 1, q],
          // as a 128-bit mask (one word per 32 columns)
          int lo[2] = {1, 1}, hi[2] = {0, 0}, base[2], s_, y_;
          int sink_hi = -1;
          if (SINK && MODE == 1 && k < 0) {
            // the sink rows: columns below min(n_sink, q - W + 1) (q absolute)
            const int64_t v = qs + qrow - wk.W + 1;
            sink_hi = static_cast<int>(v < 0 ? 0 : (v > wk.n_sink ? wk.n_sink : v)) - 1;
          } else {
            wk.segments(k, lo, hi, base, s_, y_);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              lo[g] = max(lo[g], qrow - wk.W + 1 - base[g]);
              hi[g] = min(hi[g], qrow - base[g]);
            }
            // sinks: columns 0 .. n_sink-1 of tile 0, up to the row itself
            if (SINK && MODE != 1 && k == 0) sink_hi = min(wk.n_sink - 1, qrow);
          }
          uint32_t mw[kKT / 32];
#pragma unroll
          for (int w = 0; w < kKT / 32; ++w)
            mw[w] = range_bits(lo[0] - 32 * w, hi[0] - 32 * w) |
                    range_bits(lo[1] - 32 * w, hi[1] - 32 * w) |
                    range_bits(-32 * w, sink_hi - 32 * w);
#pragma unroll
          for (int c = 0; c < kKT; ++c) s[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? s[c] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = s[i];
#pragma unroll
        for (int c = 8; c + 16 <= kKT; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], s[c + i], s[c + 8 + i]);
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[kKT - 8 + i]);
        const float m_raw = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7]));
        const float m_tile = m_raw * p.scale_log2;
        const bool grow = m_tile > m_run + kLazyRescaleLog2;
        const float m_new = grow ? m_tile : m_run;
        const float alpha = grow ? ex2(m_run - m_new) : 1.f;
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        // x = s * scale * log2(e) - m, two columns per packed FMA
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_use, -m_use);
        float2 *s2 = reinterpret_cast<float2 *>(s);
#pragma unroll
        for (int c = 0; c < kKT / 2; ++c) s2[c] = __ffma2_rn(s2[c], sc2, nm2);
        // P of keys 64h .. 64h + 63 as bf16 pairs (key 2c in the low half of
        // column c) into columns 32h .. 32h + 31 of S_X; no wait
        auto store_p = [&](int h) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pack_bf16(s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]);
          tmem_st32(tS + h * 32, pk);
        };
        auto rescale_o = [&](float a) {
#pragma unroll 1
          for (int cb2 = 0; cb2 < D / 32; ++cb2) {
            uint32_t o32[32];
            tmem_ld32(tO + cb2 * 32, o32);
#pragma unroll
            for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * a);
            tmem_st32(tO + cb2 * 32, o32);
          }
        };
        if (kSplitP) {
          // O_X is stable (PV_X of the previous tile was issued before this
          // S_X): rescale it before the first half of P hands PV_X the tile
          if (nt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) rescale_o(alpha);
          // exponentials on the MUFU (a masked column gives 2^-inf = 0) in two
          // halves of 64 keys; P of the first half (bf16 pairs, key 2c in the
          // low half of column c) goes to PV_X while the second is computed
          float2 sm2[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) sm2[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
            for (int c = h2 * 64; c < h2 * 64 + 64; ++c) s[c] = ex2(s[c]);
#pragma unroll
            for (int c = h2 * 32; c < h2 * 32 + 32; c += 4)
#pragma unroll
              for (int i = 0; i < 4; ++i) sm2[i] = __fadd2_rn(sm2[i], s2[c + i]);
            store_p(h2);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(h2 == 0 ? BAR_P + 8 * x : BAR_P2 + 8 * x);
          }
          const float2 sa = __fadd2_rn(__fadd2_rn(sm2[0], sm2[1]), __fadd2_rn(sm2[2], sm2[3]));
          l_run = l_run * alpha + (sa.x + sa.y);
          m_run = m_new;
        } else {
          // exponentials on the MUFU (a masked column gives 2^-inf = 0)
#pragma unroll
          for (int c = 0; c < kKT; ++c) s[c] = ex2(s[c]);
          float2 sm2[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) sm2[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < kKT / 2; c += 4)
#pragma unroll
            for (int i = 0; i < 4; ++i) sm2[i] = __fadd2_rn(sm2[i], s2[c + i]);
          const float2 sa = __fadd2_rn(__fadd2_rn(sm2[0], sm2[1]), __fadd2_rn(sm2[2], sm2[3]));
          l_run = l_run * alpha + (sa.x + sa.y);
          m_run = m_new;
          store_p(0);
          store_p(1);
          // O_X is stable: PV_X of the previous tile was issued before this S_X
          if (nt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) rescale_o(alpha);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(BAR_P + 8 * x);
        }
        ++nt;
      }
      if (stop) break;
      if (MODE == 1 && parts > 1) {
        // one part of a split unit: this row's unnormalised O with its running
        // max and sum, for the merge kernel (a row the part gave no key to
        // gets sum 0, which the merge skips)
        const int64_t r = (static_cast<int64_t>(slot) * 2 + x) * kQT + row;
        if (nt > 0) {
          if (!mbar_wait_warp(BAR_O + 8 * x, u_iter & 1, abort_flag)) break;
          ++u_iter;
          tc_fence_after();
          float4 *po = reinterpret_cast<float4 *>(p.ws_o + r * D);
#pragma unroll 1
          for (int c32 = 0; c32 < D / 32; ++c32) {
            uint32_t o32[32];
            tmem_ld32(tO + c32 * 32, o32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              po[c32 * 8 + i] = make_float4(__uint_as_float(o32[4 * i]), __uint_as_float(o32[4 * i + 1]),
                                            __uint_as_float(o32[4 * i + 2]),
                                            __uint_as_float(o32[4 * i + 3]));
          }
        }
        p.ws_ml[2 * r] = m_run;
        p.ws_ml[2 * r + 1] = nt > 0 ? l_run : 0.f;
      } else if (nt > 0) {
        // every PV of this unit is done
        if (!mbar_wait_warp(BAR_O + 8 * x, u_iter & 1, abort_flag)) break;
        ++u_iter;
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        const int hh = U.h[x];
        // rows of this lane's 8-lane group: whole 128-byte segments per store
        const int grp_row = U.t[x] * kQT + quad * 32 + (lane & ~7);
        store_tile_rows<D>(
            p.out + (MODE == 2 ? (qs + grp_row) * p.H + hh
                               : static_cast<int64_t>(U.b * p.H + hh) * p.n_q + grp_row) *
                        static_cast<int64_t>(D),
            MODE == 2 ? static_cast<int64_t>(p.H) * D : D, len - grp_row, tO, inv_l, lane);
        if (p.lse && qrow < len)
          p.lse[MODE == 2 ? static_cast<int64_t>(hh) * p.total + qs + qrow
                          : static_cast<int64_t>(U.b * p.H + hh) * p.n_q + qrow] =
              (m_run + __log2f(l_run)) * 0.6931471805599453f;
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace swa
