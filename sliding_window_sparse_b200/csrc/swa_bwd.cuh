// swa_bwd.cuh -- gradients of the sliding-window prefill on tcgen05 tensor cores.
//
// The M003 note (section 07) checks the Q/K/V gradients of the windowed
// attention under the same mask as the forward output; the gradients are
// those of the loss sum(out * dout):
//   P = softmax over the allowed keys of scale * Q K^T (from the forward's LSE)
//   dP = dout V^T,  D_i = <dout_i, out_i>,  dS = P o (dP - D)
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dout
// with dK and dV summed over the G query heads of a KV head.
//
// Two persistent kernels with the forward's roles, 192 threads each: one
// thread issues the MMAs, one feeds TMA, four warps (one 128-row tile, a row
// per thread) do the element-wise work between the MMAs in tensor memory.
//
//  * bwd_dq_kernel: one query tile of one head per unit.  Per live key tile:
//    S = Q K^T and dP = dO V^T on the tensor cores, dS = P o (dP - D) in
//    registers (P from the LSE, no running max), dQ += dS K with dS read from
//    tensor memory.  It also writes D_i (which it computes from out and dout
//    rows at the start of the unit) for the second kernel.
//  * bwd_dkdv_kernel: one key tile of one KV head per unit, walking every
//    (query head of the group, live query tile): S^T = K Q^T, dP^T = V dO^T,
//    P^T and dS^T in registers (a row per key), dV += P^T dO and
//    dK += dS^T Q with P^T, dS^T read from tensor memory.
//
// Key tile j and query tile t interact iff some key of j is in the window of
// some query of t (the M003 note, section 04's skip rule); partial tiles are
// masked per row with 128-bit column masks.
//
// Layouts (MODE): 0 = [B, heads, N, D] per tensor; 2 = packed token-major
// [total, heads, D] with sequence b on tokens cu_seqlens[b] .. cu_seqlens[b+1]-1
// and positions restarting at 0 in each sequence (the "Dense attention vs
// sparse SWA" blog, section 5.2 tip 4: the window is per sequence).  SINK adds
// attention sinks (sparse-attention taxonomy page, section 3.2): key j < n_sink
// stays visible to every later query of its sequence, so query tile t also
// reads key tile 0, and key tile 0 is read by every query tile.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "swa_epilogue.cuh"

namespace swa {

constexpr int kBwdT = 128;            // query and key tile rows
constexpr int kBwdThreads = 6 * 32;   // producer, MMA issuer, 4 element-wise warps

// MODE 2: out, dout, dq [total, H, D]; dk, dv [total, Hkv, D]; lse, delta [H, total].
struct BwdParams {
  const __nv_bfloat16 *out;   // [B, H, N, D]
  const __nv_bfloat16 *dout;  // [B, H, N, D]
  const float *lse;           // [B, H, N] natural log
  float *delta;               // [B, H, N] workspace: D_i
  __nv_bfloat16 *dq;          // [B, H, N, D]
  __nv_bfloat16 *dk, *dv;     // [B, Hkv, N, D]
  int B = 0, H = 0, Hkv = 0, G = 0;
  int N = 0;                  // MODE 2: the longest sequence
  int W = 0;                  // window, clamped to N + kBwdT
  float scale = 0.f, scale_log2 = 0.f;
  int nt = 0;                 // tiles per (b, head): ceil(N / 128)
  int n_units = 0;
  const int64_t *cu_seqlens = nullptr;  // MODE 2: [B + 1]
  int64_t total = 0;                    // MODE 2: packed tokens
  int n_sink = 0;                       // SINK: keys 0 .. n_sink-1 of each sequence
};

template <int D>
struct BwdLayout {
  static constexpr int PANELS = D / 64;
  static constexpr uint32_t TILE = kBwdT * D * 2;  // one 128-row bf16 tile
  static constexpr int NS = 2;                      // streamed-tile stages
  // dq kernel: Q, dO once per unit; K, V per key tile
  // dkdv kernel: K, V once per unit; Q, dO per step
  static constexpr uint32_t OFF_A0 = 0;             // Q (dq) / K (dkdv)
  static constexpr uint32_t OFF_A1 = TILE;          // dO (dq) / V (dkdv)
  static constexpr uint32_t OFF_S0 = 2 * TILE;      // NS stages of K (dq) / Q (dkdv)
  static constexpr uint32_t OFF_S1 = OFF_S0 + NS * TILE;  // NS stages of V (dq) / dO (dkdv)
  static constexpr uint32_t OFF_VEC = OFF_S1 + NS * TILE; // dkdv: lse2 and D per column, 2 copies
  static constexpr uint32_t OFF_BAR = OFF_VEC + 2 * 2 * kBwdT * 4;
  static constexpr int NBAR = 16 + 4 * NS;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t BYTES = OFF_MISC + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;
};

// Store 16 columns (32x32b.x16, one lane per thread); no wait.
__device__ __forceinline__ void tmem_st16_b(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Issue a 32-column tensor-memory load without waiting; tmem_ld_wait2 waits
// for every load this thread issued and ties the two destination arrays to
// the wait, so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait2(uint32_t (&a)[32], uint32_t (&b)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]), "+r"(a[16]), "+r"(a[17]), "+r"(a[18]), "+r"(a[19]), "+r"(a[20]), "+r"(a[21]), "+r"(a[22]), "+r"(a[23]), "+r"(a[24]), "+r"(a[25]), "+r"(a[26]), "+r"(a[27]), "+r"(a[28]), "+r"(a[29]), "+r"(a[30]), "+r"(a[31]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15]), "+r"(b[16]), "+r"(b[17]), "+r"(b[18]), "+r"(b[19]), "+r"(b[20]), "+r"(b[21]), "+r"(b[22]), "+r"(b[23]), "+r"(b[24]), "+r"(b[25]), "+r"(b[26]), "+r"(b[27]), "+r"(b[28]), "+r"(b[29]), "+r"(b[30]), "+r"(b[31])
               :
               : "memory");
}

// Columns [lo, hi] (clipped to the tile) as four 32-bit words.
__device__ __forceinline__ void col_mask(int lo, int hi, uint32_t (&mw)[4]) {
#pragma unroll
  for (int w = 0; w < 4; ++w) mw[w] = range_bits(lo - 32 * w, hi - 32 * w);
}

// The sequence of batch entry b: its first token `a` (MODE 2; 0 otherwise) and
// its length.  Returns 1 when MODE 2 offsets are out of range.
template <int MODE>
__device__ __forceinline__ int bwd_seq(const BwdParams &p, int b, int64_t &a, int &len) {
  a = 0;
  len = p.N;
  if (MODE == 2) {
    const int64_t s = p.cu_seqlens[b], e = p.cu_seqlens[b + 1];
    if (s < 0 || e < s || e - s > p.N || e > p.total) return 1;
    a = s;
    len = static_cast<int>(e - s);
  }
  return 0;
}

// The key tiles of query tile t in the dQ kernel's order: key tile 0 first
// when it holds sinks the window does not reach, then k_lo .. t.
struct DqTiles {
  int k_lo, n;
  bool sink;
  __device__ __forceinline__ int kt(int j) const {
    return sink ? (j == 0 ? 0 : k_lo + j - 1) : k_lo + j;
  }
};
template <bool SINK>
__device__ __forceinline__ DqTiles dq_tiles(const BwdParams &p, int t) {
  DqTiles r;
  r.k_lo = max(t * kBwdT - (p.W - 1), 0) / kBwdT;
  r.sink = SINK && p.n_sink > 0 && r.k_lo > 0;
  r.n = t - r.k_lo + 1 + (r.sink ? 1 : 0);
  return r;
}

// Element offset of (row r of head h) in a [B, heads, N, D] tensor (MODE 0,
// b = batch entry, r from 0) or a [total, heads, D] one (MODE 2, token a + r).
template <int MODE>
__device__ __forceinline__ int64_t bwd_row(const BwdParams &p, int b, int64_t a, int heads, int h,
                                           int r) {
  return MODE == 2 ? (a + r) * heads + h : (static_cast<int64_t>(b) * heads + h) * p.N + r;
}
// Index of (row r, head h) in the per-row fp32 arrays lse and delta.
template <int MODE>
__device__ __forceinline__ int64_t bwd_vec(const BwdParams &p, int b, int64_t a, int h, int r) {
  return MODE == 2 ? static_cast<int64_t>(h) * p.total + a + r
                   : (static_cast<int64_t>(b) * p.H + h) * p.N + r;
}

// ---------------------------------------------------------------------------------- dQ
// Unit u: (b, h, query tile t), heaviest tiles first.
template <int D, int MODE, bool SINK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + L::OFF_A0, sDO = base + L::OFF_A1;
  const uint32_t sK = base + L::OFF_S0, sV = base + L::OFF_S1;
  const uint32_t bar = base + L::OFF_BAR;
  const uint32_t BAR_QF = bar, BAR_QE = bar + 8;
  const uint32_t BAR_SF = bar + 16;        // + 8 * S buffer
  const uint32_t BAR_DPF = bar + 32;
  const uint32_t BAR_EL = bar + 40;        // element-wise done with tile j (128 arrivals)
  const uint32_t BAR_DQF = bar + 48;       // dQ final
  const uint32_t BAR_DQE = bar + 56;       // dQ read out (128 arrivals)
  const uint32_t BAR_DRAIN = bar + 64;     // the MMA thread's teardown
  const uint32_t BAR_KF = bar + 128;       // + 8 * stage
  const uint32_t BAR_KE = BAR_KF + 8 * NS;
  const uint32_t BAR_VF = BAR_KE + 8 * NS;
  const uint32_t BAR_VE = BAR_VF + 8 * NS;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + L::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR_QF, 1);
    mbar_init(BAR_QE, 1);
    mbar_init(BAR_SF, 1);
    mbar_init(BAR_SF + 8, 1);
    mbar_init(BAR_DPF, 1);
    mbar_init(BAR_EL, 4 * 32);
    mbar_init(BAR_DQF, 1);
    mbar_init(BAR_DQE, 4 * 32);
    mbar_init(BAR_DRAIN, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(BAR_KF + 8 * s, 1);
      mbar_init(BAR_KE + 8 * s, 1);
      mbar_init(BAR_VF + 8 * s, 1);
      mbar_init(BAR_VE + 8 * s, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // tensor memory: S double buffer [0, 256), dP [256, 384), dQ [384, 384 + D)
  const uint32_t T_S = 0, T_DP = 256, T_DQ = 384;

  // unit -> (b, h, t) and its sequence; 0: run it, 1: bad sequence offsets
  // (skip, flag), 2: the query tile lies past the sequence's end (skip).
  // Every role evaluates it identically, so they skip the same units.
  // Query tiles from the last down; on the packed layout sequence by
  // sequence (so the key tiles of the units in flight stay in L2), elsewhere
  // across every (b, head) at once.
  auto unit = [&](int u, int &b, int &h, int &t, int64_t &a, int &len) -> int {
    if (MODE == 2) {
      const int per_b = p.H * p.nt, r = u % per_b;
      b = u / per_b;
      t = p.nt - 1 - r / p.H;
      h = r % p.H;
    } else {
      const int per_t = p.B * p.H;
      t = p.nt - 1 - u / per_t;
      const int bh = u % per_t;
      b = bh / p.H;
      h = bh % p.H;
    }
    if (bwd_seq<MODE>(p, b, a, len)) return 1;
    return t * kBwdT >= len ? 2 : 0;
  };
  auto unit_of = [&](int i) -> int {
    const int P = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return i * P + ((i & 1) ? P - 1 - c : c);
  };

  if (warp == 0) {
    // --------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int q_iter = 0, kv_iter = 0;
      bool k_ahead = false;  // K of iteration kv_iter issued, its V not (abort between them)
      for (int it = 0, u = unit_of(0); u < p.n_units; u = unit_of(++it)) {
        int b, h, t, len;
        int64_t a;
        const int ust = unit(u, b, h, t, a, len);
        if (ust) {
          if (ust == 1) atomicOr(&g_swa_status, SWA_DEV_BADARG);
          continue;
        }
        const DqTiles tl = dq_tiles<SINK>(p, t);
        if (q_iter > 0 && !mbar_wait(BAR_QE, (q_iter - 1) & 1, abort_flag)) break;
        mbar_expect_tx(BAR_QF, 2 * L::TILE);
        // MODE 2 maps are {D, heads, tokens}: (head, token) replace (row, plane)
        const int qy = MODE == 2 ? h : t * kBwdT;
        const int qz = MODE == 2 ? static_cast<int>(a) + t * kBwdT : b * p.H + h;
#pragma unroll
        for (int pn = 0; pn < L::PANELS; ++pn) {
          tma_load_3d(sQ + pn * (kBwdT * 128), &tm_q, BAR_QF, pn * 64, qy, qz);
          tma_load_3d(sDO + pn * (kBwdT * 128), &tm_do, BAR_QF, pn * 64, qy, qz);
        }
        ++q_iter;
        for (int j = 0; j < tl.n; ++j) {
          const int kt = tl.kt(j);
          const int ky = MODE == 2 ? h / p.G : kt * kBwdT;
          const int kz = MODE == 2 ? static_cast<int>(a) + kt * kBwdT : b * p.Hkv + h / p.G;
          const int st = kv_iter % NS;
          if (kv_iter >= NS && !mbar_wait(BAR_KE + 8 * st, ((kv_iter / NS) - 1) & 1, abort_flag))
            break;
          mbar_expect_tx(BAR_KF + 8 * st, L::TILE);
#pragma unroll
          for (int pn = 0; pn < L::PANELS; ++pn)
            tma_load_3d(sK + st * L::TILE + pn * (kBwdT * 128), &tm_k, BAR_KF + 8 * st, pn * 64,
                        ky, kz);
          if (kv_iter >= NS &&
              !mbar_wait(BAR_VE + 8 * st, ((kv_iter / NS) - 1) & 1, abort_flag)) {
            k_ahead = true;
            break;
          }
          mbar_expect_tx(BAR_VF + 8 * st, L::TILE);
#pragma unroll
          for (int pn = 0; pn < L::PANELS; ++pn)
            tma_load_3d(sV + st * L::TILE + pn * (kBwdT * 128), &tm_v, BAR_VF + 8 * st, pn * 64,
                        ky, kz);
          ++kv_iter;
        }
        if (*abort_flag) break;
      }
      // every copy issued must land before the CTA ends
      if (q_iter > 0) mbar_drain(BAR_QF, (q_iter - 1) & 1);
      const int k_issued = kv_iter + (k_ahead ? 1 : 0);
      for (int i = max(0, k_issued - NS); i < k_issued; ++i)
        mbar_drain(BAR_KF + 8 * (i % NS), (i / NS) & 1);
      for (int i = max(0, kv_iter - NS); i < kv_iter; ++i)
        mbar_drain(BAR_VF + 8 * (i % NS), (i / NS) & 1);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBwdT, kBwdT, false);
      constexpr uint32_t idQ = idesc_bf16_f32(kBwdT, D, true);
      int q_iter = 0, kv_iter = 0;
      uint32_t el_cnt = 0;
      // S or dP = A (128 x D, K-major) * B (128 x D, K-major)^T
      auto issue_nt = [&](uint32_t dst, uint32_t a, uint32_t b_) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBwdT * 128) + (kk & 3) * 32;
          mma_ss(tmem + dst, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b_ + off, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
      };
      for (int it = 0, u = unit_of(0); u < p.n_units; u = unit_of(++it)) {
        int b, h, t, len;
        int64_t a;
        if (unit(u, b, h, t, a, len)) continue;
        const int n = dq_tiles<SINK>(p, t).n;
        if (!mbar_wait(BAR_QF, q_iter & 1, abort_flag)) break;
        tc_fence_after();
        const int kv0 = kv_iter;
        // S(0), dP(0), S(1)
        {
          const int st = kv0 % NS;
          if (!mbar_wait(BAR_KF + 8 * st, (kv0 / NS) & 1, abort_flag)) break;
          tc_fence_after();
          issue_nt(T_S, sQ, sK + st * L::TILE);
          tc_commit(BAR_SF);
          if (!mbar_wait(BAR_VF + 8 * st, (kv0 / NS) & 1, abort_flag)) break;
          tc_fence_after();
          issue_nt(T_DP, sDO, sV + st * L::TILE);
          tc_commit(BAR_DPF);
          tc_commit(BAR_VE + 8 * st);
          if (n > 1) {
            const int st1 = (kv0 + 1) % NS;
            if (!mbar_wait(BAR_KF + 8 * st1, ((kv0 + 1) / NS) & 1, abort_flag)) break;
            tc_fence_after();
            issue_nt(T_S + 128, sQ, sK + st1 * L::TILE);
            tc_commit(BAR_SF + 8);
          }
        }
        // the previous unit's dQ must be read out before this unit's first dQ MMA
        if (q_iter > 0 && !mbar_wait(BAR_DQE, (q_iter - 1) & 1, abort_flag)) break;
        // per tile j: dS(j) stored -> dQ(j), dP(j+1), S(j+2).  The element-wise warps
        // compute P(j+1) from S(j+1) (issued a tile earlier) while dQ(j) and dP(j+1)
        // run.  Each barrier's next phase depends on this thread having passed the
        // previous one (EL(j+1) needs dP(j+1), issued after the wait for EL(j)).
        for (int j = 0; j < n; ++j) {
          const int kj = kv0 + j;
          if (!mbar_wait(BAR_EL, el_cnt & 1, abort_flag)) break;
          ++el_cnt;
          tc_fence_after();
          // dQ += dS(j) K(j): dS in the low 64 columns of S buffer j % 2 (bf16 pairs)
          const uint32_t aS = tmem + T_S + (j & 1) * 128;
          const uint32_t kst = sK + (kj % NS) * L::TILE;
#pragma unroll
          for (int kk = 0; kk < kBwdT / 16; ++kk)
            mma_ts(tmem + T_DQ, aS + kk * 8, sdesc_sw128(kst + kk * 16 * 128, kBwdT * 128, 1024),
                   idQ, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(BAR_KE + 8 * (kj % NS));
          if (j + 1 < n) {
            const int st = (kj + 1) % NS;
            if (!mbar_wait(BAR_VF + 8 * st, ((kj + 1) / NS) & 1, abort_flag)) break;
            tc_fence_after();
            issue_nt(T_DP, sDO, sV + st * L::TILE);
            tc_commit(BAR_DPF);
            tc_commit(BAR_VE + 8 * st);
          }
          if (j + 2 < n) {
            const int st = (kj + 2) % NS;
            if (!mbar_wait(BAR_KF + 8 * st, ((kj + 2) / NS) & 1, abort_flag)) break;
            tc_fence_after();
            issue_nt(T_S + (j & 1) * 128, sQ, sK + st * L::TILE);
            tc_commit(BAR_SF + 8 * (j & 1));
          }
        }
        if (*abort_flag) break;
        kv_iter += n;
        tc_commit(BAR_QE);
        tc_commit(BAR_DQF);
        ++q_iter;
      }
      // every MMA issued must complete before the tensor memory is freed
      tc_commit(BAR_DRAIN);
      mbar_drain(BAR_DRAIN, 0);
    }
  } else {
    // --------------------------------------------------------------- element-wise
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t s_cnt[2] = {0u, 0u}, dp_cnt = 0, u_iter = 0;
    bool stop = false;  // a wait gave up (the whole warp): no more TMEM work or stores
    for (int it = 0, u = unit_of(0); u < p.n_units; u = unit_of(++it)) {
      int b, h, t, len;
      int64_t a;
      if (unit(u, b, h, t, a, len)) continue;
      const DqTiles tl = dq_tiles<SINK>(p, t);
      const int n = tl.n;
      const int qrow = t * kBwdT + row;
      const bool valid = qrow < len;
      // D_i = <dout_i, out_i> (fp32), also written for the dK/dV kernel
      float Di = 0.f, lse2 = INFINITY;
      if (valid) {
        const int64_t r = bwd_row<MODE>(p, b, a, p.H, h, qrow);
        const uint4 *po = reinterpret_cast<const uint4 *>(p.out + r * D);
        const uint4 *pg = reinterpret_cast<const uint4 *>(p.dout + r * D);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 a = po[c], g = pg[c];
          const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 af = make_float2(__uint_as_float(aw[i] << 16),
                                          __uint_as_float(aw[i] & 0xFFFF0000u));
            const float2 gf = make_float2(__uint_as_float(gw[i] << 16),
                                          __uint_as_float(gw[i] & 0xFFFF0000u));
            acc = __ffma2_rn(af, gf, acc);
          }
        }
        Di = acc.x + acc.y;
        const int64_t rv = bwd_vec<MODE>(p, b, a, h, qrow);
        p.delta[rv] = Di;
        lse2 = p.lse[rv] * 1.4426950408889634f;
      }
      for (int j = 0; j < n; ++j) {
        const int kt = tl.kt(j);
        const int x = j & 1;
        if (!mbar_wait_warp(BAR_SF + 8 * x, s_cnt[x] & 1, abort_flag)) {
          stop = true;
          break;
        }
        ++s_cnt[x];
        tc_fence_after();
        // allowed key columns of this row: positions in [qrow - W + 1, qrow] and
        // < len, and with sinks the positions below n_sink (up to the row)
        const int c0 = kt * kBwdT;
        const bool full = c0 + kBwdT - 1 <= t * kBwdT && c0 >= t * kBwdT + kBwdT - p.W &&
                          t * kBwdT + kBwdT <= len;
        uint32_t mw[4];
        col_mask(qrow - p.W + 1 - c0, min(qrow, len - 1) - c0, mw);
        if (SINK && c0 == 0) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            mw[w] |= range_bits(-32 * w, min(p.n_sink - 1, min(qrow, len - 1)) - 32 * w);
        }
        const uint32_t tS = tmem + T_S + x * 128 + lane_off;
        const uint32_t tP = tmem + T_DP + lane_off;
        // phase 1 (needs only S): P in fp32
        float pf[kBwdT];
        auto pchunk = [&](int ch, const uint32_t (&sr)[32]) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float pr = ex2(fmaf(__uint_as_float(sr[c]), p.scale_log2, -lse2));
            if (!full && !((mw[ch] >> c) & 1u)) pr = 0.f;
            pf[ch * 32 + c] = pr;
          }
        };
        {
          uint32_t r0[32], r1[32];
          tmem_ld32_issue(tS, r0);
          tmem_ld32_issue(tS + 32, r1);
          tmem_ld_wait2(r0, r1);
          pchunk(0, r0);
          tmem_ld32_issue(tS + 64, r0);
          pchunk(1, r1);
          tmem_ld32_issue(tS + 96, r1);
          tmem_ld_wait2(r0, r1);
          pchunk(2, r0);
          pchunk(3, r1);
        }
        // phase 2: dS = P o (dP - D) as bf16 over the low half of this S buffer;
        // dP is released as soon as it is read
        if (!mbar_wait_warp(BAR_DPF, dp_cnt & 1, abort_flag)) {
          stop = true;
          break;
        }
        ++dp_cnt;
        tc_fence_after();
        auto dchunk = [&](int ch, const uint32_t (&dr)[32]) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16(pf[ch * 32 + 2 * i] * (__uint_as_float(dr[2 * i]) - Di),
                              pf[ch * 32 + 2 * i + 1] * (__uint_as_float(dr[2 * i + 1]) - Di));
          tmem_st16_b(tS + ch * 16, pk);
        };
        {
          uint32_t r0[32], r1[32];
          tmem_ld32_issue(tP, r0);
          tmem_ld32_issue(tP + 32, r1);
          tmem_ld_wait2(r0, r1);
          dchunk(0, r0);
          tmem_ld32_issue(tP + 64, r0);
          dchunk(1, r1);
          tmem_ld32_issue(tP + 96, r1);
          tmem_ld_wait2(r0, r1);
          dchunk(2, r0);
          dchunk(3, r1);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(BAR_EL);
      }
      if (stop || __any_sync(0xffffffffu, *abort_flag)) break;
      if (!mbar_wait_warp(BAR_DQF, u_iter & 1, abort_flag)) break;
      ++u_iter;
      tc_fence_after();
      {
        // rows of this lane's 8-lane group: whole 128-byte segments per store
        const int g_row = t * kBwdT + quad * 32 + (lane & ~7);
        store_tile_rows<D>(p.dq + bwd_row<MODE>(p, b, a, p.H, h, g_row) * D,
                           MODE == 2 ? static_cast<int64_t>(p.H) * D : D, len - g_row,
                           tmem + T_DQ + lane_off, p.scale, lane);
      }
      tc_fence_before();
      mbar_arrive(BAR_DQE);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -------------------------------------------------------------------------------- dK dV
// Unit u: (b, kv head, key tile kt); steps over (query head g of the group, live
// query tile t in [kt, t_hi]).
template <int D, int MODE, bool SINK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw);
  const uint32_t sK = base + L::OFF_A0, sV = base + L::OFF_A1;
  const uint32_t sQ = base + L::OFF_S0, sDO = base + L::OFF_S1;
  float *vec = reinterpret_cast<float *>(gbase + L::OFF_VEC);  // [2][2][128]: lse2, D
  const uint32_t bar = base + L::OFF_BAR;
  const uint32_t BAR_KVF = bar, BAR_KVE = bar + 8;
  const uint32_t BAR_SF = bar + 16;
  const uint32_t BAR_DPF = bar + 24;
  const uint32_t BAR_PF = bar + 32;        // P^T of the step stored (128 arrivals)
  const uint32_t BAR_AF = bar + 40;        // dK, dV final
  const uint32_t BAR_AE = bar + 48;        // dK, dV read out (128 arrivals)
  const uint32_t BAR_VEC = bar + 56;       // a step's lse2 / D columns staged (128 arrivals)
  const uint32_t BAR_DSF = bar + 64;       // dS^T of the step stored (128 arrivals)
  const uint32_t BAR_DRAIN = bar + 72;     // the MMA thread's teardown
  const uint32_t BAR_QF = bar + 128;       // + 8 * stage
  const uint32_t BAR_QE = BAR_QF + 8 * NS;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + L::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR_KVF, 1);
    mbar_init(BAR_KVE, 1);
    mbar_init(BAR_SF, 1);
    mbar_init(BAR_DPF, 1);
    mbar_init(BAR_PF, 4 * 32);
    mbar_init(BAR_AF, 1);
    mbar_init(BAR_AE, 4 * 32);
    mbar_init(BAR_VEC, 4 * 32);
    mbar_init(BAR_DSF, 4 * 32);
    mbar_init(BAR_DRAIN, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(BAR_QF + 8 * s, 1);
      mbar_init(BAR_QE + 8 * s, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // tensor memory: S^T [0, 128), dP^T [128, 256), dV [256, 256 + D), dK [256 + D, 256 + 2D)
  const uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;

  // unit -> (b, kv head, kt) and its sequence; query tiles [kt, t_hi] of each
  // of the G heads (all of the sequence's for the key tile of the sinks).
  // 0: run it, 1: bad sequence offsets (skip, flag), 2: the key tile lies past
  // the sequence's end (skip).  Key tile 0 of every (b, kv head) first, then
  // key tile 1, and so on: the heaviest units first (with sinks, key tile 0
  // is read by every query tile of its sequence).  On the packed layout the
  // units run sequence by sequence and, within one, KV head by KV head, so
  // the query tiles that the units in flight read stay in L2.
  auto unit = [&](int u, int &b, int &kvh, int &kt, int &t_hi, int64_t &a, int &len) -> int {
    if (MODE == 2) {
      const int per_b = p.Hkv * p.nt, r = u % per_b;
      b = u / per_b;
      kvh = r / p.nt;
      kt = r % p.nt;
    } else {
      const int per_t = p.B * p.Hkv;
      kt = u / per_t;
      const int bk = u % per_t;
      b = bk / p.Hkv;
      kvh = bk % p.Hkv;
    }
    if (bwd_seq<MODE>(p, b, a, len)) return 1;
    if (kt * kBwdT >= len) return 2;
    const int nt_s = (len + kBwdT - 1) / kBwdT;
    t_hi = (SINK && p.n_sink > 0 && kt == 0)
               ? nt_s - 1
               : min(nt_s - 1, (kt * kBwdT + kBwdT - 1 + p.W - 1) / kBwdT);
    return 0;
  };
  auto unit_of = [&](int i) -> int {
    const int P = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return i * P + ((i & 1) ? P - 1 - c : c);
  };

  if (warp == 0) {
    // --------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int u_iter = 0, q_iter = 0;
      for (int it = 0, u = unit_of(0); u < p.n_units; u = unit_of(++it)) {
        int b, kvh, kt, t_hi, len;
        int64_t a;
        const int ust = unit(u, b, kvh, kt, t_hi, a, len);
        if (ust) {
          if (ust == 1) atomicOr(&g_swa_status, SWA_DEV_BADARG);
          continue;
        }
        if (u_iter > 0 && !mbar_wait(BAR_KVE, (u_iter - 1) & 1, abort_flag)) break;
        mbar_expect_tx(BAR_KVF, 2 * L::TILE);
        // MODE 2 maps are {D, heads, tokens}: (head, token) replace (row, plane)
        const int ky = MODE == 2 ? kvh : kt * kBwdT;
        const int kz = MODE == 2 ? static_cast<int>(a) + kt * kBwdT : b * p.Hkv + kvh;
#pragma unroll
        for (int pn = 0; pn < L::PANELS; ++pn) {
          tma_load_3d(sK + pn * (kBwdT * 128), &tm_k, BAR_KVF, pn * 64, ky, kz);
          tma_load_3d(sV + pn * (kBwdT * 128), &tm_v, BAR_KVF, pn * 64, ky, kz);
        }
        ++u_iter;
        for (int g = 0; g < p.G; ++g) {
          const int hq = kvh * p.G + g;
          for (int t = kt; t <= t_hi; ++t) {
            const int qy = MODE == 2 ? hq : t * kBwdT;
            const int qz = MODE == 2 ? static_cast<int>(a) + t * kBwdT : b * p.H + hq;
            const int st = q_iter % NS;
            if (q_iter >= NS && !mbar_wait(BAR_QE + 8 * st, ((q_iter / NS) - 1) & 1, abort_flag))
              break;
            mbar_expect_tx(BAR_QF + 8 * st, 2 * L::TILE);
#pragma unroll
            for (int pn = 0; pn < L::PANELS; ++pn) {
              tma_load_3d(sQ + st * L::TILE + pn * (kBwdT * 128), &tm_q, BAR_QF + 8 * st, pn * 64,
                          qy, qz);
              tma_load_3d(sDO + st * L::TILE + pn * (kBwdT * 128), &tm_do, BAR_QF + 8 * st,
                          pn * 64, qy, qz);
            }
            ++q_iter;
          }
          if (*abort_flag) break;
        }
        if (*abort_flag) break;
      }
      // every copy issued must land before the CTA ends
      if (u_iter > 0) mbar_drain(BAR_KVF, (u_iter - 1) & 1);
      for (int i = max(0, q_iter - NS); i < q_iter; ++i)
        mbar_drain(BAR_QF + 8 * (i % NS), (i / NS) & 1);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBwdT, kBwdT, false);
      constexpr uint32_t idA = idesc_bf16_f32(kBwdT, D, true);
      int u_iter = 0, q_iter = 0;
      uint32_t el_cnt = 0;
      auto issue_nt = [&](uint32_t dst, uint32_t a, uint32_t b_) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBwdT * 128) + (kk & 3) * 32;
          mma_ss(tmem + dst, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b_ + off, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
      };
      // dst (+)= A[tmem, 128 x 128 bf16] * B[128 queries x D, MN-major]
      auto issue_tn = [&](uint32_t dst, uint32_t a_cols, uint32_t b_, bool acc) {
#pragma unroll
        for (int kk = 0; kk < kBwdT / 16; ++kk)
          mma_ts(tmem + dst, tmem + a_cols + kk * 8,
                 sdesc_sw128(b_ + kk * 16 * 128, kBwdT * 128, 1024), idA,
                 (acc || kk > 0) ? 1u : 0u);
      };
      for (int it = 0, u = unit_of(0); u < p.n_units; u = unit_of(++it)) {
        int b, kvh, kt, t_hi, len;
        int64_t a;
        if (unit(u, b, kvh, kt, t_hi, a, len)) continue;
        const int n = p.G * (t_hi - kt + 1);
        if (!mbar_wait(BAR_KVF, u_iter & 1, abort_flag)) break;
        tc_fence_after();
        const int q0 = q_iter;
        {
          const int st = q0 % NS;
          if (!mbar_wait(BAR_QF + 8 * st, (q0 / NS) & 1, abort_flag)) break;
          tc_fence_after();
          issue_nt(T_S, sK, sQ + st * L::TILE);
          tc_commit(BAR_SF);
          issue_nt(T_DP, sV, sDO + st * L::TILE);
          tc_commit(BAR_DPF);
        }
        // the previous unit's dK, dV must be read out before this unit's first dV, dK MMAs
        if (u_iter > 0 && !mbar_wait(BAR_AE, (u_iter - 1) & 1, abort_flag)) break;
        // per step: P^T(s) stored -> dV(s), S^T(s+1); dS^T(s) stored -> dK(s), dP^T(s+1).
        // S^T(s+1) overwrites P^T(s) and dP^T(s+1) overwrites dS^T(s), each issued
        // behind the MMA that reads it; the element-wise warps compute P^T(s+1)
        // while dK(s) and dP^T(s+1) run.
        for (int s = 0; s < n; ++s) {
          const int qs = q0 + s;
          const int st = qs % NS;
          const int st1 = (qs + 1) % NS;
          if (!mbar_wait(BAR_PF, el_cnt & 1, abort_flag)) break;
          tc_fence_after();
          issue_tn(T_DV, T_S, sDO + st * L::TILE, s > 0);   // dV += P^T dO
          if (s + 1 < n) {
            if (!mbar_wait(BAR_QF + 8 * st1, ((qs + 1) / NS) & 1, abort_flag)) break;
            tc_fence_after();
            issue_nt(T_S, sK, sQ + st1 * L::TILE);
            tc_commit(BAR_SF);
          }
          if (!mbar_wait(BAR_DSF, el_cnt & 1, abort_flag)) break;
          ++el_cnt;
          tc_fence_after();
          issue_tn(T_DK, T_DP, sQ + st * L::TILE, s > 0);   // dK += dS^T Q
          tc_commit(BAR_QE + 8 * st);
          if (s + 1 < n) {
            issue_nt(T_DP, sV, sDO + st1 * L::TILE);
            tc_commit(BAR_DPF);
          }
        }
        if (*abort_flag) break;
        q_iter += n;
        tc_commit(BAR_KVE);
        tc_commit(BAR_AF);
        ++u_iter;
      }
      // every MMA issued must complete before the tensor memory is freed
      tc_commit(BAR_DRAIN);
      mbar_drain(BAR_DRAIN, 0);
    }
  } else {
    // --------------------------------------------------------------- element-wise
    const int quad = warp & 3;
    const int row = quad * 32 + lane;   // key row of the tile
    const int et = threadIdx.x - 64;    // 0..127: column this thread stages
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t s_cnt = 0, u_iter = 0, step = 0;
    for (int it = 0, u = unit_of(0); u < p.n_units; u = unit_of(++it)) {
      int b, kvh, kt, t_hi, len;
      int64_t a;
      if (unit(u, b, kvh, kt, t_hi, a, len)) continue;
      const int krow = kt * kBwdT + row;
      const int nqt = t_hi - kt + 1, n = p.G * nqt;
      // query columns this key row reaches: [krow, krow + W - 1] (a sink row:
      // every later one) within the sequence; none for rows past its end
      const int qhi = (SINK && krow < p.n_sink) ? len - 1 : min(krow + p.W - 1, len - 1);
      // lse2 and D of query column et of step s: (query head g, query tile t)
      auto col_vals = [&](int s, float &l2, float &dd) {
        const int g = s / nqt, t = kt + s % nqt;
        const int qc = t * kBwdT + et;
        const int64_t rv = bwd_vec<MODE>(p, b, a, kvh * p.G + g, qc);
        l2 = qc < len ? p.lse[rv] * 1.4426950408889634f : INFINITY;
        dd = qc < len ? p.delta[rv] : 0.f;
      };
      // stage a step's 128 (lse2, D) column values (two copies alternate).  Step
      // s + 1 is staged at the end of step s, after this thread's last read of
      // the copy it overwrites; passing step s's barrier needs every thread's
      // staging of step s, which each did after finishing step s - 1.
      auto stage = [&](uint32_t st, float l2, float dd) {
        float *v2 = vec + (st & 1) * 2 * kBwdT;
        v2[et] = l2;
        v2[kBwdT + et] = dd;
        mbar_arrive(BAR_VEC);
      };
      float l2n, ddn;
      col_vals(0, l2n, ddn);
      stage(step, l2n, ddn);
      bool stop = false;
      for (int s = 0; s < n; ++s, ++step) {
        const int t = kt + s % nqt;
        if (s + 1 < n) col_vals(s + 1, l2n, ddn);  // loads in flight during this step
        const float *v2 = vec + (step & 1) * 2 * kBwdT;
        if (!mbar_wait_warp(BAR_VEC, step & 1, abort_flag) ||
            !mbar_wait_warp(BAR_SF, s_cnt & 1, abort_flag)) {
          stop = true;
          break;
        }
        tc_fence_after();
        // allowed query columns of key row krow (see qhi above)
        const int c0 = t * kBwdT;
        const bool full = kt * kBwdT + kBwdT - 1 <= c0 && c0 + kBwdT - 1 - kt * kBwdT <= p.W - 1 &&
                          c0 + kBwdT <= len;
        uint32_t mw[4];
        col_mask(krow - c0, qhi - c0, mw);
        const uint32_t tS = tmem + T_S + lane_off;
        const uint32_t tP = tmem + T_DP + lane_off;
        // phase 1: P^T, stored as bf16 over the low half of S^T and kept for dS:
        // in fp32 on the [B, heads, N, d] layout; on the packed layout, whose
        // wider addressing leaves no room for a 128-register row, as the bf16
        // pairs just stored (the same rounded P that dV uses)
        constexpr bool kPackedP = MODE == 2;
        float pf[kPackedP ? 1 : kBwdT];
        uint32_t pw[kPackedP ? kBwdT / 2 : 1];
        auto pchunk = [&](int ch, const uint32_t (&sr)[32]) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float pr[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 2 * i + e;
              pr[e] = ex2(fmaf(__uint_as_float(sr[c]), p.scale_log2, -v2[ch * 32 + c]));
              if (!full && !((mw[ch] >> c) & 1u)) pr[e] = 0.f;
              if (!kPackedP) pf[ch * 32 + c] = pr[e];
            }
            pk[i] = pack_bf16(pr[0], pr[1]);
            if (kPackedP) pw[ch * 16 + i] = pk[i];
          }
          tmem_st16_b(tS + ch * 16, pk);
        };
        {
          uint32_t r0[32], r1[32];
          tmem_ld32_issue(tS, r0);
          tmem_ld32_issue(tS + 32, r1);
          tmem_ld_wait2(r0, r1);
          pchunk(0, r0);
          tmem_ld32_issue(tS + 64, r0);
          pchunk(1, r1);
          tmem_ld32_issue(tS + 96, r1);
          tmem_ld_wait2(r0, r1);
          pchunk(2, r0);
          pchunk(3, r1);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(BAR_PF);
        // phase 2: dS^T = P^T o (dP^T - D), stored as bf16 over the low half of dP^T
        if (!mbar_wait_warp(BAR_DPF, s_cnt & 1, abort_flag)) {
          stop = true;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        auto dchunk = [&](int ch, const uint32_t (&dr)[32]) {
          uint32_t dk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float dd[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 2 * i + e;
              float pe;
              if (kPackedP) {
                const uint32_t w = pw[ch * 16 + i];
                pe = __uint_as_float(e ? (w & 0xFFFF0000u) : (w << 16));
              } else {
                pe = pf[ch * 32 + c];
              }
              dd[e] = pe * (__uint_as_float(dr[c]) - v2[kBwdT + ch * 32 + c]);
            }
            dk[i] = pack_bf16(dd[0], dd[1]);
          }
          tmem_st16_b(tP + ch * 16, dk);
        };
        {
          uint32_t r0[32], r1[32];
          tmem_ld32_issue(tP, r0);
          tmem_ld32_issue(tP + 32, r1);
          tmem_ld_wait2(r0, r1);
          dchunk(0, r0);
          tmem_ld32_issue(tP + 64, r0);
          dchunk(1, r1);
          tmem_ld32_issue(tP + 96, r1);
          tmem_ld_wait2(r0, r1);
          dchunk(2, r0);
          dchunk(3, r1);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(BAR_DSF);
        if (s + 1 < n) stage(step + 1, l2n, ddn);
      }
      if (stop || __any_sync(0xffffffffu, *abort_flag)) break;
      if (!mbar_wait_warp(BAR_AF, u_iter & 1, abort_flag)) break;
      ++u_iter;
      tc_fence_after();
      // rows of this lane's 8-lane group: whole 128-byte segments per store
      const int g_row = kt * kBwdT + quad * 32 + (lane & ~7);
      const int64_t g_off = bwd_row<MODE>(p, b, a, p.Hkv, kvh, g_row) * D;
      const int64_t g_stride = MODE == 2 ? static_cast<int64_t>(p.Hkv) * D : D;
      store_tile_rows<D>(p.dv + g_off, g_stride, len - g_row, tmem + T_DV + lane_off, 1.f, lane);
      store_tile_rows<D>(p.dk + g_off, g_stride, len - g_row, tmem + T_DK + lane_off, p.scale,
                         lane);
      tc_fence_before();
      mbar_arrive(BAR_AE);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace swa
