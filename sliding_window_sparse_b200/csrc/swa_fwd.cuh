// swa_fwd.cuh -- tile-skipping sliding-window attention forward on sm_100a.
//
// One CTA computes one 128-row query tile of one (sequence, query head):
//   * only key tiles that hold an allowed pair are visited (M003 note
//     section 04: invisible tiles are skipped, never loaded);
//   * warp 0 stages Q once and K/V tiles into a 2-deep shared-memory ring by
//     TMA (128-byte swizzle, one box per 64 head-dim columns);
//   * one thread of warp 1 issues the 5th-generation tensor-core MMAs:
//     S = Q K^T into one of two tensor-memory buffers, then O += P V into a
//     tensor-memory accumulator;
//   * warps 2-5 (one tensor-memory lane quadrant each, one query row per
//     thread) run the online softmax in fp32: mask only partially visible or
//     ragged tiles, exponentiate in base 2 with scale * log2(e) folded in,
//     keep the running max and sum, write P as bf16 into shared memory in
//     the swizzled K-major layout the MMA reads, and rescale O in tensor
//     memory only when the running max grows by more than 2^8 (the stale max
//     is exact because O and the sum use the same one);
//   * the same warps normalise O and store bf16 rows (and the log-sum-exp).
//
// MODE 0: linear keys (prefill, query row i at position i).
// MODE 1: ring + chunk keys (chunked prefill, Chapter 10 section 10.2): the
//         ring tiles in physical slot order, then the chunk tiles; positions
//         are relative to the chunk start q_start[b].
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "swa_tile.cuh"

namespace swa {

constexpr int kBQ = 128;  // query rows per tile (MMA M, tensor-memory lanes)
constexpr int kBK = 128;  // keys per tile (MMA N of S, MMA K of P V)
constexpr int kFwdThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest unscaled P factor

struct FwdParams {
  __nv_bfloat16 *out;      // [B, H, n_q, D]
  float *lse;              // [B, H, n_q] or nullptr
  const int64_t *q_start;  // MODE 1: [B]
  int B, H, Hkv, G;
  int n_q;                 // query rows per (b, h)
  int n_k;                 // rows of the main key source (N or Tq)
  int64_t W;               // window; MODE 0 clamps it to n_k + kBQ
  float scale_log2;        // scale * log2(e)
  int nqt;                 // query tiles per (b, h)
  int n_ring_tiles;        // MODE 1
};

template <int D>
struct FwdLayout {
  static constexpr int PANELS = D / 64;  // 128-byte swizzle atoms along the head dim
  static constexpr int NST = 2;          // K/V stages
  static constexpr uint32_t Q_BYTES = kBQ * D * 2;
  static constexpr uint32_t KV_BYTES = kBK * D * 2;
  static constexpr uint32_t P_BYTES = kBQ * kBK * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NST * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + NST * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
  // q_full, k_full[NST], v_full[NST], kv_empty[NST], s_full[2], p_full, o_done
  static constexpr int NBAR = 1 + 3 * NST + 2 + 2;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
  static constexpr uint32_t BYTES = OFF_MISC + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;  // slack to align the base to 1 KB
  static constexpr uint32_t TMEM_COLS = 512;       // S0 [0,128) S1 [128,256) O [256,256+D)
};

// Walks the live key tiles of one query tile in a fixed order; every role
// of the CTA runs an identical walker, so they agree on the tile sequence.
template <int MODE>
struct TileWalker {
  int kt, kt_end;
  int64_t q_lo, q_hi, W, n_k, n_q, q_start;

  __device__ __forceinline__ bool next(KeyTile &t, int &cls) {
    while (kt < kt_end) {
      const int cur = kt++;
      if (MODE == 0)
        t = linear_tile(cur, kBK, n_k);
      else
        t = ring_chunk_tile(cur, kBK, W, n_q, q_start, q_start);
      cls = tile_class(t, q_lo, q_hi, W);
      if (cls) return true;
    }
    return false;
  }
};

template <int D, int MODE>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kr,
               const __grid_constant__ CUtensorMap tm_vr, const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr int NST = L::NST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + L::OFF_Q, sK = base + L::OFF_K, sV = base + L::OFF_V,
                 sP = base + L::OFF_P, bar = base + L::OFF_BAR;
  const uint32_t BAR_Q = bar;
  const uint32_t BAR_KF = bar + 8;                 // + 8 * stage
  const uint32_t BAR_VF = bar + 8 * (1 + NST);     // + 8 * stage
  const uint32_t BAR_KVE = bar + 8 * (1 + 2 * NST);  // + 8 * stage
  const uint32_t BAR_S = bar + 8 * (1 + 3 * NST);  // + 8 * buffer
  const uint32_t BAR_P = bar + 8 * (3 + 3 * NST);
  const uint32_t BAR_O = bar + 8 * (4 + 3 * NST);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + L::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: heavy query tiles first; heads of one kv group adjacent
  const int nbh = p.B * p.H;
  const int bh = blockIdx.x % nbh;
  const int qt = p.nqt - 1 - static_cast<int>(blockIdx.x / nbh);
  const int b = bh / p.H, h = bh % p.H;
  const int kvh = h / p.G;
  const int r_begin = qt * kBQ;
  const int r_last = (r_begin + kBQ < p.n_q ? r_begin + kBQ : p.n_q) - 1;

  TileWalker<MODE> walker;
  walker.q_lo = r_begin;
  walker.q_hi = r_last;
  walker.W = p.W;
  walker.n_k = p.n_k;
  walker.n_q = p.n_q;
  walker.q_start = 0;
  bool bad = false;
  if (MODE == 0) {
    const int64_t lo = r_begin - (p.W - 1) > 0 ? r_begin - (p.W - 1) : 0;
    walker.kt = static_cast<int>(lo / kBK);
    walker.kt_end = r_last / kBK + 1;
  } else {
    walker.q_start = p.q_start[b];
    bad = walker.q_start < 0;
    walker.kt = 0;
    walker.kt_end = bad ? 0 : p.n_ring_tiles + (p.n_q + kBK - 1) / kBK;
  }

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(BAR_KF + 8 * s, 1);
      mbar_init(BAR_VF + 8 * s, 1);
      mbar_init(BAR_KVE + 8 * s, 1);
    }
    mbar_init(BAR_S, 1);
    mbar_init(BAR_S + 8, 1);
    mbar_init(BAR_P, 4 * 32);
    mbar_init(BAR_O, 1);
    *abort_flag = 0;
    if (bad) atomicOr(&g_swa_status, SWA_DEV_BADARG);
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !bad) {
      mbar_expect_tx(BAR_Q, L::Q_BYTES);
#pragma unroll
      for (int pn = 0; pn < L::PANELS; ++pn)
        tma_load_3d(sQ + pn * (kBQ * 128), &tm_q, BAR_Q, pn * 64, r_begin, b * p.H + h);
      KeyTile t;
      int cls;
      int j = 0;
      const int z = b * p.Hkv + kvh;
      while (walker.next(t, cls)) {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(BAR_KVE + 8 * st, ((j / NST) - 1) & 1, abort_flag)) break;
        const CUtensorMap *mk = t.src == 1 ? &tm_kr : &tm_k;
        const CUtensorMap *mv = t.src == 1 ? &tm_vr : &tm_v;
        mbar_expect_tx(BAR_KF + 8 * st, L::KV_BYTES);
#pragma unroll
        for (int pn = 0; pn < L::PANELS; ++pn)
          tma_load_3d(sK + st * L::KV_BYTES + pn * (kBK * 128), mk, BAR_KF + 8 * st, pn * 64,
                      t.y0, z);
        mbar_expect_tx(BAR_VF + 8 * st, L::KV_BYTES);
#pragma unroll
        for (int pn = 0; pn < L::PANELS; ++pn)
          tma_load_3d(sV + st * L::KV_BYTES + pn * (kBK * 128), mv, BAR_VF + 8 * st, pn * 64,
                      t.y0, z);
        ++j;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && !bad) {
      constexpr uint32_t idS = idesc_bf16_f32(kBQ, kBK, false);
      constexpr uint32_t idO = idesc_bf16_f32(kBQ, D, true);
      mbar_wait(BAR_Q, 0, abort_flag);
      auto issue_s = [&](int jj) {
        const int st = jj % NST;
        mbar_wait(BAR_KF + 8 * st, (jj / NST) & 1, abort_flag);
        tc_fence_after();
        const uint32_t dS = tmem + (jj & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBQ * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kBK * 128) + (kk & 3) * 32;
          mma_ss(dS, sdesc_sw128(sQ + off, 16, 1024),
                 sdesc_sw128(sK + st * L::KV_BYTES + offk, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(BAR_S + 8 * (jj & 1));
      };
      KeyTile t;
      int cls;
      bool have = walker.next(t, cls);
      int j = 0;
      if (have) issue_s(0);
      while (have) {
        KeyTile tn;
        int clsn;
        const bool has_next = walker.next(tn, clsn);
        if (has_next) issue_s(j + 1);
        const int st = j % NST;
        mbar_wait(BAR_P, j & 1, abort_flag);
        mbar_wait(BAR_VF + 8 * st, (j / NST) & 1, abort_flag);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint32_t offp = (kk >> 2) * (kBQ * 128) + (kk & 3) * 32;
          mma_ss(tO, sdesc_sw128(sP + offp, 16, 1024),
                 sdesc_sw128(sV + st * L::KV_BYTES + kk * 16 * 128, kBK * 128, 1024), idO,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(BAR_O);
        tc_commit(BAR_KVE + 8 * st);
        have = has_next;
        ++j;
      }
    }
  } else {
    // ------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // tile row == tensor-memory lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int qrow = r_begin + row;
    const int64_t q_rel = qrow;  // MODE 0 absolute, MODE 1 relative to q_start
    float m_run = -INFINITY, l_run = 0.f;
    KeyTile t;
    int cls;
    int j = 0;
    while (walker.next(t, cls)) {
      mbar_wait(BAR_S + 8 * (j & 1), (j >> 1) & 1, abort_flag);
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(tmem + (j & 1) * 128 + lane_off, sr);
      float *s = reinterpret_cast<float *>(sr);
      if (cls == 2 || t.ncols < kBK) {
        // allowed columns of this row: c in a segment with base + c in [q-W+1, q]
        int lo[2], hi[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int64_t a = q_rel - p.W + 1 - t.seg[g].base;
          const int64_t z = q_rel - t.seg[g].base;
          lo[g] = static_cast<int>(a > t.seg[g].lo ? a : t.seg[g].lo);
          hi[g] = static_cast<int>(z < t.seg[g].hi ? z : t.seg[g].hi);
        }
#pragma unroll
        for (int c = 0; c < kBK; ++c) {
          const bool ok = (c >= lo[0] && c <= hi[0]) || (c >= lo[1] && c <= hi[1]);
          s[c] = ok ? s[c] : -INFINITY;
        }
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < kBK; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * p.scale_log2;
      const bool grow = m_tile > m_run + kRescaleThreshold;
      const float m_new = grow ? m_tile : m_run;
      const float alpha = grow ? ex2(m_run - m_new) : 1.f;
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kBK; ++c) {
        s[c] = ex2(fmaf(s[c], p.scale_log2, -m_use));
        rs += s[c];
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      // P V of the previous tile must be done: O is stable and P's buffer is free
      if (j > 0) mbar_wait(BAR_O, (j - 1) & 1, abort_flag);
      tc_fence_after();
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t o32[32];
          tmem_ld32(tO + lane_off + cb * 32, o32);
#pragma unroll
          for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * alpha);
          tmem_st32(tO + lane_off + cb * 32, o32);
        }
        tmem_st_wait();
      }
      // P as bf16, K-major with 128-byte swizzle: panel = 64 keys, row = 128 bytes,
      // 16-byte chunk c of row r stored at chunk position c ^ (r & 7)
#pragma unroll
      for (int pn = 0; pn < 2; ++pn) {
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
          const float *v = s + pn * 64 + c16 * 8;
          const uint32_t addr = sP + pn * (kBQ * 128) + row * 128 + ((c16 ^ (row & 7)) << 4);
          st_shared_v4(addr, pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                       pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(BAR_P);
      ++j;
    }
    if (j > 0) {
      mbar_wait(BAR_O, (j - 1) & 1, abort_flag);
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      __nv_bfloat16 *orow =
          p.out + (static_cast<int64_t>(b * p.H + h) * p.n_q + qrow) * static_cast<int64_t>(D);
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t o32[32];
        tmem_ld32(tO + lane_off + cb * 32, o32);
        if (qrow < p.n_q) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(o32[i + 0]) * inv_l, __uint_as_float(o32[i + 1]) * inv_l);
            v.y = pack_bf16(__uint_as_float(o32[i + 2]) * inv_l, __uint_as_float(o32[i + 3]) * inv_l);
            v.z = pack_bf16(__uint_as_float(o32[i + 4]) * inv_l, __uint_as_float(o32[i + 5]) * inv_l);
            v.w = pack_bf16(__uint_as_float(o32[i + 6]) * inv_l, __uint_as_float(o32[i + 7]) * inv_l);
            *reinterpret_cast<uint4 *>(orow + cb * 32 + i) = v;
          }
        }
      }
      if (p.lse && qrow < p.n_q)
        p.lse[static_cast<int64_t>(b * p.H + h) * p.n_q + qrow] =
            (m_run + __log2f(l_run)) * 0.6931471805599453f;
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
