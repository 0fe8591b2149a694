// swa_decode.cuh -- batched single-token decode from a W-slot ring cache.
//
// The cost of a decode step is reading the KV cache from HBM (sparse-attention
// taxonomy page, section 1), so the split kernel streams every key/value slot
// of a (sequence, kv head) exactly once, with coalesced 8-byte (d = 128) or
// 4-byte (d = 64) loads per lane, and serves all G query heads of the group
// from the same registers.  The slot range of one (b, kv head) is cut into
// `splits` CTAs; each writes an unnormalised partial (o, running max m,
// running sum l) to the workspace, and decode_combine_kernel merges them.
//
// Warp layout: lane owns DPL = d / 32 consecutive dims of q, k, v and o.
// A warp takes KEYS = 32 / G keys at a time: it forms the 32 partial dot
// products (key, head) of its lane slice, then a butterfly reduce-scatter
// over the 32 lanes leaves lane l with the full score of key l / G for head
// l % G.  Online softmax (base 2, scale * log2(e) folded into q) runs per
// head across the lanes that hold that head; the probabilities are staged in
// shared memory and every lane accumulates its o slice.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace swa {

constexpr int kDecWarps = 4;

struct DecodeParams {
  const __nv_bfloat16 *q;       // [B, H, D]
  const __nv_bfloat16 *k_ring;  // [B, Hkv, W, D]
  const __nv_bfloat16 *v_ring;  // [B, Hkv, W, D]
  const int64_t *pos;           // [B]
  float *ws_o;                  // [B*H, splits, D]
  float *ws_ml;                 // [B*H, splits, 2]  (m, l) base-2 domain
  __nv_bfloat16 *out;           // [B, H, D]
  float *lse;                   // [B, H] or nullptr
  int B, H, Hkv;
  int64_t W;
  int chunk;   // slots per split CTA
  int splits;  // CTAs per (b, kv head)
  float scale_log2;
};

template <int DPL>
struct RowVec;
template <>
struct RowVec<4> {
  using T = uint2;
};
template <>
struct RowVec<2> {
  using T = uint32_t;
};

template <int DPL>
__device__ __forceinline__ void unpack_row(const typename RowVec<DPL>::T &raw, float (&f)[DPL]);
template <>
__device__ __forceinline__ void unpack_row<4>(const uint2 &raw, float (&f)[4]) {
  f[0] = __uint_as_float(raw.x << 16);
  f[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  f[2] = __uint_as_float(raw.y << 16);
  f[3] = __uint_as_float(raw.y & 0xFFFF0000u);
}
template <>
__device__ __forceinline__ void unpack_row<2>(const uint32_t &raw, float (&f)[2]) {
  f[0] = __uint_as_float(raw << 16);
  f[1] = __uint_as_float(raw & 0xFFFF0000u);
}

template <int DPL>
__device__ __forceinline__ typename RowVec<DPL>::T load_row_nc(const __nv_bfloat16 *p) {
  using T = typename RowVec<DPL>::T;
  return __ldg(reinterpret_cast<const T *>(p));
}

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32)
    decode_split_kernel(const DecodeParams p) {
  constexpr int DPL = D / 32;
  constexpr int KEYS = 32 / G;  // keys per warp step: KEYS * G == 32 (key, head) scores
  using Raw = typename RowVec<DPL>::T;

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  __shared__ float s_p[kDecWarps][32];
  __shared__ float s_alpha[kDecWarps][G];
  __shared__ float s_m[kDecWarps][G];
  __shared__ float s_l[kDecWarps][G];
  __shared__ float s_o[kDecWarps][G][D];

  const int64_t pos = p.pos[b];
  int64_t nvalid = pos + 1 < p.W ? pos + 1 : p.W;  // slots 0..pos are filled before wrap
  if (pos < 0) {
    nvalid = 0;
    if (threadIdx.x == 0 && split == 0 && kvh == 0) atomicOr(&g_swa_status, SWA_DEV_BADARG);
  }
  const int64_t s_begin = static_cast<int64_t>(split) * p.chunk;
  int64_t s_end = s_begin + p.chunk;
  if (s_end > nvalid) s_end = nvalid;

  // q slices of the G heads of this group, pre-scaled into the base-2 domain
  float qv[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16 *qp = p.q + (static_cast<int64_t>(b) * p.H + kvh * G + g) * D + lane * DPL;
    float f[DPL];
    unpack_row<DPL>(load_row_nc<DPL>(qp), f);
#pragma unroll
    for (int i = 0; i < DPL; ++i) qv[g][i] = f[i] * p.scale_log2;
  }

  const int64_t kv_base = (static_cast<int64_t>(b) * p.Hkv + kvh) * p.W;
  const __nv_bfloat16 *kbase = p.k_ring + kv_base * D + lane * DPL;
  const __nv_bfloat16 *vbase = p.v_ring + kv_base * D + lane * DPL;

  float o[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[g][i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // for head (lane % G)

  // warp w takes steps w, w + 4, ...; a step covers KEYS consecutive slots
  const int64_t n_steps = s_end > s_begin ? (s_end - s_begin + KEYS - 1) / KEYS : 0;
  Raw kr[KEYS], vr[KEYS];
  auto load_step = [&](int64_t step, Raw (&kk)[KEYS], Raw (&vv)[KEYS]) {
    const int64_t s0 = s_begin + step * KEYS;
#pragma unroll
    for (int k = 0; k < KEYS; ++k) {
      int64_t s = s0 + k;
      if (s >= s_end) s = s_begin;  // in-bounds dummy, masked below
      kk[k] = load_row_nc<DPL>(kbase + s * D);
      vv[k] = load_row_nc<DPL>(vbase + s * D);
    }
  };
  int64_t step = warp;
  if (step < n_steps) load_step(step, kr, vr);
  for (; step < n_steps; step += kDecWarps) {
    Raw kc[KEYS], vc[KEYS];
#pragma unroll
    for (int k = 0; k < KEYS; ++k) {
      kc[k] = kr[k];
      vc[k] = vr[k];
    }
    if (step + kDecWarps < n_steps) load_step(step + kDecWarps, kr, vr);

    // partial dots of this lane's slice: part[k * G + g]
    float part[32];
#pragma unroll
    for (int k = 0; k < KEYS; ++k) {
      float kf[DPL];
      unpack_row<DPL>(kc[k], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc = fmaf(qv[g][i], kf[i], acc);
        part[k * G + g] = acc;
      }
    }
    // butterfly reduce-scatter: lane l ends with the full value of index l
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
      const bool upper = (lane & half) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float keep = upper ? part[i + half] : part[i];
        const float send = upper ? part[i] : part[i + half];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
      }
    }
    const int my_key = lane / G;
    const int64_t my_slot = s_begin + step * KEYS + my_key;
    float sc = my_slot < s_end ? part[0] : -INFINITY;
    // max and sum per head over the lanes holding that head (xor masks >= G)
    float mx = sc;
#pragma unroll
    for (int m = G; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = ex2(m_run - m_use);  // m_run = -inf gives 0
    const float pr = ex2(sc - m_use);        // masked score gives 0
    float ps = pr;
#pragma unroll
    for (int m = G; m < 32; m <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, m);
    l_run = l_run * alpha + ps;
    m_run = m_new;

    s_p[warp][lane] = pr;
    if (lane < G) s_alpha[warp][lane] = alpha;
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float a = s_alpha[warp][g];
#pragma unroll
      for (int i = 0; i < DPL; ++i) o[g][i] *= a;
    }
#pragma unroll
    for (int k = 0; k < KEYS; ++k) {
      float vf[DPL];
      unpack_row<DPL>(vc[k], vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pk = s_p[warp][k * G + g];
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[g][i] = fmaf(pk, vf[i], o[g][i]);
      }
    }
    __syncwarp();
  }

  // merge the four warps of this CTA
  if (lane < G) {
    s_m[warp][lane] = m_run;
    s_l[warp][lane] = l_run;
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < DPL; ++i) s_o[warp][g][lane * DPL + i] = o[g][i];
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w][g]);
    float acc = 0.f, L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float wt = ex2(s_m[w][g] - M);
        acc = fmaf(s_o[w][g][c], wt, acc);
        L = fmaf(s_l[w][g], wt, L);
      }
    }
    const int64_t row = (static_cast<int64_t>(b) * p.H + kvh * G + g) * p.splits + split;
    p.ws_o[row * D + c] = acc;
    if (c == 0) {
      p.ws_ml[row * 2 + 0] = M;
      p.ws_ml[row * 2 + 1] = L;
    }
  }
}

// Merge the split partials of one (b, h): o = sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M).
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  const int64_t bh = blockIdx.x;
  const int c = threadIdx.x;
  const float *ml = p.ws_ml + bh * p.splits * 2;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, ml[2 * s]);
  float acc = 0.f, L = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float m = ml[2 * s];
      if (m == -INFINITY) continue;
      const float wt = ex2(m - M);
      acc = fmaf(p.ws_o[(bh * p.splits + s) * D + c], wt, acc);
      L = fmaf(ml[2 * s + 1], wt, L);
    }
  }
  p.out[bh * D + c] = __float2bfloat16_rn(acc / L);
  if (p.lse && c == 0) p.lse[bh] = (M + __log2f(L)) * 0.6931471805599453f;
}

}  // namespace swa
