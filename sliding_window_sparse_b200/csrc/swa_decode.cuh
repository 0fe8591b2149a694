// swa_decode.cuh -- batched single-token decode from a W-slot ring cache.
//
// The cost of a decode step is reading the KV cache from HBM (sparse-attention
// taxonomy page, section 1), so the split kernel streams every key/value slot
// of a (sequence, kv head) exactly once with 16-byte coalesced loads and serves
// all G query heads of the group from the same registers.  The slot range of
// one (b, kv head) is cut into `splits` CTAs; each writes an unnormalised
// partial (o, running max m, running sum l, base 2) to the workspace, and
// decode_combine_kernel merges them.  With attention sinks (sparse-attention
// taxonomy page, section 3.2: StreamingLLM keeps the first tokens besides the
// recent W) one more CTA per (b, kv head) streams the sink rows that lie
// before the window, as one more partial.
//
// Warp layout: a key row of D bf16 is read by LPK = D / 8 lanes (16 bytes
// each), so one warp-wide load covers KPW = 32 / LPK consecutive slots.  Lane
// (kg, sub) owns head dims [8 sub, 8 sub + 8) of the keys kg, kg + KPW, ...
// A step takes R loads per lane (KPS = R * KPW slots).  The lane forms
// NV = R * G partial dot products (its 8 dims, packed f32x2 FMAs); a butterfly
// over the LPK lanes of its key group scatters them so that lane sub ends with
// the full score of value index sub / DUP (DUP = LPK / NV lanes hold each
// value).  Online softmax per head runs across the lanes holding that head;
// probabilities go through shared memory and every lane accumulates the
// partial o of its keys and dims; the KPW key groups are summed at the end.
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
  const __nv_bfloat16 *k_sink;  // [B, Hkv, n_sink, D] positions 0 .. n_sink-1, or nullptr
  const __nv_bfloat16 *v_sink;
  const int64_t *pos;           // [B]
  float *ws_o;                  // [B*H, n_part, D]
  float *ws_ml;                 // [B*H, n_part, 2]  (m, l) base-2 domain
  __nv_bfloat16 *out;           // [B, H, D]
  float *lse;                   // [B, H] or nullptr
  int B, H, Hkv;
  int64_t W;
  int chunk;   // slots per split CTA
  int splits;  // ring CTAs per (b, kv head)
  int n_sink;  // sink rows (0: none)
  int n_part;  // partials per (b, h): splits, plus one for the sinks
  float scale_log2;
};

__device__ __forceinline__ void bf16x8_to_f32x2(const uint4 &raw, float2 (&f)[4]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

__device__ __forceinline__ uint4 ldg_stream(const __nv_bfloat16 *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <int D, int G>
struct DecodeShape {
  static constexpr int LPK = D / 8;                       // lanes per key row
  static constexpr int KPW = 32 / LPK;                    // slots per warp-wide load
  static constexpr int MAXR = D == 128 ? 4 : 2;
  static constexpr int R = (LPK / G) < MAXR ? (LPK / G) : MAXR;  // loads per lane per step
  static constexpr int NV = R * G;                        // partial dots per lane
  static constexpr int DUP = LPK / NV;                    // lanes holding each full value
  static constexpr int KPS = R * KPW;                     // slots per step
  static_assert(R >= 1 && NV <= LPK && (LPK % NV) == 0, "unsupported group size");
};

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32) decode_split_kernel(const DecodeParams p) {
  using S = DecodeShape<D, G>;
  constexpr int LPK = S::LPK, KPW = S::KPW, R = S::R, NV = S::NV, DUP = S::DUP, KPS = S::KPS;

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPK;  // dims [8 sub, 8 sub + 8)
  const int kg = lane / LPK;   // key group within a warp-wide load

  __shared__ float s_p[kDecWarps][KPS * G];
  __shared__ float s_alpha[kDecWarps][G];
  __shared__ float s_m[kDecWarps][G];
  __shared__ float s_l[kDecWarps][G];
  __shared__ float s_o[kDecWarps][G][D];

  const int64_t pos = p.pos[b];
  int64_t nvalid = pos + 1 < p.W ? pos + 1 : p.W;  // slots 0..pos are filled before the wrap
  if (pos < 0) {
    nvalid = 0;
    if (threadIdx.x == 0 && split == 0 && kvh == 0) atomicOr(&g_swa_status, SWA_DEV_BADARG);
  }
  // the last CTA of a sink launch reads sink rows j < pos - W + 1 (the rest are in the ring)
  const bool sink_part = split >= p.splits;
  int64_t s_begin = static_cast<int64_t>(split) * p.chunk;
  int64_t s_end = s_begin + p.chunk;
  if (s_end > nvalid) s_end = nvalid;
  if (sink_part) {
    s_begin = 0;
    s_end = pos < 0 ? 0 : pos - p.W + 1;
    if (s_end > p.n_sink) s_end = p.n_sink;
  }

  // q slices of the G heads (8 dims each), pre-scaled into the base-2 domain
  float2 qv[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16 *qp = p.q + (static_cast<int64_t>(b) * p.H + kvh * G + g) * D + sub * 8;
    float2 f[4];
    bf16x8_to_f32x2(*reinterpret_cast<const uint4 *>(qp), f);
#pragma unroll
    for (int i = 0; i < 4; ++i) qv[g][i] = make_float2(f[i].x * p.scale_log2, f[i].y * p.scale_log2);
  }

  const int64_t kv_base = (static_cast<int64_t>(b) * p.Hkv + kvh) * (sink_part ? p.n_sink : p.W);
  const __nv_bfloat16 *kbase = (sink_part ? p.k_sink : p.k_ring) + kv_base * D + sub * 8;
  const __nv_bfloat16 *vbase = (sink_part ? p.v_sink : p.v_ring) + kv_base * D + sub * 8;

  float2 o[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[g][i] = make_float2(0.f, 0.f);
  float m_run = -INFINITY, l_run = 0.f;  // head of this lane's value index

  const int64_t n_steps = s_end > s_begin ? (s_end - s_begin + KPS - 1) / KPS : 0;
  uint4 kr[R], vr[R];
  auto load_step = [&](int64_t step, uint4 (&kk)[R], uint4 (&vv)[R]) {
    const int64_t s0 = s_begin + step * KPS + kg;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      int64_t s = s0 + r * KPW;
      if (s >= s_end) s = s_begin;  // in-bounds dummy, masked below
      kk[r] = ldg_stream(kbase + s * D);
      vv[r] = ldg_stream(vbase + s * D);
    }
  };
  int64_t step = warp;
  if (step < n_steps) load_step(step, kr, vr);
  for (; step < n_steps; step += kDecWarps) {
    uint4 kc[R], vc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      kc[r] = kr[r];
      vc[r] = vr[r];
    }
    if (step + kDecWarps < n_steps) load_step(step + kDecWarps, kr, vr);

    // partial dot products part[r * G + g] over this lane's 8 dims
    float part[NV];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 kf[4];
      bf16x8_to_f32x2(kc[r], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 acc = __fmul2_rn(qv[g][0], kf[0]);
#pragma unroll
        for (int i = 1; i < 4; ++i) acc = __ffma2_rn(qv[g][i], kf[i], acc);
        part[r * G + g] = acc.x + acc.y;
      }
    }
    // butterfly over the LPK lanes of the key group: scatter NV values, then sum duplicates
    {
      int cnt = NV;
#pragma unroll
      for (int half = LPK / 2; half >= 1; half >>= 1) {
        if (cnt > 1) {
          const int h2 = cnt / 2;
          const bool upper = (sub & half) != 0;
#pragma unroll
          for (int i = 0; i < NV / 2; ++i) {
            if (i < h2) {
              const float keep = upper ? part[i + h2] : part[i];
              const float send = upper ? part[i] : part[i + h2];
              part[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
            }
          }
          cnt = h2;
        } else {
          part[0] += __shfl_xor_sync(0xffffffffu, part[0], half);
        }
      }
    }
    const int v_idx = sub / DUP;  // value index held by this lane
    const int my_r = v_idx / G, my_g = v_idx % G;
    const int key_in_step = my_r * KPW + kg;
    const int64_t my_slot = s_begin + step * KPS + key_in_step;
    const float sc = my_slot < s_end ? part[0] : -INFINITY;
    // max and sum per head over the lanes holding that head (one copy per value)
    float mx = sc;
#pragma unroll
    for (int m = DUP * G; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = ex2(m_run - m_use);  // m_run = -inf gives 0
    const float pr = ex2(sc - m_use);        // masked score gives 0
    float ps = pr;
#pragma unroll
    for (int m = DUP * G; m < 32; m <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, m);
    l_run = l_run * alpha + ps;
    m_run = m_new;

    s_p[warp][key_in_step * G + my_g] = pr;
    if (kg == 0 && v_idx < G) s_alpha[warp][v_idx] = alpha;
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float a = s_alpha[warp][g];
      const float2 a2 = make_float2(a, a);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[g][i] = __fmul2_rn(o[g][i], a2);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 vf[4];
      bf16x8_to_f32x2(vc[r], vf);
      const int key = r * KPW + kg;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pk = s_p[warp][key * G + g];
        const float2 p2 = make_float2(pk, pk);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[g][i] = __ffma2_rn(p2, vf[i], o[g][i]);
      }
    }
    __syncwarp();
  }

  // this CTA's loads are done: let the dependent merge kernel start launching
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // sum the partial o of the KPW key groups (same dims, different slots)
#pragma unroll
  for (int m = LPK; m < 32; m <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[g][i].x += __shfl_xor_sync(0xffffffffu, o[g][i].x, m);
        o[g][i].y += __shfl_xor_sync(0xffffffffu, o[g][i].y, m);
      }
  // merge the warps of this CTA (a lane of key group 0 whose value index g < G holds head g's m, l)
  if (kg == 0 && sub / DUP < G) {
    const int g = sub / DUP;
    s_m[warp][g] = m_run;
    s_l[warp][g] = l_run;
  }
  if (kg == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s_o[warp][g][sub * 8 + 2 * i] = o[g][i].x;
        s_o[warp][g][sub * 8 + 2 * i + 1] = o[g][i].y;
      }
  }
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
    const int64_t row = (static_cast<int64_t>(b) * p.H + kvh * G + g) * p.n_part + split;
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
  // launched as a programmatic dependent of the split kernel: wait for its results
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t bh = blockIdx.x;
  const int c = threadIdx.x;
  const float *ml = p.ws_ml + bh * p.n_part * 2;
  float M = -INFINITY;
  for (int s = 0; s < p.n_part; ++s) M = fmaxf(M, ml[2 * s]);
  float acc = 0.f, L = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.n_part; ++s) {
      const float m = ml[2 * s];
      if (m == -INFINITY) continue;
      const float wt = ex2(m - M);
      acc = fmaf(p.ws_o[(bh * p.n_part + s) * D + c], wt, acc);
      L = fmaf(ml[2 * s + 1], wt, L);
    }
  }
  p.out[bh * D + c] = __float2bfloat16_rn(acc / L);
  if (p.lse && c == 0) p.lse[bh] = (M + __log2f(L)) * 0.6931471805599453f;
}

}  // namespace swa
