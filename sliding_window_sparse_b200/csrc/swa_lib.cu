// swa_lib.cu -- the C ABI declared in include/swa.h.
//
// Host code only validates arguments, encodes TMA tensor maps and enqueues
// kernels on the caller's stream.  All kernels live in the headers included
// below, compiled in this single translation unit so they share the one
// device status word g_swa_status.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <atomic>
#include <cstring>
#include <mutex>

#include "../../include/swa.h"
#include "sm100.cuh"
#include "swa_bwd.cuh"
#include "swa_decode.cuh"
#include "swa_fwd2.cuh"
#include "swa_meta.cuh"
#include "swa_selftest.cuh"
#include "swa_split.cuh"
#include "swa_tile.cuh"

namespace {

constexpr int kBQ = swa::kQT;
constexpr int kBK = swa::kKT;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D bf16 tensor map over [planes, rows, d] with a 64-column x box_rows box,
// 128-byte swizzle; rows past `rows` read as zero.
int make_map(CUtensorMap *m, const void *base, int d, int64_t rows, int64_t planes, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return SWA_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : SWA_ERR_CUDA;
}

// Token-major packed tensor [total, heads, d]: dims {d, heads, total}, box
// {64, 1, box_rows} -- the same 128-byte-row swizzled tile in shared memory as
// make_map's {64, box_rows, 1} box.
int make_map_tokens(CUtensorMap *m, const void *base, int d, int64_t heads, int64_t total,
                    int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return SWA_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(total)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(heads)};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : SWA_ERR_CUDA;
}

inline int check_launch() {
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

inline bool good_scale(float s) { return std::isfinite(s) && s > 0.f; }

int common_checks(int B, int H, int Hkv, int d, int64_t W, float scale) {
  if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0) return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  if (W < 1 || !good_scale(scale)) return SWA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H > (1 << 24)) return SWA_ERR_UNSUPPORTED;
  return SWA_OK;
}

// Work units of the forward: two query tiles that read the same key tiles
// (two heads of a GQA group, or query tiles 2p and 2p + 1 of one head).
int64_t fwd_units(swa::Fwd2Params &p) {
  p.pair_heads = (p.G % 2 == 0) ? 1 : 0;
  return p.pair_heads ? static_cast<int64_t>(p.B) * p.Hkv * (p.G / 2) * p.nqt
                      : static_cast<int64_t>(p.B) * p.H * ((p.nqt + 1) / 2);
}

int sm_count(int *sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || *sms < 1)
    return SWA_ERR_CUDA;
  return SWA_OK;
}

// tks / tvs: the sink rows of the chunk-ring path with sinks (any map otherwise).
// full_grid: one CTA per SM whatever the unit count (the split schedule's P).
template <int D, int MODE, bool SINK = false>
int launch_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
               const CUtensorMap &tkr, const CUtensorMap &tvr, swa::Fwd2Params p,
               cudaStream_t st, const CUtensorMap *tks = nullptr,
               const CUtensorMap *tvs = nullptr, bool full_grid = false) {
  using L = swa::Fwd2Layout<D>;
  auto kern = swa::fwd2_kernel<D, MODE, SINK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) !=
      cudaSuccess)
    return SWA_ERR_CUDA;
  // The kernel's warpgroups re-split the registers it is launched with
  // (setmaxnreg); that split assumes exactly kFwd2LaunchRegs per thread.
  // The count is read once per kernel variant; concurrent first calls may
  // both read it and store the same value.
  static std::atomic<int> launch_regs{-1};
  int regs = launch_regs.load(std::memory_order_relaxed);
  if (regs < 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SWA_ERR_CUDA;
    regs = fa.numRegs;
    launch_regs.store(regs, std::memory_order_relaxed);
  }
  if (regs != swa::kFwd2LaunchRegs) return SWA_ERR_UNSUPPORTED;
  const int64_t units = fwd_units(p);
  if (units > 0x7FFFFFFF) return SWA_ERR_UNSUPPORTED;
  p.n_units = static_cast<int>(units);
  int sms = 0;
  if (sm_count(&sms)) return SWA_ERR_CUDA;
  const int grid = full_grid ? sms : static_cast<int>(units < sms ? units : sms);
  kern<<<grid, swa::kFwd2Threads, L::ALLOC, st>>>(tq, tk, tv, tkr, tvr, tks ? *tks : tk,
                                                   tvs ? *tvs : tv, p);
  return check_launch();
}

// Split policy of the decode path (shared by the workspace query and the launch).
void decode_split(int B, int Hkv, int64_t W, int *chunk, int *splits) {
  int c = 512;
  while (c > 128 && static_cast<int64_t>(B) * Hkv * ((W + c - 1) / c) < 4 * 148) c >>= 1;
  *chunk = c;
  *splits = static_cast<int>((W + c - 1) / c);
}

template <int D, int G>
int launch_decode(const swa::DecodeParams &p, cudaStream_t st) {
  dim3 grid(p.n_part, p.Hkv, p.B);
  swa::decode_split_kernel<D, G><<<grid, swa::kDecWarps * 32, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  // The merge kernel is launched as a programmatic dependent of the split
  // kernel: its CTAs may start while the last split CTAs drain and wait in
  // griddepcontrol.wait until every split CTA's partials are visible.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.B * p.H));
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, swa::decode_combine_kernel<D>, p) != cudaSuccess) return SWA_ERR_CUDA;
  return check_launch();
}

template <int D>
int dispatch_decode_g(int G, const swa::DecodeParams &p, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode<D, 1>(p, st);
    case 2: return launch_decode<D, 2>(p, st);
    case 4: return launch_decode<D, 4>(p, st);
    case 8: return launch_decode<D, 8>(p, st);
    default: return SWA_ERR_UNSUPPORTED;
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The chunk forward with its key ranges split across CTAs (swa_split.cuh):
// schedule, attention over the schedule's list, merge of the split units.
template <int D, bool SINK>
int launch_chunk_split(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                       const CUtensorMap &tkr, const CUtensorMap &tvr, const CUtensorMap *tks,
                       const CUtensorMap *tvs, swa::Fwd2Params p, void *workspace,
                       cudaStream_t st) {
  const int64_t units = fwd_units(p);
  if (units > 0x7FFFFFFF) return SWA_ERR_UNSUPPORTED;
  p.n_units = static_cast<int>(units);
  int P = 0;
  if (sm_count(&P)) return SWA_ERR_CUDA;
  int *ws = static_cast<int *>(workspace);
  p.items = reinterpret_cast<const int4 *>(ws + swa::SplitLayout::kHeaderInts);
  p.ws_ml = reinterpret_cast<float *>(ws) + swa::SplitLayout::ml_offset(units, P);
  p.ws_o = reinterpret_cast<float *>(ws) + swa::SplitLayout::o_offset(units, P);
  swa::chunk_split_schedule_kernel<D><<<1, swa::kSplitThreads, 0, st>>>(p, P, ws);
  if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  int e = launch_fwd<D, 1, SINK>(tq, tk, tv, tkr, tvr, p, st, tks, tvs, true);
  if (e) return e;
  swa::chunk_split_merge_kernel<D>
      <<<dim3(P, 2, swa::kQT / swa::kMergeRowsPerCta), 32 * swa::kMergeRowsPerCta, 0, st>>>(p, P,
                                                                                        ws);
  return check_launch();
}

}  // namespace

extern "C" {

const char *swa_status_string(int status) {
  switch (status) {
    case SWA_OK: return "SWA_OK";
    case SWA_ERR_INVALID_ARG: return "SWA_ERR_INVALID_ARG";
    case SWA_ERR_UNSUPPORTED: return "SWA_ERR_UNSUPPORTED";
    case SWA_ERR_CUDA: return "SWA_ERR_CUDA";
    case SWA_ERR_WORKSPACE: return "SWA_ERR_WORKSPACE";
    case SWA_ERR_TIMEOUT: return "SWA_ERR_TIMEOUT";
    case SWA_ERR_DEVICE: return "SWA_ERR_DEVICE";
    default: return "SWA_ERR_UNKNOWN";
  }
}

int swa_version(void) { return (1 << 16) | 0; }

int swa_block_meta(int key_mode, int B, int64_t n_q, int64_t n_k, const int64_t *q_pos0,
                   int64_t W, int tile_q, int tile_k, int8_t *classes, int32_t *ranges,
                   void *stream) {
  if (key_mode != 0 && key_mode != 1) return SWA_ERR_INVALID_ARG;
  if (B < 1 || n_q < 1 || W < 1) return SWA_ERR_INVALID_ARG;
  if (key_mode == 0 && n_k < 1) return SWA_ERR_INVALID_ARG;
  if (key_mode == 1 && (q_pos0 == nullptr || W >= (int64_t(1) << 40)))
    return SWA_ERR_INVALID_ARG;
  if (tile_q < 1 || tile_q > 1024 || tile_k < 1 || tile_k > 1024) return SWA_ERR_INVALID_ARG;
  if (!classes && !ranges) return SWA_ERR_INVALID_ARG;
  swa::MetaParams p;
  p.key_mode = key_mode;
  p.B = B;
  p.n_q = n_q;
  p.n_k = n_k;
  p.W = W;
  p.tile_q = tile_q;
  p.tile_k = tile_k;
  const int64_t nqt = (n_q + tile_q - 1) / tile_q;
  const int64_t nkt = key_mode == 0 ? (n_k + tile_k - 1) / tile_k
                                    : (W + tile_k - 1) / tile_k + (n_q + tile_k - 1) / tile_k;
  if (nqt > 0x7FFFFFFF || nkt > 0x7FFFFFFF || B > 65535) return SWA_ERR_UNSUPPORTED;
  p.nqt = static_cast<int>(nqt);
  p.nkt = static_cast<int>(nkt);
  p.q_pos0 = q_pos0;
  p.classes = classes;
  p.ranges = ranges;
  dim3 grid(p.nqt, B);
  swa::block_meta_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return check_launch();
}

namespace {
int attn_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
             int Hkv, int64_t N, int d, int64_t W, int n_sink, float scale, void *stream) {
  int e = common_checks(B, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k || !v || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_INVALID_ARG;
  if (N < 1 || N >= (int64_t(1) << 29)) return SWA_ERR_INVALID_ARG;
  if (n_sink < 0 || n_sink > kBK) return SWA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if ((e = make_map(&tq, q, d, N, static_cast<int64_t>(B) * H, kBQ))) return e;
  if ((e = make_map(&tk, k, d, N, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  if ((e = make_map(&tv, v, d, N, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  swa::Fwd2Params p;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.n_q = static_cast<int>(N);
  p.n_k = static_cast<int>(N);
  p.W = W < N + kBQ ? W : N + kBQ;
  p.n_sink = n_sink;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nqt = static_cast<int>((N + kBQ - 1) / kBQ);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_sink > 0)
    return d == 128 ? launch_fwd<128, 0, true>(tq, tk, tv, tk, tv, p, st)
                    : launch_fwd<64, 0, true>(tq, tk, tv, tk, tv, p, st);
  return d == 128 ? launch_fwd<128, 0>(tq, tk, tv, tk, tv, p, st)
                  : launch_fwd<64, 0>(tq, tk, tv, tk, tv, p, st);
}
}  // namespace

int swa_attn_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                 int H, int Hkv, int64_t N, int d, int64_t W, float scale, void *stream) {
  return attn_fwd(q, k, v, out, lse, B, H, Hkv, N, d, W, 0, scale, stream);
}

int swa_attn_fwd_sink(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                      int H, int Hkv, int64_t N, int d, int64_t W, int n_sink, float scale,
                      void *stream) {
  return attn_fwd(q, k, v, out, lse, B, H, Hkv, N, d, W, n_sink, scale, stream);
}

int swa_attn_varlen(const void *q, const void *k, const void *v, const int64_t *cu_seqlens,
                    void *out, float *lse, int n_seq, int64_t total, int64_t max_seqlen, int H,
                    int Hkv, int d, int64_t W, int n_sink, float scale, void *stream) {
  int e = common_checks(n_seq, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k || !v || !cu_seqlens || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_INVALID_ARG;
  // token coordinates of the tensor maps are int32
  if (total < 1 || total >= (int64_t(1) << 31) - 2 * kBQ) return SWA_ERR_INVALID_ARG;
  if (max_seqlen < 1 || max_seqlen >= (int64_t(1) << 29)) return SWA_ERR_INVALID_ARG;
  if (n_sink < 0 || n_sink > kBK) return SWA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if ((e = make_map_tokens(&tq, q, d, H, total, kBQ))) return e;
  if ((e = make_map_tokens(&tk, k, d, Hkv, total, kBK))) return e;
  if ((e = make_map_tokens(&tv, v, d, Hkv, total, kBK))) return e;
  swa::Fwd2Params p;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.cu_seqlens = cu_seqlens;
  p.total = total;
  p.B = n_seq;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.n_q = static_cast<int>(max_seqlen);
  p.n_k = static_cast<int>(max_seqlen);
  p.W = W < max_seqlen + kBQ ? W : max_seqlen + kBQ;
  p.n_sink = n_sink;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nqt = static_cast<int>((max_seqlen + kBQ - 1) / kBQ);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_sink > 0)
    return d == 128 ? launch_fwd<128, 2, true>(tq, tk, tv, tk, tv, p, st)
                    : launch_fwd<64, 2, true>(tq, tk, tv, tk, tv, p, st);
  return d == 128 ? launch_fwd<128, 2>(tq, tk, tv, tk, tv, p, st)
                  : launch_fwd<64, 2>(tq, tk, tv, tk, tv, p, st);
}

namespace {
int ring_write(const void *k_new, const void *v_new, void *k_ring, void *v_ring,
               const int64_t *q_start, const int64_t *lens, int B, int Hkv, int64_t T, int d,
               int64_t W, void *stream) {
  if (!k_new || !v_new || !k_ring || !v_ring || !q_start) return SWA_ERR_INVALID_ARG;
  if (B < 1 || Hkv < 1 || T < 1 || W < 1 || (d != 64 && d != 128)) return SWA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_ring) || !aligned16(v_ring))
    return SWA_ERR_INVALID_ARG;
  const int vec = d * 2 / 16;
  const int64_t rows = T < W ? T : W;
  const int64_t total = static_cast<int64_t>(B) * Hkv * rows * vec;
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7FFFFFFF) return SWA_ERR_UNSUPPORTED;
  swa::ring_write_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
      static_cast<uint4 *>(k_ring), static_cast<uint4 *>(v_ring), q_start, lens, B, Hkv, T, vec,
      W);
  return check_launch();
}
}  // namespace

int swa_ring_write(const void *k_new, const void *v_new, void *k_ring, void *v_ring,
                   const int64_t *q_start, int B, int Hkv, int64_t T, int d, int64_t W,
                   void *stream) {
  return ring_write(k_new, v_new, k_ring, v_ring, q_start, nullptr, B, Hkv, T, d, W, stream);
}

namespace {
int chunk_ring(const void *q, const void *k_new, const void *v_new, void *k_ring, void *v_ring,
               const int64_t *q_start, const int64_t *chunk_len, void *out, float *lse, int B,
               int H, int Hkv, int64_t Tq, int d, int64_t W, float scale, int update_ring,
               void *stream, const void *k_sink = nullptr, const void *v_sink = nullptr,
               int n_sink = 0, void *workspace = nullptr, size_t workspace_bytes = 0) {
  int e = common_checks(B, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k_new || !v_new || !k_ring || !v_ring || !q_start || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_ring) ||
      !aligned16(v_ring) || !aligned16(out))
    return SWA_ERR_INVALID_ARG;
  if (Tq < 1 || Tq >= (int64_t(1) << 29) || W >= (int64_t(1) << 29)) return SWA_ERR_INVALID_ARG;
  if (n_sink < 0 || n_sink > kBK) return SWA_ERR_INVALID_ARG;
  if (n_sink > 0 && (!k_sink || !v_sink || !aligned16(k_sink) || !aligned16(v_sink)))
    return SWA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv, tkr, tvr, tks, tvs;
  if ((e = make_map(&tq, q, d, Tq, static_cast<int64_t>(B) * H, kBQ))) return e;
  if ((e = make_map(&tk, k_new, d, Tq, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  if ((e = make_map(&tv, v_new, d, Tq, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  if ((e = make_map(&tkr, k_ring, d, W, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  if ((e = make_map(&tvr, v_ring, d, W, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  if (n_sink > 0) {
    // one 128-row box over the n_sink rows: the rows past them read as zero
    if ((e = make_map(&tks, k_sink, d, n_sink, static_cast<int64_t>(B) * Hkv, kBK))) return e;
    if ((e = make_map(&tvs, v_sink, d, n_sink, static_cast<int64_t>(B) * Hkv, kBK))) return e;
  }
  swa::Fwd2Params p;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.q_start = q_start;
  p.chunk_len = chunk_len;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.n_q = static_cast<int>(Tq);
  p.n_k = static_cast<int>(Tq);
  p.W = W;
  p.n_sink = n_sink;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nqt = static_cast<int>((Tq + kBQ - 1) / kBQ);
  p.n_ring_tiles = static_cast<int>((W + kBK - 1) / kBK);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (workspace) {
    if (workspace_bytes < swa_chunk_split_workspace_bytes(B, H, Hkv, Tq, d, W) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return SWA_ERR_WORKSPACE;
    const CUtensorMap *ps = n_sink > 0 ? &tks : &tk, *pv = n_sink > 0 ? &tvs : &tv;
    if (n_sink > 0)
      e = d == 128 ? launch_chunk_split<128, true>(tq, tk, tv, tkr, tvr, ps, pv, p, workspace, st)
                   : launch_chunk_split<64, true>(tq, tk, tv, tkr, tvr, ps, pv, p, workspace, st);
    else
      e = d == 128 ? launch_chunk_split<128, false>(tq, tk, tv, tkr, tvr, ps, pv, p, workspace, st)
                   : launch_chunk_split<64, false>(tq, tk, tv, tkr, tvr, ps, pv, p, workspace, st);
  } else if (n_sink > 0) {
    e = d == 128 ? launch_fwd<128, 1, true>(tq, tk, tv, tkr, tvr, p, st, &tks, &tvs)
                 : launch_fwd<64, 1, true>(tq, tk, tv, tkr, tvr, p, st, &tks, &tvs);
  } else {
    e = d == 128 ? launch_fwd<128, 1>(tq, tk, tv, tkr, tvr, p, st)
                 : launch_fwd<64, 1>(tq, tk, tv, tkr, tvr, p, st);
  }
  if (e || !update_ring) return e;
  return ring_write(k_new, v_new, k_ring, v_ring, q_start, chunk_len, B, Hkv, Tq, d, W, stream);
}
}  // namespace

int swa_attn_chunk_ring(const void *q, const void *k_new, const void *v_new, void *k_ring,
                        void *v_ring, const int64_t *q_start, void *out, float *lse, int B,
                        int H, int Hkv, int64_t Tq, int d, int64_t W, float scale,
                        int update_ring, void *stream) {
  return chunk_ring(q, k_new, v_new, k_ring, v_ring, q_start, nullptr, out, lse, B, H, Hkv, Tq, d,
                    W, scale, update_ring, stream);
}

int swa_attn_chunk_ring_sink(const void *q, const void *k_new, const void *v_new,
                             void *k_ring, void *v_ring, const void *k_sink, const void *v_sink,
                             int n_sink, const int64_t *q_start, void *out, float *lse, int B,
                             int H, int Hkv, int64_t Tq, int d, int64_t W, float scale,
                             int update_ring, void *stream) {
  if (n_sink < 1) return SWA_ERR_INVALID_ARG;
  return chunk_ring(q, k_new, v_new, k_ring, v_ring, q_start, nullptr, out, lse, B, H, Hkv, Tq, d,
                    W, scale, update_ring, stream, k_sink, v_sink, n_sink);
}

size_t swa_chunk_split_workspace_bytes(int B, int H, int Hkv, int64_t Tq, int d, int64_t W) {
  if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || Tq < 1 || W < 1 || (d != 64 && d != 128))
    return 0;
  swa::Fwd2Params p;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.nqt = static_cast<int>((Tq + kBQ - 1) / kBQ);
  int P = 0;
  if (sm_count(&P)) return 0;
  return static_cast<size_t>(swa::SplitLayout::bytes(fwd_units(p), P, d));
}

int swa_attn_chunk_ring_split(const void *q, const void *k_new, const void *v_new, void *k_ring,
                              void *v_ring, const void *k_sink, const void *v_sink, int n_sink,
                              const int64_t *q_start, const int64_t *chunk_len, void *out,
                              float *lse, int B, int H, int Hkv, int64_t Tq, int d, int64_t W,
                              float scale, int update_ring, void *workspace,
                              size_t workspace_bytes, void *stream) {
  if (!workspace) return SWA_ERR_WORKSPACE;
  return chunk_ring(q, k_new, v_new, k_ring, v_ring, q_start, chunk_len, out, lse, B, H, Hkv, Tq,
                    d, W, scale, update_ring, stream, k_sink, v_sink, n_sink, workspace,
                    workspace_bytes);
}

int swa_attn_chunk_ring_ragged(const void *q, const void *k_new, const void *v_new,
                               void *k_ring, void *v_ring, const int64_t *q_start,
                               const int64_t *chunk_len, void *out, float *lse, int B, int H,
                               int Hkv, int64_t Tq, int d, int64_t W, float scale,
                               int update_ring, void *stream) {
  if (!chunk_len) return SWA_ERR_INVALID_ARG;
  return chunk_ring(q, k_new, v_new, k_ring, v_ring, q_start, chunk_len, out, lse, B, H, Hkv, Tq,
                    d, W, scale, update_ring, stream);
}

size_t swa_decode_workspace_bytes(int B, int H, int Hkv, int d, int64_t W) {
  if (B < 1 || H < 1 || Hkv < 1 || W < 1 || d < 1) return 0;
  int chunk, splits;
  decode_split(B, Hkv, W, &chunk, &splits);
  // one partial per split, plus one for the sink rows of swa_attn_decode_ring_sink
  const size_t rows = static_cast<size_t>(B) * H * (splits + 1);
  return align256(rows * d * sizeof(float)) + align256(rows * 2 * sizeof(float));
}

}  // extern "C"

namespace {
int decode_ring(const void *q, const void *k_ring, const void *v_ring, const void *k_sink,
                const void *v_sink, int n_sink, const int64_t *pos, void *out, float *lse, int B,
                int H, int Hkv, int d, int64_t W, float scale, void *workspace,
                size_t workspace_bytes, void *stream) {
  int e = common_checks(B, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k_ring || !v_ring || !pos || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out))
    return SWA_ERR_INVALID_ARG;
  if (n_sink < 0 || n_sink > 128) return SWA_ERR_INVALID_ARG;
  if (n_sink > 0 && (!k_sink || !v_sink || !aligned16(k_sink) || !aligned16(v_sink)))
    return SWA_ERR_INVALID_ARG;
  if (W >= (int64_t(1) << 31) || B > 65535 || Hkv > 65535) return SWA_ERR_UNSUPPORTED;
  const size_t need = swa_decode_workspace_bytes(B, H, Hkv, d, W);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SWA_ERR_WORKSPACE;
  swa::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.k_ring = static_cast<const __nv_bfloat16 *>(k_ring);
  p.v_ring = static_cast<const __nv_bfloat16 *>(v_ring);
  p.k_sink = static_cast<const __nv_bfloat16 *>(k_sink);
  p.v_sink = static_cast<const __nv_bfloat16 *>(v_sink);
  p.n_sink = n_sink;
  p.pos = pos;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.W = W;
  decode_split(B, Hkv, W, &p.chunk, &p.splits);
  p.n_part = p.splits + (n_sink > 0 ? 1 : 0);
  const size_t rows = static_cast<size_t>(B) * H * (p.splits + 1);
  p.ws_o = static_cast<float *>(workspace);
  p.ws_ml = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                      align256(rows * d * sizeof(float)));
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = H / Hkv;
  return d == 128 ? dispatch_decode_g<128>(G, p, st) : dispatch_decode_g<64>(G, p, st);
}
}  // namespace

extern "C" {

int swa_attn_decode_ring(const void *q, const void *k_ring, const void *v_ring,
                         const int64_t *pos, void *out, float *lse, int B, int H, int Hkv,
                         int d, int64_t W, float scale, void *workspace,
                         size_t workspace_bytes, void *stream) {
  return decode_ring(q, k_ring, v_ring, nullptr, nullptr, 0, pos, out, lse, B, H, Hkv, d, W,
                     scale, workspace, workspace_bytes, stream);
}

int swa_attn_decode_ring_sink(const void *q, const void *k_ring, const void *v_ring,
                              const void *k_sink, const void *v_sink, int n_sink,
                              const int64_t *pos, void *out, float *lse, int B, int H, int Hkv,
                              int d, int64_t W, float scale, void *workspace,
                              size_t workspace_bytes, void *stream) {
  if (n_sink < 1) return SWA_ERR_INVALID_ARG;
  return decode_ring(q, k_ring, v_ring, k_sink, v_sink, n_sink, pos, out, lse, B, H, Hkv, d, W,
                     scale, workspace, workspace_bytes, stream);
}

size_t swa_attn_bwd_workspace_bytes(int B, int H, int64_t N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return align256(static_cast<size_t>(B) * H * static_cast<size_t>(N) * sizeof(float));
}

}  // extern "C"

namespace {
template <int D, int MODE, bool SINK>
int launch_bwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
               const CUtensorMap &tdo, swa::BwdParams p, cudaStream_t st) {
  using L = swa::BwdLayout<D>;
  auto kq = swa::bwd_dq_kernel<D, MODE, SINK>;
  auto kkv = swa::bwd_dkdv_kernel<D, MODE, SINK>;
  if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) !=
          cudaSuccess)
    return SWA_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return SWA_ERR_CUDA;
  // dQ (and D_i) first: the dK/dV kernel reads D_i
  const int64_t uq = static_cast<int64_t>(p.B) * p.H * p.nt;
  const int64_t ukv = static_cast<int64_t>(p.B) * p.Hkv * p.nt;
  if (uq > 0x7FFFFFFF) return SWA_ERR_UNSUPPORTED;
  p.n_units = static_cast<int>(uq);
  kq<<<static_cast<int>(uq < sms ? uq : sms), swa::kBwdThreads, L::ALLOC, st>>>(tq, tk, tv, tdo, p);
  if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  p.n_units = static_cast<int>(ukv);
  kkv<<<static_cast<int>(ukv < sms ? ukv : sms), swa::kBwdThreads, L::ALLOC, st>>>(tq, tk, tv, tdo,
                                                                                  p);
  return check_launch();
}

int attn_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
             const float *lse, void *dq, void *dk, void *dv, int B, int H, int Hkv, int64_t N,
             int d, int64_t W, int n_sink, float scale, void *workspace, size_t workspace_bytes,
             void *stream) {
  int e = common_checks(B, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SWA_ERR_INVALID_ARG;
  if (N < 1 || N >= (int64_t(1) << 29)) return SWA_ERR_INVALID_ARG;
  if (n_sink < 0 || n_sink > kBK) return SWA_ERR_INVALID_ARG;
  const size_t need = swa_attn_bwd_workspace_bytes(B, H, N);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SWA_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv, tdo;
  if ((e = make_map(&tq, q, d, N, static_cast<int64_t>(B) * H, swa::kBwdT))) return e;
  if ((e = make_map(&tk, k, d, N, static_cast<int64_t>(B) * Hkv, swa::kBwdT))) return e;
  if ((e = make_map(&tv, v, d, N, static_cast<int64_t>(B) * Hkv, swa::kBwdT))) return e;
  if ((e = make_map(&tdo, dout, d, N, static_cast<int64_t>(B) * H, swa::kBwdT))) return e;
  swa::BwdParams p;
  p.out = static_cast<const __nv_bfloat16 *>(out);
  p.dout = static_cast<const __nv_bfloat16 *>(dout);
  p.lse = lse;
  p.delta = static_cast<float *>(workspace);
  p.dq = static_cast<__nv_bfloat16 *>(dq);
  p.dk = static_cast<__nv_bfloat16 *>(dk);
  p.dv = static_cast<__nv_bfloat16 *>(dv);
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.N = static_cast<int>(N);
  p.W = static_cast<int>(W < N + swa::kBwdT ? W : N + swa::kBwdT);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nt = static_cast<int>((N + swa::kBwdT - 1) / swa::kBwdT);
  p.n_sink = n_sink;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_sink > 0)
    return d == 128 ? launch_bwd<128, 0, true>(tq, tk, tv, tdo, p, st)
                    : launch_bwd<64, 0, true>(tq, tk, tv, tdo, p, st);
  return d == 128 ? launch_bwd<128, 0, false>(tq, tk, tv, tdo, p, st)
                  : launch_bwd<64, 0, false>(tq, tk, tv, tdo, p, st);
}
}  // namespace

extern "C" {

int swa_attn_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv, int B, int H, int Hkv, int64_t N,
                 int d, int64_t W, float scale, void *workspace, size_t workspace_bytes,
                 void *stream) {
  return attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, H, Hkv, N, d, W, 0, scale, workspace,
                  workspace_bytes, stream);
}

int swa_attn_bwd_sink(const void *q, const void *k, const void *v, const void *out,
                      const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                      int H, int Hkv, int64_t N, int d, int64_t W, int n_sink, float scale,
                      void *workspace, size_t workspace_bytes, void *stream) {
  return attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, H, Hkv, N, d, W, n_sink, scale,
                  workspace, workspace_bytes, stream);
}

size_t swa_attn_varlen_bwd_workspace_bytes(int H, int64_t total) {
  if (H < 1 || total < 1) return 0;
  return align256(static_cast<size_t>(H) * static_cast<size_t>(total) * sizeof(float));
}

int swa_attn_varlen_bwd(const void *q, const void *k, const void *v, const int64_t *cu_seqlens,
                        const void *out, const void *dout, const float *lse, void *dq, void *dk,
                        void *dv, int n_seq, int64_t total, int64_t max_seqlen, int H, int Hkv,
                        int d, int64_t W, int n_sink, float scale, void *workspace,
                        size_t workspace_bytes, void *stream) {
  int e = common_checks(n_seq, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k || !v || !cu_seqlens || !out || !dout || !lse || !dq || !dk || !dv)
    return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SWA_ERR_INVALID_ARG;
  if (total < 1 || total >= (int64_t(1) << 31) - 2 * kBQ) return SWA_ERR_INVALID_ARG;
  if (max_seqlen < 1 || max_seqlen >= (int64_t(1) << 29)) return SWA_ERR_INVALID_ARG;
  if (n_sink < 0 || n_sink > kBK) return SWA_ERR_INVALID_ARG;
  const size_t need = swa_attn_varlen_bwd_workspace_bytes(H, total);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SWA_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv, tdo;
  if ((e = make_map_tokens(&tq, q, d, H, total, swa::kBwdT))) return e;
  if ((e = make_map_tokens(&tk, k, d, Hkv, total, swa::kBwdT))) return e;
  if ((e = make_map_tokens(&tv, v, d, Hkv, total, swa::kBwdT))) return e;
  if ((e = make_map_tokens(&tdo, dout, d, H, total, swa::kBwdT))) return e;
  swa::BwdParams p;
  p.out = static_cast<const __nv_bfloat16 *>(out);
  p.dout = static_cast<const __nv_bfloat16 *>(dout);
  p.lse = lse;
  p.delta = static_cast<float *>(workspace);
  p.dq = static_cast<__nv_bfloat16 *>(dq);
  p.dk = static_cast<__nv_bfloat16 *>(dk);
  p.dv = static_cast<__nv_bfloat16 *>(dv);
  p.cu_seqlens = cu_seqlens;
  p.total = total;
  p.n_sink = n_sink;
  p.B = n_seq;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.N = static_cast<int>(max_seqlen);
  p.W = static_cast<int>(W < max_seqlen + swa::kBwdT ? W : max_seqlen + swa::kBwdT);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nt = static_cast<int>((max_seqlen + swa::kBwdT - 1) / swa::kBwdT);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_sink > 0)
    return d == 128 ? launch_bwd<128, 2, true>(tq, tk, tv, tdo, p, st)
                    : launch_bwd<64, 2, true>(tq, tk, tv, tdo, p, st);
  return d == 128 ? launch_bwd<128, 2, false>(tq, tk, tv, tdo, p, st)
                  : launch_bwd<64, 2, false>(tq, tk, tv, tdo, p, st);
}

int swa_ring_slot_positions(int B, const int64_t *n_written, int64_t W, int64_t *slot_pos,
                            void *stream) {
  if (B < 1 || W < 1 || !n_written || !slot_pos) return SWA_ERR_INVALID_ARG;
  const int64_t total = static_cast<int64_t>(B) * W;
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7FFFFFFF) return SWA_ERR_UNSUPPORTED;
  swa::ring_positions_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                               static_cast<cudaStream_t>(stream)>>>(B, n_written, W, slot_pos);
  return check_launch();
}

int swa_selftest_wait(int64_t limit_ns, int arrive, int32_t *result, void *stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000 || !result) return SWA_ERR_INVALID_ARG;
  swa::selftest_wait_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns), arrive ? 1 : 0, result);
  return check_launch();
}

int swa_get_device_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SWA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_swa_status, sizeof v) != cudaSuccess) return SWA_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_swa_status, &zero, sizeof zero) != cudaSuccess)
    return SWA_ERR_CUDA;
  if (v & SWA_DEV_TIMEOUT) return SWA_ERR_TIMEOUT;
  if (v & SWA_DEV_BADARG) return SWA_ERR_DEVICE;
  return SWA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without a caller-provided workspace.
//
// Some callers have no way to give this library device scratch: a plugin or a
// foreign-language host that owns no device allocator of its own, or a
// serving process that reserved all free device memory for its KV cache up
// front and forbids later allocations.  For them swa_attn_decode_ring_static
// runs the same split and merge kernels as swa_attn_decode_ring, with the
// split partials kept in the file-scope device array below instead of a
// workspace argument.  It calls no allocator (cudaMalloc, cudaFree or any
// library routine that allocates).
//
// The array is g_swa_static_scratch_bytes (16 MiB) long on every device that loads
// this library and stays resident until the process exits.  All calls on a
// device share it and it keeps the last call's contents; nothing in it has to
// start at zero, because every split partial is written before the merge
// reads it.  Two calls whose kernels overlap on the same device (for example
// on two streams without ordering between them) race on the array and give
// wrong results: order such calls on one stream or with events.
//
// Host code cannot use the array's name as a device address, so the first
// call on each device looks the address up with cudaGetSymbolAddress while
// that device is current and caches it; make that first call before any
// stream capture.  The cached address is valid for the life of the device's
// primary context: after a cudaDeviceReset() of that device it is stale, and
// this entry point must not be called on that device again.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t g_swa_static_scratch_bytes = size_t(16) << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_swa_static_scratch[g_swa_static_scratch_bytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mutex;
void *g_static_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
int static_scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SWA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SWA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_swa_static_scratch) != cudaSuccess || !ptr)
      return SWA_ERR_CUDA;
    g_static_scratch_ptr[dev] = ptr;
  }
  *out = g_static_scratch_ptr[dev];
  return SWA_OK;
}

}  // namespace

extern "C" {

int swa_attn_decode_ring_static(const void *q, const void *k_ring, const void *v_ring,
                                const int64_t *pos, void *out, float *lse, int B, int H, int Hkv,
                                int d, int64_t W, float scale, void *stream) {
  int e = common_checks(B, H, Hkv, d, W, scale);
  if (e) return e;
  if (!q || !k_ring || !v_ring || !pos || !out) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out))
    return SWA_ERR_INVALID_ARG;
  if (W >= (int64_t(1) << 31) || B > 65535 || Hkv > 65535) return SWA_ERR_UNSUPPORTED;
  // the split partials must fit in the static array
  const size_t need = swa_decode_workspace_bytes(B, H, Hkv, d, W);
  if (need == 0 || need > g_swa_static_scratch_bytes) return SWA_ERR_WORKSPACE;
  void *scratch = nullptr;
  if ((e = static_scratch_address(&scratch))) return e;
  return swa_attn_decode_ring(q, k_ring, v_ring, pos, out, lse, B, H, Hkv, d, W, scale, scratch,
                              g_swa_static_scratch_bytes, stream);
}

}  // extern "C"
