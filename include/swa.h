/*
 * swa.h -- C ABI of the B200 (sm_100a) causal sliding-window attention library.
 *
 * The operation (M003 note "weight sparsity vs attention sparsity", section 03;
 * Chapter 10 "local and sparse attention: SWA and DSA", section 10.1):
 *
 *   a query at logical position i may read the key at logical position j iff
 *   max(0, i - W + 1) <= j <= i   (the window of W keys includes the query's
 *   own position); scores are scale * <q_i, k_j> on those pairs only, the
 *   softmax is normalised over those pairs only, and the output is the
 *   softmax-weighted sum of the matching value rows.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major (C order), bfloat16 unless stated.  Query
 *    tensors are [B, H, rows, d]; key/value tensors are [B, Hkv, rows, d].
 *    Query head h reads key/value head h / (H / Hkv) (contiguous groups of
 *    G = H / Hkv query heads share one key/value head).
 *  - Every pointer argument named as device memory must point to memory of
 *    the current CUDA device, 16-byte aligned.  The caller owns all memory;
 *    the library never allocates, frees or retains a pointer after a call.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every compute call only validates its arguments on the host
 *    and enqueues kernels on `stream`; it returns before the work finishes.
 *  - d (head dim) must be 64 or 128.  W >= 1; W >= the sequence length means
 *    plain causal attention.  `scale` must be finite and > 0.
 *  - Return value: SWA_OK (0) or one of the positive error codes below, so
 *    that a caller can test `if (status)` and index a table by code.  Nothing
 *    is printed and no exception crosses the ABI.  Arguments are checked before
 *    anything is enqueued: an invalid argument enqueues nothing.  Errors found
 *    on the device (a negative position, a wait that timed out) set a device
 *    status word that swa_get_device_status() reads and clears.
 *  - Thread safety: calls are stateless apart from per-process caches: a
 *    driver entry point (set up once under a lock), the launch register
 *    count of each attention-kernel variant (an atomic, read once; every
 *    thread reads the same value) and the scratch address of
 *    swa_attn_decode_ring_static (set up once per device under a lock).
 *  - The prefill / chunk / varlen kernels re-split their registers between
 *    warp groups and are written for 168 registers per thread at launch; a
 *    build that compiled them otherwise makes those calls return
 *    SWA_ERR_UNSUPPORTED instead of launching.
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SWA_API __attribute__((visibility("default")))
#else
#define SWA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define SWA_OK 0
#define SWA_ERR_INVALID_ARG 1 /* a size, pointer, alignment or value is out of range   */
#define SWA_ERR_UNSUPPORTED 2 /* valid request outside what the kernels implement      */
#define SWA_ERR_CUDA 3        /* a CUDA runtime or driver call failed                  */
#define SWA_ERR_WORKSPACE 4   /* workspace missing or smaller than required            */
#define SWA_ERR_TIMEOUT 5     /* a device-side wait gave up (reported by get_status)   */
#define SWA_ERR_DEVICE 6      /* a device-side argument check failed (get_status)      */

/* Human-readable name of a status code (static string, never NULL). */
SWA_API const char *swa_status_string(int status);

/* Library ABI version: (major << 16) | minor. */
SWA_API int swa_version(void);

/*
 * swa_block_meta -- tile metadata built on the device.
 * Passage: M003 note section 04 (tiles that are entirely invisible are
 * skipped, entirely visible tiles need no mask, partially visible tiles are
 * computed whole and masked at the boundary) and section 07 (metadata is
 * built for the pattern and timed with the kernel).
 *
 * key_mode 0 (linear): query row i of sequence b sits at logical position
 *   q_pos0[b] + i (q_pos0 == NULL: 0), 0 <= i < n_q; key column j sits at
 *   position j, 0 <= j < n_k.
 * key_mode 1 (ring + chunk, Chapter 10 section 10.2): queries are a chunk at
 *   positions q_pos0[b] + i (q_pos0 is the chunk start, required); the key
 *   axis is the W slots of a ring buffer in physical order (slot s holds the
 *   most recent position p < q_pos0[b] with p mod W == s, or nothing), tiled
 *   on their own, followed by the n_q chunk keys at q_pos0[b] + t, tiled on
 *   their own.  n_k is ignored.
 *
 * Tiles are tile_q x tile_k (each 1..1024); ragged last tiles are clipped to
 * their in-range coordinates.  Outputs (device memory, caller-allocated):
 *   classes: int8 [B, nqt, nkt] (may be NULL): 0 skip, 1 full, 2 partial;
 *   ranges:  int32 [B, nqt, 4]  (may be NULL): {live tiles, full tiles,
 *            first live tile, last live tile} (-1 when there is none).  In
 *            mode 0 the live tiles of a query tile are always the contiguous
 *            run first..last (the windows of consecutive rows overlap), and
 *            the full tiles a contiguous run inside it, so the counts and the
 *            ends locate both runs; in mode 1 the ring's physical order can
 *            split the live tiles into two runs, on either side of the
 *            slots that hold the oldest, invisible positions, which a single
 *            [lo, hi) pair could not describe -- hence counts plus ends
 *            rather than two half-open ranges;
 * with nqt = ceil(n_q / tile_q) and nkt = ceil(n_k / tile_k) (mode 0) or
 * ceil(W / tile_k) + ceil(n_q / tile_k) (mode 1).
 */
SWA_API int swa_block_meta(int key_mode, int B, int64_t n_q, int64_t n_k, const int64_t *q_pos0,
                   int64_t W, int tile_q, int tile_k, int8_t *classes, int32_t *ranges,
                   void *stream);

/*
 * swa_attn_fwd -- tile-skipping prefill forward.
 * Passage: M003 note sections 03-04; Chapter 10 section 10.1.
 * No metadata argument: the class of a (query tile, key tile) pair is a
 * closed form of positions and W, which the kernel evaluates inline per tile
 * (two integer compares), the same classification swa_block_meta writes out.
 *   q:   [B, H, N, d]    bf16, device     k, v: [B, Hkv, N, d] bf16, device
 *   out: [B, H, N, d]    bf16, device (written)
 *   lse: [B, H, N] fp32, device, or NULL: natural-log log-sum-exp of the
 *        scaled scores of each row over its allowed keys.
 * Query and key row i both sit at logical position i.  Only key tiles that
 * hold an allowed pair are loaded; only partially visible tiles are masked.
 * Limits: 1 <= N < 2^29, H % Hkv == 0.
 */
SWA_API int swa_attn_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                 int H, int Hkv, int64_t N, int d, int64_t W, float scale, void *stream);

/*
 * swa_attn_fwd_sink -- swa_attn_fwd with attention sinks.
 * Passage: sparse-attention taxonomy page section 3.2 (StreamingLLM keeps the
 * first tokens visible besides the recent W).  Query i reads key j iff
 * j <= i and (j >= i - W + 1 or j < n_sink).
 *   n_sink: 0 <= n_sink <= 128 (0 is swa_attn_fwd).
 * Other arguments, layouts and limits as swa_attn_fwd.
 */
SWA_API int swa_attn_fwd_sink(const void *q, const void *k, const void *v, void *out, float *lse,
                              int B, int H, int Hkv, int64_t N, int d, int64_t W, int n_sink,
                              float scale, void *stream);

/*
 * swa_attn_varlen -- prefill over a packed batch of sequences of different
 * lengths, each with its own window.
 * Passage: "Dense attention vs sparse SWA" blog section 5.2, tip 4 (in a
 * packed batch the window is per sequence; cu_seqlens must split the samples
 * exactly or windows leak across them); M003 note section 03 within each
 * sequence; sinks as swa_attn_fwd_sink.
 *   q:   [total, H, d]   bf16, device (token-major)
 *   k, v: [total, Hkv, d] bf16, device
 *   cu_seqlens: int64 [n_seq + 1], device: sequence s is tokens
 *        cu_seqlens[s] .. cu_seqlens[s+1] - 1, at positions 0, 1, ... of its
 *        own; non-decreasing, cu_seqlens[n_seq] <= total, every length
 *        <= max_seqlen (else SWA_ERR_DEVICE is set on the device and the
 *        offending sequence is skipped).  Empty sequences are allowed.
 *   out: [total, H, d] bf16, device; rows of tokens outside every sequence are
 *        not written.
 *   lse: [H, total] fp32, device, or NULL.
 *   n_sink: 0 <= n_sink <= 128: the first n_sink positions of each sequence
 *        stay visible to all of its later queries.
 * Limits: 1 <= total < 2^31 - 256, 1 <= max_seqlen < 2^29.  Tokens of a
 * neighbouring sequence share tiles with a sequence's edges and get weight
 * zero, so all of q, k, v must be finite.
 */
SWA_API int swa_attn_varlen(const void *q, const void *k, const void *v,
                            const int64_t *cu_seqlens, void *out, float *lse, int n_seq,
                            int64_t total, int64_t max_seqlen, int H, int Hkv, int d, int64_t W,
                            int n_sink, float scale, void *stream);

/*
 * swa_attn_bwd_workspace_bytes -- bytes of scratch swa_attn_bwd needs (one
 * fp32 D_i = <dout_i, out_i> per query row: B * H * N * 4, 256-aligned).
 */
SWA_API size_t swa_attn_bwd_workspace_bytes(int B, int H, int64_t N);

/*
 * swa_attn_bwd -- gradients of the tile-skipping prefill (swa_attn_fwd).
 * Passage: M003 note sections 07-08 (outputs and Q/K/V gradients are checked
 * under the same window mask); the window rule of sections 03-04.
 * For the loss sum(out * dout), with P the softmax of scale * Q K^T over the
 * allowed keys: dV = P^T dout, dP = dout V^T, D_i = <dout_i, out_i>,
 * dS = P o (dP - D), dQ = scale * dS K, dK = scale * dS^T Q; dK and dV are
 * summed over the G query heads of each KV head.  Key tiles outside every
 * window of a query tile are skipped, as in the forward.
 *   q, out, dout: [B, H, N, d] bf16, device (out: the forward's output)
 *   k, v:         [B, Hkv, N, d] bf16, device
 *   lse:  [B, H, N] fp32, device: the forward's natural-log LSE (same scale)
 *   dq:   [B, H, N, d] bf16, device (written)
 *   dk, dv: [B, Hkv, N, d] bf16, device (written, not accumulated)
 *   workspace: device scratch of at least swa_attn_bwd_workspace_bytes(B, H,
 *         N) bytes, caller-owned; contents on entry are ignored.
 * Two kernels on `stream`: dQ (which also writes D_i), then dK/dV.
 * Limits as swa_attn_fwd: 1 <= N < 2^29, d in {64, 128}.
 */
SWA_API int swa_attn_bwd(const void *q, const void *k, const void *v, const void *out,
                         const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                         int H, int Hkv, int64_t N, int d, int64_t W, float scale,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * swa_attn_bwd_sink -- gradients of swa_attn_fwd_sink (attention sinks).
 * Passage: M003 note sections 07-08 (gradients under the same mask as the
 * outputs); sparse-attention taxonomy page section 3.2 for the mask: query i
 * reads key j iff j <= i and (j >= i - W + 1 or j < n_sink).  Key tile 0,
 * which holds the sinks, is read by every query tile.
 *   n_sink: 0 <= n_sink <= 128 (0 is swa_attn_bwd); lse: from
 *   swa_attn_fwd_sink with the same n_sink.
 * Other arguments, layouts, workspace and limits as swa_attn_bwd.
 */
SWA_API int swa_attn_bwd_sink(const void *q, const void *k, const void *v, const void *out,
                              const void *dout, const float *lse, void *dq, void *dk, void *dv,
                              int B, int H, int Hkv, int64_t N, int d, int64_t W, int n_sink,
                              float scale, void *workspace, size_t workspace_bytes, void *stream);

/*
 * swa_attn_varlen_bwd_workspace_bytes -- bytes of scratch swa_attn_varlen_bwd
 * needs: one fp32 D_i per (head, token): H * total * 4, 256-aligned.
 */
SWA_API size_t swa_attn_varlen_bwd_workspace_bytes(int H, int64_t total);

/*
 * swa_attn_varlen_bwd -- gradients of swa_attn_varlen (packed sequences, each
 * with its own window, optional sinks).
 * Passage: M003 note sections 07-08; "Dense attention vs sparse SWA" blog
 * section 5.2 tip 4 (windows per sequence, no leakage across cu_seqlens);
 * taxonomy page section 3.2 for the sinks.  Same gradients as swa_attn_bwd,
 * per sequence; nothing flows between sequences.
 *   q, out, dout, dq: [total, H, d] bf16, device (token-major, as the forward)
 *   k, v, dk, dv:     [total, Hkv, d] bf16, device
 *   cu_seqlens: int64 [n_seq + 1], device, as swa_attn_varlen (bad offsets
 *        set SWA_ERR_DEVICE and the sequence is skipped).
 *   lse: [H, total] fp32, device: the forward's natural-log LSE.
 *   n_sink: 0 <= n_sink <= 128, as in the forward.
 *   workspace: at least swa_attn_varlen_bwd_workspace_bytes(H, total) bytes.
 * Rows of tokens outside every sequence of dq, dk, dv are not written.
 * Limits as swa_attn_varlen.
 */
SWA_API int swa_attn_varlen_bwd(const void *q, const void *k, const void *v,
                                const int64_t *cu_seqlens, const void *out, const void *dout,
                                const float *lse, void *dq, void *dk, void *dv, int n_seq,
                                int64_t total, int64_t max_seqlen, int H, int Hkv, int d,
                                int64_t W, int n_sink, float scale, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * swa_attn_chunk_ring -- chunked prefill over a W-slot ring-buffer KV cache.
 * Passage: Chapter 10 section 10.2 (a chunk of T_q queries needs the union of
 * W + T_q - 1 keys; the persistent cache keeps only the last W); M003 note
 * section 06 (logical positions keep growing while slots are reused);
 * "Dense attention vs sparse SWA" blog section 3.2 (the circular cache).
 *   q:            [B, H, Tq, d]    bf16, device   chunk queries
 *   k_new, v_new: [B, Hkv, Tq, d]  bf16, device   chunk keys / values
 *   k_ring, v_ring: [B, Hkv, W, d] bf16, device   ring cache; before the call
 *                 slot s of sequence b holds the most recent position
 *                 p < q_start[b] with p mod W == s (empty if none)
 *   q_start: int64 [B], device: logical position of the chunk's first query
 *                 (>= 0; a negative value sets SWA_ERR_DEVICE on the device)
 *   out: [B, H, Tq, d] bf16, device;  lse: [B, H, Tq] fp32 or NULL.
 * Query t sits at q_start[b] + t and attends to ring keys and chunk keys by
 * logical position.  If update_ring != 0, after the attention (same stream)
 * the chunk rows whose positions are among the last W are written into slots
 * position mod W, so the ring then serves the next chunk or decode step.
 * The ring is only written when update_ring != 0.  Limits: 1 <= Tq < 2^29,
 * W < 2^29.  Empty ring slots must hold finite values (a zero-filled cache
 * does): a tile that mixes them with visible keys loads them and gives them
 * weight zero, and 0 * inf is NaN.
 */
SWA_API int swa_attn_chunk_ring(const void *q, const void *k_new, const void *v_new, void *k_ring,
                        void *v_ring, const int64_t *q_start, void *out, float *lse, int B,
                        int H, int Hkv, int64_t Tq, int d, int64_t W, float scale,
                        int update_ring, void *stream);

/*
 * swa_attn_chunk_ring_sink -- swa_attn_chunk_ring with attention sinks.
 * Passage: sparse-attention taxonomy page section 3.2 (StreamingLLM keeps the
 * first tokens visible besides the recent W) over Chapter 10 section 10.2.
 * Query t at position p = q_start[b] + t reads key j iff j <= p and
 * (j >= p - W + 1 or j < n_sink): positions in the window from the ring and
 * the chunk as in swa_attn_chunk_ring, the sinks before the window from
 * k_sink / v_sink.
 *   k_sink, v_sink: [B, Hkv, n_sink, d] bf16, device: row j holds position j
 *      for every j < n_sink, written by the caller before the call (for a
 *      chunk that contains some of them, copy those rows from k_new / v_new
 *      first).  1 <= n_sink <= 128.  The ring update leaves them untouched.
 * Other arguments, layouts and limits as swa_attn_chunk_ring.
 */
SWA_API int swa_attn_chunk_ring_sink(const void *q, const void *k_new, const void *v_new,
                                     void *k_ring, void *v_ring, const void *k_sink,
                                     const void *v_sink, int n_sink, const int64_t *q_start,
                                     void *out, float *lse, int B, int H, int Hkv, int64_t Tq,
                                     int d, int64_t W, float scale, int update_ring,
                                     void *stream);

/*
 * swa_attn_chunk_ring_ragged -- swa_attn_chunk_ring for a batch whose chunks
 * have different lengths (Chapter 10 section 10.2 applied per sequence; the
 * window is per sequence, as the blog's troubleshooting section 5.2 stresses
 * for batched requests).
 *   chunk_len: int64 [B], device: sequence b's chunk has chunk_len[b] valid
 *              rows, 0 <= chunk_len[b] <= Tq (a value outside that range sets
 *              SWA_ERR_DEVICE on the device).  Its queries t < chunk_len[b]
 *              sit at q_start[b] + t and see the ring and the chunk keys
 *              t' < chunk_len[b] only; rows t >= chunk_len[b] of q, k_new,
 *              v_new are padding: they get weight zero (so, like empty ring
 *              slots, they must be finite), their output rows and lse
 *              entries are left unwritten, and update_ring writes only the
 *              valid rows among the last W.  A sequence with chunk_len[b] = 0
 *              costs no tile work.
 * Other arguments, layouts and limits as swa_attn_chunk_ring; chunk_len may
 * not be NULL.
 */
SWA_API int swa_attn_chunk_ring_ragged(const void *q, const void *k_new, const void *v_new,
                                       void *k_ring, void *v_ring, const int64_t *q_start,
                                       const int64_t *chunk_len, void *out, float *lse, int B,
                                       int H, int Hkv, int64_t Tq, int d, int64_t W, float scale,
                                       int update_ring, void *stream);

/*
 * swa_chunk_split_workspace_bytes -- bytes of scratch swa_attn_chunk_ring_split
 * needs for these sizes on the current device (its SM count sets how many
 * parts a call can have), 256-byte aligned; 0 for invalid sizes.
 */
SWA_API size_t swa_chunk_split_workspace_bytes(int B, int H, int Hkv, int64_t Tq, int d,
                                               int64_t W);

/*
 * swa_attn_chunk_ring_split -- the chunked prefill over a ring of
 * swa_attn_chunk_ring, swa_attn_chunk_ring_ragged and swa_attn_chunk_ring_sink
 * in one call, with a caller workspace that lets it balance its work.
 * Passage: Chapter 10 section 10.2 (each query of a chunk attends to its own
 * window over the ring and chunk keys; splitting that key set changes only
 * how the softmax is summed).  Every two-query-tile unit of a chunk reads
 * about the same number of key tiles, so when the live units (those whose
 * rows hold valid chunk rows) leave the last round of units on the SMs part
 * empty -- a batch of short or few chunks -- each unit of that round is cut
 * into parts over its key tiles, one per SM; the parts write unnormalised
 * rows with their running max and sum to the workspace and a merge kernel
 * combines them (as the decode path merges its splits).  Results equal the
 * unsplit call's within rounding (a different summation order).
 *   k_sink, v_sink, n_sink: as swa_attn_chunk_ring_sink, or NULL, NULL, 0.
 *   chunk_len: as swa_attn_chunk_ring_ragged, or NULL (every chunk Tq rows).
 *   workspace: device scratch of at least swa_chunk_split_workspace_bytes(B,
 *      H, Hkv, Tq, d, W) bytes, 256-byte aligned, caller-owned; contents on
 *      entry are ignored (SWA_ERR_WORKSPACE if missing, small or unaligned).
 *      The call's kernels write it until the merge ends, so two calls in
 *      flight at once (on different streams) need workspaces of their own.
 * Other arguments, layouts, limits and the ring update as swa_attn_chunk_ring.
 * Three kernels on `stream` (schedule, attention, merge), then the ring
 * update when update_ring != 0.
 */
SWA_API int swa_attn_chunk_ring_split(const void *q, const void *k_new, const void *v_new,
                                      void *k_ring, void *v_ring, const void *k_sink,
                                      const void *v_sink, int n_sink, const int64_t *q_start,
                                      const int64_t *chunk_len, void *out, float *lse, int B,
                                      int H, int Hkv, int64_t Tq, int d, int64_t W, float scale,
                                      int update_ring, void *workspace, size_t workspace_bytes,
                                      void *stream);

/*
 * swa_ring_write -- append a chunk of keys/values to a ring cache.
 * Passage: blog section 3.2 (slot = position mod W once the ring is full);
 * M003 note section 06 (update the position-to-slot map before reuse).
 * Writes rows t of k_new/v_new [B, Hkv, T, d] whose positions
 * q_start[b] + t are among the last W (q_start[b] + t >= q_start[b] + T - W)
 * into slot (q_start[b] + t) mod W of k_ring/v_ring [B, Hkv, W, d].
 */
SWA_API int swa_ring_write(const void *k_new, const void *v_new, void *k_ring, void *v_ring,
                   const int64_t *q_start, int B, int Hkv, int64_t T, int d, int64_t W,
                   void *stream);

/*
 * swa_decode_workspace_bytes -- bytes of scratch swa_attn_decode_ring and
 * swa_attn_decode_ring_sink need for these sizes (split partial results:
 * fp32 O, running max and sum; one spare partial per (b, h) for sinks).
 */
SWA_API size_t swa_decode_workspace_bytes(int B, int H, int Hkv, int d, int64_t W);

/*
 * swa_attn_decode_ring -- batched single-token decode from a ring cache.
 * Passage: blog section 3.2 (circular cache); sparse-attention taxonomy
 * page section 1 (a decode step is bound by reading the KV cache from HBM).
 *   q: [B, H, d] bf16, device: the query of sequence b at logical position
 *      pos[b]; its own key/value are already in slot pos[b] mod W.
 *   k_ring, v_ring: [B, Hkv, W, d] bf16, device: slot s holds the most
 *      recent position p <= pos[b] with p mod W == s (empty if none).
 *   pos: int64 [B], device (>= 0).   out: [B, H, d] bf16, device.
 *   lse: [B, H] fp32 or NULL.
 *   workspace: device scratch of at least swa_decode_workspace_bytes(...)
 *      bytes, caller-owned; contents on entry are ignored.
 * Each key/value slot is read from HBM once for all G query heads of its
 * group; the key range is split across CTAs and merged in a second kernel.
 */
SWA_API int swa_attn_decode_ring(const void *q, const void *k_ring, const void *v_ring,
                         const int64_t *pos, void *out, float *lse, int B, int H, int Hkv,
                         int d, int64_t W, float scale, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * swa_attn_decode_ring_sink -- swa_attn_decode_ring with attention sinks.
 * Passage: sparse-attention taxonomy page section 3.2 (StreamingLLM keeps the
 * first tokens visible besides the recent W).  The query at pos[b] reads key
 * j iff j <= pos[b] and (j >= pos[b] - W + 1 or j < n_sink): the last W
 * positions from the ring, the sinks before the window from k_sink/v_sink.
 *   k_sink, v_sink: [B, Hkv, n_sink, d] bf16, device: row j holds position j
 *      (written once by the caller, e.g. copied from the first chunk; rows
 *      j > pos[b] are never read).   1 <= n_sink <= 128.
 * Other arguments, layouts and limits as swa_attn_decode_ring; the same
 * workspace size applies.  One extra CTA per (b, kv head) reads the sinks.
 */
SWA_API int swa_attn_decode_ring_sink(const void *q, const void *k_ring, const void *v_ring,
                                      const void *k_sink, const void *v_sink, int n_sink,
                                      const int64_t *pos, void *out, float *lse, int B, int H,
                                      int Hkv, int d, int64_t W, float scale, void *workspace,
                                      size_t workspace_bytes, void *stream);

/*
 * swa_attn_decode_ring_static -- swa_attn_decode_ring without a workspace.
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device scratch (a plugin or foreign-language host with
 * no device allocator, or a process that reserved all free device memory up
 * front).  Same arguments, layouts and results as swa_attn_decode_ring; the
 * split partials live in a fixed 16 MiB (16777216-byte) device array that
 * every device loading the library keeps until exit.  Calls no allocator.
 *  - Returns SWA_ERR_WORKSPACE, before enqueuing anything, when
 *    swa_decode_workspace_bytes(B, H, Hkv, d, W) exceeds 16777216 bytes.
 *  - All calls on a device share the array (it keeps the last call's
 *    contents; nothing needs to start zeroed): calls whose kernels overlap on
 *    one device race and must be ordered on one stream or with events.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress with that device current) and caches it; make
 *    that first call before any stream capture.
 *  - The cached address lives as long as the device's primary context: a
 *    cudaDeviceReset() on that device (or anything else that destroys its
 *    primary context) frees the array and leaves the cached address stale,
 *    so a process that resets a device must not call this entry point on it
 *    again.
 */
SWA_API int swa_attn_decode_ring_static(const void *q, const void *k_ring, const void *v_ring,
                                        const int64_t *pos, void *out, float *lse, int B, int H,
                                        int Hkv, int d, int64_t W, float scale, void *stream);

/*
 * swa_ring_slot_positions -- the logical position held by every ring slot.
 * Passage: M003 note section 06 (logical vs physical slots); blog section 3.2.
 * For sequence b after positions 0 .. n_written[b]-1 were written:
 *   slot_pos[b, s] = the largest p < n_written[b] with p mod W == s, or -1.
 * n_written: int64 [B] device; slot_pos: int64 [B, W] device (written).
 */
SWA_API int swa_ring_slot_positions(int B, const int64_t *n_written, int64_t W, int64_t *slot_pos,
                            void *stream);

/*
 * swa_selftest_wait -- runs the bounded device wait that every kernel of
 * this library uses for failure detection, in a one-CTA kernel of its own
 * (no copies, no tensor memory), so that the timeout path can be checked
 * without breaking a real kernel.  The pages have no counterpart.
 * Every mbarrier wait in the attention kernels gives up after a time limit,
 * records SWA_ERR_TIMEOUT in the device status word and raises its CTA's
 * abort flag; the CTA's other waits then give up at once, every role stops
 * issuing work, copies and MMAs already issued are waited for, and the
 * kernel returns instead of hanging the GPU.
 *   limit_ns: 1000 .. 1000000000, the time limit of the first waiter.
 *   arrive:   0: nobody arrives on the barriers: the first waiter gives up
 *             after limit_ns, the 96 others follow through the abort flag,
 *             and the next swa_get_device_status() returns SWA_ERR_TIMEOUT.
 *             Nonzero: the barriers are arrived on before anyone waits, every
 *             wait succeeds and the status word is left alone.
 *   result:   int32 [5], device (written): result[w] for w = 0..3 counts the
 *             lanes of warp w whose wait succeeded (warp 0 has one waiting
 *             lane, warps 1-3 have 32 each); result[4] is the elapsed time
 *             of the waits in microseconds.
 */
SWA_API int swa_selftest_wait(int64_t limit_ns, int arrive, int32_t *result, void *stream);

/*
 * swa_get_device_status -- synchronise `stream`, then read and clear the
 * device status word of the current device: SWA_OK, SWA_ERR_TIMEOUT (a
 * device-side wait gave up; the kernel returned early and its outputs are
 * invalid) or SWA_ERR_DEVICE (a device-side argument check failed).
 * Returns SWA_ERR_CUDA if the synchronisation itself reports an error.
 */
SWA_API int swa_get_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
