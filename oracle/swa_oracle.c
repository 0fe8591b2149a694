/*
 * swa_oracle.c -- plain fp64 CPU oracle for causal sliding-window attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file; the library under
 * sliding_window_sparse_b200/ never links, imports or calls it.  It shares
 * no code, header, table or constant with the CUDA path.
 *
 * Everything here is deliberately slow and literal: loops over the allowed
 * (query, key) pairs only, fp64 arithmetic on the exact values of the bf16
 * inputs, a two-pass softmax (max, then sum of exponentials, then the
 * weighted sum of values), and a ring buffer that is simulated write by write.
 *
 * Sources (page title, section):
 *  [M003]  "AI infra KB M003: weight sparsity vs attention sparsity"
 *          (xuujii.github.io/ai-infra-kb), sections 03-08 (07-08: outputs and
 *          Q/K/V gradients checked under the same mask, by finite differences).
 *  [CH10]  "Chapter 10 -- local and sparse attention: SWA and DSA"
 *          (book.ozine.me, LLMs from scratch), sections 10.1, 10.2, 10.3, 10.6.
 *  [BLOG]  "Dense attention vs sparse sliding window attention"
 *          (maplevalley.com.cn news 3171860), section 3.2 (circular KV cache),
 *          section 5.2 tip 4 (per-sequence windows in packed batches).
 *  [TAXO]  "Sparse attention taxonomy: what to read, what not to read"
 *          (forceinjection.github.io, kv_cache concepts), section 3.2
 *          (StreamingLLM: the first 4 tokens plus the recent W).
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact value of a bfloat16 bit pattern. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* [M003 s03], [CH10 s10.1]: position i may look at key j iff
 * max(0, i - W + 1) <= j <= i  (the window includes the current token). */
static int allowed(int64_t i, int64_t j, int64_t W)
{
    return (j <= i) && (j >= i - W + 1) && (j >= 0);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Count allowed pairs among all N x N (query, key) positions by enumeration.
 * [M003 s03] gives 21 for N=8, W=3 and 36 for full causal. */
int64_t orc_count_pairs(int64_t N, int64_t W)
{
    int64_t n = 0;
    for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < N; ++j)
            n += allowed(i, j, W);
    return n;
}

/* Softmax attention of one query over an explicit list of keys
 * [M003 s03]: dot products on the listed pairs only, softmax normalised over
 * those pairs only, output = weighted sum of the listed values.
 * Two passes: the maximum score, then exponentials and sums.
 * Returns 0, or -1 when the list is empty (no legal key: [CH10 s10.3]). */
static int attend_one(const uint16_t *qrow, const uint16_t *const *krows,
                      const uint16_t *const *vrows, int64_t nkeys, int d,
                      double scale, double *out, double *lse, double *scores)
{
    if (nkeys <= 0) {
        for (int c = 0; c < d; ++c) out[c] = NAN;
        if (lse) *lse = NAN;
        return -1;
    }
    double smax = -INFINITY;
    for (int64_t t = 0; t < nkeys; ++t) {
        double s = 0.0;
        for (int c = 0; c < d; ++c)
            s += bf16_value(qrow[c]) * bf16_value(krows[t][c]);
        s *= scale;
        scores[t] = s;
        if (s > smax) smax = s;
    }
    double denom = 0.0;
    for (int64_t t = 0; t < nkeys; ++t) {
        scores[t] = exp(scores[t] - smax);
        denom += scores[t];
    }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int64_t t = 0; t < nkeys; ++t) {
        double w = scores[t] / denom;
        for (int c = 0; c < d; ++c)
            out[c] += w * bf16_value(vrows[t][c]);
    }
    if (lse) *lse = smax + log(denom);
    return 0;
}

/* Row list helper: row r of the request is (b, h, i); NULL = every row. */
static void row_of(const int64_t *rows, int64_t r, int H, int64_t n_q,
                   int64_t *b, int64_t *h, int64_t *i)
{
    if (rows) {
        *b = rows[3 * r];
        *h = rows[3 * r + 1];
        *i = rows[3 * r + 2];
    } else {
        *i = r % n_q;
        *h = (r / n_q) % H;
        *b = r / (n_q * H);
    }
}

/* Query head h reads key/value head h / (H / Hkv) (contiguous groups). */
static int64_t kv_head(int64_t h, int H, int Hkv) { return h / (H / Hkv); }

/*
 * Prefill forward on a linear layout.
 * q: [B, H, N, d]; k, v: [B, Hkv, N, d] (bf16 bits); query row i and key row j
 * sit at logical positions q_pos0[b] + i and j (q_pos0 == NULL means 0).
 * Keys: every j with allowed(q_pos0[b] + i, j, W) and j < N, in increasing j.
 * out: [n_rows, d] (or [B, H, N, d] when rows == NULL); lse optional.
 * Returns the number of rows that had no legal key (0 for valid inputs).
 */
int64_t orc_swa_forward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        int B, int H, int Hkv, int64_t N, int d, int64_t W,
                        double scale, const int64_t *q_pos0,
                        const int64_t *rows, int64_t n_rows,
                        double *out, double *lse)
{
    int64_t total = rows ? n_rows : (int64_t)B * H * N;
    int64_t bad = 0;
#pragma omp parallel reduction(+ : bad)
    {
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(N > 0 ? N : 1));
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(N > 0 ? N : 1));
        double *sc = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            int64_t b, h, i;
            row_of(rows, r, H, N, &b, &h, &i);
            int64_t pq = (q_pos0 ? q_pos0[b] : 0) + i;
            int64_t kh = kv_head(h, H, Hkv);
            int64_t n = 0;
            for (int64_t j = 0; j < N; ++j) {
                if (!allowed(pq, j, W)) continue;
                kr[n] = k + ((b * Hkv + kh) * N + j) * d;
                vr[n] = v + ((b * Hkv + kh) * N + j) * d;
                ++n;
            }
            const uint16_t *qrow = q + ((b * H + h) * N + i) * d;
            if (attend_one(qrow, kr, vr, n, d, scale, out + r * d, lse ? lse + r : NULL, sc))
                ++bad;
        }
        free(kr);
        free(vr);
        free(sc);
    }
    return bad;
}

/*
 * Dense baseline of [M003 s07]: the full N x N score table of each (b, h),
 * forbidden entries set to -inf with the difference convention of
 * [CH10 s10.1] (diff = t - j; forbidden iff diff < 0 or diff >= W), then a
 * row softmax over the whole table.  Positions are 0..N-1.  out: [B,H,N,d].
 */
int orc_dense_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int B, int H, int Hkv, int64_t N, int d, int64_t W,
                     double scale, double *out)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)(N * N));
    if (!S) return -1;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            int64_t kh = kv_head(h, H, Hkv);
            const uint16_t *Q = q + (b * H + h) * N * d;
            const uint16_t *K = k + (b * Hkv + kh) * N * d;
            const uint16_t *V = v + (b * Hkv + kh) * N * d;
            for (int64_t t = 0; t < N; ++t)
                for (int64_t j = 0; j < N; ++j) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c)
                        s += bf16_value(Q[t * d + c]) * bf16_value(K[j * d + c]);
                    int64_t diff = t - j;
                    S[t * N + j] = (diff < 0 || diff >= W) ? -INFINITY : s * scale;
                }
            for (int64_t t = 0; t < N; ++t) {
                double m = -INFINITY;
                for (int64_t j = 0; j < N; ++j)
                    if (S[t * N + j] > m) m = S[t * N + j];
                double z = 0.0;
                for (int64_t j = 0; j < N; ++j) {
                    S[t * N + j] = exp(S[t * N + j] - m);
                    z += S[t * N + j];
                }
                double *o = out + ((b * H + h) * N + t) * d;
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < N; ++j)
                        acc += S[t * N + j] * bf16_value(V[j * d + c]);
                    o[c] = acc / z;
                }
            }
        }
    free(S);
    return 0;
}

/*
 * Ring buffer of W slots, simulated write by write as [BLOG s3.2] describes:
 * while fewer than W entries are held, the next entry goes to slot
 * `len` and len grows; once full, it overwrites slot `start` and
 * start = (start + 1) % W.  Positions 0 .. n_written-1 are written in order.
 * slot_pos[s] receives the logical position held by slot s, or -1 if empty.
 */
void orc_ring_positions(int64_t n_written, int64_t W, int64_t *slot_pos)
{
    int64_t len = 0, start = 0;
    for (int64_t s = 0; s < W; ++s) slot_pos[s] = -1;
    for (int64_t p = 0; p < n_written; ++p) {
        int64_t slot;
        if (len < W) {
            slot = len;
            ++len;
        } else {
            slot = start;
            start = (start + 1) % W;
        }
        slot_pos[slot] = p;
    }
}

/* Slot holding logical position p, or -1 (linear scan of the simulated map). */
static int64_t find_slot(const int64_t *slot_pos, int64_t W, int64_t p)
{
    for (int64_t s = 0; s < W; ++s)
        if (slot_pos[s] == p) return s;
    return -1;
}

/*
 * Chunked prefill over a ring cache ([CH10 s10.2], [M003 s06]).
 * q: [B,H,Tq,d]; k_new, v_new: [B,Hkv,Tq,d]; ring_k, ring_v: [B,Hkv,W,d].
 * Before the call the ring of sequence b holds the positions < q_start[b]
 * written by the [BLOG s3.2] procedure; the chunk holds positions
 * q_start[b] .. q_start[b] + Tq - 1.  Query t sits at q_start[b] + t and
 * reads every legal logical position in increasing order: from the ring if
 * the position is < q_start[b], else from the chunk.  The union over a chunk
 * spans W + Tq - 1 positions ([CH10 s10.2]).
 * Returns the number of rows with a missing key or no legal key.
 */
int64_t orc_swa_chunk(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                      const uint16_t *ring_k, const uint16_t *ring_v, const int64_t *q_start,
                      int B, int H, int Hkv, int64_t Tq, int d, int64_t W, double scale,
                      const int64_t *rows, int64_t n_rows, double *out, double *lse)
{
    int64_t total = rows ? n_rows : (int64_t)B * H * Tq;
    int64_t bad = 0;
    int64_t *maps = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B * W));
    for (int64_t b = 0; b < B; ++b) orc_ring_positions(q_start[b], W, maps + b * W);
#pragma omp parallel reduction(+ : bad)
    {
        int64_t cap = W + Tq;
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        double *sc = (double *)malloc(sizeof(double) * (size_t)cap);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < total; ++r) {
            int64_t b, h, t;
            row_of(rows, r, H, Tq, &b, &h, &t);
            int64_t kh = kv_head(h, H, Hkv);
            int64_t p = q_start[b] + t;
            int64_t n = 0, missing = 0;
            int64_t lo = p - W + 1 < 0 ? 0 : p - W + 1;
            for (int64_t j = lo; j <= p; ++j) {
                if (j >= q_start[b]) {
                    int64_t row = j - q_start[b];
                    kr[n] = k_new + ((b * Hkv + kh) * Tq + row) * d;
                    vr[n] = v_new + ((b * Hkv + kh) * Tq + row) * d;
                } else {
                    int64_t s = find_slot(maps + b * W, W, j);
                    if (s < 0) { ++missing; continue; }
                    kr[n] = ring_k + ((b * Hkv + kh) * W + s) * d;
                    vr[n] = ring_v + ((b * Hkv + kh) * W + s) * d;
                }
                ++n;
            }
            const uint16_t *qrow = q + ((b * H + h) * Tq + t) * d;
            int e = attend_one(qrow, kr, vr, n, d, scale, out + r * d, lse ? lse + r : NULL, sc);
            if (e || missing) ++bad;
        }
        free(kr);
        free(vr);
        free(sc);
    }
    free(maps);
    return bad;
}

/*
 * Ring update after a chunk: continue the [BLOG s3.2] write procedure for
 * positions q_start[b] .. q_start[b] + Tq - 1, copying each chunk row into the
 * slot the procedure picks (in place on ring_k / ring_v).
 */
void orc_ring_update(const uint16_t *k_new, const uint16_t *v_new,
                     uint16_t *ring_k, uint16_t *ring_v, const int64_t *q_start,
                     int B, int Hkv, int64_t Tq, int d, int64_t W)
{
    for (int64_t b = 0; b < B; ++b) {
        int64_t len = 0, start = 0;
        for (int64_t p = 0; p < q_start[b] + Tq; ++p) {
            int64_t slot;
            if (len < W) {
                slot = len;
                ++len;
            } else {
                slot = start;
                start = (start + 1) % W;
            }
            if (p < q_start[b]) continue;
            int64_t row = p - q_start[b];
            for (int64_t kh = 0; kh < Hkv; ++kh) {
                memcpy(ring_k + ((b * Hkv + kh) * W + slot) * d,
                       k_new + ((b * Hkv + kh) * Tq + row) * d, sizeof(uint16_t) * (size_t)d);
                memcpy(ring_v + ((b * Hkv + kh) * W + slot) * d,
                       v_new + ((b * Hkv + kh) * Tq + row) * d, sizeof(uint16_t) * (size_t)d);
            }
        }
    }
}

/*
 * Decode from a ring: one query per sequence at logical position pos[b],
 * whose own key/value were already written, so the ring holds positions
 * 0 .. pos[b] written by the [BLOG s3.2] procedure.  The query reads every
 * legal position max(0, pos - W + 1) .. pos from the ring.
 * q: [B,H,d]; ring_k, ring_v: [B,Hkv,W,d]; out: [B,H,d]; lse: [B,H] optional.
 */
int64_t orc_swa_decode(const uint16_t *q, const uint16_t *ring_k, const uint16_t *ring_v,
                       const int64_t *pos, int B, int H, int Hkv, int d, int64_t W,
                       double scale, double *out, double *lse)
{
    int64_t bad = 0;
    int64_t *maps = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B * W));
    for (int64_t b = 0; b < B; ++b) orc_ring_positions(pos[b] + 1, W, maps + b * W);
#pragma omp parallel reduction(+ : bad)
    {
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)W);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)W);
        double *sc = (double *)malloc(sizeof(double) * (size_t)W);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < (int64_t)B * H; ++r) {
            int64_t b = r / H, h = r % H;
            int64_t kh = kv_head(h, H, Hkv);
            int64_t p = pos[b];
            int64_t lo = p - W + 1 < 0 ? 0 : p - W + 1;
            int64_t n = 0, missing = 0;
            for (int64_t j = lo; j <= p; ++j) {
                int64_t s = find_slot(maps + b * W, W, j);
                if (s < 0) { ++missing; continue; }
                kr[n] = ring_k + ((b * Hkv + kh) * W + s) * d;
                vr[n] = ring_v + ((b * Hkv + kh) * W + s) * d;
                ++n;
            }
            int e = attend_one(q + (b * H + h) * d, kr, vr, n, d, scale, out + r * d,
                               lse ? lse + r : NULL, sc);
            if (e || missing) ++bad;
        }
        free(kr);
        free(vr);
        free(sc);
    }
    free(maps);
    return bad;
}

/* [M003 s03] with StreamingLLM's sink rule ([TAXO s3.2], StreamingLLM:
 * the first S tokens stay visible besides the recent W): key j is visible to
 * position i iff j <= i and (j >= i - W + 1 or j < S).  S = 0 is allowed(). */
static int allowed_sink(int64_t i, int64_t j, int64_t W, int64_t S)
{
    return (j <= i) && (j >= 0) && (j >= i - W + 1 || j < S);
}

/* Pairs visible under allowed_sink among all N x N positions, by enumeration. */
int64_t orc_count_pairs_sink(int64_t N, int64_t W, int64_t S)
{
    int64_t n = 0;
    for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < N; ++j)
            n += allowed_sink(i, j, W, S);
    return n;
}

/*
 * Packed variable-length prefill ([BLOG s5.2] tip 4: batches of
 * different lengths packed along one token axis with cu_seqlens; the window
 * is applied within each sequence, never across a boundary).
 * q: [total, H, d]; k, v: [total, Hkv, d] (bf16 bits, token-major).
 * Sequence s holds tokens cu_seqlens[s] .. cu_seqlens[s+1] - 1, at positions
 * 0, 1, ...  Query token t of sequence s (position i = t - cu_seqlens[s])
 * reads the tokens cu_seqlens[s] + j with allowed_sink(i, j, W, n_sink), in
 * increasing j.
 * rows: pairs (t, h), or NULL for every (t, h) with h fastest.
 * out: [n_rows, d] (or [total, H, d]); lse: [n_rows] (or [total, H]), optional.
 * Returns the number of rows with no legal key, or -1 if cu_seqlens is not
 * non-decreasing from 0.
 */
int64_t orc_swa_varlen(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int64_t *cu_seqlens, int n_seq, int H, int Hkv, int d, int64_t W,
                       int64_t n_sink, double scale, const int64_t *rows, int64_t n_rows,
                       double *out, double *lse)
{
    if (cu_seqlens[0] != 0) return -1;
    int64_t longest = 0;
    for (int s = 0; s < n_seq; ++s) {
        int64_t len = cu_seqlens[s + 1] - cu_seqlens[s];
        if (len < 0) return -1;
        if (len > longest) longest = len;
    }
    int64_t total_tok = cu_seqlens[n_seq];
    int64_t total = rows ? n_rows : total_tok * H;
    int64_t bad = 0;
#pragma omp parallel reduction(+ : bad)
    {
        int64_t cap = longest > 0 ? longest : 1;
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        double *sc = (double *)malloc(sizeof(double) * (size_t)cap);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            int64_t t = rows ? rows[2 * r] : r / H;
            int64_t h = rows ? rows[2 * r + 1] : r % H;
            int s = 0;
            while (s + 1 < n_seq && cu_seqlens[s + 1] <= t) ++s;
            int64_t first = cu_seqlens[s], len = cu_seqlens[s + 1] - first;
            int64_t i = t - first, kh = kv_head(h, H, Hkv);
            int64_t n = 0;
            for (int64_t j = 0; j < len; ++j) {
                if (!allowed_sink(i, j, W, n_sink)) continue;
                kr[n] = k + ((first + j) * Hkv + kh) * d;
                vr[n] = v + ((first + j) * Hkv + kh) * d;
                ++n;
            }
            const uint16_t *qrow = q + (t * H + h) * d;
            if (attend_one(qrow, kr, vr, n, d, scale, out + r * d, lse ? lse + r : NULL, sc))
                ++bad;
        }
        free(kr);
        free(vr);
        free(sc);
    }
    return bad;
}

/*
 * Decode with attention sinks ([TAXO s3.2]).  The ring holds the recent
 * positions exactly as in orc_swa_decode; sink_k, sink_v: [B, Hkv, S, d] hold
 * positions 0 .. S-1, written once and never overwritten.  The query at
 * pos[b] reads every position j with allowed_sink(pos[b], j, W, S) in
 * increasing order: from the ring if j is one of the last W positions, else
 * (a sink outside the window) from the sink rows.
 * q: [B,H,d]; out: [B,H,d]; lse: [B,H] optional.
 */
int64_t orc_swa_decode_sink(const uint16_t *q, const uint16_t *ring_k, const uint16_t *ring_v,
                            const uint16_t *sink_k, const uint16_t *sink_v, const int64_t *pos,
                            int B, int H, int Hkv, int d, int64_t W, int64_t S, double scale,
                            double *out, double *lse)
{
    int64_t bad = 0;
    int64_t *maps = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B * W));
    for (int64_t b = 0; b < B; ++b) orc_ring_positions(pos[b] + 1, W, maps + b * W);
#pragma omp parallel reduction(+ : bad)
    {
        int64_t cap = W + S;
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        double *sc = (double *)malloc(sizeof(double) * (size_t)cap);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < (int64_t)B * H; ++r) {
            int64_t b = r / H, h = r % H;
            int64_t kh = kv_head(h, H, Hkv);
            int64_t p = pos[b];
            int64_t n = 0, missing = 0;
            for (int64_t j = 0; j <= p; ++j) {
                if (!allowed_sink(p, j, W, S)) continue;
                if (j >= p - W + 1) {
                    int64_t s = find_slot(maps + b * W, W, j);
                    if (s < 0) { ++missing; continue; }
                    kr[n] = ring_k + ((b * Hkv + kh) * W + s) * d;
                    vr[n] = ring_v + ((b * Hkv + kh) * W + s) * d;
                } else {
                    kr[n] = sink_k + ((b * Hkv + kh) * S + j) * d;
                    vr[n] = sink_v + ((b * Hkv + kh) * S + j) * d;
                }
                ++n;
            }
            int e = attend_one(q + (b * H + h) * d, kr, vr, n, d, scale, out + r * d,
                               lse ? lse + r : NULL, sc);
            if (e || missing) ++bad;
        }
        free(kr);
        free(vr);
        free(sc);
    }
    free(maps);
    return bad;
}

/*
 * Gradients of the prefill forward ([M003 s07]: check the Q/K/V gradients,
 * by finite differences, under the same mask as the output; [M003 s08]:
 * outputs and gradients with the same mask).  For the loss sum(out * dout):
 *   P_ij  = softmax over the allowed j of scale * <q_i, k_j>
 *   dP_ij = <dout_i, v_j>,   D_i = sum_j P_ij dP_ij,   dS_ij = P_ij (dP_ij - D_i)
 *   dq_i  = scale * sum_j dS_ij k_j
 *   dk_j  = scale * sum_i dS_ij q_i     (summed over the query heads of j's group)
 *   dv_j  = sum_i P_ij dout_i           (likewise)
 * q, dout: [B,H,N,d]; k, v: [B,Hkv,N,d], fp64 values (so that finite
 * differences can move them by less than a bf16 step); positions 0..N-1.
 * dq: [B,H,N,d], dk, dv: [B,Hkv,N,d] (fp64, overwritten).
 * Returns the number of query rows with no legal key (0 for valid inputs).
 */
int64_t orc_swa_backward(const double *q, const double *k, const double *v,
                         const double *dout, int B, int H, int Hkv, int64_t N, int d,
                         int64_t W, double scale, double *dq, double *dk, double *dv)
{
    int64_t bad = 0;
    memset(dq, 0, sizeof(double) * (size_t)(B * H * N * d));
    memset(dk, 0, sizeof(double) * (size_t)(B * Hkv * N * d));
    memset(dv, 0, sizeof(double) * (size_t)(B * Hkv * N * d));
    /* one (b, kv head) per iteration: its dk, dv rows are written by it alone */
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (int64_t bk = 0; bk < (int64_t)B * Hkv; ++bk) {
        int64_t b = bk / Hkv, kh = bk % Hkv;
        int64_t cap = N > 0 ? N : 1;
        double *p = (double *)malloc(sizeof(double) * (size_t)cap);
        double *dp = (double *)malloc(sizeof(double) * (size_t)cap);
        for (int64_t h = 0; h < H; ++h) {
            if (kv_head(h, H, Hkv) != kh) continue;
            for (int64_t i = 0; i < N; ++i) {
                const double *qi = q + ((b * H + h) * N + i) * d;
                const double *gi = dout + ((b * H + h) * N + i) * d;
                int64_t lo = i - W + 1 < 0 ? 0 : i - W + 1;
                if (lo > i) { ++bad; continue; }
                /* softmax weights over the allowed keys lo..i (two passes) */
                double smax = -INFINITY;
                for (int64_t j = lo; j <= i; ++j) {
                    const double *kj = k + ((b * Hkv + kh) * N + j) * d;
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += qi[c] * kj[c];
                    p[j - lo] = s * scale;
                    if (p[j - lo] > smax) smax = p[j - lo];
                }
                double denom = 0.0;
                for (int64_t j = lo; j <= i; ++j) {
                    p[j - lo] = exp(p[j - lo] - smax);
                    denom += p[j - lo];
                }
                double Di = 0.0;
                for (int64_t j = lo; j <= i; ++j) {
                    const double *vj = v + ((b * Hkv + kh) * N + j) * d;
                    p[j - lo] /= denom;
                    double g = 0.0;
                    for (int c = 0; c < d; ++c) g += gi[c] * vj[c];
                    dp[j - lo] = g;
                    Di += p[j - lo] * g;
                }
                double *dqi = dq + ((b * H + h) * N + i) * d;
                for (int64_t j = lo; j <= i; ++j) {
                    double ds = p[j - lo] * (dp[j - lo] - Di);
                    const double *kj = k + ((b * Hkv + kh) * N + j) * d;
                    double *dkj = dk + ((b * Hkv + kh) * N + j) * d;
                    double *dvj = dv + ((b * Hkv + kh) * N + j) * d;
                    for (int c = 0; c < d; ++c) {
                        dqi[c] += scale * ds * kj[c];
                        dkj[c] += scale * ds * qi[c];
                        dvj[c] += p[j - lo] * gi[c];
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
    return bad;
}

/*
 * The prefill forward of orc_swa_forward on fp64 inputs (positions 0..N-1):
 * the function whose finite differences pin orc_swa_backward.  Same loops:
 * scores on the allowed pairs, two-pass softmax, weighted sum of values.
 * q: [B,H,N,d]; k, v: [B,Hkv,N,d]; out: [B,H,N,d].
 */
int64_t orc_swa_forward_f64(const double *q, const double *k, const double *v, int B, int H,
                            int Hkv, int64_t N, int d, int64_t W, double scale, double *out)
{
    int64_t bad = 0;
#pragma omp parallel reduction(+ : bad)
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < (int64_t)B * H * N; ++r) {
            int64_t i = r % N, h = (r / N) % H, b = r / (N * H);
            int64_t kh = kv_head(h, H, Hkv);
            const double *qi = q + r * d;
            double *o = out + r * d;
            int64_t lo = i - W + 1 < 0 ? 0 : i - W + 1;
            if (lo > i) { ++bad; continue; }
            double smax = -INFINITY;
            for (int64_t j = lo; j <= i; ++j) {
                const double *kj = k + ((b * Hkv + kh) * N + j) * d;
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += qi[c] * kj[c];
                sc[j - lo] = s * scale;
                if (sc[j - lo] > smax) smax = sc[j - lo];
            }
            double denom = 0.0;
            for (int64_t j = lo; j <= i; ++j) {
                sc[j - lo] = exp(sc[j - lo] - smax);
                denom += sc[j - lo];
            }
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t j = lo; j <= i; ++j) {
                const double *vj = v + ((b * Hkv + kh) * N + j) * d;
                for (int c = 0; c < d; ++c) o[c] += sc[j - lo] / denom * vj[c];
            }
        }
        free(sc);
    }
    return bad;
}

/*
 * Chunked prefill over a ring cache with attention sinks ([CH10 s10.2] with
 * [TAXO s3.2]).  As orc_swa_chunk, and in addition sink_k, sink_v:
 * [B, Hkv, S, d] hold positions 0 .. S-1 (written once, never evicted).
 * Query t at position p = q_start[b] + t reads every position j with
 * allowed_sink(p, j, W, S) in increasing order: from the chunk if
 * j >= q_start[b], from the ring if it is one of the last W positions before
 * the chunk and inside the window, else (a sink before the window) from the
 * sink rows.  Returns the number of rows with a missing or no legal key.
 */
int64_t orc_swa_chunk_sink(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                           const uint16_t *ring_k, const uint16_t *ring_v,
                           const uint16_t *sink_k, const uint16_t *sink_v, int64_t S,
                           const int64_t *q_start, int B, int H, int Hkv, int64_t Tq, int d,
                           int64_t W, double scale, const int64_t *rows, int64_t n_rows,
                           double *out, double *lse)
{
    int64_t total = rows ? n_rows : (int64_t)B * H * Tq;
    int64_t bad = 0;
    int64_t *maps = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B * W));
    for (int64_t b = 0; b < B; ++b) orc_ring_positions(q_start[b], W, maps + b * W);
#pragma omp parallel reduction(+ : bad)
    {
        int64_t cap = W + Tq + S;
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
        double *sc = (double *)malloc(sizeof(double) * (size_t)cap);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < total; ++r) {
            int64_t b, h, t;
            row_of(rows, r, H, Tq, &b, &h, &t);
            int64_t kh = kv_head(h, H, Hkv);
            int64_t p = q_start[b] + t;
            int64_t n = 0, missing = 0;
            for (int64_t j = 0; j <= p; ++j) {
                if (!allowed_sink(p, j, W, S)) continue;
                if (j >= q_start[b]) {
                    int64_t row = j - q_start[b];
                    kr[n] = k_new + ((b * Hkv + kh) * Tq + row) * d;
                    vr[n] = v_new + ((b * Hkv + kh) * Tq + row) * d;
                } else if (j >= p - W + 1) {
                    int64_t s = find_slot(maps + b * W, W, j);
                    if (s < 0) { ++missing; continue; }
                    kr[n] = ring_k + ((b * Hkv + kh) * W + s) * d;
                    vr[n] = ring_v + ((b * Hkv + kh) * W + s) * d;
                } else {
                    kr[n] = sink_k + ((b * Hkv + kh) * S + j) * d;
                    vr[n] = sink_v + ((b * Hkv + kh) * S + j) * d;
                }
                ++n;
            }
            const uint16_t *qrow = q + ((b * H + h) * Tq + t) * d;
            int e = attend_one(qrow, kr, vr, n, d, scale, out + r * d, lse ? lse + r : NULL, sc);
            if (e || missing) ++bad;
        }
        free(kr);
        free(vr);
        free(sc);
    }
    free(maps);
    return bad;
}

/*
 * Tile classification by brute force ([M003 s04]): every in-range
 * (query, key) coordinate of a tile is tested with the visibility rule; a tile
 * whose in-range pairs are all forbidden is skipped (class 0), one whose
 * pairs are all allowed is fully visible (class 1), anything else is
 * partially visible (class 2).  Ragged last tiles are clipped to the
 * in-range coordinates.
 *
 * mode 0 (linear): query row i at position q_pos0[b] + i (q_pos0 NULL = 0),
 *   key column j at position j, 0 <= j < n_k.
 * mode 1 (ring + chunk): queries at q_start[b] + i (q_pos0 holds q_start);
 *   the key axis is the W ring slots in physical order, tiled on their own,
 *   followed by the n_q chunk keys at q_start[b] + t, tiled on their own
 *   (n_k is ignored).  Slot positions come from orc_ring_positions(q_start,
 *   W); an empty slot is never visible.
 *
 * classes: int8 [B, nqt, nkt] (may be NULL); ranges: int32 [B, nqt, 4] =
 * {live tiles, full tiles, first live tile, last live tile} (-1 if none).
 */
int orc_tile_classes(int mode, int B, int64_t n_q, int64_t n_k, const int64_t *q_pos0,
                     int64_t W, int tile_q, int tile_k, int8_t *classes, int32_t *ranges)
{
    int64_t nqt = (n_q + tile_q - 1) / tile_q;
    int64_t n_ring_t = mode == 1 ? (W + tile_k - 1) / tile_k : 0;
    int64_t n_key_cols = mode == 1 ? W + n_q : n_k;
    int64_t nkt = mode == 1 ? n_ring_t + (n_q + tile_k - 1) / tile_k : (n_k + tile_k - 1) / tile_k;
    int64_t *kpos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_key_cols > 0 ? n_key_cols : 1));
    for (int64_t b = 0; b < B; ++b) {
        int64_t p0 = q_pos0 ? q_pos0[b] : 0;
        /* position of every key column, -1 for a column that is never visible */
        if (mode == 1) {
            orc_ring_positions(p0, W, kpos);
            for (int64_t t = 0; t < n_q; ++t) kpos[W + t] = p0 + t;
        } else {
            for (int64_t j = 0; j < n_k; ++j) kpos[j] = j;
        }
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t qt = 0; qt < nqt; ++qt) {
            int32_t n_live = 0, n_full = 0, first = -1, last = -1;
            for (int64_t kt = 0; kt < nkt; ++kt) {
                int64_t c_begin, c_end;
                if (mode == 1 && kt < n_ring_t) {
                    c_begin = kt * tile_k;
                    c_end = c_begin + tile_k < W ? c_begin + tile_k : W;
                } else if (mode == 1) {
                    c_begin = W + (kt - n_ring_t) * tile_k;
                    c_end = c_begin + tile_k < W + n_q ? c_begin + tile_k : W + n_q;
                } else {
                    c_begin = kt * tile_k;
                    c_end = c_begin + tile_k < n_k ? c_begin + tile_k : n_k;
                }
                int64_t r_begin = qt * tile_q;
                int64_t r_end = r_begin + tile_q < n_q ? r_begin + tile_q : n_q;
                int64_t n_in = 0, n_ok = 0;
                for (int64_t i = r_begin; i < r_end; ++i)
                    for (int64_t c = c_begin; c < c_end; ++c) {
                        ++n_in;
                        if (kpos[c] >= 0 && allowed(p0 + i, kpos[c], W)) ++n_ok;
                    }
                int8_t cls = n_ok == 0 ? 0 : (n_ok == n_in ? 1 : 2);
                if (classes) classes[(b * nqt + qt) * nkt + kt] = cls;
                if (cls) {
                    ++n_live;
                    if (first < 0) first = (int32_t)kt;
                    last = (int32_t)kt;
                }
                if (cls == 1) ++n_full;
            }
            if (ranges) {
                int32_t *rr = ranges + (b * nqt + qt) * 4;
                rr[0] = n_live;
                rr[1] = n_full;
                rr[2] = first;
                rr[3] = last;
            }
        }
    }
    free(kpos);
    return 0;
}

/* cu_seqlens starts at 0 and never decreases; returns the longest sequence,
 * or -1 when malformed. */
static int64_t varlen_longest(const int64_t *cu_seqlens, int n_seq)
{
    if (cu_seqlens[0] != 0) return -1;
    int64_t longest = 0;
    for (int s = 0; s < n_seq; ++s) {
        int64_t len = cu_seqlens[s + 1] - cu_seqlens[s];
        if (len < 0) return -1;
        if (len > longest) longest = len;
    }
    return longest;
}

/*
 * Packed variable-length forward on fp64 inputs ([BLOG s5.2] tip 4, with the
 * sink rule of [TAXO s3.2]): the function whose finite differences pin
 * orc_swa_varlen_backward.  q, out: [total, H, d]; k, v: [total, Hkv, d].
 * Sequence s holds tokens cu_seqlens[s] .. cu_seqlens[s+1] - 1 at positions
 * 0, 1, ...; its token i reads the keys j of the same sequence with
 * allowed_sink(i, j, W, S), in increasing j (two-pass softmax as in
 * orc_swa_forward_f64).  Returns -1 for malformed cu_seqlens, else the number
 * of rows with no legal key.
 */
int64_t orc_swa_varlen_f64(const double *q, const double *k, const double *v,
                           const int64_t *cu_seqlens, int n_seq, int H, int Hkv, int d,
                           int64_t W, int64_t S, double scale, double *out)
{
    int64_t longest = varlen_longest(cu_seqlens, n_seq);
    if (longest < 0) return -1;
    int64_t bad = 0;
    double *sc = (double *)malloc(sizeof(double) * (size_t)(longest > 0 ? longest : 1));
    int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * (size_t)(longest > 0 ? longest : 1));
    for (int s = 0; s < n_seq; ++s) {
        int64_t first = cu_seqlens[s], len = cu_seqlens[s + 1] - first;
        for (int64_t h = 0; h < H; ++h) {
            int64_t kh = kv_head(h, H, Hkv);
            for (int64_t i = 0; i < len; ++i) {
                const double *qi = q + ((first + i) * H + h) * d;
                double *o = out + ((first + i) * H + h) * d;
                int64_t n = 0;
                for (int64_t j = 0; j < len; ++j)
                    if (allowed_sink(i, j, W, S)) idx[n++] = j;
                if (n == 0) { ++bad; continue; }
                double smax = -INFINITY;
                for (int64_t t = 0; t < n; ++t) {
                    const double *kj = k + ((first + idx[t]) * Hkv + kh) * d;
                    double x = 0.0;
                    for (int c = 0; c < d; ++c) x += qi[c] * kj[c];
                    sc[t] = x * scale;
                    if (sc[t] > smax) smax = sc[t];
                }
                double denom = 0.0;
                for (int64_t t = 0; t < n; ++t) {
                    sc[t] = exp(sc[t] - smax);
                    denom += sc[t];
                }
                for (int c = 0; c < d; ++c) o[c] = 0.0;
                for (int64_t t = 0; t < n; ++t) {
                    const double *vj = v + ((first + idx[t]) * Hkv + kh) * d;
                    for (int c = 0; c < d; ++c) o[c] += sc[t] / denom * vj[c];
                }
            }
        }
    }
    free(sc);
    free(idx);
    return bad;
}

/*
 * Gradients of the packed variable-length forward, sinks included ([M003
 * s07-s08]: Q/K/V gradients under the same mask as the output; the mask is
 * that of orc_swa_varlen_f64).  For the loss sum(out * dout), per sequence:
 *   P_ij  = softmax over the visible j of scale * <q_i, k_j>
 *   dP_ij = <dout_i, v_j>,   D_i = sum_j P_ij dP_ij,   dS_ij = P_ij (dP_ij - D_i)
 *   dq_i  = scale * sum_j dS_ij k_j
 *   dk_j  = scale * sum_i dS_ij q_i   (over the query heads of j's group)
 *   dv_j  = sum_i P_ij dout_i         (likewise)
 * q, dout, dq: [total, H, d]; k, v, dk, dv: [total, Hkv, d]; fp64.
 * Returns -1 for malformed cu_seqlens, else the number of rows with no legal key.
 */
int64_t orc_swa_varlen_backward(const double *q, const double *k, const double *v,
                                const double *dout, const int64_t *cu_seqlens, int n_seq,
                                int H, int Hkv, int d, int64_t W, int64_t S, double scale,
                                double *dq, double *dk, double *dv)
{
    int64_t longest = varlen_longest(cu_seqlens, n_seq);
    if (longest < 0) return -1;
    int64_t total = cu_seqlens[n_seq];
    memset(dq, 0, sizeof(double) * (size_t)(total * H * d));
    memset(dk, 0, sizeof(double) * (size_t)(total * Hkv * d));
    memset(dv, 0, sizeof(double) * (size_t)(total * Hkv * d));
    int64_t bad = 0;
    int64_t cap = longest > 0 ? longest : 1;
    double *p = (double *)malloc(sizeof(double) * (size_t)cap);
    double *dp = (double *)malloc(sizeof(double) * (size_t)cap);
    int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
    for (int s = 0; s < n_seq; ++s) {
        int64_t first = cu_seqlens[s], len = cu_seqlens[s + 1] - first;
        for (int64_t h = 0; h < H; ++h) {
            int64_t kh = kv_head(h, H, Hkv);
            for (int64_t i = 0; i < len; ++i) {
                const double *qi = q + ((first + i) * H + h) * d;
                const double *gi = dout + ((first + i) * H + h) * d;
                int64_t n = 0;
                for (int64_t j = 0; j < len; ++j)
                    if (allowed_sink(i, j, W, S)) idx[n++] = j;
                if (n == 0) { ++bad; continue; }
                double smax = -INFINITY;
                for (int64_t t = 0; t < n; ++t) {
                    const double *kj = k + ((first + idx[t]) * Hkv + kh) * d;
                    double x = 0.0;
                    for (int c = 0; c < d; ++c) x += qi[c] * kj[c];
                    p[t] = x * scale;
                    if (p[t] > smax) smax = p[t];
                }
                double denom = 0.0;
                for (int64_t t = 0; t < n; ++t) {
                    p[t] = exp(p[t] - smax);
                    denom += p[t];
                }
                double Di = 0.0;
                for (int64_t t = 0; t < n; ++t) {
                    const double *vj = v + ((first + idx[t]) * Hkv + kh) * d;
                    p[t] /= denom;
                    double g = 0.0;
                    for (int c = 0; c < d; ++c) g += gi[c] * vj[c];
                    dp[t] = g;
                    Di += p[t] * g;
                }
                double *dqi = dq + ((first + i) * H + h) * d;
                for (int64_t t = 0; t < n; ++t) {
                    double ds = p[t] * (dp[t] - Di);
                    int64_t row = (first + idx[t]) * Hkv + kh;
                    const double *kj = k + row * d;
                    for (int c = 0; c < d; ++c) {
                        dqi[c] += scale * ds * kj[c];
                        dk[row * d + c] += scale * ds * qi[c];
                        dv[row * d + c] += p[t] * gi[c];
                    }
                }
            }
        }
    }
    free(p);
    free(dp);
    free(idx);
    return bad;
}
