/*
 * swa_oracle.c -- plain, slow, fp64 CPU reference for sliding-window GQA
 * attention and the rolling-buffer KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links,
 * loads or calls this file; only the tests, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA kernels.
 *
 * Sources (pages on the Mistral 7B paper, arXiv:2310.06825):
 *  [P1] "Mistral 7B -- Sliding Window Attention" summary
 *       (irregular6612.github.io): section "핵심 구성요소" (SWA mask
 *       mask[i,j] = 1 for (i-W) <= j <= i, causal), section "Rolling Buffer KV
 *       Cache 동작 설명" (write slot = p mod W; a query at p reads positions
 *       [p-W+1, p]), section "Pre-fill과의 상호작용" (chunks are pre-filled in
 *       order, the buffer keeps the last W entries, decode continues from it).
 *  [P2] review at manon006.tistory.com/118: section 3.3 (position i stored at
 *       i mod W, older entries overwritten), section 4.1 and Figure 3 (a chunk
 *       attends causally to itself and, through the cache, to the window).
 *  [P4] "Mistral 7B: Engineering Extreme Efficiency in LLMs"
 *       (flashpapers.ai): section 1 (GQA: query heads grouped, each group
 *       shares one K/V head; 32 query heads, 8 KV heads), section 2 (the SWA
 *       equation h_i = Attention(q_i, {k_j, v_j}) over a window of size W
 *       behind i), section 3 (rolling buffer, i mod W), section 4 (pre-fill
 *       and chunking: attention over the current chunk and the active cache).
 *
 * Readings taken where the sources above are loose or disagree:
 *  - window: query i sees keys j with i-W < j <= i (W keys, itself included).
 *    The other printed reading, i-W <= j <= i (W+1 keys), is window_mode 1.
 *  - GQA grouping is contiguous: query head h uses KV head h / (Hq/Hkv).
 *  - softmax is the standard exp-normalised form; the scale is an argument.
 *  - chunked pre-fill attends first, then writes the chunk into the buffer.
 *  - decode appends the new token first, then attends.
 *
 * Every computation is the definition written out: gather the key set of one
 * query row, score every key, subtract the maximum, exponentiate, normalise,
 * take the weighted sum of values.  All arithmetic is in double.  Rows are
 * independent, so OpenMP splits rows over threads; nothing else is reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_WINDOW_EXCL_LEFT 0 /* keys j with i-W <  j <= i */
#define ORACLE_WINDOW_INCL_LEFT 1 /* keys j with i-W <= j <= i */

/* Is key position j inside the causal window of query position i? [P1]
 * "핵심 구성요소", [P4] section 2. */
static int in_window(long i, long j, long W, int mode)
{
    if (j > i) return 0;                       /* causal: j <= i */
    if (mode == ORACLE_WINDOW_INCL_LEFT) return j >= i - W;
    return j > i - W;
}

/* Softmax attention of one query row q[D] over nk keys.  krows[t] and
 * vrows[t] point at the t-th key / value vector (length D).  scores is
 * caller scratch of length >= nk.  Writes out[D].  This is the plain
 * definition: s_t = scale * <q, k_t>; m = max s; p_t = exp(s_t - m);
 * out = sum p_t v_t / sum p_t.  Returns the normaliser sum p_t. */
static double attend_row(const double *q, const double *const *krows,
                         const double *const *vrows, long nk, int D,
                         double scale, double *scores, double *out)
{
    double m = -INFINITY;
    for (long t = 0; t < nk; ++t) {
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += q[d] * krows[t][d];
        s *= scale;
        scores[t] = s;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (long t = 0; t < nk; ++t) {
        double p = exp(scores[t] - m);
        l += p;
        for (int d = 0; d < D; ++d) out[d] += p * vrows[t][d];
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
    return l;
}

/* One-shot sliding-window GQA attention over a whole prompt.
 *   q, out : [B, N, Hq, D]      k, v : [B, N, Hkv, D]   (row-major, double)
 *   rows   : if non-NULL, the nrows query positions to compute (ascending or
 *            not); out is then [B, nrows, Hq, D].  If NULL, every position
 *            0..N-1 is computed and out is [B, N, Hq, D].
 * Query head h of batch b at position i attends to the keys of KV head
 * h / (Hq/Hkv) at positions j inside the window of i ([P1] "핵심 구성요소",
 * [P4] sections 1 and 2).  Returns 0, or -1 on bad arguments. */
int oracle_swa_prefill(const double *q, const double *k, const double *v,
                       double *out, int B, int N, int Hq, int Hkv, int D,
                       int W, double scale, int mode, const int64_t *rows,
                       int64_t nrows)
{
    if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || D < 1 || W < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const int64_t nr = rows ? nrows : N;
    const int64_t total = (int64_t)B * nr * Hq;
    int bad = 0;
#pragma omp parallel
    {
        const double **kr = malloc(sizeof(double *) * (size_t)N);
        const double **vr = malloc(sizeof(double *) * (size_t)N);
        double *sc = malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            const int h = (int)(r % Hq);
            const int64_t ri = (r / Hq) % nr;
            const int b = (int)(r / ((int64_t)Hq * nr));
            const long i = rows ? (long)rows[ri] : (long)ri;
            if (i < 0 || i >= N) { bad = 1; continue; }
            const int g = h / G;
            long nk = 0;
            for (long j = 0; j <= i; ++j) {
                if (!in_window(i, j, W, mode)) continue;
                kr[nk] = k + (((size_t)b * N + j) * Hkv + g) * D;
                vr[nk] = v + (((size_t)b * N + j) * Hkv + g) * D;
                ++nk;
            }
            const double *qr = q + (((size_t)b * N + i) * Hq + h) * D;
            double *o = out + (((size_t)b * nr + ri) * Hq + h) * D;
            attend_row(qr, kr, vr, nk, D, scale, sc, o);
        }
        free(kr); free(vr); free(sc);
    }
    return bad ? -1 : 0;
}

/* Rotary position embedding, in place (the pages give only its base:
 * "RoPE theta=10000" in Table 1 of [P1] "Methods").  Adopted reading: the
 * rotary embedding of Su et al. (RoFormer) in its original pairing, adjacent
 * elements (2i, 2i+1) form a pair rotated by the angle p * theta^(-2i/D):
 *   (x0, x1) -> (x0 cos a - x1 sin a, x0 sin a + x1 cos a).
 * x : [B, T, H, D] doubles, position of row (b, t) = pos[b] + t. */
int oracle_rope(double *x, const int32_t *pos, int B, int T, int H, int D, double theta)
{
    if (B < 1 || T < 1 || H < 1 || D < 2 || (D & 1) || !(theta > 1.0)) return -1;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const double p = (double)pos[b] + t;
            for (int h = 0; h < H; ++h) {
                double *row = x + (((size_t)b * T + t) * H + h) * D;
                for (int i = 0; i < D / 2; ++i) {
                    const double a = p * pow(theta, -2.0 * i / D);
                    const double c = cos(a), s = sin(a);
                    const double x0 = row[2 * i], x1 = row[2 * i + 1];
                    row[2 * i] = x0 * c - x1 * s;
                    row[2 * i + 1] = x0 * s + x1 * c;
                }
            }
        }
    return 0;
}

/* Rolling-buffer write ([P1] "Rolling Buffer KV Cache 동작 설명", write step;
 * [P2] section 3.3; [P4] section 3): for every sequence b and every new token
 * t, position p = pos[b] + t goes to slot p mod W.  The bytes are copied
 * unchanged (elem_bytes per element).  slot_pos [B, W] records which logical
 * position each slot holds (-1 = empty); it may be NULL.
 *   k_cache, v_cache : [B, W, Hkv, D]   k_new, v_new : [B, T, Hkv, D]  */
int oracle_cache_append(void *k_cache, void *v_cache, int32_t *slot_pos,
                        const void *k_new, const void *v_new,
                        const int32_t *pos, int B, int T, int Hkv, int D,
                        int W, int elem_bytes)
{
    if (B < 1 || T < 0 || Hkv < 1 || D < 1 || W < 1 || elem_bytes < 1) return -1;
    const size_t row = (size_t)Hkv * D * elem_bytes;
    for (int b = 0; b < B; ++b) {
        if (pos[b] < 0) return -1;
        for (int t = 0; t < T; ++t) {
            const long p = (long)pos[b] + t;
            const long slot = p % W;
            memcpy((char *)k_cache + ((size_t)b * W + slot) * row,
                   (const char *)k_new + ((size_t)b * T + t) * row, row);
            memcpy((char *)v_cache + ((size_t)b * W + slot) * row,
                   (const char *)v_new + ((size_t)b * T + t) * row, row);
            if (slot_pos) slot_pos[(size_t)b * W + slot] = (int32_t)p;
        }
    }
    return 0;
}

/* The slot -> logical position map of a buffer into which positions
 * 0 .. count[b]-1 have been written in order, one at a time, by the write
 * rule above.  Plain simulation of the writes. slot_pos : [B, W]. */
int oracle_slot_positions(const int32_t *count, int B, int W, int32_t *slot_pos)
{
    if (B < 1 || W < 1) return -1;
    for (int b = 0; b < B; ++b) {
        for (int s = 0; s < W; ++s) slot_pos[(size_t)b * W + s] = -1;
        for (long p = 0; p < count[b]; ++p) slot_pos[(size_t)b * W + p % W] = (int32_t)p;
    }
    return 0;
}

/* Chunked pre-fill attention ([P1] "Pre-fill과의 상호작용" and the chunking
 * item of "핵심 구성요소"; [P2] section 4.1, Figure 3; [P4] section 4).
 * The chunk holds positions s0 .. s0+C-1 (s0 = start_pos[b]).  Query
 * s0+t attends to
 *   - every cache entry whose recorded position p satisfies p <= s0-1 and
 *     lies inside the window of s0+t, and
 *   - the chunk's own keys s0+t' with t' <= t (causal inside the chunk),
 *     also restricted to the window.
 * The cache is read as it was before this chunk is written (attend, then
 * write; the write is a separate oracle_cache_append call).
 *   q, out : [B, C, Hq, D]   k, v : [B, C, Hkv, D]
 *   k_cache, v_cache : [B, W, Hkv, D]   slot_pos : [B, W] */
int oracle_swa_chunk(const double *q, const double *k, const double *v,
                     const double *k_cache, const double *v_cache,
                     const int32_t *slot_pos, const int32_t *start_pos,
                     double *out, int B, int C, int Hq, int Hkv, int D, int W,
                     double scale, int mode)
{
    if (B < 1 || C < 1 || Hq < 1 || Hkv < 1 || D < 1 || W < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const int64_t total = (int64_t)B * C * Hq;
#pragma omp parallel
    {
        const size_t cap = (size_t)W + (size_t)C;
        const double **kr = malloc(sizeof(double *) * cap);
        const double **vr = malloc(sizeof(double *) * cap);
        double *sc = malloc(sizeof(double) * cap);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            const int h = (int)(r % Hq);
            const int t = (int)((r / Hq) % C);
            const int b = (int)(r / ((int64_t)Hq * C));
            const int g = h / G;
            const long s0 = start_pos[b];
            const long i = s0 + t;
            long nk = 0;
            for (int s = 0; s < W; ++s) {
                const long p = slot_pos[(size_t)b * W + s];
                if (p < 0 || p > s0 - 1) continue;
                if (!in_window(i, p, W, mode)) continue;
                kr[nk] = k_cache + (((size_t)b * W + s) * Hkv + g) * D;
                vr[nk] = v_cache + (((size_t)b * W + s) * Hkv + g) * D;
                ++nk;
            }
            for (int tp = 0; tp <= t; ++tp) {
                if (!in_window(i, s0 + tp, W, mode)) continue;
                kr[nk] = k + (((size_t)b * C + tp) * Hkv + g) * D;
                vr[nk] = v + (((size_t)b * C + tp) * Hkv + g) * D;
                ++nk;
            }
            const double *qr = q + (((size_t)b * C + t) * Hq + h) * D;
            double *o = out + (((size_t)b * C + t) * Hq + h) * D;
            attend_row(qr, kr, vr, nk, D, scale, sc, o);
        }
        free(kr); free(vr); free(sc);
    }
    return 0;
}

/* Single-token decode against the rolling buffer ([P1] "Rolling Buffer KV
 * Cache 동작 설명": write slot p mod W, then the query at p reads positions
 * [p-W+1, p]).  The new token (position pos[b]) must already have been
 * appended.  Query head h attends to every cache entry of KV head
 * h / (Hq/Hkv) whose recorded position lies inside the window of pos[b].
 *   q, out : [B, Hq, D]   k_cache, v_cache : [B, W, Hkv, D]
 *   slot_pos : [B, W]    pos : [B] */
int oracle_swa_decode(const double *q, const double *k_cache,
                      const double *v_cache, const int32_t *slot_pos,
                      const int32_t *pos, double *out, int B, int Hq, int Hkv,
                      int D, int W, double scale, int mode)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || W < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq;
#pragma omp parallel
    {
        const double **kr = malloc(sizeof(double *) * (size_t)W);
        const double **vr = malloc(sizeof(double *) * (size_t)W);
        double *sc = malloc(sizeof(double) * (size_t)W);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < total; ++r) {
            const int h = (int)(r % Hq);
            const int b = (int)(r / Hq);
            const int g = h / G;
            const long p = pos[b];
            long nk = 0;
            for (int s = 0; s < W; ++s) {
                const long ps = slot_pos[(size_t)b * W + s];
                if (ps < 0) continue;
                if (!in_window(p, ps, W, mode)) continue;
                kr[nk] = k_cache + (((size_t)b * W + s) * Hkv + g) * D;
                vr[nk] = v_cache + (((size_t)b * W + s) * Hkv + g) * D;
                ++nk;
            }
            const double *qr = q + ((size_t)b * Hq + h) * D;
            double *o = out + ((size_t)b * Hq + h) * D;
            attend_row(qr, kr, vr, nk, D, scale, sc, o);
        }
        free(kr); free(vr); free(sc);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Attention sinks ([P3] aionda.blog "LLM 추론용 SWA ...", sections "왜 단순
 * sliding window만으로는 부족한가" and "추론 레이어 SWA가 주는 실용성": keep
 * the key/values of the first few tokens -- four suffice -- besides the
 * recent window; the middle is dropped).  Adopted reading: query i sees the
 * keys of its window (i-W < j <= i) and, in addition, positions j < S
 * (j <= i), each key once.
 * ---------------------------------------------------------------------- */

/* One-shot prefill with S sink positions.  Same layout as
 * oracle_swa_prefill. */
int oracle_swa_prefill_sinks(const double *q, const double *k, const double *v,
                             double *out, int B, int N, int Hq, int Hkv, int D,
                             int W, int S, double scale, const int64_t *rows,
                             int64_t nrows)
{
    if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || D < 1 || W < 1 || S < 0) return -1;
    if (Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const int64_t nr = rows ? nrows : N;
    const int64_t total = (int64_t)B * nr * Hq;
    int bad = 0;
#pragma omp parallel
    {
        const double **kr = malloc(sizeof(double *) * (size_t)N);
        const double **vr = malloc(sizeof(double *) * (size_t)N);
        double *sc = malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            const int h = (int)(r % Hq);
            const int64_t ri = (r / Hq) % nr;
            const int b = (int)(r / ((int64_t)Hq * nr));
            const long i = rows ? (long)rows[ri] : (long)ri;
            if (i < 0 || i >= N) { bad = 1; continue; }
            const int g = h / G;
            long nk = 0;
            for (long j = 0; j <= i; ++j) {
                if (!(in_window(i, j, W, ORACLE_WINDOW_EXCL_LEFT) || j < S)) continue;
                kr[nk] = k + (((size_t)b * N + j) * Hkv + g) * D;
                vr[nk] = v + (((size_t)b * N + j) * Hkv + g) * D;
                ++nk;
            }
            const double *qr = q + (((size_t)b * N + i) * Hq + h) * D;
            double *o = out + (((size_t)b * nr + ri) * Hq + h) * D;
            attend_row(qr, kr, vr, nk, D, scale, sc, o);
        }
        free(kr); free(vr); free(sc);
    }
    return bad ? -1 : 0;
}

/* Sink buffer write: new tokens whose position p is below S are also stored
 * at sink slot p.  k_sink, v_sink : [B, S, Hkv, D]; k_new, v_new :
 * [B, T, Hkv, D] (bytes copied unchanged). */
int oracle_sink_append(void *k_sink, void *v_sink, const void *k_new,
                       const void *v_new, const int32_t *pos, int B, int T,
                       int Hkv, int D, int S, int elem_bytes)
{
    if (B < 1 || T < 0 || Hkv < 1 || D < 1 || S < 0 || elem_bytes < 1) return -1;
    const size_t row = (size_t)Hkv * D * elem_bytes;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const long p = (long)pos[b] + t;
            if (p < 0) return -1;
            if (p >= S) continue;
            memcpy((char *)k_sink + ((size_t)b * S + p) * row,
                   (const char *)k_new + ((size_t)b * T + t) * row, row);
            memcpy((char *)v_sink + ((size_t)b * S + p) * row,
                   (const char *)v_new + ((size_t)b * T + t) * row, row);
        }
    return 0;
}

/* Decode with sinks: the keys of the window come from the rolling buffer
 * (recorded positions in (p-W, p]); sink positions j < S that fell out of the
 * window (j <= p-W) come from the sink buffer, which holds position j at
 * slot j. */
int oracle_swa_decode_sinks(const double *q, const double *k_cache,
                            const double *v_cache, const int32_t *slot_pos,
                            const double *k_sink, const double *v_sink,
                            const int32_t *pos, double *out, int B, int Hq,
                            int Hkv, int D, int W, int S, double scale)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || W < 1 || S < 0) return -1;
    if (Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq;
#pragma omp parallel
    {
        const size_t cap = (size_t)W + (size_t)S;
        const double **kr = malloc(sizeof(double *) * cap);
        const double **vr = malloc(sizeof(double *) * cap);
        double *sc = malloc(sizeof(double) * cap);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < total; ++r) {
            const int h = (int)(r % Hq);
            const int b = (int)(r / Hq);
            const int g = h / G;
            const long p = pos[b];
            long nk = 0;
            for (int s = 0; s < W; ++s) {
                const long ps = slot_pos[(size_t)b * W + s];
                if (ps < 0 || !in_window(p, ps, W, ORACLE_WINDOW_EXCL_LEFT)) continue;
                kr[nk] = k_cache + (((size_t)b * W + s) * Hkv + g) * D;
                vr[nk] = v_cache + (((size_t)b * W + s) * Hkv + g) * D;
                ++nk;
            }
            for (long j = 0; j < S && j <= p - W; ++j) {
                kr[nk] = k_sink + (((size_t)b * S + j) * Hkv + g) * D;
                vr[nk] = v_sink + (((size_t)b * S + j) * Hkv + g) * D;
                ++nk;
            }
            const double *qr = q + ((size_t)b * Hq + h) * D;
            double *o = out + ((size_t)b * Hq + h) * D;
            attend_row(qr, kr, vr, nk, D, scale, sc, o);
        }
        free(kr); free(vr); free(sc);
    }
    return 0;
}
