/*
 * Orthrus dual-view decode step: the CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the package smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * Everything here is the plain definition written out, in double precision,
 * with no blocking, fusion or reordering beyond what the definition states:
 *
 *   - attention (both views): textbook masked softmax attention, two passes
 *     (max, then exponentials), for each (sequence b, block slot i, query head h).
 *     Source: "Orthrus: Memory-Efficient Parallel Token Generation via Dual-View
 *     Diffusion" (gist.science technical summary), section 2.2, mask M_diff
 *     rules 1-2 (block queries see the clean context causally and the whole block
 *     bidirectionally), and section 2.3 "structural verification" (the frozen AR
 *     head sees the filled block causally).
 *   - consensus: same page, section 2.3 "consensus and commitment": strict
 *     left-to-right; a proposal is accepted only while it equals the AR greedy
 *     token; at the first mismatch the AR token replaces it.
 *   - commit: same section: keep the synchronised prefix, drop the rest of the
 *     block (rollback is truncation of the cache length).
 *
 * Readings where the pages are silent (listed with the design notes):
 *   softmax scale 1/sqrt(D) when scale <= 0; query head h reads KV head h/G
 *   (contiguous grouping); argmax ties go to the lowest index, NaN ranks above
 *   every number and the first NaN wins; accepted length a counts matching
 *   proposals (0..K); committed rows n = min(a+1, K); next anchor = AR greedy
 *   token at slot min(a, K-1).
 *
 * Layouts (row-major, element strides implied):
 *   q        [B, K, Hq, D]        float (bf16 inputs are exact in float)
 *   k_cache  [B, Hkv, S_max, D]   float; rows [ctx_b, ctx_b+K) hold the block
 *   v_cache  [B, Hkv, S_max, D]   float
 *   out      [B, K, Hq, D]        double   (or [n_rows, D] for a row subset)
 *   logits   [B, K, V]            float
 *   proposed [B, K]               int32
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_DIFF 0
#define ORACLE_AR 1

/* Number of keys query slot i of sequence b may look at.
 * DIFF (M_diff): the whole context [0, C) and the whole block [C, C+K).
 * AR (causal verification): positions [0, C+i]. */
static long visible_keys(int view, long ctx, int K, int i)
{
    return view == ORACLE_DIFF ? ctx + K : ctx + i + 1;
}

/* One output row: out = sum_j softmax_j(scale * <q, k_j>) v_j over j < n. */
static int attend_row(const float *q, const float *kc, const float *vc, int D,
                      long n, double scale, double *out)
{
    double *s = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    if (!s) return -1;
    double m = -INFINITY;
    for (long j = 0; j < n; ++j) {
        const float *kj = kc + (size_t)j * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += (double)q[d] * (double)kj[d];
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (long j = 0; j < n; ++j) {
        double w = exp(s[j] - m);
        l += w;
        const float *vj = vc + (size_t)j * D;
        for (int d = 0; d < D; ++d) out[d] += w * (double)vj[d];
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
    free(s);
    return 0;
}

/*
 * Dual-view attention.  rows == NULL computes every (b, i, h) into out laid out
 * [B, K, Hq, D]; otherwise rows holds n_rows triples (b, i, h) and out is
 * [n_rows, D].  Returns 0, or -1 on a bad argument / capacity violation.
 */
int oracle_attn(int view, int B, int Hq, int Hkv, int D, int S_max, int K,
                const int32_t *ctx_lens, const float *q, const float *k_cache,
                const float *v_cache, double scale, int n_rows,
                const int32_t *rows, double *out, int n_threads)
{
    if (view != ORACLE_DIFF && view != ORACLE_AR) return -1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || K <= 0 || Hq % Hkv) return -1;
    for (int b = 0; b < B; ++b)
        if (ctx_lens[b] < 0 || (long)ctx_lens[b] + K > S_max) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    const int G = Hq / Hkv;
    const long total = rows ? (long)n_rows : (long)B * K * Hq;
    int err = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 4) reduction(| : err)
    for (long r = 0; r < total; ++r) {
        int b, i, h;
        if (rows) {
            b = rows[3 * r]; i = rows[3 * r + 1]; h = rows[3 * r + 2];
            if (b < 0 || b >= B || i < 0 || i >= K || h < 0 || h >= Hq) { err |= 1; continue; }
        } else {
            h = (int)(r % Hq); i = (int)((r / Hq) % K); b = (int)(r / ((long)Hq * K));
        }
        const int g = h / G;
        const float *qr = q + (((size_t)b * K + i) * Hq + h) * D;
        const float *kc = k_cache + ((size_t)b * Hkv + g) * S_max * D;
        const float *vc = v_cache + ((size_t)b * Hkv + g) * S_max * D;
        long n = visible_keys(view, ctx_lens[b], K, i);
        if (attend_row(qr, kc, vc, D, n, scale, out + (size_t)r * D)) err |= 1;
    }
    return err ? -1 : 0;
}

/* The argmax order: NaN above every number, first occurrence wins ties. */
static int ranks_above(float x, float best)
{
    if (isnan(best)) return 0;
    if (isnan(x)) return 1;
    return x > best;
}

/*
 * Greedy consensus.  argmax_out (may be NULL) receives r[b, i].
 * accepted[b] = first i with proposed[b,i] != r[b,i], else K.
 * next_token[b] = r[b, min(accepted[b], K-1)].
 */
void oracle_consensus(int B, int K, int V, const float *logits,
                      const int32_t *proposed, int32_t *accepted,
                      int32_t *next_token, int32_t *argmax_out)
{
    int32_t *r = (int32_t *)malloc((size_t)K * sizeof(int32_t));
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < K; ++i) {
            const float *row = logits + ((size_t)b * K + i) * V;
            int best = 0;
            for (int v = 1; v < V; ++v)
                if (ranks_above(row[v], row[best])) best = v;
            r[i] = best;
            if (argmax_out) argmax_out[(size_t)b * K + i] = best;
        }
        int a = 0;
        while (a < K && proposed[(size_t)b * K + a] == r[a]) ++a;
        accepted[b] = a;
        next_token[b] = r[a < K ? a : K - 1];
    }
    free(r);
}

/*
 * Commit of the accepted prefix for one layer's cache pair.
 * n = min(a+1, K) rows of the block are kept.  If k_blk / v_blk are given
 * (layout [B, K, Hkv, D], elem_size bytes per element), block slots 0..n-1 are
 * copied into cache rows [ctx, ctx+n); otherwise the block already sits in the
 * cache tail.  When advance != 0, ctx_lens[b] += n.  Returns -1 on a bad
 * argument or when ctx + K would exceed S_max.
 */
int oracle_kv_commit(void *k_cache, void *v_cache, const void *k_blk,
                     const void *v_blk, int32_t *ctx_lens,
                     const int32_t *accepted, int B, int Hkv, int D, int S_max,
                     int K, int elem_size, int advance)
{
    for (int b = 0; b < B; ++b) {
        if (accepted[b] < 0 || accepted[b] > K) return -1;
        if (ctx_lens[b] < 0 || (long)ctx_lens[b] + K > S_max) return -1;
    }
    const size_t row = (size_t)D * elem_size;
    for (int b = 0; b < B; ++b) {
        int n = accepted[b] + 1 < K ? accepted[b] + 1 : K;
        if (k_blk && v_blk && k_cache && v_cache) {
            for (int g = 0; g < Hkv; ++g)
                for (int s = 0; s < n; ++s) {
                    size_t dst = (((size_t)b * Hkv + g) * S_max + ctx_lens[b] + s) * row;
                    size_t src = (((size_t)b * K + s) * Hkv + g) * row;
                    memcpy((char *)k_cache + dst, (const char *)k_blk + src, row);
                    memcpy((char *)v_cache + dst, (const char *)v_blk + src, row);
                }
        }
        if (advance) ctx_lens[b] += n;
    }
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
