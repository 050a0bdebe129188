/*
 * ReAttention CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * A plain, slow, obviously-correct fp64 restatement of what the top-k span
 * attention step computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; the two only see the same
 * seeded input bytes.
 *
 * Sources (pages about "ReAttention: Training-Free Infinite Context with
 * Finite Attention Scope", arXiv 2407.15176):
 *   [ABS]  arXiv abstract: position-agnostic top-k attention runs before the
 *          ordinary position-aware self-attention.
 *   [APP]  research-map summary, "Approach": middle KV segments are scored by
 *          the dot product of the query with un-positioned keys, concatenated
 *          with the global and local caches, and only then given positional
 *          embeddings.
 *   [DEC]  OpenReview discussion, "Decoding Phase" pseudocode: score =
 *          query . key[global:-local]^T, top-k, concatenation global ++
 *          recalled ++ local, then attention.
 *   [HYP]  OpenReview discussion, NIAH comparison settings: global 32,
 *          local 4096, seg_size 32, num_seg 127.
 * Readings taken where the pages are silent:
 *   - a span is S consecutive middle tokens, tiled from the left; the last
 *     span may be short; span score = max over its tokens (and over the
 *     chunk's queries when C > 1);
 *   - GQA: the token score sums q.k over the KV head's query heads;
 *   - ties go to the lower span index; the chosen spans keep their original
 *     (ascending) order;
 *   - window = global ++ chosen spans ++ local (last L cached) ++ current;
 *     RoPE (rotate-half pairing i, i+d/2) at window positions 0..W-1; query c
 *     sits at W-C+c; causal softmax attention with scale 1/sqrt(d).
 *
 * Everything is computed in double precision from the input bits
 * (dtype 0 = fp32, dtype 1 = bf16 stored as raw uint16).
 * Parallelism (OpenMP over heads and spans) is the only concession to speed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORA_F32 0
#define ORA_BF16 1

static double ora_elem(const void *base, int dtype, int64_t i)
{
    if (dtype == ORA_F32)
        return (double)((const float *)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

void ora_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int ora_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Partition of the T cached tokens [DEC; HYP]:
 *   global = [0, min(G,T)), local = [max(G, T-L), T), middle = [G, G+M)
 *   with M = max(0, T-G-L), NS = ceil(M / S) spans.
 * out = {global_end, local_begin, M, NS}.
 */
void ora_partition(int64_t T, int G, int L, int S, int64_t out[4])
{
    int64_t g_end = T < G ? T : G;
    int64_t loc_begin = (T - L) > G ? (T - L) : G;
    int64_t M = T - G - L;
    if (M < 0)
        M = 0;
    out[0] = g_end;
    out[1] = loc_begin;
    out[2] = M;
    out[3] = (M + S - 1) / S;
}

/* Score of cached token t for KV head h of batch b [DEC; APP]:
 *   max over queries c of  sum_{j in group(h)} sum_i q[b,j,c,i] * k[b,h,t,i]
 * on the un-rotated vectors. */
static double ora_token_score(int Hq, int Hkv, int d, int C, int64_t T, int dtype,
                              const void *q, const void *kc, int b, int h, int64_t t)
{
    int g = Hq / Hkv;
    int64_t krow = (((int64_t)b * Hkv + h) * T + t) * d;
    double best = -INFINITY;
    for (int c = 0; c < C; ++c) {
        double s = 0.0;
        for (int j = h * g; j < (h + 1) * g; ++j) {
            int64_t qrow = (((int64_t)b * Hq + j) * C + c) * d;
            for (int i = 0; i < d; ++i)
                s += ora_elem(q, dtype, qrow + i) * ora_elem(kc, dtype, krow + i);
        }
        if (s > best)
            best = s;
    }
    return best;
}

/* Span score = max over the span's tokens of the token score. Span sp of the
 * middle covers tokens [G + sp*S, min(G + (sp+1)*S, G + M)). */
static double ora_one_span(int Hq, int Hkv, int d, int C, int64_t T, int G, int L, int S,
                           int dtype, const void *q, const void *kc, int b, int h, int64_t sp)
{
    int64_t part[4];
    ora_partition(T, G, L, S, part);
    int64_t M = part[2];
    int64_t t0 = G + sp * (int64_t)S;
    int64_t t1 = t0 + S;
    if (t1 > G + M)
        t1 = G + M;
    double best = -INFINITY;
    for (int64_t t = t0; t < t1; ++t) {
        double s = ora_token_score(Hq, Hkv, d, C, T, dtype, q, kc, b, h, t);
        if (s > best)
            best = s;
    }
    return best;
}

/* All span scores, scores[(b*Hkv + h)*NS + sp]. */
void ora_span_scores(int B, int Hq, int Hkv, int d, int C, int64_t T, int G, int L, int S,
                     int dtype, const void *q, const void *kc, double *scores)
{
    int64_t part[4];
    ora_partition(T, G, L, S, part);
    int64_t NS = part[3];
    int64_t total = (int64_t)B * Hkv * NS;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t x = 0; x < total; ++x) {
        int64_t bh = x / NS, sp = x % NS;
        scores[x] = ora_one_span(Hq, Hkv, d, C, T, G, L, S, dtype, q, kc,
                                 (int)(bh / Hkv), (int)(bh % Hkv), sp);
    }
}

/* Span scores for an explicit list of (bh, sp) pairs, for sampled checks at
 * sizes where scoring every span is too slow. */
void ora_span_scores_list(int B, int Hq, int Hkv, int d, int C, int64_t T, int G, int L, int S,
                          int dtype, const void *q, const void *kc,
                          const int64_t *pairs, int64_t n, double *scores)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t x = 0; x < n; ++x) {
        int64_t bh = pairs[2 * x], sp = pairs[2 * x + 1];
        scores[x] = ora_one_span(Hq, Hkv, d, C, T, G, L, S, dtype, q, kc,
                                 (int)(bh / Hkv), (int)(bh % Hkv), sp);
    }
}

/* ---- top-k: highest score first, ties to the lower span index, then the
 * chosen indices in ascending (original) order [DEC "recalled" tokens kept
 * in cache order]. ---- */
static const double *ora_sort_keys;

static int ora_cmp_rank(const void *a, const void *b)
{
    int64_t i = *(const int64_t *)a, j = *(const int64_t *)b;
    double si = ora_sort_keys[i], sj = ora_sort_keys[j];
    if (si > sj)
        return -1;
    if (si < sj)
        return 1;
    return (i < j) ? -1 : (i > j);
}

static int ora_cmp_index(const void *a, const void *b)
{
    int64_t i = *(const int64_t *)a, j = *(const int64_t *)b;
    return (i < j) ? -1 : (i > j);
}

/* sel[0..k) = chosen span ids ascending, padded with -1 when NS < k.
 * Returns k_eff = min(k, NS).  Not thread-safe (qsort key pointer). */
int ora_topk(const double *scores, int64_t NS, int k, int32_t *sel)
{
    int64_t keff = NS < k ? NS : k;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (NS > 0 ? NS : 1));
    for (int64_t i = 0; i < NS; ++i)
        order[i] = i;
    ora_sort_keys = scores;
    qsort(order, (size_t)NS, sizeof(int64_t), ora_cmp_rank);
    qsort(order, (size_t)keff, sizeof(int64_t), ora_cmp_index);
    for (int i = 0; i < k; ++i)
        sel[i] = i < keff ? (int32_t)order[i] : -1;
    free(order);
    return (int)keff;
}

/* ---- window: global ++ chosen spans (ascending) ++ local ++ current ----
 * src[p] = cache row of window row p, or -(1+c) for current token c.
 * Returns W.  src must hold G + k*S + L + C entries. */
int64_t ora_window(int64_t T, int G, int L, int S, int C, const int32_t *sel, int k, int64_t *src)
{
    int64_t part[4];
    ora_partition(T, G, L, S, part);
    int64_t g_end = part[0], loc_begin = part[1], M = part[2];
    int64_t W = 0;
    for (int64_t t = 0; t < g_end; ++t)
        src[W++] = t;
    for (int j = 0; j < k; ++j) {
        if (sel[j] < 0)
            continue;
        int64_t t0 = G + (int64_t)sel[j] * S, t1 = t0 + S;
        if (t1 > G + M)
            t1 = G + M;
        for (int64_t t = t0; t < t1; ++t)
            src[W++] = t;
    }
    for (int64_t t = loc_begin; t < T; ++t)
        src[W++] = t;
    for (int c = 0; c < C; ++c)
        src[W++] = -(1 + (int64_t)c);
    return W;
}

/* ---- RoPE, rotate-half pairing (i, i + d/2) with frequency
 * base^(-2i/d), applied at integer position pos [ABS; APP: positional
 * embedding after concatenation].  Angles in double. ---- */
void ora_rope_row(double *x, int d, double pos, double base)
{
    int h = d / 2;
    for (int i = 0; i < h; ++i) {
        double inv_freq = pow(base, -2.0 * (double)i / (double)d);
        double a = pos * inv_freq;
        double cs = cos(a), sn = sin(a);
        double x0 = x[i], x1 = x[i + h];
        x[i] = x0 * cs - x1 * sn;
        x[i + h] = x1 * cs + x0 * sn;
    }
}

/* ---- the whole step ----
 * q [B,Hq,C,d], kc/vc [B,Hkv,T,d], kcur/vcur [B,Hkv,C,d] (dtype as above).
 * sel_in [B,Hkv,k]: when non-NULL, that selection is used instead of scoring
 *   (lets a test compare attention after a tolerated near-tie swap).
 * sel_out [B,Hkv,k], win_out [B,Hkv], scores_out [B,Hkv,NS]: optional.
 * c_list/n_c: which query positions to compute (NULL = all C).
 * out [B,Hq,C,d]: attention output for the listed queries. */
void ora_step(int B, int Hq, int Hkv, int d, int C, int64_t T, int G, int L, int S, int k,
              double base, int dtype,
              const void *q, const void *kc, const void *vc, const void *kcur, const void *vcur,
              const int32_t *sel_in, int32_t *sel_out, int64_t *win_out, double *scores_out,
              const int32_t *c_list, int n_c, double *out)
{
    int g = Hq / Hkv;
    int64_t part[4];
    ora_partition(T, G, L, S, part);
    int64_t NS = part[3];
    int64_t wcap = (int64_t)G + (int64_t)k * S + L + C;
    int ncq = c_list ? n_c : C;

    double *all_scores = NULL;
    if (!sel_in) {
        all_scores = (double *)malloc(sizeof(double) * ((int64_t)B * Hkv * NS + 1));
        ora_span_scores(B, Hq, Hkv, d, C, T, G, L, S, dtype, q, kc, all_scores);
        if (scores_out)
            memcpy(scores_out, all_scores, sizeof(double) * (size_t)((int64_t)B * Hkv * NS));
    }

    for (int bh = 0; bh < B * Hkv; ++bh) {
        int b = bh / Hkv, h = bh % Hkv;
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (k > 0 ? k : 1));
        if (sel_in)
            memcpy(sel, sel_in + (int64_t)bh * k, sizeof(int32_t) * k);
        else
            ora_topk(all_scores + (int64_t)bh * NS, NS, k, sel);
        if (sel_out)
            memcpy(sel_out + (int64_t)bh * k, sel, sizeof(int32_t) * k);

        int64_t *src = (int64_t *)malloc(sizeof(int64_t) * wcap);
        int64_t W = ora_window(T, G, L, S, C, sel, k, src);
        if (win_out)
            win_out[bh] = W;

        /* rotated keys and plain values of the window, in double */
        double *kr = (double *)malloc(sizeof(double) * (size_t)(W * d));
        double *vr = (double *)malloc(sizeof(double) * (size_t)(W * d));
#pragma omp parallel for schedule(static)
        for (int64_t p = 0; p < W; ++p) {
            for (int i = 0; i < d; ++i) {
                int64_t s = src[p];
                double kv, vv;
                if (s >= 0) {
                    int64_t off = (((int64_t)b * Hkv + h) * T + s) * d + i;
                    kv = ora_elem(kc, dtype, off);
                    vv = ora_elem(vc, dtype, off);
                } else {
                    int64_t c = -s - 1;
                    int64_t off = (((int64_t)b * Hkv + h) * C + c) * d + i;
                    kv = ora_elem(kcur, dtype, off);
                    vv = ora_elem(vcur, dtype, off);
                }
                kr[p * d + i] = kv;
                vr[p * d + i] = vv;
            }
            ora_rope_row(kr + p * d, d, (double)p, base);
        }

        /* causal softmax attention for each query head of the group */
        int nrows = g * ncq;
#pragma omp parallel for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int j = h * g + r / ncq;
            int c = c_list ? c_list[r % ncq] : r % ncq;
            int64_t qpos = W - C + c;
            double *qv = (double *)malloc(sizeof(double) * d);
            double *lg = (double *)malloc(sizeof(double) * (size_t)(qpos + 1));
            int64_t qrow = (((int64_t)b * Hq + j) * C + c) * d;
            for (int i = 0; i < d; ++i)
                qv[i] = ora_elem(q, dtype, qrow + i);
            ora_rope_row(qv, d, (double)qpos, base);
            double scale = 1.0 / sqrt((double)d), mx = -INFINITY;
            for (int64_t p = 0; p <= qpos; ++p) {
                double s = 0.0;
                for (int i = 0; i < d; ++i)
                    s += qv[i] * kr[p * d + i];
                lg[p] = s * scale;
                if (lg[p] > mx)
                    mx = lg[p];
            }
            double den = 0.0;
            for (int64_t p = 0; p <= qpos; ++p) {
                lg[p] = exp(lg[p] - mx);
                den += lg[p];
            }
            double *o = out + qrow;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int64_t p = 0; p <= qpos; ++p)
                    acc += lg[p] * vr[p * d + i];
                o[i] = acc / den;
            }
            free(qv);
            free(lg);
        }
        free(kr);
        free(vr);
        free(src);
        free(sel);
    }
    free(all_scores);
}
