/*
 * oracle.c -- fp64 reference of Flex-Prefill dynamic block-sparse prefill.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark call this code; the product path never
 * does.  It shares no code, header or constant with the CUDA library.
 *
 * Plain C, double precision, single-threaded, no blocking or fusion: every
 * function is the definition written out, in the order the sources give it.
 * Sources, cited by page title and section:
 *   [FP]  "FPGA24成果：FAST-Prefill稀疏注意力加速器，长上下文LLM推理提速2.5倍"
 *         (yunpan.plus) -- section 1.1 (attention), 1.2 (block partition, two
 *         head patterns, Jensen-Shannon decision), 2.1 (last-query-block scoring
 *         with softmax and block pooling), 3.1 (vertical and slash accumulators,
 *         selection until the cumulative sum exceeds gamma), 3.3 (INT8
 *         multiply, INT32 accumulate).
 *   [MV]  "FPGA加速动态稀疏注意力技术解析与优化" (maplevalley.com.cn) --
 *         section 1.1 (three-step index generation, tau ~ 0.1), 2.3 (signed
 *         nibble split of an int8 product).
 * Readings where the pages are silent (pooling = sum of softmax probabilities,
 * slash at token offsets pooled into offset blocks, JSD operands, QA
 * estimator from block means, VS block score v[c] + s[r-c], forced diagonal,
 * tie order, ">= gamma", int8 scale) are the written conventions of the
 * package design notes; each function below states the one it uses.
 *
 * Notation: n = ceil(S/b) blocks (the last one holds S - (n-1)b tokens when
 * b does not divide S), g = Hq/Hkv, query head h reads KV head h/g, tensors
 * are [H][S][d] row-major, the "last block" is rows (n-1)b .. S-1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int S, Hq, Hkv, d, b;
    int qk_int8;              /* 0: q, k are bf16 bits; 1: q8, k8 int8 with scales */
    const uint16_t *q, *k, *v;/* bf16 bit patterns, [H][S][d] */
    const int8_t *q8, *k8;    /* int8 [H][S][d] */
    const float *q_scale;     /* [Hq] */
    const float *k_scale;     /* [Hkv] */
} orc_problem;

enum { ORC_VS = 0, ORC_QA = 1 };

/* bf16 -> double: the 16 bits are the top half of an IEEE binary32. */
static double bf(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* [MV] 2.3, [FP] 3.3: an 8-bit signed a splits into a = aH*2^4 + aL with
 * aL = a & 0xF in 0..15 and aH signed in -8..7; then
 * a*b = aL*bL + (aH*bL + aL*bH)*2^4 + aH*bH*2^8, each term an int4 product. */
int32_t orc_nibble_mul(int32_t a, int32_t b)
{
    int32_t aL = a & 15, bL = b & 15;
    int32_t aH = (a - aL) / 16, bH = (b - bL) / 16;
    return aL * bL + (aH * bL + aL * bH) * 16 + aH * bH * 256;
}

/* Exact int8 dot product accumulated in integers ([FP] 3.3: INT8 multiply,
 * INT32 accumulate), each product formed through the nibble split. */
static int64_t dot_i8(const int8_t *a, const int8_t *b, int d)
{
    int64_t s = 0;
    for (int t = 0; t < d; ++t) s += orc_nibble_mul(a[t], b[t]);
    return s;
}

static double dot_bf(const uint16_t *a, const uint16_t *b, int d)
{
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += bf(a[t]) * bf(b[t]);
    return s;
}

/* Integer Q.K^T of query row p of head h and key row j (int8 problems). */
int64_t orc_qk_int(const orc_problem *P, int h, int p, int j)
{
    int kvh = h / (P->Hq / P->Hkv);
    const int8_t *qr = P->q8 + ((size_t)h * P->S + p) * P->d;
    const int8_t *kr = P->k8 + ((size_t)kvh * P->S + j) * P->d;
    return dot_i8(qr, kr, P->d);
}

/* Attention logit q_p . k_j / sqrt(d) ([FP] 1.1).  For int8 problems the
 * logit is the exact integer sum times q_scale[h] * k_scale[kvh] / sqrt(d). */
static double logit(const orc_problem *P, int h, int p, int j)
{
    int kvh = h / (P->Hq / P->Hkv);
    double inv = 1.0 / sqrt((double)P->d);
    if (P->qk_int8) {
        double isum = (double)orc_qk_int(P, h, p, j);
        return isum * ((double)P->q_scale[h] * (double)P->k_scale[kvh]) * inv;
    }
    const uint16_t *qr = P->q + ((size_t)h * P->S + p) * P->d;
    const uint16_t *kr = P->k + ((size_t)kvh * P->S + j) * P->d;
    return dot_bf(qr, kr, P->d) * inv;
}

static int nblocks(const orc_problem *P) { return (P->S + P->b - 1) / P->b; }

/* S1+S2 ([FP] 2.1, 3.1): score the last query block of head h against every
 * causal key, softmax each row over j <= p, and pool the probabilities over
 * the block's L = S - (n-1)b rows
 *   vhat[c] = (1/L) sum_i sum_{j in block c} A_ij                (vertical)
 *   shat[o] = (1/L) sum_i sum_{j : floor((p_i - j)/b) = o} A_ij  (slash)
 * Returns max |sum_j A_ij - 1| over the block's rows. */
double orc_last_block_stats(const orc_problem *P, int h, double *vhat, double *shat)
{
    int S = P->S, b = P->b, n = nblocks(P);
    int p0 = (n - 1) * b, rows = S - p0;
    double *s = (double *)malloc(sizeof(double) * (size_t)S);
    double worst = 0.0;
    for (int c = 0; c < n; ++c) { vhat[c] = 0.0; shat[c] = 0.0; }
    for (int i = 0; i < rows; ++i) {
        int p = p0 + i;
        double mx = -INFINITY, z = 0.0, rs = 0.0;
        for (int j = 0; j <= p; ++j) {
            s[j] = logit(P, h, p, j);
            if (s[j] > mx) mx = s[j];
        }
        for (int j = 0; j <= p; ++j) z += exp(s[j] - mx);
        for (int j = 0; j <= p; ++j) {
            double a = exp(s[j] - mx) / z;
            vhat[j / b] += a;
            shat[(p - j) / b] += a;
            rs += a;
        }
        if (fabs(rs - 1.0) > worst) worst = fabs(rs - 1.0);
    }
    for (int c = 0; c < n; ++c) { vhat[c] /= rows; shat[c] /= rows; }
    free(s);
    return worst;
}

/* Block means of the rows of head `head` of Q (which = 0) or K (which = 1):
 * out[c][t] = mean over the rows p of block c (all b of them, or the
 * S - (n-1)b of a partial last block) of x[p][t].  For int8 problems the
 * exact integer column sum is scaled by the head's scale. */
void orc_block_means(const orc_problem *P, int which, int head, double *out)
{
    int S = P->S, b = P->b, d = P->d, n = nblocks(P);
    for (int c = 0; c < n; ++c) {
        int hi = (c + 1) * b < S ? (c + 1) * b : S, cnt = hi - c * b;
        for (int t = 0; t < d; ++t) {
            if (P->qk_int8) {
                const int8_t *x = (which == 0 ? P->q8 : P->k8) + (size_t)head * S * d;
                int64_t acc = 0;
                for (int p = c * b; p < hi; ++p) acc += x[(size_t)p * d + t];
                double sc = which == 0 ? P->q_scale[head] : P->k_scale[head];
                out[(size_t)c * d + t] = (double)acc * sc / cnt;
            } else {
                const uint16_t *x = (which == 0 ? P->q : P->k) + (size_t)head * S * d;
                double acc = 0.0;
                for (int p = c * b; p < hi; ++p) acc += bf(x[(size_t)p * d + t]);
                out[(size_t)c * d + t] = acc / cnt;
            }
        }
    }
}

/* Softmax over c in [0, m) of qbar . kbar[c] / sqrt(d). */
static void block_softmax(const double *qbar, const double *kbar, int m, int d, double *out)
{
    double inv = 1.0 / sqrt((double)d), mx = -INFINITY, z = 0.0;
    for (int c = 0; c < m; ++c) {
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += qbar[t] * kbar[(size_t)c * d + t];
        out[c] = acc * inv;
        if (out[c] > mx) mx = out[c];
    }
    for (int c = 0; c < m; ++c) { out[c] = exp(out[c] - mx); z += out[c]; }
    for (int c = 0; c < m; ++c) out[c] /= z;
}

/* Estimated block distribution of the last query block: softmax over all n
 * key blocks of qbar_{n-1} . kbar_c / sqrt(d) (query-aware estimate). */
void orc_pest(const double *qbar_last, const double *kbar, int n, int d, double *pest)
{
    block_softmax(qbar_last, kbar, n, d, pest);
}

/* Jensen-Shannon divergence ([FP] 1.2), natural log, no square root:
 * JSD = 1/2 KL(p || m) + 1/2 KL(q || m), m = (p + q)/2, 0 log 0 = 0. */
double orc_jsd(const double *p, const double *q, int n)
{
    double a = 0.0, c = 0.0;
    for (int i = 0; i < n; ++i) {
        double m = 0.5 * (p[i] + q[i]);
        if (p[i] > 0.0) a += p[i] * log(p[i] / m);
        if (q[i] > 0.0) c += q[i] * log(q[i] / m);
    }
    return 0.5 * a + 0.5 * c;
}

/* Normalised block scores of query block r over its causal key blocks
 * c in [0, r] ([MV] 1.1 step 3).
 *   VS: w_c = vhat[c] + shat[r - c]
 *   QA: w_c = exp(qbar_r . kbar_c / sqrt(d) - max)
 * each divided by its sum over c in [0, r]. */
void orc_row_scores(int pattern, int r, const double *vhat, const double *shat,
                    const double *qbar_r, const double *kbar, int d, double *w)
{
    if (pattern == ORC_QA) {
        block_softmax(qbar_r, kbar, r + 1, d, w);
        return;
    }
    double z = 0.0;
    for (int c = 0; c <= r; ++c) { w[c] = vhat[c] + shat[r - c]; z += w[c]; }
    for (int c = 0; c <= r; ++c) w[c] /= z;
}

static __thread const double *g_sort_w;  /* per-thread: callers may run heads in parallel threads */
static int by_score_desc(const void *x, const void *y)
{
    int a = *(const int *)x, b = *(const int *)y;
    if (g_sort_w[a] > g_sort_w[b]) return -1;
    if (g_sort_w[a] < g_sort_w[b]) return 1;
    return a < b ? -1 : (a > b ? 1 : 0);
}

/* gamma-coverage selection ([FP] 3.1, [MV] 3.2): the diagonal block r is
 * always kept; the other causal blocks are then taken in order of score
 * (descending, ties by ascending index) while the cumulative score is below
 * gamma.  gamma >= 1 keeps every causal block.  Writes the kept indices in
 * ascending order to sel and returns their count.  info (may be NULL)
 * receives {score of the last block added (-1 if none), cumulative before
 * it, final cumulative}. */
int orc_select(const double *w, int r, double gamma, int32_t *sel, double *info)
{
    int cnt = 0;
    if (gamma >= 1.0) {
        double cum = 0.0;
        for (int c = 0; c <= r; ++c) { sel[cnt++] = c; cum += w[c]; }
        if (info) { info[0] = -1.0; info[1] = cum; info[2] = cum; }
        return cnt;
    }
    int *order = (int *)malloc(sizeof(int) * (size_t)(r + 1));
    char *keep = (char *)calloc((size_t)(r + 1), 1);
    int m = 0;
    for (int c = 0; c < r; ++c) order[m++] = c;
    g_sort_w = w;
    qsort(order, (size_t)m, sizeof(int), by_score_desc);
    keep[r] = 1;
    double cum = w[r], last = -1.0, before = w[r];
    for (int t = 0; t < m; ++t) {
        if (cum >= gamma) break;
        keep[order[t]] = 1;
        before = cum;
        last = w[order[t]];
        cum += w[order[t]];
    }
    for (int c = 0; c <= r; ++c) if (keep[c]) sel[cnt++] = c;
    if (info) { info[0] = last; info[1] = before; info[2] = cum; }
    free(order);
    free(keep);
    return cnt;
}

/* Whole index of head h ([MV] 1.1: representative query block, JSD pattern
 * decision, block-level index).  Outputs:
 *   vhat, shat, pest [n]; jsd; pattern (QA if jsd < tau else VS, unless
 *   force_pattern >= 0); counts[n]; cols padded so row r starts at r(r+1)/2;
 *   scores (may be NULL) padded the same way; info (may be NULL) [n][3].
 * Returns max |row sum - 1| of the last block's softmax rows. */
double orc_build_index_head(const orc_problem *P, int h, double gamma, double tau, int force_pattern,
                            double *vhat, double *shat, double *pest, double *jsd, int32_t *pattern,
                            int32_t *counts, int32_t *cols, double *scores, double *info)
{
    int b = P->b, d = P->d, n = nblocks(P), kvh = h / (P->Hq / P->Hkv);
    double worst = orc_last_block_stats(P, h, vhat, shat);
    double *kbar = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *qbar = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    orc_block_means(P, 1, kvh, kbar);
    orc_block_means(P, 0, h, qbar);
    orc_pest(qbar + (size_t)(n - 1) * d, kbar, n, d, pest);
    *jsd = orc_jsd(vhat, pest, n);
    *pattern = (*jsd < tau) ? ORC_QA : ORC_VS;
    if (force_pattern >= 0) *pattern = force_pattern;
    for (int r = 0; r < n; ++r) {
        size_t off = (size_t)r * (r + 1) / 2;
        orc_row_scores(*pattern, r, vhat, shat, qbar + (size_t)r * d, kbar, d, w);
        counts[r] = orc_select(w, r, gamma, cols + off, info ? info + (size_t)r * 3 : NULL);
        if (scores) memcpy(scores + off, w, sizeof(double) * (size_t)(r + 1));
    }
    free(kbar);
    free(qbar);
    free(w);
    return worst;
}

/* Block-sparse causal attention ([FP] 1.1 and figure 3) for query rows
 * p in [p_lo, p_hi) of head h, all inside one query block: the keys are the
 * union of the listed key blocks, restricted to j <= p; out[p - p_lo][t] =
 * sum_j softmax_j(q_p . k_j / sqrt(d)) v_j[t]. */
void orc_attn_rows(const orc_problem *P, int h, int p_lo, int p_hi, const int32_t *blocks,
                   int nblocks, double *out)
{
    int S = P->S, b = P->b, d = P->d, kvh = h / (P->Hq / P->Hkv);
    double *s = (double *)malloc(sizeof(double) * (size_t)nblocks * b);
    int *js = (int *)malloc(sizeof(int) * (size_t)nblocks * b);
    for (int p = p_lo; p < p_hi; ++p) {
        int m = 0;
        double mx = -INFINITY, z = 0.0;
        for (int e = 0; e < nblocks; ++e)
            for (int j = blocks[e] * b; j < (blocks[e] + 1) * b && j < S; ++j)
                if (j <= p) { js[m] = j; s[m] = logit(P, h, p, j); if (s[m] > mx) mx = s[m]; ++m; }
        for (int e = 0; e < m; ++e) { s[e] = exp(s[e] - mx); z += s[e]; }
        double *o = out + (size_t)(p - p_lo) * d;
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        for (int e = 0; e < m; ++e) {
            const uint16_t *vr = P->v + ((size_t)kvh * S + js[e]) * d;
            double a = s[e] / z;
            for (int t = 0; t < d; ++t) o[t] += a * bf(vr[t]);
        }
    }
    free(s);
    free(js);
}

/* Exact integer score tile: out[i][t] = q8[h][p0+i] . k8[kvh][j0+t] for
 * i in [0, rows), t in [0, cols) ([FP] 3.3). */
void orc_qk_int_tile(const orc_problem *P, int h, int p0, int j0, int rows, int cols, int32_t *out)
{
    for (int i = 0; i < rows; ++i)
        for (int t = 0; t < cols; ++t)
            out[(size_t)i * cols + t] = (int32_t)orc_qk_int(P, h, p0 + i, j0 + t);
}

/* ------------------------------------------------------------------------
 * Rotary embedding with block pooling: the epilogue of the projection step
 * that produces Q and K ([FP] 1.1: Q = X W_q, K = X W_k), followed by the
 * block means the index generation uses ([FP] 2.1 block pooling; [MV] 1.1
 * block-level estimate).  Rotate-half convention: for i < d/2, with c =
 * cos[p][i], s = sin[p][i] (the caller's tables),
 *   out[p][i]       = x[p][i] c - x[p][i + d/2] s
 *   out[p][i + d/2] = x[p][i + d/2] c + x[p][i] s,
 * each rounded to the nearest bf16 (ties to even), as the stored tensor is
 * bf16; means[c][t] = mean over the rows of block c (b of them, or S-(n-1)b
 * for a partial last block) of the rounded out[p][t].
 * x: H*S*d doubles (bf16 values); cos, sin: S*(d/2) doubles; out: H*S*d;
 * means: H*n*d with n = ceil(S/b). */

/* Nearest bf16 (8 significant bits, ties to even) of a finite double. */
static double round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    double m = frexp(x, &e);            /* x = m 2^e, 0.5 <= |m| < 1 */
    double r = nearbyint(ldexp(m, 8));  /* 128 <= |r| <= 256, ties to even */
    return ldexp(r, e - 8);
}

void orc_rope_pool(const double *x, const double *cosT, const double *sinT, int H, int S, int d, int b,
                   double *out, double *means)
{
    int half = d / 2, n = (S + b - 1) / b;
    for (int h = 0; h < H; ++h) {
        for (int p = 0; p < S; ++p) {
            const double *xr = x + ((size_t)h * S + p) * d;
            double *orow = out + ((size_t)h * S + p) * d;
            for (int i = 0; i < half; ++i) {
                double c = cosT[(size_t)p * half + i], sn = sinT[(size_t)p * half + i];
                orow[i] = round_bf16(xr[i] * c - xr[i + half] * sn);
                orow[i + half] = round_bf16(xr[i + half] * c + xr[i] * sn);
            }
        }
        for (int c = 0; c < n; ++c) {
            int lo = c * b, hi = (c + 1) * b < S ? (c + 1) * b : S;
            for (int t = 0; t < d; ++t) {
                double acc = 0.0;
                for (int p = lo; p < hi; ++p) acc += out[((size_t)h * S + p) * d + t];
                means[((size_t)h * n + c) * d + t] = acc / (hi - lo);
            }
        }
    }
}

/* ------------------------------------------------------------------------
 * Head-pattern sharing (maplevalley article, section 5, future directions:
 * similar heads share one sparse pattern).  The pages give no rule for
 * "similar"; the written convention: within one GQA group (the g query heads
 * of a KV head, in head order), head a joins the class of the earliest
 * earlier class representative b with JSD(vhat_a, vhat_b) < eps (natural
 * log, no square root, as for the pattern decision); a head that joins no
 * class represents its own.  Every head of a class then attends to the union
 * of the class members' block lists, so each head keeps at least its own
 * gamma-coverage.
 * vhat: [g][n] of the group's heads; cls[a] receives the representative's
 * position in the group (cls[a] = a for a representative). */
void orc_share_classes(const double *vhat, int g, int n, double eps, int32_t *cls)
{
    for (int a = 0; a < g; ++a) {
        cls[a] = a;
        for (int b = 0; b < a; ++b) {
            if (cls[b] != b) continue;
            if (orc_jsd(vhat + (size_t)a * n, vhat + (size_t)b * n, n) < eps) {
                cls[a] = b;
                break;
            }
        }
    }
}

/* Ascending union of the lists of the heads in one class for query block r:
 * lists[m] (counts[m] entries each, ascending) for the class's members m.
 * Writes the union to out and returns its size. */
int orc_union_lists(const int32_t *const *lists, const int32_t *counts, int members, int r, int32_t *out)
{
    char *seen = (char *)calloc((size_t)(r + 1), 1);
    int cnt = 0;
    for (int m = 0; m < members; ++m)
        for (int e = 0; e < counts[m]; ++e) seen[lists[m][e]] = 1;
    for (int c = 0; c <= r; ++c) if (seen[c]) out[cnt++] = c;
    free(seen);
    return cnt;
}

/* ------------------------------------------------------------------------
 * Adaptive block size (maplevalley article, section 5: block size adjusted
 * to the complexity of the content; section 4.3 lists 64, 128 and 256).  The
 * written convention: at b = 128, the concentration of head h is
 * k_h / n, where k_h is the smallest number of key blocks whose vhat
 * (the exact pooled last-block attention of that head) sums to at least
 * gamma (blocks taken by descending vhat); rho is the mean over heads.
 * Concentrated attention (rho < 0.1) gets the finer b = 64 when S/64 <= 1024
 * blocks, diffuse attention (rho >= 0.5) the coarser b = 256, anything else
 * b = 128.  vhat: [Hq][n] at b = 128. */
int orc_cover_count(const double *v, int n, double gamma)
{
    int *order = (int *)malloc(sizeof(int) * (size_t)n);
    for (int c = 0; c < n; ++c) order[c] = c;
    g_sort_w = v;
    qsort(order, (size_t)n, sizeof(int), by_score_desc);
    double cum = 0.0;
    int k = 0;
    while (k < n && cum < gamma) cum += v[order[k++]];
    free(order);
    return k;
}

int orc_choose_block_size(const double *vhat, int Hq, int n, int S, double gamma, double *rho_out)
{
    double rho = 0.0;
    for (int h = 0; h < Hq; ++h) rho += (double)orc_cover_count(vhat + (size_t)h * n, n, gamma) / n;
    rho /= Hq;
    if (rho_out) *rho_out = rho;
    if (rho < 0.1 && (S + 63) / 64 <= 1024) return 64;
    if (rho >= 0.5) return 256;
    return 128;
}
