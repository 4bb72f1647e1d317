/*
 * lsa_oracle.c -- plain, slow, fp64 CPU oracle for the Lookahead Sparse
 * Attention (LSA) decode hot path.
 *
 * TEST INFRASTRUCTURE, NOT THE PRODUCT.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline / reference leg may load this library.
 * It shares no code, header, table or helper with the CUDA path: it has its
 * own dtype codes, its own bf16 / e4m3 decoders (written from the formats'
 * definitions) and its own loops.
 *
 * Source of the method: "FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long
 * Context via Lookahead Sparse Attention" (gist.science technical summary,
 * section 2.1 "Architectural Design"), restated:
 *   - every tau decode steps a memory indexer maps the hidden state to
 *     low-rank indexer queries and computes a "lookahead index score"
 *     I_{t,s} for every preceding compressed KV entry s, a head-fused gated
 *     matching score passed through a sigmoid;
 *   - every entry with I_{t,s} >= 0.5 is fetched from the CPU cold pool into
 *     GPU memory (no rigid top-k at this stage);
 *   - inside that fetched subset the native Lightning Indexer takes a
 *     fine-grained top-k, and core attention runs over it.
 * The score is fixed as  I = sigmoid( sum_j w_j * ReLU(q_j . k_s) )  (the
 * head fusion is the gate-weighted sum over indexer heads j; section 5 of the
 * same summary says the interaction is a plain dot product).
 *
 * Every function computes the plain definition, in fp64, with no blocking,
 * fusion or reordering.  OpenMP only splits independent outputs over cores.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* dtype codes of this oracle (deliberately its own numbering) */
#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2
#define ORC_F64 3

/* ------------------------------------------------------------------ */
/* Element decoders, from the formats' definitions.                    */
/* ------------------------------------------------------------------ */

/* bfloat16: the upper 16 bits of an IEEE-754 binary32. */
double orc_bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7),
 * 3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6;
 * S.1111.111 is NaN; there are no infinities; the largest finite is 448. */
double orc_e4m3_to_f64(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

static double load_elem(const void *base, int dtype, int64_t i)
{
    switch (dtype) {
    case ORC_F32:
        return (double)((const float *)base)[i];
    case ORC_BF16:
        return orc_bf16_to_f64(((const uint16_t *)base)[i]);
    case ORC_E4M3:
        return orc_e4m3_to_f64(((const uint8_t *)base)[i]);
    case ORC_F64:
        return ((const double *)base)[i];
    default:
        return NAN;
    }
}

/* Decode n elements of any supported dtype into fp64. */
void orc_decode(const void *src, int dtype, int64_t n, double *dst)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; i++)
        dst[i] = load_elem(src, dtype, i);
}

/* Value of channel c of compressed indexer key row s.  For e4m3 keys the
 * stored code is multiplied by the row's fp32 scale; one scale covers each
 * block of 128 channels (a row of d <= 128 channels has one scale). */
static double key_value(const void *k, int k_dtype, const float *k_scale,
                        int64_t s, int d, int c)
{
    double v = load_elem(k, k_dtype, s * (int64_t)d + c);
    if (k_scale) {
        int nblk = (d + 127) / 128;
        v *= (double)k_scale[s * nblk + c / 128];
    }
    return v;
}

/* ------------------------------------------------------------------ */
/* Lookahead index score (section 2.1 "Scoring Mechanism").            */
/* ------------------------------------------------------------------ */

/* Score of one entry s of sequence b:
 *     z = sum_{j<H} w[b,j] * max(0, sum_{c<d} q[b,j,c] * k[s,c])
 * and I = 1 / (1 + exp(-z)). */
static double score_one(const void *q, int q_dtype, const float *w,
                        const void *k, int k_dtype, const float *k_scale,
                        int b, int64_t s, int H, int d)
{
    double z = 0.0;
    int j, c;
    for (j = 0; j < H; j++) {
        double dot = 0.0;
        for (c = 0; c < d; c++) {
            double qv = load_elem(q, q_dtype, ((int64_t)b * H + j) * d + c);
            dot += qv * key_value(k, k_dtype, k_scale, s, d, c);
        }
        z += (double)w[(int64_t)b * H + j] * (dot > 0.0 ? dot : 0.0);
    }
    return z;
}

/* Full scan: every entry of every sequence.  seq_off[B+1] is the CSR offset
 * of each sequence on the flat entry axis.  I may be NULL. */
void orc_index_score(const void *q, int q_dtype, const float *w,
                     const void *k, int k_dtype, const float *k_scale,
                     const int64_t *seq_off, int B, int H, int d,
                     double *z, double *I)
{
    int b;
    for (b = 0; b < B; b++) {
        int64_t s;
#pragma omp parallel for schedule(static)
        for (s = seq_off[b]; s < seq_off[b + 1]; s++) {
            double zs = score_one(q, q_dtype, w, k, k_dtype, k_scale, b, s, H, d);
            z[s] = zs;
            if (I)
                I[s] = 1.0 / (1.0 + exp(-zs));
        }
    }
}

/* Listed scan: only the entries idx[idx_off[b] .. idx_off[b+1]) of sequence
 * b (indices local to the sequence); z is written at the list position. */
void orc_index_score_list(const void *q, int q_dtype, const float *w,
                          const void *k, int k_dtype, const float *k_scale,
                          const int64_t *seq_off, const int32_t *idx,
                          const int64_t *idx_off, int B, int H, int d,
                          double *z, double *I)
{
    int b;
    for (b = 0; b < B; b++) {
        int64_t p;
#pragma omp parallel for schedule(static)
        for (p = idx_off[b]; p < idx_off[b + 1]; p++) {
            int64_t s = seq_off[b] + idx[p];
            double zs = score_one(q, q_dtype, w, k, k_dtype, k_scale, b, s, H, d);
            z[p] = zs;
            if (I)
                I[p] = 1.0 / (1.0 + exp(-zs));
        }
    }
}

/* ------------------------------------------------------------------ */
/* Threshold selection (section 2.1 "Dynamic Fetching"): keep every    */
/* entry with I >= 0.5.  Since sigmoid is strictly increasing with     */
/* sigmoid(0) = 0.5, I >= 0.5 holds exactly when z >= 0; the decision  */
/* is taken on z so that no rounding of the sigmoid can move it.       */
/* ------------------------------------------------------------------ */

/* Writes the kept entries of each sequence, as indices local to the
 * sequence in ascending order, to kept_idx[kept_off[b] ..], and the CSR
 * offsets kept_off[B+1].  mask (may be NULL) receives one byte per entry.
 * Returns the total number of kept entries. */
int64_t orc_select(const double *z, const int64_t *seq_off, int B,
                   int32_t *kept_idx, int64_t *kept_off, uint8_t *mask)
{
    int64_t n = 0;
    int b;
    kept_off[0] = 0;
    for (b = 0; b < B; b++) {
        int64_t s;
        for (s = seq_off[b]; s < seq_off[b + 1]; s++) {
            int keep = z[s] >= 0.0;
            if (mask)
                mask[s] = (uint8_t)keep;
            if (keep)
                kept_idx[n++] = (int32_t)(s - seq_off[b]);
        }
        kept_off[b + 1] = n;
    }
    return n;
}

/* ------------------------------------------------------------------ */
/* OR-mode union of indexer layers (section 2.4 "Optimal              */
/* Configuration": independent Memory Indexers on three layers, whose */
/* predictions are united at inference to decide what is fetched).    */
/* Each layer l predicts "fetch s" exactly when z_l[s] >= 0; the union */
/* fetches s when any layer does.  The union's ranking score is taken  */
/* as the largest z of the layers (the pages give none): a NaN score   */
/* is no prediction and no score.                                     */
/* ------------------------------------------------------------------ */

void orc_index_union(const double *const *z, int n_layers, int64_t n, uint8_t *keep, double *score)
{
    int64_t s;
    for (s = 0; s < n; s++) {
        int l, any = 0, have = 0;
        double best = NAN;
        for (l = 0; l < n_layers; l++) {
            double v = z[l][s];
            if (v >= 0.0)
                any = 1;
            if (v == v) {
                if (!have || v > best)
                    best = v;
                have = 1;
            }
        }
        keep[s] = (uint8_t)any;
        score[s] = best;
    }
}

/* ------------------------------------------------------------------ */
/* Indexer query encoder (section 2.1 "Memory Indexer": the current    */
/* query token's hidden state h_t is mapped to low-rank indexer        */
/* queries; section 2.3 "Query Optimization": what the encoder trains  */
/* are its low-rank projection matrices).  Read as a rank-r            */
/* factorisation with the head weights taken from h_t directly:        */
/*   c   = W_dq h            (W_dq [rank, hidden])                     */
/*   q_j = (W_uq c)[j*d .. j*d+d-1]   (W_uq [H*d, rank])               */
/*   w   = W_w h             (W_w [H, hidden])                         */
/* with no norm, activation or positional term (the pages name none).  */
/* Matrices are row-major [out, in]; every product and sum in fp64.    */
/* ------------------------------------------------------------------ */

void orc_query_encode(const void *h, int h_dtype, int B, int hidden,
                      const void *W_dq, const void *W_uq, const void *W_w, int w_dtype,
                      int rank, int H, int d, double *c, double *q, double *w)
{
    int b;
#pragma omp parallel for schedule(static)
    for (b = 0; b < B; b++) {
        const int64_t hb = (int64_t)b * hidden;
        int i, n, j, k;
        for (i = 0; i < rank; i++) {
            double acc = 0.0;
            for (k = 0; k < hidden; k++)
                acc += load_elem(W_dq, w_dtype, (int64_t)i * hidden + k) * load_elem(h, h_dtype, hb + k);
            c[(int64_t)b * rank + i] = acc;
        }
        for (n = 0; n < H * d; n++) {
            double acc = 0.0;
            for (i = 0; i < rank; i++)
                acc += load_elem(W_uq, w_dtype, (int64_t)n * rank + i) * c[(int64_t)b * rank + i];
            q[(int64_t)b * H * d + n] = acc;
        }
        for (j = 0; j < H; j++) {
            double acc = 0.0;
            for (k = 0; k < hidden; k++)
                acc += load_elem(W_w, w_dtype, (int64_t)j * hidden + k) * load_elem(h, h_dtype, hb + k);
            w[(int64_t)b * H + j] = acc;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Fine-grained top-k inside the kept subset (section 2.1 "Tiered      */
/* Selection").  Ranking is by z (the sigmoid is monotone), larger    */
/* first, equal z broken towards the lower entry index.  The chosen   */
/* set is reported in ascending entry order, padded with -1.          */
/* ------------------------------------------------------------------ */

typedef struct {
    double z;
    int32_t idx;
} orc_cand;

static int by_rank(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    if (x->z > y->z)
        return -1;
    if (x->z < y->z)
        return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int by_index(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* zk[p] is the score of the kept entry kept_idx[p]. */
void orc_topk(const double *zk, const int32_t *kept_idx, const int64_t *kept_off,
              int B, int k, int32_t *topk_idx, int32_t *topk_cnt)
{
    int b;
    for (b = 0; b < B; b++) {
        int64_t n = kept_off[b + 1] - kept_off[b], p;
        int64_t take = n < k ? n : k;
        orc_cand *c = (orc_cand *)malloc((size_t)(n > 0 ? n : 1) * sizeof *c);
        for (p = 0; p < n; p++) {
            c[p].z = zk[kept_off[b] + p];
            c[p].idx = kept_idx[kept_off[b] + p];
        }
        qsort(c, (size_t)n, sizeof *c, by_rank);
        qsort(c, (size_t)take, sizeof *c, by_index);
        for (p = 0; p < k; p++)
            topk_idx[(int64_t)b * k + p] = p < take ? c[p].idx : -1;
        topk_cnt[b] = (int32_t)take;
        free(c);
    }
}

/* ------------------------------------------------------------------ */
/* Cold-pool fetch (section 2.1 "Dynamic Fetching"; the blog page's    */
/* "fetched from the CPU Cold Pool to the GPU HBM just in time").      */
/* Row r of the hot buffer receives the cold row of the r-th kept      */
/* entry; slot_of maps every entry to its hot row or -1.               */
/* ------------------------------------------------------------------ */

void orc_gather(const uint8_t *cold, int64_t row_bytes, const int64_t *seq_off,
                const int32_t *kept_idx, const int64_t *kept_off, int B,
                uint8_t *hot, int32_t *slot_of)
{
    int b;
    int64_t s;
    for (s = 0; s < seq_off[B]; s++)
        slot_of[s] = -1;
    for (b = 0; b < B; b++) {
        int64_t p;
        for (p = kept_off[b]; p < kept_off[b + 1]; p++) {
            int64_t e = seq_off[b] + kept_idx[p];
            memcpy(hot + p * row_bytes, cold + e * row_bytes, (size_t)row_bytes);
            slot_of[e] = (int32_t)p;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Core attention over the selected entries (section 2.1 "Tiered      */
/* Selection": "final core attention computation").  Multi-query:     */
/* every query head attends over the same selected K/V rows.          */
/*   a_i = scale * Q_h . K_i,  m = max_i a_i,  p_i = exp(a_i - m)     */
/*   o_h = sum_i p_i V_i / sum_i p_i,  lse_h = m + log(sum_i p_i)     */
/* With nothing selected, o_h = 0 and lse_h = -inf.                   */
/* ------------------------------------------------------------------ */

/* kv holds one row per entry on the flat entry axis, row_stride elements
 * apart; K of entry e starts at element e*row_stride + k_off and V at
 * e*row_stride + v_off.  sel[b*k + i] is a global entry index or -1. */
void orc_sparse_attn(const void *Q, int q_dtype, const void *kv, int kv_dtype,
                     int64_t row_stride, int64_t k_off, int64_t v_off,
                     const int64_t *sel, int B, int Hq, int D, int k,
                     double scale, double *out, double *lse)
{
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (int64_t)B * Hq; bh++) {
        int b = (int)(bh / Hq);
        const int64_t *rows = sel + (int64_t)b * k;
        double *a = (double *)malloc((size_t)(k > 0 ? k : 1) * sizeof *a);
        double *o = out + bh * D;
        double m = -INFINITY, l = 0.0;
        int i, c, n = 0;
        for (c = 0; c < D; c++)
            o[c] = 0.0;
        for (i = 0; i < k; i++) {
            double dot = 0.0;
            if (rows[i] < 0) {
                a[i] = -INFINITY;
                continue;
            }
            for (c = 0; c < D; c++)
                dot += load_elem(Q, q_dtype, bh * D + c) *
                       load_elem(kv, kv_dtype, rows[i] * row_stride + k_off + c);
            a[i] = scale * dot;
            if (a[i] > m)
                m = a[i];
            n++;
        }
        if (n == 0) {
            lse[bh] = -INFINITY;
            free(a);
            continue;
        }
        for (i = 0; i < k; i++) {
            double p;
            if (rows[i] < 0)
                continue;
            p = exp(a[i] - m);
            l += p;
            for (c = 0; c < D; c++)
                o[c] += p * load_elem(kv, kv_dtype, rows[i] * row_stride + v_off + c);
        }
        for (c = 0; c < D; c++)
            o[c] /= l;
        lse[bh] = m + log(l);
        free(a);
    }
}

/* Number of OpenMP threads this library will use. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
