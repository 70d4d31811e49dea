/*
 * Plain CPU oracle for the DeepSeek Sparse Attention (DSA) layer step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Every quantity is accumulated in double.  Inputs arrive as raw buffers
 * tagged with a storage type (fp32, bf16 bit patterns, or e4m3 codes) and
 * are widened exactly to double on load.  The work is split into
 * independent query rows, each given as a (batch, query) pair, so a caller
 * can check a sample of rows of a large problem.
 *
 * Sources (the DeepSeek-V3.2 model documentation page of Transformers):
 *   [DSA-1]  section "DeepSeek Sparse Attention (DSA)", item 1, Lightning
 *            indexer: an index score between each query and all previous
 *            keys; the reference runs it in FP8 after an orthogonal
 *            Hadamard rotation, Hq.Hk = q.k.
 *   [DSA-2]  same section, item 2, fine-grained token selection: keep the
 *            top index_topk tokens per query; main MLA attention then runs
 *            over those tokens only (additive mask in the port, O(index_topk)
 *            per query with a sparse kernel).
 *   [DSA-C]  same section, paragraph on the indexer's own single-head key
 *            cache of width index_head_dim.
 *   [CFG]    section DeepseekV32Config: index_topk 2048, index_head_dim 128,
 *            index_n_heads 64, num_attention_heads 128, kv_lora_rank 512,
 *            qk_rope_head_dim 64.
 *   [USE]    section "Usage example": the indexer's weights_proj stays out of
 *            FP8 quantisation.
 *   [PROJ]   the note on the query LoRA path (the indexer scores queries from
 *            the low-rank latent q_a_layernorm(q_a_proj(x)) through `wq_b`,
 *            sized by q_lora_rank) with [CFG] and [USE]: the indexer's
 *            projections are plain linear maps kept in bf16.
 * The score's combination rule (per-head ReLU of the query-key dot product,
 * summed over index heads with the weights_proj outputs as weights) is a
 * reading of [DSA-1] + [USE]; the pages do not print the formula.
 *
 * Parity status of each function is stated at the function.  The FP8
 * indexer path is pinned only by identities (exactly representable inputs,
 * an error bound), never by printed values: the pages print none.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2 };

/* ---------------------------------------------------------------- loads -- */

static double orc_e4m3_decode_d(uint8_t c);

/* Widen element i of a typed buffer to double (exact for all three types). */
static double orc_load(const void *p, int dtype, int64_t i)
{
    if (dtype == ORC_F32) {
        return (double)((const float *)p)[i];
    } else if (dtype == ORC_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    } else {
        return orc_e4m3_decode_d(((const uint8_t *)p)[i]);
    }
}

/* ------------------------------------------------------ indexer scores -- */

/*
 * Lightning-indexer scores [DSA-1], over the single-head key cache [DSA-C].
 *
 * For each requested row r = (b, t), with query position p = q_pos0[b] + t
 * and cache length L = ctx_len[b], and for every key s < L:
 *     s <= p :  I[s] = sum_h  w[b,t,h] * max(0, scale * <q[b,t,h,:], k[b,s,:]>)
 *     s >  p :  I[s] = -inf           (only previous keys are scored)
 * Entries s >= L are set to NaN (not part of the result).
 *
 * Layouts: q [B][n_q][H][D], k [B][s_max][D], w [B][n_q][H] (fp32),
 * out [nrows][s_max] doubles.
 * Parity pins: H = 1 / w = 1 reduces to ReLU(Q K^T) (checked against a BLAS
 * matmul), one-hot w picks out one head, linearity and sign symmetry in w.
 */
void orc_indexer_scores(int n_q, int s_max, int H, int D,
                        const void *q, int q_dtype,
                        const void *k, int k_dtype,
                        const float *w,
                        const int32_t *ctx_len, const int32_t *q_pos0,
                        double scale,
                        int nrows, const int32_t *row_b, const int32_t *row_t,
                        double *out)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int b = row_b[r], t = row_t[r];
        const int p = q_pos0[b] + t;
        const int L = ctx_len[b];
        double *o = out + (int64_t)r * s_max;
        const int64_t qbase = ((int64_t)b * n_q + t) * H * D;
        const int64_t wbase = ((int64_t)b * n_q + t) * H;
        for (int s = 0; s < s_max; ++s) {
            if (s >= L) { o[s] = NAN; continue; }
            if (s > p) { o[s] = -INFINITY; continue; }
            const int64_t kbase = ((int64_t)b * s_max + s) * D;
            double acc = 0.0;
            for (int h = 0; h < H; ++h) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += orc_load(q, q_dtype, qbase + (int64_t)h * D + d) *
                           orc_load(k, k_dtype, kbase + d);
                double v = scale * dot;
                acc += (double)w[wbase + h] * (v > 0.0 ? v : 0.0);
            }
            o[s] = acc;
        }
    }
}

/* ------------------------------------------------- Hadamard rotation -- */

/*
 * y = H x for the n-point Sylvester-Hadamard matrix scaled to be
 * orthonormal: H[i][j] = (-1)^popcount(i & j) / sqrt(n), n a power of two.
 * This is the orthogonal rotation of [DSA-1] (Hq.Hk = q.k); the pages name
 * the transform but not its size or scaling, which are readings (128 points,
 * 1/sqrt(n)).  Written as the plain matrix-vector product from the entry
 * formula, O(n^2), not as a fast transform.
 * Parity pins: equals scipy.linalg.hadamard(n)/sqrt(n) applied by matmul,
 * H H = I, and dot products are preserved.
 */
void orc_hadamard(int n, int64_t rows, const double *x, double *y)
{
    const double inv = 1.0 / sqrt((double)n);
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * n;
        double *yr = y + r * n;
        for (int i = 0; i < n; ++i) {
            double acc = 0.0;
            for (int j = 0; j < n; ++j) {
                int sgn = __builtin_popcount((unsigned)(i & j)) & 1;
                acc += sgn ? -xr[j] : xr[j];
            }
            yr[i] = acc * inv;
        }
    }
}

/* ------------------------------------------------------------- e4m3 -- */

/*
 * OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN, so the largest
 * finite magnitude is 1.75 * 2^8 = 448; the smallest normal is 2^-6 and the
 * smallest subnormal 2^-9.  Written from that definition.
 */
static double orc_e4m3_decode_d(uint8_t c)
{
    const int sign = c >> 7;
    const int e = (c >> 3) & 0xF;
    const int m = c & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                 /* subnormal: m/8 * 2^-6 */
    else        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

double orc_e4m3_decode(uint8_t c) { return orc_e4m3_decode_d(c); }

/*
 * Round a finite double to E4M3 with round-to-nearest-even and saturation
 * to +-448 ("satfinite").  NaN input returns the NaN code 0x7F.
 */
uint8_t orc_e4m3_encode(double x)
{
    if (isnan(x)) return 0x7F;
    const int sign = signbit(x) ? 1 : 0;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)((sign << 7) | (0xF << 3) | 0x6);
    /* quantum of the binade that holds a (subnormal binade below 2^-6) */
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) -> floor(log2 a) = e2 - 1 */
    int ex = e2 - 1;
    if (a == 0.0 || ex < -6) ex = -6;
    const double quantum = ldexp(1.0, ex - 3);
    double r = a / quantum;       /* exact: scaling by a power of two */
    double fl = floor(r);
    double frac = r - fl;
    double n;
    if (frac > 0.5) n = fl + 1.0;
    else if (frac < 0.5) n = fl;
    else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;   /* tie: to even */
    double v = n * quantum;
    if (v > 448.0) v = 448.0;     /* cannot happen below 448, kept for clarity */
    uint8_t code;
    if (v < ldexp(1.0, -6)) {
        code = (uint8_t)(v / ldexp(1.0, -9));           /* subnormal or zero */
    } else {
        int e3;
        double f = frexp(v, &e3);  /* v = f * 2^e3, f in [0.5,1) */
        int E = e3 - 1;            /* v = (2f) * 2^E, 2f in [1,2) */
        int M = (int)((2.0 * f - 1.0) * 8.0);
        code = (uint8_t)(((E + 7) << 3) | M);
    }
    return (uint8_t)((sign << 7) | code);
}

void orc_e4m3_encode_array(int64_t n, const double *x, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

void orc_e4m3_decode_array(int64_t n, const uint8_t *c, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode_d(c[i]);
}

/*
 * FP8 quantisation of rows for the FP8 indexer of [DSA-1]: rotate each
 * n-vector by H, take sigma = max|Hx| / 448 (sigma = 1 for an all-zero
 * row), store sigma as fp32, and code each element as e4m3(Hx / sigma) with
 * that fp32 sigma.  Per-row scales (one per key token, one per query head)
 * are a reading: the pages say "FP8" only.
 * Also returns the unrounded quotient Hx / sigma (fp64) so a test can tell a
 * rounding-boundary case from a real mismatch.
 */
void orc_hadamard_quant_rows(int n, int64_t rows, const void *x, int x_dtype,
                             uint8_t *code, float *sigma, double *quotient)
{
    #pragma omp parallel
    {
        double *xr = (double *)malloc(sizeof(double) * n);
        double *yr = (double *)malloc(sizeof(double) * n);
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int i = 0; i < n; ++i) xr[i] = orc_load(x, x_dtype, r * n + i);
            orc_hadamard(n, 1, xr, yr);
            double amax = 0.0;
            for (int i = 0; i < n; ++i) amax = fmax(amax, fabs(yr[i]));
            float s = (amax > 0.0) ? (float)(amax / 448.0) : 1.0f;
            sigma[r] = s;
            for (int i = 0; i < n; ++i) {
                double qv = yr[i] / (double)s;
                if (quotient) quotient[r * n + i] = qv;
                code[r * n + i] = orc_e4m3_encode(qv);
            }
        }
        free(xr);
        free(yr);
    }
}

/*
 * FP8 indexer scores: as orc_indexer_scores, with q and k given as e4m3
 * codes plus per-row scales, the dot product taken on the decoded codes and
 * multiplied back by sigma_q[b,t,h] * sigma_k[b,s]:
 *     I[s] = sum_h w * max(0, scale * sq * sk * <q^, k^>)        (s <= p)
 * Layouts: qc [B][n_q][H][D], qs [B][n_q][H], kc [B][s_max][D], ks [B][s_max].
 */
void orc_indexer_scores_fp8(int n_q, int s_max, int H, int D,
                            const uint8_t *qc, const float *qs,
                            const uint8_t *kc, const float *ks,
                            const float *w,
                            const int32_t *ctx_len, const int32_t *q_pos0,
                            double scale,
                            int nrows, const int32_t *row_b, const int32_t *row_t,
                            double *out)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int b = row_b[r], t = row_t[r];
        const int p = q_pos0[b] + t;
        const int L = ctx_len[b];
        double *o = out + (int64_t)r * s_max;
        const int64_t qrow = ((int64_t)b * n_q + t) * H;
        for (int s = 0; s < s_max; ++s) {
            if (s >= L) { o[s] = NAN; continue; }
            if (s > p) { o[s] = -INFINITY; continue; }
            const int64_t krow = (int64_t)b * s_max + s;
            double acc = 0.0;
            for (int h = 0; h < H; ++h) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += orc_e4m3_decode_d(qc[(qrow + h) * D + d]) *
                           orc_e4m3_decode_d(kc[krow * D + d]);
                double v = scale * (double)qs[qrow + h] * (double)ks[krow] * dot;
                acc += (double)w[qrow + h] * (v > 0.0 ? v : 0.0);
            }
            o[s] = acc;
        }
    }
}

/* ------------------------------------------------------------- top-k -- */

typedef struct { float v; int32_t s; } orc_pair;

/* Order: larger score first; equal scores (including -0 == +0) by lower index. */
static int orc_pair_cmp(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

static int orc_int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Fine-grained token selection [DSA-2]: for each row with query position p,
 * the candidates are the previous keys s in [0, p]; keep the min(k, p+1)
 * best by (score descending, index ascending) -- the tie rule toward the
 * lower index is a reading; the pages are silent on ties.  The kept set
 * is written in ascending index order, padded with -1 to k entries.
 * Scores are fp32 (the precision the selection is decided in) and must be
 * finite for s <= p.
 * Layout: scores [nrows][ld] (row r holds the scores of query row r),
 * pos [nrows], idx [nrows][k].  Returns the number of rows that held a
 * non-finite candidate score (0 on success).
 * Parity pins: numpy lexsort brute force on small rows, ties, signed zeros.
 */
int orc_topk(int nrows, int64_t ld, const float *scores, const int32_t *pos,
             int k, int32_t *idx)
{
    int bad = 0;
    #pragma omp parallel reduction(+:bad)
    {
        orc_pair *buf = NULL;
        int cap = 0;
        #pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            const int n = pos[r] + 1;
            if (n > cap) { free(buf); cap = n; buf = (orc_pair *)malloc(sizeof(orc_pair) * cap); }
            const float *row = scores + (int64_t)r * ld;
            for (int s = 0; s < n; ++s) {
                if (!isfinite(row[s])) bad += 1;
                buf[s].v = row[s];
                buf[s].s = s;
            }
            qsort(buf, (size_t)n, sizeof(orc_pair), orc_pair_cmp);
            const int c = n < k ? n : k;
            int32_t *o = idx + (int64_t)r * k;
            for (int j = 0; j < c; ++j) o[j] = buf[j].s;
            qsort(o, (size_t)c, sizeof(int32_t), orc_int_cmp);
            for (int j = c; j < k; ++j) o[j] = -1;
        }
        free(buf);
    }
    return bad;
}

/* --------------------------------------------------------- attention -- */

/*
 * Attention of one query row over the keys listed in idx (entries < 0 are
 * skipped) -- the "attention only over the selected tokens" of [DSA-2].
 * Head h reads KV head g = h / (H / KVH).  Logits l_j = sm_scale * <q_h, K_j>,
 * softmax over the listed keys, O_h = sum_j softmax_j * V_j.
 * V is v[b,s,g,:] when v is given, else the first d_v columns of kv (the
 * absorbed MLA form: one shared latent row per token, value = its first
 * kv_lora_rank columns, [CFG]).
 * lse_h = max_j l_j + log(sum_j exp(l_j - max)); rows with no listed key
 * give O = 0 and lse = -inf.
 * Layouts: q [B][n_q][H][d_qk], kv [B][s_max][KVH][d_qk],
 * v [B][s_max][KVH][d_v] or NULL, idx [nrows][k], out [nrows][H][d_v],
 * lse [nrows][H] (may be NULL).
 * Parity pins: with every previous key listed it equals causal dense
 * softmax attention (torch's scaled_dot_product_attention in fp64); one key
 * gives V of that key; q = 0 gives the mean of the listed V rows; it equals
 * orc_dense_masked_attn on the same list.
 */
void orc_sparse_attn(int n_q, int s_max, int H, int KVH, int d_qk, int d_v,
                     const void *q, int q_dtype,
                     const void *kv, int kv_dtype,
                     const void *v, int v_dtype,
                     const int32_t *idx, int k, double sm_scale,
                     int nrows, const int32_t *row_b, const int32_t *row_t,
                     double *out, double *lse)
{
    #pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (k > 0 ? k : 1));
        #pragma omp for schedule(dynamic, 1) collapse(2)
        for (int r = 0; r < nrows; ++r) {
            for (int h = 0; h < H; ++h) {
                const int b = row_b[r], t = row_t[r];
                const int g = h / (H / KVH);
                const int32_t *sel = idx + (int64_t)r * k;
                const int64_t qb = (((int64_t)b * n_q + t) * H + h) * d_qk;
                double *o = out + ((int64_t)r * H + h) * d_v;
                double m = -INFINITY;
                for (int j = 0; j < k; ++j) {
                    if (sel[j] < 0) continue;
                    const int64_t kb = (((int64_t)b * s_max + sel[j]) * KVH + g) * d_qk;
                    double dot = 0.0;
                    for (int d = 0; d < d_qk; ++d)
                        dot += orc_load(q, q_dtype, qb + d) * orc_load(kv, kv_dtype, kb + d);
                    logit[j] = sm_scale * dot;
                    if (logit[j] > m) m = logit[j];
                }
                for (int c = 0; c < d_v; ++c) o[c] = 0.0;
                if (m == -INFINITY) {
                    if (lse) lse[(int64_t)r * H + h] = -INFINITY;
                    continue;
                }
                double denom = 0.0;
                for (int j = 0; j < k; ++j) {
                    if (sel[j] < 0) continue;
                    const double pj = exp(logit[j] - m);
                    denom += pj;
                    for (int c = 0; c < d_v; ++c) {
                        double vv = v ? orc_load(v, v_dtype, (((int64_t)b * s_max + sel[j]) * KVH + g) * d_v + c)
                                      : orc_load(kv, kv_dtype, (((int64_t)b * s_max + sel[j]) * KVH + g) * d_qk + c);
                        o[c] += pj * vv;
                    }
                }
                for (int c = 0; c < d_v; ++c) o[c] /= denom;
                if (lse) lse[(int64_t)r * H + h] = m + log(denom);
            }
        }
        free(logit);
    }
}

/*
 * The Transformers port's form of the same attention [DSA-2]: dense softmax
 * over every previous key s in [0, p], with an additive mask of 0 for keys
 * in the selected list and -inf for the rest.  Cost O(p) per query; it must
 * agree with orc_sparse_attn on the same list (to rounding).
 */
void orc_dense_masked_attn(int n_q, int s_max, int H, int KVH, int d_qk, int d_v,
                           const void *q, int q_dtype,
                           const void *kv, int kv_dtype,
                           const void *v, int v_dtype,
                           const int32_t *q_pos0,
                           const int32_t *idx, int k, double sm_scale,
                           int nrows, const int32_t *row_b, const int32_t *row_t,
                           double *out)
{
    #pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * s_max);
        double *mask = (double *)malloc(sizeof(double) * s_max);
        #pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            const int b = row_b[r], t = row_t[r];
            const int p = q_pos0[b] + t;
            for (int s = 0; s <= p; ++s) mask[s] = -INFINITY;
            for (int j = 0; j < k; ++j) {
                int s = idx[(int64_t)r * k + j];
                if (s >= 0 && s <= p) mask[s] = 0.0;
            }
            for (int h = 0; h < H; ++h) {
                const int g = h / (H / KVH);
                const int64_t qb = (((int64_t)b * n_q + t) * H + h) * d_qk;
                double *o = out + ((int64_t)r * H + h) * d_v;
                double m = -INFINITY;
                for (int s = 0; s <= p; ++s) {
                    const int64_t kb = (((int64_t)b * s_max + s) * KVH + g) * d_qk;
                    double dot = 0.0;
                    for (int d = 0; d < d_qk; ++d)
                        dot += orc_load(q, q_dtype, qb + d) * orc_load(kv, kv_dtype, kb + d);
                    logit[s] = sm_scale * dot + mask[s];
                    if (logit[s] > m) m = logit[s];
                }
                for (int c = 0; c < d_v; ++c) o[c] = 0.0;
                if (m == -INFINITY) continue;
                double denom = 0.0;
                for (int s = 0; s <= p; ++s) {
                    const double pj = exp(logit[s] - m);   /* exp(-inf) = 0 */
                    denom += pj;
                    for (int c = 0; c < d_v; ++c) {
                        double vv = v ? orc_load(v, v_dtype, (((int64_t)b * s_max + s) * KVH + g) * d_v + c)
                                      : orc_load(kv, kv_dtype, (((int64_t)b * s_max + s) * KVH + g) * d_qk + c);
                        o[c] += pj * vv;
                    }
                }
                for (int c = 0; c < d_v; ++c) o[c] /= denom;
            }
        }
        free(logit);
        free(mask);
    }
}

/* ------------------------------------------------------ projections -- */

/*
 * The indexer's linear projections [PROJ]: Y = X W^T, written out,
 *     Y[m][n] = sum_k X[m][k] * W[n][k],
 * with X [M][K] and W [N][K] in a stored type (fp32 or bf16 bits), summed in
 * double.  wq_b maps the query latent (K = q_lora_rank = 1536) to the
 * H_I * D_I = 64 * 128 index-query columns; the key projection and
 * weights_proj map the hidden state (K = hidden_size = 7168) to the D_I = 128
 * key columns and the H_I = 64 head weights.  Parity: pinned against a BLAS
 * matrix product and exact special cases (tests/test_oracle_pins.py).
 */
void orc_linear(int64_t M, int N, int K, const void *x, int x_dtype, const void *w, int w_dtype, double *y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += orc_load(x, x_dtype, m * K + k) * orc_load(w, w_dtype, (int64_t)n * K + k);
            y[m * N + n] = acc;
        }
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
