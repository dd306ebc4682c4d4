/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for attention: the forward
 * pass (square and general shapes, causal, explicit mask, dropout) and its
 * gradients (the backward section below), with each function's definition
 * and sources stated where it is defined.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library
 * and its Python binding) may link, load or call this file.  It is used by
 * tests/, by the smoke check, and by the CPU-baseline leg of the benchmark.
 * It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (the definition, not an algorithm):
 *
 *   For every (b, h) and query row i in [0, S):
 *     s_ij  = scale * sum_d q_id * k_jd            for j in J_i
 *     m_i   = max_j s_ij
 *     p_ij  = exp(s_ij - m_i)
 *     l_i   = sum_j p_ij
 *     O_id  = (sum_j p_ij * v_jd) / l_i
 *     LSE_i = m_i + log(l_i)                      (natural log)
 *   where J_i = [0, S) without the causal mask and J_i = [0, i] with it.
 *
 *   Sources:
 *   - Scaled dot-product attention softmax(QK^T / sqrt(d_k)) V:
 *     "FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？深度拆解 ops-transformer 的实现",
 *     section 1 (the Attention(Q,K,V) equation); and
 *     "ops-transformer FlashAttention 算子实战：让昇腾NPU算力彻底释放",
 *     section 4.2 (the naive_attention comparison function).
 *   - Causal attention (each position sees only itself and earlier tokens):
 *     the gsyq.cn catlass page (13B service moved to Ascend), section
 *     "Causal Mask的实现差异"; and the ops-transformer page, section 4.1
 *     (causal=True for autoregressive models).
 *   - The log-sum-exp per row is not defined on the pages; it is read as the
 *     natural log of sum_j exp(s_ij) with s already scaled.
 *
 * The naive path materialises each query's full score row and runs a
 * two-pass softmax (max, then exp/sum).  The tiled path is a separately
 * written online-softmax recurrence that follows the page's section 2.1
 * (tiling) and 2.2 (online softmax) of the FlashAttention-2 page, in two forms:
 *   form 0: deferred normalisation (O and l rescaled by e^{m_old-m_new},
 *           one division by l at the end);
 *   form 1: the page's printed recurrence, which normalises at every step
 *           (p_j divided by l_new, O rescaled by (l_old/l_new) e^{m_old-m_new}).
 * With the causal mask the tiled path skips key tiles whose first key lies
 * after the last query of the query tile (mode 2 "对角线跳过" of the gsyq.cn
 * catlass page; the comparison operator is lost in the page's text and is
 * read as ">=").
 *
 * Inputs are the exact 16-bit values the GPU receives (IEEE binary16 or
 * bfloat16 bit patterns), decoded here to double by this file's own decoders.
 * All arithmetic is double precision; scale is the caller's float promoted
 * to double.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -o liboracle.so attn_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* ---------------------------------------------------------------- decoders */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0) {
        mag = ldexp((double)f, -24);            /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        mag = (f == 0) ? INFINITY : NAN;
    } else {
        mag = ldexp((double)(1024 + f), e - 25); /* (1 + f/2^10) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_f64(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double mag;
    if (e == 0) {
        mag = ldexp((double)f, -133);           /* f * 2^-126 * 2^-7 */
    } else if (e == 255) {
        mag = (f == 0) ? INFINITY : NAN;
    } else {
        mag = ldexp((double)(128 + f), e - 134); /* (1 + f/2^7) * 2^(e-127) */
    }
    return sign ? -mag : mag;
}

void oracle_decode(const uint16_t *src, double *dst, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = (dtype == ORACLE_BF16) ? oracle_bf16_to_f64(src[i]) : oracle_f16_to_f64(src[i]);
}

static int check_args(int64_t B, int64_t H, int64_t S, int64_t D, int dtype)
{
    if (B < 0 || H < 0 || S < 0 || D <= 0) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    return 0;
}

/* Decode one (b,h) slice [S, D] of a BHSD tensor. */
static double *decode_head(const uint16_t *x, int64_t bh, int64_t S, int64_t D, int dtype)
{
    double *out = (double *)malloc(sizeof(double) * (size_t)(S * D > 0 ? S * D : 1));
    if (!out) return NULL;
    oracle_decode(x + bh * S * D, out, S * D, dtype);
    return out;
}

/* ------------------------------------------------------- naive definition */

/*
 * One query row of the definition above.  qi: [D]; kh, vh: [S, D] decoded.
 * srow: scratch of length S (the materialised score row).
 */
static void naive_row(const double *qi, const double *kh, const double *vh, int64_t i, int64_t S,
                      int64_t D, double scale, int causal, double *srow, double *o, double *lse)
{
    int64_t nj = causal ? (i + 1 < S ? i + 1 : S) : S; /* J_i = [0, nj) */
    /* scores */
    for (int64_t j = 0; j < nj; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kh[j * D + d];
        srow[j] = scale * dot;
    }
    /* pass 1: max */
    double m = -INFINITY;
    for (int64_t j = 0; j < nj; ++j)
        if (srow[j] > m) m = srow[j];
    /* pass 2: exponentials and their sum */
    double l = 0.0;
    for (int64_t j = 0; j < nj; ++j) {
        srow[j] = exp(srow[j] - m);
        l += srow[j];
    }
    /* P V, then normalise */
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < nj; ++j) {
        double p = srow[j];
        for (int64_t d = 0; d < D; ++d) o[d] += p * vh[j * D + d];
    }
    for (int64_t d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
}

/*
 * Full naive attention.  q, k, v: BHSD 16-bit bit patterns.
 * o: [B,H,S,D] double, lse: [B,H,S] double.  Returns 0 or a negative code.
 */
int oracle_attn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                    int64_t S, int64_t D, float scale, int causal, int dtype, double *o, double *lse)
{
    int rc = check_args(B, H, S, D, dtype);
    if (rc) return rc;
    const double sc = (double)scale;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        double *qh = decode_head(q, bh, S, D, dtype);
        double *kh = decode_head(k, bh, S, D, dtype);
        double *vh = decode_head(v, bh, S, D, dtype);
        if (!qh || !kh || !vh) {
            free(qh); free(kh); free(vh);
            return -10;
        }
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < S; ++i)
                naive_row(qh + i * D, kh, vh, i, S, D, sc, causal, srow, o + (bh * S + i) * D,
                          lse + bh * S + i);
            free(srow);
        }
        free(qh); free(kh); free(vh);
    }
    return 0;
}

/*
 * The same definition for a list of (bh, i) rows only: used to check sampled
 * rows of full-size runs.  o: [nrows, D], lse: [nrows].
 */
int oracle_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                     int64_t S, int64_t D, float scale, int causal, int dtype, const int64_t *bh_idx,
                     const int64_t *row_idx, int64_t nrows, double *o, double *lse)
{
    int rc = check_args(B, H, S, D, dtype);
    if (rc) return rc;
    for (int64_t r = 0; r < nrows; ++r)
        if (bh_idx[r] < 0 || bh_idx[r] >= B * H || row_idx[r] < 0 || row_idx[r] >= S) return -2;
    const double sc = (double)scale;
    int bad = 0;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
        double *qi = (double *)malloc(sizeof(double) * (size_t)D);
        double *kh = (double *)malloc(sizeof(double) * (size_t)(S * D > 0 ? S * D : 1));
        double *vh = (double *)malloc(sizeof(double) * (size_t)(S * D > 0 ? S * D : 1));
        int64_t cur_bh = -1;
        if (!srow || !qi || !kh || !vh) {
#pragma omp atomic write
            bad = 1;
        }
        /* rows are expected grouped by bh; each thread decodes a head once per run of rows */
#pragma omp for schedule(static)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!srow || !qi || !kh || !vh) continue;
            int64_t bh = bh_idx[r], i = row_idx[r];
            if (bh != cur_bh) {
                oracle_decode(k + bh * S * D, kh, S * D, dtype);
                oracle_decode(v + bh * S * D, vh, S * D, dtype);
                cur_bh = bh;
            }
            oracle_decode(q + (bh * S + i) * D, qi, D, dtype);
            naive_row(qi, kh, vh, i, S, D, sc, causal, srow, o + r * D, lse + r);
        }
        free(srow); free(qi); free(kh); free(vh);
    }
    return bad ? -10 : 0;
}

/*
 * Softmax probabilities P [S, S] of one (b,h) slice (tiny sizes only), by the
 * definition above; masked entries are 0.
 */
int oracle_attn_probs(const uint16_t *q, const uint16_t *k, int64_t B, int64_t H, int64_t S,
                      int64_t D, float scale, int causal, int dtype, int64_t bh, double *p)
{
    int rc = check_args(B, H, S, D, dtype);
    if (rc) return rc;
    if (bh < 0 || bh >= B * H) return -2;
    double *qh = decode_head(q, bh, S, D, dtype);
    double *kh = decode_head(k, bh, S, D, dtype);
    if (!qh || !kh) { free(qh); free(kh); return -10; }
    const double sc = (double)scale;
    for (int64_t i = 0; i < S; ++i) {
        double *row = p + i * S;
        int64_t nj = causal ? i + 1 : S;
        double m = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
            if (j >= nj) { row[j] = -INFINITY; continue; }
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += qh[i * D + d] * kh[j * D + d];
            row[j] = sc * dot;
            if (row[j] > m) m = row[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < S; ++j) {
            row[j] = (j < nj) ? exp(row[j] - m) : 0.0;
            l += row[j];
        }
        for (int64_t j = 0; j < S; ++j) row[j] /= l;
    }
    free(qh); free(kh);
    return 0;
}

/* ------------------------------------------- tiled online-softmax reference */

/*
 * Causal mode 2 of the gsyq.cn catlass page: key tile tn is skipped for query
 * tile tm when its first key comes after the last query of the query tile.
 */
static int tile_skipped(int64_t tm, int64_t tn, int64_t Br, int64_t Bc)
{
    return tn * Bc >= (tm + 1) * Br;
}

/*
 * Tiled reference: Q in tiles of Br rows, K/V in tiles of Bc rows, an outer
 * loop over Q tiles and an inner loop over K/V tiles, with the running max m
 * and running sum l of the FlashAttention-2 page, section 2.2.
 * form 0: deferred normalisation.  form 1: the page's per-step normalised
 * recurrence.  Keys beyond S in a ragged last tile are not visited.
 */
int oracle_attn_tiled(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                      int64_t S, int64_t D, float scale, int causal, int dtype, int64_t Br,
                      int64_t Bc, int form, double *o, double *lse)
{
    int rc = check_args(B, H, S, D, dtype);
    if (rc) return rc;
    if (Br <= 0 || Bc <= 0 || (form != 0 && form != 1)) return -2;
    const double sc = (double)scale;
    const int64_t nq = (S + Br - 1) / Br, nk = (S + Bc - 1) / Bc;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        double *qh = decode_head(q, bh, S, D, dtype);
        double *kh = decode_head(k, bh, S, D, dtype);
        double *vh = decode_head(v, bh, S, D, dtype);
        if (!qh || !kh || !vh) { free(qh); free(kh); free(vh); return -10; }
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t tm = 0; tm < nq; ++tm) {
            int64_t r0 = tm * Br, r1 = (r0 + Br < S) ? r0 + Br : S;
            int64_t nr = r1 - r0;
            double *m = (double *)malloc(sizeof(double) * (size_t)nr);
            double *l = (double *)malloc(sizeof(double) * (size_t)nr);
            double *acc = (double *)calloc((size_t)(nr * D), sizeof(double));
            double *s = (double *)malloc(sizeof(double) * (size_t)Bc);
            for (int64_t r = 0; r < nr; ++r) { m[r] = -INFINITY; l[r] = 0.0; }
            for (int64_t tn = 0; tn < nk; ++tn) {
                if (causal && tile_skipped(tm, tn, Br, Bc)) continue;
                int64_t c0 = tn * Bc, c1 = (c0 + Bc < S) ? c0 + Bc : S;
                for (int64_t r = 0; r < nr; ++r) {
                    int64_t i = r0 + r;
                    /* score block row, masked entries -inf */
                    double bmax = -INFINITY;
                    for (int64_t j = c0; j < c1; ++j) {
                        double x = -INFINITY;
                        if (!causal || j <= i) {
                            double dot = 0.0;
                            for (int64_t d = 0; d < D; ++d) dot += qh[i * D + d] * kh[j * D + d];
                            x = sc * dot;
                        }
                        s[j - c0] = x;
                        if (x > bmax) bmax = x;
                    }
                    if (bmax == -INFINITY) continue; /* whole block masked for this row */
                    double m_old = m[r];
                    double m_new = (bmax > m_old) ? bmax : m_old;
                    double alpha = (m_old == -INFINITY) ? 0.0 : exp(m_old - m_new);
                    double psum = 0.0;
                    for (int64_t j = c0; j < c1; ++j) {
                        double e = (s[j - c0] == -INFINITY) ? 0.0 : exp(s[j - c0] - m_new);
                        s[j - c0] = e;
                        psum += e;
                    }
                    double l_new = alpha * l[r] + psum;
                    double *a = acc + r * D;
                    if (form == 0) {
                        for (int64_t d = 0; d < D; ++d) {
                            double pv = 0.0;
                            for (int64_t j = c0; j < c1; ++j) pv += s[j - c0] * vh[j * D + d];
                            a[d] = alpha * a[d] + pv;
                        }
                    } else {
                        /* o <- p_j v_j + (l_old / l_new) e^{m_old - m_new} o, p_j = e^{s-m_new}/l_new */
                        double keep = (l[r] == 0.0) ? 0.0 : (l[r] / l_new) * alpha;
                        for (int64_t d = 0; d < D; ++d) {
                            double pv = 0.0;
                            for (int64_t j = c0; j < c1; ++j) pv += (s[j - c0] / l_new) * vh[j * D + d];
                            a[d] = pv + keep * a[d];
                        }
                    }
                    m[r] = m_new;
                    l[r] = l_new;
                }
            }
            for (int64_t r = 0; r < nr; ++r) {
                int64_t i = r0 + r;
                for (int64_t d = 0; d < D; ++d)
                    o[(bh * S + i) * D + d] = (form == 0) ? acc[r * D + d] / l[r] : acc[r * D + d];
                lse[bh * S + i] = m[r] + log(l[r]);
            }
            free(m); free(l); free(acc); free(s);
        }
        free(qh); free(kh); free(vh);
    }
    return 0;
}

/* ------------------------------------------------------ causal tile counts */

/*
 * Brute-force count of (query tile, key tile) pairs for an S x S causal
 * problem with BM x BN tiles: a pair is "computed" when at least one of its
 * (i, j) elements has j <= i, else "skipped".  total = computed + skipped.
 * This is an element-by-element enumeration, independent of any loop bound.
 */
void oracle_causal_tile_count(int64_t S, int64_t BM, int64_t BN, int64_t *total, int64_t *computed,
                              int64_t *skipped)
{
    int64_t nq = (S + BM - 1) / BM, nk = (S + BN - 1) / BN;
    int64_t c = 0, s = 0;
    for (int64_t tm = 0; tm < nq; ++tm)
        for (int64_t tn = 0; tn < nk; ++tn) {
            int any = 0;
            for (int64_t i = tm * BM; i < (tm + 1) * BM && i < S && !any; ++i)
                for (int64_t j = tn * BN; j < (tn + 1) * BN && j < S; ++j)
                    if (j <= i) { any = 1; break; }
            if (any) ++c; else ++s;
        }
    *total = nq * nk;
    *computed = c;
    *skipped = s;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* -------------------------------------------- general shapes (Sq != Sk) */

/*
 * Cross-attention and offset causal masking: queries [B,H,Sq,D], keys and
 * values [B,H,Sk,D] (contiguous).  With the causal mask query i sees key j iff
 * j <= i + (Sk - Sq): the queries are the last Sq positions of the Sk keys
 * (bottom-right alignment; with Sq = Sk this is the mask above).  A query that
 * sees no key gets O = 0 and LSE = -inf (the log of an empty sum).
 * Same definition as oracle_attn_fwd otherwise.  Sources: text-to-image
 * cross-attention with 77 text tokens ("解析CANN ops-transformer的FlashAttention
 * 算子：注意力机制的内存优化", section "Stable Diffusion中的优化"); the causal
 * mask as in oracle_attn_fwd.  The pages do not say how a causal mask aligns
 * when Sq != Sk; the bottom-right reading (queries are the newest positions,
 * as in decoding with a cache) is taken.
 */
static void naive_row_gen(const double *qi, const double *kh, const double *vh, int64_t nj, int64_t D,
                          double scale, double *srow, double *o, double *lse)
{
    if (nj <= 0) {
        for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    for (int64_t j = 0; j < nj; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kh[j * D + d];
        srow[j] = scale * dot;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < nj; ++j)
        if (srow[j] > m) m = srow[j];
    double l = 0.0;
    for (int64_t j = 0; j < nj; ++j) {
        srow[j] = exp(srow[j] - m);
        l += srow[j];
    }
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < nj; ++j)
        for (int64_t d = 0; d < D; ++d) o[d] += srow[j] * vh[j * D + d];
    for (int64_t d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
}

static int64_t visible_keys(int64_t i, int64_t Sq, int64_t Sk, int causal)
{
    if (!causal) return Sk;
    int64_t n = i + (Sk - Sq) + 1;
    if (n < 0) n = 0;
    if (n > Sk) n = Sk;
    return n;
}

int oracle_attn_fwd_gen(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                        int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype, double *o,
                        double *lse)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    const double sc = (double)scale;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        double *qh = (double *)malloc(sizeof(double) * (size_t)(Sq * D > 0 ? Sq * D : 1));
        double *kh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        double *vh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        if (!qh || !kh || !vh) { free(qh); free(kh); free(vh); return -10; }
        oracle_decode(q + bh * Sq * D, qh, Sq * D, dtype);
        oracle_decode(k + bh * Sk * D, kh, Sk * D, dtype);
        oracle_decode(v + bh * Sk * D, vh, Sk * D, dtype);
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < Sq; ++i)
                naive_row_gen(qh + i * D, kh, vh, visible_keys(i, Sq, Sk, causal), D, sc, srow,
                              o + (bh * Sq + i) * D, lse + bh * Sq + i);
            free(srow);
        }
        free(qh); free(kh); free(vh);
    }
    return 0;
}

/* The general definition for a list of (bh, i) query rows only. */
int oracle_attn_rows_gen(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                         int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype,
                         const int64_t *bh_idx, const int64_t *row_idx, int64_t nrows, double *o, double *lse)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    for (int64_t r = 0; r < nrows; ++r)
        if (bh_idx[r] < 0 || bh_idx[r] >= B * H || row_idx[r] < 0 || row_idx[r] >= Sq) return -2;
    const double sc = (double)scale;
    int bad = 0;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
        double *qi = (double *)malloc(sizeof(double) * (size_t)D);
        double *kh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        double *vh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        int64_t cur_bh = -1;
        if (!srow || !qi || !kh || !vh) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(static)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!srow || !qi || !kh || !vh) continue;
            int64_t bh = bh_idx[r], i = row_idx[r];
            if (bh != cur_bh) {
                oracle_decode(k + bh * Sk * D, kh, Sk * D, dtype);
                oracle_decode(v + bh * Sk * D, vh, Sk * D, dtype);
                cur_bh = bh;
            }
            oracle_decode(q + (bh * Sq + i) * D, qi, D, dtype);
            naive_row_gen(qi, kh, vh, visible_keys(i, Sq, Sk, causal), D, sc, srow, o + r * D, lse + r);
        }
        free(srow); free(qi); free(kh); free(vh);
    }
    return bad ? -10 : 0;
}

/* ------------------------------------------------------------------ dropout */

/*
 * Attention dropout: after the softmax each weight P_ij is kept with
 * probability 1 - p and zeroed otherwise, and the kept weights are scaled by
 * 1 / (1 - p), so O_i = sum_j P_ij z_ij v_j with z_ij = keep_ij / (1 - p)
 * (an unbiased estimate of the undropped O).  The normalisation l and the
 * LSE are those of the undropped softmax.  Source: the fused dropout of the
 * FlashAttention-2 page, sections 3.4 and 6.3 (dropout_prob = 0.1 inside the
 * kernel, random numbers drawn on the device).  That page's listing writes
 * -infinity into the score before the softmax instead; that variant is the
 * explicit mask of oracle_attn_fwd_masked with a random mask.  The standard
 * reading (drop after the softmax, rescale the kept weights) is the one
 * taken here.
 *
 * The pages name no generator.  The keep decisions come from Philox4x32-10
 * (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2,
 * 3", SC 2011): for head bh = b * H + h, query row i and key j,
 *   counter = (j / 16, i, bh, offset), key = (seed mod 2^32, seed / 2^32),
 * and element j takes byte j mod 16 of the four 32-bit output words (word
 * (j mod 16) / 4, bits 8 (j mod 4) .. 8 (j mod 4) + 7).  It is kept iff that
 * byte is >= p8, the drop threshold in 1/256 units; the drop probability is
 * p8 / 256 and the kept weights are scaled by 256 / (256 - p8).
 */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

/* Ten rounds of the Philox-4x32 bijection; the key is bumped by the Weyl
 * constants before every round after the first. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        const uint64_t a = (uint64_t)PHILOX_M0 * x0;  /* hi/lo products of the two multipliers */
        const uint64_t b = (uint64_t)PHILOX_M1 * x2;
        const uint32_t y0 = (uint32_t)(b >> 32) ^ x1 ^ k0;
        const uint32_t y1 = (uint32_t)b;
        const uint32_t y2 = (uint32_t)(a >> 32) ^ x3 ^ k1;
        const uint32_t y3 = (uint32_t)a;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

static int dropout_keep(uint64_t seed, uint32_t offset, uint32_t p8, int64_t bh, int64_t i, int64_t j)
{
    const uint32_t ctr[4] = {(uint32_t)(j >> 4), (uint32_t)i, (uint32_t)bh, offset};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    const uint32_t byte = (w[(j & 15) >> 2] >> (8 * (j & 3))) & 0xffu;
    return byte >= p8;
}

/* keep[bh][i][j] (1 = kept) for tests; BH * Sq * Sk bytes. */
int oracle_dropout_keep_mask(int64_t BH, int64_t Sq, int64_t Sk, uint32_t p8, uint64_t seed, uint32_t offset,
                             uint8_t *keep)
{
    if (BH < 0 || Sq < 0 || Sk < 0 || p8 > 255) return -2;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < BH * Sq; ++r)
        for (int64_t j = 0; j < Sk; ++j) keep[r * Sk + j] = (uint8_t)dropout_keep(seed, offset, p8, r / Sq, r % Sq, j);
    return 0;
}

/* One query row with dropout: the softmax over the nj visible keys, then
 * O = sum_j P_j z_j v_j.  An empty row gets O = 0, LSE = -inf. */
static void dropout_row(const double *qi, const double *kh, const double *vh, int64_t nj, int64_t D, double scale,
                        uint64_t seed, uint32_t offset, uint32_t p8, int64_t bh, int64_t i, const uint8_t *mrow,
                        double *srow, double *o, double *lse)
{
    /* with an explicit mask the row sees only the keys its mask row allows */
    int64_t nvis = 0;
    for (int64_t j = 0; j < nj; ++j) nvis += mrow ? (mrow[j] != 0) : 1;
    if (nvis == 0) {
        for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    const double zs = 256.0 / (256.0 - (double)p8);
    for (int64_t j = 0; j < nj; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kh[j * D + d];
        srow[j] = (mrow && !mrow[j]) ? -INFINITY : scale * dot;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < nj; ++j)
        if (srow[j] > m) m = srow[j];
    double l = 0.0;
    for (int64_t j = 0; j < nj; ++j) {
        srow[j] = exp(srow[j] - m);
        l += srow[j];
    }
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < nj; ++j) {
        if (mrow && !mrow[j]) continue;
        if (!dropout_keep(seed, offset, p8, bh, i, j)) continue;
        const double w = srow[j] * zs;
        for (int64_t d = 0; d < D; ++d) o[d] += w * vh[j * D + d];
    }
    for (int64_t d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
}

/* Attention with dropout, general shapes and the bottom-right causal mask of
 * oracle_attn_fwd_gen, and optionally an explicit mask (the convention of
 * oracle_attn_fwd_masked; mask = NULL: none).  o: [B,H,Sq,D], lse: [B,H,Sq]. */
int oracle_attn_fwd_dropout_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                                   int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype,
                                   uint32_t p8, uint64_t seed, uint32_t offset, const uint8_t *mask, int64_t mask_sb,
                                   int64_t mask_sh, int64_t mask_si, double *o, double *lse)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0 || p8 > 255) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    const double sc = (double)scale;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        double *qh = (double *)malloc(sizeof(double) * (size_t)(Sq * D > 0 ? Sq * D : 1));
        double *kh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        double *vh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        if (!qh || !kh || !vh) { free(qh); free(kh); free(vh); return -10; }
        oracle_decode(q + bh * Sq * D, qh, Sq * D, dtype);
        oracle_decode(k + bh * Sk * D, kh, Sk * D, dtype);
        oracle_decode(v + bh * Sk * D, vh, Sk * D, dtype);
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < Sq; ++i)
                dropout_row(qh + i * D, kh, vh, visible_keys(i, Sq, Sk, causal), D, sc, seed, offset, p8, bh, i,
                            mask ? mask + (bh / H) * mask_sb + (bh % H) * mask_sh + i * mask_si : NULL, srow,
                            o + (bh * Sq + i) * D, lse + bh * Sq + i);
            free(srow);
        }
        free(qh); free(kh); free(vh);
    }
    return 0;
}

int oracle_attn_fwd_dropout(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                            int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype, uint32_t p8,
                            uint64_t seed, uint32_t offset, double *o, double *lse)
{
    return oracle_attn_fwd_dropout_masked(q, k, v, B, H, Sq, Sk, D, scale, causal, dtype, p8, seed, offset, NULL, 0,
                                          0, 0, o, lse);
}

/* The dropout definition for a list of (bh, i) query rows only.  Pinned bit for
 * bit against the rows of oracle_attn_fwd_dropout (square and Sq != Sk, causal
 * and not, several thresholds, seeds and offsets): the generator's counter takes
 * the query row i, never the position r in the list. */
int oracle_attn_rows_dropout(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                             int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype, uint32_t p8,
                             uint64_t seed, uint32_t offset, const int64_t *bh_idx, const int64_t *row_idx,
                             int64_t nrows, double *o, double *lse)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0 || p8 > 255) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    for (int64_t r = 0; r < nrows; ++r)
        if (bh_idx[r] < 0 || bh_idx[r] >= B * H || row_idx[r] < 0 || row_idx[r] >= Sq) return -2;
    const double sc = (double)scale;
    int bad = 0;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
        double *qi = (double *)malloc(sizeof(double) * (size_t)D);
        double *kh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        double *vh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
        int64_t cur_bh = -1;
        if (!srow || !qi || !kh || !vh) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(static)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!srow || !qi || !kh || !vh) continue;
            const int64_t bh = bh_idx[r], i = row_idx[r];
            if (bh != cur_bh) {
                oracle_decode(k + bh * Sk * D, kh, Sk * D, dtype);
                oracle_decode(v + bh * Sk * D, vh, Sk * D, dtype);
                cur_bh = bh;
            }
            oracle_decode(q + (bh * Sq + i) * D, qi, D, dtype);
            dropout_row(qi, kh, vh, visible_keys(i, Sq, Sk, causal), D, sc, seed, offset, p8, bh, i, NULL, srow,
                        o + r * D, lse + r);
        }
        free(srow); free(qi); free(kh); free(vh);
    }
    return bad ? -10 : 0;
}

/* ------------------------------------------------------------ backward pass */

/*
 * Gradients of the attention forward pass (general shapes, bottom-right causal
 * mask as in oracle_attn_fwd_gen) for an upstream gradient dO = dL/dO:
 *
 *   P_ij  = softmax_j(s_ij),  s_ij = scale * q_i . k_j  over the visible keys
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)      (the softmax Jacobian)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * This is the chain rule through the definition, written out; the backward
 * pass recomputes S and P from Q, K and the saved row statistics instead of
 * storing P ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", the
 * recomputation row of the core-optimisation table and section 6.2; the
 * backward configuration with a deterministic switch on the gsyq.cn catlass
 * page, "反向传播的特殊处理").  Here nothing is recomputed from saved state: every
 * quantity comes from q, k, v and dO in fp64.
 *
 * Optional outputs mag_dq, mag_dk, mag_dv (NULL to skip) hold the same sums
 * over absolute values, the scale of the rounding error a 16-bit evaluation
 * of each element can carry:
 *   mag_dV_j = sum_i P_ij |dO_i|
 *   mag_dQ_i = scale * sum_j P_ij (|dP_ij| + a_i) |k_j|
 *   mag_dK_j = scale * sum_i P_ij (|dP_ij| + a_i) |q_i|,
 *   a_i = sum_k P_ik |dP_ik| + 2 sum_d |dO_id| sum_k P_ik |v_kd|
 * (the second part of a_i scales the error of sum_k P_ik dP_ik when it is
 * formed as sum_d dO_id O_id from a forward output O whose own error is at
 * most twice the unit roundoff times sum_k P_ik |v_kd|: its weights and its
 * result are each rounded once).
 * Rows with no visible key have zero gradients.
 */
/* Key j is visible to query i of head (b, h): the causal rule, and the mask
 * entry when a mask is given (see oracle_attn_fwd_masked). */
static int bwd_visible(int64_t i, int64_t j, int64_t Sq, int64_t Sk, int causal, const uint8_t *mrow)
{
    if (j >= visible_keys(i, Sq, Sk, causal)) return 0;
    return mrow ? mrow[j] != 0 : 1;
}

/*
 * With dropout (drop != 0; the keep rule and scaling z_ij of the dropout
 * section above) the forward output is O_i = sum_j P_ij z_ij v_j, so
 *   dV_j  = sum_i P_ij z_ij dO_i
 *   dP_ij = z_ij (dO_i . v_j)       (the gradient reaching the weight P_ij)
 *   dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)
 * and sum_k P_ik dP_ik is again dO_i . O_i.  The magnitudes use the same
 * weights (P z in place of P where a value is multiplied by V or dO).
 */
static int attn_bwd_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout, int64_t B,
                         int64_t H, int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype,
                         const uint8_t *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si, int drop,
                         uint32_t p8, uint64_t seed, uint32_t offset, double *dq, double *dk, double *dv,
                         double *mag_dq, double *mag_dk, double *mag_dv)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0 || p8 > 255) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    const double sc = (double)scale;
    const double zs = 256.0 / (256.0 - (double)p8);
    const size_t szq = (size_t)(Sq * D > 0 ? Sq * D : 1), szk = (size_t)(Sk * D > 0 ? Sk * D : 1);
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const uint8_t *mhead = mask ? mask + (bh / H) * mask_sb + (bh % H) * mask_sh : NULL;
        double *qh = (double *)malloc(sizeof(double) * szq);
        double *oh = (double *)malloc(sizeof(double) * szq);
        double *kh = (double *)malloc(sizeof(double) * szk);
        double *vh = (double *)malloc(sizeof(double) * szk);
        double *lse = (double *)malloc(sizeof(double) * (size_t)(Sq > 0 ? Sq : 1));
        double *dsum = (double *)malloc(sizeof(double) * (size_t)(Sq > 0 ? Sq : 1));
        double *asum = (double *)malloc(sizeof(double) * (size_t)(Sq > 0 ? Sq : 1));
        if (!qh || !oh || !kh || !vh || !lse || !dsum || !asum) {
            free(qh); free(oh); free(kh); free(vh); free(lse); free(dsum); free(asum);
            return -10;
        }
        const int64_t Dd = D;
        oracle_decode(q + bh * Sq * D, qh, Sq * D, dtype);
        oracle_decode(dout + bh * Sq * D, oh, Sq * D, dtype);  /* oh holds dO */
        oracle_decode(k + bh * Sk * D, kh, Sk * D, dtype);
        oracle_decode(v + bh * Sk * D, vh, Sk * D, dtype);
        double *dqh = dq + bh * Sq * D, *dkh = dk + bh * Sk * D, *dvh = dv + bh * Sk * D;
        double *mqh = mag_dq ? mag_dq + bh * Sq * D : NULL;
        double *mkh = mag_dk ? mag_dk + bh * Sk * D : NULL;
        double *mvh = mag_dv ? mag_dv + bh * Sk * D : NULL;

        /* pass 1, per query row: P row, dP row, the row's softmax-Jacobian sum, dQ */
#pragma omp parallel
        {
            double *prow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
            double *dprow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
            double *zrow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < Sq; ++i) {
                const uint8_t *mrow = mhead ? mhead + i * mask_si : NULL;
                const int64_t nj = visible_keys(i, Sq, Sk, causal);
                const double *qi = qh + i * D, *doi = oh + i * D;
                for (int64_t d = 0; d < D; ++d) {
                    dqh[i * D + d] = 0.0;
                    if (mqh) mqh[i * D + d] = 0.0;
                }
                int64_t nvis = 0;
                for (int64_t j = 0; j < nj; ++j) nvis += bwd_visible(i, j, Sq, Sk, causal, mrow);
                if (nvis == 0) {
                    lse[i] = -INFINITY; dsum[i] = 0.0; asum[i] = 0.0;
                    continue;
                }
                double m = -INFINITY;
                for (int64_t j = 0; j < nj; ++j) {
                    if (!bwd_visible(i, j, Sq, Sk, causal, mrow)) {
                        prow[j] = -INFINITY;
                        dprow[j] = 0.0;
                        zrow[j] = 0.0;
                        continue;
                    }
                    double dot = 0.0, dp = 0.0;
                    for (int64_t d = 0; d < D; ++d) {
                        dot += qi[d] * kh[j * D + d];
                        dp += doi[d] * vh[j * D + d];
                    }
                    zrow[j] = drop ? (dropout_keep(seed, offset, p8, bh, i, j) ? zs : 0.0) : 1.0;
                    prow[j] = sc * dot;
                    dprow[j] = zrow[j] * dp;
                    if (prow[j] > m) m = prow[j];
                }
                double l = 0.0;
                for (int64_t j = 0; j < nj; ++j) {
                    prow[j] = exp(prow[j] - m);
                    l += prow[j];
                }
                double ds = 0.0, as = 0.0;
                for (int64_t j = 0; j < nj; ++j) {
                    prow[j] /= l;
                    ds += prow[j] * dprow[j];
                    as += prow[j] * fabs(dprow[j]);
                }
                /* 2 sum_d |dO_id| sum_j P_ij |v_jd| */
                for (int64_t d = 0; d < Dd; ++d) {
                    double od = 0.0;
                    for (int64_t j = 0; j < nj; ++j)
                        if (prow[j] > 0.0) od += prow[j] * zrow[j] * fabs(vh[j * D + d]);
                    as += 2.0 * fabs(doi[d]) * od;
                }
                lse[i] = m + log(l);
                dsum[i] = ds;
                asum[i] = as;
                for (int64_t j = 0; j < nj; ++j) {
                    const double g = sc * prow[j] * (dprow[j] - ds);
                    const double gm = sc * prow[j] * (fabs(dprow[j]) + as);
                    for (int64_t d = 0; d < D; ++d) {
                        dqh[i * D + d] += g * kh[j * D + d];
                        if (mqh) mqh[i * D + d] += gm * fabs(kh[j * D + d]);
                    }
                }
            }
            free(prow); free(dprow); free(zrow);
        }
        /* pass 2, per key: dK and dV over the queries that see it */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t j = 0; j < Sk; ++j) {
            const double *kj = kh + j * D, *vj = vh + j * D;
            for (int64_t d = 0; d < D; ++d) {
                dkh[j * D + d] = 0.0;
                dvh[j * D + d] = 0.0;
                if (mkh) mkh[j * D + d] = 0.0;
                if (mvh) mvh[j * D + d] = 0.0;
            }
            for (int64_t i = 0; i < Sq; ++i) {
                if (!bwd_visible(i, j, Sq, Sk, causal, mhead ? mhead + i * mask_si : NULL)) continue;
                const double *qi = qh + i * D, *doi = oh + i * D;
                double dot = 0.0, dp = 0.0;
                for (int64_t d = 0; d < D; ++d) {
                    dot += qi[d] * kj[d];
                    dp += doi[d] * vj[d];
                }
                const double p = exp(sc * dot - lse[i]);
                const double z = drop ? (dropout_keep(seed, offset, p8, bh, i, j) ? zs : 0.0) : 1.0;
                dp *= z;
                const double g = sc * p * (dp - dsum[i]);
                const double gm = sc * p * (fabs(dp) + asum[i]);
                for (int64_t d = 0; d < D; ++d) {
                    dkh[j * D + d] += g * qi[d];
                    dvh[j * D + d] += p * z * doi[d];
                    if (mkh) mkh[j * D + d] += gm * fabs(qi[d]);
                    if (mvh) mvh[j * D + d] += p * z * fabs(doi[d]);
                }
            }
        }
        free(qh); free(oh); free(kh); free(vh); free(lse); free(dsum); free(asum);
    }
    return 0;
}

int oracle_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout, int64_t B,
                    int64_t H, int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype, double *dq,
                    double *dk, double *dv, double *mag_dq, double *mag_dk, double *mag_dv)
{
    return attn_bwd_impl(q, k, v, dout, B, H, Sq, Sk, D, scale, causal, dtype, NULL, 0, 0, 0, 0, 0, 0, 0, dq, dk, dv,
                         mag_dq, mag_dk, mag_dv);
}

/* The gradients of oracle_attn_fwd_dropout_masked (mask = NULL: none). */
int oracle_attn_bwd_dropout_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                                   int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D, float scale, int causal,
                                   int dtype, uint32_t p8, uint64_t seed, uint32_t offset, const uint8_t *mask,
                                   int64_t mask_sb, int64_t mask_sh, int64_t mask_si, double *dq, double *dk,
                                   double *dv, double *mag_dq, double *mag_dk, double *mag_dv)
{
    return attn_bwd_impl(q, k, v, dout, B, H, Sq, Sk, D, scale, causal, dtype, mask, mask_sb, mask_sh, mask_si, 1, p8,
                         seed, offset, dq, dk, dv, mag_dq, mag_dk, mag_dv);
}

/* The gradients of the attention with dropout of oracle_attn_fwd_dropout. */
int oracle_attn_bwd_dropout(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                            int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D, float scale, int causal,
                            int dtype, uint32_t p8, uint64_t seed, uint32_t offset, double *dq, double *dk,
                            double *dv, double *mag_dq, double *mag_dk, double *mag_dv)
{
    return attn_bwd_impl(q, k, v, dout, B, H, Sq, Sk, D, scale, causal, dtype, NULL, 0, 0, 0, 1, p8, seed, offset,
                         dq, dk, dv, mag_dq, mag_dk, mag_dv);
}

/* The gradients of the masked attention of oracle_attn_fwd_masked (same mask
 * convention); masked pairs contribute nothing, rows with no visible key get no
 * gradient. */
int oracle_attn_bwd_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                           int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D, float scale, int causal,
                           int dtype, const uint8_t *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si,
                           double *dq, double *dk, double *dv, double *mag_dq, double *mag_dk, double *mag_dv)
{
    return attn_bwd_impl(q, k, v, dout, B, H, Sq, Sk, D, scale, causal, dtype, mask, mask_sb, mask_sh, mask_si, 0, 0,
                         0, 0, dq, dk, dv, mag_dq, mag_dk, mag_dv);
}

/* ------------------------------------------------------------ explicit mask */

/*
 * The general definition with an explicit boolean mask: query i of head (b, h)
 * sees key j iff mask[b][h][i][j] != 0 (and, with causal = 1, j <= i + Sk - Sq).
 * The mask is uint8 with element strides mask_sb, mask_sh, mask_si over b, h
 * and the query row (0 broadcasts) and contiguous keys.  A row that sees no key
 * gets O = 0 and LSE = -inf.  Sources: the fused mask of the FlashAttention-2
 * page, section 3.4 (a score whose mask entry is false becomes -infinity
 * before the softmax); the explicit mask matrix of the gsyq.cn catlass page
 * ("Causal Mask的实现差异", mode 1).
 */
int oracle_attn_fwd_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B, int64_t H,
                           int64_t Sq, int64_t Sk, int64_t D, float scale, int causal, int dtype,
                           const uint8_t *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si, double *o,
                           double *lse)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0) return -2;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -4;
    const double sc = (double)scale;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            const int64_t bh = b * H + h;
            double *qh = (double *)malloc(sizeof(double) * (size_t)(Sq * D > 0 ? Sq * D : 1));
            double *kh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
            double *vh = (double *)malloc(sizeof(double) * (size_t)(Sk * D > 0 ? Sk * D : 1));
            if (!qh || !kh || !vh) { free(qh); free(kh); free(vh); return -10; }
            oracle_decode(q + bh * Sq * D, qh, Sq * D, dtype);
            oracle_decode(k + bh * Sk * D, kh, Sk * D, dtype);
            oracle_decode(v + bh * Sk * D, vh, Sk * D, dtype);
#pragma omp parallel
            {
                double *srow = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
                int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Sk > 0 ? Sk : 1));
#pragma omp for schedule(dynamic, 16)
                for (int64_t i = 0; i < Sq; ++i) {
                    const uint8_t *mrow = mask + b * mask_sb + h * mask_sh + i * mask_si;
                    const int64_t nvis = visible_keys(i, Sq, Sk, causal);
                    int64_t n = 0;
                    for (int64_t j = 0; j < nvis; ++j)
                        if (mrow[j]) idx[n++] = j;
                    double *oi = o + (bh * Sq + i) * D;
                    if (n == 0) {
                        for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
                        lse[bh * Sq + i] = -INFINITY;
                        continue;
                    }
                    double m = -INFINITY;
                    for (int64_t t = 0; t < n; ++t) {
                        double dot = 0.0;
                        for (int64_t d = 0; d < D; ++d) dot += qh[i * D + d] * kh[idx[t] * D + d];
                        srow[t] = sc * dot;
                        if (srow[t] > m) m = srow[t];
                    }
                    double l = 0.0;
                    for (int64_t t = 0; t < n; ++t) {
                        srow[t] = exp(srow[t] - m);
                        l += srow[t];
                    }
                    for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
                    for (int64_t t = 0; t < n; ++t)
                        for (int64_t d = 0; d < D; ++d) oi[d] += srow[t] * vh[idx[t] * D + d];
                    for (int64_t d = 0; d < D; ++d) oi[d] /= l;
                    lse[bh * Sq + i] = m + log(l);
                }
                free(srow); free(idx);
            }
            free(qh); free(kh); free(vh);
        }
    return 0;
}
