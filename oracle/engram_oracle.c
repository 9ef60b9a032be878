/*
 * engram_oracle.c -- CPU oracle for the Engram N-gram Embedding ("ple") path.
 *
 * TEST INFRASTRUCTURE ONLY. Plain, slow, scalar C that the parity tests, the
 * smoke check and the CPU-baseline leg of the benchmark compare the CUDA path
 * against. It shares no code, header, table or constant with the CUDA library
 * and is never called by the product path.
 *
 * Source: the Qwen3.8-Flash-Next engram API page (NeMo AutoModel docs),
 * class Qwen3_8_FlashNextNGramEmbedding and its methods
 * _shift_right_after_eos, _hash_input_ids, _lookup_ngram_ids and forward,
 * and class Qwen3_8_FlashNextOwnerShardedEmbedding (an owner accumulates each
 * row's gradient). Readings taken where the page is silent or cut short:
 *   - per-token terms are combined by XOR of wrapped int64 products
 *     (the page's "original DeepSeek Engram" lineage; not printed);
 *   - multiplier k multiplies the token k positions back (k = 0: current);
 *   - all heads of one order share that order's mix; heads differ only in
 *     their prime modulus and global offset;
 *   - positions lacking valid context read the value `fill` (0 by default;
 *     the page's sentence is cut off);
 *   - context also resets at every sequence start given by cu_seqlens;
 *   - backward: one fp64 sum per distinct row over its lookups in ascending
 *     lookup order, rounded once to fp32; rows reported in ascending order.
 *
 * The PLE section follows the same page's Qwen3_8_FlashNextPLELayer
 * (norm_conv, conv1d with short_conv_dilation = ngram_size, _causal_short_conv
 * with left zero history, init_weights' zero-start convolution) and the layers
 * page's Qwen3_8_FlashNextGroupedRMSNorm (Gemma-style, additive scale that
 * starts at zero, groups of group_size features). Readings taken there:
 *   - norm_conv normalises the convolution's input;
 *   - the convolution's history is zero before every start in cu_seqlens;
 *   - the optional SiLU and residual follow the Engram paper the page cites
 *     (output = x + SiLU(conv(norm(x)))); the page itself prints neither;
 *   - the tail's backward (for training the layer) is the chain rule through
 *     those same steps; the pages print no backward, so it has no reading of
 *     its own beyond the forward's.
 *
 * Parity of the hash against the released checkpoint is unpinned: the page
 * prints no worked example (see the tests for what does pin each function).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ORACLE_MUTANT (tests only) plants one known mistake so the tests can show
 * that their pins catch it; the default build defines none. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)

/* dtype codes of the raw buffers handed to the oracle */
#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_F16 2

/* ------------------------------------------------------------------ hash */

/*
 * _shift_right_after_eos(input_ids, shift), one position: read the token
 * `shift` places before t without crossing an EOS boundary. An EOS ends the
 * segment it closes, so reading across position p (p in t-shift .. t-1) is
 * forbidden when ids[p] is EOS. Positions before the sequence start also lack
 * valid context. Either way the result is `fill`.
 */
static int64_t shift_right_after_eos(const int32_t *ids, int64_t seq_begin,
                                     int64_t t, int shift, int32_t eos,
                                     int64_t fill)
{
    if (ORACLE_MUTANT == 5)
        seq_begin = 0; /* mutant: no reset at sequence starts */
    if (t - shift < seq_begin)
        return fill;
    for (int64_t p = t - shift; p < t + (ORACLE_MUTANT == 2); ++p)
        if (ids[p] == eos)
            return fill;
    return (int64_t)ids[t - shift];
}

/* Signed int64 product with two's-complement wrap ("signed int64 overflow"). */
static int64_t wrap_mul(int64_t a, int64_t b)
{
    return (int64_t)((uint64_t)a * (uint64_t)b);
}

/* Remainder in [0, m) for m > 0 ("positive remainders"). */
static int64_t positive_mod(int64_t a, int64_t m)
{
    int64_t r = a % m;
    if (r < 0 && ORACLE_MUTANT != 4)
        r += m;
    return r;
}

/*
 * _hash_input_ids: global table row of every head for every token.
 *   ids        [T] raw token IDs, cu [nseq+1] sequence bounds (NULL: one sequence)
 *   mult       [ngram_size]
 *   vocab, off [(ngram_size-1) * heads_per_ngram]
 *   out        [T, (ngram_size-1) * heads_per_ngram] int64
 * Heads 0..K-1 hash bigrams, K..2K-1 trigrams, and so on.
 */
int oracle_hash(int32_t ngram_size, int32_t heads_per_ngram,
                const int64_t *mult, const int64_t *vocab, const int64_t *off,
                int64_t fill, int32_t eos,
                const int32_t *ids, const int32_t *cu, int32_t nseq, int64_t T,
                int64_t *out)
{
    if (ngram_size < 2 || heads_per_ngram < 1 || T < 0)
        return ORACLE_EINVAL;
    const int H = (ngram_size - 1) * heads_per_ngram;
    for (int h = 0; h < H; ++h)
        if (vocab[h] <= 0)
            return ORACLE_EINVAL;

    /* shifted[k][t] = _shift_right_after_eos(ids, k)[t] for k = 1..ngram_size-1 */
    int64_t *shifted = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T > 0 ? T : 1) *
                                         (size_t)ngram_size);
    if (!shifted)
        return ORACLE_EINVAL;
    int32_t ns = cu ? nseq : 1;
    for (int32_t s = 0; s < ns; ++s) {
        int64_t b = cu ? cu[s] : 0, e = cu ? cu[s + 1] : T;
        if (b < 0 || e < b || e > T) {
            free(shifted);
            return ORACLE_EINVAL;
        }
        for (int64_t t = b; t < e; ++t) {
            shifted[t * ngram_size + 0] = ids[t];
            for (int k = 1; k < ngram_size; ++k)
                shifted[t * ngram_size + k] =
                    shift_right_after_eos(ids, b, t, k, eos, fill);
        }
    }

    for (int64_t t = 0; t < T; ++t) {
        const int64_t *x = &shifted[t * ngram_size];
        for (int n = 2; n <= ngram_size; ++n) {
            /* order-n mix: XOR of x_k * m_k over the n most recent tokens */
            int64_t mix = 0;
            for (int k = 0; k < n; ++k) {
                if (ORACLE_MUTANT == 1)
                    mix += wrap_mul(x[k], mult[k]);
                else if (ORACLE_MUTANT == 3)
                    mix ^= wrap_mul(x[k], mult[n - 1 - k]);
                else
                    mix ^= wrap_mul(x[k], mult[k]);
            }
            for (int i = 0; i < heads_per_ngram; ++i) {
                int h = (n - 2) * heads_per_ngram + i;
                out[t * H + h] = off[h] + positive_mod(mix, vocab[h]);
            }
        }
    }
    free(shifted);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- gather */

/*
 * _lookup_ngram_ids / OwnerShardedEmbedding.forward on a single-rank table:
 * out[i, :] = table[idx[i], :], copied bit for bit. Rows are `row_bytes` wide.
 */
int oracle_gather(const void *table, int64_t rows, int64_t row_bytes,
                  const int64_t *idx, int64_t n, void *out)
{
    const char *src = (const char *)table;
    char *dst = (char *)out;
    for (int64_t i = 0; i < n; ++i) {
        if (idx[i] < 0 || idx[i] >= rows)
            return ORACLE_EINVAL;
        memcpy(dst + i * row_bytes, src + idx[i] * row_bytes, (size_t)row_bytes);
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------- backward */

static double load_value(const void *buf, int dtype, int64_t i)
{
    if (dtype == ORACLE_F32) {
        return (double)((const float *)buf)[i];
    } else if (dtype == ORACLE_BF16) {
        /* bfloat16: the upper 16 bits of an IEEE binary32 */
        uint32_t bits = (uint32_t)((const uint16_t *)buf)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    } else {
        /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits */
        uint16_t h = ((const uint16_t *)buf)[i];
        int sign = h >> 15, ex = (h >> 10) & 0x1f, fr = h & 0x3ff;
        double v;
        if (ex == 0)
            v = (double)fr * (1.0 / 16777216.0); /* fr * 2^-24 */
        else if (ex == 31)
            v = fr ? (0.0 / 0.0) : (1.0 / 0.0);
        else {
            v = 1.0 + fr / 1024.0;
            int e = ex - 15;
            while (e > 0) { v *= 2.0; --e; }
            while (e < 0) { v *= 0.5; ++e; }
        }
        return sign ? -v : v;
    }
}

typedef struct { int64_t row; int64_t j; } lookup_t;

static int cmp_lookup(const void *a, const void *b)
{
    const lookup_t *x = (const lookup_t *)a, *y = (const lookup_t *)b;
    if (x->row != y->row)
        return x->row < y->row ? -1 : 1;
    return x->j < y->j ? -1 : (x->j > y->j);
}

/*
 * Row-gradient accumulation of the lookup (the owner side of the page's
 * backward): for every distinct row r among idx[0..n), in ascending order,
 *   grads[u, :] = fp32( sum over j with idx[j] == r, ascending j, of dout[j, :] )
 * with the sum taken in fp64. uniq[u] = r; *num_unique = number of rows.
 */
int oracle_backward(const int64_t *idx, int64_t n, const void *dout, int dtype,
                    int32_t dim, int64_t *uniq, float *grads, int64_t *num_unique)
{
    if (n < 0 || dim <= 0)
        return ORACLE_EINVAL;
    lookup_t *l = (lookup_t *)malloc(sizeof(lookup_t) * (size_t)(n > 0 ? n : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)dim);
    if (!l || !acc) {
        free(l);
        free(acc);
        return ORACLE_EINVAL;
    }
    for (int64_t j = 0; j < n; ++j) {
        l[j].row = idx[j];
        l[j].j = j;
    }
    qsort(l, (size_t)n, sizeof(lookup_t), cmp_lookup);

    int64_t u = 0;
    for (int64_t a = 0; a < n;) {
        int64_t b = a;
        for (int d = 0; d < dim; ++d)
            acc[d] = 0.0;
        while (b < n && (l[b].row == l[a].row ||
                         (ORACLE_MUTANT == 7 && l[b].row == l[a].row + 1))) {
            for (int d = 0; d < dim; ++d)
                acc[d] = ORACLE_MUTANT == 6
                    ? (double)((float)acc[d] + (float)load_value(dout, dtype, l[b].j * dim + d))
                    : acc[d] + load_value(dout, dtype, l[b].j * dim + d);
            ++b;
        }
        uniq[u] = l[a].row;
        for (int d = 0; d < dim; ++d)
            grads[u * dim + d] = (float)acc[d];
        ++u;
        a = b;
    }
    *num_unique = u;
    free(l);
    free(acc);
    return ORACLE_OK;
}

/* -------------------------------------------------- PLE short convolution */

/*
 * Branch-local Gemma RMS norm (layers page, Qwen3_8_FlashNextGroupedRMSNorm):
 * each row of C features is cut into C / G groups of G consecutive features
 * (one HyperConnection branch each) and every group is normalised on its own,
 *   n[c] = x[c] / sqrt(mean over the group of x^2 + eps) * (1 + w[c]),
 * where w is the additive scale that starts at zero (weight NULL = zeros).
 * All in fp64; out is fp64 [rows, C].
 */
int oracle_grouped_rms_norm(const void *x, int dtype, int64_t rows, int32_t C, int32_t G,
                            const void *weight, int wdtype, double eps, double *out)
{
    if (rows < 0 || C <= 0 || G <= 0 || C % G != 0 || eps < 0.0)
        return ORACLE_EINVAL;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t g0 = 0; g0 < C; g0 += G) {
            double ss = 0.0;
            for (int32_t c = g0; c < g0 + G; ++c) {
                const double v = load_value(x, dtype, r * C + c);
                ss += v * v;
            }
            double ms = ss / (double)G;
            if (ORACLE_MUTANT == 9)
                ms = ss / (double)C; /* mutant: mean over the whole row's width */
            const double inv = ORACLE_MUTANT == 10 ? 1.0 / (sqrt(ms) + eps)
                                                   : 1.0 / sqrt(ms + eps);
            for (int32_t c = g0; c < g0 + G; ++c) {
                const double w = weight ? load_value(weight, wdtype, c) : 0.0;
                const double scale = ORACLE_MUTANT == 8 ? w : 1.0 + w;
                out[r * C + c] = load_value(x, dtype, r * C + c) * inv * scale;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * The PLE layer's contextualising tail (engram page,
 * Qwen3_8_FlashNextPLELayer: norm_conv, conv1d, _causal_short_conv), taken
 * step by step over a [T, C] tensor of branch-flattened values:
 *   1. n = grouped RMS norm of x with norm_w (when do_norm; else n = x);
 *   2. causal depthwise convolution of width K and dilation dil with zero
 *      history before each sequence start: for token t of sequence s,
 *        y[t, c] = bias[c] + sum over k = 0 .. K-1 with t - k*dil >= cu[s] of
 *                  conv_w[c, K-1-k] * n[t - k*dil, c]
 *      (conv_w is [C, K] row-major, the [C, 1, K] weight of a depthwise
 *      conv1d whose last tap meets the current token; bias NULL = zeros);
 *   3. y = y * sigmoid(y) when do_silu;
 *   4. y = y + x when do_residual.
 * cu NULL means one sequence [0, T). out is fp64 [T, C].
 */
int oracle_short_conv(const void *x, int dtype, const int32_t *cu, int32_t nseq, int64_t T,
                      int32_t C, int32_t G, const void *norm_w, double eps,
                      const void *conv_w, const void *bias, int wdtype, int32_t K,
                      int32_t dil, int do_norm, int do_silu, int do_residual, double *out)
{
    if (T < 0 || C <= 0 || K < 1 || dil < 1 || (do_norm && (G <= 0 || C % G != 0)))
        return ORACLE_EINVAL;
    if (cu && (nseq < 0 || cu[0] != 0 || cu[nseq] != T))
        return ORACLE_EINVAL;
    double *n = (double *)malloc(sizeof(double) * (size_t)(T * C > 0 ? T * C : 1));
    if (!n)
        return ORACLE_EINVAL;
    if (do_norm) {
        const int rc = oracle_grouped_rms_norm(x, dtype, T, C, G, norm_w, wdtype, eps, n);
        if (rc != ORACLE_OK) {
            free(n);
            return rc;
        }
    } else {
        for (int64_t i = 0; i < T * C; ++i)
            n[i] = load_value(x, dtype, i);
    }
    const int32_t ns = cu ? nseq : 1;
    for (int32_t s = 0; s < ns; ++s) {
        int64_t begin = cu ? cu[s] : 0, end = cu ? cu[s + 1] : T;
        if (begin > end)
            continue;
        if (ORACLE_MUTANT == 13)
            begin = 0; /* mutant: history runs across sequence starts */
        for (int64_t t = cu ? cu[s] : 0; t < end; ++t) {
            for (int32_t c = 0; c < C; ++c) {
                double y = bias ? load_value(bias, wdtype, c) : 0.0;
                for (int32_t k = 0; k < K; ++k) {
                    const int64_t step = ORACLE_MUTANT == 11 ? (int64_t)k * (dil + 1)
                                                             : (int64_t)k * dil;
                    const int64_t src = t - step;
                    if (src < begin)
                        break;
                    const int32_t tap = ORACLE_MUTANT == 12 ? k : K - 1 - k;
                    y += load_value(conv_w, wdtype, (int64_t)c * K + tap) * n[src * C + c];
                }
                if (do_silu)
                    y = y / (1.0 + exp(-y));
                if (do_residual)
                    y += ORACLE_MUTANT == 14 ? n[t * C + c] : load_value(x, dtype, t * C + c);
                out[t * C + c] = y;
            }
        }
    }
    free(n);
    return ORACLE_OK;
}

/* ----------------------------------------------- sparse optimizer step */

/*
 * One AdamW step applied only to the rows a backward produced (the owner
 * "stores and updates each row's gradient", model card; the table's
 * optimizer tensors live in the checkpoint, model card §Current Scope). The
 * pages name no formula; this is AdamW updated lazily, with the step counter
 * global to the table. For u < U, r = rows[u], g = grads[u, :] and every
 * column c:
 *   p[r,c] *= 1 - lr * wd                          (decoupled weight decay)
 *   m[r,c]  = b1 * m[r,c] + (1 - b1) * g[c]
 *   v[r,c]  = b2 * v[r,c] + (1 - b2) * g[c]^2
 *   p[r,c] -= lr / (1 - b1^step) * m[r,c] / (sqrt(v[r,c] / (1 - b2^step)) + eps)
 * Rows not listed keep p, m and v. p, m, v are fp64 [rows, dim] in and out;
 * rows listed twice are updated twice, in order.
 */
int oracle_sparse_adam(double *p, double *m, double *v, int64_t rows, int32_t dim,
                       const int64_t *uniq, const float *grads, int64_t U, double lr,
                       double b1, double b2, double eps, double wd, int64_t step)
{
    if (rows < 0 || dim <= 0 || U < 0 || step < 1)
        return ORACLE_EINVAL;
    double bc1 = 1.0, bc2 = 1.0;
    for (int64_t s = 0; s < step; ++s) {
        bc1 *= b1;
        bc2 *= b2;
    }
    bc1 = 1.0 - bc1;
    bc2 = 1.0 - bc2;
    if (ORACLE_MUTANT == 15)
        bc1 = bc2 = 1.0; /* mutant: no bias correction */
    for (int64_t u = 0; u < U; ++u) {
        const int64_t r = uniq[u];
        if (r < 0 || r >= rows)
            return ORACLE_EINVAL;
        for (int32_t c = 0; c < dim; ++c) {
            const int64_t i = r * dim + c;
            double g = (double)grads[u * dim + c];
            if (ORACLE_MUTANT == 17)
                g += wd * p[i]; /* mutant: L2 penalty in the gradient, not decoupled */
            else
                p[i] *= 1.0 - lr * wd;
            m[i] = b1 * m[i] + (1.0 - b1) * g;
            v[i] = b2 * v[i] + (1.0 - b2) * g * g;
            const double denom = ORACLE_MUTANT == 16 ? sqrt(v[i] / bc2 + eps)
                                                     : sqrt(v[i] / bc2) + eps;
            p[i] -= lr / bc1 * m[i] / denom;
        }
    }
    return ORACLE_OK;
}

/*
 * Gradients of oracle_short_conv's output, given dout = dL/dout [T, C] (fp64),
 * by the chain rule through the same steps in reverse:
 *   dy[t,c]  = dout[t,c] * (do_silu ? s(y) (1 + y (1 - s(y))) : 1),  s = sigmoid
 *   dbias[c] = sum_t dy[t,c]
 *   for every tap k of row t that reads row src = t - k*dil (same sequence):
 *     dconv_w[c, K-1-k] += dy[t,c] * n[src,c]
 *     dn[src,c]         += conv_w[c, K-1-k] * dy[t,c]
 *   norm on (n = xh * (1 + norm_w), xh = x * inv over each group of G):
 *     dnorm_w[c] = sum_t dn[t,c] * xh[t,c]
 *     dxh = dn * (1 + norm_w);  dx = inv * (dxh - xh * mean over the group(dxh * xh))
 *   norm off: dx = dn;  residual: dx += dout.
 * Outputs are fp64: dx [T, C], dnorm_w [C], dconv_w [C, K], dbias [C].
 */
int oracle_short_conv_backward(const void *x, int dtype, const int32_t *cu, int32_t nseq,
                               int64_t T, int32_t C, int32_t G, const void *norm_w, double eps,
                               const void *conv_w, const void *bias, int wdtype, int32_t K,
                               int32_t dil, int do_norm, int do_silu, int do_residual,
                               const double *dout, double *dx, double *dnorm_w, double *dconv_w,
                               double *dbias)
{
    if (T < 0 || C <= 0 || K < 1 || dil < 1 || (do_norm && (G <= 0 || C % G != 0)))
        return ORACLE_EINVAL;
    if (cu && (nseq < 0 || cu[0] != 0 || cu[nseq] != T))
        return ORACLE_EINVAL;
    const size_t TC = (size_t)(T * C > 0 ? T * C : 1);
    double *n = (double *)calloc(TC, sizeof(double));
    double *xh = (double *)calloc(TC, sizeof(double));
    double *dy = (double *)calloc(TC, sizeof(double));
    double *dn = (double *)calloc(TC, sizeof(double));
    double *inv = (double *)calloc((size_t)(T > 0 ? T : 1) * (size_t)(do_norm ? C / G : 1),
                                   sizeof(double));
    if (!n || !xh || !dy || !dn || !inv) {
        free(n); free(xh); free(dy); free(dn); free(inv);
        return ORACLE_EINVAL;
    }
    /* forward again: xh, n */
    for (int64_t t = 0; t < T; ++t) {
        if (do_norm) {
            for (int32_t g0 = 0; g0 < C; g0 += G) {
                double ss = 0.0;
                for (int32_t c = g0; c < g0 + G; ++c) {
                    const double v = load_value(x, dtype, t * C + c);
                    ss += v * v;
                }
                const double iv = 1.0 / sqrt(ss / (double)G + eps);
                inv[t * (C / G) + g0 / G] = iv;
                for (int32_t c = g0; c < g0 + G; ++c) {
                    xh[t * C + c] = load_value(x, dtype, t * C + c) * iv;
                    n[t * C + c] = xh[t * C + c] *
                                   (1.0 + (norm_w ? load_value(norm_w, wdtype, c) : 0.0));
                }
            }
        } else {
            for (int32_t c = 0; c < C; ++c)
                n[t * C + c] = xh[t * C + c] = load_value(x, dtype, t * C + c);
        }
    }
    for (int32_t c = 0; c < C; ++c) {
        dbias[c] = 0.0;
        dnorm_w[c] = 0.0;
        for (int32_t k = 0; k < K; ++k)
            dconv_w[c * K + k] = 0.0;
    }
    /* y, dy, and the convolution's gradients */
    const int32_t ns = cu ? nseq : 1;
    for (int32_t s = 0; s < ns; ++s) {
        const int64_t begin = cu ? cu[s] : 0, end = cu ? cu[s + 1] : T;
        for (int64_t t = begin; t < end; ++t) {
            for (int32_t c = 0; c < C; ++c) {
                double y = bias ? load_value(bias, wdtype, c) : 0.0;
                for (int32_t k = 0; k < K && t - (int64_t)k * dil >= begin; ++k)
                    y += load_value(conv_w, wdtype, (int64_t)c * K + K - 1 - k) *
                         n[(t - (int64_t)k * dil) * C + c];
                double g = dout[t * C + c];
                if (do_silu) {
                    const double sg = 1.0 / (1.0 + exp(-y));
                    g *= ORACLE_MUTANT == 18 ? sg : sg * (1.0 + y * (1.0 - sg));
                }
                dy[t * C + c] = g;
                dbias[c] += g;
                for (int32_t k = 0; k < K && t - (int64_t)k * dil >= begin; ++k) {
                    const int64_t src = t - (int64_t)k * dil;
                    const double w = load_value(conv_w, wdtype, (int64_t)c * K + K - 1 - k);
                    dconv_w[(int64_t)c * K + K - 1 - k] += g * n[src * C + c];
                    if (ORACLE_MUTANT == 19) {
                        /* mutant: the taps' gradient sent forward instead of back */
                        if (t + (int64_t)k * dil < end)
                            dn[(t + (int64_t)k * dil) * C + c] += w * g;
                    } else {
                        dn[src * C + c] += w * g;
                    }
                }
            }
        }
    }
    /* the norm's gradients, then the residual */
    for (int64_t t = 0; t < T; ++t) {
        if (do_norm) {
            for (int32_t g0 = 0; g0 < C; g0 += G) {
                double dot = 0.0;
                for (int32_t c = g0; c < g0 + G; ++c) {
                    const double sc = 1.0 + (norm_w ? load_value(norm_w, wdtype, c) : 0.0);
                    dnorm_w[c] += dn[t * C + c] * xh[t * C + c];
                    dot += dn[t * C + c] * sc * xh[t * C + c];
                }
                const double mean = ORACLE_MUTANT == 20 ? 0.0 : dot / (double)G;
                const double iv = inv[t * (C / G) + g0 / G];
                for (int32_t c = g0; c < g0 + G; ++c) {
                    const double sc = 1.0 + (norm_w ? load_value(norm_w, wdtype, c) : 0.0);
                    dx[t * C + c] = iv * (dn[t * C + c] * sc - xh[t * C + c] * mean);
                }
            }
        } else {
            for (int32_t c = 0; c < C; ++c)
                dx[t * C + c] = dn[t * C + c];
        }
        if (do_residual)
            for (int32_t c = 0; c < C; ++c)
                dx[t * C + c] += dout[t * C + c];
    }
    free(n); free(xh); free(dy); free(dn); free(inv);
    return ORACLE_OK;
}
