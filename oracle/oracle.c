/*
 * oracle.c -- plain float64 CPU restatement of Attn-QAT training attention with
 * NVFP4 fake quantization (fq).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links, loads
 * or calls this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or constant with
 * the CUDA kernels; the two sides meet only at the seeded synthetic inputs.
 *
 * Sources (the web pages this method is described on):
 *  - vsqa-test-1.3b checkpoint metadata.json, "attention.precision": the fine
 *    attention is "NVFP4 fake-quant with BF16 matmul", quant_p = quant_v = true,
 *    use_global_sf_p = use_global_sf_qkv = false (no global scale),
 *    two_level_p = false.
 *  - the same metadata.json, "linear_quantization.format": NVFP4 is E2M1
 *    values in 16-element blocks with an FP8 E4M3 scale per block.
 *  - FastVideo "Attn-QAT Training" guide, "Architecture-specific Triton
 *    routing": non-causal, Lq may differ from Lk, K and V share Lk; the fast
 *    backward needs a 16-aligned KV length; the softmax statistics are
 *    recomputed in reference order so that dV stays consistent.
 *  The fq convention this library implements: values on the E2M1 grid
 *  {0, 0.5, 1, 1.5, 2, 3, 4, 6} (with sign), 16-element blocks along the
 *  contraction axis of the matmul the operand feeds, block scale =
 *  E4M3(amax / 6), round-to-nearest-even for both roundings, no global scale.
 *  Forward: S = fq(Q) fq(K)^T * c, m = row max, P~ = exp(S - m), l = sum P~,
 *  O = fq(P~) fq(V) / l, LSE = m + ln l.  Backward (straight-through):
 *  dV = (fq(P~)/l)^T dO, dP = dO fq(V)^T, dS = P o (dP - Delta),
 *  Delta = rowsum(dO o O), dQ = dS fq(K) c, dK = dS^T fq(Q) c, P = P~/l.
 *
 * Readings taken where the pages are silent:
 *  - m is the exact row max over all keys (not a running max);
 *  - l sums the unquantized P~;
 *  - dV uses the forward's fq(P~) divided by l (blocks along keys); the literal
 *    fq(P~/l) is available behind ORACLE_DV_QUANT_NORMALIZED;
 *  - both roundings are exact rational round-to-nearest, ties to the even
 *    code; a/6 above 448 saturates to 448; a scale of 0 zeroes the block;
 *  - a code nibble carries the input's sign bit (so -0.1 -> 0x8), even
 *    element in the low nibble; scale bytes have sign bit 0;
 *  - V is blocked along tokens from token 0; a ragged final block is padded
 *    with zeros (which does not change its amax);
 *  - c multiplies the fp64 dot product, never the operands before fq.
 *
 * Block-sparse fine attention (vsqa-test-1.3b metadata.json, "attention":
 * backend VSA_QAT_TRAIN_C128, kind "vsa", cube_shape 4 x 4 x 8 = 128 tokens,
 * "fine": "NVFP4 fake-quant with BF16 matmul", quantize_fine = true, top-k
 * "selection" of key blocks per query block): every function that takes
 * `sel` restricts query i to the keys j whose tiles are selected,
 * sel[(i / T) * nkt + j / T] != 0 with T-token tiles and nkt = ceil(Lk / T);
 * sel = NULL is dense attention.  Reading: the fine attention is the same
 * Attn-QAT computation over the selected keys only -- m is their exact max,
 * l their sum, and a key outside the selection has P~ = 0 (so it adds zero
 * to its fq(P~) block, which is all zeros when T is a multiple of 16); fq(Q),
 * fq(K), fq(V) do not depend on the selection.  A query row with no selected
 * key has O = 0, l = 0, m = LSE = -infinity, dQ = 0, and adds nothing to
 * dK, dV.
 *
 * Causal masking (flag ORACLE_CAUSAL, Lq == Lk): query i attends to keys
 * j <= i only.  The pages' training route is non-causal; this is the general
 * route's masking read the same way as the block selection: masked keys have
 * P~ = 0 inside their fq(P~) block, and m, l run over the unmasked keys.
 *
 * Every arithmetic step is plain float64; the only reorderings are the ones a
 * sum admits.  Loops are parallelised over independent rows with OpenMP.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_QUANT_Q 1u
#define ORACLE_QUANT_K 2u
#define ORACLE_QUANT_V 4u
#define ORACLE_QUANT_P 8u
#define ORACLE_DV_QUANT_NORMALIZED 16u
#define ORACLE_CAUSAL 32u

#define BLOCK 16

/* Does query i attend to key j?  sel == NULL: every tile; ORACLE_CAUSAL:
 * only keys j <= i (Lq == Lk, query i and key i are the same token).       */
static int selected(unsigned flags, const uint8_t *sel, long T, long nkt, long i,
                    long j)
{
    if ((flags & ORACLE_CAUSAL) && j > i)
        return 0;
    return sel == NULL || sel[(i / T) * nkt + j / T] != 0;
}

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("fn": bias 7, 3 mantissa bits, no infinities, S.1111.111 is
 * NaN).  Value of a non-negative code 0..126:
 *   exponent field 0     -> subnormal  mantissa * 2^-9
 *   exponent field e > 0 -> normal     (1 + mantissa/8) * 2^(e-7)          */
double oracle_e4m3_value(int code)
{
    int e = (code >> 3) & 15;
    int mant = code & 7;
    if (e == 0)
        return ldexp((double)mant, -9);
    return ldexp((double)(8 + mant), e - 10);
}

/* FP4 E2M1 magnitudes, indexed by the 3-bit magnitude code. */
static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int code)
{
    double v = E2M1_GRID[code & 7];
    return (code & 8) ? -v : v;
}

/* Round the exact quotient a/6 (a >= 0) to the nearest finite non-negative
 * E4M3 value; ties go to the even code; anything above 448 gives 448.
 * Exactness: with v_k <= a/6 < v_{k+1}, the comparison of a/6 against the
 * midpoint (v_k + v_{k+1})/2 is done as 2a versus 6(v_k + v_{k+1}); both
 * sides are exact in float64 (a has at most 53 bits, the right side at most
 * 8).                                                                       */
int oracle_e4m3_round_div6(double a)
{
    if (!(a > 0.0))
        return 0;
    if (a >= 6.0 * 448.0)
        return 126;
    int k = 0; /* largest code with 6 v_k <= a */
    while (k < 126 && 6.0 * oracle_e4m3_value(k + 1) <= a)
        k++;
    if (k == 126)
        return 126;
    double twice = 2.0 * a;
    double mid2 = 6.0 * (oracle_e4m3_value(k) + oracle_e4m3_value(k + 1));
    if (twice < mid2)
        return k;
    if (twice > mid2)
        return k + 1;
    return (k % 2 == 0) ? k : k + 1;
}

/* Round |x|/s (s > 0) to the nearest E2M1 magnitude code; ties to the even
 * code; above 6 saturates to 6 (code 7).  Same exact midpoint test as above:
 * 2|x| against s (g_k + g_{k+1}).                                           */
int oracle_e2m1_round(double ax, double s)
{
    int k = 0; /* largest code with g_k s <= ax */
    while (k < 7 && E2M1_GRID[k + 1] * s <= ax)
        k++;
    if (k == 7)
        return 7;
    double twice = 2.0 * ax;
    double mid2 = s * (E2M1_GRID[k] + E2M1_GRID[k + 1]);
    if (twice < mid2)
        return k;
    if (twice > mid2)
        return k + 1;
    return (k % 2 == 0) ? k : k + 1;
}

/* Element-wise oracle_e2m1_round over arrays (for exhaustive tests). */
void oracle_e2m1_round_many(const double *ax, const double *s, long n,
                            int32_t *out)
{
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; i++)
        out[i] = oracle_e2m1_round(ax[i], s[i]);
}

/* fq of one block of n <= 16 values x[i*xs].  Missing elements of a ragged
 * block count as zeros.  Writes the dequantized values y[i*ys] (may alias x),
 * optionally the 4-bit codes (one per byte, sign in bit 3) and the scale
 * code.                                                                     */
static void fq_block(const double *x, long n, long xs, double *y, long ys,
                     uint8_t *codes, uint8_t *scale_code)
{
    double a = 0.0;
    for (long i = 0; i < n; i++) {
        double ax = fabs(x[i * xs]);
        if (ax > a)
            a = ax;
    }
    int sc = oracle_e4m3_round_div6(a);
    double s = oracle_e4m3_value(sc);
    if (scale_code)
        *scale_code = (uint8_t)sc;
    for (long i = 0; i < n; i++) {
        double xi = x[i * xs];
        int neg = signbit(xi) ? 1 : 0;
        int c = (s > 0.0) ? oracle_e2m1_round(fabs(xi), s) : 0;
        double mag = E2M1_GRID[c] * s;
        if (codes)
            codes[i] = (uint8_t)((neg << 3) | c);
        y[i * ys] = neg ? -mag : mag;
    }
}

/* ------------------------------------------------------------------------ */
/* Standalone quantizer                                                      */
/* ------------------------------------------------------------------------ */

/* Quantize each of the `rows` logical rows of a bf16 view (element (r, j) at
 * x[r*srow + j*scol]) in blocks of 16 consecutive j.  cols must be a multiple
 * of 16.  Outputs (any may be NULL):
 *   codes  [rows][cols/2]  element 2i in the low nibble, 2i+1 in the high one
 *   scales [rows][cols/16] E4M3 scale codes
 *   deq    [rows][cols]    dequantized values, float64                      */
void oracle_quantize_rows(const uint16_t *x, long rows, long cols, long srow,
                          long scol, uint8_t *codes, uint8_t *scales,
                          double *deq)
{
    long nblk = cols / BLOCK;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        double xb[BLOCK], yb[BLOCK];
        uint8_t cb[BLOCK];
        for (long b = 0; b < nblk; b++) {
            for (long i = 0; i < BLOCK; i++)
                xb[i] = oracle_bf16_value(x[r * srow + (b * BLOCK + i) * scol]);
            uint8_t sc;
            fq_block(xb, BLOCK, 1, yb, 1, cb, &sc);
            if (scales)
                scales[r * nblk + b] = sc;
            if (codes)
                for (long i = 0; i < BLOCK; i += 2)
                    codes[r * (cols / 2) + (b * BLOCK + i) / 2] =
                        (uint8_t)(cb[i] | (cb[i + 1] << 4));
            if (deq)
                for (long i = 0; i < BLOCK; i++)
                    deq[r * cols + b * BLOCK + i] = yb[i];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 with an FP32 global scale                                           */
/* ------------------------------------------------------------------------ */

/* The linear-layer variant of the format (vsqa-test-1.3b metadata.json,
 * "linear_quantization": "NVFP4 W4A4: E2M1 values, 16-element blocks, FP8
 * E4M3 block scales, FP32 global scale", with the activation global scale
 * "dynamic, 448*6/max|X| recomputed every forward").  The page does not fix
 * the order of the steps; they are read as exact two-level rounding:
 *   G   = the float32 quotient 2688 / max|x| (1 when max|x| = 0; the largest
 *         finite float32 if the quotient overflows);
 *   k_b = E4M3 round-to-nearest-even (saturating) of the exact a_b * G / 6,
 *         a_b the block's max |x|;  s_b = value of k_b;
 *   c   = E2M1 round-to-nearest-even (saturating) of the exact |x| G / s_b
 *         (0 when s_b = 0);
 *   deq = sign * E2M1(c) * s_b / G, rounded once to bfloat16 (nearest, ties
 *         to even).
 * a_b * G and |x| * G are exact in float64 (8- and 24-bit significands), so
 * the roundings above reuse the exact midpoint tests of the plain format.  */

/* The float32 global scale for a tensor whose largest magnitude is amax. */
float oracle_global_scale(double amax)
{
    if (!(amax > 0.0))
        return 1.0f;
    volatile float num = 2688.0f;
    volatile float den = (float)amax; /* amax is a bf16 value: exact */
    float g = num / den;              /* IEEE float32 division */
    if (isinf(g))
        g = 3.40282347e38f;
    return g;
}

/* Value of a non-negative bfloat16 bit pattern. */
static double bf16_bits_value(uint32_t h)
{
    return oracle_bf16_value((uint16_t)h);
}

/* bfloat16 bits of the exact quotient n / g (n >= 0, g > 0, exact doubles;
 * every product below has at most 33 significant bits, so it is exact),
 * rounded to nearest, ties to even.  Start from the truncated float64
 * quotient and step along the (monotonic) bit patterns of positive bfloat16
 * values until lo <= n/g < next(lo), then compare with the midpoint.        */
static uint16_t bf16_of_quotient(double n, double g)
{
    if (n == 0.0)
        return 0;
    float qf = (float)(n / g);
    uint32_t u;
    memcpy(&u, &qf, sizeof u);
    uint32_t h = u >> 16;                          /* truncation: value <= qf */
    while (h > 0 && bf16_bits_value(h) * g > n)
        h--;
    while (bf16_bits_value(h + 1) * g <= n)
        h++;
    double mid = 0.5 * (bf16_bits_value(h) + bf16_bits_value(h + 1));
    if (n < mid * g)
        return (uint16_t)h;
    if (n > mid * g)
        return (uint16_t)(h + 1);
    return (uint16_t)((h % 2 == 0) ? h : h + 1);    /* tie: even bit pattern */
}

/* Global-scale fq of a strided bf16 view (same view as oracle_quantize_rows).
 * Outputs: codes [rows][cols/2] (element 2i in the low nibble, sign in bit 3
 * of each nibble), scales [rows][cols/16] (E4M3 codes of s_b), deq
 * [rows][cols] bfloat16 bits, and *gscale (any output may be NULL).         */
void oracle_quantize_rows_gs(const uint16_t *x, long rows, long cols, long srow,
                             long scol, uint8_t *codes, uint8_t *scales,
                             uint16_t *deq, float *gscale)
{
    long nblk = cols / BLOCK;
    double amax = 0.0;
    for (long r = 0; r < rows; r++)
        for (long j = 0; j < cols; j++) {
            double a = fabs(oracle_bf16_value(x[r * srow + j * scol]));
            if (a > amax)
                amax = a;
        }
    float gf = oracle_global_scale(amax);
    double g = (double)gf;
    if (gscale)
        *gscale = gf;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        for (long b = 0; b < nblk; b++) {
            double xb[BLOCK];
            double ab = 0.0;
            for (long i = 0; i < BLOCK; i++) {
                xb[i] = oracle_bf16_value(x[r * srow + (b * BLOCK + i) * scol]);
                if (fabs(xb[i]) > ab)
                    ab = fabs(xb[i]);
            }
            int k = oracle_e4m3_round_div6(ab * g);   /* exact product */
            double sb = oracle_e4m3_value(k);
            if (scales)
                scales[r * nblk + b] = (uint8_t)k;
            uint8_t cb[BLOCK];
            for (long i = 0; i < BLOCK; i++) {
                int neg = signbit(xb[i]) ? 1 : 0;
                int c = (sb > 0.0) ? oracle_e2m1_round(fabs(xb[i]) * g, sb) : 0;
                cb[i] = (uint8_t)((neg << 3) | c);
                if (deq) {
                    uint16_t h = bf16_of_quotient(E2M1_GRID[c] * sb, g);
                    deq[r * cols + b * BLOCK + i] = (uint16_t)(h | (neg ? 0x8000u : 0u));
                }
            }
            if (codes)
                for (long i = 0; i < BLOCK; i += 2)
                    codes[r * (cols / 2) + (b * BLOCK + i) / 2] = (uint8_t)(cb[i] | (cb[i + 1] << 4));
        }
    }
}

/* fq of float64 values, blocks of 16 along a row (used for tests of the
 * block rounding on non-bf16 inputs, e.g. probabilities).                   */
void oracle_fq_f64_rows(const double *x, long rows, long cols, double *y,
                        uint8_t *scales)
{
    long nblk = (cols + BLOCK - 1) / BLOCK;
    for (long r = 0; r < rows; r++)
        for (long b = 0; b < nblk; b++) {
            long n = cols - b * BLOCK < BLOCK ? cols - b * BLOCK : BLOCK;
            uint8_t sc;
            fq_block(x + r * cols + b * BLOCK, n, 1, y + r * cols + b * BLOCK, 1,
                     NULL, &sc);
            if (scales)
                scales[r * nblk + b] = sc;
        }
}

/* ------------------------------------------------------------------------ */
/* Attention operands                                                        */
/* ------------------------------------------------------------------------ */

/* Operands of one head as float64.  q: [Lq][D], k, v: [Lk][D] bf16.
 * Qh, Kh: fq with blocks of 16 along D (the contraction axis of Q K^T);
 * Vh: fq with blocks of 16 consecutive tokens per channel (the contraction
 * axis of P V), from token 0, ragged last block zero-padded.  A cleared flag
 * leaves that operand as its bf16 value.                                    */
void oracle_operands(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     long Lq, long Lk, long D, unsigned flags, double *Qh,
                     double *Kh, double *Vh)
{
    for (long i = 0; i < Lq * D; i++)
        Qh[i] = oracle_bf16_value(q[i]);
    for (long i = 0; i < Lk * D; i++) {
        Kh[i] = oracle_bf16_value(k[i]);
        Vh[i] = oracle_bf16_value(v[i]);
    }
    if (flags & ORACLE_QUANT_Q)
        for (long r = 0; r < Lq; r++)
            for (long b = 0; b < D / BLOCK; b++)
                fq_block(Qh + r * D + b * BLOCK, BLOCK, 1, Qh + r * D + b * BLOCK,
                         1, NULL, NULL);
    if (flags & ORACLE_QUANT_K)
        for (long r = 0; r < Lk; r++)
            for (long b = 0; b < D / BLOCK; b++)
                fq_block(Kh + r * D + b * BLOCK, BLOCK, 1, Kh + r * D + b * BLOCK,
                         1, NULL, NULL);
    if (flags & ORACLE_QUANT_V)
        for (long d = 0; d < D; d++)
            for (long t0 = 0; t0 < Lk; t0 += BLOCK) {
                long n = Lk - t0 < BLOCK ? Lk - t0 : BLOCK;
                fq_block(Vh + t0 * D + d, n, D, Vh + t0 * D + d, D, NULL, NULL);
            }
}

/* float64 dot product; four partial sums only to keep the adds independent */
static double dot(const double *a, const double *b, long n)
{
    double s0 = 0, s1 = 0, s2 = 0, s3 = 0;
    long i = 0;
    for (; i + 4 <= n; i += 4) {
        s0 += a[i] * b[i];
        s1 += a[i + 1] * b[i + 1];
        s2 += a[i + 2] * b[i + 2];
        s3 += a[i + 3] * b[i + 3];
    }
    for (; i < n; i++)
        s0 += a[i] * b[i];
    return (s0 + s1) + (s2 + s3);
}

/* One score row: S_j = c * (Qh_i . Kh_j) for j in [0, Lk). */
static void score_row(const double *Qi, const double *Kh, long Lk, long D,
                      double c, double *S)
{
    for (long j = 0; j < Lk; j++)
        S[j] = c * dot(Qi, Kh + j * D, D);
}

/* Probability row of query i: P~_j = exp(S_j - m) over the selected keys
 * (0 elsewhere) and, with QUANT_P, the fq'd P^ in blocks of 16 consecutive
 * keys from key 0.  Returns m (-inf with no selected key) and l.           */
static void prob_row(const double *Qi, long i, const double *Kh, long Lk, long D,
                     double c, unsigned flags, const uint8_t *sel, long T,
                     double *S, double *Pt, double *Phat, double *m_out,
                     double *l_out)
{
    long nkt = (Lk + T - 1) / T;
    score_row(Qi, Kh, Lk, D, c, S);
    double m = -INFINITY;
    for (long j = 0; j < Lk; j++)
        if (selected(flags, sel, T, nkt, i, j) && S[j] > m)
            m = S[j];
    double l = 0.0;
    for (long j = 0; j < Lk; j++) {
        Pt[j] = selected(flags, sel, T, nkt, i, j) ? exp(S[j] - m) : 0.0;
        l += Pt[j];
    }
    if (flags & ORACLE_QUANT_P) {
        for (long t0 = 0; t0 < Lk; t0 += BLOCK) {
            long n = Lk - t0 < BLOCK ? Lk - t0 : BLOCK;
            fq_block(Pt + t0, n, 1, Phat + t0, 1, NULL, NULL);
        }
    } else {
        memcpy(Phat, Pt, sizeof(double) * Lk);
    }
    *m_out = m;
    *l_out = l;
}

/* ------------------------------------------------------------------------ */
/* Forward                                                                   */
/* ------------------------------------------------------------------------ */

/* Forward for the query rows listed in rows[0..nrows): O (float64, [nrows][D]),
 * LSE, m and l per listed row.  Qh/Kh/Vh come from oracle_operands; sel/T
 * select key tiles per query tile (NULL: dense).                           */
void oracle_fwd_rows(const double *Qh, const double *Kh, const double *Vh,
                     long Lq, long Lk, long D, double c, unsigned flags,
                     const uint8_t *sel, long T, const long *rows, long nrows,
                     double *O, double *lse, double *m, double *l)
{
    (void)Lq;
#pragma omp parallel
    {
        double *S = malloc(sizeof(double) * Lk);
        double *Pt = malloc(sizeof(double) * Lk);
        double *Ph = malloc(sizeof(double) * Lk);
#pragma omp for schedule(dynamic, 4)
        for (long t = 0; t < nrows; t++) {
            long i = rows[t];
            double mi, li;
            prob_row(Qh + i * D, i, Kh, Lk, D, c, flags, sel, T, S, Pt, Ph, &mi,
                     &li);
            /* O_d = sum_j P^_j V^_jd / l, each sum taken in key order j =
             * 0..Lk-1 (the loop over d runs inside, along V's rows)        */
            double *acc = O + t * D;
            for (long d = 0; d < D; d++)
                acc[d] = 0.0;
            for (long j = 0; j < Lk; j++)
                for (long d = 0; d < D; d++)
                    acc[d] += Ph[j] * Vh[j * D + d];
            for (long d = 0; d < D; d++)
                acc[d] = li > 0.0 ? acc[d] / li : 0.0;
            m[t] = mi;
            l[t] = li;
            lse[t] = li > 0.0 ? mi + log(li) : -INFINITY;
        }
        free(S);
        free(Pt);
        free(Ph);
    }
}

/* Delta_i = sum_d dO_id O_id for every row (O in float64, dO bf16). */
void oracle_delta(const double *O, const uint16_t *dO, long L, long D,
                  double *delta)
{
    for (long i = 0; i < L; i++) {
        double s = 0.0;
        for (long d = 0; d < D; d++)
            s += oracle_bf16_value(dO[i * D + d]) * O[i * D + d];
        delta[i] = s;
    }
}

/* ------------------------------------------------------------------------ */
/* Backward (straight-through: every fq is the identity for the gradient)    */
/* ------------------------------------------------------------------------ */

/* dQ for the listed query rows.  m, l, delta hold all Lq rows.  dQ float64
 * [nrows][D].                                                              */
void oracle_bwd_dq_rows(const double *Qh, const double *Kh, const double *Vh,
                        const uint16_t *dO, long Lq, long Lk, long D, double c,
                        unsigned flags, const uint8_t *sel, long T,
                        const double *m, const double *l,
                        const double *delta, const long *rows, long nrows,
                        double *dQ)
{
    long nkt = (Lk + T - 1) / T;
    (void)Lq;
#pragma omp parallel
    {
        double *S = malloc(sizeof(double) * Lk);
        double *Pt = malloc(sizeof(double) * Lk);
        double *Ph = malloc(sizeof(double) * Lk);
        double *dOi = malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 4)
        for (long t = 0; t < nrows; t++) {
            long i = rows[t];
            double mi, li;
            prob_row(Qh + i * D, i, Kh, Lk, D, c, flags, sel, T, S, Pt, Ph, &mi,
                     &li);
            (void)mi;
            (void)li;
            for (long d = 0; d < D; d++)
                dOi[d] = oracle_bf16_value(dO[i * D + d]);
            for (long d = 0; d < D; d++)
                dQ[t * D + d] = 0.0;
            for (long j = 0; j < Lk; j++) {
                if (!(l[i] > 0.0) || !selected(flags, sel, T, nkt, i, j))
                    continue;
                double P = exp(S[j] - m[i]) / l[i];
                double dP = dot(dOi, Vh + j * D, D);
                double dS = P * (dP - delta[i]);
                for (long d = 0; d < D; d++)
                    dQ[t * D + d] += dS * Kh[j * D + d];
            }
            for (long d = 0; d < D; d++)
                dQ[t * D + d] *= c;
        }
        free(S);
        free(Pt);
        free(Ph);
        free(dOi);
    }
}

/* dK and dV for the keys of the listed 16-key blocks (block b covers keys
 * [16b, 16b+16) clipped to Lk).  m, l, delta hold all Lq rows.  Output
 * float64 [nblocks*16][D]; rows past Lk are left zero.                      */
void oracle_bwd_dkdv_blocks(const double *Qh, const double *Kh, const double *Vh,
                            const uint16_t *dO, long Lq, long Lk, long D,
                            double c, unsigned flags, const uint8_t *sel,
                            long T, const double *m,
                            const double *l, const double *delta,
                            const long *blocks, long nblocks, double *dK,
                            double *dV)
{
    long nkt = (Lk + T - 1) / T;
    memset(dK, 0, sizeof(double) * nblocks * BLOCK * D);
    memset(dV, 0, sizeof(double) * nblocks * BLOCK * D);
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < nblocks; t++) {
        long j0 = blocks[t] * BLOCK;
        long n = Lk - j0 < BLOCK ? Lk - j0 : BLOCK;
        double S[BLOCK], Pt[BLOCK], Ph[BLOCK], dOi[512];
        double *dKt = dK + t * BLOCK * D, *dVt = dV + t * BLOCK * D;
        for (long i = 0; i < Lq; i++) {
            if (!(l[i] > 0.0))
                continue; /* no selected key: the row adds nothing */
            for (long d = 0; d < D; d++)
                dOi[d] = oracle_bf16_value(dO[i * D + d]);
            for (long jj = 0; jj < n; jj++) {
                S[jj] = c * dot(Qh + i * D, Kh + (j0 + jj) * D, D);
                Pt[jj] = selected(flags, sel, T, nkt, i, j0 + jj) ? exp(S[jj] - m[i]) : 0.0;
            }
            /* w_j: the dV weight of key j in this query row */
            double w[BLOCK];
            if (flags & ORACLE_DV_QUANT_NORMALIZED) {
                /* literal reading: fq applied to the normalised P~/l */
                double Pn[BLOCK];
                for (long jj = 0; jj < n; jj++)
                    Pn[jj] = Pt[jj] / l[i];
                fq_block(Pn, n, 1, w, 1, NULL, NULL);
            } else if (flags & ORACLE_QUANT_P) {
                fq_block(Pt, n, 1, Ph, 1, NULL, NULL);
                for (long jj = 0; jj < n; jj++)
                    w[jj] = Ph[jj] / l[i];
            } else {
                for (long jj = 0; jj < n; jj++)
                    w[jj] = Pt[jj] / l[i];
            }
            for (long jj = 0; jj < n; jj++) {
                double P = Pt[jj] / l[i];
                double dP = dot(dOi, Vh + (j0 + jj) * D, D);
                double dS = P * (dP - delta[i]);
                for (long d = 0; d < D; d++) {
                    dVt[jj * D + d] += w[jj] * dOi[d];
                    dKt[jj * D + d] += dS * Qh[i * D + d];
                }
            }
        }
        for (long x = 0; x < n * D; x++)
            dKt[x] *= c;
    }
}

/* ------------------------------------------------------------------------ */
/* Block selection of the sparse attention (coarse scores, top-k)             */
/* ------------------------------------------------------------------------ */

/* VSA key-tile selection for one head (vsqa-test-1.3b metadata.json,
 * "attention.selection": top-k key cubes per query cube with
 * effective_topk = max(1, min(ceil((1 - sparsity) * num_blocks), num_blocks);
 * "attention.precision.coarse": BF16, quantize_coarse false).  Reading (the
 * page gives the fields, not the arithmetic): each T-token
 * tile is summarised by the mean of its valid rows; the coarse score of
 * (query tile I, key tile J) is the dot product of the two means (the softmax
 * scale and the softmax itself do not change the order); query tile I keeps
 * the topk key tiles of highest score, ties to the lower J.  The order
 * decides an integer, so it is taken in the precision a B200 kernel computes
 * it in, float32, with every step fixed: sum of the rows in token order (one
 * float32 add per row), mean = sum / count (one correctly rounded float32
 * division), score = the channels in order d = 0..D-1 accumulated with one
 * fused multiply-add each from 0.  q: [Lq][D], k: [Lk][D] bf16.  Outputs
 * mask [nq][nk] (1 = kept) and, if not NULL, the scores [nq][nk].          */
static void tile_means_f32(const uint16_t *x, long L, long D, long T, float *mean)
{
    long nt = (L + T - 1) / T;
    for (long t = 0; t < nt; t++) {
        long r0 = t * T, r1 = r0 + T < L ? r0 + T : L;
        for (long d = 0; d < D; d++) {
            float s = 0.0f;
            for (long r = r0; r < r1; r++)
                s = s + (float)oracle_bf16_value(x[r * D + d]);
            mean[t * D + d] = s / (float)(r1 - r0);
        }
    }
}

void oracle_vsa_select(const uint16_t *q, const uint16_t *k, long Lq, long Lk,
                       long D, long T, long topk, uint8_t *mask, float *scores)
{
    long nq = (Lq + T - 1) / T, nk = (Lk + T - 1) / T;
    float *qm = malloc(sizeof(float) * nq * D);
    float *km = malloc(sizeof(float) * nk * D);
    float *sc = malloc(sizeof(float) * nk);
    tile_means_f32(q, Lq, D, T, qm);
    tile_means_f32(k, Lk, D, T, km);
    if (topk > nk)
        topk = nk;
    for (long i = 0; i < nq; i++) {
        for (long j = 0; j < nk; j++) {
            float acc = 0.0f;
            for (long d = 0; d < D; d++)
                acc = fmaf(qm[i * D + d], km[j * D + d], acc);
            sc[j] = acc;
            if (scores)
                scores[i * nk + j] = acc;
            mask[i * nk + j] = 0;
        }
        /* topk rounds of "the best tile not yet kept" */
        for (long r = 0; r < topk; r++) {
            long best = -1;
            for (long j = 0; j < nk; j++)
                if (!mask[i * nk + j] && (best < 0 || sc[j] > sc[best]))
                    best = j;
            mask[i * nk + best] = 1;
        }
    }
    free(qm);
    free(km);
    free(sc);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
