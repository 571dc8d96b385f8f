/*
 * awq_oracle.c -- plain, slow, scalar CPU oracle for the AWQ W4A16 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant generator with
 * the CUDA library: every conversion below (binary16 decode/encode included) is
 * written out here from its definition.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared -pthread
 * (no FMA contraction, IEEE rounding in the default round-to-nearest-even mode).
 *
 * Sources (web pages on AWQ; cited by page and section):
 *   [P2] "AWQ 的四步链路" (four-step chain) on ai.lansai.wang/107648: a linear
 *        layer Y = XW is rewritten with a positive per-input-channel scale s as
 *        Y = (X/s)(sW); the two forms are equal before quantization; the
 *        pipeline is: collect layer-input magnitudes on calibration data ->
 *        search the scaling -> fake-quantize -> quantize and pack with bits,
 *        group size and zero point.
 *   [P3] "Awq Quantization" on skillselion.com, sections "How AWQ Works"
 *        (objective L(s) = ||Q(W*s)(s^-1*X) - W*X||), "Group Size
 *        Configuration" (q_group_size = 128, w_bit = 4), "Zero-Point
 *        Quantization" (an offset handles asymmetric weight distributions).
 *   [P1] AWQ skill card on skillsmd.top, "quant_config" example
 *        (zero_point = True, q_group_size = 128, w_bit = 4).
 *   [P3] also shows the flag zero_point = False ("symmetric quantization",
 *        for symmetric weight distributions or kernels without zero points).
 *
 * Where the pages leave a step open, the reading taken is stated at the step
 * (marked READING).  Status codes mirror the CUDA library's numbering so the
 * tests can compare error behaviour, but the values are restated here.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_NULL 1
#define OR_ERR_SHAPE 2
#define OR_ERR_NONFINITE 4

#define GROUP 128   /* [P3] "Group Size Configuration": q_group_size = 128 */
#define QMAX 15     /* [P3]/[P1] w_bit = 4 -> 16 levels, codes 0..15        */

/* ---------------------------------------------------------------------------
 * IEEE 754 binary16, written from the format definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.  Every finite
 * binary16 value is an integer multiple of 2^-24.
 * ------------------------------------------------------------------------ */
double awq_oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25);     /* (1024+f) * 2^(e-25) */
    return sign ? -v : v;
}

/* Round a double to the nearest binary16, ties to even, in one rounding.
 * The quantum of the binade that holds |x| is 2^(e-11) (x in [2^(e-1), 2^e)),
 * never finer than the subnormal quantum 2^-24; n = number of quanta rounded
 * half-to-even; the encoding of n * 2^q is ((q + 24) << 10) + n, which also
 * carries correctly into the next binade when n reaches 2048. */
uint16_t awq_oracle_double_to_half(double x)
{
    if (isnan(x))
        return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a >= 65520.0)                 /* halfway between 65504 and 2^16 -> inf */
        return sign | 0x7c00;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);
    int q = e - 11;
    if (q < -24)
        q = -24;
    double n = nearbyint(ldexp(a, -q));      /* exact scaling, then RNE */
    return (uint16_t)(sign | (uint16_t)(((q + 24) << 10) + (int)n));
}

static float h2f(uint16_t h) { return (float)awq_oracle_half_to_double(h); }
static uint16_t f2h(float x) { return awq_oracle_double_to_half((double)x); }

/* ---------------------------------------------------------------------------
 * Step 1 -- activation statistics.  [P2] four-step chain, row "采集激活"
 * (collect activations): a forward pass over calibration inputs gathers the
 * magnitude of each layer-input channel.
 * READING: the magnitude is the mean absolute value over the R calibration
 * rows, m_k = (1/R) * sum_r |x[r,k]|.  The sum is taken in double: every
 * binary16 is an integer multiple of 2^-24 below 2^16, so for R <= 8192 the
 * sum is an integer multiple of 2^-24 below 2^53 * 2^-24 and is exact (hence
 * independent of summation order).  One IEEE division by R in double, then one
 * rounding to float.
 * ------------------------------------------------------------------------ */
int awq_oracle_act_stats(const uint16_t *xcal, int64_t R, int64_t K, float *m)
{
    if (!xcal || !m)
        return OR_ERR_NULL;
    if (R < 1 || K < 1)
        return OR_ERR_SHAPE;
    for (int64_t k = 0; k < K; ++k) {
        double acc = 0.0;
        for (int64_t r = 0; r < R; ++r)
            acc += fabs(awq_oracle_half_to_double(xcal[r * K + k]));
        m[k] = (float)(acc / (double)R);
    }
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Step 2 -- per-input-channel scale s.  [P2] four-step chain: Y = (X/s)(sW)
 * with s > 0 per input channel; salient channels (large activation
 * magnitude) get their weights enlarged before quantization.  [P3] "How AWQ
 * Works": s is chosen to make ||Q(W*s)(s^-1*X) - W*X|| small.
 * READING: one point of that search, s_k = m_k^0.5 normalised:
 *   t_k = sqrt(max(m_k, 1e-8))                       (double, IEEE sqrt)
 *   c   = sqrt(max_j t_j * min_j t_j)                (geometric centre)
 *   s_k = binary16_RNE(t_k / c)
 * ------------------------------------------------------------------------ */
int awq_oracle_compute_scales(const float *m, int64_t K, uint16_t *s)
{
    if (!m || !s)
        return OR_ERR_NULL;
    if (K < 1)
        return OR_ERR_SHAPE;
    double tmax = 0.0, tmin = INFINITY;
    for (int64_t k = 0; k < K; ++k) {
        if (!isfinite(m[k]) || m[k] < 0.0f)
            return OR_ERR_NONFINITE;
        double t = sqrt(fmax((double)m[k], 1e-8));
        if (t > tmax) tmax = t;
        if (t < tmin) tmin = t;
    }
    double c = sqrt(tmax * tmin);
    for (int64_t k = 0; k < K; ++k) {
        double t = sqrt(fmax((double)m[k], 1e-8));
        s[k] = awq_oracle_double_to_half(t / c);
    }
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Scale search (next row) -- [P3] "How AWQ Works": s is chosen to make
 * L(s) = ||Q(W*s)(s^-1*X) - W*X|| small; [P2] four-step chain, row "搜索缩放"
 * (evaluate the effect of different channel scalings on the reconstruction
 * error).  The pages give neither the family nor the grid.
 * READINGS:
 *   family   s(alpha) = m^alpha normalised as in step 2 (alpha = 1/2 is step 2)
 *   grid     alpha = j/8, j = 0..8, with m^alpha formed by one fixed chain of
 *            IEEE double operations, so that every result is reproducible:
 *              u = max(m, 1e-8), r1 = sqrt(u), r2 = sqrt(r1), r3 = sqrt(r2)
 *              t = u                                   (j = 8)
 *              t = 1 * [r1 if j&4] * [r2 if j&2] * [r3 if j&1]   (j < 8, in
 *                  that order, left to right)
 *            then c = sqrt(max t * min t) and s = binary16_RNE(t / c)
 *   loss     L(j) = sum over calibration rows r and outputs n of
 *            (Yq[r,n] - Y[r,n])^2 in double, Yq from the quantized layer
 *            (steps 3-8 with s(j)) and Y = X W (both in double)
 *   choice   the smallest j whose loss is the minimum
 * ------------------------------------------------------------------------ */
int awq_oracle_scales_alpha(const float *m, int64_t K, int j, uint16_t *s)
{
    if (!m || !s)
        return OR_ERR_NULL;
    if (K < 1 || j < 0 || j > 8)
        return OR_ERR_SHAPE;
    double *t = (double *)malloc(sizeof(double) * (size_t)K);
    if (!t)
        return OR_ERR_NULL;
    double tmax = 0.0, tmin = INFINITY;
    for (int64_t k = 0; k < K; ++k) {
        if (!isfinite(m[k]) || m[k] < 0.0f) {
            free(t);
            return OR_ERR_NONFINITE;
        }
        double u = fmax((double)m[k], 1e-8);
        double r1 = sqrt(u), r2 = sqrt(r1), r3 = sqrt(r2);
        double v;
        if (j == 8) {
            v = u;
        } else {
            v = 1.0;
            if (j & 4) v = v * r1;
            if (j & 2) v = v * r2;
            if (j & 1) v = v * r3;
        }
        t[k] = v;
        if (v > tmax) tmax = v;
        if (v < tmin) tmin = v;
    }
    double c = sqrt(tmax * tmin);
    for (int64_t k = 0; k < K; ++k)
        s[k] = awq_oracle_double_to_half(t[k] / c);
    free(t);
    return OR_OK;
}

int awq_oracle_quantize_pack(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N,
                             int32_t *Q, uint16_t *scales, int32_t *zeros);
int awq_oracle_matmul(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                      const uint16_t *scales, const int32_t *zeros, int64_t M, int64_t K,
                      int64_t N, const int64_t *cols, int64_t ncols, double *Y,
                      int precision, int nthreads);

int awq_oracle_scale_search(const uint16_t *xcal, int64_t R, int64_t K, const uint16_t *W, int64_t N,
                            double *losses, uint16_t *s_best, int *j_best, int nthreads)
{
    if (!xcal || !W || !losses || !s_best || !j_best)
        return OR_ERR_NULL;
    if (R < 1 || K < GROUP || K % GROUP != 0 || N < 8 || N % 8 != 0)
        return OR_ERR_SHAPE;
    int rc = OR_ERR_NULL;
    float *m = (float *)malloc(sizeof(float) * (size_t)K);
    uint16_t *s = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)K);
    int32_t *Q = (int32_t *)malloc(sizeof(int32_t) * (size_t)((K / 8) * N));
    uint16_t *sc = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)((K / GROUP) * N));
    int32_t *z = (int32_t *)malloc(sizeof(int32_t) * (size_t)((K / GROUP) * (N / 8)));
    int64_t *cols = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    double *Yq = (double *)malloc(sizeof(double) * (size_t)(R * N));
    double *Yr = (double *)malloc(sizeof(double) * (size_t)(R * N));
    if (!m || !s || !Q || !sc || !z || !cols || !Yq || !Yr)
        goto done;
    rc = awq_oracle_act_stats(xcal, R, K, m);
    if (rc != OR_OK)
        goto done;
    for (int64_t n = 0; n < N; ++n)
        cols[n] = n;
    /* Y = X W, the unquantized layer, in double (k ascending) */
    for (int64_t r = 0; r < R; ++r)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += awq_oracle_half_to_double(xcal[r * K + k]) * awq_oracle_half_to_double(W[k * N + n]);
            Yr[r * N + n] = acc;
        }
    double best = INFINITY;
    for (int j = 0; j <= 8; ++j) {
        rc = awq_oracle_scales_alpha(m, K, j, s);
        if (rc == OR_OK) rc = awq_oracle_quantize_pack(W, s, K, N, Q, sc, z);
        if (rc == OR_OK) rc = awq_oracle_matmul(xcal, s, Q, sc, z, R, K, N, cols, N, Yq, 64, nthreads);
        if (rc != OR_OK)
            goto done;
        double loss = 0.0;
        for (int64_t i = 0; i < R * N; ++i) {
            double d = Yq[i] - Yr[i];
            loss += d * d;
        }
        losses[j] = loss;
        if (loss < best) {
            best = loss;
            *j_best = j;
            memcpy(s_best, s, sizeof(uint16_t) * (size_t)K);
        }
    }
    rc = OR_OK;
done:
    free(m); free(s); free(Q); free(sc); free(z); free(cols); free(Yq); free(Yr);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Steps 3-6 -- fold s into W, asymmetric 4-bit group quantization with a zero
 * point, and packing.
 *   [P2] four-step chain: enlarge the salient channels' weights (sW), then
 *        quantize group by group; row "真实量化/打包" (real quantize / pack):
 *        store by bits, group and zero point.
 *   [P3] "Group Size Configuration", "Zero-Point Quantization": 4-bit codes,
 *        groups of 128 consecutive weights along the input dimension, an
 *        offset (zero point) for asymmetric ranges.
 * W is [K, N] row-major (Y = X W, K = input channels), s is [K].
 * READINGS (the pages give no formula):
 *   fold     w' = float(w) * float(s_k)        exact in float (11+11 bits)
 *   group    g = rows [128g, 128g+128) of one column n
 *   range    r = max(max w' - min w', 1e-5f)   float subtraction
 *   scale    scale_h = binary16_RNE(r / 15.0f), never 0 (smallest subnormal)
 *   zero     z = clamp(rint(-min w' / float(scale_h)), 0, 15)
 *   code     q = clamp(rint(w' / float(scale_h)) + z, 0, 15)
 *   rint is round-half-to-even; every division is an IEEE float division.
 *   packing  Q[k/8, n]      bits [4j, 4j+4) hold q[8(k/8)+j, n]
 *            zeros[g, n/8]  bits [4j, 4j+4) hold z[g, 8(n/8)+j]
 * ------------------------------------------------------------------------ */
int awq_oracle_quantize_pack(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N,
                             int32_t *Q, uint16_t *scales, int32_t *zeros)
{
    if (!W || !s || !Q || !scales || !zeros)
        return OR_ERR_NULL;
    if (K < GROUP || K % GROUP != 0 || N < 8 || N % 8 != 0)
        return OR_ERR_SHAPE;
    for (int64_t k = 0; k < K; ++k) {
        float sk = h2f(s[k]);
        if (!isfinite(sk) || !(sk > 0.0f))
            return OR_ERR_NONFINITE;
    }
    for (int64_t i = 0; i < K * N; ++i)
        if (!isfinite(h2f(W[i])))
            return OR_ERR_NONFINITE;

    int64_t G = K / GROUP;
    memset(Q, 0, sizeof(int32_t) * (size_t)((K / 8) * N));
    memset(zeros, 0, sizeof(int32_t) * (size_t)(G * (N / 8)));

    for (int64_t g = 0; g < G; ++g) {
        for (int64_t n = 0; n < N; ++n) {
            float mx = -INFINITY, mn = INFINITY;
            for (int64_t k = g * GROUP; k < (g + 1) * GROUP; ++k) {
                float w = h2f(W[k * N + n]) * h2f(s[k]);
                if (w > mx) mx = w;
                if (w < mn) mn = w;
            }
            float r = mx - mn;
            if (r < 1e-5f)
                r = 1e-5f;
            uint16_t sh = f2h(r / 15.0f);
            if ((sh & 0x7fff) == 0)
                sh = 1;
            float sf = h2f(sh);
            float zf = nearbyintf(-mn / sf);
            if (zf < 0.0f) zf = 0.0f;
            if (zf > (float)QMAX) zf = (float)QMAX;
            int32_t z = (int32_t)zf;
            scales[g * N + n] = sh;
            zeros[g * (N / 8) + n / 8] |= (int32_t)((uint32_t)z << (4 * (n % 8)));
            for (int64_t k = g * GROUP; k < (g + 1) * GROUP; ++k) {
                float w = h2f(W[k * N + n]) * h2f(s[k]);
                int32_t q = (int32_t)nearbyintf(w / sf) + z;
                if (q < 0) q = 0;
                if (q > QMAX) q = QMAX;
                Q[(k / 8) * N + n] |= (int32_t)((uint32_t)q << (4 * (k % 8)));
            }
        }
    }
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Weight clipping (next row) -- "Awq Quantization", calibration parameters:
 * apply_clip = True ("Apply weight clipping"); the page names only the flag.
 * READINGS:
 *   candidates  c_i = 1 - i/20, i = 0 .. n_cand-1 (n_cand <= 11: c down to 1/2),
 *               c_0 = 1 being no clipping
 *   clipped     per group g and column n, with w' = float(w) * float(s_k):
 *               hi = c * max w', lo = c * min w' (float products), then step 4 on
 *               [lo, hi]: r = max(hi - lo, 1e-5f), scale_h = binary16_RNE(r / 15)
 *               (never 0), z = clamp(rint(-lo / scale_h), 0, 15); every code of the
 *               group (clipped weights included) q = clamp(rint(w'/scale_h) + z, 0, 15)
 *   loss        the group's share of the output error on the calibration rows:
 *               sum_r (sum_{k in g} x'_rk (w_hat_kn - w'_kn))^2 in double, with
 *               x' = x / s_k in double and w_hat = (q - z) * scale_h
 *   choice      the first candidate (largest c) with the minimum loss
 * ratio_index[g * N + n] receives the chosen i.  n_cand = 1 is step 4 exactly.
 * ------------------------------------------------------------------------ */
static void group_params(float lo, float hi, uint16_t *sh_out, int32_t *z_out)
{
    float r = hi - lo;
    if (r < 1e-5f)
        r = 1e-5f;
    uint16_t sh = f2h(r / 15.0f);
    if ((sh & 0x7fff) == 0)
        sh = 1;
    float zf = nearbyintf(-lo / h2f(sh));
    if (zf < 0.0f) zf = 0.0f;
    if (zf > (float)QMAX) zf = (float)QMAX;
    *sh_out = sh;
    *z_out = (int32_t)zf;
}

static int32_t code_of(float w, uint16_t sh, int32_t z)
{
    int32_t q = (int32_t)nearbyintf(w / h2f(sh)) + z;
    if (q < 0) q = 0;
    if (q > QMAX) q = QMAX;
    return q;
}

int awq_oracle_quantize_pack_clip(const uint16_t *W, const uint16_t *s, const uint16_t *xcal, int64_t R,
                                  int64_t K, int64_t N, int n_cand, int32_t *Q, uint16_t *scales,
                                  int32_t *zeros, int32_t *ratio_index)
{
    if (!W || !s || !xcal || !Q || !scales || !zeros || !ratio_index)
        return OR_ERR_NULL;
    if (R < 1 || K < GROUP || K % GROUP != 0 || N < 8 || N % 8 != 0 || n_cand < 1 || n_cand > 11)
        return OR_ERR_SHAPE;
    for (int64_t k = 0; k < K; ++k) {
        float sk = h2f(s[k]);
        if (!isfinite(sk) || !(sk > 0.0f))
            return OR_ERR_NONFINITE;
    }
    for (int64_t i = 0; i < K * N; ++i)
        if (!isfinite(h2f(W[i])))
            return OR_ERR_NONFINITE;
    int64_t G = K / GROUP;
    double *xp = (double *)malloc(sizeof(double) * (size_t)(R * GROUP));
    if (!xp)
        return OR_ERR_NULL;
    memset(Q, 0, sizeof(int32_t) * (size_t)((K / 8) * N));
    memset(zeros, 0, sizeof(int32_t) * (size_t)(G * (N / 8)));
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t r = 0; r < R; ++r)
            for (int64_t kk = 0; kk < GROUP; ++kk) {
                int64_t k = g * GROUP + kk;
                xp[r * GROUP + kk] = awq_oracle_half_to_double(xcal[r * K + k]) /
                                     awq_oracle_half_to_double(s[k]);
            }
        for (int64_t n = 0; n < N; ++n) {
            float wp[GROUP];
            float mx = -INFINITY, mn = INFINITY;
            for (int64_t kk = 0; kk < GROUP; ++kk) {
                int64_t k = g * GROUP + kk;
                wp[kk] = h2f(W[k * N + n]) * h2f(s[k]);
                if (wp[kk] > mx) mx = wp[kk];
                if (wp[kk] < mn) mn = wp[kk];
            }
            double best = INFINITY;
            int best_i = 0;
            uint16_t best_sh = 0;
            int32_t best_z = 0;
            for (int i = 0; i < n_cand; ++i) {
                float c = 1.0f - (float)i / 20.0f;
                uint16_t sh;
                int32_t z;
                group_params(c * mn, c * mx, &sh, &z);
                double step = awq_oracle_half_to_double(sh);
                double e[GROUP];
                for (int64_t kk = 0; kk < GROUP; ++kk)
                    e[kk] = (double)(code_of(wp[kk], sh, z) - z) * step - (double)wp[kk];
                double loss = 0.0;
                for (int64_t r = 0; r < R; ++r) {
                    double y = 0.0;
                    for (int64_t kk = 0; kk < GROUP; ++kk)
                        y += xp[r * GROUP + kk] * e[kk];
                    loss += y * y;
                }
                if (loss < best) {
                    best = loss;
                    best_i = i;
                    best_sh = sh;
                    best_z = z;
                }
            }
            ratio_index[g * N + n] = best_i;
            scales[g * N + n] = best_sh;
            zeros[g * (N / 8) + n / 8] |= (int32_t)((uint32_t)best_z << (4 * (n % 8)));
            for (int64_t kk = 0; kk < GROUP; ++kk) {
                int64_t k = g * GROUP + kk;
                Q[(k / 8) * N + n] |= (int32_t)((uint32_t)code_of(wp[kk], best_sh, best_z) << (4 * (k % 8)));
            }
        }
    }
    free(xp);
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Steps 3-6, symmetric variant -- [P3] "Zero-Point Quantization": with
 * zero_point = False the 4-bit grid has no per-group offset.  The page gives
 * only the flag.
 * READINGS:
 *   fold     w' = float(w) * float(s_k), as above
 *   range    a = max(max |w'|, 1e-5f) over the group (exact)
 *   step     scale_h = binary16_RNE(a / 7.0f), never 0: the grid is centred
 *            at zero and the largest magnitude lands on level +-7
 *   code     q = clamp(rint(w' / float(scale_h)), -8, 7) + 8, stored in the
 *            same nibbles as the asymmetric codes (0..15); no zeros tensor
 *   value    w_hat = (q - 8) * scale_h, i.e. the asymmetric decode with z = 8
 * ------------------------------------------------------------------------ */
int awq_oracle_quantize_pack_symmetric(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N,
                                       int32_t *Q, uint16_t *scales)
{
    if (!W || !s || !Q || !scales)
        return OR_ERR_NULL;
    if (K < GROUP || K % GROUP != 0 || N < 8 || N % 8 != 0)
        return OR_ERR_SHAPE;
    for (int64_t k = 0; k < K; ++k) {
        float sk = h2f(s[k]);
        if (!isfinite(sk) || !(sk > 0.0f))
            return OR_ERR_NONFINITE;
    }
    for (int64_t i = 0; i < K * N; ++i)
        if (!isfinite(h2f(W[i])))
            return OR_ERR_NONFINITE;

    int64_t G = K / GROUP;
    memset(Q, 0, sizeof(int32_t) * (size_t)((K / 8) * N));
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t n = 0; n < N; ++n) {
            float amax = 0.0f;
            for (int64_t k = g * GROUP; k < (g + 1) * GROUP; ++k) {
                float w = h2f(W[k * N + n]) * h2f(s[k]);
                if (fabsf(w) > amax) amax = fabsf(w);
            }
            if (amax < 1e-5f)
                amax = 1e-5f;
            uint16_t sh = f2h(amax / 7.0f);
            if ((sh & 0x7fff) == 0)
                sh = 1;
            float sf = h2f(sh);
            scales[g * N + n] = sh;
            for (int64_t k = g * GROUP; k < (g + 1) * GROUP; ++k) {
                float w = h2f(W[k * N + n]) * h2f(s[k]);
                float level = nearbyintf(w / sf);   /* half-to-even */
                if (level < -8.0f) level = -8.0f;
                if (level > 7.0f) level = 7.0f;
                int32_t q = (int32_t)level + 8;
                Q[(k / 8) * N + n] |= (int32_t)((uint32_t)q << (4 * (k % 8)));
            }
        }
    }
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Folding 1/s into the preceding operator -- [P2] four-step chain: Y = XW is
 * rewritten as (X/s)(sW); the X/s side can be carried by the operator that
 * produces X (a normalisation weight, or the activations themselves), so the
 * matmul receives X' = X/s.
 * READING: out[r, k] = binary16_RNE(float(a[r, k]) / float(s_k)) with one IEEE
 * float division, for rows x K inputs a (a normalisation weight is rows = 1).
 * ------------------------------------------------------------------------ */
int awq_oracle_fold_inverse_scale(const uint16_t *a, int64_t rows, int64_t K, const uint16_t *s,
                                  uint16_t *out)
{
    if (!a || !s || !out)
        return OR_ERR_NULL;
    if (rows < 1 || K < 1)
        return OR_ERR_SHAPE;
    for (int64_t k = 0; k < K; ++k) {
        float sk = h2f(s[k]);
        if (!isfinite(sk) || !(sk > 0.0f))
            return OR_ERR_NONFINITE;
    }
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = f2h(h2f(a[r * K + k]) / h2f(s[k]));
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Step 7 -- dequantization (the pages' "伪量化" fake quantization: simulate the
 * low-bit weights in floating point).  w_hat[k,n] = (q - z) * scale_h, which
 * is exact in double; zeros == NULL means the symmetric grid (z = 8).  Output
 * [K, N] row-major.
 * ------------------------------------------------------------------------ */
static int code_at(const int32_t *Q, int64_t N, int64_t k, int64_t n)
{
    return (int)(((uint32_t)Q[(k / 8) * N + n] >> (4 * (k % 8))) & 0xf);
}
/* zeros == NULL: symmetric weights, every zero point is 8 */
static int zero_at(const int32_t *zeros, int64_t N, int64_t g, int64_t n)
{
    if (!zeros)
        return 8;
    return (int)(((uint32_t)zeros[g * (N / 8) + n / 8] >> (4 * (n % 8))) & 0xf);
}

int awq_oracle_dequant(const int32_t *Q, const uint16_t *scales, const int32_t *zeros,
                       int64_t K, int64_t N, double *What)
{
    if (!Q || !scales || !What)
        return OR_ERR_NULL;
    if (K < GROUP || K % GROUP != 0 || N < 8 || N % 8 != 0)
        return OR_ERR_SHAPE;
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n) {
            int64_t g = k / GROUP;
            What[k * N + n] = (double)(code_at(Q, N, k, n) - zero_at(zeros, N, g, n)) *
                              awq_oracle_half_to_double(scales[g * N + n]);
        }
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * Step 8 -- Y = (X / s) . dequant(Q), the plain definition (no blocking, k
 * ascending), for a chosen list of output columns.  [P2] four-step chain:
 * Y = (X/s)(sW).  s == NULL: X already holds X/s (1/s folded upstream), x' = x.
 *   precision 64: x' = x / s, w_hat and the sum all in double.
 *   precision 32: x' = float(x) / float(s) (IEEE float division), w_hat =
 *                 float(q - z) * float(scale_h) (exact), float accumulation
 *                 without FMA -- the dequantise-then-float-matmul form.
 * X is [M, K] row-major; Y is [M, ncols] row-major, column j of Y is output
 * column cols[j].  Work is split over output columns across nthreads POSIX
 * threads; each Y element is computed by one thread in the same order, so the
 * result does not depend on nthreads.
 * ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *X, *s, *scales;
    const int32_t *Q, *zeros;
    int64_t M, K, N, ncols;
    const int64_t *cols;
    double *Y;
    int precision;
    int64_t j0, j1;
} mm_job;

static void *mm_worker(void *arg)
{
    mm_job *jb = (mm_job *)arg;
    for (int64_t j = jb->j0; j < jb->j1; ++j) {
        int64_t n = jb->cols[j];
        for (int64_t mrow = 0; mrow < jb->M; ++mrow) {
            if (jb->precision == 64) {
                double acc = 0.0;
                for (int64_t k = 0; k < jb->K; ++k) {
                    int64_t g = k / GROUP;
                    double xp = awq_oracle_half_to_double(jb->X[mrow * jb->K + k]);
                    if (jb->s)
                        xp = xp / awq_oracle_half_to_double(jb->s[k]);
                    double wh = (double)(code_at(jb->Q, jb->N, k, n) -
                                         zero_at(jb->zeros, jb->N, g, n)) *
                                awq_oracle_half_to_double(jb->scales[g * jb->N + n]);
                    acc += xp * wh;
                }
                jb->Y[mrow * jb->ncols + j] = acc;
            } else {
                float acc = 0.0f;
                for (int64_t k = 0; k < jb->K; ++k) {
                    int64_t g = k / GROUP;
                    float xp = h2f(jb->X[mrow * jb->K + k]);
                    if (jb->s)
                        xp = xp / h2f(jb->s[k]);
                    float wh = (float)(code_at(jb->Q, jb->N, k, n) -
                                       zero_at(jb->zeros, jb->N, g, n)) *
                               h2f(jb->scales[g * jb->N + n]);
                    float p = xp * wh;
                    acc = acc + p;
                }
                jb->Y[mrow * jb->ncols + j] = (double)acc;
            }
        }
    }
    return NULL;
}

int awq_oracle_matmul(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                      const uint16_t *scales, const int32_t *zeros, int64_t M, int64_t K,
                      int64_t N, const int64_t *cols, int64_t ncols, double *Y,
                      int precision, int nthreads)
{
    /* zeros may be NULL (symmetric weights); s may be NULL (X already holds X/s) */
    if (!X || !Q || !scales || !cols || !Y)
        return OR_ERR_NULL;
    if (M < 1 || K < GROUP || K % GROUP != 0 || N < 8 || N % 8 != 0 || ncols < 1)
        return OR_ERR_SHAPE;
    if (precision != 32 && precision != 64)
        return OR_ERR_SHAPE;
    for (int64_t j = 0; j < ncols; ++j)
        if (cols[j] < 0 || cols[j] >= N)
            return OR_ERR_SHAPE;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > ncols)
        nthreads = (int)ncols;
    mm_job *jobs = (mm_job *)calloc((size_t)nthreads, sizeof(mm_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    char *live = (char *)calloc((size_t)nthreads, 1);
    if (!jobs || !tids || !live) {
        free(jobs);
        free(tids);
        free(live);
        return OR_ERR_NULL;
    }
    for (int t = 0; t < nthreads; ++t) {
        mm_job jb = {X, s, scales, Q, zeros, M, K, N, ncols, cols, Y, precision,
                     ncols * t / nthreads, ncols * (t + 1) / nthreads};
        jobs[t] = jb;
    }
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&tids[t], NULL, mm_worker, &jobs[t]) == 0)
            live[t] = 1;
        else
            mm_worker(&jobs[t]);   /* could not start a thread: do it here */
    }
    mm_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (live[t])
            pthread_join(tids[t], NULL);
    free(jobs);
    free(tids);
    free(live);
    return OR_OK;
}
