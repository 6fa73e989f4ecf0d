/*
 * TurboQuant KV-cache oracle: a plain, slow, float64 CPU restatement of what
 * the method computes.  TEST INFRASTRUCTURE ONLY: nothing on the product path
 * may link, load or call this file.  It shares no code, header, table or
 * constant generator with the CUDA library; both sides implement the
 * published SplitMix64 generator independently.
 *
 * Sources (page title, section):
 *  - "TurboQuant and RotorQuant on DGX Spark" (dev.classmethod.jp, English
 *    edition), section "Two-stage compression: PolarQuant + QJL": random
 *    rotation before quantization, no per-block scales, a 1-bit QJL
 *    correction of the quantization error, distortion within 2.7x of the
 *    information-theoretic limit.
 *  - "What is TurboQuant? mechanism, measured accuracy, status as of July
 *    2026" (issoh.co.jp), sections "Stage 1: rotation and scalar
 *    quantization by PolarQuant" (randomized Hadamard rotation, then
 *    per-coordinate Lloyd-Max quantization) and "Stage 2: removing
 *    inner-product bias with a 1-bit QJL residual" (1-bit projection of the
 *    residual makes inner-product estimates unbiased); section on the vLLM
 *    presets (FP8 keys + 4-bit values, 3/4-bit presets).
 *  - "TurboQuant" overview (ai-work-lab.com), section "QJL: condensing the
 *    residual to 1 bit": +1/-1 sign bits of a random projection of the
 *    residual; the same codec serves inner-product vector search.
 *
 * Where the pages are silent the plainest reading is taken (all readings are
 * listed in the design notes): R = H D / sqrt(d) with H the natural-order
 * Sylvester Hadamard matrix and D a random sign diagonal; the Lloyd-Max law
 * is the coordinate law of a uniformly random unit vector in R^d; the QJL
 * matrix S is m x d iid N(0,1) rounded to bf16; the estimator is
 *   <q,k> ~ nhat*<Rq, c[idx]> + rho*sqrt(pi/2)/m * sum_j (2 s_j - 1)(S R q)_j.
 *
 * Every function is a direct, unblocked statement of its definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

/* ------------------------------------------------------------------------ */
/* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number     */
/* generators", OOPSLA 2014), used counter-style: draw(seed, stream, i) is   */
/* the (stream*2^32 + i)-th output of the generator whose state starts at    */
/* `seed`.                                                                   */
/* ------------------------------------------------------------------------ */
uint64_t orc_draw(uint64_t seed, uint64_t stream, uint64_t i)
{
    const uint64_t golden_gamma = 0x9E3779B97F4A7C15ULL;
    uint64_t counter = (stream << 32) + i + 1ULL;
    uint64_t z = seed + counter * golden_gamma;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* ------------------------------------------------------------------------ */
/* Rounding to the storage formats, each from its format definition.       */
/* ------------------------------------------------------------------------ */

/* Round |v| to `mant` fractional mantissa bits with exponent floor(log2|v|),
 * clamped below at emin (subnormal grid), ties to even.  Overflow is not
 * handled here. */
static double round_to_grid(double v, int mant, int emin)
{
    if (v == 0.0 || !isfinite(v)) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) -> exponent e-1 */
    e = e - 1;
    if (e < emin) e = emin;
    double ulp = ldexp(1.0, e - mant);
    double q = a / ulp;     /* exact: power-of-two scaling */
    double r = nearbyint(q); /* default rounding mode: ties to even */
    double out = r * ulp;
    return v < 0 ? -out : out;
}

/* IEEE binary16, round to nearest even; overflow to infinity. */
double orc_round_fp16(double v)
{
    double r = round_to_grid(v, 10, -14);
    if (fabs(r) > 65504.0) return v < 0 ? -INFINITY : INFINITY;
    return r;
}

/* bfloat16 (8 exponent bits, 7 stored mantissa bits), round to nearest even. */
double orc_round_bf16(double v)
{
    return round_to_grid(v, 7, -126);
}

/* OCP FP8 E4M3 (bias 7, max finite 448, no infinities): value of a code. */
double orc_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);            /* m/8 * 2^-6 */
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* E4M3 with round-to-nearest-even and saturation to the largest finite
 * value: the nearest finite code by exhaustive search; on an exact tie the
 * code with an even mantissa LSB. */
uint8_t orc_e4m3(double v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 0x7F; ++c) {          /* all finite non-negative codes */
        double d = fabs(orc_e4m3_value((uint8_t)c) - a);
        if (d < bestd || (d == bestd && (c & 1) == 0)) { bestd = d; best = c; }
    }
    return sign | (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* Parameters: sign diagonal D, Gaussian projection S, Lloyd-Max codebook.  */
/* ------------------------------------------------------------------------ */

/* D_i = +1 or -1 from the top bit of draw(seed, 0, i). */
void orc_signs(int d, uint64_t seed, int8_t *signs)
{
    for (int i = 0; i < d; ++i)
        signs[i] = (orc_draw(seed, 0, (uint64_t)i) >> 63) ? -1 : 1;
}

/* S is m x d, row-major, entries iid N(0,1) by the Box-Muller transform of
 * two 53-bit uniforms per pair of entries, each rounded to bf16. */
void orc_gauss_bf16(int m, int d, uint64_t seed, float *S)
{
    uint64_t total = (uint64_t)m * (uint64_t)d;
    for (uint64_t k = 0; k < total; k += 2) {
        uint64_t p = k / 2;
        uint64_t a = orc_draw(seed, 1, 2 * p), b = orc_draw(seed, 1, 2 * p + 1);
        double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53;   /* (0, 1] */
        double u2 = (double)(b >> 11) * 0x1.0p-53;           /* [0, 1) */
        double rad = sqrt(-2.0 * log(u1));
        double g0 = rad * cos(2.0 * M_PI * u2);
        double g1 = rad * sin(2.0 * M_PI * u2);
        S[k] = (float)orc_round_bf16(g0);
        if (k + 1 < total) S[k + 1] = (float)orc_round_bf16(g1);
    }
}

/* Dense random rotation (the alternative to H D / sqrt(d)).  G is d x d iid
 * N(0,1) by Box-Muller of draw(seed, 2, .) pairs, row-major, full float64.
 * Its rows are orthonormalised in order by modified Gram-Schmidt (the Q of
 * the QR factorisation of G^T with a positive diagonal, transposed), and the
 * result is stored in float32 (round to nearest even), so that both sides of
 * the computation hold the same matrix.  Outputs: G (optional), Q (float64,
 * before rounding; optional) and Rm (the stored matrix, float32 values). */
void orc_dense_rotation(int d, uint64_t seed, double *G, double *Q, double *Rm)
{
    size_t dd = (size_t)d * d;
    double *g = (double *)malloc(sizeof(double) * dd);
    for (size_t k = 0; k < dd; k += 2) {
        uint64_t p = k / 2;
        uint64_t a = orc_draw(seed, 2, 2 * p), b = orc_draw(seed, 2, 2 * p + 1);
        double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53;
        double u2 = (double)(b >> 11) * 0x1.0p-53;
        double rad = sqrt(-2.0 * log(u1));
        g[k] = rad * cos(2.0 * M_PI * u2);
        if (k + 1 < dd) g[k + 1] = rad * sin(2.0 * M_PI * u2);
    }
    if (G) memcpy(G, g, sizeof(double) * dd);
    double *q = (double *)malloc(sizeof(double) * dd);
    memcpy(q, g, sizeof(double) * dd);
    for (int j = 0; j < d; ++j) {
        double *v = q + (size_t)j * d;
        for (int k = 0; k < j; ++k) {
            const double *e = q + (size_t)k * d;
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += v[i] * e[i];
            for (int i = 0; i < d; ++i) v[i] -= dot * e[i];
        }
        double nn = 0.0;
        for (int i = 0; i < d; ++i) nn += v[i] * v[i];
        nn = sqrt(nn);
        for (int i = 0; i < d; ++i) v[i] /= nn;
    }
    if (Q) memcpy(Q, q, sizeof(double) * dd);
    for (size_t k = 0; k < dd; ++k) Rm[k] = (double)(float)q[k];   /* float32, round to nearest even */
    free(g);
    free(q);
}

/* Density of one coordinate of a uniformly random unit vector in R^d:
 *   f_d(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - t^2)^((d-3)/2). */
typedef struct { double logk; double a; int moment; } dens_t;

static double dens_eval(const dens_t *D, double t)
{
    double s = 1.0 - t * t;
    if (s <= 0.0) return 0.0;
    double f = exp(D->logk + D->a * log(s));
    return D->moment ? t * f : f;
}

static double simpson_rec(const dens_t *D, double a, double b, double fa, double fm,
                          double fb, double whole, double tol, int depth)
{
    double m = 0.5 * (a + b);
    double lm = 0.5 * (a + m), rm = 0.5 * (m + b);
    double flm = dens_eval(D, lm), frm = dens_eval(D, rm);
    double left = (m - a) / 6.0 * (fa + 4.0 * flm + fm);
    double right = (b - m) / 6.0 * (fm + 4.0 * frm + fb);
    double delta = left + right - whole;
    double floor_tol = 2e-16 * fabs(left + right);   /* rounding level */
    if (depth <= 0 || fabs(delta) <= 15.0 * (tol > floor_tol ? tol : floor_tol))
        return left + right + delta / 15.0;
    return simpson_rec(D, a, m, fa, flm, fm, left, 0.5 * tol, depth - 1) +
           simpson_rec(D, m, b, fm, frm, fb, right, 0.5 * tol, depth - 1);
}

/* Adaptive Simpson quadrature of f_d (moment 0) or t*f_d (moment 1) on
 * [a, b]; the interval is first cut into 64 panels so the narrow peak of
 * f_d at large d is always resolved. */
static double integrate(int d, int moment, double a, double b)
{
    dens_t D;
    D.logk = lgamma(d / 2.0) - lgamma((d - 1) / 2.0) - 0.5 * log(M_PI);
    D.a = (d - 3) / 2.0;
    D.moment = moment;
    double sum = 0.0;
    const int panels = 64;
    for (int p = 0; p < panels; ++p) {
        double lo = a + (b - a) * p / panels, hi = a + (b - a) * (p + 1) / panels;
        double fa = dens_eval(&D, lo), fb = dens_eval(&D, hi);
        double fm = dens_eval(&D, 0.5 * (lo + hi));
        double whole = (hi - lo) / 6.0 * (fa + 4.0 * fm + fb);
        sum += simpson_rec(&D, lo, hi, fa, fm, fb, whole, 1e-16, 50);
    }
    return sum;
}

/* Inverse of the standard normal CDF by bisection on erfc. */
static double normal_quantile(double p)
{
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        double cdf = 0.5 * erfc(-mid / sqrt(2.0));
        if (cdf < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* Lloyd-Max quantizer with 2^bits levels for f_d on [-1, 1].
 * Start: the quantiles of N(0, 1/d) at (j + 1/2) / 2^bits.  Iterate: the
 * boundaries are midpoints of adjacent levels; each level is the
 * conditional mean of its cell; stop when no level moves by 1e-13.  The law
 * is symmetric, so the converged levels are symmetrised exactly.
 * Outputs: c64 (float64 levels), c32 (levels rounded to fp32) and t32
 * (boundaries (c32_j + c32_{j+1})/2 rounded to fp32).  Returns the number of
 * iterations, or -1 if the iteration did not converge. */
int orc_codebook(int d, int bits, double *c64, float *c32, float *t32)
{
    int L = 1 << bits;
    double *c = (double *)malloc(sizeof(double) * L);
    double *t = (double *)malloc(sizeof(double) * (L + 1));
    for (int j = 0; j < L; ++j)
        c[j] = normal_quantile((j + 0.5) / L) / sqrt((double)d);
    int iters = 0, converged = 0;
    for (iters = 1; iters <= 100000; ++iters) {
        t[0] = -1.0;
        t[L] = 1.0;
        for (int j = 1; j < L; ++j) t[j] = 0.5 * (c[j - 1] + c[j]);
        double maxdelta = 0.0;
        for (int j = 0; j < L; ++j) {
            double mass = integrate(d, 0, t[j], t[j + 1]);
            double mom = integrate(d, 1, t[j], t[j + 1]);
            double nc = mom / mass;
            double dl = fabs(nc - c[j]);
            if (dl > maxdelta) maxdelta = dl;
            c[j] = nc;
        }
        if (maxdelta < 1e-13) { converged = 1; break; }
    }
    for (int j = 0; j < L / 2; ++j) {
        double s = 0.5 * (c[L - 1 - j] - c[j]);
        c[j] = -s;
        c[L - 1 - j] = s;
    }
    for (int j = 0; j < L; ++j) { c64[j] = c[j]; c32[j] = (float)c[j]; }
    for (int j = 0; j + 1 < L; ++j)
        t32[j] = (float)(0.5 * ((double)c32[j] + (double)c32[j + 1]));
    free(c);
    free(t);
    return converged ? iters : -1;
}

/* ------------------------------------------------------------------------ */
/* Rotation R = H D / sqrt(d), H the natural-order Sylvester Hadamard       */
/* matrix (H[i][j] = (-1)^popcount(i & j)), computed with the fast          */
/* Walsh-Hadamard butterfly.                                                */
/* ------------------------------------------------------------------------ */
static void fwht_inplace(int d, double *v)
{
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* y = R x.  Rm != NULL selects the dense rotation: y = Rm x, Rm row-major. */
void orc_rotate(int d, const int8_t *signs, const double *Rm, const double *x, double *y)
{
    if (Rm) {
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += Rm[(size_t)j * d + i] * x[i];
            y[j] = s;
        }
        return;
    }
    for (int i = 0; i < d; ++i) y[i] = signs[i] * x[i];
    fwht_inplace(d, y);
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) y[i] *= s;
}

/* x = R^T y = D H y / sqrt(d)  (H is symmetric); dense: x = Rm^T y. */
void orc_rotate_t(int d, const int8_t *signs, const double *Rm, const double *y, double *x)
{
    if (Rm) {
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += Rm[(size_t)j * d + i] * y[j];
            x[i] = s;
        }
        return;
    }
    for (int i = 0; i < d; ++i) x[i] = y[i];
    fwht_inplace(d, x);
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) x[i] *= s * signs[i];
}

/* ------------------------------------------------------------------------ */
/* Encode.                                                                  */
/* ------------------------------------------------------------------------ */

/* Stage 1 plus optional stage 2 for n vectors of dimension d (row-major X).
 * Per vector: n = ||x||, y = R x, u = y / n (u = 0 for the zero vector),
 * idx_i = #{j : t_j <= u_i} (fractional rates, bits2 > 0: coordinates
 * d/2 .. d-1 take the bits2-bit codebook c32b / t32b instead), nhat = fp16(n), r = y - nhat * c[idx],
 * rho = fp16(||r||), s_j = [ (S r)_j >= 0 ].
 * Diagnostics for the parity exemptions: umargin[i] = min_j |u_i - t_j|
 * (unit-vector units), zmargin[j] = |(S r)_j| / (||r|| ||S_j||), and the
 * unrounded norms nraw = ||x||, rraw = ||r||.
 * sbits / rho / zmargin are only written when qjl != 0. */
void orc_encode(int n, int d, int bits, int qjl, const double *X, const int8_t *signs,
                const double *Rm, const float *S, const float *c32, const float *t32, uint8_t *idx,
                double *nhat, double *rho, uint8_t *sbits, double *umargin,
                double *zmargin, double *nraw, double *rraw,
                int bits2, const float *c32b, const float *t32b)
{
    #pragma omp parallel
    {
    double *y = (double *)malloc(sizeof(double) * d);
    double *r = (double *)malloc(sizeof(double) * d);
    #pragma omp for schedule(static)
    for (int v = 0; v < n; ++v) {
        const double *x = X + (size_t)v * d;
        orc_rotate(d, signs, Rm, x, y);
        /* n = ||x|| (= ||R x||; the dense rotation uses ||R x|| itself) */
        const double *nsrc = Rm ? y : x;
        double nn = 0.0;
        for (int i = 0; i < d; ++i) nn += nsrc[i] * nsrc[i];
        nn = sqrt(nn);
        double nh = orc_round_fp16(nn);
        nhat[v] = nh;
        if (nraw) nraw[v] = nn;
        for (int i = 0; i < d; ++i) {
            /* fractional rates: coordinates d/2 .. d-1 use the second codebook */
            int second = bits2 > 0 && i >= d / 2;
            const float *t = second ? t32b : t32, *c = second ? c32b : c32;
            int L = 1 << (second ? bits2 : bits);
            double u = nn > 0.0 ? y[i] / nn : 0.0;
            int k = 0;
            double mg = INFINITY;
            for (int j = 0; j + 1 < L; ++j) {
                if ((double)t[j] <= u) ++k;
                double dist = fabs(u - (double)t[j]);
                if (dist < mg) mg = dist;
            }
            idx[(size_t)v * d + i] = (uint8_t)k;
            if (umargin) umargin[(size_t)v * d + i] = mg;
            r[i] = y[i] - nh * (double)c[k];
        }
        if (!qjl) continue;
        double rn = 0.0;
        for (int i = 0; i < d; ++i) rn += r[i] * r[i];
        rn = sqrt(rn);
        rho[v] = orc_round_fp16(rn);
        if (rraw) rraw[v] = rn;
        int m = d;
        for (int j = 0; j < m; ++j) {
            double z = 0.0, sn = 0.0;
            for (int i = 0; i < d; ++i) {
                z += (double)S[(size_t)j * d + i] * r[i];
                sn += (double)S[(size_t)j * d + i] * (double)S[(size_t)j * d + i];
            }
            sbits[(size_t)v * m + j] = z >= 0.0 ? 1 : 0;
            if (zmargin) zmargin[(size_t)v * m + j] = rn > 0.0 ? fabs(z) / (rn * sqrt(sn)) : INFINITY;
        }
    }
    free(y);
    free(r);
    }
}

/* FP8 keys: code_i = e4m3_rne_satfinite(sqrt(d) * u_i), nhat = fp16(||x||).
 * margin[i] = distance (unit-vector units) from u_i to the nearest E4M3
 * rounding midpoint. */
void orc_encode_fp8(int n, int d, const double *X, const int8_t *signs, const double *Rm, uint8_t *code,
                    double *nhat, double *margin, double *nraw)
{
    double sd = sqrt((double)d);
    #pragma omp parallel
    {
    double *y = (double *)malloc(sizeof(double) * d);
    #pragma omp for schedule(static)
    for (int v = 0; v < n; ++v) {
        const double *x = X + (size_t)v * d;
        orc_rotate(d, signs, Rm, x, y);
        const double *nsrc = Rm ? y : x;
        double nn = 0.0;
        for (int i = 0; i < d; ++i) nn += nsrc[i] * nsrc[i];
        nn = sqrt(nn);
        nhat[v] = orc_round_fp16(nn);
        if (nraw) nraw[v] = nn;
        for (int i = 0; i < d; ++i) {
            double u = nn > 0.0 ? y[i] / nn : 0.0;
            double a = sd * u;
            code[(size_t)v * d + i] = orc_e4m3(a);
            if (margin) {
                double mg = INFINITY;
                for (int c = 0; c + 1 < 0x7F; ++c) {
                    double mid = 0.5 * (orc_e4m3_value((uint8_t)c) + orc_e4m3_value((uint8_t)(c + 1)));
                    double dist = fabs(fabs(a) - mid) / sd;
                    if (dist < mg) mg = dist;
                }
                margin[(size_t)v * d + i] = mg;
            }
        }
    }
    free(y);
    }
}

/* ------------------------------------------------------------------------ */
/* Inner-product estimate, attention, search.                               */
/* ------------------------------------------------------------------------ */

/* Compressed key set.  kind 0: Lloyd-Max codes (idx) with optional QJL
 * (sbits, rho); kind 1: FP8 codes (fp8).  All arrays index key t first. */
typedef struct {
    int kind;               /* 0 = Lloyd-Max (+QJL), 1 = FP8 */
    int qjl;
    int d;
    const int8_t *signs;    /* rotation of this key set */
    const float *S;         /* m x d, m = d (QJL only) */
    const float *c32;       /* levels (kind 0) */
    const uint8_t *idx;     /* [L][d] (kind 0) */
    const uint8_t *fp8;     /* [L][d] (kind 1) */
    const double *nhat;     /* [L] */
    const double *rho;      /* [L] (QJL only) */
    const uint8_t *sbits;   /* [L][m] (QJL only) */
    const double *Rm;       /* dense rotation (row-major d x d) or NULL */
    const float *c32b;      /* fractional rates: levels of coordinates d/2 .. d-1, or NULL */
    const double *yhat;     /* kind 2 (polar codes): reconstruction y_hat [L][d] in the rotated basis */
} orc_keys_t;

/* Estimates of <q, k_t> for t in [0, L):
 *  Lloyd-Max: nhat_t <Rq, c[idx_t]> (+ rho_t sqrt(pi/2)/m sum_j (2 s_tj - 1)(S R q)_j)
 *  FP8:       nhat_t <Rq, e4m3(code_t)> / sqrt(d). */
void orc_estimate(const orc_keys_t *K, int L, const double *q, double *est)
{
    int d = K->d, m = d;
    double *qr = (double *)malloc(sizeof(double) * d);
    double *w = (double *)malloc(sizeof(double) * m);
    orc_rotate(d, K->signs, K->Rm, q, qr);
    if (K->kind != 1 && K->qjl) {
        for (int j = 0; j < m; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += (double)K->S[(size_t)j * d + i] * qr[i];
            w[j] = s;
        }
    }
    double cq = sqrt(M_PI / 2.0) / m;
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < L; ++t) {
        double e = 0.0;
        if (K->kind == 2) {
            for (int i = 0; i < d; ++i) e += qr[i] * K->yhat[(size_t)t * d + i];
            if (K->qjl) {
                double s = 0.0;
                for (int j = 0; j < m; ++j)
                    s += (K->sbits[(size_t)t * m + j] ? 1.0 : -1.0) * w[j];
                e += K->rho[t] * cq * s;
            }
        } else if (K->kind == 1) {
            for (int i = 0; i < d; ++i) e += qr[i] * orc_e4m3_value(K->fp8[(size_t)t * d + i]);
            e = K->nhat[t] * e / sqrt((double)d);
        } else {
            for (int i = 0; i < d; ++i) {
                const float *c = (K->c32b && i >= d / 2) ? K->c32b : K->c32;
                e += qr[i] * (double)c[K->idx[(size_t)t * d + i]];
            }
            e *= K->nhat[t];
            if (K->qjl) {
                double s = 0.0;
                for (int j = 0; j < m; ++j)
                    s += (K->sbits[(size_t)t * m + j] ? 1.0 : -1.0) * w[j];
                e += K->rho[t] * cq * s;
            }
        }
        est[t] = e;
    }
    free(qr);
    free(w);
}

/* Attention for nq queries over one compressed K/V sequence of length L.
 * Query a sees keys [0, nvis[a]) (nvis == NULL: all L).  logits = est/sqrt(d);
 * p = softmax (max-subtracted, float64); in the value rotation's basis
 * o_r = sum_t p_t nhat_v,t c_v[idx_v,t]; out = R_v^T o_r.  Optional outputs:
 * logits [nq][L] (positions past nvis set to -inf) and lse [nq] (natural log
 * of the softmax denominator of the scaled logits). */
void orc_attend(int nq, int L, int d, const double *Q, const int *nvis, const orc_keys_t *K,
                const int8_t *v_signs, const double *v_Rm, const float *v_c32, const float *v_c32b,
                const double *v_yhat, const uint8_t *v_idx,
                const double *v_nhat, double *logits, double *out, double *lse)
{
    double *est = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
    double *orot = (double *)malloc(sizeof(double) * d);
    double scale = 1.0 / sqrt((double)d);
    for (int a = 0; a < nq; ++a) {
        int nv = nvis ? nvis[a] : L;
        orc_estimate(K, nv, Q + (size_t)a * d, est);
        double mx = -INFINITY;
        for (int t = 0; t < nv; ++t) { est[t] *= scale; if (est[t] > mx) mx = est[t]; }
        double den = 0.0;
        for (int i = 0; i < d; ++i) orot[i] = 0.0;
        for (int t = 0; t < nv; ++t) {
            double p = exp(est[t] - mx);
            den += p;
            double pv = p * v_nhat[t];
            if (v_yhat) {               /* polar values: y_hat already carries nhat */
                for (int i = 0; i < d; ++i) orot[i] += p * v_yhat[(size_t)t * d + i];
                continue;
            }
            for (int i = 0; i < d; ++i) {
                const float *c = (v_c32b && i >= d / 2) ? v_c32b : v_c32;
                orot[i] += pv * (double)c[v_idx[(size_t)t * d + i]];
            }
        }
        for (int i = 0; i < d; ++i) orot[i] = den > 0.0 ? orot[i] / den : 0.0;
        orc_rotate_t(d, v_signs, v_Rm, orot, out + (size_t)a * d);
        if (logits) {
            for (int t = 0; t < L; ++t) logits[(size_t)a * L + t] = t < nv ? est[t] : -INFINITY;
        }
        if (lse) lse[a] = nv > 0 ? mx + log(den) : -INFINITY;
    }
    free(est);
    free(orot);
}

/* Textbook softmax attention with exact keys and values (the identity
 * quantizer): out_a = sum_t softmax_t(<q_a, k_t>/sqrt(d)) v_t. */
void orc_attend_exact(int nq, int L, int d, const double *Q, const double *Kx,
                      const double *Vx, double *out)
{
    double *lg = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
    for (int a = 0; a < nq; ++a) {
        double mx = -INFINITY;
        for (int t = 0; t < L; ++t) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += Q[(size_t)a * d + i] * Kx[(size_t)t * d + i];
            lg[t] = s / sqrt((double)d);
            if (lg[t] > mx) mx = lg[t];
        }
        double den = 0.0;
        for (int i = 0; i < d; ++i) out[(size_t)a * d + i] = 0.0;
        for (int t = 0; t < L; ++t) {
            double p = exp(lg[t] - mx);
            den += p;
            for (int i = 0; i < d; ++i) out[(size_t)a * d + i] += p * Vx[(size_t)t * d + i];
        }
        for (int i = 0; i < d; ++i) out[(size_t)a * d + i] /= den;
    }
    free(lg);
}

/* Top-k inner-product search: for each query, the estimates of <q, x_t> over
 * the compressed database, then the k largest with ties broken towards the
 * lower index: a single pass in increasing t keeps the k best seen so far,
 * sorted by (score descending, index ascending); a later t replaces an entry
 * only with a strictly larger score. */
void orc_search(int nq, int n_db, int k, const double *Q, const orc_keys_t *K,
                double *top_scores, int64_t *top_idx)
{
    double *est = (double *)malloc(sizeof(double) * (n_db > 0 ? n_db : 1));
    for (int a = 0; a < nq; ++a) {
        double *bs = top_scores + (size_t)a * k;
        int64_t *bi = top_idx + (size_t)a * k;
        for (int r = 0; r < k; ++r) { bs[r] = -INFINITY; bi[r] = -1; }
        orc_estimate(K, n_db, Q + (size_t)a * K->d, est);
        for (int t = 0; t < n_db; ++t) {
            if (bi[k - 1] >= 0 && !(est[t] > bs[k - 1])) continue;
            int pos = k - 1;
            while (pos > 0 && (bi[pos - 1] < 0 || est[t] > bs[pos - 1])) {
                bs[pos] = bs[pos - 1];
                bi[pos] = bi[pos - 1];
                --pos;
            }
            bs[pos] = est[t];
            bi[pos] = t;
        }
    }
    free(est);
}

/* ------------------------------------------------------------------------ */
/* PolarQuant: the polar-coordinate angle quantizer ("What is TurboQuant?",  */
/* "Stage 1": the standalone PolarQuant maps the rotated vector to polar     */
/* coordinates and quantizes the angles, so that no per-vector scale other   */
/* than the final radius is stored).                                         */
/*                                                                           */
/* Transform of y in R^d (d = 2^L): level 1 takes the pairs (y_2p, y_2p+1)   */
/* to radii r1_p and angles theta_p = atan2(y_2p+1, y_2p) in [0, 2 pi);      */
/* level l = 2 .. L takes pairs of level-(l-1) radii (a, b) to sqrt(a^2+b^2) */
/* and psi = atan2(b, a) in [0, pi/2].  The level-L radius is ||y||.         */
/* Codes: theta on 2^b1 uniform cells of [0, 2 pi) (the Lloyd-Max quantizer  */
/* of the uniform law: cell centres); psi of level l by the Lloyd-Max        */
/* quantizer, 2^bh levels, of its law for a uniformly random direction:      */
/* density proportional to (sin psi cos psi)^(k-1), k = 2^(l-1).             */
/* ------------------------------------------------------------------------ */
typedef struct { double km1; int moment; } angle_dens_t;

static double angle_dens(const angle_dens_t *D, double p)
{
    double s = sin(p) * cos(p);
    if (s <= 0.0) return 0.0;
    double f = exp(D->km1 * log(s));
    return D->moment ? p * f : f;
}

static double angle_simpson(const angle_dens_t *D, double a, double b, double fa, double fm, double fb,
                            double whole, int depth)
{
    double m = 0.5 * (a + b), lm = 0.5 * (a + m), rm = 0.5 * (m + b);
    double flm = angle_dens(D, lm), frm = angle_dens(D, rm);
    double left = (m - a) / 6.0 * (fa + 4.0 * flm + fm);
    double right = (b - m) / 6.0 * (fm + 4.0 * frm + fb);
    double delta = left + right - whole;
    if (depth <= 0 || fabs(delta) <= 15.0 * 1e-17 + 3e-16 * fabs(left + right))
        return left + right + delta / 15.0;
    return angle_simpson(D, a, m, fa, flm, fm, left, depth - 1) + angle_simpson(D, m, b, fm, frm, fb, right, depth - 1);
}

static double angle_integrate(double km1, int moment, double a, double b)
{
    angle_dens_t D = {km1, moment};
    double sum = 0.0;
    const int panels = 64;
    for (int p = 0; p < panels; ++p) {
        double lo = a + (b - a) * p / panels, hi = a + (b - a) * (p + 1) / panels;
        double fa = angle_dens(&D, lo), fb = angle_dens(&D, hi), fm = angle_dens(&D, 0.5 * (lo + hi));
        sum += angle_simpson(&D, lo, hi, fa, fm, fb, (hi - lo) / 6.0 * (fa + 4.0 * fm + fb), 50);
    }
    return sum;
}

/* Lloyd-Max levels (c64, ascending) of psi for sub-block dimension k, with
 * fp32 copies c32 and fp32 midpoint boundaries t32.  Start: pi/4 plus the
 * normal quantiles scaled by 1 / (2 sqrt(k + 1)), clamped inside (0, pi/2);
 * iterate midpoints / conditional means to 1e-13; symmetrise about pi/4.
 * Returns the iteration count or -1. */
int orc_polar_codebook(int k, int bits, double *c64, float *c32, float *t32)
{
    int L = 1 << bits;
    double *c = (double *)malloc(sizeof(double) * L), *t = (double *)malloc(sizeof(double) * (L + 1));
    const double q = M_PI / 4.0, sd = 0.5 / sqrt(k + 1.0);
    for (int j = 0; j < L; ++j) {
        double v = q + sd * normal_quantile((j + 0.5) / L);
        c[j] = fmin(fmax(v, 1e-3), M_PI / 2.0 - 1e-3);
    }
    int it, ok = 0;
    for (it = 1; it <= 100000; ++it) {
        t[0] = 0.0;
        t[L] = M_PI / 2.0;
        for (int j = 1; j < L; ++j) t[j] = 0.5 * (c[j - 1] + c[j]);
        double md = 0.0;
        for (int j = 0; j < L; ++j) {
            double nc = angle_integrate(k - 1.0, 1, t[j], t[j + 1]) / angle_integrate(k - 1.0, 0, t[j], t[j + 1]);
            md = fmax(md, fabs(nc - c[j]));
            c[j] = nc;
        }
        if (md < 1e-13) { ok = 1; break; }
    }
    for (int j = 0; j < L / 2; ++j) {
        double s = 0.5 * (c[j] + (M_PI / 2.0 - c[L - 1 - j]));
        c[j] = s;
        c[L - 1 - j] = M_PI / 2.0 - s;
    }
    for (int j = 0; j < L; ++j) { c64[j] = c[j]; c32[j] = (float)c[j]; }
    for (int j = 0; j + 1 < L; ++j) t32[j] = (float)(0.5 * ((double)c32[j] + (double)c32[j + 1]));
    free(c);
    free(t);
    return ok ? it : -1;
}

/* Angle node order of the higher-level codes: level 2's d/4 angles, then
 * level 3's d/8, ..., level L's one (d/2 - 1 in all). */
static int polar_node(int d, int level, int i)
{
    int off = 0;
    for (int l = 2; l < level; ++l) off += d >> l;
    return off + i;
}

/* Reconstruction y_hat of polar codes: the level-L radius nhat, split top
 * down by the centroid angles (fp32-stored values), level 1 by theta.
 * c1: 2^b1 level-1 centroids; ch: per level l = 2 .. L (row l - 2) 2^bh
 * centroids. */
void orc_polar_decode(int n, int d, int b1, int bh, const uint8_t *codes1, const uint8_t *codesh,
                      const double *nhat, const float *c1, const float *ch, double *yhat)
{
    int Lv = 0;
    while ((1 << Lv) < d) ++Lv;
    int H = 1 << bh;
    double *r = (double *)malloc(sizeof(double) * d), *r2 = (double *)malloc(sizeof(double) * d);
    for (int v = 0; v < n; ++v) {
        r[0] = nhat[v];
        for (int l = Lv; l >= 2; --l) {
            int nodes = d >> l;
            for (int i = 0; i < nodes; ++i) {
                double psi = (double)ch[(size_t)(l - 2) * H + codesh[(size_t)v * (d / 2 - 1) + polar_node(d, l, i)]];
                r2[2 * i] = r[i] * cos(psi);
                r2[2 * i + 1] = r[i] * sin(psi);
            }
            memcpy(r, r2, sizeof(double) * 2 * nodes);
        }
        for (int p = 0; p < d / 2; ++p) {
            double th = (double)c1[codes1[(size_t)v * (d / 2) + p]];
            yhat[(size_t)v * d + 2 * p] = r[p] * cos(th);
            yhat[(size_t)v * d + 2 * p + 1] = r[p] * sin(th);
        }
    }
    free(r);
    free(r2);
}

/* Encode with the polar quantizer: y = R x, n = ||x|| (||R x|| for the
 * dense rotation), the angles of the transform, their codes, nhat = fp16(n);
 * for QJL keys the residual r = y - y_hat(codes, nhat), rho = fp16(||r||) and
 * s_j = [(S r)_j >= 0].  Margins (unit-vector units): |angle - nearest
 * boundary| x (radius being split) / n, for level 1 the boundaries 0 and
 * 2 pi included. */
void orc_encode_polar(int n, int d, int b1, int bh, int qjl, const double *X, const int8_t *signs, const double *Rm,
                      const float *S, const float *c1, const float *t1, const float *ch, const float *th,
                      uint8_t *codes1, uint8_t *codesh, double *nhat, double *yhat, double *rho, uint8_t *sbits,
                      double *margin1, double *marginh, double *zmargin, double *nraw, double *rraw)
{
    int Lv = 0;
    while ((1 << Lv) < d) ++Lv;
    int L1 = 1 << b1, H = 1 << bh;
    #pragma omp parallel
    {
    double *y = (double *)malloc(sizeof(double) * d), *r = (double *)malloc(sizeof(double) * d);
    double *r2 = (double *)malloc(sizeof(double) * d);
    #pragma omp for schedule(static)
    for (int v = 0; v < n; ++v) {
        const double *x = X + (size_t)v * d;
        orc_rotate(d, signs, Rm, x, y);
        const double *nsrc = Rm ? y : x;
        double nn = 0.0;
        for (int i = 0; i < d; ++i) nn += nsrc[i] * nsrc[i];
        nn = sqrt(nn);
        nhat[v] = orc_round_fp16(nn);
        if (nraw) nraw[v] = nn;
        for (int p = 0; p < d / 2; ++p) {
            double a = y[2 * p], b = y[2 * p + 1];
            double t = atan2(b, a);
            if (t < 0.0) t += 2.0 * M_PI;
            int k = 0;
            double mg = fmin(t, 2.0 * M_PI - t);
            for (int j = 0; j + 1 < L1; ++j) {
                if ((double)t1[j] <= t) ++k;
                mg = fmin(mg, fabs(t - (double)t1[j]));
            }
            codes1[(size_t)v * (d / 2) + p] = (uint8_t)k;
            r[p] = sqrt(a * a + b * b);
            if (margin1) margin1[(size_t)v * (d / 2) + p] = nn > 0.0 ? mg * r[p] / nn : INFINITY;
        }
        for (int l = 2; l <= Lv; ++l) {
            int nodes = d >> l;
            for (int i = 0; i < nodes; ++i) {
                double a = r[2 * i], b = r[2 * i + 1];
                double psi = atan2(b, a), rr = sqrt(a * a + b * b);
                const float *tl = th + (size_t)(l - 2) * (H - 1);
                int k = 0;
                double mg = INFINITY;
                for (int j = 0; j + 1 < H; ++j) {
                    if ((double)tl[j] <= psi) ++k;
                    mg = fmin(mg, fabs(psi - (double)tl[j]));
                }
                codesh[(size_t)v * (d / 2 - 1) + polar_node(d, l, i)] = (uint8_t)k;
                if (marginh) marginh[(size_t)v * (d / 2 - 1) + polar_node(d, l, i)] = nn > 0.0 ? mg * rr / nn : INFINITY;
                r2[i] = rr;
            }
            memcpy(r, r2, sizeof(double) * nodes);
        }
        double *yh = yhat + (size_t)v * d;
        orc_polar_decode(1, d, b1, bh, codes1 + (size_t)v * (d / 2), codesh + (size_t)v * (d / 2 - 1), nhat + v,
                         c1, ch, yh);
        if (!qjl) continue;
        double rn = 0.0;
        for (int i = 0; i < d; ++i) { r[i] = y[i] - yh[i]; rn += r[i] * r[i]; }
        rn = sqrt(rn);
        rho[v] = orc_round_fp16(rn);
        if (rraw) rraw[v] = rn;
        for (int j = 0; j < d; ++j) {
            double z = 0.0, sn = 0.0;
            for (int i = 0; i < d; ++i) {
                z += (double)S[(size_t)j * d + i] * r[i];
                sn += (double)S[(size_t)j * d + i] * (double)S[(size_t)j * d + i];
            }
            sbits[(size_t)v * d + j] = z >= 0.0 ? 1 : 0;
            if (zmargin) zmargin[(size_t)v * d + j] = rn > 0.0 ? fabs(z) / (rn * sqrt(sn)) : INFINITY;
        }
    }
    free(y);
    free(r);
    free(r2);
    }
}
