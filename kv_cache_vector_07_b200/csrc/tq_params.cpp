// Parameter construction for libtqkv (host C++): random sign diagonal,
// bf16 Gaussian projection matrix and Lloyd-Max codebook.
//
// Page "What is TurboQuant?", "Stage 1": randomized Hadamard rotation, then
// per-coordinate Lloyd-Max quantization; "Where calibration-free pays off":
// the parameters depend on nothing but (d, bits, seed).
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_internal.h"

namespace {

// SplitMix64 (Steele, Lea, Flood 2014) evaluated at a counter: the output
// number (stream << 32) + i of the generator whose state starts at `seed`.
uint64_t splitmix_at(uint64_t seed, uint64_t stream, uint64_t i) {
    uint64_t z = seed + ((stream << 32) + i + 1ULL) * 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

// Round a double to the nearest bfloat16 (ties to even) by integer
// arithmetic on its binary64 encoding; returns the bf16 bits.
uint16_t bf16_bits_from_double(double v) {
    if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
    uint64_t u;
    std::memcpy(&u, &v, 8);
    const uint16_t sign = (u >> 63) ? 0x8000 : 0;
    int e = int((u >> 52) & 0x7FF) - 1023;         // unbiased exponent (v normal)
    uint64_t mant = (u & ((1ULL << 52) - 1)) | (1ULL << 52);   // 53-bit significand
    // bf16 keeps 8 significant bits for e >= -126; below that the grid is 2^-133
    int keep = 8;
    if (e < -126) keep = 8 - (-126 - e);
    if (keep <= 0) {
        // magnitude below half of the smallest subnormal step rounds to zero
        // (or to 2^-133 when above half of it)
        double a = std::fabs(v);
        double half_step = std::ldexp(1.0, -134);
        if (a > half_step) return sign | 0x0001;
        return sign;
    }
    const int drop = 53 - keep;
    uint64_t q = mant >> drop;
    const uint64_t rem = mant & ((1ULL << drop) - 1);
    const uint64_t halfway = 1ULL << (drop - 1);
    if (rem > halfway || (rem == halfway && (q & 1))) ++q;
    // q has `keep` significant bits, possibly carried to keep+1
    int exp_out = e;
    if (keep == 8) {
        if (q == (1ULL << 8)) { q >>= 1; ++exp_out; }
        const uint32_t biased = uint32_t(exp_out + 127);
        return sign | uint16_t((biased << 7) | (q & 0x7F));
    }
    // subnormal: value = q * 2^(e - keep + 1) = q * 2^-133
    if (q == (1ULL << 7)) return sign | uint16_t(1 << 7);   // rounded up to 2^-126
    return sign | uint16_t(q);
}

float bf16_to_float(uint16_t b) {
    uint32_t u = uint32_t(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// Gauss-Legendre nodes/weights on [-1, 1] by Newton iteration on P_n.
void gauss_legendre(int n, std::vector<double> &x, std::vector<double> &w) {
    x.resize(n);
    w.resize(n);
    for (int i = 0; i < n; ++i) {
        double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
        for (int it = 0; it < 100; ++it) {
            double p0 = 1.0, p1 = z;
            for (int k = 2; k <= n; ++k) {
                double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                p0 = p1;
                p1 = p2;
            }
            double dp = n * (z * p1 - p0) / (z * z - 1.0);
            double dz = p1 / dp;
            z -= dz;
            if (std::fabs(dz) < 1e-16) break;
        }
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
            double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
            p0 = p1;
            p1 = p2;
        }
        double dp = n * (z * p1 - p0) / (z * z - 1.0);
        x[i] = z;
        w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
}

// Coordinate law of a random unit vector in R^d, f(t) = K (1 - t^2)^a with
// a = (d-3)/2.  Cell probability by composite Gauss-Legendre; cell first
// moment in closed form, K [(1-lo^2)^(a+1) - (1-hi^2)^(a+1)] / (2(a+1)).
struct CoordLaw {
    double logK, a;
    std::vector<double> gx, gw;
    explicit CoordLaw(int d) {
        a = (d - 3) / 2.0;
        logK = std::lgamma(d / 2.0) - std::lgamma((d - 1) / 2.0) - 0.5 * std::log(M_PI);
        gauss_legendre(24, gx, gw);
    }
    double pdf(double t) const {
        double s = 1.0 - t * t;
        return s > 0.0 ? std::exp(logK + a * std::log(s)) : 0.0;
    }
    double mass(double lo, double hi) const {
        const int panels = 256;
        double sum = 0.0, h = (hi - lo) / panels;
        for (int p = 0; p < panels; ++p) {
            double c = lo + (p + 0.5) * h;
            for (size_t k = 0; k < gx.size(); ++k) sum += gw[k] * pdf(c + 0.5 * h * gx[k]);
        }
        return sum * 0.5 * h;
    }
    double moment(double lo, double hi) const {
        auto F = [&](double t) {
            double s = 1.0 - t * t;
            return s > 0.0 ? std::exp(logK + (a + 1.0) * std::log(s)) / (2.0 * (a + 1.0)) : 0.0;
        };
        return F(lo) - F(hi);
    }
};

// Positive half of the symmetric Lloyd-Max quantizer with 2^bits levels:
// cells [0, b1), [b1, b2), ..., [b_{h-1}, 1]; each level is its cell's
// conditional mean and each inner boundary the midpoint of its neighbours.
bool lloyd_max_positive(int d, int bits, std::vector<double> &pos) {
    const int h = 1 << (bits - 1);
    CoordLaw law(d);
    pos.assign(h, 0.0);
    const double sd = 1.0 / std::sqrt(double(d));
    for (int k = 0; k < h; ++k) pos[k] = sd * 2.5 * (k + 0.5) / h;   // any ordered start
    std::vector<double> edge(h + 1);
    for (int it = 0; it < 200000; ++it) {
        edge[0] = 0.0;
        edge[h] = 1.0;
        for (int k = 1; k < h; ++k) edge[k] = 0.5 * (pos[k - 1] + pos[k]);
        double change = 0.0;
        for (int k = 0; k < h; ++k) {
            double nc = law.moment(edge[k], edge[k + 1]) / law.mass(edge[k], edge[k + 1]);
            change = std::fmax(change, std::fabs(nc - pos[k]));
            pos[k] = nc;
        }
        if (change < 1e-15) return true;
    }
    return false;
}

// Law of the polar transform's angle between two k-dimensional sub-block
// radii of a random direction: density proportional to (sin p cos p)^(k-1)
// on [0, pi/2].  Cell mass and first moment by composite Gauss-Legendre.
struct AngleLaw {
    double km1;
    std::vector<double> gx, gw;
    explicit AngleLaw(int k) : km1(k - 1.0) { gauss_legendre(24, gx, gw); }
    double pdf(double p) const {
        const double s = std::sin(p) * std::cos(p);
        return s > 0.0 ? std::exp(km1 * std::log(s)) : 0.0;
    }
    template <typename F>
    double integral(double lo, double hi, F f) const {
        const int panels = 256;
        double sum = 0.0, h = (hi - lo) / panels;
        for (int q = 0; q < panels; ++q) {
            const double c = lo + (q + 0.5) * h;
            for (size_t j = 0; j < gx.size(); ++j) {
                const double x = c + 0.5 * h * gx[j];
                sum += gw[j] * f(x) * pdf(x);
            }
        }
        return sum * 0.5 * h;
    }
};

// Lloyd-Max levels of the angle law with 2^bits levels (ascending).  The law
// is symmetric about pi/4: the lower half of the levels is iterated with
// pi/4 as its last edge and mirrored.
bool lloyd_max_angle(int k, int bits, std::vector<double> &lv) {
    const int L = 1 << bits, h = L / 2;
    AngleLaw law(k);
    const double q = M_PI / 4.0;
    std::vector<double> c(h), edge(h + 1);
    for (int j = 0; j < h; ++j) c[j] = q * (j + 0.5) / h;          // any ordered start in (0, pi/4)
    bool ok = false;
    for (int it = 0; it < 200000 && !ok; ++it) {
        edge[0] = 0.0;
        edge[h] = q;
        for (int j = 1; j < h; ++j) edge[j] = 0.5 * (c[j - 1] + c[j]);
        double change = 0.0;
        for (int j = 0; j < h; ++j) {
            const double m0 = law.integral(edge[j], edge[j + 1], [](double) { return 1.0; });
            const double m1 = law.integral(edge[j], edge[j + 1], [](double x) { return x; });
            const double nc = m1 / m0;
            change = std::fmax(change, std::fabs(nc - c[j]));
            c[j] = nc;
        }
        ok = change < 1e-15;
    }
    if (!ok) return false;
    lv.assign(L, 0.0);
    for (int j = 0; j < h; ++j) {
        lv[j] = c[j];
        lv[L - 1 - j] = 2.0 * q - c[j];
    }
    return true;
}

}  // namespace

namespace {

// Host parameters: signs, S (bf16 bits and fp32 values), ascending levels and
// boundaries.  Returns false if the Lloyd-Max iteration fails to converge.
bool host_params(int d, int bits, uint64_t seed, std::vector<int8_t> &signs, std::vector<uint16_t> &S_bits,
                 std::vector<float> &levels, std::vector<float> &bounds) {
    const size_t dd = size_t(d) * d;
    signs.resize(d);
    for (int i = 0; i < d; ++i) signs[i] = (splitmix_at(seed, 0, i) >> 63) ? -1 : 1;
    // S: Box-Muller on pairs of 53-bit uniforms from stream 1, bf16-rounded
    S_bits.resize(dd);
    for (size_t k = 0; k < dd; k += 2) {
        const uint64_t pr = k / 2;
        const uint64_t a = splitmix_at(seed, 1, 2 * pr), b = splitmix_at(seed, 1, 2 * pr + 1);
        const double u1 = (double(a >> 11) + 1.0) * 0x1.0p-53;
        const double u2 = double(b >> 11) * 0x1.0p-53;
        const double rad = std::sqrt(-2.0 * std::log(u1));
        S_bits[k] = bf16_bits_from_double(rad * std::cos(2.0 * M_PI * u2));
        if (k + 1 < dd) S_bits[k + 1] = bf16_bits_from_double(rad * std::sin(2.0 * M_PI * u2));
    }
    levels.clear();
    bounds.clear();
    if (bits == 8) return true;
    if (bits == TQ_BITS_POLAR) {
        // level-1 angles: uniform cells of [0, 2 pi), centres as levels; then
        // 2-bit Lloyd-Max levels of the angle law for levels 2 .. log2 d
        const int L1 = 16;
        for (int j = 0; j < L1; ++j) levels.push_back(float((j + 0.5) * (2.0 * M_PI / L1)));
        for (int j = 0; j + 1 < L1; ++j) bounds.push_back(float(0.5 * (double(levels[j]) + double(levels[j + 1]))));
        for (int l = 2; (1 << l) <= d; ++l) {
            std::vector<double> lv;
            if (!lloyd_max_angle(1 << (l - 1), 2, lv)) return false;
            const size_t b0 = levels.size();
            for (double v : lv) levels.push_back(float(v));
            for (int j = 0; j + 1 < 4; ++j)
                bounds.push_back(float(0.5 * (double(levels[b0 + j]) + double(levels[b0 + j + 1]))));
        }
        return true;
    }
    // a fractional rate concatenates the (b + 1)-bit codebook and the b-bit one
    const int widths[2] = {(bits & TQ_BITS_HALF) ? (bits & 7) + 1 : bits, (bits & TQ_BITS_HALF) ? (bits & 7) : 0};
    for (int part = 0; part < 2 && widths[part] > 0; ++part) {
        const int L = 1 << widths[part], h = L / 2;
        std::vector<double> pos;
        if (!lloyd_max_positive(d, widths[part], pos)) return false;
        std::vector<float> lv(L, 0.0f);
        for (int k = 0; k < h; ++k) {
            const float c = float(pos[k]);
            lv[h + k] = c;
            lv[h - 1 - k] = -c;
        }
        for (int j = 0; j < L; ++j) levels.push_back(lv[j]);
        for (int j = 0; j + 1 < L; ++j) bounds.push_back(float(0.5 * (double(lv[j]) + double(lv[j + 1]))));
    }
    return true;
}

// Levels and bounds per code width: the first (or only) codebook, and for a
// fractional rate the second.
int log2i(int d) {
    int l = 0;
    while ((1 << l) < d) ++l;
    return l;
}
int n_levels(int bits, int d) {
    if (bits == 8) return 0;
    if (bits == TQ_BITS_POLAR) return 16 + 4 * (log2i(d) - 1);
    if (bits & TQ_BITS_HALF) return (2 << (bits & 7)) + (1 << (bits & 7));
    return 1 << bits;
}
int n_bounds(int bits, int d) {
    if (bits == 8) return 0;
    if (bits == TQ_BITS_POLAR) return 15 + 3 * (log2i(d) - 1);
    if (bits & TQ_BITS_HALF) return n_levels(bits, d) - 2;
    return (1 << bits) - 1;
}

// Dense rotation: rows of the d x d Gaussian matrix (SplitMix64 stream 2,
// Box-Muller, float64) orthonormalised in order, computed here as the
// Householder QR factorisation of its transpose with the columns of Q
// signed so that the triangular factor has a positive diagonal; stored in
// float32 (round to nearest even).
void dense_rotation_host(int d, uint64_t seed, std::vector<float> &R) {
    const size_t dd = size_t(d) * d;
    std::vector<double> g(dd);
    for (size_t k = 0; k < dd; k += 2) {
        const uint64_t pr = k / 2;
        const uint64_t a = splitmix_at(seed, 2, 2 * pr), b = splitmix_at(seed, 2, 2 * pr + 1);
        const double u1 = (double(a >> 11) + 1.0) * 0x1.0p-53;
        const double u2 = double(b >> 11) * 0x1.0p-53;
        const double rad = std::sqrt(-2.0 * std::log(u1));
        g[k] = rad * std::cos(2.0 * M_PI * u2);
        if (k + 1 < dd) g[k + 1] = rad * std::sin(2.0 * M_PI * u2);
    }
    // A = G^T (A[i][j] = G[j][i]); reflect columns k = 0 .. d-1 in turn
    std::vector<double> A(dd), vs(dd, 0.0), vn(d, 0.0);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) A[size_t(i) * d + j] = g[size_t(j) * d + i];
    for (int k = 0; k < d; ++k) {
        double xn = 0.0;
        for (int i = k; i < d; ++i) xn += A[size_t(i) * d + k] * A[size_t(i) * d + k];
        xn = std::sqrt(xn);
        const double x0 = A[size_t(k) * d + k];
        const double alpha = x0 >= 0.0 ? -xn : xn;
        double *v = &vs[size_t(k) * d];
        for (int i = k; i < d; ++i) v[i] = A[size_t(i) * d + k];
        v[k] -= alpha;
        double v2 = 0.0;
        for (int i = k; i < d; ++i) v2 += v[i] * v[i];
        vn[k] = v2;
        if (v2 == 0.0) continue;
        for (int j = k; j < d; ++j) {
            double t = 0.0;
            for (int i = k; i < d; ++i) t += v[i] * A[size_t(i) * d + j];
            const double f = 2.0 * t / v2;
            for (int i = k; i < d; ++i) A[size_t(i) * d + j] -= f * v[i];
        }
    }
    // Q = H_0 H_1 ... H_{d-1} I
    std::vector<double> Q(dd, 0.0);
    for (int i = 0; i < d; ++i) Q[size_t(i) * d + i] = 1.0;
    for (int k = d - 1; k >= 0; --k) {
        if (vn[k] == 0.0) continue;
        const double *v = &vs[size_t(k) * d];
        for (int j = 0; j < d; ++j) {
            double t = 0.0;
            for (int i = k; i < d; ++i) t += v[i] * Q[size_t(i) * d + j];
            const double f = 2.0 * t / vn[k];
            for (int i = k; i < d; ++i) Q[size_t(i) * d + j] -= f * v[i];
        }
    }
    R.assign(dd, 0.0f);
    for (int j = 0; j < d; ++j) {
        const double sg = A[size_t(j) * d + j] < 0.0 ? -1.0 : 1.0;     // sign of the triangular diagonal
        for (int i = 0; i < d; ++i) R[size_t(j) * d + i] = float(sg * Q[size_t(i) * d + j]);
    }
}

bool args_ok(int d, int bits) {
    if (d < 8 || d > 1024 || (d & (d - 1))) return false;
    if (bits == TQ_BITS_POLAR) return d >= 8 && d <= 256;
    if (bits & TQ_BITS_HALF) return (bits & ~TQ_BITS_HALF) >= 1 && (bits & ~TQ_BITS_HALF) <= 3 && d >= 16 && d <= 256;
    return bits == 1 || bits == 2 || bits == 3 || bits == 4 || bits == 8;
}

}  // namespace

extern "C" int tq_compute_params_host(int d, int bits, uint64_t seed, int8_t *signs, float *S, float *levels,
                                      float *bounds) {
    if (!args_ok(d, bits)) return TQ_EUNSUPPORTED;
    std::vector<int8_t> sg;
    std::vector<uint16_t> sb;
    std::vector<float> lv, bd;
    if (!host_params(d, bits, seed, sg, sb, lv, bd)) return TQ_EUNSUPPORTED;
    if (signs) std::memcpy(signs, sg.data(), size_t(d));
    if (S)
        for (size_t k = 0; k < sb.size(); ++k) S[k] = bf16_to_float(sb[k]);
    if (bits != 8) {
        if (levels) std::memcpy(levels, lv.data(), sizeof(float) * lv.size());
        if (bounds) std::memcpy(bounds, bd.data(), sizeof(float) * bd.size());
    }
    return TQ_OK;
}

extern "C" int tq_make_params(int d, int bits, uint64_t seed, tq_params **out) {
    return tq_make_params_rot(d, bits, seed, TQ_ROT_HADAMARD, out);
}

extern "C" int tq_make_params_rot(int d, int bits, uint64_t seed, int rotation, tq_params **out) {
    if (!out) return TQ_EINVAL;
    *out = nullptr;
    if (!args_ok(d, bits)) return TQ_EUNSUPPORTED;
    if (rotation != TQ_ROT_HADAMARD && rotation != TQ_ROT_DENSE) return TQ_EUNSUPPORTED;
    const bool dense = rotation == TQ_ROT_DENSE;
    if (dense && d > 256) return TQ_EUNSUPPORTED;
    std::vector<float> Rd;
    if (dense) dense_rotation_host(d, seed, Rd);

    std::vector<int8_t> sg;
    std::vector<uint16_t> S_bits;
    std::vector<float> lv, bd0;
    if (!host_params(d, bits, seed, sg, S_bits, lv, bd0)) return TQ_EUNSUPPORTED;

    tq_params *p = new (std::nothrow) tq_params();
    if (!p) return TQ_ENOMEM;
    p->d = d;
    p->bits = bits;
    p->seed = seed;
    cudaGetDevice(&p->device);
    const size_t dd = size_t(d) * d;
    const int L = n_levels(bits, d), NB = n_bounds(bits, d);
    p->h_signs = new int8_t[d];
    p->h_S = new float[dd];
    p->h_levels = L ? new float[L] : nullptr;
    p->h_bounds = L ? new float[NB] : nullptr;
    std::vector<float> signs_f(d);
    for (int i = 0; i < d; ++i) {
        p->h_signs[i] = sg[i];
        signs_f[i] = float(sg[i]);
    }
    for (size_t k = 0; k < dd; ++k) p->h_S[k] = bf16_to_float(S_bits[k]);
    // Device levels are indexed by the stored sign-magnitude code:
    // code = (neg << (w-1)) | rank.  Each codebook takes 32 floats of the
    // level area and 32 of the bound area (the second one: fractional rates).
    std::vector<float> lv_code(64, 0.0f), bd_dev(64, 0.0f);
    // polar tables: level-1 bounds [0, 16), cos / sin of the level-1 centres
    // [16, 32) / [32, 48); level l >= 2 at 48 + 12 (l - 2): 3 bounds, 4 cos, 4 sin;
    // for the encoder's half-plane tests, cos / sin pairs of the level-1 bounds
    // 0 .. 6 at 136 + 2j and of the level-l bounds at 152 + 6 (l - 2) + 2j (after
    // the level tables, which end at 132 for d = 256)
    std::vector<float> polar_tab(256, 0.0f);
    const bool polar = bits == TQ_BITS_POLAR;
    if (polar) {
        for (int j = 0; j < L; ++j) p->h_levels[j] = lv[j];
        for (int j = 0; j < NB; ++j) p->h_bounds[j] = bd0[j];
        for (int j = 0; j < 15; ++j) polar_tab[j] = bd0[j];
        for (int j = 0; j < 7; ++j) {
            polar_tab[136 + 2 * j] = float(std::cos(double(bd0[j])));
            polar_tab[137 + 2 * j] = float(std::sin(double(bd0[j])));
        }
        for (int j = 0; j < 16; ++j) {
            polar_tab[16 + j] = float(std::cos(double(lv[j])));
            polar_tab[32 + j] = float(std::sin(double(lv[j])));
        }
        for (int l = 2; (1 << l) <= d; ++l) {
            const int b = 48 + 12 * (l - 2), li = 16 + 4 * (l - 2), bi = 15 + 3 * (l - 2);
            for (int j = 0; j < 3; ++j) {
                polar_tab[b + j] = bd0[bi + j];
                polar_tab[152 + 6 * (l - 2) + 2 * j] = float(std::cos(double(bd0[bi + j])));
                polar_tab[152 + 6 * (l - 2) + 2 * j + 1] = float(std::sin(double(bd0[bi + j])));
            }
            for (int j = 0; j < 4; ++j) {
                polar_tab[b + 4 + j] = float(std::cos(double(lv[li + j])));
                polar_tab[b + 8 + j] = float(std::sin(double(lv[li + j])));
            }
        }
    }
    if (L && !polar) {
        for (int j = 0; j < L; ++j) p->h_levels[j] = lv[j];
        for (int j = 0; j < NB; ++j) p->h_bounds[j] = bd0[j];
        const bool half = (bits & TQ_BITS_HALF) != 0;
        const int wa = half ? (bits & 7) + 1 : bits;
        int lbase = 0, bbase = 0;
        for (int part = 0; part < (half ? 2 : 1); ++part) {
            const int w = part == 0 ? wa : wa - 1, Lw = 1 << w, h = Lw / 2;
            for (int k = 0; k < h; ++k) {
                lv_code[32 * part + k] = lv[lbase + h + k];
                lv_code[32 * part + h + k] = lv[lbase + h - 1 - k];
            }
            for (int j = 0; j + 1 < Lw; ++j) bd_dev[32 * part + j] = bd0[bbase + j];
            lbase += Lw;
            bbase += Lw - 1;
        }
    }

    // magnitude cells (see DevParams::cells) of a single 1- to 4-bit codebook
    std::vector<float> cells(64, 0.0f);
    float cellC = 0.0f;
    if (L && !polar && !(bits & TQ_BITS_HALF) && bits >= 1 && bits <= 4) {
        const int h = 1 << (bits - 1), nt = h - 1;
        std::vector<float> pos_t(static_cast<size_t>(nt)), pos_l(static_cast<size_t>(h));
        for (int k = 0; k < nt; ++k) pos_t[k] = bd0[h + k];          // positive thresholds, ascending
        for (int k = 0; k < h; ++k) pos_l[k] = lv_code[k];          // |level| by magnitude rank
        bool ok = nt == 0 || pos_t[0] > 0.0f;
        float C = 1.0f;
        if (ok && nt > 0) {
            for (int i = 0; i < 60 && C * pos_t[nt - 1] >= 15.0f; ++i) C *= 0.5f;
            for (int i = 0; i < 60 && 2.0f * C * pos_t[nt - 1] < 15.0f; ++i) C *= 2.0f;
            ok = C * pos_t[nt - 1] < 15.0f;
            for (int k = 0; ok && k + 1 < nt; ++k) ok = double(C * pos_t[k + 1]) - double(C * pos_t[k]) >= 1.0;
        }
        if (ok) {
            cellC = C;
            for (int c = 0; c < 16; ++c) {
                int mlo = 0;
                float X = 3.0e38f;
                for (int k = 0; k < nt; ++k) {
                    const float Xk = C * pos_t[k];
                    if (Xk <= float(c)) ++mlo;
                    else if (Xk < float(c + 1)) X = Xk;
                }
                float mlo_bits;
                std::memcpy(&mlo_bits, &mlo, sizeof mlo_bits);
                cells[4 * c] = X;
                cells[4 * c + 1] = mlo_bits;
                cells[4 * c + 2] = pos_l[mlo];
                cells[4 * c + 3] = pos_l[mlo + 1 < h ? mlo + 1 : mlo];
            }
        }
    }

    p->h_R = nullptr;
    std::vector<float> RdT;
    if (dense) {
        p->h_R = new float[dd];
        std::memcpy(p->h_R, Rd.data(), sizeof(float) * dd);
        RdT.assign(dd, 0.0f);
        for (int j = 0; j < d; ++j)
            for (int i = 0; i < d; ++i) RdT[size_t(i) * d + j] = Rd[size_t(j) * d + i];
    }

    // Operand images for the d = 128 tensor-core encoder (Hadamard rotation only).
    const bool imgs = d == 128 && !dense && bits != TQ_BITS_POLAR;
    std::vector<uint16_t> rot_img, s16_img;
    if (imgs) {
        rot_img.assign(128 * 128, 0);
        s16_img.assign(128 * 128, 0);
        for (int n = 0; n < 128; ++n)
            for (int k = 0; k < 128; ++k) {
                const bool neg = (__builtin_popcount(unsigned(n & k)) & 1) != (sg[k] < 0);
                rot_img[tq::sw128_image_offset(n, k) / 2] = neg ? 0xBF80 : 0x3F80;       // bf16 -1 / +1
                const __half h = __float2half_rn(bf16_to_float(S_bits[size_t(n) * 128 + k]));
                uint16_t hb;
                std::memcpy(&hb, &h, 2);
                s16_img[tq::sw128_image_offset(n, k) / 2] = hb;
            }
    }

    std::vector<uint16_t> S16(dd);
    for (size_t k = 0; k < dd; ++k) {
        const __half h = __float2half_rn(bf16_to_float(S_bits[k]));
        std::memcpy(&S16[k], &h, 2);
    }
    // one device block: signs | S (bf16) | levels by code | bounds | images | S (fp16) | polar | cells | dense
    const size_t off_signs = 0;
    const size_t off_S = 256 * ((sizeof(float) * d + 255) / 256);
    const size_t off_lv = off_S + 256 * ((sizeof(uint16_t) * dd + 255) / 256);
    const size_t off_bd = off_lv + 256;
    const size_t off_rot = off_bd + 256;
    const size_t off_s16 = off_rot + (imgs ? 32768 : 0);
    const size_t off_S16 = off_s16 + (imgs ? 32768 : 0);
    const size_t off_polar = off_S16 + 256 * ((sizeof(uint16_t) * dd + 255) / 256);
    const size_t off_cells = off_polar + (polar ? 1024 : 0);
    const size_t off_R = off_cells + 256;
    const size_t off_RT = off_R + (dense ? sizeof(float) * dd : 0);
    const size_t total = off_RT + (dense ? sizeof(float) * dd : 0);
    if (cudaMalloc(&p->d_block, total) != cudaSuccess) { p->d_block = nullptr; tq_free_params(p); return TQ_ENOMEM; }
    uint8_t *base = static_cast<uint8_t *>(p->d_block);
    if (cudaMemcpy(base + off_signs, signs_f.data(), sizeof(float) * d, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + off_S, S_bits.data(), sizeof(uint16_t) * dd, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + off_lv, lv_code.data(), 256, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + off_bd, bd_dev.data(), 256, cudaMemcpyHostToDevice) != cudaSuccess ||
        (imgs && (cudaMemcpy(base + off_rot, rot_img.data(), 32768, cudaMemcpyHostToDevice) != cudaSuccess ||
                  cudaMemcpy(base + off_s16, s16_img.data(), 32768, cudaMemcpyHostToDevice) != cudaSuccess)) ||
        cudaMemcpy(base + off_S16, S16.data(), sizeof(uint16_t) * dd, cudaMemcpyHostToDevice) != cudaSuccess ||
        (polar && cudaMemcpy(base + off_polar, polar_tab.data(), 1024, cudaMemcpyHostToDevice) != cudaSuccess) ||
        cudaMemcpy(base + off_cells, cells.data(), 256, cudaMemcpyHostToDevice) != cudaSuccess ||
        (dense && (cudaMemcpy(base + off_R, Rd.data(), sizeof(float) * dd, cudaMemcpyHostToDevice) != cudaSuccess ||
                   cudaMemcpy(base + off_RT, RdT.data(), sizeof(float) * dd, cudaMemcpyHostToDevice) != cudaSuccess))) {
        tq_free_params(p);
        return TQ_ECUDA;
    }
    p->dev.d = d;
    p->dev.bits = bits;
    p->dev.signs = reinterpret_cast<const float *>(base + off_signs);
    p->dev.S = reinterpret_cast<const uint16_t *>(base + off_S);
    p->dev.lv = reinterpret_cast<const float *>(base + off_lv);
    p->dev.bounds = reinterpret_cast<const float *>(base + off_bd);
    p->dev.lv2 = reinterpret_cast<const float *>(base + off_lv + 128);
    p->dev.bounds2 = reinterpret_cast<const float *>(base + off_bd + 128);
    p->dev.rot_img = imgs ? base + off_rot : nullptr;
    p->dev.s16_img = imgs ? base + off_s16 : nullptr;
    p->dev.S16 = reinterpret_cast<const uint16_t *>(base + off_S16);
    p->dev.polar = polar ? reinterpret_cast<const float *>(base + off_polar) : nullptr;
    p->dev.rot = dense ? 1 : 0;
    p->dev.Rd = dense ? reinterpret_cast<const float *>(base + off_R) : nullptr;
    p->dev.RdT = dense ? reinterpret_cast<const float *>(base + off_RT) : nullptr;
    p->dev.cells = cellC > 0.0f ? reinterpret_cast<const float4 *>(base + off_cells) : nullptr;
    p->dev.cellC = cellC;
    *out = p;
    return TQ_OK;
}

extern "C" void tq_free_params(tq_params *p) {
    if (!p) return;
    if (p->d_block) cudaFree(p->d_block);
    delete[] p->h_signs;
    delete[] p->h_S;
    delete[] p->h_levels;
    delete[] p->h_bounds;
    delete[] p->h_R;
    delete p;
}

extern "C" int tq_compute_rotation_host(int d, uint64_t seed, int rotation, float *R) {
    if (!R || d < 8 || d > 1024 || (d & (d - 1))) return TQ_EINVAL;
    if (rotation == TQ_ROT_DENSE) {
        if (d > 256) return TQ_EUNSUPPORTED;
        std::vector<float> Rd;
        dense_rotation_host(d, seed, Rd);
        std::memcpy(R, Rd.data(), sizeof(float) * Rd.size());
        return TQ_OK;
    }
    if (rotation != TQ_ROT_HADAMARD) return TQ_EUNSUPPORTED;
    std::vector<int8_t> sg;
    std::vector<uint16_t> sb;
    std::vector<float> lv, bd;
    if (!host_params(d, 8, seed, sg, sb, lv, bd)) return TQ_EUNSUPPORTED;
    const double s = 1.0 / std::sqrt(double(d));
    for (int j = 0; j < d; ++j)
        for (int i = 0; i < d; ++i)
            R[size_t(j) * d + i] = float(((__builtin_popcount(unsigned(j & i)) & 1) ? -s : s) * sg[i]);
    return TQ_OK;
}

extern "C" int tq_params_export_rotation(const tq_params *p, float *R) {
    if (!p || !R) return TQ_EINVAL;
    const int d = p->d;
    if (p->h_R) {
        std::memcpy(R, p->h_R, sizeof(float) * size_t(d) * d);
        return TQ_OK;
    }
    const double s = 1.0 / std::sqrt(double(d));
    for (int j = 0; j < d; ++j)
        for (int i = 0; i < d; ++i)
            R[size_t(j) * d + i] = float(((__builtin_popcount(unsigned(j & i)) & 1) ? -s : s) * p->h_signs[i]);
    return TQ_OK;
}

extern "C" int tq_params_export(const tq_params *p, int8_t *signs, float *S, float *levels,
                                float *bounds) {
    if (!p) return TQ_EINVAL;
    const size_t d = size_t(p->d);
    if (signs) std::memcpy(signs, p->h_signs, d);
    if (S) std::memcpy(S, p->h_S, sizeof(float) * d * d);
    if (p->bits != 8) {
        if (levels) std::memcpy(levels, p->h_levels, sizeof(float) * n_levels(p->bits, p->d));
        if (bounds) std::memcpy(bounds, p->h_bounds, sizeof(float) * n_bounds(p->bits, p->d));
    }
    return TQ_OK;
}
