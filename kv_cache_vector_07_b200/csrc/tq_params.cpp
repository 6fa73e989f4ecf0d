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
    const int L = 1 << bits, h = L / 2;
    std::vector<double> pos;
    if (!lloyd_max_positive(d, bits, pos)) return false;
    levels.assign(L, 0.0f);
    for (int k = 0; k < h; ++k) {
        const float c = float(pos[k]);
        levels[h + k] = c;
        levels[h - 1 - k] = -c;
    }
    bounds.assign(L - 1, 0.0f);
    for (int j = 0; j + 1 < L; ++j) bounds[j] = float(0.5 * (double(levels[j]) + double(levels[j + 1])));
    return true;
}

bool args_ok(int d, int bits) {
    if (d < 8 || d > 1024 || (d & (d - 1))) return false;
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
    if (!out) return TQ_EINVAL;
    *out = nullptr;
    if (!args_ok(d, bits)) return TQ_EUNSUPPORTED;

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
    const int L = bits == 8 ? 0 : (1 << bits);
    p->h_signs = new int8_t[d];
    p->h_S = new float[dd];
    p->h_levels = L ? new float[L] : nullptr;
    p->h_bounds = L ? new float[L - 1] : nullptr;
    std::vector<float> signs_f(d);
    for (int i = 0; i < d; ++i) {
        p->h_signs[i] = sg[i];
        signs_f[i] = float(sg[i]);
    }
    for (size_t k = 0; k < dd; ++k) p->h_S[k] = bf16_to_float(S_bits[k]);
    // Device levels are indexed by the stored sign-magnitude code:
    // code = (neg << (bits-1)) | rank.
    std::vector<float> lv_code(L > 0 ? L : 1, 0.0f);
    if (L) {
        const int h = L / 2;
        for (int j = 0; j < L; ++j) p->h_levels[j] = lv[j];
        for (int j = 0; j + 1 < L; ++j) p->h_bounds[j] = bd0[j];
        for (int k = 0; k < h; ++k) {
            lv_code[k] = lv[h + k];
            lv_code[h + k] = lv[h - 1 - k];
        }
    }

    // Operand images for the d = 128 tensor-core encoder.
    const bool imgs = d == 128;
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

    // one device block: signs | S (bf16) | levels by code | bounds | images
    const size_t off_signs = 0;
    const size_t off_S = 256 * ((sizeof(float) * d + 255) / 256);
    const size_t off_lv = off_S + 256 * ((sizeof(uint16_t) * dd + 255) / 256);
    const size_t off_bd = off_lv + 256;
    const size_t off_rot = off_bd + 256;
    const size_t off_s16 = off_rot + (imgs ? 32768 : 0);
    const size_t total = off_s16 + (imgs ? 32768 : 0);
    if (cudaMalloc(&p->d_block, total) != cudaSuccess) { p->d_block = nullptr; tq_free_params(p); return TQ_ENOMEM; }
    uint8_t *base = static_cast<uint8_t *>(p->d_block);
    std::vector<float> bd(L > 1 ? L - 1 : 1, 0.0f);
    for (int j = 0; j + 1 < L; ++j) bd[j] = p->h_bounds[j];
    if (cudaMemcpy(base + off_signs, signs_f.data(), sizeof(float) * d, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + off_S, S_bits.data(), sizeof(uint16_t) * dd, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + off_lv, lv_code.data(), sizeof(float) * lv_code.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + off_bd, bd.data(), sizeof(float) * bd.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
        (imgs && (cudaMemcpy(base + off_rot, rot_img.data(), 32768, cudaMemcpyHostToDevice) != cudaSuccess ||
                  cudaMemcpy(base + off_s16, s16_img.data(), 32768, cudaMemcpyHostToDevice) != cudaSuccess))) {
        tq_free_params(p);
        return TQ_ECUDA;
    }
    p->dev.d = d;
    p->dev.bits = bits;
    p->dev.signs = reinterpret_cast<const float *>(base + off_signs);
    p->dev.S = reinterpret_cast<const uint16_t *>(base + off_S);
    p->dev.lv = reinterpret_cast<const float *>(base + off_lv);
    p->dev.bounds = reinterpret_cast<const float *>(base + off_bd);
    p->dev.rot_img = imgs ? base + off_rot : nullptr;
    p->dev.s16_img = imgs ? base + off_s16 : nullptr;
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
    delete p;
}

extern "C" int tq_params_export(const tq_params *p, int8_t *signs, float *S, float *levels,
                                float *bounds) {
    if (!p) return TQ_EINVAL;
    const size_t d = size_t(p->d);
    if (signs) std::memcpy(signs, p->h_signs, d);
    if (S) std::memcpy(S, p->h_S, sizeof(float) * d * d);
    if (p->bits != 8) {
        const int L = 1 << p->bits;
        if (levels) std::memcpy(levels, p->h_levels, sizeof(float) * L);
        if (bounds) std::memcpy(bounds, p->h_bounds, sizeof(float) * (L - 1));
    }
    return TQ_OK;
}
