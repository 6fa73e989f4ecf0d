// One vector compressed by one warp: the steps of the write path shared by
// the general encoder and the fused decode step.
//
// Page "What is TurboQuant?", "Stage 1" (randomized Hadamard rotation, then
// per-coordinate Lloyd-Max codes with one norm per vector) and "Stage 2" (the
// residual of stage 1 is what the 1-bit QJL projection encodes); vLLM preset
// k8v4 (FP8 keys).
#pragma once

#include <cuda_fp8.h>

#include "tq_dev.cuh"

namespace tq {

// Shared-memory floats the per-vector encoder needs per warp: the dense
// rotation's staging (D), the polar transform (3 D) and two codebook copies
// (64 floats at codebook_offset) for d <= 256; the codebooks alone above.
template <int D>
__host__ __device__ constexpr int warp_buf_floats() { return D <= 256 ? (3 * D > 2 * D + 64 ? 3 * D : 2 * D + 64) : 64; }
// The same with room for four vectors staged for a dense rotation.
template <int D>
__host__ __device__ constexpr int dense_buf_floats() { return 4 * D > warp_buf_floats<D>() ? 4 * D : warp_buf_floats<D>(); }
template <int D>
__host__ __device__ constexpr int codebook_offset() { return D <= 256 ? 2 * D : 0; }

// Sign-magnitude codes and levels of the lane's E coordinates u = x inv for a
// W-bit codebook staged at tb (2^W - 1 ascending bounds, levels by code at
// +16): bucket = #{j : t_j <= u} by a binary search with compile-time steps.
template <int D, int W>
__device__ __forceinline__ void bucketize_lane(const float (&x)[WarpVec<D>::E], float inv, const float *tb,
                                               uint32_t (&kap)[WarpVec<D>::E], float (&cval)[WarpVec<D>::E]) {
    constexpr uint32_t half = 1u << (W - 1);
#pragma unroll
    for (int e = 0; e < WarpVec<D>::E; ++e) {
        const float u = x[e] * inv;
        uint32_t idx = 0;
#pragma unroll
        for (uint32_t step = half; step >= 1; step >>= 1)
            idx += (tb[idx + step - 1] <= u) ? step : 0u;
        const uint32_t k = idx < half ? (half | (half - 1u - idx)) : (idx - half);
        kap[e] = k;
        cval[e] = tb[16 + k];
    }
}

// Sign-magnitude code and level of one coordinate y (u = y inv) from the
// magnitude cells of DevParams staged at cs: the rank is the cell's count
// plus [x >= its threshold], x = cellC |u| (xs = cellC inv).  -0.0 counts as
// non-negative; a magnitude exactly on a threshold takes the upper rank.
__device__ __forceinline__ uint32_t cell_code(float y, float xs, const float4 *cs, int bits, float &level) {
    const uint32_t s = __float_as_uint(y + 0.0f) >> 31;
    const float x = fabsf(y) * xs;
    // floor(min(x, 15)) from the low mantissa bits of 2^23 + x (round toward zero)
    const uint32_t c = __float_as_uint(__fadd_rz(fminf(x, 15.0f), 8388608.0f)) & 15u;
    const float4 e = cs[c];
    const bool up = x >= e.x;
    const uint32_t mu = uint32_t(__float_as_int(e.y)) + (up ? 1u : 0u);
    const float a = up ? e.w : e.z;
    level = s ? -a : a;
    return (s << (bits - 1)) | mu;
}

// Store a fractional-rate code (coordinates 0 .. D/2-1 at wa bits, the rest
// at wb = wa - 1) of one token: the lanes' sign-magnitude codes are staged in
// shared memory (cb, D bytes of this warp), then each lane assembles whole
// bytes of the packed arrays (coordinate i at bit i * w; a 3-bit code as a
// 2-bit array and a 1-bit array).
template <int D>
__device__ __forceinline__ void store_half_codes(uint8_t *page, int pos, int lane, const uint32_t (&kap)[WarpVec<D>::E],
                                                 uint8_t *cb, int wa, int c_off, int c_bpt, int h_off, int h_bpt,
                                                 int c2_off, int c2_bpt, int h2_off, int h2_bpt) {
    constexpr int E = WarpVec<D>::E;
    if (lane < WarpVec<D>::LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) cb[lane * E + e] = uint8_t(kap[e]);
    }
    __syncwarp();
    constexpr int n = D / 2;
    for (int seg = 0; seg < 2; ++seg) {
        const int w = seg ? wa - 1 : wa, base = seg * n;
        const int mw = w == 3 ? 2 : w, per = 8 / mw;
        uint8_t *dst = page + (seg ? c2_off + pos * c2_bpt : c_off + pos * c_bpt);
        for (int j = lane; j < n * mw / 8; j += 32) {
            uint32_t byte = 0;
            for (int k = 0; k < per; ++k) byte |= (uint32_t(cb[base + j * per + k]) & ((1u << mw) - 1u)) << (k * mw);
            dst[j] = uint8_t(byte);
        }
        if (w == 3) {
            uint8_t *hd = page + (seg ? h2_off + pos * h2_bpt : h_off + pos * h_bpt);
            for (int j = lane; j < n / 8; j += 32) {
                uint32_t byte = 0;
                for (int k = 0; k < 8; ++k) byte |= ((uint32_t(cb[base + 8 * j + k]) >> 2) & 1u) << k;
                hd[j] = uint8_t(byte);
            }
        }
    }
    __syncwarp();
}

// Polar codes of the warp-held rotated vector y (lane l holds coordinates
// [l E, l E + E)), n = its norm and nh = fp16(n): the transform level by
// level through shared memory (wbuf: 3 D floats of this warp: y, two radius
// buffers, code bytes), angle codes by the bounds of P.polar, the packed
// arrays, the fp16 norm; then y_hat top down from the centres' cos / sin and
// r = y - y_hat into r.  No angle is computed: "angle of (a, b) >= bound t"
// is the half-plane test b cos t - a sin t >= 0, valid while both angles lie
// in one half turn (level 1 folds the lower half plane onto the upper one,
// 8 cells on); a zero pair takes the code of atan2 of its signed zeros.  An
// angle within ~1e-7 (relative to the radius it splits) of a bound may take
// either neighbour.
template <int D>
__device__ __forceinline__ bool polar_encode_warp(const Layout &L, const DevParams &P, bool is_v,
                                                  const float (&y)[WarpVec<D>::E], float n, uint16_t nh,
                                                  uint8_t *page, int pos, int lane, float (&r)[WarpVec<D>::E],
                                                  float *wbuf) {
    constexpr int E = WarpVec<D>::E;
    constexpr int H = D / 2;
    (void)n;
    float *ys = wbuf, *ra = wbuf + D, *rb = wbuf + D + H;
    uint8_t *cb = reinterpret_cast<uint8_t *>(wbuf + 2 * D);   // [H] level-1 codes, then [H] higher-level slots
    const float *tab = P.polar;
    if (lane < WarpVec<D>::LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) ys[lane * E + e] = y[e];
    }
    __syncwarp();
    for (int p = lane; p < H; p += 32) {
        const float a = ys[2 * p], b = ys[2 * p + 1];
        uint32_t k;
        if (a == 0.f && b == 0.f) {
            k = signbit(a) ? 8u : 0u;                         // atan2 of signed zeros: 0 or pi
        } else {
            const bool flip = b < 0.f || (b == 0.f && a < 0.f);   // angle in [pi, 2 pi)
            const float a2 = flip ? -a : a, b2 = flip ? -b : b;
            uint32_t c = 0;
#pragma unroll
            for (int j = 0; j < 7; ++j) c += fmaf(b2, tab[136 + 2 * j], -a2 * tab[137 + 2 * j]) >= 0.f ? 1u : 0u;
            k = flip ? 8u + c : c;
        }
        cb[p] = uint8_t(k);
        ra[p] = sqrtf(a * a + b * b);
    }
    __syncwarp();
    float *src = ra, *dst = rb;
    int slot = 0;
    for (int l = 2, nodes = H / 2; nodes >= 1; ++l, nodes >>= 1) {
        const float *tcs = tab + 152 + 6 * (l - 2);
        for (int i = lane; i < nodes; i += 32) {
            const float a = src[2 * i], b = src[2 * i + 1];    // radii: the angle lies in [0, pi/2]
            uint32_t k = 0;
            if (a != 0.f || b != 0.f) {
#pragma unroll
                for (int j = 0; j < 3; ++j) k += fmaf(b, tcs[2 * j], -a * tcs[2 * j + 1]) >= 0.f ? 1u : 0u;
            }
            cb[H + slot + i] = uint8_t(k);
            dst[i] = sqrtf(a * a + b * b);
        }
        slot += nodes;
        __syncwarp();
        float *t2 = src; src = dst; dst = t2;
    }
    if (lane == 0) cb[H + H - 1] = 0;                          // the unused last slot
    __syncwarp();
    // packed arrays: 4-bit level-1 fields, 2-bit higher-level fields
    const int c_off = is_v ? L.vc_off : L.kc_off, c_bpt = is_v ? L.vc_bpt : L.kc_bpt;
    const int c2_off = is_v ? L.vc2_off : L.kc2_off, c2_bpt = is_v ? L.vc2_bpt : L.kc2_bpt;
    for (int j = lane; j < H / 2; j += 32)
        page[c_off + pos * c_bpt + j] = uint8_t(cb[2 * j] | (cb[2 * j + 1] << 4));
    for (int j = lane; j < H / 4; j += 32)
        page[c2_off + pos * c2_bpt + j] =
            uint8_t(cb[H + 4 * j] | (cb[H + 4 * j + 1] << 2) | (cb[H + 4 * j + 2] << 4) | (cb[H + 4 * j + 3] << 6));
    if (lane == 0) *reinterpret_cast<uint16_t *>(page + (is_v ? L.vn_off : L.kn_off) + pos * 2) = nh;
    if (is_v || !L.kqjl) return false;
    // y_hat: the stored radius split top down by the centre angles
    const float nhf = h2f_bits(nh);
    src = ra; dst = rb;
    if (lane == 0) src[0] = nhf;
    __syncwarp();
    // levels log2 D .. 2 top down; level l has D >> l angles, stored from
    // slot H - 1 - (its count and those of the levels above) upward
    slot = H - 1;
    int level = 0;
    while ((1 << level) < D) ++level;
    for (int nodes = 1; nodes < H; nodes <<= 1, --level) {
        slot -= nodes;
        const float *tl = tab + 48 + 12 * (level - 2);
        for (int i = lane; i < nodes; i += 32) {
            const uint32_t k = cb[H + slot + i];
            dst[2 * i] = src[i] * tl[4 + k];
            dst[2 * i + 1] = src[i] * tl[8 + k];
        }
        __syncwarp();
        float *t2 = src; src = dst; dst = t2;
    }
    for (int p = lane; p < H; p += 32) {
        const uint32_t k = cb[p];
        ys[2 * p] = src[p] * tab[16 + k];                          // y_hat over y's staging area
        ys[2 * p + 1] = src[p] * tab[32 + k];
    }
    __syncwarp();
    float rr = 0.f;
    const bool active = lane < WarpVec<D>::LANES;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        r[e] = active ? y[e] - ys[lane * E + e] : 0.f;
        rr = fmaf(r[e], r[e], rr);
    }
    const float rho = sqrtf(warp_sum(rr));
    if (lane == 0) *reinterpret_cast<uint16_t *>(page + L.kr_off + pos * 2) = f2h_bits(rho);
    __syncwarp();
    return true;
}

// Compress the warp-held vector x (lane l holds coordinates [l E, l E + E)
// of the input, E = WarpVec<D>::E) into slot `pos` of `page`: n = ||x||,
// y = R x, codes = bucket(y / n) stored sign-magnitude, fp16 norm; FP8 keys
// store e4m3(sqrt(d) y / n).  For QJL keys the residual r = y - nhat c[code]
// is left in r (fp32, rotated basis), rho = fp16 ||r|| is stored, and the
// function returns true (the caller projects r by S).  x is overwritten.
//
// The dense rotation (P.rot) takes y = R x through wbuf (D floats of shared
// memory for this warp) and the norm of y; H D / sqrt(d) the norm of x.
// With `rotated` the caller has already applied a dense rotation: x is y.
template <int D>
__device__ __forceinline__ bool encode_vector_warp(const Layout &L, const DevParams &P, bool is_v, float (&x)[WarpVec<D>::E],
                                                   uint8_t *page, int pos, int lane, float (&r)[WarpVec<D>::E],
                                                   float *wbuf, bool rotated = false) {
    constexpr int E = WarpVec<D>::E;
    const float sqrt_d = sqrtf(float(D));
    const int bits = is_v ? L.vbits : L.kbits;
    float ss = 0.f;
    if (!P.rot) {
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
    }
    if (!rotated) rotate_warp<D>(P, x, wbuf, lane);     // y = R x
    if (P.rot) {
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
    }
    const float n = sqrtf(warp_sum(ss));
    const float inv = n > 0.f ? 1.0f / n : 0.f;
    const uint16_t nh = f2h_bits(n);
    const float nhf = h2f_bits(nh);

    if (!is_v && L.kbits == 8) {
        uint32_t f[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            // the zero vector has u = +0 (not the -0 a sign flip of a zero leaves)
            f[e] = uint32_t(__nv_cvt_float_to_fp8(n > 0.f ? sqrt_d * (x[e] * inv) : 0.f, __NV_SATFINITE, __NV_E4M3));
        store_fields<D, 8>(page + L.kc_off + pos * L.kc_bpt, lane, f);
        if (lane == 0) *reinterpret_cast<uint16_t *>(page + L.kn_off + pos * 2) = nh;
        return false;
    }

    if (is_v ? L.vpolar : L.kpolar) {
        // polar codes: transform, codes and (keys with QJL) the residual y - y_hat
        const bool res = polar_encode_warp<D>(L, P, is_v, x, n, nh, page, pos, lane, r, wbuf);
        return res && !is_v && L.kqjl;
    }
    // fractional rates: lanes holding coordinates d/2 .. d-1 use the second codebook
    const bool half = is_v ? L.vhalf : L.khalf;
    uint32_t kap[E];
    float cval[E];
    float *tbase = wbuf + codebook_offset<D>();
    if (P.cells && !half) {
        // one magnitude-cell lookup per coordinate
        __syncwarp();
        if (lane < 16) reinterpret_cast<float4 *>(tbase)[lane] = P.cells[lane];
        __syncwarp();
        const float xs = P.cellC * inv;
#pragma unroll
        for (int e = 0; e < E; ++e) kap[e] = cell_code(x[e], xs, reinterpret_cast<const float4 *>(tbase), bits, cval[e]);
        __syncwarp();
    } else {
        const bool second = half && lane >= WarpVec<D>::LANES / 2;
        const int wbits = half ? (second ? (is_v ? L.vb_bits : L.kb_bits) : (is_v ? L.va_bits : L.ka_bits)) : bits;
        // bucket = #{j : t_j <= u} by a binary search over this lane's codebook,
        // staged in the warp's buffer (lanes of the second half of a fractional
        // rate use their own copy): 2^W - 1 ascending bounds, then 2^W levels
        __syncwarp();
        for (int j = lane; j < 64; j += 32) {            // both codebooks, by all lanes
            const int seg = j >> 5, o = j & 31;
            if (seg == 1 && !half) continue;
            const int w = half ? (seg ? (is_v ? L.vb_bits : L.kb_bits) : (is_v ? L.va_bits : L.ka_bits)) : bits;
            if (o < (1 << w) - 1) tbase[j] = (seg ? P.bounds2 : P.bounds)[o];
            else if (o >= 16 && o < 16 + (1 << w)) tbase[j] = (seg ? P.lv2 : P.lv)[o - 16];
        }
        __syncwarp();
        const float *tb = tbase + (second ? 32 : 0);
        switch (wbits) {                                  // the search unrolled per width
            case 1: bucketize_lane<D, 1>(x, inv, tb, kap, cval); break;
            case 2: bucketize_lane<D, 2>(x, inv, tb, kap, cval); break;
            case 3: bucketize_lane<D, 3>(x, inv, tb, kap, cval); break;
            default: bucketize_lane<D, 4>(x, inv, tb, kap, cval); break;
        }
        __syncwarp();
    }
    const int code_off = is_v ? L.vc_off : L.kc_off;
    const int code_bpt = is_v ? L.vc_bpt : L.kc_bpt;
    uint8_t *cdst = page + code_off + pos * code_bpt;
    if (half) {
        if (is_v)
            store_half_codes<D>(page, pos, lane, kap, reinterpret_cast<uint8_t *>(wbuf), L.va_bits, L.vc_off, L.vc_bpt,
                                L.vh_off, L.vh_bpt, L.vc2_off, L.vc2_bpt, L.vh2_off, L.vh2_bpt);
        else
            store_half_codes<D>(page, pos, lane, kap, reinterpret_cast<uint8_t *>(wbuf), L.ka_bits, L.kc_off, L.kc_bpt,
                                L.kh_off, L.kh_bpt, L.kc2_off, L.kc2_bpt, L.kh2_off, L.kh2_bpt);
    } else if (bits == 1) {
        store_fields<D, 1>(cdst, lane, kap);
    } else if (bits == 2) {
        store_fields<D, 2>(cdst, lane, kap);
    } else if (bits == 4) {
        store_fields<D, 4>(cdst, lane, kap);
    } else {   // 3 bits: 2-bit magnitude array + 1-bit sign array
        uint32_t lo[E], hi[E];
#pragma unroll
        for (int e = 0; e < E; ++e) { lo[e] = kap[e] & 3u; hi[e] = kap[e] >> 2; }
        store_fields<D, 2>(cdst, lane, lo);
        const int hoff = is_v ? L.vh_off : L.kh_off;
        const int hbpt = is_v ? L.vh_bpt : L.kh_bpt;
        store_fields<D, 1>(page + hoff + pos * hbpt, lane, hi);
    }
    if (lane == 0) *reinterpret_cast<uint16_t *>(page + (is_v ? L.vn_off : L.kn_off) + pos * 2) = nh;

    if (is_v || !L.kqjl) return false;
    float rr = 0.f;
    const bool active = lane < WarpVec<D>::LANES;    // lanes past d hold no coordinate
#pragma unroll
    for (int e = 0; e < E; ++e) {
        r[e] = active ? fmaf(-nhf, cval[e], x[e]) : 0.f;
        rr = fmaf(r[e], r[e], rr);
    }
    const float rho = sqrtf(warp_sum(rr));
    if (lane == 0) *reinterpret_cast<uint16_t *>(page + L.kr_off + pos * 2) = f2h_bits(rho);
    return true;
}

// d = 1024 under H D / 32 with magnitude cells (the general encoder's
// search-database shape): the same butterflies as fwht_warp, but the five
// lane-crossing strides run in registers after a transpose through shared
// memory, so lane l ends with coordinates 32 j + l (j < 32).  Each of the
// lane's residual stores is then one coalesced 128-byte row of the warp, and
// the codes return to coordinate order through the same buffer (tbuf: 1024
// floats of this warp; cs: the staged cells).  Returns whether the residual
// (times 2^e, ||r|| 2^e in [2^10, 2^11)) was written to resid.
__device__ __forceinline__ bool encode1024_t(const Layout &L, const DevParams &P, bool is_v, float (&x)[32],
                                             uint8_t *page, int pos, int lane, float *tbuf, const float4 *cs,
                                             float *resid) {
    const int bits = is_v ? L.vbits : L.kbits;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fmaf(x[e], x[e], ss);
    const float n = sqrtf(warp_sum(ss));
    {
        float sg[32];
        load_vec<1024>(P.signs, lane, sg);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] *= sg[e];
    }
    // strides 1 .. 16 (coordinate bits 0 .. 4) inside the lane
#pragma unroll
    for (int s = 1; s < 32; s <<= 1)
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if ((e & s) == 0) {
                const float a = x[e], b = x[e + s];
                x[e] = a + b;
                x[e + s] = a - b;
            }
    // transpose: element e of lane l at row e, column l ^ e (no bank conflicts
    // either way); afterwards x[j] is coordinate 32 j + lane
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 32; ++e) tbuf[e * 32 + (lane ^ e)] = x[e];
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = tbuf[lane * 32 + (j ^ lane)];
    // strides 32 .. 512 (coordinate bits 5 .. 9), now inside the lane
#pragma unroll
    for (int s = 1; s < 32; s <<= 1)
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if ((e & s) == 0) {
                const float a = x[e], b = x[e + s];
                x[e] = a + b;
                x[e + s] = a - b;
            }
    const float inv = n > 0.f ? 1.0f / n : 0.f;
    const uint16_t nh = f2h_bits(n);
    const float nhf = h2f_bits(nh);
    const float xs = P.cellC * inv;
    const bool qjl = !is_v && L.kqjl;
    uint8_t *cb = reinterpret_cast<uint8_t *>(tbuf);
    float rr = 0.f;
    __syncwarp();                                     // every lane has read its column
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float y = x[j] * 0.03125f;              // 1 / sqrt(1024)
        float c;
        cb[32 * j + lane] = uint8_t(cell_code(y, xs, cs, bits, c));
        x[j] = fmaf(-nhf, c, y);                      // residual (used for QJL keys only)
        rr = fmaf(x[j], x[j], rr);
    }
    __syncwarp();
    // codes in coordinate order: lane l packs coordinates [32 l, 32 l + 32)
    {
        uint32_t kap[32];
        const uint4 *src = reinterpret_cast<const uint4 *>(cb + 32 * lane);
        const uint4 q0 = src[0], q1 = src[1];
        const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int e = 0; e < 32; ++e) kap[e] = (w[e >> 2] >> (8 * (e & 3))) & 0xFFu;
        uint8_t *cdst = page + (is_v ? L.vc_off : L.kc_off) + pos * (is_v ? L.vc_bpt : L.kc_bpt);
        if (bits == 1) {
            store_fields<1024, 1>(cdst, lane, kap);
        } else if (bits == 2) {
            store_fields<1024, 2>(cdst, lane, kap);
        } else if (bits == 4) {
            store_fields<1024, 4>(cdst, lane, kap);
        } else {   // 3 bits: 2-bit magnitude array + 1-bit sign array
            uint32_t hi[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) { hi[e] = kap[e] >> 2; kap[e] &= 3u; }
            store_fields<1024, 2>(cdst, lane, kap);
            store_fields<1024, 1>(page + (is_v ? L.vh_off : L.kh_off) + pos * (is_v ? L.vh_bpt : L.kh_bpt), lane, hi);
        }
    }
    __syncwarp();                                     // the buffer is free again
    if (lane == 0) *reinterpret_cast<uint16_t *>(page + (is_v ? L.vn_off : L.kn_off) + pos * 2) = nh;
    if (!qjl) return false;
    rr = warp_sum(rr);
    if (lane == 0) *reinterpret_cast<uint16_t *>(page + L.kr_off + pos * 2) = f2h_bits(sqrtf(rr));
    float sc = 1.f;
    if (rr > 0.f) {
        const int ex = ((__float_as_int(sqrtf(rr)) >> 23) & 0xff) - 127;
        sc = __int_as_float(min(254, max(1, 127 + 10 - ex)) << 23);
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) resid[32 * j + lane] = x[j] * sc;
    return true;
}

}  // namespace tq
