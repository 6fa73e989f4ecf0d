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

// Compress the warp-held vector x (lane l holds coordinates [l E, l E + E)
// of the input, E = WarpVec<D>::E) into slot `pos` of `page`: n = ||x||,
// y = R x, codes = bucket(y / n) stored sign-magnitude, fp16 norm; FP8 keys
// store e4m3(sqrt(d) y / n).  For QJL keys the residual r = y - nhat c[code]
// is left in r (fp32, rotated basis), rho = fp16 ||r|| is stored, and the
// function returns true (the caller projects r by S).  x is overwritten.
template <int D>
__device__ __forceinline__ bool encode_vector_warp(const Layout &L, const DevParams &P, bool is_v, float (&x)[WarpVec<D>::E],
                                                   uint8_t *page, int pos, int lane, float (&r)[WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E;
    const float rs = 1.0f / sqrtf(float(D));
    const float sqrt_d = sqrtf(float(D));
    const int bits = is_v ? L.vbits : L.kbits;
    float sg[E];
    load_vec<D>(P.signs, lane, sg);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        ss = fmaf(x[e], x[e], ss);
        x[e] *= sg[e];
    }
    const float n = sqrtf(warp_sum(ss));
    fwht_warp<D>(x, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] *= rs;          // y = R x
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

    const int nb = (1 << bits) - 1;
    uint32_t kap[E];
    float cval[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float u = x[e] * inv;
        uint32_t idx = 0;
        for (int j = 0; j < nb; ++j) idx += (P.bounds[j] <= u) ? 1u : 0u;
        kap[e] = kappa_of(idx, bits);
        cval[e] = P.lv[kap[e]];
    }
    const int code_off = is_v ? L.vc_off : L.kc_off;
    const int code_bpt = is_v ? L.vc_bpt : L.kc_bpt;
    uint8_t *cdst = page + code_off + pos * code_bpt;
    if (bits == 1) {
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

}  // namespace tq
