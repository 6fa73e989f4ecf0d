// Device helpers shared by the libtqkv kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "tq_internal.h"

namespace tq {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

// Per-warp register mapping of a d-vector: lane l holds coordinates
// [l*E, l*E + E) with E = max(1, D/32); lanes >= min(32, D) hold zeros.
template <int D>
struct WarpVec {
    static constexpr int E = D >= 32 ? D / 32 : 1;
    static constexpr int LANES = D >= 32 ? 32 : D;
};

// Unnormalised natural-order Walsh-Hadamard transform of the warp-held
// vector v (H[i][j] = (-1)^popcount(i & j)): butterflies of stride < E in
// registers, larger strides across lanes with __shfl_xor_sync.
template <int D>
__device__ __forceinline__ void fwht_warp(float (&v)[WarpVec<D>::E], int lane) {
    constexpr int E = WarpVec<D>::E, LANES = WarpVec<D>::LANES;
#pragma unroll
    for (int s = 1; s < E; s <<= 1) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if ((e & s) == 0) {
                float a = v[e], b = v[e + s];
                v[e] = a + b;
                v[e + s] = a - b;
            }
        }
    }
#pragma unroll
    for (int s = 1; s < LANES; s <<= 1) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float p = __shfl_xor_sync(kFull, v[e], s);
            v[e] = (lane & s) ? (p - v[e]) : (v[e] + p);
        }
    }
}

// Load the lane's E coordinates of a bf16 / fp32 vector.
template <int D>
__device__ __forceinline__ void load_vec(const __nv_bfloat16 *x, int lane, float (&v)[WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E, LANES = WarpVec<D>::LANES;
    if (lane >= LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = 0.f;
        return;
    }
    const __nv_bfloat16 *p = x + lane * E;
    if constexpr (E % 8 == 0) {
#pragma unroll
        for (int c = 0; c < E / 8; ++c) {
            uint4 u = reinterpret_cast<const uint4 *>(p)[c];
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = __bfloat1622float2(h[k]);
                v[c * 8 + 2 * k] = f.x;
                v[c * 8 + 2 * k + 1] = f.y;
            }
        }
    } else if constexpr (E == 4) {
        uint2 u = *reinterpret_cast<const uint2 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
        float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = __bfloat162float(p[e]);
    }
}
template <int D>
__device__ __forceinline__ void load_vec(const float *x, int lane, float (&v)[WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E, LANES = WarpVec<D>::LANES;
    if (lane >= LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = 0.f;
        return;
    }
    const float *p = x + lane * E;
    if constexpr (E % 4 == 0) {
#pragma unroll
        for (int c = 0; c < E / 4; ++c) {
            float4 u = reinterpret_cast<const float4 *>(p)[c];
            v[c * 4] = u.x; v[c * 4 + 1] = u.y; v[c * 4 + 2] = u.z; v[c * 4 + 3] = u.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = p[e];
    }
}

// Store the lane's E fields of W bits each (values in `f`, already < 2^W)
// into the token's packed array at `dst` (coordinate i at bit i*W).  When a
// lane holds fewer than 8 bits, neighbouring lanes are merged into bytes.
template <int D, int W>
__device__ __forceinline__ void store_fields(uint8_t *dst, int lane, const uint32_t (&f)[WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E, LANES = WarpVec<D>::LANES;
    constexpr int BITS = E * W;   // bits held by one lane
    if constexpr (BITS >= 32) {
        constexpr int WORDS = BITS / 32;
        constexpr int PER = 32 / W;
        uint32_t w[WORDS];
#pragma unroll
        for (int k = 0; k < WORDS; ++k) {
            uint32_t acc = 0;
#pragma unroll
            for (int e = 0; e < PER; ++e) acc |= f[k * PER + e] << (e * W);
            w[k] = acc;
        }
        if (lane >= LANES) return;
        uint32_t *out = reinterpret_cast<uint32_t *>(dst) + lane * WORDS;
        if constexpr (WORDS % 4 == 0) {
#pragma unroll
            for (int k = 0; k < WORDS; k += 4)
                reinterpret_cast<uint4 *>(out)[k / 4] = make_uint4(w[k], w[k + 1], w[k + 2], w[k + 3]);
        } else if constexpr (WORDS % 2 == 0) {
#pragma unroll
            for (int k = 0; k < WORDS; k += 2) reinterpret_cast<uint2 *>(out)[k / 2] = make_uint2(w[k], w[k + 1]);
        } else {
#pragma unroll
            for (int k = 0; k < WORDS; ++k) out[k] = w[k];
        }
    } else if constexpr (BITS == 16) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) acc |= f[e] << (e * W);
        if (lane < LANES) reinterpret_cast<uint16_t *>(dst)[lane] = uint16_t(acc);
    } else if constexpr (BITS == 8) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) acc |= f[e] << (e * W);
        if (lane < LANES) dst[lane] = uint8_t(acc);
    } else {
        // BITS in {1, 2, 4}: G lanes form one byte
        constexpr int G = 8 / BITS;
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) acc |= f[e] << (e * W);
        acc <<= (lane % G) * BITS;
#pragma unroll
        for (int o = 1; o < G; o <<= 1) acc |= __shfl_xor_sync(kFull, acc, o);
        if (lane < LANES && (lane % G) == 0) dst[lane / G] = uint8_t(acc);
    }
}

// Sign-magnitude storage code of bucket index idx for `bits` bits:
// top bit set for the negative half, low bits the magnitude rank.
__device__ __forceinline__ uint32_t kappa_of(uint32_t idx, int bits) {
    const uint32_t half = 1u << (bits - 1);
    return idx < half ? ((1u << (bits - 1)) | (half - 1u - idx)) : (idx - half);
}

__device__ __forceinline__ uint16_t f2h_bits(float x) {
    __half h = __float2half_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}
__device__ __forceinline__ float h2f_bits(uint16_t b) {
    __half h = *reinterpret_cast<__half *>(&b);
    return __half2float(h);
}

// z = M^T v for a dense fp32 matrix M [D][D] (row-major) and v in shared
// memory: z_j = sum_i M[i][j] v_i, lane l producing outputs [l E, l E + E).
// Row i is read as one coalesced run across the warp (lane l takes its E
// entries), v_i is a shared-memory broadcast.
template <int D>
__device__ __forceinline__ void dense_cols(const float *M, const float *vs, int lane, float (&z)[WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E;
#pragma unroll
    for (int e = 0; e < E; ++e) z[e] = 0.f;
    if (lane >= WarpVec<D>::LANES) return;
    const float *col = M + lane * E;
#pragma unroll 4
    for (int i = 0; i < D; ++i) {
        const float v = vs[i];
        if constexpr (E % 4 == 0) {
#pragma unroll
            for (int c = 0; c < E / 4; ++c) {
                const float4 m = reinterpret_cast<const float4 *>(col + size_t(i) * D)[c];
                z[4 * c] = fmaf(m.x, v, z[4 * c]);
                z[4 * c + 1] = fmaf(m.y, v, z[4 * c + 1]);
                z[4 * c + 2] = fmaf(m.z, v, z[4 * c + 2]);
                z[4 * c + 3] = fmaf(m.w, v, z[4 * c + 3]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) z[e] = fmaf(col[size_t(i) * D + e], v, z[e]);
        }
    }
}

// dense_cols for NV vectors at once (vs: NV x D floats): each row of M is
// read once for all of them.  The same sums in the same order as dense_cols.
template <int D, int NV>
__device__ __forceinline__ void dense_cols_n(const float *M, const float *vs, int lane,
                                             float (&z)[NV][WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E;
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int e = 0; e < E; ++e) z[v][e] = 0.f;
    if (lane >= WarpVec<D>::LANES) return;
    const float *col = M + lane * E;
#pragma unroll 2
    for (int i = 0; i < D; ++i) {
        float m[E];
        if constexpr (E % 4 == 0) {
#pragma unroll
            for (int c = 0; c < E / 4; ++c) {
                const float4 q = reinterpret_cast<const float4 *>(col + size_t(i) * D)[c];
                m[4 * c] = q.x; m[4 * c + 1] = q.y; m[4 * c + 2] = q.z; m[4 * c + 3] = q.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) m[e] = col[size_t(i) * D + e];
        }
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const float sv = vs[v * D + i];
#pragma unroll
            for (int e = 0; e < E; ++e) z[v][e] = fmaf(m[e], sv, z[v][e]);
        }
    }
}

// y = R x for the warp-held vector x (lane mapping of WarpVec): the dense
// rotation through the shared buffer wbuf (D floats of this warp), else
// H D / sqrt(D) by sign flip and butterflies.
template <int D>
__device__ __forceinline__ void rotate_warp(const DevParams &P, float (&x)[WarpVec<D>::E], float *wbuf, int lane) {
    constexpr int E = WarpVec<D>::E;
    if (P.rot) {
        if (lane < WarpVec<D>::LANES) {
#pragma unroll
            for (int e = 0; e < E; ++e) wbuf[lane * E + e] = x[e];
        }
        __syncwarp();
        dense_cols<D>(P.RdT, wbuf, lane, x);           // y_j = sum_i R[j][i] x_i = sum_i R^T[i][j] x_i
        __syncwarp();
        return;
    }
    float sg[E];
    load_vec<D>(P.signs, lane, sg);
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] *= sg[e];
    fwht_warp<D>(x, lane);
    const float rs = 1.0f / sqrtf(float(D));
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] *= rs;
}

// Value of an OCP E4M3 byte (CUDA's fp8 conversion; exact in fp16).
__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
    return __half2float(__half(h));
}

// Two E4M3 bytes (low byte -> low half) as an fp16 pair.
__device__ __forceinline__ uint32_t e4m3x2_to_half2_bits(uint32_t two_bytes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_bytes & 0xFFFFu),
                                                     __NV_E4M3);
    return uint32_t(h.x) | (uint32_t(h.y) << 16);
}

// Read W-bit field i (W in {1, 2, 4, 8}) of a packed token array.
__device__ __forceinline__ uint32_t read_field(const uint8_t *arr, int i, int W) {
    const int bit = i * W;
    return (uint32_t(arr[bit >> 3]) >> (bit & 7)) & ((1u << W) - 1u);
}

// Coordinates (2p, 2p + 1) of the unit-radius reconstruction of a polar
// code: the cos / sin factors of the centre angles on the path from the top
// level down to pair p, then the level-1 angle.  c1: the token's 4-bit
// level-1 codes; ch: its 2-bit higher-level slots (level 2 first); tab: the
// polar table (bounds, cos, sin per level; see DevParams::polar).
template <int D>
__device__ __forceinline__ float2 polar_pair(const uint8_t *c1, const uint8_t *ch, const float *tab, int p) {
    constexpr int H = D / 2;
    int level = 0;
    while ((1 << level) < D) ++level;
    float r = 1.f;
    int slot = H - 1;
#pragma unroll 1
    for (int nodes = 1; nodes < H; nodes <<= 1, --level) {
        slot -= nodes;
        const uint32_t k = read_field(ch, slot + (p >> (level - 1)), 2);
        const float *tl = tab + 48 + 12 * (level - 2);
        r *= ((p >> (level - 2)) & 1) ? tl[8 + k] : tl[4 + k];
    }
    const uint32_t k1 = read_field(c1, p, 4);
    return make_float2(r * tab[16 + k1], r * tab[32 + k1]);
}

}  // namespace tq
