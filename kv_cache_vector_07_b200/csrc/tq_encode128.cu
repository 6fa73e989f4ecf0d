// Fused write path for head dimension 128 with bf16 inputs: one persistent
// kernel does the rotation, the Lloyd-Max codes, the residual and the QJL
// projection, with both dense steps on the tensor cores.
//
// Page "What is TurboQuant?", "Stage 1" (randomized Hadamard rotation, then
// per-coordinate Lloyd-Max codes, no per-block scale) and "Stage 2" (1-bit
// QJL projection of the residual); ai-work-lab overview, "QJL".
//
// Per tile of 128 vectors (one vector per TMEM lane / thread row):
//   TMA     x tile [128 x 128 bf16] -> shared memory (128-byte swizzle)
//   MMA 1   Y = X (H D)^T on tcgen05 (bf16, exact +-1 operand) -> TMEM;
//           y = Y / sqrt(128) = R x
//   threads (four per vector, 32 coordinates each) read Y from TMEM: norm,
//           bucketize against the Lloyd-Max boundaries scaled by the norm,
//           sign-magnitude codes packed into the page, fp16 norm; for QJL
//           keys the residual r = y - nhat c[idx], rho = fp16 ||r||, and r
//           (scaled by a power of two) split into fp16 hi + lo -> shared
//   MMA 2   Z = (r_hi + r_lo) S^T on tcgen05 (fp16, S exact in fp16 except
//           |S| < 2^-17) -> TMEM; the sign bits of Z go to the page.
// Key and value tiles alternate so MMA 2 of a key tile overlaps the value
// tile; MMA 1 of the next tile is issued before the current tile's epilogue.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cfloat>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tc05.cuh"
#include "tq_dev.cuh"

namespace tq {

namespace {

constexpr int kRows = 128;
constexpr uint32_t kTile = 32768;          // one 128 x 128 16-bit tile
constexpr uint32_t SM_ROT_K = 0, SM_ROT_V = 32768, SM_S16 = 65536, SM_X = 98304, SM_AHI = 163840,
                   SM_ALO = 196608, SM_XCH = 229376;
constexpr uint32_t SM_BAR = SM_XCH + 2048;
constexpr uint32_t SM_TOTAL = SM_BAR + 256;        // barriers, TMEM address, level tables
constexpr uint32_t kPolls = 1u << 20;    // about a second of polling, then give up

struct Enc128Args {
    Layout L;
    const float *k_lv, *v_lv;          // levels by stored code
    const float *k_bnd, *v_bnd;        // ascending boundaries
    const uint8_t *k_rot, *v_rot, *s16;
    int64_t n_vec, n_tiles;
    const int32_t *slots;
    int64_t num_slots;
    uint8_t *cache;
    uint32_t *status;
};

// Magnitude rank mu = #{k < 2^(B-1) - 1 : a >= T[k]} of the sorted positive
// thresholds, by binary search on the float magnitude a = |Y|.
template <int B>
__device__ __forceinline__ int mag_rank(float a, const float (&T)[7]) {
    if constexpr (B == 1) {
        return 0;
    } else if constexpr (B == 2) {
        return a >= T[0] ? 1 : 0;
    } else if constexpr (B == 3) {
        const int b1 = a >= T[1] ? 1 : 0;
        const int b0 = a >= (b1 ? T[2] : T[0]) ? 1 : 0;
        return (b1 << 1) | b0;
    } else {
        const int b2 = a >= T[3] ? 1 : 0;
        const int b1 = a >= (b2 ? T[5] : T[1]) ? 1 : 0;
        const float t0 = b2 ? (b1 ? T[6] : T[4]) : (b1 ? T[2] : T[0]);
        const int b0 = a >= t0 ? 1 : 0;
        return (b2 << 2) | (b1 << 1) | b0;
    }
}

// Bucketize this thread's 32 coordinates (Y = sqrt(128) y from the rotation
// MMA) into sign-magnitude codes packed into words (B in {1,2,4}: one array
// of B words; B = 3: words 0..1 hold the 2-bit magnitudes, word 2 the sign
// bits).  T: positive boundaries scaled by ||Y||.  -0.0 counts as
// non-negative; a coordinate exactly on a boundary takes the upper magnitude
// whatever its sign.  With RESID, y is overwritten by the residual in the Y
// scale, Y - sqrt(128) nhat c[code], and rr receives its squared norm.
template <int B, bool RESID>
__device__ __forceinline__ void quantize32(float (&y)[32], const float (&T)[7], const float *lvs, float nhs,
                                           uint32_t (&cw)[4], float &rr) {
#pragma unroll
    for (int k = 0; k < 4; ++k) cw[k] = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float Y = y[i];
        const uint32_t s = Y < 0.f ? 1u : 0u;
        const uint32_t kap = (s << (B - 1)) | uint32_t(mag_rank<B>(fabsf(Y), T));
        if constexpr (B == 3) {
            cw[i >> 4] |= (kap & 3u) << (2 * (i & 15));
            cw[2] |= (kap >> 2) << i;
        } else {
            cw[(i * B) >> 5] |= kap << ((i * B) & 31);
        }
        if constexpr (RESID) {
            const float r = fmaf(-nhs, lvs[kap], Y);
            y[i] = r;
            rr = fmaf(r, r, rr);
        }
    }
}

// Stores the codes of this thread's quarter (32 coordinates) of a vector.
template <int B>
__device__ __forceinline__ void store_codes32(uint8_t *page, int pos, int q, int code_off, int code_bpt, int hi_off,
                                              int hi_bpt, const uint32_t (&cw)[4]) {
    uint8_t *dst = page + code_off + pos * code_bpt;
    if constexpr (B == 3) {
        *reinterpret_cast<uint2 *>(dst + q * 8) = make_uint2(cw[0], cw[1]);
        *reinterpret_cast<uint32_t *>(page + hi_off + pos * hi_bpt + q * 4) = cw[2];
    } else if constexpr (B == 4) {
        *reinterpret_cast<uint4 *>(dst + q * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    } else if constexpr (B == 2) {
        *reinterpret_cast<uint2 *>(dst + q * 8) = make_uint2(cw[0], cw[1]);
    } else {
        *reinterpret_cast<uint32_t *>(dst + q * 4) = cw[0];
    }
}

// Page address of vector v (nullptr = nothing to store).
__device__ __forceinline__ uint8_t *row_page(const Enc128Args &a, int64_t v, int *pos) {
    if (v >= a.n_vec) return nullptr;
    const uint32_t vv = uint32_t(v), H = uint32_t(a.L.H);
    const uint32_t t = vv / H, h = vv - t * H;
    const int slot = a.slots[t];
    if (slot < 0) return nullptr;
    if (slot >= a.num_slots) {
        atomicOr(a.status, TQ_DEV_SLOT_RANGE);
        return nullptr;
    }
    const uint32_t blk = uint32_t(slot) / uint32_t(a.L.P);
    *pos = slot - int(blk * uint32_t(a.L.P));
    return a.cache + (int64_t(blk) * a.L.H + h) * int64_t(a.L.page_bytes);
}

// 16 warps: thread (row, q) owns vector row 32*(warp%4)+lane of the tile and
// its coordinates [32q, 32q + 32), q = warp / 4 (TMEM lane slice warp % 4).
template <int KB, int VB, bool QJL>
__global__ void __launch_bounds__(512, 1)
encode128_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Enc128Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = smem_raw;
    float *xr = reinterpret_cast<float *>(sm + SM_XCH);              // [4][128] residual-norm partials
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SM_BAR);
    uint64_t *bar_const = bars, *bar_x = bars + 1, *bar_y = bars + 3, *bar_z = bars + 5;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sm + SM_BAR + 64);
    float *s_klv = reinterpret_cast<float *>(sm + SM_BAR + 128), *s_vlv = s_klv + 16;

    constexpr bool DO_V = VB > 0;
    constexpr int PER = DO_V ? 2 : 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = 32 * (warp & 3) + lane, q = warp >> 2;
    if ((tc05::smem_u32(smem_raw) & 1023u) != 0) {       // the swizzled tiles need 1024-byte alignment
        if (tid == 0) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
        return;
    }
    const int64_t n_pairs = a.n_tiles > blockIdx.x ? (a.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t n_items = n_pairs * PER;
    bool timeout = false;

    if (warp == 0) {
        tc05::tmem_alloc(tmem_holder, 512);
        tc05::tmem_relinquish();
    }
    if (tid < 16) {
        s_klv[tid] = (KB != 8 && tid < (1 << (KB == 8 ? 1 : KB))) ? a.k_lv[tid] : 0.f;
        s_vlv[tid] = (DO_V && tid < (1 << (VB > 0 ? VB : 1))) ? a.v_lv[tid] : 0.f;
    }
    auto item_tile = [&](int64_t j) { return int64_t(blockIdx.x) + (j / PER) * int64_t(gridDim.x); };
    auto item_is_v = [&](int64_t j) { return DO_V && (j % PER) == 1; };
    auto issue_x = [&](int64_t j) {
        const int st = int(j & 1);
        uint8_t *dst = sm + SM_X + st * kTile;
        tc05::mbar_expect_tx(&bar_x[st], kTile);
        const void *tm = item_is_v(j) ? static_cast<const void *>(&tmV) : static_cast<const void *>(&tmK);
        const int y = int(item_tile(j) * kRows);
        tc05::tma_load_2d(dst, tm, 0, y, &bar_x[st]);
        tc05::tma_load_2d(dst + 16384, tm, 64, y, &bar_x[st]);
    };
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) tc05::mbar_init(&bars[i], 1);
        tc05::fence_mbar_init();
        tc05::mbar_expect_tx(bar_const, kTile * (1 + (DO_V ? 1 : 0) + (QJL ? 1 : 0)));
        tc05::bulk_g2s(sm + SM_ROT_K, a.k_rot, kTile, bar_const);
        if (DO_V) tc05::bulk_g2s(sm + SM_ROT_V, a.v_rot, kTile, bar_const);
        if (QJL) tc05::bulk_g2s(sm + SM_S16, a.s16, kTile, bar_const);
        if (n_items > 0) issue_x(0);
        if (n_items > 1) issue_x(1);
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
    constexpr uint32_t idesc1 = tc05::idesc_bf16_f32(128, 128);
    constexpr uint32_t idesc2 = tc05::idesc_f16_f32(128, 128);

    auto issue_mma1 = [&](int64_t j) {
        const int st = int(j & 1);
        if (!tc05::mbar_wait_bounded(&bar_x[st], uint32_t((j >> 1) & 1), kPolls)) timeout = true;
        tc05::fence_after_sync();
        const uint32_t xa = tc05::smem_u32(sm + SM_X + st * kTile);
        const uint32_t rb = tc05::smem_u32(sm + (item_is_v(j) ? SM_ROT_V : SM_ROT_K));
        const uint32_t d = tmem + uint32_t(st * 128);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc05::mma_bf16(d, tc05::desc_kmajor_sw128(xa + c * 16384 + ks * 32),
                               tc05::desc_kmajor_sw128(rb + c * 16384 + ks * 32), idesc1, (c | ks) != 0);
        tc05::mma_commit(&bar_y[st]);
    };

    if (tid == 0 && n_items > 0) {
        if (!tc05::mbar_wait_bounded(bar_const, 0, kPolls)) timeout = true;
        issue_mma1(0);
    }

    const float rs = 0.08838834764831845f;              // 1 / sqrt(128)
    const float sq = 11.313708498984761f;               // sqrt(128)
    int64_t pending_k = -1;                             // key tile whose MMA 2 is in flight
    uint32_t z_phase = 0;

    for (int64_t j = 0; j < n_items; ++j) {
        const bool is_v = item_is_v(j);
        const int64_t tile = item_tile(j);
        const int yb = int(j & 1);
        if (tid == 0 && j + 1 < n_items) issue_mma1(j + 1);
        if (!tc05::mbar_wait_bounded(&bar_y[yb], uint32_t((j >> 1) & 1), kPolls)) timeout = true;
        tc05::fence_after_sync();
        // MMA 1 of this item has read its x stage: refill it
        if (tid == 0 && j + 2 < n_items) issue_x(j + 2);

        // this thread's quarter of Y, and ||Y||^2 summed over the four
        // quarters in a fixed order, so the four threads of a row agree
        float y[32];
        {
            uint32_t r[32];
            tc05::tmem_ld_32x32b_x32(tmem + lane_base + uint32_t(yb * 128 + q * 32), r);
            tc05::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(r[i]);
        }
        float part[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float ps = 0.f;
            if (c == q) {
#pragma unroll
                for (int i = 0; i < 32; ++i) ps = fmaf(y[i], y[i], ps);
            } else {
                uint32_t r[32];
                tc05::tmem_ld_32x32b_x32(tmem + lane_base + uint32_t(yb * 128 + c * 32), r);
                tc05::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) ps = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ps);
            }
            part[c] = ps;
        }
        const float ns = sqrtf(((part[0] + part[1]) + part[2]) + part[3]);   // ||Y|| = sqrt(128) ||x||
        const float n = ns * rs;                                               // ||x||
        const uint16_t nh = f2h_bits(n);
        const float nhf = h2f_bits(nh);
        int pos = 0;
        uint8_t *page = row_page(a, tile * kRows + row, &pos);
        const int bits = is_v ? VB : KB;
        float rr = 0.f;

        if (!is_v && KB == 8) {
            // FP8 keys: e4m3(sqrt(d) y / n) = e4m3(Y / n)
            const float inv = n > 0.f ? 1.0f / n : 0.f;
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint32_t acc = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc |= uint32_t(__nv_cvt_float_to_fp8(y[4 * k + e] * inv, __NV_SATFINITE, __NV_E4M3)) << (8 * e);
                w[k] = acc;
            }
            if (page) {
                uint4 *dst = reinterpret_cast<uint4 *>(page + a.L.kc_off + pos * a.L.kc_bpt + q * 32);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                if (q == 0) *reinterpret_cast<uint16_t *>(page + a.L.kn_off + pos * 2) = nh;
            }
        } else {
            const int nt = (1 << (bits - 1)) - 1;
            const float *bnd = is_v ? a.v_bnd : a.k_bnd;
            float T[7];
#pragma unroll
            for (int k = 0; k < 7; ++k) T[k] = (k < nt && ns > 0.f) ? bnd[(1 << (bits - 1)) + k] * ns : FLT_MAX;
            uint32_t cw[4];
            if (is_v) {
                if constexpr (DO_V) {
                    quantize32<DO_V ? VB : 1, false>(y, T, s_vlv, 0.f, cw, rr);
                    if (page) store_codes32<DO_V ? VB : 1>(page, pos, q, a.L.vc_off, a.L.vc_bpt, a.L.vh_off,
                                                            a.L.vh_bpt, cw);
                }
            } else {
                constexpr int KQ = KB == 8 ? 1 : KB;
                quantize32<KQ, QJL>(y, T, s_klv, sq * nhf, cw, rr);
                if (page) store_codes32<KQ>(page, pos, q, a.L.kc_off, a.L.kc_bpt, a.L.kh_off, a.L.kh_bpt, cw);
            }
            if (page && q == 0)
                *reinterpret_cast<uint16_t *>(page + (is_v ? a.L.vn_off : a.L.kn_off) + pos * 2) = nh;
        }

        if (!is_v && QJL) {
            // the residual (Y scale) times 2^(12 - e), ||Y|| < 2^(e + 1), so
            // |.| < 2^14, split into fp16 hi + lo; the signs of S r do not
            // depend on the positive scale
            int e = 0;
            if (ns > 0.f) e = ((__float_as_int(ns) >> 23) & 0xff) - 127;
            const int ebits = min(254, max(1, 127 + 12 - e));
            const float sc = __int_as_float(ebits << 23);
            const int c = q >> 1;                          // 64-column half of the operand tile
            uint8_t *ahi = sm + SM_AHI + c * 16384, *alo = sm + SM_ALO + c * 16384;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint32_t wh[4], wl[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float a0 = y[p * 8 + 2 * k] * sc, a1 = y[p * 8 + 2 * k + 1] * sc;
                    const __half2 h = __floats2half2_rn(a0, a1);
                    const float2 hf = __half22float2(h);
                    const __half2 l = __floats2half2_rn(a0 - hf.x, a1 - hf.y);
                    wh[k] = *reinterpret_cast<const uint32_t *>(&h);
                    wl[k] = *reinterpret_cast<const uint32_t *>(&l);
                }
                const uint32_t off = tc05::sw128_offset(uint32_t(row), uint32_t((q & 1) * 4 + p));
                *reinterpret_cast<uint4 *>(ahi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                *reinterpret_cast<uint4 *>(alo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            }
            xr[q * 128 + row] = rr;
            tc05::fence_proxy_async_smem();
            tc05::fence_before_sync();
            __syncthreads();
            if (tid == 0) {
                tc05::fence_after_sync();
                const uint32_t bh = tc05::smem_u32(sm + SM_AHI), bl = tc05::smem_u32(sm + SM_ALO);
                const uint32_t bs = tc05::smem_u32(sm + SM_S16);
                const uint32_t d = tmem + 256u;
#pragma unroll
                for (int sp = 0; sp < 2; ++sp)
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc05::mma_f16(d, tc05::desc_kmajor_sw128((sp ? bl : bh) + cc * 16384 + ks * 32),
                                          tc05::desc_kmajor_sw128(bs + cc * 16384 + ks * 32), idesc2,
                                          (sp | cc | ks) != 0);
                tc05::mma_commit(bar_z);
            }
            if (page && q == 0) {
                // rho = ||r|| = ||Y-scale residual|| / sqrt(128)
                const float rho = sqrtf(((xr[row] + xr[128 + row]) + xr[256 + row]) + xr[384 + row]) * rs;
                *reinterpret_cast<uint16_t *>(page + a.L.kr_off + pos * 2) = f2h_bits(rho);
            }
            pending_k = tile;
        }

        // sign bits of the key tile whose MMA 2 is in flight
        if (QJL && pending_k >= 0 && (is_v || !DO_V)) {
            if (!tc05::mbar_wait_bounded(bar_z, z_phase, kPolls)) timeout = true;
            z_phase ^= 1u;
            tc05::fence_after_sync();
            int kpos = 0;
            uint8_t *kpage = row_page(a, pending_k * kRows + row, &kpos);
            uint32_t r[32];
            tc05::tmem_ld_32x32b_x32(tmem + lane_base + uint32_t(256 + q * 32), r);
            tc05::tmem_wait_ld();
            // bit k = [z_k >= 0]: the complement of the float sign bit (z = -0.0
            // lies inside the zero-tolerance of the sign comparison)
            uint32_t neg = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) neg |= (r[k] >> (31 - k)) & (1u << k);
            if (kpage && !timeout)
                *reinterpret_cast<uint32_t *>(kpage + a.L.ks_off + kpos * a.L.ks_bpt + q * 4) = ~neg;
            pending_k = -1;
        }
        tc05::fence_before_sync();
        __syncthreads();
    }

    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, 512);
    }
    if (timeout) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D map over [rows][128] bf16, boxes of 64 columns x 128 rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int64_t rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {128, cuuint64_t(rows)};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KB, int VB, bool QJL>
int run(const CUtensorMap &mk, const CUtensorMap &mv, const Enc128Args &a, cudaStream_t st) {
    auto kern = encode128_kernel<KB, VB, QJL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SM_TOTAL));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = a.n_tiles < sms ? a.n_tiles : sms;
    kern<<<unsigned(grid), 512, SM_TOTAL, st>>>(mk, mv, a);
    return cudaGetLastError();
}

}  // namespace

// Returns -1 if this configuration is not handled by the fused kernel.
int launch_encode128(const tq_params *kp, const tq_params *vp, const Layout &L, const void *K, const void *V,
                     int64_t n_tokens, const int32_t *slots, uint8_t *cache, int64_t num_blocks, uint8_t *ws,
                     void *stream) {
    if (L.d != 128 || !kp->dev.rot_img) return -1;
    if (L.vbits > 0 && (!vp || !vp->dev.rot_img)) return -1;
    const int kb = L.kbits, vb = L.vbits, q = L.kqjl;
    Enc128Args a;
    a.L = L;
    a.k_lv = kp->dev.lv;
    a.k_bnd = kp->dev.bounds;
    a.k_rot = kp->dev.rot_img;
    a.s16 = kp->dev.s16_img;
    a.v_lv = vp ? vp->dev.lv : nullptr;
    a.v_bnd = vp ? vp->dev.bounds : nullptr;
    a.v_rot = vp ? vp->dev.rot_img : nullptr;
    a.n_vec = n_tokens * L.H;
    a.n_tiles = (a.n_vec + kRows - 1) / kRows;
    a.slots = slots;
    a.num_slots = num_blocks * L.P;
    a.cache = cache;
    a.status = reinterpret_cast<uint32_t *>(ws);
    CUtensorMap mk, mv;
    if (!make_map(&mk, K, a.n_vec)) return -1;
    if (vb > 0) {
        if (!make_map(&mv, V, a.n_vec)) return -1;
    } else {
        mv = mk;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (q) {
        if (kb == 4 && vb == 4) return run<4, 4, true>(mk, mv, a, st);
        if (kb == 2 && vb == 4) return run<2, 4, true>(mk, mv, a, st);
        if (kb == 2 && vb == 3) return run<2, 3, true>(mk, mv, a, st);
        if (kb == 3 && vb == 3) return run<3, 3, true>(mk, mv, a, st);
        if (kb == 3 && vb == 4) return run<3, 4, true>(mk, mv, a, st);
        if (kb == 4 && vb == 0) return run<4, 0, true>(mk, mv, a, st);
    } else {
        if (kb == 8 && vb == 4) return run<8, 4, false>(mk, mv, a, st);
        if (kb == 4 && vb == 4) return run<4, 4, false>(mk, mv, a, st);
        if (kb == 3 && vb == 3) return run<3, 3, false>(mk, mv, a, st);
    }
    return -1;
}

}  // namespace tq
