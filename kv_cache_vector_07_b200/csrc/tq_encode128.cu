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
//   threads (two per vector, 64 coordinates each) read Y from TMEM: norm,
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
constexpr uint32_t SM_BAR = SM_XCH + 1024;
constexpr uint32_t SM_TOTAL = SM_BAR + 64 + 1024;   // + alignment slack
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

// Packs W-bit fields of n consecutive coordinates into words.
template <int W, int N>
__device__ __forceinline__ void pack_fields_n(const uint32_t (&v)[N], uint32_t (&w)[N * W / 32]) {
    constexpr int PER = 32 / W;
#pragma unroll
    for (int k = 0; k < N * W / 32; ++k) {
        uint32_t acc = 0;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc |= v[k * PER + e] << (e * W);
        w[k] = acc;
    }
}

template <int NW>
__device__ __forceinline__ void store_words(uint8_t *dst, const uint32_t (&w)[NW]) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int k = 0; k < NW; k += 4) reinterpret_cast<uint4 *>(dst)[k / 4] = make_uint4(w[k], w[k + 1], w[k + 2], w[k + 3]);
    } else if constexpr (NW % 2 == 0) {
#pragma unroll
        for (int k = 0; k < NW; k += 2) reinterpret_cast<uint2 *>(dst)[k / 2] = make_uint2(w[k], w[k + 1]);
    } else {
#pragma unroll
        for (int k = 0; k < NW; ++k) reinterpret_cast<uint32_t *>(dst)[k] = w[k];
    }
}

// Bucketize this thread's 64 coordinates (Y = sqrt(128) y from the rotation
// MMA) into sign-magnitude codes packed into words (B in {1,2,4}: one
// array; B = 3: words 0..3 hold the 2-bit magnitudes, words 4..5 the sign
// bits).  T: positive boundaries scaled by sqrt(128) n, as float bits.  With
// RESID, y is overwritten by the residual y - nhat c[code] and rr receives
// its squared norm.
template <int B, bool RESID>
__device__ __forceinline__ void quantize64(float (&y)[64], const int (&T)[7], const float *lvs, float nhf, float rs,
                                           uint32_t (&cw)[8], float &rr) {
    constexpr int NT = (1 << (B - 1)) - 1;
#pragma unroll
    for (int k = 0; k < 8; ++k) cw[k] = 0;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float Y = y[i];
        const int s = Y < 0.f ? 1 : 0;          // -0.0 counts as non-negative
        const int aa = (__float_as_int(Y) & 0x7fffffff) - s;
        int mu = 0;
#pragma unroll
        for (int k = 0; k < NT; ++k) mu += aa >= T[k] ? 1 : 0;
        const uint32_t kap = uint32_t((s << (B - 1)) | mu);
        if constexpr (B == 3) {
            cw[i >> 4] |= (kap & 3u) << (2 * (i & 15));
            cw[4 + (i >> 5)] |= (kap >> 2) << (i & 31);
        } else {
            cw[(i * B) >> 5] |= kap << ((i * B) & 31);
        }
        if constexpr (RESID) {
            const float r = fmaf(-nhf, lvs[kap], Y * rs);
            y[i] = r;
            rr = fmaf(r, r, rr);
        }
    }
}

template <int B>
__device__ __forceinline__ void store_codes64(uint8_t *page, int pos, int half, int code_off, int code_bpt, int hi_off,
                                              int hi_bpt, const uint32_t (&cw)[8]) {
    if constexpr (B == 3) {
        const uint32_t lo[4] = {cw[0], cw[1], cw[2], cw[3]};
        const uint32_t hb[2] = {cw[4], cw[5]};
        store_words<4>(page + code_off + pos * code_bpt + half * 16, lo);
        store_words<2>(page + hi_off + pos * hi_bpt + half * 8, hb);
    } else {
        uint32_t w[2 * B];
#pragma unroll
        for (int k = 0; k < 2 * B; ++k) w[k] = cw[k];
        store_words<2 * B>(page + code_off + pos * code_bpt + half * (8 * B), w);
    }
}

// Row context: page address of vector v of the tile (nullptr = no store).
__device__ __forceinline__ uint8_t *row_page(const Enc128Args &a, int64_t v, int *pos) {
    if (v >= a.n_vec) return nullptr;
    const int64_t t = v / a.L.H;
    const int h = int(v - t * a.L.H);
    const int slot = a.slots[t];
    if (slot < 0) return nullptr;
    if (slot >= a.num_slots) {
        atomicOr(a.status, TQ_DEV_SLOT_RANGE);
        return nullptr;
    }
    *pos = slot % a.L.P;
    return a.cache + (int64_t(slot / a.L.P) * a.L.H + h) * int64_t(a.L.page_bytes);
}

template <int KB, int VB, bool QJL>
__global__ void __launch_bounds__(256, 1)
encode128_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Enc128Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *xch = reinterpret_cast<float *>(sm + SM_XCH);       // [2 halves][128 rows] x 2 quantities
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SM_BAR);
    uint64_t *bar_const = bars, *bar_x = bars + 1, *bar_y = bars + 3, *bar_z = bars + 5;
    __shared__ uint32_t tmem_holder;
    __shared__ float s_klv[16], s_vlv[16];

    constexpr bool DO_V = VB > 0;
    constexpr int PER = DO_V ? 2 : 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = 32 * (warp & 3) + lane, half = warp >> 2;
    const int64_t n_pairs = a.n_tiles > blockIdx.x ? (a.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t n_items = n_pairs * PER;
    bool timeout = false;

    if (warp == 0) {
        tc05::tmem_alloc(&tmem_holder, 512);
        tc05::tmem_relinquish();
    }
    if (tid < 16) {
        s_klv[tid] = (KB != 8 && tid < (1 << (KB == 8 ? 1 : KB))) ? a.k_lv[tid] : 0.f;
        s_vlv[tid] = (DO_V && tid < (1 << (VB > 0 ? VB : 1))) ? a.v_lv[tid] : 0.f;
    }
    auto item_tile = [&](int64_t j) { return int64_t(blockIdx.x) + (j / PER) * int64_t(gridDim.x); };
    auto item_is_v = [&](int64_t j) { return DO_V && (j % PER) == 1; };
    auto issue_x = [&](int64_t j) {
        const int s = int(j & 1);
        uint8_t *dst = sm + SM_X + s * kTile;
        tc05::mbar_expect_tx(&bar_x[s], kTile);
        const void *tm = item_is_v(j) ? static_cast<const void *>(&tmV) : static_cast<const void *>(&tmK);
        const int y = int(item_tile(j) * kRows);
        tc05::tma_load_2d(dst, tm, 0, y, &bar_x[s]);
        tc05::tma_load_2d(dst + 16384, tm, 64, y, &bar_x[s]);
    };
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) tc05::mbar_init(&bars[i], 1);
        tc05::fence_mbar_init();
        uint32_t cbytes = kTile;
        tc05::mbar_expect_tx(bar_const, kTile * (1 + (DO_V ? 1 : 0) + (QJL ? 1 : 0)));
        tc05::bulk_g2s(sm + SM_ROT_K, a.k_rot, kTile, bar_const);
        if (DO_V) tc05::bulk_g2s(sm + SM_ROT_V, a.v_rot, kTile, bar_const);
        if (QJL) tc05::bulk_g2s(sm + SM_S16, a.s16, kTile, bar_const);
        (void)cbytes;
        if (n_items > 0) issue_x(0);
        if (n_items > 1) issue_x(1);
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = tmem_holder;
    const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
    constexpr uint32_t idesc1 = tc05::idesc_bf16_f32(128, 128);
    constexpr uint32_t idesc2 = tc05::idesc_f16_f32(128, 128);

    auto issue_mma1 = [&](int64_t j) {
        const int s = int(j & 1);
        if (!tc05::mbar_wait_bounded(&bar_x[s], uint32_t((j >> 1) & 1), kPolls)) timeout = true;
        tc05::fence_after_sync();
        const uint32_t xa = tc05::smem_u32(sm + SM_X + s * kTile);
        const uint32_t rb = tc05::smem_u32(sm + (item_is_v(j) ? SM_ROT_V : SM_ROT_K));
        const uint32_t d = tmem + uint32_t(s * 128);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc05::mma_bf16(d, tc05::desc_kmajor_sw128(xa + c * 16384 + ks * 32),
                               tc05::desc_kmajor_sw128(rb + c * 16384 + ks * 32), idesc1, (c | ks) != 0);
        tc05::mma_commit(&bar_y[s]);
    };

    if (tid == 0 && n_items > 0) {
        if (!tc05::mbar_wait_bounded(bar_const, 0, kPolls)) timeout = true;
        issue_mma1(0);
    }

    const float rs = 0.08838834764831845f;              // 1 / sqrt(128)
    const float sq = 11.313708498984761f;               // sqrt(128)
    int64_t pending_k = -1;                             // tile whose MMA 2 is in flight
    uint32_t z_phase = 0;

    for (int64_t j = 0; j < n_items; ++j) {
        const bool is_v = item_is_v(j);
        const int64_t tile = item_tile(j);
        const int yb = int(j & 1);
        if (tid == 0 && j + 1 < n_items) issue_mma1(j + 1);
        if (!tc05::mbar_wait_bounded(&bar_y[yb], uint32_t((j >> 1) & 1), kPolls)) timeout = true;
        if (tid == 0 && j + 2 < n_items) issue_x(j + 2);
        tc05::fence_after_sync();

        // ---- epilogue 1: thread (row, half) owns coordinates [64 half, 64 half + 64)
        float y[64];
        {
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                tc05::tmem_ld_32x32b_x32(tmem + lane_base + uint32_t(yb * 128 + half * 64 + c * 32), r);
                tc05::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) y[c * 32 + i] = __uint_as_float(r[i]);
            }
        }
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) ss = fmaf(y[i], y[i], ss);
        xch[half * 128 + row] = ss;
        __syncthreads();
        const float n = sqrtf(xch[row] + xch[128 + row]) * rs;      // ||y|| = ||x||
        const uint16_t nh = f2h_bits(n);
        const float nhf = h2f_bits(nh);
        int pos = 0;
        uint8_t *page = row_page(a, tile * kRows + row, &pos);
        const int bits = is_v ? VB : KB;
        const float *lvs = is_v ? s_vlv : s_klv;
        const float *bnd = is_v ? a.v_bnd : a.k_bnd;
        float rr = 0.f;

        if (!is_v && KB == 8) {
            // FP8 keys: e4m3(sqrt(d) y / n) = e4m3(Y / n)
            const float inv = n > 0.f ? 1.0f / n : 0.f;
            uint32_t f[64];
#pragma unroll
            for (int i = 0; i < 64; ++i)
                f[i] = uint32_t(__nv_cvt_float_to_fp8(y[i] * inv, __NV_SATFINITE, __NV_E4M3));
            if (page) {
                uint32_t w[16];
                pack_fields_n<8, 64>(f, w);
                store_words<16>(page + a.L.kc_off + pos * a.L.kc_bpt + half * 64, w);
                if (half == 0) *reinterpret_cast<uint16_t *>(page + a.L.kn_off + pos * 2) = nh;
            }
        } else {
            // thresholds for |Y|: positive boundaries t' scaled by sqrt(128) n,
            // compared as integers (non-negative floats order like their bits);
            // a negative coordinate equal to a boundary belongs to the lower
            // bucket, hence the "- s" in quantize64.  A zero vector has u = 0.
            const int nt = (1 << (bits - 1)) - 1;
            const float scale = sq * n;
            int T[7];
#pragma unroll
            for (int k = 0; k < 7; ++k)
                T[k] = (k < nt && n > 0.f) ? __float_as_int(bnd[(1 << (bits - 1)) + k] * scale) : 0x7f7fffff;
            uint32_t cw[8];
            if (is_v) {
                if constexpr (DO_V) {
                    quantize64<DO_V ? VB : 1, false>(y, T, lvs, nhf, rs, cw, rr);
                    if (page) store_codes64<DO_V ? VB : 1>(page, pos, half, a.L.vc_off, a.L.vc_bpt, a.L.vh_off,
                                                            a.L.vh_bpt, cw);
                }
            } else {
                constexpr int KQ = KB == 8 ? 1 : KB;
                quantize64<KQ, QJL>(y, T, lvs, nhf, rs, cw, rr);
                if (page) store_codes64<KQ>(page, pos, half, a.L.kc_off, a.L.kc_bpt, a.L.kh_off, a.L.kh_bpt, cw);
            }
            if (page && half == 0)
                *reinterpret_cast<uint16_t *>(page + (is_v ? a.L.vn_off : a.L.kn_off) + pos * 2) = nh;
        }

        if (!is_v && QJL) {
            // rho, then r scaled by 2^k (so |r| < 2^14) split into fp16 hi + lo
            __syncthreads();                       // everyone has read the norm partials
            xch[half * 128 + row] = rr;
            __syncthreads();
            const float rho = sqrtf(xch[row] + xch[128 + row]);
            if (page && half == 0) *reinterpret_cast<uint16_t *>(page + a.L.kr_off + pos * 2) = f2h_bits(rho);
            int e = 0;
            if (rho > 0.f) e = ((__float_as_int(rho) >> 23) & 0xff) - 127;
            const int ebits = min(254, max(1, 127 + 13 - e));
            const float sc = __int_as_float(ebits << 23);
            uint8_t *ahi = sm + SM_AHI + half * 16384, *alo = sm + SM_ALO + half * 16384;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                uint32_t wh[4], wl[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a0 = y[p * 8 + 2 * q] * sc, a1 = y[p * 8 + 2 * q + 1] * sc;
                    const __half2 h = __floats2half2_rn(a0, a1);
                    const float2 hf = __half22float2(h);
                    const __half2 l = __floats2half2_rn(a0 - hf.x, a1 - hf.y);
                    wh[q] = *reinterpret_cast<const uint32_t *>(&h);
                    wl[q] = *reinterpret_cast<const uint32_t *>(&l);
                }
                const uint32_t off = tc05::sw128_offset(uint32_t(row), uint32_t(p));
                *reinterpret_cast<uint4 *>(ahi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                *reinterpret_cast<uint4 *>(alo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            }
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
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc05::mma_f16(d, tc05::desc_kmajor_sw128((sp ? bl : bh) + c * 16384 + ks * 32),
                                          tc05::desc_kmajor_sw128(bs + c * 16384 + ks * 32), idesc2,
                                          (sp | c | ks) != 0);
                tc05::mma_commit(bar_z);
            }
            pending_k = tile;
        }

        // ---- epilogue 2: sign bits of the key tile whose MMA 2 is in flight
        if (QJL && pending_k >= 0 && (is_v || !DO_V)) {
            if (!tc05::mbar_wait_bounded(bar_z, z_phase, kPolls)) timeout = true;
            z_phase ^= 1u;
            tc05::fence_after_sync();
            int kpos = 0;
            uint8_t *kpage = row_page(a, pending_k * kRows + row, &kpos);
            uint32_t r[32], wd[2];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                tc05::tmem_ld_32x32b_x32(tmem + lane_base + uint32_t(256 + half * 64 + c * 32), r);
                tc05::tmem_wait_ld();
                uint32_t b = 0;
#pragma unroll
                for (int k = 0; k < 32; ++k) b |= (__uint_as_float(r[k]) >= 0.f ? 1u : 0u) << k;
                wd[c] = b;
            }
            if (kpage && !timeout)
                *reinterpret_cast<uint2 *>(kpage + a.L.ks_off + kpos * a.L.ks_bpt + half * 8) = make_uint2(wd[0], wd[1]);
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
    kern<<<unsigned(grid), 256, SM_TOTAL, st>>>(mk, mv, a);
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
