// Chunked prefill attention over the compressed cache on the tensor cores:
// head dimension 128, pages of 64 tokens, keys b-bit Lloyd-Max + QJL
// (b in {2, 3, 4}), values b-bit (b in {2, 3, 4}).
//
// Page "What is TurboQuant?", "Stage 1"/"Stage 2" and the ai-work-lab
// overview, "QJL": the logit of key t is
//   ( nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1> ) / sqrt(d),
// then softmax and the sum of dequantized values nhat_v c_v[code] (rotated
// back by the combine kernel).  A block takes 128 query rows (positions x
// GQA heads of one KV head) and walks one key split a page at a time:
//   dequantize   all 256 threads: centroids of the page's 64 keys as fp16
//                hi + lo tiles, the QJL signs as a +-1 tile, per-key scales;
//   MMA  QK      S_mse = q_hi C_hi + q_lo C_hi + q_hi C_lo and
//                S_qjl = w_hi Sigma + w_lo Sigma on tcgen05 (TMEM
//                accumulators): the hi/lo splits keep both terms at
//                fp32-level accuracy, which large logits need;
//   softmax      one thread per row (TMEM lane): logits, causal mask, online
//                max / sum, P' = p nhat_v as fp16 hi + lo into shared memory
//                (lo over the C_lo tile, dead once QK completed), O rescaled
//                in TMEM when the row maximum grows;
//                meanwhile warps 4-7 dequantize the values as fp16 hi + lo
//                tiles (MN-major; lo over the C_hi tile);
//   MMA  PV      O += P'_hi V_hi + P'_lo V_hi + P'_hi V_lo on tcgen05: with
//                outlier value channels, fp16 weights or fp16 centroids alone
//                move outputs by more than the output tolerance.
// The split's partial (O, max, sum) goes to the workspace in the layout the
// log-sum-exp combine kernel reads.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tc05.cuh"
#include "tq_dev.cuh"

namespace tq {
namespace {

constexpr int kKeys = 64;               // keys per tile (one page)
constexpr uint32_t kPolls = 1u << 20;   // about a second of polling, then give up

// shared layout (offsets from a 1024-aligned base)
constexpr uint32_t SQH = 0, SQL = 32768, SQW = 65536, SQWL = 98304;   // [128 x 128] fp16, K-major, halves at +16 KB
constexpr uint32_t SKH = 131072, SKL = SKH + 16384, SKS = SKL + 16384;  // [64 x 128], halves at +8 KB
constexpr uint32_t SV = SKS + 16384;                              // [64 keys x 128 dims], MN-major (V_hi; V_lo at SKH)
constexpr uint32_t SP = SV + 16384;                               // [128 x 64] fp16, K-major (P'_hi; P'_lo at SKL)
constexpr uint32_t SKLUT = SP + 16384;                            // K pair table, <= 8 KB
constexpr uint32_t SVLUT = SKLUT + 8192;                          // V pair table, <= 8 KB
constexpr uint32_t SMETA = SVLUT + 8192;                          // float4 [64]: a, b, nhat_v, 0
constexpr uint32_t SBAR = SMETA + 1024;
constexpr uint32_t SM_TOTAL = SBAR + 64 + 1024;
static_assert(SM_TOTAL <= 232448, "shared memory");

struct Pf128Args {
    Layout L;
    const float *qr, *w;          // [C * Hq][128]
    int C, Hq, G, PT, base_len;   // PT = 128 / G positions per block
    const int32_t *block_table;
    int max_blocks;
    const uint8_t *cache;
    int64_t num_blocks;
    const float *k_lv, *v_lv;     // levels by stored code
    int n_splits, split_len;
    float *part_o, *part_ml;
    uint32_t *status;
};

// Pair tables: entry e holds the two coordinates' values for the pair index
// e built from the packed fields (low field bits of the two coordinates,
// then for 3-bit codes their two sign bits at bits 4..5).  Each entry is
// repeated for several lanes (lane l reads copy l mod copies) to spread
// shared-memory banks; both tables hold fp16 hi + lo pairs (8 bytes an
// entry) in 8 KB.
template <int B>
__host__ __device__ constexpr int pair_entries() { return 1 << (2 * B); }
template <int B, int BYTES, int BUDGET>
__host__ __device__ constexpr int pair_copies() {
    return BUDGET / (pair_entries<B>() * BYTES) < 32 ? BUDGET / (pair_entries<B>() * BYTES) : 32;
}

template <int B>
__device__ __forceinline__ void pair_codes(int e, int &k0, int &k1) {
    if constexpr (B == 3) {
        k0 = (e & 3) | (((e >> 4) & 1) << 2);
        k1 = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
    } else {
        k0 = e & ((1 << B) - 1);
        k1 = e >> B;
    }
}

// Pair index of pair p (coordinates 2p, 2p + 1 of this thread's 32) from the
// low-field words lo[] and, for 3-bit codes, the sign-bit word hi.
template <int B>
__device__ __forceinline__ uint32_t pair_index(const uint32_t (&lo)[4], uint32_t hi, int p) {
    if constexpr (B == 4) {
        return (lo[p >> 2] >> (8 * (p & 3))) & 0xFFu;
    } else {
        const uint32_t nib = (lo[p >> 3] >> (4 * (p & 7))) & 0xFu;
        if constexpr (B == 3) return nib | (((hi >> (2 * p)) & 3u) << 4);
        return nib;
    }
}

// This thread's 32 coordinates of a b-bit field group: low-field words and
// the 3-bit sign word.
template <int B>
__device__ __forceinline__ void load_codes(const uint8_t *lo_arr, int lo_bpt, const uint8_t *hi_arr, int hi_bpt,
                                           int pos, int qq, uint32_t (&lo)[4], uint32_t &hi) {
    if constexpr (B == 4) {
        const uint4 v = *reinterpret_cast<const uint4 *>(lo_arr + pos * lo_bpt + qq * 16);
        lo[0] = v.x; lo[1] = v.y; lo[2] = v.z; lo[3] = v.w;
        hi = 0;
    } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(lo_arr + pos * lo_bpt + qq * 8);
        lo[0] = v.x; lo[1] = v.y; lo[2] = lo[3] = 0;
        hi = 0;
        if constexpr (B == 3) hi = *reinterpret_cast<const uint32_t *>(hi_arr + pos * hi_bpt + qq * 4);
    }
}

__device__ __forceinline__ uint32_t h2u(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int KB, int VB>
__global__ void __launch_bounds__(256, 1) pf128_kernel(Pf128Args a) {
    constexpr int NCK = pair_copies<KB, 8, 8192>(), NCV = pair_copies<VB, 8, 8192>();
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_holder;
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint2 *lutk = reinterpret_cast<uint2 *>(sm + SKLUT);
    uint2 *lutv = reinterpret_cast<uint2 *>(sm + SVLUT);
    float4 *meta = reinterpret_cast<float4 *>(sm + SMETA);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SBAR);
    uint64_t *bar_qk = bars, *bar_pv = bars + 1;

    const Layout &L = a.L;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x, kvh = blockIdx.y, split = blockIdx.z;
    const int G = a.G;
    const int j_lo = qt * a.PT;
    const int j_hi = min(a.C, j_lo + a.PT);
    const int vis_max = a.base_len + j_hi;                 // keys the tile's last row sees
    const int k_begin = split * a.split_len;
    const int k_end = min(k_begin + a.split_len, vis_max);
    // row of this thread (warps 0-3 own the 128 TMEM lanes)
    const int r = tid & 127;
    const int jr = j_lo + r / G, hr = r - (r / G) * G;
    const bool row_ok = jr < a.C;
    const int vis_r = row_ok ? a.base_len + jr + 1 : 0;
    const int64_t pbase = ((int64_t(jr) * L.H + kvh) * a.n_splits + split) * G + hr;

    if (k_begin >= k_end) {                                // nothing visible in this split
        if (tid < 128 && row_ok) {
            a.part_ml[pbase * 2] = -INFINITY;
            a.part_ml[pbase * 2 + 1] = 0.f;
        }
        return;
    }

    // ---- tables
    for (int i = tid; i < pair_entries<KB>() * NCK; i += 256) {
        int k0, k1;
        pair_codes<KB>(i / NCK, k0, k1);
        const float c0 = a.k_lv[k0], c1 = a.k_lv[k1];
        const __half2 h = __floats2half2_rn(c0, c1);
        const float2 hf = __half22float2(h);
        lutk[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&h), h2u(c0 - hf.x, c1 - hf.y));
    }
    for (int i = tid; i < pair_entries<VB>() * NCV; i += 256) {
        int k0, k1;
        pair_codes<VB>(i / NCV, k0, k1);
        const float c0 = a.v_lv[k0], c1 = a.v_lv[k1];
        const __half2 h = __floats2half2_rn(c0, c1);
        const float2 hf = __half22float2(h);
        lutv[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&h), h2u(c0 - hf.x, c1 - hf.y));
    }
    // ---- query tiles: row r = 2^-e [q_r hi | q_r lo | w hi | w lo], 1 <= max |.| < 2
    float qs = 1.f;                                        // 2^e
    if (tid < 128) {
        const float *qp = a.qr + (int64_t(jr) * a.Hq + int64_t(kvh) * G + hr) * 128;
        const float *wp = a.w + (int64_t(jr) * a.Hq + int64_t(kvh) * G + hr) * 128;
        float mx = 0.f;
        if (row_ok)
            for (int i = 0; i < 128; i += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(qp + i);
                const float4 y = *reinterpret_cast<const float4 *>(wp + i);
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(y.x), fabsf(y.y)), fmaxf(fabsf(y.z), fabsf(y.w))));
            }
        int ex = 0;
        if (mx > 0.f) frexpf(mx, &ex);
        const float down = mx > 0.f ? ldexpf(1.f, 1 - ex) : 1.f;
        qs = mx > 0.f ? ldexpf(1.f, ex - 1) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
            float x[8], y[8];
            if (row_ok) {
                const float4 x0 = *reinterpret_cast<const float4 *>(qp + 8 * c);
                const float4 x1 = *reinterpret_cast<const float4 *>(qp + 8 * c + 4);
                const float4 y0 = *reinterpret_cast<const float4 *>(wp + 8 * c);
                const float4 y1 = *reinterpret_cast<const float4 *>(wp + 8 * c + 4);
                x[0] = x0.x; x[1] = x0.y; x[2] = x0.z; x[3] = x0.w; x[4] = x1.x; x[5] = x1.y; x[6] = x1.z; x[7] = x1.w;
                y[0] = y0.x; y[1] = y0.y; y[2] = y0.z; y[3] = y0.w; y[4] = y1.x; y[5] = y1.y; y[6] = y1.z; y[7] = y1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = y[e] = 0.f;
            }
            uint32_t wh[4], wl[4], ww[4], wwl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a0 = x[2 * e] * down, a1 = x[2 * e + 1] * down;
                const __half2 h = __floats2half2_rn(a0, a1);
                const float2 hf = __half22float2(h);
                wh[e] = *reinterpret_cast<const uint32_t *>(&h);
                wl[e] = h2u(a0 - hf.x, a1 - hf.y);
                const float b0 = y[2 * e] * down, b1 = y[2 * e + 1] * down;
                const __half2 g = __floats2half2_rn(b0, b1);
                const float2 gf = __half22float2(g);
                ww[e] = *reinterpret_cast<const uint32_t *>(&g);
                wwl[e] = h2u(b0 - gf.x, b1 - gf.y);
            }
            const uint32_t off = uint32_t(c >> 3) * 16384u + tc05::sw128_offset(uint32_t(r), uint32_t(c & 7));
            *reinterpret_cast<uint4 *>(sm + SQH + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
            *reinterpret_cast<uint4 *>(sm + SQL + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            *reinterpret_cast<uint4 *>(sm + SQW + off) = make_uint4(ww[0], ww[1], ww[2], ww[3]);
            *reinterpret_cast<uint4 *>(sm + SQWL + off) = make_uint4(wwl[0], wwl[1], wwl[2], wwl[3]);
        }
    }
    if (warp == 0) {
        tc05::tmem_alloc(&tmem_holder, 256);
        tc05::tmem_relinquish();
    }
    if (tid == 0) {
        tc05::mbar_init(bar_qk, 1);
        tc05::mbar_init(bar_pv, 1);
        tc05::fence_mbar_init();
    }
    tc05::fence_proxy_async_smem();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = tmem_holder;
    const uint32_t t_smse = tmem, t_sqjl = tmem + 64, t_o = tmem + 128;
    const uint32_t lrow = uint32_t((warp & 3) * 32) << 16;

    const float sl = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)
    const float cq = 1.2533141373155003f / 128.f;                    // sqrt(pi/2) / m
    float m_run = -INFINITY, l_run = 0.f;                            // log2 units
    uint32_t ph_qk = 0, ph_pv = 0;
    bool timeout = false;
    const int n_tiles = (k_end - k_begin + kKeys - 1) / kKeys;

    for (int t = 0; t < n_tiles; ++t) {
        const int k0 = k_begin + t * kKeys;
        if (t > 0) {                                   // PV of the previous tile read V and P
            if (!tc05::mbar_wait_bounded(bar_pv, ph_pv, kPolls)) timeout = true;
            ph_pv ^= 1u;
            tc05::fence_after_sync();
        }
        // ---- dequantize: key kk, coordinates [32 qq, 32 qq + 32)
        {
            const int kk = tid >> 2, qq = tid & 3;
            const int kidx = k0 + kk;
            const uint8_t *page = nullptr;
            if (kidx < k_end) {
                const int blk = a.block_table[kidx >> 6];
                if (blk >= 0 && blk < a.num_blocks)
                    page = a.cache + (int64_t(blk) * L.H + kvh) * int64_t(L.page_bytes);
                else
                    atomicOr(a.status, TQ_DEV_BLOCK_RANGE);
            }
            const int pos = kidx & 63;
            uint32_t kh[16], kl[16], ks[16];
            if (page) {
                uint32_t lo[4], hi;
                load_codes<KB>(page + L.kc_off, L.kc_bpt, page + L.kh_off, L.kh_bpt, pos, qq, lo, hi);
                const uint2 *lk = lutk + (lane & (NCK - 1));
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    const uint2 e = lk[pair_index<KB>(lo, hi, p) * NCK];
                    kh[p] = e.x;
                    kl[p] = e.y;
                }
                const uint32_t sg = *reinterpret_cast<const uint32_t *>(page + L.ks_off + pos * L.ks_bpt + qq * 4);
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    const uint32_t b = sg >> (2 * p);          // bit 0: coordinate 2p, bit 1: 2p + 1
                    ks[p] = 0xBC00BC00u ^ (((b << 15) & 0x8000u) | ((b << 30) & 0x80000000u));
                }
            } else {
#pragma unroll
                for (int p = 0; p < 16; ++p) kh[p] = kl[p] = ks[p] = 0u;
            }
            const uint32_t half = uint32_t(qq >> 1) * 8192u;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t off = half + tc05::sw128_offset(uint32_t(kk), uint32_t((qq & 1) * 4 + c));
                *reinterpret_cast<uint4 *>(sm + SKH + off) = make_uint4(kh[4 * c], kh[4 * c + 1], kh[4 * c + 2], kh[4 * c + 3]);
                *reinterpret_cast<uint4 *>(sm + SKL + off) = make_uint4(kl[4 * c], kl[4 * c + 1], kl[4 * c + 2], kl[4 * c + 3]);
                *reinterpret_cast<uint4 *>(sm + SKS + off) = make_uint4(ks[4 * c], ks[4 * c + 1], ks[4 * c + 2], ks[4 * c + 3]);
            }
            if (qq == 0) {
                float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (page) {
                    const float nk = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kn_off + pos * 2));
                    const float rk = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kr_off + pos * 2));
                    const float nv = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.vn_off + pos * 2));
                    m4 = make_float4(nk * sl, rk * cq * sl, nv, 0.f);
                }
                meta[kk] = m4;
            }
        }
        tc05::fence_proxy_async_smem();
        tc05::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc05::fence_after_sync();
            constexpr uint32_t idesc = tc05::idesc_f16_f32(128, 64);
            const uint32_t qh = tc05::smem_u32(sm + SQH), ql = tc05::smem_u32(sm + SQL);
            const uint32_t qw = tc05::smem_u32(sm + SQW), qwl = tc05::smem_u32(sm + SQWL);
            const uint32_t bh = tc05::smem_u32(sm + SKH), bl = tc05::smem_u32(sm + SKL), bs = tc05::smem_u32(sm + SKS);
            // passes: q_hi C_hi, q_lo C_hi, q_hi C_lo -> S_mse; w_hi Sigma, w_lo Sigma -> S_qjl
#pragma unroll
            for (int pass = 0; pass < 5; ++pass) {
                const uint32_t A = pass == 1 ? ql : pass == 3 ? qw : pass == 4 ? qwl : qh;
                const uint32_t B = pass == 2 ? bl : pass >= 3 ? bs : bh;
                const uint32_t D = pass >= 3 ? t_sqjl : t_smse;
                const bool first = pass == 0 || pass == 3;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = tc05::desc_kmajor_sw128(A + uint32_t(ks >> 2) * 16384u + uint32_t(ks & 3) * 32u);
                    const uint64_t bd = tc05::desc_kmajor_sw128(B + uint32_t(ks >> 2) * 8192u + uint32_t(ks & 3) * 32u);
                    tc05::mma_f16(D, ad, bd, idesc, !first || ks > 0);
                }
            }
            tc05::mma_commit(bar_qk);
        }
        // ---- values: warps 4-7, key kk, dims [64 hh, 64 hh + 64), once QK has
        // read the C_hi tile that V_lo overwrites
        if (warp >= 4) {
            const int t4 = tid - 128, kk = t4 >> 1, hh = t4 & 1;
            const int kidx = k0 + kk;
            const uint8_t *page = nullptr;
            if (kidx < k_end) {
                const int blk = a.block_table[kidx >> 6];
                if (blk >= 0 && blk < a.num_blocks) page = a.cache + (int64_t(blk) * L.H + kvh) * int64_t(L.page_bytes);
            }
            const int pos = kidx & 63;
            if (!tc05::mbar_wait_bounded(bar_qk, ph_qk, kPolls)) timeout = true;
            tc05::fence_after_sync();
            const uint2 *lv = lutv + (lane & (NCV - 1));
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
                const int qq = 2 * hh + sub;
                uint32_t vh[16], vl[16];
                if (page) {
                    uint32_t lo[4], hi;
                    load_codes<VB>(page + L.vc_off, L.vc_bpt, page + L.vh_off, L.vh_bpt, pos, qq, lo, hi);
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        const uint2 e = lv[pair_index<VB>(lo, hi, p) * NCV];
                        vh[p] = e.x;
                        vl[p] = e.y;
                    }
                } else {
#pragma unroll
                    for (int p = 0; p < 16; ++p) vh[p] = vl[p] = 0u;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t off = uint32_t(hh) * 8192u + tc05::sw128_offset(uint32_t(kk), uint32_t(sub * 4 + c));
                    *reinterpret_cast<uint4 *>(sm + SV + off) = make_uint4(vh[4 * c], vh[4 * c + 1], vh[4 * c + 2], vh[4 * c + 3]);
                    *reinterpret_cast<uint4 *>(sm + SKH + off) = make_uint4(vl[4 * c], vl[4 * c + 1], vl[4 * c + 2], vl[4 * c + 3]);
                }
            }
            tc05::fence_proxy_async_smem();
        }
        // ---- softmax: warps 0-3, thread = row
        if (warp < 4) {
            if (!tc05::mbar_wait_bounded(bar_qk, ph_qk, kPolls)) timeout = true;
            tc05::fence_after_sync();
            const int lim = min(k_end, vis_r) - k0;            // keys [0, lim) of the tile are visible
            float lp[64];
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t ra[32], rb[32];
                tc05::tmem_ld_32x32b_x32(t_smse + lrow + uint32_t(c * 32), ra);
                tc05::tmem_ld_32x32b_x32(t_sqjl + lrow + uint32_t(c * 32), rb);
                tc05::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float4 mk = meta[c * 32 + e];
                    float v = fmaf(mk.y, __uint_as_float(rb[e]), mk.x * __uint_as_float(ra[e]));
                    if (c * 32 + e >= lim) v = -INFINITY;
                    lp[c * 32 + e] = v;
                    mx = fmaxf(mx, v);
                }
            }
            const float m_new = fmaxf(m_run, qs * mx);
            const bool grow = m_new > m_run && m_run != -INFINITY && t > 0;
            const float alpha = grow ? exp2f(m_run - m_new) : 1.f;
            if (__any_sync(kFull, grow)) {
                // O rows scaled by alpha (1 for rows whose maximum did not grow)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ro[32];
                    tc05::tmem_ld_32x32b_x32(t_o + lrow + uint32_t(c * 32), ro);
                    tc05::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
                    tc05::tmem_st_32x32b_x32(t_o + lrow + uint32_t(c * 32), ro);
                }
                tc05::tmem_wait_st();
            }
            l_run *= alpha;
            m_run = m_new;
            float psum = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t pw[4], pl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = c * 8 + 2 * e;
                    float p0 = 0.f, p1 = 0.f;
                    if (m_run != -INFINITY) {
                        p0 = exp2f(fmaf(qs, lp[k], -m_run));
                        p1 = exp2f(fmaf(qs, lp[k + 1], -m_run));
                    }
                    psum += p0 + p1;
                    const float q0 = p0 * meta[k].z, q1 = p1 * meta[k + 1].z;
                    const __half2 h = __floats2half2_rn(q0, q1);
                    const float2 hf = __half22float2(h);
                    pw[e] = *reinterpret_cast<const uint32_t *>(&h);
                    pl[e] = h2u(q0 - hf.x, q1 - hf.y);
                }
                const uint32_t off = tc05::sw128_offset(uint32_t(r), uint32_t(c));
                *reinterpret_cast<uint4 *>(sm + SP + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
                *reinterpret_cast<uint4 *>(sm + SKL + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
            }
            l_run += psum;
            tc05::fence_proxy_async_smem();
        }
        ph_qk ^= 1u;
        tc05::fence_before_sync();
        if (__syncthreads_or(timeout)) break;
        if (tid == 0) {
            tc05::fence_after_sync();
            constexpr uint32_t idesc = tc05::idesc_f16_f32(128, 128) | tc05::kIdescBMajorMN;
            const uint32_t ph = tc05::smem_u32(sm + SP), pl = tc05::smem_u32(sm + SKL);
            const uint32_t vh = tc05::smem_u32(sm + SV), vl = tc05::smem_u32(sm + SKH);
            // P'_hi V_hi, P'_lo V_hi, P'_hi V_lo
#pragma unroll
            for (int part = 0; part < 3; ++part)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc05::mma_f16(t_o, tc05::desc_kmajor_sw128((part == 1 ? pl : ph) + uint32_t(ks) * 32u),
                                  tc05::desc_mnmajor_sw128((part == 2 ? vl : vh) + uint32_t(ks) * 2048u, 8192u, 1024u),
                                  idesc, t > 0 || part > 0 || ks > 0);
            tc05::mma_commit(bar_pv);
        }
    }
    // the last PV (or, after an early exit, whatever is in flight)
    if (!tc05::mbar_wait_bounded(bar_pv, ph_pv, kPolls)) timeout = true;
    tc05::fence_after_sync();
    if (warp < 4) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t ro[32];
            tc05::tmem_ld_32x32b_x32(t_o + lrow + uint32_t(c * 32), ro);
            tc05::tmem_wait_ld();
            if (row_ok) {
                float4 *dst = reinterpret_cast<float4 *>(a.part_o + pbase * 128 + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(__uint_as_float(ro[4 * e]), __uint_as_float(ro[4 * e + 1]),
                                         __uint_as_float(ro[4 * e + 2]), __uint_as_float(ro[4 * e + 3]));
            }
        }
        if (row_ok) {
            a.part_ml[pbase * 2] = m_run == -INFINITY ? -INFINITY : m_run * 0.6931471805599453f;
            a.part_ml[pbase * 2 + 1] = l_run;
        }
    }
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, 256);
    }
    if (timeout) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
}

template <int KB, int VB>
int run(const Pf128Args &a, cudaStream_t st) {
    auto kern = pf128_kernel<KB, VB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SM_TOTAL));
    if (e != cudaSuccess) return e;
    const dim3 grid(unsigned((a.C + a.PT - 1) / a.PT), unsigned(a.L.H), unsigned(a.n_splits));
    kern<<<grid, 256, SM_TOTAL, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool pf128_covers(const Layout &L, const AttnShape &s) {
    if (L.d != 128 || L.P != kKeys || !L.kqjl || s.seq_lens != nullptr) return false;
    if (L.kbits < 2 || L.kbits > 4 || L.vbits < 2 || L.vbits > 4) return false;
    if (s.Hq % L.H) return false;
    const int G = s.Hq / L.H;
    if (G < 1 || G > 128 || 128 % G) return false;
    return int64_t(s.n_seq) * G >= 64;                 // at least half a block of query rows
}

int pf128_splits(const Layout &L, const AttnShape &s, int *split_len) {
    const int G = s.Hq / L.H, PT = 128 / G;
    const int64_t blocks = int64_t((s.n_seq + PT - 1) / PT) * L.H;
    const int maxlen = s.max_len > 0 ? s.max_len : 1;
    int best = 1;
    double best_eff = 0.0;
    for (int sp = 1; sp <= 8; ++sp) {
        if (sp > 1 && int64_t(maxlen) < int64_t(sp) * 1024) break;      // keep splits of at least 1,024 keys
        const double waves = double(blocks * sp) / 148.0;
        const double eff = waves / double(int64_t(waves + 0.999999));
        if (eff > best_eff + 0.02) {
            best_eff = eff;
            best = sp;
        }
    }
    int len = (maxlen + best - 1) / best;
    len = (len + kKeys - 1) / kKeys * kKeys;
    *split_len = len;
    return (maxlen + len - 1) / len;
}

int launch_pf128(const tq_params *kp, const tq_params *vp, const Layout &L, const float *qr, const float *w,
                 const AttnShape &s, int n_splits, int split_len, const uint8_t *cache, int64_t num_blocks,
                 float *part_o, float *part_ml, uint32_t *status, cudaStream_t st) {
    Pf128Args a;
    a.L = L;
    a.qr = qr;
    a.w = w;
    a.C = s.n_seq;
    a.Hq = s.Hq;
    a.G = s.Hq / L.H;
    a.PT = 128 / a.G;
    a.base_len = s.base_len;
    a.block_table = s.block_table;
    a.max_blocks = s.max_blocks;
    a.cache = cache;
    a.num_blocks = num_blocks;
    a.k_lv = kp->dev.lv;
    a.v_lv = vp->dev.lv;
    a.n_splits = n_splits;
    a.split_len = split_len;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.status = status;
    const int kb = L.kbits, vb = L.vbits;
#define TQ_PF(KB_, VB_) \
    if (kb == KB_ && vb == VB_) return run<KB_, VB_>(a, st);
    TQ_PF(2, 2) TQ_PF(2, 3) TQ_PF(2, 4) TQ_PF(3, 2) TQ_PF(3, 3) TQ_PF(3, 4) TQ_PF(4, 2) TQ_PF(4, 3) TQ_PF(4, 4)
#undef TQ_PF
    return cudaErrorInvalidValue;
}

}  // namespace tq
