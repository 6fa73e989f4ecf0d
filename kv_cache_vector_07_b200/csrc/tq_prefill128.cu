// Chunked prefill attention over the compressed cache on the tensor cores:
// head dimension 128, pages of 64 tokens, keys b-bit Lloyd-Max + QJL
// (b in {2, 3, 4}), values b-bit (b in {2, 3, 4}).
//
// Page "What is TurboQuant?", "Stage 1"/"Stage 2" and the ai-work-lab
// overview, "QJL": the logit of key t is
//   ( nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1> ) / sqrt(d),
// then softmax and the sum of dequantized values nhat_v c_v[code] (rotated
// back by the combine kernel).  A block takes 128 query rows (positions x
// GQA heads of one KV head) and walks one key split a page (64 keys) at a
// time, with three warp roles synchronized by mbarriers:
//   producers (warps 8-11)  for page t: the key operands (centroids as fp16
//                hi + lo tiles, QJL signs as a +-1 tile, per-key logit
//                scales) into key stage t % 2 as soon as QK(t - 2) and its
//                softmax read are done, then the value operands (centroids as
//                fp16 hi + lo tiles, MN-major, and n_v) into value stage t % 2
//                once PV(t - 2) is done; raw pages arrive by bulk copy ahead;
//   MMA issuer (warp 12)    QK(t): S_mse = q_hi C_hi + q_lo C_hi + q_hi C_lo,
//                S_qjl = w_hi Sigma + w_lo Sigma, with the query tiles as the
//                A operand in tensor memory; then PV(t - 1):
//                O += P_hi V_hi + P_lo V_hi + P_hi V_lo;
//   softmax (warps 0-7)     two threads per row (TMEM lane), one per half of
//                the page's keys: read their half of S (releasing it to
//                QK(t + 1)), logits, causal mask, the row maximum met through
//                shared memory, online sum, O rescaled in TMEM when the
//                maximum grows, P' = p nhat_v as fp16 hi + lo.
// The tensor pipe alternates QK(t + 1) and PV(t) while the softmax of page t
// and the producers of pages t + 1 / t + 2 run.  The hi/lo splits keep
// logits and outputs within tolerance with outlier channels.  The split's
// partial (O, max, sum) goes to the workspace in the layout the log-sum-exp
// combine kernel reads.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tc05.cuh"
#include "tq_dev.cuh"

namespace tq {
namespace {

constexpr int kKeys = 64;               // keys per tile (one page)
constexpr int kThreads = 416;           // 8 softmax + 4 producer warps + 1 MMA warp
constexpr uint32_t kPolls = 1u << 20;   // about a second of polling, then give up

// shared layout (offsets from a 1024-aligned base)
constexpr uint32_t kKStage = 49152, kVStage = 32768;     // one page's key / value operand tiles
constexpr uint32_t SK = 0;                               // [2] key stages: C_hi, C_lo, Sigma
constexpr uint32_t OKH = 0, OKL = 16384, OKS = 32768;    //   [64 keys x 128] K-major, halves at +8 KB
constexpr uint32_t SV = 2 * kKStage;                     // [2] value stages: V_hi, V_lo
constexpr uint32_t OVH = 0, OVL = 16384;                 //   [64 keys x 128 dims] MN-major, halves at +8 KB
constexpr uint32_t SPH = SV + 2 * kVStage, SPL = SPH + 16384;   // P' hi / lo [128 rows x 64 keys] K-major
constexpr uint32_t SKLUT = SPL + 16384;                  // K pair table, 8 KB
constexpr uint32_t SVLUT = SKLUT + 8192;                 // V pair table, 8 KB
constexpr uint32_t SMK = SVLUT + 8192;                   // float2 [2][64]: logit scales a, b
constexpr uint32_t SMV = SMK + 1024;                     // float [2][64]: nhat_v
constexpr uint32_t SQS = SMV + 512;                      // float [128] query scales
constexpr uint32_t SLSUM = SQS + 512;                    // float [2][128] per-half row sums
constexpr uint32_t SXMAX = SLSUM + 1024;                 // float [2][2][128] half-row maxima
constexpr uint32_t SFLAG = SXMAX + 2048;                 // abort flag
constexpr uint32_t SBAR = SFLAG + 16;                    // 16 mbarriers, then 2 page-valid flags
constexpr uint32_t SRAW = SBAR + 160;                    // raw pages (bulk copies)
constexpr uint32_t kSmemMax = 232448;
__host__ __device__ constexpr uint32_t raw_stride(int page_bytes) { return uint32_t((page_bytes + 127) & ~127); }
// raw pages in flight: two when they fit, else one
__host__ __device__ constexpr int raw_slots(int page_bytes) {
    return SRAW + 2u * raw_stride(page_bytes) + 1024u <= kSmemMax ? 2 : 1;
}
__host__ __device__ constexpr uint32_t smem_bytes(int page_bytes) {
    return SRAW + uint32_t(raw_slots(page_bytes)) * raw_stride(page_bytes) + 1024u;
}

// TMEM columns
constexpr uint32_t TQH = 0, TQL = 64, TWH = 128, TWL = 192, TSM = 256, TSQ = 320, TO = 384;

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

// Bounded wait that also gives up once another thread has given up: after a
// few quick polls the thread naps between polls (so waiting warps leave the
// issue slots to the working ones); about a second in all.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag) {
    for (uint32_t i = 0; i < 4u; ++i)
        if (tc05::mbar_try_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < 4000000u; ++i) {
        __nanosleep(64);
        if (tc05::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    *abort_flag = 1u;
    return false;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int KB, int VB>
__global__ void __launch_bounds__(kThreads, 1) pf128_kernel(Pf128Args a) {
    constexpr int NCK = pair_copies<KB, 8, 8192>(), NCV = pair_copies<VB, 8, 8192>();
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_holder;
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint2 *lutk = reinterpret_cast<uint2 *>(sm + SKLUT);
    uint2 *lutv = reinterpret_cast<uint2 *>(sm + SVLUT);
    float2 *metak = reinterpret_cast<float2 *>(sm + SMK);
    float *metav = reinterpret_cast<float *>(sm + SMV);
    float *qs_arr = reinterpret_cast<float *>(sm + SQS);
    float *lsum = reinterpret_cast<float *>(sm + SLSUM);
    float *xmax = reinterpret_cast<float *>(sm + SXMAX);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + SFLAG);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SBAR);
    uint64_t *kfull = bars;         // [2] key operands of a page written (count 128)
    uint64_t *vfull = bars + 2;     // [2] value operands of a page written (count 128)
    uint64_t *kfree = bars + 4;     // [2] QK of the page done (commit) and its S read (256): count 257
    uint64_t *pv_done = bars + 6;   // [2] PV of the page done (commit)
    uint64_t *qk_full = bars + 8;   // QK done (commit)
    uint64_t *p_full = bars + 9;    // softmax wrote P and rescaled O (count 256)
    uint64_t *raw_full = bars + 10; // [2] raw page landed (bulk copy, or plain arrive for a missing page)
    uint64_t *raw_empty = bars + 12;// [2] producers finished reading a raw page (count 128)
    uint64_t *xbar = bars + 14;     // [2] both halves of every row posted their maximum (count 256)
    int *pvalid = reinterpret_cast<int *>(sm + SBAR + 128);   // [2] raw page present

    const Layout &L = a.L;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x, kvh = blockIdx.y, split = blockIdx.z;
    const int G = a.G;
    const int j_lo = qt * a.PT;
    const int j_hi = min(a.C, j_lo + a.PT);
    const int vis_max = a.base_len + j_hi;                 // keys the tile's last row sees
    const int k_begin = split * a.split_len;
    const int k_end = min(k_begin + a.split_len, vis_max);
    const uint32_t rstride = raw_stride(L.page_bytes);
    const int n_raw = raw_slots(L.page_bytes);
    uint8_t *raw = sm + SRAW;
    // softmax rows: warps w and w + 4 share lanes 32 (w % 4) ..
    const int r = (warp & 3) * 32 + lane;
    const int half = (warp >> 2) & 1;
    const int jr = j_lo + r / G, hr = r - (r / G) * G;
    const bool row_ok = jr < a.C;
    const int vis_r = row_ok ? a.base_len + jr + 1 : 0;
    const int64_t pbase = ((int64_t(jr) * L.H + kvh) * a.n_splits + split) * G + hr;

    if (k_begin >= k_end) {                                // nothing visible in this split
        if (warp < 4 && row_ok) {
            a.part_ml[pbase * 2] = -INFINITY;
            a.part_ml[pbase * 2 + 1] = 0.f;
        }
        return;
    }
    const int n_tiles = (k_end - k_begin + kKeys - 1) / kKeys;

    // ---- tables
    for (int i = tid; i < pair_entries<KB>() * NCK; i += kThreads) {
        int k0, k1;
        pair_codes<KB>(i / NCK, k0, k1);
        const float c0 = a.k_lv[k0], c1 = a.k_lv[k1];
        const __half2 h = __floats2half2_rn(c0, c1);
        const float2 hf = __half22float2(h);
        lutk[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&h), h2u(c0 - hf.x, c1 - hf.y));
    }
    for (int i = tid; i < pair_entries<VB>() * NCV; i += kThreads) {
        int k0, k1;
        pair_codes<VB>(i / NCV, k0, k1);
        const float c0 = a.v_lv[k0], c1 = a.v_lv[k1];
        const __half2 h = __floats2half2_rn(c0, c1);
        const float2 hf = __half22float2(h);
        lutv[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&h), h2u(c0 - hf.x, c1 - hf.y));
    }
    if (warp == 12) {
        tc05::tmem_alloc(&tmem_holder, 512);
        tc05::tmem_relinquish();
        if (lane == 0) {
            for (int i = 0; i < 2; ++i) {
                tc05::mbar_init(&kfull[i], 128);
                tc05::mbar_init(&vfull[i], 128);
                tc05::mbar_init(&kfree[i], 257);
                tc05::mbar_init(&pv_done[i], 1);
                tc05::mbar_init(&raw_full[i], 1);
                tc05::mbar_init(&raw_empty[i], 128);
                tc05::mbar_init(&xbar[i], 256);
            }
            tc05::mbar_init(qk_full, 1);
            tc05::mbar_init(p_full, 256);
            *abort_flag = 0u;
            tc05::fence_mbar_init();
        }
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = tmem_holder;
    const uint32_t lrow = uint32_t((warp & 3) * 32) << 16;

    // ---- query tiles into TMEM: row r = 2^-e [q_r hi | q_r lo | w hi | w lo],
    // 1 <= max |.| < 2, 64 columns each (two fp16 per column)
    if (warp < 4) {
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
        qs_arr[r] = mx > 0.f ? ldexpf(1.f, ex - 1) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {                      // 32 coordinates -> 16 columns per tile
            uint32_t qh[16], ql[16], wh[16], wl[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float x0 = 0.f, x1 = 0.f, y0 = 0.f, y1 = 0.f;
                if (row_ok) {
                    const float2 x = *reinterpret_cast<const float2 *>(qp + 32 * c + 2 * e);
                    const float2 y = *reinterpret_cast<const float2 *>(wp + 32 * c + 2 * e);
                    x0 = x.x * down; x1 = x.y * down; y0 = y.x * down; y1 = y.y * down;
                }
                const __half2 h = __floats2half2_rn(x0, x1);
                const float2 hf = __half22float2(h);
                qh[e] = *reinterpret_cast<const uint32_t *>(&h);
                ql[e] = h2u(x0 - hf.x, x1 - hf.y);
                const __half2 g = __floats2half2_rn(y0, y1);
                const float2 gf = __half22float2(g);
                wh[e] = *reinterpret_cast<const uint32_t *>(&g);
                wl[e] = h2u(y0 - gf.x, y1 - gf.y);
            }
            tc05::tmem_st_32x32b_x16(tmem + lrow + TQH + uint32_t(16 * c), qh);
            tc05::tmem_st_32x32b_x16(tmem + lrow + TQL + uint32_t(16 * c), ql);
            tc05::tmem_st_32x32b_x16(tmem + lrow + TWH + uint32_t(16 * c), wh);
            tc05::tmem_st_32x32b_x16(tmem + lrow + TWL + uint32_t(16 * c), wl);
        }
        tc05::tmem_wait_st();
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();

    const float sl = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)
    const float cq = 1.2533141373155003f / 128.f;                    // sqrt(pi/2) / m
    bool timeout = false;

    if (warp >= 8 && warp < 12) {
        // ================= producers: key kk (one per lane), dims [64 hh, 64 hh + 64)
        const int t4 = tid - 256, kk = t4 & 63, hh = t4 >> 6;
        const uint2 *lk = lutk + (lane & (NCK - 1));
        const uint2 *lv = lutv + (lane & (NCV - 1));
        auto issue_raw = [&](int t) {                       // thread 256 only
            const int rs = t % n_raw;
            const int kp = k_begin + t * kKeys;
            int blk = -1;
            if (kp < k_end) blk = a.block_table[kp >> 6];
            if (blk >= 0 && blk < a.num_blocks) {
                pvalid[rs] = 1;
                tc05::mbar_expect_tx(&raw_full[rs], uint32_t(L.page_bytes));
                tc05::bulk_g2s(raw + rs * rstride, a.cache + (int64_t(blk) * L.H + kvh) * int64_t(L.page_bytes),
                               uint32_t(L.page_bytes), &raw_full[rs]);
            } else {
                if (kp < k_end) atomicOr(a.status, TQ_DEV_BLOCK_RANGE);
                pvalid[rs] = 0;
                tc05::mbar_arrive(&raw_full[rs]);
            }
        };
        int issued = 0, landed = 0;                          // thread 256: raw pages requested / seen landed
        if (tid == 256) {
            for (int j = 0; j < n_raw && j < n_tiles; ++j) issue_raw(j);
            issued = min(n_raw, n_tiles);
        }
        for (int t = 0; t < n_tiles; ++t) {
            const int st = t & 1;
            const int rs = t % n_raw;
            const uint32_t ruse = uint32_t(t / n_raw) & 1u;   // phase of this raw slot's use
            if (!wait_or_abort(&raw_full[rs], ruse, abort_flag)) { timeout = true; break; }
            landed = t + 1;
            const int kidx = k_begin + t * kKeys + kk;
            const uint8_t *page = (pvalid[rs] && kidx < k_end) ? raw + rs * rstride : nullptr;
            const int pos = kk;
            // -- key operands, once QK(t - 2) and the softmax's read of its S are done
            if (t >= 2 && !wait_or_abort(&kfree[st], uint32_t((t - 2) >> 1) & 1u, abort_flag)) {
                timeout = true;
                break;
            }
            uint8_t *kb = sm + SK + uint32_t(st) * kKStage;
#pragma unroll 1
            for (int sub = 0; sub < 2; ++sub) {
                const int qq = 2 * hh + sub;
                uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi = 0u, sg = 0u;
                if (page) {
                    load_codes<KB>(page + L.kc_off, L.kc_bpt, page + L.kh_off, L.kh_bpt, pos, qq, lo, hi);
                    sg = *reinterpret_cast<const uint32_t *>(page + L.ks_off + pos * L.ks_bpt + qq * 4);
                }
                const uint32_t hoff = uint32_t(hh) * 8192u;
#pragma unroll
                for (int c = 0; c < 4; ++c) {                   // 8 coordinates: one 16-byte chunk per tile
                    uint32_t x0[4], x1[4], x2[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int p = 4 * c + q;
                        if (page) {
                            const uint2 e = lk[pair_index<KB>(lo, hi, p) * NCK];
                            const uint32_t b = sg >> (2 * p);  // bit 0: coordinate 2p, bit 1: 2p + 1
                            x0[q] = e.x;
                            x1[q] = e.y;
                            x2[q] = 0xBC00BC00u ^ (((b << 15) & 0x8000u) | ((b << 30) & 0x80000000u));
                        } else {
                            x0[q] = x1[q] = x2[q] = 0u;
                        }
                    }
                    const uint32_t off = hoff + tc05::sw128_offset(uint32_t(kk), uint32_t(sub * 4 + c));
                    *reinterpret_cast<uint4 *>(kb + OKH + off) = make_uint4(x0[0], x0[1], x0[2], x0[3]);
                    *reinterpret_cast<uint4 *>(kb + OKL + off) = make_uint4(x1[0], x1[1], x1[2], x1[3]);
                    *reinterpret_cast<uint4 *>(kb + OKS + off) = make_uint4(x2[0], x2[1], x2[2], x2[3]);
                }
            }
            if (hh == 0) {
                float2 m2 = make_float2(0.f, 0.f);
                if (page) {
                    const float nk = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kn_off + pos * 2));
                    const float rk = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kr_off + pos * 2));
                    m2 = make_float2(nk * sl, rk * cq * sl);
                }
                metak[st * 64 + kk] = m2;
            }
            tc05::fence_proxy_async_smem();
            tc05::mbar_arrive(&kfull[st]);
            // -- value operands, once PV(t - 2) is done
            if (t >= 2 && !wait_or_abort(&pv_done[st], uint32_t((t - 2) >> 1) & 1u, abort_flag)) {
                timeout = true;
                break;
            }
            uint8_t *vb = sm + SV + uint32_t(st) * kVStage;
#pragma unroll 1
            for (int sub = 0; sub < 2; ++sub) {
                const int qq = 2 * hh + sub;
                uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi = 0u;
                if (page) load_codes<VB>(page + L.vc_off, L.vc_bpt, page + L.vh_off, L.vh_bpt, pos, qq, lo, hi);
                const uint32_t hoff = uint32_t(hh) * 8192u;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t x0[4], x1[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (page) {
                            const uint2 e = lv[pair_index<VB>(lo, hi, 4 * c + q) * NCV];
                            x0[q] = e.x;
                            x1[q] = e.y;
                        } else {
                            x0[q] = x1[q] = 0u;
                        }
                    }
                    const uint32_t off = hoff + tc05::sw128_offset(uint32_t(kk), uint32_t(sub * 4 + c));
                    *reinterpret_cast<uint4 *>(vb + OVH + off) = make_uint4(x0[0], x0[1], x0[2], x0[3]);
                    *reinterpret_cast<uint4 *>(vb + OVL + off) = make_uint4(x1[0], x1[1], x1[2], x1[3]);
                }
            }
            if (hh == 0)
                metav[st * 64 + kk] =
                    page ? h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.vn_off + pos * 2)) : 0.f;
            tc05::mbar_arrive(&raw_empty[rs]);                  // raw page read
            tc05::fence_proxy_async_smem();
            tc05::mbar_arrive(&vfull[st]);
            if (tid == 256 && t + n_raw < n_tiles) {
                // the raw slot is refilled once every producer has read it
                if (!wait_or_abort(&raw_empty[rs], ruse, abort_flag)) { timeout = true; break; }
                issue_raw(t + n_raw);
                issued = t + n_raw + 1;
            }
        }
        // after an early exit, copies still in flight land before shared memory is given back
        if (tid == 256)
            for (int j = landed; j < issued; ++j)
                if (!tc05::mbar_wait_bounded(&raw_full[j % n_raw], uint32_t(j / n_raw) & 1u, kPolls)) timeout = true;
    } else if (warp == 12) {
        // ================= MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc05::idesc_f16_f32(128, 64);
            constexpr uint32_t idesc_pv = tc05::idesc_f16_f32(128, 128) | tc05::kIdescBMajorMN;
            const uint32_t ph = tc05::smem_u32(sm + SPH), pl = tc05::smem_u32(sm + SPL);
            auto issue_pv = [&](int t) {
                const uint32_t vb = tc05::smem_u32(sm + SV + uint32_t(t & 1) * kVStage);
#pragma unroll
                for (int part = 0; part < 3; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc05::mma_f16(tmem + TO, tc05::desc_kmajor_sw128((part == 1 ? pl : ph) + uint32_t(ks) * 32u),
                                      tc05::desc_mnmajor_sw128(vb + (part == 2 ? OVL : OVH) + uint32_t(ks) * 2048u,
                                                               8192u, 1024u),
                                      idesc_pv, t > 0 || part > 0 || ks > 0);
                tc05::mma_commit(&pv_done[t & 1]);
            };
            int issued_pv = 0;
            for (int t = 0; t < n_tiles && !timeout; ++t) {
                const int st = t & 1;
                if (!wait_or_abort(&kfull[st], uint32_t(t >> 1) & 1u, abort_flag)) { timeout = true; break; }
                // S free: the softmax has read S(t - 1)
                if (t >= 1 && !wait_or_abort(&kfree[(t - 1) & 1], uint32_t((t - 1) >> 1) & 1u, abort_flag)) {
                    timeout = true;
                    break;
                }
                tc05::fence_after_sync();
                const uint32_t kb = tc05::smem_u32(sm + SK + uint32_t(st) * kKStage);
                // passes: q_hi C_hi, q_lo C_hi, q_hi C_lo -> S_mse; w_hi Sigma, w_lo Sigma -> S_qjl
#pragma unroll
                for (int pass = 0; pass < 5; ++pass) {
                    const uint32_t A = tmem + (pass == 1 ? TQL : pass == 3 ? TWH : pass == 4 ? TWL : TQH);
                    const uint32_t B = kb + (pass == 2 ? OKL : pass >= 3 ? OKS : OKH);
                    const uint32_t D = tmem + (pass >= 3 ? TSQ : TSM);
                    const bool first = pass == 0 || pass == 3;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc05::mma_f16_ts(D, A + uint32_t(ks) * 8u,
                                         tc05::desc_kmajor_sw128(B + uint32_t(ks >> 2) * 8192u + uint32_t(ks & 3) * 32u),
                                         idesc_qk, !first || ks > 0);
                }
                tc05::mma_commit(qk_full);
                tc05::mma_commit(&kfree[st]);
                if (t >= 1) {
                    const int u = t - 1;
                    if (!wait_or_abort(p_full, uint32_t(u) & 1u, abort_flag) ||
                        !wait_or_abort(&vfull[u & 1], uint32_t(u >> 1) & 1u, abort_flag)) {
                        timeout = true;
                        break;
                    }
                    tc05::fence_after_sync();
                    issue_pv(u);
                    issued_pv = t;
                }
            }
            if (!timeout) {
                const int u = n_tiles - 1;
                if (wait_or_abort(p_full, uint32_t(u) & 1u, abort_flag) &&
                    wait_or_abort(&vfull[u & 1], uint32_t(u >> 1) & 1u, abort_flag)) {
                    tc05::fence_after_sync();
                    issue_pv(u);
                    issued_pv = n_tiles;
                } else {
                    timeout = true;
                }
            }
            // everything this thread issued completes before TMEM is given back
            if (issued_pv > 0 &&
                !wait_or_abort(&pv_done[(issued_pv - 1) & 1], uint32_t((issued_pv - 1) >> 1) & 1u, abort_flag))
                timeout = true;
        }
        __syncwarp();
    } else {
        // ================= softmax: row r, keys [32 half, 32 half + 32) of each page
        const float qs = qs_arr[r];
        float m_run = -INFINITY, l_run = 0.f;                    // log2 units
        // waits decided per warp, so the warp-wide TMEM accesses stay converged
        auto wait_w = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(kFull, wait_or_abort(bar, parity, abort_flag));
        };
        for (int t = 0; t < n_tiles; ++t) {
            const int st = t & 1;
            const int k0 = k_begin + t * kKeys;
            // QK(t) done; its key scales were published with the key operands
            if (!wait_w(qk_full, uint32_t(t) & 1u) || !wait_w(&kfull[st], uint32_t(t >> 1) & 1u)) {
                timeout = true;
                break;
            }
            tc05::fence_after_sync();
            const int lim = min(k_end, vis_r) - k0;            // keys [0, lim) of the page are visible
            // this thread's 32 columns of S, 16 at a time; then S (and the key
            // scales) are released
            float lp[32];
            float mx = -INFINITY;
            const bool all_visible = lim >= kKeys;
            const float2 *mk = metak + st * 64 + half * 32;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t ra[16], rb[16];
                tc05::tmem_ld_32x32b_x16(tmem + lrow + TSM + uint32_t(half * 32 + c * 16), ra);
                tc05::tmem_ld_32x32b_x16(tmem + lrow + TSQ + uint32_t(half * 32 + c * 16), rb);
                tc05::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 m2 = mk[c * 16 + e];
                    float v = fmaf(m2.y, __uint_as_float(rb[e]), m2.x * __uint_as_float(ra[e]));
                    if (!all_visible && half * 32 + c * 16 + e >= lim) v = -INFINITY;
                    lp[c * 16 + e] = v;
                    mx = fmaxf(mx, v);
                }
            }
            tc05::fence_before_sync();
            tc05::mbar_arrive(&kfree[st]);
            // the row maximum over both halves: post, meet, read the other half's
            float *xm = xmax + st * 256;
            xm[half * 128 + r] = mx;
            tc05::mbar_arrive(&xbar[st]);
            if (!wait_w(&xbar[st], uint32_t(t >> 1) & 1u)) {
                timeout = true;
                break;
            }
            mx = fmaxf(mx, xm[(half ^ 1) * 128 + r]);
            const float m_new = fmaxf(m_run, qs * mx);
            const bool grow = m_new > m_run && m_run != -INFINITY && t > 0;
            const float alpha = grow ? exp2f(m_run - m_new) : 1.f;
            // PV(t - 1) done: P is free and O stable; then the page's n_v
            if ((t > 0 && !wait_w(&pv_done[(t - 1) & 1], uint32_t((t - 1) >> 1) & 1u)) ||
                !wait_w(&vfull[st], uint32_t(t >> 1) & 1u)) {
                timeout = true;
                break;
            }
            tc05::fence_after_sync();
            if (__any_sync(kFull, grow)) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {                   // this thread's 64 columns of O
                    uint32_t ro[32];
                    const uint32_t col = TO + uint32_t(half * 64 + c * 32);
                    tc05::tmem_ld_32x32b_x32(tmem + lrow + col, ro);
                    tc05::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
                    tc05::tmem_st_32x32b_x32(tmem + lrow + col, ro);
                }
                tc05::tmem_wait_st();
            }
            l_run *= alpha;
            m_run = m_new;
            float psum = 0.f;
            const float *nvp = metav + st * 64 + half * 32;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pw[4], pl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = c * 8 + 2 * e;                // within this half
                    float p0 = 0.f, p1 = 0.f;
                    if (m_run != -INFINITY) {
                        p0 = ex2_approx(fmaf(qs, lp[k], -m_run));
                        p1 = ex2_approx(fmaf(qs, lp[k + 1], -m_run));
                    }
                    psum += p0 + p1;
                    const float q0 = p0 * nvp[k], q1 = p1 * nvp[k + 1];
                    const __half2 h = __floats2half2_rn(q0, q1);
                    const float2 hf = __half22float2(h);
                    pw[e] = *reinterpret_cast<const uint32_t *>(&h);
                    pl[e] = h2u(q0 - hf.x, q1 - hf.y);
                }
                const uint32_t off = tc05::sw128_offset(uint32_t(r), uint32_t(half * 4 + c));
                *reinterpret_cast<uint4 *>(sm + SPH + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
                *reinterpret_cast<uint4 *>(sm + SPL + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
            }
            l_run += psum;
            tc05::fence_proxy_async_smem();
            tc05::fence_before_sync();
            tc05::mbar_arrive(p_full);
        }
        // ---- partial result of this split: this thread's 64 columns of O
        if (!timeout && !wait_w(&pv_done[(n_tiles - 1) & 1], uint32_t((n_tiles - 1) >> 1) & 1u)) timeout = true;
        tc05::fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            uint32_t ro[32];
            tc05::tmem_ld_32x32b_x32(tmem + lrow + TO + uint32_t(half * 64 + c * 32), ro);
            tc05::tmem_wait_ld();
            if (row_ok) {
                float4 *dst = reinterpret_cast<float4 *>(a.part_o + pbase * 128 + half * 64 + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(__uint_as_float(ro[4 * e]), __uint_as_float(ro[4 * e + 1]),
                                         __uint_as_float(ro[4 * e + 2]), __uint_as_float(ro[4 * e + 3]));
            }
        }
        lsum[half * 128 + r] = l_run;                  // the two halves' sums meet after the barrier
        if (half == 0 && row_ok) a.part_ml[pbase * 2] = m_run == -INFINITY ? -INFINITY : m_run * 0.6931471805599453f;
    }
    tc05::fence_before_sync();
    __syncthreads();
    if (warp < 4 && row_ok) a.part_ml[pbase * 2 + 1] = lsum[r] + lsum[128 + r];
    if (warp == 12) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, 512);
    }
    if (timeout || *abort_flag) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
}

template <int KB, int VB>
int run(const Pf128Args &a, cudaStream_t st) {
    auto kern = pf128_kernel<KB, VB>;
    const uint32_t smem = smem_bytes(a.L.page_bytes);
    if (smem > 232448u) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    const dim3 grid(unsigned((a.C + a.PT - 1) / a.PT), unsigned(a.L.H), unsigned(a.n_splits));
    kern<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool pf128_covers(const Layout &L, const AttnShape &s) {
    if (L.d != 128 || L.P != kKeys || !L.kqjl || s.is_decode) return false;
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
