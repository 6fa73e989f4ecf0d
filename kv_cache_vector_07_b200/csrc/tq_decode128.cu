// Attention over the compressed cache for head dimension 128, on the tensor
// cores: logits from packed key codes plus the QJL correction, online
// softmax, value accumulation.
//
// Page "What is TurboQuant?", "Stage 2" (unbiased inner products from the
// 1-bit QJL residual; the attention-logit speed-up quoted there comes from
// scoring compressed keys); the estimator is
//   l_t = (nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1>) / sqrt(d).
//
// One block = one (query group, key split); four warps share each 64-token
// page (16 tokens each), pages arrive by bulk copy through a ring of shared
// stages.  Per 16 tokens a warp runs
//   scores  S[16 tok x 8] += A[16 tok x 16] B[16 x 8] (mma.sync m16n8k16,
//           fp16 in, fp32 out): A holds the keys' dequantized centroid pairs
//           as fp16 hi + lo (one shared-memory pair-table lookup gives both;
//           two MMAs keep the centroids' fp32 accuracy) and QJL signs
//           as +-1 (one shift and LOP3 per register); B holds the queries'
//           rotated vector and S R q, each split into fp16 hi + lo columns so
//           the products keep fp32 accuracy; scale 1/sqrt(d) * log2(e)
//           folded in.
//   softmax online per head, exp2 domain.
//   values  O^T[16 coord x 8 heads] += V^T[16 x 16 tok] P^T[16 tok x 8]: two
//           tokens' codes for one coordinate are interleaved into one byte
//           and one table lookup gives the fp16 pair.
// Warps merge in shared memory; blocks leave (m, l, o) partials for the
// log-sum-exp combine kernel.
#include <atomic>

#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include "tc05.cuh"
#include "tq_dev.cuh"

namespace tq {

namespace {

// Page stages: 4-bit-key pages (150 B per token) take two, so that four
// blocks fit in an SM's shared memory next to the 256-entry pair tables;
// smaller pages keep three.
template <int KB>
__host__ __device__ constexpr int page_stages() { return KB == 4 ? 2 : 3; }
// Key pair-table entries: two 4-bit codes (256), two 2-bit codes (16); FP8
// keys need no table (each E4M3 byte converts to fp16 exactly).
template <int KB>
__host__ __device__ constexpr int key_entries() { return KB == 4 ? 256 : (KB == 2 ? 16 : 0); }
constexpr uint32_t kPolls = 1u << 20;   // about a second of polling, then give up

struct Dec128Args {
    Layout L;
    const uint8_t *cache;
    int64_t num_blocks;
    int Hq, G, n_splits, pages_per_split;
    const int32_t *block_table;
    int bt_stride, max_blocks;
    const int32_t *seq_lens;
    int base_len;
    const float *qr, *w;           // [rows][128] from the prep kernel
    const float *k_lv, *v_lv;      // levels by stored code
    float *part_o;                 // [group][split][G][128]
    float *part_ml;                // [group][split][G][2]  (natural-log max, sum)
    float *logits;
    int64_t logits_stride;
    uint32_t *status;
    uint32_t stall_polls;          // testing aid: > 0 makes every block first wait
                                   // this many polls on a barrier nothing completes
};

// Bounded wait that also gives up once another thread of the block has given
// up (checked every 256 polls); the first thread to give up raises the flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, uint32_t max_polls,
                                              volatile int *abort_flag) {
    for (uint32_t i = 0; i < max_polls; ++i) {
        if (tc05::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    *abort_flag = 1;
    return false;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t h2bits(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// +-1 fp16 pair from sign bits j and j + 16 of a word (bit set -> +1).
__device__ __forceinline__ uint32_t sign_pair(uint32_t word, int j) {
    return 0xBC00BC00u ^ ((word << (15 - j)) & 0x80008000u);
}

__device__ __forceinline__ int visible(const Dec128Args &a, int b) {
    return a.seq_lens ? a.seq_lens[b] : a.base_len + b + 1;
}

// Pair tables are replicated so that lanes spread over the banks: 16-entry
// tables get 16 (key) / 32 (value) copies, 256-entry tables 8 copies (which
// keeps four blocks' worth of shared memory per SM).  Lane l reads copy
// l mod copies.
template <int B>
__host__ __device__ constexpr int key_copies() { return B == 4 ? 8 : (B == 2 ? 16 : 1); }
template <int B>
__host__ __device__ constexpr int val_copies() { return B == 4 ? 8 : 32; }

// Value table entry e for this lane: half2(lv[e & mask], lv[e >> shift]).
template <int VC>
__device__ __forceinline__ uint32_t lut(const uint32_t *tab_lane, uint32_t e) { return tab_lane[e * VC]; }

template <int KB, int VB, int NT>
__global__ void __launch_bounds__(128) dec128_kernel(Dec128Args a) {
    static_assert(KB == 2 || KB == 4 || KB == 8, "key bits");
    static_assert(VB == 3 || VB == 4, "value bits");
    constexpr bool FP8 = KB == 8;                   // E4M3 keys, no QJL part
    constexpr int kNS = page_stages<KB>();
    constexpr int KE = key_entries<KB>();           // key pair-table entries (two codes)
    constexpr int VE = VB == 4 ? 256 : 16;          // value pair-table entries (two codes / magnitudes)
    constexpr int KC = key_copies<KB>(), VC = val_copies<VB>();
    extern __shared__ __align__(16) uint8_t smem[];
    uint2 *lutK = reinterpret_cast<uint2 *>(smem);                  // [KE][KC copies] {hi pair, lo pair}
    uint32_t *lutV = reinterpret_cast<uint32_t *>(lutK + KE * KC);   // [VE][VC copies]
    uint2 *sB = reinterpret_cast<uint2 *>(lutV + VE * VC);          // [NT][16][32]
    uint8_t *stage0 = reinterpret_cast<uint8_t *>(sB + NT * 16 * 32);
    const Layout &L = a.L;
    const int pbytes = L.page_bytes;
    const int stage_area = max(kNS * pbytes, (64 + 4 * 8 * 128) * 4);
    uint64_t *full = reinterpret_cast<uint64_t *>(stage0 + stage_area);
    uint64_t *empty = full + kNS;
    uint64_t *never = empty + kNS;                 // completed by nothing (stall_polls only)
    int *pvalid = reinterpret_cast<int *>(never + 1);
    volatile int *abort_flag = pvalid + kNS;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int grp = blockIdx.x, split = blockIdx.y;
    const int b = grp / L.H, kvh = grp - b * L.H;
    const int G = a.G;
    const int nv = visible(a, b);
    const int n_pages_seq = (nv + L.P - 1) / L.P;
    const int p_begin = split * a.pages_per_split;
    const int p_end = min(n_pages_seq, p_begin + a.pages_per_split);
    const int n_pages = max(0, p_end - p_begin);
    const int32_t *bt = a.block_table + int64_t(b) * a.bt_stride;
    const int64_t row0 = int64_t(b) * a.Hq + int64_t(kvh) * G;

    // ---- tables: pair lookups (replicated per lane) and query fragments
    for (int i = tid; i < KE * KC; i += 128) {
        // centroid pair as fp16 hi + lo (the pair's fp32 values to ~22 bits)
        const int e = i / KC;
        float c0, c1;
        if (KB == 4) { c0 = a.k_lv[e & 15]; c1 = a.k_lv[e >> 4]; }
        else { c0 = a.k_lv[e & 3]; c1 = a.k_lv[(e >> 2) & 3]; }
        if (FP8) continue;
        const float h0 = __half2float(__float2half_rn(c0)), h1 = __half2float(__float2half_rn(c1));
        lutK[i] = make_uint2(h2bits(h0, h1), h2bits(c0 - h0, c1 - h1));
    }
    for (int i = tid; i < VE * VC; i += 128) {
        const int e = i / VC;
        float lo, hi;
        if (VB == 4) { lo = a.v_lv[e & 15]; hi = a.v_lv[e >> 4]; }
        else { lo = a.v_lv[e & 3]; hi = a.v_lv[(e >> 2) & 3]; }       // magnitudes (positive half)
        lutV[i] = h2bits(lo, hi);
    }
    {
        const float qs = 0.08838834764831845f * 1.4426950408889634f;   // 1/sqrt(128) * log2(e)
        for (int i = tid; i < NT * 16 * 32; i += 128) {
            const int ln = i & 31, ks = (i >> 5) & 15, nt = i >> 9;
            const int gg = ln >> 2, tt = ln & 3;
            const int hd = 4 * nt + (gg >> 1);
            const bool lo_part = (gg & 1) != 0;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (hd < G && !(FP8 && ks >= 8)) {
                const float *src = ks < 8 ? a.qr + (row0 + hd) * 128 : a.w + (row0 + hd) * 128;
                int c[4];
                if (ks < 8) {
                    const int base = 32 * tt + 4 * ks;
                    c[0] = base; c[1] = base + 1; c[2] = base + 2; c[3] = base + 3;
                } else {
                    const int j = 2 * (ks - 8);
                    c[0] = 32 * tt + j; c[1] = 32 * tt + j + 16; c[2] = 32 * tt + j + 1; c[3] = 32 * tt + j + 17;
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float x = src[c[k]] * qs;
                    const float h = __half2float(__float2half_rn(x));
                    v[k] = lo_part ? (x - h) : h;
                }
            }
            sB[i] = make_uint2(h2bits(v[0], v[1]), h2bits(v[2], v[3]));
        }
    }
    if (tid == 0) {
        for (int s = 0; s < kNS; ++s) {
            tc05::mbar_init(&full[s], 1);
            tc05::mbar_init(&empty[s], 4);
        }
        tc05::mbar_init(never, 1);
        *abort_flag = 0;
        tc05::fence_mbar_init();
    }
    __syncthreads();
    // Testing aid: a wait that runs out before any bulk copy is issued, so the
    // block takes the abort path with nothing in flight.
    if (a.stall_polls) wait_or_abort(never, 0, a.stall_polls, abort_flag);
    __syncthreads();

    auto issue_page = [&](int i) {          // thread 0 only
        const int st = i % kNS;
        const int pi = p_begin + i;
        const int blk = pi < a.max_blocks ? bt[pi] : -1;
        if (blk >= 0 && blk < a.num_blocks) {
            pvalid[st] = 1;
            tc05::mbar_expect_tx(&full[st], uint32_t(pbytes));
            tc05::bulk_g2s(stage0 + st * pbytes, a.cache + (int64_t(blk) * L.H + kvh) * pbytes, uint32_t(pbytes),
                           &full[st]);
        } else {
            atomicOr(a.status, TQ_DEV_BLOCK_RANGE);
            pvalid[st] = 0;
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc05::smem_u32(&full[st])) : "memory");
        }
    };
    // Pages [0, issued) have been handed to the copy engine (thread 0's count).
    // On the first wait that runs out, every warp leaves the page loop at its
    // next check, no further copy is issued, and thread 0 drains the copies
    // still in flight before the stage memory is reused for the merge.
    int issued = 0;
    if (tid == 0 && !*abort_flag)
        for (int i = 0; i < kNS - 1 && i < n_pages; ++i) { issue_page(i); issued = i + 1; }

    const uint2 *lutK_l = lutK + (lane & (KC - 1));
    const uint32_t *lutV_l = lutV + (lane & (VC - 1));
    const float cq = 1.2533141373155003f / 128.0f;       // sqrt(pi/2) / m
    float m_run[NT], l_run[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) { m_run[nt] = -INFINITY; l_run[nt] = 0.f; }
    float O[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) O[mt][k] = 0.f;

    int i_stop = n_pages;                  // thread 0: first page not consumed
    for (int i = 0; i < n_pages; ++i) {
        const int st = i % kNS;
        bool fail = *abort_flag != 0;
        if (!fail && tid == 0 && i + kNS - 1 < n_pages) {
            const int j = i + kNS - 1;            // refill the stage page i-1 used
            if (j >= kNS && !wait_or_abort(&empty[j % kNS], uint32_t(((j / kNS) - 1) & 1), kPolls, abort_flag))
                fail = true;
            else { issue_page(j); issued = j + 1; }
        }
        if (!fail) fail = !wait_or_abort(&full[st], uint32_t((i / kNS) & 1), kPolls, abort_flag);
        if (__any_sync(kFull, fail || *abort_flag)) {
            if (lane == 0) *abort_flag = 1;
            i_stop = i;
            break;
        }
        const uint8_t *pg = stage0 + st * pbytes;
        const int tok0 = (p_begin + i) * L.P + warp * 16;     // token index of row 0 of this warp
        if (pvalid[st] && tok0 < nv && warp * 16 < L.P) {
            const int pr = warp * 16;                           // position of row 0 in the page
            // ---------------- scores
            float accM[NT][4], accQ[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k) { accM[nt][k] = 0.f; accQ[nt][k] = 0.f; }
            if constexpr (FP8) {
                // E4M3 bytes [32t, 32t + 32) of tokens g and g + 8; bytes 4ks .. 4ks + 3
                // hold the coordinates of k = 2t, 2t+1 (low pair) and 2t+8, 2t+9 (high pair)
                const uint8_t *kcb = pg + L.kc_off;
                const uint4 u0 = *reinterpret_cast<const uint4 *>(kcb + (pr + g) * 128 + 32 * t);
                const uint4 u1 = *reinterpret_cast<const uint4 *>(kcb + (pr + g) * 128 + 32 * t + 16);
                const uint4 u2 = *reinterpret_cast<const uint4 *>(kcb + (pr + g + 8) * 128 + 32 * t);
                const uint4 u3 = *reinterpret_cast<const uint4 *>(kcb + (pr + g + 8) * 128 + 32 * t + 16);
                const uint32_t w0[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                const uint32_t w1[8] = {u2.x, u2.y, u2.z, u2.w, u3.x, u3.y, u3.z, u3.w};
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t A[4];
                    A[0] = e4m3x2_to_half2_bits(w0[ks]);
                    A[2] = e4m3x2_to_half2_bits(w0[ks] >> 16);
                    A[1] = e4m3x2_to_half2_bits(w1[ks]);
                    A[3] = e4m3x2_to_half2_bits(w1[ks] >> 16);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint2 bb = sB[(nt * 16 + ks) * 32 + lane];
                        mma16816(accM[nt], A, bb.x, bb.y);
                    }
                }
            } else {
                // key codes of tokens g and g + 8 for coordinates [32t, 32t + 32)
                uint32_t kc0[KB == 8 ? 1 : KB], kc1[KB == 8 ? 1 : KB];
                const uint8_t *kcb = pg + L.kc_off;
                if (KB == 4) {
                    const uint4 u0 = *reinterpret_cast<const uint4 *>(kcb + (pr + g) * 64 + 16 * t);
                    const uint4 u1 = *reinterpret_cast<const uint4 *>(kcb + (pr + g + 8) * 64 + 16 * t);
                    kc0[0] = u0.x; kc0[1] = u0.y; kc0[KB > 2 ? 2 : 0] = u0.z; kc0[KB > 2 ? 3 : 1] = u0.w;
                    kc1[0] = u1.x; kc1[1] = u1.y; kc1[KB > 2 ? 2 : 0] = u1.z; kc1[KB > 2 ? 3 : 1] = u1.w;
                } else {
                    const uint2 u0 = *reinterpret_cast<const uint2 *>(kcb + (pr + g) * 32 + 8 * t);
                    const uint2 u1 = *reinterpret_cast<const uint2 *>(kcb + (pr + g + 8) * 32 + 8 * t);
                    kc0[0] = u0.x; kc0[1] = u0.y;
                    kc1[0] = u1.x; kc1[1] = u1.y;
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t e[4];
                    if (KB == 4) {
                        // bytes 2ks, 2ks+1 of the thread's 16 code bytes: coordinate pairs
                        const uint32_t w0 = kc0[ks >> 1], w1 = kc1[ks >> 1];
                        const int sh = 16 * (ks & 1);
                        e[0] = (w0 >> sh) & 0xFF;
                        e[2] = (w0 >> (sh + 8)) & 0xFF;
                        e[1] = (w1 >> sh) & 0xFF;
                        e[3] = (w1 >> (sh + 8)) & 0xFF;
                    } else {
                        // byte ks: two 4-bit pair indices
                        const uint32_t w0 = kc0[ks >> 2], w1 = kc1[ks >> 2];
                        const int sh = 8 * (ks & 3);
                        e[0] = (w0 >> sh) & 0xF;
                        e[2] = (w0 >> (sh + 4)) & 0xF;
                        e[1] = (w1 >> sh) & 0xF;
                        e[3] = (w1 >> (sh + 4)) & 0xF;
                    }
                    uint32_t Ah[4], Al[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const uint2 v = lutK_l[e[r] * KC];
                        Ah[r] = v.x;
                        Al[r] = v.y;
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint2 bb = sB[(nt * 16 + ks) * 32 + lane];
                        mma16816(accM[nt], Ah, bb.x, bb.y);
                        mma16816(accM[nt], Al, bb.x, bb.y);
                    }
                }
                const uint32_t s0 = *reinterpret_cast<const uint32_t *>(pg + L.ks_off + (pr + g) * 16 + 4 * t);
                const uint32_t s1 = *reinterpret_cast<const uint32_t *>(pg + L.ks_off + (pr + g + 8) * 16 + 4 * t);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t A[4];
                    A[0] = sign_pair(s0, 2 * ks);
                    A[2] = sign_pair(s0, 2 * ks + 1);
                    A[1] = sign_pair(s1, 2 * ks);
                    A[3] = sign_pair(s1, 2 * ks + 1);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint2 bb = sB[(nt * 16 + 8 + ks) * 32 + lane];
                        mma16816(accQ[nt], A, bb.x, bb.y);
                    }
                }
            }
            // FP8 keys store sqrt(d) u: their estimate carries an extra 1/sqrt(d)
            const float nsc = FP8 ? 0.08838834764831845f : 1.0f;
            const float nk0 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kn_off + (pr + g) * 2)) * nsc;
            const float nk1 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kn_off + (pr + g + 8) * 2)) * nsc;
            const float rk0 = FP8 ? 0.f : h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kr_off + (pr + g) * 2)) * cq;
            const float rk1 = FP8 ? 0.f : h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kr_off + (pr + g + 8) * 2)) * cq;
            const float nv0 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.vn_off + (pr + g) * 2));
            const float nv1 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.vn_off + (pr + g + 8) * 2));
            const bool ok0 = tok0 + g < nv, ok1 = tok0 + g + 8 < nv;
            // ---------------- online softmax (log2 units) for heads t and 4 + t
            uint32_t pk[NT];           // half2(P'[token g][h], P'[token g+8][h])
            float alpha[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float l0 = ok0 ? fmaf(rk0, accQ[nt][0] + accQ[nt][1], nk0 * (accM[nt][0] + accM[nt][1])) : -INFINITY;
                float l1 = ok1 ? fmaf(rk1, accQ[nt][2] + accQ[nt][3], nk1 * (accM[nt][2] + accM[nt][3])) : -INFINITY;
                const int hd = 4 * nt + t;
                if (a.logits && hd < G) {
                    const float inv_l2e = 0.6931471805599453f;
                    if (ok0) a.logits[(row0 + hd) * a.logits_stride + tok0 + g] = l0 * inv_l2e;
                    if (ok1) a.logits[(row0 + hd) * a.logits_stride + tok0 + g + 8] = l1 * inv_l2e;
                }
                float mx = fmaxf(l0, l1);
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                const float m_new = fmaxf(m_run[nt], mx);
                const float al = m_new == -INFINITY ? 1.f : exp2f(m_run[nt] - m_new);
                const float p0 = m_new == -INFINITY ? 0.f : exp2f(l0 - m_new);
                const float p1 = m_new == -INFINITY ? 0.f : exp2f(l1 - m_new);
                l_run[nt] = fmaf(l_run[nt], al, p0 + p1);
                m_run[nt] = m_new;
                alpha[nt] = al;
                pk[nt] = h2bits(ok0 ? p0 * nv0 : 0.f, ok1 ? p1 * nv1 : 0.f);
            }
            // ---------------- P^T fragment: head column g, tokens 2t, 2t+1 (+8)
            uint32_t b0, b1;
            {
                const int src0 = 4 * (2 * t) + (g & 3), src1 = 4 * (2 * t + 1) + (g & 3);
                uint32_t v0 = __shfl_sync(kFull, pk[0], src0), v1 = __shfl_sync(kFull, pk[0], src1);
                if (NT > 1) {
                    const uint32_t u0 = __shfl_sync(kFull, pk[NT - 1], src0), u1 = __shfl_sync(kFull, pk[NT - 1], src1);
                    if (g >= 4) { v0 = u0; v1 = u1; }
                } else if (g >= 4) {
                    v0 = 0; v1 = 0;
                }
                b0 = prmt(v0, v1, 0x5410);         // tokens 2t, 2t+1
                b1 = prmt(v0, v1, 0x7632);         // tokens 2t+8, 2t+9
            }
            // ---------------- rescale O columns (heads 2t, 2t+1)
            {
                float ah[2];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int hd = 2 * t + c;
                    const float x0 = __shfl_sync(kFull, alpha[0], hd & 3);
                    const float x1 = __shfl_sync(kFull, alpha[NT - 1], hd & 3);
                    ah[c] = hd < 4 ? x0 : x1;
                }
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    O[mt][0] *= ah[0]; O[mt][1] *= ah[1]; O[mt][2] *= ah[0]; O[mt][3] *= ah[1];
                }
            }
            // ---------------- values: thread coordinates [16g, 16g + 16), tokens 2t, 2t+1, 2t+8, 2t+9
            {
                const int ta = pr + 2 * t, tb = ta + 1, tc = ta + 8, td = ta + 9;
                if (VB == 4) {
                    const uint8_t *vc = pg + L.vc_off;
                    const uint2 xa = *reinterpret_cast<const uint2 *>(vc + ta * 64 + 8 * g);
                    const uint2 xb = *reinterpret_cast<const uint2 *>(vc + tb * 64 + 8 * g);
                    const uint2 xc = *reinterpret_cast<const uint2 *>(vc + tc * 64 + 8 * g);
                    const uint2 xd = *reinterpret_cast<const uint2 *>(vc + td * 64 + 8 * g);
#pragma unroll
                    for (int wi = 0; wi < 2; ++wi) {
                        const uint32_t wa = wi ? xa.y : xa.x, wb = wi ? xb.y : xb.x;
                        const uint32_t wc = wi ? xc.y : xc.x, wd = wi ? xd.y : xd.x;
                        // byte k: (token A nibble 2k | token B nibble 2k << 4); odd nibbles likewise
                        const uint32_t eAB = (wa & 0x0F0F0F0Fu) | ((wb << 4) & 0xF0F0F0F0u);
                        const uint32_t oAB = ((wa >> 4) & 0x0F0F0F0Fu) | (wb & 0xF0F0F0F0u);
                        const uint32_t eCD = (wc & 0x0F0F0F0Fu) | ((wd << 4) & 0xF0F0F0F0u);
                        const uint32_t oCD = ((wc >> 4) & 0x0F0F0F0Fu) | (wd & 0xF0F0F0F0u);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int mt = 4 * wi + k;          // coordinates 16g + 2mt, +1
                            uint32_t A[4];
                            A[0] = lut<VC>(lutV_l, (eAB >> (8 * k)) & 0xFF);
                            A[1] = lut<VC>(lutV_l, (oAB >> (8 * k)) & 0xFF);
                            A[2] = lut<VC>(lutV_l, (eCD >> (8 * k)) & 0xFF);
                            A[3] = lut<VC>(lutV_l, (oCD >> (8 * k)) & 0xFF);
                            mma16816(O[mt], A, b0, b1);
                        }
                    }
                } else {
                    // 2-bit magnitudes (word g of each token) + sign bits (word g/2, half g&1)
                    const uint8_t *vc = pg + L.vc_off, *vh = pg + L.vh_off;
                    const uint32_t xa = *reinterpret_cast<const uint32_t *>(vc + ta * 32 + 4 * g);
                    const uint32_t xb = *reinterpret_cast<const uint32_t *>(vc + tb * 32 + 4 * g);
                    const uint32_t xc = *reinterpret_cast<const uint32_t *>(vc + tc * 32 + 4 * g);
                    const uint32_t xd = *reinterpret_cast<const uint32_t *>(vc + td * 32 + 4 * g);
                    const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;
                    const uint32_t zAB = prmt(*reinterpret_cast<const uint32_t *>(vh + ta * 16 + 4 * (g >> 1)),
                                              *reinterpret_cast<const uint32_t *>(vh + tb * 16 + 4 * (g >> 1)), sel);
                    const uint32_t zCD = prmt(*reinterpret_cast<const uint32_t *>(vh + tc * 16 + 4 * (g >> 1)),
                                              *reinterpret_cast<const uint32_t *>(vh + td * 16 + 4 * (g >> 1)), sel);
                    const uint32_t eAB = (xa & 0x33333333u) | ((xb << 2) & 0xCCCCCCCCu);
                    const uint32_t oAB = ((xa >> 2) & 0x33333333u) | (xb & 0xCCCCCCCCu);
                    const uint32_t eCD = (xc & 0x33333333u) | ((xd << 2) & 0xCCCCCCCCu);
                    const uint32_t oCD = ((xc >> 2) & 0x33333333u) | (xd & 0xCCCCCCCCu);
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        const int e0 = 2 * mt, e1 = 2 * mt + 1;     // coordinates 16g + e
                        uint32_t A[4];
                        A[0] = lut<VC>(lutV_l, (eAB >> (4 * mt)) & 0xF) ^ ((zAB << (15 - e0)) & 0x80008000u);
                        A[1] = lut<VC>(lutV_l, (oAB >> (4 * mt)) & 0xF) ^ ((zAB << (15 - e1)) & 0x80008000u);
                        A[2] = lut<VC>(lutV_l, (eCD >> (4 * mt)) & 0xF) ^ ((zCD << (15 - e0)) & 0x80008000u);
                        A[3] = lut<VC>(lutV_l, (oCD >> (4 * mt)) & 0xF) ^ ((zCD << (15 - e1)) & 0x80008000u);
                        mma16816(O[mt], A, b0, b1);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc05::smem_u32(&empty[st])) : "memory");
    }

    // ---- merge the four warps: m, l per head; O in the rotated basis
    __syncthreads();
    const bool timeout = *abort_flag != 0;
    if (timeout) {
        if (tid == 0)                      // let copies in flight land before the stages are reused
            for (int p = i_stop; p < issued; ++p)
                tc05::mbar_wait_bounded(&full[p % kNS], uint32_t((p / kNS) & 1), kPolls);
        __syncthreads();
    }
    float *mm = reinterpret_cast<float *>(stage0);               // [4 warps][8 heads]
    float *ll = mm + 32;
    float *oo = ll + 32;                                         // [4 warps][8 heads][128]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float ls = l_run[nt];
        ls += __shfl_xor_sync(kFull, ls, 4);
        ls += __shfl_xor_sync(kFull, ls, 8);
        ls += __shfl_xor_sync(kFull, ls, 16);
        if (g == 0) {
            mm[warp * 8 + 4 * nt + t] = m_run[nt];
            ll[warp * 8 + 4 * nt + t] = ls;
        }
    }
    __syncthreads();
    float scale_w[2];
    {
        // this warp's factor for heads 2t, 2t+1: exp2(m_warp - M)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int hd = 2 * t + c;
            float M = -INFINITY;
            for (int w2 = 0; w2 < 4; ++w2) M = fmaxf(M, mm[w2 * 8 + hd]);
            const float mw = mm[warp * 8 + hd];
            scale_w[c] = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        }
    }
    // each warp writes its scaled O; the four are summed in a fixed order
    float *ow = oo + warp * (8 * 128);                           // [warp][8 heads][128]
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        const int c0 = 16 * g + 2 * mt;
        ow[(2 * t) * 128 + c0] = O[mt][0] * scale_w[0];
        ow[(2 * t + 1) * 128 + c0] = O[mt][1] * scale_w[1];
        ow[(2 * t) * 128 + c0 + 1] = O[mt][2] * scale_w[0];
        ow[(2 * t + 1) * 128 + c0 + 1] = O[mt][3] * scale_w[1];
    }
    __syncthreads();
    const int64_t pbase = (int64_t(grp) * a.n_splits + split) * G;
    for (int i = tid; i < G * 128; i += 128)
        a.part_o[pbase * 128 + i] = ((oo[i] + oo[1024 + i]) + oo[2048 + i]) + oo[3072 + i];
    if (tid < G) {
        float M = -INFINITY;
        for (int w2 = 0; w2 < 4; ++w2) M = fmaxf(M, mm[w2 * 8 + tid]);
        float S = 0.f;
        for (int w2 = 0; w2 < 4; ++w2) {
            const float mw = mm[w2 * 8 + tid];
            if (mw != -INFINITY) S += ll[w2 * 8 + tid] * exp2f(mw - M);
        }
        a.part_ml[(pbase + tid) * 2] = M == -INFINITY ? -INFINITY : M * 0.6931471805599453f;
        a.part_ml[(pbase + tid) * 2 + 1] = S;
    }
    if (timeout) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
}

template <int KB, int VB, int NT>
size_t dec_smem(int page_bytes) {
    constexpr int KE = key_entries<KB>(), VE = VB == 4 ? 256 : 16;
    // the stage area also holds the final merge: 64 + 4 x 8 x 128 floats
    constexpr int kNS = page_stages<KB>();
    size_t stages = size_t(kNS) * page_bytes;
    if (stages < (64 + 4 * 8 * 128) * 4) stages = (64 + 4 * 8 * 128) * 4;
    return size_t(KE) * key_copies<KB>() * 8 + size_t(VE) * val_copies<VB>() * 4 + size_t(NT) * 16 * 32 * 8 +
           stages + (2 * kNS + 1) * 8 + kNS * 4 + 4 + 64;
}

size_t dec_smem_for(const Layout &L, int G) {
    const bool two = G > 4;
    if (L.kbits == 8 && L.vbits == 4) return two ? dec_smem<8, 4, 2>(L.page_bytes) : dec_smem<8, 4, 1>(L.page_bytes);
    if (L.kbits == 8 && L.vbits == 3) return two ? dec_smem<8, 3, 2>(L.page_bytes) : dec_smem<8, 3, 1>(L.page_bytes);
    if (L.kbits == 2 && L.vbits == 4) return two ? dec_smem<2, 4, 2>(L.page_bytes) : dec_smem<2, 4, 1>(L.page_bytes);
    if (L.kbits == 2 && L.vbits == 3) return two ? dec_smem<2, 3, 2>(L.page_bytes) : dec_smem<2, 3, 1>(L.page_bytes);
    if (L.kbits == 4 && L.vbits == 4) return two ? dec_smem<4, 4, 2>(L.page_bytes) : dec_smem<4, 4, 1>(L.page_bytes);
    return two ? dec_smem<4, 3, 2>(L.page_bytes) : dec_smem<4, 3, 1>(L.page_bytes);
}

template <int KB, int VB, int NT>
int run_dec(const Dec128Args &a, int n_groups, cudaStream_t st) {
    const size_t smem = dec_smem<KB, VB, NT>(a.L.page_bytes);
    auto kern = dec128_kernel<KB, VB, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(n_groups), unsigned(a.n_splits)), 128, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

namespace {
std::atomic<uint32_t> g_decode_stall{0};
}

uint32_t take_decode_stall() { return g_decode_stall.exchange(0); }

// Blocks of the tensor-core decode kernel that fit on one SM (shared memory:
// 228 KB per SM, 1 KB reserved per block; registers: at most 6 blocks for
// one query-head tile, 4 for two), or 0 when the configuration is not covered.
bool dec128_keys_ok(const Layout &L) {
    return ((L.kbits == 2 || L.kbits == 4) && L.kqjl) || (L.kbits == 8 && !L.kqjl);
}

int dec128_resident(const Layout &L, int G) {
    if (L.d != 128 || L.P != 64 || G > 8) return 0;
    if (!dec128_keys_ok(L) || !(L.vbits == 3 || L.vbits == 4)) return 0;
    const size_t per = dec_smem_for(L, G) + 1024;
    const int by_smem = int(233472 / per);
    const int by_regs = G > 4 ? 4 : 6;
    return by_smem < by_regs ? by_smem : by_regs;
}

// Tensor-core attention for d = 128; returns -1 when the configuration is not
// covered (the caller then uses the general kernel).
int launch_dec128(const tq_params *kp, const tq_params *vp, const Layout &L, const float *qr, const float *w,
                  const AttnShape &s, int G, int n_groups, int n_splits, int split_len, const uint8_t *cache,
                  int64_t num_blocks, float *part_o, float *part_ml, float *logits, int64_t logits_stride,
                  uint32_t *status, cudaStream_t st) {
    if (L.d != 128 || L.P != 64 || G > 8) return -1;
    if (!dec128_keys_ok(L) || !(L.vbits == 3 || L.vbits == 4)) return -1;
    if (split_len % L.P) return -1;
    Dec128Args a;
    a.L = L;
    a.cache = cache;
    a.num_blocks = num_blocks;
    a.Hq = s.Hq;
    a.G = G;
    a.n_splits = n_splits;
    a.pages_per_split = split_len / L.P;
    a.block_table = s.block_table;
    a.bt_stride = s.bt_stride;
    a.max_blocks = s.max_blocks;
    a.seq_lens = s.seq_lens;
    a.base_len = s.base_len;
    a.qr = qr;
    a.w = w;
    a.k_lv = kp->dev.lv;
    a.v_lv = vp->dev.lv;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.logits = logits;
    a.logits_stride = logits_stride;
    a.status = status;
    a.stall_polls = take_decode_stall();
    const bool two = G > 4;
    if (L.kbits == 2 && L.vbits == 4) return two ? run_dec<2, 4, 2>(a, n_groups, st) : run_dec<2, 4, 1>(a, n_groups, st);
    if (L.kbits == 2 && L.vbits == 3) return two ? run_dec<2, 3, 2>(a, n_groups, st) : run_dec<2, 3, 1>(a, n_groups, st);
    if (L.kbits == 4 && L.vbits == 4) return two ? run_dec<4, 4, 2>(a, n_groups, st) : run_dec<4, 4, 1>(a, n_groups, st);
    if (L.kbits == 4 && L.vbits == 3) return two ? run_dec<4, 3, 2>(a, n_groups, st) : run_dec<4, 3, 1>(a, n_groups, st);
    if (L.kbits == 8 && L.vbits == 4) return two ? run_dec<8, 4, 2>(a, n_groups, st) : run_dec<8, 4, 1>(a, n_groups, st);
    if (L.kbits == 8 && L.vbits == 3) return two ? run_dec<8, 3, 2>(a, n_groups, st) : run_dec<8, 3, 1>(a, n_groups, st);
    return -1;
}

void set_decode_stall(uint32_t polls) { g_decode_stall.store(polls); }

}  // namespace tq

extern "C" int tq_test_stall_next_decode(uint32_t polls) {
    tq::set_decode_stall(polls);
    return TQ_OK;
}
