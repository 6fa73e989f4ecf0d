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

// Fractional rates (FR): keys of KB bits on coordinates 0 .. 63 and KB - 1
// on 64 .. 127 (KB in {2, 3}), both halves through fp16 hi + lo pair tables;
// values of 4 bits, then 3.  K-steps 0 .. 3 cover the first half, 4 .. 7 the
// second, so no k-step mixes the two codebooks.
//
// Page stages: 4-bit-key pages (150 B per token) take two, so that four
// blocks fit in an SM's shared memory next to the 256-entry pair tables;
// smaller pages keep three.
template <int KB, bool FR = false>
__host__ __device__ constexpr int page_stages() { return KB == 4 || FR ? 2 : 3; }
// Key pair-table entries: two 4-bit codes (256), two 2-bit codes (16); FP8
// keys need no table (each E4M3 byte converts to fp16 exactly).  FR: two
// KB-bit codes (3 bits: two 2-bit magnitudes and two signs, 64), and the
// second half's two (KB - 1)-bit codes.
template <int KB, bool FR = false>
__host__ __device__ constexpr int key_entries() { return FR ? (KB == 3 ? 64 : 16) : (KB == 4 ? 256 : 0); }
template <int KB, bool FR = false>
__host__ __device__ constexpr int key_entries2() { return FR ? (KB == 3 ? 16 : 4) : 0; }
// Query-operand k-steps: 2-bit keys take a sign plane and a sign x magnitude
// plane (8 each) plus 8 for the QJL signs; 4-bit (and FR) keys 8 + 8; FP8 keys 8.
template <int KB, bool FR = false>
__host__ __device__ constexpr int query_ksteps() { return FR ? 16 : (KB == 2 ? 24 : (KB == 4 ? 16 : 8)); }
template <int KB, bool FR = false>
__host__ __device__ constexpr int qjl_kstep0() { return FR ? 8 : (KB == 2 ? 16 : 8); }
// Levels of the two codes of pair-table entry e for codes of W bits (W = 3:
// magnitudes at bits 0-1 / 2-3, signs at bits 4 / 5; else W-bit fields).
template <int W>
__device__ __forceinline__ void pair_codes_of(int e, int &k0, int &k1) {
    if constexpr (W == 3) {
        k0 = (e & 3) | (((e >> 4) & 1) << 2);
        k1 = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
    } else {
        k0 = e & ((1 << W) - 1);
        k1 = (e >> W) & ((1 << W) - 1);
    }
}
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
    const float *k_lv2, *v_lv2;    // fractional rates: the second codebooks
    const float *k_pt, *v_pt;      // polar codes: the angle tables (bounds, cos, sin per level)
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
constexpr int kFrKC = 8, kFrKC2 = 16, kFrVC2 = 32;   // FR copies: key tables, value magnitude table
template <int B>
__host__ __device__ constexpr int val_copies() { return B == 4 ? 8 : 32; }

// Table lookups with the index taken straight from a code word: field
// `pos` (width W bits, at bit W * pos) of `w`, as a byte offset into a table
// of STRIDE-byte entries (STRIDE = copies x entry size), ORed with the
// lane's copy offset (which lies below STRIDE): one shift and one LOP3.
template <int W, int STRIDE>
__device__ __forceinline__ uint32_t field_offset(uint32_t w, int pos, uint32_t lane_off) {
    constexpr int SH = __builtin_ctz(STRIDE);
    constexpr uint32_t MASK = ((1u << W) - 1u) << SH;
    const int r = W * pos - SH;
    const uint32_t x = r >= 0 ? (w >> r) : (w << (-r));
    return (x & MASK) | lane_off;
}
template <typename T>
__device__ __forceinline__ T lds_at(const void *base, uint32_t byte_off) {
    return *reinterpret_cast<const T *>(reinterpret_cast<const uint8_t *>(base) + byte_off);
}

// Polar codes (PL, keys with QJL and values, d = 128): the unit-radius
// reconstruction is rebuilt per token in registers, top down through the
// angle tree (each radius the parent's times the cos / sin of the parent's
// angle centre, the same products in the same order as polar_pair), and its
// fp16 hi + lo pairs are the MMA operands.  Keys as for 4-bit codes (thread
// t: pairs 16t .. 16t + 15), values as for 4-bit codes (thread g: pairs
// 8g .. 8g + 7); no pair tables, two 132-float angle tables.
template <int KB, int VB, int NT, bool FR = false, bool PL = false>
__global__ void __launch_bounds__(128) dec128_kernel(Dec128Args a) {
    static_assert(KB == 2 || KB == 4 || KB == 8 || (FR && KB == 3), "key bits");
    static_assert(VB == 3 || VB == 4, "value bits");
    static_assert(!FR || ((KB == 2 || KB == 3) && VB == 4), "fractional rates: keys 1.5 / 2.5 bits, values 3.5");
    static_assert(!PL || (KB == 4 && VB == 4 && !FR), "polar codes take the 4-bit slots");
    constexpr bool FP8 = KB == 8;                   // E4M3 keys, no QJL part
    constexpr int kNS = PL ? 3 : page_stages<KB, FR>();
    constexpr int KE = PL ? 0 : key_entries<KB, FR>();   // key pair-table entries (two codes)
    constexpr int KE2 = key_entries2<KB, FR>();     // FR: second-half key pair table
    constexpr int VE = PL ? 0 : (VB == 4 ? 256 : 16);    // value pair-table entries (two codes / magnitudes)
    constexpr int VE2 = FR ? 16 : 0;                // FR: second-half value magnitude pairs
    constexpr int KC = FR ? kFrKC : key_copies<KB>(), VC = val_copies<VB>();
    constexpr int NKS = query_ksteps<KB, FR>(), QK0 = qjl_kstep0<KB, FR>();
    constexpr int PT = PL ? 2 * 136 : 0;            // PL: key and value angle tables (floats)
    extern __shared__ __align__(16) uint8_t smem[];
    uint2 *lutK = reinterpret_cast<uint2 *>(smem);                  // [KE][KC copies] {hi pair, lo pair}
    uint2 *lutK2 = lutK + KE * KC;                                  // FR: [KE2][kFrKC2]
    uint2 *lutV = lutK2 + KE2 * kFrKC2;                             // [VE][VC copies] {hi pair, lo pair}
    uint2 *lutV2 = lutV + VE * VC;                                  // FR: [VE2][kFrVC2]
    uint2 *sB = lutV2 + VE2 * kFrVC2;                               // [NT][NKS][32]
    float *ptk = reinterpret_cast<float *>(sB + NT * NKS * 32);     // PL: key angle table, then values'
    float *ptv = ptk + 136;
    uint8_t *stage0 = reinterpret_cast<uint8_t *>(ptk + PT);
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
        int k0 = e & 15, k1 = e >> 4;
        if constexpr (FR) pair_codes_of<KB == 8 ? 1 : KB>(e, k0, k1);
        const float c0 = a.k_lv[k0], c1 = a.k_lv[k1];
        const float h0 = __half2float(__float2half_rn(c0)), h1 = __half2float(__float2half_rn(c1));
        lutK[i] = make_uint2(h2bits(h0, h1), h2bits(c0 - h0, c1 - h1));
    }
    if constexpr (PL) {
        for (int i = tid; i < 132; i += 128) {
            ptk[i] = a.k_pt[i];
            ptv[i] = a.v_pt[i];
        }
    }
    if constexpr (FR) {
        for (int i = tid; i < KE2 * kFrKC2; i += 128) {
            int k0, k1;
            pair_codes_of<(KB > 1 ? KB - 1 : 1)>(i / kFrKC2, k0, k1);
            const float c0 = a.k_lv2[k0], c1 = a.k_lv2[k1];
            const float h0 = __half2float(__float2half_rn(c0)), h1 = __half2float(__float2half_rn(c1));
            lutK2[i] = make_uint2(h2bits(h0, h1), h2bits(c0 - h0, c1 - h1));
        }
        for (int i = tid; i < VE2 * kFrVC2; i += 128) {
            const int e = i / kFrVC2;
            const float lo = a.v_lv2[e & 3], hi = a.v_lv2[(e >> 2) & 3];   // 3-bit magnitudes
            const float h0 = __half2float(__float2half_rn(lo)), h1 = __half2float(__float2half_rn(hi));
            lutV2[i] = make_uint2(h2bits(h0, h1), h2bits(lo - h0, hi - h1));
        }
    }
    for (int i = tid; i < VE * VC; i += 128) {
        const int e = i / VC;
        float lo, hi;
        if (VB == 4) { lo = a.v_lv[e & 15]; hi = a.v_lv[e >> 4]; }
        else { lo = a.v_lv[e & 3]; hi = a.v_lv[(e >> 2) & 3]; }       // magnitudes (positive half)
        // level pair as fp16 hi + lo: outputs of outlier channels (tens) need
        // the levels' fp32 accuracy, not fp16's 2^-12
        const float h0 = __half2float(__float2half_rn(lo)), h1 = __half2float(__float2half_rn(hi));
        lutV[i] = make_uint2(h2bits(h0, h1), h2bits(lo - h0, hi - h1));
    }
    // 2-bit keys: stored code (n, m) = (negative, larger magnitude) has level
    // (1 - 2n)(c_0 + m (c_1 - c_0)); the key side of the product is then two
    // exact planes, s = +-1 and 2 s m in {0, +-2}, and the constants c_0 and
    // (c_1 - c_0)/2 ride on the query operand, scaled by 2^kexp into [0.5, 1)
    // so that their fp16 hi + lo split keeps its precision.
    float plane_f[2] = {1.f, 1.f}, kscale = 1.f;
    if (KB == 2 && !FR) {
        const float c0 = a.k_lv[0], c1 = a.k_lv[1];
        int e2;
        frexpf(fmaxf(fabsf(c0), fabsf(0.5f * (c1 - c0))), &e2);
        plane_f[0] = ldexpf(c0, -e2);
        plane_f[1] = ldexpf(0.5f * (c1 - c0), -e2);
        kscale = ldexpf(1.f, e2);
    }
    {
        const float qs = 0.08838834764831845f * 1.4426950408889634f;   // 1/sqrt(128) * log2(e)
        for (int i = tid; i < NT * NKS * 32; i += 128) {
            const int ln = i & 31, ks = (i >> 5) % NKS, nt = (i >> 5) / NKS;
            const int gg = ln >> 2, tt = ln & 3;
            const int hd = 4 * nt + (gg >> 1);
            const bool lo_part = (gg & 1) != 0;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (hd < G) {
                const float *src = ks < QK0 ? a.qr + (row0 + hd) * 128 : a.w + (row0 + hd) * 128;
                int c[4];
                float f = 1.f;
                if (ks >= QK0) {
                    const int j = 2 * (ks - QK0);
                    c[0] = 32 * tt + j; c[1] = 32 * tt + j + 16; c[2] = 32 * tt + j + 1; c[3] = 32 * tt + j + 17;
                } else if (FR) {
                    // half ks / 4, coordinates 16 (ks % 4) + 4 tt .. + 3 of that half
                    const int base = 64 * (ks >> 2) + 16 * (ks & 3) + 4 * tt;
                    c[0] = base; c[1] = base + 1; c[2] = base + 2; c[3] = base + 3;
                } else if (KB == 2) {
                    // plane k-step kk: word kk / 4 of the thread's 32 coordinates, pair
                    // i0 = 2 (kk % 4): coordinates (i0, i0 + 8) then (i0 + 1, i0 + 9)
                    const int kk = ks & 7;
                    const int base = 32 * tt + 16 * (kk >> 2) + 2 * (kk & 3);
                    c[0] = base; c[1] = base + 8; c[2] = base + 1; c[3] = base + 9;
                    f = plane_f[ks >> 3];
                } else {
                    const int base = 32 * tt + 4 * ks;
                    c[0] = base; c[1] = base + 1; c[2] = base + 2; c[3] = base + 3;
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float x = src[c[k]] * qs * f;
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

    const uint32_t vlane_off = uint32_t(lane & (VC - 1)) * 8u;     // this lane's value-table copy
    const uint32_t klane_off = uint32_t(lane & (KC - 1)) * 8u;     // this lane's key-table copy
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
                        const uint2 bb = sB[(nt * NKS + ks) * 32 + lane];
                        mma16816(accM[nt], A, bb.x, bb.y);
                    }
                }
            } else {
                const uint8_t *kcb = pg + L.kc_off;
                if constexpr (PL) {
                    // tokens g, g + 8: radii at the level-2 nodes 8t .. 8t + 7 (the subtree of
                    // level-5 node t), then per k-step the two pairs 16t + 2ks, + 1
                    float r2[2][8];
                    uint32_t c2w[2];                           // level-2 slots 8t .. 8t + 7
                    uint2 c1w[2];                              // level-1 codes of pairs 16t .. 16t + 15
#pragma unroll
                    for (int ri = 0; ri < 2; ++ri) {
                        const int tok = pr + g + 8 * ri;
                        c1w[ri] = *reinterpret_cast<const uint2 *>(kcb + tok * L.kc_bpt + 8 * t);
                        const uint4 hq = *reinterpret_cast<const uint4 *>(pg + L.kc2_off + tok * L.kc2_bpt);
                        // slot s in word s / 16: levels 7 .. 4 (slots 48 ..) in word 3, level 3 in word 2
                        auto fld = [](uint32_t w, int sl) { return (w >> (2 * (sl & 15))) & 3u; };
                        // cos / sin of the centre of a level-l angle code
                        auto cs = [&](int l, uint32_t k, int child) { return ptk[48 + 12 * (l - 2) + (child ? 8 : 4) + k]; };
                        const float r6 = cs(7, fld(hq.w, 62), (t >> 1) & 1);
                        const float r5 = r6 * cs(6, fld(hq.w, 60 + (t >> 1)), t & 1);
                        const uint32_t k5 = fld(hq.w, 56 + t);
                        float r3[4];
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float r4 = r5 * cs(5, k5, j);
                            const uint32_t k4 = fld(hq.w, 48 + 2 * t + j);
                            r3[2 * j] = r4 * cs(4, k4, 0);
                            r3[2 * j + 1] = r4 * cs(4, k4, 1);
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t k3 = fld(hq.z, 32 + 4 * t + j);
                            r2[ri][2 * j] = r3[j] * cs(3, k3, 0);
                            r2[ri][2 * j + 1] = r3[j] * cs(3, k3, 1);
                        }
                        // level-2 slots 8t .. 8t + 7: word t / 2, bits 16 (t % 2) ..
                        c2w[ri] = ((t >> 1) ? hq.y : hq.x) >> (16 * (t & 1)) & 0xFFFFu;
                    }
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        uint32_t Ah[4], Al[4];
#pragma unroll
                        for (int ri = 0; ri < 2; ++ri) {
                            const uint32_t k2 = (c2w[ri] >> (2 * ks)) & 3u;
                            const float ra = r2[ri][ks] * ptk[48 + 4 + k2], rb = r2[ri][ks] * ptk[48 + 8 + k2];
                            // level-1 codes of pairs 16t + 2ks, + 1
                            const uint32_t cw = ks < 4 ? c1w[ri].x : c1w[ri].y;
                            const uint32_t ka = (cw >> (8 * (ks & 3))) & 15u, kb = (cw >> (8 * (ks & 3) + 4)) & 15u;
                            const float y0 = ra * ptk[16 + ka], y1 = ra * ptk[32 + ka];
                            const float y2 = rb * ptk[16 + kb], y3 = rb * ptk[32 + kb];
                            const uint32_t h01 = h2bits(y0, y1), h23 = h2bits(y2, y3);
                            const float2 f01 = __half22float2(*reinterpret_cast<const __half2 *>(&h01));
                            const float2 f23 = __half22float2(*reinterpret_cast<const __half2 *>(&h23));
                            Ah[ri] = h01;                              // a0 (row g) / a1 (row g + 8)
                            Ah[2 + ri] = h23;                          // a2 / a3
                            Al[ri] = h2bits(y0 - f01.x, y1 - f01.y);
                            Al[2 + ri] = h2bits(y2 - f23.x, y3 - f23.y);
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 bb = sB[(nt * NKS + ks) * 32 + lane];
                            mma16816(accM[nt], Ah, bb.x, bb.y);
                            mma16816(accM[nt], Al, bb.x, bb.y);
                        }
                    }
                } else if constexpr (FR) {
                    // first half: KB-bit codes of coordinates 0 .. 63 (3 bits: a 2-bit magnitude
                    // array and a sign array); second half: (KB - 1)-bit codes of 64 .. 127.
                    // K-step ks covers coordinates 16 (ks % 4) + 4t .. + 3 of half ks / 4: pair
                    // (4t, 4t + 1) for a0 / a1, (4t + 2, 4t + 3) for a2 / a3.
                    const int ta = pr + g, tb2 = pr + g + 8;
                    const uint4 m0 = *reinterpret_cast<const uint4 *>(kcb + ta * L.kc_bpt);
                    const uint4 m1 = *reinterpret_cast<const uint4 *>(kcb + tb2 * L.kc_bpt);
                    uint2 h0 = make_uint2(0u, 0u), h1 = make_uint2(0u, 0u);
                    if constexpr (KB == 3) {
                        h0 = *reinterpret_cast<const uint2 *>(pg + L.kh_off + ta * L.kh_bpt);
                        h1 = *reinterpret_cast<const uint2 *>(pg + L.kh_off + tb2 * L.kh_bpt);
                    }
                    const uint8_t *kc2 = pg + L.kc2_off;
                    uint4 n0, n1;                              // second half: 2-bit (16 B) or 1-bit (8 B)
                    if constexpr (KB == 3) {
                        n0 = *reinterpret_cast<const uint4 *>(kc2 + ta * L.kc2_bpt);
                        n1 = *reinterpret_cast<const uint4 *>(kc2 + tb2 * L.kc2_bpt);
                    } else {
                        const uint2 x0 = *reinterpret_cast<const uint2 *>(kc2 + ta * L.kc2_bpt);
                        const uint2 x1 = *reinterpret_cast<const uint2 *>(kc2 + tb2 * L.kc2_bpt);
                        n0 = make_uint4(x0.x, x0.y, 0u, 0u);
                        n1 = make_uint4(x1.x, x1.y, 0u, 0u);
                    }
                    const uint32_t mw0[4] = {m0.x, m0.y, m0.z, m0.w}, mw1[4] = {m1.x, m1.y, m1.z, m1.w};
                    const uint32_t hw0[2] = {h0.x, h0.y}, hw1[2] = {h1.x, h1.y};
                    const uint32_t nw0[4] = {n0.x, n0.y, n0.z, n0.w}, nw1[4] = {n1.x, n1.y, n1.z, n1.w};
                    // pair-table indices of pairs a0 (low) and a2 (high) of one token
                    auto idx2 = [&](uint32_t byte, uint32_t &lo, uint32_t &hi) { lo = byte & 15u; hi = byte >> 4; };
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const int kq = ks & 3;
                        uint32_t i0, i2, j0, j2;                 // tokens g, g + 8
                        uint2 v[4];
                        if (ks < 4) {
                            // 2-bit fields (KB = 3: magnitudes; KB = 2: the codes): byte 4 kq + t
                            const uint32_t b0 = (mw0[kq] >> (8 * t)) & 0xFFu, b1 = (mw1[kq] >> (8 * t)) & 0xFFu;
                            idx2(b0, i0, i2);
                            idx2(b1, j0, j2);
                            if constexpr (KB == 3) {
                                // sign bits 16 kq + 4t .. + 3: word kq / 2, bit 16 (kq % 2) + 4t
                                const int sh = 16 * (kq & 1) + 4 * t;
                                const uint32_t s0 = (hw0[kq >> 1] >> sh) & 15u, s1 = (hw1[kq >> 1] >> sh) & 15u;
                                i0 |= (s0 & 3u) << 4; i2 |= (s0 >> 2) << 4;
                                j0 |= (s1 & 3u) << 4; j2 |= (s1 >> 2) << 4;
                            }
                            v[0] = lutK[i0 * KC + (lane & (KC - 1))];
                            v[2] = lutK[i2 * KC + (lane & (KC - 1))];
                            v[1] = lutK[j0 * KC + (lane & (KC - 1))];
                            v[3] = lutK[j2 * KC + (lane & (KC - 1))];
                        } else {
                            if constexpr (KB == 3) {
                                // 2-bit codes: byte 4 kq + t
                                const uint32_t b0 = (nw0[kq] >> (8 * t)) & 0xFFu, b1 = (nw1[kq] >> (8 * t)) & 0xFFu;
                                idx2(b0, i0, i2);
                                idx2(b1, j0, j2);
                            } else {
                                // 1-bit codes: bits 16 kq + 4t .. + 3
                                const int sh = 16 * (kq & 1) + 4 * t;
                                const uint32_t b0 = (nw0[kq >> 1] >> sh) & 15u, b1 = (nw1[kq >> 1] >> sh) & 15u;
                                i0 = b0 & 3u; i2 = b0 >> 2;
                                j0 = b1 & 3u; j2 = b1 >> 2;
                            }
                            v[0] = lutK2[i0 * kFrKC2 + (lane & (kFrKC2 - 1))];
                            v[2] = lutK2[i2 * kFrKC2 + (lane & (kFrKC2 - 1))];
                            v[1] = lutK2[j0 * kFrKC2 + (lane & (kFrKC2 - 1))];
                            v[3] = lutK2[j2 * kFrKC2 + (lane & (kFrKC2 - 1))];
                        }
                        uint32_t Ah[4], Al[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            Ah[r] = v[r].x;
                            Al[r] = v[r].y;
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 bb = sB[(nt * NKS + ks) * 32 + lane];
                            mma16816(accM[nt], Ah, bb.x, bb.y);
                            mma16816(accM[nt], Al, bb.x, bb.y);
                        }
                    }
                } else if constexpr (KB == 2) {
                    // 2-bit codes of tokens g and g + 8 for coordinates [32t, 32t + 32): two words
                    // each; coordinate i of a word sits at bits 2i (magnitude) and 2i + 1 (sign)
                    const uint2 u0 = *reinterpret_cast<const uint2 *>(kcb + (pr + g) * 32 + 8 * t);
                    const uint2 u1 = *reinterpret_cast<const uint2 *>(kcb + (pr + g + 8) * 32 + 8 * t);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t w0 = (ks >> 2) ? u0.y : u0.x, w1 = (ks >> 2) ? u1.y : u1.x;
                        const int sh = 14 - 4 * (ks & 3);       // coordinate i0 -> bits 14, 15 (and 30, 31)
                        uint32_t x[4];
                        x[0] = w0 << sh;
                        x[1] = w1 << sh;
                        x[2] = w0 << (sh - 2);
                        x[3] = w1 << (sh - 2);
                        uint32_t As[4], Am[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            As[r] = (x[r] & 0x80008000u) | 0x3C003C00u;   // +-1
                            Am[r] = x[r] & 0xC000C000u;                    // 0 or +-2
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 bs = sB[(nt * NKS + ks) * 32 + lane];
                            const uint2 bm = sB[(nt * NKS + 8 + ks) * 32 + lane];
                            mma16816(accM[nt], As, bs.x, bs.y);
                            mma16816(accM[nt], Am, bm.x, bm.y);
                        }
                    }
                } else {
                    // 4-bit codes of tokens g and g + 8 for coordinates [32t, 32t + 32)
                    const uint4 u0 = *reinterpret_cast<const uint4 *>(kcb + (pr + g) * 64 + 16 * t);
                    const uint4 u1 = *reinterpret_cast<const uint4 *>(kcb + (pr + g + 8) * 64 + 16 * t);
                    const uint32_t kc0[4] = {u0.x, u0.y, u0.z, u0.w}, kc1[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        // bytes 2ks, 2ks+1 of the thread's 16 code bytes: coordinate pairs
                        const uint32_t w0 = kc0[ks >> 1], w1 = kc1[ks >> 1];
                        const int bp = 2 * (ks & 1);
                        uint2 v[4];
                        v[0] = lds_at<uint2>(lutK, field_offset<8, KC * 8>(w0, bp, klane_off));
                        v[2] = lds_at<uint2>(lutK, field_offset<8, KC * 8>(w0, bp + 1, klane_off));
                        v[1] = lds_at<uint2>(lutK, field_offset<8, KC * 8>(w1, bp, klane_off));
                        v[3] = lds_at<uint2>(lutK, field_offset<8, KC * 8>(w1, bp + 1, klane_off));
                        uint32_t Ah[4], Al[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            Ah[r] = v[r].x;
                            Al[r] = v[r].y;
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 bb = sB[(nt * NKS + ks) * 32 + lane];
                            mma16816(accM[nt], Ah, bb.x, bb.y);
                            mma16816(accM[nt], Al, bb.x, bb.y);
                        }
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
                        const uint2 bb = sB[(nt * NKS + QK0 + ks) * 32 + lane];
                        mma16816(accQ[nt], A, bb.x, bb.y);
                    }
                }
            }
            // FP8 keys store sqrt(d) u: their estimate carries an extra 1/sqrt(d)
            const float nsc = FP8 ? 0.08838834764831845f : kscale;
            const float nk0 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kn_off + (pr + g) * 2)) * nsc;
            const float nk1 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kn_off + (pr + g + 8) * 2)) * nsc;
            const float rk0 = FP8 ? 0.f : h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kr_off + (pr + g) * 2)) * cq;
            const float rk1 = FP8 ? 0.f : h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.kr_off + (pr + g + 8) * 2)) * cq;
            const float nv0 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.vn_off + (pr + g) * 2));
            const float nv1 = h2f_bits(*reinterpret_cast<const uint16_t *>(pg + L.vn_off + (pr + g + 8) * 2));
            const bool ok0 = tok0 + g < nv, ok1 = tok0 + g + 8 < nv;
            // ---------------- online softmax (log2 units) for heads t and 4 + t
            uint32_t pk[NT];           // half2(P'[token g][h], P'[token g+8][h])
            uint32_t pk_lo = 0;        // one head tile: P' - fp16(P') for the spare columns
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
                const float q0 = ok0 ? p0 * nv0 : 0.f, q1 = ok1 ? p1 * nv1 : 0.f;
                pk[nt] = h2bits(q0, q1);
                if (NT == 1) {
                    const float2 hq = __half22float2(*reinterpret_cast<const __half2 *>(&pk[nt]));
                    pk_lo = h2bits(q0 - hq.x, q1 - hq.y);
                }
            }
            // ---------------- P^T fragment: head column g, tokens 2t, 2t+1 (+8)
            uint32_t b0, b1;
            {
                const int src0 = 4 * (2 * t) + (g & 3), src1 = 4 * (2 * t + 1) + (g & 3);
                uint32_t v0 = __shfl_sync(kFull, pk[0], src0), v1 = __shfl_sync(kFull, pk[0], src1);
                if (NT > 1) {
                    const uint32_t u0 = __shfl_sync(kFull, pk[NT - 1], src0), u1 = __shfl_sync(kFull, pk[NT - 1], src1);
                    if (g >= 4) { v0 = u0; v1 = u1; }
                } else {
                    // one head tile: columns 4..7 carry the low parts of columns 0..3
                    const uint32_t u0 = __shfl_sync(kFull, pk_lo, src0), u1 = __shfl_sync(kFull, pk_lo, src1);
                    if (g >= 4) { v0 = u0; v1 = u1; }
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
                // most tiles leave every running maximum unchanged: skip the rescale then
                if (__any_sync(kFull, ah[0] != 1.f || ah[1] != 1.f)) {
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        O[mt][0] *= ah[0]; O[mt][1] *= ah[1]; O[mt][2] *= ah[0]; O[mt][3] *= ah[1];
                    }
                }
            }
            // ---------------- values: thread coordinates [16g, 16g + 16), tokens 2t, 2t+1, 2t+8, 2t+9
            {
                const int ta = pr + 2 * t, tb = ta + 1, tc = ta + 8, td = ta + 9;
                if constexpr (PL) {
                    // tokens 2t, 2t + 1, 2t + 8, 2t + 9: radii of pairs 8g .. 8g + 7 (the subtree of
                    // level-4 node g) as fp16 hi + lo pairs per token, then regrouped per
                    // coordinate into the V^T fragments
                    uint32_t ph[4][8], pl[4][8];
                    const int toks[4] = {ta, tb, tc, td};
                    auto cs = [&](int l, uint32_t k, int child) { return ptv[48 + 12 * (l - 2) + (child ? 8 : 4) + k]; };
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int tok = toks[u];
                        const uint32_t c1 = *reinterpret_cast<const uint32_t *>(pg + L.vc_off + tok * L.vc_bpt + 4 * g);
                        const uint4 hq = *reinterpret_cast<const uint4 *>(pg + L.vc2_off + tok * L.vc2_bpt);
                        // slots 48 .. 63 (levels 7 .. 4) in word 3, level 3 in word 2, the thread's
                        // level-2 slots 4g .. 4g + 3 in word g / 4
                        auto fld = [](uint32_t w, int sl) { return (w >> (2 * (sl & 15))) & 3u; };
                        const uint32_t w2 = (g >> 2) ? hq.y : hq.x;
                        const float r6 = cs(7, fld(hq.w, 62), (g >> 2) & 1);
                        const float r5 = r6 * cs(6, fld(hq.w, 60 + (g >> 2)), (g >> 1) & 1);
                        const float r4 = r5 * cs(5, fld(hq.w, 56 + (g >> 1)), g & 1);
                        const uint32_t k4 = fld(hq.w, 48 + g);
#pragma unroll
                        for (int c3 = 0; c3 < 2; ++c3) {
                            const float r3 = r4 * cs(4, k4, c3);
                            const uint32_t k3 = fld(hq.z, 32 + 2 * g + c3);
#pragma unroll
                            for (int c2 = 0; c2 < 2; ++c2) {
                                const float r2 = r3 * cs(3, k3, c2);
                                const uint32_t k2 = fld(w2, 4 * g + 2 * c3 + c2);
#pragma unroll
                                for (int c1b = 0; c1b < 2; ++c1b) {
                                    const int j = 4 * c3 + 2 * c2 + c1b;         // pair 8g + j
                                    const float r1 = r2 * cs(2, k2, c1b);
                                    const uint32_t kt = (c1 >> (4 * j)) & 15u;
                                    const float y0 = r1 * ptv[16 + kt], y1 = r1 * ptv[32 + kt];
                                    const uint32_t hh = h2bits(y0, y1);
                                    const float2 hf = __half22float2(*reinterpret_cast<const __half2 *>(&hh));
                                    ph[u][j] = hh;
                                    pl[u][j] = h2bits(y0 - hf.x, y1 - hf.y);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {              // pair 8g + mt: coordinates 16g + 2mt, + 1
                        const uint32_t Ah[4] = {prmt(ph[0][mt], ph[1][mt], 0x5410), prmt(ph[0][mt], ph[1][mt], 0x7632),
                                                prmt(ph[2][mt], ph[3][mt], 0x5410), prmt(ph[2][mt], ph[3][mt], 0x7632)};
                        const uint32_t Al[4] = {prmt(pl[0][mt], pl[1][mt], 0x5410), prmt(pl[0][mt], pl[1][mt], 0x7632),
                                                prmt(pl[2][mt], pl[3][mt], 0x5410), prmt(pl[2][mt], pl[3][mt], 0x7632)};
                        mma16816(O[mt], Ah, b0, b1);
                        mma16816(O[mt], Al, b0, b1);
                    }
                } else if constexpr (FR) {
                    // first half: 4-bit codes of coordinates [8g, 8g + 8), word g of each token's
                    // first-half array; MMAs 0 .. 3 (rows g / g + 8: coordinates 8g + 2mt, + 1)
                    const uint8_t *vc = pg + L.vc_off;
                    const uint32_t wa = *reinterpret_cast<const uint32_t *>(vc + ta * L.vc_bpt + 4 * g);
                    const uint32_t wb = *reinterpret_cast<const uint32_t *>(vc + tb * L.vc_bpt + 4 * g);
                    const uint32_t wc = *reinterpret_cast<const uint32_t *>(vc + tc * L.vc_bpt + 4 * g);
                    const uint32_t wd = *reinterpret_cast<const uint32_t *>(vc + td * L.vc_bpt + 4 * g);
                    const uint32_t eAB = (wa & 0x0F0F0F0Fu) | ((wb << 4) & 0xF0F0F0F0u);
                    const uint32_t oAB = ((wa >> 4) & 0x0F0F0F0Fu) | (wb & 0xF0F0F0F0u);
                    const uint32_t eCD = (wc & 0x0F0F0F0Fu) | ((wd << 4) & 0xF0F0F0F0u);
                    const uint32_t oCD = ((wc >> 4) & 0x0F0F0F0Fu) | (wd & 0xF0F0F0F0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint2 v[4];
                        v[0] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(eAB, k, vlane_off));
                        v[1] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(oAB, k, vlane_off));
                        v[2] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(eCD, k, vlane_off));
                        v[3] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(oCD, k, vlane_off));
                        const uint32_t Ah[4] = {v[0].x, v[1].x, v[2].x, v[3].x};
                        const uint32_t Al[4] = {v[0].y, v[1].y, v[2].y, v[3].y};
                        mma16816(O[k], Ah, b0, b1);
                        mma16816(O[k], Al, b0, b1);
                    }
                    // second half: 3-bit codes of coordinates 64 + [8g, 8g + 8): 2-bit magnitudes
                    // (half-word g) and signs (byte g); MMAs 4 .. 7
                    const uint8_t *vc2 = pg + L.vc2_off, *vh2 = pg + L.vh2_off;
                    const uint32_t xa = *reinterpret_cast<const uint16_t *>(vc2 + ta * L.vc2_bpt + 2 * g);
                    const uint32_t xb = *reinterpret_cast<const uint16_t *>(vc2 + tb * L.vc2_bpt + 2 * g);
                    const uint32_t xc = *reinterpret_cast<const uint16_t *>(vc2 + tc * L.vc2_bpt + 2 * g);
                    const uint32_t xd = *reinterpret_cast<const uint16_t *>(vc2 + td * L.vc2_bpt + 2 * g);
                    const uint32_t zAB = uint32_t(vh2[ta * L.vh2_bpt + g]) | (uint32_t(vh2[tb * L.vh2_bpt + g]) << 16);
                    const uint32_t zCD = uint32_t(vh2[tc * L.vh2_bpt + g]) | (uint32_t(vh2[td * L.vh2_bpt + g]) << 16);
                    const uint32_t fAB = (xa & 0x3333u) | ((xb << 2) & 0xCCCCu);
                    const uint32_t gAB = ((xa >> 2) & 0x3333u) | (xb & 0xCCCCu);
                    const uint32_t fCD = (xc & 0x3333u) | ((xd << 2) & 0xCCCCu);
                    const uint32_t gCD = ((xc >> 2) & 0x3333u) | (xd & 0xCCCCu);
                    const uint32_t v2off = uint32_t(lane & (kFrVC2 - 1)) * 8u;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int e0 = 2 * k, e1 = 2 * k + 1;
                        const uint32_t z[4] = {(zAB << (15 - e0)) & 0x80008000u, (zAB << (15 - e1)) & 0x80008000u,
                                               (zCD << (15 - e0)) & 0x80008000u, (zCD << (15 - e1)) & 0x80008000u};
                        uint2 v[4];
                        v[0] = lds_at<uint2>(lutV2, field_offset<4, kFrVC2 * 8>(fAB, k, v2off));
                        v[1] = lds_at<uint2>(lutV2, field_offset<4, kFrVC2 * 8>(gAB, k, v2off));
                        v[2] = lds_at<uint2>(lutV2, field_offset<4, kFrVC2 * 8>(fCD, k, v2off));
                        v[3] = lds_at<uint2>(lutV2, field_offset<4, kFrVC2 * 8>(gCD, k, v2off));
                        uint32_t Ah[4], Al[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) { Ah[r] = v[r].x ^ z[r]; Al[r] = v[r].y ^ z[r]; }
                        mma16816(O[4 + k], Ah, b0, b1);
                        mma16816(O[4 + k], Al, b0, b1);
                    }
                } else if (VB == 4) {
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
                            uint2 v[4];
                            v[0] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(eAB, k, vlane_off));
                            v[1] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(oAB, k, vlane_off));
                            v[2] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(eCD, k, vlane_off));
                            v[3] = lds_at<uint2>(lutV, field_offset<8, VC * 8>(oCD, k, vlane_off));
                            const uint32_t Ah[4] = {v[0].x, v[1].x, v[2].x, v[3].x};
                            const uint32_t Al[4] = {v[0].y, v[1].y, v[2].y, v[3].y};
                            mma16816(O[mt], Ah, b0, b1);
                            mma16816(O[mt], Al, b0, b1);
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
                        const uint32_t z[4] = {(zAB << (15 - e0)) & 0x80008000u, (zAB << (15 - e1)) & 0x80008000u,
                                               (zCD << (15 - e0)) & 0x80008000u, (zCD << (15 - e1)) & 0x80008000u};
                        uint2 v[4];
                        v[0] = lds_at<uint2>(lutV, field_offset<4, VC * 8>(eAB, mt, vlane_off));
                        v[1] = lds_at<uint2>(lutV, field_offset<4, VC * 8>(oAB, mt, vlane_off));
                        v[2] = lds_at<uint2>(lutV, field_offset<4, VC * 8>(eCD, mt, vlane_off));
                        v[3] = lds_at<uint2>(lutV, field_offset<4, VC * 8>(oCD, mt, vlane_off));
                        uint32_t Ah[4], Al[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) { Ah[r] = v[r].x ^ z[r]; Al[r] = v[r].y ^ z[r]; }
                        mma16816(O[mt], Ah, b0, b1);
                        mma16816(O[mt], Al, b0, b1);
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
            const int hd = NT == 1 ? ((2 * t + c) & 3) : 2 * t + c;   // one tile: column 4 + h is head h
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
        // FR: MMAs 0 .. 3 hold coordinates 8g + 2mt, + 1; 4 .. 7 the same of the second half
        const int c0 = FR ? 64 * (mt >> 2) + 8 * g + 2 * (mt & 3) : 16 * g + 2 * mt;
        ow[(2 * t) * 128 + c0] = O[mt][0] * scale_w[0];
        ow[(2 * t + 1) * 128 + c0] = O[mt][1] * scale_w[1];
        ow[(2 * t) * 128 + c0 + 1] = O[mt][2] * scale_w[0];
        ow[(2 * t + 1) * 128 + c0 + 1] = O[mt][3] * scale_w[1];
    }
    __syncthreads();
    const int64_t pbase = (int64_t(grp) * a.n_splits + split) * G;
    for (int i = tid; i < G * 128; i += 128) {
        float o = ((oo[i] + oo[1024 + i]) + oo[2048 + i]) + oo[3072 + i];
        if (NT == 1) o += ((oo[512 + i] + oo[1536 + i]) + oo[2560 + i]) + oo[3584 + i];
        a.part_o[pbase * 128 + i] = o;
    }
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

template <int KB, int VB, int NT, bool FR = false, bool PL = false>
size_t dec_smem(int page_bytes) {
    constexpr int KE = PL ? 0 : key_entries<KB, FR>(), VE = PL ? 0 : (VB == 4 ? 256 : 16);
    // the stage area also holds the final merge: 64 + 4 x 8 x 128 floats
    constexpr int kNS = PL ? 3 : page_stages<KB, FR>();
    size_t stages = size_t(kNS) * page_bytes;
    if (stages < (64 + 4 * 8 * 128) * 4) stages = (64 + 4 * 8 * 128) * 4;
    const size_t fr = FR ? size_t(key_entries2<KB, FR>()) * kFrKC2 * 8 + size_t(16) * kFrVC2 * 8 : 0;
    return size_t(KE) * (FR ? kFrKC : key_copies<KB>()) * 8 + size_t(VE) * val_copies<VB>() * 8 + fr +
           size_t(NT) * query_ksteps<KB, FR>() * 32 * 8 + (PL ? 2 * 136 * 4 : 0) +
           stages + (2 * kNS + 1) * 8 + kNS * 4 + 4 + 64;
}


// Blocks of one instantiation resident per SM, from the occupancy calculator
// (registers, shared memory and the 128-thread block).
// The kernel only covers d = 128 with 64-token pages, so the page size (and
// the answer) is fixed per instantiation and computed once.
template <int KB, int VB, int NT, bool FR = false, bool PL = false>
int dec_resident(int page_bytes) {
    static std::atomic<int> cached{-1};
    const int c = cached.load();
    if (c >= 0) return c;
    const size_t smem = dec_smem<KB, VB, NT, FR, PL>(page_bytes);
    auto kern = dec128_kernel<KB, VB, NT, FR, PL>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 128, smem) != cudaSuccess) return 0;
    cached.store(n);
    return n;
}

template <int KB, int VB, int NT, bool FR = false, bool PL = false>
int run_dec(const Dec128Args &a, int n_groups, cudaStream_t st) {
    const size_t smem = dec_smem<KB, VB, NT, FR, PL>(a.L.page_bytes);
    auto kern = dec128_kernel<KB, VB, NT, FR, PL>;
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
// Fractional rates the tensor-core decode covers: keys 1.5 / 2.5 bits + QJL,
// values 3.5 bits.
bool dec128_frac_ok(const Layout &L) {
    return L.khalf && L.vhalf && L.kqjl && (L.ka_bits == 2 || L.ka_bits == 3) && L.va_bits == 4;
}
// Polar codes the tensor-core decode covers: keys with QJL and values.
bool dec128_polar_ok(const Layout &L) { return L.kpolar && L.vpolar && L.kqjl; }

int dec128_resident(const Layout &L, int G) {
    if (L.d != 128 || L.P != 64 || G > 8) return 0;
    const bool two = G > 4;
    const int pb = L.page_bytes;
    if (dec128_polar_ok(L))
        return two ? dec_resident<4, 4, 2, false, true>(pb) : dec_resident<4, 4, 1, false, true>(pb);
    if (dec128_frac_ok(L)) {
        if (L.ka_bits == 3) return two ? dec_resident<3, 4, 2, true>(pb) : dec_resident<3, 4, 1, true>(pb);
        return two ? dec_resident<2, 4, 2, true>(pb) : dec_resident<2, 4, 1, true>(pb);
    }
    if (!dec128_keys_ok(L) || !(L.vbits == 3 || L.vbits == 4)) return 0;
#define TQ_DEC_RES(K, V) \
    if (L.kbits == K && L.vbits == V) return two ? dec_resident<K, V, 2>(pb) : dec_resident<K, V, 1>(pb);
    TQ_DEC_RES(2, 4) TQ_DEC_RES(2, 3) TQ_DEC_RES(4, 4) TQ_DEC_RES(4, 3) TQ_DEC_RES(8, 4) TQ_DEC_RES(8, 3)
#undef TQ_DEC_RES
    return 0;
}

// Tensor-core attention for d = 128; returns -1 when the configuration is not
// covered (the caller then uses the general kernel).
int launch_dec128(const tq_params *kp, const tq_params *vp, const Layout &L, const float *qr, const float *w,
                  const AttnShape &s, int G, int n_groups, int n_splits, int split_len, const uint8_t *cache,
                  int64_t num_blocks, float *part_o, float *part_ml, float *logits, int64_t logits_stride,
                  uint32_t *status, cudaStream_t st) {
    if (L.d != 128 || L.P != 64 || G > 8) return -1;
    const bool frac = dec128_frac_ok(L), polar = dec128_polar_ok(L);
    if (!frac && !polar && (!dec128_keys_ok(L) || !(L.vbits == 3 || L.vbits == 4))) return -1;
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
    a.k_lv2 = kp->dev.lv2;
    a.v_lv2 = vp->dev.lv2;
    a.k_pt = kp->dev.polar;
    a.v_pt = vp->dev.polar;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.logits = logits;
    a.logits_stride = logits_stride;
    a.status = status;
    a.stall_polls = take_decode_stall();
    const bool two = G > 4;
    if (polar)
        return two ? run_dec<4, 4, 2, false, true>(a, n_groups, st) : run_dec<4, 4, 1, false, true>(a, n_groups, st);
    if (frac) {
        if (L.ka_bits == 3)
            return two ? run_dec<3, 4, 2, true>(a, n_groups, st) : run_dec<3, 4, 1, true>(a, n_groups, st);
        return two ? run_dec<2, 4, 2, true>(a, n_groups, st) : run_dec<2, 4, 1, true>(a, n_groups, st);
    }
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
