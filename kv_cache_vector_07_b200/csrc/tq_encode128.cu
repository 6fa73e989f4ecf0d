// Fused write path for head dimension 128 with bf16 inputs: one persistent
// kernel does the rotation, the Lloyd-Max codes, the residual and the QJL
// projection, with both dense steps on the tensor cores.
//
// Page "What is TurboQuant?", "Stage 1" (randomized Hadamard rotation, then
// per-coordinate Lloyd-Max codes, no per-block scale) and "Stage 2" (1-bit
// QJL projection of the residual); ai-work-lab overview, "QJL".
//
// Per tile of 128 vectors (one vector per TMEM lane):
//   TMA     x tile [128 x 128 bf16] -> shared memory (128-byte swizzle)
//   MMA 1   Y = X (H D)^T on tcgen05 (bf16, exact +-1 operand) -> TMEM;
//           y = Y / sqrt(128) = R x
//   threads (two per vector, 64 coordinates each) read Y from TMEM: norm
//           (each thread sums its own 64 coordinates by quarter; the pair
//           swaps quarter sums through shared memory and adds all four in a
//           fixed order, so both agree, and neither reads columns the other
//           is about to overwrite with its residual), bucketize (3- and
//           4-bit codebooks: a 16-cell rank table over C |y| / ||y||; 1- and
//           2-bit: the boundaries scaled by the norm), sign-magnitude codes
//           packed into the page, fp16 norm; for
//           QJL keys the residual r = y - nhat c[idx] (scaled by a power of
//           two) split into fp16 hi + lo, written back over the tile's own Y
//           columns, rho = fp16 ||r||
//   MMA 2   Z = (r_hi + r_lo) S^T on tcgen05 with the residual as the A operand
//           in tensor memory (fp16, S exact in fp16 except |S| < 2^-17); the
//           sign bits of Z go to the page.
// The block runs two independent groups of eight warps, each with its own
// TMEM (Y, Z), x stage and named barrier, on alternate key/value tile pairs,
// so one group's MMAs and loads overlap the other's arithmetic.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cfloat>
#include <cstring>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tc05.cuh"
#include "tq_dev.cuh"

namespace tq {

namespace {

constexpr int kRows = 128;
constexpr uint32_t kTile = 32768;          // one 128 x 128 16-bit tile
constexpr uint32_t SM_ROT_K = 0, SM_ROT_V = 32768, SM_S16 = 65536, SM_X = 98304;   // x: one stage per group
constexpr uint32_t SM_XR = SM_X + 2 * kTile;       // float [2 groups][2 halves][128] residual-norm partials
constexpr uint32_t SM_YN = SM_XR + 2048;          // float [2 groups][4 quarters][128] ||Y||^2 partials
constexpr uint32_t SM_BAR = SM_YN + 4096;         // barriers, TMEM address, level tables
constexpr uint32_t SM_TAB = SM_BAR + 256;          // magnitude-rank cell tables (keys, values)
constexpr uint32_t SM_LV2 = SM_TAB + 4 * 128;        // second-half level tables (fractional rates)
constexpr uint32_t SM_TOTAL = SM_LV2 + 64;
constexpr int kCells = 16;                         // cells of a rank table
constexpr uint32_t kPolls = 1u << 20;    // about a second of polling, then give up

// Magnitude-rank table of a 3- or 4-bit codebook.  With x = C |y| / ||y||
// (C a power of two, so the scaled thresholds X_k = C t_k are exact) and the
// unit cells [c, c + 1), c < 15, each cell holds at most one X_k: the rank
// is mu_lo(c) + [x >= X in the cell], x clamped to 15, where no threshold
// lies.  Entry c: {X in (c, c + 1) or a large value, mu_lo(c) = #{X_k <= c}}.
struct RankTable {
    float C;
    float2 cell[kCells];
};

struct Enc128Args {
    Layout L;
    RankTable k_tab, v_tab;            // first (or only) codebooks
    RankTable k_tab2, v_tab2;          // fractional rates: codebooks of coordinates 64 .. 127
    const float *k_lv, *v_lv;          // levels by stored code
    const float *k_bnd, *v_bnd;        // ascending boundaries
    const float *k_lv2, *v_lv2, *k_bnd2, *v_bnd2;   // fractional rates: second codebooks
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
//
// For B >= 3 the rank comes from the cell table instead of the thresholds:
// xs = C / ||Y|| (0 for a zero vector), tab = shared address of the table
// minus (0x4B000000 << 3), so that the bits of 2^23 + floor(x), shifted by
// three, index its 8-byte entries directly.
template <int B>
constexpr bool use_table() { return B == 3 || B == 4; }

template <int B, bool RESID>
__device__ __forceinline__ void quantize32(float (&y)[32], const float (&T)[7], float xs, uint32_t tab,
                                           const float *lvs, float nhs, uint32_t (&cw)[4], float &rr) {
#pragma unroll
    for (int k = 0; k < 4; ++k) cw[k] = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float Y = y[i];
        uint32_t s, mu;
        if constexpr (use_table<B>()) {
            s = __float_as_uint(Y + 0.0f) >> 31;        // -0.0 + 0.0 = +0.0: zero is non-negative
            const float x = fabsf(Y) * xs;
            const uint32_t off = __float_as_uint(__fadd_rz(fminf(x, float(kCells - 1)), 8388608.0f)) << 3;
            float tb;
            uint32_t mlo;
            asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(tb), "=r"(mlo) : "r"(tab + off));
            mu = mlo + (x >= tb ? 1u : 0u);
        } else {
            s = Y < 0.f ? 1u : 0u;
            mu = uint32_t(mag_rank<B>(fabsf(Y), T));
        }
        const uint32_t kap = (s << (B - 1)) | mu;
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

// Two groups of 8 warps; in a group, thread (row, h) owns vector row
// 32*(warp%4)+lane of the tile and its coordinates [64h, 64h + 64),
// h = (warp%8)/4 (TMEM lane slice warp % 4).  Group g owns TMEM columns
// [256g, 256g + 128) (Y, then the residual operand) and [256g + 128,
// 256g + 256) (Z).
// Fractional rates (KB2 != KB or VB2 != VB): coordinates 64 .. 127, which
// are exactly the quarters of the threads with h = 1, take the second
// codebook of KB2 (VB2) bits and the second code arrays of the page.
template <int KB, int VB, bool QJL, int KB2 = KB, int VB2 = VB>
__global__ void __launch_bounds__(512, 1)
encode128_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ Enc128Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = smem_raw;
    float *xr = reinterpret_cast<float *>(sm + SM_XR);
    float *yn = reinterpret_cast<float *>(sm + SM_YN);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SM_BAR);
    uint64_t *bar_const = bars, *bar_x = bars + 1, *bar_y = bars + 3, *bar_z = bars + 5;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sm + SM_BAR + 64);
    float *s_klv = reinterpret_cast<float *>(sm + SM_BAR + 128), *s_vlv = s_klv + 16;
    float *s_klv2 = reinterpret_cast<float *>(sm + SM_LV2), *s_vlv2 = s_klv2 + 8;
    constexpr bool FRAC_K = KB2 != KB, FRAC_V = VB2 != VB;

    constexpr bool DO_V = VB > 0;
    constexpr int PER = DO_V ? 2 : 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = warp >> 3, gw = warp & 7, gtid = tid & 255;
    const int row = 32 * (gw & 3) + lane, h = gw >> 2;
    if ((tc05::smem_u32(smem_raw) & 1023u) != 0) {       // the swizzled tiles need 1024-byte alignment
        if (tid == 0) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
        return;
    }
    // tile pairs of this group: 2 blockIdx.x + grp + k * 2 gridDim.x
    const int64_t first = 2 * int64_t(blockIdx.x) + grp, stride = 2 * int64_t(gridDim.x);
    const int64_t n_my = a.n_tiles > first ? (a.n_tiles - 1 - first) / stride + 1 : 0;
    const int64_t n_items = n_my * PER;
    bool timeout = false;

    if (warp == 0) {
        tc05::tmem_alloc(tmem_holder, 512);
        tc05::tmem_relinquish();
    }
    if (tid < 16) {
        s_klv[tid] = (KB != 8 && tid < (1 << (KB == 8 ? 1 : KB))) ? a.k_lv[tid] : 0.f;
        s_vlv[tid] = (DO_V && tid < (1 << (VB > 0 ? VB : 1))) ? a.v_lv[tid] : 0.f;
    } else if (tid < 16 + 4 * kCells) {
        const int t = (tid - 16) / kCells, c = (tid - 16) % kCells;
        const RankTable &rt = t == 0 ? a.k_tab : t == 1 ? a.v_tab : t == 2 ? a.k_tab2 : a.v_tab2;
        reinterpret_cast<float2 *>(sm + SM_TAB)[t * kCells + c] = rt.cell[c];
    } else if (tid < 16 + 4 * kCells + 16) {
        const int i = tid - 16 - 4 * kCells;
        if (i < 8) s_klv2[i] = (FRAC_K && i < (1 << KB2)) ? a.k_lv2[i] : 0.f;
        else s_vlv2[i - 8] = (FRAC_V && i - 8 < (1 << (VB2 > 0 ? VB2 : 1))) ? a.v_lv2[i - 8] : 0.f;
    }
    auto item_tile = [&](int64_t j) { return first + (j / PER) * stride; };
    auto item_is_v = [&](int64_t j) { return DO_V && (j % PER) == 1; };
    uint8_t *xst = sm + SM_X + grp * kTile;
    auto issue_x = [&](int64_t j) {                       // group issuer only
        tc05::mbar_expect_tx(&bar_x[grp], kTile);
        const void *tm = item_is_v(j) ? static_cast<const void *>(&tmV) : static_cast<const void *>(&tmK);
        const int y = int(item_tile(j) * kRows);
        tc05::tma_load_2d(xst, tm, 0, y, &bar_x[grp]);
        tc05::tma_load_2d(xst + 16384, tm, 64, y, &bar_x[grp]);
    };
    if (tid == 0) {
        tc05::mbar_init(bar_const, 1);
        for (int i = 0; i < 2; ++i) {
            tc05::mbar_init(&bar_x[i], 1);
            tc05::mbar_init(&bar_y[i], 1);
            tc05::mbar_init(&bar_z[i], 1);
        }
        tc05::fence_mbar_init();
        tc05::mbar_expect_tx(bar_const, kTile * (1 + (DO_V ? 1 : 0) + (QJL ? 1 : 0)));
        tc05::bulk_g2s(sm + SM_ROT_K, a.k_rot, kTile, bar_const);
        if (DO_V) tc05::bulk_g2s(sm + SM_ROT_V, a.v_rot, kTile, bar_const);
        if (QJL) tc05::bulk_g2s(sm + SM_S16, a.s16, kTile, bar_const);
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const uint32_t ycol = tmem + uint32_t(grp * 256), zcol = ycol + 128u;
    const uint32_t lane_base = uint32_t(32 * (gw & 3)) << 16;
    constexpr uint32_t idesc1 = tc05::idesc_bf16_f32(128, 128);
    constexpr uint32_t idesc2 = tc05::idesc_f16_f32(128, 128);

    auto issue_mma1 = [&](int64_t j) {                    // group issuer only
        if (!tc05::mbar_wait_bounded(&bar_x[grp], uint32_t(j & 1), kPolls)) timeout = true;
        tc05::fence_after_sync();
        const uint32_t xa = tc05::smem_u32(xst);
        const uint32_t rb = tc05::smem_u32(sm + (item_is_v(j) ? SM_ROT_V : SM_ROT_K));
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc05::mma_bf16(ycol, tc05::desc_kmajor_sw128(xa + c * 16384 + ks * 32),
                               tc05::desc_kmajor_sw128(rb + c * 16384 + ks * 32), idesc1, (c | ks) != 0);
        tc05::mma_commit(&bar_y[grp]);
    };
    // Z = r S^T: k-step s reads the residual of quarter s / 2 (hi at +0, lo at
    // +16 columns of the quarter, coordinates 16 (s % 2) .. at +8 (s % 2))
    auto issue_mma2 = [&]() {                             // group issuer only
        const uint32_t bs = tc05::smem_u32(sm + SM_S16);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int st = 0; st < 8; ++st)
                tc05::mma_f16_ts(zcol, ycol + uint32_t(32 * (st >> 1) + 16 * part + 8 * (st & 1)),
                                 tc05::desc_kmajor_sw128(bs + (st >> 2) * 16384 + (st & 3) * 32), idesc2,
                                 (part | st) != 0);
        tc05::mma_commit(&bar_z[grp]);
    };
    auto group_sync = [&]() { asm volatile("bar.sync %0, 256;" ::"r"(1 + grp) : "memory"); };

    if (gtid == 0 && n_items > 0) {
        if (!tc05::mbar_wait_bounded(bar_const, 0, kPolls)) timeout = true;
        issue_x(0);
        issue_mma1(0);
    }

    const float rs = 0.08838834764831845f;              // 1 / sqrt(128)
    const float sq = 11.313708498984761f;               // sqrt(128)
    int64_t pending_k = -1;                             // key tile whose MMA 2 is in flight
    uint32_t z_phase = 0;

    // the pending key tile is the current tile: its page is this item's
    auto sign_pass = [&](uint8_t *kpage, int kpos) {
        if (!tc05::mbar_wait_bounded(&bar_z[grp], z_phase, kPolls)) timeout = true;
        z_phase ^= 1u;
        tc05::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int q = 2 * h + c;
            uint32_t r[32];
            tc05::tmem_ld_32x32b_x32(zcol + lane_base + uint32_t(q * 32), r);
            tc05::tmem_wait_ld();
            // bit k = [z_k >= 0]: the complement of the float sign bit (z = -0.0
            // lies inside the zero-tolerance of the sign comparison)
            uint32_t neg = 0;                           // sign bits, coordinate k at bit k
#pragma unroll
            for (int k = 31; k >= 0; --k) neg = __funnelshift_l(r[k], neg, 1);
            if (kpage && !timeout)
                *reinterpret_cast<uint32_t *>(kpage + a.L.ks_off + kpos * a.L.ks_bpt + q * 4) = ~neg;
        }
        pending_k = -1;
    };

    uint8_t *page = nullptr;
    int pos = 0;
    for (int64_t j = 0; j < n_items; ++j) {
        const bool is_v = item_is_v(j);
        const int64_t tile = item_tile(j);
        // a tile's key item finds the row's page (its value item and sign
        // pass reuse it); the slot load overlaps the wait for Y
        if (!is_v) page = row_page(a, tile * kRows + row, &pos);
        if (!tc05::mbar_wait_bounded(&bar_y[grp], uint32_t(j & 1), kPolls)) timeout = true;
        tc05::fence_after_sync();
        // MMA 1 of this item has read the group's x stage: refill it
        if (gtid == 0 && j + 1 < n_items) issue_x(j + 1);

        // ||Y||^2 of the row: each thread sums its own two quarters (the
        // partner overwrites its quarters with the residual as soon as it has
        // its norm, so neither reads the other's columns); the quarter sums
        // meet in shared memory and both threads add them in the same order
        float *ynr = yn + grp * 512 + row;
        float y[32];                                    // the quarter being quantized: 2h first
        {
            uint32_t r0[32], r1[32];
            tc05::tmem_ld_32x32b_x32(ycol + lane_base + uint32_t(2 * h * 32), r0);
            tc05::tmem_ld_32x32b_x32(ycol + lane_base + uint32_t(2 * h * 32 + 32), r1);
            tc05::tmem_wait_ld();
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                p0 = fmaf(__uint_as_float(r0[i]), __uint_as_float(r0[i]), p0);
                p1 = fmaf(__uint_as_float(r0[i + 1]), __uint_as_float(r0[i + 1]), p1);
                p2 = fmaf(__uint_as_float(r1[i]), __uint_as_float(r1[i]), p2);
                p3 = fmaf(__uint_as_float(r1[i + 1]), __uint_as_float(r1[i + 1]), p3);
            }
            ynr[2 * h * 128] = p0 + p1;
            ynr[(2 * h + 1) * 128] = p2 + p3;
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(r0[i]);
        }
        // warps gw and gw + 4 hold the two halves of the same 32 rows
        asm volatile("bar.sync %0, 64;" ::"r"(3 + 4 * grp + (gw & 3)) : "memory");
        const float ns = sqrtf(((ynr[0] + ynr[128]) + ynr[256]) + ynr[384]);   // ||Y|| = sqrt(128) ||x||
        const float n = ns * rs;                                               // ||x||
        const uint16_t nh = f2h_bits(n);
        const float nhf = h2f_bits(nh);
        // this thread's quarters 2h, 2h + 1 use the second codebook of a fractional rate
        const bool second = h == 1 && (is_v ? FRAC_V : FRAC_K);
        const int bits = is_v ? (h ? VB2 : VB) : (h ? KB2 : KB);
        // residual scale 2^(12 - e), ||Y|| < 2^(e + 1): |r * scale| < 2^14
        int e = 0;
        if (ns > 0.f) e = ((__float_as_int(ns) >> 23) & 0xff) - 127;
        const float sc = __int_as_float(min(254, max(1, 127 + 12 - e)) << 23);
        float rr = 0.f;
        float T[7];
        if (!(is_v ? (h ? use_table<VB2>() : use_table<VB>()) : (h ? use_table<KB2>() : use_table<KB>()))) {
            const int nt = (1 << (bits - 1)) - 1;
            const float *bnd = second ? (is_v ? a.v_bnd2 : a.k_bnd2) : (is_v ? a.v_bnd : a.k_bnd);
#pragma unroll
            for (int k = 0; k < 7; ++k)
                T[k] = (k < nt && ns > 0.f && !(!is_v && KB == 8)) ? bnd[(1 << (bits - 1)) + k] * ns : FLT_MAX;
        }
        const RankTable &rtab = second ? (is_v ? a.v_tab2 : a.k_tab2) : (is_v ? a.v_tab : a.k_tab);
        const float xs = ns > 0.f ? rtab.C / ns : 0.f;
        const uint32_t tab = tc05::smem_u32(sm + SM_TAB + ((is_v ? 1 : 0) + (second ? 2 : 0)) * kCells * 8) -
                             (0x4B000000u << 3);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            const int q = 2 * h + c;
            if (c == 1) {                               // quarter 2h + 1, still unwritten by anyone
                uint32_t r[32];
                tc05::tmem_ld_32x32b_x32(ycol + lane_base + uint32_t(q * 32), r);
                tc05::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(r[i]);
            }
            if (!is_v && KB == 8) {
                // FP8 keys: e4m3(sqrt(d) y / n) = e4m3(Y / n)
                const float inv = n > 0.f ? 1.0f / n : 0.f;
                uint32_t w[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2)
                        acc |= uint32_t(__nv_cvt_float_to_fp8(y[4 * k + e2] * inv, __NV_SATFINITE, __NV_E4M3))
                               << (8 * e2);
                    w[k] = acc;
                }
                if (page) {
                    uint4 *dst = reinterpret_cast<uint4 *>(page + a.L.kc_off + pos * a.L.kc_bpt + q * 32);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            } else if (is_v) {
                if constexpr (DO_V) {
                    uint32_t cw[4];
                    bool done = false;
                    if constexpr (FRAC_V) {
                        if (second) {
                            quantize32<VB2, false>(y, T, xs, tab, s_vlv2, 0.f, cw, rr);
                            if (page) store_codes32<VB2>(page, pos, q - 2, a.L.vc2_off, a.L.vc2_bpt, a.L.vh2_off,
                                                         a.L.vh2_bpt, cw);
                            done = true;
                        }
                    }
                    if (!done) {
                        quantize32<DO_V ? VB : 1, false>(y, T, xs, tab, s_vlv, 0.f, cw, rr);
                        if (page) store_codes32<DO_V ? VB : 1>(page, pos, q, a.L.vc_off, a.L.vc_bpt, a.L.vh_off,
                                                                a.L.vh_bpt, cw);
                    }
                }
            } else {
                constexpr int KQ = KB == 8 ? 1 : KB;
                uint32_t cw[4];
                bool done = false;
                if constexpr (FRAC_K) {
                    if (second) {
                        quantize32<KB2, QJL>(y, T, xs, tab, s_klv2, sq * nhf, cw, rr);
                        if (page)
                            store_codes32<KB2>(page, pos, q - 2, a.L.kc2_off, a.L.kc2_bpt, a.L.kh2_off, a.L.kh2_bpt,
                                               cw);
                        done = true;
                    }
                }
                if (!done) {
                    quantize32<KQ, QJL>(y, T, xs, tab, s_klv, sq * nhf, cw, rr);
                    if (page) store_codes32<KQ>(page, pos, q, a.L.kc_off, a.L.kc_bpt, a.L.kh_off, a.L.kh_bpt, cw);
                }
                if constexpr (QJL) {
                    // residual (Y scale) x 2^(12 - e) as fp16 hi + lo over this quarter's Y columns
#pragma unroll
                    for (int hf2 = 0; hf2 < 2; ++hf2) {
                        uint32_t wh[8], wl[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float a0 = y[16 * hf2 + 2 * k] * sc, a1 = y[16 * hf2 + 2 * k + 1] * sc;
                            const __half2 hh2 = __floats2half2_rn(a0, a1);
                            const float2 hf = __half22float2(hh2);
                            const __half2 ll2 = __floats2half2_rn(a0 - hf.x, a1 - hf.y);
                            wh[k] = *reinterpret_cast<const uint32_t *>(&hh2);
                            wl[k] = *reinterpret_cast<const uint32_t *>(&ll2);
                        }
                        tc05::tmem_st_32x32b_x8(ycol + lane_base + uint32_t(q * 32 + 8 * hf2), wh);
                        tc05::tmem_st_32x32b_x8(ycol + lane_base + uint32_t(q * 32 + 16 + 8 * hf2), wl);
                    }
                }
            }
        }
        if (page && h == 0)
            *reinterpret_cast<uint16_t *>(page + (is_v ? a.L.vn_off : a.L.kn_off) + pos * 2) = nh;
        if (!is_v && QJL) {
            tc05::tmem_wait_st();
            xr[(grp * 2 + h) * 128 + row] = rr;
        }
        // sign bits of the key tile whose MMA 2 is in flight
        if (QJL && DO_V && is_v && pending_k >= 0) sign_pass(page, pos);

        tc05::fence_before_sync();
        group_sync();                                   // Y read (and the residual written) by all
        if (gtid == 0) {
            tc05::fence_after_sync();
            if (!is_v && QJL) issue_mma2();
            if (j + 1 < n_items) {
                // MMA 1 overwrites the residual MMA 2 reads
                if (!is_v && QJL && !tc05::mbar_wait_bounded(&bar_z[grp], z_phase, kPolls)) timeout = true;
                issue_mma1(j + 1);
            }
        }
        if (!is_v && QJL) {
            if (page && h == 0) {
                // rho = ||r|| = ||Y-scale residual|| / sqrt(128)
                const float rho = sqrtf(xr[(grp * 2) * 128 + row] + xr[(grp * 2 + 1) * 128 + row]) * rs;
                *reinterpret_cast<uint16_t *>(page + a.L.kr_off + pos * 2) = f2h_bits(rho);
            }
            pending_k = tile;
            if (!DO_V) sign_pass(page, pos);
        }
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

template <int KB, int VB, bool QJL, int KB2 = KB, int VB2 = VB>
int run(const CUtensorMap &mk, const CUtensorMap &mv, const Enc128Args &a, cudaStream_t st) {
    auto kern = encode128_kernel<KB, VB, QJL, KB2, VB2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SM_TOTAL));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (a.n_tiles + 1) / 2;          // two tile groups per block
    const int64_t grid = want < sms ? want : sms;
    kern<<<unsigned(grid), 512, SM_TOTAL, st>>>(mk, mv, a);
    return cudaGetLastError();
}

// Rank table of a 3- or 4-bit codebook (see RankTable) from its ascending
// boundaries; false if no power of two puts the largest threshold below the
// last cell with every gap between scaled thresholds at least one cell wide.
// Other widths need no table (an empty one is returned).
bool make_rank_table(int bits, const float *bounds, RankTable *t) {
    *t = RankTable{};
    if (bits != 3 && bits != 4) return true;
    const int L = 1 << bits, nt = L / 2 - 1;
    const float *th = bounds + L / 2;              // positive thresholds, ascending
    if (!(th[0] > 0.f)) return false;
    float C = 1.f;
    for (int i = 0; i < 40 && C * th[nt - 1] >= float(kCells - 1); ++i) C *= 0.5f;
    for (int i = 0; i < 40 && 2.f * C * th[nt - 1] < float(kCells - 1); ++i) C *= 2.f;
    if (!(C * th[nt - 1] < float(kCells - 1))) return false;
    for (int k = 0; k + 1 < nt; ++k)
        if (double(C * th[k + 1]) - double(C * th[k]) < 1.0) return false;
    t->C = C;
    for (int c = 0; c < kCells; ++c) {
        int mlo = 0;
        float tb = 3.0e38f;
        for (int k = 0; k < nt; ++k) {
            const float X = C * th[k];
            if (X <= float(c)) ++mlo;
            else if (X < float(c + 1)) tb = X;
        }
        float mlo_bits;
        std::memcpy(&mlo_bits, &mlo, sizeof mlo_bits);   // the rank rides in the float's bits
        t->cell[c] = make_float2(tb, mlo_bits);
    }
    return true;
}

// Widths of the two halves of a codebook (equal unless the rate is
// fractional) and the host boundaries of each.
struct Halves {
    int b1, b2;
    const float *bnd1, *bnd2;
};
Halves halves_of(const tq_params *p, bool half, int ka, int kb) {
    if (!p) return Halves{0, 0, nullptr, nullptr};
    if (!half) return Halves{p->bits, p->bits, p->h_bounds, p->h_bounds};
    return Halves{ka, kb, p->h_bounds, p->h_bounds + ((1 << ka) - 1)};
}

}  // namespace

// Returns -1 if this configuration is not handled by the fused kernel.
int launch_encode128(const tq_params *kp, const tq_params *vp, const Layout &L, const void *K, const void *V,
                     int64_t n_tokens, const int32_t *slots, uint8_t *cache, int64_t num_blocks, uint8_t *ws,
                     void *stream) {
    if (L.d != 128 || !kp->dev.rot_img) return -1;
    if (L.vbits > 0 && (!vp || !vp->dev.rot_img)) return -1;
    const int q = L.kqjl;
    const Halves hk = halves_of(kp, L.khalf, L.ka_bits, L.kb_bits);
    const Halves hv = halves_of(L.vbits > 0 ? vp : nullptr, L.vhalf, L.va_bits, L.vb_bits);
    const int kb = hk.b1, kb2 = hk.b2, vb = hv.b1, vb2 = hv.b2;
    Enc128Args a;
    a.L = L;
    a.k_lv = kp->dev.lv;
    a.k_bnd = kp->dev.bounds;
    a.k_rot = kp->dev.rot_img;
    a.s16 = kp->dev.s16_img;
    a.v_lv = vp ? vp->dev.lv : nullptr;
    a.v_bnd = vp ? vp->dev.bounds : nullptr;
    a.v_rot = vp ? vp->dev.rot_img : nullptr;
    a.k_lv2 = kp->dev.lv2;
    a.k_bnd2 = kp->dev.bounds2;
    a.v_lv2 = vp ? vp->dev.lv2 : nullptr;
    a.v_bnd2 = vp ? vp->dev.bounds2 : nullptr;
    if (!make_rank_table(kb, hk.bnd1, &a.k_tab) || !make_rank_table(kb2, hk.bnd2, &a.k_tab2) ||
        !make_rank_table(vb, hv.bnd1, &a.v_tab) || !make_rank_table(vb2, hv.bnd2, &a.v_tab2))
        return -1;
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
    if (L.khalf || L.vhalf) {
        // fractional rates (both halves of keys and values): b + 1 bits, then b
        if (!L.khalf || !L.vhalf || !q) return -1;
        if (kb == 3 && vb == 4) return run<3, 4, true, 2, 3>(mk, mv, a, st);
        if (kb == 2 && vb == 3) return run<2, 3, true, 1, 2>(mk, mv, a, st);
        if (kb == 4 && vb == 4) return run<4, 4, true, 3, 3>(mk, mv, a, st);
        if (kb == 3 && vb == 3) return run<3, 3, true, 2, 2>(mk, mv, a, st);
        return -1;
    }
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
