// Compressed inner-product search on the tensor cores (4-bit Lloyd-Max +
// QJL database; head dimension 128, 256, 512 or 1024; k <= 16).
//
// ai-work-lab overview, "QJL" and the vector-search paragraphs: the codec
// used for keys also scores database vectors, with no index preprocessing.
// Estimate of <q, x_t>:
//   nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1>.
//
// As a GEMM: D[256 queries x 256 vectors] = Qf[256 x 2d] Xf[256 x 2d]^T on
// tcgen05 as two M = 128 products sharing each dequantized chunk of Xf
// (fp16 operands, fp32 accumulators in TMEM, 256 columns per query half,
// all 512 columns):
//   Qf = 2^-e [R q | S R q] per query (fp16, prepared once, TMA-loaded one
//        64-feature chunk at a time; e makes the largest feature 1 <= |f| < 2
//        and the scores are multiplied back by 2^e);
//   Xf = [nhat c[code] | rho sqrt(pi/2)/m (2 s - 1)] per database vector,
//        dequantized by the worker warps (two threads per database row, 32
//        features each) into shared memory (128-byte swizzled K-major
//        tiles) while the previous chunk's MMAs run.
// Two warp roles synchronized by mbarriers, two stages: the 16 worker warps
// dequantize chunk g into stage g % 2 once the MMAs of chunk g - 2 are done;
// the issuer warp loads the query chunk by TMA into the same stage, waits
// for both operands and issues the chunk's MMAs.  At the end of a tile the
// workers queue the next tile's first chunk, then read the tile's estimates
// from TMEM (two threads per query, half of its 256 estimates each), keep a
// running top-k (ties to the lower index) and hand the accumulators back;
// a merge kernel combines the blocks' lists.
//
// Inside every 32-coordinate group the QJL features are in the order
// (p, p + 16) for feature positions (2p, 2p + 1), so a pair of sign bits
// becomes an fp16 pair with one shift and one mask.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tc05.cuh"
#include "tq_dev.cuh"

namespace tq {
namespace {

constexpr int kQ = 256;                 // queries per block (two MMAs of M = 128, TMEM lanes)
constexpr int kN = 256;                 // database vectors per tile (MMA N)
constexpr int kWorkers = 512;          // dequantize + scan (warps 0-15)
constexpr int kThreads = kWorkers + 32; // + the TMA / MMA issuer warp (warp 16)
constexpr int kTopK = 16;               // largest k this path takes
constexpr int kSMs = 148;               // grid sizing (fixed, so workspace sizes do not depend on the device)
constexpr uint32_t kPolls = 1u << 20;   // about a second of polling, then give up

constexpr int kStages = 2;              // operand stages (query + database chunk, 64 KB each)

// shared layout (offsets from a 1024-aligned base)
constexpr uint32_t SA = 0;                                  // stages x [256 x 64] fp16 queries (32 KB each)
constexpr uint32_t SB = kStages * 32768;                    // stages x [256 x 64] fp16 database (32 KB each)
constexpr uint32_t SLUT = SB + kStages * 32768;             // [256 code bytes][32 lane copies] half2 (32 KB)
constexpr uint32_t SBAR = SLUT + 32768;                     // 3 x stages + 2 mbarriers
constexpr uint32_t SFLAG = SBAR + 8 * (3 * kStages + 2);    // abort flag
constexpr uint32_t SM_TOTAL = SFLAG + 16 + 1024;            // + slack for aligning the base
static_assert(SM_TOTAL <= 232448, "shared memory");

struct SearchTcArgs {
    Layout L;
    const float *lv;               // levels by stored code (16)
    const uint8_t *db;
    int64_t n_db;
    int n_q, k;
    int64_t n_tiles;               // ceil(n_db / 256)
    int n_groups;                  // blocks per query tile
    const float *qscale;           // [n_q_pad] 2^e
    float *part_v;                 // [n_q][2 n_groups][k]
    int64_t *part_i;
    uint32_t *status;
};

__device__ __forceinline__ uint32_t h2pack(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// The database row a thread dequantizes: tile row tid % 256 (features
// [32 p, 32 p + 32) of each chunk, p = tid / 256).  A row past the end points
// at vector 0 with zero scales, so loads and dequantization need no branches.
struct Rows {
    const uint8_t *kc, *ks;         // this row's code bytes and sign bytes
    uint32_t nbits;                 // fp16 bits: nhat | rho << 16 (loaded a chunk ahead)
    uint32_t nh2, rh2;              // nhat and -rho sqrt(pi/2)/m as fp16 pairs
};

template <int D>
__device__ __forceinline__ void rows_for(const SearchTcArgs &a, int64_t tile, int tid, Rows &r) {
    const Layout &L = a.L;
    const int64_t v = tile * kN + (tid & 255);
    const bool ok = v < a.n_db;
    const int64_t vv = ok ? v : 0;
    const uint8_t *page = a.db + (vv / L.P) * int64_t(L.page_bytes);
    const int pos = int(vv % L.P);
    r.kc = page + L.kc_off + pos * (D / 2);
    r.ks = page + L.ks_off + pos * (D / 8);
    uint32_t nb = 0;
    if (ok)
        nb = uint32_t(__ldg(reinterpret_cast<const uint16_t *>(page + L.kn_off + pos * 2))) |
             (uint32_t(__ldg(reinterpret_cast<const uint16_t *>(page + L.kr_off + pos * 2))) << 16);
    r.nbits = nb;
}

template <int D>
__device__ __forceinline__ void rows_scales(Rows &r) {
    const float cq = 1.2533141373155003f / float(D);     // sqrt(pi/2) / m
    const uint32_t nb = r.nbits;
    r.nh2 = (nb & 0xFFFFu) * 0x10001u;
    const float rh = h2f_bits(uint16_t(nb >> 16)) * cq;
    r.rh2 = h2pack(-rh, -rh);
}

// Raw bytes of part p of chunk kc of the row: 16 code bytes (MSE chunk) or
// 4 sign bytes (QJL chunk, in raw.x).
template <int D>
__device__ __forceinline__ void load_raw(const Rows &r, int kc, int p, uint4 &raw) {
    constexpr int MSE_KC = D / 64;
    if (kc < MSE_KC) raw = __ldg(reinterpret_cast<const uint4 *>(r.kc + kc * 32 + 16 * p));
    else raw.x = __ldg(reinterpret_cast<const uint32_t *>(r.ks + (kc - MSE_KC) * 8 + 4 * p));
}

// Bounded wait that also gives up once another thread has given up; about a
// second in all.  `quick` polls first, then polls with short naps (so that
// waiting warps leave the issue slots to the working ones).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag,
                                              uint32_t quick) {
    for (uint32_t i = 0; i < quick; ++i) {
        if (tc05::mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 1023u && *abort_flag) return false;
    }
    for (uint32_t i = 0; i < 4000000u; ++i) {
        __nanosleep(32);
        if (tc05::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    *abort_flag = 1u;
    return false;
}

// Per-thread state of a dequantizing / scanning worker (warps 0-15).
struct Work {
    uint8_t *sm;
    uint64_t *full_b, *empty, *acc_full, *acc_empty;
    volatile uint32_t *abort_flag;
    uint32_t tmem;
    int tid, lane, warp, qh, part;  // qh: query half (M = 128 tile) of this thread's query;
                                    // part: feature half it dequantizes, vector half it scans
    const uint32_t *lut_lane;
};

// A worker's running top-k in registers: KT scores in descending order
// (ties: the earlier, lower index first) with their indices, KT the
// multiple of 4 at or above k.  For k < KT the first KT - k slots hold
// +inf sentinels that nothing displaces, so
// the last slot is always the k-th best so far.
template <int KT>
struct TopK {
    float v[KT];
    int32_t i[KT];
};

// r[e] for a run-time e (a select tree; registers cannot be indexed).
__device__ __forceinline__ uint32_t pick32(const uint32_t (&r)[32], int e) {
    uint32_t x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = (e & 16) ? r[i + 16] : r[i];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = (e & 8) ? x[i + 8] : x[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = (e & 4) ? x[i + 4] : x[i];
#pragma unroll
    for (int i = 0; i < 2; ++i) x[i] = (e & 2) ? x[i + 2] : x[i];
    return (e & 1) ? x[1] : x[0];
}

// Insert (sv, id), known to beat the last slot: one bubble pass upwards.
template <int KT>
__device__ __forceinline__ void topk_insert(TopK<KT> &t, float sv, int32_t id) {
    t.v[KT - 1] = sv;
    t.i[KT - 1] = id;
#pragma unroll
    for (int j = KT - 1; j > 0; --j) {
        const bool up = t.v[j] > t.v[j - 1];
        const float a = t.v[j - 1], b = t.v[j];
        const int32_t ia = t.i[j - 1], ib = t.i[j];
        t.v[j - 1] = up ? b : a;
        t.v[j] = up ? a : b;
        t.i[j - 1] = up ? ib : ia;
        t.i[j] = up ? ia : ib;
    }
}

// Waits decided per warp, so that warp-wide operations stay converged.
__device__ __forceinline__ bool wait_w(const Work &w, uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, wait_or_abort(bar, parity, w.abort_flag, 64));
}

// Features [32 part, 32 part + 32) of chunk kc of row tid % 256 into stage
// tile sB (16-byte pieces 4 part .. 4 part + 3 of the row).
template <int D>
__device__ __forceinline__ void dequant_chunk(const Work &w, const Rows &cur, int kc, const uint4 &raw, uint8_t *sB) {
    constexpr int MSE_KC = D / 64;
    uint32_t v[16];
    if (kc < MSE_KC) {
        const uint32_t cw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t byte = __byte_perm(cw[i >> 2], 0, 0x4440 + (i & 3));
            v[i] = hmul2u(w.lut_lane[byte * 32], cur.nh2);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = cur.rh2 ^ ((raw.x << (15 - i)) & 0x80008000u);
    }
#pragma unroll
    for (int pc = 0; pc < 4; ++pc)
        *reinterpret_cast<uint4 *>(sB + tc05::sw128_offset(uint32_t(w.tid & 255), uint32_t(4 * w.part + pc))) =
            make_uint4(v[4 * pc], v[4 * pc + 1], v[4 * pc + 2], v[4 * pc + 3]);
}

// Running top-k over this thread's 128 estimates of tile `tile` (its query,
// vector half `part`), once the tile's MMAs are done (accumulator phase
// `use`); then hand the accumulators back to the issuer.
template <int KT>
__device__ __forceinline__ bool scan_tile(const Work &w, const SearchTcArgs &a, int64_t tile, int use, TopK<KT> &top) {
    if (!wait_w(w, w.acc_full, uint32_t(use) & 1u)) return false;
    tc05::fence_after_sync();
    // estimates stay in accumulator units (2^-e of the true value) until the end
    const int64_t rem = a.n_db - (tile * kN + 128 * w.part);
    const int lim = rem < 128 ? int(rem) : 128;
    const int32_t id0 = int32_t(tile * kN + 128 * w.part);
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tc05::tmem_ld_32x32b_x32(
            w.tmem + (uint32_t((w.warp & 3) * 32) << 16) + uint32_t(w.qh * 256 + 128 * w.part + cc * 32), r);
        tc05::tmem_wait_ld();
        // the 32 estimates' maximum first: most groups hold no candidate
        float m[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) m[e] = fmaxf(__uint_as_float(r[e]), __uint_as_float(r[e + 16]));
#pragma unroll
        for (int h = 8; h >= 1; h >>= 1)
#pragma unroll
            for (int e = 0; e < h; ++e) m[e] = fmaxf(m[e], m[e + h]);
        if (KT > 12 && m[0] > top.v[KT - 1]) {
            // 16 slots leave no registers for the select tree: one column at a time
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float sv = __uint_as_float(r[e]);
                if (sv > top.v[KT - 1] && cc * 32 + e < lim) topk_insert(top, sv, id0 + cc * 32 + e);
            }
        } else if (m[0] > top.v[KT - 1]) {
            // candidates against the threshold at the start of the group (it only
            // rises), then taken in index order: the warp loops as often as its
            // busiest lane has candidates, not once per candidate column
            const float th = top.v[KT - 1];
            uint32_t mask = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (__uint_as_float(r[e]) > th && cc * 32 + e < lim) mask |= 1u << e;
            while (mask) {
                const int e = __ffs(int(mask)) - 1;
                mask &= mask - 1u;
                const float sv = __uint_as_float(pick32(r, e));
                if (sv > top.v[KT - 1]) topk_insert(top, sv, id0 + cc * 32 + e);
            }
        }
        __syncwarp();                   // converged for the next warp-wide TMEM load
    }
    tc05::fence_before_sync();
    __syncwarp();
    if (w.lane == 0) tc05::mbar_arrive(w.acc_empty);
    return true;
}

template <int D, int KT>
__global__ void __launch_bounds__(kThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, SearchTcArgs a) {
    constexpr int NKC = 2 * D / 64;                   // 64-feature chunks per tile
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_holder;
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t *lut = reinterpret_cast<uint32_t *>(sm + SLUT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SBAR);
    uint64_t *full_a = bars;                    // [stages] query chunk landed (TMA)
    uint64_t *full_b = bars + kStages;          // [stages] database chunk written (16 worker warps)
    uint64_t *empty = bars + 2 * kStages;       // [stages] the MMAs that read the stage are done (commit)
    uint64_t *acc_full = bars + 3 * kStages;    // the tile's MMAs are done (commit)
    uint64_t *acc_empty = acc_full + 1;         // the workers have read the tile's estimates (16 warps)
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + SFLAG);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x, grp = blockIdx.y, K = a.k;

    for (int i = tid; i < 256 * 32; i += kThreads) {
        const int e = i >> 5;
        lut[i] = h2pack(a.lv[e & 15], a.lv[e >> 4]);
    }
    if (warp == 0) {
        tc05::tmem_alloc(&tmem_holder, 512);
        tc05::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            tc05::mbar_init(&full_a[i], 1);
            tc05::mbar_init(&full_b[i], kWorkers / 32);
            tc05::mbar_init(&empty[i], 1);
        }
        tc05::mbar_init(acc_full, 1);
        tc05::mbar_init(acc_empty, kWorkers / 32);
        *abort_flag = 0u;
        tc05::fence_mbar_init();
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = tmem_holder;
    bool timeout = false;
    TopK<KT> top;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        top.v[j] = j < KT - K ? INFINITY : -INFINITY;
        top.i[j] = -1;
    }

    if (warp < kWorkers / 32) {
        // ================= workers: dequantize each chunk, scan each tile
        Work w;
        w.sm = sm;
        w.full_b = full_b;
        w.empty = empty;
        w.acc_full = acc_full;
        w.acc_empty = acc_empty;
        w.abort_flag = abort_flag;
        w.tmem = tmem;
        w.tid = tid;
        w.lane = lane;
        w.warp = warp;
        w.qh = (tid >> 7) & 1;
        w.part = tid >> 8;
        w.lut_lane = lut + lane;
        Rows cur, nxt;
        uint4 raw = make_uint4(0, 0, 0, 0), nraw = raw;
        int64_t tile = grp;
        int used = 0;                   // tiles dequantized
        uint32_t g = 0;                 // chunks dequantized
        if (tile < a.n_tiles) {
            rows_for<D>(a, tile, tid, cur);
            load_raw<D>(cur, 0, w.part, raw);
        }
        while (tile < a.n_tiles && !timeout) {
            for (int kc = 0; kc < NKC; ++kc) {
                if (kc == 0) rows_scales<D>(cur);
                if (kc == NKC - 1) {
                    rows_for<D>(a, tile + a.n_groups, tid, nxt);
                    load_raw<D>(nxt, 0, w.part, nraw);
                } else {
                    load_raw<D>(cur, kc + 1, w.part, nraw);
                }
                const int s = int(g % kStages);
                // the stage is free once the MMAs that read it (chunk g - stages) are done
                if (g >= kStages && !wait_w(w, &empty[s], (g / kStages - 1u) & 1u)) { timeout = true; break; }
                dequant_chunk<D>(w, cur, kc, raw, sm + SB + uint32_t(s) * 32768u);
                tc05::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) tc05::mbar_arrive(&full_b[s]);
                ++g;
                raw = nraw;
                // the previous tile's estimates, once this tile's first chunk is queued
                if (kc == 0 && used > 0 && !scan_tile(w, a, tile - a.n_groups, used - 1, top)) {
                    timeout = true;
                    break;
                }
            }
            ++used;
            tile += a.n_groups;
            cur = nxt;
        }
        if (!timeout && used > 0 && !scan_tile(w, a, tile - a.n_groups, used - 1, top)) timeout = true;
    } else if (lane == 0) {
        // ================= issuer: query chunks by TMA, the MMAs, the commits
        uint32_t g = 0;
        int64_t last = -1;              // last chunk whose MMAs were issued
        int used = 0;
        for (int64_t tile = grp; tile < a.n_tiles && !timeout; tile += a.n_groups, ++used) {
            for (int kc = 0; kc < NKC; ++kc, ++g) {
                const int s = int(g % kStages);
                const uint32_t n = g / kStages;
                if (g >= kStages && !wait_or_abort(&empty[s], (n - 1u) & 1u, abort_flag, 1u << 20)) {
                    timeout = true;
                    break;
                }
                uint8_t *sA = sm + SA + uint32_t(s) * 32768u;
                tc05::mbar_expect_tx(&full_a[s], 32768);
                tc05::tma_load_2d(sA, &tmQ, kc * 64, qt * kQ, &full_a[s]);
                bool ok = true;
                // the accumulators are free once the workers read the previous tile
                if (kc == 0 && used > 0) ok = wait_or_abort(acc_empty, uint32_t(used - 1) & 1u, abort_flag, 1u << 20);
                ok = ok && wait_or_abort(&full_b[s], n & 1u, abort_flag, 1u << 20);
                // the copy completes whatever happened: wait for it before leaving
                if (!tc05::mbar_wait_bounded(&full_a[s], n & 1u, kPolls)) ok = false;
                if (!ok) {
                    timeout = true;
                    break;
                }
                tc05::fence_after_sync();
                const uint32_t aa = tc05::smem_u32(sA), bb = tc05::smem_u32(sm + SB + uint32_t(s) * 32768u);
                constexpr uint32_t idesc = tc05::idesc_f16_f32(128, 256);
                // query half h: A rows [128 h, 128 h + 128) (16 KB apart), columns [256 h, 256 h + 256)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t bd = tc05::desc_kmajor_sw128(bb + ks * 32);
                    const bool acc = (kc | ks) != 0;
                    tc05::mma_f16(tmem, tc05::desc_kmajor_sw128(aa + ks * 32), bd, idesc, acc);
                    tc05::mma_f16(tmem + 256, tc05::desc_kmajor_sw128(aa + 16384 + ks * 32), bd, idesc, acc);
                }
                tc05::mma_commit(&empty[s]);
                if (kc == NKC - 1) tc05::mma_commit(acc_full);
                last = int64_t(g);
            }
        }
        if (timeout) *abort_flag = 1u;
        // every MMA issued completes before TMEM is given back
        if (last >= 0 &&
            !tc05::mbar_wait_bounded(&empty[last % kStages], uint32_t(last / kStages) & 1u, kPolls))
            timeout = true;
    }
    __syncwarp();

    if (tid < kWorkers) {
        const int q = qt * kQ + (tid & 255);            // = 256 qt + 128 qh + TMEM lane
        const int part = tid >> 8;
        if (q < a.n_q) {
            const float qsc = a.qscale[q];
            const int64_t o = (int64_t(q) * (2 * a.n_groups) + 2 * grp + part) * K - (KT - K);
#pragma unroll
            for (int j = 0; j < KT; ++j)
                if (j >= KT - K) {                  // slot j is entry j - (KT - k) of the list
                    const int32_t id = top.i[j];
                    a.part_v[o + j] = id >= 0 ? top.v[j] * qsc : -INFINITY;
                    a.part_i[o + j] = id;
                }
        }
    }
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, 512);
    }
    if (timeout || *abort_flag) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
}

// Query features [n_q_pad][2d] fp16 = 2^-e [R q | S R q] (QJL half in the
// pair order described above) and qscale = 2^e.  One warp per query.
template <int D>
__global__ void __launch_bounds__(128) qfeat_kernel(const float *qr, const float *w, int n_q, int n_q_pad,
                                                    __half *out, float *qscale) {
    const int lane = threadIdx.x & 31;
    const int q = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (q >= n_q_pad) return;
    float m = 0.f;
    if (q < n_q)
        for (int i = lane; i < D; i += 32)
            m = fmaxf(m, fmaxf(fabsf(qr[int64_t(q) * D + i]), fabsf(w[int64_t(q) * D + i])));
    m = warp_max(m);
    int ex = 0;
    if (m > 0.f) frexpf(m, &ex);                 // m < 2^ex
    const float down = m > 0.f ? ldexpf(1.f, 1 - ex) : 1.f;
    if (lane == 0) qscale[q] = m > 0.f ? ldexpf(1.f, ex - 1) : 1.f;
    for (int i = lane; i < 2 * D; i += 32) {
        float v = 0.f;
        if (q < n_q) {
            if (i < D) {
                v = qr[int64_t(q) * D + i];
            } else {
                const int k = i - D, pp = k & 31;
                const int coord = (k & ~31) + ((pp & 1) ? (pp >> 1) + 16 : (pp >> 1));
                v = w[int64_t(q) * D + coord];
            }
        }
        out[int64_t(q) * 2 * D + i] = __float2half_rn(v * down);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult qr;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

template <int D>
int run_tc(const tq_params *p, const Layout &L, const uint8_t *db, int64_t n_db, int n_q, int k, const float *qr,
           const float *w, uint8_t *qf_bytes, float *qscale, float *pv, int64_t *pi, int n_groups, uint32_t *status,
           cudaStream_t st) {
    const int n_qt = (n_q + kQ - 1) / kQ;
    const int n_q_pad = n_qt * kQ;
    __half *qf = reinterpret_cast<__half *>(qf_bytes);
    qfeat_kernel<D><<<unsigned(n_q_pad / 4), 128, 0, st>>>(qr, w, n_q, n_q_pad, qf, qscale);
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap tm;
    cuuint64_t dims[2] = {cuuint64_t(2 * D), cuuint64_t(n_q_pad)};
    cuuint64_t strides[1] = {cuuint64_t(2 * D * 2)};
    cuuint32_t box[2] = {64, uint32_t(kQ)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, qf, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    SearchTcArgs a;
    a.L = L;
    a.lv = p->dev.lv;
    a.db = db;
    a.n_db = n_db;
    a.n_q = n_q;
    a.k = k;
    a.n_tiles = (n_db + kN - 1) / kN;
    a.n_groups = n_groups;
    a.qscale = qscale;
    a.part_v = pv;
    a.part_i = pi;
    a.status = status;
    auto kern = k <= 4 ? score_tc_kernel<D, 4> : k <= 8 ? score_tc_kernel<D, 8> : k <= 12 ? score_tc_kernel<D, 12>
                                                                                     : score_tc_kernel<D, kTopK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SM_TOTAL));
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(n_qt), unsigned(n_groups)), kThreads, SM_TOTAL, st>>>(tm, a);
    return cudaGetLastError();
}

}  // namespace

// Database groups (blocks per query tile) of the tensor-core search, 0 when
// the configuration is not covered.  Each group yields two candidate lists
// per query (one per vector half of its tiles).
int search_tc_groups(const Layout &L, int64_t n_db, int n_q, int k) {
    if (!(L.kbits == 4 && L.kqjl && L.vbits == 0) || k > kTopK || n_db > INT32_MAX) return 0;
    if (!(L.d == 128 || L.d == 256 || L.d == 512 || L.d == 1024)) return 0;
    const int n_qt = (n_q + kQ - 1) / kQ;
    const int64_t n_tiles = (n_db + kN - 1) / kN;
    int64_t g = kSMs / n_qt;
    if (g < 1) g = 1;
    if (g > n_tiles) g = n_tiles;
    return int(g);
}

size_t search_tc_qf_bytes(const Layout &L, int n_q) {
    const size_t n_q_pad = size_t((n_q + kQ - 1) / kQ) * kQ;
    return n_q_pad * 2 * size_t(L.d) * sizeof(__half);
}

size_t search_tc_qscale_bytes(int n_q) { return size_t((n_q + kQ - 1) / kQ) * kQ * sizeof(float); }

int launch_search_tc(const tq_params *p, const Layout &L, const uint8_t *db, int64_t n_db, int n_q, int k,
                     const float *qr, const float *w, uint8_t *qf, float *qscale, float *pv, int64_t *pi,
                     int n_groups, uint32_t *status, cudaStream_t st) {
    switch (L.d) {
        case 128: return run_tc<128>(p, L, db, n_db, n_q, k, qr, w, qf, qscale, pv, pi, n_groups, status, st);
        case 256: return run_tc<256>(p, L, db, n_db, n_q, k, qr, w, qf, qscale, pv, pi, n_groups, status, st);
        case 512: return run_tc<512>(p, L, db, n_db, n_q, k, qr, w, qf, qscale, pv, pi, n_groups, status, st);
        case 1024: return run_tc<1024>(p, L, db, n_db, n_q, k, qr, w, qf, qscale, pv, pi, n_groups, status, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tq
