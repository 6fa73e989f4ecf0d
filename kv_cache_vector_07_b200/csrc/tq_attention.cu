// Attention computed directly over the compressed cache (decode and chunked
// prefill), split over the key range and merged by log-sum-exp.
//
// Page "What is TurboQuant?", "Stage 2": the QJL bits make <q, k> estimates
// unbiased; the attention-logit figure quoted there is computed from the
// compressed keys.  Logit of key t for query q (R = H D / sqrt(d)):
//   l_t = (nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1>) / sqrt(d)
// then softmax over the visible keys and o = R_v^T sum_t p_t nhat_v,t c_v[code_v,t].
//
// Kernels: prep (per query row: q_r = R q and w = S q_r), attention (one
// block per (query group, key split): scores, online softmax, value
// accumulation in the value rotation's basis), combine (merge the splits by
// log-sum-exp, apply R_v^T with the Walsh-Hadamard butterflies, bf16 out).
#include <cuda_runtime.h>

#include "tq_dev.cuh"
#include "tq_encode_vec.cuh"

namespace tq {
namespace {

constexpr int kChunk = 128;        // keys per inner step (one per thread)
constexpr int kMaxG = 8;           // query heads per KV head handled per block

struct PrepArgs {
    const void *Q;          // [rows][D] bf16 or fp32
    int in_f32;
    int64_t rows;
    DevParams kp;
    float *qr;              // [rows][D]
    float *w;               // [rows][D]
};

// q_r = R q, one warp per query row, 4 rows per block (w = S q_r follows
// in the projection kernel).
template <int D>
__global__ void __launch_bounds__(128) prep_kernel(PrepArgs a) {
    constexpr int E = WarpVec<D>::E;
    __shared__ float wbuf[4][D <= 256 ? D : 4];          // dense rotation only (d <= 256)
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int64_t row = int64_t(blockIdx.x) * 4 + wl;
    if (row >= a.rows) return;
    float x[E];
    if (a.in_f32) load_vec<D>(reinterpret_cast<const float *>(a.Q) + row * D, lane, x);
    else load_vec<D>(reinterpret_cast<const __nv_bfloat16 *>(a.Q) + row * D, lane, x);
    rotate_warp<D>(a.kp, x, wbuf[wl], lane);
    if (lane < WarpVec<D>::LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) a.qr[row * D + lane * E + e] = x[e];
    }
}

// D = 128: q_r = R q and w = S q_r for 32 rows per block in one kernel: S
// staged transposed in shared memory (fp32, 64 KB), the rotation by one warp
// per row, the projection by thread (output j, 16 rows).
constexpr int kPQRows = 32;
constexpr size_t kPQSmem = sizeof(float) * (128 * 129 + kPQRows * 128);

// blockIdx.y selects which outputs j this block projects: all 128 (JS = 1),
// or (JS = 4, with few rows, so that more blocks share the work) a quarter of
// them, staging only those rows of S; every block rotates its own rows.  All
// 256 threads project: thread t takes output j0 + t % (128 / JS) for its
// group of 4 (JS = 4) or 16 (JS = 1) rows.
template <int JS>
__global__ void __launch_bounds__(256) prep_proj128_kernel(PrepArgs a) {
    constexpr int JN = 128 / JS, NR = JN / 8;   // outputs of this block, rows per thread
    extern __shared__ float pq_smem[];
    float *sT = pq_smem;                        // [k][j], row stride 129 (bank spread)
    float *sq = pq_smem + 128 * 129;            // [32 rows][128]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r0 = int64_t(blockIdx.x) * kPQRows;
    const int j0 = int(blockIdx.y) * JN;
    for (int i = tid; i < JN * 64; i += 256) {  // S[j][k] bf16 pairs -> sT[k][j]
        const int j = j0 + (i >> 6), k2 = (i & 63) * 2;
        const uint32_t pr = *reinterpret_cast<const uint32_t *>(a.kp.S + size_t(j) * 128 + k2);
        sT[k2 * 129 + j] = __uint_as_float(pr << 16);
        sT[(k2 + 1) * 129 + j] = __uint_as_float(pr & 0xFFFF0000u);
    }
    float sg[4];
    load_vec<128>(a.kp.signs, lane, sg);
    for (int rr = warp; rr < kPQRows; rr += 8) {
        const int64_t row = r0 + rr;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (row < a.rows) {
            if (a.in_f32) load_vec<128>(reinterpret_cast<const float *>(a.Q) + row * 128, lane, x);
            else load_vec<128>(reinterpret_cast<const __nv_bfloat16 *>(a.Q) + row * 128, lane, x);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] *= sg[e];
        fwht_warp<128>(x, lane);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float v = x[e] * 0.08838834764831845f;
            sq[rr * 128 + lane * 4 + e] = v;
            if (row < a.rows && blockIdx.y == 0) a.qr[row * 128 + lane * 4 + e] = v;
        }
    }
    __syncthreads();
    const int j = j0 + tid % JN, g = tid / JN;  // output j, rows NR g .. NR g + NR - 1
    float acc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = 0.f;
#pragma unroll 4
    for (int k = 0; k < 128; ++k) {
        const float sv = sT[k * 129 + j];
#pragma unroll
        for (int r = 0; r < NR; ++r) acc[r] = fmaf(sv, sq[(NR * g + r) * 128 + k], acc[r]);
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        const int64_t row = r0 + NR * g + r;
        if (row < a.rows) a.w[row * 128 + j] = acc[r];
    }
}

// ---------------------------------------------------------------------------
// Fused decode step, first launch: the new token's K and V of every sequence
// are compressed into the cache and the queries are prepared, one warp per
// vector.  Both need a projection by S (QJL keys: z = S r; queries: w =
// S q_r), done here from a per-warp shared copy of the vector, fp32
// products: lane l owns outputs [l E, l E + E) and reads its rows of S.
// ---------------------------------------------------------------------------
struct StepArgs {
    Layout L;
    DevParams kp, vp;
    const __nv_bfloat16 *K, *V;      // new tokens [B][H][D]
    const int32_t *slots;            // [B], < 0 = skip
    int64_t num_slots;
    uint8_t *cache;
    int B;
    PrepArgs prep;                   // queries [rows][D] -> qr, w
    uint32_t *status;
};

template <int D>
__device__ __forceinline__ void project_rows(const uint16_t *S, const float *vs, int lane,
                                             float (&z)[WarpVec<D>::E]) {
    constexpr int E = WarpVec<D>::E;
#pragma unroll
    for (int e = 0; e < E; ++e) z[e] = 0.f;
    if (lane >= WarpVec<D>::LANES) return;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const uint16_t *row = S + size_t(lane * E + e) * D;
        float acc = 0.f;
        for (int i = 0; i < D; i += 8) {
            const uint4 u = *reinterpret_cast<const uint4 *>(row + i);
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc = fmaf(__uint_as_float(w4[k] << 16), vs[i + 2 * k], acc);
                acc = fmaf(__uint_as_float(w4[k] & 0xFFFF0000u), vs[i + 2 * k + 1], acc);
            }
        }
        z[e] = acc;
    }
}

template <int D>
__global__ void __launch_bounds__(256) step_prep_kernel(StepArgs a) {
    constexpr int E = WarpVec<D>::E;
    __shared__ __align__(16) float svec[8][warp_buf_floats<D>()];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const Layout &L = a.L;
    const int64_t n_enc = int64_t(a.B) * L.H * 2;
    const int64_t job = int64_t(blockIdx.x) * 8 + wl;
    float *vs = svec[wl];
    if (job < n_enc) {
        const bool is_v = job >= int64_t(a.B) * L.H;
        const int64_t v = is_v ? job - int64_t(a.B) * L.H : job;
        const int b = int(v / L.H), h = int(v - int64_t(b) * L.H);
        const int slot = a.slots[b];
        if (slot < 0) return;
        if (slot >= a.num_slots) {
            if (lane == 0) atomicOr(a.status, TQ_DEV_SLOT_RANGE);
            return;
        }
        float x[E], r[E];
        load_vec<D>((is_v ? a.V : a.K) + v * D, lane, x);
        uint8_t *page = a.cache + (int64_t(slot / L.P) * L.H + h) * int64_t(L.page_bytes);
        const int pos = slot % L.P;
        if (!encode_vector_warp<D>(L, is_v ? a.vp : a.kp, is_v, x, page, pos, lane, r, vs)) return;
        if (lane < WarpVec<D>::LANES) {
#pragma unroll
            for (int e = 0; e < E; ++e) vs[lane * E + e] = r[e];
        }
        __syncwarp();
        float z[E];
        project_rows<D>(a.kp.S, vs, lane, z);
        uint32_t bit[E];
#pragma unroll
        for (int e = 0; e < E; ++e) bit[e] = z[e] >= 0.f ? 1u : 0u;     // s_j = [(S r)_j >= 0]
        store_fields<D, 1>(page + L.ks_off + pos * L.ks_bpt, lane, bit);
        return;
    }
    const int64_t row = job - n_enc;
    if (row >= a.prep.rows) return;
    float x[E];
    load_vec<D>(reinterpret_cast<const __nv_bfloat16 *>(a.prep.Q) + row * D, lane, x);
    rotate_warp<D>(a.kp, x, vs, lane);
    if (lane < WarpVec<D>::LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            a.prep.qr[row * D + lane * E + e] = x[e];
            vs[lane * E + e] = x[e];
        }
    }
    if (!L.kqjl) return;
    __syncwarp();
    float z[E];
    project_rows<D>(a.kp.S, vs, lane, z);
    if (lane < WarpVec<D>::LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) a.prep.w[row * D + lane * E + e] = z[e];
    }
}

struct AttnArgs {
    Layout L;
    DevParams kp, vp;
    const uint8_t *cache;
    int64_t num_blocks;
    int Hq, G, n_groups, n_splits, split_len;
    const int32_t *block_table;
    int bt_stride, max_blocks;
    const int32_t *seq_lens;
    int base_len;
    const float *qr, *w;         // [rows][D]
    float *part_o;               // [group][split][G][D]
    float *part_ml;              // [group][split][G][2]
    float *logits;               // optional
    int64_t logits_stride;
    uint32_t *status;
};

__device__ __forceinline__ int visible_len(const AttnArgs &a, int b) {
    return a.seq_lens ? a.seq_lens[b] : a.base_len + b + 1;
}

template <int D>
__global__ void __launch_bounds__(kChunk) attn_kernel(AttnArgs a) {
    constexpr int CPT = (D + kChunk - 1) / kChunk;     // coordinates per thread (value side)
    __shared__ float sq[D][kMaxG];
    __shared__ float sw[D][kMaxG];
    __shared__ float lg[kMaxG][kChunk];
    __shared__ float vn[kChunk];
    __shared__ const uint8_t *pg[kChunk];
    __shared__ float lvk[16], lvv[16], lvk2[8], lvv2[8];
    __shared__ float ptk[132], ptv[132];                  // polar tables of keys / values
    __shared__ float s_m[kMaxG], s_l[kMaxG], s_alpha[kMaxG];

    const Layout &L = a.L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = blockIdx.x, split = blockIdx.y;
    const int b = g / L.H, kvh = g - b * L.H;
    const int G = a.G;
    const int nv = visible_len(a, b);
    const int t_begin = split * a.split_len;
    const int t_end = min(nv, t_begin + a.split_len);
    const int32_t *bt = a.block_table + int64_t(b) * a.bt_stride;
    const int64_t row0 = int64_t(b) * a.Hq + int64_t(kvh) * G;

    for (int i = tid; i < D * G; i += kChunk) {
        const int h = i / D, c = i - h * D;
        sq[c][h] = a.qr[(row0 + h) * D + c];
        sw[c][h] = a.w[(row0 + h) * D + c];
    }
    if (tid < 16) {
        // first (or only) codebook of each; fractional rates add a second
        lvk[tid] = (L.ka_bits <= 4 && tid < (1 << L.ka_bits)) ? a.kp.lv[tid] : 0.f;
        lvv[tid] = tid < (1 << L.va_bits) ? a.vp.lv[tid] : 0.f;
        if (tid < 8) {
            lvk2[tid] = (L.khalf && tid < (1 << L.kb_bits)) ? a.kp.lv2[tid] : 0.f;
            lvv2[tid] = (L.vhalf && tid < (1 << L.vb_bits)) ? a.vp.lv2[tid] : 0.f;
        }
    }
    for (int i = tid; i < 132; i += kChunk) {
        ptk[i] = L.kpolar ? a.kp.polar[i] : 0.f;
        ptv[i] = L.vpolar ? a.vp.polar[i] : 0.f;
    }
    if (tid < kMaxG) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
    float acc[kMaxG][CPT];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[h][c] = 0.f;
    __syncthreads();

    const float scale = 1.0f / sqrtf(float(D));
    const float cq = 1.2533141373155003f / float(D);     // sqrt(pi/2) / m
    const int kw = L.kc_w;

    for (int c0 = t_begin; c0 < t_end; c0 += kChunk) {
        // ---- scores: one key per thread
        const int t = c0 + tid;
        float lgt[kMaxG];
        const uint8_t *page = nullptr;
        if (t < t_end) {
            const int bi = t / L.P;
            const int blk = bi < a.max_blocks ? bt[bi] : -1;
            if (blk >= 0 && blk < a.num_blocks) page = a.cache + (int64_t(blk) * L.H + kvh) * L.page_bytes;
            else atomicOr(a.status, TQ_DEV_BLOCK_RANGE);
        }
        pg[tid] = page;
        if (page) {
            const int pos = t % L.P;
            const uint8_t *kc = page + L.kc_off + pos * L.kc_bpt;
            const uint8_t *kh = L.ka_bits == 3 ? page + L.kh_off + pos * L.kh_bpt : nullptr;
            // fractional rates: coordinates nA .. D-1 in the second code arrays
            const int nA = L.khalf ? D / 2 : D;
            const uint8_t *kc2 = L.khalf ? page + L.kc2_off + pos * L.kc2_bpt : nullptr;
            const uint8_t *kh2 = (L.khalf && L.kb_bits == 3) ? page + L.kh2_off + pos * L.kh2_bpt : nullptr;
            const uint8_t *ks = L.kqjl ? page + L.ks_off + pos * L.ks_bpt : nullptr;
            float mse[kMaxG], qj[kMaxG];
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) { mse[h] = 0.f; qj[h] = 0.f; }
            // polar keys: pairs of the unit-radius reconstruction (the norm is applied below)
            for (int p = 0; L.kpolar && p < D / 2; ++p) {
                const float2 yv = polar_pair<D>(kc, page + L.kc2_off + pos * L.kc2_bpt, ptk, p);
                const bool s0 = ks ? (read_field(ks, 2 * p, 1) != 0) : true;
                const bool s1 = ks ? (read_field(ks, 2 * p + 1, 1) != 0) : true;
#pragma unroll
                for (int h = 0; h < kMaxG; ++h) {
                    if (h < G) {
                        mse[h] = fmaf(sq[2 * p][h], yv.x, fmaf(sq[2 * p + 1][h], yv.y, mse[h]));
                        qj[h] += (s0 ? sw[2 * p][h] : -sw[2 * p][h]) + (s1 ? sw[2 * p + 1][h] : -sw[2 * p + 1][h]);
                    }
                }
            }
            for (int i = 0; !L.kpolar && i < D; ++i) {
                float cv;
                if (kw == 8) {
                    cv = e4m3_to_float(kc[i]);          // FP8 key: e4m3(sqrt(d) u_i)
                } else if (i < nA) {
                    uint32_t kap = read_field(kc, i, kw);
                    if (kh) kap |= read_field(kh, i, 1) << 2;
                    cv = lvk[kap];
                } else {
                    uint32_t kap = read_field(kc2, i - nA, L.kc2_w);
                    if (kh2) kap |= read_field(kh2, i - nA, 1) << 2;
                    cv = lvk2[kap];
                }
                const bool pos_sign = ks ? (read_field(ks, i, 1) != 0) : true;
#pragma unroll
                for (int h = 0; h < kMaxG; ++h) {
                    if (h < G) {
                        mse[h] = fmaf(sq[i][h], cv, mse[h]);
                        qj[h] += pos_sign ? sw[i][h] : -sw[i][h];
                    }
                }
            }
            // FP8 keys store sqrt(d) u: the estimate is nhat <Rq, e4m3(code)> / sqrt(d)
            const float nk = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kn_off + pos * 2)) *
                             (kw == 8 ? scale : 1.0f);
            const float rk = L.kqjl ? h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kr_off + pos * 2)) : 0.f;
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                float v = nk * mse[h];
                if (L.kqjl) v = fmaf(rk * cq, qj[h], v);
                lgt[h] = v * scale;
            }
            vn[tid] = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.vn_off + pos * 2));
        } else {
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) lgt[h] = -INFINITY;
            vn[tid] = 0.f;
        }
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
            if (h < G) {
                lg[h][tid] = lgt[h];
                if (a.logits && t < t_end) a.logits[(row0 + h) * a.logits_stride + t] = lgt[h];
            }
        }
        __syncthreads();

        // ---- online softmax: warp w handles heads w, w + 4
        for (int h = warp; h < G; h += 4) {
            float mx = -INFINITY;
            for (int j = lane; j < kChunk; j += 32) mx = fmaxf(mx, lg[h][j]);
            mx = warp_max(mx);
            const float m_old = s_m[h];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.f;
            for (int j = lane; j < kChunk; j += 32) {
                const float p = m_new == -INFINITY ? 0.f : expf(lg[h][j] - m_new);
                lg[h][j] = p;
                sum += p;
            }
            sum = warp_sum(sum);
            if (lane == 0) {
                const float alpha = m_old == -INFINITY ? 0.f : expf(m_old - m_new);
                s_alpha[h] = alpha;
                s_l[h] = s_l[h] * alpha + sum;
                s_m[h] = m_new;
            }
        }
        __syncthreads();

        // ---- value accumulation: thread owns coordinates tid + kChunk * c
        float al[kMaxG];
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) al[h] = h < G ? s_alpha[h] : 0.f;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h)
#pragma unroll
            for (int c = 0; c < CPT; ++c) acc[h][c] *= al[h];
        const int nloc = min(kChunk, t_end - c0);
        for (int j = 0; j < nloc; ++j) {
            const uint8_t *page = pg[j];
            if (!page) continue;
            const int pos = (c0 + j) % L.P;
            const uint8_t *vc = page + L.vc_off + pos * L.vc_bpt;
            const uint8_t *vh = L.va_bits == 3 ? page + L.vh_off + pos * L.vh_bpt : nullptr;
            const int vA = L.vhalf ? D / 2 : D;
            const float nvv = vn[j];
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const int i = tid + c * kChunk;
                if (i < D) {
                    float lvl;
                    if (L.vpolar) {
                        const float2 yv = polar_pair<D>(vc, page + L.vc2_off + pos * L.vc2_bpt, ptv, i >> 1);
                        lvl = (i & 1) ? yv.y : yv.x;
                    } else if (i < vA) {
                        uint32_t kap = read_field(vc, i, L.vc_w);
                        if (vh) kap |= read_field(vh, i, 1) << 2;
                        lvl = lvv[kap];
                    } else {
                        const int i2 = i - vA;
                        uint32_t kap = read_field(page + L.vc2_off + pos * L.vc2_bpt, i2, L.vc2_w);
                        if (L.vb_bits == 3) kap |= read_field(page + L.vh2_off + pos * L.vh2_bpt, i2, 1) << 2;
                        lvl = lvv2[kap];
                    }
                    const float val = lvl * nvv;
#pragma unroll
                    for (int h = 0; h < kMaxG; ++h)
                        if (h < G) acc[h][c] = fmaf(lg[h][j], val, acc[h][c]);
                }
            }
        }
        __syncthreads();
    }

    // ---- partial results of this split
    const int64_t pbase = (int64_t(g) * a.n_splits + split) * G;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (h < G) {
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const int i = tid + c * kChunk;
                if (i < D) a.part_o[(pbase + h) * D + i] = acc[h][c];
            }
        }
    }
    if (tid < G) {
        a.part_ml[(pbase + tid) * 2] = s_m[tid];
        a.part_ml[(pbase + tid) * 2 + 1] = s_l[tid];
    }
}

struct CombineArgs {
    int n_groups, n_splits, G, Hq, H;
    const float *part_o, *part_ml;
    DevParams vp;
    void *out;          // bf16 [n_seq][Hq][D]
    float *lse;         // optional [n_seq][Hq]
};

// One warp per (group, head): merge splits by log-sum-exp, rotate back.  The
// split maxima and weights are reduced across lanes (lane s holds split s of a
// 32-split chunk), so the partial-output loads of a chunk are independent.
template <int D>
__global__ void __launch_bounds__(128) combine_kernel(CombineArgs a) {
    constexpr int E = WarpVec<D>::E;
    __shared__ float wbuf[4][D <= 256 ? D : 4];          // dense rotation only (d <= 256)
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (r >= int64_t(a.n_groups) * a.G) return;
    const int g = int(r / a.G), h = int(r - int64_t(g) * a.G);
    auto pb = [&](int s) { return (int64_t(g) * a.n_splits + s) * a.G + h; };
    float M = -INFINITY;
    for (int s = lane; s < a.n_splits; s += 32) M = fmaxf(M, a.part_ml[pb(s) * 2]);
    M = warp_max(M);
    float Lsum = 0.f;
    float o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.f;
    for (int s0 = 0; s0 < a.n_splits; s0 += 32) {
        const int s = s0 + lane;
        float f = 0.f;
        if (s < a.n_splits) {
            const float m = a.part_ml[pb(s) * 2];
            if (m != -INFINITY) {
                f = expf(m - M);
                Lsum = fmaf(a.part_ml[pb(s) * 2 + 1], f, Lsum);
            }
        }
        const int n = min(32, a.n_splits - s0);
        int i = 0;
        // eight splits' partials are loaded before they are added, so the
        // loads overlap (long contexts have a hundred or more splits per row)
        for (; i + 8 <= n; i += 8) {
            float v[8][E], fi[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                fi[u] = __shfl_sync(kFull, f, i + u);
                const float *src = a.part_o + pb(s0 + i + u) * D + lane * E;
#pragma unroll
                for (int e = 0; e < E; ++e) v[u][e] = (lane < WarpVec<D>::LANES && fi[u] != 0.f) ? src[e] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int e = 0; e < E; ++e) o[e] = fmaf(v[u][e], fi[u], o[e]);
        }
        for (; i < n; ++i) {
            const float fi = __shfl_sync(kFull, f, i);
            if (fi == 0.f) continue;
            if (lane < WarpVec<D>::LANES) {
                const float *src = a.part_o + pb(s0 + i) * D + lane * E;
#pragma unroll
                for (int e = 0; e < E; ++e) o[e] = fmaf(src[e], fi, o[e]);
            }
        }
    }
    Lsum = warp_sum(Lsum);
    const float inv = Lsum > 0.f ? 1.0f / Lsum : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] *= inv;
    const int b = g / a.H, kvh = g - b * a.H;
    const int64_t orow = int64_t(b) * a.Hq + int64_t(kvh) * a.G + h;
    __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out) + orow * D;
    if (a.vp.rot) {
        // o = R^T o_r with the dense rotation: rows of its transpose
        float *vs = wbuf[(threadIdx.x >> 5) & 3];
        if (lane < WarpVec<D>::LANES) {
#pragma unroll
            for (int e = 0; e < E; ++e) vs[lane * E + e] = o[e];
        }
        __syncwarp();
        dense_cols<D>(a.vp.Rd, vs, lane, o);           // o_i = sum_j R[j][i] (o_r)_j
        if (lane < WarpVec<D>::LANES) {
#pragma unroll
            for (int e = 0; e < E; ++e) out[lane * E + e] = __float2bfloat16_rn(o[e]);
        }
    } else {
        fwht_warp<D>(o, lane);
        float sg[E];
        load_vec<D>(a.vp.signs, lane, sg);
        const float rs = 1.0f / sqrtf(float(D));
        if (lane < WarpVec<D>::LANES) {
#pragma unroll
            for (int e = 0; e < E; ++e) out[lane * E + e] = __float2bfloat16_rn(o[e] * rs * sg[e]);
        }
    }
    if (a.lse && lane == 0) a.lse[orow] = Lsum > 0.f ? M + logf(Lsum) : -INFINITY;
}

struct Plan {
    int n_groups, G, n_splits, split_len;
    size_t off_qr, off_w, off_po, off_pml, total;
};

Plan make_plan(const Layout &L, const AttnShape &s) {
    Plan p;
    p.G = s.Hq / L.H;
    p.n_groups = s.n_seq * L.H;
    int sms = 148;
    const int maxlen = s.max_len > 0 ? s.max_len : 1;
    const int64_t target = int64_t(sms) * 4;
    int splits = int((target + p.n_groups - 1) / p.n_groups);
    const int max_splits = (maxlen + kChunk - 1) / kChunk;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    int split_len = (maxlen + splits - 1) / splits;
    split_len = (split_len + kChunk - 1) / kChunk * kChunk;
    splits = (maxlen + split_len - 1) / split_len;
    if (pf128_covers(L, s)) {
        splits = pf128_splits(L, s, &split_len);
    } else if (const int res = dec128_resident(L, p.G)) {
        // tensor-core decode: whole waves of resident blocks, splits of at least 8 pages
        const int64_t slots = int64_t(sms) * res;
        const int max_sp = (maxlen + 511) / 512;
        int best = 1;
        double best_eff = 0.0;
        for (int sp = 1; sp <= max_sp && sp <= 256; ++sp) {
            const double waves = double(int64_t(p.n_groups) * sp) / double(slots);
            const double eff = waves / double(int64_t(waves + 0.999999));
            // prefer more blocks only while it buys efficiency or the first full wave
            if (eff > best_eff + 0.02 || (best_eff < 0.5 && eff >= best_eff)) {
                best_eff = eff;
                best = sp;
            }
            if (waves >= 4.0) break;
        }
        split_len = (maxlen + best - 1) / best;
        split_len = (split_len + kChunk - 1) / kChunk * kChunk;
        splits = (maxlen + split_len - 1) / split_len;
    }
    p.n_splits = splits;
    p.split_len = split_len;
    const int64_t rows = int64_t(s.n_seq) * s.Hq;
    size_t off = kWsHeader;
    auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) / 256 * 256; return o; };
    p.off_qr = take(sizeof(float) * rows * L.d);
    p.off_w = take(sizeof(float) * rows * L.d);
    p.off_po = take(sizeof(float) * int64_t(p.n_groups) * splits * p.G * L.d);
    p.off_pml = take(sizeof(float) * int64_t(p.n_groups) * splits * p.G * 2);
    p.total = off;
    return p;
}

template <int D>
int run_attention(const tq_params *kp, const tq_params *vp, const Layout &L, const void *Q, const AttnShape &s,
                  const uint8_t *cache, int64_t num_blocks, void *out, float *lse, float *logits,
                  int64_t logits_stride, uint8_t *ws, cudaStream_t st, const StepTokens *step) {
    const Plan p = make_plan(L, s);
    const int64_t rows = int64_t(s.n_seq) * s.Hq;
    PrepArgs pa;
    pa.Q = Q;
    pa.in_f32 = 0;
    pa.rows = rows;
    pa.kp = kp->dev;
    pa.qr = reinterpret_cast<float *>(ws + p.off_qr);
    pa.w = reinterpret_cast<float *>(ws + p.off_w);
    if (step) {
        // decode step: the new tokens' encode shares the query-preparation launch
        StepArgs sa;
        sa.L = L;
        sa.kp = kp->dev;
        sa.vp = vp->dev;
        sa.K = static_cast<const __nv_bfloat16 *>(step->K);
        sa.V = static_cast<const __nv_bfloat16 *>(step->V);
        sa.slots = step->slots;
        sa.num_slots = num_blocks * L.P;
        sa.cache = step->cache;
        sa.B = s.n_seq;
        sa.prep = pa;
        sa.status = reinterpret_cast<uint32_t *>(ws);
        const int64_t jobs = int64_t(s.n_seq) * L.H * 2 + rows;
        step_prep_kernel<D><<<unsigned((jobs + 7) / 8), 256, 0, st>>>(sa);
    } else if (D == 128 && L.kqjl && !kp->dev.rot) {
        const unsigned rblocks = unsigned((rows + kPQRows - 1) / kPQRows);
        auto kern = rblocks < 64 ? prep_proj128_kernel<4> : prep_proj128_kernel<1>;   // few rows: 4 blocks per tile
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPQSmem));
        if (e != cudaSuccess) return e;
        kern<<<dim3(rblocks, rblocks < 64 ? 4u : 1u), 256, kPQSmem, st>>>(pa);
    } else {
        prep_kernel<D><<<unsigned((rows + 3) / 4), 128, 0, st>>>(pa);
        if (L.kqjl) {
            const int e = launch_qproj(pa.qr, rows, D, kp->dev.S, pa.w, st);
            if (e != cudaSuccess) return e;
        }
    }

    int fast;
    if (pf128_covers(L, s))
        fast = launch_pf128(kp, vp, L, pa.qr, pa.w, s, p.n_splits, p.split_len, cache, num_blocks,
                            reinterpret_cast<float *>(ws + p.off_po), reinterpret_cast<float *>(ws + p.off_pml),
                            reinterpret_cast<uint32_t *>(ws), st);
    else
        fast = launch_dec128(kp, vp, L, pa.qr, pa.w, s, p.G, p.n_groups, p.n_splits, p.split_len, cache,
                             num_blocks, reinterpret_cast<float *>(ws + p.off_po),
                             reinterpret_cast<float *>(ws + p.off_pml), logits, logits_stride,
                             reinterpret_cast<uint32_t *>(ws), st);
    if (fast > 0) return fast;

    AttnArgs a;
    a.L = L;
    a.kp = kp->dev;
    a.vp = vp->dev;
    a.cache = cache;
    a.num_blocks = num_blocks;
    a.Hq = s.Hq;
    a.G = p.G;
    a.n_groups = p.n_groups;
    a.n_splits = p.n_splits;
    a.split_len = p.split_len;
    a.block_table = s.block_table;
    a.bt_stride = s.bt_stride;
    a.max_blocks = s.max_blocks;
    a.seq_lens = s.seq_lens;
    a.base_len = s.base_len;
    a.qr = pa.qr;
    a.w = pa.w;
    a.part_o = reinterpret_cast<float *>(ws + p.off_po);
    a.part_ml = reinterpret_cast<float *>(ws + p.off_pml);
    a.logits = logits;
    a.logits_stride = logits_stride;
    a.status = reinterpret_cast<uint32_t *>(ws);
    if (fast < 0) attn_kernel<D><<<dim3(unsigned(p.n_groups), unsigned(p.n_splits)), kChunk, 0, st>>>(a);

    CombineArgs c;
    c.n_groups = p.n_groups;
    c.n_splits = p.n_splits;
    c.G = p.G;
    c.Hq = s.Hq;
    c.H = L.H;
    c.part_o = a.part_o;
    c.part_ml = a.part_ml;
    c.vp = vp->dev;
    c.out = out;
    c.lse = lse;
    const int64_t crow = int64_t(p.n_groups) * p.G;
    combine_kernel<D><<<unsigned((crow + 3) / 4), 128, 0, st>>>(c);
    return cudaGetLastError();
}

}  // namespace

size_t attn_ws_bytes(const Layout &L, const AttnShape &s) { return make_plan(L, s).total; }

int launch_attention(const tq_params *kp, const tq_params *vp, const Layout &L, const void *Q,
                     const AttnShape &s, const uint8_t *cache, int64_t num_blocks, void *out, float *lse,
                     float *logits, int64_t logits_stride, uint8_t *ws, size_t ws_bytes, void *stream,
                     const StepTokens *step) {
    (void)ws_bytes;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
#define TQ_RUN_ATT(DD) \
    case DD: return run_attention<DD>(kp, vp, L, Q, s, cache, num_blocks, out, lse, logits, logits_stride, ws, st, step);
    switch (L.d) {
        TQ_RUN_ATT(8) TQ_RUN_ATT(16) TQ_RUN_ATT(32) TQ_RUN_ATT(64) TQ_RUN_ATT(128) TQ_RUN_ATT(256)
    }
#undef TQ_RUN_ATT
    return cudaErrorInvalidValue;
}

}  // namespace tq
