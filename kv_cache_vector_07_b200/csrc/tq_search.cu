// Top-k inner-product search over compressed vectors.
//
// ai-work-lab overview ("also applies to vector search; the index needs no
// preprocessing"; recall against PQ / RabitQ): the database is encoded by
// the same codec as the keys and scored with the same unbiased estimator
//   est_t = nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1>.
// Kernels: prep (q_r = R q, w = S q_r), score (one block per (query tile,
// database split): scores plus a per-query running top-k), merge (per query,
// top-k of all split lists; ties go to the lower index).
#include <cuda_runtime.h>

#include "tq_dev.cuh"

namespace tq {
namespace {

constexpr int kQT = 8;          // queries per block
constexpr int kTile = 128;      // database vectors per inner step
constexpr int kMaxK = 64;

// q_r = R q, one warp per query, 4 per block (w = S q_r follows in the
// projection kernel).
template <int D>
__global__ void __launch_bounds__(128) prep_f32_kernel(const float *Q, int64_t rows, DevParams p, float *qr) {
    constexpr int E = WarpVec<D>::E;
    __shared__ float wbuf[4][D <= 256 ? D : 4];          // dense rotation only (d <= 256)
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int64_t row = int64_t(blockIdx.x) * 4 + wl;
    if (row >= rows) return;
    float x[E];
    load_vec<D>(Q + row * D, lane, x);
    rotate_warp<D>(p, x, wbuf[wl], lane);
    if (lane < WarpVec<D>::LANES) {
#pragma unroll
        for (int e = 0; e < E; ++e) qr[row * D + lane * E + e] = x[e];
    }
}

struct ScoreArgs {
    Layout L;
    DevParams p;
    const uint8_t *db;
    int64_t n_db;
    int n_q, k, n_splits;
    int64_t split_len;
    const float *qr, *w;
    float *part_v;          // [n_q][n_splits][k]
    int64_t *part_i;
};

template <int D>
__global__ void __launch_bounds__(128) score_kernel(ScoreArgs a) {
    extern __shared__ float smem[];
    float *sq = smem;                    // [D][kQT]
    float *sw = sq + D * kQT;            // [D][kQT]
    __shared__ float sc[kQT][kTile];
    __shared__ float topv[kQT][kMaxK];
    __shared__ int64_t topi[kQT][kMaxK];
    __shared__ float lv[16], lv2[8];

    const Layout &L = a.L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int q0 = blockIdx.x * kQT;
    const int nq = min(kQT, a.n_q - q0);
    const int split = blockIdx.y;
    const int64_t t_begin = int64_t(split) * a.split_len;
    const int64_t t_end = min(a.n_db, t_begin + a.split_len);
    const int K = a.k;

    for (int i = tid; i < D * kQT; i += 128) {
        const int q = i / D, c = i - q * D;
        sq[c * kQT + q] = q < nq ? a.qr[int64_t(q0 + q) * D + c] : 0.f;
        sw[c * kQT + q] = q < nq ? a.w[int64_t(q0 + q) * D + c] : 0.f;
    }
    if (tid < 16) lv[tid] = tid < (1 << L.ka_bits) ? a.p.lv[tid] : 0.f;
    if (tid < 8) lv2[tid] = (L.khalf && tid < (1 << L.kb_bits)) ? a.p.lv2[tid] : 0.f;   // fractional rates
    for (int i = tid; i < kQT * kMaxK; i += 128) {
        topv[i / kMaxK][i % kMaxK] = -INFINITY;
        topi[i / kMaxK][i % kMaxK] = -1;
    }
    __syncthreads();
    const float cq = 1.2533141373155003f / float(D);

    for (int64_t c0 = t_begin; c0 < t_end; c0 += kTile) {
        const int64_t t = c0 + tid;
        float est[kQT];
        if (t < t_end) {
            const uint8_t *page = a.db + (t / L.P) * int64_t(L.page_bytes);
            const int pos = int(t % L.P);
            const uint8_t *kc = page + L.kc_off + pos * L.kc_bpt;
            const uint8_t *kh = L.ka_bits == 3 ? page + L.kh_off + pos * L.kh_bpt : nullptr;
            const uint8_t *ks = L.kqjl ? page + L.ks_off + pos * L.ks_bpt : nullptr;
            const int nA = L.khalf ? D / 2 : D;
            float mse[kQT], qj[kQT];
#pragma unroll
            for (int q = 0; q < kQT; ++q) { mse[q] = 0.f; qj[q] = 0.f; }
            for (int i = 0; i < D; ++i) {
                float cv;
                if (i < nA) {
                    uint32_t kap = read_field(kc, i, L.kc_w);
                    if (kh) kap |= read_field(kh, i, 1) << 2;
                    cv = lv[kap];
                } else {
                    uint32_t kap = read_field(page + L.kc2_off + pos * L.kc2_bpt, i - nA, L.kc2_w);
                    if (L.kb_bits == 3) kap |= read_field(page + L.kh2_off + pos * L.kh2_bpt, i - nA, 1) << 2;
                    cv = lv2[kap];
                }
                const bool ps = ks ? (read_field(ks, i, 1) != 0) : true;
#pragma unroll
                for (int q = 0; q < kQT; ++q) {
                    mse[q] = fmaf(sq[i * kQT + q], cv, mse[q]);
                    qj[q] += ps ? sw[i * kQT + q] : -sw[i * kQT + q];
                }
            }
            const float nk = h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kn_off + pos * 2));
            const float rk = L.kqjl ? h2f_bits(*reinterpret_cast<const uint16_t *>(page + L.kr_off + pos * 2)) : 0.f;
#pragma unroll
            for (int q = 0; q < kQT; ++q) est[q] = L.kqjl ? fmaf(rk * cq, qj[q], nk * mse[q]) : nk * mse[q];
        } else {
#pragma unroll
            for (int q = 0; q < kQT; ++q) est[q] = -INFINITY;
        }
#pragma unroll
        for (int q = 0; q < kQT; ++q) sc[q][tid] = est[q];
        __syncthreads();
        for (int q = warp; q < nq; q += 4) {
            const float kth = topv[q][K - 1];
            const bool full = topi[q][K - 1] >= 0;
            for (int base = 0; base < kTile; base += 32) {
                const int j = base + lane;
                const bool cand = (c0 + j < t_end) && (!full || sc[q][j] > kth);
                unsigned m = __ballot_sync(kFull, cand);
                if (lane == 0) {
                    while (m) {
                        const int jj = base + __ffs(m) - 1;
                        m &= m - 1;
                        const float s = sc[q][jj];
                        const int64_t id = c0 + jj;
                        if (topi[q][K - 1] >= 0 && !(s > topv[q][K - 1])) continue;
                        int p = K - 1;
                        while (p > 0 && (topi[q][p - 1] < 0 || s > topv[q][p - 1])) {
                            topv[q][p] = topv[q][p - 1];
                            topi[q][p] = topi[q][p - 1];
                            --p;
                        }
                        topv[q][p] = s;
                        topi[q][p] = id;
                    }
                }
                __syncwarp();
            }
        }
        __syncthreads();
    }
    for (int i = tid; i < nq * K; i += 128) {
        const int q = i / K, r = i - q * K;
        const int64_t o = (int64_t(q0 + q) * a.n_splits + split) * K + r;
        a.part_v[o] = topv[q][r];
        a.part_i[o] = topi[q][r];
    }
}

// One warp per query: the k best of the n_splits * k candidates.
__global__ void __launch_bounds__(128) merge_kernel(const float *pv, const int64_t *pi, int n_q, int n_splits, int k,
                                                    float *out_v, int64_t *out_i) {
    const int lane = threadIdx.x & 31;
    const int q = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (q >= n_q) return;
    const int n = n_splits * k;
    const float *v = pv + int64_t(q) * n;
    const int64_t *ix = pi + int64_t(q) * n;
    int64_t last_i = -1;
    float last_v = INFINITY;
    for (int r = 0; r < k; ++r) {
        float bv = -INFINITY;
        int64_t bi = -1;
        for (int j = lane; j < n; j += 32) {
            const int64_t id = ix[j];
            if (id < 0) continue;
            const float s = v[j];
            // strictly after (last_v, last_i) in the order (score desc, index asc)
            const bool after = (s < last_v) || (s == last_v && id > last_i);
            if (!after) continue;
            if (bi < 0 || s > bv || (s == bv && id < bi)) { bv = s; bi = id; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int64_t oi = __shfl_xor_sync(kFull, bi, o);
            if (oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
        }
        if (lane == 0) {
            out_v[int64_t(q) * k + r] = bi >= 0 ? bv : -INFINITY;
            out_i[int64_t(q) * k + r] = bi;
        }
        last_v = bv;
        last_i = bi;
        if (bi < 0) last_v = -INFINITY;
    }
}

struct SPlan {
    int n_splits;               // candidate lists per query
    int tc_groups;              // > 0: tensor-core path with this many blocks per query tile
    int64_t split_len;
    size_t off_qr, off_w, off_pv, off_pi, off_qf, off_qs, total;
};

SPlan splan(const Layout &L, int64_t n_db, int n_q, int k) {
    SPlan s;
    s.tc_groups = search_tc_groups(L, n_db, n_q, k);
    if (s.tc_groups > 0) {
        s.n_splits = 2 * s.tc_groups;
        s.split_len = 0;
    } else {
        const int tiles = (n_q + kQT - 1) / kQT;
        const int64_t target = 148 * 6;
        int64_t splits = (target + tiles - 1) / tiles;
        const int64_t maxs = (n_db + kTile - 1) / kTile;
        if (splits > maxs) splits = maxs;
        if (splits < 1) splits = 1;
        s.split_len = ((n_db + splits - 1) / splits + kTile - 1) / kTile * kTile;
        if (s.split_len < kTile) s.split_len = kTile;
        s.n_splits = int((n_db + s.split_len - 1) / s.split_len);
        if (s.n_splits < 1) s.n_splits = 1;
    }
    size_t off = kWsHeader;
    auto take = [&](size_t b) { size_t o = off; off += (b + 255) / 256 * 256; return o; };
    s.off_qr = take(sizeof(float) * size_t(n_q) * L.d);
    s.off_w = take(sizeof(float) * size_t(n_q) * L.d);
    s.off_pv = take(sizeof(float) * size_t(n_q) * s.n_splits * k);
    s.off_pi = take(sizeof(int64_t) * size_t(n_q) * s.n_splits * k);
    s.off_qf = s.tc_groups > 0 ? take(search_tc_qf_bytes(L, n_q)) : 0;
    s.off_qs = s.tc_groups > 0 ? take(search_tc_qscale_bytes(n_q)) : 0;
    s.total = off;
    return s;
}

template <int D>
int run_score(const tq_params *p, const Layout &L, const uint8_t *db, int64_t n_db, const float *Q, int n_q, int k,
              float *top_v, int64_t *top_i, uint8_t *ws, cudaStream_t st) {
    const SPlan s = splan(L, n_db, n_q, k);
    float *qr = reinterpret_cast<float *>(ws + s.off_qr);
    float *w = reinterpret_cast<float *>(ws + s.off_w);
    prep_f32_kernel<D><<<unsigned((n_q + 3) / 4), 128, 0, st>>>(Q, n_q, p->dev, qr);
    if (L.kqjl) {
        const int e = launch_qproj(qr, n_q, D, p->dev.S, w, st);
        if (e != cudaSuccess) return e;
    }
    float *pv = reinterpret_cast<float *>(ws + s.off_pv);
    int64_t *pi = reinterpret_cast<int64_t *>(ws + s.off_pi);
    if (s.tc_groups > 0) {
        const int e = launch_search_tc(p, L, db, n_db, n_q, k, qr, w, ws + s.off_qf,
                                       reinterpret_cast<float *>(ws + s.off_qs), pv, pi, s.tc_groups,
                                       reinterpret_cast<uint32_t *>(ws), st);
        if (e != cudaSuccess) return e;
        merge_kernel<<<unsigned((n_q + 3) / 4), 128, 0, st>>>(pv, pi, n_q, s.n_splits, k, top_v, top_i);
        return cudaGetLastError();
    }
    ScoreArgs a;
    a.L = L;
    a.p = p->dev;
    a.db = db;
    a.n_db = n_db;
    a.n_q = n_q;
    a.k = k;
    a.n_splits = s.n_splits;
    a.split_len = s.split_len;
    a.qr = qr;
    a.w = w;
    a.part_v = pv;
    a.part_i = pi;
    const size_t ssm = sizeof(float) * 2 * D * kQT;
    if (ssm > 16 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(ssm));
        if (e != cudaSuccess) return e;
    }
    score_kernel<D><<<dim3(unsigned((n_q + kQT - 1) / kQT), unsigned(s.n_splits)), 128, ssm, st>>>(a);
    merge_kernel<<<unsigned((n_q + 3) / 4), 128, 0, st>>>(a.part_v, a.part_i, n_q, s.n_splits, k, top_v, top_i);
    return cudaGetLastError();
}

}  // namespace

size_t score_ws_bytes(const Layout &L, int64_t n_db, int n_q, int k) { return splan(L, n_db, n_q, k).total; }

int launch_score(const tq_params *p, const Layout &L, const uint8_t *db, int64_t n_db, const float *Q, int n_q,
                 int k, float *top_v, int64_t *top_i, uint8_t *ws, size_t ws_bytes, void *stream) {
    (void)ws_bytes;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (L.d) {
        case 8: return run_score<8>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 16: return run_score<16>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 32: return run_score<32>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 64: return run_score<64>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 128: return run_score<128>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 256: return run_score<256>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 512: return run_score<512>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
        case 1024: return run_score<1024>(p, L, db, n_db, Q, n_q, k, top_v, top_i, ws, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tq
