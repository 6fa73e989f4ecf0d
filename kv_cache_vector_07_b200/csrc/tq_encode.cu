// Write path: compress K/V vectors into the paged cache.
//
// Page "What is TurboQuant?", "Stage 1: rotation and scalar quantization by
// PolarQuant" (randomized Hadamard rotation, per-coordinate Lloyd-Max codes,
// no per-block scale) and "Stage 2: removing inner-product bias with a 1-bit
// QJL residual"; ai-work-lab overview, "QJL" (+1/-1 sign bits of a random
// projection of the residual); vLLM preset k8v4 (FP8 keys).
//
// Kernel 1 (encode_kernel, one warp per vector): load, norm, sign flip,
// Walsh-Hadamard butterflies with __shfl_xor_sync, bucketize against the
// Lloyd-Max boundaries in registers, sign-magnitude codes packed into the
// page, fp16 norm; for QJL keys also the residual r = y - nhat c[idx] (kept
// in fp32 scratch) and its fp16 norm rho.
// Kernel 2 (qjl_gemm_kernel): z = S r on the tensor cores (tcgen05.mma,
// accumulator in TMEM).  r (kept scaled by a power of two per vector) is
// split into fp16 hi + lo against the fp16 copy of S, 22 bits of r, so every
// z_j whose sign could differ from the exact product's lies within 2^-22
// ||r|| ||S_j|| of zero; the epilogue packs sign bits straight into the page.
#include <cstring>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "tc05.cuh"
#include "tq_dev.cuh"
#include "tq_encode_vec.cuh"

namespace tq {
namespace {

struct EncodeArgs {
    Layout L;
    DevParams kp, vp;
    const void *K, *V;
    int64_t n_tokens;
    const int32_t *slots;
    int64_t num_slots;
    uint8_t *cache;
    float *resid;        // [n_tokens * H][D] (QJL keys) or nullptr
    uint32_t *status;
    int do_v;
};

// Residual of a QJL key, stored times 2^e with ||r|| 2^e in [2^10, 2^11): the
// projection's fp16 hi + lo parts then stay normal, and its signs do not
// depend on a positive scale.
template <int D>
__device__ __forceinline__ void store_resid(float *resid, const float (&r)[WarpVec<D>::E], int lane) {
    constexpr int E = WarpVec<D>::E;
    float rr = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) rr = fmaf(r[e], r[e], rr);
    rr = warp_sum(rr);
    float sc = 1.f;
    if (rr > 0.f) {
        const int ex = ((__float_as_int(sqrtf(rr)) >> 23) & 0xff) - 127;
        sc = __int_as_float(min(254, max(1, 127 + 10 - ex)) << 23);
    }
    if (lane < WarpVec<D>::LANES) {
        float *dst = resid + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) dst[e] = r[e] * sc;
    }
}

template <int D, typename TIn>
__global__ void __launch_bounds__(256, D >= 512 ? 2 : 4) encode_kernel(EncodeArgs a) {
    constexpr int E = WarpVec<D>::E;
    __shared__ __align__(16) float wbuf[8][warp_buf_floats<D>()];
    // d = 1024: the transpose buffer of encode1024_t
    __shared__ __align__(16) float tbuf[D == 1024 ? 8 : 1][D == 1024 ? 1024 : 1];
    const int lane = threadIdx.x & 31;
    const Layout &L = a.L;
    const int64_t nvec = a.n_tokens * L.H;
    const int64_t total = a.do_v ? 2 * nvec : nvec;
    const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;

    for (int64_t vid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; vid < total; vid += nwarps) {
        const bool is_v = vid >= nvec;
        const int64_t v = is_v ? vid - nvec : vid;
        const int64_t t = v / L.H;
        const int h = int(v - t * L.H);
        const int slot = a.slots[t];
        if (slot < 0) continue;
        if (slot >= a.num_slots) {
            if (lane == 0) atomicOr(a.status, TQ_DEV_SLOT_RANGE);
            continue;
        }
        const DevParams &P = is_v ? a.vp : a.kp;
        float x[E], r[E];
        load_vec<D>(reinterpret_cast<const TIn *>(is_v ? a.V : a.K) + v * D, lane, x);
        uint8_t *page = a.cache + (int64_t(slot / L.P) * L.H + h) * int64_t(L.page_bytes);
        const int pos = slot % L.P;
        if constexpr (D == 1024) {
            const int bits = is_v ? L.vbits : L.kbits;
            if (P.cells && !P.rot && bits <= 4 && !(is_v ? (L.vhalf || L.vpolar) : (L.khalf || L.kpolar))) {
                float4 *cs = reinterpret_cast<float4 *>(wbuf[threadIdx.x >> 5]);
                __syncwarp();
                if (lane < 16) cs[lane] = P.cells[lane];
                __syncwarp();
                encode1024_t(L, P, is_v, x, page, pos, lane, tbuf[(threadIdx.x >> 5) & 7], cs,
                             a.resid ? a.resid + v * D : nullptr);
                continue;
            }
        }
        if (encode_vector_warp<D>(L, P, is_v, x, page, pos, lane, r, wbuf[threadIdx.x >> 5])) store_resid<D>(a.resid + v * D, r, lane);
    }
}

// Dense rotations (d <= 256): groups of four vectors of one kind (keys, then
// values), rotated together so that each row of R^T is read once per group,
// then quantized one by one.  A kernel of its own so that the others keep
// their register budget.
template <int D, typename TIn>
__global__ void __launch_bounds__(256) encode_dense_kernel(EncodeArgs a) {
    constexpr int E = WarpVec<D>::E;
    __shared__ __align__(16) float wbuf[8][dense_buf_floats<D>()];
    const int lane = threadIdx.x & 31;
    const Layout &L = a.L;
    const int64_t nvec = a.n_tokens * L.H;
    const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    // dense rotations: groups of four vectors of one kind, rotated together so
    // that each row of R^T is read once per group
    const int64_t ngk = (nvec + 3) / 4, ng = a.do_v ? 2 * ngk : ngk;
    float *wb = wbuf[threadIdx.x >> 5];
    for (int64_t gi = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; gi < ng; gi += nwarps) {
        const bool is_v = gi >= ngk;
        const int64_t v0 = (is_v ? gi - ngk : gi) * 4;
        const DevParams &P = is_v ? a.vp : a.kp;
        float x[4][E];
        uint8_t *page[4];
        int pos[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t v = v0 + k;
            page[k] = nullptr;
            pos[k] = 0;
            if (v < nvec) {
                const int64_t t = v / L.H;
                const int h = int(v - t * L.H);
                const int slot = a.slots[t];
                if (slot >= a.num_slots) {
                    if (lane == 0) atomicOr(a.status, TQ_DEV_SLOT_RANGE);
                } else if (slot >= 0) {
                    page[k] = a.cache + (int64_t(slot / L.P) * L.H + h) * int64_t(L.page_bytes);
                    pos[k] = slot % L.P;
                }
            }
            if (page[k]) load_vec<D>(reinterpret_cast<const TIn *>(is_v ? a.V : a.K) + (v0 + k) * D, lane, x[k]);
            else {
#pragma unroll
                for (int e = 0; e < E; ++e) x[k][e] = 0.f;
            }
        }
        if (P.rot) {
            __syncwarp();
            if (lane < WarpVec<D>::LANES) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int e = 0; e < E; ++e) wb[k * D + lane * E + e] = x[k][e];
            }
            __syncwarp();
            dense_cols_n<D, 4>(P.RdT, wb, lane, x);   // y_j = sum_i R^T[i][j] x_i
            __syncwarp();
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (!page[k]) continue;
            float r[E];
            if (encode_vector_warp<D>(L, P, is_v, x[k], page[k], pos[k], lane, r, wb, P.rot != 0))
                store_resid<D>(a.resid + (v0 + k) * D, r, lane);
        }
    }
}

// ---------------------------------------------------------------------------
// QJL projection on the tensor cores.
// ---------------------------------------------------------------------------
struct QjlArgs {
    Layout L;
    const uint16_t *S16;    // [m][D] fp16 bits (the tile fill when D < 64)
    const float *resid;     // [nK][D], each row scaled by a power of two
    int64_t nK;             // n_tokens * H
    const int32_t *slots;
    int64_t num_slots;
    uint8_t *cache;
    uint32_t *status;
};

constexpr int kBM = 128;       // vectors per tile (MMA M)
constexpr int kBK = 64;        // K elements per stage (one 128-byte swizzle row)
constexpr int kQThreads = 256; // two per residual row
constexpr uint32_t kMaxPolls = 1u << 20;   // about a second of polling, then give up

// z = S r for a tile of 128 residuals against BN projection rows, on the
// tensor cores.  r (fp32, scaled per row by a power of two) is split into
// fp16 hi + lo (22 bits; the scale keeps both parts normal) against the
// fp16 copy of S (exact for |S| >= 2^-14); two MMAs per k-step and per 256
// output columns, fp32 accumulators in TMEM (BN = 512 fills all of it).
// Per 64-column chunk: S arrives by TMA (128-byte swizzle, the layout the
// MMA reads), two threads per residual row convert their halves while the
// next chunk's residual is already loading into registers, and one thread
// issues the MMAs.  The epilogue packs the sign bits [z_j >= 0] into the
// page.  The grid runs the N tiles of one residual tile next to each other,
// so the tile's rows are read from DRAM once and served to the others from L2.
template <int D, int BN>
__global__ void __launch_bounds__(kQThreads, 1)
qjl_gemm_kernel(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ QjlArgs a) {
    constexpr int M = D;                                   // projection rows
    constexpr int NK = (D + kBK - 1) / kBK;
    constexpr int NI = BN < 256 ? BN : 256;                // N of one MMA (and one TMA box)
    constexpr uint32_t TCOLS = BN < 32 ? 32 : BN;
    constexpr int A_BYTES = kBM * 128;                     // one split tile
    constexpr int B_BYTES = BN * 128;
    constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
    constexpr int CW = kBK / 2;                            // columns per thread and chunk

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_mma[2], bar_b[2];
    __shared__ uint32_t tmem_holder;
    __shared__ int timed_out;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & (kBM - 1), hlf = tid >> 7;
    const int n0 = blockIdx.x * BN;
    const int64_t row0 = int64_t(blockIdx.y) * kBM;
    const int64_t g = row0 + row;

    if (warp == 0) {
        tc05::tmem_alloc(&tmem_holder, TCOLS);
        tc05::tmem_relinquish();
    }
    if (tid == 32) {
        for (int i = 0; i < 2; ++i) {
            tc05::mbar_init(&bar_mma[i], 1);
            tc05::mbar_init(&bar_b[i], 1);
        }
        tc05::fence_mbar_init();
        timed_out = 0;
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = tmem_holder;
    constexpr uint32_t idesc = tc05::idesc_f16_f32(kBM, NI < 16 ? 16 : NI);

    // this thread's columns [hlf * 32, hlf * 32 + 32) of chunk kc, zero past the data
    auto load_chunk = [&](int kc, float (&rv)[CW]) {
        const int c0 = kc * kBK + hlf * CW;
        if (g < a.nK && c0 + CW <= D) {
            const float4 *src = reinterpret_cast<const float4 *>(a.resid + g * D + c0);
#pragma unroll
            for (int q = 0; q < CW / 4; ++q) {
                const float4 f = src[q];
                rv[4 * q] = f.x; rv[4 * q + 1] = f.y; rv[4 * q + 2] = f.z; rv[4 * q + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < CW; ++q) rv[q] = (g < a.nK && c0 + q < D) ? a.resid[g * D + c0 + q] : 0.f;
        }
    };
    float rnext[CW];
    load_chunk(0, rnext);

    for (int kc = 0; kc < NK; ++kc) {
        const int st = kc & 1;
        uint8_t *sA = smem + st * STAGE_BYTES;
        uint8_t *sB = sA + 2 * A_BYTES;
        if (kc >= 2 && !tc05::mbar_wait_bounded(&bar_mma[st], ((kc - 2) >> 1) & 1, kMaxPolls)) timed_out = 1;
        if constexpr (D >= 64) {
            if (tid == 0) {                                // S rows [n0, n0 + BN), columns of chunk kc
                tc05::mbar_expect_tx(&bar_b[st], uint32_t(B_BYTES));
#pragma unroll
                for (int nb = 0; nb < BN / NI; ++nb)
                    tc05::tma_load_2d(sB + nb * NI * 128, &tmS, kc * kBK, n0 + nb * NI, &bar_b[st]);
            }
        } else {
            // rows of fewer than 64 columns: the threads fill the swizzled tile, zero-padded
            for (int q = tid; q < BN * 8; q += kQThreads) {
                const int r = q >> 3, ch = q & 7;
                const int j = n0 + r, c = ch * 8;
                uint16_t tmp[8];
#pragma unroll
                for (int z = 0; z < 8; ++z) tmp[z] = (j < M && c + z < D) ? a.S16[size_t(j) * D + c + z] : 0;
                *reinterpret_cast<uint4 *>(sB + tc05::sw128_offset(uint32_t(r), uint32_t(ch))) =
                    make_uint4(tmp[0] | (uint32_t(tmp[1]) << 16), tmp[2] | (uint32_t(tmp[3]) << 16),
                               tmp[4] | (uint32_t(tmp[5]) << 16), tmp[6] | (uint32_t(tmp[7]) << 16));
            }
        }
        float rv[CW];
#pragma unroll
        for (int q = 0; q < CW; ++q) rv[q] = rnext[q];
        if (kc + 1 < NK) load_chunk(kc + 1, rnext);       // in flight while this chunk is converted
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {                   // four 16-byte pieces of hi and of lo
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float x0 = rv[ch * 8 + 2 * k], x1 = rv[ch * 8 + 2 * k + 1];
                const __half2 h = __floats2half2_rn(x0, x1);
                const float2 hf = __half22float2(h);
                const __half2 l = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
                hi[k] = *reinterpret_cast<const uint32_t *>(&h);
                lo[k] = *reinterpret_cast<const uint32_t *>(&l);
            }
            const uint32_t o = tc05::sw128_offset(uint32_t(row), uint32_t(hlf * 4 + ch));
            *reinterpret_cast<uint4 *>(sA + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(sA + A_BYTES + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        tc05::fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            if (D >= 64 && !tc05::mbar_wait_bounded(&bar_b[st], uint32_t(kc >> 1) & 1u, kMaxPolls)) timed_out = 1;
            tc05::fence_after_sync();
            const uint32_t aBase = tc05::smem_u32(sA), bBase = tc05::smem_u32(sB);
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks) {
#pragma unroll
                for (int nb = 0; nb < BN / NI; ++nb) {
                    const uint64_t bdesc = tc05::desc_kmajor_sw128(bBase + nb * NI * 128 + ks * 32);
#pragma unroll
                    for (int sp = 0; sp < 2; ++sp) {
                        const uint64_t adesc = tc05::desc_kmajor_sw128(aBase + sp * A_BYTES + ks * 32);
                        tc05::mma_f16(tmem + uint32_t(nb * NI), adesc, bdesc, idesc, (kc | ks | sp) != 0);
                    }
                }
            }
            tc05::mma_commit(&bar_mma[st]);
        }
    }
    if (!tc05::mbar_wait_bounded(&bar_mma[(NK - 1) & 1], ((NK - 1) >> 1) & 1, kMaxPolls)) timed_out = 1;
    // a chunk's B copy that was issued is always waited for above before its MMA,
    // so no copy is in flight here
    tc05::fence_after_sync();

    // Epilogue: warps 0-3, thread = tile row (vector); TMEM lanes 32*warp .. +31.
    if (warp < 4) {
        const int64_t ge = row0 + warp * 32 + lane;
        uint8_t *ks_dst = nullptr;
        if (ge < a.nK) {
            const int64_t t = ge / a.L.H;
            const int h = int(ge - t * a.L.H);
            const int slot = a.slots[t];
            if (slot >= 0 && slot < a.num_slots) {
                uint8_t *page = a.cache + (int64_t(slot / a.L.P) * a.L.H + h) * int64_t(a.L.page_bytes);
                ks_dst = page + a.L.ks_off + (slot % a.L.P) * a.L.ks_bpt;
            }
        }
#pragma unroll 1
        for (int c = 0; c < (BN + 31) / 32; ++c) {
            uint32_t r[32];
            tc05::tmem_ld_32x32b_x32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(c * 32), r);
            tc05::tmem_wait_ld();
            uint32_t bits = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) bits |= (__uint_as_float(r[k]) >= 0.f ? 1u : 0u) << k;
            const int j0 = n0 + c * 32;
            if (ks_dst && !timed_out) {
                if (M >= 32) {
                    if (j0 < M) reinterpret_cast<uint32_t *>(ks_dst)[j0 >> 5] = bits;
                } else {
                    for (int b = 0; b < M / 8; ++b) ks_dst[b] = uint8_t(bits >> (8 * b));
                }
            }
        }
    }
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, TCOLS);
    }
    if (tid == 0 && timed_out) atomicOr(a.status, TQ_DEV_WAIT_TIMEOUT);
}

template <int D>
constexpr int qjl_bn() { return D >= 512 ? 512 : (D < 16 ? 16 : D); }

PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
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

// 2-D map over S (fp16 [D][D], row-major): boxes of 64 columns x box_rows
// rows with the 128-byte swizzle; rows past D (D < 16) read as zero.
bool make_s_map(CUtensorMap *m, const uint16_t *S16, int D, int box_rows) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(D)};
    cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    cuuint32_t box[2] = {cuuint32_t(D < 64 ? D : 64), cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(S16), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, D < 64 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
int launch_qjl(const QjlArgs &q, const uint16_t *S16, cudaStream_t st) {
    constexpr int BN = qjl_bn<D>();
    constexpr size_t smem = 2 * (2 * kBM * 128 + BN * 128) + 1024;
    CUtensorMap tm;
    std::memset(&tm, 0, sizeof(tm));
    if (D >= 64 && !make_s_map(&tm, S16, D, BN < 256 ? BN : 256)) return cudaErrorInvalidValue;
    auto kern = qjl_gemm_kernel<D, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned((D + BN - 1) / BN), unsigned((q.nK + kBM - 1) / kBM));
    kern<<<grid, kQThreads, smem, st>>>(tm, q);
    return cudaGetLastError();
}

template <int D>
int launch_encode_d(const EncodeArgs &a, int in_dtype, const tq_params *kp, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t nvec = a.n_tokens * a.L.H * (a.do_v ? 2 : 1);
    int64_t blocks = (nvec + 7) / 8;
    const int64_t cap = int64_t(sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    bool dense = false;
    if constexpr (D <= 256) dense = a.kp.rot || (a.do_v && a.vp.rot);
    if (dense) {
        if constexpr (D <= 256) {
            if (in_dtype == TQ_DTYPE_BF16) encode_dense_kernel<D, __nv_bfloat16><<<unsigned(blocks), 256, 0, st>>>(a);
            else encode_dense_kernel<D, float><<<unsigned(blocks), 256, 0, st>>>(a);
        }
    } else if (in_dtype == TQ_DTYPE_BF16) {
        encode_kernel<D, __nv_bfloat16><<<unsigned(blocks), 256, 0, st>>>(a);
    } else {
        encode_kernel<D, float><<<unsigned(blocks), 256, 0, st>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (a.L.kqjl && a.n_tokens > 0) {
        QjlArgs q;
        q.L = a.L;
        q.resid = a.resid;
        q.S16 = kp->dev.S16;
        q.nK = a.n_tokens * a.L.H;
        q.slots = a.slots;
        q.num_slots = a.num_slots;
        q.cache = a.cache;
        q.status = a.status;
        return launch_qjl<D>(q, kp->dev.S16, st);
    }
    return cudaSuccess;
}

}  // namespace

size_t encode_ws_bytes(const Layout &L, int64_t n_tokens) {
    size_t b = kWsHeader;
    if (L.kqjl) b += size_t(n_tokens) * L.H * L.d * sizeof(float);
    return b;
}

int launch_encode(const tq_params *kp, const tq_params *vp, const Layout &L, const void *K, const void *V,
                  int in_dtype, int64_t n_tokens, const int32_t *slots, uint8_t *cache, int64_t num_blocks,
                  uint8_t *ws, size_t ws_bytes, void *stream) {
    (void)ws_bytes;
    EncodeArgs a;
    a.L = L;
    a.kp = kp->dev;
    if (vp) a.vp = vp->dev;
    else a.vp = kp->dev;
    a.K = K;
    a.V = V;
    a.n_tokens = n_tokens;
    a.slots = slots;
    a.num_slots = num_blocks * L.P;
    a.cache = cache;
    a.resid = L.kqjl ? reinterpret_cast<float *>(ws + kWsHeader) : nullptr;
    a.status = reinterpret_cast<uint32_t *>(ws);
    a.do_v = L.vbits > 0 ? 1 : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (in_dtype == TQ_DTYPE_BF16) {
        const int r = launch_encode128(kp, vp, L, K, V, n_tokens, slots, cache, num_blocks, ws, stream);
        if (r >= 0) return r;
    }
    switch (L.d) {
        case 8: return launch_encode_d<8>(a, in_dtype, kp, st);
        case 16: return launch_encode_d<16>(a, in_dtype, kp, st);
        case 32: return launch_encode_d<32>(a, in_dtype, kp, st);
        case 64: return launch_encode_d<64>(a, in_dtype, kp, st);
        case 128: return launch_encode_d<128>(a, in_dtype, kp, st);
        case 256: return launch_encode_d<256>(a, in_dtype, kp, st);
        case 512: return launch_encode_d<512>(a, in_dtype, kp, st);
        case 1024: return launch_encode_d<1024>(a, in_dtype, kp, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tq
