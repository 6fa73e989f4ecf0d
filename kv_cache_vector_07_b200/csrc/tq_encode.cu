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
#include <cuda_runtime.h>
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

template <int D, typename TIn>
__global__ void __launch_bounds__(256) encode_kernel(EncodeArgs a) {
    constexpr int E = WarpVec<D>::E;
    __shared__ float wbuf[8][warp_buf_floats<D>()];
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
        if (encode_vector_warp<D>(L, P, is_v, x, page, pos, lane, r, wbuf[threadIdx.x >> 5])) {
            // the residual is stored times 2^e with ||r|| 2^e in [2^10, 2^11): the
            // projection's fp16 hi + lo parts then stay normal, and its signs do
            // not depend on a positive scale
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
                float *dst = a.resid + v * D + lane * E;
#pragma unroll
                for (int e = 0; e < E; ++e) dst[e] = r[e] * sc;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// QJL projection on the tensor cores.
// ---------------------------------------------------------------------------
struct QjlArgs {
    Layout L;
    const uint16_t *S16;    // [m][D] fp16 bits, m = D
    const float *resid;     // [nK][D], each row scaled by a power of two
    int64_t nK;             // n_tokens * H
    const int32_t *slots;
    int64_t num_slots;
    uint8_t *cache;
    uint32_t *status;
};

constexpr int kBM = 128;       // vectors per tile (MMA M)
constexpr int kBK = 64;        // K elements per stage (one 128-byte swizzle row)
constexpr uint32_t kMaxPolls = 1u << 20;   // about a second of polling, then give up

// z = S r for a tile of 128 residuals against BN projection rows, on the
// tensor cores.  r (fp32, scaled per row by a power of two) is split into
// fp16 hi + lo (22 bits; the scale keeps both parts normal) against the
// fp16 copy of S (exact for |S| >= 2^-14); two MMAs per k-step and per 256
// output columns, fp32 accumulators in TMEM (BN = 512 fills all of it).  The
// epilogue packs the sign bits [z_j >= 0] into the page.  The grid runs the
// N tiles of one residual tile next to each other, so the tile's rows are
// read from DRAM once and served to the others from L2.
template <int D, int BN>
__global__ void __launch_bounds__(128, 1) qjl_gemm_kernel(QjlArgs a) {
    constexpr int M = D;                                   // projection rows
    constexpr int NK = (D + kBK - 1) / kBK;
    constexpr int NI = BN < 256 ? BN : 256;                // N of one MMA
    constexpr uint32_t TCOLS = BN < 32 ? 32 : BN;
    constexpr int A_BYTES = kBM * 128;                     // one split tile
    constexpr int B_BYTES = BN * 128;
    constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar[2];
    __shared__ uint32_t tmem_holder;
    __shared__ int timed_out;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * BN;
    const int64_t row0 = int64_t(blockIdx.y) * kBM;

    if (warp == 0) {
        tc05::tmem_alloc(&tmem_holder, TCOLS);
        tc05::tmem_relinquish();
    }
    if (tid == 0) {
        tc05::mbar_init(&bar[0], 1);
        tc05::mbar_init(&bar[1], 1);
        tc05::fence_mbar_init();
        timed_out = 0;
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = tmem_holder;
    constexpr uint32_t idesc = tc05::idesc_f16_f32(kBM, NI < 16 ? 16 : NI);

    for (int kc = 0; kc < NK; ++kc) {
        const int st = kc & 1;
        uint8_t *sA = smem + st * STAGE_BYTES;
        uint8_t *sB = sA + 2 * A_BYTES;
        if (kc >= 2) {
            if (!tc05::mbar_wait_bounded(&bar[st], ((kc - 2) >> 1) & 1, kMaxPolls)) timed_out = 1;
        }
        // A: row tid of this tile, columns [kc*64, kc*64+64) of r as fp16 hi + lo
        {
            const int64_t g = row0 + tid;
            float rv[kBK];
            const int c0 = kc * kBK;
            if (g < a.nK && c0 + kBK <= D) {
                const float4 *src = reinterpret_cast<const float4 *>(a.resid + g * D + c0);
#pragma unroll
                for (int q = 0; q < kBK / 4; ++q) {
                    float4 f = src[q];
                    rv[4 * q] = f.x; rv[4 * q + 1] = f.y; rv[4 * q + 2] = f.z; rv[4 * q + 3] = f.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < kBK; ++q) rv[q] = (g < a.nK && c0 + q < D) ? a.resid[g * D + c0 + q] : 0.f;
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
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
                const uint32_t o = tc05::sw128_offset(tid, ch);
                *reinterpret_cast<uint4 *>(sA + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(sA + A_BYTES + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        // B: BN rows of S (fp16), same 64 columns
        for (int q = tid; q < BN * 8; q += 128) {
            const int row = q >> 3, ch = q & 7;
            const int j = n0 + row, c = kc * kBK + ch * 8;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (j < M && c + 8 <= D) {
                val = *reinterpret_cast<const uint4 *>(a.S16 + size_t(j) * D + c);
            } else if (j < M && c < D) {
                uint16_t tmp[8];
#pragma unroll
                for (int z = 0; z < 8; ++z) tmp[z] = (c + z < D) ? a.S16[size_t(j) * D + c + z] : 0;
                val = make_uint4(tmp[0] | (uint32_t(tmp[1]) << 16), tmp[2] | (uint32_t(tmp[3]) << 16),
                                 tmp[4] | (uint32_t(tmp[5]) << 16), tmp[6] | (uint32_t(tmp[7]) << 16));
            }
            *reinterpret_cast<uint4 *>(sB + tc05::sw128_offset(row, ch)) = val;
        }
        tc05::fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc05::fence_after_sync();
            const uint32_t aBase = tc05::smem_u32(sA), bBase = tc05::smem_u32(sB);
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks) {
#pragma unroll
                for (int nb = 0; nb < BN / NI; ++nb) {
                    // rows nb*NI .. of the B tile: 8-row groups are 1024 bytes apart
                    const uint64_t bdesc = tc05::desc_kmajor_sw128(bBase + nb * NI * 128 + ks * 32);
#pragma unroll
                    for (int sp = 0; sp < 2; ++sp) {
                        const uint64_t adesc = tc05::desc_kmajor_sw128(aBase + sp * A_BYTES + ks * 32);
                        tc05::mma_f16(tmem + uint32_t(nb * NI), adesc, bdesc, idesc, (kc | ks | sp) != 0);
                    }
                }
            }
            tc05::mma_commit(&bar[st]);
        }
    }
    if (!tc05::mbar_wait_bounded(&bar[(NK - 1) & 1], ((NK - 1) >> 1) & 1, kMaxPolls)) timed_out = 1;
    tc05::fence_after_sync();

    // Epilogue: thread = tile row (vector); TMEM lanes 32*warp .. +31.
    const int64_t g = row0 + warp * 32 + lane;
    uint8_t *ks_dst = nullptr;
    if (g < a.nK) {
        const int64_t t = g / a.L.H;
        const int h = int(g - t * a.L.H);
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

template <int D>
int launch_qjl(const QjlArgs &q, cudaStream_t st) {
    constexpr int BN = qjl_bn<D>();
    constexpr size_t smem = 2 * (2 * kBM * 128 + BN * 128) + 1024;
    auto kern = qjl_gemm_kernel<D, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned((D + BN - 1) / BN), unsigned((q.nK + kBM - 1) / kBM));
    kern<<<grid, 128, smem, st>>>(q);
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
    if (in_dtype == TQ_DTYPE_BF16) encode_kernel<D, __nv_bfloat16><<<unsigned(blocks), 256, 0, st>>>(a);
    else encode_kernel<D, float><<<unsigned(blocks), 256, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (a.L.kqjl && a.n_tokens > 0) {
        QjlArgs q;
        q.L = a.L;
        q.S16 = kp->dev.S16;
        q.resid = a.resid;
        q.nK = a.n_tokens * a.L.H;
        q.slots = a.slots;
        q.num_slots = a.num_slots;
        q.cache = a.cache;
        q.status = a.status;
        return launch_qjl<D>(q, st);
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
