// QJL projection of rotated queries: w = S q_r for a batch of rows.
//
// ai-work-lab overview, "QJL" (the estimator's correction term takes the
// inner product of the projected query S R q with the stored signs).  The
// projection is a small dense product [rows x d] x S^T [d x d]; it runs as a
// shared-memory tiled fp32 kernel (16 or 64 rows x 64 outputs per block), S
// read from its bf16 copy.  fp32 keeps the full-precision w that the general
// kernels use; the tensor-core paths round it afterwards.
#include <cuda_runtime.h>

#include "tq_dev.cuh"

namespace tq {
namespace {

constexpr int kTJ = 64, kTK = 32;

// TR rows x 64 outputs per block, (TR / 16) x 4 per thread.
template <int TR>
__global__ void __launch_bounds__(256) qproj_kernel(const float *qr, int64_t rows, int D, const uint16_t *S,
                                                    float *w) {
    constexpr int RPT = TR / 16;
    __shared__ float sq[kTK][TR + 4];
    __shared__ float ss[kTK][kTJ + 4];
    const int tid = threadIdx.x, tr = tid >> 4, tj = tid & 15;
    const int64_t r0 = int64_t(blockIdx.x) * TR;
    const int j0 = blockIdx.y * kTJ;
    float acc[RPT][4] = {};
    for (int k0 = 0; k0 < D; k0 += kTK) {
        // stage q_r[r0 .. r0+TR-1][k0 .. k0+31] and S[j0 .. j0+63][k0 .. k0+31], transposed
        for (int i = tid; i < TR * kTK; i += 256) {
            const int r = i / kTK, k = i % kTK;
            const int64_t row = r0 + r;
            sq[k][r] = (row < rows && k0 + k < D) ? qr[row * D + k0 + k] : 0.f;
        }
        for (int i = tid; i < kTJ * kTK; i += 256) {
            const int r = i / kTK, k = i % kTK;
            const int j = j0 + r;
            ss[k][r] = (j < D && k0 + k < D) ? __uint_as_float(uint32_t(S[size_t(j) * D + k0 + k]) << 16) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kTK; ++k) {
            float av[RPT];
#pragma unroll
            for (int x = 0; x < RPT; ++x) av[x] = sq[k][tr * RPT + x];
            const float4 b = *reinterpret_cast<const float4 *>(&ss[k][tj * 4]);
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int x = 0; x < RPT; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < RPT; ++x) {
        const int64_t row = r0 + tr * RPT + x;
        if (row >= rows) continue;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int j = j0 + tj * 4 + y;
            if (j < D) w[row * D + j] = acc[x][y];
        }
    }
}

}  // namespace

int launch_qproj(const float *qr, int64_t rows, int D, const uint16_t *S, float *w, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    if (D <= 256) {          // small products: more, smaller blocks
        const dim3 grid(unsigned((rows + 15) / 16), unsigned((D + kTJ - 1) / kTJ));
        qproj_kernel<16><<<grid, 256, 0, st>>>(qr, rows, D, S, w);
    } else {
        const dim3 grid(unsigned((rows + 63) / 64), unsigned((D + kTJ - 1) / kTJ));
        qproj_kernel<64><<<grid, 256, 0, st>>>(qr, rows, D, S, w);
    }
    return cudaGetLastError();
}

}  // namespace tq
