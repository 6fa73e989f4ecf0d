// QJL projection of rotated queries: w = S q_r for a batch of rows.
//
// ai-work-lab overview, "QJL" (the estimator's correction term takes the
// inner product of the projected query S R q with the stored signs).  The
// projection is a small dense product [rows x d] x S^T [d x d]; it runs as a
// shared-memory tiled fp32 kernel (64 rows x 64 outputs per block, 4 x 4 per
// thread), S read from its bf16 copy.  fp32 keeps the full-precision w that
// the general kernels use; the tensor-core paths round it afterwards.
#include <cuda_runtime.h>

#include "tq_dev.cuh"

namespace tq {
namespace {

constexpr int kTR = 64, kTJ = 64, kTK = 32;

__global__ void __launch_bounds__(256) qproj_kernel(const float *qr, int64_t rows, int D, const uint16_t *S,
                                                    float *w) {
    __shared__ float sq[kTK][kTR + 4];
    __shared__ float ss[kTK][kTJ + 4];
    const int tid = threadIdx.x, tr = tid >> 4, tj = tid & 15;
    const int64_t r0 = int64_t(blockIdx.x) * kTR;
    const int j0 = blockIdx.y * kTJ;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < D; k0 += kTK) {
        // stage q_r[r0 .. r0+63][k0 .. k0+31] and S[j0 .. j0+63][k0 .. k0+31], transposed
        for (int i = tid; i < kTR * kTK; i += 256) {
            const int r = i / kTK, k = i % kTK;
            const int64_t row = r0 + r;
            sq[k][r] = (row < rows && k0 + k < D) ? qr[row * D + k0 + k] : 0.f;
            const int j = j0 + r;
            ss[k][r] = (j < D && k0 + k < D) ? __uint_as_float(uint32_t(S[size_t(j) * D + k0 + k]) << 16) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kTK; ++k) {
            const float4 a = *reinterpret_cast<const float4 *>(&sq[k][tr * 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&ss[k][tj * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int64_t row = r0 + tr * 4 + x;
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
    const dim3 grid(unsigned((rows + kTR - 1) / kTR), unsigned((D + kTJ - 1) / kTJ));
    qproj_kernel<<<grid, 256, 0, st>>>(qr, rows, D, S, w);
    return cudaGetLastError();
}

}  // namespace tq
