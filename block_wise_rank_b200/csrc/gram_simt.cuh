// gram_simt.cuh -- per-block Gram matrix G_b = X_b^T X_b on CUDA cores.
//
// Step "SVD of K and of V per block" (evolve.pub review of MILO, Summary):
// the right singular vectors and singular values of X_b are the eigenvectors
// and square roots of the eigenvalues of its d x d Gram matrix.  This FP32
// FFMA kernel serves fp32 caches (tensor-core TF32 would cost the precision
// the singular values need) and is the portable fallback for bf16; the
// tcgen05 kernel in gram_tc.cuh serves bf16 caches.
#pragma once
#include "common.cuh"

namespace milo {

// grid (N_blk, 2 kinds), 256 threads; thread (ti, tj) owns the 8x8 tile
// G[8ti .. 8ti+7][8tj .. 8tj+7].  Tokens stream through shared memory in
// chunks of 32 rows.  G is written row-major to G_out[kind][blk][128][128].
template <typename T>
__global__ void __launch_bounds__(256) k_gram_simt(const T *__restrict__ K, const T *__restrict__ V,
                                                    int H, BlockGeo geo, int n_b,
                                                    float *__restrict__ G_out, int64_t n_blk) {
    __shared__ __align__(16) float xs[32][D + 4];
    const int blk = blockIdx.x;
    const int kind = blockIdx.y;
    const T *X = kind == 0 ? K : V;
    const int lh = blk / n_b, b = blk % n_b;
    const int Tb = geo.len(b);
    const T *Xb = X + ((int64_t)lh * geo.T + geo.start(b)) * D;
    const int tid = threadIdx.x;
    const int ti = tid / 16, tj = tid % 16;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;

    for (int t0 = 0; t0 < Tb; t0 += 32) {
        const int tt = min(32, Tb - t0);
        for (int e = tid; e < 32 * D; e += 256) {
            int t = e / D, j = e % D;
            xs[t][j] = t < tt ? to_f32<T>(Xb[(int64_t)(t0 + t) * D + j]) : 0.f;
        }
        __syncthreads();
        for (int t = 0; t < tt; ++t) {
            float xi[8], xj[8];
            const float4 *ri = reinterpret_cast<const float4 *>(&xs[t][8 * ti]);
            const float4 *rj = reinterpret_cast<const float4 *>(&xs[t][8 * tj]);
            float4 u0 = ri[0], u1 = ri[1], v0 = rj[0], v1 = rj[1];
            xi[0] = u0.x; xi[1] = u0.y; xi[2] = u0.z; xi[3] = u0.w;
            xi[4] = u1.x; xi[5] = u1.y; xi[6] = u1.z; xi[7] = u1.w;
            xj[0] = v0.x; xj[1] = v0.y; xj[2] = v0.z; xj[3] = v0.w;
            xj[4] = v1.x; xj[5] = v1.y; xj[6] = v1.z; xj[7] = v1.w;
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(xi[a], xj[c], acc[a][c]);
        }
        __syncthreads();
    }
    float *G = G_out + ((int64_t)kind * n_blk + blk) * D * D;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        float4 *dst = reinterpret_cast<float4 *>(&G[(8 * ti + a) * D + 8 * tj]);
        dst[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        dst[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    }
}

}  // namespace milo
