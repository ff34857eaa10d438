// refine.cuh -- singular values from the block itself: sigma_k = ||X_b w_k||.
//
// Step "SVD of K and of V per block" (evolve.pub review of MILO, Summary).
// The eigenvalues of an fp32 Gram matrix carry an error of order
// eps * sigma_1^2, i.e. eps * sigma_1^2 / sigma_k on sigma_k.  The norm of
// X_b times a computed right singular vector is a Rayleigh quotient of
// X_b^T X_b evaluated without forming it, so its error is second order in
// the eigenvector error.  This kernel recomputes every sigma_k that way, in
// FP32 on the block itself (after scaling each w_k to unit length), and
// re-sorts sigma and the columns of W in
// descending order (ties keep the eigensolver's order).  Singular values
// past min(T_b, d) are set to 0: the block's rank is at most T_b.
#pragma once
#include "common.cuh"

namespace milo {

constexpr int RF_THREADS = 256;
constexpr int RF_TT = 32;

struct RefineSmem {
    float W[D][D + 1];
    float xs[RF_TT][D + 4];
    float part[RF_THREADS];
    float sig[D];
    int rank[D];
};

// grid (n_blk, 2 kinds).  W_io: [2][n_blk][D][D] sorted eigenvectors (in),
// re-sorted by the refined sigma (out).  sigma_K/sigma_V: [n_blk][D] (out).
template <typename T>
__global__ void __launch_bounds__(RF_THREADS) k_refine_sigma(const T *__restrict__ K, const T *__restrict__ V,
                                                             float *__restrict__ W_io, float *__restrict__ sigma_K,
                                                             float *__restrict__ sigma_V, BlockGeo geo, int n_b,
                                                             int64_t n_blk) {
    extern __shared__ __align__(16) unsigned char rf_raw[];
    RefineSmem &sm = *reinterpret_cast<RefineSmem *>(rf_raw);
    const int blk = blockIdx.x, kind = blockIdx.y, tid = threadIdx.x;
    const int lh = blk / n_b, b = blk % n_b;
    const int Tb = geo.len(b);
    const T *Xb = (kind == 0 ? K : V) + ((int64_t)lh * geo.T + geo.start(b)) * D;
    float *Wg = W_io + ((int64_t)kind * n_blk + blk) * D * D;
    for (int e = tid; e < D * D; e += RF_THREADS) sm.W[e / D][e % D] = Wg[e];
    __syncthreads();
    // unit columns: rounding in the accumulated rotations lets the column
    // norms of W drift from 1 by far more than their directions move
    if (tid < D) {
        float n2 = 0.f;
        for (int j = 0; j < D; ++j) n2 = fmaf(sm.W[j][tid], sm.W[j][tid], n2);
        sm.sig[tid] = n2 > 0.f ? 1.f / sqrtf(n2) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < D * D; e += RF_THREADS) sm.W[e / D][e % D] *= sm.sig[e % D];
    const int k = tid % D, half = tid / D;   // column k, tokens of parity `half`
    float acc = 0.f;
    for (int t0 = 0; t0 < Tb; t0 += RF_TT) {
        const int tt = min(RF_TT, Tb - t0);
        __syncthreads();
        for (int e = tid; e < RF_TT * D; e += RF_THREADS) {
            const int t = e / D, j = e % D;
            sm.xs[t][j] = t < tt ? to_f32<T>(Xb[(int64_t)(t0 + t) * D + j]) : 0.f;
        }
        __syncthreads();
        for (int t = half; t < tt; t += 2) {
            float y = 0.f;
            const float4 *xr = reinterpret_cast<const float4 *>(sm.xs[t]);
#pragma unroll 8
            for (int j4 = 0; j4 < D / 4; ++j4) {
                const float4 x = xr[j4];
                y = fmaf(x.x, sm.W[4 * j4 + 0][k], y);
                y = fmaf(x.y, sm.W[4 * j4 + 1][k], y);
                y = fmaf(x.z, sm.W[4 * j4 + 2][k], y);
                y = fmaf(x.w, sm.W[4 * j4 + 3][k], y);
            }
            acc = fmaf(y, y, acc);
        }
    }
    sm.part[tid] = acc;
    __syncthreads();
    if (tid < D) sm.sig[tid] = sqrtf(sm.part[tid] + sm.part[tid + D]);
    __syncthreads();
    if (tid < D) {
        const float s = sm.sig[tid];
        int rk = 0;
        for (int j = 0; j < D; ++j) {
            const float o = sm.sig[j];
            rk += (o > s) || (o == s && j < tid);
        }
        sm.rank[tid] = rk;
        if (!isfinite(s)) raise_status(ST_NONFINITE);
        float *out = (kind == 0 ? sigma_K : sigma_V) + (int64_t)blk * D;
        out[rk] = rk < Tb ? s : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < D * D; e += RF_THREADS) {
        const int j = e / D, kk = e % D;
        Wg[j * D + sm.rank[kk]] = sm.W[j][kk];
    }
}

inline size_t refine_smem_bytes() { return sizeof(RefineSmem); }

}  // namespace milo
