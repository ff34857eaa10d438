// jacobi.cuh -- batched one-sided Jacobi on the d x d Gram tile, one CTA per
// (block, kind), the tile held in shared memory.
//
// Step "SVD of K and of V per block" (evolve.pub review of MILO, Summary).
// One-sided (Hestenes) Jacobi orthogonalises the columns of X_b by plane
// rotations; the rotation for the column pair (p, q) is decided by the three
// inner products a_p.a_p, a_q.a_q and a_p.a_q, which are the entries of the
// rotated Gram matrix G' = W^T G W.  Keeping G' (d x d) in shared memory
// instead of X_b (T_b x d) turns each column rotation into the symmetric
// update G' <- J^T G' J and the accumulation W <- W J; X_b itself is rotated
// once, at the end, by the projection A_b = X_b W (project.cuh).  The
// converged diagonal holds sigma_k^2 and W the right singular vectors.
//
// Parallel order: the round-robin ("circle") tournament -- 127 rounds of 64
// disjoint pairs per sweep; pairs of one round commute, so all 64 rotations
// of a round are applied at once.  A sweep with no rotation ends the solve;
// the sweep cap raises ST_NOT_CONVERGED and still writes the current result.
#pragma once
#include "common.cuh"

#ifndef MILO_TRACE_JACOBI
#define MILO_TRACE_JACOBI(sweeps)
#endif

namespace milo {

// plane rotations applied in the counted rounds (at most 64 per round)
__device__ unsigned long long g_jacobi_rotations;

constexpr int JAC_THREADS = 512;
constexpr int JAC_NPAIR = D / 2;                       // 64 pairs per round
constexpr int JAC_NTRI = JAC_NPAIR * (JAC_NPAIR + 1) / 2;  // 2080 pair blocks (i <= i2)
constexpr int JAC_LD = D + 1;                          // padded row stride of W
constexpr int JAC_GT = D * (D + 1) / 2;                // packed upper triangle of G

// G is symmetric and only its upper triangle is stored, packed by rows:
// entry (x, y) lives at row u = min(x, y), offset max(x, y) - u into a row
// that starts at u (2d - u + 1) / 2.  (Half of the full tile, so that two
// CTAs fit on an SM.)
__device__ __forceinline__ int jac_g(int x, int y) {
    const int u = min(x, y), v = max(x, y);
    return ((u * (2 * D + 1 - u)) >> 1) + (v - u);
}

struct JacobiSmem {
    float G[JAC_GT];
    float W[D * JAC_LD];
    float4 rot[JAC_NPAIR];   // per pair of the round: (c, s, p, q), p and q as int bits
    float t[JAC_NPAIR];
    unsigned short tri[JAC_NTRI][2];
    float lam[D];
    int rank[D];
    float floor_abs;
};

// G_io: [2][n_blk][128][128] fp32.  In: the Gram matrices.  Out: the
// eigenvectors, columns sorted by descending eigenvalue (W[j][k] = v_k[j]).
// sigma_K/sigma_V: [n_blk][128] singular values, descending; entries past
// min(T_b, d) are set to 0 (the rank of a T_b x d block).
__global__ void __launch_bounds__(JAC_THREADS, 2)
k_jacobi(float *__restrict__ G_io, float *__restrict__ sigma_K, float *__restrict__ sigma_V,
         int64_t n_blk, BlockGeo geo, int n_b, int max_sweeps, float tol) {
    extern __shared__ __align__(16) unsigned char jac_raw[];
    JacobiSmem &sm = *reinterpret_cast<JacobiSmem *>(jac_raw);
    const int tid = threadIdx.x;
    const int blk = blockIdx.x, kind = blockIdx.y;
    float *Gg = G_io + ((int64_t)kind * n_blk + blk) * D * D;

    for (int e = tid; e < D * D; e += JAC_THREADS) {
        int i = e / D, j = e % D;
        if (i <= j) sm.G[jac_g(i, j)] = Gg[e];
        sm.W[i * JAC_LD + j] = (i == j) ? 1.f : 0.f;
    }
    for (int e = tid; e < JAC_NTRI; e += JAC_THREADS) {
        // enumerate pair blocks (i, i2) with i <= i2
        int i = 0, rem = e;
        while (rem >= JAC_NPAIR - i) { rem -= JAC_NPAIR - i; ++i; }
        sm.tri[e][0] = (unsigned short)i;
        sm.tri[e][1] = (unsigned short)(i + rem);
    }
    __syncthreads();
    if (tid < 32) {
        float tr = 0.f;
        for (int k = tid; k < D; k += 32) tr += fabsf(sm.G[jac_g(k, k)]);
        for (int o = 16; o; o >>= 1) tr += __shfl_xor_sync(0xffffffffu, tr, o);
        if (tid == 0) sm.floor_abs = 1e-10f * tr;
    }
    __syncthreads();
    const float floor_abs = sm.floor_abs;

    bool converged = false;
    int sweeps_done = 0;
    unsigned rounds_applied = 0, rotations = 0;
    for (int sweep = 0; sweep < max_sweeps && !converged; ++sweep) {
        ++sweeps_done;
        int any = 0;
        for (int r = 0; r < D - 1; ++r) {
            int rot = 0;
            if (tid < JAC_NPAIR) {
                int a, b;
                if (tid == 0) { a = r; b = D - 1; }
                else { a = (r + tid) % (D - 1); b = (r - tid + (D - 1)) % (D - 1); }
                int p = min(a, b), q = max(a, b);
                float app = sm.G[jac_g(p, p)], aqq = sm.G[jac_g(q, q)], apq = sm.G[jac_g(p, q)];
                float c = 1.f, s = 0.f, tn = 0.f;
                if (fabsf(apq) > floor_abs && fabsf(apq) > tol * sqrtf(fabsf(app)) * sqrtf(fabsf(aqq))) {
                    float zeta = (aqq - app) / (2.f * apq);
                    tn = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
                    c = 1.f / sqrtf(1.f + tn * tn);
                    s = c * tn;
                    rot = 1;
                }
                sm.rot[tid] = make_float4(c, s, __int_as_float(p), __int_as_float(q));
                sm.t[tid] = tn;
            }
            const int nrot = __syncthreads_count(rot);   // rotating pairs of this round
            rot = nrot > 0;
            any |= rot;
            if (!rot) continue;   // uniform across the CTA
            ++rounds_applied;
            rotations += nrot;
            // G <- J^T G J on every 2x2 pair block (i, i2), i <= i2 (upper triangle)
            for (int e = tid; e < JAC_NTRI; e += JAC_THREADS) {
                const int i = sm.tri[e][0], i2 = sm.tri[e][1];
                const float4 r1 = sm.rot[i];
                const int p = __float_as_int(r1.z), q = __float_as_int(r1.w);
                const float c1 = r1.x, s1 = r1.y;
                if (i == i2) {
                    if (s1 != 0.f) {
                        const float tn = sm.t[i];
                        const int ipq = jac_g(p, q);
                        const float apq = sm.G[ipq];
                        sm.G[jac_g(p, p)] -= tn * apq;
                        sm.G[jac_g(q, q)] += tn * apq;
                        sm.G[ipq] = 0.f;
                    }
                    continue;
                }
                const float4 r2 = sm.rot[i2];
                const float c2 = r2.x, s2 = r2.y;
                if (s1 == 0.f && s2 == 0.f) continue;   // neither pair rotates: block unchanged
                const int p2 = __float_as_int(r2.z), q2 = __float_as_int(r2.w);
                const int ia = jac_g(p, p2), ib = jac_g(p, q2), ic = jac_g(q, p2), ie = jac_g(q, q2);
                const float a = sm.G[ia], bb = sm.G[ib];
                const float cc = sm.G[ic], ee = sm.G[ie];
                // columns (p2, q2) by J2, then rows (p, q) by J1^T
                const float a1 = c2 * a - s2 * bb, b1 = s2 * a + c2 * bb;
                const float c1_ = c2 * cc - s2 * ee, e1 = s2 * cc + c2 * ee;
                const float na = c1 * a1 - s1 * c1_, nc = s1 * a1 + c1 * c1_;
                const float nb = c1 * b1 - s1 * e1, ne = s1 * b1 + c1 * e1;
                sm.G[ia] = na;
                sm.G[ib] = nb;
                sm.G[ic] = nc;
                sm.G[ie] = ne;
            }
            // W <- W J: columns (p_i, q_i) of every row; consecutive threads take
            // consecutive rows of one pair (row stride 129: no bank conflicts)
            for (int e = tid; e < D * JAC_NPAIR; e += JAC_THREADS) {
                const int j = e % D, i = e / D;
                const float4 r1 = sm.rot[i];
                const float s1 = r1.y;
                if (s1 == 0.f) continue;
                const float c1 = r1.x;
                const int p = __float_as_int(r1.z), q = __float_as_int(r1.w);
                const float wp = sm.W[j * JAC_LD + p], wq = sm.W[j * JAC_LD + q];
                sm.W[j * JAC_LD + p] = c1 * wp - s1 * wq;
                sm.W[j * JAC_LD + q] = s1 * wp + c1 * wq;
            }
            __syncthreads();
        }
        if (!any) converged = true;
    }
    if (!converged && tid == 0) raise_status(ST_NOT_CONVERGED);
    MILO_TRACE_JACOBI(sweeps_done);
    if (tid == 0) {
        atomicAdd(&g_jacobi_rounds, (unsigned long long)rounds_applied);
        atomicAdd(&g_jacobi_rotations, (unsigned long long)rotations);
    }

    // eigenvalues, stable descending order
    if (tid < D) sm.lam[tid] = sm.G[jac_g(tid, tid)];
    __syncthreads();
    if (tid < D) {
        const float lk = sm.lam[tid];
        int rk = 0;
        for (int j = 0; j < D; ++j) {
            const float lj = sm.lam[j];
            rk += (lj > lk) || (lj == lk && j < tid);
        }
        sm.rank[tid] = rk;
        if (!isfinite(lk)) raise_status(ST_NONFINITE);
        float *sig = (kind == 0 ? sigma_K : sigma_V) + (int64_t)blk * D;
        // X_b has rank <= T_b: singular values past min(T_b, d) are exactly 0
        const int Tb = geo.len(blk % n_b);
        sig[rk] = rk < Tb ? sqrtf(fmaxf(lk, 0.f)) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < D * D; e += JAC_THREADS) {
        const int j = e / D, k = e % D;
        Gg[j * D + sm.rank[k]] = sm.W[j * JAC_LD + k];
    }
}

inline size_t jacobi_smem_bytes() { return sizeof(JacobiSmem); }

}  // namespace milo
