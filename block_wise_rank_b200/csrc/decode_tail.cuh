// decode_tail.cuh -- dense attention over each session's recent, uncompressed
// tokens, merged into the same softmax as the retrieved compressed blocks.
//
// "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression" (evolve.pub review), Summary and FAQ "What is MILO": the
// compressed cache holds the many-shot demonstrations; a query rebuilds the
// blocks it retrieves and then attends sparsely.  The tokens after the
// demonstrations (the question and what has been generated so far) are not
// part of the compressed cache, so a complete decode step also attends to
// them, uncompressed, in the same softmax.  Their keys come as the model
// cached them: already rotated to their own positions, like q.
//
// One CTA per (KV head, session, layer) reads that head's tail once for all
// of its G query heads: 32-token rounds of K and V staged in shared memory,
// score dot products split over the four warps by quarters of d, an online
// softmax per query head, and thread j accumulating output channel j.  The
// result is one more partial (max, sum, normalised output) per query row,
// which k_combine merges with the block partials.  The work is a few MACs per
// byte; the kernel streams K and V once (HBM-bound).
#pragma once
#include "decode_simt.cuh"

namespace milo {

constexpr int TAIL_CHUNK = 32;   // tail tokens per round
constexpr int TAIL_GSUB = 8;     // query heads of one KV head per pass over the tail (static smem < 48 KB)

// K and V are staged in their own element type (bf16 rows take half the
// shared-memory traffic of fp32 ones) and widened as they are read.
template <typename T> struct alignas(16) TailSmem {
    float q[TAIL_GSUB][D];
    T k[TAIL_CHUNK][D + 16 / sizeof(T)];     // padded rows: 16-byte reads of 32 different rows are conflict-free
    T v[TAIL_CHUNK][D];
    float p[TAIL_GSUB][TAIL_CHUNK];
    float part[4][TAIL_GSUB][TAIL_CHUNK];    // score partials of the four quarters of d
    float m[TAIL_GSUB], l[TAIL_GSUB], f[TAIL_GSUB];
};

// one 16-byte vector of tail elements as fp32
template <typename T> struct TailVec;
template <> struct TailVec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void get(uint4 u, float (&x)[4]) {
        x[0] = __uint_as_float(u.x);
        x[1] = __uint_as_float(u.y);
        x[2] = __uint_as_float(u.z);
        x[3] = __uint_as_float(u.w);
    }
};
template <> struct TailVec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void get(uint4 u, float (&x)[8]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
            x[2 * i] = t.x;
            x[2 * i + 1] = t.y;
        }
    }
};

// grid (H, S, L), 128 threads.
//   k_tail, v_tail: [L][S][H][tail_cap][D], 16-byte aligned; tail_len[S] tokens
//   of each session are live (a length outside [0, tail_cap] raises ST_BOUNDS
//   and counts as 0).
//   tail_o: [L][S][Hq][D] normalised outputs; tail_ml: [L][S][Hq] (max score,
//   sum of exp(score - max)); an empty tail leaves (-inf, 0) and zeros.
// Each round loads a 32-token chunk of K and V as 16-byte vectors, all issued
// before the first is used, and stages both in shared memory as they came;
// thread j then accumulates output channel j of every query head.
template <typename T>
__global__ void __launch_bounds__(128) k_tail_attn(DecodeArgs a, const T *__restrict__ k_tail,
                                                   const T *__restrict__ v_tail, int tail_cap,
                                                   const int32_t *__restrict__ tail_len, float *__restrict__ tail_o,
                                                   float2 *__restrict__ tail_ml) {
    constexpr int EPV = TailVec<T>::N;                 // elements per vector
    constexpr int VPR = D / EPV;                       // vectors per row
    constexpr int NV = TAIL_CHUNK * VPR / 128;         // vectors per thread and array (rows per thread)
    constexpr int NGRP = 128 / VPR;                    // threads loading the same channels of different rows
    static_assert(NV * NGRP == TAIL_CHUNK, "row groups");
    __shared__ TailSmem<T> sm;
    const int h = blockIdx.x, s = blockIdx.y, l = blockIdx.z;
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
    const int cgrp = j % VPR, rgrp = j / VPR;          // channels [EPV cgrp, +EPV), rows rgrp + NGRP i
    int n = tail_len[s];
    if (n < 0 || n > tail_cap) {
        if (j == 0 && h == 0 && l == 0) raise_status(ST_BOUNDS);
        n = 0;
    }
    const float scale = rsqrtf((float)D);
    const int64_t kv0 = (((int64_t)l * a.S + s) * a.H + h) * tail_cap;   // first token row of this (l, s, h)
    for (int g0 = 0; g0 < a.G; g0 += TAIL_GSUB) {
        const int gn = min(TAIL_GSUB, a.G - g0);
        const int64_t row0 = ((int64_t)l * a.S + s) * a.Hq + (int64_t)h * a.G + g0;   // first query row
        for (int g = 0; g < gn; ++g) sm.q[g][j] = a.q[(row0 + g) * D + j];
        if (j < TAIL_GSUB) {
            sm.m[j] = -INFINITY;
            sm.l[j] = 0.f;
        }
        float acc[TAIL_GSUB];
#pragma unroll
        for (int g = 0; g < TAIL_GSUB; ++g) acc[g] = 0.f;
        for (int c0 = 0; c0 < n; c0 += TAIL_CHUNK) {
            const int cn = min(TAIL_CHUNK, n - c0);
            uint4 kr[NV], vr[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int r = rgrp + NGRP * i;
                kr[i] = vr[i] = make_uint4(0u, 0u, 0u, 0u);
                if (r < cn) {
                    const int64_t row = (kv0 + c0 + r) * D;
                    kr[i] = __ldg(reinterpret_cast<const uint4 *>(k_tail + row) + cgrp);
                    vr[i] = __ldg(reinterpret_cast<const uint4 *>(v_tail + row) + cgrp);
                }
            }
            __syncthreads();   // previous round's k, p and f used; q, m, l written
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                *reinterpret_cast<uint4 *>(&sm.k[rgrp + NGRP * i][cgrp * EPV]) = kr[i];
                *reinterpret_cast<uint4 *>(&sm.v[rgrp + NGRP * i][cgrp * EPV]) = vr[i];
            }
            __syncthreads();
            // scores: warp w dots dims [32w, 32w + 32) of key t = lane with every
            // query head (each key element read once, q broadcast), then the four
            // quarters are added per (query head, token)
            {
                float sp[TAIL_GSUB];
#pragma unroll
                for (int g = 0; g < TAIL_GSUB; ++g) sp[g] = 0.f;
                // dims [32 warp, 32 warp + 32) of key `lane`: 32 / EPV vectors
                const uint4 *kt = reinterpret_cast<const uint4 *>(&sm.k[lane][32 * warp]);
#pragma unroll
                for (int vi = 0; vi < 32 / EPV; ++vi) {
                    float x[EPV];
                    TailVec<T>::get(kt[vi], x);
#pragma unroll
                    for (int e4 = 0; e4 < EPV / 4; ++e4) {
                        const int d4 = 8 * warp + vi * (EPV / 4) + e4;   // float4 index into q
#pragma unroll
                        for (int g = 0; g < TAIL_GSUB; ++g) {
                            if (g >= gn) break;
                            const float4 a4 = reinterpret_cast<const float4 *>(sm.q[g])[d4];
                            sp[g] = fmaf(a4.w, x[4 * e4 + 3],
                                         fmaf(a4.z, x[4 * e4 + 2], fmaf(a4.y, x[4 * e4 + 1], fmaf(a4.x, x[4 * e4], sp[g]))));
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < TAIL_GSUB; ++g)
                    if (g < gn) sm.part[warp][g][lane] = sp[g];
            }
            __syncthreads();
            for (int u = j; u < gn * TAIL_CHUNK; u += blockDim.x) {
                const int g = u / TAIL_CHUNK, t = u % TAIL_CHUNK;
                const float x = (sm.part[0][g][t] + sm.part[1][g][t]) + (sm.part[2][g][t] + sm.part[3][g][t]);
                sm.p[g][t] = t < cn ? x * scale : -INFINITY;
            }
            __syncthreads();
            // online softmax: warp w takes query heads w, w + 4; lane = token
            for (int g = warp; g < gn; g += 4) {
                const float x = sm.p[g][lane];
                float cm = x;
                for (int o = 16; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
                const float m_old = sm.m[g];
                const float m_new = fmaxf(m_old, cm);            // finite: every round has a live token
                const float pe = __expf(x - m_new);
                float ps = pe;
                for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
                sm.p[g][lane] = pe;
                if (lane == 0) {
                    const float fct = m_old == -INFINITY ? 0.f : __expf(m_old - m_new);
                    sm.f[g] = fct;
                    sm.l[g] = sm.l[g] * fct + ps;
                    sm.m[g] = m_new;
                }
            }
            __syncthreads();
            // o_g[j] = f_g o_g[j] + sum_t p_g[t] v[t][j]: each v[t][j] read once for
            // every query head, p read four tokens at a time (broadcast)
#pragma unroll
            for (int g = 0; g < TAIL_GSUB; ++g)
                if (g < gn) acc[g] *= sm.f[g];
#pragma unroll 2
            for (int t4 = 0; t4 < TAIL_CHUNK / 4; ++t4) {
                const float v0 = to_f32(sm.v[4 * t4][j]), v1 = to_f32(sm.v[4 * t4 + 1][j]);
                const float v2 = to_f32(sm.v[4 * t4 + 2][j]), v3 = to_f32(sm.v[4 * t4 + 3][j]);
#pragma unroll
                for (int g = 0; g < TAIL_GSUB; ++g) {
                    if (g >= gn) break;
                    const float4 p4 = reinterpret_cast<const float4 *>(sm.p[g])[t4];
                    acc[g] = fmaf(p4.w, v3, fmaf(p4.z, v2, fmaf(p4.y, v1, fmaf(p4.x, v0, acc[g]))));
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < TAIL_GSUB; ++g) {
            if (g >= gn) break;
            const float lg = sm.l[g];
            tail_o[(row0 + g) * D + j] = lg > 0.f ? acc[g] / lg : 0.f;
            if (j == 0) tail_ml[row0 + g] = make_float2(sm.m[g], lg);
        }
        __syncthreads();   // m and l read before the next pass resets them
    }
}

}  // namespace milo
