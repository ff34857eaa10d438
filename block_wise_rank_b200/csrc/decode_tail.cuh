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
// of its G query heads: 32-token chunks of K and V staged in shared memory,
// scores by thread-per-(query, token) dot products, an online softmax per
// query head, and thread j accumulating output channel j.  The result is one
// more partial (max, sum, normalised output) per query row, which k_combine
// merges with the block partials.  The work is a few MACs per byte; the
// kernel streams K and V once (HBM-bound).
#pragma once
#include "decode_simt.cuh"

namespace milo {

constexpr int TAIL_CHUNK = 32;   // tail tokens staged per round
constexpr int TAIL_GSUB = 16;    // query heads of one KV head per pass over the tail

struct TailSmem {
    float q[TAIL_GSUB][D];
    float k[TAIL_CHUNK][D + 1];   // padded rows: thread-per-token reads are conflict-free
    float v[TAIL_CHUNK][D];
    float p[TAIL_GSUB][TAIL_CHUNK];
    float m[TAIL_GSUB], l[TAIL_GSUB], f[TAIL_GSUB];
};

template <typename T> __device__ __forceinline__ float tail_elem(const T *p, int64_t i);
template <> __device__ __forceinline__ float tail_elem<float>(const float *p, int64_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float tail_elem<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
}

// grid (H, S, L), 128 threads (thread j = output channel j).
//   k_tail, v_tail: [L][S][H][tail_cap][D]; tail_len[S] tokens of each session
//   are live (a length outside [0, tail_cap] raises ST_BOUNDS and counts as 0).
//   tail_o: [L][S][Hq][D] normalised outputs; tail_ml: [L][S][Hq] (max score,
//   sum of exp(score - max)); an empty tail leaves (-inf, 0) and zeros.
template <typename T>
__global__ void __launch_bounds__(128) k_tail_attn(DecodeArgs a, const T *__restrict__ k_tail,
                                                   const T *__restrict__ v_tail, int tail_cap,
                                                   const int32_t *__restrict__ tail_len, float *__restrict__ tail_o,
                                                   float2 *__restrict__ tail_ml) {
    __shared__ TailSmem sm;
    const int h = blockIdx.x, s = blockIdx.y, l = blockIdx.z;
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
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
            __syncthreads();   // previous round's k, v, p and f fully used; q, m, l written
#pragma unroll 8
            for (int t = 0; t < TAIL_CHUNK; ++t) {
                const bool live = t < cn;
                const int64_t e = (kv0 + c0 + t) * D + j;
                sm.k[t][j] = live ? tail_elem(k_tail, e) : 0.f;
                sm.v[t][j] = live ? tail_elem(v_tail, e) : 0.f;
            }
            __syncthreads();
            // scores: pair (g, t) = (u / 32, u % 32), one lane per token
            for (int u = j; u < gn * TAIL_CHUNK; u += blockDim.x) {
                const int g = u / TAIL_CHUNK, t = u % TAIL_CHUNK;
                float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;   // four chains for the FMA latency
#pragma unroll 4
                for (int dd = 0; dd < D; dd += 4) {
                    x0 = fmaf(sm.q[g][dd], sm.k[t][dd], x0);
                    x1 = fmaf(sm.q[g][dd + 1], sm.k[t][dd + 1], x1);
                    x2 = fmaf(sm.q[g][dd + 2], sm.k[t][dd + 2], x2);
                    x3 = fmaf(sm.q[g][dd + 3], sm.k[t][dd + 3], x3);
                }
                sm.p[g][t] = t < cn ? ((x0 + x1) + (x2 + x3)) * scale : -INFINITY;
            }
            __syncthreads();
            // online softmax: warp w takes query heads w, w + 4, ...; lane = token
            for (int g = warp; g < gn; g += 4) {
                const float x = sm.p[g][lane];
                float cm = x;
                for (int o = 16; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
                const float m_old = sm.m[g];
                const float m_new = fmaxf(m_old, cm);            // finite: every round has a live token
                const float pe = __expf(x - m_new);
                float ps = pe;
                for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
                __syncwarp();
                sm.p[g][lane] = pe;
                if (lane == 0) {
                    const float fct = m_old == -INFINITY ? 0.f : __expf(m_old - m_new);
                    sm.f[g] = fct;
                    sm.l[g] = sm.l[g] * fct + ps;
                    sm.m[g] = m_new;
                }
            }
            __syncthreads();
#pragma unroll
            for (int g = 0; g < TAIL_GSUB; ++g) {
                if (g >= gn) break;
                float x = acc[g] * sm.f[g];
#pragma unroll 8
                for (int t = 0; t < TAIL_CHUNK; ++t) x = fmaf(sm.p[g][t], sm.v[t][j], x);
                acc[g] = x;
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
        __syncthreads();   // m and l are reset for the next group of query heads
    }
}

}  // namespace milo
