// decode_simt.cuh -- decode attention over retrieved compressed blocks on
// CUDA cores (FP32 throughout).
//
// Step "at inference a retriever selects blocks, whose low-rank factors are
// rebuilt before sparse attention" (evolve.pub review of MILO, Summary; FAQ
// "What is MILO": only the blocks a query needs are rebuilt).  For one
// (layer, KV head, block) the CTA rebuilds the pre-RoPE keys a_t B_K tile by
// tile, rotates them by the block-relative angle t*theta_i, scores every
// query that selected the block (each query pre-rotated by -p*theta_i, so
// that q . R(p+t) k = (R(-p) q) . (R(t) k)), runs an online softmax, and
// contracts the probabilities with A_V before multiplying by B_V.  Neither
// K-hat nor V-hat is written to memory.  Each (query, selected slot) gets a
// partial (max, sum, unnormalised output) merged by k_combine.
//
// This kernel is the FP32 path: it serves f32 factors (and bf16 / INT8
// factors of blocks longer than 512 tokens, or when MILO_FORCE_SIMT is set,
// as the tests' cross-check); the tensor-core kernel in decode_tc.cuh serves
// bf16 factors, and INT8 factors dequantised to fp16.
#pragma once
#include "common.cuh"

namespace milo {

struct DecodeArgs {
    KindView kv[2];
    int L, H, G, T, block_len, n_b, factor_dtype;
    int S, Hq, n_sel;
    const float *q;            // [L][S][Hq][D]
    const int32_t *sel;        // [S][n_sel]
    const int32_t *pos;        // [S][n_sel] or null
    const int32_t *starts;     // variable-length blocks' starts [n_b + 1], or null (BlockGeo)
    const int32_t *slot_start; // [n_b + 1] slots of each block id
    const int32_t *slot_list;  // [S * n_sel] slot = s * n_sel + j
    const float2 *rope_q;      // [S * n_sel][64] (cos, sin)(p theta_i)
    const float2 *rope_t;      // [block_len][64] (cos, sin)(t theta_i)
    float *part_o;             // [L][S][Hq][n_sel][D]
    float2 *part_ml;           // [L][S][Hq][n_sel] (max, sum)
    float *out;                // [L][S][Hq][D]
    int32_t *claim;            // tensor-core path: next unclaimed work item (zeroed before the launch)
    uint64_t wait_ns;          // tensor-core path: limit of every wait on the device
    int inject;                // tensor-core path: 1 = withhold one copy (tests of the bounded waits)
    int f16;                   // tensor-core path: kv[].data holds fp16 factors (INT8 dequantised), else bf16
    const float *tail_o;       // [L][S][Hq][D] partial of the recent uncompressed tokens, or null
    const float2 *tail_ml;     // [L][S][Hq] its (max, sum), or null
};

// (cos, sin)(p theta_i) for every selected slot and (t theta_i) for every
// in-block token, angles in double, theta_i = base^(-2i/d).
__global__ void k_rope_tables(const int32_t *__restrict__ sel, const int32_t *__restrict__ pos,
                              const int32_t *__restrict__ starts, int n_b, int n_slots, int block_len, double base,
                              float2 *__restrict__ rope_q, float2 *__restrict__ rope_t) {
    const int64_t total = (int64_t)(n_slots + block_len) * HALF;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(e % HALF);
        const int64_t row = e / HALF;
        const double theta = pow(base, -2.0 * (double)i / (double)D);
        double p;
        if (row < n_slots) {   // a selected block's start: given, else where the block starts
            const int b = sel[row];
            p = pos ? (double)pos[row]
                    : (starts ? (b >= 0 && b < n_b ? (double)starts[b] : 0.0) : (double)b * (double)block_len);
        }
        else p = (double)(row - n_slots);
        double sn, cs;
        sincos(p * theta, &sn, &cs);
        const float2 v = make_float2((float)cs, (float)sn);
        if (row < n_slots) rope_q[row * HALF + i] = v;
        else rope_t[(row - n_slots) * HALF + i] = v;
    }
}

// Inverse index: for each block id, the slots (s, j) that selected it.
__global__ void k_slot_count(const int32_t *__restrict__ sel, int n_slots, int n_b, int32_t *__restrict__ cnt) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_slots; e += gridDim.x * blockDim.x) {
        const int b = sel[e];
        if (b < 0 || b >= n_b) { raise_status(ST_BOUNDS); continue; }
        atomicAdd(&cnt[b], 1);
    }
}

// Exclusive prefix sum of the per-block slot counts (start, start[n_b] = the
// total), one CTA of 1024 threads; the counts are reset for k_slot_fill's
// cursors.
constexpr int SCAN_THREADS = 1024;
__global__ void __launch_bounds__(SCAN_THREADS) k_slot_scan(int32_t *__restrict__ cnt, int32_t *__restrict__ start,
                                                            int n_b) {
    __shared__ int wsum[SCAN_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int chunk = (n_b + SCAN_THREADS - 1) / SCAN_THREADS;
    const int b0 = min(n_b, tid * chunk), b1 = min(n_b, b0 + chunk);
    int mine = 0;
    for (int b = b0; b < b1; ++b) mine += cnt[b];
    int inc = mine;
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int v = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += x;
        }
        wsum[lane] = v;
    }
    __syncthreads();
    int acc = inc - mine + (wid > 0 ? wsum[wid - 1] : 0);
    for (int b = b0; b < b1; ++b) {
        const int c = cnt[b];
        start[b] = acc;
        acc += c;
    }
    __syncthreads();   // every count read before any is reset
    for (int b = b0; b < b1; ++b) cnt[b] = 0;
    if (tid == SCAN_THREADS - 1) start[n_b] = wsum[31];
}

__global__ void k_slot_fill(const int32_t *__restrict__ sel, int n_slots, int n_b, const int32_t *__restrict__ start,
                            int32_t *__restrict__ cursor, int32_t *__restrict__ list) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_slots; e += gridDim.x * blockDim.x) {
        const int b = sel[e];
        if (b < 0 || b >= n_b) continue;
        list[start[b] + atomicAdd(&cursor[b], 1)] = e;
    }
}

// Exclusive prefix sum of n int64 values in place (one CTA of 1024 threads);
// v[n] receives the total.
__global__ void __launch_bounds__(SCAN_THREADS) k_scan_i64(int64_t *__restrict__ v, int64_t n) {
    __shared__ long long wsum[SCAN_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t chunk = (n + SCAN_THREADS - 1) / SCAN_THREADS;
    const int64_t b0 = min(n, (int64_t)tid * chunk), b1 = min(n, b0 + chunk);
    long long mine = 0;
    for (int64_t b = b0; b < b1; ++b) mine += v[b];
    long long inc = mine;
    for (int o = 1; o < 32; o <<= 1) {
        const long long x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        long long w = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            const long long x = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += x;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    long long acc = inc - mine + (wid > 0 ? wsum[wid - 1] : 0);
    for (int64_t b = b0; b < b1; ++b) {
        const long long c = v[b];
        v[b] = acc;
        acc += c;
    }
    if (tid == SCAN_THREADS - 1) v[n] = wsum[31];
}

// Tensor-core path: query passes of every block id, ceil(slots x G / pass_q).
__global__ void k_pass_counts(const int32_t *__restrict__ start, int n_b, int G, int pass_q,
                              int32_t *__restrict__ passes) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < n_b) passes[b] = ((start[b + 1] - start[b]) * G + pass_q - 1) / pass_q;
}

// Exclusive prefix sum of n values (one CTA of 1024 threads): out[i] for i <=
// n, out[n] = the total.
__global__ void __launch_bounds__(SCAN_THREADS) k_scan_counts(const int32_t *__restrict__ in, int32_t *__restrict__ out,
                                                              int n) {
    __shared__ int wsum[SCAN_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int chunk = (n + SCAN_THREADS - 1) / SCAN_THREADS;
    const int b0 = min(n, tid * chunk), b1 = min(n, b0 + chunk);
    int mine = 0;
    for (int b = b0; b < b1; ++b) mine += in[b];
    int inc = mine;
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int v = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += x;
        }
        wsum[lane] = v;
    }
    __syncthreads();
    int acc = inc - mine + (wid > 0 ? wsum[wid - 1] : 0);
    for (int b = b0; b < b1; ++b) {
        out[b] = acc;
        acc += in[b];
    }
    if (tid == SCAN_THREADS - 1) out[n] = wsum[31];
}

constexpr int DS_QC = 16;   // queries per pass
constexpr int DS_TT = 32;   // tokens per tile

struct DecodeSimtSmem {
    float qt[DS_QC][D];
    float aK[D][DS_TT];
    float aV[D][DS_TT];
    float kt[DS_TT][D + 1];
    float sc[DS_QC][DS_TT + 1];
    float oA[DS_QC][D];
    float m[DS_QC], l[DS_QC], alpha[DS_QC];
    int qslot[DS_QC], qhead[DS_QC];
};

__device__ __forceinline__ float factor_a(const KindView &kv, int dt, int64_t blk, int64_t base, int R8, int k, int t) {
    float v = load_elem(kv.data, base + a_index(R8, t, k), dt);
    if (dt == MILO_INT8) v *= kv.scaleA[blk * D + k];
    return v;
}
__device__ __forceinline__ float factor_b(const KindView &kv, int dt, int64_t blk, int64_t base, int R8, int nt, int k,
                                          int j) {
    float v = load_elem(kv.data, base + b_index(R8, nt, k, j), dt);
    if (dt == MILO_INT8) v *= kv.scaleB[blk * D + j];
    return v;
}

// grid (n_b, H, L), 256 threads.
__global__ void __launch_bounds__(256) k_decode_simt(DecodeArgs a) {
    extern __shared__ __align__(16) unsigned char ds_raw[];
    DecodeSimtSmem &sm = *reinterpret_cast<DecodeSimtSmem *>(ds_raw);
    const int b = blockIdx.x, h = blockIdx.y, l = blockIdx.z;
    const int s0 = a.slot_start[b], ns = a.slot_start[b + 1] - s0;
    if (ns == 0) return;
    const int tid = threadIdx.x;
    const int dt = a.factor_dtype;
    const int64_t blk = ((int64_t)l * a.H + h) * a.n_b + b;
    const KindView &K = a.kv[0], &V = a.kv[1];
    const int rK = K.ranks[blk], rV = V.ranks[blk];
    const int Tb = BlockGeo{a.T, a.block_len, a.starts}.len(b);
    const int nt = token_tiles(Tb);
    const int R8K = rank_pad(rK), R8V = rank_pad(rV);
    const int64_t baseK = K.offsets[blk], baseV = V.offsets[blk];
    const float scale = rsqrtf((float)D);
    const int nq_total = ns * a.G;

    for (int q0 = 0; q0 < nq_total; q0 += DS_QC) {
        const int nq = min(DS_QC, nq_total - q0);
        // rotated queries R(-p) q
        for (int e = tid; e < DS_QC * HALF; e += 256) {
            const int qi = e / HALF, i = e % HALF;
            if (qi >= nq) { sm.qt[qi][i] = 0.f; sm.qt[qi][i + HALF] = 0.f; continue; }
            const int slot = a.slot_list[s0 + (q0 + qi) / a.G];
            const int g = (q0 + qi) % a.G;
            const int s = slot / a.n_sel;
            const int hq = h * a.G + g;
            const float *qv = a.q + (((int64_t)l * a.S + s) * a.Hq + hq) * D;
            const float2 cs = a.rope_q[(int64_t)slot * HALF + i];
            const float x0 = qv[i], x1 = qv[i + HALF];
            sm.qt[qi][i] = x0 * cs.x + x1 * cs.y;
            sm.qt[qi][i + HALF] = x1 * cs.x - x0 * cs.y;
            if (i == 0) { sm.qslot[qi] = slot; sm.qhead[qi] = hq; }
        }
        for (int e = tid; e < DS_QC * D; e += 256) sm.oA[e / D][e % D] = 0.f;
        if (tid < DS_QC) { sm.m[tid] = -INFINITY; sm.l[tid] = 0.f; }
        __syncthreads();

        for (int t0 = 0; t0 < Tb; t0 += DS_TT) {
            const int tt = min(DS_TT, Tb - t0);
            for (int e = tid; e < D * DS_TT; e += 256) {
                const int k = e / DS_TT, t = e % DS_TT;
                sm.aK[k][t] = (k < rK && t < tt) ? factor_a(K, dt, blk, baseK, R8K, k, t0 + t) : 0.f;
                sm.aV[k][t] = (k < rV && t < tt) ? factor_a(V, dt, blk, baseV, R8V, k, t0 + t) : 0.f;
            }
            __syncthreads();
            {   // rebuild pre-RoPE keys: kt[t][j] = sum_k aK[k][t] B_K[k][j]
                const int j = tid % D, th = tid / D;
                float acc[DS_TT / 2];
#pragma unroll
                for (int u = 0; u < DS_TT / 2; ++u) acc[u] = 0.f;
                for (int k = 0; k < rK; ++k) {
                    const float bk = factor_b(K, dt, blk, baseK, R8K, nt, k, j);
#pragma unroll
                    for (int u = 0; u < DS_TT / 2; ++u) acc[u] = fmaf(sm.aK[k][th * (DS_TT / 2) + u], bk, acc[u]);
                }
#pragma unroll
                for (int u = 0; u < DS_TT / 2; ++u) sm.kt[th * (DS_TT / 2) + u][j] = acc[u];
            }
            __syncthreads();
            {   // block-relative RoPE R(t) on the rebuilt keys
                const int i = tid % HALF, tg = tid / HALF;
                for (int t = tg; t < tt; t += 256 / HALF) {
                    const float2 cs = a.rope_t[(int64_t)(t0 + t) * HALF + i];
                    const float x0 = sm.kt[t][i], x1 = sm.kt[t][i + HALF];
                    sm.kt[t][i] = x0 * cs.x - x1 * cs.y;
                    sm.kt[t][i + HALF] = x1 * cs.x + x0 * cs.y;
                }
            }
            __syncthreads();
            for (int e = tid; e < DS_QC * DS_TT; e += 256) {
                const int qi = e / DS_TT, t = e % DS_TT;
                float acc = 0.f;
                if (qi < nq && t < tt)
                    for (int j = 0; j < D; ++j) acc = fmaf(sm.qt[qi][j], sm.kt[t][j], acc);
                sm.sc[qi][t] = acc * scale;
            }
            __syncthreads();
            if (tid < nq) {
                float mx = sm.m[tid];
                for (int t = 0; t < tt; ++t) mx = fmaxf(mx, sm.sc[tid][t]);
                const float al = __expf(sm.m[tid] - mx);
                float sum = 0.f;
                for (int t = 0; t < tt; ++t) {
                    const float p = __expf(sm.sc[tid][t] - mx);
                    sm.sc[tid][t] = p;
                    sum += p;
                }
                for (int t = tt; t < DS_TT; ++t) sm.sc[tid][t] = 0.f;
                sm.l[tid] = sm.l[tid] * al + sum;
                sm.m[tid] = mx;
                sm.alpha[tid] = al;
            }
            __syncthreads();
            for (int e = tid; e < DS_QC * D; e += 256) {
                const int qi = e / D, k = e % D;
                if (qi >= nq || k >= rV) continue;
                float acc = sm.oA[qi][k] * sm.alpha[qi];
                for (int t = 0; t < tt; ++t) acc = fmaf(sm.sc[qi][t], sm.aV[k][t], acc);
                sm.oA[qi][k] = acc;
            }
            __syncthreads();
        }
        // o = oA B_V, written as this slot's partial
        for (int e = tid; e < DS_QC * D; e += 256) {
            const int qi = e / D, j = e % D;
            if (qi >= nq) continue;
            float acc = 0.f;
            for (int k = 0; k < rV; ++k) acc = fmaf(sm.oA[qi][k], factor_b(V, dt, blk, baseV, R8V, nt, k, j), acc);
            const int slot = sm.qslot[qi], hq = sm.qhead[qi];
            const int s = slot / a.n_sel, jj = slot % a.n_sel;
            const int64_t pidx = (((int64_t)l * a.S + s) * a.Hq + hq) * a.n_sel + jj;
            a.part_o[pidx * D + j] = sm.l[qi] > 0.f ? acc / sm.l[qi] : 0.f;
            if (j == 0) a.part_ml[pidx] = make_float2(sm.m[qi], sm.l[qi]);
        }
        __syncthreads();
    }
}

// out[l][s][hq] = sum_j w_j l_j o_j / sum_j w_j l_j, w_j = exp(m_j - max m),
// with o_j the normalised output of slot j (fp32 from the CUDA-core path,
// fp16 from the tensor-core path), and the recent-token partial as one more
// term when there is one (an empty tail has sum 0 and adds nothing).
// grid (L * S * Hq), 128 threads.  Slots with an out-of-range block id
// contribute nothing.
template <typename PT> __device__ __forceinline__ float part_elem(const PT *p, int64_t i);
template <> __device__ __forceinline__ float part_elem<float>(const float *p, int64_t i) { return p[i]; }
template <> __device__ __forceinline__ float part_elem<__half>(const __half *p, int64_t i) {
    return __half2float(p[i]);
}

template <typename PT>
__global__ void __launch_bounds__(128) k_combine(DecodeArgs a, const PT *__restrict__ part_o) {
    const int64_t row = blockIdx.x;
    const int s = (int)((row / a.Hq) % a.S);
    const int j = threadIdx.x;
    float M = -INFINITY;
    for (int u = 0; u < a.n_sel; ++u) {
        const int bid = a.sel[(int64_t)s * a.n_sel + u];
        if (bid < 0 || bid >= a.n_b) continue;
        M = fmaxf(M, a.part_ml[row * a.n_sel + u].x);
    }
    float2 tml = make_float2(-INFINITY, 0.f);
    if (a.tail_ml) {
        tml = a.tail_ml[row];
        if (tml.y > 0.f) M = fmaxf(M, tml.x);
    }
    float num = 0.f, den = 0.f;
    if (tml.y > 0.f) {
        const float w = __expf(tml.x - M) * tml.y;
        num = w * a.tail_o[row * D + j];
        den = w;
    }
    for (int u = 0; u < a.n_sel; ++u) {
        const int bid = a.sel[(int64_t)s * a.n_sel + u];
        if (bid < 0 || bid >= a.n_b) continue;
        const float2 ml = a.part_ml[row * a.n_sel + u];
        const float w = __expf(ml.x - M) * ml.y;
        num = fmaf(w, part_elem(part_o, (row * a.n_sel + u) * D + j), num);
        den += w;
    }
    a.out[row * D + j] = den > 0.f ? num / den : 0.f;
}

}  // namespace milo
