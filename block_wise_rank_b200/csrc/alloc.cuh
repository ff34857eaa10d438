// alloc.cuh -- eps and the greedy entropy-gain rank allocation.
//
// Step "allocate each block's rank by greedily maximising
// sum log(1 + sigma^2/eps^2) under a global rank budget" (evolve.pub review
// of MILO, Summary, Eqs 5-7; Strengths, "Principled, budget-feasible rank
// allocation").  Because every gain log(1 + key) is strictly increasing in
// key = (sigma/eps)^2 and the gains of a block are non-increasing in k, the
// greedy result is exactly the set of the R' largest keys among the
// eligible components (ties to the lower linear index).  The device finds
// the R'-th largest key with an 8-pass radix select over the 64-bit key
// patterns (positive doubles order like their bit patterns), then counts
// per block the keys above it and hands the tied keys out in block order.
#pragma once
#include "common.cuh"

namespace milo {

// eps_g = eps_rel * max_b sigma_{g,b,1}, one CTA per (group, kind).
__global__ void k_eps(const float *__restrict__ sK, const float *__restrict__ sV, double *__restrict__ eK,
                      double *__restrict__ eV, int n_b, double eps_rel) {
    const int g = blockIdx.x, kind = blockIdx.y;
    const float *s = kind == 0 ? sK : sV;
    float m = 0.f;
    for (int b = threadIdx.x; b < n_b; b += blockDim.x) m = fmaxf(m, s[((int64_t)g * n_b + b) * D]);
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wm[32];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wm[w]);
        (kind == 0 ? eK : eV)[g] = eps_rel * (double)m;
    }
}

// scope "global per kind": every group takes the largest group eps
__global__ void k_eps_global(double *__restrict__ eK, double *__restrict__ eV, int n_groups) {
    double *e = blockIdx.x == 0 ? eK : eV;
    __shared__ double wm[32];
    double m = 0.0;
    for (int g = threadIdx.x; g < n_groups; g += blockDim.x) m = fmax(m, e[g]);
    for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, wm[w]);
        wm[0] = m;
    }
    __syncthreads();
    for (int g = threadIdx.x; g < n_groups; g += blockDim.x) e[g] = wm[0];
}

// Selection state of one kind (device scratch).
struct SelState {
    unsigned long long prefix;   // high bits of the threshold found so far
    unsigned long long mask;     // which bits of prefix are fixed
    long long need;              // keys still to take among those matching prefix
    unsigned int done;           // CTAs finished with the current pass
    unsigned int pad;
    unsigned int hist[256];
};

// Everything the allocation kernels need about one kind.
struct SelArgs {
    const float *sigma;      // [n_blk][D]
    const double *eps;       // [n_groups]
    int32_t *ranks;          // [n_blk] out
    int64_t *offsets;        // [n_blk + 1] out, or null
    SelState *st;
    int32_t *gt;             // [n_blk] scratch
    int32_t *eq;             // [n_blk] scratch
    long long need0;         // R - sum rmin_b
};

struct SelShape {
    int n_b, T, block_len, r_min, r_max;
    int64_t n_blk;
    int dtype;              // factor type of the offsets written (their unit: block_units)
    const int32_t *starts;  // variable-length blocks' starts, or null (BlockGeo)
    __device__ __forceinline__ int len(int b) const { return BlockGeo{T, block_len, starts}.len(b); }
};

// key bits of component k of block blk ((sigma/eps)^2 as a double, 0 if eps <= 0)
__device__ __forceinline__ unsigned long long key_bits(const SelArgs &a, int64_t blk, int k, int n_b) {
    const double e = a.eps[blk / n_b];
    if (!(e > 0.0)) return 0ull;
    const double q = (double)a.sigma[blk * D + k] / e;
    return (unsigned long long)__double_as_longlong(q * q);
}

__device__ __forceinline__ void elig_range(const SelShape &sh, int64_t blk, int &k0, int &k1) {
    const int b = (int)(blk % sh.n_b);
    const int cap = block_cap(sh.len(b), sh.r_max);
    k0 = sh.r_min < cap ? sh.r_min : cap;
    k1 = cap;
}

__global__ void k_sel_init(SelArgs a0, SelArgs a1) {
    SelArgs a = blockIdx.x == 0 ? a0 : a1;
    SelState *st = a.st;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) st->hist[i] = 0u;
    if (threadIdx.x == 0) {
        st->prefix = a.need0 > 0 ? 0ull : ~0ull;
        st->mask = a.need0 > 0 ? 0ull : ~0ull;
        st->need = a.need0;
        st->done = 0u;
    }
}

// One radix pass (digit = bits [shift, shift + 8)).  The last CTA to finish
// picks the digit of the threshold and resets the histogram.
__global__ void __launch_bounds__(256) k_sel_pass(SelArgs a0, SelArgs a1, SelShape sh, int shift) {
    const SelArgs &a = blockIdx.y == 0 ? a0 : a1;
    SelState *st = a.st;
    __shared__ unsigned int hist[256];
    __shared__ bool last;
    if (st->need <= 0) return;   // nothing to select (uniform for the grid)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    const unsigned long long prefix = st->prefix, mask = st->mask;
    const int64_t total = sh.n_blk * D;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = e / D;
        const int k = (int)(e % D);
        int k0, k1;
        elig_range(sh, blk, k0, k1);
        if (k < k0 || k >= k1) continue;
        const unsigned long long kb = key_bits(a, blk, k, sh.n_b);
        if ((kb & mask) != prefix) continue;
        atomicAdd(&hist[(kb >> shift) & 255ull], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (hist[i]) atomicAdd(&st->hist[i], hist[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = (atomicAdd(&st->done, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!last) return;
    if (threadIdx.x == 0) {
        __threadfence();
        volatile unsigned int *h = st->hist;
        long long need = st->need, cum = 0;
        int bin = 255;
        for (; bin >= 0; --bin) {
            const long long c = h[bin];
            if (cum + c >= need) break;
            cum += c;
        }
        if (bin < 0) bin = 0;   // cannot happen when need <= candidates
        st->need = need - cum;
        st->prefix = prefix | ((unsigned long long)bin << shift);
        st->mask = mask | (255ull << shift);
        st->done = 0u;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x) st->hist[i] = 0u;
}

// Per block: keys above the threshold and keys equal to it (eligible only);
// also flags keys that increase along k (sigma not sorted).  One warp per block.
__global__ void k_sel_count(SelArgs a0, SelArgs a1, SelShape sh) {
    const SelArgs &a = blockIdx.y == 0 ? a0 : a1;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= sh.n_blk) return;
    const int64_t blk = warp;
    const unsigned long long thr = a.st->prefix;
    int k0, k1;
    elig_range(sh, blk, k0, k1);
    int gt = 0, eq = 0, bad = 0;
    for (int k = k0 + lane; k < k1; k += 32) {
        const unsigned long long kb = key_bits(a, blk, k, sh.n_b);
        gt += kb > thr;
        eq += kb == thr;
        if (k + 1 < k1 && key_bits(a, blk, k + 1, sh.n_b) > kb) bad = 1;
        const float sv = a.sigma[blk * D + k];
        if (!isfinite(sv)) bad |= 2;
    }
    for (int o = 16; o; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if (lane == 0) {
        a.gt[blk] = gt;
        a.eq[blk] = eq;
        if (bad & 1) raise_status(ST_UNSORTED);
        if (bad & 2) raise_status(ST_NONFINITE);
    }
}

// Single CTA per kind: ties handed out in block order, ranks, and the
// packed-arena offsets (exclusive scan of the padded block sizes
// round_up(r_b, 8) * (128 * ceil(T_b / 128) + d)).
__global__ void __launch_bounds__(1024) k_sel_ranks(SelArgs a0, SelArgs a1, SelShape sh) {
    const SelArgs &a = blockIdx.x == 0 ? a0 : a1;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int64_t n = sh.n_blk;
    const int64_t per = (n + nt - 1) / nt;
    const int64_t lo = min((int64_t)tid * per, n), hi = min(lo + per, n);
    __shared__ long long sA[1024], sB[1024];
    long long eqsum = 0;
    for (int64_t i = lo; i < hi; ++i) eqsum += a.eq[i];
    sA[tid] = eqsum;
    __syncthreads();
    for (int o = 1; o < nt; o <<= 1) {   // inclusive Hillis-Steele scan
        long long v = tid >= o ? sA[tid - o] : 0;
        __syncthreads();
        sA[tid] += v;
        __syncthreads();
    }
    const long long need = a.st->need > 0 ? a.st->need : 0;
    long long before = sA[tid] - eqsum;
    long long elems = 0;
    for (int64_t i = lo; i < hi; ++i) {
        const int e = a.eq[i];
        long long take = need - before;
        take = take < 0 ? 0 : (take > e ? e : take);
        before += e;
        int k0, k1;
        elig_range(sh, i, k0, k1);
        const int r = k0 + a.gt[i] + (int)take;
        a.ranks[i] = r;
        const int tb = sh.len((int)(i % sh.n_b));
        elems += block_units(sh.dtype, r, tb);
    }
    if (a.offsets == nullptr) return;
    sB[tid] = elems;
    __syncthreads();
    for (int o = 1; o < nt; o <<= 1) {
        long long v = tid >= o ? sB[tid - o] : 0;
        __syncthreads();
        sB[tid] += v;
        __syncthreads();
    }
    long long off = sB[tid] - elems;
    for (int64_t i = lo; i < hi; ++i) {
        a.offsets[i] = off;
        const int tb = sh.len((int)(i % sh.n_b));
        off += block_units(sh.dtype, a.ranks[i], tb);
    }
    if (hi == n && lo < hi) a.offsets[n] = off;
    if (n == 0 && tid == 0) a.offsets[0] = 0;
}

}  // namespace milo
