// project_simt.cuh -- projection and packing of the low-rank factors.
//
// Step "keep the top r_b singular triplets of each block and store the
// cache in compressed low-rank form per block" (evolve.pub review of MILO,
// Summary and FAQ "What is MILO"): A_b = X_b W_{:,1:r_b} = U_r Sigma_r
// (T_b x r_b) and B_b = W_{:,1:r_b}^T (r_b x d), written into the packed
// arena in the tiled layout of common.cuh (A_b^T tiles, then B_b).  INT8 composition
// (same page, Summary: combined with INT8 quantisation): symmetric per-column
// absmax codes, scale = absmax / 127, round half to even, clamp to +-127.
// 2-bit composition (same page, Key claims: KIVI-style low-bit codes): A_b's
// rank columns in groups of INT2_GROUP tokens, zero = min, scale = (max -
// min) / 3 in fp16, code = clamp(rint((a - zero) / scale), 0, 3) decided in
// fp32 with the stored parameters; B_b in INT8.
#pragma once
#include "common.cuh"

namespace milo {

template <typename TO> __device__ __forceinline__ TO from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ int8_t quant_i8(float x, float s) {
    if (!(s > 0.f)) return 0;
    float q = rintf(__fdiv_rn(x, s));
    q = fminf(fmaxf(q, -127.f), 127.f);
    return (int8_t)q;
}

struct ProjArgs {
    const void *X[2];          // K, V caches [L][H][T][D]
    const float *W[2];         // sorted right singular vectors [n_blk][D][D] (W[j][k])
    KindView kv[2];
    int T, block_len, n_b, in_dtype, out_dtype;
    int64_t n_blk;
    const int32_t *starts;     // variable-length blocks' starts, or null (BlockGeo)
};

// grid (n_blk, D/32 rank chunks, 2 kinds), 256 threads.  Writes the rank
// rows k0 .. k0+31 of A_b^T (rows r_b .. R8-1 and tokens past T_b as zeros,
// in the tiled layout of common.cuh) and, for INT8, their scales.
template <typename TI>
__global__ void __launch_bounds__(256) k_project_a(ProjArgs pa) {
    __shared__ float Wc[D][33];
    __shared__ float amax[32];
    const int blk = blockIdx.x, kind = blockIdx.z;
    const int k0 = blockIdx.y * 32;
    const KindView &kv = pa.kv[kind];
    const int r = kv.ranks[blk];
    const int R8 = rank_pad(r);
    if (k0 >= R8) return;
    const int kw = min(32, R8 - k0);          // rows written (incl. zero padding)
    const int kc = max(0, min(32, r - k0));   // rows with data
    const int b = blk % pa.n_b, lh = blk / pa.n_b;
    const BlockGeo geo{pa.T, pa.block_len, pa.starts};
    const int Tb = geo.len(b);
    const int ldT = token_tiles(Tb) * FTILE;
    const TI *Xb = (const TI *)pa.X[kind] + ((int64_t)lh * pa.T + geo.start(b)) * D;
    const float *Wb = pa.W[kind] + (int64_t)blk * D * D;
    for (int e = threadIdx.x; e < D * 32; e += 256) {
        const int j = e / 32, c = e % 32;
        Wc[j][c] = c < kc ? Wb[j * D + k0 + c] : 0.f;
    }
    if (threadIdx.x < 32) amax[threadIdx.x] = 0.f;
    __syncthreads();
    const int64_t base = kv.offsets[blk];
    const bool is_i8 = pa.out_dtype == MILO_INT8;
    for (int pass = is_i8 ? 0 : 1; pass < 2; ++pass) {
        for (int t = threadIdx.x; t < ldT; t += 256) {
            float acc[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = 0.f;
            if (t < Tb) {
                const TI *xr = Xb + (int64_t)t * D;
                for (int j = 0; j < D; ++j) {
                    const float x = to_f32<TI>(xr[j]);
#pragma unroll
                    for (int c = 0; c < 32; ++c) acc[c] = fmaf(x, Wc[j][c], acc[c]);
                }
            }
            if (pass == 0) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (c < kc) atomicMax((int *)&amax[c], __float_as_int(fabsf(acc[c])));
            } else if (pa.out_dtype == MILO_INT2) {
                // a warp holds the 32 consecutive tokens of one group (ldT is a
                // multiple of 128 and t = 32 w + lane + 256 i)
                uint8_t *blkp = (uint8_t *)kv.data + base;
                const int lane = threadIdx.x & 31, g = t / INT2_GROUP, nt = ldT / FTILE;
                for (int c = 0; c < kw; ++c) {
                    const bool live = t < Tb && c < kc;
                    const float a = acc[c];
                    float lo = live ? a : INFINITY, hi = live ? a : -INFINITY;
                    for (int o = 16; o; o >>= 1) {
                        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
                    }
                    __half sh = __float2half_rn(0.f), zh = sh;   // no live token: 0, 0
                    if (lo <= hi) {
                        sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 3.f));
                        zh = __float2half_rn(lo);
                    }
                    const float s32 = __half2float(sh), z32 = __half2float(zh);
                    int q = 0;
                    if (live && s32 > 0.f) q = (int)fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(a, z32), s32)), 0.f), 3.f);
                    int byte = q << (2 * (lane & 3));   // four consecutive tokens per byte
                    byte |= __shfl_xor_sync(0xffffffffu, byte, 1);
                    byte |= __shfl_xor_sync(0xffffffffu, byte, 2);
                    if ((lane & 3) == 0) blkp[a_index(R8, t, k0 + c) >> 2] = (uint8_t)byte;
                    if (lane == 0)
                        *reinterpret_cast<__half2 *>(blkp + int2_param_off(R8, nt) +
                                                     4 * ((int64_t)(k0 + c) * (4 * nt) + g)) = __halves2half2(sh, zh);
                }
            } else {
                for (int c = 0; c < kw; ++c) {
                    const int64_t o = base + a_index(R8, t, k0 + c);
                    if (pa.out_dtype == MILO_F32) ((float *)kv.data)[o] = acc[c];
                    else if (pa.out_dtype == MILO_BF16) ((__nv_bfloat16 *)kv.data)[o] = __float2bfloat16_rn(acc[c]);
                    else ((int8_t *)kv.data)[o] = c < kc ? quant_i8(acc[c], __fdiv_rn(amax[c], 127.f)) : (int8_t)0;
                }
            }
        }
        __syncthreads();
        if (pass == 0 && threadIdx.x < 32 && k0 + threadIdx.x < D)
            kv.scaleA[(int64_t)blk * D + k0 + threadIdx.x] =
                threadIdx.x < kc ? __fdiv_rn(amax[threadIdx.x], 127.f) : 0.f;
        __syncthreads();
    }
}

// grid (n_blk, 2 kinds), 128 threads: thread j writes column j of B_b
// (B_b[k][j] = W[j][k], k < r_b; zero rows up to R8) and, for INT8, its scale.
__global__ void __launch_bounds__(128) k_project_b(ProjArgs pa) {
    const int blk = blockIdx.x, kind = blockIdx.y, j = threadIdx.x;
    const KindView &kv = pa.kv[kind];
    const int r = kv.ranks[blk];
    const int R8 = rank_pad(r);
    const int b = blk % pa.n_b;
    const int nt = token_tiles(BlockGeo{pa.T, pa.block_len, pa.starts}.len(b));
    const int64_t base = kv.offsets[blk];
    const float *Wb = pa.W[kind] + (int64_t)blk * D * D + (int64_t)j * D;
    float s = 0.f;
    const bool i8 = pa.out_dtype == MILO_INT8 || pa.out_dtype == MILO_INT2;   // B is INT8 in both
    if (i8) {
        float m = 0.f;
        for (int k = 0; k < r; ++k) m = fmaxf(m, fabsf(Wb[k]));
        s = __fdiv_rn(m, 127.f);
        kv.scaleB[(int64_t)blk * D + j] = s;
    }
    for (int k = 0; k < R8; ++k) {
        const float w = k < r ? Wb[k] : 0.f;
        const int64_t o = pa.out_dtype == MILO_INT2
                              ? base + int2_b_off(R8, nt) + (b_index(R8, nt, k, j) - (int64_t)nt * R8 * FTILE)
                              : base + b_index(R8, nt, k, j);
        if (i8) ((int8_t *)kv.data)[o] = quant_i8(w, s);
        else if (pa.out_dtype == MILO_BF16) ((__nv_bfloat16 *)kv.data)[o] = __float2bfloat16_rn(w);
        else ((float *)kv.data)[o] = w;
    }
}

}  // namespace milo
