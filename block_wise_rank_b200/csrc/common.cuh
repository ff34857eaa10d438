// common.cuh -- shared device helpers of libmilo (one translation unit).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "milo.h"

namespace milo {

constexpr int D = 128;          // head dimension served by every kernel
constexpr int HALF = D / 2;     // RoPE pairs (i, i + 64)

// Device status word (one per device that loads the library).  Kernels OR
// bits into it; milo_get_status reads and clears it.
enum : unsigned {
    ST_NOT_CONVERGED = 1u,
    ST_NONFINITE = 2u,
    ST_BOUNDS = 4u,
    ST_UNSORTED = 8u,
    ST_TIMEOUT = 16u,
};
__device__ unsigned g_status;

__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_status, bits); }
// Jacobi rounds that applied rotations, summed over all (block, kind) solves
// since the last read (work counter for the eigensolve's throughput).
__device__ unsigned long long g_jacobi_rounds;

__host__ __device__ __forceinline__ int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// tokens in block b of a (layer, head) row of T tokens
__host__ __device__ __forceinline__ int block_tokens(int T, int block_len, int b) {
    int r = T - b * block_len;
    return r < block_len ? r : block_len;
}

// Block b of every (layer, head) covers tokens [start(b), start(b) + len(b)):
// a fixed length block_len (the last block may be short), or given starts
// (variable-length blocks: starts[0] = 0, ascending, starts[n_b] = T, every
// length in [1, block_len]; `starts` is then device-readable).
struct BlockGeo {
    int T, block_len;
    const int32_t *starts;   // [n_b + 1] or null
    __device__ __forceinline__ int start(int b) const { return starts ? starts[b] : b * block_len; }
    __device__ __forceinline__ int len(int b) const {
        return starts ? starts[b + 1] - starts[b] : block_tokens(T, block_len, b);
    }
};

// largest admissible rank of a block: min(T_b, d, r_max if > 0)
__host__ __device__ __forceinline__ int block_cap(int Tb, int r_max) {
    int c = Tb < D ? Tb : D;
    if (r_max > 0 && r_max < c) c = r_max;
    return c;
}

// element loads of a factor / cache in any supported dtype, as fp32
template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f32<int8_t>(int8_t v) { return (float)v; }

__device__ __forceinline__ float load_elem(const void *base, int64_t i, int dtype) {
    switch (dtype) {
    case MILO_F32: return ((const float *)base)[i];
    case MILO_BF16: return __bfloat162float(((const __nv_bfloat16 *)base)[i]);
    default: return (float)((const int8_t *)base)[i];
    }
}

// bytes of one offset unit of the factor data (elements; bytes for 2-bit codes)
__host__ __device__ __forceinline__ int dtype_bytes(int dtype) {
    return dtype == MILO_F32 ? 4 : (dtype == MILO_BF16 ? 2 : 1);
}

// Packed factor layout of one block (element offsets from the block start).
// Ranks are padded to R8 = round_up(r_b, 8) with zero rows and tokens to
// whole tiles of FTILE = 128 with zero columns.  Tile tau of A_b^T holds
// tokens [128 tau, 128 tau + 128) as [k/8][u/8][k%8][u%8]; B_b follows the
// tiles as [k/8][j/8][k%8][j%8].  This is the tensor cores' canonical
// no-swizzle operand layout (8 x 8 core matrices, 16 bytes per bf16 row),
// so one contiguous copy lands a tile ready for the MMA.
constexpr int FTILE = 128;

__host__ __device__ __forceinline__ int rank_pad(int r) { return (r + 7) & ~7; }
__host__ __device__ __forceinline__ int token_tiles(int Tb) { return (Tb + FTILE - 1) / FTILE; }
__host__ __device__ __forceinline__ int64_t block_elems(int r, int Tb) {
    return (int64_t)rank_pad(r) * (token_tiles(Tb) * FTILE + D);
}
// A_b[t][k] (token t, rank k); R8 = rank_pad(r_b)
__host__ __device__ __forceinline__ int64_t a_index(int R8, int t, int k) {
    const int tau = t / FTILE, u = t % FTILE;
    return (int64_t)tau * R8 * FTILE + (k >> 3) * (8 * FTILE) + (u >> 3) * 64 + (k & 7) * 8 + (u & 7);
}
// B_b[k][j] (rank k, channel j)
__host__ __device__ __forceinline__ int64_t b_index(int R8, int n_tiles, int k, int j) {
    return (int64_t)n_tiles * R8 * FTILE + (k >> 3) * (8 * D) + (j >> 3) * 64 + (k & 7) * 8 + (j & 7);
}

// 2-bit factors (MILO_INT2), byte offsets from the block start: A_b's codes
// four tokens per byte at a_index / 4 (token u at bits 2 (u % 4)); B_b's
// INT8 codes after them at b_index - nt R8 FTILE; then A_b's (scale, zero)
// fp16 pairs per rank k and group of INT2_GROUP tokens, [k][t / INT2_GROUP].
constexpr int INT2_GROUP = 32;
__host__ __device__ __forceinline__ int64_t int2_b_off(int R8, int nt) { return (int64_t)nt * R8 * (FTILE / 4); }
__host__ __device__ __forceinline__ int64_t int2_param_off(int R8, int nt) {
    return int2_b_off(R8, nt) + (int64_t)R8 * D;
}
__host__ __device__ __forceinline__ int64_t int2_block_bytes(int r, int Tb) {
    const int R8 = rank_pad(r), nt = token_tiles(Tb);
    return int2_param_off(R8, nt) + (int64_t)R8 * nt * (FTILE / INT2_GROUP) * 4;
}
// a block's size in offset units of its factor type
__host__ __device__ __forceinline__ int64_t block_units(int dtype, int r, int Tb) {
    return dtype == MILO_INT2 ? int2_block_bytes(r, Tb) : block_elems(r, Tb);
}

// One kind's section of the factor arena (device pointers).
struct KindView {
    int32_t *ranks;
    int64_t *offsets;
    float *sigma;
    double *eps;
    float *scaleA;
    float *scaleB;
    void *data;
};

}  // namespace milo
