// gram_tc.cuh -- per-block Gram matrices G_b = X_b^T X_b on tcgen05 tensor
// cores (bf16 caches), fed by TMA.
//
// Step "SVD of K and of V per block" (evolve.pub review of MILO, Summary):
// the Gram matrix is the dense contraction of the per-block SVD.  One
// persistent CTA per SM walks the (kind, block) items.  Warp 0 streams
// 64-token x 128-channel tiles of X_b with 2-D TMA loads (128-byte swizzle,
// no multicast) into a 6-stage ring; warp 1 issues tcgen05.mma with M = N =
// 128 and K = 16 per instruction, the same shared-memory tile serving as both
// MN-major operands (A = X_b^T, B = X_b^T, so D = X_b^T X_b), accumulating in
// a double-buffered fp32 TMEM tile; warps 2-5 drain the finished tile with
// tcgen05.ld and write G_b to global memory while the next block accumulates.
#pragma once
#include "tc_common.cuh"

namespace milo {

constexpr int GT_STAGES = 6;
constexpr int GT_CHUNK = 64;                       // tokens per stage
constexpr int GT_STAGE_BYTES = GT_CHUNK * D * 2;   // two 64 x 64 bf16 boxes
constexpr int GT_THREADS = 192;
constexpr uint32_t GT_TMEM_COLS = 256;             // 2 x (128 x 128 fp32)

struct GramTcSmem {
    alignas(1024) uint8_t stage[GT_STAGES][GT_STAGE_BYTES];
    uint64_t full[GT_STAGES], empty[GT_STAGES];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort;
};

__global__ void __launch_bounds__(GT_THREADS, 1)
k_gram_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, float *__restrict__ G_out,
          int64_t n_blk, int n_b, int Tn, int block_len) {
    extern __shared__ __align__(1024) unsigned char gt_raw[];
    // aligned by pointer arithmetic: the compiler keeps the shared address space
    GramTcSmem &sm = *reinterpret_cast<GramTcSmem *>(gt_raw + ((1024u - (tc::smem_u32(gt_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_items = 2 * n_blk;
    const int chunks = block_len / GT_CHUNK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < GT_STAGES; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.empty[s], 1); }
        for (int a = 0; a < 2; ++a) { tc::mbar_init(&sm.acc_full[a], 1); tc::mbar_init(&sm.acc_empty[a], 128); }
        tc::mbar_init(&sm.drain, 1);
        sm.abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&sm.tmem_base, GT_TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------- producer
        tc::prefetch_tmap(&tmK);
        tc::prefetch_tmap(&tmV);
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        for (int64_t w = blockIdx.x; w < n_items && !sm.abort; w += gridDim.x) {
            const int kind = (int)(w / n_blk);
            const int64_t blk = w % n_blk;
            const CUtensorMap *map = kind == 0 ? &tmK : &tmV;
            const int row0 = (int)((blk / n_b) * Tn + (blk % n_b) * block_len);
            for (int c = 0; c < chunks; ++c) {
                if (!tc::mbar_wait(&sm.empty[stage], phase ^ 1u)) { sm.abort = 1; break; }
                tc::mbar_arrive_expect_tx(&sm.full[stage], GT_STAGE_BYTES);
                tc::tma_load_2d(sm.stage[stage], map, 0, row0 + c * GT_CHUNK, &sm.full[stage]);
                tc::tma_load_2d(sm.stage[stage] + GT_STAGE_BYTES / 2, map, 64, row0 + c * GT_CHUNK, &sm.full[stage]);
                ++issued;
                if (++stage == GT_STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        if (sm.abort) {
            // let the copies already issued land before the CTA exits
            for (int i = 0; i < GT_STAGES && i < issued; ++i) {
                if (--stage < 0) { stage = GT_STAGES - 1; phase ^= 1u; }
                tc::mbar_wait(&sm.full[stage], phase);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = tc::idesc_f16(128, 128, 1, 1, 1);
        int stage = 0;
        uint32_t phase = 0, acc = 0, acc_phase = 0;
        for (int64_t w = blockIdx.x; w < n_items && !sm.abort; w += gridDim.x) {
            if (!tc::mbar_wait(&sm.acc_empty[acc], acc_phase ^ 1u)) { sm.abort = 1; break; }
            tc::tc_fence_after();
            const uint32_t d_tmem = tmem + acc * 128;
            for (int c = 0; c < chunks; ++c) {
                if (!tc::mbar_wait(&sm.full[stage], phase)) { sm.abort = 1; break; }
                tc::tc_fence_after();
                const uint32_t base = tc::smem_u32(sm.stage[stage]);
#pragma unroll
                for (int ks = 0; ks < GT_CHUNK / 16; ++ks) {
                    // 16 tokens = two 8-row swizzle atoms (SBO = 1024 B); the
                    // two 64-channel halves sit GT_STAGE_BYTES/2 apart (LBO)
                    const uint64_t dsc = tc::smem_desc(base + ks * 2048, GT_STAGE_BYTES / 2, 1024, tc::LAYOUT_SW128);
                    tc::mma_ss(d_tmem, dsc, dsc, idesc, (c | ks) != 0);
                }
                tc::mma_commit(&sm.empty[stage]);
                if (++stage == GT_STAGES) { stage = 0; phase ^= 1u; }
            }
            if (sm.abort) break;
            tc::mma_commit(&sm.acc_full[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        tc::mma_commit(&sm.drain);
        tc::mbar_wait(&sm.drain, 0);
    } else if (warp >= 2) {
        // ---------------------------------------------------------- epilogue
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        uint32_t acc = 0, acc_phase = 0;
        for (int64_t w = blockIdx.x; w < n_items && !sm.abort; w += gridDim.x) {
            if (!tc::mbar_wait(&sm.acc_full[acc], acc_phase)) { sm.abort = 1; break; }
            tc::tc_fence_after();
            const int kind = (int)(w / n_blk);
            const int64_t blk = w % n_blk;
            float *G = G_out + ((int64_t)kind * n_blk + blk) * D * D + (int64_t)row * D;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + acc * 128 + ((uint32_t)(quad * 32) << 16) + cc * 32, r);
                tc::tmem_wait_ld();
                float4 *dst = reinterpret_cast<float4 *>(G + cc * 32);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    dst[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                         __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.acc_empty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, GT_TMEM_COLS);
}

inline size_t gram_tc_smem_bytes() { return sizeof(GramTcSmem) + 1024; }

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// 2-D map over a bf16 cache viewed as [rows][128], 64 x 64 boxes, 128B swizzle
inline bool make_cache_map(CUtensorMap *m, const void *X, uint64_t rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool gram_tc_supported(int T, int block_len) {
    if (getenv("MILO_FORCE_SIMT")) return false;
    return block_len % GT_CHUNK == 0 && T % block_len == 0 && encode_tiled_fn() != nullptr;
}

inline cudaError_t gram_tc_set_attrs() {
    return cudaFuncSetAttribute(k_gram_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gram_tc_smem_bytes());
}

inline cudaError_t launch_gram_tc(const __nv_bfloat16 *K, const __nv_bfloat16 *V, int LH, int T, int block_len,
                                  int n_b, float *G, int64_t n_blk, int sms, cudaStream_t s) {
    CUtensorMap mk, mv;
    const uint64_t rows = (uint64_t)LH * T;
    if (!make_cache_map(&mk, K, rows) || !make_cache_map(&mv, V, rows)) return cudaErrorInvalidValue;
    const int grid = (int)std::min<int64_t>(2 * n_blk, (int64_t)sms);
    k_gram_tc<<<grid, GT_THREADS, gram_tc_smem_bytes(), s>>>(mk, mv, G, n_blk, n_b, T, block_len);
    return cudaGetLastError();
}

}  // namespace milo
