// decode_tc.cuh -- decode attention over retrieved compressed blocks on
// tcgen05 tensor cores (bf16 factors).
//
// Step "at inference a retriever selects blocks, whose low-rank factors are
// rebuilt before sparse attention" (evolve.pub review of MILO, Summary; FAQ
// "What is MILO").  A prep kernel lists the work items (layer, KV head,
// block, query pass); an item covers up to 128 queries (the sessions that
// selected the block times the GQA group).  One persistent CTA per SM walks
// the items:
//
//   producer warp   bulk-copies the block's factors (already in the tensor
//                   cores' canonical layout in HBM) through a 4-stage ring:
//                   A_K tile 0, B_K, A_K tiles 1.., A_V tiles.., B_V.
//   MMA warp        K-hat tile = A_K(tile) B_K       (M=128 tokens, N=128, K=r_K, bf16)
//                   S = K-tilde (TMEM) Q-tilde^T      (M=128 tokens, N=nq, K=128, fp16)
//                   O_A^T += A_V(tile)^T P            (M=128 ranks, N=nq, K=128 tokens, fp16)
//                   O = B_V^T (O_A / l)              (M=128 channels, N=nq, K=r_V, fp16)
//   8 epilogue      rotate the queries by -p*theta_i; RoPE of each rebuilt
//   warps           key row in registers (block-relative angle t*theta_i),
//                   K-tilde back to TMEM as fp16; softmax in the exp2 domain
//                   with a per-query reference max that is raised (and the
//                   running O_A^T and sums rescaled) only when a score exceeds
//                   it by more than 2^8; P (fp16) to shared memory, each A_V
//                   tile converted to fp16 in place; a ones row in A_V makes
//                   the PV product also return the softmax denominator.
//                   Two warps share each TMEM lane quadrant and split the
//                   columns between them.
//
// Keys and values are never written to memory.  Each (query, selected slot)
// gets a partial (max, sum, normalised output) merged by k_combine.
#pragma once
#include "decode_simt.cuh"
#include "tc_common.cuh"

// Timeline hooks: empty unless a tracing build defines them.
#ifndef MILO_TRACE_EVENT
#define MILO_TRACE_EVENT(id)
#endif
#ifndef MILO_TRACE_MMA
#define MILO_TRACE_MMA(id)
#endif

namespace milo {

constexpr int DT_EPI_WARPS = 8;
constexpr int DT_EPI = 32 * DT_EPI_WARPS;             // epilogue threads
constexpr int DT_THREADS = 64 + DT_EPI;               // warp 0 producer, 1 MMA, 2.. epilogue
constexpr int DT_STAGES = 4;
constexpr int DT_STAGE_BYTES = 128 * 256;             // 128 ranks x 128 tokens (or channels) x 16 bit
constexpr int DT_NQ = 128;                            // queries per item (pass)
constexpr uint32_t DT_TMEM_COLS = 512;
constexpr uint32_t DT_COL_D1 = 0, DT_COL_KT = 128, DT_COL_D2 = 256, DT_COL_OA = 384;
constexpr float DT_RESCALE = 8.f;                     // log2 headroom before the reference max moves

// One work item, written by k_dt_items.
struct DtItem {
    int32_t l, h, b, q0;
    int32_t nq, Tb, rK, rV;
    int64_t offK, offV;     // element offsets of the block in the data sections
    int32_t slot0, pad[3];  // start of the block's slot list
};

struct DecTcSmem {
    alignas(128) uint8_t stage[DT_STAGES][DT_STAGE_BYTES];
    alignas(128) uint8_t qt[DT_NQ * D * 2];      // rotated queries, fp16, K-major
    alignas(128) uint8_t pbuf[128 * DT_NQ * 2];  // P or O_A / l (fp16), MN-major
    float2 t1[HALF][32];                         // (cos, sin)((t % 32) theta_i)
    float2 t2[HALF][16];                         // (cos, sin)(32 (t / 32) theta_i)
    float cref[DT_NQ];                           // reference max per query (log2 domain)
    float cnew[DT_NQ];
    float lsum[DT_NQ];
    float wred[4][DT_NQ];
    int qpidx[DT_NQ];
    int flag;
    uint64_t full[DT_STAGES], empty[DT_STAGES];
    uint64_t d1_full, d1_empty, kt_full[2], kt_empty[2], q_full, q_empty;
    uint64_t d2_full, d2_empty, p_full, p_empty, oa_full, oa_staged, drain;
    uint32_t tmem_base;
    volatile int abort;
};

// Items of every (layer, head, block) with selecting queries, in (l, h, b,
// pass) order: grid over l*h*n_b.
__global__ void k_dt_items(DecodeArgs a, const int32_t *__restrict__ pstart, DtItem *__restrict__ items) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)a.L * a.H * a.n_b) return;
    const int b = (int)(e % a.n_b);
    const int64_t lh = e / a.n_b;
    const int per_lh = pstart[a.n_b];
    const int slot0 = a.slot_start[b];
    const int nqt = (a.slot_start[b + 1] - slot0) * a.G;
    const int64_t blk = lh * a.n_b + b;
    DtItem it;
    it.l = (int)(lh / a.H);
    it.h = (int)(lh % a.H);
    it.b = b;
    it.Tb = block_tokens(a.T, a.block_len, b);
    it.rK = a.kv[0].ranks[blk];
    it.rV = a.kv[1].ranks[blk];
    it.offK = a.kv[0].offsets[blk];
    it.offV = a.kv[1].offsets[blk];
    it.slot0 = slot0;
    it.pad[0] = it.pad[1] = it.pad[2] = 0;
    for (int p = 0, q0 = 0; q0 < nqt; ++p, q0 += DT_NQ) {
        it.q0 = q0;
        it.nq = min(DT_NQ, nqt - q0);
        items[lh * per_lh + pstart[b] + p] = it;
    }
}

__device__ __forceinline__ int r16_of(int R8) { return R8 <= 16 ? 16 : (R8 + 15) & ~15; }

// zero rank rows [R8, R16) of a chunk stored as [r/8][16 x 128 B] groups
__device__ __forceinline__ void zero_rows(uint8_t *chunk, int R8, int R16) {
    for (int off = R8 * 256; off < R16 * 256; off += 16) *reinterpret_cast<uint4 *>(chunk + off) = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(DT_THREADS, 1)
k_decode_tc(DecodeArgs a, const int32_t *__restrict__ pstart, const DtItem *__restrict__ items) {
    extern __shared__ __align__(128) unsigned char dt_raw[];
    DecTcSmem &sm = *reinterpret_cast<DecTcSmem *>(
        (reinterpret_cast<uintptr_t>(dt_raw) + 127) & ~static_cast<uintptr_t>(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_items = (int64_t)a.L * a.H * pstart[a.n_b];

    if (threadIdx.x == 0) {
        for (int s = 0; s < DT_STAGES; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.empty[s], 1); }
        tc::mbar_init(&sm.d1_full, 1);
        tc::mbar_init(&sm.d1_empty, DT_EPI);
        for (int k = 0; k < 2; ++k) { tc::mbar_init(&sm.kt_full[k], DT_EPI); tc::mbar_init(&sm.kt_empty[k], 1); }
        tc::mbar_init(&sm.q_full, 1);
        tc::mbar_init(&sm.q_empty, 1);
        tc::mbar_init(&sm.d2_full, 1);
        tc::mbar_init(&sm.d2_empty, DT_EPI);
        tc::mbar_init(&sm.p_full, 1);
        tc::mbar_init(&sm.p_empty, 1);
        tc::mbar_init(&sm.oa_full, 1);
        tc::mbar_init(&sm.oa_staged, 1);
        tc::mbar_init(&sm.drain, 1);
        sm.abort = 0;
        tc::fence_barrier_init();
    }
    // block-relative rotation tables from the fp64-derived (cos, sin)(t theta_i)
    for (int e = threadIdx.x; e < HALF * 32; e += DT_THREADS) {
        const int i = e / 32, u = e % 32;
        sm.t1[i][u] = u < a.block_len ? a.rope_t[(int64_t)u * HALF + i] : make_float2(1.f, 0.f);
    }
    for (int e = threadIdx.x; e < HALF * 16; e += DT_THREADS) {
        const int i = e / 16, v = e % 16;
        sm.t2[i][v] = 32 * v < a.block_len ? a.rope_t[(int64_t)(32 * v) * HALF + i] : make_float2(1.f, 0.f);
    }
    if (warp == 1) {
        tc::tmem_alloc(&sm.tmem_base, DT_TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint8_t *dataK = (const uint8_t *)a.kv[0].data;
    const uint8_t *dataV = (const uint8_t *)a.kv[1].data;

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            uint32_t alloc = 0;
            auto chunk = [&](const uint8_t *src, int R8, int R16, bool ones) -> bool {
                const int s = alloc % DT_STAGES;
                const uint32_t ph = (alloc / DT_STAGES) & 1u;
                if (!tc::mbar_wait(&sm.empty[s], ph ^ 1u)) return false;
                uint8_t *dst = sm.stage[s];
                zero_rows(dst, R8, R16);
                if (ones) {   // rank row 127 = 1.0 (fp16: the tile is converted before use)
                    for (int g = 0; g < 16; ++g)
                        *reinterpret_cast<uint4 *>(dst + 15 * 2048 + g * 128 + 7 * 16) =
                            make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
                }
                tc::fence_async_smem();
                const uint32_t bytes = (uint32_t)R8 * 256u;
                tc::mbar_arrive_expect_tx(&sm.full[s], bytes);
                if (bytes) tc::bulk_g2s(dst, src, bytes, &sm.full[s]);
                ++alloc;
                return true;
            };
            bool ok = true;
            for (int64_t i = blockIdx.x; i < n_items && ok && !sm.abort; i += gridDim.x) {
                const DtItem it = items[i];
                const int nt = token_tiles(it.Tb);
                const int R8K = rank_pad(it.rK), R8V = rank_pad(it.rV);
                const int R16K = r16_of(R8K), R16V = r16_of(R8V);
                const uint8_t *bK = dataK + 2 * it.offK, *bV = dataV + 2 * it.offV;
                const int64_t tileK = (int64_t)R8K * 256, tileV = (int64_t)R8V * 256;
                const bool ones = R8V <= 120;
                ok = ok && chunk(bK, R8K, R16K, false);                          // A_K tile 0
                ok = ok && chunk(bK + nt * tileK, R8K, R16K, false);             // B_K
                for (int t = 1; t < nt && ok; ++t) ok = chunk(bK + t * tileK, R8K, R16K, false);
                for (int t = 0; t < nt && ok; ++t) ok = chunk(bV + t * tileV, R8V, R16V, ones);
                ok = ok && chunk(bV + nt * tileV, R8V, R16V, false);             // B_V
            }
            if (!ok) sm.abort = 1;
            // drain: every stage's last copy has landed before the CTA exits
            for (int s = 0; s < DT_STAGES && alloc > 0; ++s) {
                const uint32_t last = alloc - 1 - s;
                if ((int)last < 0) break;
                tc::mbar_wait(&sm.full[last % DT_STAGES], (last / DT_STAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            uint32_t alloc = 0, n_d1 = 0, n_d2 = 0, n_kt[2] = {0, 0}, n_q = 0, n_p = 0, n_oa = 0;
            bool ok = true;
            auto stage_of = [&](uint32_t k) { return k % DT_STAGES; };
            auto wait_full = [&](uint32_t k) { return tc::mbar_wait(&sm.full[stage_of(k)], (k / DT_STAGES) & 1u); };
            for (int64_t i = blockIdx.x; i < n_items && ok && !sm.abort; i += gridDim.x) {
                const DtItem it = items[i];
                const int nt = token_tiles(it.Tb);
                const int nq16 = (it.nq + 15) & ~15;
                const int R16K = r16_of(rank_pad(it.rK)), R16V = r16_of(rank_pad(it.rV));
                const uint32_t aK0 = alloc, aBK = alloc + 1;
                auto aK = [&](int t) { return t == 0 ? aK0 : aBK + t; };
                const uint32_t aV0 = aBK + nt;
                const uint32_t aBV = aV0 + nt;
                alloc = aBV + 1;
                const uint32_t id_rb = tc::idesc_f16(128, 128, 1, 1, 1);     // bf16, A/B MN-major
                const uint32_t id_sc = tc::idesc_f16(128, nq16, 0, 0, 0);    // fp16, A tmem, B K-major
                const uint32_t id_pv = tc::idesc_f16(128, nq16, 0, 0, 1);    // fp16, A K-major, B MN-major
                const uint32_t id_o = tc::idesc_f16(128, nq16, 0, 1, 1);     // fp16, A/B MN-major
                const uint32_t lbo_p = (uint32_t)(nq16 / 8) * 128u;
                auto rebuild = [&](int t) -> bool {
                    if (!wait_full(aK(t))) return false;
                    if (t == 0 && !wait_full(aBK)) return false;
                    if (!tc::mbar_wait(&sm.d1_empty, (n_d1 & 1u) ^ 1u)) return false;
                    MILO_TRACE_MMA(t);
                    tc::tc_fence_after();
                    const uint32_t sa = tc::smem_u32(sm.stage[stage_of(aK(t))]);
                    const uint32_t sb = tc::smem_u32(sm.stage[stage_of(aBK)]);
                    for (int ks = 0; ks < R16K / 16; ++ks)
                        tc::mma_ss(tmem + DT_COL_D1, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                   tc::smem_desc(sb + ks * 4096, 2048, 128, tc::LAYOUT_NONE), id_rb, ks > 0);
                    tc::mma_commit(&sm.d1_full);
                    ++n_d1;
                    tc::mma_commit(&sm.empty[stage_of(aK(t))]);
                    if (t == nt - 1) tc::mma_commit(&sm.empty[stage_of(aBK)]);
                    return true;
                };
                auto scores = [&](int t) -> bool {
                    const int slot = t & 1;
                    if (!tc::mbar_wait(&sm.kt_full[slot], n_kt[slot] & 1u)) return false;
                    if (t == 0 && !tc::mbar_wait(&sm.q_full, n_q & 1u)) return false;
                    if (!tc::mbar_wait(&sm.d2_empty, (n_d2 & 1u) ^ 1u)) return false;
                    MILO_TRACE_MMA(4 + t);
                    tc::tc_fence_after();
                    const uint32_t sq = tc::smem_u32(sm.qt);
                    for (int ks = 0; ks < D / 16; ++ks)
                        tc::mma_ts(tmem + DT_COL_D2, tmem + DT_COL_KT + slot * 64 + ks * 8,
                                   tc::smem_desc(sq + ks * 256, 128, 2048, tc::LAYOUT_NONE), id_sc, ks > 0);
                    tc::mma_commit(&sm.d2_full);
                    ++n_d2;
                    tc::mma_commit(&sm.kt_empty[slot]);
                    ++n_kt[slot];
                    if (t == nt - 1) { tc::mma_commit(&sm.q_empty); ++n_q; }
                    return true;
                };
                auto pv = [&](int t) -> bool {
                    if (!tc::mbar_wait(&sm.p_full, n_p & 1u)) return false;
                    if (!wait_full(aV0 + t)) return false;
                    MILO_TRACE_MMA(8 + t);
                    tc::tc_fence_after();
                    const uint32_t sa = tc::smem_u32(sm.stage[stage_of(aV0 + t)]);
                    const uint32_t sp = tc::smem_u32(sm.pbuf);
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_ss(tmem + DT_COL_OA, tc::smem_desc(sa + ks * 256, 128, 2048, tc::LAYOUT_NONE),
                                   tc::smem_desc(sp + ks * 2 * lbo_p, lbo_p, 128, tc::LAYOUT_NONE), id_pv,
                                   (t | ks) != 0);
                    tc::mma_commit(&sm.p_empty);
                    ++n_p;
                    tc::mma_commit(&sm.empty[stage_of(aV0 + t)]);
                    if (t == nt - 1) tc::mma_commit(&sm.oa_full);
                    return true;
                };
                ok = rebuild(0);
                if (ok && nt > 1) ok = rebuild(1);
                for (int t = 0; t < nt && ok; ++t) {
                    ok = scores(t);
                    if (ok && t + 2 < nt) ok = rebuild(t + 2);
                    if (ok && t >= 1) ok = pv(t - 1);
                }
                if (ok) ok = pv(nt - 1);
                if (ok) {   // O = B_V^T (O_A / l), into the D1 columns
                    ok = tc::mbar_wait(&sm.oa_staged, n_oa & 1u) && tc::mbar_wait(&sm.d1_empty, (n_d1 & 1u) ^ 1u);
                    ++n_oa;
                    MILO_TRACE_MMA(12);
                    if (ok) {
                        tc::tc_fence_after();
                        const uint32_t sa = tc::smem_u32(sm.stage[stage_of(aBV)]);
                        const uint32_t sp = tc::smem_u32(sm.pbuf);
                        for (int ks = 0; ks < R16V / 16; ++ks)
                            tc::mma_ss(tmem + DT_COL_D1, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                       tc::smem_desc(sp + ks * 2 * lbo_p, lbo_p, 128, tc::LAYOUT_NONE), id_o,
                                       ks > 0);
                        tc::mma_commit(&sm.d1_full);
                        ++n_d1;
                        tc::mma_commit(&sm.p_empty);   // staging buffer free again
                        tc::mma_commit(&sm.empty[stage_of(aBV)]);
                    }
                }
            }
            if (!ok) sm.abort = 1;
            tc::mma_commit(&sm.drain);
            tc::mbar_wait(&sm.drain, 0);
        }
    } else {
        // ================================================================ epilogue (8 warps)
        const int quad = warp & 3;                   // TMEM lane quadrant of this warp
        const int eh = (warp - 2) >> 2;              // which of the two warps of the quadrant
        const int row = quad * 32 + lane;            // TMEM lane of this thread
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int et = threadIdx.x - 64;             // 0 .. DT_EPI-1
        const float kscale = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(d)
        uint32_t alloc = 0, n_d1 = 0, n_d2 = 0, n_kt[2] = {0, 0}, n_q = 0, n_p = 0, n_oa = 0;
        bool ok = true;
        auto ebar = [&]() { asm volatile("bar.sync 1, %0;" ::"n"(DT_EPI) : "memory"); };
        // named-barrier AND of every epilogue thread's flag: a wait that gave up
        // in one thread ends the loop in all of them, never a lone straggler
        // named-barrier OR of a flag over the epilogue threads
        auto any_all = [&](int v) -> bool {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
                "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)v), "n"(DT_EPI)
                : "memory");
            return r != 0;
        };
        // 2^x with the hardware approximation (relative error ~2^-22)
        auto ex2 = [](float x) -> float {
            float y;
            asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
            return y;
        };
        auto all_ok = [&](bool v) -> bool {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
                "bar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)v), "n"(DT_EPI)
                : "memory");
            return r != 0;
        };
        for (int64_t i = blockIdx.x; i < n_items && ok && !sm.abort; i += gridDim.x) {
            const DtItem it = items[i];
            MILO_TRACE_EVENT(0);
            const int nt = token_tiles(it.Tb);
            const int nq = it.nq, nq16 = (nq + 15) & ~15;
            const int R8V = rank_pad(it.rV), R16V = r16_of(R8V);
            const uint32_t aV0 = alloc + 1 + nt;
            const uint32_t aBV = alloc + 1 + 2 * nt;
            alloc = aBV + 1;
            const uint32_t lbo_p = (uint32_t)(nq16 / 8) * 128u;
            const bool ones = R8V <= 120;   // rank row 127 of A_V carries ones
            const int c_first = 16 * eh;    // this warp's 16-column chunks: c_first, +32, ...

            // ---- rotated queries R(-p) q, fp16, K-major [q/8][j/8][q%8][j%8];
            // four threads per query, 16 pairs each, every load issued up front
            ok = all_ok(tc::mbar_wait(&sm.q_empty, (n_q & 1u) ^ 1u));
            if (!ok) break;
            MILO_TRACE_EVENT(1);
            for (int u = et; u < 4 * nq16; u += DT_EPI) {
                const int qi = u >> 2, part = u & 3;          // pairs 16*part .. 16*part+15
                uint8_t *qrow = sm.qt + (qi >> 3) * 2048 + (qi & 7) * 16;
                if (qi < nq) {
                    const int gq = it.q0 + qi;
                    const int slot = a.slot_list[it.slot0 + gq / a.G];
                    const int g = gq % a.G;
                    const int s = slot / a.n_sel, jj = slot % a.n_sel;
                    const int hq = it.h * a.G + g;
                    const float4 *qv = reinterpret_cast<const float4 *>(a.q + (((int64_t)it.l * a.S + s) * a.Hq + hq) * D);
                    const float4 *cs = reinterpret_cast<const float4 *>(a.rope_q + (int64_t)slot * HALF);
                    if (part == 0) sm.qpidx[qi] = (int)((((int64_t)it.l * a.S + s) * a.Hq + hq) * a.n_sel + jj);
                    float4 xa[4], xb[4], cv[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) { xa[k] = qv[4 * part + k]; xb[k] = qv[16 + 4 * part + k]; }
#pragma unroll
                    for (int k = 0; k < 8; ++k) cv[k] = cs[8 * part + k];
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {          // pairs 16*part + 8*h8 .. +7
                        const float x0[8] = {xa[2 * h8].x, xa[2 * h8].y, xa[2 * h8].z, xa[2 * h8].w,
                                             xa[2 * h8 + 1].x, xa[2 * h8 + 1].y, xa[2 * h8 + 1].z, xa[2 * h8 + 1].w};
                        const float x1[8] = {xb[2 * h8].x, xb[2 * h8].y, xb[2 * h8].z, xb[2 * h8].w,
                                             xb[2 * h8 + 1].x, xb[2 * h8 + 1].y, xb[2 * h8 + 1].z, xb[2 * h8 + 1].w};
                        uint32_t lo[4], hi[4];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const float4 c2 = cv[4 * h8 + v];   // (cos, sin) of pairs 2v, 2v+1
                            const __half2 h0 = __floats2half2_rn(x0[2 * v] * c2.x + x1[2 * v] * c2.y,
                                                                 x0[2 * v + 1] * c2.z + x1[2 * v + 1] * c2.w);
                            const __half2 h1 = __floats2half2_rn(x1[2 * v] * c2.x - x0[2 * v] * c2.y,
                                                                 x1[2 * v + 1] * c2.z - x0[2 * v + 1] * c2.w);
                            lo[v] = *reinterpret_cast<const uint32_t *>(&h0);
                            hi[v] = *reinterpret_cast<const uint32_t *>(&h1);
                        }
                        const int g8 = 2 * part + h8;
                        *reinterpret_cast<uint4 *>(qrow + g8 * 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        *reinterpret_cast<uint4 *>(qrow + (8 + g8) * 128) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    }
                } else {
                    for (int g8 = 4 * part; g8 < 4 * part + 4; ++g8)
                        *reinterpret_cast<uint4 *>(qrow + g8 * 128) = make_uint4(0, 0, 0, 0);
                }
            }
            tc::fence_async_smem();
            ebar();
            if (et == 0) tc::mbar_arrive(&sm.q_full);
            ++n_q;
            MILO_TRACE_EVENT(2);

            // ---- RoPE of a rebuilt tile, K-tilde to TMEM (fp16 pairs); this warp: 2 of the 4 pair chunks
            auto rope = [&](int t) -> bool {
                const int slot = t & 1;
                const bool w1 = tc::mbar_wait(&sm.d1_full, n_d1 & 1u);
                const bool w2 = w1 && tc::mbar_wait(&sm.kt_empty[slot], (n_kt[slot] & 1u) ^ 1u);
                if (!all_ok(w2)) return false;
                MILO_TRACE_EVENT(4 + 4 * t);
                tc::tc_fence_after();
                const int tok = t * FTILE + row;             // token of this lane
                const int tl = tok & 31, th = tok >> 5;
                uint32_t xr2[2][16], yr2[2][16];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    tc::tmem_ld16(tmem + DT_COL_D1 + lane_off + (2 * eh + c) * 16, xr2[c]);
                    tc::tmem_ld16(tmem + DT_COL_D1 + lane_off + HALF + (2 * eh + c) * 16, yr2[c]);
                }
                tc::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int pc = 2 * eh + c;
                    const uint32_t(&xr)[16] = xr2[c];
                    const uint32_t(&yr)[16] = yr2[c];
                    uint32_t px[8], py[8];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        float xo[2], yo[2];
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) {
                            const int ii = pc * 16 + 2 * v + w2;
                            const float2 c1 = sm.t1[ii][tl], c2 = sm.t2[ii][th];
                            const float c = c1.x * c2.x - c1.y * c2.y;
                            const float s = c1.y * c2.x + c1.x * c2.y;
                            const float x = __uint_as_float(xr[2 * v + w2]), y = __uint_as_float(yr[2 * v + w2]);
                            xo[w2] = x * c - y * s;
                            yo[w2] = y * c + x * s;
                        }
                        const __half2 hx = __floats2half2_rn(xo[0], xo[1]);
                        const __half2 hy = __floats2half2_rn(yo[0], yo[1]);
                        px[v] = *reinterpret_cast<const uint32_t *>(&hx);
                        py[v] = *reinterpret_cast<const uint32_t *>(&hy);
                    }
                    tc::tmem_st8(tmem + DT_COL_KT + slot * 64 + lane_off + pc * 8, px);
                    tc::tmem_st8(tmem + DT_COL_KT + slot * 64 + lane_off + 32 + pc * 8, py);
                }
                tc::tmem_wait_st();
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.d1_empty);
                ++n_d1;
                tc::mbar_arrive(&sm.kt_full[slot]);
                ++n_kt[slot];
                MILO_TRACE_EVENT(5 + 4 * t);
                return true;
            };

            // ---- softmax of one score tile, P (fp16) to shared memory.  One pass
            // over the scores: p = 2^(x - cref); a CTA-wide vote decides whether
            // any score exceeded its reference by more than 2^8, in which case
            // (rare) the reference moves to the exact maximum and the running
            // O_A^T and sums are rescaled before P is written.
            auto softmax = [&](int t) -> bool {
                {
                    const bool w1 = tc::mbar_wait(&sm.d2_full, n_d2 & 1u);
                    const bool w2 = w1 && tc::mbar_wait(&sm.p_empty, (n_p & 1u) ^ 1u);   // P buffer free
                    if (!all_ok(w2)) return false;
                }
                MILO_TRACE_EVENT(6 + 4 * t);
                tc::tc_fence_after();
                const int tok = t * FTILE + row;
                const bool valid = tok < it.Tb;
                const int nch = (nq16 - c_first + 31) / 32;   // this warp's 16-column chunks (<= 4)
                // two chunks per TMEM round trip: at most 32 score registers live
                auto load2 = [&](int k, uint32_t (&r0)[16], uint32_t (&r1)[16]) {
                    tc::tmem_ld16(tmem + DT_COL_D2 + lane_off + c_first + 32 * k, r0);
                    if (k + 1 < nch) tc::tmem_ld16(tmem + DT_COL_D2 + lane_off + c_first + 32 * (k + 1), r1);
                    tc::tmem_wait_ld();
                };
                if (t == 0) {   // reference max: the scores of the item's first token (lane 0 of quadrant 0)
                    if (quad == 0) {
                        for (int k = 0; k < nch; k += 2) {
                            uint32_t r0[16], r1[16];
                            load2(k, r0, r1);
                            if (lane == 0) {
#pragma unroll
                                for (int v = 0; v < 16; ++v) sm.cref[c_first + 32 * k + v] = __uint_as_float(r0[v]) * kscale;
                                if (k + 1 < nch)
#pragma unroll
                                    for (int v = 0; v < 16; ++v)
                                        sm.cref[c_first + 32 * (k + 1) + v] = __uint_as_float(r1[v]) * kscale;
                            }
                        }
                    }
                    ebar();
                }
                int over = 0;
                for (int k = 0; k < nch; k += 2) {
                    uint32_t r0[16], r1[16];
                    load2(k, r0, r1);
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const int q0 = c_first + 32 * k + v, q1 = q0 + 32;
                        if (valid && q0 < nq && __uint_as_float(r0[v]) * kscale > sm.cref[q0] + DT_RESCALE) over = 1;
                        if (valid && k + 1 < nch && q1 < nq && __uint_as_float(r1[v]) * kscale > sm.cref[q1] + DT_RESCALE)
                            over = 1;
                    }
                }
                if (any_all(over)) {
                    // rare path: exact column maxima of this tile, rescale running state
                    for (int k = 0; k < nch; ++k) {
                        uint32_t r0[16];
                        tc::tmem_ld16(tmem + DT_COL_D2 + lane_off + c_first + 32 * k, r0);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int v = 0; v < 16; ++v) {
                            float x = valid ? __uint_as_float(r0[v]) * kscale : -INFINITY;
                            for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                            if (lane == 0) sm.wred[quad][c_first + 32 * k + v] = x;
                        }
                    }
                    ebar();
                    if (et < nq16) {
                        const float m = fmaxf(fmaxf(sm.wred[0][et], sm.wred[1][et]), fmaxf(sm.wred[2][et], sm.wred[3][et]));
                        sm.cnew[et] = fmaxf(sm.cref[et], m);
                    }
                    ebar();
                    if (t > 0) {   // O_A^T columns (all rank lanes) scaled by 2^(cref - cnew)
                        for (int k = 0; k < nch; ++k) {
                            const int c0 = c_first + 32 * k;
                            uint32_t o[16];
                            tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0, o);
                            tc::tmem_wait_ld();
                            uint32_t w[8];
                            #pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                #pragma unroll
                                for (int v = 0; v < 8; ++v) {
                                    const int q = c0 + hh * 8 + v;
                                    w[v] = __float_as_uint(__uint_as_float(o[hh * 8 + v]) * ex2(sm.cref[q] - sm.cnew[q]));
                                }
                                tc::tmem_st8(tmem + DT_COL_OA + lane_off + c0 + hh * 8, w);
                            }
                        }
                        tc::tmem_wait_st();
                        if (et < nq16) sm.lsum[et] *= ex2(sm.cref[et] - sm.cnew[et]);
                    }
                    ebar();
                    if (et < nq16) sm.cref[et] = sm.cnew[et];
                    ebar();
                }
                // p = 2^(x - cref), fp16, MN-major [t/8][q/8][t%8][q%8]
                for (int k2 = 0; k2 < nch; k2 += 2) {
                  uint32_t rr[2][16];
                  load2(k2, rr[0], rr[1]);
#pragma unroll
                  for (int kk = 0; kk < 2; ++kk) {
                    const int k = k2 + kk;
                    if (k >= nch) break;
                    const uint32_t(&rk)[16] = rr[kk];
                    const int c0 = c_first + 32 * k;
                    uint32_t pk[8];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        float p2[2];
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) {
                            const int q = c0 + 2 * v + w2;
                            p2[w2] = (valid && q < nq) ? ex2(__uint_as_float(rk[2 * v + w2]) * kscale - sm.cref[q]) : 0.f;
                        }
                        const __half2 hb = __floats2half2_rn(p2[0], p2[1]);
                        pk[v] = *reinterpret_cast<const uint32_t *>(&hb);
                        if (!ones) {   // no spare rank row: column sums of the rounded P
                            const float2 pr = __half22float2(hb);
                            float s0 = pr.x, s1 = pr.y;
                            for (int o = 16; o; o >>= 1) {
                                s0 += __shfl_xor_sync(0xffffffffu, s0, o);
                                s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                            }
                            if (lane == 0) {
                                atomicAdd(&sm.lsum[c0 + 2 * v], s0);
                                atomicAdd(&sm.lsum[c0 + 2 * v + 1], s1);
                            }
                        }
                    }
                    uint8_t *dst = sm.pbuf + (row >> 3) * lbo_p + (c0 >> 3) * 128 + (row & 7) * 16;
                    *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4 *>(dst + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                  }
                }
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.d2_empty);
                ++n_d2;
                return true;
            };

            // ---- A_V tile to fp16 in place, then hand P and the tile to the PV
            // product.  Runs after the next RoPE: the tile's ring slot may only
            // be refilled once the last rebuild of this block has been issued.
            auto release_p = [&](int t) -> bool {
                const uint32_t av = aV0 + t;
                if (!all_ok(tc::mbar_wait(&sm.full[av % DT_STAGES], (av / DT_STAGES) & 1u))) return false;
                uint32_t *w = reinterpret_cast<uint32_t *>(sm.stage[av % DT_STAGES]);
                for (int e = et; e < R8V * 64; e += DT_EPI) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
                    const __half2 h2 = __floats2half2_rn(f.x, f.y);
                    w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                tc::fence_async_smem();
                ebar();
                if (et == 0) tc::mbar_arrive(&sm.p_full);
                ++n_p;
                MILO_TRACE_EVENT(7 + 4 * t);
                return true;
            };

            if (et < nq16) sm.lsum[et] = 0.f;
            ebar();
            ok = rope(0);
            if (ok && nt > 1) ok = rope(1);
            for (int t = 0; t < nt && ok; ++t) {
                ok = softmax(t);
                if (ok && t + 2 < nt) ok = rope(t + 2);
                if (ok) ok = release_p(t);
            }
            if (!ok) break;
            {   // B_V (bf16, landed in its stage) to fp16 in place, while the last PV runs
                const uint32_t s = aBV % DT_STAGES;
                if (!(ok = all_ok(tc::mbar_wait(&sm.full[s], (aBV / DT_STAGES) & 1u)))) break;
                uint32_t *w = reinterpret_cast<uint32_t *>(sm.stage[s]);
                for (int e = et; e < R8V * 64; e += DT_EPI) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
                    const __half2 h2 = __floats2half2_rn(f.x, f.y);
                    w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
            }
            // ---- O_A^T finished: denominators, O_A / l to fp16 staging
            {
                const bool w1 = tc::mbar_wait(&sm.oa_full, n_oa & 1u);
                const bool w2 = w1 && tc::mbar_wait(&sm.p_empty, (n_p & 1u) ^ 1u);   // last PV done
                if (!(ok = all_ok(w2))) break;
            }
            MILO_TRACE_EVENT(20);
            tc::tc_fence_after();
            if (ones && quad == 3) {   // the ones row (rank lane 127) holds sum_t p
                for (int c0 = c_first; c0 < nq16; c0 += 32) {
                    uint32_t r[16];
                    tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0, r);
                    tc::tmem_wait_ld();
                    if (lane == 31)
                        #pragma unroll
                        for (int v = 0; v < 16; ++v) sm.lsum[c0 + v] += __uint_as_float(r[v]);
                }
            }
            ebar();
            if (et < nq16) sm.cnew[et] = (et < nq && sm.lsum[et] > 0.f) ? __frcp_rn(sm.lsum[et]) : 0.f;
            ebar();
            for (int c0 = c_first; c0 < nq16; c0 += 32) {
                uint32_t r[16];
                tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0, r);
                tc::tmem_wait_ld();
                if (row < R16V) {
                    uint32_t pk[8];
                    #pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        float o2[2];
                        #pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) o2[w2] = __uint_as_float(r[2 * v + w2]) * sm.cnew[c0 + 2 * v + w2];
                        const __half2 hh = __floats2half2_rn(o2[0], o2[1]);
                        pk[v] = *reinterpret_cast<const uint32_t *>(&hh);
                    }
                    uint8_t *dst = sm.pbuf + (row >> 3) * lbo_p + (c0 >> 3) * 128 + (row & 7) * 16;
                    *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4 *>(dst + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            ebar();
            if (et == 0) tc::mbar_arrive(&sm.oa_staged);
            MILO_TRACE_EVENT(21);
            ++n_oa;
            ++n_p;   // the O product's commit frees the staging buffer
            // ---- O (lanes = channels, columns = queries) to the partials
            if (!(ok = all_ok(tc::mbar_wait(&sm.d1_full, n_d1 & 1u)))) break;
            MILO_TRACE_EVENT(22);
            tc::tc_fence_after();
            for (int c0 = c_first; c0 < nq16; c0 += 32) {
                uint32_t r[16];
                tc::tmem_ld16(tmem + DT_COL_D1 + lane_off + c0, r);
                tc::tmem_wait_ld();
                #pragma unroll
                for (int v = 0; v < 16; ++v) {
                    const int q = c0 + v;
                    if (q < nq) a.part_o[(int64_t)sm.qpidx[q] * D + row] = __uint_as_float(r[v]);
                }
            }
            if (et < nq) a.part_ml[sm.qpidx[et]] = make_float2(sm.cref[et] * 0.69314718055994531f, sm.lsum[et]);
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.d1_empty);
            ++n_d1;
            ebar();
            MILO_TRACE_EVENT(23);
        }
        if (!ok) sm.abort = 1;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, DT_TMEM_COLS);
}

inline size_t decode_tc_smem_bytes() { return sizeof(DecTcSmem) + 128; }

inline bool decode_tc_supported(const DecodeArgs &a) {
    if (getenv("MILO_FORCE_SIMT")) return false;
    return a.factor_dtype == MILO_BF16 && a.block_len <= 512;
}

inline cudaError_t decode_tc_set_attrs() {
    return cudaFuncSetAttribute(k_decode_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_tc_smem_bytes());
}

// upper bound of the number of items: sum_b ceil(q_b / 128) <= n_b + S n_sel G / 128 per (l, h)
inline int64_t decode_tc_max_items(int L, int H, int n_b, int64_t slots, int G) {
    return (int64_t)L * H * (n_b + (slots * G + DT_NQ - 1) / DT_NQ);
}

inline cudaError_t launch_decode_tc(const DecodeArgs &a, const int32_t *pstart, DtItem *items, int sms,
                                    cudaStream_t s) {
    const int64_t n = (int64_t)a.L * a.H * a.n_b;
    k_dt_items<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a, pstart, items);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_decode_tc<<<sms, DT_THREADS, decode_tc_smem_bytes(), s>>>(a, pstart, items);
    return cudaGetLastError();
}

}  // namespace milo
