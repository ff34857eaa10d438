// decode_tc.cuh -- decode attention over retrieved compressed blocks on
// tcgen05 tensor cores (bf16 factors).
//
// Step "at inference a retriever selects blocks, whose low-rank factors are
// rebuilt before sparse attention" (evolve.pub review of MILO, Summary; FAQ
// "What is MILO").  A prep kernel lists the work items (layer, KV head,
// block, query pass); an item covers up to 64 queries (the sessions that
// selected the block times the GQA group).  One persistent CTA per SM claims
// items dynamically and streams them through five roles that meet only at
// mbarriers, every wait bounded:
//
//   K producer (warp 0)  claims items and keeps their descriptors in a
//                        shared-memory table; bulk-copies each item's B_K
//                        into its own small ring and the 128-token A_K tiles
//                        into another (already in the tensor cores' canonical
//                        operand layout in HBM).
//   V producer (warp 1)  bulk-copies the A_V tiles and B_V into a third ring.
//   K MMA (warp 2)       rebuild  K-hat tile = A_K(tile) B_K          (M=128 tokens, N=128, K=r_K, bf16)
//                        scores   S = K-tilde (TMEM) Q-tilde^T         (M=128 tokens, N=nq, K=128, fp16)
//                        in the order R0 R1 S0 R2 S1 ..., two rebuild and
//                        two score buffers in tensor memory.
//   V warp (warp 3)      converts each A_V tile and B_V to fp16 in place
//                        (appending a row of ones to A_V when a rank row is
//                        free) and issues O_A^T += A_V(tile)^T P and, last,
//                        O = B_V^T (O_A / l)                           (M=128, N=nq, fp16)
//   epilogue (8 warps)   two groups of four, one warp per TMEM lane quadrant;
//                        group h owns RoPE pairs and query columns
//                        32h .. 32h+31.  Per tile, a token row per thread:
//                          RoPE of the next tile: rotate the rebuilt keys
//                          by the in-block angle t theta_i, t = 32 v + u with
//                          u the thread's lane, (cos, sin)(u theta_i) held in
//                          registers, packed f32x2 arithmetic, K-tilde packed
//                          to fp16 in place;
//                          softmax of this tile: exp2 against a per-query
//                          reference max raised only when some p exceeds
//                          2^8, P (fp16) to shared memory;
//                        and per item: the rotated queries R(-p) q of the
//                        next item, the denominators and O_A / l staging of
//                        the previous item (deferred so that its last product
//                        has run), and the previous item's O read out to the
//                        fp16 partials.
//
// The ones row makes the PV product return the softmax denominators as one
// more row of O_A^T.  Keys and values are never written to memory.  Each
// (query, selected slot) gets a partial (max, sum, normalised output in
// fp16) merged by k_combine.
#pragma once
#include "decode_simt.cuh"
#include "tc_common.cuh"

// Timeline hook: empty unless a tracing build defines it (event code, item,
// tile).
#ifndef MILO_DT_TRACE
#define MILO_DT_TRACE(code, n, t)
#endif

namespace milo {

constexpr int DT_NQ = 64;                         // queries per item (pass)
constexpr int DT_THREADS = 384;                   // 12 warps
constexpr int DT_W_EPI = 4;                       // epilogue warps 4 .. 11
constexpr int DT_NEPI = 256;                      // epilogue threads
constexpr int DT_VRING = 64 * 1024;               // A_V tiles (+ ones group) and B_V
constexpr int DT_AKRING = 48 * 1024;              // A_K tiles
constexpr int DT_BKRING = 36 * 1024;              // B_K per item
constexpr int DT_NSLOT = 16;                      // tiles in flight per tile ring
constexpr int DT_NBK = 4;                         // B_K in flight
constexpr int DT_NITAB = 16;                      // item table entries
constexpr int DT_AHEAD = 4;                       // items claimed ahead of the copies
constexpr int DT_PBUF = 128 * DT_NQ * 2;          // one P buffer: 128 tokens x 64 queries, fp16
constexpr uint32_t DT_TMEM_COLS = 512;
constexpr uint32_t DT_COL_KH = 0;                 // two 128-column rebuild buffers
constexpr uint32_t DT_COL_S = 256;                // two 64-column score buffers
constexpr uint32_t DT_COL_OA = 384;               // two 64-column O_A^T / O buffers
constexpr float DT_OVER = 8.f;                    // log2 headroom before the reference max moves

// One work item, written by k_dt_items.  l < 0 marks the end of a CTA's items
// in its table.
struct DtItem {
    int32_t l, h, b, q0;
    int32_t nq, Tb, rK, rV;
    int64_t offK, offV;     // element offsets of the block in the data sections
    int32_t slot0, pad[3];  // start of the block's slot list
};

struct DecTcSmem {
    // The V ring comes first: the PV product reads 128 rank rows from an A_V
    // tile's start, past a short tile, and those reads must stay inside the
    // CTA's shared memory (the rows they feed are never used).
    alignas(1024) uint8_t vring[DT_VRING];
    alignas(1024) uint8_t akring[DT_AKRING];
    alignas(1024) uint8_t bkring[DT_BKRING];
    alignas(1024) uint8_t qt[DT_NQ * D * 2];      // rotated queries, fp16, K-major (one item)
    alignas(1024) uint8_t pbuf[2][DT_PBUF];       // P (fp16, MN-major)
    alignas(1024) uint8_t stage[DT_PBUF];         // O_A / l for the last product (fp16, MN-major)
    float4 rhi[16][HALF / 2];                     // (cos, sin)(32 v theta_i) of pairs (2k, 2k+1): (c0, c1, s0, s1)
    DtItem itab[DT_NITAB];                        // claimed items, entry n % NITAB = this CTA's n-th
    float cref[2][DT_NQ];                         // reference max per query (log2 domain), per item parity
    float cscale[2][DT_NQ];                       // rescale factors, then 1 / l
    float lsum[2][DT_NQ];
    int cmax[DT_NQ];                              // column maxima, order-preserving int encoding
    int qpidx[4][DT_NQ];                          // partial index of each query, per item (mod 4): the
                                                  // next item's are written before the previous item's are read
    uint32_t ak_off[DT_NSLOT], v_off[DT_NSLOT], bk_off[DT_NBK];
    uint64_t item_full[DT_NITAB], item_free[DT_NITAB];
    uint64_t akfull[DT_NSLOT], akempty[DT_NSLOT];
    uint64_t vfull[DT_NSLOT], vempty[DT_NSLOT];
    uint64_t bkfull[DT_NBK], bkempty[DT_NBK];
    uint64_t kh_full[2], kh_free[2], kt_full[2];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], p_free[2];
    uint64_t qt_full, qt_free, st_full, st_free;
    uint64_t oa_full[2], oa_free[2], o_full[2];
    uint64_t drain_k, drain_v;
    uint32_t tmem_base;
    volatile int abort;
};

// readers that free an item table entry: V producer, K MMA, V warp, 8 epilogue warps
constexpr int DT_ITEM_READERS = 1 + 1 + 1 + 8;

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

__host__ __device__ __forceinline__ int r16_of(int R8) { return R8 <= 16 ? 16 : (R8 + 15) & ~15; }

// Geometry of one item as every role sees it.
struct DtGeo {
    int nt;            // 128-token tiles
    int R8K, R16K;     // key rank padded to 8 / to the MMA's K step
    int R8V, R16V;
    int rowsV;         // rank rows of an A_V tile in the ring (with the ones group)
    int nq, nq16;
    int Tb;
    bool ones;         // rank row R8V of each A_V tile is all ones (needs R8V <= 120)
};
__device__ __forceinline__ DtGeo dt_geo(const DtItem &it) {
    DtGeo g;
    g.nt = token_tiles(it.Tb);
    g.R8K = rank_pad(it.rK);
    g.R16K = r16_of(g.R8K);
    g.R8V = rank_pad(it.rV);
    g.R16V = r16_of(g.R8V);
    g.ones = g.R8V <= 120;
    g.rowsV = g.ones ? max(g.R8V + 8, g.R16V) : g.R8V;
    g.nq = it.nq;
    g.nq16 = (it.nq + 15) & ~15;
    g.Tb = it.Tb;
    return g;
}

// named-barrier helpers for one group of 128 threads, barrier id in a register
__device__ __forceinline__ void grp_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
__device__ __forceinline__ bool grp_and(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool grp_or(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}

// Bounded wait for the phase with this parity (limit in ns of %globaltimer);
// false (and ST_TIMEOUT raised) when the limit ran out.
__device__ __forceinline__ bool dt_wait(uint64_t *bar, uint32_t parity, uint64_t limit) {
    if (tc::mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = tc::globaltimer();
    for (;;) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if (tc::globaltimer() - t0 > limit) {
            raise_status(ST_TIMEOUT);
            return false;
        }
    }
}

// 2^x with the hardware approximation (relative error ~2^-22)
__device__ __forceinline__ float dt_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// order-preserving int encoding of a float (for atomicMax)
__device__ __forceinline__ int ord_enc(float x) {
    const int i = __float_as_int(x);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float ord_dec(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }

// Byte ring of variable-size tiles, placed contiguously (wrapping to 0 when
// a tile would cross the end) and released oldest first.  Producer side;
// one thread.
struct DtRing {
    uint32_t head = 0, seq = 0, tail = 0;
    // Offset for a tile of `bytes`: releases tiles from the tail (all older
    // than the new one) until the bytes and a barrier slot are free.  false
    // when a wait ran out.
    __device__ __forceinline__ bool place(uint32_t bytes, uint32_t size, uint32_t *offs, uint64_t *empty, int ns,
                                          uint64_t limit, uint32_t &off) {
        off = head + bytes > size ? 0u : head;
        while (tail < seq) {
            const uint32_t t0 = offs[tail % ns];   // start of the oldest live tile
            // live bytes run from t0 up to head, circularly
            const bool room = t0 < head ? (off == head || off + bytes <= t0) : (off == head && off + bytes <= t0);
            if (room && seq - tail < (uint32_t)ns) break;
            if (!dt_wait(&empty[tail % ns], (tail / ns) & 1u, limit)) return false;
            ++tail;
        }
        offs[seq % ns] = off;
        head = off + bytes;
        ++seq;
        return true;
    }
};

// bf16 pairs to fp16 pairs, in place, over n16 16-byte chunks
__device__ __forceinline__ void bf16_to_f16_inplace(uint8_t *base, int n16, int tid, int nthr) {
    uint4 *w = reinterpret_cast<uint4 *>(base);
#pragma unroll 4
    for (int e = tid; e < n16; e += nthr) {
        uint4 v = w[e];
        uint32_t *u = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[k]));
            u[k] = h2_bits(__floats2half2_rn(f.x, f.y));
        }
        w[e] = v;
    }
}

__global__ void __launch_bounds__(DT_THREADS, 1)
k_decode_tc(DecodeArgs a, const int32_t *__restrict__ pstart, const DtItem *__restrict__ items) {
    extern __shared__ __align__(1024) unsigned char dt_raw[];
    // aligned by pointer arithmetic, so that the compiler keeps the shared
    // address space (an integer round trip would turn every access generic)
    DecTcSmem &sm = *reinterpret_cast<DecTcSmem *>(dt_raw + ((1024u - (tc::smem_u32(dt_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_items = (int64_t)a.L * a.H * pstart[a.n_b];
    const uint64_t lim = a.wait_ns;

    // ---------------------------------------------------------------- set-up
    {   // zero the tile rings: pad rows of a tile hold older ring contents,
        // which must be finite (they meet zero rows of the other operand)
        uint4 *z = reinterpret_cast<uint4 *>(sm.vring);
        const int n16 = (DT_VRING + DT_AKRING + DT_BKRING) / 16;
        for (int e = threadIdx.x; e < n16; e += DT_THREADS) z[e] = make_uint4(0, 0, 0, 0);
        for (int e = threadIdx.x; e < 16 * (HALF / 2); e += DT_THREADS)
            sm.rhi[e / (HALF / 2)][e % (HALF / 2)] = a.rope_hi[e];
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < DT_NSLOT; ++s) {
            tc::mbar_init(&sm.akfull[s], 1);
            tc::mbar_init(&sm.akempty[s], 1);
            tc::mbar_init(&sm.vfull[s], 1);
            tc::mbar_init(&sm.vempty[s], 1);
        }
        for (int s = 0; s < DT_NBK; ++s) {
            tc::mbar_init(&sm.bkfull[s], 1);
            tc::mbar_init(&sm.bkempty[s], 1);
        }
        for (int s = 0; s < DT_NITAB; ++s) {
            tc::mbar_init(&sm.item_full[s], 1);
            tc::mbar_init(&sm.item_free[s], DT_ITEM_READERS);
        }
        for (int k = 0; k < 2; ++k) {
            tc::mbar_init(&sm.kh_full[k], 1);
            tc::mbar_init(&sm.kh_free[k], 1);
            tc::mbar_init(&sm.kt_full[k], DT_NEPI);
            tc::mbar_init(&sm.s_full[k], 1);
            tc::mbar_init(&sm.s_free[k], DT_NEPI);
            tc::mbar_init(&sm.p_full[k], DT_NEPI);
            tc::mbar_init(&sm.p_free[k], 1);
            tc::mbar_init(&sm.oa_full[k], 1);
            tc::mbar_init(&sm.oa_free[k], DT_NEPI);
            tc::mbar_init(&sm.o_full[k], 1);
        }
        tc::mbar_init(&sm.qt_full, DT_NEPI);
        tc::mbar_init(&sm.qt_free, 1);
        tc::mbar_init(&sm.st_full, DT_NEPI);
        tc::mbar_init(&sm.st_free, 1);
        tc::mbar_init(&sm.drain_k, 1);
        tc::mbar_init(&sm.drain_v, 1);
        sm.abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(&sm.tmem_base, DT_TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ============================================================ K producer
        const uint8_t *dataK = (const uint8_t *)a.kv[0].data;
        DtRing ak, bk;
        uint32_t claimed = 0;
        bool ok = true, done = false;
        int withheld = -1;                   // B_K copy never issued (tests only)
        // publish the item with global index c (or the end) as this CTA's item `claimed`
        auto publish = [&](int c) -> bool {
            const uint32_t e = claimed % DT_NITAB;
            if (claimed >= DT_NITAB && !dt_wait(&sm.item_free[e], ((claimed / DT_NITAB) - 1) & 1u, lim)) return false;
            if (c >= 0) sm.itab[e] = items[c];
            else sm.itab[e].l = -1;
            tc::mbar_arrive(&sm.item_full[e]);
            done = c < 0;
            ++claimed;
            return true;
        };
        auto claim = [&]() -> int {
            if (sm.abort) return -1;
            const int c = atomicAdd(a.claim, 1);
            return c < n_items ? c : -1;
        };
        uint32_t n = 0;
        if (lane == 0)
            while (ok && !done && claimed < DT_AHEAD) ok = publish(claim());
        ok = __shfl_sync(0xffffffffu, ok, 0);
        for (; ok; ++n) {
            // this item's descriptor, published by lane 0
            DtItem it;
            int stop = 1;
            if (lane == 0) {
                it = sm.itab[n % DT_NITAB];
                stop = it.l < 0 || sm.abort;
            }
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop) break;
            // the claim for a later item is in flight while this one's copies go out
            int c = -2;
            if (lane == 0 && !done) c = claim();
            int offK_lo = 0, offK_hi = 0, tbits = 0;
            if (lane == 0) {
                offK_lo = (int)(it.offK & 0xffffffff);
                offK_hi = (int)(it.offK >> 32);
                tbits = (it.rK << 16) | it.Tb;
            }
            offK_lo = __shfl_sync(0xffffffffu, offK_lo, 0);
            offK_hi = __shfl_sync(0xffffffffu, offK_hi, 0);
            tbits = __shfl_sync(0xffffffffu, tbits, 0);
            const int64_t offK = (int64_t)(((uint64_t)(uint32_t)offK_hi << 32) | (uint32_t)offK_lo);
            const int rK = tbits >> 16, Tb = tbits & 0xffff;
            const int nt = token_tiles(Tb), R8K = rank_pad(rK), R16K = r16_of(R8K);
            const uint8_t *src = dataK + 2 * offK;
            const uint32_t tile = (uint32_t)R8K * 256u;
            // B_K: R16K rows, the pad rows R8K .. R16K-1 zero
            uint32_t off = 0;
            if (lane == 0) ok = bk.place((uint32_t)R16K * 256u, DT_BKRING, sm.bk_off, sm.bkempty, DT_NBK, lim, off);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            off = __shfl_sync(0xffffffffu, off, 0);
            if (!ok) break;
            if (R16K > R8K) {
                uint4 *z = reinterpret_cast<uint4 *>(sm.bkring + off + tile);
                for (int e = lane; e < (R16K - R8K) * 16; e += 32) z[e] = make_uint4(0, 0, 0, 0);
                tc::fence_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                const uint32_t s = (bk.seq - 1) % DT_NBK;
                if (a.inject == 1 && n == 0) {
                    withheld = (int)s;       // no copy, no arrival: the K MMA's wait runs out
                } else {
                    tc::mbar_arrive_expect_tx(&sm.bkfull[s], tile);
                    if (tile) tc::bulk_g2s(sm.bkring + off, src + (size_t)nt * tile, tile, &sm.bkfull[s]);
                }
            }
            // A_K tiles (R16K rows reserved; rows past R8K meet B_K's zero rows)
            if (lane == 0) {
                for (int t = 0; t < nt && ok; ++t) {
                    ok = ak.place((uint32_t)R16K * 256u, DT_AKRING, sm.ak_off, sm.akempty, DT_NSLOT, lim, off);
                    if (!ok) break;
                    MILO_DT_TRACE(1, n, t);
                    const uint32_t s = (ak.seq - 1) % DT_NSLOT;
                    tc::mbar_arrive_expect_tx(&sm.akfull[s], tile);
                    if (tile) tc::bulk_g2s(sm.akring + off, src + (size_t)t * tile, tile, &sm.akfull[s]);
                }
                if (ok && c != -2) ok = publish(c);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (lane == 0) {
            if (!ok) sm.abort = 1;
            // an end marker after the last entry published, for the roles
            // still walking the table
            if (!done) publish(-1);
            // every copy issued has landed before the CTA exits
            for (uint32_t k = ak.seq > DT_NSLOT ? ak.seq - DT_NSLOT : 0; k < ak.seq; ++k)
                dt_wait(&sm.akfull[k % DT_NSLOT], (k / DT_NSLOT) & 1u, lim);
            for (uint32_t k = bk.seq > DT_NBK ? bk.seq - DT_NBK : 0; k < bk.seq; ++k)
                if (!(withheld >= 0 && k == 0)) dt_wait(&sm.bkfull[k % DT_NBK], (k / DT_NBK) & 1u, lim);
        }
    } else if (warp == 1) {
        // ============================================================ V producer
        const uint8_t *dataV = (const uint8_t *)a.kv[1].data;
        DtRing vr;
        bool ok = true;
        if (lane == 0) {
            for (uint32_t n = 0; ok; ++n) {
                if (!(ok = dt_wait(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u, lim))) break;
                const DtItem it = sm.itab[n % DT_NITAB];
                tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
                if (it.l < 0 || sm.abort) break;
                const DtGeo g = dt_geo(it);
                const uint8_t *src = dataV + 2 * it.offV;
                const uint32_t tile = (uint32_t)g.R8V * 256u;
                uint32_t off;
                for (int t = 0; t <= g.nt && ok; ++t) {   // A_V tiles, then B_V
                    const int rows = t < g.nt ? g.rowsV : g.R16V;
                    ok = vr.place((uint32_t)rows * 256u, DT_VRING, sm.v_off, sm.vempty, DT_NSLOT, lim, off);
                    if (!ok) break;
                    MILO_DT_TRACE(2, n, t);
                    const uint32_t s = (vr.seq - 1) % DT_NSLOT;
                    tc::mbar_arrive_expect_tx(&sm.vfull[s], tile);
                    if (tile) tc::bulk_g2s(sm.vring + off, src + (size_t)t * tile, tile, &sm.vfull[s]);
                }
            }
            if (!ok) sm.abort = 1;
            for (uint32_t k = vr.seq > DT_NSLOT ? vr.seq - DT_NSLOT : 0; k < vr.seq; ++k)
                dt_wait(&sm.vfull[k % DT_NSLOT], (k / DT_NSLOT) & 1u, lim);
        }
    } else if (warp == 2) {
        // ============================================================ K MMA
        if (lane == 0) {
            const uint32_t id_rb = tc::idesc_f16(128, 128, 1, 1, 1);   // bf16, A/B MN-major
            const uint32_t s_ak = tc::smem_u32(sm.akring), s_bk = tc::smem_u32(sm.bkring);
            const uint32_t s_q = tc::smem_u32(sm.qt);
            uint32_t g = 0, ka = 0, kb = 0;
            bool ok = true;
            // the tile whose scores are still to be issued
            bool have_prev = false;
            uint32_t pg = 0, pn = 0;
            int ptau = 0, pnt = 0, pnq16 = 16;
            auto scores = [&]() -> bool {
                const uint32_t b = pg & 1u;
                if (!dt_wait(&sm.kt_full[b], (pg >> 1) & 1u, lim)) return false;
                if (ptau == 0 && !dt_wait(&sm.qt_full, pn & 1u, lim)) return false;
                if (pg >= 2 && !dt_wait(&sm.s_free[b], ((pg - 2) >> 1) & 1u, lim)) return false;
                tc::tc_fence_after();
                MILO_DT_TRACE(4, pn, ptau);
                const uint32_t id_sc = tc::idesc_f16(128, pnq16, 0, 0, 0);   // fp16, A tmem, B K-major
                // K step ks: columns 8 ks .. 8 ks + 7 of K-tilde, core-matrix
                // columns 2 ks, 2 ks + 1 of the rotated queries
                for (int ks = 0; ks < D / 16; ++ks)
                    tc::mma_ts(tmem + DT_COL_S + 64 * b, tmem + DT_COL_KH + 128 * b + 8 * ks,
                               tc::smem_desc(s_q + ks * 256, 128, 2048, tc::LAYOUT_NONE), id_sc, ks > 0);
                tc::mma_commit(&sm.s_full[b]);
                tc::mma_commit(&sm.kh_free[b]);
                if (ptau == pnt - 1) tc::mma_commit(&sm.qt_free);
                return true;
            };
            for (uint32_t n = 0; ok; ++n) {
                if (!(ok = dt_wait(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u, lim))) break;
                const DtItem it = sm.itab[n % DT_NITAB];
                tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
                if (it.l < 0 || sm.abort) break;
                const DtGeo geo = dt_geo(it);
                for (int t = 0; t < geo.nt && ok; ++t) {
                    const uint32_t b = g & 1u;
                    ok = dt_wait(&sm.akfull[ka % DT_NSLOT], (ka / DT_NSLOT) & 1u, lim);
                    if (ok && t == 0) ok = dt_wait(&sm.bkfull[kb % DT_NBK], (kb / DT_NBK) & 1u, lim);
                    if (ok && g >= 2) ok = dt_wait(&sm.kh_free[b], ((g - 2) >> 1) & 1u, lim);
                    if (!ok) break;
                    tc::tc_fence_after();
                    MILO_DT_TRACE(3, n, t);
                    const uint32_t sa = s_ak + sm.ak_off[ka % DT_NSLOT];
                    const uint32_t sb = s_bk + sm.bk_off[kb % DT_NBK];
                    for (int ks = 0; ks < geo.R16K / 16; ++ks)
                        tc::mma_ss(tmem + DT_COL_KH + 128 * b, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                   tc::smem_desc(sb + ks * 4096, 2048, 128, tc::LAYOUT_NONE), id_rb, ks > 0);
                    tc::mma_commit(&sm.kh_full[b]);
                    tc::mma_commit(&sm.akempty[ka % DT_NSLOT]);
                    if (t == geo.nt - 1) tc::mma_commit(&sm.bkempty[kb % DT_NBK]);
                    ++ka;
                    if (t == geo.nt - 1) ++kb;
                    if (have_prev && !(ok = scores())) break;
                    have_prev = true;
                    pg = g;
                    pn = n;
                    ptau = t;
                    pnt = geo.nt;
                    pnq16 = geo.nq16;
                    ++g;
                }
            }
            if (ok && have_prev) ok = scores();
            if (!ok) sm.abort = 1;
            tc::mma_commit(&sm.drain_k);
            dt_wait(&sm.drain_k, 0, lim);
        }
    } else if (warp == 3) {
        // ============================================================ V warp: conversion + PV / O
        const uint32_t s_v = tc::smem_u32(sm.vring);
        const uint32_t s_p = tc::smem_u32(sm.pbuf[0]);
        const uint32_t s_st = tc::smem_u32(sm.stage);
        uint32_t g = 0, va = 0;
        uint32_t pc0 = 0, pc1 = 0;    // hand-overs of each P buffer consumed
        bool ok = true;
        auto wait_all = [&](uint64_t *bar, uint32_t par) -> bool {
            bool w = true;
            if (lane == 0) w = dt_wait(bar, par, lim);
            w = __shfl_sync(0xffffffffu, w, 0) != 0;
            __syncwarp();
            return w;
        };
        for (uint32_t n = 0; ok; ++n) {
            if (!(ok = wait_all(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u))) break;
            const DtItem it = sm.itab[n % DT_NITAB];
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
            if (it.l < 0 || sm.abort) break;
            const DtGeo geo = dt_geo(it);
            for (int t = 0; t <= geo.nt && ok; ++t) {
                const bool last = t == geo.nt;      // B_V
                const uint32_t slot = va % DT_NSLOT;
                if (!(ok = wait_all(&sm.vfull[slot], (va / DT_NSLOT) & 1u))) break;
                if (lane == 0) MILO_DT_TRACE(5, n, t);
                uint8_t *tp = sm.vring + sm.v_off[slot];
                bf16_to_f16_inplace(tp, geo.R8V * 16, lane, 32);
                if (!last && geo.ones) {            // rank row R8V: fp16 ones, rows R8V+1 .. +7: zero
                    uint4 *z = reinterpret_cast<uint4 *>(tp + geo.R8V * 256);
                    for (int e = lane; e < 128; e += 32) {
                        const uint32_t w = (e & 7) == 0 ? 0x3C003C00u : 0u;
                        z[e] = make_uint4(w, w, w, w);
                    }
                } else if (last && geo.R16V > geo.R8V) {   // B_V pad rows: zero
                    uint4 *z = reinterpret_cast<uint4 *>(tp + geo.R8V * 256);
                    for (int e = lane; e < (geo.R16V - geo.R8V) * 16; e += 32) z[e] = make_uint4(0, 0, 0, 0);
                }
                tc::fence_async_smem();
                __syncwarp();
                if (!last && t == 0 && n >= 2 && !(ok = wait_all(&sm.oa_free[n & 1u], ((n - 2) >> 1) & 1u))) break;
                const uint32_t pb = g & 1u;
                if (!last) {
                    if (!(ok = wait_all(&sm.p_full[pb], (pb ? pc1 : pc0) & 1u))) break;
                } else if (!(ok = wait_all(&sm.st_full, n & 1u))) {
                    break;
                }
                if (lane == 0) {
                    tc::tc_fence_after();
                    MILO_DT_TRACE(6, n, t);
                    const uint32_t sa = s_v + sm.v_off[slot];
                    const uint32_t dcol = tmem + DT_COL_OA + 64 * (n & 1u);
                    if (!last) {   // O_A^T += A_V(tile)^T P
                        const uint32_t sp = s_p + pb * DT_PBUF;
                        const uint32_t id_pv = tc::idesc_f16(128, geo.nq16, 0, 0, 1);   // fp16, A K-major, B MN-major
                        for (int ks = 0; ks < 8; ++ks)
                            tc::mma_ss(dcol, tc::smem_desc(sa + ks * 256, 128, 2048, tc::LAYOUT_NONE),
                                       tc::smem_desc(sp + ks * 2048, 1024, 128, tc::LAYOUT_NONE), id_pv, (t | ks) != 0);
                        tc::mma_commit(&sm.p_free[pb]);
                        if (t == geo.nt - 1) tc::mma_commit(&sm.oa_full[n & 1u]);
                    } else {       // O = B_V^T (O_A / l)
                        const uint32_t id_o = tc::idesc_f16(128, geo.nq16, 0, 1, 1);    // fp16, A/B MN-major
                        for (int ks = 0; ks < geo.R16V / 16; ++ks)
                            tc::mma_ss(dcol, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                       tc::smem_desc(s_st + ks * 2048, 1024, 128, tc::LAYOUT_NONE), id_o, ks > 0);
                        tc::mma_commit(&sm.st_free);
                        tc::mma_commit(&sm.o_full[n & 1u]);
                    }
                    tc::mma_commit(&sm.vempty[slot]);
                }
                __syncwarp();
                if (!last) {
                    if (pb) ++pc1;
                    else ++pc0;
                    ++g;
                }
                ++va;
            }
        }
        if (lane == 0) {
            if (!ok) sm.abort = 1;
            tc::mma_commit(&sm.drain_v);
            dt_wait(&sm.drain_v, 0, lim);
        }
    } else {
        // ============================================================ epilogue
        const int quad = warp & 3;
        const int half = (warp - DT_W_EPI) >> 2;          // RoPE pairs and query columns 32 half .. +31
        const int bar = 1 + half;                          // this group's named barrier
        const int gt = threadIdx.x - 32 * DT_W_EPI - 128 * half;   // thread within the group
        const int row = quad * 32 + lane;                  // TMEM lane: token row / rank row / channel
        const int c0 = 32 * half;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float kscale = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(d)
        // (cos, sin)(u theta_i) of this thread's lane u = t mod 32, pairs c0 + 2k, +1
        float2 cl[16], sl[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 v0 = a.rope_lo[lane * HALF + c0 + 2 * k];
            const float2 v1 = a.rope_lo[lane * HALF + c0 + 2 * k + 1];
            cl[k] = make_float2(v0.x, v1.x);
            sl[k] = make_float2(v0.y, v1.y);
        }
        bool ok = true;
        // one thread of the group waits; the group learns the outcome at the barrier
        auto gwait = [&](uint64_t *b, uint32_t par) -> bool {
            const bool w = gt == 0 ? (dt_wait(b, par, lim) && !sm.abort) : true;
            return grp_and(bar, w);
        };
        uint32_t hp0 = 0, hp1 = 0;                         // hand-overs of each P buffer
        uint32_t fp0 = 0, fp1 = 0;                         // their completions waited for
        // the last product that used P buffer b has completed
        auto p_ready = [&](uint32_t b) -> bool {
            const uint32_t h = b ? hp1 : hp0;
            uint32_t &f = b ? fp1 : fp0;
            if (f == h) return true;
            f = h;
            return gwait(&sm.p_free[b], (h - 1) & 1u);
        };

        // ---------------------------------------------------- RoPE, one tile
        uint32_t nr = 0, gr = 0;
        int tr = 0, ntr = 0;
        bool r_end = false;
        auto rope_step = [&]() -> bool {
            if (r_end) return true;
            if (tr == 0) {
                if (!gwait(&sm.item_full[nr % DT_NITAB], (nr / DT_NITAB) & 1u)) return false;
                const DtItem &e = sm.itab[nr % DT_NITAB];
                if (e.l < 0) {
                    r_end = true;
                    return true;
                }
                ntr = token_tiles(e.Tb);
            }
            const uint32_t b = gr & 1u;
            if (!gwait(&sm.kh_full[b], (gr >> 1) & 1u)) return false;
            tc::tc_fence_after();
            if (gt == 0) MILO_DT_TRACE(7 + half * 8, nr, tr);
            const uint32_t base = tmem + DT_COL_KH + 128 * b + lane_off;
            // (32 v theta) for the rows of this warp: v = (128 tr + 32 quad) / 32
            const float4 *hi = sm.rhi[4 * tr + quad] + c0 / 2;
#pragma unroll
            for (int j = 0; j < 2; ++j) {       // 16 pairs: x at columns i0 .., y at 64 + i0 ..
                const int i0 = c0 + 16 * j;
                uint32_t xr[16], yr[16];
                tc::tmem_ld16(base + i0, xr);
                tc::tmem_ld16(base + 64 + i0, yr);
                tc::tmem_wait_ld();
                uint32_t px[8], py[8];
#pragma unroll
                for (int v = 0; v < 8; ++v) {   // pairs i0 + 2v, i0 + 2v + 1
                    const int k = 8 * j + v;
                    const float4 h4 = hi[k];
                    const float2 ch = make_float2(h4.x, h4.y), shh = make_float2(h4.z, h4.w);
                    // (cos, sin)((32 v' + u) theta) = rotation by 32 v' theta after u theta
                    const float2 c = __ffma2_rn(ch, cl[k], __fmul2_rn(make_float2(-shh.x, -shh.y), sl[k]));
                    const float2 s = __ffma2_rn(shh, cl[k], __fmul2_rn(ch, sl[k]));
                    const float2 x = make_float2(__uint_as_float(xr[2 * v]), __uint_as_float(xr[2 * v + 1]));
                    const float2 y = make_float2(__uint_as_float(yr[2 * v]), __uint_as_float(yr[2 * v + 1]));
                    const float2 xo = __ffma2_rn(x, c, __fmul2_rn(make_float2(-y.x, -y.y), s));
                    const float2 yo = __ffma2_rn(y, c, __fmul2_rn(x, s));
                    px[v] = h2_bits(__floats2half2_rn(xo.x, xo.y));
                    py[v] = h2_bits(__floats2half2_rn(yo.x, yo.y));
                }
                // K steps i0/8 and i0/8 + 1: x pairs of 8 at columns i0 .. i0+3 and
                // i0+8 .. i0+11, y pairs at i0+4 .. i0+7 and i0+12 .. i0+15
                asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + i0),
                             "r"(px[0]), "r"(px[1]), "r"(px[2]), "r"(px[3]) : "memory");
                asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + i0 + 4),
                             "r"(py[0]), "r"(py[1]), "r"(py[2]), "r"(py[3]) : "memory");
                asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + i0 + 8),
                             "r"(px[4]), "r"(px[5]), "r"(px[6]), "r"(px[7]) : "memory");
                asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + i0 + 12),
                             "r"(py[4]), "r"(py[5]), "r"(py[6]), "r"(py[7]) : "memory");
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.kt_full[b]);
            if (gt == 0) MILO_DT_TRACE(8 + half * 8, nr, tr);
            ++gr;
            if (++tr == ntr) {
                tr = 0;
                ++nr;
            }
            return true;
        };

        // ------------------------------------- rotated queries of item j (this group's columns)
        // R(-p) q to fp16, K-major [q/8][cg][q%8][8]: core-matrix column 2c
        // holds channels 8c .. 8c+7 (x), 2c+1 holds 64+8c .. (y)
        auto qprep = [&](const DtItem &it, uint32_t nj) -> bool {
            if (nj >= 1 && !gwait(&sm.qt_free, (nj - 1) & 1u)) return false;
            const int nq = it.nq, nq16 = (nq + 15) & ~15;
            const int c = (gt >> 3) & 7;                  // pair chunk: pairs 8c .. 8c+7
#pragma unroll
            for (int k = 0; k < 2; ++k) {   // unrolled: both units' loads in flight together
                const int qi = c0 + (gt & 7) + 8 * (gt >> 6) + 16 * k;
                if (qi >= nq16) continue;
                uint8_t *qrow = sm.qt + (qi >> 3) * 2048 + (qi & 7) * 16;
                uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
                if (qi < nq) {
                    const int gq = it.q0 + qi;
                    const int slot = a.slot_list[it.slot0 + gq / a.G];
                    const int hq = it.h * a.G + gq % a.G;
                    const int s = slot / a.n_sel, jj = slot % a.n_sel;
                    const int64_t qbase = ((int64_t)it.l * a.S + s) * a.Hq + hq;
                    const float4 *qv = reinterpret_cast<const float4 *>(a.q + qbase * D);
                    const float4 *cs = reinterpret_cast<const float4 *>(a.rope_q + (int64_t)slot * HALF + 8 * c);
                    if (c == 0) sm.qpidx[nj & 3u][qi] = (int)(qbase * a.n_sel + jj);
                    const float4 x0 = qv[2 * c], x1 = qv[2 * c + 1], y0 = qv[16 + 2 * c], y1 = qv[16 + 2 * c + 1];
                    const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    const float y[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float4 c2 = cs[v];   // (cos, sin) of pairs 8c + 2v, 8c + 2v + 1
                        lo[v] = h2_bits(__floats2half2_rn(x[2 * v] * c2.x + y[2 * v] * c2.y,
                                                          x[2 * v + 1] * c2.z + y[2 * v + 1] * c2.w));
                        hi[v] = h2_bits(__floats2half2_rn(y[2 * v] * c2.x - x[2 * v] * c2.y,
                                                          y[2 * v + 1] * c2.z - x[2 * v + 1] * c2.w));
                    }
                }
                *reinterpret_cast<uint4 *>(qrow + (2 * c) * 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                *reinterpret_cast<uint4 *>(qrow + (2 * c + 1) * 128) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            }
            tc::fence_async_smem();
            tc::mbar_arrive(&sm.qt_full);
            return true;
        };

        // ---- no spare rank row: column sums of the rounded P by a transposing
        // butterfly; lanes 2c and 2c+1 end with column c of the 16
        auto colsum = [&](const uint32_t (&pk)[8], float *ls) {
            float sv[16];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const float2 pr = __half22float2(*reinterpret_cast<const __half2 *>(&pk[v]));
                sv[2 * v] = pr.x;
                sv[2 * v + 1] = pr.y;
            }
#pragma unroll
            for (int sz = 8, bit = 16; sz >= 1; sz >>= 1, bit >>= 1) {
                const bool up = lane & bit;
#pragma unroll
                for (int k = 0; k < sz; ++k) {
                    const float send = up ? sv[k] : sv[k + sz];
                    const float keep = up ? sv[k + sz] : sv[k];
                    sv[k] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
                }
            }
            sv[0] += __shfl_xor_sync(0xffffffffu, sv[0], 1);
            if (!(lane & 1)) atomicAdd(&ls[(lane >> 1) & 15], sv[0]);
        };

        // ---------------------------------------------------- softmax of tile g of item n
        auto softmax = [&](const DtGeo &geo, uint32_t g, uint32_t n, int t) -> bool {
            const uint32_t b = g & 1u;
            const uint32_t ib = n & 1u;
            float *cref = sm.cref[ib];
            float *lsum = sm.lsum[ib];
            const uint32_t dcol = tmem + DT_COL_S + 64 * b + lane_off;
            const int tok = t * FTILE + row;
            const bool valid = tok < geo.Tb;
            const int w = min(32, geo.nq16 - c0);      // this group's live columns (<= 0: none)
            const int lv = valid ? min(w, geo.nq - c0) : 0;
            tc::tc_fence_after();
            if (t == 0) {   // reference max: the scores of the item's first token; sums to 0
                if (gt < 32) lsum[c0 + gt] = 0.f;
                if (quad == 0 && w > 0) {
                    uint32_t r[16];
                    for (int h = 0; h < w; h += 16) {
                        tc::tmem_ld16(dcol + c0 + h, r);
                        tc::tmem_wait_ld();
                        if (lane == 0)
#pragma unroll
                            for (int v = 0; v < 16; ++v) cref[c0 + h + v] = __uint_as_float(r[v]) * kscale;
                    }
                }
                grp_sync(bar);
            }
            uint32_t pk[16];
            if (w > 0) {
                float emax = -INFINITY;
                // raw scores to p = 2^(x - cref), packed fp16 pairs: pk[v] <- columns 2v, 2v+1
                auto make_p = [&]() {
                    const float2 *cr = reinterpret_cast<const float2 *>(cref + c0);
                    const float2 ks2 = make_float2(kscale, kscale);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {   // 16 columns at a time
                        if (16 * h >= w) break;
                        uint32_t r[16];
                        tc::tmem_ld16(dcol + c0 + 16 * h, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            const int k = 8 * h + v;
                            const float2 crv = cr[k];
                            const float2 e = __ffma2_rn(make_float2(__uint_as_float(r[2 * v]), __uint_as_float(r[2 * v + 1])),
                                                        ks2, make_float2(-crv.x, -crv.y));
                            const float e0 = 2 * k < lv ? e.x : -INFINITY;
                            const float e1 = 2 * k + 1 < lv ? e.y : -INFINITY;
                            emax = fmaxf(emax, fmaxf(e0, e1));
                            pk[k] = h2_bits(__floats2half2_rn(dt_ex2(e0), dt_ex2(e1)));
                        }
                    }
                };
                make_p();
                // more than 2^8 (or not finite) sends the tile down the rare path
                if (grp_or(bar, !(emax <= DT_OVER))) {
                    // every P of this item handed over has been used
                    if (!p_ready(0) || !p_ready(1)) return false;
                    if (gt < w) sm.cmax[c0 + gt] = ord_enc(-INFINITY);
                    grp_sync(bar);
                    for (int h = 0; h < w; h += 16) {   // column maxima over the tile's live rows
                        uint32_t r[16];
                        tc::tmem_ld16(dcol + c0 + h, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int v = 0; v < 16; ++v) {
                            float x = h + v < lv ? __uint_as_float(r[v]) * kscale : -INFINITY;
                            for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                            if (lane == 0) atomicMax(&sm.cmax[c0 + h + v], ord_enc(x));
                        }
                    }
                    grp_sync(bar);
                    if (gt < w) {
                        const int c = c0 + gt;
                        const float cn = fmaxf(cref[c], ord_dec(sm.cmax[c]));
                        const float f = dt_ex2(cref[c] - cn);
                        sm.cscale[ib][c] = f;
                        cref[c] = cn;
                        lsum[c] *= f;
                    }
                    grp_sync(bar);
                    if (t > 0) {   // O_A^T columns (every rank lane) times 2^(cref_old - cref_new)
                        tc::tc_fence_after();
                        const uint32_t ocol = tmem + DT_COL_OA + 64 * ib + lane_off;
                        for (int h = 0; h < w; h += 16) {
                            uint32_t o[16];
                            tc::tmem_ld16(ocol + c0 + h, o);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                uint32_t wv[8];
#pragma unroll
                                for (int v = 0; v < 8; ++v)
                                    wv[v] = __float_as_uint(__uint_as_float(o[8 * hh + v]) *
                                                            sm.cscale[ib][c0 + h + 8 * hh + v]);
                                tc::tmem_st8(ocol + c0 + h + 8 * hh, wv);
                            }
                        }
                        tc::tmem_wait_st();
                        tc::tc_fence_before();
                    }
                    grp_sync(bar);
                    make_p();
                }
            }
            if (!p_ready(b)) return false;   // the P buffer's previous product has completed
            if (w > 0) {
                uint8_t *dst = sm.pbuf[b] + (row >> 3) * 1024 + (row & 7) * 16 + (c0 >> 3) * 128;
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                    if (8 * hh >= w) break;
                    *reinterpret_cast<uint4 *>(dst + hh * 128) =
                        make_uint4(pk[4 * hh], pk[4 * hh + 1], pk[4 * hh + 2], pk[4 * hh + 3]);
                }
                if (!geo.ones) {
                    colsum(*reinterpret_cast<const uint32_t(*)[8]>(&pk[0]), lsum + c0);
                    if (w == 32) colsum(*reinterpret_cast<const uint32_t(*)[8]>(&pk[8]), lsum + c0 + 16);
                }
            }
            // every score of the tile this thread needed has been read
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.s_free[b]);
            tc::fence_async_smem();
            tc::mbar_arrive(&sm.p_full[b]);
            if (b) ++hp1;
            else ++hp0;
            if (gt == 0) MILO_DT_TRACE(11 + half * 8, n, t);
            return true;
        };

        // ---- item m's O_A^T is complete: denominators, partial (max, sum), and
        // O_A / l (fp16, this group's columns) staged for the last product
        auto finalize = [&](const DtGeo &geo, uint32_t m) -> bool {
            if (!gwait(&sm.oa_full[m & 1u], (m >> 1) & 1u)) return false;
            if (gt == 0) MILO_DT_TRACE(12 + half * 8, m, 0);
            tc::tc_fence_after();
            const uint32_t ib = m & 1u;
            const int w = min(32, geo.nq16 - c0);
            const uint32_t ocol = tmem + DT_COL_OA + 64 * ib + lane_off;
            if (w > 0 && geo.ones && quad == (geo.R8V >> 5)) {   // the ones row holds sum_t p
                for (int h = 0; h < w; h += 16) {
                    uint32_t r[16];
                    tc::tmem_ld16(ocol + c0 + h, r);
                    tc::tmem_wait_ld();
                    if (row == geo.R8V)
#pragma unroll
                        for (int v = 0; v < 16; ++v) sm.lsum[ib][c0 + h + v] = __uint_as_float(r[v]);
                }
            }
            grp_sync(bar);
            if (gt < 32) {
                const int c = c0 + gt;
                const float l = sm.lsum[ib][c];
                sm.cscale[ib][c] = (c < geo.nq && l > 0.f) ? __frcp_rn(l) : 0.f;
                if (c < geo.nq) a.part_ml[sm.qpidx[m & 3u][c]] = make_float2(sm.cref[ib][c] * 0.69314718055994531f, l);
            }
            grp_sync(bar);   // every 1 / l of the group written before the staging reads them
            // the stage buffer's previous product (item m-1's O) has completed
            if (m >= 1 && !gwait(&sm.st_free, (m - 1) & 1u)) return false;
            if (w > 0 && quad * 32 < geo.R16V) {   // whole warps: tcgen05.ld is warp-collective
                uint8_t *dst = sm.stage + (row >> 3) * 1024 + (row & 7) * 16;
                for (int ch = c0; ch < c0 + w; ch += 16) {
                    uint32_t r[16];
                    tc::tmem_ld16(ocol + ch, r);
                    tc::tmem_wait_ld();
                    if (row < geo.R16V) {
                        uint32_t q8[8];
                        const bool live = row < geo.R8V;   // pad rows meet B_V's zero rows
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            q8[v] = live ? h2_bits(__floats2half2_rn(
                                               __uint_as_float(r[2 * v]) * sm.cscale[ib][ch + 2 * v],
                                               __uint_as_float(r[2 * v + 1]) * sm.cscale[ib][ch + 2 * v + 1]))
                                         : 0u;
                        *reinterpret_cast<uint4 *>(dst + (ch >> 3) * 128) = make_uint4(q8[0], q8[1], q8[2], q8[3]);
                        *reinterpret_cast<uint4 *>(dst + (ch >> 3) * 128 + 128) =
                            make_uint4(q8[4], q8[5], q8[6], q8[7]);
                    }
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.st_full);
            if (gt == 0) MILO_DT_TRACE(13 + half * 8, m, 0);
            return true;
        };

        // ---- item m's O = B_V^T (O_A / l) (lanes = channels, columns = queries)
        // to the fp16 partials; frees the item's O_A^T buffer
        auto readout = [&](int nq, uint32_t m) -> bool {
            if (!gwait(&sm.o_full[m & 1u], (m >> 1) & 1u)) return false;
            tc::tc_fence_after();
            if (gt == 0) MILO_DT_TRACE(14 + half * 8, m, 0);
            const int *qp = sm.qpidx[m & 3u];
            if (c0 < nq) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + DT_COL_OA + 64 * (m & 1u) + lane_off + c0, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int v = 0; v < 32; ++v)
                    if (c0 + v < nq) a.part_o16[(int64_t)qp[c0 + v] * D + row] = __float2half_rn(__uint_as_float(r[v]));
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.oa_free[m & 1u]);
            return true;
        };

        // ---------------------------------------------------- the item loop
        // per tile: RoPE one tile ahead, then this tile's softmax; the next
        // item's queries at the start of an item's last tile, the previous
        // item's denominators / staging after this item's first tile and its
        // read-out after the second.
        if (!(ok = gwait(&sm.item_full[0], 0))) {
            sm.abort = 1;
        } else {
            DtItem cur = sm.itab[0];
            DtGeo gprev = dt_geo(cur);
            uint32_t n = 0, g = 0;
            if (cur.l >= 0) ok = qprep(cur, 0) && rope_step();
            for (; ok && cur.l >= 0; ++n) {
                const DtGeo geo = dt_geo(cur);
                DtItem nxt;
                nxt.l = -1;
                for (int t = 0; t < geo.nt && ok; ++t, ++g) {
                    if (!(ok = rope_step())) break;
                    if (!(ok = gwait(&sm.s_full[g & 1u], (g >> 1) & 1u))) break;
                    if (gt == 0) MILO_DT_TRACE(9 + half * 8, n, t);
                    if (t == geo.nt - 1) {   // the query buffer is free once this tile's scores ran
                        if (!(ok = gwait(&sm.item_full[(n + 1) % DT_NITAB], ((n + 1) / DT_NITAB) & 1u))) break;
                        nxt = sm.itab[(n + 1) % DT_NITAB];
                        if (nxt.l >= 0 && !(ok = qprep(nxt, n + 1))) break;
                        if (gt == 0) MILO_DT_TRACE(10 + half * 8, n, t);
                    }
                    if (!(ok = softmax(geo, g, n, t))) break;
                    if (t == 0 && n >= 1 && !(ok = finalize(gprev, n - 1))) break;
                    if (t == min(1, geo.nt - 1) && n >= 1) {
                        if (!(ok = readout(gprev.nq, n - 1))) break;
                        if (lane == 0) tc::mbar_arrive(&sm.item_free[(n - 1) % DT_NITAB]);
                    }
                }
                if (!ok) break;
                gprev = geo;
                cur = nxt;
            }
            // the last item's denominators, staging and read-out
            if (ok && n >= 1) ok = finalize(gprev, n - 1) && readout(gprev.nq, n - 1);
            if (!ok) sm.abort = 1;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 2) tc::tmem_dealloc(tmem, DT_TMEM_COLS);
}

inline size_t decode_tc_smem_bytes() { return sizeof(DecTcSmem) + 1024; }
static_assert(sizeof(DecTcSmem) + 1024 <= 232448, "decode shared memory over the per-CTA limit");

inline bool decode_tc_supported(const DecodeArgs &a) {
    if (getenv("MILO_FORCE_SIMT")) return false;
    return a.factor_dtype == MILO_BF16 && a.block_len <= 512;
}

inline cudaError_t decode_tc_set_attrs() {
    return cudaFuncSetAttribute(k_decode_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_tc_smem_bytes());
}

// upper bound of the number of items: sum_b ceil(q_b / 64) <= n_b + S n_sel G / 64 per (l, h)
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
