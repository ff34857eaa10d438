// decode_tc.cuh -- decode attention over retrieved compressed blocks on
// tcgen05 tensor cores (bf16 factors, or INT8 factors dequantised to fp16 by
// k_dequant_selected).
//
// Step "at inference a retriever selects blocks, whose low-rank factors are
// rebuilt before sparse attention" (evolve.pub review of MILO, Summary; FAQ
// "What is MILO").  Prep kernels group, for every block id, the sessions that
// selected it by start position p into work items (layer, KV head, block, p,
// up to 8 sessions of G8 query heads, 64 queries at most) and pack the
// queries to fp16 in the tensor cores' operand layout.  Every query of an
// item sees the block at the same position, so the keys are rotated by the
// full angle (p + t) theta_i and the queries are used as they are:
// q . R(p + t) k_t.  One persistent CTA per SM claims items dynamically and
// streams them through warp roles that meet only at mbarriers, every wait
// bounded:
//
//   K producer (warp 0)   claims items into a shared-memory table; per item
//                         one entry of a resident ring holds its sessions'
//                         packed queries (16-byte asynchronous copies by the
//                         warp's lanes) and B_K (one bulk copy); the 128-token
//                         A_K tiles are bulk-copied into a tile ring (factors
//                         already in the canonical operand layout).
//   V producer (warp 1)   bulk-copies the A_V tiles and B_V into a third ring.
//   K MMA (warp 2)        rebuild  K-hat tile = A_K(tile) B_K        (M=128 tokens, N=128, K=r_K, bf16)
//                         scores   S = K-tilde (TMEM) Q^T             (M=128 tokens, N=nq, K=128, fp16)
//                         in the order R0 R1 S0 R2 S1 ...
//   V warp (warp 3)       issues O_A^T += A_V(tile)^T P, then
//                         O = B_V^T (O_A / l)                        (M=128, N=nq, fp16)
//   RoPE group (8 warps)  two per TMEM lane quadrant, a token row per thread,
//                         32 pairs each: rotates the rebuilt keys by
//                         (p + 32 v + u) theta_i, u = the thread's lane, with
//                         (cos, sin)(u theta_i) in registers and (p + 32 v)
//                         theta_i from a per-slot table (L2-resident), f32x2
//                         arithmetic; packs K-tilde to fp16 in place.
//                         Then converts the same tile of A_V (and, last, B_V)
//                         to fp16 in place, appending a row of ones to A_V
//                         when a rank row is free.  Also reads each item's O
//                         out (fp16, query-major in shared memory, then one
//                         bulk store of the item's rows of partials).
//   softmax group (8 w.)  two column halves of four warps, a token row per
//                         thread: exp2 against a per-query reference max
//                         raised only when some p exceeds 2^8, P (fp16) to
//                         shared memory; after the next item's first tile, the
//                         previous item's denominators and O_A / l, staged in
//                         the P buffer its last tile used.
//
// RoPE and softmax run in different warps on different tiles (two rebuild
// and two score buffers in tensor memory), so their latencies overlap.  The
// ones row makes the PV product return the softmax denominators as one more
// row of O_A^T.  Keys and values are never written to memory.  Each (query,
// selected slot) gets a partial (max, sum, normalised output in fp16)
// merged by k_combine.
#pragma once
#include "decode_simt.cuh"
#include "tc_common.cuh"

// Timeline hook: empty unless a tracing build defines it (event code, item,
// tile).
#ifndef MILO_DT_TRACE
#define MILO_DT_TRACE(code, n, t)
#endif
#ifndef MILO_DT_TRACE_STATE
#define MILO_DT_TRACE_STATE
#endif
// Copy-latency hooks (tracing builds): issue time of a ring slot's copy, and
// its landing as the consumer sees it.
#ifndef MILO_DT_STAMP
#define MILO_DT_STAMP(kind, slot)
#define MILO_DT_LAT(kind, slot)
#endif
// Debug hooks (tracing builds): the shared-memory base, and a wait that ran out.
#ifndef MILO_DT_ON_TIMEOUT
#define MILO_DT_BASE(p)
#define MILO_DT_ON_TIMEOUT(bar, parity)
#endif

namespace milo {

constexpr int DT_NQ = 64;                         // queries per item
constexpr int DT_MAXS = 8;                        // sessions per item
constexpr int DT_THREADS = 640;                   // 20 warps = 5 warpgroups
constexpr int DT_W_ROPE = 4;                      // RoPE warps 4 .. 11
constexpr int DT_W_SM = 12;                       // softmax warps 12 .. 19
constexpr int DT_NROPE = 256, DT_NSM = 256;
// registers per thread: at launch (65536 / 640, in steps of 8) and per
// warpgroup after setmaxnreg; the shares add up to the launch total
constexpr int DT_REG_LAUNCH = 96, DT_REG_CTRL = 48, DT_REG_ROPE = 128, DT_REG_SM = 88;
static_assert(DT_REG_CTRL + 2 * DT_REG_ROPE + 2 * DT_REG_SM <= 5 * DT_REG_LAUNCH, "register split over the launch");
constexpr int DT_VRING = 64 * 1024;               // A_V tiles (+ ones group) and B_V
constexpr int DT_AKRING = 48 * 1024;              // A_K tiles
constexpr int DT_RRING = 56 * 1024;               // per item: packed queries, then B_K (48 KB at most)
constexpr int DT_NSLOT = 16;                      // tiles in flight per tile ring
constexpr int DT_NRES = 4;                        // items in flight in the resident ring
constexpr int DT_NITAB = 16;                      // item table entries
constexpr int DT_AHEAD = 4;                       // items claimed ahead of the copies
constexpr int DT_PBUF = 128 * DT_NQ * 2;          // one P buffer: 128 tokens x 64 queries, fp16
constexpr uint32_t DT_TMEM_COLS = 512;
constexpr uint32_t DT_COL_KH = 0;                 // two 128-column rebuild buffers
constexpr uint32_t DT_COL_S = 256;                // two 64-column score buffers
constexpr uint32_t DT_COL_OA = 384;               // two 64-column O_A^T / O buffers
constexpr float DT_OVER = 8.f;                    // log2 headroom before the reference max moves
constexpr int DT_BAR_ROPE = 1;                    // named barrier of the RoPE group (256 threads)
constexpr int DT_BAR_SM = 2;                      // named barriers of the softmax halves (128 threads): 2, 3

// One work item, written by k_dt_items.  l < 0 marks the end of a CTA's items
// in its table.
struct DtItem {
    int32_t l, h, b, pos;   // layer, KV head, block id, start position of the block for every session
    int32_t ns, Tb, rK, rV; // sessions, tokens, ranks
    int64_t offK, offV;     // element offsets of the block in the data sections
    int32_t slots[DT_MAXS]; // the sessions' slots (s * n_sel + j); -1 past ns
    int32_t row0, pad;      // first row of the item's partial outputs (ns x G8 rows of D)
};

struct DecTcSmem {
    // The V ring comes first: the PV product reads 128 rank rows from an A_V
    // tile's start, past a short tile, and those reads must stay inside the
    // CTA's shared memory (the rows they feed are never used).
    alignas(1024) uint8_t vring[DT_VRING];
    alignas(1024) uint8_t akring[DT_AKRING];
    alignas(1024) uint8_t rring[DT_RRING];
    alignas(1024) uint8_t pbuf[2][DT_PBUF];       // P, or O_A / l for an item's last product (fp16, MN-major)
    alignas(1024) uint8_t ostage[DT_NQ * D * 2];  // an item's O, fp16, query-major, for its bulk store
    // 8 rank rows of zeros in the B_K operand layout: the second half of the
    // last K step when the padded rank is an odd multiple of 8, or both
    // halves (leading offset 0) for a block of rank 0
    alignas(1024) uint8_t zero[2048];
    DtItem itab[DT_NITAB];                        // claimed items, entry n % NITAB = this CTA's n-th
    float cref[2][DT_NQ];                         // reference max per query (log2 domain), per item parity
    float cscale[2][DT_NQ];                       // rescale factors, then 1 / l
    float lsum[2][DT_NQ];
    int cmax[DT_NQ];                              // column maxima, order-preserving int encoding
    int qp_sm[4][DT_NQ];                          // partial index of each query column (-1: none), per item
    uint32_t ak_off[DT_NSLOT], v_off[DT_NSLOT], res_off[DT_NRES];
    uint64_t item_full[DT_NITAB], item_free[DT_NITAB];
    uint64_t akfull[DT_NSLOT], akempty[DT_NSLOT];
    uint64_t vfull[DT_NSLOT], vconv[DT_NSLOT], vempty[DT_NSLOT];
    uint64_t res_full[DT_NRES], res_empty[DT_NRES];
    uint64_t kh_full[2], kh_free[2], kt_full[2];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], p_free[2];
    uint64_t oa_full[2], oa_free[2], o_full[2];
    uint64_t drain_k, drain_v;
    uint32_t tmem_base;
    volatile int abort;
};

// readers that free an item table entry: V producer, K MMA, V warp, 8 RoPE and 8 softmax warps
constexpr int DT_ITEM_READERS = 1 + 1 + 1 + 8 + 8;

// Partial index of query column c of an item (-1: a padding column).
__device__ __forceinline__ int dt_pidx(const DecodeArgs &a, const DtItem &it, int c) {
    const int k = c / a.G8, g = c % a.G8;
    if (k >= it.ns || g >= a.G) return -1;
    const int slot = it.slots[k];
    return (int)((((int64_t)it.l * a.S + slot / a.n_sel) * a.Hq + it.h * a.G + g) * a.n_sel + slot % a.n_sel);
}

// Items of every (layer, head, block): the block's slot list (sorted by
// (position, slot) by k_blk_items) cut into runs of equal position of at
// most spi sessions.  Grid over l*h*n_b; istart = exclusive scan of the
// per-block item counts, istart[n_b] = items per (l, h).
__global__ void k_dt_items(DecodeArgs a, const int32_t *__restrict__ istart, DtItem *__restrict__ items) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)a.L * a.H * a.n_b) return;
    const int b = (int)(e % a.n_b);
    const int64_t lh = e / a.n_b;
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
    int64_t out = lh * istart[a.n_b] + istart[b];
    const int s1 = a.slot_start[b + 1];
    const int64_t nslots = (int64_t)a.S * a.n_sel;
    it.pad = 0;
    for (int i = a.slot_start[b]; i < s1;) {
        const int p = slot_pos(a.sel, a.pos, a.slot_list[i], a.block_len);
        it.pos = p;
        it.ns = 0;
        // the item's rows of partials: G8 per session, in the block's slot-list order
        it.row0 = (int32_t)((lh * nslots + i) * a.G8);
        while (i < s1 && it.ns < a.spi && slot_pos(a.sel, a.pos, a.slot_list[i], a.block_len) == p)
            it.slots[it.ns++] = a.slot_list[i++];
        for (int k = it.ns; k < DT_MAXS; ++k) it.slots[k] = -1;
        for (int k = 0; k < it.ns; ++k)
            for (int g = 0; g < a.G; ++g) a.pmap[dt_pidx(a, it, k * a.G8 + g)] = it.row0 + k * a.G8 + g;
        items[out++] = it;
    }
}

// Per selected slot, (cos, sin)((p + 32 v) theta_i) for v < 16, the angle of
// the first token of each 32-token group of the block at start position p,
// by angle addition from (p theta_i) and (32 v theta_i); pairs (2k, 2k+1) as
// (c0, c1, s0, s1).  16 x 32 float4 (8 KB) per slot.
__global__ void k_rot_slots(const float2 *__restrict__ rope_q, const float4 *__restrict__ rope_hi, int n_slots,
                            float4 *__restrict__ rot) {
    const int64_t total = (int64_t)n_slots * 16 * (HALF / 2);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int k = (int)(e % (HALF / 2));
        const int v = (int)((e / (HALF / 2)) % 16);
        const int64_t slot = e / (16 * (HALF / 2));
        const float4 p = reinterpret_cast<const float4 *>(rope_q + slot * HALF)[k];   // (c0, s0, c1, s1) of p theta
        const float4 h = rope_hi[v * (HALF / 2) + k];                                   // (c0, c1, s0, s1) of 32 v theta
        const float c0 = fmaf(p.x, h.x, -p.y * h.z), s0 = fmaf(p.y, h.x, p.x * h.z);
        const float c1 = fmaf(p.z, h.y, -p.w * h.w), s1 = fmaf(p.w, h.y, p.z * h.w);
        rot[e] = make_float4(c0, c1, s0, s1);
    }
}

__host__ __device__ __forceinline__ int r16_of(int R8) { return R8 <= 16 ? 16 : (R8 + 15) & ~15; }

// Geometry of one item as the roles see it.
struct DtGeo {
    int nt;            // 128-token tiles
    int R8K, R16K;     // key rank padded to 8 / to the MMA's K step
    int R8V, R16V;
    int rowsV;         // rank rows of an A_V tile in the ring (with the ones group)
    int nq, nq16;      // query columns (sessions x G8), padded to 16
    int Tb;
    bool ones;         // rank row R8V of each A_V tile is all ones (needs R8V <= 120)
};
__device__ __forceinline__ DtGeo dt_geo(const DtItem &it, int G8) {
    DtGeo g;
    g.nt = token_tiles(it.Tb);
    g.R8K = rank_pad(it.rK);
    g.R16K = r16_of(g.R8K);
    g.R8V = rank_pad(it.rV);
    g.R16V = r16_of(g.R8V);
    g.ones = g.R8V <= 120;
    g.rowsV = g.ones ? max(g.R8V + 8, g.R16V) : g.R8V;
    g.nq = it.ns * G8;
    g.nq16 = (g.nq + 15) & ~15;
    g.Tb = it.Tb;
    return g;
}


// named barriers, id and thread count in registers
__device__ __forceinline__ void grp_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ bool grp_and(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool grp_or(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

template <int N> __device__ __forceinline__ void reg_alloc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N> __device__ __forceinline__ void reg_dealloc() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Bounded wait for the phase with this parity (limit in ns of %globaltimer);
// false (and ST_TIMEOUT raised) when the limit ran out.
__device__ __forceinline__ bool dt_wait(uint64_t *bar, uint32_t parity, uint64_t limit) {
    if (tc::mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = tc::globaltimer();
    for (;;) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if (tc::globaltimer() - t0 > limit) {
            MILO_DT_ON_TIMEOUT(bar, parity);
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
k_decode_tc(DecodeArgs a, const int32_t *__restrict__ istart, const DtItem *__restrict__ items) {
    extern __shared__ __align__(1024) unsigned char dt_raw[];
    // aligned by pointer arithmetic, so that the compiler keeps the shared
    // address space (an integer round trip would turn every access generic)
    DecTcSmem &sm = *reinterpret_cast<DecTcSmem *>(dt_raw + ((1024u - (tc::smem_u32(dt_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = a.wait_ns;
    const int G8 = a.G8;
    if (threadIdx.x == 0) MILO_DT_BASE(&sm);

    // ---------------------------------------------------------------- set-up
    {   // zero the rings (pad rows of a tile hold older ring contents, which
        // must be finite: they meet zero rows of the other operand) and the
        // zero rows
        uint4 *z = reinterpret_cast<uint4 *>(sm.vring);
        const int n16 = (DT_VRING + DT_AKRING + DT_RRING) / 16;
        for (int e = threadIdx.x; e < n16; e += DT_THREADS) z[e] = make_uint4(0, 0, 0, 0);
        for (int e = threadIdx.x; e < 2048 / 16; e += DT_THREADS) reinterpret_cast<uint4 *>(sm.zero)[e] = make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < DT_NSLOT; ++s) {
            tc::mbar_init(&sm.akfull[s], 1);
            tc::mbar_init(&sm.akempty[s], 1);
            tc::mbar_init(&sm.vfull[s], 1);
            tc::mbar_init(&sm.vconv[s], DT_NROPE);
            tc::mbar_init(&sm.vempty[s], 1);
        }
        for (int s = 0; s < DT_NRES; ++s) {
            tc::mbar_init(&sm.res_full[s], 32 + 1);   // the K producer's lanes' query copies, B_K's bulk copy
            tc::mbar_init(&sm.res_empty[s], 1);
        }
        for (int s = 0; s < DT_NITAB; ++s) {
            tc::mbar_init(&sm.item_full[s], 1);
            tc::mbar_init(&sm.item_free[s], DT_ITEM_READERS);
        }
        for (int k = 0; k < 2; ++k) {
            tc::mbar_init(&sm.kh_full[k], 1);
            tc::mbar_init(&sm.kh_free[k], 1);
            tc::mbar_init(&sm.kt_full[k], DT_NROPE);
            tc::mbar_init(&sm.s_full[k], 1);
            tc::mbar_init(&sm.s_free[k], DT_NSM);
            tc::mbar_init(&sm.p_full[k], DT_NSM);
            tc::mbar_init(&sm.p_free[k], 1);
            tc::mbar_init(&sm.oa_full[k], 1);
            tc::mbar_init(&sm.oa_free[k], DT_NROPE);
            tc::mbar_init(&sm.o_full[k], 1);
        }
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

    if (warp < DT_W_ROPE) {
        reg_dealloc<DT_REG_CTRL>();
        if (warp == 0) {
            // ======================================================== K producer
            MILO_DT_TRACE_STATE;
            const int64_t n_items = (int64_t)a.L * a.H * istart[a.n_b];
            DtRing ak, rr;
            uint32_t claimed = 0;
            bool ok = true, done = false;
            bool withheld = false;               // first B_K copy never issued (tests only)
            // publish the item with global index c (or the end) as this CTA's item `claimed`
            auto publish = [&](int c) -> bool {
                const uint32_t e = claimed % DT_NITAB;
                if (claimed >= DT_NITAB && !dt_wait(&sm.item_free[e], ((claimed / DT_NITAB) - 1) & 1u, lim))
                    return false;
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
            if (lane == 0)
                while (ok && !done && claimed < DT_AHEAD) ok = publish(claim());
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();
            for (uint32_t n = 0; ok; ++n) {
                // entries are rewritten only by this warp, so the table is read in place
                const DtItem &it = sm.itab[n % DT_NITAB];
                if (__shfl_sync(0xffffffffu, (int)(it.l < 0 || sm.abort), 0)) break;   // lane 0 decides
                // the claim for a later item is in flight while this one's copies go out
                int c = -2;
                if (lane == 0 && !done) c = claim();
                if (lane == 0) MILO_DT_TRACE(28, n, 0);
                const int R8K = rank_pad(it.rK);
                const uint32_t tile = (uint32_t)R8K * 256u;
                // resident entry: the queries (nq16 rows; rows past ns * G8 are
                // not copied: their score columns are masked), then B_K
                const uint32_t qbytes = (uint32_t)((it.ns * G8 + 15) & ~15) * 256u;
                uint32_t off = 0, rs = 0;
                if (lane == 0) {
                    ok = rr.place(qbytes + tile, DT_RRING, sm.res_off, sm.res_empty, DT_NRES, lim, off);
                    rs = (rr.seq - 1) % DT_NRES;
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                off = __shfl_sync(0xffffffffu, off, 0);
                rs = __shfl_sync(0xffffffffu, rs, 0);
                if (!ok) break;
                if (lane == 0) MILO_DT_TRACE(29, n, 0);
                // each session's G8 packed query rows (G8 x 256 bytes, contiguous in
                // the packed queries and in the entry), 16 bytes per lane and copy
                for (int k = 0; k < it.ns; ++k) {
                    const int slot = it.slots[k];
                    const int64_t lsh = ((int64_t)it.l * a.S + slot / a.n_sel) * a.H + it.h;
                    const __half *src = a.qpack + lsh * G8 * D;
                    uint8_t *dst = sm.rring + off + k * G8 * 256;
                    for (int w = lane; w < G8 * 16; w += 32) tc::cp_async16(dst + w * 16, src + w * 8);
                }
                tc::cp_async_arrive_noinc(&sm.res_full[rs]);
                __syncwarp();
                if (lane == 0) {
                    const uint8_t *src = (const uint8_t *)a.kv[0].data + 2 * it.offK;
                    const int nt = token_tiles(it.Tb);
                    if (a.inject == 1 && n == 0) {
                        withheld = true;         // no copy, no arrival: the K MMA's wait runs out
                    } else {
                        tc::mbar_arrive_expect_tx(&sm.res_full[rs], tile);
                        if (tile) tc::bulk_g2s(sm.rring + off + qbytes, src + (size_t)nt * tile, tile, &sm.res_full[rs]);
                    }
                    // A_K tiles (R16K rows reserved; rows past R8K meet B_K's zero rows)
                    const uint32_t rows16 = (uint32_t)r16_of(R8K);
                    for (int t = 0; t < nt && ok; ++t) {
                        ok = ak.place(rows16 * 256u, DT_AKRING, sm.ak_off, sm.akempty, DT_NSLOT, lim, off);
                        if (!ok) break;
                        MILO_DT_TRACE(1, n, t);
                        const uint32_t sl = (ak.seq - 1) % DT_NSLOT;
                        tc::mbar_arrive_expect_tx(&sm.akfull[sl], tile);
                        if (tile) tc::bulk_g2s(sm.akring + off, src + (size_t)t * tile, tile, &sm.akfull[sl]);
                        MILO_DT_STAMP(0, sl);
                    }
                    if (ok && c != -2) ok = publish(c);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                __syncwarp();
            }
            // every query copy of this warp has landed before the CTA exits
            tc::cp_async_wait_all();
            if (lane == 0) {
                if (!ok) sm.abort = 1;
                // an end marker after the last entry published, for the roles
                // still walking the table
                if (!done) publish(-1);
                // every bulk copy issued has landed before the CTA exits
                for (uint32_t k = ak.seq > DT_NSLOT ? ak.seq - DT_NSLOT : 0; k < ak.seq; ++k)
                    dt_wait(&sm.akfull[k % DT_NSLOT], (k / DT_NSLOT) & 1u, lim);
                for (uint32_t k = rr.seq > DT_NRES ? rr.seq - DT_NRES : 0; k < rr.seq; ++k)
                    if (!(withheld && k == 0)) dt_wait(&sm.res_full[k % DT_NRES], (k / DT_NRES) & 1u, lim);
            }
        } else if (warp == 1) {
            // ======================================================== V producer
            MILO_DT_TRACE_STATE;
            DtRing vr;
            bool ok = true;
            if (lane == 0) {
                for (uint32_t n = 0; ok; ++n) {
                    if (!(ok = dt_wait(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u, lim))) break;
                    const DtItem &e = sm.itab[n % DT_NITAB];
                    const bool live = e.l >= 0;
                    const DtGeo g = dt_geo(e, G8);
                    const uint8_t *src = (const uint8_t *)a.kv[1].data + 2 * e.offV;
                    tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
                    if (!live || sm.abort) break;
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
                        MILO_DT_STAMP(1, s);
                    }
                }
                if (!ok) sm.abort = 1;
                for (uint32_t k = vr.seq > DT_NSLOT ? vr.seq - DT_NSLOT : 0; k < vr.seq; ++k)
                    dt_wait(&sm.vfull[k % DT_NSLOT], (k / DT_NSLOT) & 1u, lim);
            }
        } else if (warp == 2) {
            // ======================================================== K MMA
            MILO_DT_TRACE_STATE;
            if (lane == 0) {
                const uint32_t id_rb = tc::idesc_f16(128, 128, a.f16 ? 0 : 1, 1, 1);   // bf16 (or fp16), A/B MN-major
                const uint32_t s_ak = tc::smem_u32(sm.akring), s_rr = tc::smem_u32(sm.rring);
                const uint32_t s_zero = tc::smem_u32(sm.zero);
                uint32_t g = 0, ka = 0, kr = 0;
                bool ok = true;
                // the tile whose scores are still to be issued: its buffer, the
                // queries of its item and the item's resident entry
                bool have_prev = false;
                uint32_t pg = 0, pq = 0, prs = 0;
                int plast = 0, pnq16 = 16;
                auto scores = [&]() -> bool {
                    const uint32_t b = pg & 1u;
                    if (!dt_wait(&sm.kt_full[b], (pg >> 1) & 1u, lim)) return false;
                    if (pg >= 2 && !dt_wait(&sm.s_free[b], ((pg - 2) >> 1) & 1u, lim)) return false;
                    tc::tc_fence_after();
                    MILO_DT_TRACE(4, 0, 0);
                    const uint32_t id_sc = tc::idesc_f16(128, pnq16, 0, 0, 0);   // fp16, A tmem, B K-major
                    // K step ks: columns 8 ks .. 8 ks + 7 of K-tilde, core-matrix
                    // columns 2 ks, 2 ks + 1 of the packed queries
                    for (int ks = 0; ks < D / 16; ++ks)
                        tc::mma_ts(tmem + DT_COL_S + 64 * b, tmem + DT_COL_KH + 128 * b + 8 * ks,
                                   tc::smem_desc(pq + ks * 256, 128, 2048, tc::LAYOUT_NONE), id_sc, ks > 0);
                    tc::mma_commit(&sm.s_full[b]);
                    tc::mma_commit(&sm.kh_free[b]);
                    if (plast) tc::mma_commit(&sm.res_empty[prs]);   // the item's queries and B_K are done
                    return true;
                };
                for (uint32_t n = 0; ok; ++n) {
                    if (!(ok = dt_wait(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u, lim))) break;
                    const DtItem &e = sm.itab[n % DT_NITAB];
                    const bool live = e.l >= 0;
                    const DtGeo geo = dt_geo(e, G8);
                    tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
                    if (!live || sm.abort) break;
                    // the item's queries and B_K.  The previous item's entry is freed by
                    // its last scores: they go first unless this entry has landed, so
                    // that no wait for an entry holds back the release of another
                    // (two large entries need not fit in the ring together)
                    const uint32_t rs = kr % DT_NRES;
                    if (have_prev && !tc::mbar_test_wait(&sm.res_full[rs], (kr / DT_NRES) & 1u)) {
                        if (!(ok = scores())) break;
                        have_prev = false;
                    }
                    if (!(ok = dt_wait(&sm.res_full[rs], (kr / DT_NRES) & 1u, lim))) break;
                    tc::fence_async_smem();   // the queries came through the generic proxy
                    const uint32_t q_addr = s_rr + sm.res_off[rs];
                    const uint32_t sb = q_addr + (uint32_t)geo.nq16 * 256u;
                    const int nks = geo.R16K / 16;
                    const bool odd = geo.R16K != geo.R8K;   // the last K step's upper 8 ranks read zeros
                    for (int t = 0; t < geo.nt && ok; ++t) {
                        const uint32_t b = g & 1u;
                        ok = dt_wait(&sm.akfull[ka % DT_NSLOT], (ka / DT_NSLOT) & 1u, lim);
                        MILO_DT_LAT(0, ka % DT_NSLOT);
                        MILO_DT_TRACE(31, n, t);
                        if (ok && g >= 2) ok = dt_wait(&sm.kh_free[b], ((g - 2) >> 1) & 1u, lim);
                        if (!ok) break;
                        tc::tc_fence_after();
                        MILO_DT_TRACE(3, n, t);
                        const uint32_t sa = s_ak + sm.ak_off[ka % DT_NSLOT];
                        for (int ks = 0; ks < nks; ++ks) {
                            const uint32_t bk = geo.R8K ? sb + ks * 4096 : s_zero;
                            const uint32_t lbo = geo.R8K == 0 ? 0u : (odd && ks == nks - 1) ? s_zero - bk : 2048u;
                            tc::mma_ss(tmem + DT_COL_KH + 128 * b, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                       tc::smem_desc(bk, lbo, 128, tc::LAYOUT_NONE), id_rb, ks > 0);
                        }
                        tc::mma_commit(&sm.kh_full[b]);
                        tc::mma_commit(&sm.akempty[ka % DT_NSLOT]);
                        ++ka;
                        if (have_prev && !(ok = scores())) break;
                        have_prev = true;
                        pg = g;
                        pq = q_addr;
                        prs = rs;
                        plast = t == geo.nt - 1;
                        pnq16 = geo.nq16;
                        ++g;
                    }
                    ++kr;
                }
                if (ok && have_prev) ok = scores();
                if (!ok) sm.abort = 1;
                tc::mma_commit(&sm.drain_k);
                dt_wait(&sm.drain_k, 0, lim);
            }
        } else {
            // ======================================================== V warp: PV / O
            MILO_DT_TRACE_STATE;
            const uint32_t s_v = tc::smem_u32(sm.vring);
            const uint32_t s_p = tc::smem_u32(sm.pbuf[0]);
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
                const DtItem &e = sm.itab[n % DT_NITAB];
                const bool live = e.l >= 0;
                const DtGeo geo = dt_geo(e, G8);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
                if (__shfl_sync(0xffffffffu, (int)(!live || sm.abort), 0)) break;   // lane 0 decides
                for (int t = 0; t <= geo.nt && ok; ++t) {
                    const bool last = t == geo.nt;      // B_V
                    const uint32_t slot = va % DT_NSLOT;
                    // the tile in fp16 (the RoPE group converts it)
                    if (!(ok = wait_all(&sm.vconv[slot], (va / DT_NSLOT) & 1u))) break;
                    if (lane == 0) MILO_DT_TRACE(5, n, t);
                    if (!last && t == 0 && n >= 2 && !(ok = wait_all(&sm.oa_free[n & 1u], ((n - 2) >> 1) & 1u)))
                        break;
                    // PV: this tile's P buffer; O: the item's O_A / l, handed over in
                    // the P buffer of its last tile
                    const uint32_t pb = (last ? g - 1 : g) & 1u;
                    if (!(ok = wait_all(&sm.p_full[pb], (pb ? pc1 : pc0) & 1u))) break;
                    if (lane == 0) {
                        tc::tc_fence_after();
                        MILO_DT_TRACE(6, n, t);
                        const uint32_t sa = s_v + sm.v_off[slot];
                        const uint32_t sp = s_p + pb * DT_PBUF;
                        const uint32_t dcol = tmem + DT_COL_OA + 64 * (n & 1u);
                        if (!last) {   // O_A^T += A_V(tile)^T P
                            const uint32_t id_pv = tc::idesc_f16(128, geo.nq16, 0, 0, 1);   // fp16, A K-major, B MN-major
                            for (int ks = 0; ks < 8; ++ks)
                                tc::mma_ss(dcol, tc::smem_desc(sa + ks * 256, 128, 2048, tc::LAYOUT_NONE),
                                           tc::smem_desc(sp + ks * 2048, 1024, 128, tc::LAYOUT_NONE), id_pv,
                                           (t | ks) != 0);
                            if (t == geo.nt - 1) tc::mma_commit(&sm.oa_full[n & 1u]);
                        } else {       // O = B_V^T (O_A / l)
                            const uint32_t id_o = tc::idesc_f16(128, geo.nq16, 0, 1, 1);    // fp16, A/B MN-major
                            for (int ks = 0; ks < geo.R16V / 16; ++ks)
                                tc::mma_ss(dcol, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                           tc::smem_desc(sp + ks * 2048, 1024, 128, tc::LAYOUT_NONE), id_o, ks > 0);
                            tc::mma_commit(&sm.o_full[n & 1u]);
                        }
                        tc::mma_commit(&sm.p_free[pb]);
                        tc::mma_commit(&sm.vempty[slot]);
                    }
                    __syncwarp();
                    if (pb) ++pc1;
                    else ++pc0;
                    if (!last) ++g;
                    ++va;
                }
            }
            if (lane == 0) {
                if (!ok) sm.abort = 1;
                tc::mma_commit(&sm.drain_v);
                dt_wait(&sm.drain_v, 0, lim);
            }
        }
    } else if (warp < DT_W_SM) {
        // ============================================================ RoPE group
        MILO_DT_TRACE_STATE;
        reg_alloc<DT_REG_ROPE>();
        const int quad = warp & 3;
        const int half = (warp - DT_W_ROPE) >> 2;         // RoPE pairs 32 half .. +31, O columns 32 half .. +31
        const int gt = threadIdx.x - 32 * DT_W_ROPE;      // thread within the group (0 .. 255)
        const int row = quad * 32 + lane;                 // TMEM lane: token row / channel of O
        const int c0 = 32 * half;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
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
            return grp_and(DT_BAR_ROPE, DT_NROPE, w);
        };
        // an item's geometry and the first row of its partials (entry m of the
        // table; read before the entry is freed)
        int nxt_live = 0, nxt_nt = 0, nxt_nq = 0, nxt_slot0 = 0, nxt_rV = 0, nxt_row0 = 0;
        auto take = [&](uint32_t m) {
            const DtItem &e = sm.itab[m % DT_NITAB];
            nxt_live = e.l >= 0;
            if (nxt_live) {
                nxt_nt = token_tiles(e.Tb);
                nxt_nq = e.ns * G8;
                nxt_slot0 = e.slots[0];
                nxt_rV = e.rV;
                nxt_row0 = e.row0;
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.item_free[m % DT_NITAB]);
        };

        // ---- the next tile of the V ring (an A_V tile, or B_V when last) to
        // fp16 in place; A_V's rank row R8V to ones and rows R8V+1 .. +7 to zero
        // when R8V <= 120, B_V's pad rows to zero
        uint32_t va = 0;
        auto vconvert = [&](int R8V, bool last, uint32_t n, int t) -> bool {
            const uint32_t slot = va % DT_NSLOT;
            if (!gwait(&sm.vfull[slot], (va / DT_NSLOT) & 1u)) return false;
            if (gt == 0) {
                MILO_DT_TRACE(27, n, t);
                MILO_DT_LAT(1, slot);
            }
            uint8_t *tp = sm.vring + sm.v_off[slot];
            if (!a.f16) bf16_to_f16_inplace(tp, R8V * 16, gt, DT_NROPE);
            const int R16V = r16_of(R8V);
            if (!last && R8V <= 120) {
                if (gt < 128) {
                    const uint32_t w = (gt & 7) == 0 ? 0x3C003C00u : 0u;
                    reinterpret_cast<uint4 *>(tp + R8V * 256)[gt] = make_uint4(w, w, w, w);
                }
            } else if (last) {
                for (int e2 = gt; e2 < (R16V - R8V) * 16; e2 += DT_NROPE)
                    reinterpret_cast<uint4 *>(tp + R8V * 256)[e2] = make_uint4(0, 0, 0, 0);
            }
            tc::fence_async_smem();
            tc::mbar_arrive(&sm.vconv[slot]);
            ++va;
            return true;
        };

        // ---- item m's O = B_V^T (O_A / l) (lanes = channels, columns = queries)
        // to its nq rows of fp16 partials: query-major in shared memory, then one
        // bulk store; frees the item's O_A^T buffer
        auto readout = [&](int nq, int row0, uint32_t m) -> bool {
            if (gt == 0) tc::bulk_wait_read_all();   // the previous item's store has read the buffer
            if (!gwait(&sm.o_full[m & 1u], (m >> 1) & 1u)) return false;
            tc::tc_fence_after();
            if (gt == 0) MILO_DT_TRACE(14, m, 0);
            if (c0 < nq) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + DT_COL_OA + 64 * (m & 1u) + lane_off + c0, r);
                tc::tmem_wait_ld();
                if (gt == 0) MILO_DT_TRACE(32, m, 0);
                __half *st = reinterpret_cast<__half *>(sm.ostage) + row;
#pragma unroll
                for (int v = 0; v < 32; ++v) st[(c0 + v) * D] = __float2half_rn(__uint_as_float(r[v]));
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.oa_free[m & 1u]);
            tc::fence_async_smem();
            grp_sync(DT_BAR_ROPE, DT_NROPE);
            if (gt == 0) {
                MILO_DT_TRACE(33, m, 0);
                tc::bulk_s2g(a.part_o16 + (int64_t)row0 * D, sm.ostage, (uint32_t)nq * D * 2u);
                tc::bulk_commit();
                MILO_DT_TRACE(15, m, 0);
            }
            return true;
        };

        // ---------------------------------------------------- the item loop
        // per item: RoPE and the V conversion of every tile, B_V's conversion,
        // then the previous item's read-out
        uint32_t g = 0, n = 0;
        int cur_nt = 0, cur_nq = 0, cur_R8V = 0, cur_slot0 = 0, cur_row0 = 0, prev_nq = 0, prev_row0 = 0;
        if (!(ok = gwait(&sm.item_full[0], 0))) {
            sm.abort = 1;
        } else {
            take(0);
            for (; ok && nxt_live; ++n) {
                cur_nt = nxt_nt;
                cur_nq = nxt_nq;
                cur_R8V = rank_pad(nxt_rV);
                cur_slot0 = nxt_slot0;
                cur_row0 = nxt_row0;
                if (!(ok = gwait(&sm.item_full[(n + 1) % DT_NITAB], ((n + 1) / DT_NITAB) & 1u))) break;
                take(n + 1);
                for (int t = 0; t < cur_nt; ++t, ++g) {
                    const uint32_t b = g & 1u;
                    if (!(ok = gwait(&sm.kh_full[b], (g >> 1) & 1u))) break;
                    tc::tc_fence_after();
                    if (gt == 0) MILO_DT_TRACE(7, n, t);
                    const uint32_t base = tmem + DT_COL_KH + 128 * b + lane_off;
                    // (p + 32 v) theta for the rows of this warp: v = (128 t + 32 quad) / 32
                    const float4 *hi = a.rot_slot + ((int64_t)cur_slot0 * 16 + 4 * t + quad) * (HALF / 2) + c0 / 2;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {       // 16 pairs: x at columns i0 .., y at 64 + i0 ..
                        const int i0 = c0 + 16 * j;
                        uint32_t xr[16], yr[16];
                        tc::tmem_ld16(base + i0, xr);
                        tc::tmem_ld16(base + HALF + i0, yr);
                        tc::tmem_wait_ld();
                        if (gt == 0 && j == 0) MILO_DT_TRACE(26, n, t);
                        uint32_t px[8], py[8];
#pragma unroll
                        for (int v = 0; v < 8; ++v) {   // pairs i0 + 2v, i0 + 2v + 1
                            const int k = 8 * j + v;
                            const float4 h4 = __ldg(hi + k);
                            const float2 ch = make_float2(h4.x, h4.y), shh = make_float2(h4.z, h4.w);
                            // (cos, sin)((p + 32 v' + u) theta): rotation by (p + 32 v') theta after u theta
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
                    if (gt == 0) MILO_DT_TRACE(8, n, t);
                    // the same tile of A_V
                    if (!(ok = vconvert(cur_R8V, false, n, t))) break;
                }
                if (!ok) break;
                if (!(ok = vconvert(cur_R8V, true, n, cur_nt))) break;   // B_V
                if (n >= 1 && !(ok = readout(prev_nq, prev_row0, n - 1))) break;
                prev_nq = cur_nq;
                prev_row0 = cur_row0;
            }
            if (ok && n >= 1) ok = readout(prev_nq, prev_row0, n - 1);
            if (!ok) sm.abort = 1;
        }
        if (gt == 0) tc::bulk_wait_all();   // the partials stored before the CTA exits
    } else {
        // ============================================================ softmax group
        MILO_DT_TRACE_STATE;
        reg_dealloc<DT_REG_SM>();
        const int quad = warp & 3;
        const int half = (warp - DT_W_SM) >> 2;           // query columns 32 half .. +31
        const int bar = DT_BAR_SM + half;                 // this half's named barrier
        const int gt = threadIdx.x - 32 * DT_W_SM - 128 * half;   // thread within the half (0 .. 127)
        const int row = quad * 32 + lane;                 // TMEM lane: token row / rank row of O_A^T
        const int c0 = 32 * half;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float kscale = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(d)
        bool ok = true;
        auto gwait = [&](uint64_t *b, uint32_t par) -> bool {
            const bool w = gt == 0 ? (dt_wait(b, par, lim) && !sm.abort) : true;
            return grp_and(bar, 128, w);
        };
        uint32_t hp0 = 0, hp1 = 0;                        // hand-overs of each P buffer
        uint32_t fp0 = 0, fp1 = 0;                        // their completions waited for
        // thread 0's wait for the last product that used P buffer b (the half
        // learns the outcome at its next barrier)
        auto p_wait0 = [&](uint32_t b) -> bool {
            const uint32_t h = b ? hp1 : hp0;
            uint32_t &f = b ? fp1 : fp0;
            if (f == h) return true;
            f = h;
            return gt == 0 ? dt_wait(&sm.p_free[b], (h - 1) & 1u, lim) : true;
        };
        auto handoff = [&](uint32_t b) {
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.p_full[b]);
            if (b) ++hp1;
            else ++hp0;
        };

        // ---- no spare rank row: column sums of the rounded P by a transposing
        // butterfly; lanes 2c and 2c+1 end with column c of the 16
        auto colsum = [&](const uint32_t *pk, float *ls) {
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

        // geometry of the current and the previous item
        int Tb = 0, nq = 0, nq16 = 0, ones = 0, R8V = 0, R16V = 0;
        int pr_nq = 0, pr_nq16 = 0, pr_ones = 0, pr_R8V = 0, pr_R16V = 0;

        // ---- softmax of tile g (item n, tile t of it)
        auto softmax = [&](uint32_t g, uint32_t n, int t) -> bool {
            const uint32_t b = g & 1u;
            const uint32_t ib = n & 1u;
            float *cref = sm.cref[ib];
            float *lsum = sm.lsum[ib];
            // this warp's wait for the scores
            bool w = true;
            if (lane == 0) w = dt_wait(&sm.s_full[b], (g >> 1) & 1u, lim);
            w = __shfl_sync(0xffffffffu, w, 0) != 0;
            __syncwarp();
            tc::tc_fence_after();
            if (gt == 0) MILO_DT_TRACE(9 + half * 8, n, t);
            const uint32_t dcol = tmem + DT_COL_S + 64 * b + lane_off;
            const int tok = t * FTILE + row;
            const int wc = min(32, nq16 - c0);         // this half's columns (<= 0: none)
            const int lv = tok < Tb ? min(wc, nq - c0) : 0;
            if (t == 0) {   // reference max: the scores of the item's first token; sums to 0
                if (gt < 32) lsum[c0 + gt] = 0.f;
                if (quad == 0 && wc > 0 && w) {
                    uint32_t r[16];
                    for (int h = 0; h < wc; h += 16) {
                        tc::tmem_ld16(dcol + c0 + h, r);
                        tc::tmem_wait_ld();
                        if (lane == 0)
#pragma unroll
                            for (int v = 0; v < 16; ++v) cref[c0 + h + v] = __uint_as_float(r[v]) * kscale;
                    }
                }
                grp_sync(bar, 128);
            }
            uint32_t pk[16];
            float emax = -INFINITY;
            // raw scores to p = 2^(x - cref), packed fp16 pairs: pk[v] <- columns 2v, 2v+1
            auto make_p = [&]() {
                const float2 *cr = reinterpret_cast<const float2 *>(cref + c0);
                const float2 ks2 = make_float2(kscale, kscale);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {   // 16 columns at a time
                    if (16 * hh >= wc) break;
                    uint32_t r[16];
                    tc::tmem_ld16(dcol + c0 + 16 * hh, r);
                    tc::tmem_wait_ld();
                    if (gt == 0 && hh == 0) MILO_DT_TRACE(22 + 2 * half, n, t);
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const int k = 8 * hh + v;
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
            if (wc > 0 && w) make_p();
            if (gt == 0) MILO_DT_TRACE(23 + 2 * half, n, t);
            // one barrier: the P buffer's previous product done (thread 0's wait),
            // no p above 2^8 (or not finite) in the half, no failed wait
            const bool pw = p_wait0(b);
            if (grp_or(bar, 128, !(emax <= DT_OVER) || !pw || !w)) {
                if (grp_or(bar, 128, !pw || !w || sm.abort)) return false;
                // rare path: raise the reference max of the columns, after every P
                // of this item handed over has been used
                const bool pw2 = p_wait0(b ^ 1u);
                if (!grp_and(bar, 128, pw2)) return false;
                if (gt < 32) sm.cmax[c0 + gt] = ord_enc(-INFINITY);
                grp_sync(bar, 128);
                for (int h = 0; h < wc; h += 16) {   // column maxima over the tile's live rows
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
                grp_sync(bar, 128);
                if (gt < wc) {
                    const int c = c0 + gt;
                    const float cn = fmaxf(cref[c], ord_dec(sm.cmax[c]));
                    const float f = dt_ex2(cref[c] - cn);
                    sm.cscale[ib][c] = f;
                    cref[c] = cn;
                    lsum[c] *= f;
                }
                grp_sync(bar, 128);
                if (t > 0) {   // O_A^T columns (every rank lane) times 2^(cref_old - cref_new)
                    tc::tc_fence_after();
                    const uint32_t ocol = tmem + DT_COL_OA + 64 * ib + lane_off;
                    for (int h = 0; h < wc; h += 16) {
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
                grp_sync(bar, 128);
                emax = -INFINITY;
                make_p();
            }
            if (gt == 0) MILO_DT_TRACE(10 + half * 8, n, t);
            if (wc > 0) {
                uint8_t *dst = sm.pbuf[b] + (row >> 3) * 1024 + (row & 7) * 16 + (c0 >> 3) * 128;
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                    if (8 * hh >= wc) break;
                    *reinterpret_cast<uint4 *>(dst + hh * 128) =
                        make_uint4(pk[4 * hh], pk[4 * hh + 1], pk[4 * hh + 2], pk[4 * hh + 3]);
                }
                if (!ones) {
                    colsum(&pk[0], lsum + c0);
                    if (wc > 16) colsum(&pk[8], lsum + c0 + 16);
                }
            }
            // every score of the tile this thread needed has been read
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.s_free[b]);
            handoff(b);
            if (gt == 0) MILO_DT_TRACE(11 + half * 8, n, t);
            return true;
        };

        // ---- item m's O_A^T is complete: denominators, partial (max, sum), and
        // O_A / l (fp16, this half's columns) staged in the P buffer sb of its
        // last tile for the last product
        auto finalize = [&](uint32_t m, uint32_t sb) -> bool {
            if (!gwait(&sm.oa_full[m & 1u], (m >> 1) & 1u)) return false;
            if (gt == 0) MILO_DT_TRACE(12 + half * 8, m, 0);
            tc::tc_fence_after();
            const uint32_t ib = m & 1u;
            const int wc = min(32, pr_nq16 - c0);
            const uint32_t ocol = tmem + DT_COL_OA + 64 * ib + lane_off;
            if (wc > 0 && pr_ones && quad == (pr_R8V >> 5)) {   // the ones row holds sum_t p
                for (int h = 0; h < wc; h += 16) {
                    uint32_t r[16];
                    tc::tmem_ld16(ocol + c0 + h, r);
                    tc::tmem_wait_ld();
                    if (row == pr_R8V)
#pragma unroll
                        for (int v = 0; v < 16; ++v) sm.lsum[ib][c0 + h + v] = __uint_as_float(r[v]);
                }
            }
            grp_sync(bar, 128);
            if (gt < 32) {
                const int c = c0 + gt;
                const float l = sm.lsum[ib][c];
                sm.cscale[ib][c] = (c < pr_nq && l > 0.f) ? __frcp_rn(l) : 0.f;
                const int pi = sm.qp_sm[m & 3u][c];
                if (pi >= 0) a.part_ml[pi] = make_float2(sm.cref[ib][c] * 0.69314718055994531f, l);
            }
            // every 1 / l written before the staging reads them; the buffer's last
            // product (this item's last PV) has completed
            const bool pw = p_wait0(sb);
            if (!grp_and(bar, 128, pw)) return false;
            if (wc > 0 && quad * 32 < pr_R16V) {   // whole warps: tcgen05.ld is warp-collective
                uint8_t *dst = sm.pbuf[sb] + (row >> 3) * 1024 + (row & 7) * 16;
                for (int ch = c0; ch < c0 + wc; ch += 16) {
                    uint32_t r[16];
                    tc::tmem_ld16(ocol + ch, r);
                    tc::tmem_wait_ld();
                    if (row < pr_R16V) {
                        uint32_t q8[8];
                        const bool live = row < pr_R8V;   // pad rows meet B_V's zero rows
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
            handoff(sb);
            if (gt == 0) MILO_DT_TRACE(13 + half * 8, m, 0);
            return true;
        };

        // ---------------------------------------------------- the item loop
        // per tile: softmax; after an item's first tile, the previous item's
        // denominators and staging
        uint32_t g = 0, n = 0;
        if (!(ok = gwait(&sm.item_full[0], 0))) {
            sm.abort = 1;
        } else {
            for (; ok; ++n) {
                if (n > 0 && !(ok = gwait(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u))) break;
                int nt = 0;
                {
                    const DtItem &e = sm.itab[n % DT_NITAB];
                    const bool live = e.l >= 0;
                    if (live) {
                        const DtGeo geo = dt_geo(e, G8);
                        nt = geo.nt;
                        Tb = geo.Tb;
                        nq = geo.nq;
                        nq16 = geo.nq16;
                        ones = geo.ones;
                        R8V = geo.R8V;
                        R16V = geo.R16V;
                        if (gt < 32) sm.qp_sm[n & 3u][c0 + gt] = dt_pidx(a, e, c0 + gt);
                    }
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&sm.item_free[n % DT_NITAB]);
                    if (!live) break;
                }
                for (int t = 0; t < nt && ok; ++t, ++g) {
                    if (!(ok = softmax(g, n, t))) break;
                    if (t == 0 && n >= 1 && !(ok = finalize(n - 1, (g - 1) & 1u))) break;
                }
                if (!ok) break;
                // this item becomes the previous one
                pr_nq = nq;
                pr_nq16 = nq16;
                pr_ones = ones;
                pr_R8V = R8V;
                pr_R16V = R16V;
            }
            // the last item's denominators and staging
            if (ok && n >= 1) ok = finalize(n - 1, (g - 1) & 1u);
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

// the GQA group padded to the queries' core-matrix height
inline int decode_tc_g8(int G) { return (G + 7) / 8 * 8; }
// sessions per work item
inline int decode_tc_spi(int G) { return std::min(DT_MAXS, DT_NQ / decode_tc_g8(G)); }

inline bool decode_tc_supported(const DecodeArgs &a) {
    if (getenv("MILO_FORCE_SIMT")) return false;
    return (a.factor_dtype == MILO_BF16 || a.factor_dtype == MILO_INT8) && a.block_len <= 512 &&
           decode_tc_g8(a.G) <= DT_NQ;
}

// INT8 factors for the tensor cores: the selected blocks' factors of both
// kinds, code x per-column scale (A: per rank, B: per channel) rounded to
// fp16, written at the same element offsets into `out` (one section per
// kind, laid out like the INT8 data).  Grid (L*H*n_b, 2); blocks no slot
// selected are skipped.  8 elements (one core-matrix row) per thread step.
__global__ void __launch_bounds__(256) k_dequant_selected(DecodeArgs a, __half *out0, __half *out1) {
    const int64_t blk = blockIdx.x;
    const int kind = blockIdx.y;
    const int b = (int)(blk % a.n_b);
    if (a.slot_start[b + 1] == a.slot_start[b]) return;
    const KindView &kv = a.kv[kind];
    const int R8 = rank_pad(kv.ranks[blk]);
    if (R8 == 0) return;
    const int Tb = block_tokens(a.T, a.block_len, b);
    const int nt = token_tiles(Tb);
    const int64_t base = kv.offsets[blk];
    const int64_t nA = (int64_t)nt * R8 * FTILE, nAll = nA + (int64_t)R8 * D;
    const int8_t *src = (const int8_t *)kv.data + base;
    __half *dst = (kind ? out1 : out0) + base;
    const float *sA = kv.scaleA + blk * D, *sB = kv.scaleB + blk * D;
    for (int64_t e = (int64_t)threadIdx.x * 8; e < nAll; e += 256 * 8) {
        const uint2 codes = *reinterpret_cast<const uint2 *>(src + e);   // 8 codes, one row of a core matrix
        const int8_t *c = reinterpret_cast<const int8_t *>(&codes);
        float sc[8];
        if (e < nA) {   // A tile: [k/8][u/8][k%8][u%8], one rank k per 8 elements
            const int r = (int)(e % (R8 * FTILE));
            const float s = sA[(r >> 10) * 8 + ((r & 63) >> 3)];
#pragma unroll
            for (int i = 0; i < 8; ++i) sc[i] = s;
        } else {        // B: [k/8][j/8][k%8][j%8], eight channels j per 8 elements
            const int r = (int)(e - nA);
            const int j0 = ((r & 1023) >> 6) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) sc[i] = sB[j0 + i];
        }
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = __floats2half2_rn((float)c[2 * i] * sc[2 * i], (float)c[2 * i + 1] * sc[2 * i + 1]);
            ow[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(dst + e) = o;
    }
}

// The warpgroups' register split assumes the launch value; a build that
// allocated another would stall its register requests, so the attribute is
// checked before the kernel is ever launched.
inline cudaError_t decode_tc_set_attrs() {
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, k_decode_tc);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != DT_REG_LAUNCH) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(k_decode_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_tc_smem_bytes());
}

// upper bound of the number of items: one per selected slot, per (l, h)
inline int64_t decode_tc_max_items(int L, int H, int64_t slots) { return (int64_t)L * H * slots; }

inline cudaError_t launch_decode_tc(const DecodeArgs &a, const int32_t *istart, DtItem *items, int sms,
                                    cudaStream_t s) {
    const int64_t n = (int64_t)a.L * a.H * a.n_b;
    k_dt_items<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a, istart, items);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_decode_tc<<<sms, DT_THREADS, decode_tc_smem_bytes(), s>>>(a, istart, items);
    return cudaGetLastError();
}

}  // namespace milo
