// decode_tc.cuh -- decode attention over retrieved compressed blocks on
// tcgen05 tensor cores (bf16 factors, or INT8 factors dequantised to fp16 by
// k_dequant_selected).
//
// Step "at inference a retriever selects blocks, whose low-rank factors are
// rebuilt before sparse attention" (evolve.pub review of MILO, Summary; FAQ
// "What is MILO").  A prep kernel lists the work items (layer, KV head,
// block, query pass); an item covers up to 128 queries (the sessions that
// selected the block times the GQA group).  One persistent CTA per SM walks
// the items with four roles that only meet at mbarriers:
//
//   producer warp   bulk-copies the block's factors (already in the tensor
//                   cores' canonical layout in HBM): B_K into its own buffer;
//                   the A_K tiles, the A_V tiles (each with a row of ones
//                   appended) and B_V into a ring of variable-size tiles.
//   MMA warp        polls three independent queues and issues whichever op
//                   is ready:
//                     rebuild  K-hat tile = A_K(tile) B_K     (M=128 tokens, N=128, K=r_K, bf16)
//                     scores   S = K-tilde (TMEM) Q-tilde^T    (M=128 tokens, N=nq, K=128, fp16)
//                     PV / O   O_A^T += A_V(tile)^T P          (M=128 ranks, N=nq, K=128 tokens, fp16)
//                              O = B_V^T (O_A / l)            (M=128 channels, N=nq, K=r_V, fp16)
//   RoPE group      8 warps, two per TMEM lane quadrant (one token row per
//                   thread, half the pairs each): rotates each rebuilt key row
//                   by its in-block angle t*theta_i and packs K-tilde to fp16 in
//                   place; two rebuild buffers let it run up to two tiles ahead
//                   of the scores.  It also reads each item's O out to the
//                   partials.
//   softmax groups  2 x 4 warps, alternate 32-query slabs: softmax in the exp2
//                   domain against a per-query reference max that is raised
//                   (with the running O_A^T and sums rescaled) only when a p
//                   exceeds 2^8; P (fp16) to shared memory; O_A / l staged for
//                   the last product.
//   helper warps    2 warps: convert each A_V tile and B_V to fp16 in place as
//                   they land; rotate the next item's queries by -p*theta_i
//                   once the current item's scores are done.
//
// The ones row makes the PV product return the softmax denominators as one
// more row of O_A^T.  Keys and values are never written to memory.  Each
// (query, selected slot) gets a partial (max, sum, normalised output) merged
// by k_combine.
#pragma once
#include "decode_simt.cuh"
#include "tc_common.cuh"

namespace milo {
// Timeline events of k_decode_tc (argument: the CTA's item n and a tile or
// ring position t).  Recorded only by the tracing build (decode_trace.cuh);
// elsewhere the hooks compile to nothing.
enum TlEvent : uint32_t {
    TL_P_CLAIM = 1,    // producer: item claimed
    TL_P_REQ,          // producer: ring position t wanted
    TL_P_PLACED,       // producer: ring space for t found
    TL_P_ISSUED,       // producer: copy of t issued (t = 31: B_K)
    TL_M_REB,          // MMA thread: rebuild of tile t issued
    TL_M_SCO,          // MMA thread: scores of tile t issued
    TL_M_PV,           // MMA thread: PV of tile t issued
    TL_M_O,            // MMA thread: output product issued
    TL_M_RET,          // MMA thread: back from an issue (t = the kind: 0 rebuild, 1 scores, 2 PV, 3 O)
    TL_R_START,        // RoPE: rebuilt keys of tile t in TMEM, rotation starts
    TL_R_END,          // RoPE: rotated keys of tile t handed to the scores
    TL_R_OUT,          // RoPE: read-out of item n's output starts
    TL_R_OUT_GOT,      // RoPE: item n's output product complete
    TL_R_OUT_END,      // RoPE: item n's output written
    TL_S_START,        // softmax: scores of tile t in TMEM
    TL_S_LOADED,       // softmax: first slab of tile t loaded from TMEM
    TL_S_MADE,         // softmax: first slab's p made and the group agreed on the rare path
    TL_S_PFREE,        // softmax: P buffer of tile t free
    TL_S_RESCALE,      // softmax: rare path taken in tile t
    TL_S_END,          // softmax: P of tile t handed over
    TL_S_OA,           // softmax: O_A of item n complete
    TL_S_DONE,         // softmax: item n's denominators and staging done
    TL_H_CONV,         // helpers: ring position t converted / passed
    TL_H_Q_START,      // helpers: queries of item n start
    TL_H_Q_END,        // helpers: queries of item n staged
};
}  // namespace milo
#ifdef MILO_DECODE_TRACE
#include "decode_trace.cuh"
#else
#define MILO_TL_LOCALS
#define MILO_TL(ev, n, t) \
    do {                  \
        (void)(n);        \
        (void)(t);        \
    } while (0)
#endif


namespace milo {

constexpr int DT_GROUP = 128;                          // threads per epilogue group
constexpr int DT_HELP = 64;                            // helper threads
constexpr int DT_RGROUP = 2 * DT_GROUP;                // RoPE threads: two warps per TMEM lane quadrant
constexpr int DT_THREADS = 64 + DT_RGROUP + 2 * DT_GROUP + DT_HELP; // warp 0 producer, 1 MMA, 2-9 RoPE,
                                                                    // 10-17 softmax, 18-19 helpers
constexpr int DT_W_S = 2 + DT_RGROUP / 32;             // first softmax warp
constexpr int DT_W_H = DT_W_S + 2 * DT_GROUP / 32;     // first helper warp
constexpr int DT_RING = 96 * 1024;                     // ring bytes for A_K, A_V and B_V tiles
constexpr int DT_NBAR = 32;                            // ring tiles in flight at most
constexpr int DT_TILE_MAX = 128 * 256;                 // 128 rank rows x 128 tokens (or channels) x 16 bit
constexpr int DT_NQ = 128;                             // queries per item (pass)
constexpr int DT_NITAB = 32;                           // claimed items in flight at most
constexpr uint32_t DT_TMEM_COLS = 512;
constexpr uint32_t DT_COL_D1 = 0;                      // two 128-column rebuild buffers
constexpr uint32_t DT_COL_D2 = 256;                    // scores: one 128-column buffer or two of 64
constexpr uint32_t DT_COL_OA = 384;                    // O_A^T, then O
constexpr float DT_RESCALE = 8.f;                      // log2 headroom before the reference max moves
constexpr int DT_BAR_S = 1, DT_BAR_R = 2, DT_BAR_H = 3, DT_BAR_S2 = 4; // named barriers of the groups

// One work item, written by k_dt_items.
struct DtItem {
    int32_t l, h, b, q0;
    int32_t nq, Tb, rK, rV;
    int64_t offK, offV;     // element offsets of the block in the data sections
    int32_t slot0, pad[3];  // start of the block's slot list
};

struct DecTcSmem {
    alignas(128) uint8_t ring[DT_RING];
    // B_K of the current item.  It follows the ring so that the 128-row
    // operand read of an A_V tile near the ring's end stays in shared memory
    // (rows past the tile only feed rows of O_A^T that are never used).
    alignas(128) uint8_t bk[DT_TILE_MAX];
    alignas(128) uint8_t qt[DT_NQ * D * 2];      // rotated queries, fp16, K-major
    alignas(128) uint8_t pbuf[128 * DT_NQ * 2];  // P or O_A / l (fp16), MN-major; two halves when nq <= 64
    float2 t1[HALF][32];                         // (cos, sin)((t % 32) theta_i)
    float2 t2[HALF][16];                         // (cos, sin)(32 (t / 32) theta_i)
    float cref[DT_NQ];                           // reference max per query (log2 domain)
    float cscale[DT_NQ];                         // rescale factors, then 1 / l
    float lsum[DT_NQ];
    int cmax[DT_NQ];                             // column maxima, order-preserving int encoding
    int qpidx[4][DT_NQ];                         // partial index of each query, per item (mod 4)
    uint32_t toff[DT_NBAR], tlen[DT_NBAR];       // ring offset and bytes of each tile in flight
    int itab[DT_NITAB];                          // n-th item claimed by this CTA (slot n % NITAB), -1: none left
    uint64_t item_full[DT_NITAB];                // slot n % NITAB holds item n
    // conv: one arrival per ring tile, in ring order, once an A_V / B_V tile
    // is fp16 (A_K tiles pass straight through), so that slot k % NBAR is in
    // phase k / NBAR exactly like full and empty
    uint64_t full[DT_NBAR], empty[DT_NBAR], conv[DT_NBAR];
    uint64_t bk_full, bk_empty;
    uint64_t d1_full[2], d1_empty[2], kt_full[2];
    uint64_t d2_full[2], d2_empty[2];
    uint64_t p_full[2], p_empty[2];
    uint64_t q_full, q_empty, oa_full, o_full, oa_free, drain;
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
    it.Tb = BlockGeo{a.T, a.block_len, a.starts}.len(b);
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
    bool ones;         // rank row R8V of each A_V tile is all ones (needs R8V <= 120)
    bool dbl;          // nq16 <= 64: scores and P double-buffered
};
__device__ __forceinline__ DtGeo dt_geo(int Tb, int rK, int rV, int nq) {
    DtGeo g;
    g.nt = token_tiles(Tb);
    g.R8K = rank_pad(rK);
    g.R16K = r16_of(g.R8K);
    g.R8V = rank_pad(rV);
    g.R16V = r16_of(g.R8V);
    g.ones = g.R8V <= 120;
    g.rowsV = g.ones ? max(g.R8V + 8, g.R16V) : g.R8V;
    g.nq = nq;
    g.nq16 = (nq + 15) & ~15;
    g.dbl = g.nq16 <= 64;
    return g;
}
__device__ __forceinline__ DtGeo dt_geo(const DtItem *__restrict__ items, int64_t i, int64_t n_items) {
    if (i >= n_items) return dt_geo(1, 0, 0, 0);
    return dt_geo(__ldg(&items[i].Tb), __ldg(&items[i].rK), __ldg(&items[i].rV), __ldg(&items[i].nq));
}

// Ring tiles of an item, 2 nt + 1 of them, in the order they are consumed:
// A_V(t) follows A_K(t + 2) (the rebuilds run two tiles ahead of the PV
// products), B_V comes last:  A_K0 A_K1 A_K2 A_V0 A_K3 A_V1 A_V2 A_V3 B_V.
__device__ __forceinline__ int dt_ring_tiles(const DtGeo &g) { return 2 * g.nt + 1; }
__host__ __device__ __forceinline__ int dt_pos_k(int t) { return t + (t > 2 ? t - 2 : 0); }
__host__ __device__ __forceinline__ int dt_pos_v(int nt, int t) { return (t + 3 < nt ? t + 3 : nt) + t; }
// kind of ring position k: 0 = A_K, 1 = A_V, 2 = B_V; *t = its tile
__host__ __device__ __forceinline__ int dt_tile_at(int nt, int k, int *t) {
    if (k == 2 * nt) { *t = nt; return 2; }
    for (int u = 0; u < nt; ++u) {
        if (dt_pos_k(u) == k) { *t = u; return 0; }
        if (dt_pos_v(nt, u) == k) { *t = u; return 1; }
    }
    *t = 0;
    return 0;
}

// Two counters selected by a runtime index without a local-memory array.
struct DtPair {
    uint32_t c0 = 0, c1 = 0;
    __device__ __forceinline__ uint32_t operator[](uint32_t b) const { return b ? c1 : c0; }
    __device__ __forceinline__ void inc(uint32_t b) {
        if (b) ++c1;
        else ++c0;
    }
};

// named-barrier helpers for one 128-thread group
template <int ID, int N = DT_GROUP>
__device__ __forceinline__ void grp_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory");
}
template <int ID, int N = DT_GROUP>
__device__ __forceinline__ bool grp_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(ID), "n"(N)
        : "memory");
    return r != 0;
}
template <int ID, int N = DT_GROUP>
__device__ __forceinline__ bool grp_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(ID), "n"(N)
        : "memory");
    return r != 0;
}

// the same with the barrier id in a register
__device__ __forceinline__ void grp_sync_rt(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(DT_GROUP) : "memory");
}
__device__ __forceinline__ bool grp_and_rt(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "n"(DT_GROUP)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool grp_or_rt(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "n"(DT_GROUP)
        : "memory");
    return r != 0;
}

// non-blocking probe of an mbarrier phase
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(tc::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
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

// bf16 pairs to fp16 pairs, in place, over n16 16-byte chunks
__device__ __forceinline__ void bf16_to_f16_inplace(uint8_t *base, int n16, int tid, int nthr) {
    uint4 *w = reinterpret_cast<uint4 *>(base);
    for (int e = tid; e < n16; e += nthr) {
        uint4 v = w[e];
        uint32_t *u = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[k]));
            const __half2 h = __floats2half2_rn(f.x, f.y);
            u[k] = *reinterpret_cast<const uint32_t *>(&h);
        }
        w[e] = v;
    }
}

__global__ void __launch_bounds__(DT_THREADS, 1)
k_decode_tc(DecodeArgs a, const int32_t *__restrict__ pstart, const DtItem *__restrict__ items) {
    extern __shared__ __align__(128) unsigned char dt_raw[];
    // aligned by pointer arithmetic, so that the compiler keeps the shared
    // address space (an integer round trip would turn every access generic)
    DecTcSmem &sm = *reinterpret_cast<DecTcSmem *>(dt_raw + ((128u - (tc::smem_u32(dt_raw) & 127u)) & 127u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_items = (int64_t)a.L * a.H * pstart[a.n_b];
    const uint64_t lim = a.wait_ns;   // limit of every wait (ns of %globaltimer)
    MILO_TL_LOCALS
    // Items are claimed dynamically: the producer takes the next unclaimed one
    // from a global counter and publishes it in the item table; every role
    // walks the same sequence n = 0, 1, ... of this CTA's items.  (The factor
    // ring keeps the producer fewer than NITAB items ahead of the slowest role,
    // so a slot is never rewritten before every role has read it.)
    auto item_ready = [&](uint32_t n) { return mbar_test(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u); };
    auto item_wait = [&](uint32_t n) { return tc::mbar_wait(&sm.item_full[n % DT_NITAB], (n / DT_NITAB) & 1u, lim); };
    auto item_at = [&](uint32_t n) -> int64_t { return sm.itab[n % DT_NITAB]; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < DT_NBAR; ++s) {
            tc::mbar_init(&sm.full[s], 1);
            tc::mbar_init(&sm.empty[s], 1);
            tc::mbar_init(&sm.conv[s], 1);
        }
        for (int s = 0; s < DT_NITAB; ++s) tc::mbar_init(&sm.item_full[s], 1);
        tc::mbar_init(&sm.bk_full, 1);
        tc::mbar_init(&sm.bk_empty, 1);
        for (int k = 0; k < 2; ++k) {
            tc::mbar_init(&sm.d1_full[k], 1);
            tc::mbar_init(&sm.d1_empty[k], 1);
            tc::mbar_init(&sm.kt_full[k], DT_RGROUP);
            tc::mbar_init(&sm.d2_full[k], 1);
            tc::mbar_init(&sm.d2_empty[k], 2 * DT_GROUP);
            tc::mbar_init(&sm.p_full[k], 2 * DT_GROUP);
            tc::mbar_init(&sm.p_empty[k], 1);
        }
        tc::mbar_init(&sm.q_full, DT_HELP);
        tc::mbar_init(&sm.q_empty, 1);
        tc::mbar_init(&sm.oa_full, 1);
        tc::mbar_init(&sm.o_full, 1);
        tc::mbar_init(&sm.oa_free, DT_RGROUP);
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

    if (warp == 0) {
        // ================================================================ producer
        const uint8_t *dataK = (const uint8_t *)a.kv[0].data;
        const uint8_t *dataV = (const uint8_t *)a.kv[1].data;
        // The ring is a FIFO byte buffer: tiles are placed at `head` (or at 0
        // when they would cross the end) and released oldest first; `tail`
        // is the oldest tile not yet seen released.
        uint32_t head = 0, seq = 0, tail = 0;
        bool withheld = false;   // the first B_K copy never issued (tests of the bounded waits)
        uint32_t trace_n = 0;   // item and ring position of the tile being placed (timeline only)
        int trace_k = 0;
        bool ok = true;
        // room for a tile of `bytes`: lane 0 releases tiles from the tail
        // (all older than the new tile, so all released without it) until the
        // bytes are free and a barrier slot is; the warp follows.  Returns
        // the tile's offset.
        auto place = [&](uint32_t bytes) -> uint32_t {
            const uint32_t off = head + bytes > (uint32_t)DT_RING ? 0u : head;
            if (lane == 0) {
                while (ok && tail < seq) {
                    const uint32_t t0 = sm.toff[tail % DT_NBAR];   // oldest live byte
                    // live bytes run from t0 up to head, circularly
                    const bool room = t0 < head ? (off == head || off + bytes <= t0)
                                                : (off >= head && off + bytes <= t0);
                    if (room && seq - tail < DT_NBAR) break;
                    if (!tc::mbar_wait(&sm.empty[tail % DT_NBAR], (tail / DT_NBAR) & 1u, lim)) { ok = false; break; }
                    ++tail;
                }
                const uint32_t s = seq % DT_NBAR;
                sm.toff[s] = off;
                sm.tlen[s] = bytes;
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            head = off + bytes;
            return off;
        };
        // rank rows [r0, r1) of a tile: zeros; with `ones`, row r0 is fp16 1.0
        // (A_V tiles are converted to fp16 before use)
        auto fill_rows = [&](uint8_t *dst, int r0, int r1, bool ones) {
            for (int e = lane; e < (r1 - r0) * 16; e += 32) {
                const uint32_t w = (ones && e < 128 && (e & 7) == 0) ? 0x3C003C00u : 0u;
                *reinterpret_cast<uint4 *>(dst + r0 * 256 + e * 16) = make_uint4(w, w, w, w);
            }
            tc::fence_async_smem();
            __syncwarp();
        };
        // one ring tile of `rows` rank rows, `copy` of them from HBM
        auto ring_tile = [&](const uint8_t *src, int rows, int copy, bool ones) {
            const uint32_t off = place((uint32_t)rows * 256u);
            if (!ok) return;
            if (lane == 0) MILO_TL(TL_P_PLACED, trace_n, trace_k);
            uint8_t *dst = sm.ring + off;
            if (rows > copy) fill_rows(dst, copy, rows, ones);
            if (lane == 0) {
                const uint32_t s = seq % DT_NBAR;
                const uint32_t bytes = (uint32_t)copy * 256u;
                tc::mbar_arrive_expect_tx(&sm.full[s], bytes);
                if (bytes) tc::bulk_g2s(dst, src, bytes, &sm.full[s]);
            }
            ++seq;
        };
        uint32_t n = 0;
        for (; ok; ++n) {
            int claimed = -1;
            if (lane == 0) {
                if (!sm.abort) {
                    const int c = atomicAdd(a.claim, 1);
                    if (c < n_items) claimed = c;
                }
                sm.itab[n % DT_NITAB] = claimed;
                tc::mbar_arrive(&sm.item_full[n % DT_NITAB]);   // releases the table entry
            }
            const int64_t i = __shfl_sync(0xffffffffu, claimed, 0);
            if (i < 0) break;
            if (lane == 0) MILO_TL(TL_P_CLAIM, n, 0);
            const DtItem it = items[i];
            const DtGeo g = dt_geo(it.Tb, it.rK, it.rV, it.nq);
            const uint8_t *bK = dataK + 2 * it.offK, *bV = dataV + 2 * it.offV;
            const int64_t tileK = (int64_t)g.R8K * 256, tileV = (int64_t)g.R8V * 256;
            trace_n = n;
            trace_k = 0;
            if (lane == 0) MILO_TL(TL_P_REQ, n, 0);
            ring_tile(bK, g.R16K, g.R8K, false);                               // A_K tile 0 (position 0)
            if (lane == 0) MILO_TL(TL_P_ISSUED, n, 0);
            if (!ok) break;
            // B_K into its own buffer once the previous item's rebuilds are done
            if (lane == 0) ok = tc::mbar_wait(&sm.bk_empty, (n & 1u) ^ 1u, lim);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (g.R16K > g.R8K) fill_rows(sm.bk, g.R8K, g.R16K, false);
            if (lane == 0 && a.inject == 1 && n == 0) {
                withheld = true;   // no copy, no arrival: the rebuild's wait runs out
            } else if (lane == 0) {
                tc::mbar_arrive_expect_tx(&sm.bk_full, (uint32_t)tileK);
                if (tileK) tc::bulk_g2s(sm.bk, bK + g.nt * tileK, (uint32_t)tileK, &sm.bk_full);
                MILO_TL(TL_P_ISSUED, n, 31);
            }
            for (int k = 1; k <= 2 * g.nt && ok; ++k) {
                int t;
                const int kind = dt_tile_at(g.nt, k, &t);
                if (lane == 0) MILO_TL(TL_P_REQ, n, k);
                trace_n = n;
                trace_k = k;
                if (kind == 0) ring_tile(bK + t * tileK, g.R16K, g.R8K, false);          // A_K(t)
                else if (kind == 1) ring_tile(bV + t * tileV, g.rowsV, g.R8V, g.ones);   // A_V(t)
                else ring_tile(bV + g.nt * tileV, g.R16V, g.R8V, false);                // B_V
                if (lane == 0) MILO_TL(TL_P_ISSUED, n, k);
            }
        }
        if (!ok && lane == 0) sm.abort = 1;
        // drain: every copy issued has landed before the CTA exits
        if (lane == 0) {
            for (uint32_t k = seq >= DT_NBAR ? seq - DT_NBAR : 0; k < seq; ++k)
                tc::mbar_wait(&sm.full[k % DT_NBAR], (k / DT_NBAR) & 1u, lim);
            if (n > 0 && !(withheld && n == 1)) tc::mbar_wait(&sm.bk_full, (n - 1) & 1u, lim);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            const uint32_t id_rb = tc::idesc_f16(128, 128, a.f16 ? 0 : 1, 1, 1);   // bf16 (or fp16), A/B MN-major
            // each queue holds its item (kPend until the producer has claimed it,
            // -1 once none is left) and the next one when already known
            constexpr int64_t kPend = -2;
            int64_t iR = kPend, iS = kPend, iP = kPend, iRn = kPend, iSn = kPend, iPn = kPend;
            DtGeo gR = dt_geo(1, 0, 0, 0), gS = gR, gP = gR, gRn = gR, gSn = gR, gPn = gR;
            // resolve a queue's current / next item from the item table
            auto resolve = [&](int64_t &i, DtGeo &g, int64_t &in, DtGeo &gn, uint32_t n) {
                if (i == kPend && in != kPend) {
                    i = in; g = gn; in = kPend;
                }
                if (i == kPend && item_ready(n)) {
                    i = item_at(n);
                    if (i >= 0) g = dt_geo(items, i, n_items);
                }
                if (i >= 0 && in == kPend && item_ready(n + 1)) {
                    in = item_at(n + 1);
                    if (in >= 0) gn = dt_geo(items, in, n_items);
                }
            };
            uint32_t nR = 0, tR = 0, seqR = 0, rc = 0;             // rebuild queue
            uint32_t nS = 0, tS = 0, rcS = 0;                      // scores queue
            uint32_t nP = 0, tP = 0, seqP = 0;                     // PV / O queue
            DtPair u2, pu;                                         // uses of each scores / P buffer
            const uint32_t sq = tc::smem_u32(sm.qt);
            const uint32_t sbk = tc::smem_u32(sm.bk);
            const uint32_t spb = tc::smem_u32(sm.pbuf);
            const uint32_t sring = tc::smem_u32(sm.ring);
            uint64_t t_last = tc::globaltimer();
            uint32_t backoff = 32;
            bool ok = true;
            while (ok) {
                resolve(iR, gR, iRn, gRn, nR);
                resolve(iS, gS, iSn, gSn, nS);
                resolve(iP, gP, iPn, gPn, nP);
                if (iR == -1 && iS == -1 && iP == -1) break;
                bool prog = false;
                // ---------------------------------------------------- rebuild
                if (iR >= 0) {
                    const uint32_t k = seqR + dt_pos_k(tR), s = k % DT_NBAR, b = rc & 1u;
                    if (mbar_test(&sm.full[s], (k / DT_NBAR) & 1u) && (tR > 0 || mbar_test(&sm.bk_full, nR & 1u)) &&
                        mbar_test(&sm.d1_empty[b], ((rc >> 1) & 1u) ^ 1u)) {
                        MILO_TL(TL_M_REB, nR, tR);
                        tc::tc_fence_after();
                        const uint32_t sa = sring + sm.toff[s];
                        for (int ks = 0; ks < gR.R16K / 16; ++ks)
                            tc::mma_ss(tmem + DT_COL_D1 + 128 * b,
                                       tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                       tc::smem_desc(sbk + ks * 4096, 2048, 128, tc::LAYOUT_NONE), id_rb, ks > 0);
                        tc::mma_commit(&sm.d1_full[b]);
                        tc::mma_commit(&sm.empty[s]);
                        if ((int)tR == gR.nt - 1) tc::mma_commit(&sm.bk_empty);
                        MILO_TL(TL_M_RET, nR, 0);
                        ++rc;
                        if ((int)++tR == gR.nt) {
                            seqR += dt_ring_tiles(gR);
                            tR = 0;
                            ++nR;
                            iR = kPend;
                        }
                        prog = true;
                    }
                }
                // ---------------------------------------------------- scores
                if (iS >= 0) {
                    const uint32_t b = rcS & 1u;
                    const uint32_t d2b = gS.dbl ? (tS & 1u) : 0u;
                    // a full-width scores buffer also covers the second half-buffer
                    if (mbar_test(&sm.kt_full[b], (rcS >> 1) & 1u) && (tS > 0 || mbar_test(&sm.q_full, nS & 1u)) &&
                        mbar_test(&sm.d2_empty[d2b], (u2[d2b] & 1u) ^ 1u) &&
                        (gS.dbl || mbar_test(&sm.d2_empty[1], (u2[1] & 1u) ^ 1u))) {
                        MILO_TL(TL_M_SCO, nS, tS);
                        tc::tc_fence_after();
                        const uint32_t id_sc = tc::idesc_f16(128, gS.nq16, 0, 0, 0);   // fp16, A tmem, B K-major
                        const uint32_t kt = tmem + DT_COL_D1 + 128 * b;
                        // K-tilde packed in place: the 16 dims of k-step ks (pairs
                        // 16(ks % 4).. of the x or y half) at columns (ks >= 4 ? 64 : 0)
                        // + {0, 8, 32, 40}[ks % 4]
                        for (int ks = 0; ks < D / 16; ++ks)
                            tc::mma_ts(tmem + DT_COL_D2 + 64 * d2b,
                                       kt + (ks >= 4 ? 64 : 0) + ((ks & 3) < 2 ? 8 * (ks & 3) : 16 + 8 * (ks & 3)),
                                       tc::smem_desc(sq + ks * 256, 128, 2048, tc::LAYOUT_NONE), id_sc, ks > 0);
                        tc::mma_commit(&sm.d2_full[d2b]);
                        tc::mma_commit(&sm.d1_empty[b]);
                        if ((int)tS == gS.nt - 1) tc::mma_commit(&sm.q_empty);
                        MILO_TL(TL_M_RET, nS, 1);
                        u2.inc(d2b);
                        ++rcS;
                        if ((int)++tS == gS.nt) {
                            tS = 0;
                            ++nS;
                            iS = kPend;
                        }
                        prog = true;
                    }
                }
                // ---------------------------------------------------- PV and O
                if (iP >= 0) {
                    const uint32_t pb = gP.dbl ? (tP & 1u) : 0u;
                    const uint32_t lbo_p = (uint32_t)(gP.nq16 / 8) * 128u;
                    const uint32_t sp = spb + pb * 16384u;
                    // A_V tile tP, or B_V when tP == nt
                    const uint32_t kv = seqP + ((int)tP < gP.nt ? dt_pos_v(gP.nt, tP) : 2 * gP.nt);
                    if (mbar_test(&sm.p_full[pb], pu[pb] & 1u) && mbar_test(&sm.conv[kv % DT_NBAR], (kv / DT_NBAR) & 1u) &&
                        (tP > 0 || mbar_test(&sm.oa_free, (nP & 1u) ^ 1u))) {
                        tc::tc_fence_after();
                        if ((int)tP < gP.nt) {   // O_A^T += A_V(tile)^T P
                            MILO_TL(TL_M_PV, nP, tP);
                            const uint32_t k = kv, s = k % DT_NBAR;
                            const uint32_t sa = sring + sm.toff[s];
                            const uint32_t id_pv = tc::idesc_f16(128, gP.nq16, 0, 0, 1);   // fp16, A K-major, B MN-major
                            for (int ks = 0; ks < 8; ++ks)
                                tc::mma_ss(tmem + DT_COL_OA, tc::smem_desc(sa + ks * 256, 128, 2048, tc::LAYOUT_NONE),
                                           tc::smem_desc(sp + ks * 2 * lbo_p, lbo_p, 128, tc::LAYOUT_NONE), id_pv,
                                           (tP | ks) != 0);
                            tc::mma_commit(&sm.p_empty[pb]);
                            tc::mma_commit(&sm.empty[s]);
                            if ((int)tP == gP.nt - 1) tc::mma_commit(&sm.oa_full);
                            MILO_TL(TL_M_RET, nP, 2);
                            pu.inc(pb);
                            ++tP;
                        } else {                 // O = B_V^T (O_A / l), over O_A's columns
                            MILO_TL(TL_M_O, nP, tP);
                            const uint32_t k = kv, s = k % DT_NBAR;
                            const uint32_t sa = sring + sm.toff[s];
                            const uint32_t id_o = tc::idesc_f16(128, gP.nq16, 0, 1, 1);    // fp16, A/B MN-major
                            for (int ks = 0; ks < gP.R16V / 16; ++ks)
                                tc::mma_ss(tmem + DT_COL_OA, tc::smem_desc(sa + ks * 4096, 2048, 128, tc::LAYOUT_NONE),
                                           tc::smem_desc(sp + ks * 2 * lbo_p, lbo_p, 128, tc::LAYOUT_NONE), id_o,
                                           ks > 0);
                            tc::mma_commit(&sm.p_empty[pb]);
                            tc::mma_commit(&sm.empty[s]);
                            tc::mma_commit(&sm.o_full);
                            MILO_TL(TL_M_RET, nP, 3);
                            pu.inc(pb);
                            seqP += dt_ring_tiles(gP);
                            tP = 0;
                            ++nP;
                            iP = kPend;
                        }
                        prog = true;
                    }
                }
                if (prog) {
                    t_last = tc::globaltimer();
                    backoff = 32;
                } else if (sm.abort || tc::globaltimer() - t_last > lim) {
                    if (!sm.abort) raise_status(ST_TIMEOUT);
                    ok = false;
                } else {
                    // idle: sleep, longer while nothing happens, so that the
                    // polling leaves issue slots and i-cache to the group warps
                    __nanosleep(backoff);
                    backoff = min(backoff * 2, 64u);
                }
            }
            if (!ok) sm.abort = 1;
            tc::mma_commit(&sm.drain);
            tc::mbar_wait(&sm.drain, 0, lim);
        }
    } else if (warp < DT_W_S) {
        // ================================================================ RoPE group
        // Two warps per TMEM lane quadrant; half rh rotates pair chunks 2rh and
        // 2rh + 1 (pairs 32rh .. 32rh + 31) of every token row of its quadrant.
        const int et = threadIdx.x - 64;
        const int rh = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        uint32_t rc = 0, n = 0;
        bool ok = true;
        (void)et;
        // O = B_V^T (O_A / l) of item m (lanes = channels, columns = queries)
        // to the partials; frees O_A^T for the next item's PV products
        int pend_nq = -1;   // queries of the item whose O is still to be read, or -1
        uint32_t pend_n = 0;
        auto readout = [&]() -> bool {
            MILO_TL(TL_R_OUT, pend_n, 0);
            if (!grp_and<DT_BAR_R, DT_RGROUP>(tc::mbar_wait(&sm.o_full, pend_n & 1u, lim) && !sm.abort)) return false;
            MILO_TL(TL_R_OUT_GOT, pend_n, 0);
            tc::tc_fence_after();
            const int *qp = sm.qpidx[pend_n & 3u];
            const int nq = pend_nq, nq16 = (nq + 15) & ~15;
            for (int c0 = 32 * rh; c0 < nq16; c0 += 64) {   // this half's 32-query slabs
                uint32_t r[32];
                tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                if (c0 + 16 < nq16)
                    tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
                tc::tmem_wait_ld();
#pragma unroll
                for (int v = 0; v < 32; ++v)
                    if (c0 + v < nq) a.part_o[(int64_t)qp[c0 + v] * D + row] = __uint_as_float(r[v]);
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.oa_free);
            MILO_TL(TL_R_OUT_END, pend_n, 0);
            pend_nq = -1;
            return true;
        };
        for (; ok; ++n) {
            ok = grp_and<DT_BAR_R, DT_RGROUP>(item_wait(n) && !sm.abort);
            if (!ok) break;
            const int64_t i = item_at(n);
            if (i < 0) break;
            const int nt = token_tiles(__ldg(&items[i].Tb));
            for (int t = 0; t < nt; ++t) {
                const uint32_t b = rc & 1u;
                ok = grp_and<DT_BAR_R, DT_RGROUP>(tc::mbar_wait(&sm.d1_full[b], (rc >> 1) & 1u, lim) && !sm.abort);
                if (!ok) break;
                MILO_TL(TL_R_START, n, t);
                tc::tc_fence_after();
                const uint32_t base = tmem + DT_COL_D1 + 128 * b + lane_off;
                const int tok = t * FTILE + row;   // in-block token of this lane
                const int tl = tok & 31, th = tok >> 5;
                // pair chunk pc (16 pairs): x at columns 16pc.., y at 64 + 16pc..;
                // packed fp16 results go to 32rh + 8j (x) and 64 + 32rh + 8j (y) for
                // the half's j-th chunk: columns of the half's first chunk, which
                // this thread has already read
                auto rot_chunk = [&](const uint32_t (&xr)[16], const uint32_t (&yr)[16], int pc, int j) {
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
                    tc::tmem_st8(base + 32 * rh + 8 * j, px);
                    tc::tmem_st8(base + 64 + 32 * rh + 8 * j, py);
                };
#pragma unroll 1
                for (int j = 0; j < 2; ++j) {
                    const int pc = 2 * rh + j;
                    uint32_t xa[16], ya[16];
                    tc::tmem_ld16(base + 16 * pc, xa);
                    tc::tmem_ld16(base + 64 + 16 * pc, ya);
                    tc::tmem_wait_ld();
                    rot_chunk(xa, ya, pc, j);
                }
                tc::tmem_wait_st();
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.kt_full[b]);
                ++rc;
                MILO_TL(TL_R_END, n, t);
                // the previous item's output, once this item's first two tiles
                // are rotated (the softmax group has work queued meanwhile)
                if (t == min(1, nt - 1) && pend_nq >= 0 && !(ok = readout())) break;
            }
            if (!ok) break;
            pend_nq = __ldg(&items[i].nq);
            pend_n = n;
        }
        if (ok && pend_nq >= 0) ok = readout();
        if (!ok) sm.abort = 1;
    } else if (warp < DT_W_H) {
        // ================================================================ softmax groups
        // Two groups of 4 warps (one per TMEM lane quadrant, one token row per
        // thread); group sg owns the 32-column query slabs sg, sg + 2, ...  The
        // reference max, sums and P of a column belong to one group, so the
        // groups only meet at the counted arrivals.
        const int sg = (warp - DT_W_S) >> 2;
        const int gt = threadIdx.x - 32 * DT_W_S - DT_GROUP * sg;   // thread within the group
        const int bar_id = sg == 0 ? DT_BAR_S : DT_BAR_S2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;                  // TMEM lane of this thread
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float kscale = 1.4426950408889634f * rsqrtf((float)D);   // log2(e) / sqrt(d)
        DtPair u2;                                         // uses of each scores buffer
        DtPair pf, pe;                                     // P buffer hand-overs / completions seen
        uint32_t n = 0;
        bool ok = true;

        // wait until P buffer b's last product (PV or O) has completed
        auto p_drain = [&](int b) -> bool {
            if (pe[b] == pf[b]) return true;
            const bool w = grp_and_rt(bar_id, tc::mbar_wait(&sm.p_empty[b], pe[b] & 1u, lim));
            pe.inc(b);
            return w;
        };

        for (; ok; ++n) {
            ok = grp_and_rt(bar_id, item_wait(n) && !sm.abort);
            if (!ok) break;
            const int64_t i = item_at(n);
            if (i < 0) break;
            const DtGeo g = dt_geo(items, i, n_items);
            const int Tb = __ldg(&items[i].Tb);
            const int nq = g.nq, nq16 = g.nq16;
            const uint32_t lbo_p = (uint32_t)(nq16 / 8) * 128u;
            int pv_issued = 0;

            // ---- P tile tt to the PV product (its A_V tile is converted by the helpers)
            auto handoff = [&](int tt) {
                tc::fence_async_smem();
                const int pb = g.dbl ? (tt & 1) : 0;
                tc::mbar_arrive(&sm.p_full[pb]);
                pf.inc(pb);
                ++pv_issued;
            };

            // ---- no spare rank row: column sums of the rounded P by a transposing
            // butterfly; lanes 2c and 2c+1 end with column c of the 16
            auto colsum = [&](const uint32_t (&pk)[8], int ch) {
                float sv[16];
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float2 pr = __half22float2(*reinterpret_cast<const __half2 *>(&pk[v]));
                    sv[2 * v] = pr.x;
                    sv[2 * v + 1] = pr.y;
                }
#pragma unroll
                for (int sz = 8, bit = 16; sz >= 1; sz >>= 1, bit >>= 1) {
                    const bool hi = lane & bit;
#pragma unroll
                    for (int j = 0; j < sz; ++j) {
                        const float send = hi ? sv[j] : sv[j + sz];
                        const float keep = hi ? sv[j + sz] : sv[j];
                        sv[j] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
                    }
                }
                sv[0] += __shfl_xor_sync(0xffffffffu, sv[0], 1);
                if (!(lane & 1)) atomicAdd(&sm.lsum[ch + ((lane >> 1) & 15)], sv[0]);
            };

            // ---- rare path: some p of columns [c0, c0 + w) exceeded 2^8 (or
            // overflowed).  Raise those columns' reference max to this tile's
            // maxima (raw scores reloaded from TMEM) and rescale the running
            // O_A^T and sums; the caller recomputes p.
            auto rescale = [&](int c0, int w, uint32_t dcol, int lim) -> bool {
                if (!p_drain(0) || !p_drain(1)) return false;   // every P handed over has been used
                if (gt < w) sm.cmax[c0 + gt] = ord_enc(-INFINITY);
                grp_sync_rt(bar_id);
                for (int h = 0; h < w; h += 16) {   // column maxima over the tile's live rows
                    uint32_t r[16];
                    tc::tmem_ld16(dcol + c0 + h, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        float x = h + v < lim ? __uint_as_float(r[v]) * kscale : -INFINITY;
                        for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                        if (lane == 0) atomicMax(&sm.cmax[c0 + h + v], ord_enc(x));
                    }
                }
                grp_sync_rt(bar_id);
                if (gt < w) {
                    const int c = c0 + gt;
                    const float cn = fmaxf(sm.cref[c], ord_dec(sm.cmax[c]));
                    const float f = dt_ex2(sm.cref[c] - cn);
                    sm.cscale[c] = f;
                    sm.cref[c] = cn;
                    sm.lsum[c] *= f;
                }
                grp_sync_rt(bar_id);
                if (pv_issued > 0) {   // O_A^T columns (every rank lane) times 2^(cref_old - cref_new)
                    tc::tc_fence_after();
                    for (int h = 0; h < w; h += 16) {
                        uint32_t o[16];
                        tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0 + h, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t wv[8];
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                wv[v] = __float_as_uint(__uint_as_float(o[8 * hh + v]) * sm.cscale[c0 + h + 8 * hh + v]);
                            tc::tmem_st8(tmem + DT_COL_OA + lane_off + c0 + h + 8 * hh, wv);
                        }
                    }
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                }
                return true;
            };

            // ---- softmax of score tile t over this group's slabs:
            // p = 2^(x - cref), fp16, MN-major [t/8][q/8][t%8][q%8]
            auto softmax = [&](int t) -> bool {
                const int d2b = g.dbl ? (t & 1) : 0;
                const uint32_t dcol = tmem + DT_COL_D2 + 64 * d2b + lane_off;
                if (!grp_and_rt(bar_id, tc::mbar_wait(&sm.d2_full[d2b], u2[d2b] & 1u, lim))) return false;
                u2.inc(d2b);
                MILO_TL(TL_S_START, n, t);
                tc::tc_fence_after();
                const int tok = t * FTILE + row;
                const bool valid = tok < Tb;
                if (t == 0) {   // reference max: the scores of the item's first token
                    for (int c0 = 32 * sg; c0 < nq16; c0 += 64) {
                        const int w = min(32, nq16 - c0);
                        if (gt < w) sm.lsum[c0 + gt] = 0.f;
                        if (quad == 0)
                            for (int h = 0; h < w; h += 16) {
                                uint32_t r[16];
                                tc::tmem_ld16(dcol + c0 + h, r);
                                tc::tmem_wait_ld();
                                if (lane == 0)
#pragma unroll
                                    for (int v = 0; v < 16; ++v) sm.cref[c0 + h + v] = __uint_as_float(r[v]) * kscale;
                            }
                    }
                    grp_sync_rt(bar_id);
                }
                const int pb = g.dbl ? (t & 1) : 0;
                uint8_t *pbase = sm.pbuf + pb * 16384 + (row >> 3) * lbo_p + (row & 7) * 16;
                // the P buffer's previous product has completed (at an item's start
                // both halves: the previous item may have used it at another width)
                auto drain = [&]() -> bool {
                    if (t == 0) return p_drain(0) && p_drain(1);
                    return p_drain(pb);
                };
                bool p_ready = false;
                for (int c0 = 32 * sg; c0 < nq16; c0 += 64) {
                    const int w = min(32, nq16 - c0);
                    const int lim = valid ? min(w, nq - c0) : 0;   // this token's live columns
                    // raw scores; p = 2^(x - cref) packed to fp16 pairs in place (pk[v] <-
                    // columns 2v, 2v+1).  More than 2^8 (or an overflow) sends the slab
                    // down the rare path, which recomputes it.
                    uint32_t pk[32];
                    tc::tmem_ld16(dcol + c0, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                    if (w == 32) tc::tmem_ld16(dcol + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
                    tc::tmem_wait_ld();
                    if (c0 == 32 * sg) MILO_TL(TL_S_LOADED, n, t);
                    auto make_p = [&](float &pmax) {
                        const float2 *c2 = reinterpret_cast<const float2 *>(sm.cref + c0);
#pragma unroll
                        for (int v = 0; v < 16; ++v) {
                            if (2 * v >= w) break;
                            const float2 cr = c2[v];
                            float e0 = dt_ex2(__uint_as_float(pk[2 * v]) * kscale - cr.x);
                            float e1 = dt_ex2(__uint_as_float(pk[2 * v + 1]) * kscale - cr.y);
                            e0 = 2 * v < lim ? e0 : 0.f;
                            e1 = 2 * v + 1 < lim ? e1 : 0.f;
                            pmax = fmaxf(pmax, fmaxf(e0, e1));
                            const __half2 hb = __floats2half2_rn(e0, e1);
                            pk[v] = *reinterpret_cast<const uint32_t *>(&hb);
                        }
                    };
                    float pmax = 0.f;
                    make_p(pmax);
                    const bool any_over = grp_or_rt(bar_id, !(pmax <= 256.f));
                    if (c0 == 32 * sg) MILO_TL(TL_S_MADE, n, t);
                    if (any_over) {
                        MILO_TL(TL_S_RESCALE, n, t);
                        if (!rescale(c0, w, dcol, lim)) return false;
                        tc::tmem_ld16(dcol + c0, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                        if (w == 32) tc::tmem_ld16(dcol + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
                        tc::tmem_wait_ld();
                        float pm2 = 0.f;
                        make_p(pm2);
                    }
                    if (!p_ready) {
                        if (!drain()) return false;
                        p_ready = true;
                        MILO_TL(TL_S_PFREE, n, t);
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (16 * hh >= w) break;
                        const int ch = c0 + 16 * hh;
                        const uint32_t(&q8)[8] = *reinterpret_cast<const uint32_t(*)[8]>(&pk[8 * hh]);
                        uint8_t *dst = pbase + (ch >> 3) * 128;
                        *reinterpret_cast<uint4 *>(dst) = make_uint4(q8[0], q8[1], q8[2], q8[3]);
                        *reinterpret_cast<uint4 *>(dst + 128) = make_uint4(q8[4], q8[5], q8[6], q8[7]);
                        if (!g.ones) colsum(q8, ch);
                    }
                }
                // every score of the tile this thread needed has been read
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.d2_empty[d2b]);
                // a group without slabs keeps the same drain sequence
                if (!p_ready && !drain()) return false;
                MILO_TL(TL_S_END, n, t);
                return true;
            };

            for (int t = 0; t < g.nt && ok; ++t) {
                ok = softmax(t);
                if (ok) handoff(t);
            }
            if (!ok) break;

            // ---- O_A^T finished: denominators, O_A / l to fp16 staging (this
            // group's columns); the last product and its read-out are the RoPE group's
            ok = grp_and_rt(bar_id, tc::mbar_wait(&sm.oa_full, n & 1u, lim));
            if (!ok) break;
            MILO_TL(TL_S_OA, n, 0);
            tc::tc_fence_after();
            if (g.ones && quad == (g.R8V >> 5)) {   // the ones row holds sum_t p
                for (int c0 = 32 * sg; c0 < nq16; c0 += 64)
                    for (int h = 0; h < min(32, nq16 - c0); h += 16) {
                        uint32_t r[16];
                        tc::tmem_ld16(tmem + DT_COL_OA + lane_off + c0 + h, r);
                        tc::tmem_wait_ld();
                        if (row == g.R8V)
#pragma unroll
                            for (int v = 0; v < 16; ++v) sm.lsum[c0 + h + v] = __uint_as_float(r[v]);
                    }
            }
            grp_sync_rt(bar_id);
            for (int c0 = 32 * sg; c0 < nq16; c0 += 64) {
                const int c = c0 + gt;
                if (gt < min(32, nq16 - c0)) sm.cscale[c] = (c < nq && sm.lsum[c] > 0.f) ? __frcp_rn(sm.lsum[c]) : 0.f;
            }
            const int pst = g.dbl ? (g.nt & 1) : 0;
            if (!p_drain(pst)) { ok = false; break; }
            grp_sync_rt(bar_id);
            if (quad * 32 < g.R16V) {
                uint8_t *sbase = sm.pbuf + pst * 16384 + (row >> 3) * lbo_p + (row & 7) * 16;
                for (int c0 = 32 * sg; c0 < nq16; c0 += 64)
                    for (int ch = c0; ch < min(c0 + 32, nq16); ch += 16) {
                        uint32_t r[16];
                        tc::tmem_ld16(tmem + DT_COL_OA + lane_off + ch, r);
                        tc::tmem_wait_ld();
                        if (row < g.R16V) {
                            uint32_t q8[8];
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                const __half2 h2 = __floats2half2_rn(__uint_as_float(r[2 * v]) * sm.cscale[ch + 2 * v],
                                                                     __uint_as_float(r[2 * v + 1]) * sm.cscale[ch + 2 * v + 1]);
                                q8[v] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                            uint8_t *dst = sbase + (ch >> 3) * 128;
                            *reinterpret_cast<uint4 *>(dst) = make_uint4(q8[0], q8[1], q8[2], q8[3]);
                            *reinterpret_cast<uint4 *>(dst + 128) = make_uint4(q8[4], q8[5], q8[6], q8[7]);
                        }
                    }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.p_full[pst]);
            pf.inc(pst);
            // the reference max and the sum of this group's queries
            for (int c0 = 32 * sg; c0 < nq16; c0 += 64) {
                const int c = c0 + gt;
                if (gt < min(32, nq16 - c0) && c < nq)
                    a.part_ml[sm.qpidx[n & 3u][c]] = make_float2(sm.cref[c] * 0.69314718055994531f, sm.lsum[c]);
            }
            // one group-wide decision per item (also orders this item's reads of
            // cref / lsum before the next item's writes)
            ok = grp_and_rt(bar_id, !sm.abort);
            MILO_TL(TL_S_DONE, n, 0);
        }
        if (!ok) sm.abort = 1;
    } else {
        // ================================================================ helper warps
        const int et = threadIdx.x - 32 * DT_W_H;
        bool ok = true;
        // ---- rotated queries R(-p) q of item j, fp16, K-major [q/8][j/8][q%8][j%8];
        // four threads per query, 16 pairs each
        auto qprep = [&](int64_t j, uint32_t nj) -> bool {
            if (!grp_and<DT_BAR_H, DT_HELP>(tc::mbar_wait(&sm.q_empty, (nj & 1u) ^ 1u, lim))) return false;
            MILO_TL(TL_H_Q_START, nj, 0);
            const int nq = __ldg(&items[j].nq), nq16 = (nq + 15) & ~15;
            const int jl = __ldg(&items[j].l), jh = __ldg(&items[j].h), jq0 = __ldg(&items[j].q0);
            const int jslot0 = __ldg(&items[j].slot0);
            for (int u = et; u < 4 * nq16; u += DT_HELP) {
                const int qi = u >> 2, part = u & 3;          // pairs 16*part .. 16*part+15
                uint8_t *qrow = sm.qt + (qi >> 3) * 2048 + (qi & 7) * 16;
                if (qi < nq) {
                    const int gq = jq0 + qi;
                    const int slot = a.slot_list[jslot0 + gq / a.G];
                    const int g = gq % a.G;
                    const int s = slot / a.n_sel, jj = slot % a.n_sel;
                    const int hq = jh * a.G + g;
                    const int64_t qbase = ((int64_t)jl * a.S + s) * a.Hq + hq;
                    const float4 *qv = reinterpret_cast<const float4 *>(a.q + qbase * D);
                    const float4 *cs = reinterpret_cast<const float4 *>(a.rope_q + (int64_t)slot * HALF);
                    if (part == 0) sm.qpidx[nj & 3u][qi] = (int)(qbase * a.n_sel + jj);
#pragma unroll 1
                    for (int h8 = 0; h8 < 2; ++h8) {          // pairs 16*part + 8*h8 .. +7
                        const int p0 = 16 * part + 8 * h8;
                        const float4 xa0 = qv[p0 / 4], xa1 = qv[p0 / 4 + 1];
                        const float4 xb0 = qv[16 + p0 / 4], xb1 = qv[16 + p0 / 4 + 1];
                        float4 cv[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) cv[k] = cs[p0 / 2 + k];
                        const float x0[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
                        const float x1[8] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w};
                        uint32_t lo[4], hi[4];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const float4 c2 = cv[v];   // (cos, sin) of pairs p0 + 2v, p0 + 2v + 1
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
            tc::mbar_arrive(&sm.q_full);
            return true;
        };

        // Two independent streams, served whichever is ready: the ring tiles
        // in order (A_K tiles pass, A_V tiles and B_V to fp16 in place), and
        // each next item's queries once the current item's scores are done.
        // Each stream's item is kPend until the producer has claimed it, -1 once
        // none is left.
        constexpr int64_t kPend = -2;
        int64_t ic = kPend, iq = kPend;
        uint32_t seqC = 0, nc = 0, nqp = 0;
        int kc = 0;
        DtGeo gc = dt_geo(1, 0, 0, 0);
        uint64_t t_last = tc::globaltimer();
        uint32_t backoff = 64;
        while (ok) {
            if (ic == kPend && grp_and<DT_BAR_H, DT_HELP>(item_ready(nc))) {
                ic = item_at(nc);
                if (ic >= 0) gc = dt_geo(items, ic, n_items);
            }
            if (iq == kPend && grp_and<DT_BAR_H, DT_HELP>(item_ready(nqp))) iq = item_at(nqp);
            if (ic == -1 && iq == -1) break;
            bool did = false;
            if (ic >= 0) {
                int tt;
                const int kind = dt_tile_at(gc.nt, kc, &tt);
                const uint32_t k = seqC + kc, s = k % DT_NBAR;
                bool go = kind == 0;
                if (!go) go = grp_and<DT_BAR_H, DT_HELP>(mbar_test(&sm.full[s], (k / DT_NBAR) & 1u));
                if (go) {
                    if (kind != 0 && !a.f16) {
                        bf16_to_f16_inplace(sm.ring + sm.toff[s], gc.R8V * 16, et, DT_HELP);
                        tc::fence_async_smem();
                        grp_sync<DT_BAR_H, DT_HELP>();
                    }
                    if (et == 0) tc::mbar_arrive(&sm.conv[s]);
                    MILO_TL(TL_H_CONV, nc, kc);
                    if (++kc == dt_ring_tiles(gc)) {
                        seqC += dt_ring_tiles(gc);
                        kc = 0;
                        ++nc;
                        ic = kPend;
                    }
                    did = true;
                }
            }
            if (iq >= 0 && grp_and<DT_BAR_H, DT_HELP>(mbar_test(&sm.q_empty, (nqp & 1u) ^ 1u))) {
                ok = qprep(iq, nqp);
                MILO_TL(TL_H_Q_END, nqp, 0);
                ++nqp;
                iq = kPend;
                did = true;
            }
            if (did) {
                t_last = tc::globaltimer();
                backoff = 64;
            } else {
                const bool stop = grp_or<DT_BAR_H, DT_HELP>(sm.abort || tc::globaltimer() - t_last > lim);
                if (stop) {
                    if (!sm.abort) raise_status(ST_TIMEOUT);
                    ok = false;
                }
                __nanosleep(backoff);
                backoff = min(backoff * 2, 256u);
            }
        }
        if (!ok) sm.abort = 1;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, DT_TMEM_COLS);
}

// Element sizes (the bf16 layout of common.cuh) of every block, for the fp16
// copy of 2-bit factors; scanned into its element offsets.  grid over nblk.
__global__ void k_elem_sizes(const int32_t *__restrict__ ranks, int64_t nblk, int n_b, BlockGeo geo,
                             int64_t *__restrict__ sizes) {
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblk;
         blk += (int64_t)gridDim.x * blockDim.x)
        sizes[blk] = block_elems(ranks[blk], geo.len((int)(blk % n_b)));
}

// 2-bit factors for the tensor cores: the selected blocks' A codes as zero +
// code * scale of their (rank, 32-token group) and B's INT8 codes times the
// channel scale, rounded to fp16, written at the element offsets eoff of the
// bf16 layout into `out` (one section per kind).  Grid (L*H*n_b, 2); blocks no
// slot selected are skipped.
__global__ void __launch_bounds__(256) k_dequant_int2(DecodeArgs a, const int64_t *__restrict__ eoff0,
                                                      const int64_t *__restrict__ eoff1, __half *out0,
                                                      __half *out1) {
    const int64_t blk = blockIdx.x;
    const int kind = blockIdx.y;
    const int b = (int)(blk % a.n_b);
    if (a.slot_start[b + 1] == a.slot_start[b]) return;
    const KindView &kv = a.kv[kind];
    const int R8 = rank_pad(kv.ranks[blk]);
    if (R8 == 0) return;
    const int nt = token_tiles(BlockGeo{a.T, a.block_len, a.starts}.len(b));
    const int64_t nA = (int64_t)nt * R8 * FTILE, nAll = nA + (int64_t)R8 * D;
    const uint8_t *src = (const uint8_t *)kv.data + kv.offsets[blk];
    __half *dst = (kind ? out1 : out0) + (kind ? eoff1 : eoff0)[blk];
    const __half2 *prm = reinterpret_cast<const __half2 *>(src + int2_param_off(R8, nt));
    const float *sB = kv.scaleB + blk * D;
    for (int64_t e = (int64_t)threadIdx.x * 8; e < nAll; e += 256 * 8) {   // one core-matrix row
        float v[8];
        if (e < nA) {   // A tile: [k/8][u/8][k%8][u%8], eight tokens of rank k
            const int tau = (int)(e / (R8 * FTILE));
            const int r = (int)(e % (R8 * FTILE));
            const int k = (r >> 10) * 8 + ((r >> 3) & 7), t0 = tau * FTILE + ((r >> 6) & 15) * 8;
            const float2 sz = __half22float2(prm[(int64_t)k * (4 * nt) + t0 / INT2_GROUP]);   // (scale, zero)
            const uint32_t codes = *reinterpret_cast<const uint16_t *>(src + (e >> 2));
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = fmaf((float)((codes >> (2 * i)) & 3u), sz.x, sz.y);
        } else {        // B: [k/8][j/8][k%8][j%8], INT8 codes of eight channels
            const int64_t r = e - nA;
            const int j0 = (int)((r & 1023) >> 6) * 8;
            const uint2 q8 = *reinterpret_cast<const uint2 *>(src + int2_b_off(R8, nt) + r);
            const int8_t *c = reinterpret_cast<const int8_t *>(&q8);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = (float)c[i] * sB[j0 + i];
        }
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
            ow[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(dst + e) = o;
    }
}

inline size_t decode_tc_smem_bytes() { return sizeof(DecTcSmem) + 128; }

inline bool decode_tc_supported(const DecodeArgs &a) {
    if (getenv("MILO_FORCE_SIMT") && a.factor_dtype != MILO_INT2) return false;   // 2-bit: no CUDA-core path
    return (a.factor_dtype == MILO_BF16 || a.factor_dtype == MILO_INT8 || a.factor_dtype == MILO_INT2) &&
           a.block_len <= 512;
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
    const int Tb = BlockGeo{a.T, a.block_len, a.starts}.len(b);
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
