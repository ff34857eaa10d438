// bm25.cuh -- block retrieval: Okapi BM25 scores of every block for every
// session's query, and each session's top n_sel blocks.
//
// "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression" (evolve.pub review), Summary: a query retrieves the relevant
// blocks of demonstrations with BM25 and only those are rebuilt.  The scoring
// function is the textbook Okapi BM25 (Robertson and Zaragoza, "The
// Probabilistic Relevance Framework: BM25 and Beyond", 2009):
//   idf(t)      = ln(1 + (N - n_t + 0.5) / (n_t + 0.5))
//   score(q, b) = sum over the block's terms t of
//                 qtf(t) idf(t) tf(t, b) (k1 + 1) / (tf(t, b) + k1 (1 - beta + beta |b| / avgdl))
// with N blocks, n_t of them containing t, |b| the block's tokens and avgdl
// their mean.  Blocks and queries are term-count tables (CSR rows: each term
// at most once per row, with its count).  Scores are fp64,
// every operation rounded separately (no fused multiply-add), the terms of a
// block added in row order.  Top n_sel by score, ties to the lower block id.
#pragma once
#include "common.cuh"

namespace milo {

struct Bm25Args {
    const int32_t *blk_ptr;    // [n_b + 1] CSR rows of the blocks' term counts
    const int32_t *blk_term;   // [nnz] term ids
    const int32_t *blk_tf;     // [nnz] counts (>= 1)
    const int32_t *blk_len;    // [n_b] tokens of each block
    const int32_t *q_ptr;      // [S + 1] CSR rows of the queries
    const int32_t *q_term;     // [nnz_q] term ids
    const int32_t *q_tf;       // [nnz_q] counts (>= 1)
    int n_b, V, S, n_sel;
    int nnz_b, nnz_q;          // entries of blk_term / q_term (row pointers are clamped to them)
    double k1, beta;
    int32_t *df;               // [V] workspace: blocks containing each term
    double *qw;                // [S][V] workspace: qtf(t) idf(t) of each session's terms, else 0
    double *avgdl;             // [1] workspace
    double *scores;            // [S][n_b]
    int32_t *selected;         // [S][n_sel]
};

// CSR row [lo, hi) clamped to [0, nnz]; a row outside raises ST_BOUNDS
__device__ __forceinline__ void bm25_row(const int32_t *ptr, int i, int nnz, int &lo, int &hi) {
    lo = ptr[i];
    hi = ptr[i + 1];
    if (lo < 0 || hi > nnz || lo > hi) {
        raise_status(ST_BOUNDS);
        lo = min(max(lo, 0), nnz);
        hi = max(lo, min(hi, nnz));
    }
}

// n_t of every term (a term id out of [0, V) raises ST_BOUNDS and is skipped)
__global__ void k_bm25_df(Bm25Args a) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < a.nnz_b; e += gridDim.x * blockDim.x) {
        const int t = a.blk_term[e];
        if (t < 0 || t >= a.V) {
            raise_status(ST_BOUNDS);
            continue;
        }
        atomicAdd(&a.df[t], 1);
    }
}

// avgdl: mean block length, summed in block order by one thread (n_b is small)
__global__ void k_bm25_avgdl(Bm25Args a) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    double sum = 0.0;
    for (int b = 0; b < a.n_b; ++b) sum = __dadd_rn(sum, (double)a.blk_len[b]);
    a.avgdl[0] = __ddiv_rn(sum, (double)a.n_b);
}

// qw[s][t] = qtf idf(t) for the session's query terms (qw zeroed before)
__global__ void k_bm25_qweights(Bm25Args a) {
    const int s = blockIdx.x;
    const double N = (double)a.n_b;
    int lo, hi;
    bm25_row(a.q_ptr, s, a.nnz_q, lo, hi);
    for (int e = lo + threadIdx.x; e < hi; e += blockDim.x) {
        const int t = a.q_term[e];
        if (t < 0 || t >= a.V) {
            raise_status(ST_BOUNDS);
            continue;
        }
        const double n = (double)a.df[t];
        const double idf = log1p(__ddiv_rn(__dadd_rn(__dsub_rn(N, n), 0.5), __dadd_rn(n, 0.5)));
        a.qw[(int64_t)s * a.V + t] = __dmul_rn((double)a.q_tf[e], idf);
    }
}

// score of every (session, block): one thread each, the block's terms in row order
__global__ void k_bm25_scores(Bm25Args a) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)a.S * a.n_b) return;
    const int s = (int)(i / a.n_b), b = (int)(i % a.n_b);
    const double k1 = a.k1;
    // k1 (1 - beta + beta |b| / avgdl)
    const double norm = __dmul_rn(k1, __dadd_rn(__dsub_rn(1.0, a.beta),
                                                 __ddiv_rn(__dmul_rn(a.beta, (double)a.blk_len[b]), a.avgdl[0])));
    const double *w = a.qw + (int64_t)s * a.V;
    double sc = 0.0;
    int lo, hi;
    bm25_row(a.blk_ptr, b, a.nnz_b, lo, hi);
    for (int e = lo; e < hi; ++e) {
        const int t = a.blk_term[e];
        if (t < 0 || t >= a.V) continue;
        const double wt = w[t];
        if (wt == 0.0) continue;   // not a query term: adds nothing
        const double tf = (double)a.blk_tf[e];
        sc = __dadd_rn(sc, __ddiv_rn(__dmul_rn(__dmul_rn(wt, tf), __dadd_rn(k1, 1.0)), __dadd_rn(tf, norm)));
    }
    a.scores[i] = sc;
}

// top n_sel of each session: the rank of block b is the number of blocks
// before it in (score descending, id ascending); one CTA per session
__global__ void k_bm25_topk(Bm25Args a) {
    const int s = blockIdx.x;
    const double *sc = a.scores + (int64_t)s * a.n_b;
    for (int b = threadIdx.x; b < a.n_b; b += blockDim.x) {
        const double x = sc[b];
        int rank = 0;
        for (int c = 0; c < a.n_b; ++c) {
            const double y = sc[c];
            rank += (y > x) || (y == x && c < b);
        }
        if (rank < a.n_sel) a.selected[(int64_t)s * a.n_sel + rank] = b;
    }
}

}  // namespace milo
