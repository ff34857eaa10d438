/*
 * milo.h -- C ABI of libmilo: block-wise low-rank compression of a many-shot
 * KV cache and decode attention over the compressed blocks, on one NVIDIA
 * B200 (sm_100a).
 *
 * The operations follow "MILO: Efficient Many-shot In-Context Learning with
 * Block-wise Low-rank Compression":
 *   - evolve.pub review, Summary: the cache is split into blocks of several
 *     demonstrations; K (taken before RoPE) and V are each decomposed by SVD
 *     per block; per-block ranks maximise sum log(1 + sigma^2/eps^2) under a
 *     global rank budget, chosen greedily (Eqs 5-7); at inference a
 *     retriever picks blocks whose low-rank factors are rebuilt before
 *     sparse attention.
 *   - same page, Strengths "Principled, budget-feasible rank allocation":
 *     greedy marginal gains log(1 + sigma^2/eps^2) under a global budget.
 *   - same page, FAQ "What is MILO": the cache is stored in compressed
 *     low-rank form per block and only the blocks a query needs are rebuilt.
 *   - shd-paper mirror, original abstract: each block holds several
 *     many-shot examples; rank budgets follow each block's information
 *     entropy.
 *
 * Conventions for every call:
 *   - Pointers documented as "device" point to memory of the current CUDA
 *     device; "host" pointers to ordinary host memory.  The caller owns and
 *     allocates every buffer (sizes come from the *_size queries); libmilo
 *     allocates no device memory.
 *   - Calls are asynchronous on the given stream and never synchronise the
 *     host, except milo_get_status, milo_factors_export and
 *     milo_factors_import, which say so.  Argument errors are returned
 *     synchronously and launch nothing.  Errors found on the device (a
 *     Jacobi sweep cap reached, non-finite input, a bad block id, a wait on
 *     the device that ran out) set bits
 *     of a per-device status word that milo_get_status reads and clears.
 *   - No C++ exception crosses this interface.
 *   - d (head dimension) must be 128.
 */
#ifndef MILO_H_
#define MILO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *milo_stream_t;

typedef enum {
    MILO_OK = 0,
    MILO_WARN_NOT_CONVERGED = 1,   /* a Jacobi eigensolve hit its sweep cap  */
    MILO_ERR_INVALID_ARG = -1,     /* bad pointer, size, shape or budget      */
    MILO_ERR_UNSUPPORTED = -2,     /* d != 128, dtype not supported here      */
    MILO_ERR_CUDA = -3,            /* a CUDA runtime call failed              */
    MILO_ERR_WORKSPACE = -4,       /* workspace or arena smaller than needed  */
    MILO_ERR_NONFINITE = -5,       /* NaN/Inf met on the device               */
    MILO_ERR_BOUNDS = -6,          /* an index out of range met on the device */
    MILO_ERR_TIMEOUT = -7          /* a bounded wait on the device ran out    */
} milo_status;

/* MILO_INT2: factor codes only (A_b in 2 bits per element, B_b in INT8; see
 * the arena layout below). */
typedef enum { MILO_F32 = 0, MILO_BF16 = 1, MILO_INT8 = 2, MILO_INT2 = 3 } milo_dtype;

/* A KV cache of one kind: [L][H][T][d] row-major (d contiguous). */
typedef struct {
    int32_t L;          /* layers                                        */
    int32_t H;          /* KV heads per layer                            */
    int32_t T;          /* tokens per (layer, head)                      */
    int32_t d;          /* head dimension; must be 128                   */
    int32_t block_len;  /* tokens per block (>= 1); the last may be short;
                           with block_starts: the longest block's tokens */
    milo_dtype in_dtype;/* MILO_F32 or MILO_BF16                         */
    /* Variable-length blocks, or 0 / NULL for fixed block_len.  Host array of
     * n_blocks + 1 token offsets shared by every (layer, head): block b =
     * tokens [block_starts[b], block_starts[b+1]); block_starts[0] = 0,
     * block_starts[n_blocks] = T, every length in [1, block_len].  Blocks
     * that each hold whole demonstrations ("MILO ... Block-wise Low-rank
     * Compression", shd-paper mirror, original abstract: each block holds
     * several many-shot examples).  The handle keeps its own copy, and the
     * arena a device copy (its `starts` array below).  With variable blocks
     * the Gram runs on CUDA cores (the tensor-core Gram needs whole
     * fixed-length blocks), and milo_compress copies the starts to the device
     * on its stream (a host-to-device copy from this array). */
    int32_t n_blocks;
    const int32_t *block_starts;
} milo_cache_shape;

typedef struct {
    /* Global rank budget R per kind (K and V have separate pools, each
     * global over all (layer, head, block)): budget_abs if > 0, else
     * floor(budget_frac * sum_b min(T_b, d)), evaluated in double. */
    double budget_frac;
    int64_t budget_abs;
    /* eps = eps_rel * max_b sigma_{b,1}; over the blocks of one
     * (layer, head, kind) when eps_scope == 0, over all of a kind when 1. */
    double eps_rel;
    int32_t eps_scope;
    /* Rank bounds per block: r_min <= r_b <= min(T_b, d, r_max or d). */
    int32_t r_min;
    int32_t r_max;                /* 0 means no cap beyond min(T_b, d) */
    milo_dtype factor_dtype;      /* MILO_F32, MILO_BF16, MILO_INT8 or MILO_INT2 */
    int32_t max_sweeps;           /* Jacobi sweep cap (0 -> 24)        */
    float jacobi_tol;             /* rotate while |g_pq| > tol*sqrt(g_pp g_qq) (0 -> 1e-7) */
} milo_compress_params;

/* Opaque host-side handle over a caller-owned factor arena. */
typedef struct milo_factors milo_factors;

/*
 * Factor arena layout (device, caller-owned, one section per kind: K then V,
 * each section start 256-byte aligned; N_blk = L*H*n_b, n_b = ceil(T /
 * block_len)):
 *   int32  starts [n_b + 1]     variable-length blocks: their token starts (unused otherwise)
 *   int32  ranks  [N_blk]
 *   int64  offsets[N_blk + 1]   element offset of block b in data (bytes for MILO_INT2)
 *   float  sigma  [N_blk][d]    singular values, descending
 *   double eps    [L*H]
 *   float  scaleA [N_blk][d]    INT8 only: scale of column k of A_b
 *   float  scaleB [N_blk][d]    INT8 and INT2: scale of column j of B_b
 *   elem   data   [...]         elem = factor dtype
 * A_b = U_r Sigma_r (T_b x r_b) and B_b = V_r^T (r_b x d), so X_b ~ A_b B_b.
 * Block b occupies R8 * (128 * nt + d) elements at data + offsets[b], with
 * R8 = round_up(r_b, 8) and nt = ceil(T_b / 128) token tiles; blocks are
 * ordered (l, h, b).  Rank rows r_b .. R8-1 and tokens T_b .. 128*nt-1 are
 * zero.  Inside a block, with t = 128*tau + u:
 *   A_b[t][k] at  tau*R8*128 + (k/8)*1024 + (u/8)*64 + (k%8)*8 + (u%8)
 *   B_b[k][j] at  nt*R8*128  + (k/8)*1024 + (j/8)*64 + (k%8)*8 + (j%8)
 * i.e. 8 x 8 element tiles, the tensor cores' canonical no-swizzle operand
 * layout, so that each 128-token tile of A_b and the whole of B_b are single
 * contiguous copies.  The data section holds at most
 * (R + 7 N_blk) * (128 * ceil(block_len / 128) + d) elements.
 *
 * MILO_INT2 (evolve.pub review, Summary and Key claims: MILO composes with
 * KIVI-style low-bit codes): A_b in 2-bit asymmetric codes per rank column k
 * and group of 32 tokens g -- zero z = the group's min, scale s = (max - min)
 * / 3, both fp16, code = clamp(rint((a - z) / s), 0, 3) in fp32 (0 when s =
 * 0), a = z + code * s -- and B_b in INT8 as above.  Block b occupies
 * R8 * (48 * nt + d) bytes: the codes of A_b at byte (index of A_b[t][k]
 * above) / 4, bits 2*(u%4) (four consecutive tokens per byte); B_b's INT8
 * codes at byte nt*R8*32 + (index of B_b[k][j] above) - nt*R8*128; then the
 * (s, z) fp16 pairs at byte nt*R8*32 + R8*d + 4 * (k * 4*nt + t / 32).
 */

/* ----------------------------------------------------------------- sizes */

/* Bytes of the factor arena for this shape and params (both kinds); 0 on
 * invalid input. */
size_t milo_factor_arena_size(const milo_cache_shape *shape, const milo_compress_params *params);

/* Bytes of scratch milo_compress needs; 0 on invalid input. */
size_t milo_compress_workspace_size(const milo_cache_shape *shape, const milo_compress_params *params);

/* R per kind for this shape and params (the formula above); -1 if invalid. */
int64_t milo_rank_budget(const milo_cache_shape *shape, const milo_compress_params *params);

/* Fill params with the defaults: budget_frac 0.5, eps_rel 1e-2, scope 0,
 * r_min 0, r_max 0, factor dtype BF16, 24 sweeps, tol 1e-7. */
void milo_default_params(milo_compress_params *params);

/* -------------------------------------------------------------- compress */

/*
 * Compress one cache (both kinds).  K_preRoPE and V: device, [L][H][T][d] in
 * shape->in_dtype, read only.  workspace: device, >= ws_bytes of
 * milo_compress_workspace_size.  arena: device, >= milo_factor_arena_size,
 * 256-byte aligned, filled in the layout above.  On MILO_OK *out receives a
 * new handle (host memory, free with milo_factors_destroy) whose views point
 * into arena.  Steps, in order and per kind: per-block Gram X_b^T X_b
 * (tensor cores for bf16), Jacobi eigensolve (sigma, right singular vectors),
 * eps, global top-R selection of the gains, ranks and offsets, projection
 * A_b = X_b W_{:,1:r_b} and packing.  Asynchronous on stream.
 */
milo_status milo_compress(const milo_cache_shape *shape, const void *K_preRoPE, const void *V,
                          const milo_compress_params *params, void *workspace, size_t ws_bytes,
                          void *arena, size_t arena_bytes, milo_factors **out, milo_stream_t stream);

/* -------------------------------------------------------------- allocate */

/* Bytes of scratch milo_allocate needs for n_blk = n_groups * n_b blocks. */
size_t milo_allocate_workspace_size(int32_t n_groups, int32_t n_b, int32_t d);

/*
 * Greedy entropy-gain rank allocation for one kind (the Eqs 5-7 reading):
 * choose ranks r_b, sum_b r_b = R, r_min_b = min(r_min, cap_b) <= r_b <=
 * cap_b = min(T_b, d, r_max or d), maximising sum_b sum_{k<r_b}
 * log(1 + sigma_{b,k}^2/eps_g^2).  Decided exactly by the global top
 * (R - sum r_min_b) keys (sigma/eps)^2 in double (one division, one
 * multiply, IEEE), ties to the lower linear index (group, block, k); this
 * equals the greedy rule when sigma is non-increasing in k.
 *   sigma:  device, float [n_groups*n_b][d], non-increasing within a block
 *   eps:    device, double [n_groups] (eps <= 0 makes every key 0)
 *   T, block_len: block b of a group has T_b = min(block_len, T - b*block_len)
 *   ranks_out: device, int32 [n_groups*n_b]
 * MILO_ERR_INVALID_ARG if R is outside [sum r_min_b, sum cap_b].
 */
milo_status milo_allocate(const float *sigma, const double *eps, int32_t n_groups, int32_t n_b,
                          int32_t d, int32_t T, int32_t block_len, int64_t R, int32_t r_min,
                          int32_t r_max, int32_t *ranks_out, void *workspace, size_t ws_bytes,
                          milo_stream_t stream);

/* Largest n_groups * n_b that milo_allocate_noalloc accepts. */
#define MILO_NOALLOC_MAX_BLOCKS 65536

/*
 * milo_allocate for callers that cannot allocate device memory: code that
 * runs under a framework owning every device byte through its own pool, or
 * a plug-in operator that is handed only its inputs and outputs.  The paper
 * has no counterpart; it is a deployment convenience.  Same arguments,
 * result and errors as milo_allocate, minus the workspace: the scratch is a
 * fixed device array inside the library (about 1 MiB, held on every device
 * that loads the library until the process exits).
 *   - n_groups * n_b > MILO_NOALLOC_MAX_BLOCKS: MILO_ERR_WORKSPACE (the
 *     built-in scratch is too small), nothing is launched.
 *   - The first call on a device looks up the array's device address (host
 *     set-up, no allocation); make that first call before any stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (on
 *     different streams, or from different threads) race and give wrong
 *     ranks.  Calls in one stream are ordered and safe.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library.
 */
milo_status milo_allocate_noalloc(const float *sigma, const double *eps, int32_t n_groups, int32_t n_b,
                                  int32_t d, int32_t T, int32_t block_len, int64_t R, int32_t r_min,
                                  int32_t r_max, int32_t *ranks_out, milo_stream_t stream);

/* ---------------------------------------------------------------- decode */

/* Bytes of scratch milo_decode_attn needs. */
size_t milo_decode_workspace_size(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel);

/*
 * GQA decode attention over retrieved compressed blocks, all layers in one
 * call.  For layer l, session s, query head hq (KV head hq / (Hq/H)), the
 * output is softmax over every token of the selected blocks of
 *   s_t = q . RoPE(a^K_t B_K, p_j + t) / sqrt(d),
 * times the rebuilt values a^V_t B_V; keys are rebuilt and rotated per token
 * (rotate-half pairs (i, i+64), theta_i = rope_base^(-2i/d)) and never
 * written to memory.
 *   q:        device, float [L][S][Hq][d], already rotated to its position
 *   selected: device, int32 [S][n_sel] block ids (0 <= id < n_b), shared by
 *             all layers and heads
 *   positions:device, int32 [S][n_sel] start position of each selected
 *             block, or NULL for id * block_len
 *   out:      device, float [L][S][Hq][d]
 * Hq must be a multiple of H.  Block ids out of range set MILO_ERR_BOUNDS in
 * the status word and contribute nothing.
 */
milo_status milo_decode_attn(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                             const int32_t *selected, const int32_t *positions, int32_t n_sel,
                             double rope_base, float *out, void *workspace, size_t ws_bytes,
                             milo_stream_t stream);

/* Bytes of scratch milo_decode_attn_tail needs (milo_decode_workspace_size
 * plus one partial per query row). */
size_t milo_decode_tail_workspace_size(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel);

/*
 * milo_decode_attn plus each session's recent, uncompressed tokens in the
 * same softmax: a complete decode step.  "MILO ... Block-wise Low-rank
 * Compression" (evolve.pub review), Summary and FAQ "What is MILO": the
 * compressed cache holds the many-shot demonstrations, a query rebuilds the
 * blocks it retrieves and attends sparsely; the tokens that follow the
 * demonstrations (the question, the tokens generated so far) stay
 * uncompressed and are attended densely.  For (l, s, hq) the output is
 * softmax over the selected blocks' tokens (as in milo_decode_attn) and the
 * tail tokens i < tail_len[s] with s_i = q . k_tail[l][s][hq / G][i] / sqrt(d),
 * times v_tail[l][s][hq / G][i].
 *   k_tail, v_tail: device, 16-byte aligned, [L][S][H][tail_cap][d] of
 *             tail_dtype (MILO_F32 or MILO_BF16; else MILO_ERR_UNSUPPORTED);
 *             keys already rotated to their own positions (as a model caches
 *             them), values plain
 *   tail_len: device, int32 [S], 0 <= tail_len[s] <= tail_cap; a length
 *             outside that range sets MILO_ERR_BOUNDS in the status word and
 *             counts as an empty tail
 * Other arguments, errors and the workspace rule as milo_decode_attn, with
 * ws_bytes >= milo_decode_tail_workspace_size.  An empty tail for every
 * session gives milo_decode_attn's output bit for bit.
 */
milo_status milo_decode_attn_tail(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                                  const int32_t *selected, const int32_t *positions, int32_t n_sel,
                                  double rope_base, const void *k_tail, const void *v_tail, milo_dtype tail_dtype,
                                  int32_t tail_cap, const int32_t *tail_len, float *out, void *workspace,
                                  size_t ws_bytes, milo_stream_t stream);

/* Bytes of scratch milo_decode_attn_offload and milo_decode_attn_offload_tail
 * need: milo_decode_tail_workspace_size plus a staging area that holds every
 * block's factors at most. */
size_t milo_decode_offload_workspace_size(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel);

/*
 * milo_decode_attn for factors kept in host memory: the handle's arena
 * (from milo_factors_wrap over a copy of a compressed arena) lives in pinned,
 * device-mapped host memory.  Each call copies the factors (and INT8 scales)
 * of the blocks some session selected into the workspace's staging area over
 * the host link, then decodes there; the output equals milo_decode_attn on a
 * device copy of the same arena bit for bit.  "MILO ... Block-wise Low-rank
 * Compression" (evolve.pub review), Summary and FAQ "How much memory saving
 * and speedup does MILO achieve?": the pages measure MILO against offloading
 * the full KV cache to CPU memory; only the retrieved blocks' factors move.
 * Arguments, errors and the result as milo_decode_attn, with ws_bytes >=
 * milo_decode_offload_workspace_size; an arena in pageable host memory gives
 * MILO_ERR_INVALID_ARG before any launch.
 */
milo_status milo_decode_attn_offload(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                                     const int32_t *selected, const int32_t *positions, int32_t n_sel,
                                     double rope_base, float *out, void *workspace, size_t ws_bytes,
                                     milo_stream_t stream);

/* milo_decode_attn_offload plus each session's recent uncompressed tokens in
 * the same softmax (their arguments as milo_decode_attn_tail; the tail stays in
 * device memory), with ws_bytes >= milo_decode_offload_workspace_size: a
 * complete decode step from host-resident factors. */
milo_status milo_decode_attn_offload_tail(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                                          const int32_t *selected, const int32_t *positions, int32_t n_sel,
                                          double rope_base, const void *k_tail, const void *v_tail,
                                          milo_dtype tail_dtype, int32_t tail_cap, const int32_t *tail_len,
                                          float *out, void *workspace, size_t ws_bytes, milo_stream_t stream);

/* ---------------------------------------------------------------- retrieval */

/* Bytes of scratch milo_bm25_select needs. */
size_t milo_bm25_workspace_size(int32_t n_b, int32_t V, int32_t S);

/*
 * Block retrieval: Okapi BM25 scores of every block for every session's query
 * and each session's top n_sel blocks.  "MILO ... Block-wise Low-rank
 * Compression" (evolve.pub review), Summary: a query retrieves its relevant
 * blocks with BM25 and only those are rebuilt.  Scoring (Robertson and
 * Zaragoza 2009): idf(t) = ln(1 + (N - n_t + 0.5) / (n_t + 0.5)) over the
 * n_b blocks, and score(s, b) = sum over the block's terms t of
 * qtf_s(t) idf(t) tf(t,b) (k1 + 1) / (tf(t,b) + k1 (1 - beta + beta len_b / avgdl)),
 * fp64 with every operation rounded separately, terms added in row order.
 *   blk_ptr [n_b + 1], blk_term / blk_tf [nnz_b]: device, the blocks' term
 *             counts in CSR form (term ids in [0, V), each once per row,
 *             counts >= 1); blk_len [n_b]: tokens of each block
 *   q_ptr [S + 1], q_term / q_tf [nnz_q]: device, each session's query terms
 *             (each once per row, with its count)
 *   selected: device, int32 [S][n_sel] out: block ids by score descending,
 *             ties to the lower id (usable as milo_decode_attn's selection)
 *   scores:   device, fp64 [S][n_b] out, or NULL
 * 1 <= n_sel <= n_b, k1 >= 0, 0 <= beta <= 1.  Row pointers outside
 * [0, nnz] and term ids outside [0, V) set MILO_ERR_BOUNDS in the status word
 * and are clamped or skipped.
 */
milo_status milo_bm25_select(const int32_t *blk_ptr, const int32_t *blk_term, const int32_t *blk_tf,
                             const int32_t *blk_len, int32_t n_b, int32_t nnz_b, int32_t V, const int32_t *q_ptr,
                             const int32_t *q_term, const int32_t *q_tf, int32_t S, int32_t nnz_q, double k1,
                             double beta, int32_t n_sel, int32_t *selected, double *scores, void *workspace,
                             size_t ws_bytes, milo_stream_t stream);

/* ------------------------------------------------------ factor handles */

/* Views (device pointers into the arena) of one kind (0 = K, 1 = V).  Any
 * output pointer may be NULL.  R receives the kind's budget. */
milo_status milo_factors_get(const milo_factors *f, int32_t kind, int32_t **ranks, int64_t **offsets,
                             float **sigma, double **eps, void **data, float **scaleA,
                             float **scaleB, int64_t *R);

/* Wrap an arena already filled in the documented layout (for instance by
 * the caller; with variable blocks its starts array holds shape's
 * block_starts, as milo_compress writes it) in a new handle.  No device
 * access. */
milo_status milo_factors_wrap(const milo_cache_shape *shape, const milo_compress_params *params,
                              void *arena, size_t arena_bytes, milo_factors **out);

/* Serialise the handle's shape, params and arena into host_buf.  With
 * host_buf NULL only *bytes is set to the size needed.  Synchronises stream. */
milo_status milo_factors_export(const milo_factors *f, void *host_buf, size_t *bytes,
                                milo_stream_t stream);

/* Copy an exported blob into a caller-owned device arena (>= the arena size
 * recorded in the blob) and return a handle over it.  Synchronises stream. */
milo_status milo_factors_import(const void *host_buf, size_t bytes, void *arena, size_t arena_bytes,
                                milo_factors **out, milo_stream_t stream);

/* The handle's shape and params.  A variable-block shape's block_starts
 * points at the handle's own copy, valid while the handle lives.  Any
 * output may be NULL. */
milo_status milo_factors_shape(const milo_factors *f, milo_cache_shape *shape, milo_compress_params *params);

/* Free the handle only; the arena stays the caller's. */
void milo_factors_destroy(milo_factors *f);

/*
 * Test hook (no counterpart on the pages): arms a fault for the next
 * milo_decode_attn call that takes the tensor-core path, then disarms.
 *   mode 1: the kernel withholds the copy of the first work item's B_K (no
 *           copy is issued, so none is in flight), every wait on the device
 *           gives up after wait_ns nanoseconds (1 .. 2e9) instead of 2 s, and
 *           the call's status word reports MILO_ERR_TIMEOUT; the kernel
 *           still waits for its issued copies and products and frees its
 *           tensor memory before it returns, so later calls run normally.
 *   mode 0: disarm.
 * MILO_ERR_INVALID_ARG for another mode or an out-of-range wait_ns.
 */
milo_status milo_test_decode_inject(int32_t mode, uint64_t wait_ns);

/* ---------------------------------------------------------------- timing */

/*
 * Kernel timing (measurement; no counterpart on the pages).  While enabled,
 * the library brackets the kernels of each stage below with CUDA events on
 * the stream the stage is launched on, and sums their elapsed times.
 */
typedef enum {
    MILO_TK_GRAM = 0,        /* Gram matrices (k_gram_tc or k_gram_simt) */
    MILO_TK_JACOBI = 1,      /* one-sided Jacobi eigensolve (k_jacobi) */
    MILO_TK_REFINE = 2,      /* singular values recomputed from the blocks (k_refine_sigma) */
    MILO_TK_SELECT = 3,      /* eps and the global top-R rank selection */
    MILO_TK_PROJECT = 4,     /* projection and packing of A and B (k_project_a, k_project_b) */
    MILO_TK_DECODE_PREP = 5, /* decode index, table and query-packing kernels */
    MILO_TK_DECODE = 6,      /* decode attention (k_decode_tc or k_decode_simt) */
    MILO_TK_COMBINE = 7,     /* merge of the per-block partials (k_combine) */
    MILO_TK_TAIL = 8,        /* attention over the recent uncompressed tokens (k_tail_attn) */
    MILO_TK_STAGE = 9,       /* host-resident factors of the selected blocks staged on the device */
    MILO_TK_RETRIEVE = 10,   /* BM25 block scores and the per-session top blocks */
    MILO_TK_COUNT = 11
} milo_timed_stage;

/* on != 0: start recording (previous records are dropped); on == 0: stop.
 * Host-side only; the events are created on the current device. */
milo_status milo_timing_enable(int32_t on);

/* Wait for every recorded event, then write per stage (n entries, stage
 * order above; n <= MILO_TK_COUNT) the summed milliseconds into ms and the
 * number of bracketed launches into count, and drop the records.  ms and
 * count are host arrays.  MILO_ERR_INVALID_ARG for n outside 0 .. 8 or a NULL
 * array; a CUDA error of the event queries is returned as MILO_ERR_CUDA. */
milo_status milo_timing_read(double *ms, int64_t *count, int32_t n);

/* Synchronise stream, then read and clear the Jacobi work counters, summed
 * over every (block, kind) eigensolve since the last read: *rounds = rounds
 * that applied rotations (one round updates the d x d Gram tile and W for up
 * to 64 disjoint plane rotations), *rotations = plane rotations applied.
 * Either pointer may be NULL.  The eigensolve's work for its throughput. */
milo_status milo_jacobi_rounds(int64_t *rounds, int64_t *rotations, milo_stream_t stream);

/* ---------------------------------------------------------------- status */

/* Synchronise stream, then read and clear the current device's status word:
 * MILO_OK, MILO_WARN_NOT_CONVERGED, or the most severe device error. */
milo_status milo_get_status(milo_stream_t stream);

/* Static description of a status code. */
const char *milo_status_string(milo_status s);

/* Library version, "major.minor.patch". */
const char *milo_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MILO_H_ */
