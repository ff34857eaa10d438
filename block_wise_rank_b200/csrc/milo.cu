// milo.cu -- libmilo: the C ABI (include/milo.h) and its launch sequences.
//
// One translation unit: the kernel headers below are included here so that
// the library has one device status word and needs no relocatable device
// code.  Every step of the path runs in these kernels; the host code only
// validates arguments, lays out caller-owned buffers and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>
#include <new>

#include "common.cuh"
#include "gram_simt.cuh"
#include "gram_tc.cuh"
#include "jacobi.cuh"
#include "refine.cuh"
#include "alloc.cuh"
#include "project_simt.cuh"
#include "decode_simt.cuh"
#include "decode_tc.cuh"
#include "decode_tail.cuh"
#include "decode_offload.cuh"
#include "bm25.cuh"

using namespace milo;

struct milo_factors {
    milo_cache_shape shape;        // shape.block_starts points at starts_host (or is null)
    milo_compress_params params;
    void *arena;
    size_t arena_bytes;
    int n_b;
    int64_t n_blk;
    int64_t R;
    KindView kv[2];
    int32_t *starts;               // variable-length blocks: the arena's starts (else null)
    std::vector<int32_t> starts_host;
};

namespace {

constexpr size_t kAlign = 256;

bool g_log = false;

void log_msg(const char *what) {
    if (g_log) fprintf(stderr, "[milo] %s\n", what);
}

struct Init {
    Init() {
        const char *e = getenv("MILO_LOG");
        g_log = e && e[0] == '1';
    }
} g_init;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

milo_compress_params effective(const milo_compress_params *p) {
    milo_compress_params q = *p;
    if (q.max_sweeps <= 0) q.max_sweeps = 24;
    if (!(q.jacobi_tol > 0.f)) q.jacobi_tol = 1e-7f;
    return q;
}

int n_blocks(const milo_cache_shape *s) {
    return s->block_starts ? s->n_blocks : (s->T + s->block_len - 1) / s->block_len;
}

// tokens of block b (host side)
int host_block_tokens(const milo_cache_shape *s, int b) {
    return s->block_starts ? s->block_starts[b + 1] - s->block_starts[b] : block_tokens(s->T, s->block_len, b);
}

bool shape_ok(const milo_cache_shape *s) {
    if (!(s && s->L > 0 && s->H > 0 && s->T > 0 && s->block_len > 0 &&
          (s->in_dtype == MILO_F32 || s->in_dtype == MILO_BF16)))
        return false;
    if (!s->block_starts) return true;
    // variable-length blocks: from 0 to T, ascending, each of 1 .. block_len tokens
    if (s->n_blocks <= 0 || s->block_starts[0] != 0 || s->block_starts[s->n_blocks] != s->T) return false;
    for (int b = 0; b < s->n_blocks; ++b) {
        const int n = s->block_starts[b + 1] - s->block_starts[b];
        if (n < 1 || n > s->block_len) return false;
    }
    return true;
}

// sum over one (layer, head) row of the rank caps and of the r_min floors
void cap_sums(const milo_cache_shape *s, int r_min, int r_max, int64_t &caps, int64_t &floors) {
    caps = 0;
    floors = 0;
    const int nb = n_blocks(s);
    for (int b = 0; b < nb; ++b) {
        const int c = block_cap(host_block_tokens(s, b), r_max);
        caps += c;
        floors += r_min < c ? r_min : c;
    }
}

int64_t budget_of(const milo_cache_shape *s, const milo_compress_params *p) {
    if (!shape_ok(s) || !p) return -1;
    if (p->budget_abs > 0) return p->budget_abs;
    if (!(p->budget_frac >= 0.0 && p->budget_frac <= 1.0)) return -1;
    int64_t total = 0;
    const int nb = n_blocks(s);
    for (int b = 0; b < nb; ++b) {
        const int tb = host_block_tokens(s, b);
        total += tb < D ? tb : D;
    }
    total *= (int64_t)s->L * s->H;
    return (int64_t)std::floor(p->budget_frac * (double)total);
}

// Byte offsets of one kind's arrays inside its arena section.
struct SectionLayout {
    size_t starts, ranks, offsets, sigma, eps, scaleA, scaleB, data, bytes;
};

SectionLayout section_layout(const milo_cache_shape *s, const milo_compress_params *p, int64_t R) {
    SectionLayout o{};
    const int64_t nblk = (int64_t)s->L * s->H * n_blocks(s);
    size_t at = 0;
    o.starts = at;  at = align_up(at + sizeof(int32_t) * (n_blocks(s) + 1));
    o.ranks = at;   at = align_up(at + sizeof(int32_t) * nblk);
    o.offsets = at; at = align_up(at + sizeof(int64_t) * (nblk + 1));
    o.sigma = at;   at = align_up(at + sizeof(float) * nblk * D);
    o.eps = at;     at = align_up(at + sizeof(double) * (size_t)s->L * s->H);
    o.scaleA = at;
    o.scaleB = at;
    if (p->factor_dtype == MILO_INT8) {
        at = align_up(at + sizeof(float) * nblk * D);
        o.scaleB = at;
        at = align_up(at + sizeof(float) * nblk * D);
    } else if (p->factor_dtype == MILO_INT2) {   // B's scales only (A's travel with its codes)
        at = align_up(at + sizeof(float) * nblk * D);
    }
    o.data = at;
    // sum_b round_up(r_b, 8) (128 ceil(T_b/128) + d) <= (R + 7 N_blk) (128 ceil(block_len/128) + d)
    // elements; 2-bit: sum_b R8 (48 ceil(T_b/128) + d) bytes
    if (p->factor_dtype == MILO_INT2)
        at = align_up(at + (size_t)(R + 7 * nblk) * (size_t)(48 * (round_up(s->block_len, FTILE) / FTILE) + D));
    else
        at = align_up(at + (size_t)(R + 7 * nblk) * (size_t)(round_up(s->block_len, FTILE) + D) *
                               dtype_bytes(p->factor_dtype));
    o.bytes = at;
    return o;
}

// the handle's shape with its own copy of the variable blocks' starts
void set_shape(milo_factors *f, const milo_cache_shape *s) {
    f->shape = *s;
    f->starts_host.clear();
    if (s->block_starts) {
        f->starts_host.assign(s->block_starts, s->block_starts + s->n_blocks + 1);
        f->shape.block_starts = f->starts_host.data();
    } else {
        f->shape.n_blocks = 0;
    }
}

void fill_views(milo_factors *f) {
    const SectionLayout o = section_layout(&f->shape, &f->params, f->R);
    f->starts = f->shape.block_starts ? (int32_t *)((char *)f->arena + o.starts) : nullptr;
    for (int k = 0; k < 2; ++k) {
        char *base = (char *)f->arena + (size_t)k * o.bytes;
        f->kv[k].ranks = (int32_t *)(base + o.ranks);
        f->kv[k].offsets = (int64_t *)(base + o.offsets);
        f->kv[k].sigma = (float *)(base + o.sigma);
        f->kv[k].eps = (double *)(base + o.eps);
        const int dt = f->params.factor_dtype;
        f->kv[k].scaleA = dt == MILO_INT8 ? (float *)(base + o.scaleA) : nullptr;
        f->kv[k].scaleB = dt == MILO_INT8 || dt == MILO_INT2 ? (float *)(base + o.scaleB) : nullptr;
        f->kv[k].data = base + o.data;
    }
}

milo_status params_ok(const milo_cache_shape *s, const milo_compress_params *p, int64_t *R_out) {
    if (!shape_ok(s) || !p) return MILO_ERR_INVALID_ARG;
    if (s->d != D) return MILO_ERR_UNSUPPORTED;
    if (p->factor_dtype != MILO_F32 && p->factor_dtype != MILO_BF16 && p->factor_dtype != MILO_INT8 &&
        p->factor_dtype != MILO_INT2)
        return MILO_ERR_INVALID_ARG;
    if (p->r_min < 0 || p->r_max < 0 || p->eps_scope < 0 || p->eps_scope > 1 || !(p->eps_rel >= 0.0))
        return MILO_ERR_INVALID_ARG;
    const int64_t R = budget_of(s, p);
    if (R < 0) return MILO_ERR_INVALID_ARG;
    int64_t caps, floors;
    cap_sums(s, p->r_min, p->r_max, caps, floors);
    const int64_t lh = (int64_t)s->L * s->H;
    if (R < floors * lh || R > caps * lh) return MILO_ERR_INVALID_ARG;
    if (R_out) *R_out = R;
    return MILO_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

milo_status cuda_check(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return MILO_OK;
    if (g_log) fprintf(stderr, "[milo] %s: %s\n", what, cudaGetErrorString(e));
    return MILO_ERR_CUDA;
}

// Limit of every wait inside the tensor-core decode kernel (ns of the GPU's
// global timer), and a fault injected into the next decode call by the test
// hook milo_test_decode_inject.
constexpr uint64_t kWaitNs = 2000000000ull;
std::mutex g_inject_mu;

// Kernel timing: event pairs per stage, recorded while enabled.
struct StageTiming {
    std::mutex mu;
    bool on = false;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev[MILO_TK_COUNT];
} g_timing;

cudaEvent_t tmark(cudaStream_t s) {
    if (!g_timing.on) return nullptr;
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    if (cudaEventRecord(e, s) != cudaSuccess) {
        cudaEventDestroy(e);
        return nullptr;
    }
    return e;
}
void tpush(int stage, cudaEvent_t a, cudaEvent_t b) {
    if (!a || !b) {
        if (a) cudaEventDestroy(a);
        if (b) cudaEventDestroy(b);
        return;
    }
    std::lock_guard<std::mutex> lk(g_timing.mu);
    g_timing.ev[stage].emplace_back(a, b);
}
void timing_drop_locked() {
    for (auto &v : g_timing.ev) {
        for (auto &p : v) {
            cudaEventDestroy(p.first);
            cudaEventDestroy(p.second);
        }
        v.clear();
    }
}
int g_inject_mode = 0;
uint64_t g_inject_wait_ns = 0;

int g_sm_count = 0;
int sm_count() {
    if (g_sm_count == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (g_sm_count <= 0) g_sm_count = 148;
    }
    return g_sm_count;
}

// Allocation scratch layout for two kinds.
struct AllocScratch {
    SelState *st;       // [2]
    int32_t *gt, *eq;   // [2][n_blk] each
    size_t bytes;
};

AllocScratch alloc_scratch(void *ws, int64_t n_blk) {
    AllocScratch a{};
    size_t at = 0;
    char *b = (char *)ws;
    a.st = (SelState *)(b + at); at = align_up(at + 2 * sizeof(SelState));
    a.gt = (int32_t *)(b + at);  at = align_up(at + 2 * sizeof(int32_t) * n_blk);
    a.eq = (int32_t *)(b + at);  at = align_up(at + 2 * sizeof(int32_t) * n_blk);
    a.bytes = at;
    return a;
}

// The selection launches for two kinds (kinds == 1 runs the first only).
milo_status launch_select(SelArgs a0, SelArgs a1, const SelShape &sh, int kinds, cudaStream_t st) {
    k_sel_init<<<kinds, 256, 0, st>>>(a0, a1);
    const int64_t elems = sh.n_blk * D;
    int grid = (int)std::min<int64_t>((elems + 255) / 256, (int64_t)sm_count() * 8);
    if (grid < 1) grid = 1;
    for (int pass = 0; pass < 8; ++pass)
        k_sel_pass<<<dim3(grid, kinds), 256, 0, st>>>(a0, a1, sh, 56 - 8 * pass);
    const int cgrid = (int)((sh.n_blk * 32 + 255) / 256);
    k_sel_count<<<dim3(cgrid > 0 ? cgrid : 1, kinds), 256, 0, st>>>(a0, a1, sh);
    k_sel_ranks<<<kinds, 1024, 0, st>>>(a0, a1, sh);
    return cuda_check(cudaGetLastError(), "select launch");
}

bool g_smem_set = false;
milo_status set_smem_attrs() {
    if (g_smem_set) return MILO_OK;
    cudaError_t e = cudaFuncSetAttribute(k_jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)jacobi_smem_bytes());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_decode_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(DecodeSimtSmem));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_refine_sigma<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)refine_smem_bytes());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_refine_sigma<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)refine_smem_bytes());
    if (e == cudaSuccess) e = gram_tc_set_attrs();
    if (e == cudaSuccess) e = decode_tc_set_attrs();
    if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute");
    g_smem_set = true;
    return MILO_OK;
}

}  // namespace

extern "C" {

const char *milo_version(void) { return "0.1.0"; }

const char *milo_status_string(milo_status s) {
    switch (s) {
    case MILO_OK: return "ok";
    case MILO_WARN_NOT_CONVERGED: return "a Jacobi eigensolve reached its sweep cap";
    case MILO_ERR_INVALID_ARG: return "invalid argument";
    case MILO_ERR_UNSUPPORTED: return "unsupported shape or dtype (d must be 128)";
    case MILO_ERR_CUDA: return "CUDA runtime error";
    case MILO_ERR_WORKSPACE: return "workspace or arena too small";
    case MILO_ERR_NONFINITE: return "non-finite value met on the device";
    case MILO_ERR_BOUNDS: return "index out of range met on the device";
    case MILO_ERR_TIMEOUT: return "a bounded wait on the device ran out (pipeline stalled)";
    }
    return "unknown status";
}

void milo_default_params(milo_compress_params *p) {
    if (!p) return;
    memset(p, 0, sizeof(*p));
    p->budget_frac = 0.5;
    p->budget_abs = 0;
    p->eps_rel = 1e-2;
    p->eps_scope = 0;
    p->r_min = 0;
    p->r_max = 0;
    p->factor_dtype = MILO_BF16;
    p->max_sweeps = 24;
    p->jacobi_tol = 1e-7f;
}

int64_t milo_rank_budget(const milo_cache_shape *shape, const milo_compress_params *params) {
    int64_t R = -1;
    if (params_ok(shape, params, &R) != MILO_OK) return -1;
    return R;
}

size_t milo_factor_arena_size(const milo_cache_shape *shape, const milo_compress_params *params) {
    int64_t R;
    if (params_ok(shape, params, &R) != MILO_OK) return 0;
    return 2 * section_layout(shape, params, R).bytes;
}

size_t milo_compress_workspace_size(const milo_cache_shape *shape, const milo_compress_params *params) {
    if (params_ok(shape, params, nullptr) != MILO_OK) return 0;
    const int64_t nblk = (int64_t)shape->L * shape->H * n_blocks(shape);
    const size_t gw = align_up(sizeof(float) * 2 * (size_t)nblk * D * D);
    return gw + alloc_scratch(nullptr, nblk).bytes;
}

milo_status milo_compress(const milo_cache_shape *shape, const void *K, const void *V,
                          const milo_compress_params *params_in, void *workspace, size_t ws_bytes,
                          void *arena, size_t arena_bytes, milo_factors **out, milo_stream_t stream) {
    if (!out) return MILO_ERR_INVALID_ARG;
    *out = nullptr;
    int64_t R;
    milo_status st = params_ok(shape, params_in, &R);
    if (st != MILO_OK) return st;
    if (!K || !V || !workspace || !arena) return MILO_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(workspace, kAlign) || !aligned(arena, kAlign))
        return MILO_ERR_INVALID_ARG;
    if (ws_bytes < milo_compress_workspace_size(shape, params_in) ||
        arena_bytes < milo_factor_arena_size(shape, params_in))
        return MILO_ERR_WORKSPACE;
    if ((st = set_smem_attrs()) != MILO_OK) return st;
    const milo_compress_params p = effective(params_in);
    milo_factors *f = new (std::nothrow) milo_factors();
    if (!f) return MILO_ERR_INVALID_ARG;
    set_shape(f, shape);
    f->params = p;
    f->arena = arena;
    f->arena_bytes = arena_bytes;
    f->n_b = n_blocks(shape);
    f->n_blk = (int64_t)shape->L * shape->H * f->n_b;
    f->R = R;
    fill_views(f);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t nblk = f->n_blk;
    float *GW = (float *)workspace;
    const BlockGeo geo{shape->T, shape->block_len, f->starts};
    if (f->starts) {   // the variable blocks' starts into the arena, for every kernel
        cudaError_t e = cudaMemcpyAsync(f->starts, f->starts_host.data(), sizeof(int32_t) * (f->n_b + 1),
                                        cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) { delete f; return cuda_check(e, "block starts copy"); }
    }
    AllocScratch as = alloc_scratch((char *)workspace + align_up(sizeof(float) * 2 * (size_t)nblk * D * D), nblk);

    // 1. Gram matrices of every block of K and V
    const dim3 grid2((unsigned)nblk, 2);
    cudaEvent_t t0 = tmark(s);
    if (shape->in_dtype == MILO_BF16 && !f->starts && gram_tc_supported(shape->T, shape->block_len)) {
        st = cuda_check(launch_gram_tc((const __nv_bfloat16 *)K, (const __nv_bfloat16 *)V, shape->L * shape->H,
                                       shape->T, shape->block_len, f->n_b, GW, nblk, sm_count(), s),
                        "Gram (tensor cores) launch");
        if (st != MILO_OK) { delete f; return st; }
    } else if (shape->in_dtype == MILO_BF16) {
        k_gram_simt<__nv_bfloat16><<<grid2, 256, 0, s>>>((const __nv_bfloat16 *)K, (const __nv_bfloat16 *)V,
                                                          shape->H, geo, f->n_b, GW, nblk);
    } else {
        k_gram_simt<float><<<grid2, 256, 0, s>>>((const float *)K, (const float *)V, shape->H, geo, f->n_b, GW,
                                                  nblk);
    }
    cudaEvent_t t1 = tmark(s);
    tpush(MILO_TK_GRAM, t0, t1);
    // 2. eigensolve: sigma into the arena, sorted eigenvectors back into GW
    t0 = tmark(s);
    k_jacobi<<<grid2, JAC_THREADS, jacobi_smem_bytes(), s>>>(GW, f->kv[0].sigma, f->kv[1].sigma, nblk, geo,
                                                             f->n_b, p.max_sweeps, p.jacobi_tol);
    tpush(MILO_TK_JACOBI, t0, tmark(s));
    // 2b. singular values recomputed from the blocks, sigma / W re-sorted
    t0 = tmark(s);
    if (shape->in_dtype == MILO_BF16)
        k_refine_sigma<__nv_bfloat16><<<grid2, RF_THREADS, refine_smem_bytes(), s>>>(
            (const __nv_bfloat16 *)K, (const __nv_bfloat16 *)V, GW, f->kv[0].sigma, f->kv[1].sigma, geo, f->n_b,
            nblk);
    else
        k_refine_sigma<float><<<grid2, RF_THREADS, refine_smem_bytes(), s>>>(
            (const float *)K, (const float *)V, GW, f->kv[0].sigma, f->kv[1].sigma, geo, f->n_b, nblk);
    tpush(MILO_TK_REFINE, t0, tmark(s));
    // 3. eps per (layer, head, kind)
    const int ngroups = shape->L * shape->H;
    t0 = tmark(s);
    k_eps<<<dim3(ngroups, 2), 256, 0, s>>>(f->kv[0].sigma, f->kv[1].sigma, f->kv[0].eps, f->kv[1].eps, f->n_b,
                                           p.eps_rel);
    if (p.eps_scope == 1) k_eps_global<<<2, 1024, 0, s>>>(f->kv[0].eps, f->kv[1].eps, ngroups);
    // 4. global top-R selection, ranks and packed offsets
    int64_t caps, floors;
    cap_sums(shape, p.r_min, p.r_max, caps, floors);
    SelShape sh{f->n_b, shape->T, shape->block_len, p.r_min, p.r_max, nblk, (int)p.factor_dtype, f->starts};
    SelArgs a[2];
    for (int k = 0; k < 2; ++k) {
        a[k].sigma = f->kv[k].sigma;
        a[k].eps = f->kv[k].eps;
        a[k].ranks = f->kv[k].ranks;
        a[k].offsets = f->kv[k].offsets;
        a[k].st = as.st + k;
        a[k].gt = as.gt + k * nblk;
        a[k].eq = as.eq + k * nblk;
        a[k].need0 = R - floors * ngroups;
    }
    if ((st = launch_select(a[0], a[1], sh, 2, s)) != MILO_OK) { delete f; return st; }
    tpush(MILO_TK_SELECT, t0, tmark(s));
    // 5. projection A_b = X_b W_{:,1:r_b}, B_b = W_{:,1:r_b}^T, packing
    ProjArgs pa{};
    pa.X[0] = K;
    pa.X[1] = V;
    pa.W[0] = GW;
    pa.W[1] = GW + (size_t)nblk * D * D;
    pa.kv[0] = f->kv[0];
    pa.kv[1] = f->kv[1];
    pa.T = shape->T;
    pa.block_len = shape->block_len;
    pa.n_b = f->n_b;
    pa.in_dtype = shape->in_dtype;
    pa.out_dtype = p.factor_dtype;
    pa.n_blk = nblk;
    pa.starts = f->starts;
    t0 = tmark(s);
    if (shape->in_dtype == MILO_BF16)
        k_project_a<__nv_bfloat16><<<dim3((unsigned)nblk, D / 32, 2), 256, 0, s>>>(pa);
    else
        k_project_a<float><<<dim3((unsigned)nblk, D / 32, 2), 256, 0, s>>>(pa);
    k_project_b<<<grid2, D, 0, s>>>(pa);
    tpush(MILO_TK_PROJECT, t0, tmark(s));
    st = cuda_check(cudaGetLastError(), "compress launch");
    if (st != MILO_OK) { delete f; return st; }
    log_msg("compress launched");
    *out = f;
    return MILO_OK;
}

size_t milo_allocate_workspace_size(int32_t n_groups, int32_t n_b, int32_t d) {
    if (n_groups <= 0 || n_b <= 0 || d != D) return 0;
    return alloc_scratch(nullptr, (int64_t)n_groups * n_b).bytes;
}

milo_status milo_allocate(const float *sigma, const double *eps, int32_t n_groups, int32_t n_b, int32_t d,
                          int32_t T, int32_t block_len, int64_t R, int32_t r_min, int32_t r_max,
                          int32_t *ranks_out, void *workspace, size_t ws_bytes, milo_stream_t stream) {
    if (d != D) return MILO_ERR_UNSUPPORTED;
    if (!sigma || !eps || !ranks_out || !workspace || n_groups <= 0 || n_b <= 0 || block_len <= 0 || T <= 0 ||
        r_min < 0 || r_max < 0 || R < 0)
        return MILO_ERR_INVALID_ARG;
    if ((int64_t)(T + block_len - 1) / block_len != n_b) return MILO_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign) || !aligned(sigma, 4) || !aligned(eps, 8) || !aligned(ranks_out, 4))
        return MILO_ERR_INVALID_ARG;
    const int64_t nblk = (int64_t)n_groups * n_b;
    if (ws_bytes < milo_allocate_workspace_size(n_groups, n_b, d)) return MILO_ERR_WORKSPACE;
    milo_cache_shape shp{1, 1, T, D, block_len, MILO_F32};
    int64_t caps, floors;
    cap_sums(&shp, r_min, r_max, caps, floors);
    if (R < floors * n_groups || R > caps * n_groups) return MILO_ERR_INVALID_ARG;
    AllocScratch as = alloc_scratch(workspace, nblk);
    SelShape sh{n_b, T, block_len, r_min, r_max, nblk, MILO_F32, nullptr};
    SelArgs a{};
    a.sigma = sigma;
    a.eps = eps;
    a.ranks = ranks_out;
    a.offsets = nullptr;
    a.st = as.st;
    a.gt = as.gt;
    a.eq = as.eq;
    a.need0 = R - floors * n_groups;
    return launch_select(a, a, sh, 1, (cudaStream_t)stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Rank allocation without a caller workspace.
//
// Some callers may not allocate device memory at all: code running inside a
// framework that owns every device byte through its own pool, or a plug-in
// operator that is handed only its inputs and outputs.  They call
// milo_allocate_noalloc, whose scratch (selection state and per-block counts
// for up to MILO_NOALLOC_MAX_BLOCKS blocks) is this file-scope device array.
// Every GPU that loads the library holds it (about 1 MiB) until exit.  In
// host code the array's name is only a host-side stand-in, so its device
// address is looked up per device with cudaGetSymbolAddress.
namespace {
constexpr int64_t kNoAllocBlocks = MILO_NOALLOC_MAX_BLOCKS;
constexpr size_t kNoAllocBytes = (2 * sizeof(SelState) + kAlign - 1) / kAlign * kAlign +
                                 2 * ((2 * sizeof(int32_t) * (size_t)kNoAllocBlocks + kAlign - 1) / kAlign * kAlign);
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {
constexpr int kMaxDevices = 64;
void *g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device; nullptr on
// failure.  Looked up again on every call made outside stream capture (a
// context torn down by cudaDeviceReset and created anew may place the array
// elsewhere); a call being captured into a graph reuses the address of the
// last lookup on that device and looks it up only if there was none.
void *noalloc_scratch(cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev] || cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cuda_check(e == cudaSuccess ? cudaErrorInvalidSymbol : e, "cudaGetSymbolAddress(noalloc scratch)");
            return nullptr;
        }
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" {

milo_status milo_allocate_noalloc(const float *sigma, const double *eps, int32_t n_groups, int32_t n_b, int32_t d,
                                  int32_t T, int32_t block_len, int64_t R, int32_t r_min, int32_t r_max,
                                  int32_t *ranks_out, milo_stream_t stream) {
    if (d != D) return MILO_ERR_UNSUPPORTED;
    if (!sigma || !eps || !ranks_out || n_groups <= 0 || n_b <= 0 || block_len <= 0 || T <= 0 || r_min < 0 ||
        r_max < 0 || R < 0)
        return MILO_ERR_INVALID_ARG;
    if ((int64_t)(T + block_len - 1) / block_len != n_b) return MILO_ERR_INVALID_ARG;
    if (!aligned(sigma, 4) || !aligned(eps, 8) || !aligned(ranks_out, 4)) return MILO_ERR_INVALID_ARG;
    const int64_t nblk = (int64_t)n_groups * n_b;
    if (nblk > kNoAllocBlocks) {
        log_msg("milo_allocate_noalloc: n_groups * n_b exceeds MILO_NOALLOC_MAX_BLOCKS");
        return MILO_ERR_WORKSPACE;
    }
    milo_cache_shape shp{1, 1, T, D, block_len, MILO_F32};
    int64_t caps, floors;
    cap_sums(&shp, r_min, r_max, caps, floors);
    if (R < floors * n_groups || R > caps * n_groups) return MILO_ERR_INVALID_ARG;
    void *scratch = noalloc_scratch((cudaStream_t)stream);
    if (!scratch) return MILO_ERR_CUDA;
    // the scratch layout for kNoAllocBlocks also holds any smaller problem
    AllocScratch as = alloc_scratch(scratch, kNoAllocBlocks);
    SelShape sh{n_b, T, block_len, r_min, r_max, nblk, MILO_F32, nullptr};
    SelArgs a{};
    a.sigma = sigma;
    a.eps = eps;
    a.ranks = ranks_out;
    a.offsets = nullptr;
    a.st = as.st;      // reset by k_sel_init at the start of every call
    a.gt = as.gt;      // written in full by k_sel_count before any read
    a.eq = as.eq;
    a.need0 = R - floors * n_groups;
    return launch_select(a, a, sh, 1, (cudaStream_t)stream);
}

// INT8 factors on the tensor cores: an fp16 copy of each kind's data section
// (the selected blocks' elements are written, at the INT8 element offsets).
static size_t shadow_bytes_per_kind(const milo_factors *f) {
    if (f->params.factor_dtype != MILO_INT8 && f->params.factor_dtype != MILO_INT2) return 0;
    return align_up(sizeof(__half) * (size_t)(f->R + 7 * f->n_blk) *
                    (size_t)(round_up(f->shape.block_len, FTILE) + D));
}

size_t milo_decode_workspace_size(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel) {
    if (!f || S <= 0 || Hq <= 0 || n_sel <= 0) return 0;
    const int64_t slots = (int64_t)S * n_sel;
    const int64_t rows = (int64_t)f->shape.L * S * Hq;
    size_t at = 0;
    at = align_up(at + sizeof(int32_t) * ((f->n_b + 1) * 3 + 1));      // counts / cursor / passes, starts, item starts, claim
    at = align_up(at + sizeof(int32_t) * slots);                       // slot list
    at = align_up(at + sizeof(float2) * (slots + f->shape.block_len) * HALF);  // rope tables
    at = align_up(at + sizeof(float) * rows * n_sel * D);              // partial o
    at = align_up(at + sizeof(float2) * rows * n_sel);                 // partial (m, l)
    at = align_up(at + sizeof(DtItem) * decode_tc_max_items(f->shape.L, f->shape.H, f->n_b, slots,
                                                            Hq / f->shape.H));  // tensor-core work items
    at += 2 * shadow_bytes_per_kind(f);                                 // INT8 / 2-bit: fp16 factors
    if (f->params.factor_dtype == MILO_INT2)                           // 2-bit: element offsets of the fp16 copy
        at += 2 * align_up(sizeof(int64_t) * (f->n_blk + 1));
    return at;
}

}  // extern "C"

namespace {
// the recent uncompressed tokens of a decode call (k == nullptr: none)
struct TailIn {
    const void *k = nullptr, *v = nullptr;
    milo_dtype dtype = MILO_F32;
    int32_t cap = 0;
    const int32_t *len = nullptr;
};

size_t tail_workspace_bytes(const milo_factors *f, int32_t S, int32_t Hq) {
    const int64_t rows = (int64_t)f->shape.L * S * Hq;
    return align_up(sizeof(float) * rows * D) + align_up(sizeof(float2) * rows);
}

milo_status decode_impl(const milo_factors *f, const float *q, int32_t S, int32_t Hq, const int32_t *selected,
                        const int32_t *positions, int32_t n_sel, double rope_base, const TailIn &tail, float *out,
                        void *workspace, size_t ws_bytes, milo_stream_t stream) {
    if (!f || !q || !selected || !out || !workspace || S <= 0 || Hq <= 0 || n_sel <= 0)
        return MILO_ERR_INVALID_ARG;
    if (Hq % f->shape.H != 0 || !(rope_base > 0.0)) return MILO_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, kAlign) || !aligned(selected, 4))
        return MILO_ERR_INVALID_ARG;
    // 2-bit factors decode on the tensor cores only (blocks of at most 512 tokens)
    if (f->params.factor_dtype == MILO_INT2 && f->shape.block_len > 512) return MILO_ERR_UNSUPPORTED;
    const size_t ws_dec = milo_decode_workspace_size(f, S, Hq, n_sel);
    if (ws_bytes < ws_dec + (tail.k ? tail_workspace_bytes(f, S, Hq) : 0)) return MILO_ERR_WORKSPACE;
    milo_status st = set_smem_attrs();
    if (st != MILO_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int n_b = f->n_b;
    const int64_t slots = (int64_t)S * n_sel;
    const int64_t rows = (int64_t)f->shape.L * S * Hq;
    char *w = (char *)workspace;
    size_t at = 0;
    int32_t *cnt = (int32_t *)(w + at);
    int32_t *start = cnt + (n_b + 1);
    int32_t *pstart = start + (n_b + 1);   // tensor-core work items of each block id, scanned
    int32_t *claim = pstart + (n_b + 1);   // next unclaimed tensor-core work item
    at = align_up(at + sizeof(int32_t) * ((n_b + 1) * 3 + 1));
    int32_t *list = (int32_t *)(w + at); at = align_up(at + sizeof(int32_t) * slots);
    float2 *rope_q = (float2 *)(w + at);
    float2 *rope_t = rope_q + slots * HALF;
    at = align_up(at + sizeof(float2) * (slots + f->shape.block_len) * HALF);
    float *part_o = (float *)(w + at); at = align_up(at + sizeof(float) * rows * n_sel * D);
    float2 *part_ml = (float2 *)(w + at); at = align_up(at + sizeof(float2) * rows * n_sel);
    DtItem *items = (DtItem *)(w + at);
    at = align_up(at + sizeof(DtItem) * decode_tc_max_items(f->shape.L, f->shape.H, f->n_b, slots,
                                                            Hq / f->shape.H));
    __half *shadow0 = (__half *)(w + at);
    __half *shadow1 = (__half *)(w + at + shadow_bytes_per_kind(f));
    int64_t *eoff0 = (int64_t *)(w + at + 2 * shadow_bytes_per_kind(f));
    int64_t *eoff1 = (int64_t *)((char *)eoff0 + align_up(sizeof(int64_t) * (f->n_blk + 1)));

    DecodeArgs a{};
    a.kv[0] = f->kv[0];
    a.kv[1] = f->kv[1];
    a.L = f->shape.L; a.H = f->shape.H; a.G = Hq / f->shape.H; a.T = f->shape.T;
    a.block_len = f->shape.block_len; a.n_b = n_b; a.factor_dtype = f->params.factor_dtype;
    a.S = S; a.Hq = Hq; a.n_sel = n_sel;
    a.q = q; a.sel = selected; a.pos = positions; a.starts = f->starts;
    a.slot_start = start; a.slot_list = list;
    a.rope_q = rope_q; a.rope_t = rope_t;
    a.part_o = part_o; a.part_ml = part_ml; a.out = out;
    a.claim = claim;
    a.f16 = 0;
    {   // a test-injected fault applies to this call only
        std::lock_guard<std::mutex> lk(g_inject_mu);
        a.wait_ns = g_inject_wait_ns ? g_inject_wait_ns : kWaitNs;
        a.inject = g_inject_mode;
        g_inject_mode = 0;
        g_inject_wait_ns = 0;
    }

    // counts and the claim counter to 0 (the starts are written by the scans)
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * ((n_b + 1) * 3 + 1), s);
    if (e != cudaSuccess) return cuda_check(e, "memset");
    const int sg = (int)std::min<int64_t>((slots + 255) / 256, 1024);
    cudaEvent_t t0 = tmark(s);
    k_slot_count<<<sg, 256, 0, s>>>(selected, (int)slots, n_b, cnt);
    k_slot_scan<<<1, SCAN_THREADS, 0, s>>>(cnt, start, n_b);
    k_slot_fill<<<sg, 256, 0, s>>>(selected, (int)slots, n_b, start, cnt, list);
    const int64_t rt = (slots + f->shape.block_len) * HALF;
    k_rope_tables<<<(int)std::min<int64_t>((rt + 255) / 256, 4096), 256, 0, s>>>(
        selected, positions, f->starts, n_b, (int)slots, f->shape.block_len, rope_base, rope_q, rope_t);
    if (decode_tc_supported(a)) {
        if (a.factor_dtype == MILO_INT8) {   // dequantised to fp16 for the tensor cores
            k_dequant_selected<<<dim3((unsigned)f->n_blk, 2), 256, 0, s>>>(a, shadow0, shadow1);
            a.kv[0].data = shadow0;
            a.kv[1].data = shadow1;
            a.f16 = 1;
        } else if (a.factor_dtype == MILO_INT2) {   // the same, into the bf16 layout's element offsets
            const int eg = (int)std::min<int64_t>((f->n_blk + 255) / 256, 4096);
            const BlockGeo geo{f->shape.T, f->shape.block_len, f->starts};
            k_elem_sizes<<<eg, 256, 0, s>>>(f->kv[0].ranks, f->n_blk, n_b, geo, eoff0);
            k_elem_sizes<<<eg, 256, 0, s>>>(f->kv[1].ranks, f->n_blk, n_b, geo, eoff1);
            k_scan_i64<<<1, SCAN_THREADS, 0, s>>>(eoff0, f->n_blk);
            k_scan_i64<<<1, SCAN_THREADS, 0, s>>>(eoff1, f->n_blk);
            k_dequant_int2<<<dim3((unsigned)f->n_blk, 2), 256, 0, s>>>(a, eoff0, eoff1, shadow0, shadow1);
            a.kv[0].data = shadow0;
            a.kv[1].data = shadow1;
            a.kv[0].offsets = eoff0;
            a.kv[1].offsets = eoff1;
            a.f16 = 1;
        }
        // work items: passes of up to DT_NQ queries per block id (counts reuse cnt)
        k_pass_counts<<<(n_b + 255) / 256, 256, 0, s>>>(start, n_b, a.G, DT_NQ, cnt);
        k_scan_counts<<<1, SCAN_THREADS, 0, s>>>(cnt, pstart, n_b);
        tpush(MILO_TK_DECODE_PREP, t0, tmark(s));
        t0 = tmark(s);
        st = cuda_check(launch_decode_tc(a, pstart, items, sm_count(), s), "decode (tensor cores) launch");
        if (st != MILO_OK) return st;
        tpush(MILO_TK_DECODE, t0, tmark(s));
    } else {
        tpush(MILO_TK_DECODE_PREP, t0, tmark(s));
        t0 = tmark(s);
        k_decode_simt<<<dim3(n_b, f->shape.H, f->shape.L), 256, sizeof(DecodeSimtSmem), s>>>(a);
        tpush(MILO_TK_DECODE, t0, tmark(s));
    }
    if (tail.k) {   // the recent tokens' partial, then merged with the blocks'
        float *tail_o = (float *)(w + ws_dec);
        float2 *tail_ml = (float2 *)(w + ws_dec + align_up(sizeof(float) * rows * D));
        t0 = tmark(s);
        const dim3 grid((unsigned)f->shape.H, (unsigned)S, (unsigned)f->shape.L);
        if (tail.dtype == MILO_BF16)
            k_tail_attn<__nv_bfloat16><<<grid, D, 0, s>>>(a, (const __nv_bfloat16 *)tail.k,
                                                          (const __nv_bfloat16 *)tail.v, tail.cap, tail.len,
                                                          tail_o, tail_ml);
        else
            k_tail_attn<float><<<grid, D, 0, s>>>(a, (const float *)tail.k, (const float *)tail.v, tail.cap,
                                                  tail.len, tail_o, tail_ml);
        tpush(MILO_TK_TAIL, t0, tmark(s));
        a.tail_o = tail_o;
        a.tail_ml = tail_ml;
    }
    t0 = tmark(s);
    k_combine<float><<<(unsigned)rows, D, 0, s>>>(a, a.part_o);
    tpush(MILO_TK_COMBINE, t0, tmark(s));
    return cuda_check(cudaGetLastError(), "decode launch");
}
}  // namespace

extern "C" {

milo_status milo_decode_attn(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                             const int32_t *selected, const int32_t *positions, int32_t n_sel, double rope_base,
                             float *out, void *workspace, size_t ws_bytes, milo_stream_t stream) {
    return decode_impl(f, q, S, Hq, selected, positions, n_sel, rope_base, TailIn{}, out, workspace, ws_bytes,
                       stream);
}

}  // extern "C"

// ---------------------------------------------------------------- offload
namespace {
struct OffloadLayout {
    size_t used, sizes[2], ranks[2], scaleA[2], scaleB[2], data[2], bytes;
};
// the staging area after the decode's own scratch
OffloadLayout offload_layout(const milo_factors *f, size_t at) {
    OffloadLayout o{};
    const SectionLayout sec = section_layout(&f->shape, &f->params, f->R);
    const bool i8 = f->params.factor_dtype == MILO_INT8;
    const bool sB = i8 || f->params.factor_dtype == MILO_INT2;   // B's scales
    o.used = at; at = align_up(at + sizeof(int32_t) * (f->n_b + 1));
    for (int k = 0; k < 2; ++k) {
        o.sizes[k] = at; at = align_up(at + sizeof(int64_t) * (f->n_blk + 1));
        o.ranks[k] = at; at = align_up(at + sizeof(int32_t) * f->n_blk);
        o.scaleA[k] = at; at = align_up(at + (i8 ? sizeof(float) * f->n_blk * D : 0));
        o.scaleB[k] = at; at = align_up(at + (sB ? sizeof(float) * f->n_blk * D : 0));
        o.data[k] = at; at = align_up(at + (sec.bytes - sec.data));   // every block selected at most
    }
    o.bytes = at;
    return o;
}

// the device address of p, a pointer into f's arena (null stays null), given
// the device address of the arena
template <typename P> P *on_device(const milo_factors *f, P *p, char *dev_arena) {
    return p ? (P *)(dev_arena + ((const char *)p - (const char *)f->arena)) : nullptr;
}
}  // namespace

namespace {
// workspace: the decode's own scratch, the recent-token partials, the staging area
size_t offload_front(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel) {
    return milo_decode_workspace_size(f, S, Hq, n_sel) + tail_workspace_bytes(f, S, Hq);
}

milo_status offload_impl(const milo_factors *f, const float *q, int32_t S, int32_t Hq, const int32_t *selected,
                         const int32_t *positions, int32_t n_sel, double rope_base, const TailIn &tail, float *out,
                         void *workspace, size_t ws_bytes, milo_stream_t stream) {
    if (!f || !f->arena || !q || !selected || !out || !workspace || S <= 0 || Hq <= 0 || n_sel <= 0)
        return MILO_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign)) return MILO_ERR_INVALID_ARG;
    const size_t ws_front = offload_front(f, S, Hq, n_sel);
    const OffloadLayout o = offload_layout(f, align_up(ws_front));
    if (ws_bytes < o.bytes) return MILO_ERR_WORKSPACE;
    // the arena must be reachable from the device: pinned, mapped host memory
    // (or device memory); pageable memory is refused before any launch
    cudaPointerAttributes attr{};
    cudaError_t e = cudaPointerGetAttributes(&attr, f->arena);
    if (e != cudaSuccess) return cuda_check(e, "arena attributes");
    if ((attr.type != cudaMemoryTypeHost && attr.type != cudaMemoryTypeDevice &&
         attr.type != cudaMemoryTypeManaged) || !attr.devicePointer)
        return MILO_ERR_INVALID_ARG;
    char *dev_arena = (char *)attr.devicePointer;
    cudaStream_t s = (cudaStream_t)stream;
    char *w = (char *)workspace;
    int32_t *used = (int32_t *)(w + o.used);
    milo_factors st = *f;   // the staged copy: same shape, params and block ids
    st.arena = nullptr;
    st.arena_bytes = 0;
    st.starts = on_device(f, f->starts, dev_arena);   // read in place over the host link (a few words)
    cudaEvent_t t0 = tmark(s);
    e = cudaMemsetAsync(used, 0, sizeof(int32_t) * (f->n_b + 1), s);
    if (e != cudaSuccess) return cuda_check(e, "memset");
    const int64_t slots = (int64_t)S * n_sel;
    k_flag_selected<<<(int)std::min<int64_t>((slots + 255) / 256, 1024), 256, 0, s>>>(selected, (int)slots, f->n_b,
                                                                                      used);
    const int esize = dtype_bytes(f->params.factor_dtype);
    for (int k = 0; k < 2; ++k) {
        KindView host = f->kv[k];
        host.ranks = on_device(f, host.ranks, dev_arena);
        host.offsets = on_device(f, host.offsets, dev_arena);
        host.scaleA = on_device(f, host.scaleA, dev_arena);
        host.scaleB = on_device(f, host.scaleB, dev_arena);
        host.data = on_device(f, (char *)host.data, dev_arena);
        KindView &sv = st.kv[k];
        sv.sigma = nullptr;
        sv.eps = nullptr;
        sv.ranks = (int32_t *)(w + o.ranks[k]);
        sv.offsets = (int64_t *)(w + o.sizes[k]);
        sv.scaleA = host.scaleA ? (float *)(w + o.scaleA[k]) : nullptr;
        sv.scaleB = host.scaleB ? (float *)(w + o.scaleB[k]) : nullptr;
        sv.data = w + o.data[k];
        k_stage_sizes<<<(int)std::min<int64_t>((f->n_blk + 255) / 256, 4096), 256, 0, s>>>(
            host.ranks, used, f->n_blk, f->n_b, BlockGeo{f->shape.T, f->shape.block_len, st.starts},
            f->params.factor_dtype, sv.offsets, sv.ranks);
        k_scan_i64<<<1, SCAN_THREADS, 0, s>>>(sv.offsets, f->n_blk);
        k_stage_copy<<<(unsigned)f->n_blk, 256, 0, s>>>(host, sv, used, f->n_b, esize);
    }
    tpush(MILO_TK_STAGE, t0, tmark(s));
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_check(e, "staging launch");
    return decode_impl(&st, q, S, Hq, selected, positions, n_sel, rope_base, tail, out, workspace, ws_front,
                       stream);
}
}  // namespace

extern "C" {

size_t milo_decode_offload_workspace_size(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel) {
    return milo_decode_workspace_size(f, S, Hq, n_sel) ? offload_layout(f, align_up(offload_front(f, S, Hq, n_sel))).bytes
                                                       : 0;
}

milo_status milo_decode_attn_offload(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                                     const int32_t *selected, const int32_t *positions, int32_t n_sel,
                                     double rope_base, float *out, void *workspace, size_t ws_bytes,
                                     milo_stream_t stream) {
    return offload_impl(f, q, S, Hq, selected, positions, n_sel, rope_base, TailIn{}, out, workspace, ws_bytes,
                        stream);
}

milo_status milo_decode_attn_offload_tail(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                                          const int32_t *selected, const int32_t *positions, int32_t n_sel,
                                          double rope_base, const void *k_tail, const void *v_tail,
                                          milo_dtype tail_dtype, int32_t tail_cap, const int32_t *tail_len,
                                          float *out, void *workspace, size_t ws_bytes, milo_stream_t stream) {
    if (!k_tail || !v_tail || !tail_len || tail_cap < 0) return MILO_ERR_INVALID_ARG;
    if (tail_dtype != MILO_F32 && tail_dtype != MILO_BF16) return MILO_ERR_UNSUPPORTED;
    if (!aligned(k_tail, 16) || !aligned(v_tail, 16) || !aligned(tail_len, 4)) return MILO_ERR_INVALID_ARG;
    TailIn t;
    t.k = k_tail;
    t.v = v_tail;
    t.dtype = tail_dtype;
    t.cap = tail_cap;
    t.len = tail_len;
    return offload_impl(f, q, S, Hq, selected, positions, n_sel, rope_base, t, out, workspace, ws_bytes, stream);
}

// ---------------------------------------------------------------- retrieval
size_t milo_bm25_workspace_size(int32_t n_b, int32_t V, int32_t S) {
    if (n_b <= 0 || V <= 0 || S <= 0) return 0;
    return align_up(sizeof(int32_t) * V) + align_up(sizeof(double) * (size_t)S * V) + align_up(sizeof(double)) +
           align_up(sizeof(double) * (size_t)S * n_b);
}

milo_status milo_bm25_select(const int32_t *blk_ptr, const int32_t *blk_term, const int32_t *blk_tf,
                             const int32_t *blk_len, int32_t n_b, int32_t nnz_b, int32_t V, const int32_t *q_ptr,
                             const int32_t *q_term, const int32_t *q_tf, int32_t S, int32_t nnz_q, double k1,
                             double beta, int32_t n_sel, int32_t *selected, double *scores, void *workspace,
                             size_t ws_bytes, milo_stream_t stream) {
    if (!blk_ptr || !blk_len || !q_ptr || !selected || !workspace) return MILO_ERR_INVALID_ARG;
    if (n_b <= 0 || V <= 0 || S <= 0 || nnz_b < 0 || nnz_q < 0 || n_sel < 1 || n_sel > n_b) return MILO_ERR_INVALID_ARG;
    if ((nnz_b > 0 && (!blk_term || !blk_tf)) || (nnz_q > 0 && (!q_term || !q_tf))) return MILO_ERR_INVALID_ARG;
    if (!(k1 >= 0.0) || !(beta >= 0.0 && beta <= 1.0) || !aligned(workspace, kAlign)) return MILO_ERR_INVALID_ARG;
    if (ws_bytes < milo_bm25_workspace_size(n_b, V, S)) return MILO_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    char *w = (char *)workspace;
    size_t at = 0;
    Bm25Args a{};
    a.blk_ptr = blk_ptr; a.blk_term = blk_term; a.blk_tf = blk_tf; a.blk_len = blk_len;
    a.q_ptr = q_ptr; a.q_term = q_term; a.q_tf = q_tf;
    a.n_b = n_b; a.V = V; a.S = S; a.n_sel = n_sel; a.nnz_b = nnz_b; a.nnz_q = nnz_q;
    a.k1 = k1; a.beta = beta;
    a.df = (int32_t *)(w + at); at = align_up(at + sizeof(int32_t) * V);
    a.qw = (double *)(w + at); at = align_up(at + sizeof(double) * (size_t)S * V);
    a.avgdl = (double *)(w + at); at = align_up(at + sizeof(double));
    a.scores = scores ? scores : (double *)(w + at);
    a.selected = selected;
    cudaEvent_t t0 = tmark(s);
    cudaError_t e = cudaMemsetAsync(a.df, 0, sizeof(int32_t) * V, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.qw, 0, sizeof(double) * (size_t)S * V, s);
    if (e != cudaSuccess) return cuda_check(e, "memset");
    k_bm25_df<<<(int)std::min<int64_t>(((int64_t)nnz_b + 255) / 256 + 1, 1024), 256, 0, s>>>(a);
    k_bm25_avgdl<<<1, 32, 0, s>>>(a);
    k_bm25_qweights<<<S, 128, 0, s>>>(a);
    k_bm25_scores<<<(unsigned)(((int64_t)S * n_b + 255) / 256), 256, 0, s>>>(a);
    k_bm25_topk<<<S, 256, 0, s>>>(a);
    tpush(MILO_TK_RETRIEVE, t0, tmark(s));
    return cuda_check(cudaGetLastError(), "retrieval launch");
}

size_t milo_decode_tail_workspace_size(const milo_factors *f, int32_t S, int32_t Hq, int32_t n_sel) {
    const size_t base = milo_decode_workspace_size(f, S, Hq, n_sel);
    return base ? base + tail_workspace_bytes(f, S, Hq) : 0;
}

milo_status milo_decode_attn_tail(const milo_factors *f, const float *q, int32_t S, int32_t Hq,
                                  const int32_t *selected, const int32_t *positions, int32_t n_sel,
                                  double rope_base, const void *k_tail, const void *v_tail, milo_dtype tail_dtype,
                                  int32_t tail_cap, const int32_t *tail_len, float *out, void *workspace,
                                  size_t ws_bytes, milo_stream_t stream) {
    if (!k_tail || !v_tail || !tail_len || tail_cap < 0) return MILO_ERR_INVALID_ARG;
    if (tail_dtype != MILO_F32 && tail_dtype != MILO_BF16) return MILO_ERR_UNSUPPORTED;
    if (!aligned(k_tail, 16) || !aligned(v_tail, 16) || !aligned(tail_len, 4)) return MILO_ERR_INVALID_ARG;
    TailIn t;
    t.k = k_tail;
    t.v = v_tail;
    t.dtype = tail_dtype;
    t.cap = tail_cap;
    t.len = tail_len;
    return decode_impl(f, q, S, Hq, selected, positions, n_sel, rope_base, t, out, workspace, ws_bytes, stream);
}

milo_status milo_factors_get(const milo_factors *f, int32_t kind, int32_t **ranks, int64_t **offsets,
                             float **sigma, double **eps, void **data, float **scaleA, float **scaleB,
                             int64_t *R) {
    if (!f || kind < 0 || kind > 1) return MILO_ERR_INVALID_ARG;
    const KindView &v = f->kv[kind];
    if (ranks) *ranks = v.ranks;
    if (offsets) *offsets = v.offsets;
    if (sigma) *sigma = v.sigma;
    if (eps) *eps = v.eps;
    if (data) *data = v.data;
    if (scaleA) *scaleA = v.scaleA;
    if (scaleB) *scaleB = v.scaleB;
    if (R) *R = f->R;
    return MILO_OK;
}

milo_status milo_factors_wrap(const milo_cache_shape *shape, const milo_compress_params *params, void *arena,
                              size_t arena_bytes, milo_factors **out) {
    if (!out) return MILO_ERR_INVALID_ARG;
    *out = nullptr;
    int64_t R;
    milo_status st = params_ok(shape, params, &R);
    if (st != MILO_OK) return st;
    if (!arena || !aligned(arena, kAlign)) return MILO_ERR_INVALID_ARG;
    if (arena_bytes < milo_factor_arena_size(shape, params)) return MILO_ERR_WORKSPACE;
    milo_factors *f = new (std::nothrow) milo_factors();
    if (!f) return MILO_ERR_INVALID_ARG;
    set_shape(f, shape);
    f->params = effective(params);
    f->arena = arena;
    f->arena_bytes = arena_bytes;
    f->n_b = n_blocks(shape);
    f->n_blk = (int64_t)shape->L * shape->H * f->n_b;
    f->R = R;
    fill_views(f);
    *out = f;
    return MILO_OK;
}

namespace {
struct BlobHeader {
    char magic[8];
    uint32_t version;
    uint32_t pad;
    milo_cache_shape shape;
    milo_compress_params params;
    uint64_t arena_bytes;
};
}  // namespace

// Blob: the header, the variable blocks' starts (n_blocks + 1 int32, only
// when the shape has them; the header's pointer is cleared), then the arena.
milo_status milo_factors_export(const milo_factors *f, void *host_buf, size_t *bytes, milo_stream_t stream) {
    if (!f || !bytes) return MILO_ERR_INVALID_ARG;
    const size_t nst = f->starts_host.size() * sizeof(int32_t);
    const size_t arena = milo_factor_arena_size(&f->shape, &f->params);
    const size_t need = sizeof(BlobHeader) + nst + arena;
    if (!host_buf) { *bytes = need; return MILO_OK; }
    if (*bytes < need) { *bytes = need; return MILO_ERR_WORKSPACE; }
    BlobHeader h{};
    memcpy(h.magic, "MILOFAC1", 8);
    h.version = 1;
    h.shape = f->shape;
    h.shape.block_starts = nullptr;
    h.params = f->params;
    h.arena_bytes = arena;
    memcpy(host_buf, &h, sizeof(h));
    if (nst) memcpy((char *)host_buf + sizeof(h), f->starts_host.data(), nst);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync((char *)host_buf + sizeof(h) + nst, f->arena, h.arena_bytes,
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    *bytes = need;
    return cuda_check(e, "export copy");
}

milo_status milo_factors_import(const void *host_buf, size_t bytes, void *arena, size_t arena_bytes,
                                milo_factors **out, milo_stream_t stream) {
    if (!out) return MILO_ERR_INVALID_ARG;
    *out = nullptr;
    if (!host_buf || bytes < sizeof(BlobHeader) || !arena) return MILO_ERR_INVALID_ARG;
    BlobHeader h;
    memcpy(&h, host_buf, sizeof(h));
    if (memcmp(h.magic, "MILOFAC1", 8) != 0 || h.version != 1) return MILO_ERR_INVALID_ARG;
    if (h.shape.n_blocks < 0 || h.shape.n_blocks > (1 << 28)) return MILO_ERR_INVALID_ARG;
    const size_t nst = h.shape.n_blocks > 0 ? sizeof(int32_t) * (size_t)(h.shape.n_blocks + 1) : 0;
    if (bytes < sizeof(h) + nst) return MILO_ERR_INVALID_ARG;
    std::vector<int32_t> starts(nst / sizeof(int32_t));
    if (nst) memcpy(starts.data(), (const char *)host_buf + sizeof(h), nst);
    h.shape.block_starts = nst ? starts.data() : nullptr;
    if (bytes < sizeof(h) + nst + h.arena_bytes) return MILO_ERR_INVALID_ARG;
    if (h.arena_bytes != milo_factor_arena_size(&h.shape, &h.params)) return MILO_ERR_INVALID_ARG;
    milo_factors *f = nullptr;
    milo_status st = milo_factors_wrap(&h.shape, &h.params, arena, arena_bytes, &f);
    if (st != MILO_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(arena, (const char *)host_buf + sizeof(h) + nst, h.arena_bytes,
                                    cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) { delete f; return cuda_check(e, "import copy"); }
    *out = f;
    return MILO_OK;
}

milo_status milo_factors_shape(const milo_factors *f, milo_cache_shape *shape, milo_compress_params *params) {
    if (!f) return MILO_ERR_INVALID_ARG;
    if (shape) *shape = f->shape;
    if (params) *params = f->params;
    return MILO_OK;
}

void milo_factors_destroy(milo_factors *f) { delete f; }

milo_status milo_test_decode_inject(int32_t mode, uint64_t wait_ns) {
    if (mode < 0 || mode > 1 || (mode == 1 && (wait_ns == 0 || wait_ns > kWaitNs))) return MILO_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_inject_mu);
    g_inject_mode = mode;
    g_inject_wait_ns = wait_ns;
    return MILO_OK;
}

milo_status milo_timing_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    if (on) timing_drop_locked();
    g_timing.on = on != 0;
    return MILO_OK;
}

milo_status milo_timing_read(double *ms, int64_t *count, int32_t n) {
    if (n < 0 || n > MILO_TK_COUNT || (n > 0 && (!ms || !count))) return MILO_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_timing.mu);
    milo_status st = MILO_OK;
    for (int k = 0; k < MILO_TK_COUNT; ++k) {
        double sum = 0.0;
        for (auto &p : g_timing.ev[k]) {
            float t = 0.f;
            cudaError_t e = cudaEventSynchronize(p.second);
            if (e == cudaSuccess) e = cudaEventElapsedTime(&t, p.first, p.second);
            if (e != cudaSuccess && st == MILO_OK) st = cuda_check(e, "timing events");
            sum += t;
        }
        if (k < n) {
            ms[k] = sum;
            count[k] = (int64_t)g_timing.ev[k].size();
        }
    }
    timing_drop_locked();
    return st;
}

milo_status milo_jacobi_rounds(int64_t *rounds, int64_t *rotations, milo_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_check(e, "stream sync");
    unsigned long long v = 0, w = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_jacobi_rounds, sizeof(v));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&w, g_jacobi_rotations, sizeof(w));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_jacobi_rounds, &zero, sizeof(zero));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_jacobi_rotations, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_check(e, "counter read");
    if (rounds) *rounds = (int64_t)v;
    if (rotations) *rotations = (int64_t)w;
    return MILO_OK;
}

milo_status milo_get_status(milo_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_check(e, "stream sync");
    unsigned bits = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&bits, g_status, sizeof(bits));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_check(e, "status read");
    if (bits & ST_BOUNDS) return MILO_ERR_BOUNDS;
    if (bits & ST_NONFINITE) return MILO_ERR_NONFINITE;
    if (bits & ST_UNSORTED) return MILO_ERR_INVALID_ARG;
    if (bits & ST_TIMEOUT) return MILO_ERR_TIMEOUT;
    if (bits & ST_NOT_CONVERGED) return MILO_WARN_NOT_CONVERGED;
    return MILO_OK;
}

#ifdef MILO_DECODE_TRACE
// Tracing build only (not part of milo.h): pick the CTA of k_decode_tc whose
// warps record the timeline, clearing earlier records (cta < 0: none), and
// copy the records out: TL_WARPS x TL_CAP TlRec rows and TL_WARPS counts.
static_assert(TL_WARPS * 32 == DT_THREADS, "one timeline row per decode warp");
milo_status milo_timeline_select(int32_t cta) {
    static uint32_t zeros[TL_WARPS];
    cudaError_t e = cudaMemcpyToSymbol(g_tl_cnt, zeros, sizeof(zeros));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_tl_cta, &cta, sizeof(cta));
    return e == cudaSuccess ? MILO_OK : cuda_check(e, "timeline select");
}
milo_status milo_timeline_read(void *records, uint32_t *counts) {
    if (!records || !counts) return MILO_ERR_INVALID_ARG;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(records, g_tl, sizeof(g_tl));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(counts, g_tl_cnt, sizeof(g_tl_cnt));
    return e == cudaSuccess ? MILO_OK : cuda_check(e, "timeline read");
}
#endif

}  // extern "C"
