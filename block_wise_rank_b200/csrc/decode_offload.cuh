// decode_offload.cuh -- decode from factors kept in host memory: each call
// stages the selected blocks' factors into device memory, then decodes there.
//
// "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression" (evolve.pub review), Summary and FAQ "How much memory saving
// and speedup does MILO achieve?": the speed-ups the pages report are measured
// against offloading the full KV cache to CPU memory; with MILO only the
// retrieved blocks' low-rank factors cross the host link, so the transfer per
// step shrinks with the compression.
//
// The arena keeps its layout (ranks, offsets, scales, data per kind) in pinned,
// device-mapped host memory.  Per call: flag the block ids some session
// selected; size each (layer, head, block) of those in offset units (0 for
// the rest) and scan the sizes into staging offsets; copy the flagged blocks'
// factors (and the INT8 / 2-bit scales) from host memory into the staging area with
// 16-byte loads (one CTA per block).  The staged copy is indexed by the
// original block ids, so the decode kernels run on it unchanged.
#pragma once
#include "decode_simt.cuh"

namespace milo {

// used[b] = 1 when some session selected block id b (ids out of range are
// left to the decode's own check)
__global__ void k_flag_selected(const int32_t *__restrict__ sel, int n_slots, int n_b, int32_t *__restrict__ used) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_slots; e += gridDim.x * blockDim.x) {
        const int b = sel[e];
        if (b >= 0 && b < n_b) used[b] = 1;
    }
}

// size (offset units of the factor type) of every (layer, head, block) of one
// kind in the staging area: the block's factors when its id is flagged, else
// 0; the ranks are copied for every block.  grid over nblk.
__global__ void k_stage_sizes(const int32_t *__restrict__ host_ranks, const int32_t *__restrict__ used, int64_t nblk,
                              int n_b, BlockGeo geo, int dtype, int64_t *__restrict__ sizes,
                              int32_t *__restrict__ ranks) {
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblk;
         blk += (int64_t)gridDim.x * blockDim.x) {
        const int b = (int)(blk % n_b);
        const int r = host_ranks[blk];
        ranks[blk] = r;
        sizes[blk] = used[b] ? block_units(dtype, r, geo.len(b)) : 0;
    }
}

// One CTA per (layer, head, block): the flagged blocks' factors from the
// host arena (device-mapped pointers) to the staging area, and their scales.
// Offsets count offset units of esize bytes; every block's size is a
// multiple of 16 bytes (1024 elements, or 16 bytes of 2-bit codes), so
// 16-byte vectors tile it exactly.
__global__ void __launch_bounds__(256) k_stage_copy(KindView host, KindView stage, const int32_t *__restrict__ used,
                                                    int n_b, int esize) {
    const int64_t blk = blockIdx.x;
    if (!used[blk % n_b]) return;
    const int64_t dst0 = stage.offsets[blk], n16 = (stage.offsets[blk + 1] - dst0) * esize / 16;
    const uint4 *src = reinterpret_cast<const uint4 *>((const char *)host.data + host.offsets[blk] * esize);
    uint4 *dst = reinterpret_cast<uint4 *>((char *)stage.data + dst0 * esize);
    int64_t e = threadIdx.x;
    for (; e + 3 * 256 < n16; e += 4 * 256) {   // four loads in flight per thread
        const uint4 a0 = __ldg(src + e), a1 = __ldg(src + e + 256), a2 = __ldg(src + e + 512), a3 = __ldg(src + e + 768);
        dst[e] = a0;
        dst[e + 256] = a1;
        dst[e + 512] = a2;
        dst[e + 768] = a3;
    }
    for (; e < n16; e += 256) dst[e] = __ldg(src + e);
    if (threadIdx.x < D) {
        if (host.scaleA) stage.scaleA[blk * D + threadIdx.x] = host.scaleA[blk * D + threadIdx.x];
        if (host.scaleB) stage.scaleB[blk * D + threadIdx.x] = host.scaleB[blk * D + threadIdx.x];
    }
}

}  // namespace milo
