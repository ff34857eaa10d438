// Timeline of one CTA of k_decode_tc, for the tracing build only
// (-DMILO_DECODE_TRACE; block_wise_rank_b200/build.py builds it as
// libmilo_trace.so).  Lane 0 of every warp of the selected CTA appends
// (SM clock, event, item, tile) records to its own row; the events are the
// TlEvent list in decode_tc.cuh.  The product library compiles none of this.
#pragma once
#include <cstdint>

namespace milo {
constexpr int TL_WARPS = 20;     // k_decode_tc's warps
constexpr int TL_CAP = 4096;     // records per warp
struct TlRec {
    long long t;                 // clock64() of the recording SM
    uint32_t code;               // event | tile << 8
    uint32_t n;                  // the CTA's item sequence number
};
__device__ TlRec g_tl[TL_WARPS][TL_CAP];
__device__ uint32_t g_tl_cnt[TL_WARPS];
__device__ int g_tl_cta = -1;
}  // namespace milo

#define MILO_TL_LOCALS                                                                     \
    uint32_t tl_cnt = 0;                                                                   \
    const bool tl_on = (int)blockIdx.x == milo::g_tl_cta && (threadIdx.x & 31) == 0;
#define MILO_TL(ev, n_, t_)                                                                \
    do {                                                                                   \
        if (tl_on && tl_cnt < (uint32_t)milo::TL_CAP) {                                    \
            milo::TlRec &r_ = milo::g_tl[threadIdx.x >> 5][tl_cnt++];                      \
            r_.t = clock64();                                                              \
            r_.code = (uint32_t)(ev) | ((uint32_t)(t_) << 8);                              \
            r_.n = (uint32_t)(n_);                                                         \
            milo::g_tl_cnt[threadIdx.x >> 5] = tl_cnt;                                     \
        }                                                                                  \
    } while (0)
