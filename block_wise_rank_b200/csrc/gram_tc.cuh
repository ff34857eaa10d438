// gram_tc.cuh -- per-block Gram matrices on tcgen05 tensor cores (bf16).
#pragma once
#include "common.cuh"

namespace milo {

inline bool gram_tc_supported(int /*block_len*/) { return false; }
inline cudaError_t gram_tc_set_attrs() { return cudaSuccess; }
inline milo_status launch_gram_tc(const __nv_bfloat16 *, const __nv_bfloat16 *, int, int, int, int, float *,
                                  int64_t, cudaStream_t) {
    return MILO_ERR_UNSUPPORTED;
}

}  // namespace milo
