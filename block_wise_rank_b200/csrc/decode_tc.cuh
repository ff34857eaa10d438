// decode_tc.cuh -- decode attention on tensor cores (bf16 / int8 factors).
#pragma once
#include "decode_simt.cuh"

namespace milo {

inline bool decode_tc_supported(const DecodeArgs &) { return false; }
inline cudaError_t decode_tc_set_attrs() { return cudaSuccess; }
inline milo_status launch_decode_tc(const DecodeArgs &, cudaStream_t) { return MILO_ERR_UNSUPPORTED; }

}  // namespace milo
