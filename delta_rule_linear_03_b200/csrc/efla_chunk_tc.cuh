// efla_chunk_tc.cuh - tensor-core (tcgen05) chunked prefill for bf16 inputs.
#pragma once
#include "efla_common.cuh"

namespace efla {

inline bool tc_path_applies(bool bf16, int d_k, int d_v) { return false; }

inline efla_status_t launch_chunk_tc(const void *, const void *, const void *, const float *, const float *, void *,
                                     bool, float *, long, int, bool, cudaStream_t) {
    return EFLA_ERR_UNSUPPORTED;
}

}  // namespace efla
