// KDA chunked prefill on the tcgen05 tensor cores (placeholder until the
// kernel lands: reports unsupported so the CUDA-core path runs).
#pragma once
#include "prefill_common.cuh"

namespace kda {

inline bool tc_prefill_supported(const kda_dims &) { return false; }

template <typename Gate>
inline kda_status launch_prefill_tc(PrefillParams &, const kda_dims &, int64_t, cudaStream_t, Gate) {
    return KDA_ERR_UNSUPPORTED;
}

}  // namespace kda
