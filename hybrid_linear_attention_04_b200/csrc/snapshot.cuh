// Bit-exact copies of whole KDA states between pools (commit a verified token,
// restore a cached block-boundary snapshot into a live slot, save a live
// state). vLLM day-0 blog, "Kimi Delta Attention": prefix caching over
// recurrent state reuses snapshots taken at block boundaries.
#pragma once
#include "common.cuh"

namespace kda {

struct SnapshotParams {
    const int64_t *src_idx, *dst_idx;
    const float *src;
    float *dst;
    int64_t n_src, n_dst;
    int64_t elems4;  // float4 per state
};

// grid = (blocks per state, n); each CTA copies a strided share of one state.
__global__ void __launch_bounds__(256) snapshot_kernel(const __grid_constant__ SnapshotParams p) {
    const int i = blockIdx.y;
    const int64_t si = p.src_idx[i], di = p.dst_idx[i];
    if (si < 0 || si >= p.n_src || di < 0 || di >= p.n_dst) {
        if (threadIdx.x == 0 && blockIdx.x == 0) record_status(KDA_ERR_RANGE);
        return;
    }
    const float4 *s = reinterpret_cast<const float4 *>(p.src) + si * p.elems4;
    float4 *d = reinterpret_cast<float4 *>(p.dst) + di * p.elems4;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < p.elems4;
         e += (int64_t)gridDim.x * blockDim.x)
        d[e] = s[e];
}

}  // namespace kda
