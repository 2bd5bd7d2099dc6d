// q/k front-end of a packed prefill batch: short causal depthwise convolution, Swish
// and L2 normalisation (Kimi K3 technical FAQ, "What is KDA": queries and keys pass
// through a short convolution, Swish and L2 normalization). The definition and the
// conv-state layout are those of the decode-side front-end in decode.cuh: per head
// and key channel y_t = sum_j w[j] x_{t-(taps-1)+j} (tap taps-1 on the current token),
// z = y sigmoid(y), out = z / max(|z|, 1e-6) over the d_k channels of the token; a
// sequence's conv state is its last taps-1 raw inputs, oldest first, laid out
// [2 (q, k), H, D, taps-1] per sequence.
//
// One CTA (D threads; thread c owns channel c for q and k) per (sequence, C-token
// tile, head): the tile's raw rows are read once, coalesced, with the window of the
// previous taps-1 inputs in registers (from the sequence's conv state for its first
// tile, from the rows before it otherwise); Swish outputs are staged in shared memory;
// each warp then normalises whole rows and writes them out. The tile that ends on a
// snapshot boundary writes the conv state there, the last tile the final conv state.
#pragma once
#include "decode.cuh"
#include "prefill_common.cuh"

namespace kda {

struct FrontendParams {
    const void *q, *k;          // raw [T, H, D]
    void *q_out, *k_out;        // normalised [T, H, D], same element type
    const float *wq, *wk;       // [H, D, taps]
    const float *conv_in;       // [n_seq, 2, H, D, taps-1] or null (zeros)
    float *conv_out;            // [n_seq, 2, H, D, taps-1] or null
    float *conv_snap;           // [n_snap, 2, H, D, taps-1] or null
    int32_t H, taps, n_seq, C, tok_first, snap_interval;
    int32_t tok0[kPrefillSeqs];
    int32_t len[kPrefillSeqs];
    int64_t start_pos[kPrefillSeqs];
    int64_t snap_off[kPrefillSeqs];
};

template <int D>
struct FrontendShape {
    static constexpr int NT = D, NW = D / 32, ROWS = 64;
    static constexpr uint32_t smem_bytes = 2u * ROWS * D * 4u;   // Swish outputs of q and k
};

template <int D, typename TIO>
__global__ void __launch_bounds__(D) qk_frontend_kernel(const __grid_constant__ FrontendParams P) {
    using Sh = FrontendShape<D>;
    extern __shared__ float fsm[];
    float *zq = fsm, *zk = fsm + Sh::ROWS * D;
    const int H = P.H, K = P.taps, C = P.C;
    const int h = blockIdx.x % H, row = blockIdx.x / H;
    // owner sequence: the last one whose first tile row is <= row (rows of different
    // sequences never collide; see prefill_split.cuh for the same indexing)
    auto first_row = [&](int i) { return (P.tok0[i] - P.tok_first) / C + i; };
    int lo = 0, hi = P.n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first_row(mid) <= row) lo = mid; else hi = mid - 1;
    }
    const int i = lo, b = row - first_row(i), len = P.len[i];
    if (b < 0 || (b > 0 && b * C >= len)) return;          // an unused row (block-uniform)
    const int c = threadIdx.x, warp = c >> 5, lane = c & 31;
    const int n = max(0, min(C, len - b * C));
    const int64_t t0 = (int64_t)P.tok0[i] + (int64_t)b * C;
    const TIO *q = static_cast<const TIO *>(P.q), *k = static_cast<const TIO *>(P.k);
    ConvWin w;
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) {
        w.wq[j] = j < K ? P.wq[((int64_t)h * D + c) * K + j] : 0.f;
        w.wk[j] = j < K ? P.wk[((int64_t)h * D + c) * K + j] : 0.f;
    }
    // the window before the tile: conv state (first tile) or the raw rows before it
#pragma unroll
    for (int j = 0; j < kMaxTaps - 1; ++j) {
        float a = 0.f, bb = 0.f;
        if (j < K - 1) {
            if (b == 0) {
                if (P.conv_in) {
                    a = P.conv_in[conv_index(2 * i, H, h, D, c, K) + j];
                    bb = P.conv_in[conv_index(2 * i + 1, H, h, D, c, K) + j];
                }
            } else {
                const int64_t r = t0 - (K - 1) + j;         // inside this sequence (b * C >= K - 1)
                a = IO<TIO>::ld(q + (r * H + h) * D + c);
                bb = IO<TIO>::ld(k + (r * H + h) * D + c);
            }
        }
        w.hq[j] = a;
        w.hk[j] = bb;
    }
    for (int r = 0; r < n; ++r) {
        const int64_t off = ((t0 + r) * H + h) * D + c;
        zq[r * D + c] = swish(conv_step(w.wq, w.hq, K, IO<TIO>::ld(q + off)));
        zk[r * D + c] = swish(conv_step(w.wk, w.hk, K, IO<TIO>::ld(k + off)));
    }
    // conv states: at a snapshot boundary that ends this tile, and after the last token
    const int64_t p_end = P.start_pos[i] + (int64_t)b * C + n;
    if (P.conv_snap && P.snap_interval > 0 && n == C && p_end % P.snap_interval == 0) {
        const int64_t j = p_end / P.snap_interval - P.start_pos[i] / P.snap_interval - 1;
        const int64_t srow = P.snap_off[i] + j;
#pragma unroll
        for (int jj = 0; jj < kMaxTaps - 1; ++jj)
            if (jj < K - 1) {
                P.conv_snap[conv_index(2 * srow, H, h, D, c, K) + jj] = w.hq[jj];
                P.conv_snap[conv_index(2 * srow + 1, H, h, D, c, K) + jj] = w.hk[jj];
            }
    }
    if (P.conv_out && (b + 1) * C >= len) {
#pragma unroll
        for (int jj = 0; jj < kMaxTaps - 1; ++jj)
            if (jj < K - 1) {
                P.conv_out[conv_index(2 * i, H, h, D, c, K) + jj] = w.hq[jj];
                P.conv_out[conv_index(2 * i + 1, H, h, D, c, K) + jj] = w.hk[jj];
            }
    }
    __syncthreads();
    // L2 normalisation of whole rows, one warp per row
    TIO *qo = static_cast<TIO *>(P.q_out), *ko = static_cast<TIO *>(P.k_out);
    for (int r = warp; r < n; r += Sh::NW) {
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e = lane; e < D; e += 32) {
            sq = fmaf(zq[r * D + e], zq[r * D + e], sq);
            sk = fmaf(zk[r * D + e], zk[r * D + e], sk);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
            sk += __shfl_xor_sync(0xffffffffu, sk, o);
        }
        const float rq = 1.f / fmaxf(sqrtf(sq), kNormEps), rk = 1.f / fmaxf(sqrtf(sk), kNormEps);
        const int64_t base = ((t0 + r) * H + h) * D;
#pragma unroll
        for (int e = lane; e < D; e += 32) {
            IO<TIO>::st(qo + base + e, zq[r * D + e] * rq);
            IO<TIO>::st(ko + base + e, zk[r * D + e] * rk);
        }
    }
}

}  // namespace kda
