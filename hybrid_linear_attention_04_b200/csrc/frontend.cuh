// q/k front-end of a packed prefill batch: short causal depthwise convolution, Swish
// and L2 normalisation (Kimi K3 technical FAQ, "What is KDA": queries and keys pass
// through a short convolution, Swish and L2 normalization). The definition and the
// conv-state layout are those of the decode-side front-end in decode.cuh: per head
// and key channel y_t = sum_j w[j] x_{t-(taps-1)+j} (tap taps-1 on the current token),
// z = y sigmoid(y), out = z / max(|z|, 1e-6) over the d_k channels of the token; a
// sequence's conv state is its last taps-1 raw inputs, oldest first, laid out
// [2 (q, k), H, D, taps-1] per sequence.
//
// One warp per (sequence, C-token tile, head), four per CTA; lane l owns the D/32
// consecutive channels from D/32 l for q and k, with their weights and conv windows in
// registers (the window from the sequence's conv state for its first tile, from the
// rows before it otherwise). Rows go in groups of four with all their loads issued
// first; each row's L2 norm is a warp reduction. The tile that ends on a snapshot
// boundary writes the conv state there, the last tile the final conv state.
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
    static constexpr int WARPS = 4;          // independent (tile, head) items per CTA
    static constexpr int NT = 32 * WARPS;
    static constexpr int CPL = D / 32;       // channels per lane: 4 lane .. (CPL lane + CPL - 1)
    static constexpr int G = 4;              // rows whose loads are issued together
};

// CPL consecutive elements of a row (one vector access)
template <typename TIO, int CPL>
__device__ __forceinline__ void ld_vec(const TIO *p, float (&x)[CPL]) {
    if (CPL == 4) {
        const float4 v = IO<TIO>::ld4(p);
        x[0] = v.x; x[1] = v.y; x[2 % CPL] = v.z; x[3 % CPL] = v.w;
    } else {
#pragma unroll
        for (int e = 0; e < CPL; ++e) x[e] = IO<TIO>::ld(p + e);
    }
}
template <typename TIO, int CPL>
__device__ __forceinline__ void st_vec(TIO *p, const float (&x)[CPL], float s) {
    if (CPL == 4) {
        IO<TIO>::st4(p, make_float4(x[0] * s, x[1 % CPL] * s, x[2 % CPL] * s, x[3 % CPL] * s));
    } else {
#pragma unroll
        for (int e = 0; e < CPL; ++e) IO<TIO>::st(p + e, x[e] * s);
    }
}

template <int D, typename TIO>
__global__ void __launch_bounds__(FrontendShape<D>::NT) qk_frontend_kernel(const __grid_constant__ FrontendParams P) {
    using Sh = FrontendShape<D>;
    constexpr int CPL = Sh::CPL, G = Sh::G;
    const int H = P.H, K = P.taps, C = P.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * Sh::WARPS + warp;
    const int h = (int)(item % H);
    const int64_t row = item / H;
    // owner sequence: the last one whose first tile row is <= row (rows of different
    // sequences never collide; see prefill_split.cuh for the same indexing)
    auto first_row = [&](int i) { return (int64_t)(P.tok0[i] - P.tok_first) / C + i; };
    int lo = 0, hi = P.n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first_row(mid) <= row) lo = mid; else hi = mid - 1;
    }
    const int i = lo, len = P.len[i];
    const int64_t bt = row - first_row(i);
    if (bt < 0 || (bt > 0 && bt * C >= len)) return;        // an unused row (warp-uniform)
    const int b = (int)bt;
    const int n = max(0, min(C, len - b * C));
    const int64_t t0 = (int64_t)P.tok0[i] + (int64_t)b * C;
    const int c0 = CPL * lane;
    const TIO *q = static_cast<const TIO *>(P.q), *k = static_cast<const TIO *>(P.k);
    // weights and windows of the lane's channels
    Win cq[CPL], ck[CPL];
    float hist[kMaxTaps - 1][2][CPL];      // the window before the tile, oldest first
#pragma unroll
    for (int j = 0; j < kMaxTaps - 1; ++j) {
#pragma unroll
        for (int e = 0; e < CPL; ++e) hist[j][0][e] = hist[j][1][e] = 0.f;
        if (j < K - 1) {
            if (b == 0) {
                if (P.conv_in) {
#pragma unroll
                    for (int e = 0; e < CPL; ++e) {
                        hist[j][0][e] = P.conv_in[conv_index(2 * i, H, h, D, c0 + e, K) + j];
                        hist[j][1][e] = P.conv_in[conv_index(2 * i + 1, H, h, D, c0 + e, K) + j];
                    }
                }
            } else {
                const int64_t r = t0 - (K - 1) + j;             // inside this sequence (b * C >= K - 1)
                ld_vec<TIO, CPL>(q + (r * H + h) * D + c0, hist[j][0]);
                ld_vec<TIO, CPL>(k + (r * H + h) * D + c0, hist[j][1]);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        const float sq[3] = {hist[0][0][e], hist[1][0][e], hist[2][0][e]};
        const float sk[3] = {hist[0][1][e], hist[1][1][e], hist[2][1][e]};
        win_load(cq[e], P.wq + ((int64_t)h * D + c0 + e) * K, sq, K);
        win_load(ck[e], P.wk + ((int64_t)h * D + c0 + e) * K, sk, K);
    }
    TIO *qo = static_cast<TIO *>(P.q_out), *ko = static_cast<TIO *>(P.k_out);
    for (int r0 = 0; r0 < n; r0 += G) {
        float xq[G][CPL], xk[G][CPL];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (r0 + g < n) {
                const int64_t off = ((t0 + r0 + g) * H + h) * D + c0;
                ld_vec<TIO, CPL>(q + off, xq[g]);
                ld_vec<TIO, CPL>(k + off, xk[g]);
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (r0 + g < n) {
                float zq[CPL], zk[CPL], sq = 0.f, sk = 0.f;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    zq[e] = swish(conv_step(cq[e], K, xq[g][e]));
                    zk[e] = swish(conv_step(ck[e], K, xk[g][e]));
                    sq = fmaf(zq[e], zq[e], sq);
                    sk = fmaf(zk[e], zk[e], sk);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                    sk += __shfl_xor_sync(0xffffffffu, sk, o);
                }
                const int64_t off = ((t0 + r0 + g) * H + h) * D + c0;
                st_vec<TIO, CPL>(qo + off, zq, 1.f / fmaxf(sqrtf(sq), kNormEps));
                st_vec<TIO, CPL>(ko + off, zk, 1.f / fmaxf(sqrtf(sk), kNormEps));
            }
        }
    }
    // conv states: at a snapshot boundary that ends this tile, and after the last token
    auto put = [&](float *dst, int64_t srow) {
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
            win_store(cq[e], dst + conv_index(2 * srow, H, h, D, c0 + e, K), K);
            win_store(ck[e], dst + conv_index(2 * srow + 1, H, h, D, c0 + e, K), K);
        }
    };
    const int64_t p_end = P.start_pos[i] + (int64_t)b * C + n;
    if (P.conv_snap && P.snap_interval > 0 && n == C && p_end % P.snap_interval == 0)
        put(P.conv_snap, P.snap_off[i] + p_end / P.snap_interval - P.start_pos[i] / P.snap_interval - 1);
    if (P.conv_out && (b + 1) * C >= len) put(P.conv_out, i);
}

}  // namespace kda
