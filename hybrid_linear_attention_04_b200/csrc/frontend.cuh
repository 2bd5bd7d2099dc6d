// q/k front-end of a packed prefill batch: short causal depthwise convolution, Swish
// and L2 normalisation (Kimi K3 technical FAQ, "What is KDA": queries and keys pass
// through a short convolution, Swish and L2 normalization). The definition and the
// conv-state layout are those of the decode-side front-end in decode.cuh: per head
// and key channel y_t = sum_j w[j] x_{t-(taps-1)+j} (tap taps-1 on the current token),
// z = y sigmoid(y), out = z / max(|z|, 1e-6) over the d_k channels of the token; a
// sequence's conv state is its last taps-1 raw inputs, oldest first, laid out
// [2 (q, k), H, D, taps-1] per sequence.
//
// One warp per (sequence, C-token tile, head, q or k), four per CTA; lane l owns the
// D/32 consecutive channels from D/32 l, with their weights and conv windows in
// registers (the window from the sequence's conv state for its first tile, from the
// rows before it otherwise). Rows go in groups of eight with all their loads issued
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
    static constexpr int WARPS = 4;          // independent (tile, head, q or k) items per CTA
    static constexpr int NT = 32 * WARPS;
    static constexpr int CPL = D / 32;       // channels per lane: CPL lane .. (CPL lane + CPL - 1)
    static constexpr int G = CPL == 4 ? 4 : 8;   // rows whose loads are issued together
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

// One warp per (tile, head, q or k): the two tensors go through the same conv, Swish and
// L2 norm independently, so each warp holds one tensor's weights and windows and keeps
// G rows of loads in flight. The tap count K is a template parameter, so that the window's
// shift through an unrolled row group is register renaming rather than moves.
template <int D, typename TIO, int K>
__global__ void __launch_bounds__(FrontendShape<D>::NT, 5) qk_frontend_kernel(const __grid_constant__ FrontendParams P) {
    using Sh = FrontendShape<D>;
    constexpr int CPL = Sh::CPL, G = Sh::G;
    const int H = P.H, C = P.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * Sh::WARPS + warp;
    const int which = (int)(item & 1);                      // 0: q, 1: k
    const int h = (int)((item >> 1) % H);
    const int64_t row = (item >> 1) / H;
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
    const TIO *x = static_cast<const TIO *>(which ? P.k : P.q);
    const float *wt = which ? P.wk : P.wq;
    // weights and windows of the lane's channels
    Win cw[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        float hist[kMaxTaps - 1] = {0.f, 0.f, 0.f};   // the window before the tile, oldest first
#pragma unroll
        for (int j = 0; j < kMaxTaps - 1; ++j) {
            if (j < K - 1) {
                if (b == 0) {
                    if (P.conv_in) hist[j] = P.conv_in[conv_index(2 * i + which, H, h, D, c0 + e, K) + j];
                } else {
                    const int64_t r = t0 - (K - 1) + j;         // inside this sequence (b * C >= K - 1)
                    hist[j] = IO<TIO>::ld(x + (r * H + h) * D + c0 + e);
                }
            }
        }
        win_load(cw[e], wt + ((int64_t)h * D + c0 + e) * K, hist, K);
    }
    // the lane's channels of the tile's rows: row r at src + r * stride (and likewise dst)
    const int64_t stride = (int64_t)H * D;
    const TIO *src = x + (t0 * H + h) * D + c0;
    TIO *dst = static_cast<TIO *>(which ? P.k_out : P.q_out) + (t0 * H + h) * D + c0;
    for (int r0 = 0; r0 < n; r0 += G) {
        float xv[G][CPL];
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (r0 + g < n) ld_vec<TIO, CPL>(src + (r0 + g) * stride, xv[g]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (r0 + g < n) {
                float z[CPL], ss = 0.f;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    z[e] = swish(conv_step(cw[e], K, xv[g][e]));
                    ss = fmaf(z[e], z[e], ss);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                // 1 / max(|z|, eps) as rsqrt(max(|z|^2, eps^2))
                st_vec<TIO, CPL>(dst + (r0 + g) * stride, z, rsqrtf(fmaxf(ss, kNormEps * kNormEps)));
            }
        }
    }
    // conv states: at a snapshot boundary that ends this tile, and after the last token
    auto put = [&](float *dst, int64_t srow) {
#pragma unroll
        for (int e = 0; e < CPL; ++e) win_store(cw[e], dst + conv_index(2 * srow + which, H, h, D, c0 + e, K), K);
    };
    const int64_t p_end = P.start_pos[i] + (int64_t)b * C + n;
    if (P.conv_snap && P.snap_interval > 0 && n == C && p_end % P.snap_interval == 0)
        put(P.conv_snap, P.snap_off[i] + p_end / P.snap_interval - P.start_pos[i] / P.snap_interval - 1);
    if (P.conv_out && (b + 1) * C >= len) put(P.conv_out, i);
}

}  // namespace kda
