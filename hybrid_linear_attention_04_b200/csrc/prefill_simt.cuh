// KDA chunked prefill on CUDA cores in fp32 (every dims/io combination; the
// all-fp32 path, and the checkable generic path for the tensor-core kernel).
//
// One CTA per (sequence, head, 32-column slice of d_v): the recurrence is
// independent across d_v columns, so slices run in parallel and each keeps its
// D x 32 fp32 state slice in shared memory across chunks. Per chunk it follows
// the chunk form in prefill_common.cuh with exact pairwise decays
// exp(b_rc - b_ic) (no reference-point factorisation, so no range condition
// on the gates), taken as 2^x of the cumsum in log2 units, and a forward
// substitution for the unit lower-triangular solve: one thread per d_v column with
// the column in registers, each solved row subtracted from the rows below it.
// Where a chunk's inputs are at most 16 values per thread and tensor, the next
// chunk's loads are issued into registers before this chunk's arithmetic, so
// their latency is hidden (the small shapes, whose chunks are latency-bound).
#pragma once
#include "prefill_common.cuh"

namespace kda {

template <int D, int C> struct SimtShape {
    static constexpr int NT = 256;
    static constexpr int DVS = 32;           // d_v columns per CTA
    static constexpr int DP = D + 1;         // padded row stride (bank-conflict free columns)
    static constexpr int CP = C + 1;
    static constexpr size_t floats =
        (size_t)D * DVS + 3 * (size_t)C * DP + 2 * (size_t)C * DVS + 2 * (size_t)C * CP + C + 2 * D;
    static constexpr size_t smem_bytes = floats * sizeof(float);
    static_assert(NT == 8 * DVS, "forward substitution uses 8 lanes per column");
};

template <int D, int C, typename TIO>
__global__ void __launch_bounds__(256)
prefill_simt_kernel(const __grid_constant__ PrefillParams p) {
    using Sh = SimtShape<D, C>;
    constexpr int NT = Sh::NT, DVS = Sh::DVS, DP = Sh::DP, CP = Sh::CP, NS = D / DVS;
    extern __shared__ float smem[];
    float *S = smem;                 // [D][DVS]   state slice
    float *Q = S + D * DVS;          // [C][DP]    q, then q . Gamma
    float *K = Q + C * DP;           // [C][DP]    k, then k . Gamma
    float *B = K + C * DP;           // [C][DP]    b (cumsum g), then k . exp(b_C - b)
    float *V = B + C * DP;           // [C][DVS]
    float *W = V + C * DVS;          // [C][DVS]
    float *Akk = W + C * DVS;        // [C][CP]    Diag(beta) A_kk (strict lower)
    float *Aqk = Akk + C * CP;       // [C][CP]    A_qk (lower incl. diagonal)
    float *bet = Aqk + C * CP;       // [C]
    float *gC = bet + C;             // [D]        Gamma_C
    float *bC = gC + D;              // [D]        b_C

    const int tid = threadIdx.x;
    const int item = blockIdx.x;
    const int rank = item / (p.H * NS);
    const int h = (item / NS) % p.H;
    const int j0 = (item % NS) * DVS;
    const int s = p.order[rank];
    const PrefillSeq sq = p.seq[s];
    const int H = p.H;
    const TIO *qg = static_cast<const TIO *>(p.q);
    const TIO *kg = static_cast<const TIO *>(p.k);
    const TIO *vg = static_cast<const TIO *>(p.v);
    TIO *og = static_cast<TIO *>(p.o);

    // initial state slice
    for (int e = tid; e < D * DVS; e += NT) {
        const int c = e / DVS, j = e % DVS;
        S[e] = p.state_in ? p.state_in[(((int64_t)s * H + h) * D + c) * D + j0 + j] : 0.f;
    }
    int64_t snap_row = sq.snap_off;
    constexpr float LOG2E = 1.4426950408889634f;

    // inputs of chunk c0 into registers (element e = tid + NT u of the C x D and C x DVS
    // tiles; rows >= n are zero: an identity token)
    constexpr int PQ = C * D / NT, PV = C * DVS / NT;
    constexpr bool PF = PQ <= 16;
    float rq[PF ? PQ : 1], rk[PF ? PQ : 1], rg[PF ? PQ : 1], rv[PF ? PV : 1], rb = 0.f;
    auto fetch = [&](int c0) {
        const int n = min(C, sq.len - c0);
#pragma unroll
        for (int u = 0; u < (PF ? PQ : 0); ++u) {
            const int e = tid + NT * u, r = e / D, c = e % D;
            rq[u] = rk[u] = rg[u] = 0.f;
            if (r < n) {
                const int64_t off = ((int64_t)(sq.tok0 + c0 + r) * H + h) * D + c;
                rq[u] = IO<TIO>::ld(qg + off);
                rk[u] = IO<TIO>::ld(kg + off);
                rg[u] = p.g[off];
            }
        }
#pragma unroll
        for (int u = 0; u < (PF ? PV : 0); ++u) {
            const int e = tid + NT * u, r = e / DVS, j = e % DVS;
            rv[u] = r < n ? IO<TIO>::ld(vg + ((int64_t)(sq.tok0 + c0 + r) * H + h) * D + j0 + j) : 0.f;
        }
        rb = tid < n ? p.beta[(int64_t)(sq.tok0 + c0 + tid) * H + h] : 0.f;
    };
    if (PF && sq.len > 0) fetch(0);

    for (int c0 = 0; c0 < sq.len; c0 += C) {
        const int n = min(C, sq.len - c0);
        __syncthreads();
        // ---- the chunk into shared memory (g in log2 units) ----
        if (PF) {
#pragma unroll
            for (int u = 0; u < (PF ? PQ : 0); ++u) {
                const int e = tid + NT * u, r = e / D, c = e % D;
                Q[r * DP + c] = rq[u];
                K[r * DP + c] = rk[u];
                B[r * DP + c] = rg[u] * LOG2E;
            }
#pragma unroll
            for (int u = 0; u < (PF ? PV : 0); ++u) V[tid + NT * u] = rv[u];
            if (tid < C) bet[tid] = rb;
            if (c0 + C < sq.len) fetch(c0 + C);      // lands while this chunk computes
        } else {
            for (int e = tid; e < C * D; e += NT) {
                const int r = e / D, c = e % D;
                float qv = 0.f, kv = 0.f, gv = 0.f;
                if (r < n) {
                    const int64_t off = ((int64_t)(sq.tok0 + c0 + r) * H + h) * D + c;
                    qv = IO<TIO>::ld(qg + off);
                    kv = IO<TIO>::ld(kg + off);
                    gv = p.g[off];
                }
                Q[r * DP + c] = qv;
                K[r * DP + c] = kv;
                B[r * DP + c] = gv * LOG2E;
            }
            for (int e = tid; e < C * DVS; e += NT) {
                const int r = e / DVS, j = e % DVS;
                V[e] = r < n ? IO<TIO>::ld(vg + ((int64_t)(sq.tok0 + c0 + r) * H + h) * D + j0 + j) : 0.f;
            }
            for (int r = tid; r < C; r += NT)
                bet[r] = r < n ? p.beta[(int64_t)(sq.tok0 + c0 + r) * H + h] : 0.f;
        }
        __syncthreads();
        // ---- b = inclusive cumsum of g over the chunk, per channel (log2 units) ----
        for (int c = tid; c < D; c += NT) {
            float run = 0.f;
            for (int r = 0; r < C; ++r) {
                run += B[r * DP + c];
                B[r * DP + c] = run;
            }
            bC[c] = run;
            gC[c] = tc::ex2(run);
        }
        __syncthreads();
        // ---- A_kk (scaled by beta_r) and A_qk with exact pairwise decays ----
        for (int e = tid; e < C * C; e += NT) {
            const int r = e / C, i = e % C;
            float kk = 0.f, qk = 0.f;
            if (i <= r) {
                for (int c = 0; c < D; ++c) {
                    const float ex = tc::ex2(B[r * DP + c] - B[i * DP + c]);
                    const float ki = K[i * DP + c] * ex;
                    kk = fmaf(K[r * DP + c], ki, kk);
                    qk = fmaf(Q[r * DP + c], ki, qk);
                }
            }
            Akk[r * CP + i] = i < r ? bet[r] * kk : 0.f;
            Aqk[r * CP + i] = i <= r ? qk : 0.f;
        }
        __syncthreads();
        // ---- Q . Gamma, K . Gamma, and K . exp(b_C - b) (into B) ----
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, c = e % D;
            const float b = B[r * DP + c];
            const float ga = tc::ex2(b);
            const float kv = K[r * DP + c];
            Q[r * DP + c] *= ga;
            K[r * DP + c] = kv * ga;
            B[r * DP + c] = kv * tc::ex2(bC[c] - b);
        }
        __syncthreads();
        // ---- right-hand side: beta (V - (K . Gamma) S_0) ----
        for (int e = tid; e < C * DVS; e += NT) {
            const int r = e / DVS, j = e % DVS;
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc = fmaf(K[r * DP + c], S[c * DVS + j], acc);
            W[e] = bet[r] * (V[e] - acc);
        }
        __syncthreads();
        // ---- forward substitution: W <- (I + Diag(beta) A_kk)^{-1} W, one thread per
        // column: row i, once solved, is subtracted from every row below it ----
        if (tid < DVS) {
            float w[C];
#pragma unroll
            for (int r = 0; r < C; ++r) w[r] = W[r * DVS + tid];
#pragma unroll
            for (int i = 0; i < C - 1; ++i)
#pragma unroll
                for (int r = i + 1; r < C; ++r) w[r] = fmaf(-Akk[r * CP + i], w[i], w[r]);
#pragma unroll
            for (int r = 0; r < C; ++r) W[r * DVS + tid] = w[r];
        }
        __syncthreads();
        // ---- outputs: scale [ (Q . Gamma) S_0 + A_qk W ] ----
        for (int e = tid; e < n * DVS; e += NT) {
            const int r = e / DVS, j = e % DVS;
            float a1 = 0.f, a2 = 0.f;
            for (int c = 0; c < D; ++c) a1 = fmaf(Q[r * DP + c], S[c * DVS + j], a1);
            for (int i = 0; i <= r; ++i) a2 = fmaf(Aqk[r * CP + i], W[i * DVS + j], a2);
            IO<TIO>::st(og + ((int64_t)(sq.tok0 + c0 + r) * H + h) * D + j0 + j, p.scale * (a1 + a2));
        }
        __syncthreads();
        // ---- state: S_C = Diag(Gamma_C) S_0 + (K . exp(b_C - b))^T W ----
        for (int e = tid; e < D * DVS; e += NT) {
            const int c = e / DVS, j = e % DVS;
            float acc = 0.f;
            for (int r = 0; r < C; ++r) acc = fmaf(B[r * DP + c], W[r * DVS + j], acc);
            S[e] = fmaf(gC[c], S[e], acc);
        }
        __syncthreads();
        // ---- snapshot at a block boundary (only full chunks can end on one) ----
        if (p.snap_interval > 0 && (sq.start_pos + c0 + n) % p.snap_interval == 0) {
            float *dst = p.snapshots + (snap_row * H + h) * (int64_t)D * D;
            for (int e = tid; e < D * DVS; e += NT) dst[(e / DVS) * D + j0 + e % DVS] = S[e];
            ++snap_row;
        }
    }
    __syncthreads();
    if (p.state_out) {
        float *dst = p.state_out + ((int64_t)s * H + h) * (int64_t)D * D;
        for (int e = tid; e < D * DVS; e += NT) dst[(e / DVS) * D + j0 + e % DVS] = S[e];
    }
}

}  // namespace kda
