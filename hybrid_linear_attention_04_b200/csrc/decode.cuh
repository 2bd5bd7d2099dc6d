// KDA decode and speculative-verify kernels (sm_100a, SIMT, HBM-bound).
//
// A CTA owns one (sequence, head) state S [D x D] fp32 (d_v contiguous) at a time and
// streams it through registers once: 128-bit loads, gate, rank-1 delta correction and
// output read in one pass per token, 128-bit stores.
//
// Per token (Kimi K3 technical FAQ, "What is KDA": delta rule with a
// per-channel forget gate; standard gated-delta form):
//     S' = Diag(alpha) S                    alpha = exp(g), per key channel
//     x  = S'^T k,   y = S'^T q             (one pass, shared reduction over d_k)
//     w  = beta (v - x)
//     S  = S' + k w^T
//     o  = scale (y + (k . q) w)            (= scale * S^T q, read after update)
//
// The d_v columns of S evolve independently (w, the update and o are per column),
// so warp w owns the 16 columns 16w .. 16w+15 over all d_k rows: lane l holds columns
// 16w + 4 (l % 4) .. +3 of rows l / 4 + 8 m, m < D / 8, as f32x2 pairs of rows. The
// column sums over d_k reduce inside the lane, then across the 8 lanes that share the
// column group (a reduce-scatter and a gather of shuffles); a token step has no barrier
// and no shared-memory reduction. Decode, verify and the commit replay run the same
// step function, so verify's state after its j-th token is bit-identical to j decode
// calls.
//
// Token vectors sit in shared memory (decode: one token; verify: batches of TMA-loaded
// rows): threads t < D own channel t of q and k (and run the q/k front-end's conv
// window in token order), threads t >= D channel t - D of v and g.
#pragma once
#include "common.cuh"
#include "tc_util.cuh"

namespace kda {

constexpr int kMaxSeqsPerLaunch = KDA_SEQS_PER_LAUNCH;

template <int D> struct DecodeShape {
    static constexpr int NT = 2 * D;     // threads per CTA: 256, 128, 64
    static constexpr int NW = NT / 32;   // warps, 16 d_v columns each
    static constexpr int R = D / 8;      // rows per lane
    static_assert(NW * 16 == D, "warps must tile the columns");
};

struct DecodeParams {
    const void *q, *k, *v;
    const float *g, *beta;
    const int32_t *slots;
    float *pool;             // decode: read/write; verify: read-only source
    float *token_states;     // verify only
    void *o;
    int32_t n_seq, H, n_slots;
    float scale;
    int32_t tok0[kMaxSeqsPerLaunch + 1];  // verify: packed token offsets (relative)
    int64_t tok_base;                     // verify: absolute offset of tok0[0]
    // q/k front-end (taps == 0: q and k are used as given)
    int32_t taps;
    const float *wq, *wk;    // [H, D, taps] conv weights
    float *conv;             // conv states [n_slots, 2, H, D, taps-1]: decode and verify+commit
                             // update them in place, verify only reads them
    float *conv_tok;         // verify: conv state after each token [T, 2, H, D, taps-1] (nullable)
};

// ---- q/k front-end (Kimi K3 technical FAQ, "What is KDA": queries and keys pass
// through a short convolution, Swish and L2 normalisation). Per head and key channel,
// a causal depthwise convolution y_t = sum_j w[j] x_{t-(taps-1)+j} (tap taps-1 on the
// current token, no bias) over the raw inputs, z = y sigmoid(y), then z / max(|z|, 1e-6)
// over the d_k channels of the token. The conv state of a sequence is its last taps-1
// raw inputs, oldest first. Thread c < D owns channel c: its weights and window are
// registers, and tokens pass through it in order.
constexpr int kMaxTaps = 4;
constexpr float kNormEps = 1e-6f;

// One channel's conv weights (tap 0 .. taps-1) and window (its last taps-1 raw inputs,
// oldest first), as scalars with the tap count branched on explicitly: an array form
// indexed through the runtime tap count lands in local memory.
struct Win {
    float w0, w1, w2, w3, h0, h1, h2;
};
struct ConvWin {
    Win q, k;
};

__device__ __forceinline__ int64_t conv_index(int64_t row2, int H, int h, int D, int c, int taps) {
    // row2 = 2 * (slot or token) + (0 for q, 1 for k)
    return ((row2 * H + h) * D + c) * (int64_t)(taps - 1);
}

// weights w[0..K-1] and the window state[0..K-2] (null: zeros)
__device__ __forceinline__ void win_load(Win &c, const float *w, const float *state, int K) {
    c.w0 = w[0];
    c.w1 = w[1];
    c.w2 = K > 2 ? w[2] : 0.f;
    c.w3 = K > 3 ? w[3] : 0.f;
    c.h0 = state ? state[0] : 0.f;
    c.h1 = (state && K > 2) ? state[1] : 0.f;
    c.h2 = (state && K > 3) ? state[2] : 0.f;
}
__device__ __forceinline__ void win_store(const Win &c, float *dst, int K) {
    dst[0] = c.h0;
    if (K > 2) dst[1] = c.h1;
    if (K > 3) dst[2] = c.h2;
}

// one causal conv step: y = sum_j w_j x_{t-(K-1)+j} over the window and x, then shift x in
__device__ __forceinline__ float conv_step(Win &c, int K, float x) {
    float y;
    if (K == 4) {
        y = c.w3 * x;
        y = fmaf(c.w0, c.h0, y); y = fmaf(c.w1, c.h1, y); y = fmaf(c.w2, c.h2, y);
        c.h0 = c.h1; c.h1 = c.h2; c.h2 = x;
    } else if (K == 3) {
        y = c.w2 * x;
        y = fmaf(c.w0, c.h0, y); y = fmaf(c.w1, c.h1, y);
        c.h0 = c.h1; c.h1 = x;
    } else {
        y = c.w1 * x;
        y = fmaf(c.w0, c.h0, y);
        c.h0 = x;
    }
    return y;
}

// weights and windows of channel c from conv state row `row` (slot or token) of `src`
__device__ __forceinline__ void conv_begin(ConvWin &w, const DecodeParams &p, const float *src, int64_t row,
                                           int h, int D, int c) {
    const int K = p.taps;
    win_load(w.q, p.wq + ((int64_t)h * D + c) * K, src + conv_index(2 * row, p.H, h, D, c, K), K);
    win_load(w.k, p.wk + ((int64_t)h * D + c) * K, src + conv_index(2 * row + 1, p.H, h, D, c, K), K);
}

__device__ __forceinline__ void conv_store(const ConvWin &w, const DecodeParams &p, float *dst, int64_t row,
                                           int h, int D, int c) {
    const int K = p.taps;
    win_store(w.q, dst + conv_index(2 * row, p.H, h, D, c, K), K);
    win_store(w.k, dst + conv_index(2 * row + 1, p.H, h, D, c, K), K);
}

// y sigmoid(y) with the fast exponential and division (a few ulp; the features go on as
// bf16 or into fp32 sums whose own rounding is larger). y below about -87 gives 0.
__device__ __forceinline__ float swish(float y) { return __fdividef(y, 1.f + __expf(-y)); }

// Where the front-end's conv state goes while a batch is staged (front-end on only):
// after every token into rows tok0 + j of `tok` (nullable), and after token snap_j
// (batch-relative; -1 = none) into row snap_row of `snap`.
struct ConvOut {
    float *tok;
    int64_t tok0;
    float *snap;
    int64_t snap_row;
    int snap_j;
};

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) --------------------------------
// One instruction does the work of two fp32 lanes; each element is rounded exactly as
// the scalar fmul / fmaf would round it, so the pairing changes no result bit.
using f2 = unsigned long long;
__device__ __forceinline__ f2 pk2(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 up2(f2 x) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(x));
    return r;
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ---- per-token vectors in shared memory ----------------------------------------
// A lane reads the gate a = exp(g), k and q at its rows rg + 8 m (rg = lane / 4,
// m < D / 8). They are stored permuted, channel c at (c % 8) * STR + c / 8, so that one
// 128-bit load gives a lane rows m .. m + 3; STR pads each row group so that the 8
// distinct addresses of a warp's load, and a warp's 32 scalar stores, hit distinct banks.
template <int D> struct TokLayout {
    static constexpr int R = D / 8;                                  // rows per lane
    static constexpr int STR = ((R + 4) / 4) % 2 ? R + 4 : R + 8;   // floats per row group
    static constexpr int SZ = 8 * STR;
    static_assert(R % 4 == 0 && (STR * 4) % 16 == 0, "128-bit rows");
};
template <int D> __device__ __forceinline__ int perm(int c) { return (c & 7) * TokLayout<D>::STR + (c >> 3); }

template <int D> struct __align__(16) TokVec {
    float a[TokLayout<D>::SZ], k[TokLayout<D>::SZ], q[TokLayout<D>::SZ];   // permuted
    float v[D];                                                          // natural order
    float beta, kq, pad0, pad1;
};

// Channel c of q and k into a token vector: with CONV through the front-end's conv window
// and Swish (token_finish normalises), else as given. with_q false: q is zero (a replayed
// token whose output is not needed; its raw q still moves the conv window).
template <int D, bool CONV>
__device__ __forceinline__ void put_qk(TokVec<D> &tv, int c, float xq, float xk, bool with_q, ConvWin &w,
                                       int taps) {
    float q = xq, k = xk;
    if (CONV) {
        const float yq = conv_step(w.q, taps, xq);
        const float yk = conv_step(w.k, taps, xk);
        q = swish(yq);
        k = swish(yk);
    }
    tv.q[perm<D>(c)] = with_q ? q : 0.f;
    tv.k[perm<D>(c)] = k;
}
template <int D>
__device__ __forceinline__ void put_vg(TokVec<D> &tv, int c, float xv, float xg) {
    tv.v[c] = xv;
    tv.a[perm<D>(c)] = expf(xg);
}

// One warp finishes a staged token: L2-normalises k and q when the front-end is on,
// then k . q (fixed reduction order) when q is used.
template <int D>
__device__ __forceinline__ void token_finish(TokVec<D> &tv, bool normalise, bool with_q) {
    const int lane = threadIdx.x & 31;
    if (normalise) {
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int c = lane; c < D; c += 32) {
            const float k = tv.k[perm<D>(c)], q = tv.q[perm<D>(c)];
            sk = fmaf(k, k, sk);
            sq = fmaf(q, q, sq);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float rk = 1.f / fmaxf(sqrtf(sk), kNormEps), rq = 1.f / fmaxf(sqrtf(sq), kNormEps);
#pragma unroll
        for (int c = lane; c < D; c += 32) {
            tv.k[perm<D>(c)] *= rk;
            tv.q[perm<D>(c)] *= rq;
        }
        __syncwarp();
    }
    if (with_q) {
        float s = 0.f;
#pragma unroll
        for (int c = lane; c < D; c += 32) s = fmaf(tv.k[perm<D>(c)], tv.q[perm<D>(c)], s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) tv.kq = s;
    }
}

// ---- the state in registers ------------------------------------------------------
// Lane (warp w, rg = lane / 4, cg = lane % 4) holds columns 16 w + 4 cg + e (e < 4) of
// rows rg + 8 m (m < R): P[i][e] pairs rows m = 2 i (low half) and 2 i + 1 (high half)
// of column e, so the gate, both column sums and the rank-1 update run as f32x2 pairs.
template <int D> using StatePairs = f2[TokLayout<D>::R / 2][4];

template <int D>
__device__ __forceinline__ int64_t lane_off(int m) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    return (int64_t)((lane >> 2) + 8 * m) * D + 16 * warp + 4 * (lane & 3);
}
__device__ __forceinline__ int lane_col() { return 16 * (threadIdx.x >> 5) + 4 * (threadIdx.x & 3); }

__device__ __forceinline__ void set_rows(f2 (&p)[4], const float4 &e, const float4 &o) {
    p[0] = pk2(e.x, o.x); p[1] = pk2(e.y, o.y); p[2] = pk2(e.z, o.z); p[3] = pk2(e.w, o.w);
}
__device__ __forceinline__ void get_rows(const f2 (&p)[4], float4 &e, float4 &o) {
    const float2 a = up2(p[0]), b = up2(p[1]), c = up2(p[2]), d = up2(p[3]);
    e = make_float4(a.x, b.x, c.x, d.x);
    o = make_float4(a.y, b.y, c.y, d.y);
}
// from global memory (read once: no L1 allocation)
template <int D>
__device__ __forceinline__ void load_state(StatePairs<D> &P, const float *S) {
#pragma unroll
    for (int i = 0; i < TokLayout<D>::R / 2; ++i) {
        float4 e, o;
        const float *se = S + lane_off<D>(2 * i), *so = S + lane_off<D>(2 * i + 1);
        asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(e.x), "=f"(e.y), "=f"(e.z), "=f"(e.w) : "l"(se));
        asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(o.x), "=f"(o.y), "=f"(o.z), "=f"(o.w) : "l"(so));
        set_rows(P[i], e, o);
    }
}
// from a row-major copy in shared memory
template <int D>
__device__ __forceinline__ void load_state_smem(StatePairs<D> &P, const float *S) {
#pragma unroll
    for (int i = 0; i < TokLayout<D>::R / 2; ++i)
        set_rows(P[i], *reinterpret_cast<const float4 *>(S + lane_off<D>(2 * i)),
                 *reinterpret_cast<const float4 *>(S + lane_off<D>(2 * i + 1)));
}
template <int D>
__device__ __forceinline__ void store_state(const StatePairs<D> &P, float *S) {
#pragma unroll
    for (int i = 0; i < TokLayout<D>::R / 2; ++i) {
        float4 e, o;
        get_rows(P[i], e, o);
        st_stream(S + lane_off<D>(2 * i), e);
        st_stream(S + lane_off<D>(2 * i + 1), o);
    }
}

// One recurrence step on the register-resident columns of this warp. With OUT =
// false the output read (y and o) is skipped; the state arithmetic is the same
// instruction for instruction, so both forms give bit-identical states.
//
// The column sums over d_k reduce inside the lane (two row halves, then added), then over
// the 8 lanes of a column group (rg = lane / 4) as a reduce-scatter: at each of lane bits
// 2, 3, 4 (rg bits 0, 1, 2) a lane keeps half of its partial sums and adds the partner's
// copy of them, so the 8 sums (x and y of 4 columns) end one per lane after 7 shuffles,
// and the 4 x sums go back to every lane by 4 indexed shuffles. Every sum has the same
// addition tree (rows paired by rg bit 0, then 1, then 2) in both forms and in every lane
// that holds it, so OUT changes no bit of x. With OUT the lane whose rg is odd holds y of
// column `oe` of its group and returns that column's output; the other lanes return 0.
template <int D, bool OUT = true>
__device__ __forceinline__ float kda_step(StatePairs<D> &P, const TokVec<D> &tv, float scale, int &oe) {
    using L = TokLayout<D>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rg = lane >> 2, cg = lane & 3;
    const bool b0 = rg & 1, b1 = (rg >> 1) & 1, b2 = (rg >> 2) & 1;
    const float *ap = tv.a + rg * L::STR, *kp = tv.k + rg * L::STR, *qp = tv.q + rg * L::STR;
    f2 xa[4] = {0ull, 0ull, 0ull, 0ull}, ya[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int i = 0; i < L::R / 4; ++i) {
        const float4 a4 = *reinterpret_cast<const float4 *>(ap + 4 * i);
        const float4 k4 = *reinterpret_cast<const float4 *>(kp + 4 * i);
        const f2 a01 = pk2(a4.x, a4.y), a23 = pk2(a4.z, a4.w);
        const f2 k01 = pk2(k4.x, k4.y), k23 = pk2(k4.z, k4.w);
        f2 q01 = 0ull, q23 = 0ull;
        if (OUT) {
            const float4 q4 = *reinterpret_cast<const float4 *>(qp + 4 * i);
            q01 = pk2(q4.x, q4.y);
            q23 = pk2(q4.z, q4.w);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const f2 s0 = mul2(P[2 * i][e], a01), s1 = mul2(P[2 * i + 1][e], a23);
            P[2 * i][e] = s0;
            P[2 * i + 1][e] = s1;
            xa[e] = fma2(k23, s1, fma2(k01, s0, xa[e]));
            if (OUT) ya[e] = fma2(q23, s1, fma2(q01, s0, ya[e]));
        }
    }
    float x[4], y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 xs = up2(xa[e]);
        x[e] = xs.x + xs.y;
        if (OUT) {
            const float2 ys = up2(ya[e]);
            y[e] = ys.x + ys.y;
        }
    }
    constexpr unsigned FULL = 0xffffffffu;
    float xr[4], own = 0.f;
    if (OUT) {
        // sums v = (x0..x3, y0..y3): keep v[4 b0 ..], then [2 b1 ..] of those, then [b2]
        float u1[4], u2[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = b0 ? x[i] : y[i], keep = b0 ? y[i] : x[i];
            u1[i] = keep + __shfl_xor_sync(FULL, send, 4);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = b1 ? u1[i] : u1[2 + i], keep = b1 ? u1[2 + i] : u1[i];
            u2[i] = keep + __shfl_xor_sync(FULL, send, 8);
        }
        {
            const float send = b2 ? u2[0] : u2[1], keep = b2 ? u2[1] : u2[0];
            own = keep + __shfl_xor_sync(FULL, send, 16);   // (b0 ? y : x)[2 b1 + b2]
        }
        // x_e sits in the lane of the group with rg = 2 (e >> 1) + 4 (e & 1)
#pragma unroll
        for (int e = 0; e < 4; ++e) xr[e] = __shfl_sync(FULL, own, 4 * (2 * (e >> 1) + 4 * (e & 1)) + cg);
    } else {
        // sums v = (x0..x3): keep v[2 b0 ..], then [b1], then the full sum over b2
        float u1[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = b0 ? x[i] : x[2 + i], keep = b0 ? x[2 + i] : x[i];
            u1[i] = keep + __shfl_xor_sync(FULL, send, 4);
        }
        const float send = b1 ? u1[0] : u1[1], keep = b1 ? u1[1] : u1[0];
        const float u2 = keep + __shfl_xor_sync(FULL, send, 8);
        own = u2 + __shfl_xor_sync(FULL, u2, 16);             // x[2 b0 + b1]
        // x_e sits in the lanes with rg = (e >> 1) + 2 (e & 1) (and + 4)
#pragma unroll
        for (int e = 0; e < 4; ++e) xr[e] = __shfl_sync(FULL, own, 4 * ((e >> 1) + 2 * (e & 1)) + cg);
    }
    const float4 vv = *reinterpret_cast<const float4 *>(tv.v + 16 * warp + 4 * cg);
    const float w0 = tv.beta * (vv.x - xr[0]), w1 = tv.beta * (vv.y - xr[1]);
    const float w2 = tv.beta * (vv.z - xr[2]), w3 = tv.beta * (vv.w - xr[3]);
    const f2 ww[4] = {pk2(w0, w0), pk2(w1, w1), pk2(w2, w2), pk2(w3, w3)};
#pragma unroll
    for (int i = 0; i < L::R / 4; ++i) {
        const float4 k4 = *reinterpret_cast<const float4 *>(kp + 4 * i);
        const f2 k01 = pk2(k4.x, k4.y), k23 = pk2(k4.z, k4.w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            P[2 * i][e] = fma2(k01, ww[e], P[2 * i][e]);
            P[2 * i + 1][e] = fma2(k23, ww[e], P[2 * i + 1][e]);
        }
    }
    oe = 2 * b1 + b2;
    float o = 0.f;
    if (OUT && b0) {
        const float w = oe == 0 ? w0 : oe == 1 ? w1 : oe == 2 ? w2 : w3;
        o = scale * fmaf(tv.kq, w, own);
    }
    return o;
}

// the lanes that hold an output after kda_step<D, true>: odd rg
__device__ __forceinline__ bool out_lane() { return ((threadIdx.x >> 2) & 1) != 0; }

// ---------------------------------------------------------------- decode
// One token per (sequence, head): one CTA each, the state read and written once.
template <int D, typename TIO, bool CONV>
__global__ void __launch_bounds__(DecodeShape<D>::NT, 2)
decode_kernel(const __grid_constant__ DecodeParams p) {
    __shared__ TokVec<D> tv;
    const int s = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int32_t slot = p.slots[s];
    if (slot < 0 || slot >= p.n_slots) {
        if (threadIdx.x == 0) record_status(KDA_ERR_RANGE);
        return;
    }
    const int t = threadIdx.x;
    float *S = p.pool + ((int64_t)slot * p.H + h) * (int64_t)D * D;
    StatePairs<D> P;
    load_state<D>(P, S);
    const int64_t row = (int64_t)s * p.H + h;
    if (t < D) {
        ConvWin w;
        if (CONV) conv_begin(w, p, p.conv, slot, h, D, t);
        const float xq = IO<TIO>::ld(static_cast<const TIO *>(p.q) + row * D + t);
        const float xk = IO<TIO>::ld(static_cast<const TIO *>(p.k) + row * D + t);
        put_qk<D, CONV>(tv, t, xq, xk, true, w, p.taps);
        if (CONV) conv_store(w, p, p.conv, slot, h, D, t);
    } else {
        const int c = t - D;
        put_vg<D>(tv, c, IO<TIO>::ld(static_cast<const TIO *>(p.v) + row * D + c), p.g[row * D + c]);
        if (c == 0) tv.beta = p.beta[row];
    }
    __syncthreads();
    if (t < 32) token_finish<D>(tv, CONV, true);
    __syncthreads();
    int oe;
    const float o = kda_step<D>(P, tv, p.scale, oe);
    store_state<D>(P, S);
    if (out_lane()) IO<TIO>::st(static_cast<TIO *>(p.o) + row * D + lane_col() + oe, o);
}

// ---------------------------------------------------------------- verify, verify + commit
// The previous step's commit, for verify + commit: the live state is read once, the
// previous step's first n_accept tokens are replayed into it (state only), it is written
// back once, and this step's draft tokens run from it with outputs only.
struct CommitParams {
    const void *q;              // the previous step's raw q (front-end on: advances the q window)
    float *conv_snapshots;      // front-end on: conv state at the boundary [rows, 2, H, D, taps-1]
    const void *k, *v;          // the previous step's tokens (packed like verify's)
    const float *g, *beta;
    const int32_t *n_accept;    // [n_seq] leading tokens of the previous batch to commit
    const int64_t *pos;         // [n_seq] tokens absorbed by the live state (snapshots only)
    const int64_t *snap_row;    // [n_seq] snapshot row for a boundary crossed, or < 0
    const uint8_t *commit_new;  // [n_seq] nonzero: this step's tokens are committed too (nullable)
    float *snapshots;
    int64_t n_snap_rows;
    int32_t snap_interval;
    int64_t tok_base;                     // absolute offset of tok0[0] in the previous batch
    int32_t tok0[kMaxSeqsPerLaunch + 1];  // previous batch offsets (relative)
};

// G CTAs over the (sequence, head) items, with the sequences in the host's order of
// decreasing token count: CTA b takes ranks b, b + G, b + 2 G, ... of that list, every
// second band of G ranks reversed (a snake), so that each CTA gets one item of every band
// and the CTAs' token totals come out nearly equal (the heads of one sequence share its
// token counts). verify + commit runs a persistent grid (two CTAs per SM); verify runs
// G = items, one CTA per item, longest first. The records of a CTA's items (slot,
// accepted count, snapshot) are read once at its start. Warp 0 is the producer: one bulk
// copy brings the next item's state (and conv window and weights) into shared memory
// while the current item runs from registers, and the item's token rows come in batches
// of TB by 3-D TMA tiles (channels x 1 head x TB rows) into two buffers, two batches ahead
// across item boundaries.
struct SpecParams {
    CUtensorMap mq, mk, mv, mg;       // this step's q, k, v, g rows: (D, H, rows), box (D, 1, TB)
    CUtensorMap pq, pk, pv, pg;       // the previous step's (replay; pq with the front-end only)
    DecodeParams p;                   // verify: token_states, conv_tok; pool read-only
    CommitParams c;                   // verify + commit only
    int32_t n_items;
    int32_t order[kMaxSeqsPerLaunch];   // sequences by decreasing token count
};

template <typename TIO> struct SpecShape {
    static constexpr int TB = sizeof(TIO) == 2 ? 8 : 4;   // tokens per batch
};
// item records per CTA (the host launches enough CTAs)
template <bool CONV> struct SpecItems {
    static constexpr int N = CONV ? 96 : 128;
};

struct ItemMeta {
    int32_t s, slot;      // slot < 0: the item is out of range
    int32_t na;           // accepted tokens to replay; bit 30: commit_new
    int32_t jsnap;        // the committed-token index after which the snapshot falls, or -1
    int64_t srow;         // snapshot row, or -1
};
constexpr int32_t kCnewBit = 1 << 30;

template <int D, typename TIO, bool CONV> struct SpecSmem {
    static constexpr int TB = SpecShape<TIO>::TB;
    static constexpr uint32_t ROW = D * sizeof(TIO);
    static constexpr uint32_t ST = 0;                                  // state [D][D] fp32
    static constexpr uint32_t CW = ST + D * D * 4;                     // conv: q, k windows, q, k weights
    static constexpr uint32_t CW_K = D * (kMaxTaps - 1) * 4, CW_WQ = 2 * CW_K, CW_WK = CW_WQ + D * kMaxTaps * 4;
    static constexpr uint32_t RAW0 = CW + (CONV ? CW_WK + D * kMaxTaps * 4 : 0);   // raw batches: q, k, v, g
    static constexpr uint32_t RAW = TB * (3 * ROW + D * 4);
    static constexpr uint32_t BETA = RAW0 + 2 * RAW;                   // beta of the raw batches [2][TB]
    static constexpr uint32_t TV = BETA + 128;                         // token vectors [TB]
    static constexpr uint32_t META = TV + TB * sizeof(TokVec<D>);      // ItemMeta [SpecItems::N]
    static constexpr uint32_t BARS = META + SpecItems<CONV>::N * sizeof(ItemMeta);   // state, raw 0, raw 1
    static constexpr uint32_t PROD = BARS + 32;                        // producer cursors
    static constexpr uint32_t BYTES = PROD + 32 + 128;                 // + alignment slack
    static_assert(RAW0 % 128 == 0 && RAW % 128 == 0 && (TB * ROW) % 128 == 0 && TV % 16 == 0, "alignment");
    static_assert(D != 128 || sizeof(TIO) != 2 || 2 * (BYTES + 1024) <= 233472, "two CTAs per SM");
};

struct ItemInfo {
    int s, h, na, n_tok, nb0, nbat;
    bool valid, cnew;
    int32_t slot;
    int64_t srow, jsnap, prev_first, tok_first;
};

// rank of the CTA's k-th item in the sorted item list (the snake over bands of G)
__device__ __forceinline__ int item_rank(int k, int n_items) {
    const int G = gridDim.x, base = k * G, pos = blockIdx.x;
    const int width = min(G, n_items - base);
    return base + ((k & 1) ? width - 1 - pos : pos);
}

// the CTA's k-th item
template <int D, typename TIO, bool COMMIT>
__device__ __forceinline__ ItemInfo item_info(const SpecParams &P, const ItemMeta *meta, int k) {
    constexpr int TB = SpecShape<TIO>::TB;
    ItemInfo I;
    const ItemMeta m = meta[k];
    I.s = m.s;
    I.h = item_rank(k, P.n_items) % P.p.H;
    I.slot = m.slot;
    I.valid = m.slot >= 0;
    I.n_tok = P.p.tok0[I.s + 1] - P.p.tok0[I.s];
    I.na = COMMIT ? (m.na & ~kCnewBit) : 0;
    I.cnew = COMMIT && (m.na & kCnewBit) != 0;
    I.srow = m.srow;
    I.jsnap = m.jsnap;
    I.nb0 = (I.na + TB - 1) / TB;
    I.nbat = I.nb0 + (I.n_tok + TB - 1) / TB;
    I.prev_first = COMMIT ? P.c.tok_base + P.c.tok0[I.s] : 0;
    I.tok_first = P.p.tok_base + P.p.tok0[I.s];
    return I;
}

struct ProdCursor {
    int kb, bb, nb_issued;     // batch cursor: local item, batch within it; batches issued
    int ks, ns_issued;         // state cursor: next local item to consider; states issued
};

// warp 0: issue the next batch of token rows (lane 0 the tiles, lanes c < nb a copy of
// their token's beta; all complete on the buffer's mbarrier)
template <int D, typename TIO, bool CONV, bool COMMIT>
__device__ __forceinline__ void produce_batch(const SpecParams &P, uint8_t *sm, const ItemMeta *meta,
                                              int n_local) {
    using SM = SpecSmem<D, TIO, CONV>;
    constexpr int TB = SM::TB;
    ProdCursor *cur = reinterpret_cast<ProdCursor *>(sm + SM::PROD);
    const int lane = threadIdx.x & 31;
    int kb = cur->kb, bb = cur->bb;
    ItemInfo I;
    for (;; ++kb, bb = 0) {
        if (kb >= n_local) return;
        I = item_info<D, TIO, COMMIT>(P, meta, kb);
        if (I.valid && bb < I.nbat) break;
    }
    const bool replay = bb < I.nb0;
    const int j0 = (replay ? bb : bb - I.nb0) * TB;
    const int nb = min(TB, (replay ? I.na : I.n_tok) - j0);
    const int64_t row0 = (replay ? I.prev_first : I.tok_first) + j0;
    const int slot = cur->nb_issued & 1;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + SM::BARS) + 1 + slot;
    if (lane < nb) {
        // before the tiles' arrival below, so that the phase cannot complete without them
        const float *beta = replay ? P.c.beta : P.p.beta;
        tc::cp_async4(reinterpret_cast<float *>(sm + SM::BETA) + slot * TB + lane, beta + (row0 + lane) * P.p.H + I.h);
        tc::cp_async_arrive(bar);
    }
    __syncwarp();
    if (lane == 0) {
        uint8_t *raw = sm + SM::RAW0 + slot * SM::RAW;
        const bool with_q = !replay || CONV;
        tc::bar_expect_tx(bar, (uint32_t)TB * ((with_q ? 3u : 2u) * SM::ROW + D * 4u));
        const int z = (int)row0;
        if (with_q) tc::tma_load3(raw, replay ? &P.pq : &P.mq, 0, I.h, z, bar);
        tc::tma_load3(raw + TB * SM::ROW, replay ? &P.pk : &P.mk, 0, I.h, z, bar);
        tc::tma_load3(raw + 2 * TB * SM::ROW, replay ? &P.pv : &P.mv, 0, I.h, z, bar);
        tc::tma_load3(raw + 3 * TB * SM::ROW, replay ? &P.pg : &P.mg, 0, I.h, z, bar);
        cur->kb = kb;
        cur->bb = bb + 1;
        cur->nb_issued += 1;
    }
    __syncwarp();
}

// thread 0: issue the state (and conv window and weights) of the next item that needs it
template <int D, typename TIO, bool CONV, bool COMMIT>
__device__ __forceinline__ void produce_state(const SpecParams &P, uint8_t *sm, const ItemMeta *meta,
                                              int n_local) {
    using SM = SpecSmem<D, TIO, CONV>;
    ProdCursor *cur = reinterpret_cast<ProdCursor *>(sm + SM::PROD);
    for (int ks = cur->ks; ks < n_local; ++ks) {
        const ItemInfo I = item_info<D, TIO, COMMIT>(P, meta, ks);
        if (!I.valid || I.nbat == 0) continue;
        const DecodeParams &p = P.p;
        uint64_t *bar = reinterpret_cast<uint64_t *>(sm + SM::BARS);
        const int K = p.taps;
        const uint32_t wb = CONV ? (uint32_t)(D * (K - 1) * 4) : 0u, cb = CONV ? (uint32_t)(D * K * 4) : 0u;
        tc::bar_expect_tx(bar, (uint32_t)(D * D * 4) + 2 * wb + 2 * cb);
        tc::bulk_load(sm + SM::ST, p.pool + ((int64_t)I.slot * p.H + I.h) * (int64_t)D * D, D * D * 4, bar);
        if (CONV) {
            tc::bulk_load(sm + SM::CW, p.conv + conv_index(2 * (int64_t)I.slot, p.H, I.h, D, 0, K), wb, bar);
            tc::bulk_load(sm + SM::CW + SM::CW_K, p.conv + conv_index(2 * (int64_t)I.slot + 1, p.H, I.h, D, 0, K),
                          wb, bar);
            tc::bulk_load(sm + SM::CW + SM::CW_WQ, p.wq + (int64_t)I.h * D * K, cb, bar);
            tc::bulk_load(sm + SM::CW + SM::CW_WK, p.wk + (int64_t)I.h * D * K, cb, bar);
        }
        cur->ks = ks + 1;
        cur->ns_issued += 1;
        return;
    }
    cur->ks = n_local;
}

// Raw rows of a batch -> token vectors: threads t < D channel t of q and k (the
// front-end's conv window in token order with CONV), threads t >= D channel t - D of v
// and g, threads t < nb token t's beta.
template <int D, typename TIO, bool CONV>
__device__ __forceinline__ void convert_batch(TokVec<D> *tv, const uint8_t *raw, const float *beta, int nb,
                                              bool read_q, bool with_q, ConvWin &w, const DecodeParams &p, int h,
                                              const ConvOut &co) {
    constexpr int TB = SpecShape<TIO>::TB;
    constexpr uint32_t ROW = D * sizeof(TIO);
    const int t = threadIdx.x;
    if (t < D) {
        const TIO *rq = reinterpret_cast<const TIO *>(raw), *rk = reinterpret_cast<const TIO *>(raw + TB * ROW);
        for (int j = 0; j < nb; ++j) {
            const float xq = read_q ? IO<TIO>::ld(rq + j * D + t) : 0.f;
            const float xk = IO<TIO>::ld(rk + j * D + t);
            put_qk<D, CONV>(tv[j], t, xq, xk, with_q, w, p.taps);
            if (CONV) {
                if (co.tok) conv_store(w, p, co.tok, co.tok0 + j, h, D, t);
                if (j == co.snap_j) conv_store(w, p, co.snap, co.snap_row, h, D, t);
            }
        }
        if (t < nb) tv[t].beta = beta[t];
    } else {
        const int c = t - D;
        const TIO *rv = reinterpret_cast<const TIO *>(raw + 2 * TB * ROW);
        const float *rgt = reinterpret_cast<const float *>(raw + 3 * TB * ROW);
        for (int j = 0; j < nb; ++j) put_vg<D>(tv[j], c, IO<TIO>::ld(rv + j * D + c), rgt[j * D + c]);
    }
}

// COMMIT = false: verify. Every token gives its output and its state (token_states row),
// and with the front-end its conv state (conv_tok row); the pool is only read.
// COMMIT = true: verify + commit. The stream of an item is the replayed prefix (state
// only; the state is written back to the pool after it, or after this step's tokens with
// commit_new), then this step's tokens (outputs); a snapshot at a crossed boundary.
template <int D, typename TIO, bool CONV, bool COMMIT>
__global__ void __launch_bounds__(DecodeShape<D>::NT, 2)
spec_kernel(const __grid_constant__ SpecParams P) {
    using SM = SpecSmem<D, TIO, CONV>;
    using Sh = DecodeShape<D>;
    constexpr int TB = SM::TB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const DecodeParams &p = P.p;
    const CommitParams &c = P.c;
    TokVec<D> *tv = reinterpret_cast<TokVec<D> *>(sm + SM::TV);
    ItemMeta *meta = reinterpret_cast<ItemMeta *>(sm + SM::META);
    uint64_t *bar_s = reinterpret_cast<uint64_t *>(sm + SM::BARS), *bar_t = bar_s + 1;
    ProdCursor *cur = reinterpret_cast<ProdCursor *>(sm + SM::PROD);
    const int t = threadIdx.x, warp = t >> 5;

    const int n_local = (int)blockIdx.x < P.n_items ? (P.n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    if (n_local == 0) return;
    if (n_local > SpecItems<CONV>::N) {         // the host never launches this
        if (t == 0) record_status(KDA_ERR_INVALID);
        return;
    }
    // the records of this CTA's items, read in parallel once
    for (int k = t; k < n_local; k += Sh::NT) {
        const int r = item_rank(k, P.n_items);
        const int s = P.order[r / p.H];
        ItemMeta m;
        m.s = s;
        m.slot = p.slots[s];
        m.na = 0;
        m.jsnap = -1;
        m.srow = -1;
        bool ok = m.slot >= 0 && m.slot < p.n_slots;
        if (COMMIT) {
            const int32_t na = c.n_accept[s];
            const int n_tok = p.tok0[s + 1] - p.tok0[s];
            const bool cnew = c.commit_new != nullptr && c.commit_new[s] != 0 && n_tok > 0;
            if (c.snap_interval > 0 && c.snap_row != nullptr && c.snap_row[s] >= 0) {
                m.srow = c.snap_row[s];
                const int64_t p0 = c.pos[s];
                m.jsnap = (int32_t)((p0 / c.snap_interval + 1) * c.snap_interval - p0 - 1);
            }
            ok = ok && na >= 0 && na <= c.tok0[s + 1] - c.tok0[s] && na < kCnewBit && m.srow < c.n_snap_rows;
            m.na = na | (cnew ? kCnewBit : 0);
        }
        if (!ok) m.slot = -1;
        meta[k] = m;
    }
    if (t == 0) {
        tc::bar_init(bar_s, 1);
        tc::bar_init(&bar_t[0], 1);
        tc::bar_init(&bar_t[1], 1);
        tc::bar_init_fence();
        // the token-row descriptors, ahead of the first copies that use them
        tc::tma_prefetch_desc(&P.mk);
        tc::tma_prefetch_desc(&P.mv);
        tc::tma_prefetch_desc(&P.mg);
        if (p.q) tc::tma_prefetch_desc(&P.mq);
        if (COMMIT && c.k) {
            tc::tma_prefetch_desc(&P.pk);
            tc::tma_prefetch_desc(&P.pv);
            tc::tma_prefetch_desc(&P.pg);
            if (CONV && c.q) tc::tma_prefetch_desc(&P.pq);
        }
        cur->kb = 0; cur->bb = 0; cur->nb_issued = 0; cur->ks = 0; cur->ns_issued = 0;
    }
    __syncthreads();
    if (t == 0) produce_state<D, TIO, CONV, COMMIT>(P, sm, meta, n_local);
    if (warp == 0) {
        produce_batch<D, TIO, CONV, COMMIT>(P, sm, meta, n_local);
        produce_batch<D, TIO, CONV, COMMIT>(P, sm, meta, n_local);
    }

    bool ok = true;
    int g = 0, vs = 0;          // batches and states consumed
    for (int kl = 0; kl < n_local && ok; ++kl) {
        int nbat;
        {
            const ItemInfo I = item_info<D, TIO, COMMIT>(P, meta, kl);
            if (!I.valid) {
                if (t == 0) record_status(KDA_ERR_RANGE);
                continue;
            }
            nbat = I.nbat;
        }
        if (nbat == 0) continue;
        const bool sok = tc::bar_wait(bar_s, (uint32_t)(vs & 1));
        vs += sok;
        ok = ok && sok;
        StatePairs<D> Pr;
        load_state_smem<D>(Pr, reinterpret_cast<const float *>(sm + SM::ST));
        ConvWin w;
        if (CONV && t < D) {
            const float *cw = reinterpret_cast<const float *>(sm + SM::CW);
            const int K = p.taps;
            win_load(w.q, cw + SM::CW_WQ / 4 + t * K, cw + t * (K - 1), K);
            win_load(w.k, cw + SM::CW_WK / 4 + t * K, cw + SM::CW_K / 4 + t * (K - 1), K);
        }
        __syncthreads();        // the state buffer is free
        if (t == 0 && ok) produce_state<D, TIO, CONV, COMMIT>(P, sm, meta, n_local);
        for (int bi = 0; bi < nbat; ++bi) {
            // the item's fields are re-read from shared memory after every barrier rather
            // than held in registers through the steps
            const ItemInfo I = item_info<D, TIO, COMMIT>(P, meta, kl);
            const bool replay = bi < I.nb0;
            const int j0 = (replay ? bi : bi - I.nb0) * TB;
            const int nb = min(TB, (replay ? I.na : I.n_tok) - j0);
            // the committed-token index of this batch's first token, and a snapshot in it
            const int64_t c0 = !COMMIT ? -1 : replay ? j0 : (I.cnew ? I.na + j0 : -1);
            const int js = (c0 >= 0 && I.jsnap >= c0 && I.jsnap < c0 + nb) ? (int)(I.jsnap - c0) : -1;
            const ConvOut co = COMMIT ? ConvOut{nullptr, 0, c.conv_snapshots, I.srow, js}
                                      : ConvOut{p.conv_tok, I.tok_first + j0, nullptr, 0, -1};
            const bool bok = tc::bar_wait(&bar_t[g & 1], (uint32_t)((g >> 1) & 1));
            convert_batch<D, TIO, CONV>(tv, sm + SM::RAW0 + (g & 1) * SM::RAW,
                                        reinterpret_cast<const float *>(sm + SM::BETA) + (g & 1) * TB, nb,
                                        CONV || !replay, !replay, w, p, I.h, co);
            ok = __syncthreads_and(ok && bok);   // vectors staged, raw buffer read
            if (!ok) break;
            ++g;
            if (warp == 0) produce_batch<D, TIO, CONV, COMMIT>(P, sm, meta, n_local);
            for (int j = warp; j < nb; j += Sh::NW) token_finish<D>(tv[j], CONV, !replay);
            __syncthreads();
            const int64_t hh = I.h;
            if (replay) {
                const bool store_after = bi == I.nb0 - 1 && !I.cnew;
                float *snap = js >= 0 ? c.snapshots + (I.srow * p.H + hh) * (int64_t)D * D : nullptr;
                for (int j = 0; j < nb; ++j) {
                    int oe;
                    kda_step<D, false>(Pr, tv[j], 0.f, oe);
                    if (j == js) store_state<D>(Pr, snap);
                }
                if (store_after) {
                    store_state<D>(Pr, p.pool + ((int64_t)I.slot * p.H + hh) * (int64_t)D * D);
                    if (CONV && t < D) conv_store(w, p, p.conv, I.slot, I.h, D, t);
                }
            } else {
                float *snap = js >= 0 ? c.snapshots + (I.srow * p.H + hh) * (int64_t)D * D : nullptr;
                const int64_t row0 = (I.tok_first + j0) * p.H + hh;
                for (int j = 0; j < nb; ++j) {
                    int oe;
                    const float o = kda_step<D>(Pr, tv[j], p.scale, oe);
                    const int64_t row = row0 + (int64_t)j * p.H;
                    if (out_lane()) IO<TIO>::st(static_cast<TIO *>(p.o) + row * D + lane_col() + oe, o);
                    if (!COMMIT) store_state<D>(Pr, p.token_states + row * (int64_t)D * D);
                    if (COMMIT && j == js) store_state<D>(Pr, snap);
                }
            }
            __syncthreads();                  // the vectors are free for the next batch
        }
        if (ok) {
            const ItemInfo I = item_info<D, TIO, COMMIT>(P, meta, kl);
            if (I.cnew) {
                store_state<D>(Pr, p.pool + ((int64_t)I.slot * p.H + I.h) * (int64_t)D * D);
                if (CONV && t < D) conv_store(w, p, p.conv, I.slot, I.h, D, t);
            }
        }
    }
    if (t == 0) {
        // copies still in flight land before the shared memory is released
        for (; vs < cur->ns_issued; ++vs) tc::bar_wait(bar_s, (uint32_t)(vs & 1), 1u << 16);
        for (; g < cur->nb_issued; ++g) tc::bar_wait(&bar_t[g & 1], (uint32_t)((g >> 1) & 1), 1u << 16);
    }
}

}  // namespace kda
