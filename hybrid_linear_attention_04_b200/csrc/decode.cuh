// KDA decode and speculative-verify kernels (sm_100a, SIMT, HBM-bound).
//
// One CTA owns one (sequence, head) state S [D x D] fp32 (d_v contiguous) and
// streams it through registers once: 128-bit loads, gate, rank-1 delta
// correction and output read in one pass, 128-bit stores.
//
// Per token (Kimi K3 technical FAQ, "What is KDA": delta rule with a
// per-channel forget gate; standard gated-delta form):
//     S' = Diag(alpha) S                    alpha = exp(g), per key channel
//     x  = S'^T k,   y = S'^T q             (one pass, shared reduction over d_k)
//     w  = beta (v - x)
//     S  = S' + k w^T
//     o  = scale (y + (k . q) w)            (= scale * S^T q, read after update)
//
// Thread map: thread t owns column group cg = t % (D/4) (four adjacent d_v
// columns, one float4) and rows rs, rs + RS, ... with rs = t / (D/4). Column
// sums over d_k reduce first across lanes of a warp that share cg (shuffles),
// then across warps through shared memory in a fixed order (deterministic).
// Decode and verify run the same step function, so verify's state after its
// j-th token is bit-identical to j decode calls.
#pragma once
#include "common.cuh"

namespace kda {

constexpr int kMaxSeqsPerLaunch = KDA_SEQS_PER_LAUNCH;

template <int D> struct DecodeShape {
    static constexpr int NT = D == 128 ? 256 : (D == 64 ? 128 : 64);  // threads per CTA
    static constexpr int CG = D / 4;                                    // column groups
    static constexpr int RS = NT / CG;                                  // row slots
    static constexpr int R = D / RS;                                    // rows per thread
    static constexpr int NW = NT / 32;                                  // warps
    static_assert(CG <= 32 && 32 % CG == 0, "column groups must tile a warp");
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

struct ConvWin {
    float wq[kMaxTaps], wk[kMaxTaps];
    float hq[kMaxTaps - 1], hk[kMaxTaps - 1];
};

__device__ __forceinline__ int64_t conv_index(int64_t row2, int H, int h, int D, int c, int taps) {
    // row2 = 2 * (slot or token) + (0 for q, 1 for k)
    return ((row2 * H + h) * D + c) * (int64_t)(taps - 1);
}

// weights and window of channel c from conv state row `row` (slot or token) of `src`
__device__ __forceinline__ void conv_begin(ConvWin &w, const DecodeParams &p, const float *src, int64_t row,
                                           int h, int D, int c) {
    const int K = p.taps;
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) {
        w.wq[j] = j < K ? p.wq[((int64_t)h * D + c) * K + j] : 0.f;
        w.wk[j] = j < K ? p.wk[((int64_t)h * D + c) * K + j] : 0.f;
    }
    const float *sq = src + conv_index(2 * row, p.H, h, D, c, K);
    const float *sk = src + conv_index(2 * row + 1, p.H, h, D, c, K);
#pragma unroll
    for (int j = 0; j < kMaxTaps - 1; ++j) {
        w.hq[j] = j < K - 1 ? sq[j] : 0.f;
        w.hk[j] = j < K - 1 ? sk[j] : 0.f;
    }
}

__device__ __forceinline__ void conv_store(const ConvWin &w, const DecodeParams &p, float *dst, int64_t row,
                                           int h, int D, int c) {
    const int K = p.taps;
    float *dq = dst + conv_index(2 * row, p.H, h, D, c, K);
    float *dk = dst + conv_index(2 * row + 1, p.H, h, D, c, K);
#pragma unroll
    for (int j = 0; j < kMaxTaps - 1; ++j)
        if (j < K - 1) { dq[j] = w.hq[j]; dk[j] = w.hk[j]; }
}

// one causal conv step of raw input x through weights wt and window hs (shifted in place)
// (every index is a compile-time constant after unrolling, so window and weights stay
// in registers)
__device__ __forceinline__ float conv_step(const float (&wt)[kMaxTaps], float (&hs)[kMaxTaps - 1], int K, float x) {
    float wl = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j)
        if (j == K - 1) wl = wt[j];
    float y = wl * x;
#pragma unroll
    for (int j = 0; j < kMaxTaps - 1; ++j)
        if (j < K - 1) y = fmaf(wt[j], hs[j], y);
#pragma unroll
    for (int j = 0; j < kMaxTaps - 1; ++j) {
        if (j < K - 2) hs[j] = hs[j + 1];
        else if (j == K - 2) hs[j] = x;
    }
    return y;
}

__device__ __forceinline__ float swish(float y) { return y / (1.f + expf(-y)); }

// Per-token vectors staged in shared memory. 16-byte aligned (and padded to a
// multiple of 16 bytes) because the step reads v with float4 loads.
template <int D> struct __align__(16) TokVec {
    float k[D], q[D], a[D], v[D];
    float beta, kq;
};
static_assert(sizeof(TokVec<128>) % 16 == 0 && sizeof(TokVec<32>) % 16 == 0, "TokVec padding");

// Stage the vectors of token row `row` (= token * H + head); q may be null (a token
// whose output is not needed). D threads (or fewer, looping) fill the vectors.
template <int D, typename TIO>
__device__ __forceinline__ void load_vectors(TokVec<D> &tv, const void *q_, const void *k_, const void *v_,
                                             const float *g_, const float *beta, int64_t row) {
    const TIO *q = q_ ? static_cast<const TIO *>(q_) + row * D : nullptr;
    const TIO *k = static_cast<const TIO *>(k_) + row * D;
    const TIO *v = static_cast<const TIO *>(v_) + row * D;
    const float *g = g_ + row * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        tv.k[i] = IO<TIO>::ld(k + i);
        tv.q[i] = q ? IO<TIO>::ld(q + i) : 0.f;
        tv.v[i] = IO<TIO>::ld(v + i);
        tv.a[i] = expf(g[i]);
    }
    if (threadIdx.x == 0) tv.beta = beta[row];
}

template <int D, typename TIO>
__device__ __forceinline__ void load_token(TokVec<D> &tv, const DecodeParams &p, int64_t row) {
    load_vectors<D, TIO>(tv, p.q, p.k, p.v, p.g, p.beta, row);
}

// Stage a token whose raw q, k pass through the front-end: the conv and Swish here
// (thread c < D, channel c, window w), the L2 normalisation in token_finish. With
// q_ == nullptr only the q window advances (a token whose output is not needed still
// moves the conv state).
template <int D, typename TIO>
__device__ __forceinline__ void load_vectors_conv(TokVec<D> &tv, ConvWin &w, int K, const void *q_, const void *k_,
                                                  const void *v_, const float *g_, const float *beta,
                                                  int64_t row, bool want_q) {
    const int c = threadIdx.x;
    if (c < D) {
        const float xq = IO<TIO>::ld(static_cast<const TIO *>(q_) + row * D + c);
        const float xk = IO<TIO>::ld(static_cast<const TIO *>(k_) + row * D + c);
        const float yq = conv_step(w.wq, w.hq, K, xq);
        const float yk = conv_step(w.wk, w.hk, K, xk);
        tv.q[c] = want_q ? swish(yq) : 0.f;
        tv.k[c] = swish(yk);
        tv.v[c] = IO<TIO>::ld(static_cast<const TIO *>(v_) + row * D + c);
        tv.a[c] = expf(g_[row * D + c]);
    }
    if (threadIdx.x == 0) tv.beta = beta[row];
}

// One warp finishes a staged token: L2-normalises k and q when the front-end is on,
// then k . q (fixed reduction order) when q is used.
template <int D>
__device__ __forceinline__ void token_finish(TokVec<D> &tv, bool normalise, bool with_q) {
    const int lane = threadIdx.x & 31;
    if (normalise) {
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int i = lane; i < D; i += 32) {
            sk = fmaf(tv.k[i], tv.k[i], sk);
            sq = fmaf(tv.q[i], tv.q[i], sq);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float rk = 1.f / fmaxf(sqrtf(sk), kNormEps), rq = 1.f / fmaxf(sqrtf(sq), kNormEps);
#pragma unroll
        for (int i = lane; i < D; i += 32) {
            tv.k[i] *= rk;
            tv.q[i] *= rq;
        }
        __syncwarp();
    }
    if (with_q) {
        float s = 0.f;
#pragma unroll
        for (int i = lane; i < D; i += 32) s = fmaf(tv.k[i], tv.q[i], s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) tv.kq = s;
    }
}

// k . q for a staged token, by one warp, fixed reduction order.
template <int D>
__device__ __forceinline__ void token_kq(TokVec<D> &tv) {
    token_finish<D>(tv, false, true);
}

// One recurrence step on the register-resident state. red: [NW][2][D] scratch
// in shared memory; the caller separates reuses of `red` by a barrier. With
// OUT = false the output read (y and o) is skipped; the state arithmetic is the
// same instruction for instruction, so both forms give bit-identical states.
template <int D, bool OUT = true>
__device__ __forceinline__ float4 kda_step(float4 (&st)[DecodeShape<D>::R], const TokVec<D> &tv,
                                           float *red, float scale) {
    using Sh = DecodeShape<D>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % Sh::CG, rs = t / Sh::CG;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) {
        const int r = rs + Sh::RS * m;
        const float a = tv.a[r], kr = tv.k[r];
        float4 s = st[m];
        s.x *= a; s.y *= a; s.z *= a; s.w *= a;
        st[m] = s;
        x.x = fmaf(kr, s.x, x.x); x.y = fmaf(kr, s.y, x.y);
        x.z = fmaf(kr, s.z, x.z); x.w = fmaf(kr, s.w, x.w);
        if (OUT) {
            const float qr = tv.q[r];
            y.x = fmaf(qr, s.x, y.x); y.y = fmaf(qr, s.y, y.y);
            y.z = fmaf(qr, s.z, y.z); y.w = fmaf(qr, s.w, y.w);
        }
    }
#pragma unroll
    for (int off = Sh::CG; off < 32; off <<= 1) {
        x.x += __shfl_xor_sync(0xffffffffu, x.x, off);
        x.y += __shfl_xor_sync(0xffffffffu, x.y, off);
        x.z += __shfl_xor_sync(0xffffffffu, x.z, off);
        x.w += __shfl_xor_sync(0xffffffffu, x.w, off);
        if (OUT) {
            y.x += __shfl_xor_sync(0xffffffffu, y.x, off);
            y.y += __shfl_xor_sync(0xffffffffu, y.y, off);
            y.z += __shfl_xor_sync(0xffffffffu, y.z, off);
            y.w += __shfl_xor_sync(0xffffffffu, y.w, off);
        }
    }
    if (lane < Sh::CG) {
        *reinterpret_cast<float4 *>(red + (warp * 2 + 0) * D + cg * 4) = x;
        if (OUT) *reinterpret_cast<float4 *>(red + (warp * 2 + 1) * D + cg * 4) = y;
    }
    __syncthreads();
    float4 X = make_float4(0.f, 0.f, 0.f, 0.f), Y = X;
#pragma unroll
    for (int w = 0; w < Sh::NW; ++w) {
        float4 a = *reinterpret_cast<const float4 *>(red + (w * 2 + 0) * D + cg * 4);
        X.x += a.x; X.y += a.y; X.z += a.z; X.w += a.w;
        if (OUT) {
            float4 b = *reinterpret_cast<const float4 *>(red + (w * 2 + 1) * D + cg * 4);
            Y.x += b.x; Y.y += b.y; Y.z += b.z; Y.w += b.w;
        }
    }
    const float4 vv = *reinterpret_cast<const float4 *>(tv.v + cg * 4);
    float4 wv;
    wv.x = tv.beta * (vv.x - X.x); wv.y = tv.beta * (vv.y - X.y);
    wv.z = tv.beta * (vv.z - X.z); wv.w = tv.beta * (vv.w - X.w);
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) {
        const float kr = tv.k[rs + Sh::RS * m];
        float4 s = st[m];
        s.x = fmaf(kr, wv.x, s.x); s.y = fmaf(kr, wv.y, s.y);
        s.z = fmaf(kr, wv.z, s.z); s.w = fmaf(kr, wv.w, s.w);
        st[m] = s;
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (OUT) {
        o.x = scale * fmaf(tv.kq, wv.x, Y.x); o.y = scale * fmaf(tv.kq, wv.y, Y.y);
        o.z = scale * fmaf(tv.kq, wv.z, Y.z); o.w = scale * fmaf(tv.kq, wv.w, Y.w);
    }
    return o;
}

template <int D, typename TIO>
__global__ void __launch_bounds__(DecodeShape<D>::NT)
decode_kernel(const __grid_constant__ DecodeParams p) {
    using Sh = DecodeShape<D>;
    __shared__ TokVec<D> tv;
    __shared__ __align__(16) float red[Sh::NW * 2 * D];
    const int s = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int32_t slot = p.slots[s];
    if (slot < 0 || slot >= p.n_slots) {
        if (threadIdx.x == 0) record_status(KDA_ERR_RANGE);
        return;
    }
    const int t = threadIdx.x, cg = t % Sh::CG, rs = t / Sh::CG;
    float *S = p.pool + ((int64_t)slot * p.H + h) * (int64_t)D * D;
    float4 st[Sh::R];
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) {
        const float *src = S + (int64_t)(rs + Sh::RS * m) * D + cg * 4;
        asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(st[m].x), "=f"(st[m].y), "=f"(st[m].z), "=f"(st[m].w)
                     : "l"(src));
    }
    const int64_t row = (int64_t)s * p.H + h;
    if (p.taps) {
        ConvWin w;
        if (t < D) conv_begin(w, p, p.conv, slot, h, D, t);
        load_vectors_conv<D, TIO>(tv, w, p.taps, p.q, p.k, p.v, p.g, p.beta, row, true);
        if (t < D) conv_store(w, p, p.conv, slot, h, D, t);
    } else {
        load_token<D, TIO>(tv, p, row);
    }
    __syncthreads();
    if (t < 32) token_finish<D>(tv, p.taps > 0, true);
    __syncthreads();
    const float4 o = kda_step<D>(st, tv, red, p.scale);
#pragma unroll
    for (int m = 0; m < Sh::R; ++m)
        st_stream(S + (int64_t)(rs + Sh::RS * m) * D + cg * 4, st[m]);
    if (rs == 0) IO<TIO>::st4(static_cast<TIO *>(p.o) + row * D + cg * 4, o);
}

// Verify: tokens are processed in batches of kTokBatch staged in shared memory.
constexpr int kTokBatch = 8;

// two CTAs per SM (register cap) keep enough state loads and stores in flight
template <int D, typename TIO>
__global__ void __launch_bounds__(DecodeShape<D>::NT, 2)
verify_kernel(const __grid_constant__ DecodeParams p) {
    using Sh = DecodeShape<D>;
    __shared__ TokVec<D> tv[kTokBatch];
    __shared__ __align__(16) float red[2][Sh::NW * 2 * D];
    const int s = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int32_t slot = p.slots[s];
    if (slot < 0 || slot >= p.n_slots) {
        if (threadIdx.x == 0) record_status(KDA_ERR_RANGE);
        return;
    }
    const int n_tok = p.tok0[s + 1] - p.tok0[s];
    const int64_t tok_first = p.tok_base + p.tok0[s];
    const int t = threadIdx.x, cg = t % Sh::CG, rs = t / Sh::CG, warp = t >> 5;
    const float *S = p.pool + ((int64_t)slot * p.H + h) * (int64_t)D * D;
    float4 st[Sh::R];
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) st[m] = ld_stream(S + (int64_t)(rs + Sh::RS * m) * D + cg * 4);
    ConvWin w;
    if (p.taps && t < D) conv_begin(w, p, p.conv, slot, h, D, t);
    int parity = 0;
    for (int j0 = 0; j0 < n_tok; j0 += kTokBatch) {
        const int nb = min(kTokBatch, n_tok - j0);
        __syncthreads();  // previous batch's vectors are no longer read
        for (int j = 0; j < nb; ++j) {
            const int64_t tok = tok_first + j0 + j;
            if (p.taps) {
                load_vectors_conv<D, TIO>(tv[j], w, p.taps, p.q, p.k, p.v, p.g, p.beta, tok * p.H + h, true);
                if (p.conv_tok && t < D) conv_store(w, p, p.conv_tok, tok, h, D, t);
            } else {
                load_token<D, TIO>(tv[j], p, tok * p.H + h);
            }
        }
        __syncthreads();
        if (warp < nb) token_finish<D>(tv[warp], p.taps > 0, true);
        for (int j = Sh::NW; j < nb; ++j)
            if (warp == 0) token_finish<D>(tv[j], p.taps > 0, true);
        __syncthreads();
        for (int j = 0; j < nb; ++j) {
            const float4 o = kda_step<D>(st, tv[j], red[parity], p.scale);
            parity ^= 1;
            const int64_t row = (tok_first + j0 + j) * p.H + h;
            float *dst = p.token_states + row * (int64_t)D * D;
#pragma unroll
            for (int m = 0; m < Sh::R; ++m)
                st_stream(dst + (int64_t)(rs + Sh::RS * m) * D + cg * 4, st[m]);
            if (rs == 0) IO<TIO>::st4(static_cast<TIO *>(p.o) + row * D + cg * 4, o);
        }
    }
}

}  // namespace kda

namespace kda {

// ---------------------------------------------------------------- verify + commit
// One speculative step with the previous step's commit fused in: the live state is
// read once, the previous step's first n_accept tokens are replayed into it (state
// only), it is written back once, and this step's draft tokens run from it with
// outputs only. No per-token state is written.
struct CommitParams {
    const void *q;              // the previous step's raw q (front-end on: advances the q window)
    float *conv_snapshots;      // front-end on: conv state at the boundary [rows, 2, H, D, taps-1]
    const void *k, *v;          // the previous step's tokens (packed like verify's)
    const float *g, *beta;
    const int32_t *n_accept;    // [n_seq] leading tokens of the previous batch to commit
    const int64_t *pos;         // [n_seq] tokens absorbed by the live state (snapshots only)
    const int64_t *snap_row;    // [n_seq] snapshot row for a boundary crossed, or < 0
    float *snapshots;
    int64_t n_snap_rows;
    int32_t snap_interval;
    int64_t tok_base;                     // absolute offset of tok0[0] in the previous batch
    int32_t tok0[kMaxSeqsPerLaunch + 1];  // previous batch offsets (relative)
};

struct VerifyCommitParams {
    DecodeParams p;   // this step: q, k, v, g, beta, o, tok0/tok_base, slots, pool (in/out)
    CommitParams c;
};

template <int D, typename TIO>
__global__ void __launch_bounds__(DecodeShape<D>::NT, 2)
verify_commit_kernel(const __grid_constant__ VerifyCommitParams P) {
    using Sh = DecodeShape<D>;
    const DecodeParams &p = P.p;
    const CommitParams &c = P.c;
    __shared__ TokVec<D> tv[kTokBatch];
    __shared__ __align__(16) float red[2][Sh::NW * 2 * D];
    const int s = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int32_t slot = p.slots[s];
    const int m_prev = c.tok0[s + 1] - c.tok0[s];
    const int32_t na = c.n_accept[s];
    int64_t srow = -1, jsnap = -1;          // snapshot row, and the replayed token after which it falls
    if (c.snap_interval > 0 && c.snap_row != nullptr && c.snap_row[s] >= 0) {
        srow = c.snap_row[s];
        const int64_t p0 = c.pos[s];
        jsnap = (p0 / c.snap_interval + 1) * c.snap_interval - p0 - 1;
    }
    if (slot < 0 || slot >= p.n_slots || na < 0 || na > m_prev || srow >= c.n_snap_rows) {
        if (threadIdx.x == 0) record_status(KDA_ERR_RANGE);
        return;
    }
    const int t = threadIdx.x, cg = t % Sh::CG, rs = t / Sh::CG, warp = t >> 5;
    float *S = p.pool + ((int64_t)slot * p.H + h) * (int64_t)D * D;
    float4 st[Sh::R];
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) {
        const float *src = S + (int64_t)(rs + Sh::RS * m) * D + cg * 4;
        asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(st[m].x), "=f"(st[m].y), "=f"(st[m].z), "=f"(st[m].w)
                     : "l"(src));
    }
    int parity = 0;
    ConvWin w;
    if (p.taps && t < D) conv_begin(w, p, p.conv, slot, h, D, t);
    // 1. commit: replay the accepted prefix of the previous batch (state only)
    const int64_t prev_first = c.tok_base + c.tok0[s];
    for (int j0 = 0; j0 < na; j0 += kTokBatch) {
        const int nb = min(kTokBatch, na - j0);
        __syncthreads();
        for (int j = 0; j < nb; ++j) {
            const int64_t row = (prev_first + j0 + j) * p.H + h;
            if (p.taps) {
                load_vectors_conv<D, TIO>(tv[j], w, p.taps, c.q, c.k, c.v, c.g, c.beta, row, false);
                if (j0 + j == jsnap && t < D) conv_store(w, p, c.conv_snapshots, srow, h, D, t);
            } else {
                load_vectors<D, TIO>(tv[j], nullptr, c.k, c.v, c.g, c.beta, row);
            }
        }
        __syncthreads();
        if (p.taps) {
            if (warp < nb) token_finish<D>(tv[warp], true, false);
            for (int j = Sh::NW; j < nb; ++j)
                if (warp == 0) token_finish<D>(tv[j], true, false);
            __syncthreads();
        }
        for (int j = 0; j < nb; ++j) {
            kda_step<D, false>(st, tv[j], red[parity], 0.f);
            parity ^= 1;
            if (j0 + j == jsnap) {
                float *dst = c.snapshots + (srow * p.H + h) * (int64_t)D * D;
#pragma unroll
                for (int m = 0; m < Sh::R; ++m) st_stream(dst + (int64_t)(rs + Sh::RS * m) * D + cg * 4, st[m]);
            }
        }
    }
    if (na > 0) {
#pragma unroll
        for (int m = 0; m < Sh::R; ++m) st_stream(S + (int64_t)(rs + Sh::RS * m) * D + cg * 4, st[m]);
        if (p.taps && t < D) conv_store(w, p, p.conv, slot, h, D, t);
    }
    // 2. verify this step's tokens from the committed state: outputs only
    const int n_tok = p.tok0[s + 1] - p.tok0[s];
    const int64_t tok_first = p.tok_base + p.tok0[s];
    for (int j0 = 0; j0 < n_tok; j0 += kTokBatch) {
        const int nb = min(kTokBatch, n_tok - j0);
        __syncthreads();
        for (int j = 0; j < nb; ++j) {
            const int64_t row = (tok_first + j0 + j) * p.H + h;
            if (p.taps)
                load_vectors_conv<D, TIO>(tv[j], w, p.taps, p.q, p.k, p.v, p.g, p.beta, row, true);
            else
                load_token<D, TIO>(tv[j], p, row);
        }
        __syncthreads();
        if (warp < nb) token_finish<D>(tv[warp], p.taps > 0, true);
        for (int j = Sh::NW; j < nb; ++j)
            if (warp == 0) token_finish<D>(tv[j], p.taps > 0, true);
        __syncthreads();
        for (int j = 0; j < nb; ++j) {
            const float4 o = kda_step<D>(st, tv[j], red[parity], p.scale);
            parity ^= 1;
            const int64_t row = (tok_first + j0 + j) * p.H + h;
            if (rs == 0) IO<TIO>::st4(static_cast<TIO *>(p.o) + row * D + cg * 4, o);
        }
    }
}

}  // namespace kda
