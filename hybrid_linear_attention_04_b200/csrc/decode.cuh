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
// The d_v columns of S evolve independently (w, the update and o are per column),
// so warp w owns the 16 columns 16w .. 16w+15 over all d_k rows: lane l holds the
// float4 of columns 16w + 4 (l % 4) .. +3 in rows l / 4 + 8 m, m < D / 8. The column
// sums over d_k reduce inside the lane, then across the 8 lanes that share the
// column group (three butterfly shuffles, so every lane holds the same sum); a
// token step has no barrier and no shared-memory reduction. Decode, verify and the
// commit replay run the same step function, so verify's state after its j-th token
// is bit-identical to j decode calls.
//
// Token vectors are staged in shared memory a batch at a time: threads t < D own
// channel t of q and k (and run the q/k front-end's conv window in token order),
// threads t >= D channel t - D of v and g; each thread issues all its loads for the
// batch before it uses any.
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

__device__ __forceinline__ float swish(float y) { return y / (1.f + expf(-y)); }

// Per-token vectors staged in shared memory. 16-byte aligned (and padded to a
// multiple of 16 bytes) because the step reads v with float4 loads.
template <int D> struct __align__(16) TokVec {
    float k[D], q[D], a[D], v[D];
    float beta, kq;
};
static_assert(sizeof(TokVec<128>) % 16 == 0 && sizeof(TokVec<32>) % 16 == 0, "TokVec padding");

// Verify: tokens are processed in batches of kTokBatch staged in shared memory.
constexpr int kTokBatch = 8;

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

// Stage nb <= kTokBatch tokens, rows row0 + j * rstride (= token * H + head) of the
// packed arrays, into tv[0..nb). q_ may be null (a replayed token whose output is not
// needed: with the front-end its q still moves the conv window). With CONV, q and k
// are raw and pass through the conv and Swish here (window w of the thread's
// channel); token_finish normalises them.
template <int D, typename TIO, bool CONV>
__device__ __forceinline__ void stage_batch(TokVec<D> *tv, int nb, int64_t row0, int64_t rstride,
                                            const void *q_, const void *k_, const void *v_,
                                            const float *g_, const float *beta, ConvWin &w,
                                            const DecodeParams &p, int h, const ConvOut &co) {
    constexpr int L = kTokBatch / 2;      // loads in flight per array (register budget)
    const int t = threadIdx.x;
    if (t < D) {
        const TIO *q = static_cast<const TIO *>(q_), *k = static_cast<const TIO *>(k_);
        for (int j0 = 0; j0 < nb; j0 += L) {
            float xq[L], xk[L];
#pragma unroll
            for (int j = 0; j < L; ++j) {
                if (j0 + j < nb) {
                    const int64_t off = (row0 + (j0 + j) * rstride) * D + t;
                    xq[j] = (q_ != nullptr) ? IO<TIO>::ld(q + off) : 0.f;
                    xk[j] = IO<TIO>::ld(k + off);
                }
            }
#pragma unroll
            for (int j = 0; j < L; ++j) {
                const int jj = j0 + j;
                if (jj < nb) {
                    if (CONV) {
                        const float yq = conv_step(w.q, p.taps, xq[j]);
                        const float yk = conv_step(w.k, p.taps, xk[j]);
                        tv[jj].q[t] = q_ != nullptr ? swish(yq) : 0.f;
                        tv[jj].k[t] = swish(yk);
                        if (co.tok) conv_store(w, p, co.tok, co.tok0 + jj, h, D, t);
                        if (jj == co.snap_j) conv_store(w, p, co.snap, co.snap_row, h, D, t);
                    } else {
                        tv[jj].q[t] = xq[j];
                        tv[jj].k[t] = xk[j];
                    }
                }
            }
        }
    } else {
        const int c = t - D;
        const TIO *v = static_cast<const TIO *>(v_);
        const float b = c < nb ? beta[row0 + c * rstride] : 0.f;
        for (int j0 = 0; j0 < nb; j0 += L) {
            float xv[L], xg[L];
#pragma unroll
            for (int j = 0; j < L; ++j) {
                if (j0 + j < nb) {
                    const int64_t off = (row0 + (j0 + j) * rstride) * D + c;
                    xv[j] = IO<TIO>::ld(v + off);
                    xg[j] = g_[off];
                }
            }
#pragma unroll
            for (int j = 0; j < L; ++j) {
                if (j0 + j < nb) {
                    tv[j0 + j].v[c] = xv[j];
                    tv[j0 + j].a[c] = expf(xg[j]);
                }
            }
        }
        if (c < nb) tv[c].beta = b;
    }
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

// Finish nb staged tokens (warp j takes token j, warp 0 the rest) between barriers.
template <int D>
__device__ __forceinline__ void finish_batch(TokVec<D> *tv, int nb, bool normalise, bool with_q) {
    const int warp = threadIdx.x >> 5;
    __syncthreads();
    if (warp < nb) token_finish<D>(tv[warp], normalise, with_q);
    for (int j = DecodeShape<D>::NW; j < nb; ++j)
        if (warp == 0) token_finish<D>(tv[j], normalise, with_q);
    __syncthreads();
}

// One recurrence step on the register-resident columns of this warp. With OUT =
// false the output read (y and o) is skipped; the state arithmetic is the same
// instruction for instruction, so both forms give bit-identical states. The
// returned o (OUT) holds the lane's four columns; every lane of a column group has it.
template <int D, bool OUT = true>
__device__ __forceinline__ float4 kda_step(float4 (&st)[DecodeShape<D>::R], const TokVec<D> &tv, float scale) {
    using Sh = DecodeShape<D>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cg = lane & 3, rg = lane >> 2;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) {
        const int r = rg + 8 * m;
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
    for (int off = 4; off < 32; off <<= 1) {
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
    const float4 vv = *reinterpret_cast<const float4 *>(tv.v + 16 * warp + 4 * cg);
    float4 wv;
    wv.x = tv.beta * (vv.x - x.x); wv.y = tv.beta * (vv.y - x.y);
    wv.z = tv.beta * (vv.z - x.z); wv.w = tv.beta * (vv.w - x.w);
#pragma unroll
    for (int m = 0; m < Sh::R; ++m) {
        const float kr = tv.k[rg + 8 * m];
        float4 s = st[m];
        s.x = fmaf(kr, wv.x, s.x); s.y = fmaf(kr, wv.y, s.y);
        s.z = fmaf(kr, wv.z, s.z); s.w = fmaf(kr, wv.w, s.w);
        st[m] = s;
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (OUT) {
        o.x = scale * fmaf(tv.kq, wv.x, y.x); o.y = scale * fmaf(tv.kq, wv.y, y.y);
        o.z = scale * fmaf(tv.kq, wv.z, y.z); o.w = scale * fmaf(tv.kq, wv.w, y.w);
    }
    return o;
}

// offset of the lane's float4 in row m of a state
template <int D>
__device__ __forceinline__ int64_t lane_off(int m) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    return (int64_t)((lane >> 2) + 8 * m) * D + 16 * warp + 4 * (lane & 3);
}
template <int D>
__device__ __forceinline__ int lane_col() {
    return 16 * (threadIdx.x >> 5) + 4 * (threadIdx.x & 3);
}

template <int D>
__device__ __forceinline__ void load_state(float4 (&st)[DecodeShape<D>::R], const float *S) {
#pragma unroll
    for (int m = 0; m < DecodeShape<D>::R; ++m) {
        const float *src = S + lane_off<D>(m);
        asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(st[m].x), "=f"(st[m].y), "=f"(st[m].z), "=f"(st[m].w)
                     : "l"(src));
    }
}
template <int D>
__device__ __forceinline__ void store_state(const float4 (&st)[DecodeShape<D>::R], float *S) {
#pragma unroll
    for (int m = 0; m < DecodeShape<D>::R; ++m) st_stream(S + lane_off<D>(m), st[m]);
}

// ---- token rows staged by bulk copies (verify, verify + commit) ----------------
// A CTA's tokens form one stream of batches of up to kTokBatch tokens (verify+commit:
// the replayed prefix, then this step's tokens). Thread 0 copies a batch's raw q, k, v
// and g rows into one of two shared-memory buffers with bulk asynchronous copies that
// complete on that buffer's mbarrier, two batches ahead of their use, so the rows of
// every batch arrive while the state is loaded and the previous batch is stepped.
template <int D, typename TIO> struct RawTok {
    static constexpr uint32_t QB = D * sizeof(TIO);     // one q, k or v row
    static constexpr uint32_t BYTES = 3 * QB + D * 4;   // + one g row (fp32)
    static constexpr uint32_t SMEM = 2 * kTokBatch * BYTES;   // dynamic shared memory
};

struct TokSrc {                 // tokens row0, row0 + H, ... of packed arrays
    const void *q, *k, *v;      // q null: not staged (a replayed token without front-end)
    const float *g, *beta;
    int64_t row0;
    int n;
};

template <int D, typename TIO>
__device__ __forceinline__ void issue_rows(uint8_t *raw, const TokSrc &src, int j0, int nb, int H,
                                           uint64_t *bar) {
    using RT = RawTok<D, TIO>;
    const uint32_t per = src.q ? RT::BYTES : RT::BYTES - RT::QB;   // every row keeps its slot
    tc::bar_expect_tx(bar, per * (uint32_t)nb);
    for (int j = 0; j < nb; ++j) {
        const int64_t row = src.row0 + (int64_t)(j0 + j) * H;
        uint8_t *dst = raw + j * RT::BYTES;
        if (src.q) tc::bulk_load(dst, static_cast<const TIO *>(src.q) + row * D, RT::QB, bar);
        tc::bulk_load(dst + RT::QB, static_cast<const TIO *>(src.k) + row * D, RT::QB, bar);
        tc::bulk_load(dst + 2 * RT::QB, static_cast<const TIO *>(src.v) + row * D, RT::QB, bar);
        tc::bulk_load(dst + 3 * RT::QB, src.g + row * D, D * 4, bar);
    }
}

// Staged raw rows -> token vectors (the front-end's conv and Swish with CONV): threads
// t < D channel t of q and k, in token order; threads t >= D channel t - D of v and g.
// b: this thread's beta (threads D .. D + nb - 1), loaded ahead.
template <int D, typename TIO, bool CONV>
__device__ __forceinline__ void convert_batch(TokVec<D> *tv, const uint8_t *raw, int nb, bool read_q,
                                              bool with_q, float b, ConvWin &w, const DecodeParams &p, int h,
                                              const ConvOut &co) {
    using RT = RawTok<D, TIO>;
    const int t = threadIdx.x;
    if (t < D) {
        for (int j = 0; j < nb; ++j) {
            const uint8_t *rj = raw + j * RT::BYTES;
            const float xq = read_q ? IO<TIO>::ld(reinterpret_cast<const TIO *>(rj) + t) : 0.f;
            const float xk = IO<TIO>::ld(reinterpret_cast<const TIO *>(rj + RT::QB) + t);
            if (CONV) {
                const float yq = conv_step(w.q, p.taps, xq);
                const float yk = conv_step(w.k, p.taps, xk);
                tv[j].q[t] = with_q ? swish(yq) : 0.f;
                tv[j].k[t] = swish(yk);
                if (co.tok) conv_store(w, p, co.tok, co.tok0 + j, h, D, t);
                if (j == co.snap_j) conv_store(w, p, co.snap, co.snap_row, h, D, t);
            } else {
                tv[j].q[t] = with_q ? xq : 0.f;
                tv[j].k[t] = xk;
            }
        }
    } else {
        const int c = t - D;
        for (int j = 0; j < nb; ++j) {
            const uint8_t *rj = raw + j * RT::BYTES;
            tv[j].v[c] = IO<TIO>::ld(reinterpret_cast<const TIO *>(rj + 2 * RT::QB) + c);
            tv[j].a[c] = expf(reinterpret_cast<const float *>(rj + 3 * RT::QB)[c]);
        }
        if (c < nb) tv[c].beta = b;
    }
}

// The batch stream of one CTA: batches of a, then of b. (Two members and selects, not
// an array indexed at run time, so that the stream stays in registers.)
struct TokStream {
    TokSrc a, b;
    int nb0, nbat;              // batches of a; all batches
    __device__ __forceinline__ void locate(int bi, int &which, int &j0, int &nb) const {
        which = bi < nb0 ? 0 : 1;
        j0 = (which ? bi - nb0 : bi) * kTokBatch;
        nb = min(kTokBatch, (which ? b.n : a.n) - j0);
    }
    __device__ __forceinline__ TokSrc pick(int which) const {
        TokSrc r;
        r.q = which ? b.q : a.q;
        r.k = which ? b.k : a.k;
        r.v = which ? b.v : a.v;
        r.g = which ? b.g : a.g;
        r.beta = which ? b.beta : a.beta;
        r.row0 = which ? b.row0 : a.row0;
        r.n = which ? b.n : a.n;
        return r;
    }
};

__device__ __forceinline__ TokStream make_stream(const TokSrc &a, const TokSrc &b) {
    TokStream s;
    s.a = a;
    s.b = b;
    s.nb0 = (a.n + kTokBatch - 1) / kTokBatch;
    s.nbat = s.nb0 + (b.n + kTokBatch - 1) / kTokBatch;
    return s;
}

template <int D, typename TIO>
__device__ __forceinline__ void issue_batch(const TokStream &ts, int bi, uint8_t *raw, uint64_t *bar, int H) {
    int which, j0, nb;
    ts.locate(bi, which, j0, nb);
    issue_rows<D, TIO>(raw, ts.pick(which), j0, nb, H, bar);
}

// beta of token c of batch bi (threads D + c), issued early as a plain load
__device__ __forceinline__ float batch_beta(const TokStream &ts, int bi, int c, int H) {
    int which, j0, nb;
    ts.locate(bi, which, j0, nb);
    const TokSrc src = ts.pick(which);
    return c < nb ? src.beta[src.row0 + (int64_t)(j0 + c) * H] : 0.f;
}

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
    float4 st[DecodeShape<D>::R];
    load_state<D>(st, S);
    const int64_t row = (int64_t)s * p.H + h;
    ConvWin w;
    if (CONV && t < D) conv_begin(w, p, p.conv, slot, h, D, t);
    const ConvOut none{nullptr, 0, nullptr, 0, -1};
    stage_batch<D, TIO, CONV>(&tv, 1, row, 0, p.q, p.k, p.v, p.g, p.beta, w, p, h, none);
    if (CONV && t < D) conv_store(w, p, p.conv, slot, h, D, t);
    finish_batch<D>(&tv, 1, CONV, true);
    const float4 o = kda_step<D>(st, tv, p.scale);
    store_state<D>(st, S);
    if ((t & 31) < 4) IO<TIO>::st4(static_cast<TIO *>(p.o) + row * D + lane_col<D>(), o);
}

// two CTAs per SM (register cap) keep enough state loads and stores in flight
template <int D, typename TIO, bool CONV>
__global__ void __launch_bounds__(DecodeShape<D>::NT, 2)
verify_kernel(const __grid_constant__ DecodeParams p) {
    using RT = RawTok<D, TIO>;
    __shared__ TokVec<D> tv[kTokBatch];
    extern __shared__ __align__(128) uint8_t dyn_smem[];   // two raw row buffers
    auto raw = [&](int i) { return dyn_smem + i * (kTokBatch * RT::BYTES); };
    __shared__ uint64_t bars[2];
    const int s = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int32_t slot = p.slots[s];
    if (slot < 0 || slot >= p.n_slots) {
        if (threadIdx.x == 0) record_status(KDA_ERR_RANGE);
        return;
    }
    const int n_tok = p.tok0[s + 1] - p.tok0[s];
    const int64_t tok_first = p.tok_base + p.tok0[s];
    const int t = threadIdx.x, warp = t >> 5;
    const TokSrc none{nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0};
    const TokStream ts = make_stream(TokSrc{p.q, p.k, p.v, p.g, p.beta, tok_first * p.H + h, n_tok}, none);
    if (t == 0) {
        tc::bar_init(&bars[0], 1);
        tc::bar_init(&bars[1], 1);
        tc::bar_init_fence();
        for (int bi = 0; bi < 2 && bi < ts.nbat; ++bi) issue_batch<D, TIO>(ts, bi, raw(bi), &bars[bi], p.H);
    }
    float bnext = (t >= D && ts.nbat > 0) ? batch_beta(ts, 0, t - D, p.H) : 0.f;
    const float *S = p.pool + ((int64_t)slot * p.H + h) * (int64_t)D * D;
    float4 st[DecodeShape<D>::R];
#pragma unroll
    for (int m = 0; m < DecodeShape<D>::R; ++m) st[m] = ld_stream(S + lane_off<D>(m));
    ConvWin w;
    if (CONV && t < D) conv_begin(w, p, p.conv, slot, h, D, t);
    __syncthreads();  // barrier initialisation visible
    bool ok = true;
    for (int bi = 0; bi < ts.nbat; ++bi) {
        int which, j0, nb;
        ts.locate(bi, which, j0, nb);
        const float b = bnext;
        if (t >= D && bi + 1 < ts.nbat) bnext = batch_beta(ts, bi + 1, t - D, p.H);
        ok = tc::bar_wait(&bars[bi & 1], (uint32_t)((bi >> 1) & 1)) && ok;
        const ConvOut co{p.conv_tok, tok_first + j0, nullptr, 0, -1};
        convert_batch<D, TIO, CONV>(tv, raw(bi & 1), nb, true, true, b, w, p, h, co);
        __syncthreads();  // vectors staged, raw buffer read
        if (t == 0 && bi + 2 < ts.nbat) issue_batch<D, TIO>(ts, bi + 2, raw(bi & 1), &bars[bi & 1], p.H);
        if (warp < nb) token_finish<D>(tv[warp], CONV, true);
        for (int j = DecodeShape<D>::NW; j < nb; ++j)
            if (warp == 0) token_finish<D>(tv[j], CONV, true);
        __syncthreads();
        for (int j = 0; j < nb; ++j) {
            const float4 o = kda_step<D>(st, tv[j], p.scale);
            const int64_t row = (tok_first + j0 + j) * p.H + h;
            store_state<D>(st, p.token_states + row * (int64_t)D * D);
            if ((t & 31) < 4) IO<TIO>::st4(static_cast<TIO *>(p.o) + row * D + lane_col<D>(), o);
        }
        __syncthreads();  // the vectors are free for the next batch
    }
    if (!ok && t == 0)  // copies still in flight land before the shared memory is released
        for (int bi = ts.nbat - 2 < 0 ? 0 : ts.nbat - 2; bi < ts.nbat; ++bi)
            tc::bar_wait(&bars[bi & 1], (uint32_t)((bi >> 1) & 1), 1u << 16);
}

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
    const uint8_t *commit_new;  // [n_seq] nonzero: this step's tokens are committed too (nullable)
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

template <int D, typename TIO, bool CONV>
__global__ void __launch_bounds__(DecodeShape<D>::NT, 2)
verify_commit_kernel(const __grid_constant__ VerifyCommitParams P) {
    using RT = RawTok<D, TIO>;
    const DecodeParams &p = P.p;
    const CommitParams &c = P.c;
    __shared__ TokVec<D> tv[kTokBatch];
    extern __shared__ __align__(128) uint8_t dyn_smem[];   // two raw row buffers
    auto raw = [&](int i) { return dyn_smem + i * (kTokBatch * RT::BYTES); };
    __shared__ uint64_t bars[2];
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
    const int n_tok = p.tok0[s + 1] - p.tok0[s];
    // committed tokens: the replayed prefix, then (mixed step) this step's tokens;
    // jsnap indexes that sequence
    const bool cnew = c.commit_new != nullptr && c.commit_new[s] != 0 && n_tok > 0;
    const int t = threadIdx.x, warp = t >> 5;
    // the stream: the replayed prefix of the previous batch (its q only for the front-end's
    // window), then this step's tokens
    const int64_t prev_first = c.tok_base + c.tok0[s];
    const int64_t tok_first = p.tok_base + p.tok0[s];
    const TokStream ts = make_stream(TokSrc{CONV ? c.q : nullptr, c.k, c.v, c.g, c.beta, prev_first * p.H + h, na},
                                     TokSrc{p.q, p.k, p.v, p.g, p.beta, tok_first * p.H + h, n_tok});
    if (t == 0) {
        tc::bar_init(&bars[0], 1);
        tc::bar_init(&bars[1], 1);
        tc::bar_init_fence();
        for (int bi = 0; bi < 2 && bi < ts.nbat; ++bi) issue_batch<D, TIO>(ts, bi, raw(bi), &bars[bi], p.H);
    }
    float bnext = (t >= D && ts.nbat > 0) ? batch_beta(ts, 0, t - D, p.H) : 0.f;
    float *S = p.pool + ((int64_t)slot * p.H + h) * (int64_t)D * D;
    float4 st[DecodeShape<D>::R];
    load_state<D>(st, S);
    ConvWin w;
    if (CONV && t < D) conv_begin(w, p, p.conv, slot, h, D, t);
    __syncthreads();  // barrier initialisation visible
    bool ok = true;
    for (int bi = 0; bi < ts.nbat; ++bi) {
        int which, j0, nb;
        ts.locate(bi, which, j0, nb);
        const bool replay = which == 0;
        const float b = bnext;
        if (t >= D && bi + 1 < ts.nbat) bnext = batch_beta(ts, bi + 1, t - D, p.H);
        ok = tc::bar_wait(&bars[bi & 1], (uint32_t)((bi >> 1) & 1)) && ok;
        // the committed-token index of this batch's first token, and a snapshot inside it
        const int64_t c0 = replay ? j0 : (cnew ? na + j0 : -1);
        const int64_t js = (c0 >= 0 && jsnap >= c0 && jsnap < c0 + nb) ? jsnap - c0 : -1;
        const ConvOut co{nullptr, 0, c.conv_snapshots, srow, (int)js};
        convert_batch<D, TIO, CONV>(tv, raw(bi & 1), nb, CONV || !replay, !replay, b, w, p, h, co);
        __syncthreads();  // vectors staged, raw buffer read
        if (t == 0 && bi + 2 < ts.nbat) issue_batch<D, TIO>(ts, bi + 2, raw(bi & 1), &bars[bi & 1], p.H);
        if (warp < nb) token_finish<D>(tv[warp], CONV, !replay);
        for (int j = DecodeShape<D>::NW; j < nb; ++j)
            if (warp == 0) token_finish<D>(tv[j], CONV, !replay);
        __syncthreads();
        if (replay) {
            // 1. commit: the accepted prefix, state only
            for (int j = 0; j < nb; ++j) {
                kda_step<D, false>(st, tv[j], 0.f);
                if (j == js) store_state<D>(st, c.snapshots + (srow * p.H + h) * (int64_t)D * D);
            }
            if (bi == ts.nb0 - 1 && !cnew) {
                store_state<D>(st, S);
                if (CONV && t < D) conv_store(w, p, p.conv, slot, h, D, t);
            }
        } else {
            // 2. this step's tokens from the committed state: outputs (and with commit_new
            // their state is committed too)
            for (int j = 0; j < nb; ++j) {
                const float4 o = kda_step<D>(st, tv[j], p.scale);
                const int64_t row = (tok_first + j0 + j) * p.H + h;
                if ((t & 31) < 4) IO<TIO>::st4(static_cast<TIO *>(p.o) + row * D + lane_col<D>(), o);
                if (j == js) store_state<D>(st, c.snapshots + (srow * p.H + h) * (int64_t)D * D);
            }
        }
        __syncthreads();  // the vectors are free for the next batch
    }
    if (cnew) {
        store_state<D>(st, S);
        if (CONV && t < D) conv_store(w, p, p.conv, slot, h, D, t);
    }
    if (!ok && t == 0)  // copies still in flight land before the shared memory is released
        for (int bi = ts.nbat - 2 < 0 ? 0 : ts.nbat - 2; bi < ts.nbat; ++bi)
            tc::bar_wait(&bars[bi & 1], (uint32_t)((bi >> 1) & 1), 1u << 16);
}

}  // namespace kda
