// KDA chunked prefill on the tcgen05 tensor cores (d_k = d_v = 128, chunk 64,
// bf16 q/k/v/o, fp32 state). The chunk form is the one in prefill_common.cuh.
//
// One CTA (128 threads) walks the chunks of one (sequence, head, 64-column
// d_v slice); d_v columns are independent, so two CTAs per head run in
// parallel. Per chunk:
//   TMA      q, k (bf16, 128B-swizzled slabs), g (fp32) and the v slice; the
//            next chunk's loads are issued as soon as this chunk's are consumed.
//   CUDA     b = cumsum(g); a per-channel reference m = b at the chunk middle;
//   cores    Qh = q.exp(b-m), Ka = k.exp(b-m), Kb = k.exp(m-b) (bf16 operands),
//            so that Qh Kb^T = A_qk and Ka Kb^T = A_kk with every exponent
//            inside the chunk bounded by half the chunk's decay range.
//   tcgen05  [Qh; Ka] Kb^T -> TMEM (M=128: A_qk rows 0-63, A_kk rows 64-127)
//   CUDA     T = (I + Diag(beta) A_kk)^{-1} Diag(beta) by blocked forward
//   cores    substitution in fp32 (16x16 diagonal blocks, then merges)
//   tcgen05  Wk = T Ka, U = T V                      (M=64)
//            W = U - Wk Sm, O = Qh Sm                (M=64; Sm = Diag(e^m) S_0)
//            O += A_qk W, D = Kb^T W                 (M=64 / M=128)
//   CUDA     o = scale O (bf16 store); S_C = Diag(Gamma_C) S_0 + Diag(e^(b_C-m)) D
//   cores    with the fp32 master state held in registers (thread = d_k row).
// Identities used: Q.Gamma = Qh.e^m and K.Gamma = Ka.e^m, so (Q.Gamma) S_0 =
// Qh Sm and (K.Gamma) S_0 = Ka Sm; K.exp(b_C-b) = Kb.e^(b_C-m) row-wise.
// A chunk whose per-channel decay from its middle exceeds 80 nats in either
// direction is reported through the status word (KDA_ERR_RANGE).
#pragma once
#include <cudaTypedefs.h>

#include "prefill_common.cuh"
#include "tc_util.cuh"

namespace kda {

struct TcParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_g;
    PrefillParams p;
};

namespace tcp {
constexpr int C = 64, D = 128, DVS = 64, NT = 128;
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t STG_Q = 0;          // q   [64 tok x 128 ch] bf16: 2 slabs of 64 rows
constexpr uint32_t STG_K = 16384;      // k   same
constexpr uint32_t STG_V = 32768;      // v   slice, 2 buffers of 1 slab [64 tok x 64]
constexpr uint32_t OP_AK = 49152;      // [Qh; Ka]: 2 slabs of 128 rows (channels 0-63, 64-127)
constexpr uint32_t OP_KB = 81920;      // Kb: 2 slabs of 64 rows
constexpr uint32_t OP_T = 98304;       // T  [64 x 64]
constexpr uint32_t OP_WK = 106496;     // Wk [64 tok x 128 ch]: 2 slabs of 64 rows
constexpr uint32_t OP_AQK = 122880;    // A_qk masked [64 x 64]
constexpr uint32_t OP_W = 131072;      // W  [64 tok x 64 dv]
constexpr uint32_t OP_SM = 139264;     // Sm [128 ch x 64 dv]: 1 slab of 128 rows
constexpr uint32_t STG_G = 155648;     // g -> b, fp32 [64][128]
constexpr uint32_t SOLVE = 188416;     // fp32 [64][65]: L, then X
constexpr uint32_t VEC = SOLVE + 64 * 65 * 4;  // mC, eM, eC, gC [128] + bet [64]
constexpr uint32_t BARS = VEC + (4 * 128 + 64) * 4;
constexpr uint32_t SMEM_USED = BARS + 32;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
// TMEM columns
constexpr uint32_t COL_A = 0, COL_WK = 64, COL_W = 192, COL_O = 256, COL_S = 320, TMEM_COLS = 512;
constexpr uint32_t CHUNK_TX = 16384 + 16384 + 32768 + 8192;   // bytes per chunk of loads
constexpr float RANGE_LIMIT = 80.f;
}  // namespace tcp

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}

__global__ void __launch_bounds__(128, 1) prefill_tc_kernel(const __grid_constant__ TcParams P) {
    using namespace tcp;
    const PrefillParams &p = P.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float *Gs = reinterpret_cast<float *>(sm + STG_G);
    float *Ls = reinterpret_cast<float *>(sm + SOLVE);
    float *mC = reinterpret_cast<float *>(sm + VEC);
    float *eM = mC + 128, *eC = mC + 256, *gC = mC + 384, *bet = mC + 512;
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(sm + BARS);   // [2]
    uint64_t *mma_bar = tma_bar + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_bar + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    const int item = blockIdx.x;
    const int rank = item / (H * 2);
    const int h = (item >> 1) % H;
    const int j0 = (item & 1) * DVS;
    const int s = p.order[rank];
    const PrefillSeq sq = p.seq[s];
    const int n_chunks = (sq.len + C - 1) / C;

    if (tid == 0) {
        tc::bar_init(&tma_bar[0], 1);
        tc::bar_init(&tma_bar[1], 1);
        tc::bar_init(mma_bar, 1);
        tc::bar_init_fence();
        tc::tma_prefetch_desc(&P.tm_q);
        tc::tma_prefetch_desc(&P.tm_k);
        tc::tma_prefetch_desc(&P.tm_v);
        tc::tma_prefetch_desc(&P.tm_g);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = (uint32_t)(32 * warp) << 16;   // this warp's TMEM sub-partition

    // fp32 master state: thread tid owns row tid (a d_k channel), 64 columns
    float S[DVS];
    {
        const float *src = p.state_in ? p.state_in + (((int64_t)s * H + h) * D + tid) * D + j0 : nullptr;
#pragma unroll
        for (int j = 0; j < DVS; j += 4) {
            float4 v = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
        }
    }

    auto issue_loads = [&](int ci) {
        uint64_t *bar = &tma_bar[ci & 1];
        const int z = sq.tok0 + ci * C;
        tc::bar_expect_tx(bar, CHUNK_TX);
        tc::tma_load3(sm + STG_Q, &P.tm_q, 0, h, z, bar);
        tc::tma_load3(sm + STG_Q + 8192, &P.tm_q, 64, h, z, bar);
        tc::tma_load3(sm + STG_K, &P.tm_k, 0, h, z, bar);
        tc::tma_load3(sm + STG_K + 8192, &P.tm_k, 64, h, z, bar);
        tc::tma_load3(sm + STG_G, &P.tm_g, 0, h, z, bar);
        tc::tma_load3(sm + STG_V + (ci & 1) * 8192, &P.tm_v, j0, h, z, bar);
    };

    int issued = 0;                 // chunks whose loads were issued (thread 0's view)
    int landed = 0;                 // chunks whose loads were waited for (all threads)
    uint32_t mma_phase = 0;
    bool ok = true;
    int64_t snap_row = sq.snap_off;
    if (tid == 0 && n_chunks > 0) {
        issue_loads(0);
        issued = 1;
    }

    for (int ci = 0; ci < n_chunks; ++ci) {
        const int n = min(C, sq.len - ci * C);
        // ---- A. this chunk's operands have landed --------------------------
        ok = tc::bar_wait(&tma_bar[ci & 1], (ci >> 1) & 1);
        if (!__syncthreads_and(ok)) { ok = false; break; }
        landed = ci + 1;
        // ---- B. beta, cumsum of g, per-channel scalars, Sm = Diag(e^m) S ---
        if (tid < C) bet[tid] = tid < n ? p.beta[(int64_t)(sq.tok0 + ci * C + tid) * H + h] : 0.f;
        {
            const int c = tid;
            float b = 0.f, m = 0.f, b0 = 0.f;
#pragma unroll 8
            for (int r = 0; r < C; ++r) {
                const float gv = r < n ? Gs[r * D + c] : 0.f;
                b += gv;
                Gs[r * D + c] = b;
                if (r == 0) b0 = b;
                if (r == C / 2 - 1) m = b;
            }
            mC[c] = m;
            const float em = expf(m);
            eM[c] = em;
            eC[c] = expf(b - m);
            gC[c] = expf(b);
            if (b0 - m > RANGE_LIMIT || m - b > RANGE_LIMIT) record_status(KDA_ERR_RANGE);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 u;
                u.x = pack_bf16(S[8 * cc + 0] * em, S[8 * cc + 1] * em);
                u.y = pack_bf16(S[8 * cc + 2] * em, S[8 * cc + 3] * em);
                u.z = pack_bf16(S[8 * cc + 4] * em, S[8 * cc + 5] * em);
                u.w = pack_bf16(S[8 * cc + 6] * em, S[8 * cc + 7] * em);
                *reinterpret_cast<uint4 *>(sm + OP_SM + tc::sw128(c, cc)) = u;
            }
        }
        __syncthreads();
        // ---- C. scaled bf16 operands Qh, Ka, Kb -----------------------------
#pragma unroll 2
        for (int j = 0; j < 8; ++j) {
            const int unit = tid + NT * j;
            const int r = unit >> 4, u = unit & 15, kb = u >> 3, cc = u & 7;
            const uint32_t so = kb * 8192 + tc::sw128(r, cc);
            const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + STG_Q + so);
            const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + STG_K + so);
            const int c0 = kb * 64 + cc * 8;
            const float4 b_lo = *reinterpret_cast<const float4 *>(Gs + r * D + c0);
            const float4 b_hi = *reinterpret_cast<const float4 *>(Gs + r * D + c0 + 4);
            const float bv[8] = {b_lo.x, b_lo.y, b_lo.z, b_lo.w, b_hi.x, b_hi.y, b_hi.z, b_hi.w};
            const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
            const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
            uint32_t oq[4], oa[4], ob[4];
            const bool live = r < n;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 qf = unpack_bf16(qw[e]), kf = unpack_bf16(kw[e]);
                const float m0 = mC[c0 + 2 * e], m1 = mC[c0 + 2 * e + 1];
                const float e10 = expf(bv[2 * e] - m0), e11 = expf(bv[2 * e + 1] - m1);
                const float e20 = expf(m0 - bv[2 * e]), e21 = expf(m1 - bv[2 * e + 1]);
                oq[e] = live ? pack_bf16(qf.x * e10, qf.y * e11) : 0u;
                oa[e] = live ? pack_bf16(kf.x * e10, kf.y * e11) : 0u;
                ob[e] = live ? pack_bf16(kf.x * e20, kf.y * e21) : 0u;
            }
            *reinterpret_cast<uint4 *>(sm + OP_AK + kb * 16384 + tc::sw128(r, cc)) =
                make_uint4(oq[0], oq[1], oq[2], oq[3]);
            *reinterpret_cast<uint4 *>(sm + OP_AK + kb * 16384 + tc::sw128(64 + r, cc)) =
                make_uint4(oa[0], oa[1], oa[2], oa[3]);
            *reinterpret_cast<uint4 *>(sm + OP_KB + kb * 8192 + tc::sw128(r, cc)) =
                make_uint4(ob[0], ob[1], ob[2], ob[3]);
        }
        tc::fence_async_smem();
        __syncthreads();
        // ---- D. next chunk's loads; A = [Qh; Ka] Kb^T ------------------------
        if (tid == 0) {
            if (ci + 1 < n_chunks) {
                issue_loads(ci + 1);
                issued = ci + 2;
            }
            tc::fence_after_sync();
            constexpr uint32_t id = tc::idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_A, tc::desc_k(sbase + OP_AK + (k >> 2) * 16384, 16 * (k & 3)),
                             tc::desc_k(sbase + OP_KB + (k >> 2) * 8192, 16 * (k & 3)), id, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
        // ---- E. A_qk (masked, bf16 operand) and L = Diag(beta) A_kk (fp32) --
        {
            const int r = tid & 63;
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + COL_A + 32 * half, a);
                tc::tmem_ld_wait();
                if (warp < 2) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = 32 * half + 8 * q4 + 2 * e;
                            w[e] = pack_bf16(jj <= r ? a[8 * q4 + 2 * e] : 0.f,
                                             jj + 1 <= r ? a[8 * q4 + 2 * e + 1] : 0.f);
                        }
                        *reinterpret_cast<uint4 *>(sm + OP_AQK + tc::sw128(r, 4 * half + q4)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
                    const float br = bet[r];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int jj = 32 * half + e;
                        Ls[r * 65 + jj] = jj < r ? br * a[e] : 0.f;
                    }
                }
            }
        }
        __syncthreads();
        // ---- F. X = (I + L)^{-1}, blocked by 16; T = X Diag(beta) -----------
        // F1: the four 16x16 diagonal blocks, one column per thread (64 threads)
        if (tid < 64) {
            const int blk = tid >> 4, c = tid & 15, base = 16 * blk;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = r == c ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) acc = fmaf(-Ls[(base + r) * 65 + base + i], x[i], acc);
                x[r] = acc;
            }
            // X overwrites L inside the diagonal block (L there is no longer needed
            // by other threads: each thread reads only its own block's rows)
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 16; ++r) Ls[(base + r) * 65 + base + c] = x[r];
        }
        __syncthreads();
        // F2: off-diagonal blocks by distance d = R - Cb = 1, 2, 3:
        //   X[R][Cb] = -X[R][R] * sum_{Cb <= J < R} L[R][J] X[J][Cb]
        // L stays in Ls (off-diagonal blocks), the diagonal blocks of Ls now
        // hold X[b][b]; the six off-diagonal X blocks and the partial sums Y
        // live in the OP_WK region, which is free until step H writes Wk.
        float *Xo = reinterpret_cast<float *>(sm + OP_WK);   // 6 blocks of 16x16
        float *Y = Xo + 6 * 256;                               // up to 3 blocks
        auto xslot = [](int dist, int bi) { return (dist == 1 ? 0 : dist == 2 ? 3 : 5) + bi; };
#pragma unroll 1
        for (int dist = 1; dist < 4; ++dist) {
            const int nb = 4 - dist;                 // blocks at this distance
            for (int e = tid; e < nb * 256; e += NT) {
                const int bi = e >> 8, a = (e >> 4) & 15, bcol = e & 15;
                const int R = bi + dist, Cb = bi;
                float acc = 0.f;
                for (int J = Cb; J < R; ++J) {
                    const float *xj = J == Cb ? Ls + (16 * J) * 65 + 16 * Cb : Xo + xslot(J - Cb, Cb) * 256;
                    const int xs = J == Cb ? 65 : 16;
#pragma unroll
                    for (int l = 0; l < 16; ++l)
                        acc = fmaf(Ls[(16 * R + a) * 65 + 16 * J + l], xj[l * xs + bcol], acc);
                }
                Y[e] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nb * 256; e += NT) {
                const int bi = e >> 8, a = (e >> 4) & 15, bcol = e & 15;
                const int R = bi + dist;
                float acc = 0.f;
#pragma unroll
                for (int l = 0; l < 16; ++l)
                    acc = fmaf(Ls[(16 * R + a) * 65 + 16 * R + l], Y[(bi << 8) + (l << 4) + bcol], acc);
                Xo[xslot(dist, bi) * 256 + a * 16 + bcol] = -acc;
            }
            __syncthreads();
        }
        // T[r][c] = X[r][c] beta_c (zero above the diagonal) -> bf16 slab
        for (int e = tid; e < 64 * 8; e += NT) {
            const int r = e >> 3, cc = e & 7;
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float x2[2];
#pragma unroll
                for (int t2 = 0; t2 < 2; ++t2) {
                    const int c = 8 * cc + 2 * q + t2;
                    const int R = r >> 4, Cb = c >> 4;
                    float x = 0.f;
                    if (R == Cb) x = c <= r ? Ls[r * 65 + c] : 0.f;
                    else if (R > Cb) x = Xo[xslot(R - Cb, Cb) * 256 + (r & 15) * 16 + (c & 15)];
                    x2[t2] = x * bet[c];
                }
                w[q] = pack_bf16(x2[0], x2[1]);
            }
            *reinterpret_cast<uint4 *>(sm + OP_T + tc::sw128(r, cc)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        // ---- G. Wk = T Ka, U = T V --------------------------------------------
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_wk = tc::idesc_bf16(64, 128, false, true);
            constexpr uint32_t id_u = tc::idesc_bf16(64, 64, false, true);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_bf16(tbase + COL_WK, tc::desc_k(sbase + OP_T, 16 * k),
                             tc::desc_mn(sbase + OP_AK + 64 * 128, 16 * k, 16384), id_wk, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_bf16(tbase + COL_W, tc::desc_k(sbase + OP_T, 16 * k),
                             tc::desc_mn(sbase + STG_V + (ci & 1) * 8192, 16 * k, 8192), id_u, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
        // ---- H. Wk -> bf16 operand (M=64 layout: lanes 32w..32w+15 = rows 16w..) ---
        {
            const int r = 16 * warp + (lane & 15);
            float a[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                tc::tmem_ld32(tbase + tlane + COL_WK + 32 * q, a);
                tc::tmem_ld_wait();
                if (lane < 16) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + OP_WK + (q >> 1) * 8192 + tc::sw128(r, 4 * (q & 1) + q4)) =
                            make_uint4(pack_bf16(a[8 * q4], a[8 * q4 + 1]), pack_bf16(a[8 * q4 + 2], a[8 * q4 + 3]),
                                       pack_bf16(a[8 * q4 + 4], a[8 * q4 + 5]), pack_bf16(a[8 * q4 + 6], a[8 * q4 + 7]));
                }
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        // ---- I. W = U - Wk Sm ; O = Qh Sm ---------------------------------------
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_w = tc::idesc_bf16(64, 64, false, true, /*a_neg=*/true);
            constexpr uint32_t id_o = tc::idesc_bf16(64, 64, false, true);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_W, tc::desc_k(sbase + OP_WK + (k >> 2) * 8192, 16 * (k & 3)),
                             tc::desc_mn(sbase + OP_SM, 16 * k, 8192), id_w, 1);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_O, tc::desc_k(sbase + OP_AK + (k >> 2) * 16384, 16 * (k & 3)),
                             tc::desc_mn(sbase + OP_SM, 16 * k, 8192), id_o, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
        // ---- J. W -> bf16 operand ------------------------------------------------
        {
            const int r = 16 * warp + (lane & 15);
            float a[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tbase + tlane + COL_W + 32 * q, a);
                tc::tmem_ld_wait();
                if (lane < 16) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + OP_W + tc::sw128(r, 4 * q + q4)) =
                            make_uint4(pack_bf16(a[8 * q4], a[8 * q4 + 1]), pack_bf16(a[8 * q4 + 2], a[8 * q4 + 3]),
                                       pack_bf16(a[8 * q4 + 4], a[8 * q4 + 5]), pack_bf16(a[8 * q4 + 6], a[8 * q4 + 7]));
                }
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        // ---- K. O += A_qk W ; D = Kb^T W -----------------------------------------
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_o = tc::idesc_bf16(64, 64, false, true);
            constexpr uint32_t id_s = tc::idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_bf16(tbase + COL_O, tc::desc_k(sbase + OP_AQK, 16 * k),
                             tc::desc_mn(sbase + OP_W, 16 * k, 8192), id_o, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_bf16(tbase + COL_S, tc::desc_mn(sbase + OP_KB, 16 * k, 8192),
                             tc::desc_mn(sbase + OP_W, 16 * k, 8192), id_s, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
        // ---- L. outputs, state update, snapshot ---------------------------------
        {
            const int r = 16 * warp + (lane & 15);
            float a[32];
            __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.o);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tbase + tlane + COL_O + 32 * q, a);
                tc::tmem_ld_wait();
                if (lane < 16 && r < n) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        og + ((int64_t)(sq.tok0 + ci * C + r) * H + h) * D + j0 + 32 * q);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(pack_bf16(p.scale * a[8 * q4], p.scale * a[8 * q4 + 1]),
                                             pack_bf16(p.scale * a[8 * q4 + 2], p.scale * a[8 * q4 + 3]),
                                             pack_bf16(p.scale * a[8 * q4 + 4], p.scale * a[8 * q4 + 5]),
                                             pack_bf16(p.scale * a[8 * q4 + 6], p.scale * a[8 * q4 + 7]));
                }
            }
            const float g_c = gC[tid], e_c = eC[tid];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tbase + tlane + COL_S + 32 * q, a);
                tc::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) S[32 * q + e] = fmaf(g_c, S[32 * q + e], e_c * a[e]);
            }
            if (p.snap_interval > 0 && (sq.start_pos + (int64_t)ci * C + n) % p.snap_interval == 0) {
                float *dst = p.snapshots + ((snap_row * H + h) * D + tid) * (int64_t)D + j0;
#pragma unroll
                for (int j = 0; j < DVS; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
                ++snap_row;
            }
        }
        tc::fence_before_sync();
        __syncthreads();
    }

    if (ok && p.state_out) {
        float *dst = p.state_out + (((int64_t)s * H + h) * D + tid) * (int64_t)D + j0;
#pragma unroll
        for (int j = 0; j < DVS; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    // teardown: on an early exit, let loads already in flight land before the
    // shared memory is released (bounded), then free TMEM
    if (tid == 0 && !ok) {
        for (int c2 = landed; c2 < issued; ++c2) tc::bar_wait(&tma_bar[c2 & 1], (c2 >> 1) & 1, 1u << 16);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, TMEM_COLS);
}

// ---------------------------------------------------------------------------- host
inline bool tc_prefill_supported(const kda_dims &d) {
    return d.dk == 128 && d.dv == 128 && d.chunk == 64 && d.io == KDA_IO_BF16;
}

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [T, H, 128] tensor, boxes of (inner, 1 head, 64 tokens)
inline bool encode_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t esize, int H,
                       int64_t T, uint32_t box_inner, CUtensorMapSwizzle sw) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)128 * esize, (cuuint64_t)H * 128 * esize};
    cuuint32_t box[3] = {box_inner, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Gate>
inline kda_status launch_prefill_tc(PrefillParams &p, const kda_dims &d, int64_t T, cudaStream_t st, Gate gate) {
    static thread_local TcParams P;
    const int H = d.H;
    if (!encode_map(&P.tm_q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map(&P.tm_k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map(&P.tm_v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map(&P.tm_g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, T, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return KDA_ERR_CUDA;
    P.p = p;
    P.p.n_items = p.n_seq * H * 2;
    static bool attr_done = false;
    if (!attr_done) {
        if (cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tcp::SMEM_BYTES) != cudaSuccess)
            return KDA_ERR_CUDA;
        attr_done = true;
    }
    if (!gate()) return KDA_ERR_CUDA;
    prefill_tc_kernel<<<P.p.n_items, tcp::NT, tcp::SMEM_BYTES, st>>>(P);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda
