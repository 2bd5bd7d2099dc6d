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
constexpr int C = 64, D = 128, DVS = 64, NT = 256;
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t STG_Q = 0;          // q   [64 tok x 128 ch] bf16: 2 slabs of 64 rows
constexpr uint32_t STG_K = 16384;      // k   same
constexpr uint32_t STG_V = 32768;      // v   slice, 2 buffers of 1 slab [64 tok x 64]
constexpr uint32_t OP_AK = 49152;      // [Qh; Ka]: 2 slabs of 128 rows (channels 0-63, 64-127)
constexpr uint32_t OP_KB = 81920;      // Kb: 2 slabs of 64 rows
constexpr uint32_t OP_T = 98304;       // T  [64 x 64]
constexpr uint32_t OP_WK = 106496;     // Wk [64 tok x 128 ch]: 2 slabs; solve scratch before that
constexpr uint32_t OP_AQK = 122880;    // A_qk masked [64 x 64]
constexpr uint32_t OP_W = 131072;      // W  [64 tok x 64 dv]
constexpr uint32_t OP_SM = 139264;     // Sm [128 ch x 64 dv]: 1 slab of 128 rows
constexpr uint32_t STG_G = 155648;     // g, fp32 [64][128]
constexpr uint32_t SOLVE = 188416;     // fp32 [64][65]: L off the diagonal, X on it
constexpr uint32_t VEC = SOLVE + 64 * 65 * 4;  // eM, eC, gC [128] + bet [64]
constexpr uint32_t BARS = VEC + (3 * 128 + 64) * 4;
constexpr uint32_t SMEM_USED = BARS + 32;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
// TMEM columns
constexpr uint32_t COL_A = 0, COL_WK = 64, COL_W = 192, COL_O = 256, COL_S = 320, TMEM_COLS = 512;
constexpr uint32_t CHUNK_TX = 16384 + 16384 + 32768 + 8192;   // bytes per chunk of loads
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RANGE_LIMIT2 = 80.f * LOG2E;    // 80 nats, in log2 units
}  // namespace tcp

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}
__device__ __forceinline__ uint4 pack8(const float *a, float s) {
    return make_uint4(pack_bf16(s * a[0], s * a[1]), pack_bf16(s * a[2], s * a[3]),
                      pack_bf16(s * a[4], s * a[5]), pack_bf16(s * a[6], s * a[7]));
}

// slot of the off-diagonal 16x16 block X[Cb + dist][Cb] in the solve scratch
__device__ __forceinline__ int xslot(int dist, int cb) { return (dist == 1 ? 0 : dist == 2 ? 3 : 5) + cb; }

__global__ void __launch_bounds__(256, 1) prefill_tc_kernel(const __grid_constant__ TcParams P) {
    using namespace tcp;
    const PrefillParams &p = P.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float *Gs = reinterpret_cast<float *>(sm + STG_G);
    float *Ls = reinterpret_cast<float *>(sm + SOLVE);
    float *eM = reinterpret_cast<float *>(sm + VEC);
    float *eC = eM + 128, *gC = eM + 256, *bet = eM + 384;
    float *Xo = reinterpret_cast<float *>(sm + OP_WK);     // 6 blocks 16x16 (solve only)
    float *Yw = Xo + 6 * 256;                                // 3 per-warp 16x16 blocks
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(sm + BARS);   // [2]
    uint64_t *mma_bar = tma_bar + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_bar + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;          // TMEM sub-partition, column half
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
    const uint32_t tlane = (uint32_t)(32 * wq) << 16;   // this warp's TMEM sub-partition

    // fp32 master state: thread owns d_k row c_own, columns [32 wh, 32 wh + 32) of the slice
    const int c_own = tid & 127;
    float S[32];
    {
        const float *src =
            p.state_in ? p.state_in + (((int64_t)s * H + h) * D + c_own) * D + j0 + 32 * wh : nullptr;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
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
    // prep-phase thread map: channel group u (8 channels), row block rb (4 rows)
    const int pu = tid >> 4, prb = tid & 15, pc0 = 8 * pu, pkb = pu >> 3, pcc = pu & 7;

    for (int ci = 0; ci < n_chunks; ++ci) {
        const int n = min(C, sq.len - ci * C);
        // ---- A. this chunk's operands have landed --------------------------
        ok = tc::bar_wait(&tma_bar[ci & 1], (ci >> 1) & 1);
        if (!__syncthreads_and(ok)) { ok = false; break; }
        landed = ci + 1;
        // ---- B. b = cumsum(g) in log2 units: local 4 rows, then a 16-lane scan
        float b[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * prb + i;
            const float4 x0 = *reinterpret_cast<const float4 *>(Gs + r * D + pc0);
            const float4 x1 = *reinterpret_cast<const float4 *>(Gs + r * D + pc0 + 4);
            const float sc = r < n ? LOG2E : 0.f;
            b[i][0] = x0.x * sc; b[i][1] = x0.y * sc; b[i][2] = x0.z * sc; b[i][3] = x0.w * sc;
            b[i][4] = x1.x * sc; b[i][5] = x1.y * sc; b[i][6] = x1.z * sc; b[i][7] = x1.w * sc;
        }
#pragma unroll
        for (int i = 1; i < 4; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) b[i][e] += b[i - 1][e];
        float m2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float tot = b[3][e];
            float incl = tot;
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off, 16);
                if (prb >= off) incl += y;
            }
            const float ex = incl - tot;
#pragma unroll
            for (int i = 0; i < 4; ++i) b[i][e] += ex;
            m2[e] = __shfl_sync(0xffffffffu, b[3][e], 7, 16);        // row 31
            const float bc = __shfl_sync(0xffffffffu, b[3][e], 15, 16);  // row 63
            const float b0 = __shfl_sync(0xffffffffu, b[0][e], 0, 16);   // row 0
            if (prb == 0) {
                const int c = pc0 + e;
                eM[c] = tc::ex2(m2[e]);
                eC[c] = tc::ex2(bc - m2[e]);
                gC[c] = tc::ex2(bc);
                if (b0 - m2[e] > RANGE_LIMIT2 || m2[e] - bc > RANGE_LIMIT2) record_status(KDA_ERR_RANGE);
            }
        }
        if (tid < C) bet[tid] = tid < n ? p.beta[(int64_t)(sq.tok0 + ci * C + tid) * H + h] : 0.f;
        // ---- C. scaled bf16 operands Qh = q 2^(b-m), Ka = k 2^(b-m), Kb = k 2^(m-b)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * prb + i;
            const uint32_t so = pkb * 8192 + tc::sw128(r, pcc);
            const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + STG_Q + so);
            const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + STG_K + so);
            const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
            const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
            uint32_t oq[4], oa[4], ob[4];
            const bool live = r < n;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 qf = unpack_bf16(qw[e]), kf = unpack_bf16(kw[e]);
                const float d0 = b[i][2 * e] - m2[2 * e], d1 = b[i][2 * e + 1] - m2[2 * e + 1];
                const float e10 = tc::ex2(d0), e11 = tc::ex2(d1);
                const float e20 = tc::ex2(-d0), e21 = tc::ex2(-d1);
                oq[e] = live ? pack_bf16(qf.x * e10, qf.y * e11) : 0u;
                oa[e] = live ? pack_bf16(kf.x * e10, kf.y * e11) : 0u;
                ob[e] = live ? pack_bf16(kf.x * e20, kf.y * e21) : 0u;
            }
            *reinterpret_cast<uint4 *>(sm + OP_AK + pkb * 16384 + tc::sw128(r, pcc)) =
                make_uint4(oq[0], oq[1], oq[2], oq[3]);
            *reinterpret_cast<uint4 *>(sm + OP_AK + pkb * 16384 + tc::sw128(64 + r, pcc)) =
                make_uint4(oa[0], oa[1], oa[2], oa[3]);
            *reinterpret_cast<uint4 *>(sm + OP_KB + pkb * 8192 + tc::sw128(r, pcc)) =
                make_uint4(ob[0], ob[1], ob[2], ob[3]);
        }
        __syncthreads();   // eM visible
        // ---- Sm = Diag(e^m) S_0 (bf16 operand of the chain products) ---------
        {
            const float em = eM[c_own];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4 *>(sm + OP_SM + tc::sw128(c_own, 4 * wh + q4)) = pack8(S + 8 * q4, em);
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
            float a[32];
            tc::tmem_ld32(tbase + tlane + COL_A + 32 * wh, a);
            tc::tmem_ld_wait();
            if (wq < 2) {
                const int r = 32 * wq + lane;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int jj = 32 * wh + 8 * q4 + 2 * e;
                        w[e] = pack_bf16(jj <= r ? a[8 * q4 + 2 * e] : 0.f, jj + 1 <= r ? a[8 * q4 + 2 * e + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(sm + OP_AQK + tc::sw128(r, 4 * wh + q4)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
                const int r = 32 * (wq - 2) + lane;
                const float br = bet[r];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int jj = 32 * wh + e;
                    Ls[r * 65 + jj] = jj < r ? br * a[e] : 0.f;
                }
            }
        }
        __syncthreads();
        // ---- F. X = (I + L)^{-1}: 16x16 diagonal blocks by forward substitution
        // (fp32), off-diagonal blocks X[R][Cb] = -X[R][R] sum_J L[R][J] X[J][Cb]
        // by distance R - Cb on tf32 mma.sync; T = X Diag(beta) -> bf16 -------
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
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 16; ++r) Ls[(base + r) * 65 + base + c] = x[r];
        }
        __syncthreads();
#pragma unroll 1
        for (int dist = 1; dist < 4; ++dist) {
            if (warp < 4 - dist) {
                const int cb = warp, R = cb + dist;
                float pacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int J = cb; J < R; ++J) {
                    const float *xj = J == cb ? Ls + (16 * J) * 65 + 16 * cb : Xo + xslot(J - cb, cb) * 256;
                    tc::mma16x16(pacc, Ls + (16 * R) * 65 + 16 * J, 65, xj, J == cb ? 65 : 16);
                }
                float *yw = Yw + warp * 256;
                tc::store16x16(yw, 16, pacc, 1.f);
                __syncwarp();
                float pr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                tc::mma16x16(pr, Ls + (16 * R) * 65 + 16 * R, 65, yw, 16);
                tc::store16x16(Xo + xslot(dist, cb) * 256, 16, pr, -1.f);
            }
            __syncthreads();
        }
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
                    if (R == Cb) x = Ls[r * 65 + c];
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
            const int r = 16 * wq + (lane & 15);
            float a[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tc::tmem_ld32(tbase + tlane + COL_WK + 64 * wh + 32 * q, a);
                tc::tmem_ld_wait();
                if (lane < 16) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + OP_WK + wh * 8192 + tc::sw128(r, 4 * q + q4)) =
                            pack8(a + 8 * q4, 1.f);
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
            const int r = 16 * wq + (lane & 15);
            float a[32];
            tc::tmem_ld32(tbase + tlane + COL_W + 32 * wh, a);
            tc::tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    *reinterpret_cast<uint4 *>(sm + OP_W + tc::sw128(r, 4 * wh + q4)) = pack8(a + 8 * q4, 1.f);
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
            float a[32];
            const int r = 16 * wq + (lane & 15);
            tc::tmem_ld32(tbase + tlane + COL_O + 32 * wh, a);
            tc::tmem_ld_wait();
            if (lane < 16 && r < n) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) +
                                                       ((int64_t)(sq.tok0 + ci * C + r) * H + h) * D + j0 + 32 * wh);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) dst[q4] = pack8(a + 8 * q4, p.scale);
            }
            const float g_c = gC[c_own], e_c = eC[c_own];
            tc::tmem_ld32(tbase + tlane + COL_S + 32 * wh, a);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) S[e] = fmaf(g_c, S[e], e_c * a[e]);
            if (p.snap_interval > 0 && (sq.start_pos + (int64_t)ci * C + n) % p.snap_interval == 0) {
                float *dst = p.snapshots + ((snap_row * H + h) * D + c_own) * (int64_t)D + j0 + 32 * wh;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
                ++snap_row;
            }
        }
        tc::fence_before_sync();
        __syncthreads();
    }

    if (ok && p.state_out) {
        float *dst = p.state_out + (((int64_t)s * H + h) * D + c_own) * (int64_t)D + j0 + 32 * wh;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
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
