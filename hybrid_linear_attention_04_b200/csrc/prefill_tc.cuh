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
//   tcgen05  (same round as A) R' = Ka Sm, O = Qh Sm  (M=64; Sm = Diag(e^m) S_0)
//   CUDA     R = V - R' (bf16), concurrently with the solve
//   tcgen05  W = T R                                 (M=64)
//            O += A_qk W, D = Kb^T W                 (M=64 / M=128)
//   CUDA     o = scale O (bf16 store); S_C = Diag(Gamma_C) S_0 + Diag(e^(b_C-m)) D
//   cores    with the fp32 master state held in registers (thread = d_k row).
// Identities used: Q.Gamma = Qh.e^m and K.Gamma = Ka.e^m, so (Q.Gamma) S_0 =
// Qh Sm and (K.Gamma) S_0 = Ka Sm; K.exp(b_C-b) = Kb.e^(b_C-m) row-wise; and
// W = T (V - (K.Gamma) S_0) = T R.
// A chunk whose per-channel decay from its middle exceeds 80 nats in either
// direction is reported through the status word (KDA_ERR_RANGE).
#pragma once
#include <cudaTypedefs.h>

#include "prefill_common.cuh"
#include "tc_util.cuh"

namespace kda {

#ifdef KDA_PHASE_TIMING
__device__ long long g_phase_clock[64][16];
#define KDA_MARK(ci, k) \
    do { if (threadIdx.x == 0 && blockIdx.x == 0 && (ci) < 64) g_phase_clock[(ci)][(k)] = clock64(); } while (0)
#else
#define KDA_MARK(ci, k) do { } while (0)
#endif

struct TcParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_g;
    PrefillParams p;
};

namespace tcp {
constexpr int C = 64, D = 128, DVS = 64, NT = 256;
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t STG_Q = 0;          // q  [64 tok x 128 ch] bf16: 2 slabs of 64 rows
constexpr uint32_t STG_K = 16384;      // k  same
constexpr uint32_t STG_V = 32768;      // v  slice, 2 buffers of 1 slab [64 tok x 64]
constexpr uint32_t OP_AK = 49152;      // [Qh; Ka]: 2 slabs of 128 rows (channels 0-63, 64-127)
constexpr uint32_t OP_KB = 81920;      // [Kb; Sm^T]: 2 slabs (channels 0-63, 64-127) of 128 rows:
                                       // rows 0-63 Kb (tokens), rows 64-127 Sm^T (d_v columns)
constexpr uint32_t OP_T = 114688;      // T  [64 x 64]
constexpr uint32_t OP_AQK = 122880;    // A_qk masked [64 x 64]
constexpr uint32_t OP_RW = 131072;     // R = V - Ka Sm, then W [64 tok x 64 dv]
constexpr uint32_t STG_G = 139264;     // g, fp32 [64][128]
constexpr uint32_t SOLVE = 172032;     // fp32 [64][65]: L off the diagonal blocks, X on them
constexpr uint32_t XO = SOLVE + 64 * 65 * 4;   // 6 off-diagonal X blocks + 3 scratch blocks (16x16 fp32)
constexpr uint32_t TOT = XO + 9 * 1024;        // per-warp row-block totals of b [8][128]
constexpr uint32_t VEC = TOT + 8 * 128 * 4;    // eM, eC, gC [128] + beta [64]
constexpr uint32_t BARS = VEC + (3 * 128 + 64) * 4;
constexpr uint32_t SMEM_USED = BARS + 48;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
// TMEM columns
// round 1 writes [A_qk | O ; A_kk | R'] into columns 0-127 (rows 0-63 | 64-127);
// W = T R lands in COL_W (M=64), D = Kb^T W in COL_S
constexpr uint32_t COL_A = 0, COL_O = 64, COL_W = 128, COL_S = 192, TMEM_COLS = 256;
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
    float *Xo = reinterpret_cast<float *>(sm + XO);     // 6 blocks 16x16
    float *Yw = Xo + 6 * 256;                             // 3 per-warp 16x16 blocks
    float *Tot = reinterpret_cast<float *>(sm + TOT);
    float *eM = reinterpret_cast<float *>(sm + VEC);
    float *eC = eM + 128, *gC = eM + 256, *bet = eM + 384;
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(sm + BARS);   // [2]
    uint64_t *mma_bar = tma_bar + 2;       // rounds 2 and 3
    uint64_t *bar_a = tma_bar + 3;         // round 1: [Qh; Ka] [Kb; Sm^T]^T
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 5);

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
        tc::bar_init(bar_a, 1);
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
    // smem matrix descriptors (start-address field advanced by 16-byte units)
    const uint64_t dAK = tc::desc_k(sbase + OP_AK, 0), dKB = tc::desc_k(sbase + OP_KB, 0);
    const uint64_t dT = tc::desc_k(sbase + OP_T, 0), dAQK = tc::desc_k(sbase + OP_AQK, 0);
    const uint64_t dRW = tc::desc_mn(sbase + OP_RW, 0, 8192);
    const uint64_t dKBmn = tc::desc_mn(sbase + OP_KB, 0, 16384);
    // T's blocks above the diagonal are always zero: clear the whole T tile once
    // (the diagonal and lower blocks are rewritten every chunk)
    for (int e = tid; e < 64 * 8; e += NT)
        *reinterpret_cast<uint4 *>(sm + OP_T + 16 * e) = make_uint4(0u, 0u, 0u, 0u);
    // prep map: warp w owns rows 8w..8w+7, lane l owns channels 4l..4l+3
    const int pkb = lane >> 4, pchk = (lane & 15) >> 1, phf = (lane & 1) * 8;

    for (int ci = 0; ci < n_chunks; ++ci) {
        const int n = min(C, sq.len - ci * C);
        KDA_MARK(ci, 0);
        // ---- A. this chunk's operands have landed --------------------------
        ok = tc::bar_wait(&tma_bar[ci & 1], (ci >> 1) & 1);
        if (!__syncthreads_and(ok)) { ok = false; break; }
        landed = ci + 1;
        KDA_MARK(ci, 1);
        // ---- B. b = cumsum(g) over the chunk, in log2 units -------------------
        float b[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 8 * warp + i;
            const float4 x = *reinterpret_cast<const float4 *>(Gs + r * D + 4 * lane);
            const float sc = r < n ? LOG2E : 0.f;
            b[i][0] = x.x * sc; b[i][1] = x.y * sc; b[i][2] = x.z * sc; b[i][3] = x.w * sc;
        }
#pragma unroll
        for (int i = 1; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) b[i][e] += b[i - 1][e];
        *reinterpret_cast<float4 *>(Tot + warp * 128 + 4 * lane) = make_float4(b[7][0], b[7][1], b[7][2], b[7][3]);
        if (tid < C) bet[tid] = tid < n ? p.beta[(int64_t)(sq.tok0 + ci * C + tid) * H + h] : 0.f;
        __syncthreads();
        float m2[4] = {0.f, 0.f, 0.f, 0.f};
        {
            float off[4] = {0.f, 0.f, 0.f, 0.f}, bc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w2 = 0; w2 < 8; ++w2) {
                const float4 t = *reinterpret_cast<const float4 *>(Tot + w2 * 128 + 4 * lane);
                const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (w2 < warp) off[e] += tv[e];
                    if (w2 < 4) m2[e] += tv[e];     // b at row 31
                    bc[e] += tv[e];                 // b at row 63
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) b[i][e] += off[e];
            if (warp == 0) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * lane + e;
                    eM[c] = tc::ex2(m2[e]);
                    eC[c] = tc::ex2(bc[e] - m2[e]);
                    gC[c] = tc::ex2(bc[e]);
                    // b <= 0, so row 0 is at most -m above the reference
                    if (-m2[e] > RANGE_LIMIT2 || m2[e] - bc[e] > RANGE_LIMIT2) record_status(KDA_ERR_RANGE);
                }
            }
        }
        // ---- C. scaled bf16 operands Qh = q 2^(b-m), Ka = k 2^(b-m), Kb = k 2^(m-b)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 8 * warp + i;
            const uint32_t so = pkb * 8192 + tc::sw128(r, pchk) + phf;
            const uint2 qv = *reinterpret_cast<const uint2 *>(sm + STG_Q + so);
            const uint2 kv = *reinterpret_cast<const uint2 *>(sm + STG_K + so);
            const float2 q01 = unpack_bf16(qv.x), q23 = unpack_bf16(qv.y);
            const float2 k01 = unpack_bf16(kv.x), k23 = unpack_bf16(kv.y);
            float e1[4], e2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float d = b[i][e] - m2[e];
                e1[e] = tc::ex2(d);
                e2[e] = tc::ex2(-d);
            }
            const bool live = r < n;
            const uint2 oq = live ? make_uint2(pack_bf16(q01.x * e1[0], q01.y * e1[1]), pack_bf16(q23.x * e1[2], q23.y * e1[3]))
                                  : make_uint2(0u, 0u);
            const uint2 oa = live ? make_uint2(pack_bf16(k01.x * e1[0], k01.y * e1[1]), pack_bf16(k23.x * e1[2], k23.y * e1[3]))
                                  : make_uint2(0u, 0u);
            const uint2 ob = live ? make_uint2(pack_bf16(k01.x * e2[0], k01.y * e2[1]), pack_bf16(k23.x * e2[2], k23.y * e2[3]))
                                  : make_uint2(0u, 0u);
            *reinterpret_cast<uint2 *>(sm + OP_AK + pkb * 16384 + tc::sw128(r, pchk) + phf) = oq;
            *reinterpret_cast<uint2 *>(sm + OP_AK + pkb * 16384 + tc::sw128(64 + r, pchk) + phf) = oa;
            *reinterpret_cast<uint2 *>(sm + OP_KB + pkb * 16384 + tc::sw128(r, pchk) + phf) = ob;
        }
        __syncthreads();   // eM visible
        KDA_MARK(ci, 2);
        // ---- Sm^T = (Diag(e^m) S_0)^T (bf16, K-major B operand of round 1) ----
        {
            const float em = eM[c_own];
            __nv_bfloat16 *st = reinterpret_cast<__nv_bfloat16 *>(sm + OP_KB + (c_own >> 6) * 16384);
            const int cch = (c_own & 63) >> 3, cin = c_own & 7;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int row = 64 + 32 * wh + j;
                st[(tc::sw128(row, cch) >> 1) + cin] = __float2bfloat16_rn(S[j] * em);
            }
        }
        tc::fence_async_smem();
        __syncthreads();
        KDA_MARK(ci, 3);
        // ---- D. round 1: A = [Qh; Ka] Kb^T; R' = Ka Sm; O = Qh Sm; then the next
        // chunk's loads (descriptors advance by 16-byte units in their low bits)
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_a = tc::idesc_bf16(128, 128, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_A, dAK + (k >> 2) * 1024 + (k & 3) * 2, dKB + (k >> 2) * 1024 + (k & 3) * 2,
                             id_a, k > 0);
            tc::mma_commit(bar_a);
            if (ci + 1 < n_chunks) {
                issue_loads(ci + 1);
                issued = ci + 2;
            }
        }
        // a timed-out wait is acted on at the block-wide vote after phase E
        ok = tc::bar_wait(bar_a, (uint32_t)(ci & 1));
        tc::fence_after_sync();
        KDA_MARK(ci, 4);
        if (warp < 4) {
            // ---- E1. A_qk (masked bf16 operand), L = Diag(beta) A_kk, then the
            // solve X = (I + L)^{-1} and T = X Diag(beta) (warps 0-3) ----------
            {
                const int r = 32 * (warp & 1) + lane;
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
            tc::named_sync(1, 128);
            KDA_MARK(ci, 10);
            // 16x16 diagonal blocks by forward substitution, one column per thread
            if (tid < 64) {
                const int blk = tid >> 4, c = tid & 15, base = 16 * blk;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float a0 = r == c ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                    const float *lr = Ls + (base + r) * 65 + base;
#pragma unroll
                    for (int i = 0; i < r; ++i) {
                        const float t = lr[i] * x[i];
                        if ((i & 3) == 0) a0 -= t;
                        else if ((i & 3) == 1) a1 -= t;
                        else if ((i & 3) == 2) a2 -= t;
                        else a3 -= t;
                    }
                    x[r] = (a0 + a1) + (a2 + a3);
                }
                __syncwarp();
                const float bc = bet[base + c];
                __nv_bfloat16 *tt = reinterpret_cast<__nv_bfloat16 *>(sm + OP_T);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    Ls[(base + r) * 65 + base + c] = x[r];
                    const int rr = base + r, cc = base + c;
                    tt[(tc::sw128(rr, cc >> 3) >> 1) + (cc & 7)] = __float2bfloat16_rn(x[r] * bc);
                }
            }
            tc::named_sync(1, 128);
            KDA_MARK(ci, 11);
            // off-diagonal blocks by distance: X[R][Cb] = -X[R][R] sum_J L[R][J] X[J][Cb]
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
                    // T[16R + row][16cb + col] = -pr * beta[col] (bf16 pairs)
                    const int g = lane >> 2, t = lane & 3;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int col = 16 * cb + 8 * nt + 2 * t;
                        const float b0 = -bet[col], b1 = -bet[col + 1];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int row = 16 * R + g + 8 * hh;
                            *reinterpret_cast<uint32_t *>(sm + OP_T + tc::sw128(row, col >> 3) + 2 * (col & 7)) =
                                pack_bf16(pr[nt][2 * hh] * b0, pr[nt][2 * hh + 1] * b1);
                        }
                    }
                }
                tc::named_sync(1, 128);
                KDA_MARK(ci, 11 + dist);
            }
        } else if (warp >= 6) {
            // ---- E2. R = V - Ka Sm (bf16 operand): R' is rows 64-127 (TMEM lanes
            // 64-127, sub-partitions 2 and 3) of columns COL_O..COL_O+63; warps 6
            // and 7 own those sub-partitions ---------------------------------------
            const int r = 32 * (wq - 2) + lane;
            const uint8_t *vs = sm + STG_V + (ci & 1) * 8192;
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + COL_O + 32 * half, a);
                tc::tmem_ld_wait();
                {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const uint32_t off = tc::sw128(r, 4 * half + q4);
                        const uint4 vv = *reinterpret_cast<const uint4 *>(vs + off);
                        const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 vf = unpack_bf16(vw[e]);
                            w[e] = pack_bf16(vf.x - a[8 * q4 + 2 * e], vf.y - a[8 * q4 + 2 * e + 1]);
                        }
                        *reinterpret_cast<uint4 *>(sm + OP_RW + off) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        if (!__syncthreads_and(ok)) { ok = false; break; }
        KDA_MARK(ci, 5);
        // ---- F. round 2: W = T R ----------------------------------------------------
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_w = tc::idesc_bf16(64, 64, false, true);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + COL_W, dT + 2 * k, dRW + 128 * k, id_w, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
        KDA_MARK(ci, 6);
        // ---- G. W -> bf16 operand (replaces R, which round 2 consumed) ----------------
        {
            const int r = 16 * wq + (lane & 15);
            float a[32];
            tc::tmem_ld32(tbase + tlane + COL_W + 32 * wh, a);
            tc::tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    *reinterpret_cast<uint4 *>(sm + OP_RW + tc::sw128(r, 4 * wh + q4)) = pack8(a + 8 * q4, 1.f);
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        KDA_MARK(ci, 7);
        // ---- H. round 3: O += A_qk W ; D = Kb^T W ---------------------------------------
        if (tid == 0) {
            tc::fence_after_sync();
            // O += A_qk W as an M=128 MMA (O1 came from the M=128 round 1): its A rows
            // 64-127 are the W tile that follows A_qk in shared memory, and land in
            // TMEM lanes 64-127 of COL_O, which are not read afterwards
            constexpr uint32_t id_o = tc::idesc_bf16(128, 64, false, true);
            constexpr uint32_t id_s = tc::idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + COL_O, dAQK + 2 * k, dRW + 128 * k, id_o, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + COL_S, dKBmn + 128 * k, dRW + 128 * k, id_s, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
        KDA_MARK(ci, 8);
        // ---- I. outputs, state update, snapshot -------------------------------------------
        {
            float a[32];
            const int r = 32 * wq + lane;          // O row in the M=128 layout (warps 0,1,4,5)
            if (wq < 2) {
                tc::tmem_ld32(tbase + tlane + COL_O + 32 * wh, a);
                tc::tmem_ld_wait();
            }
            if (wq < 2 && r < n) {
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
        KDA_MARK(ci, 9);
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
