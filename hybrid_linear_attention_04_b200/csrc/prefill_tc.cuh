// KDA chunked prefill on the tcgen05 tensor cores (d_k = d_v = 128, chunk 64,
// bf16 q/k/v/o, fp32 state). The chunk form is the one in prefill_common.cuh.
//
// One CTA (256 threads) walks the chunks of one (sequence, head, 64-column
// d_v slice); d_v columns are independent, so two CTAs per head run in
// parallel. Per chunk:
//   TMA      q, k (bf16, 128B-swizzled slabs), g (fp32) and the v slice; the
//            next chunk's loads are issued as soon as this chunk's are consumed.
//   CUDA     b = cumsum(g); a per-channel reference m = b at the chunk middle;
//   cores    Qh = q.exp(b-m), Ka = k.exp(b-m), Kb = k.exp(m-b) (bf16 operands),
//            so that Qh Kb^T = A_qk and Ka Kb^T = A_kk with every exponent
//            inside the chunk bounded by half the chunk's decay range.
//   tcgen05  [Qh; Ka] Kb^T -> TMEM (M=128: A_qk rows 0-63, A_kk rows 64-127), each
//            scaled operand split into bf16 high and low parts (three products, so A
//            is fp32-accurate)
//   tcgen05  (same MMAs as A) R' = Ka Sm, O = Qh Sm  (Sm = Diag(e^m) S_0, stored
//            transposed under Kb so one N=128 round yields all four blocks)
//   CUDA     L = Diag(beta) A_kk; inverses of its 16x16 diagonal blocks (fp32);
//   cores    R = V - R' (fp32); then W = (I + L)^{-1} Diag(beta) R by block
//            forward substitution on bf16 mma.sync, 8 d_v columns per warp
//   tcgen05  O += A_qk W, D = Kb^T W                 (M=128)
//   CUDA     o = scale O (bf16 store); S_C = Diag(Gamma_C) S_0 + Diag(e^(b_C-m)) D
//   cores    with the fp32 master state held in registers (thread = d_k row).
// Identities used: Q.Gamma = Qh.e^m and K.Gamma = Ka.e^m, so (Q.Gamma) S_0 =
// Qh Sm and (K.Gamma) S_0 = Ka Sm; K.exp(b_C-b) = Kb.e^(b_C-m) row-wise; and
// W = (I + Diag(beta) A_kk)^{-1} Diag(beta) (V - (K.Gamma) S_0).
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
constexpr uint32_t STG_Q = 0;          // q  [64 tok x 128 ch] bf16: 2 slabs of 64 rows
constexpr uint32_t STG_K = 16384;      // k  same
constexpr uint32_t STG_V = 32768;      // v  slice, 2 buffers of 1 slab [64 tok x 64]
constexpr uint32_t OP_AK = 49152;      // [Qh; Ka]: 2 slabs of 128 rows (channels 0-63, 64-127)
constexpr uint32_t OP_KB = 81920;      // [Kb; Sm^T]: 2 slabs (channels 0-63, 64-127) of 128 rows:
                                       // rows 0-63 Kb (tokens), rows 64-127 Sm^T (d_v columns)
constexpr uint32_t OP_AQK = 114688;    // A_qk masked [64 x 64] (followed by OP_W: see round 3)
constexpr uint32_t OP_W = 122880;      // W [64 tok x 64 dv] bf16
constexpr uint32_t STG_G = 131072;     // g, fp32 [64][128]
constexpr uint32_t SOLVE = 163840;     // fp32 [64][65]: L = Diag(beta) A_kk, inverse on diagonal blocks
constexpr uint32_t RF = SOLVE + 64 * 65 * 4;   // R = V - Ka Sm, fp32 [64][68]
constexpr uint32_t LB = RF + 64 * 68 * 4;      // bf16 [64][72]: L off the diagonal blocks, X on them
constexpr uint32_t WSC = LB + 64 * 72 * 2;     // per-warp Y / W columns, bf16 [8 warps][8][72]
constexpr uint32_t TOT = WSC + 8 * 8 * 72 * 2; // per-warp row-block totals of b [8][128]
// Low bf16 parts of the scaled operands (x - bf16(x), rounded to bf16), live from the
// operand pass until round 1a completes, over the solve scratch (free in that window)
constexpr uint32_t LO_AK0 = SOLVE;             // [Qh_lo; Ka_lo] channels 0-63, 128 rows
constexpr uint32_t LO_AK1 = SOLVE + 16384;     // [Qh_lo; Ka_lo] channels 64-127, 128 rows
constexpr uint32_t LO_KB = SOLVE + 32768;      // Kb_lo: 2 slabs x 64 rows
static_assert(LO_KB + 16384 <= TOT && SOLVE % 1024 == 0, "low parts overlap live data");
constexpr uint32_t VEC = TOT + 8 * 128 * 4;    // eM, eC, gC [128] + beta [64]
constexpr uint32_t BARS = VEC + (3 * 128 + 64) * 4;
constexpr uint32_t SMEM_USED = BARS + 48;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
// TMEM columns: round 1 writes [A_qk | O ; A_kk | R'] into columns 0-127 (rows
// 0-63 | 64-127); D = Kb^T W lands in COL_S
constexpr uint32_t COL_A = 0, COL_O = 64, COL_S = 128, TMEM_COLS = 256;
constexpr uint32_t CHUNK_TX = 16384 + 16384 + 32768 + 8192;   // bytes per chunk of loads
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RANGE_LIMIT2 = 80.f * LOG2E;    // 80 nats, in log2 units
// raw q, k and b of the channels beyond that range ([kMaxFast][64] fp32 each) in TOT (read
// only by the cumsum before them; a barrier separates the two when the staging is used)
constexpr int kMaxFast = 4;
constexpr uint32_t FQ = TOT, FK = TOT + kMaxFast * 256, FB = TOT + 2 * kMaxFast * 256;
static_assert(3 * kMaxFast * 256 <= 8 * 128 * 4, "fast-channel staging");
}  // namespace tcp

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}
// a, b -> bf16 pairs hi and lo with hi + lo = (a, b) to about 2^-17 relative
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    // the residuals are exact in fp32; they are truncated to bf16 (their upper halves,
    // one byte permute instead of a second conversion): error below 2^-17 of a, b
    const float ra = a - __uint_as_float(hi << 16), rb = b - __uint_as_float(hi & 0xffff0000u);
    lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
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
    float *Rf = reinterpret_cast<float *>(sm + RF);
    __nv_bfloat16 *Lb = reinterpret_cast<__nv_bfloat16 *>(sm + LB);
    __nv_bfloat16 *Wsc = reinterpret_cast<__nv_bfloat16 *>(sm + WSC);
    float *Tot = reinterpret_cast<float *>(sm + TOT);
    float *eM = reinterpret_cast<float *>(sm + VEC);
    float *eC = eM + 128, *gC = eM + 256, *bet = eM + 384;
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(sm + BARS);   // [2]
    uint64_t *mma_bar = tma_bar + 2;       // rounds 2 and 3
    uint64_t *bar_a = tma_bar + 3;         // round 1a: [Qh; Ka] Kb^T
    uint64_t *bar_b = tma_bar + 4;         // round 1b: [Qh; Ka] Sm
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
        tc::bar_init(bar_b, 1);
        tc::bar_init_fence();
        if (n_chunks > 0) {
            tc::tma_prefetch_desc(&P.tm_q);
            tc::tma_prefetch_desc(&P.tm_k);
            tc::tma_prefetch_desc(&P.tm_v);
            tc::tma_prefetch_desc(&P.tm_g);
        }
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
    const uint64_t dAQK = tc::desc_k(sbase + OP_AQK, 0);
    const uint64_t dW = tc::desc_mn(sbase + OP_W, 0, 8192);
    const uint64_t dKBmn = tc::desc_mn(sbase + OP_KB, 0, 16384);
    float bnext = (tid < C && tid < sq.len) ? p.beta[(int64_t)(sq.tok0 + tid) * H + h] : 0.f;
    // prep map: warp w owns rows 8w..8w+7, lane l owns channels 4l..4l+3
    const int pkb = lane >> 4, pchk = (lane & 15) >> 1, phf = (lane & 1) * 8;

    for (int ci = 0; ci < n_chunks; ++ci) {
        const int n = min(C, sq.len - ci * C);
        // ---- A. this chunk's operands have landed --------------------------
        ok = tc::bar_wait(&tma_bar[ci & 1], (ci >> 1) & 1);
        if (!__syncthreads_and(ok)) { ok = false; break; }
        landed = ci + 1;
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
        // beta of this chunk was fetched one chunk ahead (a strided global load)
        if (tid < C) {
            bet[tid] = bnext;
            const int nn = min(C, sq.len - (ci + 1) * C);
            bnext = (ci + 1 < n_chunks && tid < nn) ? p.beta[(int64_t)(sq.tok0 + (ci + 1) * C + tid) * H + h] : 0.f;
        }
        __syncthreads();
        float m2[4] = {0.f, 0.f, 0.f, 0.f}, r1[4], r2[4];
        int n_fast;                       // channels on the second reference (block-uniform)
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
            // references per channel: the chunk middle, or (beyond the range) 0 and b_C
            // (b <= 0, so row 0 is at most -m above the middle)
            bool fast[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                fast[e] = -m2[e] > RANGE_LIMIT2 || m2[e] - bc[e] > RANGE_LIMIT2;
                r1[e] = fast[e] ? 0.f : m2[e];
                r2[e] = fast[e] ? bc[e] : m2[e];
            }
            n_fast = fast_channels(fast).n;
            if (warp == 0) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * lane + e;
                    eM[c] = tc::ex2(r1[e]);
                    eC[c] = tc::ex2(bc[e] - r2[e]);
                    gC[c] = tc::ex2(bc[e]);
                }
                if (lane == 0 && n_fast > kMaxFast) record_status(KDA_ERR_RANGE);
            }
        }
        if (n_fast > 0) __syncthreads();   // TOT (the cumsum totals) becomes the staging below
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
                e1[e] = tc::ex2(b[i][e] - r1[e]);
                e2[e] = tc::ex2(r2[e] - b[i][e]);
            }
            if (n_fast > 0) {
                // raw values of the channels on the second reference (r1 != r2), for fast_correct
                const float qr[4] = {q01.x, q01.y, q23.x, q23.y}, kr[4] = {k01.x, k01.y, k23.x, k23.y};
                bool fast[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) fast[e] = r1[e] != r2[e];
                const FastChannels fch = fast_channels(fast);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int f = fast[e] ? fast_index(fch, lane, e) : kMaxFast;
                    if (f < kMaxFast) {
                        const bool live = r < n;
                        reinterpret_cast<float *>(sm + FQ)[f * 64 + r] = live ? qr[e] : 0.f;
                        reinterpret_cast<float *>(sm + FK)[f * 64 + r] = live ? kr[e] : 0.f;
                        reinterpret_cast<float *>(sm + FB)[f * 64 + r] = b[i][e];   // b_(n-1) past n
                    }
                }
            }
            // high parts (the MMA operands) and low parts (for the fp32-accurate A)
            uint2 oq = make_uint2(0u, 0u), lq = oq, oa = oq, la = oq, ob = oq, lb = oq;
            if (r < n) {
                split_bf16(q01.x * e1[0], q01.y * e1[1], oq.x, lq.x);
                split_bf16(q23.x * e1[2], q23.y * e1[3], oq.y, lq.y);
                split_bf16(k01.x * e1[0], k01.y * e1[1], oa.x, la.x);
                split_bf16(k23.x * e1[2], k23.y * e1[3], oa.y, la.y);
                split_bf16(k01.x * e2[0], k01.y * e2[1], ob.x, lb.x);
                split_bf16(k23.x * e2[2], k23.y * e2[3], ob.y, lb.y);
            }
            const uint32_t sr = tc::sw128(r, pchk) + phf, sr64 = tc::sw128(64 + r, pchk) + phf;
            const uint32_t lo_ak = pkb ? LO_AK1 : LO_AK0;
            *reinterpret_cast<uint2 *>(sm + OP_AK + pkb * 16384 + sr) = oq;
            *reinterpret_cast<uint2 *>(sm + OP_AK + pkb * 16384 + sr64) = oa;
            *reinterpret_cast<uint2 *>(sm + OP_KB + pkb * 16384 + sr) = ob;
            *reinterpret_cast<uint2 *>(sm + lo_ak + sr) = lq;
            *reinterpret_cast<uint2 *>(sm + lo_ak + sr64) = la;
            *reinterpret_cast<uint2 *>(sm + LO_KB + pkb * 8192 + sr) = lb;
        }
        tc::fence_async_smem();
        __syncthreads();   // operands and eM visible
        // ---- D1. round 1a: A = [Qh; Ka] Kb^T (independent of the state), issued
        // before Sm^T is written so that the L extraction can start earlier
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_a = tc::idesc_bf16(128, 64, false, false);
            // hi hi' + lo hi' + hi lo': A to fp32 accuracy (the lo lo' term is below it)
            const uint64_t dAKlo = tc::desc_k(sbase + LO_AK0, 0), dKBlo = tc::desc_k(sbase + LO_KB, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_A, dAK + (k >> 2) * 1024 + (k & 3) * 2, dKB + (k >> 2) * 1024 + (k & 3) * 2,
                             id_a, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_A, dAKlo + (k >> 2) * 1024 + (k & 3) * 2,
                             dKB + (k >> 2) * 1024 + (k & 3) * 2, id_a, 1);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_A, dAK + (k >> 2) * 1024 + (k & 3) * 2,
                             dKBlo + (k >> 2) * 512 + (k & 3) * 2, id_a, 1);
            tc::mma_commit(bar_a);
        }
        // ---- Sm^T = (Diag(e^m) S_0)^T (bf16, K-major B operand of round 1b) ----
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
        // ---- D2. round 1b: [R'; O] = [Qh; Ka] Sm; then the next chunk's loads ----
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_b = tc::idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + COL_O, dAK + (k >> 2) * 1024 + (k & 3) * 2,
                             dKB + (k >> 2) * 1024 + 512 + (k & 3) * 2, id_b, k > 0);
            tc::mma_commit(bar_b);
            if (ci + 1 < n_chunks) {
                issue_loads(ci + 1);
                issued = ci + 2;
            }
        }
        // warps 0-3 need A (round 1a), warps 6-7 need R' (round 1b); a timed-out
        // wait is acted on at the block-wide vote after phase E
        ok = tc::bar_wait(warp < 4 ? bar_a : bar_b, (uint32_t)(ci & 1));
        tc::fence_after_sync();
        // the pairwise part of the channels beyond the range, into A (each warp its own rows)
        if (n_fast > 0 && warp < 4)
            fast_correct<kMaxFast>(tbase + tlane + COL_A, 32 * warp + lane, n_fast,
                                   reinterpret_cast<const float *>(sm + FQ),
                                   reinterpret_cast<const float *>(sm + FK),
                                   reinterpret_cast<const float *>(sm + FB));
        // ---- E. warps 0,1: A_qk (masked bf16 operand). Warps 2,3: L = Diag(beta)
        // A_kk (fp32), then the inverses X of its four 16x16 diagonal blocks by
        // forward substitution (each warp owns two blocks: no block-wide sync).
        // Warps 6,7: R = V - Ka Sm (fp32) from TMEM lanes 64-127 (their sub-partitions).
        if (warp < 2) {
            const int r = 32 * warp + lane;
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + COL_A + 32 * half, a);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int jj = 32 * half + 8 * q4 + 2 * e;
                        w[e] = pack_bf16(jj <= r ? a[8 * q4 + 2 * e] : 0.f, jj + 1 <= r ? a[8 * q4 + 2 * e + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(sm + OP_AQK + tc::sw128(r, 4 * half + q4)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        } else if (warp < 4) {
            const int r = 32 * (warp - 2) + lane;
            const float br = bet[r];
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + COL_A + 32 * half, a);
                tc::tmem_ld_wait();
                // bf16 L for the forward substitution (16-byte stores: conflict-free
                // with the 144-byte row pitch); fp32 L only on the diagonal block,
                // which the inversion below reads
                const int dblk = r & ~15;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float l[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int jj = 32 * half + 8 * q4 + e;
                        l[e] = jj < r ? br * a[8 * q4 + e] : 0.f;
                        if (jj >= dblk && jj < dblk + 16) Ls[r * 65 + jj] = l[e];
                    }
                    *reinterpret_cast<uint4 *>(Lb + r * 72 + 32 * half + 8 * q4) = pack8(l, 1.f);
                }
            }
            __syncwarp();
            // diagonal block 2*(warp-2) + lane/16, column lane%16
            const int base = 16 * (2 * (warp - 2) + (lane >> 4)), c = lane & 15;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float a0 = rr == c ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                const float *lr = Ls + (base + rr) * 65 + base;
#pragma unroll
                for (int i = 0; i < rr; ++i) {
                    const float t = lr[i] * x[i];
                    if ((i & 3) == 0) a0 -= t;
                    else if ((i & 3) == 1) a1 -= t;
                    else if ((i & 3) == 2) a2 -= t;
                    else a3 -= t;
                }
                x[rr] = (a0 + a1) + (a2 + a3);
            }
            __syncwarp();
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) Lb[(base + rr) * 72 + base + c] = __float2bfloat16_rn(x[rr]);
        } else if (warp >= 6) {
            const int r = 32 * (wq - 2) + lane;
            const uint8_t *vs = sm + STG_V + (ci & 1) * 8192;
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + COL_O + 32 * half, a);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 vv = *reinterpret_cast<const uint4 *>(vs + tc::sw128(r, 4 * half + q4));
                    const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
                    float rr[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 vf = unpack_bf16(vw[e]);
                        rr[2 * e] = vf.x - a[8 * q4 + 2 * e];
                        rr[2 * e + 1] = vf.y - a[8 * q4 + 2 * e + 1];
                    }
                    float *dst = Rf + r * 68 + 32 * half + 8 * q4;
                    *reinterpret_cast<float4 *>(dst) = make_float4(rr[0], rr[1], rr[2], rr[3]);
                    *reinterpret_cast<float4 *>(dst + 4) = make_float4(rr[4], rr[5], rr[6], rr[7]);
                }
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        if (!__syncthreads_and(ok)) { ok = false; break; }
        // ---- F. W = (I + L)^{-1} Diag(beta) R by block forward substitution on bf16
        // mma.sync (fp32 accumulate): W_R = X_RR (beta R_R - sum_{J<R} L_RJ W_J).
        // Warp w owns the eight d_v columns 8w..8w+7, so the four block rows need
        // only warp syncs. Y and W columns are kept transposed (ws[col][row], bf16)
        // so that B fragments are 32-bit pairs along k.
        {
            const int g = lane >> 2, t = lane & 3, c0 = 8 * warp;
            __nv_bfloat16 *ws = Wsc + warp * 8 * 72;                // [8 cols][72]
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                const int r0 = 16 * R + g, r1 = r0 + 8;
                float y[4];
                {
                    const float2 v0 = *reinterpret_cast<const float2 *>(Rf + r0 * 68 + c0 + 2 * t);
                    const float2 v1 = *reinterpret_cast<const float2 *>(Rf + r1 * 68 + c0 + 2 * t);
                    const float b0 = bet[r0], b1 = bet[r1];
                    y[0] = b0 * v0.x; y[1] = b0 * v0.y; y[2] = b1 * v1.x; y[3] = b1 * v1.y;
                }
                float part[3][4];
#pragma unroll
                for (int J = 0; J < R; ++J) {
                    const int kc = 16 * J + 2 * t;
                    const uint32_t a[4] = {*reinterpret_cast<const uint32_t *>(Lb + r0 * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(Lb + r1 * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(Lb + r0 * 72 + kc + 8),
                                           *reinterpret_cast<const uint32_t *>(Lb + r1 * 72 + kc + 8)};
                    const uint32_t b[2] = {*reinterpret_cast<const uint32_t *>(ws + g * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(ws + g * 72 + kc + 8)};
                    float (&pp)[4] = part[J];
                    pp[0] = pp[1] = pp[2] = pp[3] = 0.f;
                    tc::mma_bf16_16816(pp, a, b);
                }
#pragma unroll
                for (int J = 0; J < R; ++J) {
                    y[0] -= part[J][0]; y[1] -= part[J][1]; y[2] -= part[J][2]; y[3] -= part[J][3];
                }
                // Y (rows of block R) -> ws, then W_R = X_RR Y
                ws[(2 * t) * 72 + r0] = __float2bfloat16_rn(y[0]);
                ws[(2 * t + 1) * 72 + r0] = __float2bfloat16_rn(y[1]);
                ws[(2 * t) * 72 + r1] = __float2bfloat16_rn(y[2]);
                ws[(2 * t + 1) * 72 + r1] = __float2bfloat16_rn(y[3]);
                __syncwarp();
                float w[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const int kc = 16 * R + 2 * t;
                    const uint32_t a[4] = {*reinterpret_cast<const uint32_t *>(Lb + r0 * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(Lb + r1 * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(Lb + r0 * 72 + kc + 8),
                                           *reinterpret_cast<const uint32_t *>(Lb + r1 * 72 + kc + 8)};
                    const uint32_t b[2] = {*reinterpret_cast<const uint32_t *>(ws + g * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(ws + g * 72 + kc + 8)};
                    tc::mma_bf16_16816(w, a, b);
                }
                __syncwarp();
                ws[(2 * t) * 72 + r0] = __float2bfloat16_rn(w[0]);
                ws[(2 * t + 1) * 72 + r0] = __float2bfloat16_rn(w[1]);
                ws[(2 * t) * 72 + r1] = __float2bfloat16_rn(w[2]);
                ws[(2 * t + 1) * 72 + r1] = __float2bfloat16_rn(w[3]);
                // bf16 W for round 3: columns c0 + 2t, c0 + 2t + 1 lie in 16-byte chunk `warp`
                *reinterpret_cast<uint32_t *>(sm + OP_W + tc::sw128(r0, warp) + 4 * t) = pack_bf16(w[0], w[1]);
                *reinterpret_cast<uint32_t *>(sm + OP_W + tc::sw128(r1, warp) + 4 * t) = pack_bf16(w[2], w[3]);
                __syncwarp();
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        // ---- H. round 3: O += A_qk W ; D = Kb^T W ---------------------------------------
        if (tid == 0) {
            tc::fence_after_sync();
            // O += A_qk W as an M=128 MMA (O1 came from the M=128 round 1): its A rows
            // 64-127 are the W tile that follows A_qk in shared memory, and land in
            // TMEM lanes 64-127 of COL_O, which are not read afterwards
            constexpr uint32_t id_o = tc::idesc_bf16(128, 64, false, true);
            constexpr uint32_t id_s = tc::idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + COL_O, dAQK + 2 * k, dW + 128 * k, id_o, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + COL_S, dKBmn + 128 * k, dW + 128 * k, id_s, k > 0);
            tc::mma_commit(mma_bar);
        }
        ok = tc::bar_wait(mma_bar, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc::fence_after_sync();
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

// [T, H, 128] tensor, boxes of (inner, 1 head, 64 tokens). An empty or absent array gets
// a zeroed map: a call without tokens has no chunk, so no launch reads it.
inline bool encode_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t esize, int H,
                       int64_t T, uint32_t box_inner, CUtensorMapSwizzle sw) {
    std::memset(m, 0, sizeof(*m));
    if (!base || T <= 0) return true;
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
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
        return fail_text("cuTensorMapEncodeTiled failed for q, k, v or g");
    P.p = p;
    P.p.n_items = p.n_seq * H * 2;
    static std::atomic<unsigned long long> attr_done{0};
    const kda_status r = set_smem_limit_once((const void *)prefill_tc_kernel, (int)tcp::SMEM_BYTES, attr_done);
    if (r != KDA_OK) return r;
    if (!gate()) return KDA_ERR_CUDA;
    prefill_tc_kernel<<<P.p.n_items, tcp::NT, tcp::SMEM_BYTES, st>>>(P);
    return launch_result();
}

}  // namespace kda
