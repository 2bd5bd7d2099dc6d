// KDA chunked prefill in two launches (d_k = d_v = 128, chunk 64, bf16 q/k/v/o,
// fp32 state), for callers that provide a workspace. The chunk form is the one in
// prefill_common.cuh; the scaled operands are those of prefill_tc.cuh (Qh, Ka, Kb
// around a per-channel reference m at the chunk middle, Sm = Diag(e^m) S_0).
//
// With T = (I + Diag(beta) A_kk)^{-1} (unit lower triangular), W' = T Diag(beta) Ka
// and U = T Diag(beta) V, the chunk update becomes
//     W   = U - W' Sm
//     O   = scale (Qh Sm + A_qk W)
//     S_C = Diag(Gamma_C) S_0 + Diag(e^(b_C - m)) Kb^T W
// so everything except two small products per chunk is independent of S_0:
//
//   prep   one CTA per (chunk, head), all chunks of all sequences at once:
//          cumsum, scaled operands, A = [Qh; Ka] Kb^T (tcgen05; each scaled operand split
//          into bf16 high and low parts, three products, so A is fp32-accurate), T by block forward
//          substitution (mma.sync), [W' | U] = (T Diag(beta)) [Ka | V] (tcgen05). Writes
//          one packet per (chunk, head) to the workspace, laid out as the shared
//          memory images the chain kernel feeds to its MMAs.
//   chain  one CTA per (sequence, head, 64-column d_v slice): per chunk, one bulk
//          copy of the packet head (three chunks in flight; U is read into registers
//          a chunk ahead), then
//            round 1  [Qh; W'] Sm          -> TMEM (M=128: rows 0-63 O, 64-127 W'Sm)
//            W = U - W'Sm (bf16)
//            round 2  D = Kb^T W, then O += A_qk W (separate commits)
//          the fp32 state update in registers and Sm of the next chunk. O and snapshots
//          leave during the following chunks through staging tiles and tiled TMA stores.
#pragma once
#include <cudaTypedefs.h>

#include "prefill_common.cuh"
#include "tc_util.cuh"

namespace kda {

namespace spl {
constexpr int C = 64, D = 128;
// ---- workspace packet of one (chunk, head); every image is 128B-swizzled slabs
constexpr uint32_t PK_QW = 0;         // [Qh; W']: 2 slabs (channels 0-63, 64-127) x 128 rows
constexpr uint32_t PK_KB = 32768;     // Kb: 2 slabs x 64 token rows
constexpr uint32_t PK_AQK = 49152;    // A_qk masked (i <= r), 1 slab x 64 rows
constexpr uint32_t PK_VEC = 57344;    // eM, eC, gC: fp32 [3][128] (1536 B, slot of 2048)
constexpr uint32_t PK_U = 59392;      // U: 2 slabs (d_v 0-63, 64-127) x 64 token rows
constexpr uint32_t PACKET = PK_U + 16384;   // 75776 bytes
// ---- prep kernel shared memory
constexpr uint32_t P_QK = 0;          // 2 slabs x 128 rows: q -> Qh (rows 0-63), k -> Ka (rows 64-127)
constexpr uint32_t P_V = 32768;       // v: 2 slabs x 64 rows (loaded once MMA A has finished: until
                                      // then slab 0 of the low parts below lives here)
constexpr uint32_t P_KB = 49152;      // Kb: 2 slabs x 64 rows
constexpr uint32_t P_TI = 65536;      // T (bf16): 1 slab x 64 rows
constexpr uint32_t P_G = 73728;       // g fp32 [64][128]; once the operands are built, the solve
                                      // scratch: Ls, Lb, Wsc below
constexpr uint32_t P_LS = P_G;                    // fp32 [64][17]: L on its diagonal 16x16 blocks
constexpr uint32_t P_LB = P_LS + 64 * 17 * 4;     // bf16 [64][72]: L, and X on the diagonal blocks
constexpr uint32_t P_WSC = P_LB + 64 * 72 * 2;    // bf16 [8 warps][8][72]
constexpr uint32_t P_AQK = P_G + 23552;           // A_qk staging (1 slab x 64 rows), 1024-aligned
constexpr uint32_t P_TOT = P_G + 32768;           // fp32 [8][128] row-block totals of b
constexpr uint32_t P_VEC = P_TOT + 4096;          // eM, eC, gC [128], beta [64]
constexpr uint32_t P_BARS = P_VEC + (3 * 128 + 64) * 4;
constexpr uint32_t P_SMEM = P_BARS + 48 + 1024;   // + slack for 1024-byte alignment
constexpr uint32_t P_TX = 16384 * 2 + 32768;      // q, k, g bytes per chunk
constexpr uint32_t P_TX_V = 16384;                // v bytes per chunk
// Low bf16 parts of the scaled operands (x - bf16(x), rounded to bf16), live from the
// operand pass until MMA A completes, in memory that is free during that window:
// [Qh_lo; Ka_lo] slab 0 over v's buffer, slab 1 and Kb_lo over T and g (g is in registers)
constexpr uint32_t P_LO0 = P_V;                   // [Qh_lo; Ka_lo] channels 0-63, 128 rows
constexpr uint32_t P_LO1 = P_TI;                  // [Qh_lo; Ka_lo] channels 64-127, 128 rows
constexpr uint32_t P_KBLO = P_TI + 16384;         // Kb_lo: 2 slabs x 64 rows
constexpr uint32_t P_COL_A = 0, P_COL_W = 0, P_COL_U = 128, P_TMEM = 256;
// ---- chain kernel shared memory
constexpr uint32_t STAGE = PK_U;                  // the packet head ([Qh; W'], Kb, A_qk, vectors)
constexpr int NSTAGE = 3;
constexpr uint32_t C_SM = NSTAGE * STAGE;         // Sm (bf16): MN-major B, 128 d_k rows x 64 d_v
constexpr uint32_t C_W = C_SM + 16384;            // W (bf16): MN-major B, 64 token rows x 64 d_v
constexpr uint32_t C_O = C_W + 8192;              // O staging for a tiled store: 64 tokens x 64 d_v bf16
constexpr uint32_t C_SN = C_O + 8192;             // snapshot staging: 64 d_k rows x 64 d_v fp32 as two
                                                  // 128B-swizzled boxes of 32 columns
constexpr uint32_t C_BARS = C_SN + 16384;
constexpr uint32_t C_SMEM = C_BARS + 64 + 1024;
// TMEM: round 1 / O of chunk c in columns 64 (c % 2) .. +63 (O is read during chunk c + 1),
// D = Kb^T W in 128 .. 191
constexpr uint32_t C_COL_R1 = 0, C_COL_D = 128, C_TMEM = 256;
// U in the packet, in the order the chain's W threads read it: 16-byte piece q4 (8 d_v
// columns) of column group wg (32 columns) of d_v half hf for token row r is at
// PK_U + ((hf * 2 + wg) * 4 + q4) * 1024 + 16 r, so a warp's 32 rows are 512 contiguous bytes
__host__ __device__ constexpr uint32_t u_piece(int hf, int wg, int q4, int r) {
    return PK_U + (uint32_t)(((hf * 2 + wg) * 4 + q4) * 1024 + 16 * r);
}
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RANGE_LIMIT2 = 80.f * LOG2E;      // 80 nats, in log2 units
// raw q, k and b of the channels beyond that range ([kMaxFast][64] fp32 each), in the tail
// of g's buffer (free once the cumsum has read g, until A_qk is staged after the correction)
constexpr int kMaxFast = 8;
constexpr uint32_t P_FQ = P_G + 24576, P_FK = P_FQ + kMaxFast * 256, P_FB = P_FK + kMaxFast * 256;
static_assert(P_WSC + 8 * 8 * 72 * 2 <= P_AQK && P_AQK + 8192 <= P_TOT && P_AQK % 1024 == 0,
              "solve scratch overlaps");
static_assert(P_KBLO + 16384 <= P_TOT && P_LO1 % 1024 == 0 && P_KBLO % 1024 == 0,
              "low parts overlap live data");
static_assert(P_FQ >= P_KBLO + 16384 && P_FB + kMaxFast * 256 <= P_TOT, "fast-channel staging");
static_assert(2 * (P_SMEM + 1024) <= 233472, "two prep CTAs per SM");
static_assert(STAGE % 1024 == 0 && PACKET % 16 == 0 && C_O % 1024 == 0 && C_SN % 1024 == 0, "alignment");
static_assert(C_SMEM <= 232448, "chain shared memory");
}  // namespace spl

// Packet row of chunk c of sequence i (launch-local index): ((tok0 - tok_first) >> 6) + i + c.
// Sequences' ranges are disjoint and increasing, and every index is below
// ((tok_end - tok_first) >> 6) + n_seq.
struct PrepParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_g;
    const float *beta;
    uint8_t *ws;
    int32_t H, n_seq, tok_first, n_packets;
    int32_t tok0[kPrefillSeqs];
    int32_t len[kPrefillSeqs];
};

struct ChainParams {
    CUtensorMap tm_o;        // o [T, H, 128] bf16, boxes of 64 d_v x 1 head x 64 tokens, 128B swizzle
    CUtensorMap tm_snap;     // snapshots as [rows, 128] fp32, boxes of 32 x 64, 128B swizzle
    PrefillParams p;
    const uint8_t *ws;
    int32_t tok_first;
    int32_t snap_tma;        // 1: snapshot rows fit the 32-bit box coordinates of tm_snap
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 bf16x2_unpack(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}
// a, b -> (bf16 pair hi, bf16 pair lo) with hi + lo = (a, b) to about 2^-17 relative:
// the operands of a three-term bf16 product hi*hi' + lo*hi' + hi*lo' that is accurate to
// fp32 level although the tensor cores take bf16
__device__ __forceinline__ void bf16x2_split(float a, float b, uint32_t &hi, uint32_t &lo) {
    hi = bf16x2(a, b);
    // the residuals are exact in fp32; they are truncated to bf16 (their upper halves,
    // one byte permute instead of a second conversion): error below 2^-17 of a, b
    const float ra = a - __uint_as_float(hi << 16), rb = b - __uint_as_float(hi & 0xffff0000u);
    lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
}
__device__ __forceinline__ uint4 bf16x8(const float *a, float s) {
    return make_uint4(bf16x2(s * a[0], s * a[1]), bf16x2(s * a[2], s * a[3]), bf16x2(s * a[4], s * a[5]),
                      bf16x2(s * a[6], s * a[7]));
}

// ============================================================================ prep
__global__ void __launch_bounds__(256, 2) prefill_prep_kernel(const __grid_constant__ PrepParams P) {
    using namespace spl;
    const int H = P.H;
    const int h = blockIdx.x % H;
    const int pk = blockIdx.x / H;
    // owner sequence: the last one whose first packet is <= pk
    auto first_packet = [&](int i) { return ((P.tok0[i] - P.tok_first) >> 6) + i; };
    int lo = 0, hi = P.n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first_packet(mid) <= pk) lo = mid; else hi = mid - 1;
    }
    const int c = pk - first_packet(lo);
    const int len = P.len[lo];
    if (c < 0 || c * C >= len) return;       // an unused packet row (block-uniform)
    const int n = min(C, len - c * C);
    const int z = P.tok0[lo] + c * C;
    uint8_t *pkt = P.ws + ((int64_t)pk * H + h) * PACKET;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(sm);
    float *Gs = reinterpret_cast<float *>(sm + P_G);
    float *Ls = reinterpret_cast<float *>(sm + P_LS);
    __nv_bfloat16 *Lb = reinterpret_cast<__nv_bfloat16 *>(sm + P_LB);
    __nv_bfloat16 *Wsc = reinterpret_cast<__nv_bfloat16 *>(sm + P_WSC);
    float *Tot = reinterpret_cast<float *>(sm + P_TOT);
    float *eM = reinterpret_cast<float *>(sm + P_VEC);
    float *eC = eM + 128, *gC = eM + 256, *bet = eM + 384;
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + P_BARS);
    uint64_t *bar_a = bar_ld + 1, *bar_w = bar_ld + 2, *bar_v = bar_ld + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_ld + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3;
    if (tid == 0) {
        tc::bar_init(bar_ld, 1);
        tc::bar_init(bar_a, 1);
        tc::bar_init(bar_w, 1);
        tc::bar_init(bar_v, 1);
        tc::bar_init_fence();
        tc::bar_expect_tx(bar_ld, P_TX);
        tc::tma_load3(sm + P_QK, &P.tm_q, 0, h, z, bar_ld);
        tc::tma_load3(sm + P_QK + 16384, &P.tm_q, 64, h, z, bar_ld);
        tc::tma_load3(sm + P_QK + 8192, &P.tm_k, 0, h, z, bar_ld);
        tc::tma_load3(sm + P_QK + 16384 + 8192, &P.tm_k, 64, h, z, bar_ld);
        tc::tma_load3(sm + P_G, &P.tm_g, 0, h, z, bar_ld);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, P_TMEM);
        tc::tmem_relinquish();
    }
    // beta (a strided load): issued now, stored once the TMA loads have landed, so the two
    // latencies overlap
    const float bv = (tid < C && tid < n) ? P.beta[(int64_t)(z + tid) * H + h] : 0.f;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = (uint32_t)(32 * wq) << 16;
    bool ok = true, stored = false, v_issued = false;

    do {
        ok = tc::bar_wait(bar_ld, 0);
        if (tid < C) bet[tid] = bv;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        // ---- b = cumsum(g) (log2 units): warp w rows 8w..8w+7, lane channels 4l..4l+3
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
                    bc[e] += tv[e];                 // b at row 63 (= row n-1)
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) b[i][e] += off[e];
            // references per channel: the chunk middle, or (beyond the range) 0 and b_C
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
                    const int ch = 4 * lane + e;
                    eM[ch] = tc::ex2(r1[e]);
                    eC[ch] = tc::ex2(bc[e] - r2[e]);
                    gC[ch] = tc::ex2(bc[e]);
                }
                if (lane == 0 && n_fast > kMaxFast) record_status(KDA_ERR_RANGE);
            }
        }
        if (n_fast > 0) {
            // raw q, k and b of the channels on the second reference (r1 != r2), for
            // fast_correct, read before the pass below scales q and k in place
            const int pkb = lane >> 4, pchk = (lane & 15) >> 1, phf = (lane & 1) * 8;
            bool fast[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) fast[e] = r1[e] != r2[e];
            const FastChannels fch = fast_channels(fast);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * warp + i;
                const uint32_t so = tc::sw128(r, pchk) + phf;
                const uint2 qv = *reinterpret_cast<const uint2 *>(sm + P_QK + pkb * 16384 + so);
                const uint2 kv = *reinterpret_cast<const uint2 *>(sm + P_QK + pkb * 16384 + 8192 + so);
                const float2 q01 = bf16x2_unpack(qv.x), q23 = bf16x2_unpack(qv.y);
                const float2 k01 = bf16x2_unpack(kv.x), k23 = bf16x2_unpack(kv.y);
                const float qr[4] = {q01.x, q01.y, q23.x, q23.y}, kr[4] = {k01.x, k01.y, k23.x, k23.y};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int f = fast[e] ? fast_index(fch, lane, e) : kMaxFast;
                    if (f < kMaxFast) {
                        const bool live = r < n;
                        reinterpret_cast<float *>(sm + P_FQ)[f * 64 + r] = live ? qr[e] : 0.f;
                        reinterpret_cast<float *>(sm + P_FK)[f * 64 + r] = live ? kr[e] : 0.f;
                        reinterpret_cast<float *>(sm + P_FB)[f * 64 + r] = b[i][e];   // b_(n-1) past n
                    }
                }
            }
            __syncwarp();
        }
        // ---- Qh = q 2^(b-r1), Ka = k 2^(b-r1) in place; Kb = k 2^(r2-b)
        {
            const int pkb = lane >> 4, pchk = (lane & 15) >> 1, phf = (lane & 1) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * warp + i;
                const uint32_t so = tc::sw128(r, pchk) + phf;
                uint8_t *qp = sm + P_QK + pkb * 16384 + so;
                uint8_t *kp = sm + P_QK + pkb * 16384 + 8192 + so;
                const uint2 qv = *reinterpret_cast<const uint2 *>(qp);
                const uint2 kv = *reinterpret_cast<const uint2 *>(kp);
                const float2 q01 = bf16x2_unpack(qv.x), q23 = bf16x2_unpack(qv.y);
                const float2 k01 = bf16x2_unpack(kv.x), k23 = bf16x2_unpack(kv.y);
                float e1[4], e2[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    e1[e] = tc::ex2(b[i][e] - r1[e]);
                    e2[e] = tc::ex2(r2[e] - b[i][e]);
                }
                // high parts in place of q and k (and Kb), low parts in the P_LO* slabs
                uint2 qh = make_uint2(0u, 0u), ql = qh, ah = qh, al = qh, bh = qh, bl = qh;
                if (r < n) {
                    bf16x2_split(q01.x * e1[0], q01.y * e1[1], qh.x, ql.x);
                    bf16x2_split(q23.x * e1[2], q23.y * e1[3], qh.y, ql.y);
                    bf16x2_split(k01.x * e1[0], k01.y * e1[1], ah.x, al.x);
                    bf16x2_split(k23.x * e1[2], k23.y * e1[3], ah.y, al.y);
                    bf16x2_split(k01.x * e2[0], k01.y * e2[1], bh.x, bl.x);
                    bf16x2_split(k23.x * e2[2], k23.y * e2[3], bh.y, bl.y);
                }
                uint8_t *lo = sm + (pkb ? P_LO1 : P_LO0) + so;
                *reinterpret_cast<uint2 *>(qp) = qh;
                *reinterpret_cast<uint2 *>(kp) = ah;
                *reinterpret_cast<uint2 *>(lo) = ql;
                *reinterpret_cast<uint2 *>(lo + 8192) = al;
                *reinterpret_cast<uint2 *>(sm + P_KB + pkb * 8192 + so) = bh;
                *reinterpret_cast<uint2 *>(sm + P_KBLO + pkb * 8192 + so) = bl;
            }
        }
        tc::fence_async_smem();
        __syncthreads();
        // ---- A = [Qh; Ka] Kb^T (M=128: A_qk rows 0-63, A_kk rows 64-127) to fp32 accuracy as
        // hi hi' + lo hi' + hi lo' (the lo lo' term is below fp32 rounding); Qh and Kb (high
        // parts) go to the packet as they are
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_a = tc::idesc_bf16(128, 64, false, false);
            const uint64_t dQK = tc::desc_k(sbase + P_QK, 0), dKB = tc::desc_k(sbase + P_KB, 0);
            const uint64_t dQKlo = tc::desc_k(sbase + P_LO0, 0), dKBlo = tc::desc_k(sbase + P_KBLO, 0);
            constexpr uint32_t lo_slab = (P_LO1 - P_LO0) >> 4;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + P_COL_A, dQK + (k >> 2) * 1024 + (k & 3) * 2, dKB + (k >> 2) * 512 + (k & 3) * 2,
                             id_a, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + P_COL_A, dQKlo + (k >> 2) * lo_slab + (k & 3) * 2,
                             dKB + (k >> 2) * 512 + (k & 3) * 2, id_a, 1);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + P_COL_A, dQK + (k >> 2) * 1024 + (k & 3) * 2,
                             dKBlo + (k >> 2) * 512 + (k & 3) * 2, id_a, 1);
            tc::mma_commit(bar_a);
        } else if (tid == 32) {
            tc::bulk_store(pkt + PK_QW, sm + P_QK, 8192);
            tc::bulk_store(pkt + PK_QW + 16384, sm + P_QK + 16384, 8192);
            tc::bulk_store(pkt + PK_KB, sm + P_KB, 16384);
            tc::bulk_commit();
            stored = true;
        }
        if (tid < 96)
            reinterpret_cast<float4 *>(pkt + PK_VEC)[tid] = reinterpret_cast<const float4 *>(eM)[tid];
        ok = tc::bar_wait(bar_a, 0);
        tc::fence_after_sync();
        if (tid == 0 && ok) {
            // the low parts are dead: v goes into its buffer (needed by the last MMAs only)
            tc::bar_expect_tx(bar_v, P_TX_V);
            tc::tma_load3(sm + P_V, &P.tm_v, 0, h, z, bar_v);
            tc::tma_load3(sm + P_V + 8192, &P.tm_v, 64, h, z, bar_v);
            v_issued = true;
        }
        if (n_fast > 0) {
            // the pairwise part of the channels beyond the range, into A (TMEM)
            if (warp < 4)
                fast_correct<kMaxFast>(tbase + tlane + P_COL_A, 32 * warp + lane, n_fast,
                                       reinterpret_cast<const float *>(sm + P_FQ),
                                       reinterpret_cast<const float *>(sm + P_FK),
                                       reinterpret_cast<const float *>(sm + P_FB));
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
        }
        if (warp < 2) {
            // A_qk, masked to i <= r, into its staging image (bulk-stored after this phase)
            const int r = 32 * warp + lane;
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + P_COL_A + 32 * half, a);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int jj = 32 * half + 8 * q4 + 2 * e;
                        w[e] = bf16x2(jj <= r ? a[8 * q4 + 2 * e] : 0.f, jj + 1 <= r ? a[8 * q4 + 2 * e + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(sm + P_AQK + tc::sw128(r, 4 * half + q4)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        } else if (warp < 4) {
            // L = Diag(beta) A_kk strictly below the diagonal: bf16 everywhere, fp32 on
            // the diagonal blocks; then the inverses X of the four diagonal blocks
            const int r = 32 * (warp - 2) + lane;
            const float br = bet[r];
            const int dblk = r & ~15;
            float a[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld32(tbase + tlane + P_COL_A + 32 * half, a);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float l[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int jj = 32 * half + 8 * q4 + e;
                        l[e] = jj < r ? br * a[8 * q4 + e] : 0.f;
                        if (jj >= dblk && jj < dblk + 16) Ls[r * 17 + (jj - dblk)] = l[e];
                    }
                    *reinterpret_cast<uint4 *>(Lb + r * 72 + 32 * half + 8 * q4) = bf16x8(l, 1.f);
                }
            }
            __syncwarp();
            const int base = 16 * (2 * (warp - 2) + (lane >> 4)), cc = lane & 15;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float a0 = rr == cc ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                const float *lr = Ls + (base + rr) * 17;
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
            for (int rr = 0; rr < 16; ++rr) Lb[(base + rr) * 72 + base + cc] = __float2bfloat16_rn(x[rr]);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        if (!__syncthreads_and(ok)) { ok = false; break; }
        if (tid == 32) {
            tc::bulk_store(pkt + PK_AQK, sm + P_AQK, 8192);
            tc::bulk_commit();
            stored = true;
        }
        // ---- T = (I + L)^{-1} by block forward substitution on bf16 mma.sync (fp32
        // accumulate): T_R = X_RR (E_R - sum_{J<R} L_RJ T_J), E = identity. Warp w
        // owns columns 8w..8w+7.
        {
            const int g = lane >> 2, t = lane & 3, c0 = 8 * warp;
            __nv_bfloat16 *ws = Wsc + warp * 8 * 72;
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                const int r0 = 16 * R + g, r1 = r0 + 8;
                float y[4] = {r0 == c0 + 2 * t ? 1.f : 0.f, r0 == c0 + 2 * t + 1 ? 1.f : 0.f,
                              r1 == c0 + 2 * t ? 1.f : 0.f, r1 == c0 + 2 * t + 1 ? 1.f : 0.f};
                float part[3][4];
#pragma unroll
                for (int J = 0; J < R; ++J) {
                    const int kc = 16 * J + 2 * t;
                    const uint32_t a[4] = {*reinterpret_cast<const uint32_t *>(Lb + r0 * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(Lb + r1 * 72 + kc),
                                           *reinterpret_cast<const uint32_t *>(Lb + r0 * 72 + kc + 8),
                                           *reinterpret_cast<const uint32_t *>(Lb + r1 * 72 + kc + 8)};
                    const uint32_t bb[2] = {*reinterpret_cast<const uint32_t *>(ws + g * 72 + kc),
                                            *reinterpret_cast<const uint32_t *>(ws + g * 72 + kc + 8)};
                    float (&pp)[4] = part[J];
                    pp[0] = pp[1] = pp[2] = pp[3] = 0.f;
                    tc::mma_bf16_16816(pp, a, bb);
                }
#pragma unroll
                for (int J = 0; J < R; ++J) {
                    y[0] -= part[J][0]; y[1] -= part[J][1]; y[2] -= part[J][2]; y[3] -= part[J][3];
                }
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
                    const uint32_t bb[2] = {*reinterpret_cast<const uint32_t *>(ws + g * 72 + kc),
                                            *reinterpret_cast<const uint32_t *>(ws + g * 72 + kc + 8)};
                    tc::mma_bf16_16816(w, a, bb);
                }
                __syncwarp();
                ws[(2 * t) * 72 + r0] = __float2bfloat16_rn(w[0]);
                ws[(2 * t + 1) * 72 + r0] = __float2bfloat16_rn(w[1]);
                ws[(2 * t) * 72 + r1] = __float2bfloat16_rn(w[2]);
                ws[(2 * t + 1) * 72 + r1] = __float2bfloat16_rn(w[3]);
                // T Diag(beta) (bf16, K-major A operand of the next MMAs: W' = T Diag(beta) Ka,
                // U = T Diag(beta) V); columns c0 + 2t, c0 + 2t + 1 are in 16-byte chunk `warp`
                const float b0 = bet[c0 + 2 * t], b1 = bet[c0 + 2 * t + 1];
                *reinterpret_cast<uint32_t *>(sm + P_TI + tc::sw128(r0, warp) + 4 * t) = bf16x2(w[0] * b0, w[1] * b1);
                *reinterpret_cast<uint32_t *>(sm + P_TI + tc::sw128(r1, warp) + 4 * t) = bf16x2(w[2] * b0, w[3] * b1);
                __syncwarp();
            }
        }
        if (tid == 32 && stored) {            // A_qk, Qh, Kb read out: the staging area is reused below
            tc::bulk_wait_read_all();
            stored = false;
        }
        if (tid == 0) ok = tc::bar_wait(bar_v, 0);    // v has landed (the MMAs below read it)
        tc::fence_async_smem();
        tc::fence_before_sync();
        if (!__syncthreads_and(ok)) { ok = false; break; }
        // ---- [W' | U] = (T Diag(beta)) [Ka | V]  (M=64: row r in TMEM lane (r % 16) + 32 (r / 16))
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_w = tc::idesc_bf16(64, 128, false, true);
            const uint64_t dT = tc::desc_k(sbase + P_TI, 0);
            const uint64_t dBK = tc::desc_mn(sbase + P_QK + 8192, 0, 16384);
            const uint64_t dBV = tc::desc_mn(sbase + P_V, 0, 8192);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + P_COL_W, dT + 2 * k, dBK + 128 * k, id_w, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + P_COL_U, dT + 2 * k, dBV + 128 * k, id_w, k > 0);
            tc::mma_commit(bar_w);
        }
        ok = tc::bar_wait(bar_w, 0);
        tc::fence_after_sync();
        {
            // warp (wq, wh): rows 16 wq .. 16 wq + 15 (lanes 0-15), columns 64 wh .. 64 wh + 63.
            // The images are staged in the solve scratch (free since T was built): W' slabs at
            // P_G, P_G + 8192; U (in the chain's read order) at P_G + 16384; then bulk-stored.
            const int wh = warp >> 2, r = 16 * wq + lane;
            float a[32];
#pragma unroll
            for (int mat = 0; mat < 2; ++mat) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    tc::tmem_ld32(tbase + tlane + (mat ? P_COL_U : P_COL_W) + 64 * wh + 32 * hh, a);
                    tc::tmem_ld_wait();
                    if (lane < 16) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint32_t off = mat ? P_G + u_piece(wh, hh, q4, r) - PK_U + 16384
                                                     : P_G + wh * 8192 + tc::sw128(r, 4 * hh + q4);
                            *reinterpret_cast<uint4 *>(sm + off) = bf16x8(a + 8 * q4, 1.f);
                        }
                    }
                }
            }
        }
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 32) {
            tc::bulk_store(pkt + PK_QW + 8192, sm + P_G, 8192);
            tc::bulk_store(pkt + PK_QW + 16384 + 8192, sm + P_G + 8192, 8192);
            tc::bulk_store(pkt + PK_U, sm + P_G + 16384, 16384);
            tc::bulk_commit();
            stored = true;
        }
    } while (0);

    if (!ok && tid == 0) {                              // loads still in flight land first
        tc::bar_wait(bar_ld, 0, 1u << 16);
        if (v_issued) tc::bar_wait(bar_v, 0, 1u << 16);
    }
    if (stored) tc::bulk_wait_read_all();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, P_TMEM);
}

// =========================================================================== chain
__global__ void __launch_bounds__(256, 1) prefill_chain_kernel(const __grid_constant__ ChainParams CP) {
    using namespace spl;
    const PrefillParams &p = CP.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(sm);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + C_BARS);   // [NSTAGE]
    uint64_t *bar_r1 = full + NSTAGE, *bar_d = full + NSTAGE + 1, *bar_o = full + NSTAGE + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + NSTAGE + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;
    const bool wwarp = wq >= 2;                   // TMEM lanes 64-127: W rows; else O rows
    const int H = p.H;
    const int item = blockIdx.x;
    const int rank = item / (H * 2);
    const int h = (item >> 1) % H;
    const int half = item & 1, j0 = 64 * half;
    const int s = p.order[rank];
    const PrefillSeq sq = p.seq[s];
    const int n_chunks = (sq.len + C - 1) / C;
    const int64_t pk0 = ((sq.tok0 - CP.tok_first) >> 6) + s;
    auto packet = [&](int ci) { return CP.ws + ((pk0 + ci) * H + h) * PACKET; };

    if (tid == 0) {
        for (int i = 0; i < NSTAGE + 3; ++i) tc::bar_init(&full[i], 1);
        tc::bar_init_fence();
        tc::tma_prefetch_desc(&CP.tm_o);
        if (p.snap_interval > 0 && CP.snap_tma) tc::tma_prefetch_desc(&CP.tm_snap);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, C_TMEM);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = (uint32_t)(32 * wq) << 16;

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
        uint64_t *bar = &full[ci % NSTAGE];
        tc::bar_expect_tx(bar, STAGE);
        tc::bulk_load(sm + (ci % NSTAGE) * STAGE, packet(ci), STAGE, bar);
    };
    int issued = 0, landed = 0;
    if (tid == 0)
        for (; issued < NSTAGE - 1 && issued < n_chunks; ++issued) issue_loads(issued);
    // U rows of a chunk for the W threads (token row r_w, columns 32 wh .. +31 of the slice),
    // read from the workspace one chunk ahead
    const int r_w = 32 * (wq - 2) + lane;
    uint4 u[4];
    auto load_u = [&](int ci) {
        const uint8_t *pkt = packet(ci);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
            u[q4] = *reinterpret_cast<const uint4 *>(pkt + u_piece(half, wh, q4, r_w));
    };
    if (wwarp && n_chunks > 0) load_u(0);
    // U of chunk ci into L2 two chunks ahead, so that the register loads of it (one chunk
    // ahead, just before the end barrier) hit L2 rather than HBM: -6 % on the chain
    auto prefetch_u = [&](int ci) {
        if ((lane & 7) == 0) {
            const uint8_t *pkt = packet(ci);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(pkt + u_piece(half, wh, q4, r_w)) : "memory");
        }
    };
    if (wwarp && n_chunks > 1) prefetch_u(1);

    const uint64_t dSM = tc::desc_mn(sbase + C_SM, 0, 16384);
    const uint64_t dW = tc::desc_mn(sbase + C_W, 0, 8192);
    bool ok = true;
    // Sm = Diag(e^m) S (bf16, MN-major: row = d_k channel, 64 d_v columns) for the chunk
    // whose packet sits in stage `st`
    auto write_sm = [&](int st) {
        const float em = reinterpret_cast<const float *>(sm + st * STAGE + PK_VEC)[c_own];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4 *>(sm + C_SM + tc::sw128(c_own, 4 * wh + q4)) = bf16x8(S + 8 * q4, em);
    };
    if (n_chunks > 0) {
        ok = tc::bar_wait(&full[0], 0);
        if (ok) write_sm(0);
        tc::fence_async_smem();
        ok = __syncthreads_and(ok);
        landed = 1;
    }

    // Snapshots: the state after a due chunk is written during the next two chunks through
    // the staging tile and tiled stores: d_k rows 0-63 (held by the O warps) during the
    // first, rows 64-127 (W warps, from the copy Ss) during the second. Threads 32 and 64
    // issue the stores and wait for their reads before the staging is written again.
    float Ss[32];
    int64_t next_snap = p.snap_interval > 0 ? (sq.start_pos / p.snap_interval + 1) * p.snap_interval : -1;
    int64_t snap_row = sq.snap_off;
    int64_t snap_pend = -1;               // snapshot row with a half still to be written
    int snap_half = 0;                    // which half goes out during this chunk
    bool stores_pending = false;          // thread 32 / 64: tiled stores issued, reads not waited for
    auto direct_snapshot = [&](int64_t row, const float *src) {
        float *dst = p.snapshots + ((row * H + h) * D + c_own) * (int64_t)D + j0 + 32 * wh;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(src[j], src[j + 1], src[j + 2], src[j + 3]);
    };
    auto stage_snapshot = [&](const float *src) {
        uint8_t *box = sm + C_SN + wh * 8192;
        const int r = c_own & 63;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4 *>(box + tc::sw128(r, q)) =
                make_float4(src[4 * q], src[4 * q + 1], src[4 * q + 2], src[4 * q + 3]);
    };
    auto store_snapshot_half = [&](int64_t row, int hf) {
        const int y = (int)((row * H + h) * D + 64 * hf);
        tc::tma_store2(&CP.tm_snap, sm + C_SN, j0, y);
        tc::tma_store2(&CP.tm_snap, sm + C_SN + 8192, j0 + 32, y);
    };

    for (int ci = 0; ok && ci < n_chunks; ++ci) {
        const int n = min(C, sq.len - ci * C);
        const int st = ci % NSTAGE;
        uint8_t *stg = sm + st * STAGE;
        const uint32_t sstg = sbase + st * STAGE;
        const uint32_t col_r1 = C_COL_R1 + 64 * (ci & 1);
        const float *eC = reinterpret_cast<const float *>(stg + PK_VEC) + 128, *gC = eC + 128;
        // ---- round 1: [Qh; W'] Sm -> rows 0-63 O, rows 64-127 W'Sm
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id1 = tc::idesc_bf16(128, 64, false, true);
            const uint64_t dQW = tc::desc_k(sstg + PK_QW, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tbase + col_r1, dQW + (k >> 2) * 1024 + (k & 3) * 2, dSM + 128 * k, id1, k > 0);
            tc::mma_commit(bar_r1);
        }
        float ov[32];          // O of chunk ci - 1 (O warps)
        if (wwarp && ci + 2 < n_chunks) prefetch_u(ci + 2);
        if (wwarp) {
            // ---- W = U - W' Sm (token rows in TMEM lanes 64-127)
            ok = tc::bar_wait(bar_r1, (uint32_t)(ci & 1));
            tc::fence_after_sync();
            float a[32];
            tc::tmem_ld32(tbase + tlane + col_r1 + 32 * wh, a);
            tc::tmem_ld_wait();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const uint32_t uw[4] = {u[q4].x, u[q4].y, u[q4].z, u[q4].w};
                float w[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 uf = bf16x2_unpack(uw[e]);
                    w[2 * e] = uf.x - a[8 * q4 + 2 * e];
                    w[2 * e + 1] = uf.y - a[8 * q4 + 2 * e + 1];
                }
                *reinterpret_cast<uint4 *>(sm + C_W + tc::sw128(r_w, 4 * wh + q4)) = bf16x8(w, 1.f);
            }
            tc::fence_async_smem();
        } else {
            // O warps, while round 1 runs: the outputs of chunk ci - 1 (its MMAs were committed
            // before the previous chunk's end barrier, so the phase awaited is bar_o's latest)
            // and half 0 of a pending snapshot leave through the staging tiles now, off the
            // recurrence's critical path
            const int pn = min(C, sq.len - (ci - 1) * C);
            const int r = 32 * wq + lane;
            const bool tiled = ci > 0 && pn == C;
            const bool snap = snap_pend >= 0 && snap_half == 0;
            if (ci > 0) {
                ok = tc::bar_wait(bar_o, (uint32_t)((ci - 1) & 1));
                tc::fence_after_sync();
                tc::tmem_ld32(tbase + tlane + C_COL_R1 + 64 * ((ci - 1) & 1) + 32 * wh, ov);
                tc::tmem_ld_wait();
            }
            if (ci > 0 && !tiled && r < pn) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) +
                                                       ((int64_t)(sq.tok0 + (ci - 1) * C + r) * H + h) * D + j0 + 32 * wh);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) dst[q4] = bf16x8(ov + 8 * q4, p.scale);
            }
            // thread 32's stores of the previous chunk have read the tiles (issued a chunk ago:
            // no wait in practice), before anyone writes them again
            if (stores_pending) {
                tc::bulk_wait_read_all();
                stores_pending = false;
            }
            if (tiled || snap) {
                tc::named_sync(1, 128);
                if (tiled) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + C_O + tc::sw128(r, 4 * wh + q4)) = bf16x8(ov + 8 * q4, p.scale);
                }
                if (snap) stage_snapshot(S);
                tc::fence_async_smem();
                tc::named_sync(1, 128);
                if (tid == 32) {
                    if (tiled) tc::tma_store3(&CP.tm_o, sm + C_O, j0, h, sq.tok0 + (ci - 1) * C);
                    if (snap) store_snapshot_half(snap_pend, 0);
                    tc::bulk_commit();
                    stores_pending = true;
                }
            }
        }
        tc::fence_before_sync();
        const bool mid_ok = __syncthreads_and(ok);
        // ---- round 2: D = Kb^T W (commit bar_d), then O += A_qk W (M=128; A rows 64-127 are
        // the bytes after A_qk and land in TMEM lanes 64-127, not read again; commit bar_o);
        // then the loads of chunk ci + NSTAGE - 1 into the stage of chunk ci - 1. Its last
        // readers were that chunk's MMAs, which completed before this chunk's round 1 did
        // (one thread issues every MMA, and a commit covers all earlier ones), and the W warps
        // saw round 1 complete before the barrier above.
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t id_o = tc::idesc_bf16(128, 64, false, true);
            constexpr uint32_t id_d = tc::idesc_bf16(128, 64, true, true);
            const uint64_t dAQK = tc::desc_k(sstg + PK_AQK, 0);
            const uint64_t dKB = tc::desc_mn(sstg + PK_KB, 0, 8192);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + C_COL_D, dKB + 128 * k, dW + 128 * k, id_d, k > 0);
            tc::mma_commit(bar_d);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::mma_bf16(tbase + col_r1, dAQK + 2 * k, dW + 128 * k, id_o, 1);
            tc::mma_commit(bar_o);
            if (mid_ok && issued < n_chunks) {
                issue_loads(issued);
                ++issued;
            }
        }
        // ---- while this chunk's MMAs run: the W warps send half 1 of a pending snapshot
        if (wwarp && snap_pend >= 0 && snap_half == 1) {
            stage_snapshot(Ss);
            tc::fence_async_smem();
            tc::named_sync(2, 128);
            if (tid == 64) {
                store_snapshot_half(snap_pend, 1);
                tc::bulk_commit();
                stores_pending = true;
            }
        }
        if (snap_pend >= 0) {                 // the same bookkeeping in every thread
            if (snap_half == 0) snap_half = 1;
            else snap_pend = -1;
        }
        // ---- state update, then Sm of the next chunk
        {
            bool okd = tc::bar_wait(bar_d, (uint32_t)(ci & 1));
            tc::fence_after_sync();
            float a[32];
            const float g_c = gC[c_own], e_c = eC[c_own];
            tc::tmem_ld32(tbase + tlane + C_COL_D + 32 * wh, a);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) S[e] = fmaf(g_c, S[e], e_c * a[e]);
            if (ci + 1 < n_chunks) {
                okd = okd && tc::bar_wait(&full[(ci + 1) % NSTAGE], (uint32_t)(((ci + 1) / NSTAGE) & 1));
                if (okd) write_sm((ci + 1) % NSTAGE);
                tc::fence_async_smem();
                if (wwarp) load_u(ci + 1);
            }
            if (sq.start_pos + (int64_t)ci * C + n == next_snap) {
                next_snap += p.snap_interval;
                // a snapshot due at consecutive chunks: the W rows of the previous one go out now
                if (wwarp && snap_pend >= 0) direct_snapshot(snap_pend, Ss);
                if (CP.snap_tma) {
                    snap_pend = snap_row;
                    snap_half = 0;
#pragma unroll
                    for (int e = 0; e < 32; ++e) Ss[e] = S[e];
                } else {
                    direct_snapshot(snap_row, S);
                }
                ++snap_row;
            }
            ok = ok && okd;
        }
        // thread 64's half-1 snapshot stores have read the tile before the end barrier: the O
        // warps may stage the next snapshot's half 0 into it early in the next chunk
        if (wwarp && stores_pending) {
            tc::bulk_wait_read_all();
            stores_pending = false;
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(ok);
        if (ok) landed = ci + 2 < n_chunks ? ci + 2 : n_chunks;
    }
    if (ok && n_chunks > 0) {
        // outputs of the last chunk; snapshot halves still pending
        if (!wwarp) {
            float a[32];
            ok = tc::bar_wait(bar_o, (uint32_t)((n_chunks - 1) & 1));
            tc::fence_after_sync();
            tc::tmem_ld32(tbase + tlane + C_COL_R1 + 64 * ((n_chunks - 1) & 1) + 32 * wh, a);
            tc::tmem_ld_wait();
            const int r = 32 * wq + lane;
            if (r < min(C, sq.len - (n_chunks - 1) * C)) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) +
                                                       ((int64_t)(sq.tok0 + (n_chunks - 1) * C + r) * H + h) * D + j0 + 32 * wh);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) dst[q4] = bf16x8(a + 8 * q4, p.scale);
            }
            if (snap_pend >= 0 && snap_half == 0) direct_snapshot(snap_pend, S);
        } else if (snap_pend >= 0) {
            direct_snapshot(snap_pend, Ss);
        }
    }

    if (ok && p.state_out) {
        float *dst = p.state_out + (((int64_t)s * H + h) * D + c_own) * (int64_t)D + j0 + 32 * wh;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    if (tid == 0 && !ok) {
        for (int c2 = landed; c2 < issued; ++c2)
            tc::bar_wait(&full[c2 % NSTAGE], (uint32_t)((c2 / NSTAGE) & 1), 1u << 16);
    }
    if (stores_pending) tc::bulk_wait_read_all();     // staging must outlive the stores' reads
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, C_TMEM);
}

// ---------------------------------------------------------------------------- host
// Workspace bytes of one launch group: packets for ((tokens >> 6) + sequences) rows x H heads.
inline size_t split_group_bytes(int64_t group_tokens, int n_seq, int H) {
    return (size_t)((group_tokens >> 6) + n_seq) * (size_t)H * spl::PACKET;
}

// snapshots viewed as [rows, 128] fp32, boxes of 32 columns x 64 rows (128B swizzle)
inline bool encode_snap_map(CUtensorMap *m, float *base, int64_t rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128 * sizeof(float)};
    cuuint32_t box[2] = {32, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Gate>
inline kda_status launch_prefill_split(PrefillParams &p, const kda_dims &d, int64_t T, int32_t tok_first,
                                       int32_t tok_end, int64_t n_snap_total, void *ws, cudaStream_t st,
                                       Gate gate) {
    using namespace spl;
    static thread_local PrepParams PP;
    static thread_local ChainParams CPm;
    const int H = d.H;
    const int64_t n_packets = ((int64_t)(tok_end - tok_first) >> 6) + p.n_seq;
    if (n_packets * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (!encode_map(&PP.tm_q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map(&PP.tm_k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map(&PP.tm_v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map(&PP.tm_g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, T, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return fail_text("cuTensorMapEncodeTiled failed for q, k, v or g");
    PP.beta = p.beta;
    PP.ws = static_cast<uint8_t *>(ws);
    PP.H = H;
    PP.n_seq = p.n_seq;
    PP.tok_first = tok_first;
    PP.n_packets = (int32_t)n_packets;
    for (int i = 0; i < p.n_seq; ++i) {
        PP.tok0[i] = p.seq[i].tok0;
        PP.len[i] = p.seq[i].len;
    }
    CPm.p = p;
    CPm.p.n_items = p.n_seq * H * 2;
    CPm.ws = static_cast<const uint8_t *>(ws);
    CPm.tok_first = tok_first;
    if (!encode_map(&CPm.tm_o, p.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return fail_text("cuTensorMapEncodeTiled failed for o");
    const int64_t snap_rows = n_snap_total * H * D;
    CPm.snap_tma = p.snapshots && n_snap_total > 0 && snap_rows < 0x7fffffffLL;
    if (CPm.snap_tma && !encode_snap_map(&CPm.tm_snap, p.snapshots, snap_rows))
        return fail_text("cuTensorMapEncodeTiled failed for the snapshots");
    static std::atomic<unsigned long long> prep_attr{0}, chain_attr{0};
    kda_status r = set_smem_limit_once((const void *)prefill_prep_kernel, (int)P_SMEM, prep_attr);
    if (r == KDA_OK) r = set_smem_limit_once((const void *)prefill_chain_kernel, (int)C_SMEM, chain_attr);
    if (r != KDA_OK) return r;
    if (n_packets > 0) {
        if (!gate()) return KDA_ERR_CUDA;
        prefill_prep_kernel<<<(unsigned)(n_packets * H), 256, P_SMEM, st>>>(PP);
        r = launch_result();
        if (r != KDA_OK) return r;
    }
    if (!gate()) return KDA_ERR_CUDA;
    prefill_chain_kernel<<<CPm.p.n_items, 256, C_SMEM, st>>>(CPm);
    return launch_result();
}

}  // namespace kda
