// Launch plan shared by the two KDA prefill kernels.
//
// Chunk-form algebra (Kimi K3 technical FAQ, "What is KDA": the state is
// updated per chunk, parallel within a chunk and recurrent across chunks; the
// algebra below is derived here from the recurrence, the pages give none).
// For one (sequence, head) and a chunk of C tokens with state S_0 on entry,
// b_r = sum_{i<=r} g_i (inclusive, per key channel), Gamma_r = exp(b_r):
//   A_kk[r,i] = sum_c k_rc k_ic exp(b_rc - b_ic)      (i <  r)
//   A_qk[r,i] = sum_c q_rc k_ic exp(b_rc - b_ic)      (i <= r)
//   (I + Diag(beta) A_kk) W = Diag(beta) (V - (K . Gamma) S_0)
//   O   = scale [ (Q . Gamma) S_0 + A_qk W ]
//   S_C = Diag(Gamma_C) S_0 + (K . exp(b_C - b))^T W
// This equals C steps of S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1}
// + beta_t k_t v_t^T, o_t = scale S_t^T q_t, in real arithmetic.
//
// Snapshots (vLLM day-0 blog, "Kimi Delta Attention": state snapshots at block
// boundaries) fall on chunk ends: the host requires snap_interval % C == 0 and
// start_pos % C == 0 whenever snapshots are requested.
#pragma once
#include "common.cuh"
#include "tc_util.cuh"

namespace kda {

struct PrefillSeq {
    int32_t tok0;       // first token of the sequence in the packed arrays (this launch)
    int32_t len;        // tokens
    int64_t start_pos;  // tokens already absorbed by the initial state
    int64_t snap_off;   // first snapshot row of this sequence
};

constexpr int kPrefillSeqs = KDA_SEQS_PER_LAUNCH;

struct PrefillParams {
    const void *q, *k, *v;
    const float *g, *beta;
    const float *state_in;   // [n_seq, H, D, D] or null (zeros); rows indexed by seq
    float *state_out;        // may be null
    void *o;
    float *snapshots;
    int32_t H, n_seq, snap_interval, n_items;
    float scale;
    int16_t order[kPrefillSeqs];  // sequences, longest first
    PrefillSeq seq[kPrefillSeqs];
};

// ---- chunks beyond the single-reference range (both tensor-core kernels) -------
// The scaled operands Qh = q 2^(b - r1), Ka = k 2^(b - r1), Kb = k 2^(r2 - b) (log2
// units) take, per key channel, r1 = r2 = m (the chunk middle) when the channel's decay
// from m stays within the range limit, and otherwise r1 = 0, r2 = b_C (every factor
// <= 1; eM = 2^r1 = 1 and eC = 2^(b_C - r2) = 1, so the chain's algebra is unchanged).
// A channel on the second reference contributes q k 2^(b_r - b_i + b_C) ~ 0 to the
// tensor-core A; its true part, q_rc k_ic 2^(b_rc - b_ic), is added to A in TMEM from
// staged raw values (fast_correct). Up to kMaxFast such channels per chunk; beyond that
// the chunk is reported as KDA_ERR_RANGE.
struct FastChannels {
    uint32_t mask[4];   // bit l of mask[e]: channel 4 l + e is on the second reference
    int n;
};

__device__ __forceinline__ FastChannels fast_channels(const bool (&fast)[4]) {
    FastChannels f;
    f.n = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f.mask[e] = __ballot_sync(0xffffffffu, fast[e]);
        f.n += __popc(f.mask[e]);
    }
    return f;
}
// compact index of channel 4 lane + e among the channels on the second reference
__device__ __forceinline__ int fast_index(const FastChannels &f, int lane, int e) {
    const uint32_t below = (1u << lane) - 1u;
    int idx = 0;
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) idx += __popc(f.mask[e2] & below) + (e2 < e ? (f.mask[e2] >> lane) & 1 : 0);
    return idx;
}

// Add the pairwise part of the channels on the second reference to the A tile in TMEM
// (rows 0-63 A_qk with q, rows 64-127 A_kk with k; columns i <= r, resp. i < r, of 64):
// the calling warp's 32 lanes = rows 32 (warp % 4) + lane. fq, fk, fb: [kMaxFast][64] raw
// q, raw k and b (log2 units) of those channels; past the chunk's length q and k are zero
// and b stays at its last live value, so that every exponent taken here is <= 0 (a zero b
// there would overflow 2^(b_r - b_i) and put 0 * inf into the rows past the length).
template <int kMaxFast>
__device__ __forceinline__ void fast_correct(uint32_t taddr_row, int r, int nf, const float *fq,
                                             const float *fk, const float *fb) {
    const bool qk = r < 64;
    const int row = r & 63;
    nf = min(nf, kMaxFast);
    for (int half = 0; half < 2; ++half) {
        float a[32];
        tc::tmem_ld32(taddr_row + 32 * half, a);
        tc::tmem_ld_wait();
        for (int f = 0; f < nf; ++f) {
            const float xr = (qk ? fq : fk)[f * 64 + row], br = fb[f * 64 + row];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int i = 32 * half + j;
                const bool on = qk ? i <= row : i < row;
                if (on) a[j] = fmaf(xr * fk[f * 64 + i], tc::ex2(br - fb[f * 64 + i]), a[j]);
            }
        }
        tc::tmem_st32(taddr_row + 32 * half, a);
    }
    tc::tmem_st_wait();
}

}  // namespace kda
