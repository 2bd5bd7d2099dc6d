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

}  // namespace kda
