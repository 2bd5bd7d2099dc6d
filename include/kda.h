/*
 * libkda — Kimi Delta Attention (KDA) hot path on NVIDIA B200 (sm_100a).
 *
 * The operation (Kimi K3 technical FAQ, runpod.io, "What is KDA, and why does a
 * serving engineer care?": a delta-rule linear-attention recurrence with a
 * per-channel forget gate and a fixed d_k x d_v state per head, computed
 * parallel within a chunk and recurrent across chunks), in the standard
 * gated-delta form, per sequence and head:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t,        alpha_t = exp(g_t) in (0, 1]^{d_k}
 *
 * State snapshots (vLLM day-0 blog, "Kimi Delta Attention": prefix caching over
 * recurrent state reuses state snapshots taken at block boundaries): the state
 * after absolute position p is a snapshot when p % snap_interval == 0.
 *
 * Conventions shared by every call
 *  - Layouts (row-major, innermost last): q, k, g: [tokens, H, d_k];
 *    v, o: [tokens, H, d_v]; beta: [tokens, H]; a state: [H, d_k, d_v] fp32 with
 *    d_v contiguous; pools of states: [n, H, d_k, d_v].
 *  - q, k, v, o are bf16 (KDA_IO_BF16) or fp32 (KDA_IO_FP32); g (= log alpha,
 *    must be <= 0), beta (in [0, 1]) and states are always fp32. q and k are
 *    used as given: the library does not normalise them.
 *  - Pointers suffixed _h are host memory read during the call only. All other
 *    pointers are device memory owned by the caller; the library allocates no
 *    memory and keeps no state between calls except a device status word.
 *    Scratch memory, where a call can use it, is a caller-provided workspace,
 *    with one exception: kda_prefill_noalloc uses a fixed device array of
 *    kda_prefill_noalloc_capacity() bytes that the library's module holds on
 *    every device it is loaded on, from module load until process exit.
 *  - Every device pointer must be 16-byte aligned (KDA_ERR_ALIGN otherwise).
 *  - Calls are asynchronous on `stream`: argument errors return synchronously
 *    before anything is launched; device-side range errors and bounded-wait
 *    timeouts are recorded in the status word read by kda_check_device_status.
 *  - Element offsets are 64-bit; tokens per call must be < 2^31.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same handle type); NULL is the legacy default stream. */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID = 1,     /* bad argument: null pointer, negative size, bad cu_seqlens ... */
    KDA_ERR_UNSUPPORTED = 2, /* dimensions outside the compiled set (see kda_dims) */
    KDA_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
    KDA_ERR_WORKSPACE = 4,   /* workspace smaller than kda_prefill_workspace_size reports */
    KDA_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
    KDA_ERR_TIMEOUT = 6,     /* a device-side wait ran out of iterations (device status) */
    KDA_ERR_RANGE = 7        /* device-side check failed: a slot or index out of range, or a
                                gate whose decay over one chunk is outside the supported
                                range of the tensor-core prefill (device status) */
} kda_status;

typedef enum { KDA_IO_BF16 = 0, KDA_IO_FP32 = 1 } kda_io;

typedef struct {
    int32_t H;     /* heads, >= 1 */
    int32_t dk;    /* key head dim;   supported: dk == dv in {32, 64, 128} */
    int32_t dv;    /* value head dim */
    int32_t chunk; /* prefill chunk length C in {16, 32, 64}; unused by decode/verify */
    int32_t io;    /* kda_io: element type of q, k, v, o */
    float scale;   /* output scale; 0 selects 1/sqrt(dk) */
} kda_dims;

/* Maximum sequences per kernel launch; larger batches are split by the library
 * into several launches on the same stream. */
#define KDA_SEQS_PER_LAUNCH 1024

/*
 * The q/k front-end (Kimi K3 technical FAQ, "What is KDA, and why does a serving
 * engineer care?": queries and keys go through a short convolution, Swish and L2
 * normalization before the recurrence). Per head h and key channel c, over the raw
 * inputs x of one sequence (q and k each with their own weights):
 *     y_t = sum_{j=0}^{taps-1} w[h][c][j] * x_{t-(taps-1)+j}   (causal, depthwise,
 *                                                              no bias; tap taps-1
 *                                                              on the current token)
 *     z_t = y_t * sigmoid(y_t)                                 (Swish)
 *     out_t = z_t / max(||z_t||_2, 1e-6)                        (over the dk channels)
 * A sequence's conv state is its last taps-1 raw inputs (zeros for a fresh
 * sequence), fp32, laid out [2 (q then k), H, dk, taps-1], oldest input first; pools
 * of conv states are [n, 2, H, dk, taps-1]. Conv states travel with the recurrent
 * states: the calls below carry them across calls and snapshot them at the same
 * block boundaries.
 */
typedef struct {
    int32_t taps;          /* 2, 3 or 4 */
    const float *w_q;      /* [H, dk, taps] fp32, device */
    const float *w_k;      /* [H, dk, taps] fp32, device */
} kda_conv;

/*
 * kda_snapshot_plan — where each sequence's snapshots go (host only, no GPU).
 * Snapshot rule of the vLLM day-0 blog, "Kimi Delta Attention" (snapshots at
 * block boundaries): sequence s (tokens cu_seqlens_h[s] .. cu_seqlens_h[s+1]-1,
 * with start_pos_h[s] tokens already absorbed by its initial state; NULL means
 * all zero) takes a snapshot after each absolute position p with
 * start_pos < p <= start_pos + len and p % snap_interval == 0, ascending.
 *   snap_offsets_h [n_seq+1] (out): exclusive prefix sum of per-sequence counts;
 *                                   snapshot j of sequence s is row
 *                                   snap_offsets_h[s] + j of the snapshot pool.
 *   snap_pos_h     [snap_offsets_h[n_seq]] (out, nullable): the positions p.
 * snap_interval == 0 means no snapshots (all offsets 0).
 * Errors: KDA_ERR_INVALID for n_seq < 0, null cu_seqlens_h / snap_offsets_h,
 * cu_seqlens_h[0] != 0, decreasing cu_seqlens_h, negative start_pos or interval.
 */
kda_status kda_snapshot_plan(int32_t n_seq, const int32_t *cu_seqlens_h,
                             const int64_t *start_pos_h, int32_t snap_interval,
                             int64_t *snap_offsets_h, int64_t *snap_pos_h);

/*
 * kda_prefill_workspace_size — bytes of device workspace that kda_prefill can
 * use for these dimensions and sequence lengths (host only, no GPU). 0 when the
 * dimensions run on the CUDA-core path, which uses none. For the tensor-core
 * dimensions (dk = dv = 128, chunk 64, bf16) it is, over each launch group of
 * at most KDA_SEQS_PER_LAUNCH sequences, the largest
 * (floor(group tokens / 64) + group sequences) * H * 75776.
 * Errors: KDA_ERR_INVALID (null `bytes` or cu_seqlens_h, bad cu_seqlens_h),
 * KDA_ERR_UNSUPPORTED as kda_prefill.
 */
kda_status kda_prefill_workspace_size(const kda_dims *dims, int32_t n_seq,
                                      const int32_t *cu_seqlens_h, size_t *bytes);

/*
 * kda_prefill — packed variable-length chunked prefill (Kimi K3 technical FAQ,
 * "What is KDA": parallel within a chunk, recurrent across chunks; the
 * chunk-form algebra is derived from the recurrence in the library's design
 * notes). Sequence s is tokens [cu_seqlens_h[s], cu_seqlens_h[s+1]) of the
 * packed q, k, v, g, beta, o arrays (T_total = cu_seqlens_h[n_seq] tokens).
 *   start_pos_h [n_seq] (nullable = zeros): tokens already absorbed by the
 *               initial state; sets the absolute positions of snapshots.
 *   state_in  [n_seq, H, dk, dv] (nullable = zero states): initial states.
 *   state_out [n_seq, H, dk, dv] (nullable): state after each sequence's last
 *               token. May alias state_in (in-place update).
 *   o         [T_total, H, dv]: outputs, written for every token.
 *   snap_interval: 0 (none) or a multiple of dims->chunk; with snapshots on,
 *               every start_pos must be a multiple of dims->chunk.
 *   snapshots [kda_snapshot_plan total, H, dk, dv] (required when any
 *               snapshot is due): fp32 states, rows as kda_snapshot_plan says.
 *   workspace (nullable), workspace_bytes: device scratch, 16-byte aligned,
 *               owned by the caller and not read back by it. With a workspace
 *               the tensor-core dimensions run in two launches per group (all
 *               chunks' state-independent work in parallel, then the
 *               recurrence across chunks); with NULL they run in one launch
 *               that keeps every intermediate on chip. Results agree to
 *               rounding, not bit for bit, between the two. The workspace must
 *               not be used by other work until the call's kernels finish.
 * A zero-length sequence writes state_out = state_in and no snapshots; in a call
 * without tokens (cu_seqlens all zero) q, k, v, g, beta and o may be NULL.
 * Errors (before launch): KDA_ERR_INVALID, KDA_ERR_UNSUPPORTED, KDA_ERR_ALIGN,
 * KDA_ERR_WORKSPACE (non-null workspace below kda_prefill_workspace_size).
 * Gate range on the tensor-core path: with b_r = g_0 + ... + g_r summed over a
 * chunk's tokens r = 0..63, a key channel with -b_31 > 80 or b_31 - b_last > 80
 * (more than 80 nats of decay from the chunk's middle in either direction) is
 * computed on a second, bounded reference with its part of the intra-chunk
 * products from pairwise exponentials; results are as for any other chunk. Up to 8
 * such channels per chunk and head (two-launch path) or 4 (single launch) are
 * handled; a chunk with more records device status KDA_ERR_RANGE and its outputs
 * are then not reliable. The CUDA-core path has no such limit.
 */
kda_status kda_prefill(const kda_dims *dims, int32_t n_seq, const int32_t *cu_seqlens_h,
                       const int64_t *start_pos_h, const void *q, const void *k,
                       const void *v, const float *g, const float *beta,
                       const float *state_in, float *state_out, void *o,
                       int32_t snap_interval, float *snapshots, void *workspace,
                       size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_prefill_noalloc — kda_prefill without a caller workspace and without any
 * allocation: the two-launch path runs on the library's fixed device scratch of
 * kda_prefill_noalloc_capacity() bytes (a module-level array, resident from the
 * library's first use on a device). When kda_prefill_workspace_size exceeds it, the
 * call runs as several two-launch pieces on the stream: consecutive sequences whose
 * workspace fits together, and a sequence too long for the scratch in windows of
 * whole chunks, with its state handed between windows in fp32 through the scratch.
 * The results are bit-identical to one kda_prefill call with a workspace. Only when a
 * piece's beta pointer would not be 16-byte aligned (H not a multiple of 4) does it
 * take the single-launch path instead. Arguments, layouts and errors as kda_prefill. For callers that cannot allocate device memory at the point of
 * the call (code running inside a captured or replayed stream region, or a host
 * that forbids allocation after start-up) and cannot set a workspace aside.
 * The scratch is shared by all calls on a device of this process and keeps the
 * last call's contents (every call writes what it reads): calls that could
 * overlap on the GPU (issued on different streams, or from different host
 * threads) race, so the caller must order them, e.g. issue them on one stream.
 * The scratch's device address is looked up once per device, on the first call
 * that uses it; make that first call before any stream capture.
 */
kda_status kda_prefill_noalloc(const kda_dims *dims, int32_t n_seq, const int32_t *cu_seqlens_h,
                               const int64_t *start_pos_h, const void *q, const void *k,
                               const void *v, const float *g, const float *beta,
                               const float *state_in, float *state_out, void *o,
                               int32_t snap_interval, float *snapshots, kda_stream_t stream);

/* Bytes of the fixed scratch kda_prefill_noalloc uses (64 MiB). */
size_t kda_prefill_noalloc_capacity(void);

/*
 * kda_decode — one token per sequence against a pool of live states, updating
 * each state in place with one read and one write of it. This is one step t of
 * the recurrence at the top of this header (Kimi K3 technical FAQ, "What is KDA,
 * and why does a serving engineer care?": the fixed d_k x d_v state per head is
 * all a decode step reads and rewrites, instead of a growing KV cache; runtimewire,
 * "The architecture is built around inference cost": KDA layers carry a
 * fixed-size recurrent state).
 *   q, k, g [n_seq, H, dk]; v, o [n_seq, H, dv]; beta [n_seq, H].
 *   slots [n_seq] (device int32): row of state_pool used by each sequence;
 *               slots must be distinct (a repeated slot is a data race).
 *   state_pool [n_slots, H, dk, dv]: read and written in place.
 * Device status KDA_ERR_RANGE if a slot is outside [0, n_slots) (that
 * sequence is skipped).
 */
kda_status kda_decode(const kda_dims *dims, int32_t n_seq, const void *q, const void *k,
                      const void *v, const float *g, const float *beta, const int32_t *slots,
                      int32_t n_slots, float *state_pool, void *o, kda_stream_t stream);

/*
 * kda_verify — speculative verify (runtimewire, "A third party tripled
 * single-user decoding speed": a draft model proposes several tokens and the
 * target accepts a prefix of them per step, 2.61 to 4.73 on average; Kimi K3
 * technical FAQ, "What is the speculative-decoding story?"). Sequence s runs its
 * draft tokens [cu_draft_h[s], cu_draft_h[s+1]) (packed like prefill) through the
 * recurrence at the top of this header from the state state_pool[slots[s]],
 * which is only read, and writes the output and the state after every token, so
 * that the caller can commit the state of the last accepted token with
 * kda_snapshot (rollback of rejected drafts).
 *   token_states [cu_draft_h[n_seq], H, dk, dv]: state after each token.
 * Errors as kda_decode.
 */
kda_status kda_verify(const kda_dims *dims, int32_t n_seq, const int32_t *cu_draft_h,
                      const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const int32_t *slots, int32_t n_slots,
                      const float *state_pool, float *token_states, void *o,
                      kda_stream_t stream);

/*
 * kda_verify_commit — one speculative step with the previous step's commit fused
 * in, so that no per-token state is ever written (vLLM day-0 blog, "Kimi Delta
 * Attention": the recurrent state lives in state blocks and is snapshotted at
 * block boundaries; runtimewire, "A third party tripled single-user decoding
 * speed": each step accepts a prefix of its draft tokens). Acceptance of a step
 * is known only after every layer has verified it, so the commit of step n-1
 * runs inside the verify of step n. For sequence s, with S = state_pool[slots[s]]
 * holding the state before the previous step's tokens:
 *   1. commit: the first n_accept[s] tokens of the previous step's batch
 *      [cu_prev_h[s], cu_prev_h[s+1]) (k_prev, v_prev, g_prev, beta_prev, packed
 *      like kda_verify's input; their q is not needed) run through the
 *      recurrence at the top of this header and S is written back in place (not
 *      written when n_accept[s] == 0). With snap_interval > 0 and snap_row[s] >= 0,
 *      the state after the committed token at absolute position p = pos[s] + j + 1
 *      with p % snap_interval == 0, if one of the committed tokens is there, is
 *      also written to snapshots[snap_row[s]] (at most one such p when
 *      snap_interval >= the batch length).
 *   2. verify: this step's tokens [cu_draft_h[s], cu_draft_h[s+1]) (q, k, v, g,
 *      beta) run from the committed state; their outputs go to o [cu_draft_h[n_seq],
 *      H, dv]; the state is not written.
 * Mixed step (a serving step of continuous batching in one launch): with
 * commit_new[s] != 0 (device uint8 [n_seq], nullable = all zero) the tokens of step 2
 * are committed too, i.e. S is written after them (after step 1's tokens otherwise):
 * a decode token (n_accept[s] = 0, one token), or a short prefill appended to a live
 * sequence, runs in the same launch as the speculative sequences. A block-boundary
 * snapshot then counts the committed tokens of both steps, in order.
 * The state after step 1 is bit-identical to kda_verify's state after token
 * n_accept[s] - 1 of the previous batch, and the outputs of step 2 to kda_verify's
 * from that state (with commit_new, the state written to kda_verify's state after the
 * last token, and for one token to kda_decode's). A pipeline drains with a call
 * whose draft batch is empty.
 *   n_accept [n_seq] (device int32), 0 <= n_accept[s] <= cu_prev_h[s+1] - cu_prev_h[s].
 *   pos [n_seq] (device int64, required with snapshots): tokens absorbed by S.
 *   snap_row [n_seq] (device int64, nullable), snapshots [n_snap_rows, H, dk, dv].
 * Device status KDA_ERR_RANGE (that sequence is skipped: neither S nor its outputs
 * are written) for a slot outside [0, n_slots), n_accept outside its range, or a
 * snap_row >= n_snap_rows. Other errors as kda_verify.
 */
kda_status kda_verify_commit(const kda_dims *dims, int32_t n_seq, const int32_t *cu_prev_h,
                             const void *k_prev, const void *v_prev, const float *g_prev,
                             const float *beta_prev, const int32_t *n_accept, const int64_t *pos,
                             int32_t snap_interval, const int64_t *snap_row, float *snapshots,
                             int64_t n_snap_rows, const int32_t *cu_draft_h, const void *q,
                             const void *k, const void *v, const float *g, const float *beta,
                             const uint8_t *commit_new, const int32_t *slots, int32_t n_slots,
                             float *state_pool, void *o, kda_stream_t stream);

/*
 * kda_snapshot — bit-exact copies of whole states between pools: for i < n,
 * dst[dst_idx[i]] = src[src_idx[i]] (each an [H, dk, dv] fp32 state). Used to
 * commit a verified token's state, restore a cached prefix snapshot into a
 * live slot, or save a live state (vLLM day-0 blog, prefix caching over
 * recurrent state).
 *   src_idx, dst_idx [n] (device int64); src [n_src, ...], dst [n_dst, ...].
 * Destinations must be distinct and must not overlap the sources read.
 * Device status KDA_ERR_RANGE for an index outside its pool (copy skipped).
 */
kda_status kda_snapshot(int32_t n, const int64_t *src_idx, const int64_t *dst_idx,
                        const float *src, int64_t n_src, float *dst, int64_t n_dst,
                        int32_t H, int32_t dk, int32_t dv, kda_stream_t stream);

/*
 * kda_qk_frontend — the front-end above over a packed prefill batch, producing the
 * normalised q and k that kda_prefill takes. Sequences, start_pos_h, snap_interval
 * and the snapshot rule are as in kda_prefill (the same kda_snapshot_plan rows).
 *   q_raw, k_raw [T_total, H, dk] (bf16 or fp32 as dims->io): raw inputs.
 *   conv_in  [n_seq, 2, H, dk, taps-1] (nullable = zeros), conv_out (nullable): the
 *            conv state before and after each sequence.
 *   q_out, k_out [T_total, H, dk]: normalised outputs (may not alias the inputs).
 *   conv_snapshots [kda_snapshot_plan total, 2, H, dk, taps-1] (required when a
 *            snapshot is due): the conv state after each snapshot position.
 * Errors: as kda_prefill, and KDA_ERR_INVALID for a null conv, taps outside 2..4
 * or null weights.
 */
kda_status kda_qk_frontend(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                           const int32_t *cu_seqlens_h, const int64_t *start_pos_h,
                           const void *q_raw, const void *k_raw, const float *conv_in,
                           float *conv_out, void *q_out, void *k_out, int32_t snap_interval,
                           float *conv_snapshots, kda_stream_t stream);

/*
 * kda_decode_conv, kda_verify_conv, kda_verify_commit_conv — kda_decode, kda_verify
 * and kda_verify_commit with the front-end fused into their token loads: q and k
 * (and q_prev, k_prev) are raw inputs, and each sequence's conv state is carried
 * next to its recurrent state in conv_pool [n_slots, 2, H, dk, taps-1]:
 *   decode:        conv_pool[slots[s]] is updated in place with the state slot.
 *   verify:        conv_pool is only read; conv_token_states [T, 2, H, dk, taps-1]
 *                  (nullable) receives the conv state after every draft token, the
 *                  companion of token_states for rollback.
 *   verify_commit: the replay of the accepted prefix advances conv_pool[slots[s]]
 *                  (written with the state); q_prev is required (it moves the q
 *                  conv state); a block-boundary snapshot also writes the conv state
 *                  to conv_snapshots[snap_row[s]] ([n_snap_rows, 2, H, dk, taps-1]).
 * Other arguments, layouts and errors as the calls without the front-end.
 */
kda_status kda_decode_conv(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                           const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const int32_t *slots, int32_t n_slots,
                           float *state_pool, float *conv_pool, void *o, kda_stream_t stream);
kda_status kda_verify_conv(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                           const int32_t *cu_draft_h, const void *q, const void *k,
                           const void *v, const float *g, const float *beta,
                           const int32_t *slots, int32_t n_slots, const float *state_pool,
                           const float *conv_pool, float *token_states,
                           float *conv_token_states, void *o, kda_stream_t stream);
kda_status kda_verify_commit_conv(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                                  const int32_t *cu_prev_h, const void *q_prev,
                                  const void *k_prev, const void *v_prev, const float *g_prev,
                                  const float *beta_prev, const int32_t *n_accept,
                                  const int64_t *pos, int32_t snap_interval,
                                  const int64_t *snap_row, float *snapshots,
                                  float *conv_snapshots, int64_t n_snap_rows,
                                  const int32_t *cu_draft_h, const void *q, const void *k,
                                  const void *v, const float *g, const float *beta,
                                  const uint8_t *commit_new, const int32_t *slots,
                                  int32_t n_slots, float *state_pool, float *conv_pool, void *o,
                                  kda_stream_t stream);

/*
 * kda_state_map_apply — out[i] = M[i] X[i] + N[i] for i < n, fp32 (N nullable = 0).
 * Splitting one long sequence across workers (runtimewire, "The architecture is
 * built around inference cost": KDA carries a fixed-size recurrent state over a
 * 1M-token context): each step S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1}
 * + beta_t k_t v_t^T is affine in the state, so a token segment maps its entering
 * state S to M S + N, where M (dk x dk) is kda_prefill's final state for the segment
 * with v = 0 from the identity state (dv = dk), and N its final state from zero.
 * Maps compose as (M2, N2) o (M1, N1) = (M2 M1, M2 N1 + N2): two calls of this
 * function. A worker holding segment r applies the maps of segments 0..r-1 to the
 * sequence's initial state, then runs kda_prefill of its segment from the result.
 *   M [n, dk, dk]; X, N, out [n, dk, dv] (per head: n = segments x H), device fp32.
 *   out may alias N; it must not overlap M or X (KDA_ERR_INVALID when equal).
 */
kda_status kda_state_map_apply(int64_t n, int32_t dk, int32_t dv, const float *M, const float *X,
                               const float *N, float *out, kda_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char *kda_status_string(kda_status s);

/*
 * kda_check_device_status — synchronises `stream`, then returns and clears the
 * device status word of the current device (KDA_OK, KDA_ERR_RANGE or
 * KDA_ERR_TIMEOUT; the first error recorded since the last check), or
 * KDA_ERR_CUDA if the synchronisation itself failed.
 */
kda_status kda_check_device_status(kda_stream_t stream);

/* Text behind the most recent KDA_ERR_CUDA (static storage): the CUDA error, a
 * failed tensor-map encoding, or an injected launch failure; "no error" if there
 * was none. */
const char *kda_last_cuda_error(void);

/* Number of kernel launches the library has issued in this process (for
 * launch accounting in benchmarks). */
int64_t kda_launch_count(void);

/* ---- Failure-injection hooks (tests) -------------------------------------
 * kda_test_fail_next_launches(n): the next n launches are not issued and
 *   report KDA_ERR_CUDA, as a failed launch would.
 * kda_test_wait_timeout(iters, stream): launches one kernel that waits on a
 *   flag that nothing sets, giving up after `iters` polls (bounded); it then
 *   records KDA_ERR_TIMEOUT in the device status word and returns. */
void kda_test_fail_next_launches(int32_t n);
kda_status kda_test_wait_timeout(int32_t iters, kda_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H */
