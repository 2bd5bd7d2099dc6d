// libkda: the C ABI of the KDA hot path (declared in include/kda.h).
//
// Host side: argument validation (every error returns before any launch), the
// ragged-batch plan (snapshot rows, longest-first sequence order, launches of
// at most KDA_SEQS_PER_LAUNCH sequences), kernel dispatch and the device
// status word. All kernels of the library live in this translation unit.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <numeric>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "frontend.cuh"
#include "prefill_simt.cuh"
#include "prefill_tc.cuh"
#include "prefill_split.cuh"
#include "snapshot.cuh"
#include "statemap.cuh"

namespace kda {

static std::atomic<int64_t> g_launches{0};
static std::atomic<int32_t> g_fail_next{0};

static kda_status cuda_fail(cudaError_t e) { return fail_cuda(e); }

// Count a launch, or simulate a failed one (failure-injection hook; the caller then
// reports KDA_ERR_CUDA, whose text says the launch was not issued).
static bool launch_gate() {
    int32_t n = g_fail_next.load();
    while (n > 0) {
        if (g_fail_next.compare_exchange_weak(n, n - 1)) {
            fail_text("launch not issued (failure injection)");
            return false;
        }
    }
    g_launches.fetch_add(1);
    return true;
}

static kda_status last_launch_status() { return launch_result(); }

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static kda_status check_dims(const kda_dims *d, bool need_chunk) {
    if (!d) return KDA_ERR_INVALID;
    if (d->H < 1 || d->dk < 1 || d->dv < 1) return KDA_ERR_INVALID;
    if (d->io != KDA_IO_BF16 && d->io != KDA_IO_FP32) return KDA_ERR_INVALID;
    if (!std::isfinite(d->scale)) return KDA_ERR_INVALID;
    if (d->dk != d->dv) return KDA_ERR_UNSUPPORTED;
    if (d->dk != 32 && d->dk != 64 && d->dk != 128) return KDA_ERR_UNSUPPORTED;
    if (need_chunk && d->chunk != 16 && d->chunk != 32 && d->chunk != 64) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

static float eff_scale(const kda_dims *d) {
    return d->scale != 0.f ? d->scale : 1.0f / std::sqrt((float)d->dk);
}

// ---------------------------------------------------------------- decode ----
template <int D, typename TIO>
static kda_status launch_decode(DecodeParams &p, int n_blocks, cudaStream_t st) {
    if (!launch_gate()) return KDA_ERR_CUDA;
    if (p.taps > 0) decode_kernel<D, TIO, true><<<n_blocks, DecodeShape<D>::NT, 0, st>>>(p);
    else decode_kernel<D, TIO, false><<<n_blocks, DecodeShape<D>::NT, 0, st>>>(p);
    return last_launch_status();
}

template <typename TIO>
static kda_status dispatch_decode(int D, DecodeParams &p, int n_blocks, cudaStream_t st) {
    switch (D) {
    case 32: return launch_decode<32, TIO>(p, n_blocks, st);
    case 64: return launch_decode<64, TIO>(p, n_blocks, st);
    case 128: return launch_decode<128, TIO>(p, n_blocks, st);
    }
    return KDA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------- verify, verify + commit ----
constexpr int kMaxDevices = 64;     // devices whose scratch address is cached

static int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static std::atomic<int> cache[kMaxDevices];
    int n = dev < kMaxDevices ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Token rows of one packed [rows, H, D] array as a 3-D tensor (channel, head, row) read
// in boxes of D channels x 1 head x `box_rows` rows. An empty or absent array gets a
// zeroed map, which no launch then reads.
static bool encode_rows(CUtensorMap *m, const void *base, bool bf16, int D, int H, int64_t rows, int box_rows) {
    std::memset(m, 0, sizeof(*m));
    if (!base || rows <= 0) return true;
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es};
    cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// sequences by decreasing token count (this step's, plus the previous step's as the bound
// on the replayed prefix), for the kernel's balanced item order; stable, so equal counts
// keep their order
static void order_by_tokens(SpecParams &P, int ng, const int32_t *tok0, const int32_t *prev0) {
    static thread_local std::vector<int32_t> cost;
    cost.resize(ng);
    for (int s = 0; s < ng; ++s)
        cost[s] = tok0[s + 1] - tok0[s] + (prev0 ? prev0[s + 1] - prev0[s] : 0);
    std::iota(P.order, P.order + ng, 0);
    std::stable_sort(P.order, P.order + ng, [&](int32_t a, int32_t b) { return cost[a] > cost[b]; });
}

template <int D, typename TIO, bool CONV, bool COMMIT>
static kda_status launch_spec_t(SpecParams &P, cudaStream_t st) {
    using SM = SpecSmem<D, TIO, CONV>;
    const void *fn = (const void *)spec_kernel<D, TIO, CONV, COMMIT>;
    static std::atomic<unsigned long long> attr{0};
    static std::atomic<int> occ_cache{0};
    kda_status r = set_smem_limit_once(fn, (int)SM::BYTES, attr);
    if (r != KDA_OK) return r;
    int occ = occ_cache.load(std::memory_order_relaxed);
    if (occ == 0) {
        const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, DecodeShape<D>::NT, SM::BYTES);
        if (e != cudaSuccess) return fail_cuda(e);
        if (occ < 1) return fail_text("the verify kernel does not fit on an SM");
        occ_cache.store(occ, std::memory_order_relaxed);
    }
    const int sms = sm_count();
    if (sms < 1) return fail_text("no multiprocessor count");
    // verify + commit: resident CTAs on every SM (more when a CTA would hold more than
    // SpecItems::N items), each walking its share of the items with the next state
    // prefetched. verify: one CTA per item, longest sequences first; its per-token state
    // writes keep HBM busy, and the hardware's block scheduler balances the tail (measured:
    // 0.96 of HBM against 0.81 for the persistent grid)
    const int64_t n_items = P.n_items;
    constexpr int64_t NI = SpecItems<CONV>::N;
    const int64_t grid = !COMMIT ? n_items
                                 : std::max<int64_t>(1, std::min<int64_t>(n_items, std::max<int64_t>(
                                                                                    (int64_t)occ * sms,
                                                                                    (n_items + NI - 1) / NI)));
    if (!launch_gate()) return KDA_ERR_CUDA;
    spec_kernel<D, TIO, CONV, COMMIT><<<(unsigned)grid, DecodeShape<D>::NT, SM::BYTES, st>>>(P);
    return last_launch_status();
}

// verify (commit false) or verify + commit over one group of sequences; T and Tp: rows of
// this step's and the previous step's packed token arrays
template <typename TIO>
static kda_status launch_spec(int D, SpecParams &P, bool commit, int64_t T, int64_t Tp, cudaStream_t st) {
    if (D != 32 && D != 64 && D != 128) return KDA_ERR_UNSUPPORTED;
    constexpr bool bf = sizeof(TIO) == 2;
    constexpr int TB = SpecShape<TIO>::TB;
    const DecodeParams &p = P.p;
    const CommitParams &c = P.c;
    const int H = p.H;
    if (!encode_rows(&P.mq, p.q, bf, D, H, T, TB) || !encode_rows(&P.mk, p.k, bf, D, H, T, TB) ||
        !encode_rows(&P.mv, p.v, bf, D, H, T, TB) || !encode_rows(&P.mg, p.g, false, D, H, T, TB) ||
        !encode_rows(&P.pq, commit ? c.q : nullptr, bf, D, H, Tp, TB) ||
        !encode_rows(&P.pk, commit ? c.k : nullptr, bf, D, H, Tp, TB) ||
        !encode_rows(&P.pv, commit ? c.v : nullptr, bf, D, H, Tp, TB) ||
        !encode_rows(&P.pg, commit ? c.g : nullptr, false, D, H, Tp, TB))
        return fail_text("cuTensorMapEncodeTiled failed for the token rows");
    const bool conv = p.taps > 0;
#define KDA_SPEC(d)                                                                                  \
    if (commit) return conv ? launch_spec_t<d, TIO, true, true>(P, st) : launch_spec_t<d, TIO, false, true>(P, st); \
    return conv ? launch_spec_t<d, TIO, true, false>(P, st) : launch_spec_t<d, TIO, false, false>(P, st);
    switch (D) {
    case 32: KDA_SPEC(32)
    case 64: KDA_SPEC(64)
    default: KDA_SPEC(128)
    }
#undef KDA_SPEC
}

// --------------------------------------------------------------- prefill ----
template <int D, int C, typename TIO>
static kda_status launch_simt(const PrefillParams &p, cudaStream_t st) {
    using Sh = SimtShape<D, C>;
    static std::atomic<unsigned long long> attr_done{0};
    const kda_status st_attr = set_smem_limit_once((const void *)prefill_simt_kernel<D, C, TIO>,
                                                   (int)Sh::smem_bytes, attr_done);
    if (st_attr != KDA_OK) return st_attr;
    if (!launch_gate()) return KDA_ERR_CUDA;
    prefill_simt_kernel<D, C, TIO><<<p.n_items, Sh::NT, Sh::smem_bytes, st>>>(p);
    return last_launch_status();
}

template <typename TIO>
static kda_status dispatch_simt(int D, int C, const PrefillParams &p, cudaStream_t st) {
#define KDA_CASE(d, c) \
    if (D == d && C == c) return launch_simt<d, c, TIO>(p, st);
    KDA_CASE(32, 16) KDA_CASE(32, 32) KDA_CASE(32, 64)
    KDA_CASE(64, 16) KDA_CASE(64, 32) KDA_CASE(64, 64)
    KDA_CASE(128, 16) KDA_CASE(128, 32) KDA_CASE(128, 64)
#undef KDA_CASE
    return KDA_ERR_UNSUPPORTED;
}

template <int D, typename TIO>
static kda_status launch_frontend(const FrontendParams &P, int64_t n_items, cudaStream_t st) {
    using Sh = FrontendShape<D>;
    if (!launch_gate()) return KDA_ERR_CUDA;
    const unsigned grid = (unsigned)((n_items + Sh::WARPS - 1) / Sh::WARPS);
    switch (P.taps) {
    case 2: qk_frontend_kernel<D, TIO, 2><<<grid, Sh::NT, 0, st>>>(P); break;
    case 3: qk_frontend_kernel<D, TIO, 3><<<grid, Sh::NT, 0, st>>>(P); break;
    default: qk_frontend_kernel<D, TIO, 4><<<grid, Sh::NT, 0, st>>>(P); break;
    }
    return last_launch_status();
}

// Forced path selection for tests: 0 = automatic, 1 = CUDA-core path only.
static std::atomic<int> g_prefill_path{0};

// Scratch of kda_prefill_noalloc: a fixed module-level device array, so that call needs
// neither an allocation nor a caller buffer. Its size bounds the workspaces it can serve.
constexpr size_t kNoallocScratchBytes = size_t(64) << 20;
__device__ __align__(1024) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

}  // namespace kda

using namespace kda;

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID: return "KDA_ERR_INVALID: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported dimensions";
    case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN: device pointer not 16-byte aligned";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace smaller than kda_prefill_workspace_size";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA call or launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: device wait ran out of iterations";
    case KDA_ERR_RANGE: return "KDA_ERR_RANGE: device-side range check failed";
    }
    return "KDA_ERR_UNKNOWN";
}

int64_t kda_launch_count(void) { return g_launches.load(); }

void kda_test_fail_next_launches(int32_t n) { g_fail_next.store(n > 0 ? n : 0); }

kda_status kda_snapshot_plan(int32_t n_seq, const int32_t *cu, const int64_t *start_pos,
                             int32_t snap_interval, int64_t *offsets, int64_t *positions) {
    if (n_seq < 0 || !cu || !offsets || snap_interval < 0) return KDA_ERR_INVALID;
    if (cu[0] != 0) return KDA_ERR_INVALID;
    for (int s = 0; s < n_seq; ++s) {
        if (cu[s + 1] < cu[s]) return KDA_ERR_INVALID;
        if (start_pos && start_pos[s] < 0) return KDA_ERR_INVALID;
    }
    int64_t total = 0;
    offsets[0] = 0;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t p0 = start_pos ? start_pos[s] : 0, len = cu[s + 1] - cu[s];
        int64_t cnt = 0;
        if (snap_interval > 0) {
            cnt = (p0 + len) / snap_interval - p0 / snap_interval;
            if (positions) {
                int64_t p = (p0 / snap_interval + 1) * snap_interval;
                for (int64_t j = 0; j < cnt; ++j, p += snap_interval) positions[total + j] = p;
            }
        }
        total += cnt;
        offsets[s + 1] = total;
    }
    return KDA_OK;
}

kda_status kda_prefill_workspace_size(const kda_dims *dims, int32_t n_seq, const int32_t *cu,
                                      size_t *bytes) {
    if (!bytes) return KDA_ERR_INVALID;
    *bytes = 0;
    kda_status st = check_dims(dims, true);
    if (st != KDA_OK) return st;
    if (n_seq < 0) return KDA_ERR_INVALID;
    if (n_seq == 0) return KDA_OK;
    if (!cu || cu[0] != 0) return KDA_ERR_INVALID;
    for (int s = 0; s < n_seq; ++s)
        if (cu[s + 1] < cu[s]) return KDA_ERR_INVALID;
    if (!tc_prefill_supported(*dims)) return KDA_OK;   // the CUDA-core path uses none
    size_t need = 0;
    for (int g0 = 0; g0 < n_seq; g0 += kPrefillSeqs) {
        const int ng = std::min(kPrefillSeqs, n_seq - g0);
        need = std::max(need, split_group_bytes((int64_t)cu[g0 + ng] - cu[g0], ng, dims->H));
    }
    *bytes = need;
    return KDA_OK;
}

kda_status kda_prefill(const kda_dims *dims, int32_t n_seq, const int32_t *cu,
                       const int64_t *start_pos, const void *q, const void *k, const void *v,
                       const float *g, const float *beta, const float *state_in,
                       float *state_out, void *o, int32_t snap_interval, float *snapshots,
                       void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    kda_status st = check_dims(dims, true);
    if (st != KDA_OK) return st;
    if (n_seq < 0 || snap_interval < 0) return KDA_ERR_INVALID;
    if (n_seq == 0) return KDA_OK;
    if (!cu) return KDA_ERR_INVALID;
    const int C = dims->chunk, D = dims->dk, H = dims->H;
    std::vector<int64_t> offs(n_seq + 1);
    st = kda_snapshot_plan(n_seq, cu, start_pos, snap_interval, offs.data(), nullptr);
    if (st != KDA_OK) return st;
    if (snap_interval > 0) {
        if (snap_interval % C != 0) return KDA_ERR_INVALID;
        for (int s = 0; s < n_seq && start_pos; ++s)
            if (start_pos[s] % C != 0) return KDA_ERR_INVALID;
    }
    const int64_t T = cu[n_seq];
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID;
    if (offs[n_seq] > 0 && !snapshots) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, g, beta, state_in, state_out, o, snapshots, workspace};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;

    // longest-first order: the hardware block scheduler hands out CTAs in
    // index order, so long chains start first and short ones fill the tail.
    std::vector<int> order(n_seq);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return cu[a + 1] - cu[a] > cu[b + 1] - cu[b]; });

    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const bool tc = g_prefill_path.load() == 0 && tc_prefill_supported(*dims);
    const bool split = tc && workspace != nullptr;
    if (split) {
        size_t need = 0;
        st = kda_prefill_workspace_size(dims, n_seq, cu, &need);
        if (st != KDA_OK) return st;
        if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
    }
    static thread_local PrefillParams p;  // ~27 KB: keep it off the stack
    for (int g0 = 0; g0 < n_seq; g0 += kPrefillSeqs) {
        const int ng = std::min(kPrefillSeqs, n_seq - g0);
        std::memset(&p, 0, sizeof(p));
        p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.o = o; p.snapshots = snapshots;
        const int64_t state_stride = (int64_t)H * D * D;
        p.state_in = state_in ? state_in + g0 * state_stride : nullptr;
        p.state_out = state_out ? state_out + g0 * state_stride : nullptr;
        p.H = H; p.n_seq = ng; p.snap_interval = snap_interval; p.scale = eff_scale(dims);
        int r = 0;
        for (int idx : order)
            if (idx >= g0 && idx < g0 + ng) p.order[r++] = (int16_t)(idx - g0);
        for (int i = 0; i < ng; ++i) {
            const int s = g0 + i;
            p.seq[i].tok0 = cu[s];
            p.seq[i].len = cu[s + 1] - cu[s];
            p.seq[i].start_pos = start_pos ? start_pos[s] : 0;
            p.seq[i].snap_off = offs[s];
        }
        if (split) {
            st = launch_prefill_split(p, *dims, T, cu[g0], cu[g0 + ng], offs[n_seq], workspace, cs,
                                      launch_gate);
        } else if (tc) {
            st = launch_prefill_tc(p, *dims, T, cs, launch_gate);
        } else {
            p.n_items = ng * H * (D / SimtShape<32, 16>::DVS);
            st = dims->io == KDA_IO_BF16 ? dispatch_simt<__nv_bfloat16>(D, C, p, cs)
                                         : dispatch_simt<float>(D, C, p, cs);
        }
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

// The fixed scratch's device address on the current device, looked up on the first call
// that needs it there (host code only sees a stand-in for the symbol).
static kda_status noalloc_scratch(void **scratch) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    static std::atomic<void *> addr[kMaxDevices];
    *scratch = dev < kMaxDevices ? addr[dev].load(std::memory_order_acquire) : nullptr;
    if (!*scratch) {
        e = cudaGetSymbolAddress(scratch, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        if (dev < kMaxDevices) addr[dev].store(*scratch, std::memory_order_release);
    }
    return KDA_OK;
}

// One sub-call of a prefill that does not fit the scratch: sequences [s0, s1) whole, or
// tokens [a, b) of sequence s0 alone (s1 = -1).
struct PrefillPiece {
    int s0, s1;
    int64_t a, b;
};

// kda_prefill_noalloc when the call's packets exceed the scratch: consecutive sequences
// are grouped while their packets fit; a sequence that alone exceeds it runs in windows of
// whole chunks, its state handed from one window to the next through two state buffers at
// the end of the scratch (fp32, exact), so that the chunks, and the results, are those of
// one call with a workspace. Returns KDA_ERR_UNSUPPORTED, with nothing launched, when a
// piece's beta would not be 16-byte aligned (H not a multiple of 4); the caller then runs
// the single-launch path.
static kda_status prefill_pieces(const kda_dims *dims, int32_t n_seq, const int32_t *cu,
                                 const int64_t *start_pos, const void *q, const void *k,
                                 const void *v, const float *g, const float *beta,
                                 const float *state_in, float *state_out, void *o,
                                 int32_t snap_interval, float *snapshots, void *scratch,
                                 kda_stream_t stream) {
    const int C = dims->chunk, H = dims->H, dk = dims->dk, dv = dims->dv;
    const size_t state_bytes = (size_t)H * dk * dv * 4;
    if (kNoallocScratchBytes < 2 * state_bytes) return KDA_ERR_UNSUPPORTED;
    const size_t cap = kNoallocScratchBytes - 2 * state_bytes;
    const int64_t max_rows = (int64_t)(cap / ((size_t)H * spl::PACKET));
    if (max_rows < 2) return KDA_ERR_UNSUPPORTED;
    // the argument checks of kda_prefill, before anything is launched
    std::vector<int64_t> offs(n_seq + 1);
    kda_status st = kda_snapshot_plan(n_seq, cu, start_pos, snap_interval, offs.data(), nullptr);
    if (st != KDA_OK) return st;
    if (snap_interval > 0) {
        if (snap_interval % C != 0) return KDA_ERR_INVALID;
        for (int s = 0; s < n_seq && start_pos; ++s)
            if (start_pos[s] % C != 0) return KDA_ERR_INVALID;
    }
    const int64_t T = cu[n_seq];
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID;
    if (offs[n_seq] > 0 && !snapshots) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, g, beta, state_in, state_out, o, snapshots};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    // the plan
    std::vector<PrefillPiece> plan;
    const int64_t wtok = (max_rows - 1) * C;          // a window's tokens: (wtok >> 6) + 1 rows
    for (int s = 0; s < n_seq;) {
        const int64_t len = cu[s + 1] - cu[s];
        if ((len >> 6) + 1 > max_rows) {
            for (int64_t a = 0; a < len; a += wtok) plan.push_back({s, -1, a, std::min(len, a + wtok)});
            ++s;
            continue;
        }
        int s1 = s;
        int64_t tok = 0;
        while (s1 < n_seq && s1 - s < kPrefillSeqs) {
            const int64_t l1 = cu[s1 + 1] - cu[s1];
            if (((tok + l1) >> 6) + (s1 - s + 1) > max_rows) break;
            tok += l1;
            ++s1;
        }
        plan.push_back({s, s1, 0, 0});
        s = s1;
    }
    const int64_t beta_row = (int64_t)H * 4;
    for (const PrefillPiece &pc : plan) {
        const int64_t row0 = cu[pc.s0] + (pc.s1 < 0 ? pc.a : 0);
        if ((row0 * beta_row) % 16 != 0) return KDA_ERR_UNSUPPORTED;
    }
    // the pieces, in order on the stream
    const size_t io = dims->io == KDA_IO_BF16 ? 2 : 4;
    const int64_t qrow = (int64_t)H * dk * io, vrow = (int64_t)H * dv * io, grow = (int64_t)H * dk * 4;
    const int64_t srow = (int64_t)H * dk * dv;                 // floats per state or snapshot row
    auto at = [](const void *p, int64_t bytes) -> const uint8_t * {
        return p ? static_cast<const uint8_t *>(p) + bytes : nullptr;
    };
    float *buf[2] = {reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + cap),
                     reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + cap + state_bytes)};
    std::vector<int32_t> cu2;
    std::vector<int64_t> start2;
    int w = 0;                                                  // window index within its sequence
    for (const PrefillPiece &pc : plan) {
        const int s = pc.s0;
        if (pc.s1 >= 0) {
            const int n = pc.s1 - pc.s0;
            cu2.assign(n + 1, 0);
            for (int i = 0; i <= n; ++i) cu2[i] = cu[s + i] - cu[s];
            const int64_t r0 = cu[s];
            st = kda_prefill(dims, n, cu2.data(), start_pos ? start_pos + s : nullptr, at(q, r0 * qrow),
                             at(k, r0 * qrow), at(v, r0 * vrow), reinterpret_cast<const float *>(at(g, r0 * grow)),
                             reinterpret_cast<const float *>(at(beta, r0 * beta_row)),
                             state_in ? state_in + s * srow : nullptr, state_out ? state_out + s * srow : nullptr,
                             const_cast<uint8_t *>(at(o, r0 * vrow)), snap_interval,
                             snapshots ? snapshots + offs[s] * srow : nullptr, scratch, cap, stream);
            w = 0;
        } else {
            const int64_t len = cu[s + 1] - cu[s], p0 = start_pos ? start_pos[s] : 0;
            const int64_t r0 = cu[s] + pc.a;
            cu2.assign(2, 0);
            cu2[1] = (int32_t)(pc.b - pc.a);
            start2.assign(1, p0 + pc.a);
            const int64_t snap0 = offs[s] + (snap_interval > 0 ? (p0 + pc.a) / snap_interval - p0 / snap_interval : 0);
            const float *sin = pc.a == 0 ? (state_in ? state_in + s * srow : nullptr) : buf[(w + 1) & 1];
            float *sout = pc.b == len ? (state_out ? state_out + s * srow : nullptr) : buf[w & 1];
            st = kda_prefill(dims, 1, cu2.data(), start2.data(), at(q, r0 * qrow), at(k, r0 * qrow),
                             at(v, r0 * vrow), reinterpret_cast<const float *>(at(g, r0 * grow)),
                             reinterpret_cast<const float *>(at(beta, r0 * beta_row)), sin, sout,
                             const_cast<uint8_t *>(at(o, r0 * vrow)), snap_interval,
                             snapshots ? snapshots + snap0 * srow : nullptr, scratch, cap, stream);
            w = pc.b == len ? 0 : w + 1;
        }
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

kda_status kda_prefill_noalloc(const kda_dims *dims, int32_t n_seq, const int32_t *cu,
                               const int64_t *start_pos, const void *q, const void *k,
                               const void *v, const float *g, const float *beta,
                               const float *state_in, float *state_out, void *o,
                               int32_t snap_interval, float *snapshots, kda_stream_t stream) {
    size_t need = 0;
    kda_status st = kda_prefill_workspace_size(dims, n_seq, cu, &need);
    if (st != KDA_OK) return st;
    void *scratch = nullptr;
    if (need > 0) {
        st = noalloc_scratch(&scratch);
        if (st != KDA_OK) return st;
        if (need > kNoallocScratchBytes) {
            st = prefill_pieces(dims, n_seq, cu, start_pos, q, k, v, g, beta, state_in, state_out, o,
                                snap_interval, snapshots, scratch, stream);
            if (st != KDA_ERR_UNSUPPORTED) return st;
            scratch = nullptr;                        // the single-launch path
        }
    }
    return kda_prefill(dims, n_seq, cu, start_pos, q, k, v, g, beta, state_in, state_out, o,
                       snap_interval, snapshots, scratch, scratch ? kNoallocScratchBytes : 0, stream);
}

size_t kda_prefill_noalloc_capacity(void) { return kNoallocScratchBytes; }

static kda_status check_conv(const kda_conv *conv) {
    if (!conv) return KDA_OK;
    if (conv->taps < 2 || conv->taps > kMaxTaps || !conv->w_q || !conv->w_k) return KDA_ERR_INVALID;
    if (!aligned16(conv->w_q) || !aligned16(conv->w_k)) return KDA_ERR_ALIGN;
    return KDA_OK;
}

static void set_conv(DecodeParams &p, const kda_conv *conv, float *pool, float *tok) {
    p.taps = conv ? conv->taps : 0;
    p.wq = conv ? conv->w_q : nullptr;
    p.wk = conv ? conv->w_k : nullptr;
    p.conv = conv ? pool : nullptr;
    p.conv_tok = conv ? tok : nullptr;
}

static kda_status decode_impl(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                              const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const int32_t *slots, int32_t n_slots, float *pool,
                              float *conv_pool, void *o, kda_stream_t stream) {
    kda_status st = check_dims(dims, false);
    if (st != KDA_OK) return st;
    if ((st = check_conv(conv)) != KDA_OK) return st;
    if (n_seq < 0 || n_slots < 0) return KDA_ERR_INVALID;
    if (n_seq == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !slots || !pool || !o) return KDA_ERR_INVALID;
    if (conv && !conv_pool) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, g, beta, slots, pool, o, conv_pool};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    if ((int64_t)n_seq * dims->H > 0x7fffffffLL) return KDA_ERR_INVALID;
    static thread_local DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.slots = slots; p.pool = pool; p.o = o;
    p.n_seq = n_seq; p.H = dims->H; p.n_slots = n_slots; p.scale = eff_scale(dims);
    set_conv(p, conv, conv_pool, nullptr);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    return dims->io == KDA_IO_BF16
               ? dispatch_decode<__nv_bfloat16>(dims->dk, p, n_seq * dims->H, cs)
               : dispatch_decode<float>(dims->dk, p, n_seq * dims->H, cs);
}

kda_status kda_decode(const kda_dims *dims, int32_t n_seq, const void *q, const void *k,
                      const void *v, const float *g, const float *beta, const int32_t *slots,
                      int32_t n_slots, float *pool, void *o, kda_stream_t stream) {
    return decode_impl(dims, nullptr, n_seq, q, k, v, g, beta, slots, n_slots, pool, nullptr, o,
                       stream);
}

kda_status kda_decode_conv(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                           const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const int32_t *slots, int32_t n_slots,
                           float *pool, float *conv_pool, void *o, kda_stream_t stream) {
    if (!conv) return KDA_ERR_INVALID;
    return decode_impl(dims, conv, n_seq, q, k, v, g, beta, slots, n_slots, pool, conv_pool, o,
                       stream);
}

static kda_status verify_impl(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                              const int32_t *cu_draft, const void *q, const void *k, const void *v,
                              const float *g, const float *beta, const int32_t *slots,
                              int32_t n_slots, const float *pool, const float *conv_pool,
                              float *token_states, float *conv_tok, void *o, kda_stream_t stream) {
    kda_status st = check_dims(dims, false);
    if (st != KDA_OK) return st;
    if ((st = check_conv(conv)) != KDA_OK) return st;
    if (conv && !conv_pool) return KDA_ERR_INVALID;
    if (n_seq < 0 || n_slots < 0) return KDA_ERR_INVALID;
    if (n_seq == 0) return KDA_OK;
    if (!cu_draft || cu_draft[0] != 0) return KDA_ERR_INVALID;
    for (int s = 0; s < n_seq; ++s)
        if (cu_draft[s + 1] < cu_draft[s]) return KDA_ERR_INVALID;
    const int64_t T = cu_draft[n_seq];
    if (!slots || !pool) return KDA_ERR_INVALID;
    if (T > 0 && (!q || !k || !v || !g || !beta || !token_states || !o)) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, v, g, beta, slots, pool, token_states, o, conv_pool, conv_tok};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    static thread_local SpecParams P;
    for (int g0 = 0; g0 < n_seq; g0 += kMaxSeqsPerLaunch) {
        const int ng = std::min(kMaxSeqsPerLaunch, n_seq - g0);
        std::memset(&P, 0, sizeof(P));
        DecodeParams &p = P.p;
        p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.slots = slots + g0;
        p.pool = const_cast<float *>(pool); p.token_states = token_states; p.o = o;
        p.n_seq = ng; p.H = dims->H; p.n_slots = n_slots; p.scale = eff_scale(dims);
        p.tok_base = cu_draft[g0];
        set_conv(p, conv, const_cast<float *>(conv_pool), conv_tok);
        for (int i = 0; i <= ng; ++i) p.tok0[i] = cu_draft[g0 + i] - cu_draft[g0];
        if ((int64_t)ng * dims->H > 0x7fffffffLL) return KDA_ERR_INVALID;
        P.n_items = ng * dims->H;
        order_by_tokens(P, ng, p.tok0, nullptr);
        st = dims->io == KDA_IO_BF16 ? launch_spec<__nv_bfloat16>(dims->dk, P, false, T, 0, cs)
                                     : launch_spec<float>(dims->dk, P, false, T, 0, cs);
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

kda_status kda_verify(const kda_dims *dims, int32_t n_seq, const int32_t *cu_draft,
                      const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const int32_t *slots, int32_t n_slots,
                      const float *pool, float *token_states, void *o, kda_stream_t stream) {
    return verify_impl(dims, nullptr, n_seq, cu_draft, q, k, v, g, beta, slots, n_slots, pool,
                       nullptr, token_states, nullptr, o, stream);
}

kda_status kda_verify_conv(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                           const int32_t *cu_draft, const void *q, const void *k, const void *v,
                           const float *g, const float *beta, const int32_t *slots,
                           int32_t n_slots, const float *pool, const float *conv_pool,
                           float *token_states, float *conv_token_states, void *o,
                           kda_stream_t stream) {
    if (!conv) return KDA_ERR_INVALID;
    return verify_impl(dims, conv, n_seq, cu_draft, q, k, v, g, beta, slots, n_slots, pool,
                       conv_pool, token_states, conv_token_states, o, stream);
}

static kda_status verify_commit_impl(
    const kda_dims *dims, const kda_conv *conv, int32_t n_seq, const int32_t *cu_prev,
    const void *q_prev, const void *k_prev, const void *v_prev, const float *g_prev,
    const float *beta_prev, const int32_t *n_accept, const int64_t *pos, int32_t snap_interval,
    const int64_t *snap_row, float *snapshots, float *conv_snapshots, int64_t n_snap_rows,
    const int32_t *cu_draft, const void *q, const void *k, const void *v, const float *g,
    const float *beta, const uint8_t *commit_new, const int32_t *slots, int32_t n_slots,
    float *pool, float *conv_pool, void *o, kda_stream_t stream) {
    kda_status st = check_dims(dims, false);
    if (st != KDA_OK) return st;
    if ((st = check_conv(conv)) != KDA_OK) return st;
    if (conv && !conv_pool) return KDA_ERR_INVALID;
    if (n_seq < 0 || n_slots < 0 || snap_interval < 0 || n_snap_rows < 0) return KDA_ERR_INVALID;
    if (n_seq == 0) return KDA_OK;
    if (!cu_prev || !cu_draft || cu_prev[0] != 0 || cu_draft[0] != 0) return KDA_ERR_INVALID;
    for (int s = 0; s < n_seq; ++s)
        if (cu_prev[s + 1] < cu_prev[s] || cu_draft[s + 1] < cu_draft[s]) return KDA_ERR_INVALID;
    const int64_t Tp = cu_prev[n_seq], T = cu_draft[n_seq];
    if (!slots || !pool || !n_accept) return KDA_ERR_INVALID;
    if (Tp > 0 && (!k_prev || !v_prev || !g_prev || !beta_prev || (conv && !q_prev)))
        return KDA_ERR_INVALID;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID;
    if (snap_interval > 0 && snap_row && (!pos || !snapshots || (conv && !conv_snapshots)))
        return KDA_ERR_INVALID;
    const void *ptrs[] = {q_prev, k_prev, v_prev, g_prev, beta_prev, n_accept, pos, snap_row,
                          snapshots, conv_snapshots, q, k, v, g, beta, slots, pool, conv_pool, o,
                          commit_new};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    static thread_local SpecParams P;
    for (int g0 = 0; g0 < n_seq; g0 += kMaxSeqsPerLaunch) {
        const int ng = std::min(kMaxSeqsPerLaunch, n_seq - g0);
        std::memset(&P, 0, sizeof(P));
        DecodeParams &p = P.p;
        p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.slots = slots + g0;
        p.pool = pool; p.o = o;
        p.n_seq = ng; p.H = dims->H; p.n_slots = n_slots; p.scale = eff_scale(dims);
        p.tok_base = cu_draft[g0];
        for (int i = 0; i <= ng; ++i) p.tok0[i] = cu_draft[g0 + i] - cu_draft[g0];
        set_conv(p, conv, conv_pool, nullptr);
        CommitParams &c = P.c;
        c.q = conv ? q_prev : nullptr;
        c.conv_snapshots = conv ? conv_snapshots : nullptr;
        c.k = k_prev; c.v = v_prev; c.g = g_prev; c.beta = beta_prev;
        c.n_accept = n_accept + g0;
        c.pos = pos ? pos + g0 : nullptr;
        c.snap_row = (snap_interval > 0 && snap_row) ? snap_row + g0 : nullptr;
        c.commit_new = commit_new ? commit_new + g0 : nullptr;
        c.snapshots = snapshots; c.n_snap_rows = n_snap_rows; c.snap_interval = snap_interval;
        c.tok_base = cu_prev[g0];
        for (int i = 0; i <= ng; ++i) c.tok0[i] = cu_prev[g0 + i] - cu_prev[g0];
        if ((int64_t)ng * dims->H > 0x7fffffffLL) return KDA_ERR_INVALID;
        P.n_items = ng * dims->H;
        order_by_tokens(P, ng, p.tok0, c.tok0);
        st = dims->io == KDA_IO_BF16 ? launch_spec<__nv_bfloat16>(dims->dk, P, true, T, Tp, cs)
                                     : launch_spec<float>(dims->dk, P, true, T, Tp, cs);
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

kda_status kda_verify_commit(const kda_dims *dims, int32_t n_seq, const int32_t *cu_prev,
                             const void *k_prev, const void *v_prev, const float *g_prev,
                             const float *beta_prev, const int32_t *n_accept, const int64_t *pos,
                             int32_t snap_interval, const int64_t *snap_row, float *snapshots,
                             int64_t n_snap_rows, const int32_t *cu_draft, const void *q,
                             const void *k, const void *v, const float *g, const float *beta,
                             const uint8_t *commit_new, const int32_t *slots, int32_t n_slots,
                             float *pool, void *o, kda_stream_t stream) {
    return verify_commit_impl(dims, nullptr, n_seq, cu_prev, nullptr, k_prev, v_prev, g_prev,
                              beta_prev, n_accept, pos, snap_interval, snap_row, snapshots, nullptr,
                              n_snap_rows, cu_draft, q, k, v, g, beta, commit_new, slots, n_slots,
                              pool, nullptr, o, stream);
}

kda_status kda_verify_commit_conv(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                                  const int32_t *cu_prev, const void *q_prev, const void *k_prev,
                                  const void *v_prev, const float *g_prev, const float *beta_prev,
                                  const int32_t *n_accept, const int64_t *pos,
                                  int32_t snap_interval, const int64_t *snap_row,
                                  float *snapshots, float *conv_snapshots, int64_t n_snap_rows,
                                  const int32_t *cu_draft, const void *q, const void *k,
                                  const void *v, const float *g, const float *beta,
                                  const uint8_t *commit_new, const int32_t *slots,
                                  int32_t n_slots, float *pool, float *conv_pool, void *o,
                                  kda_stream_t stream) {
    if (!conv) return KDA_ERR_INVALID;
    return verify_commit_impl(dims, conv, n_seq, cu_prev, q_prev, k_prev, v_prev, g_prev,
                              beta_prev, n_accept, pos, snap_interval, snap_row, snapshots,
                              conv_snapshots, n_snap_rows, cu_draft, q, k, v, g, beta, commit_new,
                              slots, n_slots, pool, conv_pool, o, stream);
}

kda_status kda_qk_frontend(const kda_dims *dims, const kda_conv *conv, int32_t n_seq,
                           const int32_t *cu, const int64_t *start_pos, const void *q,
                           const void *k, const float *conv_in, float *conv_out, void *q_out,
                           void *k_out, int32_t snap_interval, float *conv_snapshots,
                           kda_stream_t stream) {
    kda_status st = check_dims(dims, true);
    if (st != KDA_OK) return st;
    if (!conv) return KDA_ERR_INVALID;
    if ((st = check_conv(conv)) != KDA_OK) return st;
    if (n_seq < 0 || snap_interval < 0) return KDA_ERR_INVALID;
    if (n_seq == 0) return KDA_OK;
    if (!cu) return KDA_ERR_INVALID;
    const int C = dims->chunk, D = dims->dk, H = dims->H;
    std::vector<int64_t> offs(n_seq + 1);
    st = kda_snapshot_plan(n_seq, cu, start_pos, snap_interval, offs.data(), nullptr);
    if (st != KDA_OK) return st;
    if (snap_interval > 0) {
        if (snap_interval % C != 0) return KDA_ERR_INVALID;
        for (int s = 0; s < n_seq && start_pos; ++s)
            if (start_pos[s] % C != 0) return KDA_ERR_INVALID;
    }
    const int64_t T = cu[n_seq];
    if (T > 0 && (!q || !k || !q_out || !k_out)) return KDA_ERR_INVALID;
    if (offs[n_seq] > 0 && !conv_snapshots) return KDA_ERR_INVALID;
    const void *ptrs[] = {q, k, conv_in, conv_out, q_out, k_out, conv_snapshots};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    static thread_local FrontendParams P;
    const int64_t cstate = (int64_t)2 * H * D * (conv->taps - 1);
    for (int g0 = 0; g0 < n_seq; g0 += kPrefillSeqs) {
        const int ng = std::min(kPrefillSeqs, n_seq - g0);
        std::memset(&P, 0, sizeof(P));
        P.q = q; P.k = k; P.q_out = q_out; P.k_out = k_out; P.wq = conv->w_q; P.wk = conv->w_k;
        P.conv_in = conv_in ? conv_in + g0 * cstate : nullptr;
        P.conv_out = conv_out ? conv_out + g0 * cstate : nullptr;
        P.conv_snap = conv_snapshots;
        P.H = H; P.taps = conv->taps; P.n_seq = ng; P.C = C; P.tok_first = cu[g0];
        P.snap_interval = snap_interval;
        for (int i = 0; i < ng; ++i) {
            P.tok0[i] = cu[g0 + i];
            P.len[i] = cu[g0 + i + 1] - cu[g0 + i];
            P.start_pos[i] = start_pos ? start_pos[g0 + i] : 0;
            P.snap_off[i] = offs[g0 + i];
        }
        const int64_t rows = ((int64_t)cu[g0 + ng] - cu[g0]) / C + ng;
        if (2 * rows * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        const bool bf = dims->io == KDA_IO_BF16;
        switch (D) {
        case 32: st = bf ? launch_frontend<32, __nv_bfloat16>(P, 2 * rows * H, cs) : launch_frontend<32, float>(P, 2 * rows * H, cs); break;
        case 64: st = bf ? launch_frontend<64, __nv_bfloat16>(P, 2 * rows * H, cs) : launch_frontend<64, float>(P, 2 * rows * H, cs); break;
        default: st = bf ? launch_frontend<128, __nv_bfloat16>(P, 2 * rows * H, cs) : launch_frontend<128, float>(P, 2 * rows * H, cs); break;
        }
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

kda_status kda_snapshot(int32_t n, const int64_t *src_idx, const int64_t *dst_idx,
                        const float *src, int64_t n_src, float *dst, int64_t n_dst, int32_t H,
                        int32_t dk, int32_t dv, kda_stream_t stream) {
    if (n < 0 || n_src < 0 || n_dst < 0 || H < 1 || dk < 1 || dv < 1) return KDA_ERR_INVALID;
    if (n == 0) return KDA_OK;
    if (!src_idx || !dst_idx || !src || !dst) return KDA_ERR_INVALID;
    const int64_t elems = (int64_t)H * dk * dv;
    if (elems % 4 != 0) return KDA_ERR_UNSUPPORTED;
    const void *ptrs[] = {src_idx, dst_idx, src, dst};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return KDA_ERR_ALIGN;
    SnapshotParams p;
    p.src = src; p.dst = dst; p.n_src = n_src; p.n_dst = n_dst; p.elems4 = elems / 4;
    const int per_copy = (int)std::min<int64_t>(128, (p.elems4 + 1023) / 1024);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    for (int i0 = 0; i0 < n; i0 += 65535) {
        const int ni = std::min(65535, n - i0);
        p.src_idx = src_idx + i0;
        p.dst_idx = dst_idx + i0;
        if (!launch_gate()) return KDA_ERR_CUDA;
        snapshot_kernel<<<dim3(per_copy, ni), 256, 0, cs>>>(p);
        const kda_status st = last_launch_status();
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

kda_status kda_state_map_apply(int64_t n, int32_t dk, int32_t dv, const float *M, const float *X,
                               const float *N, float *out, kda_stream_t stream) {
    if (n < 0 || dk < 1 || dv < 1) return KDA_ERR_INVALID;
    if (n == 0) return KDA_OK;
    if (!M || !X || !out) return KDA_ERR_INVALID;
    if (out == X || out == M) return KDA_ERR_INVALID;      // out may alias N only
    const void *ptrs[] = {M, X, N, out};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    const int64_t tiles = (int64_t)((dk + 63) / 64) * ((dv + 63) / 64);
    if (n * tiles > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    StateMapParams p{M, X, N, out, n, dk, dv};
    if (!launch_gate()) return KDA_ERR_CUDA;
    state_map_kernel<<<(unsigned)(n * tiles), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
    return last_launch_status();
}

kda_status kda_check_device_status(kda_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e);
    if (v != 0) {
        e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return static_cast<kda_status>(v);
}

const char *kda_last_cuda_error(void) {
    return last_error_text().load();
}

// Forces the CUDA-core prefill path (1) or restores automatic selection (0).
// Not in the public header: used by the parity tests to check both paths.
void kda_internal_force_prefill_path(int32_t path) { g_prefill_path.store(path); }

}  // extern "C"

// ------------------------------------------------ failure-injection hook ----
namespace kda {
__device__ int g_never_set;

__global__ void wait_timeout_kernel(int32_t iters) {
    if (threadIdx.x != 0) return;
    volatile int *flag = &g_never_set;
    for (int32_t i = 0; i < iters; ++i) {
        if (*flag != 0) return;
        __nanosleep(1000);
    }
    record_status(KDA_ERR_TIMEOUT);
}
}  // namespace kda

extern "C" kda_status kda_test_wait_timeout(int32_t iters, kda_stream_t stream) {
    if (iters < 0) return KDA_ERR_INVALID;
    if (!launch_gate()) return KDA_ERR_CUDA;
    wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(iters);
    return last_launch_status();
}
