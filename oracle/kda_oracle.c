/*
 * KDA oracle: the plain fp64 token-by-token recurrence, on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py load this file's library. It shares no code with the
 * CUDA library and must never be reached from the product path.
 *
 * Definition followed (Kimi K3 technical FAQ, "What is KDA, and why does a
 * serving engineer care?": a delta-rule linear-attention recurrence with a
 * per-channel forget gate and a d_k x d_v state per head; written in the
 * standard gated-delta form):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t * scale            (scale = 1/sqrt(d_k) by default)
 *
 * with alpha_t = exp(g_t) per key channel. Each token is evaluated as
 *     S <- Diag(exp g_t) S ;  x = S^T k_t ;  S <- S + beta_t k_t (v_t - x)^T ;
 *     o_t = scale * S^T q_t
 * which equals the line above exactly in real arithmetic.
 *
 * State snapshots (vLLM day-0 blog, "Kimi Delta Attention": recurrent state is
 * reused from snapshots taken at block boundaries): with start_pos tokens
 * already absorbed by the initial state, the state after absolute position p is
 * recorded whenever p % snap_interval == 0, for start_pos < p <= start_pos + T,
 * in ascending p.
 *
 * Inputs are fp32 arrays (the exact values the GPU receives, widened); every
 * operation is fp64. OpenMP runs independent heads in parallel; within a head
 * the token order is the definition's order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void store(void *base, int out_f32, int64_t idx, double x) {
    if (out_f32) ((float *)base)[idx] = (float)x;
    else ((double *)base)[idx] = x;
}

/*
 * One sequence of T tokens, all H heads.
 *   q, k, g : [T, H, dk] fp32     v : [T, H, dv] fp32     beta : [T, H] fp32
 *   s0      : [H, dk, dv] initial state (fp32, or fp64 when s0_f64 != 0),
 *             or NULL for zeros
 *   o       : [T, H, dv]          s_final : [H, dk, dv]
 *   snaps   : [n_snap, H, dk, dv] or NULL (n_snap from the rule above)
 * Outputs are double, or float when out_f32 != 0. Returns the snapshot count.
 */
int64_t kda_oracle_sequence(int64_t T, int H, int dk, int dv,
                            const float *q, const float *k, const float *v,
                            const float *g, const float *beta, const void *s0,
                            int s0_f64, double scale, int64_t start_pos, int64_t snap_interval,
                            void *o, void *s_final, void *snaps, int out_f32,
                            int n_threads) {
    int64_t n_snap = 0;
    if (snap_interval > 0)
        n_snap = (start_pos + T) / snap_interval - start_pos / snap_interval;
    if (n_threads > 0) {
#ifdef _OPENMP
        omp_set_num_threads(n_threads);
#endif
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *x = (double *)malloc(sizeof(double) * (size_t)dv);
        double *kk = (double *)malloc(sizeof(double) * (size_t)dk);
        int64_t snap_no = 0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] =
                    !s0 ? 0.0
                        : s0_f64 ? ((const double *)s0)[((size_t)h * dk + i) * dv + j]
                                 : (double)((const float *)s0)[((size_t)h * dk + i) * dv + j];
        for (int64_t t = 0; t < T; ++t) {
            const float *qt = q + ((size_t)t * H + h) * dk;
            const float *kt = k + ((size_t)t * H + h) * dk;
            const float *gt = g + ((size_t)t * H + h) * dk;
            const float *vt = v + ((size_t)t * H + h) * dv;
            double b = (double)beta[(size_t)t * H + h];
            /* S <- Diag(alpha_t) S */
            for (int i = 0; i < dk; ++i) {
                double a = exp((double)gt[i]);
                kk[i] = (double)kt[i];
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
            }
            /* x = S^T k_t */
            for (int j = 0; j < dv; ++j) x[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) x[j] += S[(size_t)i * dv + j] * kk[i];
            /* S <- S + beta k (v - x)^T */
            for (int j = 0; j < dv; ++j) x[j] = b * ((double)vt[j] - x[j]);
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += kk[i] * x[j];
            /* o_t = scale * S^T q_t */
            for (int j = 0; j < dv; ++j) x[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                double qi = (double)qt[i];
                for (int j = 0; j < dv; ++j) x[j] += S[(size_t)i * dv + j] * qi;
            }
            for (int j = 0; j < dv; ++j)
                store(o, out_f32, ((int64_t)t * H + h) * dv + j, scale * x[j]);
            /* snapshot after absolute position p */
            int64_t p = start_pos + t + 1;
            if (snaps && snap_interval > 0 && p % snap_interval == 0) {
                int64_t base = ((snap_no * H + h) * (int64_t)dk) * dv;
                for (int64_t e = 0; e < (int64_t)dk * dv; ++e) store(snaps, out_f32, base + e, S[e]);
                ++snap_no;
            }
        }
        for (int64_t e = 0; e < (int64_t)dk * dv; ++e)
            store(s_final, out_f32, (int64_t)h * dk * dv + e, S[e]);
        free(S);
        free(x);
        free(kk);
    }
    return n_snap;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
