// Affine state maps of token segments, for splitting one long sequence across
// workers (runtimewire, "The architecture is built around inference cost": a 1M-token
// context on a fixed-size recurrent state). Every step of the recurrence is affine in
// the state, S_t = A_t S_{t-1} + B_t with A_t = (I - beta_t k_t k_t^T) Diag(alpha_t), so a
// segment maps the state entering it to the state leaving it as S_out = M S_in + N
// (M = product of its A_t, d_k x d_k; N = its final state from zero). Maps compose as
// (M2, N2) o (M1, N1) = (M2 M1, M2 N1 + N2). This kernel is the one product both need:
//     out[i] = M[i] X[i] + N[i]      (N nullable = 0)
// with M [n, dk, dk], X, N, out [n, dk, dv], fp32 throughout (CUDA-core FMA: the state
// carries across many segments, and tf32 tensor cores would round it to 10 bits).
// One CTA (256 threads, 4 x 4 outputs per thread) per 64 x 64 tile of out[i].
#pragma once
#include "common.cuh"

namespace kda {

struct StateMapParams {
    const float *M, *X, *N;
    float *out;
    int64_t n;
    int32_t dk, dv;
};

__global__ void __launch_bounds__(256) state_map_kernel(const __grid_constant__ StateMapParams P) {
    __shared__ float Ms[64][33];          // rows of M, a 32-wide k slice (padded)
    __shared__ __align__(16) float Xs[32][64];
    const int dk = P.dk, dv = P.dv;
    const int tiles_r = (dk + 63) / 64, tiles_c = (dv + 63) / 64;
    const int64_t item = blockIdx.x / (tiles_r * tiles_c);
    const int tile = blockIdx.x % (tiles_r * tiles_c);
    const int r0 = (tile / tiles_c) * 64, c0 = (tile % tiles_c) * 64;
    const float *M = P.M + item * dk * dk;
    const float *X = P.X + item * dk * dv;
    const int t = threadIdx.x, tr = t / 16, tc = t % 16;      // 16 x 16 threads, 4 x 4 each
    float acc[4][4] = {};
    for (int k0 = 0; k0 < dk; k0 += 32) {
        for (int e = t; e < 64 * 32; e += 256) {
            const int r = e / 32, k = e % 32;
            Ms[r][k] = (r0 + r < dk && k0 + k < dk) ? M[(int64_t)(r0 + r) * dk + k0 + k] : 0.f;
        }
        for (int e = t; e < 32 * 64; e += 256) {
            const int k = e / 64, c = e % 64;
            Xs[k][c] = (k0 + k < dk && c0 + c < dv) ? X[(int64_t)(k0 + k) * dv + c0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Ms[tr + 16 * i][k];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Xs[k][tc + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + tr + 16 * i;
        if (r >= dk) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + tc + 16 * j;
            if (c >= dv) continue;
            const int64_t off = item * dk * dv + (int64_t)r * dv + c;
            P.out[off] = acc[i][j] + (P.N ? P.N[off] : 0.f);
        }
    }
}

}  // namespace kda
