/*
 * Oracle for the two steps around the gated delta rule in the GDN token mixer:
 * the causal depthwise convolution with SiLU in front of it and the gated
 * RMSNorm after it. Plain, sequential fp64 CPU code.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path (the
 * CUDA library) shares no code with it and never calls it.
 *
 * Sources:
 *   "Qwen3.5-MoE-35B-A3B architecture teardown", section 3.3 phase 2 (the
 *   concatenated q/k/v channels go through a depthwise causal convolution of
 *   kernel size 4 with SiLU) and phase 4 (the output is RMSNorm(o) * SiLU(z));
 *   section 3.4 (the conv cache holds conv_dim x (kernel_size - 1) values per
 *   sequence);
 *   "Qwen3.5 observation notes", "Qwen3_5MoeGatedDeltaNet" (causal_conv1d with
 *   weight [conv_dim, K], optional bias, activation silu; prefill keeps the last
 *   tokens of the input as the conv cache and decode slides it by one token;
 *   RMSNormGated = RMSNorm, then times SiLU(z)).
 *
 * Readings where the pages are silent:
 *   - conv cache layout: [N][K-1][conv_dim], oldest position first; absent =>
 *     zeros before each sequence's first token (causal zero padding);
 *   - the convolution aligns the kernel's last tap with the current token:
 *     y[t][c] = silu(bias[c] + sum_{i=0}^{K-1} w[c][i] * x[t - (K-1) + i][c]);
 *   - RMSNorm epsilon 1e-6 inside the square root and a per-element weight of
 *     length d shared by all heads: y = o / sqrt(mean(o^2) + eps) * w * silu(z).
 *
 * Build: compiled together with gdn_oracle.c into liboracle.so.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double oracle_silu(double x) { return x / (1.0 + exp(-x)); }

/*
 * Causal depthwise convolution + SiLU over a packed batch.
 *   x          [T][C]           input (the concatenated q/k/v channels)
 *   w          [C][K]           per-channel taps, w[c][K-1] multiplies the current token
 *   bias       [C] or NULL
 *   state_in   [N][K-1][C] or NULL (zeros): the K-1 positions before each sequence
 *   cu_seqlens [N+1]
 *   y          [T][C]           output
 *   state_out  [N][K-1][C] or NULL: the K-1 positions ending at each sequence's
 *              last token (from state_in where the sequence is shorter than K-1)
 */
void oracle_conv1d_silu(const double* x, const double* w, const double* bias,
                        const double* state_in, const int64_t* cu_seqlens, int32_t N,
                        int32_t C, int32_t K, double* y, double* state_out) {
    const int32_t W = K - 1;
#pragma omp parallel for schedule(dynamic)
    for (int64_t nc = 0; nc < (int64_t)N * C; ++nc) {
        const int32_t n = (int32_t)(nc / C), c = (int32_t)(nc % C);
        const int64_t s0 = cu_seqlens[n], s1 = cu_seqlens[n + 1];
        /* value at position p relative to the sequence start (p < 0: the cache) */
        #define XAT(p) ((p) >= 0 ? x[(s0 + (p)) * C + c] \
                                 : (state_in ? state_in[((int64_t)n * W + (W + (p))) * C + c] : 0.0))
        for (int64_t t = 0; t < s1 - s0; ++t) {
            double acc = bias ? bias[c] : 0.0;
            for (int32_t i = 0; i < K; ++i) acc += w[(int64_t)c * K + i] * XAT(t - (K - 1) + i);
            y[(s0 + t) * C + c] = oracle_silu(acc);
        }
        if (state_out) {
            const int64_t L = s1 - s0;
            for (int32_t j = 0; j < W; ++j) state_out[((int64_t)n * W + j) * C + c] = XAT(L - W + j);
        }
        #undef XAT
    }
}

/*
 * Gated RMSNorm over rows of length d:
 *   y[r][:] = o[r][:] / sqrt(mean(o[r][:]^2) + eps) * w[:] * silu(z[r][:])
 */
void oracle_rmsnorm_gated(const double* o, const double* z, const double* w, double eps,
                          int64_t rows, int32_t d, double* y) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int32_t e = 0; e < d; ++e) ss += o[r * d + e] * o[r * d + e];
        const double inv = 1.0 / sqrt(ss / d + eps);
        for (int32_t e = 0; e < d; ++e)
            y[r * d + e] = o[r * d + e] * inv * w[e] * oracle_silu(z[r * d + e]);
    }
}
