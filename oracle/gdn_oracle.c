/*
 * Gated DeltaNet oracle: plain, slow, sequential fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path (the
 * CUDA library) shares no code with it and never calls it.
 *
 * What it computes is the plain definition of the gated delta rule, one token
 * at a time, with no chunking, blocking or reordering:
 *
 *   "Qwen3.5-MoE-35B-A3B architecture teardown", section 3.3 (phase 3, the
 *   delta rule), section 3.4 (QK heads repeat_interleave'd over V heads) and
 *   section 3.7 step 1 (L2 norm of q and k, fp32 upcast);
 *   "Qwen3.5 observation notes", sections "DeltaNet" / "Gated DeltaNet" (read,
 *   delta, outer-product write) and "Qwen3_5MoeGatedDeltaNet" (beta =
 *   sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias), the state multiplied
 *   by exp(g) before the read, delta = (v - kv_mem) * beta).
 *
 * In the value-major orientation used throughout (S is d_v x d_k, o = S q):
 *
 *   S <- alpha_t * S                      (decay first)
 *   delta = beta_t * (v_t - S k_t)        (read with the decayed state)
 *   S <- S + delta k_t^T                  (write)
 *   o_t = S q_t                           (read-out after the write)
 *
 * which expands to S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 *
 * Readings where the pages are silent (all shared with the GPU path by
 * specification, never by code):
 *   - L2-norm epsilon: x / sqrt(sum x^2 + 1e-6).
 *   - softplus: the exact stable form max(x,0) + log1p(exp(-|x|)).
 *   - query scale: a plain multiplier on the normalised query (1.0 = none).
 *   - g is taken as 0 when softplus(...) == 0, so -inf * 0 never makes a NaN.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC gdn_oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_L2_EPS 1e-6

/* Exact, overflow-free softplus: log(1 + e^x). */
static double oracle_softplus(double x) {
    return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

/*
 * Gates, per token and V head ("Qwen3.5 observation notes", section
 * "Qwen3_5MoeGatedDeltaNet": beta is the sigmoid of b; g is minus exp(A_log)
 * times softplus(a + dt_bias), computed in float).
 *   a, b      [T, H_v]
 *   A_log, dt_bias [H_v]
 *   g, beta   [T, H_v]   (outputs; either may be NULL)
 */
void oracle_gates(const double* a, const double* b, const double* A_log,
                  const double* dt_bias, int64_t T, int32_t H_v,
                  double* g, double* beta) {
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t h = 0; h < H_v; ++h) {
            int64_t i = t * H_v + h;
            if (g) {
                double sp = oracle_softplus(a[i] + dt_bias[h]);
                g[i] = (sp > 0.0) ? -exp(A_log[h]) * sp : 0.0;
            }
            if (beta) beta[i] = 1.0 / (1.0 + exp(-b[i]));
        }
    }
}

/*
 * Inclusive cumulative sum of g inside each chunk of `chunk` tokens, with
 * chunk boundaries restarting at every sequence start ("Qwen3.5-MoE-35B-A3B
 * architecture teardown", section 3.7 step 3: the cumulative sum of g inside
 * each 64-token chunk).
 *   g, G  [T, H_v];  cu_seqlens [N+1]
 */
void oracle_chunk_cumsum(const double* g, const int64_t* cu_seqlens, int32_t N,
                         int32_t H_v, int32_t chunk, double* G) {
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H_v; ++h) {
            double acc = 0.0;
            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                if ((t - cu_seqlens[n]) % chunk == 0) acc = 0.0;
                acc += g[t * H_v + h];
                G[t * H_v + h] = acc;
            }
        }
    }
}

/*
 * The recurrence itself, given the gates g (log-decay) and beta directly.
 *   q, k   [T, H_qk, d_k]       v [T, H_v, d_v]
 *   g, beta [T, H_v]
 *   S0     [N, H_v, d_v, d_k]   (NULL => zero initial state)
 *   cu_seqlens [N+1]            sequence n owns tokens cu[n] .. cu[n+1]-1
 *   o      [T, H_v, d_v]        (output)
 *   S_final [N, H_v, d_v, d_k]  (output, NULL => not written)
 *   use_l2norm: 1 => q and k are L2-normalised over the head dim (the pages'
 *               use_qk_l2norm_in_kernel=True); 0 => used as given.
 * V head h reads QK head h / (H_v / H_qk) (repeat_interleave on the head dim).
 * Units (n, h) are independent and run in parallel; within a unit every step
 * is sequential in token order.
 */
void oracle_gdn_recurrent(const double* q, const double* k, const double* v,
                          const double* g, const double* beta, const double* S0,
                          const int64_t* cu_seqlens, int32_t N, int32_t H_qk,
                          int32_t H_v, int32_t d_k, int32_t d_v, double scale,
                          int32_t use_l2norm, double* o, double* S_final) {
    const int32_t r = H_v / H_qk;
    const int64_t units = (int64_t)N * H_v;
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)d_v * d_k);
        double* qn = (double*)malloc(sizeof(double) * (size_t)d_k);
        double* kn = (double*)malloc(sizeof(double) * (size_t)d_k);
        double* delta = (double*)malloc(sizeof(double) * (size_t)d_v);
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < units; ++u) {
            const int32_t n = (int32_t)(u / H_v);
            const int32_t h = (int32_t)(u % H_v);
            const int32_t j = h / r;
            const size_t ssz = (size_t)d_v * d_k;
            if (S0)
                memcpy(S, S0 + ((size_t)n * H_v + h) * ssz, sizeof(double) * ssz);
            else
                memset(S, 0, sizeof(double) * ssz);

            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                const double* qt = q + ((size_t)t * H_qk + j) * d_k;
                const double* kt = k + ((size_t)t * H_qk + j) * d_k;
                const double* vt = v + ((size_t)t * H_v + h) * d_v;
                double qs = 1.0, ks = 1.0;
                if (use_l2norm) {
                    double sq = 0.0, sk = 0.0;
                    for (int32_t c = 0; c < d_k; ++c) {
                        sq += qt[c] * qt[c];
                        sk += kt[c] * kt[c];
                    }
                    qs = 1.0 / sqrt(sq + ORACLE_L2_EPS);
                    ks = 1.0 / sqrt(sk + ORACLE_L2_EPS);
                }
                for (int32_t c = 0; c < d_k; ++c) {
                    qn[c] = qt[c] * qs * scale;
                    kn[c] = kt[c] * ks;
                }
                const double alpha = exp(g[(size_t)t * H_v + h]);
                const double bt = beta[(size_t)t * H_v + h];

                /* decay */
                for (size_t e = 0; e < ssz; ++e) S[e] *= alpha;
                /* read with the decayed state, form the delta */
                for (int32_t i = 0; i < d_v; ++i) {
                    double kv = 0.0;
                    for (int32_t c = 0; c < d_k; ++c) kv += S[(size_t)i * d_k + c] * kn[c];
                    delta[i] = bt * (vt[i] - kv);
                }
                /* write */
                for (int32_t i = 0; i < d_v; ++i)
                    for (int32_t c = 0; c < d_k; ++c)
                        S[(size_t)i * d_k + c] += delta[i] * kn[c];
                /* read-out */
                double* ot = o + ((size_t)t * H_v + h) * d_v;
                for (int32_t i = 0; i < d_v; ++i) {
                    double acc = 0.0;
                    for (int32_t c = 0; c < d_k; ++c) acc += S[(size_t)i * d_k + c] * qn[c];
                    ot[i] = acc;
                }
            }
            if (S_final)
                memcpy(S_final + ((size_t)n * H_v + h) * ssz, S, sizeof(double) * ssz);
        }
        free(S);
        free(qn);
        free(kn);
        free(delta);
    }
}

/*
 * Gates followed by the recurrence: the whole token mixer core from the raw
 * gate inputs a, b and the per-head parameters A_log, dt_bias.
 */
void oracle_gdn_forward(const double* q, const double* k, const double* v,
                        const double* a, const double* b, const double* A_log,
                        const double* dt_bias, const double* S0,
                        const int64_t* cu_seqlens, int32_t N, int64_t T,
                        int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                        double scale, int32_t use_l2norm, double* o,
                        double* S_final) {
    double* g = (double*)malloc(sizeof(double) * (size_t)T * H_v);
    double* beta = (double*)malloc(sizeof(double) * (size_t)T * H_v);
    oracle_gates(a, b, A_log, dt_bias, T, H_v, g, beta);
    oracle_gdn_recurrent(q, k, v, g, beta, S0, cu_seqlens, N, H_qk, H_v, d_k, d_v,
                         scale, use_l2norm, o, S_final);
    free(g);
    free(beta);
}

/* Number of OpenMP threads a parallel region of the oracle uses. */
int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
