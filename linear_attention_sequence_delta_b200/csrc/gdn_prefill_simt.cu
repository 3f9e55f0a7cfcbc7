// Chunked prefill on the CUDA cores, all arithmetic in fp32.
//
// This is the precision path (fp32 q/k/v/o, tolerance 1e-4 against the fp64
// recurrence) and the plain reference design for the tensor-core kernel. It
// follows the chunkwise form of the gated delta rule ("Qwen3.5-MoE-35B-A3B
// architecture teardown", 3.7: in-chunk decay mask, triangular correction,
// inter-chunk scan, per-chunk state update), restated in the value-major
// orientation. For one chunk of L <= 64 tokens with in-chunk cumulative
// log-decay G and gates beta:
//   A    = strictly-lower(beta_i exp(G_i - G_j) k_i . k_j)
//   T    = (I + A)^-1                       (forward substitution)
//   Y    = diag(beta) (V - diag(e^G) K S^T)
//   Vnew = T Y
//   O    = diag(e^G) Q S^T + (Q K^T (.) exp(G_i - G_j))_{j<=i} Vnew
//   S   <- e^{G_L} S + Vnew^T diag(e^{G_L - G}) K
// Only differences G_i - G_j with i >= j are exponentiated, so nothing
// overflows however strong the decay.
//
// Mapping: one 256-thread block per (sequence, V head, slice of DVS value
// rows). Value rows of S evolve independently, so slices need no
// communication; the in-chunk products K K^T, Q K^T and T are recomputed per
// slice. The block walks its sequence's chunks in order.
#include "gdn_internal.cuh"

namespace gdn {

namespace {

constexpr int kThreads = 256;
constexpr int kC = kChunk;

template <int D, int DVS>
struct SimtSmem {
    static constexpr int KP = D + 1;   // padded row stride of K, Q, S (conflict-free)
    static constexpr int CP = kC + 1;  // padded row stride of the 64x64 matrices
    static constexpr int off_K = 0;
    static constexpr int off_Q = off_K + kC * KP;
    static constexpr int off_V = off_Q + kC * KP;
    static constexpr int off_Y = off_V + kC * DVS;
    static constexpr int off_N = off_Y + kC * DVS;    // Vnew
    static constexpr int off_QS = off_N + kC * DVS;
    static constexpr int off_A = off_QS + kC * DVS;
    static constexpr int off_T = off_A + kC * CP;
    static constexpr int off_P = off_T + kC * CP;
    static constexpr int off_S = off_P + kC * CP;
    static constexpr int off_G = off_S + DVS * KP;
    static constexpr int off_B = off_G + kC;
    static constexpr int off_EG = off_B + kC;
    static constexpr int off_EGL = off_EG + kC;
    static constexpr int floats = off_EGL + kC;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename IO, int D, int DVS>
__global__ void __launch_bounds__(kThreads, 1) prefill_simt_kernel(
    const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
    const float* __restrict__ Gcs, const float* __restrict__ beta,
    const float* S0, const int32_t* __restrict__ cu_seqlens, int64_t T_total,
    int H_qk, int H_v, float scale, IO* __restrict__ o, float* S_final, StateIndex sref,
    int* status, int64_t qk_tok, int64_t v_tok) {
    using L = SimtSmem<D, DVS>;
    constexpr int KP = L::KP, CP = L::CP;
    constexpr int NSL = D / DVS;
    extern __shared__ float sm[];
    float* Ks = sm + L::off_K;
    float* Qs = sm + L::off_Q;
    float* Vs = sm + L::off_V;
    float* Ys = sm + L::off_Y;
    float* Vn = sm + L::off_N;
    float* QSs = sm + L::off_QS;
    float* Am = sm + L::off_A;
    float* Tm = sm + L::off_T;
    float* Pm = sm + L::off_P;
    float* Ss = sm + L::off_S;
    float* Gs = sm + L::off_G;
    float* Bs = sm + L::off_B;
    float* eG = sm + L::off_EG;
    float* eGL = sm + L::off_EGL;

    const int tid = threadIdx.x;
    const int slice = blockIdx.x % NSL;
    const int h = (blockIdx.x / NSL) % H_v;
    const int n = blockIdx.x / (NSL * H_v);
    const int j = h / (H_v / H_qk);
    const int dv0 = slice * DVS;

    const int64_t s0 = cu_seqlens[n];
    const int64_t s1 = cu_seqlens[n + 1];
    if (s0 < 0 || s1 < s0 || s1 > T_total || (n == 0 && s0 != 0)) {
        if (tid == 0) set_status(status, kStatusBadSeqlens);
        return;
    }

    // state slice: rows dv0 .. dv0+DVS-1 of the d_v x d_k value-major state (of the
    // sequence's state, or of its pool slot); read completely before anything is written
    bool rd, wr;
    const int sidx = sref.resolve(n, rd, wr, tid == 0 ? status : nullptr);
    const float* S0s = rd ? S0 : nullptr;
    float* Sfs = wr ? S_final : nullptr;
    const size_t sbase = ((size_t)sidx * H_v + h) * D * D + (size_t)dv0 * D;
    for (int idx = tid; idx < DVS * D; idx += kThreads) {
        const int c = idx / D, kk = idx % D;
        Ss[c * KP + kk] = S0s ? S0s[sbase + idx] : 0.f;
    }

    for (int64_t t0 = s0; t0 < s1; t0 += kC) {
        const int Lc = (int)min((int64_t)kC, s1 - t0);
        __syncthreads();  // previous chunk fully consumed
        // ---- load the chunk ------------------------------------------------
        for (int idx = tid; idx < kC * D; idx += kThreads) {
            const int t = idx / D, c = idx % D;
            float kv = 0.f, qv = 0.f;
            if (t < Lc) {
                const size_t gi = (size_t)(t0 + t) * qk_tok + (size_t)j * D + c;
                kv = to_f32(k[gi]);
                qv = to_f32(q[gi]);
            }
            Ks[t * KP + c] = kv;
            Qs[t * KP + c] = qv;
        }
        for (int idx = tid; idx < kC * DVS; idx += kThreads) {
            const int t = idx / DVS, c = idx % DVS;
            Vs[idx] = t < Lc ? to_f32(v[(size_t)(t0 + t) * v_tok + (size_t)h * D + dv0 + c]) : 0.f;
        }
        if (tid < kC) {
            const bool ok = tid < Lc;
            Gs[tid] = ok ? Gcs[(size_t)(t0 + tid) * H_v + h] : 0.f;
            Bs[tid] = ok ? beta[(size_t)(t0 + tid) * H_v + h] : 0.f;
        }
        __syncthreads();
        // ---- L2 norms (warp per row), decay factors --------------------------
        {
            const int lane = tid & 31, w = tid >> 5;
            for (int t = w; t < kC; t += kThreads / 32) {
                float sk = 0.f, sq = 0.f;
                for (int c = lane; c < D; c += 32) {
                    const float kv = Ks[t * KP + c], qv = Qs[t * KP + c];
                    sk = fmaf(kv, kv, sk);
                    sq = fmaf(qv, qv, sq);
                }
                sk = warp_sum(sk);
                sq = warp_sum(sq);
                const float rk = 1.f / sqrtf(sk + kL2Eps);
                const float rq = scale / sqrtf(sq + kL2Eps);
                for (int c = lane; c < D; c += 32) {
                    Ks[t * KP + c] *= rk;
                    Qs[t * KP + c] *= rq;
                }
            }
            if (tid < kC) {
                const bool ok = tid < Lc;
                const float gl = Gs[Lc - 1];
                eG[tid] = ok ? expf(Gs[tid]) : 0.f;
                eGL[tid] = ok ? expf(gl - Gs[tid]) : 0.f;
            }
        }
        __syncthreads();
        // ---- A = strict-lower(beta_i Gamma_ij k_i.k_j), P = lower(Gamma_ij q_i.k_j)
        {
            const int ti = tid / 16, tj = tid % 16;
            float kk[4][4], qk[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) kk[x][y] = qk[x][y] = 0.f;
            for (int c = 0; c < D; ++c) {
                float ki[4], qi[4], kj[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    ki[x] = Ks[(ti + 16 * x) * KP + c];
                    qi[x] = Qs[(ti + 16 * x) * KP + c];
                    kj[x] = Ks[(tj + 16 * x) * KP + c];
                }
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        kk[x][y] = fmaf(ki[x], kj[y], kk[x][y]);
                        qk[x][y] = fmaf(qi[x], kj[y], qk[x][y]);
                    }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int i = ti + 16 * x, jj = tj + 16 * y;
                    const bool lower = jj <= i && i < Lc;
                    const float gam = lower ? expf(Gs[i] - Gs[jj]) : 0.f;
                    Am[i * CP + jj] = (jj < i && i < Lc) ? Bs[i] * gam * kk[x][y] : 0.f;
                    Pm[i * CP + jj] = lower ? gam * qk[x][y] : 0.f;
                }
        }
        __syncthreads();
        // ---- T = (I + A)^-1 by forward substitution, one row at a time --------
        // T_ij = -(A_ij + sum_{j<m<i} A_im T_mj) for j < i; T_ii = 1; T_ij = 0, j > i.
        {
            const int jj = tid >> 2, part = tid & 3;
            if (tid < kC) {
                Tm[0 * CP + tid] = tid == 0 ? 1.f : 0.f;
            }
            __syncthreads();
            for (int i = 1; i < kC; ++i) {
                float acc = 0.f;
                if (jj < i) {
                    for (int m = jj + 1 + part; m < i; m += 4)
                        acc = fmaf(Am[i * CP + m], Tm[m * CP + jj], acc);
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (part == 0 && jj < kC)
                    Tm[i * CP + jj] = jj < i ? -(Am[i * CP + jj] + acc) : (jj == i ? 1.f : 0.f);
                __syncthreads();
            }
        }
        // ---- X = K S^T, QS = Q S^T; Y = beta (V - e^G X); QS <- e^G QS --------
        {
            const int ti = tid / 8, tj = tid % 8;
            float xa[2][DVS / 8], qa[2][DVS / 8];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y) xa[x][y] = qa[x][y] = 0.f;
            for (int kk = 0; kk < D; ++kk) {
                float kt[2], qt[2], sv[DVS / 8];
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    kt[x] = Ks[(ti + 32 * x) * KP + kk];
                    qt[x] = Qs[(ti + 32 * x) * KP + kk];
                }
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y) sv[y] = Ss[(tj + 8 * y) * KP + kk];
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < DVS / 8; ++y) {
                        xa[x][y] = fmaf(kt[x], sv[y], xa[x][y]);
                        qa[x][y] = fmaf(qt[x], sv[y], qa[x][y]);
                    }
            }
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y) {
                    const int t = ti + 32 * x, c = tj + 8 * y;
                    Ys[t * DVS + c] = Bs[t] * (Vs[t * DVS + c] - eG[t] * xa[x][y]);
                    QSs[t * DVS + c] = eG[t] * qa[x][y];
                }
        }
        __syncthreads();
        // ---- Vnew = T Y -------------------------------------------------------
        {
            const int ti = tid / 8, tj = tid % 8;
            float acc[2][DVS / 8];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y) acc[x][y] = 0.f;
            for (int s = 0; s < kC; ++s) {
                float tv[2], yv[DVS / 8];
#pragma unroll
                for (int x = 0; x < 2; ++x) tv[x] = Tm[(ti + 32 * x) * CP + s];
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y) yv[y] = Ys[s * DVS + tj + 8 * y];
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < DVS / 8; ++y) acc[x][y] = fmaf(tv[x], yv[y], acc[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y)
                    Vn[(ti + 32 * x) * DVS + tj + 8 * y] = acc[x][y];
        }
        __syncthreads();
        // ---- O = e^G Q S^T + P Vnew -> global --------------------------------
        {
            const int ti = tid / 8, tj = tid % 8;
            float acc[2][DVS / 8];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y)
                    acc[x][y] = QSs[(ti + 32 * x) * DVS + tj + 8 * y];
            for (int s = 0; s < kC; ++s) {
                float pv[2], nv[DVS / 8];
#pragma unroll
                for (int x = 0; x < 2; ++x) pv[x] = Pm[(ti + 32 * x) * CP + s];
#pragma unroll
                for (int y = 0; y < DVS / 8; ++y) nv[y] = Vn[s * DVS + tj + 8 * y];
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < DVS / 8; ++y) acc[x][y] = fmaf(pv[x], nv[y], acc[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int t = ti + 32 * x;
                if (t < Lc) {
#pragma unroll
                    for (int y = 0; y < DVS / 8; ++y)
                        o[((size_t)(t0 + t) * H_v + h) * D + dv0 + tj + 8 * y] =
                            from_f32<IO>(acc[x][y]);
                }
            }
        }
        // ---- S <- e^{G_L} S + Vnew^T diag(e^{G_L - G}) K ------------------------
        {
            const int tc = tid / 32, tk = tid % 32;
            constexpr int NKB = D / 32;
            const float gL = expf(Gs[Lc - 1]);
            float acc[DVS / 8][NKB];
#pragma unroll
            for (int x = 0; x < DVS / 8; ++x)
#pragma unroll
                for (int y = 0; y < NKB; ++y) acc[x][y] = 0.f;
            for (int t = 0; t < Lc; ++t) {
                const float w = eGL[t];
                float nv[DVS / 8], kv[NKB];
#pragma unroll
                for (int x = 0; x < DVS / 8; ++x) nv[x] = Vn[t * DVS + tc + 8 * x] * w;
#pragma unroll
                for (int y = 0; y < NKB; ++y) kv[y] = Ks[t * KP + tk + 32 * y];
#pragma unroll
                for (int x = 0; x < DVS / 8; ++x)
#pragma unroll
                    for (int y = 0; y < NKB; ++y) acc[x][y] = fmaf(nv[x], kv[y], acc[x][y]);
            }
            // every (c, kk) entry of Ss is owned by exactly one thread: update in place
#pragma unroll
            for (int x = 0; x < DVS / 8; ++x)
#pragma unroll
                for (int y = 0; y < NKB; ++y) {
                    float* sp = &Ss[(tc + 8 * x) * KP + tk + 32 * y];
                    *sp = fmaf(gL, *sp, acc[x][y]);
                }
        }
    }
    __syncthreads();
    if (Sfs) {
        for (int idx = tid; idx < DVS * D; idx += kThreads) {
            const int c = idx / D, kk = idx % D;
            Sfs[sbase + idx] = Ss[c * KP + kk];
        }
    }
}

template <typename IO, int D, int DVS>
cudaError_t launch_simt_t(const void* q, const void* k, const void* v, const float* G,
                          const float* beta, const float* S0, const int32_t* cu, int32_t N,
                          int64_t T, int32_t H_qk, int32_t H_v, float scale, void* o,
                          float* S_final, StateIndex sref, int* status, cudaStream_t s,
                          int64_t qk_tok, int64_t v_tok) {
    using L = SimtSmem<D, DVS>;
    auto kern = prefill_simt_kernel<IO, D, DVS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::bytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)N * H_v * (D / DVS);
    if (blocks == 0) return cudaSuccess;
    kern<<<(unsigned)blocks, kThreads, L::bytes, s>>>(
        static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(v), G, beta,
        S0, cu, T, H_qk, H_v, scale, static_cast<IO*>(o), S_final, sref, status, qk_tok, v_tok);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const void* q, const void* k, const void* v, int io_dtype,
                                const float* G, const float* beta, const float* S0,
                                const int32_t* cu_seqlens, int32_t N, int64_t T, int32_t H_qk,
                                int32_t H_v, int32_t d, float scale, void* o, float* S_final,
                                StateIndex sref, int* status, cudaStream_t s, int64_t qk_tok,
                                int64_t v_tok) {
    if (qk_tok == 0) qk_tok = (int64_t)H_qk * d;
    if (v_tok == 0) v_tok = (int64_t)H_v * d;
#define GDN_SIMT(IO, D)                                                                      \
    return launch_simt_t<IO, D, 32>(q, k, v, G, beta, S0, cu_seqlens, N, T, H_qk, H_v, scale, \
                                    o, S_final, sref, status, s, qk_tok, v_tok)
    if (io_dtype == GDN_BF16) {
        if (d == 128) GDN_SIMT(__nv_bfloat16, 128);
        GDN_SIMT(__nv_bfloat16, 64);
    }
    if (d == 128) GDN_SIMT(float, 128);
    GDN_SIMT(float, 64);
#undef GDN_SIMT
}

}  // namespace gdn
