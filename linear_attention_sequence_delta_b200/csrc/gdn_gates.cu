// Gate prologue: beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias), and
// the inclusive cumulative sum of g inside each 64-token chunk of each sequence
// ("Qwen3.5 observation notes", "Qwen3_5MoeGatedDeltaNet"; "Qwen3.5-MoE-35B-A3B
// architecture teardown", 3.7 step 3).
//
// Layout: one block per (sequence, chunk slot); a thread owns one V head and
// walks the chunk's tokens in order, so each token row [H_v] is read and
// written as one coalesced line and the cumsum is a running sum in a register.
// The work is a few bytes per token and head: this kernel is launch- and
// latency-bound, never on the critical roofline.
#include "gdn_internal.cuh"

namespace gdn {

__global__ void __launch_bounds__(128) gates_kernel(
    const float* __restrict__ a, const float* __restrict__ b,
    const float* __restrict__ A_log, const float* __restrict__ dt_bias,
    const int32_t* __restrict__ cu_seqlens, int32_t num_seqs, int64_t total_tokens,
    int32_t H_v, float* __restrict__ G, float* __restrict__ g, float* __restrict__ beta,
    int* status) {
    const int n = blockIdx.x;
    const int64_t s0 = cu_seqlens[n];
    const int64_t s1 = cu_seqlens[n + 1];
    if (s0 < 0 || s1 < s0 || s1 > total_tokens || (n == 0 && s0 != 0)) {
        if (threadIdx.x == 0 && blockIdx.y == 0) set_status(status, kStatusBadSeqlens);
        return;
    }
    const int64_t len = s1 - s0;
    const int64_t nchunks = (len + kChunk - 1) / kChunk;
    for (int64_t c = blockIdx.y; c < nchunks; c += gridDim.y) {
        const int64_t t0 = s0 + c * kChunk;
        const int64_t t1 = min(t0 + (int64_t)kChunk, s1);
        for (int h = threadIdx.x; h < H_v; h += blockDim.x) {
            const float al = A_log[h];
            const float db = dt_bias[h];
            float acc = 0.f;
            for (int64_t t = t0; t < t1; ++t) {
                const int64_t i = t * H_v + h;
                const float gi = gate_g(a[i], al, db);
                acc += gi;
                if (G) G[i] = acc;
                if (g) g[i] = gi;
                if (beta) beta[i] = gate_beta(b[i]);
            }
        }
    }
}

cudaError_t launch_gates(const float* a, const float* b, const float* A_log,
                         const float* dt_bias, const int32_t* cu_seqlens, int32_t num_seqs,
                         int64_t total_tokens, int32_t H_v, float* G, float* g, float* beta,
                         int* status, cudaStream_t s) {
    if (num_seqs == 0) return cudaSuccess;
    // enough chunk slots per sequence to cover the average sequence in one pass
    int64_t avg_chunks = (total_tokens / num_seqs + kChunk - 1) / kChunk;
    int gy = (int)(avg_chunks < 1 ? 1 : (avg_chunks > 65535 ? 65535 : avg_chunks));
    dim3 grid(num_seqs, gy);
    int threads = H_v < 128 ? ((H_v + 31) / 32) * 32 : 128;
    gates_kernel<<<grid, threads, 0, s>>>(a, b, A_log, dt_bias, cu_seqlens, num_seqs,
                                          total_tokens, H_v, G, g, beta, status);
    return cudaGetLastError();
}

}  // namespace gdn
