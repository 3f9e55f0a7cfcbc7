// Internal declarations shared by the kernel translation units of libgdn.so.
// Not part of the public ABI (that is include/gdn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int kChunk = 64;          // chunk length of the prefill (teardown, 3.7 step 2)
constexpr float kL2Eps = 1e-6f;     // inside the square root of the QK L2 norm
// Lower clamp of the per-token log-decay g. exp(-128) is 0 in fp32, so alpha is
// unchanged (exactly 0) by the clamp, but the in-chunk cumulative sums stay
// finite: a gate of alpha = 0 (g = -inf, e.g. exp(A_log) overflowing) would
// otherwise turn G_i - G_j into inf - inf = NaN.
constexpr float kMinLogDecay = -128.f;

// Device status word values (written by kernels, read by gdn_sync_status). The status
// pointer kernels receive addresses two words: [0] the status, [1] (debug build) the
// source line of the first failed index check.
constexpr int kStatusBadSeqlens = GDN_ERR_BAD_SEQLENS;
constexpr int kStatusTimeout = GDN_ERR_TIMEOUT;
constexpr int kStatusBadSlot = GDN_ERR_BAD_SLOT;
constexpr int kStatusBadIndex = GDN_ERR_BAD_INDEX;

// The debug build (libgdn_debug.so) is compiled with GDN_DEBUG=1.
#ifndef GDN_DEBUG
#define GDN_DEBUG 0
#endif
constexpr bool kDebugBuild = GDN_DEBUG != 0;

// ---- small device helpers ---------------------------------------------------

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// softplus(x) = log(1 + e^x) in the overflow-free form max(x,0) + log1p(e^-|x|).
__device__ __forceinline__ float softplus_f32(float x) {
    return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}

// g = -exp(A_log) * softplus(a + dt_bias); 0 when the softplus is 0 (alpha = 1);
// clamped below at kMinLogDecay (where alpha is 0 in fp32 either way).
__device__ __forceinline__ float gate_g(float a, float A_log, float dt_bias) {
    const float sp = softplus_f32(a + dt_bias);
    return sp > 0.f ? fmaxf(-expf(A_log) * sp, kMinLogDecay) : 0.f;
}

__device__ __forceinline__ float gate_beta(float b) { return 1.f / (1.f + expf(-b)); }

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Index check of the debug build: true when 0 <= idx < count. Otherwise it records
// GDN_ERR_BAD_INDEX in the status word and `line` in the second word (the first failed
// check's), and the caller skips the access. Compiled out (always true) in libgdn.so.
__device__ __forceinline__ bool in_bounds_at(long long idx, long long count, int* status,
                                             int line) {
#if GDN_DEBUG
    if (idx >= 0 && idx < count) return true;
    if (status) {
        atomicCAS(status, 0, GDN_ERR_BAD_INDEX);
        atomicCAS(status + 1, 0, line);
    }
    return false;
#else
    (void)idx; (void)count; (void)status; (void)line;
    return true;
#endif
}
#define GDN_IN_BOUNDS(idx, count, status) \
    ::gdn::in_bounds_at((long long)(idx), (long long)(count), (status), __LINE__)

// Where each sequence's initial and final states live. Without slots sequence n uses
// state n of the initial / final arrays. With slots it uses entry slots[n] of one pool,
// read only where has_init is null or has_init[n] != 0 (else it starts from zeros) and
// written at the end; slot < 0 starts from zeros and writes nothing; a slot >= num_slots
// is reported (GDN_ERR_BAD_SLOT) and treated like slot < 0.
struct StateIndex {
    const int32_t* slots = nullptr;
    const int32_t* has_init = nullptr;
    int num_slots = 0;
    __device__ __forceinline__ int resolve(int n, bool& read, bool& write, int* status) const {
        read = write = true;
        if (!slots) return n;
        const int s = slots[n];
        if (s < 0 || s >= num_slots) {
            if (s >= num_slots) set_status(status, GDN_ERR_BAD_SLOT);
            read = write = false;
            return 0;
        }
        read = !has_init || has_init[n] != 0;
        return s;
    }
};

// The steps around the delta rule that gdn_mixer_prefill fuses into the tensor-core
// prefill's kernels: the causal depthwise convolution + SiLU in the preparation's loads
// of q, k and v (x != nullptr), and the gated RMSNorm in the chain's output (z != nullptr).
struct MixerFusion {
    const __nv_bfloat16* x = nullptr;         // [T][conv_dim] pre-conv, channels q | k | v
    const float* conv_w = nullptr;            // [conv_dim][K]
    const float* conv_b = nullptr;            // [conv_dim] or null
    const __nv_bfloat16* cache_in = nullptr;  // [N][K-1][conv_dim] or null (zeros)
    __nv_bfloat16* cache_out = nullptr;       // [N][K-1][conv_dim] or null
    __nv_bfloat16* qkvc = nullptr;            // [T][conv_dim] post-conv q, k, v (workspace)
    int conv_dim = 0, K = 0;
    const __nv_bfloat16* z = nullptr;         // [T][H_v][d] output gate
    const float* norm_w = nullptr;            // [d]
    float eps = 0.f;
};

// ---- host launchers (one per kernel family) ----------------------------------

// Status word of the current device (a __device__ int of this library).
int* device_status_ptr();

// ---- per-call options of the prefill (gdn_prefill_ex) ----
// Default limit of a bounded device-side wait: about 2 s at 2 GHz.
constexpr long long kDefaultWaitCycles = 4000000000LL;
struct PrefillOpts {
    int impl = GDN_IMPL_AUTO;
    int fault = GDN_FAULT_NONE;
    long long wait_cycles = kDefaultWaitCycles;
    gdn_timer* timer = nullptr;
};
// With a timer, every kernel launch of the call is bracketed by two CUDA events
// recorded on the launch stream; with NULL these do nothing.
void timer_before(gdn_timer* t, cudaStream_t s);
void timer_after(gdn_timer* t, cudaStream_t s, const char* kernel);

cudaError_t launch_gates(const float* a, const float* b, const float* A_log,
                         const float* dt_bias, const int32_t* cu_seqlens, int32_t num_seqs,
                         int64_t total_tokens, int32_t H_v, float* G, float* g, float* beta,
                         int* status, cudaStream_t s);

cudaError_t launch_decode(const void* q, const void* k, const void* v, int io_dtype,
                          const float* a, const float* b, const float* A_log,
                          const float* dt_bias, float* state, int32_t N, int32_t H_qk,
                          int32_t H_v, int32_t d, float scale, void* o, cudaStream_t s);

// Single-token decode with a bf16 state [N, H_v, d_v, d_k], updated in place.
cudaError_t launch_decode_bf16_state(const void* q, const void* k, const void* v,
                                     int io_dtype, const float* a, const float* b,
                                     const float* A_log, const float* dt_bias, void* state,
                                     int32_t N, int32_t H_qk, int32_t H_v, int32_t d,
                                     float scale, void* o, cudaStream_t s);

// L tokens per sequence from a state pool indexed by slots (NULL: slot n), optional
// per-token states; at most kMaxDecodeTokens tokens.
constexpr int kMaxDecodeTokens = 16;
cudaError_t launch_decode_multi(const void* q, const void* k, const void* v, int io_dtype,
                                const float* a, const float* b, const float* A_log,
                                const float* dt_bias, float* pool, const int32_t* slots,
                                int32_t num_slots, int32_t N, int32_t L, int32_t H_qk,
                                int32_t H_v, int32_t d, float scale, void* o, float* inter,
                                int* status, cudaStream_t s);

// qk_tok, v_tok: elements from one token's q (k) rows to the next token's, and v's
// (H_qk d and H_v d for dense [T, H, d] tensors; larger for strided views).
cudaError_t launch_prefill_simt(const void* q, const void* k, const void* v, int io_dtype,
                                const float* G, const float* beta, const float* S0,
                                const int32_t* cu_seqlens, int32_t N, int64_t T, int32_t H_qk,
                                int32_t H_v, int32_t d, float scale, void* o, float* S_final,
                                StateIndex sref, int* status, cudaStream_t s,
                                int64_t qk_tok = 0, int64_t v_tok = 0);

// Tensor-core prefill (bf16 I/O, d = 128): chunk offsets, the state-independent
// prep kernel, then the chain kernel, or both stages in one cooperative launch where
// that pays (opt.impl: GDN_IMPL_TENSOR_CORE_SPLIT forces separate launches,
// GDN_IMPL_TENSOR_CORE_WHOLE_ROWS forbids half-row chain blocks). The workspace holds
// the chunk offsets and one record (T, P and per-token factors) per (chunk, V head).
size_t prefill_tc_workspace_bytes(int32_t N, int64_t T, int32_t H_v);
bool prefill_tc_supported(int32_t H_qk, int32_t H_v);
cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, const float* a,
                              const float* b, const float* A_log, const float* dt_bias,
                              const float* S0, const int32_t* cu_seqlens, int32_t N, int64_t T,
                              int32_t H_qk, int32_t H_v, float scale, void* o, float* S_final,
                              StateIndex sref, void* workspace, const PrefillOpts& opt,
                              int* status, cudaStream_t s, const MixerFusion& mix = MixerFusion{},
                              int64_t qkv_tok = 0);

// Steps around the delta rule (gdn_mixer.cu): causal depthwise conv1d + SiLU with
// the per-sequence conv cache, its single-token decode form, and the gated RMSNorm.
cudaError_t launch_conv1d_silu(const void* x, int io_dtype, const float* w, const float* bias,
                               const void* state_in, const int32_t* cu, int N, int64_t T, int C,
                               int K, void* y, void* state_out, int* status, cudaStream_t s);
cudaError_t launch_conv1d_silu_decode(const void* x, int io_dtype, const float* w,
                                      const float* bias, void* state, const int32_t* slots,
                                      int num_slots, int N, int C, int K, void* y, int* status,
                                      cudaStream_t s);
cudaError_t launch_rmsnorm_gated(const void* o, const void* z, int io_dtype, const float* w,
                                 float eps, int64_t rows, int d, void* y, cudaStream_t s);

}  // namespace gdn
