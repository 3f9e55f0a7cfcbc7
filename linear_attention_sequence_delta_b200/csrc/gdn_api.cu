// C ABI of libgdn.so: argument checks, workspace carving and kernel dispatch.
// Declarations and the contract of every entry point are in include/gdn.h.
#include <math.h>

#include <atomic>
#include <mutex>
#include <new>

#include "gdn_internal.cuh"

namespace gdn {

// One status word per device: kernels record content errors (bad cu_seqlens,
// an expired bounded wait) here instead of trapping.
__device__ int g_status_word[2];  // [0] status, [1] first failed index check (debug build)

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int*> g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned(const void* p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline int to_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

int check_heads(int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v) {
    if (H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0) return GDN_ERR_INVALID_ARG;
    if (H_v % H_qk != 0) return GDN_ERR_INVALID_ARG;
    if (d_k != d_v || (d_k != 64 && d_k != 128)) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

size_t gate_bytes(int64_t T, int32_t H_v) { return align_up((size_t)T * H_v * sizeof(float), 256); }
}  // namespace

}  // namespace gdn

// A caller-owned kernel timer (gdn_timer_create): event pairs around each kernel of
// the most recent call that used it.
struct gdn_timer {
    static constexpr int kMax = 8;
    cudaEvent_t ev[2 * kMax] = {};
    const char* name[kMax] = {};
    int n = 0;
    bool open = false;  // an event pair is half recorded
};

namespace gdn {

void timer_before(gdn_timer* t, cudaStream_t s) {
    if (!t || t->n >= gdn_timer::kMax) return;
    t->open = cudaEventRecord(t->ev[2 * t->n], s) == cudaSuccess;
}

void timer_after(gdn_timer* t, cudaStream_t s, const char* kernel) {
    if (!t || t->n >= gdn_timer::kMax || !t->open) return;
    t->open = false;
    if (cudaEventRecord(t->ev[2 * t->n + 1], s) != cudaSuccess) return;
    t->name[t->n++] = kernel;
}

int* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    int* p = g_status_ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lk(g_status_mu);
    p = g_status_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return nullptr;
        p = static_cast<int*>(addr);
        g_status_ptr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace gdn

using namespace gdn;

extern "C" {

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_BAD_SEQLENS: return "GDN_ERR_BAD_SEQLENS";
        case GDN_ERR_BAD_SLOT: return "GDN_ERR_BAD_SLOT";
        case GDN_ERR_BAD_INDEX: return "GDN_ERR_BAD_INDEX";
        default: return "GDN_ERR_UNKNOWN";
    }
}

int gdn_version(void) { return 100; }

size_t gdn_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H_qk,
                                  int32_t H_v, int32_t d_k, int32_t d_v) {
    if (num_seqs < 0 || total_tokens < 0) return 0;
    if (check_heads(H_qk, H_v, d_k, d_v) != GDN_OK) return 0;
    if (num_seqs == 0) return 0;  // an empty batch launches nothing
    const size_t simt = 2 * gate_bytes(total_tokens, H_v);
    if (d_k != 128) return simt;
    const size_t tc = prefill_tc_workspace_bytes(num_seqs, total_tokens, H_v);
    return tc > simt ? tc : simt;
}

int gdn_gates(const float* a, const float* b, const float* A_log, const float* dt_bias,
              const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens, int32_t H_v,
              float* g_chunk_cumsum, float* g, float* beta, void* stream) {
    if (num_seqs < 0 || total_tokens < 0 || H_v <= 0) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0 && total_tokens != 0) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0 || (!g_chunk_cumsum && !g && !beta)) return GDN_OK;
    if (!a || !b || !A_log || !dt_bias || !cu_seqlens) return GDN_ERR_INVALID_ARG;
    if (!aligned(a, 4) || !aligned(b, 4) || !aligned(g_chunk_cumsum, 4) || !aligned(g, 4) ||
        !aligned(beta, 4))
        return GDN_ERR_INVALID_ARG;
    int* st = device_status_ptr();
    if (!st) return GDN_ERR_CUDA;
    return to_status(launch_gates(a, b, A_log, dt_bias, cu_seqlens, num_seqs, total_tokens, H_v,
                                  g_chunk_cumsum, g, beta, st, (cudaStream_t)stream));
}

}  // extern "C"

namespace {
// gdn_prefill(_ex) and gdn_prefill_slots(_ex): the same path, the states addressed per
// sequence or through pool slots
int prefill_common(const void* q, const void* k, const void* v, int32_t io_dtype,
                   const float* a, const float* b, const float* A_log, const float* dt_bias,
                   const float* initial_state, const int32_t* cu_seqlens, int32_t num_seqs,
                   int64_t total_tokens, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                   float scale, void* o, float* final_state, StateIndex sref, void* workspace,
                   size_t workspace_bytes, const gdn_prefill_options* options, void* stream) {
    PrefillOpts opt;
    if (options) {
        if (options->impl < GDN_IMPL_AUTO || options->impl > GDN_IMPL_TENSOR_CORE_WHOLE_ROWS)
            return GDN_ERR_INVALID_ARG;
        if (options->fault != GDN_FAULT_NONE && options->fault != GDN_FAULT_WITHHOLD_RECORDS &&
            options->fault != GDN_FAULT_BAD_INDEX)
            return GDN_ERR_INVALID_ARG;
        if (options->fault == GDN_FAULT_BAD_INDEX && !kDebugBuild) return GDN_ERR_UNSUPPORTED;
        if (options->wait_limit_cycles < 0) return GDN_ERR_INVALID_ARG;
        opt.impl = options->impl;
        opt.fault = options->fault;
        if (options->wait_limit_cycles > 0) opt.wait_cycles = options->wait_limit_cycles;
        opt.timer = options->timer;
    }
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0 || total_tokens < 0) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0 && total_tokens != 0) return GDN_ERR_INVALID_ARG;
    int hs = check_heads(H_qk, H_v, d_k, d_v);
    if (hs != GDN_OK) return hs;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if ((int64_t)num_seqs * H_v * (d_v / 32) >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if (!cu_seqlens || !A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !a || !b || !o)) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {q, k, v, o, initial_state, final_state};
    for (const void* p : ptrs16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(a, 4) || !aligned(b, 4)) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_prefill_workspace_size(num_seqs, total_tokens, H_qk, H_v, d_k, d_v);
    if (workspace_bytes < need || (need > 0 && !workspace)) return GDN_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return GDN_ERR_WORKSPACE;

    const bool tc_ok =
        io_dtype == GDN_BF16 && d_k == 128 && prefill_tc_supported(H_qk, H_v);
    const bool tc_forced = opt.impl == GDN_IMPL_TENSOR_CORE ||
                           opt.impl == GDN_IMPL_TENSOR_CORE_SPLIT ||
                           opt.impl == GDN_IMPL_TENSOR_CORE_WHOLE_ROWS;
    if (tc_forced && !tc_ok) return GDN_ERR_UNSUPPORTED;
    int* st = device_status_ptr();
    if (!st) return GDN_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    if (opt.timer) opt.timer->n = 0;
    if (tc_ok && opt.impl != GDN_IMPL_CUDA_CORE) {
        return to_status(launch_prefill_tc(q, k, v, a, b, A_log, dt_bias, initial_state,
                                           cu_seqlens, num_seqs, total_tokens, H_qk, H_v, scale,
                                           o, final_state, sref, workspace, opt, st, s));
    }
    float* G = static_cast<float*>(workspace);
    float* beta = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                           gate_bytes(total_tokens, H_v));
    if (total_tokens > 0) {
        timer_before(opt.timer, s);
        cudaError_t e = launch_gates(a, b, A_log, dt_bias, cu_seqlens, num_seqs, total_tokens,
                                     H_v, G, nullptr, beta, st, s);
        if (e != cudaSuccess) return GDN_ERR_CUDA;
        timer_after(opt.timer, s, "gates");
    }
    timer_before(opt.timer, s);
    const int rs = to_status(launch_prefill_simt(q, k, v, io_dtype, G, beta, initial_state,
                                                 cu_seqlens, num_seqs, total_tokens, H_qk, H_v,
                                                 d_k, scale, o, final_state, sref, st, s));
    timer_after(opt.timer, s, "prefill_simt");
    return rs;
}

int prefill_slots_common(const void* q, const void* k, const void* v, int32_t io_dtype,
                         const float* a, const float* b, const float* A_log,
                         const float* dt_bias, float* state_pool, const int32_t* state_slots,
                         const int32_t* has_initial_state, int32_t num_slots,
                         const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                         int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                         void* o, void* workspace, size_t workspace_bytes,
                         const gdn_prefill_options* options, void* stream) {
    if (num_seqs > 0 && (!state_slots || !state_pool)) return GDN_ERR_INVALID_ARG;
    if (num_slots < 0) return GDN_ERR_INVALID_ARG;
    if ((state_slots && !aligned(state_slots, 4)) ||
        (has_initial_state && !aligned(has_initial_state, 4)))
        return GDN_ERR_INVALID_ARG;
    StateIndex sref;
    sref.slots = state_slots;
    sref.has_init = has_initial_state;
    sref.num_slots = num_slots;
    return prefill_common(q, k, v, io_dtype, a, b, A_log, dt_bias, state_pool, cu_seqlens,
                          num_seqs, total_tokens, H_qk, H_v, d_k, d_v, scale, o, state_pool, sref,
                          workspace, workspace_bytes, options, stream);
}
}  // namespace

extern "C" {

int gdn_prefill(const void* q, const void* k, const void* v, int32_t io_dtype,
                const float* a, const float* b, const float* A_log, const float* dt_bias,
                const float* initial_state, const int32_t* cu_seqlens, int32_t num_seqs,
                int64_t total_tokens, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                float scale, void* o, float* final_state, void* workspace,
                size_t workspace_bytes, void* stream) {
    return prefill_common(q, k, v, io_dtype, a, b, A_log, dt_bias, initial_state, cu_seqlens,
                          num_seqs, total_tokens, H_qk, H_v, d_k, d_v, scale, o, final_state,
                          StateIndex{}, workspace, workspace_bytes, nullptr, stream);
}

int gdn_prefill_ex(const void* q, const void* k, const void* v, int32_t io_dtype,
                   const float* a, const float* b, const float* A_log, const float* dt_bias,
                   const float* initial_state, const int32_t* cu_seqlens, int32_t num_seqs,
                   int64_t total_tokens, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                   float scale, void* o, float* final_state, void* workspace,
                   size_t workspace_bytes, const gdn_prefill_options* options, void* stream) {
    return prefill_common(q, k, v, io_dtype, a, b, A_log, dt_bias, initial_state, cu_seqlens,
                          num_seqs, total_tokens, H_qk, H_v, d_k, d_v, scale, o, final_state,
                          StateIndex{}, workspace, workspace_bytes, options, stream);
}

int gdn_prefill_slots(const void* q, const void* k, const void* v, int32_t io_dtype,
                      const float* a, const float* b, const float* A_log, const float* dt_bias,
                      float* state_pool, const int32_t* state_slots,
                      const int32_t* has_initial_state, int32_t num_slots,
                      const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                      int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale, void* o,
                      void* workspace, size_t workspace_bytes, void* stream) {
    return prefill_slots_common(q, k, v, io_dtype, a, b, A_log, dt_bias, state_pool,
                                state_slots, has_initial_state, num_slots, cu_seqlens, num_seqs,
                                total_tokens, H_qk, H_v, d_k, d_v, scale, o, workspace,
                                workspace_bytes, nullptr, stream);
}

int gdn_prefill_slots_ex(const void* q, const void* k, const void* v, int32_t io_dtype,
                         const float* a, const float* b, const float* A_log,
                         const float* dt_bias, float* state_pool, const int32_t* state_slots,
                         const int32_t* has_initial_state, int32_t num_slots,
                         const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                         int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                         void* o, void* workspace, size_t workspace_bytes,
                         const gdn_prefill_options* options, void* stream) {
    return prefill_slots_common(q, k, v, io_dtype, a, b, A_log, dt_bias, state_pool,
                                state_slots, has_initial_state, num_slots, cu_seqlens, num_seqs,
                                total_tokens, H_qk, H_v, d_k, d_v, scale, o, workspace,
                                workspace_bytes, options, stream);
}

size_t gdn_mixer_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H_qk,
                                        int32_t H_v, int32_t d_k, int32_t d_v,
                                        int32_t io_dtype) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return 0;
    const size_t pre = gdn_prefill_workspace_size(num_seqs, total_tokens, H_qk, H_v, d_k, d_v);
    if (pre == 0) return 0;
    const size_t conv_dim = (size_t)(2 * H_qk + H_v) * d_k;
    const size_t s = io_dtype == GDN_BF16 ? 2 : 4;
    return align_up((size_t)total_tokens * conv_dim * s, 256) + pre;
}

int gdn_mixer_prefill(const void* x, int32_t io_dtype, const float* conv_weight,
                      const float* conv_bias, const void* conv_state_in, void* conv_state_out,
                      int32_t kernel_size, const float* a, const float* b, const float* A_log,
                      const float* dt_bias, const float* initial_state,
                      const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                      int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                      const void* z, const float* norm_weight, float eps, void* y,
                      float* final_state, void* workspace, size_t workspace_bytes,
                      const gdn_prefill_options* options, void* stream) {
    PrefillOpts opt;
    if (options) {
        if (options->impl < GDN_IMPL_AUTO || options->impl > GDN_IMPL_TENSOR_CORE_WHOLE_ROWS)
            return GDN_ERR_INVALID_ARG;
        if (options->fault != GDN_FAULT_NONE && options->fault != GDN_FAULT_WITHHOLD_RECORDS &&
            options->fault != GDN_FAULT_BAD_INDEX)
            return GDN_ERR_INVALID_ARG;
        if (options->fault == GDN_FAULT_BAD_INDEX && !kDebugBuild) return GDN_ERR_UNSUPPORTED;
        if (options->wait_limit_cycles < 0) return GDN_ERR_INVALID_ARG;
        opt.impl = options->impl;
        opt.fault = options->fault;
        if (options->wait_limit_cycles > 0) opt.wait_cycles = options->wait_limit_cycles;
        opt.timer = options->timer;
    }
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0 || total_tokens < 0) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0 && total_tokens != 0) return GDN_ERR_INVALID_ARG;
    int hs = check_heads(H_qk, H_v, d_k, d_v);
    if (hs != GDN_OK) return hs;
    if (kernel_size < 2 || kernel_size > 4) return GDN_ERR_UNSUPPORTED;
    if (!isfinite(scale) || !(eps >= 0.f) || !isfinite(eps)) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if ((int64_t)num_seqs * H_v * (d_v / 32) >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if (!cu_seqlens || !A_log || !dt_bias || !conv_weight || !norm_weight)
        return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!x || !a || !b || !z || !y)) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {x, z, y, conv_weight, norm_weight, conv_state_in, conv_state_out,
                            initial_state, final_state};
    for (const void* p : ptrs16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(a, 4) || !aligned(b, 4) || !aligned(conv_bias, 4)) return GDN_ERR_INVALID_ARG;
    if (y && (y == x || y == z)) return GDN_ERR_INVALID_ARG;  // y is written while x, z are read
    const size_t need = gdn_mixer_prefill_workspace_size(num_seqs, total_tokens, H_qk, H_v,
                                                         d_k, d_v, io_dtype);
    if (workspace_bytes < need || !workspace || !aligned(workspace, 256)) return GDN_ERR_WORKSPACE;

    const int conv_dim = (2 * H_qk + H_v) * d_k;
    const size_t s_io = io_dtype == GDN_BF16 ? 2 : 4;
    uint8_t* wb = static_cast<uint8_t*>(workspace);
    void* qkvc = wb;  // [T][conv_dim] post-conv q | k | v
    void* pre_ws = wb + align_up((size_t)total_tokens * conv_dim * s_io, 256);
    const bool tc_ok = io_dtype == GDN_BF16 && d_k == 128 && prefill_tc_supported(H_qk, H_v);
    const bool tc_forced = opt.impl == GDN_IMPL_TENSOR_CORE ||
                           opt.impl == GDN_IMPL_TENSOR_CORE_SPLIT ||
                           opt.impl == GDN_IMPL_TENSOR_CORE_WHOLE_ROWS;
    if (tc_forced && !tc_ok) return GDN_ERR_UNSUPPORTED;
    int* st = device_status_ptr();
    if (!st) return GDN_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    if (opt.timer) opt.timer->n = 0;
    if (tc_ok && opt.impl == GDN_IMPL_AUTO) {
        // The three steps one after another, the prefill on the tensor cores with its own
        // schedule (half-row chain blocks included) reading q, k and v from the post-conv
        // buffer through token strides and writing o to y, then the norm in place: faster
        // than the fused schedule below on every measured workload.
        timer_before(opt.timer, s);
        if (launch_conv1d_silu(x, io_dtype, conv_weight, conv_bias, conv_state_in, cu_seqlens,
                               num_seqs, total_tokens, conv_dim, kernel_size, qkvc, conv_state_out,
                               st, s) != cudaSuccess)
            return GDN_ERR_CUDA;
        timer_after(opt.timer, s, "conv1d_silu");
        const char* qc = static_cast<const char*>(qkvc);
        const int r = to_status(launch_prefill_tc(
            qc, qc + (size_t)H_qk * d_k * s_io, qc + (size_t)2 * H_qk * d_k * s_io, a, b, A_log,
            dt_bias, initial_state, cu_seqlens, num_seqs, total_tokens, H_qk, H_v, scale, y,
            final_state, StateIndex{}, pre_ws, opt, st, s, MixerFusion{}, conv_dim));
        if (r != GDN_OK) return r;
        if (total_tokens > 0) {
            timer_before(opt.timer, s);
            if (launch_rmsnorm_gated(y, z, io_dtype, norm_weight, eps, total_tokens * H_v, d_v, y,
                                     s) != cudaSuccess)
                return GDN_ERR_CUDA;
            timer_after(opt.timer, s, "rmsnorm_gated");
        }
        return GDN_OK;
    }
    if (tc_ok && opt.impl != GDN_IMPL_CUDA_CORE) {
        // the fused schedule: the convolution in the preparation's loads, the gated norm in
        // the chain's output
        MixerFusion mix;
        mix.x = static_cast<const __nv_bfloat16*>(x);
        mix.conv_w = conv_weight;
        mix.conv_b = conv_bias;
        mix.cache_in = static_cast<const __nv_bfloat16*>(conv_state_in);
        mix.cache_out = static_cast<__nv_bfloat16*>(conv_state_out);
        mix.qkvc = static_cast<__nv_bfloat16*>(qkvc);
        mix.conv_dim = conv_dim;
        mix.K = kernel_size;
        mix.z = static_cast<const __nv_bfloat16*>(z);
        mix.norm_w = norm_weight;
        mix.eps = eps;
        return to_status(launch_prefill_tc(nullptr, nullptr, nullptr, a, b, A_log, dt_bias,
                                           initial_state, cu_seqlens, num_seqs, total_tokens,
                                           H_qk, H_v, scale, y, final_state, StateIndex{}, pre_ws,
                                           opt, st, s, mix));
    }
    // The three steps one after another: the convolution into the workspace, the
    // CUDA-core prefill reading q, k and v there with o written to y, the norm in place.
    timer_before(opt.timer, s);
    if (launch_conv1d_silu(x, io_dtype, conv_weight, conv_bias, conv_state_in, cu_seqlens,
                           num_seqs, total_tokens, conv_dim, kernel_size, qkvc, conv_state_out,
                           st, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    timer_after(opt.timer, s, "conv1d_silu");
    float* G = static_cast<float*>(pre_ws);
    float* beta = reinterpret_cast<float*>(static_cast<char*>(pre_ws) +
                                           gate_bytes(total_tokens, H_v));
    if (total_tokens > 0) {
        timer_before(opt.timer, s);
        if (launch_gates(a, b, A_log, dt_bias, cu_seqlens, num_seqs, total_tokens, H_v, G,
                         nullptr, beta, st, s) != cudaSuccess)
            return GDN_ERR_CUDA;
        timer_after(opt.timer, s, "gates");
    }
    const char* qc = static_cast<const char*>(qkvc);
    timer_before(opt.timer, s);
    if (launch_prefill_simt(qc, qc + (size_t)H_qk * d_k * s_io, qc + (size_t)2 * H_qk * d_k * s_io,
                            io_dtype, G, beta, initial_state, cu_seqlens, num_seqs, total_tokens,
                            H_qk, H_v, d_k, scale, y, final_state, StateIndex{}, st, s, conv_dim,
                            conv_dim) != cudaSuccess)
        return GDN_ERR_CUDA;
    timer_after(opt.timer, s, "prefill_simt");
    if (total_tokens > 0) {
        timer_before(opt.timer, s);
        if (launch_rmsnorm_gated(y, z, io_dtype, norm_weight, eps, total_tokens * H_v, d_v, y, s) !=
            cudaSuccess)
            return GDN_ERR_CUDA;
        timer_after(opt.timer, s, "rmsnorm_gated");
    }
    return GDN_OK;
}

int gdn_decode_step(const void* q, const void* k, const void* v, int32_t io_dtype,
                    const float* a, const float* b, const float* A_log, const float* dt_bias,
                    float* state, int32_t num_seqs, int32_t H_qk, int32_t H_v, int32_t d_k,
                    int32_t d_v, float scale, void* o, void* stream) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0) return GDN_ERR_INVALID_ARG;
    int hs = check_heads(H_qk, H_v, d_k, d_v);
    if (hs != GDN_OK) return hs;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if ((int64_t)num_seqs * H_v >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {q, k, v, o, state};
    for (const void* p : ptrs16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(a, 4) || !aligned(b, 4)) return GDN_ERR_INVALID_ARG;
    return to_status(launch_decode(q, k, v, io_dtype, a, b, A_log, dt_bias, state, num_seqs,
                                   H_qk, H_v, d_k, scale, o, (cudaStream_t)stream));
}

int gdn_decode_step_bf16_state(const void* q, const void* k, const void* v, int32_t io_dtype,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, void* state, int32_t num_seqs,
                               int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                               void* o, void* stream) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0) return GDN_ERR_INVALID_ARG;
    int hs = check_heads(H_qk, H_v, d_k, d_v);
    if (hs != GDN_OK) return hs;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if ((int64_t)num_seqs * H_v >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {q, k, v, o, state};
    for (const void* p : ptrs16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(a, 4) || !aligned(b, 4)) return GDN_ERR_INVALID_ARG;
    return to_status(launch_decode_bf16_state(q, k, v, io_dtype, a, b, A_log, dt_bias, state,
                                              num_seqs, H_qk, H_v, d_k, scale, o,
                                              (cudaStream_t)stream));
}

int gdn_decode_slots(const void* q, const void* k, const void* v, int32_t io_dtype,
                     const float* a, const float* b, const float* A_log, const float* dt_bias,
                     float* state_pool, const int32_t* state_slots, int32_t num_slots,
                     int32_t num_seqs, int32_t tokens_per_seq, int32_t H_qk, int32_t H_v,
                     int32_t d_k, int32_t d_v, float scale, void* o,
                     float* intermediate_states, void* stream) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0 || num_slots < 0) return GDN_ERR_INVALID_ARG;
    if (tokens_per_seq < 1 || tokens_per_seq > kMaxDecodeTokens) return GDN_ERR_UNSUPPORTED;
    int hs = check_heads(H_qk, H_v, d_k, d_v);
    if (hs != GDN_OK) return hs;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (!state_slots && num_slots < num_seqs) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if ((int64_t)num_seqs * H_v >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !o) return GDN_ERR_INVALID_ARG;
    if (!state_pool && num_slots > 0) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {q, k, v, o, state_pool, intermediate_states};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(a, 4) || !aligned(b, 4) || (state_slots && !aligned(state_slots, 4)))
        return GDN_ERR_INVALID_ARG;
    return to_status(launch_decode_multi(q, k, v, io_dtype, a, b, A_log, dt_bias, state_pool,
                                         state_slots, num_slots, num_seqs, tokens_per_seq, H_qk,
                                         H_v, d_k, scale, o, intermediate_states,
                                         device_status_ptr(), (cudaStream_t)stream));
}

int gdn_conv1d_silu(const void* x, int32_t io_dtype, const float* weight, const float* bias,
                    const void* conv_state_in, const int32_t* cu_seqlens, int32_t num_seqs,
                    int64_t total_tokens, int32_t conv_dim, int32_t kernel_size, void* y,
                    void* conv_state_out, void* stream) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0 || total_tokens < 0 || conv_dim <= 0) return GDN_ERR_INVALID_ARG;
    if (kernel_size < 2 || kernel_size > 4 || conv_dim % 8 != 0) return GDN_ERR_UNSUPPORTED;
    if (num_seqs == 0) return total_tokens == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
    if (total_tokens == 0 && !conv_state_out) return GDN_OK;
    if (!x || !weight || !cu_seqlens || (total_tokens > 0 && !y)) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {x, y, weight, conv_state_in, conv_state_out};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 4)) return GDN_ERR_INVALID_ARG;
    if (!aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
    if (x == y) return GDN_ERR_INVALID_ARG;  // the window reads neighbouring tokens
    return to_status(launch_conv1d_silu(x, io_dtype, weight, bias, conv_state_in, cu_seqlens,
                                        num_seqs, total_tokens, conv_dim, kernel_size, y,
                                        conv_state_out, device_status_ptr(),
                                        (cudaStream_t)stream));
}

int gdn_conv1d_silu_decode(const void* x, int32_t io_dtype, const float* weight,
                           const float* bias, void* conv_state, const int32_t* cache_slots,
                           int32_t num_slots, int32_t num_seqs, int32_t conv_dim,
                           int32_t kernel_size, void* y, void* stream) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0 || num_slots < 0 || conv_dim <= 0) return GDN_ERR_INVALID_ARG;
    if (kernel_size < 2 || kernel_size > 4 || conv_dim % 8 != 0) return GDN_ERR_UNSUPPORTED;
    if (!cache_slots && num_slots < num_seqs) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if (!x || !weight || !y || (!conv_state && num_slots > 0)) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {x, y, weight, conv_state};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 4)) return GDN_ERR_INVALID_ARG;
    if (cache_slots && !aligned(cache_slots, 4)) return GDN_ERR_INVALID_ARG;
    return to_status(launch_conv1d_silu_decode(x, io_dtype, weight, bias, conv_state,
                                               cache_slots, num_slots, num_seqs, conv_dim,
                                               kernel_size, y, device_status_ptr(),
                                               (cudaStream_t)stream));
}

int gdn_rmsnorm_gated(const void* o, const void* z, int32_t io_dtype, const float* weight,
                      float eps, int64_t rows, int32_t d, void* y, void* stream) {
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (rows < 0 || !(eps >= 0.f) || !isfinite(eps)) return GDN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return GDN_ERR_UNSUPPORTED;
    if (rows == 0) return GDN_OK;
    if (!o || !z || !weight || !y) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {o, z, weight, y};
    for (const void* p : ptrs16)
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    return to_status(
        launch_rmsnorm_gated(o, z, io_dtype, weight, eps, rows, d, y, (cudaStream_t)stream));
}

gdn_timer* gdn_timer_create(void) {
    gdn_timer* t = new (std::nothrow) gdn_timer();
    if (!t) return nullptr;
    for (cudaEvent_t& e : t->ev) {
        if (cudaEventCreate(&e) != cudaSuccess) {
            e = nullptr;
            gdn_timer_destroy(t);
            return nullptr;
        }
    }
    return t;
}

void gdn_timer_destroy(gdn_timer* t) {
    if (!t) return;
    for (cudaEvent_t e : t->ev)
        if (e) cudaEventDestroy(e);
    delete t;
}

int gdn_timer_read(gdn_timer* t, float* ms, int32_t max_kernels) {
    if (!t || !ms || max_kernels < 0) return -GDN_ERR_INVALID_ARG;
    const int n = t->n < max_kernels ? t->n : max_kernels;
    for (int i = 0; i < n; ++i) {
        if (cudaEventSynchronize(t->ev[2 * i + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&ms[i], t->ev[2 * i], t->ev[2 * i + 1]) != cudaSuccess)
            return -GDN_ERR_CUDA;
    }
    return t->n;
}

const char* gdn_timer_kernel_name(const gdn_timer* t, int32_t i) {
    return (t && i >= 0 && i < t->n) ? t->name[i] : nullptr;
}

int gdn_debug_build(void) { return kDebugBuild ? 1 : 0; }

int gdn_debug_bad_index_site(void* stream) {
    int* st = device_status_ptr();
    if (!st) return -GDN_ERR_CUDA;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return -GDN_ERR_CUDA;
    int val = 0;
    if (cudaMemcpy(&val, st + 1, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return -GDN_ERR_CUDA;
    const int zero = 0;
    if (val != 0 && cudaMemcpy(st + 1, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return -GDN_ERR_CUDA;
    return val;
}

int gdn_sync_status(void* stream) {
    int* st = device_status_ptr();
    if (!st) return GDN_ERR_CUDA;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDN_ERR_CUDA;
    int val = 0;
    if (cudaMemcpy(&val, st, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int zero = 0;
    if (val != 0 && cudaMemcpy(st, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return GDN_ERR_CUDA;
    return val;
}

}  // extern "C"
