// gdn_prefill_noalloc: the chunked prefill for callers that cannot allocate
// device memory.
//
// gdn_prefill needs a caller-provided workspace. Some callers cannot provide one:
// a runtime whose device memory is fully owned by a pool it must not disturb, a
// plugin handed only input and output buffers, code that runs where an allocation
// would block or synchronise the device. This entry point keeps its scratch (the
// chunk-cumulative log-decay G and beta of every token) in a fixed array inside
// the library instead, so the caller passes only inputs and outputs and nothing is
// allocated on any call. It always runs the fp32 CUDA-core chunk kernel: the
// tensor-core path's workspace grows with the tokens (about 276 bytes per token and
// V head), which a fixed array cannot hold for useful sizes.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds it (kNoallocScratchBytes) until the process exits. In host code
// its name is only a host-side stand-in, never a device address, so its device
// address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, and cached.
#include <math.h>

#include <atomic>
#include <mutex>

#include "gdn_internal.cuh"

namespace gdn {

namespace {

// G and beta, fp32 [T, H_v] each, each half rounded up to 256 bytes.
constexpr size_t kNoallocScratchBytes = (size_t)GDN_NOALLOC_MAX_GATE_ELEMS * 2 * sizeof(float);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set-up on first use).
void* scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr)
            return nullptr;
        p = addr;
        g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
    return p;
}

size_t half_bytes(int64_t T, int32_t H_v) {
    return ((size_t)T * H_v * sizeof(float) + 255) / 256 * 256;
}

}  // namespace

}  // namespace gdn

using namespace gdn;

extern "C" int gdn_prefill_noalloc(const void* q, const void* k, const void* v, int32_t io_dtype,
                                   const float* a, const float* b, const float* A_log,
                                   const float* dt_bias, const float* initial_state,
                                   const int32_t* cu_seqlens, int32_t num_seqs,
                                   int64_t total_tokens, int32_t H_qk, int32_t H_v, int32_t d_k,
                                   int32_t d_v, float scale, void* o, float* final_state,
                                   void* stream) {
    // The same checks as gdn_prefill, minus the workspace, plus the scratch limit.
    if (io_dtype != GDN_BF16 && io_dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (num_seqs < 0 || total_tokens < 0) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0 && total_tokens != 0) return GDN_ERR_INVALID_ARG;
    if (H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0 || H_v % H_qk != 0)
        return GDN_ERR_INVALID_ARG;
    if (d_k != d_v || (d_k != 64 && d_k != 128)) return GDN_ERR_UNSUPPORTED;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if ((int64_t)num_seqs * H_v * (d_v / 32) >= (int64_t)1 << 31) return GDN_ERR_UNSUPPORTED;
    if ((size_t)total_tokens * (size_t)H_v > (size_t)GDN_NOALLOC_MAX_GATE_ELEMS ||
        2 * half_bytes(total_tokens, H_v) > kNoallocScratchBytes)
        return GDN_ERR_WORKSPACE;  // larger than the built-in scratch: use gdn_prefill
    if (!cu_seqlens || !A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !a || !b || !o)) return GDN_ERR_INVALID_ARG;
    const void* ptrs16[] = {q, k, v, o, initial_state, final_state};
    for (const void* p : ptrs16)
        if (reinterpret_cast<uintptr_t>(p) % 16) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(a) % 4 || reinterpret_cast<uintptr_t>(b) % 4)
        return GDN_ERR_INVALID_ARG;

    char* scratch = static_cast<char*>(scratch_ptr());
    int* st = device_status_ptr();
    if (!scratch || !st) return GDN_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    // Every token of every sequence gets its G and beta written by the gate
    // kernel before the chunk kernel reads them, so nothing left in the array
    // by an earlier call is ever read: no clearing is needed.
    float* G = reinterpret_cast<float*>(scratch);
    float* beta = reinterpret_cast<float*>(scratch + half_bytes(total_tokens, H_v));
    if (total_tokens > 0) {
        if (launch_gates(a, b, A_log, dt_bias, cu_seqlens, num_seqs, total_tokens, H_v, G,
                         nullptr, beta, st, s) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    return launch_prefill_simt(q, k, v, io_dtype, G, beta, initial_state, cu_seqlens, num_seqs,
                               total_tokens, H_qk, H_v, d_k, scale, o, final_state, StateIndex{},
                               st, s) ==
                   cudaSuccess
               ? GDN_OK
               : GDN_ERR_CUDA;
}
