// The steps around the gated delta rule in the GDN token mixer ("Qwen3.5-MoE-35B-A3B
// architecture teardown", 3.3 phases 2 and 4; "Qwen3.5 observation notes",
// "Qwen3_5MoeGatedDeltaNet"):
//   - causal depthwise convolution (kernel size K <= 4, one filter per channel) +
//     SiLU over the concatenated q/k/v channels, with the per-sequence conv cache of
//     the last K-1 input positions ([N][K-1][C], oldest first);
//   - gated RMSNorm of the mixer output: y = o / sqrt(mean(o^2) + eps) * w * silu(z).
// All are HBM-bound streaming passes: every thread moves 16-byte vectors of 8
// channels, consecutive threads consecutive vectors, arithmetic in fp32.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kVec = 8;        // channels per thread (one 16-byte bf16 vector)
constexpr int kDecSeqs = 2;    // sequences per thread in the decode convolution
constexpr int kMaxK = 4;

template <typename IO>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
    struct Raw {
        uint4 u;
    };
    __device__ static Raw load_raw(const __nv_bfloat16* p) {
        return Raw{*reinterpret_cast<const uint4*>(p)};
    }
    __device__ static void load(const __nv_bfloat16* p, float (&v)[kVec]) {
        unpack(load_raw(p), v);
    }
    __device__ static void unpack(const Raw& r, float (&v)[kVec]) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            v[2 * e] = f.x;
            v[2 * e + 1] = f.y;
        }
    }
    __device__ static void store(__nv_bfloat16* p, const float (&v)[kVec]) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};
template <>
struct Vec8<float> {
    struct Raw {
        float4 a, b;
    };
    __device__ static Raw load_raw(const float* p) {
        return Raw{reinterpret_cast<const float4*>(p)[0], reinterpret_cast<const float4*>(p)[1]};
    }
    __device__ static void load(const float* p, float (&v)[kVec]) { unpack(load_raw(p), v); }
    __device__ static void unpack(const Raw& r, float (&v)[kVec]) {
        v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
        v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
    }
    __device__ static void store(float* p, const float (&v)[kVec]) {
        reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
};

// x * sigmoid(x) with the fast exponential and division: two SFU operations per value
// (an IEEE division costs several times more and made the convolution compute-bound).
// Relative error a few fp32 ulp; for x < -88 the exponential overflows to inf and the
// result is 0, where the exact value is below 1e-36 in magnitude.
__device__ __forceinline__ float silu_f32(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// The prefill convolution: a thread walks kConvRange consecutive tokens of one channel
// vector, kConvGroup tokens at a time, and issues the next group's loads before it
// computes the current one; the window of the last K-1 inputs stays in registers, so
// each input is read once (plus K-1 positions per range).
constexpr int kConvRange = 32;
constexpr int kConvGroup = 4;

// sequence n with cu[n] <= t < cu[n + 1] (the last such n for empty sequences)
__device__ __forceinline__ int find_seq(const int32_t* cu, int N, int64_t t) {
    int lo = 0, hi = N;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

// Taps and bias of channels c0 .. c0+7 (w is [C][K], 16-byte aligned).
template <int K>
__device__ __forceinline__ void load_taps(const float* __restrict__ w,
                                          const float* __restrict__ bias, int c0,
                                          float (&wt)[K][kVec], float (&bs)[kVec]) {
    const float4* w4 = reinterpret_cast<const float4*>(w + (size_t)c0 * K);
#pragma unroll
    for (int f = 0; f < 2 * K; ++f) {  // 8 channels x K taps = 2K float4
        const float4 u = __ldg(w4 + f);
        const float vals[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int flat = 4 * f + j;
            wt[flat % K][flat / K] = vals[j];
        }
    }
#pragma unroll
    for (int e = 0; e < kVec; ++e) bs[e] = bias ? __ldg(bias + c0 + e) : 0.f;
}

// y for kConvRange consecutive tokens x kVec channels per thread; consecutive threads
// take consecutive channel vectors of the same token range. At a sequence's start the
// window comes from the cache (or zeros).
template <typename IO, int K>
__global__ void __launch_bounds__(128) conv1d_silu_kernel(
    const IO* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
    const IO* __restrict__ state_in, const int32_t* __restrict__ cu, int N, int64_t T, int C,
    IO* __restrict__ y, int* status) {
    using V = Vec8<IO>;
    const int nv = C / kVec;
    const int64_t gidx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t range = gidx / nv;
    const int c0 = (int)(gidx - range * nv) * kVec;
    const int64_t tb = range * kConvRange;
    if (tb >= T) return;
    const int64_t te = tb + kConvRange < T ? tb + kConvRange : T;
    // Let the cache kernel that follows start its loads (it waits before storing).
    asm volatile("griddepcontrol.launch_dependents;");
    // Loads that need no sequence bounds go first, so that they overlap the lookup in
    // cu_seqlens: the first group (index clamped to the range) and the K-1 positions
    // before the range (clamped to 0).
    typename V::Raw cur[kConvGroup], wb[K - 1];
#pragma unroll
    for (int i = 0; i < kConvGroup; ++i)
        cur[i] = V::load_raw(x + (size_t)(tb + i < te ? tb + i : te - 1) * C + c0);
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t p = tb - (K - 1) + j;
        wb[j] = V::load_raw(x + (size_t)(p > 0 ? p : 0) * C + c0);
    }
    float wt[K][kVec], bs[kVec];
    load_taps<K>(w, bias, c0, wt, bs);
    int n = find_seq(cu, N, tb);
    int64_t s0 = cu[n], s1 = cu[n + 1];
    if (s0 < 0 || tb < s0 || s1 < s0 || s1 > T) {
        set_status(status, kStatusBadSeqlens);
        return;
    }
    float win[kMaxK - 1][kVec];  // win[K-2] is the newest
    // positions t-(K-1) .. t-1 of sequence n, those before its start from the cache
    auto window_entry = [&](int64_t p, float (&v)[kVec]) {
        if (state_in) {
            V::load(state_in + ((size_t)n * (K - 1) + (K - 1) + (p - s0)) * C + c0, v);
        } else {
#pragma unroll
            for (int e = 0; e < kVec; ++e) v[e] = 0.f;
        }
    };
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t p = tb - (K - 1) + j;
        if (p >= s0) V::unpack(wb[j], win[j]);
        else window_entry(p, win[j]);
    }
    auto step = [&](const float (&xt)[kVec], int64_t t) {
        float out[kVec];
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            float acc = bs[e];
#pragma unroll
            for (int i = 0; i < K - 1; ++i) acc = fmaf(wt[i][e], win[i][e], acc);
            acc = fmaf(wt[K - 1][e], xt[e], acc);
            out[e] = silu_f32(acc);
        }
        V::store(y + (size_t)t * C + c0, out);
#pragma unroll
        for (int j = 0; j + 1 < K - 1; ++j)
#pragma unroll
            for (int e = 0; e < kVec; ++e) win[j][e] = win[j + 1][e];
#pragma unroll
        for (int e = 0; e < kVec; ++e) win[K - 2][e] = xt[e];
    };
#pragma unroll 1
    for (int64_t g0 = tb; g0 < te; g0 += kConvGroup) {
        const bool more = g0 + kConvGroup < te;
        typename V::Raw nxt[kConvGroup];
        if (more) {
#pragma unroll
            for (int i = 0; i < kConvGroup; ++i) {
                const int64_t t = g0 + kConvGroup + i;
                nxt[i] = V::load_raw(x + (size_t)(t < te ? t : te - 1) * C + c0);
            }
        }
#pragma unroll
        for (int i = 0; i < kConvGroup; ++i) {
            const int64_t t = g0 + i;
            if (t < te) {
                if (t >= s1) {  // the next non-empty sequence starts here
                    while (t >= s1) {
                        if (n + 1 >= N) {  // tokens past cu[N]
                            set_status(status, kStatusBadSeqlens);
                            return;
                        }
                        ++n;
                        s0 = s1;
                        s1 = cu[n + 1];
                        if (s1 < s0) {
                            set_status(status, kStatusBadSeqlens);
                            return;
                        }
                    }
                    if (s1 > T) {
                        set_status(status, kStatusBadSeqlens);
                        return;
                    }
                    // t == s0: the whole window precedes the sequence
#pragma unroll
                    for (int j = 0; j < K - 1; ++j) window_entry(t - (K - 1) + j, win[j]);
                }
                float xt[kVec];
                V::unpack(cur[i], xt);
                step(xt, t);
            }
        }
        if (more) {
#pragma unroll
            for (int i = 0; i < kConvGroup; ++i) cur[i] = nxt[i];
        }
    }
}

// The cache after each sequence: its last K-1 input positions (older cache entries
// where the sequence is shorter). One thread per (sequence, channel vector) reads
// everything it writes before writing, so state_out may be state_in.
template <typename IO, int K>
__global__ void __launch_bounds__(256) conv_state_kernel(const IO* __restrict__ x,
                                                         const IO* state_in,
                                                         const int32_t* __restrict__ cu,
                                                         int N, int64_t T, int C, IO* state_out) {
    const int nv = C / kVec;
    const int64_t gidx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = gidx / nv;
    const int c0 = (int)(gidx - n * nv) * kVec;
    if (n >= N) return;
    const int64_t s0 = cu[n], s1 = cu[n + 1];
    if (s0 < 0 || s1 < s0 || s1 > T) return;  // reported by the convolution
    const int64_t L = s1 - s0;
    float v[kMaxK - 1][kVec];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t p = L - (K - 1) + j;
        if (p >= 0) {
            Vec8<IO>::load(x + (size_t)(s0 + p) * C + c0, v[j]);
        } else if (state_in) {
            Vec8<IO>::load(state_in + ((size_t)n * (K - 1) + (K - 1) + p) * C + c0, v[j]);
        } else {
#pragma unroll
            for (int e = 0; e < kVec; ++e) v[j][e] = 0.f;
        }
    }
    // Launched as a programmatic dependent of the convolution: everything above only
    // reads; the stores wait for the convolution grid (which may read state_in == state_out)
    // to finish. Without that launch attribute the wait returns at once.
    asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
    for (int j = 0; j < K - 1; ++j)
        Vec8<IO>::store(state_out + ((size_t)n * (K - 1) + j) * C + c0, v[j]);
}

// One token per sequence: y = silu(bias + w . [cache, x]); the cache slides by one.
// The cache of sequence n is pool entry slots[n] (n without slots): a slot < 0 is a
// padding entry (y zeroed, no cache touched), a slot >= num_slots is reported. A thread
// takes one channel vector of kDecSeqs sequences (the taps loaded once) and loads all
// their inputs before using any.
constexpr int kDecThreads = 64;  // small blocks: 17.7 -> 16.7 us on 256 x 12288 (vs 128)

template <typename IO, int K>
__global__ void __launch_bounds__(kDecThreads) conv_decode_kernel(const IO* __restrict__ x,
                                                          const float* __restrict__ w,
                                                          const float* __restrict__ bias,
                                                          IO* state,
                                                          const int32_t* __restrict__ slots,
                                                          int num_slots, int N, int C,
                                                          IO* __restrict__ y, int* status) {
    const int nv = C / kVec;
    const int64_t gidx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t grp = gidx / nv;
    const int c0 = (int)(gidx - grp * nv) * kVec;
    const int64_t n0 = grp * kDecSeqs;
    if (n0 >= N) return;
    int64_t slot[kDecSeqs];
    typename Vec8<IO>::Raw raw[kDecSeqs][K];
#pragma unroll
    for (int q = 0; q < kDecSeqs; ++q) {
        const int64_t n = n0 + q < N ? n0 + q : n0;  // a missing last sequence re-reads n0
        slot[q] = slots ? slots[n] : n;
        const bool ok = slot[q] >= 0 && slot[q] < num_slots;
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
            raw[q][j] = Vec8<IO>::load_raw(state + ((size_t)(ok ? slot[q] : 0) * (K - 1) + j) * C
                                           + c0);
        raw[q][K - 1] = Vec8<IO>::load_raw(x + (size_t)n * C + c0);
    }
    float wt[K][kVec], bs[kVec];
    load_taps<K>(w, bias, c0, wt, bs);
#pragma unroll
    for (int q = 0; q < kDecSeqs; ++q) {
        const int64_t n = n0 + q;
        if (n >= N) break;
        float out[kVec];
        if (slot[q] < 0) {
#pragma unroll
            for (int e = 0; e < kVec; ++e) out[e] = 0.f;
            Vec8<IO>::store(y + (size_t)n * C + c0, out);
            continue;
        }
        if (slot[q] >= num_slots) {
            set_status(status, kStatusBadSlot);
            continue;
        }
        float win[K][kVec];
#pragma unroll
        for (int j = 0; j < K; ++j) Vec8<IO>::unpack(raw[q][j], win[j]);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            float acc = bs[e];
#pragma unroll
            for (int i = 0; i < K; ++i) acc = fmaf(wt[i][e], win[i][e], acc);
            out[e] = silu_f32(acc);
        }
        Vec8<IO>::store(y + (size_t)n * C + c0, out);
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
            Vec8<IO>::store(state + ((size_t)slot[q] * (K - 1) + j) * C + c0, win[j + 1]);
    }
}

// Rows of D (64 or 128) values, D/8 lanes per row, each lane 8 consecutive values.
// Each lane reads its values before writing them, so y may be o or z.
template <typename IO, int D>
__global__ void __launch_bounds__(256) rmsnorm_gated_kernel(
    const IO* o, const IO* z, const float* __restrict__ w, float eps, int64_t rows, IO* y) {
    constexpr int kLanes = D / kVec;  // 16 or 8
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t r = gt / kLanes;
    const int part = (int)(gt % kLanes);
    const bool live = r < rows;
    float ov[kVec], zv[kVec];
    if (live) {
        Vec8<IO>::load(o + (size_t)r * D + part * kVec, ov);
        Vec8<IO>::load(z + (size_t)r * D + part * kVec, zv);
    } else {
#pragma unroll
        for (int e = 0; e < kVec; ++e) ov[e] = zv[e] = 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < kVec; ++e) ss = fmaf(ov[e], ov[e], ss);
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (!live) return;
    const float inv = rsqrtf(ss * (1.f / D) + eps);
    const float4 w0 = reinterpret_cast<const float4*>(w + part * kVec)[0];
    const float4 w1 = reinterpret_cast<const float4*>(w + part * kVec)[1];
    const float wv[kVec] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float out[kVec];
#pragma unroll
    for (int e = 0; e < kVec; ++e) out[e] = ov[e] * inv * wv[e] * silu_f32(zv[e]);
    Vec8<IO>::store(y + (size_t)r * D + part * kVec, out);
}

inline unsigned blocks_for(int64_t threads_total, int threads) {
    return (unsigned)((threads_total + threads - 1) / threads);
}

template <typename IO, int K>
cudaError_t conv_launch(const void* x, const float* w, const float* bias, const void* state_in,
                        const int32_t* cu, int N, int64_t T, int C, void* y, void* state_out,
                        int* status, cudaStream_t s) {
    const int64_t nv = C / kVec;
    if (T > 0) {
        const int threads = 128;
        const int64_t ranges = (T + kConvRange - 1) / kConvRange;
        conv1d_silu_kernel<IO, K><<<blocks_for(ranges * nv, threads), threads, 0, s>>>(
            static_cast<const IO*>(x), w, bias, static_cast<const IO*>(state_in), cu, N, T, C,
            static_cast<IO*>(y), status);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (state_out && N > 0) {
        // programmatic dependent launch: its loads overlap the convolution's tail
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = T > 0 ? 1 : 0;
        cfg.gridDim = dim3(blocks_for((int64_t)N * nv, 256));
        cfg.blockDim = dim3(256);
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, conv_state_kernel<IO, K>, static_cast<const IO*>(x),
                                  static_cast<const IO*>(state_in), cu, N, T, C,
                                  static_cast<IO*>(state_out));
    }
    return cudaSuccess;
}

template <typename IO, int K>
cudaError_t conv_decode_launch(const void* x, const float* w, const float* bias, void* state,
                               const int32_t* slots, int num_slots, int N, int C, void* y,
                               int* status, cudaStream_t s) {
    const int threads = kDecThreads;
    const int64_t groups = (N + kDecSeqs - 1) / kDecSeqs;
    conv_decode_kernel<IO, K><<<blocks_for(groups * (C / kVec), threads), threads, 0, s>>>(
        static_cast<const IO*>(x), w, bias, static_cast<IO*>(state), slots, num_slots, N, C,
        static_cast<IO*>(y), status);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t conv_dispatch_k(int K, const void* x, const float* w, const float* bias,
                            const void* state_in, const int32_t* cu, int N, int64_t T, int C,
                            void* y, void* state_out, int* status, cudaStream_t s) {
    switch (K) {
        case 2: return conv_launch<IO, 2>(x, w, bias, state_in, cu, N, T, C, y, state_out, status, s);
        case 3: return conv_launch<IO, 3>(x, w, bias, state_in, cu, N, T, C, y, state_out, status, s);
        default: return conv_launch<IO, 4>(x, w, bias, state_in, cu, N, T, C, y, state_out, status, s);
    }
}

template <typename IO>
cudaError_t conv_decode_dispatch_k(int K, const void* x, const float* w, const float* bias,
                                   void* state, const int32_t* slots, int num_slots, int N,
                                   int C, void* y, int* status, cudaStream_t s) {
    switch (K) {
        case 2: return conv_decode_launch<IO, 2>(x, w, bias, state, slots, num_slots, N, C, y, status, s);
        case 3: return conv_decode_launch<IO, 3>(x, w, bias, state, slots, num_slots, N, C, y, status, s);
        default: return conv_decode_launch<IO, 4>(x, w, bias, state, slots, num_slots, N, C, y, status, s);
    }
}

template <typename IO, int D>
cudaError_t rms_launch(const void* o, const void* z, const float* w, float eps, int64_t rows,
                       void* y, cudaStream_t s) {
    const int threads = 256;
    rmsnorm_gated_kernel<IO, D><<<blocks_for(rows * (D / kVec), threads), threads, 0, s>>>(
        static_cast<const IO*>(o), static_cast<const IO*>(z), w, eps, rows, static_cast<IO*>(y));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv1d_silu(const void* x, int io_dtype, const float* w, const float* bias,
                               const void* state_in, const int32_t* cu, int N, int64_t T, int C,
                               int K, void* y, void* state_out, int* status, cudaStream_t s) {
    if (io_dtype == GDN_BF16)
        return conv_dispatch_k<__nv_bfloat16>(K, x, w, bias, state_in, cu, N, T, C, y, state_out,
                                              status, s);
    return conv_dispatch_k<float>(K, x, w, bias, state_in, cu, N, T, C, y, state_out, status, s);
}

cudaError_t launch_conv1d_silu_decode(const void* x, int io_dtype, const float* w,
                                      const float* bias, void* state, const int32_t* slots,
                                      int num_slots, int N, int C, int K, void* y, int* status,
                                      cudaStream_t s) {
    if (io_dtype == GDN_BF16)
        return conv_decode_dispatch_k<__nv_bfloat16>(K, x, w, bias, state, slots, num_slots, N,
                                                     C, y, status, s);
    return conv_decode_dispatch_k<float>(K, x, w, bias, state, slots, num_slots, N, C, y,
                                         status, s);
}

cudaError_t launch_rmsnorm_gated(const void* o, const void* z, int io_dtype, const float* w,
                                 float eps, int64_t rows, int d, void* y, cudaStream_t s) {
    if (io_dtype == GDN_BF16)
        return d == 64 ? rms_launch<__nv_bfloat16, 64>(o, z, w, eps, rows, y, s)
                       : rms_launch<__nv_bfloat16, 128>(o, z, w, eps, rows, y, s);
    return d == 64 ? rms_launch<float, 64>(o, z, w, eps, rows, y, s)
                   : rms_launch<float, 128>(o, z, w, eps, rows, y, s);
}

}  // namespace gdn
