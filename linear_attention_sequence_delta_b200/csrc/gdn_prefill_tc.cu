// Chunked prefill on the 5th-generation tensor cores (tcgen05, bf16 in, fp32
// accumulate), d_k = d_v = 128, bf16 q/k/v/o.
//
// One 128-thread block per (sequence, V head) walks the sequence's 64-token
// chunks in order with the 128x128 fp32 state resident in tensor memory (TMEM
// lane i = value row i). The chunkwise form of the gated delta rule
// ("Qwen3.5-MoE-35B-A3B architecture teardown", 3.7 steps 3-6), written in the
// value-major orientation (S is d_v x d_k, o = S q) so that every matrix product
// has the 128 value rows, or the 128 rows [K; Q] of the chunk, as its M side:
//
//   G_t   = in-chunk cumulative log-decay, beta_t = write strength (computed here
//           from a, b, A_log, dt_bias: the gate prologue is fused in)
//   KQ    = [K^; Q^] (64 + 64 rows, L2-normalised, Q^ scaled)         (smem, bf16)
//   Dkq   = KQ K^^T          -> rows 0-63: K^K^^T, rows 64-127: Q^K^^T    (MMA)
//   A     = strictly-lower(beta_i exp(G_i - G_j) K^K^^T_ij);  T = (I + A)^-1
//   P     = lower(exp(G_t - G_s) Q^K^^T_ts)                                (bf16)
//   D1    = S0 KQ^T          -> cols 0-63: S0 K^^T,  cols 64-127: S0 Q^^T  (MMA)
//   Y^T   = (V - diag(e^G) (S0 K^^T)^T)^T diag(beta)                       (bf16)
//   Vn^T  = Y^T T^T                                                         (MMA)
//   O^T   = (S0 Q^^T) diag(e^G) + Vn^T P^T                                 (MMA)
//   S    <- e^{G_L} S + (Vn^T diag(e^{G_L - G})) K^                         (MMA)
//
// Only differences G_i - G_j with i >= j are exponentiated (directly, or as a
// product of two factors that are both <= 1), so nothing overflows.
//
// The triangular inverse T = (I + A)^-1 is computed in fp32 on the CUDA cores:
// the four 16x16 diagonal blocks by forward substitution in registers (lanes
// exchange finished rows by shuffles), then the off-diagonal blocks block-row by
// block-row, T_{a,<a} = -D_a (A_{a,<a} T_{<a,<a}).
//
// Every wait on an mbarrier is bounded; on expiry the block records
// GDN_ERR_TIMEOUT in the status word, drains its copies, frees its TMEM and exits.
#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {

namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kD = 128;
constexpr int kC = kChunk;  // 64
constexpr int kTCThreads = 128;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

// ---- shared memory map (byte offsets from a 1024-byte aligned base) -----------
constexpr uint32_t SM_KQ0 = 0;            // [2 col blocks][128 rows][128 B], sw128
constexpr uint32_t SM_KQ1 = 32768;
constexpr uint32_t SM_S0 = 65536;         // [2][128][128 B] bf16 state copy, sw128
constexpr uint32_t SM_YT = 98304;         // [128][128 B] Y^T (then scaled Vn^T), sw128
constexpr uint32_t SM_VNT = 114688;       // [128][128 B] Vn^T, sw128
constexpr uint32_t SM_TT = 131072;        // [64][128 B] T (bf16), sw128
constexpr uint32_t SM_PT = 139264;        // [64][128 B] P (bf16), sw128
constexpr uint32_t SM_V0 = 147456;        // [64 t][128 i] bf16, plain rows of 256 B
constexpr uint32_t SM_V1 = 163840;
constexpr uint32_t SM_AS = 180224;        // [64][65] fp32  A
constexpr uint32_t SM_TS = 196864;        // [64][65] fp32  T
constexpr uint32_t SM_SMALL = 213504;
// small region (floats unless noted)
constexpr uint32_t SMALL_A = 0;       // [2][64] raw a
constexpr uint32_t SMALL_B = 512;     // [2][64] raw b
constexpr uint32_t SMALL_GP = 1024;   // [64] partial scan
constexpr uint32_t SMALL_G = 1280;    // [64] G
constexpr uint32_t SMALL_BETA = 1536; // [64]
constexpr uint32_t SMALL_EG = 1792;   // [64] e^{G_t}
constexpr uint32_t SMALL_EGL = 2048;  // [64] e^{G_L - G_t}
constexpr uint32_t SMALL_U = 2304;    // [4][64] e^{G_{16a} - G_j}, j < 16a
constexpr uint32_t SMALL_BAR = 3328;  // uint64 mbarrier
constexpr uint32_t SMALL_TMEM = 3336; // uint32 TMEM base
constexpr uint32_t SMALL_ERR = 3340;  // int error flag
constexpr uint32_t SMALL_BYTES = 3344;
constexpr size_t kTCSmemBytes = SM_SMALL + SMALL_BYTES + 1024;  // + alignment slack

constexpr int kAsStride = 65;

// TMEM column map (512 columns allocated)
constexpr uint32_t TM_S = 0;      // 128 cols: state, fp32
constexpr uint32_t TM_D1 = 128;   // 128 cols: S0 K^^T | S0 Q^^T
constexpr uint32_t TM_DKQ = 256;  // 64 cols: [K^;Q^] K^^T
constexpr uint32_t TM_D34 = 320;  // 64 cols: Vn^T, then (P Vn)^T
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Write 64 fp32 values as one 128-byte bf16 row (row `row` of a sw128 tile).
__device__ __forceinline__ void st_row64_bf16(uint8_t* tile, uint32_t row, const float* x) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * ch + 0], x[8 * ch + 1]);
        w.y = pack_bf16x2(x[8 * ch + 2], x[8 * ch + 3]);
        w.z = pack_bf16x2(x[8 * ch + 4], x[8 * ch + 5]);
        w.w = pack_bf16x2(x[8 * ch + 6], x[8 * ch + 7]);
        *reinterpret_cast<uint4*>(tile + sw128_off(row, ch)) = w;
    }
}

__global__ void __launch_bounds__(kTCThreads, 1) prefill_tc_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
    const float* __restrict__ a, const float* __restrict__ b, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, const float* __restrict__ S0g,
    const int32_t* __restrict__ cu_seqlens, int64_t T_total, int H_qk, int H_v, float scale,
    bf16* __restrict__ o, float* __restrict__ Sfg, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* sA = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_A);
    float* sB = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_B);
    float* sGp = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_GP);
    float* sG = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_G);
    float* sBeta = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_BETA);
    float* sEG = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_EG);
    float* sEGL = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_EGL);
    float* sU = reinterpret_cast<float*>(sm + SM_SMALL + SMALL_U);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM_SMALL + SMALL_BAR);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + SM_SMALL + SMALL_TMEM);
    int* s_err = reinterpret_cast<int*>(sm + SM_SMALL + SMALL_ERR);
    float* As = reinterpret_cast<float*>(sm + SM_AS);
    float* Ts = reinterpret_cast<float*>(sm + SM_TS);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int h = blockIdx.x % H_v;
    const int n = blockIdx.x / H_v;
    const int j = h / (H_v / H_qk);

    const int64_t s0 = cu_seqlens[n];
    const int64_t s1 = cu_seqlens[n + 1];
    if (s0 < 0 || s1 < s0 || s1 > T_total || (n == 0 && s0 != 0)) {
        if (tid == 0) set_status(status, kStatusBadSeqlens);
        return;  // before any TMEM allocation
    }

    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        *s_err = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's lane quarter
    uint32_t phase = 0;

    // ---- initial state -> TMEM ---------------------------------------------------
    const size_t sbase = ((size_t)n * H_v + h) * kD * kD + (size_t)tid * kD;
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
        float x[32];
        if (S0g) {
            const float4* src = reinterpret_cast<const float4*>(S0g + sbase + 32 * cb);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 f = src[e];
                x[4 * e] = f.x; x[4 * e + 1] = f.y; x[4 * e + 2] = f.z; x[4 * e + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = 0.f;
        }
        tmem_st32(tl + TM_S + 32 * cb, x);
    }
    tmem_wait_st();

    const float Alog_h = A_log[h];
    const float dtb_h = dt_bias[h];
    const int64_t len = s1 - s0;
    const int nchunks = (int)((len + kC - 1) / kC);

    // async loads of chunk cc into stage st
    auto issue_loads = [&](int cc, int st) {
        const int64_t t0 = s0 + (int64_t)cc * kC;
        const int L = (int)min((int64_t)kC, s1 - t0);
        uint8_t* KQ = sm + (st ? SM_KQ1 : SM_KQ0);
        uint8_t* Vt = sm + (st ? SM_V1 : SM_V0);
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int idx = tid + kTCThreads * it;  // 0 .. 1023
            const int r = idx >> 4, ch = idx & 15;
            const bool ok = r < L;
            const int64_t tok = ok ? t0 + r : 0;
            const bf16* ks = k + ((size_t)tok * H_qk + j) * kD + ch * 8;
            const bf16* qs = q + ((size_t)tok * H_qk + j) * kD + ch * 8;
            const bf16* vs = v + ((size_t)tok * H_v + h) * kD + ch * 8;
            const uint32_t cboff = (uint32_t)(ch >> 3) * 16384u;
            cp_async_16(KQ + cboff + sw128_off(r, ch & 7), ks, ok ? 16u : 0u);
            cp_async_16(KQ + cboff + sw128_off(r + 64, ch & 7), qs, ok ? 16u : 0u);
            cp_async_16(Vt + r * 256 + ch * 16, vs, ok ? 16u : 0u);
        }
        if (tid < kC) {
            const bool ok = tid < L;
            const int64_t tok = ok ? t0 + tid : 0;
            cp_async_4(sA + st * 64 + tid, a + (size_t)tok * H_v + h, ok ? 4u : 0u);
        } else {
            const int t = tid - kC;
            const bool ok = t < L;
            const int64_t tok = ok ? t0 + t : 0;
            cp_async_4(sB + st * 64 + t, b + (size_t)tok * H_v + h, ok ? 4u : 0u);
        }
    };

    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar, phase, kWaitCycles);
        phase ^= 1u;
        if (!ok) *s_err = 1;
        __syncthreads();
        tc_fence_after();
        return *s_err == 0;
    };

    bool failed = false;
    if (nchunks > 0) issue_loads(0, 0);
    cp_async_commit();

#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const int64_t t0 = s0 + (int64_t)c * kC;
        const int L = (int)min((int64_t)kC, s1 - t0);
        uint8_t* KQ = sm + (st ? SM_KQ1 : SM_KQ0);
        const uint8_t* Vt = sm + (st ? SM_V1 : SM_V0);
        if (c + 1 < nchunks) issue_loads(c + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        // ---- gates: g, beta, in-chunk inclusive cumsum --------------------------
        if (tid < kC) {
            const bool ok = tid < L;
            float g = ok ? gate_g(sA[st * 64 + tid], Alog_h, dtb_h) : 0.f;
            sBeta[tid] = ok ? gate_beta(sB[st * 64 + tid]) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, g, off);
                if (lane >= off) g += y;
            }
            sGp[tid] = g;
        }
        __syncthreads();
        if (tid < kC) sG[tid] = sGp[tid] + (tid >= 32 ? sGp[31] : 0.f);
        __syncthreads();
        const float G_last = sG[kC - 1];  // = G_{L-1}: invalid tokens add g = 0
        if (tid < kC) {
            sEG[tid] = expf(sG[tid]);
            sEGL[tid] = expf(G_last - sG[tid]);
        }
        for (int idx = tid; idx < 4 * kC; idx += kTCThreads) {
            const int ab = idx >> 6, jj = idx & 63;
            sU[idx] = (jj < 16 * ab) ? expf(sG[16 * ab] - sG[jj]) : 0.f;
        }
        const float gamma = expf(G_last);

        // ---- L2-normalise K and Q rows in place (8 threads per row) -------------
#pragma unroll 1
        for (int pass = 0; pass < 8; ++pass) {
            const int r = pass * 16 + (tid >> 3);
            const int p = tid & 7;
            uint8_t* rowbase = KQ + (uint32_t)(p >> 2) * 16384u;
            uint4* c0 = reinterpret_cast<uint4*>(rowbase + sw128_off(r, (2 * p) & 7));
            uint4* c1 = reinterpret_cast<uint4*>(rowbase + sw128_off(r, (2 * p + 1) & 7));
            uint4 w0 = *c0, w1 = *c1;
            float f[16];
            const uint32_t* u0 = &w0.x;
            const uint32_t* u1 = &w1.x;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u0[e]));
                const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u1[e]));
                f[2 * e] = x0.x; f[2 * e + 1] = x0.y;
                f[8 + 2 * e] = x1.x; f[8 + 2 * e + 1] = x1.y;
            }
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) ss = fmaf(f[e], f[e], ss);
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            ss += __shfl_xor_sync(0xffffffffu, ss, 4);
            const float inv = (r >= 64 ? scale : 1.f) / sqrtf(ss + kL2Eps);
            w0.x = pack_bf16x2(f[0] * inv, f[1] * inv);
            w0.y = pack_bf16x2(f[2] * inv, f[3] * inv);
            w0.z = pack_bf16x2(f[4] * inv, f[5] * inv);
            w0.w = pack_bf16x2(f[6] * inv, f[7] * inv);
            w1.x = pack_bf16x2(f[8] * inv, f[9] * inv);
            w1.y = pack_bf16x2(f[10] * inv, f[11] * inv);
            w1.z = pack_bf16x2(f[12] * inv, f[13] * inv);
            w1.w = pack_bf16x2(f[14] * inv, f[15] * inv);
            *c0 = w0;
            *c1 = w1;
        }

        // ---- state: bf16 copy for the MMA, then S <- gamma S in TMEM -----------
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
            float x[32];
            tmem_ld32_sync(tl + TM_S + 32 * cb, x);
            uint8_t* tile = sm + SM_S0 + (uint32_t)(cb >> 1) * 16384u;
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
                uint4 w;
                w.x = pack_bf16x2(x[8 * qd + 0], x[8 * qd + 1]);
                w.y = pack_bf16x2(x[8 * qd + 2], x[8 * qd + 3]);
                w.z = pack_bf16x2(x[8 * qd + 4], x[8 * qd + 5]);
                w.w = pack_bf16x2(x[8 * qd + 6], x[8 * qd + 7]);
                *reinterpret_cast<uint4*>(tile + sw128_off(tid, (cb & 1) * 4 + qd)) = w;
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= gamma;
            tmem_st32(tl + TM_S + 32 * cb, x);
        }
        tmem_wait_st();

        // ---- MMA 1: Dkq = KQ K^^T, D1 = S0 KQ^T -----------------------------------
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t kq = smem_u32(KQ);
            const uint32_t s0t = smem_u32(sm + SM_S0);
            constexpr uint32_t id_kq = idesc_bf16_f32(128, 64, 0, 0);
            constexpr uint32_t id_d1 = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                mma_bf16_ss(tmem + TM_DKQ, smem_desc_sw128(kq + off, 16, 1024),
                            smem_desc_sw128(kq + off, 16, 1024), id_kq, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                mma_bf16_ss(tmem + TM_D1, smem_desc_sw128(s0t + off, 16, 1024),
                            smem_desc_sw128(kq + off, 16, 1024), id_d1, ks > 0);
            }
            mma_commit(bar);
        }
        if (!wait_mma()) { failed = true; break; }

        // ---- A (rows 0-63) and P (rows 64-127) from Dkq ---------------------------
        float Ad[16];
        {
            float x[64];
            tmem_ld64_sync(tl + TM_DKQ, x);
            const int i = tid & 63;              // row inside the 64-row block
            const int ab = i >> 4, a0 = ab * 16;
            const float Gi = sG[i];
            const float ci = expf(Gi - sG[a0]);
            if (tid < 64) {
                const float bi = sBeta[i];
                float* Arow = As + i * kAsStride;
#pragma unroll
                for (int jj = 0; jj < 64; ++jj) {
                    float val = 0.f;
                    if (jj < a0) val = bi * ci * sU[ab * 64 + jj] * x[jj];
                    else if (jj < i) val = bi * expf(Gi - sG[jj]) * x[jj];
                    Arow[jj] = val;
                }
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) Ad[r2] = Arow[a0 + r2];
            } else {
#pragma unroll
                for (int jj = 0; jj < 64; ++jj) {
                    float val = 0.f;
                    if (jj < a0) val = ci * sU[ab * 64 + jj] * x[jj];
                    else if (jj <= i) val = expf(Gi - sG[jj]) * x[jj];
                    x[jj] = i < L ? val : 0.f;
                }
                st_row64_bf16(sm + SM_PT, (uint32_t)i, x);
            }
        }
        __syncthreads();

        // ---- diagonal 16x16 blocks of T by forward substitution (warps 0-1) --------
        if (tid < 64) {
            const int i = tid;
            const int r = i & 15;
            const int a0 = i & ~15;
            const int src0 = lane & 16;
            float R[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) R[jj] = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float am = Ad[m];
#pragma unroll
                for (int jj = 0; jj < m; ++jj) {
                    const float tv = -__shfl_sync(0xffffffffu, R[jj], src0 | m);
                    if (r > m) R[jj] = fmaf(am, tv, R[jj]);
                }
                if (r > m) R[m] += am;
            }
            float* Trow = Ts + i * kAsStride;
#pragma unroll
            for (int jj = 0; jj < 64; ++jj) Trow[jj] = 0.f;
#pragma unroll
            for (int jl = 0; jl < 16; ++jl)
                Trow[a0 + jl] = jl < r ? -R[jl] : (jl == r ? 1.f : 0.f);
        }
        __syncthreads();

        // ---- off-diagonal blocks: T_{a,<a} = -D_a (A_{a,<a} T_{<a,<a}) ------------
        float* Xs = reinterpret_cast<float*>(sm + SM_YT);  // 16 x 48 fp32 scratch
#pragma unroll 1
        for (int ab = 1; ab < 4; ++ab) {
            const int a0 = ab * 16;
            for (int idx = tid; idx < 16 * a0; idx += kTCThreads) {
                const int r = idx / a0, jj = idx % a0;
                const float* Arow = As + (a0 + r) * kAsStride;
                float acc = 0.f;
                for (int m = jj; m < a0; ++m) acc = fmaf(Arow[m], Ts[m * kAsStride + jj], acc);
                Xs[r * 48 + jj] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < 16 * a0; idx += kTCThreads) {
                const int r = idx / a0, jj = idx % a0;
                const float* Drow = Ts + (a0 + r) * kAsStride + a0;
                float acc = 0.f;
                for (int r2 = 0; r2 <= r; ++r2) acc = fmaf(Drow[r2], Xs[r2 * 48 + jj], acc);
                Ts[(a0 + r) * kAsStride + jj] = -acc;
            }
            __syncthreads();
        }

        // ---- T -> bf16 tile ----------------------------------------------------------
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + kTCThreads * it;  // 0..511
            const int row = idx >> 3, ch = idx & 7;
            const float* src = Ts + row * kAsStride + ch * 8;
            uint4 w;
            w.x = pack_bf16x2(src[0], src[1]);
            w.y = pack_bf16x2(src[2], src[3]);
            w.z = pack_bf16x2(src[4], src[5]);
            w.w = pack_bf16x2(src[6], src[7]);
            *reinterpret_cast<uint4*>(sm + SM_TT + sw128_off(row, ch)) = w;
        }
        __syncthreads();  // Xs (in the Y^T buffer) fully consumed

        // ---- Y^T = beta (V - e^G X)^T, row i = tid ------------------------------------
        {
            float x[64];
            tmem_ld64_sync(tl + TM_D1, x);
            const bf16* vcol = reinterpret_cast<const bf16*>(Vt) + tid;
#pragma unroll
            for (int t = 0; t < 64; ++t) {
                const float vt = __bfloat162float(vcol[t * kD]);
                x[t] = sBeta[t] * (vt - sEG[t] * x[t]);
            }
            st_row64_bf16(sm + SM_YT, (uint32_t)tid, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            constexpr uint32_t id = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t yt = smem_u32(sm + SM_YT), tt = smem_u32(sm + SM_TT);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + TM_D34, smem_desc_sw128(yt + ks * 32, 16, 1024),
                            smem_desc_sw128(tt + ks * 32, 16, 1024), id, ks > 0);
            mma_commit(bar);
        }
        if (!wait_mma()) { failed = true; break; }

        // ---- Vn^T -> bf16 (and the decay-scaled copy for the state update) ----------
        {
            float x[64];
            tmem_ld64_sync(tl + TM_D34, x);
            st_row64_bf16(sm + SM_VNT, (uint32_t)tid, x);
#pragma unroll
            for (int t = 0; t < 64; ++t) x[t] *= sEGL[t];
            st_row64_bf16(sm + SM_YT, (uint32_t)tid, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            constexpr uint32_t id_o = idesc_bf16_f32(128, 64, 0, 0);
            constexpr uint32_t id_s = idesc_bf16_f32(128, 128, 0, 1);
            const uint32_t vnt = smem_u32(sm + SM_VNT), pt = smem_u32(sm + SM_PT);
            const uint32_t yt = smem_u32(sm + SM_YT), kq = smem_u32(KQ);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + TM_D34, smem_desc_sw128(vnt + ks * 32, 16, 1024),
                            smem_desc_sw128(pt + ks * 32, 16, 1024), id_o, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + TM_S, smem_desc_sw128(yt + ks * 32, 16, 1024),
                            smem_desc_sw128(kq + ks * 2048, 16384, 1024), id_s, 1);
            mma_commit(bar);
        }
        if (!wait_mma()) { failed = true; break; }

        // ---- O = e^G (Q S0^T) + P Vn -> global ---------------------------------------
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            float xq[32], xi[32];
            tmem_ld32_sync(tl + TM_D1 + 64 + 32 * half, xq);
            tmem_ld32_sync(tl + TM_D34 + 32 * half, xi);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int t = 32 * half + e;
                if (t < L)
                    o[((size_t)(t0 + t) * H_v + h) * kD + tid] =
                        __float2bfloat16_rn(fmaf(sEG[t], xq[e], xi[e]));
            }
        }
        __syncthreads();  // stage st free for the loads of chunk c + 2
    }

    cp_async_wait<0>();
    if (!failed && Sfg) {
        float* dst = Sfg + sbase;
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
            float x[32];
            tmem_ld32_sync(tl + TM_S + 32 * cb, x);
            float4* d4 = reinterpret_cast<float4*>(dst + 32 * cb);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
        }
    }
    if (failed && tid == 0) set_status(status, kStatusTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

size_t prefill_tc_smem_bytes() { return kTCSmemBytes; }

cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, const float* a,
                              const float* b, const float* A_log, const float* dt_bias,
                              const float* S0, const int32_t* cu_seqlens, int32_t N, int64_t T,
                              int32_t H_qk, int32_t H_v, float scale, void* o, float* S_final,
                              int* status, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTCSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)N * H_v;
    if (blocks == 0) return cudaSuccess;
    prefill_tc_kernel<<<(unsigned)blocks, kTCThreads, kTCSmemBytes, s>>>(
        static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), a,
        b, A_log, dt_bias, S0, cu_seqlens, T, H_qk, H_v, scale, static_cast<bf16*>(o), S_final,
        status);
    return cudaGetLastError();
}

}  // namespace gdn
