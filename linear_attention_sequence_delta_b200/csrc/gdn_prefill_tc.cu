// Chunked prefill on the 5th-generation tensor cores (tcgen05, bf16 in, fp32
// accumulate), d_k = d_v = 128, bf16 q/k/v/o.
//
// The chunkwise form of the gated delta rule ("Qwen3.5-MoE-35B-A3B architecture
// teardown", 3.7 steps 3-6), in the value-major orientation (S is d_v x d_k,
// o = S q) so that every matrix product has the 128 value rows, or the 128 rows
// [K; Q] of a chunk, as its M side. Per 64-token chunk with in-chunk cumulative
// log-decay G and write strengths beta:
//
//   KQ   = [K^; Q^]  (L2-normalised rows, Q^ scaled)                   smem bf16
//   Dkq  = KQ K^^T   -> rows 0-63: K^K^^T, rows 64-127: Q^K^^T          MMA
//   A    = strictly-lower(beta_i exp(G_i - G_j) K^K^^T_ij),  T = (I + A)^-1
//   P    = lower(exp(G_t - G_s) Q^K^^T_ts)                              bf16
//   D1   = S0 KQ^T   -> cols 0-63: S0 K^^T, cols 64-127: S0 Q^^T        MMA
//   Y^T  = (V - diag(e^G) (S0 K^^T)^T)^T diag(beta)                     bf16
//   Vn^T = Y^T T^T                                                       MMA
//   O^T  = (S0 Q^^T) diag(e^G) + Vn^T P^T                                MMA
//   S   <- e^{G_L} S + (Vn^T diag(e^{G_L - G})) K^                       MMA
//
// Only differences G_i - G_j with i >= j are exponentiated (directly, or as a
// product of two factors that are both <= 1), so nothing overflows however strong
// the decay.
//
// One block per (sequence, V head); three warp roles run concurrently:
//   loader (1 warp)   cp.async copies of the raw K, Q rows of a chunk (and its
//                     a, b) into a 3-deep ring, completion tracked by mbarriers;
//   prep   (4 warps)  everything that does not depend on the state, one chunk
//                     ahead: gates and their in-chunk cumsum, the L2 norms, the
//                     K^K^^T / Q^K^^T MMA, A and P, and T = (I + A)^-1 in fp32
//                     (16x16 diagonal blocks by forward substitution in
//                     registers, lanes exchanging finished rows by shuffles;
//                     then the off-diagonal blocks block-row by block-row,
//                     T_{a,<a} = -D_a (A_{a,<a} T_{<a,<a}));
//   chain  (4 warps)  the state-dependent steps in chunk order, with the 128x128
//                     fp32 state resident in tensor memory (lane i = value row i)
//                     and its bf16 copy kept in tensor memory as the A operand;
//                     V tiles are fetched by cp.async one chunk ahead (the
//                     loader warms L2 with them two chunks ahead); outputs are
//                     staged in shared memory and written as full 16-byte rows.
//
// Every wait is bounded; on expiry the block records GDN_ERR_TIMEOUT in the
// status word, every role leaves its loop at its next check, copies drain, the
// tensor memory is freed and the block exits.
#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {

namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kD = 128;
constexpr int kC = kChunk;  // 64
constexpr int kThreads = 288;   // warps 0-3 chain, 4-7 prep, 8 loader
constexpr int kRing = 3;        // depth of the K/Q ring
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

// ---- shared memory map (byte offsets from a 1024-byte aligned base) -----------
constexpr uint32_t SM_KQ = 0;             // kRing x [2 col blocks][128 rows][128 B], sw128
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t SM_YT = 98304;         // [128][128 B] Y^T, then scaled Vn^T (chain)
constexpr uint32_t SM_VNT = 114688;       // [128][128 B] Vn^T (chain)
constexpr uint32_t SM_T = 131072;         // 2 x [64][128 B] T (prep -> chain)
constexpr uint32_t SM_P = 147456;         // 2 x [64][128 B] P (prep -> chain)
constexpr uint32_t TP_BYTES = 8192;
constexpr uint32_t SM_TS = 163840;        // [64][68] fp32 T (prep scratch; rows 16-B aligned)
constexpr uint32_t SM_AS = 181248;        // [48][49] fp32 A rows 16..63, cols < 48
constexpr uint32_t SM_XS = 190656;        // [32][32] fp32 (prep scratch)
constexpr uint32_t SM_AB = 194752;        // kRing x (a[64], b[64]) fp32
constexpr uint32_t SM_GATE = 196288;      // 2 x gate slot
constexpr uint32_t GATE_BYTES = 2304;     //   G, beta, eG, eGL [64 each], U [4][64], gamma
constexpr uint32_t SM_GP = 200896;        // [64] fp32 scan partials (prep)
constexpr uint32_t SM_BAR = 201152;       // 12 mbarriers
constexpr uint32_t SM_TMEMADDR = 201248;
constexpr uint32_t SM_ERR = 201252;
constexpr uint32_t SM_V = 201728;         // [64 t][128 i] bf16 V tile (chain), plain 256-B rows
constexpr size_t kSmemBytes = 218112 + 1024;  // + alignment slack

// gate slot (floats)
constexpr int GS_G = 0, GS_BETA = 64, GS_EG = 128, GS_EGL = 192, GS_U = 256, GS_GAMMA = 512;

// barriers
constexpr int B_LOADED = 0;    // [3]  loader -> prep   (32 arrivals, cp.async)
constexpr int B_KQFREE = 3;    // [3]  chain -> loader
constexpr int B_READY = 6;     // [2]  prep -> chain
constexpr int B_TPFREE = 8;    // [2]  chain -> prep
constexpr int B_MMAP = 10;     //      prep's MMA completion
constexpr int B_MMAC = 11;     //      chain's MMA completion

// tensor memory columns (512 allocated)
constexpr uint32_t TM_S = 0;      // 128: state, fp32
constexpr uint32_t TM_S0B = 128;  // 64: state as bf16 pairs (MMA A operand)
constexpr uint32_t TM_D1 = 192;   // 128: S0 K^^T | S0 Q^^T
constexpr uint32_t TM_DKQ = 320;  // 64: [K^;Q^] K^^T (prep)
constexpr uint32_t TM_D34 = 384;  // 64: Vn^T, then (P Vn)^T
constexpr uint32_t kTmemCols = 512;

constexpr int kTsStride = 68;
constexpr int kAsStride = 49;

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

// Row i of A (rows 0-63) from row i of K^K^^T: the off-diagonal-block part
// (columns < a0) into As, the diagonal-block part into Ad. AB = i / 16.
template <int AB>
__device__ __forceinline__ void a_row(const float (&x)[64], int i, float bi, float ci,
                                      const float* G, const float* U, float* As, float (&Ad)[16]) {
    constexpr int a0 = 16 * AB;
    if constexpr (AB > 0) {
        float* Arow = As + (i - 16) * kAsStride;
#pragma unroll
        for (int jj = 0; jj < a0; ++jj) Arow[jj] = bi * ci * U[AB * 64 + jj] * x[jj];
    }
    const float Gi = G[i];
#pragma unroll
    for (int r2 = 0; r2 < 16; ++r2)
        Ad[r2] = (a0 + r2 < i) ? bi * __expf(Gi - G[a0 + r2]) * x[a0 + r2] : 0.f;
}

// Row t of P from row t of Q^K^^T, rows >= L zeroed, as bf16 into the P tile.
template <int AB>
__device__ __forceinline__ void p_row(float (&x)[64], int t, int L, float ci, const float* G,
                                      const float* U, uint8_t* Ptile) {
    constexpr int a0 = 16 * AB;
    const float Gt = G[t];
    const bool live = t < L;
#pragma unroll
    for (int jj = 0; jj < 64; ++jj) {
        float val = 0.f;
        if (jj < a0) val = ci * U[AB * 64 + jj] * x[jj];
        else if (jj < a0 + 16) val = (jj <= t) ? __expf(Gt - G[jj]) * x[jj] : 0.f;
        x[jj] = live ? val : 0.f;
    }
    st_row64_bf16(Ptile, (uint32_t)t, x);
}

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
    const float* __restrict__ a, const float* __restrict__ b, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, const float* __restrict__ S0g,
    const int32_t* __restrict__ cu_seqlens, int64_t T_total, int H_qk, int H_v, float scale,
    bf16* __restrict__ o, float* __restrict__ Sfg, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + SM_TMEMADDR);
    volatile int* s_err = reinterpret_cast<volatile int*>(sm + SM_ERR);

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
        return;  // uniform across the block, before any allocation
    }
    const int nchunks = (int)((s1 - s0 + kC - 1) / kC);

    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[B_LOADED + i], 32);
        for (int i = 0; i < 3; ++i) mbar_init(&bars[B_KQFREE + i], 1);
        for (int i = 0; i < 2; ++i) mbar_init(&bars[B_READY + i], 1);
        for (int i = 0; i < 2; ++i) mbar_init(&bars[B_TPFREE + i], 1);
        mbar_init(&bars[B_MMAP], 1);
        mbar_init(&bars[B_MMAC], 1);
        *s_err = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 8) {
        // ============================ loader =========================================
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kRing;
            bool ok = true;
            if (c >= kRing)
                ok = mbar_wait_bounded(&bars[B_KQFREE + s], ((c / kRing) - 1) & 1, kWaitCycles);
            if (!ok) *s_err = 1;
            __syncwarp();
            if (*s_err) break;
            const int64_t t0 = s0 + (int64_t)c * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
            uint8_t* KQ = sm + SM_KQ + s * KQ_BYTES;
#pragma unroll 4
            for (int it = 0; it < 32; ++it) {
                const int idx = lane + 32 * it;  // 0 .. 1023
                const int r = idx >> 4, ch = idx & 15;
                const bool live = r < L;
                const int64_t tok = live ? t0 + r : 0;
                const size_t rowk = ((size_t)tok * H_qk + j) * kD + ch * 8;
                const uint32_t off = (uint32_t)(ch >> 3) * 16384u;
                cp_async_16(KQ + off + sw128_off(r, ch & 7), k + rowk, live ? 16u : 0u);
                cp_async_16(KQ + off + sw128_off(r + 64, ch & 7), q + rowk, live ? 16u : 0u);
            }
            // V rows of this chunk (read later by the chain straight from global
            // memory): bring them into L2 now, two 128-byte lines per row.
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int idx = lane + 32 * it;  // 0 .. 127
                const int r = idx >> 1;
                if (r < L) {
                    const bf16* vp = v + ((size_t)(t0 + r) * H_v + h) * kD + (idx & 1) * 64;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(vp));
                }
            }
            float* ab = reinterpret_cast<float*>(sm + SM_AB) + s * 128;
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const int t = lane + 32 * hlf;
                const bool live = t < L;
                const int64_t tok = live ? t0 + t : 0;
                cp_async_4(ab + t, a + (size_t)tok * H_v + h, live ? 4u : 0u);
                cp_async_4(ab + 64 + t, b + (size_t)tok * H_v + h, live ? 4u : 0u);
            }
            cp_async_mbar_arrive_noinc(&bars[B_LOADED + s]);
        }
        cp_async_commit();
        cp_async_wait<0>();
    } else if (warp >= 4) {
        // ============================== prep =========================================
        const int pt = tid - 128;
        const int pw = warp - 4;
        const uint32_t ptl = tmem + ((uint32_t)(pw * 32) << 16);
        float* Ts = reinterpret_cast<float*>(sm + SM_TS);
        float* As = reinterpret_cast<float*>(sm + SM_AS);
        float* Xs = reinterpret_cast<float*>(sm + SM_XS);
        float* Gp = reinterpret_cast<float*>(sm + SM_GP);
        const float Alog_h = A_log[h];
        const float dtb_h = dt_bias[h];
        uint32_t mphase = 0;
        // Entries of T above the diagonal blocks are never written: zero them once.
        for (int idx = pt; idx < 64 * kTsStride; idx += 128) Ts[idx] = 0.f;
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kRing;
            const int p = c & 1;
            bool ok = mbar_wait_bounded(&bars[B_LOADED + s], (c / kRing) & 1, kWaitCycles);
            if (ok && c >= 2)
                ok = mbar_wait_bounded(&bars[B_TPFREE + p], ((c >> 1) - 1) & 1, kWaitCycles);
            if (!ok) *s_err = 1;
            named_bar_sync(2, 128);
            if (*s_err) break;
            const int64_t t0 = s0 + (int64_t)c * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
            uint8_t* KQ = sm + SM_KQ + s * KQ_BYTES;
            const float* ab = reinterpret_cast<const float*>(sm + SM_AB) + s * 128;
            float* gs = reinterpret_cast<float*>(sm + SM_GATE + p * GATE_BYTES);
            float* sG = gs + GS_G;
            float* sBeta = gs + GS_BETA;
            float* sU = gs + GS_U;

            // ---- gates: g, beta and a per-warp inclusive scan of g -----------------
            if (pt < kC) {
                const bool live = pt < L;
                float g = live ? gate_g(ab[pt], Alog_h, dtb_h) : 0.f;
                sBeta[pt] = live ? gate_beta(ab[64 + pt]) : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, g, off);
                    if (lane >= off) g += y;
                }
                Gp[pt] = g;
            }

            // ---- L2-normalise K and Q rows in place, one row per thread ------------
            {
                const int r = pt;
                uint4 w[16];
                float ss = 0.f;
#pragma unroll
                for (int ch = 0; ch < 16; ++ch) {
                    w[ch] = *reinterpret_cast<const uint4*>(KQ + (uint32_t)(ch >> 3) * 16384u +
                                                            sw128_off(r, ch & 7));
                    const uint32_t* u = &w[ch].x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x2 =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
                        ss = fmaf(x2.x, x2.x, ss);
                        ss = fmaf(x2.y, x2.y, ss);
                    }
                }
                const float inv = (r >= 64 ? scale : 1.f) / sqrtf(ss + kL2Eps);
#pragma unroll
                for (int ch = 0; ch < 16; ++ch) {
                    uint32_t* u = &w[ch].x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x2 =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
                        u[e] = pack_bf16x2(x2.x * inv, x2.y * inv);
                    }
                    *reinterpret_cast<uint4*>(KQ + (uint32_t)(ch >> 3) * 16384u +
                                              sw128_off(r, ch & 7)) = w[ch];
                }
            }

            // ---- Dkq = KQ K^^T (overlapped with the rest of the gate arithmetic) ----
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, 128);
            tc_fence_after();
            if (pt == 0) {
                const uint32_t kq = smem_u32(KQ);
                constexpr uint32_t id_kq = idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                    mma_bf16_ss(tmem + TM_DKQ, smem_desc_sw128(kq + off, 16, 1024),
                                smem_desc_sw128(kq + off, 16, 1024), id_kq, ks > 0);
                }
                mma_commit(&bars[B_MMAP]);
            }
            if (pt < kC) sG[pt] = Gp[pt] + (pt >= 32 ? Gp[31] : 0.f);
            named_bar_sync(2, 128);
            const float G_last = sG[kC - 1];  // = G_{L-1}: tokens past L add g = 0
            if (pt < kC) {
                gs[GS_EG + pt] = __expf(sG[pt]);
                gs[GS_EGL + pt] = __expf(G_last - sG[pt]);
            }
            for (int idx = pt; idx < 4 * kC; idx += 128) {
                const int ab4 = idx >> 6, jj = idx & 63;
                sU[idx] = (jj < 16 * ab4) ? __expf(sG[16 * ab4] - sG[jj]) : 0.f;
            }
            if (pt == 0) gs[GS_GAMMA] = __expf(G_last);
            ok = mbar_wait_bounded(&bars[B_MMAP], mphase, kWaitCycles);
            mphase ^= 1u;
            if (!ok) *s_err = 1;
            named_bar_sync(2, 128);
            if (*s_err) break;
            tc_fence_after();

            // ---- A (prep warps 0-1) and P (prep warps 2-3) ---------------------------
            float Ad[16];
            {
                float x[64];
                tmem_ld64_sync(ptl + TM_DKQ, x);
                const int i = pt & 63;
                const int a0 = i & ~15;
                const float ci = __expf(sG[i] - sG[a0]);
                if (pt < 64) {
                    const float bi = sBeta[i];
                    switch (i >> 4) {
                        case 0: a_row<0>(x, i, bi, ci, sG, sU, As, Ad); break;
                        case 1: a_row<1>(x, i, bi, ci, sG, sU, As, Ad); break;
                        case 2: a_row<2>(x, i, bi, ci, sG, sU, As, Ad); break;
                        default: a_row<3>(x, i, bi, ci, sG, sU, As, Ad); break;
                    }
                } else {
                    uint8_t* Pt = sm + SM_P + p * TP_BYTES;
                    switch (i >> 4) {
                        case 0: p_row<0>(x, i, L, ci, sG, sU, Pt); break;
                        case 1: p_row<1>(x, i, L, ci, sG, sU, Pt); break;
                        case 2: p_row<2>(x, i, L, ci, sG, sU, Pt); break;
                        default: p_row<3>(x, i, L, ci, sG, sU, Pt); break;
                    }
                }
            }

            // ---- diagonal 16x16 blocks of T: forward substitution in registers -----
            if (pt < 64) {
                const int i = pt;
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
                float* Trow = Ts + i * kTsStride;
#pragma unroll
                for (int jl = 0; jl < 16; ++jl)
                    Trow[a0 + jl] = jl < r ? -R[jl] : (jl == r ? 1.f : 0.f);
            }
            named_bar_sync(2, 128);

            // ---- off-diagonal blocks by doubling ------------------------------------
            // stage 1: T_10 = -D_1 A_10 D_0 and T_32 = -D_3 A_32 D_2 (16x16 blocks)
            {
                const int which = pt >> 6;              // 0: T_10, 1: T_32
                const int q4 = pt & 63;
                const int r = q4 >> 2, c0 = (q4 & 3) * 4;
                const int cb = which ? 32 : 0;          // column block of A / D_in
                const int rb = which ? 48 : 16;         // row block of A / D_out
                const float* Arow = As + (rb + r - 16) * kAsStride + cb;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float am = Arow[m];
                    const float4 d = *reinterpret_cast<const float4*>(Ts + (cb + m) * kTsStride + cb + c0);
                    acc[0] = fmaf(am, d.x, acc[0]);
                    acc[1] = fmaf(am, d.y, acc[1]);
                    acc[2] = fmaf(am, d.z, acc[2]);
                    acc[3] = fmaf(am, d.w, acc[3]);
                }
                *reinterpret_cast<float4*>(Xs + which * 256 + r * 16 + c0) =
                    make_float4(acc[0], acc[1], acc[2], acc[3]);
                named_bar_sync(2, 128);
                const float* Drow = Ts + (rb + r) * kTsStride + rb;
                float t4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float dm = Drow[m];
                    const float4 xv = *reinterpret_cast<const float4*>(Xs + which * 256 + m * 16 + c0);
                    t4[0] = fmaf(dm, xv.x, t4[0]);
                    t4[1] = fmaf(dm, xv.y, t4[1]);
                    t4[2] = fmaf(dm, xv.z, t4[2]);
                    t4[3] = fmaf(dm, xv.w, t4[3]);
                }
                *reinterpret_cast<float4*>(Ts + (rb + r) * kTsStride + cb + c0) =
                    make_float4(-t4[0], -t4[1], -t4[2], -t4[3]);
            }
            named_bar_sync(2, 128);
            // stage 2: T[32:64, 0:32] = -T[32:64,32:64] (A[32:64, 0:32] T[0:32, 0:32])
            {
                const int r = pt >> 2, c0 = (pt & 3) * 8;
                const float* Arow = As + (16 + r) * kAsStride;
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const float am = Arow[m];
                    const float4 d0 = *reinterpret_cast<const float4*>(Ts + m * kTsStride + c0);
                    const float4 d1 = *reinterpret_cast<const float4*>(Ts + m * kTsStride + c0 + 4);
                    acc[0] = fmaf(am, d0.x, acc[0]); acc[1] = fmaf(am, d0.y, acc[1]);
                    acc[2] = fmaf(am, d0.z, acc[2]); acc[3] = fmaf(am, d0.w, acc[3]);
                    acc[4] = fmaf(am, d1.x, acc[4]); acc[5] = fmaf(am, d1.y, acc[5]);
                    acc[6] = fmaf(am, d1.z, acc[6]); acc[7] = fmaf(am, d1.w, acc[7]);
                }
                *reinterpret_cast<float4*>(Xs + r * 32 + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                *reinterpret_cast<float4*>(Xs + r * 32 + c0 + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
                named_bar_sync(2, 128);
                const float* Drow = Ts + (32 + r) * kTsStride + 32;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const float dm = Drow[m];
                    const float4 x0 = *reinterpret_cast<const float4*>(Xs + m * 32 + c0);
                    const float4 x1 = *reinterpret_cast<const float4*>(Xs + m * 32 + c0 + 4);
                    acc[0] = fmaf(dm, x0.x, acc[0]); acc[1] = fmaf(dm, x0.y, acc[1]);
                    acc[2] = fmaf(dm, x0.z, acc[2]); acc[3] = fmaf(dm, x0.w, acc[3]);
                    acc[4] = fmaf(dm, x1.x, acc[4]); acc[5] = fmaf(dm, x1.y, acc[5]);
                    acc[6] = fmaf(dm, x1.z, acc[6]); acc[7] = fmaf(dm, x1.w, acc[7]);
                }
                float* dst = Ts + (32 + r) * kTsStride + c0;
                *reinterpret_cast<float4*>(dst) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(-acc[4], -acc[5], -acc[6], -acc[7]);
            }
            named_bar_sync(2, 128);

            // ---- T -> bf16 tile; hand the chunk to the chain ------------------------
            uint8_t* Tt = sm + SM_T + p * TP_BYTES;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int idx = pt + 128 * it;  // 0..511
                const int row = idx >> 3, ch = idx & 7;
                const float* src = Ts + row * kTsStride + ch * 8;
                uint4 w;
                w.x = pack_bf16x2(src[0], src[1]);
                w.y = pack_bf16x2(src[2], src[3]);
                w.z = pack_bf16x2(src[4], src[5]);
                w.w = pack_bf16x2(src[6], src[7]);
                *reinterpret_cast<uint4*>(Tt + sw128_off(row, ch)) = w;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, 128);
            if (pt == 0) mbar_arrive(&bars[B_READY + p]);
        }
    } else {
        // ============================== chain ========================================
        const uint32_t ctl = tmem + ((uint32_t)(warp * 32) << 16);
        const size_t sbase = ((size_t)n * H_v + h) * kD * kD + (size_t)tid * kD;
        // initial state -> TMEM
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
            tmem_st32(ctl + TM_S + 32 * cb, x);
        }
        tmem_wait_st();

        // V rows of a chunk into the V tile ([t][i], 256-byte rows); rows past the
        // end of the sequence are zero-filled.
        uint8_t* Vt = sm + SM_V;
        auto load_v = [&](int cc) {
            const int64_t t0 = s0 + (int64_t)cc * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int idx = tid + 128 * it;  // 0 .. 1023
                const int r = idx >> 4, ch = idx & 15;
                const bool live = r < L;
                const int64_t tok = live ? t0 + r : 0;
                cp_async_16(Vt + r * 256 + ch * 16, v + ((size_t)tok * H_v + h) * kD + ch * 8,
                            live ? 16u : 0u);
            }
            cp_async_commit();
        };
        if (nchunks > 0) load_v(0);

        uint32_t mphase = 0;
        auto chain_mma_wait = [&]() -> bool {
            const bool ok = mbar_wait_bounded(&bars[B_MMAC], mphase, kWaitCycles);
            mphase ^= 1u;
            if (!ok) *s_err = 1;
            named_bar_sync(1, 128);
            tc_fence_after();
            return *s_err == 0;
        };

#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kRing;
            const int p = c & 1;
            const bool ok = mbar_wait_bounded(&bars[B_READY + p], (c >> 1) & 1, kWaitCycles);
            if (!ok) *s_err = 1;
            named_bar_sync(1, 128);
            if (*s_err) break;
            const int64_t t0 = s0 + (int64_t)c * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
            const float* gs = reinterpret_cast<const float*>(sm + SM_GATE + p * GATE_BYTES);
            const uint32_t kq = smem_u32(sm + SM_KQ + s * KQ_BYTES);

            // ---- state: bf16 copy (MMA operand), then S <- gamma S ------------------
            const float gamma = gs[GS_GAMMA];
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                float x[32];
                tmem_ld32_sync(ctl + TM_S + 32 * cb, x);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
                tmem_st16(ctl + TM_S0B + 16 * cb, pk);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= gamma;
                tmem_st32(ctl + TM_S + 32 * cb, x);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(1, 128);
            tc_fence_after();
            if (tid == 0) {
                constexpr uint32_t id_d1 = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                    mma_bf16_ts(tmem + TM_D1, tmem + TM_S0B + 8 * ks,
                                smem_desc_sw128(kq + off, 16, 1024), id_d1, ks > 0);
                }
                mma_commit(&bars[B_MMAC]);
            }
            cp_async_wait<0>();  // this chunk's V tile (issued one chunk earlier)
            if (!chain_mma_wait()) break;

            // ---- Y^T = beta (V - e^G X)^T, row i = tid --------------------------------
            {
                float x[64];
                tmem_ld64_sync(ctl + TM_D1, x);
                const bf16* vcol = reinterpret_cast<const bf16*>(Vt) + tid;
#pragma unroll
                for (int t = 0; t < 64; ++t)
                    x[t] = gs[GS_BETA + t] * (__bfloat162float(vcol[t * kD]) - gs[GS_EG + t] * x[t]);
                st_row64_bf16(sm + SM_YT, (uint32_t)tid, x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            tc_fence_after();
            if (c + 1 < nchunks) load_v(c + 1);  // V tile consumed: fetch the next one
            if (tid == 0) {
                constexpr uint32_t id = idesc_bf16_f32(128, 64, 0, 0);
                const uint32_t yt = smem_u32(sm + SM_YT);
                const uint32_t tt = smem_u32(sm + SM_T + p * TP_BYTES);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tmem + TM_D34, smem_desc_sw128(yt + ks * 32, 16, 1024),
                                smem_desc_sw128(tt + ks * 32, 16, 1024), id, ks > 0);
                mma_commit(&bars[B_MMAC]);
            }
            if (!chain_mma_wait()) break;

            // ---- Vn^T -> bf16, and the decay-scaled copy for the state update ----------
            {
                float x[64];
                tmem_ld64_sync(ctl + TM_D34, x);
                st_row64_bf16(sm + SM_VNT, (uint32_t)tid, x);
#pragma unroll
                for (int t = 0; t < 64; ++t) x[t] *= gs[GS_EGL + t];
                st_row64_bf16(sm + SM_YT, (uint32_t)tid, x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            tc_fence_after();
            if (tid == 0) {
                constexpr uint32_t id_o = idesc_bf16_f32(128, 64, 0, 0);
                constexpr uint32_t id_s = idesc_bf16_f32(128, 128, 0, 1);
                const uint32_t vnt = smem_u32(sm + SM_VNT);
                const uint32_t ptile = smem_u32(sm + SM_P + p * TP_BYTES);
                const uint32_t yt = smem_u32(sm + SM_YT);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tmem + TM_D34, smem_desc_sw128(vnt + ks * 32, 16, 1024),
                                smem_desc_sw128(ptile + ks * 32, 16, 1024), id_o, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tmem + TM_S, smem_desc_sw128(yt + ks * 32, 16, 1024),
                                smem_desc_sw128(kq + ks * 2048, 16384, 1024), id_s, 1);
                mma_commit(&bars[B_MMAC]);
            }
            if (!chain_mma_wait()) break;
            if (tid == 0) {  // the MMAs reading T, P and this K/Q slot are complete
                mbar_arrive(&bars[B_TPFREE + p]);
                mbar_arrive(&bars[B_KQFREE + s]);
            }

            // ---- O = e^G (Q S0^T) + P Vn: staged as [t][i] rows, then 16-byte stores ----
            uint16_t* Ost = reinterpret_cast<uint16_t*>(sm + SM_VNT);  // Vn^T tile is free now
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float xq[32], xi[32];
                tmem_ld32_sync(ctl + TM_D1 + 64 + 32 * half, xq);
                tmem_ld32_sync(ctl + TM_D34 + 32 * half, xi);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int t = 32 * half + e;
                    const bf16 ov = __float2bfloat16_rn(fmaf(gs[GS_EG + t], xq[e], xi[e]));
                    Ost[t * kD + tid] = *reinterpret_cast<const uint16_t*>(&ov);
                }
            }
            named_bar_sync(1, 128);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int idx = tid + 128 * it;  // 0 .. 1023
                const int t = idx >> 4, ch = idx & 15;
                if (t < L)
                    *reinterpret_cast<uint4*>(o + ((size_t)(t0 + t) * H_v + h) * kD + ch * 8) =
                        *reinterpret_cast<const uint4*>(Ost + t * kD + ch * 8);
            }
        }
        if (!*s_err && Sfg) {
            float* dst = Sfg + sbase;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                float x[32];
                tmem_ld32_sync(ctl + TM_S + 32 * cb, x);
                float4* d4 = reinterpret_cast<float4*>(dst + 32 * cb);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && *s_err) set_status(status, kStatusTimeout);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, const float* a,
                              const float* b, const float* A_log, const float* dt_bias,
                              const float* S0, const int32_t* cu_seqlens, int32_t N, int64_t T,
                              int32_t H_qk, int32_t H_v, float scale, void* o, float* S_final,
                              int* status, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)N * H_v;
    if (blocks == 0) return cudaSuccess;
    prefill_tc_kernel<<<(unsigned)blocks, kThreads, kSmemBytes, s>>>(
        static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), a,
        b, A_log, dt_bias, S0, cu_seqlens, T, H_qk, H_v, scale, static_cast<bf16*>(o), S_final,
        status);
    return cudaGetLastError();
}

}  // namespace gdn
