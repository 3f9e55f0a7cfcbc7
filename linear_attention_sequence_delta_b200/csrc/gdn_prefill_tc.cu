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
// One block per (sequence, V head); two warp roles run concurrently:
//   prep   (8 warps)  everything that does not depend on the state, one chunk
//                     ahead: gates and their in-chunk cumsum, the L2 norms, the
//                     K^K^^T / Q^K^^T MMA, A and P, and T = (I + A)^-1 in fp32:
//                     the 8x8 diagonal blocks by forward substitution in
//                     registers (lanes exchange finished rows by shuffles), then
//                     three doubling steps 8 -> 16 -> 32 -> 64, each block pair
//                     merged as T_{10} = -D_1 A_{10} D_0;
//   chain  (4 warps)  the state-dependent steps in chunk order, with the 128x128
//                     fp32 state resident in tensor memory (lane i = value row i).
//                     Every A operand of its MMAs (the bf16 state, Y^T, Vn^T and
//                     the decay-scaled Vn^T) is written to tensor memory by the
//                     threads that own those rows, and V^T itself is produced in
//                     tensor memory by one MMA against an identity tile, so the
//                     chain reads no operand row-by-row from shared memory.
//                     It also issues the cp.async copies: the K/Q rows and gates
//                     of chunk c + 3 into a 3-deep ring as soon as chunk c has
//                     released its slot (completion tracked by mbarriers), and
//                     the V tile of chunk c + 1. Outputs are staged in shared
//                     memory and written as full 16-byte rows.
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
constexpr int kC = kChunk;       // 64
constexpr int kThreads = 384;    // warps 0-3 chain, 4-11 prep
constexpr int kPrep = 256;
constexpr int kRing = 3;         // depth of the K/Q ring
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

// ---- shared memory map (byte offsets from a 1024-byte aligned base) -----------
constexpr uint32_t SM_KQ = 0;             // kRing x [2 col blocks][128 rows][128 B], sw128
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t SM_ID = 98304;         // [64][128 B] bf16 identity, sw128 (chain)
constexpr uint32_t SM_VNT = 114688;       // [64 t][128 i] bf16 O staging (chain)
constexpr uint32_t SM_T = 131072;         // 2 x [64][128 B] T (prep -> chain)
constexpr uint32_t SM_P = 147456;         // 2 x [64][128 B] P (prep -> chain)
constexpr uint32_t TP_BYTES = 8192;
constexpr uint32_t SM_TS = 163840;        // [64][68] fp32 T (prep; rows 16-byte aligned)
constexpr uint32_t SM_AS = 181248;        // [64][68] fp32 A, strictly-lower part used (prep)
constexpr uint32_t SM_XS = 198656;        // [1024] fp32 merge scratch (prep)
constexpr uint32_t SM_AB = 202752;        // kRing x (a[64], b[64]) fp32
constexpr uint32_t SM_GATE = 204288;      // 2 x gate slot
constexpr uint32_t GATE_BYTES = 2816;
constexpr uint32_t SM_GP = 209920;        // [64] fp32 scan partials (prep)
constexpr uint32_t SM_BAR = 210176;       // mbarriers
constexpr uint32_t SM_TMEMADDR = 210272;
constexpr uint32_t SM_ERR = 210276;
constexpr uint32_t SM_V = 210944;         // [2 col blocks][64 t][128 B] bf16 V tile, sw128 (chain)
constexpr size_t kSmemBytes = 227328 + 1024;  // + alignment slack

// gate slot (floats)
constexpr int GS_G = 0, GS_BETA = 64, GS_EG = 128, GS_EGL = 192, GS_U = 256, GS_GAMMA = 512,
              GS_BBE = 516;  // [64] x (beta_t, beta_t e^{G_t})

// barriers
constexpr int B_LOADED = 0;    // [3]  chain's cp.async copies -> prep (128 arrivals)
constexpr int B_READY = 3;     // [2]  prep -> chain
constexpr int B_TPFREE = 5;    // [2]  chain -> prep
constexpr int B_MMAP = 7;      //      prep's MMA completion
constexpr int B_MMAC = 8;      //      chain's MMA completion

// tensor memory columns (512 allocated)
constexpr uint32_t TM_S = 0;      // 128: state, fp32
constexpr uint32_t TM_S0B = 128;  // 64: state as bf16 pairs (MMA A operand)
constexpr uint32_t TM_D1 = 192;   // 128: S0 K^^T | S0 Q^^T; then Y^T as bf16 pairs in 192..223
constexpr uint32_t TM_DKQ = 320;  // 64: [K^;Q^] K^^T (prep)
constexpr uint32_t TM_D34 = 384;  // 64: Vn^T, then (P Vn)^T
constexpr uint32_t TM_DV = 448;   // 64: V^T; then Vn^T (448..479) and scaled Vn^T (480..511), bf16
constexpr uint32_t kTmemCols = 512;

constexpr int kTsStride = 68;
constexpr int kAsStride = 68;

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

// Half a row (32 columns starting at 32 H) of A (row i < 64) or of P (row t =
// i - 64), from the matching half row x of [K^;Q^] K^^T. Columns left of the
// row's 16-block use exp(G_i - G_j) = exp(G_i - G_a0) U_j (both factors <= 1);
// the at most 16 columns inside the block take their own exponential; columns
// right of the row are zero. A goes to As (fp32; its diagonal and upper entries
// are never read); P goes to the P tile as bf16 (rows >= L zero).
template <int H>
__device__ __forceinline__ void ap_half_row(const float (&x)[32], int row, int L, const float* G,
                                            const float* beta, const float* U, float* As,
                                            uint8_t* Ptile) {
    const int i = row & 63;
    const int a0 = i & ~15;
    const float Gi = G[i];
    const float ci = __expf(Gi - G[a0]);
    const float* Urow = U + (a0 >> 4) * 64 + 32 * H;
    const float* Gc = G + 32 * H;
    float val[32];
    if (a0 >= 32 * H + 32) {          // the whole half is left of the row's block
#pragma unroll
        for (int e = 0; e < 32; ++e) val[e] = ci * Urow[e] * x[e];
    } else if (a0 == 32 * H + 16) {   // 16 columns left of the block, then the block
#pragma unroll
        for (int e = 0; e < 16; ++e) val[e] = ci * Urow[e] * x[e];
#pragma unroll
        for (int e = 16; e < 32; ++e) val[e] = (32 * H + e <= i) ? __expf(Gi - Gc[e]) * x[e] : 0.f;
    } else if (a0 == 32 * H) {        // the block, then columns right of the row
#pragma unroll
        for (int e = 0; e < 16; ++e) val[e] = (32 * H + e <= i) ? __expf(Gi - Gc[e]) * x[e] : 0.f;
#pragma unroll
        for (int e = 16; e < 32; ++e) val[e] = 0.f;
    } else {                          // the whole half is right of the row
#pragma unroll
        for (int e = 0; e < 32; ++e) val[e] = 0.f;
    }
    if (row < 64) {
        const float bi = beta[i];
        float4* Arow = reinterpret_cast<float4*>(As + i * kAsStride + 32 * H);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4)
            Arow[e4] = make_float4(bi * val[4 * e4], bi * val[4 * e4 + 1], bi * val[4 * e4 + 2],
                                   bi * val[4 * e4 + 3]);
    } else {
        const bool live = i < L;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = live ? pack_bf16x2(val[8 * q4 + 0], val[8 * q4 + 1]) : 0u;
            w.y = live ? pack_bf16x2(val[8 * q4 + 2], val[8 * q4 + 3]) : 0u;
            w.z = live ? pack_bf16x2(val[8 * q4 + 4], val[8 * q4 + 5]) : 0u;
            w.w = live ? pack_bf16x2(val[8 * q4 + 6], val[8 * q4 + 7]) : 0u;
            *reinterpret_cast<uint4*>(Ptile + sw128_off((uint32_t)i, 4 * H + q4)) = w;
        }
    }
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
        for (int i = 0; i < kRing; ++i) mbar_init(&bars[B_LOADED + i], 128);
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

    if (warp >= 4) {
        // ============================== prep =========================================
        const int pt = tid - 128;           // 0 .. 255
        const int pw = warp - 4;            // 0 .. 7
        const int hh = pw >> 2;             // which half of the 64 columns
        const uint32_t ptl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int trow = (warp & 3) * 32 + lane;  // this thread's TMEM lane
        float* Ts = reinterpret_cast<float*>(sm + SM_TS);
        float* As = reinterpret_cast<float*>(sm + SM_AS);
        float* Xs = reinterpret_cast<float*>(sm + SM_XS);
        float* Gp = reinterpret_cast<float*>(sm + SM_GP);
        const float Alog_h = A_log[h];
        const float dtb_h = dt_bias[h];
        uint32_t mphase = 0;
        // Entries of T above the diagonal blocks are never written: zero them once.
        for (int idx = pt; idx < 64 * kTsStride; idx += kPrep) Ts[idx] = 0.f;
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kRing;
            const int p = c & 1;
            bool ok = mbar_wait_bounded(&bars[B_LOADED + s], (c / kRing) & 1, kWaitCycles);
            if (ok && c >= 2)
                ok = mbar_wait_bounded(&bars[B_TPFREE + p], ((c >> 1) - 1) & 1, kWaitCycles);
            if (!ok) *s_err = 1;
            named_bar_sync(2, kPrep);
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

            // ---- L2-normalise K and Q rows in place, two threads per row -----------
            {
                const int r = pt >> 1;
                uint8_t* base = KQ + (uint32_t)(pt & 1) * 16384u;
                uint4 w[8];
                float ss = 0.f;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    w[ch] = *reinterpret_cast<const uint4*>(base + sw128_off(r, ch));
                    const uint32_t* u = &w[ch].x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x2 =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
                        ss = fmaf(x2.x, x2.x, ss);
                        ss = fmaf(x2.y, x2.y, ss);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                const float inv = (r >= 64 ? scale : 1.f) / sqrtf(ss + kL2Eps);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t* u = &w[ch].x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x2 =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
                        u[e] = pack_bf16x2(x2.x * inv, x2.y * inv);
                    }
                    *reinterpret_cast<uint4*>(base + sw128_off(r, ch)) = w[ch];
                }
            }

            // ---- Dkq = KQ K^^T (overlapped with the rest of the gate arithmetic) ----
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, kPrep);
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
            named_bar_sync(2, kPrep);
            const float G_last = sG[kC - 1];  // = G_{L-1}: tokens past L add g = 0
            if (pt < kC) {
                const float eg = __expf(sG[pt]);
                const float bt = sBeta[pt];
                gs[GS_EG + pt] = eg;
                gs[GS_EGL + pt] = __expf(G_last - sG[pt]);
                *reinterpret_cast<float2*>(gs + GS_BBE + 2 * pt) = make_float2(bt, bt * eg);
            }
            {
                const int ab4 = pt >> 6, jj = pt & 63;
                sU[pt] = (jj < 16 * ab4) ? __expf(sG[16 * ab4] - sG[jj]) : 0.f;
            }
            if (pt == 0) gs[GS_GAMMA] = __expf(G_last);
            ok = mbar_wait_bounded(&bars[B_MMAP], mphase, kWaitCycles);
            mphase ^= 1u;
            if (!ok) *s_err = 1;
            named_bar_sync(2, kPrep);
            if (*s_err) break;
            tc_fence_after();

            // ---- A rows 0-63 (fp32, As) and P rows 64-127 (bf16), half a row each --
            {
                float x[32];
                tmem_ld32_sync(ptl + TM_DKQ + 32 * hh, x);
                uint8_t* Pt = sm + SM_P + p * TP_BYTES;
                if (hh == 0) ap_half_row<0>(x, trow, L, sG, sBeta, sU, As, Pt);
                else         ap_half_row<1>(x, trow, L, sG, sBeta, sU, As, Pt);
            }
            named_bar_sync(2, kPrep);

            // ---- 8x8 diagonal blocks of T: forward substitution in registers -------
            // rows 0-31 from prep warp 0 (columns 0-31), rows 32-63 from prep warp 5
            if (pw == 0 || pw == 5) {
                const int i = trow;
                const int r = i & 7;
                const int b0 = i & ~7;
                const int src0 = lane & ~7;
                float Ad[8];
#pragma unroll
                for (int r2 = 0; r2 < 8; ++r2) Ad[r2] = (r2 < r) ? As[i * kAsStride + b0 + r2] : 0.f;
                float R[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) R[jj] = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float am = Ad[m];
#pragma unroll
                    for (int jj = 0; jj < m; ++jj) {
                        const float tv = -__shfl_sync(0xffffffffu, R[jj], src0 | m);
                        if (r > m) R[jj] = fmaf(am, tv, R[jj]);
                    }
                    if (r > m) R[m] += am;
                }
                float* Trow = Ts + i * kTsStride + b0;
#pragma unroll
                for (int r2 = 0; r2 < 8; ++r2) Trow[r2] = r2 < r ? -R[r2] : (r2 == r ? 1.f : 0.f);
            }
            named_bar_sync(2, kPrep);

            // ---- doubling 8 -> 16: T_{hi,lo} = -D_hi (A_{hi,lo} D_lo) in each 16-block
            {
                const int a0 = (pt >> 6) * 16;
                const int r = (pt >> 3) & 7, cc = pt & 7;
                const float* Arow = As + (a0 + 8 + r) * kAsStride + a0;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) acc = fmaf(Arow[m], Ts[(a0 + m) * kTsStride + a0 + cc], acc);
                Xs[pt] = acc;
                named_bar_sync(2, kPrep);
                const float* Drow = Ts + (a0 + 8 + r) * kTsStride + a0 + 8;
                const float* Xb = Xs + (pt & ~63);
                float t1 = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) t1 = fmaf(Drow[m], Xb[m * 8 + cc], t1);
                Ts[(a0 + 8 + r) * kTsStride + a0 + cc] = -t1;
            }
            named_bar_sync(2, kPrep);
            // ---- doubling 16 -> 32: T_10 and T_32 ------------------------------------
            {
                const int which = pt >> 7;
                const int q7 = pt & 127;
                const int r = q7 >> 3, c0 = (q7 & 7) * 2;
                const int cb = which ? 32 : 0;
                const int rb = which ? 48 : 16;
                const float* Arow = As + (rb + r) * kAsStride + cb;
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float am = Arow[m];
                    const float2 d = *reinterpret_cast<const float2*>(Ts + (cb + m) * kTsStride + cb + c0);
                    acc.x = fmaf(am, d.x, acc.x);
                    acc.y = fmaf(am, d.y, acc.y);
                }
                *reinterpret_cast<float2*>(Xs + which * 256 + r * 16 + c0) = acc;
                named_bar_sync(2, kPrep);
                const float* Drow = Ts + (rb + r) * kTsStride + rb;
                float2 t2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float dm = Drow[m];
                    const float2 xv = *reinterpret_cast<const float2*>(Xs + which * 256 + m * 16 + c0);
                    t2.x = fmaf(dm, xv.x, t2.x);
                    t2.y = fmaf(dm, xv.y, t2.y);
                }
                *reinterpret_cast<float2*>(Ts + (rb + r) * kTsStride + cb + c0) =
                    make_float2(-t2.x, -t2.y);
            }
            named_bar_sync(2, kPrep);
            // ---- doubling 32 -> 64: T[32:64, 0:32] -----------------------------------
            {
                const int r = pt >> 3, c0 = (pt & 7) * 4;
                const float* Arow = As + (32 + r) * kAsStride;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f), acc2 = acc;
#pragma unroll
                for (int m = 0; m < 32; m += 2) {
                    const float4 am = *reinterpret_cast<const float4*>(Arow + (m & ~3));
                    const float a_0 = (m & 2) ? am.z : am.x, a_1 = (m & 2) ? am.w : am.y;
                    const float4 d = *reinterpret_cast<const float4*>(Ts + m * kTsStride + c0);
                    const float4 e = *reinterpret_cast<const float4*>(Ts + (m + 1) * kTsStride + c0);
                    acc.x = fmaf(a_0, d.x, acc.x); acc.y = fmaf(a_0, d.y, acc.y);
                    acc.z = fmaf(a_0, d.z, acc.z); acc.w = fmaf(a_0, d.w, acc.w);
                    acc2.x = fmaf(a_1, e.x, acc2.x); acc2.y = fmaf(a_1, e.y, acc2.y);
                    acc2.z = fmaf(a_1, e.z, acc2.z); acc2.w = fmaf(a_1, e.w, acc2.w);
                }
                *reinterpret_cast<float4*>(Xs + r * 32 + c0) =
                    make_float4(acc.x + acc2.x, acc.y + acc2.y, acc.z + acc2.z, acc.w + acc2.w);
                named_bar_sync(2, kPrep);
                const float* Drow = Ts + (32 + r) * kTsStride + 32;
                float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f), t5 = t4;
#pragma unroll
                for (int m = 0; m < 32; m += 2) {
                    const float4 dm = *reinterpret_cast<const float4*>(Drow + (m & ~3));
                    const float d_0 = (m & 2) ? dm.z : dm.x, d_1 = (m & 2) ? dm.w : dm.y;
                    const float4 xv = *reinterpret_cast<const float4*>(Xs + m * 32 + c0);
                    const float4 xw = *reinterpret_cast<const float4*>(Xs + (m + 1) * 32 + c0);
                    t4.x = fmaf(d_0, xv.x, t4.x); t4.y = fmaf(d_0, xv.y, t4.y);
                    t4.z = fmaf(d_0, xv.z, t4.z); t4.w = fmaf(d_0, xv.w, t4.w);
                    t5.x = fmaf(d_1, xw.x, t5.x); t5.y = fmaf(d_1, xw.y, t5.y);
                    t5.z = fmaf(d_1, xw.z, t5.z); t5.w = fmaf(d_1, xw.w, t5.w);
                }
                *reinterpret_cast<float4*>(Ts + (32 + r) * kTsStride + c0) =
                    make_float4(-(t4.x + t5.x), -(t4.y + t5.y), -(t4.z + t5.z), -(t4.w + t5.w));
            }
            named_bar_sync(2, kPrep);

            // ---- T -> bf16 tile; hand the chunk to the chain ------------------------
            uint8_t* Tt = sm + SM_T + p * TP_BYTES;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int idx = pt + kPrep * it;  // 0..511
                const int row = idx >> 3, ch = idx & 7;
                const float4 f0 = *reinterpret_cast<const float4*>(Ts + row * kTsStride + ch * 8);
                const float4 f1 = *reinterpret_cast<const float4*>(Ts + row * kTsStride + ch * 8 + 4);
                uint4 w;
                w.x = pack_bf16x2(f0.x, f0.y);
                w.y = pack_bf16x2(f0.z, f0.w);
                w.z = pack_bf16x2(f1.x, f1.y);
                w.w = pack_bf16x2(f1.z, f1.w);
                *reinterpret_cast<uint4*>(Tt + sw128_off(row, ch)) = w;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, kPrep);
            if (pt == 0) mbar_arrive(&bars[B_READY + p]);
        }
    } else {
        // ============================== chain ========================================
        const uint32_t ctl = tmem + ((uint32_t)(warp * 32) << 16);
        const size_t sbase = ((size_t)n * H_v + h) * kD * kD + (size_t)tid * kD;
        uint8_t* Vt = sm + SM_V;

        // K/Q rows and gates of chunk cc into ring slot cc % kRing (128 arrivals on
        // its mbarrier once this thread's copies land); V rows of chunk cc + 2 are
        // warmed in L2 at the same time.
        auto load_kq = [&](int cc) {
            const int st = cc % kRing;
            const int64_t t0 = s0 + (int64_t)cc * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
            uint8_t* KQ = sm + SM_KQ + st * KQ_BYTES;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int idx = tid + 128 * it;  // 0 .. 1023
                const int r = idx >> 4, ch = idx & 15;
                const bool live = r < L;
                const int64_t tok = live ? t0 + r : 0;
                const size_t rowk = ((size_t)tok * H_qk + j) * kD + ch * 8;
                const uint32_t off = (uint32_t)(ch >> 3) * 16384u;
                cp_async_16(KQ + off + sw128_off(r, ch & 7), k + rowk, live ? 16u : 0u);
                cp_async_16(KQ + off + sw128_off(r + 64, ch & 7), q + rowk, live ? 16u : 0u);
            }
            float* abp = reinterpret_cast<float*>(sm + SM_AB) + st * 128;
            {
                const int t = tid & 63;
                const bool live = t < L;
                const int64_t tok = live ? t0 + t : 0;
                const float* src = (tid < 64 ? a : b) + (size_t)tok * H_v + h;
                cp_async_4(abp + (tid < 64 ? 0 : 64) + t, src, live ? 4u : 0u);
            }
            cp_async_mbar_arrive_noinc(&bars[B_LOADED + st]);
            const int64_t tv = t0 + 2 * kC + (tid >> 1);
            if (tv < s1) {
                const bf16* vp = v + ((size_t)tv * H_v + h) * kD + (tid & 1) * 64;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(vp));
            }
        };
        // V rows of chunk cc into the V tile: [t][i] as two 64-column blocks with the
        // 128-byte swizzle (the MMA reads it as the MN-major A operand V^T); rows
        // past the end of the sequence are zero-filled.
        auto load_v = [&](int cc) {
            const int64_t t0 = s0 + (int64_t)cc * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int idx = tid + 128 * it;  // 0 .. 1023
                const int r = idx >> 4, ch = idx & 15;
                const bool live = r < L;
                const int64_t tok = live ? t0 + r : 0;
                cp_async_16(Vt + (uint32_t)(ch >> 3) * 8192u + sw128_off(r, ch & 7),
                            v + ((size_t)tok * H_v + h) * kD + ch * 8, live ? 16u : 0u);
            }
        };

        // the 64x64 bf16 identity (B operand of the MMA that transposes V into TMEM)
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = tid + 128 * it;  // 0..511
            const int row = idx >> 3, ch = idx & 7;
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if ((row >> 3) == ch) {
                const uint32_t one = 0x3F80u << (16 * (row & 1));
                uint32_t* wp = &w.x;
                wp[(row & 7) >> 1] = one;
            }
            *reinterpret_cast<uint4*>(sm + SM_ID + sw128_off(row, ch)) = w;
        }
        fence_proxy_async_smem();

        // copy groups, in order: [K/Q of chunks 0..2], [V 0], [empty]; then per
        // chunk c: [V c+1], [K/Q c+3] -- so "all but the newest group" is always
        // the V tile the next chunk needs.
        for (int cc = 0; cc < kRing && cc < nchunks; ++cc) load_kq(cc);
        cp_async_commit();
        if (nchunks > 0) load_v(0);
        cp_async_commit();
        cp_async_commit();

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
            for (int cb = 0; cb < 4; cb += 2) {
                float x[32], y[32];
                tmem_ld32x2_sync(ctl + TM_S + 32 * cb, ctl + TM_S + 32 * cb + 32, x, y);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
                tmem_st16(ctl + TM_S0B + 16 * cb, pk);
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
                tmem_st16(ctl + TM_S0B + 16 * cb + 16, pk);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    x[e] *= gamma;
                    y[e] *= gamma;
                }
                tmem_st32(ctl + TM_S + 32 * cb, x);
                tmem_st32(ctl + TM_S + 32 * cb + 32, y);
            }
            tmem_wait_st();
            cp_async_wait<1>();          // this chunk's V tile (all but the newest group)
            fence_proxy_async_smem();    // ... visible to the tensor core
            tc_fence_before();
            named_bar_sync(1, 128);
            tc_fence_after();
            if (tid == 0) {
                constexpr uint32_t id_d1 = idesc_bf16_f32(128, 128, 0, 0);
                constexpr uint32_t id_v = idesc_bf16_f32(128, 64, 1, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                    mma_bf16_ts(tmem + TM_D1, tmem + TM_S0B + 8 * ks,
                                smem_desc_sw128(kq + off, 16, 1024), id_d1, ks > 0);
                }
                const uint32_t vt = smem_u32(Vt), idt = smem_u32(sm + SM_ID);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tmem + TM_DV, smem_desc_sw128(vt + ks * 2048, 8192, 1024),
                                smem_desc_sw128(idt + ks * 32, 16, 1024), id_v, ks > 0);
                mma_commit(&bars[B_MMAC]);
            }
            if (!chain_mma_wait()) break;
            if (c + 1 < nchunks) load_v(c + 1);  // V tile consumed: fetch the next one
            cp_async_commit();

            // ---- Y^T = beta (V - e^G X)^T, row i = tid, as bf16 pairs into TMEM ---------
            {
                const float4* bbe = reinterpret_cast<const float4*>(gs + GS_BBE);
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32], vv[32];
                    tmem_ld32x2_sync(ctl + TM_D1 + 32 * hf, ctl + TM_DV + 32 * hf, x, vv);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float4 f = bbe[16 * hf + e];  // beta, beta e^G of two tokens
                        pk[e] = pack_bf16x2(fmaf(f.x, vv[2 * e], -f.y * x[2 * e]),
                                            fmaf(f.z, vv[2 * e + 1], -f.w * x[2 * e + 1]));
                    }
                    tmem_st16(ctl + TM_D1 + 16 * hf, pk);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(1, 128);
            tc_fence_after();
            if (tid == 0) {
                constexpr uint32_t id = idesc_bf16_f32(128, 64, 0, 0);
                const uint32_t tt = smem_u32(sm + SM_T + p * TP_BYTES);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TM_D34, tmem + TM_D1 + 8 * ks,
                                smem_desc_sw128(tt + ks * 32, 16, 1024), id, ks > 0);
                mma_commit(&bars[B_MMAC]);
            }
            if (!chain_mma_wait()) break;

            // ---- Vn^T -> bf16 pairs in TMEM, and the decay-scaled copy ---------------
            {
                const float4* egl4 = reinterpret_cast<const float4*>(gs + GS_EGL);
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32];
                    tmem_ld32_sync(ctl + TM_D34 + 32 * hf, x);
                    uint32_t pk[16], ps[16];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 w = egl4[8 * hf + e4];
                        pk[2 * e4] = pack_bf16x2(x[4 * e4], x[4 * e4 + 1]);
                        pk[2 * e4 + 1] = pack_bf16x2(x[4 * e4 + 2], x[4 * e4 + 3]);
                        ps[2 * e4] = pack_bf16x2(x[4 * e4] * w.x, x[4 * e4 + 1] * w.y);
                        ps[2 * e4 + 1] = pack_bf16x2(x[4 * e4 + 2] * w.z, x[4 * e4 + 3] * w.w);
                    }
                    tmem_st16(ctl + TM_DV + 16 * hf, pk);
                    tmem_st16(ctl + TM_DV + 32 + 16 * hf, ps);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(1, 128);
            tc_fence_after();
            if (tid == 0) {
                constexpr uint32_t id_o = idesc_bf16_f32(128, 64, 0, 0);
                constexpr uint32_t id_s = idesc_bf16_f32(128, 128, 0, 1);
                const uint32_t ptile = smem_u32(sm + SM_P + p * TP_BYTES);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TM_D34, tmem + TM_DV + 8 * ks,
                                smem_desc_sw128(ptile + ks * 32, 16, 1024), id_o, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TM_S, tmem + TM_DV + 32 + 8 * ks,
                                smem_desc_sw128(kq + ks * 2048, 16384, 1024), id_s, 1);
                mma_commit(&bars[B_MMAC]);
            }
            if (!chain_mma_wait()) break;
            // the MMAs reading T and P are complete: release them
            if (tid == 0) mbar_arrive(&bars[B_TPFREE + p]);

            // ---- O = e^G (Q S0^T) + P Vn: staged as [t][i] rows, then 16-byte stores ----
            uint16_t* Ost = reinterpret_cast<uint16_t*>(sm + SM_VNT);
            const float4* eg4 = reinterpret_cast<const float4*>(gs + GS_EG);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float xq[32], xi[32];
                tmem_ld32x2_sync(ctl + TM_D1 + 64 + 32 * half, ctl + TM_D34 + 32 * half, xq, xi);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 w = eg4[8 * half + e4];
                    const int e = 4 * e4;
                    uint16_t* dst = Ost + (32 * half + e) * kD + tid;
                    const __nv_bfloat162 o01 = __floats2bfloat162_rn(fmaf(w.x, xq[e], xi[e]),
                                                                     fmaf(w.y, xq[e + 1], xi[e + 1]));
                    const __nv_bfloat162 o23 = __floats2bfloat162_rn(fmaf(w.z, xq[e + 2], xi[e + 2]),
                                                                     fmaf(w.w, xq[e + 3], xi[e + 3]));
                    dst[0] = __bfloat16_as_ushort(o01.x);
                    dst[kD] = __bfloat16_as_ushort(o01.y);
                    dst[2 * kD] = __bfloat16_as_ushort(o23.x);
                    dst[3 * kD] = __bfloat16_as_ushort(o23.y);
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
            // this chunk's K/Q slot is free (its last reader, the state MMA, is done):
            // fetch chunk c + kRing into it
            if (c + kRing < nchunks) load_kq(c + kRing);
            cp_async_commit();
        }
        cp_async_wait<0>();
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
