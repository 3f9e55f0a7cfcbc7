// Chunked prefill on the 5th-generation tensor cores (tcgen05, bf16 in, fp32
// accumulate), d_k = d_v = 128, bf16 q/k/v/o.
//
// The chunkwise form of the gated delta rule ("Qwen3.5-MoE-35B-A3B architecture
// teardown", 3.7 steps 3-6), in the value-major orientation (S is d_v x d_k,
// o = S q). Per 64-token chunk with in-chunk cumulative log-decay G, write
// strengths beta, inverse row norms rk (keys) and rq (queries, times the scale):
//
//   Dkq  = [K; Q] K^T (raw bf16 rows)  -> K K^T and Q K^T                 MMA
//   A    = strictly-lower(beta_i rk_i exp(G_i - G_j) rk_j (K K^T)_ij)
//   T    = (I + A)^-1                                                     fp32
//   P    = lower(rq_t exp(G_t - G_s) rk_s (Q K^T)_ts)                       bf16
//   D1   = S0 [K; Q]^T                                                     MMA
//   Y^T  = (V - diag(e^G rk) (S0 K^T)^T)^T diag(beta)                      bf16
//   Vn^T = Y^T T^T                                                         MMA
//   O^T  = (S0 Q^T) diag(e^G rq) + Vn^T P^T                                MMA
//   S   <- e^{G_L} S + (Vn^T diag(e^{G_L - G} rk)) K                       MMA
//
// The L2 norms are folded into per-token factors, so every MMA reads the bf16
// inputs as given. Only differences G_i - G_j with i >= j are exponentiated
// (directly, or as a product of two factors that are both <= 1), so nothing
// overflows however strong the decay.
//
// Two stages:
//   prep           everything that does not depend on the state, for all chunks:
//                  workers walk (chunk, QK head) units; each loads its K and Q rows
//                  by TMA and forms [K; Q] [K; Q]^T once (one MMA into TMEM: K K^T and
//                  Q K^T, and on the diagonal the squared row norms), then for each V
//                  head sharing that QK head the gates, A, P and T = (I + A)^-1 in fp32
//                  (8x8 diagonal blocks by
//                  forward substitution in registers, then doubling steps 8 -> 16 ->
//                  32 -> 64 with T_10 = -D_1 A_10 D_0, the last two on tf32 tensor
//                  cores). T diag(beta), P and the per-token factors go to the
//                  workspace as a record per (chunk, V head): the two lower-triangular
//                  matrices as the 16-row bands the chain's MMAs read (see the record
//                  layout below), copied into the chain's shared memory as they are.
//                  Each worker finds the next unit's sequence and prefetches its rows
//                  and gate inputs one unit ahead.
//   chain          one (sequence, V head) walks its chunks in order. The fp32 state
//                  lives in the registers of eight state warps; every A operand they
//                  produce (the bf16 state, Z^T, Vn^T and its decay-scaled copy) goes to
//                  TMEM, one warp issues the MMAs, four warps turn the output
//                  accumulators into o (TMA stores) and refill a 3-deep ring of K, Q,
//                  V tiles (TMA) and records (bulk copies).
// Launches: with few chains (at most half as many as SMs) both stages run in one
// cooperative launch (fused_kernel), chain blocks consuming records as prep blocks
// publish them (per-record flags holding the call's number); with at most a quarter
// as many chains as SMs each chain is split over two blocks of 64 value rows (M = 64
// MMAs). Otherwise three launches: chunk offsets (and the chains' order, longest
// sequences first), prep_kernel, chain_kernel.
//
// Every wait is bounded; on expiry a block records GDN_ERR_TIMEOUT in the status
// word, leaves its loops, drains its copies, frees its tensor memory and exits.
#include <cuda.h>

#include <unistd.h>

#include <atomic>
#include <chrono>
#include <random>

#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {

namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kD = 128;
constexpr int kC = kChunk;  // 64
constexpr int kMaxGroup = 16;                    // V heads per QK head handled by prep

// ---- workspace record of one (chunk, V head), written by prep, bulk-copied by chain
// T diag(beta) and P are lower triangular, and each enters the chain as the B operand
// (K-major, N = K = 64) of four K steps of 16. Step s needs only the rows 16 s .. 63 of
// its 16 columns (the rows above are zero), so a matrix is kept as four bands, band s =
// those rows and columns, in the plain (unswizzled) K-major core-matrix layout: 16-byte
// chunk (row i, columns 8 c .. 8 c + 7), s = c / 2, at chunk index
//   kBandStart[s] + ((i - 16 s) / 8) * 16 + (c % 2) * 8 + i % 8
// (8-row groups 256 bytes apart, the two core matrices of a step 128 bytes apart):
// 320 chunks (5,120 bytes) instead of the 512 of the full tile.
constexpr int kTriChunks = 320;
__host__ __device__ constexpr int band_start(int s) { return 16 * s * (9 - s); }  // 0 128 224 288
__device__ __forceinline__ int tri_chunk(int i, int c) {
    const int s = c >> 1;
    return band_start(s) + ((i - 16 * s) >> 3) * 16 + (c & 1) * 8 + (i & 7);
}
constexpr uint32_t REC_T = 0;        // T diag(beta), bf16, banded
constexpr uint32_t REC_P = 5120;     // P, bf16, banded
constexpr uint32_t REC_G = 10240;    // factors (floats):
constexpr int RG_FK = 0;             //   [64] e^{G_t} rk_t
constexpr int RG_EGQ = 128;          //   [64] e^{G_t} rq_t
constexpr int RG_EGL = 192;          //   [64] e^{G_L - G_t} rk_t
constexpr int RG_GAMMA = 256;        //   e^{G_L}
constexpr uint32_t kRecBytes = 11520;  // 45 x 256
static_assert(band_start(4) == kTriChunks && 16 * kTriChunks == REC_P, "band layout");

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ bool bad_seq(int64_t s0, int64_t s1, int64_t T_total, int n) {
    return s0 < 0 || s1 < s0 || s1 > T_total || (n == 0 && s0 != 0);
}

// =============================== chunk offsets ===================================
// choff[n] = number of 64-token chunks in sequences 0 .. n-1 (choff[N] = total), and
// order[]: the sequences by chunk count, most first (ties by index), for the chain
// blocks of the separate-launch path to take the longest sequences first (a list
// schedule); with more than kOrderMax sequences, or bad lengths, the identity.
constexpr int kOrderMax = 1024;
__global__ void __launch_bounds__(256) chunk_offsets_kernel(const int32_t* __restrict__ cu,
                                                            int32_t N, int64_t T_total,
                                                            int32_t* __restrict__ choff,
                                                            int32_t* __restrict__ order,
                                                            int* status) {
    __shared__ int32_t s_nc[kOrderMax];
    __shared__ int32_t warp_tot[8];
    __shared__ int32_t carry;
    __shared__ int bad;
    if (threadIdx.x == 0) { carry = 0; bad = 0; }
    __syncthreads();
    for (int base = 0; base < N; base += 256) {
        const int n = base + threadIdx.x;
        int32_t nc = 0;
        if (n < N) {
            const int64_t s0 = cu[n], s1 = cu[n + 1];
            if (bad_seq(s0, s1, T_total, n)) bad = 1;
            else nc = (int32_t)((s1 - s0 + kC - 1) / kC);
        }
        // block-wide inclusive scan of nc
        int32_t x = nc;
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        int32_t pre = carry;
        for (int ww = 0; ww < w; ++ww) pre += warp_tot[ww];
        if (n < N) choff[n] = pre + x - nc;
        __syncthreads();
        if (threadIdx.x == 255) carry = pre + x;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        choff[N] = bad ? 0 : carry;
        if (bad) {
            set_status(status, kStatusBadSeqlens);
            for (int n = 0; n < N; ++n) choff[n] = 0;
        }
    }
    // rank of sequence n = how many sequences come before it in the order
    const bool sort = !bad && N <= kOrderMax;
    if (sort)
        for (int n = threadIdx.x; n < N; n += 256) s_nc[n] = (int32_t)((cu[n + 1] - cu[n] + kC - 1) / kC);
    __syncthreads();
    for (int n = threadIdx.x; n < N; n += 256) {
        int rank = n;
        if (sort) {
            const int32_t c = s_nc[n];
            rank = 0;
            for (int m = 0; m < N; ++m) {
                const int32_t cm = s_nc[m];
                rank += (cm > c || (cm == c && m < n)) ? 1 : 0;
            }
        }
        order[rank] = n;
    }
}

// ---- warp-level tf32 MMA (m16n8k8, fp32 accumulate) for the small products of
// the triangular solve. Fragment layouts (lane = 4 g + t): A rows g and g + 8,
// columns t and t + 4; B rows t and t + 4, column g; C rows g and g + 8, columns
// 2 t and 2 t + 1.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Four 8 x 8 matrices of 16-bit elements from shared memory, lane l giving the address of
// row l % 8 of matrix l / 8 (16-byte aligned); register i of lane l receives elements
// 2 (l % 4) and 2 (l % 4) + 1 of row l / 4 of matrix i, i.e. with 32-bit elements
// (rows of four) element l % 4 of row l / 4.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p))
                 : "memory");
}

// d (16 x 8 tile at rows r0, columns c0 of the product) += M1[r0.., k0..k0+kn) M2[k0.., c0..)
// with M1, M2 row-major fp32 in shared memory (row strides s1, s2), kn a multiple of 8.
// M1's rows and k0 are 16-byte aligned: its four 8 x 4 pieces of a step are one ldmatrix
// (rows r0 + l % 8 and r0 + 8 + l % 8, columns k and k + 4).
__device__ __forceinline__ void tile_mma_tf32(float (&d)[4], const float* M1, int s1,
                                              const float* M2, int s2, int r0, int c0, int k0,
                                              int kn, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const float* arow = M1 + (r0 + (lane & 7) + ((lane >> 3) & 1) * 8) * s1 + ((lane >> 4) << 2);
    for (int k = k0; k < k0 + kn; k += 8) {
        uint32_t ar[4];
        ldsm_x4(ar, arow + k);
        const uint32_t a[4] = {to_tf32(__uint_as_float(ar[0])), to_tf32(__uint_as_float(ar[1])),
                               to_tf32(__uint_as_float(ar[2])), to_tf32(__uint_as_float(ar[3]))};
        const uint32_t b[2] = {to_tf32(M2[(k + t) * s2 + c0 + g]),
                               to_tf32(M2[(k + t + 4) * s2 + c0 + g])};
        mma_tf32_16x8x8(d, a, b);
    }
}

// Store a 16 x 8 C fragment (times `scale`) at rows r0, columns c0 of a row-major matrix.
__device__ __forceinline__ void tile_store(float* M, int s, int r0, int c0, const float (&d)[4],
                                           float scale, int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(M + (r0 + g) * s + c0 + 2 * t) = make_float2(scale * d[0], scale * d[1]);
    *reinterpret_cast<float2*>(M + (r0 + g + 8) * s + c0 + 2 * t) =
        make_float2(scale * d[2], scale * d[3]);
}

// ==================================== prep ========================================
constexpr int kPrepThreads = 256;
constexpr int kTsStride = 68;  // rows of T and A: conflict-free as the A operand of the merges
constexpr int kAsStride = 68;
constexpr int kXsStride = 40;  // merge scratch: conflict-free as the B operand of the merges
constexpr int kEStride = 20;   // rows of the in-block exponential table (16 used): the 8 lanes
                               // of a 16-byte shared-memory access phase hit distinct banks
// Shared memory map (bytes from a 1024-byte aligned base). The first 32 KB hold the raw
// K and Q rows until the unit's MMA has read them; after that, A, the staging image of
// P and the exponential tables of the V head being worked on.
constexpr uint32_t PS_KQ = 0;      // [2 col blocks][128 rows][128 B], raw K then Q, sw128
constexpr uint32_t PS_AS = 0;      // [64][68] fp32 A (strictly-lower part used)
constexpr uint32_t PS_PST = 17408; // P, bf16, banded (the record's P; 5,120 of 8,192 B)
constexpr uint32_t PS_E = 25600;   // [4][16][20] exp(G_i - G_j) inside 16-blocks
constexpr uint32_t PS_U = 30720;   // [4][64] exp(G_{16 a} - G_j)
constexpr uint32_t PS_CI = 31744;  // [64] exp(G_i - G_{16-block start of i})
constexpr uint32_t PS_TS = 32768;  // [64][68] fp32 T (entries above its diagonal blocks stay 0)
constexpr uint32_t PS_XS = 50176;  // [32][40] fp32 merge scratch
constexpr uint32_t PS_GA = 55296;  // [kMaxGroup][64] G of every V head of the unit
constexpr uint32_t PS_BA = 59392;  // [kMaxGroup][64] beta of every V head of the unit
constexpr uint32_t PS_RK = 63488;  // [64] rk, [64] rq (rq includes the scale)
constexpr uint32_t PS_BAR = 64000; // mbarrier (MMA)
constexpr uint32_t PS_TMEM = 64008;
constexpr uint32_t PS_LDBAR = 64016; // mbarrier (TMA loads of the K and Q rows)
constexpr uint32_t PS_NEXT = 64032;  // [2][16 B] a coming unit's first token (int64),
                                     // sequence and length (int32 each)
constexpr uint32_t PS_AB = 64512;    // [2][kMaxGroup][64] fp32 a, b of the unit (copied in
                                     // during the unit before)
constexpr size_t kPrepSmem = PS_AB + 2 * kMaxGroup * 64 * 4 + 1024;
static_assert(PS_CI + 64 * 4 <= PS_TS, "the per-head area must fit where K and Q were");

// Half a row (32 columns from 32 H) of A (row i < 64, to the A matrix) or of P (row
// t = i - 64, to the banded staging image) from the matching half row x of [K; Q] K^T, whose
// columns are already scaled by rk. Columns left of the row's 16-block use
// exp(G_i - G_j) = exp(G_i - G_a0) U_j (both factors <= 1); the at most 16 columns
// inside the block take their own exponential; columns right of the row are zero.
// rowf = beta_i rk_i (A) or rq_t (P).
template <int H>
__device__ __forceinline__ void ap_half_row(const float (&x)[32], int row, const float* U,
                                            const float* E, const float* CI, float rowf,
                                            float* As, uint8_t* Pst, bool live) {
    const int i = row & 63;
    const int a0 = i & ~15;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int c0 = 32 * H + 16 * g;
        const float4* t4;
        float f;
        if (c0 < a0) {
            t4 = reinterpret_cast<const float4*>(U + (a0 >> 4) * 64 + c0);
            f = rowf * CI[i];
        } else {
            t4 = reinterpret_cast<const float4*>(E + (a0 >> 4) * (16 * kEStride) +
                                                 (i - a0) * kEStride);
            f = c0 == a0 ? rowf : 0.f;
        }
        float v[16];
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
            const float4 u = t4[e4];
            const int e = 16 * g + 4 * e4;
            v[4 * e4] = f * u.x * x[e];
            v[4 * e4 + 1] = f * u.y * x[e + 1];
            v[4 * e4 + 2] = f * u.z * x[e + 2];
            v[4 * e4 + 3] = f * u.w * x[e + 3];
        }
        if (row < 64) {
            float4* Arow = reinterpret_cast<float4*>(As + i * kAsStride + c0);
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4)
                Arow[e4] = make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
        } else if (c0 <= a0) {  // (16-column groups right of the row's block: not kept)
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                uint4 w;
                w.x = live ? pack_bf16x2(v[8 * q2 + 0], v[8 * q2 + 1]) : 0u;
                w.y = live ? pack_bf16x2(v[8 * q2 + 2], v[8 * q2 + 3]) : 0u;
                w.z = live ? pack_bf16x2(v[8 * q2 + 4], v[8 * q2 + 5]) : 0u;
                w.w = live ? pack_bf16x2(v[8 * q2 + 6], v[8 * q2 + 7]) : 0u;
                reinterpret_cast<uint4*>(Pst)[tri_chunk(i, 4 * H + 2 * g + q2)] = w;
            }
        }
    }
}

// The exponential tables of one V head's G (the thread's share of them):
//   U[a][j] = exp(G_{16 a} - G_j) for j < 16 a (both factors of a long gap are <= 1),
//   E[b][ii][jj] = exp(G_{16 b + ii} - G_{16 b + jj}) for jj <= ii, else 0,
//   CI[i] = exp(G_i - G_{16-block start of i}).
__device__ __forceinline__ void exp_tables(const float* hG, float* sU, float* sE, float* sCI,
                                           int tid) {
    const int ab4 = tid >> 6, jj = tid & 63;
    sU[tid] = (jj < 16 * ab4) ? __expf(hG[16 * ab4] - hG[jj]) : 0.f;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        // a warp writes rows ii and ii + 4 of a block (20 ii and 20 ii + 80 differ by 16
        // banks: no conflict); over the 16 row selectors rs every row ii once
        const int idx = tid + kPrepThreads * q4;  // 0..1023
        const int rs = (idx >> 4) & 15;
        const int bb = idx >> 8, ii = ((rs & 1) << 2) | ((rs >> 1) & 3) | (rs & 8), jb = idx & 15;
        sE[bb * (16 * kEStride) + ii * kEStride + jb] =
            jb <= ii ? __expf(hG[16 * bb + ii] - hG[16 * bb + jb]) : 0.f;
    }
    if (tid < kC) sCI[tid] = __expf(hG[tid] - hG[tid & ~15]);
}

__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// SiLU with one special-function operation: x sigmoid(x), sigmoid(x) = (1 + tanh(x/2)) / 2,
// tanh from the hardware's approximation (relative error about 2^-11, below half a bf16 ulp).
__device__ __forceinline__ float silu_tanh(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return x * fmaf(0.5f, t, 0.5f);
}

// The causal depthwise convolution + SiLU of one unit's channels ("Qwen3.5-MoE-35B-A3B
// architecture teardown", 3.3 phase 2: conv over the concatenated q/k/v channels, kernel
// K, then SiLU): the q and k channels of QK head j and the v channels of its r V heads,
// for the chunk's tokens t0 .. t0+L-1 of sequence n (which starts at s0). Positions
// before the sequence's start come from the conv cache (zeros without one). q and k go
// to the K/Q tile in shared memory (rows past L zero), and every channel to the post-conv
// buffer that the chain's tile loads read. The arithmetic (bias, then the taps oldest
// first with fused multiply-adds, then SiLU, one rounding to bf16) is that of the
// standalone convolution kernel, so both give the same bits. A thread takes 4 channels x
// 8 tokens at a time; consecutive threads take consecutive channel groups.
__device__ __forceinline__ void conv_unit(const MixerFusion& mix, int n, int64_t s0, int64_t t0,
                                          int L, int j, int r, int H_qk, uint8_t* KQ, int tid,
                                          int64_t T_total, int N, int* status) {
    const int C = mix.conv_dim, K = mix.K;
    const int nv4 = 64 + 32 * r;  // 4-channel groups: q 32, k 32, v 32 per V head
    const int items = nv4 * 8;    // x 8 segments of 8 tokens
    // item -> (first channel, first token) and its input window: positions
    // p = t0 + tt0 - (K-1) + s, s = 0 .. 6 + K, 4 bf16 (8 bytes) each
    auto locate = [&](int item, int& c, int& v4, int& tt0) {
        const int seg = item / nv4;
        v4 = item - seg * nv4;
        tt0 = seg * 8;
        if (v4 < 32) c = j * kD + 4 * v4;
        else if (v4 < 64) c = H_qk * kD + j * kD + 4 * (v4 - 32);
        else c = 2 * H_qk * kD + (j * r + ((v4 - 64) >> 5)) * kD + 4 * ((v4 - 64) & 31);
    };
    auto load = [&](int c, int tt0, uint2 (&raw)[11]) {
#pragma unroll
        for (int s_ = 0; s_ < 11; ++s_) {
            raw[s_] = make_uint2(0u, 0u);
            const int64_t p = t0 + tt0 - (K - 1) + s_;
            if (s_ < 7 + K && p < t0 + L) {
                if (p >= s0) {
                    if (GDN_IN_BOUNDS(p * C + c + 3, T_total * C, status))
                        raw[s_] = *reinterpret_cast<const uint2*>(mix.x + (size_t)p * C + c);
                } else if (mix.cache_in) {
                    const int64_t ci = ((int64_t)n * (K - 1) + (K - 1) + (p - s0)) * C + c;
                    if (GDN_IN_BOUNDS(ci + 3, (int64_t)N * (K - 1) * C, status))
                        raw[s_] = *reinterpret_cast<const uint2*>(mix.cache_in + ci);
                }
            }
        }
    };
    auto compute = [&](int c, int v4, int tt0, const uint2 (&raw)[11]) {
        float w[4][4], bs[4];  // w[e][i]: tap i (oldest first) of channel c + e
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            bs[e] = mix.conv_b ? mix.conv_b[c + e] : 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) w[e][i] = i < K ? mix.conv_w[(size_t)(c + e) * K + i] : 0.f;
        }
        const int cc = (v4 & 31) * 4;  // channel within the head (q, k)
        uint8_t* kq = KQ + (uint32_t)(cc >> 6) * 16384u + (uint32_t)((cc >> 2) & 1) * 8u;
        const int row0 = v4 < 32 ? 64 : 0;  // Q rows 64-127, K rows 0-63
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float acc[4] = {bs[0], bs[1], bs[2], bs[3]};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i < K) {
                    const uint2 rw = raw[u + i];
                    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw.x));
                    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw.y));
                    acc[0] = fmaf(w[0][i], lo.x, acc[0]);
                    acc[1] = fmaf(w[1][i], lo.y, acc[1]);
                    acc[2] = fmaf(w[2][i], hi.x, acc[2]);
                    acc[3] = fmaf(w[3][i], hi.y, acc[3]);
                }
            }
            const int tt = tt0 + u;
            const bool live = tt < L;
            uint2 out = make_uint2(0u, 0u);
            if (live)
                out = make_uint2(pack_bf16x2(silu_fast(acc[0]), silu_fast(acc[1])),
                                 pack_bf16x2(silu_fast(acc[2]), silu_fast(acc[3])));
            if (v4 < 64)
                *reinterpret_cast<uint2*>(kq + sw128_off((uint32_t)(row0 + tt), (uint32_t)((cc & 63) >> 3))) = out;
            if (live && GDN_IN_BOUNDS((t0 + tt) * C + c + 3, T_total * C, status))
                *reinterpret_cast<uint2*>(mix.qkvc + (size_t)(t0 + tt) * C + c) = out;
        }
    };
    // two items in flight: both windows are loaded before either is computed
#pragma unroll 1
    for (int item = tid; item < items; item += 2 * kPrepThreads) {
        int ca, va, ta, cb = 0, vb = 0, tb = 0;
        uint2 rawa[11], rawb[11];
        const bool two = item + kPrepThreads < items;
        locate(item, ca, va, ta);
        load(ca, ta, rawa);
        if (two) {
            locate(item + kPrepThreads, cb, vb, tb);
            load(cb, tb, rawb);
        }
        compute(ca, va, ta, rawa);
        if (two) compute(cb, vb, tb, rawb);
    }
}

// Record (chunk cg, V head h) is complete: publish it to the chain (release). A flag
// holds the number of the call that wrote it last; call numbers only grow within a
// process, so flags left by earlier calls never read as ready and need no reset.
__device__ __forceinline__ void publish_record(unsigned long long* flags, size_t idx,
                                               unsigned long long epoch) {
    __threadfence();
    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(flags + idx), "l"(epoch) : "memory");
}

// One prep worker of kPrepThreads threads (tid 0 .. 255, synchronised by the named
// barrier bar_id) walks the (chunk, QK head) units worker, worker + nworkers, ...
// and writes their records; with `flags`, each finished record is published.
template <bool kConv>
__device__ __forceinline__ void prep_worker(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const float* __restrict__ a,
    const float* __restrict__ b, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, const int32_t* __restrict__ cu_seqlens,
    const int32_t* __restrict__ choff, int32_t N, int H_qk, int H_v, float scale,
    uint8_t* __restrict__ rec, int* status,
    unsigned long long* flags, unsigned long long epoch, uint8_t* sm, const int tid,
    const int bar_id, const int worker, const int nworkers, const bool relinquish,
    const long long wait_cycles, const MixerFusion& mix, const int64_t qk_tok,
    const int64_t T_total, const CUtensorMap* tm_q, const CUtensorMap* tm_k) {
    uint8_t* KQ = sm + PS_KQ;
    float* Ts = reinterpret_cast<float*>(sm + PS_TS);
    float* As = reinterpret_cast<float*>(sm + PS_AS);
    float* Xs = reinterpret_cast<float*>(sm + PS_XS);
    float* sU = reinterpret_cast<float*>(sm + PS_U);   // per-head exp tables (see exp_tables)
    uint8_t* Pst = sm + PS_PST;                        // P staging image
    float* rk = reinterpret_cast<float*>(sm + PS_RK);
    float* sGall = reinterpret_cast<float*>(sm + PS_GA);
    float* sBall = reinterpret_cast<float*>(sm + PS_BA);
    float* sE = reinterpret_cast<float*>(sm + PS_E);
    float* sCI = reinterpret_cast<float*>(sm + PS_CI);
    float* rq = rk + 64;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + PS_BAR);
    uint64_t* ldbar = reinterpret_cast<uint64_t*>(sm + PS_LDBAR);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + PS_TMEM);
    int64_t* s_next = reinterpret_cast<int64_t*>(sm + PS_NEXT);
    float* AB = reinterpret_cast<float*>(sm + PS_AB);

    const int warp = tid >> 5, lane = tid & 31;
    const int r = H_v / H_qk;
    const int total_units = choff[N] * H_qk;
    // extents of the debug build's index checks: records, and q / k rows from the pointer
    // (the last token's row of the last QK head ends there)
    const int64_t total_records = (int64_t)choff[N] * H_v;
    const int64_t qk_extent = T_total > 0 ? (T_total - 1) * qk_tok + (int64_t)H_qk * kD : 0;

    constexpr uint32_t tcols = 128u;  // [K; Q] [K; Q]^T
    if (warp == 0) {
        tmem_alloc(s_tmem, tcols);
        if (relinquish) tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(ldbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // entries of T above its diagonal blocks are never written: zero them once
    for (int idx = tid; idx < 64 * kTsStride; idx += kPrepThreads) Ts[idx] = 0.f;
    tc_fence_before();
    named_bar_sync(bar_id, kPrepThreads);
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int trow = (warp & 3) * 32 + lane;  // TMEM lane = row of [K; Q] K^T
    const int hh = warp >> 2;                 // which 32 columns of that row
    uint32_t mphase = 0, lphase = 0;
    bool failed = false;
    bool ld_pending = false;  // (thread 0) a TMA load of K and Q rows not yet waited for
    uint32_t ld_phase = 0;    // (thread 0) the phase that load completes
    // A unit's sequence n (choff[n] <= chunk < choff[n + 1]), first token t0 and length L.
    // A worker's units only move forward, so each unit's are found by a short forward
    // scan from the previous one's (the first by bisection), one unit ahead: thread 0
    // looks up the next unit while the current unit's K and Q rows are in flight and
    // leaves the result in slot par ^ 1 of s_next, read after the barriers that follow
    // (by the L2 prefetch of the next unit's rows, and at the end of the iteration).
    auto locate = [&](int cgx, int& nx, int64_t& t0x, int& Lx) {
        while (GDN_IN_BOUNDS(nx + 1, N + 1, status) && choff[nx + 1] <= cgx) ++nx;
        t0x = (int64_t)cu_seqlens[nx] + (int64_t)(cgx - choff[nx]) * kC;
        Lx = (int)min((int64_t)kC, (int64_t)cu_seqlens[nx + 1] - t0x);
    };
    // a and b of a unit's V heads (tokens past its length read as zeros) into AB, element
    // i0, i0 + step, ... by this thread, as one cp.async group of it
    auto fetch_ab = [&](int64_t t0x, int Lx, int jx, int i0, int step) {
        for (int idx = i0; idx < 2 * r * kC; idx += step) {
            const int which = idx / (r * kC);            // 0: a, 1: b
            const int rem = idx - which * r * kC;
            const int hr = rem >> 6, t = rem & 63;
            const int64_t tok = t < Lx ? t0x + t : 0;
            const bool live = t < Lx && GDN_IN_BOUNDS(tok * H_v + jx * r + hr, T_total * H_v, status);
            const float* src = (which ? b : a) + (size_t)tok * H_v + jx * r + hr;
            cp_async_4(AB + (which * kMaxGroup + hr) * kC + t, src, live ? 4u : 0u);
        }
        cp_async_commit();
    };
    int n = 0, L = 0, par = 0;
    int64_t t0 = 0;
    if (worker < total_units) {
        const int cg = worker / H_qk;
        int hi = N;
        while (hi - n > 1) {
            const int mid = (n + hi) >> 1;
            if (choff[mid] <= cg) n = mid; else hi = mid;
        }
        locate(cg, n, t0, L);
        fetch_ab(t0, L, worker % H_qk, tid, kPrepThreads);
    }

#pragma unroll 1
    for (int unit = worker; unit < total_units; unit += nworkers) {
        const int cg = unit / H_qk;
        const int j = unit - cg * H_qk;

        // ---- raw K and Q rows (sw128: four TMA boxes of 64 rows x 128 bytes, the chain's
        // tile layout), or the convolution that makes them; gates of the r V heads
        if constexpr (kConv) {
            conv_unit(mix, n, cu_seqlens[n], t0, L, j, r, H_qk, KQ, tid, T_total, N, status);
        } else if (tid == 0) {
            mbar_arrive_expect_tx(ldbar, 4u * 8192u);
            tma_load_3d(KQ, tm_k, 0, j, (int32_t)t0, ldbar);
            tma_load_3d(KQ + 16384, tm_k, 64, j, (int32_t)t0, ldbar);
            tma_load_3d(KQ + 8192, tm_q, 0, j, (int32_t)t0, ldbar);
            tma_load_3d(KQ + 16384 + 8192, tm_q, 64, j, (int32_t)t0, ldbar);
            ld_pending = true;
            ld_phase = lphase;
        }
        const int un = unit + nworkers;
        if (!kConv && L < kC) {
            // the rows past the sequence's end hold the next tokens (or zeros past T): zero
            // them, 16 bytes a thread at a time (whole 128-byte rows, so no swizzle matters)
            if (!mbar_wait_bounded(ldbar, lphase, wait_cycles)) failed = true;
            else if (tid == 0) ld_pending = false;
            const int nz = (kC - L) * 8;  // 16-byte pieces per 64-row tile
            for (int idx = tid; idx < 4 * nz; idx += kPrepThreads) {
                const int tile = idx / nz, rr = L + (idx % nz) / 8, ch = idx & 7;
                *reinterpret_cast<uint4*>(KQ + (tile >> 1) * 16384 + (tile & 1) * 8192 + rr * 128 +
                                          ch * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        cp_async_wait<0>();  // this unit's a and b (copied in during the unit before)
        fence_proxy_async_smem();
        named_bar_sync(bar_id, kPrepThreads);

        // ---- Dkq = [K; Q] [K; Q]^T: columns 0-63 ([K; Q] K^T) feed A and P, the diagonal
        // gives the row norms
        if (tid == 0) {
            bool ok = true;
            if (!kConv && L == kC) {
                ok = mbar_wait_bounded(ldbar, lphase, wait_cycles);
                if (ok) ld_pending = false;
            }
            if (!ok) failed = true;
            const uint32_t kq = smem_u32(KQ);
            constexpr uint32_t id_kq = idesc_bf16_f32(128, 128, 0, 0);
            if (ok) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
                    mma_bf16_ss(tmem, smem_desc_sw128(kq + off, 16, 1024),
                                smem_desc_sw128(kq + off, 16, 1024), id_kq, ks > 0);
                }
            }
            mma_commit(bar);  // (after a failed load: arrives at once, the error follows)
        }
        if (!kConv) lphase ^= 1u;
        // ---- gates of every V head of the group: one warp per head, two tokens a lane:
        // g, beta and the in-chunk inclusive cumsum G (the record's per-token factors
        // follow once the row norms are known)
        // (warps 1.., while thread 0 waits for the rows and issues the MMA)
        for (int hr = warp - 1; hr >= 0 && hr < r; hr += kPrepThreads / 32 - 1) {
            const int hv = j * r + hr;
            const bool hok = GDN_IN_BOUNDS(hv, H_v, status);
            const float A_l = hok ? A_log[hv] : 0.f, dtb = hok ? dt_bias[hv] : 0.f;
            const int ta = 2 * lane, tb = 2 * lane + 1;
            const bool la = ta < L, lb = tb < L;
            const float2 av = *reinterpret_cast<const float2*>(AB + hr * kC + ta);
            const float2 bv = *reinterpret_cast<const float2*>(AB + (kMaxGroup + hr) * kC + ta);
            const float ga = la ? gate_g(av.x, A_l, dtb) : 0.f;
            const float gb = lb ? gate_g(av.y, A_l, dtb) : 0.f;
            const float ba = la ? gate_beta(bv.x) : 0.f;
            const float bb = lb ? gate_beta(bv.y) : 0.f;
            float sc = ga + gb;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, sc, off);
                if (lane >= off) sc += y;
            }
            *reinterpret_cast<float2*>(sGall + hr * kC + ta) = make_float2(sc - gb, sc);
            *reinterpret_cast<float2*>(sBall + hr * kC + ta) = make_float2(ba, bb);
        }
        // ---- the next unit, by the last warp meanwhile: its sequence, first token and
        // length (into slot par ^ 1 of s_next, read after the barriers that follow) and
        // its K and Q rows fetched into L2 (the four boxes its loads will read)
        if (warp == kPrepThreads / 32 - 1 && un < total_units) {
            int nn = n, Ln = 0;
            int64_t t0n = 0;
            if (lane == 0) {
                locate(un / H_qk, nn, t0n, Ln);
                s_next[2 * (par ^ 1)] = t0n;
                reinterpret_cast<int*>(s_next + 2 * (par ^ 1) + 1)[0] = nn;
                reinterpret_cast<int*>(s_next + 2 * (par ^ 1) + 1)[1] = Ln;
            }
            // (with the convolution fused in, the rows are made from x: nothing to fetch)
            if (!kConv && lane == 0 && Ln > 0) {
                const int jn = un % H_qk;
                tma_prefetch_l2_3d(tm_k, 0, jn, (int32_t)t0n);
                tma_prefetch_l2_3d(tm_k, 64, jn, (int32_t)t0n);
                tma_prefetch_l2_3d(tm_q, 0, jn, (int32_t)t0n);
                tma_prefetch_l2_3d(tm_q, 64, jn, (int32_t)t0n);
            }
        }
        const bool ok = mbar_wait_bounded(bar, mphase, wait_cycles);
        mphase ^= 1u;
        if (!ok) failed = true;
        if (named_bar_any(bar_id, kPrepThreads, failed)) { failed = true; break; }
        tc_fence_after();
        // the gates have read this unit's a and b: the next unit's come in meanwhile, asked
        // for by the warps of the second column half (the first load the row norms)
        if (un < total_units && hh == 1)
            fetch_ab(s_next[2 * (par ^ 1)],
                     reinterpret_cast<const int*>(s_next + 2 * (par ^ 1) + 1)[1], un % H_qk,
                     tid - kPrepThreads / 2, kPrepThreads / 2);
        // ---- inverse row norms from the diagonal (K K^T)_ii, (Q Q^T)_tt: the warps of the
        // first column half load the 32 columns of their own 32 rows and keep their lane's
        {
            if (hh == 0) {
                float xd[32];
                tmem_ld32_sync(tl + 32 * (warp & 3), xd);
                float d = xd[0];
#pragma unroll
                for (int e = 1; e < 32; ++e) d = lane == e ? xd[e] : d;
                const float inv = 1.f / sqrtf(d + kL2Eps);
                if (trow < 64) rk[trow] = inv;
                else rq[trow - 64] = inv * scale;
            }
        }
        named_bar_sync(bar_id, kPrepThreads);  // rk, rq
        // the record's per-token factors of every V head of the group
        for (int hr = warp; hr < r; hr += kPrepThreads / 32) {
            const int h = j * r + hr;
            const int ta = 2 * lane;
            const float2 G2 = *reinterpret_cast<const float2*>(sGall + hr * kC + ta);
            const float G_last = sGall[hr * kC + kC - 1];  // G_{L-1} (g = 0 past L)
            float* rg = reinterpret_cast<float*>(rec + ((size_t)cg * H_v + h) * kRecBytes + REC_G);
            if (!GDN_IN_BOUNDS((int64_t)cg * H_v + h, total_records, status)) continue;
            const float ea = __expf(G2.x), eb = __expf(G2.y);
            const float2 rk2 = *reinterpret_cast<const float2*>(rk + ta);
            const float2 rq2 = *reinterpret_cast<const float2*>(rq + ta);
            *reinterpret_cast<float2*>(rg + RG_FK + ta) = make_float2(ea * rk2.x, eb * rk2.y);
            *reinterpret_cast<float2*>(rg + RG_EGQ + ta) = make_float2(ea * rq2.x, eb * rq2.y);
            *reinterpret_cast<float2*>(rg + RG_EGL + ta) =
                make_float2(__expf(G_last - G2.x) * rk2.x, __expf(G_last - G2.y) * rk2.y);
            if (lane == 0) rg[RG_GAMMA] = __expf(G_last);
        }
        // this thread's half row of [K; Q] K^T, shared by the r V heads, columns scaled
        // by rk once for all of them
        float x[32];
        tmem_ld32_sync(tl + 32 * hh, x);
        {
            const float4* rk4 = reinterpret_cast<const float4*>(rk + 32 * hh);
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
                const float4 r4 = rk4[e4];
                x[4 * e4] *= r4.x;
                x[4 * e4 + 1] *= r4.y;
                x[4 * e4 + 2] *= r4.z;
                x[4 * e4 + 3] *= r4.w;
            }
        }
        // The K and Q rows have been read (MMA): their area now takes A, the P
        // staging image and the tables. The first head's tables get a phase of their own;
        // every later head's are built while the head before writes its record.
        exp_tables(sGall, sU, sE, sCI, tid);
        named_bar_sync(bar_id, kPrepThreads);

#pragma unroll 1
        for (int hr = 0; hr < r; ++hr) {
            const int h = j * r + hr;
            uint8_t* R = rec + ((size_t)cg * H_v + h) * kRecBytes;
            const bool rec_ok = GDN_IN_BOUNDS((int64_t)cg * H_v + h, total_records, status);
            const float* hBeta = sBall + hr * kC;  // this head's beta

            // ---- A rows 0-63 -> As (fp32); P rows 64-127 -> staging (bf16 image);
            // then the 8x8 diagonal blocks of T by forward substitution in registers,
            // by the two warps that wrote the A rows those blocks read (rows 0-31,
            // columns 0-31: warp 0; rows 32-63, columns 32-63: warp 5), no barrier between
            {
                const int i = trow & 63;
                const float rowf = trow < 64 ? hBeta[i] * rk[i] : rq[i];
                if (hh == 0) ap_half_row<0>(x, trow, sU, sE, sCI, rowf, As, Pst, i < L);
                else         ap_half_row<1>(x, trow, sU, sE, sCI, rowf, As, Pst, i < L);
            }
            if (warp == 0 || warp == 5) {
                const int i = trow;
                const int rr = i & 7;
                const int b0 = i & ~7;
                const int src0 = lane & ~7;
                // the row's 8 entries of its diagonal block as two 16-byte loads (the rows of a
                // load's 8-thread phase are 68 words apart: distinct bank groups)
                const float4 q0 = *reinterpret_cast<const float4*>(As + i * kAsStride + b0);
                const float4 q1 = *reinterpret_cast<const float4*>(As + i * kAsStride + b0 + 4);
                float Ad[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                for (int r2 = 0; r2 < 8; ++r2) Ad[r2] = (r2 < rr) ? Ad[r2] : 0.f;
                float Rr[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) Rr[jj] = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float am = Ad[m];
#pragma unroll
                    for (int jj = 0; jj < m; ++jj) {
                        const float tv = -__shfl_sync(0xffffffffu, Rr[jj], src0 | m);
                        if (rr > m) Rr[jj] = fmaf(am, tv, Rr[jj]);
                    }
                    if (rr > m) Rr[m] += am;
                }
                float Tv[8];
#pragma unroll
                for (int r2 = 0; r2 < 8; ++r2) Tv[r2] = r2 < rr ? -Rr[r2] : (r2 == rr ? 1.f : 0.f);
                float4* Trow = reinterpret_cast<float4*>(Ts + i * kTsStride + b0);
                Trow[0] = make_float4(Tv[0], Tv[1], Tv[2], Tv[3]);
                Trow[1] = make_float4(Tv[4], Tv[5], Tv[6], Tv[7]);
            }
            named_bar_sync(bar_id, kPrepThreads);

            // ---- doubling 8 -> 16: T_{hi,lo} = -D_hi (A_{hi,lo} D_lo) in each 16-block
            {
                const int a0 = (tid >> 6) * 16;
                const int rr = (tid >> 3) & 7, cc = tid & 7;
                const float4* Arow = reinterpret_cast<const float4*>(As + (a0 + 8 + rr) * kAsStride + a0);
                const float4 Al = Arow[0], Ah = Arow[1];
                const float Av[8] = {Al.x, Al.y, Al.z, Al.w, Ah.x, Ah.y, Ah.z, Ah.w};
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) acc = fmaf(Av[m], Ts[(a0 + m) * kTsStride + a0 + cc], acc);
                Xs[tid] = acc;
                named_bar_sync(bar_id, kPrepThreads);
                const float4* Drow = reinterpret_cast<const float4*>(Ts + (a0 + 8 + rr) * kTsStride + a0 + 8);
                const float4 Dl = Drow[0], Dh = Drow[1];
                const float Dv[8] = {Dl.x, Dl.y, Dl.z, Dl.w, Dh.x, Dh.y, Dh.z, Dh.w};
                const float* Xb = Xs + (tid & ~63);
                float t1 = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) t1 = fmaf(Dv[m], Xb[m * 8 + cc], t1);
                Ts[(a0 + 8 + rr) * kTsStride + a0 + cc] = -t1;
            }
            named_bar_sync(bar_id, kPrepThreads);
            // ---- doubling 16 -> 32 (two 32-blocks) and 32 -> 64, tf32 tensor cores ----
            // T_10 = -T_11 (A_10 T_00): X = A_10 T_00 goes through Xs
            {
                // 16 -> 32: warp w < 4: block b = w >> 1 (rows 32 b + 16 ..), column tile w & 1
                if (warp < 4) {
                    const int b = warp >> 1, nt = warp & 1;
                    const int Rb = 32 * b;
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    tile_mma_tf32(d, As, kAsStride, Ts, kTsStride, Rb + 16, Rb + 8 * nt, Rb, 16, lane);
                    tile_store(Xs + b * 16 * kXsStride, kXsStride, 0, 8 * nt, d, 1.f, lane);
                }
                named_bar_sync(bar_id, kPrepThreads);
                if (warp < 4) {
                    const int b = warp >> 1, nt = warp & 1;
                    const int Rb = 32 * b;
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    // rows Rb+16.. of T (its 16-block, columns Rb+16..Rb+31) times X (16 x 16)
                    tile_mma_tf32(d, Ts + Rb + 16, kTsStride, Xs + b * 16 * kXsStride, kXsStride,
                                  Rb + 16, 8 * nt, 0, 16, lane);
                    tile_store(Ts, kTsStride, Rb + 16, Rb + 8 * nt, d, -1.f, lane);
                }
            }
            named_bar_sync(bar_id, kPrepThreads);
            {
                // 32 -> 64: X (32 x 32) = A[32:64, 0:32] T[0:32, 0:32]; warp w: tile (w >> 2, w & 3)
                const int mt = warp >> 2, nt = warp & 3;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_mma_tf32(d, As, kAsStride, Ts, kTsStride, 32 + 16 * mt, 8 * nt, 0, 32, lane);
                tile_store(Xs, kXsStride, 16 * mt, 8 * nt, d, 1.f, lane);
                named_bar_sync(bar_id, kPrepThreads);
                float e[4] = {0.f, 0.f, 0.f, 0.f};
                // T[32:64, 0:32] = -T[32:64, 32:64] X
                tile_mma_tf32(e, Ts + 32, kTsStride, Xs, kXsStride, 32 + 16 * mt, 8 * nt, 0, 32, lane);
                tile_store(Ts, kTsStride, 32 + 16 * mt, 8 * nt, e, -1.f, lane);
            }
            named_bar_sync(bar_id, kPrepThreads);

            // ---- T diag(beta) -> record, the staged P -> record, both banded, as
            // coalesced 16-byte stores; the next head's tables meanwhile ----------------
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                // chunk o of the banded image: rows i .. of one 8-row group, columns
                // 8 c .. 8 c + 7; the 8 threads of a load phase read one column run of 8
                // consecutive rows (68 words apart: distinct bank groups)
                const int o = tid + kPrepThreads * it;
                if (o < kTriChunks) {
                    const int sb = (o >= band_start(1)) + (o >= band_start(2)) + (o >= band_start(3));
                    const int rest = o - band_start(sb);
                    const int i = 16 * sb + (rest >> 4) * 8 + (rest & 7);
                    const int c = 2 * sb + ((rest >> 3) & 1);
                    const float* trow = Ts + i * kTsStride + 8 * c;
                    const float4 ta = *reinterpret_cast<const float4*>(trow);
                    const float4 tb = *reinterpret_cast<const float4*>(trow + 4);
                    const float4 ba = *reinterpret_cast<const float4*>(hBeta + 8 * c);
                    const float4 bb = *reinterpret_cast<const float4*>(hBeta + 8 * c + 4);
                    uint4 w;  // column s of T times beta_s
                    w.x = pack_bf16x2(ta.x * ba.x, ta.y * ba.y);
                    w.y = pack_bf16x2(ta.z * ba.z, ta.w * ba.w);
                    w.z = pack_bf16x2(tb.x * bb.x, tb.y * bb.y);
                    w.w = pack_bf16x2(tb.z * bb.z, tb.w * bb.w);
                    if (rec_ok) {
                        reinterpret_cast<uint4*>(R + REC_T)[o] = w;
                        reinterpret_cast<uint4*>(R + REC_P)[o] = reinterpret_cast<const uint4*>(Pst)[o];
                    }
                }
            }
            if (hr + 1 < r) exp_tables(sGall + (hr + 1) * kC, sU, sE, sCI, tid);
            named_bar_sync(bar_id, kPrepThreads);  // Ts, As, Xs, the staging and tables are reused
            if (flags && tid == 0 && rec_ok) publish_record(flags, (size_t)cg * H_v + h, epoch);
        }
        tc_fence_before();  // this unit's TMEM reads precede the next unit's MMA
        par ^= 1;
        t0 = s_next[2 * par];
        n = reinterpret_cast<const int*>(s_next + 2 * par + 1)[0];
        L = reinterpret_cast<const int*>(s_next + 2 * par + 1)[1];
    }
    // no copy into shared memory may still be in flight when the worker ends
    cp_async_wait<0>();
    if (tid == 0 && ld_pending && !mbar_wait_bounded(ldbar, ld_phase, wait_cycles)) failed = true;
    tc_fence_before();
    named_bar_sync(bar_id, kPrepThreads);
    tc_fence_after();
    if (failed && tid == 0) set_status(status, kStatusTimeout);
    if (warp == 0) tmem_dealloc(tmem, tcols);
}

constexpr int kPrepBlocksPerSm = 3;
template <bool kConv>
__global__ void __launch_bounds__(kPrepThreads, kPrepBlocksPerSm) prep_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const bf16* __restrict__ q, const bf16* __restrict__ k, const float* __restrict__ a,
    const float* __restrict__ b, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, const int32_t* __restrict__ cu_seqlens,
    const int32_t* __restrict__ choff, int32_t N, int H_qk, int H_v, float scale,
    uint8_t* __restrict__ rec, int* status, long long wait_cycles, const MixerFusion mix,
    int64_t qk_tok, int64_t T_total) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned (128-byte swizzle), as an offset from the shared array itself so
    // that every pointer derived from it stays a shared-memory address for the compiler
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    prep_worker<kConv>(q, k, a, b, A_log, dt_bias, cu_seqlens, choff, N, H_qk, H_v, scale, rec,
                       status, nullptr, 0, sm, threadIdx.x, 1, blockIdx.x, gridDim.x, true,
                       wait_cycles, mix, qk_tok, T_total, &tm_q, &tm_k);
}

// ==================================== chain =======================================
constexpr int kChainThreads = 416;  // warps 0-7 state, warp 8 MMA issue, warps 9-12 output + loads
constexpr int kChain = 256;
constexpr int kOut = 128;
constexpr int kIssueWarp = 8;
constexpr int kRdyBar = 6;     // named barrier: state threads arrive, the issuing warp waits
constexpr int kRdyCount = 288;
constexpr int kLoadWarp = 9;
constexpr int kRing = 3;
// shared memory map (bytes from a 1024-byte aligned base)
constexpr uint32_t SLOT_KQ = 0;        // [2 col blocks][K rows 0-63, Q rows 64-127][128 B], sw128
constexpr uint32_t SLOT_V = 32768;     // [2 col blocks][64 rows][128 B] V, sw128
constexpr uint32_t SLOT_REC = 49152;   // the (chunk, V head) record: T diag(beta), P, factors
constexpr uint32_t kSlotBytes = 61440;  // (the next slot's tiles 1024-byte aligned)
static_assert(SLOT_REC + kRecBytes <= kSlotBytes && kSlotBytes % 1024 == 0, "slot layout");
constexpr uint32_t kSlotTx = 6 * 8192 + kRecBytes;  // six 64x64 tiles + the record
constexpr uint32_t CS_OST = kRing * kSlotBytes;     // [2 col blocks][64 t][128 B] o, sw128
constexpr uint32_t CS_BAR = CS_OST + 16384;         // barriers (see below)
constexpr uint32_t CS_TMEM = CS_BAR + 128;
constexpr uint32_t CS_ERR = CS_BAR + 132;
constexpr uint32_t CS_EGQ = CS_BAR + 256;           // [64] fp32: the chunk's output row factors
constexpr uint32_t CS_NW = CS_EGQ + 256;            // [128] fp32: the gated norm's weights
constexpr size_t kChainSmem = CS_NW + 512 + 1024;

// tensor memory columns (512 allocated)
constexpr uint32_t TM_U = 0;      // 128: the chunk's state increment (scaled Vn^T) K, fp32
constexpr uint32_t TM_S0B = 128;  // 64: state as bf16 pairs
constexpr uint32_t TM_D1K = 192;  // 64: S0 K^T; Z^T pairs overwrite columns 0-15 and 32-47,
                                  //     then the decay-scaled Vn^T pairs columns 0-31
constexpr uint32_t TM_D1Q0 = 256; // 64: S0 Q^T of even chunks
constexpr uint32_t TM_D3 = 320;   // 64: Vn^T; Vn^T pairs overwrite columns 0-15 and 32-47
constexpr uint32_t TM_D1Q1 = 384; // 64: S0 Q^T of odd chunks
constexpr uint32_t TM_D4 = 448;   // 64: Vn^T P^T
constexpr uint32_t kTmemCols = 512;

// Column (in 32-bit words) of the K=16 slice ks of a 64-token bf16 operand that
// two warps wrote in place over the fp32 columns they had read: tokens 0-31 at
// +0..15, tokens 32-63 at +32..47.
__device__ __forceinline__ uint32_t split_pairs_col(int ks) {
    return (uint32_t)((ks >> 1) * 32 + (ks & 1) * 8);
}

// Byte offset of element (row t, column i) of a [2 col blocks][64 rows][128 B]
// bf16 tile in the 128-byte swizzle.
__device__ __forceinline__ uint32_t tile64_off(int t, int i) {
    return (uint32_t)(i >> 6) * 8192u + (uint32_t)t * 128u +
           ((uint32_t)(((i & 63) >> 3) ^ (t & 7)) << 4) + (uint32_t)(i & 7) * 2u;
}

// One block per (sequence, V head).
//   warps 0-7   the state, fp32 in registers: two warps share each TMEM lane
//               quarter, warp w owning value rows 32 (w & 3) .. + 31 and, of every
//               64- or 128-column quantity of those rows (the state included), the
//               half w >> 2. After each step's TMEM stores they arrive on a named
//               barrier that the issuing warp waits on, and go on.
//   warp 8      issues every MMA (elect.sync), each group once its inputs are
//               ready, and commits them to mbarriers; it does nothing else, so a
//               full tensor-core queue never holds up the state warps. Both sides
//               take exactly three barrier steps per chunk, errors included.
//   warps 9-12  (one per lane quarter) turn each chunk's output accumulators into o
//               (S0 Q^T alternates between two accumulators) and, once a chunk's
//               ring slot is no longer read, load the chunk three ahead into it
//               (TMA tiles for K, Q, V and one bulk copy of the record).
// Waits (bounded) until a prep worker publishes a record in this call (acquire).
__device__ __forceinline__ bool wait_record(const unsigned long long* flag,
                                            unsigned long long epoch, long long max_cycles) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(flag) : "memory");
    if (v == epoch) return true;
    const long long t0 = clock64();
    do {
        __nanosleep(64);
        asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(flag) : "memory");
        if (v == epoch) return true;
    } while (clock64() - t0 < max_cycles);
    return false;
}

// The conv cache of sequence n after it ("Qwen3.5-MoE-35B-A3B architecture teardown",
// 3.4: conv_dim x (K-1) per sequence): the K-1 inputs ending at its last token (older
// cache entries where the sequence is shorter), for the v channels of V head h and, with
// `qk`, the q and k channels of QK head j. One thread per 4-channel group walks the
// positions oldest first, so an update in place reads every old entry before it is
// overwritten.
__device__ __forceinline__ void write_conv_cache(const MixerFusion& mix, int n, int64_t s0,
                                                 int64_t s1, int h, int j, bool qk, int H_qk,
                                                 int to, int nthreads, int64_t T_total, int N,
                                                 int* status) {
    const int C = mix.conv_dim, Km1 = mix.K - 1;
    const int64_t len = s1 - s0;
    const int ng = qk ? 96 : 32;
    for (int g = to; g < ng; g += nthreads) {
        int c;
        if (g < 32) c = 2 * H_qk * kD + h * kD + 4 * g;
        else if (g < 64) c = j * kD + 4 * (g - 32);
        else c = H_qk * kD + j * kD + 4 * (g - 64);
        for (int i = 0; i < Km1; ++i) {
            const int64_t p = len - Km1 + i;
            uint2 v = make_uint2(0u, 0u);
            const int64_t cache_extent = (int64_t)N * Km1 * C;
            if (p >= 0) {
                if (GDN_IN_BOUNDS((s0 + p) * C + c + 3, T_total * C, status))
                    v = *reinterpret_cast<const uint2*>(mix.x + (size_t)(s0 + p) * C + c);
            } else if (mix.cache_in) {
                if (GDN_IN_BOUNDS(((int64_t)n * Km1 + len + i) * C + c + 3, cache_extent, status))
                    v = *reinterpret_cast<const uint2*>(mix.cache_in + ((size_t)n * Km1 + len + i) * C + c);
            }
            if (GDN_IN_BOUNDS(((int64_t)n * Km1 + i) * C + c + 3, cache_extent, status))
                *reinterpret_cast<uint2*>(mix.cache_out + ((size_t)n * Km1 + i) * C + c) = v;
        }
    }
}

// The whole chunk chain of one (sequence n, V head h), run by the kChainThreads
// threads of a block (tid 0 .. 415, synchronised by the named barrier sync_id) on
// the tensor memory `tmem` (512 columns). With `flags`, a chunk's record is
// copied only once a prep worker has published it.
template <int kM, bool kNorm>
__device__ __forceinline__ void chain_unit(
    const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
    const CUtensorMap& tm_o, const float* S0g, const int32_t* __restrict__ cu_seqlens,
    const int32_t* __restrict__ choff, int64_t T_total, int H_qk, int H_v,
    const uint8_t* __restrict__ rec, bf16* __restrict__ o,
    float* Sfg, const StateIndex sref, int* status,
    const unsigned long long* flags, unsigned long long epoch, uint8_t* sm, const int tid,
    const int n, const int h, const int hv, const uint32_t tmem,
    const int sync_id, const long long wait_cycles, const MixerFusion& mix, const int N,
    const bool inject_bad_index) {
    static_assert(kM == 128 || kM == 64, "a chain block owns all 128 value rows or one half");
    static_assert(!kNorm || kM == 128, "the fused gated norm needs whole value rows");
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + CS_BAR);  // [3] slot landed
    uint64_t* mbar = full + kRing;         // chain MMA completions
    uint64_t* obar = mbar + 1;             // [2] chunk parity b: output accumulators complete
    uint64_t* ofree = mbar + 3;            // [2] chunk parity b: output accumulators read
    uint64_t* dbar = mbar + 5;             // drain of in-flight MMAs before the exit
    volatile int* s_err = reinterpret_cast<volatile int*>(sm + CS_ERR);

    const int warp = tid >> 5, lane = tid & 31;
    const int j = h / (H_v / H_qk);
    if (!GDN_IN_BOUNDS(n, N, status)) return;
    const int64_t s0 = cu_seqlens[n];
    const int64_t s1 = cu_seqlens[n + 1];
    if (bad_seq(s0, s1, T_total, n)) return;  // reported by the offsets kernel
    const int nchunks = (int)((s1 - s0 + kC - 1) / kC);
    const int cg0 = choff[n];
    // records of the batch: the extent of the debug build's record index checks
    const int64_t total_records = kDebugBuild ? (int64_t)choff[N] * H_v : 0;

    if (tid == 0) {
        for (int i = 0; i < kRing; ++i) mbar_init(&full[i], 1);
        mbar_init(mbar, 1);
        mbar_init(&obar[0], 1);
        mbar_init(&obar[1], 1);
        mbar_init(&ofree[0], 4);
        mbar_init(&ofree[1], 4);
        mbar_init(dbar, 1);
        *s_err = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kLoadWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
    }
    tc_fence_before();
    named_bar_sync(sync_id, kChainThreads);
    tc_fence_after();

    // chunk c of this sequence -> its ring slot (issued by one lane). The K, Q, V tiles
    // need nothing from the prep workers and go first; the record follows once its
    // flag is seen (the slot's barrier expects both). With the convolution fused into
    // the preparation the tiles are its output too, so they wait for the flag as well.
    auto load_tiles = [&](int c) {
        const int st = c % kRing;
        uint8_t* slot = sm + st * kSlotBytes;
        const int32_t t0 = (int32_t)(s0 + (int64_t)c * kC);
        mbar_arrive_expect_tx(&full[st], kSlotTx);
        tma_load_3d(slot + SLOT_KQ, &tm_k, 0, j, t0, &full[st]);
        tma_load_3d(slot + SLOT_KQ + 16384, &tm_k, 64, j, t0, &full[st]);
        tma_load_3d(slot + SLOT_KQ + 8192, &tm_q, 0, j, t0, &full[st]);
        tma_load_3d(slot + SLOT_KQ + 16384 + 8192, &tm_q, 64, j, t0, &full[st]);
        tma_load_3d(slot + SLOT_V, &tm_v, 0, h, t0, &full[st]);
        tma_load_3d(slot + SLOT_V + 8192, &tm_v, 64, h, t0, &full[st]);
    };
    // After a wait that ran out the record is copied all the same (valid memory, the
    // results are discarded), so that the slot's barrier completes and no copy is left
    // in flight when the block exits.
    auto record_ready = [&](int c) -> bool {
        if (!GDN_IN_BOUNDS((int64_t)(cg0 + c) * H_v + h, total_records, status)) return true;
        if (flags && !wait_record(flags + (size_t)(cg0 + c) * H_v + h, epoch, wait_cycles)) {
            *s_err = 1;
            return false;
        }
        return true;
    };
    auto load_record = [&](int c) {
        const int st = c % kRing;
        if (flags) asm volatile("fence.proxy.async.global;" ::: "memory");  // read by TMA
        // (debug build: an index outside copies the first record of this head instead, so
        // that the slot's transaction count still completes)
        size_t ri = (size_t)(cg0 + c) * H_v + h;
        if (!GDN_IN_BOUNDS(ri, total_records, status)) ri = (size_t)h;
        bulk_g2s(sm + st * kSlotBytes + SLOT_REC, rec + ri * kRecBytes, kRecBytes, &full[st]);
    };

    if (warp > kIssueWarp) {
        // ============================ output + loads ===================================
        const int qo = warp & 3;
        const int row = qo * 32 + lane;
        const int to = tid - (kIssueWarp + 1) * 32;  // 0..127
        const uint32_t ctl = tmem + ((uint32_t)(qo * 32) << 16);
        uint8_t* ost = sm + CS_OST;
        const bool loader = warp == kLoadWarp && lane == 0;
        float* egq = reinterpret_cast<float*>(sm + CS_EGQ);
        float* s_nw = reinterpret_cast<float*>(sm + CS_NW);
        if (kNorm && to < kD / 4)  // read by the norm after the loop's first barrier
            reinterpret_cast<float4*>(s_nw)[to] = reinterpret_cast<const float4*>(mix.norm_w)[to];
        int issued = 0;   // chunks whose tiles and record were issued
        // a test of the index checks: one index just past the record array, nothing read
        if (inject_bad_index && loader) (void)GDN_IN_BOUNDS(total_records, total_records, status);
        if (loader) {
            if (mix.x) {
                for (int c = 0; c < kRing && c < nchunks; ++c) {
                    record_ready(c);
                    if (flags) asm volatile("fence.proxy.async.global;" ::: "memory");
                    load_tiles(c);
                    load_record(c);
                    issued = c + 1;
                }
            } else {
                for (int c = 0; c < kRing && c < nchunks; ++c) load_tiles(c);
                for (int c = 0; c < kRing && c < nchunks; ++c) {
                    record_ready(c);
                    load_record(c);
                    issued = c + 1;
                }
            }
        }
        __syncwarp();
        // Gate rows for the fused norm: chunk c's are loaded into registers at the end of
        // chunk c-1's iteration (the output warps reach a chunk when its MMAs are long
        // done, so a load issued at its start would be waited for in full), after being
        // prefetched into L2 two chunks ahead.
        uint4 zv[kNorm ? 8 : 1];
        auto load_gate_rows = [&](int c) {
            const int64_t tz = s0 + (int64_t)c * kC + (to >> 1);
            if (c < nchunks && tz < s1 && GDN_IN_BOUNDS(tz, T_total, status)) {
                const bf16* zr = mix.z + ((size_t)tz * H_v + h) * kD + (to & 1) * 64;
#pragma unroll
                for (int q = 0; q < 8; ++q) zv[q] = *reinterpret_cast<const uint4*>(zr + q * 8);
            }
        };
        if constexpr (kNorm) {
            for (int c2 = 1; c2 < 3 && c2 < nchunks; ++c2) {
                const int64_t t2 = s0 + (int64_t)c2 * kC + (to >> 1);
                if (t2 < s1) prefetch_l2(mix.z + ((size_t)t2 * H_v + h) * kD + (to & 1) * 64);
            }
            load_gate_rows(0);
        }
#pragma unroll 1
        for (int cp = 0; cp < nchunks; ++cp) {
            const int b = cp & 1;
            const int cn = cp + kRing;  // the chunk that will reuse this chunk's slot
            const int64_t t0 = s0 + (int64_t)cp * kC;
            const int L = (int)min((int64_t)kC, s1 - t0);
            if constexpr (kNorm) {
                const int64_t t3 = t0 + 3 * kC + (to >> 1);
                if (t3 < s1) prefetch_l2(mix.z + ((size_t)t3 * H_v + h) * kD + (to & 1) * 64);
            }
            // its record's flag is checked while this chunk's MMAs still run
            const bool next = loader && cn < nchunks && issued == cn;
            const bool ok = mbar_wait_bounded(&obar[b], (cp >> 1) & 1, wait_cycles);
            if (!ok) *s_err = 1;
            if (loader) bulk_wait_group_read<0>();  // staging free again
            // the slot's only remaining reader is this copy of the row factors
            if (ok && to < 16)
                reinterpret_cast<float4*>(egq)[to] = reinterpret_cast<const float4*>(
                    sm + (cp % kRing) * kSlotBytes + SLOT_REC + REC_G + 4 * RG_EGQ)[to];
            if (named_bar_any(2, kOut, !ok || *s_err != 0)) break;
            tc_fence_after();
            const float4* eg4 = reinterpret_cast<const float4*>(egq);
            const uint32_t qacc = ctl + (b ? TM_D1Q1 : TM_D1Q0);
            if constexpr (kM == 128) {
                // this thread's column of the staged tile; laundered so that the 64 element
                // addresses are formed per chunk rather than held in registers across chunks
                uint32_t ocol = smem_u32(ost) + (uint32_t)(row >> 6) * 8192u + (uint32_t)(row & 7) * 2u;
                uint32_t ochk = (uint32_t)((row & 63) >> 3);
                asm volatile("" : "+r"(ocol), "+r"(ochk));
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float xq[32], xi[32];
                    tmem_ld32x2_sync(qacc + 32 * hf, ctl + TM_D4 + 32 * hf, xq, xi);
                    if (hf == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ofree[b]);  // the accumulators may be overwritten
                    }
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 w = eg4[8 * hf + e4];
                        const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int t = 32 * hf + 4 * e4 + u, e = 4 * e4 + u;
                            const uint32_t a = ocol + (uint32_t)t * 128u + ((ochk ^ (uint32_t)(t & 7)) << 4);
                            const bf16 v = __float2bfloat16_rn(fmaf(wv[u], xq[e], xi[e]));
                            asm volatile("st.shared.b16 [%0], %1;" ::"r"(a),
                                         "h"(*reinterpret_cast<const unsigned short*>(&v))
                                         : "memory");
                        }
                    }
                }
            } else {
                // value rows r0 = 16 qo + lane / 4 and r0 + 8 of this block's half; tokens
                // 8 j + 2 (lane % 4) and + 1 (16-lane accumulator layout)
                float xq[32], xi[32];
                tmem_ld16r_x8x2_sync(qacc, ctl + TM_D4, xq, xi);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ofree[b]);  // the accumulators may be overwritten
                const int r0 = qo * 16 + (lane >> 2), tp = 2 * (lane & 3);
                uint32_t obase = smem_u32(ost);
                asm volatile("" : "+r"(obase));
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const float2 w = reinterpret_cast<const float2*>(egq)[4 * jj + (lane & 3)];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = 8 * jj + tp + (e & 1), r = r0 + 8 * (e >> 1);
                        const float wt = (e & 1) ? w.y : w.x;
                        const bf16 v = __float2bfloat16_rn(fmaf(wt, xq[4 * jj + e], xi[4 * jj + e]));
                        asm volatile("st.shared.b16 [%0], %1;" ::"r"(obase + tile64_off(t, r)),
                                     "h"(*reinterpret_cast<const unsigned short*>(&v))
                                     : "memory");
                    }
                }
            }
            // The slot is free: refill it with the chunk three ahead. Its record's flag is
            // checked only now, after the accumulators were read (an acquire load of the
            // flag is an L2 round trip; before the read it delayed every chunk's output).
            if (next) {
                record_ready(cn);
                if (mix.x && flags) asm volatile("fence.proxy.async.global;" ::: "memory");
                load_tiles(cn);
                load_record(cn);
                issued = cn + 1;
            }
            __syncwarp();
            fence_proxy_async_smem();
            named_bar_sync(2, kOut);  // staged; every output warp is done with the slot
            if constexpr (kNorm) {
                {
                    // The gated RMSNorm over each staged o row ("Qwen3.5-MoE-35B-A3B architecture
                    // teardown", 3.3 phase 4: RMSNorm(o) * w * SiLU(z)): two threads per token,
                    // 64 values each, the sum of squares of the bf16 o, then y over o in place.
                    const int t = to >> 1, half = to & 1;
                    uint8_t* rowp = ost + half * 8192 + t * 128;
                    float ss = 0.f;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((ch ^ (t & 7)) << 4));
                        const uint32_t* u = &w.x;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
                            ss = fmaf(f.x, f.x, ss);
                            ss = fmaf(f.y, f.y, ss);
                        }
                    }
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    const float inv = rsqrtf(ss * (1.f / kD) + mix.eps);
                    if (t < L) {
                        const float4* wr4 = reinterpret_cast<const float4*>(s_nw + half * 64);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint4* p = reinterpret_cast<uint4*>(rowp + ((ch ^ (t & 7)) << 4));
                            const uint4 ov = *p;
                            const float4 w0 = wr4[2 * ch], w1 = wr4[2 * ch + 1];
                            const float wv[8] = {w0.x * inv, w0.y * inv, w0.z * inv, w0.w * inv,
                                                 w1.x * inv, w1.y * inv, w1.z * inv, w1.w * inv};
                            const uint32_t* ou = &ov.x;
                            const uint32_t* zu = &zv[ch].x;
                            uint32_t res[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ou[e]));
                                const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zu[e]));
                                res[e] = pack_bf16x2(of.x * wv[2 * e] * silu_tanh(zf.x),
                                                     of.y * wv[2 * e + 1] * silu_tanh(zf.y));
                            }
                            *p = make_uint4(res[0], res[1], res[2], res[3]);
                        }
                    }
                    __syncwarp();
                    fence_proxy_async_smem();
                    named_bar_sync(2, kOut);
                    load_gate_rows(cp + 1);  // the next chunk's, a whole chunk ahead of use
                }
            }
            constexpr int kOutCh = kM / 8;  // 16-byte chunks per staged row
            if (L == kC) {
                if (loader) {
                    if constexpr (kM == 128) {
                        tma_store_3d(&tm_o, 0, h, (int32_t)t0, ost);
                        tma_store_3d(&tm_o, 64, h, (int32_t)t0, ost + 8192);
                    } else {
                        tma_store_3d(&tm_o, 64 * hv, h, (int32_t)t0, ost);
                    }
                    bulk_commit_group();
                }
            } else {
                // the sequence's last rows only: plain 16-byte stores
                for (int idx = to; idx < L * kOutCh; idx += kOut) {
                    const int r = idx / kOutCh, ch = idx % kOutCh;
                    const uint4 w = *reinterpret_cast<const uint4*>(ost + tile64_off(r, ch * 8));
                    if (GDN_IN_BOUNDS(t0 + r, T_total, status))
                        *reinterpret_cast<uint4*>(o + ((size_t)(t0 + r) * H_v + h) * kD +
                                                  (kM == 64 ? 64 * hv : 0) + ch * 8) = w;
                }
                named_bar_sync(2, kOut);
            }
            __syncwarp();
        }
        if (mix.cache_out && hv == 0 && *s_err == 0)
            write_conv_cache(mix, n, s0, s1, h, j, h % (H_v / H_qk) == 0, H_qk, to, kOut, T_total,
                             N, status);
        if (loader) {
            bulk_wait_group<0>();  // o stores complete
            // Leave nothing in flight into shared memory (loads the chain did not
            // consume are only possible after an error).
            for (int c = issued - 1; c >= 0 && c >= issued - kRing; --c)
                if (!mbar_wait_bounded(&full[c % kRing], (c / kRing) & 1, wait_cycles))
                    *s_err = 1;
        }
        __syncwarp();
    } else if (warp == kIssueWarp) {
        // ================================ MMA issue =====================================
        // Three waits per chunk on the state threads' barrier, always (after an error
        // the MMAs are skipped but the waits stay, so every arrival is consumed).
        auto wait_rdy = [&](int id = kRdyBar) {
            named_bar_sync(id, kRdyCount);
            tc_fence_after();
        };
        bool dead = false;
        constexpr uint32_t id64 = idesc_bf16_f32(kM, 64, 0, 0);
        constexpr uint32_t id_s = idesc_bf16_f32(kM, 128, 0, 1);
        // the K steps of a banded B (T diag(beta), P): N = 64 - 16 s
        constexpr uint32_t id_tri[4] = {id64, idesc_bf16_f32(kM, 48, 0, 0),
                                        idesc_bf16_f32(kM, 32, 0, 0), idesc_bf16_f32(kM, 16, 0, 0)};
        constexpr uint32_t id_tri_v[4] = {idesc_bf16_f32(kM, 64, 1, 0), idesc_bf16_f32(kM, 48, 1, 0),
                                          idesc_bf16_f32(kM, 32, 1, 0), idesc_bf16_f32(kM, 16, 1, 0)};
        // TMEM A operands (fixed for the whole unit)
        uint32_t aS0[4], aS1[4], aZ[4], aU[4], aN[4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            aS0[ks] = tmem + TM_S0B + 8 * ks;
            aS1[ks] = tmem + TM_S0B + 8 * (ks + 4);
            aZ[ks] = tmem + TM_D1K + split_pairs_col(ks);
            aU[ks] = tmem + TM_D1K + 8 * ks;
            aN[ks] = tmem + TM_D3 + split_pairs_col(ks);
        }
        auto check = [&](bool ok) {  // warp-uniform: stop issuing after any failure
            dead = __any_sync(0xffffffffu, dead || !ok || *s_err != 0);
            if (dead) *s_err = 1;
        };
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int st = c % kRing;
            uint8_t* slot = sm + st * kSlotBytes;
            const uint32_t kq = smem_u32(slot + SLOT_KQ);
            const uint32_t vt = smem_u32(slot + SLOT_V);
            const uint32_t tt = smem_u32(slot + SLOT_REC + REC_T);
            const uint32_t ptile = smem_u32(slot + SLOT_REC + REC_P);
            // shared-memory descriptors of this chunk's operands, formed while waiting
            uint64_t dK0[4], dK1[4], dQ0[4], dQ1[4], dV[4], dT[4], dKm[4], dP[4];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                dK0[ks] = smem_desc_sw128(kq + ks * 32u, 16, 1024);
                dK1[ks] = smem_desc_sw128(kq + 16384u + ks * 32u, 16, 1024);
                dQ0[ks] = smem_desc_sw128(kq + 8192u + ks * 32u, 16, 1024);
                dQ1[ks] = smem_desc_sw128(kq + 16384u + 8192u + ks * 32u, 16, 1024);
                // V^T rows = value rows: this block's half of them when kM = 64
                dV[ks] = smem_desc_sw128(vt + (kM == 64 ? 8192u * hv : 0u) + ks * 2048u, 8192, 1024);
                dT[ks] = smem_desc_kmajor_plain(tt + 16u * band_start(ks), 128, 256);
                dKm[ks] = smem_desc_sw128(kq + ks * 2048u, 16384, 1024);
                dP[ks] = smem_desc_kmajor_plain(ptile + 16u * band_start(ks), 128, 256);
            }
            if (!dead) check(mbar_wait_bounded(&full[st], (c / kRing) & 1, wait_cycles));
            // (1) the bf16 state is written: S0 K^T, then V^T (T diag(beta))^T
            wait_rdy();
            check(true);
            if (!dead) {
                mma_ts_group4(tmem + TM_D1K, aS0, dK0, id64, 0);
                mma_ts_group4(tmem + TM_D1K, aS1, dK1, id64, 1);
                mma_commit_warp(mbar);
                mma_ss_tri4(tmem + TM_D3, dV, dT, id_tri_v, 0);
            }
            // (2) Z^T is written: Vn^T += Z^T (T diag(beta))^T; then S0 Q^T into the
            // accumulator of parity c & 1, last read for chunk c - 2
            wait_rdy();
            check(true);
            if (!dead) {
                mma_ts_tri4(tmem + TM_D3, aZ, dT, id_tri, 1);
                mma_commit_warp(mbar);
                if (c >= 2)
                    check(mbar_wait_bounded(&ofree[c & 1], ((c - 2) >> 1) & 1, wait_cycles));
            }
            if (!dead) {
                const uint32_t qacc = tmem + ((c & 1) ? TM_D1Q1 : TM_D1Q0);
                mma_ts_group4(qacc, aS0, dQ0, id64, 0);
                mma_ts_group4(qacc, aS1, dQ1, id64, 1);
            }
            // (3) the Vn^T pairs are written: the state increment, then Vn^T P^T
            wait_rdy();
            check(true);
            if (!dead) {
                mma_ts_group4(tmem + TM_U, aU, dKm, id_s, 0);
                mma_commit_warp(mbar);
                if (c >= 1)
                    check(mbar_wait_bounded(&ofree[(c - 1) & 1], ((c - 1) >> 1) & 1,
                                            wait_cycles));
            }
            if (!dead) {
                mma_ts_tri4(tmem + TM_D4, aN, dP, id_tri, 0);
                mma_commit_warp(&obar[c & 1]);
            }
        }
        __syncwarp();
        // no MMA may still run when the tensor memory is freed
        mma_commit_warp(dbar);
        (void)mbar_wait_bounded(dbar, 0, wait_cycles);
        if (*s_err) {  // wake the output warps so they see the error and leave
            if (lane == 0) {
                mbar_arrive(&obar[0]);
                mbar_arrive(&obar[1]);
            }
        }
        __syncwarp();
    } else {
        if constexpr (kM == 128) {
            // ================================ state ========================================
            const int qd = warp & 3;              // TMEM lane quarter
            const int hh = warp >> 2;             // column half
            const int row = qd * 32 + lane;       // value row i = TMEM lane
            const uint32_t ctl = tmem + ((uint32_t)(qd * 32) << 16);
            bool rd, wr;  // the sequence's state (or pool slot): read at the start, written at the end
            const int sidx = sref.resolve(n, rd, wr, tid == 0 ? status : nullptr);
            if (!GDN_IN_BOUNDS(sidx, sref.slots ? sref.num_slots : N, status)) rd = wr = false;
            const float* S0s = rd ? S0g : nullptr;
            float* Sfs = wr ? Sfg : nullptr;
            const size_t sbase = ((size_t)sidx * H_v + h) * kD * kD + (size_t)row * kD + 64 * hh;
            float S[64];  // S[i][64 hh + e]
            if (S0s) {
                const float4* src = reinterpret_cast<const float4*>(S0s + sbase);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float4 f = src[e];
                    S[4 * e] = f.x; S[4 * e + 1] = f.y; S[4 * e + 2] = f.z; S[4 * e + 3] = f.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 64; ++e) S[e] = 0.f;
            }

            uint32_t mphase = 0;
            bool dead = false;  // warp-uniform: after an error only the barrier arrivals remain
            auto wait_mma = [&]() {
                if (dead) return;
                bool ok = *s_err == 0 && mbar_wait_bounded(mbar, mphase, wait_cycles);
                mphase ^= 1u;
                dead = __any_sync(0xffffffffu, !ok || *s_err != 0);
                if (dead) *s_err = 1;
                tc_fence_after();
            };
            // this warp's TMEM operands of the step are written (and, before that, any
            // shared-memory writes fenced): arrive for the issuing warp, always. After an
            // error the arrival waits for the barrier to complete, so that no thread can
            // run a barrier generation ahead of the issuing warp.
            auto signal_rdy = [&]() {
                if (!dead) tmem_wait_st();
                tc_fence_before();
                if (dead) named_bar_sync(kRdyBar, kRdyCount);
                else named_bar_arrive(kRdyBar, kRdyCount);
            };
            // S <- gamma S + U (the previous chunk's decay and increment)
            auto apply_update = [&](float gamma) {
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
                    float u[32];
                    tmem_ld32_sync(ctl + TM_U + 64 * hh + 32 * cb, u);
#pragma unroll
                    for (int e = 0; e < 32; ++e) S[32 * cb + e] = fmaf(gamma, S[32 * cb + e], u[e]);
                }
            };

            float gamma = 1.f;
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % kRing;
                uint8_t* slot = sm + st * kSlotBytes;
                const float* rg = reinterpret_cast<const float*>(slot + SLOT_REC + REC_G);
                const int64_t t0 = s0 + (int64_t)c * kC;
                const int L = (int)min((int64_t)kC, s1 - t0);

                // ---- the previous chunk's state update and this chunk's data -------------
                if (c > 0) {
                    wait_mma();
                    if (!dead) apply_update(gamma);
                }
                if (!dead) {
                    const bool okf =
                        *s_err == 0 && mbar_wait_bounded(&full[st], (c / kRing) & 1, wait_cycles);
                    dead = __any_sync(0xffffffffu, !okf || *s_err != 0);
                    if (dead) *s_err = 1;
                }
                if (!dead && L < kC) {
                    // rows past the sequence's end hold the next sequence's tokens (or TMA
                    // zero fill): zero them
                    const int nz = (kC - L) * 8;  // 16-byte chunks per 64-column tile
                    for (int idx = tid; idx < 6 * nz; idx += kChain) {
                        const int tile = idx / nz, r = L + (idx % nz) / 8, ch = idx & 7;
                        const uint32_t base = tile < 4 ? SLOT_KQ + (tile >> 1) * 16384u + (tile & 1) * 8192u
                                                       : SLOT_V + (tile - 4) * 8192u;
                        *reinterpret_cast<uint4*>(slot + base + r * 128 + ch * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }

                // ---- state: bf16 copy (A operand of S0 K^T and S0 Q^T) ----------------------
                if (!dead) {
#pragma unroll
                    for (int cb = 0; cb < 2; ++cb) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(S[32 * cb + 2 * e], S[32 * cb + 2 * e + 1]);
                        tmem_st16(ctl + TM_S0B + 32 * hh + 16 * cb, pk);
                    }
                }
                signal_rdy();
                if (!dead) gamma = rg[RG_GAMMA];

                // ---- Z^T = -(e^G rk) (S0 K^T) for this thread's 32 tokens, in place ----------
                wait_mma();  // S0 K^T
                if (!dead) {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {  // 16 tokens at a time
                        const float4* fk4 = reinterpret_cast<const float4*>(rg + RG_FK) + 8 * hh + 4 * q;
                        float x[16];
                        tmem_ld16_sync(ctl + TM_D1K + 32 * hh + 16 * q, x);
                        uint32_t pk[8];
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const float4 f = fk4[e4];
                            pk[2 * e4] = pack_bf16x2(-f.x * x[4 * e4], -f.y * x[4 * e4 + 1]);
                            pk[2 * e4 + 1] = pack_bf16x2(-f.z * x[4 * e4 + 2], -f.w * x[4 * e4 + 3]);
                        }
                        // over columns this thread has already read
                        tmem_st8(ctl + TM_D1K + 32 * hh + 8 * q, pk);
                    }
                }
                signal_rdy();

                // ---- Vn^T -> bf16 pairs (for P Vn) and decay-scaled pairs (state update) --
                wait_mma();  // Vn^T
                if (!dead) {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float4* egl4 =
                            reinterpret_cast<const float4*>(rg + RG_EGL) + 8 * hh + 4 * q;
                        float x[16];
                        tmem_ld16_sync(ctl + TM_D3 + 32 * hh + 16 * q, x);
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
                        tmem_st8(ctl + TM_D3 + 32 * hh + 8 * q, pk);  // over Vn^T columns read
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const float4 w = egl4[e4];
                            pk[2 * e4] = pack_bf16x2(x[4 * e4] * w.x, x[4 * e4 + 1] * w.y);
                            pk[2 * e4 + 1] = pack_bf16x2(x[4 * e4 + 2] * w.z, x[4 * e4 + 3] * w.w);
                        }
                        tmem_st8(ctl + TM_D1K + 16 * hh + 8 * q, pk);  // Z^T there is consumed
                    }
                }
                signal_rdy();
            }
            bool done = !dead;
            if (done && nchunks > 0) {  // the last chunk's state update
                wait_mma();
                done = !dead;
                if (done) apply_update(gamma);
            }
            if (done && Sfs) {
                float4* d4 = reinterpret_cast<float4*>(Sfs + sbase);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    d4[e] = make_float4(S[4 * e], S[4 * e + 1], S[4 * e + 2], S[4 * e + 3]);
            }
        } else {
            // ======================= state, one half of the value rows =======================
            // The block's 64 value rows 64 hv .. 64 hv + 63 sit in TMEM lanes 0-15 of each lane
            // quarter (M = 64 layout): warp w takes quarter qd = w & 3 (rows 16 qd ..) and the
            // column half hh = w >> 2 of every quantity; a thread holds rows r0 and r0 + 8 and,
            // of each 8-column group, the column pair 2 (lane % 4), + 1 (16-lane accesses).
            const int qd = warp & 3;
            const int hh = warp >> 2;
            const int r0 = 64 * hv + qd * 16 + (lane >> 2);  // value row of registers e = 0, 1
            const int cp2 = 2 * (lane & 3);
            const uint32_t ctl = tmem + ((uint32_t)(qd * 32) << 16);
            bool rd, wr;  // the sequence's state (or pool slot): read at the start, written at the end
            const int sidx = sref.resolve(n, rd, wr, tid == 0 ? status : nullptr);
            if (!GDN_IN_BOUNDS(sidx, sref.slots ? sref.num_slots : N, status)) rd = wr = false;
            const float* S0s = rd ? S0g : nullptr;
            float* Sfs = wr ? Sfg : nullptr;
            const size_t hbase = ((size_t)sidx * H_v + h) * kD * kD;
            float S[32];  // S[4 j + e]: row r0 + 8 (e >> 1), column 64 hh + 8 j + cp2 + (e & 1)
            if (S0s) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int col = 64 * hh + 8 * jj + cp2;
                    const float2 f0 = *reinterpret_cast<const float2*>(S0s + hbase + (size_t)r0 * kD + col);
                    const float2 f1 =
                        *reinterpret_cast<const float2*>(S0s + hbase + (size_t)(r0 + 8) * kD + col);
                    S[4 * jj] = f0.x; S[4 * jj + 1] = f0.y; S[4 * jj + 2] = f1.x; S[4 * jj + 3] = f1.y;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) S[e] = 0.f;
            }

            uint32_t mphase = 0;
            bool dead = false;  // warp-uniform: after an error only the barrier arrivals remain
            auto wait_mma = [&]() {
                if (dead) return;
                bool ok = *s_err == 0 && mbar_wait_bounded(mbar, mphase, wait_cycles);
                mphase ^= 1u;
                dead = __any_sync(0xffffffffu, !ok || *s_err != 0);
                if (dead) *s_err = 1;
                tc_fence_after();
            };
            // as in the full-row variant: arrive for the issuing warp, always
            auto signal_rdy = [&]() {
                if (!dead) tmem_wait_st();
                tc_fence_before();
                if (dead) named_bar_sync(kRdyBar, kRdyCount);
                else named_bar_arrive(kRdyBar, kRdyCount);
            };
            // S <- gamma S + U (the previous chunk's decay and increment)
            auto apply_update = [&](float gamma) {
                float u[32];
                tmem_ld16r_x8_sync(ctl + TM_U + 64 * hh, u);
#pragma unroll
                for (int e = 0; e < 32; ++e) S[e] = fmaf(gamma, S[e], u[e]);
            };

            float gamma = 1.f;
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % kRing;
                uint8_t* slot = sm + st * kSlotBytes;
                const float* rg = reinterpret_cast<const float*>(slot + SLOT_REC + REC_G);
                const int64_t t0 = s0 + (int64_t)c * kC;
                const int L = (int)min((int64_t)kC, s1 - t0);

                // ---- the previous chunk's state update and this chunk's data -------------
                if (c > 0) {
                    wait_mma();
                    if (!dead) apply_update(gamma);
                }
                if (!dead) {
                    const bool okf =
                        *s_err == 0 && mbar_wait_bounded(&full[st], (c / kRing) & 1, wait_cycles);
                    dead = __any_sync(0xffffffffu, !okf || *s_err != 0);
                    if (dead) *s_err = 1;
                }
                if (!dead && L < kC) {
                    // rows past the sequence's end hold the next sequence's tokens (or TMA
                    // zero fill): zero them
                    const int nz = (kC - L) * 8;  // 16-byte chunks per 64-column tile
                    for (int idx = tid; idx < 6 * nz; idx += kChain) {
                        const int tile = idx / nz, r = L + (idx % nz) / 8, ch = idx & 7;
                        const uint32_t base = tile < 4 ? SLOT_KQ + (tile >> 1) * 16384u + (tile & 1) * 8192u
                                                       : SLOT_V + (tile - 4) * 8192u;
                        *reinterpret_cast<uint4*>(slot + base + r * 128 + ch * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }

                // ---- state: bf16 pairs (A operand of S0 K^T and S0 Q^T), key k at column k/2
                if (!dead) {
                    uint32_t pk[16];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        pk[2 * jj] = pack_bf16x2(S[4 * jj], S[4 * jj + 1]);
                        pk[2 * jj + 1] = pack_bf16x2(S[4 * jj + 2], S[4 * jj + 3]);
                    }
                    tmem_st16r_x8(ctl + TM_S0B + 32 * hh, pk);
                }
                signal_rdy();
                if (!dead) gamma = rg[RG_GAMMA];

                // ---- Z^T = -(e^G rk) (S0 K^T) for this thread's tokens 32 hh + 8 j + cp2, + 1
                wait_mma();  // S0 K^T
                if (!dead) {
                    float x[16];
                    tmem_ld16r_x4_sync(ctl + TM_D1K + 32 * hh, x);
                    uint32_t pk[8];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const float2 f = *reinterpret_cast<const float2*>(rg + RG_FK + 32 * hh + 8 * jj + cp2);
                        pk[2 * jj] = pack_bf16x2(-f.x * x[4 * jj], -f.y * x[4 * jj + 1]);
                        pk[2 * jj + 1] = pack_bf16x2(-f.x * x[4 * jj + 2], -f.y * x[4 * jj + 3]);
                    }
                    // over the columns just read: pairs of tokens 32 hh + 16 q .. at 32 hh + 8 q
                    tmem_st16r_x4(ctl + TM_D1K + 32 * hh, pk);
                }
                signal_rdy();

                // ---- Vn^T -> bf16 pairs (for P Vn) and decay-scaled pairs (state update) --
                wait_mma();  // Vn^T
                if (!dead) {
                    float x[16];
                    tmem_ld16r_x4_sync(ctl + TM_D3 + 32 * hh, x);
                    uint32_t pk[8], pw[8];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const float2 w = *reinterpret_cast<const float2*>(rg + RG_EGL + 32 * hh + 8 * jj + cp2);
                        pk[2 * jj] = pack_bf16x2(x[4 * jj], x[4 * jj + 1]);
                        pk[2 * jj + 1] = pack_bf16x2(x[4 * jj + 2], x[4 * jj + 3]);
                        pw[2 * jj] = pack_bf16x2(x[4 * jj] * w.x, x[4 * jj + 1] * w.y);
                        pw[2 * jj + 1] = pack_bf16x2(x[4 * jj + 2] * w.x, x[4 * jj + 3] * w.y);
                    }
                    tmem_st16r_x4(ctl + TM_D3 + 32 * hh, pk);   // over Vn^T columns read
                    tmem_st16r_x4(ctl + TM_D1K + 16 * hh, pw);  // Z^T there is consumed
                }
                signal_rdy();
            }
            bool done = !dead;
            if (done && nchunks > 0) {  // the last chunk's state update
                wait_mma();
                done = !dead;
                if (done) apply_update(gamma);
            }
            if (done && Sfs) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int col = 64 * hh + 8 * jj + cp2;
                    *reinterpret_cast<float2*>(Sfs + hbase + (size_t)r0 * kD + col) =
                        make_float2(S[4 * jj], S[4 * jj + 1]);
                    *reinterpret_cast<float2*>(Sfs + hbase + (size_t)(r0 + 8) * kD + col) =
                        make_float2(S[4 * jj + 2], S[4 * jj + 3]);
                }
            }
        }
    }

    tc_fence_before();
    named_bar_sync(sync_id, kChainThreads);
    tc_fence_after();
    if (tid == 0 && *s_err) set_status(status, kStatusTimeout);
}

template <bool kNorm>
__global__ void __launch_bounds__(kChainThreads, 1) chain_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
    const float* S0g, const int32_t* __restrict__ cu_seqlens,
    const int32_t* __restrict__ choff, int64_t T_total, int H_qk, int H_v,
    const uint8_t* __restrict__ rec, bf16* __restrict__ o, float* Sfg, const StateIndex sref,
    int* status, long long wait_cycles, const MixerFusion mix, int N, int inject_bad_index,
    const int32_t* __restrict__ order) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned (128-byte swizzle), as an offset from the shared array itself so
    // that every pointer derived from it stays a shared-memory address for the compiler
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + CS_TMEM);
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    chain_unit<128, kNorm>(tm_q, tm_k, tm_v, tm_o, S0g, cu_seqlens, choff, T_total, H_qk, H_v, rec, o,
                    Sfg, sref, status, nullptr, 0, sm, threadIdx.x, order[blockIdx.x / H_v],
                    blockIdx.x % H_v, 0, tmem, 1, wait_cycles, mix, N, inject_bad_index != 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ==================================== fused =======================================
// Prep and chain in one cooperative launch (every block resident at once), so the
// chain of the first sequences runs while prep workers produce the later records.
// Block u < c0 runs chain unit u (sequence u / H_v, V head u % H_v); the others run
// two prep workers each (256 threads, their own 72 KB of shared memory and 128 TMEM
// columns). A chain's loader waits (bounded) for each record's flag to carry this
// call's number before its bulk copy, and prep workers never wait on chains, so
// every wait ends. Nothing in the workspace needs clearing between calls.
constexpr int kFusedThreads = 512;
constexpr uint32_t kPrepRegion = 73728;
static_assert(kPrepRegion + 1024 >= kPrepSmem, "prep worker region too small");
constexpr size_t kFusedSmem =
    kChainSmem > 2 * (size_t)kPrepRegion + 1024 ? kChainSmem : 2 * (size_t)kPrepRegion + 1024;
constexpr int kChainSync = 5;  // named barrier of the chain threads in the fused kernel
constexpr int kFusedMaxSeqs = 255;  // the fused kernel computes the chunk offsets itself

template <int kM, bool kMix>
__global__ void __launch_bounds__(kFusedThreads, 1) fused_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
    const bf16* __restrict__ q, const bf16* __restrict__ k, const float* __restrict__ a,
    const float* __restrict__ b, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, const float* S0g,
    const int32_t* __restrict__ cu_seqlens, const int32_t* choff, int32_t N,
    int64_t T_total, int H_qk, int H_v, float scale, uint8_t* __restrict__ rec,
    bf16* __restrict__ o, float* Sfg, const StateIndex sref,
    int* status, unsigned long long* flags, unsigned long long epoch, int c0,
    long long wait_cycles, int withhold_records, const MixerFusion mix, int inject_bad_index,
    int64_t qk_tok) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int32_t s_choff[kFusedMaxSeqs + 1];
    __shared__ int s_bad;
    // 1024-byte aligned (128-byte swizzle), as an offset from the shared array itself so
    // that every pointer derived from it stays a shared-memory address for the compiler
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x;
    // chunk offsets of the sequences (prefix sum of ceil(len / 64)), by one warp
    if (tid < 32) {
        int32_t carry = 0;
        bool bad = false;
        for (int base = 0; base < N; base += 32) {
            const int n = base + tid;
            int32_t nc = 0;
            if (n < N) {
                const int64_t s0 = cu_seqlens[n], s1 = cu_seqlens[n + 1];
                if (bad_seq(s0, s1, T_total, n)) bad = true;
                else nc = (int32_t)((s1 - s0 + kC - 1) / kC);
            }
            int32_t x = nc;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
                if (tid >= off) x += y;
            }
            if (n < N) s_choff[n] = carry + x - nc;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        bad = __any_sync(0xffffffffu, bad);
        if (tid == 0) {
            s_choff[N] = carry;
            s_bad = bad ? 1 : 0;
            if (bad && blockIdx.x == 0) set_status(status, kStatusBadSeqlens);
        }
    }
    __syncthreads();
    if (s_bad) return;  // reported; nothing is computed
    choff = s_choff;
    if ((int)blockIdx.x >= c0) {
        const int sub = tid >> 8;
        // a fault-injection call withholds every record: the chains' waits run out
        prep_worker<kMix>(q, k, a, b, A_log, dt_bias, cu_seqlens, choff, N, H_qk, H_v, scale, rec,
                    status, withhold_records ? nullptr : flags, epoch, sm + sub * kPrepRegion,
                    tid & 255, 3 + sub, 2 * ((int)blockIdx.x - c0) + sub,
                    2 * ((int)gridDim.x - c0), false, wait_cycles, mix, qk_tok,
                    T_total, &tm_q, &tm_k);
        return;
    }
    if (tid >= kChainThreads) return;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + CS_TMEM);
    if ((tid >> 5) == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    named_bar_sync(kChainSync, kChainThreads);
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // block u: (sequence, V head) u, or with half-row blocks its half u & 1 of unit u >> 1
    const int u = kM == 64 ? (int)blockIdx.x >> 1 : (int)blockIdx.x;
    const int hv = kM == 64 ? (int)blockIdx.x & 1 : 0;
    chain_unit<kM, kMix>(tm_q, tm_k, tm_v, tm_o, S0g, cu_seqlens, choff, T_total, H_qk, H_v, rec, o,
                   Sfg, sref, status, flags, epoch, sm, tid, u / H_v, u % H_v, hv, tmem,
                   kChainSync, wait_cycles, mix, N, inject_bad_index != 0);
    tc_fence_before();
    named_bar_sync(kChainSync, kChainThreads);
    tc_fence_after();
    if ((tid >> 5) == 0) tmem_dealloc(tmem, kTmemCols);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct TcWorkspace {
    size_t off_flags, off_rec, total;
};

// Workspace: chunk offsets [N + 1], chain order [N] | record flags [records] (64-bit call
// numbers) | records [chunks][H_v].
TcWorkspace tc_workspace_layout(int32_t N, int64_t T, int32_t H_v) {
    const size_t chunks = (size_t)((T + kC - 1) / kC) + (size_t)N;
    const size_t records = chunks * H_v;
    TcWorkspace w;
    w.off_flags = align256((size_t)(2 * N + 1) * sizeof(int32_t));
    w.off_rec = w.off_flags + align256(records * sizeof(unsigned long long));
    w.total = w.off_rec + records * kRecBytes;
    return w;
}

// The number a call publishes its records under. Flags hold the number of the call
// that wrote them last, or whatever the workspace held before; a chain takes a record
// as published only when its flag equals this call's number. The numbers are a random
// 64-bit base drawn once per process (top bit set) plus a call counter, so no earlier
// call of this process used this call's number, and stale contents of any other origin
// (small integers, floats, another process's flags) match it only by chance, with
// probability 2^-64 per flag.
unsigned long long next_call_number() {
    static const unsigned long long base = [] {
        unsigned long long x = 0;
        try {
            std::random_device rd;
            x = ((unsigned long long)rd() << 32) ^ (unsigned long long)rd();
        } catch (...) {
        }
        x ^= (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() *
             0x9E3779B97F4A7C15ull;
        x ^= (unsigned long long)getpid() * 0xC2B2AE3D27D4EB4Full;
        return x | (1ull << 63);
    }();
    static std::atomic<unsigned long long> counter{0};
    return base + counter.fetch_add(1) + 1;
}

}  // namespace

size_t prefill_tc_workspace_bytes(int32_t N, int64_t T, int32_t H_v) {
    return tc_workspace_layout(N, T, H_v).total;
}

bool prefill_tc_supported(int32_t H_qk, int32_t H_v) { return H_v / H_qk <= kMaxGroup; }

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [T][heads][128] bf16 rows as a 3-D tensor (d, head, token); boxes of 64 d x 1
// head x 64 tokens move as 64 rows of 128 bytes in the 128-byte swizzle. Tokens
// past T read as zeros and are not written. token_elems: elements from one token's
// rows to the next one's (0: heads x 128, a dense tensor).
bool make_rows_map(CUtensorMap* m, const void* base, int heads, int64_t T,
                   int64_t token_elems = 0) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    if (token_elems == 0) token_elems = (int64_t)heads * kD;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)heads, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)token_elems * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kC};
    const cuuint32_t estride[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, const float* a,
                              const float* b, const float* A_log, const float* dt_bias,
                              const float* S0, const int32_t* cu_seqlens, int32_t N, int64_t T,
                              int32_t H_qk, int32_t H_v, float scale, void* o, float* S_final,
                              StateIndex sref, void* workspace, const PrefillOpts& opt,
                              int* status, cudaStream_t s, const MixerFusion& mix,
                              int64_t qkv_tok) {
    if (N == 0) return cudaSuccess;
    if (T > (int64_t)0x7FFFFFFF - kC) return cudaErrorInvalidValue;  // TMA token coordinates
    const TcWorkspace ws = tc_workspace_layout(N, T, H_v);
    uint8_t* wb = static_cast<uint8_t*>(workspace);
    int32_t* choff = reinterpret_cast<int32_t*>(wb);
    unsigned long long* flags = reinterpret_cast<unsigned long long*>(wb + ws.off_flags);
    uint8_t* rec = wb + ws.off_rec;
    // With no tokens the maps are never read; any aligned device address will do.
    // In the mixer, q, k and v are the convolution's output: views of the post-conv
    // buffer [T][conv_dim] (q | k | v), written by the preparation (convolution fused into
    // its loads) or by the standalone convolution kernel before it.
    CUtensorMap tm_q, tm_k, tm_v, tm_o;
    // q, k and v rows are token_stride apart (0: dense [T][heads][128] tensors): views of
    // one [T][conv_dim] buffer in the mixer, fused or not
    const bool mixer = mix.qkvc != nullptr;
    const int64_t tok = mixer ? (int64_t)mix.conv_dim : qkv_tok;
    const int64_t qk_tok = tok ? tok : (int64_t)H_qk * kD;  // elements from one q/k row to the next token's
    const void* qv = mixer ? (const void*)mix.qkvc : q;
    const void* kv = mixer ? (const void*)(mix.qkvc + (size_t)H_qk * kD) : k;
    const void* vv = mixer ? (const void*)(mix.qkvc + (size_t)2 * H_qk * kD) : v;
    if (!make_rows_map(&tm_q, T > 0 ? qv : workspace, H_qk, T, tok) ||
        !make_rows_map(&tm_k, T > 0 ? kv : workspace, H_qk, T, tok) ||
        !make_rows_map(&tm_v, T > 0 ? vv : workspace, H_v, T, tok) ||
        !make_rows_map(&tm_o, T > 0 ? o : workspace, H_v, T))
        return cudaErrorInvalidValue;
    int dev = 0, num_sms = 0, coop = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        num_sms <= 0)
        num_sms = 148;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) coop = 0;
    cudaError_t e;
    const int64_t chain_units = (int64_t)N * H_v;
    long long wait_cycles = opt.wait_cycles;
    const bool separate = opt.impl == GDN_IMPL_TENSOR_CORE_SPLIT;
    const bool whole_rows = opt.impl == GDN_IMPL_TENSOR_CORE_WHOLE_ROWS;

    if (!separate && coop) {
        // Overlap pays when the chains are few (latency-bound: each holds one SM for
        // its whole sequence); with many chains the separate launches keep both
        // phases at full occupancy. With at most a quarter as many chains as SMs each
        // chain runs as two blocks of 64 value rows (half the per-thread state work on
        // the critical path).
        // (the fused gated norm needs all 128 values of a token in one block)
        const bool half = !whole_rows && !mixer && 4 * chain_units <= num_sms;
        const void* kfn = mixer ? (const void*)fused_kernel<128, true>
                        : half  ? (const void*)fused_kernel<64, false>
                                : (const void*)fused_kernel<128, false>;
        e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kFusedSmem);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, kFusedThreads,
                                                          kFusedSmem);
        if (e != cudaSuccess) return e;
        const int grid = per_sm >= 1 ? num_sms : 0;
        const int64_t chain_blocks = (half ? 2 : 1) * chain_units;
        if (grid >= 2 && 2 * chain_blocks <= grid && N <= kFusedMaxSeqs) {
            unsigned long long epoch = next_call_number();
            const bf16* qb = static_cast<const bf16*>(q);
            const bf16* kb = static_cast<const bf16*>(k);
            bf16* ob = static_cast<bf16*>(o);
            int c0v = (int)chain_blocks;
            int withhold = opt.fault == GDN_FAULT_WITHHOLD_RECORDS ? 1 : 0;
            int inject = opt.fault == GDN_FAULT_BAD_INDEX ? 1 : 0;
            void* args[] = {&tm_q, &tm_k, &tm_v, &tm_o, &qb, &kb, &a, &b, &A_log, &dt_bias, &S0,
                            &cu_seqlens, &choff, &N, &T, &H_qk, &H_v, &scale, &rec, &ob,
                            &S_final, &sref, &status, &flags, &epoch, &c0v, &wait_cycles,
                            &withhold, const_cast<MixerFusion*>(&mix), &inject,
                            const_cast<int64_t*>(&qk_tok)};
            timer_before(opt.timer, s);
            e = cudaLaunchCooperativeKernel(kfn, dim3(grid), dim3(kFusedThreads), args, kFusedSmem,
                                            s);
            if (e == cudaSuccess) timer_after(opt.timer, s, half ? "fused_half_rows" : "fused");
            return e;
        }
    }

    // Separate launches. In the mixer the convolution then runs as its own streaming
    // kernel first (the preparation is the slower stage here, and the convolution would
    // add to it): it writes the post-conv buffer and the conv cache, the preparation
    // reads its q and k rows from that buffer, and the chain applies the gated norm.
    MixerFusion mix_split = mix;
    mix_split.x = nullptr;
    mix_split.cache_out = nullptr;
    if (mixer && T > 0) {
        timer_before(opt.timer, s);
        e = launch_conv1d_silu(mix.x, GDN_BF16, mix.conv_w, mix.conv_b, mix.cache_in, cu_seqlens,
                               N, T, mix.conv_dim, mix.K, mix.qkvc, mix.cache_out, status, s);
        if (e != cudaSuccess) return e;
        timer_after(opt.timer, s, "conv1d_silu");
    } else if (mixer && mix.cache_out) {  // no tokens: only the cache (kept) to write
        e = launch_conv1d_silu(mix.x, GDN_BF16, mix.conv_w, mix.conv_b, mix.cache_in, cu_seqlens,
                               N, T, mix.conv_dim, mix.K, mix.qkvc, mix.cache_out, status, s);
        if (e != cudaSuccess) return e;
    }
    const bf16* q_rows = mixer ? mix.qkvc : static_cast<const bf16*>(q);
    const bf16* k_rows = mixer ? mix.qkvc + (size_t)H_qk * kD : static_cast<const bf16*>(k);
    const auto prep_fn = prep_kernel<false>;
    const auto chain_fn = mixer ? chain_kernel<true> : chain_kernel<false>;
    e = cudaFuncSetAttribute(prep_fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPrepSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(prep_fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chain_fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kChainSmem);
    if (e != cudaSuccess) return e;
    timer_before(opt.timer, s);
    chunk_offsets_kernel<<<1, 256, 0, s>>>(cu_seqlens, N, T, choff, choff + N + 1, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    timer_after(opt.timer, s, "chunk_offsets");
    // Prep workers never wait on one another, so any grid size is safe: one wave of
    // them at the residency the launch bounds ask for (the shared-memory carveout is
    // set to its maximum so that it is reached).
    const int64_t unit_bound = (((T + kC - 1) / kC) + N) * (int64_t)H_qk;
    const int64_t grid_cap = (int64_t)kPrepBlocksPerSm * num_sms;
    const int prep_grid = (int)(unit_bound < grid_cap ? unit_bound : grid_cap);
    if (prep_grid > 0) {
        timer_before(opt.timer, s);
        prep_fn<<<prep_grid, kPrepThreads, kPrepSmem, s>>>(
            tm_q, tm_k, q_rows, k_rows, a, b, A_log, dt_bias, cu_seqlens, choff, N, H_qk, H_v, scale, rec,
            status, wait_cycles, mix_split, qk_tok, T);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        timer_after(opt.timer, s, "prep");
    }
    timer_before(opt.timer, s);
    chain_fn<<<(unsigned)chain_units, kChainThreads, kChainSmem, s>>>(
        tm_q, tm_k, tm_v, tm_o, S0, cu_seqlens, choff, T, H_qk, H_v, rec, static_cast<bf16*>(o),
        S_final, sref, status, wait_cycles, mix_split, N,
        opt.fault == GDN_FAULT_BAD_INDEX ? 1 : 0, choff + N + 1);
    e = cudaGetLastError();
    if (e == cudaSuccess) timer_after(opt.timer, s, "chain");
    return e;
}

}  // namespace gdn
