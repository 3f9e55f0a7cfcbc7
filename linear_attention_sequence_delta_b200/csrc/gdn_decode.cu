// Single-token decode: one step of the gated delta rule per (sequence, V head),
// the fp32 state updated in place ("Qwen3.5 observation notes",
// "Qwen3_5MoeGatedDeltaNet", the recurrent kernel for seq_len == 1).
//
// With the value-major state S[i][c] (i: value index, c: key index) every value
// row evolves on its own:
//   S_i <- alpha S_i;  delta_i = beta (v_i - S_i . k);  S_i <- S_i + delta_i k;
//   o_i = S_i . q = alpha (S_old_i . q) + delta_i (k . q)
// so one pass that reads a row, forms two dot products (with k and q), and
// writes the row back does the whole step. The kernel is HBM-bound: 2 * 4 * d^2
// bytes of state per head move per token, against ~7 d^2 flops.
//
// Mapping: one 128-thread block per (sequence, head). A warp covers four rows at
// a time, eight lanes per row, each lane holding d/8 consecutive-by-float4
// elements (offsets 4p + 32m), so every load and store instruction moves four
// fully used 128-byte lines. The two dot products reduce over the eight lanes
// of a row with three xor shuffles each. Loads of two row groups are issued
// before any arithmetic so each lane keeps 2 * d/32 16-byte loads in flight.
#include "gdn_internal.cuh"

namespace gdn {

namespace {

template <typename IO, int NE>
__device__ __forceinline__ void load_vec(const IO* p, float (&out)[NE]);

template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&out)[4]) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
}

template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16* p,
                                                          float (&out)[4]) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&x.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&x.y);
    const float2 l = __bfloat1622float2(lo), h = __bfloat1622float2(hi);
    out[0] = l.x; out[1] = l.y; out[2] = h.x; out[3] = h.y;
}

constexpr int kRowGroupsInFlight = 2;

template <typename IO, int D>
__global__ void __launch_bounds__(128, 4) decode_kernel(
    const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
    const float* __restrict__ a, const float* __restrict__ b,
    const float* __restrict__ A_log, const float* __restrict__ dt_bias,
    float* __restrict__ state, int H_qk, int H_v, float scale, IO* __restrict__ o) {
    constexpr int NV = D / 32;               // float4 chunks per lane per row
    constexpr int ROWS_PER_WARP = D / 4;     // 4 warps share the D rows
    constexpr int ITERS = ROWS_PER_WARP / 4; // 4 rows per warp-iteration
    constexpr int B = kRowGroupsInFlight;
    static_assert(ITERS % B == 0, "row groups must tile the warp's rows");

    const int unit = blockIdx.x;  // n * H_v + h
    const int n = unit / H_v;
    const int h = unit - n * H_v;
    const int j = h / (H_v / H_qk);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int p = lane & 7;   // position inside the row
    const int rg = lane >> 3; // which of the four rows

    // normalised q and k, in the lane's column pattern (cols 4p + 32m .. +3)
    float kr[NV][4], qr[NV][4];
    const IO* qp = q + ((size_t)n * H_qk + j) * D;
    const IO* kp = k + ((size_t)n * H_qk + j) * D;
#pragma unroll
    for (int m = 0; m < NV; ++m) {
        load_vec<IO, 4>(qp + 4 * p + 32 * m, qr[m]);
        load_vec<IO, 4>(kp + 4 * p + 32 * m, kr[m]);
    }
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int m = 0; m < NV; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sq = fmaf(qr[m][e], qr[m][e], sq);
            sk = fmaf(kr[m][e], kr[m][e], sk);
        }
#pragma unroll
    for (int x = 1; x < 8; x <<= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, x);
        sk += __shfl_xor_sync(0xffffffffu, sk, x);
    }
    const float rq = scale / sqrtf(sq + kL2Eps);
    const float rk = 1.f / sqrtf(sk + kL2Eps);
    float kq = 0.f;
#pragma unroll
    for (int m = 0; m < NV; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            qr[m][e] *= rq;
            kr[m][e] *= rk;
            kq = fmaf(kr[m][e], qr[m][e], kq);
        }
#pragma unroll
    for (int x = 1; x < 8; x <<= 1) kq += __shfl_xor_sync(0xffffffffu, kq, x);

    const float alpha = expf(gate_g(a[unit], A_log[h], dt_bias[h]));
    const float beta = gate_beta(b[unit]);

    float* S = state + (size_t)unit * D * D;
    const IO* vp = v + (size_t)unit * D;
    IO* op = o + (size_t)unit * D;

#pragma unroll 1
    for (int it0 = 0; it0 < ITERS; it0 += B) {
        float4 s[B][NV];
        float vi[B];
#pragma unroll
        for (int bb = 0; bb < B; ++bb) {
            const int row = warp * ROWS_PER_WARP + (it0 + bb) * 4 + rg;
            const float* rp = S + (size_t)row * D + 4 * p;
#pragma unroll
            for (int m = 0; m < NV; ++m) s[bb][m] = __ldcs(reinterpret_cast<const float4*>(rp + 32 * m));
            vi[bb] = to_f32(vp[row]);
        }
#pragma unroll
        for (int bb = 0; bb < B; ++bb) {
            const int row = warp * ROWS_PER_WARP + (it0 + bb) * 4 + rg;
            float dk = 0.f, dq = 0.f;
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                dk = fmaf(s[bb][m].x, kr[m][0], dk); dq = fmaf(s[bb][m].x, qr[m][0], dq);
                dk = fmaf(s[bb][m].y, kr[m][1], dk); dq = fmaf(s[bb][m].y, qr[m][1], dq);
                dk = fmaf(s[bb][m].z, kr[m][2], dk); dq = fmaf(s[bb][m].z, qr[m][2], dq);
                dk = fmaf(s[bb][m].w, kr[m][3], dk); dq = fmaf(s[bb][m].w, qr[m][3], dq);
            }
#pragma unroll
            for (int x = 1; x < 8; x <<= 1) {
                dk += __shfl_xor_sync(0xffffffffu, dk, x);
                dq += __shfl_xor_sync(0xffffffffu, dq, x);
            }
            // read with the decayed state, then write
            const float delta = beta * (vi[bb] - alpha * dk);
            float* rp = S + (size_t)row * D + 4 * p;
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                float4 w;
                w.x = fmaf(alpha, s[bb][m].x, delta * kr[m][0]);
                w.y = fmaf(alpha, s[bb][m].y, delta * kr[m][1]);
                w.z = fmaf(alpha, s[bb][m].z, delta * kr[m][2]);
                w.w = fmaf(alpha, s[bb][m].w, delta * kr[m][3]);
                __stcs(reinterpret_cast<float4*>(rp + 32 * m), w);
            }
            if (p == 0) op[row] = from_f32<IO>(fmaf(alpha, dq, delta * kq));
        }
    }
}

template <typename IO, int D>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* a,
                            const float* b, const float* A_log, const float* dt_bias,
                            float* state, int32_t N, int32_t H_qk, int32_t H_v, float scale,
                            void* o, cudaStream_t s) {
    const int64_t units = (int64_t)N * H_v;
    if (units == 0) return cudaSuccess;
    decode_kernel<IO, D><<<(unsigned)units, 128, 0, s>>>(
        static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(v), a, b,
        A_log, dt_bias, state, H_qk, H_v, scale, static_cast<IO*>(o));
    return cudaGetLastError();
}

// The same step with the state stored in bf16 ("Qwen3.5-MoE-35B-A3B architecture
// teardown", section 9.4: the fp32 state could move to bf16 to save half of its
// memory; for decode that is also half the traffic): the state is read as bf16, updated in fp32 and
// rounded to bf16 (round to nearest even) when written back. A lane holds 8
// consecutive columns per 16-byte access (columns 8p + 64m), so every load and store
// is 16 bytes as in the fp32 kernel.
template <typename IO, int D>
__global__ void __launch_bounds__(128, 5) decode_bf16_state_kernel(
    const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
    const float* __restrict__ a, const float* __restrict__ b,
    const float* __restrict__ A_log, const float* __restrict__ dt_bias,
    __nv_bfloat16* __restrict__ state, int H_qk, int H_v, float scale, IO* __restrict__ o) {
    constexpr int NV = D / 64;               // 16-byte chunks of 8 columns per lane per row
    constexpr int ROWS_PER_WARP = D / 4;
    constexpr int ITERS = ROWS_PER_WARP / 4;
    constexpr int B = 2 * kRowGroupsInFlight;  // half the bytes per row: twice the rows
    static_assert(ITERS % B == 0, "row groups must tile the warp's rows");
    // Each warp keeps its own copy of the normalised q and k in shared memory (read back
    // as 16-byte broadcasts), which leaves registers for 8 blocks per SM.
    __shared__ __align__(16) float qk_s[4][2][D];

    const int unit = blockIdx.x;
    const int n = unit / H_v;
    const int h = unit - n * H_v;
    const int j = h / (H_v / H_qk);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int p = lane & 7;
    const int rg = lane >> 3;

    __nv_bfloat16* S = state + (size_t)unit * D * D;
    const IO* vp = v + (size_t)unit * D;
    IO* op = o + (size_t)unit * D;

    // the first row groups' state loads go out before the q/k work they do not need
    uint4 raw[B][NV];
    float vi[B];
    auto load_groups = [&](int it0) {
#pragma unroll
        for (int bb = 0; bb < B; ++bb) {
            const int row = warp * ROWS_PER_WARP + (it0 + bb) * 4 + rg;
            const __nv_bfloat16* rp = S + (size_t)row * D + 8 * p;
#pragma unroll
            for (int m = 0; m < NV; ++m) raw[bb][m] = __ldcs(reinterpret_cast<const uint4*>(rp + 64 * m));
            vi[bb] = to_f32(vp[row]);
        }
    };
    load_groups(0);

    // normalised q and k (lane owns columns lane + 32 m), written to this warp's copy
    const IO* qp = q + ((size_t)n * H_qk + j) * D;
    const IO* kp = k + ((size_t)n * H_qk + j) * D;
    float qv[D / 32], kv[D / 32];
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int m = 0; m < D / 32; ++m) {
        qv[m] = to_f32(qp[lane + 32 * m]);
        kv[m] = to_f32(kp[lane + 32 * m]);
        sq = fmaf(qv[m], qv[m], sq);
        sk = fmaf(kv[m], kv[m], sk);
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    const float rq = scale / sqrtf(sq + kL2Eps);
    const float rk = 1.f / sqrtf(sk + kL2Eps);
    float kq = 0.f;
#pragma unroll
    for (int m = 0; m < D / 32; ++m) {
        qv[m] *= rq;
        kv[m] *= rk;
        kq = fmaf(kv[m], qv[m], kq);
        qk_s[warp][0][lane + 32 * m] = qv[m];
        qk_s[warp][1][lane + 32 * m] = kv[m];
    }
    kq = warp_sum(kq);
    __syncwarp();
    const float alpha = expf(gate_g(a[unit], A_log[h], dt_bias[h]));
    const float beta = gate_beta(b[unit]);
    const float* qs = qk_s[warp][0];
    const float* ks = qk_s[warp][1];

#pragma unroll 1
    for (int it0 = 0; it0 < ITERS; it0 += B) {
        if (it0 > 0) load_groups(it0);
#pragma unroll
        for (int bb = 0; bb < B; ++bb) {
            const int row = warp * ROWS_PER_WARP + (it0 + bb) * 4 + rg;
            float sv[NV][8];
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&raw[bb][m]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hp[e]);
                    sv[m][2 * e] = f.x;
                    sv[m][2 * e + 1] = f.y;
                }
            }
            float dk = 0.f, dq = 0.f;
#pragma unroll
            for (int m = 0; m < NV; ++m)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float4 k4 = *reinterpret_cast<const float4*>(ks + 8 * p + 64 * m + 4 * hh);
                    const float4 q4 = *reinterpret_cast<const float4*>(qs + 8 * p + 64 * m + 4 * hh);
                    const float* sp = sv[m] + 4 * hh;
                    dk = fmaf(sp[0], k4.x, dk); dq = fmaf(sp[0], q4.x, dq);
                    dk = fmaf(sp[1], k4.y, dk); dq = fmaf(sp[1], q4.y, dq);
                    dk = fmaf(sp[2], k4.z, dk); dq = fmaf(sp[2], q4.z, dq);
                    dk = fmaf(sp[3], k4.w, dk); dq = fmaf(sp[3], q4.w, dq);
                }
#pragma unroll
            for (int x = 1; x < 8; x <<= 1) {
                dk += __shfl_xor_sync(0xffffffffu, dk, x);
                dq += __shfl_xor_sync(0xffffffffu, dq, x);
            }
            const float delta = beta * (vi[bb] - alpha * dk);
            __nv_bfloat16* rp = S + (size_t)row * D + 8 * p;
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                const float4 k0 = *reinterpret_cast<const float4*>(ks + 8 * p + 64 * m);
                const float4 k1 = *reinterpret_cast<const float4*>(ks + 8 * p + 64 * m + 4);
                const float kk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                uint4 w;
                __nv_bfloat162* wh = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    wh[e] = __floats2bfloat162_rn(fmaf(alpha, sv[m][2 * e], delta * kk[2 * e]),
                                                  fmaf(alpha, sv[m][2 * e + 1],
                                                       delta * kk[2 * e + 1]));
                __stcs(reinterpret_cast<uint4*>(rp + 64 * m), w);
            }
            if (p == 0) op[row] = from_f32<IO>(fmaf(alpha, dq, delta * kq));
        }
    }
}

template <typename IO, int D>
cudaError_t launch_decode_bf16_state_t(const void* q, const void* k, const void* v,
                                       const float* a, const float* b, const float* A_log,
                                       const float* dt_bias, void* state, int32_t N,
                                       int32_t H_qk, int32_t H_v, float scale, void* o,
                                       cudaStream_t s) {
    const int64_t units = (int64_t)N * H_v;
    if (units == 0) return cudaSuccess;
    decode_bf16_state_kernel<IO, D><<<(unsigned)units, 128, 0, s>>>(
        static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(v), a, b,
        A_log, dt_bias, static_cast<__nv_bfloat16*>(state), H_qk, H_v, scale,
        static_cast<IO*>(o));
    return cudaGetLastError();
}

// Decode of L tokens per sequence from a state pool ("Qwen3.5 observation notes",
// section "Cache": a request keeps one batch index of the cache for its whole life;
// "Qwen3.5-MoE-35B-A3B architecture teardown", section 6.2: the main model checks an MTP
// draft token in the same forward pass, i.e. several tokens per step). The
// state of sequence n lives in pool slot slots[n] (n without slots). Each block owns one
// (sequence, V head); its rows stay in registers across the L tokens, so the state is
// read and written once per call whatever L is. Normalised q, k, the values and the gates
// of the L tokens are staged in shared memory first. With `inter`, the state after every
// token is also written out (for rolling back rejected drafts).
template <typename IO, int D>
__global__ void __launch_bounds__(128) decode_multi_kernel(
    const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
    const float* __restrict__ a, const float* __restrict__ b, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, float* __restrict__ pool,
    const int32_t* __restrict__ slots, int num_slots, int L, int H_qk, int H_v, float scale,
    IO* __restrict__ o, float* __restrict__ inter, int* status) {
    constexpr int NV = D / 32;
    constexpr int ROWS_PER_WARP = D / 4;
    constexpr int ITERS = ROWS_PER_WARP / 4;
    extern __shared__ float4 dm_smem[];
    float* qs = reinterpret_cast<float*>(dm_smem);  // [L][D] normalised, scaled q
    float* ks = qs + L * D;                          // [L][D] normalised k
    float* vs = ks + L * D;                          // [L][D] values
    float* par = vs + L * D;                         // [L][4]: alpha, beta, k.q

    const int unit = blockIdx.x;  // n * H_v + h
    const int n = unit / H_v;
    const int h = unit - n * H_v;
    const int j = h / (H_v / H_qk);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int slot = slots ? slots[n] : n;
    if (slot < 0) {  // a padding entry: zero outputs, no state touched
        for (int idx = threadIdx.x; idx < L * D; idx += blockDim.x) {
            const int t = idx / D, i = idx - t * D;
            o[(((size_t)n * L + t) * H_v + h) * D + i] = from_f32<IO>(0.f);
        }
        return;
    }
    if (slot >= num_slots) {
        if (threadIdx.x == 0) set_status(status, kStatusBadSlot);
        return;
    }
    // stage the L tokens: one warp per token, lane owns columns lane + 32 m
    for (int t = warp; t < L; t += 4) {
        const size_t tok = (size_t)n * L + t;
        const IO* qp = q + (tok * H_qk + j) * D;
        const IO* kp = k + (tok * H_qk + j) * D;
        const IO* vp = v + (tok * H_v + h) * D;
        float qv[NV], kv[NV];
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int m = 0; m < NV; ++m) {
            qv[m] = to_f32(qp[lane + 32 * m]);
            kv[m] = to_f32(kp[lane + 32 * m]);
            vs[t * D + lane + 32 * m] = to_f32(vp[lane + 32 * m]);
            sq = fmaf(qv[m], qv[m], sq);
            sk = fmaf(kv[m], kv[m], sk);
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        const float rq = scale / sqrtf(sq + kL2Eps);
        const float rk = 1.f / sqrtf(sk + kL2Eps);
        float kq = 0.f;
#pragma unroll
        for (int m = 0; m < NV; ++m) {
            qv[m] *= rq;
            kv[m] *= rk;
            kq = fmaf(kv[m], qv[m], kq);
            qs[t * D + lane + 32 * m] = qv[m];
            ks[t * D + lane + 32 * m] = kv[m];
        }
        kq = warp_sum(kq);
        if (lane == 0) {
            const size_t gi = tok * H_v + h;
            par[4 * t + 0] = expf(gate_g(a[gi], A_log[h], dt_bias[h]));
            par[4 * t + 1] = gate_beta(b[gi]);
            par[4 * t + 2] = kq;
        }
    }
    __syncthreads();

    const int p = lane & 7;
    const int rg = lane >> 3;
    float* S = pool + ((size_t)slot * H_v + h) * D * D;
#pragma unroll 1
    for (int it = 0; it < ITERS; ++it) {
        const int row = warp * ROWS_PER_WARP + it * 4 + rg;
        float4 sr[NV];
        const float* rp = S + (size_t)row * D + 4 * p;
#pragma unroll
        for (int m = 0; m < NV; ++m) sr[m] = __ldcs(reinterpret_cast<const float4*>(rp + 32 * m));
#pragma unroll 1
        for (int t = 0; t < L; ++t) {
            const float alpha = par[4 * t], beta = par[4 * t + 1], kq = par[4 * t + 2];
            float4 kr[NV], qr[NV];
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                kr[m] = *reinterpret_cast<const float4*>(ks + t * D + 4 * p + 32 * m);
                qr[m] = *reinterpret_cast<const float4*>(qs + t * D + 4 * p + 32 * m);
            }
            float dk = 0.f, dq = 0.f;
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                dk = fmaf(sr[m].x, kr[m].x, dk); dq = fmaf(sr[m].x, qr[m].x, dq);
                dk = fmaf(sr[m].y, kr[m].y, dk); dq = fmaf(sr[m].y, qr[m].y, dq);
                dk = fmaf(sr[m].z, kr[m].z, dk); dq = fmaf(sr[m].z, qr[m].z, dq);
                dk = fmaf(sr[m].w, kr[m].w, dk); dq = fmaf(sr[m].w, qr[m].w, dq);
            }
#pragma unroll
            for (int x = 1; x < 8; x <<= 1) {
                dk += __shfl_xor_sync(0xffffffffu, dk, x);
                dq += __shfl_xor_sync(0xffffffffu, dq, x);
            }
            const float delta = beta * (vs[t * D + row] - alpha * dk);
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                sr[m].x = fmaf(alpha, sr[m].x, delta * kr[m].x);
                sr[m].y = fmaf(alpha, sr[m].y, delta * kr[m].y);
                sr[m].z = fmaf(alpha, sr[m].z, delta * kr[m].z);
                sr[m].w = fmaf(alpha, sr[m].w, delta * kr[m].w);
            }
            const size_t tok = (size_t)n * L + t;
            if (p == 0) o[(tok * H_v + h) * D + row] = from_f32<IO>(fmaf(alpha, dq, delta * kq));
            if (inter) {
                float* ip = inter + (tok * H_v + h) * D * D + (size_t)row * D + 4 * p;
#pragma unroll
                for (int m = 0; m < NV; ++m) __stcs(reinterpret_cast<float4*>(ip + 32 * m), sr[m]);
            }
        }
        float* wp = S + (size_t)row * D + 4 * p;
#pragma unroll
        for (int m = 0; m < NV; ++m) __stcs(reinterpret_cast<float4*>(wp + 32 * m), sr[m]);
    }
}

template <typename IO, int D>
cudaError_t launch_decode_multi_t(const void* q, const void* k, const void* v, const float* a,
                                  const float* b, const float* A_log, const float* dt_bias,
                                  float* pool, const int32_t* slots, int32_t num_slots,
                                  int32_t N, int32_t L, int32_t H_qk, int32_t H_v, float scale,
                                  void* o, float* inter, int* status, cudaStream_t s) {
    const int64_t units = (int64_t)N * H_v;
    if (units == 0) return cudaSuccess;
    const size_t smem = (size_t)L * (3 * D + 4) * sizeof(float);
    decode_multi_kernel<IO, D><<<(unsigned)units, 128, smem, s>>>(
        static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(v), a, b,
        A_log, dt_bias, pool, slots, num_slots, L, H_qk, H_v, scale, static_cast<IO*>(o), inter,
        status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_multi(const void* q, const void* k, const void* v, int io_dtype,
                                const float* a, const float* b, const float* A_log,
                                const float* dt_bias, float* pool, const int32_t* slots,
                                int32_t num_slots, int32_t N, int32_t L, int32_t H_qk,
                                int32_t H_v, int32_t d, float scale, void* o, float* inter,
                                int* status, cudaStream_t s) {
#define GDN_DM(IO, D)                                                                          \
    return launch_decode_multi_t<IO, D>(q, k, v, a, b, A_log, dt_bias, pool, slots, num_slots, \
                                        N, L, H_qk, H_v, scale, o, inter, status, s)
    if (io_dtype == GDN_BF16) {
        if (d == 128) GDN_DM(__nv_bfloat16, 128);
        GDN_DM(__nv_bfloat16, 64);
    }
    if (d == 128) GDN_DM(float, 128);
    GDN_DM(float, 64);
#undef GDN_DM
}

cudaError_t launch_decode_bf16_state(const void* q, const void* k, const void* v,
                                     int io_dtype, const float* a, const float* b,
                                     const float* A_log, const float* dt_bias, void* state,
                                     int32_t N, int32_t H_qk, int32_t H_v, int32_t d,
                                     float scale, void* o, cudaStream_t s) {
#define GDN_DB(IO, D)                                                                       \
    return launch_decode_bf16_state_t<IO, D>(q, k, v, a, b, A_log, dt_bias, state, N, H_qk, \
                                             H_v, scale, o, s)
    if (io_dtype == GDN_BF16) {
        if (d == 128) GDN_DB(__nv_bfloat16, 128);
        GDN_DB(__nv_bfloat16, 64);
    }
    if (d == 128) GDN_DB(float, 128);
    GDN_DB(float, 64);
#undef GDN_DB
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, int io_dtype,
                          const float* a, const float* b, const float* A_log,
                          const float* dt_bias, float* state, int32_t N, int32_t H_qk,
                          int32_t H_v, int32_t d, float scale, void* o, cudaStream_t s) {
    if (io_dtype == GDN_BF16) {
        if (d == 128)
            return launch_decode_t<__nv_bfloat16, 128>(q, k, v, a, b, A_log, dt_bias, state, N,
                                                       H_qk, H_v, scale, o, s);
        return launch_decode_t<__nv_bfloat16, 64>(q, k, v, a, b, A_log, dt_bias, state, N, H_qk,
                                                  H_v, scale, o, s);
    }
    if (d == 128)
        return launch_decode_t<float, 128>(q, k, v, a, b, A_log, dt_bias, state, N, H_qk, H_v,
                                           scale, o, s);
    return launch_decode_t<float, 64>(q, k, v, a, b, A_log, dt_bias, state, N, H_qk, H_v, scale,
                                      o, s);
}

}  // namespace gdn
