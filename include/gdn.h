/*
 * gdn.h -- C ABI of the Gated DeltaNet token-mixer library (libgdn.so).
 *
 * The library computes the gated delta rule of the Qwen3.5 linear-attention
 * layers on one NVIDIA B200 (sm_100a):
 *
 *   per V head h, with QK head j = h / (H_v / H_qk):
 *     q_t, k_t <- q_t / ||q_t||, k_t / ||k_t||   (eps 1e-6 inside the root)
 *     g_t      = -exp(A_log[h]) * softplus(a_t + dt_bias[h]),  alpha_t = exp(g_t)
 *     beta_t   = sigmoid(b_t)
 *     S_t      = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t      = S_t (scale * q_t)
 *
 *   "Qwen3.5-MoE-35B-A3B architecture teardown", section 3.3 (the delta rule
 *   and the prefill / decode split), 3.4 (QK heads shared by V heads), 3.5 (QK
 *   L2 norm), 3.7 (the chunkwise prefill in seven steps);
 *   "Qwen3.5 observation notes", sections "DeltaNet", "Gated DeltaNet" and
 *   "Qwen3_5MoeGatedDeltaNet" (gates, decay before the read, the dispatch
 *   between the chunked and the recurrent kernel, initial / final state).
 *
 * Conventions shared by every call:
 *   - Pointers are DEVICE pointers unless stated, 16-byte aligned. The caller
 *     owns every buffer; the library allocates nothing on any call.
 *   - Tensors are dense, row-major, in the shapes given:
 *       q, k        [T, H_qk, d_k]      v, o   [T, H_v, d_v]
 *       a, b        [T, H_v]            A_log, dt_bias  [H_v]
 *       state       [N, H_v, d_v, d_k]  value-major: o = S q, S[i][c] with
 *                                       i a value index and c a key index.
 *                                       (The pages' HF layout is the transpose.)
 *     T is the packed token count; sequence n owns tokens cu_seqlens[n] ..
 *     cu_seqlens[n+1]-1 (cu_seqlens: int32, device, N+1 entries, cu[0] = 0,
 *     non-decreasing, cu[N] = T).
 *   - io_dtype selects the type of q, k, v and o (GDN_BF16 or GDN_FP32). The
 *     gates and the state are always fp32 (the pages' mamba_ssm_dtype float32).
 *   - Supported shapes: d_k = d_v in {64, 128}; H_v a multiple of H_qk.
 *   - `stream` is a cudaStream_t (NULL: the legacy default stream). Every call
 *     is stream-ordered and asynchronous; nothing is synchronised.
 *   - Errors: every call returns a gdn_status. Arguments are checked on the
 *     host before anything is launched; a bad argument launches nothing.
 *     Content errors that only the device can see (bad cu_seqlens, a bounded
 *     wait that ran out) set a device status word that gdn_sync_status()
 *     returns and clears. No call traps, asserts or aborts.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or count       */
    GDN_ERR_UNSUPPORTED = 2, /* a shape or type the library does not implement    */
    GDN_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required        */
    GDN_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, attribute)    */
    GDN_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out                */
    GDN_ERR_BAD_SEQLENS = 6, /* cu_seqlens not non-decreasing / out of range      */
    GDN_ERR_BAD_SLOT = 7,    /* a state / cache slot index >= the pool size       */
    GDN_ERR_BAD_INDEX = 8    /* an index a kernel formed lies outside its buffer  */
                             /* (checked only by libgdn_debug.so, see below)      */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_FP32 = 1 } gdn_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* gdn_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int gdn_version(void);

/*
 * Bytes of device workspace gdn_prefill needs for these sizes. For d = 128 it
 * covers the tensor-core path: the chunk offsets of the sequences and the order
 * in which their chains run (two int32 per sequence, plus one), then per
 * (64-token chunk, V head) an 8-byte ready flag and an 11,520-byte record (the
 * chunk's T diag(beta) and P matrices, lower triangular, in 16-row bands, and
 * per-token factors), i.e. about 180 bytes per token and V head (with one extra
 * chunk per sequence), the first two
 * parts rounded up to 256 bytes; for d = 64 (CUDA-core path) it is the per-token
 * G and beta, fp32 [T, H_v] each. Returns 0 for invalid sizes (and for
 * num_seqs = 0).
 * The workspace needs no initialisation and may hold anything (earlier calls'
 * records and flags, unrelated data): each call publishes its records under a
 * 64-bit number that no earlier call of the process used (a random per-process
 * base with the top bit set, plus a call counter), and a record counts as ready
 * only when its flag equals that number. Stale words of any other origin equal
 * it only by chance (probability 2^-64 per flag).
 */
size_t gdn_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H_qk,
                                  int32_t H_v, int32_t d_k, int32_t d_v);

/*
 * gdn_gates -- the gate prologue ("Qwen3.5 observation notes",
 * "Qwen3_5MoeGatedDeltaNet": beta = sigmoid(b), g = -exp(A_log) *
 * softplus(a + dt_bias); "Qwen3.5-MoE-35B-A3B architecture teardown", 3.7
 * step 3: the cumulative sum of g inside each 64-token chunk).
 *   a, b              [T, H_v] fp32          (in)
 *   A_log, dt_bias    [H_v] fp32             (in)
 *   cu_seqlens        [N+1] int32            (in) chunks restart at each sequence
 *   g_chunk_cumsum    [T, H_v] fp32 or NULL  (out) inclusive cumsum of g per chunk
 *   g                 [T, H_v] fp32 or NULL  (out) the log-decay itself
 *   beta              [T, H_v] fp32 or NULL  (out)
 * g is computed as 0 where softplus(...) is 0, so alpha = 1 there (no NaN),
 * and is clamped below at -128, where alpha = exp(g) is already 0 in fp32; the
 * clamp keeps the in-chunk sums finite when alpha = 0 (g = -inf).
 */
int gdn_gates(const float* a, const float* b, const float* A_log, const float* dt_bias,
              const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens, int32_t H_v,
              float* g_chunk_cumsum, float* g, float* beta, void* stream);

/*
 * gdn_prefill -- the chunked prefill (the pages' chunk_gated_delta_rule with
 * use_qk_l2norm_in_kernel=True; "Qwen3.5-MoE-35B-A3B architecture teardown",
 * 3.7 steps 1-7, chunk size 64). Runs the gate prologue, then the chunk kernel.
 *   q, k, v           io_dtype, shapes above (in)
 *   a, b, A_log, dt_bias  fp32 (in)
 *   initial_state     [N, H_v, d_v, d_k] fp32 or NULL (zeros)          (in)
 *   cu_seqlens        [N+1] int32                                        (in)
 *   scale             multiplier on the normalised query (1.0f = none)
 *   o                 [T, H_v, d_v] io_dtype                              (out)
 *   final_state       [N, H_v, d_v, d_k] fp32 or NULL (not written)      (out)
 *                     may alias initial_state (each state is read before it
 *                     is written, by the same block)
 *   workspace         >= gdn_prefill_workspace_size(...) bytes, 256-byte aligned
 *                     (the tensor-core path keeps its per-chunk intermediates
 *                     there; they are fully rewritten on every call)
 * Empty sequences are allowed: their final state equals their initial state.
 */
int gdn_prefill(const void* q, const void* k, const void* v, int32_t io_dtype,
                const float* a, const float* b, const float* A_log, const float* dt_bias,
                const float* initial_state, const int32_t* cu_seqlens, int32_t num_seqs,
                int64_t total_tokens, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                float scale, void* o, float* final_state, void* workspace,
                size_t workspace_bytes, void* stream);

/*
 * gdn_prefill_ex / gdn_prefill_slots_ex -- gdn_prefill / gdn_prefill_slots with
 * per-call options, for A/B comparison, measurement and tests of the failure
 * paths (the pages have no counterpart). A NULL options pointer, or all fields
 * zero, is exactly gdn_prefill / gdn_prefill_slots. Nothing here is process-wide
 * state: every option applies to this call only.
 *   impl               which implementation runs:
 *     GDN_IMPL_AUTO         tensor cores (tcgen05) for bf16 I/O with d = 128 and at
 *                           most 16 V heads per QK head, the fp32 CUDA-core kernel
 *                           otherwise (fp32 I/O, d = 64). On the tensor-core path,
 *                           with at most half as many (sequence, V head) chains as
 *                           SMs, preparation and chains run overlapped in one
 *                           cooperative launch (with at most a quarter as many,
 *                           each chain is split over two blocks of 64 value rows);
 *                           otherwise as separate launches.
 *     GDN_IMPL_CUDA_CORE    the fp32 CUDA-core kernel for every shape.
 *     GDN_IMPL_TENSOR_CORE  tensor cores only (GDN_ERR_UNSUPPORTED for shapes and
 *                           types they do not cover), scheduled as AUTO.
 *     GDN_IMPL_TENSOR_CORE_SPLIT       tensor cores, always separate launches.
 *     GDN_IMPL_TENSOR_CORE_WHOLE_ROWS  tensor cores, never half-row chain blocks.
 *   fault              GDN_FAULT_NONE, or GDN_FAULT_WITHHOLD_RECORDS: in the
 *                      overlapped launch the preparation publishes no record, so
 *                      every chain's bounded wait for its first record runs out;
 *                      the call then ends with GDN_ERR_TIMEOUT in the device
 *                      status word (outputs undefined) and the context stays
 *                      usable. Nothing faults. Other launches ignore it.
 *                      GDN_FAULT_BAD_INDEX (libgdn_debug.so only; GDN_ERR_UNSUPPORTED
 *                      in libgdn.so): every chain of the tensor-core path passes one
 *                      index just past the end of the record array through its index
 *                      check before its first chunk, and reads nothing there; the
 *                      check records GDN_ERR_BAD_INDEX and its site, and the call
 *                      computes its results as without the option.
 *   wait_limit_cycles  limit of every bounded device-side wait of the tensor-core
 *                      path, in SM clock cycles; 0 = the default (4e9, about 2 s).
 *   timer              NULL, or a timer from gdn_timer_create: CUDA events are
 *                      recorded on `stream` around each kernel the call launches.
 */
enum {
    GDN_IMPL_AUTO = 0,
    GDN_IMPL_CUDA_CORE = 1,
    GDN_IMPL_TENSOR_CORE = 2,
    GDN_IMPL_TENSOR_CORE_SPLIT = 3,
    GDN_IMPL_TENSOR_CORE_WHOLE_ROWS = 4
};
enum { GDN_FAULT_NONE = 0, GDN_FAULT_WITHHOLD_RECORDS = 1, GDN_FAULT_BAD_INDEX = 2 };

typedef struct gdn_timer gdn_timer;

typedef struct {
    int32_t impl;
    int32_t fault;
    int64_t wait_limit_cycles;
    gdn_timer* timer;
} gdn_prefill_options;

int gdn_prefill_ex(const void* q, const void* k, const void* v, int32_t io_dtype,
                   const float* a, const float* b, const float* A_log, const float* dt_bias,
                   const float* initial_state, const int32_t* cu_seqlens, int32_t num_seqs,
                   int64_t total_tokens, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                   float scale, void* o, float* final_state, void* workspace,
                   size_t workspace_bytes, const gdn_prefill_options* options, void* stream);

/*
 * Kernel timing of gdn_prefill_ex -- a measurement aid; the pages have no
 * counterpart. A timer owns 16 CUDA events of the device current at creation (it
 * is the only object of this library that allocates, and only here).
 *   gdn_timer_create      returns a timer, or NULL if the events cannot be made.
 *   gdn_timer_destroy     frees it (NULL is ignored).
 *   gdn_timer_read        waits for the events of the most recent call that used
 *                         the timer and writes the durations of its first
 *                         min(count, max_kernels) kernels, in milliseconds, to ms
 *                         (host array); returns the kernel count (at most 8), or
 *                         -GDN_ERR_INVALID_ARG / -GDN_ERR_CUDA.
 *   gdn_timer_kernel_name name of kernel i of that call ("chunk_offsets", "prep",
 *                         "chain", "fused", "fused_half_rows" on the tensor-core
 *                         path; "gates", "prefill_simt" on the CUDA-core path;
 *                         "conv1d_silu", "rmsnorm_gated" in gdn_mixer_prefill), or
 *                         NULL.
 * A timer may be used by one call at a time.
 */
gdn_timer* gdn_timer_create(void);
void gdn_timer_destroy(gdn_timer* timer);
int gdn_timer_read(gdn_timer* timer, float* ms, int32_t max_kernels);
const char* gdn_timer_kernel_name(const gdn_timer* timer, int32_t i);

/*
 * gdn_decode_step -- one token for each of N sequences, the state updated in
 * place (the pages' recurrent_gated_delta_rule for seq_len == 1; "Qwen3.5
 * observation notes", "Qwen3_5MoeGatedDeltaNet": state *= exp(g), kv_mem,
 * delta = (v - kv_mem) * beta, state += k delta^T, out = read-out with q).
 *   q, k   [N, H_qk, d_k] io_dtype   v [N, H_v, d_v] io_dtype          (in)
 *   a, b   [N, H_v] fp32             A_log, dt_bias [H_v] fp32          (in)
 *   state  [N, H_v, d_v, d_k] fp32                                (in/out)
 *   o      [N, H_v, d_v] io_dtype                                      (out)
 */
int gdn_decode_step(const void* q, const void* k, const void* v, int32_t io_dtype,
                    const float* a, const float* b, const float* A_log, const float* dt_bias,
                    float* state, int32_t num_seqs, int32_t H_qk, int32_t H_v, int32_t d_k,
                    int32_t d_v, float scale, void* o, void* stream);

/*
 * gdn_decode_step_bf16_state -- gdn_decode_step with the state stored in bf16
 * ("Qwen3.5-MoE-35B-A3B architecture teardown", section 9.4: moving the fp32
 * state to bf16 halves its memory; for decode it also halves the bytes moved).
 *   state  [N, H_v, d_v, d_k] bf16, value-major, updated in place      (in/out)
 *   everything else as gdn_decode_step.
 * The state is widened to fp32, updated as in gdn_decode_step and rounded to bf16
 * (round to nearest even) when written back, so each step adds a relative error
 * of up to 2^-9 to the state; the decay keeps the sum of these errors bounded.
 * Callers convert a prefill's fp32 final state to bf16 themselves.
 */
int gdn_decode_step_bf16_state(const void* q, const void* k, const void* v, int32_t io_dtype,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, void* state, int32_t num_seqs,
                               int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                               void* o, void* stream);

/*
 * gdn_decode_slots -- L tokens for each of N sequences whose states live in a pool
 * of cache slots ("Qwen3.5 observation notes", section "Cache": a request keeps
 * one batch index of the cache for its whole life, so a serving loop keeps states
 * in fixed slots; "Qwen3.5-MoE-35B-A3B architecture teardown", section 6.2: an MTP
 * draft is verified by running the main model on several tokens at once).
 *   q, k   [N, L, H_qk, d_k] io_dtype     v [N, L, H_v, d_v] io_dtype     (in)
 *   a, b   [N, L, H_v] fp32               A_log, dt_bias [H_v] fp32        (in)
 *   state_pool   [num_slots, H_v, d_v, d_k] fp32                      (in/out)
 *   state_slots  [N] int32, device, or NULL (sequence n uses slot n; then
 *                num_slots >= N). Slot < 0: a padding entry -- its outputs
 *                are written as zeros and no state is touched. Slot >=
 *                num_slots sets GDN_ERR_BAD_SLOT in the device status word
 *                and that sequence is skipped. Two sequences of one call must
 *                not share a slot (their updates would race).
 *   o      [N, L, H_v, d_v] io_dtype                                      (out)
 *   intermediate_states  [N, L, H_v, d_v, d_k] fp32, or NULL: the state after
 *                every token (entry L-1 equals the new pool state), so a
 *                caller can roll back to the last accepted draft token.   (out)
 * 1 <= L <= 16 (tokens_per_seq). The tokens of a sequence are applied in order,
 * exactly as L calls of gdn_decode_step; the state is read and written once.
 */
int gdn_decode_slots(const void* q, const void* k, const void* v, int32_t io_dtype,
                     const float* a, const float* b, const float* A_log, const float* dt_bias,
                     float* state_pool, const int32_t* state_slots, int32_t num_slots,
                     int32_t num_seqs, int32_t tokens_per_seq, int32_t H_qk, int32_t H_v,
                     int32_t d_k, int32_t d_v, float scale, void* o,
                     float* intermediate_states, void* stream);

/*
 * gdn_prefill_slots -- gdn_prefill with the states in a pool of cache slots, the
 * pool of gdn_decode_slots ("Qwen3.5 observation notes", section "Cache": a request
 * keeps one batch index of the cache for its whole life).
 *   state_pool         [num_slots, H_v, d_v, d_k] fp32                    (in/out)
 *   state_slots        [N] int32, device: sequence n's slot. Its initial state is
 *                      pool[slot] where has_initial_state is NULL or
 *                      has_initial_state[n] != 0 (else zeros, a new request); its
 *                      final state is written to pool[slot] (in place). Slot < 0:
 *                      zeros in, nothing written (outputs still computed). Slot >=
 *                      num_slots: the same, and GDN_ERR_BAD_SLOT in the device
 *                      status word. Two sequences must not share a slot.
 *   has_initial_state  [N] int32, device, or NULL (every sequence continues).
 * Everything else as gdn_prefill (same workspace size).
 */
int gdn_prefill_slots(const void* q, const void* k, const void* v, int32_t io_dtype,
                      const float* a, const float* b, const float* A_log, const float* dt_bias,
                      float* state_pool, const int32_t* state_slots,
                      const int32_t* has_initial_state, int32_t num_slots,
                      const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                      int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale, void* o,
                      void* workspace, size_t workspace_bytes, void* stream);
int gdn_prefill_slots_ex(const void* q, const void* k, const void* v, int32_t io_dtype,
                         const float* a, const float* b, const float* A_log,
                         const float* dt_bias, float* state_pool, const int32_t* state_slots,
                         const int32_t* has_initial_state, int32_t num_slots,
                         const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                         int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                         void* o, void* workspace, size_t workspace_bytes,
                         const gdn_prefill_options* options, void* stream);

/*
 * gdn_prefill_noalloc -- gdn_prefill for callers that cannot allocate device
 * memory. The pages have no counterpart: this is a deployment variant.
 *
 * gdn_prefill asks the caller for a workspace. Some callers cannot call
 * cudaMalloc or any allocator at the point where they run the mixer: a runtime
 * whose device memory is owned by a pool it must not touch, a plugin that is
 * handed only its input and output buffers, code that runs where an allocation
 * would block or synchronise the device. This call takes the same arguments minus
 * the workspace and keeps its scratch (the per-token G and beta) in a fixed
 * array inside the library.
 *   - It always runs the fp32 CUDA-core chunk kernel (the gate kernel, then the
 *     CUDA-core prefill), whatever the shape and type: the tensor-core path needs
 *     a workspace proportional to the tokens (about 180 bytes per token and V
 *     head), which a fixed array cannot hold for useful sizes. The results agree
 *     with gdn_prefill within the same tolerances; for bf16 with d = 128 the call
 *     is much slower (on the 35B-A3B layer shape, T = 4096 with 32 V heads: about
 *     3.5 ms against about 0.12 ms for gdn_prefill).
 *   - Capacity: total_tokens * H_v <= GDN_NOALLOC_MAX_GATE_ELEMS; larger calls
 *     return GDN_ERR_WORKSPACE and launch nothing (use gdn_prefill for them).
 *     The array (8 MiB) is held on every GPU that loads the library until the
 *     process exits.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture. The cached address is not renewed: after cudaDeviceReset
 *     (or anything else that destroys the device's primary context) the library
 *     must be reloaded before this call is used again.
 *   - Every call shares the one array: calls that overlap on the GPU (two
 *     streams, or two host threads on one device) race and give wrong results.
 *     Serialise them (one stream) or use gdn_prefill with separate workspaces.
 *   - Nothing from an earlier call is read: every gate value is rewritten first.
 */
#define GDN_NOALLOC_MAX_GATE_ELEMS 1048576
int gdn_prefill_noalloc(const void* q, const void* k, const void* v, int32_t io_dtype,
                        const float* a, const float* b, const float* A_log,
                        const float* dt_bias, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                        int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                        void* o, float* final_state, void* stream);

/*
 * The steps around the delta rule in the GDN token mixer ("Qwen3.5-MoE-35B-A3B
 * architecture teardown", section 3.3 phase 2 and phase 4, section 3.4 for the
 * conv cache; "Qwen3.5 observation notes", "Qwen3_5MoeGatedDeltaNet": a causal
 * depthwise conv1d with SiLU over the concatenated q/k/v channels, and
 * RMSNormGated on the mixer output).
 *
 * gdn_conv1d_silu -- causal depthwise convolution + SiLU over a packed batch:
 *   y[t][c] = silu(bias[c] + sum_{i<K} weight[c][i] * x[t-(K-1)+i][c])
 * where positions before a sequence's first token come from conv_state_in
 * (zeros when it is NULL): the last tap multiplies the current token.
 *   x               [T, conv_dim] io_dtype                               (in)
 *   weight          [conv_dim, K] fp32 (16-byte aligned)                 (in)
 *   bias            [conv_dim] fp32, or NULL (no bias)                   (in)
 *   conv_state_in   [N, K-1, conv_dim] io_dtype, oldest position first,
 *                   or NULL (zeros)                                      (in)
 *   cu_seqlens      [N+1] int32, device                                  (in)
 *   y               [T, conv_dim] io_dtype; must not be x               (out)
 *   conv_state_out  [N, K-1, conv_dim] io_dtype, or NULL: the K-1 inputs
 *                   ending at each sequence's last token (older cache
 *                   entries where the sequence is shorter than K-1; an
 *                   empty sequence keeps its cache). May be conv_state_in
 *                   (updated in place).                                 (out)
 * K = kernel_size in {2, 3, 4} (the pages' models use 4); conv_dim a multiple
 * of 8. Arithmetic in fp32; y rounded once to io_dtype; the cache holds the
 * inputs unchanged. Bad cu_seqlens contents set GDN_ERR_BAD_SEQLENS in the
 * device status word.
 */
int gdn_conv1d_silu(const void* x, int32_t io_dtype, const float* weight, const float* bias,
                    const void* conv_state_in, const int32_t* cu_seqlens, int32_t num_seqs,
                    int64_t total_tokens, int32_t conv_dim, int32_t kernel_size, void* y,
                    void* conv_state_out, void* stream);

/*
 * gdn_conv1d_silu_decode -- the same convolution for one token of each of N
 * sequences, each sequence's cache slid by one position in place:
 *   x [N, conv_dim] io_dtype (in); y [N, conv_dim] io_dtype (out);
 *   conv_state [num_slots, K-1, conv_dim] io_dtype, a pool of caches (in/out);
 *   cache_slots [N] int32, device, or NULL (sequence n uses entry n; then
 *   num_slots >= N). Slot < 0: a padding entry (y written as zeros, no cache
 *   touched); slot >= num_slots sets GDN_ERR_BAD_SLOT in the device status word
 *   and that sequence is skipped. Two sequences must not share a slot.
 *   weight, bias as above.
 * With identity slots it equals gdn_conv1d_silu on N one-token sequences with
 * conv_state_in = conv_state_out = conv_state.
 */
int gdn_conv1d_silu_decode(const void* x, int32_t io_dtype, const float* weight,
                           const float* bias, void* conv_state, const int32_t* cache_slots,
                           int32_t num_slots, int32_t num_seqs, int32_t conv_dim,
                           int32_t kernel_size, void* y, void* stream);

/*
 * gdn_rmsnorm_gated -- the mixer's output norm, per row of d values:
 *   y[r][:] = o[r][:] / sqrt(mean(o[r][:]^2) + eps) * weight[:] * silu(z[r][:])
 *   o, z   [rows, d] io_dtype (rows = tokens x V heads)                  (in)
 *   weight [d] fp32, 16-byte aligned, shared by all heads                (in)
 *   y      [rows, d] io_dtype; may be o or z                            (out)
 * d in {64, 128}; eps >= 0 (the pages' models use 1e-6). Arithmetic in fp32.
 */
int gdn_rmsnorm_gated(const void* o, const void* z, int32_t io_dtype, const float* weight,
                      float eps, int64_t rows, int32_t d, void* y, void* stream);

/*
 * gdn_mixer_prefill -- the GDN token mixer's core over a packed batch in one call:
 * the causal depthwise conv1d + SiLU over the concatenated q/k/v channels, the gated
 * delta rule, and the gated RMSNorm of its output ("Qwen3.5-MoE-35B-A3B architecture
 * teardown", section 3.3 phases 2-4 and 3.4 for the conv cache; "Qwen3.5 observation
 * notes", "Qwen3_5MoeGatedDeltaNet": causal_conv1d_fn on mixed_qkv, the split into q, k,
 * v, chunk_gated_delta_rule, then self.norm(core_attn_out, z)). It computes
 *   [q | k | v] = gdn_conv1d_silu(x)   (q, k, v rounded to io_dtype)
 *   o           = gdn_prefill(q, k, v, a, b, ...)
 *   y           = gdn_rmsnorm_gated(o, z)
 * with the same conventions as those three calls:
 *   x               [T, conv_dim] io_dtype, conv_dim = (2 H_qk + H_v) d; channels
 *                   q (H_qk heads of d) | k (H_qk heads) | v (H_v heads)     (in)
 *   conv_weight     [conv_dim, K] fp32, conv_bias [conv_dim] fp32 or NULL     (in)
 *   conv_state_in   [N, K-1, conv_dim] io_dtype or NULL (zeros)               (in)
 *   conv_state_out  [N, K-1, conv_dim] io_dtype or NULL; may be conv_state_in (out)
 *   kernel_size     K in {2, 3, 4}
 *   a, b, A_log, dt_bias, initial_state, cu_seqlens, scale: as gdn_prefill
 *   z               [T, H_v, d] io_dtype, the output gate                     (in)
 *   norm_weight     [d] fp32; eps >= 0                                        (in)
 *   y               [T, H_v, d] io_dtype; must not be x or z                  (out)
 *   final_state     [N, H_v, d, d] fp32 or NULL                               (out)
 *   workspace       >= gdn_mixer_prefill_workspace_size(...) bytes, 256-byte aligned:
 *                   the post-conv q | k | v ([T, conv_dim] io_dtype), then the
 *                   prefill's workspace
 *   options         as gdn_prefill_ex, or NULL
 * For bf16 with d = 128 (at most 16 V heads per QK head) there are two schedules:
 *   GDN_IMPL_AUTO (default): the convolution into the workspace, the tensor-core
 *     prefill with its own schedule reading q, k and v there (token stride conv_dim)
 *     and writing o to y, then the norm over y in place -- the faster schedule on
 *     every measured workload, and the same bits as the three calls.
 *   GDN_IMPL_TENSOR_CORE, _SPLIT, _WHOLE_ROWS: the steps fused into the tensor-core
 *     prefill: its preparation stage reads x (with each sequence's K-1 earlier
 *     positions from the conv cache), convolves the q and k channels it needs itself
 *     and writes all post-conv channels once for the chain stage, which applies the
 *     gated norm to each tile of o before it is stored, and writes the conv cache at
 *     the end of each sequence (with many chains the convolution runs as its own kernel
 *     first). The convolution's arithmetic is that of gdn_conv1d_silu (bit for bit);
 *     the norm's sum of squares is taken in another order than gdn_rmsnorm_gated's.
 * For other shapes and types (and with GDN_IMPL_CUDA_CORE) the call runs the convolution,
 * the CUDA-core prefill and the norm one after another on the same buffers.
 */
size_t gdn_mixer_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H_qk,
                                        int32_t H_v, int32_t d_k, int32_t d_v,
                                        int32_t io_dtype);
int gdn_mixer_prefill(const void* x, int32_t io_dtype, const float* conv_weight,
                      const float* conv_bias, const void* conv_state_in, void* conv_state_out,
                      int32_t kernel_size, const float* a, const float* b, const float* A_log,
                      const float* dt_bias, const float* initial_state,
                      const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                      int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, float scale,
                      const void* z, const float* norm_weight, float eps, void* y,
                      float* final_state, void* workspace, size_t workspace_bytes,
                      const gdn_prefill_options* options, void* stream);

/*
 * Synchronise `stream`, then return and clear the device status word of the
 * current device (GDN_OK, GDN_ERR_BAD_SEQLENS, GDN_ERR_BAD_SLOT, GDN_ERR_TIMEOUT or,
 * in libgdn_debug.so, GDN_ERR_BAD_INDEX), or GDN_ERR_CUDA if the synchronisation
 * itself failed.
 */
int gdn_sync_status(void* stream);

/*
 * The debug build. `python -m linear_attention_sequence_delta_b200.build --debug`
 * builds libgdn_debug.so: the same ABI, in which the kernels of the tensor-core
 * prefill (chunk offsets, preparation, chains, the overlapped launch, with the fused
 * convolution and norm) check each global-memory index they form against the extent
 * of its buffer before the access (the decode kernels' only index taken from data, the
 * state slot, is checked in every build: GDN_ERR_BAD_SLOT). An index outside
 * records GDN_ERR_BAD_INDEX in the device status word and the source line of the
 * first failed check in a second device word, and the access is skipped (a load
 * reads zeros): nothing faults or traps. In libgdn.so the checks are compiled out.
 * Tensor-memory-accelerator copies are not checked: the hardware bounds their
 * coordinates itself (reads past a tensor's end fill zeros, writes there are dropped).
 *   gdn_debug_build           1 in libgdn_debug.so, 0 in libgdn.so; touches no GPU.
 *   gdn_debug_bad_index_site  synchronises `stream`, then returns and clears the
 *                             source line of the first failed index check on the
 *                             current device since the last call (0: none), or
 *                             -GDN_ERR_CUDA if the synchronisation failed.
 */
int gdn_debug_build(void);
int gdn_debug_bad_index_site(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
