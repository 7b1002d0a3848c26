/*
 * llama_block.h — C ABI of a B200 (sm_100a) LLaMA pre-norm decoder block.
 *
 * The block is the pre-norm decoder layer of the "LMDrive 大语言模型（LLM）核心推理单元"
 * page (§2.5 LlamaDecoderLayer) and of chapter 02 of "LLM 核心机制交互讲义":
 *
 *   X'  = X  + o_proj( causal_softmax( RoPE(Q) RoPE(K)^T / sqrt(d_h) ) V ),
 *              with Q, K, V projected from h = RMSNorm(X; g_attn)
 *   X'' = X' + down_proj( SiLU(gate_proj(h2)) * up_proj(h2) ),  h2 = RMSNorm(X'; g_mlp)
 *
 * with grouped-query attention (query head h reads KV head h / (n_heads/n_kv_heads),
 * the repeat_kv grouping of §2.3) and a KV cache for decode (chapter 04 of the
 * mechanics page: the cache holds keys after RoPE; a decode step at cache length L
 * rotates its query and key at position L and appends k, v at index L).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *    densely packed, in the handle's (or the call's) dtype: LB_F32 = float,
 *    LB_BF16 = bfloat16 (storage) with fp32 accumulation. There is no host path.
 *  - Weights use the nn.Linear layout [out_features, in_features].
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Work is
 *    enqueued asynchronously; the call returns after the enqueue.
 *  - Argument errors are detected on the host before anything is enqueued and
 *    return LB_ERR_INVALID_ARG / LB_ERR_UNSUPPORTED / LB_ERR_CACHE_FULL; the
 *    reason is available from llama_block_last_error() (thread-local string).
 *  - Device-side waits are bounded: a wait that runs out latches an error word on
 *    the device instead of hanging; llama_block_sync_status() reads it.
 *  - Restrictions: head_dim in {64, 128}; n_kv_heads divides n_heads (any
 *    quotient); n_heads * head_dim and d are multiples of 64 for LB_BF16; y must
 *    not alias x.
 *  - A handle is not thread-safe: do not call it concurrently from several threads.
 */
#ifndef LLAMA_BLOCK_H
#define LLAMA_BLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LB_OK = 0,
    LB_ERR_INVALID_ARG = 1,  /* null pointer, non-positive or inconsistent size */
    LB_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head_dim 96) */
    LB_ERR_CUDA = 3,         /* a CUDA runtime call failed (message in last_error) */
    LB_ERR_OOM = 4,          /* device allocation failed */
    LB_ERR_CACHE_FULL = 5,   /* a sequence would grow beyond t_max */
    LB_ERR_TIMEOUT = 6,      /* a bounded device wait ran out (see sync_status) */
    LB_ERR_NO_WEIGHTS = 7    /* prefill/decode before llama_block_set_weights */
} lb_status;

typedef enum { LB_F32 = 0, LB_BF16 = 1 } lb_dtype;

typedef struct llama_block llama_block; /* opaque, library-owned */

/* Create a block handle (LMDrive page §2.3–2.5: hidden_size d, num_attention_heads,
 * num_key_value_heads, head_dim, intermediate_size f; RMSNorm eps §2.1; RoPE base
 * §2.2). `max_pos` sizes the RoPE cos/sin table (positions 0 .. max_pos-1), which
 * the library builds in fp64 on the host. Allocates library-owned device memory
 * (packed weights, RoPE table, error word) on the current device; every later call on
 * the handle (and on a llama_stack) runs on that device whatever device is current,
 * and leaves the caller's current device as it was. Its buffers and stream arguments
 * must belong to that device.
 * Returns LB_ERR_INVALID_ARG for non-positive sizes or a null `out`,
 * LB_ERR_UNSUPPORTED for head_dim not in {64,128} or n_heads not a multiple of
 * n_kv_heads. */
lb_status llama_block_create(int d, int n_heads, int n_kv_heads, int head_dim, int f,
                             float eps, float rope_base, lb_dtype dtype, int max_pos,
                             llama_block** out);

/* Copy and pack the block weights (device pointers, nn.Linear [out,in] layout,
 * handle dtype): wq [H*dh, d], wk/wv [Hkv*dh, d], wo [d, H*dh], w_gate/w_up [f, d],
 * w_down [d, f], g_attn/g_mlp [d] (input_layernorm / post_attention_layernorm
 * weights). The library keeps its own packed copies (fused Q|K|V rows; gate/up
 * rows interleaved in blocks of 128), so the caller may free its buffers once
 * `stream` has passed this call. */
lb_status llama_block_set_weights(llama_block* blk, const void* wq, const void* wk,
                                  const void* wv, const void* wo, const void* w_gate,
                                  const void* w_up, const void* w_down,
                                  const void* g_attn, const void* g_mlp, void* stream);

/* Weight-only INT8 for decode ("深入解析Llama MLP模块" page §6.4: INT8 weights reduce the
 * inference memory of the MLP; a decode step streams every weight once). enable = 1:
 * the handle quantizes its packed projection weights per output row (s = max|w|/127,
 * q = rint(w/s) in [-127, 127], decided in fp32) into library-owned INT8 copies, and
 * llama_block_decode with B <= 32 then reads those (half the weight bytes), applying
 * s in the GEMM epilogue; prefill keeps the bf16 weights. Later set_weights calls
 * re-quantize. enable = 0 frees the copies. LB_BF16 handles only; needs weights
 * (LB_ERR_NO_WEIGHTS) and every K dimension a multiple of 64 (LB_ERR_UNSUPPORTED). */
lb_status llama_block_quantize_decode_weights(llama_block* blk, int enable, void* stream);

/* Dynamic NTK scaling of the rotary embedding (LMDrive page §2.2: the rotary module
 * "supports dynamic NTK scaling" to extend the maximum sequence length; the pages give
 * no formula). With original_max_pos = L0 > 0 and factor >= 1, a later prefill, extend
 * or decode call whose longest sequence reaches L > L0 tokens rotates the Q and K of
 * its new tokens with the base
 *     base' = rope_base * (factor * L / L0 - (factor - 1)) ^ (head_dim / (head_dim - 2)),
 * calls with L <= L0 with rope_base; keys already in the cache keep the rotation they
 * were stored with. The handle rewrites the RoPE table rows a call reads (fp64 angles,
 * one extra kernel on the call's stream). original_max_pos = 0 turns it off and
 * restores the plain table on `stream`. LB_ERR_INVALID_ARG for a NULL handle,
 * original_max_pos < 0, or factor < 1 (or not finite) when turning it on. */
lb_status llama_block_set_rope_dynamic_ntk(llama_block* blk, float factor, int original_max_pos,
                                           void* stream);

/* Preallocate the workspace for up to `max_tokens` prefill rows (B*T) and
 * `max_batch` decode sequences, so that later calls allocate nothing (needed
 * before capturing calls in a CUDA graph). Optional: calls grow the workspace
 * on demand otherwise. */
lb_status llama_block_reserve(llama_block* blk, int max_tokens, int max_batch);

/* Prefill (LMDrive page §2.5 forward, positions 0..T-1 for every sequence).
 * x, y: [B, T, d]. k_cache, v_cache: [B, n_kv_heads, t_max, head_dim] (caller-owned);
 * K (after RoPE) and V of positions 0..T-1 are written to indices 0..T-1.
 * cache_len: device int32 [B], set to T. T <= t_max and T <= max_pos required
 * (else LB_ERR_CACHE_FULL). The host-side length mirror is set to T. */
lb_status llama_block_prefill(llama_block* blk, const void* x, void* y, int B, int T,
                              void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                              void* stream);

/* One decode step for B sequences with one new token each (mechanics page,
 * chapter 04 KV-cache equation). x, y: [B, 1, d]. The new token of sequence b sits
 * at position L_b = cache_len[b]; its rotated k and its v are written to cache
 * index L_b, the query attends keys 0..L_b, and cache_len[b] becomes L_b + 1.
 * The host mirror of the lengths (set by prefill or llama_block_set_lengths) is
 * checked first: L_b + 1 > t_max or L_b >= max_pos returns LB_ERR_CACHE_FULL. */
lb_status llama_block_decode(llama_block* blk, const void* x, void* y, int B,
                             void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                             void* stream);

/* Chunked prefill into an existing cache (mechanics page, chapter 04: the prefill ->
 * decode handoff; positions follow the cache length). Every sequence must hold the
 * same number L of cached tokens (host mirror: prefill, extend, decode or
 * llama_block_set_lengths), else LB_ERR_UNSUPPORTED. The T new tokens x [B, T, d]
 * sit at positions L .. L+T-1: their rotated keys and values are written to cache
 * indices L .. L+T-1, token i attends to keys 0 .. L+i, y [B, T, d] is the block
 * output, and cache_len becomes L + T. L + T <= t_max and <= max_pos required (else
 * LB_ERR_CACHE_FULL). With L = 0 this is llama_block_prefill. */
lb_status llama_block_extend(llama_block* blk, const void* x, void* y, int B, int T,
                             void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                             void* stream);

/* Tell the handle the current cache lengths (host array of B entries) when the
 * caller filled the cache itself; the device cache_len array stays the caller's
 * to set. */
lb_status llama_block_set_lengths(llama_block* blk, const int32_t* lens_host, int B);

/* KV-cache bytes of one block (mechanics page, chapter 04 memory accounting with
 * L = 1): 2 * B * t_max * n_kv_heads * head_dim * sizeof(dtype). Host-only; 0 for
 * invalid arguments. */
size_t llama_block_kv_cache_bytes(int B, int n_kv_heads, int head_dim, int t_max,
                                  lb_dtype dtype);

/* Synchronise `stream`, read and clear the device error word (of the handle, or,
 * when blk is NULL, the words of the current device's standalone entry points:
 * the one they share and the one of decode_attn_static_scratch; with blk NULL
 * this call allocates nothing). Returns LB_OK, LB_ERR_TIMEOUT
 * (a bounded wait ran out), LB_ERR_CACHE_FULL (a device-side bounds guard fired:
 * a cache index or RoPE position out of range; the write was skipped) or
 * LB_ERR_CUDA; details in last_error. */
lb_status llama_block_sync_status(llama_block* blk, void* stream);

/* Free the handle and everything it owns (synchronises the device first). */
void llama_block_destroy(llama_block* blk);

/* Thread-local description of the last error (never NULL). */
const char* llama_block_last_error(void);

/* Profiling aid: when enabled, prefill and decode bracket each of their stages
 * (one or two kernel launches) with CUDA events recorded on the caller's stream.
 * Off by default; events are created on first enable. */
lb_status llama_block_enable_timing(llama_block* blk, int enable);

/* Device durations (ms) of the stages of the last prefill/decode call with timing
 * enabled; waits for that call's events. Writes up to max_stages values into ms
 * (may be NULL) and the stage count into *n_stages. */
lb_status llama_block_stage_times(llama_block* blk, float* ms, int max_stages, int* n_stages);

/* Name of stage i of the last prefill/decode call ("" when out of range). */
const char* llama_block_stage_name(const llama_block* blk, int i);

/* Number of kernels this handle has launched since it was created. */
unsigned long long llama_block_launch_count(const llama_block* blk);

/* Self-test of the bounded-wait machinery: launch one kernel that waits on a
 * device barrier that nothing completes, with a budget of `budget_ns`
 * nanoseconds. The kernel gives up, latches the standalone error word and exits;
 * llama_block_sync_status(NULL, stream) then returns LB_ERR_TIMEOUT. No GPU fault
 * or hang is involved. */
lb_status llama_block_selftest_timeout(long long budget_ns, void* stream);

/* ---------------- stack of blocks ---------------- */

/* A stack of n_layers decoder blocks with the same shape (mechanics page, chapter 02:
 * the block repeated "x L"; LMDrive page §1: 32 decoder layers), each with its own
 * weights and KV cache; layer l's output feeds layer l+1. The stack owns its layer
 * handles, two activation buffers [B*T, d] and per-layer length arrays; the caller
 * owns the caches. */
typedef struct llama_stack llama_stack;

/* Create a stack of n_layers blocks, each as llama_block_create(d, n_heads, n_kv_heads,
 * head_dim, f, eps, rope_base, dtype, max_pos) on the current device; weights are set per
 * layer through llama_stack_layer. Returns LB_ERR_INVALID_ARG for n_layers <= 0 or a null
 * `out`, and any error of a layer's creation (the layers made so far are freed). */
lb_status llama_stack_create(int n_layers, int d, int n_heads, int n_kv_heads, int head_dim,
                             int f, float eps, float rope_base, lb_dtype dtype, int max_pos,
                             llama_stack** out);

/* The block handle of layer `layer` (for llama_block_set_weights); NULL when out of
 * range. Owned by the stack. */
llama_block* llama_stack_layer(llama_stack* st, int layer);

/* Prefill / chunked prefill / one decode step through every layer. k_caches and
 * v_caches are HOST arrays of n_layers device pointers, each cache
 * [B, n_kv_heads, t_max, head_dim]. cache_len (device int32 [B]) is read at the
 * start and holds the new lengths at the end, as for a single block. x, y as for
 * the block calls (T = 1 for decode). */
lb_status llama_stack_prefill(llama_stack* st, const void* x, void* y, int B, int T,
                              void* const* k_caches, void* const* v_caches, int t_max,
                              int32_t* cache_len, void* stream);
lb_status llama_stack_extend(llama_stack* st, const void* x, void* y, int B, int T,
                             void* const* k_caches, void* const* v_caches, int t_max,
                             int32_t* cache_len, void* stream);
lb_status llama_stack_decode(llama_stack* st, const void* x, void* y, int B,
                             void* const* k_caches, void* const* v_caches, int t_max,
                             int32_t* cache_len, void* stream);

/* Set the host length mirror of every layer (see llama_block_set_lengths). */
lb_status llama_stack_set_lengths(llama_stack* st, const int32_t* lens_host, int B);

/* Free the stack, its layers and its buffers. */
void llama_stack_destroy(llama_stack* st);

/* ---------------- tensor parallelism ---------------- */

/* "深入解析Llama MLP模块" page §6.3: the block split over W ranks, Megatron style: rank r
 * holds query heads [r H/W, (r+1) H/W), KV heads [r H_kv/W, ..), intermediate columns
 * [r f/W, ..); Q/K/V and gate/up are split by output rows, o_proj and down by input
 * columns, and an all-reduce over ranks completes each branch. A shard is an ordinary
 * handle created with (d, H/W, H_kv/W, head_dim, f/W) and given its weight slices (the
 * RMSNorm gains whole); its KV cache holds its KV heads. bf16 handles only
 * (LB_ERR_UNSUPPORTED otherwise); LB_ERR_NO_WEIGHTS before set_weights. One layer:
 *   tp_attn_*(x) -> o_part     all-reduce(o_part) -> o_sum
 *   tp_mlp(x, o_sum) -> x1, m_part     all-reduce(m_part) -> m_sum
 *   tp_add(x1, m_sum) -> y     (y = x + o + m, the block output)
 * The all-reduce is the caller's (e.g. NCCL). Partials are bf16 [rows, d]. */

/* Attention branch of a fresh prefill (T tokens per sequence at positions 0..T-1): the
 * rank's Q/K/V with RoPE (its K/V written to cache positions [0, T)), causal attention of
 * its heads, and o_part [B, T, d] = O_rank W_o[:, rank]^T (no residual). Sets cache_len
 * and the handle's lengths to T. Errors as llama_block_prefill. */
lb_status llama_block_tp_attn_prefill(llama_block* shard, const void* x, void* o_part, int B, int T,
                                      void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                                      void* stream);

/* Attention branch of one decode step (one token per sequence at position cache_len[b],
 * its K/V appended there): o_part [B, 1, d] as above; cache_len += 1. Uses the INT8
 * weights when they are enabled. Errors as llama_block_decode. */
lb_status llama_block_tp_attn_decode(llama_block* shard, const void* x, void* o_part, int B,
                                     void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                                     void* stream);

/* MLP branch for M token rows: x1 = x + o_sum (written, [M, d]), then m_part [M, d] =
 * (SiLU(RMSNorm(x1) W_gate[rank]^T) * RMSNorm(x1) W_up[rank]^T) W_down[:, rank]^T. x1
 * and m_part must not alias the inputs (LB_ERR_INVALID_ARG). */
lb_status llama_block_tp_mlp(llama_block* shard, const void* x, const void* o_sum, void* x1,
                             void* m_part, int M, void* stream);

/* out = a + b, rows x d elements of `dtype` (d % 8 == 0), fp32 add with one rounding: the
 * residual stream plus an all-reduced branch. */
lb_status llama_block_tp_add(const void* a, const void* b, void* out, int rows, int d, lb_dtype dtype,
                             void* stream);

/* ---------------- standalone entry points (testing) ---------------- */


/* RMSNorm (LMDrive page §2.1; mechanics page §02.3): y = g * x / sqrt(mean(x^2) + eps)
 * over the last axis, fp32 accumulation, one rounding. x, y: [rows, d]; g: [d].
 * rows == 0 is a no-op (pointers may then be NULL). */
lb_status rmsnorm(const void* x, const void* g, void* y, int rows, int d, float eps,
                  lb_dtype dtype, void* stream);

/* RoPE in place (LMDrive page §2.2, half-split rotate_half pairing):
 * x: [B, n_heads, T, head_dim]; pos: device int32 [B, T] positions (>= 0).
 * Angles pos * base^(-2i/head_dim) are formed in fp64 on the device. */
lb_status rope_apply(void* x, const int32_t* pos, int B, int T, int n_heads, int head_dim,
                     float base, lb_dtype dtype, void* stream);

/* Causal softmax attention with GQA (LMDrive page §2.3; mechanics page §02.1).
 * q: [B, n_heads, Tq, head_dim]; k, v: [B, n_kv_heads, k_stride_T, head_dim] of which
 * the first Tk rows are used; query row i sits at position Tk - Tq + i and attends
 * keys 0 .. Tk - Tq + i. o: [B, Tq, n_heads * head_dim] (the layout o_proj reads).
 * Scores are scaled by 1/sqrt(head_dim). Requires 1 <= Tq <= Tk <= k_stride_T. */
lb_status causal_attn(const void* q, const void* k, const void* v, void* o, int B, int Tq,
                      int Tk, int n_heads, int n_kv_heads, int head_dim, int k_stride_T,
                      lb_dtype dtype, void* stream);

/* SwiGLU MLP without residual (LMDrive page §2.4; Llama-MLP page §4.2):
 * y = down( SiLU(h gate^T) * (h up^T) ). h, y: [M, d]; w_gate, w_up: [f, d];
 * w_down: [d, f]. Packs the gate/up weights into a temporary device buffer per
 * call (allocates and frees it). */
lb_status swiglu_mlp(const void* h, const void* w_gate, const void* w_up,
                     const void* w_down, void* y, int M, int d, int f, lb_dtype dtype,
                     void* stream);

/* Decode attention that allocates nothing, for callers that may not call
 * cudaMalloc (or any allocator) while they run: code inside a region whose
 * device memory is budgeted up front, a host that hands all device memory to its
 * own pool, or a launch path that must not synchronise the device the way an
 * allocation or free can. The pages have no counterpart; it is an operational
 * variant of the split-KV decode attention that llama_block_decode runs.
 *
 * Computes, for each sequence b and query head h, the attention of the single
 * query q[b][h] (at position kv_len[b]) over keys 0..kv_len[b]:
 *   q: [B, n_heads, head_dim]; k, v: [B, n_kv_heads, k_stride_T, head_dim],
 *   16-byte aligned; kv_len: device int32 [B], 0 <= kv_len[b] < k_stride_T;
 *   o: [B, n_heads * head_dim]; all bf16 except kv_len. The caller passes inputs
 *   and outputs; the split-KV partials go to a fixed array inside the library.
 * Limit: B * n_heads * ceil(k_stride_T / 512) * (head_dim + 2) <= 6 * 2^20 floats
 * (24 MiB); larger calls return LB_ERR_INVALID_ARG before anything is launched,
 * as do misaligned k or v.
 * Every GPU that loads the library holds that array until the process exits.
 * The first call on a device looks up the array's device address on that
 * device; make that first call before any stream capture. The array belongs to
 * the process's context on that device, so all calls of one process on one
 * device share it and it keeps the last call's contents: calls that may overlap
 * on that GPU (several streams, or several host threads) race, so serialise
 * them. Separate processes each have their own copy.
 * Errors found on the device (a kv_len[b] outside [0, k_stride_T), or a bounded
 * wait that ran out) set a device word private to this entry point and leave
 * that call's output undefined; llama_block_sync_status(NULL, stream) reads and
 * clears it (LB_ERR_CACHE_FULL or LB_ERR_TIMEOUT), allocating nothing. */
lb_status decode_attn_static_scratch(const void* q, const void* k, const void* v, void* o,
                                     const int32_t* kv_len, int B, int n_heads, int n_kv_heads,
                                     int head_dim, int k_stride_T, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_BLOCK_H */
