/*
 * rod.h -- C ABI of librod.so: the Rodimus+ token-mixing hot path on one NVIDIA B200 (sm_100a).
 *
 * Two mixers, as the source pages describe them:
 *  - the Rodimus gated linear recurrence, which compresses the history into a fixed-size
 *    per-head state ("Rodimus block" paragraph of the CodeFuse article "ICLR 2025 | Rodimus*:
 *    a hybrid attention mechanism balancing performance and efficiency": a chunkwise-parallel
 *    algorithm for training/prefill, a fixed-size recurrent state at inference):
 *        S_t = diag(g_t) S_{t-1} + k_t^T v_t,      o_t = q_t S_t
 *    with the per-key-channel gates g_t in (0, 1] supplied by the caller;
 *  - SW-SKA, causal sliding-window softmax attention whose key matrix is shared by all heads
 *    while every head keeps its own values (same article, Fig. 4 and the SKA paragraph; window
 *    of the most recent W tokens: setup blog "Rodimus* ... what problem does it solve", §3):
 *        o[h,t] = sum_{j=max(0,t-W+1)}^{t} softmax_j(scale * q[h,t] . k[j]) v[h,j].
 *
 * Conventions shared by every call
 *  - Every tensor pointer is caller-owned DEVICE memory (e.g. from PyTorch), row-major and
 *    contiguous in the layout given per argument, 16-byte aligned. The library never frees or
 *    keeps caller memory and allocates no device memory of its own on these calls.
 *  - Every call is asynchronous on the given CUDA stream (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and returns a status: ROD_OK (0) or a negative ROD_ERR_*.
 *    Argument errors are detected on the host before anything is launched; nothing is
 *    written in that case. No exception crosses this ABI.
 *  - dtype ROD_BF16: q, k, v, o (and the attention caches) are bf16; gates g and recurrent
 *    states are fp32; all arithmetic accumulates in fp32.
 *    dtype ROD_FP32: every tensor is fp32 and every product is an fp32 FMA (no tensor cores).
 *  - Supported head dimensions dk, dv: 16, 32, 64, 128.
 *  - A device-side wait that exceeds its bound (it never should) makes the kernel give up,
 *    leave its outputs unspecified and raise a flag that rod_check() reports as
 *    ROD_ERR_TIMEOUT.
 */
#ifndef ROD_H
#define ROD_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ROD_API __attribute__((visibility("default")))
#else
#define ROD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ----------------------------------------------------------------------- */
#define ROD_OK 0
#define ROD_ERR_NULL (-1)        /* a required pointer is NULL                                 */
#define ROD_ERR_SHAPE (-2)       /* a size is out of range or unsupported                      */
#define ROD_ERR_ALIGN (-3)       /* a pointer is not 16-byte aligned                           */
#define ROD_ERR_DTYPE (-4)       /* dtype is neither ROD_BF16 nor ROD_FP32                     */
#define ROD_ERR_WORKSPACE (-5)   /* workspace missing or smaller than the size query returns   */
#define ROD_ERR_CUDA (-6)        /* a CUDA launch/runtime error; see rod_last_cuda_error()     */
#define ROD_ERR_TIMEOUT (-7)     /* a bounded device-side wait expired (reported by rod_check) */

/* ---- dtypes ------------------------------------------------------------------------------ */
#define ROD_BF16 1
#define ROD_FP32 2

/* Human-readable name of a status code (static string, never NULL). */
ROD_API const char* rod_status_string(int status);

/* The cudaError_t value behind the most recent ROD_ERR_CUDA returned on this host thread
 * (0 if none). */
ROD_API int rod_last_cuda_error(void);

/* Synchronise `stream`, then report ROD_ERR_TIMEOUT if any kernel of this library gave up on
 * a bounded device wait since the last rod_check (and clear that flag), ROD_ERR_CUDA on a
 * CUDA error, else ROD_OK. */
ROD_API int rod_check(void* stream);

/* Version of this ABI (incremented on any incompatible change). */
ROD_API int rod_abi_version(void);

/* Number of kernels this library has launched in this process so far (every entry point
 * counts each kernel it enqueues; host-side counter, no synchronisation). */
ROD_API uint64_t rod_launch_count(void);

/* Diagnostics for the failure-detection path (no counterpart in the source pages). Arms the
 * NEXT rod_gla_prefill call that runs the tensor-core kernels (bf16, dk = dv = 128, chunk 64):
 * its TMA producers issue no copies and every bounded device wait in its kernels gives up
 * after `probes` probes instead of the default 2^22, so the call's consumers find their first
 * input barrier never completes, abort, drain and return. rod_check() then reports
 * ROD_ERR_TIMEOUT; that call's outputs and final state are unspecified, and later calls run
 * normally (the arming is consumed by the one call). Nothing faults, traps or hangs.
 * probes = 0 disarms. Always returns ROD_OK. Not thread-safe against concurrent prefill calls
 * from other host threads (they may consume the arming). */
ROD_API int rod_test_expire_waits(uint32_t probes);

/* ---- gated linear recurrence: chunkwise prefill ------------------------------------------ */
/*
 * Bytes of device workspace rod_gla_prefill needs for these sizes (0 if none). The caller
 * allocates it; its content on entry is irrelevant. Returns 0 for invalid sizes as well.
 */
ROD_API size_t rod_gla_prefill_workspace_size(int B, int H, int T, int dk, int dv, int chunk, int dtype);

/*
 * Prefill of T tokens for B sequences x H heads (CodeFuse article, Rodimus block: the
 * chunkwise-parallel form used for training/prefill; it reaches the same result as the
 * recurrence above up to rounding).
 *   q, k  [B,H,T,dk]   dtype          queries and keys (any input gate pre-multiplied into k)
 *   v     [B,H,T,dv]   dtype          values
 *   g     [B,H,T,dk]   fp32           per-channel decay gates, expected in [0, 1]
 *   state [B,H,dk,dv]  fp32, in/out   initial state on entry (zeros for a fresh sequence),
 *                                     final state S_{T-1} on return
 *   o     [B,H,T,dv]   dtype          outputs o_t = q_t S_t (no scale, no normaliser)
 *   chunk              tokens per chunk: a multiple of 16 in [16, 128]. It changes rounding
 *                      only, never the mathematical result; a T that is not a multiple of
 *                      chunk is handled by masking the tail chunk. Only dtype ROD_BF16 with
 *                      dk = dv = 128 and chunk = 64 runs the chunkwise tensor-core kernels;
 *                      every other combination (all of ROD_FP32, other chunk sizes or head
 *                      dims) runs a sequential-in-time CUDA-core kernel with exact fp32 FMAs,
 *                      one thread per state column: correct, but far slower at long T.
 *   workspace, ws_bytes  at least rod_gla_prefill_workspace_size(...) bytes (may be NULL
 *                      when that size is 0).
 * Calling it twice, on tokens [0,T1) and then [T1,T) with the returned state, equals one
 * call on [0,T) up to rounding (chunked prefill: SALA blog §3.3).
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (B,H < 0, T < 0, dk/dv unsupported, bad chunk),
 * ROD_ERR_ALIGN, ROD_ERR_DTYPE, ROD_ERR_WORKSPACE, ROD_ERR_CUDA. T = 0 or B*H = 0 is a
 * no-op (state unchanged).
 */
ROD_API int rod_gla_prefill(const void* q, const void* k, const void* v, const float* g, float* state,
                    void* o, int B, int H, int T, int dk, int dv, int chunk, int dtype,
                    void* workspace, size_t ws_bytes, void* stream);

/* ---- gated linear recurrence: prefill for callers that cannot allocate ----------------------- */
/*
 * Not a step of the method (the source pages have no counterpart): the same computation as
 * rod_gla_prefill, for callers that cannot allocate device memory per call -- code embedded in
 * a host program that owns the GPU memory pool, plug-ins forbidden to call cudaMalloc or a
 * framework allocator (an allocation may synchronise the device or fail under memory
 * pressure), or paths that must not allocate after start-up. The scratch rod_gla_prefill takes
 * as `workspace` lives instead in one fixed device array inside the library,
 * ROD_GLA_PREFILL_NOALLOC_MAX_SCRATCH bytes, held on every GPU that uses it until the process
 * exits. The call allocates nothing; the caller still passes all inputs and outputs, with the
 * layouts and meaning of rod_gla_prefill.
 *  - The first call made with a given device current looks up the array's device address on
 *    that device; make that first call before any stream capture begins.
 *  - A problem whose rod_gla_prefill_workspace_size exceeds the maximum returns
 *    ROD_ERR_WORKSPACE before anything is launched.
 *  - Every call shares the one array and it keeps the last call's contents; nothing in it needs
 *    to start at zero. Calls that overlap on the GPU (unordered streams, concurrent host
 *    threads) race on it and produce wrong results: serialise them.
 * Other errors: as rod_gla_prefill.
 */
#define ROD_GLA_PREFILL_NOALLOC_MAX_SCRATCH ((size_t)48 << 20)
ROD_API int rod_gla_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                                    float* state, void* o, int B, int H, int T, int dk, int dv,
                                    int chunk, int dtype, void* stream);

/* ---- gated linear recurrence: backward (training path) -------------------------------------- */
/*
 * Gradients of the recurrence of rod_gla_prefill (CodeFuse article, Rodimus block: the
 * chunkwise-parallel algorithm serves training as well as prefill). For the loss gradients
 * dO_t of every output o_t and dstate_final of the final state:
 *   dq_t = S_t dO_t;  dS_t = q_t^T dO_t + diag(g_{t+1}) dS_{t+1} (dS_T from dstate_final);
 *   dk_t = dS_t v_t;  dv_t = dS_t^T k_t;  dg_t[c] = sum_j dS_t[c][j] S_{t-1}[c][j];
 *   dstate0 = diag(g_1) dS_1  (the gradient of the initial state; dstate_final when T = 0).
 *   q, k [B,H,T,dk], v [B,H,T,dv], dO [B,H,T,dv]: dtype;  g [B,H,T,dk] fp32;
 *   state0 [B,H,dk,dv] fp32: the initial state the forward started from;
 *   dstate_final [B,H,dk,dv] fp32, or NULL for no loss on the final state;
 *   outputs dq, dk [B,H,T,dk] and dv [B,H,T,dv] in dtype; dg [B,H,T,dk] and dstate0
 *   [B,H,dk,dv] fp32; workspace of rod_gla_backward_workspace_size bytes (caller-owned).
 * Two routes, chosen by dtype and shape. ROD_BF16 with dk = dv = 128 runs the chunkwise form
 * on the tensor cores in three launches: each chunk's contributions to the state and to its
 * gradient, a scan over chunks (incoming states forward, state gradients backward, both kept in
 * bf16 in the workspace), and one CTA per chunk for dq, dk, dv, dg (bf16 operands, fp32
 * accumulation). Every other case runs on CUDA cores with every product an fp32 FMA (three
 * sweeps over the sequence per (batch, head), states in registers).
 * rod_gla_backward_workspace_size does not depend on dtype: it returns enough for either route.
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE, ROD_ERR_ALIGN, ROD_ERR_DTYPE, ROD_ERR_WORKSPACE,
 * ROD_ERR_CUDA. B*H = 0 is a no-op.
 */
ROD_API size_t rod_gla_backward_workspace_size(int B, int H, int T, int dk, int dv);
ROD_API int rod_gla_backward(const void* q, const void* k, const void* v, const float* g,
                             const float* state0, const void* dO, const float* dstate_final,
                             void* dq, void* dk, void* dv, float* dg, float* dstate0, int B,
                             int H, int T, int dk_dim, int dv_dim, int dtype, void* workspace,
                             size_t ws_bytes, void* stream);

/* ---- gated linear recurrence: one decode step --------------------------------------------- */
/*
 * One token for each of N sequences x H heads, with the fixed-size state updated in place
 * (CodeFuse article, Rodimus block: O(1)-space recurrent inference; SALA blog §3.3: the state
 * stays resident on the GPU and is accumulated in place every step):
 *   S <- diag(g) S + k^T v ;  o = q S   (S after the update)
 *   q, k  [N,H,dk]  dtype;  v [N,H,dv] dtype;  g [N,H,dk] fp32;
 *   state [N,H,dk,dv] fp32, read and overwritten;  o [N,H,dv] dtype.
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE, ROD_ERR_ALIGN, ROD_ERR_DTYPE, ROD_ERR_CUDA.
 * N*H = 0 is a no-op.
 */
ROD_API int rod_gla_decode_step(const void* q, const void* k, const void* v, const float* g,
                        float* state, void* o, int N, int H, int dk, int dv, int dtype,
                        void* stream);

/* ---- SW-SKA: prefill ----------------------------------------------------------------------- */
/*
 * Causal sliding-window attention with one key matrix shared by the H heads:
 *   q [B,H,T,dk] dtype;  k [B,T,dk] dtype (shared);  v [B,H,T,dv] dtype;  o [B,H,T,dv] dtype.
 *   window W >= 1: query t sees keys max(0, t-W+1) .. t (W keys including itself);
 *   scale: multiplies q.k before the softmax; scale <= 0 selects 1/sqrt(dk).
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (window < 1, dims unsupported, H > 64), ROD_ERR_ALIGN,
 * ROD_ERR_DTYPE, ROD_ERR_CUDA. T = 0 or B*H = 0 is a no-op.
 */
ROD_API int rod_swska_prefill(const void* q, const void* k, const void* v, void* o, int B, int H,
                      int T, int dk, int dv, int window, float scale, int dtype, void* stream);

/* ---- SW-SKA: prefill that also keeps each row's log-sum-exp (for the backward) ------------- */
/*
 * rod_swska_prefill (same inputs, output, routes, window and scale rules) that also writes
 *   lse[b,h,t] = log sum_{j in the window of t} exp(scale * q[b,h,t] . k[b,j])   (natural log),
 * lse [B,H,T] fp32, 4-byte aligned, caller-owned. Together with o it is what
 * rod_swska_backward_lse needs, so a training step need not run the forward twice (the
 * statistics the backward uses are the scores' log-sum-exp and D_t = dO_t . o_t).
 * Errors: those of rod_swska_prefill; ROD_ERR_NULL also for a null lse.
 */
ROD_API int rod_swska_prefill_lse(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int B, int H, int T, int dk, int dv, int window, float scale,
                                  int dtype, void* stream);

/* ---- SW-SKA: backward (training path) -------------------------------------------------------- */
/*
 * Gradients of rod_swska_prefill for the loss gradient dO of every output row (same window
 * and scale rules; CodeFuse article, SKA paragraph: the shared K gathers every head's part):
 *   D_t = dO_t . o_t;  dS_tj = p_tj (dO_t . v_j - D_t);  dq_t = scale sum_j dS_tj k_j;
 *   dk_j = scale sum_h sum_t dS_tj q_t;  dv_j = sum_t p_tj dO_t (per head).
 *   q [B,H,T,dk], k [B,T,dk], v [B,H,T,dv], dO [B,H,T,dv]: dtype;  outputs dq, dk, dv in the
 *   layouts of q, k, v and dtype;  workspace of rod_swska_backward_workspace_size bytes
 *   (the row log-sum-exp and D_t, recomputed here from the inputs).
 * Two routes, chosen by dtype and shape: ROD_BF16 with dk = dv = 128 and T >= 128 runs four
 * tcgen05 tensor-core launches (the forward in a statistics mode for the row log-sum-exp and
 * D_t, then query tiles for dq, key tiles for dv and per-group dk partials, and a fixed-order
 * reduction of dk, so the result is deterministic); every other case runs on CUDA cores with
 * fp32 dot products (one warp per query row, then one per key).
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (window < 1, dims unsupported, H > 64), ROD_ERR_ALIGN,
 * ROD_ERR_DTYPE, ROD_ERR_WORKSPACE, ROD_ERR_CUDA. T = 0 or B*H = 0 is a no-op.
 */
ROD_API size_t rod_swska_backward_workspace_size(int B, int H, int T);
ROD_API int rod_swska_backward(const void* q, const void* k, const void* v, const void* dO,
                               void* dq, void* dk, void* dv, int B, int H, int T, int dk_dim,
                               int dv_dim, int window, float scale, int dtype, void* workspace,
                               size_t ws_bytes, void* stream);
/*
 * rod_swska_backward given the forward's output o [B,H,T,dv] (dtype) and lse [B,H,T] fp32 from
 * rod_swska_prefill_lse with the same inputs, window and scale. On the tensor-core route the
 * first launch then reads o, dO and lse (one warp per row: D_t = dO_t . o_t, and the log-sum-exp
 * in the kernels' base-2 form) instead of running the forward again; the other launches, the
 * workspace (rod_swska_backward_workspace_size) and the outputs are those of rod_swska_backward.
 * D_t is taken from the stored (rounded) o, as the pages' plain definition reads it. The
 * CUDA-core route recomputes its statistics and ignores o and lse. An o or lse that does not
 * come from these inputs gives wrong gradients (it is not checked).
 * Errors: those of rod_swska_backward; ROD_ERR_NULL also for a null o or lse.
 */
ROD_API int rod_swska_backward_lse(const void* q, const void* k, const void* v, const void* o,
                                   const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                   int B, int H, int T, int dk_dim, int dv_dim, int window,
                                   float scale, int dtype, void* workspace, size_t ws_bytes,
                                   void* stream);

/* ---- SW-SKA: decode with a ring-buffer window cache --------------------------------------- */
/*
 * One new token per sequence (SALA blog §3.3: a self-made circular buffer holds the rolling
 * window; CodeFuse article: the SKA cache holds one K and per-head V):
 *   1. writes k_new[n] to k_cache[n, pos[n] mod W] and v_new[n,h] to v_cache[n,h,pos[n] mod W];
 *   2. attends q[n,h] over the tokens at positions max(0, pos[n]-W+1) .. pos[n], whose
 *      entries sit in slots p mod W (the caller keeps the cache filled by this same rule).
 *   q [N,H,dk], k_new [N,dk], v_new [N,H,dv]: dtype;  k_cache [N,W,dk], v_cache [N,H,W,dv]:
 *   dtype, updated in place;  pos [N] int64 on the device, read only (the caller advances
 *   it);  o [N,H,dv] dtype.  window W >= 1, scale as for the prefill.
 * A negative pos[n] is not detected on the host (it lives on the device): that sequence's
 * output is set to NaN and its caches are left untouched.
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (H > 64, dims unsupported, window < 1), ROD_ERR_ALIGN,
 * ROD_ERR_DTYPE, ROD_ERR_CUDA. N = 0 is a no-op.
 */
ROD_API int rod_swska_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                     void* v_cache, const int64_t* pos, void* o, int N, int H, int dk, int dv,
                     int window, float scale, int dtype, void* stream);

/* ---- SW-SKA: decode over a paged window cache ---------------------------------------------- */
/*
 * rod_swska_decode with the ring buffer kept in pages (SALA blog §3.3: a paged KV cache split
 * into small blocks that are allocated on demand and evicted by window). The ring's W slots
 * are cut into pages_per_seq pages of page_size slots (W = pages_per_seq * page_size); logical
 * page i of sequence n is physical page block_table[n * pages_per_seq + i] of the pools:
 *   k_pool [P][page_size][dk],  v_pool [P][H][page_size][dv]   (P physical pages), bf16;
 *   ring slot s of sequence n:  K row  k_pool[t][s mod page_size],
 *                               V rows v_pool[t][h][s mod page_size],  t = table entry of s / page_size.
 * The new token is written at slot pos[n] mod W through the same mapping, then attended as in
 * rod_swska_decode (same q, k_new, v_new, pos, o, window, scale).
 *   block_table [N * pages_per_seq] int32 on the device: each entry must name a page inside the
 *   pools, and sequences must not share a page (both are the caller's to keep; they are not
 *   checked, on the host or the device).
 * Supported: dtype ROD_BF16, dk = dv = 128, 1 <= H <= 16, page_size a positive multiple of 8,
 * pages_per_seq <= ROD_MAX_PAGES_PER_SEQ.
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (unsupported shape, window != pages_per_seq *
 * page_size), ROD_ERR_ALIGN (pools, q, k_new, v_new, o, pos: 16 bytes; table: 4 bytes),
 * ROD_ERR_DTYPE, ROD_ERR_CUDA. N = 0 is a no-op.
 */
#define ROD_MAX_PAGES_PER_SEQ 512
ROD_API int rod_swska_decode_paged(const void* q, const void* k_new, const void* v_new, void* k_pool,
                                   void* v_pool, const int32_t* block_table, int page_size,
                                   int pages_per_seq, const int64_t* pos, void* o, int N, int H,
                                   int dk, int dv, int window, float scale, int dtype, void* stream);

/* ---- SW-SKA: prefill -> decode hand-off ----------------------------------------------------- */
/*
 * Fills the decode ring buffers from a prefill's keys and values (SALA blog §3.3: chunked
 * prefill, then decode over a self-managed circular window buffer; CodeFuse article, SKA
 * paragraph: one shared K, per-head V). After a prefill of T tokens every position
 * p in [max(0, T-W), T) is copied to slot p mod W:
 *   k_cache[b, p mod W, :] = k[b, p, :];   v_cache[b, h, p mod W, :] = v[b, h, p, :]
 * so that rod_swska_decode with pos = T attends over exactly the window prefill row T would.
 *   k [B,T,dk], v [B,H,T,dv]: dtype, read;  k_cache [B,W,dk], v_cache [B,H,W,dv]: dtype,
 *   written (slots not named above are left untouched).  window W >= 1.
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (H > 64, dims unsupported, window < 1), ROD_ERR_ALIGN,
 * ROD_ERR_DTYPE, ROD_ERR_CUDA. B = 0 or T = 0 is a no-op.
 */
ROD_API int rod_swska_cache_fill(const void* k, const void* v, void* k_cache, void* v_cache, int B,
                                 int H, int T, int dk, int dv, int window, int dtype, void* stream);

/* ---- SW-SKA: FP8 (E4M3) window cache ------------------------------------------------------- */
/*
 * The ring-buffer decode and the hand-off with the window cache stored in FP8 (SALA blog §4.3:
 * the KV cache in FP8 halves its memory and speeds decode). The pages name FP8 only; this
 * library reads it as the OCP E4M3 format (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, largest finite value 448) with one fp32 scale per cache:
 *   code = the E4M3 value nearest to x / scale (quotient in fp32, ties to the even code,
 *          magnitudes past 448 saturated),   value read = value(code) * scale.
 *
 * rod_swska_decode_fp8: as rod_swska_decode, with k_cache [N,W,dk] and v_cache [N,H,W,dv] of
 * E4M3 codes (one byte each). The new token's k_new / v_new (bf16) are written to slot
 * pos[n] mod W as codes first; attention then reads every window entry, the new one included,
 * from the cache. q, k_new, v_new, o: bf16 in the layouts of rod_swska_decode; k_scale,
 * v_scale > 0 (finite). Only dk = dv = 128 and 1 <= H <= 16.
 * rod_swska_cache_fill_fp8: as rod_swska_cache_fill into E4M3 rings (k, v bf16).
 * A negative pos[n] leaves that sequence's caches untouched and its output NaN.
 * Errors: ROD_ERR_NULL, ROD_ERR_SHAPE (dims or H unsupported, window < 1, a scale not positive
 * and finite), ROD_ERR_ALIGN, ROD_ERR_CUDA. N = 0 (B = 0, T = 0) is a no-op.
 */
ROD_API int rod_swska_decode_fp8(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                 void* v_cache, const int64_t* pos, void* o, int N, int H, int dk,
                                 int dv, int window, float scale, float k_scale, float v_scale,
                                 void* stream);
ROD_API int rod_swska_cache_fill_fp8(const void* k, const void* v, void* k_cache, void* v_cache, int B,
                                     int H, int T, int dk, int dv, int window, float k_scale,
                                     float v_scale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROD_H */
