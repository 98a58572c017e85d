/*
 * kda.h -- C ABI of libkda.so: KDA (fine-grained gated delta rule) chunkwise
 * prefill (dense or packed batches, optional chunk-parallel segment scan), its
 * backward pass, and the single-token decode step on NVIDIA B200 (sm_100a);
 * the delta-rule and gated-linear-attention variants run through the same
 * calls.
 *
 * The operation (pages: "Decoding Hybrid Attention Architectures", section
 * 3.4 and its variant table; "Technical Analysis ... Novel Hybrid Linear
 * Attention", section 2 item 4), per sequence and head, token by token:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with state S in R^{dk x dv} (row i = key channel i), alpha_t = exp(log_alpha_t)
 * taken elementwise (no activation is applied to log_alpha), and no scaling of q.
 * The prefill computes this with the chunkwise-parallel form of section 4 of
 * the first page (intra-chunk lower-triangular products, inter-chunk state
 * passing, precomputed U and W); the decode step is the update for one token
 * ("Decoding Hybrid Attention Architectures", sections 1 and 5: constant
 * state, cost independent of context length).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, row-major and contiguous, with
 *     the base address aligned to 16 bytes. The caller owns every buffer.
 *   - dtype selects the element type of q, k, v, log_alpha, beta and o:
 *     KDA_F32 (float) or KDA_BF16 (__nv_bfloat16). States are always float.
 *   - Nothing is allocated and nothing is synchronised: all work is enqueued
 *     on `stream` (a cudaStream_t; NULL = the legacy default stream) and the
 *     call returns once it is enqueued.
 *   - Arguments are validated before anything is launched. A call that
 *     returns anything but KDA_OK has launched nothing and written nothing,
 *     except KDA_ERR_CUDA, which reports a launch failure.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, workspace too small */
    KDA_ERR_UNSUPPORTED = 2, /* valid but not implemented (head size, chunk size, dtype) */
    KDA_ERR_CUDA = 3,        /* a CUDA launch or query failed; see cudaGetLastError */
    KDA_ERR_TIMEOUT = 4      /* a bounded device-side wait expired (kda_workspace_status, kda_noalloc_status) */
} kda_status_t;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/* Which prefill kernels to run. AUTO picks the fused tensor-core kernel when
 * it supports the shape (bf16, dk = dv = 128, chunk = 64) and the SIMT fp32
 * kernel otherwise; for a dense batch with few heads and a long T it adds the
 * chunk-parallel segment scan when that shortens the run.
 *
 * KDA_ALGO_TC_SCAN: the tensor-core kernel with the segment scan whenever T
 * spans at least 3 chunks (else plain KDA_ALGO_TC); dense batches only
 * (KDA_ERR_UNSUPPORTED for packed sequences). The update is affine in the
 * state ("Decoding Hybrid Attention Architectures" section 3.4; the chunk
 * form of section 4 passes the state between chunks the same way), so each
 * segment of a sequence maps its entry state S_in to M S_in + C. Segment 0
 * and the maps (M, C) of the middle segments are computed in parallel, an
 * fp32 scan chains the entry states, and segments 1..P-1 are then run in
 * parallel from them. Work grows by about half; the sequential depth drops
 * from T to about 2T/P tokens. The workspace holds the maps and entry states
 * (B*H*(3P-5) fp32 [dk][dv] matrices; see kda_chunk_fwd_workspace_size). */
typedef enum { KDA_ALGO_AUTO = 0, KDA_ALGO_SIMT = 1, KDA_ALGO_TC = 2, KDA_ALGO_TC_SCAN = 3 } kda_algo_t;

/* The variant table of "Decoding Hybrid Attention Architectures" (section
 * 3.4, with sections 3.1-3.3 and the per-dimension gated linear attention it
 * names) as two switches of the same kernels:
 *   erase = 1: S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *   erase = 0: S_t =                        Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *   gate: how a_t = exp(log_alpha) is given (below).
 * (erase, gate) = (1, CHANNEL) is KDA, (1, SCALAR) the scalar gated delta
 * rule, (1, NONE) the delta rule, (0, CHANNEL) per-dimension gated linear
 * attention, (0, NONE) with beta = 1 plain linear attention. */
typedef enum {
    KDA_GATE_CHANNEL = 0, /* log_alpha [B, T, H, dk]: one decay per key channel      */
    KDA_GATE_SCALAR = 1,  /* log_alpha [B, T, H]: one decay per token and head        */
    KDA_GATE_NONE = 2     /* no decay (a_t = 1); log_alpha is not read and may be NULL */
} kda_gate_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status_t status);

/*
 * Bytes of device workspace kda_chunk_fwd_ex needs for this shape and
 * algorithm (0 on invalid arguments). The workspace is scratch owned by the
 * caller, at least 256-byte aligned; its contents need not be initialised and
 * are overwritten by every call. Two calls in flight at once must not share
 * a workspace.
 */
size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, kda_dtype_t dtype,
                                    kda_algo_t algo);

/*
 * Chunkwise prefill: kda_chunk_fwd(q, k, v, log_alpha, beta, S0 -> o, S_T).
 *
 *   q, k, log_alpha : [B, T, H, dk]   dtype
 *   v               : [B, T, H, dv]   dtype
 *   beta            : [B, T, H]       dtype, the write strength in (0, 1]
 *   S0              : [B, H, dk, dv]  float, initial state; NULL means zero
 *   o               : [B, T, H, dv]   dtype, written
 *   S_T             : [B, H, dk, dv]  float, final state; NULL means not written
 *                                     (may equal S0: read fully before written)
 *   chunk           : tokens per chunk, one of 16, 32, 64 (64 is the tuned size)
 *   dk, dv          : 64 or 128, dk == dv
 *   T               : any T >= 0; a ragged last chunk is handled exactly
 *                     (as if padded with k = q = v = 0, beta = 0, log_alpha = 0)
 *   workspace       : device scratch of at least
 *                     kda_chunk_fwd_workspace_size(...) bytes (may be NULL when
 *                     that size is 0)
 *
 * Numerics: state and accumulation in fp32. With dtype KDA_F32 and the SIMT
 * algorithm every product is fp32. The tensor-core algorithm rounds MMA
 * operands (decay-scaled keys and queries, the UT inverse, W, the state copy
 * that feeds the next chunk) to bf16 and accumulates in fp32. It factors the
 * decay e^{G_r - G_s} of a chunk through a reference point: the chunk's start
 * while the chunk's decay stays within 80 (in natural-log units), its middle
 * (G_last / 2) up to 160, and exact per-pair exponentials beyond that (slower,
 * but finite for any decay).
 * Returns KDA_OK once enqueued.
 */
kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                           const void *beta, const float *S0, void *o, float *S_T, int B, int T, int H,
                           int dk, int dv, int chunk, kda_dtype_t dtype, void *workspace,
                           size_t workspace_bytes, void *stream);

/* kda_chunk_fwd with an explicit algorithm. KDA_ALGO_TC returns
 * KDA_ERR_UNSUPPORTED for shapes it does not cover. */
kda_status_t kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const void *log_alpha,
                              const void *beta, const float *S0, void *o, float *S_T, int B, int T, int H,
                              int dk, int dv, int chunk, kda_dtype_t dtype, void *workspace,
                              size_t workspace_bytes, kda_algo_t algo, void *stream);

/* kda_chunk_fwd_ex for any variant of the table above. With gate
 * KDA_GATE_SCALAR, log_alpha is [B, T, H]; with KDA_GATE_NONE it may be NULL.
 * erase must be 0 or 1 (else KDA_ERR_INVALID_ARG). Every algorithm supports
 * every variant; the workspace size does not depend on the variant. */
kda_status_t kda_chunk_fwd_v(const void *q, const void *k, const void *v, const void *log_alpha,
                             const void *beta, const float *S0, void *o, float *S_T, int B, int T, int H,
                             int dk, int dv, int chunk, kda_dtype_t dtype, int erase, kda_gate_t gate,
                             void *workspace, size_t workspace_bytes, kda_algo_t algo, void *stream);

/*
 * Packed variable-length sequences (serving: many requests of different
 * lengths in one call; "Decoding Hybrid Attention Architectures", section 5,
 * inference side: fixed-size state per request under high concurrency). The
 * operation per sequence is the one of kda_chunk_fwd_v. N sequences, their
 * tokens packed back to back:
 *   q, k            : [total_T, H, dk]   dtype
 *   log_alpha       : [total_T, H, dk] (KDA_GATE_CHANNEL), [total_T, H]
 *                     (KDA_GATE_SCALAR) or NULL (KDA_GATE_NONE)
 *   v, o            : [total_T, H, dv]   dtype
 *   beta            : [total_T, H]       dtype
 *   cu_seqlens      : DEVICE int32 [N + 1], cu_seqlens[0] = 0, non-decreasing,
 *                     cu_seqlens[N] = total_T; sequence n is tokens
 *                     [cu_seqlens[n], cu_seqlens[n+1]). The contents are read
 *                     on the device only: offsets outside [0, total_T] are
 *                     clamped and a decreasing pair is an empty sequence, so a
 *                     malformed array cannot make a kernel access memory
 *                     outside these tensors.
 *   S0, S_T         : [N, H, dk, dv] float (per sequence; NULL as above)
 * Each sequence is computed exactly as kda_chunk_fwd_v would compute it
 * alone (its own chunking from its first token; a zero-length sequence
 * copies S0 to S_T). Workspace as for kda_chunk_fwd_v with B = N.
 */
kda_status_t kda_chunk_fwd_varlen(const void *q, const void *k, const void *v, const void *log_alpha,
                                  const void *beta, const float *S0, void *o, float *S_T,
                                  const int *cu_seqlens, int N, int total_T, int H, int dk, int dv, int chunk,
                                  kda_dtype_t dtype, int erase, kda_gate_t gate, void *workspace,
                                  size_t workspace_bytes, kda_algo_t algo, void *stream);

/*
 * Backward of the prefill (training): gradients of a loss L given
 * dO = dL/do and dS_T = dL/dS_T, for any variant.
 *
 * The pages give no backward pass ("Decoding Hybrid Attention Architectures",
 * section 5, names training throughput as a goal). This is the chain rule
 * through the update of section 3.4, in the same chunked form as the forward
 * pass: a forward sweep keeps the state every 64 tokens, a backward sweep
 * walks 8-token chunks in reverse with the adjoint of the state on chip. The
 * decay gradient comes from an identity of the update (a shift of log a at
 * token t equals a rescaling of every later query and key), as one reverse
 * running sum per channel.
 *
 *   inputs as for kda_chunk_fwd_v (q, k, log_alpha, v, beta, S0 may be NULL)
 *   dO          : [B, T, H, dv]  dtype
 *   dS_T        : [B, H, dk, dv] float, or NULL (zero)
 *   d_q, d_k    : [B, T, H, dk]  dtype, written
 *   d_v         : [B, T, H, dv]  dtype, written
 *   d_log_alpha : shape of log_alpha, written (NULL allowed for KDA_GATE_NONE)
 *   d_beta      : [B, T, H]      dtype, written
 *   d_S0        : [B, H, dk, dv] float, written; NULL: not computed
 *   dk == dv in {64, 128}
 *   workspace   : device scratch of kda_chunk_bwd_workspace_size(...) bytes,
 *                 16-byte aligned. By default (KDA_BWD_AUTO) it keeps every
 *                 8-token chunk's entry state and delta (fp32) when that is at
 *                 most 16 GB, and otherwise one state per 64 tokens plus 8
 *                 (state, delta) slots per (batch, head), recomputing each
 *                 block before reversing it
 * Arithmetic: fp32 (exact per-pair decay exponentials, all with non-positive
 * exponents; the matrix products on tensor cores with each fp32 operand split
 * into two tf32 parts, which keeps fp32-level accuracy), gradients rounded to
 * dtype once. One CTA per (batch, head).
 */
size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv);

/* Workspace policy of the backward pass: AUTO (as above), STORE_ALL (every
 * chunk's state, whatever the size), LOW_MEMORY (one state per 64 tokens and
 * a recompute sweep, about a third more time). */
typedef enum { KDA_BWD_AUTO = 0, KDA_BWD_STORE_ALL = 1, KDA_BWD_LOW_MEMORY = 2 } kda_bwd_mode_t;
size_t kda_chunk_bwd_workspace_size_ex(int B, int T, int H, int dk, int dv, kda_bwd_mode_t mode);
kda_status_t kda_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                           const float *S0, const void *dO, const float *dS_T, void *d_q, void *d_k, void *d_v,
                           void *d_log_alpha, void *d_beta, float *d_S0, int B, int T, int H, int dk, int dv,
                           kda_dtype_t dtype, int erase, kda_gate_t gate, void *workspace, size_t workspace_bytes,
                           void *stream);
kda_status_t kda_chunk_bwd_ex(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                              const float *S0, const void *dO, const float *dS_T, void *d_q, void *d_k, void *d_v,
                              void *d_log_alpha, void *d_beta, float *d_S0, int B, int T, int H, int dk, int dv,
                              kda_dtype_t dtype, int erase, kda_gate_t gate, kda_bwd_mode_t mode, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Device-side status left in `workspace` by the last prefill call
 * (kda_chunk_fwd, _ex, _v, _varlen) that used it: synchronises `stream`,
 * then returns KDA_OK, or KDA_ERR_TIMEOUT if a bounded wait inside a kernel
 * gave up (that kernel's outputs are then invalid), or KDA_ERR_CUDA if the
 * stream reported an error.
 *
 * Which calls can report KDA_ERR_TIMEOUT: only the prefill calls that run the
 * tensor-core kernel (KDA_ALGO_TC, KDA_ALGO_TC_SCAN, or AUTO where it picks
 * them). Its warps hand work to one another through shared-memory barriers;
 * every wait on one gives up after about one second of SM clock, writes 1
 * into the first 4 bytes of the workspace, skips every later wait and frees
 * its tensor memory, so the kernel always returns. The call itself cannot see
 * this (it returns once the work is enqueued): read it here, or with
 * kda_noalloc_status for kda_chunk_fwd_noalloc. The SIMT prefill, the decode
 * step and the backward pass have no waits between warps that could run out
 * (only block-wide barriers) and never report it.
 */
kda_status_t kda_workspace_status(const void *workspace, size_t workspace_bytes, void *stream);

/*
 * Test hook for the timeout path above (no counterpart in the paper; not for
 * production use). Takes the arguments of kda_chunk_fwd (KDA variant,
 * algorithm KDA_ALGO_TC, T >= 1) plus wait_budget_cycles in [1, 2^31], and
 * launches the tensor-core prefill with two faults injected: every CTA
 * withholds its first k/q tile load, and every wait between warps gives up
 * after wait_budget_cycles SM cycles instead of about one second. The first
 * wait on that tile therefore expires; the kernel records KDA_ERR_TIMEOUT in
 * the workspace, skips its later waits, waits (bounded) for the copies it did
 * issue and returns. o and S_T are then undefined; kda_workspace_status
 * reports KDA_ERR_TIMEOUT. A later normal call on the same stream and
 * workspace is unaffected. Synchronous errors as kda_chunk_fwd_ex, plus
 * KDA_ERR_INVALID_ARG for T = 0 or a budget out of range.
 */
kda_status_t kda_chunk_fwd_timeout_test(const void *q, const void *k, const void *v, const void *log_alpha,
                                        const void *beta, const float *S0, void *o, float *S_T, int B, int T,
                                        int H, int dk, int dv, int chunk, kda_dtype_t dtype, void *workspace,
                                        size_t workspace_bytes, long long wait_budget_cycles, void *stream);

/*
 * One recurrent decode step: kda_decode_step(q, k, v, log_alpha, beta, S -> o, S').
 *
 *   q, k, log_alpha : [N, H, dk]      dtype
 *   v               : [N, H, dv]      dtype
 *   beta            : [N, H]          dtype
 *   S_in            : [N, H, dk, dv]  float
 *   S_out           : [N, H, dk, dv]  float, may equal S_in (in-place update)
 *   o               : [N, H, dv]      dtype
 *   dk, dv          : 64 or 128 (dk == dv)
 * Per head: S' = Diag(alpha) S; delta = beta (v - S'^T k); S_out = S' + k delta^T;
 * o = S_out^T q. State arithmetic in fp32.
 */
kda_status_t kda_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                             const void *beta, const float *S_in, float *S_out, void *o, int N, int H,
                             int dk, int dv, kda_dtype_t dtype, void *stream);

/* kda_decode_step for any variant: erase 0/1; log_alpha [N, H, dk]
 * (KDA_GATE_CHANNEL), [N, H] (KDA_GATE_SCALAR) or NULL (KDA_GATE_NONE). Per
 * head: S' = Diag(a) S; delta = beta (v - S'^T k) (erase = 1) or beta v
 * (erase = 0); S_out = S' + k delta^T; o = S_out^T q. */
kda_status_t kda_decode_step_v(const void *q, const void *k, const void *v, const void *log_alpha,
                               const void *beta, const float *S_in, float *S_out, void *o, int N, int H,
                               int dk, int dv, kda_dtype_t dtype, int erase, kda_gate_t gate, void *stream);

/*
 * Allocation-free prefill (no counterpart in the paper; an addition of this
 * library). Same operation, arguments and numerics as kda_chunk_fwd with the
 * tensor-core algorithm, minus the workspace: the kernel's scratch (its
 * 4-byte device status word) lives in a fixed 256-byte array inside libkda.so.
 * It is meant for callers that must not allocate device memory where they run
 * a prefill -- code running inside a memory allocator's own callbacks, hosts
 * that forbid cudaMalloc on their worker threads, runtimes that only expose
 * the tensors they already own. The call itself allocates nothing.
 *
 *   - Supports what the tensor-core path supports: dtype KDA_BF16,
 *     dk = dv = 128, chunk = 64 (else KDA_ERR_UNSUPPORTED). A shape whose
 *     scratch would exceed the 256-byte array is refused with
 *     KDA_ERR_INVALID_ARG (no supported shape needs more than 256 bytes).
 *   - Every call looks up the array's device address (cudaGetSymbolAddress,
 *     a host-side query) with the caller's current device, which must be the
 *     device of the tensors. The very first call in a process may also load
 *     the library's device code; make that first call before capturing any
 *     CUDA graph.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call clears the status word before its kernel runs. Calls
 *     that overlap on the GPU (different streams, no ordering) race on the
 *     array. A device-side timeout is recorded in the array and read back by
 *     kda_noalloc_status.
 */
kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *log_alpha,
                                   const void *beta, const float *S0, void *o, float *S_T, int B, int T,
                                   int H, int dk, int dv, int chunk, kda_dtype_t dtype, void *stream);

/*
 * Device-side status of the last kda_chunk_fwd_noalloc on the current device
 * (the counterpart of kda_workspace_status for the library's own array; no
 * counterpart in the paper). Synchronises `stream`, then copies the 4-byte
 * status word out of the array (no allocation): KDA_OK, KDA_ERR_TIMEOUT if a
 * bounded wait in that call's kernel gave up (its outputs are then invalid),
 * or KDA_ERR_CUDA if the stream or the copy reported an error. Racy in the
 * same way as the calls themselves when they overlap on the GPU.
 */
kda_status_t kda_noalloc_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
