/*
 * linattn.h -- C ABI of liblinattn.so: causal linear attention over a
 * recurrent state on NVIDIA B200 (sm_100a).
 *
 * The operation (slides "Chunking, causality, and parallel prefill"):
 *
 *   recurrence ("Naive recurrence", "Incoming and outgoing state")
 *       S_t = S_{t-1} + k_t v_t^T,      o_t = q_t^T S_t
 *   chunkwise prefill ("Split into chunks", "Worked case - full trace"),
 *   for each chunk c of C tokens, in order:
 *       M   = tril(Q_c K_c^T)           (j <= i, diagonal included)
 *       O_c = M V_c + Q_c S_{c-1}       (local term + incoming-state read)
 *       S_c = S_{c-1} + K_c^T V_c       (the one serial hop)
 *   decode ("Prefill and decode": one token, a 1x1 triangle)
 *       S <- S + k v^T,                 o = q^T S
 *
 * The chunk size C is an execution parameter: it never changes the result
 * in exact arithmetic ("Chunk size"), only the cost and the rounding order.
 *
 * Conventions shared by every entry point
 *   - Every pointer is device memory owned by the caller.  No entry point
 *     allocates device memory, keeps a pointer after it returns, or
 *     synchronises the stream, except la_device_status().
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued on it; errors of the kernels themselves are
 *     reported by la_device_status().
 *   - Q, K are [.., T, d_k] and V, O are [.., T, d_v], contiguous, row-major,
 *     in the dtype named by `dtype` (LA_F32 or LA_BF16).  The state is always
 *     float32 [units][d_k][d_v], row index = key dimension (the trace's
 *     S_4 = K_1^T V_1 = [[3,4],[5,5]]).
 *   - Dense layout: [B, H, T, d]; unit (b, h) = b*H + h owns rows 0..T-1.
 *     Packed variable-length layout (cu_seqlens != NULL): B must be 1, the
 *     tensors are [1, H, T_total, d], sequence n occupies rows
 *     cu_seqlens[n] .. cu_seqlens[n+1]-1 of every head, and the state is
 *     [num_seqs, H, d_k, d_v] (unit n*H + h).
 *   - An empty sequence (length 0) is a no-op that leaves its state as is.
 *   - Return value: LA_OK, or LA_ERR_INVALID_ARG (bad pointer, size or
 *     layout), LA_ERR_UNSUPPORTED (a valid request outside what the kernels
 *     implement), LA_ERR_CUDA (a launch or runtime call failed; the CUDA
 *     error string is kept for la_last_cuda_error()).  Nothing is enqueued
 *     when an argument check fails.
 */
#ifndef LINATTN_H
#define LINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,
    LA_ERR_UNSUPPORTED = 2,
    LA_ERR_CUDA = 3,
    LA_ERR_TIMEOUT = 4
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/* Initial state S_0 ("Worked case - full trace" starts from S_0 = 0).
 * state: [n_units][d_k][d_v] float32, written.  src: same shape, read; NULL
 * means zero.  n_units = B*H (dense) or num_seqs*H (packed).
 * Errors: LA_ERR_INVALID_ARG for state == NULL with n_units > 0, or a
 * non-positive d_k / d_v. */
la_status la_state_init(float* state, const float* src, int64_t n_units,
                        int d_k, int d_v, void* stream);

/* Chunkwise prefill of every unit ("Split into chunks").
 *   q, k: [.., T, d_k]; v, o: [.., T, d_v] in `dtype` (o written).
 *   state: [units][d_k][d_v] float32: S_0 on entry, S_T on return.
 *   B, H, T: dense sizes; with cu_seqlens, B == 1 and T = total rows.
 *   cu_seqlens: NULL (dense) or num_seqs+1 int32 device offsets rising from
 *     0 to T.  They are read by the kernels, not checked on the host.
 *   max_seqlen: packed mode only, an upper bound on every sequence length
 *     (host value; 0 = unknown); ignored for dense input.  When it is at
 *     most 16 the few-token kernel runs, and a sequence too long for it is
 *     left untouched and reported by la_device_status (LA_ERR_INVALID_ARG).
 *   chunk: C, the number of tokens per chunk; 0 picks the default for the
 *     shape (LINATTN_CHUNK in the environment overrides the default; like
 *     every LINATTN_* switch it is read once per process, on first use).
 *   workspace / workspace_bytes: device scratch of la_prefill_workspace_size()
 *     bytes, 16-byte aligned, owned by the caller and free for the library
 *     until the call's work on `stream` has finished.  It buys speed only:
 *     with less (or NULL) the call skips what the scratch is for (the split
 *     of few long sequences into segments; the dynamic, longest-first walk
 *     of packed sequences) and gives the same results.
 * Kernels: at most 16 tokens per unit (T, or max_seqlen), d_v a multiple of
 * 4 and a 16-byte aligned state run the few-token kernel: one pass over the
 * state, each state row stepped through the tokens (the recurrence itself),
 * fp32 CUDA cores.  Otherwise bf16 with
 * d_k == d_v in {64, 128}, 16-byte aligned q/k/v/o and chunk in
 * {16, 32, 64, 128} run on the tensor cores (TMA + tcgen05, fp32
 * accumulation, fp32 state on chip); everything else with d_k, d_v <= 128
 * runs the fp32 CUDA-core kernel.  Errors: LA_ERR_INVALID_ARG (NULL tensor
 * with T > 0, B/H/T/d negative, B != 1 with cu_seqlens), LA_ERR_UNSUPPORTED
 * (d_k or d_v above 128, a chunk the kernels cannot stage in shared
 * memory). */
la_status la_prefill(const void* q, const void* k, const void* v, void* o,
                     float* state, la_dtype dtype, int B, int H, int64_t T,
                     int d_k, int d_v, const int32_t* cu_seqlens, int num_seqs,
                     int64_t max_seqlen, int chunk, void* workspace,
                     size_t workspace_bytes, void* stream);

/* Bytes of device workspace la_prefill can use for these arguments (0 when
 * it uses none): segment states of the intra-sequence split (dense input),
 * or, for packed input, a work counter (256 bytes) followed by one int32 per
 * sequence (2 to 4096 sequences) for the longest-first order. */
size_t la_prefill_workspace_size(la_dtype dtype, int B, int H, int64_t T,
                                 int d_k, int d_v, int num_seqs, int chunk);

/* Size of the library's own static scratch buffer used by la_prefill_noalloc
 * (64 MiB, held on every GPU that loads the library until the process exits). */
#define LA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* la_prefill for callers that cannot allocate device memory.  The slides have
 * no counterpart to this entry point; it exists for callers that run inside
 * an engine which owns every byte of device memory (a serving runtime with a
 * fixed memory plan, a plugin living inside another framework's caching
 * allocator) or on a path where a cudaMalloc would synchronise the device.
 * Same arguments and results as la_prefill, without workspace: the scratch
 * that la_prefill would take from the caller (la_prefill_workspace_size
 * bytes) comes from a static device buffer of LA_NOALLOC_SCRATCH_BYTES inside
 * the library.  Nothing is allocated or freed, by this call or any library it
 * calls.
 *   - The first call on a device looks up that device's address of the
 *     buffer (again when the device's current context has changed, e.g.
 *     after cudaDeviceReset); make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one buffer, and calls that overlap
 *     on the GPU (different streams, no ordering between them) race on it.
 *     Every byte a call reads from the buffer was written earlier in the same
 *     call, so nothing needs clearing between calls.
 *   - A request whose scratch would exceed LA_NOALLOC_SCRATCH_BYTES returns
 *     LA_ERR_UNSUPPORTED before launching anything; la_last_cuda_error()
 *     then states the bytes needed and the bytes available.
 * Other errors as for la_prefill. */
la_status la_prefill_noalloc(const void* q, const void* k, const void* v,
                             void* o, float* state, la_dtype dtype, int B,
                             int H, int64_t T, int d_k, int d_v,
                             const int32_t* cu_seqlens, int num_seqs,
                             int64_t max_seqlen, int chunk, void* stream);

/* One decode token for every unit ("Prefill and decode", 1x1 triangle):
 *   S' = S + k v^T, o = q^T S' (= q^T S + (q.k) v).
 *   q, k: [B, H, d_k]; v, o: [B, H, d_v] in `dtype`; state [B*H][d_k][d_v]
 *   float32, updated in place.  Errors as for la_prefill. */
la_status la_decode_step(const void* q, const void* k, const void* v, void* o,
                         float* state, la_dtype dtype, int B, int H, int d_k,
                         int d_v, void* stream);

/* Synchronises `stream`, then reports and clears the device error word of
 * the current device: LA_ERR_TIMEOUT if a kernel gave up a bounded wait
 * (its outputs are then undefined), LA_ERR_INVALID_ARG if a packed sequence
 * was longer than the max_seqlen given to la_prefill (that unit was left
 * untouched), LA_ERR_CUDA if the synchronisation failed, else LA_OK. */
la_status la_device_status(void* stream);

/* Diagnostic of the failure path (no counterpart on the slides): launches
 * one kernel whose single thread waits on a barrier that nothing completes,
 * with the same bounded wait the prefill kernels use, limited to
 * `timeout_ms`.  The kernel gives up, records the timeout in the device
 * error word and returns; the next la_device_status() reports
 * LA_ERR_TIMEOUT and clears it.  Nothing faults or hangs; the context stays
 * usable.  Errors: LA_ERR_INVALID_ARG for timeout_ms outside (0, 10000]. */
la_status la_selftest_wait_timeout(double timeout_ms, void* stream);

/* Which chunked kernel la_prefill would run for these arguments: "tc"
 * (tensor cores), "simt" (fp32 CUDA cores) or "unsupported".  Host only. */
const char* la_prefill_path(la_dtype dtype, int d_k, int d_v, int chunk,
                            const void* q, const void* k, const void* v,
                            const void* o);

/* Which kernel la_prefill runs, given also max_tokens (T for dense input,
 * max_seqlen for packed input) and the state pointer: "short" (at most 16
 * tokens per unit: one pass over the state, fp32 CUDA cores), "tc", "simt"
 * or "unsupported".  Host only. */
const char* la_prefill_kernel(la_dtype dtype, int64_t max_tokens, int d_k,
                              int d_v, int chunk, const void* q, const void* k,
                              const void* v, const void* o,
                              const float* state);

/* The chunk size la_prefill uses for `chunk` (resolves 0 to the default). */
int la_resolve_chunk(la_dtype dtype, int d_k, int d_v, int chunk);

/* Text of a status code, and of the last CUDA error seen by this library
 * on the calling thread ("" if none). */
const char* la_status_string(la_status s);
const char* la_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LINATTN_H */
