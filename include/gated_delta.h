/*
 * gated_delta.h -- C ABI of the B200 (sm_100a) gated delta-rule library.
 *
 * The operator (thethings.ai, "The argument, in one page", table "Everything,
 * in one table", rows "KDA" and "Gated DeltaNet"), with column-vector keys:
 *
 *     S_t = Diag(a_t) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * S_t is a d_k x d_v fp32 state per (sequence, head), stored row-major
 * [d_k][d_v] (row i belongs to key channel i).  a_t = exp(g_t) with g_t <= 0 a
 * log-decay: a vector over d_k channels for KDA ("kda_*"), one scalar per
 * (token, head) for Gated DeltaNet ("gdn_*").  The decay multiplies the state
 * after the rank-one erase; the fresh write beta_t k_t v_t^T is not decayed
 * (the operator order of the table rows).  o_t reads the state after token t's
 * own update; there is no normaliser and no 1/sqrt(d_k) scale: q is used as
 * given.
 *
 * General conventions
 * -------------------
 *  - Every data pointer is a DEVICE pointer owned by the caller (except in
 *    kda_chunk_fwd_host, which takes host memory).  The library allocates no
 *    device memory (kda_chunk_fwd_noalloc's fixed array is part of its module)
 *    and keeps no state between calls except a per-device cache of attributes
 *    and kda_chunk_fwd_host's copy streams.  Work is enqueued on `stream` (a
 *    cudaStream_t; NULL = the legacy default stream) and the call returns
 *    without synchronising.
 *  - Token layout is [B, T, H, d] with d contiguous (equivalently [B*T, H, d]);
 *    for packed variable-length batches B must be 1 and T is the total token
 *    count.  g is [B, T, H_v, d_k] (KDA) or [B, T, H_v] (GDN); beta is
 *    [B, T, H_v]; states are [N, H_v, d_k, d_v] where N is the number of
 *    sequences (B, or num_seqs when cu_seqlens is given).
 *  - q/k/v/o element type is io_dtype (KDA_BF16 or KDA_F32); g, beta and the
 *    states are always fp32.  io_dtype = KDA_F32 selects the all-fp32 path.
 *  - Supported head sizes: d_k in {64, 128}, d_v in {64, 128}.
 *  - o must not alias any input.  Prefill: q, k, v, g, o and the states must
 *    be 16-byte aligned, beta and cu_seqlens 4-byte aligned.  Decode: the
 *    state 16-byte aligned, the others aligned to their element size.
 *  - The return value reports host-side validation and launch errors.  Errors
 *    found on the device (an invalid cu_seqlens array) are recorded in the
 *    workspace and reported by kda_check_device_status().
 *  - Thread safety: calls on different streams with disjoint buffers may run
 *    concurrently.
 */
#ifndef GATED_DELTA_H
#define GATED_DELTA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_ABI_VERSION 1

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,   /* bad pointer, shape, alignment or size           */
  KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d_k = 96)       */
  KDA_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed          */
  KDA_ERR_DEVICE_CHECK = 4,  /* a device-side check failed (see check call)     */
  KDA_ERR_WORKSPACE = 5      /* workspace pointer NULL or smaller than required */
} kda_status_t;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/* Where the per-channel decay sits relative to the rank-one erase (KDA only;
 * for a scalar gate the two orders are the same operator).
 *   KDA_ERASE_THEN_DECAY  S_t = Diag(a_t)(I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *                         the operator as the table row "KDA" writes it (default);
 *   KDA_DECAY_THEN_ERASE  S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *                         the erase acts on the decayed state, so that with
 *                         beta = 1 and |k| = 1 the update writes only the
 *                         difference between v and what the decayed memory
 *                         recalls (ai-explained.dataextractor.workers.dev
 *                         "The efficiency lineage", item 8 "Delta rule"). */
typedef enum { KDA_ERASE_THEN_DECAY = 0, KDA_DECAY_THEN_ERASE = 1 } kda_order_t;

/* Device-side error codes written to the workspace status word. */
#define KDA_DEVICE_OK 0
#define KDA_DEVICE_BAD_CU_SEQLENS 1  /* cu[0] != 0, decreasing, or cu[N] != T */
#define KDA_DEVICE_TIMEOUT 2         /* a bounded on-device wait expired */

/* --------------------------------------------------------------------------
 * Prefill, per-channel gate (KDA).  Chunked over tokens; the state is carried
 * across chunks on chip.  Row "KDA" of the table; the chunkwise computation
 * follows row "Chunkwise / WY" (the result is the recurrence's, whatever the
 * chunk size).
 *
 *   q, k          [B, T, H, d_k]   io_dtype
 *   v             [B, T, H, d_v]   io_dtype
 *   g             [B, T, H, d_k]   fp32 log-decay (<= 0; a = exp(g)), any
 *                                  magnitude.  (The bf16 path computes a
 *                                  chunk whose 16-token decay sum falls
 *                                  below -32 in some channel with directly
 *                                  formed pair factors: exact, but slower.)
 *   beta          [B, T, H]        fp32 write strength
 *   o             [B, T, H, d_v]   io_dtype, written
 *   initial_state [N, H, d_k, d_v] fp32, or NULL for zeros
 *   final_state   [N, H, d_k, d_v] fp32, written, or NULL
 *   cu_seqlens    [num_seqs + 1]   int32 DEVICE array of token offsets, or NULL
 *                                  (then N = B dense sequences of T tokens).
 *                                  Must satisfy cu[0] = 0, cu[i] <= cu[i+1],
 *                                  cu[num_seqs] = T; zero-length sequences are
 *                                  allowed (their final state = initial state).
 *   workspace     device scratch of at least kda_chunk_fwd_workspace_size()
 *                 bytes, 256-byte aligned; its contents are overwritten.
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, void *o, const float *initial_state,
                           float *final_state, const int32_t *cu_seqlens, int32_t num_seqs,
                           int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                           kda_dtype_t io_dtype, void *workspace, size_t workspace_bytes,
                           void *stream);

KDA_API size_t kda_chunk_fwd_workspace_size(int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                    int32_t num_seqs, kda_dtype_t io_dtype);

/* --------------------------------------------------------------------------
 * Prefill, scalar gate (Gated DeltaNet; row "Gated DeltaNet" of the table).
 * q and k have H_qk heads; v, o, g, beta and the states have H_v heads, with
 * H_v % H_qk == 0 and v-head h reading q/k head h / (H_v / H_qk).
 *
 *   q, k [B, T, H_qk, d_k]; v, o [B, T, H_v, d_v]; g, beta [B, T, H_v];
 *   states [N, H_v, d_k, d_v].  Everything else as kda_chunk_fwd, except that
 *   g has no lower bound here: with one gate value per token every scale
 *   factor of the computation is at most 1.
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, void *o, const float *initial_state,
                           float *final_state, const int32_t *cu_seqlens, int32_t num_seqs,
                           int32_t B, int32_t T, int32_t H_qk, int32_t H_v, int32_t d_k,
                           int32_t d_v, kda_dtype_t io_dtype, void *workspace,
                           size_t workspace_bytes, void *stream);

KDA_API size_t gdn_chunk_fwd_workspace_size(int32_t B, int32_t T, int32_t H_qk, int32_t H_v,
                                    int32_t d_k, int32_t d_v, int32_t num_seqs,
                                    kda_dtype_t io_dtype);

/* --------------------------------------------------------------------------
 * One decode step, per-channel gate: one token for each of N sequences; the
 * state is read once and updated IN PLACE.  Same operator as kda_chunk_fwd
 * (inferencex.semianalysis.com "Linear attention": a recurrent state of
 * constant size updated as tokens arrive).
 *
 *   q, k  [N, H, d_k] io_dtype;  v [N, H, d_v] io_dtype
 *   g     [N, H, d_k] fp32 log-decay;  beta [N, H] fp32
 *   o     [N, H, d_v] io_dtype, written
 *   state [N, H, d_k, d_v] fp32, read and overwritten
 * Needs no workspace.
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, void *o, float *state, int32_t N, int32_t H,
                             int32_t d_k, int32_t d_v, kda_dtype_t io_dtype, void *stream);

/* One decode step, scalar gate, q/k heads shared as in gdn_chunk_fwd:
 *   q, k [N, H_qk, d_k]; v, o [N, H_v, d_v]; g, beta [N, H_v];
 *   state [N, H_v, d_k, d_v] in place. */
KDA_API kda_status_t gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, void *o, float *state, int32_t N,
                             int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                             kda_dtype_t io_dtype, void *stream);

/* --------------------------------------------------------------------------
 * Prefill with the decay order and a state pool (KDA and Gated DeltaNet).
 * Same operation, arguments and errors as kda_chunk_fwd / gdn_chunk_fwd, plus:
 *
 *   order        KDA_ERASE_THEN_DECAY (what kda_chunk_fwd computes) or
 *                KDA_DECAY_THEN_ERASE; gdn has no order argument.
 *   state_slots  int32 DEVICE array [N] (N = B, or num_seqs with cu_seqlens),
 *                or NULL.  When given, initial_state and final_state are
 *                POOLS of num_slots states [num_slots, H, d_k, d_v] and
 *                sequence n reads its initial state from slot state_slots[n]
 *                and writes its final state to the same slot.  initial_state
 *                and final_state may be the same pool (in-place update of a
 *                serving state pool: inferencex.semianalysis.com "Linear
 *                attention", "Why it matters": a dropped state can only be
 *                rebuilt by replaying the sequence, so it is checkpointed).
 *                A slot outside [0, num_slots) means "no slot": the sequence
 *                starts from zeros and its final state is not stored.  Two
 *                sequences must not share a slot (the slot's contents are
 *                then unspecified).
 *   num_slots    pool capacity (ignored when state_slots is NULL).
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t kda_chunk_fwd_ex(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, void *o,
                                      const float *initial_state, float *final_state,
                                      const int32_t *state_slots, int64_t num_slots,
                                      const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                                      int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                      kda_order_t order, kda_dtype_t io_dtype, void *workspace,
                                      size_t workspace_bytes, void *stream);

KDA_API kda_status_t gdn_chunk_fwd_ex(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, void *o,
                                      const float *initial_state, float *final_state,
                                      const int32_t *state_slots, int64_t num_slots,
                                      const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                                      int32_t T, int32_t H_qk, int32_t H_v, int32_t d_k,
                                      int32_t d_v, kda_dtype_t io_dtype, void *workspace,
                                      size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * Token-by-token form for a few tokens per sequence: T consecutive tokens of
 * each of N sequences (T = 1 is one decode step; T > 1 serves speculative
 * decoding or a prompt fed in small pieces), applied one after another to
 * the state, which is read from HBM once and written back once, in place.
 * The result equals T single decode steps (and a prefill of the same tokens).
 *
 *   q, k  [N, T, H_qk, d_k] io_dtype;  v, o [N, T, H_v, d_v] io_dtype
 *   g     [N, T, H_v, d_k] fp32 (KDA) or [N, T, H_v] fp32 (GDN)
 *   beta  [N, T, H_v] fp32
 *   state the states, [N, H_v, d_k, d_v] fp32 when state_slots is NULL; else
 *         a pool [num_slots, H_v, d_k, d_v] of which sequence n uses slot
 *         state_slots[n] (int32 DEVICE array [N]).  A slot outside
 *         [0, num_slots) marks a padding entry: its o rows are written as
 *         zeros and no state is touched.  Slots of different sequences must
 *         differ.
 *   order KDA only, as in kda_chunk_fwd_ex.
 * Alignment as the decode step; state_slots 4-byte aligned.  No workspace.
 * Any T >= 0 is accepted; past a chunk's worth of tokens the chunked prefill
 * is the faster route.
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t kda_recurrent_fwd(const void *q, const void *k, const void *v,
                                       const float *g, const float *beta, void *o, float *state,
                                       const int32_t *state_slots, int64_t num_slots, int32_t N,
                                       int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                       kda_order_t order, kda_dtype_t io_dtype, void *stream);

KDA_API kda_status_t gdn_recurrent_fwd(const void *q, const void *k, const void *v,
                                       const float *g, const float *beta, void *o, float *state,
                                       const int32_t *state_slots, int64_t num_slots, int32_t N,
                                       int32_t T, int32_t H_qk, int32_t H_v, int32_t d_k,
                                       int32_t d_v, kda_dtype_t io_dtype, void *stream);

/* --------------------------------------------------------------------------
 * State checkpoint / transfer for a serving state pool
 * (inferencex.semianalysis.com "Linear attention", "How to read it in
 * InferenceX": engines checkpoint and transfer the recurrent state so that a
 * repeated turn does not pay its prefill again).  Batched copies of whole states [H, d_k, d_v] fp32 by slot:
 *
 *   kda_state_gather   out[n]  = pool[state_slots[n]]   (zeros for a slot
 *                                                        outside [0, num_slots))
 *   kda_state_scatter  pool[state_slots[n]] = src[n]    (skipped for a slot
 *                                                        outside [0, num_slots))
 *
 * pool is [num_slots, H, d_k, d_v]; out/src are dense [N, H, d_k, d_v]; all
 * DEVICE pointers, 16-byte aligned, pool and dense buffer distinct; slots
 * int32 DEVICE [N], non-NULL.  Scatter slots must be distinct.  For a copy
 * to or from host memory, gather into a dense device buffer first.
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t kda_state_gather(const float *pool, const int32_t *state_slots,
                                      int64_t num_slots, float *out, int32_t N, int32_t H,
                                      int32_t d_k, int32_t d_v, void *stream);
KDA_API kda_status_t kda_state_scatter(const float *src, float *pool,
                                       const int32_t *state_slots, int64_t num_slots, int32_t N,
                                       int32_t H, int32_t d_k, int32_t d_v, void *stream);

/* --------------------------------------------------------------------------
 * kda_chunk_fwd for callers that cannot allocate device memory (the pages
 * have no counterpart: this is a deployment convenience).  Some hosts own all
 * device memory through their own pool and do not let a library call
 * cudaMalloc, or run where an allocation (which may synchronise the device)
 * is not allowed.  This call takes the same arguments as kda_chunk_fwd minus
 * the workspace and runs the same kernels with their scratch in a fixed
 * 64 MiB array inside this library's device memory; it allocates nothing.
 *
 *  - Problems whose kda_chunk_fwd_workspace_size() exceeds 64 MiB are
 *    rejected with KDA_ERR_WORKSPACE (kda_last_error() gives the sizes);
 *    use kda_chunk_fwd with a workspace for them.
 *  - The 64 MiB are reserved on a device when the library's module holding
 *    the array is loaded there.  Under CUDA's default lazy module loading
 *    that is the first call of this function on that device (with
 *    CUDA_MODULE_LOADING=EAGER, when the library is loaded); the memory then
 *    stays reserved until the process exits or the context is destroyed.  A
 *    host whose pool claims the device's memory should make one call first:
 *    a call with T = 0 computes nothing and only reserves the array.  If it
 *    cannot be reserved the call returns KDA_ERR_CUDA (kda_last_error() says
 *    why).
 *  - The first call on each device (and the first after a device reset)
 *    looks up the array's device address (cudaGetSymbolAddress) with that
 *    device current; make that first call before capturing the stream into
 *    a CUDA graph.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents (each call resets its own status word).  Calls whose kernels
 *    overlap on the GPU (different streams or threads) race on it: order
 *    them on one stream.  A device-side error (an invalid cu_seqlens) leaves
 *    o and final_state unwritten; this call offers no status word to read.
 * ------------------------------------------------------------------------ */
KDA_API kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                           const float *g, const float *beta, void *o,
                                           const float *initial_state, float *final_state,
                                           const int32_t *cu_seqlens, int32_t num_seqs,
                                           int32_t B, int32_t T, int32_t H, int32_t d_k,
                                           int32_t d_v, kda_dtype_t io_dtype, void *stream);

/* ---------------------------------------------------------------------------
 * kda_chunk_fwd_host -- the KDA prefill of kda_chunk_fwd (dense batch, same
 * operator, same kernels) with q, k, v, g, beta, o and the states in HOST
 * memory, for a caller whose prompt is not on the device yet.  The tokens are
 * cut into `pieces` spans of equal length (a multiple of C = 64; pieces <= 0
 * means 4, at most 64): while the kernels run on span p, the host-to-device
 * copy of span p + 1 and the device-to-host copy of span p - 1's output run
 * on two internal copy streams, so the transfers overlap each other and the
 * computation.  Each span is one prefill whose initial state is the previous
 * span's final state (fp32, through device memory), which is what a single
 * call over all tokens computes between its chunks: the results equal
 * kda_chunk_fwd's.
 *
 *   q, k, v, g, beta, o, initial_state, final_state
 *                 host pointers, the layouts of kda_chunk_fwd; pinned memory
 *                 (cudaHostAlloc / cudaHostRegister) for the copies to
 *                 overlap; initial_state may be NULL (zeros), final_state
 *                 NULL (not returned)
 *   B, T, H, d_k, d_v, io_dtype    as kda_chunk_fwd; T > 0
 *   device_buffer  device memory of kda_chunk_fwd_host_buffer_size() bytes,
 *                 256-byte aligned, owned by the caller: the staged inputs
 *                 and outputs, the states and the workspace, whose status
 *                 word is at offset 0 (read it with kda_check_device_status
 *                 on device_buffer)
 *   stream        the caller's stream: the kernels run on it, the copies
 *                 start after the work queued on it before the call, and work
 *                 queued after the call starts once every copy has landed
 *
 * Asynchronous like the other calls: o and final_state are valid on the host
 * once `stream` has been synchronised.  Calls for one device serialise their
 * enqueueing on an internal lock (the copy streams are shared per device; the
 * library creates them and their events at the first call on a device and
 * keeps them until the process exits).
 * Returns KDA_ERR_INVALID_ARG / KDA_ERR_UNSUPPORTED for bad arguments (T = 0
 * included: there is nothing to stream), KDA_ERR_WORKSPACE for a missing,
 * misaligned or short device_buffer, KDA_ERR_CUDA for a failed copy or
 * launch.
 * ------------------------------------------------------------------------ */
KDA_API size_t kda_chunk_fwd_host_buffer_size(int32_t B, int32_t T, int32_t H, int32_t d_k,
                                              int32_t d_v, kda_dtype_t io_dtype, int32_t pieces);
KDA_API kda_status_t kda_chunk_fwd_host(const void *q, const void *k, const void *v,
                                        const float *g, const float *beta, void *o,
                                        const float *initial_state, float *final_state,
                                        int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                        kda_dtype_t io_dtype, int32_t pieces,
                                        void *device_buffer, size_t device_buffer_bytes,
                                        void *stream);

/* Wait for `stream`, then read the device status word of a prefill workspace.
 * Returns KDA_OK or KDA_ERR_DEVICE_CHECK (device code in *device_code when
 * non-NULL), or KDA_ERR_CUDA.  Synchronises the stream. */
KDA_API kda_status_t kda_check_device_status(const void *workspace, void *stream,
                                     int32_t *device_code);

/* Diagnostic: runs one on-device wait that nothing ever completes, bounded like
 * every wait in the library's kernels (an mbarrier poll loop of at most
 * max_polls polls; a poll of a phase that never completes returns after a few
 * microseconds on B200).  When the bound expires the kernel
 * writes KDA_DEVICE_TIMEOUT into the status word at the start of `workspace`
 * (any prefill workspace, or 4 bytes of device memory) and returns, exactly as
 * an expired wait inside a prefill does; kda_check_device_status() then
 * reports it.  Lets a caller test its handling of an expired wait without
 * faulting or hanging the GPU.  The status word is reset to KDA_DEVICE_OK
 * first.  max_polls in [1, 4096]; returns KDA_ERR_INVALID_ARG otherwise (or
 * for a NULL workspace) before touching the device.  Asynchronous on `stream`. */
KDA_API kda_status_t kda_selftest_wait_timeout(void *workspace, int32_t max_polls, void *stream);

/* Bounds-checked build (libgated_delta_checked.so, compiled with
 * -DGDR_BOUNDS_CHECK; the sanitizer substitute of this library).  In that
 * build every index a kernel computes for a global-memory access of its own
 * (inputs, outputs, states, chunk table, workspace slots; the tensor-map tile
 * copies are bounded by the TMA unit itself) is compared with the extent of
 * the buffer it addresses.  A failed comparison counts one violation and the
 * access is skipped: no trap, no access outside the buffer.  Results are
 * otherwise the same as the normal build's, a little slower.
 *
 * kda_bounds_checked(): 1 in the bounds-checked build, 0 in the normal one.
 *
 * kda_bounds_violations(): waits for `stream`, then stores in *count the
 * violations counted on the current device since the last call (and resets
 * the counters).  Always 0 in the normal build.  Returns KDA_ERR_INVALID_ARG
 * for a NULL count, KDA_ERR_CUDA if the device cannot be read. */
KDA_API int32_t kda_bounds_checked(void);
KDA_API kda_status_t kda_bounds_violations(void *stream, uint32_t *count);

/* Static text for a status code. */
KDA_API const char *kda_status_string(kda_status_t status);

/* Detail of the last error raised on the calling host thread ("" if none). */
KDA_API const char *kda_last_error(void);

/* Optional per-kernel device timing.  With kda_trace_enable(1), every kernel
 * the library launches is bracketed by two CUDA events on the caller's stream
 * (adds two event records per launch; off by default).  kda_trace_read()
 * waits for the recorded launches, writes up to `capacity` kernel names
 * (NUL-terminated, `name_stride` bytes apart) and durations in milliseconds,
 * clears the record list and returns the number of records written. */
KDA_API kda_status_t kda_trace_enable(int32_t on);
KDA_API int32_t kda_trace_read(char *names, int32_t name_stride, float *ms, int32_t capacity);

/* KDA_ABI_VERSION of the loaded library. */
KDA_API int32_t kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GATED_DELTA_H */
