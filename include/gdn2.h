/*
 * gdn2.h - C ABI of the B200 (sm_100a) Gated Delta Rule-2 operator library
 * (libgdn2.so).
 *
 * The operator ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
 * Attention"; anthology-of-the-sota LIT-802 review, "Key takeaways" 1, paper
 * Sec. 3.1 Eqs. 8-10) is, for every batch row b and head h independently,
 *
 *     S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T,
 *     D_t = diag(exp g_t),          o_t = S_t^T q_t,
 *
 * with a channel-wise log-decay g_t (key axis), erase gate b_t (key axis) and
 * write gate w_t (value axis).  The read o_t = S_t^T q_t (after the update, no
 * scale) is the reading taken for this library; the pages never print it.
 * Gate activations (sigmoid, logsigmoid) and any q/k normalisation or 1/sqrt(d)
 * scale belong to the caller: the library takes the activated values.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layouts (all contiguous, innermost dimension fastest):
 *   q, k, g, b, dq, dk, dg, db : [B, T, H, d_k]
 *   v, w, o, dO, dv, dw        : [B, T, H, d_v]
 *   S0, ST, dST, dS0           : [B, H, d_k, d_v]   (row = key channel)
 * Decode uses the same layouts with T = 1 removed: [N, H, d] and
 * [N, H, d_k, d_v].
 * Element types: q, k, v, o, dO, dq, dk, dv are float32 (GDN2_IO_F32) or
 *   bfloat16 (GDN2_IO_BF16); g, b, w, dg, db, dw are float32, or bfloat16
 *   through the *_ex entry points (gate_io); every state is float32.
 * Supported sizes: B, T, H, N >= 1; d_k, d_v in {32, 64, 128}; chunk in
 *   {16, 32, 64}.  T need not be a multiple of chunk (the last chunk is short).
 *   The chunk size changes only the order of rounding, never the result.
 * Pointers: device memory owned by the caller; the library allocates nothing
 *   and keeps no pointer after a call returns.  Every pointer must be 16-byte
 *   aligned.  Input and output buffers must not overlap (except S in
 *   gdn2_decode_step, which is updated in place).
 * Streams: every call only enqueues work on `stream` (NULL = the legacy
 *   default stream) and returns without synchronising, except
 *   gdn2_get_device_status.
 * Errors: arguments are checked on the host before anything is launched; a
 *   failed check returns a status and enqueues nothing.  A failed launch
 *   returns GDN2_ERR_CUDA.  Kernels never trap: a kernel that gives up on a
 *   bounded wait records GDN2_ERR_TIMEOUT in a device status word that
 *   gdn2_get_device_status reports.
 * Paths: bf16 I/O with d_k = d_v = 128 and chunk 64 runs on the tensor cores
 *   (fp16 and tf32 operands, fp32 accumulation and state); every other
 *   combination runs on the float32 CUDA-core path.  Both take any log-decay
 *   g <= 0.  The tensor-core path forms every decay factor so that it stays
 *   within fp16's range: state-side factors relative to the chunk's start
 *   (all <= 1), in-chunk pair factors relative to 16-row block boundaries
 *   (<= 1), and the 16 x 16 diagonal blocks in float32 relative to the block's
 *   middle with each token's log-decay floored at -9 for those factors only
 *   (a pair factor changes only where it is below e^-9 already, by at most
 *   e^-9).  Chunks whose decay stays within e^4 of the chunk's row 31 (and
 *   |q|, |k|, |b k| <= 256) take one frame for the whole chunk instead, which
 *   is exact and faster.  An fp16 operand beyond 6e4 in magnitude (inputs or
 *   states far outside the usual range) records GDN2_ERR_RANGE in the device
 *   status word (the results of that call are then not valid); the float32
 *   path has no such limit.  g > 0 is accepted but is not a decay: the
 *   tensor-core path may then report GDN2_ERR_RANGE.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Identical to cudaStream_t / CUstream. */
struct CUstream_st;
typedef struct CUstream_st *gdn2_stream_t;

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer   */
    GDN2_ERR_UNSUPPORTED = 2,  /* d_k, d_v or chunk outside the supported set  */
    GDN2_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required   */
    GDN2_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed          */
    GDN2_ERR_TIMEOUT = 5,      /* a kernel gave up on a bounded wait            */
    GDN2_ERR_RANGE = 6         /* an fp16 operand of the tensor-core path overflowed */
} gdn2_status;

typedef enum {
    GDN2_IO_F32 = 0,
    GDN2_IO_BF16 = 1
} gdn2_io;

/* Bytes of caller-provided device workspace that gdn2_fwd (for_bwd = 0) or
 * gdn2_fwd followed by gdn2_bwd (for_bwd = 1) needs for these sizes (at
 * least 256).  Returns 0 when the sizes are unsupported.  A workspace sized with for_bwd = 1 also
 * serves gdn2_fwd, and then keeps what gdn2_bwd can reuse (see ws_has_fwd). */
size_t gdn2_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, gdn2_io io,
                            int for_bwd);

/* Chunkwise forward ("Gated DeltaNet-2" LIT-802 review, "Key takeaways" 2;
 * paper Secs. 3.3-3.4 and Apps. A-B: the state is normalised by the
 * cumulative decay so that D_t folds into the two factors of each rank-one
 * erase, and one WY inverse serves the erase and the write side; only the
 * state crosses chunk borders).
 *   q, k, v, g, b, w : inputs (layouts above).
 *   S0  : initial state, or NULL for zero.
 *   o   : output [B, T, H, d_v] in the io type.
 *   ST  : final state, or NULL if not wanted.
 *   ws  : workspace of ws_bytes >= gdn2_workspace_bytes(..., for_bwd = 0).
 *         If ws_bytes >= gdn2_workspace_bytes(..., for_bwd = 1), the call also
 *         leaves in ws what gdn2_bwd reuses with ws_has_fwd = 1. */
gdn2_status gdn2_fwd(const void *q, const void *k, const void *v, const float *g,
                     const float *b, const float *w, const float *S0, void *o, float *ST,
                     void *ws, size_t ws_bytes, int B, int T, int H, int d_k, int d_v,
                     int chunk, gdn2_io io, gdn2_stream_t stream);

/* Gate-aware backward of L = <o, dO> + <S_T, dST> ("Gated DeltaNet-2"
 * LIT-802 review, "Key takeaways" 2: the per-channel gates stay inside the
 * dot products that accumulate dA instead of being pulled outside as a scalar
 * beta would be; digg thread 11/).
 *   q ... S0   : the forward's inputs (S0 may be NULL for zero).
 *   dO  : upstream gradient of o, io type.   dST : of S_T, or NULL for zero.
 *   dq, dk, dv (io type), dg, db, dw (float32) : gradients, same layouts as
 *         the inputs.  dS0 : gradient of S0 (float32), or NULL if not wanted.
 *   ws, ws_bytes >= gdn2_workspace_bytes(..., for_bwd = 1).
 *   ws_has_fwd : 1 if ws holds what gdn2_fwd left there for these same inputs
 *         and sizes (the training pattern: fwd then bwd with one workspace);
 *         0 makes the call recompute it first.  Passing 1 for a workspace that
 *         does not hold the matching forward gives wrong gradients. */
gdn2_status gdn2_bwd(const void *q, const void *k, const void *v, const float *g,
                     const float *b, const float *w, const float *S0, const void *dO,
                     const float *dST, void *dq, void *dk, void *dv, float *dg, float *db,
                     float *dw, float *dS0, void *ws, size_t ws_bytes, int ws_has_fwd,
                     int B, int T, int H, int d_k, int d_v, int chunk, gdn2_io io,
                     gdn2_stream_t stream);

/* One token of the recurrence for N independent sequences ("Gated DeltaNet-2"
 * abstract: linear-time mixing with constant-memory decoding; the update of
 * LIT-802 "Key takeaways" 1):
 *   S <- D S;  delta = w.v - S^T (b.k);  S <- S + k delta^T;  o = S^T q.
 *   q, k, v : [N, H, d] in the io type;  g, b : [N, H, d_k];  w : [N, H, d_v].
 *   S : [N, H, d_k, d_v] float32, read and overwritten in place.
 *   o : [N, H, d_v] in the io type.
 * Needs no workspace. */
gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *b, const float *w, float *S, void *o, int N, int H,
                             int d_k, int d_v, gdn2_io io, gdn2_stream_t stream);

/* Flags or-ed into gate_io (the _ex and _varlen calls): the fused gate
 * prologue.  With GDN2_GATE_LOGITS, g, b and w arrive as pre-activation logits
 * x_g, x_b, x_w and the kernels activate them on load ("Gated DeltaNet-2",
 * LIT-802 review, "Key takeaways" 1: sigmoid erase and write gates, a
 * log-sigmoid decay): g = log sigmoid(x_g), b = sigmoid(x_b), w = sigmoid(x_w);
 * dg, db, dw are then the gradients of the logits.  GDN2_GATE_B_X2 (only with
 * LOGITS) takes b = 2 sigmoid(x_b), erase eigenvalues in [-1, 1] (the review's
 * Table 5).  The chunkwise calls need the tensor-core path for either flag. */
#define GDN2_GATE_LOGITS 0x100
#define GDN2_GATE_B_X2 0x200

/* The same calls with two more choices: the gate tensors' type and grouped
 * value heads.
 *   gate_io : type of g, b, w and of dg, db, dw, or-ed with the GDN2_GATE_*
 *       flags above.  GDN2_IO_F32 without flags gives the calls
 *       above.  GDN2_IO_BF16 halves the gate bytes ("Gated DeltaNet-2"
 *       LIT-802 review, "Key takeaways" 1: b and w are sigmoid gates, values in
 *       (0, 1) or (0, 2), which bf16 holds to 3 significant digits); values
 *       are widened to float32 on load and the gradients rounded once on store.
 *       For the chunkwise calls it needs the tensor-core path (io =
 *       GDN2_IO_BF16, d_k = d_v = 128 after grouping, chunk = 64) and returns
 *       GDN2_ERR_UNSUPPORTED otherwise; the decode step takes it at every size.
 *   H_v : value heads, a multiple of H (H_v = H or 0: one value head per key
 *       head).  The LIT-802 review's "Where the hedges are" gives the write
 *       gate H_v d_v outputs against H d_k for the erase gate: value head
 *       j uses query/key head j / (H_v / H), so q, k, g, b keep H heads and v,
 *       w, o, dO, dv, dw take H_v: [B, T, H_v, d_v]; states are
 *       [B, H_v, d_k, d_v].  The G = H_v / H value heads of one key head evolve
 *       together as one state of G d_v columns, so the chunkwise calls need
 *       G d_v in {32, 64, 128} (and 128 for the tensor-core path); d_v is then
 *       32 or 64.  The decode step takes any d_k, d_v of the supported set.
 * Every other argument, the layouts and the error behaviour are those of the
 * call without the suffix.  The workspace comes from gdn2_workspace_bytes_ex,
 * which also counts two state buffers when H_v > H. */
size_t gdn2_workspace_bytes_ex(int B, int T, int H, int H_v, int d_k, int d_v, int chunk, gdn2_io io,
                               gdn2_io gate_io, int for_bwd);
gdn2_status gdn2_fwd_ex(const void *q, const void *k, const void *v, const void *g, const void *b,
                        const void *w, const float *S0, void *o, float *ST, void *ws,
                        size_t ws_bytes, int B, int T, int H, int H_v, int d_k, int d_v, int chunk,
                        gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream);
gdn2_status gdn2_bwd_ex(const void *q, const void *k, const void *v, const void *g, const void *b,
                        const void *w, const float *S0, const void *dO, const float *dST, void *dq,
                        void *dk, void *dv, void *dg, void *db, void *dw, float *dS0, void *ws,
                        size_t ws_bytes, int ws_has_fwd, int B, int T, int H, int H_v, int d_k,
                        int d_v, int chunk, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream);
gdn2_status gdn2_decode_step_ex(const void *q, const void *k, const void *v, const void *g,
                                const void *b, const void *w, float *S, void *o, int N, int H,
                                int H_v, int d_k, int d_v, gdn2_io io, gdn2_io gate_io,
                                gdn2_stream_t stream);

/* Packed variable-length sequences: N sequences stored back to back along one
 * token axis, each with its own initial and final state (no state crosses from
 * one sequence to the next; the mixer runs inside a language model, whose
 * training packs documents of mixed lengths).
 *   q, k, g, b, dq, dk, dg, db : [1, T, H, d_k];  v, w, o, dO, dv, dw : [1, T, H_v, d_v]
 *   S0, ST, dST, dS0 : [N, H_v, d_k, d_v]
 *   cu_seqlens : device int32 [N + 1]: sequence n holds tokens cu_seqlens[n]
 *       .. cu_seqlens[n + 1] - 1.  It must rise from 0 to T (a sequence may be
 *       empty: its S_T is S0).  The table is read on the device only (the call
 *       does not synchronise): a table that breaks this rule makes the call
 *       treat every sequence as empty and records GDN2_ERR_INVALID_ARG in the
 *       device status word.  4-byte alignment suffices.
 *   N : 1 .. 65535 sequences.
 * Tensor-core path only: io = GDN2_IO_BF16, d_k = 128, G d_v = 128, chunk = 64,
 * gate_io and H_v as for the _ex calls; other sizes return
 * GDN2_ERR_UNSUPPORTED.  Chunks never cross a sequence boundary: a sequence of
 * length L takes ceil(L / 64) chunks, the last one short.
 * Workspace: gdn2_workspace_bytes_varlen (for_bwd as for gdn2_workspace_bytes,
 * sized for the worst case of N sequences over T tokens); it also holds the
 * chunk table the call derives from cu_seqlens.  ws_has_fwd as for gdn2_bwd,
 * with the same cu_seqlens. */
size_t gdn2_workspace_bytes_varlen(int N, int T, int H, int H_v, int d_k, int d_v, int chunk,
                                   gdn2_io io, gdn2_io gate_io, int for_bwd);
gdn2_status gdn2_fwd_varlen(const void *q, const void *k, const void *v, const void *g,
                            const void *b, const void *w, const float *S0, void *o, float *ST,
                            void *ws, size_t ws_bytes, const int *cu_seqlens, int N, int T, int H,
                            int H_v, int d_k, int d_v, int chunk, gdn2_io io, gdn2_io gate_io,
                            gdn2_stream_t stream);
gdn2_status gdn2_bwd_varlen(const void *q, const void *k, const void *v, const void *g,
                            const void *b, const void *w, const float *S0, const void *dO,
                            const float *dST, void *dq, void *dk, void *dv, void *dg, void *db,
                            void *dw, float *dS0, void *ws, size_t ws_bytes, int ws_has_fwd,
                            const int *cu_seqlens, int N, int T, int H, int H_v, int d_k, int d_v,
                            int chunk, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream);

/* Bytes of the scratch array behind gdn2_fwd_noalloc (64 MiB). */
#define GDN2_NOALLOC_SCRATCH_BYTES (64u << 20)

/* gdn2_fwd without a workspace argument, for callers that cannot allocate
 * device memory.  The pages have no counterpart; it is a deployment aid.
 * Examples: a plugin handed only input and output pointers by a host framework
 * whose allocator owns all device memory, or a latency-critical path where the
 * implicit device synchronisation of cudaMalloc/cudaFree is unacceptable.
 * It computes the same forward as gdn2_fwd on the float32 CUDA-core path, and
 * takes the same arguments minus ws and ws_bytes.
 * Scratch: a file-scope device array of GDN2_NOALLOC_SCRATCH_BYTES, held by
 *   every GPU that loads this library until the process exits.  The call
 *   never calls cudaMalloc, cudaFree or any allocating routine.
 * Limit: problems whose float32-path workspace,
 *   gdn2_workspace_bytes(B, T, H, d_k, d_v, chunk, GDN2_IO_F32, 0), exceeds
 *   GDN2_NOALLOC_SCRATCH_BYTES are rejected with GDN2_ERR_WORKSPACE before
 *   anything is enqueued (e.g. d_k = d_v = 128, chunk 64: B*H*chunks up to
 *   292), whatever the io type.
 * Set-up: every call looks up the array's device address in the calling
 *   thread's current context (the current device must be the stream's
 *   device); the lookup allocates nothing, and no address is kept between
 *   calls, so a call after cudaDeviceReset never uses a stale address.  The
 *   first call in a context also loads the library's device code there: make
 *   that first call before any stream capture.
 * Sharing: all calls use the same array, and it keeps the last call's
 *   contents.  Calls whose work overlaps on the GPU (other streams, other
 *   threads) race on it; serialise them. */
gdn2_status gdn2_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                             const float *b, const float *w, const float *S0, void *o, float *ST,
                             int B, int T, int H, int d_k, int d_v, int chunk, gdn2_io io,
                             gdn2_stream_t stream);

/* Returns and clears the device status word once the work enqueued on
 * `stream` before this call has run: GDN2_OK, or the first error a kernel
 * recorded since the word was last read (GDN2_ERR_TIMEOUT, GDN2_ERR_RANGE).
 * The word is read and cleared in one atomic step by a one-thread kernel on
 * `stream`, and the call then waits for `stream`.
 * There is ONE status word per device, shared by every stream and thread of
 * the process: an error recorded by a call on one stream is reported to
 * whichever caller reads the word next, and work still running on other
 * streams may record an error after this call returns.  Callers that need
 * per-call attribution serialise their calls, or read the status after
 * synchronising the device.
 * Returns GDN2_ERR_CUDA if the stream reports a CUDA error. */
gdn2_status gdn2_get_device_status(gdn2_stream_t stream);

/* Self-test of the bounded-wait path every kernel uses.  Enqueues one block
 * on `stream` that waits on an mbarrier nothing will complete, gives up after
 * about `limit_cycles` SM clocks (clamped to [1e3, 4e9]) and records
 * GDN2_ERR_TIMEOUT in the device status word, as a kernel whose copy or
 * product never arrives does.  No copy or product is in flight when it
 * returns, and the context stays usable; the next gdn2_get_device_status
 * reports the timeout and clears it.  Returns GDN2_ERR_CUDA if the launch
 * fails.  Not tied to any entry in the pages. */
gdn2_status gdn2_selftest_timeout(long long limit_cycles, gdn2_stream_t stream);

/* Static, never NULL. */
const char *gdn2_status_string(gdn2_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int gdn2_version(void);

/* Number of kernels this library has enqueued in the calling process since it
 * was loaded (all threads, all devices).  A diagnostic for counting launches
 * around a region of work; not tied to any entry in the pages. */
unsigned long long gdn2_kernel_launches(void);

/* Per-kernel device timing, for benchmarks.  While enabled, every kernel the
 * library launches is bracketed by two CUDA events recorded on its launch
 * stream; gdn2_kernel_times waits for them and adds each kernel's elapsed
 * time to a per-kernel total.  Enabling resets the totals.  Not tied to any
 * entry in the pages. */
void gdn2_set_kernel_timer(int enable);
/* Number of kernel kinds the library can launch. */
int gdn2_kernel_kinds(void);
/* Static name of kernel kind `id`, or NULL. */
const char *gdn2_kernel_name(int id);
/* Waits for the recorded events, then writes for kind i < n the launches
 * counted (count[i]) and their summed device time in milliseconds (ms[i]).
 * Returns GDN2_ERR_CUDA if an event query fails. */
gdn2_status gdn2_kernel_times(unsigned long long *count, double *ms, int n);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
