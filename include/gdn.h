/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated-delta-rule library, libgdn.so.
 *
 * The operation.  Ferrite project page (bhcc2025.github.io/ferrite), Design section 03 "Chunked
 * Gated DeltaNet": the section names the method -- each linear-attention layer holds a recurrent
 * state for every request, a prompt is processed 32 rows at a time with the WY/UT chunk form of the
 * delta rule, its products on TF32 tensor cores (three-way TF32 splitting for fp32-level
 * accuracy), and the state left at the end of the prompt is what the decoder continues from.  The
 * state recurrence is the gated delta rule (Yang, Kautz and Hatamizadeh, "Gated Delta Networks"), per
 * sequence and head:
 *
 *     S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T      (S is dv x dk)
 *     o_t = S_t q_t / sqrt(dk)
 *
 * q_t and k_t must already be L2-normalised; the library does not normalise them.  g_t is the
 * log-gate (alpha_t = exp(g_t); g <= 0 is the intended range but is not enforced); beta_t is used
 * as given (intended range (0, 1), not enforced).
 *
 * Layouts (all row-major, contiguous, innermost index last):
 *     q, k        [T_total, H, dk]     dtype GDN_F32 or GDN_BF16
 *     v, out      [T_total, H, dv]     same dtype as q (out is written in that dtype)
 *     g, beta     [T_total, H]         fp32
 *     state       [N, H, dv, dk]       fp32 (dk contiguous: one row of S per dv index)
 *     cu_seqlens  int32 [N + 1]        cu[0] = 0, non-decreasing, cu[N] = T_total
 *
 * Conventions shared by every entry point.
 *   - Pointers named "device" must be device memory of the current CUDA device (or managed
 *     memory).  q, k, v, out and state pointers must be 16-byte aligned, g, beta and cu_seqlens
 *     4-byte aligned (GDN_ERR_MISALIGNED otherwise).
 *   - The caller owns every buffer; the library never allocates device memory in these calls.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All work is
 *     enqueued on it; no call synchronises the host except gdn_get_device_status.  Within a call,
 *     and from one call to the next, kernels are launched as programmatic dependents of the
 *     kernel before them: each waits on the device for its predecessor to complete before reading
 *     anything.  A caller kernel launched after a call with the programmatic-serialisation launch
 *     attribute must likewise wait (griddepcontrol.wait) before reading the call's results; a
 *     normal launch needs nothing.
 *   - Return value: GDN_OK (0) when the work was enqueued, a negative GDN_ERR_* otherwise (nothing
 *     is enqueued then).  Errors the host cannot see (bad cu_seqlens contents, an expired bounded
 *     wait) are recorded by the kernels in a per-device status word; read it with
 *     gdn_get_device_status.  Kernels never trap.
 *   - Supported head sizes: dk, dv in {64, 128}.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage type of q, k, v and out. */
typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype_t;

/*
 * Flag that may be OR'ed into the `dtype` argument of every call that takes q and k: they are
 * passed raw and the library L2-normalises each (token, head) vector, x / max(||x||_2, 1e-12) with
 * the norm summed in fp32, and rounds the result to the storage dtype before use.  The prefill
 * writes the normalised copies into its workspace (see gdn_chunk_prefill_workspace_bytes_ex);
 * decode and verify normalise in registers.  Without the flag q and k must arrive normalised
 * (the method's definition) and are used as given.
 */
#define GDN_QK_L2NORM 0x100

/* Status codes. */
enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = -1,  /* null required pointer, H < 1, N < 1, T < 0, bad dtype         */
    GDN_ERR_UNSUPPORTED = -2,  /* dk or dv not in {64, 128}                                     */
    GDN_ERR_MISALIGNED = -3,   /* a pointer breaks the alignment rule above                     */
    GDN_ERR_LAUNCH = -4,       /* a kernel launch failed (the CUDA error is left pending)        */
    GDN_ERR_WORKSPACE = -5,    /* workspace missing, misaligned (256 B) or smaller than needed   */
    GDN_ERR_BAD_SEQLENS = -6,  /* device-detected: cu_seqlens not 0..T_total non-decreasing, or
                                  cut points not increasing and strictly inside a sequence      */
    GDN_ERR_TIMEOUT = -7,      /* device-detected: a bounded wait inside a kernel expired        */
    GDN_ERR_CUDA = -8,         /* a CUDA runtime call made by the library failed                */
    GDN_ERR_BAD_PARENTS = -9   /* device-detected: a draft-tree parent index is not -1 or an
                                  earlier node of the same sequence                              */
};

/* Human-readable name of a status code (static string, never NULL). */
const char* gdn_status_string(int status);

/*
 * Detail of the last CUDA runtime error that a call of this library met on the calling thread
 * (which runtime call and CUDA's message), e.g. after GDN_ERR_LAUNCH; "" if there was none.  The
 * string belongs to the library and is overwritten by the thread's next failing call.
 */
const char* gdn_last_error(void);

/* Library ABI version (major * 100 + minor). */
int gdn_version(void);

/*
 * Bytes of device workspace that gdn_chunk_prefill needs for this problem size.  Depends only on
 * total_tokens, num_seqs, H and dk (chunk tables, the WY/UT operator and gate data per chunk or
 * pair of chunks), and covers both dtypes.
 * Returns 0 for arguments that gdn_chunk_prefill would reject.
 */
size_t gdn_chunk_prefill_workspace_bytes(int64_t total_tokens, int num_seqs, int H, int dk, int dv);

/*
 * Workspace for any prefill call: num_segments = num_seqs (+ num_cuts for gdn_chunk_prefill_cuts),
 * dtype as passed to the call (with GDN_QK_L2NORM the normalised q and k copies are included).
 * Returns 0 for arguments the calls would reject.
 */
size_t gdn_chunk_prefill_workspace_bytes_ex(int64_t total_tokens, int num_segments, int H, int dk,
                                            int dv, int dtype);

/*
 * Chunked prefill (Ferrite project page, Design section 03): runs the gated delta rule over every
 * token of N packed sequences, chunk size C = 32 with chunk boundaries relative to each sequence's
 * start, and writes every output o_t and each sequence's final state.  With bf16 q/k/v the state is
 * carried once per pair of chunks (64 rows; the pair's operator is built from the two chunks'
 * 32 x 32 inverses); with fp32 q/k/v once per chunk.
 *
 *   q, k, v       device, layouts above, dtype `dtype`
 *   g, beta       device fp32 [T_total, H]
 *   cu_seqlens    device int32 [num_seqs + 1]; NULL means num_seqs sequences of equal length
 *                 total_tokens / num_seqs (GDN_ERR_INVALID_ARG when that does not divide)
 *   num_seqs      N >= 1
 *   total_tokens  T_total >= 0, must equal cu_seqlens[N] (checked on the device)
 *   state_in      device fp32 [N, H, dv, dk] initial states, or NULL for zero states
 *   out           device [T_total, H, dv], dtype `dtype`; must not overlap any input
 *   state_out     device fp32 [N, H, dv, dk] final states, or NULL (not written).  May equal
 *                 state_in (in-place resume); must not overlap any other buffer otherwise.
 *   dtype         GDN_F32 or GDN_BF16, optionally | GDN_QK_L2NORM (raw q, k)
 *   workspace     device scratch of at least gdn_chunk_prefill_workspace_bytes(...) bytes (with
 *                 GDN_QK_L2NORM: gdn_chunk_prefill_workspace_bytes_ex(..., dtype)),
 *                 256-byte aligned; its contents on entry do not matter and are clobbered.  The
 *                 workspace must not be used by another call that runs concurrently.
 *
 * Device-detected errors (GDN_ERR_BAD_SEQLENS) leave out and state_out unwritten.
 */
int gdn_chunk_prefill(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, const int32_t* cu_seqlens, int num_seqs,
                      int64_t total_tokens, const float* state_in, void* out, float* state_out,
                      int H, int dk, int dv, int dtype, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * Chunked prefill with state snapshots at cut points (Ferrite project page, Design section 07: the
 * prompt cache saves a conversation's state where each turn ends, and a prompt is split at identical
 * places whether or not it resumes from such a save).  Same as gdn_chunk_prefill, plus: for every cut point c_i, snapshots[i]
 * receives the state of the sequence that contains c_i after its tokens before c_i.  Chunks restart
 * at every cut, so each snapshot, every output and each final state are bit for bit what a call
 * that stops at c_i and a second call resumed from that state would give.
 *
 *   cuts        device int32 [num_cuts] token offsets into the packed batch, strictly increasing,
 *               each strictly inside one sequence (start < c < end); checked on the device
 *               (GDN_ERR_BAD_SEQLENS, nothing written)
 *   num_cuts    >= 1 (GDN_ERR_INVALID_ARG otherwise; use gdn_chunk_prefill for none)
 *   snapshots   device fp32 [num_cuts, H, dv, dk], 16-byte aligned
 *   workspace   at least gdn_chunk_prefill_workspace_bytes(total_tokens, num_seqs + num_cuts, H,
 *               dk, dv) bytes (a cut adds a segment)
 * Every other argument, and the error behaviour, as gdn_chunk_prefill.
 */
int gdn_chunk_prefill_cuts(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const int32_t* cu_seqlens, int num_seqs,
                           int64_t total_tokens, const int32_t* cuts, int num_cuts,
                           const float* state_in, void* out, float* state_out, float* snapshots,
                           int H, int dk, int dv, int dtype, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * gdn_chunk_prefill without a caller-provided workspace.  The pages have no counterpart to this
 * call; it exists for callers that cannot allocate device memory when they run a prefill -- for
 * example an engine that plans every byte of GPU memory at start-up and forbids cudaMalloc later,
 * or code on a latency-critical path where cudaMalloc/cudaFree could block or synchronise the
 * device.  The call allocates nothing: its scratch is a fixed 64 MiB array inside this library,
 * one per GPU that loads the library, held until the process exits.
 *
 *   Arguments, layouts and results are those of gdn_chunk_prefill minus workspace/workspace_bytes.
 *   Limit: the problem must satisfy gdn_chunk_prefill_workspace_bytes_ex(total_tokens, num_seqs,
 *   H, dk, dv, dtype) <= 64 MiB; larger problems return GDN_ERR_WORKSPACE and enqueue nothing.
 *   The workspace is almost all operator records, one of 49,664 bytes per (pair of chunks, head)
 *   over floor(total_tokens / 64) + num_seqs pairs on the bf16 path, so the scratch holds about
 *   floor(64 MiB / (H x 49,664)) - num_seqs pairs: for H = 32, d = 128 about 2,680 tokens in one
 *   sequence.  With GDN_QK_L2NORM in dtype the normalised q/k copies live in the scratch too, which
 *   lowers the limit (about 1,600 tokens in one sequence at H = 32, d = 128, bf16).
 *   Set-up: the first call on a device looks up that device's copy of the scratch array (a CUDA
 *   runtime query, no allocation).  Make that first call before any stream capture on the device.
 *   Sharing: every call on a device uses the same scratch array and leaves its contents behind
 *   (nothing in it needs to start at zero).  Calls whose execution overlaps on the GPU -- on
 *   different streams, or from different threads -- race on the scratch and give wrong results;
 *   order them (one stream, or events).
 */
int gdn_chunk_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, const int32_t* cu_seqlens, int num_seqs,
                              int64_t total_tokens, const float* state_in, void* out,
                              float* state_out, int H, int dk, int dv, int dtype, void* stream);

/*
 * Recurrent decode step (the consumer of the written-back state, Design section 03): one token for
 * each of B sequences, state updated in place.
 *
 *   q, k          device [B, H, dk], dtype `dtype`
 *   v             device [B, H, dv], dtype `dtype`
 *   g, beta       device fp32 [B, H]
 *   state_inout   device fp32 [B, H, dv, dk]; read once and overwritten with S_t
 *   out           device [B, H, dv] in dtype `dtype`, or NULL (outputs not written)
 */
int gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* state_inout, void* out, int B, int H, int dk, int dv,
                    int dtype, void* stream);

/*
 * Multi-token recurrent verify (Ferrite project page, Design section 04: drafted tokens are checked
 * by the big model in one pass): Tk speculative tokens per sequence run through the recurrence in
 * order, as a linear chain, starting from the committed state, which is only read.  The state after
 * every token is returned, so that the caller keeps the one after the last accepted token (or the
 * committed state when none is accepted) and discards the rest.  Token t of sequence b gives exactly
 * what the t-th of Tk chained gdn_decode_step calls from state_in would give.
 *
 *   q, k          device [B, Tk, H, dk], dtype `dtype`
 *   v             device [B, Tk, H, dv], dtype `dtype`
 *   g, beta       device fp32 [B, Tk, H]
 *   state_in      device fp32 [B, H, dv, dk]; read only
 *   states_out    device fp32 [B, Tk, H, dv, dk]: S after token t at [b, t]; or NULL
 *   out           device [B, Tk, H, dv] in dtype `dtype`, or NULL (at least one of the two)
 *   Tk >= 1.  Memory: states_out holds Tk states per (b, h) (64 KB each at dk = dv = 128).
 *   Errors as gdn_decode_step; GDN_ERR_INVALID_ARG also for Tk < 1 or both outputs NULL.
 *   states_out and out must not alias the inputs.
 */
int gdn_decode_verify(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, const float* state_in, float* states_out, void* out, int B,
                      int Tk, int H, int dk, int dv, int dtype, void* stream);

/*
 * Tree verify (Ferrite project page, Design section 04: the big model checks the drafter's tokens
 * in a single pass, with the drafts arranged as a tree grown best-first).  As gdn_decode_verify, but the Tk drafted tokens of a sequence
 * form a tree: token t continues from the state after token parents[b * Tk + t], which must be an
 * earlier token (< t), or from the committed state when the parent is -1.  A linear chain
 * (parents[b * Tk + t] = t - 1) gives exactly gdn_decode_verify.
 *
 *   parents       device int32 [B, Tk], 4-byte aligned
 *   states_out    device fp32 [B, Tk, H, dv, dk]: S after token t at [b, t] -- required (the tree
 *                 reads a parent's state back from it)
 *   out           device [B, Tk, H, dv] in dtype `dtype`, or NULL
 *   Other arguments and errors as gdn_decode_verify; GDN_ERR_INVALID_ARG also for parents or
 *   states_out NULL.  A parent that is neither -1 nor an earlier token is device-detected: the
 *   token starts from the committed state and gdn_get_device_status reports GDN_ERR_BAD_PARENTS.
 */
int gdn_decode_verify_tree(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const int32_t* parents, const float* state_in,
                           float* states_out, void* out, int B, int Tk, int H, int dk, int dv, int dtype,
                           void* stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of the current device:
 * GDN_OK, or the first device-detected error (GDN_ERR_BAD_SEQLENS, GDN_ERR_TIMEOUT,
 * GDN_ERR_BAD_PARENTS) recorded since
 * the last read.  Returns GDN_ERR_CUDA when the synchronisation itself fails.
 */
int gdn_get_device_status(void* stream);

/*
 * Failure-path self-test (a test aid, not part of the computation): enqueues one kernel whose single
 * waiting thread waits on a barrier that nothing completes.  The bounded wait gives up after about
 * limit_ns nanoseconds, records GDN_ERR_TIMEOUT in the status word and the kernel returns normally,
 * so the next gdn_get_device_status returns GDN_ERR_TIMEOUT and later calls run as usual.
 *   limit_ns in [1e6, 2e9] (GDN_ERR_INVALID_ARG otherwise).
 */
int gdn_selftest_wait_timeout(long long limit_ns, void* stream);

/*
 * Measurement aid (no counterpart on the pages): per-kernel device time of the library's own
 * launches.  After gdn_profile_start, every kernel the library launches (from any host thread) is
 * bracketed by a pair of CUDA events recorded on the launch's stream.  gdn_profile_stop
 * synchronises those events, stops recording and aggregates by kernel name.
 *
 *   gdn_profile_start  GDN_OK, GDN_ERR_INVALID_ARG when already started, GDN_ERR_CUDA on failure.
 *   gdn_profile_stop   returns the number of distinct kernels seen (>= 0) or a negative status;
 *                      fills min(that, max_kernels) entries: names (host char[max_kernels][64],
 *                      NUL-terminated, may be NULL), total_ms (host double[max_kernels], may be
 *                      NULL; summed event time) and launches (host int[max_kernels], may be NULL).
 */
int gdn_profile_start(void);
int gdn_profile_stop(int max_kernels, char* names, double* total_ms, int* launches);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
