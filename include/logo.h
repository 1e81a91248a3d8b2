/*
 * logo.h -- C ABI of the B200 (sm_100a) library for the forward (prefill)
 * pass of token-level dynamic local-global attention (LoGo / L2A).
 *
 * What the library computes, and where the pages define it:
 *   - "LoGo: Token-Level Dynamic Local-Global Attention", Abstract: a layer
 *     couples a windowed branch, computed for every token, with a
 *     whole-prefix branch that a gate switches on token by token; the share
 *     of switched-on tokens is held at a set value; the kernels skip the
 *     global work of the other queries.
 *   - "Learning When to Attend", "The Architecture of Conditional Attention":
 *     windowed attention for all positions, and exact softmax attention over
 *     everything before a position only at the routed positions (about one
 *     in five).
 *   - "Local-global attention", Variants, Gemma 2: attention is causal and the
 *     windowed kind ignores keys further back than the window; Implementation
 *     sketch notes, "Packed examples (LongT5)": sequences packed together
 *     must not see each other.
 * Readings of what the pages leave open (fixed here, identical in every entry
 * point):
 *   - window: query i attends to key j iff 0 <= i - j < W;
 *   - budget: k_s = logo_num_selected(ratio, L_s) tokens per sequence, the k_s
 *     largest gate logits, equal logits broken toward the lower position,
 *     -0 equal to +0, NaN ranked below -inf; one selection per sequence,
 *     shared by every head;
 *   - global branch: exact causal attention over positions 0..i;
 *   - merge: o_i = local_i + sigmoid(g_i) * global_i on selected rows,
 *     o_i = local_i elsewhere;
 *   - GQA: query head h reads key/value head h / (Hq / Hkv);
 *   - softmax scale: 1/sqrt(d) when `scale` <= 0.
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns every buffer and the stream.  The library
 *     allocates no memory and never synchronises, except logo_check
 *     (logo_forward_host creates, once per device, two internal streams and a
 *     few events for its copy pipeline).  Every call is asynchronous on
 *     `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Device pointers: q, k, v, out, gate, sel_idx, cu_sel, cu_seqlens and ws
 *     are device (HBM) pointers on the current device, 16-byte aligned,
 *     contiguous in the stated layout (logo_forward_host takes host buffers).
 *   - Element types: q, k, v, out are bf16 (passed as raw 16-bit patterns);
 *     gate is fp32; indices are int32.
 *   - Errors: argument problems are reported synchronously as a logo_status
 *     before anything is launched.  Problems found on the device (a bounded
 *     wait that ran out) are recorded in a status word inside the workspace;
 *     logo_check reads it back.
 *   - Supported shapes: d in {64, 128}; Hq % Hkv == 0; W >= 1;
 *     0 <= ratio <= 1; sequence lengths < 2^31.
 */
#ifndef LOGO_H_
#define LOGO_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LOGO_API __attribute__((visibility("default")))
#else
#define LOGO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LOGO_OK = 0,
    LOGO_ERR_INVALID_ARG = 1,    /* a pointer, size or value is out of the supported range */
    LOGO_ERR_UNSUPPORTED = 2,    /* a shape this build does not implement (e.g. d = 96) */
    LOGO_ERR_WORKSPACE = 3,      /* workspace missing or smaller than logo_workspace_size() */
    LOGO_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed (see logo_last_error) */
    LOGO_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out (read by logo_check) */
    LOGO_ERR_CAPACITY = 6,       /* more tokens passed a threshold than the output holds (read by logo_check) */
    LOGO_ERR_BOUNDS = 7          /* debug build (LOGO_DEBUG_BOUNDS) only: a kernel's index check failed and
                                    the access was skipped (read by logo_check) */
} logo_status;

/* Raw bf16 bit pattern. */
typedef uint16_t logo_bf16;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA headers. */
typedef void *logo_stream_t;

/*
 * Problem geometry.
 * Fixed length (cu_seqlens == NULL): B sequences of L tokens; q is
 *   [B, Hq, L, d], k and v are [B, Hkv, L, d], gate is [B, L], out is
 *   [B, Hq, L, d]; nseq and max_seqlen are ignored.
 * Packed varlen (cu_seqlens != NULL): B must be 1 and L is the total token
 *   count T; sequence s occupies rows cu_seqlens[s] .. cu_seqlens[s+1]-1 of
 *   every head slab of q/k/v/out and of gate; nseq >= 1 sequences;
 *   cu_seqlens is a DEVICE int32 array of nseq+1 non-decreasing offsets with
 *   cu_seqlens[0] == 0 and cu_seqlens[nseq] <= T; max_seqlen must be >= every
 *   sequence length (it sizes the launch).  No attention crosses a sequence
 *   boundary; positions, the window and the budget are per sequence.
 */
typedef struct {
    int B, Hq, Hkv, L, d;
    const int32_t *cu_seqlens;
    int nseq;
    int max_seqlen;
} logo_shape;

/*
 * Budget count for one sequence ("LoGo", Abstract: the share of tokens on the
 * global branch is held at a set value):
 * k = ceil(ratio * len), computed in double; a product within 1e-9
 * (relative, absolute at least 1e-9) of an integer is taken as that integer,
 * so 0.07 * 100 gives 7, not 8.  Clamped to [0, len].  Host function; never
 * fails (ratio <= 0 or NaN gives 0).
 */
LOGO_API int64_t logo_num_selected(double ratio, int64_t len);

/*
 * Bytes of device workspace the calls below need for `shape` at `ratio`
 * (0 if the shape is invalid).  The workspace holds the device status word;
 * it must be zeroed once with logo_workspace_init before first use and may be
 * reused by every later call on the same stream.
 */
LOGO_API size_t logo_workspace_size(const logo_shape *shape, double ratio);

/* Zero the workspace's status word (asynchronous, on `stream`). */
LOGO_API logo_status logo_workspace_init(void *ws, size_t ws_bytes, logo_stream_t stream);

/*
 * Budget rule ("LoGo", Abstract; "Learning When to Attend", "The Architecture
 * of Conditional Attention"): per sequence, select the k_s =
 * logo_num_selected(ratio, L_s) positions with the largest gate logits
 * (ties to the lower position, -0 == +0, NaN below -inf) and write them in
 * ascending order.
 *   gate     [B, L] fp32 (device), or [1, T] packed.
 *   sel_idx  output, int32 (device): the lists of all sequences back to back;
 *            capacity sum_s k_s (fixed length: B * k with row b at b * k).
 *            Entries are positions within their sequence (0-based).
 *   cu_sel   output, int32 [nseq + 1] (device; nseq = B for fixed length):
 *            cu_sel[s] is where sequence s's list starts, cu_sel[nseq] the total.
 * Bit-exact: the result is a pure function of the logits' bit patterns.
 */
LOGO_API logo_status logo_select(const float *gate, const logo_shape *shape, double ratio, int32_t *sel_idx,
                        int32_t *cu_sel, void *ws, size_t ws_bytes, logo_stream_t stream);

/*
 * Threshold form of the budget rule ("LoGo", Abstract: the budget is kept by
 * a controller that moves a threshold on the gate, not by a fixed count).
 * Per sequence, select the positions whose logit is strictly greater than
 * *tau (never a NaN logit; nothing when *tau is NaN; -0 equals +0), ascending.
 *   tau           device pointer to one fp32 threshold (e.g. kept by
 *                 logo_threshold_update).
 *   max_selected  per-sequence capacity; a sequence with more tokens above the
 *                 threshold keeps its lowest max_selected positions and the
 *                 status word records it (logo_check: LOGO_ERR_CAPACITY).
 *   sel_idx       output, int32 (device), capacity nseq * max_selected; the
 *                 lists of all sequences back to back.
 *   cu_sel        output, int32 [nseq + 1] (device) offsets into sel_idx.
 * The workspace holds the per-sequence counts (logo_workspace_size covers them).
 * The lists feed logo_global_attn_sparse with the same max_selected.
 */
LOGO_API logo_status logo_select_threshold(const float *gate, const logo_shape *shape, const float *tau,
                                           int max_selected, int32_t *sel_idx, int32_t *cu_sel, void *ws,
                                           size_t ws_bytes, logo_stream_t stream);

/*
 * One step of the threshold controller ("LoGo", Abstract: a threshold-based
 * controller holds the share of global tokens at a target without auxiliary
 * losses).  Over all n logits of the batch (B * L, or cu_seqlens[nseq] when
 * packed) with k = logo_num_selected(ratio, n), the target q is the (k+1)-th
 * largest logit in the selection order (so, without ties, exactly k logits
 * lie above it); q = -inf when k = n or when that place holds a NaN.  Then, in
 * fp32 with a rounding after each operation, *tau = *tau + beta * (q - *tau),
 * or *tau = q when either is not finite (beta = 1 jumps to the target).
 *   tau     device pointer to one fp32 threshold, read and written.
 *   target  device pointer receiving q, or NULL.
 * One 1024-thread CTA runs the radix select over the whole batch.
 */
LOGO_API logo_status logo_threshold_update(const float *gate, const logo_shape *shape, double ratio, float beta,
                                           float *tau, float *target, void *ws, size_t ws_bytes,
                                           logo_stream_t stream);

/*
 * Local branch for every query ("LoGo", Abstract: the windowed branch runs
 * for every token; "Learning When to Attend": each position looks back over
 * a window of fixed size; "Local-global attention", Gemma 2 variant: causal,
 * keys further back than the window ignored): out[b, h, i] = softmax_j(scale * q_i . k_j) v_j over keys j of
 * the same sequence with 0 <= i - j < W.  With W >= L this is dense causal
 * attention.  q, k, v, out as in logo_shape; `scale` <= 0 means 1/sqrt(d).
 */
LOGO_API logo_status logo_local_attn(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v,
                            const logo_shape *shape, int window, float scale, logo_bf16 *out, void *ws,
                            size_t ws_bytes, logo_stream_t stream);

/*
 * Global branch on the selected queries only, and the gated merge ("Learning
 * When to Attend", "The Architecture of Conditional Attention": exact softmax
 * attention over everything before a position, run only at the routed
 * positions; "LoGo", Abstract: kernels that skip the global work of the other
 * queries).  For every selected position i of sequence s (from sel_idx /
 * cu_sel, as written by logo_select) and every query head h:
 *   global = softmax_j(scale * q_i . k_j) v_j over keys 0..i of sequence s;
 *   merge != 0: out[i] = out[i] + sigmoid(gate[i]) * global  (out must hold
 *               the local branch, e.g. from logo_local_attn);
 *   merge == 0: out[i] = global.
 * Rows that are not selected are not touched.  `max_selected` is an upper
 * bound on every sequence's count cu_sel[s+1] - cu_sel[s] (for lists written
 * by logo_select: logo_num_selected(ratio, longest sequence)); it sizes the
 * launch, and counts above it are an error the kernel reports in the status
 * word.  sel_idx entries must be strictly ascending within a sequence and in
 * [0, L_s).  The kernel checks what it reads: a 128-row chunk of a list whose
 * first or last entry lies outside [0, L_s) is skipped whole, and an entry
 * that is not above the one before it (or outside its chunk's range) is
 * skipped alone; either sets LOGO_ERR_INVALID_ARG in the status word
 * (logo_check) and writes nothing for the skipped rows.  A negative
 * cu_sel[s] or a decreasing cu_sel is reported the same way.  What the kernel
 * cannot see is the capacity of sel_idx: cu_sel must not point past it.
 */
LOGO_API logo_status logo_global_attn_sparse(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v,
                                    const float *gate, const int32_t *sel_idx, const int32_t *cu_sel,
                                    const logo_shape *shape, int max_selected, float scale, int merge,
                                    logo_bf16 *out, void *ws, size_t ws_bytes, logo_stream_t stream);

/*
 * The whole forward pass: logo_select, logo_local_attn, then
 * logo_global_attn_sparse with merge, in that order on `stream`.
 * out receives o; sel_idx / cu_sel receive the selection.
 */
LOGO_API logo_status logo_forward(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v, const float *gate,
                         const logo_shape *shape, int window, double ratio, float scale, logo_bf16 *out,
                         int32_t *sel_idx, int32_t *cu_sel, void *ws, size_t ws_bytes,
                         logo_stream_t stream);

/*
 * The same forward pass with the tensors in HOST memory (the call a user with
 * data on the host makes).  Computes exactly what logo_forward computes, with
 * the same kernels, one key/value-head group at a time: the gate is copied in
 * and the selection made once; then, per group, its Q, K and V rows are copied
 * into a device slot, the local and global kernels run on them, and its output
 * rows are copied back, the copies of neighbouring groups overlapping the
 * kernels (three rotating slots, two internal streams joined back to `stream`).
 *   q, k, v, gate, out: host buffers with logo_forward's layouts (page-locked
 *     memory lets the copies run asynchronously; pageable memory still works).
 *   shape: as for logo_forward, except that shape->cu_seqlens, when given, is a
 *     HOST array of nseq + 1 offsets.
 *   sel_idx, cu_sel: host buffers receiving the selection (nseq * k_max int32
 *     with k_max = logo_num_selected(ratio, max_seqlen), lists back to back as in
 *     logo_select, and nseq + 1 offsets), or NULL.
 *   dev_buf: a device arena of logo_forward_host_buffer_size(shape, ratio)
 *     bytes, 16-byte aligned, owned by the caller; its first bytes are the
 *     workspace: initialise it once with logo_workspace_init(dev_buf, ...) and
 *     read the device status with logo_check(dev_buf, stream).
 * Asynchronous: returns once everything is queued; `stream` completes after the
 * last output copy, so synchronise it before reading out/sel_idx/cu_sel or
 * reusing the inputs.  Calls are serialised by an internal lock.  Errors: the
 * argument errors of logo_forward, LOGO_ERR_WORKSPACE for a missing or small
 * arena, LOGO_ERR_CUDA when a copy, stream or event call fails (the stream is
 * then left partly queued: synchronise the device before reuse).
 */
LOGO_API size_t logo_forward_host_buffer_size(const logo_shape *shape, double ratio);
LOGO_API logo_status logo_forward_host(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v,
                                       const float *gate, const logo_shape *shape, int window, double ratio,
                                       float scale, logo_bf16 *out, int32_t *sel_idx, int32_t *cu_sel,
                                       void *dev_buf, size_t dev_buf_bytes, logo_stream_t stream);

/*
 * The same computation as logo_global_attn_sparse (same arguments, same
 * results) for callers that cannot allocate device memory: a layer that only
 * receives the op's tensors from a framework whose allocator owns the device
 * (and cannot ask it for a workspace), or a serving loop where cudaMalloc /
 * cudaFree would synchronise the device.  No counterpart in the pages: it is
 * a property of this library's interface.
 * Scratch: instead of a caller workspace, a fixed 256 KiB array compiled into
 * the library, held on every GPU that loads the library until exit.  Shapes
 * whose workspace (logo_workspace_size at ratio 1) exceeds it are refused with
 * LOGO_ERR_WORKSPACE.  The first call on a device looks the array's address up
 * (once per device, with that device current) and remembers the context it
 * belongs to; after a device reset (a new primary context) the next call looks
 * it up again.  Make the first call, and the first call after a reset, before
 * any stream capture.  All calls on a device share the array; each call clears its
 * status word first, and calls that overlap on the GPU race on it.  Device
 * errors of a call are recorded there but cannot be read back: use
 * logo_global_attn_sparse and logo_check when that report is needed.  This
 * entry point calls no cudaMalloc / cudaFree or allocating library routine.
 */
LOGO_API logo_status logo_global_attn_sparse_noalloc(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v,
                                                     const float *gate, const int32_t *sel_idx, const int32_t *cu_sel,
                                                     const logo_shape *shape, int max_selected, float scale, int merge,
                                                     logo_bf16 *out, logo_stream_t stream);

/*
 * Decode step ("Learning When to Attend", "Empirical Validation and System
 * Optimization": the gains carry over to time-to-first-token and generation;
 * "LoGo", Abstract: per-token gate with a threshold controller).  One new
 * query token per sequence b, at position t = cache_len[b] - 1 of its cache
 * (its key and value already written there):
 *   local  = softmax attention over positions max(0, t - W + 1) .. t;
 *   global = softmax attention over 0 .. t, computed only when gate[b] > *tau
 *            (the threshold form of the budget rule; never for NaN);
 *   out    = local + sigmoid(gate[b]) * global, or local.
 * Cache positions before the window are read only for tokens that take the
 * global branch.
 *   q        [B, Hq, d] bf16;  k_cache, v_cache [B, Hkv, Lmax, d] bf16 with
 *            shape->L = Lmax (cu_seqlens must be NULL);  cache_len int32 [B]
 *            (device, 0 <= cache_len <= Lmax; 0 gives a zero output; a
 *            larger value reads nothing, gives a zero output and is reported
 *            by logo_check as LOGO_ERR_INVALID_ARG);
 *            gate fp32 [B];  tau one fp32 (device);  out [B, Hq, d] bf16;
 *            selected int32 [B] (device; 1 iff gate[b] > *tau, the gate's
 *            decision even for an empty cache) or NULL.
 *   Hq / Hkv must be 1, 2, 4 or 8.  The workspace must hold
 *   logo_decode_workspace_size(shape) bytes (partial softmax states).
 */
LOGO_API size_t logo_decode_workspace_size(const logo_shape *shape);
LOGO_API logo_status logo_decode(const logo_bf16 *q, const logo_bf16 *k_cache, const logo_bf16 *v_cache,
                                 const int32_t *cache_len, const float *gate, const float *tau,
                                 const logo_shape *shape, int window, float scale, logo_bf16 *out,
                                 int32_t *selected, void *ws, size_t ws_bytes, logo_stream_t stream);

/*
 * Training forward: logo_forward plus what the backward pass needs ("LoGo",
 * Abstract, and "Learning When to Attend", "Empirical Validation and System
 * Optimization": the gate is learned with the model and the kernels are
 * claimed to speed up training).  Same arguments and results as logo_forward,
 * and in addition (all device, caller-owned, overwritten):
 *   sel_capacity  rows the selection list may hold (>= cu_sel[nseq]; the
 *                 row stride of lse_sel and glob; a larger selection is an
 *                 error the kernels report in the status word);
 *   lse      fp32 [B*Hq][L]: per row, log2 of the local softmax's normaliser
 *            in the scaled-score exp2 domain (m * scale * log2(e) + log2(sum));
 *            rows of a packed tensor that lie in no sequence are not written;
 *   lse_sel  fp32 [Hq][sel_capacity]: the same for the global softmax of each
 *            selected row (row r of the selection list, all sequences);
 *   glob     bf16 [Hq][sel_capacity][d]: the global branch of each selected
 *            row before the gate;
 *   loc_sel  bf16 [Hq][sel_capacity][d]: the local branch of each selected
 *            row (its value before the merge).
 */
LOGO_API logo_status logo_forward_train(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v, const float *gate,
                                        const logo_shape *shape, int window, double ratio, float scale,
                                        logo_bf16 *out, int32_t *sel_idx, int32_t *cu_sel, int sel_capacity,
                                        float *lse, float *lse_sel, logo_bf16 *glob, logo_bf16 *loc_sel, void *ws,
                                        size_t ws_bytes, logo_stream_t stream);

/*
 * Backward pass: gradients of a scalar loss given dout = dL/d(out), for the
 * forward pass logo_forward_train ran on the same q, k, v, gate, shape,
 * window and scale.  The pages print no backward formulas; this is the chain
 * rule through the forward definition, with the reading that out depends on
 * gate[i] only through sigmoid(gate[i]) on selected rows (the selection is a
 * step function and passes no gradient):
 *   dgate[i] = sigmoid'(gate[i]) * sum_h <dout[h,i], global[h,i]> on selected
 *              rows, 0 on every other row;
 *   dq, dk, dv  through both softmax branches, the global one with upstream
 *              gradient sigmoid(gate[i]) * dout[h,i]; dk and dv sum over the
 *              query heads of a GQA group.
 * Inputs: q, k, v, gate, out (the forward's output), dout [B, Hq, L, d] bf16;
 * sel_idx, cu_sel, sel_capacity, lse, lse_sel, glob, loc_sel as the forward left them;
 * max_selected bounds every sequence's count (as for logo_global_attn_sparse).
 * Outputs (device, overwritten): dq [B, Hq, L, d], dk, dv [B, Hkv, L, d] bf16,
 * dgate [B*L] fp32.  Rows of a packed tensor that lie in no sequence are left
 * as they were in dq, dk and dv.  The workspace must hold
 * logo_backward_workspace_size(shape, sel_capacity) bytes.
 */
LOGO_API size_t logo_backward_workspace_size(const logo_shape *shape, int sel_capacity);
LOGO_API logo_status logo_backward(const logo_bf16 *q, const logo_bf16 *k, const logo_bf16 *v, const float *gate,
                                   const logo_bf16 *out, const logo_bf16 *dout, const int32_t *sel_idx,
                                   const int32_t *cu_sel, int sel_capacity, int max_selected, const float *lse,
                                   const float *lse_sel, const logo_bf16 *glob, const logo_bf16 *loc_sel,
                                   const logo_shape *shape, int window, float scale, logo_bf16 *dq, logo_bf16 *dk,
                                   logo_bf16 *dv, float *dgate, void *ws, size_t ws_bytes, logo_stream_t stream);

/*
 * Synchronise `stream`, then report: LOGO_ERR_CUDA if a launch or the stream
 * failed, LOGO_ERR_DEVICE_TIMEOUT if a kernel recorded a bounded wait that ran
 * out, LOGO_ERR_INVALID_ARG if a kernel recorded an argument it could not
 * handle, else LOGO_OK.  The only entry point that blocks the host.
 */
LOGO_API logo_status logo_check(const void *ws, logo_stream_t stream);

/*
 * Diagnostic: launch one tiny kernel that waits on a barrier nothing will
 * complete, with a bound of `limit_us` microseconds; when the bound runs out
 * it records a timeout in the workspace status word and returns normally
 * (no trap, no fault).  logo_check then reports LOGO_ERR_DEVICE_TIMEOUT.
 * Used by the tests of the timeout path.
 */
LOGO_API logo_status logo_selftest_timeout(void *ws, size_t ws_bytes, unsigned limit_us, logo_stream_t stream);

/* Static text for a status code. */
LOGO_API const char *logo_status_string(logo_status status);

/* Details of the last error raised on the calling host thread ("" if none). */
LOGO_API const char *logo_last_error(void);

/* How this library was built: bit 0 (LOGO_BUILD_DEBUG_BOUNDS) is set in the
 * debug build whose kernels check every TMA coordinate, gathered row and
 * stored row before the access (make debug: liblogo_debug.so). */
#define LOGO_BUILD_DEBUG_BOUNDS 1u
LOGO_API unsigned logo_build_flags(void);

#ifdef __cplusplus
}
#endif

#endif /* LOGO_H_ */
