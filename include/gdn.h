/*
 * gdn.h -- C ABI of libgdn, the gated delta rule on NVIDIA B200 (sm_100a).
 *
 * The operation (page "Qwen3.8-27B 架构深读: Gated DeltaNet 混合线性注意力与
 * 262K 长上下文", section 三, "Gated DeltaNet: 把注意力变成可读写的记忆"):
 * a fixed-size matrix memory per head that is decayed by a per-token gate and
 * then edited by the delta rule (erase what the key recalls, write the new
 * value), read out by the query.  In the standard step order implemented here
 *
 *     S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t,
 *     a_t = exp(g_t),  b_t = beta_t,
 *
 * i.e. S <- a S; r = S k; S <- S + b (v - r) k^T; o = S q.  The same section
 * says training/prefill accumulates the state chunk-parallel and inference
 * does one fixed-size matrix update per token: gdn_prefill is the former,
 * gdn_decode_step the latter.  Readings of points the page leaves open: the
 * state is Dv x Dk (S k is a Dv-vector); the gate is one scalar per token and
 * v-head, passed as its logarithm g; o_t uses the updated state; there is no
 * 1/sqrt(Dk) scale and no feature map or normalisation inside the operation.
 *
 * Conventions shared by every call
 * --------------------------------
 * Layouts are token-major and packed over sequences, row-major, contiguous:
 *     q, k        [T][Hqk][Dk]        io_dtype
 *     v, o        [T][Hv][Dv]         io_dtype
 *     g, beta     [T][Hv]             fp32  (g finite and <= 0; beta finite)
 *     state       [N][Hv][Dv][Dk]     fp32  (row i of a head's state is S[i,:])
 *     cu_seqlens  [N+1]               int32, cu[0] = 0, non-decreasing, cu[N] = T
 * v-head h reads q/k head h / (Hv / Hqk): groups of Hv/Hqk consecutive v-heads
 * share one q/k head.
 *
 * Ownership: every pointer is a DEVICE pointer owned by the caller, except
 * the host buffers of gdn_prefill_host.  The library allocates no memory,
 * frees nothing and never synchronises; all work is enqueued on `stream` (a
 * cudaStream_t; NULL is the legacy default stream) and completes
 * asynchronously.  (gdn_prefill_host creates and releases two streams and
 * eight events per call, and its copies to or from pageable host memory are
 * synchronous, as CUDA makes them.)  Inputs are only read.  Outputs must not
 * alias inputs, except where stated.  Every pointer must be 16-byte aligned.
 *
 * Errors: argument errors are returned synchronously and nothing is launched.
 * A failed launch returns GDN_ERR_CUDA (cudaGetLastError, no synchronisation).
 * Errors only the device can see (a malformed cu_seqlens, a bounded wait that
 * expired, an fp16 range overflow of a q/k-side operand, a state slot index
 * out of range) are written as a
 * gdn_status value to *dev_error_flag when that
 * optional device int32 is given; the caller zeroes it beforehand and reads it
 * after synchronising.  A unit (sequence, head) that detects such an error
 * writes no output for itself.  No C++ exception crosses this interface.  The
 * calls keep no global mutable state and are safe to call from any thread,
 * except gdn_prefill_static_workspace, whose one scratch array per device is
 * shared by its calls (see its contract).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size, bad enum */
    GDN_ERR_UNSUPPORTED = 2,      /* valid but not implemented (head dims, dtype) */
    GDN_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed */
    GDN_ERR_TIMEOUT = 4,          /* device: a bounded wait expired */
    GDN_ERR_BAD_SEQLENS = 5,      /* device: cu_seqlens malformed */
    GDN_ERR_BAD_SLOT = 6,         /* device: a state slot index out of range */
    GDN_ERR_RANGE = 7             /* device: a q/k-side operand overflowed fp16 (see gdn_prefill) */
} gdn_status;

typedef enum gdn_dtype {
    GDN_DTYPE_BF16 = 0, /* q, k, v, o in bfloat16; o rounded once, to nearest even */
    GDN_DTYPE_F32 = 1   /* q, k, v, o in fp32 */
} gdn_dtype;

/*
 * gdn_prefill -- chunk-parallel prefill/training forward of the gated delta
 * rule over a packed batch of N sequences (section 三 of the page above: for
 * training the state is built up over chunks of tokens in parallel).
 *
 *   q, k, v, io_dtype   token inputs, layouts above.
 *   g, beta             per-token log-decay and write strength, fp32 [T][Hv].
 *   initial_state       fp32 [N][Hv][Dv][Dk] state entering each sequence,
 *                       or NULL for zeros.
 *   cu_seqlens          device int32 [N+1] sequence offsets, or NULL for a
 *                       single sequence (then N must be 1).  Never read on
 *                       the host.  Empty sequences are allowed: their final
 *                       state equals their initial state.
 *   N, T                number of sequences and total tokens (T >= 0).
 *   Hqk, Hv, Dk, Dv     head counts (Hv % Hqk == 0) and head dimensions.
 *   chunk               chunk length of the chunk-parallel form; 0 picks the
 *                       default.  It changes rounding only, never the result.
 *   o                   output [T][Hv][Dv] in io_dtype.
 *   final_state         fp32 [N][Hv][Dv][Dk] state after each sequence, or
 *                       NULL to skip.  May equal initial_state (in place).
 *   workspace, workspace_bytes
 *                       scratch of at least gdn_prefill_workspace_bytes();
 *                       may be NULL when that is 0.
 *   dev_error_flag      optional device int32 (see Errors above).
 *   stream              cudaStream_t.
 *
 * Supported: Dk = Dv = 128 with bf16 I/O and chunk 0 or 64 runs a tensor-core
 * (tcgen05) chunked kernel; every other combination with Dk, Dv in
 * {16, 32, 64, 128} and either dtype runs an exact fp32 token-recurrent CUDA
 * kernel.  Anything else returns GDN_ERR_UNSUPPORTED.  gdn_prefill_ex below
 * selects the kernel explicitly.
 *
 * Value range of the tensor-core kernels.  v, the states and every quantity
 * linear in them (U, the state increments, o) have no range limit beyond
 * fp32's: they enter the fp16 tensor-core operands with a power-of-two scale
 * chosen per chunk from their largest magnitude, so the results scale exactly
 * with v and initial_state (scaling both by 2^s scales o and final_state by
 * 2^s, bit for bit).  q and k, and the per-chunk factors built from k, beta
 * and g (the masked Q K^T, the inverse of the chunk's triangular system times
 * beta, W), are held in fp16 without scaling: an entry that reaches 65520 in
 * magnitude is reported as GDN_ERR_RANGE through dev_error_flag (the results
 * of that call are then unspecified).  q and k entries below 2^-14 in
 * magnitude lose relative precision to fp16 subnormals; rows scaled to unit
 * length, as the gated delta rule is used, are far from both limits.
 */
GDN_API gdn_status gdn_prefill(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                       const float *g, const float *beta, const float *initial_state,
                       const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk, int32_t Hv,
                       int32_t Dk, int32_t Dv, int32_t chunk, void *o, float *final_state,
                       void *workspace, size_t workspace_bytes, int32_t *dev_error_flag,
                       void *stream);

/*
 * Which prefill kernel runs.  For Dk = Dv = 128, bf16 and chunk 0 or 64, AUTO
 * picks the pool kernel when there are at most 64 (sequence, v-head) units
 * (few, long sequences: every SM of the GPU works on them) and the single-CTA
 * kernel otherwise; every other shape runs the exact recurrent kernel.
 * Naming a tensor-core kernel for a shape it does not support returns
 * GDN_ERR_UNSUPPORTED, and so does the pool kernel for more than 64 units.
 * The cluster and pool kernels need a workspace (see below).
 */
typedef enum gdn_prefill_kernel {
    GDN_PREFILL_AUTO = 0,
    GDN_PREFILL_CLUSTER = 1,     /* tcgen05, a 3-CTA cluster per (sequence, head): one CTA
                                    holds the state, two prepare alternate chunks and
                                    hand them over through an L2-resident workspace ring */
    GDN_PREFILL_SINGLE_CTA = 2,  /* tcgen05, one CTA per (sequence, head) */
    GDN_PREFILL_RECURRENT = 3,   /* exact fp32 token recurrence on CUDA cores, any shape */
    GDN_PREFILL_POOL = 4         /* tcgen05, one cooperative launch over every SM: a CTA per
                                    (sequence, head) holds the state, the other CTAs
                                    prepare chunks in chunk-major order and hand them
                                    over through the workspace ring (at most 64 units;
                                    on a GPU with too few SMs it runs as SINGLE_CTA) */
} gdn_prefill_kernel;

/*
 * gdn_prefill_ex -- gdn_prefill with an explicit kernel choice (all other
 * arguments and behaviour as gdn_prefill).  The kernels differ in speed and
 * rounding only; each meets the same tolerances.
 */
GDN_API gdn_status gdn_prefill_ex(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                                  const float *g, const float *beta, const float *initial_state,
                                  const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk,
                                  int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                                  float *final_state, void *workspace, size_t workspace_bytes,
                                  int32_t *dev_error_flag, void *stream, gdn_prefill_kernel kernel);

/*
 * gdn_prefill_workspace_bytes -- scratch bytes gdn_prefill needs for these
 * sizes (0 when none): when AUTO would run the pool kernel, 860,160 bytes per
 * (sequence, v-head) unit plus a flag block of 4 KB or more (the cluster
 * kernel, chosen explicitly, takes 430,080 bytes per unit).  Pure function of its arguments (it cannot see the dtype, so
 * it may ask for a workspace an fp32 call does not use); no device access.
 * The workspace is device memory, 256-byte aligned, owned by the caller; its
 * contents need no initialisation (the pool kernel clears its flag block on
 * the stream before it starts) and are garbage afterwards.  One workspace
 * must not serve two calls that may run at the same time.
 */
GDN_API size_t gdn_prefill_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                   int32_t Dv, int32_t chunk);

/* Scratch bytes gdn_prefill_ex needs with this kernel choice. */
GDN_API size_t gdn_prefill_ex_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv,
                                              int32_t Dk, int32_t Dv, int32_t chunk,
                                              gdn_prefill_kernel kernel);

/*
 * gdn_decode_step -- one-token inference update of N independent sequences,
 * in place on the state (section 三 of the page above: at inference time the
 * state of each head takes one update of constant size per token).
 *
 *   q, k                [N][Hqk][Dk] io_dtype, this step's query and key.
 *   v                   [N][Hv][Dv]  io_dtype.
 *   g, beta             fp32 [N][Hv].
 *   state               fp32 [N][Hv][Dv][Dk], read and overwritten in place.
 *   o                   [N][Hv][Dv] io_dtype output; must not alias anything.
 *   dev_error_flag      optional (this call detects no device-side errors
 *                       today and never writes it).
 * Supported: Dk in {16, 32, 64, 128}, any Dv >= 1, either dtype.
 */
GDN_API gdn_status gdn_decode_step(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                           const float *g, const float *beta, float *state, int32_t N,
                           int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, void *o,
                           int32_t *dev_error_flag, void *stream);

/*
 * gdn_decode_step_bf16_state -- gdn_decode_step for a state that is stored in
 * bfloat16 between steps, which halves the state bytes a decode step moves.
 * The page (section 一, the per-sequence state of the DeltaNet layers) counts
 * that state in fp32 and notes that the byte count follows the runtime dtype;
 * this entry point is that other dtype.
 *
 *   state               bfloat16 [N][Hv][Dv][Dk], read and overwritten in place.
 *   everything else     as gdn_decode_step.
 * Arithmetic: each element is widened to fp32 (exact), the step runs in fp32
 * exactly as in gdn_decode_step, o comes from the fp32 values, and the new
 * state is rounded once to bfloat16, to nearest, ties to even.
 * Supported: Dk = Dv = 128, either io dtype; other head sizes return
 * GDN_ERR_UNSUPPORTED.  Errors and ownership as gdn_decode_step.
 */
GDN_API gdn_status gdn_decode_step_bf16_state(const void *q, const void *k, const void *v,
                                              gdn_dtype io_dtype, const float *g,
                                              const float *beta, void *state, int32_t N,
                                              int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv,
                                              void *o, int32_t *dev_error_flag, void *stream);

/*
 * gdn_prefill_static_workspace -- gdn_prefill_ex with kernel
 * GDN_PREFILL_CLUSTER, but the cluster kernel's workspace ring lives in a
 * fixed device array inside libgdn, so the call allocates nothing and takes
 * no workspace argument.  The paper has no counterpart to this entry point; it exists
 * for callers that cannot hand out device memory at call time: a host program
 * that links only this C ABI and has no device allocator of its own, or a
 * runtime whose device memory is planned once up front and may not grow or be
 * carved up per call.
 *
 * All other arguments, layouts and results are those of gdn_prefill_ex; the
 * results are bit-identical to gdn_prefill_ex(..., GDN_PREFILL_CLUSTER) with
 * a caller-supplied workspace.
 *
 * Limit: N * Hv <= GDN_STATIC_WORKSPACE_MAX_UNITS (48 units, a 20,643,840-byte
 * array, 430,080 bytes per unit).  Larger calls return GDN_ERR_UNSUPPORTED
 * before any CUDA call; use gdn_prefill_ex with a workspace for them.
 * Shapes the cluster kernel does not take (not bf16, Dk or Dv != 128, chunk
 * not 0 or 64) also return GDN_ERR_UNSUPPORTED.
 *
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address and caches it for that device and its current CUDA
 * context; a failure there returns GDN_ERR_CUDA.  Make that first call before
 * any stream capture.  When the context changes (after cudaDeviceReset, the
 * primary context is created anew and the array with it), the next call looks
 * the address up again, so it too should come before any capture.  Devices
 * with an index of 64 or more are not served: the call returns
 * GDN_ERR_UNSUPPORTED for them.  Depending on the CUDA module loading mode,
 * the array's device memory is reserved when libgdn's module is loaded or at
 * that first call.
 *
 * Nothing in the array has to start at zero: within one call every ring slot
 * is written before it is read.  There is one array per device, so calls whose
 * execution overlaps on the same device (different streams, or threads not
 * ordered on one stream) race on it and give wrong results; order them.
 */
#define GDN_STATIC_WORKSPACE_MAX_UNITS 48
GDN_API gdn_status gdn_prefill_static_workspace(const void *q, const void *k, const void *v,
                                                gdn_dtype io_dtype, const float *g,
                                                const float *beta, const float *initial_state,
                                                const int32_t *cu_seqlens, int32_t N, int64_t T,
                                                int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv,
                                                int32_t chunk, void *o, float *final_state,
                                                int32_t *dev_error_flag, void *stream);

/*
 * Step order.  Section 三 of the page above states the gated rule with the
 * decay applied first and then the delta edit (the standard order used by
 * every call above), while its per-head step function takes the recall S k
 * from the state before the decay:
 *   GDN_ORDER_STANDARD      S <- a S;  r = S k;  S <- S + b (v - r) k^T;  o = S q
 *   GDN_ORDER_RECALL_FIRST  r = S k;  S <- a S;  S <- S + b (v - r) k^T;  o = S q
 * The two differ by b (1 - a) (S k) k^T per step and agree when a = 1 or b = 0.
 */
typedef enum gdn_order {
    GDN_ORDER_STANDARD = 0,
    GDN_ORDER_RECALL_FIRST = 1
} gdn_order;

/*
 * gdn_prefill_order -- gdn_prefill_ex in either step order.  All other
 * arguments, layouts, kernels, workspace sizes (gdn_prefill_ex_workspace_bytes)
 * and errors are those of gdn_prefill_ex; an order outside gdn_order returns
 * GDN_ERR_INVALID_ARGUMENT.  In the chunked kernels the recall-first order
 * changes only the decay factor of the recall terms: token r's recall of the
 * chunk's earlier writes and of the entering state is scaled by the decay up
 * to token r - 1 instead of r.
 */
GDN_API gdn_status gdn_prefill_order(const void *q, const void *k, const void *v,
                                     gdn_dtype io_dtype, const float *g, const float *beta,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                     int32_t Dv, int32_t chunk, void *o, float *final_state,
                                     void *workspace, size_t workspace_bytes,
                                     int32_t *dev_error_flag, void *stream,
                                     gdn_prefill_kernel kernel, gdn_order order);

/*
 * gdn_decode_step_order -- gdn_decode_step in either step order (fp32 state);
 * otherwise identical to gdn_decode_step.
 */
GDN_API gdn_status gdn_decode_step_order(const void *q, const void *k, const void *v,
                                         gdn_dtype io_dtype, const float *g, const float *beta,
                                         float *state, int32_t N, int32_t Hqk, int32_t Hv,
                                         int32_t Dk, int32_t Dv, void *o, int32_t *dev_error_flag,
                                         void *stream, gdn_order order);

/*
 * gdn_decode_step_slots -- gdn_decode_step for continuous batching: the head
 * states live in a pool of slots, batch entry n uses slot slot_idx[n], and an
 * entry that starts a new request starts from a zero state.  This is the
 * runtime's batch / reset rule for the state (page "Layouts híbridos: três
 * DeltaNet, uma attention", section on what the runtime must support: state
 * updates, with rules for batching and reset).
 *
 *   state_pool          fp32 [num_slots][Hv][Dv][Dk], updated in place; only
 *                       the slots named in slot_idx are read or written.
 *   num_slots           slots in the pool (>= 1 when N > 0).
 *   slot_idx            device int32 [N]: the slot of each entry.  The values
 *                       must be distinct (two entries naming one slot race);
 *                       a value outside [0, num_slots) is a device-detected
 *                       error: GDN_ERR_BAD_SLOT goes to *dev_error_flag and
 *                       that entry writes neither state nor o.
 *   reset               device int32 [N] or NULL: nonzero = the entry's step
 *                       starts from a zero state; its slot's old contents are
 *                       not read, and the step's result overwrites them.
 *   everything else     as gdn_decode_step (fp32 state, standard order).
 * Supported: as gdn_decode_step.
 */
GDN_API gdn_status gdn_decode_step_slots(const void *q, const void *k, const void *v,
                                         gdn_dtype io_dtype, const float *g, const float *beta,
                                         float *state_pool, int32_t num_slots,
                                         const int32_t *slot_idx, const int32_t *reset, int32_t N,
                                         int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, void *o,
                                         int32_t *dev_error_flag, void *stream);

/*
 * gdn_short_conv_norm -- the front end of the DeltaNet mixer before the delta
 * rule: the mixer's "kernel 4" convolution (page "Layouts híbridos: três
 * DeltaNet, uma attention", section 01) on the q, k and v channels, then q and
 * k normalised per (token, head).  Per channel c, causally within each
 * sequence,
 *     y[t, c] = w[c,0] x[t-3, c] + w[c,1] x[t-2, c] + w[c,2] x[t-1, c] + w[c,3] x[t, c],
 * inputs before a sequence's first token taken from conv_state_in (or zero);
 * q, k rows divided by their Euclidean norm (a zero row stays zero); no
 * activation (the page names none).  Computed in fp32, outputs rounded once
 * to io_dtype; the outputs are gdn_prefill's q, k, v.
 *
 *   xq, xk              [T][Hqk][Dk] io_dtype, the inputs of the q and k channels.
 *   xv                  [T][Hv][Dv] io_dtype.
 *   wq, wk              fp32 [Hqk*Dk][4] filters (tap 3 multiplies the current token).
 *   wv                  fp32 [Hv*Dv][4].
 *   conv_state_in       fp32 [N][3][2*Hqk*Dk + Hv*Dv] or NULL (zeros): per
 *                       sequence, the three inputs before its first token,
 *                       oldest first, channels in the order q, k, v.
 *   conv_state_out      the same layout, or NULL to skip: each sequence's last
 *                       three inputs (reaching into conv_state_in when it is
 *                       shorter than 3), for a later call that continues it.
 *                       May equal conv_state_in.
 *   cu_seqlens, N, T    as gdn_prefill.
 *   q, k, v             outputs [T][Hqk][Dk], [T][Hqk][Dk], [T][Hv][Dv] io_dtype;
 *                       must not alias the inputs or each other.
 * Supported: Dk = Dv = 128.  A malformed cu_seqlens is reported as
 * GDN_ERR_BAD_SEQLENS (when conv_state_out is given); the outputs are then
 * unspecified, but nothing outside the arrays is touched.
 */
GDN_API gdn_status gdn_short_conv_norm(const void *xq, const void *xk, const void *xv,
                                       gdn_dtype io_dtype, const float *wq, const float *wk,
                                       const float *wv, const float *conv_state_in,
                                       float *conv_state_out, const int32_t *cu_seqlens, int32_t N,
                                       int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv,
                                       void *q, void *k, void *v, int32_t *dev_error_flag,
                                       void *stream);

/*
 * gdn_prefill_conv -- gdn_short_conv_norm followed by gdn_prefill, as one
 * operation: the mixer's front end (the "kernel 4" convolution of the q, k, v
 * channels and the per-(token, head) normalisation of q and k, page "Layouts
 * híbridos: três DeltaNet, uma attention", section 01) is fused into the load
 * stage of the pool prefill kernel, so the convolved q, k, v never go through
 * HBM.
 *
 *   xq, xk, xv, wq, wk, wv, conv_state_in, conv_state_out
 *                       as gdn_short_conv_norm (raw channel inputs, filters,
 *                       carried conv states; conv_state_out may equal
 *                       conv_state_in).
 *   g, beta, initial_state, cu_seqlens, N, T, Hqk, Hv, Dk, Dv, chunk, o,
 *   final_state, dev_error_flag, stream
 *                       as gdn_prefill with kernel GDN_PREFILL_POOL.
 *   workspace, workspace_bytes
 *                       device scratch of at least
 *                       gdn_prefill_conv_workspace_bytes() (the pool
 *                       kernel's, then a copy of the filters rearranged for
 *                       its load stage), 16-byte aligned, caller-owned;
 *                       contents need not be preserved between calls.
 * Arithmetic: as the two calls -- the convolution and the norm in fp32, q, k
 * and v rounded to bf16 once -- up to the order in which a norm's squares are
 * summed.  Supported: the pool kernel's shapes (bf16, Dk = Dv = 128, chunk 0
 * or 64, N * Hv <= 64 and SMs enough for it on this GPU); anything else
 * returns GDN_ERR_UNSUPPORTED (run the two calls instead).  Errors as the two
 * calls, and GDN_ERR_INVALID_ARGUMENT for a workspace that is too small.
 */
/*
 * gdn_prefill_conv_workspace_bytes -- scratch bytes gdn_prefill_conv needs for
 * these sizes; 0 when T <= 0 or the shapes are outside the ones it supports
 * (the call then needs none, or returns GDN_ERR_UNSUPPORTED).
 */
GDN_API size_t gdn_prefill_conv_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv,
                                                int32_t Dk, int32_t Dv);

GDN_API gdn_status gdn_prefill_conv(const void *xq, const void *xk, const void *xv,
                                    gdn_dtype io_dtype, const float *wq, const float *wk,
                                    const float *wv, const float *conv_state_in,
                                    float *conv_state_out, const float *g, const float *beta,
                                    const float *initial_state, const int32_t *cu_seqlens,
                                    int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                    int32_t Dv, int32_t chunk, void *o, float *final_state,
                                    void *workspace, size_t workspace_bytes,
                                    int32_t *dev_error_flag, void *stream);

/*
 * gdn_prefill_slots -- gdn_prefill over a packed batch whose states live in
 * the same pool of slots as gdn_decode_step_slots (continuous batching: page
 * "Hybrid · kết hợp…", section 3, state updates with batch and reset rules).
 * Sequence n starts from state_pool[slot_idx[n]], or from zeros when reset[n]
 * is nonzero (a new request; its slot is not read), and its final state is
 * written back to that slot.  Slots no sequence names are not touched.
 *
 *   q, k, v, io_dtype, g, beta, cu_seqlens, N, T, Hqk, Hv, Dk, Dv, chunk, o,
 *   dev_error_flag, stream
 *                       as gdn_prefill.
 *   state_pool          fp32 [num_slots][Hv][Dv][Dk], device, updated in place.
 *   slot_idx            device int32 [N], distinct values in [0, num_slots).
 *                       An index out of range is reported as GDN_ERR_BAD_SLOT
 *                       through dev_error_flag; that sequence runs from zeros
 *                       and its state is not stored.  Repeated indices are a
 *                       caller error (the slot ends with one of the states).
 *   reset               device int32 [N], or NULL for none.
 *   workspace, workspace_bytes
 *                       device scratch of at least
 *                       gdn_prefill_slots_workspace_bytes(): the N gathered
 *                       states, then gdn_prefill's workspace.
 * The states are gathered into the workspace, gdn_prefill runs in place on
 * them, and they are scattered back: 2 N Hv Dv Dk fp32 values of copies.
 * Errors as gdn_prefill, and GDN_ERR_INVALID_ARGUMENT for a null pool or
 * slot list, num_slots <= 0 or a short workspace.
 */
GDN_API gdn_status gdn_prefill_slots(const void *q, const void *k, const void *v,
                                     gdn_dtype io_dtype, const float *g, const float *beta,
                                     float *state_pool, int32_t num_slots,
                                     const int32_t *slot_idx, const int32_t *reset,
                                     const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk,
                                     int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                                     void *workspace, size_t workspace_bytes,
                                     int32_t *dev_error_flag, void *stream);

/*
 * gdn_prefill_slots_workspace_bytes -- scratch bytes gdn_prefill_slots needs
 * for these sizes (0 for invalid ones).
 */
GDN_API size_t gdn_prefill_slots_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv,
                                                 int32_t Dk, int32_t Dv, int32_t chunk);

/*
 * gdn_prefill_host -- gdn_prefill of ONE sequence whose inputs and outputs
 * are in host memory.  The state carries everything one part of a sequence
 * hands to the next (page "Qwen3.8-27B 架构深读…", section 三), so the
 * sequence runs as consecutive segments of segment_tokens tokens, each a
 * gdn_prefill call on `stream` that starts from the state the previous one
 * left (in place, in scratch).  Two internal streams overlap the copies: the
 * next segment's q, k, v, g, beta go in while a segment computes and the
 * previous segment's o comes back.
 *
 *   q, k, v, g, beta    HOST memory, layouts as gdn_prefill with N = 1.  Pin
 *                       it (cudaHostAlloc / cudaHostRegister) for the copies
 *                       to overlap; pageable memory works, serialised.
 *   initial_state       HOST fp32 [Hv][Dv][Dk], or NULL for zeros.
 *   T, Hqk, Hv, Dk, Dv, chunk
 *                       as gdn_prefill.
 *   o                   HOST output [T][Hv][Dv] in io_dtype.
 *   final_state         HOST fp32 [Hv][Dv][Dk], or NULL to skip.
 *   segment_tokens      tokens per segment, a multiple of 64 so that
 *                       segments end on chunk boundaries; 0 picks 16,384.
 *   scratch, scratch_bytes
 *                       DEVICE scratch of at least
 *                       gdn_prefill_host_scratch_bytes(), 16-byte aligned,
 *                       caller-owned: the state, the prefill workspace and
 *                       two segment buffers.
 *   dev_error_flag      optional device int32, as gdn_prefill.
 *   stream              cudaStream_t.  The call is asynchronous like a copy
 *                       on `stream`: it starts after the work queued there
 *                       and `stream` sees it complete; the host buffers must
 *                       stay valid and unread until then.
 * Arithmetic: the segments' kernels are gdn_prefill's for segment_tokens
 * tokens; the result equals one gdn_prefill call over the whole sequence
 * within the prefill's tolerances (a state that crosses a segment boundary
 * passes through fp32 memory exactly).  Errors: GDN_ERR_INVALID_ARGUMENT for
 * bad sizes, a segment length that is not a multiple of 64 or a short
 * scratch; gdn_prefill's otherwise.  After GDN_ERR_CUDA (or an error from a
 * segment's gdn_prefill) copies of earlier segments may still be in flight
 * on the internal streams, which `stream` does not wait for: synchronise the
 * device before reusing the host buffers or the scratch.  It creates two
 * streams and eight events per call and releases them before returning (CUDA
 * frees them once the queued work is done).
 */
GDN_API gdn_status gdn_prefill_host(const void *q, const void *k, const void *v,
                                    gdn_dtype io_dtype, const float *g, const float *beta,
                                    const float *initial_state, int64_t T, int32_t Hqk,
                                    int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                                    float *final_state, int64_t segment_tokens, void *scratch,
                                    size_t scratch_bytes, int32_t *dev_error_flag, void *stream);

/*
 * gdn_prefill_host_scratch_bytes -- device scratch gdn_prefill_host needs for
 * these sizes (0 for invalid ones).
 */
GDN_API size_t gdn_prefill_host_scratch_bytes(int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                              int32_t Dv, int32_t chunk, gdn_dtype io_dtype,
                                              int64_t segment_tokens);

/*
 * gdn_debug_prefill_pool_stall -- FOR TESTING THE TIMEOUT PATH ONLY.
 * gdn_prefill_ex with kernel GDN_PREFILL_POOL, except that the producer CTAs
 * never prepare the chunks of (sequence, head) unit `skip_unit` (n * Hv + h),
 * and that every spin on a hand-off flag in workspace memory (a chain waiting
 * for its next chunk, a producer waiting for a free ring slot) gives up after
 * `flag_wait_cycles` SM clocks instead of about 2^31.  The chain of the skipped
 * unit therefore waits for a chunk that never comes, with no copy in flight
 * into its shared memory; when its wait gives up it reports GDN_ERR_TIMEOUT
 * through *dev_error_flag and raises the kernel's abort flag, every other CTA
 * stops at its next wait, and the launch ends.  Outputs are unspecified.  The
 * context stays usable: later calls run normally.  skip_unit < 0 or
 * flag_wait_cycles <= 0 returns GDN_ERR_INVALID_ARGUMENT; everything else as
 * gdn_prefill_ex (a shape the pool kernel does not take returns
 * GDN_ERR_UNSUPPORTED).  The page has no counterpart to this call.
 */
GDN_API gdn_status gdn_debug_prefill_pool_stall(const void *q, const void *k, const void *v,
                                                gdn_dtype io_dtype, const float *g,
                                                const float *beta, const float *initial_state,
                                                const int32_t *cu_seqlens, int32_t N, int64_t T,
                                                int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv,
                                                int32_t chunk, void *o, float *final_state,
                                                void *workspace, size_t workspace_bytes,
                                                int32_t *dev_error_flag, void *stream,
                                                int32_t skip_unit, int64_t flag_wait_cycles);

/* Human-readable name of a status code (static storage, never NULL). */
GDN_API const char *gdn_status_string(gdn_status status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
GDN_API int32_t gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
