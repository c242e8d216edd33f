/*
 * efla.h -- C ABI of the B200 (sm_100a) Exact Flow Linear Attention forward.
 *
 * The method (Exact Flow Linear Attention, arXiv 2512.12602): the delta-rule write
 * S_t = S_{t-1} - beta_t k_t (k_t^T S_{t-1} - v_t^T) is one explicit Euler step of
 * dS/dtau = -k k^T S + k v^T (summary page, Section 2 and Section 3.1).  Solving that
 * zero-order-hold ODE in closed form keeps the rank-1 write with beta_t replaced by the
 * gate (Section 3.2, with the denominator of Section 3.4 and the rank-1 algebra of App. D/E)
 *
 *     alpha_t = (1 - exp(-beta_t * lambda_t)) / lambda_t,   lambda_t = ||k_t||^2,
 *
 * and the read-out is o_t = S_t^T q_t, taken after the write.
 *
 * Conventions shared by every entry point:
 *   - Row convention: the state S of one (batch, head) stream is a d_k x d_v row-major
 *     float32 matrix and o_t^T = q_t^T S_t (the transpose of the pages' column form).
 *   - Tensors are contiguous, row-major, head-major: q, k [B, H, T, d_k]; v, o [B, H, T, d_v];
 *     beta [B, H, T]; states [B, H, d_k, d_v] float32.
 *   - q, k, v, beta and o share one element type (efla_dtype); states are always float32.
 *   - All data pointers are DEVICE pointers owned by the caller.  The library calls no
 *     allocator.  Its only global state is per-device host-side caches (SM count, kernel
 *     attributes, the scratch address below) and one 32 MiB static device array, the
 *     scratch of efla_chunk_fwd_noalloc, shared by every call of that entry point (calls
 *     that overlap on the GPU race on it).  Every other entry point works only on the
 *     caller's buffers: calls on different streams may run concurrently as long as their
 *     buffers (workspaces included) do not overlap.
 *   - Every pointer must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL: the legacy default stream) and never
 *     synchronise the host.  A non-OK status from argument checking means nothing was
 *     launched.  EFLA_ERR_CUDA reports a launch error (cudaGetLastError).
 *   - Errors detected on the device (a bounded wait that ran out) are recorded in the
 *     workspace of efla_chunk_fwd and read back with efla_workspace_status.
 */
#ifndef EFLA_H
#define EFLA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EFLA_OK = 0,
    EFLA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, non-positive size, bad workspace */
    EFLA_ERR_UNSUPPORTED = 2,  /* valid but unsupported shape (d_k, d_v, chunk) or dtype */
    EFLA_ERR_CUDA = 3,         /* a CUDA call or kernel launch failed */
    EFLA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out (see efla_workspace_status) */
    EFLA_ERR_BOUNDS = 5        /* a checked build (libefla_checked.so) recorded an out-of-range access */
} efla_status;

typedef enum {
    EFLA_DTYPE_F32 = 0,   /* float32 q, k, v, beta, o */
    EFLA_DTYPE_BF16 = 1   /* bfloat16 q, k, v, beta, o (fp32 accumulation and state) */
} efla_dtype;

/*
 * The step size each token writes with.  EFLA_RULE_EXACT is the method: the exact-flow
 * gate alpha = (1 - exp(-beta lambda)) / lambda (Section 3.2).  EFLA_RULE_EULER is the
 * delta rule the method replaces (alpha = beta: one explicit Euler step of the same ODE,
 * Section 2), run through the same kernels for comparison.
 */
typedef enum {
    EFLA_RULE_EXACT = 0,
    EFLA_RULE_EULER = 1
} efla_rule;

/* Same type as cudaStream_t, declared here so this header needs no CUDA include. */
typedef struct CUstream_st *efla_stream_t;

/* Human-readable name of a status code (static storage). */
const char *efla_status_string(int status);

/*
 * efla_gate -- the exact-flow gate alone (Section 3.2 gate, Section 3.4 denominator).
 *   k     [n, d_k] (dtype), beta [n] (dtype)  ->  alpha [n] float32
 *   lambda = sum_i k_i^2 accumulated in float32; alpha = -expm1(-beta*lambda)/lambda, and
 *   alpha = beta exactly when lambda == 0.
 * Supports any d_k in [1, 4096] with d_k*sizeof(dtype) a multiple of 16 bytes.
 */
int efla_gate(const void *k, const void *beta, float *alpha, long n, int d_k, int dtype,
              efla_stream_t stream);

/*
 * efla_chunk_fwd_workspace_bytes -- bytes of device workspace efla_chunk_fwd needs for
 * this problem (always > 0: it holds at least the device error word).  Returns 0 for
 * arguments efla_chunk_fwd would reject.
 */
size_t efla_chunk_fwd_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk,
                                      int dtype);

/*
 * efla_chunk_fwd -- chunkwise-parallel forward over B*H independent streams of T tokens
 * (Section 3.3: tokens stacked per chunk, causal lower-triangular mask, UT transform).
 *
 *   q, k [B,H,T,d_k], v [B,H,T,d_v], beta [B,H,T]         inputs, `dtype`
 *   S0   [B,H,d_k,d_v] float32 or NULL (zero initial state)
 *   o    [B,H,T,d_v]  output, `dtype`
 *   S_T  [B,H,d_k,d_v] float32 final state, or NULL (not written).  S_T may alias S0.
 *   o must not overlap any input.  No input, output or state may overlap the workspace.
 *   workspace: device memory of at least efla_chunk_fwd_workspace_bytes(...) bytes,
 *   16-byte aligned, owned by the caller; its first bytes hold a sticky device error word
 *   (zero it once before first use, e.g. with cudaMemset).  For bf16 with d = 128 it also
 *   holds every chunk's UT transform T (8 KiB per (stream, chunk)); calls that overlap
 *   on the GPU must not share a workspace.
 *
 * Supported: d_k = d_v in {64, 128}, chunk = 64, any T >= 1 (the tail chunk is padded with
 * k = 0, beta = 0 tokens, which are exact no-ops), B*H >= 1.
 * bf16 runs on the 5th-generation tensor cores (bf16 operands, fp32 accumulation, fp32
 * state); f32 runs on fp32 CUDA cores.
 */
int efla_chunk_fwd(const void *q, const void *k, const void *v, const void *beta,
                   const float *S0, void *o, float *S_T, int B, int H, int T, int d_k,
                   int d_v, int chunk, int dtype, void *workspace, size_t workspace_bytes,
                   efla_stream_t stream);

/*
 * efla_chunk_fwd_ex -- efla_chunk_fwd with the step rule chosen: `rule` is an efla_rule
 * (any other value: EFLA_ERR_INVALID_ARG, nothing launched).  efla_chunk_fwd is this call
 * with EFLA_RULE_EXACT.  Under EFLA_RULE_EULER the forward is the chunked delta rule
 * (DeltaNet form): the same UT-transform algebra with alpha = beta.  Every other argument
 * and behaviour is that of efla_chunk_fwd.
 */
int efla_chunk_fwd_ex(const void *q, const void *k, const void *v, const void *beta,
                      const float *S0, void *o, float *S_T, int B, int H, int T, int d_k,
                      int d_v, int chunk, int dtype, int rule, void *workspace,
                      size_t workspace_bytes, efla_stream_t stream);

/*
 * Gated EFLA (Section 3.4 names the method's gated variant; App. F, "exact-flow
 * formulation of Gated DeltaNet", survives on the pages only as a title, so the update
 * below is this library's reading).  Each token carries a log-decay g_t (a forget gate
 * e^{g_t}; g <= 0 decays) that joins the zero-order-hold ODE over the token's unit
 * interval together with the write rate beta_t:
 *     dS/dtau = g S - beta (k k^T S - k v^T),   tau in [0, 1].
 * Its exact flow is
 *     S_t = e^{g_t} (S_{t-1} - alpha_t k_t (k_t^T S_{t-1})) + abar_t k_t v_t^T,   o_t = S_t^T q_t,
 *     alpha_t = beta_t phi1(beta_t lambda_t),  abar_t = beta_t phi1(beta_t lambda_t - g_t),
 *     phi1(x) = (1 - e^{-x}) / x,
 * which is efla_chunk_fwd's update at g = 0.  EFLA_RULE_EULER gives the gated delta rule
 * (Gated DeltaNet), alpha = abar = beta.
 *
 * efla_chunk_fwd_gated_workspace_bytes -- workspace of efla_chunk_fwd_gated (0 for
 * arguments it would reject).
 */
size_t efla_chunk_fwd_gated_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk,
                                            int dtype);

/*
 * efla_chunk_fwd_gated -- efla_chunk_fwd_ex with the gated flow above.
 *   g [B,H,T] float32, the per-token log-decay (16-byte aligned, must not overlap o, S_T
 *   or the workspace).  Every other argument, layout, supported shape and error is that of
 *   efla_chunk_fwd_ex; the workspace must hold efla_chunk_fwd_gated_workspace_bytes.
 *   g == NULL with B*H*T > 0 is EFLA_ERR_INVALID_ARG.
 */
int efla_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *beta,
                         const float *g, const float *S0, void *o, float *S_T, int B, int H, int T,
                         int d_k, int d_v, int chunk, int dtype, int rule, void *workspace,
                         size_t workspace_bytes, efla_stream_t stream);

/*
 * efla_recurrent_step_gated -- efla_recurrent_step_ex with the gated flow above:
 *   g [N,H] float32, this token's log-decay per stream (16-byte aligned, must not overlap o
 *   or S).  One pass over S: with r = k^T S, p = q^T S, c = q.k, d = e^g,
 *   w = d alpha r - abar v:  S <- d S - k w^T,  o = d p - c w.
 */
int efla_recurrent_step_gated(const void *q, const void *k, const void *v, const void *beta,
                              const float *g, float *S, void *o, int N, int H, int d_k, int d_v,
                              int dtype, int rule, efla_stream_t stream);

/*
 * Packed variable-length batches (Section 3.3's chunkwise form, applied to each sequence
 * on its own; the pages note that long and mixed contexts are where recurrent memories are
 * used, App. A).  N sequences of different lengths are packed head-major along the token
 * axis, with no padding between them:
 *   q, k [H, total_T, d_k], v, o [H, total_T, d_v], beta [H, total_T]   (dtype)
 *   g    [H, total_T] float32 log-decay for the gated flow, or NULL (ungated)
 *   S0, S_T [N, H, d_k, d_v] float32 (each may be NULL; S_T may alias S0)
 *   cu_seqlens: HOST array of N + 1 int32 offsets, cu_seqlens[0] = 0, non-decreasing,
 *   total_T = cu_seqlens[N]; sequence n is tokens cu_seqlens[n] .. cu_seqlens[n+1] - 1 of every
 *   head.  Each (sequence, head) is an independent recurrence from its own S0 slice; its
 *   chunks start at its first token, and an empty sequence passes its state through.
 * The call copies cu_seqlens into the workspace (cudaMemcpyAsync; from pageable host memory
 * that copy may synchronise the host with `stream`, and it cannot be captured in a graph).
 *
 * efla_chunk_fwd_varlen_workspace_bytes -- workspace bytes for these offsets (gated != 0 for
 * the gated flow), or 0 for arguments efla_chunk_fwd_varlen would reject.
 */
size_t efla_chunk_fwd_varlen_workspace_bytes(const int *cu_seqlens, int N, int H, int d_k, int d_v,
                                             int chunk, int dtype, int gated);

/*
 * efla_chunk_fwd_varlen -- the chunked forward (or, with g, the gated forward) over a packed
 * variable-length batch, layouts above.  Supported shapes, dtypes, rules, alignment and
 * errors are those of efla_chunk_fwd_ex; cu_seqlens that are not valid offsets are
 * EFLA_ERR_INVALID_ARG.  No input may overlap o, S_T or the workspace.
 */
int efla_chunk_fwd_varlen(const void *q, const void *k, const void *v, const void *beta,
                          const float *g, const int *cu_seqlens, const float *S0, void *o, float *S_T,
                          int N, int H, int d_k, int d_v, int chunk, int dtype, int rule,
                          void *workspace, size_t workspace_bytes, efla_stream_t stream);

/*
 * Segmented scan for long streams (Section 3.3's chunk recurrence is affine in the state,
 * S -> (I - K^T W) S + K^T U; App. A notes long contexts as the open case).  With few streams
 * and many chunks the chain of chunks, not the hardware, sets the time; splitting each
 * stream into G segments runs them side by side:
 *   - segment 0 runs from S0 as usual;
 *   - every later segment g runs from a zero state (final state S_loc(g), outputs O_loc) and,
 *     beside it, with V = 0 from S = I (final state Phi(g), the segment's transition
 *     product, and outputs R(g), each token's linear dependence on the entering state);
 *   - S_in(g+1) = Phi(g) S_in(g) + S_loc(g) in order (S_in(1) = segment 0's final state),
 *     S_T = S_in(G), and every token of segment g >= 1 gets o += R S_in(g).
 * The results equal efla_chunk_fwd's up to rounding (the transition product and R pass
 * through the same bf16-operand, fp32-accumulate products as the state).
 *
 * efla_chunk_fwd_segmented_workspace_bytes -- workspace for `segments` (0: chosen by the
 * library) and gated != 0 for the gated flow; 0 for arguments the call would reject.
 */
size_t efla_chunk_fwd_segmented_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk,
                                                int dtype, int gated, int segments);

/*
 * efla_chunk_fwd_segmented -- efla_chunk_fwd_ex (g == NULL) or efla_chunk_fwd_gated (g given)
 * as a segmented scan.  segments >= 2 splits every stream into that many segments of equal
 * chunk counts (fewer if the stream has under 8 chunks per segment); 0 lets the library
 * choose the most segments whose chain CTAs fit one wave on the device (B*H*(4G - 2) <= SMs);
 * 1 is the plain forward.  Only bf16 with d = 128 segments; other shapes run the plain
 * forward.  Arguments, layouts and errors otherwise as efla_chunk_fwd_ex;
 * segments < 0 is EFLA_ERR_INVALID_ARG.
 */
int efla_chunk_fwd_segmented(const void *q, const void *k, const void *v, const void *beta,
                             const float *g, const float *S0, void *o, float *S_T, int B, int H,
                             int T, int d_k, int d_v, int chunk, int dtype, int rule, int segments,
                             void *workspace, size_t workspace_bytes, efla_stream_t stream);

/*
 * efla_chunk_fwd_noalloc -- efla_chunk_fwd without a caller-provided workspace.
 * The paper has no counterpart: this is an integration variant for callers that cannot
 * allocate device memory, e.g. code embedded in a host runtime that owns every device
 * allocation and hands over only the input and output tensors, or latency-critical
 * paths where cudaMalloc (which may synchronise the device) is not acceptable.
 *
 * Arguments, layouts, supported shapes and results are those of efla_chunk_fwd.  The
 * scratch is a 32 MiB static device array inside the library (held on every GPU that
 * loads it, until exit): a problem whose efla_chunk_fwd_workspace_bytes exceeds 32 MiB
 * (for bf16, d = 128: more than 4095 (stream, 64-token chunk) tiles) returns
 * EFLA_ERR_UNSUPPORTED and launches nothing.  No device memory is allocated.
 * The first call on a device looks up the array's device address (with that device
 * current); make that first call before any stream capture.  Every call shares the one
 * array and each call clears its error word first, so calls that overlap on the GPU
 * (different streams, or different host threads) race on it and must be serialised by
 * the caller.  A device-side wait timeout in this variant is recorded in the scratch's
 * error word; efla_noalloc_status reads it back (each call clears it first).
 */
int efla_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *beta,
                           const float *S0, void *o, float *S_T, int B, int H, int T, int d_k,
                           int d_v, int chunk, int dtype, efla_stream_t stream);

/*
 * efla_noalloc_status -- efla_workspace_status for the static scratch of
 * efla_chunk_fwd_noalloc on the current device: waits for `stream`, then returns
 * EFLA_ERR_TIMEOUT if the last efla_chunk_fwd_noalloc call on this device gave up on a
 * device wait (its outputs are then invalid), else EFLA_OK.  clear != 0 resets the word.
 * Like efla_chunk_fwd_noalloc, it has no counterpart in the paper.
 */
int efla_noalloc_status(int clear, efla_stream_t stream);

/*
 * efla_workspace_status -- waits for `stream`, then returns EFLA_ERR_TIMEOUT if any
 * efla_chunk_fwd that used `workspace` gave up on a device wait since the word was last
 * cleared (its outputs are then invalid), EFLA_ERR_BOUNDS if a checked build of the
 * library (libefla_checked.so: the same entry points, built with EFLA_CHECKED=1, whose
 * tensor-core forward kernels test every direct global access and computed shared-memory
 * store against its buffer and skip it when out of range) recorded an out-of-range
 * access, else EFLA_OK.  clear != 0 resets the word.
 * This is the one call that synchronises the host.
 */
int efla_workspace_status(void *workspace, int clear, efla_stream_t stream);

/*
 * efla_selftest_wait_timeout -- failure-detection self test.  Launches one CTA that waits
 * on a barrier nothing will ever arrive on, with the device-side bound `limit_ns`
 * (nanoseconds); when the bound runs out the CTA records the timeout in `workspace`'s
 * error word and exits.  efla_workspace_status then reports EFLA_ERR_TIMEOUT.  The same
 * bounded wait guards every barrier wait of efla_chunk_fwd (bound: 2 s per wait).
 */
int efla_selftest_wait_timeout(void *workspace, long long limit_ns, efla_stream_t stream);

/*
 * efla_recurrent_step -- one decode token for N*H streams, state updated in place
 * (the recurrent form: Section 3.2 update, o_t = S_t^T q_t).
 *
 *   q, k [N,H,d_k], v [N,H,d_v], beta [N,H]   inputs, `dtype`
 *   S    [N,H,d_k,d_v] float32, read and overwritten with the new state
 *   o    [N,H,d_v] output, `dtype`; must not overlap S or any input
 *
 * One pass over S: r = k^T S, p = q^T S and c = q.k are formed together, then
 * S <- S - alpha k (r - v)^T and o = p - alpha c (r - v).
 * Supported: d_k = d_v in {64, 128}; dtype f32 or bf16.
 */
int efla_recurrent_step(const void *q, const void *k, const void *v, const void *beta,
                        float *S, void *o, int N, int H, int d_k, int d_v, int dtype,
                        efla_stream_t stream);

/*
 * efla_recurrent_step_ex -- efla_recurrent_step with the step rule chosen (`rule` an
 * efla_rule, else EFLA_ERR_INVALID_ARG and nothing launched).  efla_recurrent_step is
 * this call with EFLA_RULE_EXACT; EFLA_RULE_EULER writes with alpha = beta.
 */
int efla_recurrent_step_ex(const void *q, const void *k, const void *v, const void *beta,
                           float *S, void *o, int N, int H, int d_k, int d_v, int dtype,
                           int rule, efla_stream_t stream);

/*
 * efla_backward_workspace_bytes -- bytes of device workspace efla_backward needs.  bf16 with
 * d = 128 (the chunkwise form): a 256-byte header (the device error word) and, per 64-token
 * chunk, its UT transform T (bf16 64 x 64), X = (I + A)^{-1} (fp32 64 x 64, rows padded
 * to 68), its entering state and its dS' (bf16 128 x 128 each).  Otherwise (the token sweep): B*H*T*d_v + B*H*T floats (the residuals
 * r_t = S_{t-1}^T k_t - v_t of a forward sweep, and the gate gradient).  0 for an
 * unsupported shape or dtype.
 */
size_t efla_backward_workspace_bytes(int B, int H, int T, int d_k, int d_v, int dtype);

/*
 * efla_backward -- gradients of the forward pass (efla_chunk_fwd / the recurrence of
 * Section 3.2 with o_t = S_t^T q_t) for the loss sum(dO * o) + sum(dS_T * S_T): the
 * chain rule of the recurrence taken in reverse (training, Section 4.6; the pages print
 * no backward formulas).  With G = dL/dS_t, r_t = S_{t-1}^T k_t - v_t:
 *   dq_t = S_t dO_t, dv_t = alpha_t G^T k_t, dk_t = -alpha_t (G r_t + S_{t-1} G^T k_t)
 *   + dalpha_t (d alpha / d lambda) 2 k_t, dbeta_t = dalpha_t (d alpha / d beta) with
 *   dalpha_t = -(G^T k_t) . r_t, G <- G - alpha_t k_t (G^T k_t)^T; dS0 = G at t = 0.
 *
 *   q, k [B,H,T,d_k], v, dO [B,H,T,d_v], beta [B,H,T]   inputs, `dtype`
 *   S0, dS_T [B,H,d_k,d_v] float32, or NULL (zero)
 *   dq, dk [B,H,T,d_k], dv [B,H,T,d_v], dbeta [B,H,T]   float32 outputs
 *   dS0 [B,H,d_k,d_v] float32 output, or NULL (not wanted)
 *   workspace (>= efla_backward_workspace_bytes, 16-byte aligned), caller-owned
 *
 * Supported: d_k = d_v in {64, 128}; dtype f32 or bf16; any T >= 0 (T = 0 copies dS_T
 * into dS0).  All pointers 16-byte aligned; no output may overlap an input, the
 * workspace or another output, and no input may overlap the workspace; else
 * EFLA_ERR_INVALID_ARG and nothing is launched.
 * bf16 with d = 128 runs the reverse mode of the chunkwise form (Section 3.3) on tensor
 * cores: the UT transforms and the chunk states are recomputed, a reverse chain carries
 * dL/dS across chunks, and every chunk's gradients follow from its state and dS'.  Its
 * products take bf16 operands (as the forward's do) with fp32 accumulation, and its
 * results are the same bits on every call.  The token sweep (fp32, d = 64) keeps the state
 * and the gradients in fp32; its row sums over d_v columns use atomics, so their last bits
 * depend on arrival order.  Asynchronous on `stream`; launch failures return
 * EFLA_ERR_CUDA; a device wait that runs out is reported by efla_workspace_status.
 */
int efla_backward(const void *q, const void *k, const void *v, const void *beta, const float *S0,
                  const void *dO, const float *dS_T, float *dq, float *dk, float *dv, float *dbeta,
                  float *dS0, int B, int H, int T, int d_k, int d_v, int dtype, void *workspace,
                  size_t workspace_bytes, efla_stream_t stream);

/*
 * efla_backward_ex -- efla_backward with the step rule chosen (`rule` an efla_rule, else
 * EFLA_ERR_INVALID_ARG).  EFLA_RULE_EULER differentiates the Euler step alpha = beta.
 */
int efla_backward_ex(const void *q, const void *k, const void *v, const void *beta, const float *S0,
                     const void *dO, const float *dS_T, float *dq, float *dk, float *dv, float *dbeta,
                     float *dS0, int B, int H, int T, int d_k, int d_v, int dtype, int rule,
                     void *workspace, size_t workspace_bytes, efla_stream_t stream);

/*
 * Training with saved residuals (bf16, d_k = d_v = 128, chunk 64, ungated; the exact or
 * Euler rule).  The forward keeps what the chunkwise backward needs, and the backward takes
 * it instead of recomputing it (the recompute is a full forward: the UT transforms and the
 * state chain).
 *
 * efla_train_saved_bytes -- bytes of `saved`: a 256-byte header (the forward's device error
 *   word), the UT transform T of every 64-token chunk (bf16 64 x 64) with its
 *   X = (I + A)^{-1} (fp32 64 x 64, rows padded to 68) and every chunk's entering state
 *   (bf16 128 x 128).  0 for any other shape, dtype or chunk.
 *
 * efla_chunk_fwd_save -- efla_chunk_fwd_ex with `saved` (>= efla_train_saved_bytes,
 *   16-byte aligned, caller-owned) as its workspace: the same outputs, the same bits, and
 *   on return `saved` also holds every chunk's entering state.  Unsupported shapes return
 *   EFLA_ERR_UNSUPPORTED; the other argument rules and errors are efla_chunk_fwd_ex's.
 *
 * efla_backward_saved_workspace_bytes -- bytes of workspace efla_backward_saved needs: a
 *   256-byte header (the device error word) and every chunk's dS' (bf16 128 x 128).
 *
 * efla_backward_saved -- efla_backward_ex without the recompute: T and the entering states
 *   are read from `saved`, written by efla_chunk_fwd_save for the same q, k, v, beta, S0 and
 *   rule and not modified since (S0 is not an argument: it is the first saved state).
 *   The gradients are efla_backward_ex's, bit for bit.  No output or the workspace may
 *   overlap an input, `saved` or each other; else EFLA_ERR_INVALID_ARG and nothing is
 *   launched.  Asynchronous on `stream`.
 */
size_t efla_train_saved_bytes(int B, int H, int T, int d_k, int d_v, int chunk, int dtype);
int efla_chunk_fwd_save(const void *q, const void *k, const void *v, const void *beta, const float *S0,
                        void *o, float *S_T, int B, int H, int T, int d_k, int d_v, int chunk, int dtype,
                        int rule, void *saved, size_t saved_bytes, efla_stream_t stream);
size_t efla_backward_saved_workspace_bytes(int B, int H, int T, int d_k, int d_v, int dtype);
int efla_backward_saved(const void *q, const void *k, const void *v, const void *beta, const void *dO,
                        const float *dS_T, float *dq, float *dk, float *dv, float *dbeta, float *dS0, int B,
                        int H, int T, int d_k, int d_v, int dtype, int rule, const void *saved,
                        size_t saved_bytes, void *workspace, size_t workspace_bytes, efla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EFLA_H */
