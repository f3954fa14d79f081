/*
 * scan_gated_rnns.h -- C ABI of the B200 element-wise recurrence scans.
 *
 * Three operations, all element-wise over channels and sequential in time:
 *
 *   mingru_scan   minGRU over a whole sequence (page "Mingru Pytorch", sections
 *                 "Requirements & limits" -- the log-space numerically stable
 *                 minGRU -- and "Install and apply the minGRU layer": a batched
 *                 (B, T, D) tensor in, a tensor of the same shape out):
 *                     z_t = sigmoid(k_t),  htilde_t = g(hx_t),
 *                     g(x) = x + 0.5 (x >= 0), sigmoid(x) (x < 0),
 *                     h_t = (1 - z_t) h_{t-1} + z_t htilde_t,
 *                 which the log-space form writes as
 *                     h_t = exp(a*_t + logcumsumexp_{s<=t}(log z_s + log htilde_s - a*_s)),
 *                     a*_t = sum_{r<=t} -softplus(k_r),
 *                 with an optional carried state h_0 (absent: h_0 = 0).
 *   mingru_step   one token of the same recurrence, for token-by-token decoding
 *                 with the hidden state carried between calls (page "Mingru
 *                 Pytorch", guide "Process a sequence sequentially with carried
 *                 hidden state").  It returns only the new state.
 *   minmax_scan   MinMax neuron x_{t+1} = max(min(r_t, x_t), s_t) over a whole
 *                 sequence (page "MinMax Recurrent Neural Cascades", section
 *                 "The model", item 3), with an optional carried state x_0
 *                 (absent: +0).  Exact: the result is bitwise one of the inputs.
 *
 * The input projections that produce k, hx (or r, s) are not part of this
 * library: callers pass pre-activation tensors.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layout: (B, T, D) row-major, D fastest, contiguous; output index t holds
 *    the state after token t (T outputs; the initial state is not echoed).
 *    Initial states and step operands are (B, D) rows with a batch stride in
 *    ELEMENTS; stride 0 broadcasts one D-vector to every batch row (inputs only).
 *  - Pointers are DEVICE pointers (cudaMalloc / caching-allocator memory of the
 *    current device).  The caller owns every buffer; the library keeps no
 *    pointer after a call returns and allocates nothing.
 *  - dtype selects the storage type of every tensor of a call (inputs, initial
 *    state, output).  Arithmetic is fp32 on the device in both cases; bf16
 *    inputs widen exactly and outputs round to nearest-even.
 *  - Every call is asynchronous on `stream`.  Host-detectable errors return
 *    before anything is enqueued.  A launch failure returns SGR_ERR_CUDA.
 *  - Outputs must not overlap inputs (checked on the address ranges), except
 *    that mingru_step may update its state in place (h_out == h_prev with the
 *    same batch stride).
 *  - A size of 0 in any dimension is a valid no-op; negative sizes are
 *    SGR_ERR_INVALID_ARG.
 *  - Fast path: 16-byte aligned base pointers and D a multiple of 4 (fp32) or
 *    8 (bf16) take 128-bit vector loads; anything else runs a scalar GPU
 *    variant.  Results do not depend on the variant beyond fp32 rounding order.
 *  - minGRU inputs are NaN-free; h_0 > 0 where the log-space reading matters
 *    (the linear recurrence the kernels evaluate is defined for any h_0).
 *    MinMax inputs are NaN-free; with no -0.0 among the inputs the result is
 *    bit-identical to the sequential loop, otherwise equal as a value.
 *
 * Workspace (mingru_scan, minmax_scan)
 * ------------------------------------
 *  Every non-empty call takes a small device workspace: a 256-byte header
 *  whose first 4 bytes are the status word of the kernels' bounded waits
 *  (read by sgr_workspace_status), followed, when the sequence is cut into
 *  chunks of T that run on different thread blocks, by the words through
 *  which each chunk receives its carried state from the chunks before it
 *  (per-chunk summaries and states tagged with the launch; they stay in L2).
 *  sgr_workspace_size() gives the bytes a call needs: 256 when the whole
 *  sequence runs as one chunk, more when it is cut; 0 only for an empty
 *  shape, in which case workspace may be NULL.  Before its first use a
 *  workspace must be zero-filled once (sgr_workspace_init or cudaMemset);
 *  afterwards calls keep it valid.  One workspace must not be used by two
 *  calls that can run at the same time (e.g. on two streams).
 *  Calls may be captured in a CUDA graph; a captured call zero-fills the
 *  hand-off words itself inside the graph.  When one block per chunk is
 *  launched (the tile kernels), the call also zeroes a ticket counter in the
 *  header on `stream` before the launch: blocks take their chunk numbers from
 *  it in the order they start, so no chunk ever waits for one whose block has
 *  not started.
 *  Wide batches (B x D large enough that groups of 32 channels give every SM
 *  several warps) are not cut along T at all: each warp (or pair of warps)
 *  scans its 32 channels over the whole sequence, and the plan needs only the
 *  header.  The time-decayed minGRU (mingru_scan_decay) follows the same
 *  plans; sgr_workspace_size(SGR_OP_MINGRU, ...) covers it too.  The
 *  log-space minGRU (mingru_scan_log) is always cut along T when T spans
 *  several chunks: size its workspace with SGR_OP_MINGRU_LOG.
 */
#ifndef SCAN_GATED_RNNS_H
#define SCAN_GATED_RNNS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define SGR_API __attribute__((visibility("default")))
#else
#define SGR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sgr_status {
    SGR_OK = 0,
    SGR_ERR_INVALID_ARG = 1,  /* null pointer with data to move, negative size or
                                 stride, unknown dtype/op, overlapping output      */
    SGR_ERR_UNSUPPORTED = 2,  /* sizes beyond what the kernels index (grid > 2^31-1,
                                 byte counts overflowing int64)                    */
    SGR_ERR_WORKSPACE = 3,    /* workspace needed but NULL, too small or not
                                 16-byte aligned                                   */
    SGR_ERR_CUDA = 4,         /* a CUDA runtime call or a kernel launch failed     */
    SGR_ERR_TIMEOUT = 5       /* device side: a chunk waited too long (~0.3 s) for
                                 the state of the chunk before it and gave up; its
                                 outputs are NaN.  Reported by sgr_workspace_status */
} sgr_status_t;

typedef enum sgr_dtype { SGR_F32 = 0, SGR_BF16 = 1 } sgr_dtype_t;

/* SGR_OP_MINGRU_LOG names mingru_scan_log for sgr_workspace_size and
 * sgr_scan_plan only (it has no gradient, summary or step entry points). */
typedef enum sgr_op { SGR_OP_MINGRU = 0, SGR_OP_MINMAX = 1, SGR_OP_MINGRU_LOG = 2 } sgr_op_t;

/* ---------------------------------------------------------------- scans */

/*
 * mingru_scan -- h[b, t, :] for t = 0..T-1 from k, hx (B, T, D).
 *   k, hx    : gate and candidate pre-activations, (B, T, D), dtype.
 *   h0       : optional initial state rows (B, D) with batch stride
 *              h0_batch_stride (elements, >= 0); NULL means h_0 = 0.
 *   h        : output (B, T, D), dtype; must not overlap k, hx or h0.
 *   workspace: see above; ws_bytes >= sgr_workspace_size(SGR_OP_MINGRU, ...).
 */
SGR_API sgr_status_t mingru_scan(const void *k, const void *hx,
                         const void *h0, int64_t h0_batch_stride,
                         void *h, int64_t B, int64_t T, int64_t D,
                         sgr_dtype_t dtype, void *workspace, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * mingru_scan_log -- the same result as mingru_scan, evaluated in log space
 * (page "Mingru Pytorch", Requirements & limits: the log-space numerically
 * stable minGRU): the chunked kernels carry log2 h_t through pairs
 * (sum of log a, logaddexp of log b) and exponentiate at the store.  Kept as
 * the measured alternative to the linear pairs mingru_scan evaluates: more
 * MUFU work per element and an error that grows with the log-state's range.
 * Arguments, layout, ownership and errors as mingru_scan, except:
 *   h0       : optional initial state, h0 > 0 (0 allowed: log h = -inf);
 *              h0 < 0 has no logarithm and gives NaN outputs.
 *   workspace: ws_bytes >= sgr_workspace_size(SGR_OP_MINGRU_LOG, ...); the
 *              sequence is cut into chunks whatever the batch width (no
 *              channel-sequential kernel), so wide batches need more than
 *              sgr_workspace_size(SGR_OP_MINGRU, ...).
 */
SGR_API sgr_status_t mingru_scan_log(const void *k, const void *hx,
                         const void *h0, int64_t h0_batch_stride,
                         void *h, int64_t B, int64_t T, int64_t D,
                         sgr_dtype_t dtype, void *workspace, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * minmax_scan -- x[b, t, :] = x_{t+1} for t = 0..T-1 from r, s (B, T, D).
 *   x0 : optional initial state rows (B, D), batch stride x0_batch_stride;
 *        NULL means x_0 = +0.
 *   x  : output (B, T, D), dtype; must not overlap r, s or x0.
 */
SGR_API sgr_status_t minmax_scan(const void *r, const void *s,
                         const void *x0, int64_t x0_batch_stride,
                         void *x, int64_t B, int64_t T, int64_t D,
                         sgr_dtype_t dtype, void *workspace, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * mingru_step -- one token: h_out = (1 - z) h_prev + z g(hx_t), z = sigmoid(k_t).
 *   k_t, hx_t : (B, D) rows with batch strides (elements; e.g. k[:, t, :] of a
 *               (B, T, D) tensor has stride T*D).
 *   h_prev    : (B, D) rows with batch stride, or NULL for a zero state.
 *   h_out     : (B, D) rows with batch stride (>= D when B > 1).  May equal
 *               h_prev (same pointer and stride) for an in-place update; any
 *               other overlap with an operand is SGR_ERR_INVALID_ARG.
 * No workspace.  The arithmetic per element is the one mingru_scan uses, so a
 * prefix scanned in parallel followed by step calls matches the full scan to
 * fp32 rounding.
 */
SGR_API sgr_status_t mingru_step(const void *k_t, int64_t k_batch_stride,
                         const void *hx_t, int64_t hx_batch_stride,
                         const void *h_prev, int64_t h_prev_batch_stride,
                         void *h_out, int64_t h_out_batch_stride,
                         int64_t B, int64_t D, sgr_dtype_t dtype,
                         cudaStream_t stream);

/*
 * mingru_scan_noalloc -- mingru_scan for callers that cannot allocate device
 * memory where they call it (an inference runtime's plugin whose enqueue step
 * must not allocate, a process with a fixed device-memory plan, code running
 * while its stream is captured).  There is no counterpart on the pages: this
 * is a deployment convenience of this library.  Arguments and result are those
 * of mingru_scan minus the workspace: the scratch comes from a 16 MiB array
 * inside the library (held by every GPU that loads it, until exit).  Shapes
 * whose scratch (sgr_workspace_size) exceeds 16 MiB return
 * SGR_ERR_WORKSPACE.  The first call on a device looks up the array's device
 * address and zero-fills it on `stream`, so make it before any stream capture.
 * All calls on a device share the array: calls whose kernels can overlap on
 * the GPU race and must not be made.  The array's status word is internal:
 * each call clears it on `stream` before its launch and nothing reads it
 * back, so a chunk that gave up waiting (SGR_ERR_TIMEOUT with mingru_scan)
 * shows only as NaN outputs here.
 */
SGR_API sgr_status_t mingru_scan_noalloc(const void *k, const void *hx,
                                         const void *h0, int64_t h0_batch_stride,
                                         void *h, int64_t B, int64_t T, int64_t D,
                                         sgr_dtype_t dtype, cudaStream_t stream);

/* ------------------------------- input projection fused with the scan */

/*
 * mingru_projected_scan -- the minGRU layer's input projection and scan in
 * one kernel (page "Mingru Pytorch": the layer maps a (B, T, d) input to a
 * (B, T, D) output; the two pre-activations are linear projections of the
 * input):
 *     k[b, t, c]  = sum_j x[b, t, j] W[c, j]
 *     hx[b, t, c] = sum_j x[b, t, j] W[D + c, j]
 *     h = the minGRU scan of (k, hx) from h0, as mingru_scan
 * k and hx are computed on the tensor cores (bf16 operands, fp32
 * accumulation, tcgen05.mma) in tiles of 64 channels x 256 tokens and
 * consumed in place: they are never written to memory.
 *   x   : bf16 DEVICE (B, T, d_in) contiguous, 16-byte aligned
 *   w   : bf16 DEVICE (2 D, d_in) contiguous, 16-byte aligned (a linear
 *         layer's weight, out_features = 2 D: rows 0..D-1 give k, D..2D-1 hx)
 *   h0  : fp32 DEVICE rows (B, D), batch stride h0_batch_stride, or NULL (0)
 *   h   : fp32 DEVICE (B, T, D) output
 *   D % 64 == 0 and d_in % 64 == 0 (else SGR_ERR_UNSUPPORTED); any T.
 *   workspace: sgr_projected_workspace_size(B, T, D) bytes, zero-filled once
 *         (same rules as the scans' workspace; always needed).
 */
SGR_API size_t sgr_projected_workspace_size(int64_t B, int64_t T, int64_t D);
SGR_API sgr_status_t mingru_projected_scan(const void *x, const void *w,
                                           const float *h0, int64_t h0_batch_stride,
                                           float *h, int64_t B, int64_t T, int64_t D, int64_t d_in,
                                           void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------- time axis split over devices */

/*
 * A sequence whose time axis is split into contiguous slices, one per device
 * (rank r holds steps [t_r, t_{r+1})), is scanned with one exchange: every
 * slice's summary.  The recurrences compose associatively (page "MinMax
 * Recurrent Neural Cascades", Key properties: parallel training with
 * O(log T) depth; the minGRU's affine steps likewise), so a slice is
 * summarised per channel by one pair -- minGRU: h_end = A h_start + B;
 * MinMax: x_end = max(min(x_start, U), L) -- and the state entering slice r
 * is slices 0 .. r-1's pairs applied in order to the initial state.
 *
 * sgr_scan_summary: pairs (B, D, 2) fp32 (A, B or U, L), DEVICE, for the
 *   slice in0, in1 (B, T, D); T = 0 gives the identity pair.  Workspace:
 *   sgr_summary_workspace_size(B, T, D, dtype) bytes of device memory (no
 *   initialisation needed): a 256-byte header whose first 4 bytes receive the
 *   status word of the bounded waits (sgr_workspace_status reads it), then
 *   per-segment partial pairs.  Reads the inputs once.
 * sgr_combine_summaries: out (B, D) rows (batch stride out_bs, I/O dtype) =
 *   the state entering slice `rank`, from pairs (n, B, D, 2) fp32 of all
 *   slices in rank order (only the first `rank` are read) and the initial
 *   state init (rows with batch stride init_bs; NULL: the scan's default,
 *   0 for both).  out may be init (same stride) for an in-place update.
 * The slice is then scanned with mingru_scan / minmax_scan with that state.
 * The exchange itself (an all-gather of the (B, D, 2) pairs) is the
 * caller's: the Python package does it with torch.distributed (NCCL).
 */
SGR_API size_t sgr_summary_workspace_size(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype);
SGR_API sgr_status_t sgr_scan_summary(sgr_op_t op, const void *in0, const void *in1,
                                      int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                                      float *pairs, void *workspace, size_t ws_bytes,
                                      cudaStream_t stream);
SGR_API sgr_status_t sgr_combine_summaries(sgr_op_t op, const float *pairs, int64_t rank,
                                           const void *init, int64_t init_bs,
                                           void *out, int64_t out_bs, int64_t B, int64_t D,
                                           sgr_dtype_t dtype, cudaStream_t stream);

/* ----------------------------------------------------------- time decay */

/*
 * mingru_scan_decay -- mingru_scan with time decay (page "Your first delta
 * model", Step 5: the decay contract the mixers accept -- the carried state
 * is gated once per token at the token boundary, before that token's own
 * write lands undecayed).  For the minGRU's vector state:
 *     h_t = (1 - z_t) gamma_t h_{t-1} + z_t g(hx_t),
 *     gamma_t = exp(-lambda_d u_{b,t}),  u = delta_t, or log1p(delta_t)
 *               when log1p_delta != 0 (compresses very large gaps);
 * delta_t = 0 gives gamma = 1 (no decay); lambda u > 1e4 wipes the state
 * (gamma = 0 exactly).
 *   delta_t : fp32 DEVICE array (B, T), the gap preceding each token, >= 0
 *             and finite; batch stride delta_t_batch_stride (elements, >= T
 *             when B > 1)
 *   lambda  : fp32 DEVICE array (D,), decay rates >= 0 (fixed or learnable)
 * Other arguments, workspace and errors as mingru_scan (the same workspace
 * size); h must not overlap delta_t or lambda either (SGR_ERR_INVALID_ARG).
 * Arithmetic fp32; the gate uses the MUFU exp2 like the activations.
 * Kernel: never the channel-sequential one (it would wait for the gaps one row
 * at a time); the chunked kernels with 4 rows per thread, so the plan that
 * sgr_scan_plan reports for SGR_OP_MINGRU may differ.  With delta_t and lambda
 * 16-byte aligned (and a batch stride a multiple of 4) the pipelined kernel
 * brings them in with the copy engine beside the operands.
 */
SGR_API sgr_status_t mingru_scan_decay(const void *k, const void *hx,
                                       const void *h0, int64_t h0_batch_stride,
                                       const float *delta_t, int64_t delta_t_batch_stride,
                                       const float *lambda, int log1p_delta,
                                       void *h, int64_t B, int64_t T, int64_t D,
                                       sgr_dtype_t dtype, void *workspace, size_t ws_bytes,
                                       cudaStream_t stream);

/*
 * mingru_scan_decay_backward -- gradients through mingru_scan_decay for
 * dh = dL/dh: dk, dhx, dh0 as mingru_scan_backward (with the gate:
 * dk_t = delta_t z (1 - z) (g - gamma_t h_{t-1}), state gradient
 * (1 - z) gamma), and dlambda (fp32 DEVICE (D,), or NULL) = the sum over
 * b, t of delta_t (1 - z_t) h_{t-1} dgamma_t/dlambda_d with
 * dgamma/dlambda = -u gamma (0 where the 1e4 clamp wipes).  dlambda is
 * overwritten; its sums use atomic adds, so their rounding order varies from
 * run to run.  No gradient with respect to delta_t (the gaps are data).
 * No output may overlap delta_t or lambda, and dlambda may overlap no other
 * operand (SGR_ERR_INVALID_ARG).
 * Workspace: sgr_backward_workspace_size(SGR_OP_MINGRU, ...).
 */
SGR_API sgr_status_t mingru_scan_decay_backward(const void *k, const void *hx,
                                                const void *h0, int64_t h0_batch_stride,
                                                const float *delta_t, int64_t delta_t_batch_stride,
                                                const float *lambda, int log1p_delta,
                                                const void *h, const void *dh,
                                                void *dk, void *dhx,
                                                void *dh0, int64_t dh0_batch_stride,
                                                float *dlambda,
                                                int64_t B, int64_t T, int64_t D,
                                                sgr_dtype_t dtype, void *workspace,
                                                size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ gradients */

/*
 * mingru_scan_backward -- gradients of a loss L through mingru_scan, given the
 * upstream gradient dh = dL/dh (B, T, D) for every output row.  The pages
 * show the minGRU layer as a trainable module (page "Mingru Pytorch") but
 * print no derivative; this is the chain rule through the recurrence
 * h_t = (1 - z_t) h_{t-1} + z_t g(hx_t):
 *     delta_t = dh_t + (1 - z_{t+1}) delta_{t+1}          (delta_T+1 = 0)
 *     dk_t    = delta_t z_t (1 - z_t) (g(hx_t) - h_{t-1})
 *     dhx_t   = delta_t z_t g'(hx_t),  g'(x) = 1 (x >= 0), sigmoid(x) sigmoid(-x)
 *     dh0     = (1 - z_1) delta_1  (gradient with respect to the initial state)
 * computed as a reverse-time chunked scan (one kernel, decoupled look-back).
 *   k, hx, h0, h0_batch_stride : the forward call's inputs (h0 may be NULL)
 *   h     : the forward call's output (B, T, D); h_{t-1} is read from it
 *   dh    : dL/dh (B, T, D)
 *   dk, dhx : outputs (B, T, D)
 *   dh0   : optional output rows (B, D), batch stride dh0_batch_stride
 *           (>= D when B > 1); written whether or not h0 was given (the
 *           gradient with respect to a zero initial state); NULL: not written
 *   workspace: ws_bytes >= sgr_backward_workspace_size(SGR_OP_MINGRU, ...),
 *           same rules as the forward workspace (zero-filled once).
 * All tensors share dtype; arithmetic is fp32.  Outputs must not overlap any
 * input or each other (SGR_ERR_INVALID_ARG).  T = 0 writes dh0 = 0.
 */
SGR_API sgr_status_t mingru_scan_backward(const void *k, const void *hx,
                                          const void *h0, int64_t h0_batch_stride,
                                          const void *h, const void *dh,
                                          void *dk, void *dhx,
                                          void *dh0, int64_t dh0_batch_stride,
                                          int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                                          void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * minmax_scan_backward -- gradients through minmax_scan for dx = dL/dx
 * (B, T, D), x the forward output (x[t] = x_{t+1}).  The neuron selects one
 * operand per step, x_{t+1} = max(m_t, s_t), m_t = min(r_t, x_t); the gradient
 * flows to the selected operand, and equal operands of a min or a max share
 * it evenly (the rule of PyTorch's elementwise minimum / maximum, the
 * framework the page's package is written in; the page "MinMax Recurrent
 * Neural Cascades" gives no rule for ties).  Arguments as
 * mingru_scan_backward: r, s, x0 (NULL: +0) the forward inputs; dr, ds, dx0
 * the outputs.
 */
SGR_API sgr_status_t minmax_scan_backward(const void *r, const void *s,
                                          const void *x0, int64_t x0_batch_stride,
                                          const void *x, const void *dx,
                                          void *dr, void *ds,
                                          void *dx0, int64_t dx0_batch_stride,
                                          int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                                          void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Bytes of workspace a gradient call of this shape needs (at least the 256-byte
 * header for a non-empty shape; it covers the plain and the time-decayed
 * gradient).  0 for SGR_OP_MINGRU_LOG, which has no gradient.  Pure host
 * code. */
SGR_API size_t sgr_backward_workspace_size(sgr_op_t op, int64_t B, int64_t T, int64_t D,
                                           sgr_dtype_t dtype);

/* ---------------------------------------------------- host-buffer scans */

/*
 * mingru_scan_host / minmax_scan_host -- the same scans for operands that sit
 * in HOST memory: k, hx (r, s), the optional initial state and the output h
 * (x) are host pointers, same layout, strides and dtype rules as above.  There
 * is no counterpart on the pages; this is the library's end-to-end path for
 * data that does not already live on the GPU.
 *
 * The time axis is cut into slices of Tc = ceil(T / n) rows, n = `chunks`
 * (0 picks n = round(sqrt(input MiB / 4.6)): 7 slices for 256 MiB of inputs,
 * which balances a fixed cost per slice against the pipeline's fill and
 * drain).  Slice i is copied to
 * the device on a library-owned copy stream, scanned on `stream` with the
 * last row of slice i-1's output as its initial state, and copied back on a
 * second library-owned stream, with two sets of device buffers, so the
 * upload of slice i+1, the scan of slice i and the download of slice i-1
 * overlap.  The result equals that of one device scan up to fp32 rounding
 * order (MinMax: bit-identical).
 *
 * staging: DEVICE memory of at least sgr_host_staging_size(...) bytes, 16-byte
 *   aligned, owned by the caller; its contents need no initialisation (its
 *   first bytes hold the scan workspace, which each call clears, so
 *   sgr_workspace_status(staging, ...) reports a timed-out chunk of the call).
 *   One staging buffer serves one call at a time.
 * Ordering: the call returns once everything is enqueued.  The copies wait
 *   for the work already on `stream`, and `stream` waits for the last copy, so
 *   the host output is complete when `stream` reaches the point after the
 *   call (cudaStreamSynchronize(stream)).  Host buffers must stay valid until
 *   then.  Page-locked host memory gives asynchronous, overlapped copies;
 *   pageable memory gives correct results with copies that block the host.
 * Errors: as mingru_scan, plus SGR_ERR_WORKSPACE for a missing, small or
 *   misaligned staging buffer and SGR_ERR_INVALID_ARG for a capturing stream
 *   (these calls are not graph-capturable) or overlapping host buffers.
 */
SGR_API size_t sgr_host_staging_size(sgr_op_t op, int64_t B, int64_t T, int64_t D,
                                     sgr_dtype_t dtype, int chunks);
SGR_API sgr_status_t mingru_scan_host(const void *k, const void *hx,
                                      const void *h0, int64_t h0_batch_stride,
                                      void *h, int64_t B, int64_t T, int64_t D,
                                      sgr_dtype_t dtype, int chunks,
                                      void *staging, size_t staging_bytes,
                                      cudaStream_t stream);
SGR_API sgr_status_t minmax_scan_host(const void *r, const void *s,
                                      const void *x0, int64_t x0_batch_stride,
                                      void *x, int64_t B, int64_t T, int64_t D,
                                      sgr_dtype_t dtype, int chunks,
                                      void *staging, size_t staging_bytes,
                                      cudaStream_t stream);

/* ------------------------------------------------------------ workspace */

/* Bytes of workspace a scan of this shape needs: at least the 256-byte header
 * for any non-empty shape, 0 for an empty one or an unknown op.  op selects
 * mingru_scan (and mingru_scan_decay), minmax_scan, or mingru_scan_log
 * (SGR_OP_MINGRU_LOG).  Pure host code. */
SGR_API size_t sgr_workspace_size(sgr_op_t op, int64_t B, int64_t T, int64_t D,
                          sgr_dtype_t dtype);

/* Zero-fill a workspace on `stream` (asynchronous). */
SGR_API sgr_status_t sgr_workspace_init(void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronize `stream`, then read the device-side status word of a workspace:
 * SGR_OK, or SGR_ERR_TIMEOUT if any chunk gave up waiting since the word was
 * last cleared.  clear != 0 resets the word to SGR_OK afterwards.
 */
SGR_API sgr_status_t sgr_workspace_status(void *workspace, size_t ws_bytes, int clear,
                                  cudaStream_t stream);

/* ------------------------------------------------------------- misc */

SGR_API const char *sgr_status_string(sgr_status_t status);
SGR_API const char *sgr_version(void);

/*
 * Tuning/testing knob, process-wide: force the chunk shape the scans use.
 * rows_per_thread: tile kernel {1, 2, 4, 8} (bf16 vector tiles cap it at 4),
 * pipelined kernel {2, 4}; 0 or a value a kernel does not take means
 * automatic.  channel_lanes is accepted for compatibility (0, 8 or 32) and
 * ignored: the lane layout follows from the kernel and the alignment.  The
 * chunk shape changes the workspace size: query sgr_workspace_size after
 * changing it.  Returns SGR_ERR_INVALID_ARG for other values.
 */
SGR_API sgr_status_t sgr_set_tile_override(int channel_lanes, int rows_per_thread);

/*
 * Tuning/testing knob, process-wide: 0 automatic (for aligned vector-width
 * rows: a channel-sequential kernel when the 32-channel groups B x ceil(D / 32)
 * reach 6 per SM -- two warps per group below 24 (bf16) or 32 (fp32) groups
 * per SM, above that one warp per group (fp32) or two warps per group of 64
 * channels (bf16) -- the pipelined kernel otherwise; the tile
 * kernel for anything else), 1 force the tile kernel, 2 pipelined with 7 data
 * warps per block (two blocks per SM), 3 pipelined with 15 data warps (one
 * block per SM, tiles twice as long), 4 channel-sequential with one warp per
 * group of 32 channels walking the whole sequence, 5 channel-sequential with
 * each slot's 16 rows split between the two half-warps of a warp (groups of
 * 16 channels), 6 channel-sequential with two warps per group of 32 channels
 * splitting each 32-row slot, 7 the same with groups of 64 channels, two
 * per lane (bf16 I/O; fp32 takes 6), 8 as 7 with four warps per group, 8
 * rows of each slot each (bf16 I/O; fp32 takes 6); 2-8 wherever the fast
 * path applies.
 */
SGR_API sgr_status_t sgr_set_kernel_override(int kernel);

/* ------------------------------------------------------- introspection */

/* How a scan of this shape is cut into tiles (rows x channels per block). */
typedef struct sgr_plan {
    int32_t vector_path;        /* 1: 128-bit loads; 0: scalar variant            */
    int32_t kernel;             /* 1: one block per tile; 2: pipelined persistent,
                                   7 data warps; 3: pipelined, 15 data warps;
                                   4: channel-sequential, one warp per channel
                                   group and the whole of T (one chunk; warps =
                                   warps per block, stages = load-ring slots);
                                   5: the same with 16-channel groups, the rows
                                   of each slot split between half-warps;
                                   6: two warps per 32-channel group, each slot
                                   of 32 rows split between them; 7: the same
                                   with 64-channel groups, two channels per
                                   lane (bf16); 8: as 7 with four warps per
                                   group, 8 rows of each slot per warp          */
    int32_t channels_per_thread;
    int32_t channel_lanes;      /* lanes across D per warp                         */
    int32_t rows_per_thread;
    int32_t warps;              /* data warps per block (plus one carry warp)      */
    int32_t threads;            /* threads per block                               */
    int32_t stages;             /* pipelined: tiles in flight per block            */
    int64_t tile_rows;          /* rows of T per tile                              */
    int64_t tile_channels;      /* channels of D per tile                          */
    int64_t n_channel_tiles;    /* per batch row                                   */
    int64_t n_chains;           /* B * n_channel_tiles                             */
    int64_t n_chunks;           /* tiles along T                                   */
    int64_t n_tiles;            /* n_chains * n_chunks                             */
    uint64_t smem_bytes;        /* dynamic shared memory per block                 */
    uint64_t workspace_bytes;   /* 256 (the header) when n_chunks == 1             */
    uint64_t off_words;         /* workspace offset of the hand-off words (256)    */
    uint32_t div_chains_m, div_chains_s;  /* tile -> chunk division constants   */
    uint32_t div_dt_m, div_dt_s;          /* chain -> batch division constants  */
} sgr_plan_t;

/* Fill *plan for a scan; `aligned` says whether the operands would be 16-byte
 * aligned.  Pure host code. */
SGR_API sgr_status_t sgr_scan_plan(sgr_op_t op, int64_t B, int64_t T, int64_t D,
                                   sgr_dtype_t dtype, int aligned, sgr_plan_t *plan);

/* The plan of mingru_scan_decay for this shape (the time-decayed minGRU may
 * take another kernel than sgr_scan_plan(SGR_OP_MINGRU, ...) reports, with
 * bf16 I/O only: four warps per 64-channel group from 16 groups of 32
 * channels per SM, and 8 rows per thread in 7-warp blocks of the chunked
 * kernels).  `aligned` as above.
 * Pure host code. */
SGR_API sgr_status_t sgr_scan_plan_decay(int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                                         int aligned, sgr_plan_t *plan);

/* Which kernel the gradient of this shape runs (mingru_scan_backward,
 * minmax_scan_backward and their time-decay forms): 1 the chunked tile kernel
 * (blocks take chunks by ticket), 2 the pipelined gradient (persistent blocks
 * fed by the copy engine; aligned vector-width rows with at least two tiles
 * per block: fp32 two blocks of 6 data warps per SM with 96-row tiles for the
 * decayed gradient and, below 1.5 chains of 32 channels per SM, the plain
 * ones, else one block of 15 data warps per SM with 120-row tiles; the
 * fp32 decayed gradient with too few tiles for two blocks takes one 7-warp
 * block per SM with 112-row tiles, the bf16 one two 7-warp blocks per SM with
 * 56-row tiles from 0.8 chains per SM), 4 the channel-sequential kernel (wide batches, from 5 groups of 32
 * channels per SM: one warp walks the whole sequence of 32 channels
 * backwards); 0 for invalid arguments.
 * `aligned` says whether all six (B, T, D) operands would be 16-byte aligned.
 * Kernel override 2 or 3 forces the pipelined gradient wherever the rows allow
 * it.  Pure host code. */
SGR_API int sgr_backward_kernel(sgr_op_t op, int64_t B, int64_t T, int64_t D, sgr_dtype_t dtype,
                                int aligned);

/* ------------------------------------------------------- testing hooks */

/*
 * Both hooks are process-wide and exist to exercise the bounded wait of the
 * chunk hand-off without faulting or hanging a GPU.
 * sgr_set_wait_limit: polls a chunk makes before it gives up waiting for an
 *   earlier chunk (0 restores the default of 2^18 polls, a fraction of a second).
 * sgr_set_drop_publish: the block with this tile index (chunk * n_chains +
 *   chain) skips publishing its state, so the chunk after it in the same
 *   channels waits until the limit, records SGR_ERR_TIMEOUT in the workspace
 *   status word and writes NaN for its outputs; -1 (the default) disables it.
 */
SGR_API sgr_status_t sgr_set_wait_limit(uint32_t polls);
SGR_API sgr_status_t sgr_set_drop_publish(int64_t tile);

#ifdef __cplusplus
}
#endif

#endif /* SCAN_GATED_RNNS_H */
