/*
 * stepq.h -- C ABI of the B200 (sm_100a) quantised gated Delta-rule decode step.
 *
 * The method is STEPQuant ("STEPQuant: When and Where Errors Matter in
 * Delta-Rule Recurrent State Quantization").  Each request keeps, per head, a
 * recurrent state S (d_k key rows x d_v value columns) stored packed: low-bit
 * integer codes times a row factor and a column factor, S = codes (.) (r c^T),
 * with FP16 "pivot" units kept raw (hyper.ai summary, "Method": symmetric
 * uniform quantisation, FP16 sparse pivots, key-row-aware dual-axis fitting;
 * rcap.io post, decode-step pseudocode).  One decode step of one (request,
 * head) reads the packed state, reconstructs it, applies the gated Delta
 * update, emits the readout y = X^T q before requantising, refits the row and
 * column scales and writes the state back packed (rcap.io post, decode-step
 * pseudocode; hyper.ai summary, "Method", last paragraph: a fused kernel for
 * reconstruction + Delta update + readout, and the dual-axis fit + pack
 * write-back on a separate CUDA stream).
 *
 * Conventions for every entry point:
 *   - returns STEPQ_OK (0) or an error code below; nothing else crosses the
 *     ABI (no exceptions).  stepq_last_error() gives a message for the last
 *     failing call on the calling thread.
 *   - "device" pointers are CUDA device (or managed) memory of the current
 *     device; "host" pointers are ordinary host memory.  All arrays are dense,
 *     C order, and must be aligned to 16 bytes.
 *   - `stream` arguments are cudaStream_t values passed as void* (NULL = the
 *     legacy default stream).  Device work is enqueued asynchronously; a
 *     call returns once its kernels are launched.
 *   - argument errors are reported as STEPQ_ERR_INVALID before anything is
 *     launched; CUDA launch errors as STEPQ_ERR_CUDA.  Errors found by the
 *     kernels themselves (a slot index outside the pool, a non-finite updated
 *     state, a device wait that gave up) are recorded in the pool's device
 *     status word, read with stepq_get_status().
 *   - the library allocates device memory only in stepq_plan_create (its
 *     tables) and stepq_pool_alloc (a status word); every buffer passed in
 *     stays owned by the caller.
 */
#ifndef STEPQ_H
#define STEPQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define STEPQ_API __attribute__((visibility("default")))
#else
#define STEPQ_API
#endif

/* ---- status codes ------------------------------------------------------ */
#define STEPQ_OK 0
#define STEPQ_ERR_INVALID 1     /* bad argument, caught on the host          */
#define STEPQ_ERR_CUDA 2        /* a CUDA runtime call or launch failed      */
#define STEPQ_ERR_UNSUPPORTED 3 /* valid but not built for (e.g. d_k != d_v) */

/* ---- bits of the device status word (stepq_get_status) ----------------- */
#define STEPQ_DEV_BAD_SLOT 1u   /* a slot index was outside [0, num_slots); that head was skipped */
#define STEPQ_DEV_NONFINITE 2u  /* an updated state row held NaN/Inf; it was stored as zeros       */
#define STEPQ_DEV_TIMEOUT 4u    /* a bounded device wait on a bulk copy gave up; head skipped      */

/* ---- enumerations ------------------------------------------------------ */
#define STEPQ_GATE_SCALAR 0     /* D = g I, one gate per (request, head)       (GDN) */
#define STEPQ_GATE_DIAG 1       /* D = diag(g), one gate per key row           (KDA) */
#define STEPQ_UNIT_HEAD 0       /* bit width chosen per head                         */
#define STEPQ_UNIT_ROW 1        /* bit width chosen per key row                      */
#define STEPQ_MODE_STEPQUANT 0  /* key-row-aware dual-axis fit (the method)          */
#define STEPQ_MODE_UNIFORM 1    /* uniform INT-b comparator: per-row absmax, c = 1   */
#define STEPQ_DTYPE_F32 0       /* q, k, v given as float32                          */
#define STEPQ_DTYPE_BF16 1      /* q, k, v given as bfloat16                         */

/*
 * Plan description: what the offline lifetime-aware bit allocation and pivot
 * selection hand to the runtime (hyper.ai summary, "Method": allocation and
 * FP16 pivot selection run offline, so no per-token allocation cost), plus the
 * calibrated row-impact weights (hyper.ai summary, "Method": row-impact score
 * per key row).
 *
 *   d_k, d_v   state shape per head; the library runs d_k == d_v in {64, 128}
 *              (others: STEPQ_ERR_UNSUPPORTED).
 *   n_heads    heads per layer, >= 1.
 *   gate_kind  STEPQ_GATE_SCALAR or STEPQ_GATE_DIAG.
 *   unit_kind  STEPQ_UNIT_HEAD: bits has n_heads entries;
 *              STEPQ_UNIT_ROW:  bits has n_heads * d_k entries.
 *   mode       STEPQ_MODE_STEPQUANT or STEPQ_MODE_UNIFORM.
 *   bits       host, per unit: 4, 6 or 8 (code width) or 16 (FP16 pivot).
 *   w          host, [n_heads][d_k] row-impact weights, finite and > 0.
 * Both arrays are copied; the caller keeps ownership.
 */
typedef struct stepq_plan_desc {
    int32_t d_k;
    int32_t d_v;
    int32_t n_heads;
    int32_t gate_kind;
    int32_t unit_kind;
    int32_t mode;
    const uint8_t *bits;
    const float *w;
} stepq_plan_desc;

typedef struct stepq_plan stepq_plan;
typedef struct stepq_pool stepq_pool;

/*
 * Create a plan: validates the description, computes the packed byte layout
 * of one slot and uploads the per-head / per-row tables to the current device.
 *
 * Layout of one slot (the pages give no byte format; this one is the library's own):
 * the heads' blobs in head order, each starting on a 16-byte boundary; the
 * slot stride is their total rounded up to 256 bytes.  A head blob is its key
 * rows in ascending order -- a b-bit row holds d_v codes stored as
 * code + 2^(b-1) in b bits each, LSB-first in the row's little-endian bit
 * string; an FP16 pivot row holds d_v halves -- followed by rho[d_k] and
 * c[d_v] as little-endian IEEE halves.  A head whose unit is an FP16 pivot is
 * d_k*d_v halves, row-major, with no scales.
 *
 * Ownership: the plan is library-owned; release with stepq_plan_destroy.
 * Errors: STEPQ_ERR_INVALID (bad description), STEPQ_ERR_UNSUPPORTED (shape),
 * STEPQ_ERR_CUDA (device allocation / copy failed).
 */
STEPQ_API int stepq_plan_create(const stepq_plan_desc *desc, stepq_plan **out);
STEPQ_API int stepq_plan_destroy(stepq_plan *plan);

/* Bytes of one slot (the pool's stride). */
STEPQ_API int stepq_plan_slot_bytes(const stepq_plan *plan, size_t *out);

/* Byte offset and size of head `head`'s blob inside a slot. */
STEPQ_API int stepq_plan_head_layout(const stepq_plan *plan, int32_t head, size_t *offset,
                                     size_t *bytes);

/*
 * Pool: a view over caller-owned device memory holding num_slots slots, one
 * per concurrent request ("integrated into the recurrent state pool", hyper.ai
 * summary, "Method", last paragraph).
 *   dev_buf    device, >= num_slots * slot_bytes bytes, 256-byte aligned.
 * The library allocates a 4-byte device status word, five CUDA events and two
 * CUDA streams (the copies of stepq_decode_step_host) for the pool;
 * stepq_pool_free releases those, never dev_buf.
 * Errors: STEPQ_ERR_INVALID (NULL, too small, misaligned), STEPQ_ERR_CUDA.
 */
STEPQ_API int stepq_pool_alloc(const stepq_plan *plan, int64_t num_slots, void *dev_buf,
                               size_t buf_bytes, stepq_pool **out);
STEPQ_API int stepq_pool_free(stepq_pool *pool);

/*
 * Pack: quantise the given states X and write them into slots (admitting a
 * request's state into the pool).  The quantiser is the one the decode step
 * applies to the updated state (rcap.io post, decode-step pseudocode, the
 * scale-fitting and quantise steps).
 *   slot_idx  device int32 [n], distinct, in [0, num_slots).
 *   X         device float32 [n][n_heads][d_k][d_v].
 */
STEPQ_API int stepq_pack(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                         int64_t n, const float *X, void *stream);

/*
 * Unpack: reconstruct S = codes (.) (r c^T) (pivots raw) of the given slots
 * (rcap.io post, decode-step pseudocode, its unpack step).
 *   S_out     device float32 [n][n_heads][d_k][d_v].
 */
STEPQ_API int stepq_unpack(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                           int64_t n, float *S_out, void *stream);

/* Device workspace the decode step needs for n requests (the delta vector
 * handed from the readout kernel to the fit kernel): n * n_heads * d_v floats. */
STEPQ_API int stepq_workspace_bytes(const stepq_plan *plan, int64_t n, size_t *out);

/*
 * Readout half of the step (the fused kernel of hyper.ai summary, "Method",
 * last paragraph): per (request, head) it reconstructs the packed state,
 * forms u = (D S)^T k, delta = beta (v - u), and writes
 * y = X^T q = (D S)^T q + (k.q) delta with X = D S + k delta^T (the gated
 * Delta update, rcap.io post, decode-step pseudocode, its update and readout steps).
 *   qkv_dtype STEPQ_DTYPE_F32 or STEPQ_DTYPE_BF16.
 *   q, k      device [n][n_heads][d_k];  v device [n][n_heads][d_v].
 *   beta      device float32 [n][n_heads].
 *   gate      device float32 [n][n_heads] (scalar) or [n][n_heads][d_k] (diag).
 *   y         device float32 [n][n_heads][d_v] (written).
 *   workspace device, >= stepq_workspace_bytes(n); delta is written there.
 * The slots are only read.
 */
STEPQ_API int stepq_decode_readout(const stepq_plan *plan, stepq_pool *pool,
                                   const int32_t *slot_idx, int64_t n, int32_t qkv_dtype,
                                   const void *q, const void *k, const void *v,
                                   const float *beta, const float *gate, float *y,
                                   void *workspace, size_t ws_bytes, void *stream);

/*
 * Fit-and-pack half of the step (hyper.ai summary, "Method", last paragraph:
 * key-row-aware dual-axis fitting and pack write-back): per (request, head) it
 * rebuilds X = D S + k delta^T from the still-untouched packed state and the
 * delta left in `workspace` by stepq_decode_readout, fits the row factors
 * r_i = sqrt(max_j |X_ij|) / sqrt(w_i) and the column scales by the
 * 8-candidate impact-weighted least-squares search, and writes the codes
 * clamp(rne(X / (r c)), +-qmax) back into the same slot.
 * Must run after the readout of the same step has finished (same stream, or
 * an event); k, gate and workspace must still hold that step's values.
 */
STEPQ_API int stepq_decode_fitpack(const stepq_plan *plan, stepq_pool *pool,
                                   const int32_t *slot_idx, int64_t n, int32_t qkv_dtype,
                                   const void *k, const float *gate, void *workspace,
                                   size_t ws_bytes, void *stream);

/*
 * One whole decode step: readout on `main_stream`, then -- after an event --
 * fit + pack on `side_stream`, so the caller's later work on `main_stream`
 * (the next layer) overlaps the requantisation (hyper.ai summary, "Method",
 * last paragraph; rcap.io post, "Calibration" paragraph).  y is ready in
 * stream order on main_stream.  The call first makes main_stream wait for the
 * previous step's fit on this pool, so back-to-back steps are safe.  With
 * side_stream == main_stream (or NULL) both halves run on main_stream.
 * Arguments as for the two halves.  Slots must be distinct within one call.
 * A batch whose packed state exceeds 48 MB is stepped in chunks of requests
 * (a multiple of 16 each): chunk by chunk, the readout on main_stream, an
 * event, that chunk's fit + pack on side_stream -- so the fit re-reads the
 * slots while they are still in L2 and the next chunk's readout overlaps it.
 * The results are those of one launch of each half.
 * The fit still reads k, gate and workspace after the call returns: do not
 * overwrite them, or hand the same workspace to another pool's step, until
 * side_stream has finished this step (one workspace per layer in flight).
 * Streams: the fits of different pools (layers) are independent, so a caller
 * may give consecutive layers different side streams; one layer's fit then
 * fills the SMs its predecessor's last CTAs leave idle.  A main_stream of
 * higher priority than the side streams lets each readout (which produces y)
 * take SMs ahead of pending fit CTAs.
 */
STEPQ_API int stepq_decode_step(const stepq_plan *plan, stepq_pool *pool,
                                const int32_t *slot_idx, int64_t n, int32_t qkv_dtype,
                                const void *q, const void *k, const void *v, const float *beta,
                                const float *gate, float *y, void *workspace, size_t ws_bytes,
                                void *main_stream, void *side_stream);

/*
 * The same whole step for callers whose per-token inputs live in host memory
 * (a C caller without a device allocator of its own for them): the call
 * copies q, k, v, beta and gate host -> device into `workspace`, runs
 * stepq_decode_step, and copies y device -> host.  The copies run on two
 * streams the pool owns (created and destroyed with it): the input copies
 * wait only for this pool's previous fit, not for
 * earlier work on main_stream, so they overlap the work of the layers before
 * this one; main_stream waits for them before the readout, and for the copy
 * of y after it.  So the host inputs may be reused, and y_host is valid, once
 * main_stream has reached the end of the call's work; the workspace is the
 * pool's staging area until the call's fit has finished (one workspace per
 * layer in flight, as for stepq_decode_step).  Host buffers should be pinned
 * (cudaHostAlloc) for the copies to be asynchronous.
 *   q_host..gate_host, y_host: host, same shapes and types as for
 *             stepq_decode_step.
 *   workspace device, >= stepq_host_workspace_bytes(plan, n, qkv_dtype).
 */
STEPQ_API int stepq_host_workspace_bytes(const stepq_plan *plan, int64_t n, int32_t qkv_dtype,
                                         size_t *out);
STEPQ_API int stepq_decode_step_host(const stepq_plan *plan, stepq_pool *pool,
                                     const int32_t *slot_idx, int64_t n, int32_t qkv_dtype,
                                     const void *q_host, const void *k_host, const void *v_host,
                                     const float *beta_host, const float *gate_host,
                                     float *y_host, void *workspace, size_t ws_bytes,
                                     void *main_stream, void *side_stream);

/*
 * The unquantised baseline: the same gated Delta update and readout on an
 * fp32 state pool, read and written in full (the FP32-state update the pages
 * compare against, rcap.io post, results paragraph).
 *   S          device float32 [num_slots][n_heads][d_k][d_v], updated in place.
 *   dev_status device uint32 word for STEPQ_DEV_BAD_SLOT, or NULL.
 * Other arguments as for stepq_decode_readout.
 */
STEPQ_API int stepq_fp32_step(int32_t d_k, int32_t d_v, int32_t n_heads, int32_t gate_kind,
                              int32_t qkv_dtype, float *S, int64_t num_slots,
                              const int32_t *slot_idx, int64_t n, const void *q, const void *k,
                              const void *v, const float *beta, const float *gate, float *y,
                              uint32_t *dev_status, void *stream);

/*
 * The whole decode step with no device allocation anywhere: the same kernels
 * and arguments as stepq_decode_step, minus the workspace.  (Not a step of
 * the paper's method: it exists for callers that cannot allocate device
 * memory -- a framework whose caching allocator owns all of it, a process
 * that may not grow its device footprint after start-up, a C caller with no
 * allocator.)  The delta vector handed from the readout to the fit kernel is
 * kept in a fixed array inside the library's device image, 4 MiB on every
 * GPU that loads the library, held until the process exits.
 *   - n * n_heads * d_v must not exceed STEPQ_STATIC_DELTA_FLOATS, else
 *     STEPQ_ERR_INVALID and nothing is launched.
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and keeps it for that device's current context;
 *     a call after the context changed (e.g. after cudaDeviceReset) looks it
 *     up again.  Make the first call on a device, and the first after a
 *     reset, before any stream capture.
 *   - every call shares the one array: calls whose kernels can overlap on the
 *     GPU (another stream, or the fit of the previous call on side_stream
 *     still running when the next call's readout starts on a different pool)
 *     race on it.  Serialise them, e.g. pass side_stream == main_stream.
 */
#define STEPQ_STATIC_DELTA_FLOATS 1048576
STEPQ_API int stepq_decode_step_static(const stepq_plan *plan, stepq_pool *pool,
                                       const int32_t *slot_idx, int64_t n, int32_t qkv_dtype,
                                       const void *q, const void *k, const void *v,
                                       const float *beta, const float *gate, float *y,
                                       void *main_stream, void *side_stream);

/* ------------------------------------------------------------------------
 * Offline calibration: lifetime-aware bit allocation.  hyper.ai summary,
 * section "Method" (the Lifetime-Aware Bit Allocation paragraph); rcap.io
 * post, "Temporal" part: before decoding, each state unit (a head, or one key
 * row) gets a width from {4, 6, 8} bits, or FP16 as a pivot, from its
 * reconstruction distortion at each width and its memory lifetime, under an
 * average bit budget.  The three calls below are the measurement, the
 * lifetime weight and the selection; a calibration run strings them together
 * (quantise calibration states with a plan of one width per call to
 * stepq_pack, measure, repeat for each width, then select).
 * ------------------------------------------------------------------------ */

/* Per-unit squared reconstruction error of packed slots against the states
 * they were packed from: dist[r][u] = sum over unit u's entries of
 * (X[r] - S[r])^2, S the state reconstructed from the slot slot_idx[r], each
 * difference and square in double.  Units follow the plan: one per head
 * (unit_kind HEAD, dist is [n][n_heads]) or one per key row (unit_kind ROW,
 * [n][n_heads * d_k], row i of head h at h * d_k + i).
 *   X     device, fp32 [n][n_heads][d_k][d_v] (caller-owned, read only)
 *   dist  device, float64 [n][units] (caller-owned, written)
 * Asynchronous on `stream`.  A slot index outside the pool sets
 * STEPQ_DEV_BAD_SLOT and leaves that request's entries of dist unwritten.
 * The summation order inside a unit is the kernel's own (a tree over
 * columns, then rows in ascending order). */
STEPQ_API int stepq_unit_distortion(const stepq_plan *plan, stepq_pool *pool,
                                    const int32_t *slot_idx, int64_t n, const float *X,
                                    double *dist, void *stream);

/* The same distortion summed over the n requests and added on the device to
 * dist_sum (the calibration total over all calibration states; hyper.ai
 * summary, Method, the Lifetime-Aware Bit Allocation paragraph):
 * dist_sum[u] += sum_r (X[r] - S[r])^2 over unit u's entries.
 *   dist_sum  device, float64 [units] (caller-owned, read and written;
 *             zero it before the first call of a calibration)
 * Other arguments as for stepq_unit_distortion.  The order in which the
 * requests' contributions are added is not fixed (double-precision atomic
 * adds), so repeated runs may differ in the last bits. */
STEPQ_API int stepq_unit_distortion_accumulate(const stepq_plan *plan, stepq_pool *pool,
                                               const int32_t *slot_idx, int64_t n, const float *X,
                                               double *dist_sum, void *stream);

/* Lifetime weight of each unit from its retention gates over calibration
 * steps: ell_u = mean of log(g) over the unit's gates and the steps, the error
 * left after j updates is exp(j ell_u), and the weight is
 * sum_{j >= 0} exp(j ell_u) = 1 / (1 - exp(ell_u)).
 *   gate    host, fp32 [n_steps][n_units][gates_per_unit], every value in (0, 1)
 *   weight  host, float64 [n_units]
 * Host-only (no device work).  STEPQ_ERR_INVALID if a gate is outside (0, 1)
 * or a size is not positive; nothing is written then. */
STEPQ_API int stepq_lifetime_weight(int64_t n_units, int64_t n_steps, int32_t gates_per_unit,
                                    const float *gate, double *weight);

/* Widths minimising the lifetime-weighted distortion under an average budget.
 *   weight  host, float64 [n_units] (stepq_lifetime_weight), > 0 and finite
 *   dist    host, float64 [n_units][3]: distortion at 4, 6, 8 bits, >= 0, finite
 *   budget_bits  4, 6 or 8: the average width of the non-pivot units may not
 *           exceed it
 *   n_pivots  units kept in FP16: those of largest risk weight * dist(budget
 *           width), ties to the lower unit index
 *   bits    host, uint8 [n_units]: 4, 6, 8, or 16 for a pivot (written)
 * The other units' widths are the exact minimum of sum weight_u * dist_u(b_u)
 * subject to sum b_u <= budget_bits * (n_units - n_pivots), taken by a
 * recurrence over units in ascending order with the number of 2-bit upgrades
 * left as its state; on equal sums the earlier unit takes the smaller width.
 * Host-only; memory O(n_units^2) bytes for budget 6 (16.8 MB at 4096 units).
 * STEPQ_ERR_INVALID on bad arguments (nothing written). */
STEPQ_API int stepq_allocate_bits(int64_t n_units, const double *weight, const double *dist,
                                  int32_t budget_bits, int64_t n_pivots, uint8_t *bits);

/* ------------------------------------------------------------------------
 * Offline calibration: row-impact weights.  hyper.ai summary, section
 * "Method", the paragraphs on the spatial distribution of errors and on
 * key-row-aware dual-axis fitting: the impact of a key row is the expectation,
 * over calibration tokens, of the square of the factor through which an error
 * in that row reaches the readout; it weights the row factors and the column
 * fit (the plan's w).
 * ------------------------------------------------------------------------ */

/* Add, for every (head, key row), the squared weighting factor over n
 * calibration inputs (requests x tokens):
 *     score_sum[h][i] += sum_r ((A_r^T q_r)_i)^2,
 *     A_r = (I - beta_r k_r k_r^T) D_r   (the transition of the step that
 *     reads the stored state), i.e. (A^T q)_i = g_i (q_i - beta k_i (k . q)).
 *   q, k       device, [n][n_heads][d_k] in qkv_dtype (STEPQ_DTYPE_F32 / _BF16)
 *   beta       device, fp32 [n][n_heads]
 *   gate       device, fp32 [n][n_heads] (STEPQ_GATE_SCALAR) or
 *              [n][n_heads][d_k] (STEPQ_GATE_DIAG)
 *   score_sum  device, float64 [n_heads][d_k], read and written (caller zeroes
 *              it before the first call)
 * Arithmetic in double from the input values; per head the inputs are taken
 * in ascending order.  Asynchronous on `stream`; d_k in {64, 128}. */
STEPQ_API int stepq_row_impact(int32_t d_k, int32_t n_heads, int32_t gate_kind, int32_t qkv_dtype,
                               int64_t n, const void *q, const void *k, const float *beta,
                               const float *gate, double *score_sum, void *stream);

/* The plan's row-impact weights from the accumulated scores:
 * w[i] = sqrt(score_sum[i] / count), rounded to fp32, so that the column fit's
 * weight w^2 is the mean squared weighting factor.
 *   score_sum  host, float64 [n_rows]; every entry finite and > 0
 *   w          host, fp32 [n_rows] (written)
 * Host-only.  STEPQ_ERR_INVALID on bad arguments (nothing written). */
STEPQ_API int stepq_impact_weights(int64_t n_rows, int64_t count, const double *score_sum, float *w);

/* Synchronously read the pool's device status word (STEPQ_DEV_* bits, OR-ed
 * over every call since the last clear).  Waits for the device to go idle. */
STEPQ_API int stepq_get_status(stepq_pool *pool, uint32_t *out);

/* Reset the pool's status word to 0, in stream order. */
STEPQ_API int stepq_clear_status(stepq_pool *pool, void *stream);

/*
 * Failure-detection test hook (not a step of the paper's method).  Every
 * device wait of the library is bounded: a kernel that waits on a
 * bulk-async copy gives up after a time limit, records STEPQ_DEV_TIMEOUT in
 * the pool's status word and skips that head, leaving the GPU usable.  To
 * let a test make such a wait run out without any fault, this call switches
 * the readout and fit kernels of this pool's later calls to a mode in which
 * they issue no staging copy at all (nothing is in flight) and wait at most
 * wait_limit_us microseconds per wait; their heads are then skipped: y,
 * the workspace and the pool's slots are left as they were.
 *   flags         STEPQ_TEST_NO_STAGING_COPY, or 0 to restore normal
 *                 operation (the default limit, 2 s).
 *   wait_limit_us 1 .. 1000000 when flags != 0.
 * STEPQ_ERR_INVALID on bad arguments.  Host-only; takes effect for calls
 * made after it returns.
 */
#define STEPQ_TEST_NO_STAGING_COPY 1u
STEPQ_API int stepq_pool_set_test_faults(stepq_pool *pool, uint32_t flags, uint32_t wait_limit_us);

/* Message for the last failing call on this thread ("" if none). */
STEPQ_API const char *stepq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* STEPQ_H */
