/*
 * mamba_scan.h -- C ABI of libmambascan, the B200 (sm_100a) fused selective
 * scan (S6).
 *
 * The operation (forward) follows "Mamba: Linear-Time Sequence Modeling with
 * Selective State Spaces" (chapterpal.com), Knowl 1 "Selective State Space
 * Layer (S6)" (steps 2-4 and its per-element loop), with the softplus of
 * section 3.4 "The specific functional forms" and the SiLU gate branch of
 * "The Mamba Architecture" on the paper-graph-ui summary page.  For every
 * batch b and channel d, with an N-dimensional diagonal state h (h = 0 before
 * the first step):
 *
 *     Delta_t = softplus(delta[b,d,t] + delta_bias[d])
 *     Abar_tn = exp(Delta_t * A[d,n])
 *     Bbar_tn = (exp(Delta_t * A[d,n]) - 1) / A[d,n] * B[b,n,t]   (Delta_t*B at A = 0)
 *     h_tn    = Abar_tn * h_{t-1,n} + Bbar_tn * u[b,d,t]
 *     y[b,d,t] = (sum_n C[b,n,t] * h_tn + D[d] * u[b,d,t]) * silu(z[b,d,t])
 *     last_state[b,d,n] = h_{L-1,n}
 *
 * The backward recomputes the states from the inputs instead of reading
 * stored ones (the recomputation of section 3.3 of the paper-graph-ui page and
 * Part III section 4 of the trishampatil.com walk-through) and returns the
 * gradients of sum(dy * y) with respect to every input.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device, owned
 *    by the caller.  The library never frees them and keeps no reference after
 *    the call returns.  Tensors are dense and contiguous in the stated layout
 *    (last index fastest) and aligned to their element size; 16-byte aligned
 *    tensors whose rows are 16-byte multiples take the fastest kernels.
 *  - `dtype` selects the I/O type of u, delta, z, B, C, y, dy, du, ddelta, dz,
 *    dB and dC.  A, D, delta_bias, last_state, dA, dD and ddelta_bias are
 *    always float32.  Arithmetic is float32 throughout; bf16 values are
 *    widened exactly on load and rounded to nearest-even once on store.
 *  - Calls only enqueue work on `stream` (NULL = the legacy default stream)
 *    and return.  The status reports argument validation and launch errors.
 *    Errors raised later on the device (a bounded wait that expired) are
 *    recorded in a per-device sticky error word read by
 *    mamba_scan_stream_status().
 *  - Temporary device memory (chunk-boundary states, partial sums) is taken
 *    stream-ordered on `stream` from a memory pool the library creates once
 *    per device; the pool keeps up to 4 GiB reserved between calls (until the
 *    process exits) so that repeated calls do not re-map it.  Failure returns
 *    MAMBA_ERR_OUT_OF_MEMORY.
 *  - Outputs are overwritten, never accumulated into.  No exception, abort,
 *    printf or trap crosses or happens behind this interface.  Calls are
 *    thread-safe; concurrent calls on different streams are independent.
 *  - batch, dim or L equal to 0 is an empty problem: nothing is computed, and
 *    outputs of size 0 are left alone; last_state (L = 0) is set to 0 and the
 *    parameter gradients dA, dD, ddelta_bias are set to 0.
 */
#ifndef MAMBA_SCAN_H
#define MAMBA_SCAN_H

#include <stdint.h>

#if defined(__GNUC__)
#define MAMBA_SCAN_API __attribute__((visibility("default")))
#else
#define MAMBA_SCAN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *mamba_stream_t;

typedef enum { MAMBA_F32 = 0, MAMBA_BF16 = 1 } mamba_dtype_t;

typedef enum {
  MAMBA_OK = 0,
  MAMBA_ERR_INVALID_ARG = 1,   /* null/misaligned/overlapping/host pointer, bad size */
  MAMBA_ERR_UNSUPPORTED = 2,   /* N outside 1..16, or a shape beyond the limits */
  MAMBA_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed */
  MAMBA_ERR_OUT_OF_MEMORY = 4, /* the stream-ordered workspace could not be allocated */
  MAMBA_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait expired (sticky) */
  MAMBA_ERR_OUT_OF_BOUNDS = 6   /* bounds-checking build only: a kernel computed an index
                                   outside its buffer and skipped the access (sticky) */
} mamba_status_t;

/* Kernel-path selection for mamba_scan_fwd_ex / mamba_scan_bwd_ex. */
typedef enum {
  MAMBA_PATH_AUTO = 0,       /* pick by shape and A (the default of the plain calls) */
  MAMBA_PATH_REFERENCE = 1,  /* one thread per channel, plain loads, any A */
  MAMBA_PATH_GENERIC = 2,    /* staged, chunked kernel, one exp per state element */
  MAMBA_PATH_STRUCTURED = 3  /* staged, chunked kernel for A[d,n] = (n+1)*A[d,0] < 0;
                                channels that do not have this form fall back to the
                                generic arithmetic inside the same launch */
} mamba_path_t;

typedef struct {
  int32_t path;            /* a mamba_path_t */
  int32_t chunk_len;       /* time steps per chunk of the chunked kernels; 0 = automatic,
                              else a positive multiple of 64 */
  int32_t carry;           /* how a chunk's end state (in the backward: the adjoint entering
                              from the later chunk) crosses chunk boundaries: 0 = automatic
                              (sequential when the channel groups fill the GPU),
                              1 = sequential hand-off (a bounded wait on the neighbour),
                              2 = three-phase (chunk aggregates, a scan over chunks, then every
                              chunk from its true entering value) */
  int32_t wait_timeout_us; /* bound of every device-side wait; 0 = 2,000,000 (2 s) */
  int32_t test_hook;       /* 0 in normal use.  1: the first chunk processed of the first
                              channel group (the first in time for the forward, the last for
                              the backward) never publishes its state, so that the waits on
                              it expire (tests MAMBA_ERR_DEVICE_TIMEOUT; outputs undefined) */
  int32_t reserved[3];     /* must be 0 */
} mamba_scan_options_t;

/*
 * Forward.
 *   u, delta, z, y : (batch, dim, L), dtype
 *   B, C           : (batch, N, L), dtype (input-dependent, one row per step)
 *   A              : (dim, N) float32 (diagonal of the state matrix per channel)
 *   delta_bias, D  : (dim) float32
 *   last_state     : (batch, dim, N) float32, the state after step L-1
 * Nullable: delta_bias (treated as 0), D (no skip), z (no gate), last_state
 * (not written).  1 <= N <= 16.
 */
MAMBA_SCAN_API mamba_status_t mamba_scan_fwd(const void *u, const void *delta, const float *delta_bias,
                              const float *A, const void *B, const void *C, const float *D,
                              const void *z, void *y, float *last_state, int64_t batch,
                              int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                              mamba_stream_t stream);

/* Forward with an explicit kernel path (options may be NULL = defaults). */
MAMBA_SCAN_API mamba_status_t mamba_scan_fwd_ex(const void *u, const void *delta, const float *delta_bias,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, void *y, float *last_state, int64_t batch,
                                 int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                 const mamba_scan_options_t *options, mamba_stream_t stream);

/*
 * Backward of the scalar sum(dy * y), recomputing the states from the inputs.
 *   inputs as in mamba_scan_fwd, plus dy : (batch, dim, L) dtype
 *   du, ddelta, dz : (batch, dim, L) dtype
 *   dB, dC         : (batch, N, L) dtype (summed over channels)
 *   dA             : (dim, N) float32, dD, ddelta_bias : (dim) float32
 *                    (summed over batch and time)
 * dz must be non-NULL exactly when z is, dD exactly when D is; ddelta_bias
 * may be NULL.  The reductions run in a fixed order: results are bitwise
 * reproducible run to run on the same device and shape.
 */
MAMBA_SCAN_API mamba_status_t mamba_scan_bwd(const void *u, const void *delta, const float *delta_bias,
                              const float *A, const void *B, const void *C, const float *D,
                              const void *z, const void *dy, void *du, void *ddelta, float *dA,
                              void *dB, void *dC, float *dD, void *dz, float *ddelta_bias,
                              int64_t batch, int64_t dim, int64_t L, int64_t N,
                              mamba_dtype_t dtype, mamba_stream_t stream);

MAMBA_SCAN_API mamba_status_t mamba_scan_bwd_ex(const void *u, const void *delta, const float *delta_bias,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, const void *dy, void *du, void *ddelta,
                                 float *dA, void *dB, void *dC, float *dD, void *dz,
                                 float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                 int64_t N, mamba_dtype_t dtype,
                                 const mamba_scan_options_t *options, mamba_stream_t stream);

/*
 * The training pair: a forward that also stores what its backward would
 * otherwise recompute, and a backward that reads it.  The recurrence is the
 * one of mamba_scan_fwd ("Mamba: Linear-Time Sequence Modeling with Selective
 * State Spaces", chapterpal.com, Knowl 1 "Selective State Space Model (S6)",
 * the discretized recurrence; the backward as mamba_scan_bwd).  The stored
 * states are the recurrence's h before every 16th step (for the three-phase
 * carry: h from a zero state at each chunk start, with the chunk's entering
 * state and the running sum of delta needed to complete it), so the backward
 * skips the forward pass it would run first and re-runs only 16-step tiles.
 *
 * mamba_scan_saved_bytes writes into *bytes the size of the buffer `saved`
 * for this shape, dtype and options on the current device.  It is 0 when the
 * problem takes the one-thread-per-channel kernels (path REFERENCE, N <= 2,
 * or rows of L * dtype size not a multiple of 16 bytes); the two calls are
 * then mamba_scan_fwd_ex and mamba_scan_bwd_ex and `saved` may be NULL.
 *
 * mamba_scan_fwd_save: mamba_scan_fwd_ex (same arguments and results), and
 * writes `saved` (device memory, 16-byte aligned, saved_bytes >= the size
 * above; its contents are opaque).  With a nonzero size the staged kernels
 * must take the call: u, delta, z, y, B and C 16-byte aligned, else
 * MAMBA_ERR_INVALID_ARG (nothing enqueued).
 *
 * mamba_scan_bwd_saved: mamba_scan_bwd_ex (same arguments and results),
 * reading `saved` as written by mamba_scan_fwd_save with the same u, delta,
 * delta_bias, A, B, C, shape, dtype and options on the same device (any z,
 * D and y; the stored states do not depend on them).  Stream order must put
 * the forward before it; `saved` is not modified and may serve several
 * backwards.  Anything else in `saved` gives undefined gradients.  The
 * saved states are those the recomputing backward forms, by the same
 * formulas on the same chunking when chunk_len and carry are automatic, so
 * the gradients agree with mamba_scan_bwd_ex to rounding (bit for bit where
 * the compiler forms both alike; the recomputing backward's own forward pass
 * takes the automatic chunking whatever the options).  The convolution
 * prologue, the fused Delta projection and complex A have the pair too
 * (mamba_conv_scan_fwd_save, mamba_dtproj_scan_fwd_save,
 * mamba_cplx_scan_fwd_save and their companions).
 */
MAMBA_SCAN_API mamba_status_t mamba_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L, int64_t N,
                                                     mamba_dtype_t dtype,
                                                     const mamba_scan_options_t *options,
                                                     uint64_t *bytes);

MAMBA_SCAN_API mamba_status_t mamba_scan_fwd_save(const void *u, const void *delta,
                                                  const float *delta_bias, const float *A,
                                                  const void *B, const void *C, const float *D,
                                                  const void *z, void *y, float *last_state,
                                                  int64_t batch, int64_t dim, int64_t L, int64_t N,
                                                  mamba_dtype_t dtype,
                                                  const mamba_scan_options_t *options, void *saved,
                                                  uint64_t saved_bytes, mamba_stream_t stream);

MAMBA_SCAN_API mamba_status_t mamba_scan_bwd_saved(
    const void *u, const void *delta, const float *delta_bias, const float *A, const void *B,
    const void *C, const float *D, const void *z, const void *dy, void *du, void *ddelta, float *dA,
    void *dB, void *dC, float *dD, void *dz, float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
    int64_t N, mamba_dtype_t dtype, const mamba_scan_options_t *options, const void *saved,
    uint64_t saved_bytes, mamba_stream_t stream);

/*
 * Forward with the convolution prologue of the Mamba block: the main branch
 * runs a short causal 1D convolution and SiLU before the S6 layer
 * ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
 * chapterpal.com, Knowl 3 "Mamba Block Architecture", step 3, width
 * d_conv = 4; paper-graph-ui summary, "The Mamba Architecture (Section 3.4)").
 * The pages do not spell the convolution out; it is read as depthwise (one
 * filter per channel), causal (x = 0 before the first step) and with an
 * optional bias:
 *     pre[b,d,t] = conv_b[d] + sum_{k<W} conv_w[d,k] * x[b,d,t-(W-1)+k]
 *     u[b,d,t]   = pre * sigmoid(pre)
 * and u drives the scan of mamba_scan_fwd.  u is computed inside the scan
 * kernels and never stored.
 *   x            : (batch, dim, L) dtype, in place of u
 *   conv_w       : (dim, W) float32, W = conv_width in 1..4 (4 in the Mamba
 *                  block; other widths return MAMBA_ERR_UNSUPPORTED)
 *   conv_b       : (dim) float32, nullable (no bias)
 * Everything else as in mamba_scan_fwd_ex (options may be NULL).
 */
MAMBA_SCAN_API mamba_status_t mamba_conv_scan_fwd(const void *x, const float *conv_w,
                                                  const float *conv_b, int64_t conv_width,
                                                  const void *delta, const float *delta_bias,
                                                  const float *A, const void *B, const void *C,
                                                  const float *D, const void *z, void *y,
                                                  float *last_state, int64_t batch, int64_t dim,
                                                  int64_t L, int64_t N, mamba_dtype_t dtype,
                                                  const mamba_scan_options_t *options,
                                                  mamba_stream_t stream);

/*
 * Backward of sum(dy * y) for mamba_conv_scan_fwd, recomputing the prologue
 * and the states from the inputs.  As mamba_scan_bwd_ex, with
 *   dx           : (batch, dim, L) dtype, the gradient with respect to x (in
 *                  place of du; it also serves as scratch for du, so it must
 *                  not overlap any input)
 *   dconv_w      : (dim, W) float32;  dconv_b : (dim) float32, nullable
 *                  (both summed over batch and time)
 * The scan backward writes du into dx; a second kernel then applies, in
 * place, the chain rule through SiLU and the convolution:
 *     dpre_t = du_t sigmoid(pre_t) (1 + pre_t (1 - sigmoid(pre_t)))
 *     dx[s] = sum_k conv_w[d,k] dpre_{s+(W-1)-k},
 *     dconv_w[d,k] = sum_{b,t} dpre_t x_{t-(W-1)+k},  dconv_b[d] = sum_{b,t} dpre_t.
 * In bf16, du is rounded to bf16 once before that step.  Reductions run in a
 * fixed order (bitwise reproducible).
 */
MAMBA_SCAN_API mamba_status_t mamba_conv_scan_bwd(
    const void *x, const float *conv_w, const float *conv_b, int64_t conv_width,
    const void *delta, const float *delta_bias, const float *A, const void *B, const void *C,
    const float *D, const void *z, const void *dy, void *dx, float *dconv_w, float *dconv_b,
    void *ddelta, float *dA, void *dB, void *dC, float *dD, void *dz, float *ddelta_bias,
    int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
    const mamba_scan_options_t *options, mamba_stream_t stream);

/*
 * The training pair with the convolution prologue: as mamba_scan_saved_bytes,
 * mamba_scan_fwd_save and mamba_scan_bwd_saved, for mamba_conv_scan_fwd and
 * mamba_conv_scan_bwd (same arguments; the stored states are those of the
 * scan driven by u = SiLU(conv(x)), so x, conv_w, conv_b and conv_width must
 * also be those of the forward).  The size depends on conv_width only
 * through its range check.
 */
MAMBA_SCAN_API mamba_status_t mamba_conv_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L,
                                                          int64_t N, int64_t conv_width,
                                                          mamba_dtype_t dtype,
                                                          const mamba_scan_options_t *options,
                                                          uint64_t *bytes);

MAMBA_SCAN_API mamba_status_t mamba_conv_scan_fwd_save(
    const void *x, const float *conv_w, const float *conv_b, int64_t conv_width, const void *delta,
    const float *delta_bias, const float *A, const void *B, const void *C, const float *D,
    const void *z, void *y, float *last_state, int64_t batch, int64_t dim, int64_t L, int64_t N,
    mamba_dtype_t dtype, const mamba_scan_options_t *options, void *saved, uint64_t saved_bytes,
    mamba_stream_t stream);

MAMBA_SCAN_API mamba_status_t mamba_conv_scan_bwd_saved(
    const void *x, const float *conv_w, const float *conv_b, int64_t conv_width,
    const void *delta, const float *delta_bias, const float *A, const void *B, const void *C,
    const float *D, const void *z, const void *dy, void *dx, float *dconv_w, float *dconv_b,
    void *ddelta, float *dA, void *dB, void *dC, float *dD, void *dz, float *ddelta_bias,
    int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
    const mamba_scan_options_t *options, const void *saved, uint64_t saved_bytes,
    mamba_stream_t stream);

/*
 * Forward with the low-rank Delta projection ("Mamba: Linear-Time Sequence
 * Modeling with Selective State Spaces", paper-graph-ui summary, section 3.6
 * "Parameterization of Delta's input projection": s_Delta(x) =
 * Linear_D(Linear_R(x)) with a small rank R).  The caller passes the rank-R
 * projection and the weight of Linear_D instead of delta:
 *     delta[b,d,t] = sum_r W_dt[d,r] * dt_low[b,r,t]
 * and delta_bias is Linear_D's bias (softplus(delta + delta_bias) as before).
 *   dt_low : (batch, R, L) dtype
 *   W_dt   : (dim, R) dtype (the I/O type, like a bf16 layer weight)
 * Everything else as in mamba_scan_fwd_ex.  R in 1..2^20; dim and L below
 * 2^31.  How delta is formed:
 *   - bf16 with R <= 192, the staged kernels' shapes (L a multiple of 8,
 *     16-byte aligned rows) and no MAMBA_PATH_REFERENCE: delta never reaches
 *     memory.  Each CTA keeps its 128 rows of W_dt in tensor memory and forms
 *     every 128-channel x 32-step tile of delta with one tensor-core MMA
 *     (tcgen05, fp32 accumulation) from the dt_low tile that the scan's own
 *     TMA pipeline brings in; the scan uses the fp32 result as it is.
 *   - otherwise: delta is formed first by a CUDA-core contraction (fp32
 *     accumulation, rounded once to the I/O type) into a stream-ordered
 *     workspace of delta's size, and the regular scan reads it.
 * No external library is called.
 */
MAMBA_SCAN_API mamba_status_t mamba_dtproj_scan_fwd(const void *u, const void *dt_low,
                                                    const void *W_dt, int64_t R,
                                                    const float *delta_bias, const float *A,
                                                    const void *B, const void *C, const float *D,
                                                    const void *z, void *y, float *last_state,
                                                    int64_t batch, int64_t dim, int64_t L,
                                                    int64_t N, mamba_dtype_t dtype,
                                                    const mamba_scan_options_t *options,
                                                    mamba_stream_t stream);

/*
 * Backward of sum(dy * y) for mamba_dtproj_scan_fwd.  As mamba_scan_bwd_ex,
 * with d_dt_low (batch, R, L) dtype and dW_dt (dim, R) float32 in place of
 * ddelta:
 *     d_dt_low[b] = W_dt^T . ddelta[b],   dW_dt = sum_b ddelta[b] . dt_low[b]^T
 * where ddelta (the scan backward's gradient of delta, rounded once to the
 * I/O type) lives in a workspace.  dW_dt is accumulated over the batch rows
 * in a fixed order.  Where the forward fuses the projection, so does the
 * backward (delta recomputed per tile on the tensor cores, never stored);
 * otherwise delta comes from the CUDA-core contraction into the workspace.
 * The two products run as tcgen05 GEMMs (bf16 operands, fp32 accumulation;
 * dW_dt's contraction over batch x L split across the grid and the parts
 * summed in a fixed order) for bf16 with R and L multiples of 8, R <= 256 and
 * 16-byte aligned W_dt / dt_low, else on the CUDA cores.
 */
MAMBA_SCAN_API mamba_status_t mamba_dtproj_scan_bwd(
    const void *u, const void *dt_low, const void *W_dt, int64_t R, const float *delta_bias,
    const float *A, const void *B, const void *C, const float *D, const void *z, const void *dy,
    void *du, void *d_dt_low, float *dW_dt, float *dA, void *dB, void *dC, float *dD, void *dz,
    float *ddelta_bias, int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
    const mamba_scan_options_t *options, mamba_stream_t stream);

/*
 * The training pair with the low-rank Delta projection: as
 * mamba_scan_saved_bytes, mamba_scan_fwd_save and mamba_scan_bwd_saved, for
 * mamba_dtproj_scan_fwd and mamba_dtproj_scan_bwd (same arguments; dt_low,
 * W_dt and R must also be those of the forward).  Only the fused kernels
 * (bf16, R <= 192, L a multiple of 8, no MAMBA_PATH_REFERENCE) store or read
 * states, and only on shapes whose backward carries its adjoint across the
 * sequence in one pass: elsewhere mamba_dtproj_scan_saved_bytes gives 0 and
 * the pair behaves as the plain calls.  Where it gives more, the saving
 * forward refuses (MAMBA_ERR_INVALID_ARG, nothing enqueued) a call that the
 * fused kernels cannot take, e.g. a dt_low that is not 16-byte aligned.
 */
MAMBA_SCAN_API mamba_status_t mamba_dtproj_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L,
                                                            int64_t N, int64_t R,
                                                            mamba_dtype_t dtype,
                                                            const mamba_scan_options_t *options,
                                                            uint64_t *bytes);

MAMBA_SCAN_API mamba_status_t mamba_dtproj_scan_fwd_save(
    const void *u, const void *dt_low, const void *W_dt, int64_t R, const float *delta_bias,
    const float *A, const void *B, const void *C, const float *D, const void *z, void *y,
    float *last_state, int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
    const mamba_scan_options_t *options, void *saved, uint64_t saved_bytes, mamba_stream_t stream);

MAMBA_SCAN_API mamba_status_t mamba_dtproj_scan_bwd_saved(
    const void *u, const void *dt_low, const void *W_dt, int64_t R, const float *delta_bias,
    const float *A, const void *B, const void *C, const float *D, const void *z, const void *dy,
    void *du, void *d_dt_low, float *dW_dt, float *dA, void *dB, void *dC, float *dD, void *dz,
    float *ddelta_bias, int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
    const mamba_scan_options_t *options, const void *saved, uint64_t saved_bytes,
    mamba_stream_t stream);

/*
 * Forward with a complex-valued diagonal A ("Mamba: Linear-Time Sequence
 * Modeling with Selective State Spaces", paper-graph-ui summary, section 3.6
 * "Real vs. Complex parameters"; the S4D-Lin initialization A_n = -1/2 + n i
 * of its Table 8 ablation).  A, B, C and the state are complex, u, delta, z
 * and y real; the pages say no more, and the readings are: B_t and C_t are
 * input-dependent complex vectors, the readout keeps the real part:
 *     Abar = exp(Delta A_n),  Bbar = (exp(Delta A_n) - 1) / A_n * B_n,
 *     h_n  = Abar h_n + Bbar u,   y = (Re(sum_n C_n h_n) + D u) * silu(z)
 * A complex vector of N entries is stored planar, real parts first:
 *   A          : (dim, 2N) float32
 *   B, C       : (batch, 2N, L) dtype
 *   last_state : (batch, dim, 2N) float32
 * Everything else as in mamba_scan_fwd.  One thread per (batch, channel)
 * with the B / C rows staged in shared memory; no chunking over time.
 */
MAMBA_SCAN_API mamba_status_t mamba_cplx_scan_fwd(const void *u, const void *delta,
                                                  const float *delta_bias, const float *A,
                                                  const void *B, const void *C, const float *D,
                                                  const void *z, void *y, float *last_state,
                                                  int64_t batch, int64_t dim, int64_t L, int64_t N,
                                                  mamba_dtype_t dtype, mamba_stream_t stream);

/*
 * Backward of sum(dy * y) for mamba_cplx_scan_fwd, recomputing the states.
 * As mamba_scan_bwd, with dA (dim, 2N) float32 and dB, dC (batch, 2N, L)
 * dtype in the planar layout; the gradient of a complex input is the pair
 * (d/d re, d/d im).  Reductions run in a fixed order.
 */
MAMBA_SCAN_API mamba_status_t mamba_cplx_scan_bwd(const void *u, const void *delta,
                                                  const float *delta_bias, const float *A,
                                                  const void *B, const void *C, const float *D,
                                                  const void *z, const void *dy, void *du,
                                                  void *ddelta, float *dA, void *dB, void *dC,
                                                  float *dD, void *dz, float *ddelta_bias,
                                                  int64_t batch, int64_t dim, int64_t L, int64_t N,
                                                  mamba_dtype_t dtype, mamba_stream_t stream);

/*
 * The training pair with complex A: mamba_cplx_scan_fwd_save is
 * mamba_cplx_scan_fwd that also stores the state at the start of every
 * 8-step block (the backward's block checkpoints: (batch*dim, ceil(L/8),
 * 2 NM) fp32, NM = N rounded up to 1, 2, 4, 8 or 16) into `saved` (device
 * memory, 16-byte aligned, at least mamba_cplx_scan_saved_bytes bytes);
 * mamba_cplx_scan_bwd_saved is mamba_cplx_scan_bwd reading them in place of
 * its forward sweep.  `saved` must come from mamba_cplx_scan_fwd_save with
 * the same u, delta, delta_bias, A, B, shape and dtype on the same device,
 * ordered before it on the stream; anything else gives undefined gradients.
 * The gradients are those of mamba_cplx_scan_bwd to rounding (the states are
 * the same recurrence, formed by the forward kernel).  A NULL `saved`, or one
 * smaller than the size, returns MAMBA_ERR_INVALID_ARG with nothing enqueued.
 */
MAMBA_SCAN_API mamba_status_t mamba_cplx_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L,
                                                          int64_t N, mamba_dtype_t dtype,
                                                          uint64_t *bytes);

MAMBA_SCAN_API mamba_status_t mamba_cplx_scan_fwd_save(const void *u, const void *delta,
                                                       const float *delta_bias, const float *A,
                                                       const void *B, const void *C,
                                                       const float *D, const void *z, void *y,
                                                       float *last_state, int64_t batch,
                                                       int64_t dim, int64_t L, int64_t N,
                                                       mamba_dtype_t dtype, void *saved,
                                                       uint64_t saved_bytes,
                                                       mamba_stream_t stream);

MAMBA_SCAN_API mamba_status_t mamba_cplx_scan_bwd_saved(
    const void *u, const void *delta, const float *delta_bias, const float *A, const void *B,
    const void *C, const float *D, const void *z, const void *dy, void *du, void *ddelta, float *dA,
    void *dB, void *dC, float *dD, void *dz, float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
    int64_t N, mamba_dtype_t dtype, const void *saved, uint64_t saved_bytes, mamba_stream_t stream);

/*
 * One decoding step: the recurrent mode of the selective SSM, one token per
 * call with constant work per token ("Mamba: Linear-Time Sequence Modeling
 * with Selective State Spaces", trishampatil.com walk-through, Part II
 * section 4: recurrence for autoregressive inference).  For every batch b
 * and channel d, with state[b,d,:] the state after the previous token:
 *     Delta = softplus(delta[b,d] + delta_bias[d])
 *     state[b,d,n] <- exp(Delta A[d,n]) state[b,d,n]
 *                     + (exp(Delta A[d,n]) - 1)/A[d,n] B[b,n] u[b,d]
 *     y[b,d] = (sum_n C[b,n] state[b,d,n] + D[d] u[b,d]) silu(z[b,d])
 *   state          : (batch, dim, N) float32, read and overwritten in place
 *                    (e.g. the last_state of mamba_scan_fwd over a prompt)
 *   u, delta, z, y : (batch, dim) dtype;  B, C : (batch, N) dtype
 *   A, D, delta_bias as in mamba_scan_fwd.  delta_bias, D and z may be NULL.
 * Repeating the call over the tokens of a sequence gives the same result as
 * mamba_scan_fwd over the whole sequence, up to rounding.
 */
MAMBA_SCAN_API mamba_status_t mamba_scan_step(float *state, const void *u, const void *delta,
                                              const float *delta_bias, const float *A,
                                              const void *B, const void *C, const float *D,
                                              const void *z, void *y, int64_t batch, int64_t dim,
                                              int64_t N, mamba_dtype_t dtype, mamba_stream_t stream);

/*
 * One decoding step of the block with its convolution prologue (the
 * recurrent mode of mamba_conv_scan_fwd).  x is this token's block input
 * (batch, dim) dtype; conv_state (batch, dim, W - 1) float32 holds the
 * previous W - 1 inputs of each channel, oldest first (zeros before the
 * first token; after a prompt, its last W - 1 inputs), and is shifted in
 * place; NULL is allowed only for W = 1.  u = SiLU(conv_b + sum_k conv_w[d,k]
 * (the W inputs ending with x)) then drives the step of mamba_scan_step.
 * Repeating the call over the tokens of a sequence gives the result of
 * mamba_conv_scan_fwd, up to rounding.
 */
MAMBA_SCAN_API mamba_status_t mamba_conv_scan_step(float *state, float *conv_state, const void *x,
                                                   const float *conv_w, const float *conv_b,
                                                   int64_t conv_width, const void *delta,
                                                   const float *delta_bias, const float *A,
                                                   const void *B, const void *C, const float *D,
                                                   const void *z, void *y, int64_t batch,
                                                   int64_t dim, int64_t N, mamba_dtype_t dtype,
                                                   mamba_stream_t stream);

/*
 * Decoding plans: mamba_scan_step / mamba_conv_scan_step with the argument
 * checks done once.  A decoding loop usually steps the same buffers token
 * after token (the state, this token's input slots, y); the plan records
 * them, checks every pointer (device memory of the current device, aligned,
 * no output overlapping an input) and picks the kernel, and each run is then
 * a single kernel launch.  conv_width = 0 plans mamba_scan_step (x is u, and
 * conv_state, conv_w, conv_b must be NULL); 1..4 plans mamba_conv_scan_step.
 * All other arguments as there.  The plan holds only host memory and the
 * pointers given: the caller keeps the buffers alive and unmoved while it
 * runs the plan, and writes each token's values into them between runs (on
 * the run's stream, or ordered with it).  A run on another device than the
 * creating call's returns MAMBA_ERR_INVALID_ARG; runs of one plan on streams
 * that overlap race on the state.  Destroying NULL does nothing.
 */
typedef struct mamba_step_plan_st *mamba_step_plan_t;

MAMBA_SCAN_API mamba_status_t mamba_scan_step_plan_create(
    mamba_step_plan_t *plan, float *state, float *conv_state, const void *x, const float *conv_w,
    const float *conv_b, int64_t conv_width, const void *delta, const float *delta_bias,
    const float *A, const void *B, const void *C, const float *D, const void *z, void *y,
    int64_t batch, int64_t dim, int64_t N, mamba_dtype_t dtype);

/* Enqueues one decoding token of `plan` on `stream` (one kernel launch). */
MAMBA_SCAN_API mamba_status_t mamba_scan_step_plan_run(mamba_step_plan_t plan,
                                                       mamba_stream_t stream);

MAMBA_SCAN_API void mamba_scan_step_plan_destroy(mamba_step_plan_t plan);

/*
 * The workspace pool of the current device.  The library takes its temporary
 * device memory from a pool of its own per device (see the conventions
 * above), which keeps up to a reserve -- 4 GiB unless set here -- mapped
 * between calls so that repeated calls do not map and unmap it.  That memory
 * is not visible to other allocators in the process (torch's caching
 * allocator, for one):
 *  - mamba_scan_pool_set_reserve(bytes): the pool keeps at most `bytes`
 *    reserved at each synchronization from now on (0: it gives all unused
 *    memory back every time, at the cost of re-mapping it per call).
 *  - mamba_scan_pool_trim(keep_bytes): gives unused memory back now, down to
 *    `keep_bytes`; memory of calls still running on a stream is released by a
 *    later trim, after that work completes.
 *  - mamba_scan_pool_reserved(&bytes): the memory the pool holds now.
 * Each returns MAMBA_ERR_CUDA if a CUDA call fails.
 */
MAMBA_SCAN_API mamba_status_t mamba_scan_pool_set_reserve(uint64_t bytes);
MAMBA_SCAN_API mamba_status_t mamba_scan_pool_trim(uint64_t keep_bytes);
MAMBA_SCAN_API mamba_status_t mamba_scan_pool_reserved(uint64_t *bytes);

/*
 * Test hook (not for production use): after `after` more successful
 * workspace allocations by the calling thread, the next one fails as if the
 * device were out of memory, so that tests can check that every call then
 * returns MAMBA_ERR_OUT_OF_MEMORY without launching a kernel or writing an
 * output.  A negative value disarms the hook.
 */
MAMBA_SCAN_API void mamba_scan_test_fail_alloc(int32_t after);

/*
 * Forward that allocates nothing.  (An addition of this library for callers
 * that cannot allocate; the paper has no counterpart.)
 *
 * Same arguments, layouts and results as mamba_scan_fwd.  Meant for callers
 * that cannot let a library allocate device memory -- programs that give all
 * device memory to their own allocator up front, latency-critical loops that
 * must not enter the CUDA allocator, code that runs where allocation calls
 * are not allowed.  Instead of a workspace per call, the chunked kernels keep
 * their scratch (ticket counters, hand-off flags, carried chunk-end states,
 * or the chunk aggregates of the three-phase carry) in a fixed 8 MiB array in
 * the library's device memory; every GPU that loads the library holds that
 * array until the process exits.  The call makes no cudaMalloc,
 * cudaMallocAsync or cudaFree call.
 *
 *  - Plan: the regular call's (see mamba_scan_options_t.carry) when its
 *    scratch fits the array; for the three-phase carry of few channel groups
 *    and long sequences, the variant with an aggregate pass (whose scratch
 *    does not grow with L) and then fewer, longer chunks until it fits;
 *    failing that, the sequential hand-off.
 *  - Limit: the sequential hand-off's scratch must fit: at most 1023 channel
 *    groups (batch * ceil(dim / 128)) when N > 8, 2046 when 4 < N <= 8, 4088
 *    when N <= 4.  Larger problems return MAMBA_ERR_UNSUPPORTED without
 *    enqueuing anything.  Shapes that the staged kernels do not take (see
 *    mamba_scan_fwd) run the one-thread-per-channel kernel, which needs no
 *    scratch.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) for that device; make that first call before any
 *    stream capture.
 *  - All calls on a device share the one array, and it keeps what the last
 *    call left (each call clears the parts that must start at zero).  Calls
 *    whose work overlaps on the GPU -- on different streams, or from
 *    different threads -- race on it: order them.
 */
MAMBA_SCAN_API mamba_status_t mamba_scan_fwd_noalloc(const void *u, const void *delta,
                                                     const float *delta_bias, const float *A,
                                                     const void *B, const void *C, const float *D,
                                                     const void *z, void *y, float *last_state,
                                                     int64_t batch, int64_t dim, int64_t L, int64_t N,
                                                     mamba_dtype_t dtype, mamba_stream_t stream);

/* Synchronizes `stream`, then returns MAMBA_ERR_CUDA for a pending CUDA error,
 * else MAMBA_ERR_DEVICE_TIMEOUT if a kernel of this library recorded an
 * expired wait on the current device since the last call, else (in the
 * bounds-checking build, libmambascan_debug.so) MAMBA_ERR_OUT_OF_BOUNDS if a
 * kernel computed an index outside one of its buffers (the records are
 * cleared), else MAMBA_OK. */
MAMBA_SCAN_API mamba_status_t mamba_scan_stream_status(mamba_stream_t stream);

/* Static, human-readable name of a status code (never NULL). */
MAMBA_SCAN_API const char *mamba_scan_status_string(mamba_status_t status);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all threads), for accounting in benchmarks. */
MAMBA_SCAN_API uint64_t mamba_scan_launch_count(void);

/* Version of this ABI (incremented on any incompatible change). */
MAMBA_SCAN_API int mamba_scan_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_SCAN_H */
