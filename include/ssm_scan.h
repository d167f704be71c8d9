/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective state-space scan.
 *
 * The operation is the selective scan of Mamba as stated on the page
 * "Mamba 논문 리뷰: Selective State Space Models로 Transformer를 넘어서"
 * (youngju.dev): the discretised recurrence of §2.2 (Zero-Order Hold),
 * with the input-dependent step of §3.1 (Delta = softplus(.)), the
 * simplified deltaA = exp(Delta*A), deltaB = Delta*B of the §3.3
 * selective_scan, and the D skip and y * SiLU(z) gate of the §3.4 Mamba
 * block. Per batch b, channel d and state n (state fp32):
 *
 *   Delta   = softplus(delta[b,t,d] + delta_bias[d])   (or no softplus)
 *   h[n]    = exp(Delta * A[d,n]) * h[n] + Delta * B[b,t,n] * x[b,t,d]
 *   y[b,t,d]= (sum_n C[b,t,n] * h[n] + D[d] * x[b,t,d]) * SiLU(z[b,t,d])
 *
 * starting from h0[b,d,:] (or zero) and ending in h_last[b,d,:].
 * softplus(v) is log(1 + e^v) for v <= 20 and v above 20.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, dense and
 *     row-major (C order) in the layouts given below. The library never
 *     allocates, frees or synchronises. Apart from small caches of its own
 *     (kernel attributes set once, driver entry points), its one piece of
 *     mutable global state is the fixed scratch array of the no-alloc entry
 *     (ssm_scan_fwd_noalloc below), shared by every call of that entry on a
 *     device; all other entry points keep their state in caller memory.
 *   - io_dtype selects the storage type of x, delta, z, B, C and y:
 *     SSM_DTYPE_F32 (IEEE binary32) or SSM_DTYPE_BF16 (bfloat16). A, D,
 *     delta_bias, h0, h_last and the decode state are always fp32.
 *   - Optional pointers may be NULL: D (no skip), z (no gate), delta_bias
 *     (zero bias), h0 (zero initial state), h_last (not written).
 *   - stream is a cudaStream_t (NULL = legacy default stream). Work is
 *     enqueued asynchronously; errors of the kernels themselves surface at
 *     the caller's next synchronisation.
 *   - Return value: SSM_OK, or a negative SSM_ERR_* code. Argument errors
 *     are detected on the host before anything is enqueued.
 *   - Pointers must be aligned to their element size (h0 / h_last and A
 *     of the scan and its backward to 8 bytes; for ssm_state_update the state and A to 16 bytes when
 *     dstate % 4 == 0, else 8, and B, C to four elements when dstate % 4 == 0,
 *     else two). The fast
 *     path also wants 16-byte aligned bases and rows (dim and dstate
 *     multiples of 16 bytes) and otherwise takes a slower path with plain
 *     loads (SSM_SCAN_DISABLE_TMA=1 in the environment forces that path).
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SSM_DTYPE_F32 = 0,
  SSM_DTYPE_BF16 = 1,
};

enum {
  SSM_OK = 0,
  SSM_ERR_INVALID_ARG = -1, /* null required pointer, bad size, misaligned, aliasing */
  SSM_ERR_UNSUPPORTED = -2, /* dstate, io_dtype or size this library does not support
                               (sizes: batch <= 65535, seqlen <= 2^30, dim <= 2^24, and
                               no tensor above 2^40 elements)                          */
  SSM_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required           */
  SSM_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed          */
  SSM_ERR_TIMEOUT = -5,     /* a bounded wait inside a kernel gave up (ssm_scan_status) */
};

/* dstate (N) values this library supports: 2, 4, 8, 16, 32, 64. */
#define SSM_MAX_DSTATE 64

/*
 * How ssm_scan_fwd splits a problem (see ssm_scan_plan). The sequence is cut
 * into `segments` of `segment_steps` steps; with more than one segment a
 * carry pass computes each segment's end state, the carries are composed into
 * every segment's start state (by the main pass itself up to 9 segments, by a
 * small kernel between the passes above that), and the main pass runs each
 * segment from its start (the recurrence of §2.2 is an
 * associative composition of affine maps h -> a*h + b, which the pages'
 * parallel associative scan relies on).
 */
typedef struct {
  int32_t segments;
  int32_t segment_steps;
  int32_t channel_tiles;    /* CTAs along dim                                */
  int32_t channels_per_cta;
  int32_t ctas_carry;       /* CTAs of the carry pass (0 with one segment)   */
  int32_t ctas_main;        /* CTAs of the main pass                         */
  int32_t kernels;          /* kernel launches per ssm_scan_fwd call         */
  int64_t workspace_bytes;  /* = ssm_scan_workspace_bytes(...)               */
} ssm_scan_plan_t;

/*
 * ssm_scan_workspace_bytes -- bytes of device workspace ssm_scan_fwd needs
 * for these sizes on the current device (0 when it needs none). The
 * workspace holds per-segment carries of the sequence split (§2.2
 * recurrence composed across sequence segments). Returns 0 for invalid
 * sizes too; ssm_scan_fwd then reports the size error.
 */
size_t ssm_scan_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                int io_dtype);

/*
 * ssm_scan_plan -- fill *out with the split ssm_scan_fwd will use for these
 * sizes on the current device. Host only; enqueues nothing. The split
 * targets about SSM_SCAN_CTAS_PER_SM (environment, default 4) resident CTAs
 * per SM; SSM_SCAN_SEGMENTS (environment, > 0) forces the segment count.
 * Returns SSM_OK or SSM_ERR_INVALID_ARG / SSM_ERR_UNSUPPORTED.
 */
int ssm_scan_plan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                  ssm_scan_plan_t* out);

/*
 * ssm_scan_fwd -- the selective scan (prefill / training-shaped forward).
 *
 *   x, delta, z, y : (batch, seqlen, dim)     io_dtype
 *   B, C           : (batch, seqlen, dstate)  io_dtype, shared by all channels
 *   A              : (dim, dstate)            fp32 (Mamba uses A = -exp(A_log))
 *   D, delta_bias  : (dim)                    fp32, nullable
 *   h0, h_last     : (batch, dim, dstate)     fp32, nullable
 *   softplus       : nonzero applies softplus to delta + delta_bias
 *   workspace      : device buffer of at least ssm_scan_workspace_bytes(...)
 *                    bytes (may be NULL when that is 0); contents on entry
 *                    are ignored; it must not be used by concurrent calls.
 *
 * y must not overlap any input. y may be NULL when h_last is given (only the
 * final state is wanted). h_last may alias h0 (in-place resume).
 * seqlen == 0 writes only h_last (= h0 or zero). batch or dim == 0 is a
 * no-op. Returns SSM_OK or SSM_ERR_*.
 */
int ssm_scan_fwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                 const void* x, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int softplus, const float* h0, void* y, float* h_last, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * ssm_scan_fwd_zoh -- ssm_scan_fwd with the exact zero-order-hold input term
 * of §2.2 instead of the simplified Delta * B of the §3.3 listing:
 *
 *   h[n] = exp(Delta A[d,n]) h[n] + B-bar[n] x[b,t,d],
 *   B-bar[n] = (Delta A)^-1 (exp(Delta A) - 1) Delta B = (exp(Delta A[d,n]) - 1) / A[d,n] * B[b,t,n]
 *
 * (Delta B where A[d,n] = 0). Same arguments, layouts, workspace and errors as
 * ssm_scan_fwd (the workspace size is the same).
 */
int ssm_scan_fwd_zoh(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                     const void* x, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* delta_bias,
                     int softplus, const float* h0, void* y, float* h_last, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * ssm_scan_fwd_noalloc -- ssm_scan_fwd for callers that cannot allocate
 * device memory. The Mamba pages have no counterpart to this call; it exists
 * for callers that only get their input and output buffers and may not call
 * cudaMalloc themselves (code running inside a memory pool or arena it does
 * not own, real-time paths that must not allocate after start-up, plugins of
 * a host framework). Same arguments, layouts and results as ssm_scan_fwd,
 * without the workspace.
 *
 * Scratch: a fixed 16 MiB array reserved in device memory by the library on
 * every GPU that loads it, kept until the process exits. Problems whose
 * ssm_scan_workspace_bytes(...) exceeds 16 MiB are rejected with
 * SSM_ERR_WORKSPACE (ssm_last_error_detail says how much they need); use
 * ssm_scan_fwd for those.
 *   - The first call on each device looks up the scratch's device address
 *     (with that device current); make that first call before any stream
 *     capture on the device.
 *   - Every call on a device shares the one array and finds the previous
 *     call's leftovers in it; nothing in it needs to start at zero (each call
 *     writes every scratch word it reads). Calls that can run at the same
 *     time on the GPU (different streams or host threads, without ordering
 *     between them) race on the scratch and must be serialised by the caller.
 *   - The scratch's address is cached per device together with the context
 *     it was looked up in; after cudaDeviceReset the next call (made before
 *     any stream capture, as above) looks it up again.
 *   - A bounded wait inside the kernels that times out records it in the
 *     scratch; ssm_scan_status_noalloc (below) reads it, as ssm_scan_status
 *     does for ssm_scan_fwd.
 *   - Allocates and frees nothing. Returns SSM_OK or SSM_ERR_*.
 */
int ssm_scan_fwd_noalloc(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                         int io_dtype, const void* x, const void* delta, const float* A,
                         const void* B, const void* C, const float* D, const void* z,
                         const float* delta_bias, int softplus, const float* h0, void* y,
                         float* h_last, void* stream);

/*
 * ssm_scan_status_noalloc -- ssm_scan_status for the no-alloc entry (no
 * counterpart on the pages either): synchronise `stream`, then report from
 * the reserved scratch whether every CTA of the last ssm_scan_fwd_noalloc
 * call on this device with these sizes finished normally: SSM_OK, or
 * SSM_ERR_TIMEOUT if a bounded wait gave up (y and h_last are then
 * incomplete). The status words belong to the last no-alloc call on the
 * device, whatever its sizes; pass the sizes of that call. Returns
 * SSM_ERR_WORKSPACE for sizes the scratch cannot hold, like the entry itself.
 */
int ssm_scan_status_noalloc(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                            int io_dtype, void* stream);

/*
 * ssm_state_update -- one decode step: the recurrent, O(1)-per-token form of
 * the same recurrence (the §3.3 loop body for a single t), updating the
 * carried state in place.
 *
 *   state          : (batch, dim, dstate) fp32, read and written
 *   x, delta, z, y : (batch, dim)             io_dtype (z nullable)
 *   B, C           : (batch, dstate)          io_dtype
 *   A              : (dim, dstate) fp32;  D, delta_bias : (dim) fp32, nullable
 *
 * y must not overlap any input or the state. Returns SSM_OK or SSM_ERR_*.
 */
int ssm_state_update(int64_t batch, int64_t dim, int64_t dstate, int io_dtype, float* state,
                     const void* x, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* delta_bias,
                     int softplus, void* y, void* stream);

/*
 * ssm_scan_bwd_workspace_bytes -- bytes of device workspace ssm_scan_bwd
 * needs for these sizes (0 for unsupported sizes or dtypes). It holds state
 * checkpoints every 4 steps: about 4 * batch * seqlen * dim * dstate / 4
 * bytes, plus per-segment carries and partial sums.
 */
size_t ssm_scan_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                    int io_dtype);

/*
 * ssm_scan_bwd -- gradients of the selective scan (the backward pass that the
 * §3.3 Hardware-Aware algorithm trains with: intermediate states are not
 * stored by the forward but recomputed here from the inputs). For the loss
 *
 *   sum_{b,t,d} dy[b,t,d] * y[b,t,d]  +  sum_{b,d,n} dh_last[b,d,n] * h_last[b,d,n]
 *
 * with y, h_last as ssm_scan_fwd computes them from the same inputs, it
 * writes (overwrites) the gradient with respect to every input:
 *
 *   dx, ddelta, dz : (batch, seqlen, dim)   io_dtype; ddelta is the gradient
 *                    with respect to the raw delta (before bias and softplus);
 *                    dz must be NULL exactly when z is NULL
 *   dA             : (dim, dstate) fp32
 *   dB, dC         : (batch, seqlen, dstate) fp32 (sums over channels)
 *   dD, ddelta_bias: (dim) fp32, nullable (not written when NULL); dD is
 *                    the gradient at the given D, or at D = 0 when D is NULL
 *   dh0            : (batch, dim, dstate) fp32, nullable; the gradient with
 *                    respect to the initial state (h0, or the zero state)
 *
 * Inputs x, delta, A, B, C, D, z, delta_bias, softplus, h0 are those of the
 * forward call; dy is (batch, seqlen, dim) io_dtype and dh_last (batch, dim,
 * dstate) fp32 or NULL (zero). dstate must be 2, 4, 8 or 16. No output may
 * overlap an input or another output. workspace: device memory of at least
 * ssm_scan_bwd_workspace_bytes(), 16-byte aligned, used as scratch only.
 * Sums over channels, batch rows and segments are taken in a fixed order:
 * results do not depend on scheduling. Returns SSM_OK or SSM_ERR_*.
 */
int ssm_scan_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                 const void* x, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int softplus, const float* h0, const void* dy, const float* dh_last,
                 void* dx, void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
                 float* ddelta_bias, float* dh0, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * ssm_conv1d_silu_fwd -- the Mamba block's causal depthwise convolution and
 * SiLU (§3.4 Mamba Block: nn.Conv1d(d_inner, d_inner, d_conv,
 * padding=d_conv-1, groups=d_inner), output cut to the first L steps, then
 * SiLU), the step that produces the scan's x:
 *
 *   out[b,t,d] = SiLU(bias[d] + sum_{k<width} w[d,k] * x[b, t-(width-1)+k, d])
 *
 * with x = 0 before t = 0 (silu = 0: the convolution alone).
 *   x, out : (batch, seqlen, dim) io_dtype; out must not overlap x
 *   w      : (dim, width) fp32, width 2, 3 or 4 (the block uses 4)
 *   bias   : (dim) fp32, nullable (zero)
 * dim a multiple of 4 (bf16) or 2 (fp32) with 8-byte aligned x and out takes
 * 8-byte vector accesses; other shapes one element per thread.
 * Returns SSM_OK or SSM_ERR_*.
 */
int ssm_conv1d_silu_fwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t width, int io_dtype,
                        const void* x, const float* w, const float* bias, int silu, void* out,
                        void* stream);

/*
 * ssm_conv1d_silu_update -- one decode step of the same convolution (the
 * step form for single-token decode, beside ssm_state_update):
 *   conv_state : (batch, dim, width-1) io_dtype, the channel's last width-1
 *                inputs, oldest first (zero at the start of a sequence);
 *                read and updated in place (drops the oldest, appends x)
 *   x, out     : (batch, dim) io_dtype
 *   out[b,d]   = SiLU(bias[d] + sum_(k<width-1) w[d,k] state[k] + w[d,width-1] x[b,d])
 * width 2, 3 or 4. No buffer may overlap another. Returns SSM_OK or SSM_ERR_*.
 */
int ssm_conv1d_silu_update(int64_t batch, int64_t dim, int64_t width, int io_dtype,
                           void* conv_state, const void* x, const float* w, const float* bias,
                           int silu, void* out, void* stream);

/* ssm_conv1d_silu_bwd_workspace_bytes -- workspace of ssm_conv1d_silu_bwd:
 * per-(batch row, 128-step chunk) partial sums of dw and dbias. */
size_t ssm_conv1d_silu_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim,
                                           int64_t width, int io_dtype);

/*
 * ssm_conv1d_silu_bwd -- gradients of sum(dout * out) for
 * ssm_conv1d_silu_fwd with the same x, w, bias, silu:
 *   dx    : (batch, seqlen, dim) io_dtype (overwritten)
 *   dw    : (dim, width) fp32, nullable; dbias : (dim) fp32, nullable
 * dout is (batch, seqlen, dim) io_dtype. No output may overlap an input.
 * Sums over batch rows and steps run in a fixed order. Returns SSM_OK or
 * SSM_ERR_*.
 */
int ssm_conv1d_silu_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t width, int io_dtype,
                        const void* x, const float* w, const float* bias, int silu,
                        const void* dout, void* dx, float* dw, float* dbias, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ssm_state_update_zoh -- ssm_state_update with the exact zero-order-hold
 * input term (see ssm_scan_fwd_zoh). Same arguments and errors. */
int ssm_state_update_zoh(int64_t batch, int64_t dim, int64_t dstate, int io_dtype, float* state,
                         const void* x, const void* delta, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* delta_bias,
                         int softplus, void* y, void* stream);

/*
 * Splitting one sequence across ranks (devices). A chunk of steps acts on the
 * state as the affine map h -> P h + e with P_n = exp(A[d,n] * sum_t Delta_t)
 * and e the chunk's end state from a zero start (§2.2 recurrence; the maps
 * compose associatively, which is the parallel scan of the allinfo.ai.kr
 * page). With the sequence cut into chunks 0..R-1 in order, rank r:
 *   1. ssm_scan_fwd(h0 = NULL, y = NULL, h_last = e_r) on its chunk, and
 *      ssm_delta_sum(...) -> S_r;
 *   2. gathers (e, S) of every rank (e.g. an all-gather);
 *   3. ssm_compose_carries(r, ...) -> its true entering state;
 *   4. ssm_scan_fwd(h0 = that state) on its chunk -> its y, and on the last
 *      rank the sequence's h_last.
 * (ssm_scan_fwd accepts y = NULL when h_last is given: state only.)
 */

/* ssm_delta_sum -- dsum[b,d] = sum_t Delta[b,t,d], Delta = softplus(delta +
 * delta_bias) (or delta + delta_bias), fp32 (batch, dim). delta is
 * (batch, seqlen, dim) io_dtype; delta_bias (dim) fp32, nullable. */
int ssm_delta_sum(int64_t batch, int64_t seqlen, int64_t dim, int io_dtype, const void* delta,
                  const float* delta_bias, int softplus, float* dsum, void* stream);

/* ssm_compose_carries -- h_in = the state entering chunk `rank`: starting from
 * h0 (nullable: zero), apply h <- exp(A[d,n] dsum_all[r,b,d]) h + hend_all[r,b,d,n]
 * for r = 0 .. rank-1. A (dim, dstate); h0, h_in (batch, dim, dstate);
 * hend_all (ranks, batch, dim, dstate); dsum_all (ranks, batch, dim); fp32.
 * h_in must not overlap an input. */
int ssm_compose_carries(int64_t rank, int64_t batch, int64_t dim, int64_t dstate, const float* A,
                        const float* h0, const float* hend_all, const float* dsum_all,
                        float* h_in, void* stream);

/*
 * ssm_ssd_scan_fwd -- the multi-head SSD scan of Mamba-2 (same page, §4.1
 * State Space Duality: the SSM as a semi-separable matrix, and §4.2:
 * multi-head, state 64 to 256). Head h (width headdim) has one scalar A[h]
 * and one step per token; B and C are shared by every head. Per batch b,
 * head h, with the head's state S (headdim x dstate, fp32):
 *
 *   Delta        = softplus(dt[b,t,h] + dt_bias[h])   (or no softplus)
 *   S[p][n]      = exp(Delta * A[h]) * S[p][n] + Delta * B[b,t,n] * x[b,t,h,p]
 *   y[b,t,h,p]   = sum_n C[b,t,n] * S[p][n] + D[h] * x[b,t,h,p]
 *
 * starting from h0[b,h] (or zero) and ending in h_last[b,h]. Computed chunk
 * by chunk on the tensor cores (bf16 operands, fp32 accumulation and state):
 * with dstate 64 or 128, an even nheads, a 4-byte aligned dt and 16-byte
 * aligned h0 / h_last on the fifth-generation (tcgen05) path, the state held
 * in tensor memory; otherwise (or with SSM_SSD_LEGACY=1) on the warp-level
 * MMA path.
 *   x, y     : (batch, seqlen, nheads, headdim) bf16 (io_dtype must be
 *              SSM_DTYPE_BF16); y must not overlap an input
 *   dt       : (batch, seqlen, nheads) bf16
 *   B, C     : (batch, seqlen, dstate) bf16
 *   A        : (nheads) fp32;  D, dt_bias : (nheads) fp32, nullable
 *   h0       : (batch, nheads, headdim, dstate) fp32, nullable (zero)
 *   h_last   : (batch, nheads, headdim, dstate) fp32, nullable (not written)
 * headdim must be 64 and dstate 64, 128 or 256 (else SSM_ERR_UNSUPPORTED).
 * x, B, C and y 16-byte aligned, h0 / h_last 8-byte aligned.
 * Returns SSM_OK or SSM_ERR_*.
 */
int ssm_ssd_scan_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                     int64_t dstate, int io_dtype, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* dt_bias,
                     int softplus, const float* h0, void* y, float* h_last, void* stream);

/*
 * ssm_ssd_scan_status -- synchronise `stream`, then report whether a CTA of
 * an ssm_ssd_scan_fwd call on the current device gave up a bounded wait
 * (2 s, or SSM_SCAN_WAIT_LIMIT_NS nanoseconds) since the last call of this
 * function: SSM_OK, or SSM_ERR_TIMEOUT (that call's y and h_last are then
 * incomplete). The flag is per device and cleared by this call. For testing
 * this path, SSM_SSD_TEST_STALL=1 makes the first CTA wait for data that
 * never arrives.
 */
int ssm_ssd_scan_status(void* stream);

/*
 * ssm_ssd_state_update -- one decode step of the multi-head SSD (same page,
 * §4.1: the recurrent side of the duality, O(1) work per generated token),
 * on a carried fp32 state updated in place. Per batch b, head h, row p:
 *
 *   Delta    = softplus(dt[b,h] + dt_bias[h])   (or no softplus)
 *   S[n]     = exp(Delta * A[h]) * S[n] + Delta * B[b,n] * x[b,h,p]
 *   y[b,h,p] = sum_n C[b,n] * S[n] + D[h] * x[b,h,p]
 *
 *   state    : (batch, nheads, headdim, dstate) fp32, read and written
 *   x, y     : (batch, nheads, headdim) io_dtype
 *   dt       : (batch, nheads) io_dtype
 *   B, C     : (batch, dstate) io_dtype
 *   A        : (nheads) fp32;  D, dt_bias : (nheads) fp32, nullable
 * dstate 32, 64, 128 or 256 (else SSM_ERR_UNSUPPORTED); any headdim. state,
 * B and C 16-byte aligned. No output may overlap an input.
 * Returns SSM_OK or SSM_ERR_*.
 */
int ssm_ssd_state_update(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                         int io_dtype, float* state, const void* x, const void* dt,
                         const float* A, const void* B, const void* C, const float* D,
                         const float* dt_bias, int softplus, void* y, void* stream);

/*
 * ssm_scan_status -- synchronise `stream`, then report whether every CTA of
 * the last ssm_scan_fwd call that used this workspace (with these sizes)
 * finished normally: SSM_OK, or SSM_ERR_TIMEOUT if a bounded wait inside a
 * kernel gave up (its outputs are then incomplete). The wait bound is 2 s,
 * or SSM_SCAN_WAIT_LIMIT_NS nanoseconds from the environment. For testing
 * this path, SSM_SCAN_TEST_STALL=1 in the environment makes the first CTA of
 * the main pass (TMA path) wait for data that never arrives.
 */
int ssm_scan_status(const void* workspace, size_t workspace_bytes, int64_t batch,
                    int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype, void* stream);

/* ssm_status_string -- static, human-readable text for an SSM_* code. */
const char* ssm_status_string(int status);

/*
 * ssm_last_error_detail -- text describing the last SSM_ERR_CUDA /
 * SSM_ERR_TIMEOUT failure on the calling host thread (which CUDA call failed
 * and its error name); "" if none. The pointer stays valid until the next
 * failing call on this thread.
 */
const char* ssm_last_error_detail(void);

/* ssm_scan_version -- library version as MAJOR*10000 + MINOR*100 + PATCH. */
int ssm_scan_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
