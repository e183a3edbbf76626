/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective state-space scan (S6).
 *
 * The operation (Gu & Dao, "Mamba: Linear-Time Sequence Modeling with
 * Selective State Spaces"; the selection mechanism makes dt, B and C functions
 * of the input; Mamba-1 discretises A by zero-order hold and the input term by
 * an Euler step, as the "Mamba3" post's section on the new discretisation
 * scheme recalls):
 *
 *   dt_t   = softplus(delta[b,d,t] + delta_bias[d])      (delta + bias if softplus == 0)
 *   h_t[n] = exp(dt_t * A[d,n]) * h_{t-1}[n] + dt_t * B[b,n,t] * x[b,d,t]
 *   y_t    = sum_n C[b,n,t] * h_t[n] + D[d] * x[b,d,t]
 *   out    = y_t * silu(z[b,d,t])                         (y_t when z == NULL)
 *
 * with h_{-1} = h0 (zero when NULL) and h_last = h_{L-1}.  Splitting a
 * sequence into consecutive calls, each starting from the previous call's
 * h_last, continues the same scan (Appendix D "Hardware-aware Algorithm For
 * Selective SSMs", paragraph "Speed": chunks continue from the carried state).
 *
 * Memory layout (all buffers contiguous, row-major, channel-major):
 *   x, delta, z, out : [batch][dim][seqlen]        activation dtype
 *   B, C             : [batch][dstate][seqlen]     activation dtype
 *   A                : [dim][dstate]               float32
 *   D, delta_bias    : [dim]                       float32
 *   h0, h_last       : [batch][dim][dstate]        float32
 * The activation dtype is the same for x, delta, z, B, C and out.  All
 * arithmetic is float32; the state is float32.
 *
 * Ownership and execution: every pointer is a device pointer owned by the
 * caller, and the library allocates no device memory.  ssm_scan_fwd needs a
 * workspace for its work queue, segment flags and carried states; the caller
 * sizes it with ssm_scan_fwd_workspace_size and passes it in.  Its size is
 * 16 KB + 2 KB per group of 32 channels (groups = batch * ceil(dim / 32)); when
 * the groups number fewer than half the GPU's SM sub-partitions (4 per SM),
 * the call cuts each sequence into segments and scans them in parallel in two
 * passes, and the workspace also holds 6 KB per (group, segment), with about
 * 16 * SMs segments in all (under 15 MB on a 148-SM GPU).  Calls that share a
 * workspace must not overlap on the GPU (the same stream serialises them).
 * ssm_scan_step needs no workspace.  Work is enqueued on `stream` and runs
 * asynchronously; the call returns after validating the arguments and
 * launching.  Errors that the device meets later surface through the CUDA
 * stream, and a bounded device wait that gave up is reported by
 * ssm_scan_fwd_status.  Calls are thread-safe.
 *
 * Error behaviour: every check is made on the host before anything is
 * launched; a call that returns non-zero has launched nothing and touched no
 * buffer (except SSM_ERR_CUDA, returned when a launch itself failed).
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *ssm_stream_t;

typedef enum {
    SSM_F32 = 0,  /* float32 activations */
    SSM_BF16 = 1  /* bfloat16 activations (stored as 16-bit patterns) */
} ssm_dtype_t;

typedef struct {
    int64_t batch;     /* number of sequences, >= 1 */
    int64_t seqlen;    /* L, >= 1 (ignored by ssm_scan_step) */
    int64_t dim;       /* channels D, >= 1 */
    int64_t dstate;    /* states per channel N; 16 is supported */
    int32_t act_dtype; /* ssm_dtype_t */
} ssm_dims_t;

/* Sizes of a Mamba-2 SSD call (ssm_ssd_fwd). */
typedef struct {
    int64_t batch;     /* sequences, >= 1 */
    int64_t seqlen;    /* L, >= 1 */
    int64_t heads;     /* H, >= 1, a multiple of groups */
    int64_t headdim;   /* P per head; 64 is supported */
    int64_t groups;    /* G groups of heads sharing B and C */
    int64_t dstate;    /* N; 128 is supported */
    int32_t act_dtype; /* ssm_dtype_t; SSM_BF16 is supported */
} ssm_ssd_dims_t;

enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1, /* NULL required pointer, a dimension < 1, overlapping buffers, or a too small workspace */
    SSM_ERR_UNSUPPORTED = 2, /* dstate or dtype not supported, or batch, seqlen or dim beyond 2^31 - 65 */
    SSM_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
    SSM_ERR_CUDA = 4,        /* a CUDA launch or query failed */
    SSM_ERR_TIMEOUT = 5      /* a bounded device wait gave up (from ssm_scan_fwd_status) */
};

/*
 * Workspace bytes that ssm_scan_fwd needs for the shape `dims` on a GPU with
 * `sm_count` SMs (sm_count <= 0: the current device, which needs a CUDA
 * context).  The size depends only on batch, seqlen, dim and the SM count.
 * Returns SSM_OK and writes *bytes, or an SSM_ERR_* code.
 */
int ssm_scan_fwd_workspace_size(const ssm_dims_t *dims, int sm_count, size_t *bytes);

/*
 * Forward scan over the whole sequence (the fused, chunked scan of Appendix D
 * "Speed"; recurrent computation as in the pages' recurrent mode).
 *
 *   x, delta       required, [batch][dim][seqlen]
 *   delta_bias     optional [dim] (NULL = 0)
 *   softplus       non-zero: dt = softplus(delta + bias); zero: dt = delta + bias
 *   A              required [dim][dstate]
 *   B, C           required [batch][dstate][seqlen]
 *   D              optional [dim] (NULL = no skip term)
 *   z              optional [batch][dim][seqlen] (NULL = no gate)
 *   h0             optional [batch][dim][dstate] (NULL = zero initial state)
 *   out            required [batch][dim][seqlen]; must not overlap any input
 *   h_last         optional [batch][dim][dstate] (NULL = not written); may be h0
 *   workspace      required device buffer of workspace_bytes, at least
 *                  ssm_scan_fwd_workspace_size for this shape and device; its
 *                  contents on entry do not matter; it must not overlap any
 *                  input or output
 *   dims           sizes and activation dtype
 *   stream         CUDA stream
 * Alignment: every pointer 16-byte aligned, except delta_bias and D (4 bytes).
 * Returns SSM_OK or an SSM_ERR_* code.
 */
int ssm_scan_fwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                 const float *A, const void *B, const void *C, const float *D,
                 const void *z, const float *h0, void *out, float *h_last,
                 void *workspace, size_t workspace_bytes,
                 const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * Whether the last forward call on `workspace` ran to completion: waits for
 * `stream` to finish, then reads the call's error word from the workspace.
 * Returns SSM_OK, SSM_ERR_TIMEOUT when one of the call's bounded device waits
 * gave up (its out and h_last are then void; every wait is bounded, so the
 * kernels always end), or SSM_ERR_CUDA when the stream reports a CUDA error.
 * workspace == NULL asks about the last ssm_scan_fwd_noalloc call on the
 * current device.  This call blocks the host; the forward calls never do.
 */
int ssm_scan_fwd_status(const void *workspace, ssm_stream_t stream);

/*
 * One recurrent (decode) step for every sequence: the pages' recurrent mode,
 * where inputs arrive one timestep at a time and the cache holds the SSM state
 * after the scan.  The float32 state is read and updated in place.
 *
 *   state          required [batch][dim][dstate] float32, read and written
 *   x, delta       required [batch][dim]  (one token per sequence)
 *   delta_bias     optional [dim]
 *   softplus       as for ssm_scan_fwd
 *   A              required [dim][dstate]
 *   B, C           required [batch][dstate]
 *   D              optional [dim]
 *   z              optional [batch][dim]
 *   out            required [batch][dim]; must not overlap any input or state
 *   dims           batch, dim, dstate, act_dtype (seqlen is ignored)
 * Alignment: state, A, B and C 16-byte aligned (they are read as vectors);
 * x, delta, z and out aligned to their element size; D and delta_bias 4 bytes.
 * Returns SSM_OK or an SSM_ERR_* code.
 */
int ssm_scan_step(float *state, const void *x, const void *delta, const float *delta_bias,
                  int softplus, const float *A, const void *B, const void *C,
                  const float *D, const void *z, void *out,
                  const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * The block's short causal convolution and activation fused in front of the
 * forward scan (Appendix D "Memory": input projection, convolution,
 * activation, scan, output projection; the convolution's output never goes
 * to device memory).  The scan runs on
 *
 *   xc[b,d,t] = silu( sum_{k<K} conv_w[d,k] * xin(b,d,t-K+1+k) + conv_bias[d] )
 *
 * in place of x, where xin(b,d,s) = x[b,d,s] for s >= 0 and the stored input
 * conv_state[b,d,K-1+s] for -(K-1) <= s < 0 (zero when conv_state is NULL).
 * The D skip uses xc, rounded to the activation dtype.
 *
 *   x              required [batch][dim][seqlen], the raw input
 *   conv_w         required [dim][conv_width] float32 (conv_w[d][conv_width-1]
 *                  multiplies the current input), 4-byte aligned
 *   conv_bias      optional [dim] float32 (NULL = 0), 4-byte aligned
 *   conv_width     K, 1..4
 *   conv_state     optional [batch][dim][K-1] activation dtype: the K-1 raw
 *                  inputs before t = 0, oldest first (NULL = zeros)
 *   conv_state_out optional [batch][dim][K-1] activation dtype: receives the
 *                  last K-1 raw inputs (the window for the next call or for
 *                  ssm_conv_scan_step); may be conv_state itself
 * The remaining arguments, the workspace, errors and ssm_scan_fwd_status are
 * those of ssm_scan_fwd.
 */
int ssm_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_bias, int conv_width,
                      const void *conv_state, void *conv_state_out,
                      const void *delta, const float *delta_bias, int softplus,
                      const float *A, const void *B, const void *C, const float *D,
                      const void *z, const float *h0, void *out, float *h_last,
                      void *workspace, size_t workspace_bytes,
                      const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * One decode step of the same block: the token x passes the convolution
 * window (the K-1 stored raw inputs followed by x), silu, then the recurrent
 * step of ssm_scan_step.  conv_state ([batch][dim][K-1], activation dtype,
 * element aligned; required when K > 1) is read and shifted in place: its
 * oldest input is dropped and x appended.  Other arguments as for
 * ssm_scan_step and ssm_conv_scan_fwd.
 */
int ssm_conv_scan_step(void *conv_state, float *state, const void *x, const float *conv_w,
                       const float *conv_bias, int conv_width, const void *delta,
                       const float *delta_bias, int softplus, const float *A, const void *B,
                       const void *C, const float *D, const void *z, void *out,
                       const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * Forward scan with the exponential-trapezoidal discretisation ("Mamba3"
 * posts, section on the new discretisation scheme: the integral over each
 * step is approximated with both ends of the interval, mixed by a
 * data-dependent lambda, a second-order rule):
 *
 *   h_t = alpha_t h_{t-1} + (1 - lam_t) dt_t alpha_t B_{t-1} x_{t-1} + lam_t dt_t B_t x_t
 *   alpha_t = exp(dt_t A),  y_t and out as for ssm_scan_fwd
 *
 * lam = 1 gives ssm_scan_fwd's Euler input step; lam = 1/2 the trapezoidal rule.
 *
 *   lam            required [batch][dim][seqlen], activation dtype, 16-byte aligned
 *   x_prev, B_prev optional [batch][dim] and [batch][dstate], activation dtype:
 *                  the input before t = 0 (the previous call's last x and B);
 *                  no previous input unless both are given
 * The remaining arguments, the workspace, errors and ssm_scan_fwd_status are
 * those of ssm_scan_fwd.  A sequence split into calls continues exactly when
 * each call gets the previous call's h_last and its last x and B.
 */
int ssm_trap_scan_fwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                      const void *lam, const float *A, const void *B, const void *C, const float *D,
                      const void *z, const float *h0, const void *x_prev, const void *B_prev,
                      void *out, float *h_last, void *workspace, size_t workspace_bytes,
                      const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * One recurrent step with the exponential-trapezoidal rule: ssm_scan_step's
 * arguments plus lam [batch][dim] (element aligned) and the previous token's
 * x_prev [batch][dim] (element aligned) and B_prev [batch][dstate] (16-byte
 * aligned); no previous input unless both are given.
 */
int ssm_trap_scan_step(float *state, const void *x, const void *delta, const float *delta_bias,
                       int softplus, const void *lam, const float *A, const void *B, const void *C,
                       const float *D, const void *z, const void *x_prev, const void *B_prev,
                       void *out, const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * Workspace bytes that ssm_scan_bwd needs for the shape `dims`: the scratch of
 * the forward pass that stores the checkpoints (as ssm_scan_fwd_workspace_size
 * gives it for 256 SMs; ssm_scan_fwd_status on the backward's workspace reads
 * its error word), then the states at the start of every 16-step segment (64 B
 * per channel and segment, i.e. 4 B per channel and step).  Needs no device.
 * Returns SSM_OK and writes *bytes, or an SSM_ERR_* code.
 */
int ssm_scan_bwd_workspace_size(const ssm_dims_t *dims, size_t *bytes);

/*
 * Backward pass of ssm_scan_fwd: the derivatives of a loss L with respect to
 * every input, given dout = dL/dout and dh_last = dL/dh_last.  As Appendix D
 * "Memory" describes, the intermediate states are not stored by the forward
 * pass: the call first runs the forward scan without output, storing the state
 * at the start of every 16-step segment, and recomputes each segment's states
 * from it while it runs the adjoint recurrence
 *   g_t = C_t dy_t + Abar_{t+1} g_{t+1},  dy_t = dout_t silu(z_t)
 * backwards through the chunk.
 *
 *   x .. h0        the forward call's inputs (as for ssm_scan_fwd)
 *   dout           required [batch][dim][seqlen], activation dtype
 *   dh_last        optional [batch][dim][dstate] float32 (NULL = 0)
 *   dx, ddelta     required [batch][dim][seqlen], activation dtype
 *   dz             [batch][dim][seqlen], activation dtype; required when z is given
 *   dB, dC         required [batch][dstate][seqlen] float32 (sums over channels)
 *   dA             required [dim][dstate] float32 (sum over batch and time)
 *   dD, dbias      optional [dim] float32 (NULL: not computed)
 *   dh0            optional [batch][dim][dstate] float32 (NULL: not written)
 *   workspace      at least ssm_scan_bwd_workspace_size bytes, 16-byte aligned
 * Alignment: 16 bytes for every pointer except delta_bias, D, dD, dbias (4).
 * No output may overlap an input or another output.  dB and dC (sums over
 * channels) and dA, dD, dbias (sums over the batch) are added with float
 * atomics, so their last bits may differ between calls.  Returns SSM_OK or an SSM_ERR_* code.
 */
int ssm_scan_bwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                 const float *A, const void *B, const void *C, const float *D, const void *z,
                 const float *h0, const void *dout, const float *dh_last,
                 void *dx, void *ddelta, void *dz, float *dB, float *dC, float *dA, float *dD,
                 float *dbias, float *dh0, void *workspace, size_t workspace_bytes,
                 const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * Mamba-2 state space duality (SSD) forward: a scalar-times-identity state
 * transition per head (the "Mamba3" posts: Mamba-2 reduced the transition to
 * a scalar times the identity; the Mamba-2 abstract: SSMs and attention meet
 * in structured semiseparable matrices).  Per batch b and head h:
 *
 *   dt_t = softplus(dt[b,t,h] + dt_bias[h])   (dt + dt_bias when softplus == 0)
 *   H_t  = exp(dt_t A[h]) H_{t-1} + (dt_t x_t) B_t^T      H: headdim x dstate
 *   y_t  = H_t C_t + D[h] x_t
 *
 * computed chunk by chunk (128 steps) as dense products on the tensor cores.
 *
 *   x, y           [batch][seqlen][heads][headdim] bf16, 16-byte aligned
 *   dt             [batch][seqlen][heads] bf16
 *   B, C           [batch][seqlen][groups][dstate] bf16, 16-byte aligned
 *                  (heads h*G/H .. share group h / (heads / groups))
 *   A, dt_bias, D  [heads] float32 (dt_bias and D optional)
 *   h0, h_last     optional [batch][heads][headdim][dstate] float32
 *   workspace      at least 256 bytes (the bounded-wait error word that
 *                  ssm_scan_fwd_status reads), 16-byte aligned, owned by the
 *                  caller and not used by a concurrent call.  With
 *                  ssm_ssd_fwd_workspace_size bytes or more, a call with more
 *                  sequences (batch * heads) than SMs runs one CTA per SM over
 *                  equal numbers of chunks: a sequence may be split between two
 *                  CTAs, whose state passes through the workspace.  With less,
 *                  every sequence gets its own CTA.  Results are the same
 *                  either way, up to rounding order.
 * Returns SSM_OK or an SSM_ERR_* code (SSM_ERR_UNSUPPORTED unless headdim 64,
 * dstate 128, bf16).
 */
/*
 * Workspace bytes for ssm_ssd_fwd to balance the sequences over sm_count SMs
 * (sm_count <= 0: the current device's): 256 when batch * heads is at most
 * the SM count (nothing is split), else 2048 + 32768 bytes per SM, for at most
 * 448 SMs (one hand-off flag and one headdim x dstate float32 state each).  Needs only dims.batch
 * and dims.heads.  Returns SSM_OK, SSM_ERR_INVALID_ARG (NULL pointer, batch or
 * heads < 1) or SSM_ERR_CUDA (no current device when sm_count <= 0).
 */
int ssm_ssd_fwd_workspace_size(const ssm_ssd_dims_t *dims, int sm_count, size_t *bytes);

int ssm_ssd_fwd(const void *x, const void *dt, const float *dt_bias, int softplus, const float *A,
                const void *B, const void *C, const float *D, const float *h0, void *y, float *h_last,
                void *workspace, size_t workspace_bytes, const ssm_ssd_dims_t *dims,
                ssm_stream_t stream);

/*
 * ssm_scan_fwd without a workspace.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate any device memory while
 * they run the scan, not even a workspace (code running inside an allocator or
 * memory-pool callback, runtimes that reserve all device memory up front and
 * forbid later allocations).  Arguments, layout, results and error codes are
 * those of ssm_scan_fwd without the two workspace arguments.  Its work queue,
 * segment flags and carried states use a fixed 2 MiB device array inside the
 * library (held by every GPU that loads it), so shapes with
 * batch * ceil(dim / 32) above about 1000 are rejected with
 * SSM_ERR_UNSUPPORTED.  It always scans the segments of a group in order (no
 * two-pass parallel schedule), whatever the number of groups, so shapes with
 * few channel groups run slower here than through ssm_scan_fwd.  The first
 * call on a device looks up that array's address; make that first call before
 * any stream capture.  Every call shares the one array of its device: calls
 * whose work overlaps on the GPU (for example calls on two streams of the same
 * device) race on it and must be serialised by the caller.
 * ssm_scan_fwd_status(NULL, stream) reports on the last call.  It allocates
 * nothing: no cudaMalloc/cudaFree and no memory-pool allocation.
 */
int ssm_scan_fwd_noalloc(const void *x, const void *delta, const float *delta_bias, int softplus,
                         const float *A, const void *B, const void *C, const float *D,
                         const void *z, const float *h0, void *out, float *h_last,
                         const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * Test support, not part of the operation: ssm_scan_fwd with the chained
 * schedule, where each segment's wait for its predecessor's flag awaits a
 * count that no flag ever reaches and gives up after `spin_limit` polls (0:
 * at once).  The kernels still end normally; ssm_scan_fwd_status then reports
 * SSM_ERR_TIMEOUT.  Arguments as for ssm_scan_fwd.
 */
int ssm_debug_fwd_flag_timeout(const void *x, const void *delta, const float *delta_bias, int softplus,
                               const float *A, const void *B, const void *C, const float *D,
                               const void *z, const float *h0, void *out, float *h_last,
                               void *workspace, size_t workspace_bytes, uint32_t spin_limit,
                               const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * Test support, not part of the operation: ssm_ssd_fwd where every CTA that
 * continues a sequence split between two CTAs waits for a hand-off flag value
 * that no flag ever reaches and gives up after `spin_limit` polls (0: at
 * once).  Only a call that splits sequences (more sequences than SMs, and a
 * workspace of ssm_ssd_fwd_workspace_size bytes) waits at all.  The kernel
 * still ends normally; ssm_scan_fwd_status then reports SSM_ERR_TIMEOUT.
 * Arguments as for ssm_ssd_fwd.
 */
int ssm_debug_ssd_flag_timeout(const void *x, const void *dt, const float *dt_bias, int softplus,
                               const float *A, const void *B, const void *C, const float *D,
                               const float *h0, void *y, float *h_last, void *workspace,
                               size_t workspace_bytes, uint32_t spin_limit, const ssm_ssd_dims_t *dims,
                               ssm_stream_t stream);

/* Static, human-readable text for an SSM_* code (never NULL). */
const char *ssm_strerror(int code);

/* Library version as major*10000 + minor*100 + patch. */
int ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
