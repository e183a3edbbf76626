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
 * caller.  ssm_scan_fwd takes a scratch area for its work queue (16 KB + 2 KB
 * per group of 32 channels) from a library-owned, stream-ordered memory pool per
 * device and returns it on the same stream; the pool keeps the memory between
 * calls.  When the channel groups (batch * ceil(dim / 32)) number fewer than
 * half the GPU's SM sub-partitions, the call cuts each sequence into segments
 * and scans them in parallel in two passes; the scratch then also holds 6 KB per
 * (group, segment), with about 4 * (SM sub-partitions) segments in all (under
 * 15 MB on a 148-SM GPU).  ssm_scan_step allocates nothing.  Work is enqueued on
 * `stream` and runs asynchronously; the call returns after validating the
 * arguments and launching.  Errors that the device meets later surface
 * through the CUDA stream.  Calls are thread-safe.
 *
 * Error behaviour: every check is made on the host before anything is
 * launched; a call that returns non-zero has launched nothing and touched no
 * buffer (except SSM_ERR_CUDA, returned when a launch itself failed).
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

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

enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1, /* NULL required pointer, a dimension < 1, or aliasing out with an input */
    SSM_ERR_UNSUPPORTED = 2, /* dstate or dtype not supported, or sizes beyond 32-bit indexing limits */
    SSM_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
    SSM_ERR_CUDA = 4,        /* a CUDA launch or query failed */
    SSM_ERR_TIMEOUT = 5      /* reserved: a bounded device wait gave up */
};

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
 *   dims           sizes and activation dtype
 *   stream         CUDA stream
 * Returns SSM_OK or an SSM_ERR_* code.
 */
int ssm_scan_fwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                 const float *A, const void *B, const void *C, const float *D,
                 const void *z, const float *h0, void *out, float *h_last,
                 const ssm_dims_t *dims, ssm_stream_t stream);

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
 * Returns SSM_OK or an SSM_ERR_* code.
 */
int ssm_scan_step(float *state, const void *x, const void *delta, const float *delta_bias,
                  int softplus, const float *A, const void *B, const void *C,
                  const float *D, const void *z, void *out,
                  const ssm_dims_t *dims, ssm_stream_t stream);

/*
 * ssm_scan_fwd without any device allocation.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory
 * while they run the scan (code running inside an allocator or memory-pool
 * callback, runtimes that reserve all device memory up front and forbid
 * later allocations).  Arguments, layout, results and error codes are those
 * of ssm_scan_fwd.  Its work queue, segment flags and carried states use a
 * fixed 2 MiB device array inside the library (held by every GPU that loads
 * it), so shapes with batch * ceil(dim / 32) above about 1000 are rejected
 * with SSM_ERR_UNSUPPORTED.  It always scans the segments of a group in order
 * (no two-pass parallel schedule), whatever the number of groups, so shapes
 * with few channel groups run slower here than through ssm_scan_fwd.  The
 * first call on a device looks up that array's address; make that first call
 * before any stream capture.  Every call
 * shares the one array of its device: calls whose work overlaps on the GPU
 * (for example calls on two streams of the same device) race on it and must be
 * serialised by the caller.  It allocates nothing: no cudaMalloc/cudaFree and
 * no memory-pool allocation.
 */
int ssm_scan_fwd_noalloc(const void *x, const void *delta, const float *delta_bias, int softplus,
                         const float *A, const void *B, const void *C, const float *D,
                         const void *z, const float *h0, void *out, float *h_last,
                         const ssm_dims_t *dims, ssm_stream_t stream);

/* Static, human-readable text for an SSM_* code (never NULL). */
const char *ssm_strerror(int code);

/* Library version as major*10000 + minor*100 + patch. */
int ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
