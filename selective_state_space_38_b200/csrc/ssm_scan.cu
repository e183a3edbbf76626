// ssm_scan.cu -- C ABI entry points: host-side validation and kernel launch.
//
// Every argument check happens here, before anything is enqueued; a call that
// fails a check launches nothing.  Kernels run asynchronously on the caller's
// stream.

#include <algorithm>
#include <climits>
#include <cstring>
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "ssm_scan.h"
#include "common.cuh"
#include "scan_fwd.cuh"
#include "scan_step.cuh"
#include "scan_bwd.cuh"
#include "ssd_fwd.cuh"

namespace {

using namespace ssm;

constexpr int kVersion = 10000;  // 1.0.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

struct Span {
    const void *p;
    size_t bytes;
};

bool overlap(const Span &a, const Span &b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

// sizes must be positive and every buffer must stay well inside int64 byte offsets
bool dims_ok(int64_t batch, int64_t seqlen, int64_t dim) {
    if (batch < 1 || seqlen < 1 || dim < 1) return false;
    const double elems = static_cast<double>(batch) * static_cast<double>(seqlen) * static_cast<double>(dim);
    return elems < 4.0e18 / 16.0;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// A rank-3 [d2][d1][d0] tensor (d0 contiguous) with a [1][box1][box0] box.
bool encode3d(CUtensorMap *m, CUtensorMapDataType dt, size_t es, const void *base, uint64_t d0, uint64_t d1,
              uint64_t d2, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A rank-4 [d3][d2][d1][d0] tensor (d0 contiguous) with a [1][box2][1][box0] box.
bool encode4d(CUtensorMap *m, CUtensorMapDataType dt, size_t es, const void *base, uint64_t d0, uint64_t d1,
              uint64_t d2, uint64_t d3, uint32_t box0, uint32_t box2, CUtensorMapSwizzle sw) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * es, d0 * d1 * es, d0 * d1 * d2 * es};
    const cuuint32_t box[4] = {box0, 1, box2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
bool make_maps(const FwdParams &p, TmaMaps *tm) {
    const CUtensorMapDataType dt = Act<T>::kBytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const size_t es = Act<T>::kBytes;
    const uint32_t tc = FwdSmem<T>::kTC;
    const uint64_t L = p.seqlen, D = p.dim, Bt = p.batch;
    bool ok = encode3d(&tm->x, dt, es, p.x, L, D, Bt, tc, 32, CU_TENSOR_MAP_SWIZZLE_64B) &&
              encode3d(&tm->delta, dt, es, p.delta, L, D, Bt, tc, 32, CU_TENSOR_MAP_SWIZZLE_64B) &&
              (!p.out || encode3d(&tm->out, dt, es, p.out, L, D, Bt, tc, 32, CU_TENSOR_MAP_SWIZZLE_64B)) &&
              encode3d(&tm->B, dt, es, p.B, L, kNState, Bt, tc, kNState, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              encode3d(&tm->C, dt, es, p.C, L, kNState, Bt, tc, kNState, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && p.z) ok = encode3d(&tm->z, dt, es, p.z, L, D, Bt, tc, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    if (ok && p.lam) ok = encode3d(&tm->lam, dt, es, p.lam, L, D, Bt, tc, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    return ok;
}

// The schedule for a shape.  Segments of a group form a chain; when the groups
// alone cannot keep every SM sub-partition's scan warp busy (fewer than half as
// many groups as sub-partitions), the time-parallel schedule cuts each sequence
// into enough segments for about four items per warp and pays a summary pass
// (about two thirds of a scan) to run them all at once.  Returns the segment
// count of the time-parallel schedule, or 0 for the chained one.
int64_t parallel_segments(const FwdParams &p, int sms, int64_t *seg_steps) {
    const int64_t groups = ((p.dim + 31) / 32) * p.batch;
    const int64_t workers = static_cast<int64_t>(kPairs) * sms;
    if (2 * groups > workers) return 0;
    const int64_t want = (4 * workers + groups - 1) / groups;
    int64_t steps = (p.seqlen + want - 1) / want;
    steps = (steps + 31) / 32 * 32;
    if (steps < 256) steps = 256;
    const int64_t segs = (p.seqlen + steps - 1) / steps;
    if (segs < 2) return 0;
    *seg_steps = steps;
    return segs;
}

// Persistent launch: one CTA of kPairs warp triples per SM (or fewer when there
// are fewer items); the S4D instance, then the general one.
template <typename T, bool VEC, bool CONV, bool TRAP, bool STATES>
int launch_pass(const FwdParams &p, const FwdScratch &sc, const TmaMaps &tm, int sms, cudaStream_t stream) {
    const int64_t groups = ((p.dim + 31) / 32) * p.batch;
    const int64_t items = groups * ((p.seqlen + p.seg_steps - 1) / p.seg_steps);
    const int64_t want = (items + kPairs - 1) / kPairs;
    const int64_t ctas = want < sms ? want : sms;
    const int smem = FwdSmem<T, TRAP, CONV>::kTotal;
    scan_fwd_kernel<T, VEC, true, CONV, TRAP, STATES>
        <<<static_cast<unsigned>(ctas), kFwdThreads, smem, stream>>>(p, sc, tm);
    scan_fwd_kernel<T, VEC, false, CONV, TRAP, STATES>
        <<<static_cast<unsigned>(ctas), kFwdThreads, smem, stream>>>(p, sc, tm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// The kernels of one forward call on zeroed scratch: one chained pass, or the
// summary pass, the segment combine and the second pass of the time-parallel
// schedule (the queue is re-armed between the passes).  STATES: the instances
// for a call with no output (the backward entry's checkpoint pass).
template <typename T, bool VEC, bool CONV, bool TRAP, bool STATES>
int launch_fwd_kernels(FwdParams p, void *scratch, int64_t segs, int sms, cudaStream_t stream) {
    const int64_t groups = ((p.dim + 31) / 32) * p.batch;
    const int smem = FwdSmem<T, TRAP, CONV>::kTotal;
    if (cudaFuncSetAttribute(scan_fwd_kernel<T, VEC, true, CONV, TRAP, STATES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaFuncSetAttribute(scan_fwd_kernel<T, VEC, false, CONV, TRAP, STATES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    TmaMaps tm;
    memset(&tm, 0, sizeof tm);
    if (VEC && !make_maps<T>(p, &tm)) return SSM_ERR_CUDA;
    const FwdScratch sc = fwd_scratch_view(scratch, groups, segs);
    if (segs == 0) {
        p.mode = kChained;
        p.pass = 0;
        p.seg_steps = kSegSteps;
        return launch_pass<T, VEC, CONV, TRAP, STATES>(p, sc, tm, sms, stream);
    }
    p.mode = kSummary;
    p.pass = 0;
    int rc = launch_pass<T, VEC, CONV, TRAP, STATES>(p, sc, tm, sms, stream);
    if (rc != SSM_OK) return rc;
    const int64_t threads = groups * 32;
    segment_combine_kernel<<<static_cast<unsigned>((threads + 127) / 128), 128, 0, stream>>>(p, sc);
    // the second pass takes items from its own queues; the error word of the
    // first pass stays set for the status query
    p.mode = kFromStart;
    p.pass = 1;
    return launch_pass<T, VEC, CONV, TRAP, STATES>(p, sc, tm, sms, stream);
}

// SMs of the current device (the schedule, and so the workspace size, depend on it)
int current_sms(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || *sms < 1)
        return SSM_ERR_CUDA;
    return SSM_OK;
}

// Workspace bytes of a validated shape on a GPU with `sms` SMs.
size_t fwd_workspace_bytes(const FwdParams &p, int sms) {
    FwdParams q = p;
    const int64_t groups = ((p.dim + 31) / 32) * p.batch;
    const int64_t segs = parallel_segments(q, sms, &q.seg_steps);
    return fwd_scratch_bytes(groups, segs);
}

// One forward call on the caller's workspace: zero its flag words, then the kernels.
template <typename T, bool VEC, bool CONV, bool TRAP = false, bool STATES = false>
int launch_fwd(FwdParams p, void *ws, size_t ws_bytes, int sms, bool force_chained, cudaStream_t stream) {
    const int64_t groups = ((p.dim + 31) / 32) * p.batch;
    const int64_t segs = force_chained ? 0 : parallel_segments(p, sms, &p.seg_steps);
    if (ws_bytes < fwd_scratch_bytes(groups, segs)) return SSM_ERR_INVALID_ARG;
    if (cudaMemsetAsync(ws, 0, fwd_scratch_flag_bytes(groups), stream) != cudaSuccess) return SSM_ERR_CUDA;
    return launch_fwd_kernels<T, VEC, CONV, TRAP, STATES>(p, ws, segs, sms, stream);
}

// The convolution in front of the scan, when a forward call has one.
struct ConvArgs {
    const float *w;      // [dim][k]
    const float *bias;   // [dim] or NULL
    int k;               // width, 1..4
    const void *state;   // [batch][dim][k-1] activation dtype, or NULL
    void *state_out;     // [batch][dim][k-1] activation dtype, or NULL; may be `state`
};

// The exponential-trapezoidal rule, when a forward call or step uses it.
struct TrapArgs {
    const void *lam;     // [batch][dim][seqlen] (forward) or [batch][dim] (step), activation dtype
    const void *x_prev;  // [batch][dim] activation dtype, or NULL
    const void *B_prev;  // [batch][dstate] activation dtype, or NULL
};

template <typename T, bool CONV, bool TRAP = false>
int launch_step(const StepParams &p, cudaStream_t stream) {
    const int64_t blocks = (p.batch * p.dim + kStepTile - 1) / kStepTile;
    if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
    if (p.batch * p.dim < (int64_t(1) << 31))
        scan_step_kernel<T, true, CONV, TRAP><<<static_cast<unsigned>(blocks), kStepThreads, 0, stream>>>(p);
    else
        scan_step_kernel<T, false, CONV, TRAP><<<static_cast<unsigned>(blocks), kStepThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// Every check of a decode step's arguments; on success fills `p`.  The state
// and the convolution window are read and written in place; out must not
// overlap anything.
int validate_step(float *state, const void *x, const void *delta, const float *delta_bias, int softplus,
                  const float *A, const void *B, const void *C, const float *D, const void *z, void *out,
                  const ConvArgs *conv, const ssm_dims_t *dims, StepParams *p, const TrapArgs *trap = nullptr) {
    if (!dims) return SSM_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, dim = dims->dim, N = dims->dstate;
    if (!state || !x || !delta || !A || !B || !C || !out) return SSM_ERR_INVALID_ARG;
    if (conv && (!conv->w || (conv->k > 1 && !conv->state_out))) return SSM_ERR_INVALID_ARG;
    if (trap && !trap->lam) return SSM_ERR_INVALID_ARG;
    if (!dims_ok(batch, 1, dim) || N < 1) return SSM_ERR_INVALID_ARG;
    if (N != kNState) return SSM_ERR_UNSUPPORTED;
    if (dims->act_dtype != SSM_F32 && dims->act_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    if (conv && (conv->k < 1 || conv->k > 4)) return SSM_ERR_UNSUPPORTED;
    const size_t es = dims->act_dtype == SSM_F32 ? 4 : 2;
    // state, A, B and C are read (and the state written) as 16-byte vectors per lane
    for (const void *ptr : {(const void *)state, (const void *)A, B, C, trap ? trap->B_prev : nullptr})
        if (ptr && !aligned16(ptr)) return SSM_ERR_MISALIGNED;
    for (const void *ptr : {x, delta, z, (const void *)out, trap ? trap->lam : nullptr, trap ? trap->x_prev : nullptr})
        if (ptr && reinterpret_cast<uintptr_t>(ptr) % es != 0) return SSM_ERR_MISALIGNED;
    for (const void *ptr : {(const void *)delta_bias, (const void *)D})
        if (ptr && !aligned4(ptr)) return SSM_ERR_MISALIGNED;
    if (conv) {
        for (const void *ptr : {(const void *)conv->w, (const void *)conv->bias})
            if (ptr && !aligned4(ptr)) return SSM_ERR_MISALIGNED;
        if (conv->state_out && reinterpret_cast<uintptr_t>(conv->state_out) % es != 0) return SSM_ERR_MISALIGNED;
    }

    const size_t nch = static_cast<size_t>(batch) * dim;
    const Span ins[] = {{x, nch * es}, {delta, nch * es}, {z, z ? nch * es : 0},
                        {B, static_cast<size_t>(batch) * N * es}, {C, static_cast<size_t>(batch) * N * es},
                        {A, static_cast<size_t>(dim) * N * 4}, {D, D ? static_cast<size_t>(dim) * 4 : 0},
                        {delta_bias, delta_bias ? static_cast<size_t>(dim) * 4 : 0},
                        {conv ? conv->w : nullptr, conv ? static_cast<size_t>(dim) * conv->k * 4 : 0},
                        {conv && conv->bias ? conv->bias : nullptr, static_cast<size_t>(dim) * 4},
                        {trap ? trap->lam : nullptr, nch * es}, {trap ? trap->x_prev : nullptr, nch * es},
                        {trap ? trap->B_prev : nullptr, static_cast<size_t>(batch) * N * es}};
    const Span outs[] = {{out, nch * es}, {state, nch * N * 4},
                         {conv && conv->k > 1 ? conv->state_out : nullptr, conv ? nch * (conv->k - 1) * es : 0}};
    for (int o = 0; o < 3; ++o) {
        for (const Span &in : ins)
            if (overlap(outs[o], in)) return SSM_ERR_INVALID_ARG;
        for (int q = o + 1; q < 3; ++q)
            if (overlap(outs[o], outs[q])) return SSM_ERR_INVALID_ARG;
    }

    memset(p, 0, sizeof *p);
    p->state = state; p->x = x; p->delta = delta; p->z = z; p->B = B; p->C = C;
    p->delta_bias = delta_bias; p->A = A; p->D = D; p->out = out;
    p->batch = batch; p->dim = dim; p->softplus = softplus ? 1 : 0;
    if (conv) {
        p->conv_k = conv->k;
        p->conv_w = conv->w;
        p->conv_bias = conv->bias;
        p->conv_state = conv->state_out;
    }
    if (trap) {
        p->lam = trap->lam;
        p->x_prev = trap->x_prev;
        p->B_prev = trap->B_prev;
    }
    return SSM_OK;
}

// Every check of a forward call's arguments (all forward entry points share
// it); on success fills `p` and the activation element size.  Outputs (out,
// h_last, the workspace, the new convolution state) must not overlap any
// input or each other, except that h_last may be h0 itself and the new
// convolution state may be the old one itself.
int validate_fwd(const void *x, const void *delta, const float *delta_bias, int softplus, const float *A,
                 const void *B, const void *C, const float *D, const void *z, const float *h0, void *out,
                 float *h_last, const void *ws, size_t ws_bytes, const ConvArgs *conv, const ssm_dims_t *dims,
                 FwdParams *p, size_t *es_out, const TrapArgs *trap = nullptr) {
    if (!dims) return SSM_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, dim = dims->dim, N = dims->dstate;
    if (!x || !delta || !A || !B || !C || !out) return SSM_ERR_INVALID_ARG;
    if (conv && !conv->w) return SSM_ERR_INVALID_ARG;
    if (trap && !trap->lam) return SSM_ERR_INVALID_ARG;
    if (!dims_ok(batch, L, dim) || N < 1) return SSM_ERR_INVALID_ARG;
    if (N != kNState) return SSM_ERR_UNSUPPORTED;
    if (dims->act_dtype != SSM_F32 && dims->act_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    if (conv && (conv->k < 1 || conv->k > 4)) return SSM_ERR_UNSUPPORTED;
    // TMA coordinates and the work queue's item split are 32-bit
    if (batch > INT32_MAX || L > INT32_MAX - 64 || dim > INT32_MAX - 64) return SSM_ERR_UNSUPPORTED;
    const int64_t groups = ((dim + 31) / 32) * batch;
    if (groups * ((L + 255) / 256) > static_cast<int64_t>(UINT32_MAX) / 2) return SSM_ERR_UNSUPPORTED;
    const size_t es = dims->act_dtype == SSM_F32 ? 4 : 2;
    for (const void *ptr : {x, delta, (const void *)A, B, C, z, (const void *)h0, (const void *)out,
                            (const void *)h_last, ws, trap ? trap->lam : nullptr})
        if (ptr && !aligned16(ptr)) return SSM_ERR_MISALIGNED;
    for (const void *ptr : {(const void *)delta_bias, (const void *)D})
        if (ptr && !aligned4(ptr)) return SSM_ERR_MISALIGNED;
    if (trap)
        for (const void *ptr : {trap->x_prev, trap->B_prev})
            if (ptr && reinterpret_cast<uintptr_t>(ptr) % es != 0) return SSM_ERR_MISALIGNED;
    if (conv) {
        for (const void *ptr : {(const void *)conv->w, (const void *)conv->bias})
            if (ptr && !aligned4(ptr)) return SSM_ERR_MISALIGNED;
        for (const void *ptr : {conv->state, (const void *)conv->state_out})
            if (ptr && reinterpret_cast<uintptr_t>(ptr) % es != 0) return SSM_ERR_MISALIGNED;
    }

    const size_t tok = static_cast<size_t>(batch) * dim * L;
    const size_t st = static_cast<size_t>(batch) * dim * N * 4;
    const size_t cst = conv ? static_cast<size_t>(batch) * dim * (conv->k - 1) * es : 0;
    const Span ins[] = {{x, tok * es}, {delta, tok * es}, {z, z ? tok * es : 0},
                        {B, static_cast<size_t>(batch) * N * L * es}, {C, static_cast<size_t>(batch) * N * L * es},
                        {A, static_cast<size_t>(dim) * N * 4}, {D, D ? static_cast<size_t>(dim) * 4 : 0},
                        {delta_bias, delta_bias ? static_cast<size_t>(dim) * 4 : 0}, {h0, h0 ? st : 0},
                        {conv ? conv->w : nullptr, conv ? static_cast<size_t>(dim) * conv->k * 4 : 0},
                        {conv && conv->bias ? conv->bias : nullptr, static_cast<size_t>(dim) * 4},
                        {conv ? conv->state : nullptr, cst},
                        {trap ? trap->lam : nullptr, tok * es},
                        {trap ? trap->x_prev : nullptr, static_cast<size_t>(batch) * dim * es},
                        {trap ? trap->B_prev : nullptr, static_cast<size_t>(batch) * N * es}};
    const Span outs[] = {{out, tok * es}, {h_last, h_last ? st : 0}, {ws, ws ? ws_bytes : 0},
                         {conv ? conv->state_out : nullptr, cst}};
    const void *alias_of[] = {nullptr, h0, nullptr, conv ? conv->state : nullptr};  // allowed exact alias
    for (int o = 0; o < 4; ++o) {
        for (const Span &in : ins)
            if (overlap(outs[o], in) && !(in.p == alias_of[o] && in.p == outs[o].p)) return SSM_ERR_INVALID_ARG;
        for (int q = o + 1; q < 4; ++q)
            if (overlap(outs[o], outs[q])) return SSM_ERR_INVALID_ARG;
    }
    // the chained schedule's workspace is the least any device needs (the exact
    // size, which depends on the SM count, is checked at launch)
    if (ws && ws_bytes < fwd_scratch_bytes(groups)) return SSM_ERR_INVALID_ARG;

    memset(p, 0, sizeof *p);
    p->x = x; p->delta = delta; p->z = z; p->B = B; p->C = C;
    p->delta_bias = delta_bias; p->A = A; p->D = D; p->h0 = h0;
    p->out = out; p->h_last = h_last;
    p->batch = batch; p->seqlen = L; p->dim = dim;
    p->softplus = softplus ? 1 : 0;
    p->seg_steps = kSegSteps;
    p->spin_limit = kSpinLimit;
    p->flag_bias = 0;
    if (conv) {
        p->conv_k = conv->k;
        p->conv_w = conv->w;
        p->conv_bias = conv->bias;
        p->conv_state = conv->state;
    }
    if (trap) {
        p->lam = trap->lam;
        p->x_prev = trap->x_prev;
        p->B_prev = trap->B_prev;
    }
    *es_out = es;
    return SSM_OK;
}

// The forward call on a validated shape and a workspace of ws_bytes; then,
// for a call with a convolution, the new convolution state.
int dispatch_fwd(const FwdParams &p, size_t es, int act_dtype, void *ws, size_t ws_bytes, bool force_chained,
                 void *conv_state_out, cudaStream_t s) {
    int sms = 0;
    if (current_sms(&sms) != SSM_OK) return SSM_ERR_CUDA;
    const bool vec = (static_cast<size_t>(p.seqlen) * es) % 16 == 0;
    const bool bf = act_dtype == SSM_BF16;
    int rc;
    if (p.conv_k) {
        rc = bf ? (vec ? launch_fwd<bf16raw, true, true>(p, ws, ws_bytes, sms, force_chained, s)
                       : launch_fwd<bf16raw, false, true>(p, ws, ws_bytes, sms, force_chained, s))
                : (vec ? launch_fwd<float, true, true>(p, ws, ws_bytes, sms, force_chained, s)
                       : launch_fwd<float, false, true>(p, ws, ws_bytes, sms, force_chained, s));
        if (rc == SSM_OK && conv_state_out && p.conv_k > 1) {
            const int64_t nch = p.batch * p.dim;
            const unsigned blocks = static_cast<unsigned>((nch + 255) / 256);
            if (bf)
                conv_state_kernel<bf16raw><<<blocks, 256, 0, s>>>(p, conv_state_out);
            else
                conv_state_kernel<float><<<blocks, 256, 0, s>>>(p, conv_state_out);
            rc = cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
        }
        return rc;
    }
    if (p.lam)
        return bf ? (vec ? launch_fwd<bf16raw, true, false, true>(p, ws, ws_bytes, sms, force_chained, s)
                         : launch_fwd<bf16raw, false, false, true>(p, ws, ws_bytes, sms, force_chained, s))
                  : (vec ? launch_fwd<float, true, false, true>(p, ws, ws_bytes, sms, force_chained, s)
                         : launch_fwd<float, false, false, true>(p, ws, ws_bytes, sms, force_chained, s));
    if (!p.out)  // the states alone (the backward entry's checkpoint pass)
        return bf ? (vec ? launch_fwd<bf16raw, true, false, false, true>(p, ws, ws_bytes, sms, force_chained, s)
                         : launch_fwd<bf16raw, false, false, false, true>(p, ws, ws_bytes, sms, force_chained, s))
                  : (vec ? launch_fwd<float, true, false, false, true>(p, ws, ws_bytes, sms, force_chained, s)
                         : launch_fwd<float, false, false, false, true>(p, ws, ws_bytes, sms, force_chained, s));
    return bf ? (vec ? launch_fwd<bf16raw, true, false>(p, ws, ws_bytes, sms, force_chained, s)
                     : launch_fwd<bf16raw, false, false>(p, ws, ws_bytes, sms, force_chained, s))
              : (vec ? launch_fwd<float, true, false>(p, ws, ws_bytes, sms, force_chained, s)
                     : launch_fwd<float, false, false>(p, ws, ws_bytes, sms, force_chained, s));
}

// Workspace of the backward pass: first the scratch of the forward pass that
// stores the checkpoints (so ssm_scan_fwd_status reads its error word), then
// the states at every segment start (64 B per channel and segment of kCkptSteps steps).
FwdParams bwd_ckpt_params(int64_t batch, int64_t L, int64_t dim) {
    FwdParams f;
    memset(&f, 0, sizeof f);
    f.batch = batch; f.seqlen = L; f.dim = dim;
    f.seg_steps = kSegSteps;
    f.spin_limit = kSpinLimit;
    return f;
}
// The forward scratch grows with the SM count (more segments on the two-pass
// schedule); it is sized for kBwdMaxSms, so the size needs no device.
constexpr int kBwdMaxSms = 256;
size_t bwd_fwd_scratch_bytes(int64_t batch, int64_t L, int64_t dim) {
    return (fwd_workspace_bytes(bwd_ckpt_params(batch, L, dim), kBwdMaxSms) + 255) / 256 * 256;
}
size_t bwd_workspace_bytes(int64_t batch, int64_t L, int64_t dim) {
    return bwd_fwd_scratch_bytes(batch, L, dim) +
           (static_cast<size_t>(batch) * dim * bwd_segments(L) * kNState * 4 + 255) / 256 * 256;
}

template <typename T>
int launch_bwd(BwdParams p, cudaStream_t s) {
    const int smem = static_cast<int>(sizeof(BwdSmem));
    if (cudaFuncSetAttribute(scan_bwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    const size_t bn = static_cast<size_t>(p.batch) * kNState * p.seqlen * 4;
    if (cudaMemsetAsync(p.dA, 0, static_cast<size_t>(p.dim) * kNState * 4, s) != cudaSuccess ||
        cudaMemsetAsync(p.dB, 0, bn, s) != cudaSuccess || cudaMemsetAsync(p.dC, 0, bn, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (p.dD && cudaMemsetAsync(p.dD, 0, static_cast<size_t>(p.dim) * 4, s) != cudaSuccess) return SSM_ERR_CUDA;
    if (p.dbias && cudaMemsetAsync(p.dbias, 0, static_cast<size_t>(p.dim) * 4, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    const int64_t groups = bwd_groups16(p.batch, p.dim);
    scan_bwd_kernel<T><<<static_cast<unsigned>(groups), 32, smem, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace

extern "C" {

int ssm_version(void) { return kVersion; }

const char *ssm_strerror(int code) {
    switch (code) {
        case SSM_OK: return "ok";
        case SSM_ERR_INVALID_ARG: return "invalid argument (NULL required pointer, size < 1, overlapping buffers, or a workspace that is too small)";
        case SSM_ERR_UNSUPPORTED: return "unsupported (dstate must be 16, dtype f32 or bf16, sizes within limits)";
        case SSM_ERR_MISALIGNED: return "misaligned pointer (16-byte alignment required)";
        case SSM_ERR_CUDA: return "CUDA launch or query error";
        case SSM_ERR_TIMEOUT: return "bounded device wait timed out; the call's results are void";
        default: return "unknown error code";
    }
}

int ssm_scan_fwd_workspace_size(const ssm_dims_t *dims, int sm_count, size_t *bytes) {
    if (!dims || !bytes) return SSM_ERR_INVALID_ARG;
    if (!dims_ok(dims->batch, dims->seqlen, dims->dim) || dims->dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dims->dstate != kNState) return SSM_ERR_UNSUPPORTED;
    if (sm_count <= 0 && current_sms(&sm_count) != SSM_OK) return SSM_ERR_CUDA;
    FwdParams p;
    memset(&p, 0, sizeof p);
    p.batch = dims->batch; p.seqlen = dims->seqlen; p.dim = dims->dim;
    p.seg_steps = kSegSteps;
    *bytes = fwd_workspace_bytes(p, sm_count);
    return SSM_OK;
}

int ssm_scan_fwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                 const float *A, const void *B, const void *C, const float *D, const void *z,
                 const float *h0, void *out, float *h_last, void *workspace, size_t workspace_bytes,
                 const ssm_dims_t *dims, ssm_stream_t stream) {
    if (!workspace) return SSM_ERR_INVALID_ARG;
    FwdParams p;
    size_t es = 0;
    const int rc = validate_fwd(x, delta, delta_bias, softplus, A, B, C, D, z, h0, out, h_last, workspace,
                                workspace_bytes, nullptr, dims, &p, &es);
    if (rc != SSM_OK) return rc;
    return dispatch_fwd(p, es, dims->act_dtype, workspace, workspace_bytes, false, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

int ssm_debug_fwd_flag_timeout(const void *x, const void *delta, const float *delta_bias, int softplus,
                               const float *A, const void *B, const void *C, const float *D, const void *z,
                               const float *h0, void *out, float *h_last, void *workspace,
                               size_t workspace_bytes, uint32_t spin_limit, const ssm_dims_t *dims,
                               ssm_stream_t stream) {
    if (!workspace) return SSM_ERR_INVALID_ARG;
    FwdParams p;
    size_t es = 0;
    const int rc = validate_fwd(x, delta, delta_bias, softplus, A, B, C, D, z, h0, out, h_last, workspace,
                                workspace_bytes, nullptr, dims, &p, &es);
    if (rc != SSM_OK) return rc;
    p.spin_limit = spin_limit;
    p.flag_bias = 1u << 30;  // no segment flag ever reaches this
    return dispatch_fwd(p, es, dims->act_dtype, workspace, workspace_bytes, true, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

int ssm_scan_step(float *state, const void *x, const void *delta, const float *delta_bias,
                  int softplus, const float *A, const void *B, const void *C, const float *D,
                  const void *z, void *out, const ssm_dims_t *dims, ssm_stream_t stream) {
    StepParams p;
    const int rc = validate_step(state, x, delta, delta_bias, softplus, A, B, C, D, z, out, nullptr, dims, &p);
    if (rc != SSM_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return dims->act_dtype == SSM_BF16 ? launch_step<bf16raw, false>(p, s) : launch_step<float, false>(p, s);
}

int ssm_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_bias, int conv_width,
                      const void *conv_state, void *conv_state_out, const void *delta, const float *delta_bias,
                      int softplus, const float *A, const void *B, const void *C, const float *D, const void *z,
                      const float *h0, void *out, float *h_last, void *workspace, size_t workspace_bytes,
                      const ssm_dims_t *dims, ssm_stream_t stream) {
    if (!workspace) return SSM_ERR_INVALID_ARG;
    const ConvArgs conv{conv_w, conv_bias, conv_width, conv_state, conv_state_out};
    FwdParams p;
    size_t es = 0;
    const int rc = validate_fwd(x, delta, delta_bias, softplus, A, B, C, D, z, h0, out, h_last, workspace,
                                workspace_bytes, &conv, dims, &p, &es);
    if (rc != SSM_OK) return rc;
    return dispatch_fwd(p, es, dims->act_dtype, workspace, workspace_bytes, false, conv_state_out,
                        reinterpret_cast<cudaStream_t>(stream));
}

int ssm_trap_scan_fwd(const void *x, const void *delta, const float *delta_bias, int softplus, const void *lam,
                      const float *A, const void *B, const void *C, const float *D, const void *z, const float *h0,
                      const void *x_prev, const void *B_prev, void *out, float *h_last, void *workspace,
                      size_t workspace_bytes, const ssm_dims_t *dims, ssm_stream_t stream) {
    if (!workspace) return SSM_ERR_INVALID_ARG;
    const TrapArgs trap{lam, x_prev, B_prev};
    FwdParams p;
    size_t es = 0;
    const int rc = validate_fwd(x, delta, delta_bias, softplus, A, B, C, D, z, h0, out, h_last, workspace,
                                workspace_bytes, nullptr, dims, &p, &es, &trap);
    if (rc != SSM_OK) return rc;
    return dispatch_fwd(p, es, dims->act_dtype, workspace, workspace_bytes, false, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

int ssm_trap_scan_step(float *state, const void *x, const void *delta, const float *delta_bias, int softplus,
                       const void *lam, const float *A, const void *B, const void *C, const float *D, const void *z,
                       const void *x_prev, const void *B_prev, void *out, const ssm_dims_t *dims,
                       ssm_stream_t stream) {
    const TrapArgs trap{lam, x_prev, B_prev};
    StepParams p;
    const int rc = validate_step(state, x, delta, delta_bias, softplus, A, B, C, D, z, out, nullptr, dims, &p, &trap);
    if (rc != SSM_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return dims->act_dtype == SSM_BF16 ? launch_step<bf16raw, false, true>(p, s) : launch_step<float, false, true>(p, s);
}

int ssm_scan_bwd_workspace_size(const ssm_dims_t *dims, size_t *bytes) {
    if (!dims || !bytes) return SSM_ERR_INVALID_ARG;
    if (!dims_ok(dims->batch, dims->seqlen, dims->dim) || dims->dstate < 1) return SSM_ERR_INVALID_ARG;
    if (dims->dstate != kNState) return SSM_ERR_UNSUPPORTED;
    *bytes = bwd_workspace_bytes(dims->batch, dims->seqlen, dims->dim);
    return SSM_OK;
}

int ssm_scan_bwd(const void *x, const void *delta, const float *delta_bias, int softplus, const float *A,
                 const void *B, const void *C, const float *D, const void *z, const float *h0, const void *dout,
                 const float *dh_last, void *dx, void *ddelta, void *dz, float *dB, float *dC, float *dA,
                 float *dD, float *dbias, float *dh0, void *workspace, size_t workspace_bytes,
                 const ssm_dims_t *dims, ssm_stream_t stream) {
    if (!dims) return SSM_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, dim = dims->dim, N = dims->dstate;
    if (!x || !delta || !A || !B || !C || !dout || !dx || !ddelta || !dB || !dC || !dA || !workspace)
        return SSM_ERR_INVALID_ARG;
    if (z && !dz) return SSM_ERR_INVALID_ARG;
    if (!dims_ok(batch, L, dim) || N < 1) return SSM_ERR_INVALID_ARG;
    if (N != kNState) return SSM_ERR_UNSUPPORTED;
    if (dims->act_dtype != SSM_F32 && dims->act_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    if (bwd_groups16(batch, dim) > INT32_MAX) return SSM_ERR_UNSUPPORTED;  // grid.x holds the groups
    const size_t es = dims->act_dtype == SSM_F32 ? 4 : 2;
    for (const void *ptr : {x, delta, (const void *)A, B, C, z, (const void *)h0, dout, (const void *)dx,
                            (const void *)ddelta, (const void *)(z ? dz : nullptr), (const void *)dB,
                            (const void *)dC, (const void *)dA, (const void *)dh_last, (const void *)dh0,
                            (const void *)workspace})
        if (ptr && !aligned16(ptr)) return SSM_ERR_MISALIGNED;
    for (const void *ptr : {(const void *)delta_bias, (const void *)D, (const void *)dD, (const void *)dbias})
        if (ptr && !aligned4(ptr)) return SSM_ERR_MISALIGNED;
    // the checkpoint pass is the forward kernel: its 32-bit limits apply
    if (batch > INT32_MAX || L > INT32_MAX - 64 || dim > INT32_MAX - 64) return SSM_ERR_UNSUPPORTED;
    if (((dim + 31) / 32) * batch * ((L + 255) / 256) > static_cast<int64_t>(UINT32_MAX) / 2)
        return SSM_ERR_UNSUPPORTED;
    if (workspace_bytes < bwd_workspace_bytes(batch, L, dim)) return SSM_ERR_INVALID_ARG;

    const size_t tok = static_cast<size_t>(batch) * dim * L, bn = static_cast<size_t>(batch) * N * L;
    const size_t st = static_cast<size_t>(batch) * dim * N * 4;
    const Span ins[] = {{x, tok * es}, {delta, tok * es}, {z, z ? tok * es : 0}, {B, bn * es}, {C, bn * es},
                        {A, static_cast<size_t>(dim) * N * 4}, {D, D ? static_cast<size_t>(dim) * 4 : 0},
                        {delta_bias, delta_bias ? static_cast<size_t>(dim) * 4 : 0}, {h0, h0 ? st : 0},
                        {dout, tok * es}, {dh_last, dh_last ? st : 0}};
    const Span outs[] = {{dx, tok * es}, {ddelta, tok * es}, {z ? dz : nullptr, tok * es}, {dB, bn * 4},
                         {dC, bn * 4}, {dA, static_cast<size_t>(dim) * N * 4},
                         {dD, dD ? static_cast<size_t>(dim) * 4 : 0},
                         {dbias, dbias ? static_cast<size_t>(dim) * 4 : 0}, {dh0, dh0 ? st : 0},
                         {workspace, workspace_bytes}};
    constexpr int kOuts = sizeof(outs) / sizeof(outs[0]);
    for (int o = 0; o < kOuts; ++o) {
        for (const Span &in : ins)
            if (overlap(outs[o], in)) return SSM_ERR_INVALID_ARG;
        for (int q = o + 1; q < kOuts; ++q)
            if (overlap(outs[o], outs[q])) return SSM_ERR_INVALID_ARG;
    }

    BwdParams p;
    memset(&p, 0, sizeof p);
    p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C; p.dout = dout;
    p.delta_bias = delta_bias; p.A = A; p.D = D; p.h0 = h0; p.dh_last = dh_last;
    p.dx = dx; p.ddelta = ddelta; p.dz = z ? dz : nullptr;
    p.dA = dA; p.dD = dD; p.dbias = dbias; p.dh0 = dh0; p.dB = dB; p.dC = dC;
    const size_t fws = bwd_fwd_scratch_bytes(batch, L, dim);
    p.ckpt = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + fws);
    p.batch = batch; p.seqlen = L; p.dim = dim; p.softplus = softplus ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the checkpoints: the forward scan with no output, storing its state every
    // kCkptSteps steps (its scratch at the start of the workspace)
    FwdParams f = bwd_ckpt_params(batch, L, dim);
    f.x = x; f.delta = delta; f.B = B; f.C = C;
    f.delta_bias = delta_bias; f.A = A; f.h0 = h0;
    f.softplus = p.softplus;
    f.ckpt = p.ckpt;
    f.ckpt_segs = bwd_segments(L);
    const int rc = dispatch_fwd(f, es, dims->act_dtype, workspace, fws, false, nullptr, s);
    if (rc != SSM_OK) return rc;
    return dims->act_dtype == SSM_BF16 ? launch_bwd<bf16raw>(p, s) : launch_bwd<float>(p, s);
}

// SSD workspace: bytes [0, 256) hold the CTA order counter (at 0) and the error
// word (at 16) of every workspace layout; [256, 2048) one hand-off flag per CTA;
// from 2048 one P x N float32 state per CTA.
constexpr int64_t kSsdFlagOff = 256, kSsdSlotOff = 2048, kSsdMaxCtas = (kSsdSlotOff - kSsdFlagOff) / 4;
constexpr int64_t kSsdSlotBytes = static_cast<int64_t>(kSsdP) * kSsdN * 4;

// CTAs of a split launch on sms SMs (0: sequences are not split)
static int64_t ssd_split_ctas(int64_t nseq, int sms) {
    const int64_t cap = std::min<int64_t>(sms, kSsdMaxCtas);
    return nseq > cap ? cap : 0;
}

int ssm_ssd_fwd_workspace_size(const ssm_ssd_dims_t *dims, int sm_count, size_t *bytes) {
    if (!dims || !bytes || dims->batch < 1 || dims->heads < 1) return SSM_ERR_INVALID_ARG;
    if (sm_count <= 0 && current_sms(&sm_count) != SSM_OK) return SSM_ERR_CUDA;
    const int64_t ctas = ssd_split_ctas(dims->batch * dims->heads, sm_count);
    *bytes = ctas ? static_cast<size_t>(kSsdSlotOff + ctas * kSsdSlotBytes) : 256;
    return SSM_OK;
}

// ssm_ssd_fwd with the hand-off flag value and the poll bound of the waits
static int ssd_fwd_impl(const void *x, const void *dt, const float *dt_bias, int softplus, const float *A,
                        const void *B, const void *C, const float *D, const float *h0, void *y, float *h_last,
                        void *workspace, size_t workspace_bytes, const ssm_ssd_dims_t *dims, ssm_stream_t stream,
                        uint32_t flag_want, uint32_t spin_limit) {
    if (!dims || !x || !dt || !A || !B || !C || !y || !workspace) return SSM_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, H = dims->heads, P = dims->headdim, G = dims->groups,
                  N = dims->dstate;
    if (batch < 1 || L < 1 || H < 1 || P < 1 || G < 1 || N < 1 || H % G != 0) return SSM_ERR_INVALID_ARG;
    if (P != kSsdP || N != kSsdN || dims->act_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
    // grid.x holds batch * heads; TMA coordinates and strides are 32-bit and 40-bit
    if (batch * H > INT32_MAX || L > INT32_MAX - kSsdQ ||
        static_cast<double>(batch) * L * H * P * 2 >= static_cast<double>(1ull << 40) ||
        static_cast<double>(batch) * L * G * N * 2 >= static_cast<double>(1ull << 40))
        return SSM_ERR_UNSUPPORTED;
    if (workspace_bytes < 256) return SSM_ERR_INVALID_ARG;
    for (const void *ptr : {x, B, C, (const void *)y, (const void *)h0, (const void *)h_last, (const void *)workspace})
        if (ptr && !aligned16(ptr)) return SSM_ERR_MISALIGNED;
    for (const void *ptr : {(const void *)dt_bias, (const void *)A, (const void *)D})
        if (ptr && !aligned4(ptr)) return SSM_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(dt) % 2 != 0) return SSM_ERR_MISALIGNED;
    const size_t tok = static_cast<size_t>(batch) * L * H * P * 2, bc = static_cast<size_t>(batch) * L * G * N * 2;
    const size_t st = static_cast<size_t>(batch) * H * P * N * 4;
    const Span ins[] = {{x, tok}, {dt, static_cast<size_t>(batch) * L * H * 2}, {B, bc}, {C, bc},
                        {A, static_cast<size_t>(H) * 4}, {dt_bias, dt_bias ? static_cast<size_t>(H) * 4 : 0},
                        {D, D ? static_cast<size_t>(H) * 4 : 0}, {h0, h0 ? st : 0}};
    const Span outs[] = {{y, tok}, {h_last, h_last ? st : 0}, {workspace, workspace_bytes}};
    for (int o = 0; o < 3; ++o) {
        for (const Span &in : ins)
            if (overlap(outs[o], in)) return SSM_ERR_INVALID_ARG;
        for (int q = o + 1; q < 3; ++q)
            if (overlap(outs[o], outs[q])) return SSM_ERR_INVALID_ARG;
    }
    // more sequences than SMs: persistent CTAs over equal ranges of chunks, when
    // the workspace holds the hand-offs; else one CTA per sequence
    int sms = 0;
    if (current_sms(&sms) != SSM_OK) return SSM_ERR_CUDA;
    const int64_t nseq = batch * H, chunks = (L + kSsdQ - 1) / kSsdQ;
    int64_t ctas = ssd_split_ctas(nseq, sms), per_cta = chunks;
    if (ctas && workspace_bytes < static_cast<size_t>(kSsdSlotOff + ctas * kSsdSlotBytes)) ctas = 0;
    if (ctas) {
        per_cta = (nseq * chunks + ctas - 1) / ctas;  // at least chunks, as nseq > ctas
        ctas = (nseq * chunks + per_cta - 1) / per_cta;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, ctas ? kSsdSlotOff : 256, s) != cudaSuccess) return SSM_ERR_CUDA;
    uint8_t *wb = static_cast<uint8_t *>(workspace);
    SsdParams prm;
    prm.order = ctas ? reinterpret_cast<uint32_t *>(wb) : nullptr;
    prm.flags = ctas ? reinterpret_cast<uint32_t *>(wb + kSsdFlagOff) : nullptr;
    prm.slots = ctas ? reinterpret_cast<float *>(wb + kSsdSlotOff) : nullptr;
    prm.units_per_cta = per_cta;
    prm.flag_want = flag_want;
    prm.spin_limit = spin_limit;
    prm.dt = dt;
    prm.dt_bias = dt_bias; prm.A = A; prm.D = D; prm.h0 = h0;
    prm.y = y; prm.h_last = h_last;
    prm.error = fwd_scratch_view(workspace, 0).error;
    prm.batch = batch; prm.seqlen = L; prm.heads = H; prm.groups = G; prm.softplus = softplus ? 1 : 0;
    SsdMaps tm;
    constexpr CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const uint64_t ub = static_cast<uint64_t>(batch), uL = static_cast<uint64_t>(L);
    if (!encode4d(&tm.x, bf, 2, x, kSsdP, static_cast<uint64_t>(H), uL, ub, 64, kSsdQ, sw) ||
        !encode4d(&tm.B, bf, 2, B, kSsdN, static_cast<uint64_t>(G), uL, ub, 64, kSsdQ, sw) ||
        !encode4d(&tm.C, bf, 2, C, kSsdN, static_cast<uint64_t>(G), uL, ub, 64, kSsdQ, sw))
        return SSM_ERR_CUDA;
    const int smem = SsdSmem::kTotal;
    if (cudaFuncSetAttribute(ssd_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    ssd_fwd_kernel<<<static_cast<unsigned>(ctas ? ctas : nseq), kSsdThreads, smem, s>>>(prm, tm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_ssd_fwd(const void *x, const void *dt, const float *dt_bias, int softplus, const float *A, const void *B,
                const void *C, const float *D, const float *h0, void *y, float *h_last, void *workspace,
                size_t workspace_bytes, const ssm_ssd_dims_t *dims, ssm_stream_t stream) {
    return ssd_fwd_impl(x, dt, dt_bias, softplus, A, B, C, D, h0, y, h_last, workspace, workspace_bytes, dims,
                        stream, 1u, kSsdFlagLimit);
}

int ssm_debug_ssd_flag_timeout(const void *x, const void *dt, const float *dt_bias, int softplus, const float *A,
                               const void *B, const void *C, const float *D, const float *h0, void *y,
                               float *h_last, void *workspace, size_t workspace_bytes, uint32_t spin_limit,
                               const ssm_ssd_dims_t *dims, ssm_stream_t stream) {
    return ssd_fwd_impl(x, dt, dt_bias, softplus, A, B, C, D, h0, y, h_last, workspace, workspace_bytes, dims,
                        stream, 1u << 30, spin_limit);  // no hand-off flag ever reaches this
}

int ssm_conv_scan_step(void *conv_state, float *state, const void *x, const float *conv_w,
                       const float *conv_bias, int conv_width, const void *delta, const float *delta_bias,
                       int softplus, const float *A, const void *B, const void *C, const float *D,
                       const void *z, void *out, const ssm_dims_t *dims, ssm_stream_t stream) {
    const ConvArgs conv{conv_w, conv_bias, conv_width, nullptr, conv_state};
    StepParams p;
    const int rc = validate_step(state, x, delta, delta_bias, softplus, A, B, C, D, z, out, &conv, dims, &p);
    if (rc != SSM_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return dims->act_dtype == SSM_BF16 ? launch_step<bf16raw, true>(p, s) : launch_step<float, true>(p, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Allocation-free forward scan.
//
// Some callers cannot allocate device memory while they run the scan: code
// inside a custom allocator or memory-pool callback, runtimes that reserve all
// device memory up front and forbid later allocation, and processes that must
// not touch the CUDA allocator at all.  ssm_scan_fwd_noalloc serves them: it
// runs the same kernels as ssm_scan_fwd, but its work queue, segment flags and
// carried states live in the fixed device array below instead of a caller
// workspace.  The array is part of the library image, so every GPU that loads
// the library holds kNoAllocScratchBytes for the life of the process.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // fits ~1000 groups of 32 channels
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on device `dev` (taken once per device, with
// that device current; the first call on a device does this look-up).
void *noalloc_scratch(int dev) {
    static std::mutex mu;
    static void *addr[64] = {};
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = ptr;
    }
    return addr[dev];
}

}  // namespace

extern "C" int ssm_scan_fwd_noalloc(const void *x, const void *delta, const float *delta_bias, int softplus,
                                    const float *A, const void *B, const void *C, const float *D,
                                    const void *z, const float *h0, void *out, float *h_last,
                                    const ssm_dims_t *dims, ssm_stream_t stream) {
    FwdParams p;
    size_t es = 0;
    const int rc = validate_fwd(x, delta, delta_bias, softplus, A, B, C, D, z, h0, out, h_last, nullptr, 0, nullptr,
                                dims, &p, &es);
    if (rc != SSM_OK) return rc;
    // the work queue of this shape (chained schedule: its scratch does not grow
    // with the sequence) must fit the fixed array
    const int64_t groups = ((p.dim + 31) / 32) * p.batch;
    if (fwd_scratch_bytes(groups) > kNoAllocScratchBytes) return SSM_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
    void *scratch = noalloc_scratch(dev);
    if (!scratch) return SSM_ERR_CUDA;
    // the array keeps the previous call's contents: launch_fwd zeroes the queue
    // counters, error word and segment flags (the carries need not start at zero)
    return dispatch_fwd(p, es, dims->act_dtype, scratch, kNoAllocScratchBytes, true, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int ssm_scan_fwd_status(const void *workspace, ssm_stream_t stream) {
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    if (!ws) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
        ws = static_cast<const uint8_t *>(noalloc_scratch(dev));
        if (!ws) return SSM_ERR_CUDA;
    }
    if (!aligned16(ws)) return SSM_ERR_MISALIGNED;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SSM_ERR_CUDA;
    // the error word sits in the fixed header of every workspace layout
    const FwdScratch view = fwd_scratch_view(const_cast<uint8_t *>(ws), 0);
    uint32_t err = 0;
    if (cudaMemcpy(&err, view.error, sizeof err, cudaMemcpyDeviceToHost) != cudaSuccess)
        return SSM_ERR_CUDA;
    return err ? SSM_ERR_TIMEOUT : SSM_OK;
}
