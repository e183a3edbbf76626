// scan_fwd.cuh -- forward selective scan (S6) for sm_100a.
//
// Gu & Dao, "Mamba: Linear-Time Sequence Modeling with Selective State
// Spaces", Appendix D "Hardware-aware Algorithm For Selective SSMs" ("Speed"):
// the scan is fused (discretisation, recurrence, readout and gating in one
// pass, reading x, delta, z, B, C once and writing only out and the final
// state) and chunked along L, each chunk continuing from the carried state.
//
// Work layout.  One lane owns one channel (b, d) and keeps its 16 float32
// states in registers, so the recurrence h_t = exp(dt_t A) h_{t-1} + dt_t B_t
// x_t costs one pass per element and no extra parallel-scan work.  A warp
// covers 32 consecutive channels of one sequence (a group).  Each SM runs one
// persistent CTA of four warp triples, one triple per SM sub-partition: a prep
// warp stages 32-step chunks with TMA (one 64-byte row per channel and tensor,
// 64-byte swizzle, so 32 lanes reading 32 rows hit distinct banks), widens B|C
// to a float32 time-major table and computes the per-step scalars; a scan warp
// runs the recurrence and the readout, reading B|C with warp-uniform loads; a
// post warp applies the D skip and the gate and stores the output tile with
// TMA.  The triple hands chunks along through mbarriers.
//
// Per chunk, the per-step scalar work (softplus step size, decay base r,
// input u = dt x, gate) runs stage by stage over all step pairs, which lets
// the special-function latencies of independent steps overlap; the state
// update then only carries h from step to step.
//
// Discretisation (the "Mamba3" post: Mamba-1 pairs zero-order hold with an
// Euler step): Abar = exp(dt A) = ex2(dt A log2 e).  When every A[d, n] of a
// warp's channels equals (n + 1) A[d, 0] exactly (the S4D-real family),
// Abar_n = r^(n+1) with r = exp(dt A[d, 0]) is built by multiplication (one
// MUFU op per step and channel instead of sixteen); other A rows take the
// per-state exponential in a separate kernel instance.
#pragma once

#include <type_traits>

#include <cuda.h>

#include "common.cuh"

namespace ssm {

constexpr int kCkptSteps = 16;  // spacing of the states a checkpoint pass stores

struct FwdParams {
    const void *x, *delta, *z, *B, *C;
    const float *delta_bias, *A, *D, *h0;
    void *out;      // NULL: no output (a checkpoint pass)
    float *h_last;
    // When set, the state at every kCkptSteps-th step of every channel:
    // ckpt[(b * dim + d) * ckpt_segs + t / kCkptSteps][16], the state before step t.
    float *ckpt;
    int64_t ckpt_segs;
    int64_t batch, seqlen, dim;
    int softplus;
    // kChained: segments of a group run in order, each starting from its
    // predecessor's carried state.  kSummary and kFromStart are the two scan passes
    // of the time-parallel schedule: every segment first runs from a zero state and
    // records its end state and decay product; after segment_combine_kernel has
    // turned those into start states, every segment runs again from its own.
    int mode;
    int pass;           // 0: the only or the summary pass; 1: the second pass (its own queues)
    int64_t seg_steps;  // steps per segment, a multiple of 32
    // Bound of the inter-segment flag wait (polls 64 ns apart), and an offset
    // added to the awaited segment count.  The library passes kSpinLimit and 0;
    // the wait-timeout test entry point passes a small bound and an offset no
    // flag ever reaches, so the wait gives up deterministically.
    uint32_t spin_limit;
    uint32_t flag_bias;
    // The short causal convolution in front of the scan (conv_k = 0: none).
    // x is then the raw input, and the scan's x is silu(conv(x)), with
    // conv_w[d][k] multiplying x[t - conv_k + 1 + k] (1 <= conv_k <= 4).
    int conv_k;
    const float *conv_w;        // [dim][conv_k]
    const float *conv_bias;     // [dim] or NULL
    const void *conv_state;     // [batch][dim][conv_k - 1] raw inputs before t = 0, or NULL
    // The exponential-trapezoidal rule (lam != NULL): lam [batch][dim][L] mixes
    // the interval's two ends; x_prev [batch][dim] and B_prev [batch][16] are
    // the input before t = 0 (zero unless both are given).
    const void *lam, *x_prev, *B_prev;
};
constexpr int kChained = 0, kSummary = 1, kFromStart = 2;

// TMA descriptors of the aligned path: activations as 3-D [batch][dim][L]
// tensors with [1][32][TC] boxes and the 64-byte swizzle (the same XOR layout
// as swz()), B and C as [batch][16][L] with [1][16][TC] boxes.
struct TmaMaps {
    CUtensorMap x, delta, z, B, C, out, lam;
};

constexpr int kPairs = 4;                    // warp triples per CTA (one per SM sub-partition)
constexpr int kFwdThreads = 96 * kPairs;     // warps 0..3 scan, 4..7 stage + prepare, 8..11 finish
constexpr int kRowBytes = 64;  // bytes of one channel row of a chunk
constexpr int kPieces = kRowBytes / 16;
constexpr int kBCPitch = 36;   // floats per time row of widened B|C (32 used; float 32 holds C.B with TRAP)

// Shared memory of one warp triple.  Stages hold raw chunks (x, delta, z
// tiles, the B, C rows and, with TRAP, the lambda tile); bcf, ur and g are
// double-buffered per chunk parity.  bcf, ur and g carry one spare step row
// so that the scan warp's step-ahead preparation can run unconditionally on a
// chunk's last step.  The g table holds one float per step and lane: with
// TRAP the end weight g_t, with CONV the skip term D xc_t.  TRAP and CONV keep
// two stages instead of three to make room for it (and TRAP's lambda tile).
template <typename T, bool TRAP = false, bool CONV = false>
struct FwdSmem {
    static constexpr int kTC = kRowBytes / Act<T>::kBytes;          // timesteps per chunk
    static constexpr int kTileBytes = 32 * kRowBytes;               // one [32 ch][TC] tile
    static constexpr int kStages = (TRAP || CONV) ? 2 : 3;          // staged chunks per pair
    static constexpr int kBCRawOff = 3 * kTileBytes;                // raw B|C rows in a stage
    static constexpr int kLamOff = kBCRawOff + 2 * kNState * kRowBytes;
    static constexpr int kStageBytes = kLamOff + (TRAP ? kTileBytes : 0);
    static constexpr int kBCFBytes = (kTC + 1) * kBCPitch * 4;      // widened B|C, time-major
    static constexpr int kURBytes = (kTC + 1) * 32 * 8;             // float2 (u, r) per [t][lane]
    static constexpr int kGBytes = (TRAP || CONV) ? (kTC + 1) * 32 * 4 : 0;  // float per [t][lane]
    static constexpr int kBCFOff = kStages * kStageBytes;
    static constexpr int kUROff = kBCFOff + 2 * kBCFBytes;
    static constexpr int kGOff = kUROff + 2 * kURBytes;
    static constexpr int kDescOff = kGOff + 2 * kGBytes;            // ring of 8 chunk descriptors
    static constexpr int kBarOff = kDescOff + 8 * 64;               // ready[2], done[4], posted[2], full[kStages],
                                                                    // dready[4], then the load count
    static constexpr int kPairBytes = (kBarOff + (12 + kStages) * 8 + 8 + 1023) / 1024 * 1024;
    static constexpr int kTotal = kPairs * kPairBytes + 1024;       // + slack to align the base to 1 KB
};
static_assert(FwdSmem<bf16raw, true>::kTotal <= 227 * 1024, "shared memory of the trapezoidal kernel");
static_assert(FwdSmem<bf16raw, false, true>::kTotal <= 227 * 1024, "shared memory of the convolution kernel");
static_assert(FwdSmem<bf16raw, false>::kTotal <= 227 * 1024, "shared memory of the kernel");

__device__ __forceinline__ int swz(int row, int pc) { return pc ^ ((row >> 1) & 3); }

// Row t (32 floats, one per channel of the group) of a chunk's y.  With
// YS (three stages, loads issued by the post warp) y goes to the chunk's stage,
// over the delta tile (steps 0..15) and the raw B|C rows (steps 16..31), which
// the prep warp has consumed; the (u, r) table is then free once the scan is
// done with it.  Otherwise y goes over the (u, r) table's row t (lanes 0..15's
// pairs, already consumed), as the prep warp waits for the post warp anyway.
template <bool YS>
__device__ __forceinline__ float *y_row(uint8_t *stage, const float2 *ur, int t) {
    constexpr int TB = 32 * kRowBytes;
    if constexpr (YS)
        return reinterpret_cast<float *>(stage + (t < 16 ? TB + t * 128 : 3 * TB + (t - 16) * 128));
    else
        return const_cast<float *>(reinterpret_cast<const float *>(ur + t * 32));
}

// ---- staging one chunk [t0, t0 + TC) of a warp's 32 channels element by element
// (rows that are not 16-byte aligned, L * size % 16 != 0, cannot use TMA)
template <typename T, bool TRAP = false>
__device__ __forceinline__ void load_chunk_sync(const FwdParams &p, uint8_t *stage, int64_t b,
                                                int64_t d0, int64_t t0, int lane) {
    using AT = Act<T>;
    using SM = FwdSmem<T, TRAP>;
    using W = typename std::conditional<AT::kBytes == 2, uint16_t, uint32_t>::type;
    constexpr int PP = AT::kPerPiece, TC = SM::kTC;
    const int64_t L = p.seqlen;
    const void *const srcs[4] = {p.x, p.delta, p.z, TRAP ? p.lam : nullptr};
    const int offs[4] = {0, SM::kTileBytes, 2 * SM::kTileBytes, SM::kLamOff};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (srcs[k] == nullptr) continue;
        const W *base = static_cast<const W *>(srcs[k]);
        uint8_t *tile = stage + offs[k];
        for (int row = 0; row < 32; ++row) {
            const int64_t d = d0 + row;
            for (int col = lane; col < TC; col += 32) {
                const int64_t t = t0 + col;
                const W v = (d < p.dim && t < L) ? base[(b * p.dim + d) * L + t] : W(0);
                *reinterpret_cast<W *>(tile + row * kRowBytes + (swz(row, col / PP) << 4) +
                                       (col % PP) * AT::kBytes) = v;
            }
        }
    }
    for (int j = 0; j < 2 * kNState; ++j) {
        const W *base = static_cast<const W *>(j >= kNState ? p.C : p.B);
        for (int col = lane; col < TC; col += 32) {
            const int64_t t = t0 + col;
            const W v = t < L ? base[(b * kNState + (j & 15)) * L + t] : W(0);
            *reinterpret_cast<W *>(stage + SM::kBCRawOff + j * kRowBytes + col * AT::kBytes) = v;
        }
    }
}

// Widen the chunk's B and C to float32, time-major: bcf[t][0..15] = B[.][t],
// bcf[t][16..31] = C[.][t].  Lanes take consecutive t so each 16-byte store
// of a quarter-warp lands in a distinct bank group (pitch 36 floats).
// With TRAP the B half is shifted down one row (row t holds B of step t-1,
// row TC the chunk's last B; the caller fills row 0's B half), and float 32
// of row t holds C_t . B_t.
template <typename T, bool TRAP = false>
__device__ __forceinline__ void widen_bc(const uint8_t *raw, float *bcf, int lane) {
    using AT = Act<T>;
    using W = typename std::conditional<AT::kBytes == 2, uint16_t, uint32_t>::type;
    constexpr int TC = FwdSmem<T>::kTC;
    auto rd = [&](int j, int t) {
        const W w = reinterpret_cast<const W *>(raw + j * kRowBytes)[t];
        if constexpr (AT::kBytes == 2)
            return __uint_as_float(static_cast<uint32_t>(w) << 16);
        else
            return __uint_as_float(w);
    };
#pragma unroll
    for (int item = lane; item < TC * 8; item += 32) {
        const int t = item % TC, jg = item / TC;
        float v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = rd(jg * 4 + q, t);
        const int row = (TRAP && jg < 4) ? t + 1 : t;
        *reinterpret_cast<float4 *>(bcf + row * kBCPitch + jg * 4) = make_float4(v[0], v[1], v[2], v[3]);
    }
    if constexpr (TRAP) {
        if (lane < TC) {
            float cb = 0.0f;
#pragma unroll
            for (int n = 0; n < kNState; ++n) cb = fmaf(rd(kNState + n, lane), rd(n, lane), cb);
            bcf[lane * kBCPitch + 32] = cb;
        }
    }
}

// per-channel constants, as f32x2 pairs for the packed per-step arithmetic
struct ChanConst {
    float a2_0;      // A[d, 0] * log2(e)
    float2 a2_0x2;   // (a2_0, a2_0)
    float2 Dx2;      // (D[d], D[d])
    float2 biasx2;   // (bias[d], bias[d])
    float cw[4];     // convolution taps (old to new), when the scan has a convolution in front
    float cb;        // convolution bias
};

// The convolution's input history of a lane at a segment start t0: the three
// raw inputs x[t0-3 .. t0-1], taken from x itself, from the stored state of
// the K-1 inputs before t = 0, or zero.
template <typename T>
__device__ __forceinline__ void conv_halo(const FwdParams &p, int64_t b, int64_t d, int64_t t0, float (&halo)[3]) {
    using AT = Act<T>;
    const int64_t chan = b * p.dim + d;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int64_t s = t0 - 3 + i;
        float v = 0.0f;
        if (s >= 0)
            v = AT::load(p.x, chan * p.seqlen + s);
        else if (p.conv_state && s >= -(p.conv_k - 1))
            v = AT::load(p.conv_state, chan * (p.conv_k - 1) + (p.conv_k - 1 + s));
        halo[i] = v;
    }
}

// ---- phase 1: per-step scalars of the chunk -----------------------------------
// For every step t of the chunk: dt = softplus(delta + bias) (or delta + bias),
// u = dt x and r = exp(dt A[d, 0]) (S4D) or dt (general A), stored as float2
// (u, r) in ur[t][lane].  The work is laid out stage by stage over all step
// pairs, so consecutive instructions are independent and the latency of each
// special-function op is covered by the other pairs' work.
// With CONV, x first becomes silu(conv(x)): the lane's raw row and the three
// inputs before it (halo, updated to this chunk's last three) give the
// convolution, whose output feeds u = dt x and, as the skip term D xc written
// to the g table, the post warp's output, both in float32.
//
// With TRAP (the exponential-trapezoidal rule), ur gets (s_t, r_t) and g gets
// g_t, where g_t = lam_t dt_t x_t weights the interval's end and
// s_t = g_{t-1} + (1 - lam_t) dt_t x_{t-1} its start.  The scan then carries
// h~_t = h_t - g_t B_t, for which h~_t = Abar_t (h~_{t-1} + s_t B_{t-1}): the
// same work per state as the Euler rule.  x_last and g_last hold the step
// before the chunk (updated to the chunk's last step).
template <typename T, bool S4D, bool CONV, bool TRAP = false>
__device__ __forceinline__ void chunk_prepass(uint8_t *stage, float2 *ur, int row,
                                              const ChanConst &cc, bool softplus, float (&halo)[3],
                                              float *garr = nullptr, float *x_last = nullptr,
                                              float *g_last = nullptr) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    constexpr int PP = AT::kPerPiece, TC = FwdSmem<T>::kTC, NP = TC / 2;
    constexpr int TB = FwdSmem<T>::kTileBytes;
    uint8_t *xr = stage + row * kRowBytes;
    uint4 xv[kPieces], dv[kPieces];
#pragma unroll
    for (int pc = 0; pc < kPieces; ++pc) {
        const int off = swz(row, pc) << 4;
        xv[pc] = *reinterpret_cast<const uint4 *>(xr + off);
        dv[pc] = *reinterpret_cast<const uint4 *>(xr + TB + off);
    }
    float XC[TC];  // the scan's x: the raw input, or the convolution's output
#pragma unroll
    for (int t = 0; t < TC; ++t) XC[t] = AT::piece(xv[t / PP], t % PP);
    if constexpr (CONV) {
        float raw[TC + 3];
#pragma unroll
        for (int i = 0; i < 3; ++i) raw[i] = halo[i];
#pragma unroll
        for (int t = 0; t < TC; ++t) raw[t + 3] = XC[t];
#pragma unroll
        for (int i = 0; i < 3; ++i) halo[i] = raw[TC + i];
#pragma unroll
        for (int t = 0; t < TC; ++t) {
            float acc = cc.cb;
#pragma unroll
            for (int k = 0; k < 4; ++k) acc = fmaf(cc.cw[k], raw[t + k], acc);
            XC[t] = kAccurate ? acc * (1.0f / (1.0f + expf(-acc))) : silu_fast(acc);
            garr[t * 32 + row] = cc.Dx2.x * XC[t];
        }
    }
    float2 V[NP], E[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int pc = (2 * k) / PP, i = (2 * k) % PP;
        V[k] = __fadd2_rn(make_float2(AT::piece(dv[pc], i), AT::piece(dv[pc], i + 1)), cc.biasx2);
    }
    if (softplus) {
        if constexpr (kAccurate) {
#pragma unroll
            for (int k = 0; k < NP; ++k) V[k] = make_float2(softplus_accurate(V[k].x), softplus_accurate(V[k].y));
        } else {
            // e = 2^(v log2 e) (exponent clamped so 1 + e stays finite), then
            // softplus_from_exp; max(., v) restores dt = v for large v
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                E[k] = __fmul2_rn(V[k], make_float2(kLog2e, kLog2e));
                E[k] = make_float2(fminf(E[k].x, 126.0f), fminf(E[k].y, 126.0f));
            }
#pragma unroll
            for (int k = 0; k < NP; ++k) E[k] = make_float2(ex2_approx(E[k].x), ex2_approx(E[k].y));
#pragma unroll
            for (int k = 0; k < NP; ++k)
                E[k] = make_float2(softplus_from_exp(E[k].x), softplus_from_exp(E[k].y));
#pragma unroll
            for (int k = 0; k < NP; ++k) V[k] = make_float2(fmaxf(E[k].x, V[k].x), fmaxf(E[k].y, V[k].y));
        }
    }
    // V holds dt; E becomes r (S4D) or dt
#pragma unroll
    for (int k = 0; k < NP; ++k) E[k] = S4D ? __fmul2_rn(V[k], cc.a2_0x2) : V[k];
    if constexpr (S4D) {
#pragma unroll
        for (int k = 0; k < NP; ++k) E[k] = make_float2(ex2_approx(E[k].x), ex2_approx(E[k].y));
    }
    if constexpr (TRAP) {
        const uint8_t *lr = stage + FwdSmem<T, true>::kLamOff + row * kRowBytes;
        uint4 lv[kPieces];
#pragma unroll
        for (int pc = 0; pc < kPieces; ++pc) lv[pc] = *reinterpret_cast<const uint4 *>(lr + (swz(row, pc) << 4));
        float xp = *x_last, gp = *g_last;
#pragma unroll
        for (int k = 0; k < NP; ++k) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = 2 * k + e;
                const float dt = e ? V[k].y : V[k].x;
                const float lam = AT::piece(lv[t / PP], t % PP);
                const float g = lam * dt * XC[t];
                const float sv = fmaf((1.0f - lam) * dt, xp, gp);
                ur[t * 32 + row] = make_float2(sv, e ? E[k].y : E[k].x);
                garr[t * 32 + row] = g;
                xp = XC[t];
                gp = g;
            }
        }
        *x_last = xp;
        *g_last = gp;
    } else {
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const float2 U = __fmul2_rn(V[k], make_float2(XC[2 * k], XC[2 * k + 1]));
            ur[(2 * k) * 32 + row] = make_float2(U.x, E[k].x);
            ur[(2 * k + 1) * 32 + row] = make_float2(U.y, E[k].y);
        }
    }
}

// The trapezoidal rule's history at a segment start t0 (one lane): the input
// x_{t0-1}, its end weight g_{t0-1} = lam dt x, and (lanes 0..15) B_{t0-1}[lane]
// into row 0 of the widened table; from x_prev and B_prev at t0 = 0.
template <typename T>
__device__ __forceinline__ void trap_history(const FwdParams &p, int64_t b, int64_t d, int64_t t0, int lane,
                                             const ChanConst &cc, float *bcf, float *x_last, float *g_last) {
    using AT = Act<T>;
    const int64_t chan = b * p.dim + d;
    const bool prev = p.x_prev && p.B_prev;
    if (t0 == 0) {
        *x_last = prev ? AT::load(p.x_prev, chan) : 0.0f;
        *g_last = 0.0f;
        if (lane < kNState) bcf[lane] = prev ? AT::load(p.B_prev, b * kNState + lane) : 0.0f;
        return;
    }
    const int64_t i = chan * p.seqlen + t0 - 1;
    const float xv = AT::load(p.x, i);
    float v = AT::load(p.delta, i) + cc.biasx2.x;
    if (p.softplus) v = AT::kBytes == 4 ? softplus_accurate(v) : softplus_fast(v);
    *x_last = xv;
    *g_last = AT::load(p.lam, i) * v * xv;
    if (lane < kNState) bcf[lane] = AT::load(p.B, (b * kNState + lane) * p.seqlen + t0 - 1);
}

// ---- phase 2: the recurrence ---------------------------------------------------
// Operands of one step, prepared one step ahead: a = Abar pairs, ub = u B
// pairs, c = C pairs.
struct StepOps {
    float2 a[8], ub[8], c[8];
    float gcb;  // TRAP: g_t (C_t . B_t), the readout of the interval's end term
};

// With TRAP, ur holds (s_t, r_t) and row t's B half holds B_{t-1}, so ub is
// s_t B_{t-1}; gcb comes from the g table and float 32 of the row.
template <bool S4D, bool READOUT = true, bool TRAP = false>
__device__ __forceinline__ void prepare_step(const float *bcf, const float2 *ur, int t, int row,
                                             const float (&a2)[kNState], StepOps &s, const float *garr = nullptr) {
    if constexpr (TRAP && READOUT) s.gcb = garr[t * 32 + row] * bcf[t * kBCPitch + 32];
    const float2 ut_rt = ur[t * 32 + row];
    const float4 *p = reinterpret_cast<const float4 *>(bcf + t * kBCPitch);
    const float2 U2 = make_float2(ut_rt.x, ut_rt.x);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 b4 = p[q];
        s.ub[2 * q] = __fmul2_rn(U2, make_float2(b4.x, b4.y));
        s.ub[2 * q + 1] = __fmul2_rn(U2, make_float2(b4.z, b4.w));
        if (READOUT) {
            const float4 c4 = p[4 + q];
            s.c[2 * q] = make_float2(c4.x, c4.y);
            s.c[2 * q + 1] = make_float2(c4.z, c4.w);
        }
    }
    const float Rt = ut_rt.y;
    if constexpr (S4D) {
        // Abar_n = r^(n+1): r^1..r^16 in pairs by a depth-4 tree
        const float r2 = Rt * Rt;
        const float r4 = r2 * r2;
        const float r8 = r4 * r4;
        s.a[0] = make_float2(Rt, r2);
        s.a[1] = __fmul2_rn(s.a[0], make_float2(r2, r2));
        s.a[2] = __fmul2_rn(s.a[0], make_float2(r4, r4));
        s.a[3] = __fmul2_rn(s.a[1], make_float2(r4, r4));
#pragma unroll
        for (int j = 0; j < 4; ++j) s.a[4 + j] = __fmul2_rn(s.a[j], make_float2(r8, r8));
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            s.a[j] = make_float2(ex2_approx(a2[2 * j] * Rt), ex2_approx(a2[2 * j + 1] * Rt));
    }
}

// The state update over the chunk's first `nvalid` steps, software-pipelined
// by hand: the operands of step t+1 are prepared while step t updates the
// state.  y_t = C_t . h_t (without the D skip and the gate) is stored densely
// as float `lane` of row t of ur, over (u, r) pairs the warp has already read.  Full chunks run a branch-free body (the preparation of the
// step after the chunk reads the spare table row); only the last, partial
// chunk of a sequence tests the step index.
// With TRAP the carried state is h~ (see chunk_prepass): h~ = Abar (h~ + s B_{t-1})
// and y = C . h~ + g (C . B).
template <bool S4D, bool FULL, bool TRAP, bool YS>
__device__ __forceinline__ void chunk_core(const float *bcf, const float2 *ur, uint8_t *stage, int row, int nvalid,
                                           const float (&a2)[kNState], float2 (&h)[8],
                                           const float *garr = nullptr) {
    StepOps nxt;
    prepare_step<S4D, true, TRAP>(bcf, ur, 0, row, a2, nxt, garr);
#pragma unroll 1
    for (int t0 = 0; t0 < nvalid; t0 += 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = t0 + i;
            if (!FULL && t >= nvalid) break;
            const StepOps cur = nxt;
            if (FULL || t + 1 < nvalid) prepare_step<S4D, true, TRAP>(bcf, ur, t + 1, row, a2, nxt, garr);
            float2 ya = make_float2(TRAP ? cur.gcb : 0.0f, 0.0f), yb = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if constexpr (TRAP)
                    h[j] = __fmul2_rn(cur.a[j], __fadd2_rn(h[j], cur.ub[j]));
                else
                    h[j] = __ffma2_rn(cur.a[j], h[j], cur.ub[j]);
                if (j & 1) yb = __ffma2_rn(cur.c[j], h[j], yb);
                else ya = __ffma2_rn(cur.c[j], h[j], ya);
            }
            const float2 ys = __fadd2_rn(ya, yb);
            y_row<YS>(stage, ur, t)[row] = ys.x + ys.y;  // dense: one wavefront
        }
    }
}

// The state update alone, without the readout (no C, no y), for a launch with
// no output: the backward entry's checkpoint pass.  With mid set, the state
// before the chunk's step kCkptSteps goes there as well.
template <bool S4D, bool FULL>
__device__ __forceinline__ void chunk_states(const float *bcf, const float2 *ur, int row, int nvalid,
                                             const float (&a2)[kNState], float2 (&h)[8], float4 *mid) {
    StepOps nxt;
    prepare_step<S4D, false>(bcf, ur, 0, row, a2, nxt);
#pragma unroll 1
    for (int t0 = 0; t0 < nvalid; t0 += 8) {
        if (t0 == kCkptSteps && mid) {
#pragma unroll
            for (int q = 0; q < 4; ++q) mid[q] = make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = t0 + i;
            if (!FULL && t >= nvalid) break;
            const StepOps cur = nxt;
            if (FULL || t + 1 < nvalid) prepare_step<S4D, false>(bcf, ur, t + 1, row, a2, nxt);
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = __ffma2_rn(cur.a[j], h[j], cur.ub[j]);
        }
    }
}

// The summary pass of the time-parallel schedule: the same state update, with
// the running product of the per-step decays P_n = prod_t Abar_{t,n} in place
// of the readout (so P carries the rounding of the decays the sequential scan
// applies).  No y is produced.
template <bool S4D, bool FULL, bool TRAP = false>
__device__ __forceinline__ void chunk_summary(const float *bcf, const float2 *ur, int row, int nvalid,
                                              const float (&a2)[kNState], float2 (&h)[8], float2 (&P)[8]) {
    StepOps nxt;
    prepare_step<S4D, false>(bcf, ur, 0, row, a2, nxt);
#pragma unroll 1
    for (int t0 = 0; t0 < nvalid; t0 += 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = t0 + i;
            if (!FULL && t >= nvalid) break;
            const StepOps cur = nxt;
            if (FULL || t + 1 < nvalid) prepare_step<S4D, false>(bcf, ur, t + 1, row, a2, nxt);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if constexpr (TRAP)
                    h[j] = __fmul2_rn(cur.a[j], __fadd2_rn(h[j], cur.ub[j]));
                else
                    h[j] = __ffma2_rn(cur.a[j], h[j], cur.ub[j]);
                P[j] = __fmul2_rn(cur.a[j], P[j]);
            }
        }
    }
}

// ---- phase 3: D skip, gate, output -----------------------------------------------
// out_t = (y_t + D x_t) silu(z_t), written over the lane's own x row of the
// stage (already consumed); stage by stage over step pairs as in phase 1.
// y_t is float `lane` of row t of the chunk's y (y_row).
// With CONV the skip term comes from the g table (D xc, float32) instead of D x.
template <typename T, bool CONV, bool YS>
__device__ __forceinline__ void chunk_postpass(uint8_t *stage, const float2 *ur, int row,
                                               const ChanConst &cc, bool has_z, const float *garr = nullptr) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    constexpr int PP = AT::kPerPiece, TC = FwdSmem<T>::kTC, NP = TC / 2;
    constexpr int TB = FwdSmem<T>::kTileBytes;
    uint8_t *xr = stage + row * kRowBytes;
    uint4 xv[kPieces], zv[kPieces];
#pragma unroll
    for (int pc = 0; pc < kPieces; ++pc) {
        const int off = swz(row, pc) << 4;
        xv[pc] = *reinterpret_cast<const uint4 *>(xr + off);
        zv[pc] = has_z ? *reinterpret_cast<const uint4 *>(xr + 2 * TB + off) : make_uint4(0, 0, 0, 0);
    }
    float2 O[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int pc = (2 * k) / PP, i = (2 * k) % PP;
        const float2 Y = make_float2(y_row<YS>(stage, ur, 2 * k)[row], y_row<YS>(stage, ur, 2 * k + 1)[row]);
        if constexpr (CONV)
            O[k] = __fadd2_rn(Y, make_float2(garr[(2 * k) * 32 + row], garr[(2 * k + 1) * 32 + row]));
        else
            O[k] = __ffma2_rn(make_float2(AT::piece(xv[pc], i), AT::piece(xv[pc], i + 1)), cc.Dx2, Y);
    }
    if (has_z) {
        float2 Z[NP], E[NP];
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const int pc = (2 * k) / PP, i = (2 * k) % PP;
            Z[k] = make_float2(AT::piece(zv[pc], i), AT::piece(zv[pc], i + 1));
        }
        if constexpr (kAccurate) {
#pragma unroll
            for (int k = 0; k < NP; ++k) O[k] = __fmul2_rn(O[k], make_float2(silu_accurate(Z[k].x), silu_accurate(Z[k].y)));
        } else {
            // silu(z) = z / (1 + 2^(-z log2 e))
#pragma unroll
            for (int k = 0; k < NP; ++k) E[k] = __fmul2_rn(Z[k], make_float2(-kLog2e, -kLog2e));
#pragma unroll
            for (int k = 0; k < NP; ++k) E[k] = make_float2(ex2_approx(E[k].x), ex2_approx(E[k].y));
#pragma unroll
            for (int k = 0; k < NP; ++k) E[k] = __fadd2_rn(E[k], make_float2(1.0f, 1.0f));
#pragma unroll
            for (int k = 0; k < NP; ++k) E[k] = make_float2(rcp_approx(E[k].x), rcp_approx(E[k].y));
#pragma unroll
            for (int k = 0; k < NP; ++k) O[k] = __fmul2_rn(O[k], __fmul2_rn(Z[k], E[k]));
        }
    }
#pragma unroll
    for (int pc = 0; pc < kPieces; ++pc) {
        uint4 pk;
        if constexpr (AT::kBytes == 2) {
            const int k = pc * (PP / 2);
            pk = make_uint4(pack_bf16x2(O[k].x, O[k].y), pack_bf16x2(O[k + 1].x, O[k + 1].y),
                            pack_bf16x2(O[k + 2].x, O[k + 2].y), pack_bf16x2(O[k + 3].x, O[k + 3].y));
        } else {
            const int k = pc * (PP / 2);
            pk = make_uint4(__float_as_uint(O[k].x), __float_as_uint(O[k].y), __float_as_uint(O[k + 1].x),
                            __float_as_uint(O[k + 1].y));
        }
        *reinterpret_cast<uint4 *>(xr + (swz(row, pc) << 4)) = pk;
    }
}

// ---- writing a chunk's outputs (staged in the x tile) element by element ------
// (the path without TMA, for rows that are not 16-byte aligned)
template <typename T>
__device__ __forceinline__ void store_chunk_sync(const FwdParams &p, const uint8_t *tile, int64_t b,
                                                 int64_t d0, int64_t t0, int lane) {
    using AT = Act<T>;
    using W = typename std::conditional<AT::kBytes == 2, uint16_t, uint32_t>::type;
    constexpr int PP = AT::kPerPiece, TC = FwdSmem<T>::kTC;
    const int64_t L = p.seqlen;
    W *base = static_cast<W *>(p.out);
    for (int row = 0; row < 32; ++row) {
        const int64_t d = d0 + row;
        if (d >= p.dim) break;
        for (int col = lane; col < TC; col += 32) {
            const int64_t t = t0 + col;
            if (t >= L) break;
            base[(b * p.dim + d) * L + t] = *reinterpret_cast<const W *>(
                tile + row * kRowBytes + (swz(row, col / PP) << 4) + (col % PP) * AT::kBytes);
        }
    }
}

// ---- work queue and carried state ----------------------------------------------
// The sequence of each 32-channel group is cut into segments of p.seg_steps
// steps (kSegSteps for the chained schedule).  An item is one (group, segment) pair; items are handed out in
// segment-major order through an atomic counter, so the work spreads evenly
// over the persistent workers whatever the number of groups.  A segment other
// than the first starts from the state its predecessor left in `carry` and
// published by setting flag[group] = segment index; the predecessor was taken
// from the queue earlier by a running worker, so the wait always ends.  Every
// wait is still bounded: past its limit the warp records an error and goes on.
constexpr int kSegSteps = 512;
constexpr uint32_t kSpinLimit = 1u << 24;   // flag polls (64 ns apart)
constexpr uint32_t kBarLimit = 1u << 20;    // mbarrier try_wait rounds

struct FwdScratch {
    uint32_t *counter;  // [4] next item: one queue per (pass, kernel instance S4D / general)
    uint32_t *error;    // non-zero: a bounded wait gave up (bit 0: segment flag, bit 1: mbarrier)
    uint32_t *general;  // non-zero: some group has A rows without the S4D structure
    uint32_t *flags;    // [groups]: segments of the group finished
    float *carry;       // [groups][32 lanes][16 states]
    float *summ;        // time-parallel schedule: [groups][segs][32 lanes][16 end states, 16 decay products]
    float *start;       // time-parallel schedule: [groups][segs][32 lanes][16 start states]
};

// bytes of scratch for `groups` groups (and, for the time-parallel schedule,
// `segs` segments per group); the first flag_bytes(...) bytes must be zero at launch
__host__ __device__ inline size_t fwd_scratch_flag_bytes(int64_t groups) {
    return (256 + 4 * static_cast<size_t>(groups) + 255) / 256 * 256;
}
__host__ __device__ inline size_t fwd_scratch_bytes(int64_t groups, int64_t segs = 0) {
    return fwd_scratch_flag_bytes(groups) + static_cast<size_t>(groups) * 32 * kNState * 4 +
           static_cast<size_t>(groups) * segs * 32 * 3 * kNState * 4;
}
__host__ __device__ inline FwdScratch fwd_scratch_view(void *base, int64_t groups, int64_t segs = 0) {
    uint8_t *b = static_cast<uint8_t *>(base);
    FwdScratch s;
    s.counter = reinterpret_cast<uint32_t *>(b);
    s.error = reinterpret_cast<uint32_t *>(b + 16);
    s.general = reinterpret_cast<uint32_t *>(b + 20);
    s.flags = reinterpret_cast<uint32_t *>(b + 256);
    s.carry = reinterpret_cast<float *>(b + fwd_scratch_flag_bytes(groups));
    s.summ = s.carry + static_cast<size_t>(groups) * 32 * kNState;
    s.start = s.summ + static_cast<size_t>(groups) * segs * 32 * 2 * kNState;
    return s;
}

// ---- mbarriers (shared memory), with bounded waits -------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}
// one arrival by one thread (a barrier initialised with count 1)
__device__ __forceinline__ void mbar_arrive1(uint64_t *bar) { mbar_arrive(bar); }
// Wait for the completion of the phase with the given parity.  Returns false
// when the wait gives up: after kBarLimit polls (the error word gets bit 1), or
// early, once another wait of the launch has given up (the error word is
// non-zero) -- its results are void, so the caller leaves its loop.  A caller
// that gives up never touches the chunk it waited for.
__device__ __forceinline__ bool mbar_try_parity(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *error) {
    const uint32_t addr = smem_u32(bar);
    for (uint32_t n = 0; n < kBarLimit; ++n) {
        if (mbar_try_parity(addr, parity)) return true;
        if ((n & 1023u) == 1023u && *reinterpret_cast<volatile uint32_t *>(error) != 0) return false;
    }
    atomicOr(error, 2u);
    return false;
}
// The same wait for a TMA load's completion before the CTA may exit: it does not
// stop early on the error word (a load must never be in flight when the CTA ends).
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity, uint32_t *error) {
    const uint32_t addr = smem_u32(bar);
    for (uint32_t n = 0; n < kBarLimit; ++n)
        if (mbar_try_parity(addr, parity)) return;
    atomicOr(error, 2u);
}

// One chunk of a worker's stream, as the helper hands it to the scan warp.
struct ChunkDesc {
    int64_t b, d0, t0, g, seg;
    int32_t nvalid;
    int32_t flags;  // kFirst: first chunk of its segment; kLast: last; kSeqEnd: segment ends the sequence; kStop
};
constexpr int32_t kFirst = 1, kLast = 2, kSeqEnd = 4, kStop = 8;

// Per-lane constants of a channel for the helper's passes.
__device__ __forceinline__ ChanConst chan_const(const FwdParams &p, int64_t dc) {
    ChanConst cc;
    const float a2 = p.A[dc * kNState] * kLog2e;
    const float Dd = p.D ? p.D[dc] : 0.0f;
    const float bias = p.delta_bias ? p.delta_bias[dc] : 0.0f;
    cc.a2_0 = a2;
    cc.a2_0x2 = make_float2(a2, a2);
    cc.Dx2 = make_float2(Dd, Dd);
    cc.biasx2 = make_float2(bias, bias);
    // taps padded to four at the old end: cw[k] multiplies x[t - 3 + k]
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int kk = k - (4 - p.conv_k);
        cc.cw[k] = (p.conv_k && kk >= 0) ? p.conv_w[dc * p.conv_k + kk] : 0.0f;
    }
    cc.cb = (p.conv_k && p.conv_bias) ? p.conv_bias[dc] : 0.0f;
    return cc;
}

// Whether all channels of the warp's group have S4D-structured A rows
// (A[d, n] == (n + 1) A[d, 0] exactly); lanes past the last channel agree.
__device__ __forceinline__ bool group_is_s4d(const FwdParams &p, int64_t d0, int lane) {
    const int64_t d = d0 + lane;
    bool ok = true;
    if (d < p.dim) {
        const float4 *ar = reinterpret_cast<const float4 *>(p.A + d * kNState);
        float a[kNState];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = ar[q];
            a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int n = 0; n < kNState; ++n) ok = ok && (a[n] == __fmul_rn(static_cast<float>(n + 1), a[0]));
    }
    return __all_sync(0xffffffffu, ok);
}

// The helper's walk through the queue: the next chunk of its stream.  The
// shape's counts are fixed at construction; item indices are below 2^31 (the
// host checks), so an item is split with 32-bit arithmetic.
template <typename T, bool S4D>
struct ChunkCursor {
    uint32_t tiles, groups, items;
    int64_t g = 0, seg = 0, b = 0, d0 = 0, t_begin = 0, t_next = 0, t_end = 0;
    bool open = false;

    __device__ __forceinline__ explicit ChunkCursor(const FwdParams &p) {
        tiles = static_cast<uint32_t>((p.dim + 31) / 32);
        groups = tiles * static_cast<uint32_t>(p.batch);
        items = groups * static_cast<uint32_t>((p.seqlen + p.seg_steps - 1) / p.seg_steps);
    }

    __device__ __forceinline__ ChunkDesc next(const FwdParams &p, const FwdScratch &sc, uint32_t *counter,
                                              int lane) {
        constexpr int TC = FwdSmem<T>::kTC;
        ChunkDesc dsc;
        while (!open || t_next >= t_end) {
            uint32_t item = 0;
            if (lane == 0) item = atomicAdd(counter, 1u);
            item = __shfl_sync(0xffffffffu, item, 0);
            if (item >= items) {
                dsc.flags = kStop;
                return dsc;
            }
            const uint32_t gi = item % groups;
            seg = item / groups;
            g = gi;
            b = gi / tiles;
            d0 = static_cast<int64_t>(gi % tiles) * 32;
            t_begin = seg * p.seg_steps;
            t_end = t_begin + p.seg_steps < p.seqlen ? t_begin + p.seg_steps : p.seqlen;
            t_next = t_begin;
            const bool s4d = group_is_s4d(p, d0, lane);
            if (s4d != S4D) {
                if (S4D && lane == 0) atomicOr(sc.general, 1u);
                open = false;
                continue;
            }
            open = true;
        }
        dsc.b = b; dsc.d0 = d0; dsc.t0 = t_next; dsc.g = g; dsc.seg = seg;
        dsc.nvalid = static_cast<int32_t>(t_end - t_next < TC ? t_end - t_next : TC);
        dsc.flags = (t_next == t_begin ? kFirst : 0) | (t_next + TC >= t_end ? kLast : 0) |
                    (t_end == p.seqlen ? kSeqEnd : 0);
        t_next += TC;
        return dsc;
    }
};

// ---- the kernel -----------------------------------------------------------------
// Persistent and warp-specialized.  grid: one CTA per SM; block: kPairs warp
// triples; warps w, w + 4 and w + 8 share an SM sub-partition and their own
// slice of shared memory.
//   prep (w + 4): takes items from the queue, stages chunks with TMA (or
//          element loads), widens B|C and computes the per-step scalars
//          (u, r); hands the chunk over (mbarrier ready).
//   scan (w):    the recurrence on (u, r) and B|C with the state in registers;
//          at segment boundaries it takes the state from h0 or the
//          predecessor's carry and leaves it in the carry or h_last (done).
//   post (w + 8): D skip, silu gate, bf16 pack and the TMA store of the
//          output tile (posted).
// The three instruction streams (MUFU-heavy, FMA-heavy, store) overlap on the
// sub-partition.  Two instances run back to back: the S4D one takes groups
// whose A rows are all S4D-structured and marks the scratch when it meets
// another group; the general one then takes those.
template <typename T, bool VEC, bool S4D, bool CONV, bool TRAP, bool STATES = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    scan_fwd_kernel(const FwdParams p, const FwdScratch sc, const __grid_constant__ TmaMaps tm) {
    static_assert(!STATES || (!CONV && !TRAP), "the states-only instance is the plain scan's");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // 1 KB alignment keeps every tile on a whole period of the 64-byte swizzle.  The
    // offset is added to the shared-memory pointer itself (no round trip through an
    // integer), so the compiler keeps the shared address space and emits ld/st.shared
    // rather than generic accesses, which cost twice the data-pipe passes on a
    // warp-uniform read.
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    using SM = FwdSmem<T, TRAP, CONV>;
    constexpr int TC = SM::kTC;
    constexpr int kStages = SM::kStages;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int pair = warp & (kPairs - 1);
    const int role = warp / kPairs;  // 0 scan, 1 prep, 2 post
    uint8_t *ps = smem + pair * SM::kPairBytes;
    uint64_t *ready = reinterpret_cast<uint64_t *>(ps + SM::kBarOff);
    // done[4]: the scan warp may finish up to kStages chunks ahead of the post warp
    // (the post warp issues the loads), so the barrier of chunk j is not reused
    // before the post warp has waited on it
    uint64_t *done = ready + 2;
    uint64_t *posted = ready + 6;
    uint64_t *full = ready + 8;  // [kStages]: TMA bytes of a staged chunk have landed
    ChunkDesc *ring = reinterpret_cast<ChunkDesc *>(ps + SM::kDescOff);
    auto stage_of = [&](int64_t j) { return ps + (j % kStages) * SM::kStageBytes; };
    auto bcf_of = [&](int64_t j) { return reinterpret_cast<float *>(ps + SM::kBCFOff + (j & 1) * SM::kBCFBytes); };
    auto ur_of = [&](int64_t j) { return reinterpret_cast<float2 *>(ps + SM::kUROff + (j & 1) * SM::kURBytes); };
    auto g_of = [&](int64_t j) { return reinterpret_cast<float *>(ps + SM::kGOff + (j & 1) * SM::kGBytes); };
    auto parity = [](int64_t j, int n) { return static_cast<uint32_t>((j / n) & 1); };

    uint64_t *dready = full + kStages;  // [4]: the descriptor of chunk j + kStages is in the ring
    uint32_t *load_count = reinterpret_cast<uint32_t *>(dready + 4);  // loads the post warp issued, plus one
    if (threadIdx.x < kPairs) {
        uint64_t *r = reinterpret_cast<uint64_t *>(smem + threadIdx.x * SM::kPairBytes + SM::kBarOff);
        for (int i = 0; i < 8; ++i) mbar_init(r + i, 32);
        for (int i = 0; i < kStages + 4; ++i) mbar_init(r + 8 + i, 1);
        *reinterpret_cast<uint32_t *>(r + 12 + kStages) = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    if (!S4D && *reinterpret_cast<volatile uint32_t *>(sc.general) == 0) return;
    uint32_t *counter = sc.counter + 2 * p.pass + (S4D ? 0 : 1);
    const uint32_t stage_tx = (p.z ? 3u : 2u) * SM::kTileBytes + 2u * kNState * kRowBytes +
                              (TRAP ? static_cast<uint32_t>(SM::kTileBytes) : 0u);
    // stage chunk j: TMA (one lane, completion on full[j % kStages]) or element loads
    auto load_stage = [&](const ChunkDesc &dsc, int64_t j) {
        if (dsc.flags & kStop) return;
        uint8_t *st = stage_of(j);
        if constexpr (VEC) {
            if (lane == 0) {
                uint64_t *bar = full + (j % kStages);
                mbar_arrive_expect_tx(bar, stage_tx);
                const int t0 = static_cast<int>(dsc.t0), d0 = static_cast<int>(dsc.d0), b = static_cast<int>(dsc.b);
                tma_load_3d(st, &tm.x, t0, d0, b, bar);
                tma_load_3d(st + SM::kTileBytes, &tm.delta, t0, d0, b, bar);
                if (p.z) tma_load_3d(st + 2 * SM::kTileBytes, &tm.z, t0, d0, b, bar);
                tma_load_3d(st + SM::kBCRawOff, &tm.B, t0, 0, b, bar);
                tma_load_3d(st + SM::kBCRawOff + kNState * kRowBytes, &tm.C, t0, 0, b, bar);
                if (TRAP) tma_load_3d(st + SM::kLamOff, &tm.lam, t0, d0, b, bar);
            }
        } else {
            load_chunk_sync<T, TRAP>(p, st, dsc.b, dsc.d0, dsc.t0, lane);
        }
    };
    // Who loads the stages.  Three stages with TMA: the post warp, into the stage
    // it has just posted (the prep warp keeps preparing).  Two stages: the prep
    // warp, right after it hands a chunk over (a load issued by the post warp
    // would land too late for the next chunk); element loads: the prep warp.
    constexpr bool kPrepLoads = !VEC || kStages == 2;
    // TMA loads the prep warp waited for and issued (for the drain at the end:
    // every issued load completes before the CTA exits)
    int64_t n_waited = 0, n_prep_issued = 0;

    if (role == 1) {
        // ------------------------------------------------------------------ prep
        // Buffer reuse.  Chunk j's u/r, B|C and g tables are chunk j - 2's: chunk j is
        // prepared once chunk j - 2's scan is done (and, when the prep warp loads the
        // stages or the convolution's post warp reads the g table, once chunk j - 2
        // is posted).  When the post warp loads, it loads chunk j + kStages into
        // chunk j's stage as soon as it has posted chunk j, and the prep warp puts
        // that chunk's descriptor in the ring kStages chunks ahead.
        ChunkCursor<T, S4D> cur(p);
        const bool softplus = p.softplus != 0;
        ChanConst cc;
        int64_t cc_d0 = -1;
        float halo[3] = {0.0f, 0.0f, 0.0f};  // convolution inputs before the chunk (CONV)
        float x_last = 0.0f, g_last = 0.0f;  // the step before the chunk (TRAP)
        bool stopped = false;
        auto next_desc = [&]() {
            ChunkDesc d;
            d.flags = kStop;
            if (!stopped) {
                d = cur.next(p, sc, counter, lane);
                stopped = (d.flags & kStop) != 0;
            }
            return d;
        };
        const int64_t ahead = kPrepLoads ? 1 : kStages;  // chunks loaded before the loop
        for (int64_t j = 0; j < ahead; ++j) {
            const ChunkDesc d = next_desc();
            if (lane == 0) ring[j & 7] = d;
            load_stage(d, j);
            if (!(d.flags & kStop)) n_prep_issued = j + 1;
        }
        __syncwarp();
        for (int64_t j = 0;; ++j) {
            const ChunkDesc dj = ring[j & 7];
            if (j >= 2) {
                if (!mbar_wait(done + ((j - 2) & 3), parity(j - 2, 4), sc.error)) break;
                if ((CONV || kPrepLoads) && !mbar_wait(posted + (j & 1), parity(j - 2, 2), sc.error)) break;
            }
            if constexpr (!kPrepLoads) {
                const ChunkDesc dn = next_desc();
                if (lane == 0) {
                    ring[(j + kStages) & 7] = dn;
                    mbar_arrive1(dready + (j & 3));
                }
            } else if (kStages == 3 && !(dj.flags & kStop)) {
                // the stage of chunk j + 1 is chunk j - 2's, posted above
                const ChunkDesc dn = next_desc();
                if (lane == 0) ring[(j + 1) & 7] = dn;
                load_stage(dn, j + 1);
                if (!(dn.flags & kStop)) n_prep_issued = j + 2;
            }
            if (!(dj.flags & kStop)) {
                if constexpr (VEC) {
                    if (!mbar_wait(full + (j % kStages), parity(j, kStages), sc.error)) break;
                    n_waited = j + 1;
                }
                __syncwarp();
                uint8_t *st = stage_of(j);
                widen_bc<T, TRAP>(st + SM::kBCRawOff, bcf_of(j), lane);
                if (dj.d0 != cc_d0) {  // the channel constants change only with the group
                    const int64_t d = dj.d0 + lane;
                    cc = chan_const(p, d < p.dim ? d : p.dim - 1);
                    cc_d0 = dj.d0;
                }
                if constexpr (TRAP) {
                    // row 0's B half: B of the step before the chunk
                    if (dj.flags & kFirst) {
                        const int64_t d = dj.d0 + lane;
                        trap_history<T>(p, dj.b, d < p.dim ? d : p.dim - 1, dj.t0, lane, cc, bcf_of(j), &x_last,
                                        &g_last);
                    } else if (lane < kNState) {
                        bcf_of(j)[lane] = bcf_of(j - 1)[TC * kBCPitch + lane];
                    }
                }
                if (CONV && (dj.flags & kFirst)) {
                    const int64_t d = dj.d0 + lane;
                    conv_halo<T>(p, dj.b, d < p.dim ? d : p.dim - 1, dj.t0, halo);
                }
        chunk_prepass<T, S4D, CONV, TRAP>(st, ur_of(j), lane, cc, softplus, halo, g_of(j), &x_last,
                                                  &g_last);
            }
            __syncwarp();
            mbar_arrive(ready + (j & 1));
            if (dj.flags & kStop) break;
            if (kPrepLoads && kStages == 2) {
                // the stage of chunk j + 1 is chunk j - 1's: load once it is posted
                if (j >= 1 && !mbar_wait(posted + ((j - 1) & 1), parity(j - 1, 2), sc.error)) break;
                const ChunkDesc dn = next_desc();
                if (lane == 0) ring[(j + 1) & 7] = dn;
                load_stage(dn, j + 1);
                if (!(dn.flags & kStop)) n_prep_issued = j + 2;
                __syncwarp();
            }
        }
    } else if (role == 2) {
        // ------------------------------------------------------------------ post
        const bool has_z = p.z != nullptr;
        ChanConst cc;
        int64_t cc_d0 = -1;
        uint32_t issued = 0;  // one past the last chunk this warp loaded
        for (int64_t j = 0;; ++j) {
            if (!mbar_wait(done + (j & 3), parity(j, 4), sc.error)) break;
            const ChunkDesc dj = ring[j & 7];
            if (dj.flags & kStop) break;
            uint8_t *st = stage_of(j);
            if (p.mode != kSummary && p.out) {  // the summary pass and a checkpoint pass write no output
                if (dj.d0 != cc_d0) {
                    const int64_t d = dj.d0 + lane;
                    cc = chan_const(p, d < p.dim ? d : p.dim - 1);
                    cc_d0 = dj.d0;
                }
                chunk_postpass<T, CONV, !kPrepLoads>(st, ur_of(j), lane, cc, has_z, g_of(j));
                if constexpr (VEC) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tm.out, static_cast<int>(dj.t0), static_cast<int>(dj.d0), static_cast<int>(dj.b),
                                     st);
                        tma_store_commit();
                        tma_store_wait_read();  // the stage is loaded again right after
                    }
                } else {
                    __syncwarp();
                    store_chunk_sync<T>(p, st, dj.b, dj.d0, dj.t0, lane);
                }
            }
            if constexpr (!kPrepLoads) {
                // chunk j's stage is free: load chunk j + kStages into it
                if (!mbar_wait(dready + (j & 3), parity(j, 4), sc.error)) break;
                const ChunkDesc dn = ring[(j + kStages) & 7];
                load_stage(dn, j + kStages);
                if (!(dn.flags & kStop)) issued = static_cast<uint32_t>(j + kStages + 1);
            }
            __syncwarp();
            mbar_arrive(posted + (j & 1));
        }
        if (VEC && lane == 0) {
            *load_count = issued;
            tma_store_wait_all();
        }
    } else {
        // ------------------------------------------------------------------ scan
        const int64_t segs = (p.seqlen + p.seg_steps - 1) / p.seg_steps;
        float2 h[8], P[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) h[j] = P[j] = make_float2(0.0f, 0.0f);
        float a2[kNState];
#pragma unroll
        for (int n = 0; n < kNState; ++n) a2[n] = 0.0f;
        for (int64_t k = 0;; ++k) {
            if (!mbar_wait(ready + (k & 1), parity(k, 2), sc.error)) break;
            const ChunkDesc dk = ring[k & 7];
            if (dk.flags & kStop) {
                mbar_arrive(done + (k & 3));  // lets the post warp see the end
                break;
            }
            const int64_t d = dk.d0 + lane;
            const bool active = d < p.dim;
            const int64_t gs = (dk.g * segs + dk.seg) * 32 + lane;  // (group, segment, lane) slot
            if (dk.flags & kFirst) {
                if (!S4D) {
                    const float *ar = p.A + (active ? d : p.dim - 1) * kNState;
#pragma unroll
                    for (int n = 0; n < kNState; ++n) a2[n] = ar[n] * kLog2e;
                }
                const float4 *src = nullptr;
                if (p.mode == kSummary) {
                    // every segment starts from zero; P starts as the identity
#pragma unroll
                    for (int j = 0; j < 8; ++j) P[j] = make_float2(1.0f, 1.0f);
                } else if (p.mode == kFromStart) {
                    // every segment, the first one included, starts from the state the
                    // combine kernel left; h0 is not read here, so h_last may alias it
                    src = reinterpret_cast<const float4 *>(sc.start + gs * kNState);
                } else if (dk.seg == 0) {
                    if (active && p.h0) src = reinterpret_cast<const float4 *>(p.h0 + (dk.b * p.dim + d) * kNState);
                } else {
                    const uint32_t want = static_cast<uint32_t>(dk.seg) + p.flag_bias;
                    uint32_t spins = 0;
                    while (ld_acquire(sc.flags + dk.g) < want) {
                        if (++spins > p.spin_limit) {
                            atomicOr(sc.error, 1u);
                            break;
                        }
                        __nanosleep(64);
                    }
                    src = reinterpret_cast<const float4 *>(sc.carry + (dk.g * 32 + lane) * kNState);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 v = src ? __ldcg(src + q) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    h[2 * q] = make_float2(v.x, v.y);
                    h[2 * q + 1] = make_float2(v.z, v.w);
                }
            }
            if (p.ckpt && p.mode != kSummary && active && dk.t0 % kCkptSteps == 0) {
                float4 *ck = reinterpret_cast<float4 *>(p.ckpt +
                                                        ((dk.b * p.dim + d) * p.ckpt_segs + dk.t0 / kCkptSteps) * kNState);
#pragma unroll
                for (int q = 0; q < 4; ++q) ck[q] = make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y);
            }
            if (p.mode == kSummary) {
                if (dk.nvalid == TC)
                    chunk_summary<S4D, true, TRAP>(bcf_of(k), ur_of(k), lane, TC, a2, h, P);
                else
                    chunk_summary<S4D, false, TRAP>(bcf_of(k), ur_of(k), lane, dk.nvalid, a2, h, P);
            } else if constexpr (STATES) {
                // no output: the states alone, and the checkpoint inside the chunk
                float4 *mid = nullptr;
                if (TC > kCkptSteps && p.ckpt && active)
                    mid = reinterpret_cast<float4 *>(
                        p.ckpt + ((dk.b * p.dim + d) * p.ckpt_segs + dk.t0 / kCkptSteps + 1) * kNState);
                if (dk.nvalid == TC)
                    chunk_states<S4D, true>(bcf_of(k), ur_of(k), lane, TC, a2, h, mid);
                else
                    chunk_states<S4D, false>(bcf_of(k), ur_of(k), lane, dk.nvalid, a2, h, mid);
            } else if (dk.nvalid == TC) {
                chunk_core<S4D, true, TRAP, !kPrepLoads>(bcf_of(k), ur_of(k), stage_of(k), lane, TC, a2, h, g_of(k));
            } else {
                chunk_core<S4D, false, TRAP, !kPrepLoads>(bcf_of(k), ur_of(k), stage_of(k), lane, dk.nvalid, a2, h,
                                                          g_of(k));
            }
            if (dk.flags & kLast) {
                if (p.mode == kSummary) {
                    // the segment's end state from zero and its decay product
                    float4 *sm = reinterpret_cast<float4 *>(sc.summ + gs * 2 * kNState);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        __stcg(sm + q, make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y));
                        __stcg(sm + 4 + q, make_float4(P[2 * q].x, P[2 * q].y, P[2 * q + 1].x, P[2 * q + 1].y));
                    }
                } else if (!(dk.flags & kSeqEnd)) {
                    if (p.mode == kChained) {
                        // hand the state to the next segment of this group
                        float4 *cr = reinterpret_cast<float4 *>(sc.carry + (dk.g * 32 + lane) * kNState);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            __stcg(cr + q, make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y));
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) st_release(sc.flags + dk.g, static_cast<uint32_t>(dk.seg + 1));
                    }
                } else if (active && p.h_last) {
                    float4 *hr = reinterpret_cast<float4 *>(p.h_last + (dk.b * p.dim + d) * kNState);
                    float2 hv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) hv[j] = h[j];
                    if constexpr (TRAP) {
                        // h = h~ + g B of the sequence's last step (row nvalid's B half holds B_{L-1})
                        const float g = g_of(k)[(dk.nvalid - 1) * 32 + lane];
                        const float *bl = bcf_of(k) + dk.nvalid * kBCPitch;
#pragma unroll
                        for (int j = 0; j < 8; ++j) hv[j] = __ffma2_rn(make_float2(g, g), make_float2(bl[2 * j], bl[2 * j + 1]), hv[j]);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        hr[q] = make_float4(hv[2 * q].x, hv[2 * q].y, hv[2 * q + 1].x, hv[2 * q + 1].y);
                }
            }
            __syncwarp();
            mbar_arrive(done + (k & 3));
        }
    }
    // every TMA load still in flight after a wait gave up completes before the CTA
    // exits (none on the normal path): the prep warp drains, in chunk order, the
    // loads it has not waited for
    if constexpr (VEC) {
        __syncthreads();
        if (role == 1 && lane == 0) {
            const int64_t issued = n_prep_issued > static_cast<int64_t>(*load_count) ? n_prep_issued : *load_count;
            for (int64_t j = n_waited; j < issued; ++j) mbar_drain(full + (j % kStages), parity(j, kStages), sc.error);
        }
    }
}

// Start states of every segment for the time-parallel schedule, from the
// summaries of the segments before it: h_0 = h0 (or 0), h_{s+1} = P_s h_s + e_s
// with e_s the end state of segment s run from zero and P_s its decay product
// (the splitting of the recurrence into chunks that continue from a carried
// state, applied to the carries themselves).  One thread per (group, lane).
__global__ void segment_combine_kernel(const FwdParams p, const FwdScratch sc) {
    const int64_t tiles = (p.dim + 31) / 32;
    const int64_t groups = tiles * p.batch;
    const int64_t segs = (p.seqlen + p.seg_steps - 1) / p.seg_steps;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t g = tid / 32;
    const int lane = static_cast<int>(tid % 32);
    if (g >= groups) return;
    const int64_t d = (g % tiles) * 32 + lane, b = g / tiles;
    float h[kNState];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (p.h0 && d < p.dim) v = reinterpret_cast<const float4 *>(p.h0 + (b * p.dim + d) * kNState)[q];
        h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
    }
    for (int64_t s = 0; s < segs; ++s) {
        const int64_t gs = (g * segs + s) * 32 + lane;
        float4 *st = reinterpret_cast<float4 *>(sc.start + gs * kNState);
#pragma unroll
        for (int q = 0; q < 4; ++q) st[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        if (s + 1 == segs) break;
        const float4 *sm = reinterpret_cast<const float4 *>(sc.summ + gs * 2 * kNState);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 e = sm[q], pr = sm[4 + q];
            h[4 * q] = fmaf(pr.x, h[4 * q], e.x);
            h[4 * q + 1] = fmaf(pr.y, h[4 * q + 1], e.y);
            h[4 * q + 2] = fmaf(pr.z, h[4 * q + 2], e.z);
            h[4 * q + 3] = fmaf(pr.w, h[4 * q + 3], e.w);
        }
    }
}

// The convolution state after a forward call: the last K-1 raw inputs of
// every channel, from x or (for sequences shorter than K-1) from the state
// before the call.  One thread per channel reads all its values before it
// writes, so the new state may overwrite the old one in place.
template <typename T>
__global__ void conv_state_kernel(const FwdParams p, void *state_out) {
    using AT = Act<T>;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= p.batch * p.dim) return;
    const int K1 = p.conv_k - 1;
    float v[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        v[j] = 0.0f;
        if (j >= K1) continue;
        const int64_t s = p.seqlen - K1 + j;
        if (s >= 0)
            v[j] = AT::load(p.x, c * p.seqlen + s);
        else if (p.conv_state)
            v[j] = AT::load(p.conv_state, c * K1 + (K1 + s));
    }
#pragma unroll
    for (int j = 0; j < 3; ++j)
        if (j < K1) AT::store(state_out, c * K1 + j, v[j]);
}

}  // namespace ssm
