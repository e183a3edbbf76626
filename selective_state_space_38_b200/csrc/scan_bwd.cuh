// scan_bwd.cuh -- backward pass of the selective scan (S6) for sm_100a.
//
// Gu & Dao, "Mamba", Appendix D "Hardware-aware Algorithm For Selective
// SSMs", paragraph "Memory": the backward pass does not keep the intermediate
// states; it recomputes them when the inputs are loaded into on-chip memory.
// Here a first kernel stores only the state at the start of every segment of
// kBwdSeg steps (a checkpoint, 64 B per channel and segment); the backward
// kernel walks each channel's segments from the last to the first, recomputes
// a segment's states 16 steps at a time into shared memory and runs the
// adjoint recurrence
//   g_t = C_t dy_t + Abar_{t+1} g_{t+1}
// backwards through them, carrying the decayed adjoint G = Abar_t g_t from
// step to step.
//
// Work layout: channels across lanes, as in the forward scan.  A warp owns 32
// consecutive channels of one sequence (lane = channel) and runs every step of
// them in order, so each recurrence is one sequential chain per lane with its
// 16 states in registers.  The sums over channels (dB, dC) are reduced across
// the warp's lanes with a transpose-reduce of warp shuffles (after it, lane k
// holds the warp's sum of value k) and added to the outputs with float
// atomics, four steps per atomic.  Sums over time (dA, dD, dbias) stay in the
// lane's registers until the end and are added with float atomics.
#pragma once

#include "common.cuh"

namespace ssm {

constexpr int kBwdSeg = 32;   // steps between checkpoints
constexpr int kBwdSub = 16;   // steps recomputed and run backwards at a time

struct BwdParams {
    const void *x, *delta, *z, *B, *C, *dout;
    const float *delta_bias, *A, *D, *h0, *dh_last;
    void *dx, *ddelta, *dz;          // [batch][dim][L], activation dtype (dz when z is given)
    float *dA, *dD, *dbias, *dh0;    // summed with atomics (zeroed by the host) / written
    float *ckpt;                     // [batch][dim][segments][16] states at segment starts
    float *dB, *dC;                  // [batch][16][L], summed with atomics (zeroed by the host)
    int64_t batch, seqlen, dim;
    int softplus;
};

__host__ __device__ inline int64_t bwd_segments(int64_t L) { return (L + kBwdSeg - 1) / kBwdSeg; }
__host__ __device__ inline int64_t bwd_groups(int64_t batch, int64_t dim) { return batch * ((dim + 31) / 32); }

template <typename T>
__device__ __forceinline__ float bwd_softplus(float v) {
    return Act<T>::kBytes == 4 ? softplus_accurate(v) : softplus_fast(v);
}

// exp(A[d, n] dt) for the 16 states.  all_s4d (warp-uniform): every lane's row
// has the S4D-real structure A[d, n] = (n + 1) A[d, 0], and the decays are the
// powers of r = exp(A[d, 0] dt) (one MUFU op and a multiplication tree);
// otherwise sixteen MUFU ops.
__device__ __forceinline__ void bwd_decay(const float (&a2)[kNState], bool all_s4d, float dt,
                                          float (&out)[kNState]) {
    if (all_s4d) {
        const float r = ex2_approx(a2[0] * dt);
        const float r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
        out[0] = r; out[1] = r2; out[2] = r2 * r; out[3] = r4;
#pragma unroll
        for (int n = 4; n < 8; ++n) out[n] = out[n - 4] * r4;
#pragma unroll
        for (int n = 8; n < 16; ++n) out[n] = out[n - 8] * r8;
    } else {
#pragma unroll
        for (int n = 0; n < kNState; ++n) out[n] = ex2_approx(a2[n] * dt);
    }
}

// Whether A[d, :] has the S4D-real structure A[d, n] = (n + 1) A[d, 0] exactly.
__device__ __forceinline__ bool bwd_row_is_s4d(const float *Arow) {
    bool ok = true;
#pragma unroll
    for (int n = 0; n < kNState; ++n) ok = ok && (Arow[n] == __fmul_rn(static_cast<float>(n + 1), Arow[0]));
    return ok;
}

// Sixteen consecutive activations of one channel row, t0 .. t0 + 15 (zero past
// L), widened to float: 16-byte loads when the row and t0 allow them.
template <typename T>
__device__ __forceinline__ void bwd_load16(const void *base, int64_t row_off, int64_t t0, int64_t L, bool vec,
                                           float (&v)[kBwdSub]) {
    using AT = Act<T>;
    if (vec && t0 + kBwdSub <= L) {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(base) +
                                                         (row_off + t0) * AT::kBytes);
#pragma unroll
        for (int q = 0; q < kBwdSub / AT::kPerPiece; ++q) {
            const uint4 w = __ldg(p + q);
#pragma unroll
            for (int i = 0; i < AT::kPerPiece; ++i) v[q * AT::kPerPiece + i] = AT::piece(w, i);
        }
    } else {
#pragma unroll
        for (int k = 0; k < kBwdSub; ++k) v[k] = t0 + k < L ? AT::load(base, row_off + t0 + k) : 0.0f;
    }
}

// Sixteen values to one channel row, t0 .. t0 + 15 (only those below L).
template <typename T>
__device__ __forceinline__ void bwd_store16(void *base, int64_t row_off, int64_t t0, int64_t L, bool vec,
                                            const float (&v)[kBwdSub]) {
    using AT = Act<T>;
    if (vec && t0 + kBwdSub <= L) {
        uint4 *p = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(base) + (row_off + t0) * AT::kBytes);
        if constexpr (AT::kBytes == 2) {
#pragma unroll
            for (int q = 0; q < 2; ++q)
                p[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                  pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                p[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                  __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
        }
    } else {
#pragma unroll
        for (int k = 0; k < kBwdSub; ++k)
            if (t0 + k < L) AT::store(base, row_off + t0 + k, v[k]);
    }
}

// Warp transpose-reduce: every lane holds 32 values; afterwards lane k holds
// the sum over the warp's lanes of value k.  Five butterfly levels; at the
// level of mask m a lane keeps the half of its values selected by (lane & m)
// and receives the partner's copy of that half.
__device__ __forceinline__ float warp_transpose_sum32(const float (&v)[32], int lane) {
    float w16[16], w8[8], w4[4], w2[2];
    {
        const bool up = lane & 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float send = up ? v[i] : v[i + 16], keep = up ? v[i + 16] : v[i];
            w16[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
    }
    {
        const bool up = lane & 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float send = up ? w16[i] : w16[i + 8], keep = up ? w16[i + 8] : w16[i];
            w8[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    {
        const bool up = lane & 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = up ? w8[i] : w8[i + 4], keep = up ? w8[i + 4] : w8[i];
            w4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
    }
    {
        const bool up = lane & 2;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = up ? w4[i] : w4[i + 2], keep = up ? w4[i + 2] : w4[i];
            w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        }
    }
    const bool up = lane & 1;
    const float send = up ? w2[0] : w2[1], keep = up ? w2[1] : w2[0];
    return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

// B (n < 16) and C (16 <= n < 32) of a sub-chunk's steps, widened: row k holds
// the 32 values of step t0 + k (zero past L).  Lane j loads row j of B or C.
template <typename T>
__device__ __forceinline__ void bwd_stage_bc(const BwdParams &p, int64_t b, int64_t t0, bool vec, int lane,
                                             float *bc) {
    float v[kBwdSub];
    const void *src = lane < kNState ? p.B : p.C;
    bwd_load16<T>(src, (b * kNState + (lane & (kNState - 1))) * p.seqlen, t0, p.seqlen, vec, v);
#pragma unroll
    for (int k = 0; k < kBwdSub; ++k) bc[k * 32 + lane] = v[k];
}

// B and C of step k from the staged rows (warp-uniform 16-byte reads)
__device__ __forceinline__ void bwd_bc_row(const float *bc, int k, float (&Bv)[kNState], float (&Cv)[kNState]) {
    const float4 *r = reinterpret_cast<const float4 *>(bc + k * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 b = r[q], c = r[4 + q];
        Bv[4 * q] = b.x; Bv[4 * q + 1] = b.y; Bv[4 * q + 2] = b.z; Bv[4 * q + 3] = b.w;
        Cv[4 * q] = c.x; Cv[4 * q + 1] = c.y; Cv[4 * q + 2] = c.z; Cv[4 * q + 3] = c.w;
    }
}

// One step of the forward recurrence: h = exp(A dt) h + dt x B.
__device__ __forceinline__ void bwd_fwd_step(float (&h)[kNState], const float (&a2)[kNState], bool all_s4d,
                                             float dt, float x, const float *bc, int k) {
    float a[kNState], Bv[kNState], Cv[kNState];
    bwd_decay(a2, all_s4d, dt, a);
    bwd_bc_row(bc, k, Bv, Cv);
    const float u = dt * x;
#pragma unroll
    for (int n = 0; n < kNState; ++n) h[n] = fmaf(a[n], h[n], u * Bv[n]);
}

// Per-lane constants of a channel: A row (and A log2 e), S4D structure, bias, D.
struct BwdChan {
    float a2[kNState], An[kNState];
    bool all_s4d;
    float bias, Dd;
};
__device__ __forceinline__ BwdChan bwd_chan(const BwdParams &p, int64_t dc) {
    BwdChan c;
    const float4 *ar = reinterpret_cast<const float4 *>(p.A + dc * kNState);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 v = __ldg(ar + q);
        c.An[4 * q] = v.x; c.An[4 * q + 1] = v.y; c.An[4 * q + 2] = v.z; c.An[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int n = 0; n < kNState; ++n) c.a2[n] = c.An[n] * kLog2e;
    c.all_s4d = __all_sync(0xffffffffu, bwd_row_is_s4d(c.An));
    c.bias = p.delta_bias ? p.delta_bias[dc] : 0.0f;
    c.Dd = p.D ? p.D[dc] : 0.0f;
    return c;
}

// ---- checkpoints: the state at the start of every segment -------------------------
// One warp per group of 32 channels of one sequence (four groups per CTA, each
// on its own); the forward recurrence over the whole sequence, with the state
// written at every segment start.
template <typename T>
__global__ void __launch_bounds__(128) scan_bwd_ckpt_kernel(const BwdParams p) {
    __shared__ __align__(16) float bc_all[4][kBwdSub * 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t grp = static_cast<int64_t>(blockIdx.x) * 4 + warp;
    if (grp >= bwd_groups(p.batch, p.dim)) return;  // warp-uniform
    const int64_t tiles = (p.dim + 31) / 32;
    const int64_t b = grp / tiles, d = (grp % tiles) * 32 + lane;
    const bool active = d < p.dim;
    const int64_t dc = active ? d : p.dim - 1;
    const int64_t chan = b * p.dim + dc, L = p.seqlen, segs = bwd_segments(L);
    const bool vec = (L * Act<T>::kBytes) % 16 == 0;
    const BwdChan cc = bwd_chan(p, dc);
    float *bc = bc_all[warp];
    float h[kNState];
    if (p.h0) {
        const float4 *src = reinterpret_cast<const float4 *>(p.h0 + chan * kNState);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = __ldg(src + q);
            h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int n = 0; n < kNState; ++n) h[n] = 0.0f;
    }
    for (int64_t t0 = 0; t0 < L; t0 += kBwdSub) {
        if (t0 % kBwdSeg == 0 && active) {
            float4 *dst = reinterpret_cast<float4 *>(p.ckpt + (chan * segs + t0 / kBwdSeg) * kNState);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
        float xv[kBwdSub], dv[kBwdSub];
        bwd_load16<T>(p.x, chan * L, t0, L, vec, xv);
        bwd_load16<T>(p.delta, chan * L, t0, L, vec, dv);
        __syncwarp();  // the previous sub-chunk's reads of bc are done
        bwd_stage_bc<T>(p, b, t0, vec, lane, bc);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < kBwdSub; ++k) {
            if (t0 + k >= L) break;  // warp-uniform
            const float v = dv[k] + cc.bias;
            const float dt = p.softplus ? bwd_softplus<T>(v) : v;
            bwd_fwd_step(h, cc.a2, cc.all_s4d, dt, xv[k], bc, k);
        }
    }
}

// Shared memory of a backward warp (dynamic, 44 KB).
struct BwdSmem {
    float hs[kBwdSub + 1][4][32][4];  // h_{t0-1} .. h_{t0+15} of the sub-chunk, per quarter and lane
    float bc[kBwdSub * 32];           // B|C of the sub-chunk's steps
    float io[4][kBwdSub][32];         // x, delta, z, dout per step and lane; then dx, ddelta, dz and
                                      // this lane's dB|dC sum in their places
};

__device__ __forceinline__ void bwd_put_state(BwdSmem &sm, int k, int lane, const float (&h)[kNState]) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4 *>(sm.hs[k][q][lane]) = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
}
__device__ __forceinline__ void bwd_get_state(const BwdSmem &sm, int k, int lane, float (&h)[kNState]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4 *>(sm.hs[k][q][lane]);
        h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
    }
}

// The lane's per-step scalars of step k of the staged sub-chunk.
struct BwdStep {
    float x, dt, sg, z, go;
};
template <typename T>
__device__ __forceinline__ BwdStep bwd_step_in(const BwdParams &p, const BwdSmem &sm, const BwdChan &cc, int k,
                                               int lane) {
    BwdStep s;
    s.x = sm.io[0][k][lane];
    const float v = sm.io[1][k][lane] + cc.bias;
    s.dt = p.softplus ? bwd_softplus<T>(v) : v;
    s.sg = p.softplus ? 1.0f / (1.0f + __expf(-v)) : 1.0f;  // d dt / d v
    s.z = sm.io[2][k][lane];
    s.go = sm.io[3][k][lane];
    return s;
}

// ---- the backward pass over one group of 32 channels of one sequence -------------
// grid: one warp (CTA) per group.
template <typename T>
__global__ void __launch_bounds__(32) scan_bwd_kernel(const BwdParams p) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    extern __shared__ __align__(16) uint8_t bwd_smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(bwd_smem_raw);
    const int lane = threadIdx.x;
    const int64_t tiles = (p.dim + 31) / 32;
    const int64_t b = blockIdx.x / tiles, d = (blockIdx.x % tiles) * 32 + lane;
    const bool active = d < p.dim;
    const float act = active ? 1.0f : 0.0f;
    const int64_t dc = active ? d : p.dim - 1;
    const int64_t chan = b * p.dim + dc, L = p.seqlen, segs = bwd_segments(L), row = chan * L;
    const bool vec = (L * AT::kBytes) % 16 == 0;
    const BwdChan cc = bwd_chan(p, dc);

    float G[kNState], dA[kNState];  // decayed adjoint entering the current step from the right; dA sum
#pragma unroll
    for (int n = 0; n < kNState; ++n) {
        G[n] = p.dh_last ? p.dh_last[chan * kNState + n] : 0.0f;
        dA[n] = 0.0f;
    }
    float dDs = 0.0f, dbs = 0.0f;

    // stage the inputs and B|C of the sub-chunk starting at t0 (all four inputs,
    // or only x and delta for a pass that recomputes states)
    auto stage = [&](int64_t t0, bool all) {
        __syncwarp();  // the previous users of io and bc are done
        float v[kBwdSub];
        bwd_load16<T>(p.x, row, t0, L, vec, v);
#pragma unroll
        for (int k = 0; k < kBwdSub; ++k) sm.io[0][k][lane] = v[k];
        bwd_load16<T>(p.delta, row, t0, L, vec, v);
#pragma unroll
        for (int k = 0; k < kBwdSub; ++k) sm.io[1][k][lane] = v[k];
        if (all) {
            if (p.z) {
                bwd_load16<T>(p.z, row, t0, L, vec, v);
#pragma unroll
                for (int k = 0; k < kBwdSub; ++k) sm.io[2][k][lane] = v[k];
            }
            bwd_load16<T>(p.dout, row, t0, L, vec, v);
#pragma unroll
            for (int k = 0; k < kBwdSub; ++k) sm.io[3][k][lane] = v[k];
        }
        bwd_stage_bc<T>(p, b, t0, vec, lane, sm.bc);
        __syncwarp();
    };
    // the forward recurrence over the staged sub-chunk from h (steps below L);
    // with keep, the states before and after every step go to sm.hs
    auto forward = [&](int64_t t0, float (&h)[kNState], bool keep) {
        if (keep) bwd_put_state(sm, 0, lane, h);
#pragma unroll
        for (int k = 0; k < kBwdSub; ++k) {
            if (t0 + k < L) {  // warp-uniform
                const float v = sm.io[1][k][lane] + cc.bias;
                const float dt = p.softplus ? bwd_softplus<T>(v) : v;
                bwd_fwd_step(h, cc.a2, cc.all_s4d, dt, sm.io[0][k][lane], sm.bc, k);
            }
            if (keep) bwd_put_state(sm, k + 1, lane, h);
        }
        __syncwarp();
    };
    // the adjoint over the staged sub-chunk, its steps from the last to the first,
    // with the states in sm.hs; then its outputs
    auto backward = [&](int64_t t0) {
#pragma unroll 1
        for (int k = kBwdSub - 1; k >= 0; --k) {
            if (t0 + k >= L) continue;  // warp-uniform
            const BwdStep s = bwd_step_in<T>(p, sm, cc, k, lane);
            float a[kNState], Bv[kNState], Cv[kNState], hn[kNState];
            bwd_decay(cc.a2, cc.all_s4d, s.dt, a);
            bwd_bc_row(sm.bc, k, Bv, Cv);
            bwd_get_state(sm, k + 1, lane, hn);  // h_t
            float y = cc.Dd * s.x;
#pragma unroll
            for (int n = 0; n < kNState; ++n) y = fmaf(Cv[n], hn[n], y);
            float dy = s.go, dzv = 0.0f;
            if (p.z) {
                const float sz = kAccurate ? 1.0f / (1.0f + expf(-s.z)) : rcp_approx(1.0f + ex2_approx(-s.z * kLog2e));
                dy = s.go * s.z * sz;
                dzv = s.go * y * sz * fmaf(s.z, 1.0f - sz, 1.0f);
            }
            float vals[32];  // this lane's dB (n < 16) and dC (n >= 16) terms of the step
            float g[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                g[n] = fmaf(Cv[n], dy, G[n]);
                vals[kNState + n] = act * dy * hn[n];
            }
            float hp[kNState];
            bwd_get_state(sm, k, lane, hp);  // h_{t-1}
            const float dtx = s.dt * s.x;
            float dxs = 0.0f, ddt = 0.0f;
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                vals[n] = act * g[n] * dtx;
                dxs = fmaf(g[n], Bv[n], dxs);
                const float ah = a[n] * hp[n];
                ddt = fmaf(g[n], fmaf(cc.An[n], ah, Bv[n] * s.x), ddt);
                dA[n] = fmaf(g[n] * s.dt, ah, dA[n]);
                G[n] = a[n] * g[n];
            }
            const float dd = ddt * s.sg;
            dDs = fmaf(dy, s.x, dDs);
            dbs += dd;
            sm.io[0][k][lane] = fmaf(cc.Dd, dy, s.dt * dxs);  // dx
            sm.io[1][k][lane] = dd;                            // ddelta
            sm.io[2][k][lane] = dzv;                           // dz
            sm.io[3][k][lane] = warp_transpose_sum32(vals, lane);
        }
        __syncwarp();
        float o[kBwdSub];
        if (active) {
#pragma unroll
            for (int k = 0; k < kBwdSub; ++k) o[k] = sm.io[0][k][lane];
            bwd_store16<T>(p.dx, row, t0, L, vec, o);
#pragma unroll
            for (int k = 0; k < kBwdSub; ++k) o[k] = sm.io[1][k][lane];
            bwd_store16<T>(p.ddelta, row, t0, L, vec, o);
            if (p.z) {
#pragma unroll
                for (int k = 0; k < kBwdSub; ++k) o[k] = sm.io[2][k][lane];
                bwd_store16<T>(p.dz, row, t0, L, vec, o);
            }
        }
        // the warp's dB (lanes 0..15) and dC (lanes 16..31) of the sub-chunk's steps
        float *dst = (lane < kNState ? p.dB : p.dC) + (b * kNState + (lane & (kNState - 1))) * L + t0;
        if (L % 4 == 0 && t0 + kBwdSub <= L) {
#pragma unroll
            for (int q = 0; q < kBwdSub / 4; ++q)
                atomicAdd(reinterpret_cast<float4 *>(dst) + q,
                          make_float4(sm.io[3][4 * q][lane], sm.io[3][4 * q + 1][lane], sm.io[3][4 * q + 2][lane],
                                      sm.io[3][4 * q + 3][lane]));
        } else {
            for (int k = 0; k < kBwdSub; ++k)
                if (t0 + k < L) atomicAdd(dst + k, sm.io[3][k][lane]);
        }
    };

    for (int64_t s = segs - 1; s >= 0; --s) {
        const int64_t ts = s * kBwdSeg;
        float hck[kNState], h[kNState];
        {
            const float4 *src = reinterpret_cast<const float4 *>(p.ckpt + (chan * segs + s) * kNState);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = src[q];
                hck[4 * q] = v.x; hck[4 * q + 1] = v.y; hck[4 * q + 2] = v.z; hck[4 * q + 3] = v.w;
            }
        }
        if (ts + kBwdSub < L) {
            // the segment's second sub-chunk: its start state from the first, then back through it
#pragma unroll
            for (int n = 0; n < kNState; ++n) h[n] = hck[n];
            stage(ts, false);
            forward(ts, h, false);
            stage(ts + kBwdSub, true);
            forward(ts + kBwdSub, h, true);
            backward(ts + kBwdSub);
        }
#pragma unroll
        for (int n = 0; n < kNState; ++n) h[n] = hck[n];
        stage(ts, true);
        forward(ts, h, true);
        backward(ts);
    }
    // dh0 = Abar_0 g_0, the adjoint carried out of the first step; sums over time
    if (active) {
        if (p.dh0) {
#pragma unroll
            for (int n = 0; n < kNState; ++n) p.dh0[chan * kNState + n] = G[n];
        }
#pragma unroll
        for (int n = 0; n < kNState; ++n) atomicAdd(p.dA + dc * kNState + n, dA[n]);
        if (p.dD) atomicAdd(p.dD + dc, dDs);
        if (p.dbias) atomicAdd(p.dbias + dc, dbs);
    }
}

}  // namespace ssm
