// scan_fwd_lat.cuh -- forward scan with lanes across time, for shapes with few
// channels and long sequences.
//
// "A Secret Weapon For mamba paper": the selective recurrence is not time-
// invariant but can still be parallelized with a work-efficient parallel scan;
// Gu & Dao, Appendix D "Speed": the sequence is split into chunks and each
// chunk continues from the carried state.  Here a warp owns one channel; lane
// i owns kLatK consecutive steps of a chunk of 32 kLatK steps.  Each lane folds
// its steps into an affine map h -> exp(A s) h + e (s = sum of dt, e = the
// steps' effect from a zero state); an exclusive warp-shuffle scan of those
// maps, applied to the carried state, gives every lane the state before its
// first step; the lane then reruns its steps for the readout.  The chunk's last
// state (lane 31) is carried to the next chunk.
//
// The warp's 32 lanes each need B and C of their own steps: a CTA of
// kLatWarps warps (channels of one sequence) stages the chunk's B|C once in
// shared memory, widened to float32 in lane-major slots (conflict-free
// 16-byte reads).  x, delta, z and out move as per-lane vectors straight
// between registers and global memory (coalesced over the warp).
#pragma once

#include "common.cuh"
#include "scan_bwd.cuh"  // decay16, row_is_s4d, bwd_row
#include "scan_fwd.cuh"  // FwdParams

namespace ssm {

constexpr int kLatK = 4;                     // steps per lane
constexpr int kLatChunk = 32 * kLatK;        // steps per chunk
constexpr int kLatWarps = 4;                 // channels per CTA

__device__ __forceinline__ int lat_slot(int t) { return (t % kLatK) * 32 + t / kLatK; }

// grid: ceil(dim / kLatWarps) x batch; block: kLatWarps warps.
template <typename T>
__global__ void __launch_bounds__(kLatWarps * 32) scan_fwd_lat_kernel(const FwdParams p) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    __shared__ __align__(16) float bcf[kLatChunk * kBwdPitch];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t b = blockIdx.y, L = p.seqlen;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * kLatWarps + warp;
    const bool active = d < p.dim;  // warp-uniform; inactive warps still stage B|C
    const int64_t dc = active ? d : p.dim - 1;
    const int64_t chan = b * p.dim + dc;
    float a2[kNState];
#pragma unroll
    for (int n = 0; n < kNState; ++n) a2[n] = p.A[dc * kNState + n] * kLog2e;
    const bool s4d = row_is_s4d(p.A + dc * kNState);
    const float bias = p.delta_bias ? p.delta_bias[dc] : 0.0f;
    const float Dd = p.D ? p.D[dc] : 0.0f;
    float hc[kNState];  // the carried state (the same in every lane)
#pragma unroll
    for (int n = 0; n < kNState; ++n) hc[n] = (p.h0 && active) ? p.h0[chan * kNState + n] : 0.0f;

    const int64_t chunks = (L + kLatChunk - 1) / kLatChunk;
    for (int64_t c = 0; c < chunks; ++c) {
        const int64_t t0 = c * kLatChunk;
        __syncthreads();
        for (int i = threadIdx.x; i < kLatChunk * 2 * kNState; i += blockDim.x) {
            const int t = i % kLatChunk, jn = i / kLatChunk;
            const int64_t tt = t0 + t;
            const float v = tt < L ? AT::load(jn < kNState ? p.B : p.C, (b * kNState + (jn % kNState)) * L + tt) : 0.0f;
            bcf[lat_slot(t) * kBwdPitch + jn] = v;
        }
        __syncthreads();
        if (!active) continue;

        float dts[kLatK], xs[kLatK];
        bool ok[kLatK];
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < kLatK; ++j) {
            const int64_t t = t0 + lane * kLatK + j;
            ok[j] = t < L;
            const float v = ok[j] ? AT::load(p.delta, chan * L + t) + bias : 0.0f;
            const float dt = ok[j] ? (p.softplus ? (kAccurate ? softplus_accurate(v) : softplus_fast(v)) : v) : 0.0f;
            dts[j] = dt;
            xs[j] = ok[j] ? AT::load(p.x, chan * L + t) : 0.0f;
            s += dt;
        }
        // fold the lane's steps from zero
        float e[kNState];
#pragma unroll
        for (int n = 0; n < kNState; ++n) e[n] = 0.0f;
#pragma unroll
        for (int j = 0; j < kLatK; ++j) {
            float a[kNState], Bv[kNState], Cv[kNState];
            decay16(a2, s4d, dts[j], a);
            bwd_row(bcf + (j * 32 + lane) * kBwdPitch, Bv, Cv);
            const float u = dts[j] * xs[j];
#pragma unroll
            for (int n = 0; n < kNState; ++n) e[n] = fmaf(a[n], e[n], u * Bv[n]);
        }
        // inclusive scan of the lanes' maps: (s', e') then (s, e) = (s' + s, exp(A s) e' + e)
        float si = s;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float so = __shfl_up_sync(0xffffffffu, si, off);
            float eo[kNState], P[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) eo[n] = __shfl_up_sync(0xffffffffu, e[n], off);
            if (lane >= off) {
                decay16(a2, s4d, si, P);
#pragma unroll
                for (int n = 0; n < kNState; ++n) e[n] = fmaf(P[n], eo[n], e[n]);
                si += so;
            }
        }
        // the state before this lane's first step: the maps of the lanes before it
        float h[kNState];
        {
            const float sx = __shfl_up_sync(0xffffffffu, si, 1);
            float ex[kNState], P[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                const float v = __shfl_up_sync(0xffffffffu, e[n], 1);
                ex[n] = lane ? v : 0.0f;
            }
            decay16(a2, s4d, lane ? sx : 0.0f, P);
#pragma unroll
            for (int n = 0; n < kNState; ++n) h[n] = fmaf(P[n], hc[n], ex[n]);
        }
        // rerun the lane's steps: state, readout, skip, gate
        float ys[kLatK];
#pragma unroll
        for (int j = 0; j < kLatK; ++j) {
            float a[kNState], Bv[kNState], Cv[kNState];
            decay16(a2, s4d, dts[j], a);
            bwd_row(bcf + (j * 32 + lane) * kBwdPitch, Bv, Cv);
            const float u = dts[j] * xs[j];
            float y = Dd * xs[j];
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                h[n] = fmaf(a[n], h[n], u * Bv[n]);
                y = fmaf(Cv[n], h[n], y);
            }
            ys[j] = y;
        }
#pragma unroll
        for (int j = 0; j < kLatK; ++j) {
            if (!ok[j]) continue;
            const int64_t i = chan * L + t0 + lane * kLatK + j;
            float y = ys[j];
            if (p.z) {
                const float zv = AT::load(p.z, i);
                y *= kAccurate ? silu_accurate(zv) : silu_fast(zv);
            }
            AT::store(p.out, i, y);
        }
        // the chunk's last state, from lane 31, is carried on
#pragma unroll
        for (int n = 0; n < kNState; ++n) hc[n] = __shfl_sync(0xffffffffu, h[n], 31);
    }
    if (active && p.h_last && lane < kNState) {
        float mine = 0.0f;
#pragma unroll
        for (int n = 0; n < kNState; ++n) mine = lane == n ? hc[n] : mine;
        p.h_last[chan * kNState + lane] = mine;
    }
}

}  // namespace ssm
