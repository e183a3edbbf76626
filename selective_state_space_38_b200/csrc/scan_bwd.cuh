// scan_bwd.cuh -- backward pass of the selective scan (S6) for sm_100a.
//
// Gu & Dao, "Mamba", Appendix D "Hardware-aware Algorithm For Selective
// SSMs", paragraph "Memory": the backward pass does not keep the intermediate
// states; it recomputes them when the inputs are loaded into on-chip memory.
// Here a first kernel stores only the state at the start of every chunk of
// kBwdChunk steps (a checkpoint, 64 B per channel and chunk); the backward
// kernel walks each channel's chunks from the last to the first, recomputes
// the chunk's states from its checkpoint and runs the adjoint recurrence
//   g_t = C_t dy_t + Abar_{t+1} g_{t+1}
// through it, carrying the decayed adjoint Abar_t g_t from chunk to chunk.
//
// Work layout: lanes across time.  A warp owns one channel at a time; lane i
// owns steps t0 + kBwdK i .. t0 + kBwdK i + kBwdK - 1 of the chunk.  Both
// recurrences are linear, so each lane first folds its own steps into an
// affine map (decay product, offset) and a warp-shuffle scan of those maps
// (the work-efficient associative scan over (Abar, Bbar x) pairs) gives every
// lane its starting value: forward for the states, in reverse for the adjoint.
// The decay product of a lane's steps is exp(A sum dt), so the scans carry the
// scalar sum of dt instead of 16 products.
//
// Sums over channels (dB, dC) are accumulated per CTA in shared memory and
// written as one partial per block of kBwdBlock channels; a reduce kernel adds
// the partials.  Sums over time (dA, dD, dbias) are reduced in the warp and
// added to the outputs with float atomics (one per channel and batch).
#pragma once

#include "common.cuh"

namespace ssm {

constexpr int kBwdK = 4;                   // steps per lane
constexpr int kBwdChunk = 32 * kBwdK;      // steps per chunk (128)
constexpr int kBwdWarps = 4;               // warps per CTA
constexpr int kBwdBlock = 32;              // channels per CTA (one sequence)
constexpr int kBwdPerWarp = kBwdBlock / kBwdWarps;
constexpr int kBwdPitch = 36;              // floats per widened B|C row
constexpr int kBwdAccPitch = 17;           // floats per accumulator row (odd: conflict-free lanes)

struct BwdParams {
    const void *x, *delta, *z, *B, *C, *dout;
    const float *delta_bias, *A, *D, *h0, *dh_last;
    void *dx, *ddelta, *dz;          // [batch][dim][L], activation dtype (dz when z is given)
    float *dA, *dD, *dbias, *dh0;    // summed with atomics (zeroed by the host) / written
    float *ckpt;                     // [batch][dim][chunks][16] states at chunk starts
    float *part;                     // [dim / kBwdBlock][batch][2][16][L] partial dB, dC
    float *dB, *dC;                  // [batch][16][L]
    int64_t batch, seqlen, dim;
    int softplus;
};

__host__ __device__ inline int64_t bwd_chunks(int64_t L) { return (L + kBwdChunk - 1) / kBwdChunk; }
__host__ __device__ inline int64_t bwd_blocks(int64_t dim) { return (dim + kBwdBlock - 1) / kBwdBlock; }

// Slot of step t (0 <= t < kBwdChunk) in the lane-major tables: lane i's step j
// sits at j * 32 + i, so the 32 lanes of a warp read 32 consecutive rows.
__device__ __forceinline__ int bwd_slot(int t) { return (t % kBwdK) * 32 + t / kBwdK; }

// exp(A[d, n] * s) for the 16 states: one MUFU op and a multiplication tree for
// S4D-structured rows (A[d, n] = (n + 1) A[d, 0]), sixteen otherwise.
// The choice is made per channel (s4d is the same for the whole warp).
__device__ __forceinline__ void decay16(const float (&a2)[kNState], bool s4d, float s, float (&out)[kNState]) {
    if (s4d) {
        const float r = ex2_approx(a2[0] * s);
        const float r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
        out[0] = r; out[1] = r2; out[2] = r2 * r; out[3] = r4;
#pragma unroll
        for (int n = 4; n < 8; ++n) out[n] = out[n - 4] * r4;
#pragma unroll
        for (int n = 8; n < 16; ++n) out[n] = out[n - 8] * r8;
    } else {
#pragma unroll
        for (int n = 0; n < kNState; ++n) out[n] = ex2_approx(a2[n] * s);
    }
}

// Whether A[d, :] has the S4D-real structure A[d, n] = (n + 1) A[d, 0] exactly.
__device__ __forceinline__ bool row_is_s4d(const float *Arow) {
    bool ok = true;
#pragma unroll
    for (int n = 0; n < kNState; ++n) ok = ok && (Arow[n] == __fmul_rn(static_cast<float>(n + 1), Arow[0]));
    return ok;
}

// B (n < 16) and C (n >= 16) of one step from its widened row, as 16-byte reads
// (lane-consecutive rows of pitch 36 floats: conflict-free per quarter warp).
__device__ __forceinline__ void bwd_row(const float *row, float (&Bv)[kNState], float (&Cv)[kNState]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 b = reinterpret_cast<const float4 *>(row)[q];
        const float4 c = reinterpret_cast<const float4 *>(row)[4 + q];
        Bv[4 * q] = b.x; Bv[4 * q + 1] = b.y; Bv[4 * q + 2] = b.z; Bv[4 * q + 3] = b.w;
        Cv[4 * q] = c.x; Cv[4 * q + 1] = c.y; Cv[4 * q + 2] = c.z; Cv[4 * q + 3] = c.w;
    }
}

// Shared memory of the backward CTA (dynamic: about 73 KB).
struct BwdSmem {
    float bcf[kBwdChunk * kBwdPitch];                 // B|C, lane-major slots
    float accB[kBwdChunk * kBwdAccPitch];             // the block's dB of the chunk
    float accC[kBwdChunk * kBwdAccPitch];             // the block's dC of the chunk
    float hprev[kBwdWarps][kBwdK][4][32][4];          // h_{t-1} per warp, step, quarter, lane
    float carry[kBwdBlock][kNState];                  // decayed adjoint entering a chunk
    float sumA[kBwdBlock][kNState], sumD[kBwdBlock], sumBias[kBwdBlock];
};

template <typename T>
__device__ __forceinline__ float bwd_softplus(float v) {
    return Act<T>::kBytes == 4 ? softplus_accurate(v) : softplus_fast(v);
}

// ---- checkpoints: the state at the start of every chunk -------------------------
// One warp per channel; chunks in order.  Each lane folds its kBwdK steps from a
// zero state into (sum dt, e); an inclusive warp scan of those maps gives the
// chunk's end state from its start state.
template <typename T>
__global__ void __launch_bounds__(128) scan_bwd_ckpt_kernel(const BwdParams p) {
    using AT = Act<T>;
    const int lane = threadIdx.x & 31;
    const int64_t chan = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (chan >= p.batch * p.dim) return;
    const int64_t b = chan / p.dim, d = chan % p.dim, L = p.seqlen;
    float a2[kNState];
#pragma unroll
    for (int n = 0; n < kNState; ++n) a2[n] = p.A[d * kNState + n] * kLog2e;
    const bool s4d = row_is_s4d(p.A + d * kNState);
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.0f;
    float hc[kNState];
#pragma unroll
    for (int n = 0; n < kNState; ++n) hc[n] = p.h0 ? p.h0[chan * kNState + n] : 0.0f;
    const int64_t chunks = bwd_chunks(L);
    for (int64_t c = 0; c < chunks; ++c) {
        {
            float mine = 0.0f;  // hc[lane], without indexing registers by a runtime value
#pragma unroll
            for (int n = 0; n < kNState; ++n) mine = lane == n ? hc[n] : mine;
            if (lane < kNState) p.ckpt[(chan * chunks + c) * kNState + lane] = mine;
        }
        // this lane's steps: fold into (s, e) from a zero state
        float e[kNState], s = 0.0f;
#pragma unroll
        for (int n = 0; n < kNState; ++n) e[n] = 0.0f;
#pragma unroll
        for (int j = 0; j < kBwdK; ++j) {
            const int64_t t = c * kBwdChunk + lane * kBwdK + j;
            if (t >= L) break;
            float v = AT::load(p.delta, chan * L + t) + bias;
            const float dt = p.softplus ? bwd_softplus<T>(v) : v;
            const float u = dt * AT::load(p.x, chan * L + t);
            float a[kNState];
            decay16(a2, s4d, dt, a);
#pragma unroll
            for (int n = 0; n < kNState; ++n) e[n] = fmaf(a[n], e[n], u * AT::load(p.B, (b * kNState + n) * L + t));
            s += dt;
        }
        // inclusive scan: combine (s', e') on the left with (s, e): (s' + s, exp(A s) e' + e)
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float so = __shfl_up_sync(0xffffffffu, s, off);
            float eo[kNState], P[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) eo[n] = __shfl_up_sync(0xffffffffu, e[n], off);
            if (lane >= off) {
                decay16(a2, s4d, s, P);
#pragma unroll
                for (int n = 0; n < kNState; ++n) e[n] = fmaf(P[n], eo[n], e[n]);
                s += so;
            }
        }
        // the chunk's end state: exp(A s_total) hc + e_total (from lane 31)
        float P[kNState];
        decay16(a2, s4d, s, P);
#pragma unroll
        for (int n = 0; n < kNState; ++n) {
            const float en = __shfl_sync(0xffffffffu, fmaf(P[n], hc[n], e[n]), 31);
            hc[n] = en;
        }
    }
}

// ---- the backward pass over a block of kBwdBlock channels of one sequence -------
// grid: (dim / kBwdBlock blocks) x batch; block: kBwdWarps warps.
template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32) scan_bwd_kernel(const BwdParams p) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    extern __shared__ __align__(16) uint8_t bwd_smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(bwd_smem_raw);
    float *bcf = sm.bcf, *accB = sm.accB, *accC = sm.accC;
    auto &hprev = sm.hprev;
    auto &carry = sm.carry;
    auto &sumA = sm.sumA;
    float *sumD = sm.sumD, *sumBias = sm.sumBias;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t blk = blockIdx.x, b = blockIdx.y, L = p.seqlen;
    const int64_t d0 = blk * kBwdBlock;
    const int64_t chunks = bwd_chunks(L);

    for (int i = threadIdx.x; i < kBwdBlock * kNState; i += blockDim.x) {
        const int ch = i / kNState, n = i % kNState;
        const int64_t d = d0 + ch;
        carry[ch][n] = (p.dh_last && d < p.dim) ? p.dh_last[(b * p.dim + d) * kNState + n] : 0.0f;
        sumA[ch][n] = 0.0f;
        if (n == 0) sumD[ch] = sumBias[ch] = 0.0f;
    }
    for (int i = threadIdx.x; i < kBwdChunk * kBwdAccPitch; i += blockDim.x) accB[i] = accC[i] = 0.0f;

    for (int64_t c = chunks - 1; c >= 0; --c) {
        const int64_t t0 = c * kBwdChunk;
        __syncthreads();  // the previous chunk's tables are no longer read
        // stage B and C of the chunk, widened, in lane-major slots (zero past L)
        for (int i = threadIdx.x; i < kBwdChunk * 2 * kNState; i += blockDim.x) {
            const int t = i % kBwdChunk, jn = i / kBwdChunk;  // jn: 0..15 B, 16..31 C
            const int64_t tt = t0 + t;
            const void *src = jn < kNState ? p.B : p.C;
            const float v = tt < L ? AT::load(src, (b * kNState + (jn % kNState)) * L + tt) : 0.0f;
            bcf[bwd_slot(t) * kBwdPitch + jn] = v;
        }
        __syncthreads();

        for (int k = 0; k < kBwdPerWarp; ++k) {
            const int ch = warp * kBwdPerWarp + k;
            const int64_t d = d0 + ch;
            if (d >= p.dim) break;  // warp-uniform
            const int64_t chan = b * p.dim + d;
            float a2[kNState], An[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                An[n] = p.A[d * kNState + n];
                a2[n] = An[n] * kLog2e;
            }
            const bool s4d = row_is_s4d(p.A + d * kNState);
            const float bias = p.delta_bias ? p.delta_bias[d] : 0.0f;
            const float Dd = p.D ? p.D[d] : 0.0f;

            // this lane's steps: inputs and per-step scalars
            float xs[kBwdK], dts[kBwdK], sgs[kBwdK], go[kBwdK], zs[kBwdK];
            bool ok[kBwdK];
            float s_lane = 0.0f;
#pragma unroll
            for (int j = 0; j < kBwdK; ++j) {
                const int64_t t = t0 + lane * kBwdK + j;
                ok[j] = t < L;
                const int64_t i = chan * L + t;
                const float v = ok[j] ? AT::load(p.delta, i) + bias : 0.0f;
                dts[j] = ok[j] ? (p.softplus ? bwd_softplus<T>(v) : v) : 0.0f;
                sgs[j] = p.softplus ? 1.0f / (1.0f + __expf(-v)) : 1.0f;  // d dt / d v
                xs[j] = ok[j] ? AT::load(p.x, i) : 0.0f;
                go[j] = ok[j] ? AT::load(p.dout, i) : 0.0f;
                zs[j] = (ok[j] && p.z) ? AT::load(p.z, i) : 0.0f;
                s_lane += dts[j];
            }
            const float *brow[kBwdK];
#pragma unroll
            for (int j = 0; j < kBwdK; ++j) brow[j] = bcf + (j * 32 + lane) * kBwdPitch;

            // forward fold of the lane's steps from zero, then the exclusive warp scan
            float e[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) e[n] = 0.0f;
#pragma unroll
            for (int j = 0; j < kBwdK; ++j) {
                float a[kNState], Bv[kNState], Cv[kNState];
                decay16(a2, s4d, dts[j], a);
                bwd_row(brow[j], Bv, Cv);
                const float u = dts[j] * xs[j];
#pragma unroll
                for (int n = 0; n < kNState; ++n) e[n] = fmaf(a[n], e[n], u * Bv[n]);
            }
            float s = s_lane;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float so = __shfl_up_sync(0xffffffffu, s, off);
                float eo[kNState], P[kNState];
#pragma unroll
                for (int n = 0; n < kNState; ++n) eo[n] = __shfl_up_sync(0xffffffffu, e[n], off);
                if (lane >= off) {
                    decay16(a2, s4d, s, P);
#pragma unroll
                    for (int n = 0; n < kNState; ++n) e[n] = fmaf(P[n], eo[n], e[n]);
                    s += so;
                }
            }
            // exclusive: the maps of the lanes before this one
            float h[kNState];
            {
                // every lane takes part in the shuffle (a full-mask shuffle that a lane
                // skips waits for it forever); lane 0 then discards the value
                const float sxv = __shfl_up_sync(0xffffffffu, s, 1);
                const float sx = lane ? sxv : 0.0f;
                float ex[kNState], P[kNState];
#pragma unroll
                for (int n = 0; n < kNState; ++n) {
                    const float v = __shfl_up_sync(0xffffffffu, e[n], 1);
                    ex[n] = lane ? v : 0.0f;
                }
                decay16(a2, s4d, lane ? sx : 0.0f, P);
                const float *hc = p.ckpt + (chan * chunks + c) * kNState;
#pragma unroll
                for (int n = 0; n < kNState; ++n) h[n] = fmaf(P[n], __ldg(hc + n), ex[n]);
            }

            // the lane's steps again: states, readout, gate derivative, dC; keep h_{t-1}
            float dys[kBwdK];
#pragma unroll
            for (int j = 0; j < kBwdK; ++j) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4 *>(hprev[warp][j][q][lane]) =
                        make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
                float a[kNState], Bv[kNState], Cv[kNState];
                decay16(a2, s4d, dts[j], a);
                bwd_row(brow[j], Bv, Cv);
                const float u = dts[j] * xs[j];
                float y = Dd * xs[j];
#pragma unroll
                for (int n = 0; n < kNState; ++n) {
                    h[n] = fmaf(a[n], h[n], u * Bv[n]);
                    y = fmaf(Cv[n], h[n], y);
                }
                float dy = go[j], dzv = 0.0f;
                if (p.z) {
                    const float sg = kAccurate ? 1.0f / (1.0f + expf(-zs[j])) : rcp_approx(1.0f + ex2_approx(-zs[j] * kLog2e));
                    dy = go[j] * zs[j] * sg;
                    dzv = go[j] * y * sg * fmaf(zs[j], 1.0f - sg, 1.0f);
                }
                dys[j] = dy;
                zs[j] = dzv;  // zs now holds dz
                const int row = (j * 32 + lane) * kBwdAccPitch;
                if (ok[j]) {
#pragma unroll
                    for (int n = 0; n < kNState; ++n) atomicAdd(&accC[row + n], dy * h[n]);
                }
            }

            // reverse fold of the adjoint over the lane's steps from zero, then the
            // exclusive reverse warp scan (the lanes after this one, then the carry)
            float f[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) f[n] = 0.0f;
#pragma unroll
            for (int j = kBwdK - 1; j >= 0; --j) {
                float a[kNState], Bv[kNState], Cv[kNState];
                decay16(a2, s4d, dts[j], a);
                bwd_row(brow[j], Bv, Cv);
#pragma unroll
                for (int n = 0; n < kNState; ++n) f[n] = a[n] * fmaf(Cv[n], dys[j], f[n]);
            }
            s = s_lane;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float so = __shfl_down_sync(0xffffffffu, s, off);
                float fo[kNState], P[kNState];
#pragma unroll
                for (int n = 0; n < kNState; ++n) fo[n] = __shfl_down_sync(0xffffffffu, f[n], off);
                if (lane + off < 32) {
                    decay16(a2, s4d, s, P);
#pragma unroll
                    for (int n = 0; n < kNState; ++n) f[n] = fmaf(P[n], fo[n], f[n]);
                    s += so;
                }
            }
            float G[kNState];  // decayed adjoint entering this lane's last step from the right
            {
                const float sxv = __shfl_down_sync(0xffffffffu, s, 1);  // every lane takes part
                const float sx = lane < 31 ? sxv : 0.0f;
                float fx[kNState], P[kNState];
#pragma unroll
                for (int n = 0; n < kNState; ++n) {
                    const float v = __shfl_down_sync(0xffffffffu, f[n], 1);
                    fx[n] = lane < 31 ? v : 0.0f;
                }
                decay16(a2, s4d, lane < 31 ? sx : 0.0f, P);
#pragma unroll
                for (int n = 0; n < kNState; ++n) G[n] = fmaf(P[n], carry[ch][n], fx[n]);
            }

            // the lane's steps backwards: adjoint and every derivative
            float dAl[kNState], dDl = 0.0f, dbl = 0.0f;
#pragma unroll
            for (int n = 0; n < kNState; ++n) dAl[n] = 0.0f;
            float dxs[kBwdK], dds[kBwdK];
#pragma unroll
            for (int j = kBwdK - 1; j >= 0; --j) {
                float a[kNState], hp[kNState], Bv[kNState], Cv[kNState];
                decay16(a2, s4d, dts[j], a);
                bwd_row(brow[j], Bv, Cv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 v = *reinterpret_cast<const float4 *>(hprev[warp][j][q][lane]);
                    hp[4 * q] = v.x; hp[4 * q + 1] = v.y; hp[4 * q + 2] = v.z; hp[4 * q + 3] = v.w;
                }
                const float dt = dts[j], xv = xs[j], dy = dys[j];
                float dxv = Dd * dy, ddt = 0.0f;
                const int row = (j * 32 + lane) * kBwdAccPitch;
#pragma unroll
                for (int n = 0; n < kNState; ++n) {
                    const float g = fmaf(Cv[n], dy, G[n]);
                    const float Bn = Bv[n];
                    const float ah = a[n] * hp[n];
                    if (ok[j]) atomicAdd(&accB[row + n], g * dt * xv);
                    dxv = fmaf(g * dt, Bn, dxv);
                    ddt = fmaf(g, fmaf(An[n], ah, Bn * xv), ddt);
                    dAl[n] = fmaf(g * dt, ah, dAl[n]);
                    G[n] = a[n] * g;
                }
                dxs[j] = dxv;
                dds[j] = ok[j] ? ddt * sgs[j] : 0.0f;
                dDl = fmaf(dy, xv, dDl);
                dbl += dds[j];
            }
#pragma unroll
            for (int j = 0; j < kBwdK; ++j) {
                if (!ok[j]) continue;
                const int64_t i = chan * L + t0 + lane * kBwdK + j;
                AT::store(p.dx, i, dxs[j]);
                AT::store(p.ddelta, i, dds[j]);
                if (p.z) AT::store(p.dz, i, zs[j]);
            }
            // the carry into the previous chunk: lane 0's outgoing decayed adjoint
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                const float v = __shfl_sync(0xffffffffu, G[n], 0);
                if (lane == 0) carry[ch][n] = v;
            }
            // sums over the warp's lanes (time) for dA, dD, dbias
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
                for (int n = 0; n < kNState; ++n) dAl[n] += __shfl_xor_sync(0xffffffffu, dAl[n], off);
                dDl += __shfl_xor_sync(0xffffffffu, dDl, off);
                dbl += __shfl_xor_sync(0xffffffffu, dbl, off);
            }
            {
                float mine = 0.0f;
#pragma unroll
                for (int n = 0; n < kNState; ++n) mine = lane == n ? dAl[n] : mine;
                if (lane < kNState) sumA[ch][lane] += mine;
            }
            if (lane == 0) {
                sumD[ch] += dDl;
                sumBias[ch] += dbl;
            }
        }
        __syncthreads();
        // the block's partial dB, dC of this chunk; then clear the accumulators
        float *pb = p.part + ((blk * p.batch + b) * 2) * kNState * L;
        for (int i = threadIdx.x; i < kBwdChunk * kNState; i += blockDim.x) {
            const int t = i % kBwdChunk, n = i / kBwdChunk;
            const int64_t tt = t0 + t;
            const int at = bwd_slot(t) * kBwdAccPitch + n;
            if (tt < L) {
                pb[n * L + tt] = accB[at];
                pb[(kNState + n) * L + tt] = accC[at];
            }
            accB[at] = 0.0f;
            accC[at] = 0.0f;
        }
    }
    __syncthreads();
    // dh0 = Abar_0 g_0 (the carry out of the first chunk); dA, dD, dbias summed over batch
    for (int i = threadIdx.x; i < kBwdBlock * kNState; i += blockDim.x) {
        const int ch = i / kNState, n = i % kNState;
        const int64_t d = d0 + ch;
        if (d >= p.dim) continue;
        if (p.dh0) p.dh0[(b * p.dim + d) * kNState + n] = carry[ch][n];
        if (p.dA) atomicAdd(p.dA + d * kNState + n, sumA[ch][n]);
        if (n == 0) {
            if (p.dD) atomicAdd(p.dD + d, sumD[ch]);
            if (p.dbias) atomicAdd(p.dbias + d, sumBias[ch]);
        }
    }
}

// dB and dC: the sum of the blocks' partials, in block order.
__global__ void scan_bwd_reduce_kernel(const BwdParams p) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t per = 2 * kNState * p.seqlen;  // one sequence's dB and dC
    if (i >= p.batch * per) return;
    const int64_t b = i / per, r = i % per;
    const int64_t blocks = bwd_blocks(p.dim);
    float s = 0.0f;
    for (int64_t k = 0; k < blocks; ++k) s += p.part[(k * p.batch + b) * per + r];
    if (r < kNState * p.seqlen)
        p.dB[b * kNState * p.seqlen + r] = s;
    else
        p.dC[b * kNState * p.seqlen + r - kNState * p.seqlen] = s;
}

}  // namespace ssm
