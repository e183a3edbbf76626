// scan_fwd.cuh -- forward selective scan (S6) for sm_100a.
//
// Gu & Dao, "Mamba: Linear-Time Sequence Modeling with Selective State
// Spaces", Appendix D "Hardware-aware Algorithm For Selective SSMs" ("Speed"):
// the scan is fused (discretisation, recurrence, readout and gating in one
// pass, reading x, delta, z, B, C once and writing only out and the final
// state) and chunked along L, each chunk continuing from the carried state.
//
// Layout of the work: one thread owns one channel (b, d) and keeps its 16
// float32 states in registers for the whole sequence, so the recurrence
// h_t = exp(dt_t A) h_{t-1} + dt_t B_t x_t is evaluated once per element with
// no extra parallel-scan work.  A CTA of 128 threads covers 128 channels of
// one sequence, so B_t and C_t (shared by every channel of that sequence) are
// staged once per chunk in shared memory, widened to float32 and laid out
// time-major for broadcast reads.  x, delta and z arrive through cp.async in a
// two-stage pipeline; rows are XOR-swizzled in 16-byte pieces so that the 32
// lanes of a warp (32 different channel rows) read without bank conflicts.
//
// Discretisation (the "Mamba3" post's note that Mamba-1 pairs zero-order
// hold with Euler): Abar = exp(dt A) is evaluated as ex2(dt * A log2 e); when
// A[d, n] = (n + 1) A[d, 0] exactly (the S4D-real family), Abar_n = r^(n+1)
// with r = exp(dt A[d, 0]) is built by multiplication, one MUFU op per
// (t, channel) instead of sixteen.
#pragma once

#include "common.cuh"

namespace ssm {

struct FwdParams {
    const void *x, *delta, *z, *B, *C;
    const float *delta_bias, *A, *D, *h0;
    void *out;
    float *h_last;
    int64_t batch, seqlen, dim;
    int softplus;
};

constexpr int kFwdThreads = 128;  // channels per CTA, one per thread
constexpr int kStages = 2;        // cp.async pipeline depth (chunks in flight)
constexpr int kRowBytes = 128;    // bytes of one channel's row in a chunk
constexpr int kPieces = kRowBytes / 16;
constexpr int kBCPitch = 36;      // floats per time row of widened B|C (32 used)

template <typename T>
struct FwdSmem {
    static constexpr int kTC = kRowBytes / Act<T>::kBytes;            // timesteps per chunk
    static constexpr int kTileBytes = kFwdThreads * kRowBytes;        // one [128 ch][TC] tile
    static constexpr int kBCRawBytes = 2 * kNState * kRowBytes;       // [2][16][TC] B and C
    static constexpr int kStageBytes = 3 * kTileBytes + kBCRawBytes;  // x, delta, z, B|C
    static constexpr int kOutOff = kStages * kStageBytes;
    static constexpr int kBCFOff = kOutOff + kTileBytes;
    static constexpr int kTotal = kBCFOff + kTC * kBCPitch * 4;
};

// per-channel constants kept in registers
struct ChanConst {
    float a2[kNState];  // A[d, n] * log2(e)
    float Dd, bias;
};

// ---- loading one chunk [t0, t0 + TC) of the CTA's 128 channels --------------
template <typename T>
__device__ __forceinline__ void load_chunk_async(const FwdParams &p, uint8_t *stage, int64_t b,
                                                 int64_t d0, int64_t t0, int tid) {
    using AT = Act<T>;
    constexpr int PP = AT::kPerPiece;
    const int64_t L = p.seqlen;
    const void *const srcs[3] = {p.x, p.delta, p.z};
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        if (srcs[k] == nullptr) continue;
        const uint8_t *base = static_cast<const uint8_t *>(srcs[k]);
        uint8_t *tile = stage + k * FwdSmem<T>::kTileBytes;
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
            const int idx = tid + i * kFwdThreads;
            const int row = idx >> 3, pc = idx & 7;
            const int64_t d = d0 + row, t = t0 + pc * PP;
            int bytes = 0;
            const uint8_t *src = base;
            if (d < p.dim && t < L) {
                const int64_t rem = (L - t) * AT::kBytes;
                bytes = rem >= 16 ? 16 : static_cast<int>(rem);
                src = base + ((b * p.dim + d) * L + t) * AT::kBytes;
            }
            cp_async16(smem_u32(tile + row * kRowBytes + ((pc ^ (row & 7)) << 4)), src, bytes);
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int idx = tid + i * kFwdThreads;  // 0..255
        const int which = idx >> 7, n = (idx >> 3) & 15, pc = idx & 7;
        const uint8_t *base = static_cast<const uint8_t *>(which ? p.C : p.B);
        const int64_t t = t0 + pc * PP;
        int bytes = 0;
        const uint8_t *src = base;
        if (t < L) {
            const int64_t rem = (L - t) * AT::kBytes;
            bytes = rem >= 16 ? 16 : static_cast<int>(rem);
            src = base + ((b * kNState + n) * L + t) * AT::kBytes;
        }
        cp_async16(smem_u32(stage + 3 * FwdSmem<T>::kTileBytes + which * (kNState * kRowBytes) +
                            n * kRowBytes + pc * 16),
                   src, bytes);
    }
}

// Element-wise variant for rows that are not 16-byte aligned (L * size % 16 != 0).
template <typename T>
__device__ __forceinline__ void load_chunk_sync(const FwdParams &p, uint8_t *stage, int64_t b,
                                                int64_t d0, int64_t t0, int tid) {
    using AT = Act<T>;
    using W = typename std::conditional<AT::kBytes == 2, uint16_t, uint32_t>::type;
    constexpr int PP = AT::kPerPiece, TC = FwdSmem<T>::kTC;
    const int64_t L = p.seqlen;
    const void *const srcs[3] = {p.x, p.delta, p.z};
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        if (srcs[k] == nullptr) continue;
        const W *base = static_cast<const W *>(srcs[k]);
        uint8_t *tile = stage + k * FwdSmem<T>::kTileBytes;
        for (int idx = tid; idx < kFwdThreads * TC; idx += kFwdThreads) {
            const int row = idx / TC, col = idx % TC;
            const int64_t d = d0 + row, t = t0 + col;
            const W v = (d < p.dim && t < L) ? base[(b * p.dim + d) * L + t] : W(0);
            *reinterpret_cast<W *>(tile + row * kRowBytes + (((col / PP) ^ (row & 7)) << 4) +
                                   (col % PP) * AT::kBytes) = v;
        }
    }
    for (int idx = tid; idx < 2 * kNState * TC; idx += kFwdThreads) {
        const int which = idx / (kNState * TC), n = (idx / TC) % kNState, col = idx % TC;
        const W *base = static_cast<const W *>(which ? p.C : p.B);
        const int64_t t = t0 + col;
        const W v = t < L ? base[(b * kNState + n) * L + t] : W(0);
        *reinterpret_cast<W *>(stage + 3 * FwdSmem<T>::kTileBytes + which * (kNState * kRowBytes) +
                               n * kRowBytes + col * AT::kBytes) = v;
    }
}

// Widen B and C of the chunk to float32, time-major: bcf[t][0..15] = B[.][t],
// bcf[t][16..31] = C[.][t].  Consecutive lanes take consecutive t so the
// 16-byte stores land in distinct bank groups (pitch 36 floats).
template <typename T>
__device__ __forceinline__ void widen_bc(const uint8_t *raw, float *bcf, int tid) {
    using AT = Act<T>;
    using W = typename std::conditional<AT::kBytes == 2, uint16_t, uint32_t>::type;
    constexpr int TC = FwdSmem<T>::kTC;
    for (int item = tid; item < TC * 8; item += kFwdThreads) {
        const int t = item % TC, jg = item / TC;
        float v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = jg * 4 + q;
            const W w = reinterpret_cast<const W *>(raw + (j >> 4) * (kNState * kRowBytes) +
                                                    (j & 15) * kRowBytes)[t];
            if constexpr (AT::kBytes == 2)
                v[q] = __uint_as_float(static_cast<uint32_t>(w) << 16);
            else
                v[q] = __uint_as_float(w);
        }
        *reinterpret_cast<float4 *>(bcf + t * kBCPitch + jg * 4) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// ---- the recurrence for one channel over one chunk --------------------------
template <typename T, bool S4D, bool FULL>
__device__ __forceinline__ void scan_chunk(const uint8_t *stage, const float *bcf, uint8_t *outs,
                                           int row, int nvalid, const ChanConst &cc, float2 (&h)[8],
                                           bool has_z, bool softplus) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    constexpr int PP = AT::kPerPiece;
    constexpr int TB = FwdSmem<T>::kTileBytes;
    const int sw = row & 7;
    const uint8_t *xr = stage + row * kRowBytes;
#pragma unroll 1
    for (int pc = 0; pc < kPieces; ++pc) {
        if (!FULL && pc * PP >= nvalid) break;
        const int off = (pc ^ sw) << 4;
        const uint4 xv = *reinterpret_cast<const uint4 *>(xr + off);
        const uint4 dv = *reinterpret_cast<const uint4 *>(xr + TB + off);
        const uint4 zv = has_z ? *reinterpret_cast<const uint4 *>(xr + 2 * TB + off) : make_uint4(0, 0, 0, 0);
        float o[PP];
#pragma unroll
        for (int i = 0; i < PP; ++i) {
            const int t = pc * PP + i;
            if (!FULL && t >= nvalid) {
                o[i] = 0.0f;
                continue;
            }
            const float xf = AT::piece(xv, i);
            const float v = AT::piece(dv, i) + cc.bias;
            const float dt = softplus ? (kAccurate ? softplus_accurate(v) : softplus_fast(v)) : v;
            const float u = dt * xf;
            const float4 *bc = reinterpret_cast<const float4 *>(bcf + t * kBCPitch);
            float Bv[kNState], Cv[kNState];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 b4 = bc[q], c4 = bc[4 + q];
                Bv[4 * q] = b4.x; Bv[4 * q + 1] = b4.y; Bv[4 * q + 2] = b4.z; Bv[4 * q + 3] = b4.w;
                Cv[4 * q] = c4.x; Cv[4 * q + 1] = c4.y; Cv[4 * q + 2] = c4.z; Cv[4 * q + 3] = c4.w;
            }
            const float2 U = make_float2(u, u);
            float2 ya = make_float2(cc.Dd * xf, 0.0f), yb = make_float2(0.0f, 0.0f);
            if constexpr (S4D) {
                // Abar_n = r^(n+1): pairs (r^(2j+1), r^(2j+2)) advance by r^2
                const float r = ex2_approx(cc.a2[0] * dt);
                const float r2 = r * r;
                float2 a = make_float2(r, r2);
                const float2 R2 = make_float2(r2, r2);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float2 ub = __fmul2_rn(U, make_float2(Bv[2 * j], Bv[2 * j + 1]));
                    h[j] = __ffma2_rn(a, h[j], ub);
                    if (j & 1)
                        yb = __ffma2_rn(make_float2(Cv[2 * j], Cv[2 * j + 1]), h[j], yb);
                    else
                        ya = __ffma2_rn(make_float2(Cv[2 * j], Cv[2 * j + 1]), h[j], ya);
                    if (j < 7) a = __fmul2_rn(a, R2);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float2 a = make_float2(ex2_approx(cc.a2[2 * j] * dt), ex2_approx(cc.a2[2 * j + 1] * dt));
                    const float2 ub = __fmul2_rn(U, make_float2(Bv[2 * j], Bv[2 * j + 1]));
                    h[j] = __ffma2_rn(a, h[j], ub);
                    if (j & 1)
                        yb = __ffma2_rn(make_float2(Cv[2 * j], Cv[2 * j + 1]), h[j], yb);
                    else
                        ya = __ffma2_rn(make_float2(Cv[2 * j], Cv[2 * j + 1]), h[j], ya);
                }
            }
            float y = (ya.x + yb.x) + (ya.y + yb.y);
            if (has_z) {
                const float zf = AT::piece(zv, i);
                y *= kAccurate ? silu_accurate(zf) : silu_fast(zf);
            }
            o[i] = y;
        }
        uint4 pk;
        if constexpr (AT::kBytes == 2) {
            pk = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                            pack_bf16x2(o[6], o[7]));
        } else {
            pk = make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                            __float_as_uint(o[3]));
        }
        *reinterpret_cast<uint4 *>(outs + row * kRowBytes + off) = pk;
    }
}

// ---- writing the chunk's outputs --------------------------------------------
template <typename T, bool VEC>
__device__ __forceinline__ void store_chunk(const FwdParams &p, const uint8_t *outs, int64_t b,
                                            int64_t d0, int64_t t0, int tid) {
    using AT = Act<T>;
    using W = typename std::conditional<AT::kBytes == 2, uint16_t, uint32_t>::type;
    constexpr int PP = AT::kPerPiece, TC = FwdSmem<T>::kTC;
    const int64_t L = p.seqlen;
    uint8_t *base = static_cast<uint8_t *>(p.out);
    if constexpr (VEC) {
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
            const int idx = tid + i * kFwdThreads;
            const int row = idx >> 3, pc = idx & 7;
            const int64_t d = d0 + row, t = t0 + pc * PP;
            if (d >= p.dim || t >= L) continue;
            const uint8_t *src = outs + row * kRowBytes + ((pc ^ (row & 7)) << 4);
            uint8_t *dst = base + ((b * p.dim + d) * L + t) * AT::kBytes;
            if (L - t >= PP) {
                *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
            } else {
                for (int e = 0; e < L - t; ++e)
                    reinterpret_cast<W *>(dst)[e] = reinterpret_cast<const W *>(src)[e];
            }
        }
    } else {
        for (int idx = tid; idx < kFwdThreads * TC; idx += kFwdThreads) {
            const int row = idx / TC, col = idx % TC;
            const int64_t d = d0 + row, t = t0 + col;
            if (d >= p.dim || t >= L) continue;
            const W v = *reinterpret_cast<const W *>(outs + row * kRowBytes +
                                                     (((col / PP) ^ (row & 7)) << 4) + (col % PP) * AT::kBytes);
            reinterpret_cast<W *>(base)[(b * p.dim + d) * L + t] = v;
        }
    }
}

// ---- the kernel --------------------------------------------------------------
// grid: batch * ceil(dim / 128) CTAs; block: 128 threads; dynamic smem FwdSmem<T>::kTotal
template <typename T, bool VEC>
__global__ void __launch_bounds__(kFwdThreads, 1) scan_fwd_kernel(const FwdParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    using SM = FwdSmem<T>;
    constexpr int TC = SM::kTC;
    const int tid = threadIdx.x;
    const int64_t tiles = (p.dim + kFwdThreads - 1) / kFwdThreads;
    const int64_t b = blockIdx.x / tiles;
    const int64_t d0 = (blockIdx.x % tiles) * kFwdThreads;
    const int64_t d = d0 + tid;
    const bool active = d < p.dim;
    const int64_t dc = active ? d : p.dim - 1;

    ChanConst cc;
    bool s4d = true;
    {
        const float4 *ar = reinterpret_cast<const float4 *>(p.A + dc * kNState);
        float a[kNState];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = ar[q];
            a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int n = 0; n < kNState; ++n) {
            cc.a2[n] = a[n] * kLog2e;
            s4d = s4d && (a[n] == __fmul_rn(static_cast<float>(n + 1), a[0]));
        }
        cc.Dd = p.D ? p.D[dc] : 0.0f;
        cc.bias = p.delta_bias ? p.delta_bias[dc] : 0.0f;
    }
    const bool warp_s4d = __all_sync(0xffffffffu, s4d);
    const bool has_z = p.z != nullptr;
    const bool softplus = p.softplus != 0;

    float2 h[8];
    if (active && p.h0) {
        const float4 *hr = reinterpret_cast<const float4 *>(p.h0 + (b * p.dim + d) * kNState);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = hr[q];
            h[2 * q] = make_float2(v.x, v.y);
            h[2 * q + 1] = make_float2(v.z, v.w);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) h[j] = make_float2(0.0f, 0.0f);
    }

    const int64_t L = p.seqlen;
    const int64_t nchunks = (L + TC - 1) / TC;
    uint8_t *outs = smem + SM::kOutOff;
    float *bcf = reinterpret_cast<float *>(smem + SM::kBCFOff);

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < nchunks) {
            if constexpr (VEC)
                load_chunk_async<T>(p, smem + s * SM::kStageBytes, b, d0, s * TC, tid);
            else
                load_chunk_sync<T>(p, smem + s * SM::kStageBytes, b, d0, s * TC, tid);
        }
        cp_async_commit();
    }
    for (int64_t k = 0; k < nchunks; ++k) {
        const int64_t kn = k + kStages - 1;
        if (kn < nchunks) {
            uint8_t *st = smem + (kn % kStages) * SM::kStageBytes;
            if constexpr (VEC)
                load_chunk_async<T>(p, st, b, d0, kn * TC, tid);
            else
                load_chunk_sync<T>(p, st, b, d0, kn * TC, tid);
        }
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncthreads();
        const uint8_t *stage = smem + (k % kStages) * SM::kStageBytes;
        widen_bc<T>(stage + 3 * SM::kTileBytes, bcf, tid);
        __syncthreads();
        const int nvalid = static_cast<int>(L - k * TC < TC ? L - k * TC : TC);
        if (nvalid == TC) {
            if (warp_s4d)
                scan_chunk<T, true, true>(stage, bcf, outs, tid, nvalid, cc, h, has_z, softplus);
            else
                scan_chunk<T, false, true>(stage, bcf, outs, tid, nvalid, cc, h, has_z, softplus);
        } else {
            if (warp_s4d)
                scan_chunk<T, true, false>(stage, bcf, outs, tid, nvalid, cc, h, has_z, softplus);
            else
                scan_chunk<T, false, false>(stage, bcf, outs, tid, nvalid, cc, h, has_z, softplus);
        }
        __syncthreads();
        store_chunk<T, VEC>(p, outs, b, d0, k * TC, tid);
    }
    cp_async_wait<0>();

    if (active && p.h_last) {
        float4 *hr = reinterpret_cast<float4 *>(p.h_last + (b * p.dim + d) * kNState);
#pragma unroll
        for (int q = 0; q < 4; ++q) hr[q] = make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y);
    }
}

}  // namespace ssm
