// scan_step.cuh -- one recurrent (decode) step of the selective SSM.
//
// The pages' recurrent mode: inputs arrive one timestep at a time and the
// cache holds the SSM state after the scan.  Each step reads the float32 state
// [batch][dim][16] from HBM, applies one ZOH/Euler update with the token's dt,
// B, C, and writes the state back in place plus one gated output per channel.
// The step moves 128 bytes of state per channel and does ~100 flops on it, so
// it is bound by HBM bandwidth; the kernel is laid out for coalescing: four
// consecutive lanes share one channel, each owning 4 states (one 16-byte
// vector), so a warp streams 8 channels x 64 bytes contiguously.  The partial
// readouts of the four lanes are combined with two butterfly shuffles.
#pragma once

#include "common.cuh"

namespace ssm {

struct StepParams {
    float *state;
    const void *x, *delta, *z, *B, *C;
    const float *delta_bias, *A, *D;
    void *out;
    int64_t batch, dim;
    int softplus;
    // the short causal convolution in front of the scan (conv_k = 0: none):
    // x is the raw token, the scan's x is silu(conv_w . [window, x] + conv_bias)
    int conv_k;                 // width, 1..4
    const float *conv_w;        // [dim][conv_k]
    const float *conv_bias;     // [dim] or NULL
    void *conv_state;           // [batch][dim][conv_k - 1] raw inputs, oldest first; read and shifted
    // the exponential-trapezoidal rule: lam [batch][dim]; the previous token's
    // x_prev [batch][dim] and B_prev [batch][16] (no previous input unless both)
    const void *lam, *x_prev, *B_prev;
};

constexpr int kStepThreads = 256;

// four consecutive B or C values of one sequence (an 8- or 16-byte vector load;
// the API requires 16-byte aligned B and C, and the offset is a multiple of 4)
template <typename T>
__device__ __forceinline__ float4 load4(const void *p, int64_t i) {
    if constexpr (Act<T>::kBytes == 4) {
        return *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
    } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p) + i);
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u), __uint_as_float(w.y << 16),
                           __uint_as_float(w.y & 0xffff0000u));
    }
}

// SMALL: every channel index fits in 32 bits, so (b, d) come from a 32-bit division.
// CONV: the token first passes the convolution window (every lane of a
// channel computes it; the first lane shifts the stored window).
// TRAP: h = Abar (h + (1 - lam) dt x_prev B_prev) + lam dt x B.
template <typename T, bool SMALL, bool CONV, bool TRAP = false>
__global__ void __launch_bounds__(kStepThreads) scan_step_kernel(const StepParams p) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * kStepThreads + threadIdx.x;
    const int64_t nchan = p.batch * p.dim;
    const int64_t chan = gid >> 2;
    const int q = static_cast<int>(gid & 3);
    const bool active = chan < nchan;
    const int64_t c = active ? chan : nchan - 1;  // inactive lanes still join the shuffles
    int64_t b, d;
    if constexpr (SMALL) {
        const uint32_t c32 = static_cast<uint32_t>(c), dim32 = static_cast<uint32_t>(p.dim);
        b = c32 / dim32;
        d = c32 - static_cast<uint32_t>(b) * dim32;
    } else {
        b = c / p.dim;
        d = c % p.dim;
    }

    float4 h = *reinterpret_cast<const float4 *>(p.state + c * kNState + q * 4);
    const float4 a = *reinterpret_cast<const float4 *>(p.A + d * kNState + q * 4);
    float xf = AT::load(p.x, c);
    float window[3] = {0.0f, 0.0f, 0.0f};
    if constexpr (CONV) {
        const int K1 = p.conv_k - 1;
        float acc = p.conv_bias ? p.conv_bias[d] : 0.0f;
#pragma unroll
        for (int k = 0; k < 3; ++k)
            if (k < K1) {
                window[k] = AT::load(p.conv_state, c * K1 + k);
                acc = fmaf(p.conv_w[d * p.conv_k + k], window[k], acc);
            }
        acc = fmaf(p.conv_w[d * p.conv_k + K1], xf, acc);
        // the window moves on by one input: oldest dropped, this token last
        __syncwarp();  // every lane of the channel has read the window
        if (active && q == 0) {
#pragma unroll
            for (int k = 0; k < 3; ++k)
                if (k < K1) AT::store(p.conv_state, c * K1 + k, k + 1 < K1 ? window[k + 1] : xf);
        }
        xf = kAccurate ? silu_accurate(acc) : silu_fast(acc);
    }
    float v = AT::load(p.delta, c);
    if (p.delta_bias) v += p.delta_bias[d];
    const int64_t bn = b * kNState + q * 4;
    const float4 Bv = load4<T>(p.B, bn), Cv = load4<T>(p.C, bn);
    const float dt = p.softplus ? (kAccurate ? softplus_accurate(v) : softplus_fast(v)) : v;
    const float u = dt * xf;
    const float e = kLog2e * dt;

    if constexpr (TRAP) {
        const float lam = AT::load(p.lam, c);
        const bool prev = p.x_prev && p.B_prev;
        const float f = prev ? (1.0f - lam) * dt * AT::load(p.x_prev, c) : 0.0f;
        const float4 Bp = prev ? load4<T>(p.B_prev, bn) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        const float g = lam * u;
        h.x = ex2_approx(a.x * e) * fmaf(f, Bp.x, h.x) + g * Bv.x;
        h.y = ex2_approx(a.y * e) * fmaf(f, Bp.y, h.y) + g * Bv.y;
        h.z = ex2_approx(a.z * e) * fmaf(f, Bp.z, h.z) + g * Bv.z;
        h.w = ex2_approx(a.w * e) * fmaf(f, Bp.w, h.w) + g * Bv.w;
    } else {
        h.x = ex2_approx(a.x * e) * h.x + u * Bv.x;
        h.y = ex2_approx(a.y * e) * h.y + u * Bv.y;
        h.z = ex2_approx(a.z * e) * h.z + u * Bv.z;
        h.w = ex2_approx(a.w * e) * h.w + u * Bv.w;
    }
    float y = (Cv.x * h.x + Cv.y * h.y) + (Cv.z * h.z + Cv.w * h.w);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);

    if (!active) return;
    *reinterpret_cast<float4 *>(p.state + c * kNState + q * 4) = h;
    if (q == 0) {
        if (p.D) y += p.D[d] * xf;
        if (p.z) {
            const float zf = AT::load(p.z, c);
            y *= kAccurate ? silu_accurate(zf) : silu_fast(zf);
        }
        AT::store(p.out, c, y);
    }
}

}  // namespace ssm
