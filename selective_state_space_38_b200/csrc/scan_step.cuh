// scan_step.cuh -- one recurrent (decode) step of the selective SSM.
//
// The pages' recurrent mode: inputs arrive one timestep at a time and the
// cache holds the SSM state after the scan.  Each step reads the float32 state
// [batch][dim][16] from HBM, applies one ZOH/Euler update with the token's dt,
// B, C, and writes the state back in place plus one gated output per channel.
// The step moves 128 bytes of state per channel and does ~100 flops on it, so
// it is bound by HBM bandwidth; the kernel is laid out for coalescing: four
// consecutive lanes share one channel, each owning 4 states (one 16-byte
// vector), so a warp streams 8 channels x 64 bytes contiguously, and each
// thread takes four such channels, whose states are all in flight at once.
// The partial readouts of the four lanes are combined with two butterfly
// shuffles.
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

constexpr int kStepThreads = 128;
constexpr int kStepPasses = 2;                                  // channels per four lanes
constexpr int kStepTile = kStepThreads / 4 * kStepPasses;       // channels per CTA

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

// 16 bytes global -> shared without a register round trip (src_bytes = 0: zeros,
// nothing read); one commit group per call site, waited for by count.
__device__ __forceinline__ void step_copy16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void step_copy_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// until at most n groups are pending (n known at compile time after unrolling)
__device__ __forceinline__ void step_copy_wait_upto(int n) {
    if (n >= 3) step_copy_wait<3>();
    else if (n == 2) step_copy_wait<2>();
    else if (n == 1) step_copy_wait<1>();
    else step_copy_wait<0>();
}

// Work layout: a CTA owns kStepTile consecutive channels; thread t takes the
// four states q = t & 3 of channel base + (kStepThreads / 4) k + (t >> 2) in
// pass k.  Every pass's state is copied into shared memory at the start
// (kStepPasses 16-byte copies per thread in flight at once, with no registers
// held).  Two passes of 128-thread CTAs measured best: more passes make the
// per-channel loads after an L2 flush wait longer, bigger CTAs leave a longer
// tail.
// SMALL: every channel index fits in 32 bits, so (b, d) come from a 32-bit division.
// CONV: the token first passes the convolution window (every lane of a
// channel computes it; the first lane shifts the stored window).
// TRAP: h = Abar (h + (1 - lam) dt x_prev B_prev) + lam dt x B.
template <typename T, bool SMALL, bool CONV, bool TRAP = false>
__global__ void __launch_bounds__(kStepThreads) scan_step_kernel(const StepParams p) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    __shared__ __align__(16) float4 hs[kStepPasses][kStepThreads];
    // channel indices in 32 bits when every one fits (offsets widen once, at the pointer)
    using Ix = std::conditional_t<SMALL, uint32_t, int64_t>;
    const int tid = threadIdx.x, q = tid & 3;
    const Ix nchan = static_cast<Ix>(p.batch * p.dim), dim = static_cast<Ix>(p.dim);
    const Ix base = static_cast<Ix>(blockIdx.x) * kStepTile + static_cast<Ix>(tid >> 2);
#pragma unroll
    for (int k = 0; k < kStepPasses; ++k) {
        const Ix chan = base + k * (kStepThreads / 4);
        const Ix c = chan < nchan ? chan : nchan - 1;
        step_copy16(&hs[k][tid], p.state + static_cast<uint64_t>(c) * kNState + q * 4, chan < nchan ? 16u : 0u);
    }
    // (b, d) of the first pass's channel by one division; the later passes' by
    // stepping kStepThreads / 4 channels on (inactive lanes keep the last channel)
    Ix b, d;
    {
        const Ix c = base < nchan ? base : nchan - 1;
        b = c / dim;
        d = c - b * dim;
    }
#pragma unroll
    for (int k = 0; k < kStepPasses; ++k) {
        const Ix chan = base + k * (kStepThreads / 4);
        const bool active = chan < nchan;
        const Ix c = active ? chan : nchan - 1;  // inactive lanes still join the shuffles
        if (k > 0) {
            if (active) {
                d += kStepThreads / 4;
                while (d >= dim) {  // once at most when dim >= kStepThreads / 4
                    d -= dim;
                    ++b;
                }
            } else {
                b = (nchan - 1) / dim;
                d = (nchan - 1) - b * dim;
            }
        }
        const float4 a = *reinterpret_cast<const float4 *>(p.A + static_cast<uint64_t>(d) * kNState + q * 4);
        float xf = AT::load(p.x, c);
        float v = AT::load(p.delta, c);
        const float zf = p.z && q == 0 ? AT::load(p.z, c) : 0.0f;
        if (p.delta_bias) v += p.delta_bias[d];
        const int64_t bn = static_cast<int64_t>(static_cast<uint64_t>(b) * kNState) + q * 4;
        const float4 Bv = load4<T>(p.B, bn), Cv = load4<T>(p.C, bn);
        if constexpr (CONV) {
            float window[3] = {0.0f, 0.0f, 0.0f};
            const int K1 = p.conv_k - 1;
            float acc = p.conv_bias ? p.conv_bias[d] : 0.0f;
#pragma unroll
            for (int i = 0; i < 3; ++i)
                if (i < K1) {
                    window[i] = AT::load(p.conv_state, c * K1 + i);
                    acc = fmaf(p.conv_w[d * p.conv_k + i], window[i], acc);
                }
            acc = fmaf(p.conv_w[d * p.conv_k + K1], xf, acc);
            // the window moves on by one input: oldest dropped, this token last
            __syncwarp();  // every lane of the channel has read the window
            if (active && q == 0) {
#pragma unroll
                for (int i = 0; i < 3; ++i)
                    if (i < K1) AT::store(p.conv_state, c * K1 + i, i + 1 < K1 ? window[i + 1] : xf);
            }
            xf = kAccurate ? silu_accurate(acc) : silu_fast(acc);
        }
        const float dt = p.softplus ? (kAccurate ? softplus_accurate(v) : softplus_fast(v)) : v;
        const float u = dt * xf;
        const float e = kLog2e * dt;
        // this pass's state has landed (the later passes' copies may still be in flight)
        step_copy_wait_upto(kStepPasses - 1 - k);
        float4 h = hs[k][tid];

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

        if (active) {
            *reinterpret_cast<float4 *>(p.state + static_cast<uint64_t>(c) * kNState + q * 4) = h;
            if (q == 0) {
                if (p.D) y += p.D[d] * xf;
                if (p.z) y *= kAccurate ? silu_accurate(zf) : silu_fast(zf);
                AT::store(p.out, c, y);
            }
        }
    }
}

}  // namespace ssm
