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
};

constexpr int kStepThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kStepThreads) scan_step_kernel(const StepParams p) {
    using AT = Act<T>;
    constexpr bool kAccurate = AT::kBytes == 4;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * kStepThreads + threadIdx.x;
    const int64_t nchan = p.batch * p.dim;
    const int64_t chan = gid >> 2;
    const int q = static_cast<int>(gid & 3);
    const bool active = chan < nchan;
    const int64_t c = active ? chan : nchan - 1;  // inactive lanes still join the shuffles
    const int64_t b = c / p.dim, d = c % p.dim;

    float4 h = *reinterpret_cast<const float4 *>(p.state + c * kNState + q * 4);
    const float4 a = *reinterpret_cast<const float4 *>(p.A + d * kNState + q * 4);
    const float xf = AT::load(p.x, c);
    float v = AT::load(p.delta, c);
    if (p.delta_bias) v += p.delta_bias[d];
    const float dt = p.softplus ? (kAccurate ? softplus_accurate(v) : softplus_fast(v)) : v;
    const float u = dt * xf;
    const int64_t bn = b * kNState + q * 4;
    const float B0 = AT::load(p.B, bn), B1 = AT::load(p.B, bn + 1), B2 = AT::load(p.B, bn + 2),
                B3 = AT::load(p.B, bn + 3);
    const float C0 = AT::load(p.C, bn), C1 = AT::load(p.C, bn + 1), C2 = AT::load(p.C, bn + 2),
                C3 = AT::load(p.C, bn + 3);

    h.x = ex2_approx(a.x * kLog2e * dt) * h.x + u * B0;
    h.y = ex2_approx(a.y * kLog2e * dt) * h.y + u * B1;
    h.z = ex2_approx(a.z * kLog2e * dt) * h.z + u * B2;
    h.w = ex2_approx(a.w * kLog2e * dt) * h.w + u * B3;
    float y = (C0 * h.x + C1 * h.y) + (C2 * h.z + C3 * h.w);
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
