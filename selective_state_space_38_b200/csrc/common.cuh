// common.cuh -- device helpers shared by the selective-scan kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ssm {

constexpr int kNState = 16;            // states per channel (N)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- MUFU (special-function unit) wrappers: PTX instructions, called as-is ----
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- activation element types ----------------------------------------------
// bfloat16 values travel as raw 16-bit patterns; widening is a shift.
struct bf16raw {
    uint16_t bits;
};

template <typename T>
struct Act;

template <>
struct Act<float> {
    static constexpr int kBytes = 4;
    static constexpr int kPerPiece = 4;  // elements per 16-byte piece
    __device__ static float widen(float v) { return v; }
    // element i (0..3) of a 16-byte piece
    __device__ static float piece(const uint4 &v, int i) {
        const uint32_t w = i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
        return __uint_as_float(w);
    }
    __device__ static float load(const void *p, int64_t i) { return static_cast<const float *>(p)[i]; }
    __device__ static void store(void *p, int64_t i, float v) { static_cast<float *>(p)[i] = v; }
};

template <>
struct Act<bf16raw> {
    static constexpr int kBytes = 2;
    static constexpr int kPerPiece = 8;
    __device__ static float widen(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }
    __device__ static float piece(const uint4 &v, int i) {
        const uint32_t w = (i >> 1) == 0 ? v.x : (i >> 1) == 1 ? v.y : (i >> 1) == 2 ? v.z : v.w;
        return (i & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
    }
    __device__ static float load(const void *p, int64_t i) {
        return widen(static_cast<const uint16_t *>(p)[i]);
    }
    __device__ static void store(void *p, int64_t i, float v) {
        uint32_t r;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(0.0f), "f"(v));
        static_cast<uint16_t *>(p)[i] = static_cast<uint16_t>(r & 0xffffu);
    }
};

// two floats -> packed bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---- step size, gate ----------------------------------------------------------
// softplus(v) = ln(1 + e^v) from e = e^v.  For e < 1/16 the log1p series
// e (1 - e/2 + e^2/3 - e^3/4) (truncation below e^4/5 < 3.1e-6 relative):
// there 1 + e would lose the low bits of e and lg2.approx's absolute error
// would become a large relative error of a small step size.  Otherwise
// lg2(1 + e) ln 2, whose argument is >= 1.0625 (relative error ~3e-6).
__device__ __forceinline__ float softplus_from_exp(float e) {
    const float series = e * fmaf(-e, fmaf(-e, fmaf(-e, 0.25f, 1.0f / 3.0f), 0.5f), 1.0f);
    return e < 0.0625f ? series : lg2_approx(1.0f + e) * kLn2;
}
// Fast form for bf16 activations: two MUFU ops, identity above 15 (the
// remainder e^-v < 3.1e-7 is below float resolution of v).
__device__ __forceinline__ float softplus_fast(float v) {
    const float s = softplus_from_exp(ex2_approx(fminf(v, 126.0f) * kLog2e));
    return v > 15.0f ? v : s;
}
// Accurate form for float32 activations.
__device__ __forceinline__ float softplus_accurate(float v) {
    return v > 20.0f ? v : log1pf(expf(v));
}
// silu(z) = z / (1 + e^-z); e^-z may overflow to +inf, giving -0 for z << 0.
__device__ __forceinline__ float silu_fast(float z) {
    return z * rcp_approx(1.0f + ex2_approx(-z * kLog2e));
}
__device__ __forceinline__ float silu_accurate(float z) {
    return z / (1.0f + expf(-z));
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace ssm

// ---- mbarrier + TMA (cp.async.bulk.tensor) helpers ------------------------------
namespace ssm {

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// 3-D tiled TMA load of a box at coordinates (c0, c1, c2) into shared memory;
// completion is signalled on the mbarrier as transferred bytes.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int c0, int c1, int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// 3-D tiled TMA store of a shared-memory box; tracked by the bulk-group mechanism.
__device__ __forceinline__ void tma_store_3d(const void *tmap, int c0, int c1, int c2, const void *src) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until all committed bulk stores have finished reading shared memory
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until all committed bulk stores are complete
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// order this thread's generic-proxy shared-memory writes before later async-proxy (TMA) reads
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// A flag in global memory read with acquire and written with release (GPU scope).
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

}  // namespace ssm
