// ssd_fwd.cuh -- Mamba-2 state space duality (SSD) forward on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// "A Secret Weapon For mamba paper" (the Mamba-2 abstract: SSMs and attention
// are connected through structured semiseparable matrices) and the "Mamba3"
// posts (Mamba-2 reduces the state transition to a scalar times the
// identity).  Per batch b and head h, with a_t = exp(dt_t A_h):
//   H_t = a_t H_{t-1} + (dt_t x_t) B_t^T,   y_t = H_t C_t + D_h x_t
// Because the transition is a scalar, a chunk of Q steps is a product of dense
// matrices (the semiseparable form): with cs_i the running sum of dt A over
// the chunk,
//   Y_diag = (C B^T o L) X,      L[i, j] = exp(cs_i - cs_j) dt_j (j <= i)
//   Y_off  = diag(exp(cs)) C S_in^T
//   S_out  = exp(cs_{Q-1}) S_in + (B o w)^T X,   w_j = exp(cs_{Q-1} - cs_j) dt_j
// One CTA owns one (batch, head) sequence and walks its chunks; the state
// S^T (N x P float32) stays in registers, one row per thread.  Per chunk:
//   MMA1 G = C B^T (128 x 128 x 128) and MMA3 Yo = C S_in^T (128 x 64 x 128),
//   then the epilogue forms L o G and B o w, then
//   MMA2 Yd = (L o G) X (128 x 64 x 128) and MMA4 ST = (B o w)^T X (128 x 64 x 128).
// Operands are bf16 in shared memory in the 128-byte-swizzled canonical
// layouts; the ones that are products (L o G, B o w, S) are split into a bf16
// high and low part (two MMAs each), so they keep about 16 bits.  One thread
// issues the MMAs; tcgen05.commit arrives on an mbarrier that all warps wait
// on (bounded); each thread then reads its TMEM lane with tcgen05.ld.
#pragma once

#include "common.cuh"

namespace ssm {

constexpr int kSsdQ = 128;  // chunk length
constexpr int kSsdP = 64;   // head dimension
constexpr int kSsdN = 128;  // state dimension
constexpr uint32_t kSsdWaitLimit = 1u << 24;

struct SsdParams {
    const void *x, *dt, *B, *C;  // x [b][L][H][P], dt [b][L][H], B, C [b][L][G][N] (bf16)
    const float *dt_bias, *A, *D, *h0;
    void *y;                     // [b][L][H][P] bf16
    float *h_last;               // [b][H][P][N]
    uint32_t *error;             // bounded-wait failure word
    int64_t batch, seqlen, heads, groups;
    int softplus;
};

// Shared memory (1024-byte aligned pieces; every operand tile is [rows][64] bf16
// with 128-byte rows and the 128-byte swizzle).
struct SsdSmem {
    static constexpr int kTile = 128 * 128;          // one [128][64] bf16 tile
    static constexpr int kC = 0;                     // C  [t][n]: 2 tiles (n < 64, n >= 64)
    static constexpr int kB = kC + 2 * kTile;        // B  [t][n], then B o w (high part) in place
    static constexpr int kBWlo = kB + 2 * kTile;     // B o w (low part)
    static constexpr int kX = kBWlo + 2 * kTile;     // X  [t][p]: 1 tile
    static constexpr int kMhi = kX + kTile;          // L o G [i][j] high: 2 tiles (j < 64, j >= 64)
    static constexpr int kMlo = kMhi + 2 * kTile;    // low
    static constexpr int kS = kMlo + 2 * kTile;      // S [p][n] high and low: 2 x 2 tiles of [64][64]
    static constexpr int kCs = kS + 4 * 64 * 128;    // cs[128], dt[128], warp sums[4]
    static constexpr int kBar = kCs + 3 * 128 * 4;
    static constexpr int kTotal = kBar + 64 + 1024;  // + alignment slack
};
static_assert(SsdSmem::kTotal <= 227 * 1024, "shared memory of the SSD kernel");

__device__ __forceinline__ uint32_t ssd_sw128(int r, int e) {  // byte offset of (row r, element e)
    const int c = e >> 3, w = (e & 7) * 2;
    return r * 128 + (((c ^ (r & 7)) << 4) | w);
}

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 descriptor version.
__device__ __forceinline__ uint64_t ssd_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFF) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor: bf16 x bf16 -> f32, M x N, operand majors (0 = K, 1 = MN).
__host__ __device__ constexpr uint32_t ssd_idesc(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void ssd_mma(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void ssd_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 16 consecutive float32 columns of this thread's TMEM lane
__device__ __forceinline__ void ssd_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ bool ssd_wait(uint64_t *bar, uint32_t parity, uint32_t *error) {
    const uint32_t addr = smem_u32(bar);
    for (uint32_t n = 0; n < kSsdWaitLimit; ++n) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
    }
    atomicOr(error, 2u);
    return false;
}

__device__ __forceinline__ void split_bf16(float v, uint16_t &hi, uint16_t &lo) {
    const uint32_t h = pack_bf16x2(v, 0.0f) & 0xffffu;
    hi = static_cast<uint16_t>(h);
    const float rest = v - __uint_as_float(h << 16);
    lo = static_cast<uint16_t>(pack_bf16x2(rest, 0.0f) & 0xffffu);
}

// grid: batch * heads CTAs; block: 128 threads (thread i = TMEM lane i).
__global__ void __launch_bounds__(128, 1) ssd_fwd_kernel(const SsdParams p) {
    extern __shared__ __align__(1024) uint8_t ssd_smem_raw[];
    uint8_t *sm = ssd_smem_raw + ((1024u - (smem_u32(ssd_smem_raw) & 1023u)) & 1023u);
    using S = SsdSmem;
    float *cs = reinterpret_cast<float *>(sm + S::kCs);
    float *dts = cs + 128;
    float *wsum = dts + 128;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + S::kBar);  // [0] C-stage MMAs, [1] X-stage MMAs
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + S::kBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.x / p.heads, h = blockIdx.x % p.heads;
    const int64_t g = h / (p.heads / p.groups);
    const int64_t L = p.seqlen, H = p.heads, G = p.groups;
    const float Ah = p.A[h], bias = p.dt_bias ? p.dt_bias[h] : 0.0f, Dh = p.D ? p.D[h] : 0.0f;

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar + 1)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tslot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(tslot);
    const uint32_t tG = tbase, tYd = tbase + 128, tYo = tbase + 192, tST = tbase + 256;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

    // this thread's row n of the carried state S^T (64 values over p)
    float st[kSsdP];
#pragma unroll
    for (int q = 0; q < kSsdP; ++q) st[q] = p.h0 ? p.h0[((b * H + h) * kSsdP + q) * kSsdN + tid] : 0.0f;

    const uint32_t a_c = smem_u32(sm + S::kC), a_b = smem_u32(sm + S::kB), a_bwlo = smem_u32(sm + S::kBWlo);
    const uint32_t a_x = smem_u32(sm + S::kX), a_mhi = smem_u32(sm + S::kMhi), a_mlo = smem_u32(sm + S::kMlo);
    const uint32_t a_s = smem_u32(sm + S::kS);
    const int64_t chunks = (L + kSsdQ - 1) / kSsdQ;
    bool ok = true;
    for (int64_t c = 0; c < chunks && ok; ++c) {
        const int64_t t0 = c * kSsdQ;
        __syncthreads();
        // ---- stage C, B ([t][n], 16-byte pieces), X ([t][p]) and dt; zero past L
        const uint16_t *Bg = static_cast<const uint16_t *>(p.B), *Cg = static_cast<const uint16_t *>(p.C);
        const uint16_t *Xg = static_cast<const uint16_t *>(p.x);
        for (int i = tid; i < 128 * 16; i += 128) {  // 128 rows x 16 pieces of 8 elements
            const int r = i / 16, pc = i % 16;
            const int64_t t = t0 + r;
            uint4 vb = make_uint4(0, 0, 0, 0), vc = vb;
            if (t < L) {
                const int64_t off = ((b * L + t) * G + g) * kSsdN + pc * 8;
                vb = *reinterpret_cast<const uint4 *>(Bg + off);
                vc = *reinterpret_cast<const uint4 *>(Cg + off);
            }
            const uint32_t o = (pc / 8) * S::kTile + ssd_sw128(r, (pc % 8) * 8);
            *reinterpret_cast<uint4 *>(sm + S::kB + o) = vb;
            *reinterpret_cast<uint4 *>(sm + S::kC + o) = vc;
        }
        for (int i = tid; i < 128 * 8; i += 128) {
            const int r = i / 8, pc = i % 8;
            const int64_t t = t0 + r;
            uint4 vx = make_uint4(0, 0, 0, 0);
            if (t < L) vx = *reinterpret_cast<const uint4 *>(Xg + ((b * L + t) * H + h) * kSsdP + pc * 8);
            *reinterpret_cast<uint4 *>(sm + S::kX + ssd_sw128(r, pc * 8)) = vx;
        }
        // the carried state as bf16 high/low S[p][n] (K-major for C S^T: rows p, K = n)
        for (int q = 0; q < kSsdP; ++q) {
            uint16_t hi, lo;
            split_bf16(st[q], hi, lo);
            const uint32_t o = (tid / 64) * (64 * 128) + ssd_sw128(q, tid % 64);
            *reinterpret_cast<uint16_t *>(sm + S::kS + o) = hi;
            *reinterpret_cast<uint16_t *>(sm + S::kS + 2 * 64 * 128 + o) = lo;
        }
        // dt and the running sum cs of dt A over the chunk
        {
            const int64_t t = t0 + tid;
            float dtv = 0.0f;
            if (t < L) {
                const float v = Act<bf16raw>::load(p.dt, (b * L + t) * H + h) + bias;
                dtv = p.softplus ? softplus_fast(v) : v;
            }
            float s = dtv * Ah;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, s, off);
                if (lane >= off) s += o;
            }
            if (lane == 31) wsum[warp] = s;
            dts[tid] = dtv;
            __syncthreads();
            for (int w = 0; w < warp; ++w) s += wsum[w];
            cs[tid] = s;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // ---- MMA1: G = C B^T; MMA3: Yo = C S^T (high, then low accumulated)
        if (tid == 0) {
            constexpr uint32_t i1 = ssd_idesc(128, 128, 0, 0), i3 = ssd_idesc(128, 64, 0, 0);
            for (int s = 0; s < 8; ++s) {
                const uint32_t ko = (s / 4) * S::kTile + (s % 4) * 32;
                ssd_mma(tG, ssd_desc(a_c + ko, 16, 1024), ssd_desc(a_b + ko, 16, 1024), i1, s > 0);
            }
            for (int part = 0; part < 2; ++part)
                for (int s = 0; s < 8; ++s) {
                    const uint32_t ka = (s / 4) * S::kTile + (s % 4) * 32;
                    const uint32_t kb = part * (2 * 64 * 128) + (s / 4) * (64 * 128) + (s % 4) * 32;
                    ssd_mma(tYo, ssd_desc(a_c + ka, 16, 1024), ssd_desc(a_s + kb, 16, 1024), i3, part > 0 || s > 0);
                }
            ssd_commit(bar);
        }
        // every thread takes the same branch: a wait that gave up ends the walk
        if (!__syncthreads_and(ssd_wait(bar, static_cast<uint32_t>(c & 1), p.error))) {
            ok = false;
            break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // ---- epilogue 1: row i of L o G (high/low); row j of B o w (high in place, low)
        const float total = cs[kSsdQ - 1];
        {
            const int i = tid;
            const float csi = cs[i];
            for (int j0 = 0; j0 < kSsdQ; j0 += 16) {
                float v[16];
                ssd_ld16(tG + lane_off + j0, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j = j0 + e;
                    const float m = j <= i ? v[e] * __expf(csi - cs[j]) * dts[j] : 0.0f;
                    uint16_t hi, lo;
                    split_bf16(m, hi, lo);
                    const uint32_t o = (j / 64) * S::kTile + ssd_sw128(i, j % 64);
                    *reinterpret_cast<uint16_t *>(sm + S::kMhi + o) = hi;
                    *reinterpret_cast<uint16_t *>(sm + S::kMlo + o) = lo;
                }
            }
            const int jr = tid;
            const float w = __expf(total - cs[jr]) * dts[jr];
            for (int n = 0; n < kSsdN; ++n) {
                const uint32_t o = (n / 64) * S::kTile + ssd_sw128(jr, n % 64);
                const float bv = __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<uint16_t *>(sm + S::kB + o)) << 16);
                uint16_t hi, lo;
                split_bf16(bv * w, hi, lo);
                *reinterpret_cast<uint16_t *>(sm + S::kB + o) = hi;
                *reinterpret_cast<uint16_t *>(sm + S::kBWlo + o) = lo;
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // ---- MMA2: Yd = (L o G) X; MMA4: ST = (B o w)^T X (each high + low)
        if (tid == 0) {
            constexpr uint32_t i2 = ssd_idesc(128, 64, 0, 1), i4 = ssd_idesc(128, 64, 1, 1);
            for (int part = 0; part < 2; ++part)
                for (int s = 0; s < 8; ++s) {
                    const uint32_t ka = (s / 4) * S::kTile + (s % 4) * 32;
                    ssd_mma(tYd, ssd_desc((part ? a_mlo : a_mhi) + ka, 16, 1024), ssd_desc(a_x + 2048 * s, S::kTile, 1024),
                            i2, part > 0 || s > 0);
                }
            for (int part = 0; part < 2; ++part)
                for (int s = 0; s < 8; ++s)
                    ssd_mma(tST, ssd_desc((part ? a_bwlo : a_b) + 2048 * s, S::kTile, 1024),
                            ssd_desc(a_x + 2048 * s, S::kTile, 1024), i4, part > 0 || s > 0);
            ssd_commit(bar + 1);
        }
        if (!__syncthreads_and(ssd_wait(bar + 1, static_cast<uint32_t>(c & 1), p.error))) {
            ok = false;
            break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // ---- epilogue 2: y row i; state row n
        {
            const int i = tid;
            const int64_t t = t0 + i;
            const float ecs = __expf(cs[i]);
            uint16_t *yg = static_cast<uint16_t *>(p.y);
            for (int q0 = 0; q0 < kSsdP; q0 += 16) {
                float yd[16], yo[16];
                ssd_ld16(tYd + lane_off + q0, yd);
                ssd_ld16(tYo + lane_off + q0, yo);
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    const float x0 = __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<uint16_t *>(sm + S::kX + ssd_sw128(i, q0 + e))) << 16);
                    const float x1 = __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<uint16_t *>(sm + S::kX + ssd_sw128(i, q0 + e + 1))) << 16);
                    pk[e / 2] = pack_bf16x2(fmaf(ecs, yo[e], yd[e]) + Dh * x0, fmaf(ecs, yo[e + 1], yd[e + 1]) + Dh * x1);
                }
                if (t < L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(yg + ((b * L + t) * H + h) * kSsdP + q0);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            const float et = __expf(total);
            for (int q0 = 0; q0 < kSsdP; q0 += 16) {
                float v[16];
                ssd_ld16(tST + lane_off + q0, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) st[q0 + e] = fmaf(et, st[q0 + e], v[e]);
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    }
    if (p.h_last && ok) {
#pragma unroll
        for (int q = 0; q < kSsdP; ++q) p.h_last[((b * H + h) * kSsdP + q) * kSsdN + tid] = st[q];
    }
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tbase));
}

}  // namespace ssm
