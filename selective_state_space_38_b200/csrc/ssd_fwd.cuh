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
//   S_out  = exp(cs_{Q-1}) S_in + B^T (w o X),   w_j = exp(cs_{Q-1} - cs_j) dt_j
// A CTA walks the chunks of whole sequences in order, and may begin with the
// start of one more sequence and end with the rest of another, whose state
// passes between the two CTAs through global memory (SsdRange); the state S
// (P x N float32) stays in registers, spread over the 256 threads.  Per chunk:
//   MMA1 G = C B^T (128 x 128 x 128) and MMA3 Yo = C S_in^T (128 x 64 x 128);
//   epilogue 1 forms L o G from G in tensor memory and writes it back there as
//   bf16 (the A operand of MMA2), and w o X into shared memory;
//   MMA2 Yd = (L o G) X (128 x 64 x 128) and MMA4 ST = B^T (w o X) (128 x 64 x 128);
//   epilogue 2 writes y and updates the state.
// Operands are bf16 in the 128-byte-swizzled canonical layouts; the ones that
// are products (L o G, w o X, S) are split into a bf16 high part and a low part,
// so they keep about 16 bits: the two parts of S^T and of w o X form one N = 128
// operand (the low tile is its second 64-column atom), L o G's two parts two
// MMAs, and each product's halves land side by side in TMEM and are added in
// the epilogue.  C, B and X arrive by TMA into one of two buffers, the next
// chunk's while this one is computed.  Single threads issue the MMAs (MMA2's
// halves and MMA4 from three threads at once); tcgen05.commit arrives on one
// mbarrier per MMA group that every thread waits on (bounded); each thread reads
// its TMEM lane with tcgen05.ld.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace ssm {

constexpr int kSsdQ = 128;  // chunk length
constexpr int kSsdP = 64;   // head dimension
constexpr int kSsdN = 128;  // state dimension
constexpr int kSsdConsumers = 256;               // epilogue threads (8 warps)
constexpr int kSsdThreads = kSsdConsumers + 32;  // + the producer warp
constexpr uint32_t kSsdWaitLimit = 1u << 24;
constexpr uint32_t kSsdFlagLimit = 1u << 20;  // polls of a hand-off flag, 64 ns apart at least

// TMA maps, rank 4 with the innermost dimension first: x [P][H][L][batch],
// B and C [N][G][L][batch]; every box is 64 elements x 1 x 128 steps x 1.
struct SsdMaps {
    CUtensorMap x, B, C;
};

struct SsdParams {
    const void *dt;              // [b][L][H] bf16
    const float *dt_bias, *A, *D, *h0;
    void *y;                     // [b][L][H][P] bf16
    float *h_last;               // [b][H][P][N]
    uint32_t *error;             // bounded-wait failure word
    // Split sequences (all three set, or none): the CTAs' order of start (a
    // counter), one flag and one P x N state per hand-off between two CTAs.
    uint32_t *order, *flags;
    float *slots;
    int64_t batch, seqlen, heads, groups;
    int64_t units_per_cta;       // chunks a CTA walks (the chunk count of a sequence without splits)
    uint32_t flag_want;          // a hand-off flag is set when it reaches this (1; larger: test support)
    uint32_t spin_limit;         // polls of a hand-off flag before the wait gives up
    int softplus;
};

// The chunks a CTA walks.  The batch * heads sequences, chunk by chunk, form one
// list of units; CTA k (in the order the CTAs start) owns units [k W, k W + W).
// With W at least one sequence's chunk count, such a range is: the end of one
// sequence (its "tail"), whole sequences, and the start of another (its
// "head").  The CTA walks the head first, hands its state on to CTA k + 1, then
// the whole sequences, and the tail last, from the state CTA k - 1 handed on
// at the end of its own head, which it walked first: no CTA waits on one that
// started after it.
// One unit of a CTA's walk: its sequence (batch b, head h, group g) and chunk;
// whether it starts a part, ends one, and whether that end is the hand-off.
struct SsdUnit {
    int seq, c, b, h, g;  // below 2^31: batch * heads and the chunk count are checked on the host
    bool first, last, handoff;
};

struct SsdRange {
    int64_t chunks;            // chunks per sequence
    int64_t head, full, tail;  // units in each part (full: whole sequences x chunks)
    int64_t head_seq, first_full, tail_seq, tail_chunk;
    int64_t heads, per_group;
    __device__ SsdRange(int64_t k, int64_t W, int64_t nseq, int64_t C, int64_t H, int64_t HG)
        : chunks(C), heads(H), per_group(HG) {
        const int64_t s0 = k * W, e0 = min(s0 + W, nseq * C);
        tail_chunk = s0 % C;
        tail_seq = s0 / C;
        head = e0 % C;
        head_seq = e0 / C;
        first_full = tail_chunk == 0 ? tail_seq : tail_seq + 1;
        full = (e0 / C - first_full) * C;
        tail = tail_chunk == 0 ? 0 : C - tail_chunk;
    }
    __device__ int64_t units() const { return head + full + tail; }
    __device__ void set(SsdUnit &x, int64_t u, int64_t seq, int64_t c, bool new_seq) const {
        if (new_seq) {
            const int64_t bb = seq / heads;
            x.b = static_cast<int>(bb);
            x.h = static_cast<int>(seq - bb * heads);
            x.g = static_cast<int>(x.h / per_group);
        }
        x.seq = static_cast<int>(seq);
        x.c = static_cast<int>(c);
        x.first = c == 0 || (tail > 0 && u == head + full);
        x.last = c == chunks - 1 || u == head - 1;
        x.handoff = u < head;
    }
    __device__ SsdUnit first_unit() const {
        SsdUnit x;
        if (head > 0) set(x, 0, head_seq, 0, true);
        else if (full > 0) set(x, 0, first_full, 0, true);
        else set(x, 0, tail_seq, tail_chunk, true);
        return x;
    }
    // x (unit u) becomes unit u + 1, without a division unless the sequence changes
    __device__ void advance(SsdUnit &x, int64_t u) const {
        const int64_t v = u + 1;
        if (v == head) {
            if (full > 0) set(x, v, first_full, 0, true);
            else set(x, v, tail_seq, tail_chunk, true);
        } else if (v == head + full) {
            set(x, v, tail_seq, tail_chunk, true);
        } else if (x.c + 1 == chunks) {
            set(x, v, x.seq + 1, 0, true);
        } else {
            set(x, v, x.seq, x.c + 1, false);
        }
    }
};
// Shared memory (1024-byte aligned pieces; every operand tile is [128 rows][64]
// bf16 with 128-byte rows and the 128-byte swizzle).
struct SsdSmem {
    static constexpr int kTile = 128 * 128;        // one tile, 16 KB
    static constexpr int kInC = 0;                 // C [t][n]: 2 tiles (n < 64, n >= 64)
    static constexpr int kInB = 2 * kTile;         // B [t][n]: 2 tiles
    static constexpr int kInX = 4 * kTile;         // X [t][p]: 1 tile
    static constexpr int kInBytes = 5 * kTile;     // one input buffer (two of them)
    static constexpr int kXw = 2 * kInBytes;       // w o X [t][p]: high tile, low tile
    static constexpr int kS = kXw + 2 * kTile;     // S^T [n][p]: high tile, low tile
    static constexpr int kCs = kS + 2 * kTile;     // cs[128], dt[128], F[128], warp sums[4]
    static constexpr int kBar = kCs + 1600;        // load[2], mma[5], TMEM base, CTA order (64 bytes)
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

// D (TMEM) (+)= A (shared memory) B (shared memory)
__device__ __forceinline__ void ssd_mma(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

// D (TMEM) (+)= A (TMEM: lane = row, two bf16 per column, lower index in the
// low half) B (shared memory)
__device__ __forceinline__ void ssd_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t db, uint32_t idesc,
                                           uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
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

// 16 consecutive 32-bit columns of this thread's TMEM lane from registers
__device__ __forceinline__ void ssd_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// 4-D tiled TMA load of a box at (c0, c1, c2, c3); completion as bytes on the mbarrier.
__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, int c0, int c1, int c2, int c3,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool ssd_try(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for a phase of an mbarrier; gives up early once another wait
// of the launch has given up (the error word is non-zero).
__device__ __forceinline__ bool ssd_wait(uint64_t *bar, uint32_t parity, uint32_t *error) {
    const uint32_t addr = smem_u32(bar);
    for (uint32_t n = 0; n < kSsdWaitLimit; ++n) {
        if (ssd_try(addr, parity)) return true;
        if ((n & 1023u) == 1023u && *reinterpret_cast<volatile uint32_t *>(error) != 0) return false;
    }
    atomicOr(error, 2u);
    return false;
}
// The same wait before the CTA may exit with a load or an MMA in flight: it does
// not stop early on the error word.
__device__ __forceinline__ void ssd_drain(uint64_t *bar, uint32_t parity, uint32_t *error) {
    const uint32_t addr = smem_u32(bar);
    for (uint32_t n = 0; n < kSsdWaitLimit; ++n)
        if (ssd_try(addr, parity)) return;
    atomicOr(error, 2u);
}

// v = hi + lo with hi = bf16(v) and lo = bf16(v - hi), for two values at once:
// the high parts and the low parts as bf16 pairs (first value in the low half).
__device__ __forceinline__ void split_pair(float a, float b, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16x2(a, b);
    lo = pack_bf16x2(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

// Barrier 1 among the kSsdConsumers epilogue threads (the producer warp is not
// part of it): a plain sync, and one that returns the AND of a predicate.
__device__ __forceinline__ void ssd_cbar() { asm volatile("bar.sync 1, %0;" ::"n"(kSsdConsumers) : "memory"); }
__device__ __forceinline__ bool ssd_cbar_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.cta.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(kSsdConsumers)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void ssd_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// grid: one CTA per range of units (SsdRange); block: kSsdConsumers epilogue
// threads and one producer warp.  Epilogue thread (quad, half, lane) owns row
// 32 quad + lane of every [128][..] tile (its TMEM lane) and the half `half` of
// that row's columns.  One lane of the producer warp issues every TMA load and
// every MMA; the epilogue threads hand it their results through two mbarriers
// (epilogue 1 done; the next unit's S^T in shared memory) and wait for its
// commits, so no epilogue thread is held while the tensor core takes an MMA.
__global__ void __launch_bounds__(kSsdThreads, 1)
    ssd_fwd_kernel(const SsdParams p, const __grid_constant__ SsdMaps tm) {
    extern __shared__ __align__(1024) uint8_t ssd_smem_raw[];
    uint8_t *sm = ssd_smem_raw + ((1024u - (smem_u32(ssd_smem_raw) & 1023u)) & 1023u);
    using S = SsdSmem;
    float *cs = reinterpret_cast<float *>(sm + S::kCs);
    float *dts = cs + 128;
    float *Fs = dts + 128;  // F_j = exp(-cs_j) dt_j, when every |cs| of the chunk is at most 80
    float *wsum = Fs + 128;
    uint64_t *lbar = reinterpret_cast<uint64_t *>(sm + S::kBar);  // [2] input buffer landed
    uint64_t *mG = lbar + 2, *mYo = lbar + 3, *m24 = lbar + 4;    // MMA1; MMA3; MMA2 and MMA4 done
    uint64_t *cE1 = lbar + 5, *cS = lbar + 6;  // epilogue 1 done; S^T of a unit ready (kSsdConsumers arrivals)
    uint32_t *tslot = reinterpret_cast<uint32_t *>(lbar + 7);
    uint32_t *korder = tslot + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool producer = tid >= kSsdConsumers;
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int row = quad * 32 + lane;
    const int64_t L = p.seqlen, H = p.heads, per_group = p.heads / p.groups;
    const int64_t chunks = (L + kSsdQ - 1) / kSsdQ;

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(lbar + i)));
        for (int i = 5; i < 7; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(lbar + i)), "n"(kSsdConsumers));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        // with split sequences a CTA's range is its place in the order of start
        *korder = p.order ? atomicAdd(p.order, 1u) : blockIdx.x;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tslot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(tslot);
    const int64_t kcta = *reinterpret_cast<volatile uint32_t *>(korder);
    const SsdRange rg(kcta, p.units_per_cta, p.batch * H, chunks, H, per_group);
    const int64_t units = rg.units();
    // TMEM columns: G then L o G (128); Yd and Yo (64 each: the products of the
    // high and the low operand parts accumulated, in issue order); ST (128: the
    // products with w o X high and low side by side, one N = 128 MMA); the
    // carried state S (64: lane n holds S[p][n] in column p)
    const uint32_t tG = tbase, tYd = tbase + 128, tYo = tbase + 192, tST = tbase + 256, tS = tbase + 384;
    const uint32_t a_s = smem_u32(sm + S::kS), a_xw = smem_u32(sm + S::kXw);

    if (producer) {
        if (lane == 0 && units > 0) {
            // the inputs of unit u (x) into buffer u & 1
            auto load = [&](const SsdUnit &x, int64_t u) {
                uint8_t *in = sm + (u & 1) * S::kInBytes;
                uint64_t *bar = lbar + (u & 1);
                mbar_arrive_expect_tx(bar, S::kInBytes);
                const int t0 = static_cast<int>(x.c * kSsdQ), bi = static_cast<int>(x.b), gi = static_cast<int>(x.g);
                tma_load_4d(in + S::kInC, &tm.C, 0, gi, t0, bi, bar);
                tma_load_4d(in + S::kInC + S::kTile, &tm.C, 64, gi, t0, bi, bar);
                tma_load_4d(in + S::kInB, &tm.B, 0, gi, t0, bi, bar);
                tma_load_4d(in + S::kInB + S::kTile, &tm.B, 64, gi, t0, bi, bar);
                tma_load_4d(in + S::kInX, &tm.x, 0, static_cast<int>(x.h), t0, bi, bar);
            };
            // a descriptor of base + off is the base's plus off / 16 (no carry: every
            // shared-memory address is below 2^18)
            SsdUnit x1 = rg.first_unit();  // the unit whose inputs are loaded next
            int64_t loads = 0, loads_waited = 0, nG = 0, nYo = 0, n24 = 0, w24 = 0;
            auto issue_g = [&](int64_t u) {  // MMA1: G = C B^T of unit u
                uint8_t *in = sm + (u & 1) * S::kInBytes;
                constexpr uint32_t i1 = ssd_idesc(128, 128, 0, 0);
                const uint64_t dC = ssd_desc(smem_u32(in + S::kInC), 16, 1024),
                               dB = ssd_desc(smem_u32(in + S::kInB), 16, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ko = ((k / 4) * S::kTile + (k % 4) * 32) >> 4;
                    ssd_mma(tG, dC + ko, dB + ko, i1, k > 0);
                }
                ssd_commit(mG);
                nG = u + 1;
            };
            load(x1, 0);
            loads = 1;
            if (units > 1) rg.advance(x1, 0);
            bool pok = ssd_wait(lbar, 0u, p.error);
            if (pok) {
                loads_waited = 1;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                issue_g(0);
            }
            for (int64_t u = 0; pok && u < units; ++u) {
                const uint32_t ph = static_cast<uint32_t>(u & 1);
                uint8_t *in = sm + (u & 1) * S::kInBytes;
                // S^T of unit u is written, and the previous unit's epilogue 2 is done
                // with Yo, Yd, ST and its X: the other buffer takes unit u + 1's
                // inputs (the tensor core read them before MMA2/MMA4 of the previous
                // unit completed)
                if (!ssd_wait(cS, ph, p.error)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (u + 1 < units) {
                    load(x1, u + 1);
                    loads = u + 2;
                    if (u + 2 < units) rg.advance(x1, u + 1);
                }
                // MMA3: Yo = C S^T, the high tile then the low one accumulated
                {
                    constexpr uint32_t i3 = ssd_idesc(128, 64, 0, 1);
                    const uint64_t dC = ssd_desc(smem_u32(in + S::kInC), 16, 1024), dS = ssd_desc(a_s, S::kTile, 1024);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint32_t ka = ((k / 4) * S::kTile + (k % 4) * 32) >> 4;
                            ssd_mma(tYo, dC + ka, dS + ((part * S::kTile + 2048 * k) >> 4), i3, part > 0 || k > 0);
                        }
                    ssd_commit(mYo);
                    nYo = u + 1;
                }
                // MMA2: Yd = (L o G) X, A from TMEM, the high part then the low one
                // accumulated; MMA4: ST = B^T [w o X high | w o X low] (N = 128: the low
                // tile is the operand's second 64-column atom); once epilogue 1 is done
                if (!ssd_wait(cE1, ph, p.error)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                {
                    constexpr uint32_t i2 = ssd_idesc(128, 64, 0, 1), i4 = ssd_idesc(128, 128, 1, 1);
                    const uint64_t dX = ssd_desc(smem_u32(in + S::kInX), S::kTile, 1024);
                    const uint64_t dBt = ssd_desc(smem_u32(in + S::kInB), S::kTile, 1024),
                                   dXw = ssd_desc(a_xw, S::kTile, 1024);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            // K step k covers j in [16 k, 16 k + 16): column half k / 4,
                            // 32-column block (k % 4) / 2, high or low 16 columns, 8
                            // columns per 16 j
                            const uint32_t acol = 64 * (k / 4) + 32 * ((k % 4) / 2) + 16 * part + 8 * (k % 2);
                            ssd_mma_ts(tYd, tG + acol, dX + ((2048 * k) >> 4), i2, part > 0 || k > 0);
                        }
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        ssd_mma(tST, dBt + ((2048 * k) >> 4), dXw + ((2048 * k) >> 4), i4, k > 0);
                    ssd_commit(m24);
                    n24 = u + 1;
                }
                // the next unit's G once MMA2 has read L o G out of its columns (it
                // runs during this unit's epilogue 2)
                if (u + 1 < units) {
                    if (!ssd_wait(m24, ph, p.error)) break;
                    w24 = u + 1;
                    if (!ssd_wait(lbar + ((u + 1) & 1), static_cast<uint32_t>(((u + 1) >> 1) & 1), p.error)) break;
                    loads_waited = u + 2;
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    issue_g(u + 1);
                }
            }
            // nothing in flight when the CTA ends (at most the newest phase of each
            // commit barrier is open: the tensor core completes MMAs in order, and
            // G(u + 1) is issued after MMA2/MMA4(u) are done)
            if (nG > 0) ssd_drain(mG, static_cast<uint32_t>((nG - 1) & 1), p.error);
            if (nYo > 0) ssd_drain(mYo, static_cast<uint32_t>((nYo - 1) & 1), p.error);
            if (n24 > w24) ssd_drain(m24, static_cast<uint32_t>((n24 - 1) & 1), p.error);
            for (int64_t c = loads_waited; c < loads; ++c)
                ssd_drain(lbar + (c & 1), static_cast<uint32_t>((c >> 1) & 1), p.error);
        }
        __syncwarp();
    } else {
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        // raw dt of this thread's step of unit x (zero past the end)
        auto load_dt = [&](const SsdUnit &x) -> float {
            const int64_t t = x.c * kSsdQ + tid;
            return t < L ? Act<bf16raw>::load(p.dt, (x.b * L + t) * H + x.h) : 0.0f;
        };

        // This thread's share of the state, S[p][n] for n = row and p in [32 half,
        // 32 half + 32), lives in its TMEM lane, columns tS + p; it moves through
        // registers 16 values at a time.
        const uint32_t t_s = tS + lane_off + 32 * half;
        auto put_state = [&](int q0, const float (&v)[16]) {
            uint32_t r[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(v[e]);
            ssd_st16(t_s + q0, r);
        };
        // S^T [n][p] high and low tiles, columns q0 .. q0 + 15 of this thread's half
        auto put_state_tiles = [&](int q0, const float (&v)[16]) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) split_pair(v[8 * k + 2 * e], v[8 * k + 2 * e + 1], hi[e], lo[e]);
                const uint32_t o = ssd_sw128(row, 32 * half + q0 + 8 * k);
                *reinterpret_cast<uint4 *>(sm + S::kS + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(sm + S::kS + S::kTile + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        };
        // S^T of the state in TMEM to shared memory; then the producer may issue MMA3
        auto write_state = [&]() {
#pragma unroll
            for (int q0 = 0; q0 < 32; q0 += 16) {
                float v[16];
                ssd_ld16(t_s + q0, v);
                put_state_tiles(q0, v);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            ssd_arrive(cS);
        };
        // the state a part starts from: h0 (or zero) at a sequence start, else the
        // one the previous CTA handed on (a bounded wait on its flag); into TMEM
        auto begin_part = [&](int64_t seq, int64_t c) -> bool {
            const float *src = nullptr;
            if (c == 0) {
                src = p.h0 ? p.h0 + seq * kSsdP * kSsdN : nullptr;
            } else {
                bool got = true;
                if (tid == 0) {
                    got = false;
                    const uint32_t *flag = p.flags + (kcta - 1);
                    for (uint32_t n = 0; n < p.spin_limit; ++n) {
                        if (ld_acquire(flag) >= p.flag_want) {
                            got = true;
                            break;
                        }
                        if ((n & 255u) == 255u && *reinterpret_cast<volatile uint32_t *>(p.error) != 0) break;
                        __nanosleep(64);
                    }
                    if (!got && *reinterpret_cast<volatile uint32_t *>(p.error) == 0) atomicOr(p.error, 2u);
                }
                if (!ssd_cbar_and(got)) return false;
                src = p.slots + (kcta - 1) * (kSsdP * kSsdN);
            }
#pragma unroll
            for (int q0 = 0; q0 < 32; q0 += 16) {
                float v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = src ? __ldcg(src + (32 * half + q0 + e) * kSsdN + row) : 0.0f;
                put_state(q0, v);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            return true;
        };
        // the state at the end of a part (from TMEM): h_last at a sequence end, else
        // to this CTA's hand-off slot, then its flag (release)
        auto end_part = [&](int64_t seq, bool handoff) {
            float *dst = handoff ? p.slots + kcta * (kSsdP * kSsdN) : p.h_last ? p.h_last + seq * kSsdP * kSsdN : nullptr;
            if (dst) {
#pragma unroll
                for (int q0 = 0; q0 < 32; q0 += 16) {
                    float v[16];
                    ssd_ld16(t_s + q0, v);
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[(32 * half + q0 + e) * kSsdN + row] = v[e];
                }
            }
            if (handoff) {
                ssd_cbar();
                if (tid == 0) {
                    __threadfence();
                    st_release(p.flags + kcta, 1u);
                }
            }
        };
        // the running sums of unit x's chunk: first dt and the running sum within
        // each warp (threads 0..127; the warp's total to wsum), then, after a
        // barrier, the sums of the warps before it; cs, dt and F to their tables.
        // Returns whether this thread's |cs| is at most 80 (threads 128.. true).
        float s = 0.0f, dtv = 0.0f;
        auto sums_in_warp = [&](const SsdUnit &x, float raw, float bias_x, float A_x) {
            if (tid < kSsdQ) {
                dtv = 0.0f;
                if (static_cast<int64_t>(x.c) * kSsdQ + tid < L) {
                    const float v = raw + bias_x;
                    dtv = p.softplus ? softplus_fast(v) : v;
                }
                s = dtv * A_x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float o = __shfl_up_sync(0xffffffffu, s, off);
                    if (lane >= off) s += o;
                }
                if (lane == 31) wsum[warp] = s;
            }
        };
        auto sums_across_warps = [&]() -> bool {
            if (tid >= kSsdQ) return true;
            for (int w = 0; w < warp; ++w) s += wsum[w];
            cs[tid] = s;
            dts[tid] = dtv;
            Fs[tid] = __expf(-s) * dtv;
            return fabsf(s) <= 80.0f;
        };

        // Per unit u: cur is unit u, nxt unit u + 1, nn unit u + 2 (whose dt is
        // loaded while u runs); the cs tables hold unit u's, and unit u + 1's are
        // formed while u's MMA2 and MMA4 run (epilogue 2 keeps what it needs in
        // registers).
        SsdUnit cur = rg.first_unit(), nxt = cur;
        if (units > 1) rg.advance(nxt, 0);
        bool ok = units > 0;
        // the head's A, dt bias and D (the next unit's are loaded a unit ahead)
        float Ah = 0.0f, bias = 0.0f, Dh = 0.0f;
        float dt_raw = 0.0f;
        bool factored = true;  // every |cs| of the chunk at most 80: exp(cs_i - cs_j) = exp(cs_i) exp(-cs_j)
        if (ok) {
            Ah = p.A[cur.h];
            bias = p.dt_bias ? p.dt_bias[cur.h] : 0.0f;
            Dh = p.D ? p.D[cur.h] : 0.0f;
            if (tid < kSsdQ) dt_raw = load_dt(cur);
            ok = begin_part(cur.seq, cur.c);
            if (ok) write_state();
            sums_in_warp(cur, dt_raw, bias, Ah);
            if (units > 1 && tid < kSsdQ) dt_raw = load_dt(nxt);
            ssd_cbar();
            factored = ssd_cbar_and(sums_across_warps());
        }
        for (int64_t u = 0; ok && u < units; ++u) {
            SsdUnit nn = nxt;
            if (u + 2 < units) rg.advance(nn, u + 1);
            float nAh = Ah, nbias = bias, nDh = Dh;
            if (u + 1 < units && nxt.h != cur.h) {
                nAh = p.A[nxt.h];
                nbias = p.dt_bias ? p.dt_bias[nxt.h] : 0.0f;
                nDh = p.D ? p.D[nxt.h] : 0.0f;
            }
            const int64_t b = cur.b, h = cur.h, c = cur.c;
            const int64_t t0 = c * kSsdQ;
            const uint32_t ph = static_cast<uint32_t>(u & 1);
            uint8_t *in = sm + (u & 1) * S::kInBytes;
            // G of this unit, and its inputs (X for epilogue 1)
            if (!ssd_cbar_and(ssd_wait(mG, ph, p.error) &&
                              ssd_wait(lbar + (u & 1), static_cast<uint32_t>((u >> 1) & 1), p.error))) {
                ok = false;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const float total = cs[kSsdQ - 1];
        float ecs;     // exp(cs) of this thread's row, kept for epilogue 2
        {
            // ---- epilogue 1a: row i of L o G, columns j in [64 half, 64 half + 64), 32
            // at a time: read their G, then write the high parts to the first 16 and
            // the low parts to the last 16 of the same 32 TMEM columns (two bf16 each)
            const int i = row;
            const float csi = cs[i], Ei = __expf(csi);
            ecs = Ei;
#pragma unroll 1
            for (int jp = 0; jp < 2; ++jp) {
                const uint32_t col = tG + lane_off + 64 * half + 32 * jp;
                float v[32];
                {
                    float v0[16], v1[16];
                    ssd_ld16(col, v0);
                    ssd_ld16(col + 16, v1);
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = v0[e], v[16 + e] = v1[e];
                }
                uint32_t mh[16], ml[16];
                const int j0 = 64 * half + 32 * jp;
                if (factored) {
                    const float4 *F4 = reinterpret_cast<const float4 *>(Fs + j0);
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 f = F4[e / 4];
                        const float m0 = j0 + e <= i ? v[e] * (Ei * f.x) : 0.0f;
                        const float m1 = j0 + e + 1 <= i ? v[e + 1] * (Ei * f.y) : 0.0f;
                        const float m2 = j0 + e + 2 <= i ? v[e + 2] * (Ei * f.z) : 0.0f;
                        const float m3 = j0 + e + 3 <= i ? v[e + 3] * (Ei * f.w) : 0.0f;
                        split_pair(m0, m1, mh[e / 2], ml[e / 2]);
                        split_pair(m2, m3, mh[e / 2 + 1], ml[e / 2 + 1]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int j = j0 + e;
                        const float m0 = j <= i ? v[e] * __expf(csi - cs[j]) * dts[j] : 0.0f;
                        const float m1 = j + 1 <= i ? v[e + 1] * __expf(csi - cs[j + 1]) * dts[j + 1] : 0.0f;
                        split_pair(m0, m1, mh[e / 2], ml[e / 2]);
                    }
                }
                ssd_st16(col, mh);
                ssd_st16(col + 16, ml);
            }
            // ---- epilogue 1b: row t of w o X (high and low tiles), p in [32 half, 32 half + 32)
            const int t = row;
            const float w = __expf(total - cs[t]) * dts[t];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t o = ssd_sw128(t, 32 * half + 8 * k);
                const uint4 xv = *reinterpret_cast<const uint4 *>(in + S::kInX + o);
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = __uint_as_float(xw[e] << 16), x1 = __uint_as_float(xw[e] & 0xffff0000u);
                    split_pair(w * x0, w * x1, hi[e], lo[e]);
                }
                *reinterpret_cast<uint4 *>(sm + S::kXw + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(sm + S::kXw + S::kTile + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        ssd_arrive(cE1);
        // ---- meanwhile the next unit's running sums (its dt loaded a unit ago),
        // once every epilogue thread is done with this unit's tables
        ssd_cbar();
        if (u + 1 < units) {
            sums_in_warp(nxt, dt_raw, nbias, nAh);
            if (u + 2 < units && tid < kSsdQ) dt_raw = load_dt(nn);
        }
        ssd_cbar();
        const bool fac_next = u + 1 < units ? sums_across_warps() : true;
        bool factored_next = true;
        {
            // Yo, Yd and ST of this unit, and whether every |cs| of the next unit is
            // at most 80, in one barrier (two more only when that is not so)
            const bool w = ssd_wait(mYo, ph, p.error) && ssd_wait(m24, ph, p.error);
            if (!ssd_cbar_and(w && fac_next)) {
                factored_next = ssd_cbar_and(fac_next);
                if (!ssd_cbar_and(w)) {
                    ok = false;
                    break;
                }
            }
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // ---- epilogue 2: y row i, p in [32 half, 32 half + 32); state row n, same p
        {
            const int i = row;
            const int64_t t = t0 + i;
            uint16_t *yg = static_cast<uint16_t *>(p.y);
#pragma unroll
            for (int q0 = 0; q0 < 32; q0 += 16) {
                float yd[16], yo[16];
                ssd_ld16(tYo + lane_off + 32 * half + q0, yo);
                ssd_ld16(tYd + lane_off + 32 * half + q0, yd);
                // D x of the row's 16 columns, from the X tile (not overwritten before
                // this unit's epilogue 2 is done)
                float dx[16];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(in + S::kInX + ssd_sw128(i, 32 * half + q0 + 8 * k));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        dx[8 * k + 2 * e] = Dh * __uint_as_float(xw[e] << 16);
                        dx[8 * k + 2 * e + 1] = Dh * __uint_as_float(xw[e] & 0xffff0000u);
                    }
                }
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2)
                    pk[e / 2] = pack_bf16x2(fmaf(ecs, yo[e], yd[e]) + dx[e],
                                            fmaf(ecs, yo[e + 1], yd[e + 1]) + dx[e + 1]);
                if (t < L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(yg + ((b * L + t) * H + h) * kSsdP + 32 * half + q0);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            // S <- exp(cs_last) S + ST, in TMEM
            const float et = __expf(total);
#pragma unroll
            for (int q0 = 0; q0 < 32; q0 += 16) {
                float v[16], sv[16];
                ssd_ld16(tST + lane_off + 32 * half + q0, v);
                ssd_ld16(tST + 64 + lane_off + 32 * half + q0, sv);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] += sv[e];
                ssd_ld16(t_s + q0, sv);
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[e] = fmaf(et, sv[e], v[e]);
                put_state(q0, sv);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }
        // the end of a part (h_last, or the hand-off to the next CTA); the state the
        // next unit starts from, as MMA3's operand
        if (cur.last) end_part(cur.seq, cur.handoff);
        if (u + 1 < units) {
            if (nxt.first && !begin_part(nxt.seq, nxt.c)) {
                ok = false;
                break;
            }
            write_state();
        }
        cur = nxt;
        nxt = nn;
        Ah = nAh;
        bias = nbias;
        Dh = nDh;
        factored = factored_next;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tbase));
}

}  // namespace ssm
