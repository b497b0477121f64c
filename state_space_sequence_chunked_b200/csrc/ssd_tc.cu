// Fused chunked SSD forward on 5th-generation tensor cores (tcgen05, sm_100a).
//
// One CTA owns one (batch row b, head h) stream and walks its blocks of 128 tokens
// in order, so x is read once, y is written once and the running state never
// leaves the SM. Per block (the four steps of "SSD 算法：分块和状态传递" in the
// Mamba-2 SSD write-up, with the block decomposition of "SSD 算法：分块矩阵分解"):
//   step 0  A_cs[l] = sum_{j<=l} dt_j A_h            (within the block, log2 domain)
//   step 1  G = C B^T on tensor cores (TMEM), then G'[l,s] = G[l,s] exp(A_cs[l]-A_cs[s]) dt_s
//           for s <= l (0 above the diagonal), written back to TMEM as bf16, and
//           Y_diag = G' X on tensor cores with G' as the TMEM A operand
//   step 2  dS^T = B^T X' on tensor cores, X'[s,:] = exp(A_cs[127]-A_cs[s]) dt_s x_s
//   step 3  S <- exp(A_cs[127]) S + dS                 (fp32, registers)
//   step 4  Y_off = C S_in^T on tensor cores (S_in in bf16 shared memory), and
//           y = Y_diag + exp(A_cs[l]) Y_off + D_h x
// A chunk argument of 256 is evaluated as two 128-token diagonal blocks; the
// 128x128 block between them goes through the state (its low-rank factor), which
// is the same matrix product re-associated.
//
// Warp roles (320 threads): warp 0 loads (TMA + dt), warp 1 owns TMEM and issues
// every MMA from one thread, warps 2-5 ("T") do step 0, X' and G', warps 6-9
// ("E") run the state chain and the epilogue. Every wait is bounded: on timeout
// the CTA raises a status word in the workspace, drains its own TMA loads and
// MMAs, frees TMEM and returns.
#include <cuda.h>

#include "ssd_internal.cuh"

namespace ssd {
namespace tc {

constexpr int kQ = 128;  // tokens per diagonal block
constexpr int kP = 64;   // head dimension handled by this path
constexpr int kThreads = 320;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpT = 2, kWarpE = 6;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait

template <int N>
struct Cfg {
    // N = 128: double-buffered input stages, Y accumulators and S^T; the chunk state
    // accumulates in the half of the score buffer that the packed G' leaves free.
    // N = 256: the wider state takes the room of the second buffers.
    static constexpr bool kWide = N == 256;
    static constexpr int kStages = kWide ? 1 : 2;
    static constexpr int kYBufs = kWide ? 1 : 2;
    static constexpr int kStBufs = kWide ? 1 : 2;
    static constexpr bool kDsInG = !kWide;
    static constexpr bool kXInRegs = !kWide;  // epilogue keeps its x row in registers
    static constexpr int kPanels = N / 64;           // 64-column panels of B and C
    static constexpr int kPanelBytes = kQ * 128;     // 128 rows x 128 B
    static constexpr int kCBytes = kPanels * kPanelBytes;
    static constexpr int kXBytes = kQ * 128;         // 128 rows x 64 bf16
    static constexpr int kStageBytes = 2 * kCBytes + kXBytes;  // C, B, X
    static constexpr int kStBytes = N * 128;                   // S^T bf16 [N][64]
    static constexpr int kOffXp = kStages * kStageBytes;
    static constexpr int kOffSt = kOffXp + kXBytes;
    static constexpr int kOffSmall = kOffSt + kStBufs * kStBytes;
    static constexpr int kOffDts = kOffSmall;                       // float [kStages][128]
    static constexpr int kOffAcsT = kOffDts + kStages * kQ * 4;     // float [4 warps][128]
    static constexpr int kOffCfT = kOffAcsT + 4 * kQ * 4;           // float [4 warps][128]
    static constexpr int kOffBar = kOffCfT + 4 * kQ * 4;            // uint64 barriers
    static constexpr int kNumBars = 2 * kStages + 11 + kStBufs + 2 * kYBufs;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;         // tmem base, abort flag
    static constexpr int kSmemBytes = kOffMisc + 16;
    static constexpr int kSmemAlloc = kSmemBytes + 1024;            // slack for 1024-B alignment
    // TMEM columns: score buffers j at 128 j; Y buffer i at 256 + 128 i (Y_diag, then Y_off
    // at +64); the chunk state inside score buffer j at 128 j + 64, or (wide) at 384.
    static constexpr int kTmY = 256;
    static constexpr int kTmCols = 512;
    static_assert(kSmemAlloc <= 232448, "shared memory budget");
    static constexpr uint32_t kTxBytes = kStageBytes;
};

struct Params {
    const __nv_bfloat16 *dt;
    const float *A, *D, *h0;
    float *h_final;
    __nv_bfloat16 *y;
    int *status;
    long long L;
    int H, G, nc;
};

// ---------------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on a barrier phase. Returns false (and raises the abort flag and the
// status word) when the phase does not complete within kWaitNs or another thread of
// the CTA has already aborted.
__device__ __noinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                        int *status) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = now_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (now_ns() - t0 > kWaitNs) {
                *abort_flag = 1;
                atomicOr(status, 1);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 format: version 1).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 operands and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(id), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

#define SSD_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                  "=r"(r[i + 6]), "=r"(r[i + 7])
// 32 consecutive columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : SSD_R8(0), SSD_R8(8), SSD_R8(16), SSD_R8(24)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : SSD_R8(0)
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : SSD_R8(0), SSD_R8(8)
        : "r"(taddr));
}
#undef SSD_R8
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled tile (128 B rows).
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// Warp-uniform bounded wait: every lane polls (each gets the acquire), and the
// warp agrees on the outcome, so a timeout never leaves part of a warp behind
// at a warp-collective instruction. Call only from warp-uniform control flow.
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status) {
    const bool ok = wait_phase(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}

// Within-block inclusive cumsum of dts[i] * a2, i = 0..127, by one warp on its own
// (lane handles i = lane + 32 m). v[m] is the value at index 32 m + lane; the
// block total is returned. Every warp runs the same sequence of operations, so
// every warp gets bit-identical values.
__device__ __forceinline__ float warp_block_scan(const float *dts, float a2, int lane, float (&v)[4]) {
    float carry = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float x = dts[32 * m + lane] * a2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += u;
        }
        x += carry;
        v[m] = x;
        carry = __shfl_sync(0xffffffffu, x, 31);
    }
    return carry;
}

// ---------------------------------------------------------------------------------

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
    k_ssd_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
             const __grid_constant__ CUtensorMap tm_c, const Params prm) {
    using Cf = Cfg<N>;
    constexpr int S = Cf::kStages, YB = Cf::kYBufs, SB = Cf::kStBufs;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    float *dts = reinterpret_cast<float *>(sm + Cf::kOffDts);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + Cf::kOffBar);
    uint64_t *full = bar;                // [S]   stage loaded (TMA bytes + dt)
    uint64_t *empty = full + S;          // [S]   stage consumed (MMA commit + 4 T warps + 4 E warps)
    uint64_t *gfull = empty + S;         // [2]   C B^T in score buffer j
    uint64_t *gp = gfull + 2;            // [2]   G' written back to score buffer j (T)
    uint64_t *xpr = gp + 2;              // [1]   X' written (T)
    uint64_t *dsdone = xpr + 1;          // [2]   chunk state of block c done (MMA commit), buffer c % 2
    uint64_t *dsfree = dsdone + 2;       // [2]   chunk state of block c read by E
    uint64_t *sready = dsfree + 2;       // [SB]  S_in^T of block c written (E)
    uint64_t *yfull = sready + SB;       // [YB]  Y_diag and Y_off of block c done (MMA commit)
    uint64_t *yfree = yfull + YB;        // [YB]  Y of block c read by E
    uint64_t *fin = yfree + YB;          // [1]   every MMA of this CTA done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Cf::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Cf::kOffMisc + 4);
    int *status = prm.status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = prm.H, b = blockIdx.x / H, h = blockIdx.x % H, g = h / (H / prm.G);
    const long long L = prm.L;
    const int nc = prm.nc;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1 + 4 + 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&gfull[i], 1);
            mbar_init(&gp[i], 128);
            mbar_init(&dsdone[i], 1);
            mbar_init(&dsfree[i], 128);
        }
        mbar_init(xpr, 128);
        for (int i = 0; i < SB; ++i) mbar_init(&sready[i], 128);
        for (int i = 0; i < YB; ++i) {
            mbar_init(&yfull[i], 1);
            mbar_init(&yfree[i], 128);
        }
        mbar_init(fin, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(Cf::kTmCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto stage_c = [&](int k) { return sm + k * Cf::kStageBytes; };
    auto stage_b = [&](int k) { return sm + k * Cf::kStageBytes + Cf::kCBytes; };
    auto stage_x = [&](int k) { return sm + k * Cf::kStageBytes + 2 * Cf::kCBytes; };
    unsigned char *xp = sm + Cf::kOffXp;
    auto st_buf = [&](int i) { return sm + Cf::kOffSt + i * Cf::kStBytes; };
    // TMEM column of the chunk state of block c
    auto ds_col = [&](int c) -> uint32_t { return Cf::kDsInG ? 128u * (uint32_t)(c & 1) + 64u : 384u; };

    if (warp == kWarpTma) {
        // ------------------------------------------------------------- loads
        // dt of the next block is fetched into registers one block ahead.
        float dtn[4];
        auto fetch_dt = [&](int c) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const long long t = (long long)c * kQ + lane + 32 * m;
                dtn[m] = t < L ? __bfloat162float(prm.dt[((long long)b * L + t) * H + h]) : 0.f;
            }
        };
        fetch_dt(0);
        int issued = 0;
        for (int c = 0; c < nc; ++c) {
            const int k = c % S;
            if (c >= S && !wait_warp(&empty[k], (uint32_t)((c / S) - 1) & 1u, abort_flag, status)) break;
            const int t0 = c * kQ;
#pragma unroll
            for (int m = 0; m < 4; ++m) dts[k * kQ + lane + 32 * m] = dtn[m];
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_tx(&full[k], Cf::kTxBytes);
                for (int pn = 0; pn < Cf::kPanels; ++pn) {
                    tma_load_4d(stage_c(k) + pn * Cf::kPanelBytes, &tm_c, &full[k], 64 * pn, g, t0, b);
                    tma_load_4d(stage_b(k) + pn * Cf::kPanelBytes, &tm_b, &full[k], 64 * pn, g, t0, b);
                }
                tma_load_4d(stage_x(k), &tm_x, &full[k], 0, h, t0, b);
            }
            __syncwarp();
            issued = c + 1;
            if (c + 1 < nc) fetch_dt(c + 1);
        }
        // drain: loads still in flight land before the CTA exits
        if (lane == 0) {
            for (int c = max(0, issued - S); c < issued; ++c) {
                const unsigned long long t0 = now_ns();
                while (!mbar_try(&full[c % S], (uint32_t)(c / S) & 1u) && now_ns() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------- MMA issue (one thread)
        // Each product of each block is issued as soon as its operands and its
        // accumulator are ready (non-blocking tests), so no block waits on a later one.
        if (lane == 0) {
            constexpr uint32_t kIdG = idesc(128, 128, false, false);
            constexpr uint32_t kIdDs = idesc(128, 64, true, true);
            constexpr uint32_t kIdY = idesc(128, 64, false, true);
            int nG = 0, nDS = 0, nYs = 0, nYd = 0, nDone = 0;
            unsigned long long last = now_ns();
            uint32_t spins = 0;
            while (nDone < nc) {
                bool prog = false;
                // G = C B^T   (M = l, N = s, K = n)
                if (nG < nc) {
                    const int c = nG, k = c % S, j = c & 1;
                    bool ok = mbar_test(&full[k], (uint32_t)(c / S) & 1u);
                    if (ok && c >= 2) {
                        ok = nYd > c - 2 && nDS > c - 2;
                        if (ok && Cf::kDsInG) ok = mbar_test(&dsfree[j], (uint32_t)((c - 2) >> 1) & 1u);
                    }
                    if (ok) {
                        tc_fence_after();
                        const uint32_t ca = smem_u32(stage_c(k)), ba = smem_u32(stage_b(k));
#pragma unroll
                        for (int kk = 0; kk < N / 16; ++kk) {
                            const uint32_t off = (uint32_t)((kk >> 2) * Cf::kPanelBytes + (kk & 3) * 32);
                            mma_ss(tmem + 128 * j, sdesc(ca + off, 16, 1024), sdesc(ba + off, 16, 1024), kIdG, kk > 0);
                        }
                        mma_commit(&gfull[j]);
                        ++nG;
                        prog = true;
                    }
                }
                // chunk state dS^T = B^T X'   (M = n, N = p, K = s)
                if (nDS < nG) {
                    const int c = nDS, k = c % S, j = c & 1;
                    bool ok = mbar_test(xpr, (uint32_t)c & 1u);
                    if (ok) {
                        if (Cf::kDsInG)
                            ok = mbar_test(&gp[j], (uint32_t)(c >> 1) & 1u);
                        else if (c >= 1)
                            ok = mbar_test(&dsfree[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1u);
                    }
                    if (ok) {
                        tc_fence_after();
                        const uint32_t ba = smem_u32(stage_b(k)), xa = smem_u32(xp);
#pragma unroll
                        for (int hf = 0; hf < N / 128; ++hf) {
#pragma unroll
                            for (int kk = 0; kk < kQ / 16; ++kk)
                                mma_ss(tmem + ds_col(c) + 64 * hf,
                                       sdesc(ba + 2 * hf * Cf::kPanelBytes + kk * 2048, Cf::kPanelBytes, 1024),
                                       sdesc(xa + kk * 2048, Cf::kPanelBytes, 1024), kIdDs, kk > 0);
                        }
                        mma_commit(&dsdone[j]);
                        ++nDS;
                        prog = true;
                    }
                }
                // Y_off = C S_in^T   (M = l, N = p, K = n)
                if (nYs < nG) {
                    const int c = nYs, k = c % S, yb = c % YB;
                    bool ok = mbar_test(&sready[c % SB], (uint32_t)(c / SB) & 1u);
                    if (ok && c >= YB) ok = mbar_test(&yfree[yb], (uint32_t)((c - YB) / YB) & 1u);
                    if (ok) {
                        tc_fence_after();
                        const uint32_t ca = smem_u32(stage_c(k)), sa = smem_u32(st_buf(c % SB));
#pragma unroll
                        for (int kk = 0; kk < N / 16; ++kk) {
                            const uint32_t off = (uint32_t)((kk >> 2) * Cf::kPanelBytes + (kk & 3) * 32);
                            mma_ss(tmem + Cf::kTmY + 128 * yb + 64, sdesc(ca + off, 16, 1024),
                                   sdesc(sa + kk * 2048, 1024, 1024), kIdY, kk > 0);
                        }
                        ++nYs;
                        prog = true;
                    }
                }
                // Y_diag = G' X with G' in TMEM   (M = l, N = p, K = s)
                if (nYd < nG) {
                    const int c = nYd, k = c % S, j = c & 1, yb = c % YB;
                    bool ok = mbar_test(&gp[j], (uint32_t)(c >> 1) & 1u);
                    if (ok && c >= YB) ok = mbar_test(&yfree[yb], (uint32_t)((c - YB) / YB) & 1u);
                    if (ok) {
                        tc_fence_after();
                        const uint32_t xa = smem_u32(stage_x(k));
#pragma unroll
                        for (int kk = 0; kk < kQ / 16; ++kk)
                            mma_ts(tmem + Cf::kTmY + 128 * yb, tmem + 128 * j + 8 * kk,
                                   sdesc(xa + kk * 2048, 1024, 1024), kIdY, kk > 0);
                        ++nYd;
                        prog = true;
                    }
                }
                // a block whose four products are all issued: signal its Y and release its stage
                if (nDone < nDS && nDone < nYs && nDone < nYd) {
                    mma_commit(&yfull[nDone % YB]);
                    mma_commit(&empty[nDone % S]);
                    ++nDone;
                    prog = true;
                }
                if (prog) {
                    spins = 0;
                } else if ((++spins & 255u) == 0) {
                    const unsigned long long t = now_ns();
                    if (spins == 256) last = t;
                    if (*abort_flag) break;
                    if (t - last > kWaitNs) {
                        *abort_flag = 1;
                        atomicOr(status, 1);
                        break;
                    }
                }
            }
            // every MMA issued by this thread completes before TMEM is released
            mma_commit(fin);
            const unsigned long long t0 = now_ns();
            while (!mbar_try(fin, 0) && now_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else if (warp < kWarpE) {
        // ------------------------------------------------------------- T: step 0, X', G'
        const int qtr = warp & 3;  // TMEM lane quarter of this warp
        const int row = (qtr << 5) | lane;
        float *acsW = reinterpret_cast<float *>(sm + Cf::kOffAcsT) + (warp - kWarpT) * kQ;
        float *cfW = reinterpret_cast<float *>(sm + Cf::kOffCfT) + (warp - kWarpT) * kQ;
        const float a2 = prm.A[h] * kLog2e;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        for (int c = 0; c < nc; ++c) {
            const int k = c % S, j = c & 1;
            if (!wait_warp(&full[k], (uint32_t)(c / S) & 1u, abort_flag, status)) break;
            const float *dk = dts + k * kQ;
            float v[4];
            const float tot = warp_block_scan(dk, a2, lane, v);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float vend = __shfl_sync(0xffffffffu, v[m], 31);  // A_cs at the end of 32-block m
                acsW[32 * m + lane] = v[m];
                cfW[32 * m + lane] = ex2(vend - v[m]) * dk[32 * m + lane];
            }
            __syncwarp();
            const float acs_r = acsW[row];
            const float dt_r = dk[row];
            // X' (the previous block's chunk-state MMA must be done reading X')
            if (c > 0 && !wait_warp(&dsdone[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1u, abort_flag, status)) break;
            {
                const float w = ex2(tot - acs_r) * dt_r;
                const unsigned char *xs = stage_x(k);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(xs + swz(row, ch));
                    uint4 o;
                    o.x = pack_bf16(w * bf16_lo(xv.x), w * bf16_hi(xv.x));
                    o.y = pack_bf16(w * bf16_lo(xv.y), w * bf16_hi(xv.y));
                    o.z = pack_bf16(w * bf16_lo(xv.z), w * bf16_hi(xv.z));
                    o.w = pack_bf16(w * bf16_lo(xv.w), w * bf16_hi(xv.w));
                    *reinterpret_cast<uint4 *>(xp + swz(row, ch)) = o;
                }
                fence_proxy_async();
                mbar_arrive(xpr);
            }
            // G' = (C B^T) o decay o dt, in place in TMEM as packed bf16 pairs
            if (!wait_warp(&gfull[j], (uint32_t)(c >> 1) & 1u, abort_flag, status)) break;
            tc_fence_after();
            const uint32_t gaddr = tmem + 128 * j + lane_off;
#pragma unroll 1
            for (int jb = 0; jb < 4; ++jb) {
                uint32_t out[16];
                if (jb > qtr) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) out[i] = 0u;
                } else {
                    uint32_t r[32];
                    tmem_ld32(gaddr + 32 * jb, r);
                    tmem_wait_ld();
                    if (jb < qtr) {
                        // strictly below the diagonal sub-block: exp(A_l - A_e) * [exp(A_e - A_s) dt_s]
                        const float rf = ex2(acs_r - acsW[32 * jb + 31]);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int s = 32 * jb + 2 * i;
                            out[i] = pack_bf16(__uint_as_float(r[2 * i]) * rf * cfW[s],
                                               __uint_as_float(r[2 * i + 1]) * rf * cfW[s + 1]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int s = 32 * jb + 2 * i;
                            const float v0 =
                                s <= row ? __uint_as_float(r[2 * i]) * ex2(acs_r - acsW[s]) * dk[s] : 0.f;
                            const float v1 =
                                s + 1 <= row ? __uint_as_float(r[2 * i + 1]) * ex2(acs_r - acsW[s + 1]) * dk[s + 1]
                                             : 0.f;
                            out[i] = pack_bf16(v0, v1);
                        }
                    }
                }
                tmem_st16(gaddr + 16 * jb, out);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&gp[j]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[k]);  // this warp is done with X and dt of the stage
        }
    } else {
        // ------------------------------------------------------------- E: state chain + epilogue
        const int qtr = warp & 3;
        const int row = (qtr << 5) | lane;
        const float a2 = prm.A[h] * kLog2e;
        const float Dh = prm.D ? prm.D[h] : 0.f;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        constexpr int NH = N / 128;  // state rows per thread: n = row + 128 i
        float Sr[NH][kP];
        const long long sbase = ((long long)b * H + h) * kP * N;
#pragma unroll
        for (int i = 0; i < NH; ++i)
#pragma unroll
            for (int p = 0; p < kP; ++p) Sr[i][p] = prm.h0 ? prm.h0[sbase + (long long)p * N + row + 128 * i] : 0.f;
        auto write_st = [&](int c) {  // S_in^T of block c, bf16, into its buffer
            unsigned char *stb = st_buf(c % SB);
#pragma unroll
            for (int i = 0; i < NH; ++i) {
                const int n = row + 128 * i;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 o;
                    o.x = pack_bf16(Sr[i][8 * ch + 0], Sr[i][8 * ch + 1]);
                    o.y = pack_bf16(Sr[i][8 * ch + 2], Sr[i][8 * ch + 3]);
                    o.z = pack_bf16(Sr[i][8 * ch + 4], Sr[i][8 * ch + 5]);
                    o.w = pack_bf16(Sr[i][8 * ch + 6], Sr[i][8 * ch + 7]);
                    *reinterpret_cast<uint4 *>(stb + swz(n, ch)) = o;
                }
            }
            fence_proxy_async();
            mbar_arrive(&sready[c % SB]);
        };
        write_st(0);
        bool ok = true;
        for (int c = 0; c < nc; ++c) {
            const int k = c % S, j = c & 1, yb = c % YB;
            if (!(ok = wait_warp(&full[k], (uint32_t)(c / S) & 1u, abort_flag, status))) break;
            float v[4];
            const float tot = warp_block_scan(dts + k * kQ, a2, lane, v);
            const float acs_r = v[qtr];
            uint4 xr[8];  // this thread's x row (kept only when the stage is released early)
            if (Cf::kXInRegs) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) xr[ch] = *reinterpret_cast<const uint4 *>(stage_x(k) + swz(row, ch));
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[k]);
            }
            // step 3: S <- exp(A_cs[end]) S + dS
            if (!(ok = wait_warp(&dsdone[j], (uint32_t)(c >> 1) & 1u, abort_flag, status))) break;
            tc_fence_after();
            {
                const float gam = ex2(tot);
#pragma unroll
                for (int i = 0; i < NH; ++i) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t r[32];
                        tmem_ld32(tmem + ds_col(c) + 64 * i + 32 * half + lane_off, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            Sr[i][32 * half + q] = fmaf(gam, Sr[i][32 * half + q], __uint_as_float(r[q]));
                    }
                }
                tc_fence_before();
                mbar_arrive(&dsfree[j]);
            }
            // with two S^T buffers the next one was last read by block c-1 (done: see epilogue c-1)
            if (SB == 2 && c + 1 < nc) write_st(c + 1);
            // epilogue: y = Y_diag + exp(A_cs[l]) Y_off + D x
            if (!(ok = wait_warp(&yfull[yb], (uint32_t)(c / YB) & 1u, abort_flag, status))) break;
            tc_fence_after();
            {
                const float el = ex2(acs_r);
                const long long t = (long long)c * kQ + row;
                __nv_bfloat16 *yrow = prm.y + (((long long)b * L + t) * H + h) * kP;
                const uint32_t ya = tmem + Cf::kTmY + 128 * yb + lane_off;
#pragma unroll
                for (int qq = 0; qq < 8; ++qq) {  // 8 columns at a time
                    uint32_t yd[8], ys[8];
                    tmem_ld8(ya + 8 * qq, yd);
                    tmem_ld8(ya + 64 + 8 * qq, ys);
                    tmem_wait_ld();
                    if (qq == 7) {
                        tc_fence_before();
                        mbar_arrive(&yfree[yb]);
                    }
                    const uint4 xv = Cf::kXInRegs ? xr[qq] : *reinterpret_cast<const uint4 *>(stage_x(k) + swz(row, qq));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float y0 = __uint_as_float(yd[2 * e]) + el * __uint_as_float(ys[2 * e]) + Dh * bf16_lo(xw[e]);
                        const float y1 =
                            __uint_as_float(yd[2 * e + 1]) + el * __uint_as_float(ys[2 * e + 1]) + Dh * bf16_hi(xw[e]);
                        o[e] = pack_bf16(y0, y1);
                    }
                    if (t < L) *reinterpret_cast<uint4 *>(yrow + 8 * qq) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            if (!Cf::kXInRegs) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[k]);
            }
            // with one S^T buffer it is free only now (Y_off of block c is done)
            if (SB == 1 && c + 1 < nc) write_st(c + 1);
        }
        if (ok && prm.h_final) {
#pragma unroll
            for (int i = 0; i < NH; ++i)
#pragma unroll
                for (int p = 0; p < kP; ++p) prm.h_final[sbase + (long long)p * N + row + 128 * i] = Sr[i][p];
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cf::kTmCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------------
// host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;  // process-wide cache of the driver entry point
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B, L, X, inner] bf16 tensor, box {64, 1, 128, 1}, 128-byte swizzle.
bool encode_4d(CUtensorMap *m, const void *base, int64_t inner, int64_t X, int64_t L, int64_t B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)X, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(inner * 2), (cuuint64_t)(X * inner * 2),
                                   (cuuint64_t)(L * X * inner * 2)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kQ, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N>
cudaError_t launch(const FwdProblem &p, int *status, cudaStream_t s) {
    CUtensorMap tx, tb, tcm;
    if (!encode_4d(&tx, p.x, kP, p.H, p.L, p.B) || !encode_4d(&tb, p.Bm, N, p.G, p.L, p.B) ||
        !encode_4d(&tcm, p.Cm, N, p.G, p.L, p.B))
        return cudaErrorInvalidValue;
    Params prm;
    prm.dt = static_cast<const __nv_bfloat16 *>(p.dt);
    prm.A = p.A;
    prm.D = p.D;
    prm.h0 = p.h0;
    prm.h_final = p.h_final;
    prm.y = static_cast<__nv_bfloat16 *>(p.y);
    prm.status = status;
    prm.L = p.L;
    prm.H = (int)p.H;
    prm.G = (int)p.G;
    prm.nc = (int)((p.L + kQ - 1) / kQ);
    cudaError_t e = cudaFuncSetAttribute(k_ssd_tc<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<N>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    k_ssd_tc<N><<<(unsigned)(p.B * p.H), kThreads, Cfg<N>::kSmemAlloc, s>>>(tx, tb, tcm, prm);
    return cudaGetLastError();
}

}  // namespace tc

bool tc_supported(const FwdProblem &p) {
    return p.dtype == SSD_BF16 && p.P == tc::kP && (p.N == 128 || p.N == 256) && (p.Q == 128 || p.Q == 256) &&
           p.L >= 1 && p.L < (1ll << 31) && p.B * p.H < (1ll << 31);
}

size_t tc_fwd_workspace_bytes(const FwdProblem &) { return kWsAlign; }

cudaError_t tc_fwd(const FwdProblem &p, void *ws, cudaStream_t s) {
    int *status = static_cast<int *>(ws);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    return p.N == 128 ? tc::launch<128>(p, status, s) : tc::launch<256>(p, status, s);
}

}  // namespace ssd
