// Fused chunked SSD forward on 5th-generation tensor cores (tcgen05, sm_100a).
//
// A persistent grid (one CTA per SM, or one per stream when there are fewer streams)
// splits the B*H*nc (stream, 128-token block) tasks into equal contiguous shares; within a share each stream's blocks are
// walked in order, so x is read once, y is written once and the running state
// stays on chip. Per block (the four steps of "SSD 算法：分块和状态传递" in the
// Mamba-2 SSD write-up, with the block decomposition of "SSD 算法：分块矩阵分解"):
//   step 0  A_cs[l] = sum_{j<=l} dt_j A_h            (within the block, log2 domain)
//   step 1  G = C B^T on tensor cores (TMEM); G' = causal part of G written back to TMEM
//           as bf16
//   step 2  dS^T = B^T X'' on tensor cores
//   step 3  S <- exp(A_cs[127]) S + exp(A_cs[127] - m) dS            (fp32, registers)
//   step 4  Y = C (exp(m) S_in)^T + G' X'' in one TMEM accumulator (S_in in bf16 shared
//           memory, G' as the TMEM A operand), and y = exp(A_cs[l] - m) Y
// The decay exp(A_cs[l] - A_cs[s]) of the masked block is split at the block's
// reference m (the middle of the range of A_cs): exp(A_cs[l] - m) is a row factor
// applied in the epilogue and exp(m - A_cs[s]) dt_s a column factor applied to x,
// X''[s,:] = exp(m - A_cs[s]) dt_s x_s, in place in shared memory; the state term
// exp(A_cs[l]) C S_in^T shares the row factor once S_in is scaled by exp(m). All factors
// stay within 2^64 when the block's A_cs range is at most 128 (log2 units), which holds
// for any decay that leaves more than 2^-128 of a state after 128 tokens. The D skip
// term rides on the diagonal of G' as D_h / dt_l. A block outside those bounds (a wider
// range, or a token with |dt| < 2^-40) takes the exact form instead: G'[l,s] =
// G[l,s] exp(A_cs[l] - A_cs[s]) dt_s (+ D_h on the diagonal) elementwise against x itself,
// the rows of C scaled by exp(A_cs[l]) in place, S_in unscaled, m = A_cs[127] and y = Y.
// A chunk argument of 256 is evaluated as two 128-token diagonal blocks; the 128x128
// block between them goes through the state (its low-rank factor), which is the same
// matrix product re-associated.
//
// A stream whose blocks fall into two CTAs' shares is cut: the CTA holding its
// first part runs that part first and hands the state over through global memory
// (the state passing of the sequence-parallel scheme in the same write-up); the
// CTA holding the rest runs it last, so the hand-over is ready long before it is
// read. The wait for it is bounded all the same.
//
// Warp roles (384 threads at N = 128, 512 at N = 256): warp 0 loads (TMA + dt) and runs
// step 0; warps 1, 2 and 3 issue C B^T, the chunk states and Y (one issuing thread per
// product: an MMA instruction keeps its issuing warp busy for ~100 cycles, so the products
// are issued in parallel); warps 4-7 ("T") do X'' and G'; warps 8-11 ("E"), and 12-15 at
// N = 256, run the state chain, one set of four warps per 128 state rows, and the first set
// runs the epilogue. B and C, and x with its step-0 values, have separate stage barriers, so
// the next block's B and C load as soon as the products that read them are done. Every
// wait is bounded: on timeout the CTA raises a status word in the workspace, drains its
// own TMA loads and MMAs, frees TMEM and returns.
#include <algorithm>

// the E threads keep a 64-value state row live across their waits
#define SSD_INLINE_SLOW_WAIT
#include "tc_ptx.cuh"

namespace ssd {
namespace tc {

constexpr int kQ = 128;  // tokens per diagonal block
constexpr int kP = 64;   // head dimension handled by this path
constexpr int kWarpTma = 0, kWarpG = 1, kWarpDs = 2, kWarpYs = 3, kWarpE = 8;  // warps 4-7: T
constexpr float kLog2e = 1.4426950408889634f;

template <int N>
struct Cfg {
    // N = 128: double-buffered input stages and S^T. N = 256: one of each (the wider B, C and
    // S^T fill shared memory).
    static constexpr bool kWide = N == 256;
    // E warps: one set of four per 128 state rows (each thread keeps one state row of 64
    // values in registers); the first set also runs the epilogue
    static constexpr int kESets = N / 128;
    static constexpr int kThreads = 32 * (kWarpE + 4 * kESets);
    static constexpr int kStages = kWide ? 1 : 2;
    static constexpr int kYBufs = 2;
    static constexpr int kStBufs = kWide ? 1 : 2;
    static constexpr int kPanels = N / 64;           // 64-column panels of B and C
    static constexpr int kPanelBytes = kQ * 128;     // 128 rows x 128 B
    static constexpr int kCBytes = kPanels * kPanelBytes;
    static constexpr int kXBytes = kQ * 128;         // 128 rows x 64 bf16
    static constexpr int kStageBytes = 2 * kCBytes + kXBytes;  // C, B, X
    static constexpr int kStBytes = N * 128;                   // S^T bf16 [N][64]
    static constexpr int kOffXp = kStages * kStageBytes;
    static constexpr int kOffSt = kOffXp + kXBytes;
    static constexpr int kOffSmall = kOffSt + kStBufs * kStBytes;
    // per stage: dt, A_cs (log2 domain), the block scalars {A_cs[127], m, exact?, valid tokens}
    // and the block's coordinates {b, h, c, last of its piece}; they travel with the x tile
    static constexpr int kOffDts = kOffSmall;                       // float [kStages][128]
    static constexpr int kOffAcs = kOffDts + kStages * kQ * 4;      // float [kStages][128]
    static constexpr int kOffBlk = kOffAcs + kStages * kQ * 4;      // float4 [kStages]
    static constexpr int kOffCrd = kOffBlk + kStages * 16;          // int4 [kStages]
    static constexpr int kOffBar = kOffCrd + kStages * 16;          // uint64 barriers
    // TMEM columns: score buffers j at 128 j (fp32 C B^T, then G' packed in its first 64);
    // Y buffers at 256 + 64 i; the chunk-state accumulators (64 columns per 128 state rows)
    // from 384, two of them for N = 128 and one for N = 256.
    static constexpr int kTmY = 256;
    static constexpr int kTmDs = 384;
    static constexpr int kDsCols = N / 2;
    static constexpr int kDsBufs = 128 / kDsCols;
    static constexpr int kTmCols = 512;
    static constexpr int kNumBars = 5 * kStages + 6 + 2 * kDsBufs + kStBufs + 2 * kYBufs + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;         // tmem base, abort flag
    static constexpr int kSmemBytes = kOffMisc + 16;
    static constexpr int kSmemAlloc = kSmemBytes + 1024;            // slack for 1024-B alignment
    static_assert(kSmemAlloc <= 232448, "shared memory budget");
    static constexpr uint32_t kTxBC = 2 * kCBytes, kTxX = kXBytes;
};

struct Params {
    const __nv_bfloat16 *dt;
    const float *A, *D, *h0;
    float *h_final;
    __nv_bfloat16 *y;
    int *status;         // bit 0: a bounded wait ran out
    int *flags;          // [gridDim.x] hand-over counters (zeroed before the launch)
    float *handover;     // [gridDim.x][P][N] state at the end of each CTA's first part
    long long L, total;  // total = B * H * nc tasks
    int H, G, nc;
    int wait_us;         // bounded-wait limit in microseconds (0: the built-in one)
};

// The share of CTA i is [lo, hi) in (stream-major, block-minor) task order, run as
// [B0, hi) (the start of the last stream it touches), then [A0, B0) (whole streams),
// then [lo, A0) (the rest of a stream begun by CTA i-1).
struct Share {
    long long lo, hi, a0, b0;
    __device__ __forceinline__ int count() const { return (int)(hi - lo); }
    __device__ __forceinline__ long long task(int t) const {
        const long long n1 = hi - b0, n2 = b0 - a0;
        return t < n1 ? b0 + t : (t < n1 + n2 ? a0 + (t - n1) : lo + (t - n1 - n2));
    }
};
__device__ __forceinline__ Share share_of(long long total, int nc, int i, int G) {
    const long long q = total / G, r = total % G;
    Share s;
    s.lo = q * i + (r * i) / G;
    s.hi = q * (i + 1) + (r * (i + 1)) / G;
    s.a0 = min(((s.lo + nc - 1) / nc) * nc, s.hi);
    s.b0 = max((s.hi / nc) * nc, s.a0);
    return s;
}

// ---------------------------------------------------------------------------------

// Exact form of G' for one warp's 32 rows (lane quarter qtr): every element of the causal
// part takes its own exponential, D_h on the diagonal (blocks whose decay range is too wide
// for the factored form). A_cs and dt come by explicit shared-memory loads, two columns at a
// time; volatile, so that they stay after the barrier wait that makes those values valid.
__device__ __forceinline__ void gprime_exact(uint32_t gaddr, int qtr, int row, float acs_r, const float *acsW,
                                          const float *dk, float Dh) {
    // 16 columns per TMEM load (the 512-thread N = 256 configuration caps a thread at 128 registers)
#pragma unroll 1
    for (int pc = 0; pc < 8; ++pc) {
        uint32_t out[8];
        if ((pc >> 1) > qtr) {
#pragma unroll
            for (int i = 0; i < 8; ++i) out[i] = 0u;
        } else {
            uint32_t r[16];
            tmem_ld16(gaddr + 16 * pc, r);
            tmem_wait_ld();
            const uint32_t aw = (uint32_t)__cvta_generic_to_shared(acsW + 16 * pc);
            const uint32_t dw = (uint32_t)__cvta_generic_to_shared(dk + 16 * pc);
#pragma unroll  // whole: r and out stay in registers
            for (int i = 0; i < 8; ++i) {
                const int s = 16 * pc + 2 * i;
                float a0, a1, d0, d1;
                asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(a0), "=f"(a1) : "r"(aw + 8 * i));
                asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(d0), "=f"(d1) : "r"(dw + 8 * i));
                float v0 = s <= row ? __uint_as_float(r[2 * i]) * ex2(acs_r - a0) * d0 : 0.f;
                float v1 = s + 1 <= row ? __uint_as_float(r[2 * i + 1]) * ex2(acs_r - a1) * d1 : 0.f;
                v0 += s == row ? Dh : 0.f;
                v1 += s + 1 == row ? Dh : 0.f;
                out[i] = pack_bf16(v0, v1);
            }
        }
        tmem_st8(gaddr + 8 * pc, out);
    }
}

// Bounded spin on a hand-over counter in global memory.
__device__ __noinline__ bool wait_flag(const int *flag, int want, volatile int *abort_flag, int *status) {
    const unsigned long long t0 = now_ns(), lim = wait_limit_ns(abort_flag);
    for (;;) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v >= want) return true;
        if (*abort_flag) return false;
        if (now_ns() - t0 > lim) {
            *abort_flag = 1;
            atomicOr(status, 1);
            return false;
        }
        __nanosleep(200);
    }
}

template <int N>
__global__ void __launch_bounds__(Cfg<N>::kThreads, 1)
    k_ssd_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
             const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, const Params prm) {
    using Cf = Cfg<N>;
    constexpr int S = Cf::kStages, YB = Cf::kYBufs, SB = Cf::kStBufs, DB = Cf::kDsBufs;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    float *dts = reinterpret_cast<float *>(sm + Cf::kOffDts);
    float *acs_s = reinterpret_cast<float *>(sm + Cf::kOffAcs);
    float4 *blk_s = reinterpret_cast<float4 *>(sm + Cf::kOffBlk);
    int4 *crd_s = reinterpret_cast<int4 *>(sm + Cf::kOffCrd);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + Cf::kOffBar);
    uint64_t *full_bc = bar;             // [S]   B and C of stage k loaded
    uint64_t *full_x = full_bc + S;      // [S]   x of stage k loaded and its step-0 values written
    uint64_t *empty_bc = full_x + S;     // [S]   B, C consumed: C B^T, chunk-state and Y_off commits
    uint64_t *empty_x = empty_bc + S;    // [S]   x and step-0 values consumed: 4 T + 4 E warps, 2 commits
    uint64_t *xpr = empty_x + S;         // [S]   X'' of stage k written (T)
    uint64_t *gfull = xpr + S;           // [2]   C B^T in score buffer j
    uint64_t *gp = gfull + 2;            // [2]   G' written back to score buffer j (T)
    uint64_t *ydd = gp + 2;              // [2]   Y_diag of block t done (score buffer t % 2 reusable)
    uint64_t *dsdone = ydd + 2;          // [DB]  chunk state of block t done
    uint64_t *dsfree = dsdone + DB;      // [DB]  chunk state of block t read by E
    uint64_t *sready = dsfree + DB;      // [SB]  S_in^T of block t written (E)
    uint64_t *yfull = sready + SB;       // [YB]  Y of block t done
    uint64_t *yfree = yfull + YB;        // [YB]  Y of block t read by E
    uint64_t *fin = yfree + YB;          // [1]   every MMA of this CTA done (3 issuers)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Cf::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Cf::kOffMisc + 4);
    int *status = prm.status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = prm.H, nc = prm.nc, hpg = prm.H / prm.G;
    const long long L = prm.L;
    const Share sh = share_of(prm.total, nc, blockIdx.x, gridDim.x);
    const int ntask = sh.count();

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full_bc[i], 1);
            mbar_init(&full_x[i], 1);
            mbar_init(&empty_bc[i], 3);
            mbar_init(&empty_x[i], 4 + 4 * Cf::kESets + 2);
            mbar_init(&xpr[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&gfull[i], 1);
            mbar_init(&gp[i], 128);
            mbar_init(&ydd[i], 1);
        }
        for (int i = 0; i < DB; ++i) {
            mbar_init(&dsdone[i], 1);
            mbar_init(&dsfree[i], 128 * Cf::kESets);
        }
        for (int i = 0; i < SB; ++i) mbar_init(&sready[i], 128 * Cf::kESets);
        for (int i = 0; i < YB; ++i) {
            mbar_init(&yfull[i], 1);
            mbar_init(&yfree[i], 128);
        }
        mbar_init(fin, 3);
        *abort_flag = 0;
        abort_flag[1] = prm.wait_us;  // bounded-wait limit (us; 0: the built-in one)
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpG) {
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
    // TMEM column of the chunk-state accumulator of task t
    auto ds_col = [&](int t) -> uint32_t { return (uint32_t)(Cf::kTmDs + Cf::kDsCols * (t % DB)); };
    constexpr uint32_t kIdG = idesc(128, 128, false, false);
    constexpr uint32_t kIdDs = idesc(128, 64, true, true);
    constexpr uint32_t kIdY = idesc(128, 64, false, true);

    if (warp == kWarpTma) {
        // ------------------------------------------------------------- loads and step 0
        // B and C of task t are loaded as soon as their stage is free, then x with the step-0
        // values; step 0 of task t+1 then runs on dt that was fetched one task earlier, and dt
        // of task t+2 is fetched.
        const uint64_t pol_keep = policy_evict_last(), pol_stream = policy_evict_first();
        // Lane i handles tokens 4 i .. 4 i + 3 of a block.
        float raw[4], a_raw = 0.f;  // dt and A_h of the task after the prepared one
        int nvalid_raw = 0;
        float4 dtn, acn;            // prepared step 0 of the next task to load
        float4 blkn = make_float4(0.f, 0.f, 0.f, 0.f);
        int4 crd_raw = make_int4(0, 0, 0, 0), crd_n = crd_raw;  // {b, h, c, last of its piece}
        // Task coordinates advance by one block at a time except where the share's order
        // jumps (at most twice), so the divisions run only there.
        long long cur_gi = -2;
        int cur_c = 0, cur_b = 0, cur_h = 0;
        auto fetch = [&](int t) {
            const long long gi = sh.task(t);
            if (gi == cur_gi + 1 && cur_c + 1 < nc) {
                ++cur_c;
            } else if (gi == cur_gi + 1) {
                cur_c = 0;
                if (++cur_h == H) {
                    cur_h = 0;
                    ++cur_b;
                }
            } else {
                const int sidx = (int)(gi / nc);
                cur_c = (int)(gi - (long long)sidx * nc);
                cur_b = sidx / H;
                cur_h = sidx - cur_b * H;
            }
            cur_gi = gi;
            const int b = cur_b, h = cur_h, c = cur_c;
            crd_raw = make_int4(b, h, c, (c == nc - 1 || gi == sh.hi - 1) ? 1 : 0);
            a_raw = __ldg(prm.A + h);
            nvalid_raw = (int)min((long long)kQ, L - (long long)c * kQ);
            const long long t0 = (long long)c * kQ + 4 * lane;
            const __nv_bfloat16 *src = prm.dt + ((long long)b * L + t0) * H + h;
#pragma unroll
            for (int m = 0; m < 4; ++m) raw[m] = t0 + m < L ? __bfloat162float(src[(long long)m * H]) : 0.f;
        };
        // Step 0 on the fetched dt: the within-block cumsum of dt * A_h (log2 domain), its
        // range, the reference m in the middle of it, and whether the factored form is safe.
        auto prep = [&]() {
            const float a2 = a_raw * kLog2e;
            crd_n = crd_raw;
            dtn = make_float4(raw[0], raw[1], raw[2], raw[3]);
            const float v0 = dtn.x * a2, v1 = fmaf(dtn.y, a2, v0), v2 = fmaf(dtn.z, a2, v1), v3 = fmaf(dtn.w, a2, v2);
            float incl = v3;  // inclusive scan of the lanes' sums
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            const float excl = incl - v3;
            acn = make_float4(excl + v0, excl + v1, excl + v2, incl);
            const float tot = __shfl_sync(0xffffffffu, incl, 31);
            float mx = fmaxf(fmaxf(acn.x, acn.y), fmaxf(acn.z, acn.w));
            float mn = fminf(fminf(acn.x, acn.y), fminf(acn.z, acn.w));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            }
            const int nv = nvalid_raw - 4 * lane;  // valid tokens of this lane: min(max(nv, 0), 4)
            const bool dt_ok = (nv <= 0 || fabsf(dtn.x) >= 0x1p-40f) && (nv <= 1 || fabsf(dtn.y) >= 0x1p-40f) &&
                               (nv <= 2 || fabsf(dtn.z) >= 0x1p-40f) && (nv <= 3 || fabsf(dtn.w) >= 0x1p-40f);
            // (mx - mn <= 128 is false for NaN, which then takes the exact form)
            const bool factored = __all_sync(0xffffffffu, dt_ok) && (mx - mn <= 128.f);
            blkn = make_float4(tot, factored ? 0.5f * (mx + mn) : tot, factored ? 0.f : 1.f, (float)nvalid_raw);
        };
        if (ntask > 0) {
            fetch(0);
            prep();
            if (ntask > 1) fetch(1);
        }
        int nbc = 0, nx = 0;  // loads issued
        for (int t = 0; t < ntask; ++t) {
            const int k = t % S;
            const uint32_t ph = (uint32_t)((t / S) - 1) & 1u;
            const int b = crd_n.x, h = crd_n.y, c = crd_n.z, t0 = c * kQ, g = h / hpg;
            if (t >= S && !wait_warp(&empty_bc[k], ph, abort_flag, status)) break;
            if (lane == 0) {
                mbar_arrive_tx(&full_bc[k], Cf::kTxBC);
                for (int pn = 0; pn < Cf::kPanels; ++pn) {
                    tma_load_4d_hint(stage_c(k) + pn * Cf::kPanelBytes, &tm_c, &full_bc[k], 64 * pn, g, t0, b, pol_keep);
                    tma_load_4d_hint(stage_b(k) + pn * Cf::kPanelBytes, &tm_b, &full_bc[k], 64 * pn, g, t0, b, pol_keep);
                }
            }
            nbc = t + 1;
            if (t >= S && !wait_warp(&empty_x[k], ph, abort_flag, status)) break;
            reinterpret_cast<float4 *>(dts + k * kQ)[lane] = dtn;
            reinterpret_cast<float4 *>(acs_s + k * kQ)[lane] = acn;
            if (lane == 0) {
                blk_s[k] = blkn;
                crd_s[k] = crd_n;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_tx(&full_x[k], Cf::kTxX);
                tma_load_4d_hint(stage_x(k), &tm_x, &full_x[k], 0, h, t0, b, pol_stream);
            }
            __syncwarp();
            nx = t + 1;
            if (t + 1 < ntask) {
                prep();
                if (t + 2 < ntask) fetch(t + 2);
            }
        }
        // drain: loads still in flight land before the CTA exits
        if (lane == 0) {
            for (int t = max(0, nbc - S); t < nbc; ++t) {
                const unsigned long long w0 = now_ns();
                while (!mbar_try(&full_bc[t % S], (uint32_t)(t / S) & 1u) && now_ns() - w0 < kWaitNs) {
                }
            }
            for (int t = max(0, nx - S); t < nx; ++t) {
                const unsigned long long w0 = now_ns();
                while (!mbar_try(&full_x[t % S], (uint32_t)(t / S) & 1u) && now_ns() - w0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == kWarpG) {
        // ------------------------------------------------------------- G = C B^T   (M = l, N = s, K = n)
        if (lane == 0) {
            for (int t = 0; t < ntask; ++t) {
                const int k = t % S, j = t & 1;
                if (!wait_phase(&full_bc[k], (uint32_t)(t / S) & 1u, abort_flag, status)) break;
                // score buffer j: G' of task t-2 consumed by its Y_diag
                if (t >= 2 && !wait_phase(&ydd[j], (uint32_t)((t - 2) >> 1) & 1u, abort_flag, status)) break;
                tc_fence_after();
                const uint32_t ca = smem_u32(stage_c(k)), ba = smem_u32(stage_b(k));
#pragma unroll 1
                for (int kk = 0; kk < N / 16; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * Cf::kPanelBytes + (kk & 3) * 32);
                    mma_ss(tmem + 128 * j, sdesc(ca + off, 16, 1024), sdesc(ba + off, 16, 1024), kIdG, kk > 0);
                }
                mma_commit(&gfull[j]);
                mma_commit(&empty_bc[k]);
            }
            mma_commit(fin);
        }
        __syncwarp();
    } else if (warp == kWarpDs) {
        // ------------------------------------------------------------- dS^T = B^T X''   (M = n, N = p, K = s)
        if (lane == 0) {
            for (int t = 0; t < ntask; ++t) {
                const int k = t % S, db = t % DB;
                if (!wait_phase(&xpr[k], (uint32_t)(t / S) & 1u, abort_flag, status)) break;
                if (!wait_phase(&full_bc[k], (uint32_t)(t / S) & 1u, abort_flag, status)) break;
                if (t >= DB && !wait_phase(&dsfree[db], (uint32_t)((t - DB) / DB) & 1u, abort_flag, status)) break;
                tc_fence_after();
                // X'' in place in the stage, or (exact form) X' in its own buffer
                const bool exact = blk_s[k].z != 0.f;
                const uint32_t ba = smem_u32(stage_b(k)), xa = smem_u32(exact ? xp : stage_x(k));
#pragma unroll 1
                for (int hf = 0; hf < N / 128; ++hf) {
#pragma unroll 1
                    for (int kk = 0; kk < kQ / 16; ++kk)
                        mma_ss(tmem + ds_col(t) + 64 * hf,
                               sdesc(ba + 2 * hf * Cf::kPanelBytes + kk * 2048, Cf::kPanelBytes, 1024),
                               sdesc(xa + kk * 2048, Cf::kPanelBytes, 1024), kIdDs, kk > 0);
                }
                mma_commit(&dsdone[db]);
                mma_commit(&empty_bc[k]);
                mma_commit(&empty_x[k]);
            }
            mma_commit(fin);
        }
        __syncwarp();
    } else if (warp == kWarpYs) {
        // ------------------------------------------------------------- Y = C (s S_in)^T + G' X''
        // One accumulator: Y_off first (M = l, N = p, K = n), then Y_diag (K = s) with G' as the
        // TMEM A operand. In the factored form s = exp(m) and y = exp(A_cs[l] - m) Y; in the exact
        // form T has scaled the rows of C by exp(A_cs[l]), s = 1 and y = Y.
        if (lane == 0) {
            for (int t = 0; t < ntask; ++t) {
                const int k = t % S, j = t & 1, yb = t % YB;
                const uint32_t yacc = tmem + Cf::kTmY + 64 * yb;
                if (!wait_phase(&full_bc[k], (uint32_t)(t / S) & 1u, abort_flag, status)) break;
                if (!wait_phase(&sready[t % SB], (uint32_t)(t / SB) & 1u, abort_flag, status)) break;
                if (t >= YB && !wait_phase(&yfree[yb], (uint32_t)((t - YB) / YB) & 1u, abort_flag, status)) break;
                const bool exact = blk_s[k].z != 0.f;  // written before S_in^T of task t was
                if (exact && !wait_phase(&gp[j], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                tc_fence_after();
                const uint32_t ca = smem_u32(stage_c(k)), sa = smem_u32(st_buf(t % SB));
#pragma unroll 1
                for (int kk = 0; kk < N / 16; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * Cf::kPanelBytes + (kk & 3) * 32);
                    mma_ss(yacc, sdesc(ca + off, 16, 1024), sdesc(sa + kk * 2048, 1024, 1024), kIdY, kk > 0);
                }
                mma_commit(&empty_bc[k]);
                if (!exact && !wait_phase(&gp[j], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                tc_fence_after();
                const uint32_t xa = smem_u32(stage_x(k));  // X'' in place (x itself in the exact form)
#pragma unroll 1
                for (int kk = 0; kk < kQ / 16; ++kk)
                    mma_ts(yacc, tmem + 128 * j + 8 * kk, sdesc(xa + kk * 2048, 1024, 1024), kIdY, 1);
                mma_commit(&yfull[yb]);
                mma_commit(&ydd[j]);
                mma_commit(&empty_x[k]);
            }
            mma_commit(fin);
        }
        __syncwarp();
    } else if (warp < kWarpE) {
        // ------------------------------------------------------------- T: X'' and G'
        const int qtr = warp & 3;  // TMEM lane quarter of this warp: rows 32 qtr .. 32 qtr + 31
        const int row = (qtr << 5) | lane;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        // Row `row` of x (64 bf16, 128-byte swizzled) scaled by w, from src to dst.
        auto scale_row = [&](const unsigned char *src, unsigned char *dst, float w) {
#pragma unroll 1
            for (int ch = 0; ch < 8; ++ch) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(src + swz(row, ch));
                uint4 o;
                o.x = pack_bf16(w * bf16_lo(xv.x), w * bf16_hi(xv.x));
                o.y = pack_bf16(w * bf16_lo(xv.y), w * bf16_hi(xv.y));
                o.z = pack_bf16(w * bf16_lo(xv.z), w * bf16_hi(xv.z));
                o.w = pack_bf16(w * bf16_lo(xv.w), w * bf16_hi(xv.w));
                *reinterpret_cast<uint4 *>(dst + swz(row, ch)) = o;
            }
        };
        for (int t = 0; t < ntask; ++t) {
            const int k = t % S, j = t & 1;
            if (!wait_warp(&full_x[k], (uint32_t)(t / S) & 1u, abort_flag, status)) break;
            const float Dh = prm.D ? __ldg(prm.D + crd_s[k].y) : 0.f;
            const float *dk = dts + k * kQ;
            const float *acsW = acs_s + k * kQ;
            const float4 blk = blk_s[k];  // {A_cs[127], m, exact?, valid tokens}
            const bool exact = blk.z != 0.f;  // warp-uniform
            const float acs_r = acsW[row], dt_r = dk[row];
            const uint32_t gaddr = tmem + 128 * j + lane_off;
            // X''[row,:] = exp(m - A_cs[row]) dt_row x_row, in place; in the exact form (m = A_cs[127])
            // into its own buffer, once the previous chunk-state MMA is done reading that
            if (exact && t > 0 &&
                !wait_warp(&dsdone[(t - 1) % DB], (uint32_t)((t - 1) / DB) & 1u, abort_flag, status))
                break;
            scale_row(stage_x(k), exact ? xp : stage_x(k), ex2(blk.y - acs_r) * dt_r);
            fence_proxy_async();
            mbar_arrive(&xpr[k]);
            if (!wait_warp(&gfull[j], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
            tc_fence_after();
            if (!exact) {
                const float dinv = dt_r != 0.f ? Dh / dt_r : 0.f;  // dt = 0 only on padding rows here
                // 32-column blocks jb < qtr lie below the diagonal: plain conversion to bf16 pairs
#pragma unroll 1
                for (int jb = 0; jb < qtr; ++jb) {
                    uint32_t r[32], out[16];
                    tmem_ld32(gaddr + 32 * jb, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        out[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                    tmem_st16(gaddr + 16 * jb, out);
                }
                {  // block qtr holds the diagonal: mask s > row, D_h / dt_l on s == row
                    uint32_t r[32], out[16];
                    tmem_ld32(gaddr + 32 * qtr, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int s = 2 * i, rl = lane;  // offsets within the block
                        float v0 = s <= rl ? __uint_as_float(r[2 * i]) : 0.f;
                        float v1 = s + 1 <= rl ? __uint_as_float(r[2 * i + 1]) : 0.f;
                        v0 += s == rl ? dinv : 0.f;
                        v1 += s + 1 == rl ? dinv : 0.f;
                        out[i] = pack_bf16(v0, v1);
                    }
                    tmem_st16(gaddr + 16 * qtr, out);
                }
                uint32_t zero[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll 1
                for (int jb = qtr + 1; jb < 4; ++jb) tmem_st16(gaddr + 16 * jb, zero);
            } else {
                gprime_exact(gaddr, qtr, row, acs_r, acsW, dk, Dh);
                // C[row,:] *= exp(A_cs[row]) in place (C B^T is done with C): the row factor of
                // Y_off, which the exact form cannot share with Y_diag
                if (!wait_warp(&full_bc[k], (uint32_t)(t / S) & 1u, abort_flag, status)) break;
                const float el = ex2(acs_r);
                unsigned char *cs = stage_c(k);
#pragma unroll 1
                for (int pn = 0; pn < Cf::kPanels; ++pn) scale_row(cs + pn * Cf::kPanelBytes, cs + pn * Cf::kPanelBytes, el);
                fence_proxy_async();
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&gp[j]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_x[k]);  // this warp is done with x and the step-0 values
        }
    } else {
        // ------------------------------------------------------------- E: state chain + epilogue
        const int qtr = warp & 3, set = Cf::kESets == 1 ? 0 : (warp - kWarpE) >> 2;
        const int row = (qtr << 5) | lane;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        const int nrow = row + 128 * set;  // this thread's state row n
        float Sr[kP];
        // S_in^T of task t, bf16, scaled by s = exp(m) of task t in the factored form (1 in the
        // exact form), into its buffer
        auto write_st = [&](int t) -> bool {
            if (!wait_warp(&full_x[t % S], (uint32_t)(t / S) & 1u, abort_flag, status)) return false;
            const float4 bt = blk_s[t % S];
            const float sg = bt.z != 0.f ? 1.f : ex2(bt.y);
            unsigned char *stb = st_buf(t % SB);
            // the buffer doubles as this warp's y staging slice: its last y store must have read it
            if (lane == 0) bulk_wait_read();
            __syncwarp();
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 o;
                o.x = scale2_bf16(sg, Sr[8 * ch + 0], Sr[8 * ch + 1]);
                o.y = scale2_bf16(sg, Sr[8 * ch + 2], Sr[8 * ch + 3]);
                o.z = scale2_bf16(sg, Sr[8 * ch + 4], Sr[8 * ch + 5]);
                o.w = scale2_bf16(sg, Sr[8 * ch + 6], Sr[8 * ch + 7]);
                *reinterpret_cast<uint4 *>(stb + swz(nrow, ch)) = o;
            }
            fence_proxy_async();
            mbar_arrive(&sready[t % SB]);
            return true;
        };
        // Initial state of the piece that starts at task t: h0 (or zeros) at the start of a
        // stream, otherwise the state handed over by the previous CTA.
        auto load_init = [&](int t) -> bool {
            const long long gi = sh.task(t);
            const int sidx = (int)(gi / nc), c = (int)(gi % nc);
            if (c == 0) {
                const long long base = (long long)sidx * kP * N;
#pragma unroll
                for (int p = 0; p < kP; ++p) Sr[p] = prm.h0 ? prm.h0[base + (long long)p * N + nrow] : 0.f;
                return true;
            }
            // every E thread of the previous CTA has written its row and counted itself
            if (!wait_flag(prm.flags + blockIdx.x - 1, 128 * Cf::kESets, abort_flag, status)) return false;
            const float *src = prm.handover + (long long)(blockIdx.x - 1) * kP * N;
#pragma unroll
            for (int p = 0; p < kP; ++p) Sr[p] = __ldcg(src + p * N + nrow);
            return true;
        };
        // End of a piece: the final state of the stream, or the hand-over to the next CTA.
        auto store_final = [&](int t) {
            const long long gi = sh.task(t);
            const int sidx = (int)(gi / nc), c = (int)(gi % nc);
            if (c == nc - 1) {
                if (prm.h_final) {
                    const long long base = (long long)sidx * kP * N;
#pragma unroll
                    for (int p = 0; p < kP; ++p) prm.h_final[base + (long long)p * N + nrow] = Sr[p];
                }
            } else {
                float *dst = prm.handover + (long long)blockIdx.x * kP * N;
#pragma unroll
                for (int p = 0; p < kP; ++p) __stcg(dst + p * N + nrow, Sr[p]);
                __threadfence();
                atomicAdd(prm.flags + blockIdx.x, 1);
            }
        };
        bool ok = ntask > 0 && load_init(0) && write_st(0);
        for (int t = 0; ok && t < ntask; ++t) {
            const int k = t % S, yb = t % YB, db = t % DB;
            if (!(ok = wait_warp(&full_x[k], (uint32_t)(t / S) & 1u, abort_flag, status))) break;
            const int4 crd = crd_s[k];  // {b, h, c, last of its piece}
            const int h = crd.y, c = crd.z;
            const float4 blk = blk_s[k];  // {A_cs[127], m, exact?, valid tokens}
            const float acs_r = acs_s[k * kQ + row];
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_x[k]);  // done with the step-0 values of the stage
            // step 3: S <- exp(A_cs[127]) S + exp(A_cs[127] - m) dS
            if (!(ok = wait_warp(&dsdone[db], (uint32_t)(t / DB) & 1u, abort_flag, status))) break;
            tc_fence_after();
            {
                const float gam = ex2(blk.x), dsc = ex2(blk.x - blk.y);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tmem + ds_col(t) + 64 * set + 32 * half + lane_off, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int q = 0; q < 32; q += 2)
                        fma2_state(Sr[32 * half + q], Sr[32 * half + q + 1], gam, dsc, r[q], r[q + 1]);
                }
                tc_fence_before();
                mbar_arrive(&dsfree[db]);
            }
            const bool last_of_piece = crd.w != 0;
            if (last_of_piece) store_final(t);
            // S_in^T of the next task. With two buffers the one it goes to was last read by
            // Y_off of task t-1, which is done (the epilogue of t-1 waited for it).
            if (SB == 2 && t + 1 < ntask) {
                if (last_of_piece && !(ok = load_init(t + 1))) break;
                if (!(ok = write_st(t + 1))) break;
            }
            // epilogue: y = exp(A_cs[l] - m) Y in the factored form, y = Y in the exact form (D x is
            // inside Y)
            if (!(ok = wait_warp(&yfull[yb], (uint32_t)(t / YB) & 1u, abort_flag, status))) break;
            tc_fence_after();
            if (set == 0) {
                // y rows of this warp (32 tokens x 64 values) are staged, 128-byte swizzled, in its
                // 4 KB slice of the S^T buffer of task t (free: Y_off of task t is done) and written
                // by one bulk tensor store.
                const float rd = blk.z != 0.f ? 1.f : ex2(acs_r - blk.y);
                unsigned char *stage_y = st_buf(t % SB);
                const uint32_t ya = tmem + Cf::kTmY + 64 * yb + lane_off;
#pragma unroll 1
                for (int qq = 0; qq < 4; ++qq) {  // 16 columns at a time
                    uint32_t yv[16];
                    tmem_ld16(ya + 16 * qq, yv);
                    tmem_wait_ld();
                    if (qq == 3) {
                        tc_fence_before();
                        mbar_arrive(&yfree[yb]);
                    }
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = scale2_bf16(rd, __uint_as_float(yv[2 * e]), __uint_as_float(yv[2 * e + 1]));
                    *reinterpret_cast<uint4 *>(stage_y + swz(row, 2 * qq)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4 *>(stage_y + swz(row, 2 * qq + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
                }
                fence_proxy_async();
                __syncwarp();
                const int r0 = c * kQ + 32 * qtr;
                if (lane == 0 && r0 < L) {
                    const int b = crd.x;
                    tma_store_4d(&tm_y, stage_y + 32 * qtr * 128, 0, h, r0, b, policy_evict_first());
                    bulk_commit();
                }
            }
            // with one S^T buffer it is free only now (Y_off of task t is done)
            if (SB == 1 && t + 1 < ntask) {
                if (last_of_piece && !(ok = load_init(t + 1))) break;
                if (!(ok = write_st(t + 1))) break;
            }
        }
    }

    if (warp >= kWarpE && lane == 0) bulk_wait_all();  // y stores have read their staging slices
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpG) {
        if (lane == 0) {  // every issued MMA has completed before TMEM is released
            const unsigned long long t0 = now_ns();
            while (!mbar_try(fin, 0) && now_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cf::kTmCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------------
// host side

template <int N>
cudaError_t launch(const FwdProblem &p, int *status, int *flags, float *handover, int grid, cudaStream_t s) {
    CUtensorMap tx, tb, tcm, ty;
    if (!encode_4d(&tx, p.x, kP, p.H, p.L, p.B) || !encode_4d(&tb, p.Bm, N, p.G, p.L, p.B) ||
        !encode_4d(&tcm, p.Cm, N, p.G, p.L, p.B) || !encode_4d(&ty, p.y, kP, p.H, p.L, p.B, 32))
        return cudaErrorInvalidValue;
    Params prm;
    prm.dt = static_cast<const __nv_bfloat16 *>(p.dt);
    prm.A = p.A;
    prm.D = p.D;
    prm.h0 = p.h0;
    prm.h_final = p.h_final;
    prm.y = static_cast<__nv_bfloat16 *>(p.y);
    prm.status = status;
    prm.wait_us = wait_limit_us();
    prm.flags = flags;
    prm.handover = handover;
    prm.L = p.L;
    prm.H = (int)p.H;
    prm.G = (int)p.G;
    prm.nc = (int)((p.L + kQ - 1) / kQ);
    prm.total = p.B * p.H * (long long)prm.nc;
    cudaError_t e = cudaFuncSetAttribute(k_ssd_tc<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<N>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    // All CTAs must be resident together (a CTA may wait for the state its neighbour hands
    // over), which a cooperative launch guarantees.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Cfg<N>::kThreads);
    cfg.dynamicSmemBytes = Cfg<N>::kSmemAlloc;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_ssd_tc<N>, tx, tb, tcm, ty, prm);
}

}  // namespace tc

bool tc_supported(const FwdProblem &p) {
    return p.dtype == SSD_BF16 && p.P == tc::kP && (p.N == 128 || p.N == 256) && (p.Q == 128 || p.Q == 256) &&
           p.L >= 1 && p.L < (1ll << 31) && p.B * p.H < (1ll << 31);
}

// Workspace: [status int | pad][flags int x grid | pad][hand-over states fp32 grid x P x N]
// With at least as many streams as SMs every CTA's share covers a whole stream or more,
// so a cut stream spans exactly two CTAs and the part that waits never waits on a part
// that waits itself. With fewer streams each CTA takes one whole stream.
static int tc_grid(const FwdProblem &p) {
    const int sms = tc::num_sms() > 0 ? tc::num_sms() : 148;
    const long long streams = p.B * p.H;
    return (int)std::max(1ll, streams >= sms ? (long long)sms : streams);
}

size_t tc_fwd_workspace_bytes(const FwdProblem &p) {
    if (tc_pair_supported(p)) return tc_pair_workspace_bytes(p);
    const size_t g = (size_t)tc_grid(p);
    return kWsAlign + align_up(g * sizeof(int), kWsAlign) + g * (size_t)(tc::kP * p.N) * sizeof(float);
}

// Two heads per task (C B^T shared) where the heads pair up within groups; one head otherwise.
cudaError_t tc_fwd(const FwdProblem &p, void *ws, cudaStream_t s) {
    if (tc_pair_supported(p)) return tc_pair_fwd(p, ws, s);
    const int grid = tc_grid(p);
    char *base = static_cast<char *>(ws);
    int *status = reinterpret_cast<int *>(base);
    int *flags = reinterpret_cast<int *>(base + kWsAlign);
    float *handover = reinterpret_cast<float *>(base + kWsAlign + align_up((size_t)grid * sizeof(int), kWsAlign));
    cudaError_t e = cudaMemsetAsync(base, 0, kWsAlign + (size_t)grid * sizeof(int), s);
    if (e != cudaSuccess) return e;
    return p.N == 128 ? tc::launch<128>(p, status, flags, handover, grid, s)
                      : tc::launch<256>(p, status, flags, handover, grid, s);
}

}  // namespace ssd
