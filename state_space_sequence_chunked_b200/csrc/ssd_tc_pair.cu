// Fused chunked SSD forward on tcgen05 (sm_100a) for a PAIR of heads per task.
//
// The same four steps as the one-head kernel (Mamba-2 SSD write-up, "SSD 算法：分块和状态传递",
// with the 128-token diagonal blocks of "SSD 算法：分块矩阵分解"), but a task is one 128-token
// block of two heads (2q, 2q+1) of one group, which share B and C. Per task:
//   step 0  A_cs_e[l] = sum_{j<=l} dt_{e,j} A_e            (log2 domain, per head e)
//   step 1  G = C B^T once for both heads (TMEM); G' = causal part of G in bf16, shared
//   step 2  dS^T = B^T [X''_0 | X''_1]                      (one N = 128 product)
//   step 3  S_e <- exp(A_cs_e[127]) S_e + exp(A_cs_e[127] - m_e) dS_e
//   step 4  Y = C [s_0 S_0 | s_1 S_1]^T + G' [X''_0 | X''_1]            (one accumulator)
//           y_e = exp(A_cs_e[l] - m_e) (Y_e + (D_e / dt_{e,l}) X''_e[l])
// with the factored decay of the one-head kernel: m_e is the middle of head e's A_cs range,
// X''_e[s] = exp(m_e - A_cs_e[s]) dt_{e,s} x_{e,s} in place, s_e = exp(m_e). The D skip term
// cannot ride on G''s diagonal (G' is shared), so the epilogue adds it from X''.
//
// The running state stays in TMEM, in the chunk-state accumulator itself: before the chunk-
// state product of block t the accumulator holds (gamma_t / dsc_t) S_t (gamma_t = exp(A_cs[127]),
// dsc_t the factor of dS above), the product adds dS_t, and the result is S_{t+1} / dsc_t.
// Between the two products one pass over the accumulator (the S warps) recovers S_{t+1}, writes
// its bf16 copy for step 4 of block t+1 and rescales the accumulator for block t+1.
//
// A block is factored for a head when its A_cs range is at most 192 (log2 units) and every
// valid token has |dt| >= 2^-40. The row and column factors then stay within 2^+-96, which
// leaves 2^31 of the exponent range that fp32 and bf16 share (up to 2^127) for |dt x| and the
// 128-term sums of the products; a decay factor below 2^-126 flushes to 0, as the true value
// is negligible next to the terms it is added to. A pair task in which either head's block is
// not factored runs as two single-head tasks in the exact form of head e, with N = 64 products
// on that head's columns only, factored by quarters of 32 tokens (mid_q the middle of quarter
// q's A_cs span):
//   X'''_e[s] = exp(mid_q(s) - A_cs_e[s]) dt_s x_s goes into the other head's half of the x slot
//   (x_e stays in its own half); G'_e[l,s] = G[l,s] exp(A_cs_e[l] - mid_q(s)) for s <= l (one
//   exp per row and quarter; element by element when a quarter spans more than 224); the other
//   head's X warps scale B's rows by exp(A_cs_e[127] - A_cs_e[s]) dt_s in place once C B^T has
//   read B, so the chunk state is B'^T x_e; the rows of C are scaled by exp(A_cs_e[l]) in place;
//   S_e enters unscaled and y_e = Y_e + D_e x_e. The other head's state is kept.
//
// Work split, cut streams and the hand-over are those of the one-head kernel, over pair
// streams (batch row, head pair): a persistent grid splits the pair tasks into equal shares;
// a stream cut between two CTAs hands its state over through global memory (the state
// passing of "序列并行" inside one GPU), ready long before it is read.
//
// Warp roles (1024 threads): warp 2 ("describer") fetches the dt of both heads one task ahead,
// runs step 0 for both heads at once, decides the task's form, writes a descriptor into a ring
// of four and issues the TMA loads of C and B; warp 0 loads x (each head's half as soon as its
// previous y has left the slot) and prefetches the next task's x into L2; warp 1 issues C B^T
// and the chunk states; warp 3 issues Y; warps 4-7 ("T") write G' (and scale C in the exact
// form); warps 8-15 ("X", 8 + 4 e + quarter for head e) write X'' of their head (in the exact
// form X''' or B's rows); warps 16-23 ("S", the same layout) run its state pass; warps 24-31
// ("O", the same layout) run the epilogue, staging y in the x slot it came from. The jobs
// overlap: X'' of block t+1, the state pass of block t+1 and the epilogue of block t run at the
// same time. Each warp touches only the TMEM lane quarter of its warp index. Rings: C and B in
// two 64 KB stages, x in two 32 KB slots, one S^T buffer; TMEM: two C B^T buffers, one state
// and one output accumulator of 128 columns each. Every wait is bounded; on timeout the CTA
// raises bit 0 of the status word, drains its own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "tc_ptx.cuh"

namespace ssd {
namespace tcp {
using namespace tc;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr int kThreads = 1024;
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpDesc = 2, kWarpY = 3, kWarpT = 4, kWarpX = 8, kWarpS = 16, kWarpO = 24;
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory (base 1024-byte aligned; every buffer is a whole number of swizzle atoms)
constexpr int kPanel = kQ * 128;               // 128 rows x 128 B (64 bf16)
constexpr int kOffCB = 0;                      // [2] stages: C panels 0, 1, B panels 0, 1
constexpr int kCBStage = 4 * kPanel;
constexpr int kOffX = 2 * kCBStage;            // [2] slots: x of head 0, x of head 1
constexpr int kXSlot = 2 * kPanel;
constexpr int kOffS = kOffX + 2 * kXSlot;      // S^T: [n][p] panel per head (MN-major B operand)
// Task descriptors, a ring of 4 (task t in entry t & 3): C and B of a task are loaded up to two
// tasks before its x, so a descriptor lives longer than one x slot.
constexpr int kRing = 4;
constexpr int kOffDt = kOffS + 2 * kPanel;        // bf16 dt [ring][2 heads][128]
constexpr int kOffHd = kOffDt + kRing * 2 * kQ * 2;  // Head0 [ring][2 heads]: step-0 scalars
constexpr int kOffCrd = kOffHd + kRing * 2 * 32;  // int4 [ring]: task descriptor
constexpr int kOffBar = kOffCrd + kRing * 16;
constexpr int kNumBars = 35;
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM base, abort flag
constexpr int kSmemBytes = kOffMisc + 16;
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint32_t kTxCB = 4 * kPanel, kTxXHead = kPanel;

// TMEM columns
constexpr uint32_t kTmG = 0;     // [2] x 128: C B^T (fp32), then G' (bf16) in its first 64
constexpr uint32_t kTmS = 256;   // running state / chunk states [n][(e, p)]
constexpr uint32_t kTmY = 384;   // Y [l][(e, p)]
constexpr int kTmCols = 512;

// Task descriptor: {b, pair, c, flags}
constexpr int kModePair = 0, kModeSingle0 = 1, kModeSingle1 = 2;
constexpr int kFlagLast = 4, kFlagEnd = 8;  // last task of its piece; no more tasks

struct Params {
    const __nv_bfloat16 *dt;
    const float *A, *D, *h0;
    float *h_final;
    int *status;       // bit 0: a bounded wait ran out; bit 1: shared memory misaligned
    int *flags;        // [gridDim.x] hand-over counters (zeroed before the launch)
    float *handover;   // [gridDim.x][2][P][N]
    long long L;
    int total;           // B * (H / 2) * nc pair tasks
    int H, G, nc;
    int wait_us;         // bounded-wait limit in microseconds (0: the built-in one)
};

// Share of CTA i in (pair stream, block) task order, run as [b0, hi), [a0, b0), [lo, a0): the
// start of the last stream first, whole streams, then the rest of the stream begun by CTA i-1.
// (The host admits fewer than 2^31 pair tasks.)
struct Share {
    int lo, hi, a0, b0;
    __device__ __forceinline__ int count() const { return hi - lo; }
    __device__ __forceinline__ int task(int t) const {
        const int n1 = hi - b0, n2 = b0 - a0;
        return t < n1 ? b0 + t : (t < n1 + n2 ? a0 + (t - n1) : lo + (t - n1 - n2));
    }
};
__device__ __forceinline__ Share share_of(int total, int nc, int i, int nblk) {
    const int q = total / nblk, r = total % nblk;
    Share s;
    s.lo = q * i + (int)(((long long)r * i) / nblk);
    s.hi = q * (i + 1) + (int)(((long long)r * (i + 1)) / nblk);
    s.a0 = min(((s.lo + nc - 1) / nc) * nc, s.hi);
    s.b0 = max((s.hi / nc) * nc, s.a0);
    return s;
}

// Step 0 for the 32 tokens of one lane quarter (token 32 q + lane), given the cumsum at the
// end of the previous quarters (off): the inclusive cumsum of dt A (log2 domain). Rounded
// operations only, so that every warp that runs it for the same quarter gets the same bits.
__device__ __forceinline__ float quarter_cumsum(float dt, float a2, float off, int lane) {
    float incl = __fmul_rn(dt, a2);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl = __fadd_rn(incl, u);
    }
    return __fadd_rn(off, incl);
}

// Per head and task, written by the describer warp next to the task's dt: the middle m of the
// block's A_cs range, the block total, the cumsum at the end of quarters 0, 1, 2, A_h log2(e)
// and D_h (0 without D).
struct Head0 {
    float m, tot, off1, off2, off3, a2, Dh, pad;
    __device__ __forceinline__ float off(int q) const { return q == 0 ? 0.f : (q == 1 ? off1 : (q == 2 ? off2 : off3)); }
    // the middle of quarter q's A_cs span (its bounds: the cumsum before it and at its end)
    __device__ __forceinline__ float qmid(int q) const { return 0.5f * (off(q) + (q == 3 ? tot : off(q + 1))); }
    // The exact form factors a block by quarters unless a quarter spans more than 224 of A_cs
    // (its factors then stay within 2^+-112); past that it takes exp(A_cs[l] - A_cs[s]) element
    // by element.
    __device__ __forceinline__ bool fine() const {
        const float w = fmaxf(fmaxf(-off1, off1 - off2), fmaxf(off2 - off3, off3 - tot));
        return !(w <= 224.f);  // (NaN: element by element)
    }
};

// w x for a bf16 pair x, rounded once to bf16 up to a few units in 2^-17: w is split into
// w_hi + w_lo (each bf16), and bf16(w_hi x + bf16(w_lo x)) is formed with packed bf16 ops.
__device__ __forceinline__ uint32_t scale_pair(uint32_t w_hi2, uint32_t w_lo2, uint32_t x) {
    uint32_t lo, r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(w_lo2), "r"(x));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(w_hi2), "r"(x), "r"(lo));
    return r;
}
__device__ __forceinline__ void split_bf16x2(float w, uint32_t &hi2, uint32_t &lo2) {
    hi2 = pack_bf16(w, w);
    const float r = w - bf16_lo(hi2);  // exact: w minus w rounded to 8 significant bits
    lo2 = pack_bf16(r, r);
}

// Row `row` of a 128-byte-swizzled bf16 tile, scaled by w, from src to dst (packed bf16 ops).
__device__ __forceinline__ void scale_row(const unsigned char *src, unsigned char *dst, int row, float w) {
    uint32_t wh, wl;
    split_bf16x2(w, wh, wl);
#pragma unroll 1
    for (int h4 = 0; h4 < 2; ++h4) {  // half a row at a time: four loads in flight
        uint4 xv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) xv[c] = *reinterpret_cast<const uint4 *>(src + swz(row, 4 * h4 + c));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint4 o;
            o.x = scale_pair(wh, wl, xv[c].x);
            o.y = scale_pair(wh, wl, xv[c].y);
            o.z = scale_pair(wh, wl, xv[c].z);
            o.w = scale_pair(wh, wl, xv[c].w);
            *reinterpret_cast<uint4 *>(dst + swz(row, 4 * h4 + c)) = o;
        }
    }
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// (a, b) * w on a packed fp32 pair, returned as two 32-bit words.
__device__ __forceinline__ void mul2(float w, uint32_t a, uint32_t b, uint32_t &ra, uint32_t &rb) {
    asm("{\n\t.reg .b64 v, ww;\n\t"
        "mov.b64 v, {%2, %3};\n\tmov.b64 ww, {%4, %4};\n\t"
        "mul.rn.f32x2 v, v, ww;\n\t"
        "mov.b64 {%0, %1}, v;\n\t}"
        : "=r"(ra), "=r"(rb)
        : "r"(a), "r"(b), "f"(w));
}

// bf16 pair of w (y + d x) for fp32 y = (y0, y1) and a bf16 pair x, in packed fp32 pairs: the
// same roundings as fmaf(d, x, y) then w * that, rounded to bf16.
__device__ __forceinline__ uint32_t skip2_bf16(float w, float d, uint32_t y0, uint32_t y1, uint32_t x) {
    uint32_t o;
    asm("{\n\t.reg .b64 v, xx, ww, dd;\n\t.reg .b32 xl, xh;\n\t.reg .f32 lo, hi;\n\t"
        "shl.b32 xl, %4, 16;\n\tand.b32 xh, %4, 0xFFFF0000;\n\t"
        "mov.b64 v, {%2, %3};\n\tmov.b64 xx, {xl, xh};\n\tmov.b64 ww, {%1, %1};\n\tmov.b64 dd, {%5, %5};\n\t"
        "fma.rn.f32x2 v, dd, xx, v;\n\tmul.rn.f32x2 v, v, ww;\n\t"
        "mov.b64 {lo, hi}, v;\n\tcvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(o)
        : "f"(w), "r"(y0), "r"(y1), "r"(x), "f"(d));
    return o;
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

__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ uint32_t ld_dt_pair(const __nv_bfloat16 *p, uint64_t pol) {
    uint32_t v;
    asm volatile("ld.global.nc.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(v) : "l"(p), "l"(pol));
    return v;
}

// Per head and block, the factors of the state pass (gamma = exp(A_cs[127])): dsc scales the
// block's chunk-state product (the accumulator then holds S_{t+1} / dsc), sg the bf16 copy of
// the state for the state-to-output product, rs the state the accumulator holds before the
// product ((gamma / dsc) S). Factored: dsc = exp(A_cs[127] - m), sg = rs = exp(m). The head of
// a single-head (exact) task: dsc = sg = 1, rs = gamma (its state enters unscaled). The other
// head of a single-head task keeps its state: all 1.
struct StateF {
    float dsc, sg, rs;
};
__device__ __forceinline__ StateF state_factors(const Head0 &hd, int mode, int e) {
    StateF f{1.f, 1.f, 1.f};
    if (mode == kModePair) {
        f.dsc = ex2(hd.tot - hd.m);
        f.sg = f.rs = ex2(hd.m);
    } else if (mode == kModeSingle0 + e) {
        f.rs = ex2(hd.tot);
    }
    return f;
}

// ---------------------------------------------------------------------------------------------
// The exact form's two per-task jobs, out of line: they run only for blocks whose decay range
// is too wide for the factored form, and kept inline they would lengthen the code every
// factored block runs through.

// T warp (rows 32 qtr .. 32 qtr + 31) for head ea of an exact task, once C B^T is in the G
// buffer at gaddr (this warp's lanes): G' of head ea in place, then C's rows scaled by
// exp(A_cs[l]) in place (the state term's row factor, which the exact form cannot share with the
// G' product). Factored by quarters: with X'''_s = exp(mid_q(s) - A_cs[s]) dt_s x_s (mid_q the
// middle of s's quarter), G'[l,s] = (C B^T)[l,s] exp(A_cs[l] - mid_q(s)), one factor per row and
// quarter; a quarter spanning more than 224 of A_cs instead takes X'''_s = dt_s x_s and
// G'[l,s] = (C B^T)[l,s] exp(A_cs[l] - A_cs[s]) element by element.
__device__ __noinline__ void t_exact(unsigned char *cst, uint32_t gaddr, const Head0 hx, const __nv_bfloat16 *dtrow,
                                     int qtr, int lane) {
    const int row = (qtr << 5) | lane;
    float acs_r;
    if (!hx.fine()) {
        acs_r = quarter_cumsum(__bfloat162float(dtrow[row]), hx.a2, hx.off(qtr), lane);
#pragma unroll 1
        for (int jb = 0; jb < 4; ++jb) {
            uint32_t out[16];
            if (jb > qtr) {
#pragma unroll
                for (int i = 0; i < 16; ++i) out[i] = 0u;
            } else {
                uint32_t r[32];
                tmem_ld32(gaddr + 32 * jb, r);
                const float rf = ex2(acs_r - hx.qmid(jb));
                tmem_wait_ld(r);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float v0 = __uint_as_float(r[2 * i]), v1 = __uint_as_float(r[2 * i + 1]);
                    if (jb == qtr) {  // the diagonal quarter: s = 32 jb + 2 i (+1) against l = 32 jb + lane
                        v0 = 2 * i <= lane ? v0 : 0.f;
                        v1 = 2 * i + 1 <= lane ? v1 : 0.f;
                    }
                    out[i] = scale2_bf16(rf, v0, v1);
                }
            }
            tmem_st16(gaddr + 16 * jb, out);
        }
    } else {
        // the columns need step 0 of every quarter, so this warp runs all four
        float acq[4];  // token 32 jb + lane
#pragma unroll
        for (int jb = 0; jb < 4; ++jb)
            acq[jb] = quarter_cumsum(__bfloat162float(dtrow[32 * jb + lane]), hx.a2, hx.off(jb), lane);
        acs_r = qtr == 0 ? acq[0] : (qtr == 1 ? acq[1] : (qtr == 2 ? acq[2] : acq[3]));
#pragma unroll 1
        for (int pc = 0; pc < 8; ++pc) {
            const int jb = pc >> 1;
            uint32_t out[8];
            if (jb > qtr) {
#pragma unroll
                for (int i = 0; i < 8; ++i) out[i] = 0u;
            } else {
                const float aj = jb == 0 ? acq[0] : (jb == 1 ? acq[1] : (jb == 2 ? acq[2] : acq[3]));
                uint32_t r[16];
                tmem_ld16(gaddr + 16 * pc, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float v[2];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int ci = 16 * (pc & 1) + 2 * i + hh, col = 32 * jb + ci;
                        const float ac = __shfl_sync(0xffffffffu, aj, ci);
                        v[hh] = col <= row ? __uint_as_float(r[2 * i + hh]) * ex2(acs_r - ac) : 0.f;
                    }
                    out[i] = pack_bf16(v[0], v[1]);
                }
            }
            tmem_st8(gaddr + 8 * pc, out);
        }
    }
    const float el = ex2(acs_r);
    scale_row(cst, cst, row, el);
    scale_row(cst + kPanel, cst + kPanel, row, el);
    fence_proxy_async();
}

// X warp (row `row` of the block) of an exact task of head ea. xw (the warp belongs to head ea):
// X'''_ea[row] (see t_exact) into the other head's half of the slot, x_ea staying in its own
// for the chunk-state product and the skip term. Otherwise, once C B^T has read B: B[row,:] *=
// exp(A_cs[127] - A_cs[row]) dt_row in place, the chunk-state product's decay.
__device__ __noinline__ void x_exact(unsigned char *x_own, unsigned char *x_other, unsigned char *bst, const Head0 hd,
                                     const __nv_bfloat16 *dtrow, int qtr, int lane, bool xw) {
    const int row = (qtr << 5) | lane;
    const float dt_r = __bfloat162float(dtrow[row]);
    const float acs_r = quarter_cumsum(dt_r, hd.a2, hd.off(qtr), lane);
    if (xw) {
        scale_row(x_own, x_other, row, hd.fine() ? dt_r : ex2(hd.qmid(qtr) - acs_r) * dt_r);
    } else {
        const float w = ex2(hd.tot - acs_r) * dt_r;
        scale_row(bst, bst, row, w);
        scale_row(bst + kPanel, bst + kPanel, row, w);
    }
    fence_proxy_async();
}

__global__ void __launch_bounds__(kThreads, 1)
    k_ssd_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
               const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, const Params prm) {
    extern __shared__ __align__(1024) unsigned char sm[];
    if ((smem_u32(sm) & 1023u) != 0) {  // the swizzled layouts need 1024-byte alignment
        if (threadIdx.x == 0) atomicOr(prm.status, 2);
        return;
    }
    __nv_bfloat16 *dts = reinterpret_cast<__nv_bfloat16 *>(sm + kOffDt);
    Head0 *hds = reinterpret_cast<Head0 *>(sm + kOffHd);
    int4 *crd = reinterpret_cast<int4 *>(sm + kOffCrd);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint64_t *full_cb = bar;          // [2] C, B of the stage landed
    uint64_t *empty_cb = bar + 2;     // [2] C B^T, chunk-state and Y commits
    uint64_t *full_x = bar + 4;       // [2] x of the slot landed
    uint64_t *empty_x0 = bar + 6;     // [2] head 0's half of the slot free: its y stored (4 O warps)
    uint64_t *empty_x1 = bar + 33;    // [2] the same for head 1's half
    uint64_t *xpr = bar + 8;          // [2] X'' (or X') written (X warps)
    uint64_t *gfull = bar + 10;       // [2] C B^T in G buffer j
    uint64_t *gp = bar + 12;          // [2] G' written (T)
    uint64_t *ydd = bar + 14;         // [2] the G' product of G buffer j done
    uint64_t *dsx = bar + 16;         // [2] the chunk-state product of the slot's block done (x read)
    uint64_t *dsdone = bar + 18;      // chunk states added to the state accumulator
    uint64_t *dsfree = bar + 19;      // state accumulator rescaled for the next product (S)
    uint64_t *sready = bar + 20;      // S^T written (S)
    uint64_t *soff = bar + 21;        // the state-to-output product done (S^T read)
    uint64_t *yfull = bar + 22;       // Y done
    uint64_t *yfree = bar + 23;       // Y read (O)
    uint64_t *fin = bar + 24;         // every MMA of this CTA done (3 issuers)
    uint64_t *dfull = bar + 25;       // [ring] descriptor, dt and step-0 scalars of the entry written
    uint64_t *dfree = bar + 29;       // [ring] the entry's task done with (8 O warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
    int *status = prm.status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = prm.H, nc = prm.nc, npair = prm.H / 2, hpg = prm.H / prm.G;
    const long long L = prm.L;
    const Share sh = share_of(prm.total, nc, blockIdx.x, gridDim.x);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&dfull[i], 1);
            mbar_init(&dfree[i], 8);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full_cb[i], 1);
            mbar_init(&empty_cb[i], 2);  // the two MMA issuers
            mbar_init(&full_x[i], 1);
            mbar_init(&empty_x0[i], 4);  // head 0's 4 O warps
            mbar_init(&empty_x1[i], 4);  // head 1's
            mbar_init(&xpr[i], 256);  // the 8 X warps
            mbar_init(&gfull[i], 1);
            mbar_init(&gp[i], 128);
            mbar_init(&ydd[i], 1);
        }
        mbar_init(dsdone, 1);
        mbar_init(dsfree, 256);  // the 8 S warps
        mbar_init(sready, 256);  // the 8 S warps
        mbar_init(yfull, 1);
        mbar_init(yfree, 256);  // the 8 O warps
        mbar_init(fin, 2);  // the two MMA issuers
        mbar_init(&dsx[0], 1);
        mbar_init(&dsx[1], 1);
        mbar_init(soff, 1);
        *abort_flag = 0;
        abort_flag[1] = prm.wait_us;  // bounded-wait limit (us; 0: the built-in one)
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto cb_c = [&](int k) { return sm + kOffCB + k * kCBStage; };
    auto cb_b = [&](int k) { return sm + kOffCB + k * kCBStage + 2 * kPanel; };
    auto xslot = [&](int k) { return sm + kOffX + k * kXSlot; };
    unsigned char *stb = sm + kOffS;
    constexpr uint32_t kIdG = idesc(128, 128, false, false);
    constexpr uint32_t kIdDs = idesc(128, 128, true, true), kIdDs1 = idesc(128, 64, true, true);
    constexpr uint32_t kIdY = idesc(128, 128, false, true), kIdY1 = idesc(128, 64, false, true);

    if (warp == kWarpDesc) {
        // ------------------------------------------------------------- describe, and C and B
        // For each pair task in share order: its dt of both heads (fetched one task ahead), step 0
        // over the block for both heads (the scalars the other warps need) and its form (factored
        // for both heads, or two single-head exact tasks); then one descriptor per slot task, in
        // the ring entry its slot task index selects, once the entry's previous task is done, and
        // the TMA loads of the slot task's C and B. These run up to two tasks ahead of its x.
        const uint64_t pol_keep = policy_evict_last();
        uint32_t raw[4] = {0u, 0u, 0u, 0u};  // dt of both heads at tokens 4 lane .. 4 lane + 3 (bf16 pairs)
        int4 crd_raw = make_int4(0, 0, 0, 0);
        int nvalid_raw = 0;
        auto fetch = [&](int u) {
            const int gi = sh.task(u);
            const int sidx = gi / nc, c = gi - sidx * nc;
            const int b = sidx / npair, pr = sidx - b * npair;
            crd_raw = make_int4(b, pr, c, (c == nc - 1 || gi == sh.hi - 1) ? kFlagLast : 0);
            nvalid_raw = (int)min((long long)kQ, L - (long long)c * kQ);
            const long long t0 = (long long)c * kQ + 4 * lane;
            const __nv_bfloat16 *src = prm.dt + ((long long)b * L + t0) * H + 2 * pr;
#pragma unroll
            for (int m = 0; m < 4; ++m) raw[m] = t0 + m < L ? ld_dt_pair(src + (long long)m * H, pol_keep) : 0u;
        };
        const int ntask = sh.count();
        if (ntask > 0) fetch(0);
        int td = 0;  // slot tasks described
        bool ok = true;
        // the ring entry of slot task td is free once slot task td - 4 is done with (awaited in task
        // order: no parity aliasing)
        auto take_entry = [&]() -> bool {
            return td < kRing || wait_warp(&dfree[td & (kRing - 1)], (uint32_t)((td >> 2) - 1) & 1u, abort_flag, status);
        };
        for (int u = 0; ok && u < ntask; ++u) {
            const int4 cu = crd_raw;
            const int nvalid = nvalid_raw;
            const int h0i = 2 * cu.y;
            // Both heads in one pass: lanes 16 e .. 16 e + 15 take head e, lane g of the half
            // tokens 8 g .. 8 g + 7 (from the pairs that lanes 2 g and 2 g + 1 fetched).
            const int e = lane >> 4, g = lane & 15;
            uint32_t hv[4];  // this lane's 8 dt of head e, bf16 pairs in token order
            {
                uint32_t p0[4], p1[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    p0[m] = __shfl_sync(0xffffffffu, raw[m], 2 * g);
                    p1[m] = __shfl_sync(0xffffffffu, raw[m], 2 * g + 1);
                }
                // tokens 8 g + m from lane 2 g, 8 g + 4 + m from lane 2 g + 1; head e's half of each pair
                const uint32_t sh16 = e ? 16u : 0u;
                hv[0] = ((p0[0] >> sh16) & 0xFFFFu) | (((p0[1] >> sh16) & 0xFFFFu) << 16);
                hv[1] = ((p0[2] >> sh16) & 0xFFFFu) | (((p0[3] >> sh16) & 0xFFFFu) << 16);
                hv[2] = ((p1[0] >> sh16) & 0xFFFFu) | (((p1[1] >> sh16) & 0xFFFFu) << 16);
                hv[3] = ((p1[2] >> sh16) & 0xFFFFu) | (((p1[3] >> sh16) & 0xFFFFu) << 16);
            }
            const float a2 = __fmul_rn(__ldg(prm.A + h0i + e), kLog2e);
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float dv = (i & 1) ? bf16_hi(hv[i >> 1]) : bf16_lo(hv[i >> 1]);
                v[i] = i == 0 ? __fmul_rn(dv, a2) : __fmaf_rn(dv, a2, v[i - 1]);
            }
            float incl = v[7];
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
                const float q = __shfl_up_sync(0xffffffffu, incl, o, 16);
                if (g >= o) incl = __fadd_rn(incl, q);
            }
            const float excl = __fsub_rn(incl, v[7]);
            float mx = incl, mn = incl;
#pragma unroll
            for (int i = 0; i < 7; ++i) {
                const float ac = __fadd_rn(excl, v[i]);
                mx = fmaxf(mx, ac);
                mn = fminf(mn, ac);
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o, 16));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o, 16));
            }
            const int nv = nvalid - 8 * g;
            bool dt_ok = true;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float dv = (i & 1) ? bf16_hi(hv[i >> 1]) : bf16_lo(hv[i >> 1]);
                dt_ok = dt_ok && (nv <= i || fabsf(dv) >= 0x1p-40f);
            }
            // (mx - mn <= 192 is false for NaN, which then takes the exact form)
            const bool fact = __all_sync(0xffffffffu, dt_ok && (mx - mn <= 192.f));
            // Head0 = {m, tot, off1, off2, off3, a2, Dh, 0}; off q = the cumsum through token 32 q - 1;
            // lane 16 e + f (f < 8) holds field f of head e
            const float tot = __shfl_sync(0xffffffffu, incl, 15, 16), off1 = __shfl_sync(0xffffffffu, incl, 3, 16),
                        off2 = __shfl_sync(0xffffffffu, incl, 7, 16), off3 = __shfl_sync(0xffffffffu, incl, 11, 16);
            float hd_lane = 0.f;
            if (g == 0) hd_lane = __fmul_rn(0.5f, __fadd_rn(mx, mn));
            if (g == 1) hd_lane = tot;
            if (g == 2) hd_lane = off1;
            if (g == 3) hd_lane = off2;
            if (g == 4) hd_lane = off3;
            if (g == 5) hd_lane = a2;
            if (g == 6 && prm.D) hd_lane = __ldg(prm.D + h0i + e);
            if (u + 1 < ntask) fetch(u + 1);  // the next pair task's dt, in flight while this one is written
            const int nsub = fact ? 1 : 2;
            for (int sub = 0; sub < nsub; ++sub) {
                if (!(ok = take_entry())) break;
                const int d = td & (kRing - 1);
                const int mode = fact ? kModePair : (sub == 0 ? kModeSingle0 : kModeSingle1);
                const int flags = mode | ((sub == nsub - 1) ? (cu.w & kFlagLast) : 0);
                *reinterpret_cast<uint4 *>(dts + (d * 2 + e) * kQ + 8 * g) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                if (g < 8) reinterpret_cast<float *>(hds + 2 * d)[8 * e + g] = hd_lane;
                if (lane == 0) crd[d] = make_int4(cu.x, cu.y, cu.z, flags);
                __syncwarp();
                if (lane == 0) mbar_arrive(&dfull[d]);
                // C and B of the task, once its stage is free (slot task td - 2's products done).
                // Stage completions are awaited in task order, so their parities never alias.
                const int k = td & 1;
                if (td >= 2 && !(ok = wait_warp(&empty_cb[k], (uint32_t)((td - 2) >> 1) & 1u, abort_flag, status))) break;
                if (lane == 0) {
                    const int g = h0i / hpg, t0 = cu.z * kQ;
                    mbar_arrive_tx(&full_cb[k], kTxCB);
                    for (int pn = 0; pn < 2; ++pn) {
                        tma_load_4d_hint(cb_c(k) + pn * kPanel, &tm_c, &full_cb[k], 64 * pn, g, t0, cu.x, pol_keep);
                        tma_load_4d_hint(cb_b(k) + pn * kPanel, &tm_b, &full_cb[k], 64 * pn, g, t0, cu.x, pol_keep);
                    }
                }
                __syncwarp();
                ++td;
            }
        }
        // the end marker: consumers leave their loops when they read it; it reaches the MMA
        // issuers through the stage barrier
        if (ok && take_entry()) {
            const int d = td & (kRing - 1), k = td & 1;
            if (lane == 0) {
                crd[d] = make_int4(0, 0, 0, kFlagEnd);
                mbar_arrive(&dfull[d]);
            }
            __syncwarp();
            if (td < 2 || (ok = wait_warp(&empty_cb[k], (uint32_t)((td - 2) >> 1) & 1u, abort_flag, status))) {
                if (lane == 0) mbar_arrive(&full_cb[k]);
                __syncwarp();
                ++td;
            }
        }
        // drain: C and B loads still in flight land before the CTA exits (slot tasks below td
        // arrived on full_cb; the last phase of each stage covers every earlier load)
        if (lane == 0) {
            for (int k = 0; k < 2; ++k) {
                const unsigned long long w0 = now_ns();
                const int lc = ((td - 1) & 1) == k ? td - 1 : td - 2;
                if (lc >= 0)
                    while (!mbar_try(&full_cb[k], (uint32_t)(lc >> 1) & 1u) && now_ns() - w0 < kWaitNs) {
                    }
            }
        }
        __syncwarp();
    } else if (warp == kWarpLoad) {
        // ------------------------------------------------------------- x loads
        // In task order: once slot task tx is described and its slot free (slot task tx - 2's y
        // store has read it), the TMA loads of its x; the next task's x is prefetched into L2
        // first. Slot completions are awaited in task order, so their parities never alias.
        const uint64_t pol_stream = policy_evict_first();
        int last_x[2] = {-1, -1};
        if (lane == 0) {
            for (int tx = 0;; ++tx) {
                const int d = tx & (kRing - 1), k = tx & 1;
                if (!wait_phase(&dfull[d], (uint32_t)(tx >> 2) & 1u, abort_flag, status)) break;
                const int4 cd = crd[d];
                if (cd.w & kFlagEnd) break;
                const uint32_t pe = (uint32_t)((tx - 2) >> 1) & 1u;  // slot k's previous use
                const int d1 = (tx + 1) & (kRing - 1);
                if (mbar_test(&dfull[d1], (uint32_t)((tx + 1) >> 2) & 1u)) {
                    const int4 cf = crd[d1];
                    if (!(cf.w & kFlagEnd)) {
                        if ((cf.w & 3) == kModePair || (cf.w & 3) == kModeSingle0)
                            tma_prefetch_4d(&tm_x, 0, 2 * cf.y, cf.z * kQ, cf.x);
                        if ((cf.w & 3) == kModePair || (cf.w & 3) == kModeSingle1)
                            tma_prefetch_4d(&tm_x, 0, 2 * cf.y + 1, cf.z * kQ, cf.x);
                    }
                }
                const int mode = cd.w & 3, h0i = 2 * cd.y, t0 = cd.z * kQ;
                // each half as soon as its previous y is out (the exact form writes the other half too)
                if (mode == kModePair) {
                    mbar_arrive_tx(&full_x[k], 2 * kTxXHead);
                    if (tx >= 2 && !wait_phase(&empty_x0[k], pe, abort_flag, status)) break;
                    tma_load_4d_hint(xslot(k), &tm_x, &full_x[k], 0, h0i, t0, cd.x, pol_stream);
                    last_x[k] = tx;  // (an abort here still drains this load, with the bounded wait)
                    if (tx >= 2 && !wait_phase(&empty_x1[k], pe, abort_flag, status)) break;
                    tma_load_4d_hint(xslot(k) + kPanel, &tm_x, &full_x[k], 0, h0i + 1, t0, cd.x, pol_stream);
                } else {
                    const int e = mode == kModeSingle0 ? 0 : 1;
                    if (tx >= 2 && !(wait_phase(&empty_x0[k], pe, abort_flag, status) &&
                                     wait_phase(&empty_x1[k], pe, abort_flag, status)))
                        break;
                    mbar_arrive_tx(&full_x[k], kTxXHead);
                    tma_load_4d_hint(xslot(k) + e * kPanel, &tm_x, &full_x[k], 0, h0i + e, t0, cd.x, pol_stream);
                }
                // drain bookkeeping: the last x load of each slot
                last_x[k] = tx;
            }
            // drain: x loads still in flight land before the CTA exits
            for (int k = 0; k < 2; ++k) {
                const unsigned long long w0 = now_ns();
                if (last_x[k] >= 0)
                    while (!mbar_try(&full_x[k], (uint32_t)(last_x[k] >> 1) & 1u) && now_ns() - w0 < kWaitNs) {
                    }
            }
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------- G = C B^T and S += B^T [X''_0 | X''_1]
        // One thread issues both products of a block: G (M = l, N = s, K = n) as soon as C, B and
        // its G buffer are ready, the chunk states (M = n, N = (e, p), K = s) once X'' is written
        // and the state accumulator rescaled.
        if (lane == 0) {
            for (int t = 0;; ++t) {
                const int k = t & 1, j = t & 1;
                if (!wait_phase(&full_cb[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                const int fl = crd[t & (kRing - 1)].w;
                if (fl & kFlagEnd) break;
                if (t >= 2 && !wait_phase(&ydd[j], (uint32_t)((t - 2) >> 1) & 1u, abort_flag, status)) break;
                tc_fence_after();
                {
                    const uint64_t cd0 = sdesc(smem_u32(cb_c(k)), 16, 1024), bd0 = sdesc(smem_u32(cb_b(k)), 16, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
                        mma_ss(tmem + kTmG + 128 * j, cd0 + off, bd0 + off, kIdG, kk > 0);
                    }
                }
                mma_commit(&gfull[j]);
                if (!wait_phase(&xpr[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                if (!wait_phase(dsfree, (uint32_t)t & 1u, abort_flag, status)) break;
                tc_fence_after();
                const int mode = fl & 3;
                const uint64_t ad0 = sdesc(smem_u32(cb_b(k)), kPanel, 1024);
                if (mode == kModePair) {
                    const uint64_t xd0 = sdesc(smem_u32(xslot(k)), kPanel, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kQ / 16; ++kk) mma_ss(tmem + kTmS, ad0 + 128 * kk, xd0 + 128 * kk, kIdDs, 1);
                } else {  // head e's columns only: B' (rows of B scaled by the X warps) times raw x_e
                    const int e = mode == kModeSingle0 ? 0 : 1;
                    const uint64_t xd0 = sdesc(smem_u32(xslot(k) + e * kPanel), kPanel, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kQ / 16; ++kk)
                        mma_ss(tmem + kTmS + 64 * e, ad0 + 128 * kk, xd0 + 128 * kk, kIdDs1, 1);
                }
                mma_commit(dsdone);
                mma_commit(&dsx[k]);
                mma_commit(&empty_cb[k]);  // both products of this stage issued: one commit covers them
            }
            mma_commit(fin);
        }
        __syncwarp();
    } else if (warp == kWarpY) {
        // ------------------------------------------------------------- Y = C [s S_0 | s S_1]^T + G' [X''_0 | X''_1]
        // The state term first: it needs only S^T (written while the previous block finishes),
        // so the G' product, which waits for this block's x, is the only one after it.
        if (lane == 0) {
            for (int t = 0;; ++t) {
                const int k = t & 1, j = t & 1;
                if (!wait_phase(&full_cb[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                const int fl = crd[t & (kRing - 1)].w;
                if (fl & kFlagEnd) break;
                if (t >= 1 && !wait_phase(yfree, (uint32_t)(t - 1) & 1u, abort_flag, status)) break;
                if (!wait_phase(sready, (uint32_t)t & 1u, abort_flag, status)) break;
                const int mode = fl & 3;
                const uint64_t cd0 = sdesc(smem_u32(cb_c(k)), 16, 1024);
                if (mode == kModePair) {
                    tc_fence_after();
                    const uint64_t sd0 = sdesc(smem_u32(stb), kPanel, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
                        mma_ss(tmem + kTmY, cd0 + off, sd0 + 128 * kk, kIdY, kk > 0);
                    }
                    mma_commit(soff);
                    mma_commit(&empty_cb[k]);  // C's last reader: the stage is free once this and dS are done
                    if (!wait_phase(&gp[j], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                    if (!wait_phase(&xpr[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                    tc_fence_after();
                    const uint64_t xd0 = sdesc(smem_u32(xslot(k)), kPanel, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kQ / 16; ++kk)
                        mma_ts(tmem + kTmY, tmem + kTmG + 128 * j + 8 * kk, xd0 + 128 * kk, kIdY, 1);
                } else {
                    // head e's columns only; T has scaled the rows of C before G' was written
                    const int e = mode == kModeSingle0 ? 0 : 1;
                    if (!wait_phase(&gp[j], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                    if (!wait_phase(&xpr[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                    tc_fence_after();
                    const uint64_t sd0 = sdesc(smem_u32(stb + e * kPanel), kPanel, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
                        mma_ss(tmem + kTmY + 64 * e, cd0 + off, sd0 + 128 * kk, kIdY1, kk > 0);
                    }
                    mma_commit(soff);
                    mma_commit(&empty_cb[k]);
                    const uint64_t xd0 = sdesc(smem_u32(xslot(k) + (1 - e) * kPanel), kPanel, 1024);
#pragma unroll 1
                    for (int kk = 0; kk < kQ / 16; ++kk)
                        mma_ts(tmem + kTmY + 64 * e, tmem + kTmG + 128 * j + 8 * kk, xd0 + 128 * kk, kIdY1, 1);
                }
                mma_commit(&ydd[j]);
                mma_commit(yfull);
            }
            mma_commit(fin);
        }
        __syncwarp();
    } else if (warp >= kWarpT && warp < kWarpX) {
        // ------------------------------------------------------------- T: G' (and the exact form's C rows)
        const int qtr = warp & 3;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        for (int t = 0;; ++t) {
            const int k = t & 1, j = t & 1;
            const int dq = t & (kRing - 1);
            if (!wait_warp(&dfull[dq], (uint32_t)(t >> 2) & 1u, abort_flag, status)) break;
            const int4 cd = crd[dq];
            if (cd.w & kFlagEnd) break;
            const int mode = cd.w & 3;
            const uint32_t gaddr = tmem + kTmG + 128 * j + lane_off;
            if (!wait_warp(&gfull[j], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
            tc_fence_after();
            if (mode == kModePair) {
                // 32 columns per load, 16 packed bf16 pair columns per store: blocks jb < qtr are
                // converted as they are, the diagonal block jb == qtr masks s > row, blocks above
                // it are zeros
#pragma unroll 1
                for (int jb = 0; jb < 4; ++jb) {
                    uint32_t out[16];
                    if (jb > qtr) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) out[i] = 0u;
                    } else {
                        uint32_t r[32];
                        tmem_ld32(gaddr + 32 * jb, r);
                        tmem_wait_ld(r);
                        if (jb < qtr) {  // wholly below the diagonal
#pragma unroll
                            for (int i = 0; i < 16; ++i) out[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        } else {  // the diagonal block: s = 32 jb + 2 i (+1) against row = 32 jb + lane
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float v0 = 2 * i <= lane ? __uint_as_float(r[2 * i]) : 0.f;
                                const float v1 = 2 * i + 1 <= lane ? __uint_as_float(r[2 * i + 1]) : 0.f;
                                out[i] = pack_bf16(v0, v1);
                            }
                        }
                    }
                    tmem_st16(gaddr + 16 * jb, out);
                }
            } else {
                const int ea = mode == kModeSingle0 ? 0 : 1;
                t_exact(cb_c(k), gaddr, hds[2 * dq + ea], dts + (dq * 2 + ea) * kQ, qtr, lane);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&gp[j]);
        }
    } else if (warp < kWarpS) {
        // ------------------------------------------------------------- X: X'' (factored) of head e, or in the exact form X''' or B's rows
        const int qtr = warp & 3, e = (warp - kWarpX) >> 2;
        const int row = (qtr << 5) | lane;
        for (int t = 0;; ++t) {
            const int k = t & 1;
            const int dq = t & (kRing - 1);
            if (!wait_warp(&dfull[dq], (uint32_t)(t >> 2) & 1u, abort_flag, status)) break;
            const int4 cd = crd[dq];
            if (cd.w & kFlagEnd) break;
            const int mode = cd.w & 3;
            if (mode == kModePair) {
                if (!wait_warp(&full_x[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                const Head0 hd = hds[2 * dq + e];
                unsigned char *xs = xslot(k) + e * kPanel;
                const float dt_r = __bfloat162float(dts[(dq * 2 + e) * kQ + row]);
                const float acs_r = quarter_cumsum(dt_r, hd.a2, hd.off(qtr), lane);
                scale_row(xs, xs, row, ex2(hd.m - acs_r) * dt_r);
                fence_proxy_async();
            } else {  // exact form of head ea: X''' (its warps) or B's rows (the other head's)
                const int ea = mode == kModeSingle0 ? 0 : 1;
                if (!wait_warp(ea == e ? &full_x[k] : &gfull[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                tc_fence_after();
                x_exact(xslot(k) + ea * kPanel, xslot(k) + (1 - ea) * kPanel, cb_b(k), hds[2 * dq + ea],
                        dts + (dq * 2 + ea) * kQ, qtr, lane, ea == e);
            }
            mbar_arrive(&xpr[k]);
        }
    } else if (warp < kWarpO) {
        // ------------------------------------------------------------- S: the state pass of head e
        // Before the chunk-state product of block t, the accumulator holds S_t / dsc_{t-1} (the
        // previous product's output). In 16-column pieces: S_t = dsc_{t-1} * accumulator; at the
        // end of a piece S_t goes to h_final or the hand-over and the next piece's initial state
        // (h0, zeros, or the state handed over by the previous CTA) replaces it; the bf16 copy
        // sg * S_t goes to the S^T panel and the accumulator becomes (gamma / dsc) S_t.
        const int qtr = warp & 3, e = (warp - kWarpS) >> 2;
        const int row = (qtr << 5) | lane;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        const uint32_t sacc = tmem + kTmS + 64 * e + lane_off;  // this head's state rows
        unsigned char *pb = stb + e * kPanel;
        auto init_piece = [&](const int4 cd, int qq, float (&S)[16]) {
            const int h = 2 * cd.y + e;
            if (cd.z == 0) {
                const long long base = ((long long)cd.x * H + h) * kP * kN;
#pragma unroll
                for (int p = 0; p < 16; ++p) S[p] = prm.h0 ? prm.h0[base + (long long)(16 * qq + p) * kN + row] : 0.f;
            } else {
                const float *src = prm.handover + ((long long)(blockIdx.x - 1) * 2 + e) * kP * kN;
#pragma unroll
                for (int p = 0; p < 16; ++p) S[p] = __ldcg(src + (16 * qq + p) * kN + row);
            }
        };
        auto final_piece = [&](const int4 cd, int qq, const float (&S)[16]) {
            const int h = 2 * cd.y + e;
            if (cd.z == nc - 1) {
                if (prm.h_final) {
                    const long long base = ((long long)cd.x * H + h) * kP * kN;
#pragma unroll
                    for (int p = 0; p < 16; ++p) prm.h_final[base + (long long)(16 * qq + p) * kN + row] = S[p];
                }
            } else {
                float *dst = prm.handover + ((long long)blockIdx.x * 2 + e) * kP * kN;
#pragma unroll
                for (int p = 0; p < 16; ++p) __stcg(dst + (16 * qq + p) * kN + row, S[p]);
            }
        };
        // after every piece of a hand-over is stored: publish it
        auto publish = [&](const int4 cd) {
            if (cd.z != nc - 1) {
                __threadfence();
                atomicAdd(prm.flags + blockIdx.x, 1);
            }
        };
        bool ok = true;
        float dsc_prev = 1.f;
        int4 cprev = make_int4(0, 0, 0, 0);
        for (int t = 0; ok; ++t) {
            const int dq = t & (kRing - 1);
            if (!(ok = wait_warp(&dfull[dq], (uint32_t)(t >> 2) & 1u, abort_flag, status))) break;
            const int4 cd = crd[dq];
            if (cd.w & kFlagEnd) {
                // the last product's state is the final state of the last piece
                if (t > 0) {
                    if (!(ok = wait_warp(dsdone, (uint32_t)(t - 1) & 1u, abort_flag, status))) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int qq = 0; qq < 4; ++qq) {
                        uint32_t r[16];
                        float S[16];
                        tmem_ld16(sacc + 16 * qq, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int p = 0; p < 16; ++p) S[p] = dsc_prev * __uint_as_float(r[p]);
                        final_piece(cprev, qq, S);
                    }
                    publish(cprev);
                }
                break;
            }
            const int mode = cd.w & 3;
            const StateF f = state_factors(hds[2 * dq + e], mode, e);
            const bool from_acc = t > 0, ends = t > 0 && (cprev.w & kFlagLast) != 0;
            const bool starts = t == 0 || ends;
            if (from_acc) {
                if (!(ok = wait_warp(dsdone, (uint32_t)(t - 1) & 1u, abort_flag, status))) break;
                // the S^T panel is rewritten: the state-to-output product of block t-1 has read it
                if (!(ok = wait_warp(soff, (uint32_t)(t - 1) & 1u, abort_flag, status))) break;
                tc_fence_after();
            }
            // the hand-over this piece starts from must be complete before it is read
            if (starts && cd.z != 0 &&
                !(ok = __all_sync(0xffffffffu, wait_flag(prm.flags + blockIdx.x - 1, 256, abort_flag, status))))
                break;
            if (!starts) {
                // steady state, straight from the accumulator: S_t = dsc_prev acc, then sg S_t and
                // rs S_t. In the factored form sg = rs, and the two factors fold into one,
                // cs = sg dsc_prev, unless that product is below the normal range (both factors
                // can reach 2^-96); then they are applied one after the other.
                const float cs = f.sg * dsc_prev;
                const bool fold = f.sg == f.rs && cs >= 0x1p-120f;
                const float c0 = fold ? cs : dsc_prev;
#pragma unroll 1
                for (int qq = 0; qq < 4; ++qq) {
                    uint32_t r[16], v[16];
                    tmem_ld16(sacc + 16 * qq, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 16; p += 2) mul2(c0, r[p], r[p + 1], v[p], v[p + 1]);
                    uint4 o0, o1;
                    if (fold) {
                        o0 = make_uint4(pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                                        pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                                        pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                                        pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
                        o1 = make_uint4(pack_bf16(__uint_as_float(v[8]), __uint_as_float(v[9])),
                                        pack_bf16(__uint_as_float(v[10]), __uint_as_float(v[11])),
                                        pack_bf16(__uint_as_float(v[12]), __uint_as_float(v[13])),
                                        pack_bf16(__uint_as_float(v[14]), __uint_as_float(v[15])));
                    } else {  // v holds S_t
                        o0 = make_uint4(scale2_bf16(f.sg, __uint_as_float(v[0]), __uint_as_float(v[1])),
                                        scale2_bf16(f.sg, __uint_as_float(v[2]), __uint_as_float(v[3])),
                                        scale2_bf16(f.sg, __uint_as_float(v[4]), __uint_as_float(v[5])),
                                        scale2_bf16(f.sg, __uint_as_float(v[6]), __uint_as_float(v[7])));
                        o1 = make_uint4(scale2_bf16(f.sg, __uint_as_float(v[8]), __uint_as_float(v[9])),
                                        scale2_bf16(f.sg, __uint_as_float(v[10]), __uint_as_float(v[11])),
                                        scale2_bf16(f.sg, __uint_as_float(v[12]), __uint_as_float(v[13])),
                                        scale2_bf16(f.sg, __uint_as_float(v[14]), __uint_as_float(v[15])));
#pragma unroll
                        for (int p = 0; p < 16; p += 2) mul2(f.rs, v[p], v[p + 1], v[p], v[p + 1]);
                    }
                    *reinterpret_cast<uint4 *>(pb + swz(row, 2 * qq)) = o0;
                    *reinterpret_cast<uint4 *>(pb + swz(row, 2 * qq + 1)) = o1;
                    tmem_st16(sacc + 16 * qq, v);
                }
            } else {
#pragma unroll 1
                for (int qq = 0; qq < 4; ++qq) {
                    float S[16];
                    if (from_acc) {
                        uint32_t r[16];
                        tmem_ld16(sacc + 16 * qq, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int p = 0; p < 16; ++p) S[p] = dsc_prev * __uint_as_float(r[p]);
                        final_piece(cprev, qq, S);
                    }
                    init_piece(cd, qq, S);
                    uint4 o0, o1;
                    o0.x = scale2_bf16(f.sg, S[0], S[1]);
                    o0.y = scale2_bf16(f.sg, S[2], S[3]);
                    o0.z = scale2_bf16(f.sg, S[4], S[5]);
                    o0.w = scale2_bf16(f.sg, S[6], S[7]);
                    o1.x = scale2_bf16(f.sg, S[8], S[9]);
                    o1.y = scale2_bf16(f.sg, S[10], S[11]);
                    o1.z = scale2_bf16(f.sg, S[12], S[13]);
                    o1.w = scale2_bf16(f.sg, S[14], S[15]);
                    *reinterpret_cast<uint4 *>(pb + swz(row, 2 * qq)) = o0;
                    *reinterpret_cast<uint4 *>(pb + swz(row, 2 * qq + 1)) = o1;
                    uint32_t v[16];
#pragma unroll
                    for (int p = 0; p < 16; ++p) v[p] = __float_as_uint(f.rs * S[p]);
                    tmem_st16(sacc + 16 * qq, v);
                }
                if (ends) publish(cprev);
            }
            fence_proxy_async();
            mbar_arrive(sready);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(dsfree);
            dsc_prev = f.dsc;
            cprev = cd;
        }
    } else {
        // ------------------------------------------------------------- O: epilogue of head e
        // y = rd (Y + dd X''), staged over this head's x rows, one bulk tensor store per warp
        const int qtr = warp & 3, e = (warp - kWarpO) >> 2;
        const int row = (qtr << 5) | lane;
        const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
        for (int t = 0;; ++t) {
            const int k = t & 1;
            const int dq = t & (kRing - 1);
            if (!wait_warp(&dfull[dq], (uint32_t)(t >> 2) & 1u, abort_flag, status)) break;
            const int4 cd = crd[dq];
            if (cd.w & kFlagEnd) break;
            const int mode = cd.w & 3;
            const bool act = mode == kModePair || mode == kModeSingle0 + e;
            const int h = 2 * cd.y + e;
            float rd = 1.f, dd = 0.f;
            if (mode == kModePair) {
                const Head0 hd = hds[2 * dq + e];
                const float dt_r = __bfloat162float(dts[(dq * 2 + e) * kQ + row]);
                const float acs_r = quarter_cumsum(dt_r, hd.a2, hd.off(qtr), lane);
                rd = ex2(acs_r - hd.m);
                dd = dt_r != 0.f ? hd.Dh / dt_r : 0.f;
            } else if (act) {
                dd = hds[2 * dq + e].Dh;  // exact form: y = Y + D x, x still in this head's half
            }
            if (!wait_warp(yfull, (uint32_t)t & 1u, abort_flag, status)) break;
            tc_fence_after();
            unsigned char *xs = xslot(k) + e * kPanel;
            if (act) {
                // y overwrites X'', which the chunk-state product of this block reads too; X'' was
                // written by the X warps
                if (!wait_warp(&dsx[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                if (!wait_warp(&xpr[k], (uint32_t)(t >> 1) & 1u, abort_flag, status)) break;
                const uint32_t ya = tmem + kTmY + 64 * e + lane_off;
#pragma unroll 1
                for (int qq = 0; qq < 4; ++qq) {  // 16 columns (two 16-byte chunks) at a time
                    uint32_t yv[16];
                    tmem_ld16(ya + 16 * qq, yv);
                    uint4 xv[2];
                    if (dd != 0.f) {
                        xv[0] = *reinterpret_cast<const uint4 *>(xs + swz(row, 2 * qq));
                        xv[1] = *reinterpret_cast<const uint4 *>(xs + swz(row, 2 * qq + 1));
                    }
                    tmem_wait_ld();
                    if (qq == 3) {
                        tc_fence_before();
                        mbar_arrive(yfree);
                    }
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const uint32_t *yy = yv + 8 * c2;
                        uint4 o;
                        if (dd != 0.f) {
                            o.x = skip2_bf16(rd, dd, yy[0], yy[1], xv[c2].x);
                            o.y = skip2_bf16(rd, dd, yy[2], yy[3], xv[c2].y);
                            o.z = skip2_bf16(rd, dd, yy[4], yy[5], xv[c2].z);
                            o.w = skip2_bf16(rd, dd, yy[6], yy[7], xv[c2].w);
                        } else {
                            o = make_uint4(scale2_bf16(rd, __uint_as_float(yy[0]), __uint_as_float(yy[1])),
                                           scale2_bf16(rd, __uint_as_float(yy[2]), __uint_as_float(yy[3])),
                                           scale2_bf16(rd, __uint_as_float(yy[4]), __uint_as_float(yy[5])),
                                           scale2_bf16(rd, __uint_as_float(yy[6]), __uint_as_float(yy[7])));
                        }
                        *reinterpret_cast<uint4 *>(xs + swz(row, 2 * qq + c2)) = o;
                    }
                }
                fence_proxy_async();
                __syncwarp();
                const long long r0 = (long long)cd.z * kQ + 32 * qtr;
                if (lane == 0) {
                    if (r0 < L) {
                        tma_store_4d(&tm_y, xs + 32 * qtr * 128, 0, h, (int)r0, cd.x, policy_evict_first());
                        bulk_commit();
                    }
                    bulk_wait_read();  // the slot is reloaded once every warp's store has read it
                }
            } else {
                tc_fence_before();
                mbar_arrive(yfree);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(e ? &empty_x1[k] : &empty_x0[k]);
                mbar_arrive(&dfree[dq]);
            }
        }
    }

    if (warp >= kWarpO && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) {
        if (lane == 0) {  // every issued MMA has completed before TMEM is released
            const unsigned long long t0 = now_ns();
            while (!mbar_try(fin, 0) && now_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmCols) : "memory");
    }
}

}  // namespace tcp

bool tc_pair_supported(const FwdProblem &p) {
    const long long tasks = p.B * (p.H / 2) * ((p.L + tcp::kQ - 1) / tcp::kQ);
    return p.dtype == SSD_BF16 && p.P == tcp::kP && p.N == tcp::kN && (p.Q == 128 || p.Q == 256) && p.L >= 1 &&
           p.L < (1ll << 31) && p.B * p.H < (1ll << 31) && (p.H / p.G) % 2 == 0 && tasks < (1ll << 31);
}

// With at least as many pair streams as SMs every share covers a whole stream or more, so
// a cut stream spans exactly two CTAs; with fewer, each CTA takes one whole stream.
int tc_pair_grid(const FwdProblem &p) {
    const int sms = tc::num_sms() > 0 ? tc::num_sms() : 148;
    const long long streams = p.B * (p.H / 2);
    return (int)std::max(1ll, streams >= sms ? (long long)sms : streams);
}

// Workspace: [status int | pad][flags int x grid | pad][hand-over states fp32 grid x 2 x P x N]
size_t tc_pair_workspace_bytes(const FwdProblem &p) {
    const size_t g = (size_t)tc_pair_grid(p);
    return kWsAlign + align_up(g * sizeof(int), kWsAlign) + g * 2 * (size_t)(tcp::kP * tcp::kN) * sizeof(float);
}

cudaError_t tc_pair_fwd(const FwdProblem &p, void *ws, cudaStream_t s) {
    using namespace tcp;
    const int grid = tc_pair_grid(p);
    char *base = static_cast<char *>(ws);
    int *status = reinterpret_cast<int *>(base);
    int *flags = reinterpret_cast<int *>(base + kWsAlign);
    float *handover = reinterpret_cast<float *>(base + kWsAlign + align_up((size_t)grid * sizeof(int), kWsAlign));
    cudaError_t e = cudaMemsetAsync(base, 0, kWsAlign + (size_t)grid * sizeof(int), s);
    if (e != cudaSuccess) return e;
    CUtensorMap tx, tb, tcm, ty;
    if (!encode_4d(&tx, p.x, kP, p.H, p.L, p.B) || !encode_4d(&tb, p.Bm, kN, p.G, p.L, p.B) ||
        !encode_4d(&tcm, p.Cm, kN, p.G, p.L, p.B) || !encode_4d(&ty, p.y, kP, p.H, p.L, p.B, 32))
        return cudaErrorInvalidValue;
    Params prm;
    prm.dt = static_cast<const __nv_bfloat16 *>(p.dt);
    prm.A = p.A;
    prm.D = p.D;
    prm.h0 = p.h0;
    prm.h_final = p.h_final;
    prm.status = status;
    prm.wait_us = wait_limit_us();
    prm.flags = flags;
    prm.handover = handover;
    prm.L = p.L;
    prm.H = (int)p.H;
    prm.G = (int)p.G;
    prm.nc = (int)((p.L + kQ - 1) / kQ);
    prm.total = (int)(p.B * (p.H / 2) * (long long)prm.nc);
    e = cudaFuncSetAttribute(k_ssd_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // All CTAs must be resident together (a CTA may wait for the state its neighbour hands
    // over), which a cooperative launch guarantees.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_ssd_pair, tx, tb, tcm, ty, prm);
}

}  // namespace ssd
