// The context-parallel state-to-output correction on tcgen05 tensor cores.
//
// For a segment of the sequence and the state S_in entering it (the exclusive scan of the
// ranks' end states, "序列并行" in the Mamba-2 SSD write-up), every token's output gains
//     y_t[h, :] += exp(sum_{s <= t in segment} dt_s A_h) * S_in[h] C_t
// which is step 4 of the chunked algorithm ("SSD 算法：分块和状态传递") for the incoming state.
// Over one 128-token block and two heads of one group it is a single matrix product
//     Y[t, (h, p)] = sum_n C[t, n] S_in[h, p, n]        (M = 128 tokens, N = 2 x 64, K = dstate)
// followed by a per-(token, head) scaling. A CTA takes one head pair of one batch row and a run
// of consecutive 128-token blocks, all of which share S_in, and pipelines them:
//   - the 8 epilogue warps first write S_in once, converted to bf16, K-major with 128-byte
//     swizzle;
//   - warp 8 (one thread) loads each block's C panel by panel into one buffer (a panel is
//     reloaded for the next block as soon as this block's MMAs on it are done) and the two
//     heads' y tiles (two buffers), issues the block's dstate / 16 MMAs (M = 128, N = 128),
//     panel by panel, into one of two TMEM accumulators, and stores each block's y tiles once
//     the epilogue has updated them, so block i+1's loads and MMAs run during block i's
//     epilogue;
//   - in the epilogue, warps 0-1 form the decay factors of the two heads; each warp reads its
//     TMEM lane quarter for one head and updates the y tile in shared memory.
// Every wait is bounded; a wait that runs out sets bit 0 of *status (when given) and the CTA
// skips the rest of its work.
#include <algorithm>

#include "tc_ptx.cuh"

namespace ssd {
namespace cpt {
using namespace tc;

constexpr int kBlk = 128;      // tokens per block
constexpr int kP = 64;         // head dimension this kernel takes
constexpr int kPanel = 16384;  // one 64-column panel of a 128-row K-major tile, bytes
constexpr int kThreads = 288;  // 8 epilogue warps and the producer warp
constexpr int kEpi = 256;      // epilogue threads

struct Params {
    const __nv_bfloat16 *dt;
    const float *A, *bsum, *s_in;
    int *status;
    long long L;
    int H, G, N, nblk, pairs_per_group, blocks_per_cta;
    int wait_us;  // bounded-wait limit in microseconds (0: the built-in one)
};

// Shared memory (after 1024-byte alignment): S_in tile [N/64 panels], C tile [N/64 panels],
// y tiles [2 buffers][2 heads][128 rows x 128 B], cum [2 buffers][2 heads][128] fp32, 16 barriers,
// TMEM base, abort flag and wait limit.
__host__ __device__ constexpr int smem_bytes(int N) { return 2 * (N / 64) * kPanel + 4 * kPanel + 4 * kBlk * 4 + 192; }

__global__ void __launch_bounds__(kThreads, 1)
    k_correct_tc(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, const Params prm) {
    extern __shared__ unsigned char cpt_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(cpt_raw) + 1023) & ~uintptr_t(1023));
    const int N = prm.N, npan = N / 64;
    unsigned char *s_tile = sm;
    unsigned char *c_tile = sm + npan * kPanel;
    unsigned char *y_tile = sm + 2 * npan * kPanel;  // [2][2][16 KB]
    float *cum = reinterpret_cast<float *>(y_tile + 4 * kPanel);       // [2][2][128]
    uint64_t *c_full = reinterpret_cast<uint64_t *>(cum + 4 * kBlk);  // [4] C panel p of the block landed
    uint64_t *c_free = c_full + 4;     // [4] the block's MMAs on C panel p done
    uint64_t *ld_bar = c_full + 8;     // [2] y tiles of block i landed (buffer i % 2)
    uint64_t *mma_bar = c_full + 10;   // [2] the MMAs of block i done (accumulator i % 2)
    uint64_t *acc_free = c_full + 12;  // [2] accumulator i % 2 read out by the epilogue
    uint64_t *y_done = c_full + 14;    // [2] y tiles of buffer i % 2 updated by the epilogue
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c_full + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int local_status = 0;
    int *status = prm.status ? prm.status : &local_status;

    const int b = blockIdx.z;
    const int g = blockIdx.y / prm.pairs_per_group, pr = blockIdx.y % prm.pairs_per_group;
    const int hpg = prm.H / prm.G, h0 = g * hpg + 2 * pr;
    const int blk0 = blockIdx.x * prm.blocks_per_cta, nb = min(prm.blocks_per_cta, prm.nblk - blk0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long L = prm.L;

    if (tid == 0) {
        for (int p = 0; p < 4; ++p) {
            mbar_init(&c_full[p], 1);
            mbar_init(&c_free[p], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ld_bar[i], 1);
            mbar_init(&mma_bar[i], 1);
            mbar_init(&acc_free[i], kEpi);
            mbar_init(&y_done[i], kEpi);
        }
        *abort_flag = 0;
        abort_flag[1] = prm.wait_us;  // bounded-wait limit (us; 0: the built-in one)
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 8) {
        // S_in of the two heads -> bf16, K-major: row r = 64 e + p, 16-byte chunk (n / 8) in panel
        // n / 64. chunks = 128 N / 8 is a multiple of 4 * kEpi: four chunks' loads are issued per
        // thread before any of them is converted.
        const float *src = prm.s_in + ((long long)b * prm.H + h0) * kP * N;  // the two heads are adjacent
        const int chunks = kBlk * (N / 8);
        for (int i0 = tid; i0 < chunks; i0 += 4 * kEpi) {
            float4 lo[4], hi[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kEpi, r = i / (N / 8), cc = i % (N / 8);
                lo[u] = reinterpret_cast<const float4 *>(src + (long long)r * N)[2 * cc];
                hi[u] = reinterpret_cast<const float4 *>(src + (long long)r * N)[2 * cc + 1];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kEpi, r = i / (N / 8), cc = i % (N / 8);
                uint4 o;
                o.x = pack_bf16(lo[u].x, lo[u].y);
                o.y = pack_bf16(lo[u].z, lo[u].w);
                o.z = pack_bf16(hi[u].x, hi[u].y);
                o.w = pack_bf16(hi[u].z, hi[u].w);
                *reinterpret_cast<uint4 *>(s_tile + (cc >> 3) * kPanel + swz(r, cc & 7)) = o;
            }
        }
        fence_proxy_async();  // the generic-proxy writes of S_in are visible to the tensor cores
    }
    __syncthreads();

    if (warp == 8) {
        // ------------------------------------------------------------- producer (one thread)
        if (lane == 0) {
            int last_mma = -1, last_c = -1, last_y[2] = {-1, -1};
            bool ok = true;
            auto load_c = [&](int i, int pn) {  // C panel pn of block i
                mbar_arrive_tx(&c_full[pn], kPanel);
                tma_load_4d(c_tile + pn * kPanel, &tm_c, &c_full[pn], 64 * pn, g, (blk0 + i) * kBlk, b);
            };
            auto load_y = [&](int i) {  // the two heads' y tiles of block i, into buffer i % 2
                mbar_arrive_tx(&ld_bar[i & 1], 2 * kPanel);
                for (int e = 0; e < 2; ++e)
                    tma_load_4d(y_tile + ((i & 1) * 2 + e) * kPanel, &tm_y, &ld_bar[i & 1], 0, h0 + e, (blk0 + i) * kBlk, b);
                last_y[i & 1] = i;
            };
            auto store = [&](int i) {  // y tiles of block i, once the epilogue has updated them
                ok = wait_phase(&y_done[i & 1], (uint32_t)(i >> 1) & 1u, abort_flag, status);
                if (!ok) return;
                const int t0 = (blk0 + i) * kBlk;
                for (int hh = 0; hh < 2; ++hh)
                    tma_store_4d(&tm_y, y_tile + ((i & 1) * 2 + hh) * kPanel, 0, h0 + hh, t0, b, policy_evict_first());
                bulk_commit();
            };
            if (nb > 0) {
                for (int pn = 0; pn < npan; ++pn) load_c(0, pn);
                last_c = 0;
                load_y(0);
                if (nb > 1) load_y(1);
            }
            for (int i = 0; i < nb && ok; ++i) {
                // block i's MMAs, panel by panel, into accumulator i % 2 (read out by block i-2's
                // epilogue) while the epilogue works on block i-1
                if (i >= 2 && !(ok = wait_phase(&acc_free[i & 1], (uint32_t)((i - 2) >> 1) & 1u, abort_flag, status)))
                    break;
                constexpr uint32_t kId = idesc(128, 128, false, false);
                const uint32_t ca = smem_u32(c_tile), sa = smem_u32(s_tile);
                for (int pn = 0; pn < npan && ok; ++pn) {
                    if (!(ok = wait_phase(&c_full[pn], (uint32_t)i & 1u, abort_flag, status))) break;
                    tc_fence_after();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint32_t off = (uint32_t)(pn * kPanel + k4 * 32);
                        mma_ss(tmem + 128 * (i & 1), sdesc(ca + off, 16, 1024), sdesc(sa + off, 16, 1024), kId,
                               pn > 0 || k4 > 0);
                    }
                    mma_commit(&c_free[pn]);
                }
                if (!ok) break;
                mma_commit(&mma_bar[i & 1]);
                last_mma = i;
                // block i+1's C, each panel as soon as this block's MMAs on it are done
                if (i + 1 < nb) {
                    for (int pn = 0; pn < npan && ok; ++pn) {
                        if (!(ok = wait_phase(&c_free[pn], (uint32_t)i & 1u, abort_flag, status))) break;
                        load_c(i + 1, pn);
                    }
                    if (!ok) break;
                    last_c = i + 1;
                }
                // block i-1's y tiles out, then block i+1's in once that store has read its buffer
                if (i >= 1) {
                    store(i - 1);
                    if (!ok) break;
                    if (i + 1 < nb) {
                        bulk_wait_read();
                        load_y(i + 1);
                    }
                }
            }
            if (ok && nb > 0) store(nb - 1);
            bulk_wait_all();
            if (!ok) {  // MMAs and loads still in flight end before TMEM and the CTA go
                const unsigned long long w0 = now_ns();
                while (last_mma >= 0 && !mbar_try(&mma_bar[last_mma & 1], (uint32_t)(last_mma >> 1) & 1u) &&
                       now_ns() - w0 < kWaitNs) {
                }
                for (int pn = 0; pn < npan && last_c >= 0; ++pn)
                    while (!mbar_try(&c_full[pn], (uint32_t)last_c & 1u) && now_ns() - w0 < 2 * kWaitNs) {
                    }
                for (int k = 0; k < 2; ++k)
                    while (last_y[k] >= 0 && !mbar_try(&ld_bar[k], (uint32_t)(last_y[k] >> 1) & 1u) &&
                           now_ns() - w0 < 2 * kWaitNs) {
                    }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------- epilogue (warps 0-7)
        const int q = warp & 3, e = warp >> 2, row = 32 * q + lane;  // TMEM lane quarter, head
        for (int i = 0; i < nb; ++i) {
            const int blk = blk0 + i;
            const long long t0 = (long long)blk * kBlk;
            float *ck = cum + (i & 1) * 2 * kBlk;  // (two buffers: warps 0-1 may run one block ahead)
            if (warp < 2) {  // decay factors exp(cumulative dt A) of head h0 + warp over the block's tokens
                const int h = h0 + warp;
                const float a = prm.A[h];
                const float *bs = prm.bsum + ((long long)b * prm.H + h) * prm.nblk;
                float pre = 0.f;
                for (int k = lane; k < blk; k += 32) pre += bs[k];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, o);
                const long long tt = t0 + 4 * lane;
                float v[4];
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    v[m] = tt + m < L ? __bfloat162float(prm.dt[((long long)b * L + tt + m) * prm.H + h]) * a : 0.f;
                v[1] += v[0];
                v[2] += v[1];
                v[3] += v[2];
                float incl = v[3];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += u;
                }
                const float excl = incl - v[3] + pre;
#pragma unroll
                for (int m = 0; m < 4; ++m) ck[warp * kBlk + 4 * lane + m] = expf(excl + v[m]);
            }
            // (a wait that runs out raises the abort flag before the barrier, so after it every
            // epilogue warp takes the same branch)
            // (the y tiles' landing is awaited too: that is what makes their bytes visible here)
            if (wait_phase(&ld_bar[i & 1], (uint32_t)(i >> 1) & 1u, abort_flag, status))
                wait_phase(&mma_bar[i & 1], (uint32_t)(i >> 1) & 1u, abort_flag, status);
            asm volatile("bar.sync 1, %0;" ::"n"(kEpi) : "memory");  // cum of this block written
            if (*abort_flag) break;
            tc_fence_after();
            const float w = ck[e * kBlk + row];
            const uint32_t taddr = tmem + 128 * (i & 1) + ((uint32_t)(32 * q) << 16) + 64 * e;
            unsigned char *yr = y_tile + ((i & 1) * 2 + e) * kPanel;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t acc[32];
                tmem_ld32(taddr + 32 * half, acc);
                tmem_wait_ld(acc);
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(&acc_free[i & 1]);
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {  // 16-byte chunks 4 half + c4 of the row (8 columns each)
                    uint4 *pv = reinterpret_cast<uint4 *>(yr + swz(row, 4 * half + c4));
                    const uint4 old = *pv;
                    const uint32_t ov[4] = {old.x, old.y, old.z, old.w};
                    uint32_t nv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float a0 = __uint_as_float(acc[8 * c4 + 2 * u]), a1 = __uint_as_float(acc[8 * c4 + 2 * u + 1]);
                        nv[u] = pack_bf16(fmaf(w, a0, bf16_lo(ov[u])), fmaf(w, a1, bf16_hi(ov[u])));
                    }
                    *pv = make_uint4(nv[0], nv[1], nv[2], nv[3]);
                }
            }
            fence_proxy_async();
            mbar_arrive(&y_done[i & 1]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256) : "memory");
    }
}

}  // namespace cpt

bool cp_correct_uses_tc(const CpProblem &p) {
    return p.dtype == SSD_BF16 && p.P == cpt::kP && p.N % 64 == 0 && p.N <= 256 && (p.H / p.G) % 2 == 0 &&
           p.L < (1ll << 31);
}

cudaError_t cp_correct_tc_launch(const CpProblem &p, const void *dt, const float *A, const void *Cm, const float *bsum,
                                 const float *s_in, void *y, int *status, cudaStream_t s) {
    using namespace cpt;
    const int nblk = cp_nblk(p.L);
    if (nblk == 0) return cudaSuccess;
    CUtensorMap tmc, tmy;
    if (!tc::encode_4d(&tmc, Cm, p.N, p.G, p.L, p.B) || !tc::encode_4d(&tmy, y, kP, p.H, p.L, p.B))
        return cudaErrorInvalidValue;
    Params prm;
    prm.dt = static_cast<const __nv_bfloat16 *>(dt);
    prm.A = A;
    prm.bsum = bsum;
    prm.s_in = s_in;
    prm.status = status;
    prm.wait_us = wait_limit_us();
    prm.L = p.L;
    prm.H = (int)p.H;
    prm.G = (int)p.G;
    prm.N = (int)p.N;
    prm.nblk = nblk;
    prm.pairs_per_group = (int)(p.H / p.G / 2);
    // at most one CTA per SM (one wave): each takes a run of consecutive blocks of one (batch
    // row, head pair); with more pairs than SMs, a whole stream each
    const long long pairs = p.G * prm.pairs_per_group * p.B;
    const int sms = tc::num_sms() > 0 ? tc::num_sms() : 148;
    const long long per_pair = std::max(1ll, (long long)sms / pairs);  // CTAs per pair
    prm.blocks_per_cta = (int)std::max(1ll, ((long long)nblk + per_pair - 1) / per_pair);
    const int smem = smem_bytes((int)p.N) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_correct_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((nblk + prm.blocks_per_cta - 1) / prm.blocks_per_cta), (unsigned)(p.G * prm.pairs_per_group),
              (unsigned)p.B);
    k_correct_tc<<<grid, kThreads, smem, s>>>(tmc, tmy, prm);
    return cudaGetLastError();
}

}  // namespace ssd
