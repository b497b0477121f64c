// Context (sequence) parallelism for the SSD forward: the exchange step and the
// state-to-output correction that follow a per-segment forward.
//
// The Mamba-2 SSD write-up ("序列并行", with the state passing of "SSD 算法：分块和
// 状态传递") splits a long sequence across GPUs: each GPU runs the chunked forward
// on its own segment from a zero state, keeping its outputs and its final state;
// the final states are then passed between GPUs, and each GPU adds what its true
// incoming state contributes. With segment r's total log-decay
// Lambda_r = sum_{t in r} dt_t A_h and local end state S_r, the state entering
// segment r is the exclusive scan
//     S_in(0) = 0 (rank 0 ran from h0 itself),  S_in(r+1) = exp(Lambda_r) S_in(r) + S_r,
// its true end state is exp(Lambda_r) S_in(r) + S_r, and its outputs gain
//     y_t += exp(sum_{s <= t, s in r} dt_s A_h) C_t S_in(r)^T,
// which is step 4 of the chunked algorithm (state to output) applied to the
// incoming state. Kernels here:
//   k_block_decay   per 128-token block sums of dt A (coalesced over heads)
//   k_total_decay   Lambda = the block sums added in order
//   k_combine       the exclusive scan over ranks (elementwise over the state)
//   k_correct_tc    (ssd_cp_tc.cu) the correction on tcgen05 for bf16, P = 64, N % 64 == 0,
//                   an even number of heads per group
//   k_correct_mma   the correction with bf16 mma.sync tiles (128 tokens x 64 columns of P)
//   k_correct_simt  the same in fp32 on CUDA cores (fp32 inputs, or shapes the tiles do not fit)
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kCpBlk = 128;  // tokens per decay block and per correction tile

// grid (nblk, B), 256 threads over heads. bsum[b, h, blk] = sum of dt A over the block.
template <typename T>
__global__ void __launch_bounds__(256)
    k_block_decay(const T *__restrict__ dt, const float *__restrict__ A, int64_t L, int H, int nblk,
                  float *__restrict__ bsum) {
    const int blk = blockIdx.x, b = blockIdx.y;
    const int64_t t0 = (int64_t)blk * kCpBlk;
    const int nt = (int)min((int64_t)kCpBlk, L - t0);
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        const float a = A[h];
        const T *src = dt + ((int64_t)b * L + t0) * H + h;
        float s = 0.f;
#pragma unroll 8
        for (int i = 0; i < nt; ++i) s += to_f32(src[(int64_t)i * H]) * a;
        bsum[((int64_t)b * H + h) * nblk + blk] = s;
    }
}

// One thread per (b, h): Lambda[b, h] = block sums in block order.
__global__ void k_total_decay(const float *__restrict__ bsum, int64_t BH, int nblk, float *__restrict__ total) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= BH) return;
    float s = 0.f;
    for (int k = 0; k < nblk; ++k) s += bsum[i * nblk + k];
    total[i] = s;
}

// One thread per 4 state elements. states [R, BH, PN], totals [R, BH].
__global__ void k_combine(const float *__restrict__ states, const float *__restrict__ totals, int rank,
                          int64_t BH, int64_t PN, float *__restrict__ s_in, float *__restrict__ h_final) {
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // float4 index within [BH, PN]
    const int64_t per = BH * PN / 4;
    if (v >= per) return;
    const int64_t bh = (4 * v) / PN;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < rank; ++q) {
        const float g = expf(totals[(int64_t)q * BH + bh]);
        const float4 u = reinterpret_cast<const float4 *>(states + (int64_t)q * BH * PN)[v];
        s.x = fmaf(g, s.x, u.x);
        s.y = fmaf(g, s.y, u.y);
        s.z = fmaf(g, s.z, u.z);
        s.w = fmaf(g, s.w, u.w);
    }
    reinterpret_cast<float4 *>(s_in)[v] = s;
    if (h_final) {
        const float g = expf(totals[(int64_t)rank * BH + bh]);
        const float4 u = reinterpret_cast<const float4 *>(states + (int64_t)rank * BH * PN)[v];
        reinterpret_cast<float4 *>(h_final)[v] =
            make_float4(fmaf(g, s.x, u.x), fmaf(g, s.y, u.y), fmaf(g, s.z, u.z), fmaf(g, s.w, u.w));
    }
}

// exp of the decay from the segment start through token t of this block, for the
// block's 128 tokens, into cum[] (shared memory). Warp 0: the sum of the earlier blocks,
// then a within-block inclusive scan (4 tokens per lane). Every thread must call it.
template <typename T>
__device__ __forceinline__ void block_decay_factors(const T *__restrict__ dt, float a, const float *__restrict__ bsum_row,
                                                    int blk, int64_t L, int H, int b, int h, float *cum) {
    const int tid = threadIdx.x;
    if (tid < 32) {
        const int lane = tid;
        float pre = 0.f;
        for (int k = lane; k < blk; k += 32) pre += bsum_row[k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, o);
        const int64_t t0 = (int64_t)blk * kCpBlk + 4 * lane;
        float v[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) v[m] = t0 + m < L ? to_f32(dt[((int64_t)b * L + t0 + m) * H + h]) * a : 0.f;
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
        for (int m = 0; m < 4; ++m) cum[4 * lane + m] = expf(excl + v[m]);
    }
    __syncthreads();
}

// grid (nblk, H, B), 256 threads (8 warps; warp w owns tokens 16 w .. 16 w + 15 of the
// block). Requires P % 64 == 0 and N % 16 == 0. Shared memory: C tile [128][N + 8] bf16,
// S_in chunk [64][N + 8] bf16 (rows padded by 16 bytes: conflict-free ldmatrix), cum[128].
__global__ void __launch_bounds__(256)
    k_correct_mma(const __nv_bfloat16 *__restrict__ dt, const float *__restrict__ A,
                  const __nv_bfloat16 *__restrict__ Cm, const float *__restrict__ bsum, const float *__restrict__ s_in,
                  int64_t L, int H, int P, int G, int N, int nblk, __nv_bfloat16 *__restrict__ y) {
    extern __shared__ __align__(16) unsigned char cp_smem[];
    const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ld = N + 8;  // padded row length, elements
    __nv_bfloat16 *ct = reinterpret_cast<__nv_bfloat16 *>(cp_smem);   // [128][ld]
    __nv_bfloat16 *st = ct + kCpBlk * ld;                               // [64][ld]
    float *cum = reinterpret_cast<float *>(st + 64 * ld);               // [128]
    const int64_t t0 = (int64_t)blk * kCpBlk;
    const int nt = (int)min((int64_t)kCpBlk, L - t0);
    // C rows of the block (zeros past the end of the segment), 16 bytes per asynchronous copy,
    // all in flight at once
    const int cv = N / 8;
    for (int i = tid; i < kCpBlk * cv; i += blockDim.x) {
        const int r = i / cv, c = i % cv;
        __nv_bfloat16 *dst = ct + r * ld + 8 * c;
        if (r < nt) {
            const __nv_bfloat16 *srcp = Cm + ((((int64_t)b * L + t0 + r) * G + g) * N) + 8 * c;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                         "l"(srcp)
                         : "memory");
        } else {
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    block_decay_factors(dt, A[h], bsum + ((int64_t)b * H + h) * nblk, blk, L, H, b, h, cum);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    const uint32_t ct_base = (uint32_t)__cvta_generic_to_shared(ct), st_base = (uint32_t)__cvta_generic_to_shared(st);
    // ldmatrix row addresses: A (16 x 16 of C, rows 16 warp ..), B (two 8 x 16 tiles of S_in)
    const int a_row = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1), a_col = 8 * (lane >> 4);
    const int b_row = (lane & 7) + 8 * (lane >> 4), b_col = 8 * ((lane >> 3) & 1);
    const float *srow = s_in + ((int64_t)b * H + h) * P * N;
    for (int pc = 0; pc < P; pc += 64) {
        __syncthreads();  // the previous chunk's S_in tile has been read
        // 64 rows x N fp32 of S_in to bf16: each thread's (at most 16) loads are issued
        // before any of them is converted
        {
            const int per = 64 * (N / 4);  // float4 vectors in the chunk, a multiple of 256 / 16
            float4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = tid + u * 256;
                if (i < per) v[u] = reinterpret_cast<const float4 *>(srow + (int64_t)pc * N)[i];
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = tid + u * 256;
                if (i < per) {
                    const int r = i / (N / 4), c = i % (N / 4);
                    __nv_bfloat162 lo = __floats2bfloat162_rn(v[u].x, v[u].y), hi = __floats2bfloat162_rn(v[u].z, v[u].w);
                    uint2 pk;
                    pk.x = *reinterpret_cast<uint32_t *>(&lo);
                    pk.y = *reinterpret_cast<uint32_t *>(&hi);
                    *reinterpret_cast<uint2 *>(st + r * ld + 4 * c) = pk;
                }
            }
        }
        __syncthreads();
        float acc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
        for (int k = 0; k < N; k += 16) {
            uint32_t a0, a1, a2, a3;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                         : "r"(ct_base + (uint32_t)((a_row * ld + k + a_col) * 2)));
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {  // n8 tiles 2 jj and 2 jj + 1
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(st_base + (uint32_t)(((16 * jj + b_row) * ld + k + b_col) * 2)));
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                    "{%8, %9}, {%0, %1, %2, %3};"
                    : "+f"(acc[2 * jj][0]), "+f"(acc[2 * jj][1]), "+f"(acc[2 * jj][2]), "+f"(acc[2 * jj][3])
                    : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                    "{%8, %9}, {%0, %1, %2, %3};"
                    : "+f"(acc[2 * jj + 1][0]), "+f"(acc[2 * jj + 1][1]), "+f"(acc[2 * jj + 1][2]),
                      "+f"(acc[2 * jj + 1][3])
                    : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b2), "r"(b3));
            }
        }
        // y[t, p] += cum[t] * acc: rows 16 warp + lane / 4 (+ 8), columns pc + 8 j + 2 (lane % 4) (+ 1)
        const int r0 = 16 * warp + (lane >> 2);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int r = r0 + 8 * half;
            if (r >= nt) continue;
            const float w = cum[r];
            __nv_bfloat16 *yrow = y + (((int64_t)b * L + t0 + r) * H + h) * P + pc + 2 * (lane & 3);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                __nv_bfloat162 *q = reinterpret_cast<__nv_bfloat162 *>(yrow + 8 * j);
                const float2 old = __bfloat1622float2(*q);
                *q = __floats2bfloat162_rn(fmaf(w, acc[j][2 * half], old.x), fmaf(w, acc[j][2 * half + 1], old.y));
            }
        }
    }
}

// grid (nblk, H, B), 128 threads (thread = token). fp32 arithmetic throughout; S_in is read
// in 16-row chunks of P through shared memory.
template <typename T>
__global__ void __launch_bounds__(128)
    k_correct_simt(const T *__restrict__ dt, const float *__restrict__ A, const T *__restrict__ Cm,
                   const float *__restrict__ bsum, const float *__restrict__ s_in, int64_t L, int H, int P, int G,
                   int N, int nblk, T *__restrict__ y) {
    extern __shared__ __align__(16) float cps[];
    float *sc = cps;             // [16][N]
    float *cum = sc + 16 * N;    // [128]
    const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int t = threadIdx.x;
    const int64_t t0 = (int64_t)blk * kCpBlk;
    block_decay_factors(dt, A[h], bsum + ((int64_t)b * H + h) * nblk, blk, L, H, b, h, cum);
    const bool live = t0 + t < L;
    const T *crow = Cm + (((int64_t)b * L + t0 + t) * G + g) * N;
    T *yrow = y + (((int64_t)b * L + t0 + t) * H + h) * P;
    const float w = cum[t];
    const float *srow = s_in + ((int64_t)b * H + h) * P * N;
    for (int pc = 0; pc < P; pc += 16) {
        const int np = min(16, P - pc);
        __syncthreads();
        for (int i = t; i < np * N; i += blockDim.x) sc[i] = srow[(int64_t)pc * N + i];
        __syncthreads();
        float acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = 0.f;
        if (live) {
            for (int n = 0; n < N; ++n) {
                const float c = to_f32(crow[n]);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (j < np) acc[j] = fmaf(c, sc[j * N + n], acc[j]);
            }
            for (int j = 0; j < np; ++j) store_as(yrow + pc + j, fmaf(w, acc[j], to_f32(yrow[pc + j])));
        }
    }
}

}  // namespace

int cp_nblk(int64_t L) { return (int)((L + kCpBlk - 1) / kCpBlk); }

cudaError_t cp_block_decay_launch(const CpProblem &p, const void *dt, const float *A, float *bsum, float *total,
                                  cudaStream_t s) {
    const int nblk = cp_nblk(p.L);
    if (nblk > 0) {
        dim3 grid((unsigned)nblk, (unsigned)p.B);
        if (p.dtype == SSD_F32)
            k_block_decay<float><<<grid, 256, 0, s>>>((const float *)dt, A, p.L, (int)p.H, nblk, bsum);
        else
            k_block_decay<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)dt, A, p.L, (int)p.H, nblk, bsum);
    }
    const int64_t BH = p.B * p.H;
    k_total_decay<<<(unsigned)((BH + 255) / 256), 256, 0, s>>>(bsum, BH, nblk, total);
    return cudaGetLastError();
}

cudaError_t cp_combine_launch(const CpProblem &p, int R, int rank, const float *states, const float *totals,
                              float *s_in, float *h_final, cudaStream_t s) {
    (void)R;
    const int64_t BH = p.B * p.H, PN = p.P * p.N;
    const int64_t nv = BH * PN / 4;
    k_combine<<<(unsigned)((nv + 255) / 256), 256, 0, s>>>(states, totals, rank, BH, PN, s_in, h_final);
    return cudaGetLastError();
}

bool cp_correct_uses_mma(const CpProblem &p) { return p.dtype == SSD_BF16 && p.P % 64 == 0 && p.N % 16 == 0; }

cudaError_t cp_correct_launch(const CpProblem &p, const void *dt, const float *A, const void *Cm, const float *bsum,
                              const float *s_in, void *y, int *status, cudaStream_t s) {
    const int nblk = cp_nblk(p.L);
    if (nblk == 0) return cudaSuccess;
    if (cp_correct_uses_tc(p)) return cp_correct_tc_launch(p, dt, A, Cm, bsum, s_in, y, status, s);
    dim3 grid((unsigned)nblk, (unsigned)p.H, (unsigned)p.B);
    const int H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N;
    cudaError_t e;
    if (cp_correct_uses_mma(p)) {
        const size_t smem = (size_t)(kCpBlk + 64) * (N + 8) * 2 + kCpBlk * sizeof(float);
        if ((e = cudaFuncSetAttribute(k_correct_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        k_correct_mma<<<grid, 256, smem, s>>>((const __nv_bfloat16 *)dt, A, (const __nv_bfloat16 *)Cm, bsum, s_in,
                                             p.L, H, P, G, N, nblk, (__nv_bfloat16 *)y);
    } else {
        const size_t smem = (size_t)(16 * N + kCpBlk) * sizeof(float);
        if (p.dtype == SSD_F32) {
            if ((e = cudaFuncSetAttribute(k_correct_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
                return e;
            k_correct_simt<float><<<grid, kCpBlk, smem, s>>>((const float *)dt, A, (const float *)Cm, bsum, s_in, p.L,
                                                             H, P, G, N, nblk, (float *)y);
        } else {
            using bf = __nv_bfloat16;
            if ((e = cudaFuncSetAttribute(k_correct_simt<bf>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
                return e;
            k_correct_simt<bf><<<grid, kCpBlk, smem, s>>>((const bf *)dt, A, (const bf *)Cm, bsum, s_in, p.L, H, P, G,
                                                          N, nblk, (bf *)y);
        }
    }
    return cudaGetLastError();
}

}  // namespace ssd
