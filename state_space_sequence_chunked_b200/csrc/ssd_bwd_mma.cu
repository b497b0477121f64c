// Tensor-core (mma.sync, bf16 operands, fp32 accumulation) kernels of the backward pass for
// bf16 inputs. They compute the same quantities as the fp32 CUDA-core kernels of ssd_bwd.cu
// (the formulas are listed there), with every product of the chunked backward as an
// m16n8k16 matrix multiply over 64-token tiles:
//   chunk sums      S_c = sum_l (w_l u_l) v_l^T           [P x N], K = tokens of the chunk
//   sources (s)     W1^T = B_s C_l^T, W2^T = x_s dy_l^T  (masked l >= s, decayed, to bf16)
//                   u = B_s Gend^T e + W1^T dy_l,  v = x_s Gend e + W2^T C_l
//   targets (l)     W3 = dy_l x_s^T (masked s <= l, decayed, times dt_s, to bf16)
//                   w = e dy_l S_in + W3 B_s
// The log-decay gradient is not formed from the two roles' sums (its reverse cumsum would rely
// on their bf16-rounded pair terms cancelling); instead the source kernel also forms, in fp32,
// the pair products M[l,s] = (C_l.B_s)(dy_l.x_s) dt_s exp(A_cs[l]-A_cs[s]) (l > s) with their
// row sums K_s and column sums R_l, and the state terms U_s; the target kernel the terms T_l.
// Operands sit in shared memory as bf16 rows padded by 16 bytes (conflict-free ldmatrix);
// an operand whose reduction index is not the contiguous one is read with ldmatrix.trans.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kT = 64;        // tokens per tile
constexpr int kThr = 256;     // 8 warps (chunk sums)
constexpr int kThr2 = 512;    // 16 warps (source and target kernels)

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ uint32_t su32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Fragment addresses (bytes, shared space) for a tile stored row-major with `ld` elements per row.
// A operand, 16 x 16 at (m0, k0), stored [M][K]:
__device__ __forceinline__ uint32_t a_mk(uint32_t base, int ld, int m0, int k0, int lane) {
    return base + (uint32_t)(((m0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + k0 + 8 * (lane >> 4)) * 2);
}
// A operand, 16 x 16 at (m0, k0), stored [K][M] (read transposed):
__device__ __forceinline__ uint32_t a_km(uint32_t base, int ld, int m0, int k0, int lane) {
    return base + (uint32_t)(((k0 + (lane & 7) + 8 * (lane >> 4)) * ld + m0 + 8 * ((lane >> 3) & 1)) * 2);
}
// B operand, two n8 tiles (n0, n0 + 8) x k16 at k0, stored [N][K]: regs {0,1} tile n0, {2,3} tile n0 + 8
__device__ __forceinline__ uint32_t b_nk(uint32_t base, int ld, int n0, int k0, int lane) {
    return base + (uint32_t)(((n0 + (lane & 7) + 8 * (lane >> 4)) * ld + k0 + 8 * ((lane >> 3) & 1)) * 2);
}
// B operand, the same two tiles, stored [K][N] (read transposed)
__device__ __forceinline__ uint32_t b_kn(uint32_t base, int ld, int n0, int k0, int lane) {
    return base + (uint32_t)(((k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + n0 + 8 * (lane >> 4)) * 2);
}

// rows [r0, r0 + 64) of a [rows][W] bf16 matrix (row stride `gstride` elements in global) into
// shared [64][W + 8]; rows >= nrows are zero. W % 8 == 0, 16-byte aligned rows.
template <int W>
__device__ __forceinline__ void load_rows(bf16 *dst, const bf16 *src, int64_t gstride, int nrows, int tid,
                                          int nthr) {
    constexpr int V = W / 8;
    for (int i = tid; i < kT * V; i += nthr) {
        const int r = i / V, c = i % V;
        bf16 *d = dst + r * (W + 8) + 8 * c;
        if (r < nrows) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(su32(d)), "l"(src + r * gstride + 8 * c)
                         : "memory");
        } else {
            *reinterpret_cast<uint4 *>(d) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}
__device__ __forceinline__ void async_wait() {
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// fp32 [P][N] (global) to bf16 [P][N + 8] (shared)
template <int P, int N>
__device__ __forceinline__ void load_state_bf16(bf16 *dst, const float *src, int tid, int nthr) {
    constexpr int V = N / 4;
    for (int i = tid; i < P * V; i += nthr) {
        const int r = i / V, c = i % V;
        const float4 v = reinterpret_cast<const float4 *>(src)[i];
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t *>(&lo);
        pk.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(dst + r * (N + 8) + 4 * c) = pk;
    }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---- chunk sums ---------------------------------------------------------------------
// grid (nc, H, B). Output rows are P / 16 row blocks; 8 / (P / 16) warps share a row block
// and split the N columns.
template <int P, int N, bool kAdj>
__global__ void __launch_bounds__(kThr)
    k_chunk_sums_mma(const bf16 *__restrict__ u, const bf16 *__restrict__ v, const float *__restrict__ acs,
                     const float *__restrict__ dtw, int64_t L, int H, int G, int Q, int nc, float *__restrict__ out) {
    constexpr int RB = P / 16, WPR = 8 / RB, NCW = N / WPR, NTW = NCW / 8;
    static_assert(RB * WPR == 8 && NTW % 2 == 0, "tile split");
    extern __shared__ __align__(16) unsigned char smem[];
    bf16 *us = reinterpret_cast<bf16 *>(smem);   // [64][P + 8]  weighted u rows
    bf16 *vs = us + kT * (P + 8);                 // [64][N + 8]
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    const int64_t bh = (int64_t)b * H + h, lb = (bh * nc + c) * Q;
    const float last = acs[lb + Q - 1];
    const int rb = warp / WPR, n0w = (warp % WPR) * NCW;
    float acc[NTW][4];
#pragma unroll
    for (int j = 0; j < NTW; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
    const uint32_t ub = su32(us), vb = su32(vs);
    for (int l0 = 0; l0 < q; l0 += kT) {
        const int nl = min(kT, q - l0);
        __syncthreads();
        load_rows<N>(vs, v + (((int64_t)b * L + t0 + l0) * G + g) * N, (int64_t)G * N, nl, tid, kThr);
        // u rows scaled by their weight, rounded to bf16
        constexpr int V = P / 8;
        for (int i = tid; i < kT * V; i += kThr) {
            const int r = i / V, cc = i % V;
            uint4 pk = make_uint4(0u, 0u, 0u, 0u);
            if (r < nl) {
                const int l = l0 + r;
                const float w = kAdj ? __expf(acs[lb + l]) : __expf(last - acs[lb + l]) * dtw[lb + l];
                const uint4 raw = *reinterpret_cast<const uint4 *>(u + (((int64_t)b * L + t0 + l) * H + h) * P + 8 * cc);
                const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&raw);
                float2 f0 = __bfloat1622float2(hv[0]), f1 = __bfloat1622float2(hv[1]);
                float2 f2 = __bfloat1622float2(hv[2]), f3 = __bfloat1622float2(hv[3]);
                pk.x = pack2(w * f0.x, w * f0.y);
                pk.y = pack2(w * f1.x, w * f1.y);
                pk.z = pack2(w * f2.x, w * f2.y);
                pk.w = pack2(w * f3.x, w * f3.y);
            }
            *reinterpret_cast<uint4 *>(us + r * (P + 8) + 8 * cc) = pk;
        }
        async_wait();
        __syncthreads();
#pragma unroll
        for (int k0 = 0; k0 < kT; k0 += 16) {
            uint32_t a[4];
            ldsm4t(a_km(ub, P + 8, 16 * rb, k0, lane), a);
#pragma unroll
            for (int jj = 0; jj < NTW / 2; ++jj) {
                uint32_t bb[4];
                ldsm4t(b_kn(vb, N + 8, n0w + 16 * jj, k0, lane), bb);
                mma(acc[2 * jj], a, bb[0], bb[1]);
                mma(acc[2 * jj + 1], a, bb[2], bb[3]);
            }
        }
    }
    float *o = out + (bh * nc + c) * (int64_t)P * N;
    const int r = 16 * rb + (lane >> 2);
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
        const int n = n0w + 8 * j + 2 * (lane & 3);
        *reinterpret_cast<float2 *>(o + (int64_t)r * N + n) = make_float2(acc[j][0], acc[j][1]);
        *reinterpret_cast<float2 *>(o + (int64_t)(r + 8) * N + n) = make_float2(acc[j][2], acc[j][3]);
    }
}

// ---- tokens as sources --------------------------------------------------------------
// grid (nc * nrt, H, B); a tile of 64 tokens s per CTA, 16 warps. Warp w: rows 16 (w & 3) ..,
// column quarter w >> 2 of u and v, and columns 16 (w >> 2) .. of each 64 x 64 W tile. The next
// target tile's C and dy rows load (cp.async, double buffer) while this one is multiplied.
template <int P, int N>
__global__ void __launch_bounds__(kThr2, 1)
    k_bwd_src_mma(const bf16 *__restrict__ x, const bf16 *__restrict__ Bm, const bf16 *__restrict__ Cm,
                  const bf16 *__restrict__ dy, const float *__restrict__ acs, const float *__restrict__ dtw,
                  const float *__restrict__ gend, const float *__restrict__ D, int64_t L, int H, int G, int Q, int nc,
                  int nrt, bf16 *__restrict__ dx, float *__restrict__ dB_acc, float *__restrict__ kq,
                  float *__restrict__ rq, float *__restrict__ uq, float *__restrict__ ddt_dir,
                  float *__restrict__ dDpart) {
    constexpr int LN = N + 8, LP = P + 8, LW = kT + 8;
    constexpr int TU = P / 32, TV = N / 32;  // n8 tiles per warp (a quarter of the columns)
    static_assert(TU % 2 == 0 && TV % 2 == 0, "column quarters are whole n16 pairs");
    extern __shared__ __align__(16) unsigned char smem[];
    bf16 *bs = reinterpret_cast<bf16 *>(smem);  // [64][LN]     B_s
    bf16 *xs = bs + kT * LN;                     // [64][LP]     x_s
    bf16 *cl = xs + kT * LP;                     // [2][64][LN]  C_l (double buffer)
    bf16 *dl = cl + 2 * kT * LN;                 // [2][64][LP]  dy_l
    bf16 *w1 = dl + 2 * kT * LP;                 // [64][LW]     W1^T [s][l]
    bf16 *w2 = w1 + kT * LW;                     // [64][LW]     W2^T [s][l]
    bf16 *ge = w2 + kT * LW;                     // [P][LN]      Gend
    float *as = reinterpret_cast<float *>(ge + P * LN);  // [64]
    float *al = as + kT;                                 // [2][64]
    float *ds = al + 2 * kT;                             // [64] dt_s
    float *red = ds + kT;                                // [3][4][64] + [16]

    const int c = blockIdx.x / nrt, rt = blockIdx.x % nrt, r0 = rt * kT;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    const int64_t bh = (int64_t)b * H + h, lb = (bh * nc + c) * Q;
    if (r0 >= q) {
        if (tid == 0) dDpart[(bh * nc + c) * nrt + rt] = 0.f;
        return;
    }
    const int nr = min(kT, q - r0);
    load_rows<N>(bs, Bm + (((int64_t)b * L + t0 + r0) * G + g) * N, (int64_t)G * N, nr, tid, kThr2);
    load_rows<P>(xs, x + (((int64_t)b * L + t0 + r0) * H + h) * P, (int64_t)H * P, nr, tid, kThr2);
    load_rows<N>(cl, Cm + (((int64_t)b * L + t0 + r0) * G + g) * N, (int64_t)G * N, nr, tid, kThr2);
    load_rows<P>(dl, dy + (((int64_t)b * L + t0 + r0) * H + h) * P, (int64_t)H * P, nr, tid, kThr2);
    asm volatile("cp.async.commit_group;" ::: "memory");
    load_state_bf16<P, N>(ge, gend + (bh * nc + c) * (int64_t)P * N, tid, kThr2);
    for (int i = tid; i < kT; i += kThr2) {
        as[i] = acs[lb + min(r0 + i, Q - 1)];
        al[i] = as[i];
        ds[i] = i < nr ? dtw[lb + r0 + i] : 0.f;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    const int rb = warp & 3, cq = warp >> 2;
    const int pu0 = cq * (P / 4), nv0 = cq * (N / 4);
    const uint32_t bsb = su32(bs), xsb = su32(xs), w1b = su32(w1), w2b = su32(w2), geb = su32(ge);
    float au[TU][4], av[TV][4];
#pragma unroll
    for (int j = 0; j < TU; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) au[j][e] = 0.f;
#pragma unroll
    for (int j = 0; j < TV; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) av[j][e] = 0.f;

    // state part: u = B_s Gend^T (K = N), v = x_s Gend (K = P)
#pragma unroll 2
    for (int k0 = 0; k0 < N; k0 += 16) {
        uint32_t a[4];
        ldsm4(a_mk(bsb, LN, 16 * rb, k0, lane), a);
#pragma unroll
        for (int jj = 0; jj < TU / 2; ++jj) {
            uint32_t bb[4];
            ldsm4(b_nk(geb, LN, pu0 + 16 * jj, k0, lane), bb);
            mma(au[2 * jj], a, bb[0], bb[1]);
            mma(au[2 * jj + 1], a, bb[2], bb[3]);
        }
    }
#pragma unroll 2
    for (int k0 = 0; k0 < P; k0 += 16) {
        uint32_t a[4];
        ldsm4(a_mk(xsb, LP, 16 * rb, k0, lane), a);
#pragma unroll
        for (int jj = 0; jj < TV / 2; ++jj) {
            uint32_t bb[4];
            ldsm4t(b_kn(geb, LN, nv0 + 16 * jj, k0, lane), bb);
            mma(av[2 * jj], a, bb[0], bb[1]);
            mma(av[2 * jj + 1], a, bb[2], bb[3]);
        }
    }
    const int rlo = 16 * rb + (lane >> 2), rhi = rlo + 8;
    {
        const float aend = acs[lb + Q - 1];
        const float flo = __expf(aend - as[rlo]), fhi = __expf(aend - as[rhi]);
#pragma unroll
        for (int j = 0; j < TU; ++j) {
            au[j][0] *= flo; au[j][1] *= flo; au[j][2] *= fhi; au[j][3] *= fhi;
        }
#pragma unroll
        for (int j = 0; j < TV; ++j) {
            av[j][0] *= flo; av[j][1] *= flo; av[j][2] *= fhi; av[j][3] *= fhi;
        }
    }
    // U_s = dt_s x_s . (the state part of u_s), partial over this warp's columns
    float upart[2] = {0.f, 0.f};
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int srow = rlo + 8 * hf;
#pragma unroll
        for (int j = 0; j < TU; ++j) {
            const int p = pu0 + 8 * j + 2 * (lane & 3);
            const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(xs + srow * LP + p));
            upart[hf] = fmaf(xv.x, au[j][2 * hf], fmaf(xv.y, au[j][2 * hf + 1], upart[hf]));
        }
        upart[hf] *= ds[srow];
    }
    float kpart[2] = {0.f, 0.f};  // K_s over the target tiles, rows rlo, rhi

    // within the chunk: target tiles l >= s
    const int wc = cq * 16;  // this warp's 16 columns l of a W tile (rows 16 rb ..)
    int it = 0;
    for (int l0 = r0; l0 < q; l0 += kT, ++it) {
        const int cur = it & 1, nl = min(kT, q - l0);
        bf16 *clc = cl + cur * kT * LN, *dlc = dl + cur * kT * LP;
        const float *alc = al + cur * kT;
        const int l1 = l0 + kT;
        if (l1 < q) {  // prefetch the next target tile into the other buffer
            const int n1 = min(kT, q - l1);
            load_rows<N>(cl + (cur ^ 1) * kT * LN, Cm + (((int64_t)b * L + t0 + l1) * G + g) * N, (int64_t)G * N, n1,
                         tid, kThr2);
            load_rows<P>(dl + (cur ^ 1) * kT * LP, dy + (((int64_t)b * L + t0 + l1) * H + h) * P, (int64_t)H * P, n1,
                         tid, kThr2);
            asm volatile("cp.async.commit_group;" ::: "memory");
            for (int i = tid; i < kT; i += kThr2) al[(cur ^ 1) * kT + i] = acs[lb + min(l1 + i, Q - 1)];
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const uint32_t clb = su32(clc), dlb = su32(dlc);
        float f1[2][4], f2[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) f1[j][e] = f2[j][e] = 0.f;
#pragma unroll 4
        for (int k0 = 0; k0 < N; k0 += 16) {
            uint32_t a[4], bb[4];
            ldsm4(a_mk(bsb, LN, 16 * rb, k0, lane), a);
            ldsm4(b_nk(clb, LN, wc, k0, lane), bb);
            mma(f1[0], a, bb[0], bb[1]);
            mma(f1[1], a, bb[2], bb[3]);
        }
#pragma unroll 4
        for (int k0 = 0; k0 < P; k0 += 16) {
            uint32_t a[4], bb[4];
            ldsm4(a_mk(xsb, LP, 16 * rb, k0, lane), a);
            ldsm4(b_nk(dlb, LP, wc, k0, lane), bb);
            mma(f2[0], a, bb[0], bb[1]);
            mma(f2[1], a, bb[2], bb[3]);
        }
        // mask l >= s (and the tile ends), decay exp(A_cs[l] - A_cs[s]), to bf16; and the fp32
        // pair products M (strictly l > s): row sums into K_s, column sums into R_l
        {
            float rcol[2][2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int lc = wc + 8 * j + 2 * (lane & 3);
                rcol[j][0] = rcol[j][1] = 0.f;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int s = rlo + 8 * hf;
                    float d0 = 0.f, d1 = 0.f;
                    if (s < nr) {
                        if (lc < nl && l0 + lc >= r0 + s) d0 = __expf(alc[lc] - as[s]);
                        if (lc + 1 < nl && l0 + lc + 1 >= r0 + s) d1 = __expf(alc[lc + 1] - as[s]);
                    }
                    *reinterpret_cast<uint32_t *>(w1 + s * LW + lc) = pack2(f1[j][2 * hf] * d0, f1[j][2 * hf + 1] * d1);
                    *reinterpret_cast<uint32_t *>(w2 + s * LW + lc) = pack2(f2[j][2 * hf] * d0, f2[j][2 * hf + 1] * d1);
                    const float m0 = l0 + lc != r0 + s ? f1[j][2 * hf] * f2[j][2 * hf] * d0 * ds[s] : 0.f;
                    const float m1 = l0 + lc + 1 != r0 + s ? f1[j][2 * hf + 1] * f2[j][2 * hf + 1] * d1 * ds[s] : 0.f;
                    kpart[hf] += m0 + m1;
                    rcol[j][0] += m0;
                    rcol[j][1] += m1;
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    float v = rcol[j][e2];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    const int lc = wc + 8 * j + 2 * (lane & 3) + e2;
                    if (lane < 4 && lc < nl && v != 0.f) atomicAdd(rq + lb + l0 + lc, v);
                }
        }
        __syncthreads();
        // u += W1^T dy_l, v += W2^T C_l (K = l)
#pragma unroll
        for (int k0 = 0; k0 < kT; k0 += 16) {
            uint32_t a[4];
            ldsm4(a_mk(w1b, LW, 16 * rb, k0, lane), a);
#pragma unroll
            for (int jj = 0; jj < TU / 2; ++jj) {
                uint32_t bb[4];
                ldsm4t(b_kn(dlb, LP, pu0 + 16 * jj, k0, lane), bb);
                mma(au[2 * jj], a, bb[0], bb[1]);
                mma(au[2 * jj + 1], a, bb[2], bb[3]);
            }
            ldsm4(a_mk(w2b, LW, 16 * rb, k0, lane), a);
#pragma unroll
            for (int jj = 0; jj < TV / 2; ++jj) {
                uint32_t bb[4];
                ldsm4t(b_kn(clb, LN, nv0 + 16 * jj, k0, lane), bb);
                mma(av[2 * jj], a, bb[0], bb[1]);
                mma(av[2 * jj + 1], a, bb[2], bb[3]);
            }
        }
        __syncthreads();  // this tile's buffers and W are free for the next iteration
    }

    // epilogue
    const float Dh = D ? D[h] : 0.f;
    float xu[2] = {0.f, 0.f}, dd = 0.f;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int s = rlo + 8 * hf;
        if (s >= nr) continue;
        const int64_t t = t0 + r0 + s;
        const float dts = ds[s];
        const int64_t xoff = (((int64_t)b * L + t) * H + h) * P;
#pragma unroll
        for (int j = 0; j < TU; ++j) {
            const int p = pu0 + 8 * j + 2 * (lane & 3);
            const float2 dyv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(dy + xoff + p));
            const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(xs + s * LP + p));
            const float u0 = au[j][2 * hf], u1 = au[j][2 * hf + 1];
            *reinterpret_cast<__nv_bfloat162 *>(dx + xoff + p) =
                __floats2bfloat162_rn(fmaf(dts, u0, Dh * dyv.x), fmaf(dts, u1, Dh * dyv.y));
            xu[hf] = fmaf(xv.x, u0, fmaf(xv.y, u1, xu[hf]));
            dd = fmaf(dyv.x, xv.x, fmaf(dyv.y, xv.y, dd));
        }
        float *dbrow = dB_acc + (((int64_t)b * L + t) * G + g) * N;
#pragma unroll
        for (int j = 0; j < TV; ++j) {
            const int n = nv0 + 8 * j + 2 * (lane & 3);
            atomicAdd(reinterpret_cast<float2 *>(dbrow + n), make_float2(dts * av[j][2 * hf], dts * av[j][2 * hf + 1]));
        }
    }
    // row sums: the 4 lanes of a row, then the four column quarters through shared memory
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            xu[hf] += __shfl_xor_sync(0xffffffffu, xu[hf], o);
            kpart[hf] += __shfl_xor_sync(0xffffffffu, kpart[hf], o);
            upart[hf] += __shfl_xor_sync(0xffffffffu, upart[hf], o);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
    float *rxu = red, *rk = red + 4 * kT, *ru = red + 8 * kT, *rdd = red + 12 * kT;
    if ((lane & 3) == 0) {
        rxu[cq * kT + rlo] = xu[0];
        rxu[cq * kT + rhi] = xu[1];
        rk[cq * kT + rlo] = kpart[0];
        rk[cq * kT + rhi] = kpart[1];
        ru[cq * kT + rlo] = upart[0];
        ru[cq * kT + rhi] = upart[1];
    }
    if (lane == 0) rdd[warp] = dd;
    __syncthreads();
    if (tid < nr) {
        ddt_dir[lb + r0 + tid] = rxu[tid] + rxu[kT + tid] + rxu[2 * kT + tid] + rxu[3 * kT + tid];
        kq[lb + r0 + tid] = rk[tid] + rk[kT + tid] + rk[2 * kT + tid] + rk[3 * kT + tid];
        uq[lb + r0 + tid] = ru[tid] + ru[kT + tid] + ru[2 * kT + tid] + ru[3 * kT + tid];
    }
    if (tid == 0) {
        float sacc = 0.f;
        for (int w = 0; w < kThr2 / 32; ++w) sacc += rdd[w];
        dDpart[(bh * nc + c) * nrt + rt] = sacc;
    }
}

// ---- tokens as targets --------------------------------------------------------------
// grid (nc * nrt, H, B); a tile of 64 tokens l per CTA, 16 warps; source tiles s <= l double-buffered.
template <int P, int N>
__global__ void __launch_bounds__(kThr2, 1)
    k_bwd_dst_mma(const bf16 *__restrict__ x, const bf16 *__restrict__ Bm, const bf16 *__restrict__ Cm,
                  const bf16 *__restrict__ dy, const float *__restrict__ acs, const float *__restrict__ dtw,
                  const float *__restrict__ s_in, int64_t L, int H, int G, int Q, int nc, int nrt,
                  float *__restrict__ dC_acc, float *__restrict__ tq) {
    constexpr int LN = N + 8, LP = P + 8, LW = kT + 8;
    constexpr int TV = N / 32;
    static_assert(TV % 2 == 0, "column quarters are whole n16 pairs");
    extern __shared__ __align__(16) unsigned char smem[];
    bf16 *co = reinterpret_cast<bf16 *>(smem);  // [64][LN]     C_l
    bf16 *dl = co + kT * LN;                     // [64][LP]     dy_l
    bf16 *bs = dl + kT * LP;                     // [2][64][LN]  B_s (double buffer)
    bf16 *xs = bs + 2 * kT * LN;                 // [2][64][LP]  x_s
    bf16 *w3 = xs + 2 * kT * LP;                 // [64][LW]     W3 [l][s]
    bf16 *si = w3 + kT * LW;                     // [P][LN]      S_in
    float *al = reinterpret_cast<float *>(si + P * LN);  // [64]
    float *as = al + kT;                                 // [2][64]
    float *ds = as + 2 * kT;                             // [2][64]
    float *red = ds + 2 * kT;                            // [4][64]

    const int c = blockIdx.x / nrt, r0 = (blockIdx.x % nrt) * kT;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    if (r0 >= q) return;
    const int nr = min(kT, q - r0);
    const int send = r0 + nr;  // source tokens s < send
    const int64_t bh = (int64_t)b * H + h, lb = (bh * nc + c) * Q;
    load_rows<N>(co, Cm + (((int64_t)b * L + t0 + r0) * G + g) * N, (int64_t)G * N, nr, tid, kThr2);
    load_rows<P>(dl, dy + (((int64_t)b * L + t0 + r0) * H + h) * P, (int64_t)H * P, nr, tid, kThr2);
    {
        const int n0s = min(kT, q);
        load_rows<N>(bs, Bm + (((int64_t)b * L + t0) * G + g) * N, (int64_t)G * N, n0s, tid, kThr2);
        load_rows<P>(xs, x + (((int64_t)b * L + t0) * H + h) * P, (int64_t)H * P, n0s, tid, kThr2);
        asm volatile("cp.async.commit_group;" ::: "memory");
        for (int i = tid; i < kT; i += kThr2) {
            al[i] = acs[lb + min(r0 + i, Q - 1)];
            as[i] = acs[lb + min(i, Q - 1)];
            ds[i] = i < n0s ? dtw[lb + i] : 0.f;
        }
    }
    load_state_bf16<P, N>(si, s_in + (bh * nc + c) * (int64_t)P * N, tid, kThr2);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    const int rb = warp & 3, cq = warp >> 2, nv0 = cq * (N / 4);
    const uint32_t cob = su32(co), dlb = su32(dl), w3b = su32(w3), sib = su32(si);
    (void)cob;
    float aw[TV][4];
#pragma unroll
    for (int j = 0; j < TV; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) aw[j][e] = 0.f;
    // state part: w = dy_l S_in (K = P)
#pragma unroll 2
    for (int k0 = 0; k0 < P; k0 += 16) {
        uint32_t a[4];
        ldsm4(a_mk(dlb, LP, 16 * rb, k0, lane), a);
#pragma unroll
        for (int jj = 0; jj < TV / 2; ++jj) {
            uint32_t bb[4];
            ldsm4t(b_kn(sib, LN, nv0 + 16 * jj, k0, lane), bb);
            mma(aw[2 * jj], a, bb[0], bb[1]);
            mma(aw[2 * jj + 1], a, bb[2], bb[3]);
        }
    }
    const int rlo = 16 * rb + (lane >> 2), rhi = rlo + 8;
    {
        const float flo = __expf(al[rlo]), fhi = __expf(al[rhi]);
#pragma unroll
        for (int j = 0; j < TV; ++j) {
            aw[j][0] *= flo; aw[j][1] *= flo; aw[j][2] *= fhi; aw[j][3] *= fhi;
        }
    }
    // T_l = C_l . (the state part of w_l)
    {
        float cw[2] = {0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int l = rlo + 8 * hf;
#pragma unroll
            for (int j = 0; j < TV; ++j) {
                const int n = nv0 + 8 * j + 2 * (lane & 3);
                const float2 cv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(co + l * LN + n));
                cw[hf] = fmaf(cv.x, aw[j][2 * hf], fmaf(cv.y, aw[j][2 * hf + 1], cw[hf]));
            }
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) cw[hf] += __shfl_xor_sync(0xffffffffu, cw[hf], o);
        }
        if ((lane & 3) == 0) {
            red[cq * kT + rlo] = cw[0];
            red[cq * kT + rhi] = cw[1];
        }
        __syncthreads();
        if (tid < nr) tq[lb + r0 + tid] = red[tid] + red[kT + tid] + red[2 * kT + tid] + red[3 * kT + tid];
    }
    const int wc = cq * 16;  // this warp's 16 columns s of a W3 tile
    int it = 0;
    for (int s0 = 0; s0 < send; s0 += kT, ++it) {
        const int cur = it & 1, ns = min(kT, q - s0);
        bf16 *bsc = bs + cur * kT * LN, *xsc = xs + cur * kT * LP;
        const float *asc = as + cur * kT, *dsc = ds + cur * kT;
        const int s1 = s0 + kT;
        if (s1 < send) {  // prefetch the next source tile
            const int n1 = min(kT, q - s1);
            load_rows<N>(bs + (cur ^ 1) * kT * LN, Bm + (((int64_t)b * L + t0 + s1) * G + g) * N, (int64_t)G * N, n1,
                         tid, kThr2);
            load_rows<P>(xs + (cur ^ 1) * kT * LP, x + (((int64_t)b * L + t0 + s1) * H + h) * P, (int64_t)H * P, n1,
                         tid, kThr2);
            asm volatile("cp.async.commit_group;" ::: "memory");
            for (int i = tid; i < kT; i += kThr2) {
                as[(cur ^ 1) * kT + i] = acs[lb + min(s1 + i, Q - 1)];
                ds[(cur ^ 1) * kT + i] = i < n1 ? dtw[lb + s1 + i] : 0.f;
            }
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const uint32_t bsb = su32(bsc), xsb = su32(xsc);
        float f3[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) f3[j][e] = 0.f;
#pragma unroll 4
        for (int k0 = 0; k0 < P; k0 += 16) {
            uint32_t a[4], bb[4];
            ldsm4(a_mk(dlb, LP, 16 * rb, k0, lane), a);
            ldsm4(b_nk(xsb, LP, wc, k0, lane), bb);
            mma(f3[0], a, bb[0], bb[1]);
            mma(f3[1], a, bb[2], bb[3]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int sc = wc + 8 * j + 2 * (lane & 3);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int l = rlo + 8 * hf;
                float d0 = 0.f, d1 = 0.f;
                if (l < nr) {
                    if (sc < ns && s0 + sc <= r0 + l) d0 = __expf(al[l] - asc[sc]) * dsc[sc];
                    if (sc + 1 < ns && s0 + sc + 1 <= r0 + l) d1 = __expf(al[l] - asc[sc + 1]) * dsc[sc + 1];
                }
                *reinterpret_cast<uint32_t *>(w3 + l * LW + sc) = pack2(f3[j][2 * hf] * d0, f3[j][2 * hf + 1] * d1);
            }
        }
        __syncthreads();
        // w += W3 B_s (K = s)
#pragma unroll
        for (int k0 = 0; k0 < kT; k0 += 16) {
            uint32_t a[4];
            ldsm4(a_mk(w3b, LW, 16 * rb, k0, lane), a);
#pragma unroll
            for (int jj = 0; jj < TV / 2; ++jj) {
                uint32_t bb[4];
                ldsm4t(b_kn(bsb, LN, nv0 + 16 * jj, k0, lane), bb);
                mma(aw[2 * jj], a, bb[0], bb[1]);
                mma(aw[2 * jj + 1], a, bb[2], bb[3]);
            }
        }
        __syncthreads();
    }
    // epilogue: dC (fp32 atomics, group sum)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int l = rlo + 8 * hf;
        if (l >= nr) continue;
        float *dcrow = dC_acc + (((int64_t)b * L + t0 + r0 + l) * G + g) * N;
#pragma unroll
        for (int j = 0; j < TV; ++j) {
            const int n = nv0 + 8 * j + 2 * (lane & 3);
            atomicAdd(reinterpret_cast<float2 *>(dcrow + n), make_float2(aw[j][2 * hf], aw[j][2 * hf + 1]));
        }
    }
}

// ---- dispatch -----------------------------------------------------------------------

size_t sums_smem(int P, int N) { return (size_t)kT * ((P + 8) + (N + 8)) * 2; }
size_t src_smem(int P, int N) {
    return (size_t)(3 * kT * (N + 8) + 3 * kT * (P + 8) + 2 * kT * (kT + 8) + P * (N + 8)) * 2 +
           (size_t)(4 * kT + 12 * kT + 16) * 4;
}
size_t dst_smem(int P, int N) {
    return (size_t)(3 * kT * (N + 8) + 3 * kT * (P + 8) + kT * (kT + 8) + P * (N + 8)) * 2 + (size_t)(9 * kT) * 4;
}

template <int P, int N>
cudaError_t launch_sums(const FwdProblem &p, bool adjoint, const void *u, const void *v, const float *acs,
                        const float *dtw, float *out, cudaStream_t s) {
    const size_t smem = sums_smem(P, N);
    dim3 grid((unsigned)p.nc, (unsigned)p.H, (unsigned)p.B);
    cudaError_t e;
    if (adjoint) {
        if ((e = cudaFuncSetAttribute(k_chunk_sums_mma<P, N, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)))
            return e;
        k_chunk_sums_mma<P, N, true><<<grid, kThr, smem, s>>>(static_cast<const bf16 *>(u), static_cast<const bf16 *>(v),
                                                              acs, dtw, p.L, (int)p.H, (int)p.G, (int)p.Q, (int)p.nc,
                                                              out);
    } else {
        if ((e = cudaFuncSetAttribute(k_chunk_sums_mma<P, N, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)))
            return e;
        k_chunk_sums_mma<P, N, false><<<grid, kThr, smem, s>>>(static_cast<const bf16 *>(u),
                                                               static_cast<const bf16 *>(v), acs, dtw, p.L, (int)p.H,
                                                               (int)p.G, (int)p.Q, (int)p.nc, out);
    }
    return cudaGetLastError();
}

template <int P, int N>
cudaError_t launch_src(const FwdProblem &p, const void *dy, const float *acs, const float *dtw, const float *gend,
                       void *dx, float *dB_acc, float *kq, float *rq, float *uq, float *ddt_dir, float *dDpart,
                       cudaStream_t s) {
    const size_t smem = src_smem(P, N);
    const int nrt = mma_row_tiles(p);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_bwd_src_mma<P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
        return e;
    dim3 grid((unsigned)(p.nc * nrt), (unsigned)p.H, (unsigned)p.B);
    k_bwd_src_mma<P, N><<<grid, kThr2, smem, s>>>(
        static_cast<const bf16 *>(p.x), static_cast<const bf16 *>(p.Bm), static_cast<const bf16 *>(p.Cm),
        static_cast<const bf16 *>(dy), acs, dtw, gend, p.D, p.L, (int)p.H, (int)p.G, (int)p.Q, (int)p.nc, nrt,
        static_cast<bf16 *>(dx), dB_acc, kq, rq, uq, ddt_dir, dDpart);
    return cudaGetLastError();
}

template <int P, int N>
cudaError_t launch_dst(const FwdProblem &p, const void *dy, const float *acs, const float *dtw, const float *s_in,
                       float *dC_acc, float *tq, cudaStream_t s) {
    const size_t smem = dst_smem(P, N);
    const int nrt = mma_row_tiles(p);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_bwd_dst_mma<P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
        return e;
    dim3 grid((unsigned)(p.nc * nrt), (unsigned)p.H, (unsigned)p.B);
    k_bwd_dst_mma<P, N><<<grid, kThr2, smem, s>>>(static_cast<const bf16 *>(p.x), static_cast<const bf16 *>(p.Bm),
                                                 static_cast<const bf16 *>(p.Cm), static_cast<const bf16 *>(dy), acs,
                                                 dtw, s_in, p.L, (int)p.H, (int)p.G, (int)p.Q, (int)p.nc, nrt, dC_acc,
                                                 tq);
    return cudaGetLastError();
}

// (P, N) pairs with a compiled instance
#define SSD_MMA_SHAPES(X) X(64, 64) X(64, 128) X(64, 256) X(128, 128)

}  // namespace

bool mma_bwd_supported(const FwdProblem &p) {
    if (p.dtype != SSD_BF16) return false;
#define SSD_CASE(PP, NN) \
    if (p.P == PP && p.N == NN) return true;
    SSD_MMA_SHAPES(SSD_CASE)
#undef SSD_CASE
    return false;
}

int mma_row_tiles(const FwdProblem &p) { return (int)((p.Q + kT - 1) / kT); }

cudaError_t mma_chunk_sums(const FwdProblem &p, bool adjoint, const void *u, const void *v, const float *acs,
                           const float *dtw, float *out, cudaStream_t s) {
#define SSD_CASE(PP, NN) \
    if (p.P == PP && p.N == NN) return launch_sums<PP, NN>(p, adjoint, u, v, acs, dtw, out, s);
    SSD_MMA_SHAPES(SSD_CASE)
#undef SSD_CASE
    return cudaErrorInvalidValue;
}

cudaError_t mma_bwd_src(const FwdProblem &p, const void *dy, const float *acs, const float *dtw, const float *gend,
                        void *dx, float *dB_acc, float *kq, float *rq, float *uq, float *ddt_dir, float *dDpart,
                        cudaStream_t s) {
#define SSD_CASE(PP, NN) \
    if (p.P == PP && p.N == NN)  \
        return launch_src<PP, NN>(p, dy, acs, dtw, gend, dx, dB_acc, kq, rq, uq, ddt_dir, dDpart, s);
    SSD_MMA_SHAPES(SSD_CASE)
#undef SSD_CASE
    return cudaErrorInvalidValue;
}

cudaError_t mma_bwd_dst(const FwdProblem &p, const void *dy, const float *acs, const float *dtw, const float *s_in,
                        float *dC_acc, float *tq, cudaStream_t s) {
#define SSD_CASE(PP, NN) \
    if (p.P == PP && p.N == NN) return launch_dst<PP, NN>(p, dy, acs, dtw, s_in, dC_acc, tq, s);
    SSD_MMA_SHAPES(SSD_CASE)
#undef SSD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace ssd
