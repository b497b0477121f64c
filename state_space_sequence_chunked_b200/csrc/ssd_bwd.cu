// Backward pass of the chunked SSD forward, fp32 CUDA-core arithmetic.
//
// It returns the gradient of sum(dy * y) + sum(dh_final * h_final) with respect to x, dt, A,
// B, C, D and h0. As in the hardware-aware algorithm of "A Visual Guide to Mamba and SSMs"
// (section "Recomputation"), no forward intermediate is stored: the states entering every
// chunk are recomputed here from the inputs (steps 0, 2, 3 of the chunked algorithm in the
// Mamba-2 SSD write-up, "SSD 算法：分块和状态传递").
//
// With A_cs the within-chunk cumsum of a = dt A_h, S_in[c] the state entering chunk c and
// Gend[c] the gradient with respect to the state leaving chunk c:
//   reverse state pass   Gend[nc-1] = dh_final, Gend[c-1] = exp(A_cs[c,Q-1]) Gend[c] + R[c],
//                        R[c] = sum_{l in c} exp(A_cs[l]) dy_l C_l^T, dh0 = Gend[-1]
//   tokens as sources    u_s = sum_{l >= s} exp(A_cs[l]-A_cs[s]) (C_l.B_s) dy_l + exp(A_cs[Q-1]-A_cs[s]) Gend B_s
//                        v_s = sum_{l >= s} exp(A_cs[l]-A_cs[s]) (dy_l.x_s) C_l + exp(A_cs[Q-1]-A_cs[s]) Gend^T x_s
//                        dx_s = dt_s u_s + D dy_s, dB_s += dt_s v_s, ddt_s(direct) = x_s.u_s
//   tokens as targets    w_l = sum_{s <= l} exp(A_cs[l]-A_cs[s]) dt_s (dy_l.x_s) B_s + exp(A_cs[l]) S_in^T dy_l
//                        dC_l += w_l
//   log-decay gradient   g_l = C_l.w_l - dt_l B_l.v_l (+ <dh_final, h_final> at the last token):
//                        the derivative with respect to the running sum sum_{k<=l} a_k, so the
//                        gradient of a_t is the reverse cumsum G_t = sum_{l >= t} g_l, and
//                        ddt_t = A_h G_t + ddt_t(direct), dA_h = sum_{b,t} dt_t G_t.
// dB and dC sum over the heads of a group (fp32 atomics into the workspace, then one
// conversion to the input dtype); dA and dD are reduced in a fixed order.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;        // tokens per tile
constexpr int kMaxCol = 8;       // column blocks of 32: P, N <= 256

struct BwdWs {
    float *acs, *dtw, *states, *dstates, *hfin, *dcs, *ddt_dir, *dB, *dC, *hterm, *dDpart, *dAbh, *dDbh;
    float *kq, *rq, *uq, *tq, *ec;  // chunk-local pieces of the log-decay gradient (tensor-core path)
};

size_t n_chunk_rows(const FwdProblem &p) { return (size_t)(p.B * p.H * p.nc * p.Q); }
size_t n_states(const FwdProblem &p) { return (size_t)(p.B * p.H * p.nc) * (size_t)(p.P * p.N); }
int n_row_tiles(const FwdProblem &p) { return (int)((p.Q + kRows - 1) / kRows); }

BwdWs carve(const FwdProblem &p, void *ws, size_t *total) {
    char *base = static_cast<char *>(ws);
    size_t off = 0;
    auto take = [&](size_t n) {
        float *q = base ? reinterpret_cast<float *>(base + off) : nullptr;
        off += align_up(n * sizeof(float), kWsAlign);
        return q;
    };
    const size_t BH = (size_t)(p.B * p.H), BLGN = (size_t)(p.B * p.L * p.G * p.N);
    BwdWs w;
    w.acs = take(n_chunk_rows(p));
    w.dtw = take(n_chunk_rows(p));
    w.states = take(n_states(p));
    w.dstates = take(n_states(p));
    w.hfin = take(BH * (size_t)(p.P * p.N));
    w.dcs = take(n_chunk_rows(p));
    w.ddt_dir = take(n_chunk_rows(p));
    w.dB = take(BLGN);
    w.dC = take(BLGN);
    w.hterm = take(BH);
    w.dDpart = take(BH * (size_t)p.nc * (size_t)n_row_tiles(p));
    w.dAbh = take(BH);
    w.dDbh = take(BH);
    w.kq = take(n_chunk_rows(p));
    w.rq = take(n_chunk_rows(p));
    w.uq = take(n_chunk_rows(p));
    w.tq = take(n_chunk_rows(p));
    w.ec = take(BH * (size_t)p.nc);
    if (total) *total = off;
    return w;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Reverse state pass. grid (ceil(P*N/256), H, B). R[c] (in dstates) is replaced by Gend[c].
// Also hterm[b,h] = <dh_final, h_final>, the last token's extra log-decay gradient.
// With ec != NULL (the tensor-core path) also ec[b,h,c] += <Gend[c], S_in[c]> (s_in = the
// entering states).
__global__ void __launch_bounds__(kThreads)
    k_dstate_pass(const float *__restrict__ acs, const float *__restrict__ dh_final,
                  const float *__restrict__ hfin, const float *__restrict__ s_in, int H, int PN, int Q, int nc,
                  float *__restrict__ dstates, float *__restrict__ dh0, float *__restrict__ hterm,
                  float *__restrict__ ec) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * H + h;
    const bool valid = e < PN;
    __shared__ float red[8][kThreads / 32];
    float run = (valid && dh_final) ? dh_final[bh * PN + e] : 0.f;
    if (dh_final) {
        const float part = warp_sum(valid ? run * hfin[bh * PN + e] : 0.f);
        if ((threadIdx.x & 31) == 0) atomicAdd(hterm + bh, part);
    }
    // serial in c; the loads of 8 chunks are issued before the chain
    for (int c1 = nc - 1; c1 >= 0; c1 -= 8) {
        float r[8], dec[8], si[8], part[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c1 - i;
            r[i] = (valid && c >= 0) ? dstates[(bh * nc + c) * PN + e] : 0.f;
            si[i] = (ec && valid && c >= 0) ? s_in[(bh * nc + c) * PN + e] : 0.f;
            dec[i] = c >= 0 ? acs[(bh * nc + c) * Q + Q - 1] : 0.f;
            part[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c1 - i;
            if (c >= 0) {
                if (valid) dstates[(bh * nc + c) * PN + e] = run;
                if (ec) part[i] = run * si[i];
                run = fmaf(expf(dec[i]), run, r[i]);
            }
        }
        if (ec) {  // <Gend[c], S_in[c]>: reduced over the CTA, then one atomic per chunk
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float v = warp_sum(part[i]);
                if ((threadIdx.x & 31) == 0) red[i][threadIdx.x >> 5] = v;
            }
            __syncthreads();
            if (threadIdx.x < 8 && c1 - (int)threadIdx.x >= 0) {
                float v = 0.f;
                for (int w = 0; w < kThreads / 32; ++w) v += red[threadIdx.x][w];
                atomicAdd(ec + bh * nc + c1 - threadIdx.x, v);
            }
            __syncthreads();
        }
    }
    if (valid && dh0) dh0[bh * PN + e] = run;
}

// Tokens as sources. grid (nc * nrt, H, B); a tile of 32 tokens s of one chunk.
// Warp w owns rows s = w + 8 i (i < 4); lane owns columns p (or n) = lane + 32 j.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    k_bwd_src(const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
              const T *__restrict__ dy, const float *__restrict__ acs, const float *__restrict__ dtw,
              const float *__restrict__ gend, const float *__restrict__ D, int64_t L, int H, int P, int G,
              int N, int Q, int nc, int nrt, T *__restrict__ dx, float *__restrict__ dB_acc,
              float *__restrict__ dcs, float *__restrict__ ddt_dir, float *__restrict__ dDpart) {
    extern __shared__ float sm[];
    const int NS = N + 1, PS = P + 1;
    float *bo = sm;                  // [32][N+1]  B_s of the tile
    float *xo = bo + kRows * NS;     // [32][P+1]  x_s of the tile
    float *cl = xo + kRows * PS;     // [32][N+1]  C_l of a target tile
    float *dl = cl + kRows * NS;     // [32][P+1]  dy_l of a target tile
    float *w1 = dl + kRows * PS;     // [32][33]   (C_l.B_s) exp(A_cs[l]-A_cs[s]), l >= s
    float *w2 = w1 + kRows * 33;     // [32][33]   (dy_l.x_s) exp(A_cs[l]-A_cs[s]), l >= s
    float *gs = w2 + kRows * 33;     // [P][33]    32 columns of Gend
    float *as = gs + P * 33;         // [32]       A_cs of the tile rows
    float *al = as + kRows;          // [32]       A_cs of the target rows
    float *red = al + kRows;         // [8]

    const int c = blockIdx.x / nrt, rt = blockIdx.x % nrt, r0 = rt * kRows;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    const int64_t bh = (int64_t)b * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (r0 >= q) {
        if (tid == 0) dDpart[(bh * nc + c) * nrt + rt] = 0.f;
        return;
    }
    const int nr = min(kRows, q - r0);
    const int64_t lb = (bh * nc + c) * Q;
    const int pj = (P + 31) / 32, nj = (N + 31) / 32;

    for (int i = tid; i < kRows * N; i += kThreads) {
        const int s = i / N, n = i % N;
        bo[s * NS + n] = s < nr ? to_f32(Bm[(((int64_t)b * L + t0 + r0 + s) * G + g) * N + n]) : 0.f;
    }
    for (int i = tid; i < kRows * P; i += kThreads) {
        const int s = i / P, p = i % P;
        xo[s * PS + p] = s < nr ? to_f32(x[(((int64_t)b * L + t0 + r0 + s) * H + h) * P + p]) : 0.f;
    }
    for (int i = tid; i < kRows; i += kThreads) as[i] = acs[lb + min(r0 + i, Q - 1)];

    float au[4 * kMaxCol], av[4 * kMaxCol];
#pragma unroll
    for (int k = 0; k < 4 * kMaxCol; ++k) au[k] = av[k] = 0.f;

    // state part: Gend B_s and Gend^T x_s, 32 columns n of Gend at a time
    const float *ge = gend + (bh * nc + c) * (int64_t)P * N;
    for (int n0 = 0; n0 < N; n0 += 32) {
        const int nw = min(32, N - n0);
        __syncthreads();
        for (int i = tid; i < P * 32; i += kThreads) {
            const int p = i >> 5, jj = i & 31;
            gs[p * 33 + jj] = jj < nw ? ge[(int64_t)p * N + n0 + jj] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) {
            const int p = lane + 32 * j;
            if (j < pj && p < P) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int s = warp + 8 * i;
                    float a = au[4 * j + i];
                    for (int jj = 0; jj < nw; ++jj) a = fmaf(gs[p * 33 + jj], bo[s * NS + n0 + jj], a);
                    au[4 * j + i] = a;
                }
            }
        }
        {
            const int jn = n0 >> 5;  // this column block of v
#pragma unroll
            for (int j = 0; j < kMaxCol; ++j) {
                if (j == jn && lane < nw) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int s = warp + 8 * i;
                        float a = 0.f;
                        for (int p = 0; p < P; ++p) a = fmaf(gs[p * 33 + lane], xo[s * PS + p], a);
                        av[4 * j + i] = a;
                    }
                }
            }
        }
    }
    {
        const float aend = acs[lb + Q - 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float f = expf(aend - as[warp + 8 * i]);
#pragma unroll
            for (int j = 0; j < kMaxCol; ++j) {
                au[4 * j + i] *= f;
                av[4 * j + i] *= f;
            }
        }
    }

    // within the chunk: target tiles l >= s
    for (int l0 = r0; l0 < q; l0 += kRows) {
        const int nl = min(kRows, q - l0);
        __syncthreads();
        for (int i = tid; i < kRows * N; i += kThreads) {
            const int l = i / N, n = i % N;
            cl[l * NS + n] = l < nl ? to_f32(Cm[(((int64_t)b * L + t0 + l0 + l) * G + g) * N + n]) : 0.f;
        }
        for (int i = tid; i < kRows * P; i += kThreads) {
            const int l = i / P, p = i % P;
            dl[l * PS + p] = l < nl ? to_f32(dy[(((int64_t)b * L + t0 + l0 + l) * H + h) * P + p]) : 0.f;
        }
        for (int i = tid; i < kRows; i += kThreads) al[i] = acs[lb + min(l0 + i, Q - 1)];
        __syncthreads();
        for (int i = tid; i < kRows * kRows; i += kThreads) {
            const int l = i >> 5, s = i & 31;
            float v1 = 0.f, v2 = 0.f;
            if (l0 + l >= r0 + s && l < nl && s < nr) {
                float d1 = 0.f, d2 = 0.f;
                for (int n = 0; n < N; ++n) d1 = fmaf(cl[l * NS + n], bo[s * NS + n], d1);
                for (int p = 0; p < P; ++p) d2 = fmaf(dl[l * PS + p], xo[s * PS + p], d2);
                const float dec = expf(al[l] - as[s]);
                v1 = d1 * dec;
                v2 = d2 * dec;
            }
            w1[l * 33 + s] = v1;
            w2[l * 33 + s] = v2;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) {
            const int p = lane + 32 * j;
            if (j < pj && p < P) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int s = warp + 8 * i;
                    float a = au[4 * j + i];
                    for (int l = 0; l < nl; ++l) a = fmaf(w1[l * 33 + s], dl[l * PS + p], a);
                    au[4 * j + i] = a;
                }
            }
            const int n = lane + 32 * j;
            if (j < nj && n < N) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int s = warp + 8 * i;
                    float a = av[4 * j + i];
                    for (int l = 0; l < nl; ++l) a = fmaf(w2[l * 33 + s], cl[l * NS + n], a);
                    av[4 * j + i] = a;
                }
            }
        }
    }

    // epilogue: dx, ddt (direct), dB, the source half of the log-decay gradient, dD
    const float Dh = D ? D[h] : 0.f;
    float dd = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int s = warp + 8 * i;
        const bool row = s < nr;
        const int64_t t = t0 + r0 + s;
        const float dts = row ? dtw[lb + r0 + s] : 0.f;
        float xu = 0.f, bv = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) {
            const int p = lane + 32 * j;
            if (row && j < pj && p < P) {
                const int64_t off = ((b * L + t) * H + h) * (int64_t)P + p;
                const float dyv = to_f32(dy[off]), xv = xo[s * PS + p];
                store_as(dx + off, fmaf(dts, au[4 * j + i], Dh * dyv));
                xu = fmaf(xv, au[4 * j + i], xu);
                dd = fmaf(dyv, xv, dd);
            }
            const int n = lane + 32 * j;
            if (row && j < nj && n < N) {
                const float db = dts * av[4 * j + i];
                atomicAdd(dB_acc + ((b * L + t) * G + g) * (int64_t)N + n, db);
                bv = fmaf(bo[s * NS + n], db, bv);
            }
        }
        xu = warp_sum(xu);
        bv = warp_sum(bv);
        if (row && lane == 0) {
            ddt_dir[lb + r0 + s] = xu;
            dcs[lb + r0 + s] = -bv;
        }
    }
    dd = warp_sum(dd);
    if (lane == 0) red[warp] = dd;
    __syncthreads();
    if (tid == 0) {
        float sacc = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) sacc += red[w];
        dDpart[(bh * nc + c) * nrt + rt] = sacc;
    }
}

// Tokens as targets. grid (nc * nrt, H, B); a tile of 32 tokens l of one chunk.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    k_bwd_dst(const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
              const T *__restrict__ dy, const float *__restrict__ acs, const float *__restrict__ dtw,
              const float *__restrict__ s_in, int64_t L, int H, int P, int G, int N, int Q, int nc, int nrt,
              float *__restrict__ dC_acc, float *__restrict__ dcs) {
    extern __shared__ float sm[];
    const int NS = N + 1, PS = P + 1;
    float *co = sm;                  // [32][N+1]  C_l of the tile
    float *dl = co + kRows * NS;     // [32][P+1]  dy_l of the tile
    float *bs = dl + kRows * PS;     // [32][N+1]  B_s of a source tile
    float *xs = bs + kRows * NS;     // [32][P+1]  x_s of a source tile
    float *w3 = xs + kRows * PS;     // [32][33]   (dy_l.x_s) dt_s exp(A_cs[l]-A_cs[s]), s <= l
    float *gs = w3 + kRows * 33;     // [P][33]    32 columns of S_in
    float *al = gs + P * 33;         // [32]
    float *as = al + kRows;          // [32]
    float *ds = as + kRows;          // [32]       dt of the source rows

    const int c = blockIdx.x / nrt, r0 = (blockIdx.x % nrt) * kRows;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    if (r0 >= q) return;
    const int nr = min(kRows, q - r0);
    const int64_t bh = (int64_t)b * H + h;
    const int64_t lb = (bh * nc + c) * Q;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nj = (N + 31) / 32;

    for (int i = tid; i < kRows * N; i += kThreads) {
        const int l = i / N, n = i % N;
        co[l * NS + n] = l < nr ? to_f32(Cm[(((int64_t)b * L + t0 + r0 + l) * G + g) * N + n]) : 0.f;
    }
    for (int i = tid; i < kRows * P; i += kThreads) {
        const int l = i / P, p = i % P;
        dl[l * PS + p] = l < nr ? to_f32(dy[(((int64_t)b * L + t0 + r0 + l) * H + h) * P + p]) : 0.f;
    }
    for (int i = tid; i < kRows; i += kThreads) al[i] = acs[lb + min(r0 + i, Q - 1)];

    float aw[4 * kMaxCol];
#pragma unroll
    for (int k = 0; k < 4 * kMaxCol; ++k) aw[k] = 0.f;

    // state part: exp(A_cs[l]) S_in^T dy_l
    const float *si = s_in + (bh * nc + c) * (int64_t)P * N;
    for (int n0 = 0; n0 < N; n0 += 32) {
        const int nw = min(32, N - n0);
        __syncthreads();
        for (int i = tid; i < P * 32; i += kThreads) {
            const int p = i >> 5, jj = i & 31;
            gs[p * 33 + jj] = jj < nw ? si[(int64_t)p * N + n0 + jj] : 0.f;
        }
        __syncthreads();
        const int jn = n0 >> 5;
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) {
            if (j == jn && lane < nw) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int l = warp + 8 * i;
                    float a = 0.f;
                    for (int p = 0; p < P; ++p) a = fmaf(gs[p * 33 + lane], dl[l * PS + p], a);
                    aw[4 * j + i] = a;
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float f = expf(al[warp + 8 * i]);
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) aw[4 * j + i] *= f;
    }

    // within the chunk: source tiles s <= l
    for (int s0 = 0; s0 < r0 + nr; s0 += kRows) {
        const int ns = min(kRows, q - s0);
        __syncthreads();
        for (int i = tid; i < kRows * N; i += kThreads) {
            const int s = i / N, n = i % N;
            bs[s * NS + n] = s < ns ? to_f32(Bm[(((int64_t)b * L + t0 + s0 + s) * G + g) * N + n]) : 0.f;
        }
        for (int i = tid; i < kRows * P; i += kThreads) {
            const int s = i / P, p = i % P;
            xs[s * PS + p] = s < ns ? to_f32(x[(((int64_t)b * L + t0 + s0 + s) * H + h) * P + p]) : 0.f;
        }
        for (int i = tid; i < kRows; i += kThreads) {
            as[i] = acs[lb + min(s0 + i, Q - 1)];
            ds[i] = i < ns ? dtw[lb + s0 + i] : 0.f;
        }
        __syncthreads();
        for (int i = tid; i < kRows * kRows; i += kThreads) {
            const int l = i >> 5, s = i & 31;
            float v = 0.f;
            if (s0 + s <= r0 + l && s < ns && l < nr) {
                float d = 0.f;
                for (int p = 0; p < P; ++p) d = fmaf(dl[l * PS + p], xs[s * PS + p], d);
                v = d * ds[s] * expf(al[l] - as[s]);
            }
            w3[l * 33 + s] = v;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) {
            const int n = lane + 32 * j;
            if (j < nj && n < N) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int l = warp + 8 * i;
                    float a = aw[4 * j + i];
                    for (int s = 0; s < ns; ++s) a = fmaf(w3[l * 33 + s], bs[s * NS + n], a);
                    aw[4 * j + i] = a;
                }
            }
        }
    }

    // epilogue: dC (group sum) and the target half of the log-decay gradient
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int l = warp + 8 * i;
        const bool row = l < nr;
        const int64_t t = t0 + r0 + l;
        float cw = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxCol; ++j) {
            const int n = lane + 32 * j;
            if (row && j < nj && n < N) {
                atomicAdd(dC_acc + ((b * L + t) * G + g) * (int64_t)N + n, aw[4 * j + i]);
                cw = fmaf(co[l * NS + n], aw[4 * j + i], cw);
            }
        }
        cw = warp_sum(cw);
        if (row && lane == 0) dcs[lb + r0 + l] += cw;
    }
}

// Reverse cumsum of the log-decay gradient over the whole sequence of one (b, h).
// grid (H, B), 256 threads; tiles of 256 tokens from the end.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    k_bwd_dt(const float *__restrict__ dcs, const float *__restrict__ ddt_dir, const float *__restrict__ dtw,
             const float *__restrict__ hterm, const float *__restrict__ dDpart, const float *__restrict__ A,
             int64_t L, int H, int Q, int nc, int nrt, T *__restrict__ ddt, float *__restrict__ dAbh,
             float *__restrict__ dDbh) {
    __shared__ float wsum[kThreads / 32];
    __shared__ float carry_s;
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t bh = (int64_t)b * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float Ah = A[h];
    float carry = hterm ? hterm[bh] : 0.f;  // <dh_final, h_final> enters at the last token
    float da_acc = 0.f;
    for (int64_t e0 = ((L - 1) / kThreads) * kThreads; e0 >= 0; e0 -= kThreads) {
        // thread tid handles token t = e0 + (255 - tid): a forward inclusive scan over tid is
        // then a reverse cumsum over t
        const int64_t t = e0 + (kThreads - 1 - tid);
        const bool ok = t < L;
        const int64_t ci = ok ? t / Q : 0, li = ok ? t % Q : 0;
        const int64_t wi = (bh * nc + ci) * Q + li;
        float v = ok ? dcs[wi] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (lane == 31) wsum[warp] = v;
        __syncthreads();
        float pre = carry;
        for (int w = 0; w < warp; ++w) pre += wsum[w];
        const float G = v + pre;  // sum over tokens >= t of the log-decay gradient
        if (ok) {
            const float dtv = dtw[wi];
            store_as(ddt + ((int64_t)b * L + t) * H + h, fmaf(Ah, G, ddt_dir[wi]));
            da_acc = fmaf(dtv, G, da_acc);
        }
        if (tid == kThreads - 1) carry_s = G;
        __syncthreads();
        carry = carry_s;
    }
    float dd = 0.f;
    for (int i = tid; i < nc * nrt; i += kThreads) dd += dDpart[bh * nc * nrt + i];
    da_acc = warp_sum(da_acc);
    dd = warp_sum(dd);
    __syncthreads();
    if (lane == 0) wsum[warp] = da_acc;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) s += wsum[w];
        dAbh[bh] = s;
    }
    __syncthreads();
    if (lane == 0) wsum[warp] = dd;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) s += wsum[w];
        dDbh[bh] = s;
    }
}

// Tensor-core path: the log-decay gradient of token t from chunk-local pieces only,
//   G_t = <Gbar_t, exp(a_t) S_{t-1}>
//       = sum_{u<t} (K_u - R_u)            pairs s < t <= l of the chunk (K: row sums over l > s,
//                                          R: column sums over s < l, of the same fp32 products)
//       + sum_{l>=t} T_l                   T_l = exp(A_cs[l]) dy_l^T S_in C_l
//       + sum_{s<t} U_s                    U_s = exp(A_cs[Q-1]-A_cs[s]) dt_s x_s^T Gend B_s
//       + exp(A_cs[Q-1]) <Gend, S_in>
// (the adjoint and the state of the recurrence written in the chunk's terms), then
// ddt_t = A_h G_t + ddt_t(direct) and dA_h += dt_t G_t. grid (H, B); a chunk at a time,
// thread l = token l of the chunk (Q <= 256).
template <typename T>
__global__ void __launch_bounds__(kThreads)
    k_bwd_dt_local(const float *__restrict__ kq, const float *__restrict__ rq, const float *__restrict__ uq,
                   const float *__restrict__ tq, const float *__restrict__ ec, const float *__restrict__ acs,
                   const float *__restrict__ ddt_dir, const float *__restrict__ dtw, const float *__restrict__ dDpart,
                   const float *__restrict__ A, int64_t L, int H, int Q, int nc, int nrt, T *__restrict__ ddt,
                   float *__restrict__ dAbh, float *__restrict__ dDbh) {
    __shared__ float wa[kThreads / 32], wb[kThreads / 32];
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t bh = (int64_t)b * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float Ah = A[h];
    float da = 0.f;
    for (int c = 0; c < nc; ++c) {
        const int64_t t0 = (int64_t)c * Q;
        const int q = (int)min((int64_t)Q, L - t0);
        const int64_t lb = (bh * nc + c) * Q;
        const bool ok = tid < q;
        // prefix (exclusive) of K - R + U; suffix (inclusive) of T = total - exclusive prefix
        float pv = ok ? kq[lb + tid] - rq[lb + tid] + uq[lb + tid] : 0.f;
        float tv = ok ? tq[lb + tid] : 0.f;
        float ip = pv, it = tv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float a = __shfl_up_sync(0xffffffffu, ip, o), bb = __shfl_up_sync(0xffffffffu, it, o);
            if (lane >= o) {
                ip += a;
                it += bb;
            }
        }
        __syncthreads();
        if (lane == 31) {
            wa[warp] = ip;
            wb[warp] = it;
        }
        __syncthreads();
        float pre_p = 0.f, pre_t = 0.f, tot_t = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) {
                pre_p += wa[w];
                pre_t += wb[w];
            }
            tot_t += wb[w];
        }
        const float excl_p = pre_p + ip - pv, excl_t = pre_t + it - tv;
        const float G = excl_p + (tot_t - excl_t) + __expf(acs[lb + Q - 1]) * ec[bh * nc + c];
        if (ok) {
            const float dtv = dtw[lb + tid];
            store_as(ddt + ((int64_t)b * L + t0 + tid) * H + h, fmaf(Ah, G, ddt_dir[lb + tid]));
            da = fmaf(dtv, G, da);
        }
    }
    float dd = 0.f;
    for (int i = tid; i < nc * nrt; i += kThreads) dd += dDpart[bh * nc * nrt + i];
    da = warp_sum(da);
    dd = warp_sum(dd);
    __syncthreads();
    if (lane == 0) {
        wa[warp] = da;
        wb[warp] = dd;
    }
    __syncthreads();
    if (tid == 0) {
        float s1 = 0.f, s2 = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) {
            s1 += wa[w];
            s2 += wb[w];
        }
        dAbh[bh] = s1;
        dDbh[bh] = s2;
    }
}

// dA[h] = sum_b, dD[h] = sum_b (fixed order); dB/dC from the fp32 sums to the output dtype.
__global__ void k_bwd_reduce_heads(const float *__restrict__ dAbh, const float *__restrict__ dDbh, int64_t B, int H,
                                   float *__restrict__ dA, float *__restrict__ dD) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float sa = 0.f, sd = 0.f;
    for (int64_t b = 0; b < B; ++b) {
        sa += dAbh[b * H + h];
        sd += dDbh[b * H + h];
    }
    dA[h] = sa;
    if (dD) dD[h] = sd;
}

template <typename T>
__global__ void k_convert(const float *__restrict__ src, int64_t n, T *__restrict__ dst) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        store_as(dst + i, src[i]);
}

size_t src_smem(const FwdProblem &p) {
    return (size_t)(2 * kRows * (p.N + 1) + 2 * kRows * (p.P + 1) + 2 * kRows * 33 + p.P * 33 + 2 * kRows + 8) *
           sizeof(float);
}
size_t dst_smem(const FwdProblem &p) {
    return (size_t)(2 * kRows * (p.N + 1) + 2 * kRows * (p.P + 1) + kRows * 33 + p.P * 33 + 3 * kRows) *
           sizeof(float);
}

template <typename T>
cudaError_t run(const FwdProblem &p, const BwdGrads &gr, void *ws, cudaStream_t s) {
    const BwdWs w = carve(p, ws, nullptr);
    const int H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N, Q = (int)p.Q, nc = (int)p.nc;
    const int nrt = n_row_tiles(p);
    const size_t BH = (size_t)(p.B * p.H), BLGN = (size_t)(p.B * p.L * p.G * p.N);
    const T *x = static_cast<const T *>(p.x), *Bm = static_cast<const T *>(p.Bm);
    const T *Cm = static_cast<const T *>(p.Cm), *dy = static_cast<const T *>(gr.dy);
    cudaError_t e;

    if ((e = cudaMemsetAsync(w.dB, 0, BLGN * sizeof(float), s))) return e;
    if ((e = cudaMemsetAsync(w.dC, 0, BLGN * sizeof(float), s))) return e;
    if ((e = cudaMemsetAsync(w.hterm, 0, BH * sizeof(float), s))) return e;
    // bf16 inputs of a compiled (P, N) run every product on tensor cores (ssd_bwd_mma.cu)
    const bool tc = mma_bwd_supported(p);
    if (tc) {
        if ((e = cudaMemsetAsync(w.rq, 0, n_chunk_rows(p) * sizeof(float), s))) return e;
        if ((e = cudaMemsetAsync(w.ec, 0, BH * (size_t)nc * sizeof(float), s))) return e;
    }
    const int nrt_used = tc ? mma_row_tiles(p) : nrt;
    // recompute: A_cs, dt per chunk, S_in per chunk, h_final
    if (tc) {
        if ((e = simt_cumsum(p, w.acs, w.dtw, s))) return e;
        if ((e = mma_chunk_sums(p, false, p.x, p.Bm, w.acs, w.dtw, w.states, s))) return e;
        if ((e = simt_state_pass(p, w.acs, w.states, w.hfin, s))) return e;
        if ((e = mma_chunk_sums(p, true, gr.dy, p.Cm, w.acs, w.dtw, w.dstates, s))) return e;
    } else {
        if ((e = simt_states(p, w.acs, w.dtw, w.states, w.hfin, s))) return e;
        if ((e = simt_adjoint_chunk_sums(p, gr.dy, w.acs, w.dstates, s))) return e;
    }
    // R[c] (in dstates), then the reverse state pass
    {
        dim3 grid((P * N + kThreads - 1) / kThreads, H, (unsigned)p.B);
        k_dstate_pass<<<grid, kThreads, 0, s>>>(w.acs, gr.dh_final, w.hfin, w.states, H, P * N, Q, nc, w.dstates,
                                                gr.dh0, w.hterm, tc ? w.ec : nullptr);
        if ((e = cudaGetLastError())) return e;
    }
    if (tc) {
        if ((e = mma_bwd_src(p, gr.dy, w.acs, w.dtw, w.dstates, gr.dx, w.dB, w.kq, w.rq, w.uq, w.ddt_dir, w.dDpart,
                             s)))
            return e;
        if ((e = mma_bwd_dst(p, gr.dy, w.acs, w.dtw, w.states, w.dC, w.tq, s))) return e;
    } else {
        const size_t smem = src_smem(p);
        if ((e = cudaFuncSetAttribute(k_bwd_src<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        dim3 grid(nc * nrt, H, (unsigned)p.B);
        k_bwd_src<T><<<grid, kThreads, smem, s>>>(x, Bm, Cm, dy, w.acs, w.dtw, w.dstates, p.D, p.L, H, P, G, N, Q,
                                                  nc, nrt, static_cast<T *>(gr.dx), w.dB, w.dcs, w.ddt_dir,
                                                  w.dDpart);
        if ((e = cudaGetLastError())) return e;
        const size_t smem2 = dst_smem(p);
        if ((e = cudaFuncSetAttribute(k_bwd_dst<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)))
            return e;
        k_bwd_dst<T><<<grid, kThreads, smem2, s>>>(x, Bm, Cm, dy, w.acs, w.dtw, w.states, p.L, H, P, G, N, Q, nc,
                                                  nrt, w.dC, w.dcs);
        if ((e = cudaGetLastError())) return e;
    }
    {
        dim3 grid(H, (unsigned)p.B);
        if (tc)
            k_bwd_dt_local<T><<<grid, kThreads, 0, s>>>(w.kq, w.rq, w.uq, w.tq, w.ec, w.acs, w.ddt_dir, w.dtw,
                                                        w.dDpart, p.A, p.L, H, Q, nc, nrt_used,
                                                        static_cast<T *>(gr.ddt), w.dAbh, w.dDbh);
        else
            k_bwd_dt<T><<<grid, kThreads, 0, s>>>(w.dcs, w.ddt_dir, w.dtw, gr.dh_final ? w.hterm : nullptr,
                                                  w.dDpart, p.A, p.L, H, Q, nc, nrt_used, static_cast<T *>(gr.ddt),
                                                  w.dAbh, w.dDbh);
        if ((e = cudaGetLastError())) return e;
    }
    k_bwd_reduce_heads<<<(H + 127) / 128, 128, 0, s>>>(w.dAbh, w.dDbh, p.B, H, gr.dA, gr.dD);
    if ((e = cudaGetLastError())) return e;
    const int64_t nblk = (int64_t)(BLGN + 255) / 256;
    const int cgrid = (int)(nblk < 148 * 16 ? (nblk > 0 ? nblk : 1) : 148 * 16);
    k_convert<T><<<cgrid, 256, 0, s>>>(w.dB, (int64_t)BLGN, static_cast<T *>(gr.dBm));
    if ((e = cudaGetLastError())) return e;
    k_convert<T><<<cgrid, 256, 0, s>>>(w.dC, (int64_t)BLGN, static_cast<T *>(gr.dCm));
    return cudaGetLastError();
}

}  // namespace

size_t simt_bwd_workspace_bytes(const FwdProblem &p) {
    size_t total = 0;
    carve(p, nullptr, &total);
    return total;
}

bool simt_bwd_supported(const FwdProblem &p) {
    return src_smem(p) <= 227 * 1024 && dst_smem(p) <= 227 * 1024;
}

cudaError_t simt_bwd(const FwdProblem &p, const BwdGrads &g, void *ws, cudaStream_t s) {
    return p.dtype == SSD_F32 ? run<float>(p, g, ws, s) : run<__nv_bfloat16>(p, g, ws, s);
}

}  // namespace ssd
