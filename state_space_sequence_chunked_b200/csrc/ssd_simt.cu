// Chunked SSD forward with fp32 CUDA-core arithmetic.
//
// This is the exact path (fp32 inputs must match an fp64 evaluation to 1e-4
// relative, which tensor-core tf32 would not reach) and the general-shape path.
// It follows the four steps of the chunked algorithm in the Mamba-2 SSD write-up,
// "SSD 算法：分块和状态传递", one kernel per step:
//   k_cumsum       step 0: a = dt * A_h, inclusive cumsum restarted in every chunk
//   k_chunk_state  step 2: chunk state from a zero start, decayed to the chunk end
//   k_state_pass   step 3: the short sequential scan of states across chunks
//   k_chunk_scan   steps 1 + 4: diagonal block (C B^T o L) (dt x) plus
//                  exp(A_cs) C S_in^T plus the D skip
// Workspace (fp32): A_cs [B,H,nc,Q], dt [B,H,nc,Q] (zero past the sequence end),
// states [B,H,nc,P,N] (chunk states, overwritten in place by the entering states).
//
// The backward pass recomputes steps 0, 2 and 3 with these kernels (simt_states),
// and k_chunk_state's adjoint form gives the per-chunk sums exp(A_cs[l]) dy_l C_l^T
// that its reverse state pass consumes (simt_adjoint_chunk_sums).
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;

struct WsLayout {
    float *acs, *dtw, *states;
};

WsLayout carve(const FwdProblem &p, void *ws) {
    char *base = static_cast<char *>(ws);
    const size_t n_l = (size_t)(p.B * p.H * p.nc * p.Q);
    WsLayout w;
    w.acs = reinterpret_cast<float *>(base);
    base += align_up(n_l * sizeof(float), kWsAlign);
    w.dtw = reinterpret_cast<float *>(base);
    base += align_up(n_l * sizeof(float), kWsAlign);
    w.states = reinterpret_cast<float *>(base);
    return w;
}

// step 0. grid (nc, ceil(H/32), B). Shared: dt of the chunk for 32 heads.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_cumsum(const T *__restrict__ dt,
                                                     const float *__restrict__ A, int64_t L, int H,
                                                     int Q, int nc, float *__restrict__ acs,
                                                     float *__restrict__ dtw) {
    extern __shared__ float sdt[];  // [Q][33]
    const int c = blockIdx.x, hb = blockIdx.y * 32, b = blockIdx.z;
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    for (int i = threadIdx.x; i < Q * 32; i += blockDim.x) {
        const int l = i >> 5, hh = i & 31, h = hb + hh;
        float v = 0.f;
        if (l < q && h < H) v = to_f32(dt[((int64_t)b * L + t0 + l) * H + h]);
        sdt[l * 33 + hh] = v;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int hh = warp; hh < 32; hh += kThreads / 32) {
        const int h = hb + hh;
        if (h >= H) break;
        const float ah = A[h];
        const int64_t base = (((int64_t)b * H + h) * nc + c) * Q;
        float carry = 0.f;
        for (int l0 = 0; l0 < Q; l0 += 32) {
            const int l = l0 + lane;
            const float d = l < Q ? sdt[l * 33 + hh] : 0.f;
            float v = d * ah;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            v += carry;
            carry = __shfl_sync(0xffffffffu, v, 31);
            if (l < Q) {
                acs[base + l] = v;
                dtw[base + l] = d;
            }
        }
    }
}

// step 2. grid (nc * ntile, H, B); every thread owns 16 of the P*N outputs of its tile.
// Forward: sum_l exp(A_cs[Q-1] - A_cs[l]) dt_l x_l B_l^T (u = x, v = B).
// Adjoint (kAdj): sum_l exp(A_cs[l]) dy_l C_l^T (u = dy [B,L,H,P], v = C [B,L,G,N]),
// the gradient of the chunk's state-to-output term with respect to its entering state.
constexpr int kStateTileL = 32;
constexpr int kStatePerThread = 16;
constexpr int kStateTile = kThreads * kStatePerThread;

template <typename T, bool kAdj>
__global__ void __launch_bounds__(kThreads)
    k_chunk_state(const T *__restrict__ x, const T *__restrict__ Bm, const float *__restrict__ acs,
                  const float *__restrict__ dtw, int64_t L, int H, int P, int G, int N, int Q, int nc,
                  int ntile, float *__restrict__ states) {
    extern __shared__ float sm[];
    float *xs = sm;                       // [kStateTileL][P], x scaled by the decay weight
    float *bs = xs + kStateTileL * P;     // [kStateTileL][N]
    float *ws = bs + kStateTileL * N;     // [kStateTileL]
    const int c = blockIdx.x / ntile, tile = blockIdx.x % ntile;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    const int64_t lb = (((int64_t)b * H + h) * nc + c) * Q;
    const float last = acs[lb + Q - 1];
    const int PN = P * N;

    int pp[kStatePerThread], nn[kStatePerThread];
    float acc[kStatePerThread];
#pragma unroll
    for (int k = 0; k < kStatePerThread; ++k) {
        const int e = tile * kStateTile + threadIdx.x + k * kThreads;
        pp[k] = e < PN ? e / N : 0;
        nn[k] = e < PN ? e % N : 0;
        acc[k] = 0.f;
    }
    for (int l0 = 0; l0 < q; l0 += kStateTileL) {
        const int nl = min(kStateTileL, q - l0);
        for (int i = threadIdx.x; i < kStateTileL; i += blockDim.x)
            ws[i] = i < nl ? (kAdj ? expf(acs[lb + l0 + i]) : expf(last - acs[lb + l0 + i]) * dtw[lb + l0 + i])
                           : 0.f;
        __syncthreads();
        for (int i = threadIdx.x; i < kStateTileL * P; i += blockDim.x) {
            const int l = i / P, p = i % P;
            xs[i] = l < nl ? to_f32(x[((((int64_t)b * L + t0 + l0 + l) * H) + h) * P + p]) * ws[l] : 0.f;
        }
        for (int i = threadIdx.x; i < kStateTileL * N; i += blockDim.x) {
            const int l = i / N, n = i % N;
            bs[i] = l < nl ? to_f32(Bm[((((int64_t)b * L + t0 + l0 + l) * G) + g) * N + n]) : 0.f;
        }
        __syncthreads();
        for (int l = 0; l < nl; ++l) {
#pragma unroll
            for (int k = 0; k < kStatePerThread; ++k)
                acc[k] = fmaf(xs[l * P + pp[k]], bs[l * N + nn[k]], acc[k]);
        }
        __syncthreads();
    }
    float *out = states + (((int64_t)b * H + h) * nc + c) * PN;
#pragma unroll
    for (int k = 0; k < kStatePerThread; ++k) {
        const int e = tile * kStateTile + threadIdx.x + k * kThreads;
        if (e < PN) out[e] = acc[k];
    }
}

// step 3. grid (ceil(P*N/256), H, B). S_in[c] replaces the chunk state in place.
__global__ void __launch_bounds__(kThreads)
    k_state_pass(const float *__restrict__ acs, const float *__restrict__ h0, int H, int PN, int Q,
                 int nc, float *__restrict__ states, float *__restrict__ h_final) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const int64_t bh = (int64_t)b * H + h;
    float run = h0 ? h0[bh * PN + e] : 0.f;
    // the chain is serial in c; the loads of 8 chunks are issued before it
    for (int c0 = 0; c0 < nc; c0 += 8) {
        float sc[8], dec[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c0 + i;
            sc[i] = c < nc ? states[(bh * nc + c) * PN + e] : 0.f;
            dec[i] = c < nc ? acs[(bh * nc + c) * Q + Q - 1] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c0 + i;
            if (c < nc) {
                states[(bh * nc + c) * PN + e] = run;
                run = fmaf(expf(dec[i]), run, sc[i]);
            }
        }
    }
    if (h_final) h_final[bh * PN + e] = run;
}

// steps 1 + 4. grid (nc * nrt, H, B): a tile of 32 rows of one chunk, all P columns.
constexpr int kRows = 32;

template <typename T>
__global__ void __launch_bounds__(kThreads)
    k_chunk_scan(const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
                 const float *__restrict__ acs, const float *__restrict__ dtw,
                 const float *__restrict__ states, const float *__restrict__ D, int64_t L, int H,
                 int P, int G, int N, int Q, int nc, int nrt, T *__restrict__ y) {
    extern __shared__ float sm[];
    const int NS = N + 1;
    float *cs = sm;                  // [kRows][N+1]  C rows of this tile
    float *bs = cs + kRows * NS;     // [kRows][N+1]  B rows of the source tile
    float *xs = bs + kRows * NS;     // [kRows][P]    dt * x of the source tile
    float *gs = xs + kRows * P;      // [kRows][33]   masked, decayed C B^T
    float *st = gs + kRows * 33;     // [P][33]       32 columns of S_in
    float *al = st + P * 33;         // [kRows]       A_cs of the rows
    float *as = al + kRows;          // [kRows]       A_cs of the source rows

    const int c = blockIdx.x / nrt, r0 = (blockIdx.x % nrt) * kRows;
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int64_t t0 = (int64_t)c * Q;
    const int q = (int)min((int64_t)Q, L - t0);
    if (r0 >= q) return;
    const int nr = min(kRows, q - r0);
    const int64_t lb = (((int64_t)b * H + h) * nc + c) * Q;
    const int tid = threadIdx.x;
    const int nout = kRows * P;  // <= 32 * 256
    constexpr int kMaxOut = kRows * 256 / kThreads;
    float acc[kMaxOut];
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) acc[k] = 0.f;

    for (int i = tid; i < kRows * N; i += blockDim.x) {
        const int l = i / N, n = i % N;
        cs[l * NS + n] = l < nr ? to_f32(Cm[(((int64_t)b * L + t0 + r0 + l) * G + g) * N + n]) : 0.f;
    }
    for (int i = tid; i < kRows; i += blockDim.x) al[i] = acs[lb + min(r0 + i, Q - 1)];

    // step 4: exp(A_cs[l]) * sum_n C[l, n] S_in[p, n]
    const float *sin_ = states + (((int64_t)b * H + h) * nc + c) * (int64_t)P * N;
    for (int n0 = 0; n0 < N; n0 += 32) {
        const int nw = min(32, N - n0);
        __syncthreads();
        for (int i = tid; i < P * 32; i += blockDim.x) {
            const int p = i / 32, j = i % 32;
            st[p * 33 + j] = j < nw ? sin_[(int64_t)p * N + n0 + j] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kMaxOut; ++k) {
            const int e = tid + k * kThreads;
            if (e < nout) {
                const int l = e / P, p = e % P;
                float a = acc[k];
                for (int j = 0; j < nw; ++j) a = fmaf(cs[l * NS + n0 + j], st[p * 33 + j], a);
                acc[k] = a;
            }
        }
    }
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
        const int e = tid + k * kThreads;
        if (e < nout) acc[k] *= expf(al[e / P]);
    }

    // step 1: sum_{s <= l} (C_l . B_s) exp(A_cs[l] - A_cs[s]) dt_s x_s, source tiles of 32 rows
    for (int s0 = 0; s0 < r0 + nr; s0 += kRows) {
        const int ns = min(kRows, q - s0);
        __syncthreads();
        for (int i = tid; i < kRows * N; i += blockDim.x) {
            const int s = i / N, n = i % N;
            bs[s * NS + n] = s < ns ? to_f32(Bm[(((int64_t)b * L + t0 + s0 + s) * G + g) * N + n]) : 0.f;
        }
        for (int i = tid; i < kRows * P; i += blockDim.x) {
            const int s = i / P, p = i % P;
            xs[i] = s < ns ? to_f32(x[(((int64_t)b * L + t0 + s0 + s) * H + h) * P + p]) * dtw[lb + s0 + s]
                           : 0.f;
        }
        for (int i = tid; i < kRows; i += blockDim.x) as[i] = acs[lb + min(s0 + i, Q - 1)];
        __syncthreads();
        for (int i = tid; i < kRows * kRows; i += blockDim.x) {
            const int l = i / kRows, s = i % kRows;
            float v = 0.f;
            if (s0 + s <= r0 + l && s < ns && l < nr) {
                float dot = 0.f;
                for (int n = 0; n < N; ++n) dot = fmaf(cs[l * NS + n], bs[s * NS + n], dot);
                v = dot * expf(al[l] - as[s]);
            }
            gs[l * 33 + s] = v;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kMaxOut; ++k) {
            const int e = tid + k * kThreads;
            if (e < nout) {
                const int l = e / P, p = e % P;
                float a = acc[k];
                for (int s = 0; s < ns; ++s) a = fmaf(gs[l * 33 + s], xs[s * P + p], a);
                acc[k] = a;
            }
        }
    }

    // D skip and store
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
        const int e = tid + k * kThreads;
        if (e < nout) {
            const int l = e / P, p = e % P;
            if (l < nr) {
                const int64_t off = (((int64_t)b * L + t0 + r0 + l) * H + h) * P + p;
                const float xv = to_f32(x[off]);
                store_as(y + off, acc[k] + (D ? D[h] * xv : 0.f));
            }
        }
    }
}

template <typename T, bool kAdj>
cudaError_t launch_chunk_state(const FwdProblem &p, const void *u, const void *v, const float *acs,
                               const float *dtw, float *out, cudaStream_t s) {
    const int H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N, Q = (int)p.Q, nc = (int)p.nc;
    const int ntile = (P * N + kStateTile - 1) / kStateTile;
    const size_t smem = (size_t)(kStateTileL * (P + N) + kStateTileL) * sizeof(float);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_chunk_state<T, kAdj>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
        return e;
    dim3 grid(nc * ntile, H, (unsigned)p.B);
    k_chunk_state<T, kAdj><<<grid, kThreads, smem, s>>>(static_cast<const T *>(u), static_cast<const T *>(v), acs,
                                                        dtw, p.L, H, P, G, N, Q, nc, ntile, out);
    return cudaGetLastError();
}

// steps 0, 2, 3: A_cs and dt per chunk, then the state entering every chunk (in `states`)
template <typename T>
cudaError_t run_states(const FwdProblem &p, float *acs, float *dtw, float *states, float *h_final,
                       cudaStream_t s) {
    const int H = (int)p.H, P = (int)p.P, N = (int)p.N, Q = (int)p.Q, nc = (int)p.nc;
    const T *dt = static_cast<const T *>(p.dt);
    cudaError_t e;
    {
        const size_t smem = (size_t)Q * 33 * sizeof(float);
        if ((e = cudaFuncSetAttribute(k_cumsum<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        dim3 grid(nc, (H + 31) / 32, (unsigned)p.B);
        k_cumsum<T><<<grid, kThreads, smem, s>>>(dt, p.A, p.L, H, Q, nc, acs, dtw);
        if ((e = cudaGetLastError())) return e;
    }
    if ((e = launch_chunk_state<T, false>(p, p.x, p.Bm, acs, dtw, states, s))) return e;
    {
        dim3 grid((P * N + kThreads - 1) / kThreads, H, (unsigned)p.B);
        k_state_pass<<<grid, kThreads, 0, s>>>(acs, p.h0, H, P * N, Q, nc, states, h_final);
        if ((e = cudaGetLastError())) return e;
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t run(const FwdProblem &p, void *ws, cudaStream_t s) {
    const WsLayout w = carve(p, ws);
    const int H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N, Q = (int)p.Q, nc = (int)p.nc;
    const T *x = static_cast<const T *>(p.x);
    const T *Bm = static_cast<const T *>(p.Bm), *Cm = static_cast<const T *>(p.Cm);
    cudaError_t e;
    if ((e = run_states<T>(p, w.acs, w.dtw, w.states, p.h_final, s))) return e;
    {
        const int nrt = (Q + kRows - 1) / kRows;
        const size_t smem =
            (size_t)(2 * kRows * (N + 1) + kRows * P + kRows * 33 + P * 33 + 2 * kRows) * sizeof(float);
        if ((e = cudaFuncSetAttribute(k_chunk_scan<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        dim3 grid(nc * nrt, H, (unsigned)p.B);
        k_chunk_scan<T><<<grid, kThreads, smem, s>>>(x, Bm, Cm, w.acs, w.dtw, w.states, p.D, p.L, H, P, G, N,
                                                     Q, nc, nrt, static_cast<T *>(p.y));
        if ((e = cudaGetLastError())) return e;
    }
    return cudaSuccess;
}

}  // namespace

size_t simt_fwd_workspace_bytes(const FwdProblem &p) {
    const size_t n_l = (size_t)(p.B * p.H * p.nc * p.Q);
    const size_t n_s = (size_t)(p.B * p.H * p.nc) * (size_t)(p.P * p.N);
    return 2 * align_up(n_l * sizeof(float), kWsAlign) + align_up(n_s * sizeof(float), kWsAlign);
}

cudaError_t simt_fwd(const FwdProblem &p, void *ws, cudaStream_t s) {
    return p.dtype == SSD_F32 ? run<float>(p, ws, s) : run<__nv_bfloat16>(p, ws, s);
}

cudaError_t simt_cumsum(const FwdProblem &p, float *acs, float *dtw, cudaStream_t s) {
    const int H = (int)p.H, Q = (int)p.Q, nc = (int)p.nc;
    const size_t smem = (size_t)Q * 33 * sizeof(float);
    dim3 grid(nc, (H + 31) / 32, (unsigned)p.B);
    cudaError_t e;
    if (p.dtype == SSD_F32) {
        if ((e = cudaFuncSetAttribute(k_cumsum<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        k_cumsum<float><<<grid, kThreads, smem, s>>>(static_cast<const float *>(p.dt), p.A, p.L, H, Q, nc, acs, dtw);
    } else {
        if ((e = cudaFuncSetAttribute(k_cumsum<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)))
            return e;
        k_cumsum<__nv_bfloat16><<<grid, kThreads, smem, s>>>(static_cast<const __nv_bfloat16 *>(p.dt), p.A, p.L, H,
                                                             Q, nc, acs, dtw);
    }
    return cudaGetLastError();
}

cudaError_t simt_state_pass(const FwdProblem &p, const float *acs, float *states, float *h_final, cudaStream_t s) {
    const int P = (int)p.P, N = (int)p.N;
    dim3 grid((P * N + kThreads - 1) / kThreads, (unsigned)p.H, (unsigned)p.B);
    k_state_pass<<<grid, kThreads, 0, s>>>(acs, p.h0, (int)p.H, P * N, (int)p.Q, (int)p.nc, states, h_final);
    return cudaGetLastError();
}

cudaError_t simt_states(const FwdProblem &p, float *acs, float *dtw, float *states, float *h_final,
                        cudaStream_t s) {
    return p.dtype == SSD_F32 ? run_states<float>(p, acs, dtw, states, h_final, s)
                              : run_states<__nv_bfloat16>(p, acs, dtw, states, h_final, s);
}

cudaError_t simt_adjoint_chunk_sums(const FwdProblem &p, const void *dy, const float *acs, float *out,
                                    cudaStream_t s) {
    return p.dtype == SSD_F32 ? launch_chunk_state<float, true>(p, dy, p.Cm, acs, nullptr, out, s)
                              : launch_chunk_state<__nv_bfloat16, true>(p, dy, p.Cm, acs, nullptr, out, s);
}

}  // namespace ssd
