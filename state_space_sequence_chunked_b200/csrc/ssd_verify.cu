// Speculative-decoding verify and state selection.
//
// Verify runs K draft tokens of the recurrence from a saved state and writes the
// state after every token (the Llama-to-Mamba distillation write-up, "推测解码":
// the target model checks a run of draft tokens in one pass, and the state kept
// is the one at the position where the check stops). With K small the chunked
// form has nothing to amortise, so each state row is advanced token by token in
// registers; the cost is the K state writes, a pure HBM stream.
//
// The same write-up notes that storing every intermediate state is what a
// hardware-aware verify should avoid. Two kernels serve that flow without states_out:
// verify with states_out = NULL writes only y (k_verify_y: the chunked form over the K tokens,
// without the per-token state chain), and k_advance recomputes, once the
// accepted counts are known, the state after accepted[b] tokens straight from h0
// (K small steps per state row in registers: one read of h0 and one write of the
// kept state). It applies the same fp32 operations in the same order as k_verify,
// so its result is bit-identical to the verify state it replaces. k_decode is the
// one-token step of generation, updating the state in place.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kVThreads = 256;
constexpr int kMaxVec = 2;  // float4 vectors per lane per state row: N <= 256

// Sums of 8 values across the 32 lanes of a warp at once: the halves are exchanged and
// added (xor 16, 8, 4: 4 + 2 + 1 shuffles) so that lane l ends with value (l >> 2) & 7
// summed over 8 lanes, then the 4 lanes of each group finish with xor 2 and xor 1. Each
// value is summed over the same pairs, in the same order, as the full butterfly
// (xor 16, 8, 4, 2, 1) on that value alone.
__device__ __forceinline__ float reduce8(const float (&v)[8], int lane) {
    const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
    float a[4], c[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = h16 ? v[i] : v[i + 4], keep = h16 ? v[i + 4] : v[i];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = h8 ? a[i] : a[i + 2], keep = h8 ? a[i + 2] : a[i];
        c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float r = (h4 ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, h4 ? c[0] : c[1], 4);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    return r;
}

// grid (H, B). Warp w advances rows p = w, w + 8, ...; lane owns float4 vectors
// v = lane + 32 j of the row. Shared memory: B, C (K x N), x (K x P), dt, decay (K).
template <typename T>
__global__ void __launch_bounds__(kVThreads)
    k_verify(const float *__restrict__ h0, const T *__restrict__ x, const T *__restrict__ dt,
             const float *__restrict__ A, const T *__restrict__ Bm, const T *__restrict__ Cm,
             const float *__restrict__ D, int K, int H, int P, int G, int N,
             float *__restrict__ states_out, T *__restrict__ y) {
    extern __shared__ float sm[];
    float *bsm = sm;            // [K][N]
    float *csm = bsm + K * N;   // [K][N]
    float *xsm = csm + K * N;   // [K][P]
    float *dts = xsm + K * P;   // [K]
    float *dec = dts + K;       // [K]
    const int h = blockIdx.x, b = blockIdx.y, g = h / (H / G);
    const int tid = threadIdx.x;
    for (int i = tid; i < K * N; i += blockDim.x) {
        const int k = i / N, n = i % N;
        const int64_t off = (((int64_t)b * K + k) * G + g) * N + n;
        bsm[i] = to_f32(Bm[off]);
        csm[i] = to_f32(Cm[off]);
    }
    for (int i = tid; i < K * P; i += blockDim.x) {
        const int k = i / P, p = i % P;
        xsm[i] = to_f32(x[(((int64_t)b * K + k) * H + h) * P + p]);
    }
    for (int k = tid; k < K; k += blockDim.x) {
        const float d = to_f32(dt[((int64_t)b * K + k) * H + h]);
        dts[k] = d;
        dec[k] = expf(d * A[h]);
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    const int nv = N / 4;
    const float Dh = D ? D[h] : 0.f;
    for (int p = warp; p < P; p += kVThreads / 32) {
        float4 s[kMaxVec];
        const float4 *src = reinterpret_cast<const float4 *>(h0 + (((int64_t)b * H + h) * P + p) * N);
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            s[j] = v < nv ? src[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // Tokens in groups of 8: each token's dot product with C is kept as per-lane partials
        // and the 8 of a group are reduced together (reduce8), so the sequential chain per
        // token is the state update alone.
        for (int k0 = 0; k0 < K; k0 += 8) {
            float part[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int k = k0 + kk;
                part[kk] = 0.f;
                if (k >= K) continue;  // warp-uniform
                const float dk = dec[k];
                const float dx = dts[k] * xsm[k * P + p];
                const float4 *bk = reinterpret_cast<const float4 *>(bsm + k * N);
                const float4 *ck = reinterpret_cast<const float4 *>(csm + k * N);
                float4 *dst = states_out ? reinterpret_cast<float4 *>(states_out + ((((int64_t)b * K + k) * H + h) * P + p) * N)
                                         : nullptr;
#pragma unroll
                for (int j = 0; j < kMaxVec; ++j) {
                    const int v = lane + 32 * j;
                    if (v < nv) {
                        const float4 bb = bk[v], cc = ck[v];
                        s[j].x = fmaf(dk, s[j].x, dx * bb.x);
                        s[j].y = fmaf(dk, s[j].y, dx * bb.y);
                        s[j].z = fmaf(dk, s[j].z, dx * bb.z);
                        s[j].w = fmaf(dk, s[j].w, dx * bb.w);
                        part[kk] = fmaf(s[j].x, cc.x, part[kk]);
                        part[kk] = fmaf(s[j].y, cc.y, part[kk]);
                        part[kk] = fmaf(s[j].z, cc.z, part[kk]);
                        part[kk] = fmaf(s[j].w, cc.w, part[kk]);
                        if (states_out) __stcs(dst + v, s[j]);
                    }
                }
            }
            const float tot = reduce8(part, lane);
            const int k = k0 + (lane >> 2);
            if ((lane & 3) == 0 && k < K) store_as(y + (((int64_t)b * K + k) * H + h) * P + p, tot + Dh * xsm[k * P + p]);
        }
    }
}

// grid (H, B). Verify with outputs only: no state is written, so the K-token chunked form of the
// same recurrence (the quadratic "SSD 层的对偶注意力" form within a chunk of K tokens, plus the
// initial state decayed to each token) replaces the per-token state chain:
//     y_k = exp(cum_k) (C_k . h0[p, :]) + sum_{s <= k} M[k, s] x_s[p] + D_h x_k[p],
//     M[k, s] = (C_k . B_s) exp(cum_k - cum_s) dt_s,   cum_k = sum_{j <= k} dt_j A_h.
// Each state row is read once and its K dot products with C are independent. M (K x K) is
// formed once per CTA. Shared memory: B, C (K x N), x (K x P), cum, dt (K), M (K x K).
template <typename T>
__global__ void __launch_bounds__(kVThreads)
    k_verify_y(const float *__restrict__ h0, const T *__restrict__ x, const T *__restrict__ dt,
               const float *__restrict__ A, const T *__restrict__ Bm, const T *__restrict__ Cm,
               const float *__restrict__ D, int K, int H, int P, int G, int N, T *__restrict__ y) {
    extern __shared__ float sm[];
    float *bsm = sm;            // [K][N]
    float *csm = bsm + K * N;   // [K][N]
    float *xsm = csm + K * N;   // [K][P]
    float *dts = xsm + K * P;   // [K]
    float *cum = dts + K;       // [K]
    float *msm = cum + K;       // [K][K]
    const int h = blockIdx.x, b = blockIdx.y, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < K * N; i += blockDim.x) {
        const int k = i / N, n = i % N;
        const int64_t off = (((int64_t)b * K + k) * G + g) * N + n;
        bsm[i] = to_f32(Bm[off]);
        csm[i] = to_f32(Cm[off]);
    }
    for (int i = tid; i < K * P; i += blockDim.x) {
        const int k = i / P, p = i % P;
        xsm[i] = to_f32(x[(((int64_t)b * K + k) * H + h) * P + p]);
    }
    if (warp == 0) {  // dt and the inclusive cumsum of dt A (K <= 64: two tokens per lane)
        float d[2], a[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int k = 2 * lane + m;
            d[m] = k < K ? to_f32(dt[((int64_t)b * K + k) * H + h]) : 0.f;
            a[m] = d[m] * A[h];
        }
        a[1] += a[0];
        float incl = a[1];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        const float excl = incl - a[1];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int k = 2 * lane + m;
            if (k < K) {
                dts[k] = d[m];
                cum[k] = excl + a[m];
            }
        }
    }
    __syncthreads();
    // M[k, s] for s <= k (zero above the diagonal): one warp per entry, lanes over n
    for (int e = warp; e < K * K; e += kVThreads / 32) {
        const int k = e / K, s2 = e % K;
        float v = 0.f;
        if (s2 <= k) {
            for (int n = lane; n < N; n += 32) v = fmaf(csm[k * N + n], bsm[s2 * N + n], v);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            v *= expf(cum[k] - cum[s2]) * dts[s2];
        }
        if (lane == 0) msm[e] = v;
    }
    __syncthreads();
    const int nv = N / 4;
    const float Dh = D ? D[h] : 0.f;
    for (int p = warp; p < P; p += kVThreads / 32) {
        float4 s[kMaxVec];
        const float4 *src = reinterpret_cast<const float4 *>(h0 + (((int64_t)b * H + h) * P + p) * N);
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            s[j] = v < nv ? src[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int k0 = 0; k0 < K; k0 += 8) {
            float part[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int k = k0 + kk;
                part[kk] = 0.f;
                if (k >= K) continue;  // warp-uniform
                const float4 *ck = reinterpret_cast<const float4 *>(csm + k * N);
#pragma unroll
                for (int j = 0; j < kMaxVec; ++j) {
                    const int v = lane + 32 * j;
                    if (v < nv) {
                        const float4 cc = ck[v];
                        part[kk] = fmaf(s[j].x, cc.x, part[kk]);
                        part[kk] = fmaf(s[j].y, cc.y, part[kk]);
                        part[kk] = fmaf(s[j].z, cc.z, part[kk]);
                        part[kk] = fmaf(s[j].w, cc.w, part[kk]);
                    }
                }
            }
            const float tot = reduce8(part, lane);
            const int k = k0 + (lane >> 2);
            if ((lane & 3) == 0 && k < K) {
                float acc = expf(cum[k]) * tot;
                for (int s2 = 0; s2 <= k; ++s2) acc = fmaf(msm[k * K + s2], xsm[s2 * P + p], acc);
                store_as(y + (((int64_t)b * K + k) * H + h) * P + p, acc + Dh * xsm[k * P + p]);
            }
        }
    }
}

// grid (H, B). The state after accepted[b] draft tokens, from h0: the update of
// k_verify without the outputs. Shared memory: B (K x N), x (K x P), dt, decay (K).
// A row whose count is outside 0..K is filled with quiet NaN.
template <typename T>
__global__ void __launch_bounds__(kVThreads)
    k_advance(const float *h0, const T *__restrict__ x, const T *__restrict__ dt, const float *__restrict__ A,
              const T *__restrict__ Bm, const int32_t *__restrict__ accepted, int K, int H, int P, int G, int N,
              float *h_keep) {  // h_keep may be h0 (in place): each row is read before it is written, by one warp
    extern __shared__ float sm[];
    const int h = blockIdx.x, b = blockIdx.y, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nv = N / 4;
    const int a = accepted[b];
    if (a < 0 || a > K) {
        const float qn = __int_as_float(0x7fc00000);
        float4 *dst = reinterpret_cast<float4 *>(h_keep + ((int64_t)b * H + h) * P * N);
        for (int i = tid; i < P * nv; i += blockDim.x) dst[i] = make_float4(qn, qn, qn, qn);
        return;
    }
    float *bsm = sm;            // [a][N]
    float *xsm = bsm + a * N;   // [a][P]
    float *dts = xsm + a * P;   // [a]
    float *dec = dts + a;       // [a]
    for (int i = tid; i < a * N; i += blockDim.x) {
        const int k = i / N, n = i % N;
        bsm[i] = to_f32(Bm[(((int64_t)b * K + k) * G + g) * N + n]);
    }
    for (int i = tid; i < a * P; i += blockDim.x) {
        const int k = i / P, q = i % P;
        xsm[i] = to_f32(x[(((int64_t)b * K + k) * H + h) * P + q]);
    }
    for (int k = tid; k < a; k += blockDim.x) {
        const float d = to_f32(dt[((int64_t)b * K + k) * H + h]);
        dts[k] = d;
        dec[k] = expf(d * A[h]);
    }
    __syncthreads();
    for (int p = warp; p < P; p += kVThreads / 32) {
        const float4 *src = reinterpret_cast<const float4 *>(h0 + (((int64_t)b * H + h) * P + p) * N);
        float4 *dst = reinterpret_cast<float4 *>(h_keep + (((int64_t)b * H + h) * P + p) * N);
        float4 s[kMaxVec];
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            s[j] = v < nv ? src[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int k = 0; k < a; ++k) {
            const float dk = dec[k];
            const float dx = dts[k] * xsm[k * P + p];
            const float4 *bk = reinterpret_cast<const float4 *>(bsm + k * N);
#pragma unroll
            for (int j = 0; j < kMaxVec; ++j) {
                const int v = lane + 32 * j;
                if (v < nv) {
                    const float4 bb = bk[v];
                    s[j].x = fmaf(dk, s[j].x, dx * bb.x);
                    s[j].y = fmaf(dk, s[j].y, dx * bb.y);
                    s[j].z = fmaf(dk, s[j].z, dx * bb.z);
                    s[j].w = fmaf(dk, s[j].w, dx * bb.w);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            if (v < nv) __stcs(dst + v, s[j]);
        }
    }
}

// grid (H, B). One token of generation, in place: state <- exp(dt A) state + dt x B^T,
// y = state C + D x. Each state row is read whole into registers before it is
// written back, and only its own warp touches it, so reading and writing the same
// buffer is safe (which is why `state` carries no __restrict__).
template <typename T>
__global__ void __launch_bounds__(kVThreads)
    k_decode(float *state, const T *__restrict__ x, const T *__restrict__ dt, const float *__restrict__ A,
             const T *__restrict__ Bm, const T *__restrict__ Cm, const float *__restrict__ D, int H, int P,
             int G, int N, T *__restrict__ y) {
    extern __shared__ float sm[];
    float *bsm = sm;        // [N]
    float *csm = bsm + N;   // [N]
    const int h = blockIdx.x, b = blockIdx.y, g = h / (H / G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int n = tid; n < N; n += blockDim.x) {
        const int64_t off = ((int64_t)b * G + g) * N + n;
        bsm[n] = to_f32(Bm[off]);
        csm[n] = to_f32(Cm[off]);
    }
    __syncthreads();
    const float d = to_f32(dt[(int64_t)b * H + h]);
    const float dk = expf(d * A[h]);
    const float Dh = D ? D[h] : 0.f;
    const int nv = N / 4;
    for (int p = warp; p < P; p += kVThreads / 32) {
        float4 *row = reinterpret_cast<float4 *>(state + (((int64_t)b * H + h) * P + p) * N);
        const float xk = to_f32(x[((int64_t)b * H + h) * P + p]);
        const float dx = d * xk;
        float4 s[kMaxVec];
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            s[j] = v < nv ? row[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            if (v < nv) {
                const float4 bb = reinterpret_cast<const float4 *>(bsm)[v];
                const float4 cc = reinterpret_cast<const float4 *>(csm)[v];
                s[j].x = fmaf(dk, s[j].x, dx * bb.x);
                s[j].y = fmaf(dk, s[j].y, dx * bb.y);
                s[j].z = fmaf(dk, s[j].z, dx * bb.z);
                s[j].w = fmaf(dk, s[j].w, dx * bb.w);
                part = fmaf(s[j].x, cc.x, part);
                part = fmaf(s[j].y, cc.y, part);
                part = fmaf(s[j].z, cc.z, part);
                part = fmaf(s[j].w, cc.w, part);
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = lane + 32 * j;
            if (v < nv) row[v] = s[j];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) store_as(y + ((int64_t)b * H + h) * P + p, part + Dh * xk);
    }
}

// grid (ceil(per_row / 4 / 256), B)
__global__ void k_select(const float *__restrict__ h0, const float *__restrict__ so,
                         const int32_t *__restrict__ accepted, int K, int64_t per_row,
                         float *__restrict__ out) {
    const int b = blockIdx.y;
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nv = per_row / 4;
    if (v >= nv) return;
    const int a = accepted[b];
    float4 *dst = reinterpret_cast<float4 *>(out + (int64_t)b * per_row);
    if (a < 0 || a > K) {
        const float qn = __int_as_float(0x7fc00000);
        dst[v] = make_float4(qn, qn, qn, qn);
        return;
    }
    const float *src = a == 0 ? h0 + (int64_t)b * per_row : so + ((int64_t)b * K + (a - 1)) * per_row;
    dst[v] = reinterpret_cast<const float4 *>(src)[v];
}

}  // namespace

cudaError_t verify_launch(const VerifyProblem &p, cudaStream_t s) {
    const int K = (int)p.K, H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N;
    if (!p.states_out) {  // outputs only: the chunked form, no state chain
        const size_t smem = (size_t)(2 * K * N + K * P + 2 * K + K * K) * sizeof(float);
        dim3 grid(H, (unsigned)p.B);
        cudaError_t e;
        if (p.dtype == SSD_F32) {
            if ((e = cudaFuncSetAttribute(k_verify_y<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
                return e;
            k_verify_y<float><<<grid, kVThreads, smem, s>>>(p.h0, (const float *)p.x, (const float *)p.dt, p.A,
                                                            (const float *)p.Bm, (const float *)p.Cm, p.D, K, H, P, G,
                                                            N, (float *)p.y);
        } else {
            using bf = __nv_bfloat16;
            if ((e = cudaFuncSetAttribute(k_verify_y<bf>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
                return e;
            k_verify_y<bf><<<grid, kVThreads, smem, s>>>(p.h0, (const bf *)p.x, (const bf *)p.dt, p.A, (const bf *)p.Bm,
                                                         (const bf *)p.Cm, p.D, K, H, P, G, N, (bf *)p.y);
        }
        return cudaGetLastError();
    }
    const size_t smem = (size_t)(2 * K * N + K * P + 2 * K) * sizeof(float);
    cudaError_t e;
    dim3 grid(H, (unsigned)p.B);
    if (p.dtype == SSD_F32) {
        if ((e = cudaFuncSetAttribute(k_verify<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        k_verify<float><<<grid, kVThreads, smem, s>>>(p.h0, (const float *)p.x, (const float *)p.dt, p.A,
                                                      (const float *)p.Bm, (const float *)p.Cm, p.D, K, H, P,
                                                      G, N, p.states_out, (float *)p.y);
    } else {
        using bf = __nv_bfloat16;
        if ((e = cudaFuncSetAttribute(k_verify<bf>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        k_verify<bf><<<grid, kVThreads, smem, s>>>(p.h0, (const bf *)p.x, (const bf *)p.dt, p.A,
                                                   (const bf *)p.Bm, (const bf *)p.Cm, p.D, K, H, P, G, N,
                                                   p.states_out, (bf *)p.y);
    }
    return cudaGetLastError();
}

cudaError_t advance_launch(const VerifyProblem &p, const int32_t *accepted, float *h_keep, cudaStream_t s) {
    const int K = (int)p.K, H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N;
    const size_t smem = (size_t)(K * N + K * P + 2 * K) * sizeof(float);  // room for a = K
    dim3 grid(H, (unsigned)p.B);
    cudaError_t e;
    if (p.dtype == SSD_F32) {
        if ((e = cudaFuncSetAttribute(k_advance<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        k_advance<float><<<grid, kVThreads, smem, s>>>(p.h0, (const float *)p.x, (const float *)p.dt, p.A,
                                                       (const float *)p.Bm, accepted, K, H, P, G, N, h_keep);
    } else {
        using bf = __nv_bfloat16;
        if ((e = cudaFuncSetAttribute(k_advance<bf>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        k_advance<bf><<<grid, kVThreads, smem, s>>>(p.h0, (const bf *)p.x, (const bf *)p.dt, p.A, (const bf *)p.Bm,
                                                    accepted, K, H, P, G, N, h_keep);
    }
    return cudaGetLastError();
}

cudaError_t decode_launch(const VerifyProblem &p, float *state, cudaStream_t s) {
    const int H = (int)p.H, P = (int)p.P, G = (int)p.G, N = (int)p.N;
    const size_t smem = (size_t)(2 * N) * sizeof(float);
    dim3 grid(H, (unsigned)p.B);
    if (p.dtype == SSD_F32) {
        k_decode<float><<<grid, kVThreads, smem, s>>>(state, (const float *)p.x, (const float *)p.dt, p.A,
                                                      (const float *)p.Bm, (const float *)p.Cm, p.D, H, P, G, N,
                                                      (float *)p.y);
    } else {
        using bf = __nv_bfloat16;
        k_decode<bf><<<grid, kVThreads, smem, s>>>(state, (const bf *)p.x, (const bf *)p.dt, p.A, (const bf *)p.Bm,
                                                   (const bf *)p.Cm, p.D, H, P, G, N, (bf *)p.y);
    }
    return cudaGetLastError();
}

cudaError_t select_launch(int64_t B, int64_t K, int64_t per_row, const float *h0,
                          const float *states_out, const int32_t *accepted, float *h_keep,
                          cudaStream_t s) {
    const int64_t nv = per_row / 4;
    dim3 grid((unsigned)((nv + 255) / 256), (unsigned)B);
    k_select<<<grid, 256, 0, s>>>(h0, states_out, accepted, (int)K, per_row, h_keep);
    return cudaGetLastError();
}

}  // namespace ssd
