// The Mamba-2 block around the SSD layer: the operations between the input projection and
// ssd_fwd, and between ssd_fwd and the output projection. Both kernels are HBM-bound
// elementwise/row passes; the projections themselves are plain GEMMs left to cuBLAS.
//
//   k_conv_split     the input projection's row holds [z | x B C | dt_raw]. The x, B, C channels
//                    pass through a causal depthwise convolution (kernel width W <= 4) and SiLU
//                    ("A Visual Guide to Mamba and SSMs", "The Mamba Block": a convolution
//                    before the selective SSM so that tokens are not computed independently),
//                    and are written in the layouts ssd_fwd takes. dt = softplus(dt_raw + bias)
//                    (a positive step size; the pages only say that the step size is learned).
//   k_gated_rmsnorm  out = w * RMSNorm over groups of (y * silu(z)) (the SSD write-up,
//                    "张量并行": a grouped norm whose groups split with the tensor-parallel
//                    degree, so each GPU normalises on its own).
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kConvTok = 64;   // tokens per CTA of k_conv_split
constexpr int kConvThr = 256;  // channel pairs per CTA
constexpr int kMaxW = 4;

__device__ __forceinline__ float silu(float v) { return v / (1.f + __expf(-v)); }
__device__ __forceinline__ float softplus(float v) { return v > 20.f ? v : log1pf(__expf(v)); }

template <typename T>
struct Pair;
template <>
struct Pair<__nv_bfloat16> {
    typedef __nv_bfloat162 type;
    static __device__ __forceinline__ float2 load(const __nv_bfloat16 *p) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float a, float b) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
    }
};
template <>
struct Pair<float> {
    static __device__ __forceinline__ float2 load(const float *p) { return *reinterpret_cast<const float2 *>(p); }
    static __device__ __forceinline__ void store(float *p, float a, float b) {
        *reinterpret_cast<float2 *>(p) = make_float2(a, b);
    }
};

// grid (ceil(L / 64), ceil((Cc / 2 + H) / 256), B). Thread = a pair of conv channels (or one
// head's dt), walking 64 tokens with the last W - 1 inputs in registers.
template <typename T>
__global__ void __launch_bounds__(kConvThr)
    k_conv_split(const T *__restrict__ xbc, int64_t xbc_stride, const T *__restrict__ dt_raw, int64_t dt_stride,
                 const float *__restrict__ conv_w, const float *__restrict__ conv_b, int W,
                 const float *__restrict__ dt_bias, int64_t L, int H, int P, int G, int N, T *__restrict__ x,
                 T *__restrict__ Bm, T *__restrict__ Cm, T *__restrict__ dt) {
    const int HP = H * P, GN = G * N, Cc = HP + 2 * GN;
    const int item = blockIdx.y * kConvThr + threadIdx.x;
    const int b = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.x * kConvTok;
    const int64_t t1 = t0 + kConvTok < L ? t0 + kConvTok : L;
    if (item < Cc / 2) {
        const int ch = 2 * item;
        // taps right-aligned in a fixed window of kMaxW: h[k] = input t - (kMaxW - 1) + k, and
        // we[k] = w[k - (kMaxW - W)] (zero for k < kMaxW - W), so that
        // sum_k we[k] h[k] = sum_j w[j] input[t - (W - 1) + j]
        float w0[kMaxW], w1[kMaxW];
#pragma unroll
        for (int k = 0; k < kMaxW; ++k) {
            const int j = k - (kMaxW - W);
            w0[k] = j >= 0 ? conv_w[(int64_t)ch * W + j] : 0.f;
            w1[k] = j >= 0 ? conv_w[(int64_t)(ch + 1) * W + j] : 0.f;
        }
        const float b0 = conv_b ? conv_b[ch] : 0.f, b1 = conv_b ? conv_b[ch + 1] : 0.f;
        float h0[kMaxW], h1[kMaxW];
#pragma unroll
        for (int k = 0; k < kMaxW; ++k) h0[k] = h1[k] = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxW - 1; ++k) {  // inputs before t0 (zeros before the sequence)
            const int64_t tt = t0 - (kMaxW - 1) + k;
            if (tt >= 0) {
                const float2 v = Pair<T>::load(xbc + ((int64_t)b * L + tt) * xbc_stride + ch);
                h0[k] = v.x;
                h1[k] = v.y;
            }
        }
        T *dst;
        int64_t dstride;
        int col;
        if (ch < HP) {
            dst = x, dstride = HP, col = ch;
        } else if (ch < HP + GN) {
            dst = Bm, dstride = GN, col = ch - HP;
        } else {
            dst = Cm, dstride = GN, col = ch - HP - GN;
        }
        for (int64_t t = t0; t < t1; ++t) {
            const float2 v = Pair<T>::load(xbc + ((int64_t)b * L + t) * xbc_stride + ch);
            h0[kMaxW - 1] = v.x;
            h1[kMaxW - 1] = v.y;
            float a0 = b0, a1 = b1;
#pragma unroll
            for (int k = 0; k < kMaxW; ++k) {
                a0 = fmaf(w0[k], h0[k], a0);
                a1 = fmaf(w1[k], h1[k], a1);
            }
            Pair<T>::store(dst + ((int64_t)b * L + t) * dstride + col, silu(a0), silu(a1));
#pragma unroll
            for (int k = 0; k < kMaxW - 1; ++k) {
                h0[k] = h0[k + 1];
                h1[k] = h1[k + 1];
            }
        }
    } else if (item < Cc / 2 + H) {
        const int h = item - Cc / 2;
        const float bias = dt_bias ? dt_bias[h] : 0.f;
        for (int64_t t = t0; t < t1; ++t)
            store_as(dt + ((int64_t)b * L + t) * H + h,
                     softplus(to_f32(dt_raw[((int64_t)b * L + t) * dt_stride + h]) + bias));
    }
}

// grid (rows), 256 threads. A row of `dim` elements in `ngroups` groups of dim / ngroups
// (a multiple of 64): g = y * silu(z), out = w * g / sqrt(mean over the group of g^2 + eps).
constexpr int kNormThr = 256;
constexpr int kNormMaxPer = 32;  // elements per thread: dim <= 256 * 32

template <typename T>
__global__ void __launch_bounds__(kNormThr)
    k_gated_rmsnorm(const T *__restrict__ y, const T *__restrict__ z, int64_t z_stride, const float *__restrict__ w,
                    int dim, int ngroups, float eps, T *__restrict__ out) {
    __shared__ float gsum[64];
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int gs = dim / ngroups;
    for (int i = tid; i < ngroups; i += kNormThr) gsum[i] = 0.f;
    __syncthreads();
    const T *yr = y + row * dim;
    const T *zr = z + row * z_stride;
    float g[kNormMaxPer];
#pragma unroll
    for (int k = 0; k < kNormMaxPer / 2; ++k) {
        const int i = 2 * tid + k * 2 * kNormThr;  // a warp covers 64 consecutive elements
        float s = 0.f;
        if (i < dim) {
            const float2 yv = Pair<T>::load(yr + i), zv = Pair<T>::load(zr + i);
            g[2 * k] = yv.x * silu(zv.x);
            g[2 * k + 1] = yv.y * silu(zv.y);
            s = g[2 * k] * g[2 * k] + g[2 * k + 1] * g[2 * k + 1];
        }
        if (k * 2 * kNormThr < dim) {  // warp-uniform: the whole warp's 64 elements share a group
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const int i0 = (tid & ~31) * 2 + k * 2 * kNormThr;
            if (lane == 0 && i0 < dim) atomicAdd(&gsum[i0 / gs], s);
        }
    }
    __syncthreads();
    T *orow = out + row * dim;
#pragma unroll
    for (int k = 0; k < kNormMaxPer / 2; ++k) {
        const int i = 2 * tid + k * 2 * kNormThr;
        if (i < dim) {
            const float r = rsqrtf(gsum[i / gs] / (float)gs + eps);
            const float2 wv = *reinterpret_cast<const float2 *>(w + i);
            Pair<T>::store(orow + i, g[2 * k] * r * wv.x, g[2 * k + 1] * r * wv.y);
        }
    }
}

}  // namespace

cudaError_t conv_split_launch(const BlockShape &s, ssd_dtype_t dtype, const void *xbc, int64_t xbc_stride,
                              const void *dt_raw, int64_t dt_stride, const float *conv_w, const float *conv_b,
                              int width, const float *dt_bias, void *x, void *Bm, void *Cm, void *dt,
                              cudaStream_t st) {
    const int Cc = (int)(s.H * s.P + 2 * s.G * s.N);
    dim3 grid((unsigned)((s.L + kConvTok - 1) / kConvTok), (unsigned)((Cc / 2 + s.H + kConvThr - 1) / kConvThr),
              (unsigned)s.B);
    if (dtype == SSD_F32)
        k_conv_split<float><<<grid, kConvThr, 0, st>>>(
            static_cast<const float *>(xbc), xbc_stride, static_cast<const float *>(dt_raw), dt_stride, conv_w, conv_b,
            width, dt_bias, s.L, (int)s.H, (int)s.P, (int)s.G, (int)s.N, static_cast<float *>(x),
            static_cast<float *>(Bm), static_cast<float *>(Cm), static_cast<float *>(dt));
    else
        k_conv_split<__nv_bfloat16><<<grid, kConvThr, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(xbc), xbc_stride, static_cast<const __nv_bfloat16 *>(dt_raw), dt_stride,
            conv_w, conv_b, width, dt_bias, s.L, (int)s.H, (int)s.P, (int)s.G, (int)s.N,
            static_cast<__nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(Bm), static_cast<__nv_bfloat16 *>(Cm),
            static_cast<__nv_bfloat16 *>(dt));
    return cudaGetLastError();
}

int gated_rmsnorm_max_dim() { return kNormThr * kNormMaxPer; }

cudaError_t gated_rmsnorm_launch(int64_t rows, int dim, int ngroups, ssd_dtype_t dtype, const void *y, const void *z,
                                 int64_t z_stride, const float *w, float eps, void *out, cudaStream_t st) {
    if (dtype == SSD_F32)
        k_gated_rmsnorm<float><<<(unsigned)rows, kNormThr, 0, st>>>(static_cast<const float *>(y),
                                                                   static_cast<const float *>(z), z_stride, w, dim,
                                                                   ngroups, eps, static_cast<float *>(out));
    else
        k_gated_rmsnorm<__nv_bfloat16><<<(unsigned)rows, kNormThr, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(z), z_stride, w, dim, ngroups,
            eps, static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError();
}

}  // namespace ssd
