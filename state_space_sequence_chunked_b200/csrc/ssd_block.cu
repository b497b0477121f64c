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

// V consecutive elements of a row as floats (V = 2 or 8; 4- or 16-byte aligned for bf16).
template <typename T, int V>
__device__ __forceinline__ void load_vec(const T *p, float (&f)[V]) {
    if constexpr (V == 8 && sizeof(T) == 2) {
        const uint4 r = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 v = __bfloat1622float2(h[i]);
            f[2 * i] = v.x;
            f[2 * i + 1] = v.y;
        }
    } else if constexpr (V == 8) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
    } else {
#pragma unroll
        for (int i = 0; i < V; i += 2) {
            const float2 v = Pair<T>::load(p + i);
            f[i] = v.x;
            f[i + 1] = v.y;
        }
    }
}
template <typename T, int V>
__device__ __forceinline__ void store_vec(T *p, const float (&f)[V]) {
    if constexpr (V == 8 && sizeof(T) == 2) {
        uint4 r;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&r);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        *reinterpret_cast<uint4 *>(p) = r;
    } else if constexpr (V == 8) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    } else {
#pragma unroll
        for (int i = 0; i < V; i += 2) Pair<T>::store(p + i, f[i], f[i + 1]);
    }
}

// grid (ceil(L / 64), ceil((Cc / V + H) / 256), B). Thread = V consecutive conv channels (or
// one head's dt), walking 64 tokens with the last kMaxW - 1 inputs in registers; the loads of
// 4 tokens are issued before their arithmetic.
template <typename T, int V>
__global__ void __launch_bounds__(kConvThr, 2)
    k_conv_split(const T *__restrict__ xbc, int64_t xbc_stride, const T *__restrict__ dt_raw, int64_t dt_stride,
                 const float *__restrict__ conv_w, const float *__restrict__ conv_b, int W,
                 const float *__restrict__ dt_bias, int64_t L, int H, int P, int G, int N, T *__restrict__ x,
                 T *__restrict__ Bm, T *__restrict__ Cm, T *__restrict__ dt) {
    const int HP = H * P, GN = G * N, Cc = HP + 2 * GN;
    const int item = blockIdx.y * kConvThr + threadIdx.x;
    const int b = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.x * kConvTok;
    const int64_t t1 = t0 + kConvTok < L ? t0 + kConvTok : L;
    if (item < Cc / V) {
        const int ch = V * item;
        // taps right-aligned in a fixed window of kMaxW: h[k] = input t - (kMaxW - 1) + k, and
        // we[k] = w[k - (kMaxW - W)] (zero for k < kMaxW - W), so that
        // sum_k we[k] h[k] = sum_j w[j] input[t - (W - 1) + j]
        float we[V][kMaxW], bias[V], h[V][kMaxW];
#pragma unroll
        for (int v = 0; v < V; ++v) {
#pragma unroll
            for (int k = 0; k < kMaxW; ++k) {
                const int j = k - (kMaxW - W);
                we[v][k] = j >= 0 ? conv_w[(int64_t)(ch + v) * W + j] : 0.f;
                h[v][k] = 0.f;
            }
            bias[v] = conv_b ? conv_b[ch + v] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kMaxW - 1; ++k) {  // inputs before t0 (zeros before the sequence)
            const int64_t tt = t0 - (kMaxW - 1) + k;
            if (tt >= 0) {
                float f[V];
                load_vec<T, V>(xbc + ((int64_t)b * L + tt) * xbc_stride + ch, f);
#pragma unroll
                for (int v = 0; v < V; ++v) h[v][k] = f[v];
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
        constexpr int U = V == 8 ? 2 : 4;
        for (int64_t tb = t0; tb < t1; tb += U) {
            float in[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (tb + u < t1) load_vec<T, V>(xbc + ((int64_t)b * L + tb + u) * xbc_stride + ch, in[u]);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (tb + u < t1) {
                    float o[V];
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        h[v][kMaxW - 1] = in[u][v];
                        float acc = bias[v];
#pragma unroll
                        for (int k = 0; k < kMaxW; ++k) acc = fmaf(we[v][k], h[v][k], acc);
                        o[v] = silu(acc);
#pragma unroll
                        for (int k = 0; k < kMaxW - 1; ++k) h[v][k] = h[v][k + 1];
                    }
                    store_vec<T, V>(dst + ((int64_t)b * L + tb + u) * dstride + col, o);
                }
            }
        }
    } else if (item < Cc / V + H) {
        const int hh = item - Cc / V;
        const float bias = dt_bias ? dt_bias[hh] : 0.f;
        for (int64_t t = t0; t < t1; ++t)
            store_as(dt + ((int64_t)b * L + t) * H + hh,
                     softplus(to_f32(dt_raw[((int64_t)b * L + t) * dt_stride + hh]) + bias));
    }
}

// grid (rows), 256 threads, V elements per thread and step, 32 / V steps (dim <= 256 * 32). A
// row of `dim` elements in `ngroups` groups of dim / ngroups (a multiple of 64):
// g = y * silu(z), out = w * g / sqrt(mean over the group of g^2 + eps). 64 / V consecutive
// lanes cover 64 channels, which lie in one group.
constexpr int kNormThr = 256;
constexpr int kNormPer = 32;

template <typename T, int V>
__global__ void __launch_bounds__(kNormThr)
    k_gated_rmsnorm(const T *__restrict__ y, const T *__restrict__ z, int64_t z_stride, const float *__restrict__ w,
                    int dim, int ngroups, float eps, T *__restrict__ out) {
    constexpr int S = kNormPer / V, SEG = 64 / V;
    __shared__ float gsum[64];
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int gs = dim / ngroups;
    for (int i = tid; i < ngroups; i += kNormThr) gsum[i] = 0.f;
    __syncthreads();
    const T *yr = y + row * dim;
    const T *zr = z + row * z_stride;
    float g[S][V];
#pragma unroll
    for (int k = 0; k < S; ++k) {
        const int i = V * tid + k * V * kNormThr;
        float s = 0.f;
        if (i < dim) {
            float yv[V], zv[V];
            load_vec<T, V>(yr + i, yv);
            load_vec<T, V>(zr + i, zv);
#pragma unroll
            for (int e = 0; e < V; ++e) {
                g[k][e] = yv[e] * silu(zv[e]);
                s = fmaf(g[k][e], g[k][e], s);
            }
        }
        if (k * V * kNormThr < dim) {  // warp-uniform
#pragma unroll
            for (int o = SEG / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if ((lane & (SEG - 1)) == 0 && i < dim) atomicAdd(&gsum[i / gs], s);
        }
    }
    __syncthreads();
    T *orow = out + row * dim;
#pragma unroll
    for (int k = 0; k < S; ++k) {
        const int i = V * tid + k * V * kNormThr;
        if (i < dim) {
            const float r = rsqrtf(gsum[i / gs] / (float)gs + eps);
            float wv[V], o[V];
            load_vec<float, V>(w + i, wv);
#pragma unroll
            for (int e = 0; e < V; ++e) o[e] = g[k][e] * r * wv[e];
            store_vec<T, V>(orow + i, o);
        }
    }
}

template <typename T, int V>
cudaError_t conv_split_typed(const BlockShape &s, const void *xbc, int64_t xbc_stride, const void *dt_raw,
                             int64_t dt_stride, const float *conv_w, const float *conv_b, int width,
                             const float *dt_bias, void *x, void *Bm, void *Cm, void *dt, cudaStream_t st) {
    const int Cc = (int)(s.H * s.P + 2 * s.G * s.N);
    dim3 grid((unsigned)((s.L + kConvTok - 1) / kConvTok), (unsigned)((Cc / V + s.H + kConvThr - 1) / kConvThr),
              (unsigned)s.B);
    k_conv_split<T, V><<<grid, kConvThr, 0, st>>>(static_cast<const T *>(xbc), xbc_stride,
                                                  static_cast<const T *>(dt_raw), dt_stride, conv_w, conv_b, width,
                                                  dt_bias, s.L, (int)s.H, (int)s.P, (int)s.G, (int)s.N,
                                                  static_cast<T *>(x), static_cast<T *>(Bm), static_cast<T *>(Cm),
                                                  static_cast<T *>(dt));
    return cudaGetLastError();
}

}  // namespace

// 8 channels per thread when the x, B, C boundaries, the row stride and the base allow 16-byte
// vectors; 2 otherwise.
cudaError_t conv_split_launch(const BlockShape &s, ssd_dtype_t dtype, const void *xbc, int64_t xbc_stride,
                              const void *dt_raw, int64_t dt_stride, const float *conv_w, const float *conv_b,
                              int width, const float *dt_bias, void *x, void *Bm, void *Cm, void *dt,
                              cudaStream_t st) {
    const size_t es = dtype == SSD_F32 ? 4 : 2;
    const bool wide = (s.H * s.P) % 8 == 0 && (s.G * s.N) % 8 == 0 && xbc_stride % 8 == 0 &&
                      (reinterpret_cast<uintptr_t>(xbc) % (8 * es)) == 0 && dtype == SSD_BF16;
    if (dtype == SSD_F32)
        return conv_split_typed<float, 2>(s, xbc, xbc_stride, dt_raw, dt_stride, conv_w, conv_b, width, dt_bias, x,
                                          Bm, Cm, dt, st);
    if (wide)
        return conv_split_typed<__nv_bfloat16, 8>(s, xbc, xbc_stride, dt_raw, dt_stride, conv_w, conv_b, width,
                                                  dt_bias, x, Bm, Cm, dt, st);
    return conv_split_typed<__nv_bfloat16, 2>(s, xbc, xbc_stride, dt_raw, dt_stride, conv_w, conv_b, width, dt_bias,
                                              x, Bm, Cm, dt, st);
}

int gated_rmsnorm_max_dim() { return kNormThr * kNormPer; }

// 8 elements per thread and step when every z row is 16-byte aligned; 2 otherwise.
cudaError_t gated_rmsnorm_launch(int64_t rows, int dim, int ngroups, ssd_dtype_t dtype, const void *y, const void *z,
                                 int64_t z_stride, const float *w, float eps, void *out, cudaStream_t st) {
    const int64_t es = dtype == SSD_F32 ? 4 : 2;
    const bool wide = (reinterpret_cast<uintptr_t>(z) % 16) == 0 && (z_stride * es) % 16 == 0;
    const unsigned grid = (unsigned)rows;
    if (dtype == SSD_F32) {
        if (wide)
            k_gated_rmsnorm<float, 8><<<grid, kNormThr, 0, st>>>(static_cast<const float *>(y),
                                                                 static_cast<const float *>(z), z_stride, w, dim,
                                                                 ngroups, eps, static_cast<float *>(out));
        else
            k_gated_rmsnorm<float, 2><<<grid, kNormThr, 0, st>>>(static_cast<const float *>(y),
                                                                 static_cast<const float *>(z), z_stride, w, dim,
                                                                 ngroups, eps, static_cast<float *>(out));
    } else {
        typedef __nv_bfloat16 bf;
        if (wide)
            k_gated_rmsnorm<bf, 8><<<grid, kNormThr, 0, st>>>(static_cast<const bf *>(y), static_cast<const bf *>(z),
                                                              z_stride, w, dim, ngroups, eps, static_cast<bf *>(out));
        else
            k_gated_rmsnorm<bf, 2><<<grid, kNormThr, 0, st>>>(static_cast<const bf *>(y), static_cast<const bf *>(z),
                                                              z_stride, w, dim, ngroups, eps, static_cast<bf *>(out));
    }
    return cudaGetLastError();
}

}  // namespace ssd
