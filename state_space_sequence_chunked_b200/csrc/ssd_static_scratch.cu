// ssd_fwd_static_scratch: the forward pass for callers that cannot allocate
// device memory at all.
//
// Who needs this: code that runs where cudaMalloc is unavailable or forbidden --
// inside a fixed, pre-reserved memory budget that the application manages
// itself (an inference server that carves all of HBM up front), inside a
// real-time loop where an allocation could block or fail, or in a plugin whose
// host framework owns every allocation and only hands it input and output
// buffers. Such callers cannot provide the workspace that ssd_fwd asks for.
//
// How: the per-chunk intermediates (within-chunk decay cumsums, the step sizes
// as fp32, and the chunk states) live in one file-scope device array of fixed
// size, kStaticScratchBytes (SSD_STATIC_SCRATCH_BYTES in ssd.h). The same fp32
// CUDA-core kernels as ssd_fwd's general path run on it. Every kernel writes
// each scratch element it later reads within the same call, so nothing has to
// start at zero and no clearing pass is needed.
//
// The array is a host-side stand-in in host code; only its device address may
// be passed to a kernel. That address is looked up once per device, with that
// device current, by cudaGetSymbolAddress on the first call made on the device.
#include <mutex>

#include "ssd_internal.cuh"

#define SSD_API extern "C" __attribute__((visibility("default")))

namespace ssd {
namespace {

constexpr size_t kStaticScratchBytes = SSD_STATIC_SCRATCH_BYTES;
static_assert(kStaticScratchBytes % kWsAlign == 0, "scratch size must keep 256-byte alignment");

// Shared by every call on a device; held by every GPU that loads this module until
// the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once).
cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace ssd

using namespace ssd;

SSD_API ssd_status_t ssd_fwd_static_scratch(const ssd_shape_t *s, ssd_dtype_t dtype, const void *x,
                                            const void *dt, const float *A, const void *Bm,
                                            const void *Cm, const float *D, const float *h0,
                                            int64_t chunk, void *y, float *h_final,
                                            void *stream) {
    // Same argument rules as ssd_fwd (one shared implementation).
    FwdProblem p;
    const ssd_status_t v = make_fwd(s, dtype, chunk, &p);
    if (v != SSD_OK) return v;
    if (p.B == 0) return SSD_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p.L == 0) {
        if (!h_final) return SSD_OK;
        if (!aligned16(h_final) || (h0 && !aligned16(h0))) return SSD_ERR_ALIGNMENT;
        const size_t bytes = (size_t)(p.B * p.H * p.P * p.N) * sizeof(float);
        const cudaError_t e = h0 ? cudaMemcpyAsync(h_final, h0, bytes, cudaMemcpyDeviceToDevice, st)
                                 : cudaMemsetAsync(h_final, 0, bytes, st);
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    }
    if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {x, dt, A, Bm, Cm, D, h0, y, h_final};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    // Problems whose intermediates do not fit the built-in array are refused.
    if (simt_fwd_workspace_bytes(p) > kStaticScratchBytes) return SSD_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return SSD_ERR_CUDA;
    p.x = x;
    p.dt = dt;
    p.A = A;
    p.Bm = Bm;
    p.Cm = Cm;
    p.D = D;
    p.h0 = h0;
    p.y = y;
    p.h_final = h_final;
    return simt_fwd(p, scratch, st) == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
