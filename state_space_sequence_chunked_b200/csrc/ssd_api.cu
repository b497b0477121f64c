// The C ABI: argument validation, workspace sizing and path selection.
// Every check runs before any launch; on an error nothing is launched.
#include <atomic>

#include "ssd_internal.cuh"

#define SSD_API extern "C" __attribute__((visibility("default")))

namespace ssd {

static std::atomic<int> g_wait_limit_us{0};
int wait_limit_us() { return g_wait_limit_us.load(std::memory_order_relaxed); }

namespace {

constexpr int64_t kMaxVerifyK = 64;

ssd_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA; }

// Path selection: the fused tensor-core kernel where its shape constraints hold,
// the fp32 CUDA-core kernels otherwise (fp32 inputs always take the latter).
ssd_plan_t plan_of(const FwdProblem &p) {
    ssd_plan_t out{};
    if (p.B == 0 || p.L == 0) {
        out.path = SSD_PATH_NONE;
    } else if (tc_supported(p)) {
        out.path = SSD_PATH_TCGEN05;
        out.kernels = 1;
        out.workspace_bytes = tc_fwd_workspace_bytes(p);
    } else {
        out.path = SSD_PATH_SIMT;
        out.kernels = 4;
        out.workspace_bytes = simt_fwd_workspace_bytes(p);
    }
    return out;
}

}  // namespace
}  // namespace ssd

using namespace ssd;

SSD_API const char *ssd_strerror(ssd_status_t s) {
    switch (s) {
    case SSD_OK: return "success";
    case SSD_ERR_INVALID_ARG: return "invalid argument (NULL pointer, negative or inconsistent size)";
    case SSD_ERR_UNSUPPORTED: return "unsupported size (outside the supported range)";
    case SSD_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SSD_ERR_WORKSPACE: return "workspace missing or too small";
    case SSD_ERR_CUDA: return "CUDA runtime error";
    case SSD_ERR_TIMEOUT: return "bounded device-side wait timed out";
    }
    return "unknown status";
}

SSD_API ssd_status_t ssd_fwd_workspace_bytes(const ssd_shape_t *shape, ssd_dtype_t dtype,
                                             int64_t chunk, size_t *bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    FwdProblem p;
    const ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    *bytes = plan_of(p).workspace_bytes;
    return SSD_OK;
}

SSD_API ssd_status_t ssd_fwd_plan(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                                  ssd_plan_t *plan) {
    if (!plan) return SSD_ERR_INVALID_ARG;
    FwdProblem p;
    const ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    const ssd_plan_t out = plan_of(p);
    *plan = out;
    return SSD_OK;
}

SSD_API ssd_status_t ssd_fwd(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *x,
                             const void *dt, const float *A, const void *Bm, const void *Cm,
                             const float *D, const float *h0, int64_t chunk, void *y,
                             float *h_final, void *workspace, size_t workspace_bytes,
                             void *stream) {
    FwdProblem p;
    ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    if (p.B == 0) return SSD_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)(p.B * p.H * p.P * p.N) * sizeof(float);
    if (p.L == 0) {
        if (!h_final) return SSD_OK;
        if (!aligned16(h_final) || (h0 && !aligned16(h0))) return SSD_ERR_ALIGNMENT;
        return from_cuda(h0 ? cudaMemcpyAsync(h_final, h0, state_bytes, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(h_final, 0, state_bytes, s));
    }
    if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {x, dt, A, Bm, Cm, D, h0, y, h_final, workspace};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    const ssd_plan_t plan = plan_of(p);
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes))
        return SSD_ERR_WORKSPACE;
    p.x = x;
    p.dt = dt;
    p.A = A;
    p.Bm = Bm;
    p.Cm = Cm;
    p.D = D;
    p.h0 = h0;
    p.y = y;
    p.h_final = h_final;
    return from_cuda(plan.path == SSD_PATH_TCGEN05 ? tc_fwd(p, workspace, s) : simt_fwd(p, workspace, s));
}

SSD_API ssd_status_t ssd_fwd_status(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                                    const void *workspace, void *stream) {
    FwdProblem p;
    ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSD_ERR_CUDA;
    if (plan_of(p).path != SSD_PATH_TCGEN05) return SSD_OK;  // the other paths have no waits
    if (!workspace) return SSD_ERR_INVALID_ARG;
    int32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    if (word & 1) return SSD_ERR_TIMEOUT;
    return word ? SSD_ERR_CUDA : SSD_OK;
}

SSD_API ssd_status_t ssd_set_wait_limit_us(int32_t us) {
    if (us < 0 || us > 2000000) return SSD_ERR_INVALID_ARG;
    g_wait_limit_us.store(us, std::memory_order_relaxed);
    return SSD_OK;
}

SSD_API ssd_status_t ssd_verify(const ssd_shape_t *shape, ssd_dtype_t dtype, const float *h0,
                                const void *x, const void *dt, const float *A, const void *Bm,
                                const void *Cm, const float *D, int64_t K, float *states_out,
                                void *y, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    if (K < 1 || shape->seqlen != K) return SSD_ERR_INVALID_ARG;
    if (K > kMaxVerifyK || shape->dstate % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (shape->batch == 0) return SSD_OK;
    if (!h0 || !x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;  // states_out optional
    const void *ptrs[] = {h0, x, dt, A, Bm, Cm, D, states_out, y};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    VerifyProblem p{shape->batch, K, shape->nheads, shape->headdim, shape->ngroups, shape->dstate,
                    dtype, h0, x, dt, Bm, Cm, A, D, states_out, y};
    return from_cuda(verify_launch(p, static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_select_state(const ssd_shape_t *shape, int64_t K, const float *h0,
                                      const float *states_out, const int32_t *accepted,
                                      float *h_keep, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (K < 1) return SSD_ERR_INVALID_ARG;
    if (K > kMaxVerifyK || shape->dstate % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (shape->batch == 0) return SSD_OK;
    if (!h0 || !states_out || !accepted || !h_keep) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {h0, states_out, accepted, h_keep};
    for (const void *q : ptrs)
        if (!aligned16(q)) return SSD_ERR_ALIGNMENT;
    const int64_t per_row = shape->nheads * shape->headdim * shape->dstate;
    return from_cuda(select_launch(shape->batch, K, per_row, h0, states_out, accepted, h_keep,
                                   static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_advance_state(const ssd_shape_t *shape, ssd_dtype_t dtype, const float *h0,
                                       const void *x, const void *dt, const float *A, const void *Bm,
                                       int64_t K, const int32_t *accepted, float *h_keep, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    if (K < 1 || shape->seqlen != K) return SSD_ERR_INVALID_ARG;
    if (K > kMaxVerifyK || shape->dstate % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (shape->batch == 0) return SSD_OK;
    if (!h0 || !x || !dt || !A || !Bm || !accepted || !h_keep) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {h0, x, dt, A, Bm, accepted, h_keep};
    for (const void *q : ptrs)
        if (!aligned16(q)) return SSD_ERR_ALIGNMENT;
    // h_keep may be h0 itself (in place); any other overlap is not allowed.
    const size_t state_bytes = (size_t)(shape->batch * shape->nheads * shape->headdim * shape->dstate) * sizeof(float);
    const char *a0 = reinterpret_cast<const char *>(h0), *k0 = reinterpret_cast<const char *>(h_keep);
    if (a0 != k0 && a0 < k0 + state_bytes && k0 < a0 + state_bytes) return SSD_ERR_INVALID_ARG;
    VerifyProblem p{shape->batch, K, shape->nheads, shape->headdim, shape->ngroups, shape->dstate,
                    dtype, h0, x, dt, Bm, nullptr, A, nullptr, nullptr, nullptr};
    return from_cuda(advance_launch(p, accepted, h_keep, static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_decode_step(const ssd_shape_t *shape, ssd_dtype_t dtype, float *state,
                                     const void *x, const void *dt, const float *A, const void *Bm,
                                     const void *Cm, const float *D, void *y, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    if (shape->seqlen != 1) return SSD_ERR_INVALID_ARG;
    if (shape->dstate % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (shape->batch == 0) return SSD_OK;
    if (!state || !x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {state, x, dt, A, Bm, Cm, D, y};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    VerifyProblem p{shape->batch, 1, shape->nheads, shape->headdim, shape->ngroups, shape->dstate,
                    dtype, nullptr, x, dt, Bm, Cm, A, D, nullptr, y};
    return from_cuda(decode_launch(p, state, static_cast<cudaStream_t>(stream)));
}

// ---- context parallelism ------------------------------------------------------------

namespace {
ssd::CpProblem make_cp(const ssd_shape_t *s, ssd_dtype_t dtype) {
    return ssd::CpProblem{s->batch, s->seqlen, s->nheads, s->headdim, s->ngroups, s->dstate, dtype};
}
}  // namespace

SSD_API ssd_status_t ssd_cp_decay(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *dt, const float *A,
                                  float *block_decay, float *total, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    if (shape->batch == 0) return SSD_OK;
    if (!A || !total || (shape->seqlen > 0 && (!dt || !block_decay))) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {dt, A, block_decay, total};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    return from_cuda(cp_block_decay_launch(make_cp(shape, dtype), dt, A, block_decay, total,
                                           static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_cp_combine(const ssd_shape_t *shape, int64_t nranks, int64_t rank, const float *states,
                                    const float *totals, float *s_in, float *h_final, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (nranks < 1 || rank < 0 || rank >= nranks) return SSD_ERR_INVALID_ARG;
    if (nranks > 65536) return SSD_ERR_UNSUPPORTED;
    if ((shape->headdim * shape->dstate) % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (shape->batch == 0) return SSD_OK;
    if (!states || !totals || !s_in) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {states, totals, s_in, h_final};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    return from_cuda(cp_combine_launch(make_cp(shape, SSD_F32), (int)nranks, (int)rank, states, totals, s_in,
                                       h_final, static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_cp_correct(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *dt, const float *A,
                                    const void *Cm, const float *block_decay, const float *s_in, void *y,
                                    int32_t *status, void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    if (shape->batch == 0 || shape->seqlen == 0) return SSD_OK;
    if (!dt || !A || !Cm || !block_decay || !s_in || !y) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {dt, A, Cm, block_decay, s_in, y};
    for (const void *q : ptrs)
        if (!aligned16(q)) return SSD_ERR_ALIGNMENT;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return SSD_ERR_ALIGNMENT;
    return from_cuda(cp_correct_launch(make_cp(shape, dtype), dt, A, Cm, block_decay, s_in, y, status,
                                       static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_bwd_workspace_bytes(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                                             size_t *bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    FwdProblem p;
    const ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    if (!simt_bwd_supported(p)) return SSD_ERR_UNSUPPORTED;
    *bytes = (p.B == 0 || p.L == 0) ? 0 : simt_bwd_workspace_bytes(p);
    return SSD_OK;
}

SSD_API ssd_status_t ssd_bwd_plan(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk, ssd_plan_t *plan) {
    if (!plan) return SSD_ERR_INVALID_ARG;
    FwdProblem p;
    const ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    if (!simt_bwd_supported(p)) return SSD_ERR_UNSUPPORTED;
    ssd_plan_t out{};
    if (p.B == 0 || p.L == 0) {
        out.path = SSD_PATH_NONE;
    } else {
        out.path = mma_bwd_supported(p) ? SSD_PATH_MMA : SSD_PATH_SIMT;
        out.kernels = 11;
        out.workspace_bytes = simt_bwd_workspace_bytes(p);
    }
    *plan = out;
    return SSD_OK;
}

SSD_API ssd_status_t ssd_bwd(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *x, const void *dt,
                             const float *A, const void *Bm, const void *Cm, const float *D,
                             const float *h0, int64_t chunk, const void *dy, const float *dh_final,
                             void *dx, void *ddt, float *dA, void *dBm, void *dCm, float *dD, float *dh0,
                             void *workspace, size_t workspace_bytes, void *stream) {
    FwdProblem p;
    ssd_status_t st = make_fwd(shape, dtype, chunk, &p);
    if (st != SSD_OK) return st;
    if (!simt_bwd_supported(p)) return SSD_ERR_UNSUPPORTED;
    if (!dA) return SSD_ERR_INVALID_ARG;
    const void *small[] = {dA, dD, dh0, dh_final};
    for (const void *q : small)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t head_bytes = (size_t)p.H * sizeof(float);
    if (p.B == 0 || p.L == 0) {
        cudaError_t e = cudaMemsetAsync(dA, 0, head_bytes, s);
        if (!e && dD) e = cudaMemsetAsync(dD, 0, head_bytes, s);
        if (!e && dh0 && p.B > 0) {
            const size_t state_bytes = (size_t)(p.B * p.H * p.P * p.N) * sizeof(float);
            e = dh_final ? cudaMemcpyAsync(dh0, dh_final, state_bytes, cudaMemcpyDeviceToDevice, s)
                         : cudaMemsetAsync(dh0, 0, state_bytes, s);
        }
        return from_cuda(e);
    }
    if (!x || !dt || !A || !Bm || !Cm || !dy || !dx || !ddt || !dBm || !dCm) return SSD_ERR_INVALID_ARG;
    const void *ptrs[] = {x, dt, A, Bm, Cm, D, h0, dy, dx, ddt, dBm, dCm, workspace};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < simt_bwd_workspace_bytes(p)) return SSD_ERR_WORKSPACE;
    p.x = x;
    p.dt = dt;
    p.A = A;
    p.Bm = Bm;
    p.Cm = Cm;
    p.D = D;
    p.h0 = h0;
    const BwdGrads g{dy, dh_final, dx, ddt, dBm, dCm, dA, dD, dh0};
    return from_cuda(simt_bwd(p, g, workspace, s));
}

SSD_API ssd_status_t ssd_conv_split(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *xbc, int64_t xbc_stride,
                                    const void *dt_raw, int64_t dt_stride, const float *conv_w, const float *conv_b,
                                    int64_t width, const float *dt_bias, void *x, void *Bm, void *Cm, void *dt,
                                    void *stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    const int64_t HP = shape->nheads * shape->headdim, GN = shape->ngroups * shape->dstate;
    if (width < 1 || width > 4 || xbc_stride < HP + 2 * GN || dt_stride < shape->nheads) return SSD_ERR_INVALID_ARG;
    if (HP % 2 != 0 || GN % 2 != 0 || xbc_stride % 2 != 0) return SSD_ERR_UNSUPPORTED;
    if (shape->batch == 0 || shape->seqlen == 0) return SSD_OK;
    if (!xbc || !dt_raw || !conv_w || !x || !Bm || !Cm || !dt) return SSD_ERR_INVALID_ARG;
    const uintptr_t pair = dtype == SSD_F32 ? 8 : 4, elem = dtype == SSD_F32 ? 4 : 2;
    if ((reinterpret_cast<uintptr_t>(xbc) & (pair - 1)) || (reinterpret_cast<uintptr_t>(dt_raw) & (elem - 1)))
        return SSD_ERR_ALIGNMENT;
    const void *ptrs[] = {conv_w, conv_b, dt_bias, x, Bm, Cm, dt};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return SSD_ERR_ALIGNMENT;
    const BlockShape s{shape->batch, shape->seqlen, shape->nheads, shape->headdim, shape->ngroups, shape->dstate};
    return from_cuda(conv_split_launch(s, dtype, xbc, xbc_stride, dt_raw, dt_stride, conv_w, conv_b, (int)width,
                                       dt_bias, x, Bm, Cm, dt, static_cast<cudaStream_t>(stream)));
}

SSD_API ssd_status_t ssd_gated_rmsnorm(int64_t rows, int64_t dim, int64_t ngroups, ssd_dtype_t dtype, const void *y,
                                       const void *z, int64_t z_stride, const float *weight, float eps, void *out,
                                       void *stream) {
    ssd_status_t st = check_dtype(dtype);
    if (st != SSD_OK) return st;
    if (rows < 0 || dim < 1 || ngroups < 1 || dim % ngroups != 0 || z_stride < dim || !(eps >= 0.f))
        return SSD_ERR_INVALID_ARG;
    if (dim > gated_rmsnorm_max_dim() || ngroups > 64 || (dim / ngroups) % 64 != 0 || z_stride % 2 != 0 ||
        rows > 0x7fffffffLL)
        return SSD_ERR_UNSUPPORTED;
    if (rows == 0) return SSD_OK;
    if (!y || !z || !weight || !out) return SSD_ERR_INVALID_ARG;
    const uintptr_t pair = dtype == SSD_F32 ? 8 : 4;
    if (reinterpret_cast<uintptr_t>(z) & (pair - 1)) return SSD_ERR_ALIGNMENT;
    const void *ptrs[] = {y, weight, out};
    for (const void *q : ptrs)
        if (!aligned16(q)) return SSD_ERR_ALIGNMENT;
    return from_cuda(gated_rmsnorm_launch(rows, (int)dim, (int)ngroups, dtype, y, z, z_stride, weight, eps, out,
                                          static_cast<cudaStream_t>(stream)));
}
