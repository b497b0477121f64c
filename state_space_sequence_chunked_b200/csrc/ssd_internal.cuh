// Internal declarations shared by the libssd translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// One forward problem, validated by the API layer.
struct FwdProblem {
    int64_t B, L, H, P, G, N, Q, nc;
    ssd_dtype_t dtype;
    const void *x, *dt, *Bm, *Cm;
    const float *A, *D, *h0;
    void *y;
    float *h_final;
};

struct VerifyProblem {
    int64_t B, K, H, P, G, N;
    ssd_dtype_t dtype;
    const float *h0;
    const void *x, *dt, *Bm, *Cm;
    const float *A, *D;
    float *states_out;
    void *y;
};

// Cotangents in and gradients out of the backward pass (dh_final, dD, dh0 may be NULL).
struct BwdGrads {
    const void *dy;
    const float *dh_final;
    void *dx, *ddt, *dBm, *dCm;
    float *dA, *dD, *dh0;
};

// A sequence segment for the context-parallel steps (ssd_cp_*).
struct CpProblem {
    int64_t B, L, H, P, G, N;
    ssd_dtype_t dtype;
};

constexpr size_t kWsAlign = 256;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---- argument rules shared by every forward entry point ----------------------------
constexpr int64_t kMaxDim = 256;       // headdim, dstate
constexpr int64_t kMaxChunk = 256;
constexpr int64_t kMaxGridYZ = 65535;  // batch and nheads map to grid y/z

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline ssd_status_t check_shape(const ssd_shape_t *s) {
    if (!s) return SSD_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0 || s->nheads < 1 || s->headdim < 1 || s->ngroups < 1 || s->dstate < 1)
        return SSD_ERR_INVALID_ARG;
    if (s->nheads % s->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (s->headdim > kMaxDim || s->dstate > kMaxDim) return SSD_ERR_UNSUPPORTED;
    if (s->batch > kMaxGridYZ || s->nheads > kMaxGridYZ) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

inline ssd_status_t check_dtype(ssd_dtype_t d) { return (d == SSD_F32 || d == SSD_BF16) ? SSD_OK : SSD_ERR_INVALID_ARG; }

// Shape, dtype and chunk checks, then the problem record (pointers unset).
inline ssd_status_t make_fwd(const ssd_shape_t *s, ssd_dtype_t dtype, int64_t chunk, FwdProblem *p) {
    ssd_status_t st = check_shape(s);
    if (st != SSD_OK) return st;
    if ((st = check_dtype(dtype)) != SSD_OK) return st;
    if (chunk < 1) return SSD_ERR_INVALID_ARG;
    if (chunk > kMaxChunk) return SSD_ERR_UNSUPPORTED;
    *p = FwdProblem{};
    p->B = s->batch;
    p->L = s->seqlen;
    p->H = s->nheads;
    p->P = s->headdim;
    p->G = s->ngroups;
    p->N = s->dstate;
    p->Q = chunk;
    p->nc = (s->seqlen + chunk - 1) / chunk;
    p->dtype = dtype;
    return SSD_OK;
}

// Limit, in microseconds, of each bounded device-side wait of the next launches (0: the
// built-in 2 s). Process-wide; set through ssd_set_wait_limit_us.
int wait_limit_us();

// ---- chunked path with fp32 CUDA-core arithmetic (exact path for fp32 inputs) ----
size_t simt_fwd_workspace_bytes(const FwdProblem &p);
cudaError_t simt_fwd(const FwdProblem &p, void *ws, cudaStream_t s);
// steps 0, 2, 3 alone: A_cs [B,H,nc,Q], dt [B,H,nc,Q], entering states [B,H,nc,P,N], h_final
cudaError_t simt_states(const FwdProblem &p, float *acs, float *dtw, float *states, float *h_final,
                        cudaStream_t s);
// the two halves of simt_states around step 2: step 0, and step 3 (in place on `states`)
cudaError_t simt_cumsum(const FwdProblem &p, float *acs, float *dtw, cudaStream_t s);
cudaError_t simt_state_pass(const FwdProblem &p, const float *acs, float *states, float *h_final, cudaStream_t s);
// out[b,h,c] = sum_{l in c} exp(A_cs[l]) dy_l C_l^T   (dy [B,L,H,P] in the input dtype)
cudaError_t simt_adjoint_chunk_sums(const FwdProblem &p, const void *dy, const float *acs, float *out,
                                    cudaStream_t s);

// ---- backward pass (chunked, states recomputed, fp32 CUDA-core arithmetic) ----------
bool simt_bwd_supported(const FwdProblem &p);
size_t simt_bwd_workspace_bytes(const FwdProblem &p);
cudaError_t simt_bwd(const FwdProblem &p, const BwdGrads &g, void *ws, cudaStream_t s);
// bf16 tensor-core (mma.sync) kernels of the backward, for the (P, N) pairs mma_bwd_supported
// accepts. Chunk sums: forward (x, B, exp(A_cs[Q-1] - A_cs[l]) dt_l) or adjoint (dy, C, exp(A_cs[l])).
bool mma_bwd_supported(const FwdProblem &p);
cudaError_t mma_chunk_sums(const FwdProblem &p, bool adjoint, const void *u, const void *v, const float *acs,
                           const float *dtw, float *out, cudaStream_t s);
// Sources: dx, dB (atomics), x.u, and per token K_s, U_s and (atomics) R_l; targets: dC
// (atomics) and T_l; the chunk-local pieces of the log-decay gradient (see ssd_bwd.cu).
cudaError_t mma_bwd_src(const FwdProblem &p, const void *dy, const float *acs, const float *dtw, const float *gend,
                        void *dx, float *dB_acc, float *kq, float *rq, float *uq, float *ddt_dir, float *dDpart,
                        cudaStream_t s);
cudaError_t mma_bwd_dst(const FwdProblem &p, const void *dy, const float *acs, const float *dtw, const float *s_in,
                        float *dC_acc, float *tq, cudaStream_t s);
int mma_row_tiles(const FwdProblem &p);

// ---- fused chunked path on tcgen05 tensor cores (bf16, P = 64, N in {128, 256}) ----
bool tc_supported(const FwdProblem &p);
size_t tc_fwd_workspace_bytes(const FwdProblem &p);
cudaError_t tc_fwd(const FwdProblem &p, void *ws, cudaStream_t s);
// the two-heads-per-task kernel that tc_fwd runs where it applies (N = 128, heads per group even)
bool tc_pair_supported(const FwdProblem &p);
size_t tc_pair_workspace_bytes(const FwdProblem &p);
cudaError_t tc_pair_fwd(const FwdProblem &p, void *ws, cudaStream_t s);

// ---- verify / select --------------------------------------------------------------
cudaError_t verify_launch(const VerifyProblem &p, cudaStream_t s);
// states_out may be NULL (outputs only). k_advance: state after accepted[b] tokens.
// k_decode: one token, state updated in place (p.h0 and p.states_out unused).
cudaError_t advance_launch(const VerifyProblem &p, const int32_t *accepted, float *h_keep, cudaStream_t s);
cudaError_t decode_launch(const VerifyProblem &p, float *state, cudaStream_t s);
cudaError_t select_launch(int64_t B, int64_t K, int64_t per_row, const float *h0,
                          const float *states_out, const int32_t *accepted, float *h_keep,
                          cudaStream_t s);

// ---- context parallelism: decay sums, the exchange scan, the state-to-output correction
int cp_nblk(int64_t L);
cudaError_t cp_block_decay_launch(const CpProblem &p, const void *dt, const float *A, float *bsum, float *total,
                                  cudaStream_t s);
cudaError_t cp_combine_launch(const CpProblem &p, int R, int rank, const float *states, const float *totals,
                              float *s_in, float *h_final, cudaStream_t s);
bool cp_correct_uses_mma(const CpProblem &p);
bool cp_correct_uses_tc(const CpProblem &p);
cudaError_t cp_correct_tc_launch(const CpProblem &p, const void *dt, const float *A, const void *Cm, const float *bsum,
                                 const float *s_in, void *y, int *status, cudaStream_t s);
cudaError_t cp_correct_launch(const CpProblem &p, const void *dt, const float *A, const void *Cm, const float *bsum,
                              const float *s_in, void *y, int *status, cudaStream_t s);

// ---- the Mamba-2 block around the SSD: conv + split, gated grouped RMSNorm ------------
struct BlockShape {
    int64_t B, L, H, P, G, N;
};
cudaError_t conv_split_launch(const BlockShape &s, ssd_dtype_t dtype, const void *xbc, int64_t xbc_stride,
                              const void *dt_raw, int64_t dt_stride, const float *conv_w, const float *conv_b,
                              int width, const float *dt_bias, void *x, void *Bm, void *Cm, void *dt, cudaStream_t st);
int gated_rmsnorm_max_dim();
cudaError_t gated_rmsnorm_launch(int64_t rows, int dim, int ngroups, ssd_dtype_t dtype, const void *y, const void *z,
                                 int64_t z_stride, const float *w, float eps, void *out, cudaStream_t st);

// ---- element access ---------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store_as(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_as(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

}  // namespace ssd
