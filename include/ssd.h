/*
 * libssd: the Mamba-2 SSD (state space duality) layer forward pass on B200
 * (sm_100a), evaluated with the chunked algorithm, and its speculative-decoding
 * verify step.
 *
 * Per batch row b and head h (group g = h / (nheads / ngroups)):
 *     h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T      (P x N state)
 *     y_t = h_t C_t + D_h * x_t
 * Sources: Mamba-2 SSD write-up (msbhsh.com), sections "SSD 层" (the SSD layer:
 * a selective SSM whose A is a scalar per head) and "SSD 算法：分块和状态传递"
 * (chunks of Q tokens; intra-chunk matmuls, chunk states, a short scan across
 * chunks, state-to-output); "A Visual Guide to Mamba and SSMs", "What is a SSM"
 * (D is a skip connection) and "The Recurrent Representation"; the Llama-to-Mamba
 * distillation write-up, "推测解码" (verify K draft tokens, keep the state at the
 * accepted position).
 *
 * Conventions for every entry point below:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major and
 *    contiguous, 16-byte aligned. The library allocates no memory and may be called
 *    from several host threads at once. Its only global mutable state is the test
 *    hook's wait limit (ssd_set_wait_limit_us) and the built-in device array of
 *    ssd_fwd_static_scratch.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Calls are asynchronous: SSD_OK means "validated and launched".
 *    Faults inside a kernel surface from a later CUDA call or synchronisation.
 *  - Arguments are validated before anything is launched; on an error status no
 *    kernel was launched and no output was touched. Nothing aborts or prints.
 *  - x, dt, B, C and y share one storage type (ssd_dtype_t). A, D, h0, h_final,
 *    states_out and h_keep are always fp32. Arithmetic is fp32 (accumulation in
 *    fp32; bf16 products on tensor cores where the inputs are bf16).
 *  - The head-to-group map is contiguous: head h reads group h / (nheads/ngroups).
 */
#ifndef SSD_H
#define SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ssd_shape_t {
    int64_t batch;   /* B >= 0 */
    int64_t seqlen;  /* L >= 0 (for ssd_verify: the number of draft tokens K) */
    int64_t nheads;  /* H >= 1 */
    int64_t headdim; /* P, 1..256 */
    int64_t ngroups; /* G >= 1, divides H */
    int64_t dstate;  /* N, 1..256 */
} ssd_shape_t;

typedef enum ssd_dtype_t {
    SSD_F32 = 0,  /* IEEE fp32 */
    SSD_BF16 = 1, /* bfloat16; y is rounded to nearest even from fp32 */
} ssd_dtype_t;

typedef enum ssd_status_t {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1, /* NULL required pointer, negative or inconsistent size */
    SSD_ERR_UNSUPPORTED = 2, /* a size outside the supported range */
    SSD_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned */
    SSD_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
    SSD_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch or attribute) */
    SSD_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out */
} ssd_status_t;

/* Human-readable text for a status code (static storage, never NULL). */
const char *ssd_strerror(ssd_status_t status);

/* The implementation ssd_fwd selects for a problem (see ssd_fwd_plan). */
typedef enum ssd_path_t {
    SSD_PATH_NONE = 0,    /* nothing to compute (batch == 0 or seqlen == 0) */
    SSD_PATH_SIMT = 1,    /* chunked, fp32 CUDA-core arithmetic, one kernel per step */
    SSD_PATH_TCGEN05 = 2, /* chunked, fused, bf16 tcgen05 tensor-core MMAs */
    SSD_PATH_MMA = 3,     /* chunked, bf16 mma.sync tensor-core products (ssd_bwd) */
} ssd_path_t;

typedef struct ssd_plan_t {
    int32_t path;           /* an ssd_path_t */
    int32_t kernels;        /* kernel launches per ssd_fwd call */
    size_t workspace_bytes; /* same value as ssd_fwd_workspace_bytes */
} ssd_plan_t;

/*
 * Describe what ssd_fwd would launch for this problem, without launching.
 * Errors: as ssd_fwd_workspace_bytes; *plan is untouched on error.
 */
ssd_status_t ssd_fwd_plan(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                          ssd_plan_t *plan);

/*
 * Bytes of device workspace that ssd_fwd needs for this problem
 * (written to *bytes; 0 is possible). The per-chunk intermediates (within-chunk
 * decay cumsums and, on some paths, chunk states) live there.
 * Errors: SSD_ERR_INVALID_ARG / SSD_ERR_UNSUPPORTED as ssd_fwd would return.
 */
ssd_status_t ssd_fwd_workspace_bytes(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                                     size_t *bytes);

/*
 * SSD forward pass over a whole sequence, by the chunked algorithm with chunk
 * size `chunk` (1..256; the last chunk may be shorter).
 *   x        [B, L, H, P]   dtype          input (the "V" of the attention view)
 *   dt       [B, L, H]      dtype          step size, used as given (no softplus)
 *   A        [H]            fp32           decay rate per head (A_h <= 0 expected)
 *   Bm, Cm   [B, L, G, N]   dtype          input and output projections
 *   D        [H]            fp32 or NULL   skip weight (NULL = 0)
 *   h0       [B, H, P, N]   fp32 or NULL   initial state (NULL = zeros)
 *   y        [B, L, H, P]   dtype          output
 *   h_final  [B, H, P, N]   fp32 or NULL   state after the last token
 *   workspace, workspace_bytes             >= ssd_fwd_workspace_bytes(...)
 * seqlen == 0 writes only h_final (= h0 or zeros); batch == 0 does nothing.
 * The return value reports argument and launch errors only; the call is asynchronous.
 * On SSD_PATH_TCGEN05 (ssd_fwd_plan) the kernel's CTAs wait on one another through
 * bounded waits; if one runs out, the kernel abandons the call (y and h_final are then
 * incomplete) and sets bit 0 of the workspace's first int32, the status word, which the
 * call clears before launching. ssd_fwd_status reads it.
 */
ssd_status_t ssd_fwd(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *x, const void *dt,
                     const float *A, const void *Bm, const void *Cm, const float *D,
                     const float *h0, int64_t chunk, void *y, float *h_final, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * Outcome of the last ssd_fwd on this workspace: synchronizes `stream`, then returns
 * SSD_ERR_TIMEOUT if a bounded wait ran out (status word bit 0), SSD_ERR_CUDA if the
 * kernel refused to run (any other bit: its shared memory was misaligned) or the
 * stream reported an error, SSD_OK otherwise. Paths other than SSD_PATH_TCGEN05 have
 * no waits and always give SSD_OK. shape, dtype and chunk are those of the call.
 */
ssd_status_t ssd_fwd_status(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                            const void *workspace, void *stream);

/*
 * Test hook: the limit, in microseconds, of every bounded device-side wait in the
 * kernels launched after this call, process-wide (0 restores the built-in 2 s).
 * A small limit makes a wait between CTAs run out on purpose, so that the abort path
 * (status word, drained copies, freed tensor memory) can be checked without a fault.
 * Errors: SSD_ERR_INVALID_ARG outside 0..2000000.
 */
ssd_status_t ssd_set_wait_limit_us(int32_t us);

/*
 * ssd_fwd for callers that cannot allocate device memory. No counterpart in
 * the pages describing the method: this entry point exists for deployment.
 *
 * Some callers cannot call cudaMalloc: an inference server that reserves all of
 * HBM up front and manages it itself, a real-time loop where an allocation could
 * block or fail, a plugin whose host framework owns every allocation and passes
 * in only input and output buffers. They cannot supply ssd_fwd's workspace.
 * This entry point takes the same inputs and outputs as ssd_fwd, minus the
 * workspace, and allocates nothing (no cudaMalloc, cudaFree or allocating library
 * call). Its intermediates live in one built-in device array of
 * SSD_STATIC_SCRATCH_BYTES (16 MiB), which every GPU that loads the library holds
 * until the process exits.
 *  - Always runs the fp32 CUDA-core kernels (the exact path of ssd_fwd).
 *  - Problems whose intermediates need more than SSD_STATIC_SCRATCH_BYTES return
 *    SSD_ERR_WORKSPACE before launching anything (ssd_fwd_plan's workspace_bytes,
 *    for a problem ssd_fwd runs on the CUDA-core path, is the amount needed).
 *  - The first call on each device looks up the array's device address (with that
 *    device current) and caches it; make that first call before any CUDA stream
 *    capture begins.
 *  - All calls on a device share the one array, which keeps the previous call's
 *    contents (every element read is first written by the same call, so stale
 *    contents are harmless). Calls that may overlap on the GPU -- on different
 *    streams, or from several host threads without ordering -- race on it:
 *    serialise them.
 */
#define SSD_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

ssd_status_t ssd_fwd_static_scratch(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *x,
                                    const void *dt, const float *A, const void *Bm,
                                    const void *Cm, const float *D, const float *h0,
                                    int64_t chunk, void *y, float *h_final, void *stream);

/*
 * Speculative-decoding verify: run K draft tokens from the saved state h0 and
 * return every intermediate state, so the caller can keep the state at the
 * position where verification stops. shape->seqlen must equal K (1..64).
 *   h0          [B, H, P, N]      fp32           state before the first draft token
 *   x           [B, K, H, P]      dtype
 *   dt          [B, K, H]         dtype
 *   A, D        [H]               fp32 (D may be NULL = 0)
 *   Bm, Cm      [B, K, G, N]      dtype
 *   states_out  [B, K, H, P, N]   fp32 or NULL   state after draft token k
 *   y           [B, K, H, P]      dtype          outputs of the K tokens
 * Requires dstate % 4 == 0. With states_out == NULL only y is written: the flow
 * that keeps one state (ssd_advance_state below) instead of all K. That case evaluates
 * the K tokens in the chunked form (each state row read once, no per-token state chain),
 * so its y can differ from the states_out != NULL case in the last bits.
 */
ssd_status_t ssd_verify(const ssd_shape_t *shape, ssd_dtype_t dtype, const float *h0,
                        const void *x, const void *dt, const float *A, const void *Bm,
                        const void *Cm, const float *D, int64_t K, float *states_out, void *y,
                        void *stream);

/*
 * Keep the state at the accepted position, once the caller has decided how many
 * draft tokens of each batch row were accepted:
 *   h_keep[b] = h0[b]                       if accepted[b] == 0
 *             = states_out[b, accepted[b]-1] if 1 <= accepted[b] <= K
 * A bit-exact copy. `accepted` is a device int32 array [B]. A row whose index is
 * outside 0..K is filled with quiet NaN (the host cannot see device values).
 * shape->seqlen is ignored; dims as in ssd_verify.
 */
ssd_status_t ssd_select_state(const ssd_shape_t *shape, int64_t K, const float *h0,
                              const float *states_out, const int32_t *accepted, float *h_keep,
                              void *stream);

/*
 * The kept state without storing the intermediate ones. The distillation
 * write-up ("推测解码") notes that keeping every intermediate state of a verify
 * pass costs too much memory; the state at the accepted position is what is
 * needed. Once the caller knows how many draft tokens of each batch row were
 * accepted, this recomputes that state from h0:
 *   h_keep[b] = state after the first accepted[b] tokens, starting from h0[b]
 *             (accepted[b] == 0: a copy of h0[b])
 * Same arguments and layouts as ssd_verify (shape->seqlen == K); `accepted` is a
 * device int32 array [B]. The result is bit-identical to ssd_verify's
 * states_out[b, accepted[b]-1] (the same fp32 operations in the same order). A row
 * whose count is outside 0..K is filled with quiet NaN. h_keep may be h0 itself
 * (the state advanced in place); no other overlap between them is allowed
 * (SSD_ERR_INVALID_ARG). Requires dstate % 4 == 0 and K <= 64.
 */
ssd_status_t ssd_advance_state(const ssd_shape_t *shape, ssd_dtype_t dtype, const float *h0,
                               const void *x, const void *dt, const float *A, const void *Bm,
                               int64_t K, const int32_t *accepted, float *h_keep, void *stream);

/*
 * One generated token (the recurrent form, "The Recurrent Representation" of the
 * visual guide): the state is updated in place,
 *   state <- exp(dt * A_h) * state + dt * x B^T,   y = state C + D_h * x
 * shape->seqlen must be 1.
 *   state   [B, H, P, N]   fp32           read and written
 *   x       [B, H, P]      dtype
 *   dt      [B, H]         dtype
 *   A, D    [H]            fp32 (D may be NULL = 0)
 *   Bm, Cm  [B, G, N]      dtype
 *   y       [B, H, P]      dtype
 * Requires dstate % 4 == 0. Same arithmetic as ssd_verify with K = 1.
 */
ssd_status_t ssd_decode_step(const ssd_shape_t *shape, ssd_dtype_t dtype, float *state,
                             const void *x, const void *dt, const float *A, const void *Bm,
                             const void *Cm, const float *D, void *y, void *stream);

/*
 * Context (sequence) parallelism: a long sequence split into contiguous segments,
 * one per rank (the SSD write-up, "序列并行", built on the state passing of
 * "SSD 算法：分块和状态传递"). Each rank runs ssd_fwd on its segment (rank 0 with
 * the true h0, the others from zeros), which gives its local outputs y and local
 * end state S_r; then:
 *   1. ssd_cp_decay:   the segment's decay sums (per 128-token block, and the total
 *                      Lambda_r = sum over the segment of dt_t * A_h);
 *   2. the caller all-gathers S_r [B,H,P,N] and Lambda_r [B,H] over the ranks, in
 *      rank order (one collective; ncclAllGather through torch.distributed);
 *   3. ssd_cp_combine: the state entering this segment, the exclusive scan
 *        S_in(0) = 0,  S_in(q+1) = exp(Lambda_q) S_in(q) + S_q,
 *      and the segment's true end state exp(Lambda_r) S_in(r) + S_r;
 *   4. ssd_cp_correct: y_t += exp(sum_{s<=t in segment} dt_s A_h) C_t S_in(r)^T, the
 *      state-to-output step for the incoming state (a no-op for rank 0).
 * Shapes below are those of the rank's segment (shape->seqlen = its length).
 */
#define SSD_CP_BLOCK 128 /* tokens per decay block: block_decay has ceil(seqlen/128) per (b, h) */

/*
 *   dt           [B, L, H]             dtype
 *   A            [H]                   fp32
 *   block_decay  [B, H, ceil(L/128)]   fp32   sum of dt*A over each 128-token block
 *   total        [B, H]                fp32   Lambda = the block sums added in order
 * L == 0 writes total = 0 (dt and block_decay may then be NULL).
 */
ssd_status_t ssd_cp_decay(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *dt, const float *A,
                          float *block_decay, float *total, void *stream);

/*
 *   states   [R, B, H, P, N]   fp32   every rank's local end state, in rank order
 *   totals   [R, B, H]         fp32   every rank's Lambda, in rank order
 *   s_in     [B, H, P, N]      fp32   out: the state entering segment `rank`
 *   h_final  [B, H, P, N]      fp32 or NULL   out: the true end state of segment `rank`
 *                                     (for the last rank: the whole sequence's h_final)
 * R = nranks >= 1, 0 <= rank < R. shape->seqlen and shape->ngroups are ignored.
 * Requires headdim * dstate % 4 == 0. h_final must not overlap states.
 */
ssd_status_t ssd_cp_combine(const ssd_shape_t *shape, int64_t nranks, int64_t rank, const float *states,
                            const float *totals, float *s_in, float *h_final, void *stream);

/*
 *   dt, Cm        as in ssd_fwd, for the segment
 *   A             [H] fp32
 *   block_decay   [B, H, ceil(L/128)] from ssd_cp_decay on the same segment
 *   s_in          [B, H, P, N] fp32 from ssd_cp_combine
 *   y             [B, L, H, P] dtype, read and written (y += the incoming state's term)
 *   status        int32 device word or NULL: bit 0 is set (never cleared) if a bounded
 *                 device-side wait ran out, in which case y is incomplete; zero it beforehand
 * bf16 inputs run on tensor cores with S_in rounded to bf16 and fp32 accumulation: tcgen05
 * when headdim == 64, dstate % 64 == 0 and each group has an even number of heads, mma.sync
 * when headdim % 64 == 0 and dstate % 16 == 0. Other shapes and fp32 inputs run in fp32 on
 * CUDA cores.
 */
ssd_status_t ssd_cp_correct(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *dt, const float *A,
                            const void *Cm, const float *block_decay, const float *s_in, void *y,
                            int32_t *status, void *stream);

/*
 * Backward pass of ssd_fwd: given the cotangents dy of y and dh_final of h_final, the
 * gradient of  sum(dy * y) + sum(dh_final * h_final)  with respect to every input.
 * The states are recomputed from the inputs rather than stored by the forward (the
 * recomputation of the hardware-aware algorithm, "A Visual Guide to Mamba and SSMs",
 * section "Recomputation"); the chunks follow "SSD 算法：分块和状态传递" of the SSD
 * write-up, run in reverse.
 *   x, dt, A, Bm, Cm, D, h0, chunk   the forward's inputs, as in ssd_fwd
 *   dy        [B, L, H, P]   dtype          cotangent of y
 *   dh_final  [B, H, P, N]   fp32 or NULL   cotangent of h_final (NULL = 0)
 *   dx        [B, L, H, P]   dtype          out
 *   ddt       [B, L, H]      dtype          out
 *   dA        [H]            fp32           out (summed over the batch)
 *   dBm, dCm  [B, L, G, N]   dtype          out (summed over the heads of each group)
 *   dD        [H]            fp32 or NULL   out (also when D is NULL: the gradient at D = 0)
 *   dh0       [B, H, P, N]   fp32 or NULL   out (also when h0 is NULL: the gradient at h0 = 0)
 *   workspace, workspace_bytes              >= ssd_bwd_workspace_bytes(...)
 * Arithmetic follows ssd_bwd_plan: on SSD_PATH_MMA every product runs on tensor cores
 * (mma.sync, bf16 operands, fp32 accumulation) and the rest in fp32; on SSD_PATH_SIMT
 * everything is fp32 on CUDA cores. dBm and dCm are summed with fp32 atomics, so their
 * last bits can differ between runs. batch == 0 zeroes dA and dD;
 * seqlen == 0 also writes dh0 = dh_final (or zeros).
 * Errors as ssd_fwd; SSD_ERR_UNSUPPORTED when headdim and dstate are too large for the
 * kernels' shared-memory tiles together (never for headdim, dstate <= 256).
 */
ssd_status_t ssd_bwd_workspace_bytes(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk,
                                     size_t *bytes);
/* What ssd_bwd would launch: SSD_PATH_MMA (bf16 inputs with (headdim, dstate) in {(64, 64),
 * (64, 128), (64, 256), (128, 128)}: every product on tensor cores, bf16 operands, fp32
 * accumulation), SSD_PATH_SIMT (everything else: fp32 CUDA cores) or SSD_PATH_NONE. */
ssd_status_t ssd_bwd_plan(const ssd_shape_t *shape, ssd_dtype_t dtype, int64_t chunk, ssd_plan_t *plan);
ssd_status_t ssd_bwd(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *x, const void *dt,
                     const float *A, const void *Bm, const void *Cm, const float *D, const float *h0,
                     int64_t chunk, const void *dy, const float *dh_final, void *dx, void *ddt,
                     float *dA, void *dBm, void *dCm, float *dD, float *dh0, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * The Mamba-2 block around the SSD layer. The block's input projection (a plain GEMM) writes,
 * per token, one row [z | x B C | dt_raw]; the SSD layer runs on x, B, C, dt; the gated,
 * grouped norm of its output feeds the output projection (a plain GEMM). The pages describe
 * the block in words only ("A Visual Guide to Mamba and SSMs", "The Mamba Block": an input
 * projection, then a convolution before the SSM so tokens are not computed independently; the
 * SSD write-up, "张量并行": every SSM parameter is a projection of the layer input, and the norm
 * is grouped). These two calls are the operations between the GEMMs and ssd_fwd.
 *
 * ssd_conv_split: causal depthwise convolution of the x, B, C channels, SiLU, split into the
 * layouts ssd_fwd takes, and the step size:
 *   out[t, c] = silu(conv_b[c] + sum_{j<W} conv_w[c, j] * xbc[t - (W - 1) + j, c])  (zeros before t = 0)
 *   channels c in [0, H*P) -> x [B,L,H,P]; [H*P, H*P + G*N) -> Bm [B,L,G,N]; the next G*N -> Cm
 *   dt[b, t, h] = softplus(dt_raw[b, t, h] + dt_bias[h])
 *   xbc      [B, L, *] dtype, row stride xbc_stride elements (>= H*P + 2*G*N, even), the
 *            Cc = H*P + 2*G*N conv channels at the start of each row; 4-byte (bf16) or
 *            8-byte (fp32) aligned
 *   dt_raw   [B, L, *] dtype, row stride dt_stride (>= H), H values per row
 *   conv_w   [Cc, W] fp32, 1 <= W <= 4; conv_b [Cc] fp32 or NULL (= 0); dt_bias [H] fp32 or NULL
 *   x, Bm, Cm, dt   outputs, 16-byte aligned
 * Requires H*P and G*N even. shape->... as in ssd_fwd.
 */
ssd_status_t ssd_conv_split(const ssd_shape_t *shape, ssd_dtype_t dtype, const void *xbc, int64_t xbc_stride,
                            const void *dt_raw, int64_t dt_stride, const float *conv_w, const float *conv_b,
                            int64_t width, const float *dt_bias, void *x, void *Bm, void *Cm, void *dt,
                            void *stream);

/*
 * ssd_gated_rmsnorm: for each of `rows` rows of `dim` channels, in `ngroups` groups of
 * dim / ngroups consecutive channels,
 *   g = y * silu(z),   out = weight * g / sqrt(mean over the group of g^2 + eps)
 *   y      [rows, dim] dtype, contiguous, 16-byte aligned
 *   z      [rows, *] dtype, row stride z_stride (>= dim, even), 4-byte (bf16) or 8-byte (fp32)
 *          aligned: the z columns of the input projection's rows can be passed in place (16-byte
 *          aligned rows take 16-byte loads)
 *   weight [dim] fp32; out [rows, dim] dtype, 16-byte aligned
 * Requires dim <= 8192, 1 <= ngroups <= 64 and (dim / ngroups) % 64 == 0.
 */
ssd_status_t ssd_gated_rmsnorm(int64_t rows, int64_t dim, int64_t ngroups, ssd_dtype_t dtype, const void *y,
                               const void *z, int64_t z_stride, const float *weight, float eps, void *out,
                               void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H */
