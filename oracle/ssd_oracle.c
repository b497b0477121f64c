/*
 * fp64 CPU oracle for the Mamba-2 SSD layer: the sequential recurrence.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use this file. It shares no code, header or constant with the
 * CUDA library, and the library never calls it.
 *
 * What it computes (the plain definition, evaluated token by token in fp64):
 *   for every batch row b and head h, with group g = h / (H / G):
 *     S = h0[b, h]                        (P x N; zeros when h0 is NULL)
 *     for t = 0 .. L-1:
 *       S = exp(dt[b,t,h] * A[h]) * S + dt[b,t,h] * x[b,t,h,:] B[b,t,g,:]^T
 *       y[b,t,h,:] = S C[b,t,g,:] + D[h] * x[b,t,h,:]
 *     h_final[b, h] = S
 * Sources: "A Visual Guide to Mamba and SSMs" (translated), sections
 * "What is a SSM" (state equation, output equation, D as a skip connection),
 * "From a Continuous to a Discrete Signal" (the step size Delta; the decay is the
 * zero-order-hold exp(Delta A); the input term is taken as Delta B, the reading
 * that the SSD problem statement uses) and "The Recurrent Representation"
 * (h_k = A h_{k-1} + B x_k, y_k = C h_k); "Selective SSM" (B, C, Delta depend
 * on the token, A does not); the Bi-Mamba summary, "Preliminary: Mamba Series"
 * (in SSD, A is a scalar times the identity per head, head dimension P > 1).
 *
 * Layouts (row-major, contiguous): x [B,L,H,P], dt [B,L,H], A [H], Bm/Cm
 * [B,L,G,N], D [H], h0/h_final [B,H,P,N], y [B,L,H,P], states [B,L,H,P,N]
 * (the state after each token; used by the speculative-verify reading).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One (b, h) recurrence. Output pointers may be NULL. y_bh points at y[b,0,h,0]
 * and advances by y_stride per token; st_bh likewise for the per-token states. */
static void ssd_stream(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t G,
                       int64_t N, const double *x, const double *dt, const double *A,
                       const double *Bm, const double *Cm, const double *D, const double *h0,
                       double *y_bh, int64_t y_stride, double *hf_bh, double *st_bh,
                       int64_t st_stride, double *S)
{
    const int64_t g = h / (H / G);
    const double Dh = D ? D[h] : 0.0;
    if (h0)
        memcpy(S, h0 + (b * H + h) * P * N, sizeof(double) * (size_t)(P * N));
    else
        memset(S, 0, sizeof(double) * (size_t)(P * N));

    for (int64_t t = 0; t < L; ++t) {
        const double d = dt[(b * L + t) * H + h];
        const double decay = exp(d * A[h]);
        const double *xt = x + ((b * L + t) * H + h) * P;
        const double *Bt = Bm + ((b * L + t) * G + g) * N;
        const double *Ct = Cm + ((b * L + t) * G + g) * N;
        for (int64_t p = 0; p < P; ++p) {
            double *Sp = S + p * N;
            const double dx = d * xt[p];
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                Sp[n] = decay * Sp[n] + dx * Bt[n];
                acc += Sp[n] * Ct[n];
            }
            if (y_bh)
                y_bh[t * y_stride + p] = acc + Dh * xt[p];
        }
        if (st_bh)
            memcpy(st_bh + t * st_stride, S, sizeof(double) * (size_t)(P * N));
    }
    if (hf_bh)
        memcpy(hf_bh, S, sizeof(double) * (size_t)(P * N));
}

/* Whole problem, parallel over (b, h) streams (each stream is sequential, so the
 * result does not depend on the thread count). nthreads <= 0: OpenMP default.
 * Returns 0, or -1 on a bad argument / allocation failure. */
int oracle_ssd_recurrent(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t G, int64_t N,
                         const double *x, const double *dt, const double *A, const double *Bm,
                         const double *Cm, const double *D, const double *h0, double *y,
                         double *h_final, double *states, int nthreads)
{
    if (Bsz < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || H % G != 0)
        return -1;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)(P * N));
        if (!S) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < Bsz * H; ++bh) {
            if (!S)
                continue;
            const int64_t b = bh / H, h = bh % H;
            ssd_stream(b, h, L, H, P, G, N, x, dt, A, Bm, Cm, D, h0,
                       y ? y + (b * L * H + h) * P : NULL, H * P,
                       h_final ? h_final + (b * H + h) * P * N : NULL,
                       states ? states + (b * L * H + h) * P * N : NULL, H * P * N, S);
        }
        free(S);
    }
    return err;
}
