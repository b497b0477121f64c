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

/*
 * Backward pass: the vector-Jacobian product of the recurrence above.
 *
 * Given the output cotangents dy [B,L,H,P] and dh_final [B,H,P,N] (NULL = 0), it
 * returns the gradient of  sum(dy * y) + sum(dh_final * h_final)  with respect to
 * every input. It is the recurrence differentiated token by token in reverse (the
 * adjoint of S_t = a_t S_{t-1} + dt_t x_t B_t^T, y_t = S_t C_t + D x_t, with
 * a_t = exp(dt_t A_h)). With Gbar the adjoint of S_t, walking t = L-1 .. 0:
 *   Gbar  += dy_t C_t^T                           (y_t reads S_t)
 *   dC_t  += S_t^T dy_t          dD_h += dy_t . x_t
 *   dx_t   = D_h dy_t + dt_t Gbar B_t
 *   dB_t  += dt_t Gbar^T x_t
 *   ddt_t  = x_t^T Gbar B_t + A_h a_t <Gbar, S_{t-1}>
 *   dA_h  += dt_t a_t <Gbar, S_{t-1}>
 *   Gbar   = a_t Gbar                             (now the adjoint of S_{t-1})
 * and dh0 = Gbar at the end. dC and dB sum over the heads of a group.
 *
 * The states S_t are not kept for the whole sequence. As in the hardware-aware
 * algorithm of "A Visual Guide to Mamba and SSMs" (section "Recomputation":
 * intermediate states are recomputed in the backward pass rather than stored),
 * the forward sweep keeps the state entering every segment of `seg` tokens, and
 * the reverse sweep recomputes one segment's states from it before walking back
 * through them.
 *
 * Outputs: dx [B,L,H,P], ddt [B,L,H], dA [H], dBm/dCm [B,L,G,N], dD [H] (may be
 * NULL), dh0 [B,H,P,N] (may be NULL). Every output is overwritten.
 */
static void ssd_stream_bwd(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t G,
                           int64_t N, int64_t seg, const double *x, const double *dt,
                           const double *A, const double *Bm, const double *Cm, const double *D,
                           const double *h0, const double *dy, const double *dh_final,
                           double *dx, double *ddt, double *dB_h, double *dC_h, double *dh0,
                           double *dA_bh, double *dD_bh, double *ck, double *ss, double *Gb,
                           double *tmpP)
{
    const int64_t g = h / (H / G), PN = P * N;
    const double Dh = D ? D[h] : 0.0, Ah = A[h];
    const int64_t nseg = (L + seg - 1) / seg;

    /* forward sweep: ck[k] = state entering segment k */
    double *S = ss; /* scratch: reused below as the segment's states */
    if (h0)
        memcpy(S, h0 + (b * H + h) * PN, sizeof(double) * (size_t)PN);
    else
        memset(S, 0, sizeof(double) * (size_t)PN);
    for (int64_t t = 0; t < L; ++t) {
        if (t % seg == 0)
            memcpy(ck + (t / seg) * PN, S, sizeof(double) * (size_t)PN);
        const double d = dt[(b * L + t) * H + h], decay = exp(d * Ah);
        const double *xt = x + ((b * L + t) * H + h) * P;
        const double *Bt = Bm + ((b * L + t) * G + g) * N;
        for (int64_t p = 0; p < P; ++p)
            for (int64_t n = 0; n < N; ++n)
                S[p * N + n] = decay * S[p * N + n] + d * xt[p] * Bt[n];
    }

    /* reverse sweep */
    if (dh_final)
        memcpy(Gb, dh_final + (b * H + h) * PN, sizeof(double) * (size_t)PN);
    else
        memset(Gb, 0, sizeof(double) * (size_t)PN);
    double dA_acc = 0.0, dD_acc = 0.0;
    for (int64_t k = nseg - 1; k >= 0; --k) {
        const int64_t t0 = k * seg, t1 = (t0 + seg < L) ? t0 + seg : L;
        /* recompute the segment: ss[t - t0] = S_t */
        const double *prev = ck + k * PN;
        for (int64_t t = t0; t < t1; ++t) {
            const double d = dt[(b * L + t) * H + h], decay = exp(d * Ah);
            const double *xt = x + ((b * L + t) * H + h) * P;
            const double *Bt = Bm + ((b * L + t) * G + g) * N;
            double *cur = ss + (t - t0) * PN;
            for (int64_t p = 0; p < P; ++p)
                for (int64_t n = 0; n < N; ++n)
                    cur[p * N + n] = decay * prev[p * N + n] + d * xt[p] * Bt[n];
            prev = cur;
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const double d = dt[(b * L + t) * H + h], decay = exp(d * Ah);
            const double *xt = x + ((b * L + t) * H + h) * P;
            const double *dyt = dy + ((b * L + t) * H + h) * P;
            const double *Bt = Bm + ((b * L + t) * G + g) * N;
            const double *Ct = Cm + ((b * L + t) * G + g) * N;
            const double *St = ss + (t - t0) * PN;
            const double *Sp = (t > t0) ? ss + (t - 1 - t0) * PN : ck + k * PN;
            /* y_t = S_t C_t + D x_t */
            for (int64_t p = 0; p < P; ++p)
                for (int64_t n = 0; n < N; ++n)
                    Gb[p * N + n] += dyt[p] * Ct[n];
            double *dCt = dC_h + t * N, *dBt = dB_h + t * N;
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t p = 0; p < P; ++p)
                    acc += St[p * N + n] * dyt[p];
                dCt[n] = acc;
            }
            for (int64_t p = 0; p < P; ++p)
                dD_acc += dyt[p] * xt[p];
            /* S_t = a_t S_{t-1} + dt_t x_t B_t^T */
            double direct = 0.0, inner = 0.0;
            for (int64_t p = 0; p < P; ++p) {
                double gB = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    gB += Gb[p * N + n] * Bt[n];
                tmpP[p] = gB;
                direct += xt[p] * gB;
                dx[((b * L + t) * H + h) * P + p] = Dh * dyt[p] + d * gB;
            }
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t p = 0; p < P; ++p)
                    acc += Gb[p * N + n] * xt[p];
                dBt[n] = d * acc;
            }
            for (int64_t e = 0; e < PN; ++e)
                inner += Gb[e] * Sp[e];
            ddt[(b * L + t) * H + h] = direct + Ah * decay * inner;
            dA_acc += d * decay * inner;
            for (int64_t e = 0; e < PN; ++e)
                Gb[e] *= decay;
        }
    }
    if (dh0)
        memcpy(dh0 + (b * H + h) * PN, Gb, sizeof(double) * (size_t)PN);
    *dA_bh = dA_acc;
    *dD_bh = dD_acc;
}

/* Whole problem, parallel over (b, h) streams. Per-head dB/dC rows are added into
 * the group's output under a lock; dA/dD are summed over b in a fixed order.
 * seg <= 0 picks 64. Returns 0, or -1 on a bad argument / allocation failure. */
int oracle_ssd_backward(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t G, int64_t N,
                        const double *x, const double *dt, const double *A, const double *Bm,
                        const double *Cm, const double *D, const double *h0, const double *dy,
                        const double *dh_final, double *dx, double *ddt, double *dA, double *dBm,
                        double *dCm, double *dD, double *dh0, int64_t seg, int nthreads)
{
    if (Bsz < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || H % G != 0)
        return -1;
    if (seg <= 0)
        seg = 64;
    const int64_t PN = P * N, nseg = (L + seg - 1) / seg;
    memset(dBm, 0, sizeof(double) * (size_t)(Bsz * L * G * N));
    memset(dCm, 0, sizeof(double) * (size_t)(Bsz * L * G * N));
    double *dA_bh = (double *)calloc((size_t)(Bsz * H) + 1, sizeof(double));
    double *dD_bh = (double *)calloc((size_t)(Bsz * H) + 1, sizeof(double));
    if (!dA_bh || !dD_bh) {
        free(dA_bh);
        free(dD_bh);
        return -1;
    }
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *ck = (double *)malloc(sizeof(double) * (size_t)((nseg + 1) * PN));
        double *ss = (double *)malloc(sizeof(double) * (size_t)((seg > 1 ? seg : 1) * PN + PN));
        double *Gb = (double *)malloc(sizeof(double) * (size_t)PN);
        double *tmpP = (double *)malloc(sizeof(double) * (size_t)P);
        double *dB_h = (double *)malloc(sizeof(double) * (size_t)(L * N + 1));
        double *dC_h = (double *)malloc(sizeof(double) * (size_t)(L * N + 1));
        const int ok = ck && ss && Gb && tmpP && dB_h && dC_h;
        if (!ok) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < Bsz * H; ++bh) {
            if (!ok)
                continue;
            const int64_t b = bh / H, h = bh % H, g = h / (H / G);
            ssd_stream_bwd(b, h, L, H, P, G, N, seg, x, dt, A, Bm, Cm, D, h0, dy, dh_final, dx, ddt,
                           dB_h, dC_h, dh0, dA_bh + bh, dD_bh + bh, ck, ss, Gb, tmpP);
#pragma omp critical(ssd_oracle_group_sum)
            for (int64_t t = 0; t < L; ++t) {
                double *ob = dBm + ((b * L + t) * G + g) * N, *oc = dCm + ((b * L + t) * G + g) * N;
                for (int64_t n = 0; n < N; ++n) {
                    ob[n] += dB_h[t * N + n];
                    oc[n] += dC_h[t * N + n];
                }
            }
        }
        free(ck);
        free(ss);
        free(Gb);
        free(tmpP);
        free(dB_h);
        free(dC_h);
    }
    for (int64_t h = 0; h < H; ++h) {
        double sa = 0.0, sd = 0.0;
        for (int64_t b = 0; b < Bsz; ++b) {
            sa += dA_bh[b * H + h];
            sd += dD_bh[b * H + h];
        }
        dA[h] = sa;
        if (dD)
            dD[h] = sd;
    }
    free(dA_bh);
    free(dD_bh);
    return err;
}
