/*
 * wkv_oracle.c -- plain, slow, double-precision CPU oracle for the RWKV WKV operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only the test suite, the package's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library; the two meet only in the seeded inputs they both consume.
 *
 * All arithmetic is in double.  Arrays are row-major:
 *   r, k, v, w, y, dy, dr, dk, dv, dw : [B][T][C]   (C = H * N, channel c = h*N + i)
 *   u, du                             : [C]
 * For RWKV-6 the argument w is the log-decay ew (<= 0); the per-step decay of
 * state row i is d_t[i] = exp(ew_t[i]), i.e. exp(-exp(w_raw)).
 *
 * Sources (page title, section):
 *  - "How the WKV (Weighted Key Value) Mechanism in RWKV Processes Images",
 *    CUDA Wrapper (Image Side): the kernel is handed ew = -exp(w).
 *  - "How Custom CUDA Kernels (wkv6_cuda.cu) Implement the WKV Operation",
 *    Forward Pass Implementation: a future-to-past pass without the bonus u and
 *    a past-to-future pass that adds y += r*(u*x + s); state update s = s*w + x
 *    with x = k*v; Backward Pass Gradient Computation: gradients of r, k, v, u, w.
 *  - "RWKV Architecture: How Receptance Weighted Key Value Combines RNN Linear
 *    Inference with Transformer Parallel Training": RWKV-5 matrix state
 *    S_t = diag(decay) S_{t-1} + k_t^T v_t; RWKV-6 data-dependent decay w_t;
 *    RWKV-4 recurrent formulation (a_t, b_t) and its ratio WKV_t.
 *  - yarian.com RWKV overview, section 3.2: time decay handled in log space to
 *    avoid underflow (the max-shift state p of the RWKV-4 recurrence).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define IDX(b, t, c) (((size_t)(b) * (size_t)T + (size_t)(t)) * (size_t)C + (size_t)(c))

/* ------------------------------------------------------------------------ */
/* RWKV-6 forward.                                                            */
/* Causal (RWKV Architecture page, RWKV-5/RWKV-6 matrix state; wkv6_cuda page,  */
/* past-to-future pass):                                                       */
/*   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),  S_t = diag(d_t) S_{t-1} + k_t^T v_t */
/* with S_{-1} = 0.  Bidirectional (wkv6_cuda page, Future-to-Past Pass): first */
/* a sweep t = T-1 .. 0 that reads y_t += r_t S^b and then updates            */
/* S^b = diag(d_t) S^b + k_t^T v_t (no bonus), then the causal sweep is added.  */
/* ------------------------------------------------------------------------ */
static void wkv6_head_sweep(int T, int C, int N, int b, int h, int reverse, int bonus,
                            const double *r, const double *k, const double *v,
                            const double *w, const double *u, double *y, double *S, double *M,
                            const double *s_init)
{
    /* S starts as s_init (N x N) or zero; on return it holds the state after the sweep */
    if (s_init) memcpy(S, s_init, sizeof(double) * (size_t)N * N);
    else memset(S, 0, sizeof(double) * (size_t)N * N);
    for (int step = 0; step < T; ++step) {
        const int t = reverse ? (T - 1 - step) : step;
        const double *rt = r + IDX(b, t, h * N);
        const double *kt = k + IDX(b, t, h * N);
        const double *vt = v + IDX(b, t, h * N);
        const double *wt = w + IDX(b, t, h * N);
        double *yt = y + IDX(b, t, h * N);
        /* M = S (+ diag(u) k_t^T v_t when the bonus applies) */
        for (int i = 0; i < N; ++i)
            for (int j = 0; j < N; ++j) {
                double m = S[i * N + j];
                if (bonus) m += u[h * N + i] * kt[i] * vt[j];
                M[i * N + j] = m;
            }
        /* y_t += r_t M */
        for (int j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int i = 0; i < N; ++i) acc += rt[i] * M[i * N + j];
            yt[j] += acc;
        }
        /* S = diag(exp(ew_t)) S + k_t^T v_t */
        for (int i = 0; i < N; ++i) {
            const double d = exp(wt[i]);
            for (int j = 0; j < N; ++j) S[i * N + j] = d * S[i * N + j] + kt[i] * vt[j];
        }
    }
}

int oracle_wkv6_fwd(int B, int T, int C, int H, int bidirectional,
                    const double *r, const double *k, const double *v, const double *w,
                    const double *u, double *y)
{
    if (B < 0 || T < 0 || H < 1 || C % H != 0) return -1;
    const int N = C / H;
    memset(y, 0, sizeof(double) * (size_t)B * T * C);
    double *S = (double *)malloc(sizeof(double) * (size_t)N * N);
    double *M = (double *)malloc(sizeof(double) * (size_t)N * N);
    if (!S || !M) { free(S); free(M); return -2; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            if (bidirectional) wkv6_head_sweep(T, C, N, b, h, 1, 0, r, k, v, w, u, y, S, M, NULL);
            wkv6_head_sweep(T, C, N, b, h, 0, 1, r, k, v, w, u, y, S, M, NULL);
        }
    free(S);
    free(M);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Causal RWKV-6 forward carrying the state across calls (RWKV Architecture   */
/* page, Recurrent Inference Formulation: the N x N state is all that a step  */
/* needs from the past, so a sequence may be processed in pieces).  The same */
/* recurrence as above with S_{-1} = s0 instead of 0:                          */
/*   s0 : [B][H][N][N] (row i = key channel, column j = value channel), or     */
/*        NULL for the zero state;                                             */
/*   sT : [B][H][N][N] receives S_{T-1} (s0 itself when T = 0), or NULL.       */
/* ------------------------------------------------------------------------ */
int oracle_wkv6_fwd_state(int B, int T, int C, int H, const double *r, const double *k,
                          const double *v, const double *w, const double *u, const double *s0,
                          double *y, double *sT)
{
    if (B < 0 || T < 0 || H < 1 || C % H != 0) return -1;
    const int N = C / H;
    const size_t NN = (size_t)N * N;
    memset(y, 0, sizeof(double) * (size_t)B * T * C);
    double *S = (double *)malloc(sizeof(double) * NN);
    double *M = (double *)malloc(sizeof(double) * NN);
    if (!S || !M) { free(S); free(M); return -2; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t off = ((size_t)b * H + h) * NN;
            wkv6_head_sweep(T, C, N, b, h, 0, 1, r, k, v, w, u, y, S, M, s0 ? s0 + off : NULL);
            if (sT) memcpy(sT + off, S, sizeof(double) * NN);
        }
    free(S);
    free(M);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RWKV-6 backward (wkv6_cuda page, Backward Pass Gradient Computation: the  */
/* gradients of r, k, v, u and w).  Plain reverse-mode differentiation of the */
/* forward above, with every state stored:                                    */
/*   causal: Sf[t] = S_{t-1}; the adjoint A_t = dL/dS_t obeys                 */
/*     A_{T-1} = 0,  A_{t-1} = r_t dy_t^T + diag(d_t) A_t                     */
/*   and per step                                                            */
/*     dr_t = (S_{t-1} + diag(u) k_t^T v_t) dy_t                              */
/*     dk_t = A_t v_t + u . r_t (v_t . dy_t)                                  */
/*     dv_t = A_t^T k_t + (sum_i r_t u k_t) dy_t                               */
/*     du  += r_t . k_t (v_t . dy_t)                                          */
/*     dw_t = d_t . sum_j S_{t-1}[i][j] A_t[i][j]    (d = exp(ew))            */
/*   anti-causal sweep (bidirectional only): Sb[t] = S^b_{t+1} is read by y_t, */
/*   its adjoint Ab_t = dL/dS^b_t obeys Ab_0 = 0,                             */
/*     Ab_{t+1} = r_t dy_t^T + diag(d_t) Ab_t, and                            */
/*     dr_t += S^b_{t+1} dy_t, dk_t += Ab_t v_t, dv_t += Ab_t^T k_t,          */
/*     dw_t += d_t . sum_j S^b_{t+1}[i][j] Ab_t[i][j].                         */
/* ------------------------------------------------------------------------ */
int oracle_wkv6_bwd(int B, int T, int C, int H, int bidirectional,
                    const double *r, const double *k, const double *v, const double *w,
                    const double *u, const double *dy,
                    double *dr, double *dk, double *dv, double *dw, double *du)
{
    if (B < 0 || T < 0 || H < 1 || C % H != 0) return -1;
    const int N = C / H;
    const size_t NN = (size_t)N * N;
    memset(dr, 0, sizeof(double) * (size_t)B * T * C);
    memset(dk, 0, sizeof(double) * (size_t)B * T * C);
    memset(dv, 0, sizeof(double) * (size_t)B * T * C);
    memset(dw, 0, sizeof(double) * (size_t)B * T * C);
    memset(du, 0, sizeof(double) * (size_t)C);
    if (T == 0) return 0;
    /* states[t] for t = 0..T: causal uses states[t] = S_{t-1}; the anti-causal
       sweep reuses the buffer with states[t] = S^b_{t+1}. */
    double *states = (double *)malloc(sizeof(double) * NN * (size_t)(T + 1));
    double *A = (double *)malloc(sizeof(double) * NN);
    if (!states || !A) { free(states); free(A); return -2; }

    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            /* ---- causal part ---- */
            memset(states, 0, sizeof(double) * NN);
            for (int t = 0; t < T; ++t) {
                const double *kt = k + IDX(b, t, h * N), *vt = v + IDX(b, t, h * N);
                const double *wt = w + IDX(b, t, h * N);
                const double *Sp = states + NN * (size_t)t;
                double *Sn = states + NN * (size_t)(t + 1);
                for (int i = 0; i < N; ++i) {
                    const double d = exp(wt[i]);
                    for (int j = 0; j < N; ++j) Sn[i * N + j] = d * Sp[i * N + j] + kt[i] * vt[j];
                }
            }
            memset(A, 0, sizeof(double) * NN);
            for (int t = T - 1; t >= 0; --t) {
                const double *rt = r + IDX(b, t, h * N), *kt = k + IDX(b, t, h * N);
                const double *vt = v + IDX(b, t, h * N), *wt = w + IDX(b, t, h * N);
                const double *gt = dy + IDX(b, t, h * N);
                const double *Sp = states + NN * (size_t)t; /* S_{t-1} */
                double *drt = dr + IDX(b, t, h * N), *dkt = dk + IDX(b, t, h * N);
                double *dvt = dv + IDX(b, t, h * N), *dwt = dw + IDX(b, t, h * N);
                double vdy = 0.0, ruk = 0.0;
                for (int j = 0; j < N; ++j) vdy += vt[j] * gt[j];
                for (int i = 0; i < N; ++i) ruk += rt[i] * u[h * N + i] * kt[i];
                for (int i = 0; i < N; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < N; ++j) acc += (Sp[i * N + j] + u[h * N + i] * kt[i] * vt[j]) * gt[j];
                    drt[i] += acc;
                    double acck = 0.0, accw = 0.0;
                    for (int j = 0; j < N; ++j) {
                        acck += A[i * N + j] * vt[j];
                        accw += Sp[i * N + j] * A[i * N + j];
                    }
                    dkt[i] += acck + u[h * N + i] * rt[i] * vdy;
                    dwt[i] += exp(wt[i]) * accw;
                    du[h * N + i] += rt[i] * kt[i] * vdy;
                }
                for (int j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < N; ++i) acc += A[i * N + j] * kt[i];
                    dvt[j] += acc + ruk * gt[j];
                }
                /* A_{t-1} = r_t dy_t^T + diag(d_t) A_t */
                for (int i = 0; i < N; ++i) {
                    const double d = exp(wt[i]);
                    for (int j = 0; j < N; ++j) A[i * N + j] = rt[i] * gt[j] + d * A[i * N + j];
                }
            }
            if (!bidirectional) continue;
            /* ---- anti-causal part: states[t] = S^b_{t+1} for t = 0..T-1 ----
               S^b_T = 0, and S^b_t = diag(d_t) S^b_{t+1} + k_t^T v_t for t = T-1 .. 1. */
            memset(states + NN * (size_t)(T - 1), 0, sizeof(double) * NN);
            for (int t = T - 1; t >= 1; --t) {
                const double *kt = k + IDX(b, t, h * N), *vt = v + IDX(b, t, h * N);
                const double *wt = w + IDX(b, t, h * N);
                const double *Sp = states + NN * (size_t)t;       /* S^b_{t+1} */
                double *Sn = states + NN * (size_t)(t - 1);       /* S^b_t     */
                for (int i = 0; i < N; ++i) {
                    const double d = exp(wt[i]);
                    for (int j = 0; j < N; ++j) Sn[i * N + j] = d * Sp[i * N + j] + kt[i] * vt[j];
                }
            }
            memset(A, 0, sizeof(double) * NN); /* Ab_0 = 0 */
            for (int t = 0; t < T; ++t) {
                const double *rt = r + IDX(b, t, h * N), *kt = k + IDX(b, t, h * N);
                const double *vt = v + IDX(b, t, h * N), *wt = w + IDX(b, t, h * N);
                const double *gt = dy + IDX(b, t, h * N);
                const double *Sb = states + NN * (size_t)t; /* S^b_{t+1} */
                double *drt = dr + IDX(b, t, h * N), *dkt = dk + IDX(b, t, h * N);
                double *dvt = dv + IDX(b, t, h * N), *dwt = dw + IDX(b, t, h * N);
                for (int i = 0; i < N; ++i) {
                    double accr = 0.0, acck = 0.0, accw = 0.0;
                    for (int j = 0; j < N; ++j) {
                        accr += Sb[i * N + j] * gt[j];
                        acck += A[i * N + j] * vt[j];
                        accw += Sb[i * N + j] * A[i * N + j];
                    }
                    drt[i] += accr;
                    dkt[i] += acck;
                    dwt[i] += exp(wt[i]) * accw;
                }
                for (int j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < N; ++i) acc += A[i * N + j] * kt[i];
                    dvt[j] += acc;
                }
                /* Ab_{t+1} = r_t dy_t^T + diag(d_t) Ab_t */
                for (int i = 0; i < N; ++i) {
                    const double d = exp(wt[i]);
                    for (int j = 0; j < N; ++j) A[i * N + j] = rt[i] * gt[j] + d * A[i * N + j];
                }
            }
        }
    free(states);
    free(A);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RWKV-6 forward with its decay prologue and its norm/gate epilogue          */
/* (RWKV Architecture page, RWKV-6 "Finch": w_t = w_base + tanh(x_t W1) W2;    */
/* RWKV-5 "Eagle": group normalisation over each head, SiLU output gating;    */
/* WKV processing-images page: the kernel is handed ew = -exp(w), and the     */
/* block passes the WKV output and the gate g on to its output stage).        */
/* The dense projections stay outside: the inputs are ww = tanh(x W1) W2 and  */
/* g = silu(x W_g), both [B][T][C].  Per (b, t, head h), with y the RWKV-6     */
/* output at ew = -exp(w_base + ww):                                          */
/*   mu = mean_i y[h*N+i],  var = mean_i (y[h*N+i] - mu)^2                    */
/*   out[c] = ((y[c] - mu) / sqrt(var + eps) * gn_w[c] + gn_b[c]) * g[c]      */
/* ------------------------------------------------------------------------ */
int oracle_wkv6_fwd_fused(int B, int T, int C, int H, int bidirectional,
                          const double *r, const double *k, const double *v, const double *ww,
                          const double *w_base, const double *u, const double *g,
                          const double *gn_w, const double *gn_b, double eps, double *out)
{
    if (B < 0 || T < 0 || H < 1 || C % H != 0) return -1;
    const int N = C / H;
    const size_t n = (size_t)B * T * C;
    double *ew = (double *)malloc(sizeof(double) * (n ? n : 1));
    double *y = (double *)malloc(sizeof(double) * (n ? n : 1));
    if (!ew || !y) { free(ew); free(y); return -2; }
    for (size_t e = 0; e < n; ++e) ew[e] = -exp(w_base[e % C] + ww[e]);
    int rc = oracle_wkv6_fwd(B, T, C, H, bidirectional, r, k, v, ew, u, y);
    if (rc == 0)
        for (size_t row = 0; row < (size_t)B * T; ++row)
            for (int h = 0; h < H; ++h) {
                const double *yh = y + row * C + (size_t)h * N;
                double mu = 0.0, var = 0.0;
                for (int i = 0; i < N; ++i) mu += yh[i];
                mu /= N;
                for (int i = 0; i < N; ++i) var += (yh[i] - mu) * (yh[i] - mu);
                var /= N;
                const double inv = 1.0 / sqrt(var + eps);
                for (int i = 0; i < N; ++i) {
                    const size_t c = (size_t)h * N + i;
                    out[row * C + c] = ((yh[i] - mu) * inv * gn_w[c] + gn_b[c]) * g[row * C + c];
                }
            }
    free(ew);
    free(y);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* RWKV-5 forward (RWKV Architecture page, RWKV-5 "Eagle": the matrix state   */
/* decays by the static, per-channel factor exp(-w), S_t = exp(-w) . S_{t-1}  */
/* + k_t^T v_t).  The readout is RWKV-6's with that constant decay:           */
/*   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),  S_{-1} = 0,                     */
/* w : [C], w >= 0 (decay exp(-w) of state row i = channel h*N + i).         */
/* ------------------------------------------------------------------------ */
int oracle_wkv5_fwd(int B, int T, int C, int H, const double *r, const double *k, const double *v,
                    const double *w, const double *u, double *y)
{
    if (B < 0 || T < 0 || H < 1 || C % H != 0) return -1;
    const int N = C / H;
    double *S = (double *)malloc(sizeof(double) * (size_t)N * N);
    if (!S) return -2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            memset(S, 0, sizeof(double) * (size_t)N * N);
            for (int t = 0; t < T; ++t) {
                const double *rt = r + IDX(b, t, h * N), *kt = k + IDX(b, t, h * N);
                const double *vt = v + IDX(b, t, h * N);
                double *yt = y + IDX(b, t, h * N);
                for (int j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < N; ++i)
                        acc += rt[i] * (S[i * N + j] + u[h * N + i] * kt[i] * vt[j]);
                    yt[j] = acc;
                }
                for (int i = 0; i < N; ++i) {
                    const double d = exp(-w[h * N + i]);
                    for (int j = 0; j < N; ++j) S[i * N + j] = d * S[i * N + j] + kt[i] * vt[j];
                }
            }
        }
    free(S);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RWKV-5 backward: reverse-mode differentiation of oracle_wkv5_fwd, with    */
/* every state stored.  The adjoint A_t = dL/dS_t obeys A_{T-1} = 0 and      */
/* A_{t-1} = r_t dy_t^T + exp(-w) . A_t; per step                            */
/*   dr_t = (S_{t-1} + diag(u) k_t^T v_t) dy_t                                */
/*   dk_t = A_t v_t + u . r_t (v_t . dy_t)                                    */
/*   dv_t = A_t^T k_t + (sum_i r_t u k_t) dy_t                                 */
/*   du  += r_t . k_t (v_t . dy_t)                                            */
/* and, since dS_t/dw = -exp(-w) . S_{t-1} row by row,                        */
/*   dw  -= exp(-w) . sum_j S_{t-1}[i][j] A_t[i][j]   (summed over b and t).  */
/* ------------------------------------------------------------------------ */
int oracle_wkv5_bwd(int B, int T, int C, int H, const double *r, const double *k, const double *v,
                    const double *w, const double *u, const double *dy,
                    double *dr, double *dk, double *dv, double *dw, double *du)
{
    if (B < 0 || T < 0 || H < 1 || C % H != 0) return -1;
    const int N = C / H;
    const size_t NN = (size_t)N * N;
    memset(dw, 0, sizeof(double) * (size_t)C);
    memset(du, 0, sizeof(double) * (size_t)C);
    if (T == 0) return 0;
    double *states = (double *)malloc(sizeof(double) * NN * (size_t)(T + 1));
    double *A = (double *)malloc(sizeof(double) * NN);
    if (!states || !A) { free(states); free(A); return -2; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const double *uh = u + h * N, *wh = w + h * N;
            memset(states, 0, sizeof(double) * NN);
            for (int t = 0; t < T; ++t) {   /* states[t + 1] = S_t */
                const double *kt = k + IDX(b, t, h * N), *vt = v + IDX(b, t, h * N);
                for (int i = 0; i < N; ++i)
                    for (int j = 0; j < N; ++j)
                        states[NN * (t + 1) + i * N + j] = exp(-wh[i]) * states[NN * t + i * N + j] + kt[i] * vt[j];
            }
            memset(A, 0, sizeof(double) * NN);
            for (int t = T - 1; t >= 0; --t) {
                const double *rt = r + IDX(b, t, h * N), *kt = k + IDX(b, t, h * N);
                const double *vt = v + IDX(b, t, h * N), *gt = dy + IDX(b, t, h * N);
                const double *Sp = states + NN * t;
                double vdy = 0.0, ruk = 0.0;
                for (int j = 0; j < N; ++j) vdy += vt[j] * gt[j];
                for (int i = 0; i < N; ++i) ruk += rt[i] * uh[i] * kt[i];
                for (int i = 0; i < N; ++i) {
                    double accr = 0.0, acck = 0.0, accw = 0.0;
                    for (int j = 0; j < N; ++j) {
                        accr += (Sp[i * N + j] + uh[i] * kt[i] * vt[j]) * gt[j];
                        acck += A[i * N + j] * vt[j];
                        accw += Sp[i * N + j] * A[i * N + j];
                    }
                    dr[IDX(b, t, h * N + i)] = accr;
                    dk[IDX(b, t, h * N + i)] = acck + uh[i] * rt[i] * vdy;
                    dw[h * N + i] -= exp(-wh[i]) * accw;
                    du[h * N + i] += rt[i] * kt[i] * vdy;
                }
                for (int j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < N; ++i) acc += A[i * N + j] * kt[i];
                    dv[IDX(b, t, h * N + j)] = acc + ruk * gt[j];
                }
                for (int i = 0; i < N; ++i)
                    for (int j = 0; j < N; ++j) A[i * N + j] = rt[i] * gt[j] + exp(-wh[i]) * A[i * N + j];
            }
        }
    free(states);
    free(A);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RWKV-4 forward (RWKV Architecture page, The Recurrent Inference            */
/* Formulation):                                                             */
/*   WKV_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t})                */
/*   a_t = e^{-w} a_{t-1} + e^{k_t} v_t,  b_t = e^{-w} b_{t-1} + e^{k_t}       */
/* with a_{-1} = b_{-1} = 0, carried in log space (yarian.com overview, 3.2): */
/* the stored pair (a, b) is scaled by e^{-p}, where p is the running maximum */
/* exponent; the scale cancels in the ratio.  w > 0 per channel.             */
/* ------------------------------------------------------------------------ */
int oracle_wkv4_fwd(int B, int T, int C, const double *k, const double *v, const double *w,
                    const double *u, double *y)
{
    if (B < 0 || T < 0 || C < 0) return -1;
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < C; ++c) {
            double a = 0.0, bb = 0.0, p = -INFINITY;
            for (int t = 0; t < T; ++t) {
                const double kt = k[IDX(b, t, c)], vt = v[IDX(b, t, c)];
                /* output: shift by q = max(p, u + k_t) */
                double q = fmax(p, u[c] + kt);
                double e1 = exp(p - q), e2 = exp(u[c] + kt - q);
                y[IDX(b, t, c)] = (e1 * a + e2 * vt) / (e1 * bb + e2);
                /* state: decay by e^{-w}, add e^{k_t}; new shift q = max(p - w, k_t) */
                q = fmax(p - w[c], kt);
                e1 = exp(p - w[c] - q);
                e2 = exp(kt - q);
                a = e1 * a + e2 * vt;
                bb = e1 * bb + e2;
                p = q;
            }
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RWKV-4 backward: gradients of L = sum_t dy_t . y_t for oracle_wkv4_fwd,     */
/* written from the ratio-of-sums definition (RWKV Architecture page, The     */
/* Fundamental Mathematical Duality: WKV_t = N_t / D_t with                   */
/*   N_t = sum_{s<t} E_ts v_s + E_tt v_t,  D_t = sum_{s<t} E_ts + E_tt,        */
/*   E_ts = e^{k_s - (t-1-s) w} for s < t,  E_tt = e^{u + k_t}).              */
/* Differentiating the ratio, with g_t = dy_t / D_t:                          */
/*   dv_s += g_t E_ts,   dk_s += g_t E_ts (v_s - y_t)         (s <= t)         */
/*   du   += g_t E_tt (v_t - y_t)                                             */
/*   dw   -= g_t (t-1-s) E_ts (v_s - y_t)                     (s < t)          */
/* Every E_ts and D_t of step t is scaled by e^{-m_t}, m_t the largest exponent */
/* of the step, which cancels in g_t E_ts (the log-space shift of the forward). */
/* O(T^2) per channel: a plain evaluation of the definition.                  */
/*   dk, dv : [B][T][C];  dw, du : [C], summed over B and T.                  */
/* ------------------------------------------------------------------------ */
int oracle_wkv4_bwd(int B, int T, int C, const double *k, const double *v, const double *w,
                    const double *u, const double *dy, double *dk, double *dv, double *dw, double *du)
{
    if (B < 0 || T < 0 || C < 0) return -1;
    memset(dk, 0, sizeof(double) * (size_t)B * T * C);
    memset(dv, 0, sizeof(double) * (size_t)B * T * C);
    memset(dw, 0, sizeof(double) * (size_t)C);
    memset(du, 0, sizeof(double) * (size_t)C);
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < C; ++c)
            for (int t = 0; t < T; ++t) {
                const double kt = k[IDX(b, t, c)], vt = v[IDX(b, t, c)];
                /* the step's largest exponent */
                double m = u[c] + kt;
                for (int s = 0; s < t; ++s) m = fmax(m, k[IDX(b, s, c)] - (t - 1 - s) * w[c]);
                /* N_t, D_t (scaled by e^{-m}) and y_t */
                const double ett = exp(u[c] + kt - m);
                double D = ett, N = ett * vt;
                for (int s = 0; s < t; ++s) {
                    const double e = exp(k[IDX(b, s, c)] - (t - 1 - s) * w[c] - m);
                    D += e;
                    N += e * v[IDX(b, s, c)];
                }
                const double yt = N / D, g = dy[IDX(b, t, c)] / D;
                /* the bonus term s = t */
                dv[IDX(b, t, c)] += g * ett;
                dk[IDX(b, t, c)] += g * ett * (vt - yt);
                du[c] += g * ett * (vt - yt);
                /* the decayed past s < t */
                for (int s = 0; s < t; ++s) {
                    const double vs = v[IDX(b, s, c)];
                    const double e = exp(k[IDX(b, s, c)] - (t - 1 - s) * w[c] - m);
                    dv[IDX(b, s, c)] += g * e;
                    dk[IDX(b, s, c)] += g * e * (vs - yt);
                    dw[c] -= (t - 1 - s) * g * e * (vs - yt);
                }
            }
    return 0;
}
