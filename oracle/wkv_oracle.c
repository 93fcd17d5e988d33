/*
 * wkv_oracle.c -- plain, slow, fp64 CPU reference for the WKV recurrences.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file: it exists so that the tests, the smoke check and the bench's CPU
 * baseline can compare the CUDA kernels against an obviously correct
 * evaluation. It shares no code, header or constant with the CUDA sources.
 *
 * What it computes (every function below cites the definition it follows):
 *
 *  RWKV-4 WKV (the operator that RWKV_TimeMix.forward calls as
 *  RUN_CUDA(B, T, C, time_decay, time_first, k, v) on the RWKV-LM v4 code
 *  walkthrough page "代码连连看——RWKV", section RWKV_TimeMix), per channel c with
 *  decay rate w = exp(time_decay) > 0 and bonus u = time_first:
 *
 *      a_t = sum_{i<t} e^{-(t-1-i) w + k_i} v_i        b_t = sum_{i<t} e^{-(t-1-i) w + k_i}
 *      y_t = (a_t + e^{u+k_t} v_t) / (b_t + e^{u+k_t})
 *
 *  evaluated by the plain linear recurrence a <- e^{-w} a + e^{k} v,
 *  b <- e^{-w} b + e^{k}. To stay inside fp64 range every lane first subtracts
 *  its largest key K* = max_t k_t from all keys: numerator and denominator are
 *  both multiplied by e^{-K*}, so y is unchanged (an exact identity). This
 *  oracle does NOT use the running-max (aa, bb, pp) form.
 *
 *  RWKV-4 WKV backward: the chain rule of the definition above, written out
 *  with stored per-step a_t, b_t, D_t = b_t + e^{u+k_t}, y_t.
 *
 *  RWKV-6 head-state WKV (the RWKV6_OP operator of the rwkv-ops package page,
 *  section "rwkv6op 使用方法", call and argument tables), per head with key
 *  index i and value index j:
 *
 *      o_t[j]    = sum_i r_t[i] * ( S_{t-1}[i][j] + u[i] k_t[i] v_t[j] )
 *      S_t[i][j] = w_t[i] * S_{t-1}[i][j] + k_t[i] v_t[j]
 *
 *  with S_{-1} = 0 or a caller-given initial state, and its backward (the
 *  chain rule with G_t = dL/dS_t walked down).
 *
 *  RWKV-7 generalized delta rule (generalized_delta_rule / rwkv7_op of the
 *  rwkv-ops package page; the page gives the interface, the recurrence is
 *  the diagonal-plus-rank-one transition written at oracle_wkv7_forward):
 *
 *      S_t = (diag(e^{w_t}) + b_t a_t^T) S_{t-1} + k_t^T v_t,    o_t = r_t S_t
 *
 *  and its backward (the page's generalized_delta_rule carries gradients;
 *  its _inference twin does not): the chain rule with G_t = dL/dS_t walked
 *  down, every S_t stored.
 *
 *  Time-shift mix (the prologue of RWKV_TimeMix.jit_func on the same RWKV-4
 *  page): the input shifted one token along T blended per channel with the
 *  token itself, once for each of k, v, r, and its backward.
 *
 * Layouts: activations [B][T][C] row-major, C fastest. All inputs are fp64
 * (the Python wrapper widens float32 / bf16 inputs exactly).
 * Parallelism: OpenMP over independent lanes / heads only; every lane's
 * arithmetic is sequential in t and identical to the single-thread order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <stdio.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the parallel loops that follow (timing only: the loops are over
 * independent lanes/heads, so the results do not depend on it). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

static int all_finite(const double *x, int64_t n) {
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(x[i])) return 0;
    return 1;
}

/* ------------------------------------------------------------------------ */
/* RWKV-4 forward                                                            */
/* ------------------------------------------------------------------------ */

/*
 * y[B][T][C] from w[C], u[C], k[B][T][C], v[B][T][C].
 * Optional outputs (pass NULL to skip), each [B][C]:
 *   a_end, b_end : a_T and b_T multiplied by e^{-K*}  (the state after the
 *                  last token, in the shifted scale)
 *   kmax         : K* = max_t k_t of the lane
 * Returns 0 on success, 1 if any produced value is not finite.
 */
int oracle_wkv4_forward(int64_t B, int64_t T, int64_t C,
                        const double *w, const double *u,
                        const double *k, const double *v, double *y,
                        double *a_end, double *b_end, double *kmax)
{
    int bad = 0;
    #pragma omp parallel for collapse(2) schedule(static) reduction(|:bad)
    for (int64_t bi = 0; bi < B; ++bi) {
        for (int64_t c = 0; c < C; ++c) {
            const int64_t base = bi * T * C + c;
            double K = -INFINITY;
            for (int64_t t = 0; t < T; ++t) {
                double kt = k[base + t * C];
                if (kt > K) K = kt;
            }
            if (T == 0) K = 0.0;
            const double decay = exp(-w[c]);          /* e^{-w} */
            double a = 0.0, b = 0.0;                   /* a_0 = b_0 = 0 */
            for (int64_t t = 0; t < T; ++t) {
                const int64_t idx = base + t * C;
                const double ek = exp(k[idx] - K);           /* e^{k_t}   (shifted) */
                const double eu = exp(u[c] + k[idx] - K);    /* e^{u+k_t} (shifted) */
                const double yt = (a + eu * v[idx]) / (b + eu);
                if (!isfinite(yt)) bad = 1;
                y[idx] = yt;
                a = decay * a + ek * v[idx];                 /* a_{t+1} */
                b = decay * b + ek;                          /* b_{t+1} */
            }
            if (a_end) a_end[bi * C + c] = a;
            if (b_end) b_end[bi * C + c] = b;
            if (kmax) kmax[bi * C + c] = K;
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* RWKV-4 backward                                                           */
/* ------------------------------------------------------------------------ */

/*
 * Gradients of L = sum_t gy_t . y_t with respect to k, v (per element) and
 * w, u (per channel, summed over the batch and time).
 *
 * Derivation (D_t = b_t + e^{u+k_t}, y_t as in the forward):
 *   direct terms of token t    rho_t = e^{u+k_t} / D_t
 *                              dy_t/dv_t = rho_t,  dy_t/dk_t = rho_t (v_t - y_t),
 *                              dy_t/du   = rho_t (v_t - y_t)
 *   through the past sums      dy_t/da_t = 1/D_t,  dy_t/db_t = -y_t/D_t
 *   alpha_t = gy_t / D_t,  beta_t = gy_t y_t / D_t
 *   A_i = sum_{t>i} alpha_t e^{-(t-1-i) w},  B_i likewise with beta
 *     gv_i += e^{k_i} A_i,   gk_i += e^{k_i} (v_i A_i - B_i)
 *   w enters only through a_t, b_t:  da_{t+1}/dw = e^{-w} (da_t/dw - a_t)
 *     gw = sum_t alpha_t da_t/dw - beta_t db_t/dw          (forward form)
 *   and, independently, with A'_i = sum_{t>i} (t-1-i) alpha_t e^{-(t-1-i) w}
 *     gw = -sum_i e^{k_i} (v_i A'_i - B'_i)                 (reverse form)
 *
 * gk, gv: [B][T][C]. gw, gu: [C]. gw_rev (nullable): [C], the reverse-form gw,
 * returned only so the two derivations can be checked against each other.
 * Per-lane sums are added over the batch in increasing b.
 */
int oracle_wkv4_backward(int64_t B, int64_t T, int64_t C,
                         const double *w, const double *u,
                         const double *k, const double *v, const double *gy,
                         double *gk, double *gv, double *gw, double *gu,
                         double *gw_rev)
{
    int bad = 0;
    double *lane_gw = (double *)calloc((size_t)(B * C) + 1, sizeof(double));
    double *lane_gu = (double *)calloc((size_t)(B * C) + 1, sizeof(double));
    double *lane_gwr = (double *)calloc((size_t)(B * C) + 1, sizeof(double));
    if (!lane_gw || !lane_gu || !lane_gwr) {
        free(lane_gw); free(lane_gu); free(lane_gwr);
        return 2;
    }

    #pragma omp parallel reduction(|:bad)
    {
        double *D = (double *)malloc(sizeof(double) * (size_t)(T + 1));
        double *Y = (double *)malloc(sizeof(double) * (size_t)(T + 1));
        if (!D || !Y) bad = 2;
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi) {
            for (int64_t c = 0; c < C; ++c) {
                if (!D || !Y) continue;
                const int64_t base = bi * T * C + c;
                double K = -INFINITY;
                for (int64_t t = 0; t < T; ++t)
                    if (k[base + t * C] > K) K = k[base + t * C];
                if (T == 0) K = 0.0;
                const double decay = exp(-w[c]);
                double a = 0.0, b = 0.0, da = 0.0, db = 0.0;
                double s_gw = 0.0, s_gu = 0.0;
                /* forward sweep: outputs, direct gradient terms, gw forward form */
                for (int64_t t = 0; t < T; ++t) {
                    const int64_t idx = base + t * C;
                    const double ek = exp(k[idx] - K);
                    const double eu = exp(u[c] + k[idx] - K);
                    const double Dt = b + eu;
                    const double yt = (a + eu * v[idx]) / Dt;
                    D[t] = Dt;
                    Y[t] = yt;
                    const double rho = eu / Dt;
                    gv[idx] = gy[idx] * rho;
                    gk[idx] = gy[idx] * rho * (v[idx] - yt);
                    s_gu += gy[idx] * rho * (v[idx] - yt);
                    const double alpha = gy[idx] / Dt;
                    const double beta = gy[idx] * yt / Dt;
                    s_gw += alpha * da - beta * db;
                    const double da_next = decay * (da - a);
                    const double db_next = decay * (db - b);
                    a = decay * a + ek * v[idx];
                    b = decay * b + ek;
                    da = da_next;
                    db = db_next;
                }
                /* reverse sweep: contributions through the future sums */
                double A = 0.0, Bs = 0.0, Ap = 0.0, Bp = 0.0, s_gwr = 0.0;
                for (int64_t i = T - 1; i >= 0; --i) {
                    const int64_t idx = base + i * C;
                    const double ek = exp(k[idx] - K);
                    /* A, Bs hold A_i, B_i; Ap, Bp hold A'_i, B'_i */
                    gv[idx] += ek * A;
                    gk[idx] += ek * (v[idx] * A - Bs);
                    s_gwr -= ek * (v[idx] * Ap - Bp);
                    const double alpha = gy[idx] / D[i];
                    const double beta = gy[idx] * Y[i] / D[i];
                    const double Ap_next = decay * (Ap + A);
                    const double Bp_next = decay * (Bp + Bs);
                    A = alpha + decay * A;
                    Bs = beta + decay * Bs;
                    Ap = Ap_next;
                    Bp = Bp_next;
                }
                lane_gw[bi * C + c] = s_gw;
                lane_gu[bi * C + c] = s_gu;
                lane_gwr[bi * C + c] = s_gwr;
            }
        }
        free(D);
        free(Y);
    }
    if (bad) {
        free(lane_gw); free(lane_gu); free(lane_gwr);
        return bad;
    }
    for (int64_t c = 0; c < C; ++c) {
        double sw = 0.0, su = 0.0, swr = 0.0;
        for (int64_t bi = 0; bi < B; ++bi) {
            sw += lane_gw[bi * C + c];
            su += lane_gu[bi * C + c];
            swr += lane_gwr[bi * C + c];
        }
        gw[c] = sw;
        gu[c] = su;
        if (gw_rev) gw_rev[c] = swr;
    }
    free(lane_gw); free(lane_gu); free(lane_gwr);
    if (!all_finite(gk, B * T * C) || !all_finite(gv, B * T * C) ||
        !all_finite(gw, C) || !all_finite(gu, C))
        return 1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RWKV-6 head-state forward                                                 */
/* ------------------------------------------------------------------------ */

/*
 * r, k, v, w: [B][T][H*K] (w is the per-step decay in (0, 1]); u: [H*K].
 * init_state (nullable): [n_state][H][K][K], indexed [.][h][i][j] with i the
 *   key index and j the value index. Sample b starts from
 *   init_state[state_map[b]] when state_map is given, else from
 *   init_state[0] when n_state == 1, else from init_state[b] (n_state == B).
 *   Without init_state every sample starts from S = 0.
 * o: [B][T][H*K].  final_state (nullable): [B][H][K][K], S after the last token.
 * The value dimension equals the key dimension (K), as in the package's
 * (num_heads, head_size, head_size) state shape.
 * Returns 0 on success, 1 on a non-finite output, 3 on a bad state index.
 */
int oracle_wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t K,
                        const double *r, const double *k, const double *v,
                        const double *w, const double *u,
                        const double *init_state, const int32_t *state_map,
                        int64_t n_state, double *o, double *final_state)
{
    const int64_t HK = H * K;
    int bad = 0;
    #pragma omp parallel reduction(|:bad)
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)(K * K));
        if (!S) bad = 2;
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi) {
            for (int64_t h = 0; h < H; ++h) {
                if (!S) continue;
                if (init_state) {
                    int64_t sidx;
                    if (state_map) sidx = state_map[bi];
                    else sidx = (n_state == 1) ? 0 : bi;
                    if (sidx < 0 || sidx >= n_state) { bad |= 3; continue; }
                    memcpy(S, init_state + (sidx * H + h) * K * K,
                           sizeof(double) * (size_t)(K * K));
                } else {
                    memset(S, 0, sizeof(double) * (size_t)(K * K));
                }
                for (int64_t t = 0; t < T; ++t) {
                    const int64_t row = (bi * T + t) * HK + h * K;
                    /* output uses S_{t-1} plus the bonus of the current token */
                    for (int64_t j = 0; j < K; ++j) {
                        double acc = 0.0;
                        for (int64_t i = 0; i < K; ++i)
                            acc += r[row + i] * (S[i * K + j] + u[h * K + i] * k[row + i] * v[row + j]);
                        o[row + j] = acc;
                        if (!isfinite(acc)) bad |= 1;
                    }
                    /* then the state absorbs the current token */
                    for (int64_t i = 0; i < K; ++i)
                        for (int64_t j = 0; j < K; ++j)
                            S[i * K + j] = w[row + i] * S[i * K + j] + k[row + i] * v[row + j];
                }
                if (final_state)
                    memcpy(final_state + (bi * H + h) * K * K, S,
                           sizeof(double) * (size_t)(K * K));
            }
        }
        free(S);
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* RWKV-6 head-state backward                                                */
/* ------------------------------------------------------------------------ */

/*
 * Gradients of L = sum(o * do) + sum(final_state * g_final) for the forward
 * above (RWKV6_OP is a trainable operator: the rwkv-ops package page lists
 * its PyTorch CUDA backward). The chain rule of the recurrence, written out
 * with G_t = dL/dS_t walked from the last token back:
 *
 *   G_{T-1} = g_final (or 0),   G_{t-1} = diag(w_t) G_t + r_t^T do_t
 *   gr_t[i] = sum_j S_{t-1}[i][j] do_t[j] + u[i] k_t[i] (v_t . do_t)
 *   gk_t[i] = sum_j G_t[i][j] v_t[j]     + u[i] r_t[i] (v_t . do_t)
 *   gv_t[j] = sum_i k_t[i] G_t[i][j]     + (sum_i r_t[i] u[i] k_t[i]) do_t[j]
 *   gw_t[i] = sum_j G_t[i][j] S_{t-1}[i][j]
 *   gu[i]  += r_t[i] k_t[i] (v_t . do_t)          (summed over samples, tokens)
 *   g_init  = G_{-1}                                 (per sample: [B][H][K][K])
 *
 * Every S_{t-1} of a (sample, head) is kept (T * K * K doubles), so this is
 * only for the test sizes. g_final, g_init may be NULL. gu gets the sum over
 * samples and tokens, added per (sample, head) in a fixed order.
 * Returns 0 on success, 1 on a non-finite result, 2 when out of memory,
 * 3 on a bad state index.
 */
int oracle_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t K,
                         const double *r, const double *k, const double *v,
                         const double *w, const double *u,
                         const double *init_state, const int32_t *state_map,
                         int64_t n_state, const double *dout, const double *g_final,
                         double *gr, double *gk, double *gv, double *gw,
                         double *gu, double *g_init)
{
    const int64_t HK = H * K;
    int bad = 0;
    double *gu_part = (double *)calloc((size_t)(B * HK), sizeof(double));
    if (!gu_part) return 2;
    #pragma omp parallel reduction(|:bad)
    {
        double *Sh = (double *)malloc(sizeof(double) * (size_t)((T + 1) * K * K));
        double *G = (double *)malloc(sizeof(double) * (size_t)(K * K));
        if (!Sh || !G) bad |= 2;
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi) {
            for (int64_t h = 0; h < H; ++h) {
                if (!Sh || !G) continue;
                /* forward: Sh[t] = S_{t-1} */
                if (init_state) {
                    int64_t sidx;
                    if (state_map) sidx = state_map[bi];
                    else sidx = (n_state == 1) ? 0 : bi;
                    if (sidx < 0 || sidx >= n_state) { bad |= 3; continue; }
                    memcpy(Sh, init_state + (sidx * H + h) * K * K, sizeof(double) * (size_t)(K * K));
                } else {
                    memset(Sh, 0, sizeof(double) * (size_t)(K * K));
                }
                for (int64_t t = 0; t < T; ++t) {
                    const int64_t row = (bi * T + t) * HK + h * K;
                    const double *S = Sh + t * K * K;
                    double *Sn = Sh + (t + 1) * K * K;
                    for (int64_t i = 0; i < K; ++i)
                        for (int64_t j = 0; j < K; ++j)
                            Sn[i * K + j] = w[row + i] * S[i * K + j] + k[row + i] * v[row + j];
                }
                /* reverse */
                if (g_final)
                    memcpy(G, g_final + (bi * H + h) * K * K, sizeof(double) * (size_t)(K * K));
                else
                    memset(G, 0, sizeof(double) * (size_t)(K * K));
                double *gup = gu_part + bi * HK + h * K;
                for (int64_t t = T - 1; t >= 0; --t) {
                    const int64_t row = (bi * T + t) * HK + h * K;
                    const double *S = Sh + t * K * K; /* S_{t-1} */
                    double vdo = 0.0, rku = 0.0;
                    for (int64_t j = 0; j < K; ++j) vdo += v[row + j] * dout[row + j];
                    for (int64_t i = 0; i < K; ++i) rku += r[row + i] * u[h * K + i] * k[row + i];
                    for (int64_t i = 0; i < K; ++i) {
                        double a = 0.0, b = 0.0, c = 0.0;
                        for (int64_t j = 0; j < K; ++j) {
                            a += S[i * K + j] * dout[row + j];
                            b += G[i * K + j] * v[row + j];
                            c += G[i * K + j] * S[i * K + j];
                        }
                        gr[row + i] = a + u[h * K + i] * k[row + i] * vdo;
                        gk[row + i] = b + u[h * K + i] * r[row + i] * vdo;
                        gw[row + i] = c;
                        gup[i] += r[row + i] * k[row + i] * vdo;
                    }
                    for (int64_t j = 0; j < K; ++j) {
                        double a = 0.0;
                        for (int64_t i = 0; i < K; ++i) a += k[row + i] * G[i * K + j];
                        gv[row + j] = a + rku * dout[row + j];
                    }
                    /* G_{t-1} = diag(w_t) G_t + r_t^T do_t */
                    for (int64_t i = 0; i < K; ++i)
                        for (int64_t j = 0; j < K; ++j)
                            G[i * K + j] = w[row + i] * G[i * K + j] + r[row + i] * dout[row + j];
                }
                if (g_init)
                    memcpy(g_init + (bi * H + h) * K * K, G, sizeof(double) * (size_t)(K * K));
            }
        }
        free(Sh);
        free(G);
    }
    for (int64_t c = 0; c < HK; ++c) {
        double s = 0.0;
        for (int64_t bi = 0; bi < B; ++bi) s += gu_part[bi * HK + c];
        gu[c] = s;
    }
    free(gu_part);
    const int64_t n = B * T * HK;
    if (!all_finite(gr, n) || !all_finite(gk, n) || !all_finite(gv, n) || !all_finite(gw, n) ||
        !all_finite(gu, HK))
        bad |= 1;
    return bad;
}

/* ------------------------------------------------------------------------ */
/* RWKV-7 generalized delta rule, forward                                    */
/* ------------------------------------------------------------------------ */

/*
 * generalized_delta_rule(r, w, k, v, a, b, initial_state, output_final_state)
 * of the rwkv-ops package page (section on rwkv7_op / generalized_delta_rule):
 * inputs [B][T][H][K] (w the decay in log space), state [N][H][K][V] with
 * N = B sequences, outputs o [B][T][H][V] and the final state. The page
 * prints the interface only; the recurrence taken is the plain
 * diagonal-plus-rank-one state transition of a "generalized delta rule",
 * per head with key index j and value index i (V = K here):
 *
 *   sa[i]     = sum_j a_t[j] S_{t-1}[j][i]
 *   S_t[j][i] = e^{w_t[j]} S_{t-1}[j][i] + b_t[j] sa[i] + k_t[j] v_t[i]
 *   o_t[i]    = sum_j r_t[j] S_t[j][i]          (the state after the token)
 *
 * i.e. S_t = (diag(e^{w_t}) + b_t a_t^T) S_{t-1} + k_t^T v_t, o_t = r_t S_t.
 * r, w, k, v, a, b: [B][T][H*K]; init_state (nullable): [B][H][K][K] indexed
 * [b][h][j][i]; o: [B][T][H*K]; final_state (nullable): [B][H][K][K].
 * Returns 0 on success, 1 on a non-finite output, 2 on allocation failure.
 */
int oracle_wkv7_forward(int64_t B, int64_t T, int64_t H, int64_t K,
                        const double *r, const double *w, const double *k, const double *v,
                        const double *a, const double *b, const double *init_state,
                        double *o, double *final_state)
{
    const int64_t HK = H * K;
    int bad = 0;
    #pragma omp parallel reduction(|:bad)
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)(K * K));
        double *sa = (double *)malloc(sizeof(double) * (size_t)K);
        if (!S || !sa) bad = 2;
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi) {
            for (int64_t h = 0; h < H; ++h) {
                if (!S || !sa) continue;
                if (init_state)
                    memcpy(S, init_state + (bi * H + h) * K * K, sizeof(double) * (size_t)(K * K));
                else
                    memset(S, 0, sizeof(double) * (size_t)(K * K));
                for (int64_t t = 0; t < T; ++t) {
                    const int64_t row = (bi * T + t) * HK + h * K;
                    for (int64_t i = 0; i < K; ++i) {
                        double acc = 0.0;
                        for (int64_t j = 0; j < K; ++j) acc += a[row + j] * S[j * K + i];
                        sa[i] = acc;
                    }
                    for (int64_t j = 0; j < K; ++j) {
                        const double d = exp(w[row + j]);
                        for (int64_t i = 0; i < K; ++i)
                            S[j * K + i] = d * S[j * K + i] + b[row + j] * sa[i] + k[row + j] * v[row + i];
                    }
                    for (int64_t i = 0; i < K; ++i) {
                        double acc = 0.0;
                        for (int64_t j = 0; j < K; ++j) acc += r[row + j] * S[j * K + i];
                        o[row + i] = acc;
                        if (!isfinite(acc)) bad |= 1;
                    }
                }
                if (final_state)
                    memcpy(final_state + (bi * H + h) * K * K, S, sizeof(double) * (size_t)(K * K));
            }
        }
        free(S);
        free(sa);
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* RWKV-7 generalized delta rule, backward                                   */
/* ------------------------------------------------------------------------ */

/*
 * Gradients of L = sum_t sum_i dout_t[i] o_t[i] + sum g_final o S_{T-1} for
 * the forward above (g_final nullable: 0). With G = dL/dS_t, per token from
 * the last one down (j the key index, i the value index, d = e^{w_t}):
 *
 *   G[j][i]  += r_t[j] dout_t[i]                    (o_t reads S_t)
 *   dr_t[j]   = sum_i S_t[j][i] dout_t[i]
 *   dv_t[i]   = sum_j k_t[j] G[j][i]
 *   dk_t[j]   = sum_i G[j][i] v_t[i]
 *   db_t[j]   = sum_i G[j][i] sa[i]
 *   dsa[i]    = sum_j b_t[j] G[j][i]
 *   dw_t[j]   = d[j] sum_i G[j][i] S_{t-1}[j][i]     (w is the log decay)
 *   da_t[j]   = sum_i S_{t-1}[j][i] dsa[i]           (sa = a_t S_{t-1})
 *   G[j][i]  <- d[j] G[j][i] + a_t[j] dsa[i]         (G becomes dL/dS_{t-1})
 *
 * and d_init = G after token 0. Shapes as for oracle_wkv7_forward; dout,
 * dr, dw, dk, dv, da, db [B][T][H*K]; init_state, g_final, d_init
 * [B][H][K][K] (init_state, g_final nullable; d_init written).
 * Returns 0 on success, 1 on a non-finite result, 2 on allocation failure.
 */
int oracle_wkv7_backward(int64_t B, int64_t T, int64_t H, int64_t K,
                         const double *r, const double *w, const double *k, const double *v,
                         const double *a, const double *b, const double *init_state,
                         const double *dout, const double *g_final,
                         double *dr, double *dw, double *dk, double *dv, double *da, double *db,
                         double *d_init)
{
    const int64_t HK = H * K, KK = K * K;
    int bad = 0;
    #pragma omp parallel reduction(|:bad)
    {
        double *Sh = (double *)malloc(sizeof(double) * (size_t)((T + 1) * KK));  /* Sh[t] = S_{t-1} */
        double *SA = (double *)malloc(sizeof(double) * (size_t)(T * K));         /* sa of every token */
        double *G = (double *)malloc(sizeof(double) * (size_t)KK);
        double *dsa = (double *)malloc(sizeof(double) * (size_t)K);
        if (!Sh || !SA || !G || !dsa) bad = 2;
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi) {
            for (int64_t h = 0; h < H; ++h) {
                if (!Sh || !SA || !G || !dsa) continue;
                const double *S0 = init_state ? init_state + (bi * H + h) * KK : NULL;
                for (int64_t e = 0; e < KK; ++e) Sh[e] = S0 ? S0[e] : 0.0;
                /* forward, keeping every state */
                for (int64_t t = 0; t < T; ++t) {
                    const int64_t row = (bi * T + t) * HK + h * K;
                    const double *S = Sh + t * KK;
                    double *Sn = Sh + (t + 1) * KK;
                    for (int64_t i = 0; i < K; ++i) {
                        double proj = 0.0;
                        for (int64_t j = 0; j < K; ++j) proj += a[row + j] * S[j * K + i];
                        SA[t * K + i] = proj;
                    }
                    for (int64_t j = 0; j < K; ++j)
                        for (int64_t i = 0; i < K; ++i)
                            Sn[j * K + i] = exp(w[row + j]) * S[j * K + i] + b[row + j] * SA[t * K + i]
                                            + k[row + j] * v[row + i];
                }
                /* reverse */
                const double *GF = g_final ? g_final + (bi * H + h) * KK : NULL;
                for (int64_t e = 0; e < KK; ++e) G[e] = GF ? GF[e] : 0.0;
                for (int64_t t = T - 1; t >= 0; --t) {
                    const int64_t row = (bi * T + t) * HK + h * K;
                    const double *Sp = Sh + t * KK;        /* S_{t-1} */
                    const double *St = Sh + (t + 1) * KK;  /* S_t */
                    const double *sa = SA + t * K;
                    for (int64_t j = 0; j < K; ++j)
                        for (int64_t i = 0; i < K; ++i) G[j * K + i] += r[row + j] * dout[row + i];
                    for (int64_t j = 0; j < K; ++j) {
                        double sr = 0.0, sk = 0.0, sb = 0.0, sw = 0.0;
                        for (int64_t i = 0; i < K; ++i) {
                            sr += St[j * K + i] * dout[row + i];
                            sk += G[j * K + i] * v[row + i];
                            sb += G[j * K + i] * sa[i];
                            sw += G[j * K + i] * Sp[j * K + i];
                        }
                        dr[row + j] = sr;
                        dk[row + j] = sk;
                        db[row + j] = sb;
                        dw[row + j] = exp(w[row + j]) * sw;
                    }
                    for (int64_t i = 0; i < K; ++i) {
                        double sv = 0.0, ss = 0.0;
                        for (int64_t j = 0; j < K; ++j) {
                            sv += k[row + j] * G[j * K + i];
                            ss += b[row + j] * G[j * K + i];
                        }
                        dv[row + i] = sv;
                        dsa[i] = ss;
                    }
                    for (int64_t j = 0; j < K; ++j) {
                        double s = 0.0;
                        for (int64_t i = 0; i < K; ++i) s += Sp[j * K + i] * dsa[i];
                        da[row + j] = s;
                    }
                    for (int64_t j = 0; j < K; ++j)
                        for (int64_t i = 0; i < K; ++i)
                            G[j * K + i] = exp(w[row + j]) * G[j * K + i] + a[row + j] * dsa[i];
                }
                memcpy(d_init + (bi * H + h) * KK, G, sizeof(double) * (size_t)KK);
                if (!all_finite(G, KK)) bad |= 1;
            }
        }
        free(Sh);
        free(SA);
        free(G);
        free(dsa);
    }
    if (!bad) {
        const int64_t n = B * T * HK;
        if (!all_finite(dr, n) || !all_finite(dw, n) || !all_finite(dk, n) || !all_finite(dv, n) ||
            !all_finite(da, n) || !all_finite(db, n))
            bad = 1;
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* Time-shift mix (time-mix prologue)                                        */
/* ------------------------------------------------------------------------ */

/*
 * RWKV_TimeMix.jit_func ("代码连连看——RWKV", section RWKV_TimeMix): time_shift
 * is ZeroPad2d((0, 0, 1, -1)) on [B][T][C], i.e. one row of zeros padded
 * before T and the last row cut, so row t of the shifted input xx is row t-1
 * of x and row 0 is zero. Each of k, v, r then takes
 *
 *     x_m,t = x_t * mix_m + xx_t * (1 - mix_m)        (mix_m = time_mix_{k,v,r})
 *
 * x_prev [B][C] (may be NULL: zeros) replaces the zero row, so that a
 * sequence cut into pieces gives the same result as one call (the RNN form
 * carries the last token as state).
 * mix [n_mix][C]; out [n_mix][B][T][C]. Returns 0, or 1 if a value is not finite.
 */
int oracle_time_shift_mix(int64_t B, int64_t T, int64_t C, int64_t n_mix,
                          const double *x, const double *mix, const double *x_prev,
                          double *out)
{
    int bad = 0;
    for (int64_t m = 0; m < n_mix; ++m)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t t = 0; t < T; ++t)
                for (int64_t c = 0; c < C; ++c) {
                    const double xt = x[(bi * T + t) * C + c];
                    double xx = 0.0;
                    if (t > 0)
                        xx = x[(bi * T + t - 1) * C + c];
                    else if (x_prev)
                        xx = x_prev[bi * C + c];
                    const double o = xt * mix[m * C + c] + xx * (1.0 - mix[m * C + c]);
                    out[((m * B + bi) * T + t) * C + c] = o;
                    if (!isfinite(o)) bad = 1;
                }
    return bad;
}

/*
 * Gradients of L = sum_m sum(g_m * x_m) for the time-shift mix above, by
 * scattering each output's two partial derivatives to their inputs:
 *   d x_m,t / d x_t     = mix_m
 *   d x_m,t / d xx_t    = 1 - mix_m   (xx_t = x_{t-1}, or x_prev at t = 0)
 *   d x_m,t / d mix_m   = x_t - xx_t
 * g [n_mix][B][T][C]; gx [B][T][C]; gmix [n_mix][C] (summed over b, t);
 * gx_prev [B][C] (may be NULL; written only if given).
 */
int oracle_time_shift_mix_backward(int64_t B, int64_t T, int64_t C, int64_t n_mix,
                                   const double *x, const double *mix, const double *x_prev,
                                   const double *g, double *gx, double *gmix, double *gx_prev)
{
    memset(gx, 0, sizeof(double) * (size_t)(B * T * C));
    memset(gmix, 0, sizeof(double) * (size_t)(n_mix * C));
    if (gx_prev) memset(gx_prev, 0, sizeof(double) * (size_t)(B * C));
    for (int64_t m = 0; m < n_mix; ++m)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t t = 0; t < T; ++t)
                for (int64_t c = 0; c < C; ++c) {
                    const double gm = g[((m * B + bi) * T + t) * C + c];
                    const double mc = mix[m * C + c];
                    const double xt = x[(bi * T + t) * C + c];
                    double xx = 0.0;
                    if (t > 0)
                        xx = x[(bi * T + t - 1) * C + c];
                    else if (x_prev)
                        xx = x_prev[bi * C + c];
                    gx[(bi * T + t) * C + c] += gm * mc;
                    if (t > 0)
                        gx[(bi * T + t - 1) * C + c] += gm * (1.0 - mc);
                    else if (gx_prev)
                        gx_prev[bi * C + c] += gm * (1.0 - mc);
                    gmix[m * C + c] += gm * (xt - xx);
                }
    int bad = !all_finite(gx, B * T * C) || !all_finite(gmix, n_mix * C);
    return bad;
}
