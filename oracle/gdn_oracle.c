/*
 * Oracle for the gated delta-rule layer: plain fp64 token-by-token recurrence
 * and its reverse-time adjoint.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes (StateFlow, arXiv 2608.06838, section 2.1, the generic
 * linear recurrence S_t = S_{t-1} F_t + v_t k_t^T, y_t = S_t q_t, with the
 * Gated DeltaNet transition "scalar-plus-low-rank" named in the same section),
 * written in the transposed orientation, state S in R^{dk x dv}:
 *
 *     alpha_t = exp(g_t)
 *     S_t     = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t     = scale * S_t^T q_t
 *     S_out   = S_T
 *
 * and, when the beta path is off (the scalar-identity transition of Mamba-2,
 * same section):  S_t = alpha_t S_{t-1} + k_t v_t^T.
 *
 * The backward pass differentiates the scalar
 *     L = sum_t <o_t, dO_t> + <S_out, dS_out>
 * by walking time in reverse with the adjoint D_t = dL/dS_t:
 *     D_t   = carry + scale * q_t dO_t^T          (carry starts at dS_out)
 *     dq_t  = scale * S_t dO_t
 *     dv_t  = beta_t D_t^T k_t
 *     dk_t  = beta_t D_t v_t - alpha_t beta_t (D_t S_{t-1}^T k_t + S_{t-1} D_t^T k_t)
 *     dbeta = k_t^T D_t (v_t - alpha_t S_{t-1}^T k_t)
 *     dg_t  = alpha_t (<D_t, S_{t-1}> - beta_t k_t^T D_t S_{t-1}^T k_t)
 *     carry = alpha_t (I - beta_t k_t k_t^T) D_t
 *     dS_in = carry after t = 1
 * (beta path off: dk_t = D_t v_t, dv_t = D_t^T k_t, dg_t = alpha_t <D_t, S_{t-1}>,
 *  carry = alpha_t D_t.)
 * S_{t-1} is recovered by replaying the forward recurrence from a checkpoint
 * stored every `ckpt` tokens.
 *
 * Layouts (all row-major, fp64):
 *   q, k: [B,H,T,dk]   v, o, dO: [B,H,T,dv]   g, beta: [B,H,T]
 *   S_in, S_out, dS_out, dS_in: [B,H,dk,dv]
 * Heads are independent; they are spread over OpenMP threads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One forward step on a single head: S <- alpha (I - beta k k^T) S + beta k v^T
 * (or S <- alpha S + k v^T when has_beta == 0).  tmp has room for dv values. */
static void step_forward(double* S, int dk, int dv, const double* kt, const double* vt,
                         double alpha, double beta, int has_beta, double* tmp) {
    if (has_beta) {
        /* tmp = S^T k */
        for (int b = 0; b < dv; ++b) tmp[b] = 0.0;
        for (int a = 0; a < dk; ++a) {
            const double ka = kt[a];
            const double* Sa = S + (size_t)a * dv;
            for (int b = 0; b < dv; ++b) tmp[b] += ka * Sa[b];
        }
        for (int a = 0; a < dk; ++a) {
            const double ka = kt[a];
            double* Sa = S + (size_t)a * dv;
            for (int b = 0; b < dv; ++b)
                Sa[b] = alpha * (Sa[b] - beta * ka * tmp[b]) + beta * ka * vt[b];
        }
    } else {
        for (int a = 0; a < dk; ++a) {
            const double ka = kt[a];
            double* Sa = S + (size_t)a * dv;
            for (int b = 0; b < dv; ++b) Sa[b] = alpha * Sa[b] + ka * vt[b];
        }
    }
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_gdn_fwd(int B, int H, int T, int dk, int dv, const double* q, const double* k,
                   const double* v, const double* g, const double* beta, const double* S_in,
                   double scale, double* o, double* S_out) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return 1;
    const int BH = B * H;
    const int has_beta = beta != NULL;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!S || !tmp) {
            free(S);
            free(tmp);
#pragma omp atomic write
            err = 2;
            continue;
        }
        if (S_in)
            memcpy(S, S_in + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t = 0; t < T; ++t) {
            const size_t row = (size_t)bh * T + t;
            const double* qt = q + row * dk;
            const double* kt = k + row * dk;
            const double* vt = v + row * dv;
            const double alpha = exp(g[row]);
            const double bt = has_beta ? beta[row] : 0.0;
            step_forward(S, dk, dv, kt, vt, alpha, bt, has_beta, tmp);
            double* ot = o + row * dv;
            for (int b = 0; b < dv; ++b) ot[b] = 0.0;
            for (int a = 0; a < dk; ++a) {
                const double qa = qt[a];
                const double* Sa = S + (size_t)a * dv;
                for (int b = 0; b < dv; ++b) ot[b] += qa * Sa[b];
            }
            for (int b = 0; b < dv; ++b) ot[b] *= scale;
        }
        if (S_out) memcpy(S_out + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(tmp);
    }
    return err;
}

int oracle_gdn_bwd(int B, int H, int T, int dk, int dv, const double* q, const double* k,
                   const double* v, const double* g, const double* beta, const double* S_in,
                   double scale, const double* dO, const double* dS_out, double* dq,
                   double* dk_out, double* dv_out, double* dg, double* dbeta, double* dS_in,
                   int ckpt) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || ckpt <= 0) return 1;
    const int BH = B * H;
    const int has_beta = beta != NULL;
    const size_t SS = (size_t)dk * dv;
    const int nwin = (T + ckpt - 1) / ckpt;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        /* checkpoints: ck[w] = S before token w*ckpt */
        double* ck = (double*)malloc(sizeof(double) * SS * (size_t)(nwin > 0 ? nwin : 1));
        /* window states: win[j] = S after token (w*ckpt + j - 1); win[0] = checkpoint */
        double* win = (double*)malloc(sizeof(double) * SS * (size_t)(ckpt + 1));
        double* D = (double*)malloc(sizeof(double) * SS);
        double* carry = (double*)malloc(sizeof(double) * SS);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv) * 4);
        if (!ck || !win || !D || !carry || !tmp) {
            free(ck); free(win); free(D); free(carry); free(tmp);
#pragma omp atomic write
            err = 2;
            continue;
        }
        double* S = win; /* scratch for the checkpoint pass */
        if (S_in)
            memcpy(S, S_in + (size_t)bh * SS, sizeof(double) * SS);
        else
            memset(S, 0, sizeof(double) * SS);
        for (int t = 0; t < T; ++t) {
            if (t % ckpt == 0) memcpy(ck + (size_t)(t / ckpt) * SS, S, sizeof(double) * SS);
            const size_t row = (size_t)bh * T + t;
            step_forward(S, dk, dv, k + row * dk, v + row * dv, exp(g[row]),
                         has_beta ? beta[row] : 0.0, has_beta, tmp);
        }
        if (dS_out)
            memcpy(carry, dS_out + (size_t)bh * SS, sizeof(double) * SS);
        else
            memset(carry, 0, sizeof(double) * SS);

        double* Dv = tmp;          /* D v        (dk) */
        double* DTk = tmp + dk;    /* D^T k      (dv) */
        double* Spk = DTk + dv;    /* S_{t-1}^T k (dv) ; reused */
        for (int w = nwin - 1; w >= 0; --w) {
            const int t0 = w * ckpt;
            const int t1 = (t0 + ckpt < T) ? t0 + ckpt : T;
            memcpy(win, ck + (size_t)w * SS, sizeof(double) * SS);
            for (int t = t0; t < t1; ++t) {
                const size_t row = (size_t)bh * T + t;
                double* nxt = win + (size_t)(t - t0 + 1) * SS;
                memcpy(nxt, win + (size_t)(t - t0) * SS, sizeof(double) * SS);
                step_forward(nxt, dk, dv, k + row * dk, v + row * dv, exp(g[row]),
                             has_beta ? beta[row] : 0.0, has_beta, DTk);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const size_t row = (size_t)bh * T + t;
                const double* qt = q + row * dk;
                const double* kt = k + row * dk;
                const double* vt = v + row * dv;
                const double* dOt = dO + row * dv;
                const double alpha = exp(g[row]);
                const double bt = has_beta ? beta[row] : 0.0;
                const double* Sprev = win + (size_t)(t - t0) * SS;
                const double* Scur = win + (size_t)(t - t0 + 1) * SS;

                /* D = carry + scale q dO^T */
                for (int a = 0; a < dk; ++a)
                    for (int b = 0; b < dv; ++b)
                        D[(size_t)a * dv + b] = carry[(size_t)a * dv + b] + scale * qt[a] * dOt[b];

                /* dq = scale S_t dO */
                double* dqt = dq + row * dk;
                for (int a = 0; a < dk; ++a) {
                    double s = 0.0;
                    for (int b = 0; b < dv; ++b) s += Scur[(size_t)a * dv + b] * dOt[b];
                    dqt[a] = scale * s;
                }
                /* Dv = D v ; DTk = D^T k */
                for (int a = 0; a < dk; ++a) {
                    double s = 0.0;
                    for (int b = 0; b < dv; ++b) s += D[(size_t)a * dv + b] * vt[b];
                    Dv[a] = s;
                }
                for (int b = 0; b < dv; ++b) DTk[b] = 0.0;
                for (int a = 0; a < dk; ++a)
                    for (int b = 0; b < dv; ++b) DTk[b] += D[(size_t)a * dv + b] * kt[a];
                /* <D, S_{t-1}> */
                double DS = 0.0;
                for (size_t e = 0; e < SS; ++e) DS += D[e] * Sprev[e];

                double* dkt = dk_out + row * dk;
                double* dvt = dv_out + row * dv;
                if (has_beta) {
                    /* Spk = S_{t-1}^T k */
                    for (int b = 0; b < dv; ++b) Spk[b] = 0.0;
                    for (int a = 0; a < dk; ++a)
                        for (int b = 0; b < dv; ++b) Spk[b] += Sprev[(size_t)a * dv + b] * kt[a];
                    /* k^T D S_{t-1}^T k = (D^T k) . (S_{t-1}^T k) */
                    double kDSk = 0.0, kDv = 0.0;
                    for (int b = 0; b < dv; ++b) kDSk += DTk[b] * Spk[b];
                    for (int b = 0; b < dv; ++b) kDv += DTk[b] * vt[b];
                    for (int b = 0; b < dv; ++b) dvt[b] = bt * DTk[b];
                    /* dk = beta D v - alpha beta (D S_{t-1}^T k + S_{t-1} D^T k) */
                    for (int a = 0; a < dk; ++a) {
                        double s1 = 0.0, s2 = 0.0;
                        for (int b = 0; b < dv; ++b) {
                            s1 += D[(size_t)a * dv + b] * Spk[b];
                            s2 += Sprev[(size_t)a * dv + b] * DTk[b];
                        }
                        dkt[a] = bt * Dv[a] - alpha * bt * (s1 + s2);
                    }
                    dbeta[row] = kDv - alpha * kDSk;
                    dg[row] = alpha * (DS - bt * kDSk);
                    /* carry = alpha (I - beta k k^T) D = alpha (D - beta k (D^T k)^T) */
                    for (int a = 0; a < dk; ++a)
                        for (int b = 0; b < dv; ++b)
                            carry[(size_t)a * dv + b] =
                                alpha * (D[(size_t)a * dv + b] - bt * kt[a] * DTk[b]);
                } else {
                    for (int b = 0; b < dv; ++b) dvt[b] = DTk[b];
                    for (int a = 0; a < dk; ++a) dkt[a] = Dv[a];
                    dg[row] = alpha * DS;
                    if (dbeta) dbeta[row] = 0.0;
                    for (size_t e = 0; e < SS; ++e) carry[e] = alpha * D[e];
                }
            }
        }
        memcpy(dS_in + (size_t)bh * SS, carry, sizeof(double) * SS);
        free(ck); free(win); free(D); free(carry); free(tmp);
    }
    return err;
}
