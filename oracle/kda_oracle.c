/*
 * KDA oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 token-by-token evaluation of the Kimi Delta Attention
 * recurrence.  Only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark may load this file's library; the product path never does.  It
 * shares no code, header or constant with the CUDA library.
 *
 * What it computes (per sequence n and head h, state S in R^{dk x dv}):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = scale * S_t^T q_t
 *
 * with alpha_t = exp(log_alpha_t) a per-key-channel forget gate.
 * Sources:
 *   - "Kimi Linear ... 深度解读报告" (zako-mio knowledge base), section 2.3
 *     "KDA：逐通道细粒度门控": the three parts of the update -- Diag(alpha_t)
 *     forgets per channel, (I - beta_t k_t k_t^T) erases along the new key,
 *     beta_t k_t v_t^T writes the new value.
 *   - zhaixingw.cn ai-news/151, section "KDA：把遗忘门从一个数变成一串数":
 *     the Gated DeltaNet update S_t = (I - beta k k^T) alpha_t S_{t-1}
 *     + beta k v^T, whose scalar alpha_t KDA replaces by a dk-vector.  The
 *     same page prints a second, transposed variant whose erase term uses the
 *     undecayed state; it contradicts the first formula's order (decay, then
 *     erase) and is not followed here.
 *   - the output is read from the post-update state S_t.
 *
 * The product with (I - beta k k^T) is applied as its rank-one expansion,
 *   (I - beta k k^T) X = X - k (beta k^T X),
 * which is the same matrix product written without forming the dk x dk
 * matrix.  Nothing else is reordered: one token at a time, decay first, then
 * erase and write, then read out.
 *
 * Layouts (all row-major, contiguous):
 *   q, k, log_alpha : [B, T, H, dk]      v : [B, T, H, dv]
 *   beta            : [B, T, H]
 *   initial_state   : [N, H, dk, dv] or NULL (zeros)
 *   out             : [B, T, H, dv]      final_state : [N, H, dk, dv] or NULL
 *   cu_seqlens      : [N + 1] token offsets into the flattened B*T stream, or
 *                     NULL, in which case N == B and sequence n is batch row n.
 * Inputs are fp64 copies of the exact values a GPU run receives.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One (sequence, head) chain over tokens [t0, t1) of the flattened stream. */
static void kda_chain(const double* q, const double* k, const double* v,
                      const double* log_alpha, const double* beta,
                      int64_t t0, int64_t t1, int64_t h, int64_t H,
                      int64_t dk, int64_t dv, double scale,
                      double* S /* [dk][dv], in: S_0, out: S_T */,
                      double* out, double* work /* 2*dv */)
{
    double* u = work;          /* beta (v - S_bar^T k)            */
    double* o = work + dv;     /* S_t^T q                          */
    for (int64_t t = t0; t < t1; ++t) {
        const double* qt = q + (t * H + h) * dk;
        const double* kt = k + (t * H + h) * dk;
        const double* vt = v + (t * H + h) * dv;
        const double* gt = log_alpha + (t * H + h) * dk;
        const double bt = beta[t * H + h];

        /* S_bar = Diag(alpha_t) S_{t-1}: row c scaled by exp(g_c). */
        for (int64_t c = 0; c < dk; ++c) {
            const double a = exp(gt[c]);
            double* row = S + c * dv;
            for (int64_t j = 0; j < dv; ++j) row[j] *= a;
        }
        /* u = beta (v - S_bar^T k)  -- the erase coefficient along k. */
        for (int64_t j = 0; j < dv; ++j) u[j] = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
            const double kc = kt[c];
            const double* row = S + c * dv;
            for (int64_t j = 0; j < dv; ++j) u[j] += row[j] * kc;
        }
        for (int64_t j = 0; j < dv; ++j) u[j] = bt * (vt[j] - u[j]);
        /* S_t = S_bar - beta k k^T S_bar + beta k v^T = S_bar + k u^T. */
        for (int64_t c = 0; c < dk; ++c) {
            const double kc = kt[c];
            double* row = S + c * dv;
            for (int64_t j = 0; j < dv; ++j) row[j] += kc * u[j];
        }
        /* o_t = scale * S_t^T q_t. */
        for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
            const double qc = qt[c];
            const double* row = S + c * dv;
            for (int64_t j = 0; j < dv; ++j) o[j] += row[j] * qc;
        }
        double* ot = out + (t * H + h) * dv;
        for (int64_t j = 0; j < dv; ++j) ot[j] = scale * o[j];
    }
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int kda_oracle_forward(const double* q, const double* k, const double* v,
                       const double* log_alpha, const double* beta,
                       const double* initial_state, const int64_t* cu_seqlens,
                       int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                       int64_t N, double scale,
                       double* out, double* final_state, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !out) return -1;
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || N < 0) return -1;
    if (!cu_seqlens && N != B) return -1;
    if (cu_seqlens) {
        if (B != 1 || cu_seqlens[0] != 0 || cu_seqlens[N] != T) return -1;
        for (int64_t n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    }
    const int64_t units = N * H;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)(dk * dv));
        double* work = (double*)malloc(sizeof(double) * (size_t)(2 * dv));
        if (!S || !work) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int64_t u = 0; u < units; ++u) {
                const int64_t n = u / H, h = u % H;
                const int64_t t0 = cu_seqlens ? cu_seqlens[n] : n * T;
                const int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : (n + 1) * T;
                if (initial_state)
                    memcpy(S, initial_state + u * dk * dv, sizeof(double) * (size_t)(dk * dv));
                else
                    memset(S, 0, sizeof(double) * (size_t)(dk * dv));
                kda_chain(q, k, v, log_alpha, beta, t0, t1, h, H, dk, dv, scale,
                          S, out, work);
                if (final_state)
                    memcpy(final_state + u * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
            }
        }
        free(S);
        free(work);
    }
    return err;
}

/*
 * Backward pass (reverse-mode adjoint of the recurrence above), for training
 * with this operator ("深度解读报告" 3.4: the layer is pre-trained, fine-tuned
 * and trained by RL end to end).  Per
 * chain, from the adjoints dS_T (of the final state) and do_t (of the
 * outputs), one token at a time in reverse order, each forward line of
 * kda_chain differentiated in turn:
 *
 *   o_t = scale S_t^T q_t        dS += scale q_t do_t^T ; dq_t = scale S_t do_t
 *   S_t = S_bar + k u^T          du = dS^T k ; dk_t += dS u ; dS_bar = dS
 *   u = beta (v - S_bar^T k)     dbeta_t = du . (v - S_bar^T k) ; dv_t = beta du ;
 *                                dS_bar -= beta k du^T ; dk_t -= beta S_bar du
 *   S_bar = Diag(e^g) S_{t-1}    dg_t[c] = sum_j dS_bar[c][j] S_bar[c][j] ;
 *                                dS_{t-1} = Diag(e^g) dS_bar
 *
 * S_{t-1} is needed at every step in reverse order.  The chain is run forward
 * once, keeping the state at every kBlock-th token, and each block is run
 * forward again from its checkpoint, keeping all of its states, before its
 * tokens are differentiated: the same operations in the same order as the
 * forward pass, so the recomputed states are the forward's, bit for bit.
 */
enum { kBlock = 32 };

/* S <- one forward step (decay, erase, write) of token t; u and r returned. */
static void kda_step(const double* k, const double* v, const double* log_alpha,
                     const double* beta, int64_t t, int64_t h, int64_t H, int64_t dk,
                     int64_t dv, double* S, double* u, double* r)
{
    const double* kt = k + (t * H + h) * dk;
    const double* vt = v + (t * H + h) * dv;
    const double* gt = log_alpha + (t * H + h) * dk;
    const double bt = beta[t * H + h];
    for (int64_t c = 0; c < dk; ++c) {
        const double a = exp(gt[c]);
        double* row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) row[j] *= a;
    }
    for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        const double kc = kt[c];
        const double* row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) r[j] += row[j] * kc;
    }
    for (int64_t j = 0; j < dv; ++j) {
        r[j] = vt[j] - r[j];
        u[j] = bt * r[j];
    }
    for (int64_t c = 0; c < dk; ++c) {
        const double kc = kt[c];
        double* row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) row[j] += kc * u[j];
    }
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 * d_final_state may be NULL (zero adjoint); d_initial_state may be NULL. */
int kda_oracle_backward(const double* q, const double* k, const double* v,
                        const double* log_alpha, const double* beta,
                        const double* initial_state, const int64_t* cu_seqlens,
                        const double* d_out, const double* d_final_state,
                        int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                        int64_t N, double scale,
                        double* dq, double* dkk, double* dvv, double* dg, double* dbeta,
                        double* d_initial_state, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !d_out || !dq || !dkk || !dvv || !dg || !dbeta)
        return -1;
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || N < 0) return -1;
    if (!cu_seqlens && N != B) return -1;
    if (cu_seqlens) {
        if (B != 1 || cu_seqlens[0] != 0 || cu_seqlens[N] != T) return -1;
        for (int64_t n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    }
    const int64_t units = N * H;
    const int64_t ds = dk * dv;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* dS = (double*)malloc(sizeof(double) * (size_t)ds);
        double* blk = (double*)malloc(sizeof(double) * (size_t)(ds * (kBlock + 1)));
        double* work = (double*)malloc(sizeof(double) * (size_t)(4 * dv));
        double* ckpt = NULL;
        size_t ckpt_cap = 0;
        if (!dS || !blk || !work) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int64_t w = 0; w < units; ++w) {
                const int64_t n = w / H, h = w % H;
                const int64_t t0 = cu_seqlens ? cu_seqlens[n] : n * T;
                const int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : (n + 1) * T;
                const int64_t nb = (t1 - t0 + kBlock - 1) / kBlock;
                if ((size_t)(nb + 1) * (size_t)ds > ckpt_cap) {
                    free(ckpt);
                    ckpt_cap = (size_t)(nb + 1) * (size_t)ds;
                    ckpt = (double*)malloc(sizeof(double) * ckpt_cap);
                    if (!ckpt) {
                        ckpt_cap = 0;
#ifdef _OPENMP
#pragma omp atomic write
#endif
                        err = -2;
                        continue;
                    }
                }
                double* u = work;
                double* r = work + dv;
                double* du = work + 2 * dv;
                /* forward, keeping the state before every block */
                double* S = ckpt;
                if (initial_state)
                    memcpy(S, initial_state + w * ds, sizeof(double) * (size_t)ds);
                else
                    memset(S, 0, sizeof(double) * (size_t)ds);
                for (int64_t b = 0; b < nb; ++b) {
                    double* Sn = ckpt + (b + 1) * ds;
                    memcpy(Sn, ckpt + b * ds, sizeof(double) * (size_t)ds);
                    const int64_t ta = t0 + b * kBlock;
                    const int64_t tb = ta + kBlock < t1 ? ta + kBlock : t1;
                    for (int64_t t = ta; t < tb; ++t)
                        kda_step(k, v, log_alpha, beta, t, h, H, dk, dv, Sn, u, r);
                }
                if (d_final_state)
                    memcpy(dS, d_final_state + w * ds, sizeof(double) * (size_t)ds);
                else
                    memset(dS, 0, sizeof(double) * (size_t)ds);
                for (int64_t b = nb - 1; b >= 0; --b) {
                    const int64_t ta = t0 + b * kBlock;
                    const int64_t tb = ta + kBlock < t1 ? ta + kBlock : t1;
                    /* blk[i] = state before token ta + i; blk[tb - ta] = after */
                    memcpy(blk, ckpt + b * ds, sizeof(double) * (size_t)ds);
                    for (int64_t t = ta; t < tb; ++t) {
                        double* Sn = blk + (t - ta + 1) * ds;
                        memcpy(Sn, blk + (t - ta) * ds, sizeof(double) * (size_t)ds);
                        kda_step(k, v, log_alpha, beta, t, h, H, dk, dv, Sn, u, r);
                    }
                    for (int64_t t = tb - 1; t >= ta; --t) {
                        const double* Sp = blk + (t - ta) * ds;       /* S_{t-1} */
                        const double* St = blk + (t - ta + 1) * ds;   /* S_t     */
                        const double* qt = q + (t * H + h) * dk;
                        const double* kt = k + (t * H + h) * dk;
                        const double* vt = v + (t * H + h) * dv;
                        const double* gt = log_alpha + (t * H + h) * dk;
                        const double bt = beta[t * H + h];
                        const double* dot = d_out + (t * H + h) * dv;
                        double* dqt = dq + (t * H + h) * dk;
                        double* dkt = dkk + (t * H + h) * dk;
                        double* dvt = dvv + (t * H + h) * dv;
                        double* dgt = dg + (t * H + h) * dk;
                        /* output: dS += scale q do^T ; dq = scale S_t do */
                        for (int64_t c = 0; c < dk; ++c) {
                            double acc = 0.0;
                            const double* row = St + c * dv;
                            double* drow = dS + c * dv;
                            for (int64_t j = 0; j < dv; ++j) {
                                acc += row[j] * dot[j];
                                drow[j] += scale * qt[c] * dot[j];
                            }
                            dqt[c] = scale * acc;
                        }
                        /* recompute S_bar, r = v - S_bar^T k, u = beta r */
                        for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
                        for (int64_t c = 0; c < dk; ++c) {
                            const double a = exp(gt[c]);
                            const double* row = Sp + c * dv;
                            for (int64_t j = 0; j < dv; ++j) r[j] += a * row[j] * kt[c];
                        }
                        for (int64_t j = 0; j < dv; ++j) {
                            r[j] = vt[j] - r[j];
                            u[j] = bt * r[j];
                        }
                        /* write: du = dS^T k ; dk = dS u */
                        for (int64_t j = 0; j < dv; ++j) du[j] = 0.0;
                        for (int64_t c = 0; c < dk; ++c) {
                            const double* drow = dS + c * dv;
                            double acc = 0.0;
                            for (int64_t j = 0; j < dv; ++j) {
                                du[j] += drow[j] * kt[c];
                                acc += drow[j] * u[j];
                            }
                            dkt[c] = acc;
                        }
                        /* erase: dbeta, dv, dS_bar -= beta k du^T, dk -= beta S_bar du */
                        double db = 0.0;
                        for (int64_t j = 0; j < dv; ++j) {
                            db += du[j] * r[j];
                            dvt[j] = bt * du[j];
                        }
                        dbeta[t * H + h] = db;
                        for (int64_t c = 0; c < dk; ++c) {
                            const double a = exp(gt[c]);
                            const double* row = Sp + c * dv;
                            double* drow = dS + c * dv;
                            double acc = 0.0, gacc = 0.0;
                            for (int64_t j = 0; j < dv; ++j) {
                                const double sb = a * row[j];
                                acc += sb * du[j];
                                drow[j] -= bt * kt[c] * du[j];
                                gacc += drow[j] * sb;
                            }
                            dkt[c] -= bt * acc;
                            /* decay: dg = sum_j dS_bar S_bar ; dS_{t-1} = e^g dS_bar */
                            dgt[c] = gacc;
                            for (int64_t j = 0; j < dv; ++j) drow[j] *= a;
                        }
                    }
                }
                if (d_initial_state)
                    memcpy(d_initial_state + w * ds, dS, sizeof(double) * (size_t)ds);
            }
        }
        free(dS);
        free(blk);
        free(work);
        free(ckpt);
    }
    return err;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
