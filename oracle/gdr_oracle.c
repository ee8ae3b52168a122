/*
 * gdr_oracle.c -- float64 CPU oracle of the gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (one (batch, head) pair at a time, S in R^{dk x dv}):
 *
 *     S'  = Diag(a_t) S_{t-1}                         decay rows of S
 *     e_t = S'^T k_t                                   what the key reads now
 *     S_t = S' - (b_t * k_t) e_t^T + k_t (w_t * v_t)^T  erase, then write
 *     o_t = S_t^T q_t                                  read with the query
 *
 * Sources for each step:
 *   - the update rule  S_t = (I - k~ k~^T) Diag(alpha_t) S_{t-1} + k~ v~^T
 *     with k~ = sqrt(beta) * k, v~ = sqrt(beta) * v: page "FG^2-GDN: Enhancing
 *     Long-Context Gated Delta Networks with Doubly Fine-Grained Control"
 *     (gist.science 2604.19021), section 2 "Methodology", the FG2-GDN update
 *     rule.  It fixes the order decay -> erase from the decayed state -> write.
 *   - the decoupled erase gate b_t (key side) and write gate w_t (value side),
 *     both per channel, with KDA's per-channel decay: page "Gated DeltaNet-2:
 *     decoupling erase and write in linear attention" (needhelp.icu), section
 *     "Gated DeltaNet-2: the solution", the gates table.
 *   - scalar decay (Gated DeltaNet) versus per-channel decay alpha_t in R^{dk}
 *     (KDA): FG^2-GDN page, section 1 "Problem statement".
 *   - the read-out o_t = S_t^T q_t uses the updated state; the pages print no
 *     output equation, so this is the plain reading of a memory that is read
 *     after it is written.
 *
 * The arithmetic is the definition above written out with plain loops, in
 * double precision, with no blocking and no reordering.  Inputs arrive as
 * float32 arrays (bf16 and fp32 inputs are exact in float32) and are widened
 * to double on read.
 *
 * Layouts (row-major, contiguous):
 *   q, k      [B, T, H, dk]
 *   v         [B, T, H, dv]
 *   a, b      vector gate: [B, T, H, dk]; scalar gate: [B, T, H]; none: NULL (== 1)
 *   w         vector gate: [B, T, H, dv]; scalar gate: [B, T, H]; none: NULL (== 1)
 *   s0, sT    [B, H, dk, dv]   (s0 == NULL means a zero initial state)
 *   o         [B, T, H, dv]
 */
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Gate kinds: the same three cases the recurrence admits. */
enum { ORACLE_GATE_ONE = 0, ORACLE_GATE_SCALAR = 1, ORACLE_GATE_VECTOR = 2 };

/* Value of a gate for channel c at (b, t, h). */
static double gate_at(const float *g, int kind, long long scalar_idx,
                      long long vec_base, int c) {
    if (kind == ORACLE_GATE_ONE || g == NULL) return 1.0;
    if (kind == ORACLE_GATE_SCALAR) return (double)g[scalar_idx];
    return (double)g[vec_base + c];
}

static int check_kind(int kind) {
    return kind == ORACLE_GATE_ONE || kind == ORACLE_GATE_SCALAR ||
           kind == ORACLE_GATE_VECTOR;
}

/*
 * Run the recurrence over T steps for every (b, h).
 * Returns 0 on success, -1 on a bad argument.
 * o may be NULL (not written); sT may be NULL (not written).
 * nthreads <= 0 uses the OpenMP default.
 */
int oracle_forward(int B, int T, int H, int dk, int dv,
                   int a_kind, int b_kind, int w_kind,
                   const float *q, const float *k, const float *v,
                   const float *a, const float *b, const float *w,
                   const double *s0, double *o, double *sT, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (!check_kind(a_kind) || !check_kind(b_kind) || !check_kind(w_kind)) return -1;
    if (T > 0 && (q == NULL || k == NULL || v == NULL)) return -1;
    if (a_kind != ORACLE_GATE_ONE && a == NULL && T > 0) return -1;
    if (b_kind != ORACLE_GATE_ONE && b == NULL && T > 0) return -1;
    if (w_kind != ORACLE_GATE_ONE && w == NULL && T > 0) return -1;

    const long long BH = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *e = (double *)malloc(sizeof(double) * (size_t)dv);
        double *ag = (double *)malloc(sizeof(double) * (size_t)dk);
        double *bk = (double *)malloc(sizeof(double) * (size_t)dk);
        double *wv = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !e || !ag || !bk || !wv) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long long bh = 0; bh < BH; ++bh) {
                const int bi = (int)(bh / H), hi = (int)(bh % H);
                const size_t state_off = (size_t)bh * dk * dv;
                if (s0) {
                    for (size_t x = 0; x < (size_t)dk * dv; ++x) S[x] = s0[state_off + x];
                } else {
                    memset(S, 0, sizeof(double) * (size_t)dk * dv);
                }
                for (int t = 0; t < T; ++t) {
                    const long long tok = ((long long)bi * T + t) * H + hi; /* (b,t,h) */
                    const long long kbase = tok * dk, vbase = tok * dv;
                    for (int i = 0; i < dk; ++i) {
                        ag[i] = gate_at(a, a_kind, tok, kbase, i);
                        bk[i] = gate_at(b, b_kind, tok, kbase, i) * (double)k[kbase + i];
                    }
                    for (int j = 0; j < dv; ++j)
                        wv[j] = gate_at(w, w_kind, tok, vbase, j) * (double)v[vbase + j];

                    /* S' = Diag(a_t) S_{t-1} */
                    for (int i = 0; i < dk; ++i)
                        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= ag[i];

                    /* e = S'^T k_t */
                    for (int j = 0; j < dv; ++j) e[j] = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        const double ki = (double)k[kbase + i];
                        for (int j = 0; j < dv; ++j) e[j] += S[(size_t)i * dv + j] * ki;
                    }

                    /* S_t = S' - (b*k) e^T + k (w*v)^T */
                    for (int i = 0; i < dk; ++i) {
                        const double ki = (double)k[kbase + i];
                        for (int j = 0; j < dv; ++j)
                            S[(size_t)i * dv + j] += -bk[i] * e[j] + ki * wv[j];
                    }

                    /* o_t = S_t^T q_t */
                    if (o) {
                        for (int j = 0; j < dv; ++j) {
                            double acc = 0.0;
                            for (int i = 0; i < dk; ++i)
                                acc += S[(size_t)i * dv + j] * (double)q[kbase + i];
                            o[vbase + j] = acc;
                        }
                    }
                }
                if (sT) {
                    for (size_t x = 0; x < (size_t)dk * dv; ++x) sT[state_off + x] = S[x];
                }
            }
        }
        free(S); free(e); free(ag); free(bk); free(wv);
    }
    return failed ? -1 : 0;
}

/*
 * One decode step: the same recurrence with T = 1, state updated in place.
 * q, k, a, b: [B, H, dk] (or [B, H] for scalar gates); v, w: [B, H, dv];
 * state: [B, H, dk, dv] read and overwritten; o: [B, H, dv].
 */
int oracle_decode_step(int B, int H, int dk, int dv,
                       int a_kind, int b_kind, int w_kind,
                       const float *q, const float *k, const float *v,
                       const float *a, const float *b, const float *w,
                       double *state, double *o, int nthreads) {
    if (state == NULL) return -1;
    return oracle_forward(B, 1, H, dk, dv, a_kind, b_kind, w_kind, q, k, v, a, b, w,
                          state, o, state, nthreads);
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Add the gradient of a gate at (b, t, h): vector gates take g_i, scalar gates
 * the sum over channels (the scalar multiplies every channel), GATE_ONE none. */
static void gate_grad(double *dg, int kind, long long scalar_idx, long long vec_base,
                      const double *g, int n) {
    if (dg == NULL || kind == ORACLE_GATE_ONE) return;
    if (kind == ORACLE_GATE_SCALAR) {
        double s = 0.0;
        for (int c = 0; c < n; ++c) s += g[c];
        dg[scalar_idx] = s;
        return;
    }
    for (int c = 0; c < n; ++c) dg[vec_base + c] = g[c];
}

/*
 * Gradients of  L = sum_t <o_t, do_t> + <S_T, dsT>  with respect to every
 * input of oracle_forward, by reverse-mode differentiation of the recurrence
 * above, one step at a time from t = T-1 down to 0.  G holds dL/dS_t.
 *
 *     o_t = S_t^T q_t            dq_t  = S_t do_t,   G += q_t do_t^T
 *     S_t = S' - p e^T + k u^T   (p = b*k, u = w*v)
 *                                dp = -G e,  de = -G^T p,  du = G^T k,
 *                                dk_t += G u,  dS' = G + k de^T
 *     e   = S'^T k               dk_t += S' de
 *     p   = b*k                  dk_t += b*dp,  db_t = k*dp
 *     u   = w*v                  dv_t  = w*du,  dw_t = v*du
 *     S'  = Diag(a) S_{t-1}      da_t[i] = sum_j dS'_ij S_{t-1,ij},
 *                                G <- Diag(a) dS'
 *     dS0 = G after step 0.
 *
 * The forward states S_0 .. S_T of one (b, h) are kept (T + 1 matrices of
 * dk x dv doubles).  do: [B, T, H, dv]; dsT: [B, H, dk, dv] or NULL (zero).
 * Outputs (double): dq, dk [B, T, H, dk]; dv [B, T, H, dv]; da, db in the
 * shape of a, b (NULL or GATE_ONE: not written); dw in the shape of w;
 * ds0 [B, H, dk, dv] (NULL: not written).  Returns 0, or -1 on a bad argument
 * or a failed allocation.
 */
int oracle_backward(int B, int T, int H, int dk, int dv,
                    int a_kind, int b_kind, int w_kind,
                    const float *q, const float *k, const float *v,
                    const float *a, const float *b, const float *w,
                    const double *s0, const double *dout, const double *dsT,
                    double *dq, double *dkk, double *dvv,
                    double *da, double *db, double *dw, double *ds0, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (!check_kind(a_kind) || !check_kind(b_kind) || !check_kind(w_kind)) return -1;
    if (T > 0 && (q == NULL || k == NULL || v == NULL || dout == NULL)) return -1;
    if (T > 0 && (dq == NULL || dkk == NULL || dvv == NULL)) return -1;
    if (a_kind != ORACLE_GATE_ONE && a == NULL && T > 0) return -1;
    if (b_kind != ORACLE_GATE_ONE && b == NULL && T > 0) return -1;
    if (w_kind != ORACLE_GATE_ONE && w == NULL && T > 0) return -1;

    const long long BH = (long long)B * H;
    const size_t DD = (size_t)dk * dv;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

    int failed = 0;
#pragma omp parallel
    {
        double *Ss = (double *)malloc(sizeof(double) * DD * ((size_t)T + 1));
        double *G = (double *)malloc(sizeof(double) * DD);
        double *Sp = (double *)malloc(sizeof(double) * DD);
        double *e = (double *)malloc(sizeof(double) * (size_t)dv);
        double *de = (double *)malloc(sizeof(double) * (size_t)dv);
        double *du = (double *)malloc(sizeof(double) * (size_t)dv);
        double *uu = (double *)malloc(sizeof(double) * (size_t)dv);
        double *ag = (double *)malloc(sizeof(double) * (size_t)dk);
        double *bg = (double *)malloc(sizeof(double) * (size_t)dk);
        double *p = (double *)malloc(sizeof(double) * (size_t)dk);
        double *dp = (double *)malloc(sizeof(double) * (size_t)dk);
        double *gk = (double *)malloc(sizeof(double) * (size_t)dk);
        double *gg = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
        if (!Ss || !G || !Sp || !e || !de || !du || !uu || !ag || !bg || !p || !dp || !gk ||
            !gg) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long long bh = 0; bh < BH; ++bh) {
                const int bi = (int)(bh / H), hi = (int)(bh % H);
                const size_t state_off = (size_t)bh * DD;
                /* forward, keeping S_0 .. S_T */
                if (s0) {
                    for (size_t x = 0; x < DD; ++x) Ss[x] = s0[state_off + x];
                } else {
                    memset(Ss, 0, sizeof(double) * DD);
                }
                for (int t = 0; t < T; ++t) {
                    const long long tok = ((long long)bi * T + t) * H + hi;
                    const long long kbase = tok * dk, vbase = tok * dv;
                    const double *Sprev = Ss + (size_t)t * DD;
                    double *Snext = Ss + (size_t)(t + 1) * DD;
                    for (int i = 0; i < dk; ++i) {
                        const double ai = gate_at(a, a_kind, tok, kbase, i);
                        for (int j = 0; j < dv; ++j)
                            Snext[(size_t)i * dv + j] = ai * Sprev[(size_t)i * dv + j];
                    }
                    for (int j = 0; j < dv; ++j) e[j] = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        const double ki = (double)k[kbase + i];
                        for (int j = 0; j < dv; ++j) e[j] += Snext[(size_t)i * dv + j] * ki;
                    }
                    for (int i = 0; i < dk; ++i) {
                        const double ki = (double)k[kbase + i];
                        const double pi = gate_at(b, b_kind, tok, kbase, i) * ki;
                        for (int j = 0; j < dv; ++j)
                            Snext[(size_t)i * dv + j] +=
                                -pi * e[j] + ki * gate_at(w, w_kind, tok, vbase, j) *
                                                 (double)v[vbase + j];
                    }
                }
                /* reverse */
                if (dsT) {
                    for (size_t x = 0; x < DD; ++x) G[x] = dsT[state_off + x];
                } else {
                    memset(G, 0, sizeof(double) * DD);
                }
                for (int t = T - 1; t >= 0; --t) {
                    const long long tok = ((long long)bi * T + t) * H + hi;
                    const long long kbase = tok * dk, vbase = tok * dv;
                    const double *Sprev = Ss + (size_t)t * DD;
                    const double *Scur = Ss + (size_t)(t + 1) * DD;
                    const double *dot = dout + vbase;
                    for (int i = 0; i < dk; ++i) {
                        ag[i] = gate_at(a, a_kind, tok, kbase, i);
                        bg[i] = gate_at(b, b_kind, tok, kbase, i);
                        p[i] = bg[i] * (double)k[kbase + i];
                    }
                    for (int j = 0; j < dv; ++j)
                        uu[j] = gate_at(w, w_kind, tok, vbase, j) * (double)v[vbase + j];

                    /* o_t = S_t^T q_t */
                    for (int i = 0; i < dk; ++i) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += Scur[(size_t)i * dv + j] * dot[j];
                        dq[kbase + i] = acc;
                    }
                    for (int i = 0; i < dk; ++i) {
                        const double qi = (double)q[kbase + i];
                        for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += qi * dot[j];
                    }

                    /* S' and e = S'^T k */
                    for (int i = 0; i < dk; ++i)
                        for (int j = 0; j < dv; ++j)
                            Sp[(size_t)i * dv + j] = ag[i] * Sprev[(size_t)i * dv + j];
                    for (int j = 0; j < dv; ++j) e[j] = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        const double ki = (double)k[kbase + i];
                        for (int j = 0; j < dv; ++j) e[j] += Sp[(size_t)i * dv + j] * ki;
                    }

                    /* S_t = S' - p e^T + k u^T */
                    for (int i = 0; i < dk; ++i) {
                        double s1 = 0.0, s2 = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            s1 += G[(size_t)i * dv + j] * e[j];
                            s2 += G[(size_t)i * dv + j] * uu[j];
                        }
                        dp[i] = -s1;
                        gk[i] = s2;
                    }
                    for (int j = 0; j < dv; ++j) {
                        double s1 = 0.0, s2 = 0.0;
                        for (int i = 0; i < dk; ++i) {
                            s1 += G[(size_t)i * dv + j] * p[i];
                            s2 += G[(size_t)i * dv + j] * (double)k[kbase + i];
                        }
                        de[j] = -s1;
                        du[j] = s2;
                    }
                    /* dS' = G + k de^T (kept in G) ; e = S'^T k */
                    for (int i = 0; i < dk; ++i) {
                        const double ki = (double)k[kbase + i];
                        double s = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            G[(size_t)i * dv + j] += ki * de[j];
                            s += Sp[(size_t)i * dv + j] * de[j];
                        }
                        gk[i] += s;
                    }
                    /* p = b*k */
                    for (int i = 0; i < dk; ++i) {
                        dkk[kbase + i] = gk[i] + bg[i] * dp[i];
                        gg[i] = (double)k[kbase + i] * dp[i];
                    }
                    gate_grad(db, b_kind, tok, kbase, gg, dk);
                    /* u = w*v */
                    for (int j = 0; j < dv; ++j) {
                        dvv[vbase + j] = gate_at(w, w_kind, tok, vbase, j) * du[j];
                        gg[j] = (double)v[vbase + j] * du[j];
                    }
                    gate_grad(dw, w_kind, tok, vbase, gg, dv);
                    /* S' = Diag(a) S_{t-1} */
                    for (int i = 0; i < dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < dv; ++j)
                            s += G[(size_t)i * dv + j] * Sprev[(size_t)i * dv + j];
                        gg[i] = s;
                    }
                    gate_grad(da, a_kind, tok, kbase, gg, dk);
                    for (int i = 0; i < dk; ++i)
                        for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= ag[i];
                }
                if (ds0) {
                    for (size_t x = 0; x < DD; ++x) ds0[state_off + x] = G[x];
                }
            }
        }
        free(Ss); free(G); free(Sp); free(e); free(de); free(du); free(uu);
        free(ag); free(bg); free(p); free(dp); free(gk); free(gg);
    }
    return failed ? -1 : 0;
}
