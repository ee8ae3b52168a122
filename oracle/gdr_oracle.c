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
