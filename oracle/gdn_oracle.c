/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the libgdn CUDA
 * library and its Python binding) may include, link, load or call this file.
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes (sources are named by page title and section):
 *
 *   "Qwen3.8-27B 架构深读: Gated DeltaNet 混合线性注意力与 262K 长上下文",
 *   section 三 (Gated DeltaNet: 把注意力变成可读写的记忆):
 *     - the delta rule  S <- S + beta (v - S k) k^T   (erase then write),
 *     - its gated form  S_t = g_t (.) S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T
 *       ("illustrative form"), and the illustrative per-head step function
 *       that takes the recall S k BEFORE the decay,
 *     - linear attention's read-out o_t = phi(q_t) S with S including token t,
 *     - "training accumulates the state chunk-parallel; inference does one
 *       fixed-size matrix update per step".
 *
 *   Standard form (the one the library implements):
 *       S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t,
 *       a_t = exp(g_t), b_t = beta_t.
 *   Written as steps:  S <- a S;  r = S k;  S <- S + b (v - r) k^T;  o = S q.
 *
 *   Illustrative ordering (flagged variant, the page's step function):
 *       r = S k;  S <- a S;  S <- S + b (v - r) k^T;  o = S q.
 *
 * Readings taken where the page is silent or garbled:
 *   - the state is Dv x Dk (S k is a Dv-vector), stored row-major [Dv][Dk];
 *   - the gate is one scalar per (token, v-head); the API takes its log g;
 *   - o_t is read from the post-update state;
 *   - no 1/sqrt(Dk) scale, identity feature map, no normalisation inside;
 *   - v-heads h share q/k head h / (Hv / Hqk) (contiguous groups).
 *
 * Layouts (token-major, packed over sequences):
 *   q, k  [T][Hqk][Dk]     v, o  [T][Hv][Dv]     g, beta  [T][Hv]
 *   state [N][Hv][Dv][Dk]  cu_seqlens [N+1], cu[0] = 0, cu[N] = T.
 *
 * Parity pins: every function here is pinned by the invariants and closed
 * forms in tests/test_oracle_pins.py and the hand-worked fixture under
 * tests/golden/.  The pages print no numerical worked example of their own.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_ORDER_STANDARD 0
#define ORACLE_ORDER_ILLUSTRATIVE 1
#define ORACLE_GATE_LOG 0    /* gate[] holds g, a = exp(g)      */
#define ORACLE_GATE_LINEAR 1 /* gate[] holds a itself (a may be 0) */

static int check_seqlens(const int64_t *cu, int64_t N, int64_t T) {
    if (cu[0] != 0 || cu[N] != T) return -2;
    for (int64_t n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return -2;
    return 0;
}

/* One (sequence, v-head) unit, token by token. */
static void run_unit(const double *q, const double *k, const double *v,
                     const double *gate, const double *beta, const double *s0,
                     int64_t t0, int64_t t1, int64_t Hqk, int64_t Hv,
                     int64_t Dk, int64_t Dv, int64_t h, int order,
                     int gate_kind, double *o, double *sT, double *S,
                     double *r) {
    const int64_t j = h / (Hv / Hqk);
    if (s0)
        memcpy(S, s0, sizeof(double) * Dv * Dk);
    else
        memset(S, 0, sizeof(double) * Dv * Dk);

    for (int64_t t = t0; t < t1; ++t) {
        const double *kt = k + (t * Hqk + j) * Dk;
        const double *qt = q + (t * Hqk + j) * Dk;
        const double *vt = v + (t * Hv + h) * Dv;
        const double gt = gate[t * Hv + h];
        const double a = (gate_kind == ORACLE_GATE_LOG) ? exp(gt) : gt;
        const double b = beta[t * Hv + h];

        if (order == ORACLE_ORDER_ILLUSTRATIVE) {
            /* recall from the undecayed state, then decay */
            for (int64_t i = 0; i < Dv; ++i) {
                double acc = 0.0;
                for (int64_t d = 0; d < Dk; ++d) acc += S[i * Dk + d] * kt[d];
                r[i] = acc;
            }
            for (int64_t x = 0; x < Dv * Dk; ++x) S[x] *= a;
        } else {
            /* decay, then recall from the decayed state */
            for (int64_t x = 0; x < Dv * Dk; ++x) S[x] *= a;
            for (int64_t i = 0; i < Dv; ++i) {
                double acc = 0.0;
                for (int64_t d = 0; d < Dk; ++d) acc += S[i * Dk + d] * kt[d];
                r[i] = acc;
            }
        }
        /* delta write: S <- S + b (v - r) k^T */
        for (int64_t i = 0; i < Dv; ++i) {
            const double u = b * (vt[i] - r[i]);
            for (int64_t d = 0; d < Dk; ++d) S[i * Dk + d] += u * kt[d];
        }
        /* read-out from the updated state: o = S q */
        if (o) {
            double *ot = o + (t * Hv + h) * Dv;
            for (int64_t i = 0; i < Dv; ++i) {
                double acc = 0.0;
                for (int64_t d = 0; d < Dk; ++d) acc += S[i * Dk + d] * qt[d];
                ot[i] = acc;
            }
        }
    }
    if (sT) memcpy(sT, S, sizeof(double) * Dv * Dk);
}

/*
 * Token-by-token recurrence over every (sequence, v-head) unit.
 * s0 may be NULL (zero initial state); o and sT may be NULL (not written).
 * heads_mask may be NULL (all heads) or point to Hv bytes, non-zero = run.
 * Returns 0, -1 on bad shapes, -2 on bad cu_seqlens, -3 on allocation failure.
 */
int gdn_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *gate, const double *beta,
                         const double *s0, const int64_t *cu_seqlens,
                         int64_t N, int64_t T, int64_t Hqk, int64_t Hv,
                         int64_t Dk, int64_t Dv, int order, int gate_kind,
                         const unsigned char *heads_mask, double *o,
                         double *sT) {
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return -1;
    if (Hv % Hqk != 0) return -1;
    if (check_seqlens(cu_seqlens, N, T)) return -2;
    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * Dv * Dk);
        double *r = (double *)malloc(sizeof(double) * Dv);
        if (!S || !r) {
#pragma omp atomic write
            failed = 1;
        }
        /* Every thread takes the same branch: the worksharing loop below is
           reached by the whole team or by none of it. */
#pragma omp barrier
        int any_failed;
#pragma omp atomic read
        any_failed = failed;
        if (!any_failed) {
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < N * Hv; ++u) {
                const int64_t n = u / Hv, h = u % Hv;
                if (heads_mask && !heads_mask[h]) continue;
                run_unit(q, k, v, gate, beta,
                         s0 ? s0 + (n * Hv + h) * Dv * Dk : NULL,
                         cu_seqlens[n], cu_seqlens[n + 1], Hqk, Hv, Dk, Dv, h,
                         order, gate_kind, o,
                         sT ? sT + (n * Hv + h) * Dv * Dk : NULL, S, r);
            }
        }
        free(S);
        free(r);
    }
    return failed ? -3 : 0;
}

/*
 * Chunk-parallel form of the standard rule, fp64, as a cross-check of the
 * recurrence ("训练时线性层可以用 chunk 并行累积状态", section 三 of the same
 * page; the page gives no formulas for it, so the steps below are derived
 * from the recurrence).  Per chunk of at most C tokens, starting afresh at
 * every sequence start, with S0 the state entering the chunk:
 *
 *   gamma_r = sum_{i<=r} g_i,  Gamma_r = exp(gamma_r),
 *   M_ri    = exp(gamma_r - gamma_i) for i <= r, else 0
 *   A       = strictly-lower part of diag(b) (K K^T (.) M)
 *   Tm      = (I + A)^{-1}                                (forward substitution)
 *   W       = Tm diag(b Gamma) K,   U~ = Tm diag(b) V
 *   U       = U~ - W S0^T                                 (rows u_r)
 *   O       = diag(Gamma) Q S0^T + (Q K^T (.) M) U
 *   S_C     = Gamma_C S0 + U^T diag(Gamma_C / Gamma) K
 *
 * The unroll behind it: u_r = b_r (v_r - a_r S_{r-1} k_r) and
 * S_r = Gamma_r S0 + sum_{i<=r} (Gamma_r / Gamma_i) u_i k_i^T.
 *
 * order == ORACLE_ORDER_ILLUSTRATIVE (recall before the decay): u_r = b_r (v_r -
 * S_{r-1} k_r) with the same recursion in u, so only token r's recall terms
 * change, from Gamma_r to Gamma_{r-1} (Gamma_{-1} = 1): A's row factor
 * becomes exp(gamma_{r-1} - gamma_i) and W = Tm diag(b Gamma_{.-1}) K.
 * Only the log gate is supported.
 */
int gdn_oracle_chunked(const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *s0,
                       const int64_t *cu_seqlens, int64_t N, int64_t T,
                       int64_t Hqk, int64_t Hv, int64_t Dk, int64_t Dv,
                       int64_t C, int order, double *o, double *sT) {
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || C <= 0)
        return -1;
    if (order != ORACLE_ORDER_STANDARD && order != ORACLE_ORDER_ILLUSTRATIVE) return -1;
    if (Hv % Hqk != 0) return -1;
    if (check_seqlens(cu_seqlens, N, T)) return -2;
    const int64_t G = Hv / Hqk;
    int failed = 0;
#pragma omp parallel
    {
        double *S = malloc(sizeof(double) * Dv * Dk);
        double *Sn = malloc(sizeof(double) * Dv * Dk);
        double *gam = malloc(sizeof(double) * C);
        double *A = malloc(sizeof(double) * C * C);
        double *Tm = malloc(sizeof(double) * C * C);
        double *W = malloc(sizeof(double) * C * Dk);
        double *U = malloc(sizeof(double) * C * Dv);
        if (!S || !Sn || !gam || !A || !Tm || !W || !U) {
#pragma omp atomic write
            failed = 1;
        }
        /* Every thread takes the same branch: the worksharing loop below is
           reached by the whole team or by none of it. */
#pragma omp barrier
        int any_failed;
#pragma omp atomic read
        any_failed = failed;
        if (!any_failed) {
#pragma omp for schedule(dynamic, 1)
            for (int64_t unit = 0; unit < N * Hv; ++unit) {
                const int64_t n = unit / Hv, h = unit % Hv, j = h / G;
                if (s0)
                    memcpy(S, s0 + (n * Hv + h) * Dv * Dk,
                           sizeof(double) * Dv * Dk);
                else
                    memset(S, 0, sizeof(double) * Dv * Dk);
                for (int64_t c0 = cu_seqlens[n]; c0 < cu_seqlens[n + 1];
                     c0 += C) {
                    int64_t L = cu_seqlens[n + 1] - c0;
                    if (L > C) L = C;
#define KR(r) (k + ((c0 + (r)) * Hqk + j) * Dk)
#define QR(r) (q + ((c0 + (r)) * Hqk + j) * Dk)
#define VR(r) (v + ((c0 + (r)) * Hv + h) * Dv)
#define GB(arr, r) (arr[(c0 + (r)) * Hv + h])
                    /* cumulative log-decay */
                    double acc = 0.0;
                    for (int64_t r = 0; r < L; ++r) {
                        acc += GB(g, r);
                        gam[r] = acc;
                    }
/* the log-decay of token r's recall: gamma_r, or gamma_{r-1} (0 for r = 0)
   when the recall is taken before the decay */
#define GREC(r) (order == ORACLE_ORDER_ILLUSTRATIVE ? ((r) > 0 ? gam[(r) - 1] : 0.0) : gam[r])
                    /* A = strictly lower part of diag(b)(K K^T (.) M) */
                    for (int64_t r = 0; r < L; ++r)
                        for (int64_t i = 0; i < L; ++i) {
                            double val = 0.0;
                            if (i < r) {
                                double kk = 0.0;
                                for (int64_t d = 0; d < Dk; ++d)
                                    kk += KR(r)[d] * KR(i)[d];
                                val = GB(beta, r) * kk * exp(GREC(r) - gam[i]);
                            }
                            A[r * C + i] = val;
                        }
                    /* Tm = (I + A)^{-1}, unit lower triangular: solve
                       (I + A) Tm = I column by column, row by row. */
                    for (int64_t col = 0; col < L; ++col)
                        for (int64_t r = 0; r < L; ++r) {
                            double val = (r == col) ? 1.0 : 0.0;
                            for (int64_t i = col; i < r; ++i)
                                val -= A[r * C + i] * Tm[i * C + col];
                            Tm[r * C + col] = (r < col) ? 0.0 : val;
                        }
                    /* W = Tm diag(b Gamma) K ;  U = Tm diag(b) V - W S0^T */
                    for (int64_t r = 0; r < L; ++r) {
                        for (int64_t d = 0; d < Dk; ++d) {
                            double s = 0.0;
                            for (int64_t i = 0; i <= r; ++i)
                                s += Tm[r * C + i] * GB(beta, i) *
                                     exp(GREC(i)) * KR(i)[d];
                            W[r * Dk + d] = s;
                        }
                        for (int64_t e = 0; e < Dv; ++e) {
                            double s = 0.0;
                            for (int64_t i = 0; i <= r; ++i)
                                s += Tm[r * C + i] * GB(beta, i) * VR(i)[e];
                            double ws = 0.0;
                            for (int64_t d = 0; d < Dk; ++d)
                                ws += W[r * Dk + d] * S[e * Dk + d];
                            U[r * Dv + e] = s - ws;
                        }
                    }
                    /* O = diag(Gamma) Q S0^T + (Q K^T (.) M) U */
                    if (o)
                        for (int64_t r = 0; r < L; ++r) {
                            double *orow = o + ((c0 + r) * Hv + h) * Dv;
                            for (int64_t e = 0; e < Dv; ++e) {
                                double qs = 0.0;
                                for (int64_t d = 0; d < Dk; ++d)
                                    qs += QR(r)[d] * S[e * Dk + d];
                                orow[e] = exp(gam[r]) * qs;
                            }
                            for (int64_t i = 0; i <= r; ++i) {
                                double qk = 0.0;
                                for (int64_t d = 0; d < Dk; ++d)
                                    qk += QR(r)[d] * KR(i)[d];
                                const double p = qk * exp(gam[r] - gam[i]);
                                for (int64_t e = 0; e < Dv; ++e)
                                    orow[e] += p * U[i * Dv + e];
                            }
                        }
                    /* S_C = Gamma_C S0 + U^T diag(Gamma_C / Gamma) K */
                    const double gC = gam[L - 1];
                    for (int64_t e = 0; e < Dv; ++e)
                        for (int64_t d = 0; d < Dk; ++d) {
                            double s = exp(gC) * S[e * Dk + d];
                            for (int64_t i = 0; i < L; ++i)
                                s += U[i * Dv + e] * exp(gC - gam[i]) *
                                     KR(i)[d];
                            Sn[e * Dk + d] = s;
                        }
                    memcpy(S, Sn, sizeof(double) * Dv * Dk);
#undef KR
#undef QR
#undef VR
#undef GB
#undef GREC
                }
                if (sT)
                    memcpy(sT + (n * Hv + h) * Dv * Dk, S,
                           sizeof(double) * Dv * Dk);
            }
        }
        free(S); free(Sn); free(gam); free(A); free(Tm); free(W); free(U);
    }
    return failed ? -3 : 0;
}
