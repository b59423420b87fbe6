/*
 * FP64 CPU oracle for the Gated DeltaNet-2 recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file or the library built from it; only the test suite, the smoke check
 * and the CPU-baseline leg of the bench harness use it. It shares no code,
 * header or constant with the CUDA library.
 *
 * Source: "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 * (iplexlaw.co.kr analysis of arXiv:2605.22791v1), sections "Independent
 * decisions on two axes" and "From a growing cache to a fixed state".
 *
 * Every routine below is the plain token-by-token definition, with no chunking,
 * blocking or reordering.  All tensors are row-major, double precision:
 *   per-token vectors  x[b][t][h][i]   index ((b*T + t)*H + h)*d + i
 *   per-token scalars  s[b][t][h]      index (b*T + t)*H + h
 *   states             S[b][h][i][j]   index ((b*H + h)*dk + i)*dv + j
 * i runs over key channels (dk), j over value channels (dv).  The state maps a
 * key-space vector to a value-space read: read = S^T x.
 *
 * Routines (each parallel over (b,h) with OpenMP, one head per thread):
 *   oracle_gdn2      GDN-2 recurrence (the method itself)
 *   oracle_kda       Kimi Delta Attention, written in transition-matrix form
 *   oracle_gdn       Gated DeltaNet (scalar decay), written in transition-matrix form
 *   oracle_b0_sum    closed-form decayed causal linear attention (the b = 0 case)
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define VEC(x, b, t, h, i, T, H, d) ((x)[((((size_t)(b) * (T) + (t)) * (H) + (h)) * (d)) + (i)])
#define SCAL(x, b, t, h, T, H) ((x)[(((size_t)(b) * (T) + (t)) * (H)) + (h)])
#define STATE(S, b, h, H, dk, dv) ((S) + (((size_t)(b) * (H) + (h)) * (size_t)(dk) * (dv)))

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static void load_state(double *S, const double *S0, int b, int h, int H, int dk, int dv) {
    if (S0)
        memcpy(S, STATE(S0, b, h, H, dk, dv), sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);
}

/*
 * GDN-2 ("Independent decisions on two axes"): per head and token t,
 *   Sbar = diag(alpha_t) S_{t-1}          channel-wise decay on key rows
 *   e    = b_t (.) k_t,  z = w_t (.) v_t   erase (key side) and write (value side)
 *   r    = Sbar^T e                        old read at the erase address
 *   S_t  = Sbar + k_t (z - r)^T            delta write
 *   o_t  = S_t^T q_t                       output from the state after this token's update
 * S0 may be NULL (zeros); ST may be NULL (not returned).
 */
void oracle_gdn2(int B, int T, int H, int dk, int dv,
                 const double *q, const double *k, const double *v,
                 const double *alpha, const double *bgate, const double *wgate,
                 const double *S0, double *o, double *ST) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
            double *e = (double *)malloc(sizeof(double) * dk);
            double *z = (double *)malloc(sizeof(double) * dv);
            double *r = (double *)malloc(sizeof(double) * dv);
            load_state(S, S0, b, h, H, dk, dv);
            for (int t = 0; t < T; ++t) {
                for (int i = 0; i < dk; ++i) {
                    const double a = VEC(alpha, b, t, h, i, T, H, dk);
                    for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
                    e[i] = VEC(bgate, b, t, h, i, T, H, dk) * VEC(k, b, t, h, i, T, H, dk);
                }
                for (int j = 0; j < dv; ++j)
                    z[j] = VEC(wgate, b, t, h, j, T, H, dv) * VEC(v, b, t, h, j, T, H, dv);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * e[i];
                    r[j] = acc;
                }
                for (int i = 0; i < dk; ++i) {
                    const double ki = VEC(k, b, t, h, i, T, H, dk);
                    for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += ki * (z[j] - r[j]);
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * VEC(q, b, t, h, i, T, H, dk);
                    VEC(o, b, t, h, j, T, H, dv) = acc;
                }
            }
            if (ST) memcpy(STATE(ST, b, h, H, dk, dv), S, sizeof(double) * (size_t)dk * dv);
            free(S); free(e); free(z); free(r);
        }
}

/*
 * Builds the dk x dk transition M = (I - beta k k^T) D, D = diag(d_i), and
 * applies S <- M S + beta k v^T with an explicit matrix product.
 */
static void transition_step(double *S, double *Snew, double *M, int dk, int dv,
                            const double *kk, const double *vv, const double *dgl, double beta) {
    for (int i = 0; i < dk; ++i)
        for (int l = 0; l < dk; ++l)
            M[(size_t)i * dk + l] = ((i == l) ? 1.0 : 0.0) * dgl[l] - beta * kk[i] * kk[l] * dgl[l];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
            double acc = beta * kk[i] * vv[j];
            for (int l = 0; l < dk; ++l) acc += M[(size_t)i * dk + l] * S[(size_t)l * dv + j];
            Snew[(size_t)i * dv + j] = acc;
        }
    memcpy(S, Snew, sizeof(double) * (size_t)dk * dv);
}

static void read_out(const double *S, const double *qq, double *out, int dk, int dv) {
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qq[i];
        out[j] = acc;
    }
}

/*
 * Kimi Delta Attention ("From a growing cache to a fixed state": KDA makes
 * forgetting channel-specific; "Independent decisions on two axes": tying both
 * gates to one scalar beta recovers KDA):
 *   S_t = (I - beta_t k_t k_t^T) diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
 * alpha is per key channel [B,T,H,dk]; beta is one scalar per token and head [B,T,H].
 */
void oracle_kda(int B, int T, int H, int dk, int dv,
                const double *q, const double *k, const double *v,
                const double *alpha, const double *beta,
                const double *S0, double *o, double *ST) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
            double *Sn = (double *)malloc(sizeof(double) * (size_t)dk * dv);
            double *M = (double *)malloc(sizeof(double) * (size_t)dk * dk);
            load_state(S, S0, b, h, H, dk, dv);
            for (int t = 0; t < T; ++t) {
                transition_step(S, Sn, M, dk, dv, &VEC(k, b, t, h, 0, T, H, dk), &VEC(v, b, t, h, 0, T, H, dv),
                                &VEC(alpha, b, t, h, 0, T, H, dk), SCAL(beta, b, t, h, T, H));
                read_out(S, &VEC(q, b, t, h, 0, T, H, dk), &VEC(o, b, t, h, 0, T, H, dv), dk, dv);
            }
            if (ST) memcpy(STATE(ST, b, h, H, dk, dv), S, sizeof(double) * (size_t)dk * dv);
            free(S); free(Sn); free(M);
        }
}

/*
 * Gated DeltaNet ("From a growing cache to a fixed state": a learned scalar
 * forgetting gate on the delta rule; "Independent decisions on two axes":
 * scalar decay on top of the KDA tie recovers it):
 *   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
 * alpha and beta are one scalar per token and head [B,T,H].
 */
void oracle_gdn(int B, int T, int H, int dk, int dv,
                const double *q, const double *k, const double *v,
                const double *alpha, const double *beta,
                const double *S0, double *o, double *ST) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
            double *Sn = (double *)malloc(sizeof(double) * (size_t)dk * dv);
            double *P = (double *)malloc(sizeof(double) * (size_t)dk * dk);
            load_state(S, S0, b, h, H, dk, dv);
            for (int t = 0; t < T; ++t) {
                const double a = SCAL(alpha, b, t, h, T, H);
                const double be = SCAL(beta, b, t, h, T, H);
                const double *kk = &VEC(k, b, t, h, 0, T, H, dk);
                const double *vv = &VEC(v, b, t, h, 0, T, H, dv);
                /* P = alpha (I - beta k k^T), then S <- P S + beta k v^T */
                for (int i = 0; i < dk; ++i)
                    for (int l = 0; l < dk; ++l)
                        P[(size_t)i * dk + l] = a * (((i == l) ? 1.0 : 0.0) - be * kk[i] * kk[l]);
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int l = 0; l < dk; ++l) acc += P[(size_t)i * dk + l] * S[(size_t)l * dv + j];
                        Sn[(size_t)i * dv + j] = acc + be * kk[i] * vv[j];
                    }
                memcpy(S, Sn, sizeof(double) * (size_t)dk * dv);
                read_out(S, &VEC(q, b, t, h, 0, T, H, dk), &VEC(o, b, t, h, 0, T, H, dv), dk, dv);
            }
            if (ST) memcpy(STATE(ST, b, h, H, dk, dv), S, sizeof(double) * (size_t)dk * dv);
            free(S); free(Sn); free(P);
        }
}

/*
 * The b = 0 case as an explicit causal sum (no recurrence).  With no erase the
 * read r vanishes and the state is a decayed sum of writes, so
 *   o_t[j] = sum_{s<=t} ( sum_i q_t[i] k_s[i] prod_{m=s+1..t} alpha_m[i] ) w_s[j] v_s[j]
 *          + sum_i q_t[i] ( prod_{m<=t} alpha_m[i] ) S0[i][j].
 * Every decay product is formed afresh for each (t, s, i); cost O(T^2 dk dv).
 */
void oracle_b0_sum(int B, int T, int H, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *alpha, const double *wgate,
                   const double *S0, double *o) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *coef = (double *)malloc(sizeof(double) * (size_t)dk);
            for (int t = 0; t < T; ++t) {
                double *out = &VEC(o, b, t, h, 0, T, H, dv);
                for (int j = 0; j < dv; ++j) out[j] = 0.0;
                for (int s = 0; s <= t; ++s) {
                    double score = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        double decay = 1.0;
                        for (int m = s + 1; m <= t; ++m) decay *= VEC(alpha, b, m, h, i, T, H, dk);
                        score += VEC(q, b, t, h, i, T, H, dk) * VEC(k, b, s, h, i, T, H, dk) * decay;
                    }
                    for (int j = 0; j < dv; ++j)
                        out[j] += score * VEC(wgate, b, s, h, j, T, H, dv) * VEC(v, b, s, h, j, T, H, dv);
                }
                if (S0) {
                    const double *S = STATE(S0, b, h, H, dk, dv);
                    for (int i = 0; i < dk; ++i) {
                        double decay = 1.0;
                        for (int m = 0; m <= t; ++m) decay *= VEC(alpha, b, m, h, i, T, H, dk);
                        coef[i] = VEC(q, b, t, h, i, T, H, dk) * decay;
                    }
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int i = 0; i < dk; ++i) acc += coef[i] * S[(size_t)i * dv + j];
                        out[j] += acc;
                    }
                }
            }
            free(coef);
        }
}
