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
 *   oracle_gdn2_bwd  gradient of oracle_gdn2 (reverse mode through its token loop)
 *   oracle_gdn2_prep the activations that turn pre-activation logits into the
 *                    recurrence's inputs (q, k, v, alpha, b, w)
 *   oracle_output_gate  RMS norm and sigmoid output gate applied to the recurrence's output
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

/*
 * Gradient of the GDN-2 recurrence (reverse mode through the token loop of
 * oracle_gdn2, in the same notation).  Given the upstream gradients dO of the
 * outputs and dST of the final state (NULL = zero), returns the gradients of
 * L = sum(dO * o) + sum(dST * S_T) with respect to q, k, v, alpha, b, w and S0
 * (dS0 may be NULL).  The backward pass over one token t, with G the gradient
 * with respect to S_t:
 *   G     += q_t dO_t^T                    o_t = S_t^T q_t
 *   dq_t   = S_t dO_t
 *   dk_t   = G u,    du = G^T k_t          S_t = Sbar + k_t u^T,  u = z - r
 *   dw_t   = du * v_t,  dv_t = du * w_t    z = w_t * v_t
 *   dSbar  = G - e du^T,  de = -Sbar du    r = Sbar^T e
 *   db_t   = de * k_t,   dk_t += de * b_t  e = b_t * k_t
 *   dalpha_t[i] = sum_j S_{t-1}[i][j] dSbar[i][j];  G <- diag(alpha_t) dSbar
 * The forward states S_0 .. S_{T-1} are kept (T x dk x dv doubles per head).
 */
void oracle_gdn2_bwd(int B, int T, int H, int dk, int dv,
                     const double *q, const double *k, const double *v,
                     const double *alpha, const double *bgate, const double *wgate,
                     const double *S0, const double *dO, const double *dST,
                     double *dq, double *dk_, double *dv_, double *dalpha, double *db, double *dw,
                     double *dS0) {
    const size_t D2 = (size_t)dk * dv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *Sst = (double *)malloc(sizeof(double) * D2 * (size_t)(T + 1));   /* S_0 .. S_T */
            double *G = (double *)malloc(sizeof(double) * D2);
            double *Sb = (double *)malloc(sizeof(double) * D2);
            double *e = (double *)malloc(sizeof(double) * dk);
            double *z = (double *)malloc(sizeof(double) * dv);
            double *u = (double *)malloc(sizeof(double) * dv);
            double *du = (double *)malloc(sizeof(double) * dv);
            double *de = (double *)malloc(sizeof(double) * dk);
            load_state(Sst, S0, b, h, H, dk, dv);
            /* forward, keeping every state */
            for (int t = 0; t < T; ++t) {
                const double *Sp = Sst + D2 * t;
                double *Sn = Sst + D2 * (t + 1);
                for (int i = 0; i < dk; ++i) {
                    const double a = VEC(alpha, b, t, h, i, T, H, dk);
                    for (int j = 0; j < dv; ++j) Sn[(size_t)i * dv + j] = a * Sp[(size_t)i * dv + j];
                    e[i] = VEC(bgate, b, t, h, i, T, H, dk) * VEC(k, b, t, h, i, T, H, dk);
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += Sn[(size_t)i * dv + j] * e[i];
                    u[j] = VEC(wgate, b, t, h, j, T, H, dv) * VEC(v, b, t, h, j, T, H, dv) - acc;
                }
                for (int i = 0; i < dk; ++i) {
                    const double ki = VEC(k, b, t, h, i, T, H, dk);
                    for (int j = 0; j < dv; ++j) Sn[(size_t)i * dv + j] += ki * u[j];
                }
            }
            /* backward */
            if (dST) memcpy(G, STATE(dST, b, h, H, dk, dv), sizeof(double) * D2);
            else memset(G, 0, sizeof(double) * D2);
            for (int t = T - 1; t >= 0; --t) {
                const double *Sp = Sst + D2 * t, *St = Sst + D2 * (t + 1);
                for (int i = 0; i < dk; ++i) {
                    const double qi = VEC(q, b, t, h, i, T, H, dk);
                    for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += qi * VEC(dO, b, t, h, j, T, H, dv);
                }
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * VEC(dO, b, t, h, j, T, H, dv);
                    VEC(dq, b, t, h, i, T, H, dk) = acc;
                }
                /* recompute Sbar, e, z, u of this token */
                for (int i = 0; i < dk; ++i) {
                    const double a = VEC(alpha, b, t, h, i, T, H, dk);
                    for (int j = 0; j < dv; ++j) Sb[(size_t)i * dv + j] = a * Sp[(size_t)i * dv + j];
                    e[i] = VEC(bgate, b, t, h, i, T, H, dk) * VEC(k, b, t, h, i, T, H, dk);
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += Sb[(size_t)i * dv + j] * e[i];
                    z[j] = VEC(wgate, b, t, h, j, T, H, dv) * VEC(v, b, t, h, j, T, H, dv);
                    u[j] = z[j] - acc;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += G[(size_t)i * dv + j] * VEC(k, b, t, h, i, T, H, dk);
                    du[j] = acc;
                    VEC(dw, b, t, h, j, T, H, dv) = acc * VEC(v, b, t, h, j, T, H, dv);
                    VEC(dv_, b, t, h, j, T, H, dv) = acc * VEC(wgate, b, t, h, j, T, H, dv);
                }
                for (int i = 0; i < dk; ++i) {
                    double gu = 0.0, sd = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        gu += G[(size_t)i * dv + j] * u[j];
                        sd += Sb[(size_t)i * dv + j] * du[j];
                    }
                    de[i] = -sd;
                    const double ki = VEC(k, b, t, h, i, T, H, dk), bi = VEC(bgate, b, t, h, i, T, H, dk);
                    VEC(db, b, t, h, i, T, H, dk) = de[i] * ki;
                    VEC(dk_, b, t, h, i, T, H, dk) = gu + de[i] * bi;
                }
                for (int i = 0; i < dk; ++i) {
                    const double a = VEC(alpha, b, t, h, i, T, H, dk);
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double dsb = G[(size_t)i * dv + j] - e[i] * du[j];
                        acc += Sp[(size_t)i * dv + j] * dsb;
                        G[(size_t)i * dv + j] = a * dsb;
                    }
                    VEC(dalpha, b, t, h, i, T, H, dk) = acc;
                }
            }
            if (dS0) memcpy(STATE(dS0, b, h, H, dk, dv), G, sizeof(double) * D2);
            free(Sst); free(G); free(Sb); free(e); free(z); free(u); free(du); free(de);
        }
}

/*
 * Input preparation from pre-activation logits ("Independent decisions on two
 * axes": the erase gate b and the write gate w are sigmoids of their own linear
 * projections; "Token processing and parallel training": the query and key paths
 * end in SiLU then L2 normalisation, the value path in SiLU).  The pages give the
 * channel-wise decay alpha without its parameterisation; it is taken here as
 * alpha = exp(-softplus(xa)), the usual log-space gate, which is in (0, 1).
 * Per token row and head:
 *   q = silu(xq) / ||silu(xq)||_2   (a zero row stays zero)      [dk]
 *   k = silu(xk) / ||silu(xk)||_2                                 [dk]
 *   v = silu(xv)                                                  [dv]
 *   alpha = exp(-softplus(xa)) = exp(-log(1 + exp(xa)))           [dk]
 *   b = sigmoid(xb),  w = sigmoid(xw)                             [dk], [dv]
 * with silu(x) = x sigmoid(x) and sigmoid(x) = 1 / (1 + exp(-x)).  rows = B*T*H.
 */
static double prep_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double prep_softplus(double x) { return x > 0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

static void prep_silu_l2(const double *x, double *y, int d) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) {
        y[i] = x[i] * prep_sigmoid(x[i]);
        ss += y[i] * y[i];
    }
    const double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
    for (int i = 0; i < d; ++i) y[i] *= inv;
}

void oracle_gdn2_prep(long long rows, int dk, int dv,
                      const double *xq, const double *xk, const double *xv,
                      const double *xa, const double *xb, const double *xw,
                      double *q, double *k, double *v, double *alpha, double *b, double *w) {
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        const size_t ok = (size_t)r * dk, ov = (size_t)r * dv;
        prep_silu_l2(xq + ok, q + ok, dk);
        prep_silu_l2(xk + ok, k + ok, dk);
        for (int i = 0; i < dk; ++i) {
            alpha[ok + i] = exp(-prep_softplus(xa[ok + i]));
            b[ok + i] = prep_sigmoid(xb[ok + i]);
        }
        for (int j = 0; j < dv; ++j) {
            v[ov + j] = xv[ov + j] * prep_sigmoid(xv[ov + j]);
            w[ov + j] = prep_sigmoid(xw[ov + j]);
        }
    }
}

/*
 * Output epilogue ("Token processing and parallel training": after the recurrent
 * update, RMS normalisation and a separate output gate, distinct from the write
 * gate, come before the output projection).  The pages name the two steps but
 * not their exact form; the readings taken here: the RMS norm runs over each
 * head's d_v channels with a learned per-channel scale and an epsilon, and the
 * output gate is a sigmoid of its own logits, like the pages' other gates:
 *   y = o / sqrt(mean_j(o_j^2) + eps) * weight * sigmoid(g)
 * per row (one token and head) of rows = B*T*H rows of dv channels.
 */
void oracle_output_gate(long long rows, int dv, const double *o, const double *g, const double *weight,
                        double eps, double *y) {
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        const double *orow = o + (size_t)r * dv, *grow = g + (size_t)r * dv;
        double ms = 0.0;
        for (int j = 0; j < dv; ++j) ms += orow[j] * orow[j];
        ms /= dv;
        const double inv = 1.0 / sqrt(ms + eps);
        for (int j = 0; j < dv; ++j) y[(size_t)r * dv + j] = orow[j] * inv * weight[j] / (1.0 + exp(-grow[j]));
    }
}
