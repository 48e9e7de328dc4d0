/*
 * gdr_oracle.c -- fp64 CPU oracle for the looped gated delta rule (LT2 linear mixer).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this
 * file; only the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * do.  It shares no code, header or table with the CUDA library.
 *
 * What it computes.  "LT2 transformer looped a tempo lineare" (paithon.it), section
 * "Sostituire il motore", displayed equation: the linear mixer keeps a d_k x d_v state
 * and updates it once per token as
 *
 *     S_t = A_t S_{t-1} + beta_t k_t v_t^T,     A_t = Diag(alpha_t) (I - beta_t k_t k_t^T)
 *
 * Readout (the pages never print it; it is the plainest reading): o_t = S_t^T q_t, taken
 * after token t's update, with no extra scale.  alpha_t is either one scalar per token
 * (GDN gating: Diag(alpha) = alpha I) or one value per key channel (a d_k vector).
 *
 * The gate code `per_key` of every entry point: 0 scalar gating; 1 per-key gating in the
 * order the equation is printed (delta, then decay: A_t = Diag(alpha_t)(I - beta_t k_t k_t^T));
 * 2 per-key gating with the decay first, A_t = (I - beta_t k_t k_t^T) Diag(alpha_t), the
 * order a right-multiplying convention for S would give.  For scalar alpha the two orders
 * are the same matrix.
 *
 * Loops.  Section "Profondita presa in prestito" of the same page applies one weight-tied
 * block T times; the section "Dove il quadro si incrina" lists carrying the recurrent
 * state from one loop to the next as unexplored.  So every (loop, batch, head) triple is
 * an independent recurrence with its own inputs, initial state and final state.  The
 * oracle therefore takes a flat list of U independent "head-units" (U = T*B*H in
 * row-major [T,B,H] order); the loop index changes nothing in the arithmetic.
 *
 * Three formulations, all in fp64:
 *   gdr_ref_sequential  token by token, the equation as written (primary oracle);
 *   gdr_ref_dense       materialises A_t as a d_k x d_k matrix and multiplies (brute force);
 *   gdr_ref_chunked     the chunk-parallel rewriting of the same recurrence (UT/WY form),
 *                       derived from the equation; used to pin the algebra the GPU uses.
 *
 * Layouts (all contiguous, last index fastest):
 *   q, k  [U][L][dk]      v, o  [U][L][dv]
 *   alpha [U][L] (scalar gating) or [U][L][dk] (per-key gating)
 *   beta  [U][L]          S0, S_out [U][dk][dv]   (S0 may be NULL = zeros)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX2(a, b, nb) ((a) * (nb) + (b))

/* alpha of token t, key channel i. */
static double gate_at(const double* alpha, int per_key, int64_t t, int64_t i, int64_t dk)
{
    return per_key ? alpha[t * dk + i] : alpha[t];
}

/* ------------------------------------------------------------------------------------ */
/* Sequential form: the displayed equation, one token at a time.                         */
/* ------------------------------------------------------------------------------------ */
static void seq_unit(int64_t L, int64_t dk, int64_t dv, int per_key,
                     const double* q, const double* k, const double* v,
                     const double* alpha, const double* beta, const double* S0,
                     double* o, double* S, double* e)
{
    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else    memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t = 0; t < L; ++t) {
        const double* qt = q + t * dk;
        const double* kt = k + t * dk;
        const double* vt = v + t * dv;
        const double  bt = beta[t];

        if (per_key == 2) {
            /* decay first: S <- Diag(alpha_t) S_{t-1}, then the delta step on it */
            for (int64_t i = 0; i < dk; ++i) {
                const double ai = gate_at(alpha, per_key, t, i, dk);
                for (int64_t j = 0; j < dv; ++j) S[IDX2(i, j, dv)] *= ai;
            }
        }

        /* e = k_t^T S  (a d_v row vector; S = S_{t-1}, or its decayed copy) */
        for (int64_t j = 0; j < dv; ++j) e[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j)
                e[j] += kt[i] * S[IDX2(i, j, dv)];

        if (per_key == 2) {
            /* S_t = S - beta_t k_t e + beta_t k_t v_t^T */
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j)
                    S[IDX2(i, j, dv)] += bt * kt[i] * (vt[j] - e[j]);
        } else {
            /* S_t = Diag(alpha_t) (S_{t-1} - beta_t k_t e) + beta_t k_t v_t^T */
            for (int64_t i = 0; i < dk; ++i) {
                const double ai = gate_at(alpha, per_key, t, i, dk);
                for (int64_t j = 0; j < dv; ++j)
                    S[IDX2(i, j, dv)] = ai * (S[IDX2(i, j, dv)] - bt * kt[i] * e[j]) + bt * kt[i] * vt[j];
            }
        }

        /* o_t = S_t^T q_t */
        for (int64_t j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < dk; ++i) acc += qt[i] * S[IDX2(i, j, dv)];
            o[t * dv + j] = acc;
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Dense form: build A_t explicitly and compute S_t = A_t S_{t-1} + beta_t k_t v_t^T.     */
/* ------------------------------------------------------------------------------------ */
static void dense_unit(int64_t L, int64_t dk, int64_t dv, int per_key,
                       const double* q, const double* k, const double* v,
                       const double* alpha, const double* beta, const double* S0,
                       double* o, double* S, double* A, double* Snew)
{
    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else    memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t = 0; t < L; ++t) {
        const double* qt = q + t * dk;
        const double* kt = k + t * dk;
        const double* vt = v + t * dv;
        const double  bt = beta[t];

        /* A_t[i][m] = alpha_t[i] (delta_im - beta_t k_t[i] k_t[m]);
           decay first: A_t[i][m] = (delta_im - beta_t k_t[i] k_t[m]) alpha_t[m] */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t m = 0; m < dk; ++m) {
                const double a = gate_at(alpha, per_key, t, per_key == 2 ? m : i, dk);
                A[IDX2(i, m, dk)] = a * ((i == m ? 1.0 : 0.0) - bt * kt[i] * kt[m]);
            }
        /* Snew = A_t S + beta_t k_t v_t^T */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t m = 0; m < dk; ++m) acc += A[IDX2(i, m, dk)] * S[IDX2(m, j, dv)];
                Snew[IDX2(i, j, dv)] = acc + bt * kt[i] * vt[j];
            }
        memcpy(S, Snew, sizeof(double) * dk * dv);

        for (int64_t j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < dk; ++i) acc += qt[i] * S[IDX2(i, j, dv)];
            o[t * dv + j] = acc;
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Chunked form.  Inside a chunk of n tokens (local index r = 0..n-1) with incoming      */
/* state S0, write decay(r, s)[i] for the product of alpha_{s'}[i] over s < s' <= r      */
/* (empty product = 1).  Unrolling the equation gives, with e_r = k_r^T S_{r-1}:         */
/*                                                                                        */
/*   S_r = decay(r,-1) S0 + sum_{s<=r} beta_s [ (decay(r,s) k_s) v_s^T                  */
/*                                             - (decay(r,s-1) k_s) e_s ]                */
/*                                                                                        */
/* (the delta term of token s is hit by its own alpha_s, the write term is not).  Taking */
/* k_r^T S_{r-1} of that expression gives a unit lower-triangular system for the e_r,    */
/* solved by forward substitution; o_r = S_r^T q_r and the chunk's final state follow.   */
/* With the decay first (gate code 2), e_r = k_r^T Diag(alpha_r) S_{r-1} and token s's    */
/* delta term is decayed like its write term:                                            */
/*                                                                                        */
/*   S_r = decay(r,-1) S0 + sum_{s<=r} beta_s (decay(r,s) k_s) (v_s - e_s)^T             */
/*                                                                                        */
/* so every decay(., s-1) below becomes decay(., s) and the k_r-side decay(r-1, .) of    */
/* the e system becomes decay(r, .).                                                      */
/* This "e-form" covers both gatings.  For scalar gating the same algebra with           */
/* u_r = v_r - alpha_r e_r collapses the two terms into one ("u-form"):                  */
/*                                                                                        */
/*   (I + A) U = V - diag(g) K S0,  A_rs = beta_s (g_r/g_s) k_r.k_s (s<r), g_r=decay(r,-1)*/
/*   o_r  = g_r S0^T q_r + sum_{s<=r} beta_s (g_r/g_s) (q_r.k_s) u_s                     */
/*   S_n  = g_{n-1} S0 + sum_s beta_s (g_{n-1}/g_s) k_s u_s^T                            */
/* ------------------------------------------------------------------------------------ */

/* Product of alpha_{s'}[i] for s < s' <= r, in chunk-local indices (s may be -1). */
static double decay(const double* alpha, int per_key, int64_t t0, int64_t r, int64_t s,
                    int64_t i, int64_t dk)
{
    double p = 1.0;
    for (int64_t sp = s + 1; sp <= r; ++sp) p *= gate_at(alpha, per_key, t0 + sp, i, dk);
    return p;
}

static void chunked_unit_eform(int64_t L, int64_t dk, int64_t dv, int per_key, int64_t C,
                               const double* q, const double* k, const double* v,
                               const double* alpha, const double* beta, const double* S0,
                               double* o, double* S, double* E, double* Mke, double* Mkv,
                               double* Snew)
{
    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else    memset(S, 0, sizeof(double) * dk * dv);
    const int64_t df = per_key == 2 ? 1 : 0;    /* decay first: shift the e-side indices */

    for (int64_t t0 = 0; t0 < L; t0 += C) {
        const int64_t n = (L - t0 < C) ? (L - t0) : C;
        const double* kc = k + t0 * dk;
        const double* qc = q + t0 * dk;
        const double* vc = v + t0 * dv;
        const double* bc = beta + t0;

        /* M^ke_rs = beta_s sum_i k_r[i] decay(r-1, s-1)[i] k_s[i];  M^kv uses decay(r-1, s). */
        for (int64_t r = 0; r < n; ++r)
            for (int64_t s = 0; s < r; ++s) {
                double ke = 0.0, kv = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    ke += kc[r * dk + i] * decay(alpha, per_key, t0, r - 1 + df, s - 1 + df, i, dk) * kc[s * dk + i];
                    kv += kc[r * dk + i] * decay(alpha, per_key, t0, r - 1 + df, s, i, dk) * kc[s * dk + i];
                }
                Mke[r * C + s] = bc[s] * ke;
                Mkv[r * C + s] = bc[s] * kv;
            }

        /* Forward substitution: e_r = (decay(r-1,-1) k_r)^T S0 + sum_{s<r} (Mkv_rs v_s - Mke_rs e_s) */
        for (int64_t r = 0; r < n; ++r)
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < dk; ++i)
                    acc += kc[r * dk + i] * decay(alpha, per_key, t0, r - 1 + df, -1, i, dk) * S[IDX2(i, j, dv)];
                for (int64_t s = 0; s < r; ++s)
                    acc += Mkv[r * C + s] * vc[s * dv + j] - Mke[r * C + s] * E[s * dv + j];
                E[r * dv + j] = acc;
            }

        /* o_r = (decay(r,-1) q_r)^T S0 + sum_{s<=r} beta_s [ (q_r.decay(r,s)k_s) v_s - (q_r.decay(r,s-1)k_s) e_s ] */
        for (int64_t r = 0; r < n; ++r) {
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < dk; ++i)
                    acc += qc[r * dk + i] * decay(alpha, per_key, t0, r, -1, i, dk) * S[IDX2(i, j, dv)];
                o[(t0 + r) * dv + j] = acc;
            }
            for (int64_t s = 0; s <= r; ++s) {
                double qv = 0.0, qe = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    qv += qc[r * dk + i] * decay(alpha, per_key, t0, r, s, i, dk) * kc[s * dk + i];
                    qe += qc[r * dk + i] * decay(alpha, per_key, t0, r, s - 1 + df, i, dk) * kc[s * dk + i];
                }
                for (int64_t j = 0; j < dv; ++j)
                    o[(t0 + r) * dv + j] += bc[s] * (qv * vc[s * dv + j] - qe * E[s * dv + j]);
            }
        }

        /* S_n = decay(n-1,-1) S0 + sum_s beta_s [ (decay(n-1,s) k_s) v_s^T - (decay(n-1,s-1) k_s) e_s^T ] */
        for (int64_t i = 0; i < dk; ++i) {
            const double g = decay(alpha, per_key, t0, n - 1, -1, i, dk);
            for (int64_t j = 0; j < dv; ++j) Snew[IDX2(i, j, dv)] = g * S[IDX2(i, j, dv)];
            for (int64_t s = 0; s < n; ++s) {
                const double wv = bc[s] * decay(alpha, per_key, t0, n - 1, s, i, dk) * kc[s * dk + i];
                const double we = bc[s] * decay(alpha, per_key, t0, n - 1, s - 1 + df, i, dk) * kc[s * dk + i];
                for (int64_t j = 0; j < dv; ++j)
                    Snew[IDX2(i, j, dv)] += wv * vc[s * dv + j] - we * E[s * dv + j];
            }
        }
        memcpy(S, Snew, sizeof(double) * dk * dv);
    }
}

static void chunked_unit_uform(int64_t L, int64_t dk, int64_t dv, int64_t C,
                               const double* q, const double* k, const double* v,
                               const double* alpha, const double* beta, const double* S0,
                               double* o, double* S, double* Um, double* A, double* Snew)
{
    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else    memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t0 = 0; t0 < L; t0 += C) {
        const int64_t n = (L - t0 < C) ? (L - t0) : C;
        const double* kc = k + t0 * dk;
        const double* qc = q + t0 * dk;
        const double* vc = v + t0 * dv;
        const double* bc = beta + t0;

        /* A_rs = beta_s (g_r/g_s) k_r.k_s for s < r, with g_r/g_s = decay(r, s). */
        for (int64_t r = 0; r < n; ++r)
            for (int64_t s = 0; s < r; ++s) {
                double kk = 0.0;
                for (int64_t i = 0; i < dk; ++i) kk += kc[r * dk + i] * kc[s * dk + i];
                A[r * C + s] = bc[s] * decay(alpha, 0, t0, r, s, 0, dk) * kk;
            }

        /* (I + A) U = V - diag(g) K S0, forward substitution */
        for (int64_t r = 0; r < n; ++r) {
            const double g = decay(alpha, 0, t0, r, -1, 0, dk);
            for (int64_t j = 0; j < dv; ++j) {
                double ks = 0.0;
                for (int64_t i = 0; i < dk; ++i) ks += kc[r * dk + i] * S[IDX2(i, j, dv)];
                double acc = vc[r * dv + j] - g * ks;
                for (int64_t s = 0; s < r; ++s) acc -= A[r * C + s] * Um[s * dv + j];
                Um[r * dv + j] = acc;
            }
        }

        /* o_r = g_r S0^T q_r + sum_{s<=r} beta_s (g_r/g_s) (q_r.k_s) u_s */
        for (int64_t r = 0; r < n; ++r) {
            const double g = decay(alpha, 0, t0, r, -1, 0, dk);
            for (int64_t j = 0; j < dv; ++j) {
                double qs = 0.0;
                for (int64_t i = 0; i < dk; ++i) qs += qc[r * dk + i] * S[IDX2(i, j, dv)];
                o[(t0 + r) * dv + j] = g * qs;
            }
            for (int64_t s = 0; s <= r; ++s) {
                double qk = 0.0;
                for (int64_t i = 0; i < dk; ++i) qk += qc[r * dk + i] * kc[s * dk + i];
                const double w = bc[s] * decay(alpha, 0, t0, r, s, 0, dk) * qk;
                for (int64_t j = 0; j < dv; ++j) o[(t0 + r) * dv + j] += w * Um[s * dv + j];
            }
        }

        /* S_n = g_{n-1} S0 + sum_s beta_s (g_{n-1}/g_s) k_s u_s^T */
        const double gn = decay(alpha, 0, t0, n - 1, -1, 0, dk);
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) {
                double acc = gn * S[IDX2(i, j, dv)];
                for (int64_t s = 0; s < n; ++s)
                    acc += bc[s] * decay(alpha, 0, t0, n - 1, s, 0, dk) * kc[s * dk + i] * Um[s * dv + j];
                Snew[IDX2(i, j, dv)] = acc;
            }
        memcpy(S, Snew, sizeof(double) * dk * dv);
    }
}

/* ------------------------------------------------------------------------------------ */
/* Exported entry points.  Each runs every head-unit independently (OpenMP over units).  */
/* Return 0 on success, -1 on bad arguments, -2 on allocation failure.                   */
/* ------------------------------------------------------------------------------------ */
/* ------------------------------------------------------------------------------------ */
/* The u-form in its WY arrangement (scalar gating).  With T = (I + A)^{-1} written out,  */
/* the state-independent products U_v = T V, W = T diag(g) K and Q' = diag(g) Q - P W      */
/* (P_rs = beta_s (g_r/g_s) q_r.k_s for s <= r) leave one product with S0 per chunk:      */
/*                                                                                        */
/*   U = U_v - W S0,   O = Q' S0 + P U_v,   S_n = g_{n-1} S0 + sum_s beta_s (g_{n-1}/g_s) k_s u_s^T */
/* ------------------------------------------------------------------------------------ */
static int chunked_unit_wyform(int64_t L, int64_t dk, int64_t dv, int64_t C,
                               const double* q, const double* k, const double* v,
                               const double* alpha, const double* beta, const double* S0,
                               double* o, double* S, double* Snew)
{
    double* A = (double*)calloc((size_t)(C * C), sizeof(double));
    double* T = (double*)calloc((size_t)(C * C), sizeof(double));
    double* P = (double*)calloc((size_t)(C * C), sizeof(double));
    double* Uv = (double*)malloc(sizeof(double) * C * dv);
    double* U = (double*)malloc(sizeof(double) * C * dv);
    double* W = (double*)malloc(sizeof(double) * C * dk);
    double* Qp = (double*)malloc(sizeof(double) * C * dk);
    if (!A || !T || !P || !Uv || !U || !W || !Qp) {
        free(A); free(T); free(P); free(Uv); free(U); free(W); free(Qp);
        return -1;
    }
    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else    memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t0 = 0; t0 < L; t0 += C) {
        const int64_t n = (L - t0 < C) ? (L - t0) : C;
        const double* kc = k + t0 * dk;
        const double* qc = q + t0 * dk;
        const double* vc = v + t0 * dv;
        const double* bc = beta + t0;

        /* A (s < r) and P (s <= r) */
        for (int64_t r = 0; r < n; ++r)
            for (int64_t s = 0; s <= r; ++s) {
                double kk = 0.0, qk = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    kk += kc[r * dk + i] * kc[s * dk + i];
                    qk += qc[r * dk + i] * kc[s * dk + i];
                }
                const double f = bc[s] * decay(alpha, 0, t0, r, s, 0, dk);
                A[r * C + s] = s < r ? f * kk : 0.0;
                P[r * C + s] = f * qk;
            }
        /* T = (I + A)^{-1}, unit lower triangular: T_rs = -sum_{s<=m<r} A_rm T_ms */
        for (int64_t r = 0; r < n; ++r) {
            T[r * C + r] = 1.0;
            for (int64_t s = 0; s < r; ++s) {
                double acc = 0.0;
                for (int64_t m = s; m < r; ++m) acc += A[r * C + m] * T[m * C + s];
                T[r * C + s] = -acc;
            }
        }
        /* U_v = T V,  W = T diag(g) K */
        for (int64_t r = 0; r < n; ++r) {
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t s = 0; s <= r; ++s) acc += T[r * C + s] * vc[s * dv + j];
                Uv[r * dv + j] = acc;
            }
            for (int64_t i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int64_t s = 0; s <= r; ++s)
                    acc += T[r * C + s] * decay(alpha, 0, t0, s, -1, 0, dk) * kc[s * dk + i];
                W[r * dk + i] = acc;
            }
        }
        /* Q' = diag(g) Q - P W */
        for (int64_t r = 0; r < n; ++r) {
            const double g = decay(alpha, 0, t0, r, -1, 0, dk);
            for (int64_t i = 0; i < dk; ++i) {
                double acc = g * qc[r * dk + i];
                for (int64_t s = 0; s <= r; ++s) acc -= P[r * C + s] * W[s * dk + i];
                Qp[r * dk + i] = acc;
            }
        }
        /* the one product with S0: U = U_v - W S0, O = Q' S0 + P U_v */
        for (int64_t r = 0; r < n; ++r)
            for (int64_t j = 0; j < dv; ++j) {
                double ws = 0.0, qs = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    ws += W[r * dk + i] * S[IDX2(i, j, dv)];
                    qs += Qp[r * dk + i] * S[IDX2(i, j, dv)];
                }
                U[r * dv + j] = Uv[r * dv + j] - ws;
                double pu = 0.0;
                for (int64_t s = 0; s <= r; ++s) pu += P[r * C + s] * Uv[s * dv + j];
                o[(t0 + r) * dv + j] = qs + pu;
            }
        /* S_n = g_{n-1} S0 + sum_s beta_s (g_{n-1}/g_s) k_s u_s^T */
        const double gn = decay(alpha, 0, t0, n - 1, -1, 0, dk);
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) {
                double acc = gn * S[IDX2(i, j, dv)];
                for (int64_t s = 0; s < n; ++s)
                    acc += bc[s] * decay(alpha, 0, t0, n - 1, s, 0, dk) * kc[s * dk + i] * U[s * dv + j];
                Snew[IDX2(i, j, dv)] = acc;
            }
        memcpy(S, Snew, sizeof(double) * dk * dv);
    }
    free(A); free(T); free(P); free(Uv); free(U); free(W); free(Qp);
    return 0;
}

#define UNIT_PTRS(u)                                                                     \
    const double* qu = q + (u) * L * dk;                                                 \
    const double* ku = k + (u) * L * dk;                                                 \
    const double* vu = v + (u) * L * dv;                                                 \
    const double* au = alpha + (u) * L * (per_key ? dk : 1);                             \
    const double* bu = beta + (u) * L;                                                   \
    const double* s0u = S0 ? S0 + (u) * dk * dv : NULL;                                  \
    double* ou = o + (u) * L * dv;                                                       \
    double* su = S_out + (u) * dk * dv;

static int set_threads(int nthreads)
{
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

int gdr_ref_threads(int nthreads) { return set_threads(nthreads); }

int gdr_ref_sequential(int64_t U, int64_t L, int64_t dk, int64_t dv, int per_key,
                       const double* q, const double* k, const double* v,
                       const double* alpha, const double* beta, const double* S0,
                       double* o, double* S_out, int nthreads)
{
    if (U < 0 || L < 0 || dk <= 0 || dv <= 0) return -1;
    int failed = 0;
    const int nt = set_threads(nthreads);
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(|:failed)
    for (int64_t u = 0; u < U; ++u) {
        UNIT_PTRS(u)
        double* e = (double*)malloc(sizeof(double) * dv);
        if (!e) { failed |= 1; continue; }
        seq_unit(L, dk, dv, per_key, qu, ku, vu, au, bu, s0u, ou, su, e);
        free(e);
    }
    return failed ? -2 : 0;
}

int gdr_ref_dense(int64_t U, int64_t L, int64_t dk, int64_t dv, int per_key,
                  const double* q, const double* k, const double* v,
                  const double* alpha, const double* beta, const double* S0,
                  double* o, double* S_out, int nthreads)
{
    if (U < 0 || L < 0 || dk <= 0 || dv <= 0) return -1;
    int failed = 0;
    const int nt = set_threads(nthreads);
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(|:failed)
    for (int64_t u = 0; u < U; ++u) {
        UNIT_PTRS(u)
        double* A = (double*)malloc(sizeof(double) * dk * dk);
        double* Sn = (double*)malloc(sizeof(double) * dk * dv);
        if (!A || !Sn) { free(A); free(Sn); failed |= 1; continue; }
        dense_unit(L, dk, dv, per_key, qu, ku, vu, au, bu, s0u, ou, su, A, Sn);
        free(A);
        free(Sn);
    }
    return failed ? -2 : 0;
}

/* form: 0 = u-form (scalar gating only), 1 = e-form (either gating), 2 = u-form in its WY
   arrangement (scalar gating only). */
int gdr_ref_chunked(int64_t U, int64_t L, int64_t dk, int64_t dv, int per_key, int64_t C,
                    int form, const double* q, const double* k, const double* v,
                    const double* alpha, const double* beta, const double* S0,
                    double* o, double* S_out, int nthreads)
{
    if (U < 0 || L < 0 || dk <= 0 || dv <= 0 || C <= 0) return -1;
    if ((form == 0 || form == 2) && per_key) return -1;
    int failed = 0;
    const int nt = set_threads(nthreads);
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(|:failed)
    for (int64_t u = 0; u < U; ++u) {
        UNIT_PTRS(u)
        double* E  = (double*)malloc(sizeof(double) * C * dv);
        double* M1 = (double*)calloc((size_t)(C * C), sizeof(double));
        double* M2 = (double*)calloc((size_t)(C * C), sizeof(double));
        double* Sn = (double*)malloc(sizeof(double) * dk * dv);
        if (!E || !M1 || !M2 || !Sn) {
            free(E); free(M1); free(M2); free(Sn);
            failed |= 1;
            continue;
        }
        if (form == 2)
            failed |= chunked_unit_wyform(L, dk, dv, C, qu, ku, vu, au, bu, s0u, ou, su, Sn) != 0;
        else if (form == 0)
            chunked_unit_uform(L, dk, dv, C, qu, ku, vu, au, bu, s0u, ou, su, E, M1, Sn);
        else
            chunked_unit_eform(L, dk, dv, per_key, C, qu, ku, vu, au, bu, s0u, ou, su, E, M1, M2, Sn);
        free(E); free(M1); free(M2); free(Sn);
    }
    return failed ? -2 : 0;
}
