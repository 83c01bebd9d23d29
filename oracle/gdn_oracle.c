/*
 * gdn_oracle.c -- plain fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link, load or call this file.  Only
 * the tests, the smoke check and the CPU-baseline leg of the benchmark use
 * it.  It shares no code, header, helper or constant with the CUDA path.
 *
 * What it computes (the sources are the web pages this project is built
 * from):
 *
 *   "Architecture Thread I: Gated Attention, DeltaNet, and Hybrid Models",
 *   section "Gated DeltaNet":  S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T))
 *   + beta_t v_t k_t^T, and the read-out o_t = S_t q_t used with the same
 *   state orientation in the linear-attention recurrences of
 *   "Gated Attention Architectures", section 1 (GLA) and section 3
 *   (Gated DeltaNet, "Mathematical Formulation").
 *
 * Conventions (the readings of the pages this oracle takes):
 *   - S is d_v x d_k (row = value index, key index fastest), o_t = S_t q_t.
 *   - alpha_t = exp(g_t); g and beta are given per token per VALUE head.
 *   - value head h reads query/key head h / (Hv / Hk) (contiguous groups).
 *   - q and k are used exactly as given (no renormalisation, no scale).
 *   - sequences are independent; each has its own initial / final state;
 *     a NULL initial state means zeros.
 *   - the output at t reads the state AFTER the update at t.
 *
 * Three independent formulations live here:
 *   gdn_oracle_recurrent   -- the token recurrence (the oracle proper).
 *   gdn_oracle_chunkwise   -- the chunked form with a per-chunk cumulative
 *                             decay and the WY/UT triangular factor, derived
 *                             from the recurrence ("Gated Attention
 *                             Architectures", sections 2 and 3: the WY
 *                             representation and the per-chunk cumulative
 *                             decay products; the output follows the GLA
 *                             chunkwise form of section 1 with a
 *                             decay-aware causal mask).
 *   gdn_oracle_delta_error_form -- DeltaNet written as the error-correcting
 *                             write S <- S - beta (S k - v) k^T
 *                             ("Architecture Thread I", the delta-rule
 *                             update), with no gate.
 *   gdn_oracle_kda_recurrent / gdn_oracle_kda_chunkwise -- Kimi Delta
 *                             Attention ("Gated Attention Architectures",
 *                             section 8): one decay per key channel; the
 *                             token recurrence and an independent chunked
 *                             form derived from it.
 * and the mixer's two sides around the recurrence:
 *   gdn_oracle_prepare       -- q, k L2-normalised per head; gates from
 *                             their logits (the input side).
 *   gdn_oracle_output_side   -- RMS normalisation of each output row with a
 *                             scale and an optional SiLU or sigmoid gate
 *                             (the output side).
 *
 * Layouts (all row-major, token-major, fp64):
 *   q, k          [T_total, Hk, d_k]
 *   v, o          [T_total, Hv, d_v]
 *   g, beta       [T_total, Hv]
 *   s0, s_final   [N, Hv, d_v, d_k]
 *   cu_seqlens    int64 [N + 1]; sequence n holds tokens [cu[n], cu[n+1])
 * A "unit" is one (sequence n, value head h) pair, numbered n * Hv + h.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t num_seqs;
    const int64_t *cu_seqlens;
    int32_t hk, hv, dk, dv;
    const double *q, *k, *v, *g, *beta;
    const double *s0;   /* may be NULL: zero initial state */
    double *o;          /* may be NULL: outputs not wanted */
    double *s_final;    /* may be NULL */
} gdn_oracle_problem;

/* Optional per-chunk intermediates of the chunkwise form, indexed by the
 * global chunk number (sequences in order, chunks in order inside each
 * sequence; a tail chunk keeps its C-row slot with the unused rows left
 * untouched).  Any pointer may be NULL.
 *   gcum  [chunks, Hv, C]          cumulative log-decay G inside the chunk
 *   tmat  [chunks, Hv, C, C]       T = (I + A)^-1
 *   w     [chunks, Hv, C, d_k]     W = T diag(beta * gamma) K
 *   ut    [chunks, Hv, C, d_v]     U~ = T diag(beta) V
 *   u     [chunks, Hv, C, d_v]     U = U~ - W S0^T
 *   sc    [chunks, Hv, d_v, d_k]   state at the start of the chunk      */
typedef struct {
    int32_t chunk;
    double *gcum, *tmat, *w, *ut, *u, *sc;
} gdn_oracle_chunk_out;

static int64_t seq_len_of(const gdn_oracle_problem *p, int64_t n) {
    return p->cu_seqlens[n + 1] - p->cu_seqlens[n];
}

/* ------------------------------------------------------------------ */
/* 1. Token recurrence.                                                 */
/* ------------------------------------------------------------------ */
static void recurrent_unit(const gdn_oracle_problem *p, int64_t unit, double *S, double *pk) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv;

    if (p->s0) memcpy(S, p->s0 + unit * (int64_t)dv * dk, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);

    for (int64_t t = p->cu_seqlens[n]; t < p->cu_seqlens[n + 1]; ++t) {
        const double *kt = p->k + (t * p->hk + hq) * dk;
        const double *qt = p->q + (t * p->hk + hq) * dk;
        const double *vt = p->v + (t * p->hv + h) * dv;
        const double alpha = exp(p->g[t * p->hv + h]);
        const double beta = p->beta[t * p->hv + h];

        /* prediction of the old memory for key k_t: S_{t-1} k_t */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * kt[j];
            pk[i] = acc;
        }
        /* S_t = alpha S_{t-1} (I - beta k k^T) + beta v k^T
         *     = alpha S_{t-1} + beta (v - alpha S_{t-1} k) k^T            */
        for (int i = 0; i < dv; ++i) {
            const double ui = beta * (vt[i] - alpha * pk[i]);
            for (int j = 0; j < dk; ++j) S[i * dk + j] = alpha * S[i * dk + j] + ui * kt[j];
        }
        /* o_t = S_t q_t */
        if (p->o) {
            double *ot = p->o + (t * p->hv + h) * dv;
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qt[j];
                ot[i] = acc;
            }
        }
    }
    if (p->s_final) memcpy(p->s_final + unit * (int64_t)dv * dk, S, sizeof(double) * dv * dk);
}

/* ------------------------------------------------------------------ */
/* 2. DeltaNet in its error-correcting form (no decay gate).            */
/* ------------------------------------------------------------------ */
static void delta_error_unit(const gdn_oracle_problem *p, int64_t unit, double *S, double *err) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv;

    if (p->s0) memcpy(S, p->s0 + unit * (int64_t)dv * dk, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);

    for (int64_t t = p->cu_seqlens[n]; t < p->cu_seqlens[n + 1]; ++t) {
        const double *kt = p->k + (t * p->hk + hq) * dk;
        const double *qt = p->q + (t * p->hk + hq) * dk;
        const double *vt = p->v + (t * p->hv + h) * dv;
        const double beta = p->beta[t * p->hv + h];
        /* error = S k - v */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * kt[j];
            err[i] = acc - vt[i];
        }
        /* S <- S - beta * error * k^T */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) S[i * dk + j] -= beta * err[i] * kt[j];
        if (p->o) {
            double *ot = p->o + (t * p->hv + h) * dv;
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qt[j];
                ot[i] = acc;
            }
        }
    }
    if (p->s_final) memcpy(p->s_final + unit * (int64_t)dv * dk, S, sizeof(double) * dv * dk);
}

/* ------------------------------------------------------------------ */
/* 3. Chunkwise form.                                                   */
/*                                                                      */
/* Inside a chunk of L <= C tokens r = 0..L-1 with start state S0:      */
/*   G_r   = g_0 + ... + g_r          (cumulative log-decay)             */
/*   gamma_r = exp(G_r),  Gamma_rj = exp(G_r - G_j) for j <= r          */
/*   unrolling S_r = alpha_r S_{r-1} + u_r k_r^T with                   */
/*   u_r = beta_r (v_r - alpha_r S_{r-1} k_r) gives                     */
/*   (I + A) U = diag(beta) V - diag(beta gamma) K S0^T,                */
/*   A_rj = beta_r Gamma_rj (k_r . k_j) for j < r (strictly lower), so  */
/*   U = T diag(beta) V - T diag(beta gamma) K S0^T = U~ - W S0^T,       */
/*   T = (I + A)^-1;  then                                              */
/*   O = diag(gamma) Q S0^T + (Q K^T (.) Gamma) U                        */
/*   S_L = gamma_{L-1} S0 + U^T diag(exp(G_{L-1} - G)) K.                */
/* ------------------------------------------------------------------ */
typedef struct {
    double *S, *G, *A, *T, *W, *Ut, *U, *Kc, *Qc, *Vc;
} chunk_scratch;

static void chunkwise_unit(const gdn_oracle_problem *p, const gdn_oracle_chunk_out *co,
                           int64_t unit, chunk_scratch *sc, int64_t chunk_base) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv, C = co->chunk;
    double *S = sc->S, *G = sc->G, *A = sc->A, *T = sc->T, *W = sc->W, *Ut = sc->Ut, *U = sc->U;
    double *K = sc->Kc, *Q = sc->Qc, *V = sc->Vc;

    if (p->s0) memcpy(S, p->s0 + unit * (int64_t)dv * dk, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);

    const int64_t t_begin = p->cu_seqlens[n], t_end = p->cu_seqlens[n + 1];
    int64_t chunk_idx = chunk_base;
    for (int64_t c0 = t_begin; c0 < t_end; c0 += C, ++chunk_idx) {
        const int L = (int)((t_end - c0) < C ? (t_end - c0) : C);
        const int64_t slot = chunk_idx * p->hv + h;
        if (co->sc) memcpy(co->sc + slot * (int64_t)dv * dk, S, sizeof(double) * dv * dk);

        /* gather this chunk's rows */
        for (int r = 0; r < L; ++r) {
            const int64_t t = c0 + r;
            memcpy(K + r * dk, p->k + (t * p->hk + hq) * dk, sizeof(double) * dk);
            memcpy(Q + r * dk, p->q + (t * p->hk + hq) * dk, sizeof(double) * dk);
            memcpy(V + r * dv, p->v + (t * p->hv + h) * dv, sizeof(double) * dv);
        }
        /* cumulative log-decay */
        double run = 0.0;
        for (int r = 0; r < L; ++r) {
            run += p->g[(c0 + r) * p->hv + h];
            G[r] = run;
        }
        /* A (strictly lower) */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double a = 0.0;
                if (j < r) {
                    double kk = 0.0;
                    for (int x = 0; x < dk; ++x) kk += K[r * dk + x] * K[j * dk + x];
                    a = p->beta[(c0 + r) * p->hv + h] * exp(G[r] - G[j]) * kk;
                }
                A[r * L + j] = a;
            }
        /* T = (I + A)^-1 by forward substitution: row r of (I + A) T = I
         * gives T_r = e_r - sum_{j<r} A_rj T_j.                          */
        for (int r = 0; r < L; ++r)
            for (int c = 0; c < L; ++c) {
                double x = (r == c) ? 1.0 : 0.0;
                for (int j = 0; j < r; ++j) x -= A[r * L + j] * T[j * L + c];
                T[r * L + c] = x;
            }
        /* W = T diag(beta gamma) K ;  U~ = T diag(beta) V */
        for (int r = 0; r < L; ++r) {
            for (int x = 0; x < dk; ++x) {
                double acc = 0.0;
                for (int j = 0; j < L; ++j)
                    acc += T[r * L + j] * p->beta[(c0 + j) * p->hv + h] * exp(G[j]) * K[j * dk + x];
                W[r * dk + x] = acc;
            }
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < L; ++j)
                    acc += T[r * L + j] * p->beta[(c0 + j) * p->hv + h] * V[j * dv + i];
                Ut[r * dv + i] = acc;
            }
        }
        /* U = U~ - W S0^T */
        for (int r = 0; r < L; ++r)
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int x = 0; x < dk; ++x) acc += W[r * dk + x] * S[i * dk + x];
                U[r * dv + i] = Ut[r * dv + i] - acc;
            }
        /* O = diag(gamma) Q S0^T + (Q K^T (.) Gamma) U */
        if (p->o) {
            for (int r = 0; r < L; ++r) {
                double *ot = p->o + ((c0 + r) * p->hv + h) * dv;
                for (int i = 0; i < dv; ++i) {
                    double inter = 0.0;
                    for (int x = 0; x < dk; ++x) inter += Q[r * dk + x] * S[i * dk + x];
                    double intra = 0.0;
                    for (int j = 0; j <= r; ++j) {
                        double qk = 0.0;
                        for (int x = 0; x < dk; ++x) qk += Q[r * dk + x] * K[j * dk + x];
                        intra += qk * exp(G[r] - G[j]) * U[j * dv + i];
                    }
                    ot[i] = exp(G[r]) * inter + intra;
                }
            }
        }
        /* S_L = gamma_{L-1} S0 + U^T diag(exp(G_{L-1} - G)) K */
        const double gl = G[L - 1];
        for (int i = 0; i < dv; ++i)
            for (int x = 0; x < dk; ++x) {
                double acc = 0.0;
                for (int j = 0; j < L; ++j) acc += U[j * dv + i] * exp(gl - G[j]) * K[j * dk + x];
                S[i * dk + x] = exp(gl) * S[i * dk + x] + acc;
            }

        if (co->gcum) memcpy(co->gcum + slot * C, G, sizeof(double) * L);
        if (co->tmat)
            for (int r = 0; r < L; ++r) memcpy(co->tmat + (slot * C + r) * C, T + r * L, sizeof(double) * L);
        if (co->w) memcpy(co->w + slot * (int64_t)C * dk, W, sizeof(double) * L * dk);
        if (co->ut) memcpy(co->ut + slot * (int64_t)C * dv, Ut, sizeof(double) * L * dv);
        if (co->u) memcpy(co->u + slot * (int64_t)C * dv, U, sizeof(double) * L * dv);
    }
    if (p->s_final) memcpy(p->s_final + unit * (int64_t)dv * dk, S, sizeof(double) * dv * dk);
}

/* ------------------------------------------------------------------ */
/* 4. Kimi Delta Attention (KDA): one decay per key channel.            */
/* ------------------------------------------------------------------ */
/* "Gated Attention Architectures", section 8 (Kimi Delta Attention),
 * "Mathematical Formulation": S_t = (I - beta_t k_t k_t^T) D_t S_{t-1}
 * + beta_t k_t v_t^T and o_t = S_t^T q_t, with D_t = diag(alpha_t) holding
 * one decay per key channel.  That page's state is d_k x d_v; in this
 * oracle's orientation (d_v x d_k, the transpose) the same update reads
 *     S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,
 * so each row s of S becomes s' = alpha_t .* s, then
 * s <- s' + beta_t (v_i - s' . k_t) k_t.  With every alpha_t[c] equal this
 * is the gated delta rule above (the page: KDA reduces to Gated DeltaNet
 * when the decay collapses to a scalar).
 * g is read as [T, Hv, d_k]: alpha_t[c] = exp(g[t, h, c]). */
static int kda_recurrent_unit(const gdn_oracle_problem *p, int64_t unit, double *S) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv;
    double *alpha = malloc(sizeof(double) * dk);
    double *sd = malloc(sizeof(double) * dk);
    if (!alpha || !sd) {
        free(alpha);
        free(sd);
        return -1;
    }
    if (p->s0) memcpy(S, p->s0 + unit * (int64_t)dv * dk, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);
    for (int64_t t = p->cu_seqlens[n]; t < p->cu_seqlens[n + 1]; ++t) {
        const double *kt = p->k + (t * p->hk + hq) * dk;
        const double *qt = p->q + (t * p->hk + hq) * dk;
        const double *vt = p->v + (t * p->hv + h) * dv;
        const double *gt = p->g + (t * p->hv + h) * dk;
        const double beta = p->beta[t * p->hv + h];
        for (int j = 0; j < dk; ++j) alpha[j] = exp(gt[j]);
        for (int i = 0; i < dv; ++i) {
            /* the decayed row S_{t-1} D_t, and its prediction for k_t */
            double pred = 0.0;
            for (int j = 0; j < dk; ++j) {
                sd[j] = alpha[j] * S[i * dk + j];
                pred += sd[j] * kt[j];
            }
            const double ui = beta * (vt[i] - pred);
            for (int j = 0; j < dk; ++j) S[i * dk + j] = sd[j] + ui * kt[j];
        }
        if (p->o) {
            double *ot = p->o + (t * p->hv + h) * dv;
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qt[j];
                ot[i] = acc;
            }
        }
    }
    if (p->s_final) memcpy(p->s_final + unit * (int64_t)dv * dk, S, sizeof(double) * dv * dk);
    free(alpha);
    free(sd);
    return 0;
}

/* KDA in chunks of C tokens, derived here from the recurrence above (the
 * page names a chunkwise WY algorithm with the decay absorbed into the keys;
 * it prints none).  Within a chunk with start state S0 and the per-channel
 * cumulative log-decay G_r[c] = g_0[c] + ... + g_r[c]:
 *   S_r = S0 diag(e^{G_r}) + sum_{j<=r} u_j (k_j .* e^{G_r - G_j})^T
 *   u_r = beta_r (v_r - S_{r-1} D_r k_r), which unrolls to
 *   (I + A) U = diag(beta) V - diag(beta) K+ S0^T with
 *   A_rj = beta_r sum_c k_r[c] k_j[c] e^{G_r[c] - G_j[c]}  (j < r),
 *   K+_r = k_r .* e^{G_r};  so U = T diag(beta) V - T diag(beta) K+ S0^T,
 *   T = (I + A)^-1;
 *   o_r = S0 (q_r .* e^{G_r}) + sum_{j<=r} (sum_c q_r[c] k_j[c] e^{G_r[c] - G_j[c]}) u_j;
 *   S_C = S0 diag(e^{G_last}) + sum_j u_j (k_j .* e^{G_last - G_j})^T.
 * Every exponent above is a difference G_r - G_j with j <= r (or G itself),
 * so with g <= 0 nothing overflows; the masked products are formed term by
 * term, not as products of separately scaled matrices. */
static int kda_chunk_unit(const gdn_oracle_problem *p, int C, int64_t unit, double *S) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv;
    double *G = malloc(sizeof(double) * C * dk);
    double *A = malloc(sizeof(double) * C * C);
    double *T = malloc(sizeof(double) * C * C);
    double *W = malloc(sizeof(double) * C * dk);
    double *U = malloc(sizeof(double) * C * dv);
    double *O = malloc(sizeof(double) * C * dv);
    double *Sn = malloc(sizeof(double) * dv * dk);
    int rc = 0;
    if (!G || !A || !T || !W || !U || !O || !Sn) {
        rc = -1;
        goto done;
    }
    if (p->s0) memcpy(S, p->s0 + unit * (int64_t)dv * dk, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);
    const int64_t t_begin = p->cu_seqlens[n], t_end = p->cu_seqlens[n + 1];
    for (int64_t c0 = t_begin; c0 < t_end; c0 += C) {
        const int L = (int)((t_end - c0) < C ? (t_end - c0) : C);
#define KDA_K(r, c) p->k[((c0 + (r)) * p->hk + hq) * dk + (c)]
#define KDA_Q(r, c) p->q[((c0 + (r)) * p->hk + hq) * dk + (c)]
#define KDA_V(r, i) p->v[((c0 + (r)) * p->hv + h) * dv + (i)]
#define KDA_B(r) p->beta[(c0 + (r)) * p->hv + h]
        for (int r = 0; r < L; ++r)
            for (int c = 0; c < dk; ++c)
                G[r * dk + c] = (r ? G[(r - 1) * dk + c] : 0.0) + p->g[((c0 + r) * p->hv + h) * dk + c];
        /* A (strictly lower) and T = (I + A)^-1 by forward substitution */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double a = 0.0;
                if (j < r) {
                    for (int c = 0; c < dk; ++c) a += KDA_K(r, c) * KDA_K(j, c) * exp(G[r * dk + c] - G[j * dk + c]);
                    a *= KDA_B(r);
                }
                A[r * L + j] = a;
            }
        for (int col = 0; col < L; ++col)
            for (int r = 0; r < L; ++r) {
                double x = (r == col) ? 1.0 : 0.0;
                for (int j = col; j < r; ++j) x -= A[r * L + j] * T[j * L + col];
                T[r * L + col] = r < col ? 0.0 : x;
            }
        /* W = T diag(beta) K+ */
        for (int r = 0; r < L; ++r)
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int j = 0; j <= r; ++j) acc += T[r * L + j] * KDA_B(j) * KDA_K(j, c) * exp(G[j * dk + c]);
                W[r * dk + c] = acc;
            }
        /* U = T diag(beta) V - W S0^T */
        for (int r = 0; r < L; ++r)
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j <= r; ++j) acc += T[r * L + j] * KDA_B(j) * KDA_V(j, i);
                for (int c = 0; c < dk; ++c) acc -= W[r * dk + c] * S[i * dk + c];
                U[r * dv + i] = acc;
            }
        /* outputs from the chunk's start state and the corrected values */
        for (int r = 0; r < L; ++r)
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += S[i * dk + c] * KDA_Q(r, c) * exp(G[r * dk + c]);
                for (int j = 0; j <= r; ++j) {
                    double m = 0.0;
                    for (int c = 0; c < dk; ++c) m += KDA_Q(r, c) * KDA_K(j, c) * exp(G[r * dk + c] - G[j * dk + c]);
                    acc += m * U[j * dv + i];
                }
                O[r * dv + i] = acc;
            }
        if (p->o)
            for (int r = 0; r < L; ++r)
                memcpy(p->o + ((c0 + r) * p->hv + h) * dv, O + r * dv, sizeof(double) * dv);
        /* state at the end of the chunk */
        const double *Gl = G + (L - 1) * dk;
        for (int i = 0; i < dv; ++i)
            for (int c = 0; c < dk; ++c) {
                double acc = S[i * dk + c] * exp(Gl[c]);
                for (int j = 0; j < L; ++j) acc += U[j * dv + i] * KDA_K(j, c) * exp(Gl[c] - G[j * dk + c]);
                Sn[i * dk + c] = acc;
            }
        memcpy(S, Sn, sizeof(double) * dv * dk);
#undef KDA_K
#undef KDA_Q
#undef KDA_V
#undef KDA_B
    }
    if (p->s_final) memcpy(p->s_final + unit * (int64_t)dv * dk, S, sizeof(double) * dv * dk);
done:
    free(G); free(A); free(T); free(W); free(U); free(O); free(Sn);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Threading: units are independent, so threads take units round-robin. */
/* ------------------------------------------------------------------ */
enum { KIND_RECURRENT = 0, KIND_DELTA = 1, KIND_CHUNK = 2, KIND_KDA = 3, KIND_KDA_CHUNK = 4 };

typedef struct {
    int kind;
    const gdn_oracle_problem *p;
    const gdn_oracle_chunk_out *co;
    const int64_t *units;  /* NULL = all */
    int64_t n_units;
    const int64_t *chunk_base; /* per sequence, for KIND_CHUNK */
    int tid, nthreads;
    int failed;
} worker_arg;

static void *worker(void *vp) {
    worker_arg *a = (worker_arg *)vp;
    const gdn_oracle_problem *p = a->p;
    const int dk = p->dk, dv = p->dv;
    const int C = a->co ? a->co->chunk : 1;
    const int dm = dk > dv ? dk : dv;
    double *S = malloc(sizeof(double) * dv * dk);
    double *buf = malloc(sizeof(double) * (size_t)(dm + 8));
    chunk_scratch sc = {0};
    if (a->kind == KIND_CHUNK) {
        sc.S = S;
        sc.G = malloc(sizeof(double) * C);
        sc.A = malloc(sizeof(double) * C * C);
        sc.T = malloc(sizeof(double) * C * C);
        sc.W = malloc(sizeof(double) * C * dk);
        sc.Ut = malloc(sizeof(double) * C * dv);
        sc.U = malloc(sizeof(double) * C * dv);
        sc.Kc = malloc(sizeof(double) * C * dk);
        sc.Qc = malloc(sizeof(double) * C * dk);
        sc.Vc = malloc(sizeof(double) * C * dv);
        if (!sc.G || !sc.A || !sc.T || !sc.W || !sc.Ut || !sc.U || !sc.Kc || !sc.Qc || !sc.Vc) a->failed = 1;
    }
    if (!S || !buf) a->failed = 1;
    if (!a->failed) {
        for (int64_t i = a->tid; i < a->n_units; i += a->nthreads) {
            const int64_t unit = a->units ? a->units[i] : i;
            if (a->kind == KIND_RECURRENT) recurrent_unit(p, unit, S, buf);
            else if (a->kind == KIND_DELTA) delta_error_unit(p, unit, S, buf);
            else if (a->kind == KIND_KDA) a->failed |= kda_recurrent_unit(p, unit, S) != 0;
            else if (a->kind == KIND_KDA_CHUNK) a->failed |= kda_chunk_unit(p, a->co->chunk, unit, S) != 0;
            else chunkwise_unit(p, a->co, unit, &sc, a->chunk_base[unit / p->hv]);
        }
    }
    free(S);
    free(buf);
    if (a->kind == KIND_CHUNK) {
        free(sc.G); free(sc.A); free(sc.T); free(sc.W); free(sc.Ut); free(sc.U);
        free(sc.Kc); free(sc.Qc); free(sc.Vc);
    }
    return NULL;
}

static int validate(const gdn_oracle_problem *p) {
    if (!p || !p->cu_seqlens || p->num_seqs < 0) return -1;
    if (p->hk <= 0 || p->hv <= 0 || p->dk <= 0 || p->dv <= 0) return -1;
    if (p->hv % p->hk != 0) return -1;
    if (!p->q || !p->k || !p->v || !p->g || !p->beta) return -1;
    if (p->cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < p->num_seqs; ++n)
        if (seq_len_of(p, n) < 0) return -1;
    return 0;
}

static int run(int kind, const gdn_oracle_problem *p, const gdn_oracle_chunk_out *co,
               const int64_t *units, int64_t n_units, int n_threads) {
    if (validate(p) != 0) return -1;
    const int64_t total_units = p->num_seqs * p->hv;
    if (!units) n_units = total_units;
    for (int64_t i = 0; units && i < n_units; ++i)
        if (units[i] < 0 || units[i] >= total_units) return -1;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    if (n_threads > n_units && n_units > 0) n_threads = (int)n_units;

    if (kind == KIND_KDA_CHUNK && (!co || co->chunk <= 0)) return -1;
    int64_t *chunk_base = NULL;
    if (kind == KIND_CHUNK) {
        if (!co || co->chunk <= 0) return -1;
        chunk_base = malloc(sizeof(int64_t) * (size_t)(p->num_seqs + 1));
        if (!chunk_base) return -1;
        int64_t acc = 0;
        for (int64_t n = 0; n < p->num_seqs; ++n) {
            chunk_base[n] = acc;
            acc += (seq_len_of(p, n) + co->chunk - 1) / co->chunk;
        }
        chunk_base[p->num_seqs] = acc;
    }

    pthread_t th[256];
    worker_arg args[256];
    int failed = 0;
    for (int i = 0; i < n_threads; ++i) {
        args[i] = (worker_arg){kind, p, co, units, n_units, chunk_base, i, n_threads, 0};
        if (pthread_create(&th[i], NULL, worker, &args[i]) != 0) {
            args[i].failed = 1;
            worker(&args[i]); /* run inline: correctness over speed */
            args[i].failed = 0;
            th[i] = 0;
        }
    }
    for (int i = 0; i < n_threads; ++i) {
        if (th[i]) pthread_join(th[i], NULL);
        failed |= args[i].failed;
    }
    free(chunk_base);
    return failed ? -2 : 0;
}

/* Public entry points (called through ctypes by the tests). */
int gdn_oracle_recurrent(const gdn_oracle_problem *p, const int64_t *units, int64_t n_units, int n_threads) {
    return run(KIND_RECURRENT, p, NULL, units, n_units, n_threads);
}

int gdn_oracle_delta_error_form(const gdn_oracle_problem *p, const int64_t *units, int64_t n_units,
                                int n_threads) {
    return run(KIND_DELTA, p, NULL, units, n_units, n_threads);
}

int gdn_oracle_chunkwise(const gdn_oracle_problem *p, const gdn_oracle_chunk_out *co, const int64_t *units,
                         int64_t n_units, int n_threads) {
    return run(KIND_CHUNK, p, co, units, n_units, n_threads);
}

/* KDA: the problem's g is [T, Hv, d_k] (one log-decay per key channel). */
int gdn_oracle_kda_recurrent(const gdn_oracle_problem *p, const int64_t *units, int64_t n_units, int n_threads) {
    return run(KIND_KDA, p, NULL, units, n_units, n_threads);
}

int gdn_oracle_kda_chunkwise(const gdn_oracle_problem *p, int32_t chunk, const int64_t *units, int64_t n_units,
                             int n_threads) {
    gdn_oracle_chunk_out co = {chunk, NULL, NULL, NULL, NULL, NULL, NULL};
    return run(KIND_KDA_CHUNK, p, &co, units, n_units, n_threads);
}

/* Number of chunks the chunkwise form uses (size of its intermediates). */
int64_t gdn_oracle_num_chunks(const int64_t *cu_seqlens, int64_t num_seqs, int32_t chunk) {
    int64_t acc = 0;
    for (int64_t n = 0; n < num_seqs; ++n) acc += (cu_seqlens[n + 1] - cu_seqlens[n] + chunk - 1) / chunk;
    return acc;
}

/* The input side of the mixer, for callers that hand over raw projections
 * ("Gated Attention Architectures", the Gated DeltaNet code listing: q and k
 * L2-normalised per head, the decay gate and the write gate as sigmoids of
 * per-head logits; "Architecture Thread I", "Modern Architecture
 * Improvements": L2 normalisation keeps ||k|| = 1 so that the transition's
 * eigenvalue along k, 1 - beta ||k||^2, stays in (0, 1), and beta comes from
 * a sigmoid).  In place, fp64, every array token-major as above.
 *   prep_flags & 2 : q[t, h, :] <- q / max(||q||_2, 1e-12), the same for k
 *   prep_flags & 4 : g[t, h] holds the decay logit a; alpha = sigmoid(a), so
 *                    the log-decay becomes g = log sigmoid(a) (written as
 *                    -log1p(e^-a) for a >= 0 and a - log1p(e^a) below, which
 *                    are the same function); beta[t, h] holds the write
 *                    logit b and becomes sigmoid(b) = 1 / (1 + e^-b).       */
void gdn_oracle_prepare(int64_t tokens, int32_t hk, int32_t hv, int32_t dk, double *q, double *k, double *g,
                        double *beta, uint32_t prep_flags) {
    if (prep_flags & 2u) {
        double *xs[2] = {q, k};
        for (int which = 0; which < 2; ++which) {
            double *x = xs[which];
            for (int64_t r = 0; r < tokens * hk; ++r) {
                double ss = 0.0;
                for (int32_t i = 0; i < dk; ++i) ss += x[r * dk + i] * x[r * dk + i];
                const double nrm = sqrt(ss);
                const double den = nrm > 1e-12 ? nrm : 1e-12;
                for (int32_t i = 0; i < dk; ++i) x[r * dk + i] /= den;
            }
        }
    }
    if (prep_flags & 4u) {
        for (int64_t r = 0; r < tokens * hv; ++r) {
            const double a = g[r];
            g[r] = a >= 0.0 ? -log1p(exp(-a)) : a - log1p(exp(a));
            beta[r] = 1.0 / (1.0 + exp(-beta[r]));
        }
    }
}

/* The mixer's output side, applied to the read-out o of the recurrence.
 * "Architecture Thread I", "Modern Architecture Improvements": the mixer's
 * output is RMS-normalised before the output projection (in place of a
 * softmax-style denominator).  "The Transformer Isn't Alone Anymore" lists
 * a gated RMSNorm in the Gated DeltaNet block; the Gated DeltaNet code
 * listing of "Gated Attention Architectures" multiplies the normalised
 * output by SiLU of a gate projection; the Gated Attention section of the
 * same page names the sigmoid gate; the Qwen3-Next passage of "Architecture
 * Thread I" holds the norm's scale as 1 + delta ("zero-centred").
 * For every (token, value head) row o of d_v values:
 *     ms  = (1 / d_v) sum_j o_j^2
 *     y_i = o_i / sqrt(ms + eps) * s_i * act(z_i)
 *   out_flags & 1 : act(z) = z / (1 + e^-z)      (SiLU)
 *   out_flags & 2 : act(z) = 1 / (1 + e^-z)      (sigmoid)
 *   neither       : act = 1 and z is not read
 *   out_flags & 4 : s_i = 1 + w_i (zero-centred; w NULL reads as 0)
 *   otherwise     : s_i = w_i (w NULL reads as 1)
 *   out_flags & 8 : w is [Hv, d_v], a row per value head; otherwise [d_v]
 * o, z, y are [tokens, Hv, d_v]; y may alias o. */
void gdn_oracle_output_side(int64_t tokens, int32_t hv, int32_t dv, const double *o, const double *z,
                            const double *w, double eps, uint32_t out_flags, double *y) {
    for (int64_t t = 0; t < tokens; ++t) {
        for (int32_t h = 0; h < hv; ++h) {
            const int64_t row = (t * hv + h) * dv;
            double ms = 0.0;
            for (int32_t i = 0; i < dv; ++i) ms += o[row + i] * o[row + i];
            ms /= dv;
            const double inv_rms = 1.0 / sqrt(ms + eps);
            const double *wr = w ? w + ((out_flags & 8u) ? (int64_t)h * dv : 0) : NULL;
            for (int32_t i = 0; i < dv; ++i) {
                double s;
                if (out_flags & 4u) s = 1.0 + (wr ? wr[i] : 0.0);
                else s = wr ? wr[i] : 1.0;
                double gate = 1.0;
                if (out_flags & 1u) gate = z[row + i] / (1.0 + exp(-z[row + i]));
                else if (out_flags & 2u) gate = 1.0 / (1.0 + exp(-z[row + i]));
                y[row + i] = o[row + i] * inv_rms * s * gate;
            }
        }
    }
}
