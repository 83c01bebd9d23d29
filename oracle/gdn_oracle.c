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
 * Independent formulations live here:
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
 *   gdn_oracle_backward / gdn_oracle_backward_chunkwise -- the gradients:
 *                             the reverse mode of the token recurrence, and
 *                             an independent derivation through the chunk
 *                             forms.
 * and the mixer's two sides around the recurrence:
 *   gdn_oracle_short_conv    -- the short causal depthwise convolution of
 *                             the projections, with an optional SiLU, and
 *                             its per-sequence conv state (the input side).
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

/* ------------------------------------------------------------------ */
/* 5. Gradients (training).                                             */
/* ------------------------------------------------------------------ */
/* The pages frame the chunkwise algorithm as the way to train the layer
 * ("Architecture Thread I", the DeltaNet/Gated DeltaNet training remarks;
 * "Gated Attention Architectures", sections 2 and 3).  For upstream
 * gradients dO (of every output) and dS_T (of each final state) these are
 * the gradients of L = sum dO . O + sum dS_T . S_T with respect to q, k, v,
 * g, beta and the initial state.
 *
 * gdn_oracle_backward: reverse mode of the token recurrence, written out
 * by hand.  Per token, with s' = alpha S_{t-1}, p = s' k, u = beta (v - p),
 * S_t = s' + u k^T, o = S_t q (row form of the forward above), and dS the
 * gradient of S_t accumulated from later tokens:
 *   dS += dO_t q^T;              dq += S_t^T dO_t
 *   du = dS k;                    dk += dS^T u
 *   dbeta += du . (v - p);        dv = beta du;      dp = -beta du
 *   ds' = dS + dp k^T;            dk += s'^T dp
 *   dalpha = <ds', S_{t-1}>;      dg = alpha dalpha; dS_{t-1} = alpha ds'
 * dq and dk are returned per VALUE head ([T, Hv, d_k]): summing the heads of
 * a group gives the gradient of the shared q/k head. */
typedef struct {
    const double *dO;   /* [T, Hv, dv] */
    const double *dSf;  /* [N, Hv, dv, dk] or NULL (zero) */
    double *dq, *dk;    /* [T, Hv, dk] */
    double *dv;         /* [T, Hv, dv] */
    double *dg, *dbeta; /* [T, Hv] */
    double *dS0;        /* [N, Hv, dv, dk] or NULL */
} gdn_oracle_grads;

static int backward_unit(const gdn_oracle_problem *p, const gdn_oracle_grads *gr, int64_t unit) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv;
    const int64_t t0 = p->cu_seqlens[n], T = p->cu_seqlens[n + 1] - t0;
    const size_t ssz = (size_t)dv * dk;
    double *Sh = malloc(sizeof(double) * ssz * (size_t)(T + 1)); /* S_{-1} .. S_{T-1} */
    double *dS = malloc(sizeof(double) * ssz);
    double *dsp = malloc(sizeof(double) * ssz);
    double *pk = malloc(sizeof(double) * dv), *u = malloc(sizeof(double) * dv), *du = malloc(sizeof(double) * dv);
    if (!Sh || !dS || !dsp || !pk || !u || !du) {
        free(Sh); free(dS); free(dsp); free(pk); free(u); free(du);
        return -1;
    }
    if (p->s0) memcpy(Sh, p->s0 + unit * (int64_t)ssz, sizeof(double) * ssz);
    else memset(Sh, 0, sizeof(double) * ssz);
    for (int64_t t = 0; t < T; ++t) { /* forward, keeping every state */
        const int64_t tt = t0 + t;
        const double *kt = p->k + (tt * p->hk + hq) * dk;
        const double *vt = p->v + (tt * p->hv + h) * dv;
        const double alpha = exp(p->g[tt * p->hv + h]), beta = p->beta[tt * p->hv + h];
        const double *Sp = Sh + ssz * t;
        double *Sn = Sh + ssz * (t + 1);
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += alpha * Sp[i * dk + j] * kt[j];
            const double ui = beta * (vt[i] - acc);
            for (int j = 0; j < dk; ++j) Sn[i * dk + j] = alpha * Sp[i * dk + j] + ui * kt[j];
        }
    }
    if (gr->dSf) memcpy(dS, gr->dSf + unit * (int64_t)ssz, sizeof(double) * ssz);
    else memset(dS, 0, sizeof(double) * ssz);
    for (int64_t t = T - 1; t >= 0; --t) {
        const int64_t tt = t0 + t;
        const double *kt = p->k + (tt * p->hk + hq) * dk;
        const double *qt = p->q + (tt * p->hk + hq) * dk;
        const double *vt = p->v + (tt * p->hv + h) * dv;
        const double *dOt = gr->dO + (tt * p->hv + h) * dv;
        const double alpha = exp(p->g[tt * p->hv + h]), beta = p->beta[tt * p->hv + h];
        const double *Sp = Sh + ssz * t, *St = Sh + ssz * (t + 1);
        double *dqt = gr->dq + (tt * p->hv + h) * dk, *dkt = gr->dk + (tt * p->hv + h) * dk;
        double *dvt = gr->dv + (tt * p->hv + h) * dv;
        for (int j = 0; j < dk; ++j) {
            dqt[j] = 0.0;
            dkt[j] = 0.0;
        }
        /* o = S_t q */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) {
                dS[i * dk + j] += dOt[i] * qt[j];
                dqt[j] += St[i * dk + j] * dOt[i];
            }
        /* the forward quantities of this token */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += alpha * Sp[i * dk + j] * kt[j];
            pk[i] = acc;
            u[i] = beta * (vt[i] - acc);
        }
        double dbeta = 0.0, dalpha = 0.0;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += dS[i * dk + j] * kt[j];
            du[i] = acc;
            dbeta += acc * (vt[i] - pk[i]);
            dvt[i] = beta * acc;
        }
        for (int i = 0; i < dv; ++i) {
            const double dpi = -beta * du[i];
            for (int j = 0; j < dk; ++j) {
                dkt[j] += u[i] * dS[i * dk + j] + dpi * alpha * Sp[i * dk + j];
                dsp[i * dk + j] = dS[i * dk + j] + dpi * kt[j];
                dalpha += dsp[i * dk + j] * Sp[i * dk + j];
            }
        }
        for (size_t e = 0; e < ssz; ++e) dS[e] = alpha * dsp[e];
        gr->dbeta[tt * p->hv + h] = dbeta;
        gr->dg[tt * p->hv + h] = alpha * dalpha;
    }
    if (gr->dS0) memcpy(gr->dS0 + unit * (int64_t)ssz, dS, sizeof(double) * ssz);
    free(Sh); free(dS); free(dsp); free(pk); free(u); free(du);
    return 0;
}

typedef struct {
    const gdn_oracle_problem *p;
    const gdn_oracle_grads *gr;
    int32_t chunk; /* 0: token recurrence; > 0: the chunked form */
    int tid, nthreads, failed;
} bwd_arg;

static int backward_chunk_unit(const gdn_oracle_problem *p, const gdn_oracle_grads *gr, int64_t unit, int C);

static void *bwd_worker(void *vp) {
    bwd_arg *a = (bwd_arg *)vp;
    const int64_t units = a->p->num_seqs * a->p->hv;
    for (int64_t u = a->tid; u < units; u += a->nthreads) {
        const int rc = a->chunk > 0 ? backward_chunk_unit(a->p, a->gr, u, a->chunk) : backward_unit(a->p, a->gr, u);
        if (rc != 0) a->failed = 1;
    }
    return NULL;
}

static int run_backward(const gdn_oracle_problem *p, const gdn_oracle_grads *gr, int32_t chunk, int n_threads) {
    if (validate(p) != 0 || !gr || !gr->dO || !gr->dq || !gr->dk || !gr->dv || !gr->dg || !gr->dbeta) return -1;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t th[256];
    bwd_arg args[256];
    int failed = 0;
    for (int i = 0; i < n_threads; ++i) {
        args[i] = (bwd_arg){p, gr, chunk, i, n_threads, 0};
        if (pthread_create(&th[i], NULL, bwd_worker, &args[i]) != 0) {
            bwd_worker(&args[i]);
            th[i] = 0;
        }
    }
    for (int i = 0; i < n_threads; ++i) {
        if (th[i]) pthread_join(th[i], NULL);
        failed |= args[i].failed;
    }
    return failed ? -2 : 0;
}

int gdn_oracle_backward(const gdn_oracle_problem *p, const gdn_oracle_grads *gr, int n_threads) {
    return run_backward(p, gr, 0, n_threads);
}

/* gdn_oracle_backward_chunkwise: the gradients through the chunked form
 * (the chunk forms of section 2 above), derived here by differentiating
 * those matrix expressions; an independent formulation of the same
 * gradients.  For a chunk with start state S0 and end-state gradient dS:
 *   S_C = gamma_L S0 + U^T diag(lambda) K      -> dS0 = gamma_L dS, dU_j = lambda_j dS k_j,
 *                                                 dk_j += lambda_j dS^T u_j, dlambda_j = u_j^T dS k_j
 *   O = diag(gamma) Q S0^T + P U, P = QK^T (.) Gamma (lower, with diagonal)
 *                                              -> dS0 += dO^T diag(gamma) Q, dq += diag(gamma) dO S0,
 *                                                 dU += P^T dO, dP = dO U^T
 *   U = U~ - W S0^T                             -> dW = -dU S0, dS0 -= dU^T W
 *   W = T diag(beta gamma) K, U~ = T diag(beta) V
 *                                              -> dT = dW (diag(bg) K)^T + dU (diag(beta) V)^T, ...
 *   T = (I + A)^-1                              -> dA = -T^T dT T^T (strictly lower part)
 *   A = diag(beta) (K K^T (.) Gamma) (strictly lower)
 * and the decays through G (Gamma_rj = e^(G_r - G_j), gamma_r = e^(G_r),
 * lambda_j = e^(G_last - G_j)), then dg_t = sum_{r >= t} dG_r.  The result
 * must equal the token recurrence's. */
static int backward_chunk_unit(const gdn_oracle_problem *p, const gdn_oracle_grads *gr, int64_t unit, int C) {
    const int64_t n = unit / p->hv;
    const int h = (int)(unit % p->hv);
    const int hq = h / (p->hv / p->hk);
    const int dk = p->dk, dv = p->dv;
    const int64_t t0 = p->cu_seqlens[n], T = p->cu_seqlens[n + 1] - t0;
    const int64_t nch = (T + C - 1) / C;
    const size_t ssz = (size_t)dv * dk;
    double *S0s = malloc(sizeof(double) * ssz * (size_t)(nch + 1));
    double *dS = malloc(sizeof(double) * ssz), *dS0 = malloc(sizeof(double) * ssz);
    double *G = malloc(sizeof(double) * C), *gam = malloc(sizeof(double) * C), *lam = malloc(sizeof(double) * C);
    double *A = malloc(sizeof(double) * C * C), *Tm = malloc(sizeof(double) * C * C);
    double *Gm = malloc(sizeof(double) * C * C), *KK = malloc(sizeof(double) * C * C), *QK = malloc(sizeof(double) * C * C);
    double *W = malloc(sizeof(double) * C * dk), *U = malloc(sizeof(double) * C * dv);
    double *dU = malloc(sizeof(double) * C * dv), *dW = malloc(sizeof(double) * C * dk);
    double *dT = malloc(sizeof(double) * C * C), *dA = malloc(sizeof(double) * C * C), *tmp = malloc(sizeof(double) * C * C);
    double *dGam = malloc(sizeof(double) * C * C);
    double *dQ = malloc(sizeof(double) * C * dk), *dK = malloc(sizeof(double) * C * dk);
    double *dG = malloc(sizeof(double) * C), *dgam = malloc(sizeof(double) * C), *dlam = malloc(sizeof(double) * C);
    double *dbg = malloc(sizeof(double) * C), *dbeta = malloc(sizeof(double) * C);
    int rc = 0;
    if (!S0s || !dS || !dS0 || !G || !gam || !lam || !A || !Tm || !Gm || !KK || !QK || !W || !U || !dU || !dW ||
        !dT || !dA || !tmp || !dGam || !dQ || !dK || !dG || !dgam || !dlam || !dbg || !dbeta) {
        rc = -1;
        goto done;
    }
#define BK(r, c) p->k[((t0 + c0 + (r)) * p->hk + hq) * dk + (c)]
#define BQ(r, c) p->q[((t0 + c0 + (r)) * p->hk + hq) * dk + (c)]
#define BV(r, i) p->v[((t0 + c0 + (r)) * p->hv + h) * dv + (i)]
#define BB(r) p->beta[(t0 + c0 + (r)) * p->hv + h]
#define BG(r) p->g[(t0 + c0 + (r)) * p->hv + h]
    /* forward over chunks: the start state of every chunk */
    if (p->s0) memcpy(S0s, p->s0 + unit * (int64_t)ssz, sizeof(double) * ssz);
    else memset(S0s, 0, sizeof(double) * ssz);
    for (int64_t c = 0; c < nch; ++c) {
        const int64_t c0 = c * C;
        const double *S = S0s + ssz * c;
        double *Sn = S0s + ssz * (c + 1);
        const int L = (int)((T - c0) < C ? (T - c0) : C);
        memcpy(Sn, S, sizeof(double) * ssz);
        for (int t = 0; t < L; ++t) { /* the token recurrence within the chunk */
            const double alpha = exp(BG(t)), beta = BB(t);
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += alpha * Sn[i * dk + j] * BK(t, j);
                const double ui = beta * (BV(t, i) - acc);
                for (int j = 0; j < dk; ++j) Sn[i * dk + j] = alpha * Sn[i * dk + j] + ui * BK(t, j);
            }
        }
    }
    if (gr->dSf) memcpy(dS, gr->dSf + unit * (int64_t)ssz, sizeof(double) * ssz);
    else memset(dS, 0, sizeof(double) * ssz);
    for (int64_t c = nch - 1; c >= 0; --c) {
        const int64_t c0 = c * C;
        const double *S0 = S0s + ssz * c;
        const int L = (int)((T - c0) < C ? (T - c0) : C);
        /* the chunk's forward quantities */
        for (int r = 0; r < L; ++r) G[r] = (r ? G[r - 1] : 0.0) + BG(r);
        for (int r = 0; r < L; ++r) {
            gam[r] = exp(G[r]);
            lam[r] = exp(G[L - 1] - G[r]);
        }
        const double gL = exp(G[L - 1]);
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double kk = 0.0, qk = 0.0;
                for (int x = 0; x < dk; ++x) {
                    kk += BK(r, x) * BK(j, x);
                    qk += BQ(r, x) * BK(j, x);
                }
                KK[r * L + j] = kk;
                QK[r * L + j] = qk;
                Gm[r * L + j] = j <= r ? exp(G[r] - G[j]) : 0.0;
                A[r * L + j] = j < r ? BB(r) * Gm[r * L + j] * kk : 0.0;
            }
        for (int col = 0; col < L; ++col)
            for (int r = 0; r < L; ++r) {
                double x = (r == col) ? 1.0 : 0.0;
                for (int j = col; j < r; ++j) x -= A[r * L + j] * Tm[j * L + col];
                Tm[r * L + col] = r < col ? 0.0 : x;
            }
        for (int r = 0; r < L; ++r) {
            for (int x = 0; x < dk; ++x) {
                double acc = 0.0;
                for (int j = 0; j <= r; ++j) acc += Tm[r * L + j] * BB(j) * gam[j] * BK(j, x);
                W[r * dk + x] = acc;
            }
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j <= r; ++j) acc += Tm[r * L + j] * BB(j) * BV(j, i);
                for (int x = 0; x < dk; ++x) acc -= W[r * dk + x] * S0[i * dk + x];
                U[r * dv + i] = acc;
            }
        }
        for (int r = 0; r < L; ++r) {
            dgam[r] = dlam[r] = dbg[r] = dbeta[r] = 0.0;
            for (int x = 0; x < dk; ++x) dQ[r * dk + x] = dK[r * dk + x] = 0.0;
        }
        for (int e = 0; e < L * L; ++e) dGam[e] = dT[e] = 0.0;
        /* S_C = gL S0 + U^T diag(lambda) K */
        double dgL = 0.0;
        for (size_t e = 0; e < ssz; ++e) {
            dS0[e] = gL * dS[e];
            dgL += dS[e] * S0[e];
        }
        for (int j = 0; j < L; ++j) {
            double dl = 0.0;
            for (int i = 0; i < dv; ++i) {
                double dsk = 0.0;
                for (int x = 0; x < dk; ++x) dsk += dS[i * dk + x] * BK(j, x);
                dU[j * dv + i] = lam[j] * dsk;
                dl += U[j * dv + i] * dsk;
            }
            dlam[j] = dl;
            for (int x = 0; x < dk; ++x) {
                double acc = 0.0;
                for (int i = 0; i < dv; ++i) acc += dS[i * dk + x] * U[j * dv + i];
                dK[j * dk + x] += lam[j] * acc;
            }
        }
        /* O = diag(gamma) Q S0^T + P U */
        for (int r = 0; r < L; ++r) {
            const double *dOr = gr->dO + ((t0 + c0 + r) * p->hv + h) * dv;
            for (int x = 0; x < dk; ++x) {
                double acc = 0.0;
                for (int i = 0; i < dv; ++i) {
                    acc += dOr[i] * S0[i * dk + x];
                    dS0[i * dk + x] += dOr[i] * gam[r] * BQ(r, x);
                }
                dQ[r * dk + x] += gam[r] * acc;
                dgam[r] += acc * BQ(r, x);
            }
            for (int j = 0; j <= r; ++j) {
                const double Prj = Gm[r * L + j] * QK[r * L + j];
                double dP = 0.0;
                for (int i = 0; i < dv; ++i) {
                    dU[j * dv + i] += Prj * dOr[i];
                    dP += dOr[i] * U[j * dv + i];
                }
                /* P_rj = Gamma_rj (q_r . k_j) */
                for (int x = 0; x < dk; ++x) {
                    dQ[r * dk + x] += dP * Gm[r * L + j] * BK(j, x);
                    dK[j * dk + x] += dP * Gm[r * L + j] * BQ(r, x);
                }
                dGam[r * L + j] += dP * QK[r * L + j];
            }
        }
        /* U = U~ - W S0^T;  W = T diag(beta gamma) K;  U~ = T diag(beta) V */
        for (int r = 0; r < L; ++r)
            for (int x = 0; x < dk; ++x) {
                double acc = 0.0;
                for (int i = 0; i < dv; ++i) {
                    acc -= dU[r * dv + i] * S0[i * dk + x];
                    dS0[i * dk + x] -= dU[r * dv + i] * W[r * dk + x];
                }
                dW[r * dk + x] = acc;
            }
        for (int r = 0; r < L; ++r)
            for (int j = 0; j <= r; ++j) {
                double acc = 0.0;
                for (int x = 0; x < dk; ++x) acc += dW[r * dk + x] * BB(j) * gam[j] * BK(j, x);
                for (int i = 0; i < dv; ++i) acc += dU[r * dv + i] * BB(j) * BV(j, i);
                dT[r * L + j] = acc;
            }
        for (int j = 0; j < L; ++j) {
            /* dX_j = (T^T dW)_j, dY_j = (T^T dU~)_j */
            for (int x = 0; x < dk; ++x) {
                double dx = 0.0;
                for (int r = j; r < L; ++r) dx += Tm[r * L + j] * dW[r * dk + x];
                dK[j * dk + x] += BB(j) * gam[j] * dx;
                dbg[j] += dx * BK(j, x);
            }
            double *dvj = gr->dv + ((t0 + c0 + j) * p->hv + h) * dv;
            for (int i = 0; i < dv; ++i) {
                double dy = 0.0;
                for (int r = j; r < L; ++r) dy += Tm[r * L + j] * dU[r * dv + i];
                dvj[i] = BB(j) * dy;
                dbeta[j] += dy * BV(j, i);
            }
        }
        /* T = (I + A)^-1: dA = -T^T dT T^T, strictly lower */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double acc = 0.0;
                for (int m = 0; m < L; ++m) acc += dT[r * L + m] * Tm[j * L + m]; /* (dT T^T)_rj */
                tmp[r * L + j] = acc;
            }
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double acc = 0.0;
                if (j < r)
                    for (int m = 0; m < L; ++m) acc += Tm[m * L + r] * tmp[m * L + j]; /* (T^T (dT T^T))_rj */
                dA[r * L + j] = -acc;
            }
        /* A_rj = beta_r Gamma_rj (k_r . k_j), j < r */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < r; ++j) {
                const double da = dA[r * L + j];
                dbeta[r] += da * Gm[r * L + j] * KK[r * L + j];
                dGam[r * L + j] += da * BB(r) * KK[r * L + j];
                const double dkk = da * BB(r) * Gm[r * L + j];
                for (int x = 0; x < dk; ++x) {
                    dK[r * dk + x] += dkk * BK(j, x);
                    dK[j * dk + x] += dkk * BK(r, x);
                }
            }
        /* the decays through G */
        for (int r = 0; r < L; ++r) {
            dbeta[r] += dbg[r] * gam[r];
            dgam[r] += dbg[r] * BB(r);
        }
        for (int r = 0; r < L; ++r) dG[r] = dgam[r] * gam[r] - dlam[r] * lam[r];
        dG[L - 1] += dgL * gL;
        for (int j = 0; j < L; ++j) dG[L - 1] += dlam[j] * lam[j];
        for (int r = 0; r < L; ++r)
            for (int j = 0; j <= r; ++j) {
                const double e = dGam[r * L + j] * Gm[r * L + j];
                dG[r] += e;
                dG[j] -= e;
            }
        double run = 0.0;
        for (int t = L - 1; t >= 0; --t) {
            run += dG[t];
            const int64_t tt = t0 + c0 + t;
            gr->dg[tt * p->hv + h] = run;
            gr->dbeta[tt * p->hv + h] = dbeta[t];
            memcpy(gr->dq + (tt * p->hv + h) * dk, dQ + t * dk, sizeof(double) * dk);
            memcpy(gr->dk + (tt * p->hv + h) * dk, dK + t * dk, sizeof(double) * dk);
        }
        memcpy(dS, dS0, sizeof(double) * ssz);
    }
#undef BK
#undef BQ
#undef BV
#undef BB
#undef BG
    if (gr->dS0) memcpy(gr->dS0 + unit * (int64_t)ssz, dS, sizeof(double) * ssz);
done:
    free(S0s); free(dS); free(dS0); free(G); free(gam); free(lam); free(A); free(Tm); free(Gm); free(KK); free(QK);
    free(W); free(U); free(dU); free(dW); free(dT); free(dA); free(tmp); free(dGam); free(dQ); free(dK); free(dG);
    free(dgam); free(dlam); free(dbg); free(dbeta);
    return rc;
}

int gdn_oracle_backward_chunkwise(const gdn_oracle_problem *p, const gdn_oracle_grads *gr, int32_t chunk,
                                  int n_threads) {
    if (chunk <= 0) return -1;
    return run_backward(p, gr, chunk, n_threads);
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

/* The short causal convolution of the mixer's input side, with an optional
 * SiLU after it.  "Architecture Thread I", "Modern Architecture
 * Improvements", items 2 and the module structure that follows it: after
 * the linear projections, q and k pass through a short convolution, SiLU and
 * L2 normalisation, and v through a short convolution and SiLU.  The page
 * gives neither the width nor the tap order; this oracle takes the plain
 * causal depthwise reading: one filter of W taps per channel, and
 *     y[t, c] = act( sum_{j=0}^{W-1} w[c, j] x[t - (W-1) + j, c] ),
 * so w[c, W-1] multiplies the current token.  Inputs before a sequence's
 * first token come from that sequence's conv state (its W-1 preceding
 * inputs, oldest first), or are zero when no state is given; a sequence
 * never reads another's tokens.  act is SiLU, a / (1 + e^-a), when silu is
 * set, the identity otherwise.
 *   x, y        [tokens, channels], token-major; y must not alias x
 *   w           [channels, W]
 *   cu_seqlens  [num_seqs + 1]
 *   state_in    [num_seqs, channels, W-1] or NULL (zeros)
 *   state_out   [num_seqs, channels, W-1] or NULL: the last W-1 inputs seen
 *               by the sequence (reaching into state_in when it is shorter);
 *               it may alias state_in (entry i is written after every read
 *               of entries <= i)
 * Returns 0, or -1 for W < 1 or a bad cu_seqlens. */
int gdn_oracle_short_conv(int64_t tokens, int32_t channels, int32_t width, const double *x, const double *w,
                          const int64_t *cu_seqlens, int64_t num_seqs, const double *state_in, double *y,
                          double *state_out, int32_t silu) {
    if (width < 1 || channels < 1 || num_seqs < 0) return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != tokens) return -1;
    for (int64_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    const int32_t hist = width - 1;
    for (int64_t n = 0; n < num_seqs; ++n) {
        const int64_t s = cu_seqlens[n], e = cu_seqlens[n + 1];
        for (int32_t c = 0; c < channels; ++c) {
            const double *st = state_in ? state_in + (n * channels + c) * (int64_t)hist : NULL;
            /* the input at token u of this sequence's timeline (u < s reaches into the state) */
#define CONV_IN(u) ((u) >= s ? x[(u) * channels + c] : (st ? st[hist - (s - (u))] : 0.0))
            for (int64_t t = s; t < e; ++t) {
                double acc = 0.0;
                for (int32_t j = 0; j < width; ++j) acc += w[(int64_t)c * width + j] * CONV_IN(t - hist + j);
                y[t * channels + c] = silu ? acc / (1.0 + exp(-acc)) : acc;
            }
            if (state_out)
                for (int32_t i = 0; i < hist; ++i) state_out[(n * channels + c) * (int64_t)hist + i] = CONV_IN(e - hist + i);
#undef CONV_IN
        }
    }
    return 0;
}
