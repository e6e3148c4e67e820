/*
 * fp64 reverse mode (vector-Jacobian product) of the GDN / GDN-2 token recurrence.
 *
 * TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and bench.py's CPU legs may load this code.  It
 * shares nothing with the CUDA path.
 *
 * What it differentiates: the same per-token recurrence as gdn_oracle.c (GatedDeltaNet data-flow walkthrough,
 * yfxerp.com/news/367755, section "Delta Rule: predict first, then correct"; Gated DeltaNet-2 article,
 * 7minutos.es, section "Regla-2 del Delta cerrado"), written per token t with a per-key-channel decay alpha, an
 * erase key e and a write value z:
 *     Sbar = Diag(alpha) S_{t-1};   u = z - Sbar^T e;   S_t = Sbar + k u^T;   o_t = scale S_t^T q
 *   GDN   (mode 0): alpha_i = exp(g_t), e = beta_t k_t, z = beta_t v_t
 *   GDN-2 (mode 1): alpha_i = exp(g_ti), e = b_t . k_t, z = w_t . v_t
 * The walkthrough's section "Chunked parallelism" names the full backward (gradients of q, k, v, beta, g); the
 * Gated DeltaNet-2 article's section "Entrenamiento fragmentado y reconocimiento de puertas hacia atras" says
 * the gate factors enter the gradient dot products.  Given the cotangents dO of o and dhT of the final state,
 * walking t from last to first with dS = dhT:
 *     dS += scale q do^T;  dq = scale S_t do;  du = dS^T k;  dk = dS u;  dz = du;  de = -Sbar du;
 *     dSbar = dS - e du^T;  dalpha_i = sum_j S_{t-1,ij} dSbar_ij;  dS = Diag(alpha) dSbar
 * and then through alpha = exp(g), e and z to the inputs.  dh0 is the last dS.
 * The states S_{t-1} are recomputed forward from checkpoints taken every 64 tokens (plain recomputation of the
 * same recurrence, no algebraic shortcut).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define VJP_BLOCK 64

typedef struct {
    int mode, T, H, dk, dv, row, h;
    const double *q, *k, *v, *g, *b, *w;
    double scale;
} vjp_ctx;

/* per-token gate vectors of token `tok` (global row index row * T + t) */
static void token_gates(const vjp_ctx* c, long tok, double* alpha, double* e, double* z) {
    const long kb = (tok * c->H + c->h) * c->dk, vb = (tok * c->H + c->h) * c->dv;
    const long sb = tok * c->H + c->h;
    for (int i = 0; i < c->dk; ++i) {
        alpha[i] = exp(c->mode == 0 ? c->g[sb] : c->g[kb + i]);
        e[i] = (c->mode == 0 ? c->b[sb] : c->b[kb + i]) * c->k[kb + i];
    }
    for (int j = 0; j < c->dv; ++j) z[j] = (c->mode == 0 ? c->b[sb] : c->w[vb + j]) * c->v[vb + j];
}

/* S <- S_t from S = S_{t-1}; leaves Sbar and u for the caller when asked */
static void step(const vjp_ctx* c, long tok, double* S, const double* alpha, const double* e, const double* z,
                 double* Sbar, double* u) {
    const int dk = c->dk, dv = c->dv;
    const double* kt = c->k + (tok * c->H + c->h) * dk;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(long)i * dv + j] *= alpha[i];
    if (Sbar) memcpy(Sbar, S, sizeof(double) * dk * dv);
    for (int j = 0; j < dv; ++j) {
        double r = 0.0;
        for (int i = 0; i < dk; ++i) r += e[i] * S[(long)i * dv + j];
        u[j] = z[j] - r;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(long)i * dv + j] += kt[i] * u[j];
}

/* Reverse mode of one unit (sequence n = tokens [t0, t1) of batch row `row`, head h).
 * Inputs: as oracle_gdn_unit / oracle_gdn2_unit (mode 0: b = beta [B,T,H], w unused; mode 1: b [B,T,H,dk],
 * w [B,T,H,dv]); d_o [B,T,H,dv]; dhT [n_seq,H,dk,dv] or NULL (0).  Outputs (rows of this unit overwritten):
 * dq, dk_ [B,T,H,dk], dv_ [B,T,H,dv]; mode 0: dg, db [B,T,H]; mode 1: dg, db [B,T,H,dk], dw [B,T,H,dv];
 * dh0 [n_seq,H,dk,dv] or NULL.  Returns 0, or -1 if scratch memory could not be allocated. */
int oracle_vjp_unit(int mode, const double* q, const double* k, const double* v, const double* g, const double* b,
                    const double* w, double scale, const double* h0, const double* d_o, const double* dhT, double* dq,
                    double* dk_, double* dv_, double* dg, double* db, double* dw, double* dh0, int T, int H, int dk,
                    int dv, int row, int t0, int t1, int n, int h) {
    const vjp_ctx c = {mode, T, H, dk, dv, row, h, q, k, v, g, b, w, scale};
    const long sz = (long)dk * dv;
    const int L = t1 - t0, nblk = (L + VJP_BLOCK - 1) / VJP_BLOCK;
    double* ck = malloc(sizeof(double) * sz * (nblk + 1));
    double* blk = malloc(sizeof(double) * sz * VJP_BLOCK);
    double* S = malloc(sizeof(double) * sz);
    double* Sbar = malloc(sizeof(double) * sz);
    double* dS = malloc(sizeof(double) * sz);
    double* vec = malloc(sizeof(double) * (4 * (size_t)dk + 4 * (size_t)dv));
    if (!ck || !blk || !S || !Sbar || !dS || !vec) {
        free(ck), free(blk), free(S), free(Sbar), free(dS), free(vec);
        return -1;
    }
    double *alpha = vec, *e = alpha + dk, *de = e + dk, *dalpha = de + dk;
    double *z = dalpha + dk, *u = z + dv, *du = u + dv, *tmp = du + dv;

    if (h0) memcpy(S, h0 + ((long)n * H + h) * sz, sizeof(double) * sz);
    else memset(S, 0, sizeof(double) * sz);
    for (int t = t0; t < t1; ++t) {
        if ((t - t0) % VJP_BLOCK == 0) memcpy(ck + (long)((t - t0) / VJP_BLOCK) * sz, S, sizeof(double) * sz);
        const long tok = (long)row * T + t;
        token_gates(&c, tok, alpha, e, z);
        step(&c, tok, S, alpha, e, z, NULL, u);
    }
    if (dhT) memcpy(dS, dhT + ((long)n * H + h) * sz, sizeof(double) * sz);
    else memset(dS, 0, sizeof(double) * sz);

    for (int nb = nblk - 1; nb >= 0; --nb) {
        const int b0 = t0 + nb * VJP_BLOCK, b1 = (b0 + VJP_BLOCK < t1) ? b0 + VJP_BLOCK : t1;
        /* states before each token of the block */
        memcpy(S, ck + (long)nb * sz, sizeof(double) * sz);
        for (int t = b0; t < b1; ++t) {
            memcpy(blk + (long)(t - b0) * sz, S, sizeof(double) * sz);
            const long tok = (long)row * T + t;
            token_gates(&c, tok, alpha, e, z);
            step(&c, tok, S, alpha, e, z, NULL, u);
        }
        for (int t = b1 - 1; t >= b0; --t) {
            const long tok = (long)row * T + t;
            const double* Sprev = blk + (long)(t - b0) * sz;
            const long kb = (tok * H + h) * dk, vb = (tok * H + h) * dv, sb = tok * H + h;
            const double *qt = q + kb, *kt = k + kb, *vt = v + vb, *dot = d_o + vb;
            token_gates(&c, tok, alpha, e, z);
            memcpy(S, Sprev, sizeof(double) * sz);
            step(&c, tok, S, alpha, e, z, Sbar, u); /* S = S_t, Sbar, u of token t */
            /* o_t = scale S_t^T q */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) dS[(long)i * dv + j] += scale * qt[i] * dot[j];
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += S[(long)i * dv + j] * dot[j];
                dq[kb + i] = scale * acc;
            }
            /* S_t = Sbar + k u^T */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += kt[i] * dS[(long)i * dv + j];
                du[j] = acc;
            }
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += dS[(long)i * dv + j] * u[j];
                dk_[kb + i] = acc;
            }
            /* u = z - Sbar^T e */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += Sbar[(long)i * dv + j] * du[j];
                de[i] = -acc;
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) dS[(long)i * dv + j] -= e[i] * du[j]; /* dS is now dSbar */
            /* Sbar = Diag(alpha) S_{t-1} */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += Sprev[(long)i * dv + j] * dS[(long)i * dv + j];
                dalpha[i] = acc;
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) dS[(long)i * dv + j] *= alpha[i];
            /* through the gates to the inputs (z = du since u = z - ...) */
            if (mode == 0) {
                const double bt = b[sb];
                double dbt = 0.0, dgt = 0.0;
                for (int j = 0; j < dv; ++j) {
                    dv_[vb + j] = bt * du[j];
                    dbt += vt[j] * du[j];
                }
                for (int i = 0; i < dk; ++i) {
                    dk_[kb + i] += bt * de[i];
                    dbt += kt[i] * de[i];
                    dgt += alpha[i] * dalpha[i];
                }
                db[sb] = dbt;
                dg[sb] = dgt;
            } else {
                const double *bt = b + kb, *wt = w + vb;
                for (int j = 0; j < dv; ++j) {
                    dv_[vb + j] = wt[j] * du[j];
                    dw[vb + j] = vt[j] * du[j];
                }
                for (int i = 0; i < dk; ++i) {
                    dk_[kb + i] += bt[i] * de[i];
                    db[kb + i] = kt[i] * de[i];
                    dg[kb + i] = alpha[i] * dalpha[i];
                }
            }
        }
    }
    if (dh0) memcpy(dh0 + ((long)n * H + h) * sz, dS, sizeof(double) * sz);
    (void)tmp;
    free(ck), free(blk), free(S), free(Sbar), free(dS), free(vec);
    return 0;
}
