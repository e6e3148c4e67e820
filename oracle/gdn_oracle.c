/*
 * fp64 oracle for the gated delta rule (GDN) and Gated Delta Rule-2 (GDN-2) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg
 * may load this library.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes: the plain per-token recurrence, one (sequence, head) unit at a time, in
 * double precision, with no chunking, blocking or reordering.  The chunked method is an exact
 * algebraic rearrangement of this recurrence, so the recurrence is the definition.
 *
 * GDN (GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755, section "Delta Rule: predict
 * first, then correct" -- the token-by-token reference loop; gate recipe in section "Gating"):
 *     S <- exp(g_t) * S                       decay first (the loop's order)
 *     r_j = sum_i (beta_t k_ti) S_ij          prediction of the value stored under k_t
 *     u_j = beta_t v_tj - r_j                 scaled correction
 *     S_ij <- S_ij + k_ti u_j                 rank-one write
 *     o_tj = scale * sum_i q_ti S_ij          read-out after the write (inclusive of token t)
 *   S is dk x dv: the loop sums the prediction over the key axis (dim -2), so keys index rows.
 *   The read-out is not printed on the pages; o_t = scale * S_t^T q_t with scale = dk^-1/2 is the
 *   adopted reading.  u is written beta*v - S^T(beta*k) rather than beta*(v - S^T k): equal in exact
 *   arithmetic; this order makes the GDN-2 -> GDN reduction an identical operation sequence.
 *   form == 1 selects the literal beta*(v - S^T k) order instead (used only to cross-check).
 *
 * GDN-2 (NVIDIA Gated DeltaNet-2 article, 7minutos.es, section "Regla-2 del Delta cerrado: dos
 * puertas en lugar de una"):  S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,
 * alpha_t = exp(g_t) per key channel, decay applied before the edit:
 *     S_ij <- exp(g_ti) * S_ij
 *     r_j  = sum_i (b_ti k_ti) S_ij
 *     u_j  = w_tj v_tj - r_j
 *     S_ij <- S_ij + k_ti u_j ;   o_t = scale * S^T q_t
 *
 * Layouts (row-major): q,k [B,T,H,dk]; v,o [B,T,H,dv]; GDN g,beta [B,T,H]; GDN-2 g,b [B,T,H,dk],
 * w [B,T,H,dv]; h0,hT [n_seq,H,dk,dv].  A unit is (sequence n, head h); sequence n covers tokens
 * [t0,t1) of batch row `row`.  h0 == NULL means a zero initial state.
 */
#include <math.h>
#include <stddef.h>
#include <string.h>

static void unit_init(double* S, const double* h0, long n, int H, int h, int dk, int dv) {
    const long sz = (long)dk * dv;
    if (h0) memcpy(S, h0 + ((long)n * H + h) * sz, sizeof(double) * sz);
    else memset(S, 0, sizeof(double) * sz);
}

/* One GDN unit.  S (dk*dv) and u (dv) are caller-provided scratch. */
void oracle_gdn_unit(const double* q, const double* k, const double* v, const double* g,
                     const double* beta, double scale, const double* h0, double* o, double* hT,
                     int T, int H, int dk, int dv, int row, int t0, int t1, int n, int h, int form,
                     double* S, double* u) {
    unit_init(S, h0, n, H, h, dk, dv);
    for (int t = t0; t < t1; ++t) {
        const long tok = (long)row * T + t;
        const double* kt = k + (tok * H + h) * dk;
        const double* qt = q + (tok * H + h) * dk;
        const double* vt = v + (tok * H + h) * dv;
        const double bt = beta[tok * H + h];
        const double a = exp(g[tok * H + h]);
        for (long e = 0; e < (long)dk * dv; ++e) S[e] *= a;
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;
            if (form == 0) {
                for (int i = 0; i < dk; ++i) r += (bt * kt[i]) * S[(long)i * dv + j];
                u[j] = bt * vt[j] - r;
            } else {
                for (int i = 0; i < dk; ++i) r += kt[i] * S[(long)i * dv + j];
                u[j] = bt * (vt[j] - r);
            }
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(long)i * dv + j] += kt[i] * u[j];
        double* ot = o + (tok * H + h) * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qt[i] * S[(long)i * dv + j];
            ot[j] = scale * acc;
        }
    }
    if (hT) memcpy(hT + ((long)n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
}

/* One GDN-2 unit.  S (dk*dv) and u (dv) are caller-provided scratch. */
void oracle_gdn2_unit(const double* q, const double* k, const double* v, const double* g,
                      const double* b, const double* w, double scale, const double* h0, double* o,
                      double* hT, int T, int H, int dk, int dv, int row, int t0, int t1, int n, int h,
                      double* S, double* u) {
    unit_init(S, h0, n, H, h, dk, dv);
    for (int t = t0; t < t1; ++t) {
        const long tok = (long)row * T + t;
        const double* kt = k + (tok * H + h) * dk;
        const double* qt = q + (tok * H + h) * dk;
        const double* vt = v + (tok * H + h) * dv;
        const double* gt = g + (tok * H + h) * dk;
        const double* bt = b + (tok * H + h) * dk;
        const double* wt = w + (tok * H + h) * dv;
        for (int i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            for (int j = 0; j < dv; ++j) S[(long)i * dv + j] *= a;
        }
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;
            for (int i = 0; i < dk; ++i) r += (bt[i] * kt[i]) * S[(long)i * dv + j];
            u[j] = wt[j] * vt[j] - r;
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(long)i * dv + j] += kt[i] * u[j];
        double* ot = o + (tok * H + h) * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qt[i] * S[(long)i * dv + j];
            ot[j] = scale * acc;
        }
    }
    if (hT) memcpy(hT + ((long)n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
}
