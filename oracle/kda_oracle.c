/*
 * kda_oracle.c -- fp64 CPU reference for the Kimi Delta Attention (KDA)
 * token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and
 * bench.py's CPU-baseline / reference arm load this library.  The product
 * library (gated_delta_rule_88_b200) never links, loads or calls it, and this
 * file shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (the plain definition, token by token, in fp64):
 *
 *   Kimi Linear paper notes (paper-notes-site), section 2 "core idea", the
 *   KDA recurrence equation:
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *       o_t = S_t^T q_t
 *   with a per-head state S in R^{dk x dv}, a per-channel decay alpha_t in
 *   R^{dk} and a scalar write strength beta_t.  The same formula is restated
 *   on the zhichai.net account (KDA formula paragraph) and in the hnts03
 *   summary ("Kimi Delta Attention" section: per-channel diagonal decay
 *   instead of Gated DeltaNet's scalar).
 *
 * Readings taken where the pages are silent or garbled:
 *   - The printed equation shows a bullet between the two terms; it is read
 *     as "+" (the zhichai.net formula has "+").
 *   - g = log(alpha) is the input; alpha = exp(g) is taken in fp64 here.
 *   - The readout uses the state after the token's update (o_t = S_t^T q_t).
 *   - S is stored [dk][dv] row-major: row c is key channel c.
 *
 * The update is evaluated in the algebraically identical rank-1 form
 *       S' = Diag(alpha) S
 *       u  = beta (v - S'^T k)
 *       S  = S' + k u^T
 * because (I - b k k^T) S' + b k v^T = S' + k (b (v - S'^T k))^T.  The
 * tests pin it against the dense-matrix form, DeltaNet, Gated DeltaNet,
 * closed forms and a brute-force product of transition matrices.
 *
 * Build: gcc -O2 -shared -fPIC -o libkda_oracle.so kda_oracle.c -lm
 * (no -ffast-math: the summation order is the plain loop order).
 */
#include <math.h>
#include <stdlib.h>

/*
 * One (sequence, head) recurrence over T tokens.
 *
 * Token t's vectors live at q + t*q_stride (dk doubles), k + t*k_stride (dk),
 * v + t*v_stride (dv), g + t*g_stride (dk), beta[t*beta_stride] (scalar).
 * S: [dk][dv], in = initial state, out = final state.
 * o: token t's output written to o + t*o_stride (dv doubles); o may be NULL.
 * Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int kda_oracle_recurrence(long T, int dk, int dv,
                          const double *q, long q_stride,
                          const double *k, long k_stride,
                          const double *v, long v_stride,
                          const double *g, long g_stride,
                          const double *beta, long beta_stride,
                          double *S, double *o, long o_stride)
{
    if (T < 0 || dk <= 0 || dv <= 0 || !S) return -1;
    if (T > 0 && (!q || !k || !v || !g || !beta)) return -1;
    double *kS = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!kS) return -1;

    for (long t = 0; t < T; ++t) {
        const double *qt = q + t * q_stride;
        const double *kt = k + t * k_stride;
        const double *vt = v + t * v_stride;
        const double *gt = g + t * g_stride;
        const double bt = beta[t * beta_stride];

        /* S' = Diag(alpha_t) S : row c scaled by alpha_c = exp(g_c). */
        for (int c = 0; c < dk; ++c) {
            const double a = exp(gt[c]);
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
        /* kS = S'^T k */
        for (int j = 0; j < dv; ++j) kS[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double kc = kt[c];
            const double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) kS[j] += kc * row[j];
        }
        /* u = beta (v - S'^T k), stored in kS */
        for (int j = 0; j < dv; ++j) kS[j] = bt * (vt[j] - kS[j]);
        /* S = S' + k u^T */
        for (int c = 0; c < dk; ++c) {
            const double kc = kt[c];
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] += kc * kS[j];
        }
        /* o_t = S_t^T q_t (post-update state) */
        if (o) {
            double *ot = o + t * o_stride;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int c = 0; c < dk; ++c) {
                const double qc = qt[c];
                const double *row = S + (size_t)c * dv;
                for (int j = 0; j < dv; ++j) ot[j] += qc * row[j];
            }
        }
    }
    free(kS);
    return 0;
}
