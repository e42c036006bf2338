/*
 * CARVE fp64 reference oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, token-sequential, slow and obviously correct.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may load this library; the CUDA product path never
 * does, and this file shares no code, header, table or helper with it.
 *
 * What it computes (per batch b and head h, state S in R^{V x K}, S <- S0 or 0):
 *
 *   for each chunk c = tokens [cL, min(cL+L, T)) of length n:
 *     m_c   = S . mean_{t in c} q_t               (mc_mode 0: chunk-boundary state readout;
 *                                                   CARVE paperdance abstract)
 *           | (1/n_{c-1}) sum_{t in c-1} o_t      (mc_mode 1: previous chunk's mean output;
 *                                                   CARVE blog, section 2.2; m_0 = m_prev_in or 0)
 *     z_c   = B m_c ;  Delta = A z_c                (U_b = A.B, low rank; blog section 2.2)
 *     dw_c  = Aw . z_c  (optional content term of the write gate: the same zero-initialised
 *                       low-rank projection of m_c yields the erase bias and the write bias,
 *                       blog section 2.2, Figure 1; dw_c = 0 when Aw is absent)
 *     for t in c:
 *       g_t = exp(-e^{A_dec} softplus(g_logit_t + tau))  key-axis decay (blog section 2.3, the
 *                                                 fused decay: A_dec [H] the learned log-decay
 *                                                 amplitude, tau [H,K] the bias; A_dec = 0 and
 *                                                 tau = 0 when absent)
 *       b_t = sigmoid(bx_t + Delta)               key-axis content-aware erase (blog section 2.2)
 *       a_t = g_t * b_t ;  w_t = sigmoid(w_logit_t + dw_c)  scalar write per head (blog 2.3)
 *       P   = S Diag(a_t) ; e_t = v_t - P k_t ; S = P + w_t e_t k_t^T      (blog section 2.1)
 *       o_t = S q_t
 *
 * The pages' display equations are stripped; the recurrence above is the plainest reading
 * that the symbol explanations of the blog's section 2.1-2.3 and the paperdance abstract
 * support (o_t uses the updated state; the write gate is one scalar per head; the erase and
 * decay gates multiply the state on the key axis from the right).
 *
 * Backward: back-propagation through time over the same token loop, with the chunk-start
 * states stored in fp64 and the chunk's per-token states recomputed.
 *
 * Layouts (all contiguous, row-major):
 *   q, k, g_logit, bx : [B,T,H,K]    v, o : [B,T,H,V]    w_logit : [B,T,H]
 *   (varlen: B sequences packed as [1,T,H,*] and delimited by cu_seqlens, see unit_tokens)
 *   A : [H,K,R]   Bm : [H,R,V]   Aw : [H,R]   A_dec : [H]   tau : [H,K]
 *   S0, S_final, dS : [B,H,V,K]   m vectors : [B,H,V]
 * Units (b,h) are independent and run under OpenMP; the per-head parameter gradients are
 * summed over b in a fixed order afterwards, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, H, T, K, V, R, L;
    int mc_mode;      /* 0 boundary-state readout, 1 previous-chunk mean output */
    int content_off;  /* 1: no content path at all, b = sigmoid(bx) (the key-axis baseline) */
} orc_dims;

static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }
static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

#define IX_TK(d, b, t, h, i, W) ((((size_t)(b) * (d)->T + (t)) * (d)->H + (h)) * (W) + (i))

/* the decay's parameters of head h: amplitude e^{A_dec} and the bias of channel i */
static double decay_amp(const double *A_dec, int h) { return A_dec ? exp(A_dec[h]) : 1.0; }
static double decay_bias(const orc_dims *d, const double *tau, int h, int i) {
    return tau ? tau[(size_t)h * d->K + i] : 0.0;
}

/* gate activations of one token (b,t,h): a, g, bgate over K; returns w */
static double gates(const orc_dims *d, int b, int t, int h, const double *gl, const double *bx,
                    const double *wl, const double *A_dec, const double *tau, const double *delta,
                    double dwc, double *a, double *g, double *bg) {
    const double amp = decay_amp(A_dec, h);
    for (int i = 0; i < d->K; ++i) {
        size_t ix = IX_TK(d, b, t, h, i, d->K);
        g[i] = exp(-amp * softplus(gl[ix] + decay_bias(d, tau, h, i)));
        bg[i] = d->content_off ? sigm(bx[ix]) : sigm(bx[ix] + delta[i]);
        a[i] = g[i] * bg[i];
    }
    return sigm(wl[((size_t)b * d->T + t) * d->H + h] + dwc);
}

/* dw = Aw[h] . z (0 without the write-gate content term) */
static double write_bias(const orc_dims *d, int h, const double *Aw, const double *z) {
    if (!Aw || d->content_off) return 0.0;
    double s = 0.0;
    for (int j = 0; j < d->R; ++j) s += Aw[(size_t)h * d->R + j] * z[j];
    return s;
}

/* Delta = A (B m); z = B m is returned too */
static void content_delta(const orc_dims *d, int h, const double *A, const double *Bm,
                          const double *m, double *z, double *delta) {
    const int K = d->K, V = d->V, R = d->R;
    for (int j = 0; j < R; ++j) {
        double s = 0.0;
        for (int v = 0; v < V; ++v) s += Bm[((size_t)h * R + j) * V + v] * m[v];
        z[j] = s;
    }
    for (int i = 0; i < K; ++i) {
        double s = 0.0;
        for (int j = 0; j < R; ++j) s += A[((size_t)h * K + i) * R + j] * z[j];
        delta[i] = s;
    }
}

/* one token of the recurrence on S (in place); writes e (V) and o (V) */
static void token_update(const orc_dims *d, double *S, const double *a, double w,
                         const double *k, const double *v, const double *q, double *e, double *o) {
    const int K = d->K, V = d->V;
    for (int j = 0; j < V; ++j) {
        double *row = S + (size_t)j * K;
        double p = 0.0;
        for (int i = 0; i < K; ++i) p += row[i] * a[i] * k[i];
        e[j] = v[j] - p;
        for (int i = 0; i < K; ++i) row[i] = row[i] * a[i] + w * e[j] * k[i];
        double s = 0.0;
        for (int i = 0; i < K; ++i) s += row[i] * q[i];
        o[j] = s;
    }
}

static void gather_tok(const orc_dims *d, const double *x, int b, int t, int h, int W, double *out) {
    memcpy(out, x + IX_TK(d, b, t, h, 0, W), sizeof(double) * (size_t)W);
}

/* Tokens of sequence b.  Without cu_seqlens: batch element b of [B,T,H,*] tensors, all T
 * tokens.  With cu_seqlens ([B+1], non-decreasing, cu[0] = 0, cu[B] <= T): the B sequences are
 * packed along the token axis of [1,T,H,*] tensors and sequence b is rows [cu[b], cu[b+1]);
 * each has its own state, content signal and chunk grid (chunks restart at its first token). */
static void unit_tokens(const orc_dims *d, const int *cu, int b, int *bb, int *toff, int *Tn) {
    *bb = cu ? 0 : b;
    *toff = cu ? cu[b] : 0;
    *Tn = cu ? cu[b + 1] - cu[b] : d->T;
}

static int check_seqlens(const orc_dims *d, const int *cu) {
    if (!cu) return 0;
    if (cu[0] != 0 || cu[d->B] > d->T) return -1;
    for (int b = 0; b < d->B; ++b)
        if (cu[b + 1] < cu[b]) return -1;
    return 0;
}

static int check_dims(const orc_dims *d) {
    if (d->B < 1 || d->H < 1 || d->T < 0 || d->K < 1 || d->V < 1 || d->R < 1 || d->L < 1) return -1;
    if (d->mc_mode != 0 && d->mc_mode != 1) return -1;
    return 0;
}

/* Forward.  Aw, A_dec, tau, S0, m_prev_in, m_prev_out may be NULL; so may cu_seqlens (see
   unit_tokens).  Returns 0 or -1 on bad dims. */
int orc_fwd(const orc_dims *d, const double *q, const double *k, const double *v,
            const double *gl, const double *bx, const double *wl, const double *A,
            const double *Bm, const double *Aw, const double *A_dec, const double *tau,
            const double *S0, const double *m_prev_in, double *o,
            double *S_final, double *m_prev_out, const int *cu_seqlens) {
    if (check_dims(d) || check_seqlens(d, cu_seqlens)) return -1;
    const int K = d->K, V = d->V, R = d->R, L = d->L, H = d->H;
    const int units = d->B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < units; ++u) {
        const int b = u / H, h = u % H;
        int bb, toff, Tn;
        unit_tokens(d, cu_seqlens, b, &bb, &toff, &Tn);
        double *S = (double *)calloc((size_t)V * K, sizeof(double));
        double *m = calloc(V, sizeof(double)), *z = calloc(R, sizeof(double));
        double *delta = calloc(K, sizeof(double)), *qbar = calloc(K, sizeof(double));
        double *a = calloc(K, sizeof(double)), *g = calloc(K, sizeof(double)), *bg = calloc(K, sizeof(double));
        double *qt = calloc(K, sizeof(double)), *kt = calloc(K, sizeof(double)), *vt = calloc(V, sizeof(double));
        double *e = calloc(V, sizeof(double)), *ot = calloc(V, sizeof(double));
        double *mprev = calloc(V, sizeof(double)), *osum = calloc(V, sizeof(double));
        if (S0) memcpy(S, S0 + (size_t)u * V * K, sizeof(double) * (size_t)V * K);
        if (m_prev_in) memcpy(mprev, m_prev_in + (size_t)u * V, sizeof(double) * (size_t)V);
        for (int t0 = 0; t0 < Tn; t0 += L) {
            const int t1 = t0 + L < Tn ? t0 + L : Tn, n = t1 - t0;
            if (!d->content_off) {
                if (d->mc_mode == 0) {
                    for (int i = 0; i < K; ++i) qbar[i] = 0.0;
                    for (int t = t0; t < t1; ++t)
                        for (int i = 0; i < K; ++i) qbar[i] += q[IX_TK(d, bb, toff + t, h, i, K)];
                    for (int i = 0; i < K; ++i) qbar[i] /= n;
                    for (int j = 0; j < V; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < K; ++i) s += S[(size_t)j * K + i] * qbar[i];
                        m[j] = s;
                    }
                } else {
                    memcpy(m, mprev, sizeof(double) * (size_t)V);
                }
                content_delta(d, h, A, Bm, m, z, delta);
            }
            const double dwc = write_bias(d, h, Aw, z);
            for (int j = 0; j < V; ++j) osum[j] = 0.0;
            for (int t = t0; t < t1; ++t) {
                double w = gates(d, bb, toff + t, h, gl, bx, wl, A_dec, tau, delta, dwc, a, g, bg);
                gather_tok(d, q, bb, toff + t, h, K, qt);
                gather_tok(d, k, bb, toff + t, h, K, kt);
                gather_tok(d, v, bb, toff + t, h, V, vt);
                token_update(d, S, a, w, kt, vt, qt, e, ot);
                memcpy(o + IX_TK(d, bb, toff + t, h, 0, V), ot, sizeof(double) * (size_t)V);
                for (int j = 0; j < V; ++j) osum[j] += ot[j];
            }
            for (int j = 0; j < V; ++j) mprev[j] = osum[j] / n;
        }
        if (S_final) memcpy(S_final + (size_t)u * V * K, S, sizeof(double) * (size_t)V * K);
        if (m_prev_out) memcpy(m_prev_out + (size_t)u * V, mprev, sizeof(double) * (size_t)V);
        free(S); free(m); free(z); free(delta); free(qbar); free(a); free(g); free(bg);
        free(qt); free(kt); free(vt); free(e); free(ot); free(mprev); free(osum);
    }
    return 0;
}

/*
 * Backward by back-propagation through time.  Given dO (and optionally dS_final, and
 * dm_prev_out in mc_mode 1), returns the gradient of sum(dO*o) + sum(dS_final*S_final)
 * + sum(dm_prev_out*m_prev_out) with respect to every input.  dA, dB (and dAw, dA_dec,
 * dtau when given) are overwritten; Aw, A_dec, tau and their gradients may be NULL.
 * dS0 and dm_prev_in may be NULL.
 */
int orc_bwd(const orc_dims *d, const double *q, const double *k, const double *v,
            const double *gl, const double *bx, const double *wl, const double *A,
            const double *Bm, const double *Aw, const double *A_dec, const double *tau,
            const double *S0, const double *m_prev_in, const double *dO,
            const double *dS_final, const double *dm_prev_out, double *dq, double *dk,
            double *dv, double *dgl, double *dbx, double *dwl, double *dA, double *dB, double *dAw,
            double *dA_dec, double *dtau, double *dS0, double *dm_prev_in, const int *cu_seqlens) {
    if (check_dims(d) || check_seqlens(d, cu_seqlens)) return -1;
    const int K = d->K, V = d->V, R = d->R, T = d->T, L = d->L, H = d->H;
    const int units = d->B * H;
    const size_t VK = (size_t)V * K;
    double *dA_u = calloc((size_t)units * K * R, sizeof(double));
    double *dB_u = calloc((size_t)units * R * V, sizeof(double));
    double *dAw_u = calloc((size_t)units * R, sizeof(double));
    double *dAdec_u = calloc((size_t)units, sizeof(double));
    double *dtau_u = calloc((size_t)units * K, sizeof(double));
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < units; ++u) {
        const int b = u / H, h = u % H;
        int bb, toff, Tn;
        unit_tokens(d, cu_seqlens, b, &bb, &toff, &Tn);
        const int N = (Tn + L - 1) / L;
        double *Sb = calloc((size_t)(N > 0 ? N : 1) * VK, sizeof(double)); /* chunk-start states */
        double *mc = calloc((size_t)(N > 0 ? N : 1) * V, sizeof(double));
        double *zc = calloc((size_t)(N > 0 ? N : 1) * R, sizeof(double));
        double *dc = calloc((size_t)(N > 0 ? N : 1) * K, sizeof(double));
        double *qb = calloc((size_t)(N > 0 ? N : 1) * K, sizeof(double));
        double *St = calloc((size_t)(L + 1) * VK, sizeof(double));       /* states inside a chunk */
        double *S = calloc(VK, sizeof(double)), *dS = calloc(VK, sizeof(double));
        double *dP = calloc(VK, sizeof(double));
        double *at = calloc((size_t)L * K, sizeof(double)), *gt = calloc((size_t)L * K, sizeof(double));
        double *bt = calloc((size_t)L * K, sizeof(double)), *wt = calloc(L, sizeof(double));
        double *et = calloc((size_t)L * V, sizeof(double));
        double *qt = calloc(K, sizeof(double)), *kt = calloc(K, sizeof(double)), *vt = calloc(V, sizeof(double));
        double *ot = calloc(V, sizeof(double)), *osum = calloc(V, sizeof(double)), *mprev = calloc(V, sizeof(double));
        double *dox = calloc(V, sizeof(double)), *dot = calloc(V, sizeof(double));
        double *de = calloc(V, sizeof(double)), *dd = calloc(K, sizeof(double));
        double *dz = calloc(R, sizeof(double)), *dm = calloc(V, sizeof(double)), *tmp = calloc(K, sizeof(double));
        double *dAu = dA_u + (size_t)u * K * R, *dBu = dB_u + (size_t)u * R * V, *dAwu = dAw_u + (size_t)u * R;
        double *dtauu = dtau_u + (size_t)u * K;
        const double amp = decay_amp(A_dec, h);

        /* forward pass: chunk-start states and content signals */
        if (S0) memcpy(S, S0 + (size_t)u * VK, sizeof(double) * VK);
        if (m_prev_in) memcpy(mprev, m_prev_in + (size_t)u * V, sizeof(double) * (size_t)V);
        for (int c = 0; c < N; ++c) {
            const int t0 = c * L, t1 = t0 + L < Tn ? t0 + L : Tn, n = t1 - t0;
            memcpy(Sb + (size_t)c * VK, S, sizeof(double) * VK);
            double *m = mc + (size_t)c * V, *qbar = qb + (size_t)c * K;
            for (int i = 0; i < K; ++i) qbar[i] = 0.0;
            for (int t = t0; t < t1; ++t)
                for (int i = 0; i < K; ++i) qbar[i] += q[IX_TK(d, bb, toff + t, h, i, K)];
            for (int i = 0; i < K; ++i) qbar[i] /= n;
            if (!d->content_off) {
                if (d->mc_mode == 0) {
                    for (int j = 0; j < V; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < K; ++i) s += S[(size_t)j * K + i] * qbar[i];
                        m[j] = s;
                    }
                } else {
                    memcpy(m, mprev, sizeof(double) * (size_t)V);
                }
                content_delta(d, h, A, Bm, m, zc + (size_t)c * R, dc + (size_t)c * K);
            }
            for (int j = 0; j < V; ++j) osum[j] = 0.0;
            const double dwc = write_bias(d, h, Aw, zc + (size_t)c * R);
            for (int t = t0; t < t1; ++t) {
                double w = gates(d, bb, toff + t, h, gl, bx, wl, A_dec, tau, dc + (size_t)c * K, dwc, at, gt, bt);
                gather_tok(d, q, bb, toff + t, h, K, qt);
                gather_tok(d, k, bb, toff + t, h, K, kt);
                gather_tok(d, v, bb, toff + t, h, V, vt);
                token_update(d, S, at, w, kt, vt, qt, et, ot);
                for (int j = 0; j < V; ++j) osum[j] += ot[j];
            }
            for (int j = 0; j < V; ++j) mprev[j] = osum[j] / n;
        }

        /* reverse sweep */
        if (dS_final) memcpy(dS, dS_final + (size_t)u * VK, sizeof(double) * VK);
        for (int j = 0; j < V; ++j) dox[j] = 0.0;
        if (dm_prev_out && N > 0) {
            const int nl = Tn - (N - 1) * L;
            for (int j = 0; j < V; ++j) dox[j] = dm_prev_out[(size_t)u * V + j] / nl;
        }
        for (int c = N - 1; c >= 0; --c) {
            const int t0 = c * L, t1 = t0 + L < Tn ? t0 + L : Tn, n = t1 - t0;
            const double *delta = dc + (size_t)c * K;
            const double dwc = write_bias(d, h, Aw, zc + (size_t)c * R);
            double ddw = 0.0;   /* gradient of dw_c: sum of the chunk's write-logit gradients */
            /* recompute the chunk's per-token states St[0..n] and gates */
            memcpy(St, Sb + (size_t)c * VK, sizeof(double) * VK);
            for (int ti = 0; ti < n; ++ti) {
                const int t = t0 + ti;
                wt[ti] = gates(d, bb, toff + t, h, gl, bx, wl, A_dec, tau, delta, dwc, at + (size_t)ti * K,
                                gt + (size_t)ti * K, bt + (size_t)ti * K);
                memcpy(St + (size_t)(ti + 1) * VK, St + (size_t)ti * VK, sizeof(double) * VK);
                gather_tok(d, q, bb, toff + t, h, K, qt);
                gather_tok(d, k, bb, toff + t, h, K, kt);
                gather_tok(d, v, bb, toff + t, h, V, vt);
                token_update(d, St + (size_t)(ti + 1) * VK, at + (size_t)ti * K, wt[ti], kt, vt,
                             qt, et + (size_t)ti * V, ot);
            }
            for (int i = 0; i < K; ++i) dd[i] = 0.0;
            for (int ti = n - 1; ti >= 0; --ti) {
                const int t = t0 + ti;
                const double *a = at + (size_t)ti * K, *g = gt + (size_t)ti * K, *bg = bt + (size_t)ti * K;
                const double *e = et + (size_t)ti * V, w = wt[ti];
                const double *Sprev = St + (size_t)ti * VK, *Scur = St + (size_t)(ti + 1) * VK;
                gather_tok(d, q, bb, toff + t, h, K, qt);
                gather_tok(d, k, bb, toff + t, h, K, kt);
                for (int j = 0; j < V; ++j) dot[j] = dO[IX_TK(d, bb, toff + t, h, j, V)] + dox[j];
                /* o_t = S_t q_t */
                double *dqt = dq + IX_TK(d, bb, toff + t, h, 0, K);
                for (int i = 0; i < K; ++i) dqt[i] = 0.0;
                for (int j = 0; j < V; ++j)
                    for (int i = 0; i < K; ++i) {
                        dS[(size_t)j * K + i] += dot[j] * qt[i];
                        dqt[i] += Scur[(size_t)j * K + i] * dot[j];
                    }
                /* S_t = P + w e k^T */
                double dw = 0.0;
                double *dkt = dk + IX_TK(d, bb, toff + t, h, 0, K);
                for (int i = 0; i < K; ++i) dkt[i] = 0.0;
                for (int j = 0; j < V; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < K; ++i) s += dS[(size_t)j * K + i] * kt[i];
                    de[j] = w * s;
                    dw += e[j] * s;
                    for (int i = 0; i < K; ++i) dkt[i] += w * dS[(size_t)j * K + i] * e[j];
                }
                /* e = v - P k, P = S_{t-1} Diag(a) */
                for (int j = 0; j < V; ++j) dv[IX_TK(d, bb, toff + t, h, j, V)] = de[j];
                for (int j = 0; j < V; ++j)
                    for (int i = 0; i < K; ++i) {
                        double p = Sprev[(size_t)j * K + i] * a[i];
                        dP[(size_t)j * K + i] = dS[(size_t)j * K + i] - de[j] * kt[i];
                        dkt[i] -= p * de[j];
                    }
                double *dglt = dgl + IX_TK(d, bb, toff + t, h, 0, K), *dbxt = dbx + IX_TK(d, bb, toff + t, h, 0, K);
                for (int i = 0; i < K; ++i) {
                    double da = 0.0;
                    for (int j = 0; j < V; ++j) da += Sprev[(size_t)j * K + i] * dP[(size_t)j * K + i];
                    const size_t ix = IX_TK(d, bb, toff + t, h, i, K);
                    /* a = g b, log g = -amp softplus(gl + tau) => dg/dgl = dg/dtau
                       = -g amp sigmoid(gl + tau), dg/dA_dec = g log g */
                    const double x = gl[ix] + decay_bias(d, tau, h, i);
                    dglt[i] = -da * a[i] * amp * sigm(x);
                    if (tau) dtauu[i] += dglt[i];
                    if (A_dec) dAdec_u[u] += da * a[i] * (-amp * softplus(x));   /* log g, finite where g underflows */
                    const double dbeta = da * g[i] * bg[i] * (1.0 - bg[i]);
                    dbxt[i] = dbeta;
                    dd[i] += dbeta;
                }
                for (int j = 0; j < V; ++j)
                    for (int i = 0; i < K; ++i) dS[(size_t)j * K + i] = dP[(size_t)j * K + i] * a[i];
                dwl[((size_t)bb * T + toff + t) * H + h] = dw * w * (1.0 - w);
                ddw += dw * w * (1.0 - w);
            }
            /* chunk start: Delta = A z, z = B m */
            for (int j = 0; j < V; ++j) dox[j] = 0.0;
            if (!d->content_off) {
                const double *z = zc + (size_t)c * R, *m = mc + (size_t)c * V;
                for (int j = 0; j < R; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < K; ++i) s += A[((size_t)h * K + i) * R + j] * dd[i];
                    if (Aw) s += Aw[(size_t)h * R + j] * ddw;   /* dw_c = Aw . z */
                    dz[j] = s;
                }
                if (Aw)
                    for (int j = 0; j < R; ++j) dAwu[j] += ddw * z[j];
                for (int i = 0; i < K; ++i)
                    for (int j = 0; j < R; ++j) dAu[(size_t)i * R + j] += dd[i] * z[j];
                for (int vv = 0; vv < V; ++vv) {
                    double s = 0.0;
                    for (int j = 0; j < R; ++j) s += Bm[((size_t)h * R + j) * V + vv] * dz[j];
                    dm[vv] = s;
                }
                for (int j = 0; j < R; ++j)
                    for (int vv = 0; vv < V; ++vv) dBu[(size_t)j * V + vv] += dz[j] * m[vv];
                if (d->mc_mode == 0) {
                    const double *qbar = qb + (size_t)c * K, *Sc = Sb + (size_t)c * VK;
                    for (int j = 0; j < V; ++j)
                        for (int i = 0; i < K; ++i) dS[(size_t)j * K + i] += dm[j] * qbar[i];
                    for (int i = 0; i < K; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < V; ++j) s += Sc[(size_t)j * K + i] * dm[j];
                        tmp[i] = s / n;
                    }
                    for (int t = t0; t < t1; ++t)
                        for (int i = 0; i < K; ++i) dq[IX_TK(d, bb, toff + t, h, i, K)] += tmp[i];
                } else if (c > 0) {
                    const int np = L; /* every chunk before the last is complete */
                    for (int j = 0; j < V; ++j) dox[j] = dm[j] / np;
                } else if (dm_prev_in) {
                    memcpy(dm_prev_in + (size_t)u * V, dm, sizeof(double) * (size_t)V);
                }
            }
        }
        if (dm_prev_in && N == 0) {   /* no token: m_prev_out is m_prev_in passed through */
            for (int j = 0; j < V; ++j) dm_prev_in[(size_t)u * V + j] = dm_prev_out ? dm_prev_out[(size_t)u * V + j] : 0.0;
        } else if (dm_prev_in && (d->content_off || d->mc_mode == 0)) {
            memset(dm_prev_in + (size_t)u * V, 0, sizeof(double) * (size_t)V);
        }
        if (dS0) memcpy(dS0 + (size_t)u * VK, dS, sizeof(double) * VK);
        free(Sb); free(mc); free(zc); free(dc); free(qb); free(St); free(S); free(dS); free(dP);
        free(at); free(gt); free(bt); free(wt); free(et); free(qt); free(kt); free(vt); free(ot);
        free(osum); free(mprev); free(dox); free(dot); free(de); free(dd); free(dz); free(dm); free(tmp);
    }
    /* dA, dB: per-head sums over the batch in a fixed order */
    memset(dA, 0, sizeof(double) * (size_t)H * K * R);
    memset(dB, 0, sizeof(double) * (size_t)H * R * V);
    if (dAw) memset(dAw, 0, sizeof(double) * (size_t)H * R);
    if (dA_dec) memset(dA_dec, 0, sizeof(double) * (size_t)H);
    if (dtau) memset(dtau, 0, sizeof(double) * (size_t)H * K);
    for (int u = 0; u < units; ++u) {
        const int h = u % H;
        if (dA_dec) dA_dec[h] += dAdec_u[u];
        if (dtau)
            for (int i = 0; i < K; ++i) dtau[(size_t)h * K + i] += dtau_u[(size_t)u * K + i];
        for (size_t x = 0; x < (size_t)K * R; ++x) dA[(size_t)h * K * R + x] += dA_u[(size_t)u * K * R + x];
        for (size_t x = 0; x < (size_t)R * V; ++x) dB[(size_t)h * R * V + x] += dB_u[(size_t)u * R * V + x];
        if (dAw)
            for (int j = 0; j < R; ++j) dAw[(size_t)h * R + j] += dAw_u[(size_t)u * R + j];
    }
    free(dA_u); free(dB_u); free(dAw_u); free(dAdec_u); free(dtau_u);
    return 0;
}

/*
 * One decode step for every (b,h): the recurrence above for a single token.
 *   mc_mode 0: the content signal is read from the state before this token,
 *              m = S q (the L = 1 readout; a chunk mean over future tokens is not
 *              available when decoding).
 *   mc_mode 1: the content signal is the mean output of the previous complete block of
 *              L tokens.  mstate [B,H,2,V] holds (running sum of o in the current block,
 *              mean of the previous block); pos [B,H] counts tokens consumed.
 * Inputs q, k, g_logit, bx: [B,H,K]; v: [B,H,V]; w_logit: [B,H]; Aw [H,R], A_dec [H] and
 * ti [H,K] or NULL;
 * S [B,H,V,K] in/out; o: [B,H,V].
 */
int orc_step(const orc_dims *d, const double *q, const double *k, const double *v,
             const double *gl, const double *bx, const double *wl, const double *A,
             const double *Bm, const double *Aw, const double *A_dec, const double *tau, double *S,
             double *mstate, int *pos, double *o) {
    if (check_dims(d)) return -1;
    const int K = d->K, V = d->V, R = d->R, H = d->H, L = d->L;
    const int units = d->B * H;
#pragma omp parallel for schedule(static)
    for (int u = 0; u < units; ++u) {
        const int h = u % H;
        double *Su = S + (size_t)u * V * K;
        double *m = calloc(V, sizeof(double)), *z = calloc(R, sizeof(double));
        double *delta = calloc(K, sizeof(double)), *a = calloc(K, sizeof(double));
        double *e = calloc(V, sizeof(double));
        const double *qu = q + (size_t)u * K, *ku = k + (size_t)u * K;
        if (!d->content_off) {
            if (d->mc_mode == 0) {
                for (int j = 0; j < V; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < K; ++i) s += Su[(size_t)j * K + i] * qu[i];
                    m[j] = s;
                }
            } else {
                double *msum = mstate + (size_t)u * 2 * V, *mprev = msum + V;
                if (pos[u] > 0 && pos[u] % L == 0)
                    for (int j = 0; j < V; ++j) { mprev[j] = msum[j] / L; msum[j] = 0.0; }
                memcpy(m, mprev, sizeof(double) * (size_t)V);
            }
            content_delta(d, h, A, Bm, m, z, delta);
        }
        for (int i = 0; i < K; ++i) {
            const double g = exp(-decay_amp(A_dec, h) * softplus(gl[(size_t)u * K + i] + decay_bias(d, tau, h, i)));
            const double bb = d->content_off ? sigm(bx[(size_t)u * K + i]) : sigm(bx[(size_t)u * K + i] + delta[i]);
            a[i] = g * bb;
        }
        const double w = sigm(wl[u] + write_bias(d, h, Aw, z));
        token_update(d, Su, a, w, ku, v + (size_t)u * V, qu, e, o + (size_t)u * V);
        if (d->mc_mode == 1) {
            double *msum = mstate + (size_t)u * 2 * V;
            for (int j = 0; j < V; ++j) msum[j] += o[(size_t)u * V + j];
        }
        pos[u] += 1;
        free(m); free(z); free(delta); free(a); free(e);
    }
    return 0;
}
