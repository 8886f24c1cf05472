/*
 * gdn2_oracle.c -- plain fp64 CPU oracle of the Gated Delta Rule-2 operator.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. The product path (the CUDA
 * library and its Python binding) never calls it and shares no code with it.
 *
 * What it computes -- "Gated DeltaNet-2: Decoupling Erase and Write in Linear
 * Attention":
 *   - GitHub README (NVlabs/GatedDeltaNet-2), method bullets: a channel-wise
 *     erase gate b_t in [0,1]^{d_k} picks which key-side coordinates of the
 *     DECAYED state are read and removed; a channel-wise write gate
 *     w_t in [0,1]^{d_v} picks which value-side coordinates of the new content
 *     are committed; a channel-wise decay D_t = Diag(alpha_t) (from KDA).
 *     The paragraph after the (unextracted) state equation: relative to KDA the
 *     right factor of the rank-one erase becomes channel-selective on the key
 *     axis and the write term channel-selective on the value axis.
 *   - arXiv abstract 2605.22791: delta-rule models subtract the current read
 *     before writing; the state has a fixed size; decoding is constant-memory.
 *
 * The page's state equation itself did not survive extraction. Reading adopted
 * (the plainest one consistent with the bullets above):
 *
 *     S_t = (I - k_t (b_t*k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t*v_t)^T
 *     o_t = S_t^T q_t                     (read-out after the update)
 *
 * with S_t of shape d_k x d_v, '*' the elementwise product and
 * alpha_t = exp(log_alpha_t) (the decay is passed in log form). It is computed
 * here one token at a time, in the order the words describe it:
 *
 *     P   = Diag(alpha_t) S_{t-1}          decay
 *     r   = P^T (b_t*k_t)                  read of the decayed state through the erase gate
 *     S_t = P + k_t (w_t*v_t - r)^T        remove the read, commit the gated write
 *
 * which is algebraically the same as the product form above.
 *
 * The backward is the reverse-mode adjoint of exactly these steps for the loss
 * L = <dout, o> + <dST, S_T>, with S_{t-1} recomputed from fp64 checkpoints.
 *
 * Layouts (row-major, contiguous): token tensors [B, T, H, D]; decode tensors
 * [B, H, D]; states [B, H, Dk, Dv]. Everything is double precision.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TOK(p, bb, t, hh, D, T, H) ((p) + ((((size_t)(bb) * (T) + (t)) * (H) + (hh)) * (size_t)(D)))
#define STATE(p, bb, hh, H, Dk, Dv) ((p) + (((size_t)(bb) * (H) + (hh)) * (size_t)(Dk) * (size_t)(Dv)))

int gdn2_oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One recurrence step on the value columns [j0, j1) of one head's state S
 * (d_k x d_v, row stride Dv). The columns of S never mix: the decay, the erase
 * read r_j and the write act on each column j on its own. Writes o[j] for the
 * same columns.
 */
static void step_columns(double* S, const double* q, const double* k, const double* v,
                         const double* la, const double* b, const double* w, double* o,
                         int Dk, int Dv, int j0, int j1) {
    for (int j = j0; j < j1; ++j) {
        /* P = Diag(alpha) S ; r_j = sum_i P_ij (b_i k_i) */
        double r = 0.0;
        for (int i = 0; i < Dk; ++i) {
            double p = exp(la[i]) * S[(size_t)i * Dv + j];
            S[(size_t)i * Dv + j] = p;
            r += p * (b[i] * k[i]);
        }
        /* S = P + k (w_j v_j - r_j) */
        double delta = w[j] * v[j] - r;
        double oj = 0.0;
        for (int i = 0; i < Dk; ++i) {
            double s = S[(size_t)i * Dv + j] + k[i] * delta;
            S[(size_t)i * Dv + j] = s;
            oj += s * q[i];      /* o = S^T q */
        }
        o[j] = oj;
    }
}

/*
 * Forward over a whole sequence. S0 may be NULL (zero initial state); ST may be
 * NULL (final state not wanted). Work is split over (batch, head, block of 16
 * value columns); each block runs the plain token loop on its own columns, so
 * the result does not depend on the split.
 */
int gdn2_oracle_fwd(const double* q, const double* k, const double* v, const double* log_alpha,
                    const double* b, const double* w, const double* S0, double* o, double* ST,
                    int B, int T, int H, int Dk, int Dv) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    const int CB = 16;
    const int nblk = (Dv + CB - 1) / CB;
    const long units = (long)B * H * nblk;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        int blk = (int)(u % nblk);
        int hh = (int)((u / nblk) % H);
        int bb = (int)(u / ((long)nblk * H));
        int j0 = blk * CB, j1 = j0 + CB < Dv ? j0 + CB : Dv;
        double* S = (double*)malloc((size_t)Dk * Dv * sizeof(double));
        if (!S) { err = 2; continue; }
        if (S0) memcpy(S, STATE(S0, bb, hh, H, Dk, Dv), (size_t)Dk * Dv * sizeof(double));
        else memset(S, 0, (size_t)Dk * Dv * sizeof(double));
        for (int t = 0; t < T; ++t) {
            step_columns(S, TOK(q, bb, t, hh, Dk, T, H), TOK(k, bb, t, hh, Dk, T, H),
                         TOK(v, bb, t, hh, Dv, T, H), TOK(log_alpha, bb, t, hh, Dk, T, H),
                         TOK(b, bb, t, hh, Dk, T, H), TOK(w, bb, t, hh, Dv, T, H),
                         TOK(o, bb, t, hh, Dv, T, H), Dk, Dv, j0, j1);
        }
        if (ST) {
            double* dst = STATE(ST, bb, hh, H, Dk, Dv);
            for (int i = 0; i < Dk; ++i)
                for (int j = j0; j < j1; ++j) dst[(size_t)i * Dv + j] = S[(size_t)i * Dv + j];
        }
        free(S);
    }
    return err;
}

/*
 * One decode step: the same recurrence step applied to one token per (b, h),
 * state updated in place. Inputs are [B, H, D]; S is [B, H, Dk, Dv].
 */
int gdn2_oracle_decode(const double* q, const double* k, const double* v, const double* log_alpha,
                       const double* b, const double* w, double* S, double* o,
                       int B, int H, int Dk, int Dv) {
    if (B < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    const long units = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long u = 0; u < units; ++u) {
        size_t kk = (size_t)u * Dk, vv = (size_t)u * Dv;
        step_columns(S + (size_t)u * Dk * Dv, q + kk, k + kk, v + vv, log_alpha + kk, b + kk,
                     w + vv, o + vv, Dk, Dv, 0, Dv);
    }
    return 0;
}

/*
 * Backward: reverse-mode adjoint of the token recurrence for
 *     L = <dout, o> + <dST, S_T>      (dST may be NULL: zero).
 * For each token, going backwards, with dS = dL/dS_t on entry:
 *     o_t = S_t^T q_t          dS += q_t dout_t^T ;  dq_t = S_t dout_t
 *     S_t = P + k_t delta^T    dk_t = dS delta ;     ddelta = dS^T k_t ;  dP = dS
 *     delta = u - r            du = ddelta ;         dr = -ddelta
 *     r = P^T e                dP += e dr^T ;        de = P dr
 *     u = w_t*v_t              dw_t = du*v_t ;       dv_t = du*w_t
 *     e = b_t*k_t              db_t = de*k_t ;       dk_t += de*b_t
 *     P = Diag(alpha) S_{t-1}  dlog_alpha_t,i = sum_j dP_ij P_ij ;  dS = Diag(alpha) dP
 * and dS0 = dS after the first token. S_{t-1} comes from a forward recompute
 * segment by segment, from checkpoints taken every CK tokens.
 * Any of dq..dS0 may be NULL if not wanted (dout must be given).
 */
int gdn2_oracle_bwd(const double* q, const double* k, const double* v, const double* log_alpha,
                    const double* b, const double* w, const double* S0, const double* dout,
                    const double* dST, double* dq, double* dk, double* dv, double* dlog_alpha,
                    double* db, double* dw, double* dS0, int B, int T, int H, int Dk, int Dv) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0 || !dout) return 1;
    const int CK = 64;
    const int nseg = (T + CK - 1) / CK;
    const long units = (long)B * H;
    const size_t SZ = (size_t)Dk * Dv;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        int hh = (int)(u % H), bb = (int)(u / H);
        /* ckpt[s]: state before token s*CK; seg[i]: state before token t0+i */
        double* ckpt = (double*)malloc((size_t)(nseg > 0 ? nseg : 1) * SZ * sizeof(double));
        double* seg = (double*)malloc((size_t)(CK + 1) * SZ * sizeof(double));
        double* dS = (double*)malloc(SZ * sizeof(double));
        double* P = (double*)malloc(SZ * sizeof(double));
        double* tmp_o = (double*)malloc((size_t)Dv * sizeof(double));
        double* vecs = (double*)malloc((size_t)(6 * Dk + 6 * Dv) * sizeof(double));
        if (!ckpt || !seg || !dS || !P || !tmp_o || !vecs) {
            err = 2;
            free(ckpt); free(seg); free(dS); free(P); free(tmp_o); free(vecs);
            continue;
        }
        double *e = vecs, *alpha = vecs + Dk, *dqv = vecs + 2 * Dk, *dkv = vecs + 3 * Dk,
               *de = vecs + 4 * Dk, *dla = vecs + 5 * Dk;
        double *uu = vecs + 6 * Dk, *delta = uu + Dv, *ddelta = uu + 2 * Dv, *dr = uu + 3 * Dv,
               *rr = uu + 4 * Dv, *doj = uu + 5 * Dv;
        (void)doj;

        /* forward pass: checkpoints only */
        double* S = seg;
        if (S0) memcpy(S, STATE(S0, bb, hh, H, Dk, Dv), SZ * sizeof(double));
        else memset(S, 0, SZ * sizeof(double));
        for (int t = 0; t < T; ++t) {
            if (t % CK == 0) memcpy(ckpt + (size_t)(t / CK) * SZ, S, SZ * sizeof(double));
            step_columns(S, TOK(q, bb, t, hh, Dk, T, H), TOK(k, bb, t, hh, Dk, T, H),
                         TOK(v, bb, t, hh, Dv, T, H), TOK(log_alpha, bb, t, hh, Dk, T, H),
                         TOK(b, bb, t, hh, Dk, T, H), TOK(w, bb, t, hh, Dv, T, H), tmp_o, Dk, Dv,
                         0, Dv);
        }

        if (dST) memcpy(dS, STATE(dST, bb, hh, H, Dk, Dv), SZ * sizeof(double));
        else memset(dS, 0, SZ * sizeof(double));

        for (int s = nseg - 1; s >= 0; --s) {
            int t0 = s * CK, t1 = t0 + CK < T ? t0 + CK : T;
            /* recompute seg[i] = S_{t0+i-1} (state before token t0+i), i = 0..t1-t0-1 */
            memcpy(seg, ckpt + (size_t)s * SZ, SZ * sizeof(double));
            for (int t = t0; t < t1 - 1; ++t) {
                double* nxt = seg + (size_t)(t - t0 + 1) * SZ;
                memcpy(nxt, seg + (size_t)(t - t0) * SZ, SZ * sizeof(double));
                step_columns(nxt, TOK(q, bb, t, hh, Dk, T, H), TOK(k, bb, t, hh, Dk, T, H),
                             TOK(v, bb, t, hh, Dv, T, H), TOK(log_alpha, bb, t, hh, Dk, T, H),
                             TOK(b, bb, t, hh, Dk, T, H), TOK(w, bb, t, hh, Dv, T, H), tmp_o, Dk,
                             Dv, 0, Dv);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const double* Sprev = seg + (size_t)(t - t0) * SZ;
                const double* qt = TOK(q, bb, t, hh, Dk, T, H);
                const double* kt = TOK(k, bb, t, hh, Dk, T, H);
                const double* vt = TOK(v, bb, t, hh, Dv, T, H);
                const double* lat = TOK(log_alpha, bb, t, hh, Dk, T, H);
                const double* bt = TOK(b, bb, t, hh, Dk, T, H);
                const double* wt = TOK(w, bb, t, hh, Dv, T, H);
                const double* dot = TOK(dout, bb, t, hh, Dv, T, H);
                /* recompute the step's intermediates */
                for (int i = 0; i < Dk; ++i) { alpha[i] = exp(lat[i]); e[i] = bt[i] * kt[i]; }
                for (int i = 0; i < Dk; ++i)
                    for (int j = 0; j < Dv; ++j) P[(size_t)i * Dv + j] = alpha[i] * Sprev[(size_t)i * Dv + j];
                for (int j = 0; j < Dv; ++j) {
                    double r = 0.0;
                    for (int i = 0; i < Dk; ++i) r += P[(size_t)i * Dv + j] * e[i];
                    rr[j] = r;
                    uu[j] = wt[j] * vt[j];
                    delta[j] = uu[j] - r;
                }
                /* o_t = S_t^T q_t, with S_t = P + k delta^T */
                for (int i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < Dv; ++j) {
                        double st = P[(size_t)i * Dv + j] + kt[i] * delta[j];
                        acc += st * dot[j];                    /* dq_t = S_t dout_t */
                        dS[(size_t)i * Dv + j] += qt[i] * dot[j]; /* dS += q dout^T */
                    }
                    dqv[i] = acc;
                }
                /* S_t = P + k delta^T */
                for (int i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < Dv; ++j) acc += dS[(size_t)i * Dv + j] * delta[j];
                    dkv[i] = acc;                               /* dk_t = dS delta */
                }
                for (int j = 0; j < Dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < Dk; ++i) acc += dS[(size_t)i * Dv + j] * kt[i];
                    ddelta[j] = acc;                            /* ddelta = dS^T k */
                    dr[j] = -acc;                               /* delta = u - r */
                }
                /* r = P^T e: dP = dS + e dr^T ; de = P dr */
                for (int i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < Dv; ++j) acc += P[(size_t)i * Dv + j] * dr[j];
                    de[i] = acc;
                }
                for (int i = 0; i < Dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < Dv; ++j) {
                        double dp = dS[(size_t)i * Dv + j] + e[i] * dr[j];
                        acc += dp * P[(size_t)i * Dv + j];      /* dlog_alpha = rowsum(dP * P) */
                        dS[(size_t)i * Dv + j] = alpha[i] * dp; /* dS_{t-1} = Diag(alpha) dP */
                    }
                    dla[i] = acc;
                }
                if (dq) memcpy(TOK(dq, bb, t, hh, Dk, T, H), dqv, (size_t)Dk * sizeof(double));
                if (dk) {
                    double* o_ = TOK(dk, bb, t, hh, Dk, T, H);
                    for (int i = 0; i < Dk; ++i) o_[i] = dkv[i] + de[i] * bt[i];
                }
                if (db) {
                    double* o_ = TOK(db, bb, t, hh, Dk, T, H);
                    for (int i = 0; i < Dk; ++i) o_[i] = de[i] * kt[i];
                }
                if (dlog_alpha) memcpy(TOK(dlog_alpha, bb, t, hh, Dk, T, H), dla, (size_t)Dk * sizeof(double));
                if (dv) {
                    double* o_ = TOK(dv, bb, t, hh, Dv, T, H);
                    for (int j = 0; j < Dv; ++j) o_[j] = ddelta[j] * wt[j];   /* du = ddelta */
                }
                if (dw) {
                    double* o_ = TOK(dw, bb, t, hh, Dv, T, H);
                    for (int j = 0; j < Dv; ++j) o_[j] = ddelta[j] * vt[j];
                }
            }
        }
        if (dS0) memcpy(STATE(dS0, bb, hh, H, Dk, Dv), dS, SZ * sizeof(double));
        free(ckpt); free(seg); free(dS); free(P); free(tmp_o); free(vecs);
    }
    return err;
}
