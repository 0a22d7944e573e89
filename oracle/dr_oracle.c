/*
 * Plain fp64 CPU oracle of the delta-rule recurrent-memory scan (forward).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header, table or helper with the
 * CUDA library; the two meet only through seeded inputs.
 *
 * What it computes is the per-token definition, written out one token at a time,
 * in fp64, independently for every (batch, head) sequence. There is no chunking,
 * blocking, fusion or reordering.
 *
 * Sources (the three web pages this subject is drawn from; the log-linear scan at the end
 * of this file follows the third, "Adaptive memory decay for log-linear attention"):
 *  - "Mechanisms, trade-offs and cross-layer routing of linear-attention
 *    architectures" (aitrends.kr), section "Technical details" (기술 상세) and
 *    "Understanding the key idea": memory W in R^{d_v x d_phi}, readout y = W phi(q);
 *    DeltaNet prediction vbar = W_{t-1} kappa, residual r = v - vbar, write
 *    W <- W + beta r (x) kappa; Gated DeltaNet W <- alpha W + beta r_alpha (x) kappa
 *    (scalar decay); Kimi Delta Attention decays per key-feature channel.
 *    Gated DeltaNet-2 separates a per-key-channel erase gate b and a per-value-channel
 *    write gate w: erase direction e = b (.) kappa, write target z = w (.) v, and it
 *    writes the residual r = z - W~ e. The CLVR passages of the same page route a
 *    layer's internal write signal (write value or residual) to later layers.
 *  - "Variational Linear Attention (VLA)" (gist.science 2605.11196), section 2.1
 *    (plain accumulation S_t = S_{t-1} + v_t k_t^T), section 2.2 (inverse penalty
 *    A_t = M_t^{-1} kept by a Sherman-Morrison rank-1 update) and section 2.3
 *    (steps 1-3: A-update, alpha_hat = A_t k_hat / ||A_t k_hat||,
 *    S_t = S_{t-1} + (v_t - S_{t-1} k_hat_t) alpha_hat_t^T).
 *
 * Readings where the pages are silent or garbled (each is listed in the design notes):
 *  - Gated variants take the residual against the DECAYED state:
 *    S' = alpha (.) S_{t-1};  r = v - S' k;  S_t = S' + beta r k^T.
 *    This is the only reading under which "unit k, beta = 1 => S_t k_t = v_t"
 *    holds for alpha != 1. The literal reading r = v - S_{t-1} k is kept behind
 *    the flag `residual_pre_decay` (oracle-only option).
 *  - KDA's alpha_t in (0,1)^{d_k} scales the COLUMNS of S (key-feature axis).
 *  - Readout after the write: o_t = S_t q_t. No feature map and no 1/sqrt(d_k)
 *    scale inside the scan; q and k arrive as the caller prepared them.
 *  - Plain linear attention ignores beta and gate.
 *  - Gated DeltaNet-2: W~ is the decayed memory alpha_t S_{t-1} (scalar alpha, as in
 *    Gated DeltaNet), and the residual is written along the erase direction e:
 *    S_t = W~ + beta r e^T, so that with a unit e and beta = 1, S_t e = z exactly.
 *    With b = w = 1 it is Gated DeltaNet.
 *  - The exported write value of a token is u_t = beta_t r_t, the vector the step adds
 *    to memory along its key (along e for Gated DeltaNet-2); plain linear attention
 *    writes u_t = v_t.
 *  - VLA: z_t = A_{t-1} u_t (Sherman-Morrison for M_t = M_{t-1} + u_t u_t^T),
 *    A_0 = I / lambda0, readout o_t = S_t q_hat_t, no beta and no decay.
 *  - VLA ratio readout (section 2.3: the output is a ratio of recurrences, as in linear
 *    attention, with an ELU+1 feature map): the denominator recurrence is the same write
 *    applied to one more value channel held at 1, n_t = n_{t-1} + (1 - n_{t-1} k_hat_t)
 *    alpha_hat_t^T (n_0 = 0 unless given), and o_t = S_t q_t / (n_t q_t). The feature map
 *    is the caller's, like every other feature map here: q arrives as phi(q) and k_hat as
 *    phi(k) / ||phi(k)||.
 *
 * Layouts (all row-major, contiguous):
 *   q, k   [B, H, T, dk]      v, out [B, H, T, dv]      beta [B, H, T]
 *   gate   GDN, GDN2: [B, H, T]   KDA: [B, H, T, dk]    (alpha values, not logs)
 *   erase  GDN2: [B, H, T, dk]   write  GDN2: [B, H, T, dv]   u_out [B, H, T, dv]
 *   S0, S_final [B, H, dv, dk]   (S maps keys to values: S k in R^{dv})
 *   VLA: q, k, v, u, out [B, H, T, d];  S0, S_final, A0, A_final [B, H, d, d]
 */
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_LINEAR 0
#define ORACLE_DELTANET 1
#define ORACLE_GDN 2
#define ORACLE_KDA 3
#define ORACLE_GDN2 4

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One (batch, head) sequence of the delta-rule family. S is dv x dk, updated in place.
 * work holds dk + dv doubles (Gated DeltaNet-2's e and z). */
static void dr_sequence(const double* q, const double* k, const double* v,
                        const double* beta, const double* gate, const double* erase,
                        const double* write, double* S, double* out, double* u_out,
                        double* decay, double* pred, double* work,
                        long T, int dk, int dv, int mode, int residual_pre_decay) {
    for (long t = 0; t < T; ++t) {
        const double* kt = k + t * dk;
        const double* qt = q + t * dk;
        const double* vt = v + t * dv;
        double* ot = out + t * dv;
        double* ut = u_out ? u_out + t * dv : NULL;

        if (mode == ORACLE_LINEAR) {
            /* S_t = S_{t-1} + v_t k_t^T  (VLA page, section 2.1) */
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    S[(long)i * dk + j] += vt[i] * kt[j];
            if (ut)
                for (int i = 0; i < dv; ++i) ut[i] = vt[i];
        } else {
            /* Gated DeltaNet-2 reads and writes along e = b (.) k with the target z = w (.) v;
             * every other variant along k with the target v */
            const double* kk = kt;
            const double* vv = vt;
            if (mode == ORACLE_GDN2) {
                double* e = work;
                double* z = work + dk;
                for (int j = 0; j < dk; ++j) e[j] = erase[t * dk + j] * kt[j];
                for (int i = 0; i < dv; ++i) z[i] = write[t * dv + i] * vt[i];
                kk = e;
                vv = z;
            }
            /* decay factor per key channel j: 1 (DeltaNet), alpha_t (GDN, GDN2), alpha_t[j] (KDA) */
            for (int j = 0; j < dk; ++j) {
                if (mode == ORACLE_DELTANET) decay[j] = 1.0;
                else if (mode == ORACLE_GDN || mode == ORACLE_GDN2) decay[j] = gate[t];
                else decay[j] = gate[t * dk + j];
            }
            /* prediction vbar = S' k, with S' = S (.) decay (or S itself, literal reading) */
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) {
                    double s = S[(long)i * dk + j];
                    if (!residual_pre_decay) s *= decay[j];
                    acc += s * kk[j];
                }
                pred[i] = acc;
            }
            /* S_t = S' + beta_t (v_t - vbar) k_t^T */
            const double b = beta[t];
            for (int i = 0; i < dv; ++i) {
                const double r = vv[i] - pred[i];
                for (int j = 0; j < dk; ++j) {
                    long ij = (long)i * dk + j;
                    S[ij] = decay[j] * S[ij] + b * r * kk[j];
                }
                if (ut) ut[i] = b * r;
            }
        }
        /* readout after the write: o_t = S_t q_t */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(long)i * dk + j] * qt[j];
            ot[i] = acc;
        }
    }
}

/*
 * Delta-rule family scan with every option. beta may be NULL for LINEAR; gate is NULL for
 * LINEAR and DELTANET, [B,H,T] for GDN and GDN2, [B,H,T,dk] for KDA; erase [B,H,T,dk] and
 * write [B,H,T,dv] are GDN2's gates (NULL otherwise). S0 NULL means zeros; S_final and
 * u_out (the per-token write values) NULL mean not written. Returns 0, or -1 on a bad
 * argument.
 */
int oracle_dr_scan_ex(const double* q, const double* k, const double* v,
                      const double* beta, const double* gate, const double* erase,
                      const double* write, const double* S0,
                      double* out, double* S_final, double* u_out,
                      int B, int H, int T, int dk, int dv, int mode, int residual_pre_decay) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    if (mode < ORACLE_LINEAR || mode > ORACLE_GDN2) return -1;
    if (!q || !k || !v || !out) return -1;
    if (mode != ORACLE_LINEAR && !beta) return -1;
    if ((mode == ORACLE_GDN || mode == ORACLE_KDA || mode == ORACLE_GDN2) && !gate) return -1;
    if (mode == ORACLE_GDN2 && (!erase || !write)) return -1;
    const long BH = (long)B * H;
    const long state = (long)dv * dk;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double* S = (double*)malloc(sizeof(double) * (size_t)state);
        double* decay = (double*)malloc(sizeof(double) * (size_t)dk);
        double* pred = (double*)malloc(sizeof(double) * (size_t)dv);
        double* work = (double*)malloc(sizeof(double) * (size_t)(dk + dv));
        if (!S || !decay || !pred || !work) {
            failed = 1;
        } else {
            if (S0) memcpy(S, S0 + bh * state, sizeof(double) * (size_t)state);
            else memset(S, 0, sizeof(double) * (size_t)state);
            const double* g = NULL;
            if (mode == ORACLE_GDN || mode == ORACLE_GDN2) g = gate + bh * T;
            if (mode == ORACLE_KDA) g = gate + bh * (long)T * dk;
            const int gdn2 = mode == ORACLE_GDN2;
            dr_sequence(q + bh * (long)T * dk, k + bh * (long)T * dk, v + bh * (long)T * dv,
                        beta ? beta + bh * T : NULL, g,
                        gdn2 ? erase + bh * (long)T * dk : NULL,
                        gdn2 ? write + bh * (long)T * dv : NULL, S, out + bh * (long)T * dv,
                        u_out ? u_out + bh * (long)T * dv : NULL, decay, pred, work, T, dk, dv,
                        mode, residual_pre_decay);
            if (S_final) memcpy(S_final + bh * state, S, sizeof(double) * (size_t)state);
        }
        free(S);
        free(decay);
        free(pred);
        free(work);
    }
    return failed ? -1 : 0;
}

/* The delta-rule family scan without Gated DeltaNet-2 and without write values. */
int oracle_dr_scan(const double* q, const double* k, const double* v,
                   const double* beta, const double* gate, const double* S0,
                   double* out, double* S_final,
                   int B, int H, int T, int dk, int dv, int mode, int residual_pre_decay) {
    if (mode == ORACLE_GDN2) return -1;
    return oracle_dr_scan_ex(q, k, v, beta, gate, NULL, NULL, S0, out, S_final, NULL, B, H, T,
                             dk, dv, mode, residual_pre_decay);
}

/* One VLA sequence. S and A are d x d, updated in place; work holds 3*d doubles. n (d
 * doubles) is the ratio readout's denominator state, NULL for the plain readout. */
static void vla_sequence(const double* q, const double* k, const double* v, const double* u,
                         double* S, double* A, double* n, double* out, double* work, long T,
                         int d) {
    double* z = work;          /* z_t = A_{t-1} u_t */
    double* y = work + d;      /* A_t k_hat_t, then alpha_hat_t */
    double* r = work + 2 * d;  /* v_t - S_{t-1} k_hat_t */
    for (long t = 0; t < T; ++t) {
        const double* ut = u + t * d;
        const double* kt = k + t * d;
        const double* vt = v + t * d;
        const double* qt = q + t * d;
        double* ot = out + t * d;

        /* step 1: A_t = A_{t-1} - z z^T / (1 + u^T z), z = A_{t-1} u  (section 2.3, Sherman-Morrison) */
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += A[(long)i * d + j] * ut[j];
            z[i] = acc;
        }
        double den = 1.0;
        for (int i = 0; i < d; ++i) den += ut[i] * z[i];
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) A[(long)i * d + j] -= z[i] * z[j] / den;

        /* step 2: alpha_hat = A_t k_hat / ||A_t k_hat|| */
        double nrm2 = 0.0;
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += A[(long)i * d + j] * kt[j];
            y[i] = acc;
            nrm2 += acc * acc;
        }
        const double inv = 1.0 / sqrt(nrm2);
        for (int i = 0; i < d; ++i) y[i] *= inv;

        /* step 3: S_t = S_{t-1} + (v - S_{t-1} k_hat) alpha_hat^T */
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += S[(long)i * d + j] * kt[j];
            r[i] = vt[i] - acc;
        }
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) S[(long)i * d + j] += r[i] * y[j];

        /* ratio readout: the same write on the value 1, n_t = n + (1 - n k_hat) alpha_hat^T */
        double nq = 1.0;
        if (n) {
            double nk = 0.0;
            for (int j = 0; j < d; ++j) nk += n[j] * kt[j];
            for (int j = 0; j < d; ++j) n[j] += (1.0 - nk) * y[j];
            nq = 0.0;
            for (int j = 0; j < d; ++j) nq += n[j] * qt[j];
        }

        /* readout o_t = S_t q_hat_t (divided by n_t q_t for the ratio readout) */
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += S[(long)i * d + j] * qt[j];
            ot[i] = n ? acc / nq : acc;
        }
    }
}

/*
 * VLA Sherman-Morrison scan with either readout. S0 NULL = zeros; A0 NULL = I / lambda0;
 * n0 [B,H,d] NULL = zeros (ratio readout only). S_final / A_final / n_final NULL = not
 * written. readout 0: o_t = S_t q_t; 1: o_t = S_t q_t / (n_t q_t). Returns 0, or -1 on a
 * bad argument.
 */
int oracle_vla_scan_ex(const double* q, const double* k, const double* v, const double* u,
                       const double* S0, const double* A0, const double* n0, double lambda0,
                       double* out, double* S_final, double* A_final, double* n_final,
                       int B, int H, int T, int d, int readout) {
    if (B < 0 || H < 0 || T < 0 || d <= 0) return -1;
    if (readout != 0 && readout != 1) return -1;
    if (!q || !k || !v || !u || !out) return -1;
    if (!A0 && !(lambda0 > 0.0)) return -1;
    const long BH = (long)B * H;
    const long dd = (long)d * d;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double* S = (double*)malloc(sizeof(double) * (size_t)dd);
        double* A = (double*)malloc(sizeof(double) * (size_t)dd);
        double* work = (double*)malloc(sizeof(double) * 3 * (size_t)d);
        double* n = readout ? (double*)malloc(sizeof(double) * (size_t)d) : NULL;
        if (!S || !A || !work || (readout && !n)) {
            failed = 1;
        } else {
            if (S0) memcpy(S, S0 + bh * dd, sizeof(double) * (size_t)dd);
            else memset(S, 0, sizeof(double) * (size_t)dd);
            if (A0) {
                memcpy(A, A0 + bh * dd, sizeof(double) * (size_t)dd);
            } else {
                memset(A, 0, sizeof(double) * (size_t)dd);
                for (int i = 0; i < d; ++i) A[(long)i * d + i] = 1.0 / lambda0;
            }
            if (n) {
                if (n0) memcpy(n, n0 + bh * d, sizeof(double) * (size_t)d);
                else memset(n, 0, sizeof(double) * (size_t)d);
            }
            const long off = bh * (long)T * d;
            vla_sequence(q + off, k + off, v + off, u + off, S, A, n, out + off, work, T, d);
            if (S_final) memcpy(S_final + bh * dd, S, sizeof(double) * (size_t)dd);
            if (A_final) memcpy(A_final + bh * dd, A, sizeof(double) * (size_t)dd);
            if (n && n_final) memcpy(n_final + bh * d, n, sizeof(double) * (size_t)d);
        }
        free(S);
        free(A);
        free(work);
        free(n);
    }
    return failed ? -1 : 0;
}

/* VLA scan with the plain readout o_t = S_t q_hat_t (see oracle_vla_scan_ex). */
int oracle_vla_scan(const double* q, const double* k, const double* v, const double* u,
                    const double* S0, const double* A0, double lambda0,
                    double* out, double* S_final, double* A_final,
                    int B, int H, int T, int d) {
    return oracle_vla_scan_ex(q, k, v, u, S0, A0, NULL, lambda0, out, S_final, A_final, NULL,
                              B, H, T, d, 0);
}

/*
 * Log-linear attention ("Adaptive memory decay for log-linear attention", problem definition
 * and method sections): the memory is a Fenwick-tree hierarchy, the state grows as O(log T),
 * and each output is a weighted sum of memory levels with weights lambda_t^(l).
 *
 * Reading taken (plain linear-attention memories, no decay or delta rule inside a level):
 * at step t (0-based) the prefix [0, t] is split into level 0 = {t} and, for every set bit b
 * of t, level b + 1 = the 2^b tokens before the block of every lower set bit (the Fenwick
 * decomposition of the prefix), and
 *     o_t = lambda_t^(0) (v_t k_t^T) q_t + sum_{b : bit b of t} lambda_t^(b+1) M_b q_t,
 * M_b = sum of v_s k_s^T over level b+1's tokens. The levels are kept as a binary counter:
 * after token t, with j = the number of trailing ones of t, M_j = v_t k_t^T + sum_{b<j} M_b
 * and M_b = 0 for b < j (the blocks of the next step). lambda is [B,H,T,L] with
 * L >= bits(T-1) + 1 levels (level l at index l).
 */
static void loglinear_sequence(const double* q, const double* k, const double* v,
                               const double* lam, double* M, double* cur, double* out,
                               long T, int dk, int dv, int L) {
    const long state = (long)dv * dk;
    memset(M, 0, sizeof(double) * (size_t)state * (size_t)(L > 1 ? L - 1 : 1));
    for (long t = 0; t < T; ++t) {
        const double* kt = k + t * dk;
        const double* qt = q + t * dk;
        const double* vt = v + t * dv;
        const double* lt = lam + t * L;
        double* ot = out + t * dv;
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) cur[(long)i * dk + j] = vt[i] * kt[j];
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += cur[(long)i * dk + j] * qt[j];
            acc *= lt[0];
            for (int b = 0; b + 1 < L; ++b) {
                if (!((t >> b) & 1)) continue;
                double lev = 0.0;
                for (int j = 0; j < dk; ++j) lev += M[b * state + (long)i * dk + j] * qt[j];
                acc += lt[b + 1] * lev;
            }
            ot[i] = acc;
        }
        /* advance the binary counter to t + 1 */
        int jt = 0;
        while ((t >> jt) & 1) ++jt;
        if (jt + 1 < L) {
            double* Mj = M + jt * state;
            for (long e = 0; e < state; ++e) {
                double x = cur[e];
                for (int b = 0; b < jt; ++b) x += M[b * state + e];
                Mj[e] = x;
            }
            for (int b = 0; b < jt; ++b) memset(M + b * state, 0, sizeof(double) * (size_t)state);
        }
    }
}

/*
 * Log-linear attention scan: q, k [B,H,T,dk], v [B,H,T,dv], lambda [B,H,T,L] (weights of
 * levels 0..L-1), out [B,H,T,dv]. L must cover every position: T <= 2^(L-1). Returns 0, or
 * -1 on a bad argument.
 */
int oracle_loglinear_scan(const double* q, const double* k, const double* v, const double* lam,
                          double* out, int B, int H, int T, int dk, int dv, int L) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || L < 1 || L > 40) return -1;
    if (T > 1 && (long)(T - 1) >> (L - 1)) return -1;
    if (!q || !k || !v || !lam || !out) return -1;
    const long BH = (long)B * H;
    const long state = (long)dv * dk;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double* M = (double*)malloc(sizeof(double) * (size_t)state * (size_t)(L > 1 ? L - 1 : 1));
        double* cur = (double*)malloc(sizeof(double) * (size_t)state);
        if (!M || !cur) {
            failed = 1;
        } else {
            loglinear_sequence(q + bh * (long)T * dk, k + bh * (long)T * dk,
                               v + bh * (long)T * dv, lam + bh * (long)T * L,
                               M, cur, out + bh * (long)T * dv, T, dk, dv, L);
        }
        free(M);
        free(cur);
    }
    return failed ? -1 : 0;
}
