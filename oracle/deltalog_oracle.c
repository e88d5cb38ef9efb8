/*
 * deltalog_oracle.c -- plain fp64 CPU oracle for DeltaLog recurrent-state decode.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the checker, not the product: only
 * the test suite, the package smoke check and the benchmark's CPU-baseline leg
 * may load it. It shares no code, header, table or helper with the CUDA path.
 *
 * Source: "DeltaLog: Deferred Materialization of Recurrent States for Linear
 * Attention Decoding" (arXiv 2608.15533), as summarised on its gist.science
 * page (technical summary: "Meccanismo Core: Base + Log", "Modello di
 * Traffico", the operator list GDN / KDA / RWKV6) and on its signal-papers
 * page (Fig. 4 caption: append while L < C, materialise into the base when
 * L = C).  The pages do not print the recurrences; the forms below are the
 * plainest standard ones consistent with the operator descriptions:
 *
 *   state per head S in R^{dk x dv}, row i = key channel, column c = value channel
 *
 *   GDN   (scalar decay per head, delta rule)
 *         a = exp(g) (scalar), S' = a S, u = beta (v - S'^T k),
 *         S = S' + k u^T, o = scale S^T q
 *   KDA   (per-key decay, delta rule)
 *         a = exp(g) in (0,1)^dk, S' = D(a) S, then the same delta rule
 *   RWKV6 (per-key decay, raw value update, bonus u)
 *         o = scale (S^T r + (r . (bonus * k)) v)   with the pre-update S,
 *         S = D(exp(g)) S + k v^T
 *
 * Two independent formulations are given:
 *   1. the eager recurrence (the plain definition; ground truth), and
 *   2. the base + bounded log formulation, step by step in the pages' order:
 *      append while L < C (base untouched, compact factors k_t, u_t and the
 *      cumulative log-decay snapshot Lambda_t appended), merge when L = C
 *      (the logical state is materialised back into the base, log reset).
 *      Logical state after t appends:
 *        S_t = D(exp(Lambda_t)) Sbar + sum_{j<=t} D(exp(Lambda_t - Lambda_j)) k_j u_j^T
 *
 * Everything is double precision; no blocking, fusion or reordering beyond
 * the formulas above.  Heads are independent and are spread over threads.
 *
 * Layouts (row-major, all double):
 *   S, base  [nh, dk, dv]      q, k  [T, nh, dk]      v  [T, nh, dv]
 *   beta     [T, nh]           g     [T, nh, m]       (m = 1 GDN, dk otherwise)
 *   bonus    [nh, dk]          out   [T, nh, dv]
 *   logK     [nh, C, dk]       logU  [nh, C, dv]      logLam [nh, C, m]
 */
#include <math.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_GDN = 0, OR_KDA = 1, OR_RWKV6 = 2 };

static int decay_width(int op, int dk) { return op == OR_GDN ? 1 : dk; }

/* decay index for key channel i: the scalar for GDN, channel i otherwise */
static int didx(int op, int i) { return op == OR_GDN ? 0 : i; }

/* ---------------------------------------------------------------- eager -- */

/* One eager decode step for one head, in place on S (dk x dv).
 * u_out (dv, may be NULL) receives the value-side factor written this step:
 * the delta-rule u for GDN/KDA, the raw v for RWKV6. */
static void eager_step_head(int op, int dk, int dv, double scale, double *S,
                            const double *q, const double *k, const double *v,
                            double beta, const double *g, const double *bonus,
                            double *out, double *u_out)
{
    if (op == OR_RWKV6) {
        /* output from the pre-update state plus the bonus term */
        double rb = 0.0;
        for (int i = 0; i < dk; ++i) rb += q[i] * bonus[i] * k[i];
        for (int c = 0; c < dv; ++c) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + c] * q[i];
            out[c] = scale * (acc + rb * v[c]);
        }
        /* S = D(w) S + k v^T */
        for (int i = 0; i < dk; ++i) {
            double w = exp(g[i]);
            for (int c = 0; c < dv; ++c)
                S[(size_t)i * dv + c] = w * S[(size_t)i * dv + c] + k[i] * v[c];
        }
        if (u_out) for (int c = 0; c < dv; ++c) u_out[c] = v[c];
        return;
    }
    /* GDN / KDA: decay, delta rule, readout of the updated state */
    for (int i = 0; i < dk; ++i) {
        double a = exp(g[didx(op, i)]);
        for (int c = 0; c < dv; ++c) S[(size_t)i * dv + c] *= a;
    }
    for (int c = 0; c < dv; ++c) {
        double pred = 0.0;
        for (int i = 0; i < dk; ++i) pred += S[(size_t)i * dv + c] * k[i];
        double u = beta * (v[c] - pred);
        if (u_out) u_out[c] = u;
        for (int i = 0; i < dk; ++i) S[(size_t)i * dv + c] += k[i] * u;
    }
    for (int c = 0; c < dv; ++c) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + c] * q[i];
        out[c] = scale * acc;
    }
}

/* T eager steps over nh heads.  u_trace [T, nh, dv] may be NULL. */
int oracle_eager_run(int op, int nh, int dk, int dv, int T, double scale,
                     double *S, const double *q, const double *k, const double *v,
                     const double *beta, const double *g, const double *bonus,
                     double *out, double *u_trace, int n_threads)
{
    if (op < 0 || op > 2 || nh < 0 || dk <= 0 || dv <= 0 || T < 0) return 1;
    const int m = decay_width(op, dk);
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h) {
        double *Sh = S + (size_t)h * dk * dv;
        for (int t = 0; t < T; ++t) {
            size_t th = (size_t)t * nh + h;
            eager_step_head(op, dk, dv, scale, Sh, q + th * dk, k + th * dk,
                            v + th * dv, beta ? beta[th] : 0.0, g + th * m,
                            bonus ? bonus + (size_t)h * dk : NULL,
                            out + th * dv, u_trace ? u_trace + th * dv : NULL);
        }
    }
    return 0;
}

/* ------------------------------------------------------------ base + log -- */

/* Append phase for one head (log holds L < C entries): read-out of the
 * logical state from the untouched base plus the replayed log, then append
 * (k_t, u_t, Lambda_t) at slot L. */
static void append_step_head(int op, int dk, int dv, int C, double scale,
                             const double *base, double *K, double *U, double *Lam,
                             int L, const double *q, const double *k, const double *v,
                             double beta, const double *g, const double *bonus,
                             double *out)
{
    const int m = decay_width(op, dk);
    (void)C;
    /* cumulative log-decay snapshot: previous entry's (0 right after a merge) */
    double lam_prev[1024], lam_t[1024];
    for (int x = 0; x < m; ++x) {
        lam_prev[x] = L > 0 ? Lam[(size_t)(L - 1) * m + x] : 0.0;
        lam_t[x] = lam_prev[x] + g[x];
    }

    if (op == OR_RWKV6) {
        /* output reads the logical state before this step's update:
         * S_{t-1}^T r = Sbar^T (Gamma_{t-1} * r) + sum_j d_j v_j */
        double d[64];
        for (int j = 0; j < L; ++j) {
            double s = 0.0;
            for (int i = 0; i < dk; ++i)
                s += q[i] * K[(size_t)j * dk + i] * exp(lam_prev[i] - Lam[(size_t)j * m + i]);
            d[j] = s;
        }
        double rb = 0.0;
        for (int i = 0; i < dk; ++i) rb += q[i] * bonus[i] * k[i];
        for (int c = 0; c < dv; ++c) {
            double xr = 0.0;
            for (int i = 0; i < dk; ++i)
                xr += base[(size_t)i * dv + c] * exp(lam_prev[i]) * q[i];
            double rr = 0.0;
            for (int j = 0; j < L; ++j) rr += d[j] * U[(size_t)j * dv + c];
            out[c] = scale * (xr + rr + rb * v[c]);
        }
        for (int i = 0; i < dk; ++i) K[(size_t)L * dk + i] = k[i];
        for (int c = 0; c < dv; ++c) U[(size_t)L * dv + c] = v[c];
        for (int x = 0; x < m; ++x) Lam[(size_t)L * m + x] = lam_t[x];
        return;
    }

    /* GDN / KDA.  ReplayPrep: key-side replay coefficients against the
     * current token, c_j for the key and d_j for the query. */
    double cj[64], dj[64];
    for (int j = 0; j < L; ++j) {
        double sc = 0.0, sd = 0.0;
        for (int i = 0; i < dk; ++i) {
            int x = didx(op, i);
            double e = exp(lam_t[x] - Lam[(size_t)j * m + x]) * K[(size_t)j * dk + i];
            sc += k[i] * e;
            sd += q[i] * e;
        }
        cj[j] = sc;
        dj[j] = sd;
    }
    double kq = 0.0;
    for (int i = 0; i < dk; ++i) kq += k[i] * q[i];
    double u[1024];
    for (int c = 0; c < dv; ++c) {
        /* base read-out through the decay since the last merge */
        double xk = 0.0, xq = 0.0;
        for (int i = 0; i < dk; ++i) {
            double gam = exp(lam_t[didx(op, i)]);
            xk += base[(size_t)i * dv + c] * gam * k[i];
            xq += base[(size_t)i * dv + c] * gam * q[i];
        }
        /* value-side log replay */
        double rk = 0.0, rq = 0.0;
        for (int j = 0; j < L; ++j) {
            rk += cj[j] * U[(size_t)j * dv + c];
            rq += dj[j] * U[(size_t)j * dv + c];
        }
        u[c] = beta * (v[c] - xk - rk);
        out[c] = scale * (xq + rq + kq * u[c]);
    }
    for (int i = 0; i < dk; ++i) K[(size_t)L * dk + i] = k[i];
    for (int c = 0; c < dv; ++c) U[(size_t)L * dv + c] = u[c];
    for (int x = 0; x < m; ++x) Lam[(size_t)L * m + x] = lam_t[x];
}

/* Materialise the logical state of one head (base + L log entries) into dst.
 * dst may alias base (that is the merge). */
static void materialize_head(int op, int dk, int dv, const double *base,
                             const double *K, const double *U, const double *Lam,
                             int L, double *dst)
{
    const int m = decay_width(op, dk);
    for (int i = 0; i < dk; ++i) {
        int x = didx(op, i);
        double lamL = L > 0 ? Lam[(size_t)(L - 1) * m + x] : 0.0;
        double gam = exp(lamL);
        double coef[64];
        for (int j = 0; j < L; ++j)
            coef[j] = exp(lamL - Lam[(size_t)j * m + x]) * K[(size_t)j * dk + i];
        for (int c = 0; c < dv; ++c) {
            double s = gam * base[(size_t)i * dv + c];
            for (int j = 0; j < L; ++j) s += coef[j] * U[(size_t)j * dv + c];
            dst[(size_t)i * dv + c] = s;
        }
    }
}

/* Base+log decode of T tokens over nh heads with log capacity C.
 * *L_io is the log length shared by all heads on entry and on exit.
 * L_trace[t] = log length after token t, merged[t] = 1 when a merge ran
 * after token t (either may be NULL).  Returns 0, or 1 on bad arguments. */
int oracle_deltalog_run(int op, int nh, int dk, int dv, int C, int T, double scale,
                        double *base, double *K, double *U, double *Lam, int *L_io,
                        const double *q, const double *k, const double *v,
                        const double *beta, const double *g, const double *bonus,
                        double *out, int *L_trace, int *merged, int n_threads)
{
    if (op < 0 || op > 2 || nh < 0 || dk <= 0 || dv <= 0 || T < 0) return 1;
    if (C < 1 || C > 64 || dk > 1024 || dv > 1024) return 1;
    if (*L_io < 0 || *L_io >= C) return 1;
    const int m = decay_width(op, dk);
    const int L0 = *L_io;
    /* the schedule (append, then merge when the log is full) is the same for
     * every head and does not depend on the data */
    int Ls = L0;
    for (int t = 0; t < T; ++t) {
        Ls += 1;
        int dm = 0;
        if (Ls == C) { Ls = 0; dm = 1; }
        if (L_trace) L_trace[t] = Ls;
        if (merged) merged[t] = dm;
    }
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h) {
        double *bh = base + (size_t)h * dk * dv;
        double *Kh = K + (size_t)h * C * dk;
        double *Uh = U + (size_t)h * C * dv;
        double *Lh = Lam + (size_t)h * C * m;
        int L = L0;
        for (int t = 0; t < T; ++t) {
            size_t th = (size_t)t * nh + h;
            append_step_head(op, dk, dv, C, scale, bh, Kh, Uh, Lh, L,
                             q + th * dk, k + th * dk, v + th * dv,
                             beta ? beta[th] : 0.0, g + th * m,
                             bonus ? bonus + (size_t)h * dk : NULL, out + th * dv);
            L += 1;
            if (L == C) {               /* merge phase: fold the log into the base */
                materialize_head(op, dk, dv, bh, Kh, Uh, Lh, L, bh);
                L = 0;
            }
        }
    }
    *L_io = Ls;
    return 0;
}

/* Base+log decode with a log length per slot (continuous batching: slots
 * join, leave and idle independently, so their logs fill at different
 * tokens).  Heads are grouped by slot, head = s * H + h for slot s < nslots.
 * Slot s takes part in token t only when active[t * nslots + s] is nonzero:
 * then each of its heads appends at the slot's own log length, and the slot
 * merges when its log is full; an idle slot's heads, log and output rows are
 * left untouched.  Ls[s] is slot s's log length on entry and on exit;
 * L_trace[t * nslots + s] = slot s's length after token t (may be NULL).
 * Returns 0, or 1 on bad arguments. */
int oracle_deltalog_slots_run(int op, int nslots, int H, int dk, int dv, int C, int T,
                              double scale, double *base, double *K, double *U, double *Lam,
                              int *Ls, const unsigned char *active,
                              const double *q, const double *k, const double *v,
                              const double *beta, const double *g, const double *bonus,
                              double *out, int *L_trace, int n_threads)
{
    if (op < 0 || op > 2 || nslots < 0 || H < 1 || dk <= 0 || dv <= 0 || T < 0) return 1;
    if (C < 1 || C > 64 || dk > 1024 || dv > 1024) return 1;
    for (int s = 0; s < nslots; ++s)
        if (Ls[s] < 0 || Ls[s] >= C) return 1;
    const int m = decay_width(op, dk);
    const int nh = nslots * H;
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1)
    for (int hh = 0; hh < nh; ++hh) {
        const int s = hh / H;
        double *bh = base + (size_t)hh * dk * dv;
        double *Kh = K + (size_t)hh * C * dk;
        double *Uh = U + (size_t)hh * C * dv;
        double *Lh = Lam + (size_t)hh * C * m;
        int L = Ls[s];
        for (int t = 0; t < T; ++t) {
            if (!active[(size_t)t * nslots + s]) continue;
            size_t th = (size_t)t * nh + hh;
            append_step_head(op, dk, dv, C, scale, bh, Kh, Uh, Lh, L,
                             q + th * dk, k + th * dk, v + th * dv,
                             beta ? beta[th] : 0.0, g + th * m,
                             bonus ? bonus + (size_t)hh * dk : NULL, out + th * dv);
            L += 1;
            if (L == C) {
                materialize_head(op, dk, dv, bh, Kh, Uh, Lh, L, bh);
                L = 0;
            }
        }
    }
    /* the per-slot schedule depends only on the activity pattern */
    for (int s = 0; s < nslots; ++s) {
        int L = Ls[s];
        for (int t = 0; t < T; ++t) {
            if (active[(size_t)t * nslots + s]) {
                L += 1;
                if (L == C) L = 0;
            }
            if (L_trace) L_trace[(size_t)t * nslots + s] = L;
        }
        Ls[s] = L;
    }
    return 0;
}

/* Out-of-place materialisation of nh heads with log length L. */
int oracle_materialize(int op, int nh, int dk, int dv, int C, int L,
                       const double *base, const double *K, const double *U,
                       const double *Lam, double *S_out)
{
    if (op < 0 || op > 2 || L < 0 || L > C || dk > 1024 || C > 64) return 1;
    const int m = decay_width(op, dk);
    for (int h = 0; h < nh; ++h)
        materialize_head(op, dk, dv, base + (size_t)h * dk * dv,
                         K + (size_t)h * C * dk, U + (size_t)h * C * dv,
                         Lam + (size_t)h * C * m, L, S_out + (size_t)h * dk * dv);
    return 0;
}

/* In-place merge of nh heads with log length L (L = 0 leaves the base as is). */
int oracle_merge(int op, int nh, int dk, int dv, int C, int L, double *base,
                 const double *K, const double *U, const double *Lam)
{
    if (L == 0) return 0;
    return oracle_materialize(op, nh, dk, dv, C, L, base, K, U, Lam, base);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
