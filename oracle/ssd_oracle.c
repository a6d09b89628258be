/*
 * ssd_oracle.c -- plain, slow, fp64 CPU oracle for the chunked SSD forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What is computed (all in double precision, libm exp):
 *
 *   y_t = sum_{s<=t} C_t^T B_s * exp(sum_{k=s+1..t} a_k) * x_s + D * x_t
 *
 * equivalently the state recurrence
 *
 *   h_t = exp(a_t) * h_{t-1} + B_t x_t^T,   h_{-1} = 0,   y_t = C_t^T h_t + D x_t,
 *
 * per (batch b, head h), with B/C taken from group g = h / (H/G).
 * Sources:
 *  - "State Space Models and Mamba ..." (llms.blog), section "The SSD
 *    Theoretical Equivalence": the 1-semiseparable matrix M_{i,j} =
 *    C_i^T (prod_{k=j+1..i} a_k) B_j for i >= j, and the state-space view
 *    h_t = a_t h_{t-1} + K_t^T V_t, y_t = Q_t h_t.  The decays a_k there are
 *    multiplicative; here a holds log-decays, so prod a_k -> exp(sum a_k).
 *  - same page, "Continuous-to-Discrete Discretization": the skip term D x_t.
 *  - "State Space Duality" (aiwiki), section "Two algorithms for one
 *    operator": the chunked evaluation (quadratic form inside a chunk,
 *    summarised state between chunks), with log-space cumulative decay.
 *  - "On Structured State-Space Duality" (ICML 2026 poster abstract), item
 *    (i): the diagonal generalisation -- one log-decay per state index n.
 *
 * Three independent routes:
 *   O1 oracle_recurrence : the step recurrence (primary oracle).
 *   O2 oracle_brute      : materialise M[t][s] with the decay exponent summed
 *                          directly (no cumsum difference); tiny T only.
 *   O3 oracle_chunked    : the chunked algorithm written step by step
 *                          (chunk cumsum, chunk states, state pass, output),
 *                          exposing every intermediate.
 *
 * Layouts (row-major, all double):
 *   x[B][T][H][P]; a[B][T][H] (scalar) or a[B][T][H][N] (per-state);
 *   Bm, Cm[B][T][G][N]; D[H] (NULL means 0).
 * Outputs are per listed chain c = (b, h):
 *   y[c][T][P], final[c][N][P], bounds[c][nc][N][P] (state after each chunk).
 *
 * A planted-mistake switch (oracle_set_mutation) exists so that the tests can
 * show that the oracle's pins catch plausible errors; it is 0 (off) unless a
 * test sets it.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, H, P, G, N, chunk, a_per_state;
} oracle_shape;

/* Planted mistakes, applied consistently to every route that has the
 * concept (so route-vs-route comparisons alone cannot catch them). */
enum {
    MUT_NONE = 0,
    MUT_DROP_D = 1,          /* skip term forgotten                           */
    MUT_DECAY_INCLUSIVE = 2, /* decay from s to t also applies a_s            */
    MUT_SWAP_BC = 3,         /* B and C roles exchanged                       */
    MUT_GROUP_MOD = 4,       /* head->group as h % G instead of h / (H/G)     */
    MUT_SIGN_A = 5,          /* exp(-a) instead of exp(a)                     */
    MUT_NO_INTER_DECAY = 6,  /* O3: inter-chunk output term lacks exp(cum_t)  */
    MUT_STATE_NO_WEIGHT = 7, /* O3: chunk state lacks the within-chunk decay  */
    MUT_DIAG_SHIFT_N = 8,    /* per-state decay read from index n+1 (mod N)   */
    MUT_Y_BEFORE_UPDATE = 9  /* output taken from h_{t-1} instead of h_t      */
};
static int g_mutation = 0;

void oracle_set_mutation(int m) { g_mutation = m; }
int oracle_get_mutation(void) { return g_mutation; }

static int group_of(const oracle_shape* s, int h) {
    if (g_mutation == MUT_GROUP_MOD) return h % s->G;
    return h / (s->H / s->G);
}

/* log-decay for (b, t, h, n) */
static double logdecay(const oracle_shape* s, const double* a, int b, int t, int h, int n) {
    double v;
    if (s->a_per_state) {
        int nn = n;
        if (g_mutation == MUT_DIAG_SHIFT_N) nn = (n + 1) % s->N;
        v = a[(((size_t)b * s->T + t) * s->H + h) * s->N + nn];
    } else {
        v = a[((size_t)b * s->T + t) * s->H + h];
    }
    if (g_mutation == MUT_SIGN_A) v = -v;
    return v;
}

static const double* Bptr(const oracle_shape* s, const double* Bm, const double* Cm,
                          int b, int t, int g) {
    const double* base = (g_mutation == MUT_SWAP_BC) ? Cm : Bm;
    return base + (((size_t)b * s->T + t) * s->G + g) * s->N;
}
static const double* Cptr(const oracle_shape* s, const double* Bm, const double* Cm,
                          int b, int t, int g) {
    const double* base = (g_mutation == MUT_SWAP_BC) ? Bm : Cm;
    return base + (((size_t)b * s->T + t) * s->G + g) * s->N;
}
static const double* Xptr(const oracle_shape* s, const double* x, int b, int t, int h) {
    return x + (((size_t)b * s->T + t) * s->H + h) * s->P;
}
static double Dval(const double* D, int h) {
    if (!D || g_mutation == MUT_DROP_D) return 0.0;
    return D[h];
}

/* ---------------------------------------------------------------- O1 ---- */
/* One chain of the step recurrence.  h_t = exp(a_t) h_{t-1} + B_t x_t^T;
 * y_t = C_t^T h_t + D x_t.  (llms.blog, "The SSD Theoretical Equivalence",
 * state space view; "Continuous-to-Discrete Discretization", D x_t.) */
static void recurrence_chain(const oracle_shape* s, const double* x, const double* a,
                             const double* Bm, const double* Cm, const double* D,
                             const double* init, int b, int h, int t_end, double* y,
                             double* fin, double* bounds) {
    const int N = s->N, P = s->P, Q = s->chunk;
    const int g = group_of(s, h);
    double* st = (double*)calloc((size_t)N * P, sizeof(double));
    /* h_{-1}: zero, or the given state of this (b, h) chain (resuming a
     * sequence from the state a previous call ended with) */
    if (init) memcpy(st, init + ((size_t)b * s->H + h) * N * P, (size_t)N * P * sizeof(double));
    double* e = (double*)malloc((size_t)N * sizeof(double));
    double* prev = (double*)malloc((size_t)N * P * sizeof(double));
    const double dh = Dval(D, h);
    for (int t = 0; t < t_end; ++t) {
        const double* Bt = Bptr(s, Bm, Cm, b, t, g);
        const double* Ct = Cptr(s, Bm, Cm, b, t, g);
        const double* xt = Xptr(s, x, b, t, h);
        for (int n = 0; n < N; ++n) e[n] = exp(logdecay(s, a, b, t, h, n));
        if (g_mutation == MUT_Y_BEFORE_UPDATE) memcpy(prev, st, (size_t)N * P * sizeof(double));
        for (int n = 0; n < N; ++n) {
            for (int p = 0; p < P; ++p) {
                double inp = Bt[n] * xt[p];
                if (g_mutation == MUT_DECAY_INCLUSIVE)
                    st[(size_t)n * P + p] = e[n] * (st[(size_t)n * P + p] + inp);
                else
                    st[(size_t)n * P + p] = e[n] * st[(size_t)n * P + p] + inp;
            }
        }
        const double* hs = (g_mutation == MUT_Y_BEFORE_UPDATE) ? prev : st;
        if (y) {
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) acc += Ct[n] * hs[(size_t)n * P + p];
                y[(size_t)t * P + p] = acc + dh * xt[p];
            }
        }
        if (bounds && Q > 0 && (t + 1) % Q == 0) {
            memcpy(bounds + (size_t)((t + 1) / Q - 1) * N * P, st, (size_t)N * P * sizeof(double));
        }
    }
    if (fin) memcpy(fin, st, (size_t)N * P * sizeof(double));
    free(st);
    free(e);
    free(prev);
}

/* ---------------------------------------------------------------- O2 ---- */
/* Materialise M[t][s] = sum_n C_t[n] B_s[n] exp(sum_{k=s+1..t} a_k[n]) (the
 * 1-semiseparable matrix of llms.blog "The SSD Theoretical Equivalence"),
 * summing the exponent term by term; y = M x + D x.  final state =
 * sum_s exp(sum_{k=s+1..T-1} a_k) B_s x_s^T.  O(T^3 N): tiny inputs only. */
static void brute_chain(const oracle_shape* s, const double* x, const double* a,
                        const double* Bm, const double* Cm, const double* D, int b,
                        int h, double* y, double* fin) {
    const int T = s->T, N = s->N, P = s->P;
    const int g = group_of(s, h);
    const double dh = Dval(D, h);
    const int k0_off = (g_mutation == MUT_DECAY_INCLUSIVE) ? 0 : 1;
    if (y) {
        for (int t = 0; t < T; ++t) {
            const double* Ct = Cptr(s, Bm, Cm, b, t, g);
            const double* xt = Xptr(s, x, b, t, h);
            for (int p = 0; p < P; ++p) y[(size_t)t * P + p] = dh * xt[p];
            int s_hi = (g_mutation == MUT_Y_BEFORE_UPDATE) ? t - 1 : t;
            for (int sidx = 0; sidx <= s_hi; ++sidx) {
                const double* Bs = Bptr(s, Bm, Cm, b, sidx, g);
                const double* xs = Xptr(s, x, b, sidx, h);
                double m = 0.0;
                for (int n = 0; n < N; ++n) {
                    double ex = 0.0;
                    /* with the output taken before the update, the decay
                     * runs to t-1 */
                    int k_hi = (g_mutation == MUT_Y_BEFORE_UPDATE) ? t - 1 : t;
                    for (int k = sidx + k0_off; k <= k_hi; ++k) ex += logdecay(s, a, b, k, h, n);
                    m += Ct[n] * Bs[n] * exp(ex);
                }
                for (int p = 0; p < P; ++p) y[(size_t)t * P + p] += m * xs[p];
            }
        }
    }
    if (fin) {
        memset(fin, 0, (size_t)N * P * sizeof(double));
        for (int sidx = 0; sidx < T; ++sidx) {
            const double* Bs = Bptr(s, Bm, Cm, b, sidx, g);
            const double* xs = Xptr(s, x, b, sidx, h);
            for (int n = 0; n < N; ++n) {
                double ex = 0.0;
                for (int k = sidx + k0_off; k <= T - 1; ++k) ex += logdecay(s, a, b, k, h, n);
                double w = Bs[n] * exp(ex);
                for (int p = 0; p < P; ++p) fin[(size_t)n * P + p] += w * xs[p];
            }
        }
    }
}

/* ---------------------------------------------------------------- O3 ---- */
/* The chunked algorithm ("State Space Duality", "Two algorithms for one
 * operator"; llms.blog "The Chunk-Wise SSD Algorithm"), step by step, with the
 * two readings the pages leave open fixed as follows: the inter-chunk output
 * term carries exp(cum_t) (decay from the chunk start to t), and the chunk
 * state weights each token by its decay to the chunk end.
 *   S1 cum[k][j][n]  = sum_{i<=j} a[kQ+i][n]
 *   S2 S_k[n][p]     = sum_j B_{kQ+j}[n] exp(cum[k][Q-1][n] - cum[k][j][n]) x_{kQ+j}[p]
 *   S3 Hin_0 = 0;  Hin_{k+1} = exp(cum[k][Q-1][n]) Hin_k + S_k;  final = Hin_nc
 *   S4 y_{kQ+j} = sum_{i<=j} sum_n C[n] B_i[n] exp(cum_j[n]-cum_i[n]) x_i
 *               + sum_n C[n] exp(cum_j[n]) Hin_k[n][:] + D x
 * cum has N columns only for the per-state variant (else 1).
 * Outputs (any may be NULL): cum[nc][Q][Na], S[nc][N][P], Hin[nc][N][P],
 * y[T][P], fin[N][P]. */
static void chunked_chain(const oracle_shape* s, const double* x, const double* a,
                          const double* Bm, const double* Cm, const double* D, int b,
                          int h, double* cum_o, double* S_o, double* Hin_o, double* y,
                          double* fin) {
    const int T = s->T, N = s->N, P = s->P, Q = s->chunk;
    const int nc = T / Q;
    const int Na = s->a_per_state ? N : 1;
    const int g = group_of(s, h);
    const double dh = Dval(D, h);
    double* cum = (double*)malloc((size_t)nc * Q * Na * sizeof(double));
    double* S = (double*)calloc((size_t)nc * N * P, sizeof(double));
    double* Hin = (double*)calloc((size_t)nc * N * P, sizeof(double));
    double* hcur = (double*)calloc((size_t)N * P, sizeof(double));

    /* S1: inclusive prefix sum restarting at each chunk */
    for (int k = 0; k < nc; ++k)
        for (int na = 0; na < Na; ++na) {
            double run = 0.0;
            for (int j = 0; j < Q; ++j) {
                run += logdecay(s, a, b, k * Q + j, h, na);
                cum[((size_t)k * Q + j) * Na + na] = run;
            }
        }
#define CUM(k, j, n) cum[((size_t)(k) * Q + (j)) * Na + (Na == 1 ? 0 : (n))]

    /* S2: chunk states from a zero start */
    for (int k = 0; k < nc; ++k)
        for (int j = 0; j < Q; ++j) {
            const double* Bs = Bptr(s, Bm, Cm, b, k * Q + j, g);
            const double* xs = Xptr(s, x, b, k * Q + j, h);
            for (int n = 0; n < N; ++n) {
                double w = (g_mutation == MUT_STATE_NO_WEIGHT)
                               ? 1.0
                               : exp(CUM(k, Q - 1, n) - CUM(k, j, n));
                if (g_mutation == MUT_DECAY_INCLUSIVE) w *= exp(logdecay(s, a, b, k * Q + j, h, n));
                for (int p = 0; p < P; ++p) S[((size_t)k * N + n) * P + p] += Bs[n] * w * xs[p];
            }
        }

    /* S3: sequential pass over chunks */
    for (int k = 0; k < nc; ++k) {
        memcpy(Hin + (size_t)k * N * P, hcur, (size_t)N * P * sizeof(double));
        for (int n = 0; n < N; ++n) {
            double e = exp(CUM(k, Q - 1, n));
            for (int p = 0; p < P; ++p)
                hcur[(size_t)n * P + p] = e * hcur[(size_t)n * P + p] + S[((size_t)k * N + n) * P + p];
        }
    }

    /* S4: chunk outputs */
    if (y) {
        for (int k = 0; k < nc; ++k)
            for (int j = 0; j < Q; ++j) {
                const int t = k * Q + j;
                const double* Ct = Cptr(s, Bm, Cm, b, t, g);
                const double* xt = Xptr(s, x, b, t, h);
                double* yt = y + (size_t)t * P;
                for (int p = 0; p < P; ++p) yt[p] = dh * xt[p];
                int i_hi = (g_mutation == MUT_Y_BEFORE_UPDATE) ? j - 1 : j;
                for (int i = 0; i <= i_hi; ++i) {
                    const double* Bi = Bptr(s, Bm, Cm, b, k * Q + i, g);
                    const double* xi = Xptr(s, x, b, k * Q + i, h);
                    double m = 0.0;
                    for (int n = 0; n < N; ++n) {
                        double ex = CUM(k, j, n) - CUM(k, i, n);
                        if (g_mutation == MUT_DECAY_INCLUSIVE) ex += logdecay(s, a, b, k * Q + i, h, n);
                        if (g_mutation == MUT_Y_BEFORE_UPDATE) ex -= logdecay(s, a, b, t, h, n);
                        m += Ct[n] * Bi[n] * exp(ex);
                    }
                    for (int p = 0; p < P; ++p) yt[p] += m * xi[p];
                }
                for (int n = 0; n < N; ++n) {
                    double f = (g_mutation == MUT_NO_INTER_DECAY) ? 1.0 : exp(CUM(k, j, n));
                    if (g_mutation == MUT_Y_BEFORE_UPDATE) f *= exp(-logdecay(s, a, b, t, h, n));
                    double cf = Ct[n] * f;
                    const double* hk = Hin + (size_t)k * N * P + (size_t)n * P;
                    for (int p = 0; p < P; ++p) yt[p] += cf * hk[p];
                }
            }
    }
#undef CUM
    if (cum_o) memcpy(cum_o, cum, (size_t)nc * Q * Na * sizeof(double));
    if (S_o) memcpy(S_o, S, (size_t)nc * N * P * sizeof(double));
    if (Hin_o) memcpy(Hin_o, Hin, (size_t)nc * N * P * sizeof(double));
    if (fin) memcpy(fin, hcur, (size_t)N * P * sizeof(double));
    free(cum);
    free(S);
    free(Hin);
    free(hcur);
}

/* ------------------------------------------------------ thread driver ---- */
typedef struct {
    int route; /* 1 = O1, 2 = O2, 3 = O3 */
    const oracle_shape* s;
    const double *x, *a, *Bm, *Cm, *D;
    const double* init; /* [B][H][N][P] initial states (O1 only), or NULL */
    const int* chains; /* pairs (b, h) */
    int n_chains;
    int t_end;
    double *y, *fin, *bounds, *cum, *S, *Hin;
    int next; /* shared work counter */
    pthread_mutex_t mu;
} job_t;

static void* worker(void* arg) {
    job_t* j = (job_t*)arg;
    const oracle_shape* s = j->s;
    const int nc = s->chunk > 0 ? s->T / s->chunk : 0;
    const size_t NP = (size_t)s->N * s->P;
    const int Na = s->a_per_state ? s->N : 1;
    for (;;) {
        pthread_mutex_lock(&j->mu);
        int c = j->next++;
        pthread_mutex_unlock(&j->mu);
        if (c >= j->n_chains) break;
        int b = j->chains[2 * c], h = j->chains[2 * c + 1];
        double* y = j->y ? j->y + (size_t)c * s->T * s->P : NULL;
        double* fin = j->fin ? j->fin + (size_t)c * NP : NULL;
        if (j->route == 1) {
            double* bd = j->bounds ? j->bounds + (size_t)c * nc * NP : NULL;
            recurrence_chain(s, j->x, j->a, j->Bm, j->Cm, j->D, j->init, b, h, j->t_end, y, fin, bd);
        } else if (j->route == 2) {
            brute_chain(s, j->x, j->a, j->Bm, j->Cm, j->D, b, h, y, fin);
        } else {
            double* cum = j->cum ? j->cum + (size_t)c * nc * s->chunk * Na : NULL;
            double* S = j->S ? j->S + (size_t)c * nc * NP : NULL;
            double* Hin = j->Hin ? j->Hin + (size_t)c * nc * NP : NULL;
            chunked_chain(s, j->x, j->a, j->Bm, j->Cm, j->D, b, h, cum, S, Hin, y, fin);
        }
    }
    return NULL;
}

static int run(job_t* j, int nthreads) {
    if (j->s->H % j->s->G != 0) return -1;
    if (j->route == 3 && (j->s->chunk <= 0 || j->s->T % j->s->chunk != 0)) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > j->n_chains) nthreads = j->n_chains > 0 ? j->n_chains : 1;
    j->next = 0;
    pthread_mutex_init(&j->mu, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, j);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j->mu);
    return 0;
}

/* O1.  t_end <= T: run the recurrence over t in [0, t_end) only (y rows past
 * t_end are left untouched).  bounds needs s->chunk > 0. */
int oracle_recurrence(const oracle_shape* s, const double* x, const double* a,
                      const double* Bm, const double* Cm, const double* D,
                      const int* chains, int n_chains, int t_end, double* y, double* fin,
                      double* bounds, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.route = 1; j.s = s; j.x = x; j.a = a; j.Bm = Bm; j.Cm = Cm; j.D = D;
    j.chains = chains; j.n_chains = n_chains; j.t_end = t_end;
    j.y = y; j.fin = fin; j.bounds = bounds;
    return run(&j, nthreads);
}

/* O1 from given initial states init[B][H][N][P] (NULL: zero). */
int oracle_recurrence_init(const oracle_shape* s, const double* x, const double* a,
                           const double* Bm, const double* Cm, const double* D,
                           const double* init, const int* chains, int n_chains, int t_end,
                           double* y, double* fin, double* bounds, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.route = 1; j.s = s; j.x = x; j.a = a; j.Bm = Bm; j.Cm = Cm; j.D = D; j.init = init;
    j.chains = chains; j.n_chains = n_chains; j.t_end = t_end;
    j.y = y; j.fin = fin; j.bounds = bounds;
    return run(&j, nthreads);
}

int oracle_brute(const oracle_shape* s, const double* x, const double* a, const double* Bm,
                 const double* Cm, const double* D, const int* chains, int n_chains,
                 double* y, double* fin, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.route = 2; j.s = s; j.x = x; j.a = a; j.Bm = Bm; j.Cm = Cm; j.D = D;
    j.chains = chains; j.n_chains = n_chains; j.t_end = s->T;
    j.y = y; j.fin = fin;
    return run(&j, nthreads);
}

int oracle_chunked(const oracle_shape* s, const double* x, const double* a,
                   const double* Bm, const double* Cm, const double* D, const int* chains,
                   int n_chains, double* cum, double* S, double* Hin, double* y,
                   double* fin, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.route = 3; j.s = s; j.x = x; j.a = a; j.Bm = Bm; j.Cm = Cm; j.D = D;
    j.chains = chains; j.n_chains = n_chains; j.t_end = s->T;
    j.cum = cum; j.S = S; j.Hin = Hin; j.y = y; j.fin = fin;
    return run(&j, nthreads);
}
