/*
 * sf_oracle.c -- plain fp64 CPU oracle for the chunkwise linear-recurrence layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes (token by token, no chunking, no blocking, no reordering):
 *
 *   The layer is the linear recurrence with a d_k x d_v matrix state that the
 *   StateFlow pages build on ("StateFlow: Sequence Pipeline Parallelism for
 *   Long-Context Modeling with Linear Recurrence", Abstract: linear attention
 *   and state-space models, boundary states carried across chunks) and that the
 *   Sequence Accumulation page calls the accumulated d x d memory state
 *   ("Sequence Accumulation and Beyond: Infinite Context Length on Single GPU
 *   and Large Clusters", Approach).  The evaluated architecture is Gated
 *   DeltaNet (gptget.net StateFlow summary, section 实验设计), whose update is
 *   the gated delta rule:
 *
 *       S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,   o_t = S_t^T q_t
 *
 *   with a_t = exp(g_t) (g is a log-decay).  Variants, selected by NULL
 *   pointers:
 *       g == NULL     -> a_t = 1 (no decay)
 *       beta == NULL  -> plain (gated) linear attention S_t = a_t S_{t-1} + k_t v_t^T
 *   The output uses the state after the update of token t (inclusive).
 *
 *   The backward pass is the reverse-mode derivative of that token loop,
 *   derived by hand (one step at a time, see oracle_bwd_head), of any loss
 *   L(o, S_out) given dO = dL/do and dS_out = dL/dS_out.  The gradient with
 *   respect to S_in is returned too, which is the boundary-gradient hand-off
 *   between sub-sequences (StateFlow Abstract: "propagating boundary states and
 *   gradients across chunks"; Sequence Accumulation, Approach: backward pass
 *   over stored states).
 *
 * Layouts (all double, C order):
 *   q, k: [B, T, H, dk]   v, o: [B, T, H, dv]   g, beta: [B, T, H]
 *   S_in, S_out, dS_*: [B, H, dk, dv]
 *
 * Parallelism: OpenMP over the independent (b, h) pairs only; each (b, h) is a
 * plain sequential loop over t.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, T, H, dk, dv;
} dims_t;

static size_t tok_idx(const dims_t* d, int b, int t, int h) {
    return ((size_t)b * d->T + t) * d->H + h;
}

/* One token step of the forward recurrence, in place on S (dk x dv). */
static void step_fwd(const dims_t* d, double* S, const double* kt, const double* vt,
                     double a, int has_beta, double bt, double* y) {
    const int dk = d->dk, dv = d->dv;
    if (has_beta) {
        /* y = S^T k  (the value the state currently returns for key k) */
        for (int j = 0; j < dv; ++j) y[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) y[j] += S[i * dv + j] * kt[i];
        /* S <- a (S - b k y^T) + b k v^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[i * dv + j] = a * (S[i * dv + j] - bt * kt[i] * y[j]) + bt * kt[i] * vt[j];
    } else {
        /* S <- a S + k v^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] = a * S[i * dv + j] + kt[i] * vt[j];
    }
}

static void oracle_fwd_head(const dims_t* d, int b, int h, const double* q, const double* k,
                            const double* v, const double* g, const double* beta,
                            const double* S_in, double* o, double* S_out) {
    const int dk = d->dk, dv = d->dv;
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* y = (double*)malloc(sizeof(double) * (size_t)dv);
    const size_t s_off = ((size_t)b * d->H + h) * dk * dv;
    if (S_in)
        memcpy(S, S_in + s_off, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);
    for (int t = 0; t < d->T; ++t) {
        const size_t ti = tok_idx(d, b, t, h);
        const double* kt = k + ti * dk;
        const double* vt = v + ti * dv;
        const double* qt = q + ti * dk;
        const double a = g ? exp(g[ti]) : 1.0;
        step_fwd(d, S, kt, vt, a, beta != NULL, beta ? beta[ti] : 0.0, y);
        double* ot = o + ti * dv;
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qt[i];
    }
    if (S_out) memcpy(S_out + s_off, S, sizeof(double) * (size_t)dk * dv);
    free(S);
    free(y);
}

/*
 * Backward for one (b, h).  dS holds dL/dS_t for the state after token t while
 * walking t from T-1 down to 0.  Per token (state before = P, after = S_t):
 *
 *   o_t = S_t^T q_t          : dq_t = S_t do_t ;  dS += q_t do_t^T
 *   delta rule, y = P^T k, X = P - b k y^T, S_t = a X + b k v^T:
 *       dv_t = b dS^T k ;  db = k^T dS v ;  dk_t = b dS v
 *       da = <dS, X> ;  dX = a dS ;  z = dX^T k
 *       dk_t += -b (dX y + P z) ;  db += -y^T z ;  dP = dX - b k z^T
 *   linear attention, S_t = a P + k v^T:
 *       dv_t = dS^T k ;  dk_t = dS v ;  da = <dS, P> ;  dP = a dS
 *   a = exp(g): dg_t = a da
 *
 * States before each token are recomputed segment by segment from checkpoints
 * taken every `seg` tokens during a first forward sweep, so host memory stays
 * O(T/seg + seg) states per (b, h).
 */
static void oracle_bwd_head(const dims_t* d, int b, int h, int seg, const double* q,
                            const double* k, const double* v, const double* g,
                            const double* beta, const double* S_in, const double* dO,
                            const double* dS_out, double* dq, double* dk_out, double* dv_out,
                            double* dg, double* dbeta, double* dS_in) {
    const int dk = d->dk, dv = d->dv, T = d->T;
    const size_t SS = (size_t)dk * dv;
    const int nseg = (T + seg - 1) / seg;
    const size_t s_off = ((size_t)b * d->H + h) * SS;
    double* ckpt = (double*)malloc(sizeof(double) * SS * (size_t)(nseg > 0 ? nseg : 1));
    double* states = (double*)malloc(sizeof(double) * SS * (size_t)(seg + 1));
    double* dS = (double*)malloc(sizeof(double) * SS);
    double* dX = (double*)malloc(sizeof(double) * SS);
    double* y = (double*)malloc(sizeof(double) * (size_t)dv);
    double* z = (double*)malloc(sizeof(double) * (size_t)dv);
    double* S = states; /* scratch for the checkpoint sweep */

    /* Sweep 1: forward, storing the state before the first token of each segment. */
    if (S_in)
        memcpy(S, S_in + s_off, sizeof(double) * SS);
    else
        memset(S, 0, sizeof(double) * SS);
    for (int t = 0; t < T; ++t) {
        if (t % seg == 0) memcpy(ckpt + (size_t)(t / seg) * SS, S, sizeof(double) * SS);
        const size_t ti = tok_idx(d, b, t, h);
        step_fwd(d, S, k + ti * dk, v + ti * dv, g ? exp(g[ti]) : 1.0, beta != NULL,
                 beta ? beta[ti] : 0.0, y);
    }

    if (dS_out)
        memcpy(dS, dS_out + s_off, sizeof(double) * SS);
    else
        memset(dS, 0, sizeof(double) * SS);

    for (int sgi = nseg - 1; sgi >= 0; --sgi) {
        const int t0 = sgi * seg;
        const int t1 = (t0 + seg < T) ? t0 + seg : T;
        /* Recompute states[i] = state before token t0 + i, states[t1 - t0] = after. */
        memcpy(states, ckpt + (size_t)sgi * SS, sizeof(double) * SS);
        for (int t = t0; t < t1; ++t) {
            const size_t ti = tok_idx(d, b, t, h);
            double* nxt = states + (size_t)(t - t0 + 1) * SS;
            memcpy(nxt, states + (size_t)(t - t0) * SS, sizeof(double) * SS);
            step_fwd(d, nxt, k + ti * dk, v + ti * dv, g ? exp(g[ti]) : 1.0, beta != NULL,
                     beta ? beta[ti] : 0.0, y);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const size_t ti = tok_idx(d, b, t, h);
            const double* P = states + (size_t)(t - t0) * SS;      /* S_{t-1} */
            const double* St = states + (size_t)(t - t0 + 1) * SS; /* S_t */
            const double* qt = q + ti * dk;
            const double* kt = k + ti * dk;
            const double* vt = v + ti * dv;
            const double* dot = dO + ti * dv;
            double* dqt = dq + ti * dk;
            double* dkt = dk_out + ti * dk;
            double* dvt = dv_out + ti * dv;
            const double a = g ? exp(g[ti]) : 1.0;

            /* output read-out */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += St[i * dv + j] * dot[j];
                dqt[i] = acc;
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) dS[i * dv + j] += qt[i] * dot[j];

            double da = 0.0;
            if (beta) {
                const double bt = beta[ti];
                double db = 0.0;
                /* y = P^T k and dv_t = b dS^T k, accumulated row by row */
                for (int j = 0; j < dv; ++j) y[j] = 0.0, dvt[j] = 0.0;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        y[j] += P[i * dv + j] * kt[i];
                        dvt[j] += dS[i * dv + j] * kt[i];
                    }
                for (int j = 0; j < dv; ++j) dvt[j] *= bt;
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dS[i * dv + j] * vt[j];
                    dkt[i] = bt * acc;
                    db += kt[i] * acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        const double X = P[i * dv + j] - bt * kt[i] * y[j];
                        da += dS[i * dv + j] * X;
                        dX[i * dv + j] = a * dS[i * dv + j];
                    }
                /* z = dX^T k */
                for (int j = 0; j < dv; ++j) z[j] = 0.0;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) z[j] += dX[i * dv + j] * kt[i];
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dX[i * dv + j] * y[j] + P[i * dv + j] * z[j];
                    dkt[i] += -bt * acc;
                }
                for (int j = 0; j < dv; ++j) db -= y[j] * z[j];
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) dS[i * dv + j] = dX[i * dv + j] - bt * kt[i] * z[j];
                dbeta[ti] = db;
            } else {
                /* dv_t = dS^T k */
                for (int j = 0; j < dv; ++j) dvt[j] = 0.0;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) dvt[j] += dS[i * dv + j] * kt[i];
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dS[i * dv + j] * vt[j];
                    dkt[i] = acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        da += dS[i * dv + j] * P[i * dv + j];
                        dS[i * dv + j] *= a;
                    }
            }
            if (g) dg[ti] = a * da;
        }
    }
    if (dS_in) memcpy(dS_in + s_off, dS, sizeof(double) * SS);
    free(ckpt);
    free(states);
    free(dS);
    free(dX);
    free(y);
    free(z);
}

static int check_dims(int B, int T, int H, int dk, int dv) {
    return (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) ? -1 : 0;
}

/* Forward.  Returns 0 on success, -1 on bad sizes. */
int sfo_fwd(int B, int T, int H, int dk, int dv, const double* q, const double* k,
            const double* v, const double* g, const double* beta, const double* S_in, double* o,
            double* S_out, int nthreads) {
    if (check_dims(B, T, H, dk, dv)) return -1;
    dims_t d = {B, T, H, dk, dv};
    const int n = B * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int bh = 0; bh < n; ++bh)
        oracle_fwd_head(&d, bh / H, bh % H, q, k, v, g, beta, S_in, o, S_out);
    return 0;
}

/* Backward.  dS_out may be NULL (zero).  dg must be non-NULL iff g is; dbeta iff beta is. */
int sfo_bwd(int B, int T, int H, int dk, int dv, const double* q, const double* k,
            const double* v, const double* g, const double* beta, const double* S_in,
            const double* dO, const double* dS_out, double* dq, double* dk_out, double* dv_out,
            double* dg, double* dbeta, double* dS_in, int seg, int nthreads) {
    if (check_dims(B, T, H, dk, dv)) return -1;
    if ((g == NULL) != (dg == NULL) || (beta == NULL) != (dbeta == NULL)) return -1;
    if (seg <= 0) seg = 64;
    dims_t d = {B, T, H, dk, dv};
    const int n = B * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int bh = 0; bh < n; ++bh)
        oracle_bwd_head(&d, bh / H, bh % H, seg, q, k, v, g, beta, S_in, dO, dS_out, dq, dk_out,
                        dv_out, dg, dbeta, dS_in);
    return 0;
}

int sfo_max_threads(void) {
#ifdef _OPENMP
    return omp_get_num_procs();
#else
    return 1;
#endif
}
