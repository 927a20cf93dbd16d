/*
 * Oracle: the eager recurrent decode step, in fp64, one (slot, layer, head)
 * trajectory at a time.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline / reference legs load this code.  It shares no code,
 * header, table or constant with the CUDA path.
 *
 * What it computes (DeltaLog paper, "Background": the common decode form
 * S_t = Diag(exp(lambda_t)) S_{t-1} + a_t b_t^T,  o_t = S_t^T q_t, with the
 * per-operator instantiations of its Table 1 as restated in the prose around it):
 *
 *   for t = 1..T
 *     g      = exp(lambda_t)              vector over d_k; one value shared by all
 *                                         coordinates for scalar decay; 1 for none
 *     Shat   = Diag(g) S_{t-1}
 *     b_t    = v_t                                   additive (LA, RetNet, GLA, RWKV6)
 *            = beta_t (v_t - Shat^T k_t)             delta rule on the decayed state
 *            = beta_t (v_t - S_{t-1}^T k_t)          delta rule, undecayed reading
 *     S_t    = Shat + k_t b_t^T                      (a_t = k_t for every operator)
 *     o_t    = S_t^T q_t
 *
 * The delta-rule default uses the decayed state, which makes the common form
 * reproduce the gated delta rule S_t = (I - beta k k^T) Diag(g) S_{t-1} + beta k v^T
 * of GDN and KDA (paper: "Delta-rule models ... construct the value-side factor
 * using the previous state"; the exact equation did not survive extraction).
 * The undecayed reading is kept as a second mode.
 *
 * Plain loops, no blocking, no reordering beyond the definition.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_DECAY_NONE = 0, OR_DECAY_SCALAR = 1, OR_DECAY_DIAG = 2 };
enum { OR_UPDATE_ADD = 0, OR_UPDATE_DELTA = 1, OR_UPDATE_DELTA_UNDECAYED = 2 };

typedef struct {
    int d_k, d_v, steps;
    int decay;      /* OR_DECAY_* */
    int update;     /* OR_UPDATE_* */
    int n_ckpt;     /* number of state checkpoints written per task */
} oracle_dims;

/* One trajectory.  Arrays are row-major:
 *   S0 [d_k][d_v]; q,k [steps][d_k]; v [steps][d_v];
 *   lam [steps][d_k] (diag) | [steps] (scalar) | unused (none); beta [steps];
 *   out [steps][d_v]; S_ckpt [n_ckpt][d_k][d_v], where checkpoint j holds the
 *   state after ckpt_steps[j] steps (0 = the initial state).
 *   work: 2*d_k*d_v + d_k + d_v doubles. */
static void eager_task(const oracle_dims *dm, const double *S0, const double *q,
                       const double *k, const double *v, const double *lam,
                       const double *beta, const int *ckpt_steps, double *out,
                       double *S_ckpt, double *work)
{
    const int dk = dm->d_k, dv = dm->d_v, T = dm->steps;
    double *S = work;                 /* S_{t-1}, then S_t      */
    double *Shat = S + (size_t)dk * dv;
    double *g = Shat + (size_t)dk * dv;
    double *b = g + dk;

    memcpy(S, S0, sizeof(double) * (size_t)dk * dv);
    for (int j = 0; j < dm->n_ckpt; ++j)
        if (ckpt_steps[j] == 0)
            memcpy(S_ckpt + (size_t)j * dk * dv, S, sizeof(double) * (size_t)dk * dv);

    for (int t = 0; t < T; ++t) {
        const double *qt = q + (size_t)t * dk;
        const double *kt = k + (size_t)t * dk;
        const double *vt = v + (size_t)t * dv;

        /* g = exp(lambda_t) */
        for (int r = 0; r < dk; ++r) {
            if (dm->decay == OR_DECAY_NONE)
                g[r] = 1.0;
            else if (dm->decay == OR_DECAY_SCALAR)
                g[r] = exp(lam[t]);
            else
                g[r] = exp(lam[(size_t)t * dk + r]);
        }

        /* Shat = Diag(g) S_{t-1} */
        for (int r = 0; r < dk; ++r)
            for (int c = 0; c < dv; ++c)
                Shat[(size_t)r * dv + c] = g[r] * S[(size_t)r * dv + c];

        /* value-side factor b_t */
        if (dm->update == OR_UPDATE_ADD) {
            for (int c = 0; c < dv; ++c)
                b[c] = vt[c];
        } else {
            const double *P = (dm->update == OR_UPDATE_DELTA) ? Shat : S;
            for (int c = 0; c < dv; ++c) {
                double u = 0.0;                      /* (P^T k_t)[c] */
                for (int r = 0; r < dk; ++r)
                    u += P[(size_t)r * dv + c] * kt[r];
                b[c] = beta[t] * (vt[c] - u);
            }
        }

        /* S_t = Shat + k_t b_t^T */
        for (int r = 0; r < dk; ++r)
            for (int c = 0; c < dv; ++c)
                S[(size_t)r * dv + c] = Shat[(size_t)r * dv + c] + kt[r] * b[c];

        /* o_t = S_t^T q_t */
        for (int c = 0; c < dv; ++c) {
            double o = 0.0;
            for (int r = 0; r < dk; ++r)
                o += S[(size_t)r * dv + c] * qt[r];
            out[(size_t)t * dv + c] = o;
        }

        for (int j = 0; j < dm->n_ckpt; ++j)
            if (ckpt_steps[j] == t + 1)
                memcpy(S_ckpt + (size_t)j * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    }
}

/* n_task independent trajectories, each laid out as in eager_task() with a leading
 * [n_task] dimension.  lam/beta may be NULL when unused.  n_threads <= 0 uses the
 * OpenMP default.  Returns 0, or -1 on bad arguments / allocation failure. */
int oracle_eager_run(const oracle_dims *dm, long n_task, const double *S0,
                     const double *q, const double *k, const double *v,
                     const double *lam, const double *beta, const int *ckpt_steps,
                     double *out, double *S_ckpt, int n_threads)
{
    if (!dm || dm->d_k <= 0 || dm->d_v <= 0 || dm->steps < 0 || n_task < 0 || dm->n_ckpt < 0)
        return -1;
    if (dm->decay < OR_DECAY_NONE || dm->decay > OR_DECAY_DIAG)
        return -1;
    if (dm->update < OR_UPDATE_ADD || dm->update > OR_UPDATE_DELTA_UNDECAYED)
        return -1;
    if (dm->decay != OR_DECAY_NONE && !lam)
        return -1;
    if (dm->update != OR_UPDATE_ADD && !beta)
        return -1;
    if (dm->n_ckpt > 0 && (!S_ckpt || !ckpt_steps))
        return -1;
    const size_t dk = (size_t)dm->d_k, dv = (size_t)dm->d_v, T = (size_t)dm->steps;
    const size_t lam_per_task = dm->decay == OR_DECAY_DIAG ? T * dk : T;
    const size_t work_len = 2 * dk * dv + dk + dv;
    int failed = 0;

#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif

#pragma omp parallel
    {
        double *work = (double *)malloc(sizeof(double) * work_len);
        if (!work) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long i = 0; i < n_task; ++i) {
            if (!work)
                continue;
            eager_task(dm, S0 + (size_t)i * dk * dv, q + (size_t)i * T * dk,
                       k + (size_t)i * T * dk, v + (size_t)i * T * dv,
                       lam ? lam + (size_t)i * lam_per_task : NULL,
                       beta ? beta + (size_t)i * T : NULL, ckpt_steps,
                       out + (size_t)i * T * dv,
                       S_ckpt ? S_ckpt + (size_t)i * dm->n_ckpt * dk * dv : NULL, work);
        }
        free(work);
    }
    return failed ? -1 : 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
