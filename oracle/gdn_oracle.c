/*
 * gdn_oracle.c -- fp64 CPU oracle of the Gated Delta Rule forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code with the CUDA path.
 *
 * What it computes is the token-by-token recurrence of the page
 * "lite_boost.ops.recurrent_gated_delta_rule" (section "algorithm flow", the
 * four update equations: state decay, memory retrieval, delta update, output),
 * with the query scaled as that page's `scale_value` parameter states, and the
 * q/k L2 normalisation of the page "Qwen3Next Samples" (chunk_gated_delta_rule,
 * equation "L2 Normalization", epsilon inside the square root).  The scalar
 * gate is per (token, v-head); the per-key gate gk of the decode page is not
 * part of this operator.
 *
 * For each sequence b (tokens cu[b] .. cu[b+1]-1) and each v-head h, with
 * qk-head hq = h / (Nv / Nqk), in double precision:
 *
 *     S        = initial state of (b, h)  [Dk x Dv], or zero
 *     for each token t:
 *         kh   = k[t,hq] / sqrt(sum(k[t,hq]^2) + eps)
 *         qh   = scale * q[t,hq] / sqrt(sum(q[t,hq]^2) + eps)
 *         S    = exp(g[t,h]) * S                      (state decay)
 *         kv   = S^T kh                               (memory retrieval)
 *         u    = beta[t,h] * (v[t,h] - kv)
 *         S    = S + kh u^T                           (delta update)
 *         o    = S^T qh                               (output, updated state)
 *     final state of (b, h) = S
 *
 * Layouts (all row-major, contiguous):
 *     q, k  [T, Nqk, Dk]      v, out  [T, Nv, Dv]      g, beta  [T, Nv]
 *     state pool [P, Nv, Dk, Dv]   final state [B, Nv, Dk, Dv]
 * The initial state of sequence b is pool[idx[b]] where idx = state_indices,
 * or slot b when state_indices is NULL; no pool means a zero initial state.
 *
 * Element types are passed as tags so that the same loop reads the bf16 bits
 * the GPU reads (converted exactly to double) or arbitrary doubles for the
 * small analytic tests.  Work is split over (sequence, v-head) pairs with
 * POSIX threads; each pair runs the plain loop above on its own.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

static double ld(const void *p, int dtype, int64_t i)
{
    if (dtype == ORC_F64) return ((const double *)p)[i];
    if (dtype == ORC_F32) return (double)((const float *)p)[i];
    /* bf16: the upper 16 bits of an IEEE binary32 */
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *q, *k, *v, *g, *beta, *pool;
    int dt_q, dt_k, dt_v, dt_g, dt_beta, dt_pool;
    const int32_t *cu, *state_indices;
    int32_t B, Nqk, Nv, Dk, Dv, P;
    double scale, eps;
    double *out, *final_state;
    int32_t nout; /* heads in the out / final_state layouts */
    const int32_t *pairs; /* flattened (b, h, slot) triples */
    int64_t npairs;
    int64_t next; /* next pair to take, guarded by lock */
    pthread_mutex_t lock;
} job_t;

static void run_pair(const job_t *J, int32_t b, int32_t h, int32_t hslot, double *S, double *kh,
                     double *qh, double *kv, double *u)
{
    const int32_t Dk = J->Dk, Dv = J->Dv;
    const int32_t G = J->Nv / J->Nqk;
    const int32_t hq = h / G;

    /* initial state */
    if (J->pool) {
        int64_t slot = J->state_indices ? J->state_indices[b] : b;
        int64_t base = (slot * J->Nv + h) * (int64_t)Dk * Dv;
        for (int64_t i = 0; i < (int64_t)Dk * Dv; ++i) S[i] = ld(J->pool, J->dt_pool, base + i);
    } else {
        for (int64_t i = 0; i < (int64_t)Dk * Dv; ++i) S[i] = 0.0;
    }

    for (int64_t t = J->cu[b]; t < J->cu[b + 1]; ++t) {
        const int64_t qk_base = (t * J->Nqk + hq) * Dk;
        const int64_t v_base = (t * J->Nv + h) * Dv;
        const int64_t o_base = (t * J->nout + hslot) * Dv;
        const int64_t gh = t * J->Nv + h;

        double ssk = 0.0, ssq = 0.0;
        for (int32_t d = 0; d < Dk; ++d) {
            double kd = ld(J->k, J->dt_k, qk_base + d);
            double qd = ld(J->q, J->dt_q, qk_base + d);
            ssk += kd * kd;
            ssq += qd * qd;
        }
        const double kden = sqrt(ssk + J->eps);
        const double qden = sqrt(ssq + J->eps);
        for (int32_t d = 0; d < Dk; ++d) {
            kh[d] = ld(J->k, J->dt_k, qk_base + d) / kden;
            qh[d] = J->scale * (ld(J->q, J->dt_q, qk_base + d) / qden);
        }

        /* state decay */
        const double decay = exp(ld(J->g, J->dt_g, gh));
        for (int64_t i = 0; i < (int64_t)Dk * Dv; ++i) S[i] = decay * S[i];

        /* memory retrieval kv = S^T kh */
        for (int32_t j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int32_t d = 0; d < Dk; ++d) acc += S[(int64_t)d * Dv + j] * kh[d];
            kv[j] = acc;
        }

        /* delta update S += kh u^T with u = beta (v - kv) */
        const double bt = ld(J->beta, J->dt_beta, gh);
        for (int32_t j = 0; j < Dv; ++j) u[j] = bt * (ld(J->v, J->dt_v, v_base + j) - kv[j]);
        for (int32_t d = 0; d < Dk; ++d)
            for (int32_t j = 0; j < Dv; ++j) S[(int64_t)d * Dv + j] += kh[d] * u[j];

        /* output from the updated state o = S^T qh */
        for (int32_t j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int32_t d = 0; d < Dk; ++d) acc += S[(int64_t)d * Dv + j] * qh[d];
            J->out[o_base + j] = acc;
        }
    }

    if (J->final_state) {
        int64_t base = ((int64_t)b * J->nout + hslot) * (int64_t)Dk * Dv;
        for (int64_t i = 0; i < (int64_t)Dk * Dv; ++i) J->final_state[base + i] = S[i];
    }
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = malloc(sizeof(double) * (size_t)J->Dk * J->Dv);
    double *kh = malloc(sizeof(double) * (size_t)J->Dk);
    double *qh = malloc(sizeof(double) * (size_t)J->Dk);
    double *kv = malloc(sizeof(double) * (size_t)J->Dv);
    double *u = malloc(sizeof(double) * (size_t)J->Dv);
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t p = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (p >= J->npairs) break;
        run_pair(J, J->pairs[3 * p], J->pairs[3 * p + 1], J->pairs[3 * p + 2], S, kh, qh, kv, u);
    }
    free(S);
    free(kh);
    free(qh);
    free(kv);
    free(u);
    return NULL;
}

/*
 * Run the recurrence.  `heads` (length nheads) restricts the v-heads that are
 * computed (NULL: all Nv).  With a head list, `out` is [T, nheads, Dv] and
 * `final_state` is [B, nheads, Dk, Dv], head slot i holding v-head heads[i].
 * nthreads <= 0 uses every online core.
 * Returns the number of threads used, or a negative value on a bad argument.
 */
int gdn_oracle_recurrent(const void *q, int dt_q, const void *k, int dt_k, const void *v, int dt_v,
                         const void *g, int dt_g, const void *beta, int dt_beta, const int32_t *cu,
                         const void *pool, int dt_pool, const int32_t *state_indices, int32_t B,
                         int32_t Nqk, int32_t Nv, int32_t Dk, int32_t Dv, int32_t P, double scale,
                         double eps, double *out, double *final_state, const int32_t *heads,
                         int32_t nheads, int32_t nthreads)
{
    if (B < 0 || Nqk <= 0 || Nv <= 0 || Dk <= 0 || Dv <= 0 || Nv % Nqk != 0) return -1;
    if (pool && !state_indices && P < B) return -2;
    if (!heads) nheads = Nv;

    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.pool = pool;
    J.dt_q = dt_q; J.dt_k = dt_k; J.dt_v = dt_v; J.dt_g = dt_g; J.dt_beta = dt_beta;
    J.dt_pool = dt_pool;
    J.cu = cu; J.state_indices = state_indices;
    J.B = B; J.Nqk = Nqk; J.Nv = Nv; J.Dk = Dk; J.Dv = Dv; J.P = P;
    J.scale = scale; J.eps = eps; J.out = out; J.final_state = final_state;
    J.npairs = (int64_t)B * nheads;
    J.nout = nheads;
    int32_t *pairs = malloc(sizeof(int32_t) * 3 * (size_t)(J.npairs > 0 ? J.npairs : 1));
    int64_t n = 0;
    for (int32_t b = 0; b < B; ++b)
        for (int32_t i = 0; i < nheads; ++i) {
            if (heads && (heads[i] < 0 || heads[i] >= Nv)) { free(pairs); return -3; }
            pairs[3 * n] = b;
            pairs[3 * n + 1] = heads ? heads[i] : i;
            pairs[3 * n + 2] = i;
            ++n;
        }
    J.pairs = pairs;
    pthread_mutex_init(&J.lock, NULL);

    if (nthreads <= 0) nthreads = (int32_t)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if ((int64_t)nthreads > J.npairs) nthreads = (int32_t)(J.npairs > 0 ? J.npairs : 1);

    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int32_t i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int32_t i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    free(pairs);
    return nthreads;
}
