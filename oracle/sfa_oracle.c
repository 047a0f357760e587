/*
 * CPU oracle for frame-restricted softmax attention.  TEST INFRASTRUCTURE ONLY:
 * this file is compiled into liboracle.so and is used by the tests, by smoke()
 * and by the bench's CPU-baseline leg.  The product library never links or
 * calls it, and it shares no code with the CUDA path.
 *
 * What it computes is the plain definition, in float64, with no blocking,
 * no online softmax and no reordering:
 *
 *   "LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de Video Largo",
 *   §2 Mecanismo Central: a query frame t attends only to the frames of A(t)
 *   instead of {0..T-1}; §Complejidad: cost O(|A(t)| * P * d) per query.
 *   "ISPA", §2.1 Dual-Stream Warmup: attention kernels track the per-row
 *   log-sum-exp, which is what lets two partial attentions be merged later.
 *
 * For query row i of frame t in head h, batch b, with key index set
 *   K(h,t) = union over f in A(h,t) of the token range [f*P, (f+1)*P):
 *     s_j   = scale * sum_k q_ik * k_jk                 (j in K)
 *     m     = max_j s_j
 *     l     = sum_j exp(s_j - m)
 *     O_i   = (sum_j exp(s_j - m) * v_j) / l
 *     LSE_i = m + ln(l)            (natural log of sum_j exp(s_j))
 *   K empty  ->  O_i = 0, LSE_i = -inf.
 *
 * Inputs are bf16 bit patterns, widened exactly to double.  Layout is
 * contiguous [B][H][L][d] for q (L = Tq*P) and k, v (L = Tkv*P).  Frame lists
 * are [H][Tq][Amax] int32 (entries beyond counts[h][t] are ignored) with
 * counts [H][Tq]; they are shared by every batch entry.
 *
 * Parity status: pinned (see tests/test_oracle_attention.py): dense case vs
 * a library SDPA, gathered-key case vs a library SDPA, closed forms
 * (Q = 0, constant V, key-shift invariance, key permutation invariance).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    int B, H, Tq, Tkv, P, d, Amax;
    double scale;
    const uint16_t *q, *k, *v;
    const int32_t *frames, *counts;
    const int64_t *rows;   /* flat row ids (b*H + h)*Lq + i, or NULL for all rows */
    int64_t n_rows;
    double *o, *lse;       /* [n_rows][d], [n_rows] */
    int n_threads;
    int thread_id;
    int status;
} job_t;

static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;   /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void *worker(void *arg)
{
    job_t *jb = (job_t *)arg;
    const int64_t Lq = (int64_t)jb->Tq * jb->P;
    const int64_t Lkv = (int64_t)jb->Tkv * jb->P;
    const int d = jb->d;
    double *s = (double *)malloc(sizeof(double) * (size_t)(Lkv > 0 ? Lkv : 1));
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Lkv > 0 ? Lkv : 1));
    double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !keys || !qrow) {
        jb->status = -1;
        free(s); free(keys); free(qrow);
        return NULL;
    }
    for (int64_t r = jb->thread_id; r < jb->n_rows; r += jb->n_threads) {
        const int64_t flat = jb->rows ? jb->rows[r] : r;
        const int64_t bh = flat / Lq;
        const int64_t i = flat % Lq;
        const int64_t b = bh / jb->H;
        const int h = (int)(bh % jb->H);
        const int t = (int)(i / jb->P);
        const uint16_t *qi = jb->q + (bh * Lq + i) * d;
        const uint16_t *kb = jb->k + bh * Lkv * d;
        const uint16_t *vb = jb->v + bh * Lkv * d;
        double *orow = jb->o + r * d;
        (void)b;

        /* K(h,t): every token of every attended frame */
        int64_t nk = 0;
        const int cnt = jb->counts[h * jb->Tq + t];
        const int32_t *fl = jb->frames + ((int64_t)h * jb->Tq + t) * jb->Amax;
        for (int a = 0; a < cnt; ++a) {
            const int64_t f = fl[a];
            for (int64_t p = 0; p < jb->P; ++p) keys[nk++] = f * jb->P + p;
        }

        for (int c = 0; c < d; ++c) qrow[c] = widen_bf16(qi[c]);
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        if (nk == 0) {
            jb->lse[r] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int64_t n = 0; n < nk; ++n) {
            const uint16_t *kj = kb + keys[n] * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qrow[c] * widen_bf16(kj[c]);
            s[n] = jb->scale * dot;
            if (s[n] > m) m = s[n];
        }
        double l = 0.0;
        for (int64_t n = 0; n < nk; ++n) {
            const double e = exp(s[n] - m);
            const uint16_t *vj = vb + keys[n] * d;
            l += e;
            for (int c = 0; c < d; ++c) orow[c] += e * widen_bf16(vj[c]);
        }
        for (int c = 0; c < d; ++c) orow[c] /= l;
        jb->lse[r] = m + log(l);
    }
    free(s); free(keys); free(qrow);
    return NULL;
}

/* Returns 0 on success, -1 on allocation failure, -2 on bad arguments. */
int oracle_attention(int B, int H, int Tq, int Tkv, int P, int d, double scale,
                     const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *frames, const int32_t *counts, int Amax,
                     const int64_t *rows, int64_t n_rows,
                     double *o, double *lse, int n_threads)
{
    if (B < 0 || H <= 0 || Tq <= 0 || Tkv <= 0 || P <= 0 || d <= 0 || Amax < 0) return -2;
    const int64_t total = (int64_t)B * H * Tq * P;
    if (!rows) n_rows = total;
    for (int h = 0; h < H; ++h)
        for (int t = 0; t < Tq; ++t) {
            const int c = counts[h * Tq + t];
            if (c < 0 || c > Amax) return -2;
            for (int a = 0; a < c; ++a) {
                const int32_t f = frames[((int64_t)h * Tq + t) * Amax + a];
                if (f < 0 || f >= Tkv) return -2;
            }
        }
    if (rows)
        for (int64_t r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= total) return -2;
    if (n_threads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = nc > 0 ? (int)nc : 1;
    }
    if (n_threads > 256) n_threads = 256;
    if (n_rows < n_threads) n_threads = n_rows > 0 ? (int)n_rows : 1;

    job_t *jobs = (job_t *)calloc((size_t)n_threads, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return -1; }
    for (int i = 0; i < n_threads; ++i) {
        job_t *jb = &jobs[i];
        jb->B = B; jb->H = H; jb->Tq = Tq; jb->Tkv = Tkv; jb->P = P; jb->d = d;
        jb->Amax = Amax; jb->scale = scale; jb->q = q; jb->k = k; jb->v = v;
        jb->frames = frames; jb->counts = counts; jb->rows = rows; jb->n_rows = n_rows;
        jb->o = o; jb->lse = lse; jb->n_threads = n_threads; jb->thread_id = i;
        pthread_create(&th[i], NULL, worker, jb);
    }
    int status = 0;
    for (int i = 0; i < n_threads; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].status) status = jobs[i].status;
    }
    free(jobs); free(th);
    return status;
}
