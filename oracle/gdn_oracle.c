/*
 * gdn_oracle.c -- fp64 CPU oracle for the Gated DeltaNet (GDN) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (bjdmk.com.cn article "为什么 Qwen3.8-Flash-Next 值得单独
 * 跑一遍", section 2.1 "Gated DeltaNet 负责廉价压缩历史", state-update formula):
 *
 *     S_t = alpha_t * (I - beta_t * k_t k_t^T) * S_{t-1} + beta_t * k_t v_t^T
 *
 * with S_t a d_k x d_v matrix, alpha_t the forget gate and beta_t the write
 * strength.  The same passage describes the write as storing the new value
 * minus what the memory already predicts for k_t; the loop below evaluates
 * exactly that expanded form, which equals the formula above term by term:
 *
 *     p   = S_{t-1}^T k_t                      (memory's prediction of v_t)
 *     S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t p)^T
 *
 * Readout (the pages are silent; the plainest reading, adopted throughout):
 * o_t = S_t^T q_t with the post-update state and no scale factor.
 *
 * Head layout (same article, section 2.1, and the jianying88.com article
 * "Qwen3.8-Flash-Next混合注意力深度解析", section 三, config fields
 * linear_num_value_heads / linear_num_key_heads): H_v value heads share H_qk
 * query/key heads; value head h reads query/key head h / (H_v / H_qk).
 * Gates are one scalar per (token, value head).
 *
 * Arithmetic: every input is widened exactly to double (bf16 bits are the top
 * half of an IEEE binary32); all accumulation is in double, sequential in the
 * token order, with no blocking or reordering.
 *
 * Work is split into independent "units" (t0, t1, h): the token range
 * [t0, t1) of one sequence and one value head.  Units run on a pthread pool.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BF16 1
#define ORACLE_F32 2

typedef struct {
    const void *q, *k, *v;
    int io_dtype;
    const float *log_alpha, *beta;
    int T, H_qk, H_v, dk, dv;
    const int32_t *units; /* n_units x 3 : t0, t1, h */
    const int64_t *o_offsets; /* row offset of each unit's o block, or NULL */
    int n_units;
    const double *S_init; /* n_units x dk x dv, or NULL for zeros */
    double *S_out;        /* n_units x dk x dv */
    double *o_out;        /* rows x dv, or NULL */
    int next;             /* work counter */
    pthread_mutex_t lock;
} oracle_job;

static double widen(const void *base, int io_dtype, size_t idx) {
    if (io_dtype == ORACLE_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[idx];
}

static void run_unit(oracle_job *J, int u, double *kbuf, double *qbuf) {
    const int t0 = J->units[3 * u], t1 = J->units[3 * u + 1], h = J->units[3 * u + 2];
    const int dk = J->dk, dv = J->dv;
    const int group = J->H_v / J->H_qk;
    const int hq = h / group;
    double *S = J->S_out + (size_t)u * dk * dv;
    double *p = (double *)malloc(sizeof(double) * dv);
    if (J->S_init)
        memcpy(S, J->S_init + (size_t)u * dk * dv, sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * dk * dv);

    for (int t = t0; t < t1; ++t) {
        const double alpha = exp((double)J->log_alpha[(size_t)t * J->H_v + h]);
        const double beta = (double)J->beta[(size_t)t * J->H_v + h];
        const size_t qk_base = ((size_t)t * J->H_qk + hq) * dk;
        const size_t v_base = ((size_t)t * J->H_v + h) * dv;
        for (int i = 0; i < dk; ++i) {
            kbuf[i] = widen(J->k, J->io_dtype, qk_base + i);
            qbuf[i] = widen(J->q, J->io_dtype, qk_base + i);
        }
        /* p = S^T k */
        for (int j = 0; j < dv; ++j) p[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double ki = kbuf[i];
            const double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) p[j] += Si[j] * ki;
        }
        /* p <- beta * (v - alpha p): the corrected write */
        for (int j = 0; j < dv; ++j)
            p[j] = beta * (widen(J->v, J->io_dtype, v_base + j) - alpha * p[j]);
        /* S <- alpha S + k p^T */
        for (int i = 0; i < dk; ++i) {
            const double ki = kbuf[i];
            double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] = alpha * Si[j] + ki * p[j];
        }
        /* o_t = S_t^T q_t */
        if (J->o_out) {
            double *o = J->o_out + ((size_t)J->o_offsets[u] + (t - t0)) * dv;
            for (int j = 0; j < dv; ++j) o[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double qi = qbuf[i];
                const double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) o[j] += Si[j] * qi;
            }
        }
    }
    free(p);
}

static void *worker(void *arg) {
    oracle_job *J = (oracle_job *)arg;
    double *kbuf = (double *)malloc(sizeof(double) * J->dk);
    double *qbuf = (double *)malloc(sizeof(double) * J->dk);
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        run_unit(J, u, kbuf, qbuf);
    }
    free(kbuf);
    free(qbuf);
    return NULL;
}

/*
 * Run the recurrence over every unit.  Returns 0 on success, -1 on a bad
 * argument.  o_offsets[u] is the first row of unit u in o_out (rows of dv
 * doubles); it may be NULL only when o_out is NULL.
 */
int gdn_oracle_run(const void *q, const void *k, const void *v, int io_dtype,
                   const float *log_alpha, const float *beta,
                   int T, int H_qk, int H_v, int dk, int dv,
                   const int32_t *units, int n_units,
                   const double *S_init, double *S_out,
                   double *o_out, const int64_t *o_offsets, int n_threads) {
    if (!q || !k || !v || !log_alpha || !beta || !units || !S_out) return -1;
    if (io_dtype != ORACLE_BF16 && io_dtype != ORACLE_F32) return -1;
    if (H_qk <= 0 || H_v <= 0 || H_v % H_qk != 0 || dk <= 0 || dv <= 0 || T < 0) return -1;
    if (o_out && !o_offsets) return -1;
    for (int u = 0; u < n_units; ++u) {
        const int t0 = units[3 * u], t1 = units[3 * u + 1], h = units[3 * u + 2];
        if (t0 < 0 || t1 < t0 || t1 > T || h < 0 || h >= H_v) return -1;
    }
    oracle_job J;
    J.q = q; J.k = k; J.v = v; J.io_dtype = io_dtype;
    J.log_alpha = log_alpha; J.beta = beta;
    J.T = T; J.H_qk = H_qk; J.H_v = H_v; J.dk = dk; J.dv = dv;
    J.units = units; J.o_offsets = o_offsets; J.n_units = n_units;
    J.S_init = S_init; J.S_out = S_out; J.o_out = o_out;
    J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_units) n_threads = n_units > 0 ? n_units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
