/*
 * kda_oracle.c -- fp64 CPU oracle for the Kimi Delta Attention (KDA) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker of the CUDA
 * library.  Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may build, load or call it.  It shares no code, header, helper or
 * constant with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (source: aiblin.ru, "Kimi K3 -- открытая модель, которая
 * обошла закрытых лидеров рынка", section "Как хранить миллион токенов в
 * памяти"): a fixed-size state S (d_k x d_v) is rewritten at every token -- the
 * old content is partly erased, then new content is written -- with a write
 * strength beta in (0,1) and a per-channel forget coefficient alpha, and alpha is
 * clamped to [e^-5, 1].  The exact update taken here (the page's formula did not
 * survive extraction; this is the plainest reading consistent with the prose):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                                (uses the UPDATED state)
 *     alpha_t = exp(clamp(log_alpha_t, -5, 0))       (d_k vector, scales rows)
 *
 * Two independent evaluations are provided:
 *   (A) kda_oracle_recurrent: the token-by-token definition above.
 *   (B) kda_oracle_chunked:   the chunkwise reformulation that the section
 *       "Как распараллелили последовательное обновление" of the same page
 *       describes ("all tokens of a chunk in parallel, then the state is passed
 *       from chunk to chunk"), written out in fp64 with plain exp(+g)/exp(-g)
 *       (safe in fp64 for any chunk up to a few hundred tokens: exp(+-5*128) is
 *       far inside the fp64 range).
 *
 * Both take inputs as fp32 or bf16 bit patterns (the exact values a GPU kernel
 * receives) and widen them exactly to fp64 before any arithmetic.
 *
 * Layouts (row-major, last index fastest; B folded into T, sequences given by
 * cu_seqlens over the packed token axis):
 *   q, k        [T, H, d_k]      qkv_dtype (0 = fp32, 1 = bf16 bits)
 *   v           [T, H, d_v]      qkv_dtype
 *   log_alpha   [T, H, d_k]      fp32
 *   beta        [T, H]           fp32
 *   s0          [N, H, d_k, d_v] fp32 or NULL (= zero state)
 *   cu_seqlens  [N + 1]          int64, cu[0] = 0, non-decreasing, cu[N] = T
 *   o           [o_tokens, H, d_v] fp64: written only for packed token index
 *               t < o_tokens (o_tokens <= T); pass 0 to skip outputs
 *   s_final     [N, H, d_k, d_v] fp64 or NULL
 *
 * Threads: one work item per (sequence, head); n_threads <= 0 means all cores.
 * Return 0 on success, nonzero on bad arguments.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *s0;
    const int64_t *cu;
    int64_t n_seqs, T, H, dk, dv, o_tokens, chunk;
    int qkv_dtype;
    double *o, *s_final;
    int64_t next_item; /* guarded by lock */
    pthread_mutex_t lock;
    int mode; /* 0 = recurrent, 1 = chunked */
} job_t;

static double widen(const void *base, int dtype, int64_t idx) {
    if (dtype == 0) return (double)((const float *)base)[idx];
    /* bf16: the 16 stored bits are the top half of an fp32 word */
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double clamp_log_alpha(float x) {
    /* clamp applied to the fp32 input; both bounds are exactly representable */
    float c = x < -5.0f ? -5.0f : x;
    c = c > 0.0f ? 0.0f : c;
    return (double)c;
}

/* (A) token recurrence for one (sequence n, head h). */
static void run_recurrent(const job_t *J, int64_t n, int64_t h, double *S, double *p) {
    const int64_t dk = J->dk, dv = J->dv, H = J->H;
    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const int64_t rk = (t * H + h) * dk, rv = (t * H + h) * dv;
        /* forget, row by row: Diag(alpha_t) S_{t-1} scales row i (key channel i);
         * in the same pass p = (Diag(alpha_t) S_{t-1})^T k_t, what the decayed
         * state returns for k_t */
        for (int64_t j = 0; j < dv; ++j) p[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i) {
            double a = exp(clamp_log_alpha(J->log_alpha[rk + i]));
            double ki = widen(J->k, J->qkv_dtype, rk + i);
            double *row = S + i * dv;
            for (int64_t j = 0; j < dv; ++j) {
                row[j] *= a;
                p[j] += row[j] * ki;
            }
        }
        /* erase-then-write: S += beta k (v - p)^T
         * == (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T;
         * in the same pass o_t = S_t^T q_t (the UPDATED state) */
        double b = (double)J->beta[t * H + h];
        for (int64_t j = 0; j < dv; ++j) p[j] = b * (widen(J->v, J->qkv_dtype, rv + j) - p[j]);
        const int want_o = t < J->o_tokens;
        double *o = want_o ? J->o + rv : p + dv; /* scratch row when o is not kept */
        for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i) {
            double ki = widen(J->k, J->qkv_dtype, rk + i);
            double qi = widen(J->q, J->qkv_dtype, rk + i);
            double *row = S + i * dv;
            for (int64_t j = 0; j < dv; ++j) {
                row[j] += ki * p[j];
                o[j] += row[j] * qi;
            }
        }
    }
}

/* (B) chunkwise reformulation for one (sequence n, head h).
 *
 * Inside a chunk with incoming state S0 and tokens r = 0..L-1 (g_r = inclusive
 * cumulative sum of the clamped log-gates over the chunk, per key channel):
 *   Kt = K*exp(g), Kh = K*exp(-g), Qt = Q*exp(g)
 *   A  = strict_lower(diag(beta) Kt Kh^T)
 *   (I + A) W  = diag(beta) Kt        (forward substitution)
 *   (I + A) U' = diag(beta) V
 *   U  = U' - W S0
 *   O  = Qt S0 + lower_incl_diag(Qt Kh^T) U
 *   S_L = Diag(exp(g_{L-1})) S0 + (K*exp(g_{L-1} - g))^T U
 * Derivation: with u_r = beta_r (v_r - (Diag(alpha_r) S_{r-1})^T k_r) the
 * recurrence reads S_r = Diag(alpha_r) S_{r-1} + k_r u_r^T; unrolling it inside
 * the chunk gives the lines above. */
static void run_chunked(const job_t *J, int64_t n, int64_t h, double *S, double *ws) {
    const int64_t dk = J->dk, dv = J->dv, H = J->H, C = J->chunk;
    double *g = ws;                /* C x dk */
    double *Kt = g + C * dk;       /* C x dk */
    double *Kh = Kt + C * dk;      /* C x dk */
    double *Qt = Kh + C * dk;      /* C x dk */
    double *A = Qt + C * dk;       /* C x C  */
    double *W = A + C * C;         /* C x dk */
    double *U = W + C * dk;        /* C x dv */
    double *Snew = U + C * dv;     /* dk x dv */
    for (int64_t c0 = J->cu[n]; c0 < J->cu[n + 1]; c0 += C) {
        int64_t L = J->cu[n + 1] - c0;
        if (L > C) L = C;
        for (int64_t r = 0; r < L; ++r) {
            const int64_t rk = ((c0 + r) * H + h) * dk;
            for (int64_t i = 0; i < dk; ++i) {
                double prev = r ? g[(r - 1) * dk + i] : 0.0;
                g[r * dk + i] = prev + clamp_log_alpha(J->log_alpha[rk + i]);
                double ki = widen(J->k, J->qkv_dtype, rk + i);
                double qi = widen(J->q, J->qkv_dtype, rk + i);
                Kt[r * dk + i] = ki * exp(g[r * dk + i]);
                Kh[r * dk + i] = ki * exp(-g[r * dk + i]);
                Qt[r * dk + i] = qi * exp(g[r * dk + i]);
            }
        }
        for (int64_t r = 0; r < L; ++r) {
            double br = (double)J->beta[(c0 + r) * H + h];
            for (int64_t j = 0; j < r; ++j) {
                double s = 0.0;
                for (int64_t i = 0; i < dk; ++i) s += Kt[r * dk + i] * Kh[j * dk + i];
                A[r * C + j] = br * s;
            }
        }
        /* forward substitution: row r of X = rhs_r - sum_{j<r} A[r,j] X_j */
        for (int64_t r = 0; r < L; ++r) {
            double br = (double)J->beta[(c0 + r) * H + h];
            const int64_t rv = ((c0 + r) * H + h) * dv;
            for (int64_t i = 0; i < dk; ++i) W[r * dk + i] = br * Kt[r * dk + i];
            for (int64_t e = 0; e < dv; ++e) U[r * dv + e] = br * widen(J->v, J->qkv_dtype, rv + e);
            for (int64_t j = 0; j < r; ++j) {
                double a = A[r * C + j];
                for (int64_t i = 0; i < dk; ++i) W[r * dk + i] -= a * W[j * dk + i];
                for (int64_t e = 0; e < dv; ++e) U[r * dv + e] -= a * U[j * dv + e];
            }
        }
        /* U = U' - W S0 */
        for (int64_t r = 0; r < L; ++r)
            for (int64_t i = 0; i < dk; ++i) {
                double w = W[r * dk + i];
                for (int64_t e = 0; e < dv; ++e) U[r * dv + e] -= w * S[i * dv + e];
            }
        /* O = Qt S0 + lower_incl_diag(Qt Kh^T) U */
        for (int64_t r = 0; r < L; ++r) {
            const int64_t t = c0 + r;
            if (t >= J->o_tokens) continue;
            double *o = J->o + (t * H + h) * dv;
            for (int64_t e = 0; e < dv; ++e) o[e] = 0.0;
            for (int64_t i = 0; i < dk; ++i) {
                double qi = Qt[r * dk + i];
                for (int64_t e = 0; e < dv; ++e) o[e] += qi * S[i * dv + e];
            }
            for (int64_t j = 0; j <= r; ++j) {
                double pj = 0.0;
                for (int64_t i = 0; i < dk; ++i) pj += Qt[r * dk + i] * Kh[j * dk + i];
                for (int64_t e = 0; e < dv; ++e) o[e] += pj * U[j * dv + e];
            }
        }
        /* S_L = Diag(exp(g_last)) S0 + (K * exp(g_last - g))^T U */
        const double *gl = g + (L - 1) * dk;
        for (int64_t i = 0; i < dk; ++i) {
            double decay = exp(gl[i]);
            for (int64_t e = 0; e < dv; ++e) Snew[i * dv + e] = decay * S[i * dv + e];
        }
        for (int64_t r = 0; r < L; ++r) {
            const int64_t rk = ((c0 + r) * H + h) * dk;
            for (int64_t i = 0; i < dk; ++i) {
                double kd = widen(J->k, J->qkv_dtype, rk + i) * exp(gl[i] - g[r * dk + i]);
                for (int64_t e = 0; e < dv; ++e) Snew[i * dv + e] += kd * U[r * dv + e];
            }
        }
        memcpy(S, Snew, (size_t)(dk * dv) * sizeof(double));
    }
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    const int64_t dk = J->dk, dv = J->dv, C = J->chunk;
    size_t ws_n = (size_t)(dk * dv + 2 * dv);
    if (J->mode == 1) ws_n += (size_t)(5 * C * dk + C * C + C * dv + dk * dv);
    double *S = (double *)malloc(ws_n * sizeof(double));
    if (!S) return (void *)1;
    double *ws = S + dk * dv;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t item = J->next_item++;
        pthread_mutex_unlock(&J->lock);
        if (item >= J->n_seqs * J->H) break;
        int64_t n = item / J->H, h = item % J->H;
        if (J->s0) {
            const float *src = J->s0 + (n * J->H + h) * dk * dv;
            for (int64_t x = 0; x < dk * dv; ++x) S[x] = (double)src[x];
        } else {
            memset(S, 0, (size_t)(dk * dv) * sizeof(double));
        }
        if (J->mode == 0)
            run_recurrent(J, n, h, S, ws);
        else
            run_chunked(J, n, h, S, ws);
        if (J->s_final) memcpy(J->s_final + (n * J->H + h) * dk * dv, S, (size_t)(dk * dv) * sizeof(double));
    }
    free(S);
    return NULL;
}

static int run_job(job_t *J, int n_threads) {
    if (J->n_seqs < 0 || J->H <= 0 || J->dk <= 0 || J->dv <= 0 || J->T < 0) return 1;
    if (J->cu[0] != 0 || J->cu[J->n_seqs] != J->T) return 2;
    for (int64_t n = 0; n < J->n_seqs; ++n)
        if (J->cu[n + 1] < J->cu[n]) return 3;
    if (J->o_tokens < 0 || J->o_tokens > J->T || (J->o_tokens > 0 && !J->o)) return 4;
    if (J->mode == 1 && J->chunk <= 0) return 5;
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    int64_t items = J->n_seqs * J->H;
    if (n_threads > items) n_threads = (int)(items > 0 ? items : 1);
    J->next_item = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int rc = 0;
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, worker, J);
    for (int i = 0; i < n_threads; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret) rc = 6;
    }
    free(th);
    pthread_mutex_destroy(&J->lock);
    return rc;
}

int kda_oracle_recurrent(const void *q, const void *k, const void *v, int qkv_dtype,
                         const float *log_alpha, const float *beta, const float *s0,
                         const int64_t *cu_seqlens, int64_t n_seqs, int64_t T, int64_t H,
                         int64_t dk, int64_t dv, double *o, int64_t o_tokens, double *s_final,
                         int n_threads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.qkv_dtype = qkv_dtype;
    J.log_alpha = log_alpha; J.beta = beta; J.s0 = s0; J.cu = cu_seqlens;
    J.n_seqs = n_seqs; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.o = o; J.o_tokens = o_tokens; J.s_final = s_final; J.mode = 0; J.chunk = 1;
    return run_job(&J, n_threads);
}

int kda_oracle_chunked(const void *q, const void *k, const void *v, int qkv_dtype,
                       const float *log_alpha, const float *beta, const float *s0,
                       const int64_t *cu_seqlens, int64_t n_seqs, int64_t T, int64_t H,
                       int64_t dk, int64_t dv, int64_t chunk, double *o, int64_t o_tokens,
                       double *s_final, int n_threads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.qkv_dtype = qkv_dtype;
    J.log_alpha = log_alpha; J.beta = beta; J.s0 = s0; J.cu = cu_seqlens;
    J.n_seqs = n_seqs; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.o = o; J.o_tokens = o_tokens; J.s_final = s_final; J.mode = 1; J.chunk = chunk;
    return run_job(&J, n_threads);
}
