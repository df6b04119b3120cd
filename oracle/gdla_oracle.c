/*
 * GDLA oracle: plain, slow, fp64 CPU implementation of the Grouped
 * Differential Latent Attention core (prefill, its backward, decode and decode
 * over the compressed cache).
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library. The CUDA library never calls
 * it and shares no code, header or constant with it.
 *
 * What it follows (aitrends.kr/articles/94908, "314B MoE 언어 모델 Motif 3의
 * 구조와 학습 시스템", GDLA paragraphs):
 *  - the two attention paths (signal and noise) share one KV head, and the
 *    noise output is subtracted from the signal output:
 *        D_t = H_{S,t} - lambda_t (.) Repeat_g(H_{N,t})
 *    followed by the query-based element-wise output gate ("GDLA query path"
 *    paragraph);
 *  - 80 query heads / 16 KV heads, 64 signal + 16 noise, dqk = 192, dv = 128
 *    ("GDLA head configuration" paragraph; also Table 1 of the metalmedia.ai
 *    digest of arXiv 2608.09119);
 *  - group ratio g = 4, n_N = n_H/(g+1), n_S = g n_N; each signal head is
 *    paired with the noise head of its own group; lambda_t = sigmoid(x_t W^l)
 *    lies in (0, 1) ("group ratio" paragraph);
 *  - full causal attention, or sliding-window attention over 128 tokens
 *    (Table 1 "Hybrid GDLA (1 full / 3 sliding-window)"; idailynews article,
 *    hybrid-attention paragraph).
 *
 * Readings taken where the pages are silent (each stated once here):
 *  - lambda is one fp32 scalar per (token, signal head), broadcast over dv;
 *  - Repeat_g is contiguous: noise head j serves signal heads 4j..4j+3, and
 *    both use KV head j;
 *  - the softmax scale is 1/sqrt(192);
 *  - a window of W keys includes the query itself: keys u in [t-W+1, t];
 *    window <= 0 means full causal;
 *  - the gate is out = sigmoid(gate_logit) * D, element-wise per (token,
 *    signal head, d); nothing else (no per-head norm) follows the subtract;
 *  - decode: the single query of sequence b sits at position L_b - 1 and the
 *    cache already holds its key and value.
 *
 * Arithmetic: every bf16 input is widened exactly to double, every fp32 lambda
 * is widened exactly to double, and all arithmetic is in double with no tiling
 * or reordering beyond the sums written below.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GROUP 4     /* signal heads per noise head (g) */
#define DQK 192     /* query/key head dim */
#define DV 128      /* value head dim */

static double bf16_to_double(uint16_t x) {
    uint32_t bits = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * One softmax-attention head for one query row:
 *   s_u = (q . k_u) / sqrt(192),  w_u = exp(s_u - max_u s_u),
 *   H = sum_u w_u v_u / sum_u w_u,
 * over the keys u = 0..nkeys-1 whose rows start at k_rows + u*kstride and
 * v_rows + u*vstride. `scores` has room for nkeys doubles.
 */
static void attend(const uint16_t *q, const uint16_t *k_rows, const uint16_t *v_rows,
                   long kstride, long vstride, long nkeys, double *scores, double *h) {
    double qd[DQK];
    for (int d = 0; d < DQK; ++d) qd[d] = bf16_to_double(q[d]);
    const double root = sqrt((double)DQK);
    double smax = -INFINITY;
    for (long u = 0; u < nkeys; ++u) {
        const uint16_t *kr = k_rows + u * kstride;
        double s = 0.0;
        for (int d = 0; d < DQK; ++d) s += qd[d] * bf16_to_double(kr[d]);
        s = s / root;
        scores[u] = s;
        if (s > smax) smax = s;
    }
    double den = 0.0;
    for (int d = 0; d < DV; ++d) h[d] = 0.0;
    for (long u = 0; u < nkeys; ++u) {
        const uint16_t *vr = v_rows + u * vstride;
        double w = exp(scores[u] - smax);
        den += w;
        for (int d = 0; d < DV; ++d) h[d] += w * bf16_to_double(vr[d]);
    }
    for (int d = 0; d < DV; ++d) h[d] /= den;
}

/*
 * One output row of one group: the 4 signal heads and the noise head of group
 * j attend over the same keys; then D_i = H_S,i - lambda_i * H_N and
 * out_i = D_i / (1 + exp(-g_i)).
 *   qs      : 4 signal query rows (4*DQK, consecutive heads 4j..4j+3)
 *   qn      : the noise query row of group j
 *   k_rows, v_rows : first visible key/value row of group j
 *   lam     : 4 lambda values for heads 4j..4j+3
 *   gate    : 4 x DV gate logits
 *   out     : 4 x DV doubles
 */
static void group_row(const uint16_t *qs, const uint16_t *qn, const uint16_t *k_rows,
                      const uint16_t *v_rows, long kstride, long vstride, long nkeys,
                      const float *lam, const uint16_t *gate, double *scores, double *out) {
    double hn[DV], hs[DV];
    attend(qn, k_rows, v_rows, kstride, vstride, nkeys, scores, hn);
    for (int i = 0; i < GROUP; ++i) {
        attend(qs + (long)i * DQK, k_rows, v_rows, kstride, vstride, nkeys, scores, hs);
        const double l = (double)lam[i];
        for (int d = 0; d < DV; ++d) {
            const double dd = hs[d] - l * hn[d];
            const double g = bf16_to_double(gate[(long)i * DV + d]);
            out[(long)i * DV + d] = dd / (1.0 + exp(-g));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Prefill                                                                  */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q_sig, *q_noise, *k, *v, *gate;
    const float *lambda;
    int hkv, window;
    const int64_t *row_token;  /* packed token index of each requested row */
    const int64_t *row_seq_start; /* packed index of the row's sequence start */
    int64_t num_rows;
    double *out;               /* [num_rows, 4*hkv, DV] */
    long max_keys;
    int nthreads, tid;
} prefill_job_t;

static void *prefill_worker(void *arg) {
    prefill_job_t *J = (prefill_job_t *)arg;
    const int hs = GROUP * J->hkv;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(J->max_keys > 0 ? J->max_keys : 1));
    if (!scores) return (void *)1;
    const int64_t ntasks = J->num_rows * J->hkv;
    for (int64_t task = J->tid; task < ntasks; task += J->nthreads) {
        const int64_t r = task / J->hkv;
        const int j = (int)(task % J->hkv);
        const int64_t n = J->row_token[r];        /* packed token index */
        const int64_t s0 = J->row_seq_start[r];   /* sequence start */
        const int64_t t = n - s0;                 /* position in sequence */
        int64_t lo = 0;
        if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;
        const long nkeys = (long)(t - lo + 1);
        const long kstride = (long)J->hkv * DQK, vstride = (long)J->hkv * DV;
        const uint16_t *krow = J->k + (s0 + lo) * kstride + (long)j * DQK;
        const uint16_t *vrow = J->v + (s0 + lo) * vstride + (long)j * DV;
        const uint16_t *qs = J->q_sig + (n * hs + (long)GROUP * j) * DQK;
        const uint16_t *qn = J->q_noise + (n * J->hkv + j) * DQK;
        const float *lam = J->lambda + n * hs + GROUP * j;
        const uint16_t *gate = J->gate + (n * hs + (long)GROUP * j) * DV;
        double *out = J->out + (r * hs + (long)GROUP * j) * DV;
        group_row(qs, qn, krow, vrow, kstride, vstride, nkeys, lam, gate, scores, out);
    }
    free(scores);
    return NULL;
}

static int run_threads(void *(*fn)(void *), void *jobs, size_t job_size, int nthreads) {
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -1;
    int rc = 0, started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, fn, (char *)jobs + (size_t)i * job_size) != 0) { rc = -1; break; }
        ++started;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret != NULL) rc = -1;
    }
    free(th);
    return rc;
}

/*
 * Packed varlen prefill. Inputs are laid out exactly as the CUDA library's
 * (row-major, N = sum(seqlens)):
 *   q_sig [N, 4*hkv, 192] bf16 bits, q_noise [N, hkv, 192], k [N, hkv, 192],
 *   v [N, hkv, 128], lambda [N, 4*hkv] fp32, gate [N, 4*hkv, 128] bf16 bits.
 * rows: the packed token indices to evaluate (num_rows of them); out receives
 * [num_rows, 4*hkv, 128] doubles. Returns 0, or -1 on a bad argument or an
 * allocation/thread failure.
 */
int gdla_oracle_prefill(const uint16_t *q_sig, const uint16_t *q_noise, const uint16_t *k,
                        const uint16_t *v, const float *lambda, const uint16_t *gate,
                        int hkv, int batch, const int32_t *seqlens, int window,
                        const int64_t *rows, int64_t num_rows, double *out, int nthreads) {
    if (hkv < 1 || batch < 0 || num_rows < 0 || nthreads < 1) return -1;
    int64_t total = 0;
    long max_len = 0;
    for (int b = 0; b < batch; ++b) {
        if (seqlens[b] < 0) return -1;
        total += seqlens[b];
        if (seqlens[b] > max_len) max_len = seqlens[b];
    }
    int64_t *seq_start = (int64_t *)malloc(sizeof(int64_t) * (size_t)(num_rows > 0 ? num_rows : 1));
    if (!seq_start) return -1;
    for (int64_t r = 0; r < num_rows; ++r) {
        const int64_t n = rows[r];
        if (n < 0 || n >= total) { free(seq_start); return -1; }
        int64_t s0 = 0;
        for (int b = 0; b < batch; ++b) {
            if (n < s0 + seqlens[b]) break;
            s0 += seqlens[b];
        }
        seq_start[r] = s0;
    }
    prefill_job_t *jobs = (prefill_job_t *)malloc(sizeof(prefill_job_t) * (size_t)nthreads);
    if (!jobs) { free(seq_start); return -1; }
    for (int i = 0; i < nthreads; ++i) {
        prefill_job_t J = {q_sig, q_noise, k, v, gate, lambda, hkv, window, rows, seq_start,
                           num_rows, out, max_len, nthreads, i};
        jobs[i] = J;
    }
    int rc = run_threads(prefill_worker, jobs, sizeof(prefill_job_t), nthreads);
    free(jobs);
    free(seq_start);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Decode                                                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q_sig, *q_noise, *k, *v, *gate;
    const float *lambda;
    const int64_t *cu;  /* [batch+1] packed cache offsets */
    int batch, hkv, window;
    double *out;        /* [batch, 4*hkv, DV] */
    long max_keys;
    int nthreads, tid;
} decode_job_t;

static void *decode_worker(void *arg) {
    decode_job_t *J = (decode_job_t *)arg;
    const int hs = GROUP * J->hkv;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(J->max_keys > 0 ? J->max_keys : 1));
    if (!scores) return (void *)1;
    const int64_t ntasks = (int64_t)J->batch * J->hkv;
    for (int64_t task = J->tid; task < ntasks; task += J->nthreads) {
        const int64_t b = task / J->hkv;
        const int j = (int)(task % J->hkv);
        const int64_t s0 = J->cu[b];
        const int64_t len = J->cu[b + 1] - s0;
        const int64_t t = len - 1;              /* the query's own position */
        int64_t lo = 0;
        if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;
        const long nkeys = (long)(t - lo + 1);
        const long kstride = (long)J->hkv * DQK, vstride = (long)J->hkv * DV;
        const uint16_t *krow = J->k + (s0 + lo) * kstride + (long)j * DQK;
        const uint16_t *vrow = J->v + (s0 + lo) * vstride + (long)j * DV;
        const uint16_t *qs = J->q_sig + (b * hs + (long)GROUP * j) * DQK;
        const uint16_t *qn = J->q_noise + (b * J->hkv + j) * DQK;
        const float *lam = J->lambda + b * hs + GROUP * j;
        const uint16_t *gate = J->gate + (b * hs + (long)GROUP * j) * DV;
        double *out = J->out + (b * hs + (long)GROUP * j) * DV;
        group_row(qs, qn, krow, vrow, kstride, vstride, nkeys, lam, gate, scores, out);
    }
    free(scores);
    return NULL;
}

/*
 * Varlen decode: one query per sequence at position L_b - 1.
 *   q_sig [B, 4*hkv, 192], q_noise [B, hkv, 192], k_cache [Nk, hkv, 192],
 *   v_cache [Nk, hkv, 128] (sequence b owns rows cu[b]..cu[b+1]-1),
 *   lambda [B, 4*hkv] fp32, gate [B, 4*hkv, 128]; out [B, 4*hkv, 128] doubles.
 * Every L_b must be >= 1. Returns 0, or -1 on a bad argument.
 */
int gdla_oracle_decode(const uint16_t *q_sig, const uint16_t *q_noise, const uint16_t *k_cache,
                       const uint16_t *v_cache, const int64_t *cu_seqlens_k, const float *lambda,
                       const uint16_t *gate, int batch, int hkv, int window, double *out,
                       int nthreads) {
    if (hkv < 1 || batch < 0 || nthreads < 1) return -1;
    long max_len = 0;
    for (int b = 0; b < batch; ++b) {
        const int64_t len = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        if (len < 1) return -1;
        if (len > max_len) max_len = (long)len;
    }
    decode_job_t *jobs = (decode_job_t *)malloc(sizeof(decode_job_t) * (size_t)nthreads);
    if (!jobs) return -1;
    for (int i = 0; i < nthreads; ++i) {
        decode_job_t J = {q_sig, q_noise, k_cache, v_cache, gate, lambda, cu_seqlens_k,
                          batch, hkv, window, out, max_len, nthreads, i};
        jobs[i] = J;
    }
    int rc = run_threads(decode_worker, jobs, sizeof(decode_job_t), nthreads);
    free(jobs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Decode over the compressed (latent) KV cache, with the projections        */
/* absorbed                                                                  */
/* ------------------------------------------------------------------------ */
/*
 * What it follows ([A], head-configuration paragraph): the KV path keeps one
 * compressed KV row per token (KV low-rank dimension 512) and one rotary key
 * (64) shared by every KV head; the 16 KV heads are an up-projection of the
 * compressed row. Readings: the 192 query-key dims are 128 non-rotary then 64
 * rotary; per KV head j,
 *     K_j,u = [ W^UK_j c_u (128) | kr_u (64) ],   V_j,u = W^UV_j c_u (128),
 * with W^UK_j and W^UV_j of shape [128 x 512]. A query of group j with its
 * non-rotary part absorbed, q_abs = [ W^UK_j^T q_nope (512) | q_rope (64) ],
 * gives q . K_j,u = q_abs . [c_u | kr_u], and sum_u p_u V_j,u = W^UV_j sum_u p_u c_u.
 * So every head attends over the shared 576-wide rows [c_u | kr_u] (same
 * 1/sqrt(192) scale) and its 512-wide latent output is projected by W^UV_j.
 */
#define DC 512      /* KV low-rank (latent) dim */
#define DR 64       /* shared rotary key dim */
#define DL (DC + DR)

/* One head over the latent rows: the 512-wide softmax-weighted latent average. */
static void attend_latent(const uint16_t *q, const uint16_t *rows, long nkeys, double *scores, double *o) {
    double qd[DL];
    for (int e = 0; e < DL; ++e) qd[e] = bf16_to_double(q[e]);
    const double root = sqrt((double)DQK);
    double smax = -INFINITY;
    for (long u = 0; u < nkeys; ++u) {
        const uint16_t *r = rows + u * DL;
        double s = 0.0;
        for (int e = 0; e < DL; ++e) s += qd[e] * bf16_to_double(r[e]);
        s = s / root;
        scores[u] = s;
        if (s > smax) smax = s;
    }
    double den = 0.0;
    for (int e = 0; e < DC; ++e) o[e] = 0.0;
    for (long u = 0; u < nkeys; ++u) {
        const uint16_t *r = rows + u * DL;
        const double w = exp(scores[u] - smax);
        den += w;
        for (int e = 0; e < DC; ++e) o[e] += w * bf16_to_double(r[e]);
    }
    for (int e = 0; e < DC; ++e) o[e] /= den;
}

/* H = W^UV_j o: [128 x 512] times a 512-vector. */
static void up_project(const uint16_t *w_uv_j, const double *o, double *h) {
    for (int d = 0; d < DV; ++d) {
        double acc = 0.0;
        for (int e = 0; e < DC; ++e) acc += bf16_to_double(w_uv_j[(long)d * DC + e]) * o[e];
        h[d] = acc;
    }
}

typedef struct {
    const uint16_t *q_sig, *q_noise, *ckv, *w_uv, *gate;
    const float *lambda;
    const int64_t *cu;
    int batch, hkv, window;
    double *out;
    long max_keys;
    int nthreads, tid;
} latent_job_t;

static void *latent_worker(void *arg) {
    latent_job_t *J = (latent_job_t *)arg;
    const int hs = GROUP * J->hkv;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(J->max_keys > 0 ? J->max_keys : 1));
    if (!scores) return (void *)1;
    const int64_t ntasks = (int64_t)J->batch * J->hkv;
    for (int64_t task = J->tid; task < ntasks; task += J->nthreads) {
        const int64_t b = task / J->hkv;
        const int j = (int)(task % J->hkv);
        const int64_t s0 = J->cu[b];
        const int64_t t = J->cu[b + 1] - s0 - 1;   /* the query's own position */
        int64_t lo = 0;
        if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;
        const long nkeys = (long)(t - lo + 1);
        const uint16_t *rows = J->ckv + (s0 + lo) * DL;
        const uint16_t *w_uv_j = J->w_uv + (long)j * DV * DC;
        double o[DC], hn[DV], hsig[DV];
        attend_latent(J->q_noise + (b * J->hkv + j) * DL, rows, nkeys, scores, o);
        up_project(w_uv_j, o, hn);
        for (int i = 0; i < GROUP; ++i) {
            const int64_t head = b * hs + (long)GROUP * j + i;
            attend_latent(J->q_sig + head * DL, rows, nkeys, scores, o);
            up_project(w_uv_j, o, hsig);
            const double l = (double)J->lambda[head];
            for (int d = 0; d < DV; ++d) {
                const double dd = hsig[d] - l * hn[d];
                const double g = bf16_to_double(J->gate[head * DV + d]);
                J->out[head * DV + d] = dd / (1.0 + exp(-g));
            }
        }
    }
    free(scores);
    return NULL;
}

/*
 * Varlen decode over the latent cache: one query per sequence at position
 * L_b - 1, queries already absorbed.
 *   q_abs_sig [B, 4*hkv, 576], q_abs_noise [B, hkv, 576] bf16 bits,
 *   ckv [Nk, 576] = [c (512) | kr (64)] bf16 bits (sequence b owns rows
 *   cu[b]..cu[b+1]-1), w_uv [hkv, 128, 512] bf16 bits, lambda [B, 4*hkv] fp32,
 *   gate [B, 4*hkv, 128]; out [B, 4*hkv, 128] doubles.
 * Every L_b must be >= 1. Returns 0, or -1 on a bad argument.
 */
int gdla_oracle_decode_latent(const uint16_t *q_abs_sig, const uint16_t *q_abs_noise, const uint16_t *ckv,
                              const int64_t *cu_seqlens_k, const uint16_t *w_uv, const float *lambda,
                              const uint16_t *gate, int batch, int hkv, int window, double *out,
                              int nthreads) {
    if (hkv < 1 || batch < 0 || nthreads < 1) return -1;
    long max_len = 0;
    for (int b = 0; b < batch; ++b) {
        const int64_t len = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        if (len < 1) return -1;
        if (len > max_len) max_len = (long)len;
    }
    latent_job_t *jobs = (latent_job_t *)malloc(sizeof(latent_job_t) * (size_t)nthreads);
    if (!jobs) return -1;
    for (int i = 0; i < nthreads; ++i) {
        latent_job_t J = {q_abs_sig, q_abs_noise, ckv, w_uv, gate, lambda, cu_seqlens_k,
                          batch, hkv, window, out, max_len, nthreads, i};
        jobs[i] = J;
    }
    int rc = run_threads(latent_worker, jobs, sizeof(latent_job_t), nthreads);
    free(jobs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Prefill backward                                                         */
/* ------------------------------------------------------------------------ */
/*
 * Gradients of L = sum(dout * out) with respect to every input of the packed
 * prefill, by the chain rule written out on the definition above (the pages
 * train GDLA end to end; they print no gradient, so this is the plain
 * derivative of the forward as read here):
 *   sigma_i = 1 / (1 + exp(-g_i)),  out_i = sigma_i D_i,  D_i = H_S,i - lambda_i H_N
 *   dgate_i   = dout_i * D_i * sigma_i (1 - sigma_i)
 *   dD_i      = dout_i * sigma_i
 *   dlambda_i = -sum_d dD_i[d] H_N[d]
 *   dH_S,i    = dD_i,   dH_N = -sum_i lambda_i dD_i
 * and for every head h of the group with P_u = softmax_u(s_u), s_u = q_h.k_u / sqrt(192),
 * H_h = sum_u P_u v_u:
 *   dv_u += P_u dH_h
 *   dP_u  = dH_h . v_u,   dS_u = P_u (dP_u - sum_w P_w dP_w)
 *   dq_h += sum_u dS_u k_u / sqrt(192),   dk_u += dS_u q_h / sqrt(192)
 * One job is one (sequence, group): it owns the dk, dv rows of that group in
 * that sequence, so the accumulation needs no locking.
 */
typedef struct {
    const uint16_t *q_sig, *q_noise, *k, *v, *gate, *dout;
    const float *lambda;
    int hkv, window, batch;
    const int32_t *seqlens;
    const int64_t *seq_start;
    double *dq_sig, *dq_noise, *dk, *dv, *dlambda, *dgate;
    long max_len;
    int nthreads, tid;
} bwd_job_t;

/* Softmax weights of one head over keys u = 0..nkeys-1 (rows k_rows + u*kstride). */
static void softmax_weights(const uint16_t *q, const uint16_t *k_rows, long kstride, long nkeys, double *p) {
    double qd[DQK];
    for (int d = 0; d < DQK; ++d) qd[d] = bf16_to_double(q[d]);
    const double root = sqrt((double)DQK);
    double smax = -INFINITY;
    for (long u = 0; u < nkeys; ++u) {
        const uint16_t *kr = k_rows + u * kstride;
        double s = 0.0;
        for (int d = 0; d < DQK; ++d) s += qd[d] * bf16_to_double(kr[d]);
        p[u] = s / root;
        if (p[u] > smax) smax = p[u];
    }
    double den = 0.0;
    for (long u = 0; u < nkeys; ++u) {
        p[u] = exp(p[u] - smax);
        den += p[u];
    }
    for (long u = 0; u < nkeys; ++u) p[u] /= den;
}

/* Backward of one head for one query row: given P (nkeys) and dH, accumulate
 * dq (DQK), dk rows and dv rows (doubles, strided like the keys). */
static void head_backward(const uint16_t *q, const uint16_t *k_rows, const uint16_t *v_rows, long kstride,
                          long vstride, long nkeys, const double *p, const double *dh, double *dp, double *dq,
                          double *dk_rows, double *dv_rows, long dkstride, long dvstride) {
    const double root = sqrt((double)DQK);
    double drow = 0.0;
    for (long u = 0; u < nkeys; ++u) {
        const uint16_t *vr = v_rows + u * vstride;
        double s = 0.0;
        for (int d = 0; d < DV; ++d) s += dh[d] * bf16_to_double(vr[d]);
        dp[u] = s;
        drow += p[u] * s;
    }
    for (long u = 0; u < nkeys; ++u) {
        const double ds = p[u] * (dp[u] - drow);
        const uint16_t *kr = k_rows + u * kstride;
        double *dkr = dk_rows + u * dkstride;
        double *dvr = dv_rows + u * dvstride;
        for (int d = 0; d < DQK; ++d) {
            dq[d] += ds * bf16_to_double(kr[d]) / root;
            dkr[d] += ds * bf16_to_double(q[d]) / root;
        }
        for (int d = 0; d < DV; ++d) dvr[d] += p[u] * dh[d];
    }
}

static void *bwd_worker(void *arg) {
    bwd_job_t *J = (bwd_job_t *)arg;
    const int hkv = J->hkv, hs = GROUP * hkv;
    const long n1 = J->max_len > 0 ? J->max_len : 1;
    double *p = (double *)malloc(sizeof(double) * (size_t)n1 * (GROUP + 1));
    double *dp = (double *)malloc(sizeof(double) * (size_t)n1);
    if (!p || !dp) { free(p); free(dp); return (void *)1; }
    const long kstride = (long)hkv * DQK, vstride = (long)hkv * DV;
    for (int64_t task = J->tid; task < (int64_t)J->batch * hkv; task += J->nthreads) {
        const int b = (int)(task / hkv), j = (int)(task % hkv);
        const int64_t s0 = J->seq_start[b];
        const long L = J->seqlens[b];
        for (long t = 0; t < L; ++t) {
            const int64_t n = s0 + t;
            long lo = 0;
            if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;
            const long nkeys = t - lo + 1;
            const uint16_t *krow = J->k + (s0 + lo) * kstride + (long)j * DQK;
            const uint16_t *vrow = J->v + (s0 + lo) * vstride + (long)j * DV;
            double *dkrow = J->dk + (s0 + lo) * kstride + (long)j * DQK;
            double *dvrow = J->dv + (s0 + lo) * vstride + (long)j * DV;
            const uint16_t *qs = J->q_sig + (n * hs + (long)GROUP * j) * DQK;
            const uint16_t *qn = J->q_noise + (n * hkv + j) * DQK;
            /* forward: P and H of the 4 signal heads (h = 0..3) and the noise head (h = 4) */
            double hh[GROUP + 1][DV];
            for (int h = 0; h <= GROUP; ++h) {
                const uint16_t *q = (h < GROUP) ? qs + (long)h * DQK : qn;
                double *ph = p + (long)h * n1;
                softmax_weights(q, krow, kstride, nkeys, ph);
                for (int d = 0; d < DV; ++d) hh[h][d] = 0.0;
                for (long u = 0; u < nkeys; ++u)
                    for (int d = 0; d < DV; ++d) hh[h][d] += ph[u] * bf16_to_double(vrow[u * vstride + d]);
            }
            /* the gate and the subtract */
            double dh[GROUP + 1][DV];
            for (int d = 0; d < DV; ++d) dh[GROUP][d] = 0.0;
            for (int i = 0; i < GROUP; ++i) {
                const long row = n * hs + (long)GROUP * j + i;
                const double l = (double)J->lambda[row];
                double dl = 0.0;
                for (int d = 0; d < DV; ++d) {
                    const double g = bf16_to_double(J->gate[row * DV + d]);
                    const double sg = 1.0 / (1.0 + exp(-g));
                    const double dd = hh[i][d] - l * hh[GROUP][d];
                    const double go = bf16_to_double(J->dout[row * DV + d]);
                    J->dgate[row * DV + d] = go * dd * sg * (1.0 - sg);
                    const double ddd = go * sg;
                    dl -= ddd * hh[GROUP][d];
                    dh[i][d] = ddd;
                    dh[GROUP][d] -= l * ddd;
                }
                J->dlambda[row] = dl;
            }
            /* attention backward of the five heads */
            for (int h = 0; h <= GROUP; ++h) {
                const uint16_t *q = (h < GROUP) ? qs + (long)h * DQK : qn;
                double *dq = (h < GROUP) ? J->dq_sig + (n * hs + (long)GROUP * j + h) * DQK
                                         : J->dq_noise + (n * hkv + j) * DQK;
                head_backward(q, krow, vrow, kstride, vstride, nkeys, p + (long)h * n1, dh[h], dp, dq, dkrow,
                              dvrow, kstride, vstride);
            }
        }
    }
    free(p);
    free(dp);
    return NULL;
}

/*
 * Packed varlen prefill backward. Inputs as gdla_oracle_prefill, plus dout
 * [N, 4*hkv, 128] bf16 bits (the gradient of the output). Outputs, all double
 * and zeroed here: dq_sig [N, 4*hkv, 192], dq_noise [N, hkv, 192],
 * dk [N, hkv, 192], dv [N, hkv, 128], dlambda [N, 4*hkv], dgate [N, 4*hkv, 128].
 * Returns 0, or -1 on a bad argument or an allocation/thread failure.
 */
int gdla_oracle_prefill_bwd(const uint16_t *q_sig, const uint16_t *q_noise, const uint16_t *k, const uint16_t *v,
                            const float *lambda, const uint16_t *gate, const uint16_t *dout, int hkv, int batch,
                            const int32_t *seqlens, int window, double *dq_sig, double *dq_noise, double *dk,
                            double *dv, double *dlambda, double *dgate, int nthreads) {
    if (hkv < 1 || batch < 0 || nthreads < 1) return -1;
    int64_t total = 0;
    long max_len = 0;
    int64_t *seq_start = (int64_t *)malloc(sizeof(int64_t) * (size_t)(batch > 0 ? batch : 1));
    if (!seq_start) return -1;
    for (int b = 0; b < batch; ++b) {
        if (seqlens[b] < 0) { free(seq_start); return -1; }
        seq_start[b] = total;
        total += seqlens[b];
        if (seqlens[b] > max_len) max_len = seqlens[b];
    }
    const int hs = GROUP * hkv;
    memset(dq_sig, 0, sizeof(double) * (size_t)total * hs * DQK);
    memset(dq_noise, 0, sizeof(double) * (size_t)total * hkv * DQK);
    memset(dk, 0, sizeof(double) * (size_t)total * hkv * DQK);
    memset(dv, 0, sizeof(double) * (size_t)total * hkv * DV);
    memset(dlambda, 0, sizeof(double) * (size_t)total * hs);
    memset(dgate, 0, sizeof(double) * (size_t)total * hs * DV);
    bwd_job_t *jobs = (bwd_job_t *)malloc(sizeof(bwd_job_t) * (size_t)nthreads);
    if (!jobs) { free(seq_start); return -1; }
    for (int i = 0; i < nthreads; ++i) {
        bwd_job_t J = {q_sig, q_noise, k, v, gate, dout, lambda, hkv, window, batch, seqlens, seq_start,
                       dq_sig, dq_noise, dk, dv, dlambda, dgate, max_len, nthreads, i};
        jobs[i] = J;
    }
    int rc = run_threads(bwd_worker, jobs, sizeof(bwd_job_t), nthreads);
    free(jobs);
    free(seq_start);
    return rc;
}
