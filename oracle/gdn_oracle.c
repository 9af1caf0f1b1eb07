/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle of the Gated DeltaNet gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library (gated_deltanet_05_b200/) calls,
 * links or includes this file; only the tests, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py use it. It shares no source with the CUDA path.
 *
 * What it computes (joezjh.github.io notes page "Qwen3.8-Flash-Next", section
 * "Gated DeltaNet 核心机制", the four-line update rule): per head, with the state
 * S in R^{d_k x d_v} (the pages' orientation, row index = key dimension),
 *
 *     S~      = alpha_t * S_{t-1}                 (decay first)
 *     e_t     = v_t - S~^T k_t                    (error against the decayed state)
 *     S_t     = S~ + beta_t * k_t e_t^T           (rank-one write of the error)
 *     y_t     = S_t^T (scale * q_t)               (read AFTER the write)
 *
 * token by token, one (sequence, head) chain at a time, in the order of the pages.
 * The `scale` factor multiplies q; the pages use none, so every workload passes 1.
 *
 * The output epilogue (same page, section "GDN 参数化细节", output-gate equation, and
 * the pwwt.cn translation, section 2.1.1, "sigmoid output gate ... zero-centred
 * RMSNorm") is o = sigmoid(z) * RMSNorm(y), with RMSNorm taken per (token, head)
 * over d_v and the zero-centred weight stored as w, multiplying as (1 + w).
 *
 * All arithmetic is IEEE fp64 in the order written; build without -ffast-math.
 * Chains are independent, so they are spread over POSIX threads; each chain's
 * arithmetic is the same whatever the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------ prefill */

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    const int64_t *cu_seqlens;
    int n_seq, H, dk, dv;
    double scale;
    double *y, *S_T;
    /* work distribution */
    int n_threads, tid;
} rec_args;

/* One chain: sequence i, head h. S is d_k x d_v, row-major (S[a*dv + b] = S_{a,b}). */
static void recurrent_chain(const rec_args *A, int i, int h, double *S, double *e, double *qs)
{
    const int H = A->H, dk = A->dk, dv = A->dv;
    const int64_t bos = A->cu_seqlens[i], eos = A->cu_seqlens[i + 1];
    const size_t state_off = ((size_t)i * H + h) * (size_t)dk * dv;

    if (A->S0)
        memcpy(S, A->S0 + state_off, sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t = bos; t < eos; ++t) {
        const double *kt = A->k + ((size_t)t * H + h) * dk;
        const double *qt = A->q + ((size_t)t * H + h) * dk;
        const double *vt = A->v + ((size_t)t * H + h) * dv;
        const double alpha = exp(A->log_alpha[(size_t)t * H + h]);
        const double beta = A->beta[(size_t)t * H + h];

        /* S~ = alpha * S */
        for (int a = 0; a < dk * dv; ++a)
            S[a] *= alpha;
        /* e = v - S~^T k : e_b = v_b - sum_a S~_{a,b} k_a */
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a)
                acc += S[a * dv + b] * kt[a];
            e[b] = vt[b] - acc;
        }
        /* S = S~ + beta k e^T */
        for (int a = 0; a < dk; ++a)
            for (int b = 0; b < dv; ++b)
                S[a * dv + b] += beta * kt[a] * e[b];
        /* y = S^T (scale q) */
        for (int a = 0; a < dk; ++a)
            qs[a] = A->scale * qt[a];
        double *yt = A->y + ((size_t)t * H + h) * dv;
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a)
                acc += S[a * dv + b] * qs[a];
            yt[b] = acc;
        }
    }
    if (A->S_T)
        memcpy(A->S_T + state_off, S, sizeof(double) * dk * dv);
}

static void *recurrent_worker(void *p)
{
    const rec_args *A = (const rec_args *)p;
    double *S = (double *)malloc(sizeof(double) * A->dk * A->dv);
    double *e = (double *)malloc(sizeof(double) * A->dv);
    double *qs = (double *)malloc(sizeof(double) * A->dk);
    if (S && e && qs) {
        const int n_chain = A->n_seq * A->H;
        for (int c = A->tid; c < n_chain; c += A->n_threads)
            recurrent_chain(A, c / A->H, c % A->H, S, e, qs);
    }
    free(S);
    free(e);
    free(qs);
    return NULL;
}

static int resolve_threads(int n_threads, int n_work)
{
    if (n_threads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = n > 0 ? (int)n : 1;
    }
    if (n_threads > n_work)
        n_threads = n_work > 0 ? n_work : 1;
    return n_threads;
}

/*
 * Token recurrence over packed variable-length sequences.
 *   q, k      [N_tok][H][dk]      (N_tok = cu_seqlens[n_seq])
 *   v         [N_tok][H][dv]
 *   log_alpha [N_tok][H]          alpha_t = exp(log_alpha)
 *   beta      [N_tok][H]
 *   S0        [n_seq][H][dk][dv]  or NULL for zeros (the pages' orientation)
 *   y         [N_tok][H][dv]      out
 *   S_T       [n_seq][H][dk][dv]  out, or NULL
 * Returns the number of threads used (>= 1), or -1 on a bad argument.
 */
int gdn_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *S0,
                         const int64_t *cu_seqlens, int n_seq, int H, int dk, int dv,
                         double scale, double *y, double *S_T, int n_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !y || n_seq < 0 || H <= 0 ||
        dk <= 0 || dv <= 0)
        return -1;
    const int n_chain = n_seq * H;
    n_threads = resolve_threads(n_threads, n_chain);
    rec_args *args = (rec_args *)calloc((size_t)n_threads, sizeof(rec_args));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!args || !th) {
        free(args);
        free(th);
        return -1;
    }
    for (int i = 0; i < n_threads; ++i) {
        rec_args a = {q, k, v, log_alpha, beta, S0, cu_seqlens, n_seq, H, dk, dv, scale,
                      y, S_T, n_threads, i};
        args[i] = a;
    }
    for (int i = 1; i < n_threads; ++i)
        pthread_create(&th[i], NULL, recurrent_worker, &args[i]);
    recurrent_worker(&args[0]);
    for (int i = 1; i < n_threads; ++i)
        pthread_join(th[i], NULL);
    free(args);
    free(th);
    return n_threads;
}

/* ------------------------------------------------------------------- decode */

/*
 * One token for each of n_chain = n_seq*H independent chains (same update as above,
 * alpha given directly instead of its log).
 *   q, k [n_chain][dk]; v [n_chain][dv]; alpha, beta [n_chain]
 *   S    [n_chain][dk][dv]  updated in place (the pages' orientation)
 *   y    [n_chain][dv]      out
 */
typedef struct {
    const double *q, *k, *v, *alpha, *beta;
    double *S, *y;
    int n_chain, dk, dv;
    double scale;
    int n_threads, tid;
} dec_args;

static void *decode_worker(void *p)
{
    const dec_args *A = (const dec_args *)p;
    const int dk = A->dk, dv = A->dv;
    double *e = (double *)malloc(sizeof(double) * dv);
    if (!e)
        return NULL;
    for (int c = A->tid; c < A->n_chain; c += A->n_threads) {
        double *S = A->S + (size_t)c * dk * dv;
        const double *kt = A->k + (size_t)c * dk, *qt = A->q + (size_t)c * dk;
        const double *vt = A->v + (size_t)c * dv;
        const double alpha = A->alpha[c], beta = A->beta[c];
        for (int a = 0; a < dk * dv; ++a)
            S[a] *= alpha;
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a)
                acc += S[a * dv + b] * kt[a];
            e[b] = vt[b] - acc;
        }
        for (int a = 0; a < dk; ++a)
            for (int b = 0; b < dv; ++b)
                S[a * dv + b] += beta * kt[a] * e[b];
        double *yt = A->y + (size_t)c * dv;
        for (int b = 0; b < dv; ++b) {
            double acc = 0.0;
            for (int a = 0; a < dk; ++a)
                acc += S[a * dv + b] * (A->scale * qt[a]);
            yt[b] = acc;
        }
    }
    free(e);
    return NULL;
}

int gdn_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *alpha, const double *beta, double *S, double *y,
                           int n_chain, int dk, int dv, double scale, int n_threads)
{
    if (!q || !k || !v || !alpha || !beta || !S || !y || n_chain < 0 || dk <= 0 || dv <= 0)
        return -1;
    n_threads = resolve_threads(n_threads, n_chain);
    dec_args *args = (dec_args *)calloc((size_t)n_threads, sizeof(dec_args));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!args || !th) {
        free(args);
        free(th);
        return -1;
    }
    for (int i = 0; i < n_threads; ++i) {
        dec_args a = {q, k, v, alpha, beta, S, y, n_chain, dk, dv, scale, n_threads, i};
        args[i] = a;
    }
    for (int i = 1; i < n_threads; ++i)
        pthread_create(&th[i], NULL, decode_worker, &args[i]);
    decode_worker(&args[0]);
    for (int i = 1; i < n_threads; ++i)
        pthread_join(th[i], NULL);
    free(args);
    free(th);
    return n_threads;
}

/* ---------------------------------------------------------------- gate-norm */

/*
 * o[r][j] = sigmoid(z[r][j]) * y[r][j] / sqrt(mean_j y[r][j]^2 + eps) * (1 + w[j])
 * for r < n_rows (= N_tok * H), j < dv. Row-local, single threaded.
 */
int gdn_oracle_gate_norm(const double *y, const double *z, const double *w, int64_t n_rows,
                         int dv, double eps, double *o)
{
    if (!y || !z || !w || !o || n_rows < 0 || dv <= 0)
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const double *yr = y + (size_t)r * dv, *zr = z + (size_t)r * dv;
        double ss = 0.0;
        for (int j = 0; j < dv; ++j)
            ss += yr[j] * yr[j];
        const double inv_rms = 1.0 / sqrt(ss / dv + eps);
        for (int j = 0; j < dv; ++j) {
            const double gate = 1.0 / (1.0 + exp(-zr[j]));
            o[(size_t)r * dv + j] = gate * (yr[j] * inv_rms) * (1.0 + w[j]);
        }
    }
    return 1;
}

/* ---------------------------------------------------------------- featurisation */

/*
 * The feature and gate computation in front of the recurrence (joezjh.github.io notes
 * page "Qwen3.8-Flash-Next", section "GDN 参数化细节", the q/k/v equations and the gate
 * equations; pwwt.cn translation, section 2.1.1, Figure 2 caption: a short causal
 * convolution on the projected q, k, v streams, L2 normalisation of q and k only).
 * The projections W x are inputs here (plain GEMMs outside this step):
 *
 *   c_t     = sum_{j < W} w[ch][j] * x_{t - (W-1) + j}     per channel, x = 0 before the
 *                                                           sequence's first token
 *   f_t     = SiLU(c_t) = c_t / (1 + exp(-c_t))
 *   q_t,k_t = f_t / sqrt(sum_ch f_t^2 + eps)               per (token, head), over d
 *   v_t     = f_t
 *   beta_t  = 1 / (1 + exp(-beta_logit_t))
 *   log alpha_t = -exp(A_h) * softplus(alpha_logit_t + b_alpha_h)
 *
 * Tap j of a channel's W weights multiplies the token W-1-j places back (the weight
 * layout of a depthwise PyTorch Conv1d padded by W-1 and cut to its first T outputs).
 * x*, out*: [n_tok][H][d] (d = dk for q, k and dv for v); conv_*: [H*d][W];
 * logits, beta, log_alpha: [n_tok][H]; A, b_alpha: [H]. Single threaded.
 */
static void featurize_stream(const double *x, const double *cw, int W, const int64_t *cu, int n_seq,
                             int H, int d, int l2, double eps, double *out)
{
    for (int i = 0; i < n_seq; ++i)
        for (int64_t t = cu[i]; t < cu[i + 1]; ++t)
            for (int h = 0; h < H; ++h) {
                double *o = out + ((size_t)t * H + h) * d;
                for (int c = 0; c < d; ++c) {
                    const double *w = cw + ((size_t)h * d + c) * W;
                    double acc = 0.0;
                    for (int j = 0; j < W; ++j) {
                        const int64_t s = t - (W - 1) + j;
                        if (s >= cu[i])
                            acc += w[j] * x[((size_t)s * H + h) * d + c];
                    }
                    o[c] = acc / (1.0 + exp(-acc));
                }
                if (l2) {
                    double ss = 0.0;
                    for (int c = 0; c < d; ++c)
                        ss += o[c] * o[c];
                    const double inv = 1.0 / sqrt(ss + eps);
                    for (int c = 0; c < d; ++c)
                        o[c] *= inv;
                }
            }
}

static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

int gdn_oracle_featurize(const double *xq, const double *xk, const double *xv, const double *conv_q,
                         const double *conv_k, const double *conv_v, int W, const double *beta_logit,
                         const double *alpha_logit, const double *A, const double *b_alpha,
                         const int64_t *cu, int n_seq, int H, int dk, int dv, double eps, double *q,
                         double *k, double *v, double *beta, double *log_alpha)
{
    if (!xq || !xk || !xv || !conv_q || !conv_k || !conv_v || !beta_logit || !alpha_logit || !A ||
        !b_alpha || !cu || !q || !k || !v || !beta || !log_alpha || W < 1 || n_seq < 0 || H <= 0 ||
        dk <= 0 || dv <= 0)
        return -1;
    featurize_stream(xq, conv_q, W, cu, n_seq, H, dk, 1, eps, q);
    featurize_stream(xk, conv_k, W, cu, n_seq, H, dk, 1, eps, k);
    featurize_stream(xv, conv_v, W, cu, n_seq, H, dv, 0, eps, v);
    for (int64_t t = cu[0]; t < cu[n_seq]; ++t)
        for (int h = 0; h < H; ++h) {
            const size_t e = (size_t)t * H + h;
            beta[e] = 1.0 / (1.0 + exp(-beta_logit[e]));
            log_alpha[e] = -exp(A[h]) * softplus(alpha_logit[e] + b_alpha[h]);
        }
    return 1;
}

/* ---------------------------------------------------------------- backward */

/*
 * Gradients of the token recurrence above (the reverse-mode adjoint of its four lines,
 * taken step by step in reverse order). Given dy_t = dL/dy_t for every token and
 * dS_T = dL/dS_T for the final state of every sequence (NULL: zero), with G = dL/dS_t
 * carried backwards from G = dS_T:
 *
 *   y_t = S_t^T (scale q_t):       G += scale q_t dy_t^T;   dq_t = scale S_t dy_t
 *   S_t = S~_t + beta_t k_t e_t^T: dbeta_t = k_t^T G e_t;   dk_t = beta_t G e_t;
 *                                  de_t = beta_t G^T k_t;   G~ = G
 *   e_t = v_t - S~_t^T k_t:        dv_t = de_t;   G~ -= k_t de_t^T;   dk_t -= S~_t de_t
 *   S~_t = alpha_t S_{t-1}:        dalpha_t = <G~, S_{t-1}>;   G = alpha_t G~
 *
 * and dlog_alpha_t = alpha_t dalpha_t, dS0 = G after the first token. The states S_t are
 * recomputed forward from a copy kept every kCkpt tokens (the same operations in the same
 * order as the forward pass, so the same values). Layouts as gdn_oracle_recurrent; dS_T,
 * dS0 [n_seq][H][dk][dv] in the pages' orientation. Single threaded.
 */
enum { kCkpt = 64 };

static void forward_step(double *S_out, const double *S_in, const double *kt, const double *vt,
                         double alpha, double beta, int dk, int dv, double *e)
{
    for (int a = 0; a < dk * dv; ++a)
        S_out[a] = alpha * S_in[a];
    for (int b = 0; b < dv; ++b) {
        double acc = 0.0;
        for (int a = 0; a < dk; ++a)
            acc += S_out[a * dv + b] * kt[a];
        e[b] = vt[b] - acc;
    }
    for (int a = 0; a < dk; ++a)
        for (int b = 0; b < dv; ++b)
            S_out[a * dv + b] += beta * kt[a] * e[b];
}

int gdn_oracle_backward(const double *q, const double *k, const double *v, const double *log_alpha,
                        const double *beta, const double *S0, const int64_t *cu, int n_seq, int H,
                        int dk, int dv, double scale, const double *dy, const double *dS_T,
                        double *dq, double *dk_out, double *dv_out, double *dlog_alpha,
                        double *dbeta, double *dS0)
{
    if (!q || !k || !v || !log_alpha || !beta || !cu || !dy || !dq || !dk_out || !dv_out ||
        !dlog_alpha || !dbeta || n_seq < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return -1;
    const size_t SZ = (size_t)dk * dv;
    int64_t max_len = 0;
    for (int i = 0; i < n_seq; ++i)
        if (cu[i + 1] - cu[i] > max_len)
            max_len = cu[i + 1] - cu[i];
    const int64_t n_ck = max_len / kCkpt + 1;
    double *ck = (double *)malloc(sizeof(double) * SZ * (size_t)n_ck);
    double *seg = (double *)malloc(sizeof(double) * SZ * (kCkpt + 1));
    double *G = (double *)malloc(sizeof(double) * SZ);
    double *Gt = (double *)malloc(sizeof(double) * SZ);
    double *e = (double *)malloc(sizeof(double) * dv);
    double *de = (double *)malloc(sizeof(double) * dv);
    int rc = (ck && seg && G && Gt && e && de) ? 1 : -1;
    for (int i = 0; rc > 0 && i < n_seq; ++i)
        for (int h = 0; h < H; ++h) {
            const int64_t bos = cu[i], T = cu[i + 1] - cu[i];
            const size_t soff = ((size_t)i * H + h) * SZ;
            /* forward: keep S at t = 0, kCkpt, 2 kCkpt, ... */
            if (S0)
                memcpy(seg, S0 + soff, sizeof(double) * SZ);
            else
                memset(seg, 0, sizeof(double) * SZ);
            memcpy(ck, seg, sizeof(double) * SZ);
            for (int64_t t = 0; t < T; ++t) {
                const size_t r = (size_t)(bos + t) * H + h;
                forward_step(seg + SZ, seg, k + r * dk, v + r * dv, exp(log_alpha[r]), beta[r], dk, dv, e);
                memcpy(seg, seg + SZ, sizeof(double) * SZ);
                if ((t + 1) % kCkpt == 0)
                    memcpy(ck + (size_t)((t + 1) / kCkpt) * SZ, seg, sizeof(double) * SZ);
            }
            /* backward, one checkpoint segment at a time from the end */
            if (dS_T)
                memcpy(G, dS_T + soff, sizeof(double) * SZ);
            else
                memset(G, 0, sizeof(double) * SZ);
            for (int64_t s0 = (T == 0 ? 0 : (T - 1) / kCkpt * kCkpt); s0 >= 0 && T > 0; s0 -= kCkpt) {
                const int64_t s1 = s0 + kCkpt < T ? s0 + kCkpt : T;
                /* seg[j] = S_{s0 + j}, j = 0 .. s1 - s0 */
                memcpy(seg, ck + (size_t)(s0 / kCkpt) * SZ, sizeof(double) * SZ);
                for (int64_t t = s0; t < s1; ++t) {
                    const size_t r = (size_t)(bos + t) * H + h;
                    forward_step(seg + (size_t)(t - s0 + 1) * SZ, seg + (size_t)(t - s0) * SZ, k + r * dk,
                                 v + r * dv, exp(log_alpha[r]), beta[r], dk, dv, e);
                }
                for (int64_t t = s1 - 1; t >= s0; --t) {
                    const size_t r = (size_t)(bos + t) * H + h;
                    const double *St = seg + (size_t)(t - s0 + 1) * SZ;      /* S_t */
                    const double *Sp = seg + (size_t)(t - s0) * SZ;          /* S_{t-1} */
                    const double *qt = q + r * dk, *kt = k + r * dk, *vt = v + r * dv, *dyt = dy + r * dv;
                    const double alpha = exp(log_alpha[r]), bt = beta[r];
                    double *dqt = dq + r * dk, *dkt = dk_out + r * dk, *dvt = dv_out + r * dv;
                    /* y_t = S_t^T (scale q_t) */
                    for (int a = 0; a < dk; ++a) {
                        double acc = 0.0;
                        for (int b = 0; b < dv; ++b)
                            acc += St[a * dv + b] * dyt[b];
                        dqt[a] = scale * acc;
                    }
                    for (int a = 0; a < dk; ++a)
                        for (int b = 0; b < dv; ++b)
                            G[a * dv + b] += scale * qt[a] * dyt[b];
                    /* e_t and S~_t = alpha S_{t-1} */
                    for (int b = 0; b < dv; ++b) {
                        double acc = 0.0;
                        for (int a = 0; a < dk; ++a)
                            acc += alpha * Sp[a * dv + b] * kt[a];
                        e[b] = vt[b] - acc;
                    }
                    /* S_t = S~_t + beta k e^T */
                    double db = 0.0;
                    for (int a = 0; a < dk; ++a) {
                        double ge = 0.0;
                        for (int b = 0; b < dv; ++b)
                            ge += G[a * dv + b] * e[b];
                        db += kt[a] * ge;
                        dkt[a] = bt * ge;
                    }
                    dbeta[r] = db;
                    for (int b = 0; b < dv; ++b) {
                        double acc = 0.0;
                        for (int a = 0; a < dk; ++a)
                            acc += G[a * dv + b] * kt[a];
                        de[b] = bt * acc;
                        dvt[b] = de[b];
                    }
                    /* e = v - S~^T k */
                    for (int a = 0; a < dk * dv; ++a)
                        Gt[a] = G[a];
                    for (int a = 0; a < dk; ++a) {
                        double sd = 0.0;
                        for (int b = 0; b < dv; ++b) {
                            Gt[a * dv + b] -= kt[a] * de[b];
                            sd += alpha * Sp[a * dv + b] * de[b];
                        }
                        dkt[a] -= sd;
                    }
                    /* S~ = alpha S_{t-1} */
                    double dal = 0.0;
                    for (int a = 0; a < dk * dv; ++a) {
                        dal += Gt[a] * Sp[a];
                        G[a] = alpha * Gt[a];
                    }
                    dlog_alpha[r] = alpha * dal;
                }
            }
            if (dS0)
                memcpy(dS0 + soff, G, sizeof(double) * SZ);
        }
    free(ck);
    free(seg);
    free(G);
    free(Gt);
    free(e);
    free(de);
    return rc;
}
