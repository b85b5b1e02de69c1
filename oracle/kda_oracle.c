/*
 * kda_oracle.c -- plain, slow, fp64 CPU oracle for the Kimi Delta Attention (KDA) operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this file;
 * only tests/, the smoke check and the bench's CPU-baseline leg use it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (per sequence n, per head h, state S of shape d_k x d_v, row = key channel):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t
 *
 *   - recurrence: "Kimi Linear: redefining long-context inference efficiency" (xugj520.cn),
 *     section "Kimi Delta Attention的技术内核", the recurrent-form state update; the same formula
 *     with the per-channel Diag(alpha_t) appears in the 2025 attention/MoE review (lanjinlin.com.cn),
 *     entry "KLA 25.10 kimi", and its readout o_t = S_t^T q_t is the linear-attention formula
 *     stated there.
 *   - alpha_t = exp(log_alpha_t) per key channel, beta_t a per-head scalar per token.
 *   - the decode step follows the per-token loop of the review's GDN pseudo-code (state decay,
 *     value modification by S'^T k, rank-1 state update with beta, output from the UPDATED state).
 *   - the chunked form follows the explainer's "硬件效率的深度优化" list: chunk-parallel compute
 *     inside a chunk, recurrent state passing between chunks, a WY representation of the
 *     chunk's rank-1 updates and a UT transform (the triangular inverse (I+A)^{-1}).
 *
 * Inputs are float32 arrays (the exact values the GPU receives; bf16 values are exactly
 * representable in float32) and are widened to fp64.  All arithmetic is fp64.
 *
 * Layout: token-major.  q, k, log_alpha: [Ttot][H][dk]; v: [Ttot][H][dv]; beta: [Ttot][H];
 * out: [Ttot][H][dv]; S0 / S_final: [N][H][dk][dv].  Sequence n owns tokens
 * cu_seqlens[n] .. cu_seqlens[n+1]-1.  A regular batch of B sequences of length T is
 * cu_seqlens = {0, T, 2T, ..., BT}.
 *
 * Three independent formulations:
 *   kda_oracle_seq        the recurrence as written, step by step            (the definition)
 *   kda_oracle_bruteforce the dense transition matrix M_t = (I - b k k^T) Diag(a), S = M S + b k v^T
 *   kda_oracle_chunked    the chunk/WY/UT re-association, chunk size C        (exact up to rounding)
 * and kda_oracle_decode_step, one token per sequence, in the review's loop order.
 * kda_oracle_bwd is the reverse-mode derivative of kda_oracle_seq (the training backward pass):
 * the same step differentiated as written, tokens walked backwards, states recomputed from
 * checkpoints.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX3(t, h, c, H, D) (((size_t)(t) * (size_t)(H) + (size_t)(h)) * (size_t)(D) + (size_t)(c))
/* q and k of value head h: head h / (H / Hk) of the Hk q/k heads */
#define QKIDX(J, t, h, c) IDX3(t, (h) / ((J)->H / (J)->Hk), c, (J)->Hk, (J)->dk)

typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double* S0;
    const int64_t* cu_seqlens;
    const int32_t* pair_mask;
    int N, H, dk, dv, C;
    int Hk; /* q/k heads; value head h reads q/k head h / (H / Hk) (grouped heads); Hk = H: one each */
    double *out, *S_final;
    int mode; /* 0 = sequential, 1 = chunked, 2 = brute force */
    int next_pair;
    pthread_mutex_t lock;
    int status;
} job_t;

/* ------------------------------------------------------------------------------------------
 * The definition, one (sequence, head) pair.
 *   S' = Diag(alpha_t) S            (row c scaled by alpha_c = exp(log_alpha_c))
 *   S  = S' - beta k (k^T S') + beta k v^T      ((I - beta k k^T) S' + beta k v^T, expanded)
 *   o  = S^T q
 * ------------------------------------------------------------------------------------------ */
static void pair_seq(const job_t* J, int n, int h, double* S, double* w)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int64_t t0 = J->cu_seqlens[n], t1 = J->cu_seqlens[n + 1];
    for (int64_t t = t0; t < t1; ++t) {
        const float* kt = J->k + QKIDX(J, t, h, 0);
        const float* qt = J->q + QKIDX(J, t, h, 0);
        const float* vt = J->v + IDX3(t, h, 0, H, dv);
        const float* la = J->log_alpha + IDX3(t, h, 0, H, dk);
        const double b = (double)J->beta[(size_t)t * H + h];
        /* S' = Diag(alpha) S */
        for (int c = 0; c < dk; ++c) {
            const double a = exp((double)la[c]);
            for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;
        }
        /* w = k^T S'  (a d_v row vector) */
        for (int j = 0; j < dv; ++j) w[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double kc = (double)kt[c];
            for (int j = 0; j < dv; ++j) w[j] += kc * S[(size_t)c * dv + j];
        }
        /* S = S' - b k w + b k v^T */
        for (int c = 0; c < dk; ++c) {
            const double kc = (double)kt[c];
            for (int j = 0; j < dv; ++j)
                S[(size_t)c * dv + j] += -b * kc * w[j] + b * kc * (double)vt[j];
        }
        /* o = S^T q */
        if (J->out) {
            double* o = J->out + IDX3(t, h, 0, H, dv);
            for (int j = 0; j < dv; ++j) o[j] = 0.0;
            for (int c = 0; c < dk; ++c) {
                const double qc = (double)qt[c];
                for (int j = 0; j < dv; ++j) o[j] += qc * S[(size_t)c * dv + j];
            }
        }
    }
}

/* ------------------------------------------------------------------------------------------
 * Brute force: materialise the dense d_k x d_k transition M_t = (I - b k k^T) Diag(alpha) and
 * apply S = M_t S + b k v^T with a textbook matrix product.  Meant for short sequences.
 * ------------------------------------------------------------------------------------------ */
static void pair_bruteforce(const job_t* J, int n, int h, double* S, double* M, double* S2)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int64_t t0 = J->cu_seqlens[n], t1 = J->cu_seqlens[n + 1];
    for (int64_t t = t0; t < t1; ++t) {
        const float* kt = J->k + QKIDX(J, t, h, 0);
        const float* qt = J->q + QKIDX(J, t, h, 0);
        const float* vt = J->v + IDX3(t, h, 0, H, dv);
        const float* la = J->log_alpha + IDX3(t, h, 0, H, dk);
        const double b = (double)J->beta[(size_t)t * H + h];
        for (int r = 0; r < dk; ++r)
            for (int c = 0; c < dk; ++c) {
                const double id = (r == c) ? 1.0 : 0.0;
                M[(size_t)r * dk + c] = (id - b * (double)kt[r] * (double)kt[c]) * exp((double)la[c]);
            }
        for (int r = 0; r < dk; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += M[(size_t)r * dk + c] * S[(size_t)c * dv + j];
                S2[(size_t)r * dv + j] = acc + b * (double)kt[r] * (double)vt[j];
            }
        memcpy(S, S2, sizeof(double) * (size_t)dk * dv);
        if (J->out) {
            double* o = J->out + IDX3(t, h, 0, H, dv);
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * (double)qt[c];
                o[j] = acc;
            }
        }
    }
}

/* ------------------------------------------------------------------------------------------
 * Chunked form (chunk-parallel inside, recurrent between chunks; WY representation; UT transform).
 * Inside a chunk with start state S0 and local index r = 0..L-1:
 *   g_r      = sum_{i<=r} log_alpha_i                     (per key channel; restarts every chunk)
 *   A[r][i]  = beta_r sum_c k_rc k_ic exp(g_rc - g_ic),  i < r       (strictly lower)
 *   T        = (I + A)^{-1} Diag(beta)                    (UT transform, forward substitution)
 *   Kt[r][c] = k_rc exp(g_rc),  W = T Kt,  Uv = T V       (WY factors)
 *   U        = Uv - W S0                                   (the chunk's corrected values u_r)
 *   o_r      = sum_c q_rc exp(g_rc) S0[c][:] + sum_{i<=r} P[r][i] U[i],
 *              P[r][i] = sum_c q_rc k_ic exp(g_rc - g_ic)
 *   S_end    = Diag(exp(g_last)) S0 + sum_i (k_i * exp(g_last - g_i)) U_i^T
 * Derivation: unrolling the recurrence inside the chunk gives
 *   S_r = Diag(gamma_r) S0 + sum_{i<=r} Diag(gamma_r/gamma_i) k_i u_i^T,  gamma_r = exp(g_r),
 *   u_r = beta_r (v_r - S'_r^T k_r), which is the unit-lower-triangular system
 *   (I + A) U = Diag(beta)(V - Kt S0).
 * ------------------------------------------------------------------------------------------ */
static void pair_chunked(const job_t* J, int n, int h, double* S, double* scratch)
{
    const int H = J->H, dk = J->dk, dv = J->dv, C = J->C;
    const int64_t t0 = J->cu_seqlens[n], t1 = J->cu_seqlens[n + 1];
    double* g = scratch;                          /* C * dk */
    double* A = g + (size_t)C * dk;               /* C * C */
    double* Tm = A + (size_t)C * C;               /* C * C */
    double* W = Tm + (size_t)C * C;               /* C * dk */
    double* Uv = W + (size_t)C * dk;              /* C * dv */
    double* U = Uv + (size_t)C * dv;              /* C * dv */
    double* Snew = U + (size_t)C * dv;            /* dk * dv */
    for (int64_t cs = t0; cs < t1; cs += C) {
        const int L = (int)((t1 - cs) < C ? (t1 - cs) : C);
        /* cumulative log gate */
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int r = 0; r < L; ++r) {
                acc += (double)J->log_alpha[IDX3(cs + r, h, c, H, dk)];
                g[(size_t)r * dk + c] = acc;
            }
        }
        /* A (strictly lower) */
        for (int r = 0; r < L; ++r) {
            const double br = (double)J->beta[(size_t)(cs + r) * H + h];
            for (int i = 0; i < L; ++i) {
                double acc = 0.0;
                if (i < r)
                    for (int c = 0; c < dk; ++c)
                        acc += (double)J->k[QKIDX(J, cs + r, h, c)] * (double)J->k[QKIDX(J, cs + i, h, c)] *
                               exp(g[(size_t)r * dk + c] - g[(size_t)i * dk + c]);
                A[(size_t)r * C + i] = br * acc;
            }
        }
        /* T = (I + A)^{-1} Diag(beta): row r of (I+A) T = Diag(beta) gives
           T[r][j] = beta_r [r==j] - sum_{i<r} A[r][i] T[i][j] */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < L; ++j) {
                double acc = (r == j) ? (double)J->beta[(size_t)(cs + r) * H + h] : 0.0;
                for (int i = 0; i < r; ++i) acc -= A[(size_t)r * C + i] * Tm[(size_t)i * C + j];
                Tm[(size_t)r * C + j] = acc;
            }
        /* W = T Kt, Uv = T V */
        for (int r = 0; r < L; ++r) {
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int i = 0; i < L; ++i)
                    acc += Tm[(size_t)r * C + i] * (double)J->k[QKIDX(J, cs + i, h, c)] * exp(g[(size_t)i * dk + c]);
                W[(size_t)r * dk + c] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < L; ++i) acc += Tm[(size_t)r * C + i] * (double)J->v[IDX3(cs + i, h, j, H, dv)];
                Uv[(size_t)r * dv + j] = acc;
            }
        }
        /* U = Uv - W S0 */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = Uv[(size_t)r * dv + j];
                for (int c = 0; c < dk; ++c) acc -= W[(size_t)r * dk + c] * S[(size_t)c * dv + j];
                U[(size_t)r * dv + j] = acc;
            }
        /* outputs */
        if (J->out) {
            for (int r = 0; r < L; ++r) {
                double* o = J->out + IDX3(cs + r, h, 0, H, dv);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c)
                        acc += (double)J->q[QKIDX(J, cs + r, h, c)] * exp(g[(size_t)r * dk + c]) * S[(size_t)c * dv + j];
                    o[j] = acc;
                }
                for (int i = 0; i <= r; ++i) {
                    double p = 0.0;
                    for (int c = 0; c < dk; ++c)
                        p += (double)J->q[QKIDX(J, cs + r, h, c)] * (double)J->k[QKIDX(J, cs + i, h, c)] *
                             exp(g[(size_t)r * dk + c] - g[(size_t)i * dk + c]);
                    for (int j = 0; j < dv; ++j) o[j] += p * U[(size_t)i * dv + j];
                }
            }
        }
        /* state at the chunk end */
        const double* glast = g + (size_t)(L - 1) * dk;
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < dv; ++j) {
                double acc = exp(glast[c]) * S[(size_t)c * dv + j];
                for (int i = 0; i < L; ++i)
                    acc += (double)J->k[QKIDX(J, cs + i, h, c)] * exp(glast[c] - g[(size_t)i * dk + c]) *
                           U[(size_t)i * dv + j];
                Snew[(size_t)c * dv + j] = acc;
            }
        memcpy(S, Snew, sizeof(double) * (size_t)dk * dv);
    }
}

static void* worker(void* arg)
{
    job_t* J = (job_t*)arg;
    const int dk = J->dk, dv = J->dv, C = J->C > 0 ? J->C : 1;
    const size_t sz = (size_t)dk * dv;
    size_t extra;
    if (J->mode == 0) extra = (size_t)dv;
    else if (J->mode == 2) extra = (size_t)dk * dk + sz;
    else extra = (size_t)C * dk * 2 + (size_t)C * C * 2 + (size_t)C * dv * 2 + sz;
    double* S = (double*)malloc(sizeof(double) * (sz + extra));
    if (!S) {
        pthread_mutex_lock(&J->lock);
        J->status = -2;
        pthread_mutex_unlock(&J->lock);
        return NULL;
    }
    double* work = S + sz;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int p = J->next_pair++;
        pthread_mutex_unlock(&J->lock);
        if (p >= J->N * J->H) break;
        if (J->pair_mask && !J->pair_mask[p]) continue;
        const int n = p / J->H, h = p % J->H;
        if (J->S0) memcpy(S, J->S0 + (size_t)p * sz, sizeof(double) * sz);
        else memset(S, 0, sizeof(double) * sz);
        if (J->mode == 0) pair_seq(J, n, h, S, work);
        else if (J->mode == 2) pair_bruteforce(J, n, h, S, work, work + (size_t)dk * dk);
        else pair_chunked(J, n, h, S, work);
        if (J->S_final) memcpy(J->S_final + (size_t)p * sz, S, sizeof(double) * sz);
    }
    free(S);
    return NULL;
}

static int run(job_t* J, int num_threads)
{
    if (!J->q || !J->k || !J->v || !J->log_alpha || !J->beta || !J->cu_seqlens) return -1;
    if (J->N < 0 || J->H <= 0 || J->dk <= 0 || J->dv <= 0) return -1;
    if (J->Hk <= 0 || J->H % J->Hk != 0) return -1;
    for (int n = 0; n < J->N; ++n)
        if (J->cu_seqlens[n + 1] < J->cu_seqlens[n]) return -1;
    if (num_threads < 1) num_threads = 1;
    J->next_pair = 0;
    J->status = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)num_threads);
    int started = 0;
    for (int i = 0; i < num_threads; ++i)
        if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->status;
}

#define FILL_JOB(J, mode_, C_)                                                                    \
    job_t J;                                                                                      \
    memset(&J, 0, sizeof(J));                                                                     \
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;                \
    J.cu_seqlens = cu_seqlens; J.pair_mask = pair_mask; J.N = N; J.H = H; J.dk = dk; J.dv = dv;   \
    J.C = (C_); J.out = out; J.S_final = S_final; J.mode = (mode_); J.Hk = H;

/* The definition (sequential recurrence).  pair_mask: [N*H] (index n*H+h), nonzero = compute
 * that pair, NULL = all pairs.  Returns 0 on success, -1 on bad arguments, -2 out of memory. */
int kda_oracle_seq(const float* q, const float* k, const float* v, const float* log_alpha, const float* beta,
                   const double* S0, const int64_t* cu_seqlens, int N, int H, int dk, int dv, double* out,
                   double* S_final, const int32_t* pair_mask, int num_threads)
{
    FILL_JOB(J, 0, 1);
    return run(&J, num_threads);
}

/* Dense transition-matrix form; for short sequences only. */
int kda_oracle_bruteforce(const float* q, const float* k, const float* v, const float* log_alpha,
                          const float* beta, const double* S0, const int64_t* cu_seqlens, int N, int H, int dk,
                          int dv, double* out, double* S_final, const int32_t* pair_mask, int num_threads)
{
    FILL_JOB(J, 2, 1);
    return run(&J, num_threads);
}

/* Chunked WY/UT form with chunk size C >= 1. */
int kda_oracle_chunked(const float* q, const float* k, const float* v, const float* log_alpha, const float* beta,
                       const double* S0, const int64_t* cu_seqlens, int N, int H, int dk, int dv, double* out,
                       double* S_final, const int32_t* pair_mask, int C, int num_threads)
{
    if (C < 1) return -1;
    FILL_JOB(J, 1, C);
    return run(&J, num_threads);
}

/* Grouped q/k heads: q and k are [Ttot][Hk][dk] and value head h reads q/k head h / (H / Hk);
 * v, log_alpha, beta, out and the states keep their H heads.  Hk = H is kda_oracle_seq /
 * kda_oracle_chunked. */
int kda_oracle_seq_grouped(const float* q, const float* k, const float* v, const float* log_alpha,
                           const float* beta, const double* S0, const int64_t* cu_seqlens, int N, int H, int Hk,
                           int dk, int dv, double* out, double* S_final, const int32_t* pair_mask, int num_threads)
{
    FILL_JOB(J, 0, 1);
    J.Hk = Hk;
    return run(&J, num_threads);
}

int kda_oracle_chunked_grouped(const float* q, const float* k, const float* v, const float* log_alpha,
                               const float* beta, const double* S0, const int64_t* cu_seqlens, int N, int H, int Hk,
                               int dk, int dv, double* out, double* S_final, const int32_t* pair_mask, int C,
                               int num_threads)
{
    if (C < 1) return -1;
    FILL_JOB(J, 1, C);
    J.Hk = Hk;
    return run(&J, num_threads);
}

/* One decode step for N independent sequences, in the loop order of the review's pseudo-code:
 *   (a) decay       S' = S * exp(log_alpha)    (row c scaled)
 *   (b) delta       d  = S'^T k,   v_mod = v - d
 *   (c) update      S  = S' + k (beta v_mod)^T
 *   (d) output      o  = S^T q                  (from the updated state)
 * q, k: [N][Hk][dk] (value head h reads q/k head h / (H / Hk)); log_alpha: [N][H][dk]; v: [N][H][dv];
 * beta: [N][H]; S: [N][H][dk][dv] in/out; out: [N][H][dv]. */
int kda_oracle_decode_step_grouped(const float* q, const float* k, const float* v, const float* log_alpha,
                                   const float* beta, double* S, int N, int H, int Hk, int dk, int dv, double* out)
{
    if (!q || !k || !v || !log_alpha || !beta || !S || N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (Hk <= 0 || H % Hk != 0) return -1;
    double* d = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!d) return -2;
    for (int p = 0; p < N * H; ++p) {
        double* Sp = S + (size_t)p * dk * dv;
        const size_t pk = (size_t)(p / H) * Hk + (size_t)((p % H) / (H / Hk));  /* q/k head of pair p */
        const float* kp = k + pk * dk;
        const float* qp = q + pk * dk;
        const float* vp = v + (size_t)p * dv;
        const float* lp = log_alpha + (size_t)p * dk;
        const double b = (double)beta[p];
        for (int c = 0; c < dk; ++c) {
            const double a = exp((double)lp[c]);
            for (int j = 0; j < dv; ++j) Sp[(size_t)c * dv + j] *= a;
        }
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += Sp[(size_t)c * dv + j] * (double)kp[c];
            d[j] = (double)vp[j] - acc; /* v_mod */
        }
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < dv; ++j) Sp[(size_t)c * dv + j] += (double)kp[c] * (b * d[j]);
        if (out)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += (double)qp[c] * Sp[(size_t)c * dv + j];
                out[(size_t)p * dv + j] = acc;
            }
    }
    free(d);
    return 0;
}

/* Hk = H: one q/k head per value head. */
int kda_oracle_decode_step(const float* q, const float* k, const float* v, const float* log_alpha,
                           const float* beta, double* S, int N, int H, int dk, int dv, double* out)
{
    return kda_oracle_decode_step_grouped(q, k, v, log_alpha, beta, S, N, H, H, dk, dv, out);
}

/* ==========================================================================================
 * Backward pass (reverse-mode derivative of the recurrence), for a scalar loss
 *     f = sum_t <dout_t, o_t> + <dS_final, S_final>
 * given the cotangents dout ([Ttot][H][dv]) and dS_final ([N][H][dk][dv], or NULL = 0).
 * Returns df/dq, df/dk ([Ttot][H][dk], one entry per VALUE head), df/dv, df/dlog_alpha,
 * df/dbeta and df/dS0.
 *
 * The forward step, written the way the derivative is taken (the same update as pair_seq):
 *   M   = Diag(alpha_t) S_{t-1}                 (alpha = exp(log_alpha), row c scaled)
 *   w   = M^T k_t,   u = beta_t (v_t - w)       (u: the corrected value written at step t)
 *   S_t = M + k_t u^T                           (= (I - beta k k^T) M + beta k v^T)
 *   o_t = S_t^T q_t
 * Walking t backwards with G = df/dS_t (starting from dS_final):
 *   G    += q_t dout_t^T,          dq_t = S_t dout_t
 *   du    = G^T k_t,               dk_t = G u
 *   dbeta = du . (v_t - w),        dv_t = beta du,        dw = -beta du
 *   dk_t += M dw,                  dM   = G + k_t dw^T
 *   dlog_alpha_c = alpha_c sum_j dM[c][j] S_{t-1}[c][j],  G <- Diag(alpha) dM   (= df/dS_{t-1})
 * The states S_{t-1}, S_t are recomputed forward from checkpoints kept every kBwdSeg steps, so
 * memory stays O(T/kBwdSeg + kBwdSeg) states per pair whatever the sequence length.
 * ========================================================================================== */
#define kBwdSeg 64

typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double *S0, *dout, *dS_final;
    const int64_t* cu_seqlens;
    const int32_t* pair_mask;
    int N, H, dk, dv;
    double *dq, *dk_, *dv_, *dla, *dbeta, *dS0;
    int next_pair;
    pthread_mutex_t lock;
    int status;
} bjob_t;

/* one forward step S <- step(S) at token t of head h (the update of pair_seq, outputs omitted) */
static void bwd_step_fwd(const bjob_t* J, int64_t t, int h, double* S, double* w)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const float* kt = J->k + IDX3(t, h, 0, H, dk);
    const float* vt = J->v + IDX3(t, h, 0, H, dv);
    const float* la = J->log_alpha + IDX3(t, h, 0, H, dk);
    const double b = (double)J->beta[(size_t)t * H + h];
    for (int c = 0; c < dk; ++c) {
        const double a = exp((double)la[c]);
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;
    }
    for (int j = 0; j < dv; ++j) w[j] = 0.0;
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) w[j] += (double)kt[c] * S[(size_t)c * dv + j];
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += (double)kt[c] * b * ((double)vt[j] - w[j]);
}

static void pair_bwd(const bjob_t* J, int n, int h, double* ck, double* seg, double* G, double* M, double* w,
                     double* du)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const size_t sz = (size_t)dk * dv;
    const size_t p = (size_t)n * H + h;
    const int64_t t0 = J->cu_seqlens[n], t1 = J->cu_seqlens[n + 1];
    const int64_t nseg = (t1 - t0 + kBwdSeg - 1) / kBwdSeg;
    /* checkpoints: ck[s] = state before token t0 + s * kBwdSeg */
    double* S = seg;
    if (J->S0) memcpy(S, J->S0 + p * sz, sizeof(double) * sz);
    else memset(S, 0, sizeof(double) * sz);
    for (int64_t s = 0; s < nseg; ++s) {
        memcpy(ck + (size_t)s * sz, S, sizeof(double) * sz);
        const int64_t e = (t0 + (s + 1) * kBwdSeg < t1) ? t0 + (s + 1) * kBwdSeg : t1;
        for (int64_t t = t0 + s * kBwdSeg; t < e; ++t) bwd_step_fwd(J, t, h, S, w);
    }
    /* G = df/dS_final */
    if (J->dS_final) memcpy(G, J->dS_final + p * sz, sizeof(double) * sz);
    else memset(G, 0, sizeof(double) * sz);
    for (int64_t s = nseg - 1; s >= 0; --s) {
        const int64_t ts = t0 + s * kBwdSeg;
        const int64_t e = (ts + kBwdSeg < t1) ? ts + kBwdSeg : t1;
        /* seg[i] = state before token ts + i, i = 0 .. e - ts */
        memcpy(seg, ck + (size_t)s * sz, sizeof(double) * sz);
        for (int64_t t = ts; t < e; ++t) {
            memcpy(seg + (size_t)(t - ts + 1) * sz, seg + (size_t)(t - ts) * sz, sizeof(double) * sz);
            bwd_step_fwd(J, t, h, seg + (size_t)(t - ts + 1) * sz, w);
        }
        for (int64_t t = e - 1; t >= ts; --t) {
            const double* Sp = seg + (size_t)(t - ts) * sz;     /* S_{t-1} */
            const double* St = seg + (size_t)(t - ts + 1) * sz; /* S_t */
            const float* qt = J->q + IDX3(t, h, 0, H, dk);
            const float* kt = J->k + IDX3(t, h, 0, H, dk);
            const float* vt = J->v + IDX3(t, h, 0, H, dv);
            const float* la = J->log_alpha + IDX3(t, h, 0, H, dk);
            const double* dot = J->dout + IDX3(t, h, 0, H, dv);
            const double b = (double)J->beta[(size_t)t * H + h];
            double* dqt = J->dq + IDX3(t, h, 0, H, dk);
            double* dkt = J->dk_ + IDX3(t, h, 0, H, dk);
            double* dvt = J->dv_ + IDX3(t, h, 0, H, dv);
            double* dlat = J->dla + IDX3(t, h, 0, H, dk);
            /* readout o_t = S_t^T q_t */
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    G[(size_t)c * dv + j] += (double)qt[c] * dot[j];
                    acc += St[(size_t)c * dv + j] * dot[j];
                }
                dqt[c] = acc;
            }
            /* M = Diag(alpha) S_{t-1},  w = M^T k,  u = beta (v - w) */
            for (int c = 0; c < dk; ++c) {
                const double a = exp((double)la[c]);
                for (int j = 0; j < dv; ++j) M[(size_t)c * dv + j] = a * Sp[(size_t)c * dv + j];
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += M[(size_t)c * dv + j] * (double)kt[c];
                w[j] = acc;
            }
            /* S_t = M + k u^T */
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += G[(size_t)c * dv + j] * (double)kt[c];
                du[j] = acc;                               /* du = G^T k */
                db += acc * ((double)vt[j] - w[j]);        /* u = beta (v - w) */
                dvt[j] = b * acc;
            }
            J->dbeta[(size_t)t * H + h] = db;
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0, acc2 = 0.0;
                for (int j = 0; j < dv; ++j) {
                    acc += G[(size_t)c * dv + j] * b * ((double)vt[j] - w[j]);  /* G u */
                    acc2 += M[(size_t)c * dv + j] * (-b * du[j]);               /* M dw */
                }
                dkt[c] = acc + acc2;
            }
            /* dM = G + k dw^T, then the decay */
            for (int c = 0; c < dk; ++c) {
                const double a = exp((double)la[c]);
                double da = 0.0;
                for (int j = 0; j < dv; ++j) {
                    const double dm = G[(size_t)c * dv + j] + (double)kt[c] * (-b * du[j]);
                    da += dm * Sp[(size_t)c * dv + j];
                    G[(size_t)c * dv + j] = a * dm;
                }
                dlat[c] = a * da;
            }
        }
    }
    if (J->dS0) memcpy(J->dS0 + p * sz, G, sizeof(double) * sz);
}

static void* bwd_worker(void* arg)
{
    bjob_t* J = (bjob_t*)arg;
    const int dk = J->dk, dv = J->dv;
    const size_t sz = (size_t)dk * dv;
    int64_t maxlen = 0;
    for (int n = 0; n < J->N; ++n)
        if (J->cu_seqlens[n + 1] - J->cu_seqlens[n] > maxlen) maxlen = J->cu_seqlens[n + 1] - J->cu_seqlens[n];
    const size_t nck = (size_t)((maxlen + kBwdSeg - 1) / kBwdSeg) + 1;
    double* buf = (double*)malloc(sizeof(double) * (sz * (nck + kBwdSeg + 1 + 2) + 2 * (size_t)dv));
    if (!buf) {
        pthread_mutex_lock(&J->lock);
        J->status = -2;
        pthread_mutex_unlock(&J->lock);
        return NULL;
    }
    double* ck = buf;
    double* seg = ck + sz * nck;
    double* G = seg + sz * (kBwdSeg + 1);
    double* M = G + sz;
    double* w = M + sz;
    double* du = w + dv;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int p = J->next_pair++;
        pthread_mutex_unlock(&J->lock);
        if (p >= J->N * J->H) break;
        if (J->pair_mask && !J->pair_mask[p]) continue;
        pair_bwd(J, p / J->H, p % J->H, ck, seg, G, M, w, du);
    }
    free(buf);
    return NULL;
}

/* Backward of kda_oracle_seq (one q/k head per value head).  Inputs as kda_oracle_seq plus
 * dout [Ttot][H][dv] and dS_final [N][H][dk][dv] (NULL = 0); outputs (all fp64, caller-owned):
 * dq, dk [Ttot][H][dk], dv [Ttot][H][dv], dlog_alpha [Ttot][H][dk], dbeta [Ttot][H],
 * dS0 [N][H][dk][dv] (NULL = not wanted).  Pairs outside pair_mask are left untouched.
 * Returns 0, -1 on bad arguments, -2 out of memory. */
int kda_oracle_bwd(const float* q, const float* k, const float* v, const float* log_alpha, const float* beta,
                   const double* S0, const double* dout, const double* dS_final, const int64_t* cu_seqlens, int N,
                   int H, int dk, int dv, double* dq, double* dk_out, double* dv_out, double* dlog_alpha,
                   double* dbeta, double* dS0, const int32_t* pair_mask, int num_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || !dout || !cu_seqlens) return -1;
    if (!dq || !dk_out || !dv_out || !dlog_alpha || !dbeta) return -1;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    bjob_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta;
    J.S0 = S0; J.dout = dout; J.dS_final = dS_final; J.cu_seqlens = cu_seqlens; J.pair_mask = pair_mask;
    J.N = N; J.H = H; J.dk = dk; J.dv = dv;
    J.dq = dq; J.dk_ = dk_out; J.dv_ = dv_out; J.dla = dlog_alpha; J.dbeta = dbeta; J.dS0 = dS0;
    if (num_threads < 1) num_threads = 1;
    pthread_mutex_init(&J.lock, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)num_threads);
    int started = 0;
    if (th)
        for (int i = 0; i < num_threads; ++i)
            if (pthread_create(&th[i], NULL, bwd_worker, &J) == 0) ++started;
    if (started == 0) bwd_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return J.status;
}
