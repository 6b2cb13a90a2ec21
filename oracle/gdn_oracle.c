/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the Gated DeltaNet token mixer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg load this library. The CUDA library never links or calls it,
 * and this file includes nothing from the CUDA sources.
 *
 * What it computes (sources: "Inside Qwen3.5: a hybrid linear + full attention LLM",
 * romaanj.github.io/study/models/hybrid-attention, sections 2, 4, 5 and the config
 * footnote; "Hybrid Mamba-Transformer MoE", sotaaz.com, the DeltaNet equation in the
 * "Gated DeltaNet" section):
 *
 *   conv   : y[t,c] = SiLU( sum_{j=0..3} w[c][j] * x[t-3+j, c] ), a width-4 depthwise
 *            causal convolution (Qwen3.5 config "conv kernel 4"); positions before a
 *            sequence start read the carried conv state, or zero.
 *   L2     : q <- q / sqrt(|q|^2 + eps), same for k (the page's stabiliser that keeps the
 *            recurrence bounded, section 5).
 *   update : S' = alpha_t * S_{t-1}                      (alpha = exp(g): the forgetting)
 *            S_t = S' + beta_t * (v_t - S' k_t) k_t^T    (the delta rule: predict S k,
 *                                                         write the error along k)
 *            which equals S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 *   output : o_t = scale * S_t q_t                        (o = S q, section 2).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - decay first, then the delta write against the decayed state;
 *   - the output is read after the write;
 *   - eps = 1e-6 inside the square root; scale defaults to 1;
 *   - SiLU z/(1+exp(-z)) after the conv; PyTorch cross-correlation tap order
 *     (w[c][3] multiplies the current token), no bias, zero padding;
 *   - alpha and beta belong to v-heads; v-head h reads k-head h / (Hv/Hk).
 *
 * Layouts (all row-major, fp64):
 *   x, y        [T][Cc]             conv input / output
 *   w           [Cc][4]
 *   conv state  [n_seq][3][Cc]      taps oldest .. newest
 *   q, k        [T][Hk][dk]
 *   v, o        [T][Hv][dv]
 *   g, beta     [T][Hv]
 *   S           [n_seq][Hv][dv][dk] row index = value dimension, column = key dimension
 *   cu_seqlens  int32 [n_seq+1], host memory, cu[0]=0, cu[n_seq]=T; NULL = one sequence.
 *
 * Parallelism: independent (sequence, v-head) chains run on n_threads POSIX threads;
 * inside a chain every operation runs in token order, as written above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ conv + SiLU */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* x value at absolute position s of the sequence that starts at bos; positions before
 * bos come from the carried taps (index 3 + (s - bos)), or are zero. */
static double conv_input(const double* x, int32_t Cc, int64_t bos, int64_t s, int32_t c,
                         const double* taps /* [3][Cc] or NULL */) {
    if (s >= bos) return x[s * (int64_t)Cc + c];
    int64_t j = 3 + (s - bos);
    if (j < 0 || taps == NULL) return 0.0;
    return taps[j * (int64_t)Cc + c];
}

int gdn_oracle_conv1d_silu(const double* x, double* y, int64_t T, int32_t Cc,
                           const double* w, const int32_t* cu_seqlens, int32_t n_seq,
                           const double* state_in, double* state_out) {
    int32_t one_seq[2] = {0, (int32_t)T};
    if (cu_seqlens == NULL) { cu_seqlens = one_seq; n_seq = 1; }
    for (int32_t n = 0; n < n_seq; ++n) {
        int64_t bos = cu_seqlens[n], eos = cu_seqlens[n + 1];
        const double* taps = state_in ? state_in + (int64_t)n * 3 * Cc : NULL;
        for (int64_t t = bos; t < eos; ++t) {
            for (int32_t c = 0; c < Cc; ++c) {
                double z = 0.0;
                for (int j = 0; j < 4; ++j)
                    z += w[(int64_t)c * 4 + j] * conv_input(x, Cc, bos, t - 3 + j, c, taps);
                y[t * (int64_t)Cc + c] = silu(z);
            }
        }
        if (state_out) {
            double* dst = state_out + (int64_t)n * 3 * Cc;
            for (int j = 0; j < 3; ++j)
                for (int32_t c = 0; c < Cc; ++c)
                    dst[j * (int64_t)Cc + c] = conv_input(x, Cc, bos, eos - 3 + j, c, taps);
        }
    }
    return 0;
}

/* ------------------------------------------------------------ delta-rule recurrence */

typedef struct {
    const double *q, *k, *v, *g, *beta, *init;
    double *o, *final_state;
    int64_t T;
    int32_t Hk, Hv, dk, dv, n_seq, l2norm;
    const int32_t* cu;
    double scale, eps;
    int64_t n_chains;
    int64_t next;              /* next chain index to take */
    pthread_mutex_t lock;
} rec_job;

static void l2_normalise(const double* src, double* dst, int32_t d, int32_t on, double eps) {
    if (!on) { memcpy(dst, src, sizeof(double) * (size_t)d); return; }
    double ss = 0.0;
    for (int32_t j = 0; j < d; ++j) ss += src[j] * src[j];
    double inv = 1.0 / sqrt(ss + eps);
    for (int32_t j = 0; j < d; ++j) dst[j] = src[j] * inv;
}

static void run_chain(rec_job* J, int64_t chain) {
    const int32_t n = (int32_t)(chain / J->Hv), h = (int32_t)(chain % J->Hv);
    const int32_t G = J->Hv / J->Hk, hk = h / G;
    const int32_t dk = J->dk, dv = J->dv;
    const int64_t bos = J->cu[n], eos = J->cu[n + 1];
    double* S = (double*)calloc((size_t)dv * dk, sizeof(double));
    double* qh = (double*)malloc(sizeof(double) * (size_t)dk);
    double* kh = (double*)malloc(sizeof(double) * (size_t)dk);
    double* p = (double*)malloc(sizeof(double) * (size_t)dv);
    if (J->init) memcpy(S, J->init + ((int64_t)n * J->Hv + h) * dv * dk, sizeof(double) * (size_t)dv * dk);
    for (int64_t t = bos; t < eos; ++t) {
        l2_normalise(J->q + (t * J->Hk + hk) * dk, qh, dk, J->l2norm, J->eps);
        l2_normalise(J->k + (t * J->Hk + hk) * dk, kh, dk, J->l2norm, J->eps);
        const double* vt = J->v + (t * J->Hv + h) * dv;
        const double alpha = exp(J->g[t * J->Hv + h]);
        const double b = J->beta[t * J->Hv + h];
        /* forget: S' = alpha S */
        for (int64_t e = 0; e < (int64_t)dv * dk; ++e) S[e] *= alpha;
        /* predict: p = S' k */
        for (int32_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int32_t j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * kh[j];
            p[i] = acc;
        }
        /* write the error along k: S = S' + beta (v - p) k^T */
        for (int32_t i = 0; i < dv; ++i) {
            const double err = b * (vt[i] - p[i]);
            for (int32_t j = 0; j < dk; ++j) S[(int64_t)i * dk + j] += err * kh[j];
        }
        /* read out: o = scale * S q */
        double* ot = J->o + (t * J->Hv + h) * dv;
        for (int32_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int32_t j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * qh[j];
            ot[i] = J->scale * acc;
        }
    }
    if (J->final_state)
        memcpy(J->final_state + ((int64_t)n * J->Hv + h) * dv * dk, S, sizeof(double) * (size_t)dv * dk);
    free(S); free(qh); free(kh); free(p);
}

static void* rec_worker(void* arg) {
    rec_job* J = (rec_job*)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t c = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (c >= J->n_chains) break;
        run_chain(J, c);
    }
    return NULL;
}

int gdn_oracle_recurrence(const double* q, const double* k, const double* v,
                          const double* g, const double* beta, double* o,
                          int64_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                          const int32_t* cu_seqlens, int32_t n_seq,
                          const double* initial_state, double* final_state,
                          double scale, int32_t l2norm, double eps, int32_t n_threads) {
    if (Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || dk <= 0 || dv <= 0 || T < 0) return 1;
    int32_t one_seq[2] = {0, (int32_t)T};
    if (cu_seqlens == NULL) { cu_seqlens = one_seq; n_seq = 1; }
    rec_job J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.init = initial_state;
    J.o = o; J.final_state = final_state; J.T = T;
    J.Hk = Hk; J.Hv = Hv; J.dk = dk; J.dv = dv; J.n_seq = n_seq; J.l2norm = l2norm;
    J.cu = cu_seqlens; J.scale = scale; J.eps = eps;
    J.n_chains = (int64_t)n_seq * Hv; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > J.n_chains) n_threads = (int32_t)(J.n_chains > 0 ? J.n_chains : 1);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int32_t started = 0;
    for (int32_t i = 0; i + 1 < n_threads; ++i)
        if (pthread_create(&th[started], NULL, rec_worker, &J) == 0) ++started;
    rec_worker(&J); /* the calling thread works too */
    for (int32_t i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/* ------------------------------------------------------------------- byte counts */

/* Constant per-layer footprint of one sequence: the recurrent matrices (Hv heads of
 * dv x dk, state_bytes each element) plus the conv buffer (channels x taps elements of
 * conv_bytes each). The Qwen3.5-27B page quotes 3 MB + 80 KB = 3,227,648 bytes with fp32
 * state and a bf16 buffer counted at 4 taps (section 6). */
int64_t gdn_oracle_layer_state_bytes(int32_t Hv, int32_t dk, int32_t dv, int32_t state_bytes,
                                     int32_t conv_channels, int32_t conv_taps, int32_t conv_bytes) {
    return (int64_t)Hv * dk * dv * state_bytes + (int64_t)conv_channels * conv_taps * conv_bytes;
}
