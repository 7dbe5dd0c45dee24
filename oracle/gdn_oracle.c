/*
 * Gated DeltaNet token mixer: plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or helper with the
 * CUDA path.
 *
 * What it computes, token by token, for every packed sequence and every
 * selected value head (sources in brackets):
 *
 *   1. Short causal depthwise convolution of kernel 4 over the q|k|v channels,
 *      then SiLU.  ["Qwen3.8-Flash-Next" (llm-architectures-explained),
 *      "Every architecture field": mixers.linear.conv_kernel = 4;
 *      "Qwen3.8-Flash-Next anatomy" (frontier-model-atlas), "Decoder
 *      microscope": "Short conv: kernel 4"; SiLU from hidden_act, "Raw config
 *      fields" (llm-atlas-9r2).]  Tap i of channel c multiplies x[t-K+1+i];
 *      the K-1 inputs before a sequence start come from conv_state (oldest
 *      first); no bias.
 *   2. q and k L2-normalised per key head: x / sqrt(sum x^2 + l2_eps).
 *   3. Gates per value head h: alpha = exp(-exp(A_log[h]) * softplus(a + dt_bias[h])),
 *      beta = sigmoid(b).  softplus(x) = max(x,0) + log1p(exp(-|x|)).
 *   4. Gated delta rule with a fixed-size state per head ("Decoder microscope":
 *      "Recurrent state ... fixed-size state update rather than a full KV
 *      history"; state kept in float32 by the model, mamba_ssm_dtype, "Raw
 *      config fields" -- here fp64):
 *         S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *         o_t = S_t q_t / sqrt(d_k)
 *      S is d_v x d_k.  Value head h reads key head h / (H_v / H_k)
 *      (16 key heads, 48 value heads: "Every architecture field",
 *      mixers.linear.k_heads / v_heads).
 *   5. Output gated RMSNorm per value head:
 *         out = o * (mean(o^2) + norm_eps)^(-1/2) * w_norm * z * sigmoid(z)
 *      (rms_norm_eps = 1e-6, "Raw config fields").
 *
 * The product S(I - beta k k^T) is expanded as S - beta (S k) k^T: that is the
 * same matrix product written out entry by entry, with no reassociation across
 * tokens.  No blocking, chunking or fusion beyond that.
 *
 * Build: gcc -O2 -fPIC -shared (no -ffast-math) -lpthread -lm.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

typedef struct {
    int n_k_heads, n_v_heads, d_k, d_v, conv_kernel;
    double l2_eps, norm_eps;
} gdn_oracle_config;

typedef struct {
    const gdn_oracle_config* cfg;
    const double *conv_w, *A_log, *dt_bias, *norm_w;
    const void *q, *k, *v, *a, *b, *z;
    int act_dtype;
    const double* conv_state_in;   /* [N][Ctot][K-1] */
    double* rec_state;             /* [N][n_sel][d_v][d_k] in/out */
    const int32_t* cu_seqlens;
    int n_seqs;
    const int32_t* heads;          /* [n_sel] value-head indices */
    int n_sel;
    double* out;                   /* [T][n_sel][d_v] */
    double* o_pre;                 /* [T][n_sel][d_v] or NULL */
    int next_item;
    pthread_mutex_t lock;
} oracle_job;

/* bf16 -> double is exact: the 16 bits are the top half of an IEEE binary32. */
static double load_act(const void* base, int dtype, int64_t idx) {
    if (dtype == ORC_F64) return ((const double*)base)[idx];
    if (dtype == ORC_F32) return (double)((const float*)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double silu(double x) { return x / (1.0 + exp(-x)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double softplus(double x) { return (x > 0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* One (sequence, value head) pair, all of its tokens in order. */
static void run_item(oracle_job* J, int seq, int sel) {
    const gdn_oracle_config* c = J->cfg;
    const int Hk = c->n_k_heads, Hv = c->n_v_heads, dk = c->d_k, dv = c->d_v, K = c->conv_kernel;
    const int h = J->heads[sel];
    const int j = h / (Hv / Hk);
    const int Cq = Hk * dk, Ck = Hk * dk;
    const int Ctot = Cq + Ck + Hv * dv;
    const int64_t t0 = J->cu_seqlens[seq], t1 = J->cu_seqlens[seq + 1];

    /* channels this head reads: q of key head j, k of key head j, v of value head h */
    const int nch = 2 * dk + dv;
    int* chan = (int*)malloc(sizeof(int) * nch);
    for (int i = 0; i < dk; i++) chan[i] = j * dk + i;
    for (int i = 0; i < dk; i++) chan[dk + i] = Cq + j * dk + i;
    for (int i = 0; i < dv; i++) chan[2 * dk + i] = Cq + Ck + h * dv + i;

    /* window[ch][0..K-2] = previous inputs, oldest first */
    double* win = (double*)malloc(sizeof(double) * nch * (K - 1));
    for (int i = 0; i < nch; i++)
        for (int p = 0; p < K - 1; p++)
            win[i * (K - 1) + p] = J->conv_state_in[((int64_t)seq * Ctot + chan[i]) * (K - 1) + p];

    double* y = (double*)malloc(sizeof(double) * nch);      /* conv+SiLU outputs */
    double* S = J->rec_state + ((int64_t)seq * J->n_sel + sel) * dv * dk;
    double* Sk = (double*)malloc(sizeof(double) * dv);
    double* o = (double*)malloc(sizeof(double) * dv);
    const double inv_sqrt_dk = 1.0 / sqrt((double)dk);
    const double A = exp(J->A_log[h]);

    for (int64_t t = t0; t < t1; t++) {
        /* 1. conv + SiLU */
        for (int i = 0; i < nch; i++) {
            double x;
            int ch = chan[i];
            if (i < dk)            x = load_act(J->q, J->act_dtype, t * (int64_t)Cq + ch);
            else if (i < 2 * dk)   x = load_act(J->k, J->act_dtype, t * (int64_t)Ck + (ch - Cq));
            else                   x = load_act(J->v, J->act_dtype, t * (int64_t)(Hv * dv) + (ch - Cq - Ck));
            double acc = 0.0;
            for (int p = 0; p < K - 1; p++) acc += J->conv_w[(int64_t)ch * K + p] * win[i * (K - 1) + p];
            acc += J->conv_w[(int64_t)ch * K + (K - 1)] * x;
            for (int p = 0; p + 1 < K - 1; p++) win[i * (K - 1) + p] = win[i * (K - 1) + p + 1];
            if (K > 1) win[i * (K - 1) + K - 2] = x;
            y[i] = silu(acc);
        }
        double* qh = y;
        double* kh = y + dk;
        double* vh = y + 2 * dk;
        /* 2. L2 norm of q and k */
        double sq = 0.0, sk = 0.0;
        for (int i = 0; i < dk; i++) { sq += qh[i] * qh[i]; sk += kh[i] * kh[i]; }
        double rq = 1.0 / sqrt(sq + c->l2_eps), rk = 1.0 / sqrt(sk + c->l2_eps);
        for (int i = 0; i < dk; i++) { qh[i] *= rq; kh[i] *= rk; }
        /* 3. gates */
        double av = load_act(J->a, J->act_dtype, t * (int64_t)Hv + h);
        double bv = load_act(J->b, J->act_dtype, t * (int64_t)Hv + h);
        double alpha = exp(-A * softplus(av + J->dt_bias[h]));
        double beta = sigmoid(bv);
        /* 4. S <- alpha * (S - beta (S k) k^T) + beta v k^T ;  o = S q / sqrt(dk) */
        for (int r = 0; r < dv; r++) {
            double acc = 0.0;
            for (int i = 0; i < dk; i++) acc += S[(int64_t)r * dk + i] * kh[i];
            Sk[r] = acc;
        }
        for (int r = 0; r < dv; r++) {
            double* Sr = S + (int64_t)r * dk;
            for (int i = 0; i < dk; i++)
                Sr[i] = alpha * (Sr[i] - beta * Sk[r] * kh[i]) + beta * vh[r] * kh[i];
        }
        for (int r = 0; r < dv; r++) {
            double acc = 0.0;
            for (int i = 0; i < dk; i++) acc += S[(int64_t)r * dk + i] * qh[i];
            o[r] = acc * inv_sqrt_dk;
        }
        /* 5. gated RMSNorm */
        double ms = 0.0;
        for (int r = 0; r < dv; r++) ms += o[r] * o[r];
        ms /= (double)dv;
        double rs = 1.0 / sqrt(ms + c->norm_eps);
        int64_t ob = (t * (int64_t)J->n_sel + sel) * dv;
        for (int r = 0; r < dv; r++) {
            double zz = load_act(J->z, J->act_dtype, t * (int64_t)(Hv * dv) + (int64_t)h * dv + r);
            J->out[ob + r] = o[r] * rs * J->norm_w[r] * zz * sigmoid(zz);
            if (J->o_pre) J->o_pre[ob + r] = o[r];
        }
    }
    free(chan); free(win); free(y); free(Sk); free(o);
}

static void* worker(void* arg) {
    oracle_job* J = (oracle_job*)arg;
    const int total = J->n_seqs * J->n_sel;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int it = J->next_item++;
        pthread_mutex_unlock(&J->lock);
        if (it >= total) break;
        run_item(J, it / J->n_sel, it % J->n_sel);
    }
    return NULL;
}

/*
 * Forward pass over packed sequences.
 *   q, k: [T][H_k*d_k]; v, z: [T][H_v*d_v]; a, b: [T][H_v]   (act_dtype)
 *   conv_w [Ctot][K], Ctot = 2*H_k*d_k + H_v*d_v, channel order q|k|v
 *   conv_state [N][Ctot][K-1] in/out (oldest first)
 *   rec_state  [N][n_sel][d_v][d_k] in/out, for value heads heads[0..n_sel)
 *   out, o_pre [T][n_sel][d_v]  (o_pre: output before the gated norm; may be NULL)
 *   heads == NULL selects all value heads in order (n_sel must then be H_v).
 * Returns 0, or -1 on a bad argument.
 */
int gdn_oracle_forward(const gdn_oracle_config* cfg,
                       const double* conv_w, const double* A_log, const double* dt_bias,
                       const double* norm_w,
                       const void* q, const void* k, const void* v,
                       const void* a, const void* b, const void* z, int act_dtype,
                       double* conv_state, double* rec_state,
                       const int32_t* cu_seqlens, int n_seqs,
                       const int32_t* heads, int n_sel,
                       double* out, double* o_pre, int n_threads) {
    if (!cfg || cfg->n_k_heads <= 0 || cfg->n_v_heads % cfg->n_k_heads != 0 || cfg->conv_kernel < 1)
        return -1;
    if (n_seqs < 0 || n_sel < 0) return -1;
    const int Ctot = 2 * cfg->n_k_heads * cfg->d_k + cfg->n_v_heads * cfg->d_v;
    const int K = cfg->conv_kernel;
    int32_t* all = NULL;
    if (!heads) {
        if (n_sel != cfg->n_v_heads) return -1;
        all = (int32_t*)malloc(sizeof(int32_t) * n_sel);
        for (int i = 0; i < n_sel; i++) all[i] = i;
        heads = all;
    }
    for (int i = 0; i < n_sel; i++)
        if (heads[i] < 0 || heads[i] >= cfg->n_v_heads) { free(all); return -1; }

    /* every worker reads the state as it was on entry */
    size_t cs_n = (size_t)n_seqs * Ctot * (K - 1);
    double* cs_in = (double*)malloc(sizeof(double) * (cs_n ? cs_n : 1));
    memcpy(cs_in, conv_state, sizeof(double) * cs_n);

    oracle_job J;
    memset(&J, 0, sizeof J);
    J.cfg = cfg; J.conv_w = conv_w; J.A_log = A_log; J.dt_bias = dt_bias; J.norm_w = norm_w;
    J.q = q; J.k = k; J.v = v; J.a = a; J.b = b; J.z = z; J.act_dtype = act_dtype;
    J.conv_state_in = cs_in; J.rec_state = rec_state; J.cu_seqlens = cu_seqlens; J.n_seqs = n_seqs;
    J.heads = heads; J.n_sel = n_sel; J.out = out; J.o_pre = o_pre;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * n_threads);
    for (int i = 0; i < n_threads; i++) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < n_threads; i++) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);

    /* final conv state of every channel: the last K-1 inputs of the sequence,
       continuing the old state when the sequence is shorter than K-1 */
    const int Cq = cfg->n_k_heads * cfg->d_k;
    const int Cv = cfg->n_v_heads * cfg->d_v;
    for (int s = 0; s < n_seqs; s++) {
        int64_t t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
        for (int ch = 0; ch < Ctot; ch++) {
            double* dst = conv_state + ((int64_t)s * Ctot + ch) * (K - 1);
            const double* src = cs_in + ((int64_t)s * Ctot + ch) * (K - 1);
            for (int p = 0; p < K - 1; p++) {
                int64_t t = t1 - (K - 1) + p;     /* token this slot holds */
                double x;
                if (t >= t0) {
                    if (ch < Cq)            x = load_act(q, act_dtype, t * (int64_t)Cq + ch);
                    else if (ch < 2 * Cq)   x = load_act(k, act_dtype, t * (int64_t)Cq + (ch - Cq));
                    else                    x = load_act(v, act_dtype, t * (int64_t)Cv + (ch - 2 * Cq));
                } else {
                    x = src[(K - 1) - (t0 - t)];  /* t0 - t slots before the start */
                }
                dst[p] = x;
            }
        }
    }
    free(cs_in);
    free(all);
    return 0;
}
