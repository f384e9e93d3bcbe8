/*
 * dg_oracle.c -- ORACLE: plain, slow, fp64 CPU definition of one denoising step of a
 * block-autoregressive, uniform-state text-diffusion decoder (a Gemma-4-26B-A4B-shaped MoE).
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark may load it.  It shares no source, header, table or helper with the CUDA path.
 *
 * Sources (web pages about DiffusionGemma, cited by title and section):
 *   [guide]  "diffusion-gemma developer guide" (aisparkup.com wiki): sections "256-token Canvas
 *            parallel generation", "Uniform State Diffusion", "Block Autoregressive Diffusion",
 *            "Dual attention of prefill and denoising", "Serving with vLLM".
 *   [report] "DiffusionGemma: a diffusion LLM that refines 256-token blocks in parallel"
 *            (42jerrykim.github.io, a summary of the technical report): section "Composition of
 *            DiffusionGemma" (flowchart, training recipe, sampler settings).
 *   [news]   "DiffusionGemma: 4x faster text generation" (news.hada.io summary of the Google post).
 *   [philox] J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
 *            SC'11 -- definition of the Philox4x32-10 counter-based generator.
 *
 * The pages fix only: canvas of 256 positions, at most 48 denoising steps, temperature decaying
 * linearly 0.8 -> 0.4, entropy bound 0.1 for committing a position, adaptive-stop threshold 0.005,
 * uniform random placeholder start, re-randomisation of low-confidence positions, bidirectional
 * attention inside the canvas with the prompt/committed blocks held as cache, and commit of a
 * finished block to the KV cache.  Every other detail below is the plainest standard reading
 * (pre-norm residual block, RMSNorm, NeoX RoPE, GQA, top-k softmax router, SwiGLU experts); each
 * such reading is stated where it is used.
 *
 * Everything is computed in fp64.  Weights arrive as bf16 bit patterns (upcast exactly) or as
 * e4m3 bytes with one fp32 scale per 128x128 tile (dequantised exactly to q*s).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* number formats                                                                              */
/* ------------------------------------------------------------------------------------------ */

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite magnitude 448. */
double orc_e4m3_to_double(uint8_t q)
{
    int sign = (q >> 7) & 1, e = (q >> 3) & 15, m = q & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* The 256 decoded e4m3 values, filled once when the library loads (a table of orc_e4m3_to_double,
 * so that expanding FP8 weight rows costs a lookup per element). */
static double e4m3_value[256];

__attribute__((constructor)) static void fill_e4m3_table(void)
{
    for (int q = 0; q < 256; ++q)
        e4m3_value[q] = orc_e4m3_to_double((uint8_t)q);
}

/* A weight matrix [rows][cols], row-major: bf16 bits, or e4m3 bytes with one fp32 scale per
 * 128x128 tile (scale index [r/128][c/128], row-major over ceil(cols/128) tiles). */
typedef struct {
    const uint16_t *bf16;
    const uint8_t *e4m3;
    const float *scale;
    int rows, cols;
} orc_mat;

static void mat_row(const orc_mat *w, int r, double *out)
{
    if (w->bf16) {
        const uint16_t *p = w->bf16 + (size_t)r * w->cols;
        for (int c = 0; c < w->cols; ++c)
            out[c] = bf16_bits_to_double(p[c]);
    } else {
        const uint8_t *p = w->e4m3 + (size_t)r * w->cols;
        int tiles_c = (w->cols + 127) / 128;
        for (int c = 0; c < w->cols; ++c)
            out[c] = e4m3_value[p[c]] * (double)w->scale[(size_t)(r / 128) * tiles_c + c / 128];
    }
}

/* out[t][r] = sum_c W[r][c] * x[t][c] for t < n_tok (plain definition of x W^T). */
static void mat_apply(const orc_mat *w, int n_tok, const double *x, double *out, int out_stride)
{
    #pragma omp parallel
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)w->cols);
        #pragma omp for schedule(static)
        for (int r = 0; r < w->rows; ++r) {
            mat_row(w, r, row);
            for (int t = 0; t < n_tok; ++t) {
                const double *xt = x + (size_t)t * w->cols;
                double acc = 0.0;
                for (int c = 0; c < w->cols; ++c)
                    acc += row[c] * xt[c];
                out[(size_t)t * out_stride + r] = acc;
            }
        }
        free(row);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Philox4x32-10 [philox]: 10 rounds of the 4-word Philox S-box with multipliers 0xD2511F53,    */
/* 0xCD9E8D57 and Weyl key increments 0x9E3779B9, 0xBB67AE85.                                   */
/* ------------------------------------------------------------------------------------------ */

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {            /* key schedule: bump by the Weyl constants between rounds */
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;   /* multiplies word 0 */
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;   /* multiplies word 2 */
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The sampler's random stream (a reading; the pages name no generator): key = the 64-bit seed
 * split low/high; counter = (v/4, absolute position, step, tag); word v mod 4.
 * tag 0 = Gumbel noise, tag 1 = re-randomisation, tag 2 = canvas initialisation. */
uint32_t orc_rng_word(uint64_t seed, uint32_t c0, uint32_t pos, uint32_t step, uint32_t tag, int word)
{
    uint32_t ctr[4] = {c0, pos, step, tag}, key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)}, out[4];
    orc_philox4x32_10(ctr, key, out);
    return out[word & 3];
}

/* uniform on the open interval: (2*(x>>9)+1) * 2^-24, in [2^-24, 1-2^-24], exact in fp32 */
double orc_uniform(uint32_t x)
{
    return (2.0 * (double)(x >> 9) + 1.0) * ldexp(1.0, -24);
}

/* standard Gumbel variate -ln(-ln u) */
double orc_gumbel(uint32_t x)
{
    return -log(-log(orc_uniform(x)));
}

/* uniform token id in [0, V): floor(x * V / 2^32) */
int32_t orc_token_from_word(uint32_t x, uint32_t vocab)
{
    return (int32_t)(((uint64_t)x * (uint64_t)vocab) >> 32);
}

/* ------------------------------------------------------------------------------------------ */
/* Sampler schedule [report, "Composition", sampler settings]: temperature decays linearly      */
/* from t_start (0.8) to t_end (0.4) over the maximum step budget (48), step s counted from 0.    */
/* Reading: the schedule spans the 48-step budget even when a block stops earlier; the value    */
/* handed to the sampler is rounded to fp32.                                                    */
/* ------------------------------------------------------------------------------------------ */

float orc_temperature(int s, int max_steps, float t_start, float t_end)
{
    double frac = max_steps > 1 ? (double)s / (double)(max_steps - 1) : 0.0;
    return (float)((double)t_start - ((double)t_start - (double)t_end) * frac);
}

/* ------------------------------------------------------------------------------------------ */
/* Model pieces                                                                                */
/* ------------------------------------------------------------------------------------------ */

/* RMSNorm: x / sqrt(mean(x^2) + eps) * g  (plain reading of "Gemma-style" pre-norm; gain g) */
void orc_rmsnorm(int n, int d, const double *x, const float *g, double eps, double *out)
{
    for (int t = 0; t < n; ++t) {
        const double *xt = x + (size_t)t * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j)
            ss += xt[j] * xt[j];
        double r = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j)
            out[(size_t)t * d + j] = xt[j] * r * (double)g[j];
    }
}

/* RoPE, NeoX half-split: for i < dh/2 the pair (i, i + dh/2) is rotated by angle
 * pos * theta^(-2i/dh).  x is [n_tok][n_head][dh], rotated in place. */
void orc_rope(int n_tok, int n_head, int dh, const int32_t *pos, double theta, double *x)
{
    int half = dh / 2;
    for (int t = 0; t < n_tok; ++t)
        for (int h = 0; h < n_head; ++h) {
            double *v = x + ((size_t)t * n_head + h) * dh;
            for (int i = 0; i < half; ++i) {
                double ang = (double)pos[t] * pow(theta, -2.0 * i / dh);
                double c = cos(ang), s = sin(ang);
                double a = v[i], b = v[i + half];
                v[i] = a * c - b * s;
                v[i + half] = b * c + a * s;
            }
        }
}

/* Masked multi-head attention, plain definition with an explicit mask matrix:
 *   out[i][h] = sum_j p_ij v[j][h'] , p_i = softmax_j( q[i][h].k[j][h'] / sqrt(dh) ) over the
 *   keys j with mask[i][j] = 1, where h' = floor(h * n_kv / n_q) (grouped-query attention).
 * q [n_rows][n_q][dh], k,v [n_keys][n_kv][dh], mask [n_rows][n_keys], out [n_rows][n_q][dh].
 * A row with no visible key gets zeros. */
void orc_attention(int n_rows, int n_keys, int n_q, int n_kv, int dh, const double *q,
                   const double *k, const double *v, const uint8_t *mask, double *out)
{
    double scale = 1.0 / sqrt((double)dh);
    #pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
        #pragma omp for collapse(2) schedule(static)
        for (int i = 0; i < n_rows; ++i)
            for (int h = 0; h < n_q; ++h) {
                int hk = (int)((long)h * n_kv / n_q);
                const double *qi = q + ((size_t)i * n_q + h) * dh;
                double mx = -INFINITY;
                for (int j = 0; j < n_keys; ++j) {
                    if (!mask[(size_t)i * n_keys + j]) { sc[j] = -INFINITY; continue; }
                    const double *kj = k + ((size_t)j * n_kv + hk) * dh;
                    double s = 0.0;
                    for (int c = 0; c < dh; ++c)
                        s += qi[c] * kj[c];
                    sc[j] = s * scale;
                    if (sc[j] > mx) mx = sc[j];
                }
                double *o = out + ((size_t)i * n_q + h) * dh;
                for (int c = 0; c < dh; ++c) o[c] = 0.0;
                if (mx == -INFINITY) continue;
                double den = 0.0;
                for (int j = 0; j < n_keys; ++j) {
                    if (sc[j] == -INFINITY) continue;
                    double p = exp(sc[j] - mx);
                    den += p;
                    const double *vj = v + ((size_t)j * n_kv + hk) * dh;
                    for (int c = 0; c < dh; ++c)
                        o[c] += p * vj[c];
                }
                for (int c = 0; c < dh; ++c)
                    o[c] /= den;
            }
        free(sc);
    }
}

/* Router [reading]: logits = h . W_r^T; the top_k experts by logit (ties -> lower expert id);
 * gates = softmax over the selected logits only.  sel/gate are [n][top_k] in rank order.
 * flip (nullable, [n]): a token with flip[t] != 0 takes its (top_k+1)-th expert in place of its
 * top_k-th one (the other choice of a token whose k-th and (k+1)-th logits are a near-tie); the
 * gates are the softmax over the logits it then selects.  Used by the tests to measure how much
 * such a choice moves the other tokens; flip = NULL is the router of the model. */
void orc_router_topk_flip(int n, int n_exp, int top_k, const double *logits, const uint8_t *flip, int32_t *sel,
                          double *gate)
{
    int32_t ranked[257];
    for (int t = 0; t < n; ++t) {
        const double *l = logits + (size_t)t * n_exp;
        const int alt = flip && flip[t] && top_k < n_exp;
        const int n_rank = top_k + alt;
        for (int r = 0; r < n_rank; ++r) {
            int best = -1;
            for (int e = 0; e < n_exp; ++e) {
                int taken = 0;
                for (int q = 0; q < r; ++q) taken |= (ranked[q] == e);
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict '>' keeps the lower id on ties */
            }
            ranked[r] = best;
        }
        if (alt) ranked[top_k - 1] = ranked[top_k];
        int32_t *s = sel + (size_t)t * top_k;
        for (int r = 0; r < top_k; ++r) s[r] = ranked[r];
        double mx = l[s[0]];
        for (int r = 1; r < top_k; ++r) if (l[s[r]] > mx) mx = l[s[r]];
        double den = 0.0;
        for (int r = 0; r < top_k; ++r) den += exp(l[s[r]] - mx);
        for (int r = 0; r < top_k; ++r) gate[(size_t)t * top_k + r] = exp(l[s[r]] - mx) / den;
    }
}

void orc_router_topk(int n, int n_exp, int top_k, const double *logits, int32_t *sel, double *gate)
{
    orc_router_topk_flip(n, n_exp, top_k, logits, NULL, sel, gate);
}

static double silu(double a) { return a / (1.0 + exp(-a)); }

typedef struct {
    int d_model, n_q, n_kv, d_head, n_exp, top_k, d_ff, n_layers, vocab;
    double rms_eps, rope_theta;
} orc_config;

typedef struct {
    const float *attn_norm;   /* [d] */
    orc_mat w_qkv;            /* [(n_q + 2 n_kv) dh][d]: Q rows, then K rows, then V rows */
    orc_mat w_o;              /* [d][n_q dh] */
    const float *ffn_norm;    /* [d] */
    orc_mat w_router;         /* [E][d] (bf16) */
    orc_mat w_gate_up;        /* [E * 2F][d]: expert e owns rows [2F e, 2F e + F) gate, [2F e + F, 2F(e+1)) up */
    orc_mat w_down;           /* [E * d][F]: expert e owns rows [d e, d (e+1)) */
} orc_layer_weights;

typedef struct {
    const uint16_t *emb;        /* [V][d] bf16 */
    const float *final_norm;    /* [d] */
    const uint16_t *head;       /* [V][d] bf16 (untied LM head) */
    const orc_layer_weights *layers;
} orc_model_weights;

/* Mixture of experts for n tokens: y_t = sum over the top-k experts e (in rank order) of
 * gate_{t,e} * W_down_e( silu(W_gate_e h_t) * (W_up_e h_t) ).  Computes only the selected experts. */
static void moe_apply(const orc_config *c, const orc_layer_weights *w, int n, int K, const double *h,
                      const int32_t *sel, const double *gate, double *y)
{
    int d = c->d_model, F = c->d_ff;
    memset(y, 0, sizeof(double) * (size_t)n * d);
    #pragma omp parallel
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)(d > F ? d : F));
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < n; ++t) {
            const double *ht = h + (size_t)t * d;
            for (int r = 0; r < K; ++r) {
                int e = sel[(size_t)t * K + r];
                for (int j = 0; j < F; ++j) {
                    double g = 0.0, u = 0.0;
                    mat_row(&w->w_gate_up, 2 * F * e + j, row);
                    for (int q = 0; q < d; ++q) g += row[q] * ht[q];
                    mat_row(&w->w_gate_up, 2 * F * e + F + j, row);
                    for (int q = 0; q < d; ++q) u += row[q] * ht[q];
                    a[j] = silu(g) * u;
                }
                for (int i = 0; i < d; ++i) {
                    mat_row(&w->w_down, d * e + i, row);
                    double acc = 0.0;
                    for (int j = 0; j < F; ++j) acc += row[j] * a[j];
                    o[i] = acc;
                }
                double gw = gate[(size_t)t * K + r];
                for (int i = 0; i < d; ++i) y[(size_t)t * d + i] += gw * o[i];
            }
        }
        free(row); free(a); free(o);
    }
}

/* sel/gate are [n][k] (k selected experts per token, any k <= E) */
void orc_moe(const orc_config *c, const orc_layer_weights *w, int n, int k, const double *h,
             const int32_t *sel, const double *gate, double *y)
{
    moe_apply(c, w, n, k, h, sel, gate, y);
}

/* One pre-norm decoder layer on n rows [reading of "same architecture as Gemma 4 26B A4B",
 * guide "Integration with existing serving frameworks"]:
 *   x <- x + W_o Attn(RoPE(Q), RoPE(K), V) of RMSNorm_1(x);   x <- x + MoE(RMSNorm_2(x)).
 * Keys are the cache rows [0, P) followed by the n rows themselves.  causal = 0: every row sees
 * every key (canvas step: bidirectional inside the canvas, full view of the committed prefix;
 * guide "Dual attention of prefill and denoising", report "Composition", training recipe);
 * causal = 1: row i sees cache and rows j <= i (prompt prefill).
 * k_new/v_new receive the rows' post-RoPE K and V ([n][n_kv][dh]); router_logits is [n][E];
 * x_mid (nullable) receives x after the attention residual.  flip (nullable, [n]): the routing
 * alternative of orc_router_topk_flip for the flagged tokens (test use; NULL is the model). */
int orc_layer_forward_flip(const orc_config *c, const orc_layer_weights *w, int n, const int32_t *pos,
                           double *x, int P, const double *k_cache, const double *v_cache, int causal,
                           double *k_new, double *v_new, double *router_logits, double *x_mid, const uint8_t *flip)
{
    int d = c->d_model, nq = c->n_q, nkv = c->n_kv, dh = c->d_head, E = c->n_exp;
    int nqkv = (nq + 2 * nkv) * dh, nkeys = P + n;
    double *h = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *qkv = (double *)malloc(sizeof(double) * (size_t)n * nqkv);
    double *q = (double *)malloc(sizeof(double) * (size_t)n * nq * dh);
    double *keys = (double *)malloc(sizeof(double) * (size_t)nkeys * nkv * dh);
    double *vals = (double *)malloc(sizeof(double) * (size_t)nkeys * nkv * dh);
    uint8_t *mask = (uint8_t *)malloc((size_t)n * nkeys);
    double *att = (double *)malloc(sizeof(double) * (size_t)n * nq * dh);
    double *o = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *rl = (double *)malloc(sizeof(double) * (size_t)n * E);
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)n * c->top_k);
    double *gate = (double *)malloc(sizeof(double) * (size_t)n * c->top_k);
    if (!h || !qkv || !q || !keys || !vals || !mask || !att || !o || !rl || !sel || !gate) return -1;

    /* attention block */
    orc_rmsnorm(n, d, x, w->attn_norm, c->rms_eps, h);
    mat_apply(&w->w_qkv, n, h, qkv, nqkv);
    double *kn = keys + (size_t)P * nkv * dh, *vn = vals + (size_t)P * nkv * dh;
    for (int t = 0; t < n; ++t) {
        const double *src = qkv + (size_t)t * nqkv;
        memcpy(q + (size_t)t * nq * dh, src, sizeof(double) * nq * dh);
        memcpy(kn + (size_t)t * nkv * dh, src + nq * dh, sizeof(double) * nkv * dh);
        memcpy(vn + (size_t)t * nkv * dh, src + (nq + nkv) * dh, sizeof(double) * nkv * dh);
    }
    orc_rope(n, nq, dh, pos, c->rope_theta, q);
    orc_rope(n, nkv, dh, pos, c->rope_theta, kn);
    if (P > 0) {
        memcpy(keys, k_cache, sizeof(double) * (size_t)P * nkv * dh);
        memcpy(vals, v_cache, sizeof(double) * (size_t)P * nkv * dh);
    }
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < nkeys; ++j)
            mask[(size_t)i * nkeys + j] = (uint8_t)(j < P || !causal || (j - P) <= i);
    orc_attention(n, nkeys, nq, nkv, dh, q, keys, vals, mask, att);
    mat_apply(&w->w_o, n, att, o, d);
    for (size_t i = 0; i < (size_t)n * d; ++i) x[i] += o[i];
    if (x_mid) memcpy(x_mid, x, sizeof(double) * (size_t)n * d);
    if (k_new) memcpy(k_new, kn, sizeof(double) * (size_t)n * nkv * dh);
    if (v_new) memcpy(v_new, vn, sizeof(double) * (size_t)n * nkv * dh);

    /* MoE block */
    orc_rmsnorm(n, d, x, w->ffn_norm, c->rms_eps, h);
    mat_apply(&w->w_router, n, h, rl, E);
    orc_router_topk_flip(n, E, c->top_k, rl, flip, sel, gate);
    moe_apply(c, w, n, c->top_k, h, sel, gate, o);
    for (size_t i = 0; i < (size_t)n * d; ++i) x[i] += o[i];
    if (router_logits) memcpy(router_logits, rl, sizeof(double) * (size_t)n * E);

    free(h); free(qkv); free(q); free(keys); free(vals); free(mask); free(att); free(o);
    free(rl); free(sel); free(gate);
    return 0;
}

int orc_layer_forward(const orc_config *c, const orc_layer_weights *w, int n, const int32_t *pos,
                      double *x, int P, const double *k_cache, const double *v_cache, int causal,
                      double *k_new, double *v_new, double *router_logits, double *x_mid)
{
    return orc_layer_forward_flip(c, w, n, pos, x, P, k_cache, v_cache, causal, k_new, v_new, router_logits, x_mid,
                                  NULL);
}

/* Embedding lookup: rows of the bf16 embedding table (no scaling; reading). */
void orc_embed(const orc_config *c, const uint16_t *emb, int n, const int32_t *ids, double *x)
{
    for (int t = 0; t < n; ++t)
        for (int j = 0; j < c->d_model; ++j)
            x[(size_t)t * c->d_model + j] = bf16_bits_to_double(emb[(size_t)ids[t] * c->d_model + j]);
}

/* LM head ("diffusion head" read as an ordinary vocabulary projection): logits = RMSNorm_f(x) W_head^T */
void orc_head(const orc_config *c, const orc_model_weights *m, int n, const double *x, double *logits)
{
    int d = c->d_model;
    double *h = (double *)malloc(sizeof(double) * (size_t)n * d);
    orc_rmsnorm(n, d, x, m->final_norm, c->rms_eps, h);
    orc_mat W = {m->head, NULL, NULL, c->vocab, d};
    mat_apply(&W, n, h, logits, c->vocab);
    free(h);
}

/* Full forward of n rows at positions pos, against caches [layer][P][n_kv][dh].
 * write_cache: also store each layer's post-RoPE K and V of the rows into cache rows [P, P+n).
 * hidden_dbg (nullable): [L+1][n][d] residual stream before layer 0 .. after the last layer.
 * logits (nullable): [n][V].  flip (nullable, [L][n]): per layer, the tokens that take the routing
 * alternative of orc_router_topk_flip (test use; NULL is the model). */
int orc_forward_flip(const orc_config *c, const orc_model_weights *m, int n, const int32_t *ids,
                     const int32_t *pos, int P, double *const *k_cache, double *const *v_cache, int causal,
                     int write_cache, double *hidden_dbg, double *router_dbg, double *logits, const uint8_t *flip)
{
    int d = c->d_model, kvw = c->n_kv * c->d_head;
    double *x = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *kn = (double *)malloc(sizeof(double) * (size_t)n * kvw);
    double *vn = (double *)malloc(sizeof(double) * (size_t)n * kvw);
    if (!x || !kn || !vn) return -1;
    orc_embed(c, m->emb, n, ids, x);
    if (hidden_dbg) memcpy(hidden_dbg, x, sizeof(double) * (size_t)n * d);
    for (int l = 0; l < c->n_layers; ++l) {
        double *rl = router_dbg ? router_dbg + (size_t)l * n * c->n_exp : NULL;
        if (orc_layer_forward_flip(c, &m->layers[l], n, pos, x, P, k_cache[l], v_cache[l], causal, kn, vn, rl, NULL,
                                   flip ? flip + (size_t)l * n : NULL))
            return -1;
        if (write_cache) {
            memcpy(k_cache[l] + (size_t)P * kvw, kn, sizeof(double) * (size_t)n * kvw);
            memcpy(v_cache[l] + (size_t)P * kvw, vn, sizeof(double) * (size_t)n * kvw);
        }
        if (hidden_dbg) memcpy(hidden_dbg + (size_t)(l + 1) * n * d, x, sizeof(double) * (size_t)n * d);
    }
    if (logits) orc_head(c, m, n, x, logits);
    free(x); free(kn); free(vn);
    return 0;
}

int orc_forward(const orc_config *c, const orc_model_weights *m, int n, const int32_t *ids,
                const int32_t *pos, int P, double *const *k_cache, double *const *v_cache, int causal,
                int write_cache, double *hidden_dbg, double *router_dbg, double *logits)
{
    return orc_forward_flip(c, m, n, ids, pos, P, k_cache, v_cache, causal, write_cache, hidden_dbg, router_dbg,
                            logits, NULL);
}

/* ------------------------------------------------------------------------------------------ */
/* Sampler [report "Composition", sampler settings; guide "Uniform State Diffusion",            */
/* "Serving with vLLM" (entropy_bound sampler, bound 0.1)].                                     */
/* ------------------------------------------------------------------------------------------ */

/* Per-row statistics at temperature T for absolute position pos and step s:
 *   z_v = l_v / T,  H = entropy of softmax(z) in nats = ln S - A/S with S = sum e^(z-m),
 *   A = sum e^(z-m)(z-m), m = max z;
 *   y = argmax_v (z_v + g_v), g_v Gumbel from word v of the stream (tag 0), ties -> lower v;
 *   margin = best - second-best perturbed score;  rr = uniform id from the stream (tag 1, word 0). */
static void sample_row(int V, const double *l, double T, uint64_t seed, uint32_t pos, uint32_t step,
                       double *H, int32_t *y, double *margin, int32_t *rr)
{
    double m = -INFINITY;
    for (int v = 0; v < V; ++v) {
        double z = l[v] / T;
        if (z > m) m = z;
    }
    double S = 0.0, A = 0.0, best = -INFINITY, second = -INFINITY;
    int arg = 0;
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)}, words[4];
    for (int v = 0; v < V; ++v) {
        double z = l[v] / T;
        double e = exp(z - m);
        S += e;
        A += e * (z - m);
        if ((v & 3) == 0) {
            uint32_t ctr[4] = {(uint32_t)(v >> 2), pos, step, 0u};
            orc_philox4x32_10(ctr, key, words);
        }
        double sc = z + orc_gumbel(words[v & 3]);
        if (sc > best) { second = best; best = sc; arg = v; }
        else if (sc > second) second = sc;
    }
    *H = log(S) - A / S;
    *y = arg;
    *margin = best - second;
    *rr = orc_token_from_word(orc_rng_word(seed, 0u, pos, step, 1u, 0), (uint32_t)V);
}

/* Rows with skip[i] != 0 (already committed) are not read: H = 0, y = rr = -1, margin = +inf. */
void orc_sample_rows_f32(int n, int V, const float *logits, const uint8_t *skip, const int32_t *pos,
                         float T, uint64_t seed, int step, double *H, int32_t *y, double *margin, int32_t *rr)
{
    #pragma omp parallel
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)V);
        #pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n; ++i) {
            if (skip && skip[i]) { H[i] = 0.0; y[i] = -1; margin[i] = INFINITY; rr[i] = -1; continue; }
            for (int v = 0; v < V; ++v) row[v] = (double)logits[(size_t)i * V + v];
            sample_row(V, row, (double)T, seed, (uint32_t)pos[i], (uint32_t)step, &H[i], &y[i], &margin[i], &rr[i]);
        }
        free(row);
    }
}

void orc_sample_rows_f64(int n, int V, const double *logits, const uint8_t *skip, const int32_t *pos,
                         float T, uint64_t seed, int step, double *H, int32_t *y, double *margin, int32_t *rr)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; ++i) {
        if (skip && skip[i]) { H[i] = 0.0; y[i] = -1; margin[i] = INFINITY; rr[i] = -1; continue; }
        sample_row(V, logits + (size_t)i * V, (double)T, seed, (uint32_t)pos[i], (uint32_t)step,
                   &H[i], &y[i], &margin[i], &rr[i]);
    }
}

/* Sort key of the cumulative rule: entropy, then position. */
static const double *g_sort_H;
static int cmp_entropy_then_index(const void *a, const void *b)
{
    int i = *(const int *)a, j = *(const int *)b;
    if (g_sort_H[i] < g_sort_H[j]) return -1;
    if (g_sort_H[i] > g_sort_H[j]) return 1;
    return (i > j) - (i < j);
}

/* Decision rule of one step [reading of the entropy-bound sampler, self-correction and adaptive
 * stop]:
 *   - a committed position keeps its id (committed positions are anchors and never change);
 *   - cumulative == 0: an uncommitted position with H <= entropy_bound commits with id y;
 *     cumulative == 1: the uncommitted positions in ascending (H, position) order commit with id y
 *     while the running sum of their entropies stays <= entropy_bound (the longest such prefix);
 *     cum (nullable) receives each uncommitted position's running sum in that order;
 *   - otherwise it is re-randomised (id rr) when H > rerand_entropy, else takes y;
 *   - stop after this step when every position is committed, or mean(H over all n positions,
 *     committed ones counting 0) <= stop_mean_entropy, or s + 1 == max_steps; with
 *     fixed_steps > 0 the adaptive tests are off and the block stops exactly at s + 1 == fixed_steps;
 *   - on stop every still-uncommitted position takes y and is committed.
 * Returns the stop flag; *mean_H receives the canvas-mean entropy. */
int orc_step_rule(int n, const uint8_t *commit_in, const int32_t *ids_in, const double *H,
                  const int32_t *y, const int32_t *rr, double entropy_bound, double rerand_entropy,
                  double stop_mean_entropy, int s, int max_steps, int fixed_steps, int cumulative,
                  int32_t *ids_out, uint8_t *commit_out, double *mean_H, double *cum)
{
    uint8_t *commits_now = (uint8_t *)calloc((size_t)n, 1);
    if (!commits_now) return -1;
    if (cumulative) {
        int *order = (int *)malloc(sizeof(int) * (size_t)n);
        if (!order) { free(commits_now); return -1; }
        int m = 0;
        for (int i = 0; i < n; ++i)
            if (!commit_in[i]) order[m++] = i;
        g_sort_H = H;
        qsort(order, (size_t)m, sizeof(int), cmp_entropy_then_index);
        double run = 0.0;
        for (int k = 0; k < m; ++k) {
            run += H[order[k]];
            if (cum) cum[order[k]] = run;
            if (run <= entropy_bound) commits_now[order[k]] = 1;
        }
        free(order);
    } else {
        for (int i = 0; i < n; ++i)
            commits_now[i] = !commit_in[i] && H[i] <= entropy_bound;
    }
    double sumH = 0.0;
    int all = 1;
    for (int i = 0; i < n; ++i) {
        if (commit_in[i]) {
            ids_out[i] = ids_in[i];
            commit_out[i] = 1;
            if (cum) cum[i] = 0.0;
            continue;
        }
        sumH += H[i];
        if (commits_now[i]) {
            ids_out[i] = y[i];
            commit_out[i] = 1;
        } else {
            ids_out[i] = H[i] > rerand_entropy ? rr[i] : y[i];
            commit_out[i] = 0;
            all = 0;
        }
    }
    free(commits_now);
    double mean = sumH / n;
    *mean_H = mean;
    int stop;
    if (fixed_steps > 0)
        stop = (s + 1 >= fixed_steps);
    else
        stop = all || mean <= stop_mean_entropy || (s + 1 >= max_steps);
    if (stop)
        for (int i = 0; i < n; ++i)
            if (!commit_out[i]) {
                ids_out[i] = y[i];
                commit_out[i] = 1;
            }
    return stop;
}

/* Canvas initialisation [guide "Uniform State Diffusion": random placeholder tokens]:
 * position j of the block starting at P gets a uniform id from the stream (tag 2, step 0). */
void orc_canvas_init(int n, int P, uint64_t seed, int V, int32_t *ids, uint8_t *commit)
{
    for (int j = 0; j < n; ++j) {
        ids[j] = orc_token_from_word(orc_rng_word(seed, 0u, (uint32_t)(P + j), 0u, 2u, 0), (uint32_t)V);
        commit[j] = 0;
    }
}
