/*
 * amk_oracle.c -- fp64 CPU oracle for one batch-1 decode step of a
 * Llama-family decoder (the computation the AutoMegaKernel megakernel runs as
 * one persistent launch per token).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the bench's CPU-baseline leg and the smoke check
 * do.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes is the plain definition, written out op by op in fp64:
 *   "RightNow-AI/AutoMegaKernel" README (bittide mirror), section "What is
 *   built and verified": the whole Llama-style decode forward, matching eager
 *   PyTorch; multi-token greedy decode with a KV cache carried across steps.
 *   paperfeed "RightNow-AI/AutoMegaKernel", section "How it works": the
 *   instruction set (GEMV tiles, attention tile, RMSNorm, RoPE, SwiGLU,
 *   dequant).
 *   Same README, results section: W8A16 int8 weights (per output channel),
 *   correctness gated on an exact argmax.
 *   gist.science technical summary of the paper, "Belangrijkste Bijdragen"
 *   (the quantised-megakernels item): int8 and int4 weight-only kernels from
 *   the same IR path.  The pages give no int4 format; the one
 *   read here is symmetric 4-bit codes with one fp16 scale per group of 128
 *   consecutive inputs of a row (the last group shorter when the row length
 *   is not a multiple of 128), two codes per byte, input 2i in the low nibble.
 * Where the pages leave a step open, the HuggingFace Llama definition is used
 * (the pages reproduce HF greedy generate token for token): RoPE is HF
 * rotate_half, GQA maps query head h to KV head h / (n_heads / n_kv_heads),
 * the softmax is the max-subtracted form over positions 0..pos inclusive.
 *
 * Precision: weights arrive as the exact bf16 (or int8/int4 + fp16 scale) bytes the
 * GPU consumes and are widened to double; everything else is double.  The KV
 * cache is stored as bf16 (round to nearest even), which is how the workload
 * defines the cache ("bf16 activations/KV"); every K and V row is rounded
 * once when it is appended, and attention reads the rounded rows.
 *
 * KV cache layout (caller-owned, bf16 bits):
 *   kv[((layer * 2 + which) * n_kv_heads + g) * max_ctx + position][d]
 * with which = 0 for K (after RoPE) and 1 for V.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t hidden, n_layers, n_heads, n_kv_heads, head_dim, ffn, vocab, max_ctx;
    double rms_eps, rope_theta;
    int32_t tied;  /* 1: the LM head is the embedding table */
    int32_t quant; /* 0: bf16 linear weights; 1: int8 + fp16 row scales;
                      2: packed int4 + fp16 scales per 128-input group */
} orc_config;

typedef struct {
    const uint16_t *embed;      /* bf16 [vocab][hidden] */
    const uint16_t *final_norm; /* bf16 [hidden] */
    const void *lm_head;        /* bf16, int8 or packed int4 [vocab][hidden]; unused if tied */
    const uint16_t *lm_head_scale; /* fp16 [vocab] (int8) or [vocab][groups] (int4), untied */
    const uint16_t *const *attn_norm; /* [n_layers] -> bf16 [hidden] */
    const uint16_t *const *ffn_norm;
    const void *const *wq, *const *wk, *const *wv, *const *wo;
    const void *const *wgate, *const *wup, *const *wdown;
    const uint16_t *const *sq, *const *sk, *const *sv, *const *so;
    const uint16_t *const *sgate, *const *sup, *const *sdown;
} orc_weights;

/* ---- number formats ---------------------------------------------------- */

/* bf16 is the top half of an IEEE binary32. */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_fp16_to_double(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);
    return s ? -v : v;
}

/* Round a double to the nearest bf16 (8 significant bits, ties to even) and
 * return its bits.  bf16 shares binary32's exponent range; its smallest
 * subnormal step is 2^-133. */
uint16_t orc_double_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    if (v == 0.0)
        return signbit(v) ? 0x8000 : 0x0000;
    int e;
    frexp(v, &e);          /* |v| = f * 2^e, f in [0.5, 1) */
    int step = e - 8;      /* spacing of 8-significant-bit numbers near v */
    if (step < -133)
        step = -133;
    double q = nearbyint(ldexp(v, -step)); /* default mode: ties to even */
    double r = ldexp(q, step);
    if (fabs(r) >= ldexp(1.0, 128))
        return v < 0 ? 0xFF80 : 0x7F80;
    float f = (float)r;    /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ---- the ops ----------------------------------------------------------- */

/* RMSNorm: out_i = g_i * x_i / sqrt(mean_j x_j^2 + eps). */
void orc_rmsnorm(const double *x, const uint16_t *g, int32_t n, double eps,
                 double *out)
{
    double ss = 0.0;
    for (int32_t i = 0; i < n; ++i)
        ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss / n + eps);
    for (int32_t i = 0; i < n; ++i)
        out[i] = orc_bf16_to_double(g[i]) * (x[i] * inv);
}

#define ORC_INT4_GROUP 128

/* The signed value of input k's 4-bit code in a packed int4 row: byte k / 2,
 * low nibble for even k, high nibble for odd k, two's complement. */
static int orc_int4_code(const uint8_t *row, int32_t k)
{
    int nib = (row[k >> 1] >> ((k & 1) * 4)) & 0xF;
    return nib >= 8 ? nib - 16 : nib;
}

/* y = W x for row-major W [rows][cols].  quant 0: W is bf16.  quant 1: W is
 * int8 and row j's weights are scale_j * q_jk, so y_j = scale_j * sum_k q_jk x_k.
 * quant 2: W is packed int4 (cols / 2 bytes per row) and weight (j, k) is
 * scale[j][k / 128] * q_jk, the scales fp16 [rows][ceil(cols / 128)]. */
void orc_matvec(const void *W, const uint16_t *scale, int32_t quant,
                int32_t rows, int32_t cols, const double *x, double *y)
{
#pragma omp parallel for schedule(static)
    for (int32_t j = 0; j < rows; ++j) {
        double acc = 0.0;
        if (quant == 0) {
            const uint16_t *w = (const uint16_t *)W + (size_t)j * cols;
            for (int32_t k = 0; k < cols; ++k)
                acc += orc_bf16_to_double(w[k]) * x[k];
            y[j] = acc;
        } else if (quant == 1) {
            const int8_t *w = (const int8_t *)W + (size_t)j * cols;
            for (int32_t k = 0; k < cols; ++k)
                acc += (double)w[k] * x[k];
            y[j] = orc_fp16_to_double(scale[j]) * acc;
        } else {
            const uint8_t *w = (const uint8_t *)W + (size_t)j * (cols / 2);
            const int32_t ng = (cols + ORC_INT4_GROUP - 1) / ORC_INT4_GROUP;
            const uint16_t *sj = scale + (size_t)j * ng;
            for (int32_t k = 0; k < cols; ++k)
                acc += orc_fp16_to_double(sj[k / ORC_INT4_GROUP]) * orc_int4_code(w, k) * x[k];
            y[j] = acc;
        }
    }
}

/* RoPE on one head vector v[head_dim] at position pos, HF rotate_half form:
 * for i < hd/2, w_i = theta^(-2i/hd), a = pos * w_i,
 *   v'_i        = v_i cos a - v_{i+hd/2} sin a
 *   v'_{i+hd/2} = v_{i+hd/2} cos a + v_i sin a. */
void orc_rope(double *v, int32_t head_dim, int32_t pos, double theta)
{
    int32_t half = head_dim / 2;
    for (int32_t i = 0; i < half; ++i) {
        double w = pow(theta, -2.0 * i / head_dim);
        double a = (double)pos * w;
        double c = cos(a), s = sin(a);
        double x0 = v[i], x1 = v[i + half];
        v[i] = x0 * c - x1 * s;
        v[i + half] = x1 * c + x0 * s;
    }
}

/* One query head attending over npos cached rows (bf16 bits, row stride
 * head_dim): s_j = q . K_j / sqrt(hd), p = softmax(s), out = sum_j p_j V_j.
 * If probs is not NULL it receives p. */
void orc_attention_head(const double *q, const uint16_t *K, const uint16_t *V,
                        int32_t npos, int32_t head_dim, double *out,
                        double *probs)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1));
    double scale = 1.0 / sqrt((double)head_dim);
    double mx = -INFINITY;
    for (int32_t j = 0; j < npos; ++j) {
        double d = 0.0;
        for (int32_t t = 0; t < head_dim; ++t)
            d += q[t] * orc_bf16_to_double(K[(size_t)j * head_dim + t]);
        s[j] = d * scale;
        if (s[j] > mx)
            mx = s[j];
    }
    double den = 0.0;
    for (int32_t j = 0; j < npos; ++j) {
        s[j] = exp(s[j] - mx);
        den += s[j];
    }
    for (int32_t t = 0; t < head_dim; ++t)
        out[t] = 0.0;
    for (int32_t j = 0; j < npos; ++j) {
        double p = s[j] / den;
        if (probs)
            probs[j] = p;
        for (int32_t t = 0; t < head_dim; ++t)
            out[t] += p * orc_bf16_to_double(V[(size_t)j * head_dim + t]);
    }
    free(s);
}

/* SiLU(z) = z / (1 + e^-z). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* Index of the largest value; the lowest index wins a tie. */
int32_t orc_argmax(const double *v, int32_t n)
{
    int32_t best = 0;
    for (int32_t i = 1; i < n; ++i)
        if (v[i] > v[best])
            best = i;
    return best;
}

/* ---- one decode step ---------------------------------------------------- */

static const uint16_t *sel_scale(const orc_config *c, const uint16_t *const *s,
                                 int32_t l)
{
    return c->quant ? s[l] : NULL;
}

/* Runs the decode step for token `token` at position `pos`: appends this
 * position's K and V to every layer's cache, writes the vocab logits and the
 * greedy token.  If trace is not NULL it receives, per layer, the residual
 * stream after attention and after the FFN: trace[(l*2 + {0,1}) * hidden + i].
 * Returns 0, or -1 on bad arguments. */
int32_t orc_decode_step(const orc_config *c, const orc_weights *w,
                        uint16_t *kv, int32_t token, int32_t pos,
                        double *logits, int32_t *argmax_out, double *trace)
{
    const int32_t h = c->hidden, nh = c->n_heads, nkv = c->n_kv_heads;
    const int32_t hd = c->head_dim, F = c->ffn;
    if (token < 0 || token >= c->vocab || pos < 0 || pos >= c->max_ctx ||
        nkv <= 0 || nh % nkv != 0 || (hd & 1) || c->quant < 0 || c->quant > 2)
        return -1;
    if (c->quant == 2 && ((h & 1) || ((nh * hd) & 1) || (F & 1)))
        return -1; /* packed int4 rows hold whole bytes */
    const int32_t group = nh / nkv;
    const int32_t qr = nh * hd, kr = nkv * hd;

    double *x = (double *)calloc((size_t)h, sizeof(double));
    double *u = (double *)calloc((size_t)h, sizeof(double));
    double *q = (double *)calloc((size_t)qr, sizeof(double));
    double *k = (double *)calloc((size_t)kr, sizeof(double));
    double *v = (double *)calloc((size_t)kr, sizeof(double));
    double *att = (double *)calloc((size_t)qr, sizeof(double));
    double *o = (double *)calloc((size_t)h, sizeof(double));
    double *gt = (double *)calloc((size_t)F, sizeof(double));
    double *up = (double *)calloc((size_t)F, sizeof(double));
    double *a = (double *)calloc((size_t)F, sizeof(double));
    double *dn = (double *)calloc((size_t)h, sizeof(double));

    /* embedding gather */
    for (int32_t i = 0; i < h; ++i)
        x[i] = orc_bf16_to_double(w->embed[(size_t)token * h + i]);

    for (int32_t l = 0; l < c->n_layers; ++l) {
        /* attention block */
        orc_rmsnorm(x, w->attn_norm[l], h, c->rms_eps, u);
        orc_matvec(w->wq[l], sel_scale(c, w->sq, l), c->quant, qr, h, u, q);
        orc_matvec(w->wk[l], sel_scale(c, w->sk, l), c->quant, kr, h, u, k);
        orc_matvec(w->wv[l], sel_scale(c, w->sv, l), c->quant, kr, h, u, v);
        for (int32_t hh = 0; hh < nh; ++hh)
            orc_rope(q + (size_t)hh * hd, hd, pos, c->rope_theta);
        for (int32_t g = 0; g < nkv; ++g)
            orc_rope(k + (size_t)g * hd, hd, pos, c->rope_theta);
        for (int32_t g = 0; g < nkv; ++g) {
            uint16_t *Kc = kv + (((size_t)l * 2 + 0) * nkv + g) * c->max_ctx * hd;
            uint16_t *Vc = kv + (((size_t)l * 2 + 1) * nkv + g) * c->max_ctx * hd;
            for (int32_t t = 0; t < hd; ++t) {
                Kc[(size_t)pos * hd + t] = orc_double_to_bf16(k[(size_t)g * hd + t]);
                Vc[(size_t)pos * hd + t] = orc_double_to_bf16(v[(size_t)g * hd + t]);
            }
        }
#pragma omp parallel for schedule(static)
        for (int32_t hh = 0; hh < nh; ++hh) {
            int32_t g = hh / group;
            const uint16_t *Kc = kv + (((size_t)l * 2 + 0) * nkv + g) * c->max_ctx * hd;
            const uint16_t *Vc = kv + (((size_t)l * 2 + 1) * nkv + g) * c->max_ctx * hd;
            orc_attention_head(q + (size_t)hh * hd, Kc, Vc, pos + 1, hd,
                               att + (size_t)hh * hd, NULL);
        }
        orc_matvec(w->wo[l], sel_scale(c, w->so, l), c->quant, h, qr, att, o);
        for (int32_t i = 0; i < h; ++i)
            x[i] += o[i];
        if (trace)
            memcpy(trace + ((size_t)l * 2 + 0) * h, x, sizeof(double) * h);

        /* SwiGLU FFN block */
        orc_rmsnorm(x, w->ffn_norm[l], h, c->rms_eps, u);
        orc_matvec(w->wgate[l], sel_scale(c, w->sgate, l), c->quant, F, h, u, gt);
        orc_matvec(w->wup[l], sel_scale(c, w->sup, l), c->quant, F, h, u, up);
        for (int32_t j = 0; j < F; ++j)
            a[j] = orc_silu(gt[j]) * up[j];
        orc_matvec(w->wdown[l], sel_scale(c, w->sdown, l), c->quant, h, F, a, dn);
        for (int32_t i = 0; i < h; ++i)
            x[i] += dn[i];
        if (trace)
            memcpy(trace + ((size_t)l * 2 + 1) * h, x, sizeof(double) * h);
    }

    /* final norm, LM head (the embedding table when tied), greedy token */
    orc_rmsnorm(x, w->final_norm, h, c->rms_eps, u);
    if (c->tied)
        orc_matvec(w->embed, NULL, 0, c->vocab, h, u, logits);
    else
        orc_matvec(w->lm_head, c->quant ? w->lm_head_scale : NULL, c->quant,
                   c->vocab, h, u, logits);
    if (argmax_out)
        *argmax_out = orc_argmax(logits, c->vocab);

    free(x); free(u); free(q); free(k); free(v); free(att); free(o);
    free(gt); free(up); free(a); free(dn);
    return 0;
}

/* Thread count for the OpenMP loops (the CPU baseline reports it). */
int32_t orc_set_threads(int32_t n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
