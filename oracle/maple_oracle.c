/*
 * maple_oracle.c -- plain, slow, single-threaded CPU oracle for the forward
 * pass of one ternary-weight mixture-of-experts FFN layer (and the stack of
 * such layers with RMSNorm + residual between them).
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark may load or call this library.  The CUDA
 * library never links, loads or calls it, and shares no source with it.
 *
 * What it computes, and where each step comes from:
 *
 *  - Ternary linear layers: every weight is one of {-alpha, 0, +alpha} with one
 *    alpha per output row, so a product becomes add (+alpha), subtract
 *    (-alpha) or skip (0).  ("linlog.top/article/1232", section
 *    三值权重; its model table in section 架构设计 lists the weights as
 *    2-bit ternary with one alpha per row.)  Here the accumulation over the input
 *    dimension is done in int32 on int8 activation codes and the scales are
 *    applied afterwards.
 *  - Routing: every token scores all experts and keeps the top-8 of 256
 *    (same page, 架构设计 table: top-8 routing over 256 experts).
 *  - Everything the pages leave open (SwiGLU expert MLP, the per-token int8
 *    absmax quantiser, fp32 router, rounding and summation orders, exp, the
 *    2-bit code map) follows one fixed reading, stated at each function.
 *    All float steps are single IEEE-754 binary32 operations rounded to
 *    nearest even; build with -ffp-contract=off so that no product and sum are
 *    fused unless fmaf() is written.
 *
 * Parity pins: every function here is checked against something other than
 * itself by the CPU tests (dense int64 matmul on expanded codes, numpy float64
 * references, full-sort top-k, closed forms and invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_NAN (-2)
#define ORC_ERR_OOM (-3)

/* ------------------------------------------------------------------ */
/* 2-bit ternary interchange format                                    */
/* ------------------------------------------------------------------ */
/*
 * A row of `cols` ternary values is stored as cols/16 uint32 words.  Value j
 * of the row sits in word j/16, bits 2*(j%16) and 2*(j%16)+1.  Code 0 means 0,
 * code 1 means +1, code 2 means -1.  Code 3 is never written; a reader treats
 * it as 0.  Two bits per weight is what makes the 20.2B-parameter model a
 * 5.31 GB checkpoint ("linlog.top/article/1232", 架构设计 table).
 */
int orc_pack_ternary(const int8_t *t, int64_t rows, int32_t cols, uint32_t *out)
{
    if (cols <= 0 || cols % 16 != 0 || rows < 0) return ORC_ERR_ARG;
    int32_t words = cols / 16;
    for (int64_t r = 0; r < rows; r++) {
        for (int32_t w = 0; w < words; w++) {
            uint32_t word = 0;
            for (int32_t i = 0; i < 16; i++) {
                int8_t v = t[r * cols + (int64_t)w * 16 + i];
                uint32_t code;
                if (v == 0) code = 0;
                else if (v == 1) code = 1;
                else if (v == -1) code = 2;
                else return ORC_ERR_ARG;
                word |= code << (2 * i);
            }
            out[r * words + w] = word;
        }
    }
    return ORC_OK;
}

static int orc_code_value(uint32_t code)
{
    if (code == 1) return 1;
    if (code == 2) return -1;
    return 0;                    /* 0, and the invalid code 3 */
}

/* value j of a packed row */
static int orc_ternary_at(const uint32_t *row, int32_t j)
{
    uint32_t code = (row[j / 16] >> (2 * (j % 16))) & 3u;
    return orc_code_value(code);
}

int orc_unpack_ternary(const uint32_t *p, int64_t rows, int32_t cols, int8_t *out)
{
    if (cols <= 0 || cols % 16 != 0 || rows < 0) return ORC_ERR_ARG;
    for (int64_t r = 0; r < rows; r++)
        for (int32_t j = 0; j < cols; j++)
            out[r * cols + j] = (int8_t)orc_ternary_at(p + r * (cols / 16), j);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* exp                                                                 */
/* ------------------------------------------------------------------ */
/*
 * exp(x) written out from the mathematics, so that the CPU and the GPU can
 * take bit-identical decisions that depend on it (SiLU feeds the int8 codes
 * of the down-projection input):
 *   clamp x to [-87, 88];
 *   n = rint(x * log2(e));
 *   r = x - n*ln2, with ln2 split in two (Cody and Waite) and fmaf;
 *   p = sum_{k=0..7} r^k / k!  (Taylor polynomial, Horner form with fmaf);
 *   result = p * 2^n, 2^n built from its exponent bits.
 * Constants: ln2_hi = 0.693145751953125 (ln 2 truncated to 17 significant
 * bits), ln2_lo = ln 2 - ln2_hi, log2(e) and 1/k!, each rounded once to
 * binary32 from its double value.
 */
static float orc_c_log2e, orc_c_ln2_hi, orc_c_ln2_lo, orc_c_inv_fact[8];
static int orc_exp_ready = 0;

static void orc_exp_init(void)
{
    double f = 1.0;
    for (int k = 0; k < 8; k++) {
        if (k > 0) f *= (double)k;
        orc_c_inv_fact[k] = (float)(1.0 / f);
    }
    orc_c_log2e = (float)(1.0 / log(2.0));
    orc_c_ln2_hi = 0.693145751953125f;
    orc_c_ln2_lo = (float)(log(2.0) - 0.693145751953125);
    orc_exp_ready = 1;
}

float orc_exp(float x)
{
    if (!orc_exp_ready) orc_exp_init();
    if (x < -87.0f) x = -87.0f;
    if (x > 88.0f) x = 88.0f;
    float n = rintf(x * orc_c_log2e);
    float r = fmaf(-n, orc_c_ln2_hi, x);
    r = fmaf(-n, orc_c_ln2_lo, r);
    float p = orc_c_inv_fact[7];
    for (int k = 6; k >= 0; k--) p = fmaf(p, r, orc_c_inv_fact[k]);
    uint32_t bits = (uint32_t)((int32_t)n + 127) << 23;
    float scale;
    memcpy(&scale, &bits, sizeof scale);
    return p * scale;
}

void orc_exp_array(const float *x, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_exp(x[i]);
}

/* ------------------------------------------------------------------ */
/* bf16                                                                */
/* ------------------------------------------------------------------ */
static float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* round a finite float to bf16, nearest with ties to even */
static uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* int8 absmax quantiser                                               */
/* ------------------------------------------------------------------ */
/*
 * Symmetric per-row absmax quantisation of a float vector to int8:
 *   amax = max_j |v_j|;  if amax == 0: q = 0, s = 0;
 *   inv = 127 / amax;  q_j = clamp(rint(v_j * inv), -127, 127);  s = amax / 127.
 * (one rounded division for inv, one rounded product per element, rint with
 * ties to even; -128 is never produced.)  Used for the token activations
 * before gate/up and for each (token, expert) SwiGLU output before down.
 */
void orc_quantize_row(const float *v, int32_t n, int8_t *q, float *s)
{
    float amax = 0.0f;
    for (int32_t j = 0; j < n; j++) {
        float a = fabsf(v[j]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        for (int32_t j = 0; j < n; j++) q[j] = 0;
        *s = 0.0f;
        return;
    }
    float inv = 127.0f / amax;
    for (int32_t j = 0; j < n; j++) {
        float t = rintf(v[j] * inv);
        if (t > 127.0f) t = 127.0f;
        if (t < -127.0f) t = -127.0f;
        q[j] = (int8_t)t;
    }
    *s = amax / 127.0f;
}

/* ------------------------------------------------------------------ */
/* Router logit with the fixed fp32 summation order                    */
/* ------------------------------------------------------------------ */
/*
 * logit = sum_j x_j * w_j in binary32, in this fixed order (D a multiple of
 * 256): partial sum number l (l = 0..31) runs over j = 256*i + 8*l + m for
 * i = 0..D/256-1, m = 0..7, acc = fmaf(x_j, w_j, acc) from 0; the 32 partial
 * sums are then added pairwise, first partial l with partial l^16, then the
 * results with distance 8, 4, 2 and 1 (a binary tree over the index bits from
 * high to low).  The pages fix no order; one is needed so that the choice of
 * the top-k experts is reproducible bit for bit.
 */
static float orc_tree_sum32(float p[32])
{
    float a[32];
    for (int l = 0; l < 32; l++) a[l] = p[l];
    for (int dist = 16; dist >= 1; dist /= 2) {
        float b[32];
        for (int l = 0; l < 32; l++) b[l] = a[l] + a[l ^ dist];
        for (int l = 0; l < 32; l++) a[l] = b[l];
    }
    return a[0];
}

float orc_router_logit(const float *x, const float *w, int32_t D)
{
    float p[32];
    for (int l = 0; l < 32; l++) {
        float acc = 0.0f;
        for (int32_t i = 0; i < D / 256; i++)
            for (int m = 0; m < 8; m++) {
                int32_t j = 256 * i + 8 * l + m;
                acc = fmaf(x[j], w[j], acc);
            }
        p[l] = acc;
    }
    return orc_tree_sum32(p);
}

/* ------------------------------------------------------------------ */
/* top-k and softmax over the kept logits                              */
/* ------------------------------------------------------------------ */
/*
 * The K largest logits in descending order; equal logits are ordered by the
 * lower expert index first.  A NaN logit is an error.
 */
int orc_topk(const float *logits, int32_t E, int32_t K, int32_t *idx)
{
    if (K < 1 || K > E) return ORC_ERR_ARG;
    for (int32_t e = 0; e < E; e++)
        if (isnan(logits[e])) return ORC_ERR_NAN;
    for (int32_t k = 0; k < K; k++) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; e++) {
            int taken = 0;
            for (int32_t q = 0; q < k; q++)
                if (idx[q] == e) taken = 1;
            if (taken) continue;
            if (best < 0 || logits[e] > logits[best]) best = e;  /* strict: ties keep the lower index */
        }
        idx[k] = best;
    }
    return ORC_OK;
}

/*
 * Softmax over the K kept logits (sorted descending):
 *   e_k = exp(l_k - l_0);  S = e_0 + e_1 + ... (left to right, from 0);  w_k = e_k / S.
 * Mathematically equal to a softmax over all experts renormalised over the
 * kept ones.
 */
void orc_softmax_kept(const float *kept, int32_t K, float *w)
{
    float e[1024];
    float S = 0.0f;
    for (int32_t k = 0; k < K; k++) {
        e[k] = orc_exp(kept[k] - kept[0]);
        S = S + e[k];
    }
    for (int32_t k = 0; k < K; k++) w[k] = e[k] / S;
}

/* ------------------------------------------------------------------ */
/* token -> expert permutation                                         */
/* ------------------------------------------------------------------ */
/*
 * Slot s = t*K + k is token t's k-th choice idx[s].  counts[e] = number of
 * slots routed to e; offsets = exclusive prefix sum of counts (E+1 entries);
 * perm lists, expert by expert, that expert's slots in increasing s (hence
 * increasing token); inv[s] is the position of slot s in perm.  This is a
 * stable counting sort.
 */
int orc_permute(const int32_t *idx, int32_t T, int32_t K, int32_t E,
                int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv)
{
    int64_t S = (int64_t)T * K;
    for (int32_t e = 0; e < E; e++) counts[e] = 0;
    for (int64_t s = 0; s < S; s++) {
        if (idx[s] < 0 || idx[s] >= E) return ORC_ERR_ARG;
        counts[idx[s]]++;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor) return ORC_ERR_OOM;
    for (int32_t e = 0; e < E; e++) cursor[e] = offsets[e];
    for (int64_t s = 0; s < S; s++) {
        int32_t p = cursor[idx[s]]++;
        perm[p] = (int32_t)s;
        inv[s] = p;
    }
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* the layer                                                           */
/* ------------------------------------------------------------------ */
typedef struct {
    int32_t d_model, n_experts, top_k, d_ff;
} orc_shape;

/* packed weights in the interchange format, scales and router */
typedef struct {
    const uint32_t *w_gate;      /* [E][F][D/16] */
    const uint32_t *w_up;        /* [E][F][D/16] */
    const uint32_t *w_down;      /* [E][D][F/16] */
    const float *alpha_gate;     /* [E][F] */
    const float *alpha_up;       /* [E][F] */
    const float *alpha_down;     /* [E][D] */
    const float *router_w;       /* [E][D] */
    const float *router_bias;    /* [E] or NULL */
} orc_weights;

/* optional intermediate results; row n of every array belongs to tokens[n] */
typedef struct {
    int8_t *q_x;        /* [n][D] */
    float *s_x;         /* [n] */
    float *logits;      /* [n][E] */
    int32_t *topk_idx;  /* [n][K] */
    float *topk_w;      /* [n][K] */
    int32_t *acc_gate;  /* [n][K][F] */
    int32_t *acc_up;    /* [n][K][F] */
    float *h;           /* [n][K][F] */
    int8_t *q_h;        /* [n][K][F] */
    float *s_h;         /* [n][K] */
    int32_t *acc_down;  /* [n][K][D] */
    float *y_e;         /* [n][K][D] */
} orc_taps;

/* route one token: logits over all experts, top-k, softmax over kept */
static int orc_route_token(const orc_shape *sh, const orc_weights *wt, const float *xf,
                           float *logits, int32_t *idx, float *w)
{
    int32_t D = sh->d_model, E = sh->n_experts, K = sh->top_k;
    for (int32_t e = 0; e < E; e++) {
        float l = orc_router_logit(xf, wt->router_w + (int64_t)e * D, D);
        if (wt->router_bias) l = l + wt->router_bias[e];
        logits[e] = l;
    }
    int rc = orc_topk(logits, E, K, idx);
    if (rc) return rc;
    float kept[1024];
    for (int32_t k = 0; k < K; k++) kept[k] = logits[idx[k]];
    orc_softmax_kept(kept, K, w);
    return ORC_OK;
}

int orc_route(const orc_shape *sh, const orc_weights *wt, const uint16_t *x, int32_t T,
              float *logits /*[T][E] or NULL*/, int32_t *idx /*[T][K]*/, float *w /*[T][K]*/)
{
    int32_t D = sh->d_model, E = sh->n_experts, K = sh->top_k;
    if (D % 256 || K < 1 || K > E || E > 1024) return ORC_ERR_ARG;
    float *xf = (float *)malloc(sizeof(float) * (size_t)D);
    float *lg = (float *)malloc(sizeof(float) * (size_t)E);
    if (!xf || !lg) { free(xf); free(lg); return ORC_ERR_OOM; }
    int rc = ORC_OK;
    for (int32_t t = 0; t < T && rc == ORC_OK; t++) {
        for (int32_t j = 0; j < D; j++) xf[j] = orc_bf16_to_f32(x[(int64_t)t * D + j]);
        rc = orc_route_token(sh, wt, xf, lg, idx + (int64_t)t * K, w + (int64_t)t * K);
        if (logits) memcpy(logits + (int64_t)t * E, lg, sizeof(float) * (size_t)E);
    }
    free(xf);
    free(lg);
    return rc;
}

/*
 * Forward pass for the listed tokens (each token is independent of the
 * others).  For token t with choices idx[k] and weights w[k]:
 *   q_x, s_x  = quantise(x_t)
 *   accG[r]   = sum_j tG[e][r][j] * q_x[j]      (int32; add / subtract / skip)
 *   accU[r]   = sum_j tU[e][r][j] * q_x[j]
 *   g = f32(accG[r]) * (alphaG[e][r] * s_x),  u likewise  (the product of the
 *       two scales is rounded first)
 *   h[r]      = (g / (1 + exp(-g))) * u          (SiLU(g) * u, i.e. SwiGLU)
 *   q_h, s_h  = quantise(h)
 *   accD[c]   = sum_r tD[e][c][r] * q_h[r]
 *   yE[c]     = f32(accD[c]) * (alphaD[e][c] * s_h)
 *   y[c]      = fmaf(w[k], yE_k[c], y[c]) for k = 0..K-1, from y = 0.
 */
int orc_forward_tokens(const orc_shape *sh, const orc_weights *wt, const uint16_t *x,
                       const int32_t *tokens, int32_t n, float *y, const orc_taps *taps)
{
    int32_t D = sh->d_model, E = sh->n_experts, K = sh->top_k, F = sh->d_ff;
    if (D % 256 || F % 16 || K < 1 || K > E || E > 1024) return ORC_ERR_ARG;
    float *xf = (float *)malloc(sizeof(float) * (size_t)D);
    int8_t *qx = (int8_t *)malloc((size_t)D);
    float *lg = (float *)malloc(sizeof(float) * (size_t)E);
    int32_t *ag = (int32_t *)malloc(sizeof(int32_t) * (size_t)F);
    int32_t *au = (int32_t *)malloc(sizeof(int32_t) * (size_t)F);
    float *h = (float *)malloc(sizeof(float) * (size_t)F);
    int8_t *qh = (int8_t *)malloc((size_t)F);
    int32_t *ad = (int32_t *)malloc(sizeof(int32_t) * (size_t)D);
    float *ye = (float *)malloc(sizeof(float) * (size_t)D);
    int rc = ORC_OK;
    if (!xf || !qx || !lg || !ag || !au || !h || !qh || !ad || !ye) rc = ORC_ERR_OOM;
    int32_t idx[1024];
    float w[1024];
    const int32_t WD = D / 16, WF = F / 16;

    for (int32_t i = 0; i < n && rc == ORC_OK; i++) {
        int32_t t = tokens[i];
        for (int32_t j = 0; j < D; j++) xf[j] = orc_bf16_to_f32(x[(int64_t)t * D + j]);
        rc = orc_route_token(sh, wt, xf, lg, idx, w);
        if (rc) break;
        float sx;
        orc_quantize_row(xf, D, qx, &sx);
        if (taps) {
            if (taps->q_x) memcpy(taps->q_x + (int64_t)i * D, qx, (size_t)D);
            if (taps->s_x) taps->s_x[i] = sx;
            if (taps->logits) memcpy(taps->logits + (int64_t)i * E, lg, sizeof(float) * (size_t)E);
            if (taps->topk_idx) memcpy(taps->topk_idx + (int64_t)i * K, idx, sizeof(int32_t) * (size_t)K);
            if (taps->topk_w) memcpy(taps->topk_w + (int64_t)i * K, w, sizeof(float) * (size_t)K);
        }
        float *yt = y + (int64_t)i * D;
        for (int32_t c = 0; c < D; c++) yt[c] = 0.0f;

        for (int32_t k = 0; k < K; k++) {
            int32_t e = idx[k];
            /* gate and up: ternary rows of length D against q_x */
            for (int32_t r = 0; r < F; r++) {
                const uint32_t *rg = wt->w_gate + ((int64_t)e * F + r) * WD;
                const uint32_t *ru = wt->w_up + ((int64_t)e * F + r) * WD;
                int32_t sg = 0, su = 0;
                for (int32_t j = 0; j < D; j++) {
                    int vg = orc_ternary_at(rg, j), vu = orc_ternary_at(ru, j);
                    if (vg == 1) sg += qx[j]; else if (vg == -1) sg -= qx[j];
                    if (vu == 1) su += qx[j]; else if (vu == -1) su -= qx[j];
                }
                ag[r] = sg;
                au[r] = su;
                float g = (float)sg * (wt->alpha_gate[(int64_t)e * F + r] * sx);
                float u = (float)su * (wt->alpha_up[(int64_t)e * F + r] * sx);
                float silu = g / (1.0f + orc_exp(-g));
                h[r] = silu * u;
            }
            float sh_;
            orc_quantize_row(h, F, qh, &sh_);
            /* down: ternary rows of length F against q_h */
            for (int32_t c = 0; c < D; c++) {
                const uint32_t *rd = wt->w_down + ((int64_t)e * D + c) * WF;
                int32_t sd = 0;
                for (int32_t r = 0; r < F; r++) {
                    int v = orc_ternary_at(rd, r);
                    if (v == 1) sd += qh[r]; else if (v == -1) sd -= qh[r];
                }
                ad[c] = sd;
                ye[c] = (float)sd * (wt->alpha_down[(int64_t)e * D + c] * sh_);
                yt[c] = fmaf(w[k], ye[c], yt[c]);
            }
            if (taps) {
                int64_t sk = (int64_t)i * K + k;
                if (taps->acc_gate) memcpy(taps->acc_gate + sk * F, ag, sizeof(int32_t) * (size_t)F);
                if (taps->acc_up) memcpy(taps->acc_up + sk * F, au, sizeof(int32_t) * (size_t)F);
                if (taps->h) memcpy(taps->h + sk * F, h, sizeof(float) * (size_t)F);
                if (taps->q_h) memcpy(taps->q_h + sk * F, qh, (size_t)F);
                if (taps->s_h) taps->s_h[sk] = sh_;
                if (taps->acc_down) memcpy(taps->acc_down + sk * D, ad, sizeof(int32_t) * (size_t)D);
                if (taps->y_e) memcpy(taps->y_e + sk * D, ye, sizeof(float) * (size_t)D);
            }
        }
    }
    free(xf); free(qx); free(lg); free(ag); free(au); free(h); free(qh); free(ad); free(ye);
    return rc;
}

/* ------------------------------------------------------------------ */
/* stack glue: RMSNorm to bf16, residual add                           */
/* ------------------------------------------------------------------ */
/*
 * Pre-norm before each layer, norm weights 1:  ms = (sum_j r_j^2) / D with the
 * sum in the same fixed order as the router logit (fmaf(r_j, r_j, acc) per
 * partial, pairwise tree), rms = sqrt(ms + 1e-6), x_j = bf16(r_j / rms).
 */
void orc_rmsnorm_bf16(const float *r, int32_t D, uint16_t *out)
{
    float p[32];
    for (int l = 0; l < 32; l++) {
        float acc = 0.0f;
        for (int32_t i = 0; i < D / 256; i++)
            for (int m = 0; m < 8; m++) {
                int32_t j = 256 * i + 8 * l + m;
                acc = fmaf(r[j], r[j], acc);
            }
        p[l] = acc;
    }
    float ms = orc_tree_sum32(p) / (float)D;
    float rms = sqrtf(ms + 1e-6f);
    for (int32_t j = 0; j < D; j++) out[j] = orc_f32_to_bf16(r[j] / rms);
}

/*
 * One step of the layer stack for the listed tokens: for each layer l,
 * x = RMSNorm(resid) to bf16, resid = resid + MoE_l(x).  resid is [n][D],
 * row i belonging to tokens[i]; layers[l] are the layer weights.
 */
int orc_stack_forward(const orc_shape *sh, const orc_weights *layers, int32_t n_layers,
                      float *resid, int32_t n)
{
    int32_t D = sh->d_model;
    uint16_t *xb = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n * D);
    float *y = (float *)malloc(sizeof(float) * (size_t)n * D);
    int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int rc = (xb && y && tok) ? ORC_OK : ORC_ERR_OOM;
    for (int32_t i = 0; i < n && rc == ORC_OK; i++) tok[i] = i;
    for (int32_t l = 0; l < n_layers && rc == ORC_OK; l++) {
        for (int32_t i = 0; i < n; i++) orc_rmsnorm_bf16(resid + (int64_t)i * D, D, xb + (int64_t)i * D);
        rc = orc_forward_tokens(sh, &layers[l], xb, tok, n, y, NULL);
        for (int64_t j = 0; rc == ORC_OK && j < (int64_t)n * D; j++) resid[j] = resid[j] + y[j];
    }
    free(xb); free(y); free(tok);
    return rc;
}
