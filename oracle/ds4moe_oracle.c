/*
 * ds4moe_oracle.c -- fp64 oracle of the routed Q2_K mixture-of-experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded C99
 * restatement of what the layer computes, written so that it can be checked
 * against the sources by eye.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the library's product path never
 * links, loads or calls it, and it shares no code, header or table with the
 * CUDA path.  Everything is computed in double precision; sums run
 * sequentially in index order.
 *
 * Sources (cited by page and section):
 *  [README-2bit]   "antirez/ds4" README, Korean translation (molayo1419.me),
 *                  paragraph on the 2-bit models: only the routed MoE experts
 *                  are quantised (up/gate IQ2_XXS, down Q2_K); shared experts,
 *                  projections and routing stay unquantised.
 *  [README-GLM]    same page, GLM 5.2 paragraph: routed gate/up may be Q2_K,
 *                  routed down Q2_K.
 *  [README-ack]    same page, acknowledgements: GGUF quantisation layouts and
 *                  tables were kept from llama.cpp/GGML, so the Q2_K block here
 *                  is the GGUF Q2_K super-block.
 *  [FAQ-softplus]  opensource-hub.com "antirez/ds4" FAQ, first entry (the
 *                  M1 Ultra router numeric check): the router score is
 *                  sqrt(softplus(x)); the naive fp32 log(1 + exp(x)) loses
 *                  precision near x = -12; the checked tolerance is 3e-6.
 *  [Layer]         the layer as the benchmark workloads state it: score =
 *                  sqrt(softplus(x . Wr (+ bias))), top-k with ties to the
 *                  lower expert index, weights normalised to sum 1,
 *                  y = sum_e w_e down_e(silu(gate_e x) * up_e x) + shared(x),
 *                  w = d*scale*q - dmin*min over 16 sub-blocks of 16.
 *
 * Readings where the sources are silent:
 *  - Q2_K byte order: scales[16], qs[64], d (fp16 LE), dmin (fp16 LE); 84 B.
 *  - Quant i of a block: h = i/128, r = i%128, j = r/32, l = r%32 gives
 *    q = (qs[32h + l] >> 2j) & 3, and its sub-block is i/16 (the GGUF order).
 *  - Selection ranks by the fp64 logit (sqrt o softplus is increasing); ties
 *    go to the lower expert index; slots are kept in descending order.
 *  - If the selected scores sum to 0, every selected weight is 1/k.
 *  - The logit bias is added before softplus, so it moves the weights too.
 *  - RMS renormalisation between chained layers: x' = bf16_rne(y /
 *    sqrt(mean(y^2) + 1e-6)) per token, no learned scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_QK 256          /* weights per Q2_K super-block                */
#define ORA_BLOCK_BYTES 84  /* 16 scales + 64 quant bytes + d + dmin       */

/* ---------------------------------------------------------------- formats */

/* bf16 bit pattern -> double (exact: bf16 is the top half of an fp32). */
double ora_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16 bit pattern -> double (exact). */
double ora_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* double -> bf16 bit pattern, rounded to nearest, ties to even (finite, normal range). */
uint16_t ora_double_to_bf16(double v)
{
    if (v == 0.0)
        return signbit(v) ? 0x8000 : 0;
    int e;
    double m = frexp(v, &e);                      /* |m| in [0.5, 1) */
    double r = nearbyint(ldexp(m, 8));            /* 8 significant bits, RNE */
    double q = ldexp(r, e - 8);                   /* exactly representable in bf16 */
    float f = (float)q;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ Q2_K */

/* Dequantise one 84-byte Q2_K super-block into 256 doubles  [README-2bit], [Layer].
 * For weight i: sub-block sb = i/16 with scale = low nibble of scales[sb] and
 * min = high nibble; q is the 2-bit quant at the reading's position; the value
 * is d*scale*q - dmin*min. */
void ora_q2k_dequant(const uint8_t *blk, double *w)
{
    const uint8_t *scales = blk;
    const uint8_t *qs = blk + 16;
    double d = ora_f16_to_double((uint16_t)(blk[80] | (blk[81] << 8)));
    double dmin = ora_f16_to_double((uint16_t)(blk[82] | (blk[83] << 8)));
    for (int i = 0; i < ORA_QK; ++i) {
        int sb = i / 16;
        int scale = scales[sb] & 0xF;
        int mn = scales[sb] >> 4;
        int h = i / 128, r = i % 128, j = r / 32, l = r % 32;
        int q = (qs[32 * h + l] >> (2 * j)) & 3;
        w[i] = d * scale * q - dmin * mn;
    }
}

/* Dot product of one Q2_K row (K/256 blocks) with a double vector, sequential in i. */
static double ora_q2k_row_dot(const uint8_t *row, int K, const double *v)
{
    double w[ORA_QK];
    double acc = 0.0;
    for (int b = 0; b < K / ORA_QK; ++b) {
        ora_q2k_dequant(row + (size_t)b * ORA_BLOCK_BYTES, w);
        for (int i = 0; i < ORA_QK; ++i)
            acc += w[i] * v[b * ORA_QK + i];
    }
    return acc;
}

/* ---------------------------------------------------------------- router */

/* softplus(l) = log(1 + e^l), in the overflow-free form max(l,0) + log1p(e^-|l|)  [FAQ-softplus]. */
double ora_softplus(double l)
{
    return fmax(l, 0.0) + log1p(exp(-fabs(l)));
}

/* Router score s = sqrt(softplus(l))  [FAQ-softplus]. */
double ora_score(double l)
{
    return sqrt(ora_softplus(l));
}

/* Router logit of one (token, expert): sum_i x_i * Wr_i in index order, then + bias. */
double ora_logit(const uint16_t *x, const uint16_t *wr_row, int H, const float *bias_e)
{
    double acc = 0.0;
    for (int i = 0; i < H; ++i)
        acc += ora_bf16_to_double(x[i]) * ora_bf16_to_double(wr_row[i]);
    if (bias_e)
        acc += (double)*bias_e;
    return acc;
}

/* Top-k of one token: k rounds of "largest logit not yet taken, lower index on ties",
 * then weights w_j = s_j / sum s (1/k each if the sum is 0)  [Layer]. */
void ora_route_token(const uint16_t *x, const uint16_t *wr, const float *bias, int E, int H, int k,
                     int32_t *idx, double *wts, double *logits)
{
    double *lg = logits ? logits : (double *)malloc(sizeof(double) * (size_t)E);
    char *taken = (char *)calloc((size_t)E, 1);
    for (int e = 0; e < E; ++e)
        lg[e] = ora_logit(x, wr + (size_t)e * H, H, bias ? bias + e : NULL);
    double ssum = 0.0;
    double s[64];
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || lg[e] > lg[best]))
                best = e;                          /* strict '>' keeps the lower index on ties */
        taken[best] = 1;
        idx[j] = best;
        s[j] = ora_score(lg[best]);
        ssum += s[j];
    }
    for (int j = 0; j < k; ++j)
        wts[j] = ssum > 0.0 ? s[j] / ssum : 1.0 / k;
    free(taken);
    if (!logits)
        free(lg);
}

/* Route T tokens: idx [T][k], weights [T][k], logits [T][E] (optional). */
void ora_route(const uint16_t *x, int T, int H, const uint16_t *wr, const float *bias, int E, int k,
               int32_t *idx, double *wts, double *logits)
{
    for (int t = 0; t < T; ++t)
        ora_route_token(x + (size_t)t * H, wr, bias, E, H, k, idx + (size_t)t * k, wts + (size_t)t * k,
                        logits ? logits + (size_t)t * E : NULL);
}

/* Token->expert permutation: counts per expert, exclusive scan into offsets[E+1], and each
 * (token, slot) pair placed at offsets[e] + (number of earlier pairs of e in token order).
 * sorted_token/sorted_slot list the pairs in that order; inv_pos[t*k+j] is the position. */
void ora_permute(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *sorted_token,
                 int32_t *sorted_slot, int32_t *inv_pos)
{
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int e = 0; e <= E; ++e)
        offsets[e] = 0;
    for (int p = 0; p < T * k; ++p)
        offsets[idx[p] + 1] += 1;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] += offsets[e];
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            int pos = offsets[e] + fill[e]++;
            sorted_token[pos] = t;
            sorted_slot[pos] = j;
            inv_pos[t * k + j] = pos;
        }
    free(fill);
}

/* ---------------------------------------------------------------- experts */

static double ora_silu(double g)
{
    return g / (1.0 + exp(-g));
}

/* One routed expert on one token  [Layer]:
 * g_r = W_g[r,:].x, u_r = W_u[r,:].x, h_r = silu(g_r) u_r (r < I); o_c = W_d[c,:].h (c < H).
 * gate/up: I rows of H/256 blocks; down: H rows of I/256 blocks.  g, u, h, o may be NULL. */
void ora_expert(const uint8_t *gate, const uint8_t *up, const uint8_t *down, int H, int I, const double *x,
                double *g_out, double *u_out, double *h_out, double *o_out)
{
    size_t row_gu = (size_t)(H / ORA_QK) * ORA_BLOCK_BYTES;
    size_t row_d = (size_t)(I / ORA_QK) * ORA_BLOCK_BYTES;
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    for (int r = 0; r < I; ++r) {
        double g = ora_q2k_row_dot(gate + r * row_gu, H, x);
        double u = ora_q2k_row_dot(up + r * row_gu, H, x);
        h[r] = ora_silu(g) * u;
        if (g_out) g_out[r] = g;
        if (u_out) u_out[r] = u;
        if (h_out) h_out[r] = h[r];
    }
    if (o_out)
        for (int c = 0; c < H; ++c)
            o_out[c] = ora_q2k_row_dot(down + c * row_d, I, h);
    free(h);
}

/* Shared expert on one token, bf16 weights  [README-2bit] (kept unquantised):
 * S = W_sd (silu(W_sg x) * (W_su x)); W_sg, W_su [Is][H], W_sd [H][Is], row-major. */
void ora_shared(const uint16_t *sg, const uint16_t *su, const uint16_t *sd, int H, int Is, const double *x,
                double *h_out, double *s_out)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)(Is > 0 ? Is : 1));
    for (int r = 0; r < Is; ++r) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < H; ++i) {
            g += ora_bf16_to_double(sg[(size_t)r * H + i]) * x[i];
            u += ora_bf16_to_double(su[(size_t)r * H + i]) * x[i];
        }
        h[r] = ora_silu(g) * u;
        if (h_out) h_out[r] = h[r];
    }
    for (int c = 0; c < H; ++c) {
        double acc = 0.0;
        for (int r = 0; r < Is; ++r)
            acc += ora_bf16_to_double(sd[(size_t)c * Is + r]) * h[r];
        s_out[c] = acc;
    }
    free(h);
}

/* ------------------------------------------------------------------ layer */

typedef struct {
    int hidden, n_experts, top_k, inter, shared_inter;
    const uint8_t *gate, *up, *down;      /* [E][rows][K/256][84] */
    const uint16_t *router;               /* [E][H] bf16 */
    const float *bias;                    /* [E] or NULL */
    const uint16_t *sg, *su, *sd;         /* shared expert, NULL if shared_inter == 0 */
} ora_layer;

/* Layer output for the tokens listed in `tokens` (n of them; all T when tokens == NULL):
 * y[n][H] = sum_j w_j o^(j) + S, slots summed in ascending order, then the shared output.
 * idx/wts ([n][k], optional) receive the routing of those tokens. */
void ora_layer_forward(const ora_layer *L, const uint16_t *x, int T, const int32_t *tokens, int n,
                       double *y, int32_t *idx_out, double *wts_out)
{
    int H = L->hidden, E = L->n_experts, k = L->top_k, I = L->inter, Is = L->shared_inter;
    size_t mat_gu = (size_t)I * (H / ORA_QK) * ORA_BLOCK_BYTES;
    size_t mat_d = (size_t)H * (I / ORA_QK) * ORA_BLOCK_BYTES;
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *o = (double *)malloc(sizeof(double) * (size_t)H);
    double *s = (double *)malloc(sizeof(double) * (size_t)H);
    int32_t idx[64];
    double wts[64];
    int count = tokens ? n : T;
    for (int a = 0; a < count; ++a) {
        int t = tokens ? tokens[a] : a;
        const uint16_t *xt = x + (size_t)t * H;
        for (int i = 0; i < H; ++i)
            xd[i] = ora_bf16_to_double(xt[i]);
        ora_route_token(xt, L->router, L->bias, E, H, k, idx, wts, NULL);
        double *yt = y + (size_t)a * H;
        for (int c = 0; c < H; ++c)
            yt[c] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[j];
            ora_expert(L->gate + e * mat_gu, L->up + e * mat_gu, L->down + e * mat_d, H, I, xd,
                       NULL, NULL, NULL, o);
            for (int c = 0; c < H; ++c)
                yt[c] += wts[j] * o[c];
        }
        if (Is > 0) {
            ora_shared(L->sg, L->su, L->sd, H, Is, xd, NULL, s);
            for (int c = 0; c < H; ++c)
                yt[c] += s[c];
        }
        if (idx_out)
            for (int j = 0; j < k; ++j) {
                idx_out[(size_t)a * k + j] = idx[j];
                wts_out[(size_t)a * k + j] = wts[j];
            }
    }
    free(xd);
    free(o);
    free(s);
}

/* Brute-force dense evaluation for tiny shapes: every expert runs on every token from fully
 * dequantised dense matrices, and each output is multiplied by a mask weight that is w_j if
 * the expert holds slot j and 0 otherwise.  The slot comes from rank counting (how many
 * experts beat e: a larger logit, or an equal one at a lower index), not from the iterative
 * selection of ora_route_token, so the two formulations check each other. */
int ora_dense_forward(const ora_layer *L, const uint16_t *x, int T, double *y)
{
    int H = L->hidden, E = L->n_experts, k = L->top_k, I = L->inter, Is = L->shared_inter;
    int nbh = H / ORA_QK, nbi = I / ORA_QK;
    double *Wg = (double *)malloc(sizeof(double) * (size_t)E * I * H);
    double *Wu = (double *)malloc(sizeof(double) * (size_t)E * I * H);
    double *Wd = (double *)malloc(sizeof(double) * (size_t)E * H * I);
    double *lg = (double *)malloc(sizeof(double) * (size_t)E);
    double *mask = (double *)malloc(sizeof(double) * (size_t)E);
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *hh = (double *)malloc(sizeof(double) * (size_t)(I > Is ? I : Is));
    char *sel = (char *)malloc((size_t)E);
    if (!Wg || !Wu || !Wd || !lg || !mask || !xd || !hh || !sel)
        return -1;
    /* dense dequantisation of every matrix */
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < I; ++r)
            for (int b = 0; b < nbh; ++b) {
                size_t blk = (((size_t)e * I + r) * nbh + b) * ORA_BLOCK_BYTES;
                ora_q2k_dequant(L->gate + blk, Wg + ((size_t)e * I + r) * H + b * ORA_QK);
                ora_q2k_dequant(L->up + blk, Wu + ((size_t)e * I + r) * H + b * ORA_QK);
            }
    for (int e = 0; e < E; ++e)
        for (int c = 0; c < H; ++c)
            for (int b = 0; b < nbi; ++b) {
                size_t blk = (((size_t)e * H + c) * nbi + b) * ORA_BLOCK_BYTES;
                ora_q2k_dequant(L->down + blk, Wd + ((size_t)e * H + c) * I + b * ORA_QK);
            }
    for (int t = 0; t < T; ++t) {
        const uint16_t *xt = x + (size_t)t * H;
        for (int i = 0; i < H; ++i)
            xd[i] = ora_bf16_to_double(xt[i]);
        for (int e = 0; e < E; ++e)
            lg[e] = ora_logit(xt, L->router + (size_t)e * H, H, L->bias ? L->bias + e : NULL);
        /* mask from ranks: expert e is selected when fewer than k experts beat it */
        double ssum = 0.0;
        for (int e = 0; e < E; ++e) {
            int rank = 0;
            for (int f = 0; f < E; ++f)
                if (lg[f] > lg[e] || (lg[f] == lg[e] && f < e))
                    ++rank;
            sel[e] = rank < k;
            mask[e] = sel[e] ? ora_score(lg[e]) : 0.0;
            ssum += mask[e];
        }
        for (int e = 0; e < E; ++e)
            mask[e] = !sel[e] ? 0.0 : (ssum > 0.0 ? mask[e] / ssum : 1.0 / k);
        double *yt = y + (size_t)t * H;
        for (int c = 0; c < H; ++c)
            yt[c] = 0.0;
        for (int e = 0; e < E; ++e) {
            for (int r = 0; r < I; ++r) {
                double g = 0.0, u = 0.0;
                for (int i = 0; i < H; ++i) {
                    g += Wg[((size_t)e * I + r) * H + i] * xd[i];
                    u += Wu[((size_t)e * I + r) * H + i] * xd[i];
                }
                hh[r] = ora_silu(g) * u;
            }
            for (int c = 0; c < H; ++c) {
                double acc = 0.0;
                for (int r = 0; r < I; ++r)
                    acc += Wd[((size_t)e * H + c) * I + r] * hh[r];
                yt[c] += mask[e] * acc;
            }
        }
        if (Is > 0) {
            for (int r = 0; r < Is; ++r) {
                double g = 0.0, u = 0.0;
                for (int i = 0; i < H; ++i) {
                    g += ora_bf16_to_double(L->sg[(size_t)r * H + i]) * xd[i];
                    u += ora_bf16_to_double(L->su[(size_t)r * H + i]) * xd[i];
                }
                hh[r] = ora_silu(g) * u;
            }
            for (int c = 0; c < H; ++c) {
                double acc = 0.0;
                for (int r = 0; r < Is; ++r)
                    acc += ora_bf16_to_double(L->sd[(size_t)c * Is + r]) * hh[r];
                yt[c] += acc;
            }
        }
    }
    free(Wg); free(Wu); free(Wd); free(lg); free(mask); free(xd); free(hh); free(sel);
    return 0;
}

/* RMS renormalisation between chained layers, per token:
 * x'[t,i] = bf16_rne( y[t,i] / sqrt(mean_i y[t,i]^2 + 1e-6) ). */
void ora_rms_renorm(const double *y, int T, int H, uint16_t *x_next)
{
    for (int t = 0; t < T; ++t) {
        const double *yt = y + (size_t)t * H;
        double ss = 0.0;
        for (int i = 0; i < H; ++i)
            ss += yt[i] * yt[i];
        double denom = sqrt(ss / H + 1e-6);
        for (int i = 0; i < H; ++i)
            x_next[(size_t)t * H + i] = ora_double_to_bf16(yt[i] / denom);
    }
}
