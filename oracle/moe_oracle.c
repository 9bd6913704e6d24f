/*
 * ORACLE - test infrastructure, not product code.
 *
 * A plain, slow, fp64 CPU restatement of the quantized sparse-MoE feed-forward
 * layer.  Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg
 * (and its reference arm) call it.  It shares no code, header, table or helper
 * with the CUDA library; it reads the canonical packed layout that the public
 * header defines in words, and nothing else.
 *
 * What the layer is, from the pages:
 *   - "Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB GPU?" (video transcript,
 *     1:37-2:16): each of the 48 layers holds 512 small expert networks; for
 *     every token a router in every layer picks 10 of them, plus one shared
 *     expert that always runs.
 *   - same transcript, 3:36-3:47: the routed experts' results and the rest of
 *     the token's work are combined into one result ("same ticket").
 *   - "Qwen3.8-Flash-Next on RTX 5090 + 64GB" (en.wiselychen.com), section
 *     "The 30-Second Overview": 512 experts per layer, 10 routed + 1 shared.
 * What the pages leave open and this library's specification fixes (readings
 * that the design notes list):
 *   - expert network = SwiGLU: h = silu(W_g x) * (W_u x), y = W_d h;
 *   - routing weights = softmax over all E logits, renormalised over the
 *     chosen k; shared expert weight 1;
 *   - block formats Q4B32 and Q3B32 (the pages name IQ3_S, IQ2_XS, Q2_0 ...
 *     but never define a layout; "Running Qwen3.8-Flash-Next on a 4090 24GB",
 *     section "The engine rejects Unsloth's embedding format"), and the
 *     2-bit Q2B32 for the pages' fastest size, Q2_0 ("Strata: Qwen3.8-Flash-
 *     Next (125B Moe) on a 8GB+ Nvidia GPU", tables "How fast?" and "The
 *     size"; video transcript 6:18-6:32), defined the same way: 32 codes and
 *     one fp16 scale, the zero point at half the code range.
 *
 * Every function below computes in fp64.  Parity of each is pinned by the
 * CPU tests against hand-built blocks, closed forms, brute force and the
 * invariants of the specification.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_Q4B32 1
#define ORACLE_Q3B32 2
#define ORACLE_Q2B32 3

/* IEEE 754 binary16 -> double, written from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h)
{
    int sign = h >> 15, ex = (h >> 10) & 31, fr = h & 1023;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -24);               /* subnormal: fr * 2^-10 * 2^-14 */
    else if (ex == 31)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + fr), ex - 25);  /* (1 + fr/1024) * 2^(ex-15) */
    return sign ? -v : v;
}

/* bfloat16 -> double: the upper half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Code j (0..31) of one packed block.
 * Q4B32: 16 bytes, two 4-bit codes per byte; byte b holds code 2b in its low
 *        nibble and code 2b+1 in its high nibble.
 * Q3B32: 12 bytes read as one 96-bit little-endian integer; code j is bits
 *        3j..3j+2 (bit 0 of byte 0 is the least significant bit).
 * Q2B32: 8 bytes read as one 64-bit little-endian integer; code j is bits
 *        2j..2j+1, i.e. byte j/4, starting at bit 2*(j mod 4). */
int oracle_code(int fmt, const uint8_t *blk, int j)
{
    if (fmt == ORACLE_Q4B32) {
        uint8_t byte = blk[j >> 1];
        return (j & 1) ? (byte >> 4) : (byte & 15);
    }
    if (fmt == ORACLE_Q2B32)
        return (blk[j >> 2] >> (2 * (j & 3))) & 3;
    int v = 0;
    for (int t = 0; t < 3; ++t) {
        int bit = 3 * j + t;
        v |= ((blk[bit >> 3] >> (bit & 7)) & 1) << t;
    }
    return v;
}

/* Weight j of a block: w = s * (q - 8) for Q4B32, w = s * (q - 4) for Q3B32,
 * w = s * (q - 2) for Q2B32, s the block's fp16 scale. */
double oracle_weight(int fmt, const uint8_t *blk, uint16_t scale, int j)
{
    int zero = (fmt == ORACLE_Q4B32) ? 8 : (fmt == ORACLE_Q2B32) ? 2 : 4;
    return oracle_half_to_double(scale) * (double)(oracle_code(fmt, blk, j) - zero);
}

static int block_bytes(int fmt) { return fmt == ORACLE_Q4B32 ? 16 : (fmt == ORACLE_Q2B32) ? 8 : 12; }

/* y[r] = sum_k W[r][k] x[k] for a packed matrix of `rows` rows and K columns,
 * blocks of 32 running along k: codes [rows][K/32][B], scales [rows][K/32]. */
void oracle_qmatvec(int fmt, int rows, int K, const uint8_t *codes,
                    const uint16_t *scales, const double *x, double *y)
{
    int nb = K / 32, B = block_bytes(fmt);
    for (int r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int b = 0; b < nb; ++b) {
            const uint8_t *blk = codes + ((size_t)r * nb + b) * B;
            uint16_t s = scales[(size_t)r * nb + b];
            for (int j = 0; j < 32; ++j)
                acc += oracle_weight(fmt, blk, s, j) * x[b * 32 + j];
        }
        y[r] = acc;
    }
}

/* Dense fp64 copy of a packed matrix: out[r][k] = W[r][k] = s_rb * (q - zero)
 * for k in block b, straight from the block definition (one scale decode per
 * block).  codes [rows][K/32][B], scales [rows][K/32], out [rows][K]. */
void oracle_dequant(int fmt, int rows, int K, const uint8_t *codes,
                    const uint16_t *scales, double *out)
{
    int nb = K / 32, B = block_bytes(fmt);
    int zero = (fmt == ORACLE_Q4B32) ? 8 : (fmt == ORACLE_Q2B32) ? 2 : 4;
    for (int r = 0; r < rows; ++r)
        for (int b = 0; b < nb; ++b) {
            const uint8_t *blk = codes + ((size_t)r * nb + b) * B;
            double s = oracle_half_to_double(scales[(size_t)r * nb + b]);
            double *o = out + (size_t)r * K + (size_t)b * 32;
            for (int j = 0; j < 32; ++j)
                o[j] = s * (double)(oracle_code(fmt, blk, j) - zero);
        }
}

/* silu(z) = z / (1 + e^-z). */
double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/* One SwiGLU expert on one token: g = W_g x, u = W_u x, h = silu(g) * u,
 * y = W_d h.  Gate/up are [I][d] (blocks along d), down is [d][I] (blocks
 * along I).  h_out (length I) may be NULL. */
void oracle_expert(int fmt, int d, int I,
                   const uint8_t *gc, const uint16_t *gs,
                   const uint8_t *uc, const uint16_t *us,
                   const uint8_t *dc, const uint16_t *ds,
                   const double *x, double *y, double *h_out)
{
    double *g = malloc(sizeof(double) * I);
    double *u = malloc(sizeof(double) * I);
    double *h = malloc(sizeof(double) * I);
    oracle_qmatvec(fmt, I, d, gc, gs, x, g);
    oracle_qmatvec(fmt, I, d, uc, us, x, u);
    for (int i = 0; i < I; ++i)
        h[i] = oracle_silu(g[i]) * u[i];
    oracle_qmatvec(fmt, d, I, dc, ds, h, y);
    if (h_out)
        memcpy(h_out, h, sizeof(double) * I);
    free(g);
    free(u);
    free(h);
}

/* Router: logit[e] = sum_i x[i] W_r[e][i] (+ bias[e]); W_r fp32 [E][d],
 * bias fp32 [E] or NULL. */
void oracle_router_logits(int d, int E, const double *x, const float *Wr,
                          const float *bias, double *logits)
{
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += x[i] * (double)Wr[(size_t)e * d + i];
        logits[e] = acc + (bias ? (double)bias[e] : 0.0);
    }
}

typedef struct { double v; int id; } scored;

static int by_logit_desc(const void *a, const void *b)
{
    const scored *p = a, *q = b;
    if (p->v > q->v) return -1;
    if (p->v < q->v) return 1;
    return p->id - q->id;              /* equal logits: lower expert id first */
}

/* Routing of one token.  p = softmax over all E logits; the k experts with
 * the largest p are chosen (ordered by p descending, equal p -> lower id;
 * softmax is strictly increasing in the logit, so this is the logit order);
 * w_j = p_j / sum of the chosen p.  gap = (k-th largest logit) - ((k+1)-th),
 * +inf when k == E. */
void oracle_route(int E, int k, const double *logits, int32_t *ids, double *w,
                  double *gap)
{
    scored *s = malloc(sizeof(scored) * E);
    double *p = malloc(sizeof(double) * E);
    double mx = -INFINITY, z = 0.0;
    for (int e = 0; e < E; ++e)
        if (logits[e] > mx) mx = logits[e];
    for (int e = 0; e < E; ++e) {
        p[e] = exp(logits[e] - mx);
        z += p[e];
    }
    for (int e = 0; e < E; ++e) {
        p[e] /= z;
        s[e].v = logits[e];
        s[e].id = e;
    }
    qsort(s, E, sizeof(scored), by_logit_desc);
    double sel = 0.0;
    for (int j = 0; j < k; ++j) {
        ids[j] = s[j].id;
        sel += p[s[j].id];
    }
    for (int j = 0; j < k; ++j)
        w[j] = p[ids[j]] / sel;
    *gap = (k < E) ? s[k - 1].v - s[k].v : INFINITY;
    free(s);
    free(p);
}

/* The whole layer for T tokens, each token on its own:
 *   logits -> route -> y_t = sum_j w_tj * expert_{ids_tj}(x_t) + sum_s shared_s(x_t).
 * x: bf16 bits [T][d].  Routed expert tensors are the canonical arrays of all
 * E experts: gate/up codes [E][I][d/32][B], down codes [E][d][I/32][B], scales
 * without the last dim.  Shared: same with n_shared experts of size I_s.
 * Outputs: y fp64 [T][d], ids [T][k], w fp64 [T][k], gap fp64 [T]. */
void oracle_moe_layer(int fmt, int d, int E, int I, int k, int n_shared, int I_s,
                      int T, const uint16_t *x_bf16,
                      const float *Wr, const float *bias,
                      const uint8_t *gc, const uint16_t *gs,
                      const uint8_t *uc, const uint16_t *us,
                      const uint8_t *dc, const uint16_t *ds,
                      const uint8_t *sgc, const uint16_t *sgs,
                      const uint8_t *suc, const uint16_t *sus,
                      const uint8_t *sdc, const uint16_t *sds,
                      double *y, int32_t *ids, double *w, double *gap)
{
    int B = block_bytes(fmt);
    size_t gu_codes = (size_t)I * (d / 32) * B, gu_sc = (size_t)I * (d / 32);
    size_t dn_codes = (size_t)d * (I / 32) * B, dn_sc = (size_t)d * (I / 32);
    size_t sgu_codes = (size_t)I_s * (d / 32) * B, sgu_sc = (size_t)I_s * (d / 32);
    size_t sdn_codes = (size_t)d * (I_s / 32) * B, sdn_sc = (size_t)d * (I_s / 32);
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double *x = malloc(sizeof(double) * d);
        double *lg = malloc(sizeof(double) * E);
        double *ye = malloc(sizeof(double) * d);
        double *yt = y + (size_t)t * d;
        for (int i = 0; i < d; ++i)
            x[i] = oracle_bf16_to_double(x_bf16[(size_t)t * d + i]);
        oracle_router_logits(d, E, x, Wr, bias, lg);
        oracle_route(E, k, lg, ids + (size_t)t * k, w + (size_t)t * k, gap + t);
        for (int i = 0; i < d; ++i)
            yt[i] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[(size_t)t * k + j];
            oracle_expert(fmt, d, I, gc + e * gu_codes, gs + e * gu_sc,
                          uc + e * gu_codes, us + e * gu_sc,
                          dc + e * dn_codes, ds + e * dn_sc, x, ye, NULL);
            double wj = w[(size_t)t * k + j];
            for (int i = 0; i < d; ++i)
                yt[i] += wj * ye[i];
        }
        for (int s = 0; s < n_shared; ++s) {
            oracle_expert(fmt, d, I_s, sgc + s * sgu_codes, sgs + s * sgu_sc,
                          suc + s * sgu_codes, sus + s * sgu_sc,
                          sdc + s * sdn_codes, sds + s * sdn_sc, x, ye, NULL);
            for (int i = 0; i < d; ++i)
                yt[i] += ye[i];
        }
        free(x);
        free(lg);
        free(ye);
    }
}

/* Pre-normalisation of the 48-layer stack (a reading: the pages only say
 * the layers are stacked; see the design notes): out = r / sqrt(mean(r^2) + eps). */
void oracle_rmsnorm(int d, const double *r, double eps, double *out)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i)
        ss += r[i] * r[i];
    double inv = 1.0 / sqrt(ss / d + eps);
    for (int i = 0; i < d; ++i)
        out[i] = r[i] * inv;
}

/* double -> bfloat16 bits with one round-to-nearest-even step, written from
 * the format's definition (8 significant bits, binary32's exponent range,
 * subnormal spacing 2^-133).  Used for the bf16 layer input of the stack and
 * to compare bf16 outputs. */
uint16_t oracle_round_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    double a = fabs(v), q;
    if (a == 0.0) {
        q = 0.0;
    } else if (a < ldexp(1.0, -126)) {
        q = nearbyint(ldexp(a, 133));
        q = ldexp(q, -133);
    } else {
        int e;
        double m = frexp(a, &e);                 /* a = m * 2^e, m in [0.5, 1) */
        q = ldexp(nearbyint(ldexp(m, 8)), e - 8);
    }
    float f = (float)q;                          /* exact: q has <= 9 significant bits */
    if (q > 3.3895313892515355e38)               /* beyond the largest finite bf16 */
        f = INFINITY;
    uint32_t u;
    memcpy(&u, &f, 4);
    u >>= 16;
    if (v < 0 || (v == 0.0 && signbit(v)))
        u |= 0x8000;
    return (uint16_t)u;
}

void oracle_round_bf16_array(size_t n, const double *v, uint16_t *out)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_round_bf16(v[i]);
}

void oracle_bf16_to_double_array(size_t n, const uint16_t *b, double *out)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_to_double(b[i]);
}

void oracle_half_to_double_array(size_t n, const uint16_t *h, double *out)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_half_to_double(h[i]);
}
