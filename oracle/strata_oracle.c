/*
 * strata_oracle.c -- plain CPU oracle of the Strata MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What the layer is.  The pages fix the outline: 512 experts per layer, 10
 * routed and 1 shared expert per token ("Strata Runs 125B Qwen3.8-Flash-Next on
 * a 12GB Gaming GPU at Up to 94 Tokens/s", section "What it is"; "Strata ...
 * gaming PC", spec table, rows "Experts" and "Hidden dimension"), routers and
 * shared experts evaluated on the GPU ("How a 125B model fits in 12 GB"), and
 * 2-3 bit quantised expert builds ("Caveats"; the Q2_0 build in "The numbers,
 * measured by the author").  The layer specification this library implements
 * fills in the rest: fp32 router logits plus an optional per-expert bias,
 * softmax over all experts, top-k with the lower expert id winning ties,
 * renormalisation over the k picks, SwiGLU experts whose weights are 2-bit
 * (w = d*(q-1.5)) or 3-bit (w = d*(q-3.5)) codes in blocks of 32 along the
 * input dimension with one fp16 scale d per block, one always-on shared expert
 * added with weight 1, and a fixed-order combine rounded once to bf16.
 *
 * Precision.  Expert arithmetic runs in fp64 (the pages fix no precision for
 * it).  Two steps decide integers or bf16 codes, and there both sides of a
 * parity test must decide in the same precision, so they are fp32 here, in a
 * stated summation order:
 *   - router logits: fp32, 32 interleaved partial sums p_l over i = l, l+32,
 *     ... (each p_l = fmaf(x_i, W_i, p_l) in ascending i), then a halving tree
 *     p_l += p_{l+s} for s = 16, 8, 4, 2, 1, then + bias;
 *   - RMSNorm of the 48-layer stack: the sum of squares in the same order,
 *     r = 1/sqrtf(ss/H + 1e-6f), xn = bf16(h*r).
 * Every other value is computed in double.
 *
 * Build: gcc -O2 -ffp-contract=off -mfma -shared -fPIC (no SIMD intrinsics;
 * -mfma only makes the explicit fmaf calls a single instruction).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* IEEE binary16 bit pattern -> exact double. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (ex == 0)
        v = ldexp((double)man, -24);            /* subnormal: man * 2^-24 */
    else if (ex == 31)
        v = man ? NAN : INFINITY;
    else
        v = ldexp((double)(man | 0x400), ex - 25); /* (1024+man) * 2^(ex-15-10) */
    return sign ? -v : v;
}

/* bf16 bit pattern -> exact float. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to a binary format with `mbits` explicit mantissa bits,
 * exponent range [emin, emax] for normals, round to nearest even, directly
 * from the double (no intermediate rounding).  Returns the rounded value as a
 * double (exact), +-inf on overflow. */
static double round_to_format(double v, int mbits, int emin, int emax)
{
    if (v == 0.0 || isnan(v) || isinf(v))
        return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) -> unbiased exp = e-1 */
    int ue = e - 1;
    if (ue < emin)
        ue = emin;                /* subnormal range: fixed quantum */
    double q = ldexp(1.0, ue - mbits); /* quantum (ulp) at this exponent */
    double n = nearbyint(a / q);  /* a/q is exact (power-of-two scaling); default mode is RNE */
    double r = n * q;
    /* the largest finite value is (2 - 2^-mbits) * 2^emax */
    double maxf = ldexp(2.0 - ldexp(1.0, -mbits), emax);
    if (r > maxf)
        r = INFINITY;
    return v < 0 ? -r : r;
}

/* double -> bf16 bit pattern, round to nearest even (directly from double). */
uint16_t orc_f64_to_bf16(double v)
{
    double r = round_to_format(v, 7, -126, 127);
    float f = (float)r;           /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(v))
        return 0x7fc0;
    return (uint16_t)(u >> 16);
}

/* double -> fp16 bit pattern, round to nearest even. */
uint16_t orc_f64_to_f16(double v)
{
    if (isnan(v))
        return 0x7e00;
    double r = round_to_format(v, 10, -14, 15);
    uint16_t sign = (r < 0 || (r == 0 && signbit(r))) ? 0x8000 : 0;
    double a = fabs(r);
    if (isinf(a))
        return sign | 0x7c00;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);
    int ue = e - 1;
    if (ue < -14)                 /* subnormal: a = man * 2^-24 */
        return sign | (uint16_t)(a / ldexp(1.0, -24));
    uint16_t man = (uint16_t)(ldexp(a, -ue) * 1024.0 - 1024.0);
    return sign | (uint16_t)((ue + 15) << 10) | man;
}

/* ------------------------------------------------------------------------ */
/* Quantised block format                                                    */
/* ------------------------------------------------------------------------ */

/* Code q of element j (0..31) of one block.
 *  1-bit: 4 bytes; element j is bit j%8 of byte j/8.
 *  2-bit: 8 bytes; element j sits in bits 2*(j%4) .. 2*(j%4)+1 of byte j/4.
 *  3-bit: 12 bytes read as one little-endian 96-bit integer; element j sits in
 *         bits 3j .. 3j+2.
 * (All three: element j occupies bits bits*j .. bits*j+bits-1 of the block
 * read as one little-endian integer.) */
int orc_code(const uint8_t *block, int bits, int j)
{
    if (bits == 2)
        return (block[j >> 2] >> (2 * (j & 3))) & 3;
    int bit = bits * j, q = 0;
    for (int b = 0; b < bits; b++) {
        int p = bit + b;
        q |= ((block[p >> 3] >> (p & 7)) & 1) << b;
    }
    return q;
}

/* Centre of the code range: w = d * (q - centre), centre = (2^bits - 1) / 2
 * (0.5, 1.5, 3.5 for 1, 2, 3 bits). */
static double code_centre(int bits) { return ((double)(1 << bits) - 1.0) / 2.0; }

/* Exact dequantised weight (row r, column c) of a rows x cols matrix stored in
 * the packed format: codes [rows][cols/32][4*bits], scales [rows][cols/32]. */
double orc_weight(const uint8_t *codes, const uint16_t *scales, int bits, int cols,
                  int r, int c)
{
    int nb = cols / 32;
    const uint8_t *blk = codes + ((size_t)r * nb + c / 32) * (size_t)(4 * bits);
    double d = orc_f16_to_f64(scales[(size_t)r * nb + c / 32]);
    int q = orc_code(blk, bits, c % 32);
    return d * ((double)q - code_centre(bits));
}

/* Dequantise rows [row0, row0+nrows) of one matrix into out[nrows][cols]
 * (exact values; test hook for the bit-exact dequant check). */
void orc_dequant_rows(const uint8_t *codes, const uint16_t *scales, int bits, int cols,
                      int row0, int nrows, double *out)
{
    for (int r = 0; r < nrows; r++)
        for (int c = 0; c < cols; c++)
            out[(size_t)r * cols + c] = orc_weight(codes, scales, bits, cols, row0 + r, c);
}

/* Matrix m (0 gate [I,H], 1 up [I,H], 2 down [H,I]) of one expert whose
 * packed codes/scales start at codes_e/scales_e. */
static void mat_ptrs(const uint8_t *codes_e, const uint16_t *scales_e, int bits, int H, int I,
                     int m, const uint8_t **c, const uint16_t **s)
{
    size_t w = (size_t)H * I;
    *c = codes_e + (size_t)m * (w * bits / 8);
    *s = scales_e + (size_t)m * (w / 32);
}

/* ------------------------------------------------------------------------ */
/* Router                                                                    */
/* ------------------------------------------------------------------------ */

/* fp32 dot product of a bf16 vector and an fp32 vector in the canonical order
 * (32 interleaved fma partial sums, then a halving tree). */
static float canon_dot(const uint16_t *x, const float *w, int n)
{
    float p[32];
    for (int l = 0; l < 32; l++) {
        p[l] = 0.0f;
        for (int i = l; i < n; i += 32)
            p[l] = fmaf(orc_bf16_to_f32(x[i]), w[i], p[l]);
    }
    for (int s = 16; s >= 1; s >>= 1)
        for (int l = 0; l < s; l++)
            p[l] = p[l] + p[l + s];
    return p[0];
}

/* logits[t][e] = canonical fp32 dot(x[t], W[e]) (+ b[e] when b != NULL). */
void orc_router_logits(const uint16_t *x, int T, int H, const float *W, const float *b, int E,
                       float *logits)
{
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            float s = canon_dot(x + (size_t)t * H, W + (size_t)e * H, H);
            logits[(size_t)t * E + e] = b ? s + b[e] : s;
        }
}

/* Softmax over all E experts (fp64, from the fp32 logits), then the k largest
 * probabilities (a tie goes to the lower expert id), renormalised to sum 1.
 * idx[j] lists the picks in descending probability; w[j] their weights. */
void orc_route_token(const float *logit, int E, int k, int32_t *idx, double *w)
{
    double m = -INFINITY, z = 0.0;
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    char *taken = (char *)calloc((size_t)E, 1);
    for (int e = 0; e < E; e++)
        if ((double)logit[e] > m)
            m = logit[e];
    for (int e = 0; e < E; e++) {
        p[e] = exp((double)logit[e] - m);
        z += p[e];
    }
    for (int e = 0; e < E; e++)
        p[e] /= z;
    double kept = 0.0;
    for (int j = 0; j < k; j++) {
        int best = -1;
        for (int e = 0; e < E; e++)
            if (!taken[e] && (best < 0 || p[e] > p[best]))
                best = e;   /* strict '>' keeps the lower id on a tie */
        taken[best] = 1;
        idx[j] = best;
        kept += p[best];
    }
    for (int j = 0; j < k; j++)
        w[j] = p[idx[j]] / kept;
    free(p);
    free(taken);
}

void orc_route(const float *logits, int T, int E, int k, int32_t *idx, double *w)
{
    for (int t = 0; t < T; t++)
        orc_route_token(logits + (size_t)t * E, E, k, idx + (size_t)t * k, w + (size_t)t * k);
}

/* ------------------------------------------------------------------------ */
/* Dispatch                                                                  */
/* ------------------------------------------------------------------------ */

/* cnt[e] = number of (t, j) with idx[t][j] == e; off = exclusive prefix sum of
 * cnt (E+1 entries, off[E] = T*k); list[off[e] + r] = r-th token (ascending)
 * that picked e; slot[t][j] = position of (t, j) in list. */
void orc_dispatch(const int32_t *idx, int T, int k, int E, int32_t *cnt, int32_t *off,
                  int32_t *list, int32_t *slot)
{
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; e++)
        cnt[e] = 0;
    for (size_t i = 0; i < (size_t)T * k; i++)
        cnt[idx[i]]++;
    off[0] = 0;
    for (int e = 0; e < E; e++)
        off[e + 1] = off[e] + cnt[e];
    for (int e = 0; e < E; e++)
        fill[e] = off[e];
    for (int t = 0; t < T; t++)
        for (int j = 0; j < k; j++) {
            int e = idx[(size_t)t * k + j];
            int pos = fill[e]++;
            list[pos] = t;
            slot[(size_t)t * k + j] = pos;
        }
    free(fill);
}

/* ------------------------------------------------------------------------ */
/* Experts                                                                   */
/* ------------------------------------------------------------------------ */

/* y[r] = sum_c W[r][c] * v[c], fp64, ascending c. */
static void qmatvec(const uint8_t *codes, const uint16_t *scales, int bits, int rows, int cols,
                    const double *v, double *y)
{
    for (int r = 0; r < rows; r++) {
        double acc = 0.0;
        for (int c = 0; c < cols; c++)
            acc += orc_weight(codes, scales, bits, cols, r, c) * v[c];
        y[r] = acc;
    }
}

/* SwiGLU expert: g = Wg x, u = Wu x, a = silu(g) * u, y = Wd a (fp64). */
void orc_expert_ffn(const uint8_t *codes_e, const uint16_t *scales_e, int bits, int H, int I,
                    const double *x, double *y)
{
    const uint8_t *c;
    const uint16_t *s;
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    mat_ptrs(codes_e, scales_e, bits, H, I, 0, &c, &s);
    qmatvec(c, s, bits, I, H, x, g);
    mat_ptrs(codes_e, scales_e, bits, H, I, 1, &c, &s);
    qmatvec(c, s, bits, I, H, x, u);
    for (int r = 0; r < I; r++)
        g[r] = g[r] / (1.0 + exp(-g[r])) * u[r];
    mat_ptrs(codes_e, scales_e, bits, H, I, 2, &c, &s);
    qmatvec(c, s, bits, H, I, g, y);
    free(g);
    free(u);
}

/* ------------------------------------------------------------------------ */
/* Layer                                                                     */
/* ------------------------------------------------------------------------ */

typedef struct {
    int H, E, k, I, bits;
    const uint8_t *codes;          /* [E][3][...] packed */
    const uint16_t *scales;
    const float *router_w;         /* [E][H] */
    const float *router_b;         /* [E] or NULL */
    const uint8_t *shared_codes;   /* [3][...] packed */
    const uint16_t *shared_scales;
} orc_layer;

/* Forward of one token: y_f64[H] (before the final bf16 rounding), y_bf16[H],
 * idx[k], w[k].  Combine: shared expert first, then the routed experts in
 * ascending expert id, each added as w_j * expert_j(x). */
static void layer_token(const orc_layer *L, const uint16_t *x_t, double *y, uint16_t *yb,
                        int32_t *idx, double *w)
{
    int H = L->H, E = L->E, k = L->k, I = L->I;
    size_t ex_codes = (size_t)3 * H * I * L->bits / 8, ex_scales = (size_t)3 * H * I / 32;
    float *logit = (float *)malloc(sizeof(float) * (size_t)E);
    double *xf = (double *)malloc(sizeof(double) * (size_t)H);
    double *ye = (double *)malloc(sizeof(double) * (size_t)H);
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);

    orc_router_logits(x_t, 1, H, L->router_w, L->router_b, E, logit);
    orc_route_token(logit, E, k, idx, w);
    for (int i = 0; i < H; i++)
        xf[i] = (double)orc_bf16_to_f32(x_t[i]);

    orc_expert_ffn(L->shared_codes, L->shared_scales, L->bits, H, I, xf, y);

    /* routed experts in ascending id */
    for (int j = 0; j < k; j++)
        order[j] = j;
    for (int a = 0; a < k; a++)
        for (int b = a + 1; b < k; b++)
            if (idx[order[b]] < idx[order[a]]) {
                int32_t tmp = order[a];
                order[a] = order[b];
                order[b] = tmp;
            }
    for (int jj = 0; jj < k; jj++) {
        int j = order[jj], e = idx[j];
        orc_expert_ffn(L->codes + (size_t)e * ex_codes, L->scales + (size_t)e * ex_scales,
                       L->bits, H, I, xf, ye);
        for (int i = 0; i < H; i++)
            y[i] += w[j] * ye[i];
    }
    for (int i = 0; i < H; i++)
        yb[i] = orc_f64_to_bf16(y[i]);
    free(logit);
    free(xf);
    free(ye);
    free(order);
}

/* MoE layer forward for the tokens listed in sel[0..n_sel) (all T tokens when
 * sel == NULL, n_sel = T).  Tokens do not interact in this layer, so any
 * subset is computed exactly as in the full batch.  Outputs are indexed by
 * position in sel: y_bf16[n_sel][H]; y_f64 [n_sel][H], idx [n_sel][k] and
 * w [n_sel][k] may be NULL. */
int orc_moe_forward(int H, int E, int k, int I, int bits, const uint8_t *codes,
                    const uint16_t *scales, const float *router_w, const float *router_b,
                    const uint8_t *shared_codes, const uint16_t *shared_scales,
                    const uint16_t *x, int T, const int32_t *sel, int n_sel, uint16_t *y_bf16,
                    double *y_f64, int32_t *idx, double *w)
{
    if (bits < 1 || bits > 3 || H % 32 || I % 32 || k < 1 || k > E)
        return -1;
    orc_layer L = {H, E, k, I, bits, codes, scales, router_w, router_b, shared_codes,
                   shared_scales};
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    int32_t *ti = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    double *tw = (double *)malloc(sizeof(double) * (size_t)k);
    if (!sel)
        n_sel = T;
    for (int n = 0; n < n_sel; n++) {
        int t = sel ? sel[n] : n;
        if (t < 0 || t >= T)
            return -2;
        layer_token(&L, x + (size_t)t * H, y, y_bf16 + (size_t)n * H, ti, tw);
        if (y_f64)
            memcpy(y_f64 + (size_t)n * H, y, sizeof(double) * (size_t)H);
        if (idx)
            memcpy(idx + (size_t)n * k, ti, sizeof(int32_t) * (size_t)k);
        if (w)
            memcpy(w + (size_t)n * k, tw, sizeof(double) * (size_t)k);
    }
    free(y);
    free(ti);
    free(tw);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 48-layer stack pieces: RMSNorm (weight 1, eps 1e-6) and the residual      */
/* ------------------------------------------------------------------------ */

static uint16_t f32_to_bf16_rne(float f) { return orc_f64_to_bf16((double)f); }

/* xn = bf16(h * r), r = 1 / sqrtf(ss / H + 1e-6f), ss = canonical fp32 sum of
 * squares (same order as the router's dot product). */
void orc_rmsnorm(const uint16_t *h, int T, int H, uint16_t *xn)
{
    for (int t = 0; t < T; t++) {
        const uint16_t *row = h + (size_t)t * H;
        float p[32];
        for (int l = 0; l < 32; l++) {
            p[l] = 0.0f;
            for (int i = l; i < H; i += 32) {
                float v = orc_bf16_to_f32(row[i]);
                p[l] = fmaf(v, v, p[l]);
            }
        }
        for (int s = 16; s >= 1; s >>= 1)
            for (int l = 0; l < s; l++)
                p[l] = p[l] + p[l + s];
        float r = 1.0f / sqrtf(p[0] / (float)H + 1e-6f);
        for (int i = 0; i < H; i++)
            xn[(size_t)t * H + i] = f32_to_bf16_rne(orc_bf16_to_f32(row[i]) * r);
    }
}

/* h = bf16(f32(h) + f32(y)), elementwise. */
void orc_residual_add(uint16_t *h, const uint16_t *y, size_t n)
{
    for (size_t i = 0; i < n; i++)
        h[i] = f32_to_bf16_rne(orc_bf16_to_f32(h[i]) + orc_bf16_to_f32(y[i]));
}
