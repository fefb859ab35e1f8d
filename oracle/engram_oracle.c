/*
 * engram_oracle.c -- plain, slow, single-threaded CPU definition of the
 * Engram conditional-memory forward (lookup and gate).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file.  It shares no code, header, table or
 * constant generator with the CUDA path, and it includes none of its files.
 *
 * Every step follows "Conditional Memory via Scalable Lookup: A New Axis of
 * Sparsity for Large Language Models" (DeepSeek-AI & Peking University),
 * section 2, in the order the paper gives it:
 *
 *   compress   x'_t = P(x_t)                          section 2.2, "Tokenizer compression"
 *   n-grams    g_{t,n} = (x'_{t-n+1}, ..., x'_t)      section 2.2
 *   hash       z_{t,n,k} = phi_{n,k}(g_{t,n})         section 2.2, Eq. (1)
 *   gather     e_t = concat_n concat_k E_{n,k}[z]     section 2.2, Eq. (1)-(2)
 *   project    k_t = W_K e_t,  v_t = W_V e_t          section 2.3, Eq. (3)
 *   gate       alpha_t = sigmoid(RMSNorm(h_t) . RMSNorm(k_t) / sqrt(d))
 *                                                     section 2.3, Eq. (4);
 *                                                     per branch, section 2.4, Eq. (6)
 *   output     out = h + alpha * v                    section 2.3 (gated value,
 *                                                     residual H <- H + Y) and
 *                                                     section 2.4 (u = alpha (W_V e))
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - phi is called a "lightweight multiplicative-XOR hash" and nothing more.
 *    The form used: x = 0; for j < n: x ^= c[t-j] * m[s][j] (wrapping 64-bit),
 *    z = x mod p[s].  j = 0 is the current token.
 *  - multipliers m[s][j] = splitmix64_next() | 1, drawn from one SplitMix64
 *    stream seeded with the hash seed, slot s ascending, then j ascending,
 *    max_order draws per slot.  SplitMix64 is the published generator of
 *    Steele, Lea and Flood, "Fast splittable pseudorandom number generators"
 *    (OOPSLA 2014), in the 64-bit mixing form of Vigna's reference code.
 *  - table sizes: "prime size" only.  The primes are the ascending primes
 *    >= a target, one per slot, slot order = order ascending, head ascending.
 *  - positions before the start of a sequence read the pad id; n-grams never
 *    cross sequences.
 *  - RMSNorm(x) = x / sqrt(mean(x^2) + eps) * w, with a learnable weight w
 *    per branch for the query and for the key; the key is normalised after
 *    the projection (Eq. 4), the scale is 1/sqrt(d) with d the hidden size.
 *  - the FP8 form of the projection (section 2.4) quantises e and W to E4M3
 *    with a power-of-two scale per row; its reading is stated beside
 *    eo_e4m3_encode below.
 *  - ShortConv (Eq. 5) is zero-initialised in the paper (Table 5), so at
 *    initialisation its output equals the gated value and out = h + alpha v.
 *    With trained (non-zero) weights it is the last step below.
 *
 *   short conv Y = SiLU(Conv1D(RMSNorm(V~))) + V~,  H <- H + Y
 *                                                     section 2.3, Eq. (5)
 *
 *  - Conv1D is depthwise and causal over the positions of one sequence, with
 *    kernel size W and dilation delta (the paper sets W = 4 and delta to the
 *    largest n-gram order): tap i of channel c multiplies channel c of the
 *    normalised gated value at position t - i*delta; positions before the
 *    sequence start contribute zero.  No bias.  RMSNorm has its own weight
 *    per channel and the same epsilon as the gate.  In the multi-branch form
 *    one set of conv and norm weights is applied to each branch's sequence
 *    u^(m) = alpha^(m) v separately.
 *
 * Floating point: every sum is accumulated in double over the exact values of
 * the fp32 or bf16 inputs.  bf16 outputs are rounded to nearest-even
 * (through float: double -> float -> bf16).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define EO_F32 0
#define EO_BF16 1
#define EO_F64 2 /* double operands: the dequantised FP8 values below */

/* ---------------------------------------------------------------- SplitMix64 */

uint64_t eo_splitmix64_next(uint64_t *state)
{
    uint64_t z;
    *state += 0x9E3779B97F4A7C15ULL;
    z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* mult[s * max_order + j], s < num_tables, j < max_order; every value odd. */
void eo_hash_multipliers(uint64_t seed, int32_t num_tables, int32_t max_order, uint64_t *mult)
{
    uint64_t st = seed;
    int32_t s, j;
    for (s = 0; s < num_tables; ++s)
        for (j = 0; j < max_order; ++j)
            mult[(int64_t)s * max_order + j] = eo_splitmix64_next(&st) | 1ULL;
}

/* ------------------------------------------------------------------- primes */

int eo_is_prime(int64_t n)
{
    int64_t f;
    if (n < 2) return 0;
    if (n < 4) return 1;
    if (n % 2 == 0) return 0;
    for (f = 3; f * f <= n; f += 2)
        if (n % f == 0) return 0;
    return 1;
}

/* The num_tables ascending primes >= target.  Returns 0, or -1 if target < 2. */
int eo_table_primes(int64_t target, int32_t num_tables, int64_t *primes)
{
    int64_t n = target;
    int32_t s;
    if (target < 2) return -1;
    for (s = 0; s < num_tables; ++s) {
        while (!eo_is_prime(n)) ++n;
        primes[s] = n;
        ++n;
    }
    return 0;
}

/* ------------------------------------------------------------ compression */

/* c[i] = map[x[i]].  Returns the number of tokens outside [0, V) (their c is -1). */
int64_t eo_compress(const int32_t *x, int64_t n, const int32_t *map, int32_t V, int32_t *c)
{
    int64_t i, bad = 0;
    for (i = 0; i < n; ++i) {
        if (x[i] < 0 || x[i] >= V) { c[i] = -1; ++bad; continue; }
        c[i] = map[x[i]];
    }
    return bad;
}

/* ------------------------------------------------------------------ hashing */

/*
 * z[(b * (T - t_begin) + (t - t_begin)) * S + s] for t in [t_begin, T),
 * slot s = order_index * heads + head.  c is the compressed sequence [B, T].
 */
void eo_hash(const int32_t *c, int32_t B, int32_t T, int32_t t_begin, int32_t pad,
             int32_t num_orders, const int32_t *orders, int32_t heads,
             const uint64_t *mult, int32_t max_order, const int64_t *primes, int64_t *z)
{
    int32_t S = num_orders * heads;
    int32_t b, t, oi, k, j;
    for (b = 0; b < B; ++b) {
        for (t = t_begin; t < T; ++t) {
            int64_t row = (int64_t)b * (T - t_begin) + (t - t_begin);
            for (oi = 0; oi < num_orders; ++oi) {
                int32_t n = orders[oi];
                for (k = 0; k < heads; ++k) {
                    int32_t s = oi * heads + k;
                    uint64_t x = 0;
                    for (j = 0; j < n; ++j) {
                        int32_t pos = t - j;
                        int32_t tok = pos >= 0 ? c[(int64_t)b * T + pos] : pad;
                        x ^= (uint64_t)(uint32_t)tok * mult[(int64_t)s * max_order + j];
                    }
                    z[row * S + s] = (int64_t)(x % (uint64_t)primes[s]);
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ gather */

/* e[r][s * d_head + i] = tables[s][z[r][s]][i], copied byte for byte. */
void eo_gather(const void *const *tables, int32_t elem_bytes, int32_t d_head,
               const int64_t *z, int64_t rows, int32_t S, void *e)
{
    int64_t r;
    int32_t s;
    size_t row_bytes = (size_t)d_head * (size_t)elem_bytes;
    for (r = 0; r < rows; ++r)
        for (s = 0; s < S; ++s) {
            const char *src = (const char *)tables[s] + (size_t)z[r * S + s] * row_bytes;
            char *dst = (char *)e + ((size_t)r * S + s) * row_bytes;
            memcpy(dst, src, row_bytes);
        }
}

/* --------------------------------------------------------- element access */

static double eo_load(const void *p, int32_t dtype, int64_t i)
{
    if (dtype == EO_F64) return ((const double *)p)[i];
    if (dtype == EO_F32) return (double)((const float *)p)[i];
    {
        uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
}

static size_t eo_elem_bytes(int32_t dtype)
{
    return dtype == EO_F64 ? 8 : dtype == EO_F32 ? 4 : 2;
}

static uint16_t eo_bf16_rne(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------- projection */

/* y[r][o] = sum_j w[o][j] * e[r][j], accumulated in double (Eq. 3). */
void eo_project(const void *e, int32_t dtype, int64_t rows, int32_t d_mem,
                const void *w, int32_t n_out, double *y)
{
    int64_t r;
    int32_t o, j;
    for (r = 0; r < rows; ++r)
        for (o = 0; o < n_out; ++o) {
            double acc = 0.0;
            for (j = 0; j < d_mem; ++j)
                acc += eo_load(w, dtype, (int64_t)o * d_mem + j) * eo_load(e, dtype, r * d_mem + j);
            y[r * n_out + o] = acc;
        }
}

/* ------------------------------------------------------------------- gate */

/*
 * alpha = sigmoid( RMSNorm_q(h) . RMSNorm_k(k) / sqrt(d) )        (Eq. 4)
 * RMSNorm_w(x)_i = x_i / sqrt(mean(x^2) + eps) * w_i.
 */
double eo_gate(const double *h, const double *k, const float *wq, const float *wk,
               int32_t d, double eps)
{
    double sh = 0.0, sk = 0.0, dot = 0.0, rh, rk, s;
    int32_t i;
    for (i = 0; i < d; ++i) { sh += h[i] * h[i]; sk += k[i] * k[i]; }
    rh = 1.0 / sqrt(sh / d + eps);
    rk = 1.0 / sqrt(sk / d + eps);
    for (i = 0; i < d; ++i) {
        double q = h[i] * rh * (double)wq[i];
        double kn = k[i] * rk * (double)wk[i];
        dot += q * kn;
    }
    s = dot / sqrt((double)d);
    return 1.0 / (1.0 + exp(-s));
}

/* ---------------------------------------------------------------- forward */

/*
 * Projection, gate and output for `rows` rows whose memory vectors e are given
 * (Eq. 3, Eq. 4 / Eq. 6, gated residual).
 *   e     [rows, d_mem]          wdtype
 *   w_k   [M, d, d_mem]          wdtype  (one key projection per branch)
 *   w_v   [d, d_mem]             wdtype  (shared value projection)
 *   wq,wk [M, d]                 float   (RMSNorm weights of query and key)
 *   h     [rows, M, d]           hdtype  (fp32 or bf16)
 *   alpha [rows, M]              double  (out)
 *   delta [rows, M, d]           double  (out; alpha * v; may be NULL)
 *   out   [rows, M, d]           hdtype  (out; h + alpha * v rounded to hdtype)
 * Scratch: kbuf [M * d], vbuf [d], hbuf [d] doubles supplied by the caller.
 */
void eo_project_gate_mixed(const void *e, int32_t wdtype, int64_t rows, int32_t d_mem,
                           const void *w_k, const void *w_v, const float *wq, const float *wk,
                           int32_t M, int32_t d, double eps, const void *h, int32_t hdtype,
                           double *alpha, double *delta, void *out,
                           double *kbuf, double *vbuf, double *hbuf)
{
    int64_t r;
    int32_t m, i;
    for (r = 0; r < rows; ++r) {
        const char *er = (const char *)e + (size_t)r * d_mem * eo_elem_bytes(wdtype);
        eo_project(er, wdtype, 1, d_mem, w_k, M * d, kbuf);
        eo_project(er, wdtype, 1, d_mem, w_v, d, vbuf);
        for (m = 0; m < M; ++m) {
            int64_t base = (r * M + m) * (int64_t)d;
            double a;
            for (i = 0; i < d; ++i) hbuf[i] = eo_load(h, hdtype, base + i);
            a = eo_gate(hbuf, kbuf + (int64_t)m * d, wq + (int64_t)m * d, wk + (int64_t)m * d, d, eps);
            alpha[r * M + m] = a;
            for (i = 0; i < d; ++i) {
                double dl = a * vbuf[i];
                double o = hbuf[i] + dl;
                if (delta) delta[base + i] = dl;
                if (hdtype == EO_F64) ((double *)out)[base + i] = o;
                else if (hdtype == EO_F32) ((float *)out)[base + i] = (float)o;
                else ((uint16_t *)out)[base + i] = eo_bf16_rne(o);
            }
        }
    }
}

/* The same with one dtype for every operand. */
void eo_project_gate(const void *e, int32_t dtype, int64_t rows, int32_t d_mem,
                     const void *w_k, const void *w_v, const float *wq, const float *wk,
                     int32_t M, int32_t d, double eps, const void *h,
                     double *alpha, double *delta, void *out,
                     double *kbuf, double *vbuf, double *hbuf)
{
    eo_project_gate_mixed(e, dtype, rows, d_mem, w_k, w_v, wq, wk, M, d, eps, h, dtype,
                          alpha, delta, out, kbuf, vbuf, hbuf);
}

/* ------------------------------------------------------- FP8 projection */

/*
 * Section 2.4 fuses W_V and the M key projections W_K into one dense FP8
 * matmul.  The pages name neither the FP8 format nor how values are scaled
 * into it; the reading taken here:
 *  - the operands e and W are E4M3 (1 sign bit, 4 exponent bits with bias 7,
 *    3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9; no
 *    infinities; S.1111.111 is NaN; the largest finite magnitude is 448);
 *  - one scale per row of e (per position) and one per row of W (per output
 *    channel), each a power of two 2^E, E the smallest integer for which the
 *    row's largest magnitude is at most 448 * 2^E (E = 0 for an all-zero row);
 *  - code = E4M3(x * 2^-E), rounded to nearest with ties to even, saturating
 *    at +-448, the sign kept for values that round to zero; the dequantised
 *    value is E4M3value(code) * 2^E.
 * Both scales factor out of every dot product of Eq. (3), so k and v are the
 * projections of the dequantised operands, and the gate and output follow
 * unchanged (eo_project_gate_mixed with EO_F64 operands).
 */

/* The value of an E4M3 code (NaN for S.1111.111). */
double eo_e4m3_decode(uint8_t code)
{
    const int sign = code >> 7, ex = (code >> 3) & 15, man = code & 7;
    double v;
    if (ex == 15 && man == 7) return NAN;
    v = ex == 0 ? ldexp((double)man, -9) : ldexp(8.0 + man, ex - 10); /* (1 + m/8) 2^(ex-7) */
    return sign ? -v : v;
}

/* E4M3 code of y: round to nearest, ties to even, saturate at +-448. */
uint8_t eo_e4m3_encode(double y)
{
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    const double a = fabs(y);
    double step, v;
    int ex;
    if (isnan(y)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    /* spacing of the representable values around a: 2^-9 below the smallest
       normal 2^-6, else 2^(floor(log2 a) - 3) */
    if (a < ldexp(1.0, -6)) {
        step = ldexp(1.0, -9);
    } else {
        frexp(a, &ex); /* a = f 2^ex, 0.5 <= f < 1: floor(log2 a) = ex - 1 */
        step = ldexp(1.0, ex - 4);
    }
    v = nearbyint(a / step) * step; /* a / step is exact; ties to even */
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -6)) return sign | (uint8_t)(v / ldexp(1.0, -9));
    frexp(v, &ex);
    return sign | (uint8_t)((ex - 1 + 7) << 3) | (uint8_t)(ldexp(v, 4 - ex) - 8.0);
}

/* E of the power-of-two scale 2^E for a row whose largest magnitude is amax. */
int32_t eo_e4m3_scale_exp(double amax)
{
    int ex;
    double f;
    if (!(amax > 0.0)) return 0;
    f = frexp(amax, &ex); /* amax = f 2^ex; 448 = 0.875 2^9 */
    return f <= 0.875 ? ex - 9 : ex - 8;
}

/* codes [rows, cols] and scales [rows] (2^E as float) of x [rows, cols]. */
void eo_quantize_e4m3_rows(const void *x, int32_t dtype, int64_t rows, int32_t cols,
                           uint8_t *code, float *scale)
{
    int64_t r;
    int32_t j;
    for (r = 0; r < rows; ++r) {
        double amax = 0.0;
        int32_t E;
        for (j = 0; j < cols; ++j) {
            const double a = fabs(eo_load(x, dtype, r * cols + j));
            if (a > amax) amax = a;
        }
        E = eo_e4m3_scale_exp(amax);
        for (j = 0; j < cols; ++j)
            code[r * cols + j] = eo_e4m3_encode(ldexp(eo_load(x, dtype, r * cols + j), -E));
        scale[r] = (float)ldexp(1.0, E);
    }
}

/* y [rows, cols] = E4M3value(code) * scale[row]. */
void eo_dequantize_e4m3_rows(const uint8_t *code, const float *scale, int64_t rows, int32_t cols,
                             double *y)
{
    int64_t r;
    int32_t j;
    for (r = 0; r < rows; ++r)
        for (j = 0; j < cols; ++j)
            y[r * cols + j] = eo_e4m3_decode(code[r * cols + j]) * (double)scale[r];
}

/* -------------------------------------------------------------- short conv */

static double eo_silu(double x) { return x / (1.0 + exp(-x)); }

/*
 * Y at one position t of one sequence and branch (Eq. 5):
 *   Y_t = SiLU( sum_i cw[c][i] * RMSNorm(V~_{t - i*dil})[c] ) + V~_t[c]
 *   taps  [W][d] double: V~ at positions t, t - dil, ..., t - (W-1) dil
 *   have  [W]    int:    0 where that position lies before the sequence start
 *   cw    [d][W] float, nw [d] float (RMSNorm weight), y [d] double (out).
 * Scratch: norm [d] doubles supplied by the caller.
 */
void eo_short_conv_at(const double *taps, const int32_t *have, int32_t W, int32_t d,
                      const float *cw, const float *nw, double eps, double *y, double *norm)
{
    int32_t i, c;
    for (c = 0; c < d; ++c) y[c] = 0.0;
    for (i = 0; i < W; ++i) {
        const double *x = taps + (int64_t)i * d;
        double ss = 0.0, r;
        if (!have[i]) continue;
        for (c = 0; c < d; ++c) ss += x[c] * x[c];
        r = 1.0 / sqrt(ss / d + eps);
        for (c = 0; c < d; ++c) norm[c] = x[c] * r * (double)nw[c];
        for (c = 0; c < d; ++c) y[c] += (double)cw[(int64_t)c * W + i] * norm[c];
    }
    for (c = 0; c < d; ++c) y[c] = eo_silu(y[c]) + taps[c];
}

/*
 * Y for every position of one sequence and branch: vt [n_pos, d] double
 * (V~ at positions 0 .. n_pos-1), y [n_pos, d] double (out).
 * Scratch: taps [W * d], norm [d] doubles, have [W] ints.
 */
void eo_short_conv(const double *vt, int32_t n_pos, int32_t d, const float *cw, int32_t W,
                   int32_t dil, const float *nw, double eps, double *y,
                   double *taps, int32_t *have, double *norm)
{
    int32_t t, i, c;
    for (t = 0; t < n_pos; ++t) {
        for (i = 0; i < W; ++i) {
            const int32_t p = t - i * dil;
            have[i] = p >= 0;
            for (c = 0; c < d; ++c) taps[(int64_t)i * d + c] = p >= 0 ? vt[(int64_t)p * d + c] : 0.0;
        }
        eo_short_conv_at(taps, have, W, d, cw, nw, eps, y + (int64_t)t * d, norm);
    }
}

/* out = h + Y rounded to the h dtype, for n values. */
void eo_add_round(const void *h, int32_t dtype, int64_t n, const double *y, void *out)
{
    int64_t i;
    for (i = 0; i < n; ++i) {
        double o = eo_load(h, dtype, i) + y[i];
        if (dtype == EO_F32) ((float *)out)[i] = (float)o;
        else ((uint16_t *)out)[i] = eo_bf16_rne(o);
    }
}

/* ---------------------------------------------------------------- backward */

/*
 * Gradients of the forward above (Eq. 3, Eq. 4 / Eq. 6 and the gated
 * residual) for a scalar loss whose gradient with respect to out is dout.
 * The pages give only the forward; the backward is its exact derivative,
 * written out per row r and branch m (all in double):
 *
 *   k = W_K^(m) e, v = W_V e, rh = (mean(h^2) + eps)^-1/2, rk likewise for k,
 *   qn = h rh w_q, kn = k rk w_k, s = qn . kn / sqrt(d), alpha = sigmoid(s),
 *   out = h + alpha v.
 *
 *   dalpha = dout . v                  dv   += alpha dout
 *   ds     = dalpha alpha (1 - alpha)
 *   dqn    = ds kn / sqrt(d)           dkn   = ds qn / sqrt(d)
 *   dw_q  += dqn h rh                  dw_k += dkn k rk
 *   RMSNorm x^ = x r: with u = dqn w_q (resp. dkn w_k),
 *     dx = r u - r^3 / d x (u . x)
 *   dh     = dout + rh u_q - rh^3 / d h (u_q . h)
 *   dk     = rk u_k - rk^3 / d k (u_k . k)
 *   dW_K^(m) += dk e^T,  dW_V += dv e^T,
 *   de     = sum_m W_K^(m)T dk + W_V^T dv,
 *   dE_s[z_s] += the slot-s slice of de (slot_rows_grad below).
 *
 * round_dkv != 0: dk and dv are rounded to bf16 (nearest-even, through
 * float) before they multiply e and W, as a bf16 training step feeds them to
 * its tensor-core GEMMs; the gradients are then exact functions of those
 * rounded values.  dh is returned in double.
 *   e     [rows, d_mem] wdtype;  w_k [M, d, d_mem], w_v [d, d_mem] wdtype
 *   h     [rows, M, d] hdtype;   dout [rows, M, d] double
 *   dh    [rows, M, d] double (out)
 *   dkv   [rows, (M + 1) d] double (out): dk of each branch, then dv, as used
 *         by the weight GEMMs (rounded when round_dkv)
 *   dw    [(M + 1) d, d_mem] double, accumulated: dW_K rows, then dW_V
 *   dwq, dwk [M, d] double, accumulated
 *   de    [rows, d_mem] double (out)
 * Scratch: kbuf [M d], vbuf [d], hbuf [d] doubles.
 */
void eo_backward(const void *e, int32_t wdtype, int64_t rows, int32_t d_mem,
                 const void *w_k, const void *w_v, const float *wq, const float *wk,
                 int32_t M, int32_t d, double eps, const void *h, int32_t hdtype,
                 const double *dout, int32_t round_dkv, double *dh, double *dkv, double *dw,
                 double *dwq, double *dwk, double *de,
                 double *kbuf, double *vbuf, double *hbuf)
{
    const int64_t nkv = (int64_t)(M + 1) * d;
    const double isd = 1.0 / sqrt((double)d);
    int64_t r, o;
    int32_t m, i, j;
    for (r = 0; r < rows; ++r) {
        const char *er = (const char *)e + (size_t)r * d_mem * eo_elem_bytes(wdtype);
        double *gkv = dkv + r * nkv;
        double *dv = gkv + (int64_t)M * d;
        eo_project(er, wdtype, 1, d_mem, w_k, M * d, kbuf);
        eo_project(er, wdtype, 1, d_mem, w_v, d, vbuf);
        for (i = 0; i < d; ++i) dv[i] = 0.0;
        for (m = 0; m < M; ++m) {
            const int64_t base = (r * M + m) * (int64_t)d;
            const double *k = kbuf + (int64_t)m * d;
            const float *wqm = wq + (int64_t)m * d, *wkm = wk + (int64_t)m * d;
            const double *g = dout + base;
            double sh = 0.0, sk = 0.0, s = 0.0, da = 0.0, uh = 0.0, uk = 0.0;
            double rh, rk, a, ds;
            for (i = 0; i < d; ++i) hbuf[i] = eo_load(h, hdtype, base + i);
            for (i = 0; i < d; ++i) { sh += hbuf[i] * hbuf[i]; sk += k[i] * k[i]; }
            rh = 1.0 / sqrt(sh / d + eps);
            rk = 1.0 / sqrt(sk / d + eps);
            for (i = 0; i < d; ++i) s += (hbuf[i] * rh * wqm[i]) * (k[i] * rk * wkm[i]);
            a = 1.0 / (1.0 + exp(-s * isd));
            for (i = 0; i < d; ++i) { da += g[i] * vbuf[i]; dv[i] += a * g[i]; }
            ds = da * a * (1.0 - a);
            /* u_q = dqn w_q, u_k = dkn w_k, with dqn = ds kn / sqrt(d), dkn = ds qn / sqrt(d) */
            for (i = 0; i < d; ++i) {
                const double qn = hbuf[i] * rh * wqm[i], kn = k[i] * rk * wkm[i];
                const double dqn = ds * kn * isd, dkn = ds * qn * isd;
                dwq[(int64_t)m * d + i] += dqn * hbuf[i] * rh;
                dwk[(int64_t)m * d + i] += dkn * k[i] * rk;
                uh += dqn * wqm[i] * hbuf[i];
                uk += dkn * wkm[i] * k[i];
            }
            for (i = 0; i < d; ++i) {
                const double qn = hbuf[i] * rh * wqm[i], kn = k[i] * rk * wkm[i];
                const double dqn = ds * kn * isd, dkn = ds * qn * isd;
                dh[base + i] = g[i] + rh * dqn * wqm[i] - rh * rh * rh / d * hbuf[i] * uh;
                gkv[(int64_t)m * d + i] = rk * dkn * wkm[i] - rk * rk * rk / d * k[i] * uk;
            }
        }
        if (round_dkv)
            for (o = 0; o < nkv; ++o) {
                const uint16_t b = eo_bf16_rne(gkv[o]);
                uint32_t u = (uint32_t)b << 16;
                float f;
                memcpy(&f, &u, 4);
                gkv[o] = (double)f;
            }
        /* weight gradients and de (Eq. 3 transposed) */
        for (o = 0; o < nkv; ++o)
            for (j = 0; j < d_mem; ++j)
                dw[o * d_mem + j] += gkv[o] * eo_load(e, wdtype, r * d_mem + j);
        for (j = 0; j < d_mem; ++j) {
            double acc = 0.0;
            for (o = 0; o < nkv; ++o) {
                const void *w = o < (int64_t)M * d ? w_k : w_v;
                const int64_t wo = o < (int64_t)M * d ? o : o - (int64_t)M * d;
                acc += gkv[o] * eo_load(w, wdtype, wo * d_mem + j);
            }
            de[r * d_mem + j] = acc;
        }
    }
}

/*
 * Table gradients (Eq. 2 transposed): for every row r and slot s,
 * dtab[s][z[r][s]][i] += de[r][s d_h + i].  dtab is an array of S pointers to
 * double [p_s, d_h]; z [rows, S] the indices of the forward.
 */
void eo_table_grad(const double *de, const int64_t *z, int64_t rows, int32_t S, int32_t d_head,
                   double *const *dtab)
{
    int64_t r;
    int32_t s, i;
    for (r = 0; r < rows; ++r)
        for (s = 0; s < S; ++s) {
            double *row = dtab[s] + z[r * S + s] * d_head;
            for (i = 0; i < d_head; ++i) row[i] += de[r * (int64_t)S * d_head + (int64_t)s * d_head + i];
        }
}
