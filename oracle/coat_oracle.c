/*
 * coat_oracle.c -- plain, slow, double-precision CPU oracle for the COAT
 * FP8-optimizer-state AdamW step and its per-group FP8 codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no source, header, table or constant with
 * the CUDA path.
 *
 * Sources (web pages describing COAT: "Compressing Optimizer states and
 * Activation for memory-efficient FP8 Training"):
 *   [P1] "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍"
 *        (blob.wenxiaobai.com), sections "FP8优化器状态" (FP8 optimizer
 *        states) and "解决方案：动态范围扩展" (dynamic range expansion).
 *   [P4] "FP8量化训练实战指南：解决大模型训练效率瓶颈的终极方案", section
 *        "格式选择：E4M3与E5M2的智能搭配" (bit layouts 1+4+3 and 1+5+2).
 * The pages name the expansion function but its formula was lost from the
 * extracted text; the formulas below are the problem statement's:
 *   f(x) = sign(x)|x|^k,  k = ln(448 / 2^-9) / ln(max|x| / min_nonzero|x|),
 *   clamped to [1, 16]; an all-zero group has k = 1 and scale 1;
 *   dequantisation x = sign(q) |q s|^(1/k).
 * Readings taken where the pages are silent (each is listed in the design
 * notes):
 *   - R = 448 / 2^-9 = 229376 sets k for both E4M3 and E5M2.
 *   - The stored per-group scale is the k-th root s_r = s^(1/k) = M FMT_MAX^(-1/k)
 *     (s itself underflows FP32 for second moments), so x = sign(q) s_r |q|^(1/k).
 *   - k is rounded to FP32 first; the scale and the expansion use that FP32 k,
 *     which is the k that dequantisation will see.
 *   - The FP8 encode decision is taken on an FP32 value (the kernel's
 *     precision): the double y is rounded to float, then to the nearest finite
 *     FP8 value, ties to the even code, saturating; a zero magnitude is code 0.
 *   - AdamW follows torch.optim.AdamW: decoupled decay p <- p (1 - lr wd),
 *     eps added after sqrt(v)/sqrt(1 - b2^t), bias corrections in double; the
 *     update uses the unquantised new moments; requantisation only affects
 *     what is stored for the next step.
 * Pinned by tests/test_oracle_*.py (decode tables from the bit definitions and
 * torch's float8 casts, brute-force nearest encode, expansion invariants,
 * hand-derived worked examples, torch.optim.AdamW in float64, closed forms).
 * Parity unpinned: the choice of R for E5M2 and the "optimal k" claim of [P1];
 * the formula is a definition, not a proven optimum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_E4M3 0
#define ORC_E5M2 1
/* E5M2 codes whose expansion targets E5M2's own span (57344 / 2^-16) instead
 * of E4M3's; as a number format it is E5M2. */
#define ORC_E5M2_FULL 2

/* ------------------------------------------------------------------ */
/* FP8 formats, straight from the bit definitions ([P4] 格式选择).     */
/* ------------------------------------------------------------------ */

/* Value of an 8-bit code.  E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa
 * bits; exponent 15 with mantissa 7 is NaN; there is no infinity.
 * E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits; exponent 31 is
 * infinity (mantissa 0) or NaN.  Exponent 0 is subnormal. */
double orc_fp8_decode(int fmt, unsigned code)
{
    int neg = (code >> 7) & 1;
    double mag;
    if (fmt == ORC_E4M3) {
        int e = (code >> 3) & 15, m = code & 7;
        if (e == 15 && m == 7)
            return NAN;
        if (e == 0)
            mag = ldexp((double)m / 8.0, 1 - 7);
        else
            mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    } else {
        int e = (code >> 2) & 31, m = code & 3;
        if (e == 31) {
            if (m != 0)
                return NAN;
            return neg ? -INFINITY : INFINITY;
        }
        if (e == 0)
            mag = ldexp((double)m / 4.0, 1 - 15);
        else
            mag = ldexp(1.0 + (double)m / 4.0, e - 15);
    }
    return neg ? -mag : mag;
}

/* Largest finite code and value of each format. */
static unsigned orc_max_code(int fmt) { return fmt == ORC_E4M3 ? 0x7Eu : 0x7Bu; }
double orc_fmt_max(int fmt) { return orc_fp8_decode(fmt, orc_max_code(fmt)); }

/* Positive finite values by code, filled on first use from orc_fp8_decode. */
static double g_table[3][128];
static int g_table_ready[3];

static const double *orc_table(int fmt)
{
    if (!g_table_ready[fmt]) {
        for (unsigned c = 0; c < 128; c++)
            g_table[fmt][c] = orc_fp8_decode(fmt, c);
        g_table_ready[fmt] = 1;
    }
    return g_table[fmt];
}

/* Nearest finite FP8 magnitude code to a non-negative FP32 value: a plain
 * scan over every finite positive code.  On an exact tie between two codes the
 * even one wins; anything at or above the largest finite value (infinity
 * included) saturates to it. */
static unsigned orc_encode_mag(int fmt, float yf)
{
    const double *t = orc_table(fmt);
    unsigned top = orc_max_code(fmt);
    double a = fabs((double)yf);
    if (a >= t[top])
        return top;
    unsigned best = 0;
    double bestd = a; /* distance to code 0, whose value is 0 */
    for (unsigned c = 1; c <= top; c++) {
        double d = fabs(t[c] - a);
        if (d < bestd || (d == bestd && (c & 1u) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* FP32 -> FP8 code, round to nearest even, saturating to the largest finite
 * value.  NaN gives 0x7F with the input's sign.  A magnitude that rounds to
 * zero gives code 0x00 whatever the sign. */
unsigned orc_fp8_encode(int fmt, float y)
{
    if (isnan(y))
        return (signbit(y) ? 0x80u : 0u) | 0x7Fu;
    unsigned mag = orc_encode_mag(fmt, y);
    if (mag == 0)
        return 0;
    return (signbit(y) ? 0x80u : 0u) | mag;
}

/* Element-wise orc_fp8_encode over an array (for exhaustive tests). */
void orc_fp8_encode_array(int fmt, const float *y, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)orc_fp8_encode(fmt, y[i]);
}

/* bf16 bit pattern -> double (exact). */
static double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* FP32 -> bf16 bit pattern, round to nearest even (NaN stays NaN). */
uint16_t orc_float_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(f))
        return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* Dynamic range expansion and per-group quantisation                 */
/* ([P1] 解决方案：动态范围扩展; problem-statement formulas).           */
/* ------------------------------------------------------------------ */

/* The span the expansion aims for: E4M3's largest over smallest positive
 * value, 448 / 2^-9 ([P1] FP8优化器状态: 0.00195 ... 448, about 200000), for
 * E4M3 and E5M2 alike; for ORC_E5M2_FULL, E5M2's own largest over smallest
 * positive value, 57344 / 2^-16 (the reading under which [P1] 解决方案：动态范围扩展's
 * "E4M3 and E5M2 almost the same after expansion" for v holds). */
double orc_target_range(int fmt)
{
    if (fmt == ORC_E5M2_FULL)
        return orc_fp8_decode(ORC_E5M2, 0x7B) / orc_fp8_decode(ORC_E5M2, 0x01);
    return orc_fp8_decode(ORC_E4M3, 0x7E) / orc_fp8_decode(ORC_E4M3, 0x01);
}

/* Group statistics and parameters.  M = max|x|, mu = min{|x| : x != 0}.
 * k = clamp(ln R / ln(M/mu), 1, 16); M == mu (one distinct magnitude) gives
 * k = 16; without expansion k = 1; an all-zero group gives k = 1, s_r = 1.
 * k is stored as float and the root scale s_r = M * FMT_MAX^(-1/k) uses that
 * float k.  Returns M. */
double orc_group_params(const double *x, int64_t cnt, int expand, int fmt,
                        float *k_out, float *s_out)
{
    double M = 0.0, mu = INFINITY;
    for (int64_t i = 0; i < cnt; i++) {
        double a = fabs(x[i]);
        if (a > M)
            M = a;
        if (a != 0.0 && a < mu)
            mu = a;
    }
    if (M == 0.0) {
        *k_out = 1.0f;
        *s_out = 1.0f;
        return 0.0;
    }
    double k;
    if (!expand)
        k = 1.0;
    else if (M == mu)
        k = 16.0;
    else {
        k = log(orc_target_range(fmt)) / log(M / mu);
        if (k < 1.0)
            k = 1.0;
        if (k > 16.0)
            k = 16.0;
    }
    float kf = (float)k;
    double s_r = M * pow(orc_fmt_max(fmt), -1.0 / (double)kf);
    *k_out = kf;
    *s_out = (float)s_r;
    return M;
}

/* Quantise one group of cnt values: k and s_r as above, then
 * y_i = FMT_MAX (|x_i| / M)^k, rounded to FP32 and encoded; the sign of x_i
 * goes in the code's top bit. */
void orc_quantize_group(const double *x, int64_t cnt, int expand, int fmt,
                        uint8_t *codes, float *k_out, float *s_out)
{
    double M = orc_group_params(x, cnt, expand, fmt, k_out, s_out);
    double k = (double)*k_out;
    double fmax = orc_fmt_max(fmt);
    for (int64_t i = 0; i < cnt; i++) {
        if (M == 0.0) {
            codes[i] = 0;
            continue;
        }
        double y = fmax * pow(fabs(x[i]) / M, k);
        float yf = (float)y;
        if (x[i] < 0)
            yf = -yf;
        codes[i] = (uint8_t)orc_fp8_encode(fmt, yf);
    }
}

/* x = sign(q) * s_r * |dec(q)|^(1/k). */
double orc_dequant_value(int fmt, uint8_t code, float s_r, float k)
{
    double d = orc_fp8_decode(fmt, code);
    if (d == 0.0 || isnan(d))
        return d == 0.0 ? 0.0 : d;
    double mag = (double)s_r * pow(fabs(d), 1.0 / (double)k);
    return d < 0 ? -mag : mag;
}

/* 2-D grouping.  x is rows x cols, row-major with leading dimension ldx
 * (elements); groups are gr x gc blocks (partial blocks at the bottom and
 * right edges hold only the valid elements); q is rows x cols bytes with
 * leading dimension ldq; scale and k are ceil(rows/gr) x ceil(cols/gc),
 * row-major.  Returns 0, or -1 on bad arguments. */
int orc_group_quantize(const double *x, int64_t rows, int64_t cols, int64_t ldx,
                       int gr, int gc, int expand, int fmt, uint8_t *q,
                       int64_t ldq, float *scale, float *kk)
{
    if (rows < 0 || cols < 0 || gr < 1 || gc < 1 || ldx < cols || ldq < cols)
        return -1;
    int64_t nbr = (rows + gr - 1) / gr, nbc = (cols + gc - 1) / gc;
    double *buf = (double *)malloc(sizeof(double) * (size_t)gr * (size_t)gc);
    uint8_t *cb = (uint8_t *)malloc((size_t)gr * (size_t)gc);
    if (!buf || !cb) {
        free(buf);
        free(cb);
        return -1;
    }
    for (int64_t bi = 0; bi < nbr; bi++)
        for (int64_t bj = 0; bj < nbc; bj++) {
            int64_t r0 = bi * gr, c0 = bj * gc;
            int64_t r1 = r0 + gr < rows ? r0 + gr : rows;
            int64_t c1 = c0 + gc < cols ? c0 + gc : cols;
            int64_t cnt = 0;
            for (int64_t r = r0; r < r1; r++)
                for (int64_t c = c0; c < c1; c++)
                    buf[cnt++] = x[r * ldx + c];
            orc_quantize_group(buf, cnt, expand, fmt, cb, &kk[bi * nbc + bj],
                               &scale[bi * nbc + bj]);
            cnt = 0;
            for (int64_t r = r0; r < r1; r++)
                for (int64_t c = c0; c < c1; c++)
                    q[r * ldq + c] = cb[cnt++];
        }
    free(buf);
    free(cb);
    return 0;
}

int orc_group_dequantize(const uint8_t *q, int64_t ldq, const float *scale,
                         const float *kk, int64_t rows, int64_t cols, int gr,
                         int gc, int fmt, double *out, int64_t ldo)
{
    if (rows < 0 || cols < 0 || gr < 1 || gc < 1 || ldq < cols || ldo < cols)
        return -1;
    int64_t nbc = (cols + gc - 1) / gc;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            int64_t g = (r / gr) * nbc + c / gc;
            out[r * ldo + c] = orc_dequant_value(fmt, q[r * ldq + c], scale[g], kk[g]);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* AdamW over FP8 moments ([P1] FP8优化器状态: first and second        */
/* moments kept in FP8, per-group; torch.optim.AdamW semantics).      */
/* ------------------------------------------------------------------ */

/* One step on n elements split into groups of `group` (the last may be
 * partial).  master (float) is updated in place; weight_out (bf16 bits, may
 * be NULL) receives RNE(master); grad holds bf16 bits.  m_q / v_q hold
 * ceil(n/group)*group codes (padding written 0); *_scale / *_k hold one
 * float per group.  If upd_out is not NULL it receives, per element, the
 * adaptive update evaluated on the magnitudes of the two summands of m',
 * lr/bc1 * (|b1 m| + |(1-b1) g|) / (sqrt(v')/sqrt(bc2) + eps): the size of
 * the update before any cancellation between the old moment and the new
 * gradient.  Tests use it to size the master-weight tolerance (it is not part
 * of the method's result).  Returns 0, or -1 on bad arguments. */
int orc_adamw_step_scaled(float *master, uint16_t *weight_out, const uint16_t *grad,
                          uint8_t *m_q, float *m_scale, float *m_k, uint8_t *v_q,
                          float *v_scale, float *v_k, int64_t n, int group, float lr,
                          float beta1, float beta2, float eps, float wd, int64_t step,
                          int fmt_m, int fmt_v, double gscale, double *upd_out);

int orc_adamw_step(float *master, uint16_t *weight_out, const uint16_t *grad,
                   uint8_t *m_q, float *m_scale, float *m_k, uint8_t *v_q,
                   float *v_scale, float *v_k, int64_t n, int group, float lr,
                   float beta1, float beta2, float eps, float wd, int64_t step,
                   int fmt_m, int fmt_v, double *upd_out)
{
    return orc_adamw_step_scaled(master, weight_out, grad, m_q, m_scale, m_k, v_q, v_scale, v_k,
                                 n, group, lr, beta1, beta2, eps, wd, step, fmt_m, fmt_v, 1.0,
                                 upd_out);
}

/* The step on the clipped gradient gscale * g (gradient-norm clipping, see
 * orc_clip_coef; gscale = 1 is the plain step). */
int orc_adamw_step_scaled(float *master, uint16_t *weight_out, const uint16_t *grad,
                          uint8_t *m_q, float *m_scale, float *m_k, uint8_t *v_q,
                          float *v_scale, float *v_k, int64_t n, int group, float lr,
                          float beta1, float beta2, float eps, float wd, int64_t step,
                          int fmt_m, int fmt_v, double gscale, double *upd_out)
{
    if (n < 0 || group < 1 || step < 1)
        return -1;
    double b1 = beta1, b2 = beta2, dlr = lr, deps = eps, dwd = wd;
    double bc1 = 1.0 - pow(b1, (double)step);
    double bc2 = 1.0 - pow(b2, (double)step);
    int64_t ngroups = (n + group - 1) / group;
    double *mb = (double *)malloc(sizeof(double) * (size_t)group);
    double *vb = (double *)malloc(sizeof(double) * (size_t)group);
    if (!mb || !vb) {
        free(mb);
        free(vb);
        return -1;
    }
    for (int64_t g = 0; g < ngroups; g++) {
        int64_t base = g * group;
        int64_t cnt = n - base < group ? n - base : group;
        for (int64_t j = 0; j < cnt; j++) {
            int64_t i = base + j;
            double m = orc_dequant_value(fmt_m, m_q[i], m_scale[g], m_k[g]);
            double v = orc_dequant_value(fmt_v, v_q[i], v_scale[g], v_k[g]);
            double gi = gscale * orc_bf16_to_double(grad[i]);
            double m1 = b1 * m + (1.0 - b1) * gi;
            double v1 = b2 * v + (1.0 - b2) * gi * gi;
            double p = (double)master[i];
            p = p * (1.0 - dlr * dwd);
            double adapt = (dlr / bc1) * m1 / (sqrt(v1) / sqrt(bc2) + deps);
            p = p - adapt;
            master[i] = (float)p;
            if (weight_out)
                weight_out[i] = orc_float_to_bf16(master[i]);
            if (upd_out)
                upd_out[i] = (dlr / bc1) * (fabs(b1 * m) + fabs((1.0 - b1) * gi)) /
                             (sqrt(v1) / sqrt(bc2) + deps);
            mb[j] = m1;
            vb[j] = v1;
        }
        orc_quantize_group(mb, cnt, 1, fmt_m, m_q + base, &m_k[g], &m_scale[g]);
        orc_quantize_group(vb, cnt, 1, fmt_v, v_q + base, &v_k[g], &v_scale[g]);
        for (int64_t j = cnt; j < group; j++) {
            m_q[base + j] = 0;
            v_q[base + j] = 0;
        }
    }
    free(mb);
    free(vb);
    return 0;
}

/* The same step with the moments kept unquantised in double: the plain
 * AdamW recurrence, used to pin the optimizer arithmetic against closed
 * forms and torch.optim.AdamW. */
/* ------------------------------------------------------------------ */
/* Global gradient-norm clipping and the non-finite check before the   */
/* step (not on the pages; the usual training-loop pre-step, as        */
/* torch.nn.utils.clip_grad_norm_ defines it).                          */
/* ------------------------------------------------------------------ */

/* Sum of squares of n bf16 gradient values, in double, in element order;
 * *nonfinite is set to 1 if any value is infinite or NaN (left as is
 * otherwise, so that calls over several tensors accumulate). */
double orc_grad_sumsq(const uint16_t *grad, int64_t n, int *nonfinite)
{
    double s = 0.0;
    for (int64_t i = 0; i < n; i++) {
        double g = orc_bf16_to_double(grad[i]);
        if (!isfinite(g))
            *nonfinite = 1;
        s += g * g;
    }
    return s;
}

/* Clip coefficient for a total sum of squares: min(1, max_norm / (norm +
 * 1e-6)) with norm = sqrt(sumsq), rounded to FP32 (max_norm = +inf: 1). */
float orc_clip_coef(double sumsq, float max_norm)
{
    double c = (double)max_norm / (sqrt(sumsq) + 1e-6);
    return (float)(c < 1.0 ? c : 1.0);
}

int orc_adamw_step_unquantized(double *p, double *m, double *v, const double *g,
                               int64_t n, double lr, double beta1, double beta2,
                               double eps, double wd, int64_t step)
{
    if (n < 0 || step < 1)
        return -1;
    double bc1 = 1.0 - pow(beta1, (double)step);
    double bc2 = 1.0 - pow(beta2, (double)step);
    for (int64_t i = 0; i < n; i++) {
        m[i] = beta1 * m[i] + (1.0 - beta1) * g[i];
        v[i] = beta2 * v[i] + (1.0 - beta2) * g[i] * g[i];
        p[i] = p[i] * (1.0 - lr * wd);
        p[i] = p[i] - (lr / bc1) * m[i] / (sqrt(v[i]) / sqrt(bc2) + eps);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* FP8 precision flow through a non-linear layer ([P1] sections        */
/* "FP8激活" and "解决方案：混合粒度FP8精度流"): the layer's inputs and  */
/* output are FP8 tensors in 1x128 per-token groups, and the FP8 inputs */
/* are what the backward pass reads (nothing is requantised for it).   */
/* The layer is Llama's gated activation h = silu(gate) * up (SwiGLU),  */
/* silu(g) = g sigmoid(g) = g / (1 + e^-g).                            */
/* Readings: the activation value h is rounded to FP32 before it is     */
/* quantised (the kernel's precision decides the codes); a sigmoid      */
/* below FP32's normal range (2^-126, i.e. g < -87.3) counts as 0, as   */
/* in FP32 arithmetic that flushes subnormals; the incoming gradient    */
/* and the outgoing input gradients are bf16, the gradients rounded     */
/* double -> FP32 -> bf16 (RNE both times).                             */
/* ------------------------------------------------------------------ */

static double orc_sigmoid(double g)
{
    double s = 1.0 / (1.0 + exp(-g));
    return s < 0x1p-126 ? 0.0 : s;
}

/* silu(g) * u */
double orc_swiglu(double g, double u)
{
    return g * orc_sigmoid(g) * u;
}

/* Partial derivatives of dh * silu(g) u:
 *   d/du = dh silu(g),
 *   d/dg = dh u (sigmoid(g) + g sigmoid(g)(1 - sigmoid(g))). */
void orc_swiglu_grad(double g, double u, double dh, double *dg, double *du)
{
    double s = orc_sigmoid(g);
    *du = dh * g * s;
    *dg = dh * u * s * (1.0 + g * (1.0 - s));
}

/* Forward over a rows x cols FP8 layer.  gate / up / out: codes with row
 * stride ld*_q bytes; per-group scale and k with row stride ld*_s floats
 * (groups of 128 along a row, the last one partial when cols % 128 != 0).
 * The output is quantised per 1x128 group with or without expansion.
 * Returns 0, or -1 on bad arguments. */
int orc_swiglu_fp8_forward(const uint8_t *gq, int64_t ldgq, const float *gs, const float *gk,
                           int64_t ldgs, const uint8_t *uq, int64_t lduq, const float *us,
                           const float *uk, int64_t ldus, int64_t rows, int64_t cols, int fmt,
                           int expand, uint8_t *oq, int64_t ldoq, float *os, float *ok,
                           int64_t ldos)
{
    if (rows < 0 || cols < 0 || ldgq < cols || lduq < cols || ldoq < cols)
        return -1;
    int64_t ng = (cols + 127) / 128;
    if (ldgs < ng || ldus < ng || ldos < ng)
        return -1;
    double h[128];
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < ng; j++) {
            int64_t c0 = j * 128, cnt = cols - c0 < 128 ? cols - c0 : 128;
            for (int64_t i = 0; i < cnt; i++) {
                double g = orc_dequant_value(fmt, gq[r * ldgq + c0 + i], gs[r * ldgs + j],
                                             gk[r * ldgs + j]);
                double u = orc_dequant_value(fmt, uq[r * lduq + c0 + i], us[r * ldus + j],
                                             uk[r * ldus + j]);
                h[i] = (double)(float)orc_swiglu(g, u);
            }
            orc_quantize_group(h, cnt, expand, fmt, oq + r * ldoq + c0, &ok[r * ldos + j],
                               &os[r * ldos + j]);
        }
    return 0;
}

/* Backward: dh (bf16 bits, row stride lddh elements) and the forward's FP8
 * inputs give dgate and dup (bf16 bits, row strides lddg / lddu). */
int orc_swiglu_fp8_backward(const uint16_t *dh, int64_t lddh, const uint8_t *gq, int64_t ldgq,
                            const float *gs, const float *gk, int64_t ldgs, const uint8_t *uq,
                            int64_t lduq, const float *us, const float *uk, int64_t ldus,
                            int64_t rows, int64_t cols, int fmt, uint16_t *dg, int64_t lddg,
                            uint16_t *du, int64_t lddu)
{
    if (rows < 0 || cols < 0 || lddh < cols || ldgq < cols || lduq < cols || lddg < cols ||
        lddu < cols)
        return -1;
    int64_t ng = (cols + 127) / 128;
    if (ldgs < ng || ldus < ng)
        return -1;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            int64_t j = c / 128;
            double g = orc_dequant_value(fmt, gq[r * ldgq + c], gs[r * ldgs + j], gk[r * ldgs + j]);
            double u = orc_dequant_value(fmt, uq[r * lduq + c], us[r * ldus + j], uk[r * ldus + j]);
            double a, b;
            orc_swiglu_grad(g, u, orc_bf16_to_double(dh[r * lddh + c]), &a, &b);
            dg[r * lddg + c] = orc_float_to_bf16((float)a);
            du[r * lddu + c] = orc_float_to_bf16((float)b);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* The second non-linear layer of the FP8 precision flow: Llama's      */
/* RMSNorm, y = x / sqrt(mean(x^2) + eps) * w, per row of d features,   */
/* with FP8 1x128 input and output and a bf16 weight; the backward      */
/* reads the saved FP8 input and a bf16 output gradient.                */
/* Readings: y is quantised from its double value (no FP32 rounding of  */
/* y itself: within a group y_i / y_max = x_i w_i / (x_max w_max), and  */
/* for k = 1 inputs that ratio is one of exact FP8 x bf16 products, so  */
/* the code is decided on the exact real number, ties to even, as the   */
/* kernel does); dx is rounded double -> FP32 -> bf16; dw (summed over  */
/* rows) is returned in double and compared with a tolerance, its       */
/* summation order being the kernel's own.                              */
/* ------------------------------------------------------------------ */

/* 1 / sqrt(mean(x^2) + eps) of one row of d values. */
static double orc_rstd(const double *x, int64_t d, double eps)
{
    double s = 0.0;
    for (int64_t i = 0; i < d; i++)
        s += x[i] * x[i];
    return 1.0 / sqrt(s / (double)d + eps);
}

static void orc_dequant_row(const uint8_t *q, const float *s, const float *k, int64_t d, int fmt,
                            double *x)
{
    for (int64_t i = 0; i < d; i++)
        x[i] = orc_dequant_value(fmt, q[i], s[i / 128], k[i / 128]);
}

/* Forward over rows x d: x codes (row stride ldxq bytes) with per-group
 * scale / k (row stride ldxs floats); w: d bf16 values; the output quantised
 * per 1x128 group into oq / os / ok.  rstd_out (may be NULL) receives each
 * row's 1 / sqrt(mean(x^2) + eps).  Returns 0, or -1 on bad arguments. */
int orc_rmsnorm_fp8_forward(const uint8_t *xq, int64_t ldxq, const float *xs, const float *xk,
                            int64_t ldxs, const uint16_t *w, int64_t rows, int64_t d, double eps,
                            int fmt, int expand, uint8_t *oq, int64_t ldoq, float *os, float *ok,
                            int64_t ldos, double *rstd_out)
{
    if (rows < 0 || d < 0 || ldxq < d || ldoq < d || !(eps > 0.0))
        return -1;
    int64_t ng = (d + 127) / 128;
    if (ldxs < ng || ldos < ng)
        return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
    double *y = (double *)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
    if (!x || !y) {
        free(x);
        free(y);
        return -1;
    }
    for (int64_t r = 0; r < rows; r++) {
        orc_dequant_row(xq + r * ldxq, xs + r * ldxs, xk + r * ldxs, d, fmt, x);
        double rs = orc_rstd(x, d, eps);
        if (rstd_out)
            rstd_out[r] = rs;
        for (int64_t i = 0; i < d; i++)
            y[i] = x[i] * rs * orc_bf16_to_double(w[i]);
        for (int64_t j = 0; j < ng; j++) {
            int64_t c0 = j * 128, cnt = d - c0 < 128 ? d - c0 : 128;
            orc_quantize_group(y + c0, cnt, expand, fmt, oq + r * ldoq + c0, &ok[r * ldos + j],
                               &os[r * ldos + j]);
        }
    }
    free(x);
    free(y);
    return 0;
}

/* Backward: with xh = x rstd and g = dy w,
 *   dx = rstd (g - xh mean(g xh)),   dw = sum over rows of dy xh.
 * dy: bf16 (row stride lddy); dx: bf16 (row stride lddx); dw: d doubles. */
int orc_rmsnorm_fp8_backward(const uint16_t *dy, int64_t lddy, const uint8_t *xq, int64_t ldxq,
                             const float *xs, const float *xk, int64_t ldxs, const uint16_t *w,
                             int64_t rows, int64_t d, double eps, int fmt, uint16_t *dx,
                             int64_t lddx, double *dw)
{
    if (rows < 0 || d < 0 || lddy < d || ldxq < d || lddx < d || !(eps > 0.0))
        return -1;
    int64_t ng = (d + 127) / 128;
    if (ldxs < ng)
        return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
    if (!x)
        return -1;
    for (int64_t i = 0; i < d; i++)
        dw[i] = 0.0;
    for (int64_t r = 0; r < rows; r++) {
        orc_dequant_row(xq + r * ldxq, xs + r * ldxs, xk + r * ldxs, d, fmt, x);
        double rs = orc_rstd(x, d, eps);
        double dot = 0.0;   /* sum of g xh */
        for (int64_t i = 0; i < d; i++)
            dot += orc_bf16_to_double(dy[r * lddy + i]) * orc_bf16_to_double(w[i]) * x[i] * rs;
        double mean = dot / (double)d;
        for (int64_t i = 0; i < d; i++) {
            double dyi = orc_bf16_to_double(dy[r * lddy + i]);
            double xh = x[i] * rs;
            double g = dyi * orc_bf16_to_double(w[i]);
            dx[r * lddx + i] = orc_float_to_bf16((float)(rs * (g - xh * mean)));
            dw[i] += dyi * xh;
        }
    }
    free(x);
    return 0;
}
