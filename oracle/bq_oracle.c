/*
 * Oracle for the quantized linear layer: plain, slow, obviously correct host C.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the timed
 * CPU baseline of the benchmark use it.  It shares no code, header, table or
 * constant with the CUDA library; the two only meet through the seeded input
 * generator, which holds none of the arithmetic below.
 *
 * Every routine works in double precision (IEEE binary64), uses no blocking,
 * no reordering and no fused multiply-add (build with -ffp-contract=off), and
 * follows the pages it cites step by step:
 *
 *   [BitLinear]  "Class BitLinear" (LLaMA-BitNet utils.py), class docstring
 *                "Forward pass (training)" steps 1-5 and forward().
 *   [common]     "Common Attention Utilities" (frankenstein-transformer
 *                src.model.attention.common): activation_quant, weight_quant,
 *                BitLinear.bake_ternary_weights.
 *   [ATB]        "Per-token Quantization for Matmul" (Huawei CANN ATB):
 *                Input / Output tables and the Example.
 *   [linear_4bit] "vyre_libs/nn/linear/inner/linear_4bit/mod.rs" (docs.rs
 *                vyre-libs 0.7.2): module doc, QuantizedLinear4BitSpec.
 *   [Q4Linear]   "bitorch_engine.layers.qlinear.nbit.cutlass.q4_layer.
 *                Q4LinearFunction" (bitorch-engine docs): forward(x, weight,
 *                scale_a, scale_w, eps, is_train) and backward(output_gradient).
 *
 * Readings taken where the pages are silent (each is also listed in the
 * design notes): RMSNorm puts eps inside the square root; the activation
 * scale maps the row's absolute maximum to 127; absmax and absmean are
 * clamped below at 1e-5; rounding is half-to-even; the ternary code is stored
 * offset-binary (w+1) two bits per weight; INT4 nibbles are packed low-nibble
 * first along the reduction axis; the INT4 affine form is s*(q - z).
 *
 * Pins: every function here is checked by the CPU test-suite against values
 * the pages print (the ATB example), closed forms, invariants, library
 * routines on special cases, and (for the backward passes) autograd of the
 * straight-through forward.  The BitLinear composition is pinned through its
 * steps, closed-form special cases and a one-code-per-row case that fixes
 * the weight indexing.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_ABSMAX_FLOOR 1e-5   /* absmax / absmean lower clamp            */
#define ORACLE_ACT_QMAX 127.0      /* int8 activations scaled to +-127        */

/* Round half to even, written out: floor, then compare the remainder. */
double bq_oracle_round_half_even(double v)
{
    double f = floor(v);
    double d = v - f; /* exact for |v| < 2^52 */
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

static double clampd(double v, double lo, double hi)
{
    return v < lo ? lo : (v > hi ? hi : v);
}

/*
 * Per-token activation quantization after a parameter-free RMSNorm.
 * [BitLinear] steps 1-2 (internal RMSNorm, 8-bit per-token quantization);
 * [common] activation_quant (per-token scale over the last dimension into
 * [-128, 127], round to integer).
 *
 *   r[m]        = sqrt( (1/K) sum_k x[m,k]^2 + eps )
 *   y[m,k]      = x[m,k] / r[m]
 *   a[m]        = max( max_k |y[m,k]|, 1e-5 )
 *   pre[m,k]    = y[m,k] * 127 / a[m]              (pre-rounding value)
 *   xq[m,k]     = clamp( round_half_even(pre), -128, 127 )
 *   act_scale[m]= a[m] / 127                       (multiplied back in step 5)
 *   rowsum[m]   = sum_k xq[m,k]
 *
 * x is read as float (bf16 inputs are passed widened, which is exact).
 * Optional outputs (pre, y, rowsum) may be NULL.  Dense row-major [M,K].
 */
void bq_oracle_act_quant(const float *x, int64_t M, int64_t K, double eps,
                         int8_t *xq, double *act_scale, int64_t *rowsum,
                         double *pre, double *y_out)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *xr = x + m * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += (double)xr[k] * (double)xr[k];
        double r = sqrt(ss / (double)K + eps);

        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double y = (double)xr[k] / r;
            if (y_out) y_out[m * K + k] = y;
            if (fabs(y) > amax) amax = fabs(y);
        }
        double a = amax > ORACLE_ABSMAX_FLOOR ? amax : ORACLE_ABSMAX_FLOOR;

        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            double y = (double)xr[k] / r;
            double v = y * ORACLE_ACT_QMAX / a;
            if (pre) pre[m * K + k] = v;
            double q = clampd(bq_oracle_round_half_even(v), -128.0, 127.0);
            xq[m * K + k] = (int8_t)q;
            sum += (int64_t)q;
        }
        act_scale[m] = a / ORACLE_ACT_QMAX;
        if (rowsum) rowsum[m] = sum;
    }
}

/*
 * Per-token activation quantization after a LayerNorm, the normaliser of the
 * BitLinear and BitConv1d layers of [common] ("Applies LayerNorm to inputs
 * before quantization"; BitConv1d normalises over the channel dimension),
 * followed by the same 8-bit per-token quantization as above:
 *
 *   mu[m]      = (1/K) sum_k x[m,k]
 *   var[m]     = (1/K) sum_k (x[m,k] - mu[m])^2          (biased, as LayerNorm)
 *   y[m,k]     = (x[m,k] - mu[m]) / sqrt(var[m] + eps) * g[k] + b[k]
 *   a[m]       = max( max_k |y[m,k]|, 1e-5 )
 *   pre[m,k]   = y[m,k] * 127 / a[m]
 *   xq[m,k]    = clamp( round_half_even(pre), -128, 127 )
 *   act_scale[m] = a[m] / 127,   rowsum[m] = sum_k xq[m,k]
 *
 * g (ln_weight) and b (ln_bias) are the LayerNorm's elementwise affine
 * parameters, [K] each; NULL stands for g = 1 and b = 0 (a parameter-free
 * LayerNorm).  Optional outputs (rowsum, pre, y) may be NULL.
 */
void bq_oracle_act_quant_layernorm(const float *x, int64_t M, int64_t K, double eps,
                                   const float *g, const float *b, int8_t *xq,
                                   double *act_scale, int64_t *rowsum, double *pre,
                                   double *y_out)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *xr = x + m * K;
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k) sum += (double)xr[k];
        double mu = sum / (double)K;
        double sq = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double d = (double)xr[k] - mu;
            sq += d * d;
        }
        double sd = sqrt(sq / (double)K + eps);

        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double y = ((double)xr[k] - mu) / sd * (g ? (double)g[k] : 1.0) + (b ? (double)b[k] : 0.0);
            if (y_out) y_out[m * K + k] = y;
            if (fabs(y) > amax) amax = fabs(y);
        }
        double a = amax > ORACLE_ABSMAX_FLOOR ? amax : ORACLE_ABSMAX_FLOOR;

        int64_t total = 0;
        for (int64_t k = 0; k < K; ++k) {
            double y = ((double)xr[k] - mu) / sd * (g ? (double)g[k] : 1.0) + (b ? (double)b[k] : 0.0);
            double v = y * ORACLE_ACT_QMAX / a;
            if (pre) pre[m * K + k] = v;
            double q = clampd(bq_oracle_round_half_even(v), -128.0, 127.0);
            xq[m * K + k] = (int8_t)q;
            total += (int64_t)q;
        }
        act_scale[m] = a / ORACLE_ACT_QMAX;
        if (rowsum) rowsum[m] = total;
    }
}

/*
 * Ternary Conv1d ([common] BitConv1d: "the same ternary weight ({-1, 0, 1}) +
 * int8 activation quantization as BitLinear"; "Inputs are LayerNorm-
 * normalized over the channel dimension before activation quantization";
 * forward maps (B, C_in, L) to (B, C_out, L_out)), from the quantized
 * operands:
 *
 *   xq [B, L, C_in] and act_scale [B, L]: the per-position codes and scales
 *       of the LayerNorm-normalised input (position-major, as act quant of
 *       the rows of x transposed to (B, L, C_in));
 *   wq [C_out, C_in / groups, KS] ternary codes with one scale gamma;
 *   out[b, co, lo] = gamma * sum_t sum_c wq[co, c, t] * xq[b, p, g * Cg + c]
 *                    * act_scale[b, p]      (+ bias[co])
 *       with p = lo * stride + t - pad (taps outside [0, L) add nothing),
 *       Cg = C_in / groups, g = co / (C_out / groups),
 *       L_out = (L + 2 pad - KS) / stride + 1.
 *
 * Each tap's integer dot product is exact; it is scaled by the scale of the
 * position it reads, and the taps are summed in double.
 */
void bq_oracle_bitconv1d_from_codes(const int8_t *xq, const double *act_scale, const int8_t *wq,
                                    double gamma, const float *bias, int64_t B, int64_t C_in,
                                    int64_t L, int64_t C_out, int64_t KS, int64_t stride,
                                    int64_t pad, int64_t groups, double *out)
{
    int64_t L_out = (L + 2 * pad - KS) / stride + 1;
    int64_t Cg = C_in / groups, Cog = C_out / groups;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t co = 0; co < C_out; ++co) {
            int64_t g = co / Cog;
            for (int64_t lo = 0; lo < L_out; ++lo) {
                double sum = 0.0;
                for (int64_t t = 0; t < KS; ++t) {
                    int64_t p = lo * stride + t - pad;
                    if (p < 0 || p >= L) continue;
                    int64_t acc = 0;
                    for (int64_t c = 0; c < Cg; ++c)
                        acc += (int64_t)wq[(co * Cg + c) * KS + t] * (int64_t)xq[(b * L + p) * C_in + g * Cg + c];
                    sum += (double)acc * act_scale[b * L + p];
                }
                double v = gamma * sum;
                if (bias) v += (double)bias[co];
                out[(b * C_out + co) * L_out + lo] = v;
            }
        }
}

/*
 * Absmean ternary weight quantization with the bake rule.
 * [BitLinear] step 3 (ternary {-1,0,+1} via absmean); [common] weight_quant
 * (scale by the inverse mean absolute value, round to the nearest integer in
 * [-1, 1]) and bake_ternary_weights (a weight whose nonzero entries all equal
 * +-max|w| is already ternary and is left as it is, so its scale is max|w|).
 *
 *   if some w != 0 and every nonzero |w| == max|w| = c:   gamma = c
 *   else:  gamma = max( (1/(N K)) sum |w|, 1e-5 )
 *   pre = w / gamma;   wq = clamp( round_half_even(pre), -1, 1 )
 *
 * Returns 1 when the bake rule applied, 0 otherwise.  pre may be NULL.
 */
int bq_oracle_ternary_quant(const float *w, int64_t N, int64_t K, double *gamma,
                            int8_t *wq, double *pre)
{
    int64_t n_el = N * K;
    double c = 0.0;
    for (int64_t i = 0; i < n_el; ++i)
        if (fabs((double)w[i]) > c) c = fabs((double)w[i]);

    int already_ternary = c > 0.0;
    for (int64_t i = 0; i < n_el && already_ternary; ++i) {
        double aw = fabs((double)w[i]);
        if (aw != 0.0 && aw != c) already_ternary = 0;
    }

    double g;
    if (already_ternary) {
        g = c;
    } else {
        double s = 0.0;
        for (int64_t i = 0; i < n_el; ++i) s += fabs((double)w[i]);
        g = s / (double)n_el;
        if (g < ORACLE_ABSMAX_FLOOR) g = ORACLE_ABSMAX_FLOOR;
    }
    *gamma = g;

    for (int64_t i = 0; i < n_el; ++i) {
        double v = (double)w[i] / g;
        if (pre) pre[i] = v;
        wq[i] = (int8_t)clampd(bq_oracle_round_half_even(v), -1.0, 1.0);
    }
    return already_ternary;
}

/* bake(W) = wq * gamma, the weight that bake_ternary_weights stores. */
void bq_oracle_ternary_bake(const int8_t *wq, double gamma, int64_t n_el, float *out)
{
    for (int64_t i = 0; i < n_el; ++i) out[i] = (float)((double)wq[i] * gamma);
}

/*
 * Two-bit ternary packing (the pages fix no bit layout; this is the layout
 * the library documents).  Row n of wq [N,K] becomes K/16 words; the code of
 * element k = 16*w + 4*j + b is (wq + 1) in {0,1,2}, stored in bits
 * [8*b + 2*j, 8*b + 2*j + 1] of word w.  K must be a multiple of 16.
 */
void bq_oracle_ternary_pack(const int8_t *wq, int64_t N, int64_t K, uint32_t *packed)
{
    int64_t words = K / 16;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t wi = 0; wi < words; ++wi) {
            uint32_t word = 0;
            for (int j = 0; j < 4; ++j)
                for (int b = 0; b < 4; ++b) {
                    int64_t k = 16 * wi + 4 * j + b;
                    uint32_t code = (uint32_t)(wq[n * K + k] + 1);
                    word |= code << (8 * b + 2 * j);
                }
            packed[n * words + wi] = word;
        }
}

/* Inverse of bq_oracle_ternary_pack; returns the number of invalid codes (3). */
int64_t bq_oracle_ternary_unpack(const uint32_t *packed, int64_t N, int64_t K, int8_t *wq)
{
    int64_t words = K / 16, bad = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t wi = k / 16, j = (k % 16) / 4, b = k % 4;
            uint32_t code = (packed[n * words + wi] >> (8 * b + 2 * j)) & 3u;
            if (code == 3u) ++bad;
            wq[n * K + k] = (int8_t)((int)code - 1);
        }
    return bad;
}

/*
 * Nibble packing along the last axis, eight per 32-bit word ([linear_4bit]
 * module doc: the kernel loads the packed u32 word and extracts the nibble
 * for k).  Element c of a row sits in bits [4*(c%8), 4*(c%8)+3] of word c/8
 * (low nibble first); a ragged last word is zero-padded.  Values must be
 * 0..15.  Used for weights [N,K] and for zero-points [N,G].
 */
void bq_oracle_int4_pack(const uint8_t *q, int64_t rows, int64_t cols, uint32_t *packed)
{
    int64_t words = (cols + 7) / 8;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t wi = 0; wi < words; ++wi) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) {
                int64_t c = 8 * wi + j;
                if (c < cols) word |= ((uint32_t)q[r * cols + c] & 15u) << (4 * j);
            }
            packed[r * words + wi] = word;
        }
}

void bq_oracle_int4_unpack(const uint32_t *packed, int64_t rows, int64_t cols, uint8_t *q)
{
    int64_t words = (cols + 7) / 8;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            q[r * cols + c] = (uint8_t)((packed[r * words + c / 8] >> (4 * (c % 8))) & 15u);
}

/*
 * IEEE 754 binary16 bits to double, from the format's definition:
 * sign, 5-bit exponent (bias 15), 10-bit fraction; exponent 0 is subnormal.
 */
double bq_oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/*
 * Per-token W8A8 matmul with dequantization ([ATB] Input/Output tables and
 * the Example, whose printed arithmetic fixes the formula):
 *
 *   acc[m,n] = sum_k x[m,k] * weight(k,n)          (exact, int64)
 *   out[m,n] = (acc * deqScale[n]) * perTokenScale[m]  (+ bias[n])
 *
 * weight(k,n) = w[n*ldw + k] for layout 0 ([N,K], the nn.Linear layout,
 * ATB transposeB = true) or w[k*ldw + n] for layout 1 ([K,N], the ATB
 * default).  bias may be NULL.  out is dense [M,N].
 * Returns the number of accumulators outside the int32 range (must be 0).
 */
int64_t bq_oracle_gemm_i8_pertoken(const int8_t *x, int64_t ldx, const int8_t *w,
                                   int layout, int64_t ldw, const float *deq_scale,
                                   const float *per_token_scale, const float *bias,
                                   int64_t M, int64_t N, int64_t K, double *out)
{
    int64_t overflow = 0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t wv = layout == 0 ? w[n * ldw + k] : w[k * ldw + n];
                acc += (int64_t)x[m * ldx + k] * wv;
            }
            if (acc > 2147483647LL || acc < -2147483648LL) ++overflow;
            double v = ((double)acc * (double)deq_scale[n]) * (double)per_token_scale[m];
            if (bias) v += (double)bias[n];
            out[m * N + n] = v;
        }
    return overflow;
}

/*
 * Batched and transposed forms of the per-token W8A8 matmul ([ATB] Input /
 * Output tables: x [m,k] or [batch,m,k], weight [k,n] or [batch,k,n],
 * output [batch,m,n]; Parameters: transposeA and transposeB).  For each batch
 * b the 2-D formula above, with
 *
 *   x(b,m,k)      = x[b*sx + m*ldx + k]       (trans_a = 0: x is [M,K] per batch)
 *                 = x[b*sx + k*ldx + m]       (trans_a = 1: x is stored [K,M])
 *   weight(b,k,n) = w[b*sw + n*ldw + k]       (layout 0, [N,K])
 *                 = w[b*sw + k*ldw + n]       (layout 1, [K,N])
 *   deqScale(b,n) = deq[b*sdeq + n],  perTokenScale(b,m) = pts[b*spts + m]
 *
 * (sdeq = spts = 0 is the tables' reading: one [n] and one [m] vector shared
 * by every batch; the strides N and M give one per batch).  out is dense
 * [batch,M,N].  Returns the number of accumulators outside int32.
 */
int64_t bq_oracle_gemm_i8_pertoken_batched(const int8_t *x, int64_t ldx, int64_t sx, int trans_a,
                                           const int8_t *w, int layout, int64_t ldw, int64_t sw,
                                           const float *deq, int64_t sdeq, const float *pts, int64_t spts,
                                           const float *bias, int64_t batch, int64_t M, int64_t N,
                                           int64_t K, double *out)
{
    int64_t overflow = 0;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = 0; n < N; ++n) {
                int64_t acc = 0;
                for (int64_t k = 0; k < K; ++k) {
                    int64_t xv = trans_a ? x[b * sx + k * ldx + m] : x[b * sx + m * ldx + k];
                    int64_t wv = layout == 0 ? w[b * sw + n * ldw + k] : w[b * sw + k * ldw + n];
                    acc += xv * wv;
                }
                if (acc > 2147483647LL || acc < -2147483648LL) ++overflow;
                double v = ((double)acc * (double)deq[b * sdeq + n]) * (double)pts[b * spts + m];
                if (bias) v += (double)bias[n];
                out[(b * M + m) * N + n] = v;
            }
    return overflow;
}

/*
 * 4-bit quantization with a given step size ([Q4Linear] forward: activations
 * and weights are quantized "to 4-bits using specified scale factors"; eps
 * "to avoid division by zero").  Row r of v [rows, cols] uses the step
 *   s_r = max(scale[r * scale_stride], eps)       (stride 0: one step for all)
 *   pre = v / s_r;   q = clamp(round_half_even(pre), -8, 7)
 * pre may be NULL.
 */
void bq_oracle_q4_quant(const float *v, int64_t rows, int64_t cols, const float *scale,
                        int64_t scale_stride, double eps, int8_t *q, double *pre)
{
    for (int64_t r = 0; r < rows; ++r) {
        double st = (double)scale[r * scale_stride];
        if (st < eps) st = eps;
        for (int64_t c = 0; c < cols; ++c) {
            double x = (double)v[r * cols + c] / st;
            if (pre) pre[r * cols + c] = x;
            q[r * cols + c] = (int8_t)clampd(bq_oracle_round_half_even(x), -8.0, 7.0);
        }
    }
}

/*
 * The Q4Linear forward ([Q4Linear] forward: quantize x and weight to 4 bits,
 * then the linear operation), from 4-bit codes:
 *   out[m,n] = ((sum_k xq[m,k] * wq[n,k]) * s_w[n]) * s_a   (+ bias[n])
 * with s_a = max(scale_a, eps) and s_w[n] = max(scale_w[n * sw_stride], eps).
 */
void bq_oracle_linear_w4a4_from_codes(const int8_t *xq, const int8_t *wq, const float *scale_a,
                                      const float *scale_w, int64_t sw_stride, double eps,
                                      const float *bias, int64_t M, int64_t N, int64_t K,
                                      double *out)
{
    double sa = (double)scale_a[0];
    if (sa < eps) sa = eps;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)xq[m * K + k] * (int64_t)wq[n * K + k];
            double sw = (double)scale_w[n * sw_stride];
            if (sw < eps) sw = eps;
            double v = ((double)acc * sw) * sa;
            if (bias) v += (double)bias[n];
            out[m * N + n] = v;
        }
}

/*
 * The Q4Linear backward ([Q4Linear] backward: gradients for the input, the
 * weight and the activation scale, "adjusted based on quantization ranges";
 * none for scale_w and eps), read as straight-through rounding passed only
 * inside the clamp range.  With the forward's steps s_a = max(scale_a, eps),
 * s_w[n] = max(scale_w[n * sw_stride], eps), quotients u = x / s_a,
 * v = w / s_w[n], codes xq = clamp(rne(u), -8, 7), wq = clamp(rne(v), -8, 7),
 * and the dequantized operands xh = s_a * xq, wh[n,:] = s_w[n] * wq[n,:]
 * (out = xh wh^T + bias):
 *
 *   g[m,k]   = sum_n dout[m,n] * wh[n,k]                (gradient reaching xh)
 *   dx[m,k]  = g[m,k]          if -8 <= u[m,k] <= 7, else 0
 *   dw[n,k]  = sum_m dout[m,n] * xh[m,k]   if -8 <= v[n,k] <= 7, else 0
 *   dscale_a = sum_{m,k} g[m,k] * d xh[m,k] / d s_a,
 *              d xh / d s_a = xq - u inside the range, xq (the bound) outside,
 *              and dscale_a = 0 when scale_a < eps (s_a is then the constant eps).
 *
 * g (optional) receives g[m,k].
 */
void bq_oracle_linear_w4a4_backward(const float *x, const float *w, const float *dout,
                                    const float *scale_a, const float *scale_w, int64_t sw_stride,
                                    double eps, int64_t M, int64_t N, int64_t K, double *dx,
                                    double *dw, double *dscale_a, double *g)
{
    int8_t *xq = (int8_t *)malloc((size_t)(M * K));
    int8_t *wq = (int8_t *)malloc((size_t)(N * K));
    double *u = (double *)malloc((size_t)(M * K) * sizeof(double));
    double *v = (double *)malloc((size_t)(N * K) * sizeof(double));
    double sa = (double)scale_a[0];
    int sa_clamped = sa < eps;
    if (sa_clamped) sa = eps;
    bq_oracle_q4_quant(x, M, K, scale_a, 0, eps, xq, u);
    bq_oracle_q4_quant(w, N, K, scale_w, sw_stride, eps, wq, v);
    double ds = 0.0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double gk = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double sw = (double)scale_w[n * sw_stride];
                if (sw < eps) sw = eps;
                gk += (double)dout[m * N + n] * (sw * (double)wq[n * K + k]);
            }
            if (g) g[m * K + k] = gk;
            double um = u[m * K + k];
            int inside = um >= -8.0 && um <= 7.0;
            dx[m * K + k] = inside ? gk : 0.0;
            double dxh_ds = inside ? (double)xq[m * K + k] - um : (double)xq[m * K + k];
            ds += gk * dxh_ds;
        }
    *dscale_a = sa_clamped ? 0.0 : ds;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t m = 0; m < M; ++m) s += (double)dout[m * N + n] * (sa * (double)xq[m * K + k]);
            double vn = v[n * K + k];
            dw[n * K + k] = (vn >= -8.0 && vn <= 7.0) ? s : 0.0;
        }
    free(xq);
    free(wq);
    free(u);
    free(v);
}

/*
 * Signed 4-bit codes packed eight per 32-bit word along the row, low nibble
 * first (element c of a row in bits [4*(c%8), 4*(c%8)+3] of word c/8, as the
 * two's-complement nibble of a value in [-8, 7]).  cols % 8 == 0.
 */
void bq_oracle_s4_pack(const int8_t *q, int64_t rows, int64_t cols, uint32_t *packed)
{
    int64_t words = cols / 8;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t wi = 0; wi < words; ++wi) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j)
                word |= ((uint32_t)q[r * cols + 8 * wi + j] & 15u) << (4 * j);
            packed[r * words + wi] = word;
        }
}

/*
 * BitLinear steps 4-5 from the quantized operands ([BitLinear] forward:
 * F.linear(x_q, w_q) then out * act_scale * w_scale):
 *
 *   out[m,n] = ((sum_k xq[m,k] * wq[n,k]) * act_scale[m]) * gamma  (+ bias[n])
 *
 * xq [M,K], wq [N,K] dense; bias may be NULL (the page disables it by
 * default).  Also writes the exact integer accumulators when acc != NULL.
 */
void bq_oracle_bitlinear_from_codes(const int8_t *xq, const double *act_scale,
                                    const int8_t *wq, double gamma, const float *bias,
                                    int64_t M, int64_t N, int64_t K, double *out,
                                    int64_t *acc_out)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)xq[m * K + k] * (int64_t)wq[n * K + k];
            if (acc_out) acc_out[m * N + n] = acc;
            double v = ((double)acc * act_scale[m]) * gamma;
            if (bias) v += (double)bias[n];
            out[m * N + n] = v;
        }
}

/*
 * Backward of the BitLinear forward under the straight-through estimator
 * ([BitLinear] "Quantise ... (STE)" in steps 2-3; [common] activation_quant and
 * weight_quant: the STE "passes gradients through the rounding operation
 * unchanged").  The forward used xt = xq * act_scale in place of the
 * normalised y and wt = wq * gamma in place of w, with identity gradients
 * through both, so for dout [M,N]:
 *
 *   dW[n,k] = sum_m dout[m,n] * xq[m,k] * act_scale[m]
 *   dy[m,k] = sum_n dout[m,n] * wq[n,k] * gamma
 *   dx[m,k] = (dy[m,k] - y[m,k] * (1/K) sum_j dy[m,j] * y[m,j]) / r[m]
 *
 * the last line being the backward of the parameter-free RMSNorm
 * y = x / r, r = sqrt(mean(x^2) + eps).  x [M,K], w [N,K], dout [M,N].
 */
void bq_oracle_bitlinear_backward(const float *x, const float *w, const float *dout, int64_t M,
                                  int64_t N, int64_t K, double eps, double *dx, double *dw)
{
    int8_t *xq = (int8_t *)malloc((size_t)(M * K));
    int8_t *wq = (int8_t *)malloc((size_t)(N * K));
    double *act = (double *)malloc((size_t)M * sizeof(double));
    double *y = (double *)malloc((size_t)(M * K) * sizeof(double));
    double *dy = (double *)malloc((size_t)K * sizeof(double));
    double gamma;
    bq_oracle_act_quant(x, M, K, eps, xq, act, NULL, NULL, y);
    bq_oracle_ternary_quant(w, N, K, &gamma, wq, NULL);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t m = 0; m < M; ++m)
                s += (double)dout[m * N + n] * ((double)xq[m * K + k] * act[m]);
            dw[n * K + k] = s;
        }
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += (double)x[m * K + k] * (double)x[m * K + k];
        double r = sqrt(ss / (double)K + eps);
        double dot = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t n = 0; n < N; ++n) s += (double)dout[m * N + n] * ((double)wq[n * K + k] * gamma);
            dy[k] = s;
            dot += s * y[m * K + k];
        }
        for (int64_t k = 0; k < K; ++k)
            dx[m * K + k] = (dy[k] - y[m * K + k] * (dot / (double)K)) / r;
    }
    free(xq);
    free(wq);
    free(act);
    free(y);
    free(dy);
}

/*
 * Grouped affine INT4 linear ([linear_4bit] module doc: unpack-on-demand
 * nibble extraction inside the k loop; grouped affine path with a scale and
 * a zero-point per group, plus bias):
 *
 *   g = k / group_size
 *   q = nibble k of row n of qweight [N, K/8];  z = nibble g of row n of
 *   qzeros [N, ceil(G/8)];  s = scales[n, g] (binary16 bits)
 *   out[m,n] = bias[n] + sum_k x[m,k] * s * (q - z)
 *
 * accumulated in double.  bias may be NULL.  out is dense [M,N].
 */
void bq_oracle_linear_w4_grouped(const float *x, int64_t M, int64_t K,
                                 const uint32_t *qweight, const uint16_t *scales_f16,
                                 const uint32_t *qzeros, const float *bias, int64_t N,
                                 int64_t group_size, double *out)
{
    int64_t G = K / group_size;
    int64_t wwords = K / 8, zwords = (G + 7) / 8;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t g = k / group_size;
                int q = (int)((qweight[n * wwords + k / 8] >> (4 * (k % 8))) & 15u);
                int z = (int)((qzeros[n * zwords + g / 8] >> (4 * (g % 8))) & 15u);
                double s = bq_oracle_half_to_double(scales_f16[n * G + g]);
                sum += (double)x[m * K + k] * s * (double)(q - z);
            }
            out[m * N + n] = (bias ? (double)bias[n] : 0.0) + sum;
        }
}
