/*
 * bq.h - C ABI of libbq.so, a B200 (sm_100a) implementation of the quantized
 * linear layer: per-token int8 activation quantization after a
 * parameter-free RMSNorm, ternary (absmean) or grouped affine INT4 weights,
 * and integer matmuls with a fused dequantizing epilogue.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensor pointers are device pointers owned by the caller.  The library
 *    never allocates, frees or synchronizes: scratch memory is the caller's
 *    `workspace`, sized with bq_workspace_bytes().
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) on the calling thread's current device.
 *  - Matrices are row-major.  Leading dimensions (ld*) count elements.
 *    Unless a call says otherwise, base pointers must be 16-byte aligned and
 *    ld * element size must be a multiple of 16 bytes (TMA and vector-load
 *    requirement); a violation returns BQ_ERR_MISALIGNED.
 *  - Arguments are validated before anything is launched; an invalid call
 *    returns a status != BQ_OK and leaves every output untouched.  M == 0 or
 *    N == 0 is a valid empty call (BQ_OK, nothing launched); K must be >= 1.
 *  - A CUDA error raised by a launch is returned as BQ_ERR_CUDA.
 *  - Kernels bound every wait they perform.  A wait that runs out (it cannot
 *    happen with a correct build) or an invalid value met inside a kernel
 *    (a nibble > 15) is recorded in a per-device status word and the kernel
 *    returns early; read and clear it with bq_device_status().
 *  - Inputs must be finite.  Rounding is to nearest, ties to even.
 *  - Per-device state (the status word's and the static scratch's device
 *    addresses, kernel shared-memory opt-ins) is cached against the device's
 *    current context and looked up again when that context changes (e.g.
 *    after cudaDeviceReset); calls racing with a reset are not supported.
 *
 * Data formats
 * ------------
 *  - Ternary weights (bq_weight_quant_ternary_pack, bq_bitlinear_w2a8):
 *    uint32 wpacked[N][K/16].  Element k = 16*w + 4*j + b of row n has the
 *    offset-binary code (w_q + 1) in {0,1,2} in bits [8b+2j, 8b+2j+1] of
 *    word w, so (word >> 2j) & 0x03030303 yields the codes of k = 16w+4j+0..3
 *    as four bytes.  One fp32 scale gamma per tensor.
 *  - INT4 weights (bq_weight_pack_int4_grouped, bq_linear_w4_grouped):
 *    uint32 qweight[N][K/8], element k of row n in bits [4*(k%8), 4*(k%8)+3]
 *    of word k/8 (low nibble first); zero-points uint32 qzeros[N][ceil(G/8)]
 *    packed the same way along the group axis (G = K / group_size, ragged
 *    last word zero-padded); scales IEEE binary16 [N][G]; dequantized weight
 *    w[n,k] = scale[n,g] * (q[n,k] - zero[n,g]) with g = k / group_size.
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *bq_stream_t; /* a cudaStream_t */

typedef enum {
    BQ_OK = 0,
    BQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad enum, value out of range */
    BQ_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. no sm_100 device)   */
    BQ_ERR_MISALIGNED = 3,  /* pointer / leading-dimension alignment rule broken   */
    BQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required          */
    BQ_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed                 */
    BQ_ERR_TIMEOUT = 6      /* (device status only) a bounded wait ran out         */
} bq_status;

typedef enum { BQ_F32 = 0, BQ_BF16 = 1, BQ_F16 = 2 } bq_dtype;

typedef enum {
    BQ_W_NK = 0, /* weight [N][K], K contiguous: nn.Linear layout (ATB transposeB = true) */
    BQ_W_KN = 1  /* weight [K][N], N contiguous: the ATB operator's default layout        */
} bq_wlayout;

typedef enum {
    BQ_OP_ACT_QUANT_INT8 = 0,
    BQ_OP_WEIGHT_QUANT_TERNARY_PACK = 1,
    BQ_OP_WEIGHT_PACK_INT4_GROUPED = 2,
    BQ_OP_GEMM_I8_PERTOKEN = 3,
    BQ_OP_BITLINEAR_W2A8 = 4,
    BQ_OP_LINEAR_W4_GROUPED = 5,
    BQ_OP_LINEAR_W4A4 = 6,
    BQ_OP_BITLINEAR_W2A8_BACKWARD = 7,
    BQ_OP_LINEAR_W4A4_BACKWARD = 8
} bq_op;

/*
 * Per-token int8 activation quantization after a parameter-free RMSNorm.
 * Source: "Class BitLinear" (LLaMA-BitNet utils.py), forward steps 1-2, and
 * "Common Attention Utilities" (frankenstein-transformer), activation_quant.
 *
 *   r[m] = sqrt(mean_k x[m,k]^2 + eps),  a[m] = max(max_k |x[m,k]| / r[m], 1e-5)
 *   xq[m,k] = clamp(rne(x[m,k] / r[m] * 127 / a[m]), -128, 127)   (|xq| <= 127)
 *   act_scale[m] = a[m] / 127,   rowsum[m] = sum_k xq[m,k]
 *
 * x: [M][ldx] of x_dtype BQ_F32 or BQ_BF16 (row base 16-byte aligned when
 * ldx*size % 16 == 0; any K >= 1).  xq: int8 [M][ldq], 16-byte aligned,
 * ldq % 16 == 0, ldq >= K.  act_scale: fp32 [M].  rowsum: int32 [M] or NULL.
 */
bq_status bq_act_quant_int8(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, int64_t ldx,
                            float eps, int8_t *xq, int64_t ldq, float *act_scale, int32_t *rowsum,
                            bq_stream_t stream);

/*
 * Absmean ternary quantization and 2-bit packing of a weight matrix.
 * Source: "Common Attention Utilities", weight_quant and
 * BitLinear.bake_ternary_weights; "Class BitLinear", forward step 3.
 *
 *   gamma = max|w| if w has a nonzero entry and every nonzero |w| equals
 *           max|w| (already ternary: the bake rule keeps it unchanged);
 *           otherwise max(mean|w|, 1e-5), the mean taken in fp64.
 *   w_q = clamp(rne(w / gamma), -1, 1);  wpacked as in "Data formats".
 *
 * w: dense [N][K] of w_dtype BQ_F32 or BQ_BF16, 16-byte aligned; K % 16 == 0.
 * wpacked: uint32 [N][K/16], 16-byte aligned.  w_scale: one fp32 on the
 * device (written without a host round trip).  workspace: at least
 * bq_workspace_bytes(BQ_OP_WEIGHT_QUANT_TERNARY_PACK, 0, N, K, 0) bytes,
 * 256-byte aligned.  The result is deterministic (fixed reduction order).
 */
bq_status bq_weight_quant_ternary_pack(const void *w, bq_dtype w_dtype, int64_t N, int64_t K,
                                       uint32_t *wpacked, float *w_scale, void *workspace,
                                       size_t workspace_bytes, bq_stream_t stream);

/*
 * Pack INT4 codes and zero-points into u32 words of eight nibbles.
 * Source: "vyre_libs/nn/linear/inner/linear_4bit/mod.rs" (docs.rs vyre-libs),
 * module doc (packed u32 weight, nibble extracted in the k loop) and
 * QuantizedLinear4BitSpec (typed packed-word layout).
 *
 * q: uint8 [N][K] codes 0..15, K % 8 == 0.  zeros: uint8 [N][G] codes 0..15,
 * G = K / group_size; group_size >= 1 divides K.  qweight: uint32 [N][K/8];
 * qzeros: uint32 [N][ceil(G/8)].  All 4-byte aligned (q 8-byte aligned).
 * A code > 15 is masked to its low nibble and flagged in the device status
 * word as BQ_ERR_INVALID_ARG.
 */
bq_status bq_weight_pack_int4_grouped(const uint8_t *q, const uint8_t *zeros, int64_t N, int64_t K,
                                      int64_t group_size, uint32_t *qweight, uint32_t *qzeros,
                                      bq_stream_t stream);

/*
 * Per-token W8A8 matmul with a fused dequantizing epilogue.
 * Source: "Per-token Quantization for Matmul" (Huawei CANN ATB), Input and
 * Output tables and the Example (acc * deqScale[n] * perTokenScale[m]).
 *
 *   acc[m,n] = sum_k x[m,k] * w(k,n)   (exact int32; K <= 131071)
 *   out[m,n] = (float(acc) * deq_scale[n]) * per_token_scale[m] (+ bias[n])
 *
 * x: int8 [M][ldx].  w: int8 [N][ldw] (BQ_W_NK) or [K][ldw] (BQ_W_KN).
 * deq_scale: fp32 [N], 32-byte aligned (as the ATB page requires).
 * per_token_scale: fp32 [M].  bias: fp32 [N] or NULL.  out: out_dtype
 * (BQ_BF16, BQ_F16 or BQ_F32) [M][ldo], computed in fp32 and rounded once.
 * Runs on the tcgen05 tensor cores; M, N and K tails are handled.
 */
bq_status bq_gemm_i8_pertoken(const int8_t *x, int64_t ldx, const int8_t *w, bq_wlayout w_layout,
                              int64_t ldw, const float *deq_scale, const float *per_token_scale,
                              const float *bias, int64_t M, int64_t N, int64_t K, bq_dtype out_dtype,
                              void *out, int64_t ldo, bq_stream_t stream);

/*
 * Batched and transposed forms of the per-token W8A8 matmul.
 * Source: "Per-token Quantization for Matmul" (Huawei CANN ATB), Parameters
 * (transposeA, transposeB) and Input / Output tables (x [batch,m,k],
 * weight [batch,k,n], output [batch,m,n]).
 *
 * For every b in [0, batch):
 *   acc[b,m,n] = sum_k x(b,m,k) * w(b,k,n)             (exact int32)
 *   out[b,m,n] = (float(acc) * deq_scale[b*stride_deq + n])
 *                * per_token_scale[b*stride_pts + m]  (+ bias[n])
 * x(b,m,k) = x[b*stride_x + m*ldx + k]  (trans_a = 0: [batch][M][ldx])
 *          = x[b*stride_x + k*ldx + m]  (trans_a = 1: [batch][K][ldx], M contiguous)
 * w(b,k,n) as in bq_gemm_i8_pertoken at w + b*stride_w.  out: out_dtype
 * [batch][M][ldo] at out + b*stride_out.  Strides count elements.
 * stride_deq = stride_pts = 0 shares one deq_scale [N] and one
 * per_token_scale [M] among all batches (the tables' [n] and [m]); N and M
 * give each batch its own.  bias [N] (or NULL) is shared.  With batch > 1:
 * stride_x >= rows(x) * ldx, stride_w >= rows(w) * ldw, stride_out >= M * ldo,
 * each a multiple of 16 bytes, and stride_deq * 4 a multiple of 32.  The
 * alignment rules of bq_gemm_i8_pertoken hold for each batch.  All batches
 * run in one launch (the tile schedule spans them); transposeA runs on
 * single-CTA tiles.  bq_gemm_i8_pertoken is this call with batch = 1.
 */
bq_status bq_gemm_i8_pertoken_batched(const int8_t *x, int64_t ldx, int64_t stride_x, int trans_a,
                                      const int8_t *w, bq_wlayout w_layout, int64_t ldw, int64_t stride_w,
                                      const float *deq_scale, int64_t stride_deq,
                                      const float *per_token_scale, int64_t stride_pts, const float *bias,
                                      int64_t batch, int64_t M, int64_t N, int64_t K, bq_dtype out_dtype,
                                      void *out, int64_t ldo, int64_t stride_out, bq_stream_t stream);

/*
 * BitLinear forward with ternary weights and int8 activations (W1.58A8).
 * Source: "Class BitLinear" (LLaMA-BitNet utils.py), forward steps 1-5.
 *
 *   (xq, act_scale, rowsum) = bq_act_quant_int8(x)   into the workspace
 *   acc[m,n] = sum_k xq[m,k] * w_q[n,k]              (exact int32)
 *   out[m,n] = (float(acc) * act_scale[m]) * gamma  (+ bias[n])
 *
 * x: dense [M][K] of x_dtype BQ_F32 or BQ_BF16; K % 16 == 0, any N.
 * wpacked, w_scale: as written by bq_weight_quant_ternary_pack.  bias: fp32
 * [N] or NULL (the page disables it by default).  out: dense [M][N] of
 * out_dtype.  M <= 16 runs a bandwidth-bound decode kernel, larger M the
 * tcgen05 GEMM that unpacks the 2-bit tiles in shared memory (for K % 64 != 0
 * it first copies the packed rows to a 16-byte pitch in the workspace, and
 * for N * size(out) % 16 != 0 it stages the output rows there and copies
 * them out; bq_bitlinear_w2a8_path() tells which kernels a shape runs).
 * workspace: at least bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8, M, N, K, 0)
 * bytes, 256-byte aligned; bq_bitlinear_workspace_layout() gives where
 * xq [M][K] int8, act_scale fp32 [M] and rowsum int32 [M] sit, so they can
 * be read back.
 */
bq_status bq_bitlinear_w2a8(const void *x, bq_dtype x_dtype, int64_t M, int64_t K,
                            const uint32_t *wpacked, const float *w_scale, int64_t N,
                            const float *bias, float eps, bq_dtype out_dtype, void *out,
                            void *workspace, size_t workspace_bytes, bq_stream_t stream);

/*
 * Per-token int8 activation quantization after a LayerNorm (the normaliser of
 * BitLinear and BitConv1d in "Common Attention Utilities", frankenstein-
 * transformer: "Applies LayerNorm to inputs before quantization"):
 *
 *   mu[m] = mean_k x[m,k],  var[m] = mean_k (x[m,k] - mu[m])^2
 *   y[m,k] = (x[m,k] - mu[m]) / sqrt(var[m] + eps) * g[k] + b[k]
 *   a[m] = max(max_k |y[m,k]|, 1e-5),  xq = clamp(rne(y * 127 / a), -128, 127)
 *   act_scale[m] = a[m] / 127,  rowsum[m] = sum_k xq[m,k]
 *
 * ln_weight (g) and ln_bias (b): fp32 [K] each, 4-byte aligned, or NULL for
 * g = 1 / b = 0 (a parameter-free LayerNorm).  The mean and variance are taken
 * in binary64 (the mean subtraction cancels); y in binary64 or, for at least
 * eight aligned rows, in fp32 with the row constants split into two fp32 parts
 * under a per-row error check (rows that fail it take binary64), so every code
 * agrees with the binary64 one except within 1e-6 (relative) of a rounding
 * tie.  Other arguments and rules as bq_act_quant_int8.
 */
bq_status bq_act_quant_int8_layernorm(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, int64_t ldx,
                                      const float *ln_weight, const float *ln_bias, float eps, int8_t *xq,
                                      int64_t ldq, float *act_scale, int32_t *rowsum, bq_stream_t stream);

/*
 * BitLinear forward with the LayerNorm normaliser ("Common Attention
 * Utilities", BitLinear: LayerNorm, 8-bit per-token activations, absmean
 * ternary weights, rescale): bq_act_quant_int8_layernorm into the workspace,
 * then the ternary linear and rescale of bq_bitlinear_w2a8
 * (out = (float(acc) * act_scale[m]) * gamma (+ bias[n])) on the mma.sync
 * weight-streaming kernel or the split GEMV kernel (M <= 16) or the tcgen05
 * GEMM (M > 16); one token with K in {2048, 4096, 8192} (fp32: up to 4096),
 * a 16-byte aligned x and at most 5120 * 64 / K weight rows per SM (N up to
 * 11840 at K = 4096 on 148 SMs) runs the normaliser inside the
 * weight-streaming kernel, one launch, which also writes the codes, act_scale
 * and rowsum to the workspace.  Arguments, workspace
 * (bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8, M, N, K, 0) and its layout) and
 * rules as bq_bitlinear_w2a8, plus ln_weight / ln_bias as above.
 */
bq_status bq_bitlinear_w2a8_layernorm(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const float *ln_weight,
                                      const float *ln_bias, const uint32_t *wpacked, const float *w_scale, int64_t N,
                                      const float *bias, float eps, bq_dtype out_dtype, void *out, void *workspace,
                                      size_t workspace_bytes, bq_stream_t stream);

/*
 * Backward of the BitLinear forward under the straight-through estimator.
 * Source: "Class BitLinear" (LLaMA-BitNet utils.py), forward steps 2-3
 * ("Quantise ... (STE)"); "Common Attention Utilities", activation_quant and
 * weight_quant (the STE "passes gradients through the rounding operation
 * unchanged").  With the forward's xq, act_scale (recomputed from x) and the
 * ternary codes wq with scale gamma:
 *
 *   dw[n,k] = sum_m dout[m,n] * act_scale[m] * xq[m,k]
 *   dy[m,k] = gamma * sum_n dout[m,n] * wq[n,k]
 *   dx[m,k] = (dy[m,k] - y[m,k] * mean_j(dy[m,j] * y[m,j])) / r[m],
 *   y = x / r, r = sqrt(mean(x^2) + eps)   (the parameter-free RMSNorm's backward)
 *
 * x: dense [M][K] fp32 or bf16; dout: dense bf16 [M][N] (the incoming
 * gradient); wpacked, w_scale as bq_bitlinear_w2a8; K % 16 == 0, N % 8 == 0.
 * dx: fp32 [M][K]; dw: fp32 [N][K] (the gradient of the master weight).  The
 * contractions run on the bf16 tensor cores (tcgen05 kind::f16, fp32
 * accumulation): dout and the codes are exact in bf16, and the products
 * dout * act_scale of dw are split into two bf16 parts (16 significant bits).
 * workspace: bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8_BACKWARD, M, N, K, 0)
 * bytes, 256-byte aligned.  M == 0 or N == 0: the gradients that exist are
 * written as zeros (dw when M == 0, dx when N == 0) and nothing else runs.
 */
bq_status bq_bitlinear_w2a8_backward(const void *x, bq_dtype x_dtype, const void *dout, int64_t M, int64_t K,
                                     const uint32_t *wpacked, const float *w_scale, int64_t N, float eps, float *dx,
                                     float *dw, void *workspace, size_t workspace_bytes, bq_stream_t stream);

/*
 * Which kernels bq_bitlinear_w2a8 runs for a shape on the current device (for
 * tests and profiling; the choice depends on M, N, K, the activation dtype,
 * the 16-byte alignment of x and the device's SM count).  *path receives a
 * bq_bitlinear_path.  Needs an sm_100 device (else BQ_ERR_UNSUPPORTED).
 */
typedef enum {
    BQ_PATH_DECODE_STREAM = 1,  /* 1 token: activation quant fused, dp4a register-streaming kernel    */
    BQ_PATH_DECODE_MMA = 2,     /* 2..16 tokens, K 2048/4096: fused, mma.sync register-streaming      */
    BQ_PATH_DECODE_SMEM = 3,    /* other M <= 16 with K % 512 == 0: fused, shared-memory staged kernel */
    BQ_PATH_ACT_QUANT_GEMV = 4, /* other M <= 16: activation-quant kernel, then a split GEMV kernel    */
    BQ_PATH_TC_SINGLE = 5,      /* M > 16: activation quant, tcgen05 GEMM on single CTAs               */
    BQ_PATH_TC_PAIR = 6         /* M > 16: activation quant, tcgen05 GEMM on CTA pairs (cta_group::2)  */
} bq_bitlinear_path;
bq_status bq_bitlinear_w2a8_path(const void *x, bq_dtype x_dtype, int64_t M, int64_t N, int64_t K, int *path);

/*
 * Grouped affine INT4 linear with fp32 activations.
 * Source: "vyre_libs/nn/linear/inner/linear_4bit/mod.rs", module doc (fused
 * unpack-on-demand; grouped affine path with scale and zero-point per group)
 * and the grouped output drift tolerance constant.
 *
 *   out[m,n] = bias[n] + sum_k x[m,k] * scale[n,g] * (q[n,k] - zero[n,g])
 *
 * x: dense fp32 [M][K], K % 8 == 0, group_size % 8 == 0 and divides K.
 * qweight, scales_f16, qzeros: as in "Data formats".  bias: fp32 [N] or NULL.
 * out: dense fp32 [M][N].  Internally x is split per (token, group) into a
 * 24-bit fixed-point value held as three byte planes so that the inner
 * products are exact integer dot products; the representation error is below
 * 1e-6 of the group's absolute maximum.  workspace: at least
 * bq_workspace_bytes(BQ_OP_LINEAR_W4_GROUPED, M, N, K, group_size) bytes,
 * 256-byte aligned.
 */
bq_status bq_linear_w4_grouped(const float *x, int64_t M, int64_t K, const uint32_t *qweight,
                               const uint16_t *scales_f16, const uint32_t *qzeros,
                               const float *bias, int64_t N, int64_t group_size, float *out,
                               void *workspace, size_t workspace_bytes, bq_stream_t stream);

/*
 * 4-bit activations and 4-bit weights with given step sizes (W4A4).
 * Source: "bitorch_engine.layers.qlinear.nbit.cutlass.q4_layer.
 * Q4LinearFunction" (bitorch-engine), forward(x, weight, scale_a, scale_w,
 * eps, is_train): the inputs and the weights are quantized to 4 bits with the
 * given scale factors, eps avoids a division by zero, then the linear.
 *
 *   s_a = max(scale_a, eps),  s_w[n] = max(scale_w[per_channel ? n : 0], eps)
 *   xq[m,k] = clamp(rne(x[m,k] / s_a), -8, 7),  wq[n,k] = clamp(rne(w[n,k] / s_w[n]), -8, 7)
 *   out[m,n] = (float(sum_k xq * wq) * s_w[n]) * s_a (+ bias[n])
 *
 * Steps are device fp32 values (read by the kernels, no host round trip):
 * scale_a one value, scale_w one value or [N] (scale_w_per_channel = 1).
 * eps > 0.  Quotients are correctly rounded fp32 divisions rounded to
 * nearest even.  is_train only decides what a training framework keeps for
 * its backward; the forward result is the same.
 *
 * bq_weight_quant_int4_pack: w dense [N][K] fp32 or bf16 -> wpacked uint32
 * [N][K/8], eight signed (two's-complement) nibbles per word, element k of a
 * row in bits [4*(k%8), 4*(k%8)+3] of word k/8.  K % 8 == 0.
 * bq_act_quant_int4: x [M][ldx] fp32 or bf16 -> xq int8 [M][ldq] in [-8, 7].
 * bq_linear_w4a4: x dense [M][K] (K % 32 == 0, any N), wpacked as above
 * (16-byte aligned), bias fp32 [N] or NULL, out dense [M][N] of out_dtype.
 * The activation codes go to the workspace
 * (bq_workspace_bytes(BQ_OP_LINEAR_W4A4, M, N, K, 0) bytes, 256-byte aligned);
 * up to 16 tokens run a dp4a GEMV kernel, more run the tcgen05 kind::i8 GEMM
 * with the packed weights sign-extended to int8 in shared memory (no int8
 * copy of the weights in global memory).
 */
bq_status bq_weight_quant_int4_pack(const void *w, bq_dtype w_dtype, int64_t N, int64_t K, const float *scale_w,
                                    int scale_w_per_channel, float eps, uint32_t *wpacked, bq_stream_t stream);
bq_status bq_act_quant_int4(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, int64_t ldx, const float *scale_a,
                            float eps, int8_t *xq, int64_t ldq, bq_stream_t stream);
bq_status bq_linear_w4a4(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const float *scale_a,
                         const uint32_t *wpacked, const float *scale_w, int scale_w_per_channel, int64_t N,
                         const float *bias, float eps, bq_dtype out_dtype, void *out, void *workspace,
                         size_t workspace_bytes, bq_stream_t stream);

/*
 * Straight-through backward of the 4-bit activation and weight linear.
 * Source: "bitorch_engine.layers.qlinear.nbit.cutlass.q4_layer.
 * Q4LinearFunction", backward(output_gradient): gradients for the input, the
 * weight and the activation scale, adjusted by the quantization ranges; none
 * for scale_w and eps.  Read as rounding passed straight through inside the
 * clamp range of the unrounded quotient.  With the forward's s_a, s_w[n],
 * u = x / s_a, v = w / s_w[n], xq, wq (bq_linear_w4a4):
 *
 *   g[m,k]   = sum_n dout[m,n] * s_w[n] * wq[n,k]
 *   dx[m,k]  = g[m,k] where -8 <= u[m,k] <= 7, else 0
 *   dw[n,k]  = s_a * sum_m dout[m,n] * xq[m,k] where -8 <= v[n,k] <= 7, else 0
 *   dscale_a = sum_{m,k} g[m,k] * (inside ? xq[m,k] - u[m,k] : xq[m,k]),
 *              0 when scale_a < eps
 *
 * x: dense [M][K] fp32 or bf16; w: dense fp32 [N][K] (the master weights the
 * forward quantized); dout: dense bf16 [M][N]; scale_a: one fp32, scale_w: one
 * fp32 or [N] (scale_w_per_channel), both on the device; K % 16 == 0,
 * N % 8 == 0, eps > 0.  dx fp32 [M][K], dw fp32 [N][K], dscale_a one fp32, all
 * on the device (16-byte aligned; dscale_a 4-byte).  The quotients are the
 * forward's correctly rounded fp32 divisions.  The two contractions run on the
 * bf16 tensor cores (fp32 accumulation; codes and dout exact in bf16, per-channel
 * steps folded into dout as two bf16 parts, 16 significant bits); dscale_a is a
 * binary64 sum in a fixed order (deterministic).  M == 0 or N == 0: the
 * gradients are written as zeros.  workspace:
 * bq_workspace_bytes(BQ_OP_LINEAR_W4A4_BACKWARD, M, N, K, 0) bytes, 256-byte
 * aligned.
 */
bq_status bq_linear_w4a4_backward(const void *x, bq_dtype x_dtype, const float *w, const void *dout, int64_t M,
                                  int64_t K, int64_t N, const float *scale_a, const float *scale_w,
                                  int scale_w_per_channel, float eps, float *dx, float *dw, float *dscale_a,
                                  void *workspace, size_t workspace_bytes, bq_stream_t stream);

/*
 * Ternary Conv1d with LayerNorm-normalised 8-bit activations.
 * Source: "Common Attention Utilities" (frankenstein-transformer), BitConv1d:
 * the ternary weights and int8 activations of BitLinear, the input (B, C_in,
 * L) LayerNorm-normalised over the channel dimension before the activation
 * quantization, forward (B, C_in, L) -> (B, C_out, L_out) with kernel_size,
 * stride, padding and groups.
 *
 *   per position (b, p): LayerNorm over the C_in channels (optional affine
 *     ln_weight / ln_bias [C_in]), then bq_act_quant_int8_layernorm's codes
 *     xq[b,p,:] and act_scale[b,p];
 *   gamma, wq = absmean ternary quantization of all weights (bake rule);
 *   out[b,co,lo] = gamma * sum_t act_scale[b,p] * sum_c wq[co,c,t] * xq[b,p,g*Cg+c]
 *                  (+ bias[co]),  p = lo*stride + t - pad (padding adds nothing),
 *   Cg = C_in / groups, g = co / (C_out / groups),
 *   L_out = (L + 2*pad - KS) / stride + 1.
 * Each tap is an exact integer contraction over the group's channels, scaled
 * by the scale of the position it reads; the taps are summed in fp32 and the
 * result rounded once to out_dtype.
 *
 * bq_bitconv1d_weight_pack: w dense [C_out][Cg][KS] (the Conv1d weight) fp32
 * or bf16, Cg % 16 == 0 -> wpacked uint32 [KS][C_out][Cgp/16] (Cgp = Cg
 * rounded up to 64; per tap the 2-bit layout of bq_weight_quant_ternary_pack
 * along the channels, rows Cgp/16 words apart) and w_scale (one fp32 on the
 * device).  workspace: bq_bitconv1d_weight_pack_workspace_bytes().
 * bq_bitconv1d: x dense (B, C_in, L), C_in % 16 == 0, Cg % 16 == 0, groups
 * <= 1024 and, with groups > 1, (C_out / groups) % 4 == 0; out dense
 * (B, C_out, L_out).  Runs a
 * transpose to position-major rows, the binary64 LayerNorm quantization, per
 * tap a row gather and per group the tcgen05 ternary GEMM into fp32
 * partials, and a tap-sum / transpose kernel.  workspace:
 * bq_bitconv1d_workspace_bytes(), 256-byte aligned.
 */
size_t bq_bitconv1d_weight_pack_workspace_bytes(int64_t C_out, int64_t Cg, int64_t KS);
bq_status bq_bitconv1d_weight_pack(const void *w, bq_dtype w_dtype, int64_t C_out, int64_t Cg, int64_t KS,
                                   uint32_t *wpacked, float *w_scale, void *workspace, size_t workspace_bytes,
                                   bq_stream_t stream);
size_t bq_bitconv1d_workspace_bytes(int64_t B, int64_t C_in, int64_t L, int64_t C_out, int64_t KS, int64_t stride,
                                    int64_t pad, int64_t groups);
bq_status bq_bitconv1d(const void *x, bq_dtype x_dtype, int64_t B, int64_t C_in, int64_t L, const float *ln_weight,
                       const float *ln_bias, const uint32_t *wpacked, const float *w_scale, int64_t C_out, int64_t KS,
                       int64_t stride, int64_t pad, int64_t groups, const float *bias, float eps, bq_dtype out_dtype,
                       void *out, void *workspace, size_t workspace_bytes, bq_stream_t stream);

/*
 * BitLinear forward with the contract and results of bq_bitlinear_w2a8, for
 * callers that cannot allocate device memory or hand over a workspace: a
 * plugin or custom op whose host framework owns every device allocation and
 * forbids cudaMalloc, or a latency-critical decode loop where an allocation
 * would synchronize the device.  The pages have no counterpart of this entry
 * point.
 *
 * The caller passes inputs and outputs as for bq_bitlinear_w2a8, and the
 * arguments are checked in the same way and order, with the same results.
 * The scratch (int8 activations, per-token scales, row sums, and for more
 * than 16 tokens the re-pitched weights or staged outputs of ragged shapes)
 * lives in one static device array of BQ_NOALLOC_SCRATCH_BYTES bytes, which
 * every GPU that loads the library holds until the process exits.  A valid
 * call whose scratch would exceed it (bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8,
 * M, N, K, 0) > BQ_NOALLOC_SCRATCH_BYTES, i.e. M*K above about 2 MB) returns
 * BQ_ERR_WORKSPACE before launching anything.  The call never allocates (no
 * cudaMalloc / cudaFree, no allocating library routine).
 *
 * The first call on a device (and the first after its context was destroyed
 * and re-created) looks up the array's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any
 * stream capture.  All calls on a device share the array and it keeps the
 * last call's contents; each call writes all the scratch it reads, so nothing
 * needs clearing, but calls that overlap on the GPU (unordered streams) race
 * on it.
 */
#define BQ_NOALLOC_SCRATCH_BYTES (2u * 1024u * 1024u)
bq_status bq_bitlinear_w2a8_noalloc(const void *x, bq_dtype x_dtype, int64_t M, int64_t K,
                                    const uint32_t *wpacked, const float *w_scale, int64_t N,
                                    const float *bias, float eps, bq_dtype out_dtype, void *out,
                                    bq_stream_t stream);

/* Workspace bytes a call needs (0 for calls that need none). */
size_t bq_workspace_bytes(bq_op op, int64_t M, int64_t N, int64_t K, int64_t group_size);

/* Byte offsets of xq [M][K], act_scale [M] and rowsum [M] inside the
 * bq_bitlinear_w2a8 workspace. */
void bq_bitlinear_workspace_layout(int64_t M, int64_t K, size_t *xq_offset, size_t *act_scale_offset,
                                   size_t *rowsum_offset);

/* Static description of a status code. */
const char *bq_status_string(bq_status status);

/*
 * Synchronizes `stream`, then reads and clears the current device's status
 * word.  Returns BQ_OK or the first error a kernel recorded; *detail (may be
 * NULL) receives the raw word (bits 0-7 status, bits 8-31 the site).
 */
bq_status bq_device_status(bq_stream_t stream, uint32_t *detail);

/*
 * Failure-detection check (diagnostic; the pages have no counterpart).  Runs
 * the single-CTA W8A8 tensor-core GEMM kernel on one 128 x 256 tile:
 * x int8 [128][256], w int8 [256][256] (BQ_W_NK), deq_scale fp32 [256]
 * (32-byte aligned), per_token_scale fp32 [128], out bf16 [128][256], with
 * every bounded wait limited to wait_limit_ns (1e5 .. 2e9) and the producer
 * withholding the copies of the second K block.  The MMA issuer's and the
 * epilogue's waits on that block run out: the kernel records BQ_ERR_TIMEOUT
 * (site: MMA issuer 2 or epilogue 3) in the device status word, waits for
 * its own copies and MMAs in flight, frees its tensor memory and returns
 * within a few limits; no fault, no trap, the context stays usable.  `out`
 * is left partly unwritten.  Read the outcome with bq_device_status().
 */
bq_status bq_diag_gemm_withheld_arrival(const int8_t *x, const int8_t *w, const float *deq_scale,
                                        const float *per_token_scale, void *out_bf16, uint64_t wait_limit_ns,
                                        bq_stream_t stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int bq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
