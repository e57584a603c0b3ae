// Host-side launch entry points of the kernel files, called by bq_api.cu after
// argument validation.  Each returns the launch's cudaError_t (or a bq_status
// where the launch itself can fail validation, e.g. tensor-map encoding).
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/bq.h"

namespace bq {

constexpr int kMaxDevices = 64;

struct DevInfo {
    int device = -1;
    uint64_t ctx = 0;            // identity of the device's current context (never 0 once known)
    int num_sms = 0;
    int cc_major = 0, cc_minor = 0;
    size_t max_smem_optin = 0;
    uint32_t *status = nullptr;  // device address of the status word
};

// Identity of the calling thread's current CUDA context (its driver-assigned
// unique id, + 1 so that it is never 0); 1 when no context is current or the
// driver entry points are unavailable.  Per-device state that a context owns
// (symbol addresses, kernel attributes) is cached against this value, so a
// context destroyed and re-created (cudaDeviceReset) is noticed.
uint64_t current_context_id();

// Opt-in to `bytes` of dynamic shared memory for kernel `kern`, once per
// context and only when it grows (the attribute belongs to the context).
struct SmemOptIn {
    std::mutex mu;
    uint64_t ctx[kMaxDevices] = {};
    size_t bytes[kMaxDevices] = {};
};
inline cudaError_t smem_opt_in(SmemOptIn &c, const DevInfo &dev, const void *kern, size_t bytes) {
    std::lock_guard<std::mutex> lk(c.mu);
    const int d = dev.device;
    if (c.ctx[d] == dev.ctx && bytes <= c.bytes[d]) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e != cudaSuccess) return e;
    if (c.ctx[d] != dev.ctx) c.bytes[d] = 0;
    c.ctx[d] = dev.ctx;
    if (bytes > c.bytes[d]) c.bytes[d] = bytes;
    return cudaSuccess;
}

// The calling thread's current device, with its cached properties
// (refreshed when the device's context changes).  BQ_ERR_UNSUPPORTED unless
// it is an sm_100 device.
bq_status current_device(DevInfo *out);

// Every check of bq_bitlinear_w2a8 except the workspace ones; *empty is set
// for a valid call with M == 0 or N == 0 (nothing to launch).
bq_status bitlinear_check_args(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const uint32_t *wpacked,
                               const float *w_scale, int64_t N, const float *bias, float eps, bq_dtype out_dtype,
                               void *out, bool *empty);

cudaError_t launch_act_quant(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, float eps,
                             int8_t *xq, int64_t ldq, float *act_scale, int32_t *rowsum, cudaStream_t s,
                             const DevInfo &dev);

// LayerNorm (optional affine ln_weight / ln_bias [K]) + per-token int8
// quantization, in binary64 (act_quant_ln.cu).
cudaError_t launch_act_quant_ln(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *ln_weight,
                                const float *ln_bias, float eps, int8_t *xq, int64_t ldq, float *act_scale,
                                int32_t *rowsum, cudaStream_t s, const DevInfo &dev);

// Workspace of the ternary reduction (fp64 partial sums and extrema).
size_t ternary_pack_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_ternary_pack(const void *w, bq_dtype wt, int64_t N, int64_t K, uint32_t *wpacked,
                                float *w_scale, void *ws, cudaStream_t s, const DevInfo &dev);

cudaError_t launch_int4_pack(const uint8_t *q, const uint8_t *zeros, int64_t N, int64_t K, int64_t group_size,
                             uint32_t *qweight, uint32_t *qzeros, cudaStream_t s, const DevInfo &dev);

// Epilogue of the integer GEMMs:
//   W8A8, W4A4: out = (float(acc) * colscale[n]) * rowscale[m] (+ bias[n])
//   W2A8:       out = (float(acc - rowcorr[m]) * rowscale[m]) * (*colscale_scalar) (+ bias[n])
struct GemmArgs {
    const int8_t *a = nullptr;      // [M][lda] int8, K-major (or [K][lda], M-major, with a_mn)
    int64_t lda = 0;
    const void *b = nullptr;        // int8 [N][ldb] / [K][ldb], or packed u32 [N][ldb] (K * b_pack / 32 words)
    int64_t ldb = 0;                // elements (bytes for int8, words for packed)
    bq_wlayout b_layout = BQ_W_NK;
    int b_pack = 0;                 // 0: int8 B; 2: ternary offset-binary codes; 4: signed 4-bit codes
    const float *colscale = nullptr;  // [N] (W8A8) or one device scalar (W2A8)
    const float *rowscale = nullptr;  // [M]
    const int32_t *rowcorr = nullptr; // [M] (W2A8) or nullptr
    const float *bias = nullptr;      // [N] or nullptr
    int64_t M = 0, N = 0, K = 0;
    bq_dtype out_dtype = BQ_BF16;
    void *out = nullptr;
    int64_t ldo = 0;
    bool a_mn = false;              // A stored [K][lda], M contiguous (ATB transposeA = true)
    int64_t batch = 1;              // independent products of the same shape
    int64_t sa = 0, sb = 0, so = 0; // elements (words for packed B) between batches of a, b, out
    int64_t s_col = 0, s_row = 0;   // elements between batches of colscale / rowscale and rowcorr (0: shared)
    // (packed B, K-major A) rows of A per batch (0: M); output row m reads A row
    // m + a_row_off, and rows outside [0, a_rows) read as zeros
    int64_t a_rows = 0, a_row_off = 0;
    // launched as a programmatic dependent of the kernel just before it (the
    // kernel's producer and epilogue wait for it before reading anything)
    bool pdl = false;
    uint64_t wait_ns = 2000000000ull;  // limit of the kernel's bounded waits
    int withhold_kb = -1;              // failure-detection check only (single-CTA kernel)
};
bq_status launch_gemm_tc(const GemmArgs &g, cudaStream_t s, const DevInfo &dev);
// Whether launch_gemm_tc runs a product of this shape on CTA pairs.
bool gemm_uses_pair(bool packed, bq_wlayout b_layout, int64_t M, int64_t N, const DevInfo &dev, int64_t batch = 1);

// Decode path (M <= 16) of the ternary linear: reads the packed weights once.
cudaError_t launch_gemv_w2a8(const int8_t *xq, int64_t ldq, const float *act_scale, const int32_t *rowsum,
                             const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t M,
                             int64_t N, int64_t K, bq_dtype out_dtype, void *out, cudaStream_t s,
                             const DevInfo &dev);

// Fused single-launch decode path (M <= 16) of the ternary linear: per-CTA
// activation quantization + bulk-streamed packed weights.  Writes xq,
// act_scale and rowsum to the workspace as well.
bool decode_w2a8_supported(const void *x, int64_t M, int64_t N, int64_t K, const DevInfo &dev);
// Which decode kernel launch_decode_w2a8 runs for a supported shape
// (BQ_PATH_DECODE_STREAM, BQ_PATH_DECODE_MMA or BQ_PATH_DECODE_SMEM).
int decode_w2a8_kind(int64_t M, int64_t N, int64_t K, bq_dtype xt, const DevInfo &dev);
// The weight-streaming half of the 2..16-token decode path on codes already in
// global memory (written by a kernel launched just before it that waits for
// its own predecessors before it releases its dependents, as every quantizer
// of this library does).  1..16 tokens, K 2048 or 4096.
bool decode_mma_from_codes_supported(int64_t M, int64_t N, int64_t K, const DevInfo &dev);
cudaError_t launch_decode_mma_from_codes(const int8_t *xq, const float *act_scale, const int32_t *rowsum, int64_t M,
                                         int64_t K, const uint32_t *wpacked, const float *w_scale, const float *bias,
                                         int64_t N, bq_dtype out_dtype, void *out, cudaStream_t s,
                                         const DevInfo &dev);
cudaError_t launch_decode_w2a8(const void *x, bq_dtype xt, int64_t M, int64_t K, float eps, const uint32_t *wpacked,
                               const float *w_scale, const float *bias, int64_t N, bq_dtype out_dtype, void *out,
                               int8_t *ws_xq, float *ws_scale, int32_t *ws_rowsum, cudaStream_t s,
                               const DevInfo &dev);
// One-token BitLinear with the LayerNorm normaliser fused into the
// weight-streaming kernel (one launch; codes, act_scale and rowsum also go to
// the workspace, as in launch_decode_w2a8).
bool decode_ln1_supported(const void *x, int64_t M, int64_t N, int64_t K, bq_dtype xt, const DevInfo &dev);
cudaError_t launch_decode_ln1(const void *x, bq_dtype xt, int64_t K, const float *ln_w, const float *ln_b, float eps,
                              const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t N,
                              bq_dtype out_dtype, void *out, int8_t *ws_xq, float *ws_scale, int32_t *ws_rowsum,
                              cudaStream_t s, const DevInfo &dev);

// W4A4 (4-bit activations and weights with given steps, w4a4.cu).
cudaError_t launch_q4_weight_pack(const void *w, bq_dtype wt, int64_t N, int64_t K, const float *scale_w,
                                  int per_channel, float eps, uint32_t *wpacked, cudaStream_t s, const DevInfo &dev);
cudaError_t launch_q4_act_quant(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *scale_a,
                                float eps, int8_t *xq, int64_t ldq, float *row_step, const float *scale_w,
                                int per_channel, int64_t N, float *col_step, cudaStream_t s, const DevInfo &dev);
cudaError_t launch_w4a4_gemv(const int8_t *xq, int64_t M, int64_t K, const uint32_t *wpacked, const float *row_step,
                             const float *col_step, const float *bias, int64_t N, bq_dtype out_dtype, void *out,
                             cudaStream_t s, const DevInfo &dev);

// Ternary Conv1d (bitconv1d.cu): workspace layout, weight transpose to
// [KS][C_out * Cg], and the forward.
struct BitconvLayout {
    int64_t L_out = 0, ldp = 0;  // output length; row pitch of the fp32 tap partials
    size_t xt = 0, xq = 0, scale = 0, a = 0, rs = 0, rc = 0, part = 0, total = 0;
};
BitconvLayout bitconv_layout(int64_t B, int64_t C_in, int64_t L, int64_t C_out, int64_t KS, int64_t stride,
                             int64_t pad, int64_t groups);
cudaError_t launch_bitconv_weight_transpose(const void *w, bq_dtype wt, int64_t C_out, int64_t Cg, int64_t KS,
                                            void *dst, cudaStream_t s);
bq_status launch_bitconv1d(const void *x, bq_dtype xt, int64_t B, int64_t C_in, int64_t L, const float *ln_weight,
                           const float *ln_bias, const uint32_t *wpacked, const float *w_scale, int64_t C_out,
                           int64_t KS, int64_t stride, int64_t pad, int64_t groups, const float *bias, float eps,
                           bq_dtype out_dtype, void *out, void *workspace, cudaStream_t s, const DevInfo &dev);

// bf16 x bf16 -> fp32 tensor-core GEMM (gemm_bf16.cu):
//   out[m,n] = (*scale or 1) * sum_k A(m,k) * B(k,n)
// A [M][lda] K-major or [K][lda] M-major (a_mn); B [N][ldb] K-major or
// [K][ldb] N-major (b_mn); out fp32 [M][ldo].  lda, ldb % 8 == 0, ldo % 4 == 0.
struct Bf16Args {
    const void *a = nullptr;
    int64_t lda = 0;
    bool a_mn = false;
    const void *b = nullptr;
    int64_t ldb = 0;
    bool b_mn = false;
    int64_t M = 0, N = 0, K = 0;
    const float *scale = nullptr;
    float *out = nullptr;
    int64_t ldo = 0;
};
bq_status launch_gemm_bf16(const Bf16Args &g, cudaStream_t s, const DevInfo &dev);

// Straight-through backward of the W4A4 linear (w4a4.cu): workspace layout
// (epilogue steps, bf16 codes of x and of w (twice), the per-channel dout
// operand, g, the dscale_a partials) and the launch.
struct W4a4BwdLayout {
    size_t steps, xq, wq, a2, g, part, total;
};
W4a4BwdLayout w4a4_bwd_layout(int64_t M, int64_t N, int64_t K);
bq_status launch_w4a4_backward(const void *x, bq_dtype xt, const float *w, const void *dout, int64_t M, int64_t K,
                               int64_t N, const float *scale_a, const float *scale_w, int per_channel, float eps,
                               float *dx, float *dw, float *dscale_a, void *workspace, cudaStream_t s,
                               const DevInfo &dev);

// Straight-through backward of BitLinear (bitlinear_bwd.cu): workspace layout
// (xq, act_scale, bf16 ternary weights, the dW operands, dy) and the launch.
struct BwdLayout {
    size_t xq = 0, scale = 0, wt = 0, a2 = 0, b2 = 0, dy = 0, total = 0;
};
BwdLayout bitlinear_bwd_layout(int64_t M, int64_t N, int64_t K);
bq_status launch_bitlinear_backward(const void *x, bq_dtype xt, const void *dout, int64_t M, int64_t K,
                                    const uint32_t *wpacked, const float *w_scale, int64_t N, float eps, float *dx,
                                    float *dw, void *workspace, cudaStream_t s, const DevInfo &dev);

// Grouped INT4 linear.
size_t linear_w4_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group_size);
// Multi-token path on the tensor cores (2..32 tokens, K % 1024 == 0, groups of 128k).
bool w4_tc_supported(int64_t M, int64_t N, int64_t K, int64_t gs, const DevInfo &dev);
size_t w4_tc_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_w4_tc(const float *x, int64_t M, int64_t K, const uint32_t *qweight, const uint16_t *scales,
                         const uint32_t *qzeros, const float *bias, int64_t N, int64_t gs, float *out, void *ws,
                         cudaStream_t s, const DevInfo &dev);
cudaError_t launch_linear_w4(const float *x, int64_t M, int64_t K, const uint32_t *qweight,
                             const uint16_t *scales, const uint32_t *qzeros, const float *bias, int64_t N,
                             int64_t group_size, float *out, void *ws, cudaStream_t s, const DevInfo &dev);

}  // namespace bq
