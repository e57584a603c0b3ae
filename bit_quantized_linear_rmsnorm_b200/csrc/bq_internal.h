// Host-side launch entry points of the kernel files, called by bq_api.cu after
// argument validation.  Each returns the launch's cudaError_t (or a bq_status
// where the launch itself can fail validation, e.g. tensor-map encoding).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/bq.h"

namespace bq {

struct DevInfo {
    int device = -1;
    int num_sms = 0;
    int cc_major = 0, cc_minor = 0;
    size_t max_smem_optin = 0;
    uint32_t *status = nullptr;  // device address of the status word
};

cudaError_t launch_act_quant(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, float eps,
                             int8_t *xq, int64_t ldq, float *act_scale, int32_t *rowsum, cudaStream_t s,
                             const DevInfo &dev);

// Workspace of the ternary reduction (fp64 partial sums and extrema).
size_t ternary_pack_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_ternary_pack(const void *w, bq_dtype wt, int64_t N, int64_t K, uint32_t *wpacked,
                                float *w_scale, void *ws, cudaStream_t s, const DevInfo &dev);

cudaError_t launch_int4_pack(const uint8_t *q, const uint8_t *zeros, int64_t N, int64_t K, int64_t group_size,
                             uint32_t *qweight, uint32_t *qzeros, cudaStream_t s, const DevInfo &dev);

// Epilogue of the integer GEMMs:
//   W8A8: out = (float(acc) * colscale[n]) * rowscale[m] (+ bias[n])
//   W2A8: out = (float(acc - rowcorr[m]) * rowscale[m]) * (*colscale_scalar) (+ bias[n])
struct GemmArgs {
    const int8_t *a = nullptr;      // [M][lda] int8, K-major
    int64_t lda = 0;
    const void *b = nullptr;        // int8 [N][ldb] / [K][ldb], or packed 2-bit u32 [N][K/16]
    int64_t ldb = 0;                // elements (bytes for int8, words for packed)
    bq_wlayout b_layout = BQ_W_NK;
    bool b_packed2 = false;         // ternary offset-binary codes
    const float *colscale = nullptr;  // [N] (W8A8) or one device scalar (W2A8)
    const float *rowscale = nullptr;  // [M]
    const int32_t *rowcorr = nullptr; // [M] (W2A8) or nullptr
    const float *bias = nullptr;      // [N] or nullptr
    int64_t M = 0, N = 0, K = 0;
    bq_dtype out_dtype = BQ_BF16;
    void *out = nullptr;
    int64_t ldo = 0;
};
bq_status launch_gemm_tc(const GemmArgs &g, cudaStream_t s, const DevInfo &dev);

// Decode path (M <= 16) of the ternary linear: reads the packed weights once.
cudaError_t launch_gemv_w2a8(const int8_t *xq, int64_t ldq, const float *act_scale, const int32_t *rowsum,
                             const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t M,
                             int64_t N, int64_t K, bq_dtype out_dtype, void *out, cudaStream_t s,
                             const DevInfo &dev);

// Fused single-launch decode path (M <= 16) of the ternary linear: per-CTA
// activation quantization + bulk-streamed packed weights.  Writes xq,
// act_scale and rowsum to the workspace as well.
bool decode_w2a8_supported(const void *x, int64_t M, int64_t N, int64_t K, const DevInfo &dev);
cudaError_t launch_decode_w2a8(const void *x, bq_dtype xt, int64_t M, int64_t K, float eps, const uint32_t *wpacked,
                               const float *w_scale, const float *bias, int64_t N, bq_dtype out_dtype, void *out,
                               int8_t *ws_xq, float *ws_scale, int32_t *ws_rowsum, cudaStream_t s,
                               const DevInfo &dev);

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
