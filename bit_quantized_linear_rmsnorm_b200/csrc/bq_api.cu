// C ABI of libbq (declared in include/bq.h): argument validation, workspace
// layout, device capability checks and the per-device status word.  Every
// check runs before anything is launched, so a rejected call has no effect.
#include <cmath>
#include <cstring>
#include <mutex>

#include "bq_common.cuh"
#include "bq_internal.h"

// Per-device status word written by kernels (first error wins).
__device__ uint32_t bq_dev_status_word = 0;

namespace bq {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DevInfo g_dev[kMaxDevices];

bq_status current_device(DevInfo *out) {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return BQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo &di = g_dev[d];
    if (di.device != d) {
        DevInfo n;
        n.device = d;
        if (cudaDeviceGetAttribute(&n.num_sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess ||
            cudaDeviceGetAttribute(&n.cc_major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess ||
            cudaDeviceGetAttribute(&n.cc_minor, cudaDevAttrComputeCapabilityMinor, d) != cudaSuccess)
            return BQ_ERR_CUDA;
        int smem = 0;
        if (cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess)
            return BQ_ERR_CUDA;
        n.max_smem_optin = static_cast<size_t>(smem);
        void *sym = nullptr;
        if (cudaGetSymbolAddress(&sym, bq_dev_status_word) != cudaSuccess) return BQ_ERR_CUDA;
        n.status = static_cast<uint32_t *>(sym);
        di = n;
    }
    *out = di;
    // The kernels are built for sm_100a only.
    if (di.cc_major != 10 || di.cc_minor != 0) return BQ_ERR_UNSUPPORTED;
    return BQ_OK;
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
inline int esize(bq_dtype t) { return t == BQ_F32 ? 4 : 2; }
inline bool act_dtype_ok(bq_dtype t) { return t == BQ_F32 || t == BQ_BF16; }
inline bool out_dtype_ok(bq_dtype t) { return t == BQ_F32 || t == BQ_BF16 || t == BQ_F16; }

constexpr int64_t kMaxK = 131071;          // keeps |acc| <= 2^31 - 1 for int8 x int8
constexpr int64_t kMaxDim = 2147483647LL;  // tile indices are 32-bit
constexpr int64_t kMaxKW4 = 65536;         // activation planes staged in shared memory
constexpr int kGemvMaxM = 16;

void bitlinear_layout(int64_t M, int64_t K, size_t *xq, size_t *sc, size_t *rs, size_t *total) {
    *xq = 0;
    *sc = align256(static_cast<size_t>(M) * static_cast<size_t>(K));
    *rs = *sc + align256(static_cast<size_t>(M) * 4);
    *total = *rs + align256(static_cast<size_t>(M) * 4);
}

inline bq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA; }

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" {

int bq_version(void) { return 100; }

const char *bq_status_string(bq_status s) {
    switch (s) {
        case BQ_OK:
            return "ok";
        case BQ_ERR_INVALID_ARG:
            return "invalid argument";
        case BQ_ERR_UNSUPPORTED:
            return "unsupported (needs an sm_100 device or a supported shape)";
        case BQ_ERR_MISALIGNED:
            return "misaligned pointer or leading dimension";
        case BQ_ERR_WORKSPACE:
            return "workspace missing or too small";
        case BQ_ERR_CUDA:
            return "CUDA error";
        case BQ_ERR_TIMEOUT:
            return "a bounded device wait ran out";
    }
    return "unknown status";
}

size_t bq_workspace_bytes(bq_op op, int64_t M, int64_t N, int64_t K, int64_t group_size) {
    if (M < 0 || N < 0 || K < 0) return 0;
    switch (op) {
        case BQ_OP_WEIGHT_QUANT_TERNARY_PACK:
            return ternary_pack_workspace_bytes(N, K);
        case BQ_OP_BITLINEAR_W2A8: {
            size_t a, b, c, t;
            bitlinear_layout(M, K, &a, &b, &c, &t);
            return t;
        }
        case BQ_OP_LINEAR_W4_GROUPED:
            if (group_size <= 0) return 0;
            return linear_w4_workspace_bytes(M, N, K, group_size);
        default:
            return 0;
    }
}

void bq_bitlinear_workspace_layout(int64_t M, int64_t K, size_t *xq_offset, size_t *act_scale_offset,
                                   size_t *rowsum_offset) {
    size_t a, b, c, t;
    bitlinear_layout(M, K, &a, &b, &c, &t);
    if (xq_offset) *xq_offset = a;
    if (act_scale_offset) *act_scale_offset = b;
    if (rowsum_offset) *rowsum_offset = c;
}

bq_status bq_device_status(bq_stream_t stream, uint32_t *detail) {
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st == BQ_ERR_CUDA) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BQ_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, bq_dev_status_word, sizeof(v)) != cudaSuccess) return BQ_ERR_CUDA;
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(bq_dev_status_word, &zero, sizeof(zero)) != cudaSuccess) return BQ_ERR_CUDA;
    if (detail) *detail = v;
    return static_cast<bq_status>(v & 0xffu);
}

bq_status bq_act_quant_int8(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, int64_t ldx, float eps,
                            int8_t *xq, int64_t ldq, float *act_scale, int32_t *rowsum, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || M < 0 || K < 1 || ldx < K || ldq < K || !std::isfinite(eps) || eps < 0.0f)
        return BQ_ERR_INVALID_ARG;
    if (M > 0 && (x == nullptr || xq == nullptr || act_scale == nullptr)) return BQ_ERR_INVALID_ARG;
    if (M == 0) return BQ_OK;
    if (!aligned(x, esize(x_dtype)) || !aligned(xq, 16) || ldq % 16 != 0 || !aligned(act_scale, 4) ||
        !aligned(rowsum, 4))
        return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(launch_act_quant(x, x_dtype, M, K, ldx, eps, xq, ldq, act_scale, rowsum,
                                      static_cast<cudaStream_t>(stream), dev));
}

bq_status bq_weight_quant_ternary_pack(const void *w, bq_dtype w_dtype, int64_t N, int64_t K, uint32_t *wpacked,
                                       float *w_scale, void *workspace, size_t workspace_bytes,
                                       bq_stream_t stream) {
    if (!act_dtype_ok(w_dtype) || N < 0 || K < 1 || K % 16 != 0) return BQ_ERR_INVALID_ARG;
    if (N > 0 && (w == nullptr || wpacked == nullptr || w_scale == nullptr)) return BQ_ERR_INVALID_ARG;
    if (N == 0) return BQ_OK;
    if (!aligned(w, 16) || !aligned(wpacked, 16) || !aligned(w_scale, 4)) return BQ_ERR_MISALIGNED;
    const size_t need = ternary_pack_workspace_bytes(N, K);
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(
        launch_ternary_pack(w, w_dtype, N, K, wpacked, w_scale, workspace, static_cast<cudaStream_t>(stream), dev));
}

bq_status bq_weight_pack_int4_grouped(const uint8_t *q, const uint8_t *zeros, int64_t N, int64_t K,
                                      int64_t group_size, uint32_t *qweight, uint32_t *qzeros,
                                      bq_stream_t stream) {
    if (N < 0 || K < 1 || K % 8 != 0 || group_size < 1 || K % group_size != 0) return BQ_ERR_INVALID_ARG;
    if (N > 0 && (q == nullptr || zeros == nullptr || qweight == nullptr || qzeros == nullptr))
        return BQ_ERR_INVALID_ARG;
    if (N == 0) return BQ_OK;
    if (!aligned(q, 8) || !aligned(qweight, 4) || !aligned(qzeros, 4)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(launch_int4_pack(q, zeros, N, K, group_size, qweight, qzeros, static_cast<cudaStream_t>(stream),
                                      dev));
}

bq_status bq_gemm_i8_pertoken(const int8_t *x, int64_t ldx, const int8_t *w, bq_wlayout w_layout, int64_t ldw,
                              const float *deq_scale, const float *per_token_scale, const float *bias, int64_t M,
                              int64_t N, int64_t K, bq_dtype out_dtype, void *out, int64_t ldo,
                              bq_stream_t stream) {
    if (M < 0 || N < 0 || K < 1 || K > kMaxK || M > kMaxDim || N > kMaxDim) return BQ_ERR_INVALID_ARG;
    if (w_layout != BQ_W_NK && w_layout != BQ_W_KN) return BQ_ERR_INVALID_ARG;
    if (!out_dtype_ok(out_dtype)) return BQ_ERR_INVALID_ARG;
    if (ldx < K || ldw < (w_layout == BQ_W_NK ? K : N) || ldo < N) return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BQ_OK;
    if (x == nullptr || w == nullptr || deq_scale == nullptr || per_token_scale == nullptr || out == nullptr)
        return BQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(out, 16) || ldx % 16 != 0 || ldw % 16 != 0 ||
        (ldo * esize(out_dtype)) % 16 != 0 || !aligned(deq_scale, 32) || !aligned(per_token_scale, 4) ||
        !aligned(bias, 4))
        return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    GemmArgs g;
    g.a = x;
    g.lda = ldx;
    g.b = w;
    g.ldb = ldw;
    g.b_layout = w_layout;
    g.colscale = deq_scale;
    g.rowscale = per_token_scale;
    g.bias = bias;
    g.M = M;
    g.N = N;
    g.K = K;
    g.out_dtype = out_dtype;
    g.out = out;
    g.ldo = ldo;
    return launch_gemm_tc(g, static_cast<cudaStream_t>(stream), dev);
}

bq_status bq_bitlinear_w2a8(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const uint32_t *wpacked,
                            const float *w_scale, int64_t N, const float *bias, float eps, bq_dtype out_dtype,
                            void *out, void *workspace, size_t workspace_bytes, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || !out_dtype_ok(out_dtype) || M < 0 || N < 0 || K < 1 || K > kMaxK ||
        K % 16 != 0 || M > kMaxDim || N > kMaxDim || !std::isfinite(eps) || eps < 0.0f)
        return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BQ_OK;
    if (x == nullptr || wpacked == nullptr || w_scale == nullptr || out == nullptr) return BQ_ERR_INVALID_ARG;
    size_t xq_off, sc_off, rs_off, need;
    bitlinear_layout(M, K, &xq_off, &sc_off, &rs_off, &need);
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256) || !aligned(x, esize(x_dtype)) || !aligned(wpacked, 16) || !aligned(out, 16) ||
        !aligned(w_scale, 4) || !aligned(bias, 4))
        return BQ_ERR_MISALIGNED;
    const bool gemm_path = M > kGemvMaxM;
    // the tensor-core path stores rows of out and loads packed rows with TMA
    if (gemm_path && ((N * esize(out_dtype)) % 16 != 0 || K % 64 != 0)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + xq_off);
    float *act_scale = reinterpret_cast<float *>(ws + sc_off);
    int32_t *rowsum = reinterpret_cast<int32_t *>(ws + rs_off);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!gemm_path && decode_w2a8_supported(x, M, N, K, dev))
        return from_cuda(launch_decode_w2a8(x, x_dtype, M, K, eps, wpacked, w_scale, bias, N, out_dtype, out, xq,
                                            act_scale, rowsum, s, dev));
    cudaError_t e = launch_act_quant(x, x_dtype, M, K, K, eps, xq, K, act_scale, rowsum, s, dev);
    if (e != cudaSuccess) return BQ_ERR_CUDA;
    if (!gemm_path)
        return from_cuda(
            launch_gemv_w2a8(xq, K, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out_dtype, out, s, dev));
    GemmArgs g;
    g.a = xq;
    g.lda = K;
    g.b = wpacked;
    g.ldb = K / 16;
    g.b_packed2 = true;
    g.colscale = w_scale;
    g.rowscale = act_scale;
    g.rowcorr = rowsum;
    g.bias = bias;
    g.M = M;
    g.N = N;
    g.K = K;
    g.out_dtype = out_dtype;
    g.out = out;
    g.ldo = N;
    return launch_gemm_tc(g, s, dev);
}

bq_status bq_linear_w4_grouped(const float *x, int64_t M, int64_t K, const uint32_t *qweight,
                               const uint16_t *scales_f16, const uint32_t *qzeros, const float *bias, int64_t N,
                               int64_t group_size, float *out, void *workspace, size_t workspace_bytes,
                               bq_stream_t stream) {
    if (M < 0 || N < 0 || K < 1 || K % 8 != 0 || K > kMaxKW4 || group_size < 8 || group_size % 8 != 0 ||
        K % group_size != 0 || N > kMaxDim)
        return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BQ_OK;
    if (x == nullptr || qweight == nullptr || scales_f16 == nullptr || qzeros == nullptr || out == nullptr)
        return BQ_ERR_INVALID_ARG;
    const size_t need = linear_w4_workspace_bytes(M, N, K, group_size);
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256) || !aligned(x, 4) || !aligned(qweight, 4) || !aligned(scales_f16, 2) ||
        !aligned(qzeros, 4) || !aligned(bias, 4) || !aligned(out, 4))
        return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(launch_linear_w4(x, M, K, qweight, scales_f16, qzeros, bias, N, group_size, out, workspace,
                                      static_cast<cudaStream_t>(stream), dev));
}

}  // extern "C"
