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

uint64_t current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 1;
    return static_cast<uint64_t>(id) + 2;
}

namespace {

std::mutex g_mu;
DevInfo g_dev[kMaxDevices];

}  // namespace

bq_status current_device(DevInfo *out) {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return BQ_ERR_CUDA;
    uint64_t ctx = current_context_id();
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo &di = g_dev[d];
    if (di.device != d || di.ctx != ctx) {
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
        // (the lookup makes the device's primary context current if it was not)
        void *sym = nullptr;
        if (cudaGetSymbolAddress(&sym, bq_dev_status_word) != cudaSuccess) return BQ_ERR_CUDA;
        n.status = static_cast<uint32_t *>(sym);
        n.ctx = ctx == 1 ? current_context_id() : ctx;
        di = n;
    }
    *out = di;
    // The kernels are built for sm_100a only.
    if (di.cc_major != 10 || di.cc_minor != 0) return BQ_ERR_UNSUPPORTED;
    return BQ_OK;
}

namespace {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
inline int esize(bq_dtype t) { return t == BQ_F32 ? 4 : 2; }
inline bool act_dtype_ok(bq_dtype t) { return t == BQ_F32 || t == BQ_BF16; }
inline bool out_dtype_ok(bq_dtype t) { return t == BQ_F32 || t == BQ_BF16 || t == BQ_F16; }

constexpr int64_t kMaxK = 131071;          // keeps |acc| <= 2^31 - 1 for int8 x int8
constexpr int64_t kMaxDim = 2147483647LL;  // tile indices are 32-bit
constexpr int64_t kMaxKW4 = 65536;         // activation planes staged in shared memory
constexpr int kGemvMaxM = 16;

// Workspace of bq_bitlinear_w2a8: xq [M][K], act_scale [M], rowsum [M]; for
// more than 16 tokens also, where the tensor-core path needs them, the packed
// weight rows re-pitched to a multiple of 64 codes (the tensor copy wants
// 16-byte row strides) and an output staging buffer with rows padded to 8
// elements of up to 4 bytes.
struct BitlinearLayout {
    size_t xq, scale, rowsum, wpad, opad, total;
};
// Workspace of bq_linear_w4a4: xq [M][K] int8, the per-row step [M] and the
// per-channel step [N] (fp32), and for more than 16 tokens with
// N * size(out) % 16 != 0 an output staging buffer (rows padded to 8 elements).
struct W4a4Layout {
    size_t xq, row, col, opad, total;
};
W4a4Layout w4a4_layout(int64_t M, int64_t N, int64_t K) {
    W4a4Layout l;
    l.xq = 0;
    l.row = align256(static_cast<size_t>(M) * static_cast<size_t>(K));
    l.col = l.row + align256(static_cast<size_t>(M) * 4);
    l.opad = l.col + align256(static_cast<size_t>(N) * 4);
    l.total = l.opad;
    if (M > kGemvMaxM && N % 8 != 0) l.total += align256(static_cast<size_t>(M) * static_cast<size_t>((N + 7) / 8 * 8) * 4);
    return l;
}

BitlinearLayout bitlinear_layout(int64_t M, int64_t N, int64_t K) {
    BitlinearLayout l;
    l.xq = 0;
    l.scale = align256(static_cast<size_t>(M) * static_cast<size_t>(K));
    l.rowsum = l.scale + align256(static_cast<size_t>(M) * 4);
    l.wpad = l.rowsum + align256(static_cast<size_t>(M) * 4);
    l.opad = l.wpad;
    if (M > kGemvMaxM && K % 64 != 0)
        l.opad += align256(static_cast<size_t>(N) * static_cast<size_t>((K + 63) / 64 * 4) * 4);
    l.total = l.opad;
    if (M > kGemvMaxM && N % 8 != 0) l.total += align256(static_cast<size_t>(M) * static_cast<size_t>((N + 7) / 8 * 8) * 4);
    return l;
}

inline bq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA; }

// Which kernels a BitLinear call of this shape runs (a bq_bitlinear_path).
int bitlinear_path(const void *x, bq_dtype x_dtype, int64_t M, int64_t N, int64_t K, const DevInfo &dev) {
    if (M > kGemvMaxM) return gemm_uses_pair(true, BQ_W_NK, M, N, dev) ? BQ_PATH_TC_PAIR : BQ_PATH_TC_SINGLE;
    if (decode_w2a8_supported(x, M, N, K, dev)) return decode_w2a8_kind(M, N, K, x_dtype, dev);
    return BQ_PATH_ACT_QUANT_GEMV;
}

}  // namespace

bq_status bitlinear_check_args(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const uint32_t *wpacked,
                               const float *w_scale, int64_t N, const float *bias, float eps, bq_dtype out_dtype,
                               void *out, bool *empty) {
    *empty = false;
    if (!act_dtype_ok(x_dtype) || !out_dtype_ok(out_dtype) || M < 0 || N < 0 || K < 1 || K > kMaxK ||
        K % 16 != 0 || M > kMaxDim || N > kMaxDim || !std::isfinite(eps) || eps < 0.0f)
        return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) {
        *empty = true;
        return BQ_OK;
    }
    if (x == nullptr || wpacked == nullptr || w_scale == nullptr || out == nullptr) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(wpacked, 16) || !aligned(out, 16) || !aligned(w_scale, 4) ||
        !aligned(bias, 4))
        return BQ_ERR_MISALIGNED;
    return BQ_OK;
}

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
        case BQ_OP_BITLINEAR_W2A8:
            return bitlinear_layout(M, N, K).total;
        case BQ_OP_LINEAR_W4_GROUPED:
            if (group_size <= 0) return 0;
            return linear_w4_workspace_bytes(M, N, K, group_size);
        case BQ_OP_LINEAR_W4A4:
            return w4a4_layout(M, N, K).total;
        case BQ_OP_BITLINEAR_W2A8_BACKWARD:
            return bitlinear_bwd_layout(M, N, K).total;
        case BQ_OP_LINEAR_W4A4_BACKWARD:
            return w4a4_bwd_layout(M, N, K).total;
        default:
            return 0;
    }
}

void bq_bitlinear_workspace_layout(int64_t M, int64_t K, size_t *xq_offset, size_t *act_scale_offset,
                                   size_t *rowsum_offset) {
    const BitlinearLayout l = bitlinear_layout(M, 0, K);
    if (xq_offset) *xq_offset = l.xq;
    if (act_scale_offset) *act_scale_offset = l.scale;
    if (rowsum_offset) *rowsum_offset = l.rowsum;
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

bq_status bq_gemm_i8_pertoken_batched(const int8_t *x, int64_t ldx, int64_t stride_x, int trans_a, const int8_t *w,
                                      bq_wlayout w_layout, int64_t ldw, int64_t stride_w, const float *deq_scale,
                                      int64_t stride_deq, const float *per_token_scale, int64_t stride_pts,
                                      const float *bias, int64_t batch, int64_t M, int64_t N, int64_t K,
                                      bq_dtype out_dtype, void *out, int64_t ldo, int64_t stride_out,
                                      bq_stream_t stream) {
    if (batch < 0 || M < 0 || N < 0 || K < 1 || K > kMaxK || M > kMaxDim || N > kMaxDim) return BQ_ERR_INVALID_ARG;
    if (trans_a != 0 && trans_a != 1) return BQ_ERR_INVALID_ARG;
    if (w_layout != BQ_W_NK && w_layout != BQ_W_KN) return BQ_ERR_INVALID_ARG;
    if (!out_dtype_ok(out_dtype)) return BQ_ERR_INVALID_ARG;
    const int64_t x_rows = trans_a ? K : M, x_cols = trans_a ? M : K;
    const int64_t w_rows = w_layout == BQ_W_NK ? N : K, w_cols = w_layout == BQ_W_NK ? K : N;
    if (ldx < x_cols || ldw < w_cols || ldo < N) return BQ_ERR_INVALID_ARG;
    if (batch > 1 && (stride_x < x_rows * ldx || stride_w < w_rows * ldw || stride_out < M * ldo ||
                      (stride_deq != 0 && stride_deq < N) || (stride_pts != 0 && stride_pts < M)))
        return BQ_ERR_INVALID_ARG;
    if (stride_deq < 0 || stride_pts < 0) return BQ_ERR_INVALID_ARG;
    if (batch == 0 || M == 0 || N == 0) return BQ_OK;
    // tile indices are 32-bit
    if (((M + 127) / 128) * ((N + 255) / 256) * batch > kMaxDim) return BQ_ERR_INVALID_ARG;
    if (x == nullptr || w == nullptr || deq_scale == nullptr || per_token_scale == nullptr || out == nullptr)
        return BQ_ERR_INVALID_ARG;
    const int esz = esize(out_dtype);
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(out, 16) || ldx % 16 != 0 || ldw % 16 != 0 ||
        (ldo * esz) % 16 != 0 || !aligned(deq_scale, 32) || !aligned(per_token_scale, 4) || !aligned(bias, 4))
        return BQ_ERR_MISALIGNED;
    if (batch > 1 && (stride_x % 16 != 0 || stride_w % 16 != 0 || (stride_out * esz) % 16 != 0 ||
                      (stride_deq * 4) % 32 != 0))
        return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    GemmArgs g;
    g.a = x;
    g.lda = ldx;
    g.a_mn = trans_a != 0;
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
    g.batch = batch;
    g.sa = batch > 1 ? stride_x : 0;
    g.sb = batch > 1 ? stride_w : 0;
    g.so = batch > 1 ? stride_out : 0;
    g.s_col = batch > 1 ? stride_deq : 0;
    g.s_row = batch > 1 ? stride_pts : 0;
    return launch_gemm_tc(g, static_cast<cudaStream_t>(stream), dev);
}

bq_status bq_gemm_i8_pertoken(const int8_t *x, int64_t ldx, const int8_t *w, bq_wlayout w_layout, int64_t ldw,
                              const float *deq_scale, const float *per_token_scale, const float *bias, int64_t M,
                              int64_t N, int64_t K, bq_dtype out_dtype, void *out, int64_t ldo,
                              bq_stream_t stream) {
    return bq_gemm_i8_pertoken_batched(x, ldx, 0, 0, w, w_layout, ldw, 0, deq_scale, 0, per_token_scale, 0, bias, 1,
                                       M, N, K, out_dtype, out, ldo, 0, stream);
}

// The ternary linear and rescale of a BitLinear call whose activations are
// already quantized into the workspace (xq [M][K], act_scale, rowsum).
static bq_status bitlinear_linear(int path, const BitlinearLayout &l, uint8_t *ws, int64_t M, int64_t K,
                                  const uint32_t *wpacked, const float *w_scale, int64_t N, const float *bias,
                                  bq_dtype out_dtype, void *out, cudaStream_t s, const DevInfo &dev) {
    const int8_t *xq = reinterpret_cast<const int8_t *>(ws + l.xq);
    const float *act_scale = reinterpret_cast<const float *>(ws + l.scale);
    const int32_t *rowsum = reinterpret_cast<const int32_t *>(ws + l.rowsum);
    if (path == BQ_PATH_ACT_QUANT_GEMV)
        return from_cuda(
            launch_gemv_w2a8(xq, K, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out_dtype, out, s, dev));
    // tensor-core path: its tensor copies need 16-byte row pitches, so packed
    // rows of K % 64 != 0 codes are re-pitched into the workspace first, and
    // output rows of N * size % 16 != 0 bytes are staged there and copied out
    const uint32_t *wrows = wpacked;
    int64_t ldb = K / 16;
    if (K % 64 != 0) {
        uint32_t *wpad = reinterpret_cast<uint32_t *>(ws + l.wpad);
        ldb = (K + 63) / 64 * 4;
        const cudaError_t e =
            cudaMemcpy2DAsync(wpad, static_cast<size_t>(ldb) * 4, wpacked, static_cast<size_t>(K / 16) * 4,
                              static_cast<size_t>(K / 16) * 4, static_cast<size_t>(N), cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return BQ_ERR_CUDA;
        wrows = wpad;
    }
    const bool stage_out = (N * esize(out_dtype)) % 16 != 0;
    GemmArgs g;
    g.a = xq;
    g.lda = K;
    g.b = wrows;
    g.ldb = ldb;
    g.b_pack = 2;
    g.colscale = w_scale;
    g.rowscale = act_scale;
    g.rowcorr = rowsum;
    g.bias = bias;
    g.pdl = K % 64 == 0;  // straight after the quantizer (no re-pitch copy in between)
    g.M = M;
    g.N = N;
    g.K = K;
    g.out_dtype = out_dtype;
    g.out = stage_out ? static_cast<void *>(ws + l.opad) : out;
    g.ldo = stage_out ? (N + 7) / 8 * 8 : N;
    const bq_status st = launch_gemm_tc(g, s, dev);
    if (st != BQ_OK || !stage_out) return st;
    const size_t row = static_cast<size_t>(N) * esize(out_dtype);
    return from_cuda(cudaMemcpy2DAsync(out, row, g.out, static_cast<size_t>(g.ldo) * esize(out_dtype), row,
                                       static_cast<size_t>(M), cudaMemcpyDeviceToDevice, s));
}

bq_status bq_bitlinear_w2a8(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const uint32_t *wpacked,
                            const float *w_scale, int64_t N, const float *bias, float eps, bq_dtype out_dtype,
                            void *out, void *workspace, size_t workspace_bytes, bq_stream_t stream) {
    bool empty = false;
    bq_status st = bitlinear_check_args(x, x_dtype, M, K, wpacked, w_scale, N, bias, eps, out_dtype, out, &empty);
    if (st != BQ_OK || empty) return st;
    const BitlinearLayout l = bitlinear_layout(M, N, K);
    if (workspace == nullptr || workspace_bytes < l.total) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    st = current_device(&dev);
    if (st != BQ_OK) return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + l.xq);
    float *act_scale = reinterpret_cast<float *>(ws + l.scale);
    int32_t *rowsum = reinterpret_cast<int32_t *>(ws + l.rowsum);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int path = bitlinear_path(x, x_dtype, M, N, K, dev);
    if (path == BQ_PATH_DECODE_STREAM || path == BQ_PATH_DECODE_MMA || path == BQ_PATH_DECODE_SMEM)
        return from_cuda(launch_decode_w2a8(x, x_dtype, M, K, eps, wpacked, w_scale, bias, N, out_dtype, out, xq,
                                            act_scale, rowsum, s, dev));
    if (launch_act_quant(x, x_dtype, M, K, K, eps, xq, K, act_scale, rowsum, s, dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    return bitlinear_linear(path, l, ws, M, K, wpacked, w_scale, N, bias, out_dtype, out, s, dev);
}

bq_status bq_act_quant_int8_layernorm(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, int64_t ldx,
                                      const float *ln_weight, const float *ln_bias, float eps, int8_t *xq,
                                      int64_t ldq, float *act_scale, int32_t *rowsum, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || M < 0 || K < 1 || ldx < K || ldq < K || !std::isfinite(eps) || eps < 0.0f)
        return BQ_ERR_INVALID_ARG;
    if (M > 0 && (x == nullptr || xq == nullptr || act_scale == nullptr)) return BQ_ERR_INVALID_ARG;
    if (M == 0) return BQ_OK;
    if (!aligned(x, esize(x_dtype)) || !aligned(xq, 16) || ldq % 16 != 0 || !aligned(act_scale, 4) ||
        !aligned(rowsum, 4) || !aligned(ln_weight, 4) || !aligned(ln_bias, 4))
        return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(launch_act_quant_ln(x, x_dtype, M, K, ldx, ln_weight, ln_bias, eps, xq, ldq, act_scale, rowsum,
                                         static_cast<cudaStream_t>(stream), dev));
}

bq_status bq_bitlinear_w2a8_layernorm(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const float *ln_weight,
                                      const float *ln_bias, const uint32_t *wpacked, const float *w_scale, int64_t N,
                                      const float *bias, float eps, bq_dtype out_dtype, void *out, void *workspace,
                                      size_t workspace_bytes, bq_stream_t stream) {
    bool empty = false;
    bq_status st = bitlinear_check_args(x, x_dtype, M, K, wpacked, w_scale, N, bias, eps, out_dtype, out, &empty);
    if (st != BQ_OK || empty) return st;
    if (!aligned(ln_weight, 4) || !aligned(ln_bias, 4)) return BQ_ERR_MISALIGNED;
    const BitlinearLayout l = bitlinear_layout(M, N, K);
    if (workspace == nullptr || workspace_bytes < l.total) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    st = current_device(&dev);
    if (st != BQ_OK) return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (decode_ln1_supported(x, M, N, K, x_dtype, dev))  // one token: normaliser fused into the weight stream
        return from_cuda(launch_decode_ln1(x, x_dtype, K, ln_weight, ln_bias, eps, wpacked, w_scale, bias, N, out_dtype,
                                           out, reinterpret_cast<int8_t *>(ws + l.xq),
                                           reinterpret_cast<float *>(ws + l.scale),
                                           reinterpret_cast<int32_t *>(ws + l.rowsum), s, dev));
    if (launch_act_quant_ln(x, x_dtype, M, K, K, ln_weight, ln_bias, eps, reinterpret_cast<int8_t *>(ws + l.xq), K,
                            reinterpret_cast<float *>(ws + l.scale), reinterpret_cast<int32_t *>(ws + l.rowsum), s,
                            dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (M <= kGemvMaxM && decode_mma_from_codes_supported(M, N, K, dev))
        return from_cuda(launch_decode_mma_from_codes(reinterpret_cast<int8_t *>(ws + l.xq),
                                                      reinterpret_cast<float *>(ws + l.scale),
                                                      reinterpret_cast<int32_t *>(ws + l.rowsum), M, K, wpacked,
                                                      w_scale, bias, N, out_dtype, out, s, dev));
    const int path = M > kGemvMaxM ? bitlinear_path(x, x_dtype, M, N, K, dev) : BQ_PATH_ACT_QUANT_GEMV;
    return bitlinear_linear(path, l, ws, M, K, wpacked, w_scale, N, bias, out_dtype, out, s, dev);
}

bq_status bq_bitlinear_w2a8_path(const void *x, bq_dtype x_dtype, int64_t M, int64_t N, int64_t K, int *path) {
    if (path == nullptr || !act_dtype_ok(x_dtype) || M < 1 || N < 1 || K < 1 || K % 16 != 0 || K > kMaxK ||
        M > kMaxDim || N > kMaxDim)
        return BQ_ERR_INVALID_ARG;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    *path = bitlinear_path(x, x_dtype, M, N, K, dev);
    return BQ_OK;
}

bq_status bq_diag_gemm_withheld_arrival(const int8_t *x, const int8_t *w, const float *deq_scale,
                                        const float *per_token_scale, void *out_bf16, uint64_t wait_limit_ns,
                                        bq_stream_t stream) {
    if (x == nullptr || w == nullptr || deq_scale == nullptr || per_token_scale == nullptr || out_bf16 == nullptr ||
        wait_limit_ns < 100000ull || wait_limit_ns > 2000000000ull)
        return BQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(out_bf16, 16) || !aligned(deq_scale, 32) ||
        !aligned(per_token_scale, 4))
        return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    // one 128 x 256 tile (a single CTA), two 128-wide K blocks: the second is withheld
    GemmArgs g;
    g.a = x;
    g.lda = 256;
    g.b = w;
    g.ldb = 256;
    g.colscale = deq_scale;
    g.rowscale = per_token_scale;
    g.M = 128;
    g.N = 256;
    g.K = 256;
    g.out_dtype = BQ_BF16;
    g.out = out_bf16;
    g.ldo = 256;
    g.wait_ns = wait_limit_ns;
    g.withhold_kb = 1;
    if (gemm_uses_pair(false, BQ_W_NK, g.M, g.N, dev)) return BQ_ERR_UNSUPPORTED;  // (a one-tile grid never pairs)
    return launch_gemm_tc(g, static_cast<cudaStream_t>(stream), dev);
}

bq_status bq_weight_quant_int4_pack(const void *w, bq_dtype w_dtype, int64_t N, int64_t K, const float *scale_w,
                                    int scale_w_per_channel, float eps, uint32_t *wpacked, bq_stream_t stream) {
    if (!act_dtype_ok(w_dtype) || N < 0 || K < 1 || K % 8 != 0 || !std::isfinite(eps) || eps <= 0.0f ||
        (scale_w_per_channel != 0 && scale_w_per_channel != 1))
        return BQ_ERR_INVALID_ARG;
    if (N == 0) return BQ_OK;
    if (w == nullptr || scale_w == nullptr || wpacked == nullptr) return BQ_ERR_INVALID_ARG;
    if (!aligned(w, esize(w_dtype)) || !aligned(scale_w, 4) || !aligned(wpacked, 4)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(launch_q4_weight_pack(w, w_dtype, N, K, scale_w, scale_w_per_channel, eps, wpacked,
                                           static_cast<cudaStream_t>(stream), dev));
}

bq_status bq_act_quant_int4(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, int64_t ldx, const float *scale_a,
                            float eps, int8_t *xq, int64_t ldq, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || M < 0 || K < 1 || ldx < K || ldq < K || !std::isfinite(eps) || eps <= 0.0f)
        return BQ_ERR_INVALID_ARG;
    if (M == 0) return BQ_OK;
    if (x == nullptr || scale_a == nullptr || xq == nullptr) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(scale_a, 4)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return from_cuda(launch_q4_act_quant(x, x_dtype, M, K, ldx, scale_a, eps, xq, ldq, nullptr, nullptr, 0, 0, nullptr,
                                         static_cast<cudaStream_t>(stream), dev));
}

bq_status bq_linear_w4a4(const void *x, bq_dtype x_dtype, int64_t M, int64_t K, const float *scale_a,
                         const uint32_t *wpacked, const float *scale_w, int scale_w_per_channel, int64_t N,
                         const float *bias, float eps, bq_dtype out_dtype, void *out, void *workspace,
                         size_t workspace_bytes, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || !out_dtype_ok(out_dtype) || M < 0 || N < 0 || K < 1 || K % 32 != 0 ||
        K > kMaxK || M > kMaxDim || N > kMaxDim || !std::isfinite(eps) || eps <= 0.0f ||
        (scale_w_per_channel != 0 && scale_w_per_channel != 1))
        return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BQ_OK;
    if (x == nullptr || scale_a == nullptr || wpacked == nullptr || scale_w == nullptr || out == nullptr)
        return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(scale_a, 4) || !aligned(wpacked, 16) || !aligned(scale_w, 4) ||
        !aligned(bias, 4) || !aligned(out, 16))
        return BQ_ERR_MISALIGNED;
    const W4a4Layout l = w4a4_layout(M, N, K);
    if (workspace == nullptr || workspace_bytes < l.total) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + l.xq);
    float *row_step = reinterpret_cast<float *>(ws + l.row);
    float *col_step = reinterpret_cast<float *>(ws + l.col);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_q4_act_quant(x, x_dtype, M, K, K, scale_a, eps, xq, K, row_step, scale_w, scale_w_per_channel, N,
                            col_step, s, dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (M <= kGemvMaxM)
        return from_cuda(launch_w4a4_gemv(xq, M, K, wpacked, row_step, col_step, bias, N, out_dtype, out, s, dev));
    const bool stage_out = (N * esize(out_dtype)) % 16 != 0;
    GemmArgs g;
    g.a = xq;
    g.lda = K;
    g.b = wpacked;
    g.ldb = K / 8;
    g.b_pack = 4;
    g.colscale = col_step;
    g.rowscale = row_step;
    g.bias = bias;
    g.pdl = true;  // straight after the quantizer
    g.M = M;
    g.N = N;
    g.K = K;
    g.out_dtype = out_dtype;
    g.out = stage_out ? static_cast<void *>(ws + l.opad) : out;
    g.ldo = stage_out ? (N + 7) / 8 * 8 : N;
    st = launch_gemm_tc(g, s, dev);
    if (st != BQ_OK || !stage_out) return st;
    const size_t row = static_cast<size_t>(N) * esize(out_dtype);
    return from_cuda(cudaMemcpy2DAsync(out, row, g.out, static_cast<size_t>(g.ldo) * esize(out_dtype), row,
                                       static_cast<size_t>(M), cudaMemcpyDeviceToDevice, s));
}

size_t bq_bitconv1d_weight_pack_workspace_bytes(int64_t C_out, int64_t Cg, int64_t KS) {
    if (C_out < 0 || Cg < 0 || KS < 0) return 0;
    const size_t n = static_cast<size_t>(C_out) * static_cast<size_t>(Cg) * static_cast<size_t>(KS);
    return align256(n * 4) + align256(ternary_pack_workspace_bytes(KS * C_out, Cg)) + align256(n / 4 + 16);
}

size_t bq_bitconv1d_workspace_bytes(int64_t B, int64_t C_in, int64_t L, int64_t C_out, int64_t KS, int64_t stride,
                                    int64_t pad, int64_t groups) {
    if (B < 0 || C_in < 1 || L < 1 || C_out < 1 || KS < 1 || stride < 1 || pad < 0 || groups < 1) return 0;
    if (L + 2 * pad < KS) return 0;
    return bitconv_layout(B, C_in, L, C_out, KS, stride, pad, groups).total;
}

bq_status bq_bitconv1d_weight_pack(const void *w, bq_dtype w_dtype, int64_t C_out, int64_t Cg, int64_t KS,
                                   uint32_t *wpacked, float *w_scale, void *workspace, size_t workspace_bytes,
                                   bq_stream_t stream) {
    if (!act_dtype_ok(w_dtype) || C_out < 0 || Cg < 16 || Cg % 16 != 0 || KS < 1) return BQ_ERR_INVALID_ARG;
    if (C_out == 0) return BQ_OK;
    if (w == nullptr || wpacked == nullptr || w_scale == nullptr) return BQ_ERR_INVALID_ARG;
    if (!aligned(w, esize(w_dtype)) || !aligned(wpacked, 16) || !aligned(w_scale, 4)) return BQ_ERR_MISALIGNED;
    const size_t need = bq_bitconv1d_weight_pack_workspace_bytes(C_out, Cg, KS);
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = static_cast<size_t>(C_out) * static_cast<size_t>(Cg) * static_cast<size_t>(KS);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *wt = ws;                                   // [KS][C_out][Cg] in the weight's dtype
    uint8_t *tws = ws + align256(n * 4);                // reduction partials of the ternary pack
    uint32_t *dense = reinterpret_cast<uint32_t *>(tws + align256(ternary_pack_workspace_bytes(KS * C_out, Cg)));
    if (launch_bitconv_weight_transpose(w, w_dtype, C_out, Cg, KS, wt, s) != cudaSuccess) return BQ_ERR_CUDA;
    const int64_t Cgp = (Cg + 63) / 64 * 64;
    uint32_t *dst = Cgp == Cg ? wpacked : dense;
    if (launch_ternary_pack(wt, w_dtype, KS * C_out, Cg, dst, w_scale, tws, s, dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (Cgp == Cg) return BQ_OK;
    return from_cuda(cudaMemcpy2DAsync(wpacked, static_cast<size_t>(Cgp / 16) * 4, dense,
                                       static_cast<size_t>(Cg / 16) * 4, static_cast<size_t>(Cg / 16) * 4,
                                       static_cast<size_t>(KS * C_out), cudaMemcpyDeviceToDevice, s));
}

bq_status bq_bitconv1d(const void *x, bq_dtype x_dtype, int64_t B, int64_t C_in, int64_t L, const float *ln_weight,
                       const float *ln_bias, const uint32_t *wpacked, const float *w_scale, int64_t C_out, int64_t KS,
                       int64_t stride, int64_t pad, int64_t groups, const float *bias, float eps, bq_dtype out_dtype,
                       void *out, void *workspace, size_t workspace_bytes, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || !out_dtype_ok(out_dtype) || B < 0 || C_in < 16 || L < 1 || C_out < 1 || KS < 1 ||
        stride < 1 || pad < 0 || groups < 1 || C_in % groups != 0 || C_out % groups != 0 || !std::isfinite(eps) ||
        eps < 0.0f || L + 2 * pad < KS)
        return BQ_ERR_INVALID_ARG;
    const int64_t Cg = C_in / groups, Cog = C_out / groups;
    if (C_in % 16 != 0 || Cg % 16 != 0 || Cg > kMaxK || (groups > 1 && Cog % 4 != 0) || groups > 1024)
        return BQ_ERR_INVALID_ARG;
    if (B * L > kMaxDim || B * ((L + 2 * pad - KS) / stride + 1) > kMaxDim) return BQ_ERR_INVALID_ARG;
    if (B == 0) return BQ_OK;
    if (x == nullptr || wpacked == nullptr || w_scale == nullptr || out == nullptr) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(wpacked, 16) || !aligned(w_scale, 4) || !aligned(bias, 4) ||
        !aligned(ln_weight, 4) || !aligned(ln_bias, 4) || !aligned(out, esize(out_dtype)))
        return BQ_ERR_MISALIGNED;
    const size_t need = bitconv_layout(B, C_in, L, C_out, KS, stride, pad, groups).total;
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return launch_bitconv1d(x, x_dtype, B, C_in, L, ln_weight, ln_bias, wpacked, w_scale, C_out, KS, stride, pad, groups,
                            bias, eps, out_dtype, out, workspace, static_cast<cudaStream_t>(stream), dev);
}

bq_status bq_bitlinear_w2a8_backward(const void *x, bq_dtype x_dtype, const void *dout, int64_t M, int64_t K,
                                     const uint32_t *wpacked, const float *w_scale, int64_t N, float eps, float *dx,
                                     float *dw, void *workspace, size_t workspace_bytes, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || M < 0 || N < 0 || K < 1 || K % 16 != 0 || N % 8 != 0 || K > kMaxK ||
        M > kMaxDim / 2 || N > kMaxDim || !std::isfinite(eps) || eps < 0.0f)
        return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) {  // the gradients that exist are zero
        if ((M > 0 && dx == nullptr) || (N > 0 && dw == nullptr)) return BQ_ERR_INVALID_ARG;
        const cudaStream_t s = static_cast<cudaStream_t>(stream);
        if (M > 0 && cudaMemsetAsync(dx, 0, static_cast<size_t>(M) * static_cast<size_t>(K) * 4, s) != cudaSuccess)
            return BQ_ERR_CUDA;
        if (N > 0 && cudaMemsetAsync(dw, 0, static_cast<size_t>(N) * static_cast<size_t>(K) * 4, s) != cudaSuccess)
            return BQ_ERR_CUDA;
        return BQ_OK;
    }
    if (x == nullptr || dout == nullptr || wpacked == nullptr || w_scale == nullptr || dx == nullptr || dw == nullptr)
        return BQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(dout, 16) || !aligned(wpacked, 16) || !aligned(w_scale, 4) || !aligned(dx, 16) ||
        !aligned(dw, 16))
        return BQ_ERR_MISALIGNED;
    const size_t need = bitlinear_bwd_layout(M, N, K).total;
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return launch_bitlinear_backward(x, x_dtype, dout, M, K, wpacked, w_scale, N, eps, dx, dw, workspace,
                                     static_cast<cudaStream_t>(stream), dev);
}

bq_status bq_linear_w4a4_backward(const void *x, bq_dtype x_dtype, const float *w, const void *dout, int64_t M,
                                  int64_t K, int64_t N, const float *scale_a, const float *scale_w,
                                  int scale_w_per_channel, float eps, float *dx, float *dw, float *dscale_a,
                                  void *workspace, size_t workspace_bytes, bq_stream_t stream) {
    if (!act_dtype_ok(x_dtype) || M < 0 || N < 0 || K < 1 || K % 16 != 0 || N % 8 != 0 || K > kMaxK ||
        M > kMaxDim || N > kMaxDim / 2 || !std::isfinite(eps) || eps <= 0.0f ||
        (scale_w_per_channel != 0 && scale_w_per_channel != 1))
        return BQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) {  // the gradients are zero
        if ((M > 0 && dx == nullptr) || (N > 0 && dw == nullptr) || dscale_a == nullptr) return BQ_ERR_INVALID_ARG;
        const cudaStream_t s = static_cast<cudaStream_t>(stream);
        if (M > 0 && cudaMemsetAsync(dx, 0, static_cast<size_t>(M) * static_cast<size_t>(K) * 4, s) != cudaSuccess)
            return BQ_ERR_CUDA;
        if (N > 0 && cudaMemsetAsync(dw, 0, static_cast<size_t>(N) * static_cast<size_t>(K) * 4, s) != cudaSuccess)
            return BQ_ERR_CUDA;
        if (cudaMemsetAsync(dscale_a, 0, 4, s) != cudaSuccess) return BQ_ERR_CUDA;
        return BQ_OK;
    }
    if (x == nullptr || w == nullptr || dout == nullptr || scale_a == nullptr || scale_w == nullptr || dx == nullptr ||
        dw == nullptr || dscale_a == nullptr)
        return BQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(dout, 16) || !aligned(scale_a, 4) || !aligned(scale_w, 4) ||
        !aligned(dx, 16) || !aligned(dw, 16) || !aligned(dscale_a, 4))
        return BQ_ERR_MISALIGNED;
    const size_t need = w4a4_bwd_layout(M, N, K).total;
    if (workspace == nullptr || workspace_bytes < need) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BQ_ERR_MISALIGNED;
    DevInfo dev;
    const bq_status st = current_device(&dev);
    if (st != BQ_OK) return st;
    return launch_w4a4_backward(x, x_dtype, w, dout, M, K, N, scale_a, scale_w, scale_w_per_channel, eps, dx, dw,
                                dscale_a, workspace, static_cast<cudaStream_t>(stream), dev);
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
