// bq_bitlinear_w2a8_noalloc: the BitLinear W2A8 forward for callers that may
// not allocate device memory and cannot hand over a workspace.
//
// Who needs it: code running inside a host framework that owns every device
// allocation (a plugin or custom op whose host forbids cudaMalloc after start
// up, or whose memory pool is fixed), and latency-critical decode loops where
// a cudaMalloc / cudaFree would synchronize the device.  Such callers still
// pass their inputs and outputs; the scratch that bq_bitlinear_w2a8 keeps in
// the caller's workspace (the int8 activations, their per-token scales and
// row sums) lives here instead, in one fixed-size array in device memory that
// every GPU loading the library holds until the process exits.
//
// The array is shared by every call on a device and keeps the last call's
// contents.  A call writes all the scratch it reads (the activation
// quantization fills xq, act_scale and rowsum before the linear kernel reads
// them), so nothing needs clearing; but two calls that overlap on the GPU
// (different streams, no ordering between them) race on the array.
#include <mutex>

#include "bq_internal.h"

namespace {

static __device__ __align__(256) uint8_t bq_noalloc_scratch[BQ_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
uint8_t *g_scratch[bq::kMaxDevices] = {};
uint64_t g_ctx[bq::kMaxDevices] = {};

// In host code `bq_noalloc_scratch` names a host-side stand-in, not device
// memory: the device address is looked up once per device context, with that
// device current, and cached against the context's identity.
bq_status scratch_of(const bq::DevInfo &dev, uint8_t **out) {
    std::lock_guard<std::mutex> lk(g_mu);
    const int d = dev.device;
    if (g_scratch[d] == nullptr || g_ctx[d] != dev.ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, bq_noalloc_scratch) != cudaSuccess || p == nullptr) return BQ_ERR_CUDA;
        g_scratch[d] = static_cast<uint8_t *>(p);
        g_ctx[d] = dev.ctx;
    }
    *out = g_scratch[d];
    return BQ_OK;
}

}  // namespace

extern "C" bq_status bq_bitlinear_w2a8_noalloc(const void *x, bq_dtype x_dtype, int64_t M, int64_t K,
                                               const uint32_t *wpacked, const float *w_scale, int64_t N,
                                               const float *bias, float eps, bq_dtype out_dtype, void *out,
                                               bq_stream_t stream) {
    // the same argument checks as bq_bitlinear_w2a8, before anything else
    bool empty = false;
    bq_status st = bq::bitlinear_check_args(x, x_dtype, M, K, wpacked, w_scale, N, bias, eps, out_dtype, out, &empty);
    if (st != BQ_OK || empty) return st;
    if (bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8, M, N, K, 0) > static_cast<size_t>(BQ_NOALLOC_SCRATCH_BYTES))
        return BQ_ERR_WORKSPACE;
    bq::DevInfo dev;
    st = bq::current_device(&dev);
    if (st != BQ_OK) return st;
    uint8_t *scratch = nullptr;
    st = scratch_of(dev, &scratch);
    if (st != BQ_OK) return st;
    return bq_bitlinear_w2a8(x, x_dtype, M, K, wpacked, w_scale, N, bias, eps, out_dtype, out, scratch,
                             static_cast<size_t>(BQ_NOALLOC_SCRATCH_BYTES), stream);
}
