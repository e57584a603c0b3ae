// Per-token int8 activation quantization after a LayerNorm: the normaliser of
// BitLinear and BitConv1d in "Common Attention Utilities" (frankenstein-
// transformer: "Applies LayerNorm to inputs before quantization"), followed by
// the same per-token absmax quantization as the RMSNorm path:
//   mu = mean(x), var = mean((x - mu)^2), y = (x - mu) / sqrt(var + eps) * g + b,
//   a = max(max|y|, 1e-5), xq = clamp(rne(y * 127 / a), -128, 127), act_scale = a / 127.
//
// The arithmetic is binary64.  Subtracting the mean cancels: in fp32 the
// pre-rounding value of a code near +-0.5 would move by ~1e-5 (the mean's own
// rounding, scaled by 127 / max|y|), far more than the 1e-6 relative band in
// which a code may round either way, so codes would not be reproducible.  In
// binary64 every pre-rounding value is within a few 2^-53 of the exact one.
//
// One CTA per row (grid-stride over rows).  Pass 1 reads the row from HBM
// (sum), passes 2-4 (sum of squared deviations, max|y|, codes) re-read it from
// L1/L2 (a row of 4096 bf16 is 8 KB).  HBM-bound on the first read; the fp64
// work per element is a handful of operations.
#include <cuda_bf16.h>

#include "bq_internal.h"

namespace bq {
namespace {

constexpr int kLnThreads = 256;

__device__ __forceinline__ double load_x(const float *p, int64_t k) { return static_cast<double>(__ldg(p + k)); }
__device__ __forceinline__ double load_x(const __nv_bfloat16 *p, int64_t k) {
    return static_cast<double>(__bfloat162float(p[k]));
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, T *red, Op op) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();  // the previous use of `red` is finished
    if (lane == 0) red[warp] = v;
    __syncthreads();
    T r = red[0];
#pragma unroll
    for (int w = 1; w < kLnThreads / 32; ++w) r = op(r, red[w]);
    return r;
}

template <typename In>
__global__ void __launch_bounds__(kLnThreads)
    act_quant_ln_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, double eps,
                        const float *__restrict__ g, const float *__restrict__ b, int8_t *__restrict__ xq,
                        int64_t ldq, float *__restrict__ act_scale, int32_t *__restrict__ rowsum) {
    __shared__ double red_d[kLnThreads / 32];
    __shared__ int red_i[kLnThreads / 32];
    auto add = [](double p, double q) { return p + q; };
    auto mx = [](double p, double q) { return fmax(p, q); };
    auto addi = [](int p, int q) { return p + q; };
    const double inv_k = 1.0 / static_cast<double>(K);
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const In *xr = x + m * ldx;
        double s = 0.0;
        for (int64_t k = threadIdx.x; k < K; k += kLnThreads) s += load_x(xr, k);
        const double mu = block_reduce(s, red_d, add) * inv_k;
        double q = 0.0;
        for (int64_t k = threadIdx.x; k < K; k += kLnThreads) {
            const double d = load_x(xr, k) - mu;
            q = fma(d, d, q);
        }
        const double var = block_reduce(q, red_d, add) * inv_k;
        const double sd = sqrt(var + eps);
        auto y_of = [&](int64_t k) {
            const double d = (load_x(xr, k) - mu) / sd;
            const double gk = g != nullptr ? static_cast<double>(__ldg(g + k)) : 1.0;
            const double bk = b != nullptr ? static_cast<double>(__ldg(b + k)) : 0.0;
            return fma(d, gk, bk);
        };
        double amax = 0.0;
        for (int64_t k = threadIdx.x; k < K; k += kLnThreads) amax = fmax(amax, fabs(y_of(k)));
        const double a = fmax(block_reduce(amax, red_d, mx), 1e-5);
        const double f = 127.0 / a;
        int isum = 0;
        int8_t *qr = xq + m * ldq;
        for (int64_t k = threadIdx.x; k < K; k += kLnThreads) {
            int c = __double2int_rn(y_of(k) * f);  // nearest, ties to even
            c = c < -128 ? -128 : (c > 127 ? 127 : c);
            qr[k] = static_cast<int8_t>(c);
            isum += c;
        }
        isum = block_reduce(isum, red_i, addi);
        if (threadIdx.x == 0) {
            act_scale[m] = static_cast<float>(a / 127.0);
            if (rowsum != nullptr) rowsum[m] = isum;
        }
    }
}

}  // namespace

cudaError_t launch_act_quant_ln(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *ln_weight,
                                const float *ln_bias, float eps, int8_t *xq, int64_t ldq, float *act_scale,
                                int32_t *rowsum, cudaStream_t s, const DevInfo &dev) {
    const int64_t grid = std::min<int64_t>(M, static_cast<int64_t>(dev.num_sms) * 8);
    if (xt == BQ_BF16)
        act_quant_ln_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), kLnThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), M, K, ldx, static_cast<double>(eps), ln_weight, ln_bias, xq, ldq,
            act_scale, rowsum);
    else
        act_quant_ln_kernel<float><<<static_cast<unsigned>(grid), kLnThreads, 0, s>>>(
            static_cast<const float *>(x), M, K, ldx, static_cast<double>(eps), ln_weight, ln_bias, xq, ldq,
            act_scale, rowsum);
    return cudaGetLastError();
}

}  // namespace bq
