// Backward of the BitLinear forward under the straight-through estimator
// ("Class BitLinear" (LLaMA-BitNet utils.py): steps 2-3 quantize "(STE)";
// "Common Attention Utilities": activation_quant / weight_quant "pass gradients
// through the rounding operation unchanged").  The forward used
// xt = xq * act_scale for the normalised input y and wt = wq * gamma for w,
// with identity gradients through both, so for dout [M,N]:
//
//   dW[n,k] = sum_m dout[m,n] * act_scale[m] * xq[m,k]
//   dy[m,k] = gamma * sum_n dout[m,n] * wq[n,k]
//   dx[m,k] = (dy[m,k] - y[m,k] * mean_j(dy[m,j] * y[m,j])) / r[m]   (RMSNorm backward)
//
// The two contractions run on the bf16 tensor cores (gemm_bf16.cu) with
// operands that are exact in bf16: dout (bf16), the ternary codes wq
// (-1 / 0 / 1), the int8 codes xq; act_scale runs along the contraction of
// dW, so the products dout * act_scale are split into hi + lo bf16 parts
// stacked along the contraction (rows m and M + m), each pair carrying the
// product to 16 significant bits.  The RMSNorm backward takes its row
// reductions in binary64.
#include <cuda_bf16.h>

#include <algorithm>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

// wpacked [N][K/16] 2-bit offset-binary codes -> wt [N][K] bf16 (w_q = code - 1).
__global__ void ternary_to_bf16_kernel(const uint32_t *__restrict__ wpacked, int64_t N, int64_t K,
                                       __nv_bfloat16 *__restrict__ wt) {
    const int64_t words = N * (K / 16);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint32_t u = __ldg(wpacked + i);
        uint32_t out[8];  // 16 bf16, k = 16 w + 4 j + b at bits [8b + 2j, 8b + 2j + 1]
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint16_t h[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t c = (u >> (8 * b + 2 * j)) & 3u;
                h[b] = c == 0u ? 0xBF80u : (c == 2u ? 0x3F80u : 0u);  // -1, +1, 0
            }
            out[2 * j] = h[0] | (static_cast<uint32_t>(h[1]) << 16);
            out[2 * j + 1] = h[2] | (static_cast<uint32_t>(h[3]) << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(wt + i * 16);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
}

// Operands of dW: a2 [2M][N] bf16 with rows m = hi(dout[m,:] * s[m]) and
// M + m = lo(...) (hi = bf16(p), lo = bf16(p - hi), p the fp32 product), and
// b2 [2M][K] bf16 = the codes xq[m,:] in rows m and M + m.  Eight elements
// per thread and step (N % 8 == 0, K % 16 == 0): 16-byte loads and stores.
__global__ void dw_operands_kernel(const __nv_bfloat16 *__restrict__ dout, const float *__restrict__ act_scale,
                                   const int8_t *__restrict__ xq, int64_t M, int64_t N, int64_t K,
                                   __nv_bfloat16 *__restrict__ a2, __nv_bfloat16 *__restrict__ b2) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t nth = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t n8 = N / 8, k8 = K / 8;
    for (int64_t i = tid; i < M * n8; i += nth) {
        const int64_t m = i / n8;
        const float sm = __ldg(act_scale + m);
        const uint4 d = __ldcs(reinterpret_cast<const uint4 *>(dout) + i);
        const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t h2 = 0, l2 = 0;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float prod = __fmul_rn(__uint_as_float(e ? (dw[j] & 0xffff0000u) : (dw[j] << 16)), sm);
                const __nv_bfloat16 h = __float2bfloat16_rn(prod);
                const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(prod, __bfloat162float(h)));
                h2 |= static_cast<uint32_t>(__bfloat16_as_ushort(h)) << (16 * e);
                l2 |= static_cast<uint32_t>(__bfloat16_as_ushort(l)) << (16 * e);
            }
            hi[j] = h2;
            lo[j] = l2;
        }
        reinterpret_cast<uint4 *>(a2)[i] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        reinterpret_cast<uint4 *>(a2 + M * N)[i] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    for (int64_t i = tid; i < M * k8; i += nth) {
        const uint2 q = __ldg(reinterpret_cast<const uint2 *>(xq) + i);
        const uint32_t qw[2] = {q.x, q.y};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c0 = static_cast<int8_t>((qw[j >> 1] >> (16 * (j & 1))) & 0xffu);
            const int c1 = static_cast<int8_t>((qw[j >> 1] >> (16 * (j & 1) + 8)) & 0xffu);
            o[j] = static_cast<uint32_t>(__bfloat16_as_ushort(__int2bfloat16_rn(c0))) |
                   (static_cast<uint32_t>(__bfloat16_as_ushort(__int2bfloat16_rn(c1))) << 16);
        }
        const uint4 v = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4 *>(b2)[i] = v;
        reinterpret_cast<uint4 *>(b2 + M * K)[i] = v;
    }
}

// 8 consecutive elements of x as floats
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}

// dx = (dy - y * mean(dy * y)) / r, y = x / r, r = sqrt(mean(x^2) + eps): one
// CTA per row, row reductions in binary64, eight elements per thread and step
// (K % 16 == 0).
template <typename In>
__global__ void __launch_bounds__(256) rms_backward_kernel(const In *__restrict__ x, const float *__restrict__ dy,
                                                           int64_t M, int64_t K, double eps, float *__restrict__ dx) {
    __shared__ double red[2][8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const In *xr = x + m * K;
        const float *dr = dy + m * K;
        double ss = 0.0, dot = 0.0;
        for (int64_t k = 8 * threadIdx.x; k < K; k += 8 * 256) {
            float xv[8], dv[8];
            load8(xr + k, xv);
            load8(dr + k, dv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double xd = static_cast<double>(xv[e]);
                ss = fma(xd, xd, ss);
                dot = fma(static_cast<double>(dv[e]), xd, dot);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            dot += __shfl_xor_sync(0xffffffffu, dot, o);
        }
        __syncthreads();
        if (lane == 0) {
            red[0][warp] = ss;
            red[1][warp] = dot;
        }
        __syncthreads();
        ss = 0.0;
        dot = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            ss += red[0][w];
            dot += red[1][w];
        }
        const double r = sqrt(ss / static_cast<double>(K) + eps);
        // mean(dy * y) = dot / (r K); dx = (dy - x / r * mean(dy * y)) / r
        const double c = dot / (r * r * static_cast<double>(K));
        const double inv_r = 1.0 / r;
        for (int64_t k = 8 * threadIdx.x; k < K; k += 8 * 256) {
            float xv[8], dv[8], o[8];
            load8(xr + k, xv);
            load8(dr + k, dv);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                o[e] = static_cast<float>((static_cast<double>(dv[e]) - static_cast<double>(xv[e]) * c) * inv_r);
            float4 *dst = reinterpret_cast<float4 *>(dx + m * K + k);
            dst[0] = make_float4(o[0], o[1], o[2], o[3]);
            dst[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
    }
}

int grid_of_items(int64_t items, const DevInfo &dev) {
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, dev.num_sms * 16)));
}

}  // namespace

BwdLayout bitlinear_bwd_layout(int64_t M, int64_t N, int64_t K) {
    auto a256 = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
    const size_t m = static_cast<size_t>(M), n = static_cast<size_t>(N), k = static_cast<size_t>(K);
    BwdLayout l;
    l.xq = 0;
    l.scale = l.xq + a256(m * k);
    l.wt = l.scale + a256(m * 4);
    l.a2 = l.wt + a256(n * k * 2);
    l.b2 = l.a2 + a256(2 * m * n * 2);
    l.dy = l.b2 + a256(2 * m * k * 2);
    l.total = l.dy + a256(m * k * 4);
    return l;
}

bq_status launch_bitlinear_backward(const void *x, bq_dtype xt, const void *dout, int64_t M, int64_t K,
                                    const uint32_t *wpacked, const float *w_scale, int64_t N, float eps, float *dx,
                                    float *dw, void *workspace, cudaStream_t s, const DevInfo &dev) {
    const BwdLayout l = bitlinear_bwd_layout(M, N, K);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + l.xq);
    float *act_scale = reinterpret_cast<float *>(ws + l.scale);
    __nv_bfloat16 *wt = reinterpret_cast<__nv_bfloat16 *>(ws + l.wt);
    __nv_bfloat16 *a2 = reinterpret_cast<__nv_bfloat16 *>(ws + l.a2);
    __nv_bfloat16 *b2 = reinterpret_cast<__nv_bfloat16 *>(ws + l.b2);
    float *dy = reinterpret_cast<float *>(ws + l.dy);
    // the forward's codes and scales, again from x
    if (launch_act_quant(x, xt, M, K, K, eps, xq, K, act_scale, nullptr, s, dev) != cudaSuccess) return BQ_ERR_CUDA;
    ternary_to_bf16_kernel<<<grid_of_items(N * K / 16, dev), 256, 0, s>>>(wpacked, N, K, wt);
    dw_operands_kernel<<<grid_of_items(M * std::max(N, K) / 8, dev), 256, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(dout), act_scale, xq, M, N, K, a2, b2);
    if (cudaGetLastError() != cudaSuccess) return BQ_ERR_CUDA;
    // dy [M][K] = gamma * dout [M][N] . wt [N][K]   (A K-major, B N-major)
    Bf16Args g;
    g.a = dout;
    g.lda = N;
    g.a_mn = false;
    g.b = wt;
    g.ldb = K;
    g.b_mn = true;
    g.M = M;
    g.N = K;
    g.K = N;
    g.scale = w_scale;
    g.out = dy;
    g.ldo = K;
    bq_status st = launch_gemm_bf16(g, s, dev);
    if (st != BQ_OK) return st;
    // dW [N][K] = a2^T [N][2M] . b2 [2M][K]   (A M-major, B N-major)
    Bf16Args h;
    h.a = a2;
    h.lda = N;
    h.a_mn = true;
    h.b = b2;
    h.ldb = K;
    h.b_mn = true;
    h.M = N;
    h.N = K;
    h.K = 2 * M;
    h.scale = nullptr;
    h.out = dw;
    h.ldo = K;
    st = launch_gemm_bf16(h, s, dev);
    if (st != BQ_OK) return st;
    const int rgrid = static_cast<int>(std::min<int64_t>(M, dev.num_sms * 8));
    if (xt == BQ_BF16)
        rms_backward_kernel<__nv_bfloat16><<<rgrid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), dy, M, K,
                                                                 static_cast<double>(eps), dx);
    else
        rms_backward_kernel<float><<<rgrid, 256, 0, s>>>(static_cast<const float *>(x), dy, M, K,
                                                         static_cast<double>(eps), dx);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace bq
