// Decode path (M <= 16 tokens) of the BitLinear W1.58A8 linear ("Class
// BitLinear" (LLaMA-BitNet utils.py), forward steps 4-5; the page notes that
// specialised ternary kernels are only needed at inference time).
//
//   acc[m,n] = sum_k xq[m,k] * (c[n,k] - 1)  with c the offset-binary code
//            = dot(c, xq) - rowsum[m]
//   out[m,n] = (float(acc) * act_scale[m]) * gamma  (+ bias[n])
//
// Bandwidth-bound on the packed weights (2 bits per weight, read once).  One
// warp owns a pair of output rows at a time; lane l reads 16-byte chunks
// l, l+32, ... of each row, so a warp load is 512 contiguous bytes.  The
// activations (M x K int8) sit in shared memory.  For each packed word
// (16 weights) the code bytes of k = 16w+4j+b are (word >> 2j) & 0x03030303,
// matched with the j-th 32-bit slice of the 16 activation bytes; the dot
// products run on dp4a (u8 codes x s8 activations).  With one token the
// shift is folded into four accumulators: (word & (3 << 2j)) * x sums to
// 4^j times the code dot product, shifted back once per row.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

constexpr int kWarps = 8;
constexpr int kRows = 2;  // output rows per warp iteration

template <typename OutT>
__device__ __forceinline__ OutT to_out(float v);
template <>
__device__ __forceinline__ float to_out<float>(float v) {
    return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half to_out<__half>(float v) {
    return __float2half_rn(v);
}

__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// MT: compile-time upper bound of the token count; M <= MT at run time.
template <int MT, typename OutT>
__global__ void __launch_bounds__(kWarps * 32)
    gemv_w2a8_kernel(const int8_t *__restrict__ xq, int64_t ldq, const float *__restrict__ act_scale,
                     const int32_t *__restrict__ rowsum, const uint32_t *__restrict__ wpacked,
                     const float *__restrict__ w_scale, const float *__restrict__ bias, int M, int64_t N,
                     int64_t K, OutT *__restrict__ out) {
    extern __shared__ __align__(16) uint8_t xs[];  // [M][K] int8
    const int lane = threadIdx.x & 31;
    const int64_t words = K / 16;    // per weight row
    const int64_t chunks = words / 4;  // 16-byte chunks per row (K % 64 == 0 on this path)

    // stage the activations
    for (int m = 0; m < M; ++m) {
        const uint4 *src = reinterpret_cast<const uint4 *>(xq + m * ldq);
        uint4 *dst = reinterpret_cast<uint4 *>(xs + m * K);
        for (int64_t i = threadIdx.x; i < K / 16; i += blockDim.x) dst[i] = src[i];
    }
    __syncthreads();
    const float gamma = __ldg(w_scale);

    const int64_t warp = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t n0 = warp * kRows; n0 < N; n0 += nwarps * kRows) {
        int acc[kRows][MT];
        int acc4[kRows][4];  // single-token split accumulators
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) acc4[r][j] = 0;
        }
        for (int64_t c = lane; c < chunks; c += 32) {
            uint4 wv[kRows];
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                const int64_t n = n0 + r < N ? n0 + r : N - 1;
                wv[r] = __ldcs(reinterpret_cast<const uint4 *>(wpacked + n * words) + c);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // word 4c + q covers k = 64c + 16q .. +16
                const int64_t koff = 64 * c + 16 * q;
                if constexpr (MT == 1) {
                    const uint4 x4 = *reinterpret_cast<const uint4 *>(xs + koff);
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        const uint32_t u = q == 0 ? wv[r].x : q == 1 ? wv[r].y : q == 2 ? wv[r].z : wv[r].w;
                        acc4[r][0] = dp4a_us(u & 0x03030303u, x4.x, acc4[r][0]);
                        acc4[r][1] = dp4a_us(u & 0x0c0c0c0cu, x4.y, acc4[r][1]);
                        acc4[r][2] = dp4a_us(u & 0x30303030u, x4.z, acc4[r][2]);
                        acc4[r][3] = dp4a_us(u & 0xc0c0c0c0u, x4.w, acc4[r][3]);
                    }
                } else {
                    uint32_t cj[kRows][4];
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        const uint32_t u = q == 0 ? wv[r].x : q == 1 ? wv[r].y : q == 2 ? wv[r].z : wv[r].w;
#pragma unroll
                        for (int j = 0; j < 4; ++j) cj[r][j] = (u >> (2 * j)) & 0x03030303u;
                    }
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m < M) {
                            const uint4 x4 = *reinterpret_cast<const uint4 *>(xs + m * K + koff);
#pragma unroll
                            for (int r = 0; r < kRows; ++r) {
                                int a = acc[r][m];
                                a = dp4a_us(cj[r][0], x4.x, a);
                                a = dp4a_us(cj[r][1], x4.y, a);
                                a = dp4a_us(cj[r][2], x4.z, a);
                                a = dp4a_us(cj[r][3], x4.w, a);
                                acc[r][m] = a;
                            }
                        }
                    }
                }
            }
        }
        if constexpr (MT == 1) {
#pragma unroll
            for (int r = 0; r < kRows; ++r)
                acc[r][0] = acc4[r][0] + (acc4[r][1] >> 2) + (acc4[r][2] >> 4) + (acc4[r][3] >> 6);
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const int64_t n = n0 + r;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const int dot = warp_isum(acc[r][m]);
                    if (lane == 0 && n < N) {
                        const int a = dot - __ldg(rowsum + m);
                        float v = __fmul_rn(__fmul_rn(static_cast<float>(a), __ldg(act_scale + m)), gamma);
                        if (bias) v = __fadd_rn(v, __ldg(bias + n));
                        out[static_cast<int64_t>(m) * N + n] = to_out<OutT>(v);
                    }
                }
            }
        }
    }
}

// Generic path: any K % 16 == 0, one packed word per lane step.
template <typename OutT>
__global__ void __launch_bounds__(kWarps * 32)
    gemv_w2a8_word_kernel(const int8_t *__restrict__ xq, int64_t ldq, const float *__restrict__ act_scale,
                          const int32_t *__restrict__ rowsum, const uint32_t *__restrict__ wpacked,
                          const float *__restrict__ w_scale, const float *__restrict__ bias, int M, int64_t N,
                          int64_t K, OutT *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t words = K / 16;
    const float gamma = __ldg(w_scale);
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t n = warp; n < N; n += nwarps) {
        for (int m = 0; m < M; ++m) {
            int a = 0;
            for (int64_t w = lane; w < words; w += 32) {
                const uint32_t u = __ldg(wpacked + n * words + w);
                const uint4 x4 = *reinterpret_cast<const uint4 *>(xq + m * ldq + 16 * w);
                a = dp4a_us(u & 0x03030303u, x4.x, a);
                a = dp4a_us((u >> 2) & 0x03030303u, x4.y, a);
                a = dp4a_us((u >> 4) & 0x03030303u, x4.z, a);
                a = dp4a_us((u >> 6) & 0x03030303u, x4.w, a);
            }
            const int dot = warp_isum(a);
            if (lane == 0) {
                const int acc = dot - __ldg(rowsum + m);
                float v = __fmul_rn(__fmul_rn(static_cast<float>(acc), __ldg(act_scale + m)), gamma);
                if (bias) v = __fadd_rn(v, __ldg(bias + n));
                out[static_cast<int64_t>(m) * N + n] = to_out<OutT>(v);
            }
        }
    }
}

template <int MT, typename OutT>
cudaError_t launch_mt(const int8_t *xq, int64_t ldq, const float *act_scale, const int32_t *rowsum,
                      const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t M, int64_t N,
                      int64_t K, OutT *out, cudaStream_t s, const DevInfo &dev) {
    const size_t smem = static_cast<size_t>(M) * static_cast<size_t>(K);
    auto kern = gemv_w2a8_kernel<MT, OutT>;
    static SmemOptIn opt_in;
    if (smem > 48 * 1024) {
        const cudaError_t e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t rows_per_block = static_cast<int64_t>(kWarps) * kRows;
    int64_t grid = (N + rows_per_block - 1) / rows_per_block;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * 8;
    if (grid > cap) grid = cap;
    kern<<<static_cast<unsigned>(grid), kWarps * 32, smem, s>>>(xq, ldq, act_scale, rowsum, wpacked, w_scale,
                                                                bias, static_cast<int>(M), N, K, out);
    return cudaGetLastError();
}

template <typename OutT>
cudaError_t launch_typed(const int8_t *xq, int64_t ldq, const float *act_scale, const int32_t *rowsum,
                         const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t M, int64_t N,
                         int64_t K, OutT *out, cudaStream_t s, const DevInfo &dev) {
    const bool vec = (K % 64 == 0) && (reinterpret_cast<uintptr_t>(wpacked) % 16 == 0) &&
                     static_cast<size_t>(M) * static_cast<size_t>(K) <= 160 * 1024;
    if (!vec) {
        int64_t grid = (N + kWarps - 1) / kWarps;
        const int64_t cap = static_cast<int64_t>(dev.num_sms) * 8;
        if (grid > cap) grid = cap;
        gemv_w2a8_word_kernel<OutT><<<static_cast<unsigned>(grid), kWarps * 32, 0, s>>>(
            xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, static_cast<int>(M), N, K, out);
        return cudaGetLastError();
    }
    if (M == 1) return launch_mt<1, OutT>(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out, s, dev);
    if (M <= 2) return launch_mt<2, OutT>(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out, s, dev);
    if (M <= 4) return launch_mt<4, OutT>(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out, s, dev);
    if (M <= 8) return launch_mt<8, OutT>(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out, s, dev);
    return launch_mt<16, OutT>(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K, out, s, dev);
}

}  // namespace

cudaError_t launch_gemv_w2a8(const int8_t *xq, int64_t ldq, const float *act_scale, const int32_t *rowsum,
                             const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t M,
                             int64_t N, int64_t K, bq_dtype out_dtype, void *out, cudaStream_t s,
                             const DevInfo &dev) {
    switch (out_dtype) {
        case BQ_F32:
            return launch_typed(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K,
                                static_cast<float *>(out), s, dev);
        case BQ_F16:
            return launch_typed(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K,
                                static_cast<__half *>(out), s, dev);
        default:
            return launch_typed(xq, ldq, act_scale, rowsum, wpacked, w_scale, bias, M, N, K,
                                static_cast<__nv_bfloat16 *>(out), s, dev);
    }
}

}  // namespace bq
