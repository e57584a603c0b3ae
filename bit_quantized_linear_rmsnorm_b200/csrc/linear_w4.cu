// Grouped affine INT4 linear with fp32 activations
// ("vyre_libs/nn/linear/inner/linear_4bit/mod.rs" (docs.rs vyre-libs), module
// doc: the packed u32 word is loaded and the nibble for k is extracted inside
// the k loop, so no dequantized weight ever exists; grouped affine path with a
// scale and a zero-point per group, plus bias):
//
//   out[m,n] = bias[n] + sum_k x[m,k] * s[n,g] * (q[n,k] - z[n,g]),  g = k / gs
//
// Prologue: each (token, group) slice of x becomes a 24-bit fixed-point
// integer X = rne(x / sx) with sx = max|x| / (2^23 - 1), stored as three byte
// planes X = 65536*P0 + 256*P1 + P2 (P0 signed, P1 and P2 unsigned), plus
// sx and sum(X) per (token, group).  The representation error is at most
// sx (one unit: the quotient's fp32 rounding plus the integer rounding),
// i.e. max|x| * 1.2e-7.
//
// Main kernel: inner products D_p = sum_k q[n,k] * P_p[k] are exact int32
// dp4a dot products; per 32-weight chunk (one group)
//   contribution = s[n,g] * sx[m,g] * (65536*D0 + 256*D1 + D2)
// and per group the zero-point term  - s[n,g] * z[n,g] * sx[m,g] * sum(X).
// Within a packed word, (word & 0x0f0f0f0f) holds the nibbles of elements
// 0,2,4,6 and ((word >> 4) & 0x0f0f0f0f) those of 1,3,5,7; the planes are
// stored in that interleaved order so each matches one dp4a.
#include <cuda_fp16.h>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

constexpr int kWarps = 8;

struct W4Workspace {
    int8_t *planes;  // [3][M][K], byte order within each 8-chunk: 0,2,4,6,1,3,5,7
    float *sx;       // [M][G]
    int32_t *sumX;   // [M][G]
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

__host__ __device__ inline W4Workspace carve(void *ws, int64_t M, int64_t K, int64_t G) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    W4Workspace w;
    w.planes = reinterpret_cast<int8_t *>(p);
    size_t off = align256(static_cast<size_t>(3 * M * K));
    w.sx = reinterpret_cast<float *>(p + off);
    off += align256(static_cast<size_t>(M * G) * 4);
    w.sumX = reinterpret_cast<int32_t *>(p + off);
    return w;
}

__device__ __forceinline__ int perm8(int64_t k) {
    const int j = static_cast<int>(k & 7);
    return static_cast<int>(k & ~7ll) + ((j & 1) ? 4 + (j >> 1) : (j >> 1));
}

// One warp per (token, group).
__global__ void __launch_bounds__(256)
    w4_split_x_kernel(const float *__restrict__ x, int64_t M, int64_t K, int64_t gs, W4Workspace ws) {
    const int lane = threadIdx.x & 31;
    const int64_t G = K / gs;
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
    for (int64_t t = warp; t < M * G; t += nwarps) {
        const int64_t m = t / G, g = t % G;
        const float *xr = x + m * K + g * gs;
        float amax = 0.f;
        for (int64_t i = lane; i < gs; i += 32) amax = fmaxf(amax, fabsf(xr[i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sx = __fdiv_rn(amax, 8388607.0f);
        int sum = 0;
        for (int64_t i = lane; i < gs; i += 32) {
            int X = 0;
            if (amax > 0.f) {
                X = __float2int_rn(__fdiv_rn(xr[i], sx));
                X = max(-8388607, min(8388607, X));
            }
            sum += X;
            const int64_t k = g * gs + i;
            const int64_t pos = m * K + perm8(k);
            ws.planes[pos] = static_cast<int8_t>(X >> 16);
            ws.planes[M * K + pos] = static_cast<int8_t>((X >> 8) & 255);
            ws.planes[2 * M * K + pos] = static_cast<int8_t>(X & 255);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            ws.sx[t] = sx;
            ws.sumX[t] = sum;
        }
    }
}

__device__ __forceinline__ float warp_fsum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Tokens [m0, m0 + MT) of one pass; planes of those tokens staged in shared
// memory as [3][MT][K].  VEC: K % 32 == 0 and gs % 32 == 0, one group per
// 16-byte chunk of packed weights.
template <int MT, bool VEC>
__global__ void __launch_bounds__(kWarps * 32)
    w4_linear_dp4a_kernel(const uint32_t *__restrict__ qweight, const uint16_t *__restrict__ scales,
                          const uint32_t *__restrict__ qzeros, const float *__restrict__ bias, int64_t N,
                          int64_t K, int64_t gs, W4Workspace ws, int64_t M, int64_t m0, float *__restrict__ out) {
    extern __shared__ __align__(16) uint8_t sp[];  // [3][MT][K]
    const int lane = threadIdx.x & 31;
    const int64_t G = K / gs;
    const int64_t wrow = K / 8;
    const int64_t zrow = (G + 7) / 8;
    const int mt = static_cast<int>(M - m0 < MT ? M - m0 : MT);

    for (int p = 0; p < 3; ++p)
        for (int m = 0; m < mt; ++m) {
            const uint2 *src = reinterpret_cast<const uint2 *>(ws.planes + (p * M + m0 + m) * K);
            uint2 *dst = reinterpret_cast<uint2 *>(sp + (p * MT + m) * K);
            for (int64_t i = threadIdx.x; i < K / 8; i += blockDim.x) dst[i] = src[i];
        }
    __syncthreads();

    const int64_t warp = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t n = warp; n < N; n += nwarps) {
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.f;

        if constexpr (VEC) {
            const uint4 *wr = reinterpret_cast<const uint4 *>(qweight + n * wrow);
            for (int64_t c = lane; c < wrow / 4; c += 32) {
                const uint4 wv = __ldcs(wr + c);
                const int64_t k0 = 32 * c;
                const int64_t g = k0 / gs;
                const float sw = __half2float(__ushort_as_half(__ldg(scales + n * G + g)));
                int D[MT][3];
#pragma unroll
                for (int m = 0; m < MT; ++m) D[m][0] = D[m][1] = D[m][2] = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // words 2h, 2h+1
                    const uint32_t wa = h == 0 ? wv.x : wv.z;
                    const uint32_t wb = h == 0 ? wv.y : wv.w;
                    const uint32_t lo_a = wa & 0x0f0f0f0fu, hi_a = (wa >> 4) & 0x0f0f0f0fu;
                    const uint32_t lo_b = wb & 0x0f0f0f0fu, hi_b = (wb >> 4) & 0x0f0f0f0fu;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m < mt) {
#pragma unroll
                            for (int p = 0; p < 3; ++p) {
                                const uint4 pv = *reinterpret_cast<const uint4 *>(sp + (p * MT + m) * K + k0 + 16 * h);
                                if (p == 0) {
                                    int d = D[m][0];
                                    d = dp4a_us(lo_a, pv.x, d);
                                    d = dp4a_us(hi_a, pv.y, d);
                                    d = dp4a_us(lo_b, pv.z, d);
                                    d = dp4a_us(hi_b, pv.w, d);
                                    D[m][0] = d;
                                } else {
                                    uint32_t d = static_cast<uint32_t>(D[m][p]);
                                    d = dp4a_uu(lo_a, pv.x, d);
                                    d = dp4a_uu(hi_a, pv.y, d);
                                    d = dp4a_uu(lo_b, pv.z, d);
                                    d = dp4a_uu(hi_b, pv.w, d);
                                    D[m][p] = static_cast<int>(d);
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < mt) {
                        const float T = fmaf(65536.0f, static_cast<float>(D[m][0]),
                                             fmaf(256.0f, static_cast<float>(D[m][1]), static_cast<float>(D[m][2])));
                        const float f = __fmul_rn(sw, ws.sx[(m0 + m) * G + g]);
                        acc[m] = fmaf(f, T, acc[m]);
                    }
                }
            }
        } else {
            const uint32_t *wr = qweight + n * wrow;
            for (int64_t w = lane; w < wrow; w += 32) {
                const uint32_t u = __ldg(wr + w);
                const int64_t k0 = 8 * w;
                const int64_t g = k0 / gs;
                const float sw = __half2float(__ushort_as_half(__ldg(scales + n * G + g)));
                const uint32_t lo = u & 0x0f0f0f0fu, hi = (u >> 4) & 0x0f0f0f0fu;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < mt) {
                        const uint2 p0 = *reinterpret_cast<const uint2 *>(sp + (0 * MT + m) * K + k0);
                        const uint2 p1 = *reinterpret_cast<const uint2 *>(sp + (1 * MT + m) * K + k0);
                        const uint2 p2 = *reinterpret_cast<const uint2 *>(sp + (2 * MT + m) * K + k0);
                        const int d0 = dp4a_us(hi, p0.y, dp4a_us(lo, p0.x, 0));
                        const int d1 = static_cast<int>(dp4a_uu(hi, p1.y, dp4a_uu(lo, p1.x, 0u)));
                        const int d2 = static_cast<int>(dp4a_uu(hi, p2.y, dp4a_uu(lo, p2.x, 0u)));
                        const float T = fmaf(65536.0f, static_cast<float>(d0),
                                             fmaf(256.0f, static_cast<float>(d1), static_cast<float>(d2)));
                        acc[m] = fmaf(__fmul_rn(sw, ws.sx[(m0 + m) * G + g]), T, acc[m]);
                    }
                }
            }
        }
        // zero-point term, one group per lane step
        for (int64_t g = lane; g < G; g += 32) {
            const float sw = __half2float(__ushort_as_half(__ldg(scales + n * G + g)));
            const uint32_t z = (__ldg(qzeros + n * zrow + g / 8) >> (4 * (g % 8))) & 15u;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < mt) {
                    const int64_t t = (m0 + m) * G + g;
                    const float corr = __fmul_rn(__fmul_rn(sw, static_cast<float>(z)), ws.sx[t]);
                    acc[m] = fmaf(-corr, static_cast<float>(ws.sumX[t]), acc[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m < mt) {
                const float v = warp_fsum(acc[m]);
                if (lane == 0) out[(m0 + m) * N + n] = (bias ? __ldg(bias + n) : 0.0f) + v;
            }
        }
    }
}

template <int MT, bool VEC>
cudaError_t launch_pass(const uint32_t *qweight, const uint16_t *scales, const uint32_t *qzeros, const float *bias,
                        int64_t N, int64_t K, int64_t gs, const W4Workspace &ws, int64_t M, int64_t m0, float *out,
                        cudaStream_t s, const DevInfo &dev) {
    const size_t smem = static_cast<size_t>(3 * MT) * static_cast<size_t>(K);
    auto kern = w4_linear_dp4a_kernel<MT, VEC>;
    static size_t attr_smem[64] = {};  // largest opt-in set so far, per device
    if (smem > 48 * 1024 && smem > attr_smem[dev.device]) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        attr_smem[dev.device] = smem;
    }
    int64_t grid = (N + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * 8;
    if (grid > cap) grid = cap;
    kern<<<static_cast<unsigned>(grid), kWarps * 32, smem, s>>>(qweight, scales, qzeros, bias, N, K, gs, ws, M, m0,
                                                                out);
    return cudaGetLastError();
}

template <bool VEC>
cudaError_t launch_all(const uint32_t *qweight, const uint16_t *scales, const uint32_t *qzeros, const float *bias,
                       int64_t N, int64_t K, int64_t gs, const W4Workspace &ws, int64_t M, float *out,
                       cudaStream_t s, const DevInfo &dev) {
    // widest pass whose planes fit in shared memory
    const bool fit4 = 3 * 4 * K <= 192 * 1024;
    const bool fit2 = 3 * 2 * K <= 192 * 1024;
    for (int64_t m0 = 0; m0 < M;) {
        const int64_t left = M - m0;
        cudaError_t e;
        if (left >= 3 && fit4) {
            e = launch_pass<4, VEC>(qweight, scales, qzeros, bias, N, K, gs, ws, M, m0, out, s, dev);
            m0 += 4;
        } else if (left >= 2 && fit2) {
            e = launch_pass<2, VEC>(qweight, scales, qzeros, bias, N, K, gs, ws, M, m0, out, s, dev);
            m0 += 2;
        } else {
            e = launch_pass<1, VEC>(qweight, scales, qzeros, bias, N, K, gs, ws, M, m0, out, s, dev);
            m0 += 1;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

size_t linear_w4_workspace_bytes(int64_t M, int64_t K, int64_t group_size) {
    const int64_t G = K / group_size;
    return align256(static_cast<size_t>(3 * M * K)) + align256(static_cast<size_t>(M * G) * 4) +
           align256(static_cast<size_t>(M * G) * 4);
}

cudaError_t launch_linear_w4(const float *x, int64_t M, int64_t K, const uint32_t *qweight, const uint16_t *scales,
                             const uint32_t *qzeros, const float *bias, int64_t N, int64_t group_size, float *out,
                             void *ws_ptr, cudaStream_t s, const DevInfo &dev) {
    const int64_t G = K / group_size;
    const W4Workspace ws = carve(ws_ptr, M, K, G);
    int64_t grid = (M * G + 7) / 8;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * 8;
    if (grid > cap) grid = cap;
    w4_split_x_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(x, M, K, group_size, ws);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const bool vec = (K % 32 == 0) && (group_size % 32 == 0) && (reinterpret_cast<uintptr_t>(qweight) % 16 == 0);
    if (vec) return launch_all<true>(qweight, scales, qzeros, bias, N, K, group_size, ws, M, out, s, dev);
    return launch_all<false>(qweight, scales, qzeros, bias, N, K, group_size, ws, M, out, s, dev);
}

}  // namespace bq
