// Per-token int8 activation quantization after a parameter-free RMSNorm.
//
// Follows "Class BitLinear" (LLaMA-BitNet utils.py), forward steps 1-2, and
// activation_quant of "Common Attention Utilities" (frankenstein-transformer):
//   r = sqrt(mean(x^2) + eps), y = x / r, a = max(max|y|, 1e-5),
//   xq = clamp(rne(y * 127 / a), -128, 127), act_scale = a / 127.
//
// One warp per row.  Each lane reads its share of the row with 16-byte loads
// and keeps it in registers (rows of up to 512 16-byte chunks, i.e. 4096 bf16
// or 2048 fp32 values; longer rows are read a second time), reduces sum(x^2)
// and max|x| with warp shuffles, then quantizes from registers.  HBM-bound:
// one read of x, one int8 write.
//
// Rounding of the code: t = fma(x, f, 1.5 * 2^23) with f = (1/r) * (127/a)
// rounds x*f to the nearest integer, ties to even, in the low bits of t (the
// product is exact inside the fma, so the value rounded is x*f itself).  The
// factor 1/r cancels between y and a, so the pre-rounding value differs from
// the exact x*127/max|x| by at most three fp32 roundings (<= 1.8e-7
// relative).  |x*f| <= 127 * (1 + 2^-22) always rounds inside [-127, 127], so
// the clamp of the definition never changes a value.
#include <cuda_bf16.h>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kCacheChunks = 16;  // 16-byte chunks per lane kept in registers
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

template <typename In>
struct Elt;
template <>
struct Elt<float> {
    static constexpr int kPerChunk = 4;
    __device__ static float get(const float *p, int64_t i) { return p[i]; }
    __device__ static void unpack(const uint4 &v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
};
template <>
struct Elt<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;
    __device__ static float get(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
    __device__ static void unpack(const uint4 &v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Low byte of t holds the rounded code (two's complement).
__device__ __forceinline__ uint32_t pack4(float t0, float t1, float t2, float t3) {
    const uint32_t p01 = __byte_perm(__float_as_uint(t0), __float_as_uint(t1), 0x0040);
    const uint32_t p23 = __byte_perm(__float_as_uint(t2), __float_as_uint(t3), 0x0040);
    return __byte_perm(p01, p23, 0x5410);
}

// Row statistics -> the code factor f and the row's act_scale.
__device__ __forceinline__ void row_factor(float ss, float amax, int64_t K, float eps, float &f,
                                           float &act_scale) {
    const float ms = __fdiv_rn(ss, static_cast<float>(K));
    const float r = __fsqrt_rn(__fadd_rn(ms, eps));
    const float inv_r = __fdiv_rn(1.0f, r);
    const float a = fmaxf(__fmul_rn(amax, inv_r), 1e-5f);
    const float qs = __fdiv_rn(127.0f, a);
    f = __fmul_rn(inv_r, qs);
    act_scale = __fdiv_rn(a, 127.0f);
}

// Vector path: row base and stride keep 16-byte alignment.
template <typename In>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    act_quant_vec_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
                         int8_t *__restrict__ xq, int64_t ldq, float *__restrict__ act_scale,
                         int32_t *__restrict__ rowsum) {
    constexpr int EPC = Elt<In>::kPerChunk;
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock) + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarpsPerBlock;
    const int64_t nchunks = K / EPC;             // full 16-byte chunks
    const bool cached = nchunks <= 32 * kCacheChunks;

    for (int64_t m = warp; m < M; m += nwarps) {
        const In *xr = x + m * ldx;
        const uint4 *xv = reinterpret_cast<const uint4 *>(xr);
        int8_t *qr = xq + m * ldq;

        uint4 cache[kCacheChunks];
        float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
        if (cached) {
#pragma unroll
            for (int i = 0; i < kCacheChunks; ++i) {
                const int64_t c = lane + 32 * i;
                if (c < nchunks) cache[i] = __ldcs(xv + c);
            }
#pragma unroll
            for (int i = 0; i < kCacheChunks; ++i) {
                const int64_t c = lane + 32 * i;
                if (c < nchunks) {
                    float f[EPC];
                    Elt<In>::unpack(cache[i], f);
#pragma unroll
                    for (int e = 0; e < EPC; e += 2) {
                        ss0 = fmaf(f[e], f[e], ss0);
                        ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                        amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
                    }
                }
            }
        } else {
            for (int64_t c = lane; c < nchunks; c += 32) {
                float f[EPC];
                Elt<In>::unpack(__ldg(xv + c), f);
#pragma unroll
                for (int e = 0; e < EPC; e += 2) {
                    ss0 = fmaf(f[e], f[e], ss0);
                    ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                    amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
                }
            }
        }
        // ragged tail (fewer than EPC elements)
        const int64_t tail0 = nchunks * EPC;
        float xt = 0.f;
        if (tail0 + lane < K) {
            xt = Elt<In>::get(xr, tail0 + lane);
            ss0 = fmaf(xt, xt, ss0);
            amax = fmaxf(amax, fabsf(xt));
        }
        const float ss = warp_sum(ss0 + ss1);
        amax = warp_max(amax);
        float f, scale;
        row_factor(ss, amax, K, eps, f, scale);

        int isum = 0;
        auto quant_chunk = [&](const uint4 &v, int64_t c) {
            float e[EPC];
            Elt<In>::unpack(v, e);
            uint32_t w[EPC / 4];
#pragma unroll
            for (int j = 0; j < EPC / 4; ++j) {
                w[j] = pack4(fmaf(e[4 * j], f, kMagic), fmaf(e[4 * j + 1], f, kMagic),
                             fmaf(e[4 * j + 2], f, kMagic), fmaf(e[4 * j + 3], f, kMagic));
                isum = dp4a_ss(w[j], 0x01010101u, isum);
            }
            if constexpr (EPC == 8) {
                *reinterpret_cast<uint2 *>(qr + c * 8) = make_uint2(w[0], w[1]);
            } else {
                *reinterpret_cast<uint32_t *>(qr + c * 4) = w[0];
            }
        };
        if (cached) {
#pragma unroll
            for (int i = 0; i < kCacheChunks; ++i) {
                const int64_t c = lane + 32 * i;
                if (c < nchunks) quant_chunk(cache[i], c);
            }
        } else {
            for (int64_t c = lane; c < nchunks; c += 32) quant_chunk(__ldg(xv + c), c);
        }
        if (tail0 + lane < K) {
            const float t = fmaf(xt, f, kMagic);
            const int code = static_cast<int>(__float_as_uint(t)) - 0x4B400000;
            qr[tail0 + lane] = static_cast<int8_t>(code);
            isum += code;
        }
        isum = warp_isum(isum);
        if (lane == 0) {
            act_scale[m] = scale;
            if (rowsum) rowsum[m] = isum;
        }
    }
}

// Scalar path for rows without 16-byte alignment: two passes over x.
template <typename In>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    act_quant_scalar_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
                            int8_t *__restrict__ xq, int64_t ldq, float *__restrict__ act_scale,
                            int32_t *__restrict__ rowsum) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock) + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarpsPerBlock;
    for (int64_t m = warp; m < M; m += nwarps) {
        const In *xr = x + m * ldx;
        float ss = 0.f, amax = 0.f;
        for (int64_t k = lane; k < K; k += 32) {
            const float v = Elt<In>::get(xr, k);
            ss = fmaf(v, v, ss);
            amax = fmaxf(amax, fabsf(v));
        }
        ss = warp_sum(ss);
        amax = warp_max(amax);
        float f, scale;
        row_factor(ss, amax, K, eps, f, scale);
        int isum = 0;
        for (int64_t k = lane; k < K; k += 32) {
            const float t = fmaf(Elt<In>::get(xr, k), f, kMagic);
            const int code = static_cast<int>(__float_as_uint(t)) - 0x4B400000;
            xq[m * ldq + k] = static_cast<int8_t>(code);
            isum += code;
        }
        isum = warp_isum(isum);
        if (lane == 0) {
            act_scale[m] = scale;
            if (rowsum) rowsum[m] = isum;
        }
    }
}

template <typename In>
cudaError_t launch_typed(const In *x, int64_t M, int64_t K, int64_t ldx, float eps, int8_t *xq, int64_t ldq,
                         float *act_scale, int32_t *rowsum, cudaStream_t s, const DevInfo &dev) {
    const int64_t want = (M + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * 16;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    const bool vec = (reinterpret_cast<uintptr_t>(x) % 16 == 0) &&
                     ((ldx * static_cast<int64_t>(sizeof(In))) % 16 == 0);
    if (vec)
        act_quant_vec_kernel<In><<<grid, kWarpsPerBlock * 32, 0, s>>>(x, M, K, ldx, eps, xq, ldq, act_scale,
                                                                       rowsum);
    else
        act_quant_scalar_kernel<In><<<grid, kWarpsPerBlock * 32, 0, s>>>(x, M, K, ldx, eps, xq, ldq,
                                                                          act_scale, rowsum);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_act_quant(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, float eps,
                             int8_t *xq, int64_t ldq, float *act_scale, int32_t *rowsum, cudaStream_t s,
                             const DevInfo &dev) {
    if (xt == BQ_BF16)
        return launch_typed(static_cast<const __nv_bfloat16 *>(x), M, K, ldx, eps, xq, ldq, act_scale, rowsum,
                            s, dev);
    return launch_typed(static_cast<const float *>(x), M, K, ldx, eps, xq, ldq, act_scale, rowsum, s, dev);
}

}  // namespace bq
