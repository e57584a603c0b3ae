// Per-token activation quantization arithmetic shared by the standalone
// quantization kernel and the fused decode kernels, so that every path takes
// the same fp32 decisions ("Class BitLinear" (LLaMA-BitNet utils.py) forward
// steps 1-2; activation_quant of "Common Attention Utilities").
//
//   r = sqrt(mean(x^2) + eps), a = max(max|x| / r, 1e-5)
//   code = rne(x * f) with f = (1/r) * (127/a), act_scale = a / 127
//
// The code is the low byte of fma(x, f, 1.5 * 2^23): the product is exact
// inside the fma, so x*f is rounded once, to nearest even.  1/r cancels
// between y = x/r and a, so the pre-rounding value is within three fp32
// roundings of the exact x*127/max|x|; |x*f| <= 127*(1 + 2^-22) never rounds
// outside [-127, 127], so the definition's clamp to [-128, 127] is a no-op.
#pragma once

#include <cuda_bf16.h>

#include "bq_common.cuh"

namespace bq {

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

template <typename In>
struct Elt;
template <>
struct Elt<float> {
    static constexpr int kPerChunk = 4;  // elements per 16-byte chunk
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

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Four rounded codes (low bytes of the magic-number sums) packed into a word.
__device__ __forceinline__ uint32_t pack_codes4(float t0, float t1, float t2, float t3) {
    const uint32_t p01 = __byte_perm(__float_as_uint(t0), __float_as_uint(t1), 0x0040);
    const uint32_t p23 = __byte_perm(__float_as_uint(t2), __float_as_uint(t3), 0x0040);
    return __byte_perm(p01, p23, 0x5410);
}

__device__ __forceinline__ int code_of(float t) { return static_cast<int>(__float_as_uint(t)) - 0x4B400000; }

// Row statistics -> the code factor f and the row's act_scale.
__device__ __forceinline__ void quant_row_factor(float ss, float amax, int64_t K, float eps, float &f,
                                                 float &act_scale) {
    const float ms = __fdiv_rn(ss, static_cast<float>(K));
    const float r = __fsqrt_rn(__fadd_rn(ms, eps));
    const float inv_r = __fdiv_rn(1.0f, r);
    const float a = fmaxf(__fmul_rn(amax, inv_r), 1e-5f);
    const float qs = __fdiv_rn(127.0f, a);
    f = __fmul_rn(inv_r, qs);
    act_scale = __fdiv_rn(a, 127.0f);
}

// One warp quantizes one row of K values whose start is 16-byte aligned and
// K % (16 / sizeof(In)) == 0.  Two passes over the row (the second hits L1).
// Codes go to dst0 (and dst1 when not null); returns act_scale and rowsum in
// every lane.
template <typename In>
__device__ __forceinline__ void warp_quant_row_vec(const In *__restrict__ xr, int64_t K, float eps, int8_t *dst0,
                                                   int8_t *dst1, float &act_scale, int &rowsum) {
    constexpr int EPC = Elt<In>::kPerChunk;
    const int lane = threadIdx.x & 31;
    const uint4 *xv = reinterpret_cast<const uint4 *>(xr);
    const int64_t nchunks = K / EPC;
    float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
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
    const float ss = warp_sum_f(ss0 + ss1);
    amax = warp_max_f(amax);
    float fac;
    quant_row_factor(ss, amax, K, eps, fac, act_scale);
    int isum = 0;
    for (int64_t c = lane; c < nchunks; c += 32) {
        float e[EPC];
        Elt<In>::unpack(__ldg(xv + c), e);
        uint32_t w[EPC / 4];
#pragma unroll
        for (int j = 0; j < EPC / 4; ++j) {
            w[j] = pack_codes4(fmaf(e[4 * j], fac, kRoundMagic), fmaf(e[4 * j + 1], fac, kRoundMagic),
                               fmaf(e[4 * j + 2], fac, kRoundMagic), fmaf(e[4 * j + 3], fac, kRoundMagic));
            isum = dp4a_ss(w[j], 0x01010101u, isum);
        }
        if constexpr (EPC == 8) {
            *reinterpret_cast<uint2 *>(dst0 + c * 8) = make_uint2(w[0], w[1]);
            if (dst1) *reinterpret_cast<uint2 *>(dst1 + c * 8) = make_uint2(w[0], w[1]);
        } else {
            *reinterpret_cast<uint32_t *>(dst0 + c * 4) = w[0];
            if (dst1) *reinterpret_cast<uint32_t *>(dst1 + c * 4) = w[0];
        }
    }
    rowsum = warp_sum_i(isum);
}

}  // namespace bq
