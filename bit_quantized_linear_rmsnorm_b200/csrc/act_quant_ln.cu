// Per-token int8 activation quantization after a LayerNorm: the normaliser of
// BitLinear and BitConv1d in "Common Attention Utilities" (frankenstein-
// transformer: "Applies LayerNorm to inputs before quantization"), followed by
// the same per-token absmax quantization as the RMSNorm path:
//   mu = mean(x), var = mean((x - mu)^2), y = (x - mu) / sqrt(var + eps) * g + b,
//   a = max(max|y|, 1e-5), xq = clamp(rne(y * 127 / a), -128, 127), act_scale = a / 127.
//
// Subtracting the mean cancels: with the mean rounded to fp32 first, the
// pre-rounding value of a code near +-0.5 would move by ~1e-5 (the mean's own
// rounding, scaled by 127 / max|y|), far more than the 1e-6 relative band in
// which a code may round either way.  So the mean and variance are taken in
// binary64, and y is formed either in binary64 or, in the warp-per-row kernel,
// in fp32 with the row constants 1/sqrt(var + eps) and -mean/sqrt(var + eps)
// split into two fp32 parts: the mean then cancels exactly inside one fused
// multiply-add before its only rounding, and y stays within a few fp32
// roundings of itself (the bound and the per-row check that sends other rows
// to binary64 are at the kernel).  Either way every pre-rounding value is well
// inside the tie band of the exact one.
//
// Aligned rows are read once from HBM and every pass (mean and variance,
// max|y|, codes) works from on-chip copies: at least eight rows of up to
// 768 16-byte chunks take one warp per row with the row staged in shared
// memory; fewer rows of up to 1024 chunks take one CTA per row, the row in
// registers; other rows take the general kernel, which re-reads the row from
// L1/L2 in each pass.  HBM-bound: one read of x, one write of the codes.
#include <cuda_bf16.h>

#include <algorithm>

#include "bq_common.cuh"
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
    pdl_wait();  // x may come from the previous kernel; its readers of xq are done
    pdl_launch_dependents();
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
        const double rsd = 1.0 / sqrt(var + eps);  // one division per row
        auto y_of = [&](int64_t k) {
            const double d = (load_x(xr, k) - mu) * rsd;
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

// Rows with 16-byte aligned bases and K a multiple of the elements per
// 16-byte chunk, at most 256 * CPT chunks: one read of the row from HBM into
// registers (chunk c of a row held by thread c % 256), then the mean, the
// variance, max|y| and the codes from registers.
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
    static constexpr int kElts = 4;
    __device__ static void unpack(const uint4 &v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
};
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int kElts = 8;
    __device__ static void unpack(const uint4 &v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <typename In, int CPT>
__global__ void __launch_bounds__(kLnThreads)
    act_quant_ln_vec_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, double eps,
                            const float *__restrict__ g, const float *__restrict__ b, int8_t *__restrict__ xq,
                            int64_t ldq, float *__restrict__ act_scale, int32_t *__restrict__ rowsum) {
    constexpr int E = Vec16<In>::kElts;
    __shared__ double red_d[kLnThreads / 32];
    __shared__ int red_i[kLnThreads / 32];
    auto add = [](double p, double q) { return p + q; };
    auto mx = [](double p, double q) { return fmax(p, q); };
    auto addi = [](int p, int q) { return p + q; };
    const double inv_k = 1.0 / static_cast<double>(K);
    const int nch = static_cast<int>(K / E);
    pdl_wait();  // x may come from the previous kernel; its readers of xq are done
    pdl_launch_dependents();
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + m * ldx);
        float v[CPT][E];
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + kLnThreads * i;
            const uint4 u = c < nch ? __ldcs(xr + c) : make_uint4(0u, 0u, 0u, 0u);
            Vec16<In>::unpack(u, v[i]);
        }
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < CPT; ++i)
#pragma unroll
            for (int e = 0; e < E; ++e) s += static_cast<double>(v[i][e]);
        const double mu = block_reduce(s, red_d, add) * inv_k;
        double q = 0.0;
#pragma unroll
        for (int i = 0; i < CPT; ++i)
            if (threadIdx.x + kLnThreads * i < nch)
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const double d = static_cast<double>(v[i][e]) - mu;
                    q = fma(d, d, q);
                }
        const double rsd = 1.0 / sqrt(block_reduce(q, red_d, add) * inv_k + eps);  // one division per row
        auto y_of = [&](int i, int e) {
            const int64_t k = static_cast<int64_t>(threadIdx.x + kLnThreads * i) * E + e;
            const double d = (static_cast<double>(v[i][e]) - mu) * rsd;
            const double gk = g != nullptr ? static_cast<double>(__ldg(g + k)) : 1.0;
            const double bk = b != nullptr ? static_cast<double>(__ldg(b + k)) : 0.0;
            return fma(d, gk, bk);
        };
        double amax = 0.0;
#pragma unroll
        for (int i = 0; i < CPT; ++i)
            if (threadIdx.x + kLnThreads * i < nch)
#pragma unroll
                for (int e = 0; e < E; ++e) amax = fmax(amax, fabs(y_of(i, e)));
        const double a = fmax(block_reduce(amax, red_d, mx), 1e-5);
        const double f = 127.0 / a;
        int isum = 0;
        int8_t *qr = xq + m * ldq;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + kLnThreads * i;
            if (c < nch) {
                uint32_t w[E / 4];
#pragma unroll
                for (int j = 0; j < E / 4; ++j) {
                    uint32_t word = 0;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int code = __double2int_rn(y_of(i, 4 * j + u) * f);  // nearest, ties to even
                        code = code < -128 ? -128 : (code > 127 ? 127 : code);
                        isum += code;
                        word |= (static_cast<uint32_t>(code) & 0xffu) << (8 * u);
                    }
                    w[j] = word;
                }
                if constexpr (E == 8)
                    *reinterpret_cast<uint2 *>(qr + static_cast<int64_t>(c) * 8) = make_uint2(w[0], w[1]);
                else
                    *reinterpret_cast<uint32_t *>(qr + static_cast<int64_t>(c) * 4) = w[0];
            }
        }
        isum = block_reduce(isum, red_i, addi);
        if (threadIdx.x == 0) {
            act_scale[m] = static_cast<float>(a / 127.0);
            if (rowsum != nullptr) rowsum[m] = isum;
        }
    }
}

// One warp per row (aligned rows, K a multiple of the chunk's elements):
// each lane copies its 16-byte chunks of the row into the warp's slice of
// shared memory with cp.async (all in flight at once), then the passes read
// the row from there; reductions by warp shuffles only (no block barrier),
// eight rows in flight per CTA.  In the passes lane l owns the four
// consecutive elements k = 4 l + 128 i, so one warp instruction reads 128
// consecutive elements of the row, of g and of b, and writes 128 consecutive
// codes (every access coalesced; g and b are L1-resident across rows).  The
// first pass accumulates the sum and the sum of squares of x - x[0] in
// binary64 together.
__device__ __forceinline__ void quad_of(const uint8_t *rowb, int k0, const float *, float (&v)[4]) {
    const float4 t = *reinterpret_cast<const float4 *>(rowb + 4 * k0);
    v[0] = t.x;
    v[1] = t.y;
    v[2] = t.z;
    v[3] = t.w;
}
__device__ __forceinline__ void quad_of(const uint8_t *rowb, int k0, const __nv_bfloat16 *, float (&v)[4]) {
    const uint2 t = *reinterpret_cast<const uint2 *>(rowb + 2 * k0);
    v[0] = __uint_as_float(t.x << 16);
    v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16);
    v[3] = __uint_as_float(t.y & 0xffff0000u);
}
// p[k0 .. k0 + 3] (def where p is null); v16: p is 16-byte aligned
__device__ __forceinline__ void affine_quad(const float *p, bool v16, int k0, float def, double (&o)[4]) {
    if (p == nullptr) {
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = def;
    } else if (v16) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p + k0));
        o[0] = t.x;
        o[1] = t.y;
        o[2] = t.z;
        o[3] = t.w;
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = __ldg(p + k0 + j);
    }
}

__device__ __forceinline__ void affine_quad_f(const float *p, bool v16, int k0, float def, float (&o)[4]) {
    if (p == nullptr) {
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = def;
    } else if (v16) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p + k0));
        o[0] = t.x;
        o[1] = t.y;
        o[2] = t.z;
        o[3] = t.w;
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = __ldg(p + k0 + j);
    }
}

template <typename In>
__global__ void __launch_bounds__(kLnThreads)
    act_quant_ln_warp_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, double eps,
                             const float *__restrict__ g, const float *__restrict__ b, int8_t *__restrict__ xq,
                             int64_t ldq, float *__restrict__ act_scale, int32_t *__restrict__ rowsum) {
    constexpr int E = Vec16<In>::kElts;
    extern __shared__ uint4 srows[];  // [8][nch]
    const int lane = threadIdx.x & 31;
    const int nch = static_cast<int>(K / E);
    const int kk = static_cast<int>(K);
    uint4 *row = srows + static_cast<int64_t>(threadIdx.x >> 5) * nch;
    const uint8_t *rowb = reinterpret_cast<const uint8_t *>(row);
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kLnThreads / 32) + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kLnThreads / 32);
    const double inv_k = 1.0 / static_cast<double>(K);
    const bool g16 = reinterpret_cast<uintptr_t>(g) % 16 == 0;
    const bool b16 = reinterpret_cast<uintptr_t>(b) % 16 == 0;
    pdl_wait();  // x may come from the previous kernel; its readers of xq are done
    pdl_launch_dependents();
    float gmax = 1.0f;  // max |g| over the row (the same for every row)
    if (g != nullptr) {
        gmax = 0.0f;
        for (int k0 = 4 * lane; k0 < kk; k0 += 128) {
            float gk[4];
            affine_quad_f(g, g16, k0, 1.0f, gk);
#pragma unroll
            for (int e = 0; e < 4; ++e) gmax = fmaxf(gmax, fabsf(gk[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
    }
    for (int64_t m = warp; m < M; m += nwarps) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + m * ldx);
        __syncwarp();  // the previous row's readers are done with the slice
        for (int ch = lane; ch < nch; ch += 32) cp_async_16(smem_u32(row + ch), xr + ch, 16);
        cp_async_commit();
        cp_async_wait_all();
        __syncwarp();
        // sums of d = x - c and d^2 with c the row's first element (x - c is
        // exact in binary64), so the variance E[d^2] - E[d]^2 cancels only by
        // (mu - c)^2 / var, a few units for any row, not by mu^2 / var
        double c;
        {
            float v0[4];
            quad_of(rowb, 0, x, v0);
            c = static_cast<double>(v0[0]);
        }
        double s = 0.0, s2 = 0.0;
        for (int k0 = 4 * lane; k0 < kk; k0 += 128) {
            float v[4];
            quad_of(rowb, k0, x, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const double d = static_cast<double>(v[e]) - c;
                s += d;
                s2 = fma(d, d, s2);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, o);
            s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        }
        const double md = s * inv_k;
        const double mu = c + md;
        const double var = fmax(s2 * inv_k - md * md, 0.0);
        const double rsd = 1.0 / sqrt(var + eps);  // one division per row
        const double nmr = -mu * rsd;
        int8_t *qr = xq + m * ldq;
        int isum = 0;
        float scale;

        // Passes 2 and 3 in fp32 with the row constants split into two fp32
        // parts: x * rsd_h + nmr_h is formed exactly inside one FMA (the mean
        // cancels before the only rounding) and corrected by the low parts, so
        // y is within about three fp32 roundings of itself plus an absolute
        // 6 u^2 |nmr| |g| (u = 2^-24).  Scaled by f = 127 / max|y|, that term
        // stays below 4.3e-8 when |nmr| * max|g| * f < 2^21, far inside the
        // 1e-6 band around a rounding tie (5e-7 at the smallest tie, 0.5), so
        // the codes agree with binary64 ones outside it.  Rows that fail the
        // check (a near-constant row far from zero, say) take the binary64 passes.
        const float rsd_h = static_cast<float>(rsd), rsd_l = static_cast<float>(rsd - static_cast<double>(rsd_h));
        const float nmr_h = static_cast<float>(nmr), nmr_l = static_cast<float>(nmr - static_cast<double>(nmr_h));
        auto y_quad_f = [&](int k0, float (&y)[4]) {
            float v[4], gk[4], bk[4];
            quad_of(rowb, k0, x, v);
            affine_quad_f(g, g16, k0, 1.0f, gk);
            affine_quad_f(b, b16, k0, 0.0f, bk);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float yn = __fadd_rn(__fmaf_rn(v[e], rsd_h, nmr_h), __fmaf_rn(v[e], rsd_l, nmr_l));
                y[e] = __fmaf_rn(yn, gk[e], bk[e]);
            }
        };
        float amax_f = 0.0f;
        for (int k0 = 4 * lane; k0 < kk; k0 += 128) {
            float y[4];
            y_quad_f(k0, y);
#pragma unroll
            for (int e = 0; e < 4; ++e) amax_f = fmaxf(amax_f, fabsf(y[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax_f = fmaxf(amax_f, __shfl_xor_sync(0xffffffffu, amax_f, o));
        const float a_f = fmaxf(amax_f, 1e-5f);
        const float f_f = __fdiv_rn(127.0f, a_f);
        if (fabs(nmr) * static_cast<double>(gmax) * static_cast<double>(f_f) < 2097152.0) {
            for (int k0 = 4 * lane; k0 < kk; k0 += 128) {
                float y[4];
                y_quad_f(k0, y);
                uint32_t word = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // nearest, ties to even: y * f added to 1.5 * 2^23 in one rounding
                    int code = __float_as_int(__fmaf_rn(y[e], f_f, 12582912.0f)) - 0x4B400000;
                    code = code < -128 ? -128 : (code > 127 ? 127 : code);
                    isum += code;
                    word |= (static_cast<uint32_t>(code) & 0xffu) << (8 * e);
                }
                *reinterpret_cast<uint32_t *>(qr + k0) = word;
            }
            scale = __fdiv_rn(a_f, 127.0f);
        } else {
            // binary64 passes: y for the quad at k0 = (x - mu) / sqrt(var + eps) * g + b
            auto y_quad = [&](int k0, double (&y)[4]) {
                float v[4];
                quad_of(rowb, k0, x, v);
                double gk[4], bk[4];
                affine_quad(g, g16, k0, 1.0f, gk);
                affine_quad(b, b16, k0, 0.0f, bk);
#pragma unroll
                for (int e = 0; e < 4; ++e) y[e] = fma(fma(static_cast<double>(v[e]), rsd, nmr), gk[e], bk[e]);
            };
            double amax = 0.0;
            for (int k0 = 4 * lane; k0 < kk; k0 += 128) {
                double y[4];
                y_quad(k0, y);
#pragma unroll
                for (int e = 0; e < 4; ++e) amax = fmax(amax, fabs(y[e]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const double a = fmax(amax, 1e-5);
            const double f = 127.0 / a;
            for (int k0 = 4 * lane; k0 < kk; k0 += 128) {
                double y[4];
                y_quad(k0, y);
                uint32_t word = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int code = __double2int_rn(y[e] * f);  // nearest, ties to even
                    code = code < -128 ? -128 : (code > 127 ? 127 : code);
                    isum += code;
                    word |= (static_cast<uint32_t>(code) & 0xffu) << (8 * e);
                }
                *reinterpret_cast<uint32_t *>(qr + k0) = word;
            }
            scale = static_cast<float>(a / 127.0);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(0xffffffffu, isum, o);
        if (lane == 0) {
            act_scale[m] = scale;
            if (rowsum != nullptr) rowsum[m] = isum;
        }
    }
}

template <typename In>
cudaError_t launch_ln_typed(const In *x, int64_t M, int64_t K, int64_t ldx, double eps, const float *g, const float *b,
                            int8_t *xq, int64_t ldq, float *act_scale, int32_t *rowsum, cudaStream_t s,
                            const DevInfo &dev) {
    constexpr int E = Vec16<In>::kElts;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(M, static_cast<int64_t>(dev.num_sms) * 8));
    const bool vec = reinterpret_cast<uintptr_t>(x) % 16 == 0 && (ldx * static_cast<int64_t>(sizeof(In))) % 16 == 0 &&
                     K % E == 0 && reinterpret_cast<uintptr_t>(xq) % 8 == 0 && ldq % 8 == 0;
    const int64_t cpt = (K / E + kLnThreads - 1) / kLnThreads;
    // launched as a programmatic dependent of the previous kernel; it waits for
    // it before touching memory and then releases its own dependent
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kLnThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int64_t nch = K / E;
    const size_t wsmem = static_cast<size_t>(kLnThreads / 32) * static_cast<size_t>(nch) * 16;
    if (vec && M >= 8 && wsmem <= 96 * 1024) {
        // one warp per row, rows staged in shared memory
        static SmemOptIn opt_in;
        if (wsmem > 48 * 1024) {
            const cudaError_t e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(act_quant_ln_warp_kernel<In>),
                                              wsmem);
            if (e != cudaSuccess) return e;
        }
        cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>((M + 7) / 8, static_cast<int64_t>(dev.num_sms) * 8)));
        cfg.dynamicSmemBytes = wsmem;
        return cudaLaunchKernelEx(&cfg, act_quant_ln_warp_kernel<In>, x, M, K, ldx, eps, g, b, xq, ldq, act_scale,
                                  rowsum);
    }
    if (vec && cpt <= 1)
        return cudaLaunchKernelEx(&cfg, act_quant_ln_vec_kernel<In, 1>, x, M, K, ldx, eps, g, b, xq, ldq, act_scale,
                                  rowsum);
    if (vec && cpt <= 2)
        return cudaLaunchKernelEx(&cfg, act_quant_ln_vec_kernel<In, 2>, x, M, K, ldx, eps, g, b, xq, ldq, act_scale,
                                  rowsum);
    if (vec && cpt <= 4)
        return cudaLaunchKernelEx(&cfg, act_quant_ln_vec_kernel<In, 4>, x, M, K, ldx, eps, g, b, xq, ldq, act_scale,
                                  rowsum);
    return cudaLaunchKernelEx(&cfg, act_quant_ln_kernel<In>, x, M, K, ldx, eps, g, b, xq, ldq, act_scale, rowsum);
}

}  // namespace

cudaError_t launch_act_quant_ln(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *ln_weight,
                                const float *ln_bias, float eps, int8_t *xq, int64_t ldq, float *act_scale,
                                int32_t *rowsum, cudaStream_t s, const DevInfo &dev) {
    if (xt == BQ_BF16)
        return launch_ln_typed(static_cast<const __nv_bfloat16 *>(x), M, K, ldx, static_cast<double>(eps), ln_weight,
                               ln_bias, xq, ldq, act_scale, rowsum, s, dev);
    return launch_ln_typed(static_cast<const float *>(x), M, K, ldx, static_cast<double>(eps), ln_weight, ln_bias, xq,
                           ldq, act_scale, rowsum, s, dev);
}

}  // namespace bq
