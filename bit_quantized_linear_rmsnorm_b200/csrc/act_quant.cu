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
#include <algorithm>

#include "bq_internal.h"
#include "quant_common.cuh"

namespace bq {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kCacheChunks = 16;  // 16-byte chunks per lane kept in registers

// Vector path: row base and stride keep 16-byte alignment.
template <typename In>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    act_quant_vec_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
                         int8_t *__restrict__ xq, int64_t ldq, float *__restrict__ act_scale,
                         int32_t *__restrict__ rowsum) {
    constexpr int EPC = Elt<In>::kPerChunk;
    pdl_launch_dependents();  // a dependent GEMM reads the codes only after its wait
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
        const float ss = warp_sum_f(ss0 + ss1);
        amax = warp_max_f(amax);
        float f, scale;
        quant_row_factor(ss, amax, K, eps, f, scale);

        int isum = 0;
        auto quant_chunk = [&](const uint4 &v, int64_t c) {
            float e[EPC];
            Elt<In>::unpack(v, e);
            uint32_t w[EPC / 4];
#pragma unroll
            for (int j = 0; j < EPC / 4; ++j) {
                w[j] = pack_codes4(fmaf(e[4 * j], f, kRoundMagic), fmaf(e[4 * j + 1], f, kRoundMagic),
                                   fmaf(e[4 * j + 2], f, kRoundMagic), fmaf(e[4 * j + 3], f, kRoundMagic));
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
            const int code = code_of(fmaf(xt, f, kRoundMagic));
            qr[tail0 + lane] = static_cast<int8_t>(code);
            isum += code;
        }
        isum = warp_sum_i(isum);
        if (lane == 0) {
            act_scale[m] = scale;
            if (rowsum) rowsum[m] = isum;
        }
    }
}

// Block-per-row path for many rows (M of at least four CTAs per SM): a CTA of
// 128 threads takes rows b, b + G, ...; thread t holds chunks t + 128 j
// (j < CPT) of the row, so every load and store instruction of a warp covers
// contiguous bytes, and it loads the chunks of its next row before reducing
// and writing the current one (two rows in flight per CTA).  The rows spread
// evenly over all CTAs, where one warp per row leaves a partial last wave of
// rows.  Same arithmetic as the warp-per-row path.
constexpr int kRowThreads = 128;
template <typename In, int CPT>
__global__ void __launch_bounds__(kRowThreads)
    act_quant_row_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
                         int8_t *__restrict__ xq, int64_t ldq, float *__restrict__ act_scale,
                         int32_t *__restrict__ rowsum) {
    constexpr int EPC = Elt<In>::kPerChunk;
    pdl_launch_dependents();  // a dependent GEMM reads the codes only after its wait
    __shared__ float s_ss[kRowThreads / 32], s_mx[kRowThreads / 32];
    __shared__ int s_rs[kRowThreads / 32];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int nchunks = static_cast<int>(K / EPC);  // K % EPC == 0 on this path
    uint4 cur[CPT], nxt[CPT];
    auto load_row = [&](int64_t m, uint4 (&dst)[CPT]) {
        const uint4 *xv = reinterpret_cast<const uint4 *>(x + m * ldx);
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + kRowThreads * j;
            dst[j] = (m < M && c < nchunks) ? __ldcs(xv + c) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    int64_t m = blockIdx.x;
    load_row(m, cur);
    for (; m < M; m += gridDim.x) {
        load_row(m + gridDim.x, nxt);
        float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            float f[EPC];
            Elt<In>::unpack(cur[j], f);
#pragma unroll
            for (int e = 0; e < EPC; e += 2) {
                ss0 = fmaf(f[e], f[e], ss0);
                ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
            }
        }
        const float wss = warp_sum_f(ss0 + ss1), wmx = warp_max_f(amax);
        if (lane == 0) {
            s_ss[warp] = wss;
            s_mx[warp] = wmx;
        }
        __syncthreads();
        float ss = 0.f, mx = 0.f;
#pragma unroll
        for (int w = 0; w < kRowThreads / 32; ++w) {
            ss += s_ss[w];
            mx = fmaxf(mx, s_mx[w]);
        }
        float f, scale;
        quant_row_factor(ss, mx, K, eps, f, scale);
        int8_t *qr = xq + m * ldq;
        int isum = 0;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + kRowThreads * j;
            if (c < nchunks) {
                float e[EPC];
                Elt<In>::unpack(cur[j], e);
                uint32_t w[EPC / 4];
#pragma unroll
                for (int q = 0; q < EPC / 4; ++q) {
                    w[q] = pack_codes4(fmaf(e[4 * q], f, kRoundMagic), fmaf(e[4 * q + 1], f, kRoundMagic),
                                       fmaf(e[4 * q + 2], f, kRoundMagic), fmaf(e[4 * q + 3], f, kRoundMagic));
                    isum = dp4a_ss(w[q], 0x01010101u, isum);
                }
                if constexpr (EPC == 8) {
                    *reinterpret_cast<uint2 *>(qr + c * 8) = make_uint2(w[0], w[1]);
                } else {
                    *reinterpret_cast<uint32_t *>(qr + c * 4) = w[0];
                }
            }
        }
        isum = warp_sum_i(isum);
        if (lane == 0) s_rs[warp] = isum;
        __syncthreads();
        if (t == 0) {
            int r = 0;
#pragma unroll
            for (int w = 0; w < kRowThreads / 32; ++w) r += s_rs[w];
            act_scale[m] = scale;
            if (rowsum) rowsum[m] = r;
        }
#pragma unroll
        for (int j = 0; j < CPT; ++j) cur[j] = nxt[j];
    }
}

// Scalar path for rows without 16-byte alignment: two passes over x.
template <typename In>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    act_quant_scalar_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
                            int8_t *__restrict__ xq, int64_t ldq, float *__restrict__ act_scale,
                            int32_t *__restrict__ rowsum) {
    pdl_launch_dependents();  // a dependent GEMM reads the codes only after its wait
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
        ss = warp_sum_f(ss);
        amax = warp_max_f(amax);
        float f, scale;
        quant_row_factor(ss, amax, K, eps, f, scale);
        int isum = 0;
        for (int64_t k = lane; k < K; k += 32) {
            const int code = code_of(fmaf(Elt<In>::get(xr, k), f, kRoundMagic));
            xq[m * ldq + k] = static_cast<int8_t>(code);
            isum += code;
        }
        isum = warp_sum_i(isum);
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
    constexpr int EPC = Elt<In>::kPerChunk;
    const int64_t nch = K / EPC;
    const int64_t rgrid = std::min<int64_t>(M, static_cast<int64_t>(dev.num_sms) * 12);
    const bool rows_path = vec && K % EPC == 0 && nch <= 8 * kRowThreads && M >= 4 * dev.num_sms &&
                           reinterpret_cast<uintptr_t>(xq) % 8 == 0 && ldq % 8 == 0;
    if (rows_path) {
        const int cpt = static_cast<int>((nch + kRowThreads - 1) / kRowThreads);
        auto kern = cpt <= 1   ? act_quant_row_kernel<In, 1>
                    : cpt <= 2 ? act_quant_row_kernel<In, 2>
                    : cpt <= 4 ? act_quant_row_kernel<In, 4>
                               : act_quant_row_kernel<In, 8>;
        kern<<<static_cast<unsigned>(rgrid), kRowThreads, 0, s>>>(x, M, K, ldx, eps, xq, ldq, act_scale, rowsum);
        return cudaGetLastError();
    }
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
