// 4-bit activations and 4-bit weights with given step sizes: the forward of
// Q4LinearFunction ("bitorch_engine.layers.qlinear.nbit.cutlass.q4_layer",
// bitorch-engine: "quantizes inputs and weights to 4-bits using specified
// scale factors and performs linear"; eps "to avoid division by zero").
//
//   s_a = max(scale_a, eps), s_w[n] = max(scale_w[n or 0], eps)
//   xq = clamp(rne(x / s_a), -8, 7),  wq = clamp(rne(w / s_w[n]), -8, 7)
//   out[m,n] = (float(sum_k xq * wq) * s_w[n]) * s_a (+ bias[n])
//
// sm_100 has no 4-bit integer tensor-core kind, so the weights stay packed
// (eight signed nibbles per word) in HBM and are sign-extended to int8 where
// they are used: in shared memory ahead of the tcgen05 kind::i8 MMA for more
// than 16 tokens (the packed-B path of the GEMM), in registers ahead of dp4a
// in the GEMV below for up to 16 tokens.  The activation codes are int8.
//
// The quotient v / s is the correctly rounded fp32 division, rounded to
// nearest-even by rintf: within half an fp32 ulp of the exact quotient, so a
// code differs from the exact decision only inside the 1e-6 tie band.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

__device__ __forceinline__ float load_v(const float *p, int64_t i) { return __ldg(p + i); }
__device__ __forceinline__ float load_v(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }

__device__ __forceinline__ int q4_code(float v, float step) {
    const float q = rintf(__fdiv_rn(v, step));
    return static_cast<int>(fminf(fmaxf(q, -8.0f), 7.0f));
}

__device__ __forceinline__ float step_of(const float *scale, int64_t i, float eps) {
    return fmaxf(__ldg(scale + i), eps);
}

// One thread per packed word (eight weights of one row).
template <typename In>
__global__ void q4_weight_pack_kernel(const In *__restrict__ w, int64_t N, int64_t K, const float *__restrict__ scale_w,
                                      int per_channel, float eps, uint32_t *__restrict__ wpacked) {
    const int64_t words = K / 8, total = N * words;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t n = i / words, k0 = (i - n * words) * 8;
        const float st = step_of(scale_w, per_channel ? n : 0, eps);
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            word |= (static_cast<uint32_t>(q4_code(load_v(w, n * K + k0 + j), st)) & 15u) << (4 * j);
        wpacked[i] = word;
    }
}

// Activation codes (int8 [M][ldq]) plus, for the linear, the per-row step
// s_a [M] and the per-channel step s_w [N] the epilogue multiplies by.
template <typename In>
__global__ void q4_act_quant_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx,
                                    const float *__restrict__ scale_a, float eps, int8_t *__restrict__ xq,
                                    int64_t ldq, float *__restrict__ row_step, const float *__restrict__ scale_w,
                                    int per_channel, int64_t N, float *__restrict__ col_step) {
    const float sa = step_of(scale_a, 0, eps);
    const int64_t total = M * K;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = tid; i < total; i += stride) {
        const int64_t m = i / K, k = i - m * K;
        xq[m * ldq + k] = static_cast<int8_t>(q4_code(load_v(x, m * ldx + k), sa));
    }
    if (row_step != nullptr)
        for (int64_t m = tid; m < M; m += stride) row_step[m] = sa;
    if (col_step != nullptr)
        for (int64_t n = tid; n < N; n += stride) col_step[n] = step_of(scale_w, per_channel ? n : 0, eps);
}

// The same for rows whose base is 16-byte aligned and K % 8 == 0: eight
// elements (one or two 16-byte loads) per thread and step, eight codes stored
// at once.
template <typename In>
__global__ void q4_act_quant_vec_kernel(const In *__restrict__ x, int64_t M, int64_t K, int64_t ldx,
                                        const float *__restrict__ scale_a, float eps, int8_t *__restrict__ xq,
                                        int64_t ldq, float *__restrict__ row_step, const float *__restrict__ scale_w,
                                        int per_channel, int64_t N, float *__restrict__ col_step) {
    const float sa = step_of(scale_a, 0, eps);
    const int64_t cpr = K / 8, total = M * cpr;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = tid; i < total; i += stride) {
        const int64_t m = i / cpr, k0 = (i - m * cpr) * 8;
        float v[8];
        if constexpr (sizeof(In) == 2) {
            const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(x + m * ldx + k0));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[2 * j] = __uint_as_float(w[j] << 16);
                v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
        } else {
            const float4 a = __ldcs(reinterpret_cast<const float4 *>(x + m * ldx + k0));
            const float4 b = __ldcs(reinterpret_cast<const float4 *>(x + m * ldx + k0 + 4));
            v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
        }
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            lo |= (static_cast<uint32_t>(q4_code(v[j], sa)) & 0xffu) << (8 * j);
            hi |= (static_cast<uint32_t>(q4_code(v[4 + j], sa)) & 0xffu) << (8 * j);
        }
        *reinterpret_cast<uint2 *>(xq + m * ldq + k0) = make_uint2(lo, hi);
    }
    if (row_step != nullptr)
        for (int64_t m = tid; m < M; m += stride) row_step[m] = sa;
    if (col_step != nullptr)
        for (int64_t n = tid; n < N; n += stride) col_step[n] = step_of(scale_w, per_channel ? n : 0, eps);
}

// Up to 16 tokens: one warp per weight row at a time (grid-stride over rows),
// lanes stride over 16-byte pieces (32 weights) of the row; the codes of all
// tokens sit in shared memory.  Each nibble n goes to the high half of a byte,
// which read as s8 is exactly 16 n; dp4a sums 16 x the products, and the
// final sum is shifted down by 4 (exact).
constexpr int kGemvWarps = 8;

template <int MT, typename OutT>
__global__ void __launch_bounds__(kGemvWarps * 32)
    w4a4_gemv_kernel(const int8_t *__restrict__ xq, int M, int64_t K, const uint32_t *__restrict__ wpacked,
                     const float *__restrict__ row_step, const float *__restrict__ col_step,
                     const float *__restrict__ bias, int64_t N, OutT *__restrict__ out) {
    extern __shared__ __align__(16) int8_t xs[];  // [MT][K]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t chunks = static_cast<int64_t>(M) * K / 16;
    for (int64_t i = threadIdx.x; i < chunks; i += blockDim.x)
        reinterpret_cast<uint4 *>(xs)[i] = __ldg(reinterpret_cast<const uint4 *>(xq) + i);
    __syncthreads();
    const int64_t pieces = K / 32;  // 16-byte pieces of a packed row
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * kGemvWarps + warp; n < N;
         n += static_cast<int64_t>(gridDim.x) * kGemvWarps) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(wpacked + n * (K / 8));
        int acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0;
#pragma unroll 4
        for (int64_t pc = lane; pc < pieces; pc += 32) {
            const uint4 u = __ldcs(wr + pc);
            const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
            uint32_t b[8];  // 32 sign-extended codes, k = 32 pc + 4 j + 0..3 in b[j]
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const uint32_t lo = (ws[h] << 4) & 0xF0F0F0F0u, hi = ws[h] & 0xF0F0F0F0u;
                b[2 * h] = __byte_perm(lo, hi, 0x5140);
                b[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const uint4 *xr = reinterpret_cast<const uint4 *>(xs + static_cast<int64_t>(m) * K + 32 * pc);
                    const uint4 a0 = xr[0], a1 = xr[1];
                    int s = acc[m];
                    s = dp4a_ss(a0.x, b[0], s);
                    s = dp4a_ss(a0.y, b[1], s);
                    s = dp4a_ss(a0.z, b[2], s);
                    s = dp4a_ss(a0.w, b[3], s);
                    s = dp4a_ss(a1.x, b[4], s);
                    s = dp4a_ss(a1.y, b[5], s);
                    s = dp4a_ss(a1.z, b[6], s);
                    s = dp4a_ss(a1.w, b[7], s);
                    acc[m] = s;
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            int v = acc[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[m] = v;
        }
        if (lane < M) {
            int v = acc[0];
#pragma unroll
            for (int m = 1; m < MT; ++m)
                if (lane == m) v = acc[m];
            v >>= 4;  // the sum of 16 x the products
            float o = __fmul_rn(__fmul_rn(static_cast<float>(v), __ldg(col_step + n)), __ldg(row_step + lane));
            if (bias != nullptr) o = __fadd_rn(o, __ldg(bias + n));
            if constexpr (sizeof(OutT) == 4)
                out[static_cast<int64_t>(lane) * N + n] = o;
            else if constexpr (std::is_same<OutT, __half>::value)
                out[static_cast<int64_t>(lane) * N + n] = __float2half_rn(o);
            else
                out[static_cast<int64_t>(lane) * N + n] = __float2bfloat16_rn(o);
        }
    }
}

template <int MT, typename OutT>
cudaError_t launch_gemv_mt(const int8_t *xq, int M, int64_t K, const uint32_t *wpacked, const float *row_step,
                           const float *col_step, const float *bias, int64_t N, void *out, cudaStream_t s,
                           const DevInfo &dev) {
    auto kern = w4a4_gemv_kernel<MT, OutT>;
    const size_t smem = static_cast<size_t>(M) * static_cast<size_t>(K);
    static SmemOptIn opt_in;
    if (smem > 48 * 1024) {
        const cudaError_t e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), smem);
        if (e != cudaSuccess) return e;
    }
    int64_t grid = (N + kGemvWarps - 1) / kGemvWarps;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * (smem > 100 * 1024 ? 2 : smem > 24 * 1024 ? 4 : 8);
    if (grid > cap) grid = cap;
    kern<<<static_cast<unsigned>(grid), kGemvWarps * 32, smem, s>>>(xq, M, K, wpacked, row_step, col_step, bias, N,
                                                                     static_cast<OutT *>(out));
    return cudaGetLastError();
}

template <typename OutT>
cudaError_t launch_gemv_out(const int8_t *xq, int M, int64_t K, const uint32_t *wpacked, const float *row_step,
                            const float *col_step, const float *bias, int64_t N, void *out, cudaStream_t s,
                            const DevInfo &dev) {
    if (M <= 4) return launch_gemv_mt<4, OutT>(xq, M, K, wpacked, row_step, col_step, bias, N, out, s, dev);
    if (M <= 8) return launch_gemv_mt<8, OutT>(xq, M, K, wpacked, row_step, col_step, bias, N, out, s, dev);
    return launch_gemv_mt<16, OutT>(xq, M, K, wpacked, row_step, col_step, bias, N, out, s, dev);
}

int grid_for(int64_t items, const DevInfo &dev) {
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, dev.num_sms * 16)));
}

}  // namespace

cudaError_t launch_q4_weight_pack(const void *w, bq_dtype wt, int64_t N, int64_t K, const float *scale_w,
                                  int per_channel, float eps, uint32_t *wpacked, cudaStream_t s, const DevInfo &dev) {
    const int grid = grid_for(N * K / 8, dev);
    if (wt == BQ_BF16)
        q4_weight_pack_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(w), N, K, scale_w,
                                                                  per_channel, eps, wpacked);
    else
        q4_weight_pack_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float *>(w), N, K, scale_w, per_channel,
                                                          eps, wpacked);
    return cudaGetLastError();
}

cudaError_t launch_q4_act_quant(const void *x, bq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *scale_a,
                                float eps, int8_t *xq, int64_t ldq, float *row_step, const float *scale_w,
                                int per_channel, int64_t N, float *col_step, cudaStream_t s, const DevInfo &dev) {
    const bool vec = K % 8 == 0 && reinterpret_cast<uintptr_t>(x) % 16 == 0 &&
                     (ldx * (xt == BQ_BF16 ? 2 : 4)) % 16 == 0 && reinterpret_cast<uintptr_t>(xq) % 8 == 0 &&
                     ldq % 8 == 0;
    if (vec) {
        const int vgrid = grid_for(std::max<int64_t>(M * K / 8, N), dev);
        if (xt == BQ_BF16)
            q4_act_quant_vec_kernel<__nv_bfloat16><<<vgrid, 256, 0, s>>>(
                static_cast<const __nv_bfloat16 *>(x), M, K, ldx, scale_a, eps, xq, ldq, row_step, scale_w, per_channel,
                N, col_step);
        else
            q4_act_quant_vec_kernel<float><<<vgrid, 256, 0, s>>>(static_cast<const float *>(x), M, K, ldx, scale_a, eps,
                                                                 xq, ldq, row_step, scale_w, per_channel, N, col_step);
        return cudaGetLastError();
    }
    const int grid = grid_for(std::max<int64_t>(M * K, N), dev);
    if (xt == BQ_BF16)
        q4_act_quant_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), M, K, ldx,
                                                                scale_a, eps, xq, ldq, row_step, scale_w, per_channel,
                                                                N, col_step);
    else
        q4_act_quant_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float *>(x), M, K, ldx, scale_a, eps, xq, ldq,
                                                        row_step, scale_w, per_channel, N, col_step);
    return cudaGetLastError();
}

cudaError_t launch_w4a4_gemv(const int8_t *xq, int64_t M, int64_t K, const uint32_t *wpacked, const float *row_step,
                             const float *col_step, const float *bias, int64_t N, bq_dtype out_dtype, void *out,
                             cudaStream_t s, const DevInfo &dev) {
    const int m = static_cast<int>(M);
    switch (out_dtype) {
        case BQ_F32:
            return launch_gemv_out<float>(xq, m, K, wpacked, row_step, col_step, bias, N, out, s, dev);
        case BQ_F16:
            return launch_gemv_out<__half>(xq, m, K, wpacked, row_step, col_step, bias, N, out, s, dev);
        default:
            return launch_gemv_out<__nv_bfloat16>(xq, m, K, wpacked, row_step, col_step, bias, N, out, s, dev);
    }
}

}  // namespace bq
