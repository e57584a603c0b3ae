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
    pdl_launch_dependents();  // the GEMV may be scheduled (it reads the codes only after its wait)
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
    pdl_launch_dependents();  // the GEMV may be scheduled (it reads the codes only after its wait)
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
    // launched as a programmatic dependent of the act-quant kernel: before the
    // dependency wait a warp only prefetches its first weight row into L2
    // (which consumes nothing); everything is read after it
    {
        const int64_t n = static_cast<int64_t>(blockIdx.x) * kGemvWarps + warp;
        if (n < N)
            for (int64_t l = lane; l < (K / 2 + 127) / 128; l += 32)
                prefetch_l2(reinterpret_cast<const uint8_t *>(wpacked + n * (K / 8)) + l * 128);
    }
    pdl_launch_dependents();
    pdl_wait();
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
        // four pieces per lane in flight before any of them is used
        for (int64_t base = lane; base < pieces; base += 32 * 4) {
            uint4 u4[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t pc = base + 32 * j;
                u4[j] = pc < pieces ? __ldcs(wr + pc) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t pc = base + 32 * j;
                if (pc >= pieces) break;
                const uint32_t ws[4] = {u4[j].x, u4[j].y, u4[j].z, u4[j].w};
                uint32_t b[8];  // 32 sign-extended codes, k = 32 pc + 4 i + 0..3 in b[i]
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xq, M, K, wpacked, row_step, col_step, bias, N, static_cast<OutT *>(out));
}

template <typename OutT>
cudaError_t launch_gemv_out(const int8_t *xq, int M, int64_t K, const uint32_t *wpacked, const float *row_step,
                            const float *col_step, const float *bias, int64_t N, void *out, cudaStream_t s,
                            const DevInfo &dev) {
    if (M <= 4) return launch_gemv_mt<4, OutT>(xq, M, K, wpacked, row_step, col_step, bias, N, out, s, dev);
    if (M <= 8) return launch_gemv_mt<8, OutT>(xq, M, K, wpacked, row_step, col_step, bias, N, out, s, dev);
    return launch_gemv_mt<16, OutT>(xq, M, K, wpacked, row_step, col_step, bias, N, out, s, dev);
}

// ---------------------------------------------------------------------------
// Straight-through backward (gradients for x, w and scale_a; none for scale_w
// and eps): the reading of Q4LinearFunction.backward ("adjusts gradients
// based on quantization ranges").  With the forward's quotients u = x / s_a
// and v = w / s_w[n]:
//   g  = dout . wh,  wh[n,:] = s_w[n] * wq[n,:]     (bf16 tensor cores)
//   dx = g where -8 <= u <= 7, else 0
//   dw = s_a * (dout^T . xq) where -8 <= v <= 7, else 0
//   dscale_a = sum g * (inside ? xq - u : xq); 0 when scale_a < eps
// The codes are exact in bf16.  Per-channel weight steps run along the
// contraction of g, so they are folded into dout as hi + lo bf16 parts
// stacked along it (2N), each pair carrying the fp32 product to 16
// significant bits; one step for all weights is applied in the epilogue.
// ---------------------------------------------------------------------------
constexpr int kBwdPartMax = 1024;  // CTAs of the dx kernel = binary64 partials of dscale_a

__device__ __forceinline__ void load8v(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x;
    v[1] = a.y;
    v[2] = a.z;
    v[3] = a.w;
    v[4] = b.x;
    v[5] = b.y;
    v[6] = b.z;
    v[7] = b.w;
}
__device__ __forceinline__ void load8v(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

// the steps the GEMM epilogues multiply by: max(scale_a, eps), max(scale_w[0], eps)
__global__ void w4a4_bwd_steps_kernel(const float *__restrict__ scale_a, const float *__restrict__ scale_w, float eps,
                                      float *__restrict__ steps) {
    steps[0] = fmaxf(__ldg(scale_a), eps);
    steps[1] = fmaxf(__ldg(scale_w), eps);
}

// codes clamp(rne(v / s_r), -8, 7) of v [rows][cols] as bf16, s_r = max(scale[r * stride], eps),
// eight per thread (cols % 8 == 0); copies == 2 writes the matrix a second time below itself
template <typename In>
__global__ void q4_codes_bf16_kernel(const In *__restrict__ v, int64_t rows, int64_t cols,
                                     const float *__restrict__ scale, int64_t stride, float eps,
                                     __nv_bfloat16 *__restrict__ out, int copies) {
    const int64_t c8 = cols / 8, total = rows * c8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / c8;
        const float st = fmaxf(__ldg(scale + r * stride), eps);
        float e[8];
        load8v(v + i * 8, e);
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = bf16x2_bits(static_cast<float>(q4_code(e[2 * j], st)), static_cast<float>(q4_code(e[2 * j + 1], st)));
        const uint4 val = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4 *>(out)[i] = val;
        if (copies > 1) reinterpret_cast<uint4 *>(out + rows * cols)[i] = val;
    }
}

// per-channel weight steps folded into dout: a2 [M][2N], column n = hi(p), N + n = lo(p),
// p = dout[m,n] * s_w[n] (fp32), hi = bf16(p), lo = bf16(p - hi); eight per thread (N % 8 == 0)
__global__ void dout_steps_kernel(const __nv_bfloat16 *__restrict__ dout, int64_t M, int64_t N,
                                  const float *__restrict__ scale_w, float eps, __nv_bfloat16 *__restrict__ a2) {
    const int64_t n8 = N / 8, total = M * n8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / n8, c = i - m * n8;
        float d[8];
        load8v(dout + i * 8, d);
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float p = __fmul_rn(d[j], fmaxf(__ldg(scale_w + c * 8 + j), eps));
            hi[j] = __bfloat162float(__float2bfloat16_rn(p));
            lo[j] = __fsub_rn(p, hi[j]);
        }
        uint4 *row = reinterpret_cast<uint4 *>(a2 + m * 2 * N);
        row[c] = make_uint4(bf16x2_bits(hi[0], hi[1]), bf16x2_bits(hi[2], hi[3]), bf16x2_bits(hi[4], hi[5]),
                            bf16x2_bits(hi[6], hi[7]));
        row[n8 + c] = make_uint4(bf16x2_bits(lo[0], lo[1]), bf16x2_bits(lo[2], lo[3]), bf16x2_bits(lo[4], lo[5]),
                                 bf16x2_bits(lo[6], lo[7]));
    }
}

// dx = g inside the range, 0 outside; this CTA's binary64 sum of
// g * (inside ? q - u : q) into part[blockIdx.x] (q - u is exact in fp32:
// an integer minus a quotient within half a unit of it)
template <typename In>
__global__ void __launch_bounds__(256) w4a4_dx_kernel(const In *__restrict__ x, const float *__restrict__ g,
                                                     int64_t M, int64_t K, const float *__restrict__ steps,
                                                     float *__restrict__ dx, double *__restrict__ part) {
    __shared__ double red[8];
    const float sa = steps[0];
    const int64_t total = M * K / 8;
    double acc = 0.0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float e[8], gv[8], o[8];
        load8v(x + i * 8, e);
        load8v(g + i * 8, gv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float u = __fdiv_rn(e[j], sa);  // the forward's quotient
            const float q = fminf(fmaxf(rintf(u), -8.0f), 7.0f);
            const bool in = u >= -8.0f && u <= 7.0f;
            o[j] = in ? gv[j] : 0.0f;
            acc += static_cast<double>(gv[j]) * static_cast<double>(in ? __fsub_rn(q, u) : q);
        }
        float4 *dst = reinterpret_cast<float4 *>(dx + i * 8);
        dst[0] = make_float4(o[0], o[1], o[2], o[3]);
        dst[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += red[w];
        part[blockIdx.x] = t;
    }
}

// dscale_a = the partials summed in a fixed order (one warp), 0 when scale_a < eps
__global__ void w4a4_dscale_kernel(const double *__restrict__ part, int n, const float *__restrict__ scale_a,
                                   float eps, float *__restrict__ dscale) {
    double t = 0.0;
    for (int i = threadIdx.x; i < n; i += 32) t += part[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (threadIdx.x == 0) *dscale = __ldg(scale_a) < eps ? 0.0f : static_cast<float>(t);
}

// dw = 0 where the weight quotient lies outside [-8, 7]; eight per thread (K % 8 == 0)
__global__ void w4a4_dw_mask_kernel(const float *__restrict__ w, int64_t N, int64_t K,
                                    const float *__restrict__ scale_w, int64_t stride, float eps,
                                    float *__restrict__ dw) {
    const int64_t k8 = K / 8, total = N * k8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float st = fmaxf(__ldg(scale_w + (i / k8) * stride), eps);
        float e[8];
        load8v(w + i * 8, e);
        float4 *d = reinterpret_cast<float4 *>(dw + i * 8);
        float4 a = d[0], b = d[1];
        float o[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float u = __fdiv_rn(e[j], st);
            if (!(u >= -8.0f && u <= 7.0f)) o[j] = 0.0f;
        }
        d[0] = make_float4(o[0], o[1], o[2], o[3]);
        d[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
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

W4a4BwdLayout w4a4_bwd_layout(int64_t M, int64_t N, int64_t K) {
    auto a256 = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
    const size_t m = static_cast<size_t>(M), n = static_cast<size_t>(N), k = static_cast<size_t>(K);
    W4a4BwdLayout l;
    l.steps = 0;
    l.xq = 256;
    l.wq = l.xq + a256(m * k * 2);
    l.a2 = l.wq + a256(2 * n * k * 2);
    l.g = l.a2 + a256(m * 2 * n * 2);
    l.part = l.g + a256(m * k * 4);
    l.total = l.part + a256(static_cast<size_t>(kBwdPartMax) * 8);
    return l;
}

bq_status launch_w4a4_backward(const void *x, bq_dtype xt, const float *w, const void *dout, int64_t M, int64_t K,
                               int64_t N, const float *scale_a, const float *scale_w, int per_channel, float eps,
                               float *dx, float *dw, float *dscale_a, void *workspace, cudaStream_t s,
                               const DevInfo &dev) {
    const W4a4BwdLayout l = w4a4_bwd_layout(M, N, K);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *steps = reinterpret_cast<float *>(ws + l.steps);
    __nv_bfloat16 *xqb = reinterpret_cast<__nv_bfloat16 *>(ws + l.xq);
    __nv_bfloat16 *wqb = reinterpret_cast<__nv_bfloat16 *>(ws + l.wq);
    __nv_bfloat16 *a2 = reinterpret_cast<__nv_bfloat16 *>(ws + l.a2);
    float *g = reinterpret_cast<float *>(ws + l.g);
    double *part = reinterpret_cast<double *>(ws + l.part);
    const __nv_bfloat16 *db = static_cast<const __nv_bfloat16 *>(dout);
    w4a4_bwd_steps_kernel<<<1, 1, 0, s>>>(scale_a, scale_w, eps, steps);
    if (xt == BQ_BF16)
        q4_codes_bf16_kernel<__nv_bfloat16><<<grid_for(M * K / 8, dev), 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), M, K, scale_a, 0, eps, xqb, 1);
    else
        q4_codes_bf16_kernel<float><<<grid_for(M * K / 8, dev), 256, 0, s>>>(static_cast<const float *>(x), M, K,
                                                                             scale_a, 0, eps, xqb, 1);
    q4_codes_bf16_kernel<float><<<grid_for(N * K / 8, dev), 256, 0, s>>>(w, N, K, scale_w, per_channel ? 1 : 0, eps,
                                                                         wqb, per_channel ? 2 : 1);
    if (per_channel) dout_steps_kernel<<<grid_for(M * N / 8, dev), 256, 0, s>>>(db, M, N, scale_w, eps, a2);
    if (cudaGetLastError() != cudaSuccess) return BQ_ERR_CUDA;
    // g [M][K] = dout [M][N] . wh [N][K]   (A K-major, B N-major)
    Bf16Args gg;
    gg.a = per_channel ? static_cast<const void *>(a2) : dout;
    gg.lda = per_channel ? 2 * N : N;
    gg.a_mn = false;
    gg.b = wqb;
    gg.ldb = K;
    gg.b_mn = true;
    gg.M = M;
    gg.N = K;
    gg.K = per_channel ? 2 * N : N;
    gg.scale = per_channel ? nullptr : steps + 1;
    gg.out = g;
    gg.ldo = K;
    bq_status st = launch_gemm_bf16(gg, s, dev);
    if (st != BQ_OK) return st;
    // dw [N][K] = s_a * dout^T [N][M] . xq [M][K]   (A M-major, B N-major)
    Bf16Args h;
    h.a = dout;
    h.lda = N;
    h.a_mn = true;
    h.b = xqb;
    h.ldb = K;
    h.b_mn = true;
    h.M = N;
    h.N = K;
    h.K = M;
    h.scale = steps;
    h.out = dw;
    h.ldo = K;
    st = launch_gemm_bf16(h, s, dev);
    if (st != BQ_OK) return st;
    const int pg = std::min(grid_for(M * K / 8, dev), kBwdPartMax);
    if (xt == BQ_BF16)
        w4a4_dx_kernel<__nv_bfloat16><<<pg, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), g, M, K, steps, dx, part);
    else
        w4a4_dx_kernel<float><<<pg, 256, 0, s>>>(static_cast<const float *>(x), g, M, K, steps, dx, part);
    w4a4_dscale_kernel<<<1, 32, 0, s>>>(part, pg, scale_a, eps, dscale_a);
    w4a4_dw_mask_kernel<<<grid_for(N * K / 8, dev), 256, 0, s>>>(w, N, K, scale_w, per_channel ? 1 : 0, eps, dw);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace bq
