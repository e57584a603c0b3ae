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

#include <algorithm>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "quant_common.cuh"

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


// ---------------------------------------------------------------------------
// One-token decode kernel: a single launch that splits x into its 24-bit
// planes in shared memory (every CTA, for all of K) and streams the packed
// weights with a deep per-thread load pipeline.
//
// One CTA per SM (512 threads), CTA b owns rows [b N / G, (b+1) N / G).  With
// CQ = K / 32 chunk columns (a chunk = 4 packed words = 32 weights, inside one
// group), thread t always works on chunk column q = t % CQ, so the 96 bytes of
// activation planes its chunks need stay in registers; its rows are
// rg + RG i (rg = t / CQ, RG = 512 / CQ).  The chunks of a thread are loaded
// kW4Ahead ahead of their use in a fully unrolled loop, so about 128 KB per
// SM is in flight.  Per chunk: D_p = sum q * P_p by dp4a, then
//   v = s[n,g] * sx[g] * (65536 D0 + 256 D1 + D2)  (- s z sx sumX once per group)
// and the partial row sums of four chunks are reduced across the warp at once
// (the lanes of a warp share each chunk's row when CQ >= 32).
// ---------------------------------------------------------------------------
constexpr int kW4Threads = 512;
constexpr int kW4Warps = kW4Threads / 32;
constexpr int kW4Chunks = 28;   // chunks per thread (rows per thread)
constexpr int kW4Ahead = 16;    // loads in flight per thread
constexpr int kW4MaxRows = 224;

__device__ __forceinline__ float warp_fsum4(float v0, float v1, float v2, float v3) {
    const int lane = threadIdx.x & 31;
    const bool h16 = lane & 16, h8 = lane & 8;
    float k0 = h16 ? v2 : v0, k1 = h16 ? v3 : v1;
    k0 += __shfl_xor_sync(0xffffffffu, h16 ? v0 : v2, 16);
    k1 += __shfl_xor_sync(0xffffffffu, h16 ? v1 : v3, 16);
    float k = h8 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;
}

struct W4DecodeArgs {
    const float *x;
    const uint32_t *qweight;
    const uint16_t *scales;
    const uint32_t *qzeros;
    const float *bias;
    float *out;
    int N, K, gs;
};

__global__ void __launch_bounds__(kW4Threads, 1) w4_decode_kernel(const W4DecodeArgs p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int K = p.K, gs = p.gs, G = K / gs, CQ = K / 32, RG = kW4Threads / CQ;
    int8_t *planes = reinterpret_cast<int8_t *>(smem);                  // [3][K], perm8 order
    float *s_sx = reinterpret_cast<float *>(smem + 3 * K);              // [G]
    int *s_sumx = reinterpret_cast<int *>(s_sx + G);                    // [G]
    float *s_part = reinterpret_cast<float *>(s_sumx + G);              // [kW4MaxRows][4]
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t b = blockIdx.x, Gc = gridDim.x;
    const int n0 = static_cast<int>((b * p.N) / Gc), rows = static_cast<int>(((b + 1) * p.N) / Gc) - n0;
    const int q = t % CQ, rg = t / CQ;
    const int g = q / (gs / 32);                  // group of this chunk column
    const bool zlead = (q % (gs / 32)) == 0;      // first chunk of its group: adds the zero-point term
    const int wrow = K / 8, zrow = (G + 7) / 8;
    const uint4 *wq = reinterpret_cast<const uint4 *>(p.qweight + static_cast<int64_t>(n0) * wrow) + q;

    pdl_launch_dependents();
    pdl_wait();

    // weight pipeline head: the first kW4Ahead chunks of this thread
    uint4 w[kW4Ahead];
    uint16_t sc[kW4Ahead];
    uint32_t zw[kW4Ahead];
#pragma unroll
    for (int i = 0; i < kW4Ahead; ++i) {
        const int r = rg + RG * i;
        const bool in = r < rows;
        w[i] = in ? __ldcs(wq + static_cast<int64_t>(r) * (wrow / 4)) : make_uint4(0u, 0u, 0u, 0u);
        sc[i] = in ? __ldg(p.scales + static_cast<int64_t>(n0 + r) * G + g) : static_cast<uint16_t>(0);
        zw[i] = (in && zlead) ? __ldg(p.qzeros + static_cast<int64_t>(n0 + r) * zrow + g / 8) : 0u;
    }

    // scales and zero-points of this CTA's rows -> shared memory (loads batched)
    uint16_t *s_scale = reinterpret_cast<uint16_t *>(s_part + kW4MaxRows * (CQ / 32));   // [rows][G]
    uint32_t *s_zero = reinterpret_cast<uint32_t *>(s_scale + ((kW4MaxRows * G + 1) & ~1));  // [rows][zrow]
    {
        const int ns = rows * G, nz = rows * zrow;
        const uint16_t *sg = p.scales + static_cast<int64_t>(n0) * G;
        const uint32_t *zg = p.qzeros + static_cast<int64_t>(n0) * zrow;
        for (int base = 0; base < ns; base += 8 * kW4Threads) {
            uint16_t v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = base + t + j * kW4Threads;
                v[j] = i < ns ? __ldg(sg + i) : static_cast<uint16_t>(0);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = base + t + j * kW4Threads;
                if (i < ns) s_scale[i] = v[j];
            }
        }
        for (int i = t; i < nz; i += kW4Threads) s_zero[i] = __ldg(zg + i);
    }

    // activation planes: thread t splits elements EPT t .. EPT t + EPT - 1
    // (EPT = K / 512, one group spans TPG = gs / EPT threads).  X = rne(x / sx),
    // sx = max|x| / (2^23 - 1) per group, x / sx taken as x * (1 / sx): at
    // most one more unit of error than the exact quotient.
    {
        const int EPT = K / kW4Threads, nv = EPT / 4, TPG = gs / EPT;
        const float4 *x4 = reinterpret_cast<const float4 *>(p.x) + static_cast<int64_t>(t) * nv;
        float4 xv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) xv[j] = j < nv ? __ldg(x4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(xv[j].x), fabsf(xv[j].y)), fmaxf(fabsf(xv[j].z), fabsf(xv[j].w))));
        for (int o = TPG / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sx = __fdiv_rn(amax, 8388607.0f);
        const float inv = amax > 0.f ? __fdiv_rn(1.0f, sx) : 0.f;
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j < nv) {
                const float e4[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int X = __float2int_rn(__fmul_rn(e4[u], inv));
                    X = max(-8388607, min(8388607, X));
                    sum += X;
                    const int k = EPT * t + 4 * j + u, jj = k & 7;
                    const int pos = (k & ~7) + ((jj & 1) ? 4 + (jj >> 1) : (jj >> 1));
                    planes[pos] = static_cast<int8_t>(X >> 16);
                    planes[K + pos] = static_cast<int8_t>((X >> 8) & 255);
                    planes[2 * K + pos] = static_cast<int8_t>(X & 255);
                }
            }
        }
        for (int o = TPG / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (t % TPG == 0) {
            s_sx[(EPT * t) / gs] = sx;
            s_sumx[(EPT * t) / gs] = sum;
        }
    }
    __syncthreads();
    uint4 xp[3][2];
#pragma unroll
    for (int pl = 0; pl < 3; ++pl)
#pragma unroll
        for (int h = 0; h < 2; ++h) xp[pl][h] = *reinterpret_cast<const uint4 *>(planes + pl * K + 32 * q + 16 * h);
    const float sxg = s_sx[g];
    const float zterm = sxg * static_cast<float>(s_sumx[g]);

    float v[4];
#pragma unroll
    for (int i = 0; i < kW4Chunks; ++i) {
        const int slot = i % kW4Ahead;
        const int r = rg + RG * i;
        float val = 0.f;
        if (r < rows) {
            const uint32_t wd[4] = {w[slot].x, w[slot].y, w[slot].z, w[slot].w};
            int d0 = 0;
            uint32_t d1 = 0u, d2 = 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // word j: elements 8 j .. 8 j + 7 of the chunk
                const uint32_t lo = wd[j] & 0x0f0f0f0fu, hi = (wd[j] >> 4) & 0x0f0f0f0fu;
                const uint4 &a = xp[0][j >> 1], &bq = xp[1][j >> 1], &c = xp[2][j >> 1];
                const uint32_t p0l = (j & 1) ? a.z : a.x, p0h = (j & 1) ? a.w : a.y;
                const uint32_t p1l = (j & 1) ? bq.z : bq.x, p1h = (j & 1) ? bq.w : bq.y;
                const uint32_t p2l = (j & 1) ? c.z : c.x, p2h = (j & 1) ? c.w : c.y;
                d0 = dp4a_us(hi, p0h, dp4a_us(lo, p0l, d0));
                d1 = dp4a_uu(hi, p1h, dp4a_uu(lo, p1l, d1));
                d2 = dp4a_uu(hi, p2h, dp4a_uu(lo, p2l, d2));
            }
            const float T = fmaf(65536.0f, static_cast<float>(d0),
                                 fmaf(256.0f, static_cast<float>(d1), static_cast<float>(d2)));
            const float s = __half2float(__ushort_as_half(s_scale[r * G + g]));
            val = __fmul_rn(__fmul_rn(s, sxg), T);
            if (zlead) {
                const float z = static_cast<float>((s_zero[r * zrow + g / 8] >> (4 * (g % 8))) & 15u);
                val = fmaf(-__fmul_rn(s, z), zterm, val);
            }
        }
        // refill the slot
        if (i + kW4Ahead < kW4Chunks) {
            const int rn = rg + RG * (i + kW4Ahead);
            w[slot] = rn < rows ? __ldcs(wq + static_cast<int64_t>(rn) * (wrow / 4)) : make_uint4(0u, 0u, 0u, 0u);
        }
        v[i & 3] = val;
        if ((i & 3) == 3) {
            const float k = warp_fsum4(v[0], v[1], v[2], v[3]);
            const int rr = rg + RG * (i - 3 + (lane >> 3));
            if ((lane & 7) == 0 && rr < rows) s_part[rr * (CQ / 32) + q / 32] = k;
        }
    }
    __syncthreads();
    for (int r = t; r < rows; r += kW4Threads) {
        float acc = 0.f;
        for (int j = 0; j < CQ / 32; ++j) acc += s_part[r * (CQ / 32) + j];
        p.out[n0 + r] = (p.bias ? __ldg(p.bias + n0 + r) : 0.0f) + acc;
    }
}

size_t w4_decode_smem(int K, int gs) {
    const int G = K / gs, CQ = K / 32, zrow = (G + 7) / 8;
    size_t b = static_cast<size_t>(3 * K) + 8u * G + 4u * kW4MaxRows * (CQ / 32);
    b += 2u * ((kW4MaxRows * G + 1) & ~1) + 4u * kW4MaxRows * zrow;
    return b;
}

bool w4_decode_supported(int64_t M, int64_t N, int64_t K, int64_t gs, const DevInfo &dev) {
    if (M != 1 || gs % 32 != 0 || K % gs != 0 || K < 2048 || K > 8192 || (gs & (gs - 1)) != 0) return false;
    if (gs / (K / kW4Threads) > 32) return false;  // a group spans at most one warp in the split
    const int64_t CQ = K / 32;
    if (kW4Threads % CQ != 0) return false;
    const int64_t RG = kW4Threads / CQ, Gc = std::min<int64_t>(N, dev.num_sms);
    const int64_t rb = (N + Gc - 1) / Gc;
    if (rb > kW4Chunks * RG || rb > kW4MaxRows) return false;
    return w4_decode_smem(static_cast<int>(K), static_cast<int>(gs)) <= dev.max_smem_optin;
}

cudaError_t launch_w4_decode(const float *x, int64_t K, const uint32_t *qweight, const uint16_t *scales,
                             const uint32_t *qzeros, const float *bias, int64_t N, int64_t gs, float *out,
                             cudaStream_t s, const DevInfo &dev) {
    W4DecodeArgs a;
    a.x = x;
    a.qweight = qweight;
    a.scales = scales;
    a.qzeros = qzeros;
    a.bias = bias;
    a.out = out;
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.gs = static_cast<int>(gs);
    const int smem = static_cast<int>(w4_decode_smem(a.K, a.gs));
    static int attr_smem[64] = {};
    if (smem > 48 * 1024 && smem > attr_smem[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(w4_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_smem[dev.device] = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(N, dev.num_sms)));
    cfg.blockDim = dim3(kW4Threads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4_decode_kernel, a);
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
    if (w4_decode_supported(M, N, K, group_size, dev) && reinterpret_cast<uintptr_t>(qweight) % 16 == 0 &&
        reinterpret_cast<uintptr_t>(x) % 16 == 0)
        return launch_w4_decode(x, K, qweight, scales, qzeros, bias, N, group_size, out, s, dev);
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
