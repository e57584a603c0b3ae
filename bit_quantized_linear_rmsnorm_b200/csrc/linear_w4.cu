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
#include <cudaTypedefs.h>

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
    static SmemOptIn opt_in;
    if (smem > 48 * 1024) {
        const cudaError_t e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), smem);
        if (e != cudaSuccess) return e;
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
// One-token decode kernel on the mma.sync tensor path: a single launch.  One
// CTA per SM takes a range of 8-row boxes of the packed weights; one thread of
// a producer warp streams them with TMA into a ring of box slots (a 3-D tensor
// view of the rows, {128 bytes, 8 rows, K/256 column pairs}, 128-byte
// swizzle: one copy moves 8 x K/2 bytes), and 16 computing warps consume them
// while the next boxes are in flight.  After the dependency wait the
// computing warps also split x into 23-bit planes (each warp keeps the plane
// fragments of its own spans in registers) and fold scale and activation
// scale into one pair of factors per (row, group).
//
// The planes use signed base-256 digits, X = 65536 P0 + 256 P1 + P2 with
// P0 in [-64, 64] and P1, P2 in [-128, 127] (|X| <= 2^22 - 1), so all three are s8 columns of
// one B operand: one m16n8k32 (u8 weights x s8 planes) gives D0, D1 and D2 of
// 16 rows in columns 0, 1, 2.
//
// Work unit = (two boxes = 16 rows, one 128-weight span).  Warp w takes the
// spans sp = w + 16 c (c < K / 2048).  MMA row g (0..7) is row sigma(g) of
// the first box and MMA row g + 8 row sigma(g) of the second, with
// sigma(g) = (g >> 1) | 4 (g & 1): the lanes that share a shared-memory phase
// then read rows whose swizzle differs in bit 2, i.e. opposite halves of the
// 128-byte line, so the fragment loads are free of bank conflicts.  Lane
// (g, t) reads words 4t .. 4t+3 of the span for both of its rows.  MMA pair e
// takes words 2e and 2e+1: the low nibbles (word & 0x0f0f0f0f) as one A
// operand and the high nibbles masked in place (word & 0xf0f0f0f0 = 16 q) as
// another, into two accumulators combined as C_lo + C_hi / 16 (exact).  The
// k-slots of lane t map to the elements of words 4t + 2e and 4t + 2e + 1,
// whose plane bytes (stored in the order 0,2,4,6,1,3,5,7 within each 8) are
// one 16-byte load: .x / .z feed the low-nibble MMA, .y / .w the high one.
//
//   out[n] = bias[n] + sum_g s[n,g] sx[g] T[n,g] - sum_g s[n,g] sx[g] z[n,g] sumX[g]
//
// with T[n,g] = sum_{k in g} q[n,k] X[k] = 65536 D0 + 256 D1 + D2.
// ---------------------------------------------------------------------------
constexpr int kW4Threads = 512;  // computing threads
constexpr int kW4Warps = kW4Threads / 32;
constexpr int kW4Block = kW4Threads + 32;  // + the producer warp
constexpr int kW4MaxRows = 128;
constexpr int kW4MaxSlots = 12;
constexpr int kW4MinSlots = 4;
constexpr int kW4XMax = 4194303;  // 2^22 - 1: |X| stays in the exact range of the rounding FMA

struct W4DecodeArgs {
    const float *x;
    const uint16_t *scales;
    const uint32_t *qzeros;
    const float *bias;
    float *out;
    int N, K, gs, nslots, rows_cap, nbox;  // nbox: 8-row boxes of the whole matrix
    uint32_t *status;
};

__device__ __forceinline__ int digit_s8(int v) { return ((v + 128) & 255) - 128; }

// float(v) for |v| < 2^22 on the FMA pipe: v added to the mantissa of 1.5 * 2^23
// gives 1.5 * 2^23 + v exactly, then the offset is subtracted (both exact).
// One 16-row x 128-weight inner product stays below 15 * 128 * 128 < 2^18.
__device__ __forceinline__ float exact_float(int v) { return __int_as_float(0x4B400000 + v) - 12582912.0f; }

// mbar_wait with the polling loop out of line (keeps the consumers' loop body
// small: the phase has usually completed by the time it is checked).
__device__ __noinline__ bool w4_wait_slow(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status) {
    return mbar_wait(bar, parity, abort, status, SITE_W4_STAGE);
}
__device__ __forceinline__ bool w4_wait(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status) {
    return mbar_try_wait(bar, parity) || w4_wait_slow(bar, parity, abort, status);
}

// Arrival on named barrier `id` without waiting (the producer waits on it).
__device__ __forceinline__ void w4_bar_arrive(uint32_t id, uint32_t threads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y, int32_t z,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// Shared-memory layout of the kernel (host and device), from a 1024-byte
// aligned base: the ring first (one box per slot, K/2 bytes per row).  The
// per-(row, group) factors are stored group-major with an odd row stride rs,
// so the lanes of one row block (consecutive rows) and the lanes of one row
// (consecutive groups) both hit distinct banks.
struct W4Layout {
    int G, zrow, rs;
    uint32_t slot, off_planes, off_sx, off_sumx, off_part, off_tab, off_zero, off_bars, total;
    __host__ __device__ static uint32_t a16(uint32_t v) { return (v + 15u) & ~15u; }
    __host__ __device__ W4Layout(int K, int gs, int nslots, int rows_cap) {
        G = K / gs;
        zrow = (G + 7) / 8;
        rs = (rows_cap + 8) | 1;  // (a row block may reach 8 rows past the last box)
        slot = 8u * static_cast<uint32_t>(K / 2);
        off_planes = slot * static_cast<uint32_t>(nslots);
        off_sx = a16(off_planes + 3u * K);
        off_sumx = off_sx + 4u * G;
        off_part = a16(off_sumx + 4u * G);
        off_tab = a16(off_part + 4u * rows_cap * kW4Warps);
        off_zero = a16(off_tab + 8u * rs * G);
        off_bars = (off_zero + 4u * rows_cap * zrow + 7u) & ~7u;
        total = off_bars + 16u * kW4MaxSlots + 1024u;  // + alignment slack of the base
    }
};

template <int SPW>  // spans per warp: K / 2048
__global__ void __launch_bounds__(kW4Block, 1) w4_decode_kernel(const __grid_constant__ CUtensorMap wmap,
                                                                const W4DecodeArgs p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ int s_abort;
    const int K = p.K, gs = p.gs, NS = p.nslots;
    const W4Layout L(K, gs, NS, p.rows_cap);
    const int G = L.G, zrow = L.zrow, rs = L.rs;
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t ring = smem_u32(smem);
    int8_t *planes = reinterpret_cast<int8_t *>(smem + L.off_planes);    // [3][K], order 0,2,4,6,1,3,5,7
    float *s_sx = reinterpret_cast<float *>(smem + L.off_sx);             // [G]
    float *s_sumx = reinterpret_cast<float *>(smem + L.off_sumx);         // [G]: sum of X
    float *s_part = reinterpret_cast<float *>(smem + L.off_part);         // [kW4Warps][rows_cap]
    float2 *s_tab = reinterpret_cast<float2 *>(smem + L.off_tab);         // [G][rs]: s sx, s sx z sumX
    uint32_t *s_zero = reinterpret_cast<uint32_t *>(smem + L.off_zero);   // [rows][zrow]
    const uint32_t fbar = smem_u32(smem + L.off_bars), ebar = fbar + 8u * kW4MaxSlots;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    // boxes [j0, j1) of the matrix; rows n0 .. n0 + rows - 1
    const int64_t b = blockIdx.x, Gc = gridDim.x;
    const int j0 = static_cast<int>((b * p.nbox) / Gc), j1 = static_cast<int>(((b + 1) * p.nbox) / Gc);
    const int nb = j1 - j0, n0 = 8 * j0, rows = min(8 * j1, p.N) - n0;

    if (t == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(fbar + 8 * s, 1);
            mbar_init(ebar + 8 * s, kW4Warps);
        }
        s_abort = 0;
        fence_mbarrier_init();
    }
    if (warp == kW4Warps && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&wmap) : "memory");
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();

    if (warp == kW4Warps) {  // producer: box i of this CTA into slot i % NS
        // the small loads of x, scales and zero-points enter the memory system
        // ahead of the weight stream (they head the computing warps' critical path)
        named_bar_sync(2, kW4Block);
        if (lane == 0) {
            int i = 0;
            for (; i < nb; ++i) {
                const int slot = i % NS;
                if (i >= NS && !mbar_wait(ebar + 8 * slot, ((i / NS) - 1) & 1, &s_abort, p.status, SITE_W4_STAGE))
                    break;
                mbar_arrive_expect_tx(fbar + 8 * slot, L.slot);
                tma_load_3d(ring + static_cast<uint32_t>(slot) * L.slot, &wmap, 0, n0 + 8 * i, 0, fbar + 8 * slot);
            }
            // the copies in flight land before the CTA exits, whatever happened
            for (int k = max(0, i - NS); k < i; ++k)
                mbar_wait_timed(fbar + 8 * (k % NS), (k / NS) & 1, p.status, SITE_W4_DRAIN);
        }
        return;
    }

    // activations, zero-points and scales (the weight stream is already running)
    const int ns = rows * G, nz = rows * zrow;
    const int sgo = n0 * G, zgo = n0 * zrow;
    float4 xv[SPW];  // EPT = K / 512 = 4 SPW elements of x per thread
    {
        const float4 *x4 = reinterpret_cast<const float4 *>(p.x) + static_cast<int64_t>(t) * SPW;
#pragma unroll
        for (int j = 0; j < SPW; ++j) xv[j] = __ldg(x4 + j);
    }
    uint16_t sv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = t + j * kW4Threads;
        sv[j] = i < ns ? __ldg(p.scales + sgo + i) : static_cast<uint16_t>(0);
    }
    // the bias of row t (rows <= 128 < threads), added at the very end
    const float bias_t = p.bias && t < rows ? __ldg(p.bias + n0 + t) : 0.0f;
    {
        uint32_t zv[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = t + j * kW4Threads;
            zv[j] = i < nz ? __ldg(p.qzeros + zgo + i) : 0u;
        }
        w4_bar_arrive(2, kW4Block);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = t + j * kW4Threads;
            if (i < nz) s_zero[i] = zv[j];
        }
    }

    // activation planes: thread t splits elements EPT t .. EPT t + EPT - 1 (a
    // group spans TPG = gs / EPT threads).  X = rne(x / sx) with
    // sx = max|x| / (2^22 - 1) per group, x / sx taken as x * (1 / sx) and
    // rounded by one FMA that adds 1.5 * 2^23 (exact while |x / sx| <= 2^22):
    // at most one more unit of error than the exact quotient, on the FMA pipe.
    // The digits are bytes of X: P2 = X (mod 256) as a signed byte,
    // X1 = (X + 128) >> 8, P1 = X1 (mod 256), P0 = (X1 + 128) >> 8.
    {
        constexpr int EPT = 4 * SPW;
        const int TPG = gs / EPT;
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < SPW; ++j)
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(xv[j].x), fabsf(xv[j].y)), fmaxf(fabsf(xv[j].z), fabsf(xv[j].w))));
        for (int o = TPG / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sx = __fdiv_rn(amax, static_cast<float>(kW4XMax));
        const float inv = amax > 0.f ? __fdiv_rn(1.0f, sx) : 0.f;
        int sum = 0;
        int xd[3][EPT];  // per element: X, X1, X0 (their low bytes are P2, P1, P0)
#pragma unroll
        for (int j = 0; j < SPW; ++j) {
            const float e4[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                int X = __float_as_int(fmaf(e4[u], inv, 12582912.0f)) - 0x4B400000;
                X = max(-kW4XMax, min(kW4XMax, X));
                sum += X;
                const int X1 = (X + 128) >> 8;
                xd[2][4 * j + u] = X;
                xd[1][4 * j + u] = X1;
                xd[0][4 * j + u] = (X1 + 128) >> 8;
            }
        }
        // low bytes of four values -> one word
        auto pack4 = [](int a, int b, int c, int d) -> uint32_t {
            return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
        };
        if (EPT >= 8) {  // whole 8-chunks: even elements (positions 0..3), odd (4..7)
#pragma unroll
            for (int q = 0; q < 3; ++q)
#pragma unroll
                for (int h = 0; h < EPT / 8; ++h) {
                    const int *v = xd[q] + 8 * h;
                    *reinterpret_cast<uint2 *>(planes + q * K + EPT * t + 8 * h) =
                        make_uint2(pack4(v[0], v[2], v[4], v[6]), pack4(v[1], v[3], v[5], v[7]));
                }
        } else {  // half a chunk: elements 0..3 or 4..7 of it, at positions hb, hb + 1, 4 + hb, 5 + hb
            const int base = (EPT * t) & ~7, hb = ((EPT * t) & 7) ? 2 : 0;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                planes[q * K + base + hb] = static_cast<int8_t>(xd[q][0]);
                planes[q * K + base + hb + 1] = static_cast<int8_t>(xd[q][2]);
                planes[q * K + base + 4 + hb] = static_cast<int8_t>(xd[q][1]);
                planes[q * K + base + 4 + hb + 1] = static_cast<int8_t>(xd[q][3]);
            }
        }
        for (int o = TPG / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (t % TPG == 0) {
            s_sx[(EPT * t) / gs] = sx;
            s_sumx[(EPT * t) / gs] = static_cast<float>(sum);
        }
    }
    named_bar_sync(1, kW4Threads);

    // per (row, group): s sx and s sx z sumX (G is a power of two)
    const int g_shift = __ffs(G) - 1;
    auto tab_items = [&](int base, const uint16_t(&v)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + t + j * kW4Threads;
            if (i < ns) {
                const int r = i >> g_shift, grp = i & (G - 1);
                const float fs = __fmul_rn(__half2float(__ushort_as_half(v[j])), s_sx[grp]);
                const float z = exact_float(static_cast<int>((s_zero[r * zrow + grp / 8] >> (4 * (grp % 8))) & 15u));
                s_tab[grp * rs + r] = make_float2(fs, __fmul_rn(__fmul_rn(fs, z), s_sumx[grp]));
            }
        }
    };
    tab_items(0, sv);
    for (int base = 8 * kW4Threads; base < ns; base += 8 * kW4Threads) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + t + j * kW4Threads;
            sv[j] = i < ns ? __ldg(p.scales + sgo + i) : static_cast<uint16_t>(0);
        }
        tab_items(base, sv);
    }
    // this warp's plane fragments (the same for every row block)
    uint4 bx[SPW][2];
#pragma unroll
    for (int c = 0; c < SPW; ++c) {
        const int sp = warp + kW4Warps * c;
#pragma unroll
        for (int e = 0; e < 2; ++e)
            bx[c][e] = gq < 3 ? *reinterpret_cast<const uint4 *>(planes + gq * K + 128 * sp + 32 * tq + 16 * e)
                              : make_uint4(0u, 0u, 0u, 0u);
    }
    named_bar_sync(1, kW4Threads);

    // C columns: lane t = 0 holds D0, D1 of MMA rows g and g + 8, lane t = 1
    // holds D2 (column 2) of both.  Each accumulates its share of
    // s sx T = s sx (65536 D0 + 256 D1) + s sx D2 (lane t = 0 also subtracts
    // the zero-point term once per group); the two shares meet once per block.
    const int SPG = gs / 128, spg_shift = __ffs(SPG) - 1;  // spans per group (a power of two)
    const int sg = (gq >> 1) | ((gq & 1) << 2);             // sigma(g): row of the box
    // byte offset of this lane's 16 bytes of span sp within a box: column pair
    // sp / 2 (1 KB each), row sg (128 bytes), 16-byte chunk (4 (sp & 1) + t) ^ sg
    auto frag_off = [&](int sp) -> uint32_t {
        return static_cast<uint32_t>((sp >> 1) * 1024 + sg * 128 + ((((sp & 1) << 2) + tq) ^ sg) * 16);
    };
    const int nrb = (nb + 1) / 2;
    int s0 = 0;        // slot of box 2 rb
    uint32_t ph0 = 0;  // and the parity of its phase
    for (int rb = 0; rb < nrb; ++rb) {
        const bool has1 = 2 * rb + 1 < nb;
        const int s1 = s0 + 1 == NS ? 0 : s0 + 1;
        const uint32_t ph1 = s0 + 1 == NS ? ph0 ^ 1u : ph0;
        bool ok = w4_wait(fbar + 8 * s0, ph0, &s_abort, p.status);
        if (has1) ok = ok && w4_wait(fbar + 8 * s1, ph1, &s_abort, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            const uint32_t b0 = ring + static_cast<uint32_t>(s0) * L.slot;
            const uint32_t b1 = ring + static_cast<uint32_t>(s1) * L.slot;
            const int r0 = 16 * rb + sg, r1 = r0 + 8;  // this lane's rows (MMA rows g, g + 8)
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int c = 0; c < SPW; ++c) {
                const int sp = warp + kW4Warps * c;
                const uint32_t off = frag_off(sp);
                // (without a second box, the other slot's stale bytes only reach rows
                // past the end, whose sums are never stored)
                uint4 wa, wb;
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wa.x), "=r"(wa.y), "=r"(wa.z), "=r"(wa.w) : "r"(b0 + off));
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wb.x), "=r"(wb.y), "=r"(wb.z), "=r"(wb.w) : "r"(b1 + off));
                int clo[4] = {0, 0, 0, 0}, chi[4] = {0, 0, 0, 0};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t a0 = e ? wa.z : wa.x, a2 = e ? wa.w : wa.y;
                    const uint32_t a1 = e ? wb.z : wb.x, a3 = e ? wb.w : wb.y;
                    const uint32_t lo[4] = {a0 & 0x0f0f0f0fu, a1 & 0x0f0f0f0fu, a2 & 0x0f0f0f0fu, a3 & 0x0f0f0f0fu};
                    const uint32_t hi[4] = {a0 & 0xf0f0f0f0u, a1 & 0xf0f0f0f0u, a2 & 0xf0f0f0f0u, a3 & 0xf0f0f0f0u};
                    mma_u8s8_16832(clo, lo, bx[c][e].x, bx[c][e].z);
                    mma_u8s8_16832(chi, hi, bx[c][e].y, bx[c][e].w);
                }
                // every lane takes the same steps (no divergence): lane t = 0 adds
                // 65536 D0 + 256 D1 and subtracts the zero-point term once per group,
                // lane t = 1 adds D2; lanes t = 2, 3 hold zero columns
                const int grp = sp >> spg_shift;
                const float2 f0 = s_tab[grp * rs + r0], f1 = s_tab[grp * rs + r1];
                const float zt = tq == 0 && (sp & (SPG - 1)) == 0 ? 1.0f : 0.0f;
                const float d0 = exact_float(clo[0] + (chi[0] >> 4)), d1 = exact_float(clo[1] + (chi[1] >> 4));
                const float d2 = exact_float(clo[2] + (chi[2] >> 4)), d3 = exact_float(clo[3] + (chi[3] >> 4));
                const float u0 = tq == 0 ? fmaf(65536.0f, d0, 256.0f * d1) : d0;
                const float u1 = tq == 0 ? fmaf(65536.0f, d2, 256.0f * d3) : d2;
                acc0 = fmaf(f0.x, u0, fmaf(-zt, f0.y, acc0));
                acc1 = fmaf(f1.x, u1, fmaf(-zt, f1.y, acc1));
            }
            acc0 += __shfl_down_sync(0xffffffffu, acc0, 1);
            acc1 += __shfl_down_sync(0xffffffffu, acc1, 1);
            if (tq == 0) {
                if (r0 < rows) s_part[warp * p.rows_cap + r0] = acc0;
                if (r1 < rows) s_part[warp * p.rows_cap + r1] = acc1;
            }
        }
        __syncwarp();
        if (lane == 0) {  // this warp is done with both slots
            mbar_arrive(ebar + 8 * s0);
            if (has1) mbar_arrive(ebar + 8 * s1);
        }
        s0 = s1 + 1 == NS ? 0 : s1 + 1;
        ph0 = s1 + 1 == NS ? ph1 ^ 1u : ph1;
    }
    named_bar_sync(1, kW4Threads);
    if (t < rows) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kW4Warps; ++w) acc += s_part[w * p.rows_cap + t];
        p.out[n0 + t] = bias_t + acc;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 w4_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

int w4_boxes(int64_t N) { return static_cast<int>((N + 7) / 8); }

int w4_rows_cap(int64_t N, const DevInfo &dev) {
    const int64_t nb = w4_boxes(N), Gc = std::min<int64_t>(nb, dev.num_sms);
    return static_cast<int>(8 * ((nb + Gc - 1) / Gc));
}

int w4_decode_slots(int K, int gs, int rows_cap, const DevInfo &dev) {
    const W4Layout L0(K, gs, 0, rows_cap);
    const int64_t room = static_cast<int64_t>(dev.max_smem_optin) - 1024 - L0.total;  // (static shared memory)
    const int64_t n = std::min<int64_t>(kW4MaxSlots, room / L0.slot);
    return n < kW4MinSlots ? 0 : static_cast<int>(n);
}

bool w4_decode_supported(int64_t M, int64_t N, int64_t K, int64_t gs, const DevInfo &dev) {
    if (M != 1 || K % 2048 != 0 || K > 8192 || gs % 128 != 0 || K % gs != 0 || (gs & (gs - 1)) != 0) return false;
    if (gs > K / 16) return false;  // a group spans at most one warp in the split of x
    if (w4_rows_cap(N, dev) > kW4MaxRows || w4_encode_fn() == nullptr) return false;
    return w4_decode_slots(static_cast<int>(K), static_cast<int>(gs), w4_rows_cap(N, dev), dev) > 0;
}

cudaError_t launch_w4_decode(const float *x, int64_t K, const uint32_t *qweight, const uint16_t *scales,
                             const uint32_t *qzeros, const float *bias, int64_t N, int64_t gs, float *out,
                             cudaStream_t s, const DevInfo &dev) {
    // the packed rows as {128-byte column pairs of 16 u64, rows, column pairs}
    CUtensorMap map;
    {
        const cuuint64_t dims[3] = {16, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K / 256)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2), 128};
        const cuuint32_t box[3] = {16, 8, static_cast<cuuint32_t>(K / 256)};
        const cuuint32_t estr[3] = {1, 1, 1};
        const CUresult r = w4_encode_fn()(&map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<uint32_t *>(qweight),
                                          dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    W4DecodeArgs a;
    a.x = x;
    a.scales = scales;
    a.qzeros = qzeros;
    a.bias = bias;
    a.out = out;
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.gs = static_cast<int>(gs);
    a.rows_cap = w4_rows_cap(N, dev);
    a.nslots = w4_decode_slots(a.K, a.gs, a.rows_cap, dev);
    a.nbox = w4_boxes(N);
    a.status = dev.status;
    const int smem = static_cast<int>(W4Layout(a.K, a.gs, a.nslots, a.rows_cap).total);
    auto kern = K == 2048 ? w4_decode_kernel<1> : K == 4096 ? w4_decode_kernel<2> : w4_decode_kernel<4>;
    static SmemOptIn opt_in[3];
    if (smem > 48 * 1024) {
        const cudaError_t e = smem_opt_in(opt_in[K == 2048 ? 0 : K == 4096 ? 1 : 2], dev,
                                          reinterpret_cast<const void *>(kern), static_cast<size_t>(smem));
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(a.nbox, dev.num_sms)));
    cfg.blockDim = dim3(kW4Block);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, map, a);
}

}  // namespace

size_t linear_w4_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group_size) {
    const int64_t G = K / group_size;
    const size_t planes = align256(static_cast<size_t>(3 * M * K)) + align256(static_cast<size_t>(M * G) * 4) +
                          align256(static_cast<size_t>(M * G) * 4);
    // room for the tensor-core path whenever it may be taken (it depends on the device only through the grid)
    const bool tc = M >= 2 && M <= 32 && K % 1024 == 0 && group_size % 128 == 0 && K % group_size == 0;
    return tc ? std::max(planes, w4_tc_workspace_bytes(N, K)) : planes;
}

cudaError_t launch_linear_w4(const float *x, int64_t M, int64_t K, const uint32_t *qweight, const uint16_t *scales,
                             const uint32_t *qzeros, const float *bias, int64_t N, int64_t group_size, float *out,
                             void *ws_ptr, cudaStream_t s, const DevInfo &dev) {
    if (w4_decode_supported(M, N, K, group_size, dev) && reinterpret_cast<uintptr_t>(qweight) % 16 == 0 &&
        reinterpret_cast<uintptr_t>(x) % 16 == 0)
        return launch_w4_decode(x, K, qweight, scales, qzeros, bias, N, group_size, out, s, dev);
    if (w4_tc_supported(M, N, K, group_size, dev) && reinterpret_cast<uintptr_t>(qweight) % 16 == 0 &&
        reinterpret_cast<uintptr_t>(x) % 16 == 0)
        return launch_w4_tc(x, M, K, qweight, scales, qzeros, bias, N, group_size, out, ws_ptr, s, dev);
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
