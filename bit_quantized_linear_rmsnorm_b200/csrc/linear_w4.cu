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
// One-token decode kernel on the mma.sync tensor path: a single launch that
// splits x into 24-bit planes in shared memory (every CTA, for all of K) and
// streams the CTA's packed weight rows into a ring of 16-row stages.  One
// extra warp only issues those copies (16-byte cp.async through the load /
// store path, measured faster per SM than bulk copies for this stream), and
// refills a slot as soon as the 16 computing warps have released it (full /
// empty mbarriers per slot), so the HBM stream keeps going while the other
// warps split x and compute.
//
// The planes use signed base-256 digits, X = 65536 P0 + 256 P1 + P2 with
// P0, P1, P2 in [-128, 127] (|X| <= 8355711), so all three are s8 columns of
// one B operand: one m16n8k32 (u8 weights x s8 planes) gives D0, D1 and D2 of
// 16 rows in columns 0, 1, 2.
//
// A stage holds 16 rows at a pitch of K/2 + 64 bytes (the extra 64 bytes put
// rows g and g + 1 in different bank groups).  Warp w takes the 128-weight
// spans sp = w + 16 c (c < K / 2048) of every stage (one group each when
// gs % 128 == 0).  Lane (g, t) reads words 4t .. 4t+3 of the span for rows g
// and g + 8.  MMA pair e takes words 2e and 2e+1: the low nibbles
// (word & 0x0f0f0f0f) as one A operand and the high nibbles masked in place
// (word & 0xf0f0f0f0 = 16 q) as another, into two accumulators combined as
// C_lo + C_hi / 16 (exact).  The k-slots of lane t map to the elements of words
// 4t + 2e and 4t + 2e + 1, whose plane bytes (stored in the order 0,2,4,6,1,3,5,7
// within each 8) are one 16-byte load: .x / .z feed the low-nibble MMA, .y / .w
// the high-nibble one.
// ---------------------------------------------------------------------------
constexpr int kW4Threads = 512;                 // computing threads
constexpr int kW4Warps = kW4Threads / 32;
constexpr int kW4Streamers = 8;                  // warps that only stream the weights
constexpr int kW4Block = kW4Threads + 32 * kW4Streamers;
constexpr int kW4MaxRows = 128;
constexpr int kW4MaxStages = 8;
constexpr int kW4XMax = 8355711;  // 127 * (65536 + 256 + 1)

struct W4DecodeArgs {
    const float *x;
    const uint32_t *qweight;
    const uint16_t *scales;
    const uint32_t *qzeros;
    const float *bias;
    float *out;
    int N, K, gs, nstg, rows_cap;
    uint32_t *status;
};

__device__ __forceinline__ int digit_s8(int v) { return ((v + 128) & 255) - 128; }

// Shared-memory layout of the kernel (host and device).
struct W4Layout {
    int G, zrow, pitch;
    uint32_t off_sx, off_sumx, off_part, off_tab, off_zero, off_bars, off_ring, total;
    __host__ __device__ static uint32_t a16(uint32_t v) { return (v + 15u) & ~15u; }
    __host__ __device__ W4Layout(int K, int gs, int nstg, int rows_cap) {
        G = K / gs;
        zrow = (G + 7) / 8;
        pitch = K / 2 + 64;
        off_sx = a16(3u * K);
        off_sumx = off_sx + 4u * G;
        off_part = a16(off_sumx + 4u * G);
        off_tab = a16(off_part + 4u * rows_cap * kW4Warps);
        off_zero = a16(off_tab + 8u * rows_cap * G);
        off_bars = a16(off_zero + 4u * rows_cap * zrow);
        off_ring = (off_bars + 16u * kW4MaxStages + 127u) & ~127u;
        total = off_ring + static_cast<uint32_t>(nstg) * 16u * pitch;
    }
};

template <int SPW>  // spans per warp and stage: K / 2048
__global__ void __launch_bounds__(kW4Block, 1) w4_decode_kernel(const W4DecodeArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_abort;
    const int K = p.K, gs = p.gs, nstg = p.nstg;
    const W4Layout L(K, gs, nstg, p.rows_cap);
    const int G = L.G, zrow = L.zrow, pitch = L.pitch;
    int8_t *planes = reinterpret_cast<int8_t *>(smem);                  // [3][K], order 0,2,4,6,1,3,5,7
    float *s_sx = reinterpret_cast<float *>(smem + L.off_sx);           // [G]
    int *s_sumx = reinterpret_cast<int *>(smem + L.off_sumx);           // [G]
    float *s_part = reinterpret_cast<float *>(smem + L.off_part);       // [rows][kW4Warps]
    float2 *s_tab = reinterpret_cast<float2 *>(smem + L.off_tab);       // [rows][G]: s sx, s sx z sumX
    uint32_t *s_zero = reinterpret_cast<uint32_t *>(smem + L.off_zero);    // [rows][zrow]
    // full[s] at bars + 8 s (one arrival + the copy bytes), empty[s] at bars + 8 (kW4MaxStages + s)
    const uint32_t bars = smem_u32(smem + L.off_bars), ring = smem_u32(smem + L.off_ring);
    const uint32_t ebars = bars + 8u * kW4MaxStages;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int64_t b = blockIdx.x, Gc = gridDim.x;
    const int n0 = static_cast<int>((b * p.N) / Gc), rows = static_cast<int>(((b + 1) * p.N) / Gc) - n0;
    const int nst = (rows + 15) / 16;  // stages of this CTA
    const uint32_t rowb = static_cast<uint32_t>(K / 2);  // packed bytes per row
    const uint8_t *wsrc = reinterpret_cast<const uint8_t *>(p.qweight) + static_cast<int64_t>(n0) * rowb;

    if (t == 0) {
        for (int s = 0; s < nstg; ++s) {
            mbar_init(bars + 8 * s, 32 * kW4Streamers);  // one arrival per streaming lane
            mbar_init(ebars + 8 * s, kW4Warps);
        }
        s_abort = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();

    // the streaming warp copies stage s (rows 16 s .. 16 s + 15) into ring slot
    // s % nstg, each lane then arriving on the slot's full barrier once its
    // own copies have landed
    const int ppr_shift = __ffs(static_cast<int>(rowb / 16)) - 1;  // 16-byte pieces per row (a power of two)
    const int sl = t - kW4Threads;  // lane among the streaming warps
    auto issue = [&](int s) {
        const int slot = s % nstg, r0 = 16 * s, nr = min(16, rows - r0);
        const uint32_t dst = ring + static_cast<uint32_t>(slot) * 16u * pitch;
        const int npc = nr << ppr_shift;
        for (int i = sl; i < npc; i += 32 * kW4Streamers) {
            const int j = i >> ppr_shift, c = i & ((1 << ppr_shift) - 1);
            cp_async_16(dst + static_cast<uint32_t>(j) * pitch + 16u * c,
                        wsrc + static_cast<int64_t>(r0 + j) * rowb + 16 * c, 16u);
        }
        cp_async_mbar_arrive_noinc(bars + 8 * slot);
    };
    if (warp >= kW4Warps) {  // the streaming warps
        int s = 0;
        for (; s < nst; ++s) {
            const int slot = s % nstg;
            if (s >= nstg) {  // the slot's previous stage must be released by every computing warp
                bool ok = mbar_wait(ebars + 8 * slot, ((s / nstg) - 1) & 1, &s_abort, p.status, SITE_W4_STAGE);
                if (!__all_sync(0xffffffffu, ok)) break;
            }
            issue(s);
        }
        cp_async_wait_all();  // (the copies land before the warp exits, whatever happened)
        return;
    }

    // activations, scales and zero-points (the weight stream is already running)
    const int EPT = K / kW4Threads, nv = EPT / 4, TPG = gs / EPT;
    float4 xv[4];
    {
        const float4 *x4 = reinterpret_cast<const float4 *>(p.x) + static_cast<int64_t>(t) * nv;
#pragma unroll
        for (int j = 0; j < 4; ++j) xv[j] = j < nv ? __ldg(x4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int ns = rows * G;
    uint16_t sv[16];
    {
        const int nz = rows * zrow;
        const uint16_t *sg = p.scales + static_cast<int64_t>(n0) * G;
        const uint32_t *zg = p.qzeros + static_cast<int64_t>(n0) * zrow;
        uint32_t zv[2];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int i = t + j * kW4Threads;
            sv[j] = i < ns ? __ldg(sg + i) : static_cast<uint16_t>(0);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = t + j * kW4Threads;
            zv[j] = i < nz ? __ldg(zg + i) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = t + j * kW4Threads;
            if (i < nz) s_zero[i] = zv[j];
        }
    }

    // activation planes: thread t splits elements EPT t .. EPT t + EPT - 1
    // (EPT = K / 512; a group spans TPG = gs / EPT threads).  X = rne(x / sx)
    // with sx = max|x| / 8355711 per group, x / sx taken as x * (1 / sx): at
    // most one more unit of error than the exact quotient.
    {
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(xv[j].x), fabsf(xv[j].y)), fmaxf(fabsf(xv[j].z), fabsf(xv[j].w))));
        for (int o = TPG / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sx = __fdiv_rn(amax, static_cast<float>(kW4XMax));
        const float inv = amax > 0.f ? __fdiv_rn(1.0f, sx) : 0.f;
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j < nv) {
                const float e4[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int X = __float2int_rn(__fmul_rn(e4[u], inv));
                    X = max(-kW4XMax, min(kW4XMax, X));
                    sum += X;
                    const int P2 = digit_s8(X), X1 = (X - P2) >> 8;
                    const int P1 = digit_s8(X1), P0 = (X1 - P1) >> 8;
                    const int k = EPT * t + 4 * j + u, jj = k & 7;
                    const int pos = (k & ~7) + ((jj & 1) ? 4 + (jj >> 1) : (jj >> 1));
                    planes[pos] = static_cast<int8_t>(P0);
                    planes[K + pos] = static_cast<int8_t>(P1);
                    planes[2 * K + pos] = static_cast<int8_t>(P2);
                }
            }
        }
        for (int o = TPG / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (t % TPG == 0) {
            s_sx[(EPT * t) / gs] = sx;
            s_sumx[(EPT * t) / gs] = sum;
        }
    }
    named_bar_sync(1, kW4Threads);
    // per (row, group): s sx and s sx z sumX (G is a power of two)
    const int g_shift = __ffs(G) - 1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int i = t + j * kW4Threads;
        if (i < ns) {
            const int r = i >> g_shift, grp = i & (G - 1);
            const float fs = __fmul_rn(__half2float(__ushort_as_half(sv[j])), s_sx[grp]);
            const float z = static_cast<float>((s_zero[r * zrow + grp / 8] >> (4 * (grp % 8))) & 15u);
            s_tab[i] = make_float2(fs, __fmul_rn(__fmul_rn(fs, z), static_cast<float>(s_sumx[grp])));
        }
    }
    named_bar_sync(1, kW4Threads);

    const int SPG = gs / 128, spg_shift = __ffs(SPG) - 1;  // spans per group (a power of two)
    for (int s = 0; s < nst; ++s) {
        const int slot = s % nstg;
        bool ok = mbar_wait(bars + 8 * slot, (s / nstg) & 1, &s_abort, p.status, SITE_W4_STAGE);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            const uint32_t sbase = ring + static_cast<uint32_t>(slot) * 16u * pitch;
            const int r0 = 16 * s + gq, r1 = r0 + 8;
            float acc0 = 0.f;  // row g (lane t = 0) or g + 8 (lane t = 2)
#pragma unroll
            for (int c = 0; c < SPW; ++c) {
                const int sp = warp + kW4Warps * c;
                uint4 wa, wb;
                const uint32_t wad = sbase + static_cast<uint32_t>(gq) * pitch + 64u * sp + 16u * tq;
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wa.x), "=r"(wa.y), "=r"(wa.z), "=r"(wa.w) : "r"(wad));
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wb.x), "=r"(wb.y), "=r"(wb.z), "=r"(wb.w) : "r"(wad + 8u * pitch));
                uint4 bx[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
                if (gq < 3) {
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        bx[e] = *reinterpret_cast<const uint4 *>(planes + gq * K + 128 * sp + 32 * tq + 16 * e);
                }
                int clo[4] = {0, 0, 0, 0}, chi[4] = {0, 0, 0, 0};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t a0 = e ? wa.z : wa.x, a2 = e ? wa.w : wa.y;
                    const uint32_t a1 = e ? wb.z : wb.x, a3 = e ? wb.w : wb.y;
                    const uint32_t lo[4] = {a0 & 0x0f0f0f0fu, a1 & 0x0f0f0f0fu, a2 & 0x0f0f0f0fu, a3 & 0x0f0f0f0fu};
                    const uint32_t hi[4] = {a0 & 0xf0f0f0f0u, a1 & 0xf0f0f0f0u, a2 & 0xf0f0f0f0u, a3 & 0xf0f0f0f0u};
                    mma_u8s8_16832(clo, lo, bx[e].x, bx[e].z);
                    mma_u8s8_16832(chi, hi, bx[e].y, bx[e].w);
                }
                int d[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) d[q] = clo[q] + (chi[q] >> 4);
                // lane t = 0 finishes row g, lane t = 2 row g + 8 (D0, D1 in columns 0, 1 of
                // lane t = 0, D2 in column 2 of lane t = 1)
                const int e0 = __shfl_down_sync(0xffffffffu, d[0], 1);
                const int e1 = __shfl_up_sync(0xffffffffu, d[2], 2), e2 = __shfl_up_sync(0xffffffffu, d[3], 2);
                const int e3 = __shfl_up_sync(0xffffffffu, d[2], 1);
                if ((tq & 1) == 0) {
                    const int row = tq == 0 ? r0 : r1;
                    const int D0 = tq == 0 ? d[0] : e1, D1 = tq == 0 ? d[1] : e2, D2 = tq == 0 ? e0 : e3;
                    if (row < rows) {
                        const float T = fmaf(65536.0f, static_cast<float>(D0),
                                             fmaf(256.0f, static_cast<float>(D1), static_cast<float>(D2)));
                        const float2 f = s_tab[row * G + (sp >> spg_shift)];
                        acc0 += fmaf(f.x, T, (sp & (SPG - 1)) == 0 ? -f.y : 0.0f);
                    }
                }
            }
            if ((tq & 1) == 0) {
                const int row = tq == 0 ? r0 : r1;
                if (row < rows) s_part[row * kW4Warps + warp] = acc0;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(ebars + 8 * slot);  // this warp is done with the slot
    }
    named_bar_sync(1, kW4Threads);
    for (int r = t; r < rows; r += kW4Threads) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kW4Warps; ++w) acc += s_part[r * kW4Warps + w];
        p.out[n0 + r] = (p.bias ? __ldg(p.bias + n0 + r) : 0.0f) + acc;
    }
}

int w4_rows_cap(int64_t N, const DevInfo &dev) {
    const int64_t Gc = std::min<int64_t>(N, dev.num_sms);
    return static_cast<int>((N + Gc - 1) / Gc);
}

int w4_decode_stages(int K, int gs, int rows_cap, const DevInfo &dev) {
    const W4Layout L0(K, gs, 0, rows_cap);
    const int64_t room = static_cast<int64_t>(dev.max_smem_optin) - L0.total;
    return static_cast<int>(std::min<int64_t>(kW4MaxStages, room / (16 * (K / 2 + 64))));
}

bool w4_decode_supported(int64_t M, int64_t N, int64_t K, int64_t gs, const DevInfo &dev) {
    if (M != 1 || K % 2048 != 0 || K > 8192 || gs % 128 != 0 || K % gs != 0 || (gs & (gs - 1)) != 0) return false;
    if (gs / (K / kW4Threads) > 32) return false;  // a group spans at most one warp in the split
    const int64_t Gc = std::min<int64_t>(N, dev.num_sms), rb = (N + Gc - 1) / Gc, G = K / gs;
    if (rb > kW4MaxRows) return false;
    if (rb * G > 16 * kW4Threads || rb * ((G + 7) / 8) > 2 * kW4Threads) return false;  // scale / zero registers
    return w4_decode_stages(static_cast<int>(K), static_cast<int>(gs), static_cast<int>(rb), dev) >= 2;
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
    a.rows_cap = w4_rows_cap(N, dev);
    a.nstg = w4_decode_stages(a.K, a.gs, a.rows_cap, dev);
    a.status = dev.status;
    const int smem = static_cast<int>(W4Layout(a.K, a.gs, a.nstg, a.rows_cap).total);
    auto kern = K == 2048 ? w4_decode_kernel<1> : K == 4096 ? w4_decode_kernel<2> : w4_decode_kernel<4>;
    static int attr_smem[3][64] = {};
    int &done = attr_smem[K == 2048 ? 0 : K == 4096 ? 1 : 2][dev.device];
    if (smem > 48 * 1024 && smem > done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        done = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(N, dev.num_sms)));
    cfg.blockDim = dim3(kW4Block);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
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
