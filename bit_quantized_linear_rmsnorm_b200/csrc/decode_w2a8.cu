// Fused BitLinear W1.58A8 decode (M <= 16 tokens): one launch per call.
//
// "Class BitLinear" (LLaMA-BitNet utils.py), forward steps 1-5, at inference
// time (the page: specialised ternary kernels are only needed at inference):
//   xq, act_scale = per-token int8 quantization of RMSNorm(x)
//   acc[m,n] = sum_k xq[m,k] * w_q[n,k],   out = (float(acc) * act_scale[m]) * gamma (+ bias)
//
// Kernels, each one launch per call with the tokens quantized inside it:
// decode_w2a8_stream_kernel (one token, K a multiple of 2048, dp4a from
// registers), decode_w2a8_fused_kernel (2..16 tokens, K = 2048 or 4096,
// masked mma.sync from registers), and decode_w2a8_kernel below for the other
// shapes with K % 512 == 0.  decode_w2a8_mma_kernel serves the LayerNorm
// BitLinear, whose quantizer has already written the codes.
//
// decode_w2a8_kernel: bandwidth-bound on the 2-bit weights.  One CTA owns RB consecutive output
// rows and copies them into shared memory with 16-byte cp.async (many copies
// in flight per SM through the load/store path -- measured faster than 2-D
// TMA boxes for this short HBM stream), laid out in 128-byte K slices of
// every row with the 128-byte XOR swizzle (chunk c of row r at c ^ (r % 8))
// so that the fragment loads below are free of bank conflicts.
//
// Overlap across calls.  Each kernel lets the next kernel of the stream
// launch at once (programmatic dependent launch); a CTA small enough to share
// an SM (256 threads, <= 128 registers) starts while the previous call runs,
// and before griddepcontrol.wait it only prefetches its weight lines into L2
// -- nothing is consumed, so this is correct whatever the previous kernel
// wrote.  After the wait it issues its weight copies, then quantizes the
// activations while they are in flight (CTA 0 also writes xq, act_scale and
// rowsum to the workspace), then:
//   * M <= 2: warp w owns rows w, w+8, ...; per slice each lane takes one
//     packed word (16 weights) of a row: dp4a of the u8 codes with the s8
//     activations (one token: the 2-bit fields are masked in place, so
//     (word & (3 << 2j)) . x accumulates 4^j times the code dot product).
//   * M >= 3: mma.sync m16n8k32 u8 x s8.  The packed layout puts the codes of
//     k = 16w + 4j + b at bits [8b+2j, 8b+2j+1] of word w, so
//     (word >> 2j) & 0x03030303 is the A fragment of quad thread j; warp w
//     takes k-steps 2w and 2w+1 of every slice for all 16-row blocks, and
//     the partial accumulators are reduced across warps once, at the end.
// The codes are offset binary (w_q + 1), so acc = dot(codes, xq) - rowsum.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <algorithm>

#include "bq_internal.h"
#include "quant_common.cuh"

namespace bq {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSliceWords = 32;               // 128 bytes of each packed row per slice
constexpr int kChunksPerRow16 = 8;            // 16-byte chunks per row and slice
constexpr int kMaxSlices = 16;                // K <= 8192
constexpr int kMaxRB = 96;                    // rows per CTA
constexpr int kMaxBlocks = kMaxRB / 16;       // 16-row blocks of the mma path
constexpr int kMaxRowsPerWarp = kMaxRB / kWarps;

struct DecodeArgs {
    const void *x;
    int M, K;
    float eps;
    const uint32_t *wpacked;
    const float *w_scale;
    const float *bias;
    int N;
    void *out;
    int8_t *ws_xq;
    float *ws_scale;
    int32_t *ws_rowsum;
    int rb;  // rows per CTA
    uint32_t *status;
    bq_dtype out_dtype;
    const float *ln_w = nullptr, *ln_b = nullptr;  // LayerNorm normaliser (one-token stream kernel): affine or NULL
};

struct Layout {
    uint32_t slice_bytes, nslices, xs, off_x, off_sc, off_rs, off_red, off_qred, total;
    __host__ __device__ Layout(int K, int MT, int rb) {
        nslices = static_cast<uint32_t>(K / (16 * kSliceWords));
        slice_bytes = (static_cast<uint32_t>(rb) * 128u + 1023u) & ~1023u;  // 1024-aligned for the swizzle
        xs = static_cast<uint32_t>(K) + 16u;                                 // padded token rows
        off_x = nslices * slice_bytes;
        off_sc = a16(off_x + MT * xs);
        off_rs = a16(off_sc + 4 * MT);
        off_red = a16(off_rs + 4 * MT);
        off_qred = a16(off_red + (MT > 2 ? kMaxRB * 16 * 4 : 0));
        total = a16(off_qred + 3 * kWarps * 2 * 4);  // cooperative prologue partials
    }
    __host__ __device__ static uint32_t a16(uint32_t v) { return (v + 15u) & ~15u; }
};

template <typename OutT>
__device__ __forceinline__ OutT to_out(float v);
template <>
__device__ __forceinline__ float to_out<float>(float v) {
    return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half to_out<__half>(float v) {
    return __float2half_rn(v);
}

// Byte offset of packed word `w` (0..31) of row `r` inside a 128-byte-swizzled
// slice: 16-byte chunk w/4 of the row sits at chunk position (w/4) ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int r, int w) {
    return static_cast<uint32_t>(r) * 128u + ((static_cast<uint32_t>(w >> 2) ^ static_cast<uint32_t>(r & 7)) << 4) +
           (static_cast<uint32_t>(w & 3) << 2);
}

// Rows of the CTA: the grid has one CTA per SM (or one per row when N is
// smaller), and CTA b owns rows [b N / G, (b+1) N / G), so the ranges differ
// by at most one row.  A grid of exactly one CTA per SM also keeps two CTAs of
// the same call off one SM when consecutive calls overlap: each call's CTAs
// can only take the slot that a CTA of the call before the previous one left.
struct RowRange {
    int begin, rows;
};
__device__ __forceinline__ RowRange row_range(int N) {
    const int64_t b = blockIdx.x, G = gridDim.x;
    const int n0 = static_cast<int>((b * N) / G), n1 = static_cast<int>(((b + 1) * N) / G);
    return {n0, n1 - n0};
}

// One warp quantizes one token row (16-byte aligned, K % (16/sizeof(In)) == 0)
// into shared memory (and the workspace when ws != nullptr).  Rows of up to
// 512 chunks sit in registers, so their loads are all in flight at once.
template <typename InT>
__device__ __forceinline__ void warp_quant_token(const InT *__restrict__ xr, int K, float eps, int8_t *dst,
                                                 int8_t *ws, float &scale, int &rowsum) {
    constexpr int EPC = Elt<InT>::kPerChunk;
    constexpr int CPL = 16;  // cached chunks per lane
    const int lane = threadIdx.x & 31;
    const int nch = K / EPC;
    if (nch > 32 * CPL) {
        warp_quant_row_vec<InT>(xr, K, eps, dst, ws, scale, rowsum);
        return;
    }
    const uint4 *xv = reinterpret_cast<const uint4 *>(xr);
    uint4 c[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int ch = lane + 32 * i;
        if (ch < nch) c[i] = __ldg(xv + ch);
    }
    float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int ch = lane + 32 * i;
        if (ch < nch) {
            float f[EPC];
            Elt<InT>::unpack(c[i], f);
#pragma unroll
            for (int e = 0; e < EPC; e += 2) {
                ss0 = fmaf(f[e], f[e], ss0);
                ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
            }
        }
    }
    const float ss = warp_sum_f(ss0 + ss1);
    amax = warp_max_f(amax);
    float fac;
    quant_row_factor(ss, amax, K, eps, fac, scale);
    int isum = 0;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int ch = lane + 32 * i;
        if (ch < nch) {
            float e[EPC];
            Elt<InT>::unpack(c[i], e);
            uint32_t w[EPC / 4];
#pragma unroll
            for (int j = 0; j < EPC / 4; ++j) {
                w[j] = pack_codes4(fmaf(e[4 * j], fac, kRoundMagic), fmaf(e[4 * j + 1], fac, kRoundMagic),
                                   fmaf(e[4 * j + 2], fac, kRoundMagic), fmaf(e[4 * j + 3], fac, kRoundMagic));
                isum = dp4a_ss(w[j], 0x01010101u, isum);
            }
            if constexpr (EPC == 8) {
                *reinterpret_cast<uint2 *>(dst + ch * 8) = make_uint2(w[0], w[1]);
                if (ws) *reinterpret_cast<uint2 *>(ws + ch * 8) = make_uint2(w[0], w[1]);
            } else {
                *reinterpret_cast<uint32_t *>(dst + ch * 4) = w[0];
                if (ws) *reinterpret_cast<uint32_t *>(ws + ch * 4) = w[0];
            }
        }
    }
    rowsum = warp_sum_i(isum);
}

// All warps quantize the (one or two) token rows together: warp w takes an
// eighth of each row, partial sums and maxima meet in shared memory, and
// every thread derives the same code factor from them.
template <int MT, typename InT>
__device__ __forceinline__ void cta_quant_small(const InT *__restrict__ x, int M, int K, float eps, int8_t *xs,
                                                int xs_pitch, int8_t *ws_xq, float *s_scale, int *s_rowsum,
                                                float *ws_scale, int32_t *ws_rowsum, float *q) {
    constexpr int EPC = Elt<InT>::kPerChunk;
    constexpr int CPL = 4;  // chunks per lane and row (K <= 4096 bf16 / 2048 fp32 fit in one pass)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = K / EPC;
    const int per_warp = (nch + kWarps - 1) / kWarps;
    const int c0 = warp * per_warp;
    const int c1 = min(nch, c0 + per_warp);
    float *q_ss = q, *q_mx = q + 2 * kWarps;
    int *q_rs = reinterpret_cast<int *>(q + 4 * kWarps);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
        const uint4 *xv = reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(m) * K);
        uint4 v[CPL];
        const bool cached = c1 - c0 <= 32 * CPL;
        float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
        auto stats = [&](const uint4 &u) {
            float f[EPC];
            Elt<InT>::unpack(u, f);
#pragma unroll
            for (int e = 0; e < EPC; e += 2) {
                ss0 = fmaf(f[e], f[e], ss0);
                ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
            }
        };
        if (cached) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = c0 + lane + 32 * i;
                if (c < c1) v[i] = __ldg(xv + c);
            }
#pragma unroll
            for (int i = 0; i < CPL; ++i)
                if (c0 + lane + 32 * i < c1) stats(v[i]);
        } else {
            for (int c = c0 + lane; c < c1; c += 32) stats(__ldg(xv + c));
        }
        const float a = warp_sum_f(ss0 + ss1), b = warp_max_f(amax);
        if (lane == 0) {
            q_ss[m * kWarps + warp] = a;
            q_mx[m * kWarps + warp] = b;
        }
        __syncthreads();
        float ss = 0.f, mx = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            ss += q_ss[m * kWarps + w];
            mx = fmaxf(mx, q_mx[m * kWarps + w]);
        }
        float fac, sc;
        quant_row_factor(ss, mx, K, eps, fac, sc);
        int isum = 0;
        auto codes = [&](const uint4 &u, int c) {
            float e[EPC];
            Elt<InT>::unpack(u, e);
            uint32_t w[EPC / 4];
#pragma unroll
            for (int j = 0; j < EPC / 4; ++j) {
                w[j] = pack_codes4(fmaf(e[4 * j], fac, kRoundMagic), fmaf(e[4 * j + 1], fac, kRoundMagic),
                                   fmaf(e[4 * j + 2], fac, kRoundMagic), fmaf(e[4 * j + 3], fac, kRoundMagic));
                isum = dp4a_ss(w[j], 0x01010101u, isum);
            }
            int8_t *d0 = xs + m * xs_pitch + c * EPC;
            int8_t *d1 = ws_xq ? ws_xq + static_cast<int64_t>(m) * K + c * EPC : nullptr;
            if constexpr (EPC == 8) {
                *reinterpret_cast<uint2 *>(d0) = make_uint2(w[0], w[1]);
                if (d1) *reinterpret_cast<uint2 *>(d1) = make_uint2(w[0], w[1]);
            } else {
                *reinterpret_cast<uint32_t *>(d0) = w[0];
                if (d1) *reinterpret_cast<uint32_t *>(d1) = w[0];
            }
        };
        if (cached) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = c0 + lane + 32 * i;
                if (c < c1) codes(v[i], c);
            }
        } else {
            for (int c = c0 + lane; c < c1; c += 32) codes(__ldg(xv + c), c);
        }
        const int r = warp_sum_i(isum);
        if (lane == 0) q_rs[m * kWarps + warp] = r;
        if (threadIdx.x == 0) {
            s_scale[m] = sc;
            if (ws_scale) ws_scale[m] = sc;
        }
    }
    __syncthreads();
    if (threadIdx.x < M) {
        const int m = threadIdx.x;
        int r = 0;
        for (int w = 0; w < kWarps; ++w) r += q_rs[m * kWarps + w];
        s_rowsum[m] = r;
        if (ws_rowsum) ws_rowsum[m] = r;
    }
}

template <int MT, bool MMA, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 2)
    decode_w2a8_kernel(const DecodeArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int K = p.K, M = p.M;
    const Layout L(K, MT, p.rb);
    const int ns = static_cast<int>(L.nslices);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const RowRange rr = row_range(p.N);
    const int n_begin = rr.begin, rows = rr.rows;
    const uint32_t sbase = smem_u32(smem);
    int8_t *xs = reinterpret_cast<int8_t *>(smem + L.off_x);
    float *s_scale = reinterpret_cast<float *>(smem + L.off_sc);
    int *s_rowsum = reinterpret_cast<int *>(smem + L.off_rs);
    int *red = reinterpret_cast<int *>(smem + L.off_red);
    const int words = K / 16;
    const uint8_t *wbase = reinterpret_cast<const uint8_t *>(p.wpacked + static_cast<int64_t>(n_begin) * words);
    const int row_bytes = K / 4;

    // pull this CTA's weight lines toward L2 while the previous grid finishes
    for (int l = threadIdx.x; l < rows * (row_bytes / 128); l += kThreads)
        prefetch_l2(wbase + static_cast<int64_t>(l) * 128);
    if constexpr (MMA)
        for (int i = threadIdx.x; i < kMaxRB * 16; i += kThreads) red[i] = 0;
    pdl_launch_dependents();
    pdl_wait();  // previous grid complete and visible: data may be consumed from here on

    // weight copies: 16-byte chunk q of row r -> slice q / 8, swizzled chunk (q % 8) ^ (r % 8)
    {
        const int cpr = row_bytes / 16;  // chunks per row
        for (int j = threadIdx.x; j < p.rb * cpr; j += kThreads) {
            const int r = j / cpr, q = j - r * cpr;
            const int sl = q / kChunksPerRow16, c = q % kChunksPerRow16;
            const uint32_t dst = sbase + sl * L.slice_bytes + r * 128 + ((c ^ (r & 7)) << 4);
            const bool in = r < rows;
            cp_async_16(dst, wbase + (in ? static_cast<int64_t>(r) * row_bytes + q * 16 : 0), in ? 16u : 0u);
        }
        cp_async_commit();
    }
    const float gamma = __ldg(p.w_scale);

    // per-token activation quantization (the weight copies are in flight)
    if constexpr (MT <= 2) {
        cta_quant_small<MT, InT>(static_cast<const InT *>(p.x), M, K, p.eps, xs, L.xs,
                                 blockIdx.x == 0 ? p.ws_xq : nullptr, s_scale, s_rowsum,
                                 blockIdx.x == 0 ? p.ws_scale : nullptr, blockIdx.x == 0 ? p.ws_rowsum : nullptr,
                                 reinterpret_cast<float *>(smem + L.off_qred));
    } else {
        for (int m = warp; m < M; m += kWarps) {
            float sc;
            int rsum;
            warp_quant_token<InT>(static_cast<const InT *>(p.x) + static_cast<int64_t>(m) * K, K, p.eps,
                                  xs + m * L.xs, blockIdx.x == 0 ? p.ws_xq + static_cast<int64_t>(m) * K : nullptr,
                                  sc, rsum);
            if (lane == 0) {
                s_scale[m] = sc;
                s_rowsum[m] = rsum;
                if (blockIdx.x == 0) {
                    p.ws_scale[m] = sc;
                    p.ws_rowsum[m] = rsum;
                }
            }
        }
    }
    cp_async_wait_all();
    __syncthreads();
    OutT *out = static_cast<OutT *>(p.out);


    if constexpr (!MMA) {
        // rows r = warp + 8 i of this CTA; lane l takes word l of each slice
        int acc[kMaxRowsPerWarp][MT];
        int acc4[kMaxRowsPerWarp][4];
#pragma unroll
        for (int i = 0; i < kMaxRowsPerWarp; ++i) {
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[i][m] = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) acc4[i][j] = 0;
        }
        for (int s = 0; s < ns; ++s) {
            const uint8_t *sl = smem + s * L.slice_bytes;
            uint4 x4[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m)
                x4[m] = m < M ? *reinterpret_cast<const uint4 *>(xs + m * L.xs + 16 * (s * kSliceWords + lane))
                              : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int i = 0; i < kMaxRowsPerWarp; ++i) {
                const int r = warp + kWarps * i;
                if (r < rows) {
                    const uint32_t u = *reinterpret_cast<const uint32_t *>(sl + swz(r, lane));
                    if constexpr (MT == 1) {
                        acc4[i][0] = dp4a_us(u & 0x03030303u, x4[0].x, acc4[i][0]);
                        acc4[i][1] = dp4a_us(u & 0x0c0c0c0cu, x4[0].y, acc4[i][1]);
                        acc4[i][2] = dp4a_us(u & 0x30303030u, x4[0].z, acc4[i][2]);
                        acc4[i][3] = dp4a_us(u & 0xc0c0c0c0u, x4[0].w, acc4[i][3]);
                    } else {
                        const uint32_t c0 = u & 0x03030303u, c1 = (u >> 2) & 0x03030303u;
                        const uint32_t c2 = (u >> 4) & 0x03030303u, c3 = (u >> 6) & 0x03030303u;
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            int a = acc[i][m];
                            a = dp4a_us(c0, x4[m].x, a);
                            a = dp4a_us(c1, x4[m].y, a);
                            a = dp4a_us(c2, x4[m].z, a);
                            a = dp4a_us(c3, x4[m].w, a);
                            acc[i][m] = a;
                        }
                    }
                }
            }
        }
        {
#pragma unroll
            for (int i = 0; i < kMaxRowsPerWarp; ++i) {
                const int r = warp + kWarps * i;
                if (r < rows) {
                    if constexpr (MT == 1)
                        acc[i][0] = acc4[i][0] + (acc4[i][1] >> 2) + (acc4[i][2] >> 4) + (acc4[i][3] >> 6);
                    const int n = n_begin + r;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m < M) {
                            const int dot = warp_sum_i(acc[i][m]);
                            if (lane == 0) {
                                float v = __fmul_rn(__fmul_rn(static_cast<float>(dot - s_rowsum[m]), s_scale[m]),
                                                    gamma);
                                if (p.bias) v = __fadd_rn(v, __ldg(p.bias + n));
                                out[static_cast<int64_t>(m) * p.N + n] = to_out<OutT>(v);
                            }
                        }
                    }
                }
            }
        }
    } else {
        constexpr int NT = (MT + 7) / 8;  // n8 tiles
        const int g = lane >> 2, t = lane & 3;
        const int nblk = (rows + 15) / 16;
        int C[kMaxBlocks][NT][4];
#pragma unroll
        for (int b = 0; b < kMaxBlocks; ++b)
#pragma unroll
            for (int tile = 0; tile < NT; ++tile) C[b][tile][0] = C[b][tile][1] = C[b][tile][2] = C[b][tile][3] = 0;
        for (int s = 0; s < ns; ++s) {
            const uint8_t *sl = smem + s * L.slice_bytes;
            const uint32_t sh = 2 * t;
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // k-steps 2*warp + h of this slice
                const int ks = 2 * warp + h;
                const int k0 = 32 * (s * 16 + ks);
                uint32_t bf[NT][2];
#pragma unroll
                for (int tile = 0; tile < NT; ++tile) {
                    const int tok = tile * 8 + g;
                    bf[tile][0] = tok < M ? *reinterpret_cast<const uint32_t *>(xs + tok * L.xs + k0 + 4 * t) : 0u;
                    bf[tile][1] = tok < M ? *reinterpret_cast<const uint32_t *>(xs + tok * L.xs + k0 + 16 + 4 * t) : 0u;
                }
#pragma unroll
                for (int b = 0; b < kMaxBlocks; ++b) {
                    if (b < nblk) {
                        const int rg = 16 * b + g, rh = rg + 8;
                        uint32_t a[4];
                        a[0] = (*reinterpret_cast<const uint32_t *>(sl + swz(rg, 2 * ks)) >> sh) & 0x03030303u;
                        a[1] = (*reinterpret_cast<const uint32_t *>(sl + swz(rh, 2 * ks)) >> sh) & 0x03030303u;
                        a[2] = (*reinterpret_cast<const uint32_t *>(sl + swz(rg, 2 * ks + 1)) >> sh) & 0x03030303u;
                        a[3] = (*reinterpret_cast<const uint32_t *>(sl + swz(rh, 2 * ks + 1)) >> sh) & 0x03030303u;
#pragma unroll
                        for (int tile = 0; tile < NT; ++tile) mma_u8s8_16832(C[b][tile], a, bf[tile][0], bf[tile][1]);
                    }
                }
            }
        }
        // reduce across warps (every warp reaches the barrier)
#pragma unroll
        for (int b = 0; b < kMaxBlocks; ++b) {
            if (b < nblk) {
                int *rb = red + b * 16 * 16;
#pragma unroll
                for (int tile = 0; tile < NT; ++tile) {
                    const int col = tile * 8 + 2 * t;
                    atomicAdd(rb + g * 16 + col, C[b][tile][0]);
                    atomicAdd(rb + g * 16 + col + 1, C[b][tile][1]);
                    atomicAdd(rb + (g + 8) * 16 + col, C[b][tile][2]);
                    atomicAdd(rb + (g + 8) * 16 + col + 1, C[b][tile][3]);
                }
            }
        }
        __syncthreads();
        {
            for (int e = threadIdx.x; e < rows * 16; e += kThreads) {
                const int r = e >> 4, m = e & 15;
                if (m < M) {
                    const int n = n_begin + r;
                    float v = __fmul_rn(__fmul_rn(static_cast<float>(red[e] - s_rowsum[m]), s_scale[m]), gamma);
                    if (p.bias) v = __fadd_rn(v, __ldg(p.bias + n));
                    out[static_cast<int64_t>(m) * p.N + n] = to_out<OutT>(v);
                }
            }
        }
    }
}

// Register-streaming variant for one token.  256 threads at most 128
// registers each, so a CTA of the next call fits on the SM beside a running
// one: it starts as soon as this call's CTAs have started (programmatic
// dependent launch), prefetches its own weight lines into L2, and waits.
// After the dependency wait each thread loads its activation chunks first
// (they head the critical path: statistics -> code factor -> codes), then,
// once its statistics are in shared memory, its weight chunks
// j = t + 256 i (i < kStreamChunks) straight into registers.  With
// 256 % (K/64) == 0 every chunk of a thread covers the same 64-wide K range
// [64 q, 64 q + 64), q = t % (K/64), so it needs the same 64 activation bytes,
// held in registers.  dp4a per packed word (the 2-bit fields are masked in
// place: (word & (3 << 2j)) . x accumulates 4^j times the code dot product),
// then the partial row sums of four chunks are reduced across the warp at
// once (K/64 >= 32: the lanes of a warp share each chunk's row).
constexpr int kStreamThreads = 256;
constexpr int kStreamWarps = kStreamThreads / 32;
constexpr int kStreamChunks = 20;      // weight chunks per thread (multiple of 4)
constexpr int kStreamMaxRows = 160;    // rows per CTA
constexpr int kStreamXPitch = 8192 + 16;

template <int MT>
struct StreamX {
    static constexpr int kChunks = 4;  // activation chunks per thread and token
};

// Sum over the 32 lanes of four values at once: returns, in lanes 8c..8c+7,
// the warp sum of value c (6 shuffles instead of 20).
__device__ __forceinline__ int warp_sum4(int v0, int v1, int v2, int v3) {
    const int lane = threadIdx.x & 31;
    const bool h16 = lane & 16, h8 = lane & 8;
    int k0 = h16 ? v2 : v0, k1 = h16 ? v3 : v1;
    k0 += __shfl_xor_sync(0xffffffffu, h16 ? v0 : v2, 16);
    k1 += __shfl_xor_sync(0xffffffffu, h16 ? v1 : v3, 16);
    int k = h8 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;
}

// Code dot product of one 16-byte chunk (64 weights) with its 64 activations.
__device__ __forceinline__ int chunk_dot(const uint4 &w, const uint4 (&x)[4]) {
    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
    for (int h = 0; h < 4; ++h) {  // word h covers k = 64 q + 16 h .. + 16
        a0 = dp4a_us(wd[h] & 0x03030303u, x[h].x, a0);
        a1 = dp4a_us(wd[h] & 0x0c0c0c0cu, x[h].y, a1);
        a2 = dp4a_us(wd[h] & 0x30303030u, x[h].z, a2);
        a3 = dp4a_us(wd[h] & 0xc0c0c0c0u, x[h].w, a3);
    }
    return a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
}

// eight affine parameters of chunk c (k = 8 c .. 8 c + 7 for bf16, 4 c .. for fp32) as floats
template <int EPC>
__device__ __forceinline__ void ln_param8(const float *p, int c, float def, float (&o)[EPC]) {
    if (p == nullptr) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) o[e] = def;
    } else if (reinterpret_cast<uintptr_t>(p) % 16 == 0) {
#pragma unroll
        for (int h = 0; h < EPC / 4; ++h) {
            const float4 t = __ldg(reinterpret_cast<const float4 *>(p + c * EPC) + h);
            o[4 * h] = t.x;
            o[4 * h + 1] = t.y;
            o[4 * h + 2] = t.z;
            o[4 * h + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < EPC; ++e) o[e] = __ldg(p + c * EPC + e);
    }
}

// LN = true (one token): the LayerNorm normaliser instead of the RMSNorm one.
// Mean and variance from binary64 sums of x - x[0] (the shifted form cancels
// only by (mean - x[0])^2 / var); y = x * rsd + nmr with rsd = 1/sqrt(var +
// eps) and nmr = -mean * rsd split into two fp32 parts each, so the mean
// cancels inside one fused multiply-add before its only rounding, then the
// affine step in fp32.  y is then within about three fp32 roundings of itself
// plus an absolute 6 u^2 |nmr| max|g| (u = 2^-24), which, scaled by
// f = 127 / max|y|, stays below 4.3e-8 when |nmr| max|g| f < 2^21: far inside
// the 1e-6 band around a rounding tie.  A row that fails the check takes
// binary64 passes (the decision is the same for the whole CTA).
template <int MT, typename InT, typename OutT, bool LN>
__global__ void __launch_bounds__(kStreamThreads, 2) decode_w2a8_stream_kernel(const DecodeArgs p) {
    constexpr int EPC = Elt<InT>::kPerChunk;
    constexpr int XC = StreamX<MT>::kChunks;
    static_assert(!LN || MT == 1, "the LayerNorm form streams one token");
    __shared__ __align__(16) int8_t xs[MT][kStreamXPitch];
    __shared__ int rowacc[kStreamMaxRows][MT];
    __shared__ float q_ss[MT][kStreamWarps], q_mx[MT][kStreamWarps];
    __shared__ double q_d[2][kStreamWarps];  // LN: sums of x - x[0] and of its square
    __shared__ int q_rs[MT][kStreamWarps];
    const int K = p.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const RowRange rr = row_range(p.N);
    const int cpr = K / 64;  // 16-byte chunks per packed row
    const uint4 *wv = reinterpret_cast<const uint4 *>(p.wpacked + static_cast<int64_t>(rr.begin) * (K / 16));
    const int total = rr.rows * cpr;

    // L2 prefetch of this CTA's weight lines before the dependency wait
    // (consumes nothing, so it is correct whatever the previous kernel wrote)
    for (int l = threadIdx.x; l < total / 8; l += kStreamThreads) prefetch_l2(wv + 8 * l);
    for (int i = threadIdx.x; i < kStreamMaxRows * MT; i += kStreamThreads) (&rowacc[0][0])[i] = 0;
    pdl_launch_dependents();
    pdl_wait();

    // activations first
    const int nch = K / EPC;
    uint4 xc[MT][XC];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const uint4 *xv = reinterpret_cast<const uint4 *>(static_cast<const InT *>(p.x) + static_cast<int64_t>(m) * K);
#pragma unroll
        for (int i = 0; i < XC; ++i) {
            const int c = threadIdx.x + kStreamThreads * i;
            xc[m][i] = c < nch ? __ldg(xv + c) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    double ln_c = 0.0;  // LN: the row's first element
    if constexpr (LN) {
        ln_c = static_cast<double>(static_cast<float>(static_cast<const InT *>(p.x)[0]));
        double s = 0.0, s2 = 0.0;
#pragma unroll
        for (int i = 0; i < XC; ++i) {
            const int c = threadIdx.x + kStreamThreads * i;
            if (c < nch) {
                float f[EPC];
                Elt<InT>::unpack(xc[0][i], f);
#pragma unroll
                for (int e = 0; e < EPC; ++e) {
                    const double d = static_cast<double>(f[e]) - ln_c;
                    s += d;
                    s2 = fma(d, d, s2);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, o);
            s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        }
        if (lane == 0) {
            q_d[0][warp] = s;
            q_d[1][warp] = s2;
        }
    } else {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
#pragma unroll
            for (int i = 0; i < XC; ++i) {
                float f[EPC];
                Elt<InT>::unpack(xc[m][i], f);
#pragma unroll
                for (int e = 0; e < EPC; e += 2) {
                    ss0 = fmaf(f[e], f[e], ss0);
                    ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                    amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
                }
            }
            const float ss = warp_sum_f(ss0 + ss1), mx = warp_max_f(amax);
            if (lane == 0) {
                q_ss[m][warp] = ss;
                q_mx[m][warp] = mx;
            }
        }
    }

    // then the weights (issued behind the activation loads)
    uint4 w[kStreamChunks];
#pragma unroll
    for (int i = 0; i < kStreamChunks; ++i) {
        const int j = threadIdx.x + kStreamThreads * i;
        w[i] = j < total ? __ldcs(wv + j) : make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
    }
    const float gamma = __ldg(p.w_scale);
    __syncthreads();

    // code factor of each token (every thread derives the same one), codes
    float sc[MT];
    if constexpr (LN) {
        double S = 0.0, S2 = 0.0;
#pragma unroll
        for (int w2 = 0; w2 < kStreamWarps; ++w2) {
            S += q_d[0][w2];
            S2 += q_d[1][w2];
        }
        const double md = S / static_cast<double>(K);
        const double mu = ln_c + md;
        const double var = fmax(S2 / static_cast<double>(K) - md * md, 0.0);
        const double rsd = 1.0 / sqrt(var + static_cast<double>(p.eps));
        const double nmr = -mu * rsd;
        const float rsd_h = static_cast<float>(rsd), rsd_l = static_cast<float>(rsd - static_cast<double>(rsd_h));
        const float nmr_h = static_cast<float>(nmr), nmr_l = static_cast<float>(nmr - static_cast<double>(nmr_h));
        float gmax = 0.0f;  // max |g| (for the error check), gathered with max|y|
        auto y_f = [&](int i, float (&y)[EPC]) {
            const int c = threadIdx.x + kStreamThreads * i;
            float f[EPC], gk[EPC], bk[EPC];
            Elt<InT>::unpack(xc[0][i], f);
            ln_param8<EPC>(p.ln_w, c, 1.0f, gk);
            ln_param8<EPC>(p.ln_b, c, 0.0f, bk);
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                y[e] = __fmaf_rn(__fadd_rn(__fmaf_rn(f[e], rsd_h, nmr_h), __fmaf_rn(f[e], rsd_l, nmr_l)), gk[e], bk[e]);
                gmax = fmaxf(gmax, fabsf(gk[e]));
            }
        };
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < XC; ++i)
            if (threadIdx.x + kStreamThreads * i < nch) {
                float y[EPC];
                y_f(i, y);
#pragma unroll
                for (int e = 0; e < EPC; ++e) amax = fmaxf(amax, fabsf(y[e]));
            }
        amax = warp_max_f(amax);
        gmax = warp_max_f(gmax);
        if (lane == 0) {
            q_ss[0][warp] = amax;
            q_mx[0][warp] = gmax;
        }
        __syncthreads();
        amax = 0.0f;
        gmax = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < kStreamWarps; ++w2) {
            amax = fmaxf(amax, q_ss[0][w2]);
            gmax = fmaxf(gmax, q_mx[0][w2]);
        }
        const float a_f = fmaxf(amax, 1e-5f);
        const float fac = __fdiv_rn(127.0f, a_f);
        const bool fast = fabs(nmr) * static_cast<double>(gmax) * static_cast<double>(fac) < 2097152.0;
        double fd = 0.0;
        if (fast) {
            sc[0] = __fdiv_rn(a_f, 127.0f);
        } else {  // binary64 passes (uniform over the CTA)
            double ad = 0.0;
#pragma unroll
            for (int i = 0; i < XC; ++i) {
                const int c = threadIdx.x + kStreamThreads * i;
                if (c < nch) {
                    float f[EPC], gk[EPC], bk[EPC];
                    Elt<InT>::unpack(xc[0][i], f);
                    ln_param8<EPC>(p.ln_w, c, 1.0f, gk);
                    ln_param8<EPC>(p.ln_b, c, 0.0f, bk);
#pragma unroll
                    for (int e = 0; e < EPC; ++e)
                        ad = fmax(ad, fabs(fma(fma(static_cast<double>(f[e]), rsd, nmr), static_cast<double>(gk[e]),
                                               static_cast<double>(bk[e]))));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ad = fmax(ad, __shfl_xor_sync(0xffffffffu, ad, o));
            if (lane == 0) q_d[0][warp] = ad;
            __syncthreads();
            ad = 0.0;
#pragma unroll
            for (int w2 = 0; w2 < kStreamWarps; ++w2) ad = fmax(ad, q_d[0][w2]);
            ad = fmax(ad, 1e-5);
            fd = 127.0 / ad;
            sc[0] = static_cast<float>(ad / 127.0);
        }
        int isum = 0;
#pragma unroll
        for (int i = 0; i < XC; ++i) {
            const int c = threadIdx.x + kStreamThreads * i;
            if (c < nch) {
                uint32_t wq[EPC / 4];
                if (fast) {
                    float y[EPC];
                    y_f(i, y);
#pragma unroll
                    for (int j = 0; j < EPC / 4; ++j)
                        wq[j] = pack_codes4(__fmaf_rn(y[4 * j], fac, kRoundMagic), __fmaf_rn(y[4 * j + 1], fac, kRoundMagic),
                                            __fmaf_rn(y[4 * j + 2], fac, kRoundMagic),
                                            __fmaf_rn(y[4 * j + 3], fac, kRoundMagic));
                } else {
                    float f[EPC], gk[EPC], bk[EPC];
                    Elt<InT>::unpack(xc[0][i], f);
                    ln_param8<EPC>(p.ln_w, c, 1.0f, gk);
                    ln_param8<EPC>(p.ln_b, c, 0.0f, bk);
#pragma unroll
                    for (int j = 0; j < EPC / 4; ++j) {
                        uint32_t word = 0;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int e = 4 * j + u;
                            const double y = fma(fma(static_cast<double>(f[e]), rsd, nmr), static_cast<double>(gk[e]),
                                                 static_cast<double>(bk[e]));
                            int code = __double2int_rn(y * fd);
                            code = code < -128 ? -128 : (code > 127 ? 127 : code);
                            word |= (static_cast<uint32_t>(code) & 0xffu) << (8 * u);
                        }
                        wq[j] = word;
                    }
                }
#pragma unroll
                for (int j = 0; j < EPC / 4; ++j) isum = dp4a_ss(wq[j], 0x01010101u, isum);
                int8_t *ws = blockIdx.x == 0 ? p.ws_xq + c * EPC : nullptr;
                if constexpr (EPC == 8) {
                    *reinterpret_cast<uint2 *>(&xs[0][c * 8]) = make_uint2(wq[0], wq[1]);
                    if (ws) *reinterpret_cast<uint2 *>(ws) = make_uint2(wq[0], wq[1]);
                } else {
                    *reinterpret_cast<uint32_t *>(&xs[0][c * 4]) = wq[0];
                    if (ws) *reinterpret_cast<uint32_t *>(ws) = wq[0];
                }
            }
        }
        isum = warp_sum_i(isum);
        if (lane == 0) q_rs[0][warp] = isum;
        if (blockIdx.x == 0 && threadIdx.x == 0) p.ws_scale[0] = sc[0];
    } else {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float ss = 0.f, mx = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kStreamWarps; ++w2) {
            ss += q_ss[m][w2];
            mx = fmaxf(mx, q_mx[m][w2]);
        }
        float fac;
        quant_row_factor(ss, mx, K, p.eps, fac, sc[m]);
        int isum = 0;
#pragma unroll
        for (int i = 0; i < XC; ++i) {
            const int c = threadIdx.x + kStreamThreads * i;
            if (c < nch) {
                float e[EPC];
                Elt<InT>::unpack(xc[m][i], e);
                uint32_t wq[EPC / 4];
#pragma unroll
                for (int j = 0; j < EPC / 4; ++j) {
                    wq[j] = pack_codes4(fmaf(e[4 * j], fac, kRoundMagic), fmaf(e[4 * j + 1], fac, kRoundMagic),
                                        fmaf(e[4 * j + 2], fac, kRoundMagic), fmaf(e[4 * j + 3], fac, kRoundMagic));
                    isum = dp4a_ss(wq[j], 0x01010101u, isum);
                }
                int8_t *ws = blockIdx.x == 0 ? p.ws_xq + static_cast<int64_t>(m) * K + c * EPC : nullptr;
                if constexpr (EPC == 8) {
                    *reinterpret_cast<uint2 *>(&xs[m][c * 8]) = make_uint2(wq[0], wq[1]);
                    if (ws) *reinterpret_cast<uint2 *>(ws) = make_uint2(wq[0], wq[1]);
                } else {
                    *reinterpret_cast<uint32_t *>(&xs[m][c * 4]) = wq[0];
                    if (ws) *reinterpret_cast<uint32_t *>(ws) = wq[0];
                }
            }
        }
        isum = warp_sum_i(isum);
        if (lane == 0) q_rs[m][warp] = isum;
        if (blockIdx.x == 0 && threadIdx.x == 0) p.ws_scale[m] = sc[m];
    }
    }
    __syncthreads();

    // dot products: chunk i of this thread is row r0 + rstep * i
    const int qk = threadIdx.x % cpr, r0 = threadIdx.x / cpr, rstep = kStreamThreads / cpr;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        uint4 xr[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) xr[h] = *reinterpret_cast<const uint4 *>(&xs[m][64 * qk + 16 * h]);
#pragma unroll
        for (int g = 0; g < kStreamChunks / 4; ++g) {
            const int k = warp_sum4(chunk_dot(w[4 * g], xr), chunk_dot(w[4 * g + 1], xr),
                                    chunk_dot(w[4 * g + 2], xr), chunk_dot(w[4 * g + 3], xr));
            const int r = r0 + rstep * (4 * g + (lane >> 3));
            if ((lane & 7) == 0 && r < rr.rows) atomicAdd(&rowacc[r][m], k);
        }
    }
    __syncthreads();

    // epilogue: out = ((acc - rowsum) * act_scale) * gamma (+ bias)
    int rsum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int r = 0;
#pragma unroll
        for (int w2 = 0; w2 < kStreamWarps; ++w2) r += q_rs[m][w2];
        rsum[m] = r;
        if (blockIdx.x == 0 && threadIdx.x == 0) p.ws_rowsum[m] = r;
    }
    OutT *out = static_cast<OutT *>(p.out);
    for (int r = threadIdx.x; r < rr.rows; r += kStreamThreads) {
        const int n = rr.begin + r;
        const float bias = p.bias ? __ldg(p.bias + n) : 0.f;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = __fmul_rn(__fmul_rn(static_cast<float>(rowacc[r][m] - rsum[m]), sc[m]), gamma);
            if (p.bias) v = __fadd_rn(v, bias);
            out[static_cast<int64_t>(m) * p.N + n] = to_out<OutT>(v);
        }
    }
}

template <typename InT, typename OutT, bool LN = false>
cudaError_t launch_stream(const DecodeArgs &a, int MT, cudaStream_t s, int grid) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kStreamThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    (void)MT;  // one token (two would not fit the register budget)
    return cudaLaunchKernelEx(&cfg, decode_w2a8_stream_kernel<1, InT, OutT, LN>, a);
}

template <typename InT, bool LN = false>
cudaError_t launch_stream_out(const DecodeArgs &a, bq_dtype ot, int MT, cudaStream_t s, int grid) {
    switch (ot) {
        case BQ_F32:
            return launch_stream<InT, float, LN>(a, MT, s, grid);
        case BQ_F16:
            return launch_stream<InT, __half, LN>(a, MT, s, grid);
        default:
            return launch_stream<InT, __nv_bfloat16, LN>(a, MT, s, grid);
    }
}

// 2..16 tokens whose codes are already in the workspace (the LayerNorm
// BitLinear, after its quantizer): decode_w2a8_mma_kernel, launched as a
// programmatic dependent of the quantizer.  The quantizer waits for the work
// before it in the stream (griddepcontrol.wait) before it lets its dependent
// start (griddepcontrol.launch_dependents), so this kernel starts only once
// everything before the call is complete and visible: it loads its packed
// weights into registers at once (they stream from HBM while the tokens are
// quantized) and waits only for the codes; it copies them into shared memory
// and runs mma.sync m16n8k32 (u8 fields x s8 codes) from registers.
//
// Work unit = (16-row block rb, 256-wide K block kb); warp w takes the K
// blocks kb = w + 8 c (c < KBW, K = 2048 KBW) of every row block.  Lane
// (g = lane / 4, t = lane % 4) holds words 16 kb + 4 t .. + 3 of rows g and
// g + 8 of the block (two 16-byte loads).  MMA (s, j) takes field j of words
// 2 s and 2 s + 1 masked in place, (word & (3 << 2j)) = code * 4^j in each
// byte, as the A fragment; its k-slots 4 t + b and 16 + 4 t + b hold the
// codes of k = 16 (16 kb + 4 t + 2 s) + 4 j + b and of the next word, so the
// matching B fragment of token g is bytes 4 j .. 4 j + 3 of the two 16-byte
// activation chunks 16 kb + 4 t + 2 s and + 1.  The four fields accumulate in
// four accumulators, combined as acc0 + acc1 / 4 + acc2 / 16 + acc3 / 64
// (each acc_j is a multiple of 4^j, so the shifts are exact).  Each masked
// fragment serves both token groups (tokens 0-7 and 8-15).
constexpr int kMmaThreads = 256;
constexpr int kMmaWarps = kMmaThreads / 32;
constexpr int kMmaUnits = 10;  // units per warp held in registers

// 16-byte chunk c of a token row sits at chunk c ^ (2 ((c >> 3) & 1)): the
// B-fragment loads of lanes t = 0..3 (chunks 4 t + const) and of consecutive
// tokens (row pitch K + 16 bytes) then fall in distinct bank groups.
__device__ __forceinline__ int xchunk_swz(int c) { return c ^ (((c >> 3) & 1) << 1); }

template <typename OutT>
__device__ __forceinline__ void store_out(void *out, int64_t i, float v) {
    static_cast<OutT *>(out)[i] = to_out<OutT>(v);
}

template <int MT, int KBW>
struct MmaLayout {
    static constexpr int kMaxRows = 16 * (kMmaUnits / KBW);
    static __host__ __device__ int pitch(int K) { return K + 16; }
    static __host__ __device__ int off_acc(int K) { return MT * pitch(K); }
    static __host__ __device__ int off_scale(int K) { return off_acc(K) + kMaxRows * MT * 4; }
    static __host__ __device__ int off_rowsum(int K) { return off_scale(K) + MT * 4; }
    static __host__ __device__ int bytes(int K) { return off_rowsum(K) + MT * 4; }
};

template <int MT, int KBW>
__global__ void __launch_bounds__(kMmaThreads, 1) decode_w2a8_mma_kernel(const DecodeArgs p) {
    using L = MmaLayout<MT, KBW>;
    constexpr int NH = MT / 8;  // token groups of eight
    extern __shared__ __align__(16) uint8_t smem[];
    const int K = p.K, M = p.M;
    const int xp = L::pitch(K);
    int8_t *xs = reinterpret_cast<int8_t *>(smem);
    int *rowacc = reinterpret_cast<int *>(smem + L::off_acc(K));
    float *s_scale = reinterpret_cast<float *>(smem + L::off_scale(K));
    int *s_rowsum = reinterpret_cast<int *>(smem + L::off_rowsum(K));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const RowRange rr = row_range(p.N);
    const int wpr = K / 16;  // packed words per row
    const uint32_t *wrow = p.wpacked + static_cast<int64_t>(rr.begin) * wpr;

    // this warp's weight words (unit i: row block i / KBW, K block warp + 8 (i % KBW)),
    // read before the dependency wait: the token kernel released this grid only
    // after everything before the call had completed
    const int nrb = (rr.rows + 15) / 16;
    uint4 wa[kMmaUnits], wb[kMmaUnits];
#pragma unroll
    for (int i = 0; i < kMmaUnits; ++i) {
        const int rb = i / KBW, kb = warp + kMmaWarps * (i % KBW);
        const int r0 = rb * 16 + g, r1 = r0 + 8;
        const uint32_t *base = wrow + 16 * kb + 4 * t;
        wa[i] = r0 < rr.rows ? __ldcs(reinterpret_cast<const uint4 *>(base + static_cast<int64_t>(r0) * wpr))
                             : make_uint4(0u, 0u, 0u, 0u);
        wb[i] = r1 < rr.rows ? __ldcs(reinterpret_cast<const uint4 *>(base + static_cast<int64_t>(r1) * wpr))
                             : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = threadIdx.x; i < L::kMaxRows * MT; i += kMmaThreads) rowacc[i] = 0;
    const float gamma = __ldg(p.w_scale);
    pdl_launch_dependents();
    pdl_wait();  // the token codes are written and visible

    // token codes -> shared memory (swizzled rows) with asynchronous 16-byte
    // copies, all of a thread's in flight at once; per-token scale and row sum
    const int cpr = K / 16;  // 16-byte chunks per token row
    for (int i = threadIdx.x; i < M * cpr; i += kMmaThreads) {
        const int m = i / cpr, c = i - m * cpr;
        cp_async_16(smem_u32(xs + m * xp + xchunk_swz(c) * 16), p.ws_xq + static_cast<int64_t>(m) * K + 16 * c, 16);
    }
    cp_async_commit();
    if (threadIdx.x < M) {
        s_scale[threadIdx.x] = __ldcg(p.ws_scale + threadIdx.x);
        s_rowsum[threadIdx.x] = __ldcg(p.ws_rowsum + threadIdx.x);
    }
    cp_async_wait_all();
    __syncthreads();

    // per unit: the masked A fragments once, both token groups; the
    // accumulators of a row block are kept across its KBW K blocks
    int acc[NH][4][4];
#pragma unroll
    for (int i = 0; i < kMmaUnits; ++i) {
        const int rb = i / KBW, kb = warp + kMmaWarps * (i % KBW);
        if (i % KBW == 0) {
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[h][j][0] = acc[h][j][1] = acc[h][j][2] = acc[h][j][3] = 0;
        }
        if (rb < nrb) {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint32_t w0 = s ? wa[i].z : wa[i].x, w1 = s ? wa[i].w : wa[i].y;
                const uint32_t v0 = s ? wb[i].z : wb[i].x, v1 = s ? wb[i].w : wb[i].y;
                const int c0 = 16 * kb + 4 * t + 2 * s;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const int tok = g + 8 * h;
                    uint4 bx0 = make_uint4(0u, 0u, 0u, 0u), bx1 = make_uint4(0u, 0u, 0u, 0u);
                    if (tok < M) {
                        bx0 = *reinterpret_cast<const uint4 *>(xs + tok * xp + xchunk_swz(c0) * 16);
                        bx1 = *reinterpret_cast<const uint4 *>(xs + tok * xp + xchunk_swz(c0 + 1) * 16);
                    }
                    const uint32_t b0[4] = {bx0.x, bx0.y, bx0.z, bx0.w}, b1[4] = {bx1.x, bx1.y, bx1.z, bx1.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t mk = 0x03030303u << (2 * j);
                        const uint32_t a[4] = {w0 & mk, v0 & mk, w1 & mk, v1 & mk};
                        mma_u8s8_16832(acc[h][j], a, b0[j], b1[j]);
                    }
                }
            }
            if (i % KBW == KBW - 1) {  // last K block of this row block: combine and flush
                const int r0 = rb * 16 + g, r1 = r0 + 8;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    int v[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        v[c] = acc[h][0][c] + (acc[h][1][c] >> 2) + (acc[h][2][c] >> 4) + (acc[h][3][c] >> 6);
                    const int m0 = 2 * t + 8 * h, m1 = m0 + 1;
                    if (r0 < rr.rows && m0 < M) atomicAdd(&rowacc[r0 * MT + m0], v[0]);
                    if (r0 < rr.rows && m1 < M) atomicAdd(&rowacc[r0 * MT + m1], v[1]);
                    if (r1 < rr.rows && m0 < M) atomicAdd(&rowacc[r1 * MT + m0], v[2]);
                    if (r1 < rr.rows && m1 < M) atomicAdd(&rowacc[r1 * MT + m1], v[3]);
                }
            }
        }
    }
    __syncthreads();

    // epilogue: out = ((acc - rowsum) * act_scale) * gamma (+ bias)
    for (int e = threadIdx.x; e < rr.rows * M; e += kMmaThreads) {
        const int r = e / M, m = e - r * M;
        const int n = rr.begin + r;
        float v = __fmul_rn(__fmul_rn(static_cast<float>(rowacc[r * MT + m] - s_rowsum[m]), s_scale[m]), gamma);
        if (p.bias) v = __fadd_rn(v, __ldg(p.bias + n));
        const int64_t o = static_cast<int64_t>(m) * p.N + n;
        if (p.out_dtype == BQ_F32)
            store_out<float>(p.out, o, v);
        else if (p.out_dtype == BQ_F16)
            store_out<__half>(p.out, o, v);
        else
            store_out<__nv_bfloat16>(p.out, o, v);
    }
}

// 2..16 tokens in one launch.  One CTA per SM over a range of output rows (as
// decode_w2a8_mma_kernel), 16 warps; the tokens are quantized inside the
// launch, every CTA quantizing all of them (M x K activations, read from L2):
// with TOK = 4, 8 or 16 token slots, warp w takes part w % (16 / TOK) of
// token w / (16 / TOK); the partial statistics of a token's warps meet in
// shared memory and are added in part order, so every CTA derives the same
// code factor.  Weights: before the dependency wait only L2 prefetches of
// this CTA's lines; after it, each warp loads its units (16 rows x 256 K)
// into registers, all in flight while the tokens are quantized.  Warp w takes
// the 256-wide K block w % G (G = K / 256) of row blocks w / G, w / G +
// 16 / G, ..., so its token fragments are loaded from shared memory once;
// masked mma.sync as decode_w2a8_mma_kernel (one or two token groups, tokens
// >= M read as zero), partial row sums added in shared memory, then the
// epilogue.
constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedUnits = 5;  // 16-row units per warp held in registers

template <int KK, int TOK>
struct FusedLayout {
    static constexpr int kG = KK / 256;                     // 256-wide K blocks
    static constexpr int kRBS = kFusedWarps / kG;              // row-block stride of a warp
    static constexpr int kMaxRows = 16 * kFusedUnits * kRBS;   // rows per CTA
    static constexpr int kPitch = KK + 16;                  // padded token rows
    static constexpr int kOffAcc = TOK * kPitch;            // [rows][TOK] partial row sums
    static constexpr int kOffStat = kOffAcc + kMaxRows * TOK * 4;     // [warp] (sum x^2, max|x|)
    static constexpr int kOffRs = kOffStat + kFusedWarps * 8;            // [warp] code sums
    static constexpr int kOffScale = kOffRs + kFusedWarps * 4;           // [token] act_scale
    static constexpr int kBytes = kOffScale + TOK * 4;
};

template <int KK, int TOK, typename InT>
__global__ void __launch_bounds__(kFusedThreads, 1) decode_w2a8_fused_kernel(const DecodeArgs p) {
    using L = FusedLayout<KK, TOK>;
    constexpr int EPC = Elt<InT>::kPerChunk;
    constexpr int NH = TOK > 8 ? 2 : 1;        // token groups of eight
    constexpr int WPT = kFusedWarps / TOK;        // warps per token
    constexpr int KP = KK / WPT;               // a warp's part of a token
    constexpr int XC = KP / EPC / 32;          // 16-byte activation chunks per lane
    constexpr int XR = XC <= 8 ? XC : 8;       // of them held in registers at once (more: read twice)
    constexpr int G = L::kG, RBS = L::kRBS;
    extern __shared__ __align__(16) uint8_t smem[];
    const int M = p.M;
    int8_t *xs = reinterpret_cast<int8_t *>(smem);
    int *rowacc = reinterpret_cast<int *>(smem + L::kOffAcc);
    float *s_stat = reinterpret_cast<float *>(smem + L::kOffStat);
    int *s_rs = reinterpret_cast<int *>(smem + L::kOffRs);
    float *s_scale = reinterpret_cast<float *>(smem + L::kOffScale);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const RowRange rr = row_range(p.N);
    const int R = rr.rows, nrb = (R + 15) / 16;
    constexpr int wpr = KK / 16;  // packed words per row
    const uint32_t *wrow = p.wpacked + static_cast<int64_t>(rr.begin) * wpr;
    const int kb = warp % G, rb0 = warp / G;

    // before the dependency wait: L2 prefetches of this CTA's weight lines
    // (nothing is consumed) and shared-memory set-up
    for (int l = threadIdx.x; l < R * (wpr / 32); l += kFusedThreads) prefetch_l2(wrow + 32 * l);
    for (int i = threadIdx.x; i < R * TOK; i += kFusedThreads) rowacc[i] = 0;
    pdl_wait();  // x, the weights and w_scale may come from the kernels before
    pdl_launch_dependents();

    // this warp's part of its token, then its weight units
    const int tok = warp / WPT, part = warp % WPT;
    const bool tokw = tok < M;
    const uint4 *xv =
        reinterpret_cast<const uint4 *>(static_cast<const InT *>(p.x) + static_cast<int64_t>(tok) * KK + part * KP);
    uint4 xc[XR];
    if (tokw) {
#pragma unroll
        for (int j = 0; j < XR; ++j) xc[j] = __ldg(xv + lane + 32 * j);
    }
    uint4 wa[kFusedUnits], wb[kFusedUnits];
#pragma unroll
    for (int i = 0; i < kFusedUnits; ++i) {
        const int r0 = (rb0 + RBS * i) * 16 + g, r1 = r0 + 8;
        const uint32_t *base = wrow + 16 * kb + 4 * t;
        wa[i] = r0 < R ? __ldcs(reinterpret_cast<const uint4 *>(base + static_cast<int64_t>(r0) * wpr))
                       : make_uint4(0u, 0u, 0u, 0u);
        wb[i] = r1 < R ? __ldcs(reinterpret_cast<const uint4 *>(base + static_cast<int64_t>(r1) * wpr))
                       : make_uint4(0u, 0u, 0u, 0u);
    }
    const float gamma = __ldg(p.w_scale);

    // partial statistics of the part
    if (tokw) {
        float ss0 = 0.f, ss1 = 0.f, amax = 0.f;
#pragma unroll
        for (int b = 0; b < XC; b += XR) {
            if (b > 0) {
#pragma unroll
                for (int j = 0; j < XR; ++j) xc[j] = __ldg(xv + lane + 32 * (b + j));
            }
#pragma unroll
            for (int j = 0; j < XR; ++j) {
                float f[EPC];
                Elt<InT>::unpack(xc[j], f);
#pragma unroll
                for (int e = 0; e < EPC; e += 2) {
                    ss0 = fmaf(f[e], f[e], ss0);
                    ss1 = fmaf(f[e + 1], f[e + 1], ss1);
                    amax = fmaxf(amax, fmaxf(fabsf(f[e]), fabsf(f[e + 1])));
                }
            }
        }
        const float ss = warp_sum_f(ss0 + ss1);
        amax = warp_max_f(amax);
        if (lane == 0) {
            s_stat[2 * warp] = ss;
            s_stat[2 * warp + 1] = amax;
        }
    }
    __syncthreads();

    // the token's statistics (parts added in order), codes of the part into
    // shared memory (and the workspace, CTA 0)
    if (tokw) {
        float ss = 0.f, amax = 0.f;
#pragma unroll
        for (int c = 0; c < WPT; ++c) {
            ss += s_stat[2 * (WPT * tok + c)];
            amax = fmaxf(amax, s_stat[2 * (WPT * tok + c) + 1]);
        }
        float fac, scale;
        quant_row_factor(ss, amax, KK, p.eps, fac, scale);
        int8_t *xrow = xs + tok * L::kPitch;
        int8_t *wsrow = blockIdx.x == 0 ? p.ws_xq + static_cast<int64_t>(tok) * KK : nullptr;
        int isum = 0;
#pragma unroll
        for (int j = 0; j < XC; ++j) {
            const int c = part * (KP / EPC) + lane + 32 * j;  // chunk of EPC activations in the token
            if (XC > XR && j % XR == 0) {                     // read again (from L1)
#pragma unroll
                for (int i = 0; i < XR; ++i) xc[i] = __ldg(xv + lane + 32 * (j + i));
            }
            float e[EPC];
            Elt<InT>::unpack(xc[j % XR], e);
            uint32_t w[EPC / 4];
#pragma unroll
            for (int i = 0; i < EPC / 4; ++i) {
                w[i] = pack_codes4(fmaf(e[4 * i], fac, kRoundMagic), fmaf(e[4 * i + 1], fac, kRoundMagic),
                                   fmaf(e[4 * i + 2], fac, kRoundMagic), fmaf(e[4 * i + 3], fac, kRoundMagic));
                isum = dp4a_ss(w[i], 0x01010101u, isum);
            }
            if constexpr (EPC == 8) {
                *reinterpret_cast<uint2 *>(xrow + xchunk_swz(c >> 1) * 16 + (c & 1) * 8) = make_uint2(w[0], w[1]);
                if (wsrow) *reinterpret_cast<uint2 *>(wsrow + 8 * c) = make_uint2(w[0], w[1]);
            } else {
                *reinterpret_cast<uint32_t *>(xrow + xchunk_swz(c >> 2) * 16 + (c & 3) * 4) = w[0];
                if (wsrow) *reinterpret_cast<uint32_t *>(wsrow + 4 * c) = w[0];
            }
        }
        isum = warp_sum_i(isum);
        if (lane == 0) {
            s_rs[warp] = isum;
            if (part == 0) s_scale[tok] = scale;
        }
    }
    __syncthreads();  // the codes are in shared memory

    // this warp's B fragments (K block kb; tokens >= M read as zero)
    uint4 bx[2][NH][2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int c0 = 16 * kb + 4 * t + 2 * s;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const int tb = g + 8 * h;
            bx[s][h][0] = bx[s][h][1] = make_uint4(0u, 0u, 0u, 0u);
            if (tb < M) {
                bx[s][h][0] = *reinterpret_cast<const uint4 *>(xs + tb * L::kPitch + xchunk_swz(c0) * 16);
                bx[s][h][1] = *reinterpret_cast<const uint4 *>(xs + tb * L::kPitch + xchunk_swz(c0 + 1) * 16);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kFusedUnits; ++i) {
        const int rb = rb0 + RBS * i;
        if (rb < nrb) {
            int acc[NH][4][4];
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[h][j][0] = acc[h][j][1] = acc[h][j][2] = acc[h][j][3] = 0;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint32_t w0 = s ? wa[i].z : wa[i].x, w1 = s ? wa[i].w : wa[i].y;
                const uint32_t v0 = s ? wb[i].z : wb[i].x, v1 = s ? wb[i].w : wb[i].y;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const uint32_t b0[4] = {bx[s][h][0].x, bx[s][h][0].y, bx[s][h][0].z, bx[s][h][0].w};
                    const uint32_t b1[4] = {bx[s][h][1].x, bx[s][h][1].y, bx[s][h][1].z, bx[s][h][1].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t mk = 0x03030303u << (2 * j);
                        const uint32_t a[4] = {w0 & mk, v0 & mk, w1 & mk, v1 & mk};
                        mma_u8s8_16832(acc[h][j], a, b0[j], b1[j]);
                    }
                }
            }
            const int r0 = rb * 16 + g, r1 = r0 + 8;
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                int v[4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    v[c] = acc[h][0][c] + (acc[h][1][c] >> 2) + (acc[h][2][c] >> 4) + (acc[h][3][c] >> 6);
                const int m0 = 2 * t + 8 * h, m1 = m0 + 1;
                if (r0 < R && m0 < M) atomicAdd(&rowacc[r0 * TOK + m0], v[0]);
                if (r0 < R && m1 < M) atomicAdd(&rowacc[r0 * TOK + m1], v[1]);
                if (r1 < R && m0 < M) atomicAdd(&rowacc[r1 * TOK + m0], v[2]);
                if (r1 < R && m1 < M) atomicAdd(&rowacc[r1 * TOK + m1], v[3]);
            }
        }
    }
    __syncthreads();

    // epilogue: out = ((acc - rowsum) * act_scale) * gamma (+ bias), rows fastest
    for (int e = threadIdx.x; e < R * M; e += kFusedThreads) {
        const int m = e / R, r = e - m * R;
        int rs = 0;
#pragma unroll
        for (int c = 0; c < WPT; ++c) rs += s_rs[WPT * m + c];
        const int n = rr.begin + r;
        float o = __fmul_rn(__fmul_rn(static_cast<float>(rowacc[r * TOK + m] - rs), s_scale[m]), gamma);
        if (p.bias) o = __fadd_rn(o, __ldg(p.bias + n));
        const int64_t oi = static_cast<int64_t>(m) * p.N + n;
        if (p.out_dtype == BQ_F32)
            store_out<float>(p.out, oi, o);
        else if (p.out_dtype == BQ_F16)
            store_out<__half>(p.out, oi, o);
        else
            store_out<__nv_bfloat16>(p.out, oi, o);
    }
    if (blockIdx.x == 0 && threadIdx.x < M) {
        const int m = threadIdx.x;
        int rs = 0;
#pragma unroll
        for (int c = 0; c < WPT; ++c) rs += s_rs[WPT * m + c];
        p.ws_scale[m] = s_scale[m];
        p.ws_rowsum[m] = rs;
    }
}

cudaError_t launch_pdl_cfg(const void *kern, const DecodeArgs &a, int grid, int threads, int smem, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {const_cast<DecodeArgs *>(&a)};
    return cudaLaunchKernelExC(&cfg, kern, args);
}

template <int MT, bool MMA, typename InT, typename OutT>
cudaError_t launch_t(const DecodeArgs &a, int smem, const DevInfo &dev, cudaStream_t s, int grid) {
    auto kern = decode_w2a8_kernel<MT, MMA, InT, OutT>;
    static SmemOptIn opt_in;
    const cudaError_t e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), static_cast<size_t>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename InT, typename OutT>
cudaError_t dispatch_m(const DecodeArgs &a, int MT, int smem, const DevInfo &dev, cudaStream_t s, int grid) {
    switch (MT) {
        case 1:
            return launch_t<1, false, InT, OutT>(a, smem, dev, s, grid);
        case 2:
            return launch_t<2, false, InT, OutT>(a, smem, dev, s, grid);
        case 8:
            return launch_t<8, true, InT, OutT>(a, smem, dev, s, grid);
        default:
            return launch_t<16, true, InT, OutT>(a, smem, dev, s, grid);
    }
}

template <typename InT>
cudaError_t dispatch_out(const DecodeArgs &a, bq_dtype ot, int MT, int smem, const DevInfo &dev, cudaStream_t s,
                         int grid) {
    switch (ot) {
        case BQ_F32:
            return dispatch_m<InT, float>(a, MT, smem, dev, s, grid);
        case BQ_F16:
            return dispatch_m<InT, __half>(a, MT, smem, dev, s, grid);
        default:
            return dispatch_m<InT, __nv_bfloat16>(a, MT, smem, dev, s, grid);
    }
}

// One CTA per SM (fewer when N is smaller); the largest row range of a CTA.
int grid_of(int64_t N, const DevInfo &dev) { return static_cast<int>(std::min<int64_t>(N, dev.num_sms)); }
int rows_per_cta(int64_t N, const DevInfo &dev) {
    const int64_t G = grid_of(N, dev);
    return static_cast<int>((N + G - 1) / G);
}

template <int KK, int TOK, typename InT>
cudaError_t launch_fused_t(const DecodeArgs &a, const DevInfo &dev, int grid, cudaStream_t s) {
    auto kern = decode_w2a8_fused_kernel<KK, TOK, InT>;
    constexpr int smem = FusedLayout<KK, TOK>::kBytes;
    static SmemOptIn opt_in;
    const cudaError_t e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), static_cast<size_t>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl_cfg(reinterpret_cast<const void *>(kern), a, grid, kFusedThreads, smem, s);
}

// Shapes of the one-launch kernel: 2..16 tokens, K = 2048 or 4096, every
// unit of a warp in registers.
bool fused_supported(int64_t M, int64_t N, int64_t K, const DevInfo &dev) {
    if (M < 2 || M > 16 || (K != 2048 && K != 4096)) return false;
    const int64_t max_rows = K == 2048 ? FusedLayout<2048, 4>::kMaxRows : FusedLayout<4096, 4>::kMaxRows;
    return rows_per_cta(N, dev) <= max_rows;
}

template <int KK, typename InT>
cudaError_t launch_fused_k(const DecodeArgs &a, const DevInfo &dev, int grid, cudaStream_t s) {
    if (a.M <= 4) return launch_fused_t<KK, 4, InT>(a, dev, grid, s);
    if (a.M <= 8) return launch_fused_t<KK, 8, InT>(a, dev, grid, s);
    return launch_fused_t<KK, 16, InT>(a, dev, grid, s);
}

template <typename InT>
cudaError_t launch_fused(const DecodeArgs &a, const DevInfo &dev, int grid, cudaStream_t s) {
    if (a.K == 2048) return launch_fused_k<2048, InT>(a, dev, grid, s);
    return launch_fused_k<4096, InT>(a, dev, grid, s);
}

// Shapes of the register-streaming kernel: one token, 256 % (K/64) == 0
// with K/64 >= 32, the activation chunks of a thread cached in registers, and
// every weight chunk of the CTA in flight at once.
bool stream_supported(int64_t M, int64_t N, int64_t K, bq_dtype xt, const DevInfo &dev) {
    if (M != 1 || K % 64 != 0 || K > kStreamXPitch - 16) return false;
    const int64_t cpr = K / 64;
    if (cpr < 32 || kStreamThreads % cpr != 0) return false;
    const int64_t epc = xt == BQ_BF16 ? 8 : 4;
    if (K / epc > static_cast<int64_t>(kStreamThreads) * StreamX<1>::kChunks) return false;
    const int64_t rb = rows_per_cta(N, dev);
    return rb <= kStreamMaxRows && rb * cpr <= static_cast<int64_t>(kStreamThreads) * kStreamChunks;
}

// Shapes of the mma.sync register-streaming kernel: 2..16 tokens, K = 2048 or
// 4096, every unit of the CTA in registers, two CTAs per SM.
bool mma_stream_supported(int64_t M, int64_t N, int64_t K, const DevInfo &dev) {
    if (M < 2 || M > 16 || (K != 2048 && K != 4096)) return false;
    const int64_t max_rows = 16 * (kMmaUnits / (K / 2048));
    const int smem = M > 8 ? MmaLayout<16, 1>::bytes(static_cast<int>(K)) : MmaLayout<8, 1>::bytes(static_cast<int>(K));
    return rows_per_cta(N, dev) <= max_rows && 2 * static_cast<size_t>(smem + 1024) <= dev.max_smem_optin * 2 &&
           static_cast<size_t>(smem) <= dev.max_smem_optin;
}

int mt_of(int64_t M) { return M == 1 ? 1 : M == 2 ? 2 : M <= 8 ? 8 : 16; }

}  // namespace

bool decode_w2a8_supported(const void *x, int64_t M, int64_t N, int64_t K, const DevInfo &dev) {
    if (M < 1 || M > 16 || K % 512 != 0 || K > 512 * kMaxSlices || reinterpret_cast<uintptr_t>(x) % 16 != 0)
        return false;
    const int rb = rows_per_cta(N, dev);
    if (rb > kMaxRB || rb < 1) return false;
    return Layout(static_cast<int>(K), mt_of(M), rb).total + 1024 <= dev.max_smem_optin;
}

bool decode_mma_from_codes_supported(int64_t M, int64_t N, int64_t K, const DevInfo &dev) {
    return M >= 1 && mma_stream_supported(M < 2 ? 2 : M, N, K, dev);
}

cudaError_t launch_decode_mma_from_codes(const int8_t *xq, const float *act_scale, const int32_t *rowsum, int64_t M,
                                         int64_t K, const uint32_t *wpacked, const float *w_scale, const float *bias,
                                         int64_t N, bq_dtype out_dtype, void *out, cudaStream_t s,
                                         const DevInfo &dev) {
    DecodeArgs a;
    a.x = nullptr;
    a.M = static_cast<int>(M);
    a.K = static_cast<int>(K);
    a.eps = 0.0f;
    a.wpacked = wpacked;
    a.w_scale = w_scale;
    a.bias = bias;
    a.N = static_cast<int>(N);
    a.out = out;
    a.ws_xq = const_cast<int8_t *>(xq);
    a.ws_scale = const_cast<float *>(act_scale);
    a.ws_rowsum = const_cast<int32_t *>(rowsum);
    a.rb = rows_per_cta(N, dev);
    a.status = dev.status;
    a.out_dtype = out_dtype;
    const int grid = grid_of(N, dev);
    const bool two = M > 8;
    const void *kern;
    int smem;
    if (K == 2048) {
        kern = two ? reinterpret_cast<const void *>(decode_w2a8_mma_kernel<16, 1>)
                   : reinterpret_cast<const void *>(decode_w2a8_mma_kernel<8, 1>);
        smem = two ? MmaLayout<16, 1>::bytes(2048) : MmaLayout<8, 1>::bytes(2048);
    } else {
        kern = two ? reinterpret_cast<const void *>(decode_w2a8_mma_kernel<16, 2>)
                   : reinterpret_cast<const void *>(decode_w2a8_mma_kernel<8, 2>);
        smem = two ? MmaLayout<16, 2>::bytes(4096) : MmaLayout<8, 2>::bytes(4096);
    }
    static SmemOptIn opt_in[4];
    const cudaError_t e = smem_opt_in(opt_in[(K == 2048 ? 0 : 2) + (two ? 1 : 0)], dev, kern, static_cast<size_t>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl_cfg(kern, a, grid, kMmaThreads, smem, s);
}

int decode_w2a8_kind(int64_t M, int64_t N, int64_t K, bq_dtype xt, const DevInfo &dev) {
    if (fused_supported(M, N, K, dev)) return BQ_PATH_DECODE_MMA;
    if (stream_supported(M, N, K, xt, dev)) return BQ_PATH_DECODE_STREAM;
    return BQ_PATH_DECODE_SMEM;
}

cudaError_t launch_decode_w2a8(const void *x, bq_dtype xt, int64_t M, int64_t K, float eps, const uint32_t *wpacked,
                               const float *w_scale, const float *bias, int64_t N, bq_dtype out_dtype, void *out,
                               int8_t *ws_xq, float *ws_scale, int32_t *ws_rowsum, cudaStream_t s,
                               const DevInfo &dev) {
    const int MT = mt_of(M);
    const int rb = rows_per_cta(N, dev);
    const int grid = grid_of(N, dev);
    DecodeArgs a;
    a.x = x;
    a.M = static_cast<int>(M);
    a.K = static_cast<int>(K);
    a.eps = eps;
    a.wpacked = wpacked;
    a.w_scale = w_scale;
    a.bias = bias;
    a.N = static_cast<int>(N);
    a.out = out;
    a.ws_xq = ws_xq;
    a.ws_scale = ws_scale;
    a.ws_rowsum = ws_rowsum;
    a.rb = rb;
    a.status = dev.status;
    a.out_dtype = out_dtype;
    const int kind = decode_w2a8_kind(M, N, K, xt, dev);
    if (kind == BQ_PATH_DECODE_MMA) {
        if (xt == BQ_BF16) return launch_fused<__nv_bfloat16>(a, dev, grid, s);
        return launch_fused<float>(a, dev, grid, s);
    }
    if (kind == BQ_PATH_DECODE_STREAM) {
        if (xt == BQ_BF16) return launch_stream_out<__nv_bfloat16>(a, out_dtype, static_cast<int>(M), s, grid);
        return launch_stream_out<float>(a, out_dtype, static_cast<int>(M), s, grid);
    }
    const int smem = static_cast<int>(Layout(static_cast<int>(K), MT, rb).total) + 1024;
    if (xt == BQ_BF16) return dispatch_out<__nv_bfloat16>(a, out_dtype, MT, smem, dev, s, grid);
    return dispatch_out<float>(a, out_dtype, MT, smem, dev, s, grid);
}

bool decode_ln1_supported(const void *x, int64_t M, int64_t N, int64_t K, bq_dtype xt, const DevInfo &dev) {
    return M == 1 && reinterpret_cast<uintptr_t>(x) % 16 == 0 && stream_supported(M, N, K, xt, dev);
}

cudaError_t launch_decode_ln1(const void *x, bq_dtype xt, int64_t K, const float *ln_w, const float *ln_b, float eps,
                              const uint32_t *wpacked, const float *w_scale, const float *bias, int64_t N,
                              bq_dtype out_dtype, void *out, int8_t *ws_xq, float *ws_scale, int32_t *ws_rowsum,
                              cudaStream_t s, const DevInfo &dev) {
    DecodeArgs a;
    a.x = x;
    a.M = 1;
    a.K = static_cast<int>(K);
    a.eps = eps;
    a.wpacked = wpacked;
    a.w_scale = w_scale;
    a.bias = bias;
    a.N = static_cast<int>(N);
    a.out = out;
    a.ws_xq = ws_xq;
    a.ws_scale = ws_scale;
    a.ws_rowsum = ws_rowsum;
    a.rb = rows_per_cta(N, dev);
    a.status = dev.status;
    a.out_dtype = out_dtype;
    a.ln_w = ln_w;
    a.ln_b = ln_b;
    const int grid = grid_of(N, dev);
    if (xt == BQ_BF16) return launch_stream_out<__nv_bfloat16, true>(a, out_dtype, 1, s, grid);
    return launch_stream_out<float, true>(a, out_dtype, 1, s, grid);
}

}  // namespace bq
