// Fused BitLinear W1.58A8 decode (M <= 16 tokens): one launch per call.
//
// "Class BitLinear" (LLaMA-BitNet utils.py), forward steps 1-5, at inference
// time (the page: specialised ternary kernels are only needed at inference):
//   xq, act_scale = per-token int8 quantization of RMSNorm(x)
//   acc[m,n] = sum_k xq[m,k] * w_q[n,k],   out = (float(acc) * act_scale[m]) * gamma (+ bias)
//
// Bandwidth-bound on the 2-bit weights.  One CTA per SM owns a contiguous
// slice of output rows.  Thread 0 streams the slice's packed rows into a
// shared-memory ring with cp.async.bulk (16 rows per stage, rows padded by 16
// bytes so that fragment loads from different rows fall in different banks),
// while every CTA quantizes the M activation rows itself into shared memory
// (CTA 0 also writes them to the workspace).  Consumers:
//   * M <= 2: one warp per weight row, one packed word (16 weights) per lane
//     step, dp4a of the u8 codes with the s8 activations (for one token the
//     activations sit in registers and the 2-bit fields are masked in place,
//     so (word & (3 << 2j)) . x accumulates 4^j times the code dot product).
//   * M >= 3: mma.sync m16n8k32 u8 x s8 over register fragments.  The packed
//     layout puts the codes of k = 16w + 4j + b at bits [8b+2j, 8b+2j+1] of
//     word w, so (word >> 2j) & 0x03030303 is exactly the A fragment of
//     thread j of a quad (k = 4j..4j+3); the K range is split across the 16
//     warps and the partial accumulators are reduced in shared memory.
// The codes are offset binary (w_q + 1), so acc = dot(codes, xq) - rowsum.
//
// Programmatic dependent launch: the kernel lets the next kernel of the
// stream start early and waits for the previous one (griddepcontrol.wait)
// before its first global memory access.  Every mbarrier wait is bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "bq_internal.h"
#include "quant_common.cuh"

namespace bq {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int CR = 16;             // weight rows per stage
constexpr int kMaxKSteps = 16;     // k32 steps per warp in the mma path (K <= 8192)
constexpr int kMaxWordsPerLane = 16;  // packed words per lane and row in the dp4a path (K <= 8192)
constexpr int kRound = 5;          // chunks per reduction round of the mma path

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
    int rows_per_cta;
    int stages;
    uint32_t *status;
};

struct Layout {
    uint32_t rs, xs, off_w, off_x, off_sc, off_rs, off_red, off_qred, off_bar, total;
    __host__ __device__ Layout(int K, int MT, int S) {
        rs = K / 4 + 16;
        xs = K + 16;
        // every region starts on a 16-byte boundary (bulk-copy targets, uint4
        // accesses and the 8-byte mbarriers all rely on it)
        off_w = 0;
        off_x = a16(off_w + S * CR * rs);
        off_sc = a16(off_x + MT * xs);
        off_rs = a16(off_sc + 4 * MT);
        off_red = a16(off_rs + 4 * MT);
        off_qred = a16(off_red + kRound * CR * 16 * 4);
        // [2][MT][warps] sums/maxima, [MT] code factors, [MT][warps] row sums
        off_bar = a16(off_qred + (3 * MT * kWarps + MT) * 4);
        total = off_bar + 2 * S * 8;
    }
    __host__ __device__ static uint32_t a16(uint32_t v) { return (v + 15u) & ~15u; }
    __host__ bool aligned_ok() const {
        return rs % 16 == 0 && xs % 16 == 0 && off_x % 16 == 0 && off_red % 16 == 0 && off_qred % 16 == 0 &&
               off_bar % 8 == 0;
    }
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

// The whole CTA quantizes the M activation rows: every thread issues its
// 16-byte loads of all rows at once (two passes; the second hits L1/L2), the
// per-row sums and maxima are reduced warp by warp and then across the 16
// warps in a fixed order, with the same fp32 arithmetic as the standalone
// quantization kernel (quant_common.cuh).
template <int MT, typename InT>
__device__ __forceinline__ void cta_quant_rows(const InT *__restrict__ x, int M, int K, float eps, int8_t *xs,
                                               int xs_pitch, int8_t *ws_xq, float *s_scale, int *s_rowsum,
                                               float *ws_scale, int32_t *ws_rowsum, float *redf, int *redi) {
    constexpr int EPC = Elt<InT>::kPerChunk;
    constexpr int CPT = MT <= 4 ? 4 : (MT <= 8 ? 2 : 1);  // cached 16-byte chunks per thread and row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cpr = K / EPC;  // 16-byte chunks per row
    const bool cached = cpr <= CPT * kThreads;
    uint4 v[MT][CPT];
    float ss[MT], mx[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) ss[m] = mx[m] = 0.f;
    auto stats = [&](const uint4 &q, int m) {
        float f[EPC];
        Elt<InT>::unpack(q, f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            ss[m] = fmaf(f[e], f[e], ss[m]);
            mx[m] = fmaxf(mx[m], fabsf(f[e]));
        }
    };
    if (cached) {
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + i * kThreads;
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M && c < cpr) v[m][i] = __ldg(reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(m) * K) + c);
        }
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + i * kThreads;
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M && c < cpr) stats(v[m][i], m);
        }
    } else {
        for (int c = threadIdx.x; c < cpr; c += kThreads) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) stats(__ldg(reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(m) * K) + c), m);
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m < M) {
            const float a = warp_sum_f(ss[m]), b = warp_max_f(mx[m]);
            if (lane == 0) {
                redf[m * kWarps + warp] = a;
                redf[(MT + m) * kWarps + warp] = b;
            }
        }
    }
    __syncthreads();
    if (threadIdx.x < M) {
        const int m = threadIdx.x;
        float a = 0.f, b = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            a += redf[m * kWarps + w];
            b = fmaxf(b, redf[(MT + m) * kWarps + w]);
        }
        float fac, sc;
        quant_row_factor(a, b, K, eps, fac, sc);
        redf[2 * MT * kWarps + m] = fac;
        s_scale[m] = sc;
        if (ws_scale) ws_scale[m] = sc;
    }
    __syncthreads();
    int isum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) isum[m] = 0;
    auto codes = [&](const uint4 &q, int m, int c) {
        const float fac = redf[2 * MT * kWarps + m];
        float e[EPC];
        Elt<InT>::unpack(q, e);
        uint32_t w[EPC / 4];
#pragma unroll
        for (int j = 0; j < EPC / 4; ++j) {
            w[j] = pack_codes4(fmaf(e[4 * j], fac, kRoundMagic), fmaf(e[4 * j + 1], fac, kRoundMagic),
                               fmaf(e[4 * j + 2], fac, kRoundMagic), fmaf(e[4 * j + 3], fac, kRoundMagic));
            isum[m] = dp4a_ss(w[j], 0x01010101u, isum[m]);
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
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + i * kThreads;
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M && c < cpr) codes(v[m][i], m, c);
        }
    } else {
        for (int c = threadIdx.x; c < cpr; c += kThreads) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) codes(__ldg(reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(m) * K) + c), m, c);
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m < M) {
            const int q = warp_sum_i(isum[m]);
            if (lane == 0) redi[m * kWarps + warp] = q;
        }
    }
    __syncthreads();
    if (threadIdx.x < M) {
        const int m = threadIdx.x;
        int q = 0;
        for (int w = 0; w < kWarps; ++w) q += redi[m * kWarps + w];
        s_rowsum[m] = q;
        if (ws_rowsum) ws_rowsum[m] = q;
    }
    __syncthreads();
}

template <int MT, bool MMA, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 1) decode_w2a8_kernel(const DecodeArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int S = p.stages;
    const Layout L(p.K, MT, S);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = p.K, M = p.M;
    const int words = K / 16;
    const uint32_t rowbytes = static_cast<uint32_t>(K / 4);
    const int n_begin = blockIdx.x * p.rows_per_cta;
    const int n_end = min(p.N, n_begin + p.rows_per_cta);
    const int rows = n_end - n_begin;
    const int nchunks = (rows + CR - 1) / CR;
    const uint32_t sbase = smem_u32(smem);
    auto full = [&](int s) { return sbase + L.off_bar + 8u * s; };
    auto empty = [&](int s) { return sbase + L.off_bar + 8u * (S + s); };
    int8_t *xs = reinterpret_cast<int8_t *>(smem + L.off_x);
    float *s_scale = reinterpret_cast<float *>(smem + L.off_sc);
    int *s_rowsum = reinterpret_cast<int *>(smem + L.off_rs);
    int *red = reinterpret_cast<int *>(smem + L.off_red);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), kWarps);
        }
        fence_mbarrier_init();
    }
    if constexpr (MMA)
        for (int i = threadIdx.x; i < kRound * CR * 16; i += kThreads) red[i] = 0;
    pdl_launch_dependents();
    __syncthreads();
    pdl_wait();  // previous grid complete and visible: global memory may be touched from here on

    // Warp 0 streams the slice's packed rows: lane 0 arms each stage with its
    // byte count, then the 32 lanes issue the row copies.
    auto issue = [&](int c) {  // warp 0 only
        const int stage = c % S;
        const int rc = min(CR, rows - c * CR);
        if (lane == 0) mbar_arrive_expect_tx(full(stage), rc * rowbytes);
        __syncwarp();
        for (int r = lane; r < rc; r += 32)
            bulk_load(sbase + L.off_w + (stage * CR + r) * L.rs,
                      p.wpacked + static_cast<int64_t>(n_begin + c * CR + r) * words, rowbytes, full(stage));
    };
    int issued = min(S, nchunks);
    if (warp == 0)
        for (int c = 0; c < issued; ++c) issue(c);

    // per-token activation quantization into shared memory (overlaps the weight stream)
    cta_quant_rows<MT, InT>(static_cast<const InT *>(p.x), M, K, p.eps, xs, L.xs,
                            blockIdx.x == 0 ? p.ws_xq : nullptr, s_scale, s_rowsum,
                            blockIdx.x == 0 ? p.ws_scale : nullptr, blockIdx.x == 0 ? p.ws_rowsum : nullptr,
                            reinterpret_cast<float *>(smem + L.off_qred),
                            reinterpret_cast<int *>(smem + L.off_qred) + 2 * MT * kWarps + MT);
    const float gamma = __ldg(p.w_scale);
    OutT *out = static_cast<OutT *>(p.out);

    // Waits (bounded) for chunk c; warp-uniform result.
    auto wait_chunk = [&](int c) -> bool {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_timed(full(c % S), static_cast<uint32_t>(c / S) & 1u, p.status, SITE_DECODE_FULL);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };
    // Warp 0 refills the stage of chunk c with chunk c + S once every warp released it.
    auto refill = [&](int c) {
        if (warp == 0 && issued < nchunks) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait_timed(empty(c % S), static_cast<uint32_t>(c / S) & 1u, p.status, SITE_DECODE_EMPTY);
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                issue(issued);
                ++issued;
            }
        }
    };

    if constexpr (!MMA) {
        // one weight row per warp and chunk: warp w owns row w of every chunk
        uint4 xr[kMaxWordsPerLane];
        if constexpr (MT == 1) {
#pragma unroll
            for (int j = 0; j < kMaxWordsPerLane; ++j) {
                const int w = lane + 32 * j;
                xr[j] = w < words ? *reinterpret_cast<const uint4 *>(xs + 16 * w) : make_uint4(0, 0, 0, 0);
            }
        }
        for (int c = 0; c < nchunks; ++c) {
            if (!wait_chunk(c)) break;
            const int stage = c % S;
            const int rc = min(CR, rows - c * CR);
            const int r = warp;
            if (r < rc) {
                const uint32_t *wr = reinterpret_cast<const uint32_t *>(smem + L.off_w + (stage * CR + r) * L.rs);
                int acc[MT];
                int acc4[4] = {0, 0, 0, 0};
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0;
#pragma unroll
                for (int j = 0; j < kMaxWordsPerLane; ++j) {
                    const int w = lane + 32 * j;
                    if (w < words) {
                        const uint32_t u = wr[w];
                        if constexpr (MT == 1) {
                            acc4[0] = dp4a_us(u & 0x03030303u, xr[j].x, acc4[0]);
                            acc4[1] = dp4a_us(u & 0x0c0c0c0cu, xr[j].y, acc4[1]);
                            acc4[2] = dp4a_us(u & 0x30303030u, xr[j].z, acc4[2]);
                            acc4[3] = dp4a_us(u & 0xc0c0c0c0u, xr[j].w, acc4[3]);
                        } else {
                            const uint32_t c0 = u & 0x03030303u, c1 = (u >> 2) & 0x03030303u;
                            const uint32_t c2 = (u >> 4) & 0x03030303u, c3 = (u >> 6) & 0x03030303u;
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                if (m < M) {
                                    const uint4 x4 = *reinterpret_cast<const uint4 *>(xs + m * L.xs + 16 * w);
                                    int a = acc[m];
                                    a = dp4a_us(c0, x4.x, a);
                                    a = dp4a_us(c1, x4.y, a);
                                    a = dp4a_us(c2, x4.z, a);
                                    a = dp4a_us(c3, x4.w, a);
                                    acc[m] = a;
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(stage));  // the row has been read
                if constexpr (MT == 1) acc[0] = acc4[0] + (acc4[1] >> 2) + (acc4[2] >> 4) + (acc4[3] >> 6);
                const int n = n_begin + c * CR + r;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const int dot = warp_sum_i(acc[m]);
                        if (lane == 0) {
                            float v = __fmul_rn(__fmul_rn(static_cast<float>(dot - s_rowsum[m]), s_scale[m]), gamma);
                            if (p.bias) v = __fadd_rn(v, __ldg(p.bias + n));
                            out[static_cast<int64_t>(m) * p.N + n] = to_out<OutT>(v);
                        }
                    }
                }
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(stage));
            }
            refill(c);
        }
    } else {
        // K split across the 16 warps; each warp keeps one accumulator set per
        // chunk of a round and the round ends with one shared-memory reduction.
        constexpr int NT = (MT + 7) / 8;  // n8 tiles
        const int g = lane >> 2, t = lane & 3;
        uint32_t bf[kMaxKSteps][NT][2];
#pragma unroll
        for (int j = 0; j < kMaxKSteps; ++j) {
            const int s = warp + kWarps * j;
#pragma unroll
            for (int tile = 0; tile < NT; ++tile) {
                const int tok = tile * 8 + g;
                const bool ok = s < K / 32 && tok < M;
                bf[j][tile][0] = ok ? *reinterpret_cast<const uint32_t *>(xs + tok * L.xs + 32 * s + 4 * t) : 0u;
                bf[j][tile][1] = ok ? *reinterpret_cast<const uint32_t *>(xs + tok * L.xs + 32 * s + 16 + 4 * t) : 0u;
            }
        }
        for (int c0 = 0; c0 < nchunks; c0 += kRound) {
            const int cn = min(kRound, nchunks - c0);
            int C[kRound][NT][4];
#pragma unroll
            for (int i = 0; i < kRound; ++i)
#pragma unroll
                for (int tile = 0; tile < NT; ++tile) C[i][tile][0] = C[i][tile][1] = C[i][tile][2] = C[i][tile][3] = 0;
            bool ok = true;
#pragma unroll
            for (int i = 0; i < kRound; ++i) {
                if (i < cn && ok) {
                    const int c = c0 + i;
                    ok = wait_chunk(c);
                    if (ok) {
                        const int stage = c % S;
                        const uint8_t *wst = smem + L.off_w + stage * CR * L.rs;
                        const uint32_t *rg = reinterpret_cast<const uint32_t *>(wst + g * L.rs);
                        const uint32_t *rh = reinterpret_cast<const uint32_t *>(wst + (g + 8) * L.rs);
#pragma unroll
                        for (int j = 0; j < kMaxKSteps; ++j) {
                            const int s = warp + kWarps * j;
                            if (s < K / 32) {
                                const uint32_t sh = 2 * t;
                                uint32_t a[4];
                                a[0] = (rg[2 * s] >> sh) & 0x03030303u;
                                a[1] = (rh[2 * s] >> sh) & 0x03030303u;
                                a[2] = (rg[2 * s + 1] >> sh) & 0x03030303u;
                                a[3] = (rh[2 * s + 1] >> sh) & 0x03030303u;
#pragma unroll
                                for (int tile = 0; tile < NT; ++tile)
                                    mma_u8s8_16832(C[i][tile], a, bf[j][tile][0], bf[j][tile][1]);
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(empty(stage));
                        refill(c);
                    }
                }
            }
            // reduce the round across warps (every warp reaches this barrier)
#pragma unroll
            for (int i = 0; i < kRound; ++i) {
                if (i < cn) {
                    int *rb = red + i * CR * 16;
#pragma unroll
                    for (int tile = 0; tile < NT; ++tile) {
                        const int col = tile * 8 + 2 * t;
                        atomicAdd(rb + g * 16 + col, C[i][tile][0]);
                        atomicAdd(rb + g * 16 + col + 1, C[i][tile][1]);
                        atomicAdd(rb + (g + 8) * 16 + col, C[i][tile][2]);
                        atomicAdd(rb + (g + 8) * 16 + col + 1, C[i][tile][3]);
                    }
                }
            }
            __syncthreads();
            for (int e = threadIdx.x; e < cn * CR * 16; e += kThreads) {
                const int i = e / (CR * 16), r = (e / 16) % CR, m = e % 16;
                const int c = c0 + i;
                const int rc = min(CR, rows - c * CR);
                if (r < rc && m < M) {
                    const int n = n_begin + c * CR + r;
                    float v = __fmul_rn(__fmul_rn(static_cast<float>(red[e] - s_rowsum[m]), s_scale[m]), gamma);
                    if (p.bias) v = __fadd_rn(v, __ldg(p.bias + n));
                    out[static_cast<int64_t>(m) * p.N + n] = to_out<OutT>(v);
                }
                red[e] = 0;
            }
            __syncthreads();
        }
    }
    // let every issued copy land before the CTA exits
    if (warp == 0 && lane == 0) {
        for (int c = max(0, issued - S); c < issued; ++c) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(full(c % S), static_cast<uint32_t>(c / S) & 1u) &&
                   globaltimer_ns() - t0 < kWaitLimitNs) {
            }
        }
    }
}

template <int MT, bool MMA, typename InT, typename OutT>
cudaError_t launch_t(const DecodeArgs &a, int smem, const DevInfo &dev, cudaStream_t s, int grid) {
    auto kern = decode_w2a8_kernel<MT, MMA, InT, OutT>;
    static int attr_smem[64] = {};
    if (smem > attr_smem[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_smem[dev.device] = smem;
    }
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

}  // namespace

bool decode_w2a8_supported(const void *x, int64_t M, int64_t K) {
    return M >= 1 && M <= 16 && K % 64 == 0 && K <= 8192 && reinterpret_cast<uintptr_t>(x) % 16 == 0;
}

cudaError_t launch_decode_w2a8(const void *x, bq_dtype xt, int64_t M, int64_t K, float eps, const uint32_t *wpacked,
                               const float *w_scale, const float *bias, int64_t N, bq_dtype out_dtype, void *out,
                               int8_t *ws_xq, float *ws_scale, int32_t *ws_rowsum, cudaStream_t s,
                               const DevInfo &dev) {
    const int MT = M == 1 ? 1 : M == 2 ? 2 : M <= 8 ? 8 : 16;
    const int rpc = static_cast<int>((N + dev.num_sms - 1) / dev.num_sms);
    const int grid = static_cast<int>((N + rpc - 1) / rpc);
    const int nchunks = (rpc + CR - 1) / CR;
    const int budget = static_cast<int>(dev.max_smem_optin) - 1024;
    int S = nchunks;
    while (S > 2 && static_cast<int>(Layout(static_cast<int>(K), MT, S).total) > budget) --S;
    if (static_cast<int>(Layout(static_cast<int>(K), MT, S).total) > budget) return cudaErrorInvalidConfiguration;
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
    a.rows_per_cta = rpc;
    a.stages = S;
    a.status = dev.status;
    const Layout lay(static_cast<int>(K), MT, S);
    if (!lay.aligned_ok()) return cudaErrorInvalidConfiguration;
    const int smem = static_cast<int>(lay.total);
    if (xt == BQ_BF16) return dispatch_out<__nv_bfloat16>(a, out_dtype, MT, smem, dev, s, grid);
    return dispatch_out<float>(a, out_dtype, MT, smem, dev, s, grid);
}

}  // namespace bq
