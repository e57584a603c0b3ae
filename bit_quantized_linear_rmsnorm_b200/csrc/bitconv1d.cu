// Ternary Conv1d ("Common Attention Utilities", frankenstein-transformer,
// BitConv1d: the ternary weights and 8-bit activations of BitLinear; the input
// (B, C_in, L) is LayerNorm-normalised over the channels at every position
// before the activation quantization; output (B, C_out, L_out)).
//
//   out[b,co,lo] = gamma * sum_t act_scale[b,p] * sum_c wq[co,c,t] * xq[b,p,g Cg + c]  (+ bias[co])
//   p = lo * stride + t - pad,  L_out = (L + 2 pad - KS) / stride + 1
//
// The activation scale belongs to the input position, so each tap is its own
// integer contraction over the channels, scaled by the scale of the position
// it reads.  The path:
//   1. x (B, C_in, L) -> rows [B*L][C_in] (tiled transpose through shared memory);
//   2. LayerNorm + per-position int8 quantization of those rows (the binary64
//      kernel of act_quant_ln.cu): codes and scales;
//   3. per tap t: the rows read by the tap gathered into [B*L_out][C_in]
//      (zero rows and scale where the tap falls into the padding) with their
//      code sums per channel group, then per group the ternary tcgen05 GEMM
//      against the tap's packed weights [C_out/groups][C_in/groups], which
//      computes (acc - rowsum) * scale * gamma in fp32;
//   4. the taps summed in fp32 (+ bias), rounded once and transposed into
//      (B, C_out, L_out).
// Weights are packed per tap by bq_bitconv1d_weight_pack: [KS][C_out][Cgp/16]
// words with Cgp = Cg rounded up to 64 (16-byte row pitch for the tensor copy).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "bq_internal.h"

namespace bq {
namespace {

// 64 x 64 tiles: src [batch][R][C] -> dst [batch][C][R] (element type T,
// 2 or 4 bytes).  A thread loads 4 consecutive elements of a source row as
// one vector and, after the tile is in shared memory, writes 4 consecutive
// elements of a destination row as one vector (8 or 16 bytes per access on
// both sides); the tile rows are padded by one element, which leaves at most
// a 2-way bank conflict on the column reads.  Ragged or unaligned edges fall
// back to element accesses.
template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
    using V = float4;
    __device__ static void split(const V &v, float (&e)[4]) {
        e[0] = v.x;
        e[1] = v.y;
        e[2] = v.z;
        e[3] = v.w;
    }
    __device__ static V join(const float (&e)[4]) { return make_float4(e[0], e[1], e[2], e[3]); }
};
template <>
struct Vec4<__nv_bfloat16> {
    using V = uint2;
    __device__ static void split(const V &v, __nv_bfloat16 (&e)[4]) {
        e[0] = __ushort_as_bfloat16(static_cast<unsigned short>(v.x & 0xffffu));
        e[1] = __ushort_as_bfloat16(static_cast<unsigned short>(v.x >> 16));
        e[2] = __ushort_as_bfloat16(static_cast<unsigned short>(v.y & 0xffffu));
        e[3] = __ushort_as_bfloat16(static_cast<unsigned short>(v.y >> 16));
    }
    __device__ static V join(const __nv_bfloat16 (&e)[4]) {
        return make_uint2(static_cast<uint32_t>(__bfloat16_as_ushort(e[0])) |
                              (static_cast<uint32_t>(__bfloat16_as_ushort(e[1])) << 16),
                          static_cast<uint32_t>(__bfloat16_as_ushort(e[2])) |
                              (static_cast<uint32_t>(__bfloat16_as_ushort(e[3])) << 16));
    }
};

constexpr int kTr = 64;  // tile edge
template <typename T>
__global__ void __launch_bounds__(256) transpose_kernel(const T *__restrict__ src, int64_t R, int64_t C,
                                                       T *__restrict__ dst) {
    using V = typename Vec4<T>::V;
    __shared__ T tile[kTr][kTr + 1];
    const int64_t b = blockIdx.z;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTr, c0 = static_cast<int64_t>(blockIdx.x) * kTr;
    const T *s = src + b * R * C;
    T *d = dst + b * R * C;
    const int q = threadIdx.x & 15, h = threadIdx.x >> 4;  // 4-element group q of a line, line h (+ 16 i)
    const bool cvec = C % 4 == 0 && reinterpret_cast<uintptr_t>(src) % sizeof(V) == 0;
    const bool rvec = R % 4 == 0 && reinterpret_cast<uintptr_t>(dst) % sizeof(V) == 0;
#pragma unroll
    for (int i = 0; i < kTr / 16; ++i) {
        const int tr = h + 16 * i;
        const int64_t r = r0 + tr, c = c0 + 4 * q;
        T e[4];
        if (r < R && cvec && c + 3 < C) {
            Vec4<T>::split(__ldg(reinterpret_cast<const V *>(s + r * C + c)), e);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) e[j] = (r < R && c + j < C) ? s[r * C + c + j] : T{};
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) tile[tr][4 * q + j] = e[j];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kTr / 16; ++i) {
        const int tc = h + 16 * i;
        const int64_t c = c0 + tc, r = r0 + 4 * q;
        if (c >= C) continue;
        T e[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) e[j] = tile[4 * q + j][tc];
        if (rvec && r + 3 < R) {
            *reinterpret_cast<V *>(d + c * R + r) = Vec4<T>::join(e);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (r + j < R) d[c * R + r + j] = e[j];
        }
    }
}

template <typename T>
cudaError_t transpose(const T *src, int64_t batch, int64_t R, int64_t C, T *dst, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>((C + kTr - 1) / kTr), static_cast<unsigned>((R + kTr - 1) / kTr),
                    static_cast<unsigned>(batch));
    transpose_kernel<T><<<grid, 256, 0, s>>>(src, R, C, dst);
    return cudaGetLastError();
}

// Rows of tap t: row (b, lo) of the gathered codes is row (b, p) of xq, p =
// lo * stride + t - pad, or zeros outside [0, L); rs[row] is that position's
// scale (0 outside) and rc[g * rows + row] the sum of its codes over the
// channels of group g (the offset-binary correction of that group's product).
// With a == nullptr only rs and rc are written (stride 1: the padded scale and
// code-sum arrays, L_out = L + 2 pad rows per batch, t = 0).
// One warp per row; a 16-byte chunk lies inside one group (Cg % 16 == 0), its
// code sum goes to the warp's group counters in shared memory.
constexpr int kGatherWarps = 8;
__global__ void __launch_bounds__(kGatherWarps * 32)
    tap_gather_kernel(const int8_t *__restrict__ xq, const float *__restrict__ act_scale, int64_t B, int64_t C_in,
                      int64_t L, int64_t L_out, int64_t stride, int64_t pad, int64_t t, int64_t groups,
                      int8_t *__restrict__ a, float *__restrict__ rs, int32_t *__restrict__ rc) {
    extern __shared__ int gsum[];  // [kGatherWarps][groups]
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    int *mine = gsum + wib * groups;
    const int64_t rows = B * L_out, chunks = C_in / 16, cpg = (C_in / groups) / 16;
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * kGatherWarps + wib; row < rows;
         row += static_cast<int64_t>(gridDim.x) * kGatherWarps) {
        const int64_t b = row / L_out, lo = row - b * L_out, p = lo * stride + t - pad;
        const bool in = p >= 0 && p < L;
        for (int64_t gi = lane; gi < groups; gi += 32) mine[gi] = 0;
        __syncwarp();
        const uint4 *src = reinterpret_cast<const uint4 *>(xq + (b * L + (in ? p : 0)) * C_in);
        uint4 *dst = a != nullptr ? reinterpret_cast<uint4 *>(a + row * C_in) : nullptr;
        int lsum = 0;  // one group: this lane's part of the row sum
        for (int64_t c = lane; c < chunks; c += 32) {
            const uint4 v = in ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            if (dst != nullptr) dst[c] = v;
            int sum = __dp4a(static_cast<int>(v.x), 0x01010101, 0);
            sum = __dp4a(static_cast<int>(v.y), 0x01010101, sum);
            sum = __dp4a(static_cast<int>(v.z), 0x01010101, sum);
            sum = __dp4a(static_cast<int>(v.w), 0x01010101, sum);
            if (groups == 1)
                lsum += sum;
            else
                atomicAdd(mine + c / cpg, sum);
        }
        if (groups == 1) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
            if (lane == 0) mine[0] = lsum;
        }
        __syncwarp();
        for (int64_t gi = lane; gi < groups; gi += 32) rc[gi * rows + row] = mine[gi];
        if (lane == 0) rs[row] = in ? __ldg(act_scale + b * L + p) : 0.0f;
        __syncwarp();
    }
}

// out[b, co, lo] = sum_t part[t][(b L_out + lo) * ldp + co] (+ bias[co]), through a
// 32 (lo) x 128 (co) shared-memory tile: 16-byte reads along co, writes along lo.
template <typename OutT>
__global__ void __launch_bounds__(256) tap_sum_kernel(const float *__restrict__ part, int64_t KS, int64_t B,
                                                      int64_t L_out, int64_t C_out, int64_t ldp,
                                                      const float *__restrict__ bias, OutT *__restrict__ out) {
    __shared__ float tile[32][129];
    const int64_t b = blockIdx.z;
    const int64_t l0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 128;
    const int64_t tap_stride = B * L_out * ldp;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    const int64_t co = c0 + 4 * tx;
    for (int i = ty; i < 32; i += 8) {
        const int64_t lo = l0 + i;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lo < L_out && co < C_out) {
            const float *p = part + (b * L_out + lo) * ldp + co;
            if (co + 4 <= ldp) {
                for (int64_t t = 0; t < KS; ++t) {
                    const float4 q = __ldcs(reinterpret_cast<const float4 *>(p + t * tap_stride));
                    v.x = __fadd_rn(v.x, q.x);
                    v.y = __fadd_rn(v.y, q.y);
                    v.z = __fadd_rn(v.z, q.z);
                    v.w = __fadd_rn(v.w, q.w);
                }
            }
        }
        const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float r = e[j];
            if (bias != nullptr && co + j < C_out) r = __fadd_rn(r, __ldg(bias + co + j));
            tile[i][4 * tx + j] = r;
        }
    }
    __syncthreads();
    for (int cc = ty; cc < 128; cc += 8) {
        const int64_t c = c0 + cc, lo = l0 + tx;
        if (c < C_out && lo < L_out) {
            const float v = tile[tx][cc];
            OutT o;
            if constexpr (sizeof(OutT) == 4)
                o = v;
            else if constexpr (std::is_same<OutT, __half>::value)
                o = __float2half_rn(v);
            else
                o = __float2bfloat16_rn(v);
            out[(b * C_out + c) * L_out + lo] = o;
        }
    }
}

inline size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

}  // namespace

BitconvLayout bitconv_layout(int64_t B, int64_t C_in, int64_t L, int64_t C_out, int64_t KS, int64_t stride,
                             int64_t pad, int64_t groups) {
    BitconvLayout l;
    l.L_out = (L + 2 * pad - KS) / stride + 1;
    l.ldp = (C_out + 3) / 4 * 4;
    const size_t rows = static_cast<size_t>(B * L), orows = static_cast<size_t>(B * l.L_out);
    l.xt = 0;
    l.xq = l.xt + a256(rows * static_cast<size_t>(C_in) * 4);
    l.scale = l.xq + a256(rows * static_cast<size_t>(C_in));
    l.a = l.scale + a256(rows * 4);
    size_t a_bytes = orows * static_cast<size_t>(C_in);  // gathered codes, or (stride 1) the padded arrays
    if (stride == 1) {
        const size_t lp = static_cast<size_t>(B * (L + 2 * pad));
        a_bytes = std::max(a_bytes, a256(lp * 4) + static_cast<size_t>(groups) * lp * 4);
    }
    l.rs = l.a + a256(a_bytes);
    l.rc = l.rs + a256(orows * 4);
    l.part = l.rc + a256(orows * static_cast<size_t>(groups) * 4);
    l.total = l.part + a256(static_cast<size_t>(KS) * orows * static_cast<size_t>(l.ldp) * 4);
    return l;
}

cudaError_t launch_bitconv_weight_transpose(const void *w, bq_dtype wt, int64_t C_out, int64_t Cg, int64_t KS,
                                            void *dst, cudaStream_t s) {
    // [C_out * Cg][KS] -> [KS][C_out * Cg]
    if (wt == BQ_BF16)
        return transpose(static_cast<const __nv_bfloat16 *>(w), 1, C_out * Cg, KS, static_cast<__nv_bfloat16 *>(dst),
                         s);
    return transpose(static_cast<const float *>(w), 1, C_out * Cg, KS, static_cast<float *>(dst), s);
}

bq_status launch_bitconv1d(const void *x, bq_dtype xt, int64_t B, int64_t C_in, int64_t L, const float *ln_weight,
                           const float *ln_bias, const uint32_t *wpacked, const float *w_scale, int64_t C_out,
                           int64_t KS, int64_t stride, int64_t pad, int64_t groups, const float *bias, float eps,
                           bq_dtype out_dtype, void *out, void *workspace, cudaStream_t s, const DevInfo &dev) {
    const BitconvLayout l = bitconv_layout(B, C_in, L, C_out, KS, stride, pad, groups);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // 1. (B, C_in, L) -> [B*L][C_in]
    cudaError_t e = xt == BQ_BF16 ? transpose(static_cast<const __nv_bfloat16 *>(x), B, C_in, L,
                                              reinterpret_cast<__nv_bfloat16 *>(ws + l.xt), s)
                                  : transpose(static_cast<const float *>(x), B, C_in, L,
                                              reinterpret_cast<float *>(ws + l.xt), s);
    if (e != cudaSuccess) return BQ_ERR_CUDA;
    // 2. per-position LayerNorm + int8 codes
    int8_t *xq = reinterpret_cast<int8_t *>(ws + l.xq);
    float *act_scale = reinterpret_cast<float *>(ws + l.scale);
    e = launch_act_quant_ln(ws + l.xt, xt, B * L, C_in, C_in, ln_weight, ln_bias, eps, xq, C_in, act_scale, nullptr, s,
                            dev);
    if (e != cudaSuccess) return BQ_ERR_CUDA;
    // 3. per tap: gather, ternary GEMM into the tap's fp32 partial
    const int64_t orows = B * l.L_out, Cg = C_in / groups, Cog = C_out / groups, Cgp = (Cg + 63) / 64 * 64;
    int8_t *a = reinterpret_cast<int8_t *>(ws + l.a);
    float *rs = reinterpret_cast<float *>(ws + l.rs);
    int32_t *rc = reinterpret_cast<int32_t *>(ws + l.rc);  // [groups][rows]
    float *part = reinterpret_cast<float *>(ws + l.part);
    const size_t gsmem = static_cast<size_t>(kGatherWarps) * static_cast<size_t>(groups) * 4;
    auto gather_grid = [&](int64_t nrows) {
        return static_cast<int>(
            std::max<int64_t>(1, std::min<int64_t>((nrows + kGatherWarps - 1) / kGatherWarps, dev.num_sms * 16)));
    };
    if (stride == 1) {
        // Tap t of output row (b, lo) reads codes row (b, lo + t - pad): the GEMM reads
        // the codes in place as [B][L][C_in] at a row offset, the tensor copies
        // filling rows outside [0, L) with zeros (the padding); the scale and the code
        // sums come from per-batch arrays padded with zeros, L + 2 pad long, built once.
        const int64_t Lp = L + 2 * pad;
        float *rsp = reinterpret_cast<float *>(a);
        int32_t *rcp = reinterpret_cast<int32_t *>(a + a256(static_cast<size_t>(B * Lp) * 4));  // [groups][B][Lp]
        tap_gather_kernel<<<gather_grid(B * Lp), kGatherWarps * 32, gsmem, s>>>(xq, act_scale, B, C_in, L, Lp, 1, pad,
                                                                               0, groups, nullptr, rsp, rcp);
        if (cudaGetLastError() != cudaSuccess) return BQ_ERR_CUDA;
        for (int64_t t = 0; t < KS; ++t)
            for (int64_t gr = 0; gr < groups; ++gr) {
                GemmArgs g;
                g.a = xq + gr * Cg;
                g.lda = C_in;
                g.batch = B;
                g.sa = L * C_in;
                g.a_rows = L;
                g.a_row_off = t - pad;
                g.b = wpacked + (t * C_out + gr * Cog) * (Cgp / 16);
                g.ldb = Cgp / 16;
                g.b_pack = 2;
                g.colscale = w_scale;
                g.rowscale = rsp + t;
                g.rowcorr = rcp + gr * B * Lp + t;
                g.s_row = Lp;
                g.M = l.L_out;
                g.N = Cog;
                g.K = Cg;
                g.out_dtype = BQ_F32;
                g.out = part + t * orows * l.ldp + gr * Cog;
                g.ldo = l.ldp;
                g.so = l.L_out * l.ldp;
                const bq_status st = launch_gemm_tc(g, s, dev);
                if (st != BQ_OK) return st;
            }
    } else {
        for (int64_t t = 0; t < KS; ++t) {
            tap_gather_kernel<<<gather_grid(orows), kGatherWarps * 32, gsmem, s>>>(xq, act_scale, B, C_in, L, l.L_out,
                                                                                 stride, pad, t, groups, a, rs, rc);
            if (cudaGetLastError() != cudaSuccess) return BQ_ERR_CUDA;
            for (int64_t gr = 0; gr < groups; ++gr) {  // group gr: its channels, weight rows and output columns
                GemmArgs g;
                g.a = a + gr * Cg;
                g.lda = C_in;
                g.b = wpacked + (t * C_out + gr * Cog) * (Cgp / 16);
                g.ldb = Cgp / 16;
                g.b_pack = 2;
                g.colscale = w_scale;
                g.rowscale = rs;
                g.rowcorr = rc + gr * orows;
                g.M = orows;
                g.N = Cog;
                g.K = Cg;
                g.out_dtype = BQ_F32;
                g.out = part + t * orows * l.ldp + gr * Cog;
                g.ldo = l.ldp;
                const bq_status st = launch_gemm_tc(g, s, dev);
                if (st != BQ_OK) return st;
            }
        }
    }
    // 4. sum the taps (+ bias), transpose to (B, C_out, L_out)
    const dim3 grid(static_cast<unsigned>((C_out + 127) / 128), static_cast<unsigned>((l.L_out + 31) / 32),
                    static_cast<unsigned>(B));
    switch (out_dtype) {
        case BQ_F32:
            tap_sum_kernel<float><<<grid, 256, 0, s>>>(part, KS, B, l.L_out, C_out, l.ldp, bias,
                                                       static_cast<float *>(out));
            break;
        case BQ_F16:
            tap_sum_kernel<__half><<<grid, 256, 0, s>>>(part, KS, B, l.L_out, C_out, l.ldp, bias,
                                                        static_cast<__half *>(out));
            break;
        default:
            tap_sum_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(part, KS, B, l.L_out, C_out, l.ldp, bias,
                                                               static_cast<__nv_bfloat16 *>(out));
    }
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace bq
