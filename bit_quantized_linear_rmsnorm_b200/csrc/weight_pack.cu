// Weight preparation kernels (one-time, HBM-bound):
//
//  * Absmean ternary quantization + 2-bit packing ("Common Attention
//    Utilities" (frankenstein-transformer): weight_quant and
//    BitLinear.bake_ternary_weights; "Class BitLinear" forward step 3).
//    Pass 1 reduces sum|w| in fp64 plus max|w| and the smallest nonzero |w|
//    into a fixed number of partials (deterministic: the partition depends
//    only on the tensor size).  Pass 2 re-reduces the partials in every
//    block in the same order, derives gamma (the bake rule: a tensor whose
//    nonzero magnitudes all equal max|w| keeps gamma = max|w|), then writes
//    one packed word per 16 weights.
//
//  * INT4 packing ("vyre_libs/nn/linear/inner/linear_4bit/mod.rs", module
//    doc and QuantizedLinear4BitSpec): eight nibbles per u32, low nibble
//    first, for the codes [N][K] and the zero-points [N][G].
#include <cuda_bf16.h>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

struct Partial {
    double sum;   // sum |w|
    float amax;   // max |w|
    float minnz;  // min nonzero |w| (+inf if none)
};
static_assert(sizeof(Partial) == 16, "Partial layout");

constexpr int kReduceThreads = 256;
constexpr int kMaxPartials = 1024;

__host__ __device__ inline int64_t num_partials(int64_t n_el) {
    int64_t p = (n_el + 4095) / 4096;
    if (p < 1) p = 1;
    if (p > kMaxPartials) p = kMaxPartials;
    return p;
}

__device__ __forceinline__ void accum(float v, double &s, float &mx, float &mn) {
    const float a = fabsf(v);
    s += static_cast<double>(a);
    mx = fmaxf(mx, a);
    if (a != 0.0f) mn = fminf(mn, a);
}

// Block reduction in a fixed tree order.
__device__ void block_reduce(double &s, float &mx, float &mn) {
    __shared__ double ss[kReduceThreads];
    __shared__ float sx[kReduceThreads], sn[kReduceThreads];
    const int t = threadIdx.x;
    ss[t] = s;
    sx[t] = mx;
    sn[t] = mn;
    __syncthreads();
    for (int o = kReduceThreads / 2; o > 0; o >>= 1) {
        if (t < o) {
            ss[t] += ss[t + o];
            sx[t] = fmaxf(sx[t], sx[t + o]);
            sn[t] = fminf(sn[t], sn[t + o]);
        }
        __syncthreads();
    }
    s = ss[0];
    mx = sx[0];
    mn = sn[0];
    __syncthreads();
}

template <typename In>
__device__ __forceinline__ float ld_elt(const In *p, int64_t i);
template <>
__device__ __forceinline__ float ld_elt<float>(const float *p, int64_t i) {
    return __ldg(p + i);
}
template <>
__device__ __forceinline__ float ld_elt<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
}

template <typename In>
__global__ void __launch_bounds__(kReduceThreads)
    ternary_reduce_kernel(const In *__restrict__ w, int64_t n_el, Partial *__restrict__ parts) {
    double s = 0.0;
    float mx = 0.0f, mn = __int_as_float(0x7f800000);
    // contiguous slice per block, strided by thread inside it
    const int64_t P = gridDim.x;
    const int64_t per = (n_el + P - 1) / P;
    const int64_t lo = blockIdx.x * per;
    const int64_t hi = lo + per < n_el ? lo + per : n_el;
    for (int64_t i = lo + threadIdx.x; i < hi; i += kReduceThreads) accum(ld_elt(w, i), s, mx, mn);
    block_reduce(s, mx, mn);
    if (threadIdx.x == 0) parts[blockIdx.x] = Partial{s, mx, mn};
}

template <typename In>
__global__ void __launch_bounds__(kReduceThreads)
    ternary_pack_kernel(const In *__restrict__ w, int64_t N, int64_t K, const Partial *__restrict__ parts,
                        int64_t nparts, uint32_t *__restrict__ wpacked, float *__restrict__ w_scale) {
    double s = 0.0;
    float mx = 0.0f, mn = __int_as_float(0x7f800000);
    for (int64_t p = threadIdx.x; p < nparts; p += kReduceThreads) {
        const Partial q = parts[p];
        s += q.sum;
        mx = fmaxf(mx, q.amax);
        mn = fminf(mn, q.minnz);
    }
    block_reduce(s, mx, mn);
    const bool already_ternary = (mx > 0.0f) && (mn == mx);
    double g = already_ternary ? static_cast<double>(mx) : s / static_cast<double>(N * K);
    if (!already_ternary && g < 1e-5) g = 1e-5;
    const float gf = static_cast<float>(g);
    if (blockIdx.x == 0 && threadIdx.x == 0) *w_scale = gf;

    const int64_t words = N * (K / 16);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kReduceThreads + threadIdx.x; i < words;
         i += static_cast<int64_t>(gridDim.x) * kReduceThreads) {
        const In *src = w + i * 16;  // rows are whole words: K % 16 == 0
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float v = __fdiv_rn(ld_elt(src, e), gf);
            const float q = fminf(fmaxf(rintf(v), -1.0f), 1.0f);
            const uint32_t code = static_cast<uint32_t>(static_cast<int>(q) + 1);
            const int j = e >> 2, b = e & 3;  // element 4j + b of the word
            word |= code << (8 * b + 2 * j);
        }
        wpacked[i] = word;
    }
}

__global__ void int4_pack_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ zeros, int64_t N,
                                 int64_t K, int64_t G, uint32_t *__restrict__ qweight,
                                 uint32_t *__restrict__ qzeros, uint32_t *status) {
    const int64_t wwords = N * (K / 8);
    const int64_t zrow = (G + 7) / 8;
    const int64_t zwords = N * zrow;
    bool bad = false;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < wwords + zwords;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint32_t word = 0;
        if (i < wwords) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(q) + i);
            bad |= ((v.x | v.y) & 0xf0f0f0f0u) != 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                word |= ((v.x >> (8 * j)) & 15u) << (4 * j);
                word |= ((v.y >> (8 * j)) & 15u) << (4 * (j + 4));
            }
            qweight[i] = word;
        } else {
            const int64_t zi = i - wwords;
            const int64_t n = zi / zrow, wi = zi % zrow;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int64_t g = wi * 8 + j;
                if (g < G) {
                    const uint32_t z = zeros[n * G + g];
                    bad |= z > 15u;
                    word |= (z & 15u) << (4 * j);
                }
            }
            qzeros[zi] = word;
        }
    }
    if (bad) report(status, BQ_ERR_INVALID_ARG, SITE_INT4_PACK);
}

template <typename In>
cudaError_t ternary_typed(const In *w, int64_t N, int64_t K, uint32_t *wpacked, float *w_scale, void *ws,
                          cudaStream_t s, const DevInfo &dev) {
    const int64_t n_el = N * K;
    const int64_t P = num_partials(n_el);
    Partial *parts = static_cast<Partial *>(ws);
    ternary_reduce_kernel<In><<<static_cast<unsigned>(P), kReduceThreads, 0, s>>>(w, n_el, parts);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t words = N * (K / 16);
    int64_t grid = (words + kReduceThreads - 1) / kReduceThreads;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    ternary_pack_kernel<In><<<static_cast<unsigned>(grid), kReduceThreads, 0, s>>>(w, N, K, parts, P, wpacked,
                                                                                  w_scale);
    return cudaGetLastError();
}

}  // namespace

size_t ternary_pack_workspace_bytes(int64_t N, int64_t K) {
    return static_cast<size_t>(num_partials(N * K)) * sizeof(Partial);
}

cudaError_t launch_ternary_pack(const void *w, bq_dtype wt, int64_t N, int64_t K, uint32_t *wpacked,
                                float *w_scale, void *ws, cudaStream_t s, const DevInfo &dev) {
    if (wt == BQ_BF16)
        return ternary_typed(static_cast<const __nv_bfloat16 *>(w), N, K, wpacked, w_scale, ws, s, dev);
    return ternary_typed(static_cast<const float *>(w), N, K, wpacked, w_scale, ws, s, dev);
}

cudaError_t launch_int4_pack(const uint8_t *q, const uint8_t *zeros, int64_t N, int64_t K, int64_t group_size,
                             uint32_t *qweight, uint32_t *qzeros, cudaStream_t s, const DevInfo &dev) {
    const int64_t G = K / group_size;
    const int64_t total = N * (K / 8) + N * ((G + 7) / 8);
    int64_t grid = (total + 255) / 256;
    const int64_t cap = static_cast<int64_t>(dev.num_sms) * 16;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    int4_pack_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(q, zeros, N, K, G, qweight, qzeros,
                                                                 dev.status);
    return cudaGetLastError();
}

}  // namespace bq
