// bf16 x bf16 -> fp32 GEMM on the sm_100a tensor cores (tcgen05.mma
// kind::f16), used by the straight-through backward of BitLinear ("Class
// BitLinear" (LLaMA-BitNet utils.py): activations and weights quantized "with
// STE"; "Common Attention Utilities": the STE "passes gradients through the
// rounding operation unchanged"):
//
//   D[m,n] = scale * sum_k A(m,k) * B(k,n)          (fp32 accumulators in TMEM)
//
// A is K-major ([M][lda], k contiguous) or M-major ([K][lda], m contiguous);
// B is K-major ([N][ldb]) or N-major ([K][ldb], n contiguous).  The operands
// of the backward are exact in bf16 (gradients given in bf16, ternary codes
// -1/0/1, int8 activation codes) or split into exact hi + lo bf16 parts by
// the caller, so the only roundings are the fp32 accumulation and the scale.
//
// One CTA per SM, persistent over 128 x 256 output tiles:
//   warp 0      TMA producer: per 64-element K step a 128 x 64 A tile and a
//               256 x 64 B tile (128-byte swizzle; M- or N-major tiles arrive
//               as 64-wide boxes), mbarrier transaction counts.
//   warp 1      MMA issuer: one thread, 4 x tcgen05.mma (K = 16 each) per
//               stage into a TMEM accumulator, commits to free the stage.
//   warp 2      allocates / frees 512 TMEM columns (two 256-column
//               accumulators: the epilogue of tile t overlaps tile t + 1).
//   warps 4-7   epilogue: tcgen05.ld 32 columns at a time, scale, stage
//               through a 64-byte-swizzled buffer, TMA store (clipped at the
//               matrix edges).
// Every wait is bounded; on expiry the kernel records BQ_ERR_TIMEOUT in the
// status word, drains its own asynchronous work and exits.
#include <cudaTypedefs.h>

#include <algorithm>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

constexpr int FBM = 128;
constexpr int FBN = 256;
constexpr int FBK = 64;   // bf16 elements per stage = one 128-byte swizzle row
constexpr int FUK = 16;   // K of one kind::f16 MMA
constexpr int FS = 4;     // stages
constexpr uint32_t FA_BYTES = FBM * 128;   // 16 KB
constexpr uint32_t FB_BYTES = FBN * 128;   // 32 KB
constexpr uint32_t FSTG_BYTES = FBM * 64;  // 8 KB epilogue staging
constexpr uint32_t kFTmemCols = 512;

struct FCfg {
    static constexpr uint32_t OFF_A = 0;
    static constexpr uint32_t OFF_B = OFF_A + FS * FA_BYTES;
    static constexpr uint32_t OFF_STG = OFF_B + FS * FB_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_STG + 2 * FSTG_BYTES;
    static constexpr uint32_t NBAR = 2 * FS + 5;  // full[S], empty[S], tfull[2], tempty[2], drain
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;
};
static_assert(FCfg::SMEM <= 232448, "stages exceed the shared memory of a CTA");

struct Bf16Dev {
    int M, N, K;
    const float *scale;  // one fp32 on the device, or nullptr for 1
    uint32_t *status;
};

// Instruction descriptor of kind::f16 with bf16 A and B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                                 // D format: f32
           | (1u << 7)                               // A format: bf16
           | (1u << 10)                              // B format: bf16
           | ((a_mn ? 1u : 0u) << 15)                // A major
           | ((b_mn ? 1u : 0u) << 16)                // B major
           | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// M- / N-major tile of 64-element-wide blocks (128-byte swizzle): K rows 128
// bytes apart, 8-row groups 1024 bytes apart (stride byte offset), the next
// 64-wide block FBK * 128 bytes further (leading byte offset).
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3fffu);
    d |= static_cast<uint64_t>((FBK * 128u) >> 4) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(256, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmO, const Bf16Dev p) {
    using C = FCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (FS + s); };
    auto tfull = [&](int b) { return bar0 + 8u * (2 * FS + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (2 * FS + 2 + b); };
    const uint32_t drain = bar0 + 8u * (2 * FS + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *epi_fail = reinterpret_cast<int *>(smem + C::OFF_MISC + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (p.M + FBM - 1) / FBM, num_n = (p.N + FBN - 1) / FBN;
    const int num_tiles = num_m * num_n;
    const int nkb = (p.K + FBK - 1) / FBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < FS; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *epi_fail = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), kFTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const int m0 = (t % num_m) * FBM, n0 = (t / num_m) * FBN;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, p.status, SITE_GEMM_PRODUCER)) {
                    ok = false;
                    break;
                }
                const uint32_t a_dst = sbase + C::OFF_A + stage * FA_BYTES;
                const uint32_t b_dst = sbase + C::OFF_B + stage * FB_BYTES;
                const int k0 = kb * FBK;
                mbar_arrive_expect_tx(full(stage), FA_BYTES + FB_BYTES);
                if constexpr (A_MN) {
                    tma_load_2d(a_dst, &tmA, m0, k0, full(stage));
                    tma_load_2d(a_dst + FBK * 128, &tmA, m0 + 64, k0, full(stage));
                } else {
                    tma_load_2d(a_dst, &tmA, k0, m0, full(stage));
                }
                if constexpr (B_MN) {
#pragma unroll
                    for (int j = 0; j < FBN / 64; ++j) tma_load_2d(b_dst + j * FBK * 128, &tmB, n0 + 64 * j, k0, full(stage));
                } else {
                    tma_load_2d(b_dst, &tmB, k0, n0, full(stage));
                }
                ++issued;
                if (++stage == FS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // let the copies issued land before the CTA can go away
        for (int64_t i = issued > FS ? issued - FS : 0; i < issued; ++i)
            mbar_drain(full(static_cast<int>(i % FS)), static_cast<uint32_t>((i / FS) & 1), kWaitLimitNs);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_bf16(FBM, FBN, A_MN, B_MN);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int i = 0;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++i) {
            const int abuf = i & 1;
            const uint32_t aphase = static_cast<uint32_t>(i >> 1) & 1u;
            if (!mbar_wait(tempty(abuf), aphase ^ 1u, abort_flag, p.status, SITE_GEMM_MMA)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tbase + static_cast<uint32_t>(abuf * FBN);
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(full(stage), phase, abort_flag, p.status, SITE_GEMM_MMA)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = sbase + C::OFF_A + stage * FA_BYTES;
                const uint32_t b_addr = sbase + C::OFF_B + stage * FB_BYTES;
#pragma unroll
                for (int ks = 0; ks < FBK / FUK; ++ks) {
                    // a K step of 16 elements: 32 bytes along a K-major row, 16 rows of a M/N-major tile
                    const uint64_t ad = A_MN ? desc_mn_sw128(a_addr + ks * FUK * 128)
                                             : smem_desc_kmajor_sw128(a_addr + ks * FUK * 2);
                    const uint64_t bd = B_MN ? desc_mn_sw128(b_addr + ks * FUK * 128)
                                             : smem_desc_kmajor_sw128(b_addr + ks * FUK * 2);
                    tc_mma_f16(d_tmem, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
                }
                tc_commit(empty(stage));
                if (++stage == FS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit(tfull(abuf));
        }
        if (!ok) {
            tc_commit(drain);
            mbar_drain(drain, 0, kWaitLimitNs);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int q = warp - 4, r = 32 * q + lane, et = threadIdx.x - 128;
        uint8_t *stg = smem + C::OFF_STG;
        const float scale = p.scale != nullptr ? __ldg(p.scale) : 1.0f;
        uint32_t chunk_ctr = 0;
        int i = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++i) {
            const int m0 = (t % num_m) * FBM, n0 = (t / num_m) * FBN;
            const int abuf = i & 1;
            const uint32_t aphase = static_cast<uint32_t>(i >> 1) & 1u;
            bool ok = true;
            if (lane == 0) ok = mbar_wait_timed(tfull(abuf), aphase, p.status, SITE_GEMM_EPILOGUE);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok && lane == 0) {
                atomicOr(epi_fail, 1);
                *abort_flag = 1;
            }
            named_bar_sync(1, 128);
            if (*reinterpret_cast<volatile int *>(epi_fail)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c32 = 0; c32 < FBN / 32; ++c32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(abuf * FBN + c32 * 32) +
                                       (static_cast<uint32_t>(32 * q) << 16),
                                   v);
                tmem_wait_ld();
                if (c32 == FBN / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(tempty(abuf));
                }
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(__fmul_rn(__uint_as_float(v[j]), scale));
#pragma unroll
                for (int sc = 0; sc < 2; ++sc) {  // 16 fp32 columns = one 64-byte staging row
                    const uint32_t sb = chunk_ctr & 1u;
                    if (et == 0) bulk_wait_read<1>();
                    named_bar_sync(1, 128);
                    uint8_t *rowp = stg + sb * FSTG_BYTES + r * 64;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int pj = j ^ ((r >> 1) & 3);
                        *reinterpret_cast<uint4 *>(rowp + pj * 16) =
                            make_uint4(w[sc * 16 + 4 * j], w[sc * 16 + 4 * j + 1], w[sc * 16 + 4 * j + 2],
                                       w[sc * 16 + 4 * j + 3]);
                    }
                    fence_proxy_async_smem();
                    named_bar_sync(1, 128);
                    if (et == 0) {
                        tma_store_2d(&tmO, smem_u32(stg + sb * FSTG_BYTES), n0 + c32 * 32 + sc * 16, m0);
                        bulk_commit();
                    }
                    ++chunk_ctr;
                }
            }
        }
        if (et == 0) bulk_wait_all();
    }

    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, kFTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_bf16() {
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

bool map2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
           uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    auto fn = encode_fn_bf16();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN>
bq_status launch_bf16_t(const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mO, const Bf16Dev &p,
                        cudaStream_t s, const DevInfo &dev) {
    auto kern = gemm_bf16_kernel<A_MN, B_MN>;
    static SmemOptIn opt_in;
    if (smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), static_cast<size_t>(FCfg::SMEM)) != cudaSuccess)
        return BQ_ERR_CUDA;
    const int64_t tiles = static_cast<int64_t>((p.M + FBM - 1) / FBM) * ((p.N + FBN - 1) / FBN);
    const int grid = static_cast<int>(std::min<int64_t>(tiles, dev.num_sms));
    kern<<<grid, 256, FCfg::SMEM, s>>>(mA, mB, mO, p);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace

bq_status launch_gemm_bf16(const Bf16Args &g, cudaStream_t s, const DevInfo &dev) {
    CUtensorMap mA, mB, mO;
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const bool okA = g.a_mn ? map2d(&mA, bf, g.a, g.M, g.K, g.lda * 2, 64, FBK, CU_TENSOR_MAP_SWIZZLE_128B)
                            : map2d(&mA, bf, g.a, g.K, g.M, g.lda * 2, FBK, FBM, CU_TENSOR_MAP_SWIZZLE_128B);
    const bool okB = g.b_mn ? map2d(&mB, bf, g.b, g.N, g.K, g.ldb * 2, 64, FBK, CU_TENSOR_MAP_SWIZZLE_128B)
                            : map2d(&mB, bf, g.b, g.K, g.N, g.ldb * 2, FBK, FBN, CU_TENSOR_MAP_SWIZZLE_128B);
    const bool okO = map2d(&mO, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.out, g.N, g.M, g.ldo * 4, 16, FBM,
                           CU_TENSOR_MAP_SWIZZLE_64B);
    if (!okA || !okB || !okO) return BQ_ERR_CUDA;
    Bf16Dev p;
    p.M = static_cast<int>(g.M);
    p.N = static_cast<int>(g.N);
    p.K = static_cast<int>(g.K);
    p.scale = g.scale;
    p.status = dev.status;
    if (g.a_mn) return g.b_mn ? launch_bf16_t<true, true>(mA, mB, mO, p, s, dev) : launch_bf16_t<true, false>(mA, mB, mO, p, s, dev);
    return g.b_mn ? launch_bf16_t<false, true>(mA, mB, mO, p, s, dev) : launch_bf16_t<false, false>(mA, mB, mO, p, s, dev);
}

}  // namespace bq
