// Integer GEMMs on the sm_100a tensor cores (tcgen05.mma kind::i8) with a
// fused dequantizing epilogue.
//
//  * W8A8 per-token ("Per-token Quantization for Matmul", Huawei CANN ATB:
//    Input/Output tables and the Example):
//        out[m,n] = (float(acc) * deqScale[n]) * perTokenScale[m] (+ bias[n])
//    with the weight either [N][K] (K-major) or [K][N] (N-major operand).
//  * W2A8 BitLinear prefill ("Class BitLinear", LLaMA-BitNet utils.py,
//    forward steps 4-5): the weight arrives as 2-bit offset-binary codes;
//    unpack warps expand each TMA-staged packed tile to u8 codes in the
//    swizzled shared-memory layout the MMA reads, so no int8 copy of the
//    weight ever exists in global memory.  acc(codes) - rowsum(xq) is the
//    exact ternary accumulator:
//        out[m,n] = (float(acc - rowsum[m]) * act_scale[m]) * gamma (+ bias[n])
//
// Two kernels share the roles below.  Large products with K-major (or
// packed) weights run on clusters of two CTAs (gemm_pair_kernel, 256 x 256
// tiles per pair, tcgen05 cta_group::2; described at its definition); the
// rest on single CTAs (gemm_tc_kernel).
//
// Single-CTA structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: A tile (128 x 128 B) and B tile (256 x 128 B, or
//               the 256 x 32 B packed tile) per stage, mbarrier tx-count.
//   warp 1      MMA issuer: one thread issues 4 x tcgen05.mma (K = 32 each)
//               per stage into a TMEM accumulator, commits to free the stage.
//   warp 2      allocates / frees 512 TMEM columns (two 256-column
//               accumulators, so the epilogue of tile t overlaps tile t+1).
//   warps 4-7   epilogue: tcgen05.ld 32 columns at a time (warp w reads TMEM
//               lanes 32*(w%4)..), scale in fp32, round once, stage through a
//               64-byte-swizzled buffer, TMA store (out-of-range rows/cols are
//               clipped by the TMA unit).
//   warps 8-15  (W2A8 only) unpack 2-bit codes into the B stage.
// Every mbarrier wait is bounded; on expiry the kernel records
// BQ_ERR_TIMEOUT in the status word, drains its own async work and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // K bytes per stage = one 128-byte swizzle row
constexpr int UMMA_K = 32;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t A_BYTES = BM * BK;           // 16 KB
constexpr uint32_t B_BYTES = BN * BK;           // 32 KB
constexpr uint32_t STG_BYTES = BM * 64;         // 8 KB epilogue staging buffer

// Packed weights: PK = 0 for int8 B, 2 for ternary offset-binary codes (2 bits,
// unsigned), 4 for signed 4-bit codes.  A 128-K slab of one weight row is
// BK * PK / 32 words.
template <int PK>
constexpr int slab_words() { return PK == 0 ? 0 : BK * PK / 32; }
template <int PK>
constexpr uint32_t p_bytes(int rows) { return static_cast<uint32_t>(rows * slab_words<PK>() * 4); }

template <int PK>
struct Cfg {
    static constexpr bool PACKED = PK != 0;
    static constexpr uint32_t P_BYTES = p_bytes<PK>(BN);  // 8 KB (2-bit) / 16 KB (4-bit) tile
    static constexpr int kStages = PACKED ? 3 : 4;
    static constexpr int kUnpack = 256;  // unpack threads (packed weights)
    static constexpr int kThreads = PACKED ? 256 + kUnpack : 256;
    static constexpr uint32_t OFF_A = 0;
    static constexpr uint32_t OFF_B = OFF_A + kStages * A_BYTES;
    static constexpr uint32_t OFF_P = OFF_B + kStages * B_BYTES;
    static constexpr uint32_t OFF_STG = OFF_P + (PACKED ? kStages * P_BYTES : 0);
    static constexpr uint32_t OFF_VEC = OFF_STG + 2 * STG_BYTES;   // colscale[BN], bias[BN]
    static constexpr uint32_t OFF_BAR = OFF_VEC + 2 * BN * 4;
    // barriers: full[S], empty[S], bready[S], tfull[2], tempty[2], drain
    static constexpr uint32_t NBAR = 3 * kStages + 5;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;      // tmem base, abort flag
    static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;         // + alignment slack
};

struct GemmDev {
    const float *colscale;
    const float *rowscale;
    const int32_t *rowcorr;
    const float *bias;
    int M, N, K;
    int batch;              // independent products (tile coordinate z)
    int64_t s_col, s_row;   // colscale / rowscale (and rowcorr) elements between batches (0: shared)
    int a_row_off;          // (packed B) A row of output row m: m + a_row_off
    int b_shared;           // one B for all batches (batch > 1 with a zero B stride): B tiles at batch 0
    uint32_t *status;
    uint64_t wait_ns;  // limit of every bounded wait
    int withhold_kb;   // (failure-detection check only) K block of the first tile whose copies are never issued
};

template <typename OutT>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Shared-memory descriptor of the N-major B tile (TMA box 128 N x 128 K,
// 128-byte swizzle): K rows 128 bytes apart, 8-row groups 1024 bytes apart
// (stride byte offset), the second 128-wide N half 16 KB further (leading
// byte offset).
__device__ __forceinline__ uint64_t smem_desc_mnmajor_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3fffu);
    d |= static_cast<uint64_t>((BK * 128u) >> 4) << 16;  // leading byte offset: next 128-wide N block
    d |= static_cast<uint64_t>(1024u >> 4) << 32;        // stride byte offset: next 8 K rows
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Work items of the persistent schedule (CTA b takes items b, b + G, ...): the
// full waves of 128 x 256 tiles, then, when the last wave would leave at
// least half of the CTAs idle, each of its tiles as two 128 x 128 halves, so
// the busiest CTAs end half a tile earlier.
struct Items {
    int num_m, per_batch, big, count;
    __device__ Items(int num_tiles, int num_m_, int per_batch_, int G, bool allow)
        : num_m(num_m_), per_batch(per_batch_) {
        const int full = (num_tiles / G) * G, left = num_tiles - full;
        const bool split = allow && left > 0 && 2 * left <= G;
        big = split ? full : num_tiles;
        count = split ? full + 2 * left : num_tiles;
    }
    __device__ void tile(int item, int &b, int &m0, int &n0, bool &half) const {
        const int t = item < big ? item : big + ((item - big) >> 1);
        b = t / per_batch;
        const int r = t - b * per_batch;
        m0 = (r % num_m) * BM;
        n0 = (r / num_m) * BN + (item < big ? 0 : ((item - big) & 1) * (BN / 2));
        half = item >= big;
    }
};

// 16 weights of one 16-byte chunk from the packed slab word(s): ternary codes
// are expanded to u8 codes (w + 1); a signed 4-bit code n goes to the high
// half of its byte, which read as s8 is exactly 16 n (the epilogue divides the
// accumulator by 16, exactly).
template <int PK>
__device__ __forceinline__ uint4 unpack_chunk(const uint32_t *words, int c) {
    if constexpr (PK == 2) {
        const uint32_t u = words[c];
        return make_uint4(u & 0x03030303u, (u >> 2) & 0x03030303u, (u >> 4) & 0x03030303u, (u >> 6) & 0x03030303u);
    } else {
        const uint2 u = reinterpret_cast<const uint2 *>(words)[c];
        uint32_t r[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t w = h ? u.y : u.x;
            const uint32_t lo = (w << 4) & 0xF0F0F0F0u, hi = w & 0xF0F0F0F0u;  // even / odd nibbles, 16 n as s8
            r[2 * h] = __byte_perm(lo, hi, 0x5140);
            r[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
        }
        return make_uint4(r[0], r[1], r[2], r[3]);
    }
}

template <int PK, bool A_MN, bool B_KN, typename OutT>
__global__ void __launch_bounds__(Cfg<PK>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmO,
                   const GemmDev p) {
    using C = Cfg<PK>;
    constexpr bool PACKED = PK != 0;
    constexpr bool TERN = PK == 2;  // ternary codes: acc - rowsum, one scalar weight scale
    constexpr uint32_t P_BYTES = C::P_BYTES;
    constexpr int S = C::kStages;
    constexpr int CC = 64 / static_cast<int>(sizeof(OutT));  // output columns per staging chunk

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (S + s); };
    auto bready = [&](int s) { return bar0 + 8u * (2 * S + s); };
    auto tfull = [&](int b) { return bar0 + 8u * (3 * S + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (3 * S + 2 + b); };
    const uint32_t drain = bar0 + 8u * (3 * S + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *epi_fail = reinterpret_cast<int *>(smem + C::OFF_MISC + 8);
    float *vcol = reinterpret_cast<float *>(smem + C::OFF_VEC);
    float *vbias = vcol + BN;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (p.M + BM - 1) / BM;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n * p.batch;
    const int nkb = (p.K + BK - 1) / BK;
    // (the 2-bit path keeps whole tiles: its unpack warps expand the full B tile)
    const Items items(num_tiles, num_m, num_m * num_n, static_cast<int>(gridDim.x), !PACKED);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
            mbar_init(bready(s), C::kUnpack);
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
        tma_prefetch_desc(&tmBh);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ producer
        pdl_wait();  // (a programmatic dependent of the act-quant kernel: its codes are ready)
        int stage = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < items.count && ok; item += gridDim.x) {
            int bz, m0, n0;
            bool half;
            items.tile(item, bz, m0, n0, half);
            const uint32_t b_bytes = half ? B_BYTES / 2 : B_BYTES;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, p.status, SITE_GEMM_PRODUCER, p.wait_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t a_dst = sbase + C::OFF_A + stage * A_BYTES;
                if (kb == p.withhold_kb && item == static_cast<int>(blockIdx.x)) {
                    // failure-detection check: this stage's barrier never completes
                } else if constexpr (PACKED) {
                    mbar_arrive_expect_tx(full(stage), A_BYTES + P_BYTES);
                    tma_load_3d(a_dst, &tmA, kb * BK, m0 + p.a_row_off, bz, full(stage));
                    tma_load_3d(sbase + C::OFF_P + stage * P_BYTES, &tmB, kb * slab_words<PK>(), n0, p.b_shared ? 0 : bz,
                                full(stage));
                } else {
                    mbar_arrive_expect_tx(full(stage), A_BYTES + b_bytes);
                    // A: a 128 (K) x 128 (M) box when M-major, 128 (M) x 128 (K) otherwise
                    if constexpr (A_MN)
                        tma_load_3d(a_dst, &tmA, m0, kb * BK, bz, full(stage));
                    else
                        tma_load_3d(a_dst, &tmA, kb * BK, m0, bz, full(stage));
                    const uint32_t b_dst = sbase + C::OFF_B + stage * B_BYTES;
                    if constexpr (B_KN) {
                        tma_load_3d(b_dst, &tmB, n0, kb * BK, p.b_shared ? 0 : bz, full(stage));
                        if (!half)
                            tma_load_3d(b_dst + B_BYTES / 2, &tmB, n0 + 128, kb * BK, p.b_shared ? 0 : bz, full(stage));
                    } else {
                        tma_load_3d(b_dst, half ? &tmBh : &tmB, kb * BK, n0, p.b_shared ? 0 : bz, full(stage));
                    }
                }
                ++issued;
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // let the copies already issued land before the CTA can go away: at
        // once when the MMA consumed them, bounded when another role gave up
        // (a withheld block's barrier runs to the limit)
        for (int64_t i = issued > S ? issued - S : 0; i < issued; ++i)
            mbar_drain(full(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1), p.wait_ns);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_i8(BM, BN, true, !TERN, B_KN, A_MN);
        constexpr uint32_t idesc_half = idesc_i8(BM, BN / 2, true, !TERN, B_KN, A_MN);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int t = 0;
        for (int item = blockIdx.x; item < items.count && ok; item += gridDim.x, ++t) {
            const uint32_t id = item < items.big ? idesc : idesc_half;
            const int abuf = t & 1;
            const uint32_t aphase = static_cast<uint32_t>(t >> 1) & 1u;
            if (!mbar_wait(tempty(abuf), aphase ^ 1u, abort_flag, p.status, SITE_GEMM_MMA, p.wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tbase + static_cast<uint32_t>(abuf * BN);
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(full(stage), phase, abort_flag, p.status, SITE_GEMM_MMA, p.wait_ns)) {
                    ok = false;
                    break;
                }
                if constexpr (PACKED) {
                    if (!mbar_wait(bready(stage), phase, abort_flag, p.status, SITE_GEMM_MMA, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                }
                tc_fence_after();
                const uint32_t a_addr = sbase + C::OFF_A + stage * A_BYTES;
                const uint32_t b_addr = sbase + C::OFF_B + stage * B_BYTES;
#pragma unroll
                for (int ks = 0; ks < BK / UMMA_K; ++ks) {
                    const uint64_t ad = A_MN ? smem_desc_mnmajor_sw128(a_addr + ks * UMMA_K * 128)
                                             : smem_desc_kmajor_sw128(a_addr + ks * UMMA_K);
                    const uint64_t bd = B_KN ? smem_desc_mnmajor_sw128(b_addr + ks * UMMA_K * 128)
                                             : smem_desc_kmajor_sw128(b_addr + ks * UMMA_K);
                    tc_mma_i8(d_tmem, ad, bd, id, (kb | ks) != 0 ? 1u : 0u);
                }
                tc_commit(empty(stage));
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit(tfull(abuf));
        }
        if (!ok) {
            // wait until every MMA issued so far has completed
            tc_commit(drain);
            mbar_drain(drain, 0, p.wait_ns);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ epilogue
        pdl_wait();  // the row scales and sums come from the kernel before
        const int q = warp - 4;  // TMEM lane quarter
        const int r = 32 * q + lane;
        const int et = threadIdx.x - 128;  // 0..127
        uint8_t *stg = smem + C::OFF_STG;
        const float colscale_scalar = TERN ? __ldg(p.colscale) : 0.0f;
        uint32_t chunk_ctr = 0;
        int t = 0;
        for (int item = blockIdx.x; item < items.count; item += gridDim.x, ++t) {
            int bz, m0, n0;
            bool half;
            items.tile(item, bz, m0, n0, half);
            const float *colscale = p.colscale + bz * p.s_col;
            const float *rowscale = p.rowscale + bz * p.s_row;
            const int nc32 = half ? BN / 64 : BN / 32;  // 32-column chunks of this item
            const int abuf = t & 1;
            const uint32_t aphase = static_cast<uint32_t>(t >> 1) & 1u;

            named_bar_sync(1, 128);  // previous tile finished reading vcol / vbias
            for (int i = et; i < BN; i += 128) {
                const int n = n0 + i;
                vcol[i] = (!TERN && n < p.N) ? __ldg(colscale + n) : 0.0f;
                vbias[i] = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + n) : 0.0f;
            }
            named_bar_sync(1, 128);

            // The 128 epilogue threads take the same decision, so none is left
            // alone at a named barrier: each waits (time-bounded only), then
            // they agree through a shared flag.
            // one lane per warp waits (polling by 128 threads would take shared-
            // memory bandwidth from the TMA and MMA), the warp follows it
            bool ok = true;
            if (lane == 0) ok = mbar_wait_timed(tfull(abuf), aphase, p.status, SITE_GEMM_EPILOGUE, p.wait_ns);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok && lane == 0) {
                atomicOr(epi_fail, 1);
                *abort_flag = 1;
            }
            named_bar_sync(1, 128);
            if (*reinterpret_cast<volatile int *>(epi_fail)) break;
            tc_fence_after();
            const int row = m0 + r;
            const float rs = row < p.M ? __ldg(rowscale + row) : 0.0f;
            const int corr = (TERN && row < p.M) ? __ldg(p.rowcorr + bz * p.s_row + row) : 0;

#pragma unroll 1
            for (int c32 = 0; c32 < nc32; ++c32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(abuf * BN + c32 * 32) +
                                       (static_cast<uint32_t>(32 * q) << 16),
                                   v);
                tmem_wait_ld();
                if (c32 == nc32 - 1) {
                    tc_fence_before();
                    mbar_arrive(tempty(abuf));
                }
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float a = static_cast<float>(static_cast<int>(v[j]) - corr);
                    if constexpr (PK == 4) a = __fmul_rn(a, 0.0625f);  // 16 x the code products, exact
                    float o;
                    if constexpr (TERN)
                        o = __fmul_rn(__fmul_rn(a, rs), colscale_scalar);
                    else
                        o = __fmul_rn(__fmul_rn(a, vcol[c32 * 32 + j]), rs);
                    f[j] = __fadd_rn(o, vbias[c32 * 32 + j]);
                }
                uint32_t w[32];
                constexpr int kSub = sizeof(OutT) == 2 ? 1 : 2;  // 64-byte staging rows per 32 columns
                if constexpr (sizeof(OutT) == 2) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[j] = pack2<OutT>(f[2 * j], f[2 * j + 1]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(f[j]);
                }
#pragma unroll
                for (int sc = 0; sc < kSub; ++sc) {
                    const uint32_t sb = chunk_ctr & 1u;
                    if (et == 0) bulk_wait_read<1>();
                    named_bar_sync(1, 128);
                    uint8_t *rowp = stg + sb * STG_BYTES + r * 64;
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
                        tma_store_3d(&tmO, smem_u32(stg + sb * STG_BYTES), n0 + c32 * 32 + sc * CC, m0, bz);
                        bulk_commit();
                    }
                    ++chunk_ctr;
                }
            }
        }
        if (et == 0) bulk_wait_all();
    } else if (PACKED && warp >= 8) {
        // ------------------------------------------------------------ unpack packed codes
        const int ut = threadIdx.x - 256;  // 0 .. C::kUnpack - 1
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < items.count && ok; item += gridDim.x) {
            for (int kb = 0; kb < nkb; ++kb) {
                bool got = true;
                if (lane == 0) got = mbar_wait(full(stage), phase, abort_flag, p.status, SITE_GEMM_UNPACK, p.wait_ns);
                if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
                    ok = false;
                    break;
                }
                const uint32_t *pk = reinterpret_cast<const uint32_t *>(smem + C::OFF_P + stage * P_BYTES);
                uint8_t *bt = smem + C::OFF_B + stage * B_BYTES;
#pragma unroll 4
                for (int i = 0; i < (BN * 8) / C::kUnpack; ++i) {
                    const int idx = ut + C::kUnpack * i;
                    const int n = idx >> 3, c = idx & 7;  // weight row, 16-element chunk of the 128-K slab
                    const uint4 codes = unpack_chunk<PK>(pk + n * slab_words<PK>(), c);
                    *reinterpret_cast<uint4 *>(bt + n * 128 + ((c ^ (n & 7)) << 4)) = codes;
                }
                fence_proxy_async_smem();
                mbar_arrive(bready(stage));
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Pair kernel (W8A8 with K-major weights, large problems): clusters of two
// CTAs on two SMs share one tcgen05.mma.cta_group::2 per 32 K of a 256 x 256
// output tile.  CTA rank r stages its own 128 rows of A (rows m0 + 128 r) and
// its half of B (rows n0 + 128 r), so each SM moves half of the B tile
// through TMA and shared memory; the MMA of the leader (rank 0) reads both
// CTAs' stages and writes each CTA's 128 rows x 256 columns into that CTA's
// tensor memory.
//   warp 0      TMA producer (both CTAs): waits for its own stage to be free,
//               loads A and B with the pair form of the tensor copy, whose
//               completion bytes count on the leader's full barrier (the
//               leader's producer announces the bytes of both CTAs).
//   warp 1      MMA issuer (leader only): 4 x tcgen05.mma.cta_group::2 per
//               stage; the commit arrives on the stage's empty barrier in both
//               CTAs.
//   warp 2      allocates / frees 512 TMEM columns in both CTAs together.
//   warps 4-7   epilogue (both CTAs): as in the single-CTA kernel, on the
//               CTA's own rows; all 256 epilogue threads of the pair release
//               an accumulator on the leader's barrier.
// A short last wave runs as 256 x 128 halves (each CTA 64 rows of B).
// W2A8 (PACKED): each CTA loads A and its half of the packed 2-bit codes with
// plain tensor copies on its own full barrier; its unpack warps (8-15, two
// groups of four taking the k-blocks in turn) expand only that half into the B
// stage and arrive on the leader's bready barrier, which is what the MMA waits
// for (both CTAs' stages complete).
// Every wait is bounded; both CTAs always reach the closing cluster barrier.
// ---------------------------------------------------------------------------
constexpr uint32_t PA_BYTES = 128 * BK;              // own 128 rows of A
constexpr uint32_t PB_BYTES = 128 * BK;              // own half of a 256-wide B tile
template <int PK>
struct PairCfg {
    static constexpr bool PACKED = PK != 0;
    static constexpr int kUnpackGroups = 2;  // unpack warp groups, taking k-blocks in turn
    static constexpr uint32_t PP_BYTES = p_bytes<PK>(128);  // its packed form
    static constexpr int kStages = PACKED ? 5 : 6;
    static constexpr int kUnpack = 256;  // unpack threads (packed weights)
    static constexpr int kThreads = PACKED ? 256 + kUnpack : 256;
    static constexpr uint32_t OFF_A = 0;
    static constexpr uint32_t OFF_B = OFF_A + kStages * PA_BYTES;
    static constexpr uint32_t OFF_P = OFF_B + kStages * PB_BYTES;
    static constexpr uint32_t OFF_STG = OFF_P + (PACKED ? kStages * PP_BYTES : 0);
    static constexpr uint32_t OFF_VEC = OFF_STG + 2 * STG_BYTES;  // colscale[BN], bias[BN]
    static constexpr uint32_t OFF_BAR = OFF_VEC + 2 * BN * 4;
    // full[S], empty[S], bready[S], tfull[2], tempty[2], drain
    static constexpr uint32_t NBAR = 3 * kStages + 5;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, epilogue failure
    static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;
};

static_assert(Cfg<0>::SMEM <= 232448 && Cfg<2>::SMEM <= 232448 && Cfg<4>::SMEM <= 232448,
              "single-CTA stages exceed the 227 KB of shared memory per CTA");
static_assert(PairCfg<0>::SMEM <= 232448 && PairCfg<2>::SMEM <= 232448 && PairCfg<4>::SMEM <= 232448,
              "pair stages exceed the 227 KB of shared memory per CTA");

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the object at CTA-local address `addr` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// Arrival (default release semantics) on the barrier at cluster address `caddr`.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
// Tensor copy into this CTA's shared memory whose completion counts on the
// barrier at cluster address `bar` (the leader's).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                                 int32_t z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives (once) on the barrier at CTA-local address `bar` in both CTAs of the
// pair when the MMAs issued so far have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

template <int PK, typename OutT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<PK>::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmO,
                     const GemmDev p) {
    using C = PairCfg<PK>;
    constexpr bool PACKED = PK != 0;
    constexpr bool TERN = PK == 2;
    constexpr uint32_t PP_BYTES = C::PP_BYTES;
    constexpr int S = C::kStages;
    constexpr uint32_t OFF_A = C::OFF_A, OFF_B = C::OFF_B, OFF_P = C::OFF_P, OFF_STG = C::OFF_STG;
    constexpr uint32_t OFF_VEC = C::OFF_VEC, OFF_BAR = C::OFF_BAR, OFF_MISC = C::OFF_MISC;
    constexpr int CC = 64 / static_cast<int>(sizeof(OutT));

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (S + s); };
    auto bready = [&](int s) { return bar0 + 8u * (2 * S + s); };
    auto tfull = [&](int b) { return bar0 + 8u * (3 * S + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (3 * S + 2 + b); };
    const uint32_t drain = bar0 + 8u * (3 * S + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    int *epi_fail = reinterpret_cast<int *>(smem + OFF_MISC + 8);
    float *vcol = reinterpret_cast<float *>(smem + OFF_VEC);
    float *vbias = vcol + BN;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int num_m = (p.M + 2 * BM - 1) / (2 * BM);  // 256-row tiles
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n * p.batch;
    const int nkb = (p.K + BK - 1) / BK;
    const int cl = static_cast<int>(blockIdx.x >> 1), ncl = static_cast<int>(gridDim.x >> 1);
    // items as in the single-CTA schedule, over pairs and 256 x 256 tiles
    const int full_w = (num_tiles / ncl) * ncl, left = num_tiles - full_w;
    const bool split = left > 0 && 2 * left <= ncl;
    const int big = split ? full_w : num_tiles, count = split ? full_w + 2 * left : num_tiles;
    auto tile_of = [&](int item, int &b, int &m0, int &n0, bool &half) {
        const int t = item < big ? item : big + ((item - big) >> 1);
        b = t / (num_m * num_n);
        const int r = t - b * num_m * num_n;
        m0 = (r % num_m) * 2 * BM;
        n0 = (r / num_m) * BN + (item < big ? 0 : ((item - big) & 1) * (BN / 2));
        half = item >= big;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
            mbar_init(bready(s), 2 * (C::kUnpack / 32) / C::kUnpackGroups);  // one unpack group per CTA (leader's)
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), 256);  // the epilogue threads of both CTAs (leader's barrier)
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *epi_fail = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmBh);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 2) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
        tc_fence_before();
    }
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers initialized before any remote arrival
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        pdl_wait();  // (a programmatic dependent of the act-quant kernel: its codes are ready)
        int stage = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        bool ok = true;
        for (int item = cl; item < count && ok; item += ncl) {
            int bz, m0, n0;
            bool half;
            tile_of(item, bz, m0, n0, half);
            const uint32_t b_bytes = half ? PB_BYTES / 2 : PB_BYTES;
            const int nb0 = n0 + (half ? BN / 4 : BN / 2) * static_cast<int>(rank);  // this CTA's B rows
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait_spin(empty(stage), phase ^ 1u, abort_flag, p.status, SITE_GEMM_PRODUCER, p.wait_ns)) {
                    ok = false;
                    break;
                }
                if constexpr (PACKED) {  // own barrier: this CTA's unpack warps wait on it
                    const uint32_t p_bytes = half ? PP_BYTES / 2 : PP_BYTES;
                    mbar_arrive_expect_tx(full(stage), PA_BYTES + p_bytes);
                    tma_load_3d(sbase + OFF_A + stage * PA_BYTES, &tmA, kb * BK,
                                m0 + BM * static_cast<int>(rank) + p.a_row_off, bz, full(stage));
                    tma_load_3d(sbase + OFF_P + stage * PP_BYTES, half ? &tmBh : &tmB, kb * slab_words<PK>(), nb0,
                                p.b_shared ? 0 : bz,
                                full(stage));
                } else {  // the leader's barrier counts both CTAs' copies
                    if (leader) mbar_arrive_expect_tx(full(stage), 2u * (PA_BYTES + b_bytes));
                    const uint32_t lbar = cluster_addr(full(stage), 0);
                    tma_load_3d_pair(sbase + OFF_A + stage * PA_BYTES, &tmA, kb * BK, m0 + BM * static_cast<int>(rank),
                                     bz, lbar);
                    tma_load_3d_pair(sbase + OFF_B + stage * PB_BYTES, half ? &tmBh : &tmB, kb * BK, nb0,
                                     p.b_shared ? 0 : bz, lbar);
                }
                ++issued;
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && (leader || PACKED)) {
            // let the copies this full barrier counts land (both CTAs' on the leader without 2-bit codes)
            for (int64_t i = issued > S ? issued - S : 0; i < issued; ++i) {
                mbar_drain(full(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1), p.wait_ns);
            }
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------------------------ MMA issuer (leader)
        constexpr uint32_t idesc = idesc_i8(2 * BM, BN, true, !TERN, false);
        constexpr uint32_t idesc_half = idesc_i8(2 * BM, BN / 2, true, !TERN, false);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int t = 0;
        for (int item = cl; item < count && ok; item += ncl, ++t) {
            const uint32_t id = item < big ? idesc : idesc_half;
            const int abuf = t & 1;
            const uint32_t aphase = static_cast<uint32_t>(t >> 1) & 1u;
            if (!mbar_wait(tempty(abuf), aphase ^ 1u, abort_flag, p.status, SITE_GEMM_MMA, p.wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tbase + static_cast<uint32_t>(abuf * BN);
            for (int kb = 0; kb < nkb; ++kb) {
                // (polled: the last arrival is often the peer CTA's)
                if (!mbar_wait_spin(PACKED ? bready(stage) : full(stage), phase, abort_flag, p.status, SITE_GEMM_MMA, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = sbase + OFF_A + stage * PA_BYTES;
                const uint32_t b_addr = sbase + OFF_B + stage * PB_BYTES;
#pragma unroll
                for (int ks = 0; ks < BK / UMMA_K; ++ks)
                    tc_mma_i8_pair(d_tmem, smem_desc_kmajor_sw128(a_addr + ks * UMMA_K),
                                   smem_desc_kmajor_sw128(b_addr + ks * UMMA_K), id, (kb | ks) != 0 ? 1u : 0u);
                tc_commit_pair(empty(stage));
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit_pair(tfull(abuf));
        }
        if (!ok) {
            tc_commit_pair(drain);
            mbar_drain(drain, 0, p.wait_ns);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        pdl_wait();  // the row scales and sums come from the kernel before
        const int q = warp - 4;
        const int r = 32 * q + lane;
        const int et = threadIdx.x - 128;
        uint8_t *stg = smem + OFF_STG;
        const float colscale_scalar = TERN ? __ldg(p.colscale) : 0.0f;
        uint32_t chunk_ctr = 0;
        int t = 0;
        for (int item = cl; item < count; item += ncl, ++t) {
            int bz, m0, n0;
            bool half;
            tile_of(item, bz, m0, n0, half);
            const float *colscale = p.colscale + bz * p.s_col;
            const float *rowscale = p.rowscale + bz * p.s_row;
            const int mr = m0 + BM * static_cast<int>(rank);  // this CTA's first row
            const int nc32 = half ? BN / 64 : BN / 32;
            const int abuf = t & 1;
            const uint32_t aphase = static_cast<uint32_t>(t >> 1) & 1u;

            named_bar_sync(1, 128);
            for (int i = et; i < BN; i += 128) {
                const int n = n0 + i;
                vcol[i] = (!TERN && n < p.N) ? __ldg(colscale + n) : 0.0f;
                vbias[i] = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + n) : 0.0f;
            }
            named_bar_sync(1, 128);

            bool ok = true;
            if (lane == 0) ok = mbar_wait_timed(tfull(abuf), aphase, p.status, SITE_GEMM_EPILOGUE, p.wait_ns);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok && lane == 0) {
                atomicOr(epi_fail, 1);
                *abort_flag = 1;
            }
            named_bar_sync(1, 128);
            if (*reinterpret_cast<volatile int *>(epi_fail)) break;
            tc_fence_after();
            const int row = mr + r;
            const float rs = row < p.M ? __ldg(rowscale + row) : 0.0f;
            const int corr = (TERN && row < p.M) ? __ldg(p.rowcorr + bz * p.s_row + row) : 0;

#pragma unroll 1
            for (int c32 = 0; c32 < nc32; ++c32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(abuf * BN + c32 * 32) +
                                       (static_cast<uint32_t>(32 * q) << 16),
                                   v);
                tmem_wait_ld();
                if (c32 == nc32 - 1) {
                    tc_fence_before();
                    mbar_arrive_remote(cluster_addr(tempty(abuf), 0));
                }
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float a = static_cast<float>(static_cast<int>(v[j]) - corr);
                    if constexpr (PK == 4) a = __fmul_rn(a, 0.0625f);  // 16 x the code products, exact
                    const float o = TERN ? __fmul_rn(__fmul_rn(a, rs), colscale_scalar)
                                           : __fmul_rn(__fmul_rn(a, vcol[c32 * 32 + j]), rs);
                    f[j] = __fadd_rn(o, vbias[c32 * 32 + j]);
                }
                uint32_t w[32];
                constexpr int kSub = sizeof(OutT) == 2 ? 1 : 2;
                if constexpr (sizeof(OutT) == 2) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[j] = pack2<OutT>(f[2 * j], f[2 * j + 1]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(f[j]);
                }
#pragma unroll
                for (int sc = 0; sc < kSub; ++sc) {
                    const uint32_t sb = chunk_ctr & 1u;
                    if (et == 0) bulk_wait_read<1>();
                    named_bar_sync(1, 128);
                    uint8_t *rowp = stg + sb * STG_BYTES + r * 64;
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
                        tma_store_3d(&tmO, smem_u32(stg + sb * STG_BYTES), n0 + c32 * 32 + sc * CC, mr, bz);
                        bulk_commit();
                    }
                    ++chunk_ctr;
                }
            }
        }
        if (et == 0) bulk_wait_all();
    } else if (PACKED && warp >= 8) {
        // ------------------------------------------------------------ unpack own half of B (both CTAs)
        // The unpack warps form kUnpackGroups groups that take the k-blocks in
        // turn, each expanding a whole stage: the wait -> expand -> fence ->
        // arrive chains of consecutive stages overlap, instead of all eight warps
        // walking every stage's chain together.  Every warp follows the same
        // stage / phase sequence, so the barrier parities stay in step.
        constexpr int kGroup = C::kUnpack / C::kUnpackGroups;  // threads per group
        const int ut = threadIdx.x - 256;
        const int grp = ut / kGroup, gt = ut - grp * kGroup;
        int stage = 0, step = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int item = cl; item < count && ok; item += ncl) {
            const int chunks = (item < big ? 128 : 64) * 8;  // 16-weight chunks of this CTA's rows
            for (int kb = 0; kb < nkb; ++kb, ++step) {
                if (step % C::kUnpackGroups != grp) {  // another group's k-block
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    continue;
                }
                bool got = true;
                if (lane == 0) got = mbar_wait_spin(full(stage), phase, abort_flag, p.status, SITE_GEMM_UNPACK, p.wait_ns);
                if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
                    ok = false;
                    break;
                }
                const uint32_t *pk = reinterpret_cast<const uint32_t *>(smem + OFF_P + stage * PP_BYTES);
                uint8_t *bt = smem + OFF_B + stage * PB_BYTES;
#pragma unroll 4
                for (int idx = gt; idx < chunks; idx += kGroup) {
                    const int n = idx >> 3, c = idx & 7;  // weight row, 16-element chunk of the 128-K slab
                    const uint4 codes = unpack_chunk<PK>(pk + n * slab_words<PK>(), c);
                    *reinterpret_cast<uint4 *>(bt + n * 128 + ((c ^ (n & 7)) << 4)) = codes;
                }
                // every lane orders its stores before the tensor core's reads, then the
                // warp's arrival on the leader releases them
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(cluster_addr(bready(stage), 0));
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    __syncthreads();
    cluster_sync_all();  // no remote arrival or MMA of the pair is left in flight
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 3-D tiled tensor map: {inner, outer, batch} elements with row and batch
// strides in bytes (both multiples of 16), box {box_inner, box_outer, 1}.
// batches of the B tensor maps: one when all batches share B (zero B stride)
uint64_t b_batches(const GemmArgs &g) { return g.batch > 1 && g.sb == 0 ? 1 : static_cast<uint64_t>(g.batch); }

bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw, uint64_t batch = 1,
              uint64_t batch_bytes = 0) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    if (batch <= 1 || batch_bytes == 0) batch_bytes = (row_bytes * outer + 15) / 16 * 16;
    const cuuint64_t dims[3] = {inner, outer, batch < 1 ? 1 : batch};
    const cuuint64_t strides[2] = {row_bytes, batch_bytes};
    const cuuint32_t box[3] = {box_inner, box_outer, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

GemmDev dev_args(const GemmArgs &g, const DevInfo &dev) {
    GemmDev p;
    p.colscale = g.colscale;
    p.rowscale = g.rowscale;
    p.rowcorr = g.rowcorr;
    p.bias = g.bias;
    p.M = static_cast<int>(g.M);
    p.N = static_cast<int>(g.N);
    p.K = static_cast<int>(g.K);
    p.batch = static_cast<int>(g.batch);
    p.s_col = g.s_col;
    p.s_row = g.s_row;
    p.a_row_off = static_cast<int>(g.a_row_off);
    p.b_shared = g.batch > 1 && g.sb == 0 ? 1 : 0;
    p.status = dev.status;
    p.wait_ns = g.wait_ns;
    p.withhold_kb = g.withhold_kb;
    return p;
}

template <int PK, bool A_MN, bool B_KN, typename OutT>
bq_status launch_t(const GemmArgs &g, const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mBh,
                   const CUtensorMap &mO,
                   cudaStream_t s, const DevInfo &dev) {
    using C = Cfg<PK>;
    auto kern = gemm_tc_kernel<PK, A_MN, B_KN, OutT>;
    static SmemOptIn opt_in;  // once per context (also keeps later calls capture-safe)
    if (smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), static_cast<size_t>(C::SMEM)) != cudaSuccess)
        return BQ_ERR_CUDA;
    const int64_t tiles = ((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN) * g.batch;
    const int grid = static_cast<int>(tiles < dev.num_sms ? tiles : dev.num_sms);
    if (g.pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = C::SMEM;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, mA, mB, mBh, mO, dev_args(g, dev)) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
    }
    kern<<<grid, C::kThreads, C::SMEM, s>>>(mA, mB, mBh, mO, dev_args(g, dev));
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <int PK, typename OutT>
bq_status launch_pair(const GemmArgs &g, const CUtensorMap &mA, const CUtensorMap &mB128, const CUtensorMap &mB64,
                      const CUtensorMap &mO, cudaStream_t s, const DevInfo &dev) {
    using C = PairCfg<PK>;
    auto kern = gemm_pair_kernel<PK, OutT>;
    static SmemOptIn opt_in;  // once per context (also keeps later calls capture-safe)
    if (smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(kern), static_cast<size_t>(C::SMEM)) != cudaSuccess)
        return BQ_ERR_CUDA;
    const int64_t tiles = ((g.M + 2 * BM - 1) / (2 * BM)) * ((g.N + BN - 1) / BN) * g.batch;
    const int64_t pairs = std::min<int64_t>(tiles, dev.num_sms / 2);
    GemmDev p = dev_args(g, dev);
    p.withhold_kb = -1;  // (the failure-detection check runs on a single CTA)
    if (g.pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = C::SMEM;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, mA, mB128, mB64, mO, p) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
    }
    kern<<<static_cast<unsigned>(2 * pairs), C::kThreads, C::SMEM, s>>>(mA, mB128, mB64, mO, p);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

// The pair kernel takes products with K-major A and K-major (or 2-bit packed)
// weights that fill at least one wave of CTA pairs with 256 x 256 tiles.
bool use_pair(const GemmArgs &g, const DevInfo &dev) {
    return !g.a_mn && gemm_uses_pair(g.b_pack != 0, g.b_layout, g.M, g.N, dev, g.batch);
}

template <int PK, typename OutT>
bq_status dispatch_packed(const GemmArgs &g, const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mO,
                          cudaStream_t s, const DevInfo &dev) {
    if (use_pair(g, dev)) {
        // per CTA of a pair: its half of the packed tile (128 rows), 64 rows for half tiles
        CUtensorMap mP128, mP64;
        const uint64_t words = static_cast<uint64_t>(g.K) * PK / 32;
        if (!make_map(&mP128, CU_TENSOR_MAP_DATA_TYPE_UINT32, g.b, words, g.N, g.ldb * 4, slab_words<PK>(), BN / 2,
                      CU_TENSOR_MAP_SWIZZLE_NONE, b_batches(g), g.sb * 4) ||
            !make_map(&mP64, CU_TENSOR_MAP_DATA_TYPE_UINT32, g.b, words, g.N, g.ldb * 4, slab_words<PK>(), BN / 4,
                      CU_TENSOR_MAP_SWIZZLE_NONE, b_batches(g), g.sb * 4))
            return BQ_ERR_CUDA;
        return launch_pair<PK, OutT>(g, mA, mP128, mP64, mO, s, dev);
    }
    return launch_t<PK, false, false, OutT>(g, mA, mB, mB, mO, s, dev);
}

template <typename OutT>
bq_status dispatch(const GemmArgs &g, const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mBh,
                   const CUtensorMap &mO,
                   cudaStream_t s, const DevInfo &dev) {
    if (g.b_pack == 2) return dispatch_packed<2, OutT>(g, mA, mB, mO, s, dev);
    if (g.b_pack == 4) return dispatch_packed<4, OutT>(g, mA, mB, mO, s, dev);
    if (use_pair(g, dev)) {
        // per CTA of a pair: 128-row boxes of B (half of a 256-wide tile), 64-row boxes for half tiles
        CUtensorMap mBq;
        if (!make_map(&mBq, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b, g.K, g.N, g.ldb, BK, BN / 4,
                      CU_TENSOR_MAP_SWIZZLE_128B, b_batches(g), g.sb))
            return BQ_ERR_CUDA;
        return launch_pair<0, OutT>(g, mA, mBh, mBq, mO, s, dev);
    }
    if (g.a_mn) {
        if (g.b_layout == BQ_W_KN) return launch_t<0, true, true, OutT>(g, mA, mB, mBh, mO, s, dev);
        return launch_t<0, true, false, OutT>(g, mA, mB, mBh, mO, s, dev);
    }
    if (g.b_layout == BQ_W_KN) return launch_t<0, false, true, OutT>(g, mA, mB, mBh, mO, s, dev);
    return launch_t<0, false, false, OutT>(g, mA, mB, mBh, mO, s, dev);
}

}  // namespace

bool gemm_uses_pair(bool packed, bq_wlayout b_layout, int64_t M, int64_t N, const DevInfo &dev, int64_t batch) {
    if ((!packed && b_layout == BQ_W_KN) || dev.num_sms < 2) return false;
    const int64_t tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + BN - 1) / BN) * batch;
    return tiles >= dev.num_sms / 2;
}

bq_status launch_gemm_tc(const GemmArgs &g, cudaStream_t s, const DevInfo &dev) {
    const uint64_t nb = static_cast<uint64_t>(g.batch);
    CUtensorMap mA, mB, mBh, mO;
    const bool okA = g.a_mn ? make_map(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, g.M, g.K, g.lda, BM, BK,
                                       CU_TENSOR_MAP_SWIZZLE_128B, nb, g.sa)
                            : make_map(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, g.K, g.a_rows > 0 ? g.a_rows : g.M,
                                       g.lda, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B, nb, g.sa);
    if (!okA) return BQ_ERR_CUDA;
    bool okB;
    if (g.b_pack != 0)
        okB = make_map(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT32, g.b, static_cast<uint64_t>(g.K) * g.b_pack / 32, g.N,
                       g.ldb * 4, BK * g.b_pack / 32, BN, CU_TENSOR_MAP_SWIZZLE_NONE, b_batches(g), g.sb * 4);
    else if (g.b_layout == BQ_W_KN)
        okB = make_map(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b, g.N, g.K, g.ldb, 128, BK, CU_TENSOR_MAP_SWIZZLE_128B,
                       b_batches(g), g.sb);
    else
        okB = make_map(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b, g.K, g.N, g.ldb, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B,
                       b_batches(g), g.sb);
    if (!okB) return BQ_ERR_CUDA;
    // K-major weights: a 128-row box too, for the half tiles of a last partial wave
    mBh = mB;
    if (g.b_pack == 0 && g.b_layout != BQ_W_KN &&
        !make_map(&mBh, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b, g.K, g.N, g.ldb, BK, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B,
                  b_batches(g), g.sb))
        return BQ_ERR_CUDA;
    CUtensorMapDataType odt = g.out_dtype == BQ_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                              : g.out_dtype == BQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int esz = g.out_dtype == BQ_F32 ? 4 : 2;
    if (!make_map(&mO, odt, g.out, g.N, g.M, g.ldo * esz, 64 / esz, BM, CU_TENSOR_MAP_SWIZZLE_64B, nb, g.so * esz))
        return BQ_ERR_CUDA;
    switch (g.out_dtype) {
        case BQ_F32:
            return dispatch<float>(g, mA, mB, mBh, mO, s, dev);
        case BQ_F16:
            return dispatch<__half>(g, mA, mB, mBh, mO, s, dev);
        default:
            return dispatch<__nv_bfloat16>(g, mA, mB, mBh, mO, s, dev);
    }
}

}  // namespace bq
