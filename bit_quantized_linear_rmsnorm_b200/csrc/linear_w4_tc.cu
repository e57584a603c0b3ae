// Multi-token grouped INT4 linear on the sm_100a tensor cores
// ("vyre_libs/nn/linear/inner/linear_4bit/mod.rs" (docs.rs vyre-libs), module
// doc: grouped affine INT4 linear, one scale and zero-point per group):
//
//   out[m,n] = bias[n] + sum_k x[m,k] * s[n,g] * (q[n,k] - z[n,g]),  g = k / gs
//
// Three launches (programmatic dependent launch between them):
//  1. w4_planes_kernel: per token m and 1024-wide K slice s, X = rne(x / sx)
//     with sx[m,s] = max|x| / 8355711 over the slice, written as signed
//     base-256 digits P0, P1, P2
//     (X = 65536 P0 + 256 P1 + P2, each digit in [-128, 127]).  Plane p of
//     token m is row 32 p + m of a [96][K] int8 matrix (rows of absent tokens
//     are zero).  The representation error is at most one unit of sx
//     (x / sx taken as x * (1 / sx)), i.e. about max|x| * 1.2e-7.
//  2. w4_tc_kernel: a CTA owns the rows of one row tile and one 1024-wide K
//     slice.  Per 128-wide K block (one group when gs % 128 == 0) it computes
//       D[n, 32 p + m] = sum_k (q[n,k] - z[n,g]) * P_p[m,k]
//     with tcgen05.mma kind::i8 (M = 128 weight rows, N = 96, K = 32 per
//     instruction, s8 x s8, 32-bit accumulators in TMEM): eight expander warps
//     turn the packed codes minus the zero-point into s8 in a 128-byte-swizzled
//     A stage (no dequantized weight reaches global memory); the plane slice
//     (96 rows x 1024 B) stays resident in shared memory as B.  Per group the
//     eight epilogue warps (two per TMEM lane quarter, 16 tokens each) read the
//     three planes of their tokens, T = 65536 D0 + (256 D1 + D2) (the bracket in
//     int32, T in fp32), acc[m] += s[n,g] * T[m], and write one partial sum per
//     (K slice, token, row).  Four TMEM accumulators let the MMAs run ahead.
//  3. w4_reduce_kernel: out = bias + sum over the K slices, in slice order, of
//     sx[m,s] * partial, so the result does not depend on scheduling.
// Every mbarrier wait is bounded; on expiry the kernel records BQ_ERR_TIMEOUT
// in the status word, drains its own async work and exits.
#include <cuda_fp16.h>

#include <algorithm>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

constexpr int kTcTok = 32;                 // token slots (columns per plane)
constexpr int kTcCols = 3 * kTcTok;        // MMA N
constexpr int kTcRows = 128;               // MMA M: weight rows per tile
constexpr int kTcKB = 128;                 // K per stage (one 128-byte swizzle row)
constexpr int kTcKS = 1024;                // K per CTA slice
constexpr int kTcBlocks = kTcKS / kTcKB;   // K blocks per slice
constexpr int kTcStages = 4;               // A stages
constexpr int kTcMaxTiles = 4;             // row tiles of 128 per CTA
constexpr int kTcXMax = 8355711;           // 127 * (65536 + 256 + 1)
constexpr int kTcThreads = 576;            // warps 0-7 expand, 8-15 epilogue, 16 MMA, 17 TMEM
constexpr int kTcBufs = 4;                 // TMEM accumulators (96 columns each)
constexpr int kTcRing = 6;                 // packed weight steps in flight per expander thread
constexpr uint32_t kTcABytes = kTcRows * kTcKB;       // 16 KB
constexpr uint32_t kTcBBlock = kTcCols * kTcKB;       // 12 KB
constexpr uint32_t kTcBBytes = kTcBBlock * kTcBlocks; // 96 KB
constexpr uint32_t kTcTmemCols = 512;                 // four 96-column accumulators at 0, 128, 256, 384

struct TcLayout {
    static constexpr uint32_t OFF_B = 0;
    static constexpr uint32_t OFF_A = OFF_B + kTcBBytes;
    // packed weights: [kTcRing][2 rows][256 expander threads][16 B] (each thread its own pieces)
    static constexpr uint32_t OFF_P = OFF_A + kTcStages * kTcABytes;
    static constexpr uint32_t P_BYTES = kTcRing * 2 * 256 * 16;
    static constexpr uint32_t OFF_Z = OFF_P + P_BYTES;  // zero-point word of each row for the slice
    static constexpr uint32_t OFF_BAR = OFF_Z + kTcMaxTiles * kTcRows * 4;
    // a_full[S], a_empty[S], t_full[B], t_empty[B], drain
    static constexpr uint32_t NBAR = 2 * kTcStages + 2 * kTcBufs + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
    static constexpr uint32_t OFF_GT = OFF_MISC + 16;         // per K block: group index, zero-point shift
    // the scales of every step, [tile][K block][row] fp16, loaded once after the dependency wait
    static constexpr uint32_t OFF_SC = OFF_GT + 8 * kTcBlocks;
    static constexpr uint32_t SC_BYTES = kTcMaxTiles * kTcBlocks * kTcRows * 2;
    static constexpr uint32_t SMEM = OFF_SC + SC_BYTES + 1024;  // + alignment slack
};

__device__ __forceinline__ int tc_digit(int v) { return ((v + 128) & 255) - 128; }

// float(v) for |v| < 2^22 on the FMA pipe (v added to the mantissa of
// 1.5 * 2^23, then the offset subtracted; both steps exact).  A 128-deep
// inner product of codes minus zero-point (|.| <= 15) and plane digits
// (|.| <= 128) stays below 2^18.
__device__ __forceinline__ float tc_exact_float(int v) { return __int_as_float(0x4B400000 + v) - 12582912.0f; }

// ---------------------------------------------------------------------------
// 1. activation planes, one CTA per (token slot, K slice) (256 threads x 4 elements)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) w4_planes_kernel(const float *__restrict__ x, int M, int K,
                                                       int8_t *__restrict__ planes, float *__restrict__ sx_out) {
    __shared__ float red[8];
    const int S = K / kTcKS;
    const int m = blockIdx.x / S, s = blockIdx.x - m * S, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    pdl_launch_dependents();
    pdl_wait();
    const int k = s * kTcKS + 4 * t;
    int8_t *p0 = planes + static_cast<int64_t>(m) * K + k;
    int8_t *p1 = planes + static_cast<int64_t>(kTcTok + m) * K + k;
    int8_t *p2 = planes + static_cast<int64_t>(2 * kTcTok + m) * K + k;
    if (m >= M) {  // absent token: zero planes
        *reinterpret_cast<uint32_t *>(p0) = 0u;
        *reinterpret_cast<uint32_t *>(p1) = 0u;
        *reinterpret_cast<uint32_t *>(p2) = 0u;
        if (t == 0) sx_out[m * S + s] = 0.0f;
        return;
    }
    const float4 v = __ldg(reinterpret_cast<const float4 *>(x + static_cast<int64_t>(m) * K + k));
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float sx = __fdiv_rn(amax, static_cast<float>(kTcXMax));
    const float inv = amax > 0.f ? __fdiv_rn(1.0f, sx) : 0.f;
    if (t == 0) sx_out[m * S + s] = sx;
    const float e[4] = {v.x, v.y, v.z, v.w};
    uint32_t w0 = 0u, w1 = 0u, w2 = 0u;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int X = __float2int_rn(__fmul_rn(e[u], inv));
        X = max(-kTcXMax, min(kTcXMax, X));
        const int d2 = tc_digit(X), X1 = (X - d2) >> 8;
        const int d1 = tc_digit(X1), d0 = (X1 - d1) >> 8;
        w0 |= (static_cast<uint32_t>(d0) & 255u) << (8 * u);
        w1 |= (static_cast<uint32_t>(d1) & 255u) << (8 * u);
        w2 |= (static_cast<uint32_t>(d2) & 255u) << (8 * u);
    }
    *reinterpret_cast<uint32_t *>(p0) = w0;
    *reinterpret_cast<uint32_t *>(p1) = w1;
    *reinterpret_cast<uint32_t *>(p2) = w2;
}

// ---------------------------------------------------------------------------
// 3. out[m][n] = bias[n] + sum_s sx[m,s] * part[s][m][n]  (slices in order)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) w4_reduce_kernel(const float *__restrict__ part, const float *__restrict__ sx,
                                                       const float *__restrict__ bias, int M, int N, int S,
                                                       float *__restrict__ out) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t total = static_cast<int64_t>(N) * M;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int m = static_cast<int>(i / N), n = static_cast<int>(i - static_cast<int64_t>(m) * N);
        float acc = 0.f;
        for (int s = 0; s < S; ++s)
            acc = fmaf(sx[m * S + s], part[(static_cast<int64_t>(s) * kTcTok + m) * N + n], acc);
        out[static_cast<int64_t>(m) * N + n] = (bias ? __ldg(bias + n) : 0.0f) + acc;
    }
}

// ---------------------------------------------------------------------------
// 2. tensor-core kernel
// ---------------------------------------------------------------------------
struct TcArgs {
    const uint32_t *qweight;
    const uint16_t *scales;
    const uint32_t *qzeros;
    const int8_t *planes;  // [96][K]
    float *part;           // [S][32][N]
    int N, K, gs, S, R;    // K slices, row tiles
    uint32_t *status;
};

__global__ void __launch_bounds__(kTcThreads, 1) w4_tc_kernel(const TcArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + TcLayout::OFF_BAR;
    auto a_full = [&](int s) { return bar0 + 8u * s; };
    auto a_empty = [&](int s) { return bar0 + 8u * (kTcStages + s); };
    auto t_full = [&](int b) { return bar0 + 8u * (2 * kTcStages + b); };
    auto t_empty = [&](int b) { return bar0 + 8u * (2 * kTcStages + kTcBufs + b); };
    const uint32_t drain = bar0 + 8u * (2 * kTcStages + 2 * kTcBufs);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + TcLayout::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + TcLayout::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rt = blockIdx.x / p.S, ks = blockIdx.x - rt * p.S;  // row tile, K slice
    const int n0 = static_cast<int>((static_cast<int64_t>(rt) * p.N) / p.R);
    const int rows = static_cast<int>((static_cast<int64_t>(rt + 1) * p.N) / p.R) - n0;
    const int ntiles = (rows + kTcRows - 1) / kTcRows;  // <= kTcMaxTiles (host check)
    const int nsteps = ntiles * kTcBlocks;
    const int K = p.K, G = K / p.gs, zrow = (G + 7) / 8;
    const int kbase = ks * kTcKS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(a_full(s), 8);  // one arrival per expander warp
            mbar_init(a_empty(s), 1);
        }
        for (int b = 0; b < kTcBufs; ++b) {
            mbar_init(t_full(b), 1);
            mbar_init(t_empty(b), 8);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 17) {
        tmem_alloc(smem_u32(tmem_slot), kTcTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    pdl_launch_dependents();
    pdl_wait();  // the planes come from the previous launch

    // resident B: the plane slice (96 rows x 1024 B) as 8 swizzled K blocks
    for (int i = threadIdx.x; i < kTcCols * (kTcKS / 16); i += kTcThreads) {
        const int r = i >> 6, c = i & 63, g = c >> 3, cc = c & 7;
        cp_async_16(sbase + TcLayout::OFF_B + g * kTcBBlock + r * 128 + ((cc ^ (r & 7)) << 4),
                    p.planes + static_cast<int64_t>(r) * K + kbase + 16 * c, 16u);
    }
    {  // the zero-point word (8 nibbles) covering this slice's groups, per row
        uint32_t *zs = reinterpret_cast<uint32_t *>(smem + TcLayout::OFF_Z);
        const int zw = (kbase / p.gs) / 8;
        for (int r = threadIdx.x; r < rows; r += kTcThreads) zs[r] = __ldg(p.qzeros + static_cast<int64_t>(n0 + r) * zrow + zw);
        int *gt = reinterpret_cast<int *>(smem + TcLayout::OFF_GT);  // (no division in the step loops)
        if (threadIdx.x < kTcBlocks) {
            const int grp = (kbase + kTcKB * static_cast<int>(threadIdx.x)) / p.gs;
            gt[threadIdx.x] = grp;
            gt[kTcBlocks + threadIdx.x] = 4 * (grp % 8);
        }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp < 8) {
        // ------------------------------------------------------------ expanders
        // thread e: 16-byte piece pc = e % 4 (32 codes) of the block's 64 packed
        // bytes, for rows rr = e / 4 and rr + 64 of the tile; four lanes cover a
        // row's block, so every copy instruction reads whole 64-byte segments.
        // The pieces are copied kTcRing steps ahead (cp.async into this
        // thread's own ring slots, read back by the same thread).
        const int e = threadIdx.x, pc = e & 3, rr = e >> 2;
        const uint32_t *zs = reinterpret_cast<const uint32_t *>(smem + TcLayout::OFF_Z);
        const int *zshift = reinterpret_cast<const int *>(smem + TcLayout::OFF_GT) + kTcBlocks;
        auto slot_addr = [&](int j, int half) {
            return sbase + TcLayout::OFF_P + static_cast<uint32_t>((((j % kTcRing) * 2 + half) * 256 + e) * 16);
        };
        auto issue = [&](int j) {
            const int t = j / kTcBlocks, g = j - t * kTcBlocks;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = t * kTcRows + rr + 64 * half;
                const bool in = j < nsteps && r < rows;
                const uint32_t *src = p.qweight + static_cast<int64_t>(n0 + (in ? r : 0)) * (K / 8) +
                                      (kbase + g * kTcKB + 32 * pc) / 8;
                cp_async_16(slot_addr(j, half), src, in ? 16u : 0u);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < kTcRing; ++i) issue(i);
        // expand one row's piece: codes minus the zero-point as s8, two 16-byte
        // chunks.  Per byte, q + (128 - z) lies in [113, 143] (no carry into the
        // next byte), and flipping bit 7 leaves q - z in two's complement.
        auto expand = [&](uint8_t *row, int r_t, const uint4 &w, uint32_t zw) {
            const uint32_t zoff = 0x80808080u - (zw & 15u) * 0x01010101u;
            const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // word k: codes 8 k .. 8 k + 7 of the piece
                const uint32_t lo = wd[k] & 0x0f0f0f0fu, hi = (wd[k] >> 4) & 0x0f0f0f0fu;
                o[2 * k] = (__byte_perm(lo, hi, 0x5140) + zoff) ^ 0x80808080u;
                o[2 * k + 1] = (__byte_perm(lo, hi, 0x7362) + zoff) ^ 0x80808080u;
            }
            *reinterpret_cast<uint4 *>(row + (((2 * pc) ^ (r_t & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4 *>(row + (((2 * pc + 1) ^ (r_t & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        };
        bool ok = true;
#pragma unroll
        for (int j = 0; j < kTcMaxTiles * kTcBlocks; ++j) {
            if (j < nsteps && ok) {
                const int s = j % kTcStages;
                if (j >= kTcStages) {
                    ok = mbar_wait_spin(a_empty(s), static_cast<uint32_t>((j / kTcStages) - 1) & 1u, abort_flag, p.status,
                                   SITE_W4_STAGE);
                    ok = __all_sync(0xffffffffu, ok);
                }
                if (ok) {
                    const int t = j / kTcBlocks, g = j - t * kTcBlocks;
                    // this step's copies have landed (at most kTcRing - 1 later groups pending)
                    cp_async_wait_pending(min(kTcRing, kTcMaxTiles * kTcBlocks - j) - 1);
                    uint4 wa, wb;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(wa.x), "=r"(wa.y), "=r"(wa.z), "=r"(wa.w) : "r"(slot_addr(j, 0)));
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(wb.x), "=r"(wb.y), "=r"(wb.z), "=r"(wb.w) : "r"(slot_addr(j, 1)));
                    const int zsh = zshift[g];
                    uint8_t *stage = smem + TcLayout::OFF_A + s * kTcABytes;
                    if (t * kTcRows + rr < rows) expand(stage + rr * 128, rr, wa, zs[t * kTcRows + rr] >> zsh);
                    if (t * kTcRows + rr + 64 < rows)
                        expand(stage + (rr + 64) * 128, rr + 64, wb, zs[t * kTcRows + rr + 64] >> zsh);
                    // the slot's pieces are in registers: refill it
                    if (j + kTcRing < kTcMaxTiles * kTcBlocks) issue(j + kTcRing);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(a_full(s));
                }
            }
        }
        cp_async_wait_all();  // (copies issued past the last step land before the CTA exits)
    } else if (warp == 16 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_i8(kTcRows, kTcCols, true, true, false);
        bool ok = true;
        for (int j = 0; j < nsteps && ok; ++j) {
            const int s = j % kTcStages, b = j % kTcBufs, g = j % kTcBlocks;
            if (j >= kTcBufs && !mbar_wait_spin(t_empty(b), static_cast<uint32_t>((j / kTcBufs) - 1) & 1u, abort_flag,
                                           p.status, SITE_W4_STAGE)) {
                ok = false;
                break;
            }
            if (!mbar_wait_spin(a_full(s), static_cast<uint32_t>(j / kTcStages) & 1u, abort_flag, p.status,
                           SITE_W4_STAGE)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = sbase + TcLayout::OFF_A + s * kTcABytes;
            const uint32_t b_addr = sbase + TcLayout::OFF_B + g * kTcBBlock;
            const uint32_t d_tmem = tbase + static_cast<uint32_t>(b * 128);
#pragma unroll
            for (int kk = 0; kk < kTcKB / 32; ++kk)
                tc_mma_i8(d_tmem, smem_desc_kmajor_sw128(a_addr + 32 * kk), smem_desc_kmajor_sw128(b_addr + 32 * kk),
                          idesc, kk != 0 ? 1u : 0u);
            tc_commit(a_empty(s));
            tc_commit(t_full(b));
        }
        if (!ok) {  // wait until every MMA issued so far has completed
            tc_commit(drain);
            mbar_drain(drain, 0, kWaitLimitNs);
        }
    } else if (warp >= 8 && warp < 16) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;          // TMEM lane quarter
        const int th = (warp - 8) >> 2;  // tokens 16 th .. 16 th + 15
        const int r_in = 32 * q + lane;
        const int *grp_of = reinterpret_cast<const int *>(smem + TcLayout::OFF_GT);
        // every scale of this CTA's steps into shared memory at once (one
        // memory latency for all of them, not one per step): the two warps of
        // a lane quarter take two tiles each
        uint16_t *sc_tab = reinterpret_cast<uint16_t *>(smem + TcLayout::OFF_SC);
#pragma unroll
        for (int tt = 0; tt < kTcMaxTiles / 2; ++tt) {
            const int t = 2 * th + tt, r = t * kTcRows + r_in;
#pragma unroll
            for (int g = 0; g < kTcBlocks; ++g)
                sc_tab[(t * kTcBlocks + g) * kTcRows + r_in] =
                    t < ntiles && r < rows ? __ldg(p.scales + static_cast<int64_t>(n0 + r) * G + grp_of[g])
                                           : static_cast<uint16_t>(0);
        }
        named_bar_sync(1, 256);  // the eight epilogue warps
        float acc[16];
        for (int j = 0; j < nsteps; ++j) {
            const int t = j / kTcBlocks, g = j - t * kTcBlocks, b = j % kTcBufs;
            const int r = t * kTcRows + r_in;
            const bool valid = r < rows;
            if (g == 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = 0.f;
            }
            const float sc = __half2float(__ushort_as_half(sc_tab[j * kTcRows + r_in]));
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait_spin(t_full(b), static_cast<uint32_t>(j / kTcBufs) & 1u, abort_flag, p.status,
                               SITE_W4_STAGE);
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
            tc_fence_after();
            uint32_t d0[16], d1[16], d2[16];
            const uint32_t taddr = tbase + static_cast<uint32_t>(b * 128 + 16 * th) +
                                   (static_cast<uint32_t>(32 * q) << 16);
            tmem_ld_32x32b_x16(taddr, d0);
            tmem_ld_32x32b_x16(taddr + kTcTok, d1);
            tmem_ld_32x32b_x16(taddr + 2 * kTcTok, d2);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(t_empty(b));
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float T = fmaf(65536.0f, tc_exact_float(static_cast<int>(d0[i])),
                                     fmaf(256.0f, tc_exact_float(static_cast<int>(d1[i])),
                                          tc_exact_float(static_cast<int>(d2[i]))));
                acc[i] = fmaf(sc, T, acc[i]);
            }
            if (g == kTcBlocks - 1 && valid) {
                float *dst = p.part + (static_cast<int64_t>(ks) * kTcTok + 16 * th) * p.N + n0 + r;
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[static_cast<int64_t>(i) * p.N] = acc[i];
            }
        }
    }

    __syncthreads();
    if (warp == 17) {
        tc_fence_after();
        tmem_dealloc(tbase, kTcTmemCols);
    }
}

size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int tc_slices(int64_t K) { return static_cast<int>(K / kTcKS); }

int tc_row_tiles(int64_t N, int64_t K, const DevInfo &dev) {
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(N, dev.num_sms / tc_slices(K))));
}

template <typename KernT, typename... Args>
cudaError_t launch_pdl(KernT kern, unsigned grid, unsigned block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

bool w4_tc_supported(int64_t M, int64_t N, int64_t K, int64_t gs, const DevInfo &dev) {
    if (M < 2 || M > kTcTok || K % kTcKS != 0 || K > 16 * kTcKS || gs % kTcKB != 0 || K % gs != 0) return false;
    const int64_t R = tc_row_tiles(N, K, dev);
    if (R * tc_slices(K) > dev.num_sms) return false;  // one wave
    if ((N + R - 1) / R > static_cast<int64_t>(kTcMaxTiles) * kTcRows) return false;
    return TcLayout::SMEM <= dev.max_smem_optin;
}

size_t w4_tc_workspace_bytes(int64_t N, int64_t K) {
    return a256(static_cast<size_t>(kTcCols) * K) + a256(4 * kTcTok * (K / kTcKS)) +
           static_cast<size_t>(K / kTcKS) * N * kTcTok * 4;
}

cudaError_t launch_w4_tc(const float *x, int64_t M, int64_t K, const uint32_t *qweight, const uint16_t *scales,
                         const uint32_t *qzeros, const float *bias, int64_t N, int64_t gs, float *out, void *ws,
                         cudaStream_t s, const DevInfo &dev) {
    uint8_t *w = static_cast<uint8_t *>(ws);
    int8_t *planes = reinterpret_cast<int8_t *>(w);
    float *sx = reinterpret_cast<float *>(w + a256(static_cast<size_t>(kTcCols) * K));
    float *part = reinterpret_cast<float *>(w + a256(static_cast<size_t>(kTcCols) * K) +
                                            a256(4 * kTcTok * static_cast<size_t>(K / kTcKS)));
    cudaError_t e = launch_pdl(w4_planes_kernel, static_cast<unsigned>(kTcTok * (K / kTcKS)), 256, 0, s, x,
                               static_cast<int>(M), static_cast<int>(K), planes, sx);
    if (e != cudaSuccess) return e;
    TcArgs a;
    a.qweight = qweight;
    a.scales = scales;
    a.qzeros = qzeros;
    a.planes = planes;
    a.part = part;
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.gs = static_cast<int>(gs);
    a.S = tc_slices(K);
    a.R = tc_row_tiles(N, K, dev);
    a.status = dev.status;
    static SmemOptIn opt_in;
    e = smem_opt_in(opt_in, dev, reinterpret_cast<const void *>(w4_tc_kernel), static_cast<size_t>(TcLayout::SMEM));
    if (e != cudaSuccess) return e;
    e = launch_pdl(w4_tc_kernel, static_cast<unsigned>(a.R * a.S), kTcThreads, TcLayout::SMEM, s, a);
    if (e != cudaSuccess) return e;
    const int64_t total = N * M;
    const unsigned rgrid = static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, 4 * dev.num_sms));
    return launch_pdl(w4_reduce_kernel, rgrid, 256, 0, s, static_cast<const float *>(part),
                      static_cast<const float *>(sx), bias, static_cast<int>(M), static_cast<int>(N), a.S, out);
}

}  // namespace bq
