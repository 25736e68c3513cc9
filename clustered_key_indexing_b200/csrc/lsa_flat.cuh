// lsa_flat.cuh -- flat search of the LSA path on sm_100a [essay "《卡片柜》——
// 当注意力学会先查目录再翻书", ch. 3: score every centroid, expand the best
// buckets until k long-range keys are filled; ch. 5: native max over heads].
//
// Per chunk of query positions:
//   sample_gather_kernel (once per call)  every 8th centroid of each kv-head
//       and its (first eligible position, key count), packed contiguously;
//   flat_tc_kernel  one CTA per 128 latent rows of one kv-head, on the 5th-
//       generation tensor cores (TMA -> shared memory -> tcgen05.mma ->
//       TMEM, bf16 in, fp32 accumulate).  Phase 1 scores the rows against the
//       sampled centroids and builds a per-row weighted histogram (bins
//       scaled to the row's latent norm, which bounds its scores) whose upper
//       tail gives a threshold tau expected to keep about twice the k keys
//       needed; phase 2 scores every eligible centroid and appends scores
//       >= tau to the row's candidate list in ascending bucket id;
//   flat_resolve_kernel  one warp per (query, kv-head): eligibility and
//       exact key counts, weighted radix select on the fp32 scores for the
//       cut c32, exact fp64 rescoring of the buckets within 2e of c32 only,
//       key emission in bucket id order, sinks and window.
// Exactness: |fp32 score - exact score| < e = 1e-4 (the error is below
// 64 * 2^-23 * |y||c|, whatever order the tensor core sums in).  The exact
// score E* of the k-th key then lies in [c32 - e, c32 + e]: buckets with fp32
// score > c32 + 2e rank strictly above it, buckets below c32 - 2e strictly
// below, and only the band between is ranked on exact fp64 scores (score
// desc, bucket id asc).  The band must lie above tau (every bucket in it is
// then a candidate); rows where it does not, or whose list overflowed, go to
// the exact fallback kernel.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"
#include "lsa_tc.cuh"

namespace lsa {

constexpr int kCandCap = 1024;       // candidates kept per (query, kv-head)
constexpr int kSampleStride = 8;     // every 8th bucket scored by the sample phase
constexpr int kOversample = 2;       // tau targets kOversample * k keys
constexpr float kScoreErr = 1e-4f;   // bound on |fp32 score - exact score|

// tcgen05 tile of the flat pass.  A CTA scores 256 latent rows (two M = 128
// blocks, each its own MMA) against 128 centroids per tile: K = 64 (four MMAs
// of K = 16) plus, in the candidate phase, one more K = 16 step that adds -tau
// to every row (A holds -tau in its first extra column, B a 1 there), so TMEM
// holds s - tau and a hit is a clear sign bit.  A 3-stage TMA ring of centroid
// tiles; TMEM = 2 buffers x 2 blocks x 128 fp32 columns; eight epilogue warps,
// each owning 32 rows of one block (TMEM lane quarter = warp % 4), a thread
// per row.
constexpr int kTcBlocks = 2;
constexpr int kTcRows = 128 * kTcBlocks;
constexpr int kTcCols = 128;
constexpr int kTcStages = 3;
constexpr int kTcEpi = 32 * 4 * kTcBlocks;         // epilogue threads, one per row
constexpr int kTcThreads = 64 + kTcEpi;            // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-9 epilogue
constexpr int kHBins = 128;                        // sample histogram bins per row
constexpr uint32_t kTcABytes = 128 * kDL * 2;      // 16 KB per block, 128-byte swizzle
constexpr uint32_t kTcAxBytes = 128 * 16 * 2;      // 4 KB per block, extra K = 16 of A, no swizzle
constexpr uint32_t kTcBxBytes = kTcCols * 16 * 2;  // 4 KB, extra K = 16 of B, no swizzle
constexpr uint32_t kTcBBytes = kTcCols * kDL * 2;  // 16 KB per stage
constexpr uint32_t kTcTmemCols = 2 * kTcBlocks * kTcCols;
constexpr uint32_t kTcHistBytes = kHBins * kTcRows * 4;       // [bin][row] counts (sample phase)
constexpr int kTcStgStride = 36;                              // floats per row in the staging rows
constexpr uint32_t kTcStgBytes = kTcRows * kTcStgStride * 4;  // candidate phase; shares the histogram's space
constexpr uint32_t kTcScratchBytes = kTcHistBytes > kTcStgBytes ? kTcHistBytes : kTcStgBytes;
constexpr size_t kTcSmemBytes = 1024 + kTcBlocks * (kTcABytes + kTcAxBytes) + kTcBxBytes + kTcStages * kTcBBytes +
                                kTcScratchBytes + 256;
constexpr uint32_t kTcIdesc = umma_idesc_bf16(128, kTcCols);
static_assert(kTcSmemBytes <= 232448, "flat_tc_kernel shared memory");

struct PassArgs {
    const uint16_t* Y;       // chunk latents [nqc, hkv, 64] (mean) / [nqc, hq, 64] (native)
    int64_t cap_buckets, ns_cap, NB, nqc, t_first;
    int32_t W, hkv, G, agg, k, S;
    float* tau;              // [nqc * hkv]
    int2* cand;              // [nqc * hkv, kCandCap] (bucket id, fp32 score bits)
    int32_t* cand_n;         // [nqc * hkv]
};

__host__ __device__ __forceinline__ int64_t flat_ncol_d(int64_t t, int32_t W, int64_t NB) {
    const int64_t lim = t - W;
    if (lim < 0) return 0;
    const int64_t n = (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1);
    return n < NB ? n : NB;
}

// cent_s[h, j] = cent[h, 8j] for 8j < NB (zero past it).
__global__ void sample_gather_kernel(const uint16_t* __restrict__ cent, int64_t cap_buckets, int64_t NB,
                                     int64_t ns_cap, int32_t hkv, uint16_t* __restrict__ cent_s) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)hkv * ns_cap * 8) return;
    const int64_t row = idx >> 3;
    const int c = (int)(idx & 7);
    const int64_t h = row / ns_cap, b = (row % ns_cap) * kSampleStride;
    reinterpret_cast<uint4*>(cent_s + row * kDL)[c] =
        b < NB ? reinterpret_cast<const uint4*>(cent + (h * cap_buckets + b) * kDL)[c] : make_uint4(0, 0, 0, 0);
}

template <int G>
__device__ __forceinline__ void group_max(uint32_t (&v)[32]) {
#pragma unroll
    for (int off = 1; off < G; off <<= 1)
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = __float_as_uint(fmaxf(__uint_as_float(v[i]), __uint_as_float(__shfl_xor_sync(0xffffffffu, v[i], off))));
}

// Largest bf16 value <= x (x finite or -inf).
__device__ __forceinline__ float bf16_floor(float x) {
    uint32_t u = __float_as_uint(x);
    const uint32_t low = u & 0xFFFFu;
    u &= 0xFFFF0000u;
    if ((u >> 31) && low) u += 0x10000u;  // negative: truncation went up, step one ulp down
    return __uint_as_float(u);
}

// Element (row, k) of a K = 16, no-swizzle K-major operand: 8-row x 16-byte
// core matrices; 128 bytes between the two K halves, 256 between row groups.
__device__ __forceinline__ uint32_t noswz_off(int row, int khalf) {
    return (uint32_t)((row >> 3) * 256 + khalf * 128 + (row & 7) * 16);
}

// G: latent rows per query (1 for the group-mean score, hq / hkv for the
// native per-head max).
template <int G>
__global__ void __launch_bounds__(kTcThreads, 1)
flat_tc_kernel(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmS, PassArgs a) {
    extern __shared__ uint8_t tsm_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t* tsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sA = tsm;                                   // [block] 16 KB
    uint8_t* sB = sA + kTcBlocks * kTcABytes;            // [stage] 16 KB
    uint8_t* sAx = sB + kTcStages * kTcBBytes;           // [block] 4 KB
    uint8_t* sBx = sAx + kTcBlocks * kTcAxBytes;         // 4 KB
    uint8_t* scratch = sBx + kTcBxBytes;                 // histogram, then staging rows
    uint32_t* hist = reinterpret_cast<uint32_t*>(scratch);
    float* stg = reinterpret_cast<float*>(scratch);
    uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + kTcScratchBytes);
    // bars: full[S], empty[S], tfull[2], tempty[2], tau_ready, drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kTcStages + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    constexpr int qpt = kTcRows / G;
    const int64_t q0 = (int64_t)blockIdx.x * qpt;
    if (q0 >= a.nqc) return;
    const int64_t qlast = min(a.nqc - 1, q0 + qpt - 1);
    const int64_t ncol_max = flat_ncol_d(a.t_first + qlast, a.W, a.NB);
    const int64_t ncol_min = flat_ncol_d(a.t_first + q0, a.W, a.NB);
    const int ns_tiles = (int)ceil_div<int64_t>(ceil_div<int64_t>(ncol_max, kSampleStride), kTcCols);
    const int ntiles = ns_tiles + (int)ceil_div<int64_t>(ncol_max, kTcCols);

    const uint32_t bar0 = smem_u32(bars);
    const uint32_t tau_ready = bar0 + 8u * (2 * kTcStages + 4);
    const uint32_t drain = bar0 + 8u * (2 * kTcStages + 5);
#define FULL(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY(s) (bar0 + 8u * (uint32_t)(kTcStages + (s)))
#define TFULL(b) (bar0 + 8u * (uint32_t)(2 * kTcStages + (b)))
#define TEMPTY(b) (bar0 + 8u * (uint32_t)(2 * kTcStages + 2 + (b)))

    if (tid == 0) {
        for (int s = 0; s < kTcStages; ++s) { mbar_init(FULL(s), 1); mbar_init(EMPTY(s), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(TFULL(b), 1); mbar_init(TEMPTY(b), kTcEpi); }
        mbar_init(tau_ready, kTcEpi);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTcTmemCols);
    for (int i = tid; i < kHBins * kTcRows; i += kTcThreads) hist[i] = 0u;
    // extra K step: B = 1 in its first column (bf16 0x3F80); A filled in once tau is known
    for (int i = tid; i < kTcCols * 2; i += kTcThreads) {
        const int n = i >> 1, kh = i & 1;
        *reinterpret_cast<uint4*>(sBx + noswz_off(n, kh)) = make_uint4(kh == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    if (tid >= 64) {
        // A: the CTA's 256 latent rows (block r / 128), 128-byte swizzled;
        // rows past the chunk are zero
        const int r = tid - 64;
        const int64_t q = q0 + r / G;
        uint4* dst = reinterpret_cast<uint4*>(sA + (r >> 7) * kTcABytes + (r & 127) * 128);
        if (q < a.nqc) {
            const int64_t yrow = G > 1 ? (q * a.hkv + h) * G + r % G : q * a.hkv + h;
            const uint4* src = reinterpret_cast<const uint4*>(a.Y + yrow * kDL);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c ^ (r & 7)] = src[c];
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // producer: sampled tiles first, then every eligible tile
            int issued = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % kTcStages;
                if (!mbar_wait(EMPTY(s), ((uint32_t)(it / kTcStages) & 1u) ^ 1u, abort_flag)) break;
                mbar_expect_tx(FULL(s), kTcBBytes);
                if (it < ns_tiles)
                    tma_load_2d(smem_u32(sB + s * kTcBBytes), &tmS, 0,
                                (int32_t)((int64_t)h * a.ns_cap + (int64_t)it * kTcCols), FULL(s));
                else
                    tma_load_2d(smem_u32(sB + s * kTcBBytes), &tmF, 0,
                                (int32_t)((int64_t)h * a.cap_buckets + (int64_t)(it - ns_tiles) * kTcCols), FULL(s));
                ++issued;
            }
            // after an abort, let this thread's copies land before the CTA exits
            if (*abort_flag)
                for (int it = max(0, issued - kTcStages); it < issued; ++it)
                    mbar_wait(FULL(it % kTcStages), (uint32_t)(it / kTcStages) & 1u, abort_flag, false);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint64_t bxd = noswz_desc(smem_u32(sBx), 128, 256);
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % kTcStages, b = it & 1;
                if (!mbar_wait(TEMPTY(b), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag)) break;
                if (!mbar_wait(FULL(s), (uint32_t)(it / kTcStages) & 1u, abort_flag)) break;
                if (it == ns_tiles && !mbar_wait(tau_ready, 0, abort_flag)) break;
                tc_fence_after();
                const uint32_t b0 = smem_u32(sB + s * kTcBBytes);
#pragma unroll
                for (int blk = 0; blk < kTcBlocks; ++blk) {
                    const uint32_t d = tmem + (uint32_t)((b * kTcBlocks + blk) * kTcCols);
                    const uint32_t a0 = smem_u32(sA + blk * kTcABytes);
#pragma unroll
                    for (int k = 0; k < kDL / 16; ++k)
                        umma_bf16(d, sw128_desc(a0 + 32u * k), sw128_desc(b0 + 32u * k), kTcIdesc, k > 0 ? 1u : 0u);
                    if (it >= ns_tiles)
                        umma_bf16(d, noswz_desc(smem_u32(sAx + blk * kTcAxBytes), 128, 256), bxd, kTcIdesc, 1u);
                }
                umma_commit(EMPTY(s));
                umma_commit(TFULL(b));
            }
            // every MMA this thread issued has completed once `drain` fires
            umma_commit(drain);
            mbar_wait(drain, 0, abort_flag, false);
        }
    } else {
        // epilogue: warp w owns rows 128 * blk + 32 * (w % 4) + lane of block
        // blk = (w - 2) / 4 (TMEM lane quarter w % 4)
        const int quarter = warp & 3, blk = (warp - 2) >> 2;
        const int r = blk * 128 + quarter * 32 + lane;
        const int64_t q = q0 + r / G;
        const bool valid = q < a.nqc;
        const bool owner = valid && (r % G) == 0;
        const int64_t qq = valid ? q : 0;
        const int64_t t = a.t_first + qq;
        const int ncol = (int)flat_ncol_d(t, a.W, a.NB);
        const int64_t orow = qq * a.hkv + h;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(blk * kTcCols);

        // R bounds |score| of the row: |s| <= |y| |c| < 1.01 |y| (|c| <= 1 + 2^-8)
        float n2 = 0.f;
        {
            const int64_t yrow = G > 1 ? (qq * a.hkv + h) * G + r % G : orow;
            const uint4* yp = reinterpret_cast<const uint4*>(a.Y + yrow * kDL);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 u = yp[c];
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float lo = __uint_as_float(w4[x] << 16), hi = __uint_as_float(w4[x] & 0xFFFF0000u);
                    n2 += lo * lo + hi * hi;
                }
            }
#pragma unroll
            for (int off = 1; off < G; off <<= 1) n2 = fmaxf(n2, __shfl_xor_sync(0xffffffffu, n2, off));
        }
        const float R = sqrtf(n2) * 1.01f + 1e-6f;
        // Eligible long-range keys of the row: positions S .. t - W.  Rows
        // with at most kOversample * k of them and no more than kCandCap
        // buckets in range take every bucket (tau = -inf).  Histogram range
        // [lo, R): rows with at least four times that target bin [0, R) only
        // (their tau lies in the upper tail), others the whole [-R, R).  Bin of s:
        // round(s * bsc + boff - 0.5), computed by adding 1.5 * 2^23 (the
        // float's last place is then 1) and clamped to [0, kHBins).
        const long long n_elig = max(0LL, (long long)(t - a.W) - a.S + 1);
        const bool take_all = n_elig <= (long long)kOversample * a.k && ncol <= kCandCap;
        const bool upper = n_elig >= 4LL * kOversample * a.k;
        const float lo = upper ? 0.f : -R;
        const float bsc = (float)kHBins / (R - lo);
        const float boff = -lo * bsc - 0.5f + 12582912.0f;

        uint32_t va[32], vb[32];
        int it = 0;
        // phase 1: histogram of the sampled scores, one count per sampled
        // bucket (buckets hold 8 keys on average, a block's 512 keys in 64)
        for (; it < ns_tiles; ++it) {
            const int b = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(TFULL(b), (uint32_t)(it >> 1) & 1u, abort_flag))) break;
            tc_fence_after();
            const uint32_t tb = trow + (uint32_t)(b * kTcBlocks * kTcCols);
            auto sample_chunk = [&](uint32_t (&v)[32], uint32_t (&vn)[32], int c) {
                if (c + 1 < kTcCols / 32) tmem_ld32_async(tb + (uint32_t)((c + 1) * 32), vn);
                group_max<G>(v);
                const int j0 = it * kTcCols + c * 32;  // sampled column; its bucket is 8 j
                // columns a row may score: 8 j < ncol
                const int nval = !owner ? 0 : min(32, max(0, (ncol + kSampleStride - 1) / kSampleStride - j0));
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int bin = min(kHBins - 1, max(0, __float_as_int(fmaf(__uint_as_float(v[i]), bsc, boff)) - 0x4B400000));
                    if (i < nval) atomicAdd(&hist[bin * kTcRows + r], 1u);
                }
                if (c + 1 < kTcCols / 32) tmem_wait_ld(vn);
            };
            tmem_ld32_async(tb, va);
            tmem_wait_ld(va);
#pragma unroll 1
            for (int c = 0; c < kTcCols / 32; c += 2) {
                sample_chunk(va, vb, c);
                sample_chunk(vb, va, c + 1);
            }
            tc_fence_before();
            mbar_arrive(TEMPTY(b));
        }
        // tau: lower edge of the bin where the sampled key estimate (8 keys
        // per bucket, every 8th bucket) from the top first reaches
        // kOversample * k, rounded down to bf16 (it enters the extra K step);
        // -inf if never (the upper-only range then still reports the whole
        // count at bin 0, so an upper row whose target lies below 0 gets 0)
        float tau = -CUDART_INF_F;
        if (!take_all) {
            long long cum = 0;
            const long long need = ((long long)kOversample * a.k + 63) / 64;  // sampled buckets
            for (int bn = kHBins - 1; bn >= 0; --bn) {
                cum += hist[bn * kTcRows + r];
                if (cum >= need) { tau = lo + bn * ((R - lo) / kHBins); break; }
            }
        }
        tau = bf16_floor(tau);
        if (G > 1) tau = __shfl_sync(0xffffffffu, tau, lane & ~(G - 1));  // the query's owner lane
        const bool tau_inf = tau == -CUDART_INF_F;
        const float tau_add = tau_inf ? 0.f : tau;
        if (owner) a.tau[orow] = tau;
        {
            uint8_t* ax = sAx + blk * kTcAxBytes;
            const int rb = quarter * 32 + lane;
            const uint32_t nb = (uint32_t)(__float_as_uint(-tau_add) >> 16);  // exact: tau_add is a bf16 value
            *reinterpret_cast<uint4*>(ax + noswz_off(rb, 0)) = make_uint4(nb, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(ax + noswz_off(rb, 1)) = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem();
            mbar_arrive(tau_ready);
        }
        // the histogram's space becomes the staging rows: every epilogue
        // thread has read its bins past this barrier
        asm volatile("bar.sync 1, %0;\n" ::"n"(kTcEpi) : "memory");
        float* my_stg = stg + r * kTcStgStride;

        // phase 2: TMEM holds s - tau_add; candidates (score >= tau) are
        // appended in ascending bucket id (the thread owns its row)
        int2* cand = a.cand + orow * (int64_t)kCandCap;
        int cnt = 0;
        for (; it < ntiles; ++it) {
            const int b = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(TFULL(b), (uint32_t)(it >> 1) & 1u, abort_flag))) break;
            tc_fence_after();
            const uint32_t tb = trow + (uint32_t)(b * kTcBlocks * kTcCols);
            const int tbase = (it - ns_tiles) * kTcCols;
            auto cand_chunk = [&](uint32_t (&v)[32], uint32_t (&vn)[32], int c) {
                if (c + 1 < kTcCols / 32) tmem_ld32_async(tb + (uint32_t)((c + 1) * 32), vn);
                group_max<G>(v);
                const int col0 = tbase + c * 32;
                const int rem = ncol - col0;
                const uint32_t lm = !owner || rem <= 0 ? 0u : (rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u));
                // sign bits of s - tau: bit i set = miss
                uint32_t shi = 0u, slo = 0u;
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    shi = __funnelshift_l(v[16 + i], shi, 1);
                    slo = __funnelshift_l(v[i], slo, 1);
                }
                uint32_t hits = (tau_inf ? 0xffffffffu : ~((shi << 16) | slo)) & lm;
                if (__any_sync(0xffffffffu, hits)) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        reinterpret_cast<uint4*>(my_stg)[j] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    while (hits) {
                        const int i = __ffs(hits) - 1;
                        hits &= hits - 1u;
                        if (cnt < kCandCap) cand[cnt] = make_int2(col0 + i, __float_as_int(my_stg[i] + tau_add));
                        ++cnt;
                    }
                }
                if (c + 1 < kTcCols / 32) tmem_wait_ld(vn);
            };
            tmem_ld32_async(tb, va);
            tmem_wait_ld(va);
#pragma unroll 1
            for (int c = 0; c < kTcCols / 32; c += 2) {
                cand_chunk(va, vb, c);
                cand_chunk(vb, va, c + 1);
            }
            tc_fence_before();
            mbar_arrive(TEMPTY(b));
        }
        if (owner) a.cand_n[orow] = cnt;
    }
#undef FULL
#undef EMPTY
#undef TFULL
#undef TEMPTY
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

// --------------------------------------------------------------- resolve

constexpr int kResWarps = 4;

struct ResolveArgs {
    const int32_t* units;
    const int32_t* offsets;
    const int32_t* members;
    const int32_t* cnt_lr;
    const int32_t* minlr;
    const int32_t* maxpos;
    const uint16_t* cent;
    int64_t cap_units, cap_buckets, NB, T_built;
    int32_t hkv, G, agg, k, S, W;
    const uint16_t* Y;
    int64_t nqc, t_first;
    const float* tau;
    const int2* cand;
    const int32_t* cand_n;
    int32_t* idx;
    int32_t* ovf_rows;
    int32_t* ovf_count;
    int32_t ovf_cap;
};

constexpr int kBandCap = 128;  // buckets ranked on exact scores per row

struct ResWarp {
    double bex[kBandCap];     // exact scores of the band
    int32_t col[kCandCap];    // eligible candidates, ascending bucket id
    float sc[kCandCap];       // their fp32 scores
    int32_t w[kCandCap];      // key weights, then taken counts
    int32_t pk[kCandCap];     // packed member units
    int32_t bidx[kBandCap];   // band members (index into col)
    uint32_t hist[256];
    uint16_t ylat[8 * kDL];
};

__device__ __forceinline__ uint32_t order_key_f(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);
    return (u >> 31) ? ~u : (u | 0x80000000u);
}

// Keys of bucket b in [S, lim]; `pk` is the bucket's packed member units.
__device__ __forceinline__ int weight_packed(const ResolveArgs& a, int64_t b, int32_t pk, int64_t lim) {
    const int64_t ubase = (b / kBucketsPerBlock) * kUnitsPerBlock;
    const int cnt = (pk >> 28) & 7;
    int w = 0;
    for (int i = 0; i < cnt; ++i) {
        const int64_t j = ubase + ((pk >> (7 * i)) & 127);
        for (int64_t p = j * kPool; p < j * kPool + kPool && p < a.T_built; ++p)
            if (p >= a.S && p <= lim) ++w;
    }
    return w;
}

// First `tk` keys of bucket b in [S, lim], ascending (member units are
// packed in ascending order).  Fast path: a bucket taken whole that lies
// inside [S, lim] with full units writes 4 consecutive positions per unit.
__device__ void emit_keys(const ResolveArgs& a, int64_t b, int32_t pk, int tk, int64_t lim,
                          int32_t* out) {
    const int64_t ubase = (b / kBucketsPerBlock) * kUnitsPerBlock;
    const int cnt = (pk >> 28) & 7;
    const int64_t j0 = ubase + (pk & 127);
    if (tk == cnt * kPool && j0 * kPool >= a.S) {
        int o = 0;
        for (int i = 0; i < cnt; ++i) {
            const int32_t p = (int32_t)((ubase + ((pk >> (7 * i)) & 127)) * kPool);
            out[o] = p; out[o + 1] = p + 1; out[o + 2] = p + 2; out[o + 3] = p + 3;
            o += 4;
        }
        return;
    }
    int o = 0;
    for (int i = 0; i < cnt && o < tk; ++i) {
        const int64_t j = ubase + ((pk >> (7 * i)) & 127);
        for (int64_t p = j * kPool; p < j * kPool + kPool && p < a.T_built && o < tk; ++p)
            if (p >= a.S && p <= lim) out[o++] = (int32_t)p;
    }
}

// Exact score (fp64, ascending dims) of one centroid row against the warp's
// query latent(s) in shared memory; the row is read with 16-byte loads.
__device__ __forceinline__ double exact_row(const uint16_t* ylat, int ng, const uint16_t* c) {
    uint4 cv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) cv[i] = __ldg(reinterpret_cast<const uint4*>(c) + i);
    double best = -CUDART_INF;
    for (int g = 0; g < ng; ++g) {
        const uint16_t* y = ylat + g * kDL;
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t wv[4] = {cv[i].x, cv[i].y, cv[i].z, cv[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s = fma(bf16_to_f64(y[8 * i + 2 * e]), (double)__uint_as_float(wv[e] << 16), s);
                s = fma(bf16_to_f64(y[8 * i + 2 * e + 1]), (double)__uint_as_float(wv[e] & 0xFFFF0000u), s);
            }
        }
        best = s > best ? s : best;
    }
    return best;
}

__device__ __forceinline__ void push_fallback(const ResolveArgs& a, int64_t row) {
    atomicAdd(&g_lsa_fallback_rows, 1ull);
    const int slot = atomicAdd(a.ovf_count, 1);
    if (slot < a.ovf_cap) a.ovf_rows[slot] = (int32_t)row;
    else raise_device_error(kErrSelectOverflow);
}

__global__ void __launch_bounds__(32 * kResWarps, 4) flat_resolve_kernel(ResolveArgs a) {
    extern __shared__ __align__(16) uint8_t rsm[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    ResWarp& sw = reinterpret_cast<ResWarp*>(rsm)[wid];
    const int64_t row = (int64_t)blockIdx.x * kResWarps + wid;
    if (row >= a.nqc * a.hkv) return;
    const int64_t q = row / a.hkv;
    const int h = (int)(row % a.hkv);
    const int64_t t = a.t_first + q;
    const int64_t lim = t - a.W;
    int32_t* out = a.idx + row * (int64_t)(a.S + a.k + a.W);

    // sinks and window
    for (int i = lane; i < a.S; i += 32) out[i] = (i <= t) ? i : -1;
    const int64_t w0 = max((int64_t)a.S, t - a.W + 1);
    const int64_t nw = t >= a.S ? t - w0 + 1 : 0;
    for (int i = lane; i < a.W; i += 32) out[a.S + a.k + i] = i < nw ? (int32_t)(w0 + i) : -1;
    if (lim < a.S) {
        for (int i = lane; i < a.k; i += 32) out[a.S + i] = -1;
        return;
    }
    const int n = a.cand_n[row];
    if (n > kCandCap) {
        if (lane == 0) push_fallback(a, row);
        return;
    }
    const float tau = a.tau[row];

    // eligible candidates (kept in ascending bucket id) and their key counts
    const int64_t hb0 = (int64_t)h * a.cap_buckets;
    int m = 0;
    long long wtot = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        bool el = false;
        int col = 0, wgt = 0;
        float sc = 0.f;
        int32_t pk = 0;
        if (i < n) {
            const int2 cv = a.cand[row * kCandCap + i];
            col = cv.x;
            sc = __int_as_float(cv.y);
            const int64_t hb = hb0 + col;
            const int32_t mlr = a.minlr[hb], mxp = a.maxpos[hb], clr = a.cnt_lr[hb];
            pk = a.units[hb];
            el = (int64_t)mlr <= lim;
            wgt = (int64_t)mxp <= lim ? clr : weight_packed(a, col, pk, lim);
        }
        if (el) wtot += wgt;
        const unsigned bal = __ballot_sync(0xffffffffu, el);
        if (el) {
            const int pos = m + __popc(bal & ((1u << lane) - 1u));
            sw.col[pos] = col;
            sw.sc[pos] = sc;
            sw.w[pos] = wgt;
            sw.pk[pos] = pk;
        }
        m += __popc(bal);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wtot += __shfl_xor_sync(0xffffffffu, wtot, off);
    __syncwarp();

    if (wtot > a.k) {
        // weighted radix select on the fp32 scores: cut key K32 with
        // weight(key > K32) < k <= weight(key >= K32)
        uint32_t prefix = 0;
        long long above = 0;
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = lane; i < 256; i += 32) sw.hist[i] = 0u;
            __syncwarp();
            for (int i = lane; i < m; i += 32) {
                const uint32_t key = order_key_f(sw.sc[i]);
                if (pass > 0 && (key >> (shift + 8)) != (prefix >> (shift + 8))) continue;
                atomicAdd(&sw.hist[(key >> shift) & 255u], (unsigned)sw.w[i]);
            }
            __syncwarp();
            long long s8 = 0;
            for (int d = 0; d < 8; ++d) s8 += sw.hist[255 - 8 * lane - d];
            long long incl = s8;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const long long excl = incl - s8;
            const unsigned hitm = __ballot_sync(0xffffffffu, above + incl >= a.k && above + excl < a.k);
            if (hitm == 0u) {  // cannot happen while the weight above the prefix reaches k
                if (lane == 0) push_fallback(a, row);
                return;
            }
            const int src = __ffs(hitm) - 1;
            int dig = 0;
            long long cum = 0;
            if (lane == src) {
                cum = above + excl;
                dig = 255 - 8 * lane;
                for (int d = 0; d < 8; ++d) {
                    const int dd = 255 - 8 * lane - d;
                    if (cum + sw.hist[dd] >= a.k) { dig = dd; break; }
                    cum += sw.hist[dd];
                }
            }
            dig = __shfl_sync(0xffffffffu, dig, src);
            above = __shfl_sync(0xffffffffu, cum, src);
            prefix |= (uint32_t)dig << shift;
            __syncwarp();
        }
        const float c32 = __uint_as_float((prefix >> 31) ? (prefix & 0x7FFFFFFFu) : ~prefix);
        const float hi = c32 + 2.f * kScoreErr, lo = c32 - 2.f * kScoreErr;
        // every bucket that can rank above the exact cut must be a candidate:
        // non-candidates score <= tau (s - tau < 0 rounds to at most tau)
        if (tau > -CUDART_INF_F && !(lo > tau)) {
            if (lane == 0) push_fallback(a, row);
            return;
        }
        // in (> hi): taken whole; out (< lo): not taken; band: exact ranking
        long long win = 0;
        int nb = 0;
        for (int base = 0; base < m; base += 32) {
            const int i = base + lane;
            const float sc = i < m ? sw.sc[i] : -CUDART_INF_F;
            const bool band = i < m && sc >= lo && sc <= hi;
            if (i < m && sc > hi) win += sw.w[i];
            const unsigned bal = __ballot_sync(0xffffffffu, band);
            if (band) {
                const int pos = nb + __popc(bal & ((1u << lane) - 1u));
                if (pos < kBandCap) sw.bidx[pos] = i;
            }
            nb += __popc(bal);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) win += __shfl_xor_sync(0xffffffffu, win, off);
        if (nb > kBandCap) {
            if (lane == 0) push_fallback(a, row);
            return;
        }
        const int ng = a.agg ? a.G : 1;
        const uint16_t* ysrc = a.agg ? a.Y + (q * (int64_t)a.hkv * a.G + (int64_t)h * a.G) * kDL
                                     : a.Y + row * kDL;
        for (int i = lane; i < ng * kDL; i += 32) sw.ylat[i] = ysrc[i];
        __syncwarp();
        for (int i = lane; i < nb; i += 32)
            sw.bex[i] = exact_row(sw.ylat, ng, a.cent + (hb0 + sw.col[sw.bidx[i]]) * kDL);
        __syncwarp();
        // taken counts: in -> whole, out -> 0, band -> pending (negative)
        for (int i = lane; i < m; i += 32) {
            const float sc = sw.sc[i];
            sw.w[i] = sc > hi ? sw.w[i] : (sc >= lo ? -sw.w[i] : 0);
        }
        __syncwarp();
        long long need = a.k - win;
        while (need > 0) {
            // best pending band bucket: exact score desc, bucket id asc
            double bs = -CUDART_INF;
            int bb = -1, bcol = 0x7FFFFFFF;
            for (int i = lane; i < nb; i += 32) {
                const int ci = sw.bidx[i];
                if (sw.w[ci] >= 0) continue;
                const double e = sw.bex[i];
                if (bb < 0 || e > bs || (e == bs && sw.col[ci] < bcol)) { bs = e; bb = ci; bcol = sw.col[ci]; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double os = __shfl_xor_sync(0xffffffffu, bs, off);
                const int ob = __shfl_xor_sync(0xffffffffu, bb, off);
                const int oc = __shfl_xor_sync(0xffffffffu, bcol, off);
                if (ob >= 0 && (bb < 0 || os > bs || (os == bs && oc < bcol))) { bs = os; bb = ob; bcol = oc; }
            }
            if (bb < 0) break;
            const int wv = -sw.w[bb];
            const int tk = wv < need ? wv : (int)need;
            __syncwarp();
            if (lane == 0) sw.w[bb] = tk;
            need -= tk;
            __syncwarp();
        }
        for (int i = lane; i < m; i += 32)
            if (sw.w[i] < 0) sw.w[i] = 0;
        __syncwarp();
    } else if (tau > -CUDART_INF_F) {
        // fewer than k keys among the candidates, but buckets below tau exist
        if (lane == 0) push_fallback(a, row);
        return;
    }
    // emit keys in ascending bucket id (candidates are already in that order)
    int run = 0;
    for (int base = 0; base < m; base += 32) {
        const int i = base + lane;
        const int tk = i < m ? sw.w[i] : 0;
        int incl = tk;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (tk > 0) emit_keys(a, sw.col[i], sw.pk[i], tk, lim, out + a.S + run + incl - tk);
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int i = run + lane; i < a.k; i += 32) out[a.S + i] = -1;
}

// ------------------------------------------------------------ host side

// Sampled centroids, once per call (the cache does not change between
// chunks).
lsa_status launch_sample_gather(const uint16_t* cent, int64_t cap_buckets, int64_t NB, int64_t ns_cap, int32_t hkv,
                                uint16_t* cent_s, cudaStream_t st) {
    const int64_t n = (int64_t)hkv * ns_cap * 8;
    sample_gather_kernel<<<(unsigned)ceil_div<int64_t>(n, 256), 256, 0, st>>>(cent, cap_buckets, NB, ns_cap, hkv,
                                                                              cent_s);
    return check_launch("sample_gather_kernel");
}

lsa_status launch_flat(const PassArgs& pa, const ResolveArgs& ra, const CUtensorMap& tmF, const CUtensorMap& tmS,
                       cudaStream_t st) {
    const int G = pa.agg ? pa.G : 1;
    const int qpt = kTcRows / G;
    dim3 grid((unsigned)ceil_div<int64_t>(pa.nqc, qpt), (unsigned)pa.hkv);
    auto kern = G == 1 ? flat_tc_kernel<1> : G == 2 ? flat_tc_kernel<2> : G == 4 ? flat_tc_kernel<4> : flat_tc_kernel<8>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmemBytes);
    kern<<<grid, kTcThreads, kTcSmemBytes, st>>>(tmF, tmS, pa);
    lsa_status s = check_launch("flat_tc_kernel");
    if (s != LSA_OK) return s;
    const size_t smem_r = sizeof(ResWarp) * kResWarps;
    cudaFuncSetAttribute(flat_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_r);
    const int64_t rows = pa.nqc * pa.hkv;
    flat_resolve_kernel<<<(unsigned)ceil_div<int64_t>(rows, kResWarps), 32 * kResWarps, smem_r, st>>>(ra);
    return check_launch("flat_resolve_kernel");
}

}  // namespace lsa
