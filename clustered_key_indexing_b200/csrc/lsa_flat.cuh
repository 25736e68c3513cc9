// lsa_flat.cuh -- flat search of the LSA path on sm_100a [essay "《卡片柜》——
// 当注意力学会先查目录再翻书", ch. 3: score every centroid, expand the best
// buckets until k long-range keys are filled; ch. 5: native max over heads].
//
// Per chunk of query positions:
//   sample_gather_kernel (once per call)  every 8th centroid of each kv-head,
//       packed contiguously;
//   flat_sample_kernel  tensor-core scores of the rows against the sampled
//       centroids; a per-row histogram (bins scaled to the row's latent norm,
//       which bounds its scores) whose upper tail gives a threshold tau
//       expected to keep about twice the k keys needed;
//   flat_cand_kernel  tensor-core scores against every eligible centroid;
//       scores >= tau are appended to the row's candidate list in ascending
//       bucket id;
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

// The flat pass runs on the 5th-generation tensor cores in two kernels per
// chunk, both TMA -> shared memory -> tcgen05.mma (bf16 in, fp32 accumulate
// in TMEM) -> tcgen05.ld, with one producer thread (warp 0), one MMA thread
// (warp 1, which also owns the TMEM allocation) and sixteen epilogue warps
// (TMEM lane quarter = warp % 4):
//   flat_sample_kernel  256 rows (two M = 128 blocks) x 128 sampled centroids
//       per tile, two epilogue threads per row, one per 64-column half of a
//       tile; per-row histogram of the sampled scores (both threads of a row
//       count into it) -> tau;
//   flat_cand_kernel    512 rows (four blocks) x 64 centroids per tile, plus
//       one K = 16 step that adds -tau to every row (A holds -tau in its first
//       extra column, B a 1 there), so TMEM holds s - tau and a hit is a clear
//       sign bit; hits are appended in ascending bucket id.  One epilogue
//       thread per row takes a whole tile row into registers with one TMEM
//       load, and the buffer goes back to the MMA thread before the scan.
//       (Two blocks of 128 columns read a third fewer operand bytes per
//       score; with a thread per 64-column half of a row and a per-tile
//       exchange of hit counts between the two, they ran 14% slower.)
constexpr uint32_t kTcABytes = 128 * kDL * 2;      // one M = 128 block of latents, 128-byte swizzle
constexpr uint32_t kTcAxBytes = 128 * 16 * 2;      // extra K = 16 of a block, no swizzle
constexpr int kHBins = 256;                        // sample histogram bins per row (16-bit counts)

constexpr int kSmBlocks = 2, kSmCols = 128, kSmStages = 3;
constexpr int kSmRows = 128 * kSmBlocks;
constexpr int kSmEpi = 2 * kSmRows;                  // epilogue threads: two per row
constexpr int kSmThreads = 64 + kSmEpi;
constexpr uint32_t kSmBBytes = kSmCols * kDL * 2;
constexpr uint32_t kSmHistBytes = kHBins / 2 * kSmRows * 4;  // [bin / 2][row] words, two counts each
constexpr size_t kSmSmemBytes = 1024 + kSmBlocks * kTcABytes + kSmStages * kSmBBytes + kSmHistBytes + 256;
static_assert(kSmSmemBytes <= 232448, "flat_sample_kernel shared memory");

constexpr int kCdBlocks = 4, kCdCols = 64, kCdStages = 4;  // the epilogue scans a tile as two 32-column halves
constexpr int kCdRows = 128 * kCdBlocks;
constexpr int kCdThreads = 64 + kCdRows;
constexpr uint32_t kCdBBytes = kCdCols * kDL * 2;
constexpr uint32_t kCdBxBytes = kCdCols * 16 * 2;
constexpr int kTcStgStride = 36;                               // floats per row in the staging rows
constexpr uint32_t kCdStgBytes = kCdRows * kTcStgStride * 4;
constexpr size_t kCdSmemBytes = 1024 + kCdBlocks * (kTcABytes + kTcAxBytes) + kCdStages * kCdBBytes + kCdBxBytes +
                                kCdStgBytes + 256;
static_assert(kCdSmemBytes <= 232448, "flat_cand_kernel shared memory");
static_assert(kCdCols == 64, "flat_cand_kernel epilogue: one 64-column TMEM load per tile");
static_assert(2 * kSmBlocks * kSmCols <= 512 && 2 * kCdBlocks * kCdCols <= 512, "TMEM columns");

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

// Latent row r of the CTA (query q0 + r / G) into block r / 128 of A,
// 128-byte swizzled (16-byte chunk c of row i at c ^ (i & 7)); zero past the chunk.
template <int G>
__device__ __forceinline__ void fill_a_row(uint8_t* sA, const PassArgs& a, int64_t q0, int h, int r) {
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

// Barrier layout shared by both kernels: full[S], empty[S], tfull[2],
// tempty[2], drain.
template <int STAGES>
struct TcBars {
    uint32_t b0;
    __device__ uint32_t full(int s) const { return b0 + 8u * (uint32_t)s; }
    __device__ uint32_t empty(int s) const { return b0 + 8u * (uint32_t)(STAGES + s); }
    __device__ uint32_t tfull(int b) const { return b0 + 8u * (uint32_t)(2 * STAGES + b); }
    __device__ uint32_t tempty(int b) const { return b0 + 8u * (uint32_t)(2 * STAGES + 2 + b); }
    __device__ uint32_t drain() const { return b0 + 8u * (uint32_t)(2 * STAGES + 4); }
    static constexpr int kCount = 2 * STAGES + 5;
    __device__ void init(int epi_threads) const {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(tfull(b), 1); mbar_init(tempty(b), (uint32_t)epi_threads); }
        mbar_init(drain(), 1);
    }
};

// Producer (one thread): tile `it` is rows row0 + it * ROWS of `map`.
template <int STAGES, int ROWS>
__device__ void tc_produce(const CUtensorMap* map, int64_t row0, int ntiles, uint8_t* sB, const TcBars<STAGES>& bar,
                           volatile int* abort_flag) {
    constexpr uint32_t bytes = ROWS * kDL * 2;
    int issued = 0;
    for (int it = 0; it < ntiles; ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(bar.empty(s), ((uint32_t)(it / STAGES) & 1u) ^ 1u, abort_flag)) break;
        mbar_expect_tx(bar.full(s), bytes);
        tma_load_2d(smem_u32(sB + s * bytes), map, 0, (int32_t)(row0 + (int64_t)it * ROWS), bar.full(s));
        ++issued;
    }
    // after an abort, let this thread's copies land before the CTA exits
    if (*abort_flag)
        for (int it = max(0, issued - STAGES); it < issued; ++it)
            mbar_wait(bar.full(it % STAGES), (uint32_t)(it / STAGES) & 1u, abort_flag, false);
}

// MMA issuer (one thread): per tile and block, D[(buf * BLK + blk) * N] =
// A_blk * B_tile^T over K = 64 (+ the extra K = 16 step when EXTRA).
template <int BLK, int N, int STAGES, bool EXTRA>
__device__ void tc_mma(uint32_t tmem, const uint8_t* sA, const uint8_t* sB, const uint8_t* sAx, const uint8_t* sBx,
                       int ntiles, const TcBars<STAGES>& bar, volatile int* abort_flag) {
    constexpr uint32_t idesc = umma_idesc_bf16(128, N);
    constexpr uint32_t bbytes = N * kDL * 2;
    for (int it = 0; it < ntiles; ++it) {
        const int s = it % STAGES, b = it & 1;
        if (!mbar_wait(bar.tempty(b), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag)) break;
        if (!mbar_wait(bar.full(s), (uint32_t)(it / STAGES) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t b0 = smem_u32(sB + s * bbytes);
#pragma unroll
        for (int blk = 0; blk < BLK; ++blk) {
            const uint32_t d = tmem + (uint32_t)((b * BLK + blk) * N);
            const uint32_t a0 = smem_u32(sA + blk * kTcABytes);
#pragma unroll
            for (int k = 0; k < kDL / 16; ++k)
                umma_bf16(d, sw128_desc(a0 + 32u * k), sw128_desc(b0 + 32u * k), idesc, k > 0 ? 1u : 0u);
            if (EXTRA)
                umma_bf16(d, noswz_desc(smem_u32(sAx + blk * kTcAxBytes), 128, 256), noswz_desc(smem_u32(sBx), 128, 256),
                          idesc, 1u);
        }
        umma_commit(bar.empty(s));
        umma_commit(bar.tfull(b));
    }
    // every MMA this thread issued has completed once `drain` fires
    umma_commit(bar.drain());
    mbar_wait(bar.drain(), 0, abort_flag, false);
}

// Epilogue row of a CTA: row r of the CTA's latent rows.
struct EpiRow {
    int64_t q, qq, t, orow;
    int ncol;
    bool valid, owner;
};

template <int G>
__device__ __forceinline__ EpiRow epi_row(const PassArgs& a, int64_t q0, int h, int r) {
    EpiRow e;
    e.q = q0 + r / G;
    e.valid = e.q < a.nqc;
    e.owner = e.valid && (r % G) == 0;
    e.qq = e.valid ? e.q : 0;
    e.t = a.t_first + e.qq;
    e.ncol = (int)flat_ncol_d(e.t, a.W, a.NB);
    e.orow = e.qq * a.hkv + h;
    return e;
}

// G: latent rows per query (1 for the group-mean score, hq / hkv for the
// native per-head max).
template <int G>
__global__ void __launch_bounds__(kSmThreads, 1)
flat_sample_kernel(const __grid_constant__ CUtensorMap tmS, PassArgs a) {
    extern __shared__ uint8_t tsm_raw[];
    uint8_t* tsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sA = tsm;                                   // [block] 16 KB
    uint8_t* sB = sA + kSmBlocks * kTcABytes;            // [stage] 16 KB
    uint32_t* hist = reinterpret_cast<uint32_t*>(sB + kSmStages * kSmBBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(hist) + kSmHistBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + TcBars<kSmStages>::kCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const TcBars<kSmStages> bar{smem_u32(bars)};

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    constexpr int qpt = kSmRows / G;
    const int64_t q0 = (int64_t)blockIdx.x * qpt;
    if (q0 >= a.nqc) return;
    const int64_t qlast = min(a.nqc - 1, q0 + qpt - 1);
    const int64_t ncol_max = flat_ncol_d(a.t_first + qlast, a.W, a.NB);
    const int ntiles = (int)ceil_div<int64_t>(ceil_div<int64_t>(ncol_max, kSampleStride), kSmCols);

    if (tid == 0) {
        bar.init(kSmEpi);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    for (int i = tid; i < kHBins / 2 * kSmRows; i += kSmThreads) hist[i] = 0u;
    // epilogue warps 2 .. 17: TMEM lane quarter warp % 4, then column half, then block
    const int quarter = warp & 3, half = ((warp - 2) >> 2) & 1, blk = (warp - 2) >> 3;
    const int r = blk * 128 + quarter * 32 + lane;  // epilogue row of this thread
    if (warp >= 2 && half == 0) fill_a_row<G>(sA, a, q0, h, r);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) tc_produce<kSmStages, kSmCols>(&tmS, (int64_t)h * a.ns_cap, ntiles, sB, bar, abort_flag);
    } else if (warp == 1) {
        if (lane == 0) tc_mma<kSmBlocks, kSmCols, kSmStages, false>(tmem, sA, sB, nullptr, nullptr, ntiles, bar, abort_flag);
    } else {
        const EpiRow e = epi_row<G>(a, q0, h, r);
        const uint32_t trow =
            tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(blk * kSmCols + half * (kSmCols / 2));
        // R bounds |score| of the row: |s| <= |y| |c| < 1.01 |y| (|c| <= 1 + 2^-8)
        float n2 = 0.f;
        {
            const int64_t yrow = G > 1 ? (e.qq * a.hkv + h) * G + r % G : e.orow;
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
        // (their tau lies in the upper tail), others the whole [-R, R).  Bin
        // of s: round(s * bsc + boff - 0.5), computed by adding 1.5 * 2^23
        // (the float's last place is then 1) and clamped to [0, kHBins).
        const long long n_elig = max(0LL, (long long)(e.t - a.W) - a.S + 1);
        const bool take_all = n_elig <= (long long)kOversample * a.k && e.ncol <= kCandCap;
        const bool upper = n_elig >= 4LL * kOversample * a.k;
        const float lo = upper ? 0.f : -R;
        const float bsc = (float)kHBins / (R - lo);
        const float boff = -lo * bsc - 0.5f + 12582912.0f;
        const int ns_row = e.owner ? (e.ncol + kSampleStride - 1) / kSampleStride : 0;

        // one count per sampled bucket (buckets hold 8 keys on average: a
        // block's 512 keys in 64); 16-bit counts, two bins per word
        for (int it = 0; it < ntiles; ++it) {
            const int b = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(bar.tfull(b), (uint32_t)(it >> 1) & 1u, abort_flag))) break;
            tc_fence_after();
            uint32_t v[64];
            tmem_ld64(trow + (uint32_t)(b * kSmBlocks * kSmCols), v);
            tc_fence_before();
            mbar_arrive(bar.tempty(b));
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t(&vv)[32] = *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c);
                group_max<G>(vv);
                const int nval = min(32, max(0, ns_row - (it * kSmCols + half * (kSmCols / 2) + c * 32)));
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int bin =
                        min(kHBins - 1, max(0, __float_as_int(fmaf(__uint_as_float(vv[i]), bsc, boff)) - 0x4B400000));
                    if (i < nval) atomicAdd(&hist[(bin >> 1) * kSmRows + r], 1u << ((bin & 1) << 4));
                }
            }
        }
        // both halves' counts are in before the row's tau is read off
        asm volatile("bar.sync 1, %0;\n" ::"n"(kSmEpi) : "memory");
        // tau: lower edge of the bin where the sampled key estimate (8 keys
        // per bucket, every 8th bucket) from the top first reaches
        // kOversample * k, rounded down to bf16 (it enters the extra K step
        // of the candidate kernel); -inf if never (an upper-range row whose
        // target lies below 0 gets 0: bin 0 holds every score below 0)
        float tau = -CUDART_INF_F;
        if (!take_all && half == 0) {
            long long cum = 0;
            const long long need = ((long long)kOversample * a.k + 63) / 64;  // sampled buckets
            for (int bn = kHBins - 1; bn >= 0; --bn) {
                cum += (hist[(bn >> 1) * kSmRows + r] >> ((bn & 1) << 4)) & 0xFFFFu;
                if (cum >= need) { tau = lo + bn * ((R - lo) / kHBins); break; }
            }
        }
        if (e.owner && half == 0) a.tau[e.orow] = bf16_floor(tau);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int G>
__global__ void __launch_bounds__(kCdThreads, 1)
flat_cand_kernel(const __grid_constant__ CUtensorMap tmF, PassArgs a) {
    extern __shared__ uint8_t tsm_raw[];
    uint8_t* tsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sA = tsm;                                   // [block] 16 KB
    uint8_t* sB = sA + kCdBlocks * kTcABytes;            // [stage] 8 KB
    uint8_t* sAx = sB + kCdStages * kCdBBytes;           // [block] 4 KB
    uint8_t* sBx = sAx + kCdBlocks * kTcAxBytes;         // 2 KB
    float* stg = reinterpret_cast<float*>(sBx + kCdBxBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stg) + kCdStgBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + TcBars<kCdStages>::kCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const TcBars<kCdStages> bar{smem_u32(bars)};

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    constexpr int qpt = kCdRows / G;
    const int64_t q0 = (int64_t)blockIdx.x * qpt;
    if (q0 >= a.nqc) return;
    const int64_t qlast = min(a.nqc - 1, q0 + qpt - 1);
    const int ntiles = (int)ceil_div<int64_t>(flat_ncol_d(a.t_first + qlast, a.W, a.NB), kCdCols);

    if (tid == 0) {
        bar.init(kCdRows);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    // extra K step: B = 1 in its first column (bf16 0x3F80)
    for (int i = tid; i < kCdCols * 2; i += kCdThreads) {
        const int n = i >> 1, kh = i & 1;
        *reinterpret_cast<uint4*>(sBx + noswz_off(n, kh)) = make_uint4(kh == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    const int quarter = warp & 3, blk = (warp - 2) >> 2;
    const int r = blk * 128 + quarter * 32 + lane;  // epilogue row of this thread
    float tau = -CUDART_INF_F;
    EpiRow e{};
    if (warp >= 2) {
        fill_a_row<G>(sA, a, q0, h, r);
        e = epi_row<G>(a, q0, h, r);
        tau = e.valid ? a.tau[e.orow] : -CUDART_INF_F;
        // A's extra column: -tau (exact: tau is a bf16 value), 0 when tau = -inf
        const float tau_add = tau == -CUDART_INF_F ? 0.f : tau;
        uint8_t* ax = sAx + blk * kTcAxBytes;
        const int rb = r & 127;
        *reinterpret_cast<uint4*>(ax + noswz_off(rb, 0)) =
            make_uint4((uint32_t)(__float_as_uint(-tau_add) >> 16), 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(ax + noswz_off(rb, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) tc_produce<kCdStages, kCdCols>(&tmF, (int64_t)h * a.cap_buckets, ntiles, sB, bar, abort_flag);
    } else if (warp == 1) {
        if (lane == 0) tc_mma<kCdBlocks, kCdCols, kCdStages, true>(tmem, sA, sB, sAx, sBx, ntiles, bar, abort_flag);
    } else {
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(blk * kCdCols);
        const bool tau_inf = tau == -CUDART_INF_F;
        const float tau_add = tau_inf ? 0.f : tau;
        float* my_stg = stg + r * kTcStgStride;
        int2* cand = a.cand + e.orow * (int64_t)kCandCap;
        int cnt = 0;
        // TMEM holds s - tau_add; candidates (score >= tau) are appended in
        // ascending bucket id (the thread owns its row)
        for (int it = 0; it < ntiles; ++it) {
            const int b = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(bar.tfull(b), (uint32_t)(it >> 1) & 1u, abort_flag))) break;
            tc_fence_after();
            const uint32_t tb = trow + (uint32_t)(b * kCdBlocks * kCdCols);
            uint32_t v[64];
            tmem_ld64(tb, v);
            // the whole tile is in registers: its TMEM buffer goes back to the
            // MMA thread before the scan
            tc_fence_before();
            mbar_arrive(bar.tempty(b));
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t* vv = v + 32 * c;
#pragma unroll
                for (int off = 1; off < G; off <<= 1)   // native: max over the query's head rows
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        vv[i] = __float_as_uint(fmaxf(__uint_as_float(vv[i]), __uint_as_float(__shfl_xor_sync(0xffffffffu, vv[i], off))));
                const int col0 = it * kCdCols + c * 32;
                const int rem = e.ncol - col0;
                const uint32_t lm = !e.owner || rem <= 0 ? 0u : (rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u));
                // sign bits of s - tau (bit i set = miss), four independent chains
                uint32_t sg[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int i = 7; i >= 0; --i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) sg[j] = __funnelshift_l(vv[8 * j + i], sg[j], 1);
                const uint32_t miss = sg[0] | (sg[1] << 8) | (sg[2] << 16) | (sg[3] << 24);
                uint32_t hits = (tau_inf ? 0xffffffffu : ~miss) & lm;
                if (__any_sync(0xffffffffu, hits)) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        reinterpret_cast<uint4*>(my_stg)[j] = make_uint4(vv[4 * j], vv[4 * j + 1], vv[4 * j + 2], vv[4 * j + 3]);
                    while (hits) {
                        const int i = __ffs(hits) - 1;
                        hits &= hits - 1u;
                        if (cnt < kCandCap) cand[cnt] = make_int2(col0 + i, __float_as_int(my_stg[i] + tau_add));
                        ++cnt;
                    }
                }
            }
        }
        if (e.owner) a.cand_n[e.orow] = cnt;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------- resolve

constexpr int kResWarps = 4;
constexpr int kBandCap = 128;  // buckets ranked on exact scores per row

// One record of a shard's local fill (sequence-sharded selection): a bucket
// the shard's own fill of k keys took, its global id, the keys it took and
// its exact fp64 score.
struct ShardRec {
    int32_t bucket;
    int32_t taken;
    double score;
};

struct ResolveArgs {
    const int4* meta;        // [hkv, NB] (minlr, maxpos, cnt_lr, packed member units)
    const uint16_t* cent;
    int64_t cap_buckets, NB, T_built;
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
    // candidate-record mode (rec != NULL): no index rows; per row the taken
    // buckets as records [rows, rec_cap] in ascending id, ids offset by id_base
    ShardRec* rec;
    int32_t* rec_n;
    int32_t rec_cap;
    int64_t id_base;
};

// meta[h * NB + b] = (minlr, maxpos, cnt_lr, units) of bucket b < NB: one 16-byte
// record per bucket for the resolve's gathers.
__global__ void meta_gather_kernel(const int32_t* __restrict__ minlr, const int32_t* __restrict__ maxpos,
                                   const int32_t* __restrict__ cnt_lr, const int32_t* __restrict__ units,
                                   int64_t cap_buckets, int64_t NB, int32_t hkv, int4* __restrict__ meta) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)hkv * NB) return;
    const int64_t hb = (idx / NB) * cap_buckets + idx % NB;
    meta[idx] = make_int4(minlr[hb], maxpos[hb], cnt_lr[hb], units[hb]);
}

struct ResWarp {
    double bex[kBandCap];     // exact scores of the band
    int2 cs[kCandCap];        // eligible candidates (bucket id, fp32 score bits), ascending id
    uint8_t w[kCandCap];      // key weights (<= 16), then taken counts
    int32_t pk[kCandCap];     // packed member units of each candidate (from its record)
    int16_t bidx[kBandCap];   // band members (index into cs)
    uint32_t hist[256];
    uint16_t ylat[8 * kDL];
};

// Keys of bucket b in [S, lim]; `pk` is the bucket's packed member units.
__device__ __noinline__ int weight_packed(int64_t b, int32_t pk, int64_t lim, int32_t S, int64_t T_built) {
    const int64_t ubase = (b / kBucketsPerBlock) * kUnitsPerBlock;
    const int cnt = (pk >> 28) & 7;
    int w = 0;
    for (int i = 0; i < cnt; ++i) {
        const int64_t j = ubase + ((pk >> (7 * i)) & 127);
        for (int64_t p = j * kPool; p < j * kPool + kPool && p < T_built; ++p)
            if (p >= S && p <= lim) ++w;
    }
    return w;
}

// First `tk` keys of bucket b in [S, lim], ascending (member units are
// packed in ascending order), written to out[o ..].  Fast path: a bucket
// taken whole whose units are full and >= S writes 4 consecutive positions
// per unit, as one 16-byte store where out + o is 16-byte aligned.
__device__ __forceinline__ void emit_keys(int64_t b, int32_t pk, int tk, int64_t lim, int32_t S, int64_t T_built,
                                          int32_t* out, int o) {
    const int64_t ubase = (b / kBucketsPerBlock) * kUnitsPerBlock;
    const int cnt = (pk >> 28) & 7;
    const int64_t j0 = ubase + (pk & 127);
    if (tk == cnt * kPool && j0 * kPool >= S) {
        const bool al = ((((uintptr_t)(out + o)) & 15u) == 0u);
        for (int i = 0; i < cnt; ++i) {
            const int32_t p = (int32_t)((ubase + ((pk >> (7 * i)) & 127)) * kPool);
            if (al) {
                reinterpret_cast<int4*>(out + o)[i] = make_int4(p, p + 1, p + 2, p + 3);
            } else {
                out[o + 4 * i] = p; out[o + 4 * i + 1] = p + 1; out[o + 4 * i + 2] = p + 2; out[o + 4 * i + 3] = p + 3;
            }
        }
        return;
    }
    for (int i = 0; i < cnt && tk > 0; ++i) {
        const int64_t j = ubase + ((pk >> (7 * i)) & 127);
        for (int64_t p = j * kPool; p < j * kPool + kPool && p < T_built && tk > 0; ++p)
            if (p >= S && p <= lim) { out[o++] = (int32_t)p; --tk; }
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

// exact_row against an FP8 centroid (64 e4m3 codes of 2^8 c): products of a
// bf16 and a 2^-8 e4m3 value are exact in fp64, ascending dimension order.
__device__ __forceinline__ double exact_row8(const uint16_t* ylat, int ng, const uint8_t* c8) {
    uint4 cv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cv[i] = __ldg(reinterpret_cast<const uint4*>(c8) + i);
    double best = -CUDART_INF;
    for (int g = 0; g < ng; ++g) {
        const uint16_t* y = ylat + g * kDL;
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t wv[4] = {cv[i].x, cv[i].y, cv[i].z, cv[i].w};
#pragma unroll
            for (int e = 0; e < 16; ++e)
                s = fma(bf16_to_f64(y[16 * i + e]), e4m3_to_f64((wv[e >> 2] >> (8 * (e & 3))) & 0xFFu) * 0x1p-8, s);
        }
        best = s > best ? s : best;
    }
    return best;
}

// exact_row for four centroids at once: four independent fma chains (each
// in ascending dimension order, so every score equals exact_row's).
__device__ __forceinline__ void exact_rows4(const uint16_t* ylat, int ng, const uint16_t* const (&c)[4],
                                            double (&out)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) out[j] = -CUDART_INF;
    for (int g = 0; g < ng; ++g) {
        const uint16_t* y = ylat + g * kDL;
        double s[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 2
        for (int i = 0; i < 8; ++i) {
            uint4 cv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) cv[j] = __ldg(reinterpret_cast<const uint4*>(c[j]) + i);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const double y0 = bf16_to_f64(y[8 * i + 2 * e]), y1 = bf16_to_f64(y[8 * i + 2 * e + 1]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t w = e == 0 ? cv[j].x : e == 1 ? cv[j].y : e == 2 ? cv[j].z : cv[j].w;
                    s[j] = fma(y0, (double)__uint_as_float(w << 16), s[j]);
                    s[j] = fma(y1, (double)__uint_as_float(w & 0xFFFF0000u), s[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) out[j] = s[j] > out[j] ? s[j] : out[j];
    }
}

__device__ __forceinline__ void push_fallback(const ResolveArgs& a, int64_t row) {
    atomicAdd(&g_lsa_fallback_rows, 1ull);
    const int slot = atomicAdd(a.ovf_count, 1);
    if (slot < a.ovf_cap) a.ovf_rows[slot] = (int32_t)row;
    else raise_device_error(kErrSelectOverflow);
}

// Weighted cut over 256 bins (descending): the bin where the weight from the
// top first reaches `need`; *above = the weight of the bins above it.
// -1 if the bins hold less than `need`.
__device__ __forceinline__ int cut_bin(const uint32_t* hist, long long need, long long* above) {
    const int lane = threadIdx.x & 31;
    long long s8 = 0;
#pragma unroll
    for (int d = 0; d < 8; ++d) s8 += hist[255 - 8 * lane - d];
    long long incl = s8;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const long long excl = incl - s8;
    const unsigned hitm = __ballot_sync(0xffffffffu, incl >= need && excl < need);
    if (hitm == 0u) return -1;
    const int src = __ffs(hitm) - 1;
    int dig = 0;
    long long cum = 0;
    if (lane == src) {
        cum = excl;
        dig = 255 - 8 * lane;
        for (int d = 0; d < 8; ++d) {
            const int dd = 255 - 8 * lane - d;
            if (cum + hist[dd] >= need) { dig = dd; break; }
            cum += hist[dd];
        }
    }
    *above = __shfl_sync(0xffffffffu, cum, src);
    return __shfl_sync(0xffffffffu, dig, src);
}

__device__ __forceinline__ float warp_minf(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}
__device__ __forceinline__ float warp_maxf(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// CANDS: write the row's taken buckets as records (ascending id, exact
// scores) instead of its index row.
template <bool CANDS>
__global__ void __launch_bounds__(32 * kResWarps, 3) flat_resolve_kernel(ResolveArgs a) {
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

    if constexpr (!CANDS) {
        // sinks and window (16-byte stores when the row layout keeps them aligned)
        for (int i = lane; i < a.S; i += 32) out[i] = (i <= t) ? i : -1;
        const int64_t w0 = max((int64_t)a.S, t - a.W + 1);
        const int nw = t >= a.S ? (int)(t - w0 + 1) : 0;
        int32_t* wout = out + a.S + a.k;
        if ((((uintptr_t)wout) & 15u) == 0u && (a.W & 3) == 0) {
            for (int i4 = lane; i4 < a.W / 4; i4 += 32) {
                const int i = 4 * i4;
                reinterpret_cast<int4*>(wout)[i4] =
                    make_int4(i < nw ? (int)w0 + i : -1, i + 1 < nw ? (int)w0 + i + 1 : -1,
                              i + 2 < nw ? (int)w0 + i + 2 : -1, i + 3 < nw ? (int)w0 + i + 3 : -1);
            }
        } else {
            for (int i = lane; i < a.W; i += 32) wout[i] = i < nw ? (int32_t)(w0 + i) : -1;
        }
    }
    if (lim < a.S) {
        if constexpr (CANDS) {
            if (lane == 0) a.rec_n[row] = 0;
        } else {
            for (int i = lane; i < a.k; i += 32) out[a.S + i] = -1;
        }
        return;
    }
    const int n = a.cand_n[row];
    if (n > kCandCap) {
        if (lane == 0) push_fallback(a, row);
        return;
    }
    const float tau = a.tau[row];

    // eligible candidates (kept in ascending bucket id), their key counts
    // and score range
    const int64_t hb0 = (int64_t)h * a.cap_buckets;
    const int4* mrow = a.meta + (int64_t)h * a.NB;
    const int2* crow = a.cand + row * kCandCap;
    // (1) the candidate list into shared memory, (2) every candidate's
    // record gathered with the loads of a lane in flight together, its key
    // count (0: not eligible) kept, (3) in-place compaction of the eligible
    // ones (a chunk's reads precede its writes, which land at or below it)
#pragma unroll 4
    for (int i = lane; i < n; i += 32) sw.cs[i] = crow[i];
    __syncwarp();
    // the records of 8 candidates per lane are requested before any is used
    for (int i0 = lane; i0 < n; i0 += 32 * 8) {
        int4 md[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u;
            md[u] = i < n ? __ldg(mrow + sw.cs[i].x) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u;
            if (i < n) {
                int wgt = 0;
                if ((int64_t)md[u].x <= lim)
                    wgt = (int64_t)md[u].y <= lim ? md[u].z : weight_packed(sw.cs[i].x, md[u].w, lim, a.S, a.T_built);
                sw.w[i] = (uint8_t)wgt;
                sw.pk[i] = md[u].w;
            }
        }
    }
    __syncwarp();
    int m = 0;
    long long wtot = 0;
    float smin = CUDART_INF_F, smax = -CUDART_INF_F;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const int2 cv = i < n ? sw.cs[i] : make_int2(0, 0);
        const int wgt = i < n ? sw.w[i] : 0;
        const int32_t pkv = i < n ? sw.pk[i] : 0;
        const bool el = wgt > 0;
        if (el) {
            wtot += wgt;
            smin = fminf(smin, __int_as_float(cv.y));
            smax = fmaxf(smax, __int_as_float(cv.y));
        }
        const unsigned bal = __ballot_sync(0xffffffffu, el);
        __syncwarp();
        if (el) {
            const int pos = m + __popc(bal & ((1u << lane) - 1u));
            sw.cs[pos] = cv;
            sw.w[pos] = (uint8_t)wgt;
            sw.pk[pos] = pkv;
        }
        m += __popc(bal);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wtot += __shfl_xor_sync(0xffffffffu, wtot, off);
    smin = warp_minf(smin);
    smax = warp_maxf(smax);
    __syncwarp();

    if (wtot > a.k) {
        // the fp32 score of the k-th key lies in [lo_s, hi_s], the score
        // range of the members of the cut bin: two passes of 256 linear bins
        // over [smin, smax] (the second inside the first pass's cut bin)
        const float inv = smax > smin ? 256.f / (smax - smin) : 0.f;
        auto bin1 = [&](float s) { return min(255, (int)((s - smin) * inv)); };
        for (int i = lane; i < 256; i += 32) sw.hist[i] = 0u;
        __syncwarp();
        for (int i = lane; i < m; i += 32) atomicAdd(&sw.hist[bin1(__int_as_float(sw.cs[i].y))], (unsigned)sw.w[i]);
        __syncwarp();
        long long above = 0;
        const int b1 = cut_bin(sw.hist, a.k, &above);
        __syncwarp();
        auto bin2 = [&](float s) { return min(255, max(0, (int)(((s - smin) * inv - (float)b1) * 256.f))); };
        for (int i = lane; i < 256; i += 32) sw.hist[i] = 0u;
        __syncwarp();
        for (int i = lane; i < m; i += 32) {
            const float s = __int_as_float(sw.cs[i].y);
            if (bin1(s) == b1) atomicAdd(&sw.hist[bin2(s)], (unsigned)sw.w[i]);
        }
        __syncwarp();
        long long above2 = 0;
        const int b2 = cut_bin(sw.hist, a.k - above, &above2);
        if (b1 < 0 || b2 < 0) {  // cannot happen while the weights above reach k
            if (lane == 0) push_fallback(a, row);
            return;
        }
        float lo_s = CUDART_INF_F, hi_s = -CUDART_INF_F;
        for (int i = lane; i < m; i += 32) {
            const float s = __int_as_float(sw.cs[i].y);
            if (bin1(s) == b1 && bin2(s) == b2) { lo_s = fminf(lo_s, s); hi_s = fmaxf(hi_s, s); }
        }
        lo_s = warp_minf(lo_s);
        hi_s = warp_maxf(hi_s);
        const float hi = hi_s + 2.f * kScoreErr, lo = lo_s - 2.f * kScoreErr;
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
            const float sc = i < m ? __int_as_float(sw.cs[i].y) : -CUDART_INF_F;
            const bool band = i < m && sc >= lo && sc <= hi;
            if (i < m && sc > hi) win += sw.w[i];
            const unsigned bal = __ballot_sync(0xffffffffu, band);
            if (band) {
                const int pos = nb + __popc(bal & ((1u << lane) - 1u));
                if (pos < kBandCap) sw.bidx[pos] = (int16_t)i;
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
            sw.bex[i] = exact_row(sw.ylat, ng, a.cent + (hb0 + sw.cs[sw.bidx[i]].x) * kDL);
        __syncwarp();
        // taken counts: in -> whole, out -> 0, band -> pending (marked 0x80 | w)
        for (int i = lane; i < m; i += 32) {
            const float sc = __int_as_float(sw.cs[i].y);
            sw.w[i] = sc > hi ? sw.w[i] : (sc >= lo ? (uint8_t)(0x80u | sw.w[i]) : (uint8_t)0);
        }
        __syncwarp();
        // the greedy fill of the band (best exact score first, lower bucket id
        // on ties) in closed form: a band bucket takes what is left of the
        // need after the weight of every band bucket ranked above it
        const long long need = a.k - win;
        int tk_reg[kBandCap / 32];
#pragma unroll
        for (int u = 0; u < kBandCap / 32; ++u) {
            const int i = lane + 32 * u;
            tk_reg[u] = 0;
            if (i < nb) {
                const int ci = sw.bidx[i];
                const double ei = sw.bex[i];
                const int coli = sw.cs[ci].x;
                long long above = 0;
                for (int j = 0; j < nb; ++j) {
                    const double ej = sw.bex[j];
                    const int cj = sw.bidx[j];
                    if (ej > ei || (ej == ei && sw.cs[cj].x < coli)) above += sw.w[cj] & 0x7F;
                }
                const long long left = need - above;
                const int wv = sw.w[ci] & 0x7F;
                tk_reg[u] = left <= 0 ? 0 : (left < wv ? (int)left : wv);
            }
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kBandCap / 32; ++u) {
            const int i = lane + 32 * u;
            if (i < nb) sw.w[sw.bidx[i]] = (uint8_t)tk_reg[u];
        }
        __syncwarp();
        for (int i = lane; i < m; i += 32)
            if (sw.w[i] & 0x80u) sw.w[i] = 0;
        __syncwarp();
    } else if (tau > -CUDART_INF_F) {
        // fewer than k keys among the candidates, but buckets below tau exist
        if (lane == 0) push_fallback(a, row);
        return;
    }
    if constexpr (CANDS) {
        // records of the taken buckets, ascending id, with their exact scores
        const int ng = a.agg ? a.G : 1;
        const uint16_t* ysrc = a.agg ? a.Y + (q * (int64_t)a.hkv * a.G + (int64_t)h * a.G) * kDL
                                     : a.Y + row * kDL;
        __syncwarp();
        for (int i = lane; i < ng * kDL; i += 32) sw.ylat[i] = ysrc[i];
        __syncwarp();
        ShardRec* rec = a.rec + row * (int64_t)a.rec_cap;
        int nrec = 0;
        for (int base = 0; base < m; base += 32) {
            const int i = base + lane;
            const int tk = i < m ? sw.w[i] : 0;
            const unsigned bal = __ballot_sync(0xffffffffu, tk > 0);
            const int pos = nrec + __popc(bal & ((1u << lane) - 1u));
            if (tk > 0 && pos < a.rec_cap) {
                const int col = sw.cs[i].x;
                rec[pos] = ShardRec{(int32_t)(a.id_base + col), tk,
                                    exact_row(sw.ylat, ng, a.cent + (hb0 + col) * kDL)};
            }
            nrec += __popc(bal);
        }
        if (lane == 0) {
            a.rec_n[row] = min(nrec, a.rec_cap);
            if (nrec > a.rec_cap) raise_device_error(kErrSelectOverflow);
        }
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
        if (tk > 0) {
            const int col = sw.cs[i].x;
            emit_keys(col, sw.pk[i], tk, lim, a.S, a.T_built, out, a.S + run + incl - tk);
        }
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

// Packed bucket records for the resolve, once per call.
lsa_status launch_meta_gather(const lsa_cache* c, int64_t NB, int4* meta, cudaStream_t st) {
    const int64_t n = (int64_t)c->hkv * NB;
    if (n == 0) return LSA_OK;
    meta_gather_kernel<<<(unsigned)ceil_div<int64_t>(n, 256), 256, 0, st>>>(c->minlr, c->maxpos, c->cnt_lr, c->units,
                                                                            c->cap_buckets, NB, c->hkv, meta);
    return check_launch("meta_gather_kernel");
}

// tmF: centroids [hkv * cap_buckets, 64] in 64-row boxes; tmS: sampled
// centroids [hkv * ns_cap, 64] in 128-row boxes.
lsa_status launch_flat(const PassArgs& pa, const ResolveArgs& ra, const CUtensorMap& tmF, const CUtensorMap& tmS,
                       cudaStream_t st) {
    const int G = pa.agg ? pa.G : 1;
    auto ks = G == 1 ? flat_sample_kernel<1> : G == 2 ? flat_sample_kernel<2> : G == 4 ? flat_sample_kernel<4>
                                                                                          : flat_sample_kernel<8>;
    auto kc = G == 1 ? flat_cand_kernel<1> : G == 2 ? flat_cand_kernel<2> : G == 4 ? flat_cand_kernel<4>
                                                                                    : flat_cand_kernel<8>;
    cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmSmemBytes);
    cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCdSmemBytes);
    {
        KTime kt_("flat_sample_kernel", st);
        ks<<<dim3((unsigned)ceil_div<int64_t>(pa.nqc, kSmRows / G), (unsigned)pa.hkv), kSmThreads, kSmSmemBytes, st>>>(tmS,
                                                                                                                   pa);
    }
    lsa_status s = check_launch("flat_sample_kernel");
    if (s != LSA_OK) return s;
    {
        KTime kt_("flat_cand_kernel", st);
        kc<<<dim3((unsigned)ceil_div<int64_t>(pa.nqc, kCdRows / G), (unsigned)pa.hkv), kCdThreads, kCdSmemBytes, st>>>(tmF,
                                                                                                                   pa);
    }
    if ((s = check_launch("flat_cand_kernel")) != LSA_OK) return s;
    const size_t smem_r = sizeof(ResWarp) * kResWarps;
    auto kr = ra.rec ? flat_resolve_kernel<true> : flat_resolve_kernel<false>;
    cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_r);
    const int64_t rows = pa.nqc * pa.hkv;
    {
        KTime kt_("flat_resolve_kernel", st);
        kr<<<(unsigned)ceil_div<int64_t>(rows, kResWarps), 32 * kResWarps, smem_r, st>>>(ra);
    }
    return check_launch("flat_resolve_kernel");
}

}  // namespace lsa
