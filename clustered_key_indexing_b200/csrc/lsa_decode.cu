// lsa_decode.cu -- batched decode of the LSA path on sm_100a.
//
// One new token per request per step [essay "《卡片柜》——当注意力学会先查目录
// 再翻书", ch. 2: clustering is done once per completed 512-key block while
// streaming and never redone; ch. 3/4: the query then searches the bucket
// cache flat or down the tree; tutorial "隐空间稀疏注意力 (LSA)", section 二:
// exact attention over the selected keys].
//
// The cache of a decode batch is one lsa_cache whose heads are
// (request, kv-head) pairs: head r*hkv + h.  Per step:
//   decode_append_kernel   K/V rows of the new token; its key latent (fp64)
//                          added to the pooled unit being filled (block ring
//                          U_blk), divided by 4 when the unit completes;
//   ward_kernel (jobs)     every request whose token completed a block
//                          clusters it; the tree is updated above its slots;
//   query latents, then flat (decode_score_kernel + decode_resolve_kernel)
//                          or tree (tree_warp_kernel) selection;
//   attn_kernel<8>         eight warps share each (request, kv-head) row.
// Flat scores: one HBM pass over the request's eligible centroids (TMA into a
// shared-memory ring, mma.sync bf16 scores with fp32 accumulation) storing
// each slot's score bin (2048 bins of width >= 2e over the row's score range)
// and key weight; then one CTA per row: weighted histogram of the bins, the
// two bins around the k-th key kept (warp-ordered compaction), exact fp64
// rescoring, weighted radix select, key emission in bucket-id order.  Rows
// whose kept bins overflow shared memory take exact fp64 scores of every
// eligible bucket in a global slot.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"
#include "lsa_common.cuh"
#include "lsa_mma.cuh"
#include "lsa_tc.cuh"

namespace lsa {

lsa_status launch_key_latent(const uint16_t* K, int64_t T, int32_t hkv, const float* W, int64_t unit0,
                             int64_t unit1, int64_t cap_units, double* U, cudaStream_t st);
lsa_status launch_query_latent(const uint16_t* Q, int64_t nq, int32_t hq, int32_t hkv, const float* W,
                               int agg, uint16_t* Y, cudaStream_t st);
lsa_status launch_ward_u(const lsa_cache* c, const double* U, int64_t U_stride, int64_t T, int32_t sinks,
                         int64_t blk0, int64_t blk1, cudaStream_t st);
lsa_status launch_ward_jobs(const lsa_cache* c, const double* U_blk, int32_t hkv, int32_t sinks, int n_jobs,
                            const int32_t* head0, const int64_t* blk, cudaStream_t st);
lsa_status launch_clear_slots(const lsa_cache* c, int64_t b0, int64_t b1, cudaStream_t st);
lsa_status launch_tree_update(const lsa_cache* c, lsa_tree* t, int64_t b0, int64_t b1, cudaStream_t st);
lsa_status launch_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                       int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t T, uint16_t* O,
                       cudaStream_t st, int64_t kv_q_stride, int split, int32_t n_use, const float* Ow,
                       const float* lse, const uint16_t* Ks, const uint16_t* Vs, int64_t shared_len);

// ------------------------------------------------------------- key latent

// z = normalise(k W) for one 128-value bf16 row held in shared memory as
// doubles; lane computes dims c = lane, lane + 32; |v|^2 summed in ascending
// dim order.  Returns z for the lane's two dims.
__device__ __forceinline__ void latent_row(const double* krow, const float* __restrict__ W,
                                           int lane, double& z0, double& z1) {
    double v0 = 0.0, v1 = 0.0;
    for (int e = 0; e < kD; ++e) {
        const double k = krow[e];
        v0 = fma(k, (double)__ldg(W + e * kDL + lane), v0);
        v1 = fma(k, (double)__ldg(W + e * kDL + lane + 32), v1);
    }
    double n2 = 0.0;
    for (int c = 0; c < kDL; ++c) {
        const double v = __shfl_sync(0xffffffffu, c < 32 ? v0 : v1, c & 31);
        n2 = __dadd_rn(n2, __dmul_rn(v, v));
    }
    const double nrm = sqrt(n2);
    z0 = nrm > 0.0 ? __ddiv_rn(v0, nrm) : 0.0;
    z1 = nrm > 0.0 ? __ddiv_rn(v1, nrm) : 0.0;
}

constexpr int kDecBins = 2048;       // histogram bins over the row's score range

struct AppendArgs {
    const uint16_t* k;   // [batch, hkv, 128] new keys
    const uint16_t* v;   // [batch, hkv, 128] new values
    uint16_t* K;         // [batch, tail, hkv, 128] (tail = cap - shared_len)
    uint16_t* V;
    const float* W;      // W_k [128, 64]
    double* U_blk;       // [batch * hkv, 128, 64]
    int64_t tail, shared_len;
    int32_t hkv, batch;
    uint32_t* hist;      // flat search: [batch * hkv, kDecBins] zeroed here for this step's scores ...
    unsigned long long* tot;  // ... and [batch * hkv] row totals
    int64_t pos[LSA_MAX_BATCH];
};

// One warp per (request, kv-head).
__global__ void __launch_bounds__(256) decode_append_kernel(AppendArgs a) {
    __shared__ double krow[8][kD];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t w = (int64_t)blockIdx.x * 8 + wid;
    if (w >= (int64_t)a.batch * a.hkv) return;
    const int64_t r = w / a.hkv, h = w % a.hkv;
    const int64_t t = a.pos[r];
    if (a.hist) {
        for (int i = lane; i < kDecBins; i += 32) a.hist[w * kDecBins + i] = 0u;
        if (lane == 0) a.tot[w] = 0ull;
    }
    const uint16_t* ks = a.k + w * kD;
    const uint16_t* vs = a.v + w * kD;
    const int64_t dst = ((r * a.tail + (t - a.shared_len)) * a.hkv + h) * kD;
    if (lane < 16) {
        reinterpret_cast<uint4*>(a.K + dst)[lane] = reinterpret_cast<const uint4*>(ks)[lane];
        reinterpret_cast<uint4*>(a.V + dst)[lane] = reinterpret_cast<const uint4*>(vs)[lane];
    }
    for (int e = lane; e < kD; e += 32) krow[wid][e] = bf16_to_f64(ks[e]);
    __syncwarp();
    double z0, z1;
    latent_row(krow[wid], a.W, lane, z0, z1);
    double* u = a.U_blk + (w * kUnitsPerBlock + (t / kPool) % kUnitsPerBlock) * kDL;
    const int i = (int)(t % kPool);
    double s0 = (i == 0) ? __dadd_rn(0.0, z0) : __dadd_rn(u[lane], z0);
    double s1 = (i == 0) ? __dadd_rn(0.0, z1) : __dadd_rn(u[lane + 32], z1);
    if (i == kPool - 1) {
        s0 = __ddiv_rn(s0, (double)kPool);
        s1 = __ddiv_rn(s1, (double)kPool);
    }
    u[lane] = s0;
    u[lane + 32] = s1;
}

// Tail of a loaded prompt: pooled units [j0, j1) of one request into its
// block ring (complete units divided by 4, the last partial unit left as the
// running sum the next appends continue).  One warp per (head, unit).
__global__ void __launch_bounds__(256) tail_units_kernel(const uint16_t* __restrict__ K,
                                                         const float* __restrict__ W, double* U_blk,
                                                         int64_t n, int64_t j0, int64_t j1, int32_t hkv,
                                                         int64_t head0, int64_t row0) {
    __shared__ double krow[8][kD];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t w = (int64_t)blockIdx.x * 8 + wid;
    if (w >= (j1 - j0) * hkv) return;
    const int64_t j = j0 + w / hkv, h = w % hkv;
    double s0 = 0.0, s1 = 0.0;
    int cnt = 0;
    for (int64_t t = j * kPool; t < j * kPool + kPool && t < n; ++t) {
        const uint16_t* ks = K + ((t - row0) * hkv + h) * kD;   // K holds positions row0 ..
        __syncwarp();
        for (int e = lane; e < kD; e += 32) krow[wid][e] = bf16_to_f64(ks[e]);
        __syncwarp();
        double z0, z1;
        latent_row(krow[wid], W, lane, z0, z1);
        s0 = __dadd_rn(s0, z0);
        s1 = __dadd_rn(s1, z1);
        ++cnt;
    }
    if (cnt == kPool) {
        s0 = __ddiv_rn(s0, (double)kPool);
        s1 = __ddiv_rn(s1, (double)kPool);
    }
    double* u = U_blk + ((head0 + h) * kUnitsPerBlock + j % kUnitsPerBlock) * kDL;
    u[lane] = s0;
    u[lane + 32] = s1;
}

// ------------------------------------------------------ flat decode scores


struct DecScoreArgs {
    const uint16_t* Y;        // [batch, hkv, 64] (mean) / [batch, hq, 64] (native)
    const uint16_t* cent;     // [heads, cap_buckets, 64]
    const int32_t* minlr;
    const int32_t* maxpos;
    const int32_t* cnt_lr;
    const int32_t* units;
    int64_t cap_buckets, ld;
    int32_t hkv, G, agg, S, W, k;
    int64_t T_built;
    uint16_t* bin;            // [rows, ld] score bin of every slot
    uint8_t* wt;              // [rows, ld] keys of the slot in [S, t-W] (0 = not eligible)
    uint32_t* hist;           // [rows, kDecBins] key weight per bin (zeroed by the append kernel)
    unsigned long long* tot;  // [rows] key weight of the row (zeroed by the append kernel)
    int64_t pos[LSA_MAX_BATCH];
};

__device__ __forceinline__ int weight_units(int64_t b, int32_t pk, int64_t lim, int32_t S, int64_t T_built) {
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

// Score range of a row: |score| <= |y| (native: max over its heads); the
// floor 0.25 keeps every one of the 2048 bins at least 2e = 2e-4 wide.
__device__ __forceinline__ float row_radius(const uint16_t* y, int ng) {
    float R = 0.f;
    for (int g = 0; g < ng; ++g) {
        float n2 = 0.f;
        for (int i = 0; i < kDL; ++i) { const float v = bf16_to_f32(y[g * kDL + i]); n2 += v * v; }
        R = fmaxf(R, sqrtf(n2));
    }
    return fmaxf(0.25f, fminf(1.0625f, R * 1.01f + 1e-6f));
}

__device__ __forceinline__ int score_to_bin(float s, float R) {
    int bin = __float2int_rd((s + R) * ((float)kDecBins / (2.f * R)));
    return bin < 0 ? 0 : (bin >= kDecBins ? kDecBins - 1 : bin);
}

// Cut of a key-weight histogram h (kDecBins bins in shared memory, bin
// kDecBins - 1 the highest scores), computed by all 128 threads of a block
// (each sums 16 bins, then a block scan): returns j - 1 (not below 0) for the
// highest bin j whose weight counted from the top reaches k, and in *tot the
// histogram's total weight.  Every slot in bins >= j - 1 is kept for exact
// rescoring: the k-th key's exact score lies in bin j or j - 1 (bins are at
// least 2e wide).  Contains __syncthreads: every thread of the block calls it.
__device__ int dec_cut_block(const uint32_t* h, int64_t k, long long* tot) {
    __shared__ long long wsum[4];
    __shared__ int s_j;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int top = kDecBins - 1 - 16 * tid;  // this thread's bins: top, top - 1, .., top - 15
    long long s = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) s += (long long)h[top - i];
    long long incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[wid] = incl;
    if (tid == 0) s_j = 1;  // no bin reaches k: cut 0
    __syncthreads();
    for (int i = 0; i < wid; ++i) incl += wsum[i];
    const long long all = wsum[0] + wsum[1] + wsum[2] + wsum[3];
    const long long excl = incl - s;
    if (excl < k && incl >= k) {
        long long cum = excl;
        int j = top;
        for (int i = 0; i < 16; ++i) {
            cum += (long long)h[top - i];
            if (cum >= k) { j = top - i; break; }
        }
        s_j = j;
    }
    __syncthreads();
    const int j = s_j;
    __syncthreads();  // s_j and wsum are reused by the next call
    *tot = all;
    return j > 0 ? j - 1 : 0;
}

// grid (column chunks, rows), 4 warps.  The chunk's centroids stream through
// a 3-stage shared-memory ring of 256-row tiles (TMA, 128-byte swizzle, one
// thread issues; bounded mbarrier waits, no multicast).  Each warp scores 64
// centroids of a tile with mma.sync m16n8k16 (centroids as M, the row's NG
// query latents as N, fp32 accumulate), the lane pairs' scores are reduced
// to the max over latents, binned, and the tile's bins and weights are
// written with coalesced stores (weights from cnt_lr, and below the frontier
// block no minlr / maxpos reads: those buckets lie wholly in [S, t - W]).
constexpr int kDecScanCols = 16384;   // bucket slots per CTA
constexpr int kDecTile = 256;        // centroids per ring stage (32 KB)
constexpr int kDecStages = 3;
constexpr size_t kDecScanSmem = 1024 + (size_t)kDecStages * kDecTile * kDL * 2 + kDecTile * 4 + 64;

template <int NG>
__global__ void __launch_bounds__(128) decode_score_kernel(const __grid_constant__ CUtensorMap tmC, DecScoreArgs a) {
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* ring = dsm;
    float* best_s = reinterpret_cast<float*>(ring + kDecStages * kDecTile * kDL * 2);  // [kDecTile]
    uint64_t* bars = reinterpret_cast<uint64_t*>(best_s + kDecTile);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kDecStages);
    __shared__ float rad;
    __shared__ uint32_t shist[kDecBins];  // key weight per score bin over this CTA's slots
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.y;
    const int64_t r = row / a.hkv;
    const int64_t t = a.pos[r];
    const int64_t lim = t - a.W;
    const int64_t ncol = lim < 0 ? 0 : min(a.cap_buckets, (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1));
    const int64_t c0 = (int64_t)blockIdx.x * kDecScanCols;
    if (c0 >= ncol) return;
    const int64_t cend = min(ncol, c0 + kDecScanCols);
    const int ntiles = (int)((cend - c0 + kDecTile - 1) / kDecTile);
    const uint32_t bar0 = smem_u32(bars);
    for (int i = tid; i < kDecBins; i += 128) shist[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) mbar_init(bar0 + 8u * s, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    const uint16_t* yb = a.Y + (row * NG) * kDL;  // native: row*G = r*hq + h*G
    if (tid == 0) rad = row_radius(yb, NG);
    // B operand: Y^T (k = dims, n = latent rows, zero past NG)
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t yq[4][2];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        yq[kk][0] = gq < NG ? *reinterpret_cast<const uint32_t*>(yb + gq * kDL + kk * 16 + 2 * tq) : 0u;
        yq[kk][1] = gq < NG ? *reinterpret_cast<const uint32_t*>(yb + gq * kDL + kk * 16 + 8 + 2 * tq) : 0u;
    }
    __syncthreads();
    const int64_t rowbase = row * a.cap_buckets;
    if (tid == 0) {
        for (int i = 0; i < kDecStages && i < ntiles; ++i) {
            mbar_expect_tx(bar0 + 8u * i, kDecTile * kDL * 2);
            tma_load_2d(smem_u32(ring + i * kDecTile * kDL * 2), &tmC, 0, (int32_t)(rowbase + c0 + i * kDecTile),
                        bar0 + 8u * i);
        }
    }
    const float R = rad;
    const int64_t hb0 = rowbase;
    const int64_t frontier = ncol - kBucketsPerBlock;  // first bucket of the last block in range
    int done = 0;  // tiles consumed
    for (int it = 0; it < ntiles; ++it) {
        const int s = it % kDecStages;
        // this tile's key counts, requested before the scores so that their
        // latency overlaps the MMAs (two slots per thread)
        const int64_t tb0 = c0 + (int64_t)it * kDecTile;
        int32_t clr_pre[kDecTile / 128];
#pragma unroll
        for (int u = 0; u < kDecTile / 128; ++u) {
            const int64_t b = tb0 + tid + 128 * u;
            clr_pre[u] = b < cend ? __ldg(a.cnt_lr + hb0 + b) : 0;
        }
        const bool ok = mbar_wait(bar0 + 8u * s, (uint32_t)(it / kDecStages) & 1u, abort_flag);
        if (!__syncthreads_and(ok)) break;
        const uint32_t tb = smem_u32(ring + s * kDecTile * kDL * 2);
        // warp w: centroids 64 w .. 64 w + 63 of the tile, four m16 tiles
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const int m0 = 64 * warp + 16 * mt;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t af[4];
                const int rr = m0 + (lane & 15);
                const int ch = 2 * kk + (lane >> 4);
                ldsm_x4(af, tb + (uint32_t)(rr * 128 + ((ch ^ (rr & 7)) << 4)));
                mma_16816(acc, af, yq[kk][0], yq[kk][1]);
            }
            // acc: (centroid gq, latents 2tq, 2tq+1), (centroid gq + 8, same)
            float b0 = NG > 1 ? fmaxf(acc[0], acc[1]) : acc[0];
            float b1 = NG > 1 ? fmaxf(acc[2], acc[3]) : acc[2];
            if (NG > 2) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, 1));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, 1));
            }
            if (NG > 4) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, 2));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, 2));
            }
            if (tq == 0) {
                best_s[m0 + gq] = b0;
                best_s[m0 + gq + 8] = b1;
            }
        }
        __syncthreads();
        // the stage is free: the next tile of the chunk into it
        if (tid == 0 && it + kDecStages < ntiles) {
            fence_proxy_async_smem();
            mbar_expect_tx(bar0 + 8u * s, kDecTile * kDL * 2);
            tma_load_2d(smem_u32(ring + s * kDecTile * kDL * 2), &tmC, 0,
                        (int32_t)(rowbase + c0 + (it + kDecStages) * kDecTile), bar0 + 8u * s);
        }
        // bins and weights of the tile, coalesced
#pragma unroll
        for (int u = 0; u < kDecTile / 128; ++u) {
            const int j = tid + 128 * u;
            const int64_t b = tb0 + j;
            if (b >= cend) break;
            const int32_t clr = clr_pre[u];
            int w = clr;
            if (b >= frontier) {
                const int32_t mlr = __ldg(a.minlr + hb0 + b), mxp = __ldg(a.maxpos + hb0 + b);
                w = 0;
                if ((int64_t)mlr <= lim)
                    w = (int64_t)mxp <= lim ? clr : weight_units(b, __ldg(a.units + hb0 + b), lim, a.S, a.T_built);
            }
            const int bn = score_to_bin(best_s[j], R);
            a.bin[row * a.ld + b] = (uint16_t)bn;
            a.wt[row * a.ld + b] = (uint8_t)w;
            if (w > 0) atomicAdd(&shist[bn], (uint32_t)w);
        }
        __syncthreads();  // best_s is rewritten by the next tile
        done = it + 1;
    }
    // after an abort, let the copies already issued land before the CTA exits
    if (tid == 0 && *abort_flag) {
        const int issued = min(ntiles, done + kDecStages);
        for (int i = done; i < issued; ++i)
            mbar_wait(bar0 + 8u * (i % kDecStages), (uint32_t)(i / kDecStages) & 1u, abort_flag, false);
    }
    // The CTA's bin weights into the row's histogram, from its own cut bin
    // down by one: the row's cut bin j (where the weight from the top reaches
    // k) is at or above every CTA's, so the row histogram is exact on every
    // bin >= j - 1, the only bins the cut and the kept slots read.  The
    // total weight goes into the row total.
    __syncthreads();
    long long tc;
    const int jc = dec_cut_block(shist, a.k, &tc);
    if (tid == 0 && tc) atomicAdd(a.tot + row, (unsigned long long)tc);
    for (int i = jc + tid; i < kDecBins; i += 128)
        if (shist[i]) atomicAdd(a.hist + row * kDecBins + i, shist[i]);
}

// The same scan over FP8 centroids (lsa_cache.cent8: e4m3 codes of 2^8 c,
// 64 bytes per bucket).  TMA brings 256-row tiles of the codes (16 KB, no
// swizzle) through a 6-stage ring; each lane converts its rows' codes to
// fp16 pairs (exact) and scores them with fp16 mma.sync against the row's
// query latents (bf16 -> fp16: exact for components >= 2^-14, the smaller
// ones move a score by under 2^-21) with fp32 accumulation.  The MMA's K
// order is a permutation of the 64 dims, the same on both operands: lane
// (g, t) takes dims 16 t .. 16 t + 15 of its two centroid rows with one
// 16-byte load each (rows 64 bytes apart: a quarter-warp reads 128
// contiguous bytes), k-step kk of the MMA covering dims 16 t + 4 kk .. + 3.
// Scores come out times 2^8 and are scaled back exactly.  Their error stays
// below 1e-5 < e, and |score| <= 1.07 |y| (an e4m3 component is within
// 2^-4 of its value relative, so |c8| <= 1.0625 + 2^-17): the row radius
// grows by that factor and the binning, keep and exact fp64 rescoring
// (against the same FP8 values) are unchanged.
constexpr int kDec8Stages = 6;
constexpr size_t kDec8ScanSmem = 1024 + (size_t)kDec8Stages * kDecTile * kDL + kDecTile * 4 + 64;

__device__ __forceinline__ float row_radius8(const uint16_t* y, int ng) {
    float R = 0.f;
    for (int g = 0; g < ng; ++g) {
        float n2 = 0.f;
        for (int i = 0; i < kDL; ++i) { const float v = bf16_to_f32(y[g * kDL + i]); n2 += v * v; }
        R = fmaxf(R, sqrtf(n2));
    }
    return fmaxf(0.25f, fminf(1.14f, R * 1.07f + 1e-6f));
}

__device__ __forceinline__ uint32_t bf16_pair_to_f16x2(uint16_t lo, uint16_t hi) {
    const __half2 h = __floats2half2_rn(bf16_to_f32(lo), bf16_to_f32(hi));
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <int NG>
__global__ void __launch_bounds__(128) decode_score8_kernel(const __grid_constant__ CUtensorMap tmC, DecScoreArgs a) {
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* ring = dsm;
    float* best_s = reinterpret_cast<float*>(ring + kDec8Stages * kDecTile * kDL);  // [kDecTile]
    uint64_t* bars = reinterpret_cast<uint64_t*>(best_s + kDecTile);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kDec8Stages);
    __shared__ float rad;
    __shared__ uint32_t shist[kDecBins];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.y;
    const int64_t r = row / a.hkv;
    const int64_t t = a.pos[r];
    const int64_t lim = t - a.W;
    const int64_t ncol = lim < 0 ? 0 : min(a.cap_buckets, (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1));
    const int64_t c0 = (int64_t)blockIdx.x * kDecScanCols;
    if (c0 >= ncol) return;
    const int64_t cend = min(ncol, c0 + kDecScanCols);
    const int ntiles = (int)((cend - c0 + kDecTile - 1) / kDecTile);
    const uint32_t bar0 = smem_u32(bars);
    constexpr uint32_t kTileB = kDecTile * kDL;  // 16 KB
    for (int i = tid; i < kDecBins; i += 128) shist[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < kDec8Stages; ++s) mbar_init(bar0 + 8u * s, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    const uint16_t* yb = a.Y + (row * NG) * kDL;
    if (tid == 0) rad = row_radius8(yb, NG);
    // B operand in the permuted K order: k-step kk, lane (g, t): dims
    // 16 t + 4 kk + {0, 1} (b0) and + {2, 3} (b1) of latent row g
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t yq[4][2];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint16_t* yr = yb + gq * kDL + 16 * tq + 4 * kk;
        yq[kk][0] = gq < NG ? bf16_pair_to_f16x2(yr[0], yr[1]) : 0u;
        yq[kk][1] = gq < NG ? bf16_pair_to_f16x2(yr[2], yr[3]) : 0u;
    }
    __syncthreads();
    const int64_t rowbase = row * a.cap_buckets;
    if (tid == 0) {
        for (int i = 0; i < kDec8Stages && i < ntiles; ++i) {
            mbar_expect_tx(bar0 + 8u * i, kTileB);
            tma_load_2d(smem_u32(ring + i * kTileB), &tmC, 0, (int32_t)(rowbase + c0 + i * kDecTile), bar0 + 8u * i);
        }
    }
    const float R = rad;
    const int64_t hb0 = rowbase;
    const int64_t frontier = ncol - kBucketsPerBlock;
    int done = 0;
    for (int it = 0; it < ntiles; ++it) {
        const int s = it % kDec8Stages;
        const int64_t tb0 = c0 + (int64_t)it * kDecTile;
        int32_t clr_pre[kDecTile / 128];
#pragma unroll
        for (int u = 0; u < kDecTile / 128; ++u) {
            const int64_t b = tb0 + tid + 128 * u;
            clr_pre[u] = b < cend ? __ldg(a.cnt_lr + hb0 + b) : 0;
        }
        const bool ok = mbar_wait(bar0 + 8u * s, (uint32_t)(it / kDec8Stages) & 1u, abort_flag);
        if (!__syncthreads_and(ok)) break;
        const uint8_t* tile = ring + s * kTileB;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            const int m0 = 64 * warp + 16 * mt;
            const uint4 ra = *reinterpret_cast<const uint4*>(tile + (m0 + gq) * kDL + 16 * tq);
            const uint4 rb = *reinterpret_cast<const uint4*>(tile + (m0 + gq + 8) * kDL + 16 * tq);
            const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w}, wb[4] = {rb.x, rb.y, rb.z, rb.w};
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t af[4] = {e4m3x2_to_f16x2(wa[kk] & 0xFFFFu), e4m3x2_to_f16x2(wb[kk] & 0xFFFFu),
                                        e4m3x2_to_f16x2(wa[kk] >> 16), e4m3x2_to_f16x2(wb[kk] >> 16)};
                mma_16816_f16(acc, af, yq[kk][0], yq[kk][1]);
            }
            float b0 = NG > 1 ? fmaxf(acc[0], acc[1]) : acc[0];
            float b1 = NG > 1 ? fmaxf(acc[2], acc[3]) : acc[2];
            if (NG > 2) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, 1));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, 1));
            }
            if (NG > 4) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, 2));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, 2));
            }
            if (tq == 0) {
                best_s[m0 + gq] = b0 * 0x1p-8f;
                best_s[m0 + gq + 8] = b1 * 0x1p-8f;
            }
        }
        __syncthreads();
        if (tid == 0 && it + kDec8Stages < ntiles) {
            fence_proxy_async_smem();
            mbar_expect_tx(bar0 + 8u * s, kTileB);
            tma_load_2d(smem_u32(ring + s * kTileB), &tmC, 0, (int32_t)(rowbase + c0 + (it + kDec8Stages) * kDecTile),
                        bar0 + 8u * s);
        }
#pragma unroll
        for (int u = 0; u < kDecTile / 128; ++u) {
            const int j = tid + 128 * u;
            const int64_t b = tb0 + j;
            if (b >= cend) break;
            const int32_t clr = clr_pre[u];
            int w = clr;
            if (b >= frontier) {
                const int32_t mlr = __ldg(a.minlr + hb0 + b), mxp = __ldg(a.maxpos + hb0 + b);
                w = 0;
                if ((int64_t)mlr <= lim)
                    w = (int64_t)mxp <= lim ? clr : weight_units(b, __ldg(a.units + hb0 + b), lim, a.S, a.T_built);
            }
            const int bn = score_to_bin(best_s[j], R);
            a.bin[row * a.ld + b] = (uint16_t)bn;
            a.wt[row * a.ld + b] = (uint8_t)w;
            if (w > 0) atomicAdd(&shist[bn], (uint32_t)w);
        }
        __syncthreads();
        done = it + 1;
    }
    if (tid == 0 && *abort_flag) {
        const int issued = min(ntiles, done + kDec8Stages);
        for (int i = done; i < issued; ++i)
            mbar_wait(bar0 + 8u * (i % kDec8Stages), (uint32_t)(i / kDec8Stages) & 1u, abort_flag, false);
    }
    __syncthreads();
    long long tc;
    const int jc = dec_cut_block(shist, a.k, &tc);
    if (tid == 0 && tc) atomicAdd(a.tot + row, (unsigned long long)tc);
    for (int i = jc + tid; i < kDecBins; i += 128)
        if (shist[i]) atomicAdd(a.hist + row * kDecBins + i, shist[i]);
}

// ------------------------------------------------------ flat decode cut

// Slots of chunk [c0, c0 + kDecScanCols) of a row with a key in [S, t - W]
// and a bin >= the row's cut, in ascending id, into the chunk's segment
// (kCap ids; the count is stored whole, so an overflow shows).  grid
// (chunks, rows), 4 warps; warp w takes a contiguous quarter of the chunk.
struct DecKeepArgs {
    const uint32_t* hist;    // [rows, kDecBins]
    const unsigned long long* tot;  // [rows]
    const uint16_t* bin;     // [rows, ld]
    const uint8_t* wt;       // [rows, ld]
    int32_t* seg;            // [rows, nch, kCap]
    int32_t* segn;           // [rows, nch]
    int64_t ld, cap_buckets, nch;
    int32_t hkv, k, S, W;
    int64_t pos[LSA_MAX_BATCH];
};

__device__ __forceinline__ int64_t dec_ncol(int64_t t, int32_t S, int32_t W, int64_t cap_buckets) {
    const int64_t lim = t - W;
    if (lim < S) return 0;
    return min(cap_buckets, (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1));
}

__global__ void __launch_bounds__(128) decode_keep_kernel(DecKeepArgs a) {
    __shared__ int wc[4];
    __shared__ __align__(16) uint32_t h[kDecBins];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.y, chunk = blockIdx.x;
    const int64_t ncol = dec_ncol(a.pos[row / a.hkv], a.S, a.W, a.cap_buckets);
    int32_t* nout = a.segn + row * a.nch + chunk;
    const int64_t c0 = chunk * (int64_t)kDecScanCols;
    if (c0 >= ncol) {
        if (tid == 0) *nout = 0;
        return;
    }
    if ((long long)a.tot[row] <= a.k) {  // the resolve takes every eligible key
        if (tid == 0) *nout = 0;
        return;
    }
    for (int i = tid; i < kDecBins / 4; i += 128)
        reinterpret_cast<uint4*>(h)[i] = reinterpret_cast<const uint4*>(a.hist + row * kDecBins)[i];
    __syncthreads();
    long long hsum;
    const int jt = dec_cut_block(h, a.k, &hsum);
    const uint16_t* brow = a.bin + row * a.ld;
    const uint8_t* wrow = a.wt + row * a.ld;
    auto hits16 = [&](int64_t g16) -> uint32_t {
        const uint4 wv = *reinterpret_cast<const uint4*>(wrow + g16 * 16);
        const uint4 bv0 = *reinterpret_cast<const uint4*>(brow + g16 * 16);
        const uint4 bv1 = *reinterpret_cast<const uint4*>(brow + g16 * 16 + 8);
        const uint32_t wu[4] = {wv.x, wv.y, wv.z, wv.w};
        const uint32_t bu[8] = {bv0.x, bv0.y, bv0.z, bv0.w, bv1.x, bv1.y, bv1.z, bv1.w};
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t w = (wu[i >> 2] >> (8 * (i & 3))) & 0xFFu;
            const int b = (int)((bu[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
            m |= (uint32_t)(w > 0 && b >= jt && g16 * 16 + i < ncol) << i;
        }
        return m;
    };
    const int64_t g0 = c0 / 16, g1 = (min(ncol, c0 + (int64_t)kDecScanCols) + 15) / 16;
    const int64_t per = (g1 - g0 + 3) / 4;
    const int64_t g_lo = g0 + wid * per, g_hi = min(g1, g_lo + per);
    int c = 0;
    for (int64_t g = g_lo + lane; g < g_hi; g += 32) c += __popc(hits16(g));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    if (lane == 0) wc[wid] = c;
    __syncthreads();
    int base = 0, total = 0;
    for (int i = 0; i < 4; ++i) {
        if (i < wid) base += wc[i];
        total += wc[i];
    }
    if (tid == 0) *nout = total;
    if (total > kCap) return;  // the resolve falls back to exact scores
    int32_t* out = a.seg + (row * a.nch + chunk) * (int64_t)kCap;
    for (int64_t s0 = g_lo; s0 < g_hi; s0 += 32) {
        const int64_t g = s0 + lane;
        uint32_t m = g < g_hi ? hits16(g) : 0u;
        const int nh = __popc(m);
        int incl = nh;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        int o = base + incl - nh;
        while (m) {
            const int i = __ffs(m) - 1;
            m &= m - 1;
            out[o++] = (int32_t)(g * 16 + i);
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// ---------------------------------------------------- flat decode resolve

struct DecResolveArgs {
    SelectArgs s;            // cache, cfg, idx, decode positions (row_info)
    const uint16_t* bin;
    uint8_t* wt;             // weights in, taken counts out (fallback rows)
    double* slot;            // [rows, ld] exact scores (fallback rows)
    int64_t ld;
    int64_t cap_buckets;
    const unsigned long long* tot;  // [rows] key weight of the row
    const int32_t* seg;      // [rows, nch, kCap] kept slots per chunk (decode_keep_kernel)
    const int32_t* segn;     // [rows, nch]
    int64_t nch;
};

__global__ void __launch_bounds__(kSelThreads) decode_resolve_kernel(DecResolveArgs d) {
    __shared__ SelShared sh;
    __shared__ int wcnt[kSelThreads / 32];
    const SelectArgs& a = d.s;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    const RowInfo r = row_info(a, row);
    write_sinks_window(a, r);
    if (r.lim < a.S) {
        for (int i = tid; i < a.k; i += kSelThreads) r.out[a.S + i] = -1;
        return;
    }
    load_latents(a, r, sh);
    const int ng = a.agg ? a.G : 1;
    const int64_t ncol = min(d.cap_buckets, (int64_t)kBucketsPerBlock * (r.lim / kBlockKeys + 1));
    uint8_t* wrow = d.wt + row * d.ld;
    // the row's key weight (summed by the score kernel); the cut itself is
    // the keep kernel's, which left the kept slots in per-chunk segments
    const long long totw = (long long)d.tot[row];
    if (totw <= a.k) {
        emit_range(a, r, ncol, [&](int64_t b) -> int { return (int)wrow[b]; }, sh);
        return;
    }
    // candidates: the keep kernel's per-chunk segments, concatenated in
    // chunk order (ascending ids)
    const int64_t nch = (ncol + kDecScanCols - 1) / kDecScanCols;
    const int32_t* sn = d.segn + row * d.nch;
    int my = 0;
    for (int64_t c = tid; c < nch; c += kSelThreads) my += sn[c];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) my += __shfl_xor_sync(0xffffffffu, my, off);
    if (lane == 0) wcnt[wid] = my;
    __syncthreads();
    int ncand = 0;
    for (int i = 0; i < kSelThreads / 32; ++i) ncand += wcnt[i];
    __syncthreads();
    if (ncand <= kCap) {
        int base = 0;
        for (int64_t cb = 0; cb < nch; cb += kSelThreads) {
            const int64_t c = cb + tid;
            const int n = c < nch ? sn[c] : 0;
            int incl = n;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            if (lane == 31) wcnt[wid] = incl;
            __syncthreads();
            int wbase = base;
            int gtot = 0;
            for (int i = 0; i < kSelThreads / 32; ++i) {
                if (i < wid) wbase += wcnt[i];
                gtot += wcnt[i];
            }
            const int32_t* src = d.seg + (row * d.nch + c) * (int64_t)kCap;
            const int o = wbase + incl - n;
            for (int j = 0; j < n; ++j) sh.cid[o + j] = src[j];
            base += gtot;
            __syncthreads();
        }
        __syncthreads();
        const int n = ncand;
        const int64_t hb0 = (int64_t)r.h * d.cap_buckets;
        for (int i = tid; i < n; i += kSelThreads) {
            const int64_t b = sh.cid[i];
            sh.csc[i] = a.cent8 ? exact_row8(sh.ylat, ng, a.cent8 + (hb0 + b) * kDL)
                                : exact_row(sh.ylat, ng, a.cent + (hb0 + b) * kDL);
            sh.cw[i] = wrow[b];
        }
        __syncthreads();
        radix_fill(
            n, a.k, [&](int64_t i) { return sh.csc[i]; }, [&](int64_t i) { return sh.cw[i]; },
            [&](int64_t i, int tk) { sh.ctk[i] = tk; }, sh);
        emit_candidates(a, r, n, sh);
        return;
    }
    // band overflow (dense ties): exact scores of every eligible bucket
    double* fs = d.slot + row * d.ld;
    const int64_t hb0 = (int64_t)r.h * d.cap_buckets;
    for (int64_t b = tid; b < ncol; b += kSelThreads)
        fs[b] = wrow[b] == 0 ? 0.0
                : a.cent8 ? exact_row8(sh.ylat, ng, a.cent8 + (hb0 + b) * kDL)
                          : exact_row(sh.ylat, ng, a.cent + (hb0 + b) * kDL);
    __syncthreads();
    radix_fill(
        ncol, a.k, [&](int64_t i) { return fs[i]; }, [&](int64_t i) { return (int)wrow[i]; },
        [&](int64_t i, int tk) { wrow[i] = (uint8_t)tk; }, sh);
    __syncthreads();
    emit_range(a, r, ncol, [&](int64_t b) -> int { return (int)wrow[b]; }, sh);
}

// ------------------------------------------------------------- host side

static int64_t decode_row_len(const lsa_cfg* cfg) { return cfg->sinks + cfg->k + cfg->window; }

struct DecodeWs {
    uint16_t* Y;
    int32_t* idx;
    uint16_t* bin;
    uint8_t* wt;
    double* slot;
    uint32_t* hist;
    unsigned long long* tot;
    int32_t* seg;
    int32_t* segn;
    int64_t nch;
    double* Utmp;
    size_t step_bytes, load_bytes;
};

static DecodeWs carve_decode(const lsa_cfg* cfg, const lsa_decode* d, char* base) {
    DecodeWs w{};
    const int64_t rows = (int64_t)d->batch * d->hkv;
    const int64_t ld = (d->cache.cap_buckets + 127) / 128 * 128;
    const int32_t hy = cfg->agg ? d->hq : d->hkv;
    size_t o = 0;
    auto take = [&](size_t n) { size_t at = o; o += (n + 255) & ~(size_t)255; return base + at; };
    w.Y = (uint16_t*)take((size_t)d->batch * hy * kDL * 2);
    w.idx = (int32_t*)take((size_t)rows * decode_row_len(cfg) * 4);
    if (cfg->mode == 0) {
        w.bin = (uint16_t*)take((size_t)rows * ld * 2);
        w.wt = (uint8_t*)take((size_t)rows * ld);
        w.slot = (double*)take((size_t)rows * ld * 8);
        w.nch = (d->cache.cap_buckets + kDecScanCols - 1) / kDecScanCols;
        w.hist = (uint32_t*)take((size_t)rows * kDecBins * 4);
        w.tot = (unsigned long long*)take((size_t)rows * 8);
        w.seg = (int32_t*)take((size_t)rows * w.nch * kCap * 4);
        w.segn = (int32_t*)take((size_t)rows * w.nch * 4);
    }
    w.step_bytes = o;
    // a request load reuses the same bytes for its temporary pooled units
    w.Utmp = (double*)base;
    w.load_bytes = (size_t)d->hkv * (d->cap / kPool) * kDL * 8;
    return w;
}

static lsa_cache request_view(const lsa_decode* d, int32_t r) {
    lsa_cache v = d->cache;
    const int64_t h0 = (int64_t)r * d->hkv;
    v.hkv = d->hkv;
    v.U = nullptr;
    v.bucket_of_unit += h0 * v.cap_units;
    v.members += h0 * v.cap_units;
    v.offsets += h0 * (v.cap_buckets + 1);
    v.cnt_lr += h0 * v.cap_buckets;
    v.minlr += h0 * v.cap_buckets;
    v.maxpos += h0 * v.cap_buckets;
    v.sum += h0 * v.cap_buckets * kDL;
    v.cent += h0 * v.cap_buckets * kDL;
    v.units += h0 * v.cap_buckets;
    if (v.cent8) v.cent8 += h0 * v.cap_buckets * kDL;
    return v;
}

static lsa_tree tree_view(const lsa_decode* d, int32_t r) {
    lsa_tree t = d->tree;
    const int64_t h0 = (int64_t)r * d->hkv;
    t.sum += h0 * t.n_nodes * kDL;
    t.minlr += h0 * t.n_nodes;
    t.cent += h0 * t.n_nodes * kDL;
    return t;
}

static lsa_status check_decode(const lsa_decode* d, const lsa_cfg* cfg) {
    if (!d) return set_error(LSA_EINVAL, "decode state is NULL");
    if (d->batch < 1 || d->batch > LSA_MAX_BATCH) return set_error(LSA_EUNSUPPORTED, "decode: batch must be 1..%d", LSA_MAX_BATCH);
    if (d->hkv < 1 || d->hq < 1 || d->hq % d->hkv) return set_error(LSA_EINVAL, "decode: need hq %% hkv == 0");
    const int G = d->hq / d->hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return set_error(LSA_EUNSUPPORTED, "decode: hq / hkv must be 1, 2, 4 or 8");
    if (d->cap < kBlockKeys || d->cap % kBlockKeys) return set_error(LSA_EINVAL, "decode: cap must be a positive multiple of 512");
    if (!d->K || !d->V || !d->U_blk) return set_error(LSA_EINVAL, "decode: K, V or U_blk is NULL");
    if (d->shared_len < 0 || d->shared_len % kBlockKeys || d->shared_len >= d->cap)
        return set_error(LSA_EINVAL, "decode: shared_len must be a multiple of 512 in [0, cap)");
    if (d->shared_len > 0 && (!d->K_shared || !d->V_shared))
        return set_error(LSA_EINVAL, "decode: shared_len > 0 needs K_shared and V_shared");
    const lsa_cache& c = d->cache;
    if (c.hkv != d->batch * d->hkv) return set_error(LSA_EINVAL, "decode: cache.hkv must be batch * hkv");
    if (c.cap_units != d->cap / kPool || c.cap_buckets != d->cap / kBlockKeys * kBucketsPerBlock)
        return set_error(LSA_EINVAL, "decode: cache capacities must match cap");
    if (!c.bucket_of_unit || !c.members || !c.offsets || !c.cnt_lr || !c.minlr || !c.maxpos || !c.sum ||
        !c.cent || !c.units)
        return set_error(LSA_EINVAL, "decode: a cache array is NULL");
    if (cfg->mode == 1) {
        lsa_tree ref;
        lsa_tree_layout(c.cap_buckets, &ref);
        if (!d->tree.sum || !d->tree.minlr || !d->tree.cent || d->tree.levels != ref.levels ||
            d->tree.n_nodes != ref.n_nodes)
            return set_error(LSA_EINVAL, "decode: tree mode needs a tree laid out over cache.cap_buckets");
    }
    return LSA_OK;
}

static int lstar_for(const lsa_cfg* cfg) {
    int l = 0;
    while ((int64_t)cfg->beam * cfg->bucket_mean * ((int64_t)1 << l) < cfg->k && l < 62) ++l;
    return l;
}

static void fill_select_args(SelectArgs& a, const lsa_decode* d, const lsa_cfg* cfg, const uint16_t* Y,
                             int32_t* idx) {
    const lsa_cache& c = d->cache;
    a.offsets = c.offsets; a.members = c.members; a.cnt_lr = c.cnt_lr; a.minlr = c.minlr;
    a.maxpos = c.maxpos; a.cent = c.cent; a.cap_units = c.cap_units; a.cap_buckets = c.cap_buckets;
    a.NB = c.cap_buckets; a.T_built = d->cap;
    a.hkv = d->hkv; a.G = d->hq / d->hkv; a.agg = cfg->agg; a.k = cfg->k; a.S = cfg->sinks; a.W = cfg->window;
    a.mode = cfg->mode;
    if (cfg->mode == 1) {
        a.tminlr = d->tree.minlr; a.tcent = d->tree.cent; a.n_nodes = d->tree.n_nodes;
        a.levels = d->tree.levels; a.beam = cfg->beam; a.lstar = lstar_for(cfg);
        for (int l = 0; l < d->tree.levels; ++l) { a.level_n[l] = d->tree.level_n[l]; a.level_off[l] = d->tree.level_off[l]; }
    }
    a.Y = Y; a.nqc = d->batch; a.t_first = 0; a.idx = idx;
    a.decode = 1;
    a.cent8 = cfg->mode == 0 ? c.cent8 : nullptr;  // the flat decode search scores the FP8 centroids
    for (int r = 0; r < d->batch; ++r) a.pos[r] = d->len[r];
}

}  // namespace lsa

using namespace lsa;

extern "C" {

size_t lsa_decode_workspace_bytes(const lsa_cfg* cfg, const lsa_decode* d) {
    if (check_cfg(cfg) != LSA_OK || check_decode(d, cfg) != LSA_OK) return 0;
    const DecodeWs w = carve_decode(cfg, d, nullptr);
    return w.step_bytes > w.load_bytes ? w.step_bytes : w.load_bytes;
}

lsa_status lsa_decode_load(lsa_decode* d, int32_t r, int64_t n, const float* W_k, const lsa_cfg* cfg,
                           void* ws, size_t ws_bytes, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_decode(d, cfg)) != LSA_OK) return s;
    if (r < 0 || r >= d->batch) return set_error(LSA_EINVAL, "lsa_decode_load: request %d out of range", r);
    if (n < 0 || n >= d->cap) return set_error(LSA_ENOSPACE, "lsa_decode_load: n must be in [0, cap)");
    if (n < d->shared_len) return set_error(LSA_EINVAL, "lsa_decode_load: n below the shared prefix");
    if (!W_k || !ws) return set_error(LSA_EINVAL, "lsa_decode_load: W_k or ws is NULL");
    const DecodeWs w = carve_decode(cfg, d, (char*)ws);
    if (ws_bytes < w.load_bytes || ws_bytes < w.step_bytes)
        return set_error(LSA_ENOSPACE, "lsa_decode_load: workspace too small");
    cudaStream_t st = (cudaStream_t)stream;
    const lsa_cache view = request_view(d, r);
    const int64_t sl = d->shared_len;
    const uint16_t* Kr = d->K + (int64_t)r * (d->cap - sl) * d->hkv * kD;   // the request's rows from sl on
    const int64_t nb = n / kBlockKeys, nc = nb * kBlockKeys;                 // nc >= sl (sl is whole blocks)
    if (nb > 0) {
        if (sl > 0 &&
            (s = launch_key_latent(d->K_shared, sl, d->hkv, W_k, 0, sl / kPool, nc / kPool, w.Utmp, st)) != LSA_OK)
            return s;
        if (nc > sl && (s = launch_key_latent(Kr, nc - sl, d->hkv, W_k, 0, (nc - sl) / kPool, nc / kPool,
                                              w.Utmp + (sl / kPool) * kDL, st)) != LSA_OK)
            return s;
        if ((s = launch_ward_u(&view, w.Utmp, nc / kPool, nc, cfg->sinks, 0, nb, st)) != LSA_OK) return s;
    }
    if ((s = launch_clear_slots(&view, nb * kBucketsPerBlock, view.cap_buckets, st)) != LSA_OK) return s;
    const int64_t j0 = nc / kPool, j1 = (n + kPool - 1) / kPool;
    if (j1 > j0) {
        const int64_t warps = (j1 - j0) * d->hkv;
        tail_units_kernel<<<(unsigned)ceil_div<int64_t>(warps, 8), 256, 0, st>>>(
            Kr, W_k, d->U_blk, n, j0, j1, d->hkv, (int64_t)r * d->hkv, sl);
        if ((s = check_launch("tail_units_kernel")) != LSA_OK) return s;
    }
    if (cfg->mode == 1) {
        lsa_tree tv = tree_view(d, r);
        if ((s = launch_tree_update(&view, &tv, 0, view.cap_buckets, st)) != LSA_OK) return s;
    }
    d->len[r] = n;
    return LSA_OK;
}

lsa_status lsa_decode_step(lsa_decode* d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const float* W_k, const float* W_q, const lsa_cfg* cfg, uint16_t* o,
                           int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_decode(d, cfg)) != LSA_OK) return s;
    if (!q || !k || !v || !W_k || !W_q || !o || !ws) return set_error(LSA_EINVAL, "lsa_decode_step: NULL pointer");
    for (int r = 0; r < d->batch; ++r)
        if (d->len[r] < 0 || d->len[r] >= d->cap)
            return set_error(LSA_ENOSPACE, "lsa_decode_step: request %d is full (len %lld, cap %lld)", r,
                             (long long)d->len[r], (long long)d->cap);
    const DecodeWs w = carve_decode(cfg, d, (char*)ws);
    if (ws_bytes < w.step_bytes) return set_error(LSA_ENOSPACE, "lsa_decode_step: workspace too small");
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t rows = (int64_t)d->batch * d->hkv;

    // (1) append k/v and pool the new key
    AppendArgs ap{};
    ap.k = k; ap.v = v; ap.K = d->K; ap.V = d->V; ap.W = W_k; ap.U_blk = d->U_blk;
    ap.tail = d->cap - d->shared_len; ap.shared_len = d->shared_len;
    ap.hkv = d->hkv; ap.batch = d->batch;
    ap.hist = cfg->mode == 0 ? w.hist : nullptr;
    ap.tot = w.tot;
    for (int r = 0; r < d->batch; ++r) ap.pos[r] = d->len[r];
    {
        KTime kt_("decode_append_kernel", st);
        decode_append_kernel<<<(unsigned)ceil_div<int64_t>(rows, 8), 256, 0, st>>>(ap);
    }
    if ((s = check_launch("decode_append_kernel")) != LSA_OK) return s;

    // (2) cluster every block this token completed
    int32_t head0[LSA_MAX_BATCH];
    int64_t blk[LSA_MAX_BATCH];
    int nj = 0;
    for (int r = 0; r < d->batch; ++r)
        if ((d->len[r] + 1) % kBlockKeys == 0) { head0[nj] = r * d->hkv; blk[nj] = d->len[r] / kBlockKeys; ++nj; }
    if ((s = launch_ward_jobs(&d->cache, d->U_blk, d->hkv, cfg->sinks, nj, head0, blk, st)) != LSA_OK) return s;
    if (cfg->mode == 1) {
        for (int j = 0; j < nj; ++j) {
            const int r = head0[j] / d->hkv;
            lsa_cache cv = request_view(d, r);
            lsa_tree tv = tree_view(d, r);
            if ((s = launch_tree_update(&cv, &tv, blk[j] * kBucketsPerBlock, (blk[j] + 1) * kBucketsPerBlock, st)) != LSA_OK)
                return s;
        }
    }
    // the new token is part of the context from here on
    for (int r = 0; r < d->batch; ++r) d->len[r] += 1;

    // (3) query latents, selection
    if ((s = launch_query_latent(q, d->batch, d->hq, d->hkv, W_q, cfg->agg, w.Y, st)) != LSA_OK) return s;
    int32_t* idx = idx_out ? idx_out : w.idx;
    SelectArgs a{};
    fill_select_args(a, d, cfg, w.Y, idx);
    for (int r = 0; r < d->batch; ++r) a.pos[r] = d->len[r] - 1;
    if (cfg->mode == 1) {
        if ((s = launch_tree_select(a, rows, st)) != LSA_OK) return s;
    } else {
        const int64_t ld = (d->cache.cap_buckets + 127) / 128 * 128;
        DecScoreArgs sa{};
        sa.Y = w.Y; sa.cent = d->cache.cent; sa.minlr = d->cache.minlr; sa.maxpos = d->cache.maxpos;
        sa.cnt_lr = d->cache.cnt_lr; sa.units = d->cache.units; sa.cap_buckets = d->cache.cap_buckets;
        sa.ld = ld; sa.hkv = d->hkv; sa.G = d->hq / d->hkv; sa.agg = cfg->agg; sa.S = cfg->sinks;
        sa.W = cfg->window; sa.T_built = d->cap; sa.bin = w.bin; sa.wt = w.wt; sa.hist = w.hist;
        sa.tot = w.tot; sa.k = cfg->k;
        for (int r = 0; r < d->batch; ++r) sa.pos[r] = a.pos[r];
        dim3 grid((unsigned)ceil_div<int64_t>(d->cache.cap_buckets, kDecScanCols), (unsigned)rows);
        const int ng = cfg->agg ? d->hq / d->hkv : 1;
        CUtensorMap tmC;
        if (d->cache.cent8) {
            if ((s = make_rows64_u8_map(&tmC, d->cache.cent8, rows * d->cache.cap_buckets, kDecTile)) != LSA_OK)
                return s;
            auto kern = ng == 1 ? decode_score8_kernel<1> : ng == 2 ? decode_score8_kernel<2>
                      : ng == 4 ? decode_score8_kernel<4> : decode_score8_kernel<8>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDec8ScanSmem);
            {
                KTime kt_("decode_score_kernel", st);
                kern<<<grid, 128, kDec8ScanSmem, st>>>(tmC, sa);
            }
        } else {
            if ((s = make_rows64_map(&tmC, d->cache.cent, rows * d->cache.cap_buckets, kDecTile)) != LSA_OK) return s;
            auto kern = ng == 1 ? decode_score_kernel<1> : ng == 2 ? decode_score_kernel<2>
                      : ng == 4 ? decode_score_kernel<4> : decode_score_kernel<8>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecScanSmem);
            {
                KTime kt_("decode_score_kernel", st);
                kern<<<grid, 128, kDecScanSmem, st>>>(tmC, sa);
            }
        }
        if ((s = check_launch("decode_score_kernel")) != LSA_OK) return s;
        DecKeepArgs ka{};
        ka.hist = w.hist; ka.tot = w.tot; ka.bin = w.bin; ka.wt = w.wt; ka.seg = w.seg; ka.segn = w.segn; ka.ld = ld;
        ka.cap_buckets = d->cache.cap_buckets; ka.nch = w.nch; ka.hkv = d->hkv; ka.k = cfg->k; ka.S = cfg->sinks;
        ka.W = cfg->window;
        for (int r = 0; r < d->batch; ++r) ka.pos[r] = a.pos[r];
        {
            KTime kt_("decode_keep_kernel", st);
            decode_keep_kernel<<<dim3((unsigned)w.nch, (unsigned)rows), 128, 0, st>>>(ka);
        }
        if ((s = check_launch("decode_keep_kernel")) != LSA_OK) return s;
        DecResolveArgs ra{};
        ra.s = a; ra.bin = w.bin; ra.wt = w.wt; ra.slot = w.slot; ra.ld = ld; ra.cap_buckets = d->cache.cap_buckets;
        ra.tot = w.tot; ra.seg = w.seg; ra.segn = w.segn; ra.nch = w.nch;
        {
            KTime kt_("decode_resolve_kernel", st);
            decode_resolve_kernel<<<(unsigned)rows, kSelThreads, 0, st>>>(ra);
        }
        if ((s = check_launch("decode_resolve_kernel")) != LSA_OK) return s;
    }
    // (4) attention: each request reads its own K/V rows
    return launch_attn(q, d->K, d->V, idx, d->batch, d->hq, d->hkv, (int32_t)decode_row_len(cfg), d->cap,
                       o, st, d->cap - d->shared_len, 8, -1, nullptr, nullptr, d->K_shared, d->V_shared,
                       d->shared_len);
}

}  // extern "C"
