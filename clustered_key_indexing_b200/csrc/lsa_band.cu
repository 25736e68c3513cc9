// lsa_band.cu -- the sliding-window part of an LSA index row as banded dense
// attention on the 5th-generation tensor cores [tutorial "隐空间稀疏注意力
// (LSA)" (diosapp.com.cn), section 二: every query always attends to its
// sinks and its last W positions; the attention formula is unchanged].
//
// Query t's window is positions max(S, t - W + 1) .. t: consecutive queries
// share almost all of it.  A CTA takes 128 (query, head) rows of one kv-head
// (128 / G consecutive queries x the G heads of the group) and streams the
// union of their windows in 64-key tiles, so each K/V tile is read once for
// all 128 rows.  Per CTA (two per SM):
//   warp 0 (one thread)  TMA loads of K and V tiles (3-D tensor maps over
//       [position, kv-head, dim], 128-byte swizzle), two stages each;
//   warp 1 (one thread)  tcgen05.mma: S = Q K^T (M = 128 rows, N = 64 keys,
//       K = 128 dims; Q and K from shared memory) into TMEM, and O += P V
//       (M = 128, N = 128 dims, K = 64 keys) with P read from TMEM and V
//       from shared memory as an MN-major operand; O accumulates in TMEM.
//       S(i + 1) is computed as soon as the softmax threads hold S(i) in
//       registers, and P is double-buffered, so the softmax of tile i
//       overlaps both products of its neighbours;
//   warps 2-5  one row per thread (TMEM lane = row): S from TMEM, band
//       masks, online softmax in fp32 with independent max / sum chains
//       (exp2 with log2(e)/sqrt(d) folded into one FFMA), P as bf16 into
//       TMEM.  The running max is moved (and O, l rescaled) only when a
//       row's max grows by more than 2^8, so P stays <= 256 and O is rarely
//       touched.  (Two threads per row, each exponentiating half the keys,
//       measured 5% slower: both must read all 64 scores for the row max.)
// Output: the normalised window output O_w (fp32) and its log-sum-exp (log2
// domain) per row, merged with the sinks and long-range part by the gather
// kernel's epilogue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"
#include "lsa_tc.cuh"

namespace lsa {

constexpr int kBandRows = 128;                              // (query, head) rows per CTA
constexpr int kBandKeys = 64;                               // keys per tile
constexpr int kBandSoftmax = kBandRows;                     // softmax threads: one per row
constexpr int kBandThreads = 64 + kBandSoftmax;             // producer warp, MMA warp, four softmax warps
constexpr uint32_t kBandQBlk = kBandRows * 128;             // 16 KB: 64 dims of the CTA's rows
constexpr uint32_t kBandKBlk = kBandKeys * 128;             // 8 KB: 64 dims of a tile's keys
constexpr uint32_t kBandTileBytes = 2 * kBandKBlk;          // one K or V tile
constexpr uint32_t kBandTmemCols = 256;                     // S [0, 64), P [64, 128) twice, O [128, 256)
constexpr uint32_t kBandColP = 64, kBandColO = 128;
constexpr int kBandBars = 15;
constexpr size_t kBandSmemBytes = 1024 + 2 * kBandQBlk + 4 * kBandTileBytes + 8 * kBandBars + 16;
static_assert(2 * (kBandSmemBytes + 1024) <= 233472, "two band CTAs per SM");

struct BandArgs {
    const uint16_t* Q;       // [nq, hq, 128]: query i of the call sits at position t0 + i
    int64_t nq, t0, T;
    int32_t hq, hkv, S, W;
    float* Ow;               // [nq, hq, 128] normalised window output
    float* lse;              // [nq, hq] log2-domain log-sum-exp of the scaled scores; -inf: empty window
    float scale_log2;
};

// Barriers: K full/empty and V full/empty per stage; S full (QK done), S
// free (the softmax threads hold S in registers); per P buffer, P full (P
// written) and P done (O += P V from it has landed); drain.  Every wait is
// for the phase right after the last one its thread saw of that barrier, and
// the phase after it cannot complete before the waiter's own next step.
struct BandBars {
    uint32_t b0;
    __device__ uint32_t kfull(int s) const { return b0 + 8u * (uint32_t)s; }
    __device__ uint32_t kempty(int s) const { return b0 + 8u * (uint32_t)(2 + s); }
    __device__ uint32_t vfull(int s) const { return b0 + 8u * (uint32_t)(4 + s); }
    __device__ uint32_t vempty(int s) const { return b0 + 8u * (uint32_t)(6 + s); }
    __device__ uint32_t sfull() const { return b0 + 64u; }
    __device__ uint32_t sfree() const { return b0 + 72u; }
    __device__ uint32_t pfull(int b) const { return b0 + 80u + 8u * (uint32_t)b; }
    __device__ uint32_t pdone(int b) const { return b0 + 96u + 8u * (uint32_t)b; }
    __device__ uint32_t drain() const { return b0 + 112u; }
    __device__ void init() const {
        for (int s = 0; s < 2; ++s) {
            mbar_init(kfull(s), 1); mbar_init(kempty(s), 1);
            mbar_init(vfull(s), 1); mbar_init(vempty(s), 1);
        }
        mbar_init(sfull(), 1);
        mbar_init(sfree(), kBandSoftmax);
        mbar_init(pfull(0), kBandSoftmax);
        mbar_init(pfull(1), kBandSoftmax);
        mbar_init(pdone(0), 1);
        mbar_init(pdone(1), 1);
        mbar_init(drain(), 1);
    }
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

template <int G>
__global__ void __launch_bounds__(kBandThreads, 2)
band_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BandArgs a) {
    extern __shared__ uint8_t bsm_raw[];
    uint8_t* bsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = bsm;                                  // [2 dim blocks][128 rows][128 B]
    uint8_t* sK = sQ + 2 * kBandQBlk;                   // [2 stages][2 dim blocks][64 keys][128 B]
    uint8_t* sV = sK + 2 * kBandTileBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 2 * kBandTileBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBandBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const BandBars bar{smem_u32(bars)};

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int QB = kBandRows / G;  // queries per CTA
    const int h = blockIdx.y;
    const int64_t qb0 = (int64_t)blockIdx.x * QB;
    if (qb0 >= a.nq) return;
    const int64_t qlast = min(a.nq - 1, qb0 + QB - 1);
    // positions fit in int32 (T < 2^31)
    const int t_first = (int)(a.t0 + qb0), t_last = (int)(a.t0 + qlast);
    // keys some row of the CTA attends to: [P0, t_last]
    const int P0 = max(a.S, t_first - a.W + 1);
    const int nkeys = t_last - P0 + 1;
    const int n = nkeys > 0 ? (nkeys + kBandKeys - 1) / kBandKeys : 0;
    // a tile [p0, p0 + 63] is inside every row's window when p0 >= lo_max and p0 + 63 <= t_first
    const int lo_max = max(a.S, t_last - a.W + 1);

    if (tid == 0) {
        bar.init();
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kBandTmemCols);
    // softmax thread of row r = TMEM lane r (warp % 4 selects the lane quarter)
    const int r = (warp & 3) * 32 + lane;
    if (warp >= 2) {
        // the CTA's Q rows (row r = query r / G, head r % G; zero past the
        // call's queries), K-major with the 128-byte swizzle
        const int64_t qq = qb0 + r / G;
        const uint4* src = qq <= qlast ? reinterpret_cast<const uint4*>(a.Q + (qq * a.hq + (int64_t)h * G + r % G) * kD)
                                       : nullptr;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint4 v = src ? src[c] : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(sQ + (c >> 3) * kBandQBlk + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = v;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && n > 0) {
            int nk = 0, nv = 0;
            auto load = [&](bool isk, int i) -> bool {
                const int s = i & 1;
                if (!mbar_wait(isk ? bar.kempty(s) : bar.vempty(s), ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag))
                    return false;
                const uint32_t full = isk ? bar.kfull(s) : bar.vfull(s);
                const uint32_t dst = smem_u32((isk ? sK : sV) + s * kBandTileBytes);
                const CUtensorMap* map = isk ? &tmK : &tmV;
                const int p0 = P0 + i * kBandKeys;
                mbar_expect_tx(full, kBandTileBytes);
                tma_load_3d(dst, map, 0, h, p0, full);
                tma_load_3d(dst + kBandKBlk, map, 64, h, p0, full);
                return true;
            };
            bool ok = load(true, 0);
            nk = ok ? 1 : 0;
            for (int i = 0; ok && i < n; ++i) {
                if (i + 1 < n) {
                    ok = load(true, i + 1);
                    if (ok) ++nk;
                }
                if (ok) ok = load(false, i);
                if (ok) ++nv;
            }
            // after an abort, let this thread's copies land before the CTA exits
            if (*abort_flag) {
                for (int i = max(0, nk - 2); i < nk; ++i) mbar_wait(bar.kfull(i & 1), (uint32_t)(i >> 1) & 1u, abort_flag, false);
                for (int i = max(0, nv - 2); i < nv; ++i) mbar_wait(bar.vfull(i & 1), (uint32_t)(i >> 1) & 1u, abort_flag, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(128, kBandKeys);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(128, kD) | (1u << 16);  // B (V) MN-major
            const uint32_t qa = smem_u32(sQ), kb0 = smem_u32(sK), vb0 = smem_u32(sV);
            auto qk = [&](int i) -> bool {
                const int s = i & 1;
                if (!mbar_wait(bar.kfull(s), (uint32_t)(i >> 1) & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t kb = kb0 + (uint32_t)s * kBandTileBytes;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t off = (uint32_t)(k & 3) * 32u;  // K step within a 64-dim block
                    umma_bf16(tmem, sw128_desc(qa + (uint32_t)(k >> 2) * kBandQBlk + off),
                              sw128_desc(kb + (uint32_t)(k >> 2) * kBandKBlk + off), idesc_qk, k > 0 ? 1u : 0u);
                }
                umma_commit(bar.kempty(s));
                umma_commit(bar.sfull());
                return true;
            };
            auto pv = [&](int i) -> bool {
                const int s = i & 1;
                if (!mbar_wait(bar.pfull(s), (uint32_t)(i >> 1) & 1u, abort_flag)) return false;
                if (!mbar_wait(bar.vfull(s), (uint32_t)(i >> 1) & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t vb = vb0 + (uint32_t)s * kBandTileBytes;
#pragma unroll
                for (int j = 0; j < kBandKeys / 16; ++j)  // keys 16 j .. 16 j + 15: P columns 8 j .., V rows 16 j ..
                    umma_bf16_ts(tmem + kBandColO, tmem + kBandColP + (uint32_t)(32 * s + 8 * j),
                                 sw128_mn_desc(vb + (uint32_t)j * 2048u, kBandKBlk, 1024u), idesc_pv,
                                 (i > 0 || j > 0) ? 1u : 0u);
                umma_commit(bar.vempty(s));
                umma_commit(bar.pdone(s));
                return true;
            };
            bool ok = qk(0);
            for (int i = 0; ok && i < n; ++i) {
                if (i + 1 < n) {
                    // S(i) is in the softmax threads' registers
                    ok = mbar_wait(bar.sfree(), (uint32_t)i & 1u, abort_flag);
                    if (ok) ok = qk(i + 1);
                }
                if (ok) ok = pv(i);
            }
            // every MMA this thread issued has completed once `drain` fires
            umma_commit(bar.drain());
            mbar_wait(bar.drain(), 0, abort_flag, false);
        }
    } else {
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int t = t_first + r / G;
        const int lo_r = max(a.S, t - a.W + 1), hi_r = t;
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar.sfull(), (uint32_t)i & 1u, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t v[64];
            tmem_ld64(trow, v);
            tc_fence_before();
            mbar_arrive(bar.sfree());
            const int p0 = P0 + i * kBandKeys;
            // band edges: keys outside the row's window become -inf (a tile
            // inside every row's window needs no test)
            if (!(p0 >= lo_max && p0 + kBandKeys - 1 <= t_first)) {
#pragma unroll
                for (int c = 0; c < kBandKeys; ++c)
                    if (p0 + c < lo_r || p0 + c > hi_r) v[c] = 0xFF800000u;
            }
            // row max of the raw scores, eight independent chains
            float mx8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mx8[j] = __uint_as_float(v[j]);
#pragma unroll
            for (int c = 8; c < kBandKeys; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(v[c]));
#pragma unroll
            for (int w = 4; w > 0; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) mx8[j] = fmaxf(mx8[j], mx8[j + w]);
            // move the reference max (log2 domain) only when it grows by more than 2^8
            const float m_new = fmaxf(m, mx8[0] * a.scale_log2);
            float alpha = 1.f;
            bool rescale_o = false;
            if (m_new > m + 8.f) {
                if (l > 0.f) {
                    alpha = ex2_approx(m - m_new);
                    rescale_o = true;
                }
                m = m_new;
            }
            // p = 2^(s * scale - m): one FFMA and one ex2 per key (-inf -> 0)
            const float nmu = m == -CUDART_INF_F ? 0.f : -m;
            float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float e0 = ex2_approx(fmaf(__uint_as_float(v[2 * c]), a.scale_log2, nmu));
                const float e1 = ex2_approx(fmaf(__uint_as_float(v[2 * c + 1]), a.scale_log2, nmu));
                rs8[c & 7] += e0 + e1;
                pk[c] = pack_bf16x2(e0, e1);
            }
#pragma unroll
            for (int w = 4; w > 0; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) rs8[j] += rs8[j + w];
            l = l * alpha + rs8[0];
            // P buffer i % 2 is free once O += P(i - 2) V has run
            if (i > 1 && !__all_sync(0xffffffffu, mbar_wait(bar.pdone(i & 1), (uint32_t)((i - 2) >> 1) & 1u, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st32(trow + kBandColP + (uint32_t)(32 * (i & 1)), pk);
            if (__any_sync(0xffffffffu, rescale_o)) {
                // O must hold O += P(i - 1) V before it is rescaled
                if (!__all_sync(0xffffffffu,
                                mbar_wait(bar.pdone((i - 1) & 1), (uint32_t)((i - 1) >> 1) & 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c4 = 0; c4 < kD / 32; ++c4) {
                    uint32_t ov[32];
                    const uint32_t col = kBandColO + (uint32_t)(32 * c4);
                    tmem_ld32_async(trow + col, ov);
                    tmem_wait_ld(ov);
#pragma unroll
                    for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                    tmem_st32(trow + col, ov);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar.pfull(i & 1));
        }
        // O += P(n - 1) V has landed: normalise and store the row
        if (ok && n > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(bar.pdone((n - 1) & 1), (uint32_t)((n - 1) >> 1) & 1u, abort_flag)))
            ok = false;
        tc_fence_after();
        const int64_t rq = qb0 + r / G;
        const int64_t rrow = rq * a.hq + (int64_t)h * G + r % G;
        const bool mine = rq <= qlast;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float* orow = a.Ow + rrow * kD;
#pragma unroll 1
        for (int c4 = 0; c4 < kD / 32; ++c4) {
            uint32_t ov[32];
            if (ok && n > 0) {
                tmem_ld32_async(trow + kBandColO + (uint32_t)(32 * c4), ov);
                tmem_wait_ld(ov);
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) ov[c] = 0u;
            }
            if (mine) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    reinterpret_cast<float4*>(orow + 32 * c4)[c] =
                        make_float4(__uint_as_float(ov[4 * c]) * inv, __uint_as_float(ov[4 * c + 1]) * inv,
                                    __uint_as_float(ov[4 * c + 2]) * inv, __uint_as_float(ov[4 * c + 3]) * inv);
            }
        }
        if (mine) a.lse[rrow] = l > 0.f ? m + log2f(l) : -CUDART_INF_F;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kBandTmemCols);
    }
}

lsa_status launch_band_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t nq, int64_t t0,
                            int64_t T, int32_t hq, int32_t hkv, int32_t S, int32_t W, float* Ow, float* lse,
                            cudaStream_t st) {
    if (nq <= 0) return LSA_OK;
    CUtensorMap tmK, tmV;
    lsa_status s;
    if ((s = make_kv_map(&tmK, K, T, hkv, kBandKeys)) != LSA_OK) return s;
    if ((s = make_kv_map(&tmV, V, T, hkv, kBandKeys)) != LSA_OK) return s;
    BandArgs a{};
    a.Q = Q; a.nq = nq; a.t0 = t0; a.T = T; a.hq = hq; a.hkv = hkv; a.S = S; a.W = W;
    a.Ow = Ow; a.lse = lse;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    const int G = hq / hkv;
    auto kern = G == 1 ? band_attn_kernel<1> : G == 2 ? band_attn_kernel<2> : G == 4 ? band_attn_kernel<4>
                                                                                     : band_attn_kernel<8>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBandSmemBytes);
    {
        KTime kt_("band_attn_kernel", st);
        kern<<<dim3((unsigned)ceil_div<int64_t>(nq, kBandRows / G), (unsigned)hkv), kBandThreads, kBandSmemBytes,
               st>>>(tmK, tmV, a);
    }
    return check_launch("band_attn_kernel");
}

}  // namespace lsa
