// lsa_flat.cuh -- flat search of the LSA path on sm_100a [essay "《卡片柜》——
// 当注意力学会先查目录再翻书", ch. 3: score every centroid, expand the best
// buckets until k long-range keys are filled; ch. 5: native max over heads].
//
// Three kernels per chunk of query positions:
//   flat_pass_kernel<sample=true>   bf16 tensor-core scores (mma.sync
//       m16n8k16, fp32 accumulate) of 64 query rows against every 8th
//       centroid; a per-row weighted histogram of those scores (bins scaled to
//       the row's latent norm, which bounds its scores) gives a threshold tau
//       expected to keep about twice the k keys needed;
//   flat_pass_kernel<sample=false>  the same contraction over every eligible
//       centroid; scores >= tau are appended to the row's candidate list in
//       ascending bucket id;
//   flat_resolve_kernel             one warp per (query, kv-head): eligibility
//       and exact key counts, weighted radix select on the fp32 scores for the
//       cut c32, exact fp64 rescoring of the buckets within 2e of c32 only,
//       key emission in bucket id order, sinks and window.
// Exactness: |fp32 score - exact score| < e = 1e-4 (the error is below
// 64 * 2^-23 * |y||c|).  The exact score E* of the k-th key then lies in
// [c32 - e, c32 + e]: buckets with fp32 score > c32 + 2e rank strictly above
// it, buckets below c32 - 2e strictly below, and only the band between is
// ranked on exact fp64 scores (score desc, bucket id asc).  The band must lie
// above tau (every bucket in it is then a candidate); rows where it does not,
// or whose list overflowed, go to the exact fallback kernel.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"

namespace lsa {

constexpr int kCandCap = 1024;       // candidates kept per (query, kv-head)
constexpr int kSampleStride = 8;     // every 8th bucket scored by the sample pass
constexpr int kSBins = 256;          // sample histogram bins over [-R, R], R = row latent norm
constexpr int kOversample = 2;       // tau targets kOversample * k keys
constexpr float kScoreErr = 1e-4f;   // bound on |fp32 score - exact score|
constexpr int kPassCols = 128;

struct PassArgs {
    const uint16_t* Y;       // chunk latents [nqc, hkv, 64] (mean) / [nqc, hq, 64] (native)
    const uint16_t* cent;    // [hkv, cap_buckets, 64]
    const int32_t* minlr;    // [hkv, cap_buckets]
    const int32_t* cnt_lr;   // [hkv, cap_buckets]
    int64_t cap_buckets, NB, nqc, t_first;
    int32_t W, hkv, G, agg, k;
    float* tau;              // [nqc * hkv]
    int32_t* cand_col;       // [nqc * hkv, kCandCap]
    float* cand_s;           // [nqc * hkv, kCandCap]
    int32_t* cand_n;         // [nqc * hkv]
};

__device__ __forceinline__ int64_t flat_ncol_d(int64_t t, int32_t W, int64_t NB) {
    const int64_t lim = t - W;
    if (lim < 0) return 0;
    const int64_t n = (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1);
    return n < NB ? n : NB;
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}

template <bool SAMPLE>
__global__ void __launch_bounds__(128) flat_pass_kernel(PassArgs a) {
    extern __shared__ __align__(128) uint8_t psm[];
    uint16_t* ctile = reinterpret_cast<uint16_t*>(psm);                       // [2][128*64]
    int32_t* mminlr = reinterpret_cast<int32_t*>(psm + 2 * kPassCols * kDL * 2);  // [2][128]
    int32_t* mcnt = mminlr + 2 * kPassCols;                                   // [2][128]
    float* rads = reinterpret_cast<float*>(mcnt + 2 * kPassCols);             // [64] row radii
    uint32_t* hist = reinterpret_cast<uint32_t*>(rads + 64);                  // sample: [qpt][256]; full: [qpt]

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int h = blockIdx.y;
    const int G = a.agg ? a.G : 1;
    const int qpt = 64 / G;
    const int64_t q0 = (int64_t)blockIdx.x * qpt;
    if (q0 >= a.nqc) return;
    const int64_t qlast = min(a.nqc - 1, q0 + qpt - 1);
    const int64_t ncol_max = flat_ncol_d(a.t_first + qlast, a.W, a.NB);
    const int64_t stride = SAMPLE ? kSampleStride : 1;
    const int64_t nv = ceil_div<int64_t>(ncol_max, stride);
    const int ntile = (int)ceil_div<int64_t>(nv, kPassCols);

    for (int i = tid; i < qpt * (SAMPLE ? kSBins : 1); i += 128) hist[i] = 0u;

    // A fragments (rows of this warp) and per-row limits
    const int g = lane >> 2, tq = lane & 3;
    uint32_t af[4][4];
    int64_t lim[2], ncol[2], row[2];
    float tau[2], rad[2];
    int qloc[2];
    bool rowok[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int r = w * 16 + g + 8 * hh;
        qloc[hh] = r / G;
        const int64_t q = q0 + qloc[hh];
        rowok[hh] = q < a.nqc;
        const int64_t t = a.t_first + (rowok[hh] ? q : 0);
        lim[hh] = t - a.W;
        ncol[hh] = flat_ncol_d(t, a.W, a.NB);
        row[hh] = (rowok[hh] ? q : 0) * a.hkv + h;
        tau[hh] = SAMPLE ? 0.f : a.tau[row[hh]];
        const int64_t yrow = a.agg ? ((rowok[hh] ? q : 0) * (int64_t)a.hkv * G + (int64_t)h * G + r % G) : row[hh];
        const uint16_t* yp = a.Y + yrow * kDL;
        float n2 = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int c0 = kk * 16 + 2 * tq;
            af[kk][hh] = rowok[hh] ? *reinterpret_cast<const uint32_t*>(yp + c0) : 0u;
            af[kk][hh + 2] = rowok[hh] ? *reinterpret_cast<const uint32_t*>(yp + c0 + 8) : 0u;
            const uint32_t u[2] = {af[kk][hh], af[kk][hh + 2]};
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const float lo = __uint_as_float(u[x] << 16), hi = __uint_as_float(u[x] & 0xFFFF0000u);
                n2 += lo * lo + hi * hi;
            }
        }
        // |y| of the row (native: max over the group's heads) bounds |score|
        n2 += __shfl_xor_sync(0xffffffffu, n2, 1);
        n2 += __shfl_xor_sync(0xffffffffu, n2, 2);
        for (int off = 4; off < 4 * G; off <<= 1) n2 = fmaxf(n2, __shfl_xor_sync(0xffffffffu, n2, off));
        rad[hh] = fminf(1.0625f, sqrtf(n2) * 1.01f + 1e-6f);
        if (SAMPLE && rowok[hh] && (g % G) == 0 && tq == 0) rads[qloc[hh]] = rad[hh];
    }

    const uint16_t* cb = a.cent + (int64_t)h * a.cap_buckets * kDL;
    auto load_tile = [&](int tile, int buf) {
        const int64_t v0 = (int64_t)tile * kPassCols;
        uint16_t* dst = ctile + buf * kPassCols * kDL;
#pragma unroll
        for (int i = 0; i < (kPassCols * 8) / 128; ++i) {
            const int idx = tid + 128 * i;
            const int n = idx >> 3, c = idx & 7;
            const bool ok = v0 + n < nv;
            const int64_t b = (v0 + n) * stride;
            cp_async_16(smem_u32(dst + n * kDL + ((c ^ (n & 7)) << 3)),
                        ok ? (const void*)(cb + b * kDL + c * 8) : (const void*)cb, ok ? 16 : 0);
        }
        if (SAMPLE) {
            const bool ok = v0 + tid < nv;
            const int64_t b = (v0 + tid) * stride;
            const int64_t hb = (int64_t)h * a.cap_buckets + (ok ? b : 0);
            cp_async_4(smem_u32(mminlr + buf * kPassCols + tid), a.minlr + hb, ok ? 4 : 0);
            cp_async_4(smem_u32(mcnt + buf * kPassCols + tid), a.cnt_lr + hb, ok ? 4 : 0);
        }
        cp_async_commit();
    };

    if (ntile > 0) load_tile(0, 0);
    __syncthreads();  // histogram / counters cleared
    for (int tile = 0; tile < ntile; ++tile) {
        const int buf = tile & 1;
        if (tile + 1 < ntile) load_tile(tile + 1, buf ^ 1);
        else cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        float acc[16][4];
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
        const uint32_t base = smem_u32(ctile + buf * kPassCols * kDL);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
                const int mi = lane >> 3, ri = lane & 7;
                const int n = (2 * jp + (mi >> 1)) * 8 + ri;
                const int c = 2 * kk + (mi & 1);
                uint32_t b[4];
                ldsm_x4(b, base + (uint32_t)(n * kDL + ((c ^ (n & 7)) << 3)) * 2u);
                mma_16816(acc[2 * jp], af[kk], b[0], b[1]);
                mma_16816(acc[2 * jp + 1], af[kk], b[2], b[3]);
            }
        }
        const int64_t v0 = (int64_t)tile * kPassCols;
        uint32_t hit[2] = {0u, 0u};  // bit 2j+e: element (n8 tile j, column e) kept
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float v[4] = {acc[j][0], acc[j][1], acc[j][2], acc[j][3]};
            for (int off = 4; off < 4 * G; off <<= 1)
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = fmaxf(v[i], __shfl_xor_sync(0xffffffffu, v[i], off));
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[j][i] = v[i];
            if ((g % G) != 0) continue;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                if (!rowok[hh]) continue;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cl = j * 8 + 2 * tq + e;
                    const int64_t vc = v0 + cl;
                    const float sc = v[2 * hh + e];
                    if (SAMPLE) {
                        if (vc * kSampleStride < ncol[hh] && (int64_t)mminlr[buf * kPassCols + cl] <= lim[hh]) {
                            int bin = __float2int_rd((sc + rad[hh]) * ((float)kSBins / (2.f * rad[hh])));
                            bin = bin < 0 ? 0 : (bin >= kSBins ? kSBins - 1 : bin);
                            atomicAdd(&hist[qloc[hh] * kSBins + bin], (uint32_t)mcnt[buf * kPassCols + cl]);
                        }
                    } else if (sc >= tau[hh] && vc < ncol[hh]) {
                        hit[hh] |= 1u << (2 * j + e);
                    }
                }
            }
        }
        if (!SAMPLE) {
            // ordered append: the 4 lanes of a quad hold one row's columns
            // 8j + 2tq + e; a hit's rank in the tile counts the quad's hits
            // in earlier n8 tiles and in earlier lanes of its own tile
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int qb = lane & ~3;
                const uint32_t m0 = __shfl_sync(0xffffffffu, hit[hh], qb);
                const uint32_t m1 = __shfl_sync(0xffffffffu, hit[hh], qb | 1);
                const uint32_t m2 = __shfl_sync(0xffffffffu, hit[hh], qb | 2);
                const uint32_t m3 = __shfl_sync(0xffffffffu, hit[hh], qb | 3);
                const int tot = __popc(m0) + __popc(m1) + __popc(m2) + __popc(m3);
                int base = 0;
                if (tq == 0 && tot > 0) base = (int)atomicAdd(&hist[qloc[hh]], (uint32_t)tot);
                base = __shfl_sync(0xffffffffu, base, qb);
                if (tot == 0) continue;
                const uint32_t mine = hit[hh];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (!((mine >> (2 * j + e)) & 1u)) continue;
                        const uint32_t below = (1u << (2 * j)) - 1u, here = 3u << (2 * j);
                        int pos = __popc(m0 & below) + __popc(m1 & below) + __popc(m2 & below) +
                                  __popc(m3 & below);
                        if (tq > 0) pos += __popc(m0 & here);
                        if (tq > 1) pos += __popc(m1 & here);
                        if (tq > 2) pos += __popc(m2 & here);
                        if (e) pos += (mine >> (2 * j)) & 1u;
                        const int slot = base + pos;
                        if (slot < kCandCap) {
                            a.cand_col[row[hh] * kCandCap + slot] = (int32_t)(v0 + j * 8 + 2 * tq + e);
                            a.cand_s[row[hh] * kCandCap + slot] = acc[j][2 * hh + e];
                        }
                    }
                }
            }
        }
        __syncthreads();  // buffer `buf` is refilled two iterations later
    }
    cp_async_wait<0>();
    __syncthreads();
    if (tid < qpt && q0 + tid < a.nqc) {
        const int64_t r = (q0 + tid) * a.hkv + h;
        if (SAMPLE) {
            // tau: lower edge of the bin where the scaled sample weight from
            // the top first reaches kOversample * k; -inf if it never does
            const float R = rads[tid];
            float t = -CUDART_INF_F;
            long long cum = 0;
            for (int b = kSBins - 1; b >= 0; --b) {
                cum += (long long)hist[tid * kSBins + b] * kSampleStride;
                if (cum >= (long long)kOversample * a.k) { t = -R + b * (2.f * R / kSBins); break; }
            }
            a.tau[r] = t;
        } else {
            a.cand_n[r] = (int32_t)hist[tid];
        }
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
    const int32_t* cand_col;
    const float* cand_s;
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
            col = a.cand_col[row * kCandCap + i];
            sc = a.cand_s[row * kCandCap + i];
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
        // every bucket that can rank above the exact cut must be a candidate
        if (tau > -CUDART_INF_F && !(lo >= tau)) {
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

lsa_status launch_flat(const PassArgs& pa, const ResolveArgs& ra, cudaStream_t st) {
    const int G = pa.agg ? pa.G : 1;
    const int qpt = 64 / G;
    dim3 grid((unsigned)ceil_div<int64_t>(pa.nqc, qpt), (unsigned)pa.hkv);
    const size_t base = 2 * kPassCols * kDL * 2 + 4 * kPassCols * 4 + 64 * 4;
    const size_t smem_s = base + (size_t)qpt * kSBins * 4;
    const size_t smem_f = base + (size_t)qpt * 4;
    cudaFuncSetAttribute(flat_pass_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s);
    cudaFuncSetAttribute(flat_pass_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_f);
    flat_pass_kernel<true><<<grid, 128, smem_s, st>>>(pa);
    lsa_status s = check_launch("flat_pass_kernel<sample>");
    if (s != LSA_OK) return s;
    flat_pass_kernel<false><<<grid, 128, smem_f, st>>>(pa);
    if ((s = check_launch("flat_pass_kernel<full>")) != LSA_OK) return s;
    const size_t smem_r = sizeof(ResWarp) * kResWarps;
    cudaFuncSetAttribute(flat_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_r);
    const int64_t rows = pa.nqc * pa.hkv;
    flat_resolve_kernel<<<(unsigned)ceil_div<int64_t>(rows, kResWarps), 32 * kResWarps, smem_r, st>>>(ra);
    return check_launch("flat_resolve_kernel");
}

}  // namespace lsa
