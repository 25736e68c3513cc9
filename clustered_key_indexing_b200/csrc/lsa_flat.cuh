// lsa_flat.cuh -- flat search of the LSA path on sm_100a [essay "《卡片柜》——
// 当注意力学会先查目录再翻书", ch. 3: score every centroid, expand the best
// buckets until k long-range keys are filled; ch. 5: native max over heads].
//
// Three kernels per chunk of query positions:
//   flat_pass_kernel<sample=true>   bf16 tensor-core scores (mma.sync
//       m16n8k16, fp32 accumulate) of 64 query rows against every 16th
//       centroid; a per-row weighted histogram of those scores gives a
//       threshold tau expected to keep about twice the k keys needed;
//   flat_pass_kernel<sample=false>  the same contraction over every eligible
//       centroid; scores >= tau are appended to the row's candidate list;
//   flat_resolve_kernel             one warp per (query, kv-head): eligibility
//       and exact key counts, exact fp64 rescoring, weighted radix select on
//       the exact scores (score desc, bucket id asc), sort of the chosen
//       buckets by id, key emission, sinks and window.
// The resolve step checks that the buckets with fp32 score >= tau + 2e
// already hold k keys (e = 1e-4 bounds the fp32 score error, which is below
// 64 * 2^-23 * |y||c|): then every bucket that can rank above the exact cut
// is a candidate.  Rows that fail the check, or whose list overflowed, go to
// the exact fallback kernel (exact scores of every eligible bucket).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"

namespace lsa {

constexpr int kCandCap = 1024;       // candidates kept per (query, kv-head)
constexpr int kSampleStride = 16;    // every 16th bucket scored by the sample pass
constexpr int kSBins = 256;          // sample histogram bins over [-1.0625, 1.0625)
constexpr float kSBinLo = -1.0625f;
constexpr float kSBinW = 2.125f / kSBins;
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
    uint32_t* hist = reinterpret_cast<uint32_t*>(mcnt + 2 * kPassCols);       // sample: [qpt][256]; full: [qpt]

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
    float tau[2];
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
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int c0 = kk * 16 + 2 * tq;
            af[kk][hh] = rowok[hh] ? *reinterpret_cast<const uint32_t*>(yp + c0) : 0u;
            af[kk][hh + 2] = rowok[hh] ? *reinterpret_cast<const uint32_t*>(yp + c0 + 8) : 0u;
        }
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
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float v[4] = {acc[j][0], acc[j][1], acc[j][2], acc[j][3]};
            for (int off = 4; off < 4 * G; off <<= 1)
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = fmaxf(v[i], __shfl_xor_sync(0xffffffffu, v[i], off));
            if ((g % G) != 0) continue;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                if (!rowok[hh]) continue;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cl = j * 8 + 2 * tq + e;
                    const int64_t vc = v0 + cl;
                    const float s = v[2 * hh + e];
                    if (SAMPLE) {
                        if (vc * kSampleStride < ncol[hh] && (int64_t)mminlr[buf * kPassCols + cl] <= lim[hh]) {
                            int bin = __float2int_rd((s - kSBinLo) * (1.0f / kSBinW));
                            bin = bin < 0 ? 0 : (bin >= kSBins ? kSBins - 1 : bin);
                            atomicAdd(&hist[qloc[hh] * kSBins + bin], (uint32_t)mcnt[buf * kPassCols + cl]);
                        }
                    } else if (s >= tau[hh] && vc < ncol[hh]) {
                        const uint32_t slot = atomicAdd(&hist[qloc[hh]], 1u);
                        if (slot < (uint32_t)kCandCap) {
                            a.cand_col[row[hh] * kCandCap + slot] = (int32_t)vc;
                            a.cand_s[row[hh] * kCandCap + slot] = s;
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
            float t = -CUDART_INF_F;
            long long cum = 0;
            for (int b = kSBins - 1; b >= 0; --b) {
                cum += (long long)hist[tid * kSBins + b] * kSampleStride;
                if (cum >= (long long)kOversample * a.k) { t = kSBinLo + b * kSBinW; break; }
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

struct ResWarp {
    double ex[kCandCap];      // exact scores
    int32_t col[kCandCap];    // bucket ids; later packed (id << 5 | taken)
    int32_t w[kCandCap];      // key weights; later taken counts (negative = tied)
    uint32_t hist[256];
    uint16_t ylat[8 * kDL];
};

__device__ __forceinline__ unsigned long long order_key_d(double s) {
    s = s + 0.0;
    const unsigned long long u = (unsigned long long)__double_as_longlong(s);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ int weight_of(const ResolveArgs& a, int h, int64_t b, int64_t lim) {
    const int64_t hb = (int64_t)h * a.cap_buckets + b;
    if ((int64_t)a.maxpos[hb] <= lim) return a.cnt_lr[hb];
    const int32_t* off = a.offsets + (int64_t)h * (a.cap_buckets + 1);
    const int32_t* mem = a.members + (int64_t)h * a.cap_units;
    int w = 0;
    for (int32_t m = off[b]; m < off[b + 1]; ++m) {
        const int64_t j = mem[m];
        for (int64_t p = j * kPool; p < j * kPool + kPool && p < a.T_built; ++p)
            if (p >= a.S && p <= lim) ++w;
    }
    return w;
}

__device__ void emit_keys(const ResolveArgs& a, int h, int64_t b, int tk, int64_t lim, int32_t* out) {
    const int32_t* off = a.offsets + (int64_t)h * (a.cap_buckets + 1);
    const int32_t* mem = a.members + (int64_t)h * a.cap_units;
    int o = 0;
    for (int32_t m = off[b]; m < off[b + 1] && o < tk; ++m) {
        const int64_t j = mem[m];
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
    const int slot = atomicAdd(a.ovf_count, 1);
    if (slot < a.ovf_cap) a.ovf_rows[slot] = (int32_t)row;
    else raise_device_error(kErrSelectOverflow);
}

__global__ void __launch_bounds__(32 * kResWarps) flat_resolve_kernel(ResolveArgs a) {
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
    const int ng = a.agg ? a.G : 1;
    const uint16_t* ysrc = a.agg ? a.Y + (q * (int64_t)a.hkv * a.G + (int64_t)h * a.G) * kDL
                                 : a.Y + row * kDL;
    for (int i = lane; i < ng * kDL; i += 32) sw.ylat[i] = ysrc[i];
    __syncwarp();

    // eligible candidates, exact weights and scores
    const int64_t hb0 = (int64_t)h * a.cap_buckets;
    int m = 0;
    long long whi = 0, wtot = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        bool el = false;
        int col = 0, wgt = 0;
        float s = 0.f;
        if (i < n) {
            col = a.cand_col[row * kCandCap + i];
            s = a.cand_s[row * kCandCap + i];
            el = (int64_t)a.minlr[hb0 + col] <= lim;
        }
        if (el) {
            wgt = weight_of(a, h, col, lim);
            wtot += wgt;
            if (s >= tau + 2.0f * kScoreErr) whi += wgt;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, el);
        const int pos = m + __popc(bal & ((1u << lane) - 1u));
        if (el) {
            sw.col[pos] = col;
            sw.w[pos] = wgt;
            sw.ex[pos] = exact_row(sw.ylat, ng, a.cent + (hb0 + col) * kDL);
        }
        m += __popc(bal);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        whi += __shfl_xor_sync(0xffffffffu, whi, off);
        wtot += __shfl_xor_sync(0xffffffffu, wtot, off);
    }
    // tau = -inf means every eligible bucket is in the list
    if (tau > -CUDART_INF_F && whi < a.k) {
        if (lane == 0) push_fallback(a, row);
        return;
    }
    __syncwarp();

    if (wtot > a.k) {
        // weighted radix select on the exact scores (8 digits of 8 bits)
        unsigned long long prefix = 0;
        long long above = 0;
        for (int pass = 0; pass < 8; ++pass) {
            const int shift = 56 - 8 * pass;
            for (int i = lane; i < 256; i += 32) sw.hist[i] = 0u;
            __syncwarp();
            for (int i = lane; i < m; i += 32) {
                const unsigned long long key = order_key_d(sw.ex[i]);
                if (pass > 0 && (key >> (shift + 8)) != (prefix >> (shift + 8))) continue;
                atomicAdd(&sw.hist[(key >> shift) & 255ull], (unsigned)sw.w[i]);
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
            if (hitm == 0u) {  // cannot happen while the weights above the prefix reach k
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
            prefix |= (unsigned long long)dig << shift;
            __syncwarp();
        }
        // taken counts: above the cut fully, below not at all, ties pending
        for (int i = lane; i < m; i += 32) {
            const unsigned long long key = order_key_d(sw.ex[i]);
            sw.w[i] = key > prefix ? sw.w[i] : (key == prefix ? -sw.w[i] : 0);
        }
        __syncwarp();
        // ties at the cut: lowest bucket ids first
        long long need = a.k - above;
        while (need > 0) {
            int best = 0x7FFFFFFF, bi = -1;
            for (int i = lane; i < m; i += 32)
                if (sw.w[i] < 0 && sw.col[i] < best) { best = sw.col[i]; bi = i; }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const int ob = __shfl_xor_sync(0xffffffffu, best, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (ob < best) { best = ob; bi = oi; }
            }
            if (bi < 0) break;
            const int wv = -sw.w[bi];
            const int tk = wv < need ? wv : (int)need;
            __syncwarp();
            if (lane == 0) sw.w[bi] = tk;
            need -= tk;
            __syncwarp();
        }
        for (int i = lane; i < m; i += 32)
            if (sw.w[i] < 0) sw.w[i] = 0;
        __syncwarp();
    }
    // chosen buckets packed (id << 5 | taken), compacted, sorted by id
    int nsel = 0;
    for (int base = 0; base < m; base += 32) {
        const int i = base + lane;
        const int tk = i < m ? sw.w[i] : 0;
        const int col = i < m ? sw.col[i] : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, tk > 0);
        __syncwarp();
        if (tk > 0) sw.col[nsel + __popc(bal & ((1u << lane) - 1u))] = (col << 5) | tk;
        nsel += __popc(bal);
        __syncwarp();
    }
    int P = 1;
    while (P < nsel) P <<= 1;
    for (int i = nsel + lane; i < P; i += 32) sw.col[i] = 0x7FFFFFFF;
    __syncwarp();
    for (int k2 = 2; k2 <= P; k2 <<= 1) {
        for (int j = k2 >> 1; j > 0; j >>= 1) {
            for (int i = lane; i < P; i += 32) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const int x = sw.col[i], y = sw.col[ixj];
                    if ((x > y) == ((i & k2) == 0)) { sw.col[i] = y; sw.col[ixj] = x; }
                }
            }
            __syncwarp();
        }
    }
    // emit keys in ascending bucket id
    int run = 0;
    for (int base = 0; base < nsel; base += 32) {
        const int i = base + lane;
        const int pk = i < nsel ? sw.col[i] : 0;
        const int tk = i < nsel ? (pk & 31) : 0;
        int incl = tk;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (tk > 0) emit_keys(a, h, pk >> 5, tk, lim, out + a.S + run + incl - tk);
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int i = run + lane; i < a.k; i += 32) out[a.S + i] = -1;
}

// ------------------------------------------------------------ host side

lsa_status launch_flat(const PassArgs& pa, const ResolveArgs& ra, cudaStream_t st) {
    const int G = pa.agg ? pa.G : 1;
    const int qpt = 64 / G;
    dim3 grid((unsigned)ceil_div<int64_t>(pa.nqc, qpt), (unsigned)pa.hkv);
    const size_t base = 2 * kPassCols * kDL * 2 + 4 * kPassCols * 4;
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
