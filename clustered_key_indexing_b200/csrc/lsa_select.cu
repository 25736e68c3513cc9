// lsa_select.cu -- query scoring, long-range selection and index assembly of
// the LSA path on sm_100a [essay "《卡片柜》——当注意力学会先查目录再翻书",
// ch. 3 (flat search, sinks, window) and ch. 4 (tree beam search); ch. 5 for
// the native max-over-heads score].
//
// Flat search runs in three kernels per chunk of query positions:
//   score_kernel    bf16 tensor-core contraction (mma.sync m16n8k16, fp32
//                   accumulate) of query latents against centroid tiles;
//   select_kernel   one CTA per (query, kv-head): weighted histogram of the
//                   fp32 scores locates the k-th key's score bin, the band of
//                   candidates at or above the bin below it is rescored
//                   exactly in fp64, a weighted radix select on the exact
//                   scores finds the cut (score desc, bucket id asc), and the
//                   chosen buckets' keys are written in ascending bucket id;
//   select_fallback for rows whose candidate band overflows shared memory:
//                   exact scores of every eligible bucket in a global slot,
//                   same radix select.
// Tree search is a mode of select_kernel: beam descent over the node
// centroids with exact scores, then the same fill over the final leaves.
//
// Exactness: the fp32 scores only steer which buckets are rescored.  Their
// error is below 64 * 2^-23 * |y||c| < 1e-5; a histogram bin is 1.04e-3 wide,
// so every bucket whose exact score can reach the cut lies in the two bins
// kept, and the decision itself is taken on exact fp64 scores.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"

namespace lsa {

// --------------------------------------------------------------- scoring

constexpr int kScoreCols = 128;  // centroid columns per CTA tile
constexpr int kScoreRows = 64;   // MMA rows per CTA (4 warps x 16)

struct ScoreArgs {
    const uint16_t* Y;    // chunk query latents: [nqc, hkv, 64] (mean) / [nqc, hq, 64] (native)
    const uint16_t* cent; // [hkv, cap_buckets, 64]
    int64_t cap_buckets;
    int64_t NB;
    int64_t nqc;
    int64_t t_first;
    int32_t W, hkv, G, agg;
    float* S;             // [nqc * hkv, ld]
    int64_t ld;
};

// Columns (bucket slots) that can hold an eligible bucket for query t: only
// blocks that start at or before t - W.
__host__ __device__ __forceinline__ int64_t flat_ncol(int64_t t, int32_t W, int64_t NB) {
    const int64_t lim = t - W;
    if (lim < 0) return 0;
    const int64_t n = (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1);
    return n < NB ? n : NB;
}

__global__ void __launch_bounds__(128) score_kernel(ScoreArgs a) {
    __shared__ __align__(128) uint16_t ctile[kScoreCols * kDL];  // 16 KB, 16B-chunk swizzled
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int h = blockIdx.z;
    const int G = a.agg ? a.G : 1;
    const int64_t n0 = (int64_t)blockIdx.x * kScoreCols;
    const int64_t qrow0 = (int64_t)blockIdx.y * (kScoreRows / G);  // first query of the tile
    if (qrow0 >= a.nqc) return;
    const int64_t qlast = min(a.nqc - 1, qrow0 + kScoreRows / G - 1);
    if (n0 >= flat_ncol(a.t_first + qlast, a.W, a.NB)) return;

    // centroid tile -> shared (chunk c of row n at position c ^ (n & 7))
    const uint16_t* cb = a.cent + ((int64_t)h * a.cap_buckets + n0) * kDL;
#pragma unroll
    for (int i = 0; i < (kScoreCols * 8) / 128; ++i) {
        const int idx = tid + 128 * i;
        const int n = idx >> 3, c = idx & 7;
        const bool ok = n0 + n < a.NB;
        cp_async_16(smem_u32(ctile + n * kDL + ((c ^ (n & 7)) << 3)),
                    ok ? (const void*)(cb + (int64_t)n * kDL + c * 8) : (const void*)cb, ok ? 16 : 0);
    }
    cp_async_commit();

    // A fragments straight from global: MMA row r of this warp
    const int g = lane >> 2, tq = lane & 3;
    uint32_t af[4][4];
    const uint16_t* rowp[2];
    bool rowok[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int r = w * 16 + g + 8 * hh;
        const int64_t q = qrow0 + r / G;
        rowok[hh] = q < a.nqc;
        const int64_t yrow = a.agg ? (q * (int64_t)a.hkv * G + (int64_t)h * G + r % G)
                                   : (q * (int64_t)a.hkv + h);
        rowp[hh] = a.Y + (rowok[hh] ? yrow : 0) * kDL;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const int c0 = kk * 16 + 2 * tq;
        af[kk][0] = rowok[0] ? *reinterpret_cast<const uint32_t*>(rowp[0] + c0) : 0u;
        af[kk][1] = rowok[1] ? *reinterpret_cast<const uint32_t*>(rowp[1] + c0) : 0u;
        af[kk][2] = rowok[0] ? *reinterpret_cast<const uint32_t*>(rowp[0] + c0 + 8) : 0u;
        af[kk][3] = rowok[1] ? *reinterpret_cast<const uint32_t*>(rowp[1] + c0 + 8) : 0u;
    }
    cp_async_wait<0>();
    __syncthreads();

    float acc[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
    const uint32_t base = smem_u32(ctile);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) {
            // matrices: (n-tile 2jp, k lo), (2jp, k hi), (2jp+1, k lo), (2jp+1, k hi)
            const int mi = lane >> 3, ri = lane & 7;
            const int n = (2 * jp + (mi >> 1)) * 8 + ri;
            const int c = 2 * kk + (mi & 1);
            uint32_t b[4];
            ldsm_x4(b, base + (uint32_t)(n * kDL + ((c ^ (n & 7)) << 3)) * 2u);
            mma_16816(acc[2 * jp], af[kk], b[0], b[1]);
            mma_16816(acc[2 * jp + 1], af[kk], b[2], b[3]);
        }
    }

    // epilogue: rows g and g+8 of this warp (native: max over the G heads)
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float v[4] = {acc[j][0], acc[j][1], acc[j][2], acc[j][3]};
        for (int off = 4; off < 4 * G; off <<= 1)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = fmaxf(v[i], __shfl_xor_sync(0xffffffffu, v[i], off));
        if ((g % G) != 0) continue;
        const int64_t col = n0 + j * 8 + 2 * tq;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = w * 16 + g + 8 * hh;
            const int64_t q = qrow0 + r / G;
            if (q >= a.nqc) continue;
            float2* dst = reinterpret_cast<float2*>(a.S + (q * a.hkv + h) * a.ld + col);
            *dst = make_float2(v[2 * hh], v[2 * hh + 1]);
        }
    }
}

// ------------------------------------------------------------- selection

constexpr int kSelThreads = 128;
constexpr int kCap = 1024;      // candidates held in shared memory
constexpr int kBins = 2048;     // fp32 score bins over [-1.0625, 1.0625)
constexpr float kBinLo = -1.0625f;
constexpr float kBinScale = 2048.0f / 2.125f;

struct SelectArgs {
    const int32_t* offsets;
    const int32_t* members;
    const int32_t* cnt_lr;
    const int32_t* minlr;
    const int32_t* maxpos;
    const uint16_t* cent;
    int64_t cap_units, cap_buckets, NB, T_built;
    // tree (mode 1)
    const int32_t* tminlr;
    const uint16_t* tcent;
    int64_t n_nodes;
    int32_t levels, lstar, beam;
    int64_t level_n[LSA_MAX_LEVELS];
    int64_t level_off[LSA_MAX_LEVELS];
    int32_t hkv, G, agg, k, S, W, mode;
    const uint16_t* Y;     // chunk latents
    int64_t nqc, t_first;
    const float* scores;
    int64_t ld;
    int32_t* idx;          // chunk rows [nqc, hkv, S+k+W]
    int32_t* ovf_rows;
    int32_t* ovf_count;
    int32_t ovf_cap;
    double* fb_score;      // [n_slots, ld]
    int32_t* fb_w;         // [n_slots, ld]
};

__device__ __forceinline__ unsigned long long order_key(double s) {
    s = s + 0.0;  // -0 -> +0
    const unsigned long long u = (unsigned long long)__double_as_longlong(s);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ int score_bin(float s) {
    int b = __float2int_rd((s - kBinLo) * kBinScale);
    return b < 0 ? 0 : (b >= kBins ? kBins - 1 : b);
}

// Number of keys of bucket b (head h) in [S, lim].
__device__ int bucket_weight(const SelectArgs& a, int h, int64_t b, int64_t lim) {
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

// Write the first `tk` keys of bucket b in [S, lim], ascending.
__device__ void emit_bucket(const SelectArgs& a, int h, int64_t b, int tk, int64_t lim,
                            int32_t* out) {
    const int32_t* off = a.offsets + (int64_t)h * (a.cap_buckets + 1);
    const int32_t* mem = a.members + (int64_t)h * a.cap_units;
    int o = 0;
    for (int32_t m = off[b]; m < off[b + 1] && o < tk; ++m) {
        const int64_t j = mem[m];
        for (int64_t p = j * kPool; p < j * kPool + kPool && p < a.T_built && o < tk; ++p)
            if (p >= a.S && p <= lim) out[o++] = (int32_t)p;
    }
}

// Exact (fp64) score of node centroid c against the query latent(s) in shared memory.
__device__ __forceinline__ double exact_score(const uint16_t* ylat, int ng, const uint16_t* c) {
    double best = -CUDART_INF;
    for (int g = 0; g < ng; ++g) {
        const double v = dot_bf16_exact(ylat + g * kDL, c);
        best = v > best ? v : best;
    }
    return best;
}

// Block-wide exclusive scan of one int per thread; returns the prefix and the total.
__device__ __forceinline__ int block_exscan(int v, int* total, int* sh4) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    __syncthreads();
    if (lane == 31) sh4[wid] = x;
    __syncthreads();
    int before = 0, tot = 0;
    for (int i = 0; i < kSelThreads / 32; ++i) {
        if (i < wid) before += sh4[i];
        tot += sh4[i];
    }
    *total = tot;
    return before + x - v;
}

struct SelShared {
    unsigned long long hist[kBins];   // packed (count << 32 | weight)
    int cid[kCap];
    double csc[kCap];
    int cw[kCap];
    int ctk[kCap];
    uint16_t ylat[8 * kDL];
    int sh4[4];
    long long beam_id[16];
    double beam_sc[16];
    int nbeam;
    int misc[8];
    unsigned long long thr;
};

// Weighted radix select on exact scores of n candidates (id order) with
// total weight > k: taken count per candidate so that exactly k keys are
// taken from the best (score desc, id asc).  Candidate data via accessors.
template <typename GetS, typename GetW, typename SetTk>
__device__ void radix_fill(int64_t n, int k, GetS gs, GetW gw, SetTk st, SelShared& sh) {
    const int tid = threadIdx.x, lane = tid & 31;
    unsigned int* h256 = reinterpret_cast<unsigned int*>(sh.hist);
    unsigned long long prefix = 0;
    long long above = 0;
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = tid; i < 256; i += kSelThreads) h256[i] = 0;
        __syncthreads();
        for (int64_t i = tid; i < n; i += kSelThreads) {
            const int w = gw(i);
            if (w <= 0) continue;
            const unsigned long long key = order_key(gs(i));
            if (pass > 0 && (key >> (shift + 8)) != (prefix >> (shift + 8))) continue;
            atomicAdd(&h256[(key >> shift) & 255ull], (unsigned)w);
        }
        __syncthreads();
        if (tid < 32) {
            // lane l holds digits 255-8l .. 248-8l (descending)
            long long s = 0;
            for (int d = 0; d < 8; ++d) s += h256[255 - 8 * lane - d];
            long long incl = s;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const long long excl = incl - s;
            const bool hit = above + incl >= k && above + excl < k;
            const unsigned mask = __ballot_sync(0xffffffffu, hit);
            const int src = __ffs(mask) - 1;
            if (lane == src) {
                long long cum = above + excl;
                int dig = 255 - 8 * lane;
                for (int d = 0; d < 8; ++d) {
                    const int dd = 255 - 8 * lane - d;
                    if (cum + h256[dd] >= k) { dig = dd; break; }
                    cum += h256[dd];
                }
                sh.misc[0] = dig;
                reinterpret_cast<long long*>(sh.misc)[1] = cum;  // weight strictly above
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)sh.misc[0] << shift;
        above = reinterpret_cast<long long*>(sh.misc)[1];
        __syncthreads();
    }
    // ties at the cut: lowest ids first
    const long long need = k - above;
    long long run = 0;
    const int64_t per = (n + kSelThreads - 1) / kSelThreads;
    const int64_t i0 = tid * per, i1 = min(n, i0 + per);
    int mine = 0;
    for (int64_t i = i0; i < i1; ++i)
        if (gw(i) > 0 && order_key(gs(i)) == prefix) mine += gw(i);
    int tot;
    run = block_exscan(mine, &tot, sh.sh4);
    for (int64_t i = i0; i < i1; ++i) {
        const int w = gw(i);
        int tk = 0;
        if (w > 0) {
            const unsigned long long key = order_key(gs(i));
            if (key > prefix) {
                tk = w;
            } else if (key == prefix) {
                if (run + w <= need) tk = w;
                else if (run < need) tk = (int)(need - run);
                run += w;
            }
        }
        st(i, tk);
    }
    __syncthreads();
}

// Row bookkeeping shared by the kernels.
struct RowInfo {
    int64_t q, t, lim;
    int h;
    int32_t* out;
};

__device__ __forceinline__ RowInfo row_info(const SelectArgs& a, int64_t row) {
    RowInfo r;
    r.q = row / a.hkv;
    r.h = (int)(row % a.hkv);
    r.t = a.t_first + r.q;
    r.lim = r.t - a.W;
    r.out = a.idx + row * (int64_t)(a.S + a.k + a.W);
    return r;
}

__device__ void write_sinks_window(const SelectArgs& a, const RowInfo& r) {
    for (int i = threadIdx.x; i < a.S; i += kSelThreads) r.out[i] = (i <= r.t) ? i : -1;
    const int64_t w0 = max((int64_t)a.S, r.t - a.W + 1);
    const int64_t nw = r.t >= a.S ? r.t - w0 + 1 : 0;
    for (int i = threadIdx.x; i < a.W; i += kSelThreads)
        r.out[a.S + a.k + i] = i < nw ? (int32_t)(w0 + i) : -1;
}

__device__ void load_latents(const SelectArgs& a, const RowInfo& r, SelShared& sh) {
    const int ng = a.agg ? a.G : 1;
    const uint16_t* src = a.agg ? a.Y + (r.q * (int64_t)a.hkv * a.G + (int64_t)r.h * a.G) * kDL
                                : a.Y + (r.q * (int64_t)a.hkv + r.h) * kDL;
    for (int i = threadIdx.x; i < ng * kDL; i += kSelThreads) sh.ylat[i] = src[i];
}

// Emit candidates (id order, taken counts in sh.ctk) to the long-range part.
__device__ void emit_candidates(const SelectArgs& a, const RowInfo& r, int n, SelShared& sh) {
    const int per = (n + kSelThreads - 1) / kSelThreads;
    const int i0 = threadIdx.x * per, i1 = min(n, i0 + per);
    int mine = 0;
    for (int i = i0; i < i1; ++i) mine += sh.ctk[i];
    int tot;
    int o = block_exscan(mine, &tot, sh.sh4);
    for (int i = i0; i < i1; ++i) {
        if (sh.ctk[i] > 0) emit_bucket(a, r.h, sh.cid[i], sh.ctk[i], r.lim, r.out + a.S + o);
        o += sh.ctk[i];
    }
    for (int i = tot + threadIdx.x; i < a.k; i += kSelThreads) r.out[a.S + i] = -1;
}

// Emit every eligible bucket of [0, ncol) with taken count tk(b) (id order).
template <typename TkOf>
__device__ void emit_range(const SelectArgs& a, const RowInfo& r, int64_t ncol, TkOf tkof,
                           SelShared& sh) {
    int64_t base = 0;
    constexpr int per = 8;
    for (int64_t c0 = 0; c0 < ncol; c0 += (int64_t)per * kSelThreads) {
        const int64_t b0 = c0 + (int64_t)threadIdx.x * per;
        int tk[per];
        int mine = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int64_t b = b0 + i;
            tk[i] = (b < ncol) ? tkof(b) : 0;
            mine += tk[i];
        }
        int tot;
        int o = block_exscan(mine, &tot, sh.sh4);
#pragma unroll
        for (int i = 0; i < per; ++i) {
            if (tk[i] > 0) emit_bucket(a, r.h, b0 + i, tk[i], r.lim, r.out + a.S + base + o);
            o += tk[i];
        }
        base += tot;
    }
    for (int64_t i = base + threadIdx.x; i < a.k; i += kSelThreads) r.out[a.S + i] = -1;
}

// Beam descent [essay ch. 4]: leaves end up as candidates (id order) in
// sh.cid / sh.csc / sh.cw; returns their count.
__device__ int tree_candidates(const SelectArgs& a, const RowInfo& r, SelShared& sh) {
    const int tid = threadIdx.x;
    const int ng = a.agg ? a.G : 1;
    const int64_t hn = (int64_t)r.h * a.n_nodes;
    const int top = a.levels - 1;
    if (tid == 0) {
        sh.nbeam = 0;
        if (top <= a.lstar) {
            sh.beam_id[0] = 0;
            sh.nbeam = 1;
        } else if ((int64_t)a.tminlr[hn + a.level_off[top]] <= r.lim) {
            sh.beam_id[0] = 0;
            sh.nbeam = 1;
        }
    }
    __syncthreads();
    int lvl = top;
    while (lvl > a.lstar && sh.nbeam > 0) {
        const int nb = sh.nbeam;
        const int64_t nl = a.level_n[lvl - 1];
        double sc = -CUDART_INF;
        long long node = -1;
        if (tid < 2 * nb) {
            const long long ch = 2 * sh.beam_id[tid >> 1] + (tid & 1);
            if (ch < nl) {
                const int64_t gi = hn + a.level_off[lvl - 1] + ch;
                if ((int64_t)a.tminlr[gi] <= r.lim) {
                    sc = exact_score(sh.ylat, ng, a.tcent + gi * kDL);
                    node = ch;
                }
            }
        }
        __syncthreads();
        if (tid < 16) { sh.beam_sc[tid] = sc; sh.beam_id[tid] = node; }
        __syncthreads();
        if (tid == 0) {
            // keep the best `beam` eligible children (score desc, index asc)
            double bs[16];
            long long bi[16];
            int m = 0;
            for (int i = 0; i < 2 * nb; ++i) {
                if (sh.beam_id[i] < 0) continue;
                int j = m++;
                while (j > 0 && (bs[j - 1] < sh.beam_sc[i] ||
                                 (bs[j - 1] == sh.beam_sc[i] && bi[j - 1] > sh.beam_id[i]))) {
                    bs[j] = bs[j - 1];
                    bi[j] = bi[j - 1];
                    --j;
                }
                bs[j] = sh.beam_sc[i];
                bi[j] = sh.beam_id[i];
            }
            const int keep = m < a.beam ? m : a.beam;
            // ascending node index for the next level / the leaf list
            for (int i = 1; i < keep; ++i)
                for (int j = i; j > 0 && bi[j - 1] > bi[j]; --j) {
                    long long t2 = bi[j]; bi[j] = bi[j - 1]; bi[j - 1] = t2;
                }
            for (int i = 0; i < keep; ++i) sh.beam_id[i] = bi[i];
            sh.nbeam = keep;
        }
        __syncthreads();
        --lvl;
    }
    // leaves below the final beam, ascending
    const int nb = sh.nbeam;
    const int64_t span = (int64_t)1 << a.lstar;
    int n = 0;
    for (int i = 0; i < nb; ++i) {
        const int64_t b0 = (top <= a.lstar) ? 0 : (int64_t)sh.beam_id[i] * span;
        const int64_t b1 = (top <= a.lstar) ? a.NB : min(a.NB, b0 + span);
        for (int64_t c0 = b0; c0 < b1; c0 += kSelThreads) {
            const int64_t b = c0 + tid;
            const bool el = b < b1 && (int64_t)a.minlr[(int64_t)r.h * a.cap_buckets + b] <= r.lim;
            const unsigned bal = __ballot_sync(0xffffffffu, el);
            int tot;
            const int o = block_exscan(el ? 1 : 0, &tot, sh.sh4);
            (void)bal;
            if (el && n + o < kCap) sh.cid[n + o] = (int)b;
            n += tot;
        }
    }
    __syncthreads();
    if (n > kCap) return n;
    for (int i = tid; i < n; i += kSelThreads) {
        const int64_t b = sh.cid[i];
        sh.csc[i] = exact_score(sh.ylat, ng, a.cent + ((int64_t)r.h * a.cap_buckets + b) * kDL);
        sh.cw[i] = bucket_weight(a, r.h, b, r.lim);
    }
    __syncthreads();
    return n;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
    __shared__ SelShared sh;
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    const RowInfo r = row_info(a, row);
    write_sinks_window(a, r);
    if (r.lim < a.S) {
        for (int i = tid; i < a.k; i += kSelThreads) r.out[a.S + i] = -1;
        return;
    }
    load_latents(a, r, sh);
    const int ng = a.agg ? a.G : 1;
    const int64_t hb0 = (int64_t)r.h * a.cap_buckets;

    if (a.mode == 1) {
        __syncthreads();
        const int n = tree_candidates(a, r, sh);
        if (n > kCap) {
            if (tid == 0) raise_device_error(kErrSelectOverflow);
            return;
        }
        long long totw = 0;
        for (int i = 0; i < n; ++i) totw += sh.cw[i];
        if (totw <= a.k) {
            for (int i = tid; i < n; i += kSelThreads) sh.ctk[i] = sh.cw[i];
            __syncthreads();
        } else {
            radix_fill(
                n, a.k, [&](int64_t i) { return sh.csc[i]; }, [&](int64_t i) { return sh.cw[i]; },
                [&](int64_t i, int tk) { sh.ctk[i] = tk; }, sh);
        }
        emit_candidates(a, r, n, sh);
        return;
    }

    // ---- flat: pass 1, weighted histogram of the fp32 scores
    const int64_t ncol = flat_ncol(r.t, a.W, a.NB);
    const float* srow = a.scores + row * a.ld;
    for (int i = tid; i < kBins; i += kSelThreads) sh.hist[i] = 0ull;
    __syncthreads();
    long long myw = 0;
    for (int64_t b = tid; b < ncol; b += kSelThreads) {
        if ((int64_t)a.minlr[hb0 + b] > r.lim) continue;
        const int w = bucket_weight(a, r.h, b, r.lim);
        myw += w;
        atomicAdd(&sh.hist[score_bin(srow[b])], (1ull << 32) | (unsigned long long)w);
    }
    // total weight
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) myw += __shfl_xor_sync(0xffffffffu, myw, off);
    __shared__ long long wsum[4];
    if ((tid & 31) == 0) wsum[tid >> 5] = myw;
    __syncthreads();
    const long long totw = wsum[0] + wsum[1] + wsum[2] + wsum[3];
    if (totw <= a.k) {
        emit_range(a, r, ncol,
                   [&](int64_t b) -> int {
                       return ((int64_t)a.minlr[hb0 + b] <= r.lim) ? bucket_weight(a, r.h, b, r.lim) : 0;
                   },
                   sh);
        return;
    }
    // cut bin: highest j with weight(bins >= j) >= k; keep bins >= j - 1
    if (tid < 32) {
        const int lane = tid;
        long long s = 0, c = 0;
        for (int d = 0; d < kBins / 32; ++d) {
            const unsigned long long v = sh.hist[kBins - 1 - (kBins / 32) * lane - d];
            s += (long long)(v & 0xffffffffull);
            c += (long long)(v >> 32);
        }
        long long incl = s;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const long long excl = incl - s;
        const unsigned mask = __ballot_sync(0xffffffffu, incl >= a.k && excl < a.k);
        const int src = __ffs(mask) - 1;
        if (lane == src) {
            long long cum = excl;
            int j = kBins - 1 - (kBins / 32) * lane;
            for (int d = 0; d < kBins / 32; ++d) {
                const int jj = kBins - 1 - (kBins / 32) * lane - d;
                cum += (long long)(sh.hist[jj] & 0xffffffffull);
                if (cum >= a.k) { j = jj; break; }
            }
            sh.misc[0] = j > 0 ? j - 1 : 0;
        }
    }
    __syncthreads();
    const int jt = sh.misc[0];
    // candidate count
    int cnt = 0;
    for (int i = jt + tid; i < kBins; i += kSelThreads) cnt += (int)(sh.hist[i] >> 32);
    int ncand;
    block_exscan(cnt, &ncand, sh.sh4);
    if (ncand > kCap) {
        if (tid == 0) {
            const int slot = atomicAdd(a.ovf_count, 1);
            if (slot < a.ovf_cap) a.ovf_rows[slot] = (int)row;
            else raise_device_error(kErrSelectOverflow);
        }
        return;
    }
    // pass 2: ordered compaction of the band, then exact rescoring
    int n = 0;
    for (int64_t c0 = 0; c0 < ncol; c0 += kSelThreads) {
        const int64_t b = c0 + tid;
        const bool el = b < ncol && (int64_t)a.minlr[hb0 + b] <= r.lim && score_bin(srow[b]) >= jt;
        int tot;
        const int o = block_exscan(el ? 1 : 0, &tot, sh.sh4);
        if (el) sh.cid[n + o] = (int)b;
        n += tot;
    }
    __syncthreads();
    for (int i = tid; i < n; i += kSelThreads) {
        const int64_t b = sh.cid[i];
        sh.csc[i] = exact_score(sh.ylat, ng, a.cent + (hb0 + b) * kDL);
        sh.cw[i] = bucket_weight(a, r.h, b, r.lim);
    }
    __syncthreads();
    radix_fill(
        n, a.k, [&](int64_t i) { return sh.csc[i]; }, [&](int64_t i) { return sh.cw[i]; },
        [&](int64_t i, int tk) { sh.ctk[i] = tk; }, sh);
    emit_candidates(a, r, n, sh);
}

// Rows whose candidate band overflowed: exact scores of every eligible
// bucket in a global slot (one per CTA), then the same radix fill.
__global__ void __launch_bounds__(kSelThreads) select_fallback_kernel(SelectArgs a) {
    __shared__ SelShared sh;
    const int tid = threadIdx.x;
    const int nrows = min(*a.ovf_count, a.ovf_cap);
    double* fs = a.fb_score + (int64_t)blockIdx.x * a.ld;
    int32_t* fw = a.fb_w + (int64_t)blockIdx.x * a.ld;
    for (int it = blockIdx.x; it < nrows; it += gridDim.x) {
        const int64_t row = a.ovf_rows[it];
        const RowInfo r = row_info(a, row);
        __syncthreads();
        load_latents(a, r, sh);
        __syncthreads();
        const int ng = a.agg ? a.G : 1;
        const int64_t hb0 = (int64_t)r.h * a.cap_buckets;
        const int64_t ncol = flat_ncol(r.t, a.W, a.NB);
        for (int64_t b = tid; b < ncol; b += kSelThreads) {
            const bool el = (int64_t)a.minlr[hb0 + b] <= r.lim;
            fw[b] = el ? bucket_weight(a, r.h, b, r.lim) : 0;
            fs[b] = el ? exact_score(sh.ylat, ng, a.cent + (hb0 + b) * kDL) : 0.0;
        }
        __syncthreads();
        // taken counts are written back into fw
        radix_fill(
            ncol, a.k, [&](int64_t i) { return fs[i]; }, [&](int64_t i) { return (int)fw[i]; },
            [&](int64_t i, int tk) { fw[i] = tk; }, sh);
        __syncthreads();
        emit_range(a, r, ncol, [&](int64_t b) -> int { return fw[b]; }, sh);
    }
}

// ------------------------------------------------------------ host side

struct SelectPlan {
    int64_t ld;        // score row stride (floats)
    int64_t chunk;     // query positions per chunk
    int32_t hy;        // latent rows per query
    int32_t fb_slots;
};

static SelectPlan plan_select(const lsa_cfg* cfg, int64_t nq, int32_t hq, int32_t hkv, int64_t NB) {
    SelectPlan p;
    p.ld = ceil_div<int64_t>(NB > 0 ? NB : 1, kScoreCols) * kScoreCols;
    p.hy = cfg->agg ? hq : hkv;
    const int64_t budget = (int64_t)512 << 20;  // score rows per chunk
    int64_t c = budget / (hkv * p.ld * (int64_t)sizeof(float));
    c = c / 64 * 64;
    if (c < 64) c = 64;
    if (c > nq) c = nq;
    if (c < 1) c = 1;
    p.chunk = c;
    p.fb_slots = 64;
    return p;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct SelectWs {
    uint16_t* Y;
    float* S;
    int32_t* ovf_rows;
    int32_t* ovf_count;
    double* fb_score;
    int32_t* fb_w;
    size_t bytes;
};

static SelectWs carve_select(const SelectPlan& p, int32_t hkv, int mode, char* base) {
    SelectWs w{};
    size_t o = 0;
    w.Y = (uint16_t*)(base + o); o += align256((size_t)p.chunk * p.hy * kDL * 2);
    if (mode == 0) {
        w.S = (float*)(base + o); o += align256((size_t)p.chunk * hkv * p.ld * 4);
        w.ovf_rows = (int32_t*)(base + o); o += align256((size_t)p.chunk * hkv * 4);
        w.ovf_count = (int32_t*)(base + o); o += 256;
        w.fb_score = (double*)(base + o); o += align256((size_t)p.fb_slots * p.ld * 8);
        w.fb_w = (int32_t*)(base + o); o += align256((size_t)p.fb_slots * p.ld * 4);
    }
    w.bytes = o;
    return w;
}

size_t select_ws_bytes(const lsa_cfg* cfg, int64_t nq, int32_t hq, int32_t hkv, int64_t NB) {
    const SelectPlan p = plan_select(cfg, nq, hq, hkv, NB);
    return carve_select(p, hkv, cfg->mode, nullptr).bytes;
}

lsa_status launch_query_latent(const uint16_t* Q, int64_t nq, int32_t hq, int32_t hkv,
                               const float* W, int agg, uint16_t* Y, cudaStream_t st);

static int lstar_of(const lsa_cfg* cfg) {
    int l = 0;
    while ((int64_t)cfg->beam * cfg->bucket_mean * ((int64_t)1 << l) < cfg->k && l < 62) ++l;
    return l;
}

lsa_status run_select(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq, const float* W_q,
                      const lsa_cache* c, const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                      uint16_t* Y_out, void* ws, size_t ws_bytes, cudaStream_t st) {
    const int32_t hkv = c->hkv;
    const int64_t NU = ceil_div<int64_t>(c->n_tokens, kPool);
    const int64_t NB = ceil_div<int64_t>(NU, kUnitsPerBlock) * kBucketsPerBlock;
    const SelectPlan p = plan_select(cfg, nq, hq, hkv, NB);
    const SelectWs w = carve_select(p, hkv, cfg->mode, (char*)ws);
    if (ws_bytes < w.bytes)
        return set_error(LSA_ENOSPACE, "lsa_select: workspace %zu bytes < %zu needed", ws_bytes, w.bytes);
    const int row_len = cfg->sinks + cfg->k + cfg->window;

    SelectArgs a{};
    a.offsets = c->offsets; a.members = c->members; a.cnt_lr = c->cnt_lr; a.minlr = c->minlr;
    a.maxpos = c->maxpos; a.cent = c->cent; a.cap_units = c->cap_units; a.cap_buckets = c->cap_buckets;
    a.NB = NB; a.T_built = c->n_tokens;
    a.hkv = hkv; a.G = hq / hkv; a.agg = cfg->agg; a.k = cfg->k; a.S = cfg->sinks; a.W = cfg->window;
    a.mode = cfg->mode;
    if (cfg->mode == 1) {
        a.tminlr = tree->minlr; a.tcent = tree->cent; a.n_nodes = tree->n_nodes;
        a.levels = tree->levels; a.beam = cfg->beam; a.lstar = lstar_of(cfg);
        for (int l = 0; l < tree->levels; ++l) { a.level_n[l] = tree->level_n[l]; a.level_off[l] = tree->level_off[l]; }
    }
    a.ld = p.ld;
    a.scores = w.S;
    a.ovf_rows = w.ovf_rows; a.ovf_count = w.ovf_count; a.ovf_cap = (int32_t)(p.chunk * hkv);
    a.fb_score = w.fb_score; a.fb_w = w.fb_w;

    for (int64_t c0 = 0; c0 < nq; c0 += p.chunk) {
        const int64_t nqc = (nq - c0) < p.chunk ? (nq - c0) : p.chunk;
        uint16_t* Y = Y_out ? Y_out + c0 * p.hy * kDL : w.Y;
        lsa_status s = launch_query_latent(Q + c0 * hq * kD, nqc, hq, hkv, W_q, cfg->agg, Y, st);
        if (s != LSA_OK) return s;
        a.Y = Y; a.nqc = nqc; a.t_first = t0 + c0; a.idx = idx + c0 * hkv * row_len;
        if (cfg->mode == 0) {
            ScoreArgs sa{};
            sa.Y = Y; sa.cent = c->cent; sa.cap_buckets = c->cap_buckets; sa.NB = NB; sa.nqc = nqc;
            sa.t_first = t0 + c0; sa.W = cfg->window; sa.hkv = hkv; sa.G = hq / hkv; sa.agg = cfg->agg;
            sa.S = w.S; sa.ld = p.ld;
            const int64_t ncol = flat_ncol(t0 + c0 + nqc - 1, cfg->window, NB);
            if (ncol > 0) {
                const int qpt = kScoreRows / (cfg->agg ? hq / hkv : 1);
                dim3 grid((unsigned)ceil_div<int64_t>(ncol, kScoreCols),
                          (unsigned)ceil_div<int64_t>(nqc, qpt), (unsigned)hkv);
                score_kernel<<<grid, 128, 0, st>>>(sa);
                if ((s = check_launch("score_kernel")) != LSA_OK) return s;
            }
            if (cudaMemsetAsync(w.ovf_count, 0, sizeof(int32_t), st) != cudaSuccess)
                return set_error(LSA_ECUDA, "lsa_select: memset failed");
        }
        select_kernel<<<(unsigned)(nqc * hkv), kSelThreads, 0, st>>>(a);
        if ((s = check_launch("select_kernel")) != LSA_OK) return s;
        if (cfg->mode == 0) {
            select_fallback_kernel<<<(unsigned)p.fb_slots, kSelThreads, 0, st>>>(a);
            if ((s = check_launch("select_fallback_kernel")) != LSA_OK) return s;
        }
    }
    return LSA_OK;
}

}  // namespace lsa
