// lsa_select.cu -- long-range selection and index assembly of the LSA path
// on sm_100a [essay "《卡片柜》——当注意力学会先查目录再翻书", ch. 3 (flat
// search, sinks, window) and ch. 4 (tree beam search); ch. 5 for the native
// max-over-heads score].
//
//   tree_warp_kernel        tree search, one warp per (query, kv-head): beam
//                           descent over the node centroids with exact fp64
//                           scores, then exact scores of the leaves below the
//                           final beam and a weighted radix fill of k keys;
//   select_fallback_kernel  the exact flat search for the rows the flat
//                           resolve flags (band below tau, or a candidate
//                           list that overflowed): exact scores of every
//                           eligible bucket in a global slot, the same fill;
//   run_select              the selection driver: query latents, then per
//                           chunk of query positions the flat kernels of
//                           lsa_flat.cuh (tcgen05 scores, candidates, resolve)
//                           or the tree kernel, then the fallback.
// The record modes of the resolve and fallback kernels write a shard's taken
// buckets with their exact scores instead of index rows (sequence sharding).
//
// Exactness: every ranking decision is taken on exact fp64 scores (score
// desc, bucket id asc); fp32 tensor-core scores only steer which buckets are
// rescored (lsa_flat.cuh states the bound).
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_flat.cuh"
#include "lsa_mma.cuh"

namespace lsa {

// Columns (bucket slots) that can hold an eligible bucket for query t: only
// blocks that start at or before t - W.
__host__ __device__ __forceinline__ int64_t flat_ncol(int64_t t, int32_t W, int64_t NB) {
    const int64_t lim = t - W;
    if (lim < 0) return 0;
    const int64_t n = (int64_t)kBucketsPerBlock * (lim / kBlockKeys + 1);
    return n < NB ? n : NB;
}

// ------------------------------------------------------------- selection

constexpr int kSelThreads = 128;
constexpr int kCap = 1024;      // candidates held in shared memory (fallback, decode resolve); decode keep slots per row chunk

struct SelectArgs {
    const int32_t* offsets;
    const int32_t* members;
    const int32_t* cnt_lr;
    const int32_t* minlr;
    const int32_t* maxpos;
    const uint16_t* cent;
    const uint8_t* cent8;  // decode, flat search: FP8 centroids scored instead of cent (NULL: bf16)
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
    // decode rows: row = request * hkv + head is also the cache head, and
    // each request has its own position
    int32_t decode;
    int64_t pos[LSA_MAX_BATCH];
    // candidate-record mode of the flat fallback (sequence-sharded selection)
    ShardRec* rec;
    int32_t* rec_n;
    int32_t rec_cap;
    int64_t id_base;
};

__device__ __forceinline__ unsigned long long order_key(double s) {
    s = s + 0.0;  // -0 -> +0
    const unsigned long long u = (unsigned long long)__double_as_longlong(s);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
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
    // 8-byte members first: every field below stays naturally aligned
    double csc[kCap];
    long long above;                  // radix select: weight strictly above the prefix
    unsigned int hist[256];           // radix select: weight per digit
    int cid[kCap];
    int cw[kCap];
    int ctk[kCap];
    int sh4[kSelThreads / 32];
    int misc[4];
    uint16_t ylat[8 * kDL];
};

// Weighted radix select on exact scores of n candidates (id order) with
// total weight > k: taken count per candidate so that exactly k keys are
// taken from the best (score desc, id asc).  Candidate data via accessors.
template <typename GetS, typename GetW, typename SetTk>
__device__ void radix_fill(int64_t n, int k, GetS gs, GetW gw, SetTk st, SelShared& sh) {
    const int tid = threadIdx.x, lane = tid & 31;
    unsigned int* h256 = sh.hist;
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
                sh.above = cum;  // weight strictly above the chosen digit
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)sh.misc[0] << shift;
        above = sh.above;
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
    if (a.decode) {
        r.q = 0;
        r.h = (int)row;
        r.t = a.pos[row / a.hkv];
    } else {
        r.q = row / a.hkv;
        r.h = (int)(row % a.hkv);
        r.t = a.t_first + r.q;
    }
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

// Tree search [essay ch. 4]: one warp per (query, kv-head).
//   descent: from the root down to level L*, the children of the beam are
//     scored exactly (fp64, ascending dims, one child per lane) and the best
//     `beam` eligible ones kept (score desc, node index asc), then ordered by
//     node index;
//   leaves: the eligible buckets below the final beam, ascending id, scored
//     exactly, weighted by their keys in [S, t - W];
//   fill: exactly k keys from the best (score desc, id asc) by a warp radix
//     select on the fp64 order keys (8 digits of 8 bits); at the cut the
//     lowest ids first; keys emitted in ascending bucket id.
constexpr int kTreeWarps = 4;

// Leaves a row can reach: at most beam subtrees of 2^L* buckets.
static inline int tree_max_cands(int beam, int lstar) { return beam << lstar; }

// Exponent spread of the nonzero bf16 values among `b` (biased exponents,
// subnormals counted as exponent 1): returns (max << 8) | min, or 0 if all
// are zero.
__device__ __forceinline__ uint32_t bf16_exp_span(uint32_t lo_bits, uint32_t hi_bits) {
    uint32_t mn = 255u, mx = 0u;
    const uint32_t v[2] = {lo_bits, hi_bits};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t b = v[i] & 0xFFFFu;
        if (b & 0x7FFFu) {
            const uint32_t e = max(1u, (b >> 7) & 0xFFu);
            mn = min(mn, e);
            mx = max(mx, e);
        }
    }
    return mx ? (mx << 8) | mn : 0u;
}

// Exactness test of a dot product of two bf16 vectors in fp64: with every
// product exact (8-bit significands) and the spreads of the two vectors'
// nonzero exponents summing to at most 30, every partial sum is an integer
// multiple of the smallest product quantum below 2^53 of them, so any order
// of summation gives the exact sum -- the ascending sequential sum included.
__device__ __forceinline__ int exp_range(uint32_t span) { return span ? (int)(span >> 8) - (int)(span & 0xFFu) : 0; }
__device__ __forceinline__ uint32_t span_merge(uint32_t a, uint32_t b) {
    if (!a) return b;
    if (!b) return a;
    return (max(a >> 8, b >> 8) << 8) | min(a & 0xFFu, b & 0xFFu);
}

__host__ __device__ inline size_t tree_warp_bytes(int maxn) {
    return (((size_t)maxn * 16 + 256 * 4 + 8 * kDL * 2) + 15) & ~(size_t)15;
}

__global__ void __launch_bounds__(32 * kTreeWarps, 4) tree_warp_kernel(SelectArgs a, int64_t nrows, int maxn) {
    extern __shared__ __align__(16) uint8_t tsm[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kTreeWarps + wid;
    if (row >= nrows) return;
    uint8_t* base = tsm + (size_t)wid * tree_warp_bytes(maxn);
    double* sc = reinterpret_cast<double*>(base);          // exact leaf scores
    int* id = reinterpret_cast<int*>(sc + maxn);          // leaf bucket ids, ascending
    int* wt = id + maxn;                                  // key weights, then taken counts
    uint32_t* hist = reinterpret_cast<uint32_t*>(wt + maxn);
    uint16_t* ylat = reinterpret_cast<uint16_t*>(hist + 256);
    const RowInfo r = row_info(a, row);

    for (int i = lane; i < a.S; i += 32) r.out[i] = (i <= r.t) ? i : -1;
    const int64_t w0 = max((int64_t)a.S, r.t - a.W + 1);
    const int64_t nw = r.t >= a.S ? r.t - w0 + 1 : 0;
    for (int i = lane; i < a.W; i += 32) r.out[a.S + a.k + i] = i < nw ? (int32_t)(w0 + i) : -1;
    if (r.lim < a.S) {
        for (int i = lane; i < a.k; i += 32) r.out[a.S + i] = -1;
        return;
    }
    const int ng = a.agg ? a.G : 1;
    const uint16_t* ysrc = a.agg ? a.Y + (r.q * (int64_t)a.hkv * a.G + (int64_t)r.h * a.G) * kDL
                                 : a.Y + (r.q * (int64_t)a.hkv + r.h) * kDL;
    for (int i = lane; i < ng * kDL; i += 32) ylat[i] = ysrc[i];
    __syncwarp();
    // the widest exponent spread over the row's latent(s), for the exactness test
    int yrange = 0;
    for (int g = 0; g < ng; ++g) {
        uint32_t sp = bf16_exp_span(ylat[g * kDL + 2 * lane], ylat[g * kDL + 2 * lane + 1]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sp = span_merge(sp, __shfl_xor_sync(0xffffffffu, sp, off));
        yrange = max(yrange, exp_range(sp));
    }

    // descent: lane i < nbeam holds beam node i (ascending index)
    const int64_t hn = (int64_t)r.h * a.n_nodes;
    const int top = a.levels - 1;
    int nbeam = 0;
    long long mybeam = -1;
    if (top <= a.lstar || (int64_t)a.tminlr[hn + a.level_off[top]] <= r.lim) {
        nbeam = 1;
        mybeam = lane == 0 ? 0 : -1;
    }
    for (int lvl = top; lvl > a.lstar && nbeam > 0; --lvl) {
        const int64_t nl = a.level_n[lvl - 1];
        const int nc = 2 * nbeam;  // children of the beam (<= 16)
        // exact scores of the children, 8 lanes per child (8 dimensions each,
        // combined in a fixed tree), four children per pass; a child whose
        // vectors fail the exactness test is scored sequentially instead
        double s_all = -CUDART_INF;  // lane j < nc: child j's score
        for (int p0 = 0; p0 < nc; p0 += 4) {
            const int j = p0 + (lane >> 3), part = lane & 7;
            const long long parj = __shfl_sync(0xffffffffu, mybeam, (j >> 1) & 31);
            const long long chj = 2 * parj + (j & 1);
            const bool act = j < nc && chj < nl;
            const int64_t gj = hn + a.level_off[lvl - 1] + (act ? chj : 0);
            const uint4 cv = act ? __ldg(reinterpret_cast<const uint4*>(a.tcent + gj * kDL) + part)
                                 : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
            uint32_t sp = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) sp = span_merge(sp, bf16_exp_span(cw[e] & 0xFFFFu, cw[e] >> 16));
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) sp = span_merge(sp, __shfl_xor_sync(0xffffffffu, sp, off));
            double best = -CUDART_INF;
            for (int g = 0; g < ng; ++g) {
                const uint16_t* y = ylat + g * kDL + 8 * part;
                double ps = 0.0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    ps = fma(bf16_to_f64(y[2 * e]), (double)__uint_as_float(cw[e] << 16), ps);
                    ps = fma(bf16_to_f64(y[2 * e + 1]), (double)__uint_as_float(cw[e] & 0xFFFF0000u), ps);
                }
#pragma unroll
                for (int off = 1; off < 8; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
                best = ps > best ? ps : best;
            }
            if (act && part == 0 && yrange + exp_range(sp) > 30) best = exact_row(ylat, ng, a.tcent + gj * kDL);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const double v = __shfl_sync(0xffffffffu, best, 8 * q4);
                if (lane == p0 + q4) s_all = v;
            }
        }
        const long long par = __shfl_sync(0xffffffffu, mybeam, (lane >> 1) & 31);
        double s = -CUDART_INF;
        long long node = -1;
        if (lane < nc) {
            const long long ch = 2 * par + (lane & 1);
            if (ch < nl) {
                const int64_t gi = hn + a.level_off[lvl - 1] + ch;
                if ((int64_t)a.tminlr[gi] <= r.lim) {
                    s = s_all;
                    node = ch;
                }
            }
        }
        // rank among the eligible children (score desc, index asc)
        int rank = 0;
        for (int j = 0; j < nc; ++j) {
            const double sj = __shfl_sync(0xffffffffu, s, j);
            const long long nj = __shfl_sync(0xffffffffu, node, j);
            if (nj >= 0 && (sj > s || (sj == s && nj < node))) ++rank;
        }
        const bool keep = node >= 0 && rank < a.beam;
        const unsigned km = __ballot_sync(0xffffffffu, keep);
        // the kept nodes, ascending index, into lanes 0 .. popc(km) - 1
        int pos = 0;
        for (int j = 0; j < nc; ++j) {
            const long long nj = __shfl_sync(0xffffffffu, node, j);
            if (((km >> j) & 1u) && nj < node) ++pos;
        }
        long long nb_new = -1;
        for (int j = 0; j < nc; ++j) {
            const int pj = __shfl_sync(0xffffffffu, pos, j);
            const long long nj = __shfl_sync(0xffffffffu, node, j);
            if (((km >> j) & 1u) && pj == lane) nb_new = nj;
        }
        mybeam = nb_new;
        nbeam = __popc(km);
    }

    // leaves below the final beam (the whole cache when the tree is not
    // taller than L*), eligible ones in ascending id
    const int64_t span = (int64_t)1 << a.lstar;
    const int64_t hb0 = (int64_t)r.h * a.cap_buckets;
    int n = 0;
    for (int i = 0; i < nbeam; ++i) {
        const long long bnode = __shfl_sync(0xffffffffu, mybeam, i);
        const int64_t b0 = (top <= a.lstar) ? 0 : (int64_t)bnode * span;
        const int64_t b1 = (top <= a.lstar) ? a.NB : min(a.NB, b0 + span);
        for (int64_t c0 = b0; c0 < b1; c0 += 32) {
            const int64_t b = c0 + lane;
            const bool el = b < b1 && (int64_t)a.minlr[hb0 + b] <= r.lim;
            const unsigned bal = __ballot_sync(0xffffffffu, el);
            const int o = n + __popc(bal & ((1u << lane) - 1u));
            if (el && o < maxn) id[o] = (int)b;
            n += __popc(bal);
        }
    }
    if (n > maxn) {  // cannot happen: at most beam subtrees of 2^L* leaves
        if (lane == 0) raise_device_error(kErrSelectOverflow);
        return;
    }
    __syncwarp();
    long long totw = 0;
    // leaves four per lane at a time (i, i + 32, i + 64, i + 96): four
    // independent exact-score chains in flight
    for (int i0 = 0; i0 < n; i0 += 128) {
        const uint16_t* cp[4];
        int ii[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            ii[j] = i0 + lane + 32 * j;
            cp[j] = a.cent + (hb0 + (ii[j] < n ? id[ii[j]] : id[0])) * kDL;
        }
        double sv[4];
        exact_rows4(ylat, ng, cp, sv);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (ii[j] < n) {
                sc[ii[j]] = sv[j];
                wt[ii[j]] = bucket_weight(a, r.h, id[ii[j]], r.lim);
                totw += wt[ii[j]];
            }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) totw += __shfl_xor_sync(0xffffffffu, totw, off);
    __syncwarp();

    if (totw > a.k) {
        // weighted radix select: prefix = the order key of the k-th key,
        // above = the weight strictly above it
        unsigned long long prefix = 0ull;
        long long above = 0;
        for (int pass = 0; pass < 8; ++pass) {
            const int shift = 56 - 8 * pass;
            for (int i = lane; i < 256; i += 32) hist[i] = 0u;
            __syncwarp();
            for (int i = lane; i < n; i += 32) {
                const int w = wt[i];
                if (w <= 0) continue;
                const unsigned long long key = order_key(sc[i]);
                if (pass > 0 && (key >> (shift + 8)) != (prefix >> (shift + 8))) continue;
                atomicAdd(&hist[(key >> shift) & 255ull], (unsigned)w);
            }
            __syncwarp();
            long long ab = 0;
            const int dig = cut_bin(hist, a.k - above, &ab);
            if (dig < 0) {  // cannot happen while the weight above the prefix reaches k
                if (lane == 0) raise_device_error(kErrSelectOverflow);
                return;
            }
            above += ab;
            prefix |= (unsigned long long)dig << shift;
            __syncwarp();
        }
        // taken counts: above the cut whole, at the cut lowest ids first
        const long long need = a.k - above;
        long long run = 0;
        for (int b0 = 0; b0 < n; b0 += 32) {
            const int i = b0 + lane;
            const int w = i < n ? wt[i] : 0;
            const unsigned long long key = i < n ? order_key(sc[i]) : 0ull;
            const long long eq = (w > 0 && key == prefix) ? w : 0;
            long long incl = eq;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            int tk = 0;
            if (w > 0) {
                if (key > prefix) tk = w;
                else if (key == prefix) tk = (int)max(0LL, min((long long)w, need - (run + incl - eq)));
            }
            __syncwarp();
            if (i < n) wt[i] = tk;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncwarp();
    }
    // emit the taken keys in ascending bucket id
    int o = 0;
    for (int b0 = 0; b0 < n; b0 += 32) {
        const int i = b0 + lane;
        const int tk = i < n ? wt[i] : 0;
        int incl = tk;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (tk > 0) emit_bucket(a, r.h, id[i], tk, r.lim, r.out + a.S + o + incl - tk);
        o += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int i = o + lane; i < a.k; i += 32) r.out[a.S + i] = -1;
}

lsa_status launch_tree_select(const SelectArgs& a, int64_t nrows, cudaStream_t st) {
    const int maxn = tree_max_cands(a.beam, a.lstar);
    const size_t smem = (size_t)kTreeWarps * tree_warp_bytes(maxn);
    if (smem > 227 * 1024) return set_error(LSA_EUNSUPPORTED, "tree search: beam * 2^L* = %d leaves too many", maxn);
    cudaFuncSetAttribute(tree_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    {
        KTime kt_("tree_select_kernel", st);
        tree_warp_kernel<<<(unsigned)ceil_div<int64_t>(nrows, kTreeWarps), 32 * kTreeWarps, smem, st>>>(a, nrows,
                                                                                                       maxn);
    }
    return check_launch("tree_warp_kernel");
}

// Records (ascending id) of the buckets of [0, ncol) with taken count tk(b) >
// 0 and exact score sc(b), for the candidate-record mode.
template <typename TkOf, typename ScOf>
__device__ void emit_records(const SelectArgs& a, int64_t row, int64_t ncol, TkOf tkof, ScOf scof,
                             SelShared& sh) {
    ShardRec* rec = a.rec + row * (int64_t)a.rec_cap;
    int64_t base = 0;
    constexpr int per = 8;
    for (int64_t c0 = 0; c0 < ncol; c0 += (int64_t)per * kSelThreads) {
        const int64_t b0 = c0 + (int64_t)threadIdx.x * per;
        int mine = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) mine += (b0 + i < ncol && tkof(b0 + i) > 0) ? 1 : 0;
        int tot;
        int o = block_exscan(mine, &tot, sh.sh4);
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int64_t b = b0 + i;
            if (b < ncol && tkof(b) > 0) {
                if (base + o < a.rec_cap) rec[base + o] = ShardRec{(int32_t)(a.id_base + b), tkof(b), scof(b)};
                ++o;
            }
        }
        base += tot;
    }
    if (threadIdx.x == 0) {
        a.rec_n[row] = (int32_t)min(base, (int64_t)a.rec_cap);
        if (base > a.rec_cap) raise_device_error(kErrSelectOverflow);
    }
}

// Rows whose candidate band overflowed: exact scores of every eligible
// bucket in a global slot (one per CTA), then the same radix fill.  CANDS:
// the taken buckets as records instead of the index row.
template <bool CANDS>
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
        int myw = 0;
        for (int64_t b = tid; b < ncol; b += kSelThreads) {
            const bool el = (int64_t)a.minlr[hb0 + b] <= r.lim;
            fw[b] = el ? bucket_weight(a, r.h, b, r.lim) : 0;
            fs[b] = el ? exact_row(sh.ylat, ng, a.cent + (hb0 + b) * kDL) : 0.0;
            myw += fw[b];
        }
        int totw;
        block_exscan(myw, &totw, sh.sh4);
        __syncthreads();
        // taken counts are written back into fw (every eligible key when
        // there are no more than k of them)
        if (totw > a.k)
            radix_fill(
                ncol, a.k, [&](int64_t i) { return fs[i]; }, [&](int64_t i) { return (int)fw[i]; },
                [&](int64_t i, int tk) { fw[i] = tk; }, sh);
        __syncthreads();
        if constexpr (CANDS)
            emit_records(a, row, ncol, [&](int64_t b) -> int { return fw[b]; },
                         [&](int64_t b) -> double { return fs[b]; }, sh);
        else
            emit_range(a, r, ncol, [&](int64_t b) -> int { return fw[b]; }, sh);
    }
}

// ------------------------------------------------------------ host side

struct SelectPlan {
    int64_t ld;        // fallback slot stride (bucket slots, rounded up)
    int64_t chunk;     // query positions per chunk
    int32_t hy;        // latent rows per query
    int32_t fb_slots;
    int64_t ns_cap;    // sampled buckets per kv-head (every 8th)
    int64_t nb;        // buckets per kv-head (packed records)
};

// Query positions per flat-search chunk: the candidate kernel launches one CTA
// per (512 / G latent rows, kv-head), so a chunk of a multiple of
// num_sms / gcd(num_sms, hkv) CTA row blocks fills whole waves; candidate
// lists (kCandCap x 8 bytes per query and kv-head) stay within 2 GiB.
int64_t select_wave_rows(const lsa_cfg* cfg, int32_t hq, int32_t hkv) {
    const int64_t qpt = kCdRows / (cfg->agg ? hq / hkv : 1);
    int64_t g = num_sms(), x = hkv;
    while (x) { const int64_t y = g % x; g = x; x = y; }
    return qpt * (num_sms() / g);
}

int64_t select_chunk(const lsa_cfg* cfg, int32_t hq, int32_t hkv) {
    const int64_t wave = select_wave_rows(cfg, hq, hkv);
    const int64_t per_wave = wave * hkv * (int64_t)kCandCap * 8;
    int64_t m = ((int64_t)2 << 30) / per_wave;
    if (m < 1) m = 1;
    return wave * m;
}

static SelectPlan plan_select(const lsa_cfg* cfg, int64_t nq, int32_t hq, int32_t hkv, int64_t NB) {
    SelectPlan p;
    p.ld = ceil_div<int64_t>(NB > 0 ? NB : 1, 128) * 128;
    p.hy = cfg->agg ? hq : hkv;
    int64_t c = select_chunk(cfg, hq, hkv);
    if (c > nq) c = nq;
    if (c < 1) c = 1;
    p.chunk = c;
    p.fb_slots = 64;
    p.ns_cap = ceil_div<int64_t>(NB > 0 ? NB : 1, kSampleStride);
    p.nb = NB > 0 ? NB : 1;
    return p;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct SelectWs {
    uint16_t* Y;
    float* tau;
    int2* cand;
    int32_t* cand_n;
    int32_t* ovf_rows;
    int32_t* ovf_count;
    double* fb_score;
    int32_t* fb_w;
    uint16_t* cent_s;
    int4* meta;
    size_t bytes;
};

static SelectWs carve_select(const SelectPlan& p, int32_t hkv, int mode, char* base) {
    SelectWs w{};
    size_t o = 0;
    const size_t rows = (size_t)p.chunk * hkv;
    w.Y = (uint16_t*)(base + o); o += align256((size_t)p.chunk * p.hy * kDL * 2);
    if (mode == 0) {
        w.tau = (float*)(base + o); o += align256(rows * 4);
        w.cand = (int2*)(base + o); o += align256(rows * kCandCap * 8);
        w.cand_n = (int32_t*)(base + o); o += align256(rows * 4);
        w.ovf_rows = (int32_t*)(base + o); o += align256(rows * 4);
        w.ovf_count = (int32_t*)(base + o); o += 256;
        w.fb_score = (double*)(base + o); o += align256((size_t)p.fb_slots * p.ld * 8);
        w.fb_w = (int32_t*)(base + o); o += align256((size_t)p.fb_slots * p.ld * 4);
        w.cent_s = (uint16_t*)(base + o); o += align256((size_t)hkv * p.ns_cap * kDL * 2);
        w.meta = (int4*)(base + o); o += align256((size_t)hkv * p.nb * 16);
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

// Candidate-record output of a flat selection (sequence-sharded selection):
// per (query, kv-head) row, the buckets its own fill of k keys took.
struct ShardOut {
    ShardRec* rec;      // [nq, hkv, cap]
    int32_t* rec_n;     // [nq, hkv]
    int32_t cap;
    int64_t id_base;    // added to local bucket ids
};

lsa_status run_select(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq, const float* W_q,
                      const lsa_cache* c, const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                      uint16_t* Y_out, void* ws, size_t ws_bytes, cudaStream_t st, const ShardOut* so) {
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
    a.ovf_rows = w.ovf_rows; a.ovf_count = w.ovf_count; a.ovf_cap = (int32_t)(p.chunk * hkv);
    a.fb_score = w.fb_score; a.fb_w = w.fb_w;
    if (so && cfg->mode != 0) return set_error(LSA_EUNSUPPORTED, "candidate records: flat search only");
    if (so) { a.rec_cap = so->cap; a.id_base = so->id_base; }

    CUtensorMap tmF, tmS;
    if (cfg->mode == 0) {
        lsa_status s = launch_sample_gather(c->cent, c->cap_buckets, NB, p.ns_cap, hkv, w.cent_s, st);
        if (s != LSA_OK) return s;
        if ((s = launch_meta_gather(c, NB, w.meta, st)) != LSA_OK) return s;
        if ((s = make_rows64_map(&tmF, c->cent, (int64_t)hkv * c->cap_buckets, kCdCols)) != LSA_OK) return s;
        if ((s = make_rows64_map(&tmS, w.cent_s, (int64_t)hkv * p.ns_cap, kSmCols)) != LSA_OK) return s;
    }

    for (int64_t c0 = 0; c0 < nq; c0 += p.chunk) {
        const int64_t nqc = (nq - c0) < p.chunk ? (nq - c0) : p.chunk;
        uint16_t* Y = Y_out ? Y_out + c0 * p.hy * kDL : w.Y;
        lsa_status s = launch_query_latent(Q + c0 * hq * kD, nqc, hq, hkv, W_q, cfg->agg, Y, st);
        if (s != LSA_OK) return s;
        a.Y = Y; a.nqc = nqc; a.t_first = t0 + c0; a.idx = idx ? idx + c0 * hkv * row_len : nullptr;
        if (so) { a.rec = so->rec + c0 * hkv * so->cap; a.rec_n = so->rec_n + c0 * hkv; }
        if (cfg->mode == 1) {
            if ((s = launch_tree_select(a, nqc * hkv, st)) != LSA_OK) return s;
            continue;
        }
        if (cudaMemsetAsync(w.ovf_count, 0, sizeof(int32_t), st) != cudaSuccess)
            return set_error(LSA_ECUDA, "lsa_select: memset failed");
        PassArgs pa{};
        pa.Y = Y; pa.ns_cap = p.ns_cap;
        pa.cap_buckets = c->cap_buckets; pa.NB = NB; pa.nqc = nqc; pa.t_first = t0 + c0;
        pa.W = cfg->window; pa.S = cfg->sinks; pa.hkv = hkv; pa.G = hq / hkv; pa.agg = cfg->agg; pa.k = cfg->k;
        pa.tau = w.tau; pa.cand = w.cand; pa.cand_n = w.cand_n;
        ResolveArgs ra{};
        ra.meta = w.meta; ra.cent = c->cent;
        ra.cap_buckets = c->cap_buckets; ra.NB = NB; ra.T_built = c->n_tokens;
        ra.hkv = hkv; ra.G = hq / hkv; ra.agg = cfg->agg; ra.k = cfg->k; ra.S = cfg->sinks;
        ra.W = cfg->window; ra.Y = Y; ra.nqc = nqc; ra.t_first = t0 + c0; ra.tau = w.tau;
        ra.cand = w.cand; ra.cand_n = w.cand_n; ra.idx = a.idx;
        ra.ovf_rows = w.ovf_rows; ra.ovf_count = w.ovf_count; ra.ovf_cap = a.ovf_cap;
        ra.rec = a.rec; ra.rec_n = a.rec_n; ra.rec_cap = a.rec_cap; ra.id_base = a.id_base;
        if ((s = launch_flat(pa, ra, tmF, tmS, st)) != LSA_OK) return s;
        {
            KTime kt_("select_fallback_kernel", st);
            if (so) select_fallback_kernel<true><<<(unsigned)p.fb_slots, kSelThreads, 0, st>>>(a);
            else select_fallback_kernel<false><<<(unsigned)p.fb_slots, kSelThreads, 0, st>>>(a);
        }
        if ((s = check_launch("select_fallback_kernel")) != LSA_OK) return s;
    }
    return LSA_OK;
}

}  // namespace lsa
