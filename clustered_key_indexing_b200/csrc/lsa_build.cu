// lsa_build.cu -- key build of the LSA path on sm_100a:
//   * latent rows: z = normalise(x W) in fp64 for keys (pooled into units)
//     and queries (group mean / per head, rounded to bf16)
//     [essay "《卡片柜》——当注意力学会先查目录再翻书", ch. 2; tutorial
//     "隐空间稀疏注意力 (LSA)", section 二; essay ch. 5 for the native variant];
//   * capped Ward clustering of one 512-key block per CTA [essay ch. 2;
//     Ward 1963];
//   * one level of the complete binary centroid tree [essay ch. 4].
//
// All latent and clustering arithmetic is fp64 in a fixed order (ascending
// index sums, separately rounded squares), so the bucket sets, sums and bf16
// centroids are reproducible bit for bit by any implementation that follows
// the same order.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"

namespace lsa {


// ---------------------------------------------------------------- latents

// Rows of 128 bf16 values are processed 16 at a time per warp.  Lane l owns
// key group kg = l / 16 (rows 8kg .. 8kg+7) and dim group cg = l % 16 (dims
// cg, cg+16, cg+32, cg+48): 32 fp64 accumulators, one fma per (row, dim, e).
// The product of a bf16 key and an fp32 weight is exact in fp64, so the fma
// chain equals "sum of products in ascending e, one rounding per add".
constexpr int kLatWarps = 8;  // 204 KB of shared memory: one CTA, 8 warps per SM
constexpr int kKT = 17;        // padded row stride (doubles) of the staged tile
constexpr int kVS = 65;        // padded row stride of the projected rows

enum LatentMode { kKeyPool = 0, kQueryMean = 1, kQueryHead = 2 };

struct LatentArgs {
    const uint16_t* X;   // bf16 rows: keys [T, hkv, 128] or queries [nq, hq, 128]
    const float* W;      // [128, 64] fp32
    int64_t n_items;     // units (key mode) or output rows (query modes)
    // key mode
    int64_t T;           // valid key rows (tokens)
    int32_t hkv;
    int64_t unit0;       // first unit to compute
    int64_t cap_units;
    double* U;           // [hkv, cap_units, 64]
    // query modes
    int32_t hq, G;
    uint16_t* Y;         // [nq, hkv or hq, 64]
};

template <int MODE>
__device__ __forceinline__ void item_rows(const LatentArgs& a, int64_t item, int r,
                                          int64_t& row, bool& valid) {
    if (MODE == kKeyPool) {
        const int64_t j = a.unit0 + item / a.hkv, h = item % a.hkv;
        const int64_t t = j * kPool + r;
        valid = item < a.n_items && t < a.T;
        row = t * a.hkv + h;
    } else if (MODE == kQueryMean) {
        const int64_t q = item / a.hkv, g = item % a.hkv;
        valid = item < a.n_items;
        row = q * a.hq + g * a.G + r;
    } else {
        valid = item < a.n_items;
        row = item;
    }
}

template <int MODE>
__global__ void __launch_bounds__(32 * kLatWarps)
latent_kernel(LatentArgs a) {
    extern __shared__ double lat_smem[];
    double* Ws = lat_smem;                                   // [128][64]
    double* wk = Ws + kD * kDL + (threadIdx.x / 32) * (kD * kKT + 16);
    double* nrm = wk + kD * kKT;                             // [16]
    const int lane = threadIdx.x & 31;
    const int rows_per_item = (MODE == kKeyPool) ? kPool : (MODE == kQueryMean ? a.G : 1);
    const int items_per_iter = 16 / rows_per_item;

    for (int i = threadIdx.x; i < kD * kDL; i += blockDim.x) Ws[i] = (double)a.W[i];
    __syncthreads();

    const int64_t warp0 = (int64_t)blockIdx.x * kLatWarps + threadIdx.x / 32;
    const int64_t nwarps = (int64_t)gridDim.x * kLatWarps;
    const int kg = lane >> 4, cg = lane & 15;

    for (int64_t base = warp0 * items_per_iter; base < a.n_items; base += nwarps * items_per_iter) {
        // stage 16 rows (row = lane%16, 16-byte parts lane/16 + 2m) as doubles, e-major
        const int row = lane & 15;
        int64_t grow;
        bool valid;
        item_rows<MODE>(a, base + row / rows_per_item, row % rows_per_item, grow, valid);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int part = (lane >> 4) + 2 * m;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (valid) v = __ldg(reinterpret_cast<const uint4*>(a.X + grow * kD) + part);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                wk[(part * 8 + 2 * i) * kKT + row] = (double)__uint_as_float(w4[i] << 16);
                wk[(part * 8 + 2 * i + 1) * kKT + row] = (double)__uint_as_float(w4[i] & 0xFFFF0000u);
            }
        }
        __syncwarp();
        double acc[8][4];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][i] = 0.0;
#pragma unroll 2
        for (int e = 0; e < kD; ++e) {
            double w[4], kv[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = Ws[e * kDL + cg + 16 * i];
#pragma unroll
            for (int r = 0; r < 8; ++r) kv[r] = wk[e * kKT + kg * 8 + r];
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[r][i] = fma(kv[r], w[i], acc[r][i]);
        }
        __syncwarp();
        double* vs = wk;  // reuse: [16][kVS] projected rows
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) vs[(kg * 8 + r) * kVS + cg + 16 * i] = acc[r][i];
        __syncwarp();
        if (lane < 16) {
            double n2 = 0.0;
            for (int c = 0; c < kDL; ++c) {
                const double v = vs[lane * kVS + c];
                n2 = __dadd_rn(n2, __dmul_rn(v, v));
            }
            nrm[lane] = sqrt(n2);
        }
        __syncwarp();
        for (int it = 0; it < items_per_iter; ++it) {
            const int64_t item = base + it;
            if (item >= a.n_items) break;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int c = lane + 32 * half;
                double s = 0.0;
                int n = 0;
                for (int r = 0; r < rows_per_item; ++r) {
                    int64_t gr;
                    bool ok;
                    item_rows<MODE>(a, item, r, gr, ok);
                    if (!ok) break;
                    const int lr = it * rows_per_item + r;
                    const double nn = nrm[lr];
                    const double z = nn > 0.0 ? __ddiv_rn(vs[lr * kVS + c], nn) : 0.0;
                    s = __dadd_rn(s, z);
                    ++n;
                }
                if (MODE == kKeyPool) {
                    const int64_t j = a.unit0 + item / a.hkv, h = item % a.hkv;
                    a.U[(h * a.cap_units + j) * kDL + c] = __ddiv_rn(s, (double)n);
                } else if (MODE == kQueryMean) {
                    a.Y[item * kDL + c] = f64_to_bf16_rne(__ddiv_rn(s, (double)a.G));
                } else {
                    a.Y[item * kDL + c] = f64_to_bf16_rne(s);
                }
            }
        }
        __syncwarp();
    }
}

static size_t latent_smem() {
    return sizeof(double) * (kD * kDL + kLatWarps * (kD * kKT + 16));
}

template <int MODE>
static lsa_status launch_latent(const LatentArgs& a, cudaStream_t st) {
    if (a.n_items <= 0) return LSA_OK;
    const size_t smem = latent_smem();
    cudaFuncSetAttribute(latent_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int rows_per_item = (MODE == kKeyPool) ? kPool : (MODE == kQueryMean ? a.G : 1);
    const int64_t iters = ceil_div<int64_t>(a.n_items, 16 / rows_per_item);
    int64_t grid = ceil_div<int64_t>(iters, kLatWarps);
    const int64_t cap = (int64_t)num_sms() * 4;
    if (grid > cap) grid = cap;
    {
        KTime kt_("latent_kernel", st);
        latent_kernel<MODE><<<(unsigned)grid, 32 * kLatWarps, smem, st>>>(a);
    }
    return check_launch("latent_kernel");
}

lsa_status launch_key_latent(const uint16_t* K, int64_t T, int32_t hkv, const float* W,
                             int64_t unit0, int64_t unit1, int64_t cap_units, double* U,
                             cudaStream_t st) {
    LatentArgs a{};
    a.X = K; a.W = W; a.T = T; a.hkv = hkv; a.unit0 = unit0; a.cap_units = cap_units; a.U = U;
    a.n_items = (unit1 - unit0) * hkv;
    return launch_latent<kKeyPool>(a, st);
}

lsa_status launch_query_latent(const uint16_t* Q, int64_t nq, int32_t hq, int32_t hkv,
                               const float* W, int agg, uint16_t* Y, cudaStream_t st) {
    LatentArgs a{};
    a.X = Q; a.W = W; a.hq = hq; a.hkv = hkv; a.G = hq / hkv; a.Y = Y;
    if (agg == 0) {
        a.n_items = nq * hkv;
        return launch_latent<kQueryMean>(a, st);
    }
    a.n_items = nq * hq;
    return launch_latent<kQueryHead>(a, st);
}

// ------------------------------------------------------------------- Ward

// One CTA (128 threads, thread r = row r) clusters one block of n <= 128
// pooled units to m = ceil(n/2) buckets.  Shared memory: the units (UT) and
// the cluster means (MU), both dim-major with a padded stride, and the upper
// triangle of the Delta matrix.  Each merge step: block argmin over the
// rows' nearest neighbours (Delta, lo, hi), merge (id = lower), recompute the
// merged cluster's mean from its members in ascending order, recompute its
// Delta row, refresh nearest neighbours (warp-parallel rescans of the rows
// that pointed at either merged cluster).
constexpr int kWT = 129;  // padded stride of UT / MU (doubles)

constexpr int kMaxWardJobs = 256;

struct WardArgs {
    const double* U;
    int64_t U_stride;    // units per head in U
    int32_t U_local;     // 1: U holds only the clustered block (decode block ring)
    int32_t n_jobs;      // > 0: decode jobs, blockIdx.x -> (head base, block) below
    int32_t job_head0[kMaxWardJobs];
    int64_t job_blk[kMaxWardJobs];
    int64_t cap_units, cap_buckets;
    int64_t NU;          // units in use
    int64_t T;           // tokens in use (key ranges clip to it)
    int32_t sinks;
    int64_t blk0;        // first block of this launch
    int32_t* bucket_of_unit;
    int32_t* members;
    int32_t* offsets;
    int32_t* cnt_lr;
    int32_t* minlr;
    int32_t* maxpos;
    double* sum;
    uint16_t* cent;
    int32_t* units;
    uint8_t* cent8;      // optional FP8 centroids (NULL: none)
};

__device__ __forceinline__ int tri_index(int i, int j) {  // i < j < 128
    return i * kUnitsPerBlock - (i * (i + 1)) / 2 + (j - i - 1);
}

__device__ __forceinline__ double dget(const double* D, int i, int j) {
    return i < j ? D[tri_index(i, j)] : D[tri_index(j, i)];
}

__device__ __forceinline__ bool better(double d1, int lo1, int hi1, double d2, int lo2, int hi2) {
    if (d1 != d2) return d1 < d2;
    if (lo1 != lo2) return lo1 < lo2;
    return hi1 < hi2;
}

// Delta between cluster a (mean column a of MU, na units) and column k.
__device__ __forceinline__ double ward_delta_cols(const double* MU, int a, int na, int k, int nk) {
    double ss = 0.0;
    for (int c = 0; c < kDL; ++c) {
        const double df = __dsub_rn(MU[c * kWT + a], MU[c * kWT + k]);
        ss = __dadd_rn(ss, __dmul_rn(df, df));
    }
    const double f = __ddiv_rn((double)(na * nk), (double)(na + nk));
    return __dmul_rn(f, ss);
}

__global__ void __launch_bounds__(128, 1) ward_kernel(WardArgs a) {
    extern __shared__ double wsm[];
    double* UT = wsm;                       // [64][kWT]
    double* MU = UT + kDL * kWT;            // [64][kWT]
    double* D = MU + kDL * kWT;             // 8128 upper-triangle entries
    __shared__ int size_[128];
    __shared__ int mem_[128][kMaxUnits];
    __shared__ int nn_[128];
    __shared__ double nnd_[128];
    __shared__ double red_d[4];
    __shared__ int red_lo[4], red_hi[4];
    __shared__ int resc_[128];
    __shared__ int n_resc;
    __shared__ int scan_[4];
    __shared__ int scan2_[4];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int h = a.n_jobs > 0 ? a.job_head0[blockIdx.x] + (int)blockIdx.y : (int)blockIdx.y;
    const int64_t blk = a.n_jobs > 0 ? a.job_blk[blockIdx.x] : a.blk0 + blockIdx.x;
    const int64_t u0 = blk * kUnitsPerBlock;
    const int n = (int)min((int64_t)kUnitsPerBlock, a.NU - u0);
    const int m = (n * kBucketsPerBlock + kUnitsPerBlock - 1) / kUnitsPerBlock;
    const double* Ub = a.U + ((int64_t)h * a.U_stride + (a.U_local ? 0 : u0)) * kDL;

    for (int i = tid; i < n * kDL; i += 128) {
        const int unit = i / kDL, c = i % kDL;
        const double v = Ub[i];
        UT[c * kWT + unit] = v;
        MU[c * kWT + unit] = v;
    }
    size_[tid] = tid < n ? 1 : 0;
    mem_[tid][0] = tid;
    __syncthreads();

    // initial Delta of singletons: 1/2 |u_i - u_j|^2 (pairs (i, i+d mod 128))
    for (int d = 1; d <= 64; ++d) {
        if (d == 64 && tid >= 64) break;
        const int j = (tid + d) & 127;
        const int lo = min(tid, j), hi = max(tid, j);
        if (hi < n) {
            double ss = 0.0;
            for (int c = 0; c < kDL; ++c) {
                const double df = __dsub_rn(MU[c * kWT + lo], MU[c * kWT + hi]);
                ss = __dadd_rn(ss, __dmul_rn(df, df));
            }
            D[tri_index(lo, hi)] = __dmul_rn(0.5, ss);
        }
    }
    __syncthreads();
    // nearest neighbour of every row (smallest Delta, lowest column on ties)
    {
        double bd = CUDART_INF;
        int bc = -1;
        if (tid < n) {
            for (int c = 0; c < n; ++c) {
                if (c == tid) continue;
                const double v = dget(D, tid, c);
                if (v < bd) { bd = v; bc = c; }
            }
        }
        nn_[tid] = bc;
        nnd_[tid] = bd;
    }
    __syncthreads();

    int clusters = n;
    while (clusters > m) {
        // (1) global best pair
        double bd = CUDART_INF;
        int blo = 1 << 20, bhi = 1 << 20;
        if (size_[tid] > 0 && nn_[tid] >= 0 && nnd_[tid] < CUDART_INF) {
            bd = nnd_[tid];
            blo = min(tid, nn_[tid]);
            bhi = max(tid, nn_[tid]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const double od = __shfl_xor_sync(0xffffffffu, bd, off);
            const int olo = __shfl_xor_sync(0xffffffffu, blo, off);
            const int ohi = __shfl_xor_sync(0xffffffffu, bhi, off);
            if (better(od, olo, ohi, bd, blo, bhi)) { bd = od; blo = olo; bhi = ohi; }
        }
        if (lane == 0) { red_d[wid] = bd; red_lo[wid] = blo; red_hi[wid] = bhi; }
        __syncthreads();
        bd = red_d[0]; blo = red_lo[0]; bhi = red_hi[0];
        for (int w = 1; w < 4; ++w)
            if (better(red_d[w], red_lo[w], red_hi[w], bd, blo, bhi)) {
                bd = red_d[w]; blo = red_lo[w]; bhi = red_hi[w];
            }
        if (!(bd < CUDART_INF)) {
            if (tid == 0) raise_device_error(kErrWardInfeasible);
            break;
        }
        const int A = blo, B = bhi;
        // (2) merge B into A; members stay ascending
        if (tid == 0) {
            int tmp[kMaxUnits];
            const int na = size_[A], nb = size_[B];
            int i = 0, j = 0, o = 0;
            while (i < na || j < nb) {
                if (j >= nb || (i < na && mem_[A][i] < mem_[B][j])) tmp[o++] = mem_[A][i++];
                else tmp[o++] = mem_[B][j++];
            }
            for (int k = 0; k < o; ++k) mem_[A][k] = tmp[k];
            size_[A] = na + nb;
            size_[B] = 0;
            n_resc = 0;
        }
        __syncthreads();
        // (3) mean of the merged cluster from its members, ascending
        const int na = size_[A];
        if (tid < kDL) {
            double s = 0.0;
            for (int i = 0; i < na; ++i) s = __dadd_rn(s, UT[tid * kWT + mem_[A][i]]);
            MU[tid * kWT + A] = __ddiv_rn(s, (double)na);
        }
        __syncthreads();
        // (4) Delta row of the merged cluster
        double dA = CUDART_INF;
        const int nk = size_[tid];
        if (tid != A && nk > 0) {
            if (na + nk <= kMaxUnits) dA = ward_delta_cols(MU, A, na, tid, nk);
            D[tid < A ? tri_index(tid, A) : tri_index(A, tid)] = dA;
        }
        __syncthreads();
        // (5) nearest-neighbour refresh
        if (nk > 0) {
            const int cur = nn_[tid];
            if (tid == A || cur == A || cur == B) {
                const int slot = atomicAdd(&n_resc, 1);
                resc_[slot] = tid;
            } else if (dA < nnd_[tid] || (dA == nnd_[tid] && dA < CUDART_INF && A < cur)) {
                nnd_[tid] = dA;
                nn_[tid] = A;
            }
        } else {
            nn_[tid] = -1;
            nnd_[tid] = CUDART_INF;
        }
        __syncthreads();
        for (int q = wid; q < n_resc; q += 4) {
            const int r = resc_[q];
            double best = CUDART_INF;
            int bc = 1 << 20;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = lane + 32 * i;
                if (c < n && c != r && size_[c] > 0) {
                    const double v = dget(D, r, c);
                    if (v < best) { best = v; bc = c; }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double ob = __shfl_xor_sync(0xffffffffu, best, off);
                const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
                if (ob < best || (ob == best && oc < bc)) { best = ob; bc = oc; }
            }
            if (lane == 0) {
                nn_[r] = best < CUDART_INF ? bc : -1;
                nnd_[r] = best;
            }
        }
        __syncthreads();
        --clusters;
    }
    __syncthreads();

    // ---- epilogue: buckets in ascending cluster id
    const bool active = tid < n && size_[tid] > 0;
    const unsigned bal = __ballot_sync(0xffffffffu, active);
    const int sz = active ? size_[tid] : 0;
    int incl = sz;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) { scan_[wid] = __popc(bal); scan2_[wid] = incl; }
    __syncthreads();
    int before_b = 0, before_u = 0;
    for (int w = 0; w < wid; ++w) { before_b += scan_[w]; before_u += scan2_[w]; }
    const int lb = before_b + __popc(bal & ((1u << lane) - 1u));
    const int pos_in_blk = before_u + incl - sz;
    const int64_t hb0 = (int64_t)h * a.cap_buckets;
    int32_t* offs = a.offsets + (int64_t)h * (a.cap_buckets + 1);
    if (active) {
        const int64_t b = blk * kBucketsPerBlock + lb;
        const int64_t pos = u0 + pos_in_blk;
        offs[b] = (int32_t)pos;
        int c_lr = 0, mlr = kIMax, mxp = -1;
        for (int i = 0; i < sz; ++i) {
            const int64_t j = u0 + mem_[tid][i];
            a.members[(int64_t)h * a.cap_units + pos + i] = (int32_t)j;
            a.bucket_of_unit[(int64_t)h * a.cap_units + j] = (int32_t)b;
            for (int64_t p = j * kPool; p < j * kPool + kPool && p < a.T; ++p) {
                if (p > mxp) mxp = (int32_t)p;
                if (p >= a.sinks) { ++c_lr; if (p < mlr) mlr = (int32_t)p; }
            }
        }
        int32_t pk = sz << 28;
        for (int i = 0; i < sz; ++i) pk |= mem_[tid][i] << (7 * i);
        a.units[hb0 + b] = pk;
        a.cnt_lr[hb0 + b] = c_lr;
        a.minlr[hb0 + b] = mlr;
        a.maxpos[hb0 + b] = mxp;
        double* sb = a.sum + (hb0 + b) * kDL;
        double n2 = 0.0;
        for (int c = 0; c < kDL; ++c) {
            double s = 0.0;
            for (int i = 0; i < sz; ++i) s = __dadd_rn(s, UT[c * kWT + mem_[tid][i]]);
            sb[c] = s;
            n2 = __dadd_rn(n2, __dmul_rn(s, s));
        }
        const double nrm = sqrt(n2);
        uint16_t* cb = a.cent + (hb0 + b) * kDL;
        for (int c = 0; c < kDL; ++c)
            cb[c] = f64_to_bf16_rne(nrm > 0.0 ? __ddiv_rn(sb[c], nrm) : 0.0);
        if (a.cent8) {  // e4m3 of 2^8 times the same fp64 component (exact scaling)
            uint8_t* c8 = a.cent8 + (hb0 + b) * kDL;
            for (int c = 0; c < kDL; ++c)
                c8[c] = f64_to_e4m3_rne(nrm > 0.0 ? __ddiv_rn(sb[c], nrm) * 256.0 : 0.0);
        }
    }
    if (tid >= m && tid < kBucketsPerBlock) {
        const int64_t b = blk * kBucketsPerBlock + tid;
        offs[b] = (int32_t)(u0 + n);
        a.cnt_lr[hb0 + b] = 0;
        a.minlr[hb0 + b] = kIMax;
        a.maxpos[hb0 + b] = -1;
        a.units[hb0 + b] = 0;
        for (int c = 0; c < kDL; ++c) {
            a.sum[(hb0 + b) * kDL + c] = 0.0;
            a.cent[(hb0 + b) * kDL + c] = 0;
            if (a.cent8) a.cent8[(hb0 + b) * kDL + c] = 0;
        }
    }
    if (tid == 0) offs[(blk + 1) * kBucketsPerBlock] = (int32_t)(u0 + n);
}

static void fill_ward_cache(WardArgs& a, const lsa_cache* c) {
    a.cap_units = c->cap_units; a.cap_buckets = c->cap_buckets;
    a.bucket_of_unit = c->bucket_of_unit; a.members = c->members; a.offsets = c->offsets;
    a.cnt_lr = c->cnt_lr; a.minlr = c->minlr; a.maxpos = c->maxpos; a.sum = c->sum; a.cent = c->cent;
    a.units = c->units; a.cent8 = c->cent8;
}

static size_t ward_smem() {
    return sizeof(double) * (2 * kDL * kWT + kUnitsPerBlock * (kUnitsPerBlock - 1) / 2);
}

// Blocks [blk0, blk1) of every head of `c`, units read from U (U_stride
// units per head).
lsa_status launch_ward_u(const lsa_cache* c, const double* U, int64_t U_stride, int64_t T,
                         int32_t sinks, int64_t blk0, int64_t blk1, cudaStream_t st) {
    if (blk1 <= blk0) return LSA_OK;
    WardArgs a{};
    fill_ward_cache(a, c);
    a.U = U; a.U_stride = U_stride; a.U_local = 0; a.n_jobs = 0;
    a.NU = ceil_div<int64_t>(T, kPool); a.T = T; a.sinks = sinks; a.blk0 = blk0;
    const size_t smem = ward_smem();
    cudaFuncSetAttribute(ward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((unsigned)(blk1 - blk0), (unsigned)c->hkv);
    {
        KTime kt_("ward_kernel", st);
        ward_kernel<<<grid, 128, smem, st>>>(a);
    }
    return check_launch("ward_kernel");
}

lsa_status launch_ward(const lsa_cache* c, int64_t T, int32_t sinks, int64_t blk0, int64_t blk1,
                       cudaStream_t st) {
    return launch_ward_u(c, c->U, c->cap_units, T, sinks, blk0, blk1, st);
}

// Decode: cluster one completed block per job; job j covers heads
// head0[j] .. head0[j] + hkv - 1 of the (request-combined) cache, and its
// units come from the block ring U_blk [heads, 128, 64].
lsa_status launch_ward_jobs(const lsa_cache* c, const double* U_blk, int32_t hkv, int32_t sinks,
                            int n_jobs, const int32_t* head0, const int64_t* blk, cudaStream_t st) {
    if (n_jobs <= 0) return LSA_OK;
    if (n_jobs > kMaxWardJobs) return set_error(LSA_EUNSUPPORTED, "more than %d blocks completed in one step", kMaxWardJobs);
    WardArgs a{};
    fill_ward_cache(a, c);
    a.U = U_blk; a.U_stride = kUnitsPerBlock; a.U_local = 1; a.n_jobs = n_jobs;
    for (int j = 0; j < n_jobs; ++j) { a.job_head0[j] = head0[j]; a.job_blk[j] = blk[j]; }
    a.NU = c->cap_units; a.T = c->cap_units * kPool; a.sinks = sinks; a.blk0 = 0;
    const size_t smem = ward_smem();
    cudaFuncSetAttribute(ward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((unsigned)n_jobs, (unsigned)hkv);
    {
        KTime kt_("ward_kernel", st);
        ward_kernel<<<grid, 128, smem, st>>>(a);
    }
    return check_launch("ward_kernel(decode)");
}

// Mark bucket slots [b0, b1) of every head empty.
__global__ void clear_slots_kernel(int32_t* cnt_lr, int32_t* minlr, int32_t* maxpos, double* sum,
                                   uint16_t* cent, int32_t* units, uint8_t* cent8, int64_t cap_buckets,
                                   int64_t b0, int64_t b1, int32_t hkv) {
    const int64_t span = b1 - b0;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= span * hkv * kDL) return;
    const int64_t h = i / (span * kDL), r = i % (span * kDL);
    const int64_t b = b0 + r / kDL, c = r % kDL;
    const int64_t hb = h * cap_buckets + b;
    sum[hb * kDL + c] = 0.0;
    cent[hb * kDL + c] = 0;
    if (cent8) cent8[hb * kDL + c] = 0;
    if (c == 0) {
        cnt_lr[hb] = 0;
        minlr[hb] = kIMax;
        maxpos[hb] = -1;
        units[hb] = 0;
    }
}

lsa_status launch_clear_slots(const lsa_cache* c, int64_t b0, int64_t b1, cudaStream_t st) {
    if (b1 <= b0) return LSA_OK;
    const int64_t n = (b1 - b0) * c->hkv * kDL;
    clear_slots_kernel<<<(unsigned)ceil_div<int64_t>(n, 256), 256, 0, st>>>(
        c->cnt_lr, c->minlr, c->maxpos, c->sum, c->cent, c->units, c->cent8, c->cap_buckets, b0, b1, c->hkv);
    return check_launch("clear_slots_kernel");
}

// ------------------------------------------------------------------- tree

// One warp per node i in [i0, i1) of level l: sum = left + right child sum
// (a missing right child copies the left), minlr = min, centroid =
// bf16(sum / |sum|) with |sum|^2 accumulated in ascending dim order.
__global__ void tree_level_kernel(double* tsum, int32_t* tminlr, uint16_t* tcent, int64_t n_nodes,
                                  int64_t off_l, int64_t off_c, int64_t n_c, int64_t i0, int64_t i1,
                                  int32_t hkv) {
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int64_t span = i1 - i0;
    if (w >= span * hkv) return;
    const int64_t h = w / span, i = i0 + w % span;
    const int64_t base = h * n_nodes;
    const int64_t ca = base + off_c + 2 * i, cb = ca + 1;
    const bool has_b = 2 * i + 1 < n_c;
    double s0 = tsum[ca * kDL + lane], s1 = tsum[ca * kDL + lane + 32];
    if (has_b) {
        s0 = __dadd_rn(s0, tsum[cb * kDL + lane]);
        s1 = __dadd_rn(s1, tsum[cb * kDL + lane + 32]);
    }
    const int64_t node = base + off_l + i;
    tsum[node * kDL + lane] = s0;
    tsum[node * kDL + lane + 32] = s1;
    double n2 = 0.0;
    for (int c = 0; c < kDL; ++c) {
        const double v = __shfl_sync(0xffffffffu, c < 32 ? s0 : s1, c & 31);
        n2 = __dadd_rn(n2, __dmul_rn(v, v));
    }
    const double nrm = sqrt(n2);
    tcent[node * kDL + lane] = f64_to_bf16_rne(nrm > 0.0 ? __ddiv_rn(s0, nrm) : 0.0);
    tcent[node * kDL + lane + 32] = f64_to_bf16_rne(nrm > 0.0 ? __ddiv_rn(s1, nrm) : 0.0);
    if (lane == 0) {
        const int32_t ma = tminlr[ca];
        const int32_t mb = has_b ? tminlr[cb] : kIMax;
        tminlr[node] = mb < ma ? mb : ma;
    }
}

// Copy buckets [b0, b1) into tree level 0, then rebuild every ancestor of
// them level by level.
lsa_status launch_tree_update(const lsa_cache* c, lsa_tree* t, int64_t b0, int64_t b1,
                              cudaStream_t st) {
    if (b1 <= b0) return LSA_OK;
    const int64_t hkv = c->hkv;
    cudaError_t e;
    e = cudaMemcpy2DAsync(t->sum + b0 * kDL, t->n_nodes * kDL * sizeof(double),
                          c->sum + b0 * kDL, c->cap_buckets * kDL * sizeof(double),
                          (b1 - b0) * kDL * sizeof(double), hkv, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(t->cent + b0 * kDL, t->n_nodes * kDL * sizeof(uint16_t),
                              c->cent + b0 * kDL, c->cap_buckets * kDL * sizeof(uint16_t),
                              (b1 - b0) * kDL * sizeof(uint16_t), hkv, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(t->minlr + b0, t->n_nodes * sizeof(int32_t), c->minlr + b0,
                              c->cap_buckets * sizeof(int32_t), (b1 - b0) * sizeof(int32_t), hkv,
                              cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return set_error(LSA_ECUDA, "tree level-0 copy: %s", cudaGetErrorString(e));
    int64_t lo = b0, hi = b1;  // node range [lo, hi) on the current level
    for (int l = 1; l < t->levels; ++l) {
        lo >>= 1;
        hi = (hi + 1) >> 1;
        const int64_t warps = (hi - lo) * hkv;
        const int threads = 256;
        const int64_t blocks = ceil_div<int64_t>(warps * 32, threads);
        tree_level_kernel<<<(unsigned)blocks, threads, 0, st>>>(
            t->sum, t->minlr, t->cent, t->n_nodes, t->level_off[l], t->level_off[l - 1],
            t->level_n[l - 1], lo, hi, c->hkv);
        lsa_status s = check_launch("tree_level_kernel");
        if (s != LSA_OK) return s;
    }
    return LSA_OK;
}

}  // namespace lsa
