// lsa_shard.cu -- the sequence-sharded LSA layer: each GPU of a job holds a
// contiguous range of whole 512-key cluster blocks [p0, p1) of the context
// (its K/V and their bucket cache), the way the LSA pages' deployments split
// the context over GPUs (news page, "开源内容": DCP8 / CP8 context
// parallelism), while the query positions are shared.  Per chunk of queries:
//
//   lsa_shard_candidates  every shard runs the flat search [essay
//       "《卡片柜》——当注意力学会先查目录再翻书", ch. 3] over its own buckets
//       and keeps the buckets its own fill of k keys takes, as records
//       (global bucket id, keys taken, exact fp64 score);
//   all-gather of the records (NCCL, by the caller);
//   lsa_shard_merge  the global fill over every shard's records: the
//       buckets of the fill over all buckets are among them (a bucket the
//       global fill takes has less than k keys ranked above it in its own
//       shard too), and a bucket's own-shard taken count bounds what the
//       global fill can take from it, so the weighted radix select over the
//       records (score desc, global id asc) reproduces the single-GPU
//       selection; each shard then emits its own keys, its part of the
//       window and (first shard) the sinks;
//   lsa_sparse_attn_partial  exact attention over the shard's own entries,
//       normalised O with its base-2 log-sum-exp [tutorial "隐空间稀疏注意力
//       (LSA)", section 二];
//   all-gather of the partials, then lsa_lse_combine: O = sum_r 2^(L_r - M) O_r
//       / sum_r 2^(L_r - M), the exact softmax over the union of the
//       shards' entries.
// No TMA load here or in the kernels these calls run reads another GPU's
// memory: the exchange goes through the caller's collectives.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"
#include "lsa_common.cuh"

namespace lsa {

lsa_status launch_attn_partial(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                               int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t p0, int64_t n_keys,
                               float* Opart, float* lse, cudaStream_t st);

static int32_t shard_cap(const lsa_cfg* cfg) { return cfg->k / kPool + 4; }

// Sinks apply to positions below S, all of which lie in the first shard.
static int32_t shard_sinks(const lsa_cfg* cfg, int64_t p0) { return p0 == 0 ? cfg->sinks : 0; }

static lsa_status check_shard(const lsa_cfg* cfg, int64_t p0) {
    if (p0 < 0 || p0 % kBlockKeys) return set_error(LSA_EINVAL, "shard: p0 must be a non-negative multiple of 512");
    if (cfg->sinks > kBlockKeys) return set_error(LSA_EUNSUPPORTED, "shard: sinks beyond the first block");
    if (cfg->mode != 0) return set_error(LSA_EUNSUPPORTED, "shard: flat search only");
    return LSA_OK;
}

struct MergeArgs {
    const ShardRec* rec_all;   // [world, rows, cap]
    const int32_t* n_all;      // [world, rows]
    int32_t world, rank, cap;
    int64_t rows;
    // the shard's own cache (positions local to the shard)
    const int32_t* offsets;
    const int32_t* members;
    int64_t cap_units, cap_buckets, n_local;
    int32_t hkv, k, S, W, S_loc;
    int64_t p0, t0, id_base;
    int32_t* idx;              // [nq, hkv, S + k + W]
};

// CTA per (query, kv-head) row; dynamic shared memory holds every shard's
// records of the row (score, weight, taken).
__global__ void __launch_bounds__(kSelThreads) shard_merge_kernel(MergeArgs a) {
    extern __shared__ __align__(16) uint8_t msm[];
    __shared__ SelShared sh;
    __shared__ int offs[65];
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    const int64_t q = row / a.hkv;
    const int h = (int)(row % a.hkv);
    const int64_t t = a.t0 + q;
    const int64_t lim = t - a.W;                      // global
    const int64_t p1 = a.p0 + a.n_local;
    const int nmax = a.world * a.cap;
    double* sc = reinterpret_cast<double*>(msm);
    int* w = reinterpret_cast<int*>(sc + nmax);
    int* tk = w + nmax;
    int32_t* out = a.idx + row * (int64_t)(a.S + a.k + a.W);

    // sinks (first shard) and this shard's part of the window, compacted
    for (int i = tid; i < a.S; i += kSelThreads) out[i] = (a.p0 == 0 && i <= t) ? i : -1;
    const int64_t w0 = max(max((int64_t)a.S, t - a.W + 1), a.p0), w1 = min(t + 1, p1);
    for (int i = tid; i < a.W; i += kSelThreads) out[a.S + a.k + i] = (w0 + i < w1) ? (int32_t)(w0 + i) : -1;

    if (tid == 0) {
        int o = 0;
        for (int r = 0; r < a.world; ++r) {
            offs[r] = o;
            o += min(a.n_all[(int64_t)r * a.rows + row], a.cap);
        }
        offs[a.world] = o;
    }
    __syncthreads();
    const int n = offs[a.world];
    int mine = 0;
    for (int r = 0; r < a.world; ++r) {
        const ShardRec* src = a.rec_all + ((int64_t)r * a.rows + row) * a.cap;
        const int nr = offs[r + 1] - offs[r];
        for (int i = tid; i < nr; i += kSelThreads) {
            const ShardRec rc = src[i];
            sc[offs[r] + i] = rc.score;
            w[offs[r] + i] = rc.taken;
            mine += rc.taken;
        }
    }
    int tot;
    block_exscan(mine, &tot, sh.sh4);
    __syncthreads();
    if (tot > a.k)
        radix_fill(
            n, a.k, [&](int64_t i) { return sc[i]; }, [&](int64_t i) { return w[i]; },
            [&](int64_t i, int v) { tk[i] = v; }, sh);
    else
        for (int i = tid; i < n; i += kSelThreads) tk[i] = w[i];
    __syncthreads();

    // this shard's records: their keys in [S, t - W], ascending within a
    // bucket, buckets in ascending id
    const ShardRec* own = a.rec_all + ((int64_t)a.rank * a.rows + row) * a.cap;
    const int o0 = offs[a.rank], no = offs[a.rank + 1] - o0;
    const int per = (no + kSelThreads - 1) / kSelThreads;
    const int i0 = tid * per, i1 = min(no, i0 + per);
    int cnt = 0;
    for (int i = i0; i < i1; ++i) cnt += tk[o0 + i];
    int total;
    int o = block_exscan(cnt, &total, sh.sh4);
    const int32_t* off = a.offsets + (int64_t)h * (a.cap_buckets + 1);
    const int32_t* mem = a.members + (int64_t)h * a.cap_units;
    const int64_t lim_loc = lim - a.p0;
    for (int i = i0; i < i1; ++i) {
        int rem = tk[o0 + i];
        const int64_t b = own[i].bucket - a.id_base;
        for (int32_t m = off[b]; m < off[b + 1] && rem > 0; ++m)
            for (int64_t p = (int64_t)mem[m] * kPool; p < (int64_t)mem[m] * kPool + kPool && p < a.n_local && rem > 0; ++p)
                if (p >= a.S_loc && p <= lim_loc) {
                    out[a.S + o++] = (int32_t)(p + a.p0);
                    --rem;
                }
    }
    for (int i = total + tid; i < a.k; i += kSelThreads) out[a.S + i] = -1;
}

// O = sum_r 2^(L_r - M) O_r / sum_r 2^(L_r - M) per (query, head), M = max_r L_r.
__global__ void lse_combine_kernel(const float* __restrict__ Op, const float* __restrict__ L, int32_t world,
                                   int64_t nqh, uint16_t* __restrict__ O) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= nqh * kD) return;
    const int64_t i = e / kD;
    float M = -CUDART_INF_F;
    for (int r = 0; r < world; ++r) M = fmaxf(M, L[(int64_t)r * nqh + i]);
    float num = 0.f, den = 0.f;
    if (M > -CUDART_INF_F) {
        for (int r = 0; r < world; ++r) {
            const float lr = L[(int64_t)r * nqh + i];
            if (!(lr > -CUDART_INF_F)) continue;
            const float wr = exp2f(lr - M);
            num += wr * Op[(int64_t)r * nqh * kD + e];
            den += wr;
        }
    }
    const __nv_bfloat16 ob = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
    O[e] = *reinterpret_cast<const uint16_t*>(&ob);
}

}  // namespace lsa

using namespace lsa;

extern "C" {

int32_t lsa_shard_cand_cap(const lsa_cfg* cfg) {
    if (!cfg || check_cfg(cfg) != LSA_OK) return 0;
    return shard_cap(cfg);
}

lsa_status lsa_shard_build_buckets(const uint16_t* K, int64_t n, int32_t hkv, const float* W_k, const lsa_cfg* cfg,
                                   int64_t p0, lsa_cache* cache, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK || (s = check_shard(cfg, p0)) != LSA_OK) return s;
    lsa_cfg c = *cfg;
    c.sinks = shard_sinks(cfg, p0);
    return lsa_build_buckets(K, n, hkv, W_k, &c, cache, stream);
}

lsa_status lsa_shard_candidates(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq, const float* W_q,
                                const lsa_cache* cache, int64_t p0, const lsa_cfg* cfg, void* rec, int32_t* rec_n,
                                void* ws, size_t ws_bytes, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK || (s = check_shard(cfg, p0)) != LSA_OK) return s;
    if ((s = check_cache(cache, true)) != LSA_OK) return s;
    if ((s = check_heads(hq, cache->hkv)) != LSA_OK) return s;
    if (!Q || !W_q || !rec || !rec_n) return set_error(LSA_EINVAL, "lsa_shard_candidates: NULL pointer");
    if (nq < 0 || t0 < 0) return set_error(LSA_EINVAL, "lsa_shard_candidates: negative nq or t0");
    if (((uintptr_t)rec & 15u) != 0) return set_error(LSA_EINVAL, "lsa_shard_candidates: rec must be 16-byte aligned");
    if (nq == 0) return LSA_OK;
    lsa_cfg c = *cfg;
    c.sinks = shard_sinks(cfg, p0);
    const int32_t hkv = cache->hkv, cap = shard_cap(cfg);
    cudaStream_t st = (cudaStream_t)stream;
    // queries before p0 + W + S have no eligible key in this shard
    const int64_t qf = min(nq, max((int64_t)0, p0 + c.window + c.sinks - t0));
    if (qf > 0 && cudaMemsetAsync(rec_n, 0, (size_t)qf * hkv * 4, st) != cudaSuccess)
        return set_error(LSA_ECUDA, "lsa_shard_candidates: memset failed");
    if (qf == nq) return LSA_OK;
    ShardOut so{reinterpret_cast<ShardRec*>(rec) + qf * hkv * cap, rec_n + qf * hkv, cap,
                p0 / kBlockKeys * kBucketsPerBlock};
    return run_select(Q + qf * hq * kD, t0 + qf - p0, nq - qf, hq, W_q, cache, nullptr, &c, nullptr, nullptr, ws,
                      ws_bytes, st, &so);
}

lsa_status lsa_shard_merge(const void* rec_all, const int32_t* rec_n_all, int32_t world, int32_t rank, int64_t t0,
                           int64_t nq, const lsa_cache* cache, int64_t p0, const lsa_cfg* cfg, int32_t* idx,
                           void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK || (s = check_shard(cfg, p0)) != LSA_OK) return s;
    if ((s = check_cache(cache, true)) != LSA_OK) return s;
    if (!rec_all || !rec_n_all || !idx) return set_error(LSA_EINVAL, "lsa_shard_merge: NULL pointer");
    if (world < 1 || world > 64 || rank < 0 || rank >= world)
        return set_error(LSA_EINVAL, "lsa_shard_merge: need 0 <= rank < world <= 64");
    if (nq < 0 || t0 < 0) return set_error(LSA_EINVAL, "lsa_shard_merge: negative nq or t0");
    if (nq == 0) return LSA_OK;
    MergeArgs a{};
    a.rec_all = reinterpret_cast<const ShardRec*>(rec_all); a.n_all = rec_n_all;
    a.world = world; a.rank = rank; a.cap = shard_cap(cfg); a.rows = nq * cache->hkv;
    a.offsets = cache->offsets; a.members = cache->members; a.cap_units = cache->cap_units;
    a.cap_buckets = cache->cap_buckets; a.n_local = cache->n_tokens;
    a.hkv = cache->hkv; a.k = cfg->k; a.S = cfg->sinks; a.W = cfg->window; a.S_loc = shard_sinks(cfg, p0);
    a.p0 = p0; a.t0 = t0; a.id_base = p0 / kBlockKeys * kBucketsPerBlock; a.idx = idx;
    const size_t smem = (size_t)world * a.cap * (8 + 4 + 4);
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaFuncSetAttribute(shard_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return set_error(LSA_EUNSUPPORTED, "lsa_shard_merge: %zu bytes of records per row do not fit", smem);
    {
        KTime kt_("shard_merge_kernel", st);
        shard_merge_kernel<<<(unsigned)a.rows, kSelThreads, smem, st>>>(a);
    }
    return check_launch("shard_merge_kernel");
}

lsa_status lsa_sparse_attn_partial(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                                   int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t p0, int64_t n_keys,
                                   float* O_part, float* lse, void* stream) {
    lsa_status s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!Q || !K || !V || !idx || !O_part || !lse) return set_error(LSA_EINVAL, "lsa_sparse_attn_partial: NULL pointer");
    if (nq < 0 || n_idx < 0 || p0 < 0 || n_keys < 0)
        return set_error(LSA_EINVAL, "lsa_sparse_attn_partial: negative size");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O_part))
        return set_error(LSA_EINVAL, "lsa_sparse_attn_partial: Q, K, V, O_part must be 16-byte aligned");
    if (p0 + n_keys > (int64_t)INT32_MAX) return set_error(LSA_EUNSUPPORTED, "lsa_sparse_attn_partial: positions beyond 2^31");
    return launch_attn_partial(Q, K, V, idx, nq, hq, hkv, n_idx, p0, n_keys, O_part, lse, (cudaStream_t)stream);
}

lsa_status lsa_lse_combine(const float* O_parts, const float* lse_parts, int32_t world, int64_t nq, int32_t hq,
                           uint16_t* O, void* stream) {
    if (!O_parts || !lse_parts || !O) return set_error(LSA_EINVAL, "lsa_lse_combine: NULL pointer");
    if (world < 1 || nq < 0 || hq < 1) return set_error(LSA_EINVAL, "lsa_lse_combine: bad sizes");
    const int64_t n = nq * hq * kD;
    if (n == 0) return LSA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    {
        KTime kt_("lse_combine_kernel", st);
        lse_combine_kernel<<<(unsigned)ceil_div<int64_t>(n, 256), 256, 0, st>>>(O_parts, lse_parts, world, nq * hq, O);
    }
    return check_launch("lse_combine_kernel");
}

}  // extern "C"
