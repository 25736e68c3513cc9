// lsa_api.cu -- extern "C" entry points of liblsa.so: argument checks,
// status codes, launch sequencing.  Every kernel lives in lsa_build.cu,
// lsa_select.cu or lsa_attn.cu; nothing here computes on the host.
#include <cuda_runtime.h>
#include <stdarg.h>

#include <atomic>
#include <mutex>
#include <stdint.h>
#include <vector>
#include <stdio.h>
#include <string.h>

#include "lsa.h"
#include "lsa_common.cuh"

namespace lsa {

static thread_local char g_err[512] = "";
static std::atomic<long long> g_launches{0};

lsa_status set_error(lsa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

lsa_status check_launch(const char* what) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(LSA_ECUDA, "%s: %s", what, cudaGetErrorString(e));
    return LSA_OK;
}

// ---------------------------------------------------------- kernel timing

struct TimerRec {
    const char* name;
    std::vector<cudaEvent_t> start, stop;
    size_t used = 0;
};
static std::atomic<bool> g_timing{false};
static std::mutex g_tmu;
static std::vector<TimerRec> g_trec;

KTime::KTime(const char* name, cudaStream_t s) : st(s) {
    if (!g_timing.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_tmu);
    int r = -1;
    for (size_t i = 0; i < g_trec.size(); ++i)
        if (strcmp(g_trec[i].name, name) == 0) { r = (int)i; break; }
    if (r < 0) {
        g_trec.push_back(TimerRec{name, {}, {}, 0});
        r = (int)g_trec.size() - 1;
    }
    TimerRec& t = g_trec[r];
    if (t.used == t.start.size()) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return;
        if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return; }
        t.start.push_back(a);
        t.stop.push_back(b);
    }
    rec = r;
    slot = (int)t.used++;
    cudaEventRecord(t.start[slot], st);
}

KTime::~KTime() {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_tmu);
    cudaEventRecord(g_trec[rec].stop[slot], st);
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// kernels (other translation units)
int64_t select_chunk(const lsa_cfg* cfg, int32_t hq, int32_t hkv);
int64_t select_wave_rows(const lsa_cfg* cfg, int32_t hq, int32_t hkv);
lsa_status launch_key_latent(const uint16_t* K, int64_t T, int32_t hkv, const float* W, int64_t unit0,
                             int64_t unit1, int64_t cap_units, double* U, cudaStream_t st);
lsa_status launch_query_latent(const uint16_t* Q, int64_t nq, int32_t hq, int32_t hkv, const float* W,
                               int agg, uint16_t* Y, cudaStream_t st);
lsa_status launch_ward(const lsa_cache* c, int64_t T, int32_t sinks, int64_t blk0, int64_t blk1,
                       cudaStream_t st);
lsa_status launch_clear_slots(const lsa_cache* c, int64_t b0, int64_t b1, cudaStream_t st);
lsa_status launch_tree_update(const lsa_cache* c, lsa_tree* t, int64_t b0, int64_t b1, cudaStream_t st);
size_t select_ws_bytes(const lsa_cfg* cfg, int64_t nq, int32_t hq, int32_t hkv, int64_t NB);
lsa_status run_select(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq, const float* W_q,
                      const lsa_cache* c, const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                      uint16_t* Y_out, void* ws, size_t ws_bytes, cudaStream_t st, const ShardOut* so);
lsa_status launch_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                       int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t T, uint16_t* O,
                       cudaStream_t st, int64_t kv_q_stride, int split, int32_t n_use, const float* Ow,
                       const float* lse, const uint16_t* Ks, const uint16_t* Vs, int64_t shared_len);
lsa_status launch_band_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t nq, int64_t t0,
                            int64_t T, int32_t hq, int32_t hkv, int32_t S, int32_t W, float* Ow, float* lse,
                            cudaStream_t st);

static lsa_status check_cfg(const lsa_cfg* c) {
    if (!c) return set_error(LSA_EINVAL, "cfg is NULL");
    if (c->d_head <= 0 || c->d_latent <= 0 || c->pool <= 0 || c->block <= 0 || c->bucket_mean <= 0 ||
        c->bucket_max <= 0)
        return set_error(LSA_EINVAL, "cfg: sizes must be positive");
    if (c->k < 1 || c->sinks < 0 || c->window < 1 || c->beam < 1)
        return set_error(LSA_EINVAL, "cfg: need k >= 1, sinks >= 0, window >= 1, beam >= 1");
    if (c->mode != 0 && c->mode != 1) return set_error(LSA_EINVAL, "cfg: mode must be 0 (flat) or 1 (tree)");
    if (c->agg != 0 && c->agg != 1) return set_error(LSA_EINVAL, "cfg: agg must be 0 (mean) or 1 (max)");
    if (c->d_head != kD || c->d_latent != kDL || c->pool != kPool || c->block != kBlockKeys ||
        c->bucket_mean != 8 || c->bucket_max != 16)
        return set_error(LSA_EUNSUPPORTED,
                         "cfg: this library implements d_head 128, d_latent 64, pool 4, block 512, "
                         "bucket_mean 8, bucket_max 16");
    if (c->k > 4096) return set_error(LSA_EUNSUPPORTED, "cfg: k > 4096");
    if (c->beam > 8) return set_error(LSA_EUNSUPPORTED, "cfg: beam > 8");
    if ((int64_t)c->sinks + c->k + c->window > (1 << 20))
        return set_error(LSA_EUNSUPPORTED, "cfg: index row longer than 2^20");
    return LSA_OK;
}

static lsa_status check_heads(int32_t hq, int32_t hkv) {
    if (hkv <= 0 || hq <= 0 || hq % hkv != 0) return set_error(LSA_EINVAL, "heads: need hq %% hkv == 0, both > 0");
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return set_error(LSA_EUNSUPPORTED, "heads: hq / hkv must be 1, 2, 4 or 8 (got %d)", G);
    if (hkv > 65535) return set_error(LSA_EUNSUPPORTED, "heads: hkv > 65535");
    return LSA_OK;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static lsa_status check_cache(const lsa_cache* c, bool need_built) {
    if (!c) return set_error(LSA_EINVAL, "cache is NULL");
    if (c->hkv <= 0) return set_error(LSA_EINVAL, "cache: hkv must be positive");
    if (!c->U || !c->bucket_of_unit || !c->members || !c->offsets || !c->cnt_lr || !c->minlr ||
        !c->maxpos || !c->sum || !c->cent || !c->units)
        return set_error(LSA_EINVAL, "cache: a device array is NULL");
    if (c->cap_units <= 0 || c->cap_buckets <= 0) return set_error(LSA_EINVAL, "cache: capacities must be positive");
    if (c->cap_buckets < ceil_div<int64_t>(c->cap_units, kUnitsPerBlock) * kBucketsPerBlock)
        return set_error(LSA_EINVAL, "cache: cap_buckets < 64 * ceil(cap_units / 128)");
    if (c->cap_units > (int64_t)1 << 30) return set_error(LSA_EUNSUPPORTED, "cache: more than 2^30 units");
    if (!aligned16(c->cent) || !aligned16(c->sum) || !aligned16(c->U) || !aligned16(c->cent8))
        return set_error(LSA_EINVAL, "cache: U, sum, cent and cent8 must be 16-byte aligned");
    if (need_built && c->n_tokens <= 0) return set_error(LSA_EINVAL, "cache: not built (n_tokens == 0)");
    if (c->n_tokens > c->cap_units * kPool) return set_error(LSA_EINVAL, "cache: n_tokens beyond capacity");
    return LSA_OK;
}

}  // namespace lsa

using namespace lsa;

extern "C" {

const char* lsa_last_error(void) { return g_err; }

int64_t lsa_launch_count(void) { return (int64_t)g_launches.load(std::memory_order_relaxed); }

void lsa_timing_begin(void) {
    std::lock_guard<std::mutex> lk(g_tmu);
    for (auto& t : g_trec) t.used = 0;
    g_timing.store(true, std::memory_order_relaxed);
}

void lsa_timing_end(void) { g_timing.store(false, std::memory_order_relaxed); }

lsa_status lsa_timing_get(const char* name, double* total_ms, int64_t* launches) {
    if (!name || !total_ms || !launches) return set_error(LSA_EINVAL, "lsa_timing_get: NULL pointer");
    std::lock_guard<std::mutex> lk(g_tmu);
    *total_ms = 0.0;
    *launches = 0;
    for (auto& t : g_trec) {
        if (strcmp(t.name, name) != 0) continue;
        for (size_t i = 0; i < t.used; ++i) {
            if (cudaEventSynchronize(t.stop[i]) != cudaSuccess)
                return set_error(LSA_ECUDA, "lsa_timing_get: event synchronize failed");
            float ms = 0.f;
            if (cudaEventElapsedTime(&ms, t.start[i], t.stop[i]) != cudaSuccess)
                return set_error(LSA_ECUDA, "lsa_timing_get: elapsed time failed");
            *total_ms += ms;
        }
        *launches = (int64_t)t.used;
    }
    return LSA_OK;
}

const char* lsa_version(void) { return "lsa-b200 0.1 (sm_100a)"; }

lsa_status lsa_cfg_default(lsa_cfg* cfg) {
    if (!cfg) return set_error(LSA_EINVAL, "cfg is NULL");
    cfg->d_head = 128; cfg->d_latent = 64; cfg->pool = 4; cfg->block = 512;
    cfg->bucket_mean = 8; cfg->bucket_max = 16; cfg->k = 2048; cfg->sinks = 4;
    cfg->window = 1024; cfg->beam = 2; cfg->mode = 0; cfg->agg = 0;
    return LSA_OK;
}

lsa_status lsa_cfg_check(const lsa_cfg* cfg) { return check_cfg(cfg); }

int64_t lsa_cache_units(const lsa_cfg* cfg, int64_t n_tokens) {
    if (!cfg || cfg->pool <= 0 || n_tokens < 0) return -1;
    return (n_tokens + cfg->pool - 1) / cfg->pool;
}

int64_t lsa_cache_buckets(const lsa_cfg* cfg, int64_t n_tokens) {
    if (!cfg || cfg->pool <= 0 || cfg->block <= 0 || cfg->bucket_mean <= 0 || n_tokens < 0) return -1;
    const int64_t units = (n_tokens + cfg->pool - 1) / cfg->pool;
    const int64_t upb = cfg->block / cfg->pool;
    return (units + upb - 1) / upb * (cfg->block / cfg->bucket_mean);
}

lsa_status lsa_tree_layout(int64_t n_buckets, lsa_tree* t) {
    if (!t) return set_error(LSA_EINVAL, "tree is NULL");
    if (n_buckets <= 0) return set_error(LSA_EINVAL, "tree: n_buckets must be positive");
    int32_t L = 0;
    int64_t n = n_buckets, off = 0;
    for (;;) {
        if (L >= LSA_MAX_LEVELS) return set_error(LSA_EUNSUPPORTED, "tree: too many levels");
        t->level_n[L] = n;
        t->level_off[L] = off;
        off += n;
        ++L;
        if (n <= 1) break;
        n = (n + 1) / 2;
    }
    t->levels = L;
    t->n_nodes = off;
    return LSA_OK;
}

int64_t lsa_fallback_rows(void) {
    unsigned long long v = 0ull, zero = 0ull;
    if (cudaMemcpyFromSymbol(&v, g_lsa_fallback_rows, sizeof(v)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_lsa_fallback_rows, &zero, sizeof(zero));
    return (int64_t)v;
}

lsa_status lsa_check_device_error(void) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_lsa_device_error, sizeof(int));
    if (e != cudaSuccess) return set_error(LSA_ECUDA, "reading device error word: %s", cudaGetErrorString(e));
    if (v == 0) return LSA_OK;
    const int zero = 0;
    cudaMemcpyToSymbol(g_lsa_device_error, &zero, sizeof(int));
    const char* what = v == kErrWardInfeasible ? "Ward: no eligible merge left"
                     : v == kErrSelectOverflow ? "select: candidate list overflow"
                     : v == kErrIndexRange ? "attention: index entry >= T"
                     : v == kErrTcTimeout  ? "tensor-core pipeline wait timed out" : "unknown";
    return set_error(LSA_EDEVICE, "device error %d: %s", v, what);
}

lsa_status lsa_build_buckets(const uint16_t* K, int64_t T, int32_t hkv, const float* W_k,
                             const lsa_cfg* cfg, lsa_cache* cache, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_cache(cache, false)) != LSA_OK) return s;
    if (!K || !W_k) return set_error(LSA_EINVAL, "lsa_build_buckets: K or W_k is NULL");
    if (T <= 0) return set_error(LSA_EINVAL, "lsa_build_buckets: T must be positive");
    if (hkv != cache->hkv) return set_error(LSA_EINVAL, "lsa_build_buckets: hkv != cache->hkv");
    if (!aligned16(K)) return set_error(LSA_EINVAL, "lsa_build_buckets: K must be 16-byte aligned");
    const int64_t NU = ceil_div<int64_t>(T, kPool);
    if (NU > cache->cap_units)
        return set_error(LSA_ENOSPACE, "lsa_build_buckets: %lld units > cap_units %lld", (long long)NU,
                         (long long)cache->cap_units);
    cudaStream_t st = (cudaStream_t)stream;
    if ((s = launch_key_latent(K, T, hkv, W_k, 0, NU, cache->cap_units, cache->U, st)) != LSA_OK) return s;
    const int64_t nblk = ceil_div<int64_t>(NU, kUnitsPerBlock);
    if ((s = launch_ward(cache, T, cfg->sinks, 0, nblk, st)) != LSA_OK) return s;
    // unused slots after the last block stay empty
    const int64_t NB = nblk * kBucketsPerBlock;
    if ((s = launch_clear_slots(cache, NB, cache->cap_buckets, st)) != LSA_OK) return s;
    cache->n_tokens = T;
    return LSA_OK;
}

lsa_status lsa_build_tree(const lsa_cache* cache, const lsa_cfg* cfg, lsa_tree* tree, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_cache(cache, true)) != LSA_OK) return s;
    if (!tree || !tree->sum || !tree->minlr || !tree->cent) return set_error(LSA_EINVAL, "lsa_build_tree: tree arrays are NULL");
    lsa_tree ref;
    lsa_tree_layout(cache->cap_buckets, &ref);
    if (tree->levels != ref.levels || tree->n_nodes != ref.n_nodes)
        return set_error(LSA_EINVAL, "lsa_build_tree: tree layout does not match cache->cap_buckets");
    return launch_tree_update(cache, tree, 0, cache->cap_buckets, (cudaStream_t)stream);
}

lsa_status lsa_query_latent(const uint16_t* Q, int64_t nq, int32_t hq, int32_t hkv, const float* W_q,
                            const lsa_cfg* cfg, uint16_t* Y, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!Q || !W_q || !Y) return set_error(LSA_EINVAL, "lsa_query_latent: NULL pointer");
    if (nq < 0) return set_error(LSA_EINVAL, "lsa_query_latent: nq < 0");
    if (!aligned16(Q)) return set_error(LSA_EINVAL, "lsa_query_latent: Q must be 16-byte aligned");
    return launch_query_latent(Q, nq, hq, hkv, W_q, cfg->agg, Y, (cudaStream_t)stream);
}

size_t lsa_select_workspace_bytes(const lsa_cfg* cfg, int64_t nq, int32_t hq, const lsa_cache* cache) {
    if (check_cfg(cfg) != LSA_OK || !cache || cache->hkv <= 0 || nq <= 0) return 0;
    const int64_t NU = ceil_div<int64_t>(cache->n_tokens > 0 ? cache->n_tokens : cache->cap_units * kPool, kPool);
    const int64_t NB = ceil_div<int64_t>(NU, kUnitsPerBlock) * kBucketsPerBlock;
    return select_ws_bytes(cfg, nq, hq, cache->hkv, NB);
}

lsa_status lsa_select(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq, const float* W_q,
                      const lsa_cache* cache, const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                      uint16_t* Y_out, void* ws, size_t ws_bytes, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_cache(cache, true)) != LSA_OK) return s;
    if ((s = check_heads(hq, cache->hkv)) != LSA_OK) return s;
    if (!Q || !W_q || !idx) return set_error(LSA_EINVAL, "lsa_select: NULL pointer");
    if (!aligned16(Q)) return set_error(LSA_EINVAL, "lsa_select: Q must be 16-byte aligned");
    if (Y_out && !aligned16(Y_out)) return set_error(LSA_EINVAL, "lsa_select: Y_out must be 16-byte aligned");
    if (nq <= 0 || t0 < 0) return set_error(LSA_EINVAL, "lsa_select: need nq > 0 and t0 >= 0");
    if (t0 + nq > (int64_t)INT32_MAX) return set_error(LSA_EUNSUPPORTED, "lsa_select: positions beyond 2^31");
    if (cfg->mode == 1) {
        if (!tree || !tree->minlr || !tree->cent) return set_error(LSA_EINVAL, "lsa_select: tree mode needs a built tree");
        lsa_tree ref;
        lsa_tree_layout(cache->cap_buckets, &ref);
        if (tree->levels != ref.levels || tree->n_nodes != ref.n_nodes)
            return set_error(LSA_EINVAL, "lsa_select: tree layout does not match the cache");
    }
    if (!ws && ws_bytes > 0) return set_error(LSA_EINVAL, "lsa_select: ws is NULL");
    return run_select(Q, t0, nq, hq, W_q, cache, tree, cfg, idx, Y_out, ws, ws_bytes, (cudaStream_t)stream, nullptr);
}

lsa_status lsa_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                           int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t T, uint16_t* O,
                           void* stream) {
    lsa_status s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!Q || !K || !V || !idx || !O) return set_error(LSA_EINVAL, "lsa_sparse_attn: NULL pointer");
    if (nq < 0 || n_idx < 0 || T < 0) return set_error(LSA_EINVAL, "lsa_sparse_attn: negative size");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return set_error(LSA_EINVAL, "lsa_sparse_attn: Q, K, V, O must be 16-byte aligned");
    if (T > (int64_t)INT32_MAX) return set_error(LSA_EUNSUPPORTED, "lsa_sparse_attn: T beyond 2^31");
    return launch_attn(Q, K, V, idx, nq, hq, hkv, n_idx, T, O, (cudaStream_t)stream, 0, 1, -1, nullptr, nullptr,
                       nullptr, nullptr, 0);
}

size_t lsa_select_attn_workspace_bytes(int64_t nq, int32_t hq) {
    if (nq <= 0 || hq <= 0) return 0;
    return (((size_t)nq * hq * kD * 4 + 255) & ~(size_t)255) + (((size_t)nq * hq * 4 + 255) & ~(size_t)255);
}

lsa_status lsa_select_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx, int64_t t0,
                           int64_t nq, int32_t hq, int32_t hkv, int64_t T, const lsa_cfg* cfg, uint16_t* O, void* ws,
                           size_t ws_bytes, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!Q || !K || !V || !idx || !O || (!ws && nq > 0)) return set_error(LSA_EINVAL, "lsa_select_attn: NULL pointer");
    if (nq < 0 || t0 < 0 || T < 0) return set_error(LSA_EINVAL, "lsa_select_attn: negative size");
    if (t0 + nq > T) return set_error(LSA_EINVAL, "lsa_select_attn: query positions beyond T");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(ws))
        return set_error(LSA_EINVAL, "lsa_select_attn: Q, K, V, O, ws must be 16-byte aligned");
    if (T > (int64_t)INT32_MAX) return set_error(LSA_EUNSUPPORTED, "lsa_select_attn: T beyond 2^31");
    if (nq == 0) return LSA_OK;
    const size_t need = lsa_select_attn_workspace_bytes(nq, hq);
    if (ws_bytes < need) return set_error(LSA_ENOSPACE, "lsa_select_attn: workspace %zu < %zu bytes", ws_bytes, need);
    float* Ow = (float*)ws;
    float* lse = (float*)((char*)ws + (((size_t)nq * hq * kD * 4 + 255) & ~(size_t)255));
    const cudaStream_t st = (cudaStream_t)stream;
    const int32_t row = cfg->sinks + cfg->k + cfg->window;
    // the rows' window part [S + k, S + k + W) is the contiguous range
    // max(S, t - W + 1) .. t: attend to it as a band, then gather the sinks
    // and long-range entries and merge the two softmax states
    if ((s = launch_band_attn(Q, K, V, nq, t0, T, hq, hkv, cfg->sinks, cfg->window, Ow, lse, st)) != LSA_OK) return s;
    return launch_attn(Q, K, V, idx, nq, hq, hkv, row, T, O, st, 0, 1, cfg->sinks + cfg->k, Ow, lse,
                       nullptr, nullptr, 0);
}


// Query positions per prefill chunk: `chunk` (all of T if <= 0 or larger);
// in flat mode the nearest multiple of the flat search's own wave-aligned
// chunk (at least one, at most T), so every select call but the last fills
// whole waves.
// Prefill workspace ahead of the select workspace: the chunk's index rows,
// then the sliding-window partial output (fp32) and its log-sum-exp.
struct PrefillWs {
    size_t idx_bytes, ow_bytes, lse_bytes, total;
};
static PrefillWs prefill_ws_layout(const lsa_cfg* cfg, int64_t chunk, int32_t hq, int32_t hkv) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    PrefillWs w;
    w.idx_bytes = al((size_t)chunk * hkv * (cfg->sinks + cfg->k + cfg->window) * 4);
    w.ow_bytes = al((size_t)chunk * hq * kD * 4);
    w.lse_bytes = al((size_t)chunk * hq * 4);
    w.total = w.idx_bytes + w.ow_bytes + w.lse_bytes;
    return w;
}

static int64_t prefill_chunk(const lsa_cfg* cfg, int64_t T, int32_t hq, int32_t hkv, int64_t chunk) {
    if (chunk <= 0 || chunk > T) chunk = T;
    if (cfg->mode == 0 && hkv > 0 && hq > 0 && chunk < T) {
        const int64_t sc = lsa::select_wave_rows(cfg, hq, hkv);
        int64_t m = (chunk + sc / 2) / sc;
        if (m < 1) m = 1;
        chunk = m * sc < T ? m * sc : T;
    }
    return chunk;
}

int64_t lsa_prefill_chunk(const lsa_cfg* cfg, int64_t T, int32_t hq, int32_t hkv, int64_t chunk) {
    if (check_cfg(cfg) != LSA_OK || T <= 0 || hq <= 0 || hkv <= 0) return -1;
    return prefill_chunk(cfg, T, hq, hkv, chunk);
}

size_t lsa_prefill_workspace_bytes(const lsa_cfg* cfg, int64_t T, int32_t hq, int32_t hkv, int64_t chunk) {
    if (check_cfg(cfg) != LSA_OK || T <= 0 || hkv <= 0) return 0;
    chunk = prefill_chunk(cfg, T, hq, hkv, chunk);
    const int64_t NU = ceil_div<int64_t>(T, kPool);
    const int64_t NB = ceil_div<int64_t>(NU, kUnitsPerBlock) * kBucketsPerBlock;
    return prefill_ws_layout(cfg, chunk, hq, hkv).total + select_ws_bytes(cfg, chunk, hq, hkv, NB);
}

lsa_status lsa_prefill(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t T, int32_t hq,
                       int32_t hkv, const float* W_k, const float* W_q, const lsa_cfg* cfg,
                       lsa_cache* cache, lsa_tree* tree, uint16_t* O, int64_t chunk, void* ws,
                       size_t ws_bytes, void* stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!Q || !K || !V || !O || !W_k || !W_q || !ws) return set_error(LSA_EINVAL, "lsa_prefill: NULL pointer");
    chunk = prefill_chunk(cfg, T, hq, hkv, chunk);
    const size_t need = lsa_prefill_workspace_bytes(cfg, T, hq, hkv, chunk);
    if (ws_bytes < need) return set_error(LSA_ENOSPACE, "lsa_prefill: workspace %zu < %zu bytes", ws_bytes, need);
    if ((s = lsa_build_buckets(K, T, hkv, W_k, cfg, cache, stream)) != LSA_OK) return s;
    if (cfg->mode == 1 && (s = lsa_build_tree(cache, cfg, tree, stream)) != LSA_OK) return s;
    const PrefillWs pw = prefill_ws_layout(cfg, chunk, hq, hkv);
    int32_t* idx = (int32_t*)ws;
    void* aws = (char*)ws + pw.idx_bytes;
    void* sws = (char*)ws + pw.total;
    const size_t sws_bytes = ws_bytes - pw.total;
    for (int64_t t0 = 0; t0 < T; t0 += chunk) {
        const int64_t n = (T - t0) < chunk ? (T - t0) : chunk;
        const uint16_t* Qc = Q + t0 * hq * kD;
        if ((s = lsa_select(Qc, t0, n, hq, W_q, cache, tree, cfg, idx, nullptr, sws, sws_bytes, stream)) != LSA_OK)
            return s;
        if ((s = lsa_select_attn(Qc, K, V, idx, t0, n, hq, hkv, T, cfg, O + t0 * hq * kD, aws,
                                 pw.ow_bytes + pw.lse_bytes, stream)) != LSA_OK)
            return s;
    }
    return LSA_OK;
}

lsa_status lsa_prefill_host(const uint16_t* hQ, const uint16_t* hK, const uint16_t* hV, uint16_t* hO,
                            uint16_t* Q, uint16_t* K, uint16_t* V, uint16_t* O, int64_t T, int32_t hq,
                            int32_t hkv, const float* W_k, const float* W_q, const lsa_cfg* cfg,
                            lsa_cache* cache, lsa_tree* tree, int64_t chunk, void* ws, size_t ws_bytes,
                            void* stream, void* h2d_stream, void* d2h_stream) {
    lsa_status s;
    if ((s = check_cfg(cfg)) != LSA_OK) return s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!hQ || !hK || !hV || !hO) return set_error(LSA_EINVAL, "lsa_prefill_host: NULL host pointer");
    if (!Q || !K || !V || !O || !W_k || !W_q || !ws) return set_error(LSA_EINVAL, "lsa_prefill_host: NULL pointer");
    if (T <= 0) return set_error(LSA_EINVAL, "lsa_prefill_host: T must be positive");
    chunk = prefill_chunk(cfg, T, hq, hkv, chunk);
    const size_t need = lsa_prefill_workspace_bytes(cfg, T, hq, hkv, chunk);
    if (ws_bytes < need) return set_error(LSA_ENOSPACE, "lsa_prefill_host: workspace %zu < %zu bytes", ws_bytes, need);
    cudaStream_t st = (cudaStream_t)stream, up = (cudaStream_t)h2d_stream, down = (cudaStream_t)d2h_stream;
    const int64_t nch = (T + chunk - 1) / chunk;
    const size_t qrow = (size_t)hq * kD * 2, kvrow = (size_t)hkv * kD * 2;
    // events: start, K landed, per chunk (Q and V rows landed, O written, O copied back)
    std::vector<cudaEvent_t> ev((size_t)(2 + 3 * nch), nullptr);
    auto cleanup = [&]() {
        for (auto& e : ev)
            if (e) cudaEventDestroy(e);  // released once complete
    };
    for (auto& e : ev)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
            e = nullptr;
            cleanup();
            return set_error(LSA_ECUDA, "lsa_prefill_host: cudaEventCreate failed");
        }
    cudaEvent_t e_start = ev[0], e_k = ev[1];
    auto e_in = [&](int64_t i) { return ev[2 + 3 * i]; };
    auto e_out = [&](int64_t i) { return ev[3 + 3 * i]; };
    auto e_back = [&](int64_t i) { return ev[4 + 3 * i]; };
    auto fail = [&](const char* what) {
        cleanup();
        return set_error(LSA_ECUDA, "lsa_prefill_host: %s: %s", what, cudaGetErrorString(cudaGetLastError()));
    };
    // uploads: K whole (the build needs every key), then per chunk its Q rows
    // and V rows; they start after the work already queued on `stream`
    if (cudaEventRecord(e_start, st) != cudaSuccess || cudaStreamWaitEvent(up, e_start, 0) != cudaSuccess)
        return fail("event");
    if (cudaMemcpyAsync(K, hK, (size_t)T * kvrow, cudaMemcpyHostToDevice, up) != cudaSuccess) return fail("K upload");
    if (cudaEventRecord(e_k, up) != cudaSuccess) return fail("event");
    for (int64_t i = 0; i < nch; ++i) {
        const int64_t t0 = i * chunk, n = (T - t0) < chunk ? (T - t0) : chunk;
        if (cudaMemcpyAsync(Q + t0 * hq * kD, hQ + t0 * hq * kD, (size_t)n * qrow, cudaMemcpyHostToDevice, up) !=
                cudaSuccess ||
            cudaMemcpyAsync(V + t0 * hkv * kD, hV + t0 * hkv * kD, (size_t)n * kvrow, cudaMemcpyHostToDevice, up) !=
                cudaSuccess)
            return fail("Q/V upload");
        if (cudaEventRecord(e_in(i), up) != cudaSuccess) return fail("event");
    }
    // compute, with each chunk's output copied back as soon as it is written
    if (cudaStreamWaitEvent(st, e_k, 0) != cudaSuccess) return fail("event");
    if ((s = lsa_build_buckets(K, T, hkv, W_k, cfg, cache, stream)) != LSA_OK) { cleanup(); return s; }
    if (cfg->mode == 1 && (s = lsa_build_tree(cache, cfg, tree, stream)) != LSA_OK) { cleanup(); return s; }
    const PrefillWs pw = prefill_ws_layout(cfg, chunk, hq, hkv);
    int32_t* idx = (int32_t*)ws;
    void* aws = (char*)ws + pw.idx_bytes;
    void* sws = (char*)ws + pw.total;
    const size_t sws_bytes = ws_bytes - pw.total;
    for (int64_t i = 0; i < nch; ++i) {
        const int64_t t0 = i * chunk, n = (T - t0) < chunk ? (T - t0) : chunk;
        if (cudaStreamWaitEvent(st, e_in(i), 0) != cudaSuccess) return fail("event");
        const uint16_t* Qc = Q + t0 * hq * kD;
        if ((s = lsa_select(Qc, t0, n, hq, W_q, cache, tree, cfg, idx, nullptr, sws, sws_bytes, stream)) != LSA_OK ||
            (s = lsa_select_attn(Qc, K, V, idx, t0, n, hq, hkv, T, cfg, O + t0 * hq * kD, aws,
                                 pw.ow_bytes + pw.lse_bytes, stream)) != LSA_OK) {
            cleanup();
            return s;
        }
        if (cudaEventRecord(e_out(i), st) != cudaSuccess || cudaStreamWaitEvent(down, e_out(i), 0) != cudaSuccess)
            return fail("event");
        if (cudaMemcpyAsync(hO + t0 * hq * kD, O + t0 * hq * kD, (size_t)n * qrow, cudaMemcpyDeviceToHost, down) !=
            cudaSuccess)
            return fail("O download");
        if (cudaEventRecord(e_back(i), down) != cudaSuccess) return fail("event");
    }
    // the call is complete on `stream` once the last copy back has landed
    if (cudaStreamWaitEvent(st, e_back(nch - 1), 0) != cudaSuccess) return fail("event");
    cleanup();
    return LSA_OK;
}

}  // extern "C"
