/*
 * lsa.h -- C ABI of the B200 (sm_100a) Latent Sparse Attention library
 * (liblsa.so).
 *
 * The library implements the data-parallel path of "Latent Sparse Attention:
 * Towards Subquadratic Ultra-Long Context Attention" (arXiv:2610.42147) as the
 * LSA web pages describe it:
 *   (1) key build -- every key is projected by W_k into a 64-d latent, L2
 *       normalised; every 4 consecutive keys are pooled; every 512-key cluster
 *       block is Ward-clustered into buckets (mean 8 keys, max 16) whose
 *       normalised centroids form the bucket cache  [essay "《卡片柜》——当注意力
 *       学会先查目录再翻书" (zhichai.net), ch. 2 "卡片柜的灵感——语义聚类"];
 *   (2) query scoring -- the query is projected by W_q into the same space and
 *       scored against every centroid (flat search), or taken down a complete
 *       binary tree of merged centroids by beam search (tree search); the top
 *       buckets are expanded until k long-range keys are filled
 *       [same essay, ch. 3 "查询来了怎么办" and ch. 4 "树——当卡片柜变成楼层图"];
 *       the native variant scores a bucket by the max over the group's heads
 *       [same essay, ch. 5 "两种生产方式"];
 *   (3) assembly of sinks + long-range keys + local window under a causal
 *       mask [ch. 3];
 *   (4) exact softmax attention over that index set [tutorial "隐空间稀疏注意力
 *       (LSA)" (diosapp.com.cn), section 二 "LSA 怎么工作"].
 *
 * Conventions (all entry points):
 *   - Every tensor argument is a DEVICE pointer owned by the caller, unless
 *     stated otherwise.  The library allocates no device memory and keeps no
 *     state between calls; scratch space is passed in as `ws`/`ws_bytes`.
 *   - bf16 tensors are passed as uint16_t bit patterns.  Layouts are
 *     row-major; K/V are token-major [T, hkv, d_head]; Q is [nq, hq, d_head]
 *     with query head h reading kv-head h / (hq / hkv).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous: a return of LSA_OK means the work was enqueued.
 *   - Every call returns an lsa_status; on failure nothing is enqueued and
 *     lsa_last_error() (thread-local) describes the reason.  Errors found by
 *     kernels at run time (LSA_EDEVICE) are reported through
 *     lsa_check_device_error().
 *   - Supported geometry: d_head 128, d_latent 64, pool 4, block 512,
 *     bucket_mean 8, bucket_max 16, hq / hkv in {1,2,4,8}; other values give
 *     LSA_EUNSUPPORTED.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t lsa_status;
#define LSA_OK            0
#define LSA_EINVAL        1  /* bad argument (null pointer, size, range)     */
#define LSA_EUNSUPPORTED  2  /* valid but not implemented on this library    */
#define LSA_ECUDA         3  /* a CUDA runtime call failed                   */
#define LSA_ENOSPACE      4  /* workspace or capacity too small              */
#define LSA_EDEVICE       5  /* a kernel raised its device-side error word   */

/* Method parameters; names follow the pages' notation. */
typedef struct lsa_cfg {
    int32_t d_head;      /* key/query width (128)                                 */
    int32_t d_latent;    /* latent width (64)                 [ch. 2]             */
    int32_t pool;        /* consecutive keys pooled per unit (4)  [ch. 2]         */
    int32_t block;       /* keys per cluster block (512)      [ch. 2]             */
    int32_t bucket_mean; /* mean keys per bucket (8)          [ch. 2]             */
    int32_t bucket_max;  /* max keys per bucket (16)          [ch. 2]             */
    int32_t k;           /* long-range keys per query         [ch. 3]             */
    int32_t sinks;       /* S: keys 0..S-1 always attended    [ch. 3]             */
    int32_t window;      /* W: keys t-W+1..t always attended  [ch. 3], >= 1       */
    int32_t beam;        /* beam width of tree search, 1..8   [ch. 4]             */
    int32_t mode;        /* 0 flat search, 1 tree search      [ch. 3, ch. 4]      */
    int32_t agg;         /* 0 group-mean query latent, 1 max over heads (native)  */
} lsa_cfg;

/*
 * Bucket cache of one layer (all kv-heads), caller-owned device arrays.
 * Sizes per head: cap_units >= ceil(n_tokens / pool) units and cap_buckets =
 * (block / bucket_mean) * ceil(cap_units / (block / pool)) bucket slots.
 * Bucket b of block beta is slot beta*64 + local; local ids are ordered by the
 * bucket's lowest unit; unused slots are empty (cnt_lr 0, minlr INT32_MAX,
 * maxpos -1, zero sum/centroid).
 */
typedef struct lsa_cache {
    int32_t   hkv;
    int64_t   n_tokens;        /* tokens clustered (set by the build calls)       */
    int64_t   cap_units;       /* allocated units per head                        */
    int64_t   cap_buckets;     /* allocated bucket slots per head                 */
    double*   U;               /* [hkv, cap_units, d_latent] pooled unit latents  */
    int32_t*  bucket_of_unit;  /* [hkv, cap_units]                                */
    int32_t*  members;         /* [hkv, cap_units] unit ids grouped by bucket     */
    int32_t*  offsets;         /* [hkv, cap_buckets + 1] CSR into members         */
    int32_t*  cnt_lr;          /* [hkv, cap_buckets] keys at positions >= sinks   */
    int32_t*  minlr;           /* [hkv, cap_buckets] smallest key >= sinks        */
    int32_t*  maxpos;          /* [hkv, cap_buckets] largest key                  */
    double*   sum;             /* [hkv, cap_buckets, d_latent] fp64 unit sums     */
    uint16_t* cent;            /* [hkv, cap_buckets, d_latent] bf16 centroids     */
    int32_t*  units;           /* [hkv, cap_buckets] member units packed: bits
                                  7i..7i+6 = i-th member's unit index within its
                                  128-unit block (ascending), bits 28..30 = count */
    uint8_t*  cent8;           /* optional (NULL = none), [hkv, cap_buckets,
                                  d_latent], 16-byte aligned: FP8 centroids, the
                                  OCP e4m3 code of 2^8 * c for each component c
                                  of the normalised centroid, rounded to nearest
                                  even straight from fp64 [ch. 8: the bucket
                                  cache stacks with FP8 quantisation].  When
                                  present, every build call writes them and the
                                  flat decode step (lsa_decode_step, mode 0)
                                  scores the buckets against them (64 bytes per
                                  bucket instead of 128); prefill selection
                                  (lsa_select) always scores the bf16 cent.    */
} lsa_cache;

#define LSA_MAX_LEVELS 48
#define LSA_MAX_BATCH 128

/*
 * Complete binary tree over the bucket slots of a cache [ch. 4]: level 0 =
 * the cap_buckets slots, level l+1 has ceil(n_l / 2) nodes, node i merging
 * children 2i and 2i+1.  lsa_tree_layout() fills levels/level_n/level_off/
 * n_nodes; the caller then allocates the arrays (per head n_nodes entries).
 */
typedef struct lsa_tree {
    int32_t   levels;
    int64_t   level_n[LSA_MAX_LEVELS];
    int64_t   level_off[LSA_MAX_LEVELS];
    int64_t   n_nodes;         /* nodes per head                                   */
    double*   sum;             /* [hkv, n_nodes, d_latent]                         */
    int32_t*  minlr;           /* [hkv, n_nodes]                                   */
    uint16_t* cent;            /* [hkv, n_nodes, d_latent] bf16                    */
} lsa_tree;

/* ---------------------------------------------------------------- misc */

/* Human-readable reason of the last failure on this thread ("" if none). */
const char* lsa_last_error(void);
/* Library version string. */
const char* lsa_version(void);
/* Fill *cfg with the pages' parameters (d 128, latent 64, pool 4, block 512,
 * bucket mean 8 / max 16, k 2048, S 4, W 1024, beam 2, flat, mean). */
lsa_status lsa_cfg_default(lsa_cfg* cfg);
/* LSA_OK if *cfg is supported by this library, else the reason. */
lsa_status lsa_cfg_check(const lsa_cfg* cfg);
/* Units ceil(n_tokens / pool) and bucket slots for a capacity of n_tokens. */
int64_t lsa_cache_units(const lsa_cfg* cfg, int64_t n_tokens);
int64_t lsa_cache_buckets(const lsa_cfg* cfg, int64_t n_tokens);
/* Fill the tree geometry for `n_buckets` leaf slots (host-only, no CUDA). */
lsa_status lsa_tree_layout(int64_t n_buckets, lsa_tree* tree);
/* Kernels this library has launched in this process (host-side counter,
 * for diagnostics and launch accounting). */
int64_t lsa_launch_count(void);
/* Flat-search rows (query, kv-head) that took the exact fallback since the
 * last call, on the current device (diagnostics; synchronous; -1 on error). */
int64_t lsa_fallback_rows(void);
/* Read back and clear the device-side error word of the current device:
 * LSA_OK, or LSA_EDEVICE with a description in lsa_last_error(). Synchronous. */
lsa_status lsa_check_device_error(void);

/* ------------------------------------------------------------ (1) build */

/*
 * lsa_build_buckets -- key build [ch. 2].
 * K [T, hkv, d_head] bf16, W_k [d_head, d_latent] fp32 row-major (one matrix
 * per layer, shared by all heads [ch. 5]).  For every head: pooled unit
 * latents u_j = mean of normalise(k W_k) over keys 4j..4j+3 (fp64, not
 * re-normalised) -> cache->U; every 128-unit block (a 512-key cluster block;
 * a ragged last block of n units gets ceil(n/2) buckets) is Ward-clustered:
 * greedy least-Delta-SSE merges of units, clusters capped at 4 units (16
 * keys), ties to the lowest (id_A, id_B), until 64 clusters remain.  Fills
 * every cache array for tokens [0, T) and sets cache->n_tokens = T.
 * Requires cache->cap_units >= ceil(T/4) (else LSA_ENOSPACE).
 */
lsa_status lsa_build_buckets(const uint16_t* K, int64_t T, int32_t hkv,
                             const float* W_k, const lsa_cfg* cfg,
                             lsa_cache* cache, void* stream);

/*
 * lsa_build_tree -- complete binary tree over the cache's bucket slots
 * [ch. 4]: node sum = sum of its two children (fp64), minlr = min of the
 * children, centroid = bf16(sum / |sum|) (the normalised mean of every key
 * below it).  `tree` must carry lsa_tree_layout(cache->cap_buckets, ...).
 */
lsa_status lsa_build_tree(const lsa_cache* cache, const lsa_cfg* cfg,
                          lsa_tree* tree, void* stream);

/* ------------------------------------------------------ (2)+(3) select */

/*
 * lsa_query_latent -- query latents [tutorial section 二; ch. 5]:
 * y_{t,h} = normalise(q_{t,h} W_q) in fp64; agg 0 writes the group mean
 * rounded to bf16, Y [nq, hkv, d_latent]; agg 1 writes every head,
 * Y [nq, hq, d_latent].
 */
lsa_status lsa_query_latent(const uint16_t* Q, int64_t nq, int32_t hq,
                            int32_t hkv, const float* W_q, const lsa_cfg* cfg,
                            uint16_t* Y, void* stream);

/* Workspace bytes lsa_select needs for nq queries over `cache`. */
size_t lsa_select_workspace_bytes(const lsa_cfg* cfg, int64_t nq, int32_t hq,
                                  const lsa_cache* cache);

/*
 * lsa_select -- long-range key selection and index assembly [ch. 3, ch. 4].
 * Queries are the positions t = t0 .. t0+nq-1 with rows Q [nq, hq, d_head].
 * A bucket is eligible for t iff minlr <= t - W; its weight is its number of
 * keys in [S, t - W].  Flat (cfg->mode 0): eligible buckets ranked by exact
 * score (desc; lower bucket id first on ties) are expanded until exactly k
 * keys are taken, the last bucket truncated to its lowest keys.  Tree
 * (cfg->mode 1, `tree` built): beam descent from the root to level
 * L* = min{l : beam * bucket_mean * 2^l >= k}, keeping the best `beam`
 * eligible children per level, then the same fill over the buckets below the
 * final beam.  Output idx [nq, hkv, S + k + W] int32:
 *   [0,S) sinks 0..min(S,t+1)-1 | [S,S+k) long-range keys, chosen buckets in
 *   ascending id, keys ascending | [S+k, S+k+W) window max(S,t-W+1)..t;
 *   every part padded with -1.
 * Y_out (optional, may be NULL, 16-byte aligned) receives the bf16 query latents.
 * ws / ws_bytes: scratch of at least lsa_select_workspace_bytes().
 */
lsa_status lsa_select(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq,
                      const float* W_q, const lsa_cache* cache,
                      const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                      uint16_t* Y_out, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------- kernel timing */

/*
 * Kernel timing (tracing; no counterpart on the pages).  Between
 * lsa_timing_begin() and lsa_timing_end(), every launch of the library's
 * compute kernels is bracketed by two CUDA events recorded on its stream;
 * lsa_timing_get() synchronises on them and returns, for one kernel name
 * (e.g. "flat_cand_kernel", "attn_kernel"), the summed duration in ms and
 * the number of launches recorded since the last begin.  Events are created
 * on first use and reused.  A name never launched gives 0 and 0.  Host
 * thread safe; one device per process.
 */
void lsa_timing_begin(void);
void lsa_timing_end(void);
lsa_status lsa_timing_get(const char* name, double* total_ms, int64_t* launches);

/*
 * L2-to-SM read bandwidth (measurement; no counterpart on the pages).  The
 * gathered attention re-reads K/V rows that stay in L2, so its bound is the
 * rate at which the SMs can read from L2, which this kernel measures:
 * lsa_l2_read streams the device buffer `buf` (16-byte aligned, at least
 * 128 KiB; choose it well under the L2 size so it stays resident) `passes`
 * times with 16-byte loads that bypass L1, from `ctas` CTAs of 512 threads,
 * and writes one word per thread to `sink` (device, at least
 * lsa_l2_read_sink_bytes(ctas) bytes).  lsa_l2_read_bytes() gives the bytes
 * one launch reads (whole 128 KiB chunks of the buffer, each once a pass);
 * the caller times the launch with CUDA events on `stream`.  LSA_EINVAL on
 * NULL, misaligned or too small buffers or passes/ctas out of range.
 */
size_t lsa_l2_read_sink_bytes(int32_t ctas);
int64_t lsa_l2_read_bytes(size_t bytes, int32_t passes);
lsa_status lsa_l2_read(const void* buf, size_t bytes, int32_t passes, int32_t ctas, uint32_t* sink,
                       void* stream);

/* ------------------------------------------------------- (4) attention */

/*
 * lsa_sparse_attn -- exact softmax attention over index lists [tutorial
 * section 二]: O_{q,h} = sum_j softmax_j(q_{q,h} . k_j / sqrt(d_head)) v_j
 * over the entries j >= 0 of idx[q, h / G, 0:n_idx] (G = hq / hkv; the G
 * query heads of a group share the list).  Q [nq, hq, d_head], K/V
 * [T, hkv, d_head] bf16, idx [nq, hkv, n_idx] int32 (-1 = padding; entries
 * must be < T), O [nq, hq, d_head] bf16.  fp32 accumulation; a list with no
 * valid entry gives O = 0.
 */
lsa_status lsa_sparse_attn(const uint16_t* Q, const uint16_t* K,
                           const uint16_t* V, const int32_t* idx, int64_t nq,
                           int32_t hq, int32_t hkv, int32_t n_idx, int64_t T,
                           uint16_t* O, void* stream);

/* Workspace bytes lsa_select_attn needs for nq query positions (the
 * window's fp32 partial output and its log-sum-exp). */
size_t lsa_select_attn_workspace_bytes(int64_t nq, int32_t hq);

/*
 * lsa_select_attn -- lsa_sparse_attn for index rows in lsa_select's layout
 * (same cfg): the same result over the same entries, computed in two parts
 * [tutorial section 二: sinks and the local window are always attended].
 * The window part [S + k, S + k + W) of a row is by construction the
 * contiguous range max(S, t - W + 1) .. t, so it is not read: queries
 * t0 .. t0 + nq - 1 attend to their windows as a band (consecutive queries
 * share K/V tiles), then the sinks and long-range entries [0, S + k) are
 * gathered and the two softmax states merged.  Q [nq, hq, d_head], K/V
 * [T, hkv, d_head], O [nq, hq, d_head] bf16; idx [nq, hkv, S + k + W];
 * ws (16-byte aligned): at least lsa_select_attn_workspace_bytes(nq, hq).
 */
lsa_status lsa_select_attn(const uint16_t* Q, const uint16_t* K,
                           const uint16_t* V, const int32_t* idx, int64_t t0,
                           int64_t nq, int32_t hq, int32_t hkv, int64_t T,
                           const lsa_cfg* cfg, uint16_t* O, void* ws,
                           size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ decode */

/*
 * Batched decode state of one layer, `batch` requests of one geometry
 * [essay ch. 2: each completed 512-key block is clustered once, while
 * streaming].  All arrays are caller-owned device memory except `len`.
 * The cache's heads are (request, kv-head) pairs: head r*hkv + h.
 *   K, V    [batch, cap, hkv, d_head] bf16: request r's token t is row r*cap + t.
 *   U_blk   [batch*hkv, 128, d_latent] fp64: pooled units of the block each
 *           request is filling (a complete unit holds its mean, the unit in
 *           progress the running sum of its key latents).
 *   cache   lsa_cache with hkv = batch*hkv, cap_units = cap/4,
 *           cap_buckets = 64*cap/512; cache.U is not used (may be NULL).
 *   tree    tree mode only: lsa_tree_layout(cache.cap_buckets), arrays
 *           [batch*hkv, n_nodes, ...].
 *   len     tokens each request holds (host memory, in this struct); set by
 *           lsa_decode_load and advanced by lsa_decode_step.
 * cap must be a multiple of 512; batch <= LSA_MAX_BATCH.
 *
 * Shared prefix (optional; K_shared = V_shared = NULL, shared_len = 0 for
 * none): every request starts with the same shared_len tokens, whose rows
 * are read from K_shared / V_shared [shared_len, hkv, d_head] (caller-owned,
 * read only).  The pools K, V then hold only each request's tail:
 * [batch, cap - shared_len, hkv, d_head], request r's token t >= shared_len
 * at row r*(cap - shared_len) + (t - shared_len).  shared_len is a multiple
 * of 512 below cap, and lsa_decode_load needs n >= shared_len.  Each request
 * keeps its own cache (its blocks are clustered once per request).
 */
typedef struct lsa_decode {
    int32_t   batch, hkv, hq;
    int64_t   cap;
    uint16_t* K;
    uint16_t* V;
    double*   U_blk;
    lsa_cache cache;
    lsa_tree  tree;
    int64_t   len[LSA_MAX_BATCH];
    const uint16_t* K_shared;
    const uint16_t* V_shared;
    int64_t   shared_len;
} lsa_decode;

/* Workspace bytes of lsa_decode_load / lsa_decode_step for this state. */
size_t lsa_decode_workspace_bytes(const lsa_cfg* cfg, const lsa_decode* d);

/*
 * lsa_decode_load -- make request r hold the n tokens whose K/V rows the
 * caller has written at rows r*cap .. r*cap+n-1: clusters its complete
 * blocks (as lsa_build_buckets), pools the keys of the block in progress into
 * U_blk, empties the later bucket slots, builds its tree (tree mode) and
 * sets len[r] = n.  Requires n < cap.
 */
lsa_status lsa_decode_load(lsa_decode* d, int32_t r, int64_t n, const float* W_k,
                           const lsa_cfg* cfg, void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_decode_step -- one new token per request [essay ch. 2-4; tutorial §二].
 * q [batch, hq, d], k/v [batch, hkv, d] bf16 (token t = len[r] of request r),
 * o [batch, hq, d] bf16.  Appends k/v at t; pools its key latent; clusters a
 * block completed by t (Ward, exactly as prefill) and updates the tree above
 * it; then selects for query position t over the clustered blocks (flat or
 * tree, as lsa_select) and attends over sinks + long-range keys + window
 * (the window includes the new token).  len[r] advances by one.  With
 * W >= 512 the selection equals lsa_select's at the same position.
 * idx_out (optional, may be NULL): [batch, hkv, S+k+W] receives the index
 * rows (positions within each request), as lsa_select writes them.
 */
lsa_status lsa_decode_step(lsa_decode* d, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const float* W_k, const float* W_q,
                           const lsa_cfg* cfg, uint16_t* o, int32_t* idx_out, void* ws,
                           size_t ws_bytes, void* stream);

/* ---------------------------------------------- selection without ws */

/*
 * lsa_select_noalloc -- lsa_select for callers that cannot allocate device
 * memory (a host framework that owns all device memory through its own
 * pool, or a latency-critical path that must not call cudaMalloc).  The
 * pages have no counterpart of this call; it is a deployment convenience.
 * Same arguments and results as lsa_select, minus Y_out and the workspace:
 * the scratch is one built-in device array of
 * lsa_select_noalloc_scratch_bytes() bytes (64 MiB) that every GPU loading
 * this library reserves until the process exits.
 *   - A request whose lsa_select_workspace_bytes() exceeds that size is
 *     refused with LSA_ENOSPACE (split the query range into smaller calls;
 *     e.g. 512 queries fit at 131072 keys x 8 kv-heads).  Flat search also
 *     needs scratch that grows with the cache, about 1 KB per bucket slot
 *     for 8 kv-heads, whatever nq: the largest flat-mode cache is about 512K
 *     tokens at 8 kv-heads, and a larger one is refused with LSA_ENOSPACE
 *     and a message saying so.  Tree mode's scratch does not grow with the
 *     cache.
 *   - `stream` must belong to the current device (the scratch address is
 *     that device's); another device's stream gives LSA_EINVAL.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first
 *     call before any stream capture.
 *   - Every call shares the one array: calls that can overlap on the GPU
 *     (different streams, different host threads) race and must be
 *     serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
lsa_status lsa_select_noalloc(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq,
                              const float* W_q, const lsa_cache* cache,
                              const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                              void* stream);
/* Size in bytes of lsa_select_noalloc's built-in scratch array. */
size_t lsa_select_noalloc_scratch_bytes(void);

/* --------------------------------------------------- whole-layer prefill */

/* The query chunk lsa_prefill uses for a requested `chunk` (see below);
 * -1 on invalid arguments. */
int64_t lsa_prefill_chunk(const lsa_cfg* cfg, int64_t T, int32_t hq,
                          int32_t hkv, int64_t chunk);

/* Workspace bytes lsa_prefill needs (T tokens, queries processed in chunks
 * of `chunk` positions; chunk <= 0 means all of T; in flat mode the chunk
 * becomes the nearest multiple of the flat search's wave-aligned chunk,
 * at least one and at most T). */
size_t lsa_prefill_workspace_bytes(const lsa_cfg* cfg, int64_t T, int32_t hq,
                                   int32_t hkv, int64_t chunk);

/*
 * lsa_prefill -- one LSA attention layer over a prompt of T tokens:
 * lsa_build_buckets, lsa_build_tree (tree mode), then per chunk of `chunk`
 * query positions lsa_select + lsa_select_attn.  Q [T, hq, d], K/V
 * [T, hkv, d], O [T, hq, d] bf16; cache/tree as for the calls above.
 */
lsa_status lsa_prefill(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                       int64_t T, int32_t hq, int32_t hkv, const float* W_k,
                       const float* W_q, const lsa_cfg* cfg, lsa_cache* cache,
                       lsa_tree* tree, uint16_t* O, int64_t chunk, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * lsa_prefill_host -- lsa_prefill from pinned HOST buffers hQ, hK, hV into
 * the pinned host buffer hO, with the transfers overlapped with the compute:
 * on `h2d_stream` K is uploaded whole (the build needs every key), then per
 * chunk its Q rows and V rows; the layer runs on `stream` (each chunk waits
 * for its rows only); each chunk's O rows go back on `d2h_stream` as soon as
 * they are written.  Q, K, V, O are the caller's device buffers for the
 * layer ([T, hq or hkv, d] bf16), the rest as for lsa_prefill.  The uploads
 * start after the work already queued on `stream`, and the call is complete
 * on `stream` once the last O rows are on the host.  The three streams
 * should be distinct for the copies to overlap (NULL = the legacy default
 * stream, which serialises them).  Events are created and released inside.
 */
lsa_status lsa_prefill_host(const uint16_t* hQ, const uint16_t* hK, const uint16_t* hV,
                            uint16_t* hO, uint16_t* Q, uint16_t* K, uint16_t* V, uint16_t* O,
                            int64_t T, int32_t hq, int32_t hkv, const float* W_k,
                            const float* W_q, const lsa_cfg* cfg, lsa_cache* cache,
                            lsa_tree* tree, int64_t chunk, void* ws, size_t ws_bytes,
                            void* stream, void* h2d_stream, void* d2h_stream);

/* ------------------------------------------- training-free projection */

/* Workspace bytes of lsa_fit_pca (independent of T beyond T > 0). */
size_t lsa_fit_pca_workspace_bytes(int64_t T, int32_t hkv);

/*
 * lsa_fit_pca -- the training-free projection of the distilled variant: the
 * leading d_latent principal directions of the layer's keys, used as W_k
 * (and as W_q: queries are projected onto the same directions)
 * [tutorial "隐空间稀疏注意力 (LSA)"; essay ch. 5 and closing remarks: PCA of
 * the keys, the leading 64 directions as the projection, no training].
 * K [T, hkv, d_head] bf16, 16-byte aligned; every key of every kv-head
 * counts once.  Computes the centred covariance C = (1/N) sum (k - mean)
 * (k - mean)^T (fp64, N = T*hkv) and its eigen-decomposition (cyclic Jacobi,
 * fp64); directions ordered by eigenvalue, largest first (equal eigenvalues:
 * lower Jacobi index first); each direction's first largest-magnitude
 * component is positive.  W_out [d_head, d_latent] fp32 row-major, column r
 * = direction r (rounded to nearest).  eig_out (optional, may be NULL):
 * [d_head] fp64 eigenvalues, descending.  Requires ws_bytes >=
 * lsa_fit_pca_workspace_bytes(T, hkv).
 */
lsa_status lsa_fit_pca(const uint16_t* K, int64_t T, int32_t hkv, int32_t d_latent,
                       float* W_out, double* eig_out, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Gradient of the sparse attention over saved index lists [tutorial
 * "隐空间稀疏注意力 (LSA)", section 二: the attention; essay "《卡片柜》",
 * ch. 6: the natively trained variant's backward keeps every query's
 * selected key indices].  The selection carries no gradient.  For every
 * (query, head h) with row idx[q, h / G, :] (entries < 0 are padding), with
 * s_j = q.k_j / sqrt(d), p = softmax(s) and D = dO . O:
 *   dQ[q, h]  = (1/sqrt(d)) sum_j p_j (dO . v_j - D) k_j      (written)
 *   dK[j, g] += (1/sqrt(d)) p_j (dO . v_j - D) q              (added)
 *   dV[j, g] += p_j dO                                        (added)
 * Q, O, dO [nq, hq, d_head] bf16 (O: the forward's output for the same rows);
 * K, V [T, hkv, d_head] bf16; all five 16-byte aligned.  idx [nq, hkv, n_idx]
 * int32; an entry >= T raises the device error word (LSA_EDEVICE at the next
 * lsa_check_device_error) and is skipped.  dQ [nq, hq, d_head] fp32; dK, dV
 * [T, hkv, d_head] fp32, 8-byte aligned, accumulated into so that query
 * chunks add up: the caller zeroes them first.  fp32 accumulation; P and dS
 * enter the tensor-core products rounded to bf16.  Asynchronous on `stream`;
 * no workspace.  hq / hkv must be 1, 2, 4 or 8.
 */
lsa_status lsa_attn_backward(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const uint16_t* O, const uint16_t* dO, const int32_t* idx,
                             int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t T,
                             float* dQ, float* dK, float* dV, void* stream);

/* ------------------------------------------------- sequence-sharded layer */

/*
 * The layer split over the GPUs of a job by sequence position, as the pages'
 * deployments split the context (news page "开源内容": DCP8 / CP8 context
 * parallelism).  Shard r of a job holds the keys of positions [p0, p1): whole
 * 512-key blocks (p0 a multiple of 512; the last shard may end ragged), its
 * K/V rows 0 .. p1 - p0 - 1 and the bucket cache of those keys (positions
 * local to the shard).  Every shard sees every query position.  Flat search
 * only.  Per chunk of queries [t0, t0 + nq):
 *   1. lsa_shard_candidates on every shard;
 *   2. the caller all-gathers the records and counts (rank order);
 *   3. lsa_shard_merge on every shard -> its part of every index row;
 *   4. lsa_sparse_attn_partial on every shard -> (O_r, L_r);
 *   5. the caller all-gathers the partials; lsa_lse_combine -> O.
 * The union over shards of the index rows' valid entries equals lsa_select's
 * row for the whole context (sinks in the first shard, long-range keys in
 * ascending bucket id shard by shard, the window in position order), and O
 * is the attention over that union.
 */

/* Records per (query, kv-head) row of a candidate list: k / 4 + 4 (every
 * bucket a fill takes, except at most the one holding the window's edge, a
 * sink unit or the ragged last unit, holds at least one whole 4-key unit of
 * eligible keys).  0 if cfg is invalid. */
int32_t lsa_shard_cand_cap(const lsa_cfg* cfg);

/*
 * lsa_shard_build_buckets -- lsa_build_buckets over a shard's n keys K
 * [n, hkv, d_head] (positions p0 .. p0 + n - 1): sinks count only in the
 * first shard (p0 = 0).  Errors as lsa_build_buckets; LSA_EINVAL if p0 is
 * not a multiple of 512; LSA_EUNSUPPORTED for sinks > 512.
 */
lsa_status lsa_shard_build_buckets(const uint16_t* K, int64_t n, int32_t hkv, const float* W_k,
                                   const lsa_cfg* cfg, int64_t p0, lsa_cache* cache, void* stream);

/*
 * lsa_shard_candidates -- the shard's own flat fill [essay ch. 3] of k keys
 * for query positions t0 .. t0 + nq - 1 (global), over its cache built by
 * lsa_shard_build_buckets: per (query, kv-head) row the buckets that fill
 * takes, as 16-byte records {int32 global bucket id (64 p0 / 512 + local),
 * int32 keys taken, double exact fp64 score}, in ascending id, into rec
 * [nq, hkv, lsa_shard_cand_cap(cfg)] (device, 16-byte aligned); rec_n
 * [nq, hkv] int32 the counts.  Q [nq, hq, d_head] bf16 (the chunk's rows),
 * W_q as lsa_select; ws / ws_bytes >= lsa_select_workspace_bytes(cfg, nq,
 * hq, cache).  The global fill takes a bucket only if its shard's own fill
 * does, and at most the keys that one takes, so these records carry every
 * decision of the global fill.  LSA_EUNSUPPORTED for tree mode.
 */
lsa_status lsa_shard_candidates(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq,
                                const float* W_q, const lsa_cache* cache, int64_t p0,
                                const lsa_cfg* cfg, void* rec, int32_t* rec_n, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * lsa_shard_merge -- the global fill of k keys over every shard's records
 * (rec_all [world, nq, hkv, cap], rec_n_all [world, nq, hkv], in rank order,
 * as an all-gather leaves them): weighted radix select on the exact scores,
 * score desc, global bucket id asc, exactly k keys.  Writes shard `rank`'s
 * part of each row into idx [nq, hkv, S + k + W] (global positions): the
 * sinks (first shard only), the keys its buckets give in [S, t - W] in
 * ascending bucket id (each bucket's lowest first), and the window
 * positions [max(S, t - W + 1), t] inside [p0, p0 + n_tokens); every part
 * packed at its segment's start, -1 after.  `cache` is the shard's own.
 * LSA_EUNSUPPORTED if world * cap records do not fit shared memory.
 */
lsa_status lsa_shard_merge(const void* rec_all, const int32_t* rec_n_all, int32_t world,
                           int32_t rank, int64_t t0, int64_t nq, const lsa_cache* cache,
                           int64_t p0, const lsa_cfg* cfg, int32_t* idx, void* stream);

/*
 * lsa_sparse_attn_partial -- lsa_sparse_attn over a shard's part of the
 * index rows: entries are global positions p0 .. p0 + n_keys - 1 of the K/V
 * rows 0 .. n_keys - 1 given here (others raise the device error word and
 * are skipped).  Writes the normalised fp32 O_part [nq, hq, d_head]
 * (16-byte aligned) and lse [nq, hq] fp32, the base-2 log-sum-exp of the
 * scores scaled by log2(e) / sqrt(d_head) (-inf and O = 0 for an empty row).
 */
lsa_status lsa_sparse_attn_partial(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                   const int32_t* idx, int64_t nq, int32_t hq, int32_t hkv,
                                   int32_t n_idx, int64_t p0, int64_t n_keys, float* O_part,
                                   float* lse, void* stream);

/*
 * lsa_lse_combine -- the shards' partial attentions merged into O [nq, hq,
 * d_head] bf16: O = sum_r 2^(L_r - M) O_r / sum_r 2^(L_r - M), M = max_r L_r
 * (fp32), from O_parts [world, nq, hq, d_head] and lse_parts [world, nq, hq]
 * as lsa_sparse_attn_partial writes them.  Rows no shard attends give 0.
 */
lsa_status lsa_lse_combine(const float* O_parts, const float* lse_parts, int32_t world, int64_t nq,
                           int32_t hq, uint16_t* O, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
