/*
 * lsa_oracle.c -- plain, single-threaded fp64 CPU restatement of the Latent
 * Sparse Attention (LSA) indexer + attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or table with the CUDA library.
 *
 * Sources (web pages about "Latent Sparse Attention: Towards Subquadratic
 * Ultra-Long Context Attention", arXiv:2610.42147):
 *   [CC2] essay "《卡片柜》——当注意力学会先查目录再翻书" (zhichai.net),
 *         ch. 2 "卡片柜的灵感——语义聚类": 64-d latent, L2 normalisation,
 *         pool 4 consecutive keys, 512-key cluster block, Ward clustering to
 *         buckets of mean 8 / max 16 keys, normalised-mean centroid, bucket
 *         cache, clustering done once per completed block.
 *   [CC3] same essay, ch. 3 "查询来了怎么办": score every centroid, take the
 *         top buckets until k long-range keys are filled, plus sinks and a
 *         local window; cost ~T/8 per query.
 *   [CC4] same essay, ch. 4 "树——当卡片柜变成楼层图": complete binary tree
 *         over buckets, node = merge of two siblings, centroid = mean of all
 *         its keys, beam descent, O(log T) comparisons.
 *   [CC5] same essay, ch. 5 "两种生产方式": one W_k / W_q pair per layer;
 *         native variant scores a bucket by the max over heads.
 *   [CC6] same essay, ch. 6 "数字不说谎": natively trained LSA (N-LSA) runs
 *         forward + backward per layer; its backward keeps every query's
 *         selected key indices.
 *   [DA2] tutorial "隐空间稀疏注意力 (LSA)" (diosapp.com.cn), section 二
 *         "LSA 怎么工作": the query is projected into the same latent space;
 *         exact softmax attention over the gathered keys, scale 1/sqrt(d).
 *   [CC8] same essay, ch. 8 "亚平方版图上的新坐标": the bucket cache is
 *         compatible with FP8 / INT4 quantisation.
 *   [W63] Ward, "Hierarchical Grouping to Optimize an Objective Function",
 *         JASA 1963 (cited in the essay's references): merge the pair whose
 *         union increases the within-cluster sum of squares least.
 *
 * Where the pages leave a step open, the readings are the ones the design
 * notes list (pool before the block, no re-normalisation of pooled units,
 * Delta-SSE Ward distance with a 4-unit cap, lower index wins ties, mean over
 * the GQA group for the default variant, exact-k fill with truncation of the
 * last bucket, positional sibling pairing, beam stop level L*).
 *
 * Arithmetic order (fixed so that a second implementation can reproduce the
 * fp64 values bit for bit): every dot product and every sum runs in ascending
 * index order, accumulator starting at +0.0, one rounding per operation.
 * Compile with -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define LSAO_IMAX 2147483647

/* ------------------------------------------------------------------ bf16 */

static inline double bf(uint16_t h)
{
    union { uint32_t u; float f; } v;
    v.u = ((uint32_t)h) << 16;
    return (double)v.f;
}

double lsao_bf16_to_double(uint16_t h) { return bf(h); }

/* Round a double straight to bfloat16 (8 significant bits), ties to even. */
uint16_t lsao_bf16_rne(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    frexp(a, &e);                  /* a in [2^(e-1), 2^e) */
    int ulp_exp = e - 8;           /* spacing of 8-significant-bit numbers */
    if (e - 1 < -126) ulp_exp = -133; /* bf16 subnormal spacing */
    double r = nearbyint(ldexp(a, -ulp_exp)); /* exact scale, RNE */
    double y = ldexp(r, ulp_exp);
    float f = (float)y;            /* exact, or +inf past the bf16 range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void lsao_bf16_rne_array(const double* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = lsao_bf16_rne(x[i]);
}

/* ----------------------------------------------------- fp8 e4m3 [CC8] */

/*
 * FP8 (e4m3) centroid cache [CC8]: the essay's closing chapter names FP8 and
 * INT4 quantisation of the bucket cache as compatible with the method.
 * Reading: a centroid component c (|c| <= 1) is stored as the e4m3 code of
 * 2^8 * c, rounded to nearest, ties to even, from the fp64 normalised value
 * (no intermediate bf16); |2^8 c| <= 256 < 448, so no code saturates; its
 * value is the code's value times 2^-8.  e4m3 (OCP FP8 E4M3, "fn"): 1 sign,
 * 4 exponent bits (bias 7), 3 mantissa bits, no infinities, largest finite
 * 448, smallest subnormal 2^-9; exponent field 0 holds the subnormals m 2^-9.
 * Every such value times 2^-8 is a bf16 number, so a bf16 array can carry it
 * exactly.
 */
double lsao_e4m3_to_double(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a double straight to e4m3, ties to even, saturating at +-448. */
uint8_t lsao_e4m3_rne(double x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int ulp_exp = e - 4;          /* spacing of 4-significant-bit numbers */
    if (e - 1 < -6) ulp_exp = -9; /* subnormal spacing 2^-9 */
    double r = nearbyint(ldexp(a, -ulp_exp)) ; /* exact scale, RNE */
    double y = ldexp(r, ulp_exp);
    if (y > 448.0) y = 448.0;
    /* encode y (exactly representable now) */
    int ye;
    if (y < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)ldexp(y, 9)); /* subnormal or zero */
    frexp(y, &ye);                /* y in [2^(ye-1), 2^ye) */
    int E = ye - 1 + 7;
    int M = (int)ldexp(y, -(ye - 1) + 3) - 8;
    return (uint8_t)(sign | (uint8_t)(E << 3) | (uint8_t)M);
}

/* FP8 centroids of n fp64 bucket sums [n, dl]: code of 2^8 * s / |s| per
 * component (0 for an empty sum). */
void lsao_cent_fp8(const double* sum, int64_t n, int32_t dl, uint8_t* out)
{
    for (int64_t b = 0; b < n; ++b) {
        const double* s = sum + b * dl;
        double n2 = 0.0;
        for (int32_t c = 0; c < dl; ++c) n2 = n2 + s[c] * s[c];
        double nrm = sqrt(n2);
        for (int32_t c = 0; c < dl; ++c)
            out[b * dl + c] = lsao_e4m3_rne(nrm > 0.0 ? ldexp(s[c] / nrm, 8) : 0.0);
    }
}

/* ------------------------------------------------------- latent [CC2][DA2] */

/* z = v/|v| with v = x W (x: d bf16 values, W: d x dl fp32 row-major). */
static void latent_of(const uint16_t* x, int32_t d, const float* W, int32_t dl,
                      double* v, double* z)
{
    for (int32_t c = 0; c < dl; ++c) {
        double s = 0.0;
        for (int32_t e = 0; e < d; ++e)
            s = s + bf(x[e]) * (double)W[(int64_t)e * dl + c];
        v[c] = s;
    }
    double n2 = 0.0;
    for (int32_t c = 0; c < dl; ++c) n2 = n2 + v[c] * v[c];
    double nrm = sqrt(n2);
    for (int32_t c = 0; c < dl; ++c) z[c] = (nrm > 0.0) ? v[c] / nrm : 0.0;
}

/*
 * Key latent + pooling [CC2]: for every (kv-head h, unit j) the pooled unit
 * u_j = (1/n_j) * sum of the latents z of keys pool*j .. pool*j+n_j-1
 * (n_j = pool except for a ragged last unit).  Pooled units are not
 * re-normalised.  K: [T, H, d] bf16 bits.  U: [H, NU, dl].
 */
int lsao_key_latent_pool(const uint16_t* K, int64_t T, int32_t H, int32_t d,
                         const float* W, int32_t dl, int32_t pool, double* U)
{
    if (T < 0 || H <= 0 || d <= 0 || dl <= 0 || pool <= 0) return -1;
    int64_t NU = (T + pool - 1) / pool;
    double* v = (double*)malloc(sizeof(double) * dl);
    double* z = (double*)malloc(sizeof(double) * dl);
    double* acc = (double*)malloc(sizeof(double) * dl);
    for (int32_t h = 0; h < H; ++h) {
        for (int64_t j = 0; j < NU; ++j) {
            int64_t t0 = j * pool;
            int32_t n = (int32_t)((T - t0) < pool ? (T - t0) : pool);
            for (int32_t c = 0; c < dl; ++c) acc[c] = 0.0;
            for (int32_t i = 0; i < n; ++i) {
                latent_of(K + ((t0 + i) * H + h) * (int64_t)d, d, W, dl, v, z);
                for (int32_t c = 0; c < dl; ++c) acc[c] = acc[c] + z[c];
            }
            double* u = U + ((int64_t)h * NU + j) * dl;
            for (int32_t c = 0; c < dl; ++c) u[c] = acc[c] / (double)n;
        }
    }
    free(v); free(z); free(acc);
    return 0;
}

/*
 * Query latent [DA2][CC5]: y_{t,h} = normalise(q_{t,h} W_q).
 * agg == 0 (default, distilled variant): one vector per GQA group,
 *   ybar = (y_{g*G} + ... + y_{g*G+G-1}) / G, rounded to bf16.  Y: [nq, hkv, dl].
 * agg == 1 (native variant): every head's y rounded to bf16.  Y: [nq, hq, dl].
 */
int lsao_query_latent(const uint16_t* Q, int64_t nq, int32_t hq, int32_t hkv,
                      int32_t d, const float* W, int32_t dl, int32_t agg,
                      uint16_t* Y)
{
    if (hkv <= 0 || hq % hkv != 0) return -1;
    int32_t G = hq / hkv;
    double* v = (double*)malloc(sizeof(double) * dl);
    double* z = (double*)malloc(sizeof(double) * dl);
    double* acc = (double*)malloc(sizeof(double) * dl);
    for (int64_t t = 0; t < nq; ++t) {
        if (agg == 1) {
            for (int32_t h = 0; h < hq; ++h) {
                latent_of(Q + (t * hq + h) * (int64_t)d, d, W, dl, v, z);
                for (int32_t c = 0; c < dl; ++c)
                    Y[(t * hq + h) * (int64_t)dl + c] = lsao_bf16_rne(z[c]);
            }
        } else {
            for (int32_t g = 0; g < hkv; ++g) {
                for (int32_t c = 0; c < dl; ++c) acc[c] = 0.0;
                for (int32_t i = 0; i < G; ++i) {
                    latent_of(Q + (t * hq + g * G + i) * (int64_t)d, d, W, dl, v, z);
                    for (int32_t c = 0; c < dl; ++c) acc[c] = acc[c] + z[c];
                }
                for (int32_t c = 0; c < dl; ++c)
                    Y[(t * hkv + g) * (int64_t)dl + c] = lsao_bf16_rne(acc[c] / (double)G);
            }
        }
    }
    free(v); free(z); free(acc);
    return 0;
}

/* ----------------------------------------------------------- Ward [CC2][W63] */

/*
 * Increase of the within-cluster sum of squares when clusters A and B merge:
 *   Delta(A,B) = |A||B|/(|A|+|B|) * |mu_A - mu_B|^2,  mu = (sum of units)/|A|.
 */
double lsao_ward_delta(const double* sA, int32_t nA, const double* sB, int32_t nB,
                       int32_t dl)
{
    double ss = 0.0;
    for (int32_t c = 0; c < dl; ++c) {
        double df = sA[c] / (double)nA - sB[c] / (double)nB;
        ss = ss + df * df;
    }
    double f = (double)(nA * nB) / (double)(nA + nB);
    return f * ss;
}

typedef struct {
    int32_t n, dl, max_units;
    const double* U;   /* [n, dl] */
    int32_t* size;     /* units per cluster (0 = merged away) */
    int32_t* mem;      /* [n, max_units] member unit indices, ascending */
    double* sum;       /* [n, dl] canonical sums */
} ward_state;

/* Canonical cluster sum: member units added in ascending order from +0.0. */
static void cluster_sum(ward_state* w, int32_t a)
{
    double* s = w->sum + (int64_t)a * w->dl;
    for (int32_t c = 0; c < w->dl; ++c) s[c] = 0.0;
    for (int32_t i = 0; i < w->size[a]; ++i) {
        const double* u = w->U + (int64_t)w->mem[a * w->max_units + i] * w->dl;
        for (int32_t c = 0; c < w->dl; ++c) s[c] = s[c] + u[c];
    }
}

static double pair_delta(ward_state* w, int32_t a, int32_t b)
{
    if (a == b || w->size[a] == 0 || w->size[b] == 0) return INFINITY;
    if (w->size[a] + w->size[b] > w->max_units) return INFINITY;
    return lsao_ward_delta(w->sum + (int64_t)a * w->dl, w->size[a],
                           w->sum + (int64_t)b * w->dl, w->size[b], w->dl);
}

static void merge_into(ward_state* w, int32_t a, int32_t b)
{
    /* a < b; merged cluster keeps id a (its lowest member). */
    int32_t na = w->size[a], nb = w->size[b];
    int32_t tmp[64];
    int32_t i = 0, j = 0, o = 0;
    const int32_t* ma = w->mem + a * w->max_units;
    const int32_t* mb = w->mem + b * w->max_units;
    while (i < na || j < nb) {
        if (j >= nb || (i < na && ma[i] < mb[j])) tmp[o++] = ma[i++];
        else tmp[o++] = mb[j++];
    }
    for (int32_t k = 0; k < o; ++k) w->mem[a * w->max_units + k] = tmp[k];
    w->size[a] = na + nb;
    w->size[b] = 0;
    cluster_sum(w, a);
}

/*
 * Capped Ward agglomeration of one cluster block [CC2][W63].
 * Start from n singleton clusters (the block's pooled units), repeatedly merge
 * the eligible pair (size sum <= max_units) with the least Delta until
 * m_target clusters remain.  Ties: smallest (id_A, id_B), id = lowest member.
 * Result: bucket_of[i] = rank of unit i's cluster among surviving clusters
 * ordered by id.  naive != 0 recomputes every pair at every step (O(n^3 dl))
 * and reports the smallest gap between the chosen and the next-best Delta in
 * *margin; naive == 0 keeps a nearest-neighbour row array (same arithmetic).
 * Returns 0, or -1 if no eligible pair exists before m_target is reached.
 */
int lsao_ward_block(const double* U, int32_t n, int32_t dl, int32_t m_target,
                    int32_t max_units, int32_t naive, int32_t* bucket_of,
                    double* margin)
{
    if (n <= 0 || m_target <= 0 || max_units <= 0 || max_units > 64) return -1;
    ward_state w;
    w.n = n; w.dl = dl; w.max_units = max_units; w.U = U;
    w.size = (int32_t*)malloc(sizeof(int32_t) * n);
    w.mem = (int32_t*)malloc(sizeof(int32_t) * n * max_units);
    w.sum = (double*)malloc(sizeof(double) * (int64_t)n * dl);
    for (int32_t i = 0; i < n; ++i) {
        w.size[i] = 1;
        w.mem[i * max_units] = i;
        cluster_sum(&w, i);
    }
    double best_margin = INFINITY;
    int32_t clusters = n;
    int rc = 0;
    if (naive) {
        while (clusters > m_target) {
            double d1 = INFINITY, d2 = INFINITY;
            int32_t ba = -1, bb = -1;
            for (int32_t a = 0; a < n; ++a) {
                if (w.size[a] == 0) continue;
                for (int32_t b = a + 1; b < n; ++b) {
                    double dd = pair_delta(&w, a, b);
                    if (dd == INFINITY) continue;
                    if (dd < d1) { d2 = d1; d1 = dd; ba = a; bb = b; }
                    else if (dd < d2) d2 = dd;
                }
            }
            if (ba < 0) { rc = -1; break; }
            if (d2 < INFINITY && d2 - d1 < best_margin) best_margin = d2 - d1;
            merge_into(&w, ba, bb);
            --clusters;
        }
    } else {
        double* D = (double*)malloc(sizeof(double) * (int64_t)n * n);
        int32_t* nn = (int32_t*)malloc(sizeof(int32_t) * n);
        double* nnd = (double*)malloc(sizeof(double) * n);
        for (int32_t a = 0; a < n; ++a)
            for (int32_t b = 0; b < n; ++b)
                D[(int64_t)a * n + b] = (b > a) ? pair_delta(&w, a, b)
                                       : (b < a ? D[(int64_t)b * n + a] : INFINITY);
        for (int32_t r = 0; r < n; ++r) {
            nn[r] = -1; nnd[r] = INFINITY;
            for (int32_t c = 0; c < n; ++c)
                if (D[(int64_t)r * n + c] < nnd[r]) { nnd[r] = D[(int64_t)r * n + c]; nn[r] = c; }
        }
        while (clusters > m_target) {
            int32_t ba = -1, bb = -1;
            double bd = INFINITY;
            for (int32_t r = 0; r < n; ++r) {
                if (w.size[r] == 0 || nn[r] < 0) continue;
                int32_t lo = r < nn[r] ? r : nn[r], hi = r < nn[r] ? nn[r] : r;
                if (nnd[r] < bd || (nnd[r] == bd && (lo < ba || (lo == ba && hi < bb)))) {
                    bd = nnd[r]; ba = lo; bb = hi;
                }
            }
            if (ba < 0) { rc = -1; break; }
            merge_into(&w, ba, bb);
            --clusters;
            for (int32_t c = 0; c < n; ++c) {
                D[(int64_t)bb * n + c] = INFINITY;
                D[(int64_t)c * n + bb] = INFINITY;
            }
            for (int32_t c = 0; c < n; ++c) {
                double dd = pair_delta(&w, ba, c);
                D[(int64_t)ba * n + c] = dd;
                D[(int64_t)c * n + ba] = dd;
            }
            for (int32_t r = 0; r < n; ++r) {
                if (w.size[r] == 0) { nn[r] = -1; nnd[r] = INFINITY; continue; }
                if (r == ba || nn[r] == ba || nn[r] == bb) {
                    nn[r] = -1; nnd[r] = INFINITY;
                    for (int32_t c = 0; c < n; ++c)
                        if (D[(int64_t)r * n + c] < nnd[r]) { nnd[r] = D[(int64_t)r * n + c]; nn[r] = c; }
                } else {
                    double dd = D[(int64_t)r * n + ba];
                    if (dd < nnd[r] || (dd == nnd[r] && dd < INFINITY && ba < nn[r])) {
                        nnd[r] = dd; nn[r] = ba;
                    }
                }
            }
        }
        free(D); free(nn); free(nnd);
    }
    if (rc == 0) {
        int32_t rank = 0;
        for (int32_t a = 0; a < n; ++a) {
            if (w.size[a] == 0) continue;
            for (int32_t i = 0; i < w.size[a]; ++i) bucket_of[w.mem[a * max_units + i]] = rank;
            ++rank;
        }
    }
    if (margin) *margin = best_margin;
    free(w.size); free(w.mem); free(w.sum);
    return rc;
}

/* ------------------------------------------------- bucket cache [CC2][CC3] */

/*
 * Build the bucket cache of every kv-head from its pooled units U [H, NU, dl].
 * Block b of units [b*bu, min(b*bu+bu, NU)) with n units is Ward-clustered to
 * ceil(n*bpb/bu) buckets (bpb for a full block); bucket slots are
 * blk*bpb + local, local ordered by lowest member; unused slots stay empty.
 * Per bucket: CSR members (ascending unit ids), cnt_lr (#keys >= sinks),
 * minlr (smallest key >= sinks, IMAX if none), maxpos (largest key, -1 if
 * empty), canonical fp64 sum of member units, centroid = bf16(sum/|sum|).
 */
int lsao_build(const double* U, int64_t T, int32_t H, int32_t dl, int32_t pool,
               int32_t bu, int32_t bpb, int32_t max_units, int32_t sinks,
               int32_t naive, int32_t* bucket_of_unit, int32_t* members,
               int32_t* offsets, int32_t* cnt_lr, int32_t* minlr, int32_t* maxpos,
               double* sum, uint16_t* cent, double* ward_margin)
{
    int64_t NU = (T + pool - 1) / pool;
    int64_t nblk = (NU + bu - 1) / bu;
    int64_t NB = nblk * bpb;
    int32_t* loc = (int32_t*)malloc(sizeof(int32_t) * bu);
    double* s = (double*)malloc(sizeof(double) * dl);
    for (int32_t h = 0; h < H; ++h) {
        const double* Uh = U + (int64_t)h * NU * dl;
        int32_t* off = offsets + (int64_t)h * (NB + 1);
        for (int64_t blk = 0; blk < nblk; ++blk) {
            int64_t u0 = blk * bu;
            int32_t n = (int32_t)((NU - u0) < bu ? (NU - u0) : bu);
            int32_t m = (int32_t)(((int64_t)n * bpb + bu - 1) / bu);
            double mg = INFINITY;
            if (lsao_ward_block(Uh + u0 * dl, n, dl, m, max_units, naive, loc, &mg) != 0) {
                free(loc); free(s);
                return -1;
            }
            if (ward_margin) ward_margin[(int64_t)h * nblk + blk] = mg;
            int32_t pos = (int32_t)u0;
            for (int32_t lb = 0; lb < bpb; ++lb) {
                int64_t b = blk * bpb + lb;
                int64_t hb = (int64_t)h * NB + b;
                off[b] = pos;
                int32_t c_lr = 0, mlr = LSAO_IMAX, mxp = -1;
                for (int32_t c = 0; c < dl; ++c) s[c] = 0.0;
                for (int32_t i = 0; i < n; ++i) {
                    if (lb >= m || loc[i] != lb) continue;
                    int64_t j = u0 + i;
                    members[(int64_t)h * NU + pos] = (int32_t)j;
                    bucket_of_unit[(int64_t)h * NU + j] = (int32_t)b;
                    ++pos;
                    const double* u = Uh + j * dl;
                    for (int32_t c = 0; c < dl; ++c) s[c] = s[c] + u[c];
                    for (int64_t p = j * pool; p < j * pool + pool && p < T; ++p) {
                        if (p > mxp) mxp = (int32_t)p;
                        if (p >= sinks) { ++c_lr; if (p < mlr) mlr = (int32_t)p; }
                    }
                }
                cnt_lr[hb] = c_lr;
                minlr[hb] = mlr;
                maxpos[hb] = mxp;
                double n2 = 0.0;
                for (int32_t c = 0; c < dl; ++c) n2 = n2 + s[c] * s[c];
                double nrm = sqrt(n2);
                for (int32_t c = 0; c < dl; ++c) {
                    sum[hb * dl + c] = s[c];
                    cent[hb * dl + c] = lsao_bf16_rne(nrm > 0.0 ? s[c] / nrm : 0.0);
                }
            }
        }
        off[NB] = (int32_t)NU;
    }
    free(loc); free(s);
    return 0;
}

/* ------------------------------------------------------------ tree [CC4] */

/* Number of nodes on every level: n_0 = NB, n_{l+1} = ceil(n_l / 2) down to 1. */
int32_t lsao_tree_levels(int64_t NB, int64_t* level_n, int64_t* level_off)
{
    int32_t L = 0;
    int64_t n = NB, off = 0;
    for (;;) {
        level_n[L] = n;
        level_off[L] = off;
        off += n;
        ++L;
        if (n <= 1) break;
        n = (n + 1) / 2;
    }
    return L;
}

/*
 * Complete binary tree over the buckets of every head [CC4]: level 0 = the
 * buckets in id order; node i of level l merges children 2i and 2i+1 of
 * level l-1 (a missing second child gives a one-child node).  Node sum =
 * left sum + right sum (fp64), minlr = min of the children, centroid =
 * bf16(sum/|sum|) -- the normalised mean of all keys below the node.
 * tsum [H, ntot, dl], tminlr [H, ntot], tcent [H, ntot, dl].
 */
int lsao_build_tree(int64_t NB, int32_t H, int32_t dl, const double* sum,
                    const int32_t* minlr, double* tsum, int32_t* tminlr,
                    uint16_t* tcent)
{
    int64_t ln[64], lo[64];
    int32_t L = lsao_tree_levels(NB, ln, lo);
    int64_t ntot = lo[L - 1] + ln[L - 1];
    for (int32_t h = 0; h < H; ++h) {
        double* S = tsum + (int64_t)h * ntot * dl;
        int32_t* M = tminlr + (int64_t)h * ntot;
        uint16_t* C = tcent + (int64_t)h * ntot * dl;
        for (int64_t b = 0; b < NB; ++b) {
            for (int32_t c = 0; c < dl; ++c) S[b * dl + c] = sum[((int64_t)h * NB + b) * dl + c];
            M[b] = minlr[(int64_t)h * NB + b];
        }
        for (int32_t l = 1; l < L; ++l) {
            for (int64_t i = 0; i < ln[l]; ++i) {
                int64_t node = lo[l] + i, a = lo[l - 1] + 2 * i, b = a + 1;
                int has_b = (2 * i + 1) < ln[l - 1];
                for (int32_t c = 0; c < dl; ++c)
                    S[node * dl + c] = has_b ? S[a * dl + c] + S[b * dl + c] : S[a * dl + c];
                M[node] = (has_b && M[b] < M[a]) ? M[b] : M[a];
            }
        }
        for (int64_t node = 0; node < ntot; ++node) {
            double n2 = 0.0;
            for (int32_t c = 0; c < dl; ++c) n2 = n2 + S[node * dl + c] * S[node * dl + c];
            double nrm = sqrt(n2);
            for (int32_t c = 0; c < dl; ++c)
                C[node * dl + c] = lsao_bf16_rne(nrm > 0.0 ? S[node * dl + c] / nrm : 0.0);
        }
    }
    return 0;
}

/* -------------------------------------------------- selection [CC3][CC4] */

/* Exact score of a bf16 query latent against a bf16 centroid (products of two
 * bf16 numbers are exact in fp64). */
static double score1(const uint16_t* y, const uint16_t* c, int32_t dl)
{
    double s = 0.0;
    for (int32_t i = 0; i < dl; ++i)
        s = s + bf(y[i]) * bf(c[i]);
    return s;
}

typedef struct { double s; int64_t id; } scored;

/* Score of one node: the mean-variant latent, or the max over the ng heads of
 * the native variant.  Adds the number of dot products to *nc. */
static double node_score(const uint16_t* yq, int32_t ng, int32_t dl,
                         const uint16_t* c, int64_t* nc)
{
    double best = -INFINITY;
    for (int32_t g = 0; g < ng; ++g) {
        double v = score1(yq + (int64_t)g * dl, c, dl);
        if (v > best) best = v;
    }
    *nc += ng;
    return best;
}

static int cmp_scored(const void* pa, const void* pb)
{
    const scored* a = (const scored*)pa;
    const scored* b = (const scored*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->id < b->id) ? -1 : (a->id > b->id);
}

static int cmp_i64(const void* pa, const void* pb)
{
    int64_t a = ((const scored*)pa)->id, b = ((const scored*)pb)->id;
    return (a < b) ? -1 : (a > b);
}

/*
 * Selection of long-range keys for a list of queries [CC3][CC4][CC5].
 * For query position t and kv-head h, a bucket is eligible iff
 * minlr <= t - W; its weight is the number of its keys in R_t = [S, t-W].
 * Score: mean variant s = ybar . c (Y [nq, H, dl]); native variant
 * s = max over the group's G heads of y_h . c (Y [nq, H*G, dl]).
 * mode 0 (flat): rank all eligible buckets by (s desc, id asc) and take their
 *   keys in R_t (ascending within a bucket) until exactly k are taken; the
 *   last bucket is truncated to its lowest positions.
 * mode 1 (tree): beam descent from the root of the complete binary tree to
 *   level L* = min{l : beam * bucket_mean * 2^l >= k}; on every level the
 *   eligible children of the beam are scored and the best `beam` kept
 *   (score desc, node index asc); then the flat fill runs over the buckets
 *   under the final beam nodes.
 * Output row [S + k + W] per (query, head):
 *   [0, S)       sinks 0 .. min(S, t+1)-1, then -1;
 *   [S, S+k)     long-range keys: chosen buckets in ascending id, each
 *                bucket's chosen keys ascending, then -1;
 *   [S+k, S+k+W) window max(S, t-W+1) .. t ascending, then -1.
 * margin: smallest score gap around any decision (fill cut; each beam cut);
 * INFINITY if none.  ncmp: centroid evaluations (native counts G per node).
 * Tree arrays: ntot nodes per head, levels as lsao_tree_levels gives them.
 */
int lsao_select(int64_t NB, int32_t H, int32_t dl, int32_t pool, int64_t T_built,
                const int32_t* offsets, const int32_t* members,
                const int32_t* cnt_lr, const int32_t* minlr, const int32_t* maxpos,
                const uint16_t* cent, const int32_t* tminlr, const uint16_t* tcent,
                const uint16_t* Y, int32_t G, const int64_t* tpos, int64_t nq,
                int32_t k, int32_t S, int32_t W, int32_t beam, int32_t bucket_mean,
                int32_t mode, int32_t agg, int32_t* idx, double* margin,
                int64_t* ncmp)
{
    int64_t NU = (T_built + pool - 1) / pool;
    int32_t row = S + k + W;
    int64_t ln[64], lo[64];
    int32_t L = lsao_tree_levels(NB, ln, lo);
    int64_t ntot = lo[L - 1] + ln[L - 1];
    int32_t Lstar = 0;
    while ((int64_t)beam * bucket_mean * ((int64_t)1 << Lstar) < k && Lstar < 62) ++Lstar;
    int32_t hy = (agg == 1) ? H * G : H;
    scored* cand = (scored*)malloc(sizeof(scored) * (NB > 0 ? NB : 1));
    scored* lvl = (scored*)malloc(sizeof(scored) * (2 * (beam > 0 ? beam : 1) + 2));
    int64_t* bm = (int64_t*)malloc(sizeof(int64_t) * (beam > 0 ? beam : 1));
    int64_t* bm2 = (int64_t*)malloc(sizeof(int64_t) * (beam > 0 ? beam : 1));
    scored* taken = (scored*)malloc(sizeof(scored) * (NB > 0 ? NB : 1));
    int32_t* takecnt = (int32_t*)malloc(sizeof(int32_t) * (NB > 0 ? NB : 1));

    for (int64_t q = 0; q < nq; ++q) {
        int64_t t = tpos[q];
        int64_t lim = t - W;   /* last long-range key position */
        for (int32_t h = 0; h < H; ++h) {
            const int32_t* off = offsets + (int64_t)h * (NB + 1);
            const int32_t* mem = members + (int64_t)h * NU;
            const int32_t* clr = cnt_lr + (int64_t)h * NB;
            const int32_t* mlr = minlr + (int64_t)h * NB;
            const int32_t* mxp = maxpos + (int64_t)h * NB;
            const uint16_t* C = cent + (int64_t)h * NB * dl;
            const uint16_t* yq = Y + (q * hy + (agg == 1 ? h * G : h)) * (int64_t)dl;
            int32_t ng = (agg == 1) ? G : 1;
            double mg = INFINITY;
            int64_t nc = 0;
            int64_t ncand = 0;
            if (mode == 0 || Lstar >= L - 1) {
                for (int64_t b = 0; b < NB; ++b) {
                    if ((int64_t)mlr[b] > lim) continue;
                    cand[ncand].s = node_score(yq, ng, dl, C + b * dl, &nc);
                    cand[ncand].id = b;
                    ++ncand;
                }
            } else {
                const int32_t* tm = tminlr + (int64_t)h * ntot;
                const uint16_t* TC = tcent + (int64_t)h * ntot * dl;
                int32_t nbm = 0;
                if ((int64_t)tm[lo[L - 1]] <= lim) bm[nbm++] = 0;
                for (int32_t l = L - 1; l > Lstar && nbm > 0; --l) {
                    int32_t nl = 0;
                    for (int32_t i = 0; i < nbm; ++i) {
                        for (int64_t ch = 2 * bm[i]; ch <= 2 * bm[i] + 1; ++ch) {
                            if (ch >= ln[l - 1]) continue;
                            int64_t node = lo[l - 1] + ch;
                            if ((int64_t)tm[node] > lim) continue;
                            lvl[nl].s = node_score(yq, ng, dl, TC + node * dl, &nc);
                            lvl[nl].id = ch;
                            ++nl;
                        }
                    }
                    qsort(lvl, nl, sizeof(scored), cmp_scored);
                    int32_t keep = nl < beam ? nl : beam;
                    if (nl > keep) {
                        double gap = lvl[keep - 1].s - lvl[keep].s;
                        if (gap < mg) mg = gap;
                    }
                    for (int32_t i = 0; i < keep; ++i) bm2[i] = lvl[i].id;
                    nbm = keep;
                    for (int32_t i = 0; i < nbm; ++i) bm[i] = bm2[i];
                }
                /* leaves under the final beam nodes, in ascending order */
                for (int32_t i = 0; i < nbm; ++i) bm2[i] = bm[i];
                for (int32_t i = 1; i < nbm; ++i)
                    for (int32_t j2 = i; j2 > 0 && bm2[j2 - 1] > bm2[j2]; --j2) {
                        int64_t tt = bm2[j2]; bm2[j2] = bm2[j2 - 1]; bm2[j2 - 1] = tt;
                    }
                for (int32_t i = 0; i < nbm; ++i) {
                    int64_t b0 = bm2[i] << Lstar, b1 = (bm2[i] + 1) << Lstar;
                    if (b1 > NB) b1 = NB;
                    for (int64_t b = b0; b < b1; ++b) {
                        if ((int64_t)mlr[b] > lim) continue;
                        cand[ncand].s = node_score(yq, ng, dl, C + b * dl, &nc);
                        cand[ncand].id = b;
                        ++ncand;
                    }
                }
            }
            qsort(cand, ncand, sizeof(scored), cmp_scored);
            /* fill exactly k keys */
            int64_t need = k, ntaken = 0;
            int64_t last = -1;
            int last_trunc = 0;
            for (int64_t i = 0; i < ncand && need > 0; ++i) {
                int64_t b = cand[i].id;
                int64_t w;
                if ((int64_t)mxp[b] <= lim) {
                    w = clr[b];
                } else {
                    w = 0;
                    for (int32_t m = off[b]; m < off[b + 1]; ++m)
                        for (int64_t p = (int64_t)mem[m] * pool; p < (int64_t)mem[m] * pool + pool && p < T_built; ++p)
                            if (p >= S && p <= lim) ++w;
                }
                if (w <= 0) continue;
                int32_t tk = (int32_t)(w < need ? w : need);
                last_trunc = (tk < w);
                need -= tk;
                taken[ntaken].id = b;
                taken[ntaken].s = cand[i].s;
                takecnt[ntaken] = tk;
                ++ntaken;
                last = i;
            }
            if (need == 0 && last >= 0) {
                /* gap to the best untaken bucket that has a key in R_t */
                for (int64_t i = last + 1; i < ncand; ++i) {
                    double gap = cand[last].s - cand[i].s;
                    if (gap < mg) mg = gap;
                    break;
                }
                if (last_trunc && ntaken >= 2) {
                    double gap = taken[ntaken - 2].s - taken[ntaken - 1].s;
                    if (gap < mg) mg = gap;
                }
            }
            /* canonical order: ascending bucket id */
            for (int64_t i = 0; i < ntaken; ++i) taken[i].s = (double)takecnt[i];
            qsort(taken, ntaken, sizeof(scored), cmp_i64);
            int32_t* out = idx + (q * H + h) * (int64_t)row;
            for (int32_t i = 0; i < row; ++i) out[i] = -1;
            for (int32_t i = 0; i < S && i <= t; ++i) out[i] = i;
            int32_t o = S;
            for (int64_t i = 0; i < ntaken; ++i) {
                int64_t b = taken[i].id;
                int32_t rem = (int32_t)taken[i].s;
                /* keys of the bucket in R_t, ascending (members ascending) */
                for (int32_t m = off[b]; m < off[b + 1] && rem > 0; ++m)
                    for (int64_t p = (int64_t)mem[m] * pool; p < (int64_t)mem[m] * pool + pool && p < T_built && rem > 0; ++p)
                        if (p >= S && p <= lim) { out[o++] = (int32_t)p; --rem; }
            }
            if (t >= S) {
                int64_t w0 = t - W + 1 > S ? t - W + 1 : S;
                int32_t o2 = S + k;
                for (int64_t p = w0; p <= t; ++p) out[o2++] = (int32_t)p;
            }
            if (margin) margin[q * H + h] = mg;
            if (ncmp) ncmp[q * H + h] = nc;
        }
    }
    free(cand); free(lvl); free(bm); free(bm2); free(taken); free(takecnt);
    return 0;
}

/* ------------------------------------------------------ attention [DA2] */

/*
 * Exact softmax attention over an index list [DA2]:
 *   O_{q,h} = sum_j softmax_j(q_{q,h} . k_j / sqrt(d)) v_j over the valid
 *   (>= 0) entries j of idx[q, h/G, :].  Q [nq, hq, d], K/V [T, hkv, d] bf16
 *   bits, O [nq, hq, d] fp64.  An empty list gives O = 0.
 */
int lsao_attention(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                   const int32_t* idx, int64_t nq, int32_t hq, int32_t hkv,
                   int32_t d, int32_t n_idx, double* O)
{
    int32_t G = hq / hkv;
    double* lg = (double*)malloc(sizeof(double) * (n_idx > 0 ? n_idx : 1));
    double sc = 1.0 / sqrt((double)d);
    for (int64_t q = 0; q < nq; ++q) {
        for (int32_t h = 0; h < hq; ++h) {
            const int32_t* list = idx + (q * hkv + h / G) * (int64_t)n_idx;
            const uint16_t* qv = Q + (q * hq + h) * (int64_t)d;
            double* o = O + (q * hq + h) * (int64_t)d;
            double mx = -INFINITY;
            for (int32_t i = 0; i < n_idx; ++i) {
                if (list[i] < 0) continue;
                const uint16_t* kv = K + ((int64_t)list[i] * hkv + h / G) * d;
                double s = 0.0;
                for (int32_t e = 0; e < d; ++e)
                    s = s + bf(qv[e]) * bf(kv[e]);
                lg[i] = s * sc;
                if (lg[i] > mx) mx = lg[i];
            }
            for (int32_t e = 0; e < d; ++e) o[e] = 0.0;
            double den = 0.0;
            for (int32_t i = 0; i < n_idx; ++i) {
                if (list[i] < 0) continue;
                double p = exp(lg[i] - mx);
                den = den + p;
                const uint16_t* vv = V + ((int64_t)list[i] * hkv + h / G) * d;
                for (int32_t e = 0; e < d; ++e) o[e] = o[e] + p * bf(vv[e]);
            }
            if (den > 0.0)
                for (int32_t e = 0; e < d; ++e) o[e] = o[e] / den;
        }
    }
    free(lg);
    return 0;
}

/* ------------------------------------------ attention backward [DA2][CC6] */

/*
 * Gradient of the exact sparse attention above with respect to Q, K and V,
 * for saved index lists [CC6].  The selection is a discrete choice and
 * carries no gradient.  For one (query, head) with valid entries i of its list,
 * s_i = sc q.k_i (sc = 1/sqrt(d)), p = softmax(s), O = sum_i p_i v_i and the
 * output gradient g = dO:
 *   dV[k_i] += p_i g
 *   dp_i     = g . v_i,   D = g . O
 *   ds_i     = p_i (dp_i - D)
 *   dQ       = sc sum_i ds_i k_i
 *   dK[k_i] += sc ds_i q
 * Q, dO [nq, hq, d], K, V [T, hkv, d] as fp64; idx [nq, hkv, n_idx] (entries
 * < 0 are padding; every valid entry < T).  dQ [nq, hq, d], dK, dV
 * [T, hkv, d] are overwritten.  Order: queries ascending, heads ascending,
 * list entries in list order; every sum from +0.0 in ascending index order.
 */
int lsao_attention_backward(const double* Q, const double* K, const double* V,
                            const double* dO, const int32_t* idx, int64_t nq,
                            int32_t hq, int32_t hkv, int32_t d, int32_t n_idx,
                            int64_t T, double* dQ, double* dK, double* dV)
{
    if (hkv <= 0 || hq % hkv != 0 || d <= 0 || n_idx < 0 || nq < 0 || T < 0) return -1;
    int32_t G = hq / hkv;
    for (int64_t i = 0; i < T * hkv * d; ++i) { dK[i] = 0.0; dV[i] = 0.0; }
    double* p = (double*)malloc(sizeof(double) * (n_idx > 0 ? n_idx : 1));
    double* o = (double*)malloc(sizeof(double) * d);
    double sc = 1.0 / sqrt((double)d);
    for (int64_t q = 0; q < nq; ++q) {
        for (int32_t h = 0; h < hq; ++h) {
            int32_t g = h / G;
            const int32_t* list = idx + (q * hkv + g) * (int64_t)n_idx;
            const double* qv = Q + (q * hq + h) * (int64_t)d;
            const double* gv = dO + (q * hq + h) * (int64_t)d;
            double* dq = dQ + (q * hq + h) * (int64_t)d;
            for (int32_t e = 0; e < d; ++e) dq[e] = 0.0;
            /* forward again: probabilities and output */
            double mx = -INFINITY;
            for (int32_t i = 0; i < n_idx; ++i) {
                if (list[i] < 0) continue;
                if (list[i] >= T) { free(p); free(o); return -1; }
                const double* kv = K + ((int64_t)list[i] * hkv + g) * d;
                double s = 0.0;
                for (int32_t e = 0; e < d; ++e) s = s + qv[e] * kv[e];
                p[i] = s * sc;
                if (p[i] > mx) mx = p[i];
            }
            double den = 0.0;
            for (int32_t i = 0; i < n_idx; ++i) {
                if (list[i] < 0) continue;
                p[i] = exp(p[i] - mx);
                den = den + p[i];
            }
            if (!(den > 0.0)) continue;             /* empty list: no gradient */
            for (int32_t e = 0; e < d; ++e) o[e] = 0.0;
            for (int32_t i = 0; i < n_idx; ++i) {
                if (list[i] < 0) continue;
                p[i] = p[i] / den;
                const double* vv = V + ((int64_t)list[i] * hkv + g) * d;
                for (int32_t e = 0; e < d; ++e) o[e] = o[e] + p[i] * vv[e];
            }
            double D = 0.0;
            for (int32_t e = 0; e < d; ++e) D = D + gv[e] * o[e];
            /* backward */
            for (int32_t i = 0; i < n_idx; ++i) {
                if (list[i] < 0) continue;
                int64_t r = ((int64_t)list[i] * hkv + g) * d;
                double dp = 0.0;
                for (int32_t e = 0; e < d; ++e) dp = dp + gv[e] * V[r + e];
                double ds = p[i] * (dp - D);
                for (int32_t e = 0; e < d; ++e) {
                    dV[r + e] = dV[r + e] + p[i] * gv[e];
                    dq[e] = dq[e] + ds * K[r + e];
                    dK[r + e] = dK[r + e] + (sc * ds) * qv[e];
                }
            }
            for (int32_t e = 0; e < d; ++e) dq[e] = sc * dq[e];
        }
    }
    free(p); free(o);
    return 0;
}
