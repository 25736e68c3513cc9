// lsa_attn.cu -- exact softmax attention over gathered index lists
// [tutorial "隐空间稀疏注意力 (LSA)" (diosapp.com.cn), section 二: the attention
// formula is unchanged, only the set of keys read changes; project card
// "Prefrontal-AI/latent-sparse-attention", 项目介绍].
//
// One warp per (query, kv-head).  The G <= 8 query heads of the GQA group
// share the index list, so the warp computes S^T = K_sel Q^T with the keys as
// the MMA's M dimension (16 keys per tile) and the heads as N (8 columns),
// then O^T += V_sel^T P^T.  Keys are gathered 16 at a time with 16-byte
// cp.async copies into a per-warp 12 KB shared-memory ring: two K tiles and
// one V tile (16-byte chunks XOR-swizzled by row so ldmatrix reads are
// conflict-free), so that 16 warps fit on an SM; the next V tile is fetched
// while the next tile's scores are computed.  Index tiles with no valid
// entry are skipped.  Online softmax in fp32 (exp2 with the
// log2(e)/sqrt(d) scale folded in), P rounded to bf16 for the PV product.
// Warps are ordered kv-head-major so the warps resident at one time read one
// head's K/V, which keeps that head's rows in L2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"

namespace lsa {

constexpr int kAttnWarps = 8;  // 12 KB of ring each: two CTAs, 16 warps per SM
constexpr int kTileKeys = 16;
constexpr int kTileBytes = kTileKeys * kD * 2;           // 4 KB per tensor
constexpr int kWarpBytes = 3 * kTileBytes;               // per-warp ring: K twice, V once

struct AttnArgs {
    const uint16_t* Q;
    const uint16_t* K;
    const uint16_t* V;
    const int32_t* idx;
    int64_t nq;
    int32_t hq, hkv, n_idx;
    int32_t n_use;        // entries of each list to attend to (<= n_idx, the list stride)
    const float* Ow;      // optional [nq, hq, 128] partial output over other keys (normalised) ...
    const float* lse;     // ... and its log2-domain log-sum-exp, merged into the result
    int64_t T;            // index entries must be < T
    int64_t kv_q_stride;  // token rows of K/V per query row (decode: each request's capacity); 0 = shared
    const uint16_t* Ks;   // decode's shared prefix [shared_len, hkv, 128] (SPLIT > 1 only) ...
    const uint16_t* Vs;
    int64_t shared_len;   // ... positions below it are read there; 0 = none
    uint16_t* O;
    float scale_log2;
    int64_t pos0;         // index entries are positions pos0 .. pos0 + T - 1 (K/V row p - pos0)
    float* Opart;         // optional (SPLIT == 1, Ow == NULL): normalised fp32 O [nq, hq, 128] ...
    float* lse_out;       // ... and the base-2 log-sum-exp of the scaled scores [nq, hq], instead of O
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)(row * (kD * 2) + ((chunk ^ (row & 7)) << 4));
}

// SPLIT == 1: one warp per (query, kv-head), 4 warps per CTA (prefill).
// SPLIT > 1: SPLIT warps share one (query, kv-head) row, each taking a
// contiguous slice of its index tiles; partial softmax states are combined
// through shared memory (decode, where rows are few).
template <int SPLIT>
__global__ void __launch_bounds__(32 * (SPLIT == 1 ? kAttnWarps : SPLIT), SPLIT == 1 ? 2 : 1) attn_kernel(AttnArgs a) {
    extern __shared__ __align__(128) uint8_t asmem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t wg = SPLIT == 1 ? (int64_t)blockIdx.x * kAttnWarps + wid : (int64_t)blockIdx.x;
    if (wg >= a.nq * a.hkv) return;
    const int64_t g = wg / a.nq, q = wg % a.nq;  // kv-head major
    const int G = a.hq / a.hkv;
    const int32_t* list = a.idx + (q * a.hkv + g) * (int64_t)a.n_idx;
    uint8_t* wbuf = asmem + wid * kWarpBytes;
    const uint32_t wbase = smem_u32(wbuf);

    // Q^T as B fragments (k = dim, n = head)
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t qb[8][2];
    {
        const uint16_t* qrow = a.Q + ((q * a.hq) + g * G + (gq < G ? gq : 0)) * (int64_t)kD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qb[kk][0] = gq < G ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * tq) : 0u;
            qb[kk][1] = gq < G ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * tq + 8) : 0u;
        }
    }

    const int ntot = (a.n_use + kTileKeys - 1) / kTileKeys;
    const int tbeg = SPLIT == 1 ? 0 : (int)(((int64_t)ntot * wid) / SPLIT);
    const int ntiles = SPLIT == 1 ? ntot : (int)(((int64_t)ntot * (wid + 1)) / SPLIT);  // tile end
    const int64_t kv_stride = (int64_t)a.hkv * kD;
    const uint16_t* Kg = a.K + (q * a.kv_q_stride * a.hkv + g) * kD;
    const uint16_t* Vg = a.V + (q * a.kv_q_stride * a.hkv + g) * kD;
    const uint16_t* Ksg = SPLIT > 1 && a.shared_len > 0 ? a.Ks + (int64_t)g * kD : Kg;
    const uint16_t* Vsg = SPLIT > 1 && a.shared_len > 0 ? a.Vs + (int64_t)g * kD : Vg;

    // positions of one 16-key tile: lanes l and l+16 both hold entry l
    auto tile_pos = [&](int tile) -> int {
        const int e = tile * kTileKeys + (lane & 15);
        int p = (tile < ntiles && e < a.n_use) ? __ldg(list + e) : -1;
        if (p >= 0) {
            const int64_t pl = (int64_t)p - a.pos0;
            if (pl < 0 || pl >= a.T) {
                raise_device_error(kErrIndexRange);
                p = -1;
            } else {
                p = (int)pl;
            }
        }
        return p;
    };
    // one 16-key tile of K (into K slot `slot`) or of V (its one slot), as a
    // cp.async group of its own
    auto issue = [&](int tile, uint32_t dst, const uint16_t* src, const uint16_t* src_sh, int p) {
        if (tile < ntiles) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = 2 * m + (lane >> 4), part = lane & 15;
                const int pr = __shfl_sync(0xffffffffu, p, r);
                if constexpr (SPLIT == 1) {
                    const int64_t off = (pr >= 0 ? (int64_t)pr : 0) * kv_stride + part * 8;
                    cp_async_16(dst + swz(r, part), src + off, pr >= 0 ? 16 : 0);
                } else {  // decode: the shared prefix, then the request's own rows
                    const bool sh = pr >= 0 && pr < a.shared_len;
                    const int64_t row = pr < 0 ? 0 : (sh ? (int64_t)pr : (int64_t)pr - a.shared_len);
                    const int64_t off = row * kv_stride + part * 8;
                    cp_async_16(dst + swz(r, part), (sh ? src_sh : src) + off, pr >= 0 ? 16 : 0);
                }
            }
        }
        cp_async_commit();
    };
    const uint32_t vslot = wbase + 2 * kTileBytes;
    auto issue_k = [&](int tile, int p) { issue(tile, wbase + (tile & 1) * kTileBytes, Kg, Ksg, p); };
    auto issue_v = [&](int tile, int p) { issue(tile, vslot, Vg, Vsg, p); };

    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;
    float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F};
    float l_run[2] = {0.f, 0.f};

    // Tile i: K in slot i % 2, V in the one V slot.  Groups are committed in
    // the order K(i), V(i), K(i + 1): S and the softmax of tile i wait for
    // K(i) only, the PV product for V(i); then V(i + 1) and K(i + 2) go out.
    int pr0 = tile_pos(tbeg), pr1 = tile_pos(tbeg + 1);
    issue_k(tbeg, pr0);
    issue_v(tbeg, pr0);
    issue_k(tbeg + 1, pr1);

    for (int i = tbeg; i < ntiles; ++i) {
        const int pnext = tile_pos(i + 2);
        const unsigned vmask = __ballot_sync(0xffffffffu, pr0 >= 0) & 0xFFFFu;
        const uint32_t kb = wbase + (i & 1) * kTileBytes, vb = vslot;
        uint32_t b0 = 0u, b1 = 0u;
        cp_async_wait<2>();
        __syncwarp();
        if (vmask != 0) {
            // S^T (16 keys x 8 heads): two independent accumulation chains
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t af[4];
                const int row = ((lane >> 3) & 1) * 8 + (lane & 7);
                const int chunk = 2 * kk + (lane >> 4);
                ldsm_x4(af, kb + swz(row, chunk));
                if (kk & 1) mma_16816(sb, af, qb[kk][0], qb[kk][1]);
                else mma_16816(sa, af, qb[kk][0], qb[kk][1]);
            }
            float s[4] = {sa[0] + sb[0], sa[1] + sb[1], sa[2] + sb[2], sa[3] + sb[3]};
            const bool v0 = (vmask >> gq) & 1u, v1 = (vmask >> (gq + 8)) & 1u;
            s[0] = v0 ? s[0] * a.scale_log2 : -CUDART_INF_F;
            s[1] = v0 ? s[1] * a.scale_log2 : -CUDART_INF_F;
            s[2] = v1 ? s[2] * a.scale_log2 : -CUDART_INF_F;
            s[3] = v1 ? s[3] * a.scale_log2 : -CUDART_INF_F;
            float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
            const bool grew = __any_sync(0xffffffffu, mn0 != m_run[0] || mn1 != m_run[1]);
            if (grew) {
                const float al0 = exp2f(m_run[0] - mn0), al1 = exp2f(m_run[1] - mn1);
                l_run[0] *= al0;
                l_run[1] *= al1;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[mt][0] *= al0; o[mt][1] *= al1; o[mt][2] *= al0; o[mt][3] *= al1;
                }
                m_run[0] = mn0;
                m_run[1] = mn1;
            }
            const float e0 = exp2f(s[0] - mn0), e1 = exp2f(s[1] - mn1);
            const float e2 = exp2f(s[2] - mn0), e3 = exp2f(s[3] - mn1);
            l_run[0] += e0 + e2;
            l_run[1] += e1 + e3;
            // P^T as B fragments: lane (head gq, tq) needs keys 2tq, 2tq+1, 2tq+8, 2tq+9
            const uint32_t pk_lo = pack_bf16x2(e0, e1), pk_hi = pack_bf16x2(e2, e3);
            const int src1 = (2 * tq) * 4 + (gq >> 1), src2 = (2 * tq + 1) * 4 + (gq >> 1);
            const uint32_t x1 = __shfl_sync(0xffffffffu, pk_lo, src1);
            const uint32_t x2 = __shfl_sync(0xffffffffu, pk_lo, src2);
            const uint32_t y1 = __shfl_sync(0xffffffffu, pk_hi, src1);
            const uint32_t y2 = __shfl_sync(0xffffffffu, pk_hi, src2);
            const uint32_t sel = (gq & 1) ? 0x7632u : 0x5410u;
            b0 = __byte_perm(x1, x2, sel);
            b1 = __byte_perm(y1, y2, sel);
            if (gq >= G) { b0 = 0u; b1 = 0u; }
        }
        cp_async_wait<1>();
        __syncwarp();
        if (vmask != 0) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t af[4];
                const int row = (lane >> 4) * 8 + (lane & 7);
                const int chunk = 2 * mt + ((lane >> 3) & 1);
                ldsm_x4_t(af, vb + swz(row, chunk));
                mma_16816(o[mt], af, b0, b1);
            }
        }
        __syncwarp();
        issue_v(i + 1, pr1);
        issue_k(i + 2, pnext);
        pr0 = pr1;
        pr1 = pnext;
    }
    cp_async_wait<0>();
    __syncwarp();

#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
    }
    if (SPLIT == 1 && a.Ow != nullptr) {
        // merge with the partial (O_w, lse) of the other keys: stage the
        // unnormalised O [8 heads][128] fp32 and (m, l) per head, then each
        // lane combines (head, dim) elements with coalesced reads and writes
        float* op = reinterpret_cast<float*>(wbuf);
        float* ml = op + 8 * kD;  // [8][2]
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d0 = mt * 16 + gq;
            op[(2 * tq) * kD + d0] = o[mt][0];
            op[(2 * tq + 1) * kD + d0] = o[mt][1];
            op[(2 * tq) * kD + d0 + 8] = o[mt][2];
            op[(2 * tq + 1) * kD + d0 + 8] = o[mt][3];
        }
        if (gq == 0) {
            ml[4 * tq] = m_run[0]; ml[4 * tq + 1] = l_run[0];
            ml[4 * tq + 2] = m_run[1]; ml[4 * tq + 3] = l_run[1];
        }
        __syncwarp();
        const int64_t r0 = q * a.hq + g * G;
        for (int e = lane; e < G * kD; e += 32) {
            const int hh = e / kD, d = e % kD;
            const float mb = ml[2 * hh], lb = ml[2 * hh + 1];
            const float la = a.lse[r0 + hh];
            const float M = fmaxf(mb, la);
            float out = 0.f;
            if (M > -CUDART_INF_F) {
                const float wb = exp2f(mb - M), wa = exp2f(la - M);
                out = (op[hh * kD + d] * wb + a.Ow[(r0 + hh) * kD + d] * wa) / (lb * wb + wa);
            }
            const __nv_bfloat16 ob = __float2bfloat16_rn(out);
            a.O[(r0 + hh) * kD + d] = *reinterpret_cast<const uint16_t*>(&ob);
        }
    } else if (SPLIT == 1 && a.Opart != nullptr) {
        // partial attention of a shard: normalised fp32 O and the base-2
        // log-sum-exp of each head (-inf, with O = 0, for an empty list)
        const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
        const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
        float* op = reinterpret_cast<float*>(wbuf);  // [8][128]
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d0 = mt * 16 + gq;
            op[(2 * tq) * kD + d0] = o[mt][0] * inv0;
            op[(2 * tq + 1) * kD + d0] = o[mt][1] * inv1;
            op[(2 * tq) * kD + d0 + 8] = o[mt][2] * inv0;
            op[(2 * tq + 1) * kD + d0 + 8] = o[mt][3] * inv1;
        }
        const int64_t r0 = q * a.hq + g * G;
        if (gq == 0) {
            if (2 * tq < G)
                a.lse_out[r0 + 2 * tq] = l_run[0] > 0.f ? m_run[0] + log2f(l_run[0]) : -CUDART_INF_F;
            if (2 * tq + 1 < G)
                a.lse_out[r0 + 2 * tq + 1] = l_run[1] > 0.f ? m_run[1] + log2f(l_run[1]) : -CUDART_INF_F;
        }
        __syncwarp();
        float* orow = a.Opart + r0 * (int64_t)kD;
        for (int c = lane; c < G * kD / 4; c += 32)
            reinterpret_cast<float4*>(orow)[c] = reinterpret_cast<const float4*>(op)[c];
    } else if constexpr (SPLIT == 1) {
        // normalise and stage O (heads x dims, bf16) for a coalesced store
        const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
        const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
        uint16_t* os = reinterpret_cast<uint16_t*>(wbuf);  // [8][128]
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d0 = mt * 16 + gq;
            const uint32_t lo = pack_bf16x2(o[mt][0] * inv0, o[mt][1] * inv1);
            const uint32_t hi = pack_bf16x2(o[mt][2] * inv0, o[mt][3] * inv1);
            os[(2 * tq) * kD + d0] = (uint16_t)(lo & 0xFFFF);
            os[(2 * tq + 1) * kD + d0] = (uint16_t)(lo >> 16);
            os[(2 * tq) * kD + d0 + 8] = (uint16_t)(hi & 0xFFFF);
            os[(2 * tq + 1) * kD + d0 + 8] = (uint16_t)(hi >> 16);
        }
        __syncwarp();
        uint16_t* orow = a.O + (q * a.hq + g * G) * (int64_t)kD;
        const int nchunk = G * kD / 8;  // 16-byte chunks
        for (int c = lane; c < nchunk; c += 32)
            reinterpret_cast<uint4*>(orow)[c] = reinterpret_cast<const uint4*>(os)[c];
    } else {
        // partial states: unnormalised O [8 heads][128] fp32 per warp + (m, l)
        __shared__ float ml[SPLIT][8][2];
        float* op = reinterpret_cast<float*>(wbuf);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d0 = mt * 16 + gq;
            op[(2 * tq) * kD + d0] = o[mt][0];
            op[(2 * tq + 1) * kD + d0] = o[mt][1];
            op[(2 * tq) * kD + d0 + 8] = o[mt][2];
            op[(2 * tq + 1) * kD + d0 + 8] = o[mt][3];
        }
        if (gq == 0) {
            ml[wid][2 * tq][0] = m_run[0]; ml[wid][2 * tq][1] = l_run[0];
            ml[wid][2 * tq + 1][0] = m_run[1]; ml[wid][2 * tq + 1][1] = l_run[1];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < G * kD; e += 32 * SPLIT) {
            const int hh = e / kD, d = e % kD;
            float mx = -CUDART_INF_F;
            for (int w = 0; w < SPLIT; ++w) mx = fmaxf(mx, ml[w][hh][0]);
            float l = 0.f, acc = 0.f;
            if (mx > -CUDART_INF_F) {
                for (int w = 0; w < SPLIT; ++w) {
                    const float mw = ml[w][hh][0];
                    if (!(mw > -CUDART_INF_F)) continue;
                    const float sc = exp2f(mw - mx);
                    l += ml[w][hh][1] * sc;
                    acc += reinterpret_cast<const float*>(asmem + w * kWarpBytes)[hh * kD + d] * sc;
                }
            }
            const float out = l > 0.f ? acc / l : 0.f;
            const __nv_bfloat16 ob = __float2bfloat16_rn(out);
            a.O[(q * a.hq + g * G + hh) * (int64_t)kD + d] = *reinterpret_cast<const uint16_t*>(&ob);
        }
    }
}

// Partial attention of one sequence shard: entries are positions p0 ..
// p0 + n_keys - 1 of K/V rows 0 .. n_keys - 1; writes the normalised fp32 O
// and base-2 log-sum-exp per (query, head).
lsa_status launch_attn_partial(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                               int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t p0, int64_t n_keys,
                               float* Opart, float* lse, cudaStream_t st) {
    if (nq <= 0) return LSA_OK;
    AttnArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.idx = idx; a.nq = nq; a.hq = hq; a.hkv = hkv; a.n_idx = n_idx;
    a.n_use = n_idx; a.T = n_keys; a.pos0 = p0; a.kv_q_stride = 0;
    a.Opart = Opart; a.lse_out = lse;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    const int64_t rows = nq * hkv;
    const size_t smem = (size_t)kAttnWarps * kWarpBytes;
    cudaFuncSetAttribute(attn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    {
        KTime kt_("attn_kernel", st);
        attn_kernel<1><<<(unsigned)ceil_div<int64_t>(rows, kAttnWarps), 32 * kAttnWarps, smem, st>>>(a);
    }
    return check_launch("attn_kernel(partial)");
}

// n_use < 0: every entry of each list; Ow / lse: optional partial state of
// other keys to merge (prefill: the sliding window, from the band kernel);
// Ks / Vs / shared_len: decode's shared prefix (positions below shared_len
// read Ks / Vs, the others row p - shared_len of the query row's own K / V).
lsa_status launch_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                       int64_t nq, int32_t hq, int32_t hkv, int32_t n_idx, int64_t T, uint16_t* O,
                       cudaStream_t st, int64_t kv_q_stride, int split, int32_t n_use, const float* Ow,
                       const float* lse, const uint16_t* Ks, const uint16_t* Vs, int64_t shared_len) {
    if (nq <= 0) return LSA_OK;
    AttnArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.idx = idx; a.nq = nq; a.hq = hq; a.hkv = hkv; a.n_idx = n_idx;
    a.n_use = n_use < 0 || n_use > n_idx ? n_idx : n_use;
    a.Ow = split == 1 ? Ow : nullptr;
    a.lse = split == 1 ? lse : nullptr;
    a.T = T; a.O = O; a.kv_q_stride = kv_q_stride;
    if (split == 1 && shared_len > 0) return set_error(LSA_EUNSUPPORTED, "attention: shared prefix is decode only");
    a.Ks = Ks; a.Vs = Vs; a.shared_len = shared_len;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    const int64_t rows = nq * hkv;
    if (split == 1) {
        const size_t smem = (size_t)kAttnWarps * kWarpBytes;
        cudaFuncSetAttribute(attn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        {
            KTime kt_("attn_kernel", st);
            attn_kernel<1><<<(unsigned)ceil_div<int64_t>(rows, kAttnWarps), 32 * kAttnWarps, smem, st>>>(a);
        }
        return check_launch("attn_kernel");
    }
    constexpr int kSplit = 8;
    const size_t smem = (size_t)kSplit * kWarpBytes;
    cudaFuncSetAttribute(attn_kernel<kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    {
        KTime kt_("attn_kernel_split", st);
        attn_kernel<kSplit><<<(unsigned)rows, 32 * kSplit, smem, st>>>(a);
    }
    return check_launch("attn_kernel(split)");
}

}  // namespace lsa
