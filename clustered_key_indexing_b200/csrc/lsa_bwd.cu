// lsa_bwd.cu -- gradient of the exact sparse attention over saved index
// lists [tutorial "隐空间稀疏注意力 (LSA)" (diosapp.com.cn), section 二: the
// attention itself; essay "《卡片柜》" (zhichai.net), ch. 6: the natively
// trained variant runs forward and backward per layer, and its backward keeps
// every query's selected key indices].  The selection is discrete and carries
// no gradient.
//
// One warp per (query, kv-head), as in the forward gather: the 16 keys of a
// tile are the MMA's M dimension, the G <= 8 query heads of the group its N.
// Pass 1 runs over the list's K tiles for the softmax statistics (the
// log-sum-exp of every head); pass 2 gathers the K and V tiles again and per
// tile forms
//   S^T = K Q^T,  P^T = exp(S^T / sqrt(d) - lse),  dP^T = V dO^T,
//   dS^T = P^T (dP^T - D),  dQ^T += K^T dS^T,
//   dV[keys] += P dO,  dK[keys] += dS Q / sqrt(d),
// with D = dO . O per head from the forward's output O.  P and dS enter the
// MMAs rounded to bf16; every accumulation is fp32.  The dV and dK tile
// products take P and dS straight from the accumulator layout of S^T as A
// operands (heads padded to K = 16) and are added to global memory with
// vector reductions, since several queries select the same key.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"

namespace lsa {

constexpr int kBwdWarps = 4;
constexpr int kBwdTileBytes = 16 * kD * 2;          // one 16-key tile of K or V
constexpr int kBwdWarpBytes = 4 * kBwdTileBytes;    // K and V, two slots each

struct BwdArgs {
    const uint16_t* Q;    // [nq, hq, 128]
    const uint16_t* K;    // [T, hkv, 128]
    const uint16_t* V;
    const uint16_t* O;    // forward output [nq, hq, 128]
    const uint16_t* dO;   // [nq, hq, 128]
    const int32_t* idx;   // [nq, hkv, n_idx]
    int64_t nq, T;
    int32_t hq, hkv, n_idx;
    float* dQ;            // [nq, hq, 128], written
    float* dK;            // [T, hkv, 128], added to
    float* dV;
    float scale_log2, scale;
};

__device__ __forceinline__ uint32_t bswz(int row, int chunk) {
    return (uint32_t)(row * (kD * 2) + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float bf2f(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

__device__ __forceinline__ void red_add_v2(float* p, float x, float y) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};\n" ::"l"(p), "f"(x), "f"(y) : "memory");
}

// C fragment of a 16 x 8 tile (rows = keys, columns = heads) to the B
// fragment of the same matrix as K x N (keys x heads), rounded to bf16.
__device__ __forceinline__ void c_to_b(const float (&c)[4], int lane, int G, uint32_t& b0, uint32_t& b1) {
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t lo = pack_bf16x2(c[0], c[1]), hi = pack_bf16x2(c[2], c[3]);
    const int src1 = (2 * tq) * 4 + (gq >> 1), src2 = (2 * tq + 1) * 4 + (gq >> 1);
    const uint32_t x1 = __shfl_sync(0xffffffffu, lo, src1);
    const uint32_t x2 = __shfl_sync(0xffffffffu, lo, src2);
    const uint32_t y1 = __shfl_sync(0xffffffffu, hi, src1);
    const uint32_t y2 = __shfl_sync(0xffffffffu, hi, src2);
    const uint32_t sel = (gq & 1) ? 0x7632u : 0x5410u;
    b0 = __byte_perm(x1, x2, sel);
    b1 = __byte_perm(y1, y2, sel);
    if (gq >= G) { b0 = 0u; b1 = 0u; }
}

__global__ void __launch_bounds__(32 * kBwdWarps) attn_bwd_kernel(BwdArgs a) {
    extern __shared__ __align__(128) uint8_t bsmem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t wg = (int64_t)blockIdx.x * kBwdWarps + wid;
    if (wg >= a.nq * a.hkv) return;
    const int64_t g = wg / a.nq, q = wg % a.nq;  // kv-head major, as the forward
    const int G = a.hq / a.hkv;
    const int32_t* list = a.idx + (q * a.hkv + g) * (int64_t)a.n_idx;
    const uint32_t wbase = smem_u32(bsmem + wid * kBwdWarpBytes);
    const int gq = lane >> 2, tq = lane & 3;
    const int64_t hrow0 = q * a.hq + g * G;  // the group's first query-head row
    const int h0 = 2 * tq, h1 = 2 * tq + 1;  // the heads of this lane's accumulator columns

    // Q^T and dO^T as B fragments of S^T and dP^T (k = dim, n = head gq)
    uint32_t qb[8][2], db[8][2];
    {
        const bool hv = gq < G;
        const uint16_t* qrow = a.Q + (hrow0 + (hv ? gq : 0)) * kD;
        const uint16_t* drow = a.dO + (hrow0 + (hv ? gq : 0)) * kD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qb[kk][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * tq) : 0u;
            qb[kk][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * tq + 8) : 0u;
            db[kk][0] = hv ? *reinterpret_cast<const uint32_t*>(drow + kk * 16 + 2 * tq) : 0u;
            db[kk][1] = hv ? *reinterpret_cast<const uint32_t*>(drow + kk * 16 + 2 * tq + 8) : 0u;
        }
    }
    // Q and dO as B fragments of the tile products (k = heads h0, h1; n = dim)
    uint32_t qn[16], dn[16];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        const int dim = nt * 8 + gq;
        const uint32_t q0 = h0 < G ? a.Q[(hrow0 + h0) * kD + dim] : 0u, q1 = h1 < G ? a.Q[(hrow0 + h1) * kD + dim] : 0u;
        const uint32_t d0 = h0 < G ? a.dO[(hrow0 + h0) * kD + dim] : 0u, d1 = h1 < G ? a.dO[(hrow0 + h1) * kD + dim] : 0u;
        qn[nt] = q0 | (q1 << 16);
        dn[nt] = d0 | (d1 << 16);
    }
    // D = dO . O of heads h0 and h1
    float D0 = 0.f, D1 = 0.f;
    for (int hh = 0; hh < G; ++hh) {
        const uint16_t* orow = a.O + (hrow0 + hh) * kD + lane * 4;
        const uint16_t* drow = a.dO + (hrow0 + hh) * kD + lane * 4;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) part = fmaf(bf2f(orow[e]), bf2f(drow[e]), part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (hh == h0) D0 = part;
        if (hh == h1) D1 = part;
    }

    const int ntiles = (a.n_idx + 15) / 16;
    const int64_t kv_stride = (int64_t)a.hkv * kD;
    const uint16_t* Kg = a.K + g * kD;
    const uint16_t* Vg = a.V + g * kD;
    // positions of one 16-key tile: lanes l and l + 16 both hold entry l
    auto tile_pos = [&](int tile) -> int {
        const int e = tile * 16 + (lane & 15);
        int p = (tile < ntiles && e < a.n_idx) ? __ldg(list + e) : -1;
        if (p >= a.T) {
            raise_device_error(kErrIndexRange);
            p = -1;
        }
        return p < 0 ? -1 : p;
    };
    // one 16-key tile (rows of absent entries are zero-filled), as one cp.async group
    auto issue = [&](int tile, uint32_t dst, const uint16_t* src, int p) {
        if (tile < ntiles) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = 2 * m + (lane >> 4), part = lane & 15;
                const int pr = __shfl_sync(0xffffffffu, p, r);
                const int64_t off = (pr >= 0 ? (int64_t)pr : 0) * kv_stride + part * 8;
                cp_async_16(dst + bswz(r, part), src + off, pr >= 0 ? 16 : 0);
            }
        }
        cp_async_commit();
    };
    // S^T (16 keys x 8 heads) of the K tile at `kb`, in the log2 domain;
    // absent keys -inf
    auto scores = [&](uint32_t kb, unsigned vmask, float (&s)[4]) {
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t af[4];
            ldsm_x4(af, kb + bswz(((lane >> 3) & 1) * 8 + (lane & 7), 2 * kk + (lane >> 4)));
            if (kk & 1) mma_16816(sb, af, qb[kk][0], qb[kk][1]);
            else mma_16816(sa, af, qb[kk][0], qb[kk][1]);
        }
        const bool v0 = (vmask >> gq) & 1u, v1 = (vmask >> (gq + 8)) & 1u;
        s[0] = v0 ? (sa[0] + sb[0]) * a.scale_log2 : -CUDART_INF_F;
        s[1] = v0 ? (sa[1] + sb[1]) * a.scale_log2 : -CUDART_INF_F;
        s[2] = v1 ? (sa[2] + sb[2]) * a.scale_log2 : -CUDART_INF_F;
        s[3] = v1 ? (sa[3] + sb[3]) * a.scale_log2 : -CUDART_INF_F;
    };

    // ---- pass 1: log-sum-exp of heads h0, h1 (K tiles only, two slots)
    float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};
    {
        int pa = tile_pos(0), pb = tile_pos(1);
        issue(0, wbase, Kg, pa);
        issue(1, wbase + kBwdTileBytes, Kg, pb);
        for (int i = 0; i < ntiles; ++i) {
            const int pn = tile_pos(i + 2);
            const unsigned vmask = __ballot_sync(0xffffffffu, pa >= 0) & 0xFFFFu;
            cp_async_wait<1>();
            __syncwarp();
            if (vmask != 0) {
                float s[4];
                scores(wbase + (i & 1) * kBwdTileBytes, vmask, s);
                float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
                l_run[0] = l_run[0] * exp2f(m_run[0] - mn0) + exp2f(s[0] - mn0) + exp2f(s[2] - mn0);
                l_run[1] = l_run[1] * exp2f(m_run[1] - mn1) + exp2f(s[1] - mn1) + exp2f(s[3] - mn1);
                m_run[0] = mn0;
                m_run[1] = mn1;
            }
            __syncwarp();
            issue(i + 2, wbase + (i & 1) * kBwdTileBytes, Kg, pn);
            pa = pb;
            pb = pn;
        }
        cp_async_wait<0>();
        __syncwarp();
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
    }
    // an empty list leaves lse = +inf: every p below is 0 and no gradient flows
    const float lse0 = l_run[0] > 0.f && h0 < G ? m_run[0] + log2f(l_run[0]) : CUDART_INF_F;
    const float lse1 = l_run[1] > 0.f && h1 < G ? m_run[1] + log2f(l_run[1]) : CUDART_INF_F;

    // ---- pass 2: K tile i in slot i % 2, V tile i in slot 2 + i % 2
    float dq[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) dq[mt][i] = 0.f;
    {
        auto kslot = [&](int t) { return wbase + (uint32_t)((t & 1) * kBwdTileBytes); };
        auto vslot = [&](int t) { return wbase + (uint32_t)((2 + (t & 1)) * kBwdTileBytes); };
        int pa = tile_pos(0), pb = tile_pos(1);
        issue(0, kslot(0), Kg, pa);
        issue(0, vslot(0), Vg, pa);
        issue(1, kslot(1), Kg, pb);
        issue(1, vslot(1), Vg, pb);
        for (int i = 0; i < ntiles; ++i) {
            const int pn = tile_pos(i + 2);
            const unsigned vmask = __ballot_sync(0xffffffffu, pa >= 0) & 0xFFFFu;
            cp_async_wait<2>();  // K(i) and V(i) have landed
            __syncwarp();
            if (vmask != 0) {
                float s[4];
                scores(kslot(i), vmask, s);
                float p[4];
                p[0] = exp2f(s[0] - lse0);
                p[1] = exp2f(s[1] - lse1);
                p[2] = exp2f(s[2] - lse0);
                p[3] = exp2f(s[3] - lse1);
                // dP^T = V dO^T
                float pa_[4] = {0.f, 0.f, 0.f, 0.f}, pb_[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t af[4];
                    ldsm_x4(af, vslot(i) + bswz(((lane >> 3) & 1) * 8 + (lane & 7), 2 * kk + (lane >> 4)));
                    if (kk & 1) mma_16816(pb_, af, db[kk][0], db[kk][1]);
                    else mma_16816(pa_, af, db[kk][0], db[kk][1]);
                }
                float ds[4];
                ds[0] = p[0] * (pa_[0] + pb_[0] - D0);
                ds[1] = p[1] * (pa_[1] + pb_[1] - D1);
                ds[2] = p[2] * (pa_[2] + pb_[2] - D0);
                ds[3] = p[3] * (pa_[3] + pb_[3] - D1);
                // dQ^T += K^T dS^T
                uint32_t b0, b1;
                c_to_b(ds, lane, G, b0, b1);
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    uint32_t af[4];
                    ldsm_x4_t(af, kslot(i) + bswz((lane >> 4) * 8 + (lane & 7), 2 * mt + ((lane >> 3) & 1)));
                    mma_16816(dq[mt], af, b0, b1);
                }
                // dV[keys] += P dO and dK[keys] += dS Q / sqrt(d): A = P, dS in
                // the S^T accumulator layout (rows = keys, k = heads, 8..15 zero)
                const int pos0 = __shfl_sync(0xffffffffu, pa, gq), pos1 = __shfl_sync(0xffffffffu, pa, gq + 8);
                float* dv0 = a.dV + ((int64_t)(pos0 < 0 ? 0 : pos0) * a.hkv + g) * kD + 2 * tq;
                float* dv1 = a.dV + ((int64_t)(pos1 < 0 ? 0 : pos1) * a.hkv + g) * kD + 2 * tq;
                float* dk0 = a.dK + ((int64_t)(pos0 < 0 ? 0 : pos0) * a.hkv + g) * kD + 2 * tq;
                float* dk1 = a.dK + ((int64_t)(pos1 < 0 ? 0 : pos1) * a.hkv + g) * kD + 2 * tq;
                const uint32_t ap[4] = {pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), 0u, 0u};
                const uint32_t as[4] = {pack_bf16x2(ds[0] * a.scale, ds[1] * a.scale),
                                        pack_bf16x2(ds[2] * a.scale, ds[3] * a.scale), 0u, 0u};
#pragma unroll
                for (int nt = 0; nt < 16; ++nt) {
                    float cv[4] = {0.f, 0.f, 0.f, 0.f}, ck[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_16816(cv, ap, dn[nt], 0u);
                    mma_16816(ck, as, qn[nt], 0u);
                    if (pos0 >= 0) {
                        red_add_v2(dv0 + nt * 8, cv[0], cv[1]);
                        red_add_v2(dk0 + nt * 8, ck[0], ck[1]);
                    }
                    if (pos1 >= 0) {
                        red_add_v2(dv1 + nt * 8, cv[2], cv[3]);
                        red_add_v2(dk1 + nt * 8, ck[2], ck[3]);
                    }
                }
            }
            __syncwarp();
            issue(i + 2, kslot(i), Kg, pn);
            issue(i + 2, vslot(i), Vg, pn);
            pa = pb;
            pb = pn;
        }
        cp_async_wait<0>();
        __syncwarp();
    }
    // dQ = (dQ^T)^T / sqrt(d): dq[mt] holds dims mt * 16 + gq (+ 8) of heads h0, h1
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        const int d0 = mt * 16 + gq;
        if (h0 < G) {
            a.dQ[(hrow0 + h0) * kD + d0] = dq[mt][0] * a.scale;
            a.dQ[(hrow0 + h0) * kD + d0 + 8] = dq[mt][2] * a.scale;
        }
        if (h1 < G) {
            a.dQ[(hrow0 + h1) * kD + d0] = dq[mt][1] * a.scale;
            a.dQ[(hrow0 + h1) * kD + d0 + 8] = dq[mt][3] * a.scale;
        }
    }
}

}  // namespace lsa

extern "C" {

lsa_status lsa_attn_backward(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* O,
                             const uint16_t* dO, const int32_t* idx, int64_t nq, int32_t hq, int32_t hkv,
                             int32_t n_idx, int64_t T, float* dQ, float* dK, float* dV, void* stream) {
    using namespace lsa;
    lsa_status s;
    if ((s = check_heads(hq, hkv)) != LSA_OK) return s;
    if (!Q || !K || !V || !O || !dO || !idx || !dQ || !dK || !dV)
        return set_error(LSA_EINVAL, "lsa_attn_backward: NULL pointer");
    if (nq < 0 || n_idx < 0 || T < 0) return set_error(LSA_EINVAL, "lsa_attn_backward: negative size");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO))
        return set_error(LSA_EINVAL, "lsa_attn_backward: Q, K, V, O, dO must be 16-byte aligned");
    if ((((uintptr_t)dQ | (uintptr_t)dK | (uintptr_t)dV) & 7u) != 0)
        return set_error(LSA_EINVAL, "lsa_attn_backward: dQ, dK, dV must be 8-byte aligned");
    if (T > (int64_t)INT32_MAX) return set_error(LSA_EUNSUPPORTED, "lsa_attn_backward: T beyond 2^31");
    if (nq == 0) return LSA_OK;
    BwdArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.O = O; a.dO = dO; a.idx = idx;
    a.nq = nq; a.T = T; a.hq = hq; a.hkv = hkv; a.n_idx = n_idx;
    a.dQ = dQ; a.dK = dK; a.dV = dV;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    a.scale = 1.0f / sqrtf((float)kD);
    const cudaStream_t st = (cudaStream_t)stream;
    const size_t smem = (size_t)kBwdWarps * kBwdWarpBytes;
    cudaFuncSetAttribute(attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    {
        KTime kt_("attn_bwd_kernel", st);
        attn_bwd_kernel<<<(unsigned)ceil_div<int64_t>(nq * hkv, kBwdWarps), 32 * kBwdWarps, smem, st>>>(a);
    }
    return check_launch("attn_bwd_kernel");
}

}  // extern "C"
