// lsa_band.cu -- the sliding-window part of an LSA index row as banded dense
// attention [tutorial "隐空间稀疏注意力 (LSA)" (diosapp.com.cn), section 二:
// every query always attends to its sinks and its last W positions; the
// attention formula is unchanged].
//
// Query t's window is positions max(S, t - W + 1) .. t: consecutive queries
// share almost all of it.  A CTA takes 128 (query, head) rows of one kv-head
// (128 / G consecutive queries x the G heads of the group, 16 rows per warp)
// and streams the union of their windows through shared memory in 64-key
// tiles (K and V, 16-byte cp.async copies, 2-stage ring, XOR-swizzled
// chunks), so each tile is read once for all 128 rows instead of once per
// query.  The CTA's Q rows sit in shared memory too.  Per warp: S = Q K^T
// with mma.sync m16n8k16 (bf16 in, fp32
// accumulate; the accumulator layout is reused as the A operand of P V),
// online softmax in fp32 (exp2, log2(e)/sqrt(d) folded into the scale),
// per-row masks on the band edges only.  Output: the normalised window
// output O_w (fp32) and its log-sum-exp (log2 domain) per row, merged with
// the sinks and long-range part by the gather kernel's epilogue.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_mma.cuh"

namespace lsa {

constexpr int kBandRows = 128;                     // (query, head) rows per CTA
constexpr int kBandWarps = kBandRows / 16;
constexpr int kBandTile = 64;                      // keys per tile
constexpr int kBandTileBytes = kBandTile * kD * 2;  // 16 KB per tensor
constexpr int kBandStageBytes = 2 * kBandTileBytes;
constexpr int kBandQBytes = kBandRows * kD * 2;      // the CTA's Q rows, 32 KB
constexpr size_t kBandSmemBytes = 2 * (size_t)kBandStageBytes + kBandQBytes;

struct BandArgs {
    const uint16_t* Q;       // [nq, hq, 128]: query i of the call sits at position t0 + i
    const uint16_t* K;       // [T, hkv, 128]
    const uint16_t* V;
    int64_t nq, t0, T;
    int32_t hq, hkv, S, W;
    float* Ow;               // [nq, hq, 128] normalised window output
    float* lse;              // [nq, hq] log2-domain log-sum-exp of the scaled scores; -inf: empty window
    float scale_log2;
};

__device__ __forceinline__ uint32_t band_swz(int row, int chunk) {
    return (uint32_t)(row * (kD * 2) + ((chunk ^ (row & 7)) << 4));
}

template <int G>
__global__ void __launch_bounds__(32 * kBandWarps, 2) band_attn_kernel(BandArgs a) {
    extern __shared__ __align__(128) uint8_t bsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int QB = kBandRows / G;  // queries per CTA
    const int h = blockIdx.y;
    const int64_t qb0 = (int64_t)blockIdx.x * QB;
    if (qb0 >= a.nq) return;
    const int64_t qlast = min(a.nq - 1, qb0 + QB - 1);
    // positions fit in int32 (T < 2^31)
    const int t_first = (int)(a.t0 + qb0), t_last = (int)(a.t0 + qlast);
    // keys some row of the CTA attends to: [P0, t_last]
    const int P0 = max(a.S, t_first - a.W + 1);
    const int nkeys = t_last - P0 + 1;
    const int ntiles = nkeys > 0 ? (nkeys + kBandTile - 1) / kBandTile : 0;
    // a tile [p0, p0 + 63] is inside every row's window when p0 >= lo_max and p0 + 63 <= t_first
    const int lo_max = max(a.S, t_last - a.W + 1);

    // this lane's rows 16 warp + gq and + 8: row r is query r / G, head r % G
    const int gq = lane >> 2, tq = lane & 3;
    int lo_r[2], hi_r[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int r = 16 * warp + gq + 8 * hh;
        const int t = t_first + r / G;
        lo_r[hh] = max(a.S, t - a.W + 1);
        hi_r[hh] = t;
    }
    // the CTA's Q rows into shared memory (row r = query r / G, head r % G;
    // zero past the call's queries), read back per k-step with ldmatrix
    uint8_t* sQ = bsm + 2 * kBandStageBytes;
    for (int c = tid; c < kBandRows * 16; c += 32 * kBandWarps) {
        const int r = c >> 4, part = c & 15;
        const int64_t qq = qb0 + r / G;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (qq <= qlast)
            v = *reinterpret_cast<const uint4*>(a.Q + (qq * a.hq + (int64_t)h * G + r % G) * kD + part * 8);
        *reinterpret_cast<uint4*>(sQ + band_swz(r, part)) = v;
    }
    const uint32_t qbase = smem_u32(sQ);
    const int qrow = 16 * warp + (lane & 7) + (((lane >> 3) & 1) << 3);

    const uint32_t sbase = smem_u32(bsm);
    auto issue = [&](int tile, int stage) {
        if (tile < ntiles) {
            const int p0 = P0 + tile * kBandTile;
            const uint32_t kb = sbase + stage * kBandStageBytes, vb = kb + kBandTileBytes;
#pragma unroll
            for (int c = tid; c < kBandTile * 16; c += 32 * kBandWarps) {
                const int r = c >> 4, part = c & 15;
                const int p = p0 + r;
                const bool ok = p <= t_last;
                const int64_t off = ((int64_t)(ok ? p : 0) * a.hkv + h) * kD + part * 8;
                cp_async_16(kb + band_swz(r, part), a.K + off, ok ? 16 : 0);
                cp_async_16(vb + band_swz(r, part), a.V + off, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
    float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};

    issue(0, 0);
    __syncthreads();  // Q rows staged
    for (int i = 0; i < ntiles; ++i) {
        issue(i + 1, (i + 1) & 1);
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t kb = sbase + (i & 1) * kBandStageBytes, vb = kb + kBandTileBytes;
        const int p0 = P0 + i * kBandTile;
        const bool full = p0 >= lo_max && p0 + kBandTile - 1 <= t_first;
        // two halves of 32 keys, each its own online-softmax step (fewer live
        // registers than one 64-key step)
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const int kh = 32 * half;
            // S = Q K^T: 16 rows x 32 keys (n-tile nt: keys kh + 8 nt .. + 7)
            float s[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) s[nt][j] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t qa[4];
                ldsm_x4(qa, qbase + band_swz(qrow, 2 * kk + (lane >> 4)));
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t b[4];
                    const int key = kh + 16 * np + ((lane >> 4) << 3) + (lane & 7);
                    ldsm_x4(b, kb + band_swz(key, 2 * kk + ((lane >> 3) & 1)));
                    mma_16816(s[2 * np], qa, b[0], b[1]);
                    mma_16816(s[2 * np + 1], qa, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int hh = j >> 1;
                    const int p = p0 + kh + 8 * nt + 2 * tq + (j & 1);
                    const bool ok = full || (p >= lo_r[hh] && p <= hi_r[hh]);
                    s[nt][j] = ok ? s[nt][j] * a.scale_log2 : -CUDART_INF_F;
                }
            // online softmax per row (a row's scores sit in the 4 lanes of a quad)
            float alpha[2], m_use[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float mx = -CUDART_INF_F;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * hh], s[nt][2 * hh + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mn = fmaxf(m_run[hh], mx);
                m_use[hh] = mn == -CUDART_INF_F ? 0.f : mn;
                alpha[hh] = exp2f(m_run[hh] - m_use[hh]);
                m_run[hh] = mn;
            }
            uint32_t pa[2][4];
            float rs[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float e0 = exp2f(s[nt][0] - m_use[0]), e1 = exp2f(s[nt][1] - m_use[0]);
                const float e2 = exp2f(s[nt][2] - m_use[1]), e3 = exp2f(s[nt][3] - m_use[1]);
                rs[0] += e0 + e1;
                rs[1] += e2 + e3;
                pa[nt >> 1][(nt & 1) * 2] = pack_bf16x2(e0, e1);
                pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(e2, e3);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) l_run[hh] = l_run[hh] * alpha[hh] + rs[hh];
#pragma unroll
            for (int dt = 0; dt < 16; ++dt) {
                o[dt][0] *= alpha[0]; o[dt][1] *= alpha[0];
                o[dt][2] *= alpha[1]; o[dt][3] *= alpha[1];
            }
            // O += P V: 16 rows x 128 dims, k-step j = keys kh + 16 j .. + 15
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#pragma unroll
                for (int dp = 0; dp < 8; ++dp) {
                    uint32_t b[4];
                    const int key = kh + 16 * j + (((lane >> 3) & 1) << 3) + (lane & 7);
                    ldsm_x4_t(b, vb + band_swz(key, 2 * dp + (lane >> 4)));
                    mma_16816(o[2 * dp], pa[j], b[0], b[1]);
                    mma_16816(o[2 * dp + 1], pa[j], b[2], b[3]);
                }
            }
        }
        __syncthreads();  // stage (i & 1) is refilled by the next iteration's issue
    }
    cp_async_wait<0>();

#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int r = 16 * warp + gq + 8 * hh;
        const int64_t rq = qb0 + r / G;
        if (rq > qlast) continue;
        const int64_t rrow = rq * a.hq + (int64_t)h * G + r % G;
        const float inv = l_run[hh] > 0.f ? 1.f / l_run[hh] : 0.f;
        float* orow = a.Ow + rrow * kD;
#pragma unroll
        for (int dt = 0; dt < 16; ++dt)
            *reinterpret_cast<float2*>(orow + 8 * dt + 2 * tq) =
                make_float2(o[dt][2 * hh] * inv, o[dt][2 * hh + 1] * inv);
        if (tq == 0)
            a.lse[rrow] = l_run[hh] > 0.f ? m_run[hh] + log2f(l_run[hh]) : -CUDART_INF_F;
    }
}

lsa_status launch_band_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t nq, int64_t t0,
                            int64_t T, int32_t hq, int32_t hkv, int32_t S, int32_t W, float* Ow, float* lse,
                            cudaStream_t st) {
    if (nq <= 0) return LSA_OK;
    BandArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.nq = nq; a.t0 = t0; a.T = T; a.hq = hq; a.hkv = hkv; a.S = S; a.W = W;
    a.Ow = Ow; a.lse = lse;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    const int G = hq / hkv;
    auto kern = G == 1 ? band_attn_kernel<1> : G == 2 ? band_attn_kernel<2> : G == 4 ? band_attn_kernel<4>
                                                                                     : band_attn_kernel<8>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBandSmemBytes);
    {
        KTime kt_("band_attn_kernel", st);
        kern<<<dim3((unsigned)ceil_div<int64_t>(nq, kBandRows / G), (unsigned)hkv), 32 * kBandWarps, kBandSmemBytes,
               st>>>(a);
    }
    return check_launch("band_attn_kernel");
}

}  // namespace lsa
