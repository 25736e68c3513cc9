// lsa_pca.cu -- training-free projection of the distilled LSA variant: the
// leading d_latent principal directions of a layer's keys, used as W_k
// [tutorial "隐空间稀疏注意力 (LSA)" and the essay's closing remarks: PCA of
// the keys, the leading 64 directions taken as the projection, no training].
//
//   pca_moments_kernel  per CTA, over a contiguous slice of the key rows: the
//       raw second moments sum_t k_t k_t^T (fp64; every product of two bf16
//       values is exact, one rounding per add) and the sums sum_t k_t;
//   pca_reduce_kernel   the CTAs' partials in CTA order, then the centred
//       covariance C = (S2 - S1 S1^T / N) / N (exactly symmetric);
//   pca_jacobi_kernel   one CTA: cyclic Jacobi on C (fp64) with the
//       round-robin ordering, 64 disjoint rotations per step applied as a row
//       pass then a column pass, until the off-diagonal norm is below 1e-15
//       of the matrix norm; eigenvalues sorted descending (ties: lower
//       index), each direction's largest-magnitude component made positive;
//       W[e][r] = direction r, rounded to fp32.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"
#include "lsa_common.cuh"

namespace lsa {

constexpr int kPcaThreads = 256;
constexpr int kPcaRows = 32;       // key rows staged per step
constexpr int kPcaLd = kD + 1;     // padded row stride of the Jacobi matrix
constexpr int kPcaSweeps = 40;

// thread t owns entries (i, j) = (t / 16 + 16 r, t % 16 + 16 c), r, c < 8
__global__ void __launch_bounds__(kPcaThreads) pca_moments_kernel(const uint16_t* __restrict__ K, int64_t N,
                                                                 int64_t rows_per_blk, double* __restrict__ part2,
                                                                 double* __restrict__ part1) {
    __shared__ double xs[kPcaRows][kD];
    const int tid = threadIdx.x, bi = tid >> 4, bj = tid & 15;
    double acc[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.0;
    double s1 = 0.0;
    const int64_t r0 = (int64_t)blockIdx.x * rows_per_blk;
    const int64_t r1 = min(N, r0 + rows_per_blk);
    for (int64_t base = r0; base < r1; base += kPcaRows) {
        const int n = (int)(r1 - base < kPcaRows ? r1 - base : kPcaRows);
        for (int u = tid; u < kPcaRows * (kD / 8); u += kPcaThreads) {
            const int row = u / (kD / 8), part = u % (kD / 8);
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row < n) v = __ldg(reinterpret_cast<const uint4*>(K + (base + row) * kD) + part);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xs[row][part * 8 + 2 * i] = (double)__uint_as_float(w4[i] << 16);
                xs[row][part * 8 + 2 * i + 1] = (double)__uint_as_float(w4[i] & 0xFFFF0000u);
            }
        }
        __syncthreads();
        for (int row = 0; row < n; ++row) {
            double xi[8], xj[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) xi[r] = xs[row][bi + 16 * r];
#pragma unroll
            for (int c = 0; c < 8; ++c) xj[c] = xs[row][bj + 16 * c];
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = fma(xi[r], xj[c], acc[r][c]);
            if (tid < kD) s1 = __dadd_rn(s1, xs[row][tid]);
        }
        __syncthreads();
    }
    double* p2 = part2 + (int64_t)blockIdx.x * kD * kD;
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) p2[(bi + 16 * r) * kD + bj + 16 * c] = acc[r][c];
    if (tid < kD) part1[(int64_t)blockIdx.x * kD + tid] = s1;
}

// C[i][j] = (S2[i][j] - S1[i] S1[j] / N) / N, partials summed in CTA order.
__global__ void __launch_bounds__(128) pca_reduce_kernel(const double* __restrict__ part2,
                                                        const double* __restrict__ part1, int nblk, int64_t N,
                                                        double* __restrict__ C) {
    const int e = blockIdx.x * 128 + threadIdx.x;
    if (e >= kD * kD) return;
    const int i = e / kD, j = e % kD;
    double s2 = 0.0, si = 0.0, sj = 0.0;
    for (int b = 0; b < nblk; ++b) {
        s2 = __dadd_rn(s2, part2[(int64_t)b * kD * kD + e]);
        si = __dadd_rn(si, part1[(int64_t)b * kD + i]);
        sj = __dadd_rn(sj, part1[(int64_t)b * kD + j]);
    }
    const double n = (double)N;
    C[e] = __ddiv_rn(__dsub_rn(s2, __ddiv_rn(__dmul_rn(si, sj), n)), n);
}

// Block-wide sum over 1024 threads (result in every thread).
__device__ double pca_block_sum(double v, double* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == 0) red[wid] = v;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < 32; ++w) s = __dadd_rn(s, red[w]);
    __syncthreads();
    return s;
}

// One CTA of 1024 threads; A (the covariance) in shared memory, the
// eigenvectors V [d][d] in global memory (ws).
__global__ void __launch_bounds__(1024) pca_jacobi_kernel(const double* __restrict__ C, double* __restrict__ V,
                                                         int d_latent, float* __restrict__ W, double* __restrict__ eig) {
    extern __shared__ double A[];   // [kD][kPcaLd]
    __shared__ int P[kD / 2], Q[kD / 2];
    __shared__ double cs[kD / 2], sn[kD / 2], red[32], lam[kD];
    const int tid = threadIdx.x;
    for (int e = tid; e < kD * kD; e += 1024) {
        const int i = e / kD, j = e % kD;
        A[i * kPcaLd + j] = C[e];
        V[e] = i == j ? 1.0 : 0.0;
    }
    __syncthreads();
    for (int sweep = 0; sweep < kPcaSweeps; ++sweep) {
        double off = 0.0, all = 0.0;
        for (int e = tid; e < kD * kD; e += 1024) {
            const int i = e / kD, j = e % kD;
            const double a = A[i * kPcaLd + j];
            all = fma(a, a, all);
            if (i != j) off = fma(a, a, off);
        }
        off = pca_block_sum(off, red);
        all = pca_block_sum(all, red);
        if (off <= 1e-30 * all) break;
        for (int s = 0; s < kD - 1; ++s) {
            if (tid < kD / 2) {
                // round robin: position 0 fixed, positions 1..127 rotate by s
                auto pos = [&](int i) { return i == 0 ? 0 : 1 + ((i - 1 + s) % (kD - 1)); };
                const int p = pos(tid), q = pos(kD - 1 - tid);
                const double app = A[p * kPcaLd + p], aqq = A[q * kPcaLd + q], apq = A[p * kPcaLd + q];
                double c = 1.0, sv = 0.0;
                if (apq != 0.0) {
                    const double th = (aqq - app) / (2.0 * apq);
                    const double t = (th >= 0.0 ? 1.0 : -1.0) / (fabs(th) + sqrt(th * th + 1.0));
                    c = 1.0 / sqrt(t * t + 1.0);
                    sv = t * c;
                }
                P[tid] = p;
                Q[tid] = q;
                cs[tid] = c;
                sn[tid] = sv;
            }
            __syncthreads();
            // rows: A <- J^T A (rows p and q of every pair)
            for (int it = tid; it < (kD / 2) * kD; it += 1024) {
                const int k = it / kD, j = it % kD;
                const int p = P[k], q = Q[k];
                const double c = cs[k], sv = sn[k];
                const double ap = A[p * kPcaLd + j], aq = A[q * kPcaLd + j];
                A[p * kPcaLd + j] = c * ap - sv * aq;
                A[q * kPcaLd + j] = sv * ap + c * aq;
            }
            __syncthreads();
            // columns: A <- A J, V <- V J
            for (int it = tid; it < (kD / 2) * kD; it += 1024) {
                const int k = it / kD, i = it % kD;
                const int p = P[k], q = Q[k];
                const double c = cs[k], sv = sn[k];
                const double ap = A[i * kPcaLd + p], aq = A[i * kPcaLd + q];
                A[i * kPcaLd + p] = c * ap - sv * aq;
                A[i * kPcaLd + q] = sv * ap + c * aq;
                const double vp = V[i * kD + p], vq = V[i * kD + q];
                V[i * kD + p] = c * vp - sv * vq;
                V[i * kD + q] = sv * vp + c * vq;
            }
            __syncthreads();
        }
    }
    if (tid < kD) lam[tid] = A[tid * kPcaLd + tid];
    __syncthreads();
    if (tid < kD) {
        const double li = lam[tid];
        int rk = 0;
        for (int j = 0; j < kD; ++j) rk += (lam[j] > li) || (lam[j] == li && j < tid);
        if (eig) eig[rk] = li;
        // sign: the first largest-magnitude component positive
        int m = 0;
        double best = -1.0;
        for (int e = 0; e < kD; ++e) {
            const double a = fabs(V[e * kD + tid]);
            if (a > best) { best = a; m = e; }
        }
        const double sgn = V[m * kD + tid] < 0.0 ? -1.0 : 1.0;
        if (rk < d_latent)
            for (int e = 0; e < kD; ++e) W[e * d_latent + rk] = __double2float_rn(sgn * V[e * kD + tid]);
    }
}

static int pca_blocks() { return 2 * num_sms(); }

static size_t pca_ws_bytes() {
    const size_t nb = (size_t)pca_blocks();
    return nb * kD * kD * 8 + nb * kD * 8 + 2 * (size_t)kD * kD * 8 + 1024;
}

}  // namespace lsa

using namespace lsa;

extern "C" {

size_t lsa_fit_pca_workspace_bytes(int64_t T, int32_t hkv) {
    if (T <= 0 || hkv <= 0) return 0;
    return pca_ws_bytes();
}

lsa_status lsa_fit_pca(const uint16_t* K, int64_t T, int32_t hkv, int32_t d_latent, float* W_out, double* eig_out,
                       void* ws, size_t ws_bytes, void* stream) {
    if (!K || !W_out || !ws) return set_error(LSA_EINVAL, "lsa_fit_pca: K, W_out or ws is NULL");
    if (T <= 0 || hkv <= 0) return set_error(LSA_EINVAL, "lsa_fit_pca: need T > 0 and hkv > 0");
    if (d_latent < 1 || d_latent > kD) return set_error(LSA_EINVAL, "lsa_fit_pca: d_latent must be in 1..128");
    if (((uintptr_t)K & 15u) != 0) return set_error(LSA_EINVAL, "lsa_fit_pca: K must be 16-byte aligned");
    if (ws_bytes < pca_ws_bytes()) return set_error(LSA_ENOSPACE, "lsa_fit_pca: workspace too small");
    cudaStream_t st = (cudaStream_t)stream;
    const int nblk = pca_blocks();
    const int64_t N = T * hkv;
    char* base = (char*)(((uintptr_t)ws + 255) & ~(uintptr_t)255);
    double* part2 = (double*)base;
    double* part1 = part2 + (size_t)nblk * kD * kD;
    double* C = part1 + (size_t)nblk * kD;
    double* V = C + (size_t)kD * kD;
    lsa_status s;
    {
        KTime kt_("pca_moments_kernel", st);
        pca_moments_kernel<<<nblk, kPcaThreads, 0, st>>>(K, N, ceil_div<int64_t>(N, nblk), part2, part1);
    }
    if ((s = check_launch("pca_moments_kernel")) != LSA_OK) return s;
    pca_reduce_kernel<<<(kD * kD + 127) / 128, 128, 0, st>>>(part2, part1, nblk, N, C);
    if ((s = check_launch("pca_reduce_kernel")) != LSA_OK) return s;
    const size_t smem = (size_t)kD * kPcaLd * 8;
    cudaFuncSetAttribute(pca_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    {
        KTime kt_("pca_jacobi_kernel", st);
        pca_jacobi_kernel<<<1, 1024, smem, st>>>(C, V, d_latent, W_out, eig_out);
    }
    return check_launch("pca_jacobi_kernel");
}

}  // extern "C"
