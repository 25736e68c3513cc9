// lsa_probe.cu -- the measured peak of the L2-to-SM read path, the bound of
// the gathered attention (its K/V rows are re-read from L2 by many queries).
// No counterpart on the pages: measurement only.
//
// l2_read_kernel streams a caller buffer small enough to stay resident in L2
// `passes` times with 16-byte loads that bypass L1 (ld.global.cg, the cache
// path the gather's row copies take), eight loads in flight per thread,
// folding the words into one value per thread so the loads are not removed.
// Every CTA walks the buffer from its own offset, so the requests of the SMs
// at one time are spread over the whole buffer (and over both L2 halves).
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"
#include "lsa_common.cuh"

namespace lsa {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 8;

__global__ void __launch_bounds__(kProbeThreads) l2_read_kernel(const uint4* __restrict__ buf, int64_t n16,
                                                                int32_t passes, uint32_t* __restrict__ sink) {
    const int64_t per_cta = (int64_t)kProbeThreads * kProbeUnroll;
    const int64_t nchunks = n16 / per_cta;  // whole chunks of the buffer
    uint32_t acc = 0u;
    for (int32_t p = 0; p < passes; ++p) {
        for (int64_t c = 0; c < nchunks; c += gridDim.x) {
            if (c + blockIdx.x >= nchunks) break;
            // chunk c + blockIdx.x of this pass, rotated by the pass number
            const int64_t chunk = (c + blockIdx.x + (int64_t)p * 37) % nchunks;
            const uint4* src = buf + chunk * per_cta + threadIdx.x;
            uint4 v[kProbeUnroll];
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u) v[u] = __ldcg(src + u * kProbeThreads);
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
        }
    }
    sink[(int64_t)blockIdx.x * kProbeThreads + threadIdx.x] = acc;
}

}  // namespace lsa

using namespace lsa;

extern "C" {

size_t lsa_l2_read_sink_bytes(int32_t ctas) { return ctas > 0 ? (size_t)ctas * kProbeThreads * 4 : 0; }

int64_t lsa_l2_read_bytes(size_t bytes, int32_t passes) {
    const int64_t per_cta = (int64_t)kProbeThreads * kProbeUnroll * 16;
    if (passes <= 0) return 0;
    return (int64_t)(bytes / (size_t)per_cta) * per_cta * passes;  // whole chunks, each read once a pass
}

lsa_status lsa_l2_read(const void* buf, size_t bytes, int32_t passes, int32_t ctas, uint32_t* sink, void* stream) {
    if (!buf || !sink) return set_error(LSA_EINVAL, "lsa_l2_read: NULL pointer");
    if (((uintptr_t)buf & 15u) != 0) return set_error(LSA_EINVAL, "lsa_l2_read: buffer must be 16-byte aligned");
    if (passes <= 0 || ctas <= 0 || ctas > 65535) return set_error(LSA_EINVAL, "lsa_l2_read: passes, ctas out of range");
    const int64_t per_cta = (int64_t)kProbeThreads * kProbeUnroll * 16;
    if ((int64_t)bytes < per_cta) return set_error(LSA_EINVAL, "lsa_l2_read: buffer under %lld bytes", (long long)per_cta);
    l2_read_kernel<<<(unsigned)ctas, kProbeThreads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4*>(buf), (int64_t)(bytes / 16), passes, sink);
    return check_launch("l2_read_kernel");
}

}  // extern "C"
