// lsa_noalloc.cu -- lsa_select_noalloc: the selection call for callers that
// cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: a host framework that owns
// every byte of device memory through its own pre-allocated pool, or a
// latency-critical path where an allocation (with its possible implicit
// synchronisation and its possible failure) is not acceptable.  This entry
// point gives them lsa_select without a caller-provided workspace: the
// scratch lives in one fixed-size array in device global memory that the
// library reserves when its module is loaded (every GPU that loads the
// library holds it until the process exits).
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "lsa.h"
#include "lsa_common.cuh"

namespace lsa {

constexpr size_t kNoAllocScratchBytes = (size_t)64 << 20;  // 64 MiB

// The scratch array.  In host code its name is only a host-side stand-in,
// not a device address; the device address comes from
// cudaGetSymbolAddress (see noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

size_t select_ws_bytes(const lsa_cfg* cfg, int64_t nq, int32_t hq, int32_t hkv, int64_t NB);

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
static lsa_status noalloc_scratch(void** out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* ptrs[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(LSA_ECUDA, "lsa_select_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return set_error(LSA_EUNSUPPORTED, "lsa_select_noalloc: device %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return set_error(LSA_ECUDA, "lsa_select_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return LSA_OK;
}

}  // namespace lsa

using namespace lsa;

extern "C" size_t lsa_select_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" lsa_status lsa_select_noalloc(const uint16_t* Q, int64_t t0, int64_t nq, int32_t hq,
                                         const float* W_q, const lsa_cache* cache,
                                         const lsa_tree* tree, const lsa_cfg* cfg, int32_t* idx,
                                         void* stream) {
    // size checks before anything touches the device.  Part of the flat
    // search's scratch grows with the cache (about 1 KB per bucket slot and
    // kv-head group of 8 heads), not with nq: if even one query does not fit,
    // splitting the query range cannot help.
    const size_t need = lsa_select_workspace_bytes(cfg, nq, hq, cache);
    if (need == 0) {
        lsa_status s = lsa_cfg_check(cfg);
        if (s != LSA_OK) return s;
        return set_error(LSA_EINVAL, "lsa_select_noalloc: invalid cache or nq");
    }
    if (need > kNoAllocScratchBytes) {
        const size_t one = lsa_select_workspace_bytes(cfg, 1, hq, cache);
        if (one > kNoAllocScratchBytes)
            return set_error(LSA_ENOSPACE,
                             "lsa_select_noalloc: the cache is too large for the built-in scratch: flat search "
                             "over it needs %zu bytes even for one query, the scratch holds %zu (about 512K "
                             "tokens at 8 kv-heads is the largest flat-mode cache; tree mode has no such limit)",
                             one, kNoAllocScratchBytes);
        return set_error(LSA_ENOSPACE,
                         "lsa_select_noalloc: this call needs %zu scratch bytes; the built-in scratch holds "
                         "%zu (split the queries into smaller ranges)",
                         need, kNoAllocScratchBytes);
    }
    // the scratch address is the current device's: the stream must be one
    // of that device's streams
    int dev = 0, sdev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaStreamGetDevice((cudaStream_t)stream, &sdev) == cudaSuccess &&
        sdev != dev)
        return set_error(LSA_EINVAL, "lsa_select_noalloc: the stream belongs to device %d, the current device is %d",
                         sdev, dev);
    void* ws = nullptr;
    lsa_status s = noalloc_scratch(&ws);
    if (s != LSA_OK) return s;
    return lsa_select(Q, t0, nq, hq, W_q, cache, tree, cfg, idx, nullptr, ws, kNoAllocScratchBytes, stream);
}
