// noalloc.cu -- tkv_quantize_append_noalloc: the bulk append without any
// caller-provided scratch.
//
// A multi-token append needs, per batch row, the rank of every new token among
// the new tokens of its class (and the per-class totals).  The regular entry
// point keeps those in the scratch part of the caller's workspace.  Some callers
// cannot allocate device memory at all -- code that runs where cudaMalloc is
// forbidden or unavailable (inside a host callback, under an allocator that
// must not grow, in a process that only receives pre-registered buffers) -- and
// cannot size a workspace for the largest T they might append.  This variant
// keeps the ranks in a fixed, file-scope device array instead, so it needs
// nothing beyond the cache's state and the inputs.
//
// The array is kNoallocScratchInts int32 (2 MiB); every GPU that loads the
// library holds it until the process exits.  Host code must not use the array's
// name as a device address: the first call on each device looks the address up
// with cudaGetSymbolAddress (with that device current) and caches it, so that
// first call should be made before any stream capture begins.  The cached address
// is valid only for the device context that was current at that first call: a
// process that calls cudaDeviceReset (or otherwise tears the primary context down
// and creates it again) must not use this entry point afterwards.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "tkv.h"
#include "tkv_internal.cuh"

namespace {

constexpr long long kNoallocScratchInts = 1ll << 19;  // 2 MiB of int32
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocScratchInts];

std::mutex g_mu;
int32_t *g_addr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t scratch_address(int32_t **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = static_cast<int32_t *>(p);
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

// Defined in tkv_api.cu: the cache's device view and the error-string setter.
namespace tkv {
const Dev *cache_dev(const tkv_cache *c, int *max_append);
void note_append(tkv_cache *c, int64_t launches, int T);
tkv_status api_fail(tkv_status st, const std::string &msg);
}  // namespace tkv

extern "C" TKV_API tkv_status tkv_quantize_append_noalloc(tkv_cache *cache, const void *k,
                                                          const void *v, const uint8_t *cls,
                                                          const int32_t *pos, int32_t T,
                                                          void *stream) {
    if (!cache) return tkv::api_fail(TKV_ERR_INVALID, "cache is NULL");
    if (!k || !v || !cls || !pos) return tkv::api_fail(TKV_ERR_INVALID, "NULL input pointer");
    int max_append = 0;
    const tkv::Dev *d0 = tkv::cache_dev(cache, &max_append);
    if (T < 1 || T > max_append) return tkv::api_fail(TKV_ERR_INVALID, "T out of [1, max_append]");
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
         reinterpret_cast<uintptr_t>(pos)) & 15u)
        return tkv::api_fail(TKV_ERR_INVALID, "k, v and pos must be 16-byte aligned");
    const long long need = (long long)d0->B * T + 4ll * d0->B;
    if (T > 1 && need > kNoallocScratchInts)
        return tkv::api_fail(TKV_ERR_INVALID,
                             "B*(T+4) exceeds the 524288-entry scratch of the no-alloc append");
    tkv::Dev d = *d0;
    if (T > 1) {
        int32_t *base = nullptr;
        cudaError_t e = scratch_address(&base);
        if (e != cudaSuccess)
            return tkv::api_fail(TKV_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
        // ranks [B][T] then totals [B][4]; both are fully rewritten by every call
        d.rank = base;
        d.totals = base + (size_t)d.B * T;
        d.max_append = T;
    }
    int64_t launches = 0;
    cudaError_t e = tkv::launch_append(d, k, v, cls, pos, T, static_cast<cudaStream_t>(stream), &launches);
    tkv::note_append(cache, launches, T);
    if (e != cudaSuccess) return tkv::api_fail(TKV_ERR_CUDA, cudaGetErrorString(e));
    return TKV_OK;
}
