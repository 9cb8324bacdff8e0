// selftest.cu -- tkv_selftest_wait_timeout: exercises the bounded-wait path the
// decode kernels use for their copy barriers, without any fault.  A one-warp
// kernel waits on an mbarrier that nothing ever arrives on; after `limit` SM
// cycles the wait gives up and the kernel latches TKV_ERR_TIMEOUT in the cache's
// device error word, exactly as a decode kernel does when a copy never lands.
#include "attn_common.cuh"

namespace tkv {
namespace {

__global__ void wait_timeout_kernel(uint32_t *err, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = attn::smem_addr(&bar);
    if (threadIdx.x == 0) {
        attn::mbar_init(b);   // expects one arrival, which never comes
        attn::mbar_init_fence();
    }
    __syncwarp();
    const bool ok = attn::mbar_wait_for(b, 0u, limit);
    if (!__all_sync(attn::kFull, ok) && threadIdx.x == 0) raise_error(err, kErrTimeout, 0xffffffffu);
}

}  // namespace

cudaError_t launch_wait_timeout(const Dev &d, long long limit, cudaStream_t st, int64_t *launches) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(d.err, limit);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tkv
