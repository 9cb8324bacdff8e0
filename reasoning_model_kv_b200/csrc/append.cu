// append.cu -- tkv_quantize_append: thought-adaptive group quantisation of new
// tokens (ThinKV, Metodologia / TBQ) into paged per-precision pools with
// in-place reuse of evicted slots (ThinKV, Implementacao do Sistema /
// Continuous Thinking).  The per-token work (for T == 1 two warps per (stream, token),
// one quantising the K row and the other the V row; for T > 1 one warp per (stream,
// token)) is in append_token.cuh.
//
// Slot allocation needs, per (stream, class), the rank of each new token among
// the new tokens of its class.  For T == 1 that rank is 0 and the packing warp
// also updates the stream's counters (one kernel).  For T > 1 a scan kernel per
// batch row computes the ranks (they are shared by all kv heads of the row), the
// pack kernel runs on every (stream, token) in parallel against the pre-call
// counters, and a finalize kernel advances the counters.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "append_token.cuh"

namespace tkv {
namespace {

using app::kFull;
using app::token_class;

__global__ void append_rank_kernel(Dev d, const uint8_t *__restrict__ cls,
                                   const int32_t *__restrict__ pos, int T) {
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    __shared__ int carry[4];
    __shared__ int wtot[32][4];
    if (threadIdx.x < 4) carry[threadIdx.x] = 0;
    __syncthreads();
    for (int t0 = 0; t0 < T; t0 += blockDim.x) {
        const int t = t0 + threadIdx.x;
        int c = -2;
        if (t < T) c = token_class(d, cls[(size_t)b * T + t], pos[(size_t)b * T + t]);
        int myrank = 0;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const unsigned m = __ballot_sync(kFull, c == cc);
            if (lane == 0) wtot[warp][cc] = __popc(m);
            if (c == cc) myrank = __popc(m & ((1u << lane) - 1u));
        }
        __syncthreads();
        if (c >= 0) {
            int pre = carry[c];
            for (int w = 0; w < warp; ++w) pre += wtot[w][c];
            d.rank[(size_t)b * d.max_append + t] = pre + myrank;
        } else if (t < T) {
            d.rank[(size_t)b * d.max_append + t] = -1;
        }
        __syncthreads();
        if (threadIdx.x < 4) {
            int sum = 0;
            for (int w = 0; w < nwarps; ++w) sum += wtot[w][threadIdx.x];
            carry[threadIdx.x] += sum;
        }
        __syncthreads();
    }
    if (threadIdx.x < 4) d.totals[b * 4 + threadIdx.x] = carry[threadIdx.x];
}

// kCodec: the class record formats (0 integer codes, 1 FP codes), a template argument so
// that each instantiation holds only its own quantiser (the T = 1 append overlaps the
// decode attention launched after it, and a leaner kernel leaves it more room).
template <bool kSingle, int kCodec>
__global__ void __launch_bounds__(256) append_pack_kernel(
    Dev d, const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
    const uint8_t *__restrict__ cls, const int32_t *__restrict__ pos, int T) {
    __shared__ __align__(16) uint8_t stage_all[8 * 2 * kD];   // per warp: a row by head dim
    // let the next kernel in the stream (decode attention) launch now; it waits for
    // this grid's completion before it reads the cache
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // T == 1: two warps per (stream, token), warps 2i (K) and 2i + 1 (V) of the grid;
    // T > 1: one warp per (stream, token)
    constexpr int kShift = kSingle ? 1 : 0;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if ((gw >> kShift) >= d.S * T) return;   // (both warps of a pair)
    app::append_token<kSingle, kCodec>(d, k, v, cls, pos, T, gw >> kShift, gw & 1, lane,
                                       stage_all + (threadIdx.x >> 5) * 2 * kD, 1 + ((threadIdx.x >> 5) >> 1));
}

__global__ void append_finalize_kernel(Dev d) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= d.S * 4) return;
    const int s = i >> 2, c = i & 3, b = s / d.Hkv;
    const int tot = d.totals[b * 4 + c];
    const int ft = d.ft[i], hw = d.hw[i];
    const int pops = tot < ft ? tot : ft;
    int fresh = tot - pops;
    if (fresh > d.cap[c] - hw) fresh = d.cap[c] - hw;
    d.ft[i] = ft - pops;
    d.hw[i] = hw + fresh;
    d.n[i] += pops + fresh;
}

}  // namespace

cudaError_t launch_append(const Dev &d, const void *k, const void *v, const uint8_t *cls,
                          const int32_t *pos, int T, cudaStream_t st, int64_t *launches) {
    const auto *kk = static_cast<const __nv_bfloat16 *>(k);
    const auto *vv = static_cast<const __nv_bfloat16 *>(v);
    // T == 1: a K warp and a V warp per (stream, token); T > 1: one warp per (stream, token)
    const long long warps = (T == 1 ? 2ll : 1ll) * d.S * T;
    const int threads = 256;
    const unsigned blocks = (unsigned)((warps * 32 + threads - 1) / threads);
    if (T == 1) {
        if (d.codec == 0) append_pack_kernel<true, 0><<<blocks, threads, 0, st>>>(d, kk, vv, cls, pos, T);
        else append_pack_kernel<true, 1><<<blocks, threads, 0, st>>>(d, kk, vv, cls, pos, T);
        *launches += 1;
        return cudaGetLastError();
    }
    append_rank_kernel<<<d.B, 1024, 0, st>>>(d, cls, pos, T);
    if (d.codec == 0) append_pack_kernel<false, 0><<<blocks, threads, 0, st>>>(d, kk, vv, cls, pos, T);
    else append_pack_kernel<false, 1><<<blocks, threads, 0, st>>>(d, kk, vv, cls, pos, T);
    append_finalize_kernel<<<(d.S * 4 + 255) / 256, 256, 0, st>>>(d);
    *launches += 3;
    return cudaGetLastError();
}

}  // namespace tkv
