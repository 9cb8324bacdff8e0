// tkv_internal.cuh -- device-side view of a cache workspace and the launchers
// of the sm_100a kernels.  Internal to libtkv (the C ABI is include/tkv.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace tkv {

constexpr int kD = 128;       // head dim
constexpr int kGroup = 32;    // quantisation group along head dim
constexpr int kNG = kD / kGroup;
constexpr int kMaxG = 8;      // query heads per kv head supported

// Record bytes of a class with `bits` bits per element (bits == 16: bf16) under codec 0
// (integer codes, fp16 scale + zero per group) or codec 1 (floating-point codes: FP8
// and ternary with an fp16 scale per group, NVFP4 with an E4M3 scale per 16 dims).
__host__ __device__ constexpr int record_bytes(int bits, int codec = 0) {
    return bits == 16 ? 4 * kD
           : codec == 0 ? 2 * (kD * bits / 8) + 4 * kNG * 2
           : bits == 4 ? 2 * (kD / 2) + 2 * (kD / 16)
                       : 2 * (kD * bits / 8) + 2 * kNG * 2;
}

// Everything a kernel needs to address one cache.  Passed by value.
struct Dev {
    int B, Hkv, G, S, n_protect, max_append;
    int dense;              // 1: live records contiguous in table order (handle[i] == i)
    int attn_kernel;        // 0: warp-tile kernel, 1: tensor-memory (tcgen05) kernel, 2: warp-tile on a TMA pipeline
    int codec;              // 0: integer class records, 1: FP8 / NVFP4 / ternary class records
    int cap[4];
    int rec[4];
    int32_t *n, *ft, *hw;   // [S][4]
    uint32_t *err;          // [0] first status, [1] count, [2] detail
    int32_t *handle[4], *pos[4], *fs[4];
    float *score[4];
    uint8_t *pool[4];
    // scratch
    int32_t *rank;     // [B][max_append] rank of a new token within its class
    int32_t *totals;   // [B][4] tokens per class in the current append
    float *logits;     // [S][ncap][G] raw logits (log2 domain) of the current step
    int ncap;          // sum of cap[c], rounded up to a multiple of 32
    // tensor-core decode attention (attention_i8.cu): per (stream, CTA, warpgroup)
    // partial results, slot 2 (s + cta) + warpgroup, part_floats(G) floats each, and
    // the first / last CTA of every stream
    float *part;       // [2 (S + ncta_max)][part_floats(G)]
    int32_t *seg_lo, *seg_hi;   // [S]
    int ncta_max;
};

// Floats of one partial result of the tensor-core decode attention: running max,
// sum and sum p*(x - m) per head, then the unnormalised O [G][D].
__host__ __device__ constexpr int part_floats(int G) { return G * (3 + kD); }
constexpr int kNctaMax = 1024;   // upper bound on the persistent grid (one CTA per SM)
__host__ __device__ constexpr size_t part_bytes(size_t S, int G) {
    return 2 * (S + kNctaMax) * (size_t)part_floats(G) * sizeof(float);
}

// TMA descriptors of the record pools for the tensor-core decode attention:
// m[class][0 = code boxes, 1 = scale / zero box][0 = a whole tile's rows, 1 = 16 rows].
struct I8Maps {
    CUtensorMap m[4][2][2];
};

enum : uint32_t { kErrInvalid = 1, kErrCapacity = 2, kErrTimeout = 4 };

__device__ __forceinline__ void raise_error(uint32_t *err, uint32_t code, uint32_t detail) {
    if (atomicCAS(err, 0u, code) == 0u) err[2] = detail;
    atomicAdd(err + 1, 1u);
}

// Bounds checks of the TKV_DEBUG build (libtkv_debug.so; the pages' pipeline has no
// counterpart: it stands in for a memory checker).  Before a table or pool access the
// kernels check the counters and slot handles they index with against the cache's
// capacities; a failed check latches TKV_ERR_INVALID with the check's id as detail
// (kDbg* below, + class) and the access is skipped or its index clamped into range.
// Release builds compile every check to `true` / the unchanged value.
enum : uint32_t { kDbgAppend = 0x100, kDbgAttention = 0x200, kDbgEvict = 0x300, kDbgSegments = 0x400 };
#ifdef TKV_DEBUG
__device__ __forceinline__ bool dcheck(uint32_t *err, bool ok, uint32_t id) {
    if (!ok) raise_error(err, kErrInvalid, id);
    return ok;
}
__device__ __forceinline__ int dclamp(uint32_t *err, int v, int hi, uint32_t id) {
    if (v < 0 || v > hi) {
        raise_error(err, kErrInvalid, id);
        return v < 0 ? 0 : hi;
    }
    return v;
}
#else
__device__ __forceinline__ bool dcheck(uint32_t *, bool, uint32_t) { return true; }
__device__ __forceinline__ int dclamp(uint32_t *, int v, int, uint32_t) { return v; }
#endif

// Host-side per-device facts, looked up once per device and thread-safe (racing
// first calls compute and store the same value).
constexpr int kMaxDevices = 64;
// SM count of the current device; 0 (and the CUDA error) if it cannot be read.
cudaError_t device_sm_count(int *sms);
// Resident CTAs per SM of `kernel` with `threads` threads and `smem` dynamic shared
// bytes on the current device, cached in slot[device] (0 means "not yet known").
cudaError_t cached_blocks_per_sm(int *slot_per_device, const void *kernel, int threads, size_t smem,
                                 int *blocks);
// Clusters of C CTAs of `kernel` (threads per CTA, dynamic shared memory smem, already set
// up by cached_blocks_per_sm) that the current device holds at once, cached per device in
// slot_per_device.  A cluster lives within one GPC, so on a part whose GPCs hold an odd
// number of SMs this is below blocks-per-SM x SMs / C.
cudaError_t cached_max_clusters(int *slot_per_device, const void *kernel, int threads, size_t smem, int C,
                                int *clusters);

// Launchers (each returns the CUDA error of its launches and adds the number
// of kernels it launched to *launches).
cudaError_t launch_append(const Dev &d, const void *k, const void *v, const uint8_t *cls,
                          const int32_t *pos, int T, cudaStream_t st, int64_t *launches);
// Warp-tile decode attention; with `sparsity` non-NULL it also writes, per (stream, query
// head), the attention sparsity and (thought non-NULL) its thought class.  q_ready: the
// kernel before it on `st` is launch_append's (launched in plain stream order), so the
// query may be read before that kernel completes.
cudaError_t launch_attention(const Dev &d, const void *q, float scale, float *out,
                             long long live_ub, cudaStream_t st, int64_t *launches, float *sparsity = nullptr,
                             uint8_t *thought = nullptr, float th_r = 0.f, float th_t = 0.f, bool q_ready = false);
// Dense placement: the tensor-core kernel with integer operands (attention_i8.cu).  With
// sparsity / thought non-NULL it also writes, per (stream, query head), the attention
// sparsity 1 - H(p) / ln N and its thought class under the thresholds th_r <= th_t.
cudaError_t launch_attention_i8(const Dev &d, const I8Maps &maps, const void *q, float scale, float *out,
                                float *sparsity, uint8_t *thought, float th_r, float th_t, long long live_ub,
                                cudaStream_t st, int64_t *launches);
// Encodes the TMA descriptors of d's pools (host only; needs the CUDA driver).
cudaError_t make_i8_maps(const Dev &d, I8Maps *maps);
// Dense placement, attn_kernel 2: the warp-tile math fed by a persistent TMA pipeline
// (attention_ws.cu).
cudaError_t launch_attention_ws(const Dev &d, const I8Maps &maps, const void *q, float scale, float *out,
                                long long live_ub, cudaStream_t st, int64_t *launches);
// Self-test of the bounded device waits (selftest.cu).
cudaError_t launch_wait_timeout(const Dev &d, long long limit, cudaStream_t st, int64_t *launches);
cudaError_t launch_evict(const Dev &d, int budget, int keep_from, cudaStream_t st, int64_t *launches);
// Segment-level eviction (evict_segments.cu); evict_segments_max() segments per row.
int evict_segments_max();
cudaError_t launch_evict_segments(const Dev &d, const int32_t *seg_start, const uint8_t *seg_label,
                                  const int32_t *seg_keep, const int32_t *nseg, int max_seg, cudaStream_t st,
                                  int64_t *launches);
// Thought-aware segment budgets with pivotal tokens (evict_segments.cu, TAM mode).
cudaError_t launch_evict_tam(const Dev &d, const int32_t *seg_start, const uint8_t *seg_label, const int32_t *nseg,
                             int max_seg, int budget, double c, cudaStream_t st, int64_t *launches);

}  // namespace tkv
