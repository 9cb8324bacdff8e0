// evict_segments.cu -- tkv_evict_segments: segment-level eviction (ThinKV,
// Metodologia, TBE paragraph: when a Transition thought starts, the tokens of
// earlier R/E thought segments are evicted progressively on an annealing
// schedule, segment by segment rather than token by token, and a few Transition
// tokens are kept as a safety net).  The caller gives each batch row's segments
// and the retention of each (tkv_tbe_schedule computes it from the labels);
// inside a segment the kept tokens are the first under the same order as the
// token-level eviction (score desc, position asc), then table index.
//
// One CTA per stream.  The row's segment table is staged in shared memory.  A
// first sweep over the class tables marks every entry kept and records, for
// each segment, the run of its label's class table that holds it (a class table
// is ordered by position, so a segment is one contiguous run).  Then a warp per
// segment that must shrink ranks the run: every lane counts, for the entries it
// owns, the run's keys that precede them (keys staged in shared memory 256 at a
// time); protected entries rank first and add to the retention.  A retention of
// 0 needs no ranking, and a small one (about r < n / 2) is taken by r warp
// arg-max rounds instead (O(r n / 32) rather than O(n^2 / 32)).  The keep flags
// (a byte per entry, in the step's logits scratch, which the next decode call
// rewrites anyway) then drive the shared table compaction.
#include "compact.cuh"

namespace tkv {
namespace {

using namespace evict;

constexpr int kMaxSeg = 4096;   // segments per batch row
constexpr int kStage = 256;     // keys a warp stages in shared memory at a time
constexpr int kOwn = 8;         // entries a lane ranks per round (32 * kOwn per warp)

__host__ __device__ constexpr int seg_table_bytes(int ms) {
    return (17 * ms + 15) & ~15;   // starts, keep, lo, hi (int32) and label (uint8) per segment
}
constexpr int kUnionBytes = kWarpsE * kStage * 8 > kMoveBytes ? kWarpsE * kStage * 8 : kMoveBytes;

__global__ void __launch_bounds__(kThreads) tbe_kernel(Dev d, const int32_t *__restrict__ seg_start,
                                                       const uint8_t *__restrict__ seg_label,
                                                       const int32_t *__restrict__ seg_keep,
                                                       const int32_t *__restrict__ nseg, int max_seg) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ int move_src[kPer * kThreads];
    __shared__ int scratch[33];
    const int ms = (max_seg + 3) & ~3;
    int *starts = reinterpret_cast<int *>(dyn);
    int *keep = starts + ms;
    int *lo = keep + ms;
    int *hi = lo + ms;
    uint8_t *label = reinterpret_cast<uint8_t *>(hi + ms);
    uint8_t *un = dyn + seg_table_bytes(ms);   // ranking stage, later the record move staging
    uint4 *move_buf = reinterpret_cast<uint4 *>(un);

    const int s = blockIdx.x, b = s / d.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ns = min(max(nseg[b], 0), max_seg);
    for (int j = tid; j < ns; j += kThreads) {
        starts[j] = seg_start[(size_t)b * max_seg + j];
        keep[j] = seg_keep[(size_t)b * max_seg + j];
        label[j] = seg_label[(size_t)b * max_seg + j];
        lo[j] = 0;
        hi[j] = 0;
    }
    int n[4], cbase[4];
    {
        int acc = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            n[c] = d.n[s * 4 + c];
            cbase[c] = acc;   // the flags of class c start here
            acc += d.cap[c];
        }
    }
    uint8_t *flags = reinterpret_cast<uint8_t *>(d.logits + (size_t)s * d.ncap * d.G);
    __syncthreads();

    // segment of position p: the last j with starts[j] <= p, -1 before the first
    auto seg_of = [&](int32_t p) -> int {
        int a = 0, e = ns;
        while (a < e) {
            const int mid = (a + e) >> 1;
            if (starts[mid] <= p) a = mid + 1; else e = mid;
        }
        return a - 1;
    };

    // 1. every entry kept; each segment's run [lo, hi) in its label's class table
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
        for (int i = tid; i < n[c]; i += kThreads) {
            flags[cbase[c] + i] = 1;
            const int32_t p = pc[i];
            const int j = seg_of(p);
            if (j < 0 || label[j] != c) continue;   // before the first segment, or foreign: kept
            if (i == 0 || pc[i - 1] < starts[j]) lo[j] = i;
            if (i == n[c] - 1 || (j + 1 < ns && pc[i + 1] >= starts[j + 1])) hi[j] = i + 1;
        }
    }
    __syncthreads();

    // 2. a warp per segment that must shrink: entry idx of the run is kept iff fewer
    //    than (retention + protected entries of the run) keys precede it
    uint64_t *st = reinterpret_cast<uint64_t *>(un) + warp * kStage;
    int shrunk = 0;
    for (int j = warp; j < ns; j += kWarpsE) {
        const int r = keep[j], c = label[j];
        if (r < 0 || c > 3) continue;
        const int a = lo[j], e = hi[j];
        if (e - a <= r) continue;
        const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
        const float *sc = d.score[c] + (size_t)s * d.cap[c];
        auto key_of = [&](int i) -> uint64_t {
            const int32_t p = pc[i];
            return p < d.n_protect ? ~0ull : entry_key(sc[i], p);
        };
        int np = 0;
        for (int i = a + lane; i < e; i += 32) np += pc[i] < d.n_protect;
        const int budget = r + __reduce_add_sync(kFull, np);
        if (e - a <= budget) continue;
        shrunk = 1;
        if (r == 0) {   // only the protected entries stay
            for (int i = a + lane; i < e; i += 32) flags[cbase[c] + i] = pc[i] < d.n_protect;
            continue;
        }
        const int cnt = e - a, per = (cnt + 31) >> 5;
        if (cnt <= 32 * kOwn && budget * 64 < cnt * per * 32) {
            // small retention: pick the first key under (key desc, index asc) budget
            // times; a warp arg-max per pick
            uint64_t ok[kOwn];
            bool sel[kOwn];
#pragma unroll
            for (int m = 0; m < kOwn; ++m) {
                const int idx = a + lane + 32 * m;
                ok[m] = idx < e ? key_of(idx) : 0ull;
                sel[m] = idx >= e;   // not a candidate
            }
            for (int it = 0; it < budget; ++it) {
                uint64_t bk = 0ull;
                int bi = INT_MAX, have = 0;
#pragma unroll
                for (int m = 0; m < kOwn; ++m) {
                    const int idx = a + lane + 32 * m;
                    if (!sel[m] && (!have || ok[m] > bk || (ok[m] == bk && idx < bi))) {
                        bk = ok[m];
                        bi = idx;
                        have = 1;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const uint64_t k2 = __shfl_xor_sync(kFull, bk, o);
                    const int i2 = __shfl_xor_sync(kFull, bi, o), h2 = __shfl_xor_sync(kFull, have, o);
                    if (h2 && (!have || k2 > bk || (k2 == bk && i2 < bi))) {
                        bk = k2;
                        bi = i2;
                        have = 1;
                    }
                }
#pragma unroll
                for (int m = 0; m < kOwn; ++m)
                    if (a + lane + 32 * m == bi) sel[m] = true;
            }
#pragma unroll
            for (int m = 0; m < kOwn; ++m) {
                const int idx = a + lane + 32 * m;
                if (idx < e) flags[cbase[c] + idx] = sel[m];
            }
            continue;
        }
        for (int base = a; base < e; base += 32 * kOwn) {
            uint64_t ok[kOwn];
            int rk[kOwn];
#pragma unroll
            for (int m = 0; m < kOwn; ++m) {
                const int idx = base + lane + 32 * m;
                ok[m] = idx < e ? key_of(idx) : 0ull;
                rk[m] = 0;
            }
            for (int cb = a; cb < e; cb += kStage) {
                const int cn = min(kStage, e - cb);
                __syncwarp();
                for (int t = lane; t < cn; t += 32) st[t] = key_of(cb + t);
                __syncwarp();
                for (int t = 0; t < cn; ++t) {
                    const uint64_t kt = st[t];
                    const int it = cb + t;
#pragma unroll
                    for (int m = 0; m < kOwn; ++m) {
                        if (base + 32 * m >= e) break;   // warp-uniform
                        const int im = base + lane + 32 * m;
                        rk[m] += (kt > ok[m]) || (kt == ok[m] && it < im);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < kOwn; ++m) {
                const int idx = base + lane + 32 * m;
                if (idx < e) flags[cbase[c] + idx] = rk[m] < budget;
            }
        }
    }
    if (!__syncthreads_or(shrunk)) return;   // every segment within its retention

    // 3. evicted entries per class, then the shared compaction
    int evicted[4];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        int ev = 0;
        for (int i = tid; i < n[c]; i += kThreads) ev += !flags[cbase[c] + i];
        evicted[c] = block_sum(ev, scratch);
    }
    auto keep_of = [&](int c, int i, int32_t, float, int &tie) -> int {
        tie = 0;
        return flags[cbase[c] + i];
    };
    compact_tables(d, s, n, evicted, keep_of, true, 0, scratch, move_src, move_buf);
}

}  // namespace

int evict_segments_max() { return kMaxSeg; }

cudaError_t launch_evict_segments(const Dev &d, const int32_t *seg_start, const uint8_t *seg_label,
                                  const int32_t *seg_keep, const int32_t *nseg, int max_seg, cudaStream_t st,
                                  int64_t *launches) {
    static bool configured = false;
    const int smem = seg_table_bytes((max_seg + 3) & ~3) + kUnionBytes;
    if (!configured) {
        const cudaError_t e = cudaFuncSetAttribute(tbe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   seg_table_bytes(kMaxSeg) + kUnionBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    tbe_kernel<<<d.S, kThreads, smem, st>>>(d, seg_start, seg_label, seg_keep, nseg, max_seg);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tkv
