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
//
// The same kernel, instantiated with TAM = true, serves tkv_evict_tam: the
// thought-aware budget allocation of the TAM page (sections 2.B and 2.C) as a
// selection policy.  After the first sweep a warp per segment counts the
// segment's candidates (unprotected entries of its run) and sums their scores
// exactly (integer digits: the same sum in any order); the block forms the stream's mean, delta = c * mean, the pivotal
// candidates (score >= delta: kept, ranked first like protected entries) and the
// budgets t_j = min(n_j - p_j, floor(T' (a_j / D) + 1e-9)) with a_j = sqrt(w_j) n_j,
// D = sum a_j, T' = max(0, budget - pivotal), which then play the role of the
// retentions.
#include <cmath>

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
__host__ __device__ constexpr int tam_table_bytes(int ms) {
    return 16 * ms;                // score sum (fp64), candidates and pivotal (int32) per segment
}
constexpr int kUnionBytes = kWarpsE * kStage * 8 > kMoveBytes ? kWarpsE * kStage * 8 : kMoveBytes;

// Exact sums of fp32 scores for the TAM means.  A finite non-negative fp32 is
// m * 2^(b - 149) (m < 2^24, 0 <= b <= 253), so a sum of them is an integer times
// 2^-149 held in nine 32-bit digits, each in a 64-bit counter with room for the
// carries of 2^32 terms: integer adds, so every summation order gives the same sum.
// Negative and non-finite scores (attention mass is neither) count as 0.
constexpr int kDig = 9;
__device__ __forceinline__ void xsum_add(unsigned long long (&a)[kDig], float v) {
    const uint32_t u = __float_as_uint(v);
    const uint32_t eb = u >> 23;
    if (u == 0u || eb >= 255u) return;
    const unsigned long long m = eb ? ((u & 0x7FFFFFu) | 0x800000u) : (u & 0x7FFFFFu);
    const int b = eb ? (int)eb - 1 : 0;
    const unsigned long long x = m << (b & 31);
    const int i = b >> 5;
#pragma unroll
    for (int k = 0; k < kDig; ++k) {   // register-resident digits: no indexed access
        if (k == i) a[k] += x & 0xFFFFFFFFull;
        if (k == i + 1) a[k] += x >> 32;
    }
}
// The sum rounded to the nearest double (ties to even): the leading 64 bits, with every
// bit below them folded into the lowest (sticky), converted once and scaled by 2^e.
__device__ double xsum_value(const unsigned long long (&a)[kDig]) {
    uint32_t dig[kDig + 2];
    unsigned long long carry = 0;
#pragma unroll
    for (int k = 0; k < kDig; ++k) {
        const unsigned long long t = a[k] + carry;
        dig[k] = (uint32_t)t;
        carry = t >> 32;
    }
    dig[kDig] = (uint32_t)carry;
    dig[kDig + 1] = (uint32_t)(carry >> 32);
    int top = kDig + 1;
    while (top >= 0 && dig[top] == 0u) --top;
    if (top < 0) return 0.0;
    const unsigned long long w2 = dig[top], w1 = top >= 1 ? dig[top - 1] : 0u, w0 = top >= 2 ? dig[top - 2] : 0u;
    bool sticky = false;
    for (int k = 0; k < top - 2; ++k) sticky |= dig[k] != 0u;
    const int lz = __clz((int)(uint32_t)w2);
    unsigned long long t = ((w2 << 32) | w1) << lz;
    if (lz) t |= w0 >> (32 - lz);
    if (((w0 << lz) & 0xFFFFFFFFull) != 0ull || sticky) t |= 1ull;
    const int e = 32 - lz + 32 * (top - 2) - 149;   // in [-212, 202]: 2^e is a normal double
    return __dmul_rn(__ull2double_rn(t), __longlong_as_double((long long)(1023 + e) << 52));
}

template <bool TAM>
__global__ void __launch_bounds__(kThreads) tbe_kernel(Dev d, const int32_t *__restrict__ seg_start,
                                                       const uint8_t *__restrict__ seg_label,
                                                       const int32_t *__restrict__ seg_keep,
                                                       const int32_t *__restrict__ nseg, int max_seg,
                                                       int budget, double cpiv) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ int move_src[kPer * kThreads];
    __shared__ int scratch[33];
    const int ms = (max_seg + 3) & ~3;
    int *starts = reinterpret_cast<int *>(dyn);
    int *keep = starts + ms;
    int *lo = keep + ms;
    int *hi = lo + ms;
    uint8_t *label = reinterpret_cast<uint8_t *>(hi + ms);
    double *ssum = reinterpret_cast<double *>(dyn + seg_table_bytes(ms));   // TAM only: w_j n_j, then a_j
    int *scnt = reinterpret_cast<int *>(ssum + ms);
    int *spiv = scnt + ms;
    uint8_t *un = dyn + seg_table_bytes(ms) + (TAM ? tam_table_bytes(ms) : 0);   // ranking stage, then moves
    uint4 *move_buf = reinterpret_cast<uint4 *>(un);
    __shared__ double sh_delta, sh_D;
    __shared__ unsigned long long tot_dig[kDig];   // TAM: exact sum of every candidate's score

    const int s = blockIdx.x, b = s / d.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ns = min(max(nseg[b], 0), max_seg);
    for (int j = tid; j < ns; j += kThreads) {
        starts[j] = seg_start[(size_t)b * max_seg + j];
        keep[j] = TAM ? 0 : seg_keep[(size_t)b * max_seg + j];
        label[j] = seg_label[(size_t)b * max_seg + j];
        lo[j] = 0;
        hi[j] = 0;
    }
    int n[4], cbase[4];
    {
        int acc = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            n[c] = dclamp(d.err, d.n[s * 4 + c], d.cap[c], kDbgSegments + c);
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

    double delta = 0.0;   // TAM: candidates scoring at least delta are pivotal
    if constexpr (TAM) {
        if (tid < kDig) tot_dig[tid] = 0ull;
        __syncthreads();
        // T1. per segment: candidates and the exact sum of their scores
        for (int j = warp; j < ns; j += kWarpsE) {
            const int c = label[j];
            int n = 0;
            unsigned long long a[kDig];
#pragma unroll
            for (int k = 0; k < kDig; ++k) a[k] = 0ull;
            if (c <= 3) {
                const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
                const float *sc = d.score[c] + (size_t)s * d.cap[c];
                for (int i = lo[j] + lane; i < hi[j]; i += 32)
                    if (pc[i] >= d.n_protect) { ++n; xsum_add(a, sc[i]); }
            }
            n = __reduce_add_sync(kFull, n);
#pragma unroll
            for (int k = 0; k < kDig; ++k)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) a[k] += __shfl_xor_sync(kFull, a[k], o);
            if (lane == 0) {
                scnt[j] = n;
                ssum[j] = xsum_value(a);
#pragma unroll
                for (int k = 0; k < kDig; ++k)
                    if (a[k]) atomicAdd(&tot_dig[k], a[k]);
            }
        }
        __syncthreads();   // every segment's count and sum written
        // T2. the stream's mean score over all candidates -> delta
        {
            int n = 0;
            for (int j = tid; j < ns; j += kThreads) n += scnt[j];
            const int ntot = block_sum(n, scratch);   // ends with a barrier: tot_dig complete
            if (tid == 0) {
                unsigned long long t[kDig];
#pragma unroll
                for (int k = 0; k < kDig; ++k) t[k] = tot_dig[k];
                sh_delta = ntot > 0 ? __dmul_rn(cpiv, __ddiv_rn(xsum_value(t), (double)ntot)) : -1.0;
            }
            __syncthreads();
            if (ntot == 0) return;   // no candidates: nothing to evict
            delta = sh_delta;
        }
        // T3. pivotal candidates per segment
        for (int j = warp; j < ns; j += kWarpsE) {
            const int c = label[j];
            int p = 0;
            if (c <= 3) {
                const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
                const float *sc = d.score[c] + (size_t)s * d.cap[c];
                for (int i = lo[j] + lane; i < hi[j]; i += 32)
                    p += pc[i] >= d.n_protect && (double)sc[i] >= delta;
            }
            p = __reduce_add_sync(kFull, p);
            if (lane == 0) spiv[j] = p;
        }
        __syncthreads();
        // T4. budgets: T' = max(0, budget - pivotal), t_j = min(n_j - p_j, floor(T' a_j / D + 1e-9)),
        // a_j = sqrt(w_j) n_j and D = sum a_j in segment order (every operation rounded once,
        // no fused multiply-add: the same doubles as a plain sequential evaluation)
        {
            int P = 0;
            for (int j = tid; j < ns; j += kThreads) {
                const int n = scnt[j];
                ssum[j] = n > 0 ? __dmul_rn(__dsqrt_rn(__ddiv_rn(ssum[j], (double)n)), (double)n) : 0.0;
                P += spiv[j];
            }
            const int Ptot = block_sum(P, scratch);   // ends with a barrier: every a_j written
            if (tid == 0) {
                double D = 0.0;
                for (int j = 0; j < ns; ++j)
                    if (scnt[j] > 0) D = __dadd_rn(D, ssum[j]);
                sh_D = D;
            }
            __syncthreads();
            const double D = sh_D;
            const double Tp = budget > Ptot ? (double)(budget - Ptot) : 0.0;
            for (int j = tid; j < ns; j += kThreads) {
                long long t = 0;
                if (scnt[j] > 0 && D > 0.0)
                    t = (long long)floor(__dadd_rn(__dmul_rn(Tp, __ddiv_rn(ssum[j], D)), 1e-9));
                const int cap_j = scnt[j] - spiv[j];
                keep[j] = (int)(t < cap_j ? t : cap_j);
            }
            __syncthreads();
        }
    }

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
        // protected (and, for TAM, pivotal) entries always stay: they rank first
        auto fixed = [&](int i) -> bool {
            return pc[i] < d.n_protect || (TAM && (double)sc[i] >= delta);
        };
        auto key_of = [&](int i) -> uint64_t { return fixed(i) ? ~0ull : entry_key(sc[i], pc[i]); };
        int np = 0;
        for (int i = a + lane; i < e; i += 32) np += fixed(i);
        const int budget = r + __reduce_add_sync(kFull, np);
        if (e - a <= budget) continue;
        shrunk = 1;
        if (r == 0) {   // only the protected (pivotal) entries stay
            for (int i = a + lane; i < e; i += 32) flags[cbase[c] + i] = fixed(i);
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

template <bool TAM>
cudaError_t launch_mode(const Dev &d, const int32_t *seg_start, const uint8_t *seg_label, const int32_t *seg_keep,
                        const int32_t *nseg, int max_seg, int budget, double cpiv, cudaStream_t st,
                        int64_t *launches) {
    static bool configured = false;
    const int ms = (max_seg + 3) & ~3;
    const int smem = seg_table_bytes(ms) + (TAM ? tam_table_bytes(ms) : 0) + kUnionBytes;
    if (!configured) {
        const cudaError_t e = cudaFuncSetAttribute(
            tbe_kernel<TAM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
            seg_table_bytes(kMaxSeg) + (TAM ? tam_table_bytes(kMaxSeg) : 0) + kUnionBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    tbe_kernel<TAM><<<d.S, kThreads, smem, st>>>(d, seg_start, seg_label, seg_keep, nseg, max_seg, budget, cpiv);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_evict_segments(const Dev &d, const int32_t *seg_start, const uint8_t *seg_label,
                                  const int32_t *seg_keep, const int32_t *nseg, int max_seg, cudaStream_t st,
                                  int64_t *launches) {
    return launch_mode<false>(d, seg_start, seg_label, seg_keep, nseg, max_seg, 0, 0.0, st, launches);
}

cudaError_t launch_evict_tam(const Dev &d, const int32_t *seg_start, const uint8_t *seg_label, const int32_t *nseg,
                             int max_seg, int budget, double c, cudaStream_t st, int64_t *launches) {
    return launch_mode<true>(d, seg_start, seg_label, nullptr, nseg, max_seg, budget, c, st, launches);
}

int evict_segments_max() { return kMaxSeg; }

}  // namespace tkv
