// evict.cu -- tkv_evict_compact: per-stream budgeted top-k on accumulated
// attention mass (DYNTS page, section 2.3, selection window: keep the k
// highest-scoring tokens and evict the rest; protected question-window tokens
// are never evicted) and stable compaction of the block table, with evicted
// slots handed to the class's free stack for in-place reuse (ThinKV,
// Implementacao do Sistema / Continuous Thinking).
//
// One CTA per stream.  Every unprotected entry gets a 64-bit key whose
// descending order is the eviction order: the high word maps the fp32 score
// bits monotonically onto uint32 (higher score = larger), the low word maps
// the position so that a lower position is larger.  An MSB-first radix select
// (8 bits per pass, shared-memory histogram) finds the key of the budget-th
// entry, stopping early once every entry sharing the selected prefix is kept.
// Exact 64-bit ties (equal score and position) fall back to class, then table
// index order, resolved by a block scan during compaction.  Compaction runs
// each class table chunk by chunk; a chunk is read into registers before any
// thread writes, and every write goes to an index no larger than its source,
// so the table compacts in place.  In dense placement (handle[i] == i) the kept
// records move the same way, from slot i to slot = new index, staged through
// shared memory in batches.
#include "tkv_internal.cuh"

namespace tkv {
namespace {

constexpr int kThreads = 512;
constexpr int kMoveBytes = 16384;   // dense placement: records staged per move batch
constexpr int kWarpsE = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint32_t score_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t entry_key(float score, int32_t pos) {
    const uint32_t p = ~(static_cast<uint32_t>(pos) ^ 0x80000000u);
    return (static_cast<uint64_t>(score_key(score)) << 32) | p;
}

__device__ __forceinline__ uint64_t top_bits(uint64_t k, int nbits) {
    return nbits == 0 ? 0ull : (k >> (64 - nbits));
}

// Exclusive block scan of v; *total receives the block sum.  scratch: >= 33 ints.
__device__ __forceinline__ int block_scan(int v, int *total, int *scratch) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[w] = x;
    __syncthreads();
    if (w == 0) {
        int y = lane < kWarpsE ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int z = __shfl_up_sync(kFull, y, o);
            if (lane >= o) y += z;
        }
        scratch[lane] = y;
    }
    __syncthreads();
    const int pre = (w > 0 ? scratch[w - 1] : 0) + x - v;
    *total = scratch[kWarpsE - 1];
    __syncthreads();
    return pre;
}

__device__ __forceinline__ int block_sum(int v, int *scratch) {
    int total;
    block_scan(v, &total, scratch);
    return total;
}

__global__ void __launch_bounds__(kThreads) evict_kernel(Dev d, int budget) {
    const int s = blockIdx.x;
    __shared__ unsigned hist[256];
    __shared__ int scratch[33];
    __shared__ int move_src[kThreads];                       // dense: source slot per kept entry
    __shared__ uint4 move_buf[kMoveBytes / sizeof(uint4)];
    __shared__ unsigned long long sh_prefix;
    __shared__ int sh_bits, sh_rem, sh_done;

    int n[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) n[c] = d.n[s * 4 + c];

    // 1. number of unprotected entries
    int cnt = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
        for (int i = threadIdx.x; i < n[c]; i += kThreads) cnt += pc[i] >= d.n_protect;
    }
    const int cand = block_sum(cnt, scratch);
    if (cand <= budget) return;

    // 2. radix select of the budget-th largest key (budget == 0: nothing kept)
    if (threadIdx.x == 0) {
        sh_prefix = 0ull;
        sh_bits = 0;
        sh_rem = budget;
        sh_done = budget == 0;
    }
    __syncthreads();
    for (int pass = 0; pass < 8 && !sh_done; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0u;
        __syncthreads();
        const uint64_t want = top_bits(sh_prefix, 8 * pass);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
            const float *sc = d.score[c] + (size_t)s * d.cap[c];
            // whole warps iterate together so equal digits can be counted with one
            // atomic per warp (scores cluster in a few exponents: per-lane atomics on
            // one bin would serialise)
            for (int base = 0; base < n[c]; base += kThreads) {
                const int i = base + threadIdx.x;
                unsigned digit = 256u;                     // 256: lane adds nothing
                if (i < n[c]) {
                    const int32_t p = pc[i];
                    if (p >= d.n_protect) {
                        const uint64_t key = entry_key(sc[i], p);
                        if (top_bits(key, 8 * pass) == want) digit = (unsigned)(key >> shift) & 255u;
                    }
                }
                const unsigned peers = __match_any_sync(kFull, digit);
                if (digit < 256u && (threadIdx.x & 31) == __ffs(peers) - 1)
                    atomicAdd(&hist[digit], (unsigned)__popc(peers));
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int acc = 0, dg = 255;
            for (; dg > 0; --dg) {
                if (acc + (int)hist[dg] >= sh_rem) break;
                acc += hist[dg];
            }
            sh_rem -= acc;
            sh_prefix |= static_cast<unsigned long long>(dg) << shift;
            sh_bits = 64 - shift;
            if ((int)hist[dg] == sh_rem) sh_done = 1;
        }
        __syncthreads();
    }
    const int nb = sh_bits, done = sh_done, rem0 = sh_rem;
    const uint64_t pref = top_bits(sh_prefix, nb);
    const bool keep_none = budget == 0;

    // 3. keep flags -> per-class evicted counts (first sweep), then the writes
    //    (second sweep).  Both sweeps replay the same tie order.
    int evicted[4];
    int tie_carry = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
        const float *sc = d.score[c] + (size_t)s * d.cap[c];
        int ev = 0;
        for (int base = 0; base < n[c]; base += kThreads) {
            const int i = base + threadIdx.x;
            int keep = 1, tie = 0;
            if (i < n[c]) {
                const int32_t p = pc[i];
                if (p >= d.n_protect) {
                    if (keep_none) {
                        keep = 0;
                    } else {
                        const uint64_t tb = top_bits(entry_key(sc[i], p), nb);
                        keep = tb > pref || (tb == pref && done);
                        tie = tb == pref && !done;
                    }
                }
            }
            int ntie;
            const int tr = block_scan(tie, &ntie, scratch) + tie_carry;
            tie_carry += ntie;
            if (tie) keep = tr < rem0;
            ev += block_sum(i < n[c] ? !keep : 0, scratch);
        }
        evicted[c] = ev;
    }
    tie_carry = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const size_t base_e = (size_t)s * d.cap[c];
        int32_t *hc = d.handle[c] + base_e;
        int32_t *pc = d.pos[c] + base_e;
        float *sc = d.score[c] + base_e;
        int32_t *fsc = d.fs[c] + base_e;
        const int ft0 = d.ft[s * 4 + c];
        const int m = evicted[c];
        const int rec = d.rec[c];
        uint8_t *pool = d.pool[c] + base_e * rec;
        int kept_carry = 0, ev_carry = 0;
        for (int base = 0; base < n[c]; base += kThreads) {
            const int i = base + threadIdx.x;
            int keep = 1, tie = 0;
            int32_t hd = 0, p = 0;
            float scv = 0.f;
            if (i < n[c]) {
                hd = hc[i];
                p = pc[i];
                scv = sc[i];
                if (p >= d.n_protect) {
                    if (keep_none) {
                        keep = 0;
                    } else {
                        const uint64_t tb = top_bits(entry_key(scv, p), nb);
                        keep = tb > pref || (tb == pref && done);
                        tie = tb == pref && !done;
                    }
                }
            }
            int ntie;
            const int tr = block_scan(tie, &ntie, scratch) + tie_carry;
            tie_carry += ntie;
            if (tie) keep = tr < rem0;
            const int valid = i < n[c];
            int nkeep, nev;
            const int wk = block_scan(valid && keep, &nkeep, scratch) + kept_carry;
            const int r = block_scan(valid && !keep, &nev, scratch) + ev_carry;
            // block_scan ends with a barrier: the whole chunk has been read
            if (valid) {
                if (keep) {
                    hc[wk] = d.dense ? wk : hd;
                    pc[wk] = p;
                    sc[wk] = scv;
                    if (d.dense) move_src[wk - kept_carry] = i;
                } else if (!d.dense) {
                    fsc[ft0 + (m - 1 - r)] = hd;
                }
            }
            if (d.dense) {
                // move this chunk's kept records from slot i to slot wk (wk <= i), in
                // batches staged through shared memory: a batch is read completely before
                // any of it is written, and later batches only read slots above this one's
                __syncthreads();
                const int per_rec = rec / 16;
                const int batch = kMoveBytes / rec;
                for (int b0 = 0; b0 < nkeep; b0 += batch) {
                    const int nb_rec = min(batch, nkeep - b0);
                    const int pieces = nb_rec * per_rec;
                    for (int q = threadIdx.x; q < pieces; q += kThreads) {
                        const int k = q / per_rec, part = q - k * per_rec;
                        move_buf[k * per_rec + part] =
                            reinterpret_cast<const uint4 *>(pool + (size_t)move_src[b0 + k] * rec)[part];
                    }
                    __syncthreads();
                    for (int q = threadIdx.x; q < pieces; q += kThreads) {
                        const int k = q / per_rec, part = q - k * per_rec;
                        reinterpret_cast<uint4 *>(pool + (size_t)(kept_carry + b0 + k) * rec)[part] =
                            move_buf[k * per_rec + part];
                    }
                    __syncthreads();
                }
            }
            kept_carry += nkeep;
            ev_carry += nev;
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            d.n[s * 4 + c] = n[c] - m;
            if (d.dense) {
                d.ft[s * 4 + c] = 0;
                d.hw[s * 4 + c] = n[c] - m;
            } else {
                d.ft[s * 4 + c] = ft0 + m;
            }
        }
    }
}

}  // namespace

cudaError_t launch_evict(const Dev &d, int budget, cudaStream_t st, int64_t *launches) {
    evict_kernel<<<d.S, kThreads, 0, st>>>(d, budget);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tkv
