// compact.cuh -- per-stream table compaction shared by the eviction kernels
// (tkv_evict_compact and tkv_evict_segments): given a keep decision per entry,
// each class table keeps its surviving entries in table order (scores carried
// over) and the slots of the evicted ones go on the class's free stack in
// reverse table order (ThinKV, Implementacao do Sistema / Continuous Thinking:
// freed slots are reused in place); in dense placement the kept records move
// down to slot = new table index instead.  Internal to libtkv.
#pragma once

#include <climits>

#include "tkv_internal.cuh"

namespace tkv {
namespace evict {

constexpr int kThreads = 512;
constexpr int kMoveBytes = 16384;   // dense placement: records staged per move batch
constexpr int kPer = 4;             // entries per thread in flight (passes) / per chunk (compaction)
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

// Compacts every class table of stream s.  keep_of(c, i, pos, score, tie) is the
// keep decision of entry i of class c (its pre-compaction index, position and
// score); it sets tie for entries whose decision is settled in table order among
// equal keys: the first rem0 such entries (over the classes in order) are kept.
// no_ties: keep_of never sets tie.  evicted[c] must equal the number of entries of
// class c that are not kept.  Called by all kThreads threads of the CTA.
template <class KeepFn>
__device__ __forceinline__ void compact_tables(const Dev &d, int s, const int (&n)[4], const int (&evicted)[4],
                                               KeepFn keep_of, bool no_ties, int rem0, int *scratch,
                                               int *move_src, uint4 *move_buf) {
    int tie_carry = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const size_t base_e = (size_t)s * d.cap[c];
        int32_t *hc = d.handle[c] + base_e;
        int32_t *pc = d.pos[c] + base_e;
        float *sc = d.score[c] + base_e;
        int32_t *fsc = d.fs[c] + base_e;
        const int m = evicted[c];
        const int ft0 = dclamp(d.err, d.ft[s * 4 + c], d.cap[c] - m, kDbgEvict + 0x10 + c);
        const int rec = d.rec[c];
        uint8_t *pool = d.pool[c] + base_e * rec;
        int kept_carry = 0, ev_carry = 0;
        // chunks of kPer * kThreads entries; thread t owns kPer consecutive entries, so
        // an exclusive block scan of per-thread counts plus a running count inside the
        // thread gives every entry its rank in table order
        for (int base = 0; base < n[c]; base += kPer * kThreads) {
            const int i0 = base + kPer * threadIdx.x;
            int32_t hd[kPer], pv[kPer];
            float sv[kPer];
            int keep[kPer], tie[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = i0 + j;
                const bool valid = i < n[c];
                hd[j] = valid ? hc[i] : 0;
                pv[j] = valid ? pc[i] : 0;
                sv[j] = valid ? sc[i] : 0.f;
            }
            int nt = 0, nk = 0, nv = 0;
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const bool valid = i0 + j < n[c];
                keep[j] = valid ? keep_of(c, i0 + j, pv[j], sv[j], tie[j]) : 0;
                if (!valid) tie[j] = 0;
                nt += tie[j];
                nv += valid;
            }
            if (!no_ties) {
                int ntie;
                int tr = block_scan(nt, &ntie, scratch) + tie_carry;
                tie_carry += ntie;
#pragma unroll
                for (int j = 0; j < kPer; ++j)
                    if (tie[j]) keep[j] = tr++ < rem0;
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) nk += keep[j];
            int nkeep;
            int wk = block_scan(nk, &nkeep, scratch) + kept_carry;
            int er = 0, nev = 0;
            if (!no_ties) er = block_scan(nv - nk, &nev, scratch) + ev_carry;
            else nev = min(kPer * kThreads, n[c] - base) - nkeep;
            // block_scan ends with a barrier: the whole chunk has been read
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = i0 + j;
                if (i >= n[c]) continue;
                if (keep[j]) {
                    hc[wk] = d.dense ? wk : hd[j];
                    pc[wk] = pv[j];
                    sc[wk] = sv[j];
                    if (d.dense) move_src[wk - kept_carry] = i;
                    ++wk;
                } else {
                    const int r = no_ties ? i - wk : er++;   // evicted entries of this class before i
                    if (!d.dense) fsc[ft0 + (m - 1 - r)] = hd[j];
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
            // writes of this chunk go to indices below the next chunk's reads; the
            // scan scratch and the move staging are protected by their own barriers
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

}  // namespace evict
}  // namespace tkv
