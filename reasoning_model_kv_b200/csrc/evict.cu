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
#include "compact.cuh"

namespace tkv {
namespace {

using namespace evict;

// keep_from: positions >= keep_from (a local window of recent tokens) are kept and
// are not candidates; INT32_MAX disables the window.
__global__ void __launch_bounds__(kThreads) evict_kernel(Dev d, int budget, int keep_from) {
    const int s = blockIdx.x;
    __shared__ unsigned hist[256];
    __shared__ int scratch[33];
    __shared__ int move_src[kPer * kThreads];                // dense: source slot per kept entry
    __shared__ uint4 move_buf[kMoveBytes / sizeof(uint4)];
    __shared__ unsigned long long sh_prefix;
    __shared__ int sh_bits, sh_rem, sh_done, sh_cand;

    int n[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) n[c] = dclamp(d.err, d.n[s * 4 + c], d.cap[c], kDbgEvict + c);

    // 1+2. radix select of the budget-th largest key (budget == 0: nothing kept);
    //      pass 0 also counts the unprotected entries
    if (threadIdx.x == 0) {
        sh_prefix = 0ull;
        sh_bits = 0;
        sh_rem = budget;
        sh_done = budget == 0;
        sh_cand = 0;
    }
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
        if (pass > 0 && sh_done) break;
        const int shift = 56 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0u;
        __syncthreads();
        const uint64_t want = top_bits(sh_prefix, 8 * pass);
        int cnt = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
            const float *sc = d.score[c] + (size_t)s * d.cap[c];
            // whole warps iterate together so equal digits can be counted with one
            // atomic per warp (scores cluster in a few exponents: per-lane atomics on
            // one bin would serialise)
            for (int base = 0; base < n[c]; base += kPer * kThreads) {
                int32_t pv[kPer];
                float sv[kPer];
#pragma unroll
                for (int j = 0; j < kPer; ++j) {             // all loads first: kPer in flight
                    const int i = base + j * kThreads + threadIdx.x;
                    pv[j] = i < n[c] ? pc[i] : INT_MIN;
                    sv[j] = i < n[c] ? sc[i] : 0.f;
                }
#pragma unroll
                for (int j = 0; j < kPer; ++j) {
                    unsigned digit = 256u;                     // 256: lane adds nothing
                    if (pv[j] >= d.n_protect && pv[j] < keep_from) {
                        ++cnt;
                        const uint64_t key = entry_key(sv[j], pv[j]);
                        if (top_bits(key, 8 * pass) == want) digit = (unsigned)(key >> shift) & 255u;
                    }
                    const unsigned peers = __match_any_sync(kFull, digit);
                    if (digit < 256u && (threadIdx.x & 31) == __ffs(peers) - 1)
                        atomicAdd(&hist[digit], (unsigned)__popc(peers));
                }
            }
        }
        if (pass == 0) {
            cnt = __reduce_add_sync(kFull, cnt);
            if ((threadIdx.x & 31) == 0) atomicAdd(&sh_cand, cnt);
        }
        __syncthreads();
        if (sh_cand <= budget) return;   // nothing to evict (uniform: read after the barrier)
        if (sh_done) break;              // budget 0: every unprotected entry goes
        // warp 0 picks the digit: the first bin, from the top, where the count of
        // keys at or above it reaches the remaining rank (bin 0 if none does)
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            unsigned h[8];
            int sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                h[j] = hist[255 - 8 * lane - j];
                sum += (int)h[j];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            const int rem = sh_rem;
            const unsigned hit = __ballot_sync(kFull, incl >= rem);
            const int owner = hit ? __ffs(hit) - 1 : 31;
            if (lane == owner) {
                int acc = incl - sum, j = 0;
                for (; j < 7; ++j) {
                    if (acc + (int)h[j] >= rem) break;
                    acc += (int)h[j];
                }
                const int dg = 255 - 8 * lane - j;
                sh_rem = rem - acc;
                sh_prefix |= static_cast<unsigned long long>(dg) << shift;
                sh_bits = 64 - shift;
                if ((int)h[j] == rem - acc) sh_done = 1;
            }
        }
        __syncthreads();
    }
    const int nb = sh_bits, done = sh_done, rem0 = sh_rem;
    const uint64_t pref = top_bits(sh_prefix, nb);
    const bool keep_none = budget == 0;

    // 3. keep flags -> per-class evicted counts (first sweep), then the writes
    //    (second sweep).  Without exact key ties (`done`, or nothing kept) the keep
    //    flag is a function of the key alone: the first sweep needs one block
    //    reduction per class and the second one scan per chunk (an evicted entry's
    //    rank in its class is its index minus the kept entries before it).  With
    //    ties, both sweeps replay the same tie order with block scans.
    const bool no_ties = done || keep_none;
    auto keep_of = [&](int, int, int32_t p, float scv, int &tie) -> int {
        tie = 0;
        if (p < d.n_protect || p >= keep_from) return 1;
        if (keep_none) return 0;
        const uint64_t tb = top_bits(entry_key(scv, p), nb);
        tie = tb == pref && !done;
        return tb > pref || (tb == pref && done);
    };
    int evicted[4];
    int tie_carry = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int32_t *pc = d.pos[c] + (size_t)s * d.cap[c];
        const float *sc = d.score[c] + (size_t)s * d.cap[c];
        int ev = 0;
        if (no_ties) {
            for (int base = 0; base < n[c]; base += kPer * kThreads) {
                int32_t pv[kPer];
                float sv[kPer];
#pragma unroll
                for (int j = 0; j < kPer; ++j) {
                    const int i = base + j * kThreads + threadIdx.x;
                    pv[j] = i < n[c] ? pc[i] : INT_MIN;
                    sv[j] = i < n[c] ? sc[i] : 0.f;
                }
#pragma unroll
                for (int j = 0; j < kPer; ++j) {
                    int tie;
                    if (pv[j] != INT_MIN) ev += !keep_of(c, 0, pv[j], sv[j], tie);
                }
            }
            evicted[c] = block_sum(ev, scratch);
            continue;
        }
        for (int base = 0; base < n[c]; base += kThreads) {
            const int i = base + threadIdx.x;
            int keep = 1, tie = 0;
            if (i < n[c]) keep = keep_of(c, i, pc[i], sc[i], tie);
            int ntie;
            const int tr = block_scan(tie, &ntie, scratch) + tie_carry;
            tie_carry += ntie;
            if (tie) keep = tr < rem0;
            ev += block_sum(i < n[c] ? !keep : 0, scratch);
        }
        evicted[c] = ev;
    }
    compact_tables(d, s, n, evicted, keep_of, no_ties, rem0, scratch, move_src, move_buf);
}

}  // namespace

cudaError_t launch_evict(const Dev &d, int budget, int keep_from, cudaStream_t st, int64_t *launches) {
    evict_kernel<<<d.S, kThreads, 0, st>>>(d, budget, keep_from);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tkv
