// persist.cuh -- the parts the persistent decode-attention kernels share: the work
// split (every stream's class tables cut into class-homogeneous tiles -- 64 records for
// bf16, 128 for the code classes -- laid on one line weighted by bytes plus a fixed cost
// per tile; CTA c takes the tiles that start in the c-th equal share), the tile iterator
// and descriptor ring, the TMA producer, and the merge + score pass over the per-(stream,
// CTA) partial results.  Internal to libtkv.
#pragma once

#include <cuda.h>

#include "attn_common.cuh"

namespace tkv {
namespace attn {

constexpr int kRawBytes = 36864;      // a tile's boxes: int8 128 x (128 K + 128 V + 32 meta)
constexpr int kTileOverhead = 4096;   // cost of a tile beyond its bytes, for the work split
constexpr int kMaxStreamTable = 64;   // streams whose counts a CTA keeps in shared memory

__host__ __device__ constexpr int rows_of(int c) { return c == 0 ? 64 : 128; }
__host__ __device__ constexpr int rec_of(int c) { return c == 0 ? 512 : c == 1 ? 288 : c == 2 ? 160 : 96; }
// box layout inside a raw stage: K and V code boxes and the scale / zero box
__host__ __device__ constexpr int v_off(int c) { return c == 0 ? 16384 : c == 1 ? 16384 : c == 2 ? 8192 : 4096; }
__host__ __device__ constexpr int meta_off(int c) { return c == 1 ? 32768 : c == 2 ? 16384 : 8192; }
__host__ __device__ constexpr int code_box_bytes(int c) { return c <= 1 ? 128 : c == 2 ? 64 : 32; }

// ------------------------------------------------------------ barrier and TMA wrappers
__device__ __forceinline__ void mbar_init_n(uint32_t bar, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(n) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Non-blocking probe of phase `parity` of a barrier.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return done != 0;
}


// ------------------------------------------------------------ the work split
struct Counts {
    int n[4];
};

// tiles of class c holding n records (64-row bf16 tiles, 128-row code tiles)
__device__ __forceinline__ int ntiles(int n, int c) { return c == 0 ? (n + 63) >> 6 : (n + 127) >> 7; }
__device__ __forceinline__ unsigned long long class_cost(int n, int c) {
    return (unsigned long long)n * rec_of(c) + (unsigned long long)ntiles(n, c) * kTileOverhead;
}
__device__ __forceinline__ unsigned long long stream_cost(const Counts &k) {
    return class_cost(k.n[0], 0) + class_cost(k.n[1], 1) + class_cost(k.n[2], 2) + class_cost(k.n[3], 3);
}
__device__ __forceinline__ unsigned long long tile_cost_full(int c) {
    return (unsigned long long)rows_of(c) * rec_of(c) + kTileOverhead;
}
// floor(c * Q / NC) without overflow
__device__ __forceinline__ unsigned long long split_at(unsigned long long Q, int NC, int c) {
    if (c >= NC) return Q;
    return (Q / NC) * c + ((Q % NC) * c) / NC;
}
__device__ __forceinline__ Counts load_counts(const Dev &d, int s) {
    // counts are clamped into [0, cap] in every build (the split reads them for every
    // stream); the debug build also reports a count out of range
    const int4 v = *reinterpret_cast<const int4 *>(d.n + 4 * s);
    Counts k;
    k.n[0] = min(max(v.x, 0), d.cap[0]);
    k.n[1] = min(max(v.y, 0), d.cap[1]);
    k.n[2] = min(max(v.z, 0), d.cap[2]);
    k.n[3] = min(max(v.w, 0), d.cap[3]);
    dcheck(d.err, k.n[0] == v.x && k.n[1] == v.y && k.n[2] == v.z && k.n[3] == v.w, kDbgAttention + 0x20);
    return k;
}

struct SharedPlan {
    unsigned long long red[32];
    unsigned long long total, cstart, cend, p0;
    int s0;
    int nst;                               // streams in the table
    int cnt[kMaxStreamTable][4];
};

// One tile of the CTA's sequence.
struct Tile {
    int s;          // stream
    int c;          // class
    int e;          // first table entry of the tile within the class
    int nr;         // records in the tile
    int oc;         // entries of classes before c (offset in entry order)
    bool first;     // first tile of the stream
    bool last;      // last tile of the stream
};

// Iterator over the tiles a CTA owns.  The current stream's counts live in scalars
// (no indexed register arrays, which would go to local memory) and each step costs a
// few integer operations: the iterator runs on a single producer thread whose every
// instruction is on the tile pipeline's critical path.
__device__ __forceinline__ int pick(int c, int a0, int a1, int a2, int a3) {
    return c == 0 ? a0 : c == 1 ? a1 : c == 2 ? a2 : a3;
}
struct TileIter {
    int S, s, c, j;
    int n0, n1, n2, n3, mask;        // the stream's counts, classes holding records (bit c)
    int n, nt, oc;                   // current class: records, tiles, entries before it
    unsigned long long start, cend, cls_end, full;   // costs: current tile, share end, class end, per tile

    __device__ __forceinline__ void load(const Dev &d, const SharedPlan &pl, int stream) {
        const int i = stream - pl.s0;
        if (i >= 0 && i < pl.nst) {
            n0 = pl.cnt[i][0]; n1 = pl.cnt[i][1]; n2 = pl.cnt[i][2]; n3 = pl.cnt[i][3];
        } else {
            const Counts k = load_counts(d, stream);
            n0 = k.n[0]; n1 = k.n[1]; n2 = k.n[2]; n3 = k.n[3];
        }
        mask = (n0 > 0) | ((n1 > 0) << 1) | ((n2 > 0) << 2) | ((n3 > 0) << 3);
    }
    // enter class cc of the current stream; its region starts at cost `at`
    __device__ __forceinline__ void enter(int cc, unsigned long long at) {
        c = cc;
        n = pick(cc, n0, n1, n2, n3);
        nt = ntiles(n, cc);
        oc = pick(cc, 0, n0, n0 + n1, n0 + n1 + n2);
        full = tile_cost_full(cc);
        start = at;
        cls_end = at + class_cost(n, cc);
        j = 0;
    }
    // first class of the next stream holding records (streams without records cost 0)
    __device__ __forceinline__ void next_stream(const Dev &d, const SharedPlan &pl, unsigned long long at) {
        for (++s; s < S; ++s) {
            load(d, pl, s);
            if (mask) { enter(__ffs(mask) - 1, at); return; }
        }
        start = ~0ull;
    }
    __device__ __forceinline__ bool valid() const { return s < S && start < cend; }
    __device__ __forceinline__ void begin(const Dev &d, const SharedPlan &pl) {
        S = d.S;
        cend = pl.cend;
        s = pl.s0;
        start = ~0ull;
        if (s >= S) return;
        load(d, pl, s);
        if (!mask) { next_stream(d, pl, pl.p0); return; }
        enter(__ffs(mask) - 1, pl.p0);
        // skip the tiles of s0 that start before cstart
        while (cls_end <= pl.cstart) {
            const int rest = mask & ~((2 << c) - 1);
            if (!rest) { next_stream(d, pl, cls_end); return; }
            enter(__ffs(rest) - 1, cls_end);
        }
        if (pl.cstart > start) {
            j = (int)((pl.cstart - start + full - 1) / full);
            start += (unsigned long long)j * full;
            if (j >= nt) advance_class(d, pl);
        }
    }
    __device__ __forceinline__ void advance_class(const Dev &d, const SharedPlan &pl) {
        const int rest = mask & ~((2 << c) - 1);
        if (rest) enter(__ffs(rest) - 1, cls_end);
        else next_stream(d, pl, cls_end);
    }
    __device__ __forceinline__ void advance(const Dev &d, const SharedPlan &pl) {
        ++j;
        start += full;
        if (j >= nt) advance_class(d, pl);
    }
    __device__ __forceinline__ Tile tile() const {
        Tile t;
        t.s = s;
        t.c = c;
        t.e = j << (c == 0 ? 6 : 7);
        t.nr = min(c == 0 ? 64 : 128, n - t.e);
        t.oc = oc;
        t.first = j == 0 && c == __ffs(mask) - 1;
        t.last = j == nt - 1 && c == 31 - __clz(mask);
        return t;
    }
};

// The producer walks the tile sequence once and publishes each tile to the other roles
// through a small ring in shared memory (written before the tile's copies are issued,
// so a role that has waited for the tile's copies -- directly or through a warpgroup's
// barrier -- reads a complete descriptor).  No role lags the producer by more than a
// few tiles: the producer reuses the stage of tile k - R only after that tile's PV has
// completed, and the MMA issuer takes tiles in order, so neither warpgroup can run more
// than two tiles ahead of the other.
constexpr int kDescRing = 16;
struct __align__(16) TileDesc {
    int32_t s;       // stream
    int32_t e;       // first table entry of the tile within its class
    int32_t oc;      // entries of the classes before its class
    uint32_t meta;   // class (bits 0-1), records (bits 2-10), first / last tile of the stream
                     // (bits 11 / 12); bit 31: no more tiles
};
__device__ __forceinline__ int td_c(const TileDesc &t) { return (int)(t.meta & 3u); }
__device__ __forceinline__ int td_nr(const TileDesc &t) { return (int)((t.meta >> 2) & 511u); }
__device__ __forceinline__ bool td_first(const TileDesc &t) { return (t.meta >> 11) & 1u; }
__device__ __forceinline__ bool td_last(const TileDesc &t) { return (t.meta >> 12) & 1u; }
__device__ __forceinline__ bool td_end(const TileDesc &t) { return (t.meta >> 31) & 1u; }

// Every thread (NT of them): total cost, this CTA's share and the stream containing its start.
template <int NT>
__device__ void plan_work(const Dev &d, SharedPlan &pl, int cta, int ncta) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = NT / 32;
    unsigned long long part = 0;
    for (int s = tid; s < d.S; s += NT) part += stream_cost(load_counts(d, s));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(kFull, part, o);
    if (lane == 0) pl.red[warp] = part;
    if (tid == 0) pl.s0 = d.S;
    __syncthreads();
    if (tid == 0) {
        unsigned long long q = 0;
        for (int w = 0; w < NW; ++w) q += pl.red[w];
        pl.total = q;
        pl.cstart = split_at(q, ncta, cta);
        pl.cend = split_at(q, ncta, cta + 1);
    }
    __syncthreads();
    const unsigned long long cstart = pl.cstart;
    unsigned long long running = 0;
    for (int base = 0; base < d.S; base += NT) {
        const int s = base + tid;
        const unsigned long long cost = s < d.S ? stream_cost(load_counts(d, s)) : 0ull;
        unsigned long long incl = cost;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        __syncthreads();   // pl.red free again
        if (lane == 31) pl.red[warp] = incl;
        __syncthreads();
        unsigned long long before = running, chunk = 0;
        for (int w = 0; w < NW; ++w) {
            if (w < warp) before += pl.red[w];
            chunk += pl.red[w];
        }
        const unsigned long long excl = before + incl - cost;
        if (cost > 0 && excl <= cstart && cstart < excl + cost) {
            pl.s0 = s;
            pl.p0 = excl;
        }
        running += chunk;
        __syncthreads();
        if (pl.s0 < d.S) break;   // uniform: read after the barrier
    }
    __syncthreads();
    if (tid == 0) pl.nst = pl.s0 < d.S ? min(kMaxStreamTable, d.S - pl.s0) : 0;
    if (pl.s0 < d.S && tid < min(kMaxStreamTable, d.S - pl.s0)) {
        const Counts k = load_counts(d, pl.s0 + tid);
#pragma unroll
        for (int q = 0; q < 4; ++q) pl.cnt[tid][q] = k.n[q];
    }
    __syncthreads();
}




// ------------------------------------------------------------ the producer
// One thread: walks the CTA's tiles, publishes each descriptor in the ring and issues the
// tile's TMA boxes into stage k % R (a tail tile as 16-row boxes); after the last tile it
// publishes `nend` "no more tiles" descriptors, one for the next tile of each consumer
// group, and before returning waits for every copy still in flight.  Returns false on a
// timeout (no further copies are issued then).
template <int R>
__device__ bool produce_tiles(const Dev &d, const I8Maps &maps, const SharedPlan &pl, TileDesc *desc,
                              uint64_t *bar_full, uint64_t *bar_empty, uint32_t stage0, int nend) {
    const uint64_t pol = policy_evict_first();
    bool ok = true;
    TileIter it;
    it.begin(d, pl);
    uint32_t pending = 0;   // bit i: stage i holds a copy not yet seen consumed
    int k = 0, ncopied = 0; // tiles copied: stage i last received tile ncopied-1-((ncopied-1-i) mod R)
    for (; ok; ++k) {
        const int slot = k % R;
        if (k >= R) {
            ok = mbar_wait_sleep(smem_addr(&bar_empty[slot]), (uint32_t)((k / R - 1) & 1));
            if (!ok) break;
            pending &= ~(1u << slot);   // its previous copy was consumed
        }
        if (!it.valid()) break;
        const Tile t = it.tile();
        TileDesc td;
        td.s = t.s; td.e = t.e; td.oc = t.oc;
        td.meta = (uint32_t)t.c | ((uint32_t)t.nr << 2) | ((uint32_t)t.first << 11) | ((uint32_t)t.last << 12);
        desc[k % kDescRing] = td;
        const bool full = t.nr == rows_of(t.c);
        const int nb = full ? 1 : (t.nr + 15) >> 4;                 // 16-row boxes of a tail tile
        const int rows = full ? rows_of(t.c) : 16 * nb;
        const uint32_t bar = smem_addr(&bar_full[slot]);
        mbar_expect_tx(bar, (uint32_t)(rows * rec_of(t.c)));
        const uint32_t dst = stage0 + slot * kRawBytes;
        const int y0 = t.s * pick(t.c, d.cap[0], d.cap[1], d.cap[2], d.cap[3]) + t.e;
        const int nbox = t.c == 0 ? 4 : 3;
        const int cw = code_box_bytes(t.c);
        for (int bx = 0; bx < nbox; ++bx) {
            const bool is_meta = t.c != 0 && bx == 2;
            const int wbytes = is_meta ? 32 : cw;
            const int x = bx * cw;
            const uint32_t bdst = dst + (uint32_t)(bx * rows_of(t.c) * cw);
            const CUtensorMap *mp = &maps.m[t.c][is_meta ? 1 : 0][full ? 0 : 1];
            for (int j = 0; j < nb; ++j)
                tma_load_2d(bdst + (uint32_t)(j * 16 * wbytes), mp, x, y0 + 16 * j, bar, pol);
        }
        pending |= 1u << slot;
        ncopied = k + 1;
        it.advance(d, pl);
    }
    // "no more tiles" for the next tile of each consumer group (stage free: waited above or unused)
    if (ok) {
        for (int u = 0; u < nend; ++u) {
            const int kk = k + u, slot = kk % R;
            if (u >= 1 && kk >= R) {
                ok = mbar_wait_sleep(smem_addr(&bar_empty[slot]), (uint32_t)((kk / R - 1) & 1));
                if (!ok) break;
                pending &= ~(1u << slot);
            }
            TileDesc td;
            td.s = -1; td.e = 0; td.oc = 0; td.meta = 1u << 31;
            desc[kk % kDescRing] = td;
            mbar_arrive(smem_addr(&bar_full[slot]));
        }
    }
    // every copy still unconsumed lands before the CTA may exit (each stage holds at most one)
    for (int i = 0; i < R; ++i) {
        if (!((pending >> i) & 1u)) continue;
        const int kl = ncopied - 1 - ((ncopied - 1 - i) % R);   // >= 0: stage i received a copy
        if (!mbar_wait_sleep(smem_addr(&bar_full[i]), (uint32_t)((kl / R) & 1))) ok = false;
    }
    return ok;
}

// Prefetch of the pools' TMA descriptors (kernel parameters) into the descriptor cache.
__device__ __forceinline__ void prefetch_maps(const I8Maps &maps) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int z = 0; z < 2; ++z) asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.m[i][j][z]) : "memory");
}

// ------------------------------------------------------------ merge + score pass
// One CTA row per stream: merges the stream's partials (slots SPC (s + c) + w for the
// CTAs c of its first .. last tile and their SPC consumer groups w; empty ones have
// l = 0), writes O and the sparsity statistic, then adds p = 2^(x - M) / L to the scores
// of its slice.
template <int G, bool STATS, int SPC>
__global__ void __launch_bounds__(256, 4) attn_finalize_kernel(const __grid_constant__ Dev d, float *__restrict__ out,
                                                            float *__restrict__ sparsity,
                                                            uint8_t *__restrict__ thought, float th_r, float th_t,
                                                            int ncta) {
    constexpr int kParts = 64;   // partials staged in shared memory (more are read from global)
    __shared__ float gM[kMaxG], gInvL[kMaxG], gH[kMaxG];
    __shared__ float fac[kParts][kMaxG];
    __shared__ float hm[kParts][kMaxG], hl[kParts][kMaxG], he[kParts][kMaxG];
    grid_dependency_wait();
    const int s = blockIdx.x, split = blockIdx.y, nsplit = gridDim.y;
    const int tid = threadIdx.x;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;
    const Counts k = load_counts(d, s);
    const int o1 = k.n[0], o2 = o1 + k.n[1], o3 = o2 + k.n[2], N = o3 + k.n[3];
    float *orow = out + ((size_t)b * d.Hkv * G + (size_t)kvh * G) * kD;
    if (N == 0) {
        if (split == 0) {
            for (int i = tid; i < G * kD; i += 256) orow[i] = 0.f;
            if (STATS && tid < G) {
                if (sparsity) sparsity[(size_t)s * G + tid] = 0.f;
                if (thought) thought[(size_t)s * G + tid] = thought_of(0.f, th_r, th_t);
            }
        }
        return;
    }
    const int c_lo = d.seg_lo[s], c_hi = d.seg_hi[s];
    if (c_lo < 0 || c_hi < c_lo || c_hi >= ncta) {
        if (tid == 0 && split == 0) raise_error(d.err, kErrInvalid, (uint32_t)s);
        return;
    }
    const int nparts = SPC * (c_hi - c_lo + 1);
    const float *part0 = d.part + (size_t)SPC * (s + c_lo) * part_floats(G);
    // (m, l, e) of the first kParts partials, loaded by all threads at once
    const int nstage = min(nparts, kParts);
    for (int i = tid; i < nstage * G; i += 256) {
        const int j = i / G, h = i - j * G;
        const float *pp = part0 + (size_t)j * part_floats(G);
        hm[j][h] = pp[h];
        hl[j][h] = pp[G + h];
        if (STATS) he[j][h] = pp[2 * G + h];
    }
    __syncthreads();
    auto pm = [&](int j, int h) { return j < kParts ? hm[j][h] : part0[(size_t)j * part_floats(G) + h]; };
    auto pl_ = [&](int j, int h) { return j < kParts ? hl[j][h] : part0[(size_t)j * part_floats(G) + G + h]; };
    auto pe = [&](int j, int h) { return j < kParts ? he[j][h] : part0[(size_t)j * part_floats(G) + 2 * G + h]; };
    if (tid < G) {
        float M = kNoMax;
        for (int j = 0; j < nparts; ++j)
            if (pl_(j, tid) > 0.f) M = fmaxf(M, pm(j, tid));
        float L = 0.f, E = 0.f;
        for (int j = 0; j < nparts; ++j) {
            const float lj = pl_(j, tid), mj = pm(j, tid);
            const float f = lj > 0.f ? ex2(mj - M) : 0.f;
            if (j < kParts) fac[j][tid] = f;
            L += f * lj;
            if (STATS && lj > 0.f) E += f * (pe(j, tid) + (mj - M) * lj);
        }
        gM[tid] = M;
        gInvL[tid] = L > 0.f ? 1.f / L : 0.f;
        if (STATS) {
            gH[tid] = sparsity_of(L, E, N);
        }
    }
    __syncthreads();
    // the output: the stream's G x 128 elements spread over its nsplit CTAs, each element's
    // partials summed by sub threads (partials j, j + sub, ...; sub = the power of two that
    // leaves each thread at most 4, up to 16) and then reduced over those threads (a fixed
    // order, so the result does not depend on timing)
    {
        int sub = 1;
        while (sub < 16 && sub * 4 < nparts) sub *= 2;
        const int E = G * kD, per = (E + nsplit - 1) / nsplit;
        const int e_lo = split * per, e_hi = min(E, e_lo + per);
        const int k = tid % sub;
        for (int base = e_lo; base < e_hi; base += 256 / sub) {
            const int i = base + tid / sub;
            const int h = (i < e_hi ? i : e_lo) / kD;
            float acc = 0.f;
            if (i < e_hi) {
                for (int j = k; j < nparts; j += sub) {
                    const float *pp = part0 + (size_t)j * part_floats(G);
                    const float f = j < kParts ? fac[j][h] : (pp[G + h] > 0.f ? ex2(pp[h] - gM[h]) : 0.f);
                    if (f > 0.f) acc = fmaf(f, pp[3 * G + i], acc);
                }
            }
            for (int o = sub / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
            if (k == 0 && i < e_hi) orow[i] = acc * gInvL[h];
        }
    }
    if (split == 0) {
        if (STATS && tid < G) {
            if (sparsity) sparsity[(size_t)s * G + tid] = gH[tid];
            if (thought) thought[(size_t)s * G + tid] = thought_of(gH[tid], th_r, th_t);
        }
    }
    // scores of this CTA's slice of the stream (slices start on 32-entry boundaries)
    const int chunk = ((N + nsplit - 1) / nsplit + 31) & ~31;
    const int t0 = min(N, split * chunk), t1 = min(N, t0 + chunk);
    if (t0 < t1) add_scores<G, 256>(d, s, d.logits + (size_t)s * d.ncap * G, t0, t1, o1, o2, o3, gM, gInvL, tid);
}


// The merge + score pass after a persistent kernel of ncta CTAs with SPC partial slots
// each: one CTA per stream, more for long streams.
template <int G, bool STATS, int SPC>
cudaError_t launch_finalize(const Dev &d, float *out, float *sparsity, uint8_t *thought, float th_r, float th_t,
                            int ncta, long long live_ub, cudaStream_t st, int64_t *launches) {
    // about 2048 entries per CTA of the score pass, at most 64 CTAs per stream (four
    // resident per SM; more CTAs than one resident wave measured slower: each is bound by
    // its own latencies)
    const int nsplit = (int)(live_ub < 2048 ? 1 : live_ub >= 64ll * 2048 ? 64 : (live_ub + 2047) / 2048);
    cudaLaunchConfig_t cf = {};
    cf.gridDim = dim3((unsigned)d.S, (unsigned)nsplit, 1);
    cf.blockDim = dim3(256, 1, 1);
    cf.dynamicSmemBytes = 0;
    cf.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the launch with the kernel before
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cf.attrs = attr;
    cf.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cf, attn_finalize_kernel<G, STATS, SPC>, d, out, sparsity, thought,
                                             th_r, th_t, ncta);
    *launches += 1;
    return e;
}

}  // namespace attn
}  // namespace tkv
