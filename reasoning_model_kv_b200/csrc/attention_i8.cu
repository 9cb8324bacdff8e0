// attention_i8.cu -- tkv_decode_attention for dense record placement on the
// 5th-generation tensor cores with integer operands (tcgen05.mma kind::i8): one
// GQA decode step over the mixed-precision pools with exact integer accumulation
// of the code products, online softmax, and accumulation of each token's attention
// mass into its score (ThinKV decode over the Continuous Thinking block table;
// cumulative attention scores as on the "Back from the Future" page, problem
// statement).
//
// Two kernels.  attn_i8_kernel runs one persistent CTA per SM.  The work of the
// whole step -- every stream's class tables cut into class-homogeneous tiles
// (64 records for bf16, 112 for int8, 128 for int4 / int2) -- is laid on one line
// weighted by bytes (+ a fixed cost per tile), and CTA c takes the tiles that
// start in the c-th equal share, so every SM streams the same number of bytes
// whatever the streams' lengths and class mixes.  A stream split over several
// CTAs leaves one partial (running max m, sum l, O) per CTA; attn_finalize_kernel
// merges the partials of each stream, writes the output and adds p to the scores
// (from the raw logits the first kernel left in an L2-resident scratch).
//
// Roles inside a CTA (320 threads):
//   warp 0      producer: one bulk copy per tile into a 3-deep ring of raw stages;
//   warp 1      tensor-memory owner and MMA issuer (one thread);
//   warps 2-5   stager: thread r takes record r of the tile, puts its K and V
//               codes in head-dim order into the MMA operand layouts in shared
//               memory (int4 / int2 codes widened to one byte each), copies the
//               scale / zero block, and builds the query operands per stream;
//   warps 6-9   softmax: thread r owns row r of the tile's accumulators in tensor
//               memory (token r for QK, head dim r for PV).
//
// Math (per tile; exact integer products, no per-element dequantisation):
//   QK  q is written once per stream as three signed 8-bit digits per element,
//       q = (d0 * 2^14 + d1 * 2^7 + d2) * 2^(E_gh - 146), E_gh the exponent of the
//       largest |q| of head h in group g (exact for every bf16 within 2^12 of that
//       largest value), so for each 32-dim group g one kind::i8 MMA (A = the
//       tile's codes, u8; B = the digits, s8; M 128, K 32) gives
//       c_s = sum_d code_d * digit_s,d exactly in s32.  Thread t folds
//       x_h = sum_g kscale_g * 2^(E_gh-146) * (c0 2^14 + c1 2^7 + c2) + kzero_g * sum_g(q_h).
//   PV  W_t,(g,h) = p_h,t * vscale_g,t becomes an unsigned integer below 2^22 under a
//       per-tile power-of-two scale; its three bytes are three u8 columns, so one
//       kind::i8 MMA chain (A = V codes, MN-major, M = 128 head dims; B = W,
//       MN-major; K = the tile's tokens) gives exact s32 byte sums, which thread
//       d scales back into its fp32 O; the zero term sum_t p * vzero_g is
//       accumulated by the token threads in fp32.
//   bf16 tiles (protected tokens) use kind::f16 with bf16 operands: q exact, P
//   split into a bf16 high and low part (two columns), so nothing is narrowed.
// The running max only moves (and l, O are rescaled) when a tile exceeds it by
// more than 2^8.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "attn_common.cuh"

namespace tkv {
namespace {

using namespace attn;

constexpr int kThreads = 320;
constexpr int kRawStages = 3;
constexpr int kRawBytes = 32768;      // >= rows * record bytes of every class
constexpr int kStgBytes = 32768;      // staged K (16 KB) + V (16 KB)
constexpr int kStgV = 16384;
constexpr int kMetaBytes = 5120;      // 128 rows x 32 B of fp16 scale / zero + vmax header (4 warps x 4)
constexpr int kMetaHdr = 4096;
constexpr int kTileOverhead = 4096;   // cost of a tile beyond its bytes, for the work split
constexpr int kTmemCols = 512;
constexpr int kMaxStreamTable = 64;   // streams whose counts a CTA keeps in shared memory

__host__ __device__ constexpr int rows_of(int c) { return c == 0 ? 64 : c == 1 ? 112 : 128; }
__host__ __device__ constexpr int rec_of(int c) { return c == 0 ? 512 : c == 1 ? 288 : c == 2 ? 160 : 96; }
__host__ __device__ constexpr int ng_of(int G) { return 3 * G <= 16 ? 16 : 32; }   // QK columns per group
__host__ __device__ constexpr int gs_of(int G) { return 4 * G < 16 ? 16 : 4 * G; }  // PV columns per group
__host__ __device__ constexpr int no_of(int G) { return 4 * gs_of(G); }              // PV columns (i8 tiles)
__host__ __device__ constexpr int w_bytes(int G) { return 128 * no_of(G); }
__host__ __device__ constexpr int qi8_bytes(int G) { return 4 * 32 * ng_of(G); }
constexpr int kQbfBytes = 16 * 128 * 2;
__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int q_bytes(int G) { return align1k(qi8_bytes(G) + kQbfBytes + 2 * 4 * kMaxG * 4); }
// dynamic shared memory layout (from a 1024-byte aligned base)
constexpr int kOffRaw = 0;
constexpr int kOffStg = kOffRaw + kRawStages * kRawBytes;
constexpr int kOffMeta = kOffStg + 2 * kStgBytes;
constexpr int kOffW = kOffMeta + 2 * kMetaBytes;
__host__ __device__ constexpr int off_q(int G) { return kOffW + 2 * w_bytes(G); }
__host__ __device__ constexpr int smem_bytes(int G) { return 1024 + off_q(G) + 2 * q_bytes(G); }
// tensor memory: buffer b holds the QK accumulators at column 256b and the PV
// accumulators at column 256b + 128
__host__ __device__ constexpr uint32_t col_s(int b) { return 256u * b; }
__host__ __device__ constexpr uint32_t col_o(int b) { return 256u * b + 128u; }

// ------------------------------------------------------------ tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor without swizzle: lbo = byte stride between core
// matrices along K, sbo = along M / N (both multiples of 16).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}
// Instruction descriptor: accumulator format (1 f32, 2 s32), A / B formats (kind::i8:
// 0 u8, 1 s8; kind::f16: 1 bf16), A / B major (0 K, 1 MN), N, M = 128.
__host__ __device__ constexpr uint32_t idesc(uint32_t cfmt, uint32_t afmt, uint32_t bfmt, uint32_t amn, uint32_t bmn,
                                             uint32_t n) {
    return (cfmt << 4) | (afmt << 7) | (bfmt << 10) | (amn << 15) | (bmn << 16) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d), "l"(a), "l"(b), "r"(id),
                 "r"(acc)
                 : "memory");
}
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d), "l"(a), "l"(b), "r"(id),
                 "r"(acc)
                 : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void mbar_init_n(uint32_t bar, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

#define TKV_LD_REGS16(r) "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), \
    "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : TKV_LD_REGS16(r)
        : "r"(taddr)
        : "memory");
}
#undef TKV_LD_REGS16

// ------------------------------------------------------------ the work split
struct Counts {
    int n[4];
};

__device__ __forceinline__ int ntiles(int n, int c) { return (n + rows_of(c) - 1) / rows_of(c); }
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
    unsigned long long red[kThreads / 32];
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

// Iterator over the tiles a CTA owns (the same sequence in every role).
struct TileIter {
    int s, c, j;
    Counts k;
    unsigned long long sbase, cbase, start, cend;
    int S;

    __device__ __forceinline__ void load(const Dev &d, const SharedPlan &pl, int stream) {
        const int i = stream - pl.s0;
        if (i >= 0 && i < pl.nst) {
#pragma unroll
            for (int q = 0; q < 4; ++q) k.n[q] = pl.cnt[i][q];
        } else {
            k = load_counts(d, stream);
        }
    }
    // first class >= c0 with entries, 4 if none; cbase advanced over skipped classes
    __device__ __forceinline__ int next_class(int c0) {
        int cc = c0;
        while (cc < 4 && k.n[cc] == 0) ++cc;
        return cc;
    }
    __device__ __forceinline__ bool valid() const { return s < S && start < cend; }
    __device__ __forceinline__ void settle(const Dev &d, const SharedPlan &pl) {
        // move to the next tile that exists (possibly in a later stream)
        while (s < S) {
            if (c < 4 && j < ntiles(k.n[c], c)) {
                start = cbase + (unsigned long long)j * tile_cost_full(c);
                return;
            }
            if (c < 4) {
                cbase += class_cost(k.n[c], c);
                c = next_class(c + 1);
                j = 0;
                continue;
            }
            sbase += stream_cost(k);
            ++s;
            if (s >= S) break;
            load(d, pl, s);
            c = next_class(0);
            cbase = sbase;
            j = 0;
        }
        start = ~0ull;
    }
    __device__ __forceinline__ void begin(const Dev &d, const SharedPlan &pl) {
        S = d.S;
        cend = pl.cend;
        s = pl.s0;
        if (s >= S) { start = ~0ull; return; }
        load(d, pl, s);
        sbase = pl.p0;
        cbase = sbase;
        c = next_class(0);
        j = 0;
        // skip the tiles of s0 that start before cstart
        while (c < 4) {
            const unsigned long long span = class_cost(k.n[c], c);
            if (cbase + span <= pl.cstart) {
                cbase += span;
                c = next_class(c + 1);
                continue;
            }
            const unsigned long long full = tile_cost_full(c);
            j = pl.cstart > cbase ? (int)((pl.cstart - cbase + full - 1) / full) : 0;
            break;
        }
        settle(d, pl);
    }
    __device__ __forceinline__ void advance(const Dev &d, const SharedPlan &pl) {
        ++j;
        settle(d, pl);
    }
    __device__ __forceinline__ Tile tile() const {
        Tile t;
        t.s = s;
        t.c = c;
        t.e = j * rows_of(c);
        t.nr = min(rows_of(c), k.n[c] - t.e);
        t.oc = 0;
        for (int q = 0; q < c; ++q) t.oc += k.n[q];
        int cf = 0;
        while (cf < 4 && k.n[cf] == 0) ++cf;
        int cl = 3;
        while (cl >= 0 && k.n[cl] == 0) --cl;
        t.first = (c == cf && j == 0);
        t.last = (c == cl && j == ntiles(k.n[c], c) - 1);
        return t;
    }
};

// The producer walks the tile sequence once and publishes each tile to the other roles
// through a small ring in shared memory (written before the tile's copy is issued, so
// a role that has waited for the tile's copy -- directly or through the stager's
// barriers -- reads a complete descriptor).  No role lags the producer by more than
// kDescRing - 4 tiles: the producer needs the raw stage of tile k - 3, which the stager
// releases only after staging it, which needs tile k - 5's PV complete, which needs its
// softmax done.
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

// Every thread: total cost, this CTA's share and the stream containing its start.
__device__ void plan_work(const Dev &d, SharedPlan &pl, int cta, int ncta) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kThreads / 32;
    unsigned long long part = 0;
    for (int s = tid; s < d.S; s += kThreads) part += stream_cost(load_counts(d, s));
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
    for (int base = 0; base < d.S; base += kThreads) {
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

// ------------------------------------------------------------ staging (code order)
// Head-dim ("natural") order for the MMA operands.  Word layouts of the records:
// see stored_dim in append.cu.  Each function writes the 16-byte chunk kc of the
// row's natural-order codes as 4 words (K: K-major rows; V: MN-major columns --
// the same byte formula for both: chunk kc at kc*2048 + (r/8)*128 + (r%8)*16).

__device__ __forceinline__ void sts128(uint8_t *p, uint32_t a, uint32_t b, uint32_t c, uint32_t dd) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, dd);
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) { return __byte_perm(a, b, sel); }

// int8: K word (q, w) holds dims base + {0, 2, 1, 3}, base = 32(w/2) + 8q + 4(w%2);
// V word (q, w) holds dims 16w + 2q + {0, 8, 1, 9}.
__device__ __forceinline__ void stage_row_i8(const uint8_t *rec, uint8_t *k_dst, uint8_t *v_dst) {
    uint32_t kw[4][8], vw[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 a = *reinterpret_cast<const uint4 *>(rec + 32 * q);
        const uint4 b = *reinterpret_cast<const uint4 *>(rec + 32 * q + 16);
        kw[q][0] = a.x; kw[q][1] = a.y; kw[q][2] = a.z; kw[q][3] = a.w;
        kw[q][4] = b.x; kw[q][5] = b.y; kw[q][6] = b.z; kw[q][7] = b.w;
        const uint4 c = *reinterpret_cast<const uint4 *>(rec + 128 + 32 * q);
        const uint4 e = *reinterpret_cast<const uint4 *>(rec + 128 + 32 * q + 16);
        vw[q][0] = c.x; vw[q][1] = c.y; vw[q][2] = c.z; vw[q][3] = c.w;
        vw[q][4] = e.x; vw[q][5] = e.y; vw[q][6] = e.z; vw[q][7] = e.w;
    }
    // K chunk kc = 2(w/2) + q/2, position 2(q%2) + w%2
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
        const int w0 = 2 * (kc / 2), q0 = 2 * (kc % 2);
        sts128(k_dst + kc * 2048, prmt(kw[q0][w0], 0, 0x3120), prmt(kw[q0][w0 + 1], 0, 0x3120),
               prmt(kw[q0 + 1][w0], 0, 0x3120), prmt(kw[q0 + 1][w0 + 1], 0, 0x3120));
    }
    // V chunk w: [p(0,1,0x6420), p(2,3,0x6420), p(0,1,0x7531), p(2,3,0x7531)]
#pragma unroll
    for (int w = 0; w < 8; ++w)
        sts128(v_dst + w * 2048, prmt(vw[0][w], vw[1][w], 0x6420), prmt(vw[2][w], vw[3][w], 0x6420),
               prmt(vw[0][w], vw[1][w], 0x7531), prmt(vw[2][w], vw[3][w], 0x7531));
}

// int4: K word (q, w) = group w, dims 32w + 8q + {0..7}, nibble e at offset
// 2(e%4) + e/4; V word (q, w) nibble e = dim 32w + 8(e%4) + 2q + e/4.
__device__ __forceinline__ void stage_row_i4(const uint8_t *rec, uint8_t *k_dst, uint8_t *v_dst) {
    uint32_t kw[4][4], vw[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 a = *reinterpret_cast<const uint4 *>(rec + 16 * q);
        kw[q][0] = a.x; kw[q][1] = a.y; kw[q][2] = a.z; kw[q][3] = a.w;
        const uint4 b = *reinterpret_cast<const uint4 *>(rec + 64 + 16 * q);
        vw[q][0] = b.x; vw[q][1] = b.y; vw[q][2] = b.z; vw[q][3] = b.w;
    }
    // K: natural words 8w + 2q + {0,1} = (prmt(lo,hi,0x6420), prmt(lo,hi,0x7531)); chunk 2w + q/2
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t nat[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t lo = kw[q][w] & 0x0F0F0F0Fu, hi = (kw[q][w] >> 4) & 0x0F0F0F0Fu;
            nat[2 * q] = prmt(lo, hi, 0x6420);
            nat[2 * q + 1] = prmt(lo, hi, 0x7531);
        }
        sts128(k_dst + (2 * w) * 2048, nat[0], nat[1], nat[2], nat[3]);
        sts128(k_dst + (2 * w + 1) * 2048, nat[4], nat[5], nat[6], nat[7]);
    }
    // V: natural word 8w + 2m + r from A = (2r, w), B = (2r+1, w); chunk 2w + m/2,
    // position 2(m%2) + r
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t nat[8];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t alo = vw[2 * r][w] & 0x0F0F0F0Fu, ahi = (vw[2 * r][w] >> 4) & 0x0F0F0F0Fu;
            const uint32_t blo = vw[2 * r + 1][w] & 0x0F0F0F0Fu, bhi = (vw[2 * r + 1][w] >> 4) & 0x0F0F0F0Fu;
            nat[2 * 0 + r] = prmt(alo, blo, 0x6420);   // m = 0
            nat[2 * 1 + r] = prmt(ahi, bhi, 0x6420);   // m = 1
            nat[2 * 2 + r] = prmt(alo, blo, 0x7531);   // m = 2
            nat[2 * 3 + r] = prmt(ahi, bhi, 0x7531);   // m = 3
        }
        sts128(v_dst + (2 * w) * 2048, nat[0], nat[1], nat[2], nat[3]);
        sts128(v_dst + (2 * w + 1) * 2048, nat[4], nat[5], nat[6], nat[7]);
    }
}

// int2: K word (q, w) field e = dim 32(2w + (e%8)/4) + 8q + 2(e%4) + e/8;
// V word (q, w) field e = dim 64w + 8(e%8) + 2q + e/8.
__device__ __forceinline__ void stage_row_i2(const uint8_t *rec, uint8_t *k_dst, uint8_t *v_dst) {
    uint32_t kw[4][2], vw[4][2];
    {
        const uint4 a = *reinterpret_cast<const uint4 *>(rec);
        const uint4 b = *reinterpret_cast<const uint4 *>(rec + 16);
        kw[0][0] = a.x; kw[0][1] = a.y; kw[1][0] = a.z; kw[1][1] = a.w;
        kw[2][0] = b.x; kw[2][1] = b.y; kw[3][0] = b.z; kw[3][1] = b.w;
        const uint4 c = *reinterpret_cast<const uint4 *>(rec + 32);
        const uint4 e = *reinterpret_cast<const uint4 *>(rec + 48);
        vw[0][0] = c.x; vw[0][1] = c.y; vw[1][0] = c.z; vw[1][1] = c.w;
        vw[2][0] = e.x; vw[2][1] = e.y; vw[3][0] = e.z; vw[3][1] = e.w;
    }
    // K: group 2w + gg, dims 8q + {0..3} = prmt(e0, e1, sel(gg)), 8q + {4..7} = prmt(e2, e3, sel(gg));
    // natural word 16w + 8gg + 2q + {0,1}: chunk 4w + 2gg + q/2, position 2(q%2) + {0,1}
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        uint32_t nat[2][8];   // [gg][2q + half]
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t x = kw[q][w];
            const uint32_t e0 = x & 0x03030303u, e1 = (x >> 2) & 0x03030303u;
            const uint32_t e2 = (x >> 4) & 0x03030303u, e3 = (x >> 6) & 0x03030303u;
            nat[0][2 * q] = prmt(e0, e1, 0x6420);
            nat[0][2 * q + 1] = prmt(e2, e3, 0x6420);
            nat[1][2 * q] = prmt(e0, e1, 0x7531);
            nat[1][2 * q + 1] = prmt(e2, e3, 0x7531);
        }
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            sts128(k_dst + (4 * w + 2 * gg) * 2048, nat[gg][0], nat[gg][1], nat[gg][2], nat[gg][3]);
            sts128(k_dst + (4 * w + 2 * gg + 1) * 2048, nat[gg][4], nat[gg][5], nat[gg][6], nat[gg][7]);
        }
    }
    // V: natural word 16w + 2m + r = prmt(A.e_{m%4}, B.e_{m%4}, m/4 ? 0x7531 : 0x6420), A = (2r, w),
    // B = (2r+1, w); chunk 4w + m/2, position 2(m%2) + r
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        uint32_t nat[16];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t A = vw[2 * r][w], Bw = vw[2 * r + 1][w];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t ea = (A >> (2 * kk)) & 0x03030303u, eb = (Bw >> (2 * kk)) & 0x03030303u;
                nat[2 * kk + r] = prmt(ea, eb, 0x6420);         // m = kk
                nat[2 * (kk + 4) + r] = prmt(ea, eb, 0x7531);   // m = kk + 4
            }
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
            sts128(v_dst + (4 * w + ch) * 2048, nat[4 * ch], nat[4 * ch + 1], nat[4 * ch + 2], nat[4 * ch + 3]);
    }
}

// bf16: K word (q, w) = dims 32(w/4) + 8q + 2(w%4) + {0,1}: chunk kc (dims 8kc..8kc+7)
// is the 16 bytes at 64(kc%4) + 16(kc/4); V word (q, w) = dims 8w + 2q + {0,1}: chunk
// kc = words (q, kc) for q = 0..3.  Layout: chunk kc at kc*1024 + (r/8)*128 + (r%8)*16.
__device__ __forceinline__ void stage_row_bf16(const uint8_t *rec, uint8_t *dst, bool is_v, int rot) {
    // rows are 512 bytes apart, so every row starts on the same bank: each thread walks
    // the chunks from a different starting chunk (rot = row) to spread a phase's loads
    if (!is_v) {
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
            const int kc = (i + rot) & 15;
            *reinterpret_cast<uint4 *>(dst + kc * 1024) =
                *reinterpret_cast<const uint4 *>(rec + 64 * (kc % 4) + 16 * (kc / 4));
        }
    } else {
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
            const int kc = (i + rot) & 15;
            const uint32_t *src = reinterpret_cast<const uint32_t *>(rec + 256 + 4 * kc);
            sts128(dst + kc * 1024, src[0], src[16], src[32], src[48]);
        }
    }
}

__device__ __forceinline__ void zero_row(uint8_t *dst, int nchunks, int stride) {
    for (int i = 0; i < nchunks; ++i) *reinterpret_cast<uint4 *>(dst + i * stride) = make_uint4(0u, 0u, 0u, 0u);
}

// Order-preserving uint32 image of a float (for max reductions with redux).
__device__ __forceinline__ uint32_t fkey(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_inv(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// 2^-ceil(log2 x) for x > 0 (a power of two), with e_out = ceil(log2 x)
__device__ __forceinline__ float inv_pow2_ceil(float x, int &e_out) {
    const uint32_t u = __float_as_uint(x);
    const int be = (int)((u >> 23) & 0xff);
    const int e = be - 127 + ((u & 0x7fffff) != 0 ? 1 : 0);
    e_out = e;
    return __uint_as_float((uint32_t)(127 - e) << 23);
}
__device__ __forceinline__ float pow2f(int e) {   // 2^e for -126 <= e <= 127
    return __uint_as_float((uint32_t)(e + 127) << 23);
}
__device__ __forceinline__ float i2f_exact(int32_t c) { return __int2float_rn(c); }

template <int G>
struct QConst {   // per-stream constants of the query operand, in shared memory
    float a[4][kMaxG];      // 2^(E_gh - 146): weight of one unit of the digit combination
    float qsum[4][kMaxG];   // sum over group g of head h's (digit-exact) query
};

// ------------------------------------------------------------ the attention kernel
template <int G, bool STATS>
__global__ void __launch_bounds__(kThreads, 1)
    attn_i8_kernel(const __grid_constant__ Dev d, const __nv_bfloat16 *__restrict__ q, float xscale) {
    constexpr int NG = ng_of(G);
    constexpr int NO = no_of(G);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_raw_full[kRawStages], bar_raw_empty[kRawStages];
    __shared__ __align__(8) uint64_t bar_stg_full[2], bar_stg_empty[2], bar_meta_full[2], bar_meta_empty[2];
    __shared__ __align__(8) uint64_t bar_s_full[2], bar_w_full[2], bar_o_full[2];
    __shared__ uint32_t tmem_base;
    __shared__ SharedPlan pl;
    __shared__ uint32_t xred[2][4][kMaxG];      // tile max keys per softmax warp (double-buffered)
    __shared__ float fred[4][6 * kMaxG];        // segment flush reductions
    __shared__ float zsum[4][kMaxG];            // reduced zero-term sums of the segment being flushed
    __shared__ uint32_t err_timeout;
    __shared__ TileDesc desc[kDescRing];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x, ncta = gridDim.x;

    // ---- set-up (independent of the append, so before the dependency wait)
    if (warp == 1) tmem_alloc(smem_addr(&tmem_base), kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < kRawStages; ++i) {
            mbar_init_n(smem_addr(&bar_raw_full[i]), 1);
            mbar_init_n(smem_addr(&bar_raw_empty[i]), 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init_n(smem_addr(&bar_stg_full[i]), 4);
            mbar_init_n(smem_addr(&bar_stg_empty[i]), 1);
            mbar_init_n(smem_addr(&bar_meta_full[i]), 4);
            mbar_init_n(smem_addr(&bar_meta_empty[i]), 4);
            mbar_init_n(smem_addr(&bar_s_full[i]), 1);
            mbar_init_n(smem_addr(&bar_w_full[i]), 4);
            mbar_init_n(smem_addr(&bar_o_full[i]), 1);
        }
        err_timeout = 0;
        mbar_init_fence();
    }
    // query operand buffers: padding rows and columns stay zero
    for (int i = tid; i < 2 * q_bytes(G) / 16; i += kThreads)
        reinterpret_cast<uint4 *>(sm + off_q(G))[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base;

    grid_dependency_wait();   // the append's counters and records are visible from here
    plan_work(d, pl, cta, ncta);

    bool ok = true;
    const uint32_t smb = smem_addr(sm);

    if (warp == 0) {
        // ================================================= producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            TileIter it;
            it.begin(d, pl);
            int k = 0;
            for (;; ++k) {
                const int slot = k % kRawStages;
                if (k >= kRawStages && ok)
                    ok = mbar_wait_sleep(smem_addr(&bar_raw_empty[slot]), (uint32_t)((k / kRawStages - 1) & 1));
                const uint32_t bar = smem_addr(&bar_raw_full[slot]);
                if (!it.valid()) {
                    TileDesc td;
                    td.s = -1; td.e = 0; td.oc = 0; td.meta = 1u << 31;
                    desc[k % kDescRing] = td;
                    mbar_arrive(bar);   // completes the stage's phase without a copy: "no more tiles"
                    break;
                }
                const Tile t = it.tile();
                TileDesc td;
                td.s = t.s; td.e = t.e; td.oc = t.oc;
                td.meta = (uint32_t)t.c | ((uint32_t)t.nr << 2) | ((uint32_t)t.first << 11) | ((uint32_t)t.last << 12);
                desc[k % kDescRing] = td;
                const uint32_t bytes = (uint32_t)(t.nr * rec_of(t.c));
                const uint8_t *src = d.pool[t.c] + ((size_t)t.s * d.cap[t.c] + t.e) * rec_of(t.c);
                mbar_expect_tx(bar, bytes);
                bulk_copy(smb + kOffRaw + slot * kRawBytes, src, bytes, bar, pol);
                it.advance(d, pl);
            }
            // every copy this CTA issued (tiles 0 .. k-1) has landed before the CTA may exit;
            // the stage of tile k ended with the "no more tiles" arrival
            for (int i = 0; i < kRawStages; ++i) {
                if (k < 1 || i == k % kRawStages) continue;
                const int kl = k - 1 - ((k - 1 - i) % kRawStages);   // last tile copied into stage i
                if (kl < 0) continue;
                if (!mbar_wait_sleep(smem_addr(&bar_raw_full[i]), (uint32_t)((kl / kRawStages) & 1))) ok = false;
            }
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            int k = 0, prev_c = -1, seg = -1, prev_s = -1;
            auto issue_pv = [&](int kp, int cp) {
                const int b = kp & 1;
                if (ok) ok = mbar_wait_sleep(smem_addr(&bar_w_full[b]), (uint32_t)((kp >> 1) & 1));
                tc_fence_after();
                const uint32_t av = smb + kOffStg + b * kStgBytes + kStgV;
                const uint32_t bw = smb + kOffW + b * w_bytes(G);
                if (cp == 0) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16(tb + col_o(b), sdesc(av + ks * 256, 128, 1024), sdesc(bw + ks * 256, 128, 1024),
                                idesc(1, 1, 1, 1, 1, 16), ks > 0);
                } else {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_i8(tb + col_o(b), sdesc(av + ks * 512, 128, 2048), sdesc(bw + ks * 512, 128, 2048),
                               idesc(2, 0, 0, 1, 1, NO), ks > 0);
                }
                mma_commit(smem_addr(&bar_o_full[b]));
                mma_commit(smem_addr(&bar_stg_empty[b]));
            };
            for (;; ++k) {
                const int b = k & 1;
                if (ok) ok = mbar_wait_sleep(smem_addr(&bar_stg_full[b]), (uint32_t)((k >> 1) & 1));
                const TileDesc td = desc[k % kDescRing];
                if (td_end(td)) break;
                const int tc = td_c(td);
                if (td.s != prev_s) { ++seg; prev_s = td.s; }
                tc_fence_after();
                const uint32_t ak = smb + kOffStg + b * kStgBytes;
                const uint32_t qb = smb + off_q(G) + (seg & 1) * q_bytes(G);
                if (tc == 0) {
                    const uint32_t bq = qb + qi8_bytes(G);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_f16(tb + col_s(b), sdesc(ak + ks * 2048, 1024, 128), sdesc(bq + ks * 512, 256, 128),
                                idesc(1, 1, 1, 0, 0, 16), ks > 0);
                } else {
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        mma_i8(tb + col_s(b) + g * NG, sdesc(ak + 2 * g * 2048, 2048, 128),
                               sdesc(qb + g * 32 * NG, NG * 16, 128), idesc(2, 0, 1, 0, 0, NG), 0u);
                }
                mma_commit(smem_addr(&bar_s_full[b]));
                if (k > 0) issue_pv(k - 1, prev_c);
                prev_c = tc;
            }
            if (k > 0) issue_pv(k - 1, prev_c);
        }
    } else if (warp < 6) {
        // ================================================= stager
        const int r = tid - 64;            // row of the tile, also head dim for the query operand
        const int sw = warp - 2;           // stager warp = query group it builds
        int k = 0, seg = -1, prev_s = -1;
        for (;; ++k) {
            const int b = k & 1, slot = k % kRawStages;
            if (k >= 2) {
                if (ok) ok = mbar_wait_sleep(smem_addr(&bar_stg_empty[b]), (uint32_t)(((k - 2) >> 1) & 1));
                if (ok) ok = mbar_wait_sleep(smem_addr(&bar_meta_empty[b]), (uint32_t)(((k - 2) >> 1) & 1));
            }
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_raw_full[slot]), (uint32_t)((k / kRawStages) & 1));
            const TileDesc td = desc[k % kDescRing];
            if (td_end(td)) {
                // pass "no more tiles" on to the MMA issuer and the softmax warps
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_addr(&bar_stg_full[b]));
                    mbar_arrive(smem_addr(&bar_meta_full[b]));
                }
                break;
            }
            Tile t;
            t.s = td.s; t.c = td_c(td); t.e = td.e; t.nr = td_nr(td); t.oc = td.oc;
            t.first = td_first(td); t.last = td_last(td);
            if (t.s != prev_s) {
                // ---- query operands of stream t.s: thread r takes head dim r
                ++seg;
                prev_s = t.s;
                uint8_t *qbuf = sm + off_q(G) + (seg & 1) * q_bytes(G);
                QConst<G> *qc = reinterpret_cast<QConst<G> *>(qbuf + qi8_bytes(G) + kQbfBytes);
                const int bb = t.s / d.Hkv, kvh = t.s - bb * d.Hkv;
                const uint16_t *qrow =
                    reinterpret_cast<const uint16_t *>(q) + ((size_t)bb * d.Hkv * G + (size_t)kvh * G) * kD;
                const int g = sw, kk = r & 31;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const uint32_t bits = qrow[h * kD + r];
                    // bf16 operand: element (n = h, k = r), K-major
                    *reinterpret_cast<uint16_t *>(qbuf + qi8_bytes(G) + (r / 8) * 256 + (h / 8) * 128 + (h % 8) * 16 +
                                                  (r % 8) * 2) = (uint16_t)bits;
                    // digits: q = v * 2^(Emax - 146) with v = m * 2^(e - Emax + 12) (rounded)
                    const int ex = (int)((bits >> 7) & 0xff);
                    const int m = ex == 0 ? (int)(bits & 0x7f) : (int)((bits & 0x7f) | 0x80);
                    const int e_eff = ex == 0 ? 1 : ex;
                    const int emax = (int)__reduce_max_sync(kFull, (unsigned)e_eff);
                    const int sh = e_eff - emax + 12;
                    int v;
                    if (sh >= 0) v = m << sh;
                    else if (sh > -9) v = (m + (1 << (-sh - 1))) >> (-sh);
                    else v = 0;
                    if (bits & 0x8000) v = -v;
                    const int d2 = ((v + 64) & 127) - 64;
                    const int v1 = (v - d2) >> 7;
                    const int d1 = ((v1 + 64) & 127) - 64;
                    const int d0 = (v1 - d1) >> 7;
                    uint8_t *gb = qbuf + g * 32 * NG;
                    const int n0 = 0 * G + h, n1 = 1 * G + h, n2 = 2 * G + h;
                    const int ko = (kk / 16) * (NG * 16) + kk % 16;
                    gb[ko + (n0 / 8) * 128 + (n0 % 8) * 16] = (uint8_t)(int8_t)d0;
                    gb[ko + (n1 / 8) * 128 + (n1 % 8) * 16] = (uint8_t)(int8_t)d1;
                    gb[ko + (n2 / 8) * 128 + (n2 % 8) * 16] = (uint8_t)(int8_t)d2;
                    const int vsum = __reduce_add_sync(kFull, v);
                    if (lane == 0) {
                        const int ea = emax - 146;
                        const float a = ea >= -126 ? pow2f(ea) : pow2f(ea + 64) * 5.421010862427522e-20f;   // 2^-64
                        qc->a[g][h] = a;
                        qc->qsum[g][h] = (float)vsum * a;
                    }
                }
            }
            // ---- the tile
            const uint8_t *raw = sm + kOffRaw + slot * kRawBytes;
            uint8_t *stg = sm + kOffStg + b * kStgBytes;
            uint8_t *meta = sm + kOffMeta + b * kMetaBytes;
            const int R = rec_of(t.c);
            if (t.c == 0) {
                // 64 rows: threads 0..63 take K, 64..127 take V of row r % 64
                const int rr = r & 63;
                const bool is_v = r >= 64;
                uint8_t *dst = stg + (is_v ? kStgV : 0) + (rr / 8) * 128 + (rr % 8) * 16;
                if (rr < t.nr) stage_row_bf16(raw + rr * R, dst, is_v, rr);
                else zero_row(dst, 16, 1024);
            } else {
                uint8_t *kd = stg + (r / 8) * 128 + (r % 8) * 16;
                uint8_t *vd = kd + kStgV;
                uint32_t vkey[4] = {0u, 0u, 0u, 0u};
                if (r < t.nr) {
                    const uint8_t *rec = raw + r * R;
                    if (t.c == 1) stage_row_i8(rec, kd, vd);
                    else if (t.c == 2) stage_row_i4(rec, kd, vd);
                    else stage_row_i2(rec, kd, vd);
                    const int cb = R == 288 ? 128 : R == 160 ? 64 : 32;
                    const uint4 km = *reinterpret_cast<const uint4 *>(rec + 2 * cb);
                    const uint4 vm = *reinterpret_cast<const uint4 *>(rec + 2 * cb + 16);
                    *reinterpret_cast<uint4 *>(meta + r * 32) = km;
                    *reinterpret_cast<uint4 *>(meta + r * 32 + 16) = vm;
                    // v scales are >= 0: their fp16 bits order as integers
                    vkey[0] = vm.x & 0xffffu; vkey[1] = vm.x >> 16; vkey[2] = vm.y & 0xffffu; vkey[3] = vm.y >> 16;
                } else {
                    zero_row(kd, 8, 2048);
                    zero_row(vd, 8, 2048);
                    *reinterpret_cast<uint4 *>(meta + r * 32) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(meta + r * 32 + 16) = make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t mx = __reduce_max_sync(kFull, vkey[g]);
                    if (lane == 0) reinterpret_cast<uint32_t *>(meta + kMetaHdr)[sw * 4 + g] = mx;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_addr(&bar_stg_full[b]));
                mbar_arrive(smem_addr(&bar_meta_full[b]));
                mbar_arrive(smem_addr(&bar_raw_empty[slot]));
            }
        }
    } else {
        // ================================================= softmax / epilogue
        const int wq = warp & 3;                 // lane quarter of tensor memory
        const int r = 32 * wq + lane;            // token row (QK) and head dim (PV)
        const int gr = r >> 5;                   // group of head dim r
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        float m[G], l[G], e[G], z[4][G], oacc[G];
        float alpha_prev[G], bp_prev[G], bv_prev = 1.f;
        int c_prev = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = kNoMax; l[h] = 0.f; e[h] = 0.f; oacc[h] = 0.f; alpha_prev[h] = 1.f; bp_prev[h] = 1.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) z[g][h] = 0.f;
        }
        int k = 0, seg = -1, prev_s = -1;
        Tile tp;                                 // previous tile
        tp.s = -1; tp.first = false; tp.last = false;
        int seg_first_cta_tile = 0;              // the current segment began with the stream's first tile

        // reduce the per-thread partial sums of the softmax warps; thread 0..: write the
        // segment's (m, l, e) and keep the zero-term sums in shared memory
        auto flush_softmax_side = [&](int s_old, bool first_flag) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float vl = l[h], ve = e[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    vl += __shfl_xor_sync(kFull, vl, o);
                    if (STATS) ve += __shfl_xor_sync(kFull, ve, o);
                }
                if (lane == 0) { fred[wq][h] = vl; fred[wq][G + h] = ve; }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float vz = z[g][h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) vz += __shfl_xor_sync(kFull, vz, o);
                    if (lane == 0) fred[wq][2 * G + g * G + h] = vz;
                }
            }
            named_sync(1, 128);
            float *part = d.part + (size_t)(s_old + cta) * part_floats(G);
            if (r < 6 * G) {
                const float v = fred[0][r] + fred[1][r] + fred[2][r] + fred[3][r];
                if (r < G) part[G + r] = v;                        // l
                else if (r < 2 * G) part[2 * G + (r - G)] = v;     // e
                else zsum[(r - 2 * G) / G][(r - 2 * G) % G] = v;   // zero term
            }
            if (r == 0) {
#pragma unroll
                for (int h = 0; h < G; ++h) part[h] = m[h];
                if (first_flag) d.seg_lo[s_old] = cta;
            }
            named_sync(1, 128);
        };
        auto flush_o_side = [&](int s_old, bool last_flag) {
            float *part = d.part + (size_t)(s_old + cta) * part_floats(G);
#pragma unroll
            for (int h = 0; h < G; ++h) part[3 * G + h * kD + r] = oacc[h] + zsum[gr][h];
            if (r == 0 && last_flag) d.seg_hi[s_old] = cta;
        };
        // add the PV result of own tile kp (class cp) to O
        auto o_accumulate = [&](int kp, int cp) {
            const int b = kp & 1;
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_o_full[b]), (uint32_t)((kp >> 1) & 1));
            tc_fence_after();
            if (cp == 0) {
                uint32_t dv[16];
                tmem_ld16(tb + lane_off + col_o(b), dv);
                tc_wait_ld();
#pragma unroll
                for (int h = 0; h < G; ++h)
                    oacc[h] = fmaf(oacc[h], alpha_prev[h], __uint_as_float(dv[h]) + __uint_as_float(dv[G + h]));
            } else {
                uint32_t dv[gs_of(G)];
#pragma unroll
                for (int i = 0; i < gs_of(G); i += 16) tmem_ld16(tb + lane_off + col_o(b) + gr * gs_of(G) + i, dv + i);
                tc_wait_ld();
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float v = fmaf(i2f_exact((int32_t)dv[4 * h + 2]), 65536.f,
                                         fmaf(i2f_exact((int32_t)dv[4 * h + 1]), 256.f,
                                              i2f_exact((int32_t)dv[4 * h])));
                    oacc[h] = fmaf(oacc[h], alpha_prev[h], v * bp_prev[h] * bv_prev);
                }
            }
            tc_fence_before();
        };

        float *lgs_base = d.logits;
        for (;; ++k) {
            const int b = k & 1;
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_meta_full[b]), (uint32_t)((k >> 1) & 1));
            const TileDesc td = desc[k % kDescRing];
            if (td_end(td)) break;
            Tile t;
            t.s = td.s; t.c = td_c(td); t.e = td.e; t.nr = td_nr(td); t.oc = td.oc;
            t.first = td_first(td); t.last = td_last(td);
            const bool newseg = t.s != prev_s;
            if (newseg && k > 0) flush_softmax_side(prev_s, seg_first_cta_tile != 0);
            if (newseg) {
                ++seg;
                prev_s = t.s;
                seg_first_cta_tile = t.first ? 1 : 0;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    m[h] = kNoMax; l[h] = 0.f; e[h] = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) z[g][h] = 0.f;
                }
            }
            const QConst<G> *qc =
                reinterpret_cast<const QConst<G> *>(sm + off_q(G) + (seg & 1) * q_bytes(G) + qi8_bytes(G) + kQbfBytes);
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_s_full[b]), (uint32_t)((k >> 1) & 1));
            tc_fence_after();
            const bool valid = r < t.nr;
            float x[G];
            float vsc[4] = {0.f, 0.f, 0.f, 0.f}, vze[4] = {0.f, 0.f, 0.f, 0.f};
            if (t.c == 0) {
                uint32_t sv[16];
                tmem_ld16(tb + lane_off + col_s(b), sv);
                tc_wait_ld();
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = valid ? __uint_as_float(sv[h]) * xscale : -INFINITY;
            } else {
                const uint8_t *meta = sm + kOffMeta + b * kMetaBytes;
                const uint4 km = *reinterpret_cast<const uint4 *>(meta + r * 32);
                const uint4 vm = *reinterpret_cast<const uint4 *>(meta + r * 32 + 16);
                const float2 ks01 = __half22float2(u32_as_h2(km.x)), ks23 = __half22float2(u32_as_h2(km.y));
                const float2 kz01 = __half22float2(u32_as_h2(km.z)), kz23 = __half22float2(u32_as_h2(km.w));
                const float2 vs01 = __half22float2(u32_as_h2(vm.x)), vs23 = __half22float2(u32_as_h2(vm.y));
                const float2 vz01 = __half22float2(u32_as_h2(vm.z)), vz23 = __half22float2(u32_as_h2(vm.w));
                const float ks[4] = {ks01.x, ks01.y, ks23.x, ks23.y}, kz[4] = {kz01.x, kz01.y, kz23.x, kz23.y};
                vsc[0] = vs01.x; vsc[1] = vs01.y; vsc[2] = vs23.x; vsc[3] = vs23.y;
                vze[0] = vz01.x; vze[1] = vz01.y; vze[2] = vz23.x; vze[3] = vz23.y;
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = 0.f;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t sv[NG];
#pragma unroll
                    for (int i = 0; i < NG; i += 16) tmem_ld16(tb + lane_off + col_s(b) + g * NG + i, sv + i);
                    tc_wait_ld();
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float tsum = fmaf(i2f_exact((int32_t)sv[h]), 16384.f,
                                                fmaf(i2f_exact((int32_t)sv[G + h]), 128.f,
                                                     i2f_exact((int32_t)sv[2 * G + h])));
                        x[h] = fmaf(ks[g] * qc->a[g][h], tsum, fmaf(kz[g], qc->qsum[g][h], x[h]));
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = valid ? x[h] * xscale : -INFINITY;
            }
            // raw logits for the score pass (entry order of the stream)
            if (valid) {
                float *lg = lgs_base + ((size_t)t.s * d.ncap + t.oc + t.e + r) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) lg[h] = x[h];
            }
            // tile max per head (and the stager's v-scale maxima) across the softmax warps
            const int par = k & 1;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint32_t mk = __reduce_max_sync(kFull, fkey(x[h]));
                if (lane == 0) xred[par][wq][h] = mk;
            }
            named_sync(1, 128);
            float alpha[G], tmax[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint32_t mk = max(max(xred[par][0][h], xred[par][1][h]), max(xred[par][2][h], xred[par][3][h]));
                tmax[h] = fkey_inv(mk);
                alpha[h] = 1.f;
                if (tmax[h] > m[h] + kRescaleSlack) {
                    alpha[h] = ex2(m[h] - tmax[h]);
                    if (STATS) e[h] = alpha[h] * (e[h] + (m[h] - tmax[h]) * l[h]);
                    l[h] *= alpha[h];
#pragma unroll
                    for (int g = 0; g < 4; ++g) z[g][h] *= alpha[h];
                    m[h] = tmax[h];
                }
            }
            float p[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                p[h] = ex2(x[h] - m[h]);   // 0 for masked rows
                l[h] += p[h];
                if (STATS) e[h] = fmaf(p[h], valid ? x[h] - m[h] : 0.f, e[h]);
            }
            // ---- W (the B operand of PV) for row r
            uint8_t *wbuf = sm + kOffW + b * w_bytes(G);
            float bp_cur[G], bv_cur = 1.f;
            if (t.c == 0) {
                if (r < 64) {
                    uint32_t pw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};   // 16 bf16 columns: hi then lo
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const __nv_bfloat16 hi = __float2bfloat16_rn(p[h]);
                        const __nv_bfloat16 lo = __float2bfloat16_rn(p[h] - __bfloat162float(hi));
                        const uint32_t hb = *reinterpret_cast<const uint16_t *>(&hi);
                        const uint32_t lb = *reinterpret_cast<const uint16_t *>(&lo);
                        pw[h >> 1] |= hb << (16 * (h & 1));
                        pw[(G + h) >> 1] |= lb << (16 * ((G + h) & 1));
                    }
                    uint8_t *dst = wbuf + (r / 8) * 128 + (r % 8) * 16;
                    sts128(dst, pw[0], pw[1], pw[2], pw[3]);
                    sts128(dst + 1024, pw[4], pw[5], pw[6], pw[7]);
                }
#pragma unroll
                for (int h = 0; h < G; ++h) bp_cur[h] = 1.f;
            } else {
                const uint32_t *hdr = reinterpret_cast<const uint32_t *>(sm + kOffMeta + b * kMetaBytes + kMetaHdr);
                float iv[4], ip[G];
                int ev[4], ep[G];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t vk = max(max(hdr[0 * 4 + g], hdr[1 * 4 + g]), max(hdr[2 * 4 + g], hdr[3 * 4 + g]));
                    const float vmax = __half2float(__ushort_as_half((unsigned short)vk));
                    if (vmax > 0.f) {
                        iv[g] = inv_pow2_ceil(vmax, ev[g]) * 4194304.f;   // 2^(22 - ceil log2 vmax)
                    } else {
                        iv[g] = 0.f; ev[g] = 0;
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float pmax = ex2(tmax[h] - m[h]);
                    if (pmax > 1e-30f) {
                        ip[h] = inv_pow2_ceil(pmax, ep[h]);
                    } else {
                        ip[h] = 0.f; ep[h] = 0;
                    }
                    bp_cur[h] = pow2f(ep[h]);
                }
                bv_cur = pow2f(ev[gr] - 22);
                uint32_t wv[4 * G];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float vv = vsc[g] * iv[g];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float pv = p[h] * ip[h];
                        const float wf = pv * vv;   // in [0, 2^22)
                        wv[g * G + h] = __float_as_uint(wf + 12582912.f) - 0x4B400000u;
                        z[g][h] = fmaf(p[h], vze[g], z[g][h]);
                    }
                }
                // row r: group g's columns start at g * gs_of(G); column 4h + byte of a group is
                // byte `byte` of wv[g*G + h]; 16-column chunks 2048 B apart
                uint8_t *dst = wbuf + (r / 8) * 128 + (r % 8) * 16;
                constexpr int CPG = gs_of(G) / 16;   // chunks per group
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int i = 0; i < CPG; ++i) {
                        uint32_t a4[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) a4[j] = 4 * i + j < G ? wv[g * G + 4 * i + j] : 0u;
                        sts128(dst + (g * CPG + i) * 2048, a4[0], a4[1], a4[2], a4[3]);
                    }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_addr(&bar_w_full[b]));
                mbar_arrive(smem_addr(&bar_meta_empty[b]));
            }
            // ---- O of the previous tile
            if (k > 0) {
                o_accumulate(k - 1, c_prev);
                if (newseg) {
                    flush_o_side(tp.s, tp.last);
#pragma unroll
                    for (int h = 0; h < G; ++h) oacc[h] = 0.f;
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) { alpha_prev[h] = alpha[h]; bp_prev[h] = bp_cur[h]; }
            bv_prev = bv_cur;
            c_prev = t.c;
            tp = t;
        }
        if (k > 0) {
            flush_softmax_side(prev_s, seg_first_cta_tile != 0);
            o_accumulate(k - 1, c_prev);
            flush_o_side(tp.s, tp.last);
        } else if (pl.s0 < d.S && r < G) {
            // no tile starts in this CTA's share, which lies inside stream s0 between two
            // tiles: the merge reads this slot, so mark it empty
            d.part[(size_t)(pl.s0 + cta) * part_floats(G) + G + r] = 0.f;
        }
    }

    if (!ok) atomicExch(&err_timeout, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tb, kTmemCols);
    }
    if (tid == 0 && err_timeout) raise_error(d.err, kErrTimeout, (uint32_t)cta);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ merge + score pass
template <int G, bool STATS>
__global__ void __launch_bounds__(256) attn_finalize_kernel(const __grid_constant__ Dev d, float *__restrict__ out,
                                                            float *__restrict__ sparsity,
                                                            uint8_t *__restrict__ thought, float th_r, float th_t,
                                                            int ncta) {
    __shared__ float gM[kMaxG], gInvL[kMaxG], gH[kMaxG];
    __shared__ float fac[64][kMaxG];
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
                if (thought) thought[(size_t)s * G + tid] = (uint8_t)(0.f >= th_t ? 3 : 0.f >= th_r ? 1 : 2);
            }
        }
        return;
    }
    const int c_lo = d.seg_lo[s], c_hi = d.seg_hi[s];
    if (c_lo < 0 || c_hi < c_lo || c_hi >= ncta) {
        if (tid == 0 && split == 0) raise_error(d.err, kErrInvalid, (uint32_t)s);
        return;
    }
    const int nparts = c_hi - c_lo + 1;
    if (tid < G) {
        float M = kNoMax;
        for (int j = 0; j < nparts; ++j) {
            const float *pp = d.part + (size_t)(s + c_lo + j) * part_floats(G);
            if (pp[G + tid] > 0.f) M = fmaxf(M, pp[tid]);
        }
        float L = 0.f, E = 0.f;
        for (int j = 0; j < nparts; ++j) {
            const float *pp = d.part + (size_t)(s + c_lo + j) * part_floats(G);
            const float lj = pp[G + tid];
            const float f = lj > 0.f ? ex2(pp[tid] - M) : 0.f;
            if (j < 64) fac[j][tid] = f;
            L += f * lj;
            if (STATS && lj > 0.f) E += f * (pp[2 * G + tid] + (pp[tid] - M) * lj);
        }
        gM[tid] = M;
        gInvL[tid] = L > 0.f ? 1.f / L : 0.f;
        if (STATS) {
            // H = ln L - ln 2 * sum p (x - M) / L  (x, M in log2 units)
            const float Hh = L > 0.f ? logf(L) - 0.6931471805599453f * E / L : 0.f;
            gH[tid] = N > 1 ? 1.f - Hh / logf((float)N) : 0.f;
        }
    }
    __syncthreads();
    if (split == 0) {
        for (int i = tid; i < G * kD; i += 256) {
            const int h = i / kD;
            float acc = 0.f;
            for (int j = 0; j < nparts; ++j) {
                const float *pp = d.part + (size_t)(s + c_lo + j) * part_floats(G);
                const float f = j < 64 ? fac[j][h] : (pp[G + h] > 0.f ? ex2(pp[h] - gM[h]) : 0.f);
                if (f > 0.f) acc = fmaf(f, pp[3 * G + i], acc);
            }
            orow[i] = acc * gInvL[h];
        }
        if (STATS && tid < G) {
            if (sparsity) sparsity[(size_t)s * G + tid] = gH[tid];
            if (thought) thought[(size_t)s * G + tid] = (uint8_t)(gH[tid] >= th_t ? 3 : gH[tid] >= th_r ? 1 : 2);
        }
    }
    // scores of this CTA's slice of the stream (slices start on 32-entry boundaries)
    const int chunk = ((N + nsplit - 1) / nsplit + 31) & ~31;
    const int t0 = min(N, split * chunk), t1 = min(N, t0 + chunk);
    if (t0 < t1) add_scores<G, 256>(d, s, d.logits + (size_t)s * d.ncap * G, t0, t1, o1, o2, o3, gM, gInvL, tid);
}

int g_bps_i8[kMaxG + 1][2][kMaxDevices] = {};

template <int G, bool STATS>
cudaError_t launch_i8_g(const Dev &d, const void *q, float scale, float *out, float *sparsity, uint8_t *thought,
                        float th_r, float th_t, long long live_ub, cudaStream_t st, int64_t *launches) {
    constexpr int smem = smem_bytes(G);
    int sms = 0, bps = 0;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = cached_blocks_per_sm(g_bps_i8[G][STATS], reinterpret_cast<const void *>(attn_i8_kernel<G, STATS>), kThreads,
                             smem, &bps);
    if (e != cudaSuccess) return e;
    // one CTA per SM (fixed by the device alone, so the split of a given state is always
    // the same and so are the results)
    const int ncta = std::min(sms, d.ncta_max);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ncta, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the launch with the append
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float xscale = scale * 1.4426950408889634f;   // logits in the log2 domain
    e = cudaLaunchKernelEx(&cfg, attn_i8_kernel<G, STATS>, d, static_cast<const __nv_bfloat16 *>(q), xscale);
    *launches += 1;
    if (e != cudaSuccess) return e;
    // the merge + score pass: one CTA per stream, more for long streams
    const int nsplit = (int)std::min<long long>(64, std::max<long long>(1, (live_ub + 4095) / 4096));
    cudaLaunchConfig_t cf2 = {};
    cf2.gridDim = dim3((unsigned)d.S, (unsigned)nsplit, 1);
    cf2.blockDim = dim3(256, 1, 1);
    cf2.dynamicSmemBytes = 0;
    cf2.stream = st;
    cf2.attrs = attr;
    cf2.numAttrs = 1;
    e = cudaLaunchKernelEx(&cf2, attn_finalize_kernel<G, STATS>, d, out, sparsity, thought, th_r, th_t, ncta);
    *launches += 1;
    return e;
}

}  // namespace

cudaError_t launch_attention_i8(const Dev &d, const void *q, float scale, float *out, float *sparsity,
                                uint8_t *thought, float th_r, float th_t, long long live_ub, cudaStream_t st,
                                int64_t *launches) {
    const bool stats = sparsity != nullptr || thought != nullptr;
    switch (d.G) {
        case 1: return stats ? launch_i8_g<1, true>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches)
                             : launch_i8_g<1, false>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches);
        case 2: return stats ? launch_i8_g<2, true>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches)
                             : launch_i8_g<2, false>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches);
        case 4: return stats ? launch_i8_g<4, true>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches)
                             : launch_i8_g<4, false>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches);
        case 8: return stats ? launch_i8_g<8, true>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches)
                             : launch_i8_g<8, false>(d, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st, launches);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tkv
