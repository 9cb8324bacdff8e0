// attention.cu -- tkv_decode_attention: one GQA decode step over the
// mixed-precision pools with fused dequantisation, online softmax, and
// accumulation of each token's attention mass into its score (ThinKV decode over
// the Continuous Thinking block table; cumulative attention scores as described
// on the "Back from the Future" page, problem statement).
//
// Work decomposition.  Stream s = (b, kv head) is processed by a cluster of C
// CTAs of kWarps (4) warps (grid (C, S), cluster (C, 1, 1)); CTA r takes a
// contiguous range of the stream's entries (class 0, 1, 2, 3 tables concatenated)
// and cuts it into class-homogeneous tiles (16 records; 8 for bf16).  Warp w
// computes tiles w, w+4, w+8, ... with its own online-softmax state, so the warps
// of a CTA run through the class loops (and their code) together.  C is picked on
// the host so that the whole grid is resident (C = 1 for many streams).  When even
// clusters of 8 would leave SMs idle (a few long streams), a stream gets as many CTAs
// as fill the grid (at least 1024 entries each, and 16 or more) without a cluster: each
// writes its partial (m, l, O) and the merge + score pass of the persistent kernels
// finishes.
//
// Memory path.  Each warp stages its tiles in a 3-deep shared-memory ring: with
// dense placement one bulk copy per tile (the records are contiguous; completion
// on an mbarrier), otherwise 16-byte cp.async copies, eight lanes per record so
// every instruction reads whole 128-byte lines.  Both use the L2 evict_first
// policy; two tiles are in flight while one is computed.  Tile descriptors and the
// record handles are read three tiles ahead into a small register ring.
//
// Math path (tensor cores, mma.sync m16n8k16, f16 x f16 -> f32):
//   S[t][h] = K[t][:] . Q[h][:]      M = 16 tokens, N = 8 heads (G used), one fp32
//            accumulator per 32-dim group; the group's scale multiplies it and its
//            zero adds zero * sum_group(q);
//   O[d][h] += V^T[d][t] . (P * vscale)[t][h]   M = 16 dims, N = 8 heads, K = 16
//            tokens, plus sum_t p * vzero per group (fp32, outside the MMA).
// Integer codes are exact in f16 (magic-number conversion, 1-2 ALU ops per pair);
// the query is f16 too, each (group, head) scaled by a power of two into f16's range
// when needed.  bf16 tiles use bf16 MMAs on the raw keys, values and query (P as a
// bf16 high part plus the bf16 of the remainder), so nothing is narrowed.  The
// record storage order puts each lane's operand pairs 16 bits apart in one word,
// so a row's quarter loads with one or two 16-byte shared-memory reads; the V
// operand and P are transposed in registers with movmatrix.  The running max is
// only moved (and O, l rescaled) when a tile exceeds it by more than 2^8.
//
// Epilogue.  The CTA merges its warps in shared memory; with C > 1 every CTA
// then reads its peers' (m, l) over DSMEM after a cluster barrier and rank r
// merges its slice of the output.  Finally every CTA adds p = exp2(x - M) / L,
// summed over the G heads, to the scores of its own tokens.  Raw logits (log2
// domain) go through a global scratch that stays in L2 and is discarded (no
// write-back) once read.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_tile.cuh"
#include "persist.cuh"

namespace tkv {
namespace {

using namespace attn;

// Warps per CTA and the minimum resident CTAs per SM the register budget is fitted to.
#ifndef TKV_ATTN_WARPS
#define TKV_ATTN_WARPS 4
#endif
#ifndef TKV_ATTN_MIN_BLOCKS
#define TKV_ATTN_MIN_BLOCKS 4
#endif
constexpr int kWarps = TKV_ATTN_WARPS;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 3;
constexpr int kStageBytes = 16 * 288;   // the largest tile: 16 int8 records (rows unpadded, swizzled)
constexpr int kRingBytes = kWarps * kStages * kStageBytes;
constexpr int kSplitTokens = 1024;   // fewest entries per CTA of a stream split beyond a cluster

// Record bytes, reuse-placement stage row stride and rows per tile of class C_ under
// codec CODEC.  Int8 rows (codec 0) are unpadded and chunk-swizzled on odd rows (SWZ);
// the other strides make a quad's row reads fall in distinct banks.
template <int C_, int CODEC>
struct ClassShape {
    static constexpr int REC = C_ == 0 ? 512 : CODEC == 0 ? (C_ == 1 ? 288 : C_ == 2 ? 160 : 96)
                                                          : (C_ == 1 ? 272 : C_ == 2 ? 144 : 80);
    static constexpr int STRIDE = C_ == 0 ? 528 : (CODEC == 0 && C_ == 2) ? 192 : REC;
    static constexpr int ROWS = C_ == 0 ? 8 : 16;
    static constexpr bool SWZ = CODEC == 0 && C_ == 1;
};

// Copy a tile of class C_ into a stage with coalesced 16-byte cp.async: eight
// consecutive lanes cover 128 contiguous bytes of one record, so one instruction
// reads four whole 128-byte lines (records r = lane/8 + 4i).  `hd` holds, in lane
// j < 16, the slot of the tile's record j (any valid slot past the tile).  Rows at
// or beyond nr are zero-filled without reading memory, so the copy has no
// branches and the compute reads zeros (finite) there.  Int8 rows are unpadded and
// odd rows store 16-byte chunk k at k ^ 1.
template <int C_, int CODEC>
__device__ __forceinline__ void issue_tile(uint32_t stage, const uint8_t *pool, int hd, int nr,
                                           int lane, uint64_t pol) {
    using CS = ClassShape<C_, CODEC>;
    constexpr int REC = CS::REC, STRIDE = CS::STRIDE, ROWS = CS::ROWS;
    constexpr int NCH = REC / 16;                  // 16-byte chunks per record
    constexpr int NBLK = (NCH + 7) / 8;            // 8-chunk blocks per record
    const int sub = lane & 7;
#pragma unroll
    for (int i = 0; i < ROWS / 4; ++i) {
        const int r = (lane >> 3) + 4 * i;
        const int slot = __shfl_sync(kFull, hd, r);
        const uint32_t bytes = r < nr ? 16u : 0u;
        const uint8_t *src = pool + (size_t)slot * REC + 16 * sub;
        int dpos = 16 * sub;
        if constexpr (CS::SWZ) dpos += (r & 1) ? ((sub & 1) ? -16 : 16) : 0;   // k ^ 1 on odd rows
        const uint32_t dst = stage + r * STRIDE + dpos;
#pragma unroll
        for (int j = 0; j < NBLK; ++j)
            if (8 * j + sub < NCH) cp_async16_zfill(dst + 128 * j, src + 128 * j, bytes, pol);
    }
}

// Dense placement: the tile's nr records are nr * REC contiguous bytes of the pool,
// copied by one bulk copy into an unpadded stage (row stride REC).  Rows nr..ROWS-1
// of the stage are zeroed first by the warp (generic stores, then a proxy fence so
// they are ordered before later bulk writes of the stage).
template <int C_, int CODEC>
__device__ __forceinline__ void issue_tile_dense(uint8_t *stage_ptr, uint32_t stage, const uint8_t *src,
                                                 int nr, int lane, uint32_t bar, uint64_t pol) {
    constexpr int REC = ClassShape<C_, CODEC>::REC, ROWS = ClassShape<C_, CODEC>::ROWS;
    if (nr < ROWS) {
        uint4 *z = reinterpret_cast<uint4 *>(stage_ptr + nr * REC);
        const int nz = (ROWS - nr) * (REC / 16);
        for (int i = lane; i < nz; i += 32) z[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        __syncwarp();
    }
    if (lane == 0) {
        const uint32_t bytes = (uint32_t)(nr * REC);
        mbar_expect_tx(bar, bytes);
        bulk_copy(stage, src, bytes, bar, pol);
    }
}

// split: C CTAs per stream without a cluster (more than one holds); each writes its
// partial (m, l, O) to slot s C + rank and the merge + score pass of the persistent
// kernels (attn_finalize_kernel) completes the stream.
// STATS: also the attention sparsity 1 - H(p) / ln N of every (stream, query head) and its
// thought class (tkv_decode_attention_sparsity), from the score pass's exp2(x - M).
template <int G, bool DENSE, int CODEC, bool STATS>
__global__ void __launch_bounds__(kThreads, TKV_ATTN_MIN_BLOCKS) attn_kernel(const __grid_constant__ Dev d,
                                                           const __nv_bfloat16 *__restrict__ q,
                                                           float xscale, float *__restrict__ out,
                                                           int C, int split, float *__restrict__ sparsity,
                                                           uint8_t *__restrict__ thought, float th_r, float th_t,
                                                           int q_ready) {
    extern __shared__ __align__(128) uint8_t ring[];   // kRingBytes, dynamic
    __shared__ float cta_m[kMaxG], cta_l[kMaxG];
    __shared__ float fac[kMaxCluster][kMaxG];     // exp2(m_j - M) per warp / peer rank and head
    __shared__ float gM[kMaxG], gInvL[kMaxG];
    __shared__ __align__(8) uint64_t bars[kWarps][kStages];   // dense placement only
    __shared__ float se[kWarps][kMaxG], ce[kMaxG];   // STATS: entropy terms per warp, per CTA
    __shared__ float sqinv[kWarps][4][2][4];          // query inverse scales per warp and tig (rarely read)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int rank = blockIdx.x;
    const int s = blockIdx.y;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;

    // the previous kernel's writes (an append's counters and records, or the caller's
    // query) are visible from here: nothing it may write is read before it, since this
    // kernel may launch while the previous one still runs (programmatic dependent
    // launch).  q_ready: the previous kernel is this library's append, itself launched
    // in plain stream order (so the query was complete before it started), and the
    // query is read while the append still runs.
    if (!q_ready) grid_dependency_wait();

    // ---- query operand (B of S = K Q^T): head g, dims 32grp + 8tig + 4hh + 0..3.
    //      qbb: the raw bf16 pairs (bf16 keys); qb: f16 pairs for the integer codes,
    //      each (group, head) scaled by a power of two when its largest |q| lies
    //      outside [2^-10, 2^14) so that f16 neither overflows nor goes subnormal on
    //      it; qinv holds the inverse scale of heads 2tig, 2tig+1 per group.
    //      One copy lives through the tile loops: qf holds the raw pairs while the bf16
    //      tiles (the first class loop) run, then the scaled f16 pairs.
    //      The inverse scales (used only by queries that needed a scale) wait in shared
    //      memory, one copy per warp and tig, rather than in registers.
    uint32_t qf[4][2][2];
    float qs[2][4];
    bool qscaled;
    uint32_t scexp;
    {
        uint32_t qb_unused[4][2][2];
        float qinv[2][4];
        query_frags<G>(q + ((size_t)b * d.Hkv * G + (size_t)kvh * G) * kD, lane, qb_unused, qf, qs, qinv, qscaled,
                       &scexp);
        if (g == 0) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int grp = 0; grp < 4; ++grp) sqinv[warp][tig][hh][grp] = qinv[hh][grp];
        }
        __syncwarp();
    }
    const float (&qinv)[2][4] = sqinv[warp][tig];
    if (q_ready) grid_dependency_wait();

    // ---- this CTA's entry range and its tiles (class by class)
    const int n0 = dclamp(d.err, d.n[s * 4 + 0], d.cap[0], kDbgAttention + 0);
    const int n1 = dclamp(d.err, d.n[s * 4 + 1], d.cap[1], kDbgAttention + 1);
    const int n2 = dclamp(d.err, d.n[s * 4 + 2], d.cap[2], kDbgAttention + 2);
    const int n3 = dclamp(d.err, d.n[s * 4 + 3], d.cap[3], kDbgAttention + 3);
    const int o1 = n0, o2 = o1 + n1, o3 = o2 + n2, N = o3 + n3;
    const int chunk = ((N + C - 1) / C + 31) & ~31;
    const int t0 = min(N, rank * chunk), t1 = min(N, t0 + chunk);
    const int lo0 = min(t0, o1), hi0 = min(t1, o1);
    const int lo1 = min(max(t0 - o1, 0), n1), hi1 = min(max(t1 - o1, 0), n1);
    const int lo2 = min(max(t0 - o2, 0), n2), hi2 = min(max(t1 - o2, 0), n2);
    const int lo3 = min(max(t0 - o3, 0), n3), hi3 = min(max(t1 - o3, 0), n3);
    const int p1 = (hi0 - lo0 + 7) / 8;                 // tile prefix counts
    const int p2 = p1 + (hi1 - lo1 + 15) / 16;
    const int p3 = p2 + (hi2 - lo2 + 15) / 16;
    const int p4 = p3 + (hi3 - lo3 + 15) / 16;
    float *lgs = d.logits + (size_t)s * d.ncap * G;   // this stream's logits, by entry order

    WarpState ws;
    ws.m[0] = ws.m[1] = kNoMax;
    ws.l[0] = ws.l[1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) ws.o[mt][0] = ws.o[mt][1] = ws.o[mt][2] = ws.o[mt][3] = 0.f;
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) ws.z[0][grp] = ws.z[1][grp] = 0.f;

    const uint64_t pol = policy_evict_first();
    const uint32_t ring0 = smem_addr(ring) + warp * kStages * kStageBytes;
    uint8_t *ring_w = ring + warp * kStages * kStageBytes;
    const uint32_t bar0 = smem_addr(&bars[warp][0]);   // stage i: bar0 + 8 i
    uint32_t phase = 0;                                // dense: parity bit per stage
    if constexpr (DENSE) {
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kStages; ++i) mbar_init(bar0 + 8 * i);
            mbar_init_fence();
        }
        __syncwarp();
    }

    // tile T -> packed descriptor: entry e (bits 0-23), rows nr (24-28), class c (29-30)
    auto tile_of = [&](int T) -> int {
        if (T >= p4) return -1;
        const int c = (T >= p1) + (T >= p2) + (T >= p3);
        const int rows = c == 0 ? 8 : 16;
        const int e = sel4(c, lo0, lo1, lo2, lo3) + (T - sel4(c, 0, p1, p2, p3)) * rows;
        const int nr = min(rows, sel4(c, hi0, hi1, hi2, hi3) - e);
        return e | (nr << 24) | (c << 29);
    };
    // lane j holds the slot of record min(j, nr - 1) of a tile (slot = entry when dense)
    auto handle_of = [&](int dsc) -> int {
        if constexpr (DENSE) {
            return 0;
        } else {
            if (dsc < 0) return 0;
            const int e = dsc & 0xffffff, nr = (dsc >> 24) & 31, c = dsc >> 29;
            const int h = d.handle[c][(size_t)s * d.cap[c] + e + min(lane, nr - 1)];
            return dclamp(d.err, h, d.cap[c] - 1, kDbgAttention + 0x10 + c);
        }
    };
    auto issue = [&](int dsc, int stage, int hd) {
        const int nr = (dsc >> 24) & 31, c = dsc >> 29;
        const uint32_t st = ring0 + stage * kStageBytes;
        const uint8_t *pool = d.pool[c] + (size_t)s * d.cap[c] * d.rec[c];
        if constexpr (DENSE) {
            const int e = dsc & 0xffffff;
            uint8_t *sp = ring_w + stage * kStageBytes;
            const uint32_t bar = bar0 + 8 * stage;
            switch (c) {
                case 0: issue_tile_dense<0, CODEC>(sp, st, pool + (size_t)e * 512, nr, lane, bar, pol); break;
                case 1:
                    issue_tile_dense<1, CODEC>(sp, st, pool + (size_t)e * ClassShape<1, CODEC>::REC, nr, lane, bar, pol);
                    break;
                case 2:
                    issue_tile_dense<2, CODEC>(sp, st, pool + (size_t)e * ClassShape<2, CODEC>::REC, nr, lane, bar, pol);
                    break;
                default:
                    issue_tile_dense<3, CODEC>(sp, st, pool + (size_t)e * ClassShape<3, CODEC>::REC, nr, lane, bar, pol);
                    break;
            }
        } else {
            switch (c) {
                case 0: issue_tile<0, CODEC>(st, pool, hd, nr, lane, pol); break;
                case 1: issue_tile<1, CODEC>(st, pool, hd, nr, lane, pol); break;
                case 2: issue_tile<2, CODEC>(st, pool, hd, nr, lane, pol); break;
                default: issue_tile<3, CODEC>(st, pool, hd, nr, lane, pol); break;
            }
        }
    };
    // wait until the tile in `stage` has landed (dense: its barrier phase; otherwise
    // the cp.async groups, two of which may stay in flight)
    auto arrive_wait = [&](int stage) {
        if constexpr (DENSE) {
            const bool ok = mbar_wait(bar0 + 8 * stage, (phase >> stage) & 1u);
            phase ^= 1u << stage;
            if (!__all_sync(kFull, ok) && lane == 0) raise_error(d.err, kErrTimeout, (uint32_t)s);
        } else {
            cp_async_wait_2();
        }
        __syncwarp();
    };
    const uint32_t magic = magic_f16();

    // Warp tiles t_k = warp + kWarps * k.  Iteration k computes t_k (stage k % 3)
    // after issuing t_{k+2}; descriptors (and handles) of t_{k+2..k+4} sit in a
    // register ring and t_{k+5}'s are loaded each iteration, three iterations
    // before use.  The consumer runs one loop per class (compile-time class).
    {
        const int d0 = tile_of(warp), d1 = tile_of(warp + kWarps);
        if (d0 >= 0) issue(d0, 0, handle_of(d0));
        if constexpr (!DENSE) cp_async_commit();
        if (d1 >= 0) issue(d1, 1, handle_of(d1));
        if constexpr (!DENSE) cp_async_commit();
    }
    int dr0 = tile_of(warp + 2 * kWarps), dr1 = tile_of(warp + 3 * kWarps), dr2 = tile_of(warp + 4 * kWarps);
    int hr0 = handle_of(dr0), hr1 = handle_of(dr1), hr2 = handle_of(dr2);
    int stage = 0;
    int T = warp;
    auto produce = [&]() {
        if (dr0 >= 0) issue(dr0, stage == 0 ? 2 : stage - 1, hr0);
        if constexpr (!DENSE) cp_async_commit();
        dr0 = dr1; dr1 = dr2; hr0 = hr1; hr1 = hr2;
        dr2 = tile_of(T + 5 * kWarps);
        hr2 = handle_of(dr2);
        arrive_wait(stage);
    };
#define TKV_CONSUME(CLS, BITS, PLO, PHI, LO, HI, OFF)                                             \
    for (; T < (PHI); T += kWarps) {                                                          \
        using CS = ClassShape<CLS, CODEC>;                                                    \
        produce();                                                                            \
        const int e = (LO) + (T - (PLO)) * CS::ROWS;                                          \
        const int nr = min(CS::ROWS, (HI) - e);                                               \
        constexpr int FMT_ = (CLS) > 0 ? CODEC : 0;                                          \
        const RowLoader<BITS, (DENSE ? CS::REC : CS::STRIDE), (!DENSE && CS::SWZ), FMT_> ldr(   \
            ring + (warp * kStages + stage) * kStageBytes, lane >> 2);                        \
        tile_compute<BITS, CS::ROWS, G, FMT_>(ldr, nr, lane, qf, qf, qs, qinv, qscaled, xscale, ws, \
                                              lgs + (size_t)((OFF) + e) * G, magic);          \
        __syncwarp();                                                                         \
        stage = stage == 2 ? 0 : stage + 1;                                                   \
    }
    TKV_CONSUME(0, 16, 0, p1, lo0, hi0, 0)
    query_to_f16(qf, scexp);   // the code classes take the scaled f16 query
    TKV_CONSUME(1, 8, p1, p2, lo1, hi1, o1)
    TKV_CONSUME(2, 4, p2, p3, lo2, hi2, o2)
    TKV_CONSUME(3, 2, p3, p4, lo3, hi3, o3)
#undef TKV_CONSUME
    if constexpr (!DENSE) cp_async_wait_0();

    // ---- warp partials: reduce the lane partials over the 8 row lanes, fold z into O
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        ws.l[0] += __shfl_xor_sync(kFull, ws.l[0], o);
        ws.l[1] += __shfl_xor_sync(kFull, ws.l[1], o);
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            ws.z[0][grp] += __shfl_xor_sync(kFull, ws.z[0][grp], o);
            ws.z[1][grp] += __shfl_xor_sync(kFull, ws.z[1][grp], o);
        }
    }
    __syncthreads();                                   // every warp is done with the ring
    float *wm = reinterpret_cast<float *>(ring);       // [kWarps][kMaxG]
    float *wl = wm + kWarps * kMaxG;                   // [kWarps][kMaxG]
    float *wo = wl + kWarps * kMaxG;                   // [kWarps][G][kD]
    float *co = wo + kWarps * G * kD;                  // [G][kD] the CTA's merged O
    if (g == 0) {
        if (2 * tig < G) { wm[warp * kMaxG + 2 * tig] = ws.m[0]; wl[warp * kMaxG + 2 * tig] = ws.l[0]; }
        if (2 * tig + 1 < G) { wm[warp * kMaxG + 2 * tig + 1] = ws.m[1]; wl[warp * kMaxG + 2 * tig + 1] = ws.l[1]; }
    }
    {
        float *w = wo + warp * G * kD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d0 = 16 * mt + g, grp = mt >> 1;
            if (2 * tig < G) {
                w[(2 * tig) * kD + d0] = ws.o[mt][0] + ws.z[0][grp];
                w[(2 * tig) * kD + d0 + 8] = ws.o[mt][2] + ws.z[0][grp];
            }
            if (2 * tig + 1 < G) {
                w[(2 * tig + 1) * kD + d0] = ws.o[mt][1] + ws.z[1][grp];
                w[(2 * tig + 1) * kD + d0 + 8] = ws.o[mt][3] + ws.z[1][grp];
            }
        }
    }
    __syncthreads();
    // ---- CTA merge of the warps
    if (tid < G) {
        float M = kNoMax;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * kMaxG + tid]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = ex2(wm[w * kMaxG + tid] - M);   // warps without tokens carry l = 0
            fac[w][tid] = f;
            L += f * wl[w * kMaxG + tid];
        }
        cta_m[tid] = M;
        cta_l[tid] = L;
    }
    __syncthreads();
    for (int idx = tid; idx < G * kD; idx += kThreads) {
        const int h = idx / kD;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) acc += fac[w][h] * wo[w * G * kD + idx];
        co[idx] = acc;
    }
    __syncthreads();

    // per-warp slots -> ce[h] (a fixed order): the CTA's sum of this thread's e[h], written
    // by thread h (which alone reads it afterwards, or its peers after a cluster barrier)
    auto cta_sum = [&](const float (&e)[G]) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float v = e[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
            if (lane == 0) se[warp][h] = v;
        }
        __syncthreads();
        if (tid < G) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += se[w][tid];
            ce[tid] = v;
        }
    };

    // ---- split: this CTA's partial of the stream for the merge + score pass
    if (split) {
        if constexpr (STATS) {
            // e relative to this CTA's reference max, from the raw logits of its entries
            float e[G];
#pragma unroll
            for (int h = 0; h < G; ++h) e[h] = 0.f;
            for (int t = t0 + tid; t < t1; t += kThreads)
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float x = lgs[(size_t)t * G + h];
                    e[h] = fmaf(exp2f(x - cta_m[h]), x - cta_m[h], e[h]);
                }
            cta_sum(e);
        }
        float *pp = d.part + (size_t)(s * C + rank) * part_floats(G);
        if (tid < G) {
            pp[tid] = cta_m[tid];
            pp[G + tid] = cta_l[tid];
            pp[2 * G + tid] = STATS ? ce[tid] : 0.f;
        }
        for (int idx = tid; idx < G * kD; idx += kThreads) pp[3 * G + idx] = co[idx];
        if (rank == 0 && tid == 0) {   // the stream's partial slots: s + c_lo .. s + c_hi
            d.seg_lo[s] = s * (C - 1);
            d.seg_hi[s] = s * (C - 1) + C - 1;
        }
        return;
    }

    // ---- cluster merge: global (M, L) per head; this rank writes its output slice
    float *orow = out + ((size_t)b * d.Hkv * G + (size_t)kvh * G) * kD;
    if (C == 1) {
        if (tid < G) {
            gM[tid] = cta_m[tid];
            gInvL[tid] = cta_l[tid] > 0.f ? 1.f / cta_l[tid] : 0.f;
        }
        __syncthreads();
        for (int idx = tid; idx < G * kD; idx += kThreads) orow[idx] = co[idx] * gInvL[idx / kD];
    } else {
        cluster_sync();
        if (tid < G) {
            float M = kNoMax;
            for (int j = 0; j < C; ++j) M = fmaxf(M, dsmem_ld(dsmem_addr(cta_m + tid, (uint32_t)j)));
            float L = 0.f;
            for (int j = 0; j < C; ++j) {
                const float mj = dsmem_ld(dsmem_addr(cta_m + tid, (uint32_t)j));
                const float f = ex2(mj - M);
                fac[j][tid] = f;
                L += f * dsmem_ld(dsmem_addr(cta_l + tid, (uint32_t)j));
            }
            gM[tid] = M;
            gInvL[tid] = L > 0.f ? 1.f / L : 0.f;
        }
        __syncthreads();
        const int E = G * kD;
        const int per = (E + C - 1) / C;
        const int e0 = rank * per, e1 = min(E, e0 + per);
        for (int idx = e0 + tid; idx < e1; idx += kThreads) {
            const int h = idx / kD;
            float acc = 0.f;
            for (int j = 0; j < C; ++j) acc += fac[j][h] * dsmem_ld(dsmem_addr(co + idx, (uint32_t)j));
            orow[idx] = acc * gInvL[h];
        }
    }

    // ---- scores of this CTA's tokens: += sum_h exp2(x - M_h) / L_h (none if the stream is empty)
    float e[G];
#pragma unroll
    for (int h = 0; h < G; ++h) e[h] = 0.f;
    if (N > 0) add_scores<G, kThreads, STATS>(d, s, lgs, t0, t1, o1, o2, o3, gM, gInvL, tid, e);
    if constexpr (STATS) {
        // the stream's entropy term: this CTA's, plus its peers' over DSMEM (rank 0 writes)
        cta_sum(e);
        if (C > 1) cluster_sync();
        if (rank == 0 && tid < G) {
            float E = 0.f;
            if (C == 1) E = ce[tid];
            else
                for (int j = 0; j < C; ++j) E += dsmem_ld(dsmem_addr(ce + tid, (uint32_t)j));
            const float L = gInvL[tid] > 0.f ? 1.f / gInvL[tid] : 0.f;
            const float sp = sparsity_of(L, E, N);
            sparsity[(size_t)s * G + tid] = sp;
            if (thought) thought[(size_t)s * G + tid] = thought_of(sp, th_r, th_t);
        }
    }
    if (C > 1) cluster_sync();   // peers may still be reading this CTA's shared memory
}

int g_blocks_per_sm[2][2][2][kMaxG + 1][kMaxDevices] = {};   // per codec, placement, stats, G and device
int g_max_clusters[2][2][2][kMaxG + 1][kMaxCluster + 1][kMaxDevices] = {};   // ... and cluster size

template <int G, bool DENSE, int CODEC, bool STATS>
cudaError_t launch_g(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                     cudaStream_t st, int64_t *launches, float *sparsity, uint8_t *thought, float th_r,
                     float th_t, bool q_ready) {
    int sms = 0, bps = 0;
    cudaError_t e0 = device_sm_count(&sms);
    if (e0 != cudaSuccess) return e0;
    e0 = cached_blocks_per_sm(g_blocks_per_sm[CODEC][DENSE][STATS][G],
                              reinterpret_cast<const void *>(attn_kernel<G, DENSE, CODEC, STATS>), kThreads, kRingBytes,
                              &bps);
    if (e0 != cudaSuccess) return e0;
    // Largest cluster (<= 8) whose grid is fully resident, never splitting a stream
    // below ~128 tokens per CTA; one CTA per stream when the streams fill the GPU.
    // Few long streams (the clusters would leave SMs idle): as many CTAs per stream as
    // fill the resident grid, at least kSplitTokens entries each, merged by a second pass,
    // once that is at least twice a cluster.
    const long long slots = (long long)bps * sms;
    long long C = slots / d.S;
    const long long c_split = std::min<long long>({C, live_ub / kSplitTokens, 2ll * (d.S + kNctaMax) / d.S});
    const bool split = c_split >= 2 * kMaxCluster;   // (a few more CTAs do not pay for the second pass)
    if (split) {
        C = c_split;
    } else {
        if (C > kMaxCluster) C = kMaxCluster;
        if (C > live_ub / 128) C = live_ub / 128;
        if (C < 1) C = 1;
        // clusters are placed within one GPC, where a few SMs' slots can stay unusable for
        // a cluster size: shrink it until every stream's cluster is resident at once (a
        // second wave would double the call)
        while (C > 1) {
            int fit = 0;
            e0 = cached_max_clusters(g_max_clusters[CODEC][DENSE][STATS][G][C],
                                     reinterpret_cast<const void *>(attn_kernel<G, DENSE, CODEC, STATS>), kThreads,
                                     kRingBytes, (int)C, &fit);
            if (e0 != cudaSuccess) return e0;
            if (fit >= d.S) break;
            --C;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)d.S, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kRingBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the launch with the kernel before
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = split ? 1 : 2;
    const float xscale = scale * 1.4426950408889634f;   // logits in the log2 domain
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_kernel<G, DENSE, CODEC, STATS>, d,
                                       static_cast<const __nv_bfloat16 *>(q), xscale, out, (int)C, (int)split,
                                       sparsity, thought, th_r, th_t, (int)q_ready);
    *launches += 1;
    if (e != cudaSuccess || !split) return e;
    return launch_finalize<G, STATS, 1>(d, out, sparsity, thought, th_r, th_t, (int)(d.S * C), live_ub, st, launches);
}

}  // namespace

cudaError_t launch_attention(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                             cudaStream_t st, int64_t *launches, float *sparsity, uint8_t *thought, float th_r,
                             float th_t, bool q_ready) {
    if (d.dense && d.attn_kernel != 0) return cudaErrorInvalidValue;   // the persistent kernels'
#define TKV_G_CASES(DN, CD, ST)                                                                              \
    switch (d.G) {                                                                                           \
        case 1: return launch_g<1, DN, CD, ST>(d, q, scale, out, live_ub, st, launches, sparsity, thought, th_r, th_t, q_ready); \
        case 2: return launch_g<2, DN, CD, ST>(d, q, scale, out, live_ub, st, launches, sparsity, thought, th_r, th_t, q_ready); \
        case 4: return launch_g<4, DN, CD, ST>(d, q, scale, out, live_ub, st, launches, sparsity, thought, th_r, th_t, q_ready); \
        case 8: return launch_g<8, DN, CD, ST>(d, q, scale, out, live_ub, st, launches, sparsity, thought, th_r, th_t, q_ready); \
        default: return cudaErrorInvalidValue;                                                               \
    }
    // one compound statement per (placement, codec): both switches return
#define TKV_ST_CASES(DN, CD)                     \
    {                                            \
        if (sparsity) TKV_G_CASES(DN, CD, true)  \
        TKV_G_CASES(DN, CD, false)               \
    }
    if (d.codec == 0) {
        if (d.dense) TKV_ST_CASES(true, 0)
        TKV_ST_CASES(false, 0)
    }
    if (d.dense) TKV_ST_CASES(true, 1)
    TKV_ST_CASES(false, 1)
#undef TKV_ST_CASES
#undef TKV_G_CASES
}

}  // namespace tkv
