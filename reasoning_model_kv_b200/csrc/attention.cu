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
// the host so that the whole grid is resident (C = 1 for many streams).
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

#include <type_traits>

#include "attn_common.cuh"

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

struct WarpState {
    float m[2], l[2];   // reference max / (lane-partial) sum for heads 2*tig, 2*tig+1
    float o[8][4];      // O^T fragments: dims 16*mt + g (+8), heads 2*tig, 2*tig+1
    float z[2][4];      // lane-partial sum_t p * vzero per (head, group)
};

// One tile: up to ROWS records of one class, resident in shared memory (row stride
// STRIDE; int8 odd rows chunk-swizzled when SWZ).  Lane (g, tig) owns rows g and
// g + 8.  Rows at or beyond nr hold zeros (the copy zero-fills them); their logits
// are masked to -inf, so they contribute p = 0 everywhere.
template <int BITS, int ROWS, int STRIDE, int G, bool SWZ, int FMT = 0>
__device__ __forceinline__ void tile_compute(const uint8_t *st, int nr, int lane,
                                             const uint32_t (&qb)[4][2][2], const uint32_t (&qbb)[4][2][2],
                                             const float (&qs)[2][4], const float (&qinv)[2][4], bool qscaled,
                                             float xscale, WarpState &ws, float *lg, uint32_t magic) {
    const int g = lane >> 2, tig = lane & 3;
    constexpr int QB = 4 * BITS;     // bytes of one quarter of a code block
    constexpr int CB = 16 * BITS;    // bytes of a code block
    const bool v0 = g < nr;
    const bool v1 = ROWS == 16 && g + 8 < nr;
    const int i0 = g, i1 = g + 8;
    const uint8_t *r0 = st + i0 * STRIDE;
    const uint8_t *r1 = st + i1 * STRIDE;
    const int odd0 = (BITS == 8 && SWZ) ? (i0 & 1) : 0, odd1 = (BITS == 8 && SWZ) ? (i1 & 1) : 0;
    // meta chunk positions (int8 rows: chunks 16 and 17 swap on odd rows)
    const int km_off0 = 2 * CB + 16 * odd0, vm_off0 = 2 * CB + 16 - 16 * odd0;
    const int km_off1 = 2 * CB + 16 * odd1, vm_off1 = 2 * CB + 16 - 16 * odd1;

    // ---- phase 1: S = K . Q^T
    float x[4] = {0.f, 0.f, 0.f, 0.f};   // (row g, head 2tig), (g, 2tig+1), (g+8, 2tig), (g+8, 2tig+1)
    {
        uint32_t k0[BITS], k1[BITS];
        float2 km0[4], km1[4];
        load_quarter<BITS>(r0, QB * tig, odd0, k0);
        if constexpr (ROWS == 16) {
            load_quarter<BITS>(r1, QB * tig, odd1, k1);
        } else {
#pragma unroll
            for (int i = 0; i < BITS; ++i) k1[i] = 0u;
        }
        if constexpr (FMT == 1) {
            // scales: fp16 per group (FP8, ternary) or E4M3 per 16 dims (NVFP4) at 2 CB
            const uint2 ka = *reinterpret_cast<const uint2 *>(r0 + 2 * CB);
            const uint2 kc = *reinterpret_cast<const uint2 *>(r1 + 2 * CB);
            qk_group_fp<BITS, 0>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
            qk_group_fp<BITS, 1>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
            qk_group_fp<BITS, 2>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
            qk_group_fp<BITS, 3>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
        } else {
            if constexpr (BITS < 16) {
                load_meta(r0 + km_off0, km0);
                load_meta(r1 + km_off1, km1);
            }
            qk_group<BITS, 0>(x, k0, k1, qb, qbb, qs, qinv, qscaled, km0, km1, magic);
            qk_group<BITS, 1>(x, k0, k1, qb, qbb, qs, qinv, qscaled, km0, km1, magic);
            qk_group<BITS, 2>(x, k0, k1, qb, qbb, qs, qinv, qscaled, km0, km1, magic);
            qk_group<BITS, 3>(x, k0, k1, qb, qbb, qs, qinv, qscaled, km0, km1, magic);
        }
    }
    const bool h0 = 2 * tig < G, h1 = 2 * tig + 1 < G;
    x[0] = (v0 && h0) ? x[0] * xscale : -INFINITY;
    x[1] = (v0 && h1) ? x[1] * xscale : -INFINITY;
    x[2] = (v1 && h0) ? x[2] * xscale : -INFINITY;
    x[3] = (v1 && h1) ? x[3] * xscale : -INFINITY;
    // raw logits (log2 domain) for the score pass
    if constexpr (G >= 2) {
        if (h0 && v0) *reinterpret_cast<float2 *>(lg + g * G + 2 * tig) = make_float2(x[0], x[1]);
        if (h0 && v1) *reinterpret_cast<float2 *>(lg + (g + 8) * G + 2 * tig) = make_float2(x[2], x[3]);
    } else {
        if (tig == 0 && v0) lg[g] = x[0];
        if (tig == 0 && v1) lg[g + 8] = x[2];
    }

    // ---- online softmax.  The reference max moves only when a tile exceeds it by more
    //      than the slack, so the column maxima (heads are columns: a reduction over the
    //      8 row lanes) are formed only then; the reference starts at a finite
    //      sentinel, so p needs no -inf guard
    float t0 = fmaxf(x[0], x[2]), t1 = fmaxf(x[1], x[3]);
    if (__any_sync(kFull, t0 > ws.m[0] + kRescaleSlack || t1 > ws.m[1] + kRescaleSlack)) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            t0 = fmaxf(t0, __shfl_xor_sync(kFull, t0, o));
            t1 = fmaxf(t1, __shfl_xor_sync(kFull, t1, o));
        }
        const float mn0 = fmaxf(ws.m[0], t0), mn1 = fmaxf(ws.m[1], t1);
        const float a0 = ex2(ws.m[0] - mn0), a1 = ex2(ws.m[1] - mn1);
        ws.m[0] = mn0;
        ws.m[1] = mn1;
        ws.l[0] *= a0;
        ws.l[1] *= a1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            ws.o[mt][0] *= a0; ws.o[mt][1] *= a1; ws.o[mt][2] *= a0; ws.o[mt][3] *= a1;
        }
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) { ws.z[0][grp] *= a0; ws.z[1][grp] *= a1; }
    }
    float p[4];
    p[0] = ex2(x[0] - ws.m[0]);
    p[2] = ex2(x[2] - ws.m[0]);
    p[1] = ex2(x[1] - ws.m[1]);
    p[3] = ex2(x[3] - ws.m[1]);
    ws.l[0] += p[0] + p[2];
    ws.l[1] += p[1] + p[3];

    // ---- phase 2: O += V^T . (P * vscale) per group; zero term accumulated apart.
    //      bf16 values: bf16 MMAs with P split into a bf16 high part and the bf16 of
    //      the remainder (two MMAs), so P keeps ~16 bits and V is never narrowed
    uint32_t bfr[4][2];
    uint32_t blo0 = 0u, blo1 = 0u;
    if constexpr (BITS == 16) {
        const uint32_t h01 = f32x2_to_bf16x2(p[0], p[1]);
        const uint32_t l01 = f32x2_to_bf16x2(p[0] - __uint_as_float(h01 << 16), p[1] - __uint_as_float(h01 & 0xffff0000u));
        const uint32_t b0 = transpose8x8(h01);
        blo0 = transpose8x8(l01);
        uint32_t b1 = 0u;
        if constexpr (ROWS == 16) {
            const uint32_t h23 = f32x2_to_bf16x2(p[2], p[3]);
            const uint32_t l23 =
                f32x2_to_bf16x2(p[2] - __uint_as_float(h23 << 16), p[3] - __uint_as_float(h23 & 0xffff0000u));
            b1 = transpose8x8(h23);
            blo1 = transpose8x8(l23);
        }
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) { bfr[grp][0] = b0; bfr[grp][1] = b1; }
    } else if constexpr (FMT == 1 && BITS == 4) {
        // NVFP4 values are dequantised exactly in f16 (scale folded into V): P alone
        const uint32_t b0 = transpose8x8(f32x2_to_f16x2(p[0], p[1]));
        const uint32_t b1 = transpose8x8(f32x2_to_f16x2(p[2], p[3]));
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) { bfr[grp][0] = b0; bfr[grp][1] = b1; }
    } else if constexpr (FMT == 1) {
        // FP8 / ternary: the group's fp16 scale folds into P; no zero term
        const uint2 va = *reinterpret_cast<const uint2 *>(r0 + 2 * CB + 8);
        const uint2 vc = *reinterpret_cast<const uint2 *>(r1 + 2 * CB + 8);
        const float2 a01 = __half22float2(u32_as_h2(va.x)), a23 = __half22float2(u32_as_h2(va.y));
        const float2 c01 = __half22float2(u32_as_h2(vc.x)), c23 = __half22float2(u32_as_h2(vc.y));
        const float s0[4] = {a01.x, a01.y, a23.x, a23.y}, s1[4] = {c01.x, c01.y, c23.x, c23.y};
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            bfr[grp][0] = transpose8x8(f32x2_to_f16x2(p[0] * s0[grp], p[1] * s0[grp]));
            bfr[grp][1] = transpose8x8(f32x2_to_f16x2(p[2] * s1[grp], p[3] * s1[grp]));
        }
    } else {
        float2 vm0[4], vm1[4];
        load_meta(r0 + vm_off0, vm0);
        load_meta(r1 + vm_off1, vm1);
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            ws.z[0][grp] = fmaf(p[2], vm1[grp].y, fmaf(p[0], vm0[grp].y, ws.z[0][grp]));
            ws.z[1][grp] = fmaf(p[3], vm1[grp].y, fmaf(p[1], vm0[grp].y, ws.z[1][grp]));
            bfr[grp][0] = transpose8x8(f32x2_to_f16x2(p[0] * vm0[grp].x, p[1] * vm0[grp].x));
            bfr[grp][1] = transpose8x8(f32x2_to_f16x2(p[2] * vm1[grp].x, p[3] * vm1[grp].x));
        }
    }
    uint32_t w0[BITS], w1[BITS];
    load_quarter<BITS>(r0, CB + QB * tig, odd0, w0);
    if constexpr (ROWS == 16) {
        load_quarter<BITS>(r1, CB + QB * tig, odd1, w1);
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w1[i] = 0u;
    }
    // NVFP4: each row's E4M3 scale of block MT (dims 16 MT .. 16 MT + 15) as f16x2
    uint2 vb0 = make_uint2(0u, 0u), vb1 = make_uint2(0u, 0u);
    if constexpr (FMT == 1 && BITS == 4) {
        vb0 = *reinterpret_cast<const uint2 *>(r0 + 2 * CB + 8);
        vb1 = *reinterpret_cast<const uint2 *>(r1 + 2 * CB + 8);
    }
    auto vpair = [&](auto pc, const uint32_t (&w)[BITS], const uint2 &vb) -> uint32_t {
        constexpr int P = decltype(pc)::value;
        if constexpr (FMT == 1 && BITS == 4) {
            const uint32_t code = ((P / 2 < 4 ? vb.x : vb.y) >> (8 * ((P / 2) & 3))) & 0xFFu;
            return hmul2_u32(quarter_pair_fp<BITS, P>(w), e4m3_h2(code));
        } else if constexpr (FMT == 1) {
            return quarter_pair_fp<BITS, P>(w);
        } else {
            return quarter_pair<BITS, P>(w, magic);
        }
    };
#define TKV_VMMA(MT)                                                                              \
    {                                                                                             \
        using P0 = std::integral_constant<int, 2 * (MT)>;                                         \
        using P1 = std::integral_constant<int, 2 * (MT) + 1>;                                     \
        const uint32_t e0 = transpose8x8(vpair(P0{}, w0, vb0));                                   \
        const uint32_t e1 = transpose8x8(vpair(P1{}, w0, vb0));                                   \
        const uint32_t e2 = ROWS == 16 ? transpose8x8(vpair(P0{}, w1, vb1)) : 0u;                 \
        const uint32_t e3 = ROWS == 16 ? transpose8x8(vpair(P1{}, w1, vb1)) : 0u;                 \
        if constexpr (BITS == 16) {                                                               \
            mma16816_bf16(ws.o[MT], e0, e1, e2, e3, bfr[(MT) >> 1][0], bfr[(MT) >> 1][1]);        \
            mma16816_bf16(ws.o[MT], e0, e1, e2, e3, blo0, blo1);                                  \
        } else {                                                                                  \
            mma16816(ws.o[MT], e0, e1, e2, e3, bfr[(MT) >> 1][0], bfr[(MT) >> 1][1]);             \
        }                                                                                         \
    }
    TKV_VMMA(0) TKV_VMMA(1) TKV_VMMA(2) TKV_VMMA(3) TKV_VMMA(4) TKV_VMMA(5) TKV_VMMA(6) TKV_VMMA(7)
#undef TKV_VMMA
}

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

template <int G, bool DENSE, int CODEC>
__global__ void __launch_bounds__(kThreads, TKV_ATTN_MIN_BLOCKS) attn_kernel(const __grid_constant__ Dev d,
                                                           const __nv_bfloat16 *__restrict__ q,
                                                           float xscale, float *__restrict__ out,
                                                           int C) {
    extern __shared__ __align__(128) uint8_t ring[];   // kRingBytes, dynamic
    __shared__ float cta_m[kMaxG], cta_l[kMaxG];
    __shared__ float fac[kMaxCluster][kMaxG];     // exp2(m_j - M) per warp / peer rank and head
    __shared__ float gM[kMaxG], gInvL[kMaxG];
    __shared__ __align__(8) uint64_t bars[kWarps][kStages];   // dense placement only

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int rank = blockIdx.x;
    const int s = blockIdx.y;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;

    // ---- query operand (B of S = K Q^T; independent of the previous kernel, so it is
    //      loaded before the dependency wait): head g, dims 32grp + 8tig + 4hh + 0..3.
    //      qbb: the raw bf16 pairs (bf16 keys); qb: f16 pairs for the integer codes,
    //      each (group, head) scaled by a power of two when its largest |q| lies
    //      outside [2^-10, 2^14) so that f16 neither overflows nor goes subnormal on
    //      it; qinv holds the inverse scale of heads 2tig, 2tig+1 per group.
    uint32_t qb[4][2][2], qbb[4][2][2];
    float qs[2][4], qinv[2][4];
    bool qscaled;
    {
        float qsg[4], qsc[4];
        const __nv_bfloat16 *qr = q + ((size_t)b * d.Hkv * G + (size_t)kvh * G + (g < G ? g : 0)) * kD;
        uint2 raw[4][2];
#pragma unroll
        for (int grp = 0; grp < 4; ++grp)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                raw[grp][hh] = make_uint2(0u, 0u);
                if (g < G) raw[grp][hh] = *reinterpret_cast<const uint2 *>(qr + 32 * grp + 8 * tig + 4 * hh);
            }
        bool any = false;
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            float sum = 0.f, mx = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint2 r2 = raw[grp][hh];
                const float f0 = __uint_as_float(r2.x << 16), f1 = __uint_as_float(r2.x & 0xffff0000u);
                const float f2 = __uint_as_float(r2.y << 16), f3 = __uint_as_float(r2.y & 0xffff0000u);
                sum += (f0 + f1) + (f2 + f3);
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3))));
            }
            sum += __shfl_xor_sync(kFull, sum, 1);
            sum += __shfl_xor_sync(kFull, sum, 2);
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
            qsg[grp] = sum;                              // sum over group grp of q[head g]
            // scale 2^(13 - floor(log2 mx)) puts the largest |q| in [2^13, 2^14)
            float sc = 1.f;
            if (mx >= 16384.f || (mx > 0.f && mx < 0.0009765625f)) {
                const int e = (int)((__float_as_uint(mx) >> 23) & 0xff) - 127;
                sc = __uint_as_float((uint32_t)(127 + 13 - e) << 23);
                any = true;
            }
            qsc[grp] = sc;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint2 r2 = raw[grp][hh];
                qbb[grp][hh][0] = r2.x;
                qbb[grp][hh][1] = r2.y;
                qb[grp][hh][0] = f32x2_to_f16x2(__uint_as_float(r2.x << 16) * sc, __uint_as_float(r2.x & 0xffff0000u) * sc);
                qb[grp][hh][1] = f32x2_to_f16x2(__uint_as_float(r2.y << 16) * sc, __uint_as_float(r2.y & 0xffff0000u) * sc);
            }
        }
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            qs[0][grp] = __shfl_sync(kFull, qsg[grp], (2 * tig) * 4);
            qs[1][grp] = __shfl_sync(kFull, qsg[grp], (2 * tig + 1) * 4);
            qinv[0][grp] = 1.f / __shfl_sync(kFull, qsc[grp], (2 * tig) * 4);
            qinv[1][grp] = 1.f / __shfl_sync(kFull, qsc[grp], (2 * tig + 1) * 4);
        }
        qscaled = __any_sync(kFull, any);
    }

    grid_dependency_wait();   // the append's counters and records are visible from here

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
        tile_compute<BITS, CS::ROWS, (DENSE ? CS::REC : CS::STRIDE), G, (!DENSE && CS::SWZ),  \
                     ((CLS) > 0 ? CODEC : 0)>(ring + (warp * kStages + stage) * kStageBytes,  \
                                            nr, lane, qb, qbb, qs, qinv, qscaled, xscale, ws, \
                                            lgs + (size_t)((OFF) + e) * G, magic);            \
        __syncwarp();                                                                         \
        stage = stage == 2 ? 0 : stage + 1;                                                   \
    }
    TKV_CONSUME(0, 16, 0, p1, lo0, hi0, 0)
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
    if (N > 0) {
        add_scores<G, kThreads>(d, s, lgs, t0, t1, o1, o2, o3, gM, gInvL, tid);

    }
    if (C > 1) cluster_sync();   // peers may still be reading this CTA's shared memory
}

int g_blocks_per_sm[2][2][kMaxG + 1][kMaxDevices] = {};   // per codec, placement, G and device

template <int G, bool DENSE, int CODEC>
cudaError_t launch_g(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                     cudaStream_t st, int64_t *launches) {
    int sms = 0, bps = 0;
    cudaError_t e0 = device_sm_count(&sms);
    if (e0 != cudaSuccess) return e0;
    e0 = cached_blocks_per_sm(g_blocks_per_sm[CODEC][DENSE][G], reinterpret_cast<const void *>(attn_kernel<G, DENSE, CODEC>),
                              kThreads, kRingBytes, &bps);
    if (e0 != cudaSuccess) return e0;
    // Largest cluster (<= 8) whose grid is fully resident, never splitting a stream
    // below ~128 tokens per CTA; one CTA per stream when the streams fill the GPU.
    const long long slots = (long long)bps * sms;
    long long C = slots / d.S;
    if (C > kMaxCluster) C = kMaxCluster;
    if (C > live_ub / 128) C = live_ub / 128;
    if (C < 1) C = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)d.S, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kRingBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the launch with the append
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const float xscale = scale * 1.4426950408889634f;   // logits in the log2 domain
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_kernel<G, DENSE, CODEC>, d, static_cast<const __nv_bfloat16 *>(q),
                                       xscale, out, (int)C);
    *launches += 1;
    return e;
}

}  // namespace

cudaError_t launch_attention(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                             cudaStream_t st, int64_t *launches) {
    if (d.dense && d.attn_kernel == 1) return cudaErrorInvalidValue;   // launch_attention_i8's
#define TKV_G_CASES(DN, CD)                                                           \
    switch (d.G) {                                                                    \
        case 1: return launch_g<1, DN, CD>(d, q, scale, out, live_ub, st, launches);  \
        case 2: return launch_g<2, DN, CD>(d, q, scale, out, live_ub, st, launches);  \
        case 4: return launch_g<4, DN, CD>(d, q, scale, out, live_ub, st, launches);  \
        case 8: return launch_g<8, DN, CD>(d, q, scale, out, live_ub, st, launches);  \
        default: return cudaErrorInvalidValue;                                        \
    }
    if (d.codec == 0) {
        if (d.dense) TKV_G_CASES(true, 0)
        TKV_G_CASES(false, 0)
    }
    if (d.dense) TKV_G_CASES(true, 1)
    TKV_G_CASES(false, 1)
#undef TKV_G_CASES
}

}  // namespace tkv
