// attention.cu -- tkv_decode_attention: one GQA decode step over the
// mixed-precision pools with fused dequantisation, online softmax split over a
// thread-block cluster, and accumulation of each token's attention mass into its
// score (ThinKV decode over the Continuous Thinking block table; cumulative
// attention scores as described on the "Back from the Future" page, problem
// statement).
//
// Work decomposition.  Stream s = (b, kv head) is processed by one cluster of C
// one-warp CTAs (grid (C, S), cluster (C, 1, 1)); CTA r takes a contiguous range
// of the stream's entries (class 0, 1, 2, 3 tables concatenated).  C is chosen
// on the host so that the whole grid is resident at once.
//
// Memory path.  A CTA walks its range in class-homogeneous tiles (16 records;
// 8 for bf16).  For each tile, the lanes of the warp issue one TMA bulk copy per
// record (cp.async.bulk, L2 evict_first) into a 3-stage shared-memory ring, so
// two tiles are in flight while one is computed; an mbarrier per stage tracks
// the bytes.  Handles are prefetched one tile further ahead.
//
// Math path (tensor cores, mma.sync m16n8k16, f16 x f16 -> f32):
//   S[t][h] = K[t][:] . Q[h][:]   M = 16 tokens, N = 8 heads (G used), per 32-dim
//            group, so the group's scale multiplies the fp32 accumulator and
//            its zero adds zero * sum_g(q);
//   O[d][h] += V^T[d][t] . (P * vscale)[t][h]   M = 16 dims, N = 8 heads, K = 16 tokens,
//            plus sum_t p * vzero per group.
// Integer codes are exact in f16 (magic-number conversion, 1-2 ALU ops per pair);
// bf16 keys/values and queries convert exactly to f16 in its normal range.  The
// record storage order puts each lane's operand pairs 16 bits apart in one word,
// so fragments load with one or two 16-byte shared-memory reads per row; the V
// operand and P are transposed with movmatrix.
//
// Epilogue.  Each CTA leaves (m, l, O) in shared memory; after a cluster barrier
// every CTA reads its peers' (m, l) over DSMEM, rank r merges its slice of the
// output, and every CTA adds p = exp2(x - M) / L, summed over the G heads, to
// the scores of its own tokens.  Raw logits (log2 domain) go through a global
// scratch that stays in L2 and is discarded (no write-back) after use.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tkv_internal.cuh"

namespace tkv {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kStages = 3;
constexpr int kStageBytes = 16 * 304;   // the largest tile: 16 int8 records at a 304-byte stride
constexpr long long kSpinLimit = 1ll << 24;  // bounded mbarrier waits (seconds, never reached)

// Per class: bits per element, record bytes, shared-memory row stride (padded so
// the fragment loads of 2-4 rows per phase hit distinct banks) and tile rows.
__device__ __forceinline__ int class_rec(int c) { return c == 0 ? 512 : c == 1 ? 288 : c == 2 ? 160 : 96; }
__device__ __forceinline__ int class_stride(int c) { return c == 0 ? 528 : c == 1 ? 304 : c == 2 ? 192 : 96; }
__device__ __forceinline__ int class_rows(int c) { return c == 0 ? 8 : 16; }

// ----------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: false if the phase did not complete within kSpinLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    for (long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// One record: global -> this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t dsmem_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ float dsmem_ld(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void discard_l2_line(const void *p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    return h2_as_u32(__floats2half2_rn(lo, hi));
}

// ------------------------------------------------- code pair -> f16x2 operand
// A 32-bit word of a BITS-bit code block holds 16/BITS dim pairs; pair s has its
// members at bits BITS*s and BITS*s + 16.  OR-ing the masked word into 0x6400
// (f16 1024) gives 1024 + m*code in each half (m = 2^(BITS*s') after an optional
// 8-bit shift); one f16x2 FMA, exact, turns that into the code.
template <int BITS, int S>
__device__ __forceinline__ uint32_t code_pair(uint32_t word) {
    if constexpr (BITS == 16) {
        return f32x2_to_f16x2(__uint_as_float(word << 16), __uint_as_float(word & 0xffff0000u));
    } else if constexpr (BITS == 8) {
        const uint32_t x = __byte_perm(word, 0x64646464u, S == 0 ? 0x4240 : 0x4341);
        return h2_as_u32(__hsub2(u32_as_h2(x), u32_as_h2(0x64006400u)));
    } else {
        constexpr int kPerShift = BITS == 4 ? 2 : 4;        // pairs reachable without a shift
        constexpr int ss = S % kPerShift;
        const uint32_t w = (S >= kPerShift) ? (word >> 8) : word;
        constexpr uint32_t mask = ((1u << BITS) - 1u) * 0x00010001u;
        const uint32_t x = (w & (mask << (BITS * ss))) | 0x64006400u;
        if constexpr (ss == 0) {
            return h2_as_u32(__hsub2(u32_as_h2(x), u32_as_h2(0x64006400u)));
        } else {
            // x = 1024 + 2^(BITS*ss) * code: multiply by 2^-(BITS*ss), subtract 1024 * 2^-(BITS*ss)
            constexpr int e = BITS * ss;   // 2, 4 or 6
            constexpr uint32_t mul = e == 2 ? 0x34003400u : e == 4 ? 0x2C002C00u : 0x24002400u;
            constexpr uint32_t add = e == 2 ? 0xDC00DC00u : e == 4 ? 0xD400D400u : 0xCC00CC00u;
            return h2_as_u32(__hfma2(u32_as_h2(x), u32_as_h2(mul), u32_as_h2(add)));
        }
    }
}

// Pair P (0..15) of a quarter held as BITS words.
template <int BITS, int P>
__device__ __forceinline__ uint32_t quarter_pair(const uint32_t (&w)[BITS]) {
    constexpr int ppw = 16 / BITS;
    return code_pair<BITS, P % ppw>(w[P / ppw]);
}

template <int BITS>
__device__ __forceinline__ void load_quarter(const uint8_t *src, uint32_t (&w)[BITS]) {
    if constexpr (BITS == 2) {
        const uint2 v = *reinterpret_cast<const uint2 *>(src);
        w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < BITS / 4; ++i) {
            const uint4 v = reinterpret_cast<const uint4 *>(src)[i];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    }
}

// S += K . Q^T over head-dim group GRP (32 dims = 2 k-steps).  Pair p = 4*GRP + 2*hh
// of a quarter carries k-indices 2tig, 2tig+1 of k-step hh; pair p + 1 carries
// 2tig+8, 2tig+9.  The group's K scale multiplies the fp32 result and its zero adds
// zero * sum_group(q).
template <int BITS, int GRP>
__device__ __forceinline__ void qk_group(float (&x)[4], const uint32_t (&k0)[BITS],
                                         const uint32_t (&k1)[BITS], const uint32_t (&qb)[4][2][2],
                                         const float (&qs)[2][4], const float (&ks)[2][4],
                                         const float (&kz)[2][4]) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    mma16816(acc, quarter_pair<BITS, 4 * GRP>(k0), quarter_pair<BITS, 4 * GRP>(k1),
             quarter_pair<BITS, 4 * GRP + 1>(k0), quarter_pair<BITS, 4 * GRP + 1>(k1),
             qb[GRP][0][0], qb[GRP][0][1]);
    mma16816(acc, quarter_pair<BITS, 4 * GRP + 2>(k0), quarter_pair<BITS, 4 * GRP + 2>(k1),
             quarter_pair<BITS, 4 * GRP + 3>(k0), quarter_pair<BITS, 4 * GRP + 3>(k1),
             qb[GRP][1][0], qb[GRP][1][1]);
    if constexpr (BITS == 16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] += acc[i];
    } else {
        x[0] = fmaf(ks[0][GRP], acc[0], fmaf(kz[0][GRP], qs[0][GRP], x[0]));
        x[1] = fmaf(ks[0][GRP], acc[1], fmaf(kz[0][GRP], qs[1][GRP], x[1]));
        x[2] = fmaf(ks[1][GRP], acc[2], fmaf(kz[1][GRP], qs[0][GRP], x[2]));
        x[3] = fmaf(ks[1][GRP], acc[3], fmaf(kz[1][GRP], qs[1][GRP], x[3]));
    }
}

struct Softmax {
    float m[2], l[2];       // running max / sum for heads 2*tig, 2*tig+1 (partial over this lane's rows)
    float o[8][4];          // O^T fragments: dims 16*mt + g (+8), heads 2*tig, 2*tig+1
    float z[2][4];          // sum_t p * vzero per (head, group)
};

// One tile: up to 16 (ROWS) records of one class, resident in shared memory.
template <int BITS, int ROWS, int G>
__device__ __forceinline__ void tile_compute(const uint8_t *st, int stride, int nr, int lane,
                                             const uint32_t (&qb)[4][2][2], const float (&qs)[2][4],
                                             float xscale, Softmax &sm, float *lg) {
    const int g = lane >> 2, tig = lane & 3;
    constexpr int QB = 4 * BITS;     // bytes of one quarter of a code block
    constexpr int CB = 16 * BITS;    // bytes of a code block
    const bool v0 = g < nr;
    const bool v1 = ROWS == 16 && g + 8 < nr;
    uint32_t k0[BITS], k1[BITS], w0[BITS], w1[BITS];
#pragma unroll
    for (int i = 0; i < BITS; ++i) k0[i] = k1[i] = w0[i] = w1[i] = 0u;
    float ks[2][4], kz[2][4], vs[2][4], vz[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) ks[0][i] = ks[1][i] = kz[0][i] = kz[1][i] = vs[0][i] = vs[1][i] = vz[0][i] = vz[1][i] = 0.f;
    auto load_row = [&](const uint8_t *row, uint32_t (&kw)[BITS], uint32_t (&vw)[BITS], int ri) {
        load_quarter<BITS>(row + QB * tig, kw);
        load_quarter<BITS>(row + CB + QB * tig, vw);
        if constexpr (BITS < 16) {
            const uint4 ma = *reinterpret_cast<const uint4 *>(row + 2 * CB);
            const uint4 mb = *reinterpret_cast<const uint4 *>(row + 2 * CB + 16);
            const uint32_t mw[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float2 a = __half22float2(u32_as_h2(mw[j]));       // K scales
                const float2 bz = __half22float2(u32_as_h2(mw[2 + j]));  // K zeros
                const float2 c = __half22float2(u32_as_h2(mw[4 + j]));   // V scales
                const float2 e = __half22float2(u32_as_h2(mw[6 + j]));   // V zeros
                ks[ri][2 * j] = a.x; ks[ri][2 * j + 1] = a.y;
                kz[ri][2 * j] = bz.x; kz[ri][2 * j + 1] = bz.y;
                vs[ri][2 * j] = c.x; vs[ri][2 * j + 1] = c.y;
                vz[ri][2 * j] = e.x; vz[ri][2 * j + 1] = e.y;
            }
        }
    };
    if (v0) load_row(st + g * stride, k0, w0, 0);
    if (v1) load_row(st + (g + 8) * stride, k1, w1, 1);

    // ---- S = K . Q^T, one fp32 accumulator per 32-dim group
    float x[4] = {0.f, 0.f, 0.f, 0.f};   // (row g, head 2tig), (g, 2tig+1), (g+8, 2tig), (g+8, 2tig+1)
    qk_group<BITS, 0>(x, k0, k1, qb, qs, ks, kz);
    qk_group<BITS, 1>(x, k0, k1, qb, qs, ks, kz);
    qk_group<BITS, 2>(x, k0, k1, qb, qs, ks, kz);
    qk_group<BITS, 3>(x, k0, k1, qb, qs, ks, kz);
    const bool h0 = 2 * tig < G, h1 = 2 * tig + 1 < G;
    x[0] = (v0 && h0) ? x[0] * xscale : -INFINITY;
    x[1] = (v0 && h1) ? x[1] * xscale : -INFINITY;
    x[2] = (v1 && h0) ? x[2] * xscale : -INFINITY;
    x[3] = (v1 && h1) ? x[3] * xscale : -INFINITY;
    // raw logits (log2 domain) for the score pass
    if constexpr (G >= 2) {
        if (h0) {
            if (v0) *reinterpret_cast<float2 *>(lg + g * G + 2 * tig) = make_float2(x[0], x[1]);
            if (v1) *reinterpret_cast<float2 *>(lg + (g + 8) * G + 2 * tig) = make_float2(x[2], x[3]);
        }
    } else {
        if (tig == 0) {
            if (v0) lg[g] = x[0];
            if (v1) lg[g + 8] = x[2];
        }
    }

    // ---- online softmax (heads are columns: reduce over the 8 row lanes)
    float t0 = fmaxf(x[0], x[2]), t1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(kFull, t0, o));
        t1 = fmaxf(t1, __shfl_xor_sync(kFull, t1, o));
    }
    const float mn0 = fmaxf(sm.m[0], t0), mn1 = fmaxf(sm.m[1], t1);
    const float a0 = mn0 == -INFINITY ? 1.f : ex2(sm.m[0] - mn0);
    const float a1 = mn1 == -INFINITY ? 1.f : ex2(sm.m[1] - mn1);
    float p[4];
    p[0] = mn0 == -INFINITY ? 0.f : ex2(x[0] - mn0);
    p[2] = mn0 == -INFINITY ? 0.f : ex2(x[2] - mn0);
    p[1] = mn1 == -INFINITY ? 0.f : ex2(x[1] - mn1);
    p[3] = mn1 == -INFINITY ? 0.f : ex2(x[3] - mn1);
    sm.l[0] = sm.l[0] * a0 + p[0] + p[2];
    sm.l[1] = sm.l[1] * a1 + p[1] + p[3];
    sm.m[0] = mn0;
    sm.m[1] = mn1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        sm.o[mt][0] *= a0; sm.o[mt][1] *= a1; sm.o[mt][2] *= a0; sm.o[mt][3] *= a1;
    }
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) { sm.z[0][grp] *= a0; sm.z[1][grp] *= a1; }

    // ---- O += V^T . (P * vscale) per group; zero term accumulated separately
    uint32_t bfr[4][2];
    if constexpr (BITS == 16) {
        const uint32_t b0 = transpose8x8(f32x2_to_f16x2(p[0], p[1]));
        const uint32_t b1 = ROWS == 16 ? transpose8x8(f32x2_to_f16x2(p[2], p[3])) : 0u;
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) { bfr[grp][0] = b0; bfr[grp][1] = b1; }
    } else {
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            sm.z[0][grp] += p[0] * vz[0][grp] + p[2] * vz[1][grp];
            sm.z[1][grp] += p[1] * vz[0][grp] + p[3] * vz[1][grp];
            bfr[grp][0] = transpose8x8(f32x2_to_f16x2(p[0] * vs[0][grp], p[1] * vs[0][grp]));
            bfr[grp][1] = transpose8x8(f32x2_to_f16x2(p[2] * vs[1][grp], p[3] * vs[1][grp]));
        }
    }
#define TKV_VMMA(MT)                                                                          \
    {                                                                                         \
        const uint32_t e0 = transpose8x8(quarter_pair<BITS, 2 * (MT)>(w0));                   \
        const uint32_t e1 = transpose8x8(quarter_pair<BITS, 2 * (MT) + 1>(w0));               \
        const uint32_t e2 = ROWS == 16 ? transpose8x8(quarter_pair<BITS, 2 * (MT)>(w1)) : 0u; \
        const uint32_t e3 = ROWS == 16 ? transpose8x8(quarter_pair<BITS, 2 * (MT) + 1>(w1)) : 0u; \
        mma16816(sm.o[MT], e0, e1, e2, e3, bfr[(MT) >> 1][0], bfr[(MT) >> 1][1]);             \
    }
    TKV_VMMA(0) TKV_VMMA(1) TKV_VMMA(2) TKV_VMMA(3) TKV_VMMA(4) TKV_VMMA(5) TKV_VMMA(6) TKV_VMMA(7)
#undef TKV_VMMA
}

// Tile cursor over the CTA's entry range, class by class.
struct Cursor {
    int c, e;
    __device__ __forceinline__ void skip_empty(const int (&lo)[4], const int (&hi)[4]) {
        while (c < 4 && e >= hi[c]) { ++c; if (c < 4) e = lo[c]; }
    }
    __device__ __forceinline__ void advance(const int (&lo)[4], const int (&hi)[4]) {
        e += class_rows(c);
        skip_empty(lo, hi);
    }
    __device__ __forceinline__ int rows(const int (&hi)[4]) const {
        return min(class_rows(c), hi[c] - e);
    }
};

template <int G>
__global__ void __launch_bounds__(32) attn_kernel(Dev d, const __nv_bfloat16 *__restrict__ q,
                                                  float xscale, float *__restrict__ out, int C) {
    __shared__ __align__(128) uint8_t ring[kStages * kStageBytes];
    __shared__ __align__(8) uint64_t bars[kStages];
    __shared__ float fac[16][kMaxG];     // exp2(m_j - M) per peer rank and head
    __shared__ float gM[kMaxG], gInvL[kMaxG];

    const int lane = threadIdx.x;
    const int g = lane >> 2, tig = lane & 3;
    const int rank = blockIdx.x;
    const int s = blockIdx.y;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;

    int n[4], off[5];
    off[0] = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) { n[c] = d.n[s * 4 + c]; off[c + 1] = off[c] + n[c]; }
    const int N = off[4];
    const int chunk = ((N + C - 1) / C + 31) & ~31;
    const int t0 = min(N, rank * chunk), t1 = min(N, t0 + chunk);
    int lo[4], hi[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        lo[c] = min(max(t0 - off[c], 0), n[c]);
        hi[c] = min(max(t1 - off[c], 0), n[c]);
    }
    float *lgs = d.logits + (size_t)s * d.ncap * G;   // this stream's logits, by entry order

    // ---- query operand (B of S = K Q^T): head g, dims 32grp + 8tig + 4hh + 0..3
    uint32_t qb[4][2][2];
    float qsg[4];
    {
        const __nv_bfloat16 *qr = q + ((size_t)b * d.Hkv * G + (size_t)kvh * G + (g < G ? g : 0)) * kD;
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            float sum = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint2 raw = make_uint2(0u, 0u);
                if (g < G) raw = *reinterpret_cast<const uint2 *>(qr + 32 * grp + 8 * tig + 4 * hh);
                const float f0 = __uint_as_float(raw.x << 16), f1 = __uint_as_float(raw.x & 0xffff0000u);
                const float f2 = __uint_as_float(raw.y << 16), f3 = __uint_as_float(raw.y & 0xffff0000u);
                qb[grp][hh][0] = f32x2_to_f16x2(f0, f1);
                qb[grp][hh][1] = f32x2_to_f16x2(f2, f3);
                sum += (f0 + f1) + (f2 + f3);
            }
            sum += __shfl_xor_sync(kFull, sum, 1);
            sum += __shfl_xor_sync(kFull, sum, 2);
            qsg[grp] = sum;                              // sum over group grp of q[head g]
        }
    }
    float qs[2][4];
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {
        qs[0][grp] = __shfl_sync(kFull, qsg[grp], (2 * tig) * 4);
        qs[1][grp] = __shfl_sync(kFull, qsg[grp], (2 * tig + 1) * 4);
    }

    Softmax sm;
    sm.m[0] = sm.m[1] = -INFINITY;
    sm.l[0] = sm.l[1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) sm.o[mt][0] = sm.o[mt][1] = sm.o[mt][2] = sm.o[mt][3] = 0.f;
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) sm.z[0][grp] = sm.z[1][grp] = 0.f;

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
        fence_mbarrier_init();
    }
    __syncwarp();
    const uint64_t pol = policy_evict_first();

    // cursors: consumer, producer (2 tiles ahead), handle prefetch (3 ahead)
    Cursor cc{0, lo[0]}, cp{0, lo[0]}, ch{0, lo[0]};
    cc.skip_empty(lo, hi);
    cp.skip_empty(lo, hi);
    ch.skip_empty(lo, hi);
    auto handle_of = [&](const Cursor &cu) -> int {
        if (cu.c >= 4 || lane >= cu.rows(hi)) return 0;
        return d.handle[cu.c][(size_t)s * d.cap[cu.c] + cu.e + lane];
    };
    auto issue = [&](const Cursor &cu, int stage, int hd) {
        const int c = cu.c, nr = cu.rows(hi), rb = class_rec(c);
        fence_proxy_async();
        if (lane == 0) mbar_arrive_expect_tx(&bars[stage], (uint32_t)(nr * rb));
        __syncwarp();
        if (lane < nr)
            bulk_load(ring + stage * kStageBytes + lane * class_stride(c),
                      d.pool[c] + ((size_t)s * d.cap[c] + hd) * rb, (uint32_t)rb, &bars[stage], pol);
    };

    int issued = 0;
    int h_next = 0;
    for (int k = 0; k < 2 && cp.c < 4; ++k) {
        issue(cp, issued % kStages, handle_of(cp));
        ++issued;
        cp.advance(lo, hi);
    }
    ch = cp;
    h_next = handle_of(ch);
    if (ch.c < 4) ch.advance(lo, hi);

    bool ok = true;
    int consumed = 0;
    while (cc.c < 4) {
        if (cp.c < 4) {
            issue(cp, issued % kStages, h_next);
            ++issued;
            cp.advance(lo, hi);
            h_next = handle_of(ch);
            if (ch.c < 4) ch.advance(lo, hi);
        }
        const int stage = consumed % kStages;
        // every lane waits (acquire of the TMA writes); the outcome is made warp-uniform
        const bool arrived = mbar_wait(&bars[stage], (uint32_t)((consumed / kStages) & 1));
        if (!__all_sync(kFull, arrived)) {
            ok = false;
            break;
        }
        const uint8_t *st = ring + stage * kStageBytes;
        const int nr = cc.rows(hi);
        float *lg = lgs + (size_t)(off[cc.c] + cc.e) * G;
        switch (cc.c) {
            case 0: tile_compute<16, 8, G>(st, 528, nr, lane, qb, qs, xscale, sm, lg); break;
            case 1: tile_compute<8, 16, G>(st, 304, nr, lane, qb, qs, xscale, sm, lg); break;
            case 2: tile_compute<4, 16, G>(st, 192, nr, lane, qb, qs, xscale, sm, lg); break;
            default: tile_compute<2, 16, G>(st, 96, nr, lane, qb, qs, xscale, sm, lg); break;
        }
        __syncwarp();
        ++consumed;
        cc.advance(lo, hi);
    }
    if (!ok) {
        if (lane == 0) raise_error(d.err, kErrTimeout, (uint32_t)s);
        // let every copy still in flight land before the ring is reused (bounded)
        for (int i = consumed; i < issued; ++i) mbar_wait(&bars[i % kStages], (uint32_t)((i / kStages) & 1));
    }

    // ---- finish this CTA's partial: reduce over the 8 row lanes, fold the zero term
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        sm.l[0] += __shfl_xor_sync(kFull, sm.l[0], o);
        sm.l[1] += __shfl_xor_sync(kFull, sm.l[1], o);
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            sm.z[0][grp] += __shfl_xor_sync(kFull, sm.z[0][grp], o);
            sm.z[1][grp] += __shfl_xor_sync(kFull, sm.z[1][grp], o);
        }
    }
    float *ep_m = reinterpret_cast<float *>(ring);    // [kMaxG]
    float *ep_l = ep_m + kMaxG;                        // [kMaxG]
    float *ep_o = ep_m + 2 * kMaxG;                    // [G][kD]
    __syncwarp();
    if (g == 0) {
        if (2 * tig < G) { ep_m[2 * tig] = sm.m[0]; ep_l[2 * tig] = sm.l[0]; }
        if (2 * tig + 1 < G) { ep_m[2 * tig + 1] = sm.m[1]; ep_l[2 * tig + 1] = sm.l[1]; }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        const int d0 = 16 * mt + g, grp = mt >> 1;
        if (2 * tig < G) {
            ep_o[(2 * tig) * kD + d0] = sm.o[mt][0] + sm.z[0][grp];
            ep_o[(2 * tig) * kD + d0 + 8] = sm.o[mt][2] + sm.z[0][grp];
        }
        if (2 * tig + 1 < G) {
            ep_o[(2 * tig + 1) * kD + d0] = sm.o[mt][1] + sm.z[1][grp];
            ep_o[(2 * tig + 1) * kD + d0 + 8] = sm.o[mt][3] + sm.z[1][grp];
        }
    }
    cluster_sync();

    // ---- merge the cluster: global (M, L) per head, then this rank's output slice
    if (lane < G) {
        float M = -INFINITY;
        for (int j = 0; j < C; ++j) M = fmaxf(M, dsmem_ld(dsmem_addr(ep_m + lane, (uint32_t)j)));
        float L = 0.f;
        for (int j = 0; j < C; ++j) {
            const float mj = dsmem_ld(dsmem_addr(ep_m + lane, (uint32_t)j));
            const float f = M == -INFINITY ? 0.f : ex2(mj - M);
            fac[j][lane] = f;
            L += f * dsmem_ld(dsmem_addr(ep_l + lane, (uint32_t)j));
        }
        gM[lane] = M;
        gInvL[lane] = L > 0.f ? 1.f / L : 0.f;
    }
    __syncwarp();
    {
        const int E = G * kD;
        const int per = (E + C - 1) / C;
        const int e0 = rank * per, e1 = min(E, e0 + per);
        float *orow = out + ((size_t)b * d.Hkv * G + (size_t)kvh * G) * kD;
        for (int idx = e0 + lane; idx < e1; idx += 32) {
            const int h = idx / kD;
            float acc = 0.f;
            for (int j = 0; j < C; ++j) acc += fac[j][h] * dsmem_ld(dsmem_addr(ep_o + idx, (uint32_t)j));
            orow[idx] = acc * gInvL[h];
        }
    }

    // ---- scores of this CTA's tokens: += sum_h exp2(x - M_h) / L_h
    if (ok && gM[0] != -INFINITY) {
        float Mh[kMaxG], Ih[kMaxG];
#pragma unroll
        for (int h = 0; h < G; ++h) { Mh[h] = gM[h]; Ih[h] = gInvL[h]; }
        for (int t = t0 + lane; t < t1; t += 32) {
            const float *xt = lgs + (size_t)t * G;
            float inc = 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h) inc += ex2(xt[h] - Mh[h]) * Ih[h];
            int c = 0;
            while (t >= off[c + 1]) ++c;
            d.score[c][(size_t)s * d.cap[c] + (t - off[c])] += inc;
        }
        __syncwarp();
        const char *base = reinterpret_cast<const char *>(lgs + (size_t)t0 * G);
        const int nlines = (int)(((size_t)(t1 - t0) * G * sizeof(float) + 127) / 128);
        for (int i = lane; i < nlines; i += 32) discard_l2_line(base + (size_t)i * 128);
    }
    cluster_sync();   // peers may still be reading this CTA's shared memory
}

int g_blocks_per_sm[kMaxG + 1] = {0};
int g_sms = 0;

template <int G>
cudaError_t launch_g(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                     cudaStream_t st, int64_t *launches) {
    if (g_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    if (g_blocks_per_sm[G] == 0) {
        int nb = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, attn_kernel<G>, 32, 0);
        if (e != cudaSuccess) return e;
        g_blocks_per_sm[G] = nb > 0 ? nb : 1;
    }
    const long long slots = (long long)g_blocks_per_sm[G] * g_sms;
    long long C = slots / d.S;
    C = C < 1 ? 1 : (C > 8 ? 8 : C);
    const long long by_tokens = live_ub / 64;
    if (C > by_tokens) C = by_tokens < 1 ? 1 : by_tokens;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)d.S, 1);
    cfg.blockDim = dim3(32, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float xscale = scale * 1.4426950408889634f;   // logits in the log2 domain
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_kernel<G>, d, static_cast<const __nv_bfloat16 *>(q),
                                       xscale, out, (int)C);
    *launches += 1;
    return e;
}

}  // namespace

cudaError_t launch_attention(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                             cudaStream_t st, int64_t *launches) {
    switch (d.G) {
        case 1: return launch_g<1>(d, q, scale, out, live_ub, st, launches);
        case 2: return launch_g<2>(d, q, scale, out, live_ub, st, launches);
        case 4: return launch_g<4>(d, q, scale, out, live_ub, st, launches);
        case 8: return launch_g<8>(d, q, scale, out, live_ub, st, launches);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tkv
