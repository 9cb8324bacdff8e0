// attn_common.cuh -- device helpers shared by the two decode-attention kernels
// (inline PTX wrappers, the exact code -> f16 conversions, the per-group QK
// fragment product).  Internal to libtkv.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "tkv_internal.cuh"

namespace tkv {
namespace attn {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxCluster = 8;
constexpr float kRescaleSlack = 8.f;    // log2 units the running max may lag behind
constexpr float kNoMax = -1e30f;        // reference max before any token: finite, so that
                                        // exp2(-inf - kNoMax) = 0 and exp2(kNoMax - kNoMax) = 1

// ----------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 16-byte copy that reads only `src_size` bytes (0 or 16) and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, uint32_t src_size,
                                                 uint64_t policy) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src),
                 "r"(src_size), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_2() { asm volatile("cp.async.wait_group 2;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---- dense placement: one bulk copy per tile, completion tracked by an mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival (release: this thread's earlier writes are visible to whoever waits on
// the phase).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done;
}

// Bounded wait for phase `parity` of the barrier: false after ~1 s without it.
constexpr long long kWaitCycles = 1ll << 31;
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > limit) return false;
    return true;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    return mbar_wait_for(bar, parity, kWaitCycles);
}

// The same bounded wait, but each probe lets the hardware suspend the warp until the
// phase completes (or a 10 ms hint runs out), so a waiting warp takes no issue slots
// from the warps that work on the same scheduler.
__device__ __forceinline__ uint32_t mbar_try_wait_suspend(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 10000000;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait_suspend(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_suspend(bar, parity))
        if (clock64() - t0 > kWaitCycles) return false;
    return true;
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, "
        "[%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// Programmatic dependent launch: block until the previous kernel in the stream has
// completed and its writes are visible (returns at once when launched without the
// programmatic-serialisation attribute).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

// bf16 x bf16 -> f32 (the operands of bf16-class tiles: raw bf16 keys / values and
// the query, no conversion and no narrowing).
__device__ __forceinline__ void mma16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
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

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ int sel4(int c, int a0, int a1, int a2, int a3) {
    return c == 0 ? a0 : c == 1 ? a1 : c == 2 ? a2 : a3;
}

// ------------------------------------------------- code pair -> f16x2 operand
// (BITS == 16: the raw bf16 pair, the operand of a bf16 MMA.)
// A 32-bit word of a BITS-bit code block holds 16/BITS dim pairs; pair s has its
// members at bits BITS*s and BITS*s + 16.  OR-ing the masked word into 0x6400
// (f16 1024) gives 1024 + m*code in each half (m = 2^(BITS*s') after an optional
// 8-bit shift); one f16x2 FMA, exact, turns that into the code.
// 0x64006400 held in a register (opaque to constant folding), so that
// (w & mask) | magic compiles to a single three-input LOP3.
__device__ __forceinline__ uint32_t magic_f16() {
    uint32_t m;
    asm volatile("mov.b32 %0, 0x64006400;" : "=r"(m));
    return m;
}

template <int BITS, int S>
__device__ __forceinline__ uint32_t code_pair(uint32_t word, uint32_t magic) {
    if constexpr (BITS == 16) {
        return word;
    } else if constexpr (BITS == 8) {
        const uint32_t x = __byte_perm(word, 0x64646464u, S == 0 ? 0x4240 : 0x4341);
        return h2_as_u32(__hsub2(u32_as_h2(x), u32_as_h2(0x64006400u)));
    } else {
        constexpr int kPerShift = BITS == 4 ? 2 : 4;   // pairs reachable without a shift
        constexpr int ss = S % kPerShift;
        const uint32_t w = (S >= kPerShift) ? (word >> 8) : word;
        constexpr uint32_t mask = ((1u << BITS) - 1u) * 0x00010001u;
        const uint32_t x = (w & (mask << (BITS * ss))) | magic;
        if constexpr (ss == 0) {
            return h2_as_u32(__hsub2(u32_as_h2(x), u32_as_h2(0x64006400u)));
        } else {
            // x = 1024 + 2^e * code: multiply by 2^-e, add -1024 * 2^-e (exact in f16)
            constexpr int e = BITS * ss;   // 2, 4 or 6
            constexpr uint32_t mul = e == 2 ? 0x34003400u : e == 4 ? 0x2C002C00u : 0x24002400u;
            constexpr uint32_t add = e == 2 ? 0xDC00DC00u : e == 4 ? 0xD400D400u : 0xCC00CC00u;
            return h2_as_u32(__hfma2(u32_as_h2(x), u32_as_h2(mul), u32_as_h2(add)));
        }
    }
}

// Pair P (0..15) of a quarter held as BITS words.
template <int BITS, int P>
__device__ __forceinline__ uint32_t quarter_pair(const uint32_t (&w)[BITS], uint32_t magic) {
    constexpr int ppw = 16 / BITS;
    return code_pair<BITS, P % ppw>(w[P / ppw], magic);
}

// ------------------------------------------------- floating-point code pair -> f16x2
// (codec 1; same storage order as the integer codes: pair S at elements S and
// S + 16/BITS, i.e. 16 bits apart.)  8: E4M3 and 4: E2M1 through the hardware
// conversions (every value is exact in f16); 2: ternary 1 -> +1, 3 -> -1, 0 -> 0.
template <int BITS, int S>
__device__ __forceinline__ uint32_t code_pair_fp(uint32_t word) {
    if constexpr (BITS == 8) {
        const uint32_t b2 = __byte_perm(word, 0u, S == 0 ? 0x0020u : 0x0031u);   // bytes S, S + 2
        const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)b2, __NV_E4M3);
        return (uint32_t)h.x | ((uint32_t)h.y << 16);
    } else if constexpr (BITS == 4) {
        const uint32_t b = ((word >> (4 * S)) & 0xFu) | ((word >> (4 * S + 12)) & 0xF0u);   // nibbles S, S + 4
        const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)b, __NV_E2M1);
        return (uint32_t)h.x | ((uint32_t)h.y << 16);
    } else {
        const uint32_t c = (word >> (2 * S)) & 0x00030003u;
        return (c & 0x00010001u) * 0x3C00u | ((c & 0x00020002u) << 14);
    }
}

template <int BITS, int P>
__device__ __forceinline__ uint32_t quarter_pair_fp(const uint32_t (&w)[BITS]) {
    constexpr int ppw = 16 / BITS;
    return code_pair_fp<BITS, P % ppw>(w[P / ppw]);
}

// f16x2 with both halves the value of E4M3 code `code` (exact).
__device__ __forceinline__ uint32_t e4m3_h2(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return (uint32_t)h.x * 0x00010001u;
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    return h2_as_u32(__hmul2(u32_as_h2(a), u32_as_h2(b)));
}

// One row's quarter (4*BITS bytes at byte offset `off` of the record).  Int8 tiles keep
// rows unpadded (288 bytes) and store odd rows with 16-byte chunks k and k ^ 1
// swapped, which spreads the two rows a load phase touches over all 32 banks.
template <int BITS>
__device__ __forceinline__ void load_quarter(const uint8_t *row, int off, int odd, uint32_t (&w)[BITS]) {
    if constexpr (BITS == 8) {
        const uint4 a = *reinterpret_cast<const uint4 *>(row + off + 16 * odd);
        const uint4 b = *reinterpret_cast<const uint4 *>(row + off + 16 - 16 * odd);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        return;
    }
    const uint8_t *src = row + off;
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
// 2tig+8, 2tig+9.  Codes: f16 MMA against the f16 query qb (each head's group scaled
// by a power of two into f16's range when its magnitudes need it; qinv undoes the
// scale on the fp32 product); the group's K scale multiplies the fp32 result and its
// zero adds zero * sum_group(q).  bf16 keys: bf16 MMA against the raw bf16 query qbb.
template <int BITS, int GRP>
__device__ __forceinline__ void qk_group(float (&x)[4], const uint32_t (&k0)[BITS],
                                         const uint32_t (&k1)[BITS], const uint32_t (&qb)[4][2][2],
                                         const uint32_t (&qbb)[4][2][2], const float (&qs)[2][4],
                                         const float (&qinv)[2][4], bool qscaled, const float2 (&km0)[4],
                                         const float2 (&km1)[4], uint32_t magic) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (BITS == 16) {
        mma16816_bf16(acc, quarter_pair<BITS, 4 * GRP>(k0, magic), quarter_pair<BITS, 4 * GRP>(k1, magic),
                      quarter_pair<BITS, 4 * GRP + 1>(k0, magic), quarter_pair<BITS, 4 * GRP + 1>(k1, magic),
                      qbb[GRP][0][0], qbb[GRP][0][1]);
        mma16816_bf16(acc, quarter_pair<BITS, 4 * GRP + 2>(k0, magic), quarter_pair<BITS, 4 * GRP + 2>(k1, magic),
                      quarter_pair<BITS, 4 * GRP + 3>(k0, magic), quarter_pair<BITS, 4 * GRP + 3>(k1, magic),
                      qbb[GRP][1][0], qbb[GRP][1][1]);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] += acc[i];
    } else {
        mma16816(acc, quarter_pair<BITS, 4 * GRP>(k0, magic), quarter_pair<BITS, 4 * GRP>(k1, magic),
                 quarter_pair<BITS, 4 * GRP + 1>(k0, magic), quarter_pair<BITS, 4 * GRP + 1>(k1, magic),
                 qb[GRP][0][0], qb[GRP][0][1]);
        mma16816(acc, quarter_pair<BITS, 4 * GRP + 2>(k0, magic), quarter_pair<BITS, 4 * GRP + 2>(k1, magic),
                 quarter_pair<BITS, 4 * GRP + 3>(k0, magic), quarter_pair<BITS, 4 * GRP + 3>(k1, magic),
                 qb[GRP][1][0], qb[GRP][1][1]);
        if (qscaled) {
            acc[0] *= qinv[0][GRP]; acc[1] *= qinv[1][GRP]; acc[2] *= qinv[0][GRP]; acc[3] *= qinv[1][GRP];
        }
        // km = (scale, zero) of the group for row g (0) and row g + 8 (1)
        x[0] = fmaf(km0[GRP].x, acc[0], fmaf(km0[GRP].y, qs[0][GRP], x[0]));
        x[1] = fmaf(km0[GRP].x, acc[1], fmaf(km0[GRP].y, qs[1][GRP], x[1]));
        x[2] = fmaf(km1[GRP].x, acc[2], fmaf(km1[GRP].y, qs[0][GRP], x[2]));
        x[3] = fmaf(km1[GRP].x, acc[3], fmaf(km1[GRP].y, qs[1][GRP], x[3]));
    }
}

// The two MMAs of qk_group for integer codes alone: acc = codes . q over group GRP (the
// f16 query as scaled), with no scale, zero or inverse query scale applied yet.  Used
// when a tile's four groups are formed first and folded together (see tile_compute).
template <int BITS, int GRP>
__device__ __forceinline__ void qk_acc(float (&acc)[4], const uint32_t (&k0)[BITS], const uint32_t (&k1)[BITS],
                                       const uint32_t (&qb)[4][2][2], uint32_t magic) {
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    mma16816(acc, quarter_pair<BITS, 4 * GRP>(k0, magic), quarter_pair<BITS, 4 * GRP>(k1, magic),
             quarter_pair<BITS, 4 * GRP + 1>(k0, magic), quarter_pair<BITS, 4 * GRP + 1>(k1, magic),
             qb[GRP][0][0], qb[GRP][0][1]);
    mma16816(acc, quarter_pair<BITS, 4 * GRP + 2>(k0, magic), quarter_pair<BITS, 4 * GRP + 2>(k1, magic),
             quarter_pair<BITS, 4 * GRP + 3>(k0, magic), quarter_pair<BITS, 4 * GRP + 3>(k1, magic),
             qb[GRP][1][0], qb[GRP][1][1]);
}

// S += K . Q^T over head-dim group GRP for floating-point codes (codec 1), pairs as in
// qk_group.  FP8 / ternary: the code values against the f16 query, times the group's
// fp16 scale (ka / kc: the four K scales of rows g / g + 8); no zero term.  NVFP4: each
// code times its 16-dim block's E4M3 scale (ka / kc: the eight block scales) is exact
// in f16, so the products need no scale afterwards.  Lane tig holds quarter tig, whose
// dims of group GRP lie in block 2 GRP + tig / 2.
template <int BITS, int GRP>
__device__ __forceinline__ void qk_group_fp(float (&x)[4], const uint32_t (&k0)[BITS], const uint32_t (&k1)[BITS],
                                            const uint32_t (&qb)[4][2][2], const float (&qinv)[2][4], bool qscaled,
                                            const uint2 &ka, const uint2 &kc, int tig) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t a[4][2];   // pairs 4 GRP + j of rows g (0) and g + 8 (1)
    a[0][0] = quarter_pair_fp<BITS, 4 * GRP>(k0); a[0][1] = quarter_pair_fp<BITS, 4 * GRP>(k1);
    a[1][0] = quarter_pair_fp<BITS, 4 * GRP + 1>(k0); a[1][1] = quarter_pair_fp<BITS, 4 * GRP + 1>(k1);
    a[2][0] = quarter_pair_fp<BITS, 4 * GRP + 2>(k0); a[2][1] = quarter_pair_fp<BITS, 4 * GRP + 2>(k1);
    a[3][0] = quarter_pair_fp<BITS, 4 * GRP + 3>(k0); a[3][1] = quarter_pair_fp<BITS, 4 * GRP + 3>(k1);
    float s0 = 1.f, s1 = 1.f;
    if constexpr (BITS == 4) {
        const int sh = 8 * ((2 * GRP + (tig >> 1)) & 3);
        const uint32_t b0 = e4m3_h2(((GRP < 2 ? ka.x : ka.y) >> sh) & 0xFFu);
        const uint32_t b1 = e4m3_h2(((GRP < 2 ? kc.x : kc.y) >> sh) & 0xFFu);
#pragma unroll
        for (int j = 0; j < 4; ++j) { a[j][0] = hmul2_u32(a[j][0], b0); a[j][1] = hmul2_u32(a[j][1], b1); }
    } else {
        const int sh = 16 * (GRP & 1);
        s0 = __half2float(__ushort_as_half((unsigned short)(((GRP < 2 ? ka.x : ka.y) >> sh) & 0xFFFFu)));
        s1 = __half2float(__ushort_as_half((unsigned short)(((GRP < 2 ? kc.x : kc.y) >> sh) & 0xFFFFu)));
    }
    mma16816(acc, a[0][0], a[0][1], a[1][0], a[1][1], qb[GRP][0][0], qb[GRP][0][1]);
    mma16816(acc, a[2][0], a[2][1], a[3][0], a[3][1], qb[GRP][1][0], qb[GRP][1][1]);
    if (qscaled) {
        acc[0] *= qinv[0][GRP]; acc[1] *= qinv[1][GRP]; acc[2] *= qinv[0][GRP]; acc[3] *= qinv[1][GRP];
    }
    x[0] = fmaf(s0, acc[0], x[0]);
    x[1] = fmaf(s0, acc[1], x[1]);
    x[2] = fmaf(s1, acc[2], x[2]);
    x[3] = fmaf(s1, acc[3], x[3]);
}

// (scale, zero) pairs of the 4 groups from half of a record's meta block.
__device__ __forceinline__ void load_meta(const uint8_t *meta, float2 (&out)[4]) {
    const uint4 m = *reinterpret_cast<const uint4 *>(meta);   // scale x4 then zero x4 (fp16)
    const float2 s01 = __half22float2(u32_as_h2(m.x)), s23 = __half22float2(u32_as_h2(m.y));
    const float2 z01 = __half22float2(u32_as_h2(m.z)), z23 = __half22float2(u32_as_h2(m.w));
    out[0] = make_float2(s01.x, z01.x);
    out[1] = make_float2(s01.y, z01.y);
    out[2] = make_float2(s23.x, z23.x);
    out[3] = make_float2(s23.y, z23.y);
}

// The attention sparsity 1 - H(p) / ln N of one head (0 when N < 2) from the softmax sum
// L = sum_t exp2(x_t - M) and e = sum_t exp2(x_t - M) (x_t - M) (x, M in log2 units):
// H = ln L - ln 2 * e / L.  Its thought class: 3 (Transition) at or above th_t, else 1
// (Reasoning) at or above th_r, else 2 (Execution).
__device__ __forceinline__ float sparsity_of(float L, float e, int N) {
    const float Hh = L > 0.f ? logf(L) - 0.6931471805599453f * e / L : 0.f;
    return N > 1 ? 1.f - Hh / logf((float)N) : 0.f;
}
__device__ __forceinline__ uint8_t thought_of(float sp, float th_r, float th_t) {
    return (uint8_t)(sp >= th_t ? 3 : sp >= th_r ? 1 : 2);
}

// Scores of this CTA's entries [t0, t1) of stream s: score += sum_h exp2(x_h - M_h) *
// invL_h, x the step's raw logits (log2 domain, entry order, from the L2 scratch).
// Entry t0 + k*NT + tid belongs to thread tid (coalesced), kPer of them per round
// with every load issued before any use (one round covers NT*kPer entries).  A
// warp's 32 consecutive entries fill exactly G whole 128-byte scratch lines (a CTA's
// range starts on a 32-entry boundary), so once the warp has its logits in registers
// it drops those lines from L2 without write-back.
// STATS: e[h] (this thread's share) also accumulates sum_t exp2(x_t - M_h) (x_t - M_h), the
// attention-entropy term H(p) = ln L - ln 2 * e / L of the sparsity statistic.
template <int G, int NT, bool STATS = false>
__device__ __forceinline__ void add_scores(const Dev &d, int s, const float *lgs, int t0, int t1, int o1, int o2,
                                           int o3, const float *gM, const float *gInvL, int tid,
                                           float *e = nullptr) {
    constexpr int kPer = G >= 8 ? 4 : G >= 4 ? 8 : 16;   // x[kPer][G] fits the registers
    const int lane = tid & 31;
    float Mh[G], Ih[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { Mh[h] = gM[h]; Ih[h] = gInvL[h]; }
    // score row of class c, indexed by entry (class c's entries start at o_c)
    float *const r0 = d.score[0] + (size_t)s * d.cap[0], *const r1 = d.score[1] + (size_t)s * d.cap[1] - o1;
    float *const r2 = d.score[2] + (size_t)s * d.cap[2] - o2, *const r3 = d.score[3] + (size_t)s * d.cap[3] - o3;
    auto srow = [&](int t) { return t >= o3 ? r3 : t >= o2 ? r2 : t >= o1 ? r1 : r0; };
    for (int base = t0; base < t1; base += kPer * NT) {
        float x[kPer][G], sv[kPer];
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int t = base + k * NT + tid;
            sv[k] = 0.f;
            if (t < t1) {
                const float *xt = lgs + (size_t)t * G;
                if constexpr (G % 4 == 0) {
#pragma unroll
                    for (int h = 0; h < G; h += 4) {
                        const float4 v = *reinterpret_cast<const float4 *>(xt + h);
                        x[k][h] = v.x; x[k][h + 1] = v.y; x[k][h + 2] = v.z; x[k][h + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) x[k][h] = xt[h];
                }
                sv[k] = srow(t)[t];
            }
        }
        __syncwarp();   // the warp's logits are in registers
        if (lane < G) {
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int w0 = base + k * NT + (tid & ~31);   // first entry of this warp's group
                if (w0 < t1) discard_l2_line(lgs + (size_t)w0 * G + 32 * lane);
            }
        }
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int t = base + k * NT + tid;
            if (t >= t1) continue;
            float inc = 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float ex = exp2f(x[k][h] - Mh[h]);   // full-precision exp2
                inc += ex * Ih[h];
                if constexpr (STATS) e[h] = fmaf(ex, x[k][h] - Mh[h], e[h]);
            }
            srow(t)[t] = sv[k] + inc;
        }
    }
}

}  // namespace attn
}  // namespace tkv
