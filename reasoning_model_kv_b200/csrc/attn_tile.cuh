// attn_tile.cuh -- the per-warp tile computation of the warp-tile decode kernels
// (mma.sync m16n8k16: S = K.Q^T per 32-dim group, online softmax, O += V^T.(P.vscale))
// and the row loaders that present a tile's records to it: records packed in rows of
// a staging ring (RowLoader), or the TMA boxes of a swizzled tile (TmaLoader).
// Internal to libtkv.
#pragma once

#include <type_traits>

#include "attn_common.cuh"

namespace tkv {
namespace attn {

struct WarpState {
    float m[2], l[2];   // reference max / (lane-partial) sum for heads 2*tig, 2*tig+1
    float o[8][4];      // O^T fragments: dims 16*mt + g (+8), heads 2*tig, 2*tig+1
    float z[2][4];      // lane-partial sum_t p * vzero per (head, group)
};

// One tile: up to ROWS records of one class, resident in shared memory (row stride
// STRIDE; int8 odd rows chunk-swizzled when SWZ).  Lane (g, tig) owns rows g and
// g + 8.  Rows at or beyond nr hold zeros (the copy zero-fills them); their logits
// are masked to -inf, so they contribute p = 0 everywhere.
// FOLD4 (integer codes): the four groups' products are formed before one query-scaling
// branch and then folded (the warp-tile kernel); otherwise group by group, each with its
// own branch (the persistent pipeline, whose register budget favours it).  Both give the
// same arithmetic.
template <int BITS, int ROWS, int G, int FMT, bool FOLD4 = true, class Loader>
__device__ __forceinline__ void tile_compute(const Loader &ld, int nr, int lane,
                                             const uint32_t (&qb)[4][2][2], const uint32_t (&qbb)[4][2][2],
                                             const float (&qs)[2][4], const float (&qinv)[2][4], bool qscaled,
                                             float xscale, WarpState &ws, float *lg, uint32_t magic) {
    const int g = lane >> 2, tig = lane & 3;
    const bool v0 = g < nr;
    const bool v1 = ROWS == 16 && g + 8 < nr;

    // ---- phase 1: S = K . Q^T
    float x[4] = {0.f, 0.f, 0.f, 0.f};   // (row g, head 2tig), (g, 2tig+1), (g+8, 2tig), (g+8, 2tig+1)
    {
        uint32_t k0[BITS], k1[BITS];
        float2 km0[4], km1[4];
        ld.k_quarter(0, tig, k0);
        if constexpr (ROWS == 16) {
            ld.k_quarter(1, tig, k1);
        } else {
#pragma unroll
            for (int i = 0; i < BITS; ++i) k1[i] = 0u;
        }
        if constexpr (FMT == 1) {
            // scales: fp16 per group (FP8, ternary) or E4M3 per 16 dims (NVFP4) at 2 CB
            const uint2 ka = *reinterpret_cast<const uint2 *>(ld.k_meta(0));
            const uint2 kc = *reinterpret_cast<const uint2 *>(ld.k_meta(1));
            qk_group_fp<BITS, 0>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
            qk_group_fp<BITS, 1>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
            qk_group_fp<BITS, 2>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
            qk_group_fp<BITS, 3>(x, k0, k1, qb, qinv, qscaled, ka, kc, tig);
        } else if constexpr (BITS < 16 && FOLD4) {
            // the four groups' products first, one branch for the (rare) query scale, then
            // the folds in group order (the same arithmetic as qk_group, group by group)
            load_meta(ld.k_meta(0), km0);
            load_meta(ld.k_meta(1), km1);
            float acc[4][4];
            qk_acc<BITS, 0>(acc[0], k0, k1, qb, magic);
            qk_acc<BITS, 1>(acc[1], k0, k1, qb, magic);
            qk_acc<BITS, 2>(acc[2], k0, k1, qb, magic);
            qk_acc<BITS, 3>(acc[3], k0, k1, qb, magic);
            if (qscaled) {
#pragma unroll
                for (int grp = 0; grp < 4; ++grp) {
                    acc[grp][0] *= qinv[0][grp]; acc[grp][1] *= qinv[1][grp];
                    acc[grp][2] *= qinv[0][grp]; acc[grp][3] *= qinv[1][grp];
                }
            }
#pragma unroll
            for (int grp = 0; grp < 4; ++grp) {
                x[0] = fmaf(km0[grp].x, acc[grp][0], fmaf(km0[grp].y, qs[0][grp], x[0]));
                x[1] = fmaf(km0[grp].x, acc[grp][1], fmaf(km0[grp].y, qs[1][grp], x[1]));
                x[2] = fmaf(km1[grp].x, acc[grp][2], fmaf(km1[grp].y, qs[0][grp], x[2]));
                x[3] = fmaf(km1[grp].x, acc[grp][3], fmaf(km1[grp].y, qs[1][grp], x[3]));
            }
        } else {
            if constexpr (BITS < 16) {
                load_meta(ld.k_meta(0), km0);
                load_meta(ld.k_meta(1), km1);
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
        const uint2 va = *reinterpret_cast<const uint2 *>(ld.v_meta(0));
        const uint2 vc = *reinterpret_cast<const uint2 *>(ld.v_meta(1));
        const float2 a01 = __half22float2(u32_as_h2(va.x)), a23 = __half22float2(u32_as_h2(va.y));
        const float2 c01 = __half22float2(u32_as_h2(vc.x)), c23 = __half22float2(u32_as_h2(vc.y));
        const float s0[4] = {v0 ? a01.x : 0.f, v0 ? a01.y : 0.f, v0 ? a23.x : 0.f, v0 ? a23.y : 0.f};
        const float s1[4] = {v1 ? c01.x : 0.f, v1 ? c01.y : 0.f, v1 ? c23.x : 0.f, v1 ? c23.y : 0.f};
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            bfr[grp][0] = transpose8x8(f32x2_to_f16x2(p[0] * s0[grp], p[1] * s0[grp]));
            bfr[grp][1] = transpose8x8(f32x2_to_f16x2(p[2] * s1[grp], p[3] * s1[grp]));
        }
    } else {
        float2 vm0[4], vm1[4];
        load_meta(ld.v_meta(0), vm0);
        load_meta(ld.v_meta(1), vm1);
        if constexpr (!Loader::kZeroFilled) {
#pragma unroll
            for (int grp = 0; grp < 4; ++grp) {
                vm0[grp] = v0 ? vm0[grp] : make_float2(0.f, 0.f);
                vm1[grp] = v1 ? vm1[grp] : make_float2(0.f, 0.f);
            }
        }
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
            ws.z[0][grp] = fmaf(p[2], vm1[grp].y, fmaf(p[0], vm0[grp].y, ws.z[0][grp]));
            ws.z[1][grp] = fmaf(p[3], vm1[grp].y, fmaf(p[1], vm0[grp].y, ws.z[1][grp]));
            bfr[grp][0] = transpose8x8(f32x2_to_f16x2(p[0] * vm0[grp].x, p[1] * vm0[grp].x));
            bfr[grp][1] = transpose8x8(f32x2_to_f16x2(p[2] * vm1[grp].x, p[3] * vm1[grp].x));
        }
    }
    uint32_t w0[BITS], w1[BITS];
    ld.v_quarter(0, tig, w0);
    if constexpr (ROWS == 16) {
        ld.v_quarter(1, tig, w1);
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w1[i] = 0u;
    }
    // rows past the tile's records may hold anything (a TMA box's trailing rows): their
    // values must not reach the MMA, where 0 * inf would poison the sums (a staging ring
    // zero-fills them already)
    if constexpr (!Loader::kZeroFilled) {
#pragma unroll
        for (int i = 0; i < BITS; ++i) {
            w0[i] = v0 ? w0[i] : 0u;
            w1[i] = v1 ? w1[i] : 0u;
        }
    }
    // NVFP4: each row's E4M3 scale of block MT (dims 16 MT .. 16 MT + 15) as f16x2
    uint2 vb0 = make_uint2(0u, 0u), vb1 = make_uint2(0u, 0u);
    if constexpr (FMT == 1 && BITS == 4) {
        vb0 = v0 ? *reinterpret_cast<const uint2 *>(ld.v_meta(0)) : make_uint2(0u, 0u);
        vb1 = v1 ? *reinterpret_cast<const uint2 *>(ld.v_meta(1)) : make_uint2(0u, 0u);
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


// Query operands of one stream (qh: its G heads x 128 bf16) in m16n8k16 B-fragment order:
// lane (g, tig) holds head g, dims 32 grp + 8 tig + 4 hh + 0..3.  qbb: the raw bf16 pairs
// (bf16 keys); qb: f16 pairs for the codes, each (group, head) scaled by a power of two
// when its largest |q| lies outside [2^-10, 2^14), so that f16 neither overflows nor goes
// subnormal on it; qinv: the inverse scales of heads 2 tig, 2 tig + 1 per group; qs: the
// group sums of q (for the zero term); qscaled: any scale differs from 1.
// scexp (optional): the biased exponents of this lane's own four group scales (head g),
// one byte per group, for query_to_f16 below.
template <int G>
__device__ __forceinline__ void query_frags(const __nv_bfloat16 *__restrict__ qh, int lane, uint32_t (&qb)[4][2][2],
                                            uint32_t (&qbb)[4][2][2], float (&qs)[2][4], float (&qinv)[2][4],
                                            bool &qscaled, uint32_t *scexp = nullptr) {
    const int g = lane >> 2, tig = lane & 3;
    {
        float qsg[4], qsc[4];
        const __nv_bfloat16 *qr = qh + (size_t)(g < G ? g : 0) * kD;
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
            if (scexp) *scexp = (grp == 0 ? 0u : *scexp) | (((__float_as_uint(sc) >> 23) & 0xFFu) << (8 * grp));
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
}

// The raw bf16 query pairs (qbb of query_frags) turned, in place, into the scaled f16 pairs
// (its qb) -- the same arithmetic -- from the lane's scale exponents (scexp): a kernel that
// runs its bf16 tiles first keeps one copy of the query through the tile loops.
__device__ __forceinline__ void query_to_f16(uint32_t (&qf)[4][2][2], uint32_t scexp) {
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {
        const float sc = __uint_as_float(((scexp >> (8 * grp)) & 0xFFu) << 23);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint32_t r = qf[grp][hh][k];
                qf[grp][hh][k] = f32x2_to_f16x2(__uint_as_float(r << 16) * sc, __uint_as_float(r & 0xffff0000u) * sc);
            }
    }
}

// ---- rows of a staging ring: record i at st + i * STRIDE, quarter q of a code block at
// 4 BITS q (K) and 16 BITS + 4 BITS q (V); int8 odd rows swap 16-byte chunks k and k ^ 1
// (SWZ); meta (codec 0: scale x4 + zero x4 per block; codec 1: scales) after the codes.
template <int BITS, int STRIDE, bool SWZ, int FMT>
struct RowLoader {
    static constexpr bool kZeroFilled = true;   // the copies zero-fill rows past the tile
    static constexpr int QB = 4 * BITS, CB = 16 * BITS;
    const uint8_t *r[2];
    int odd[2];
    __device__ __forceinline__ RowLoader(const uint8_t *st, int g) {
        r[0] = st + g * STRIDE;
        r[1] = st + (g + 8) * STRIDE;
        odd[0] = (BITS == 8 && SWZ) ? (g & 1) : 0;
        odd[1] = (BITS == 8 && SWZ) ? ((g + 8) & 1) : 0;
    }
    __device__ __forceinline__ void k_quarter(int i, int tig, uint32_t (&w)[BITS]) const {
        load_quarter<BITS>(r[i], QB * tig, odd[i], w);
    }
    __device__ __forceinline__ void v_quarter(int i, int tig, uint32_t (&w)[BITS]) const {
        load_quarter<BITS>(r[i], CB + QB * tig, odd[i], w);
    }
    __device__ __forceinline__ const uint8_t *k_meta(int i) const {
        return FMT == 1 ? r[i] + 2 * CB : r[i] + 2 * CB + 16 * odd[i];
    }
    __device__ __forceinline__ const uint8_t *v_meta(int i) const {
        return FMT == 1 ? r[i] + 2 * CB + 8 : r[i] + 2 * CB + 16 - 16 * odd[i];
    }
};

// ---- a tile brought by TMA (codec 0): K and V codes in boxes whose rows are the
// record's 128 / 64 / 32-byte code blocks with the 128 / 64 / 32-byte hardware swizzle
// (16-byte chunk j of row r at r * W + 16 (j ^ f(r))), the scale / zero block in a
// 32-byte-row box; bf16 tiles are four 128-byte 128B-swizzled boxes of 64 rows (K bytes
// 0-127, 128-255, then V).  Rows r0 + g and r0 + g + 8 of the tile.
template <int BITS>
struct TmaLoader {
    static constexpr bool kZeroFilled = false;  // trailing rows hold what the pool or an earlier tile left
    static constexpr int W = BITS == 16 ? 128 : 16 * BITS;   // box row bytes
    static constexpr int KOFF = 0;
    static constexpr int VOFF = BITS == 16 ? 16384 : BITS == 8 ? 16384 : BITS == 4 ? 8192 : 4096;
    static constexpr int MOFF = BITS == 8 ? 32768 : BITS == 4 ? 16384 : 8192;
    const uint8_t *st;
    int row[2];
    __device__ __forceinline__ TmaLoader(const uint8_t *stage, int r0, int g) : st(stage) {
        row[0] = r0 + g;
        row[1] = r0 + g + 8;
    }
    __device__ __forceinline__ static uint4 chunk(const uint8_t *box, int r, int j) {
        int x;
        if constexpr (W == 128) x = j ^ (r & 7);
        else if constexpr (W == 64) x = j ^ ((r >> 1) & 3);
        else x = j ^ ((r >> 2) & 1);
        return *reinterpret_cast<const uint4 *>(box + r * W + 16 * x);
    }
    __device__ __forceinline__ void quarter(int off, int i, int tig, uint32_t (&w)[BITS]) const {
        const int r = row[i];
        if constexpr (BITS == 16) {
            const uint8_t *box = st + off + (tig >> 1) * 8192;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = chunk(box, r, 4 * (tig & 1) + j);
                w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
            }
        } else if constexpr (BITS == 8) {
            const uint4 a = chunk(st + off, r, 2 * tig), b = chunk(st + off, r, 2 * tig + 1);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        } else if constexpr (BITS == 4) {
            const uint4 a = chunk(st + off, r, tig);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        } else {
            const uint4 a = chunk(st + off, r, tig >> 1);
            w[0] = (tig & 1) ? a.z : a.x;
            w[1] = (tig & 1) ? a.w : a.y;
        }
    }
    __device__ __forceinline__ void k_quarter(int i, int tig, uint32_t (&w)[BITS]) const { quarter(KOFF, i, tig, w); }
    __device__ __forceinline__ void v_quarter(int i, int tig, uint32_t (&w)[BITS]) const { quarter(VOFF, i, tig, w); }
    __device__ __forceinline__ const uint8_t *k_meta(int i) const { return st + MOFF + 32 * row[i]; }
    __device__ __forceinline__ const uint8_t *v_meta(int i) const { return st + MOFF + 32 * row[i] + 16; }
};

}  // namespace attn
}  // namespace tkv
