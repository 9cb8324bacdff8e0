// append_token.cuh -- the per-token work of tkv_quantize_append: thought-adaptive
// group quantisation of one new token's K/V row (ThinKV, Metodologia / TBQ) into its
// class record, slot allocation in the per-precision pool with in-place reuse of
// evicted slots (ThinKV, Implementacao do Sistema / Continuous Thinking), and the
// table / counter updates.  One warp per token; the append kernels' device code.
// Internal to libtkv.
//
// Lane l owns head-dim elements [4l, 4l+4), so a 32-element group is 8 lanes and its
// min/max is a 3-step xor-shuffle reduction.  Codes are then re-gathered through shared
// memory into the record's storage order (see stored_dim), which the decode kernels read
// with wide loads straight into tensor-core operand registers.  The quantiser uses only
// correctly rounded fp32 operations (__fsub_rn, __fdiv_rn, __float2int_rn) and the
// hardware's directed fp32->fp16 conversions, so codes, scales and zeros are bit-exact
// with any IEEE implementation of the same definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tkv_internal.cuh"

namespace tkv {
namespace app {

constexpr unsigned kFull = 0xffffffffu;

// Class a new token is stored in; -1 for an invalid class id.
__device__ __forceinline__ int token_class(const Dev &d, uint8_t c, int32_t p) {
    if (p < d.n_protect) return 0;
    return c <= 3 ? static_cast<int>(c) : -1;
}

// Head-dim index held by storage element e of word w in quarter q of a code
// block (K or V) with BITS-bit elements.  Quarter q holds 16 dim pairs:
//   K pair p: 32*(p/4) + 8*q + 2*(p%4) + {0,1}   (the lane-quad operand of one
//             m16n8k16 k-step per group half),
//   V pair p: 8*p + 2*q + {0,1}                   (one column pair of an 8x8 block);
// a word holds 16/BITS pairs, pair s at elements s and s + 16/BITS, so the two
// members of a pair are always 16 bits apart.
template <int BITS, bool IS_V>
__device__ __forceinline__ int stored_dim(int q, int w, int e) {
    constexpr int ppw = 16 / BITS;
    const int p = w * ppw + e % ppw, hi = e / ppw;
    return IS_V ? 8 * p + 2 * q + hi : 32 * (p / 4) + 8 * q + 2 * (p % 4) + hi;
}

// Word `word` (0 .. 4*BITS-1) of a code block whose codes, indexed by head dim,
// are in shared memory.
template <int BITS, bool IS_V>
__device__ __forceinline__ uint32_t code_word(const uint8_t *codes, int word) {
    const int q = word / BITS, w = word % BITS;
    uint32_t r = 0;
#pragma unroll
    for (int e = 0; e < 32 / BITS; ++e)
        r |= static_cast<uint32_t>(codes[stored_dim<BITS, IS_V>(q, w, e)]) << (BITS * e);
    return r;
}

// Quantise one 128-element bf16 row held as 4 elements per lane (lane l owns dims
// 4l..4l+3, so a group is 8 lanes); write the codes in storage order and the
// group's (scale, zero).
template <int BITS, bool IS_V>
__device__ __forceinline__ void quantize_row(const float (&x)[4], int lane, uint8_t *codes_out,
                                             __half *meta /* [scale x4][zero x4] */,
                                             uint8_t *stage /* 128 bytes of this warp */) {
    constexpr int kQmax = (1 << BITS) - 1;
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    }
    const __half zh = __float2half_rd(mn);
    const float zf = __half2float(zh);
    const float step = __fdiv_rn(__fsub_rn(mx, zf), static_cast<float>(kQmax));
    const __half sh = __float2half_ru(step);
    const float sf = __half2float(sh);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int v = 0;
        if (sf != 0.0f) {
            v = __float2int_rn(__fdiv_rn(__fsub_rn(x[i], zf), sf));
            v = v < 0 ? 0 : (v > kQmax ? kQmax : v);
        }
        packed |= static_cast<uint32_t>(v) << (8 * i);
    }
    __syncwarp();
    reinterpret_cast<uint32_t *>(stage)[lane] = packed;   // codes by head dim
    __syncwarp();
    if (lane < 4 * BITS)
        reinterpret_cast<uint32_t *>(codes_out)[lane] = code_word<BITS, IS_V>(stage, lane);
    if ((lane & 7) == 0) {
        const int g = lane >> 3;
        meta[g] = sh;
        meta[kNG + g] = zh;
    }
}

// ---- floating-point class codes (codec 1; ThinKV page, Metodologia, TBQ: FP8 or
//      NVFP4 for Reasoning tokens, ternary for Transition tokens).  Every step is a
//      correctly rounded fp32 operation or a hardware conversion with round-to-nearest-
//      even and saturation to the format's largest finite value, so the codes and
//      scales are bit-exact with any IEEE implementation of the same definition.
// E4M3 code of x: nearest, ties to even, |x| >= 448 saturating to 448, NaN -> 0x7F
// (both halves of the packed conversion get x, so the byte order does not matter).
__device__ __forceinline__ uint32_t e4m3_rn(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(x));
    return r & 0xFFu;
}
// E2M1 code of x: nearest, ties to the even code, saturating at 6.
__device__ __forceinline__ uint32_t e2m1_rn(float x) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(x));
    return r & 0xFu;
}
// Value of a positive E4M3 code (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    return e == 0 ? (float)m * 0.001953125f                                   // m/8 * 2^-6
                  : __uint_as_float(((e + 120u) << 23) | (m << 20));         // (1 + m/8) * 2^(e-7)
}
// Smallest E4M3 value >= y > 0, saturated at 448 (y <= 0: code 0).
__device__ __forceinline__ uint32_t e4m3_round_up(float y) {
    if (!(y > 0.f)) return 0u;
    if (y >= 448.f) return 0x7Eu;
    uint32_t c = e4m3_rn(y);
    if (e4m3_value(c) < y) ++c;   // positive codes are ordered
    return c;
}

// Codes (by head dim, into the warp's stage) and scales of one 128-element row under
// codec 1.  BITS 8: FP8 per 32-dim group, scale = fp16 round-up of amax / 448, code =
// E4M3 of x / scale.  BITS 4: NVFP4 per 16-dim block, scale = E4M3 round-up of amax / 6,
// code = E2M1 of x / scale.  BITS 2: ternary per group, delta = 0.7 * mean |x|, scale =
// fp16 nearest of the mean |x| over |x| > delta, code 1 / 3 / 0 for x > delta /
// x < -delta / else (sums in head-dim order).  Lane l holds dims 4l .. 4l+3.
template <int BITS>
__device__ __forceinline__ void quantize_row_fp(const float (&x)[4], int lane, uint8_t *scales, uint8_t *stage) {
    uint32_t packed = 0;
    if constexpr (BITS == 8 || BITS == 4) {
        float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
        constexpr int span = BITS == 8 ? 8 : 4;   // lanes of a group / block
#pragma unroll
        for (int o = 1; o < span; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
        float sf;
        if constexpr (BITS == 8) {
            const __half sh = __float2half_ru(__fdiv_rn(amax, 448.f));
            sf = __half2float(sh);
            if ((lane & 7) == 0) reinterpret_cast<__half *>(scales)[lane >> 3] = sh;
        } else {
            const uint32_t sc = e4m3_round_up(__fdiv_rn(amax, 6.f));
            sf = e4m3_value(sc);
            if ((lane & 3) == 0) scales[lane >> 2] = (uint8_t)sc;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t c = 0;
            if (sf != 0.f) c = BITS == 8 ? e4m3_rn(__fdiv_rn(x[i], sf)) : e2m1_rn(__fdiv_rn(x[i], sf));
            packed |= c << (8 * i);
        }
    } else {
        // the group's 32 values in head-dim order, gathered from its 8 lanes
        const int base = lane & ~7;
        float sa = 0.f;
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) sa = __fadd_rn(sa, fabsf(__shfl_sync(kFull, x[i], base + j)));
        const float delta = __fmul_rn(0.7f, __fdiv_rn(sa, 32.f));
        float sb = 0.f;
        int cnt = 0;
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = fabsf(__shfl_sync(kFull, x[i], base + j));
                if (a > delta) { sb = __fadd_rn(sb, a); ++cnt; }
            }
        const float alpha = cnt ? __fdiv_rn(sb, (float)cnt) : 0.f;
        // fp16 nearest; a finite value above the largest finite fp16 takes that value (65504)
        const bool big = alpha >= 65520.f && alpha <= 3.402823466e38f;
        const __half sh = big ? __ushort_as_half((unsigned short)0x7BFFu) : __float2half_rn(alpha);
        if ((lane & 7) == 0) reinterpret_cast<__half *>(scales)[lane >> 3] = sh;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t c = x[i] > delta ? 1u : (x[i] < -delta ? 3u : 0u);
            packed |= c << (8 * i);
        }
    }
    __syncwarp();
    reinterpret_cast<uint32_t *>(stage)[lane] = packed;   // codes by head dim
    __syncwarp();
}

__device__ __forceinline__ void row_floats(const uint2 &raw, float (&x)[4]) {
    x[0] = __uint_as_float(raw.x << 16);
    x[1] = __uint_as_float(raw.x & 0xffff0000u);
    x[2] = __uint_as_float(raw.y << 16);
    x[3] = __uint_as_float(raw.y & 0xffff0000u);
}

// bf16 row -> storage order: word w of quarter q holds the pair (p = w) of 16-bit values.
template <bool IS_V>
__device__ __forceinline__ void store_bf16_row(const uint2 &raw, int lane, uint8_t *dst,
                                               uint16_t *stage /* 128 halves */) {
    __syncwarp();
    reinterpret_cast<uint2 *>(stage)[lane] = raw;          // values by head dim
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int word = lane + 32 * k, q = word / 16, w = word % 16;
        const uint32_t lo = stage[stored_dim<16, IS_V>(q, w, 0)];
        const uint32_t hi = stage[stored_dim<16, IS_V>(q, w, 1)];
        reinterpret_cast<uint32_t *>(dst)[word] = lo | (hi << 16);
    }
}

// One half of a record -- the K (IS_V false) or the V row -- from this lane's 4 elements
// of that row (raw bf16 pairs).  Codec 0 record: [K codes][V codes][K meta][V meta] (bf16
// rows for class 0); codec 1: [K codes][V codes][K scales][V scales].
template <int BITS, bool IS_V>
__device__ __forceinline__ void pack_half(const uint2 &raw, uint8_t *rec, int lane, uint8_t *stage) {
    if constexpr (BITS == 16) {
        store_bf16_row<IS_V>(raw, lane, rec + (IS_V ? 2 * kD : 0), reinterpret_cast<uint16_t *>(stage));
    } else {
        constexpr int cb = kD * BITS / 8;
        __half *meta = reinterpret_cast<__half *>(rec + 2 * cb);
        float x[4];
        row_floats(raw, x);
        quantize_row<BITS, IS_V>(x, lane, rec + (IS_V ? cb : 0), meta + (IS_V ? 2 * kNG : 0), stage);
    }
}
template <int BITS, bool IS_V>
__device__ __forceinline__ void pack_half_fp(const uint2 &raw, uint8_t *rec, int lane, uint8_t *stage) {
    constexpr int cb = kD * BITS / 8;
    constexpr int sb = BITS == 4 ? kD / 16 : 2 * kNG;   // scale bytes of one block
    float x[4];
    row_floats(raw, x);
    quantize_row_fp<BITS>(x, lane, rec + 2 * cb + (IS_V ? sb : 0), stage);
    if (lane < 4 * BITS) reinterpret_cast<uint32_t *>(rec + (IS_V ? cb : 0))[lane] = code_word<BITS, IS_V>(stage, lane);
}

__device__ __forceinline__ int pick4(const int4 &v, int c) {
    return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// Where a new token of stream s goes, from its class id and position and the stream's
// counters before the call (n4 entries, ft4 free slots, hw4 slots ever used per class);
// r is its rank among the new tokens of its class in its batch row.  Returns its class
// and *slot, or -1 when it is dropped: an invalid class id (TKV_ERR_INVALID) or a class
// with neither a free nor a fresh slot (TKV_ERR_CAPACITY), latched when `report` (one
// lane of the warp reports).
__device__ __forceinline__ int append_decide(const Dev &d, int s, uint8_t craw, int32_t p, int r, const int4 &n4,
                                             const int4 &ft4, const int4 &hw4, uint32_t detail, bool report,
                                             int *slot) {
    auto check = [&](bool ok, uint32_t id) {   // the debug build's range checks
#ifdef TKV_DEBUG
        if (!ok && report) raise_error(d.err, kErrInvalid, id);
        return ok;
#else
        (void)ok;
        (void)id;
        return true;
#endif
    };
    const int c = token_class(d, craw, p);
    if (c < 0) {
        if (report) raise_error(d.err, kErrInvalid, detail);
        return -1;
    }
    const int cap = d.cap[c];
    const int ft = pick4(ft4, c), hw = pick4(hw4, c), n = pick4(n4, c);
    if (!check(n >= 0 && n + r < cap && ft >= 0 && ft <= cap && hw >= 0 && hw <= cap && r >= 0, kDbgAppend + c))
        return -1;
    if (r < ft) {
        *slot = d.fs[c][(size_t)s * cap + ft - 1 - r];
        if (!check(*slot >= 0 && *slot < cap, kDbgAppend + 0x10 + c)) return -1;
    } else {
        *slot = hw + (r - ft);
        if (*slot >= cap) {
            if (report) raise_error(d.err, kErrCapacity, (uint32_t)(s * 4 + c));
            return -1;
        }
    }
    return c;
}

// A record of class c from this warp's rows: kBoth, the K row `raw` and the V row `rawv`;
// otherwise the K row (half 0) or the V row (half 1) in `raw`.
template <int kCodec, bool kBoth>
__device__ __forceinline__ void pack_row(int c, int half, const uint2 &raw, const uint2 &rawv, uint8_t *rec, int lane,
                                         uint8_t *stage) {
#define TKV_PACK_HALF(FN, BITS)                                      \
    {                                                                \
        if (kBoth) {                                                 \
            FN<BITS, false>(raw, rec, lane, stage);                  \
            FN<BITS, true>(rawv, rec, lane, stage);                  \
        } else if (half) {                                           \
            FN<BITS, true>(raw, rec, lane, stage);                   \
        } else {                                                     \
            FN<BITS, false>(raw, rec, lane, stage);                  \
        }                                                            \
    }
    if constexpr (kCodec == 0) {
        switch (c) {
            case 0: TKV_PACK_HALF(pack_half, 16) break;
            case 1: TKV_PACK_HALF(pack_half, 8) break;
            case 2: TKV_PACK_HALF(pack_half, 4) break;
            default: TKV_PACK_HALF(pack_half, 2) break;
        }
    } else {
        switch (c) {
            case 0: TKV_PACK_HALF(pack_half, 16) break;
            case 1: TKV_PACK_HALF(pack_half_fp, 8) break;
            case 2: TKV_PACK_HALF(pack_half_fp, 4) break;
            default: TKV_PACK_HALF(pack_half_fp, 2) break;
        }
    }
#undef TKV_PACK_HALF
}

// Appends token t of stream s, tok = s * T + t, from the callers' K / V rows (bf16,
// [S][T][128]), class ids and positions ([B][T]).
// kSingle (T == 1, a decode step): two warps share the token, `half` 0 packing the K row
// and writing the table entry, half 1 the V row (both reach the same slot decision from
// the same inputs); the token's rank r among the new tokens of its class is 0, and the
// pair meets at named barrier `pair_bar` (64 threads) once both have read the stream's
// counters, before half 0 advances them.  Otherwise (a prefill, where throughput rather
// than one token's latency counts) one warp packs both rows (`half` unused), the ranks
// come from the scan kernel and a finalize kernel advances the counters.
// `stage`: 256 bytes of this warp's shared memory.
template <bool kSingle, int kCodec>
__device__ __forceinline__ void append_token(const Dev &d, const __nv_bfloat16 *__restrict__ k,
                                             const __nv_bfloat16 *__restrict__ v, const uint8_t *__restrict__ cls,
                                             const int32_t *__restrict__ pos, int T, int tok, int half, int lane,
                                             uint8_t *stage, int pair_bar) {
    if constexpr (!kSingle) half = 0;
    const int s = tok / T, t = tok - s * T;
    const int b = s / d.Hkv;
    // every independent load first (one round trip): the row(s), the token's position
    // and class, and the stream's counters of all four classes
    const size_t row = ((size_t)s * T + t) * kD;
    const uint2 raw = reinterpret_cast<const uint2 *>((half ? v : k) + row)[lane];
    uint2 rawv = make_uint2(0u, 0u);
    if constexpr (!kSingle) rawv = reinterpret_cast<const uint2 *>(v + row)[lane];
    const int32_t p = pos[(size_t)b * T + t];
    const uint8_t craw = cls[(size_t)b * T + t];
    const int4 n4 = *reinterpret_cast<const int4 *>(d.n + s * 4);
    const int4 ft4 = *reinterpret_cast<const int4 *>(d.ft + s * 4);
    const int4 hw4 = *reinterpret_cast<const int4 *>(d.hw + s * 4);
    const int r = kSingle ? 0 : d.rank[(size_t)b * d.max_append + t];
    int slot = 0;
    const int c = append_decide(d, s, craw, p, r, n4, ft4, hw4, (uint32_t)tok, half == 0 && lane == 0, &slot);
    if (c < 0) return;   // (both warps of a pair)
    const int cap = d.cap[c];
    const size_t e = (size_t)s * cap + pick4(n4, c) + r;
    if (half == 0 && lane == 0) {
        d.handle[c][e] = slot;
        d.pos[c][e] = p;
        d.score[c][e] = 0.0f;
    }
    uint8_t *rec = d.pool[c] + ((size_t)s * cap + slot) * d.rec[c];
    pack_row<kCodec, !kSingle>(c, half, raw, rawv, rec, lane, stage);
    if constexpr (kSingle) {
        // both warps of the pair have read the pre-call counters
        asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
        if (half == 0 && lane == 0) {
            const int sc = s * 4 + c, ft = pick4(ft4, c);
            if (ft > 0) d.ft[sc] = ft - 1; else d.hw[sc] = pick4(hw4, c) + 1;   // popped, or a fresh slot
            d.n[sc] = pick4(n4, c) + 1;
        }
    }
}

}  // namespace app
}  // namespace tkv
