/*
 * tkv_oracle.c -- plain, slow CPU oracle of the thought-adaptive compressed
 * KV-cache decode step (ThinKV-style).  TEST INFRASTRUCTURE ONLY: it is used by
 * the test-suite, by the smoke check and by the benchmark's CPU-baseline leg; the
 * product path never links, loads or calls it.  It shares no code with the CUDA
 * library (its own structs, its own fp16 conversion, its own packing).
 *
 * What it computes, and where the pages define it:
 *
 *  - Thought-adaptive group quantisation ("ThinKV", section Metodologia, TBQ
 *    paragraph: precision chosen by thought type, importance R > E > T,
 *    tokens group-quantised per category).  Reading used here: asymmetric
 *    integer codes of 8/4/2 bits for R/E/T, groups of 32 consecutive head_dim
 *    elements, one fp16 scale and one fp16 zero (an offset value) per group,
 *    for K and for V of every token; zero = min rounded down to fp16, scale =
 *    (max - zero)/(2^b - 1) rounded up to fp16; code = round-half-even of
 *    (x - zero)/scale in fp32, clamped to [0, 2^b-1].  Tokens whose position is
 *    below n_protect (attention sinks / question window: "DYNTS", section 2.3,
 *    question window never evicted) are stored as bf16.
 *  - Paged per-precision pools with in-place slot reuse ("ThinKV", section
 *    Implementacao do Sistema, Continuous Thinking: a block table tracks
 *    thought type and eviction, and new tokens of the same type overwrite
 *    evicted slots without gather-based compaction).
 *  - Decode attention over the dequantised cache, in fp64, and accumulation of
 *    each token's attention mass as its importance score (H2O-style cumulative
 *    attention; "Back from the Future", problem statement; "ThinKV",
 *    Resultados names H2O/R-KV as the baselines).
 *  - Budgeted top-k eviction ("DYNTS", section 2.3, selection window: keep
 *    the k highest-scoring tokens, evict the rest) followed by a stable
 *    compaction of the block table; evicted slots go to a per-class free stack.
 *  - Segment-level eviction ("ThinKV", section Metodologia, TBE paragraph: when
 *    a Transition thought starts, earlier R/E segments are cut down segment by
 *    segment on an annealing schedule, retention 64, 32, 16, ...; a few
 *    Transition tokens are always kept).  Reading used here: a completed R/E
 *    segment followed by k >= 1 Transition segments keeps r0 >> (k - 1) of its
 *    tokens, a completed T segment followed by another keeps t_keep, the open
 *    segment and bf16-labelled segments keep everything; inside a segment the
 *    kept tokens are the first under (score desc, position asc).
 *  - Thought-aware budgets with pivotal-token protection ("Compactacao de Cache KV
 *    Consciente do Pensamento ... (TAM)", sections 2.B-2.C), as a selection policy:
 *    segment j keeps floor(T' sqrt(w_j) n_j / sum_i sqrt(w_i) n_i) of its tokens
 *    (w_j = mean accumulated score of its candidates), tokens scoring at least
 *    c times the stream's mean are kept on top.  The attention-matching refit of
 *    the kept keys that TAM performs is not specified on the page and not modelled.
 *
 * Floating point: quantisation is done in IEEE fp32 with round-to-nearest-even
 * and no contraction (build with -ffp-contract=off, no fast-math).  The
 * fp32 -> fp16 directed conversions are written here from the IEEE-754
 * definition (largest fp16 <= x, smallest fp16 >= x).  Attention, softmax and
 * scores are fp64; output is rounded to fp32 and the score is stored as fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_INVALID 1
#define ORC_ERR_CAPACITY 2

typedef struct {
    int32_t B, Hkv, G, D, group, n_protect;
    int32_t bits[4];   /* 16 (bf16), 8, 4, 2 for classes 0..3 */
    int32_t cap[4];    /* slots per stream per class */
    int32_t dense;     /* 0: evicted slots reused in place; 1: dense placement */
    uint8_t *pool[4];  /* [S][cap[c]][rec_bytes(c)] */
    int32_t *n, *ft, *hw;          /* [S][4] */
    int32_t *handle[4], *pos[4], *fs[4];  /* [S][cap[c]] */
    float *score[4];               /* [S][cap[c]] */
    int32_t codec;     /* 0: integer codes; 1: FP codes for classes 1-3 (FP8, NVFP4, ternary) */
} orc_state;

/* ------------------------------------------------------------------ */
/* bf16 / fp16 scalar helpers (IEEE-754 definitions)                   */
/* ------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

double orc_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* fp16 bit pattern of a double that is exactly representable in fp16
 * (or +-inf). */
static uint16_t exact_to_f16_bits(double v) {
    uint16_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a)) return sign | 0x7C00;
    if (a == 0) return sign;
    if (a < ldexp(1.0, -14)) return sign | (uint16_t)(a / ldexp(1.0, -24));
    int E;
    frexp(a, &E);          /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;         /* a in [2^e, 2^(e+1)) */
    double mant = a / ldexp(1.0, e) - 1.0;  /* [0, 1) */
    return sign | (uint16_t)((e + 15) << 10) | (uint16_t)(mant * 1024.0);
}

/* spacing of fp16 values at magnitude a (a finite, >= 0) */
static double f16_quantum(double a) {
    if (a < ldexp(1.0, -14)) return ldexp(1.0, -24);
    int E;
    frexp(a, &E);
    int e = E - 1;
    if (e > 15) e = 15;
    return ldexp(1.0, e - 10);
}

/* largest fp16 value <= x (round toward -inf) */
uint16_t orc_f32_to_f16_rd(float xf) {
    double x = xf;
    if (isnan(x)) return 0x7FFF;
    if (isinf(x)) return x > 0 ? 0x7C00 : 0xFC00;
    if (x == 0) return signbit(x) ? 0x8000 : 0;
    double q = f16_quantum(fabs(x));
    double v = floor(x / q) * q;
    if (v > 65504.0) v = 65504.0;
    if (v < -65504.0) v = -INFINITY;
    if (v == 0) v = 0.0; /* floor of a tiny positive value is +0 */
    return exact_to_f16_bits(v);
}

/* smallest fp16 value >= x (round toward +inf) */
uint16_t orc_f32_to_f16_ru(float xf) {
    double x = xf;
    if (isnan(x)) return 0x7FFF;
    if (isinf(x)) return x > 0 ? 0x7C00 : 0xFC00;
    if (x == 0) return signbit(x) ? 0x8000 : 0;
    double q = f16_quantum(fabs(x));
    double v = ceil(x / q) * q;
    if (v < -65504.0) v = -65504.0;
    if (v > 65504.0) v = INFINITY;
    if (v == 0) v = -0.0; /* ceil of a tiny negative value is -0 */
    return exact_to_f16_bits(v);
}

/* ------------------------------------------------------------------ */
/* Group quantisation and record packing                               */
/* ------------------------------------------------------------------ */
/* ------------------------------------------------------------------ */
/* Floating-point class codecs (the ThinKV page, Metodologia, TBQ: FP8 or NVFP4 */
/* for Reasoning tokens, ternary for Transition tokens).                          */
/* ------------------------------------------------------------------ */

/* FP8 E4M3 in its "fn" form (OCP 8-bit floating point): sign, 4 exponent bits
 * (bias 7), 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite
 * value 1.75 * 2^8 = 448, subnormals m/8 * 2^-6. */
double orc_e4m3_decode(uint8_t code) {
    const int sg = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return sg ? -v : v;
}

/* Nearest E4M3 value, ties to an even mantissa; magnitudes at or above 448
 * saturate to 448 (the format has no infinity); NaN encodes as 0x7F. */
uint8_t orc_e4m3_encode(float xf) {
    if (isnan(xf)) return 0x7F;
    const uint8_t sg = signbit(xf) ? 0x80 : 0x00;
    const double a = fabs((double)xf);
    if (a >= 448.0) return sg | 0x7E;
    if (a == 0.0) return sg;
    int E;
    frexp(a, &E);                                  /* a = f 2^E, f in [0.5, 1) */
    const int ex = a < ldexp(1.0, -6) ? -6 : E - 1;   /* binade (subnormals: -6) */
    const double q = ldexp(1.0, ex - 3);           /* spacing of the binade */
    const double r = a / q, fl = floor(r), fr = r - fl;
    const double n = (fr > 0.5 || (fr == 0.5 && fmod(fl, 2.0) != 0.0)) ? fl + 1.0 : fl;
    const double v = n * q;                        /* <= 448: a < 448 and 448 is on the grid */
    if (v == 0.0) return sg;
    int E2;
    frexp(v, &E2);
    const int e2 = E2 - 1;
    if (e2 < -6) return sg | (uint8_t)(v / ldexp(1.0, -9));          /* subnormal */
    const int m = (int)((v / ldexp(1.0, e2) - 1.0) * 8.0);
    return sg | (uint8_t)(((e2 + 7) << 3) | m);
}

/* Smallest E4M3 value >= y > 0 (saturated at 448). */
uint8_t orc_e4m3_round_up(float y) {
    if (!(y > 0.0f)) return 0x00;
    if ((double)y >= 448.0) return 0x7E;
    uint8_t c = orc_e4m3_encode(y);
    if (orc_e4m3_decode(c) < (double)y) c = (uint8_t)(c + 1);   /* positive codes are ordered */
    return c;
}

/* FP4 E2M1 (the element type of NVFP4): bit 3 sign, magnitudes of codes 0..7. */
static const double k_e2m1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_decode(uint8_t code) {
    const double v = k_e2m1[code & 7];
    return (code & 8) ? -v : v;
}

/* Nearest E2M1 value, ties to the even code (even mantissa); saturates at 6. */
uint8_t orc_e2m1_encode(float xf) {
    const uint8_t sg = signbit(xf) ? 8 : 0;
    const double a = fabs((double)xf);
    int k = 7;
    for (int j = 0; j < 7; ++j) {
        const double mid = 0.5 * (k_e2m1[j] + k_e2m1[j + 1]);
        if (a < mid) { k = j; break; }
        if (a == mid) { k = (j % 2 == 0) ? j : j + 1; break; }
    }
    return sg | (uint8_t)k;
}

/* fp16 nearest (ties to even) of an fp32 value, from the directed roundings. */
static uint16_t f16_rn(float x);

/* FP8 class group: scale = smallest fp16 >= amax / 448 (fp32 division); code =
 * E4M3 nearest of x / scale (fp32 division); all codes 0 when amax == 0.  The
 * group's x_hat = decode(code) * scale. */
void orc_quantize_group_fp8(const float *x, int n, uint16_t *scale_h, uint8_t *codes) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const uint16_t sh = orc_f32_to_f16_ru(amax / 448.0f);
    const float sf = (float)orc_f16_to_f64(sh);
    *scale_h = sh;
    for (int i = 0; i < n; ++i) codes[i] = sf == 0.0f ? 0 : orc_e4m3_encode(x[i] / sf);
}

/* NVFP4 block (16 values): scale = smallest E4M3 >= amax / 6 (fp32 division,
 * saturated at 448); code = E2M1 nearest of x / scale (fp32 division); all codes 0
 * when amax == 0. */
void orc_quantize_block_nvfp4(const float *x, int n, uint8_t *scale_e4m3, uint8_t *codes) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const uint8_t sc = orc_e4m3_round_up(amax / 6.0f);
    const float sf = (float)orc_e4m3_decode(sc);
    *scale_e4m3 = sc;
    for (int i = 0; i < n; ++i) codes[i] = sf == 0.0f ? 0 : orc_e2m1_encode(x[i] / sf);
}

/* Ternary group (threshold ternarisation): delta = 0.7 * mean |x|, alpha = mean of
 * |x| over the elements with |x| > delta, scale = fp16 nearest of alpha; code 1 for
 * x > delta, 3 (-1 in two bits) for x < -delta, else 0 (all fp32, sums left to
 * right).  x_hat = {0, +scale, -scale}. */
void orc_quantize_group_ternary(const float *x, int n, uint16_t *scale_h, uint8_t *codes) {
    float sa = 0.0f;
    for (int i = 0; i < n; ++i) sa += fabsf(x[i]);
    const float delta = 0.7f * (sa / (float)n);
    float sb = 0.0f;
    int cnt = 0;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > delta) { sb += fabsf(x[i]); ++cnt; }
    const float alpha = cnt ? sb / (float)cnt : 0.0f;
    *scale_h = f16_rn(alpha);
    for (int i = 0; i < n; ++i) codes[i] = x[i] > delta ? 1 : (x[i] < -delta ? 3 : 0);
}

static uint16_t f16_rn(float x) {
    const uint16_t lo = orc_f32_to_f16_rd(x), hi = orc_f32_to_f16_ru(x);
    if (lo == hi) return lo;
    const double dl = (double)x - orc_f16_to_f64(lo), dh = orc_f16_to_f64(hi) - (double)x;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;   /* tie: the even fp16 */
}

int orc_record_bytes(int bits, int D, int group) {
    if (bits == 16) return 2 * D * 2;
    int ngroups = D / group;
    return 2 * (D * bits / 8) + 4 * ngroups * 2;
}

/* Quantise one group of n fp32 values (exact bf16 values) at `bits`. */
void orc_quantize_group(const float *x, int n, int bits, uint16_t *scale_h,
                        uint16_t *zero_h, uint8_t *codes) {
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    const int qmax = (1 << bits) - 1;
    uint16_t z = orc_f32_to_f16_rd(mn);
    float zf = (float)orc_f16_to_f64(z);
    float range = mx - zf;                 /* fp32, round to nearest even */
    float step = range / (float)qmax;      /* fp32 IEEE division */
    uint16_t s = orc_f32_to_f16_ru(step);
    float sf = (float)orc_f16_to_f64(s);
    *zero_h = z;
    *scale_h = s;
    for (int i = 0; i < n; ++i) {
        if (sf == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float d = x[i] - zf;
        float r = d / sf;
        float q = nearbyintf(r);           /* round half to even (default mode) */
        if (q < 0) q = 0;
        if (q > (float)qmax) q = (float)qmax;
        codes[i] = (uint8_t)q;
    }
}

/* Storage order of a 128-element code block (K or V).  The block is four
 * quarters of 32 elements; quarter q holds 16 pairs of head-dim indices:
 *   K pair p: dims 32*(p/4) + 8*q + 2*(p%4) + {0, 1}
 *   V pair p: dims  8*p     + 2*q           + {0, 1}
 * Each 32-bit word of the quarter holds 32/b elements (b bits each, element e
 * at bits b*e) and 16/b pairs: pair p = w*(16/b) + s of word w puts its lower
 * dim at element s and its upper dim at element s + 16/b (16 bits higher).
 * Returns the head-dim index stored at element i (0..127) of the block. */
static int storage_dim(int is_v, int bits, int i) {
    int q = i / 32, u = i % 32;
    int per_word = 32 / bits, pairs_per_word = 16 / bits;
    int w = u / per_word, e = u % per_word;
    int p = w * pairs_per_word + e % pairs_per_word;
    int hi = e / pairs_per_word;
    if (is_v) return 8 * p + 2 * q + hi;
    return 32 * (p / 4) + 8 * q + 2 * (p % 4) + hi;
}

/* Pack codes (indexed by head dim) in storage order, little-endian within each
 * byte: storage element i at bit bits*(i % (8/bits)) of byte i*bits/8. */
static void pack_codes(const uint8_t *codes, int n, int bits, int is_v, uint8_t *out) {
    int per = 8 / bits;
    memset(out, 0, (size_t)n * bits / 8);
    for (int i = 0; i < n; ++i)
        out[i / per] |= (uint8_t)(codes[storage_dim(is_v, bits, i)] << (bits * (i % per)));
}

static void unpack_codes(const uint8_t *in, int n, int bits, int is_v, uint8_t *codes) {
    int per = 8 / bits;
    int mask = (1 << bits) - 1;
    for (int i = 0; i < n; ++i)
        codes[storage_dim(is_v, bits, i)] = (in[i / per] >> (bits * (i % per))) & mask;
}

static void put_u16(uint8_t *p, uint16_t v) {
    p[0] = (uint8_t)(v & 0xFF);
    p[1] = (uint8_t)(v >> 8);
}

static uint16_t get_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Record layout (all little-endian):
 *   bf16:  [K: D x bf16][V: D x bf16], each block in the storage order above (b = 16)
 *   b-bit: [K codes: D*b/8 bytes][V codes: D*b/8 bytes]  (storage order above)
 *          [K scale x ngroups][K zero x ngroups][V scale x ngroups][V zero x ngroups] (fp16)
 * Groups are 32 consecutive head dims; only the placement of codes is permuted.
 */
void orc_pack_record(int bits, int D, int group, const uint16_t *k, const uint16_t *v,
                     uint8_t *rec) {
    if (bits == 16) {
        for (int i = 0; i < D; ++i) put_u16(rec + 2 * i, k[storage_dim(0, 16, i)]);
        for (int i = 0; i < D; ++i) put_u16(rec + 2 * D + 2 * i, v[storage_dim(1, 16, i)]);
        return;
    }
    int ng = D / group;
    int cb = D * bits / 8;
    uint8_t *meta = rec + 2 * cb;
    uint8_t codes[512];
    float x[512];
    for (int which = 0; which < 2; ++which) {
        const uint16_t *src = which == 0 ? k : v;
        uint8_t allc[512];
        for (int g = 0; g < ng; ++g) {
            uint16_t s, z;
            for (int i = 0; i < group; ++i) x[i] = bf16_to_f32(src[g * group + i]);
            orc_quantize_group(x, group, bits, &s, &z, codes);
            memcpy(allc + g * group, codes, group);
            put_u16(meta + (which * 2 * ng + g) * 2, s);
            put_u16(meta + (which * 2 * ng + ng + g) * 2, z);
        }
        pack_codes(allc, D, bits, which, rec + which * cb);
    }
}

/* Dequantise a record: x_hat = code * scale + zero, evaluated in fp64. */
void orc_unpack_record(int bits, int D, int group, const uint8_t *rec, double *k_hat,
                       double *v_hat) {
    if (bits == 16) {
        for (int i = 0; i < D; ++i) k_hat[storage_dim(0, 16, i)] = bf16_to_f32(get_u16(rec + 2 * i));
        for (int i = 0; i < D; ++i)
            v_hat[storage_dim(1, 16, i)] = bf16_to_f32(get_u16(rec + 2 * D + 2 * i));
        return;
    }
    int ng = D / group;
    int cb = D * bits / 8;
    const uint8_t *meta = rec + 2 * cb;
    uint8_t codes[512];
    for (int which = 0; which < 2; ++which) {
        double *dst = which == 0 ? k_hat : v_hat;
        unpack_codes(rec + which * cb, D, bits, which, codes);
        for (int d = 0; d < D; ++d) {
            int g = d / group;
            double s = orc_f16_to_f64(get_u16(meta + (which * 2 * ng + g) * 2));
            double z = orc_f16_to_f64(get_u16(meta + (which * 2 * ng + ng + g) * 2));
            dst[d] = (double)codes[d] * s + z;
        }
    }
}

/* Record formats: 16 bf16, 8 / 4 / 2 integer codes (above), and the floating-point
 * class codecs 108 FP8 (E4M3), 104 NVFP4 (E2M1, blocks of 16), 102 ternary.  FP
 * records place their 8-, 4- and 2-bit codes in the storage order of the integer
 * records of the same width (storage_dim / pack_codes above):
 *   108: [K codes: D bytes][V codes: D bytes][K scale x ngroups][V scale x ngroups] (fp16)
 *   104: [K codes: D/2 bytes, 4-bit E2M1 fields][V codes]
 *        [K block scales: D/16 bytes (E4M3), block j = dims 16j..16j+15][V block scales]
 *   102: [K codes: D/4 bytes, 2-bit fields: 1 = +1, 3 = -1, 0 = 0][V codes]
 *        [K scale x ngroups][V scale x ngroups] (fp16) */
int orc_record_bytes_fmt(int fmt, int D, int group) {
    const int ng = D / group;
    switch (fmt) {
        case 108: return 2 * D + 4 * ng;
        case 104: return D + 2 * (D / 16);
        case 102: return D / 2 + 4 * ng;
        default: return orc_record_bytes(fmt, D, group);
    }
}

static int class_fmt(const orc_state *st, int c) {
    return (st->codec && st->bits[c] < 16) ? 100 + st->bits[c] : st->bits[c];
}

void orc_pack_record_fmt(int fmt, int D, int group, const uint16_t *k, const uint16_t *v, uint8_t *rec) {
    if (fmt < 100) {
        orc_pack_record(fmt, D, group, k, v, rec);
        return;
    }
    const int ng = D / group;
    float x[512];
    uint8_t codes[512];
    for (int which = 0; which < 2; ++which) {
        const uint16_t *src = which == 0 ? k : v;
        for (int i = 0; i < D; ++i) x[i] = bf16_to_f32(src[i]);
        if (fmt == 108) {
            for (int g = 0; g < ng; ++g) {
                uint16_t sh;
                orc_quantize_group_fp8(x + g * group, group, &sh, codes + g * group);
                put_u16(rec + 2 * D + (which * ng + g) * 2, sh);
            }
            pack_codes(codes, D, 8, which, rec + which * D);
        } else if (fmt == 104) {
            for (int blk = 0; blk < D / 16; ++blk) {
                uint8_t sc;
                orc_quantize_block_nvfp4(x + blk * 16, 16, &sc, codes + blk * 16);
                rec[D + which * (D / 16) + blk] = sc;
            }
            pack_codes(codes, D, 4, which, rec + which * (D / 2));
        } else {   /* 102 */
            for (int g = 0; g < ng; ++g) {
                uint16_t sh;
                orc_quantize_group_ternary(x + g * group, group, &sh, codes + g * group);
                put_u16(rec + D / 2 + (which * ng + g) * 2, sh);
            }
            pack_codes(codes, D, 2, which, rec + which * (D / 4));
        }
    }
}

/* Dequantise a record of any format, in fp64. */
void orc_unpack_record_fmt(int fmt, int D, int group, const uint8_t *rec, double *k_hat, double *v_hat) {
    if (fmt < 100) {
        orc_unpack_record(fmt, D, group, rec, k_hat, v_hat);
        return;
    }
    uint8_t codes[512];
    for (int which = 0; which < 2; ++which) {
        double *dst = which == 0 ? k_hat : v_hat;
        if (fmt == 108) unpack_codes(rec + which * D, D, 8, which, codes);
        else if (fmt == 104) unpack_codes(rec + which * (D / 2), D, 4, which, codes);
        else unpack_codes(rec + which * (D / 4), D, 2, which, codes);
        for (int d = 0; d < D; ++d) {
            const int g = d / group;
            if (fmt == 108) {
                const double sc = orc_f16_to_f64(get_u16(rec + 2 * D + (which * (D / group) + g) * 2));
                dst[d] = orc_e4m3_decode(codes[d]) * sc;
            } else if (fmt == 104) {
                dst[d] = orc_e2m1_decode(codes[d]) * orc_e4m3_decode(rec[D + which * (D / 16) + d / 16]);
            } else {
                const double sc = orc_f16_to_f64(get_u16(rec + D / 2 + (which * (D / group) + g) * 2));
                dst[d] = codes[d] == 1 ? sc : (codes[d] == 3 ? -sc : 0.0);
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Cache operations                                                    */
/* ------------------------------------------------------------------ */
static int n_streams(const orc_state *st) { return st->B * st->Hkv; }

static uint8_t *record_ptr(const orc_state *st, int s, int c, int slot) {
    size_t rb = (size_t)orc_record_bytes_fmt(class_fmt(st, c), st->D, st->group);
    return st->pool[c] + ((size_t)s * st->cap[c] + slot) * rb;
}

/* Append T tokens per stream.  k, v: bf16 [B][Hkv][T][D]; cls, pos: [B][T].
 * Tokens are processed in order; a token at position < n_protect is stored in
 * class 0 (bf16).  Slot: pop the stream's free stack for that class if it is
 * non-empty, else take the next never-used slot; if neither exists the token
 * is dropped and CAPACITY is reported.  (In dense placement the free stack is
 * always empty, so the slot is always the next never-used one.)  A class id > 3 drops the token and
 * reports INVALID.  New table entries start with score 0. */
int orc_append(orc_state *st, const uint16_t *k, const uint16_t *v, const uint8_t *cls,
               const int32_t *pos, int T) {
    int status = ORC_OK;
    const int D = st->D;
    for (int b = 0; b < st->B; ++b)
        for (int h = 0; h < st->Hkv; ++h) {
            int s = b * st->Hkv + h;
            for (int t = 0; t < T; ++t) {
                int32_t p = pos[(size_t)b * T + t];
                int c = p < st->n_protect ? 0 : cls[(size_t)b * T + t];
                if (c < 0 || c > 3) {
                    if (status == ORC_OK) status = ORC_ERR_INVALID;
                    continue;
                }
                int32_t slot;
                int32_t *ft = &st->ft[s * 4 + c], *hw = &st->hw[s * 4 + c];
                if (*ft > 0) {
                    *ft -= 1;
                    slot = st->fs[c][(size_t)s * st->cap[c] + *ft];
                } else if (*hw < st->cap[c]) {
                    slot = *hw;
                    *hw += 1;
                } else {
                    if (status == ORC_OK) status = ORC_ERR_CAPACITY;
                    continue;
                }
                int32_t i = st->n[s * 4 + c]++;
                size_t e = (size_t)s * st->cap[c] + i;
                st->handle[c][e] = slot;
                st->pos[c][e] = p;
                st->score[c][e] = 0.0f;
                size_t off = (((size_t)b * st->Hkv + h) * T + t) * D;
                orc_pack_record_fmt(class_fmt(st, c), D, st->group, k + off, v + off,
                                    record_ptr(st, s, c, slot));
            }
        }
    return status;
}

/* One decode step of attention for every stream s = (b, kv head):
 *   logit[j][t] = softmax_scale * sum_d q[b][kvh*G + j][d] * k_hat[t][d]
 *   p = softmax over all live tokens of the stream (every class);
 *   out[b][kvh*G + j][:] = sum_t p[j][t] * v_hat[t][:]   (fp64, stored fp32)
 *   score[t] += sum_j p[j][t]                          (fp64 add, stored fp32)
 * q: bf16 [B][Hkv*G][D]; out: fp32 [B][Hkv*G][D].  An empty stream gives a zero
 * output.  If p_out is non-NULL it receives p for stream s_dbg in entry order
 * (class 0 entries, then class 1, ...), [G][N]. */
void orc_attend(orc_state *st, const uint16_t *q, float softmax_scale, float *out,
                int s_dbg, double *p_out) {
    const int D = st->D, G = st->G, S = n_streams(st);
    const int Hq = st->Hkv * G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int s = 0; s < S; ++s) {
        int b = s / st->Hkv, kvh = s % st->Hkv;
        int N = 0;
        for (int c = 0; c < 4; ++c) N += st->n[s * 4 + c];
        double *qd = malloc(sizeof(double) * G * D);
        double *logit = malloc(sizeof(double) * G * (N > 0 ? N : 1));
        double *vh = malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * D);
        double *kh = malloc(sizeof(double) * D);
        float **sc = malloc(sizeof(float *) * (N > 0 ? N : 1));
        for (int j = 0; j < G; ++j)
            for (int d = 0; d < D; ++d)
                qd[j * D + d] = bf16_to_f32(q[((size_t)b * Hq + kvh * G + j) * D + d]);
        int t = 0;
        for (int c = 0; c < 4; ++c)
            for (int i = 0; i < st->n[s * 4 + c]; ++i, ++t) {
                size_t e = (size_t)s * st->cap[c] + i;
                orc_unpack_record_fmt(class_fmt(st, c), D, st->group,
                                      record_ptr(st, s, c, st->handle[c][e]), kh, vh + (size_t)t * D);
                sc[t] = &st->score[c][e];
                for (int j = 0; j < G; ++j) {
                    double acc = 0;
                    for (int d = 0; d < D; ++d) acc += qd[j * D + d] * kh[d];
                    logit[(size_t)j * N + t] = acc * (double)softmax_scale;
                }
            }
        double *incr = calloc((size_t)(N > 0 ? N : 1), sizeof(double));
        for (int j = 0; j < G; ++j) {
            double *o = calloc(D, sizeof(double));
            if (N > 0) {
                double m = -INFINITY;
                for (t = 0; t < N; ++t) m = fmax(m, logit[(size_t)j * N + t]);
                double l = 0;
                for (t = 0; t < N; ++t) l += exp(logit[(size_t)j * N + t] - m);
                for (t = 0; t < N; ++t) {
                    double p = exp(logit[(size_t)j * N + t] - m) / l;
                    incr[t] += p;
                    if (p_out && s == s_dbg) p_out[(size_t)j * N + t] = p;
                    for (int d = 0; d < D; ++d) o[d] += p * vh[(size_t)t * D + d];
                }
            }
            for (int d = 0; d < D; ++d)
                out[((size_t)b * Hq + kvh * G + j) * D + d] = (float)o[d];
            free(o);
        }
        for (t = 0; t < N; ++t) *sc[t] = (float)((double)*sc[t] + incr[t]);
        free(incr);
        free(qd); free(logit); free(vh); free(kh); free(sc);
    }
}

/* ------------------------------------------------------------------ */
/* Budgeted top-k eviction + table compaction                          */
/* ------------------------------------------------------------------ */
typedef struct {
    uint32_t skey;  /* order-preserving image of the fp32 score bits */
    int32_t pos;
    int32_t c, i;
} cand_t;

/* Monotone map of fp32 bit patterns onto uint32: a < b as floats (with -0 < +0)
 * iff key(a) < key(b). */
static uint32_t score_key(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

/* Total order: higher score first, then lower position, then lower class,
 * then lower table index. */
static int cand_cmp(const void *pa, const void *pb) {
    const cand_t *a = pa, *b = pb;
    if (a->skey != b->skey) return a->skey > b->skey ? -1 : 1;
    if (a->pos != b->pos) return a->pos < b->pos ? -1 : 1;
    if (a->c != b->c) return a->c < b->c ? -1 : 1;
    if (a->i != b->i) return a->i < b->i ? -1 : 1;
    return 0;
}

/* For every stream: entries with pos < n_protect are always kept; among the
 * others keep the `budget` first under the total order above and evict the
 * rest.  Each class list keeps its surviving entries in their previous order
 * (scores carried over).  The slots of evicted entries are pushed on the
 * class's free stack in reverse table order, so the earliest evicted entry
 * ends on top and is reused first.  budget >= candidates is a no-op.
 * Dense placement instead moves the record of the entry that ends at table
 * index i to slot i, empties the free stack and sets the next never-used slot
 * to the new entry count: a class's live records stay contiguous, in table
 * order. */
static void compact_stream(orc_state *st, int s, uint8_t *evict[4]);

int orc_evict_window(orc_state *st, int budget, int32_t keep_from);

int orc_evict(orc_state *st, int budget) { return orc_evict_window(st, budget, INT32_MAX); }

/* The same eviction with a local window ("DYNTS", section 2.3, local window: the
 * most recently generated tokens are kept for local coherence): entries at
 * positions >= keep_from are kept as well and are not candidates, so the budget
 * applies to the selection window [n_protect, keep_from) only. */
int orc_evict_window(orc_state *st, int budget, int32_t keep_from) {
    if (budget < 0) return ORC_ERR_INVALID;
    const int S = n_streams(st);
    for (int s = 0; s < S; ++s) {
        int N = 0;
        for (int c = 0; c < 4; ++c) N += st->n[s * 4 + c];
        cand_t *cand = malloc(sizeof(cand_t) * (N > 0 ? N : 1));
        int nc = 0;
        for (int c = 0; c < 4; ++c)
            for (int i = 0; i < st->n[s * 4 + c]; ++i) {
                size_t e = (size_t)s * st->cap[c] + i;
                if (st->pos[c][e] < st->n_protect || st->pos[c][e] >= keep_from) continue;
                cand[nc].skey = score_key(st->score[c][e]);
                cand[nc].pos = st->pos[c][e];
                cand[nc].c = c;
                cand[nc].i = i;
                ++nc;
            }
        if (nc > budget) {
            qsort(cand, nc, sizeof(cand_t), cand_cmp);
            uint8_t *evict[4];
            for (int c = 0; c < 4; ++c) evict[c] = calloc(st->n[s * 4 + c] + 1, 1);
            for (int r = budget; r < nc; ++r) evict[cand[r].c][cand[r].i] = 1;
            compact_stream(st, s, evict);
            for (int c = 0; c < 4; ++c) free(evict[c]);
        }
        free(cand);
    }
    return ORC_OK;
}

/* Removes the entries flagged in evict[c][i] from every class list of stream s:
 * each list keeps its surviving entries in their previous order (scores carried
 * over); the slots of evicted entries are pushed on the class's free stack in
 * reverse table order, so the earliest evicted entry ends on top and is reused
 * first.  Dense placement instead moves the record of the entry that ends at
 * table index i to slot i, empties the free stack and sets the next never-used
 * slot to the new entry count. */
static void compact_stream(orc_state *st, int s, uint8_t *evict[4]) {
    for (int c = 0; c < 4; ++c) {
        int n = st->n[s * 4 + c];
        size_t base = (size_t)s * st->cap[c];
        int m = 0;
        for (int i = 0; i < n; ++i) m += evict[c][i];
        int ft0 = st->ft[s * 4 + c];
        int w = 0, r = 0;
        size_t rb = (size_t)orc_record_bytes_fmt(class_fmt(st, c), st->D, st->group);
        uint8_t *moved = st->dense ? malloc(rb * (n - m > 0 ? n - m : 1)) : NULL;
        for (int i = 0; i < n; ++i) {
            if (evict[c][i]) {
                if (!st->dense) st->fs[c][base + ft0 + (m - 1 - r)] = st->handle[c][base + i];
                ++r;
            } else {
                if (st->dense)
                    memcpy(moved + (size_t)w * rb, record_ptr(st, s, c, st->handle[c][base + i]), rb);
                st->handle[c][base + w] = st->handle[c][base + i];
                st->pos[c][base + w] = st->pos[c][base + i];
                st->score[c][base + w] = st->score[c][base + i];
                ++w;
            }
        }
        st->n[s * 4 + c] = w;
        if (st->dense) {
            for (int i = 0; i < w; ++i) {
                memcpy(record_ptr(st, s, c, i), moved + (size_t)i * rb, rb);
                st->handle[c][base + i] = i;
            }
            st->hw[s * 4 + c] = w;
            st->ft[s * 4 + c] = 0;
            free(moved);
        } else {
            st->ft[s * 4 + c] = ft0 + m;
        }
    }
}

/* Thought segment of position p: the last j with seg_start[j] <= p, or -1 when p
 * lies before the first segment (seg_start strictly increasing, nseg of them). */
/* Exact sums of fp32 scores (TAM page, sections 2.B-2.C: w_j is the mean attention
 * score of segment j and delta = c times the stream's mean score; the means are taken
 * of the exact sums).  A finite non-negative fp32 value is m * 2^(b - 149) with m < 2^24
 * and 0 <= b <= 253, so the exact sum of up to 2^32 of them is a 288-bit integer times
 * 2^-149: nine 32-bit digits.  Negative and non-finite values (attention mass never is
 * either) count as 0.  The sum is then rounded to the nearest double (ties to even). */
typedef struct { uint64_t d[9]; } exact_sum;

static void exact_add(exact_sum *a, float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    const uint32_t eb = u >> 23;                  /* sign bit set: eb >= 256 */
    if (u == 0 || eb >= 255) return;
    const uint64_t m = eb ? (uint64_t)((u & 0x7FFFFFu) | 0x800000u) : (uint64_t)(u & 0x7FFFFFu);
    const int b = eb ? (int)eb - 1 : 0;           /* bit of m's lowest bit above 2^-149 */
    const uint64_t x = m << (b % 32);
    a->d[b / 32] += x & 0xFFFFFFFFull;
    a->d[b / 32 + 1] += x >> 32;                  /* b / 32 <= 7 */
}

static void exact_merge(exact_sum *a, const exact_sum *b) {
    for (int i = 0; i < 9; ++i) a->d[i] += b->d[i];
}

static double exact_value(const exact_sum *a) {
    uint32_t dig[11];
    uint64_t carry = 0;
    for (int i = 0; i < 9; ++i) {
        const uint64_t t = a->d[i] + carry;       /* digits below 2^64 - 2^32: no overflow */
        dig[i] = (uint32_t)t;
        carry = t >> 32;
    }
    dig[9] = (uint32_t)carry;
    dig[10] = (uint32_t)(carry >> 32);
    int top = 10;
    while (top >= 0 && dig[top] == 0) --top;
    if (top < 0) return 0.0;
    /* the 64 bits below the leading one of the 96-bit window dig[top..top-2], the bits
     * under them folded into bit 0 (sticky), converted with one rounding */
    const uint64_t w2 = dig[top], w1 = top >= 1 ? dig[top - 1] : 0, w0 = top >= 2 ? dig[top - 2] : 0;
    int sticky = 0;
    for (int i = 0; i < top - 2; ++i) sticky |= dig[i] != 0;
    int lz = 0;
    while (!((w2 << lz) & 0x80000000ull)) ++lz;
    uint64_t t = ((w2 << 32) | w1) << lz;
    if (lz) t |= w0 >> (32 - lz);
    if (((w0 << lz) & 0xFFFFFFFFull) != 0 || sticky) t |= 1;
    return ldexp((double)t, 32 - lz + 32 * (top - 2) - 149);
}

double orc_sum_f32_exact(const float *v, int n) {
    exact_sum a;
    memset(&a, 0, sizeof(a));
    for (int i = 0; i < n; ++i) exact_add(&a, v[i]);
    return exact_value(&a);
}

static int segment_of(const int32_t *seg_start, int nseg, int32_t p) {
    int j = -1;
    for (int k = 0; k < nseg && seg_start[k] <= p; ++k) j = k;
    return j;
}

/* Segment-level eviction.  Row b of the segment arrays (stride max_seg) lists the
 * thought segments of batch row b: segment j starts at seg_start[j] and ends where
 * segment j + 1 starts (the last one is open), its tokens are stored in class
 * seg_label[j], and seg_keep[j] is its retention (-1: keep all).  For every stream
 * (b, kv head): an entry is kept when its position is below n_protect, lies before
 * the first segment, or its class differs from its segment's label; the other
 * entries of segment j are ranked by (score desc, position asc, table index asc)
 * and the first seg_keep[j] of them are kept.  The tables are then compacted as
 * by orc_evict. */
int orc_evict_segments(orc_state *st, const int32_t *seg_start, const uint8_t *seg_label,
                       const int32_t *seg_keep, const int32_t *nseg, int max_seg) {
    if (max_seg < 0) return ORC_ERR_INVALID;
    const int S = n_streams(st);
    for (int s = 0; s < S; ++s) {
        const int b = s / st->Hkv;
        const int ns = nseg[b] < 0 ? 0 : (nseg[b] > max_seg ? max_seg : nseg[b]);
        const int32_t *starts = seg_start + (size_t)b * max_seg;
        const uint8_t *labels = seg_label + (size_t)b * max_seg;
        const int32_t *keeps = seg_keep + (size_t)b * max_seg;
        uint8_t *evict[4];
        int any = 0;
        for (int c = 0; c < 4; ++c) evict[c] = calloc(st->n[s * 4 + c] + 1, 1);
        for (int j = 0; j < ns; ++j) {
            if (keeps[j] < 0) continue;
            const int c = labels[j];
            if (c < 0 || c > 3) continue;
            const size_t base = (size_t)s * st->cap[c];
            const int n = st->n[s * 4 + c];
            cand_t *cand = malloc(sizeof(cand_t) * (n > 0 ? n : 1));
            int nc = 0;
            for (int i = 0; i < n; ++i) {
                const int32_t p = st->pos[c][base + i];
                if (p < st->n_protect || segment_of(starts, ns, p) != j) continue;
                cand[nc].skey = score_key(st->score[c][base + i]);
                cand[nc].pos = p;
                cand[nc].c = c;
                cand[nc].i = i;
                ++nc;
            }
            if (nc > keeps[j]) {
                qsort(cand, nc, sizeof(cand_t), cand_cmp);
                for (int r = keeps[j]; r < nc; ++r) evict[c][cand[r].i] = 1;
                any = 1;
            }
            free(cand);
        }
        if (any) compact_stream(st, s, evict);
        for (int c = 0; c < 4; ++c) free(evict[c]);
    }
    return ORC_OK;
}

/* Thought-aware budget allocation with pivotal-token protection (page "Compactacao
 * de Cache KV Consciente do Pensamento ... (TAM)", sections 2.B and 2.C), as a
 * selection policy over the accumulated scores.  For every stream (b, kv head), with
 * the segments of batch row b as in orc_evict_segments (entries before the first
 * segment, protected and foreign entries kept): the candidates of segment j are its
 * unprotected entries in its label's class; n_j their number, w_j their mean score;
 * a candidate is pivotal when its score >= delta = c * (mean score of all candidates
 * of the stream) and is kept; the rest of the budget, T' = max(0, budget - pivotal),
 * is split t_j = min(n_j - p_j, floor(T' * (a_j / D) + 1e-9)), a_j = sqrt(w_j) * n_j,
 * D = sum_i a_i (all in fp64; segments with n_j = 0 get nothing; the 1e-9 absorbs the
 * rounding of a share that is an exact integer), and segment j keeps its t_j first
 * non-pivotal candidates under (score desc, position asc, table index asc). */
int orc_evict_tam(orc_state *st, const int32_t *seg_start, const uint8_t *seg_label, const int32_t *nseg,
                  int max_seg, int budget, double c) {
    if (max_seg < 0 || budget < 0 || !(c >= 0.0)) return ORC_ERR_INVALID;
    const int S = n_streams(st);
    for (int s = 0; s < S; ++s) {
        const int b = s / st->Hkv;
        const int ns = nseg[b] < 0 ? 0 : (nseg[b] > max_seg ? max_seg : nseg[b]);
        const int32_t *starts = seg_start + (size_t)b * max_seg;
        const uint8_t *labels = seg_label + (size_t)b * max_seg;
        if (ns == 0) continue;
        int *cnt = calloc(ns, sizeof(int)), *piv = calloc(ns, sizeof(int));
        double *sum = calloc(ns, sizeof(double));
        /* 1. candidates per segment: count and exact score sum; the stream's mean */
        exact_sum tot_x;
        memset(&tot_x, 0, sizeof(tot_x));
        long long ntot = 0;
        for (int j = 0; j < ns; ++j) {
            const int c = labels[j];
            if (c > 3) continue;
            const size_t base = (size_t)s * st->cap[c];
            exact_sum seg;
            memset(&seg, 0, sizeof(seg));
            for (int i = 0; i < st->n[s * 4 + c]; ++i) {
                const int32_t p = st->pos[c][base + i];
                if (p < st->n_protect || segment_of(starts, ns, p) != j) continue;
                cnt[j] += 1;
                exact_add(&seg, st->score[c][base + i]);
            }
            sum[j] = exact_value(&seg);
            exact_merge(&tot_x, &seg);
            ntot += cnt[j];
        }
        if (ntot == 0) { free(cnt); free(piv); free(sum); continue; }
        const double tot = exact_value(&tot_x);
        const double delta = c * (tot / (double)ntot);
        /* 2. pivotal candidates */
        long long P = 0;
        for (int j = 0; j < ns; ++j) {
            const int c = labels[j];
            if (c > 3) continue;
            const size_t base = (size_t)s * st->cap[c];
            for (int i = 0; i < st->n[s * 4 + c]; ++i) {
                const int32_t p = st->pos[c][base + i];
                if (p < st->n_protect || segment_of(starts, ns, p) != j) continue;
                if ((double)st->score[c][base + i] >= delta) piv[j] += 1;
            }
            P += piv[j];
        }
        /* 3. budgets t_j proportional to sqrt(w_j) n_j */
        const long long Tp = budget > P ? budget - P : 0;
        double D = 0.0;
        for (int j = 0; j < ns; ++j)
            if (cnt[j] > 0) D += sqrt(sum[j] / cnt[j]) * cnt[j];
        int32_t *keep = malloc(sizeof(int32_t) * ns);
        for (int j = 0; j < ns; ++j) {
            long long t = 0;
            /* share T' a_j / D with a_j = sqrt(w_j) n_j; 1e-9 keeps a share that is an
             * integer in exact arithmetic from flooring one below it */
            if (cnt[j] > 0 && D > 0.0) t = (long long)floor((double)Tp * (sqrt(sum[j] / cnt[j]) * cnt[j] / D) + 1e-9);
            if (t > cnt[j] - piv[j]) t = cnt[j] - piv[j];
            keep[j] = (int32_t)t;
        }
        /* 4. selection: pivotal kept, then the t_j first of the rest */
        uint8_t *evict[4];
        int any = 0;
        for (int k = 0; k < 4; ++k) evict[k] = calloc(st->n[s * 4 + k] + 1, 1);
        for (int j = 0; j < ns; ++j) {
            const int c = labels[j];
            if (c > 3 || cnt[j] == 0) continue;
            const size_t base = (size_t)s * st->cap[c];
            const int n = st->n[s * 4 + c];
            cand_t *cand = malloc(sizeof(cand_t) * (n > 0 ? n : 1));
            int nc = 0;
            for (int i = 0; i < n; ++i) {
                const int32_t p = st->pos[c][base + i];
                if (p < st->n_protect || segment_of(starts, ns, p) != j) continue;
                if ((double)st->score[c][base + i] >= delta) continue;   /* pivotal: kept */
                cand[nc].skey = score_key(st->score[c][base + i]);
                cand[nc].pos = p;
                cand[nc].c = c;
                cand[nc].i = i;
                ++nc;
            }
            if (nc > keep[j]) {
                qsort(cand, nc, sizeof(cand_t), cand_cmp);
                for (int r = keep[j]; r < nc; ++r) evict[c][cand[r].i] = 1;
                any = 1;
            }
            free(cand);
        }
        if (any) compact_stream(st, s, evict);
        for (int k = 0; k < 4; ++k) free(evict[k]);
        free(keep); free(cnt); free(piv); free(sum);
    }
    return ORC_OK;
}

/* Retention of each of the nseg thought segments of one batch row under the
 * annealing schedule (labels 0 bf16, 1 R, 2 E, 3 T; the last segment is the open
 * one).  k = number of Transition segments after segment j:
 *   open segment, bf16 label, or k = 0          -> -1 (keep all);
 *   R or E segment with k >= 1                   -> r0 >> (k - 1)  (64, 32, 16, ... for r0 = 64);
 *   T segment with k >= 1                        -> t_keep (the safety net). */
int orc_tbe_schedule(const uint8_t *label, int nseg, int r0, int t_keep, int32_t *keep) {
    if (nseg < 0 || r0 < 0 || t_keep < 0) return ORC_ERR_INVALID;
    for (int j = 0; j < nseg; ++j)
        if (label[j] > 3) return ORC_ERR_INVALID;
    for (int j = 0; j < nseg; ++j) {
        int k = 0;
        for (int i = j + 1; i < nseg; ++i) k += label[i] == 3;
        if (j == nseg - 1 || label[j] == 0 || k == 0) keep[j] = -1;
        else if (label[j] == 3) keep[j] = t_keep;
        else keep[j] = (k - 1 >= 31) ? 0 : (r0 >> (k - 1));
    }
    return ORC_OK;
}

/* Attention sparsity of one decode step (the ThinKV page, Metodologia: thought
 * types differ in the sparsity of their attention weights -- Transition the
 * sparsest, then Reasoning, Execution the least).  The page gives no measure;
 * reading used here: for every stream s and query head j, with p the step's
 * softmax over the stream's N live tokens (as orc_attend computes it, scores not
 * touched), sparsity = 1 - H(p) / ln N with H(p) = -sum p ln p (fp64): 0 for
 * uniform attention, 1 for attention on one token; 0 when N < 2.
 * out: [S][G]. */
void orc_attention_sparsity(orc_state *st, const uint16_t *q, float softmax_scale, double *out) {
    const int D = st->D, G = st->G, S = n_streams(st);
    const int Hq = st->Hkv * G;
    for (int s = 0; s < S; ++s) {
        const int b = s / st->Hkv, kvh = s % st->Hkv;
        int N = 0;
        for (int c = 0; c < 4; ++c) N += st->n[s * 4 + c];
        if (N < 2) {
            for (int j = 0; j < G; ++j) out[(size_t)s * G + j] = 0.0;
            continue;
        }
        double *logit = malloc(sizeof(double) * (size_t)G * N);
        double *kh = malloc(sizeof(double) * D), *vh = malloc(sizeof(double) * D);
        int t = 0;
        for (int c = 0; c < 4; ++c)
            for (int i = 0; i < st->n[s * 4 + c]; ++i, ++t) {
                const size_t e = (size_t)s * st->cap[c] + i;
                orc_unpack_record_fmt(class_fmt(st, c), D, st->group, record_ptr(st, s, c, st->handle[c][e]),
                                      kh, vh);
                for (int j = 0; j < G; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d)
                        acc += (double)bf16_to_f32(q[((size_t)b * Hq + kvh * G + j) * D + d]) * kh[d];
                    logit[(size_t)j * N + t] = acc * (double)softmax_scale;
                }
            }
        for (int j = 0; j < G; ++j) {
            const double *x = logit + (size_t)j * N;
            double m = x[0];
            for (int u = 1; u < N; ++u) m = x[u] > m ? x[u] : m;
            double z = 0.0;
            for (int u = 0; u < N; ++u) z += exp(x[u] - m);
            double h = 0.0;   /* H = ln z - sum p (x - m) */
            for (int u = 0; u < N; ++u) h -= exp(x[u] - m) / z * (x[u] - m);
            h += log(z);
            out[(size_t)s * G + j] = 1.0 - h / log((double)N);
        }
        free(logit); free(kh); free(vh);
    }
}

/* Thought type from a sparsity value with thresholds th_r <= th_t (parameters: the
 * page gives none): 3 (Transition) when s >= th_t, 1 (Reasoning) when s >= th_r,
 * else 2 (Execution). */
int orc_classify_sparsity(double s, double th_r, double th_t) {
    return s >= th_t ? 3 : (s >= th_r ? 1 : 2);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
