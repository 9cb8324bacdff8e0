// attention_i8.cu -- tkv_decode_attention for dense record placement on the
// 5th-generation tensor cores with integer operands (tcgen05.mma kind::i8): one
// GQA decode step over the mixed-precision pools with exact integer accumulation
// of the code products, online softmax, and accumulation of each token's attention
// mass into its score (ThinKV decode over the Continuous Thinking block table;
// cumulative attention scores as on the "Back from the Future" page, problem
// statement).
//
// Two kernels.  attn_i8_kernel runs one persistent CTA per SM.  The work of the
// whole step -- every stream's class tables cut into class-homogeneous tiles (64
// records for bf16, 128 for int8 / int4 / int2) -- is laid on one line weighted by
// bytes (+ a fixed cost per tile), and CTA c takes the tiles that start in the c-th
// equal share, so every SM streams the same number of bytes whatever the streams'
// lengths and class mixes.  Each (stream, CTA, warpgroup) leaves one partial
// (running max m, sum l, sum p*(x - m), O); attn_finalize_kernel merges the
// partials of each stream, writes the output and adds p to the scores (from the raw
// logits the first kernel left in an L2-resident scratch).
//
// Memory path.  A tile arrives by TMA in 2-3 boxes whose 32- to 128-byte rows are
// the records' K codes, V codes and scale / zero block, written with the matching
// hardware swizzle: int8 K and V then ARE the MMA operands (K-major and MN-major
// layouts with 128-byte swizzle), with no copy through registers.  int4 / int2 codes
// are widened to bytes in the int8 records' element order: K into tensor memory (the
// A operand of QK), V into a swizzled shared buffer; bf16 keys are the A operand as
// they arrive, bf16 values are regathered into the same element order.
//
// Roles (320 threads): warp 0 issues the TMA boxes and publishes each tile's
// descriptor; warp 1 owns tensor memory and issues the MMAs (one thread); warps 2-5
// and 6-9 are two compute warpgroups taking alternate tiles: thread r widens row r,
// owns row r of the QK accumulators (token r) and of the PV accumulators (head dim
// r of the int8 element order), forms logits, softmax and the PV operand.
//
// Math (per tile):
//   QK  q is written once per stream and warpgroup as three signed 8-bit digits per
//       element, q = (d0 * 2^14 + d1 * 2^7 + d2) * 2^(E_gh - 146), E_gh the exponent
//       of the largest |q| of head h in 32-dim group g (exact for every bf16 within
//       2^12 of that largest value); one kind::i8 MMA chain (A = codes, u8; B = the
//       digits, s8, zero outside the column's group; M 128, K 128) gives
//       c_s = sum_{d in g} code_d * digit_s,d exactly in s32.  Thread t folds
//       x_h = sum_g kscale_g * 2^(E_gh-146) * (c0 2^14 + c1 2^7 + c2) + kzero_g * sum_g(q_h).
//   PV  W_t,(g,h) = p_h,t * vscale_g,t becomes an unsigned integer below 2^22 under a
//       per-tile power-of-two scale; its bytes are u8 columns, so one kind::i8 MMA
//       chain (A = V codes, M = 128 head dims; B = W; K = the tile's tokens) gives
//       exact s32 byte sums, which thread d scales back into its fp32 O; the zero
//       term sum_t p * vzero_g is accumulated by the token threads in fp32.
//   bf16 tiles (protected tokens) use kind::f16 with bf16 operands: q exact, P split
//   into a bf16 high and low part (two columns), so nothing is narrowed.
// The running max only moves (and l, O are rescaled) when a tile exceeds it by
// more than 2^8.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "persist.cuh"

namespace tkv {
namespace {

using namespace attn;

constexpr int kThreads = 320;
constexpr int kStgV = 16384;          // widened V of one tile (128 rows x 128 B)
constexpr int kTmemCols = 512;

__host__ __device__ constexpr int raw_stages(int G) { return G <= 4 ? 4 : 3; }
__host__ __device__ constexpr int ns_of(int G) { return (12 * G + 15) / 16 * 16; }   // QK columns (i8 tiles)
__host__ __device__ constexpr int gs_of(int G) { return 4 * G < 16 ? 16 : 4 * G; }   // PV columns per group
__host__ __device__ constexpr int no_of(int G) { return 4 * gs_of(G); }              // PV columns (i8 tiles)
__host__ __device__ constexpr int w_bytes(int G) { return 128 * no_of(G); }
constexpr uint32_t kSw128 = 2;        // shared-memory descriptor layout: 128-byte swizzle
__host__ __device__ constexpr int qi8_bytes(int G) { return 128 * ns_of(G); }
constexpr int kQbfBytes = 16 * 128 * 2;
__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int q_bytes(int G) { return align1k(qi8_bytes(G) + kQbfBytes + 2 * 4 * kMaxG * 4); }
// dynamic shared memory layout (from a 1024-byte aligned base); per warpgroup wg: the
// widened V, the PV operand W and the query operands
constexpr int kOffRaw = 0;
__host__ __device__ constexpr int off_stg(int G) { return kOffRaw + raw_stages(G) * kRawBytes; }
__host__ __device__ constexpr int off_w(int G) { return off_stg(G) + 2 * kStgV; }
__host__ __device__ constexpr int off_q(int G) { return off_w(G) + 2 * w_bytes(G); }
__host__ __device__ constexpr int smem_bytes(int G) { return 1024 + off_q(G) + 2 * q_bytes(G); }
// tensor memory of warpgroup wg: widened K at 256 wg, QK accumulators at 256 wg + 32,
// PV accumulators at 256 wg + 128
__host__ __device__ constexpr uint32_t col_a(int wg) { return 256u * wg; }
__host__ __device__ constexpr uint32_t col_s(int wg) { return 256u * wg + 32u; }
__host__ __device__ constexpr uint32_t col_o(int wg) { return 256u * wg + 128u; }

// ------------------------------------------------------------ tcgen05 / TMA wrappers
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
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: lbo / sbo in bytes, layout 0 = no swizzle, 2 = 128B swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout = 0) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
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
// A in tensor memory
__device__ __forceinline__ void mma_i8_tmem(uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d), "r"(a), "l"(b), "r"(id),
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
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}


// ------------------------------------------------------------ widening to the int8 element order
// All classes are brought to the element order of the int8 records (tkv.h: quarters of
// 32-bit words, word w of quarter q at byte 32q + 4w, pairs 16 bits apart), so one query
// operand serves every integer class and the PV accumulator rows (= V byte positions)
// mean the same head dim for every class.
//   int4 word (q, w) of a code block (nibbles n0..n7) -> int8 words (q, 2w), (q, 2w+1):
//     lo = nibbles 0,2,4,6; hi = nibbles 1,3,5,7; (q,2w) = [lo0 hi0 lo2 hi2], (q,2w+1) = [lo1 hi1 lo3 hi3]
//   int2 word (q, w) (fields f0..f15) -> int8 words (q, 4w + m): e_k = field bytes k, k+4, k+8, k+12;
//     m = 0: [e0.0 e1.0 e0.2 e1.2], 1: [e2.0 e3.0 e2.2 e3.2], 2: [e0.1 e1.1 e0.3 e1.3], 3: [e2.1 e3.1 e2.3 e3.3]
// (the same for K and V blocks: both formats store head-dim pair p of quarter q in the
// same place, only the pair -> dim maps of K and V differ, and those are shared).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) { return __byte_perm(a, b, sel); }
__device__ __forceinline__ void sts128(uint8_t *p, uint32_t a, uint32_t b, uint32_t c, uint32_t dd) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, dd);
}

// Row r of a [row][64 B] box with 64-byte swizzle: the 16-byte chunk j of the row.
__device__ __forceinline__ uint4 ld_sw64(const uint8_t *base, int r, int j) {
    return *reinterpret_cast<const uint4 *>(base + r * 64 + 16 * (j ^ ((r >> 1) & 3)));
}
// Row r of a [row][32 B] box with 32-byte swizzle.
__device__ __forceinline__ uint4 ld_sw32(const uint8_t *base, int r, int j) {
    return *reinterpret_cast<const uint4 *>(base + r * 32 + 16 * (j ^ ((r >> 2) & 1)));
}
// Row r of a [row][128 B] box with 128-byte swizzle.
__device__ __forceinline__ uint4 ld_sw128(const uint8_t *base, int r, int j) {
    return *reinterpret_cast<const uint4 *>(base + r * 128 + 16 * (j ^ (r & 7)));
}
__device__ __forceinline__ void st_sw128(uint8_t *base, int r, int j, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    *reinterpret_cast<uint4 *>(base + r * 128 + 16 * (j ^ (r & 7))) = make_uint4(a, b, c, d);
}

// 32 int8-order words (128 bytes) of an int4 code block held as row r of a 64B-swizzled box.
__device__ __forceinline__ void widen_i4(const uint8_t *box, int r, uint32_t (&o)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = ld_sw64(box, r, q);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t lo = w4[w] & 0x0F0F0F0Fu, hi = (w4[w] >> 4) & 0x0F0F0F0Fu;
            o[8 * q + 2 * w] = prmt(lo, hi, 0x6240);
            o[8 * q + 2 * w + 1] = prmt(lo, hi, 0x7351);
        }
    }
}
// 32 int8-order words of an int2 code block held as row r of a 32B-swizzled box.
__device__ __forceinline__ void widen_i2(const uint8_t *box, int r, uint32_t (&o)[32]) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint4 v = ld_sw32(box, r, j);   // quarters 2j (words x, y) and 2j + 1 (z, w)
        const uint32_t w2[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int q = 2 * j + i / 2, w = i % 2;
            const uint32_t x = w2[i];
            const uint32_t e0 = x & 0x03030303u, e1 = (x >> 2) & 0x03030303u;
            const uint32_t e2 = (x >> 4) & 0x03030303u, e3 = (x >> 6) & 0x03030303u;
            o[8 * q + 4 * w + 0] = prmt(e0, e1, 0x6240);
            o[8 * q + 4 * w + 1] = prmt(e2, e3, 0x6240);
            o[8 * q + 4 * w + 2] = prmt(e0, e1, 0x7351);
            o[8 * q + 4 * w + 3] = prmt(e2, e3, 0x7351);
        }
    }
}
// 32 int8-order words -> row r of a [row][128 B] 128B-swizzled buffer (chunk j = words 4j..4j+3)
__device__ __forceinline__ void store_row_sw128(uint8_t *buf, int r, const uint32_t (&o)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) st_sw128(buf, r, j, o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}
// bf16 V of row r (two 128B-swizzled atoms of 64 rows) regathered into the int8 element
// order, half `a` (positions 64a .. 64a + 63): output word u (positions 2u, 2u + 1) of
// quarter q = u / 16, word w8 = (u % 16) / 2 takes the low (u even) or high (u odd)
// halves of bf16 words (q, 2 w8) and (q, 2 w8 + 1) (bf16 word (q, w) sits at byte
// 64 q + 4 w of the value block).  Output chunk c (8 positions) of atom a of the
// staged buffer: row r, chunk c ^ (r % 8).
__device__ __forceinline__ void regather_bf16_v(const uint8_t *vbox, uint8_t *stg, int r, int a) {
    // the atom a of the value block holds quarters 2a, 2a + 1 (bytes 128 a .. 128 a + 127)
    uint32_t w[2][16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 v = ld_sw128(vbox + a * 8192, r, j);   // bytes 16 j.. of the atom: quarter 2a + j/4
        w[j / 4][4 * (j % 4)] = v.x; w[j / 4][4 * (j % 4) + 1] = v.y;
        w[j / 4][4 * (j % 4) + 2] = v.z; w[j / 4][4 * (j % 4) + 3] = v.w;
    }
    uint8_t *dst = stg + a * 8192;
#pragma unroll
    for (int c = 0; c < 8; ++c) {   // output chunk c holds words u = 32a + 4c .. + 3
        uint32_t ow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int u = 32 * a + 4 * c + i;
            const int ql = (u / 16) - 2 * a, w8 = (u % 16) / 2;
            ow[i] = prmt(w[ql][2 * w8], w[ql][2 * w8 + 1], (u & 1) ? 0x7632 : 0x5410);
        }
        st_sw128(dst, r, c, ow[0], ow[1], ow[2], ow[3]);
    }
}

// Head dim of position m (0..127) of an int8 K / V block (tkv.h element order).
__device__ __forceinline__ int dim_of_k8(int m) {
    const int q = m >> 5, w = (m & 31) >> 2, e = m & 3;
    return 32 * (w >> 1) + 8 * q + 4 * (w & 1) + ((e & 1) << 1) + (e >> 1);
}
__device__ __forceinline__ int dim_of_v8(int m) {
    const int q = m >> 5, w = (m & 31) >> 2, e = m & 3;
    return 16 * w + 8 * (e & 1) + 2 * q + (e >> 1);
}
// Position of head dim d in an int8 K block (inverse of dim_of_k8) and of bf16 K.
__device__ __forceinline__ int pos_k8(int d) {
    const int g = d >> 5, q = (d >> 3) & 3, o = d & 7;
    const int w = 2 * g + (o >> 2), e = ((o & 1) << 1) | ((o >> 1) & 1);
    return 32 * q + 4 * w + e;
}
__device__ __forceinline__ int pos_kbf(int d) {
    const int g = d >> 5, q = (d >> 3) & 3, o = d & 7;
    return 32 * q + 8 * g + o;
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

template <int G>
struct QConst {   // per-stream constants of the query operand, in shared memory
    float a[4][kMaxG];      // 2^(E_gh - 146): weight of one unit of the digit combination
    float qsum[4][kMaxG];   // sum over group g of head h's (digit-exact) query
};


// ------------------------------------------------------------ the attention kernel
__device__ __forceinline__ bool wg_any(int id, bool pred) {   // OR of pred over the 128 threads of a warpgroup
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, 128, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)pred), "r"(id)
                 : "memory");
    return r != 0;
}
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t *r) {
    if constexpr (N >= 16) {
#pragma unroll
        for (int i = 0; i < N; i += 16) tmem_ld16(taddr + i, r + i);
    } else if constexpr (N == 8) {
        tmem_ld8(taddr, r);
    } else {
        static_assert(N == 4, "column count");
        tmem_ld4(taddr, r);
    }
}

template <int G, bool STATS>
__global__ void __launch_bounds__(kThreads, 1)
    attn_i8_kernel(const __grid_constant__ Dev d, const __grid_constant__ I8Maps maps,
                   const __nv_bfloat16 *__restrict__ q, float xscale) {
    constexpr int NS = ns_of(G);
    constexpr int NO = no_of(G);
    constexpr int GS = gs_of(G);
    constexpr int R = raw_stages(G);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_raw_full[R], bar_raw_empty[R];
    __shared__ __align__(8) uint64_t bar_kready[2], bar_s_full[2], bar_w_full[2], bar_o_full[2], bar_mma_done;
    __shared__ uint32_t tmem_base;
    __shared__ SharedPlan pl;
    __shared__ uint32_t xred[2][2][4][kMaxG + 4];   // [wg][parity][warp]: tile max keys per head, v-scale max keys
    __shared__ float fred[2][4][6 * kMaxG];         // segment flush reductions
    __shared__ float zsum[2][4][kMaxG];             // reduced zero-term sums of the segment being flushed
    __shared__ uint32_t err_timeout;
    __shared__ TileDesc desc[kDescRing];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x, ncta = gridDim.x;

    // ---- set-up (independent of the append, so before the dependency wait)
    if (warp == 1) tmem_alloc(smem_addr(&tmem_base), kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < R; ++i) {
            mbar_init_n(smem_addr(&bar_raw_full[i]), 1);
            mbar_init_n(smem_addr(&bar_raw_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init_n(smem_addr(&bar_kready[i]), 4);
            mbar_init_n(smem_addr(&bar_s_full[i]), 1);
            mbar_init_n(smem_addr(&bar_w_full[i]), 4);
            mbar_init_n(smem_addr(&bar_o_full[i]), 1);
        }
        mbar_init_n(smem_addr(&bar_mma_done), 1);
        err_timeout = 0;
        mbar_init_fence();
    }
    if (warp == 0 && lane == 0) prefetch_maps(maps);
    // query operand buffers: the block-diagonal zeros and padding columns stay zero
    for (int i = tid; i < 2 * q_bytes(G) / 16; i += kThreads)
        reinterpret_cast<uint4 *>(sm + off_q(G))[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base;

    grid_dependency_wait();   // the append's counters and records are visible from here
    plan_work<kThreads>(d, pl, cta, ncta);

    bool ok = true;
    const uint32_t smb = smem_addr(sm);

    if (warp == 0) {
        // ================================================= producer
        if (lane == 0) ok = produce_tiles<R>(d, maps, pl, desc, bar_raw_full, bar_raw_empty, smb + kOffRaw, 2);
    } else if (warp == 1) {
        // ================================================= MMA issuer
        // Two independent in-order streams: QK(kq) once its warpgroup has the tile ready,
        // PV(kpv) once that warpgroup has written W; whichever is ready is issued, so
        // neither warpgroup waits on the other's progress.  QK(k) always precedes PV(k)
        // (W needs the logits).  Descriptors stay in the ring until the tile's PV is
        // issued (the producer reuses a ring slot only 16 tiles later, after the PV of
        // an even later tile).
        if (lane == 0) {
            // descriptor templates (start address 0): a descriptor is template | (address >> 4)
            const uint64_t dA = sdesc(0, 16, 1024, kSw128);     // tiles and staged values, 128B swizzle
            const uint64_t dVb = sdesc(0, 8192, 1024, kSw128);  // staged bf16 values (two 64-dim atoms)
            const uint64_t dQi = sdesc(0, NS * 16, 128);        // query digits
            const uint64_t dQb = sdesc(0, 256, 128);            // bf16 query
            const uint64_t dWi = sdesc(0, 128, 2048);           // W, integer columns
            const uint64_t dWb = sdesc(0, 128, 1024);           // W, bf16 columns
            auto at = [](uint64_t t, uint32_t addr) { return t | (uint64_t)(addr >> 4); };
            int kq = 0, kpv = 0;
            bool q_done = false;
            long long t_idle = 0;
            while (ok) {
                bool progress = false;
                if (!q_done && mbar_test(smem_addr(&bar_kready[kq & 1]), (uint32_t)((kq >> 1) & 1))) {
                    const TileDesc td = desc[kq % kDescRing];
                    progress = true;
                    if (td_end(td)) {
                        q_done = true;
                    } else {
                        tc_fence_after();
                        const int wg = kq & 1, tc = td_c(td);
                        const uint32_t raw = smb + kOffRaw + (kq % R) * kRawBytes;
                        const uint32_t qb = smb + off_q(G) + wg * q_bytes(G);
                        const uint32_t dcol = tb + col_s(wg);
                        if (tc == 0) {
                            const uint32_t bq = qb + qi8_bytes(G);
#pragma unroll
                            for (int ks = 0; ks < 8; ++ks)
                                mma_f16(dcol, at(dA, raw + (ks >> 2) * 8192 + (ks & 3) * 32), at(dQb, bq + ks * 512),
                                        idesc(1, 1, 1, 0, 0, 16), ks > 0);
                        } else if (tc == 1) {
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_i8(dcol, at(dA, raw + ks * 32), at(dQi, qb + ks * 32 * NS), idesc(2, 0, 1, 0, 0, NS), ks > 0);
                        } else {
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_i8_tmem(dcol, tb + col_a(wg) + 8 * ks, at(dQi, qb + ks * 32 * NS), idesc(2, 0, 1, 0, 0, NS),
                                            ks > 0);
                        }
                        mma_commit(smem_addr(&bar_s_full[wg]));
                        ++kq;
                    }
                }
                if (kpv < kq && mbar_test(smem_addr(&bar_w_full[kpv & 1]), (uint32_t)((kpv >> 1) & 1))) {
                    tc_fence_after();
                    const TileDesc tp = desc[kpv % kDescRing];
                    const int wg = kpv & 1, cp = td_c(tp);
                    const uint32_t raw = smb + kOffRaw + (kpv % R) * kRawBytes;
                    const uint32_t stg = smb + off_stg(G) + wg * kStgV;
                    const uint32_t bw = smb + off_w(G) + wg * w_bytes(G);
                    const uint32_t dcol = tb + col_o(wg);
                    if (cp == 0) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_f16(dcol, at(dVb, stg + ks * 2048), at(dWb, bw + ks * 256), idesc(1, 1, 1, 1, 1, 16), ks > 0);
                    } else {
                        const uint32_t av = cp == 1 ? raw + v_off(1) : stg;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_i8(dcol, at(dA, av + ks * 4096), at(dWi, bw + ks * 512), idesc(2, 0, 0, 1, 1, NO), ks > 0);
                    }
                    mma_commit(smem_addr(&bar_o_full[wg]));
                    mma_commit(smem_addr(&bar_raw_empty[kpv % R]));
                    ++kpv;
                    progress = true;
                }
                if (q_done && kpv == kq) break;
                if (progress) {
                    t_idle = 0;
                } else {
                    // bounded: a second without a ready operand is a timeout
                    const long long now = clock64();
                    if (t_idle == 0) t_idle = now;
                    else if (now - t_idle > kWaitCycles) ok = false;
                }
            }
            // every MMA issued has completed before tensor memory is released
            mma_commit(smem_addr(&bar_mma_done));
            if (!mbar_wait_sleep(smem_addr(&bar_mma_done), 0u)) ok = false;
        }
    } else {
        // ================================================= compute warpgroups (warps 2-5, 6-9)
        const int wg = (warp - 2) >> 2;
        const int wq = warp & 3;                         // lane quarter of tensor memory
        const int r = 32 * wq + lane;                    // token row (QK), element m of the V order (PV), dim (q)
        const int gr = (r & 31) >> 3;                    // group of the head dim at V position r
        const int bid = 1 + wg;                          // named barrier of the warpgroup
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        uint8_t *qbuf = sm + off_q(G) + wg * q_bytes(G);
        QConst<G> *qc = reinterpret_cast<QConst<G> *>(qbuf + qi8_bytes(G) + kQbfBytes);
        uint8_t *stg = sm + off_stg(G) + wg * kStgV;
        uint8_t *wbuf = sm + off_w(G) + wg * w_bytes(G);
        float m[G], l[G], e[G], z[4][G], oacc[G];
        float alpha_prev[G], bp_prev[G], bv_prev = 1.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = kNoMax; l[h] = 0.f; e[h] = 0.f; oacc[h] = 0.f; alpha_prev[h] = 1.f; bp_prev[h] = 1.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) z[g][h] = 0.f;
        }
        int cur_s = -1, c_prev = 0, kp = -1;
        bool cta_empty = false;
        // an empty partial (l = 0: the merge skips it) in this warpgroup's slot of stream s
        auto write_empty = [&](int s) {
            float *part = d.part + (size_t)(2 * (s + cta) + wg) * part_floats(G);
            part[r] = kNoMax;
            part[G + r] = 0.f;
            part[2 * G + r] = 0.f;
        };

        // add the PV result of own tile kp (class cp) to O
        auto o_accumulate = [&](int kpp, int cp) {
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_o_full[wg]), (uint32_t)((kpp >> 1) & 1));
            tc_fence_after();
            if (cp == 0) {
                uint32_t dv[16];
                tmem_ld16(tb + lane_off + col_o(wg), dv);
                tc_wait_ld();
#pragma unroll
                for (int h = 0; h < G; ++h)
                    oacc[h] = fmaf(oacc[h], alpha_prev[h], __uint_as_float(dv[h]) + __uint_as_float(dv[G + h]));
            } else {
                uint32_t sel[4 * G];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t dv[4 * G];
                    tmem_ldn<4 * G>(tb + lane_off + col_o(wg) + g * GS, dv);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4 * G; ++i) sel[i] = g == gr ? dv[i] : (g == 0 ? 0u : sel[i]);
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float v = fmaf(__int2float_rn((int32_t)sel[4 * h + 2]), 65536.f,
                                         fmaf(__int2float_rn((int32_t)sel[4 * h + 1]), 256.f,
                                              __int2float_rn((int32_t)sel[4 * h])));
                    oacc[h] = fmaf(oacc[h], alpha_prev[h], v * bp_prev[h] * bv_prev);
                }
            }
            tc_fence_before();
        };
        // write the partial of segment s_old: (m, l, e) per head and O + zero term
        auto flush = [&](int s_old) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float vl = l[h], ve = e[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    vl += __shfl_xor_sync(kFull, vl, o);
                    if (STATS) ve += __shfl_xor_sync(kFull, ve, o);
                }
                if (lane == 0) { fred[wg][wq][h] = vl; fred[wg][wq][G + h] = ve; }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float vz = z[g][h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) vz += __shfl_xor_sync(kFull, vz, o);
                    if (lane == 0) fred[wg][wq][2 * G + g * G + h] = vz;
                }
            }
            named_sync(bid, 128);
            float *part = d.part + (size_t)(2 * (s_old + cta) + wg) * part_floats(G);
            if (r < 6 * G) {
                const float v = fred[wg][0][r] + fred[wg][1][r] + fred[wg][2][r] + fred[wg][3][r];
                if (r < G) part[G + r] = v;                                 // l
                else if (r < 2 * G) part[2 * G + (r - G)] = v;              // e
                else zsum[wg][(r - 2 * G) / G][(r - 2 * G) % G] = v;        // zero term
            }
            if (r == 0) {
#pragma unroll
                for (int h = 0; h < G; ++h) part[h] = m[h];
            }
            named_sync(bid, 128);
            const int dim = dim_of_v8(r);
#pragma unroll
            for (int h = 0; h < G; ++h) part[3 * G + h * kD + dim] = oacc[h] + zsum[wg][gr][h];
        };

        for (int k = wg;; k += 2) {
            const int slot = k % R;
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_raw_full[slot]), (uint32_t)((k / R) & 1));
            const TileDesc td = desc[k % kDescRing];
            const bool end = td_end(td);
            if (k == wg) cta_empty = end && (wg == 0 || td_end(desc[0]));
            // a stream whose tiles in this CTA all went to the other warpgroup (the tile
            // between this warpgroup's previous tile and this one) gets an empty partial
            if (ok && k >= 1 && r < G) {
                const TileDesc to = desc[(k - 1) % kDescRing];
                if (!td_end(to) && to.s != cur_s && (end || to.s != td.s)) write_empty(to.s);
            }
            if (wg_any(bid, end || !ok)) {
                if (end && ok) {   // let the MMA issuer see the end
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&bar_kready[wg]));
                }
                break;
            }
            const int tcls = td_c(td), nr = td_nr(td);
            const uint8_t *raw = sm + kOffRaw + slot * kRawBytes;
            const bool newseg = td.s != cur_s;
            if (newseg) {
                // ---- query operands of stream td.s: thread r takes head dim r (group wq)
                const int bb = td.s / d.Hkv, kvh = td.s - bb * d.Hkv;
                const uint16_t *qrow =
                    reinterpret_cast<const uint16_t *>(q) + ((size_t)bb * d.Hkv * G + (size_t)kvh * G) * kD;
                const int kb = pos_kbf(r), m8 = pos_k8(r);
                uint32_t qraw[G];
#pragma unroll
                for (int h = 0; h < G; ++h) qraw[h] = qrow[h * kD + r];   // every load in flight at once
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const uint32_t bits = qraw[h];
                    *reinterpret_cast<uint16_t *>(qbuf + qi8_bytes(G) + (kb / 8) * 256 + (h / 8) * 128 + (h % 8) * 16 +
                                                  (kb % 8) * 2) = (uint16_t)bits;
                    // digits: q = v * 2^(Emax - 146) with v = m * 2^(e - Emax + 12) (rounded)
                    const int ex = (int)((bits >> 7) & 0xff);
                    const int mant = ex == 0 ? (int)(bits & 0x7f) : (int)((bits & 0x7f) | 0x80);
                    const int e_eff = ex == 0 ? 1 : ex;
                    const int emax = (int)__reduce_max_sync(kFull, (unsigned)e_eff);
                    const int sh = e_eff - emax + 12;
                    int v;
                    if (sh >= 0) v = mant << sh;
                    else if (sh > -9) v = (mant + (1 << (-sh - 1))) >> (-sh);
                    else v = 0;
                    if (bits & 0x8000) v = -v;
                    const int d2 = ((v + 64) & 127) - 64;
                    const int v1 = (v - d2) >> 7;
                    const int d1 = ((v1 + 64) & 127) - 64;
                    const int d0 = (v1 - d1) >> 7;
                    const int dg[3] = {d0, d1, d2};
#pragma unroll
                    for (int s3 = 0; s3 < 3; ++s3) {
                        const int n = wq * 3 * G + s3 * G + h;
                        qbuf[(m8 / 16) * (NS * 16) + (n / 8) * 128 + (n % 8) * 16 + (m8 % 16)] = (uint8_t)(int8_t)dg[s3];
                    }
                    const int vsum = __reduce_add_sync(kFull, v);
                    if (lane == 0) {
                        const int ea = emax - 146;
                        const float a = ea >= -126 ? pow2f(ea) : pow2f(ea + 64) * 5.421010862427522e-20f;   // 2^-64
                        qc->a[wq][h] = a;
                        qc->qsum[wq][h] = (float)vsum * a;
                    }
                }
            }
            // ---- keys of int4 / int2 tiles: widened into tensor memory (row r = token r)
            if (tcls >= 2) {
                uint32_t o[32];
                if (tcls == 2) widen_i4(raw, r, o);
                else widen_i2(raw, r, o);
                tmem_st16(tb + lane_off + col_a(wg), o);
                tmem_st16(tb + lane_off + col_a(wg) + 16, o + 16);
                tc_wait_st();
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bar_kready[wg]));
            if (r == 0) {
                if (td_first(td)) d.seg_lo[td.s] = cta;
                if (td_last(td)) d.seg_hi[td.s] = cta;
            }

            // ---- O of the previous own tile: at a stream change now (the segment's partial
            //      is written); otherwise after this tile's logits, so that the PV of the
            //      previous tile runs meanwhile.  Its values (staged) and W must be read
            //      before this tile overwrites them.
            const bool o_late = kp >= 0 && !newseg;
            if (kp >= 0 && newseg) {
                o_accumulate(kp, c_prev);
                flush(cur_s);
#pragma unroll
                for (int h = 0; h < G; ++h) oacc[h] = 0.f;
            }
            if (o_late && tcls != 1 && ok)
                ok = mbar_wait_sleep(smem_addr(&bar_o_full[wg]), (uint32_t)((kp >> 1) & 1));
            if (newseg) {
                cur_s = td.s;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    m[h] = kNoMax; l[h] = 0.f; e[h] = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) z[g][h] = 0.f;
                }
            }

            // ---- values of int4 / int2 / bf16 tiles: widened / regathered into the staged buffer
            if (tcls >= 2) {
                uint32_t o[32];
                if (tcls == 2) widen_i4(raw + v_off(2), r, o);
                else widen_i2(raw + v_off(3), r, o);
                store_row_sw128(stg, r, o);
            } else if (tcls == 0) {
                const int t = r & 63, a = r >> 6;
                if (t < nr) {
                    regather_bf16_v(raw + 16384, stg, t, a);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) st_sw128(stg + a * 8192, t, j, 0u, 0u, 0u, 0u);
                }
            }

            // ---- logits
            if (ok) ok = mbar_wait_sleep(smem_addr(&bar_s_full[wg]), (uint32_t)((k >> 1) & 1));
            tc_fence_after();
            const bool valid = r < nr;
            float x[G];
            float vsc[4] = {0.f, 0.f, 0.f, 0.f}, vze[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t vkey[4] = {0u, 0u, 0u, 0u};
            if (tcls == 0) {
                uint32_t sv[16];
                tmem_ld16(tb + lane_off + col_s(wg), sv);
                tc_wait_ld();
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = valid ? __uint_as_float(sv[h]) * xscale : -INFINITY;
            } else {
                const uint8_t *meta = raw + meta_off(tcls) + 32 * r;
                const uint4 km = *reinterpret_cast<const uint4 *>(meta);
                const uint4 vm = *reinterpret_cast<const uint4 *>(meta + 16);
                const float2 ks01 = __half22float2(u32_as_h2(km.x)), ks23 = __half22float2(u32_as_h2(km.y));
                const float2 kz01 = __half22float2(u32_as_h2(km.z)), kz23 = __half22float2(u32_as_h2(km.w));
                const float2 vs01 = __half22float2(u32_as_h2(vm.x)), vs23 = __half22float2(u32_as_h2(vm.y));
                const float2 vz01 = __half22float2(u32_as_h2(vm.z)), vz23 = __half22float2(u32_as_h2(vm.w));
                const float ks[4] = {ks01.x, ks01.y, ks23.x, ks23.y}, kz[4] = {kz01.x, kz01.y, kz23.x, kz23.y};
                if (valid) {
                    vsc[0] = vs01.x; vsc[1] = vs01.y; vsc[2] = vs23.x; vsc[3] = vs23.y;
                    vze[0] = vz01.x; vze[1] = vz01.y; vze[2] = vz23.x; vze[3] = vz23.y;
                    // v scales are >= 0: their fp16 bits order as integers
                    vkey[0] = vm.x & 0xffffu; vkey[1] = vm.x >> 16; vkey[2] = vm.y & 0xffffu; vkey[3] = vm.y >> 16;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = 0.f;
                constexpr int GPL = G == 8 ? 2 : 4;                       // groups per accumulator load
                constexpr int NL = (GPL * 3 * G + 15) / 16 * 16;
#pragma unroll
                for (int g0 = 0; g0 < 4; g0 += GPL) {
                    uint32_t sv[NL];
                    tmem_ldn<NL>(tb + lane_off + col_s(wg) + g0 * 3 * G, sv);
                    tc_wait_ld();
#pragma unroll
                    for (int gi = 0; gi < GPL; ++gi) {
                        const int g = g0 + gi;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float tsum = fmaf(__int2float_rn((int32_t)sv[gi * 3 * G + h]), 16384.f,
                                                    fmaf(__int2float_rn((int32_t)sv[gi * 3 * G + G + h]), 128.f,
                                                         __int2float_rn((int32_t)sv[gi * 3 * G + 2 * G + h])));
                            x[h] = fmaf(ks[g] * qc->a[g][h], tsum, fmaf(kz[g], qc->qsum[g][h], x[h]));
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = valid ? x[h] * xscale : -INFINITY;
            }
            tc_fence_before();
            // raw logits for the score pass (entry order of the stream)
            if (valid) {
                float *lg = d.logits + ((size_t)td.s * d.ncap + td.oc + td.e + r) * G;
                if constexpr (G == 4) {
                    *reinterpret_cast<float4 *>(lg) = make_float4(x[0], x[1], x[2], x[3]);
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) lg[h] = x[h];
                }
            }
            // tile max per head and v-scale max per group across the warpgroup
            const int par = (k >> 1) & 1;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint32_t mk = __reduce_max_sync(kFull, fkey(x[h]));
                if (lane == 0) xred[wg][par][wq][h] = mk;
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const uint32_t mx = __reduce_max_sync(kFull, vkey[g]);
                if (lane == 0) xred[wg][par][wq][kMaxG + g] = mx;
            }
            named_sync(bid, 128);
            float alpha[G], tmax[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint32_t mk = max(max(xred[wg][par][0][h], xred[wg][par][1][h]),
                                        max(xred[wg][par][2][h], xred[wg][par][3][h]));
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
            if (o_late) o_accumulate(kp, c_prev);
            // ---- W (the B operand of PV) for row r
            float bp_cur[G], bv_cur = 1.f;
            if (tcls == 0) {
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
                float iv[4], ip[G];
                int ev[4], ep[G];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t vk = max(max(xred[wg][par][0][kMaxG + g], xred[wg][par][1][kMaxG + g]),
                                            max(xred[wg][par][2][kMaxG + g], xred[wg][par][3][kMaxG + g]));
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
                const int evr = gr == 0 ? ev[0] : gr == 1 ? ev[1] : gr == 2 ? ev[2] : ev[3];
                bv_cur = pow2f(evr - 22);
                uint32_t wv[4 * G];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float vv = vsc[g] * iv[g];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float wf = (p[h] * ip[h]) * vv;   // in [0, 2^22)
                        wv[g * G + h] = __float_as_uint(wf + 12582912.f) - 0x4B400000u;
                        z[g][h] = fmaf(p[h], vze[g], z[g][h]);
                    }
                }
                // row r: group g's columns start at g * GS; column 4h + byte of a group is byte
                // `byte` of wv[g*G + h]; 16-column chunks 2048 B apart
                uint8_t *dst = wbuf + (r / 8) * 128 + (r % 8) * 16;
                constexpr int CPG = GS / 16;   // chunks per group
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
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bar_w_full[wg]));
#pragma unroll
            for (int h = 0; h < G; ++h) { alpha_prev[h] = alpha[h]; bp_prev[h] = bp_cur[h]; }
            bv_prev = bv_cur;
            c_prev = tcls;
            kp = k;
        }
        if (!wg_any(bid, !ok)) {
            if (kp >= 0) {
                o_accumulate(kp, c_prev);
                flush(cur_s);
            } else if (cta_empty && pl.s0 < d.S && r < G) {
                // no tile starts in this CTA's share, which lies inside stream s0 between
                // two tiles: the merge reads this CTA's slots of s0
                write_empty(pl.s0);
            }
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

int g_bps_i8[kMaxG + 1][2][kMaxDevices] = {};

template <int G, bool STATS>
cudaError_t launch_i8_g(const Dev &d, const I8Maps &maps, const void *q, float scale, float *out, float *sparsity,
                        uint8_t *thought, float th_r, float th_t, long long live_ub, cudaStream_t st,
                        int64_t *launches) {
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
    e = cudaLaunchKernelEx(&cfg, attn_i8_kernel<G, STATS>, d, maps, static_cast<const __nv_bfloat16 *>(q), xscale);
    *launches += 1;
    if (e != cudaSuccess) return e;
    return launch_finalize<G, STATS, 2>(d, out, sparsity, thought, th_r, th_t, ncta, live_ub, st, launches);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

cudaError_t make_i8_maps(const Dev &d, I8Maps *maps) {
    std::memset(maps, 0, sizeof(*maps));
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr);
    if (e != cudaSuccess) return e;
    if (fn == nullptr || qr != cudaDriverEntryPointSuccess) return cudaErrorNotSupported;
    const auto encode = reinterpret_cast<EncodeTiledFn>(fn);
    for (int c = 0; c < 4; ++c) {
        const long long rows = (long long)d.S * d.cap[c];
        if (rows == 0) continue;   // the class holds no records: no tile ever reads it
        if (rows + 128 > (long long)INT32_MAX) return cudaErrorInvalidValue;
        const int rec = rec_of(c);
        if (d.rec[c] != rec) return cudaErrorInvalidValue;
        const cuuint64_t gdim[2] = {(cuuint64_t)rec, (cuuint64_t)rows};
        const cuuint64_t gstride[1] = {(cuuint64_t)rec};
        const cuuint32_t es[2] = {1, 1};
        const CUtensorMapSwizzle sw = c <= 1 ? CU_TENSOR_MAP_SWIZZLE_128B
                                             : c == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
        for (int kind = 0; kind < (c == 0 ? 1 : 2); ++kind)
            for (int small = 0; small < 2; ++small) {
                const cuuint32_t box[2] = {(cuuint32_t)(kind == 0 ? code_box_bytes(c) : 32),
                                           (cuuint32_t)(small ? 16 : rows_of(c))};
                const CUresult r = encode(&maps->m[c][kind][small], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, d.pool[c], gdim,
                                          gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                          kind == 0 ? sw : CU_TENSOR_MAP_SWIZZLE_NONE,
                                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
                if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
            }
    }
    return cudaSuccess;
}

size_t i8_part_bytes(int S, int G) { return (size_t)2 * (S + kNctaMax) * part_floats(G) * sizeof(float); }

cudaError_t launch_attention_i8(const Dev &d, const I8Maps &maps, const void *q, float scale, float *out,
                                float *sparsity, uint8_t *thought, float th_r, float th_t, long long live_ub,
                                cudaStream_t st, int64_t *launches) {
    const bool stats = sparsity != nullptr || thought != nullptr;
#define TKV_I8_CASE(GG)                                                                                             \
    case GG:                                                                                                        \
        return stats ? launch_i8_g<GG, true>(d, maps, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st,   \
                                             launches)                                                              \
                     : launch_i8_g<GG, false>(d, maps, q, scale, out, sparsity, thought, th_r, th_t, live_ub, st,  \
                                              launches);
    switch (d.G) {
        TKV_I8_CASE(1)
        TKV_I8_CASE(2)
        TKV_I8_CASE(4)
        TKV_I8_CASE(8)
        default: return cudaErrorInvalidValue;
    }
#undef TKV_I8_CASE
}

}  // namespace tkv
