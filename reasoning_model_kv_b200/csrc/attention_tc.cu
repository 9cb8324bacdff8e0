// attention_tc.cu -- tkv_decode_attention for dense record placement on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory): one GQA
// decode step over the mixed-precision pools with fused dequantisation, online
// softmax and accumulation of each token's attention mass into its score
// (ThinKV decode; cumulative attention scores as on the "Back from the Future"
// page, problem statement).
//
// Work decomposition.  Stream s = (b, kv head) is processed by a cluster of C
// CTAs of 128 threads; CTA r takes a contiguous range of the stream's entries
// (class 0..3 tables concatenated) cut into class-homogeneous tiles of up to 128
// records (64 for bf16, 112 for int8, so a tile fits a 32 KB stage).  Thread t
// owns row t of every tile: it dequantises its token and owns lane t of the
// tensor-memory accumulators, so the softmax and score work is per thread.
//
// Per tile (dense placement: the tile's records are one contiguous bulk copy,
// two tiles in flight):
//   QK   thread t converts its K codes to f16 (exact integers) and stores them to
//        tensor memory as row t of A [128 x 128 dims].  B = q stacked per group:
//        row g*G + h holds q_h on the dims of group g and 0 elsewhere, so one
//        chain of 8 MMAs (M 128, N 16, K 16) gives S[t][g*G + h] = (k_t . q_h) over
//        group g.  Thread t reads its row and folds the group scales and zeros:
//        x_h = sum_g kscale_g * S_g,h + kzero_g * sum_{d in g} q_h,d.
//   softmax  tile max per head (warp shuffles + shared memory); the reference max
//        moves, and the accumulators are rescaled, only when a tile exceeds it by
//        more than 2^8.  p = exp2(x - m); thread t adds p to l and p * vzero_g to
//        the zero sums z_g,h.
//   PV   B = V codes as f16 [128 tokens x 128 dims] in shared memory (MN-major);
//        A = P' in tensor memory, row g*G + h = p_h * vscale_g over the tile's tokens
//        (written by warp 0 from a shared-memory transpose).  For each group g, 8
//        MMAs (M 128, N 32, K 16) accumulate dims 32g..32g+31 into one 32-column
//        accumulator O, with only rows g*G..g*G+G-1 enabled, so row g*G + h of O
//        holds sum_t p_h,t vscale_g,t code_t,d for the dims of group g.
// bf16 tiles use bf16 operands for QK (q is bf16: exact) and f16 V (exact in the
// f16 range) with vscale 1, vzero 0.
//
// Epilogue: O_h,d = O[g*G + h][d - 32g] + z_g,h; CTA (m, l, O) merged across the
// cluster over DSMEM; scores += sum_h exp2(x - M_h) / L_h from the raw-logit scratch.
#include "attn_common.cuh"

namespace tkv {
namespace {

using namespace attn;

constexpr int kTT = 128;                 // threads = tile rows = tensor-memory lanes
constexpr int kTcStages = 2;
constexpr int kTcStage = 32768;          // >= rows * record bytes of every class
constexpr int kTmemCols = 256;
// tensor-memory columns
constexpr uint32_t kColAK = 0;           // A of QK: [128][64 f16 pairs]
constexpr uint32_t kColS = 64;           // QK accumulators: [128][NS] f32
constexpr uint32_t kColAP = 96;          // A of PV: [128][64 f16 pairs]
constexpr uint32_t kColO = 160;          // PV accumulator: [128][32] f32
// shared memory (dynamic, from a 1024-byte aligned base)
constexpr int kOffStage = 0;                            // [kTcStages][kTcStage] records
constexpr int kOffBV = kOffStage + kTcStages * kTcStage;  // V as f16, MN-major: 32 KB
constexpr int kBVKBlock = 2048;                         // bytes between 8-token blocks (16 dim blocks x 128 B)
constexpr int kOffBQ = kOffBV + 16 * kBVKBlock;         // q stacked, f16 then bf16: 2 x NS x 256 B
__host__ __device__ constexpr int tc_ns(int G) { return 4 * G < 16 ? 16 : 4 * G; }
__host__ __device__ constexpr int off_pbuf(int G) { return kOffBQ + 2 * tc_ns(G) * 256; }
__host__ __device__ constexpr int tc_smem_bytes(int G) { return 1024 + off_pbuf(G) + 4 * G * kTT * 2; }

__host__ __device__ constexpr int tc_rows(int c) { return c == 0 ? 64 : c == 1 ? 112 : 128; }
__host__ __device__ constexpr int tc_rec(int c) { return c == 0 ? 512 : c == 1 ? 288 : c == 2 ? 160 : 96; }

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
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle: lbo / sbo in bytes (multiples of 16).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}

// D[tmem] (+)= A[tmem] . B[smem]^T, kind::f16; rows whose bit is set in mask are left untouched.
__device__ __forceinline__ void mma_tmem_a(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc,
                                           uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(acc), "r"(m0), "r"(m1), "r"(m2), "r"(m3)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Instruction descriptor, kind::f16: f32 accumulator, A/B format (0 f16, 1 bf16),
// B major (0 K, 1 MN), N, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t fmt, uint32_t b_mn, uint32_t n) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (b_mn << 16) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

#define TKV_R8(r, i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), \
                     "r"(r[i + 6]), "r"(r[i + 7])
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {"
        "%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
        "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
        "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
        TKV_R8(r, 0), TKV_R8(r, 8), TKV_R8(r, 16), TKV_R8(r, 24), TKV_R8(r, 32), TKV_R8(r, 40), TKV_R8(r, 48),
        TKV_R8(r, 56)
        : "memory");
}
#undef TKV_R8

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::
            "r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// ------------------------------------------------------------ per-row dequantisation
// The record's code block `blk` (BITS-bit codes of 128 dims, storage order: four
// quarters of 16 dim pairs) as 64 f16x2 words in storage-pair order.
template <int BITS>
__device__ __forceinline__ void codes_to_f16(const uint8_t *blk, uint32_t (&out)[64], uint32_t magic) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t w[BITS];
        const uint8_t *src = blk + 4 * BITS * q4;
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
#define TKV_P(P) out[16 * q4 + (P)] = quarter_pair<BITS, P>(w, magic);
        TKV_P(0) TKV_P(1) TKV_P(2) TKV_P(3) TKV_P(4) TKV_P(5) TKV_P(6) TKV_P(7)
        TKV_P(8) TKV_P(9) TKV_P(10) TKV_P(11) TKV_P(12) TKV_P(13) TKV_P(14) TKV_P(15)
#undef TKV_P
    }
}

// bf16 code block as raw words (bf16 pairs in storage order).
__device__ __forceinline__ void raw_words(const uint8_t *blk, uint32_t (&out)[64]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint4 v = reinterpret_cast<const uint4 *>(blk)[i];
        out[4 * i] = v.x; out[4 * i + 1] = v.y; out[4 * i + 2] = v.z; out[4 * i + 3] = v.w;
    }
}

template <int G>
__global__ void __launch_bounds__(kTT, 1)
    attn_tc_kernel(const __grid_constant__ Dev d, const __nv_bfloat16 *__restrict__ q, float xscale,
                   float *__restrict__ out, int C) {
    constexpr int NS = tc_ns(G);
    constexpr int NR = 4 * G;                  // rows of P' / O in use
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t full_bar[kTcStages];
    __shared__ __align__(8) uint64_t s_bar, o_bar;
    __shared__ uint32_t tmem_base;
    __shared__ float qsum[4][kMaxG];
    __shared__ float wmax[4][kMaxG];
    __shared__ float red[4][5 * kMaxG];
    __shared__ float cta_m[kMaxG], cta_l[kMaxG];
    __shared__ float fac[kMaxCluster][kMaxG];
    __shared__ float gM[kMaxG], gInvL[kMaxG];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = blockIdx.x;
    const int s = blockIdx.y;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

    // ---- set-up: tensor memory, barriers, the stacked q operand
    if (warp == 0) tmem_alloc(smem_addr(&tmem_base), kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < kTcStages; ++i) mbar_init(smem_addr(&full_bar[i]));
        mbar_init(smem_addr(&s_bar));
        mbar_init(smem_addr(&o_bar));
        mbar_init_fence();
    }
    const __nv_bfloat16 *qrow = q + ((size_t)b * d.Hkv * G + (size_t)kvh * G) * kD;
    {
        // element (n, k) of the K-major operand: k-step (k / 16) blocks of NS * 32 bytes
        uint8_t *bq = sm + kOffBQ, *bqb = bq + NS * 256;
        for (int i = tid; i < NS * kD; i += kTT) {
            const int n = i / kD, k = i - n * kD;
            // storage element k -> dim: pair c = k / 2 of quarter c / 16, slot p = c % 16
            const int c = k >> 1, q4 = c >> 4, pp = c & 15;
            const int grp = pp >> 2;
            const int dim = 32 * grp + 8 * q4 + 2 * (pp & 3) + (k & 1);
            uint16_t v = 0;
            if (n < NR && (n / G) == grp) v = reinterpret_cast<const uint16_t *>(qrow + (n % G) * kD)[dim];
            const int off = (k >> 4) * (NS * 32) + (n >> 3) * 256 + ((k & 15) >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
            const float f = __uint_as_float((uint32_t)v << 16);
            *reinterpret_cast<__half *>(bq + off) = __float2half_rn(f);
            *reinterpret_cast<uint16_t *>(bqb + off) = v;
        }
        if (tid < 4 * G) {
            const int grp = tid / G, h = tid % G;
            float sum = 0.f;
            for (int j = 0; j < 32; ++j) sum += __bfloat162float(qrow[h * kD + 32 * grp + j]);
            qsum[grp][h] = sum;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dependency_wait();   // the append's counters and records are visible from here
    // ---- this CTA's entry range and its tiles (class by class)
    const int n0 = d.n[s * 4 + 0], n1 = d.n[s * 4 + 1], n2 = d.n[s * 4 + 2], n3 = d.n[s * 4 + 3];
    const int o1 = n0, o2 = o1 + n1, o3 = o2 + n2, N = o3 + n3;
    const int chunk = ((N + C - 1) / C + 31) & ~31;
    const int t0 = min(N, rank * chunk), t1 = min(N, t0 + chunk);
    const int lo0 = min(t0, o1), hi0 = min(t1, o1);
    const int lo1 = min(max(t0 - o1, 0), n1), hi1 = min(max(t1 - o1, 0), n1);
    const int lo2 = min(max(t0 - o2, 0), n2), hi2 = min(max(t1 - o2, 0), n2);
    const int lo3 = min(max(t0 - o3, 0), n3), hi3 = min(max(t1 - o3, 0), n3);
    const int p1 = (hi0 - lo0 + tc_rows(0) - 1) / tc_rows(0);
    const int p2 = p1 + (hi1 - lo1 + tc_rows(1) - 1) / tc_rows(1);
    const int p3 = p2 + (hi2 - lo2 + tc_rows(2) - 1) / tc_rows(2);
    const int P = p3 + (hi3 - lo3 + tc_rows(3) - 1) / tc_rows(3);
    float *lgs = d.logits + (size_t)s * d.ncap * G;
    // tile T -> packed descriptor: entry e (bits 0-23), class c (bits 29-30); rows via nr_of
    auto tile_c = [&](int T) { return (T >= p1) + (T >= p2) + (T >= p3); };
    auto tile_e = [&](int T, int c) { return sel4(c, lo0, lo1, lo2, lo3) + (T - sel4(c, 0, p1, p2, p3)) * tc_rows(c); };
    auto tile_nr = [&](int c, int e) { return min(tc_rows(c), sel4(c, hi0, hi1, hi2, hi3) - e); };

    const uint32_t tb = tmem_base;
    const uint64_t pol = policy_evict_first();
    const uint32_t magic = magic_f16();

    auto issue_tile = [&](int T) {   // thread 0: bulk copy of tile T's records into stage T % 2
        const int c = tile_c(T), e = tile_e(T, c), nr = tile_nr(c, e);
        const int st = T & 1;
        const uint32_t bytes = (uint32_t)(nr * tc_rec(c));
        const uint8_t *src = d.pool[c] + ((size_t)s * d.cap[c] + e) * tc_rec(c);
        const uint32_t bar = smem_addr(&full_bar[st]);
        mbar_expect_tx(bar, bytes);
        bulk_copy(smem_addr(sm + kOffStage + st * kTcStage), src, bytes, bar, pol);
    };
    if (tid == 0) {
        if (P > 0) issue_tile(0);
        if (P > 1) issue_tile(1);
    }

    float Mref[G], L[G], z[4][G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        Mref[h] = kNoMax;
        L[h] = 0.f;
        z[0][h] = z[1][h] = z[2][h] = z[3][h] = 0.f;
    }
    bool ok = true;
    __half *pbuf = reinterpret_cast<__half *>(sm + off_pbuf(G));

    for (int T = 0; T < P; ++T) {
        const int c = tile_c(T), e = tile_e(T, c), nr = tile_nr(c, e);
        const int st = T & 1;
        const bool live = tid < nr;
        if (ok) ok = mbar_wait(smem_addr(&full_bar[st]), (uint32_t)((T >> 1) & 1));
        const uint8_t *rec = sm + kOffStage + st * kTcStage + tid * tc_rec(c);

        // ---- K row -> A of QK (tensor memory)
        {
            uint32_t kw[64];
            if (live) {
                switch (c) {
                    case 0: raw_words(rec, kw); break;
                    case 1: codes_to_f16<8>(rec, kw, magic); break;
                    case 2: codes_to_f16<4>(rec, kw, magic); break;
                    default: codes_to_f16<2>(rec, kw, magic); break;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) kw[i] = 0u;
            }
            tmem_st64(tb + lane_off + kColAK, kw);
        }
        tc_wait_st();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idq = idesc_f16(c == 0 ? 1u : 0u, 0u, NS);
            const uint32_t bq = smem_addr(sm + kOffBQ) + (c == 0 ? NS * 256 : 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tmem_a(tb + kColS, tb + kColAK + 8 * ks, smem_desc(bq + ks * NS * 32, 128, 256), idq, ks > 0,
                           0u, 0u, 0u, 0u);
            mma_commit(smem_addr(&s_bar));
        }

        // ---- scale / zero of this row
        float ks4[4], kz4[4], vs4[4], vz4[4];
        if (c == 0 || !live) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                ks4[g] = live ? 1.f : 0.f; kz4[g] = 0.f; vs4[g] = live ? 1.f : 0.f; vz4[g] = 0.f;
            }
        } else {
            const int cb = c == 1 ? 128 : c == 2 ? 64 : 32;
            float2 km[4], vm[4];
            load_meta(rec + 2 * cb, km);
            load_meta(rec + 2 * cb + 16, vm);
#pragma unroll
            for (int g = 0; g < 4; ++g) { ks4[g] = km[g].x; kz4[g] = km[g].y; vs4[g] = vm[g].x; vz4[g] = vm[g].y; }
        }

        // ---- V row -> B of PV (shared memory, MN-major), once the previous PV is done
        {
            uint32_t vw[64];
            if (live) {
                switch (c) {
                    case 0: codes_to_f16<16>(rec + 256, vw, magic); break;
                    case 1: codes_to_f16<8>(rec + 128, vw, magic); break;
                    case 2: codes_to_f16<4>(rec + 64, vw, magic); break;
                    default: codes_to_f16<2>(rec + 32, vw, magic); break;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) vw[i] = 0u;
            }
            if (T > 0 && ok) ok = mbar_wait(smem_addr(&o_bar), (uint32_t)((T - 1) & 1));
            uint8_t *bv = sm + kOffBV + (tid >> 3) * kBVKBlock + (tid & 7) * 16;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                *reinterpret_cast<uint4 *>(bv + j * 128) = make_uint4(vw[j], vw[16 + j], vw[32 + j], vw[48 + j]);
        }

        // ---- logits of this row
        float x[G];
        {
            if (ok) ok = mbar_wait(smem_addr(&s_bar), (uint32_t)(T & 1));
            tc_fence_after();
            uint32_t sr[16];
            tmem_ld16(tb + lane_off + kColS, sr);
            uint32_t sr2[16];
            if constexpr (NS > 16) tmem_ld16(tb + lane_off + kColS + 16, sr2);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float acc = 0.f;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int n = g * G + h;
                    const float sv = __uint_as_float(n < 16 ? sr[n & 15] : sr2[n & 15]);
                    acc = fmaf(ks4[g], sv, fmaf(kz4[g], qsum[g][h], acc));
                }
                x[h] = live ? acc * xscale : -INFINITY;
            }
            if (live) {
                float *lg = lgs + (size_t)(sel4(c, 0, o1, o2, o3) + e + tid) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) lg[h] = x[h];
            }
        }

        // ---- tile max, lazy move of the reference max
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float m = x[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
            if (lane == 0) wmax[warp][h] = m;
        }
        __syncthreads();
        float alpha[G];
        bool moved = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float tm = fmaxf(fmaxf(wmax[0][h], wmax[1][h]), fmaxf(wmax[2][h], wmax[3][h]));
            alpha[h] = 1.f;
            if (tm > Mref[h] + kRescaleSlack) {
                alpha[h] = ex2(Mref[h] - tm);
                Mref[h] = tm;
                moved = true;
            }
        }
        if (moved) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                L[h] *= alpha[h];
                z[0][h] *= alpha[h]; z[1][h] *= alpha[h]; z[2][h] *= alpha[h]; z[3][h] *= alpha[h];
            }
            if (T > 0 && warp == 0) {   // O holds earlier tiles (their PV is complete): rescale its rows
                uint32_t orow[16];
                float a = 1.f;
#pragma unroll
                for (int h = 0; h < G; ++h) a = (lane < NR && lane % G == h) ? alpha[h] : a;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld16(tb + lane_off + kColO + 16 * half, orow);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) orow[j] = __float_as_uint(__uint_as_float(orow[j]) * a);
                    tmem_st16(tb + lane_off + kColO + 16 * half, orow);
                }
                tc_wait_st();
            }
        }

        // ---- p, l, zero sums, P' rows (transposed through shared memory)
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float p = ex2(x[h] - Mref[h]);
            L[h] += p;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                z[g][h] = fmaf(p, vz4[g], z[g][h]);
                pbuf[(g * G + h) * kTT + tid] = __float2half_rn(p * vs4[g]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && T + 2 < P) issue_tile(T + 2);   // the stage's records have all been read

        // ---- warp 0: P' rows -> A of PV; thread 0 issues the four masked group chains
        if (warp == 0) {
            uint32_t pw[64];
            if (lane < NR) {
                const uint4 *src = reinterpret_cast<const uint4 *>(pbuf + lane * kTT);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint4 v = src[i];
                    pw[4 * i] = v.x; pw[4 * i + 1] = v.y; pw[4 * i + 2] = v.z; pw[4 * i + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) pw[i] = 0u;
            }
            tc_fence_after();
            tmem_st64(tb + kColAP, pw);   // warp 0 owns lanes 0..31
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                tc_fence_after();
                const uint32_t idv = idesc_f16(0u, 1u, 32u);
                const uint32_t bv = smem_addr(sm + kOffBV);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    // enable rows g*G .. g*G+G-1 only
                    uint32_t m[4] = {~0u, ~0u, ~0u, ~0u};
                    m[0] &= ~(((1u << G) - 1u) << (g * G));
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_tmem_a(tb + kColO, tb + kColAP + 8 * ks,
                                   smem_desc(bv + ks * 2 * kBVKBlock + 4 * g * 128, kBVKBlock, 128), idv,
                                   (T > 0 || ks > 0) ? 1u : 0u, m[0], m[1], m[2], m[3]);
                }
                mma_commit(smem_addr(&o_bar));
            }
            __syncwarp();
        }
    }
    if (P > 0 && ok) ok = mbar_wait(smem_addr(&o_bar), (uint32_t)((P - 1) & 1));
    if (!__all_sync(kFull, ok) && lane == 0) raise_error(d.err, kErrTimeout, (uint32_t)s);
    tc_fence_after();

    // ---- CTA sums of l and the zero sums; O rows out of tensor memory
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float v = L[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        if (lane == 0) red[warp][h] = v;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            float zz = z[g][h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(kFull, zz, o);
            if (lane == 0) red[warp][G + g * G + h] = zz;
        }
    }
    __syncthreads();
    float *co = reinterpret_cast<float *>(sm + kOffStage);   // [G][kD] the CTA's O (stages are free)
    if (warp == 0) {
        uint32_t orow[16];
        const int g = lane / G, h = lane % G;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tmem_ld16(tb + kColO + 16 * half, orow);
            tc_wait_ld();
            if (lane < NR) {
                const float zt = red[0][G + g * G + h] + red[1][G + g * G + h] + red[2][G + g * G + h] +
                                 red[3][G + g * G + h];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    co[h * kD + 32 * g + 16 * half + j] = (P > 0 ? __uint_as_float(orow[j]) : 0.f) + zt;
            }
        }
    }
    if (tid < G) {
        cta_l[tid] = red[0][tid] + red[1][tid] + red[2][tid] + red[3][tid];
        float m = Mref[0];
#pragma unroll
        for (int h = 1; h < G; ++h) m = tid == h ? Mref[h] : m;
        cta_m[tid] = m;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, kTmemCols);
    }

    // ---- cluster merge: global (M, L) per head; this rank writes its output slice
    float *orow_out = out + ((size_t)b * d.Hkv * G + (size_t)kvh * G) * kD;
    if (C == 1) {
        if (tid < G) {
            gM[tid] = cta_m[tid];
            gInvL[tid] = cta_l[tid] > 0.f ? 1.f / cta_l[tid] : 0.f;
        }
        __syncthreads();
        for (int idx = tid; idx < G * kD; idx += kTT) orow_out[idx] = co[idx] * gInvL[idx / kD];
    } else {
        cluster_sync();
        if (tid < G) {
            float Mx = kNoMax;
            for (int j = 0; j < C; ++j) Mx = fmaxf(Mx, dsmem_ld(dsmem_addr(cta_m + tid, (uint32_t)j)));
            float Lx = 0.f;
            for (int j = 0; j < C; ++j) {
                const float f = ex2(dsmem_ld(dsmem_addr(cta_m + tid, (uint32_t)j)) - Mx);
                fac[j][tid] = f;
                Lx += f * dsmem_ld(dsmem_addr(cta_l + tid, (uint32_t)j));
            }
            gM[tid] = Mx;
            gInvL[tid] = Lx > 0.f ? 1.f / Lx : 0.f;
        }
        __syncthreads();
        const int E = G * kD;
        const int per = (E + C - 1) / C;
        const int e0 = rank * per, e1 = min(E, e0 + per);
        for (int idx = e0 + tid; idx < e1; idx += kTT) {
            const int h = idx / kD;
            float acc = 0.f;
            for (int j = 0; j < C; ++j) acc += fac[j][h] * dsmem_ld(dsmem_addr(co + idx, (uint32_t)j));
            orow_out[idx] = acc * gInvL[h];
        }
    }

    // ---- scores of this CTA's tokens: += sum_h exp2(x - M_h) / L_h
    if (N > 0) {
        add_scores<G, kTT>(d, s, lgs, t0, t1, o1, o2, o3, gM, gInvL, tid);

    }
    if (C > 1) cluster_sync();   // peers may still be reading this CTA's shared memory
}

int g_tc_bps[kMaxG + 1] = {0};
int g_tc_sms = 0;

template <int G>
cudaError_t launch_tc_g(const Dev &d, const void *q, float scale, float *out, long long live_ub, cudaStream_t st,
                        int64_t *launches) {
    constexpr int smem = tc_smem_bytes(G);
    if (g_tc_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_tc_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    if (g_tc_bps[G] == 0) {
        cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, attn_tc_kernel<G>, kTT, smem);
        if (e != cudaSuccess) return e;
        // each CTA holds kTmemCols of the 512 tensor-memory columns
        g_tc_bps[G] = nb < 1 ? 1 : nb > 512 / kTmemCols ? 512 / kTmemCols : nb;
    }
    const long long slots = (long long)g_tc_bps[G] * g_tc_sms;
    long long C = slots / d.S;
    if (C > kMaxCluster) C = kMaxCluster;
    if (C > live_ub / 256) C = live_ub / 256;
    if (C < 1) C = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)d.S, 1);
    cfg.blockDim = dim3(kTT, 1, 1);
    cfg.dynamicSmemBytes = smem;
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<G>, d, static_cast<const __nv_bfloat16 *>(q), xscale,
                                       out, (int)C);
    *launches += 1;
    return e;
}

}  // namespace

cudaError_t launch_attention_tc(const Dev &d, const void *q, float scale, float *out, long long live_ub,
                                cudaStream_t st, int64_t *launches) {
    switch (d.G) {
        case 1: return launch_tc_g<1>(d, q, scale, out, live_ub, st, launches);
        case 2: return launch_tc_g<2>(d, q, scale, out, live_ub, st, launches);
        case 4: return launch_tc_g<4>(d, q, scale, out, live_ub, st, launches);
        case 8: return launch_tc_g<8>(d, q, scale, out, live_ub, st, launches);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tkv
