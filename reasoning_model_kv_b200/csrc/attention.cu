// attention.cu -- tkv_decode_attention: one GQA decode step over the
// mixed-precision pools with fused dequantisation, split-K online softmax and
// accumulation of each token's attention mass into its score (ThinKV decode
// over the Continuous Thinking block table; cumulative attention scores as in
// H2O, described on the "Back from the Future" page, problem statement).
//
// Work split: grid (splits, S).  CTA (j, s) takes entry range j of stream s
// (entries ordered class 0, 1, 2, 3, each class in table order) and keeps an
// online-softmax state per query head; it writes (m, l, O) for its range and
// the raw logits of its tokens.  The combine kernel merges the splits of a
// stream, writes the output, and adds p = exp(logit - m)/l, summed over the G
// heads, to every token's score.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tkv_internal.cuh"

namespace tkv {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarps = 8;

// Dequantise the 4 K and 4 V elements [4*lane, 4*lane+4) of one record.
template <int BITS>
__device__ __forceinline__ void dequant4(const uint8_t *rec, int lane, float (&k)[4],
                                         float (&v)[4]) {
    if constexpr (BITS == 16) {
        const uint2 rk = reinterpret_cast<const uint2 *>(rec)[lane];
        const uint2 rv = reinterpret_cast<const uint2 *>(rec + 2 * kD)[lane];
        k[0] = __uint_as_float(rk.x << 16); k[1] = __uint_as_float(rk.x & 0xffff0000u);
        k[2] = __uint_as_float(rk.y << 16); k[3] = __uint_as_float(rk.y & 0xffff0000u);
        v[0] = __uint_as_float(rv.x << 16); v[1] = __uint_as_float(rv.x & 0xffff0000u);
        v[2] = __uint_as_float(rv.y << 16); v[3] = __uint_as_float(rv.y & 0xffff0000u);
    } else {
        constexpr int cb = kD * BITS / 8;
        constexpr uint32_t mask = (1u << BITS) - 1u;
        const __half *meta = reinterpret_cast<const __half *>(rec + 2 * cb);
        const int g = lane >> 3;
        const float ks = __half2float(meta[g]), kz = __half2float(meta[kNG + g]);
        const float vs = __half2float(meta[2 * kNG + g]), vz = __half2float(meta[3 * kNG + g]);
        uint32_t wk, wv;
        if constexpr (BITS == 8) {
            wk = reinterpret_cast<const uint32_t *>(rec)[lane];
            wv = reinterpret_cast<const uint32_t *>(rec + cb)[lane];
        } else if constexpr (BITS == 4) {
            wk = reinterpret_cast<const uint16_t *>(rec)[lane];
            wv = reinterpret_cast<const uint16_t *>(rec + cb)[lane];
        } else {
            wk = rec[lane];
            wv = rec[cb + lane];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            k[i] = __fmaf_rn(static_cast<float>((wk >> (BITS * i)) & mask), ks, kz);
            v[i] = __fmaf_rn(static_cast<float>((wv >> (BITS * i)) & mask), vs, vz);
        }
    }
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32) attn_split_kernel(
    Dev d, const __nv_bfloat16 *__restrict__ q, float scale, int splits) {
    const int j = blockIdx.x, s = blockIdx.y;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int off[5];
    off[0] = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) off[c + 1] = off[c] + d.n[s * 4 + c];
    const int N = off[4];
    const int chunk = (N + splits - 1) / splits;
    const int t0 = min(N, j * chunk), t1 = min(N, t0 + chunk);

    float qf[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const __nv_bfloat16 *qr = q + ((size_t)b * d.Hkv * G + kvh * G + h) * kD;
        const uint2 r = reinterpret_cast<const uint2 *>(qr)[lane];
        qf[h][0] = __uint_as_float(r.x << 16); qf[h][1] = __uint_as_float(r.x & 0xffff0000u);
        qf[h][2] = __uint_as_float(r.y << 16); qf[h][3] = __uint_as_float(r.y & 0xffff0000u);
    }
    float m[G], l[G], o[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY; l[h] = 0.f;
        o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
    }
    float *lg = d.logits + (size_t)s * d.ncap * G;
    for (int t = t0 + warp; t < t1; t += kWarps) {
        int c = 0;
        while (t >= off[c + 1]) ++c;
        const int i = t - off[c];
        const size_t e = (size_t)s * d.cap[c] + i;
        const uint8_t *rec = d.pool[c] + ((size_t)s * d.cap[c] + d.handle[c][e]) * d.rec[c];
        float kx[4], vx[4];
        switch (c) {
            case 0: dequant4<16>(rec, lane, kx, vx); break;
            case 1: dequant4<8>(rec, lane, kx, vx); break;
            case 2: dequant4<4>(rec, lane, kx, vx); break;
            default: dequant4<2>(rec, lane, kx, vx); break;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float dot = qf[h][0] * kx[0] + qf[h][1] * kx[1] + qf[h][2] * kx[2] + qf[h][3] * kx[3];
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) dot += __shfl_xor_sync(kFull, dot, o2);
            const float x = dot * scale;
            if (lane == h) lg[(size_t)t * G + h] = x;
            const float mn = fmaxf(m[h], x);
            const float corr = expf(m[h] - mn);
            const float p = expf(x - mn);
            l[h] = l[h] * corr + p;
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) o[h][e2] = o[h][e2] * corr + p * vx[e2];
            m[h] = mn;
        }
    }
    // merge the warps of the CTA
    __shared__ float sm[kWarps][G], sl[kWarps][G];
    __shared__ float so[kWarps][G][kD];
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) { sm[warp][h] = m[h]; sl[warp][h] = l[h]; }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) so[warp][h][4 * lane + e2] = o[h][e2];
    __syncthreads();
    float *part = d.part + ((size_t)s * d.max_splits + j) * G * (kD + 2);
    for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
        const int h = idx / kD, dd = idx - h * kD;
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm[w][h]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < kWarps; ++w) {
                const float f = expf(sm[w][h] - M);
                L += sl[w][h] * f;
                O += so[w][h][dd] * f;
            }
        }
        part[h * (kD + 2) + 2 + dd] = O;
        if (dd == 0) { part[h * (kD + 2)] = M; part[h * (kD + 2) + 1] = L; }
    }
}

template <int G>
__global__ void __launch_bounds__(kD) attn_combine_kernel(Dev d, float *__restrict__ out,
                                                          int splits) {
    const int s = blockIdx.x;
    const int b = s / d.Hkv, kvh = s - b * d.Hkv;
    const float *part = d.part + (size_t)s * d.max_splits * G * (kD + 2);
    __shared__ float Ms[G], Ls[G];
    const int dd = threadIdx.x;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
        for (int j = 0; j < splits; ++j) M = fmaxf(M, part[(j * G + h) * (kD + 2)]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int j = 0; j < splits; ++j) {
                const float *pj = part + (j * G + h) * (kD + 2);
                const float f = expf(pj[0] - M);
                L += pj[1] * f;
                O += pj[2 + dd] * f;
            }
        }
        out[((size_t)b * d.Hkv * G + kvh * G + h) * kD + dd] = L > 0.f ? O / L : 0.f;
        if (dd == 0) { Ms[h] = M; Ls[h] = L; }
    }
    __syncthreads();
    if (Ms[0] == -INFINITY) return;  // empty stream: no token to score
    int off[5];
    off[0] = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) off[c + 1] = off[c] + d.n[s * 4 + c];
    const float *lg = d.logits + (size_t)s * d.ncap * G;
    for (int t = threadIdx.x; t < off[4]; t += blockDim.x) {
        float inc = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) inc += expf(lg[(size_t)t * G + h] - Ms[h]) / Ls[h];
        int c = 0;
        while (t >= off[c + 1]) ++c;
        d.score[c][(size_t)s * d.cap[c] + (t - off[c])] += inc;
    }
}

template <int G>
cudaError_t launch_g(const Dev &d, const void *q, float scale, float *out, int splits,
                     cudaStream_t st, int64_t *launches) {
    attn_split_kernel<G><<<dim3(splits, d.S), kWarps * 32, 0, st>>>(
        d, static_cast<const __nv_bfloat16 *>(q), scale, splits);
    attn_combine_kernel<G><<<d.S, kD, 0, st>>>(d, out, splits);
    *launches += 2;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Dev &d, const void *q, float scale, float *out, int splits,
                             cudaStream_t st, int64_t *launches) {
    switch (d.G) {
        case 1: return launch_g<1>(d, q, scale, out, splits, st, launches);
        case 2: return launch_g<2>(d, q, scale, out, splits, st, launches);
        case 4: return launch_g<4>(d, q, scale, out, splits, st, launches);
        case 8: return launch_g<8>(d, q, scale, out, splits, st, launches);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tkv
