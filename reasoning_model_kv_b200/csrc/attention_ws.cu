// attention_ws.cu -- tkv_decode_attention for dense record placement with
// attn_kernel = 2: the warp-tile math of attention.cu (mma.sync m16n8k16, fused
// dequantisation, online softmax, score accumulation; ThinKV decode over the
// Continuous Thinking block table, cumulative attention scores as on the "Back from the
// Future" page, problem statement) fed by a warp-specialised TMA pipeline over the
// whole GPU.
//
// Work.  Persistent CTAs, two per SM; the step's tiles (64 bf16 / 128 code records,
// one class each) are split over the CTAs evenly by bytes (persist.cuh), so every SM
// streams the same share whatever the streams' lengths and class mixes, and a long
// stream is spread over many SMs without a cluster limit.
//
// Roles (288 threads): warp 8 issues each tile's TMA boxes (K codes, V codes, scale /
// zero block, each with the hardware swizzle of its row width) into one of two stages.
// The consumer warps form kGroups groups of eight that take alternate tiles (one group:
// every tile; a layout with two groups and one CTA per SM measured slower, 116 against
// 98 us at 64 x 32k post-eviction); in a group, warp w takes rows
// 16w .. 16w+15 of a code tile (8w .. 8w+7 of a bf16 tile) and runs the tile math on them
// straight from the swizzled boxes, with its own online-softmax state.  A group's warps
// see the same tiles, so they change stream together: then each writes its (m, l, O) to
// shared memory and the group merges them into one partial per (stream, CTA, group);
// a group writes an empty partial for a stream of its CTA that only the other group saw.
// The merge + score pass (persist.cuh) combines a stream's partials and adds every
// token's attention mass to its score.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_tile.cuh"
#include "persist.cuh"

namespace tkv {
namespace {

using namespace attn;

constexpr int kConsumers = 8;                       // warps of a consumer group
constexpr int kGroups = 1;                          // consumer groups (alternate tiles)
constexpr int kCtasPerSm = kGroups == 1 ? 2 : 1;    // resident CTAs per SM
constexpr int kProducerWarp = kConsumers * kGroups;
constexpr int kThreadsWS = 32 * (kProducerWarp + 1);
__host__ __device__ constexpr int ws_stages(int G) { return kGroups == 1 ? 2 : G <= 4 ? 4 : 3; }
__host__ __device__ constexpr int ws_merge_bytes(int G) { return kConsumers * G * kD * 4; }   // per group
__host__ __device__ constexpr int ws_smem_bytes(int G) {
    return 1024 + ws_stages(G) * kRawBytes + kGroups * ws_merge_bytes(G);
}

// The stream's query operands (query_frags) per lane, shared by the consumer warps (they
// all work on the same stream) and read from shared memory where the tile math uses
// them: 49 words per lane, an odd stride, so a warp's reads hit 32 distinct banks.
struct QFrag {
    uint32_t qb[4][2][2], qbb[4][2][2];
    float qs[2][4], qinv[2][4];
    uint32_t pad;
};

template <int G>
__global__ void __launch_bounds__(kThreadsWS, kCtasPerSm)
    attn_ws_kernel(const __grid_constant__ Dev d, const __grid_constant__ I8Maps maps,
                   const __nv_bfloat16 *__restrict__ q, float xscale) {
    constexpr int R = ws_stages(G);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);   // stages: 1024-aligned
    __shared__ __align__(8) uint64_t bar_full[R], bar_empty[R];
    // per group: its warps' partials written / read (the two halves of a merge), and the
    // stream's query operands published; bounded waits, so a warp that gave up on a
    // timeout never leaves the others stuck at a barrier
    __shared__ __align__(8) uint64_t bar_written[kGroups], bar_read[kGroups], bar_query[kGroups];
    __shared__ SharedPlan pl;
    __shared__ TileDesc desc[kDescRing];
    __shared__ float wm[kGroups][kConsumers][kMaxG], wl[kGroups][kConsumers][kMaxG];
    __shared__ QFrag qf[kGroups][32];
    __shared__ int qscaled_sh[kGroups];
    __shared__ uint32_t err_timeout;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cta = blockIdx.x, ncta = gridDim.x;
    if (tid == 0) {
        for (int i = 0; i < R; ++i) {
            mbar_init_n(smem_addr(&bar_full[i]), 1);
            mbar_init_n(smem_addr(&bar_empty[i]), kConsumers);
        }
        for (int i = 0; i < kGroups; ++i) {
            mbar_init_n(smem_addr(&bar_written[i]), kConsumers);
            mbar_init_n(smem_addr(&bar_read[i]), kConsumers);
            mbar_init_n(smem_addr(&bar_query[i]), 1);
        }
        err_timeout = 0;
        mbar_init_fence();
    }
    if (warp == kProducerWarp && lane == 0) prefetch_maps(maps);
    __syncthreads();

    grid_dependency_wait();   // the append's counters and records are visible from here
    plan_work<kThreadsWS>(d, pl, cta, ncta);
    bool ok = true;
    const uint32_t smb = smem_addr(sm);

    if (warp == kProducerWarp) {
        // ================================================= producer
        if (lane == 0) ok = produce_tiles<R>(d, maps, pl, desc, bar_full, bar_empty, smb, kGroups);
    } else {
        // ================================================= consumer group grp, warp cw of it
        const int grp = warp / kConsumers, cw = warp - grp * kConsumers;
        const int gt = tid - grp * 32 * kConsumers;     // thread index inside the group
        int nmerge = 0, nquery = 0;                     // phases used of bar_written / bar_read, bar_query
        // every warp of the group at a merge point (lane 0 arrives after the warp's writes)
        auto group_sync = [&](uint64_t *bar, int &uses) {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(bar));
            if (ok) ok = mbar_wait(smem_addr(bar), (uint32_t)(uses & 1));
            ok = __all_sync(kFull, ok);
            ++uses;
        };
        const int g = lane >> 2, tig = lane & 3;
        const uint32_t magic = magic_f16();
        float *wo = reinterpret_cast<float *>(sm + R * kRawBytes + grp * ws_merge_bytes(G));   // [cw][G][kD]
        const QFrag &Q = qf[grp][lane];
        bool qscaled = false;
        WarpState ws;
        int cur_s = -1;

        auto reset = [&]() {
            ws.m[0] = ws.m[1] = kNoMax;
            ws.l[0] = ws.l[1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) ws.o[mt][0] = ws.o[mt][1] = ws.o[mt][2] = ws.o[mt][3] = 0.f;
#pragma unroll
            for (int grp = 0; grp < 4; ++grp) ws.z[0][grp] = ws.z[1][grp] = 0.f;
        };
        // the CTA's partial of stream s_old: every consumer warp's (m, l, O) merged
        auto flush = [&](int s_old) {
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                ws.l[0] += __shfl_xor_sync(kFull, ws.l[0], o);
                ws.l[1] += __shfl_xor_sync(kFull, ws.l[1], o);
#pragma unroll
                for (int zg = 0; zg < 4; ++zg) {
                    ws.z[0][zg] += __shfl_xor_sync(kFull, ws.z[0][zg], o);
                    ws.z[1][zg] += __shfl_xor_sync(kFull, ws.z[1][zg], o);
                }
            }
            if (g == 0) {
                if (2 * tig < G) { wm[grp][cw][2 * tig] = ws.m[0]; wl[grp][cw][2 * tig] = ws.l[0]; }
                if (2 * tig + 1 < G) { wm[grp][cw][2 * tig + 1] = ws.m[1]; wl[grp][cw][2 * tig + 1] = ws.l[1]; }
            }
            float *w = wo + cw * G * kD;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int d0 = 16 * mt + g, zg = mt >> 1;
                if (2 * tig < G) {
                    w[(2 * tig) * kD + d0] = ws.o[mt][0] + ws.z[0][zg];
                    w[(2 * tig) * kD + d0 + 8] = ws.o[mt][2] + ws.z[0][zg];
                }
                if (2 * tig + 1 < G) {
                    w[(2 * tig + 1) * kD + d0] = ws.o[mt][1] + ws.z[1][zg];
                    w[(2 * tig + 1) * kD + d0 + 8] = ws.o[mt][3] + ws.z[1][zg];
                }
            }
            int u = nmerge;
            group_sync(&bar_written[grp], u);
            float *part = d.part + (size_t)(kGroups * (s_old + cta) + grp) * part_floats(G);
            for (int i = gt; i < G * kD; i += 32 * kConsumers) {
                const int h = i / kD;
                float M = kNoMax;
#pragma unroll
                for (int v = 0; v < kConsumers; ++v)
                    if (wl[grp][v][h] > 0.f) M = fmaxf(M, wm[grp][v][h]);
                float L = 0.f, acc = 0.f;
#pragma unroll
                for (int v = 0; v < kConsumers; ++v) {
                    const float f = wl[grp][v][h] > 0.f ? ex2(wm[grp][v][h] - M) : 0.f;   // warps without tokens: l = 0
                    L = fmaf(f, wl[grp][v][h], L);
                    acc = fmaf(f, wo[(v * G + h) * kD + (i - h * kD)], acc);
                }
                part[3 * G + i] = acc;
                if (i - h * kD == 0) {
                    part[h] = M;
                    part[G + h] = L;
                    part[2 * G + h] = 0.f;
                }
            }
            u = nmerge;
            group_sync(&bar_read[grp], u);   // wm / wl / wo free again
            ++nmerge;
        };
        // an empty partial (l = 0: the merge skips it) in this group's slot of stream s
        auto write_empty = [&](int s) {
            if (cw == 0 && lane < G) {
                float *part = d.part + (size_t)(kGroups * (s + cta) + grp) * part_floats(G);
                part[lane] = kNoMax;
                part[G + lane] = 0.f;
                part[2 * G + lane] = 0.f;
            }
        };
        bool cta_empty = false;

        for (int k = grp;; k += kGroups) {
            const int slot = k % R;
            if (ok) ok = mbar_wait(smem_addr(&bar_full[slot]), (uint32_t)((k / R) & 1));
            const TileDesc td = desc[k % kDescRing];
            const bool end = td_end(td);
            if (k == grp) cta_empty = end && (grp == 0 || td_end(desc[0]));
            // a stream whose tiles in this CTA all went to the other group (the tile
            // between this group's previous tile and this one) gets an empty partial
            if (ok && k >= 1) {
                const TileDesc to = desc[(k - 1) % kDescRing];
                if (!td_end(to) && to.s != cur_s && (end || to.s != td.s)) write_empty(to.s);
            }
            const bool wok = __all_sync(kFull, ok);
            if (end || !wok) { ok = wok; break; }
            if (td.s != cur_s) {
                if (cur_s >= 0) flush(cur_s);
                cur_s = td.s;
                if (cw == 0) {
                    const int bb = td.s / d.Hkv, kvh = td.s - bb * d.Hkv;
                    QFrag f;
                    bool sc;
                    query_frags<G>(q + ((size_t)bb * d.Hkv * G + (size_t)kvh * G) * kD, lane, f.qb, f.qbb, f.qs,
                                   f.qinv, sc);
                    qf[grp][lane] = f;
                    if (lane == 0) qscaled_sh[grp] = sc;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&bar_query[grp]));
                }
                if (ok) ok = mbar_wait(smem_addr(&bar_query[grp]), (uint32_t)(nquery & 1));   // operands in place
                ok = __all_sync(kFull, ok);
                ++nquery;
                qscaled = qscaled_sh[grp] != 0;
                reset();
            }
            const int tcls = td_c(td), nr = td_nr(td);
            const int rows = tcls == 0 ? 8 : 16;
            const int r0 = cw * rows;
            const int nw = min(max(nr - r0, 0), rows);
            if (nw > 0) {
                const uint8_t *stage = sm + slot * kRawBytes;
                float *lg = d.logits + ((size_t)td.s * d.ncap + td.oc + td.e + r0) * G;
                switch (tcls) {
                    case 0:
                        tile_compute<16, 8, G, 0, false>(TmaLoader<16>(stage, r0, g), nw, lane, Q.qb, Q.qbb, Q.qs, Q.qinv,
                                                  qscaled, xscale, ws, lg, magic);
                        break;
                    case 1:
                        tile_compute<8, 16, G, 0, false>(TmaLoader<8>(stage, r0, g), nw, lane, Q.qb, Q.qbb, Q.qs, Q.qinv,
                                                  qscaled, xscale, ws, lg, magic);
                        break;
                    case 2:
                        tile_compute<4, 16, G, 0, false>(TmaLoader<4>(stage, r0, g), nw, lane, Q.qb, Q.qbb, Q.qs, Q.qinv,
                                                  qscaled, xscale, ws, lg, magic);
                        break;
                    default:
                        tile_compute<2, 16, G, 0, false>(TmaLoader<2>(stage, r0, g), nw, lane, Q.qb, Q.qbb, Q.qs, Q.qinv,
                                                  qscaled, xscale, ws, lg, magic);
                        break;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bar_empty[slot]));
            if (cw == 0 && lane == 0) {
                if (td_first(td)) d.seg_lo[td.s] = cta;
                if (td_last(td)) d.seg_hi[td.s] = cta;
            }
        }
        // every warp of the group left the loop at its end tile (or gave up on a timeout,
        // in which case the bounded merge waits of the others run out as well)
        if (ok) {
            if (cur_s >= 0) {
                flush(cur_s);
            } else if (cta_empty && pl.s0 < d.S) {
                // no tile starts in this CTA's share, which lies inside stream s0 between
                // two tiles: the merge reads this CTA's slots of s0
                write_empty(pl.s0);
            }
        }
    }

    if (!ok) atomicExch(&err_timeout, 1u);
    __syncthreads();
    if (tid == 0 && err_timeout) raise_error(d.err, kErrTimeout, (uint32_t)cta);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

int g_bps_ws[kMaxG + 1][kMaxDevices] = {};

template <int G>
cudaError_t launch_ws_g(const Dev &d, const I8Maps &maps, const void *q, float scale, float *out,
                        long long live_ub, cudaStream_t st, int64_t *launches) {
    constexpr int smem = ws_smem_bytes(G);
    int sms = 0, bps = 0;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = cached_blocks_per_sm(g_bps_ws[G], reinterpret_cast<const void *>(attn_ws_kernel<G>), kThreadsWS, smem, &bps);
    if (e != cudaSuccess) return e;
    // kCtasPerSm CTAs per SM when they fit (fixed by the device alone, so the split of a
    // given state, and so the results, are always the same)
    const int ncta = std::min(sms * std::min(bps, kCtasPerSm), d.ncta_max);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ncta, 1, 1);
    cfg.blockDim = dim3(kThreadsWS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the launch with the append
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float xscale = scale * 1.4426950408889634f;   // logits in the log2 domain
    e = cudaLaunchKernelEx(&cfg, attn_ws_kernel<G>, d, maps, static_cast<const __nv_bfloat16 *>(q), xscale);
    *launches += 1;
    if (e != cudaSuccess) return e;
    return launch_finalize<G, false, kGroups>(d, out, nullptr, nullptr, 0.f, 0.f, ncta, live_ub, st, launches);
}

}  // namespace

cudaError_t launch_attention_ws(const Dev &d, const I8Maps &maps, const void *q, float scale, float *out,
                                long long live_ub, cudaStream_t st, int64_t *launches) {
    switch (d.G) {
        case 1: return launch_ws_g<1>(d, maps, q, scale, out, live_ub, st, launches);
        case 2: return launch_ws_g<2>(d, maps, q, scale, out, live_ub, st, launches);
        case 4: return launch_ws_g<4>(d, maps, q, scale, out, live_ub, st, launches);
        case 8: return launch_ws_g<8>(d, maps, q, scale, out, live_ub, st, launches);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tkv
