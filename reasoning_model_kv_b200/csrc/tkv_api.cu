// tkv_api.cu -- host side of the C ABI in include/tkv.h: configuration checks,
// the workspace layout, argument validation and kernel launches.  No device
// memory is allocated here; nothing synchronises except poll/export/import.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include "tkv.h"
#include "tkv_internal.cuh"

struct tkv_cache {
    tkv_config cfg;
    tkv_layout lay;
    tkv::Dev dev;
    uint8_t *base;
    long long live_ub;   // host-side upper bound of live entries in any stream
    int64_t launches;
    tkv::I8Maps maps;    // TMA descriptors of the pools (tensor-core attention), made on first use
    bool maps_ready;
};

namespace {

thread_local std::string g_last_error;

tkv_status fail(tkv_status st, const std::string &msg) {
    g_last_error = msg;
    return st;
}

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool valid_config(const tkv_config *c, std::string *why) {
    if (!c) { *why = "config is NULL"; return false; }
    if (c->B < 1 || c->Hkv < 1) { *why = "B and Hkv must be >= 1"; return false; }
    if (!(c->G == 1 || c->G == 2 || c->G == 4 || c->G == 8)) { *why = "G must be 1, 2, 4 or 8"; return false; }
    if (c->D != tkv::kD) { *why = "D must be 128"; return false; }
    if (c->group != tkv::kGroup) { *why = "group must be 32"; return false; }
    const int want[4] = {16, 8, 4, 2};
    for (int i = 0; i < 4; ++i)
        if (c->bits[i] != want[i]) { *why = "bits must be {16, 8, 4, 2}"; return false; }
    if (c->n_protect < 0) { *why = "n_protect must be >= 0"; return false; }
    long long ncap = 0;
    for (int i = 0; i < 4; ++i) {
        if (c->cap[i] < 0) { *why = "cap[c] must be >= 0"; return false; }
        ncap += c->cap[i];
    }
    if (ncap > (1ll << 30)) { *why = "sum of cap too large"; return false; }
    if (c->max_append < 1 || c->max_append > (1 << 24)) { *why = "max_append must be in [1, 2^24]"; return false; }
    if ((long long)c->B * c->Hkv > 65535) { *why = "B * Hkv must be <= 65535"; return false; }
    if (c->dense != 0 && c->dense != 1) { *why = "dense must be 0 or 1"; return false; }
    if (c->attn_kernel < 0 || c->attn_kernel > 2) { *why = "attn_kernel must be 0, 1 or 2"; return false; }
    if (c->attn_kernel != 0 && c->dense != 1) { *why = "attn_kernel 1 and 2 need dense placement"; return false; }
    if (c->codec != 0 && c->codec != 1) { *why = "codec must be 0 or 1"; return false; }
    if (c->codec == 1 && c->attn_kernel != 0) { *why = "codec 1 needs attn_kernel 0"; return false; }
    for (int i = 0; i < 4; ++i)
        if (c->cap[i] >= (1 << 24)) { *why = "cap[c] must be < 2^24"; return false; }
    return true;
}

// Lays the workspace out; fills *lay and, if base != NULL, the device view.
void make_layout(const tkv_config &c, tkv_layout *lay, tkv::Dev *dev, uint8_t *base) {
    const size_t S = (size_t)c.B * c.Hkv;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes); return o; };
    lay->n = take(S * 4 * sizeof(int32_t));
    lay->ft = take(S * 4 * sizeof(int32_t));
    lay->hw = take(S * 4 * sizeof(int32_t));
    lay->err = take(16 * sizeof(uint32_t));
    for (int k = 0; k < 4; ++k) {
        const size_t e = S * (size_t)c.cap[k];
        lay->handle[k] = take(e * sizeof(int32_t));
        lay->pos[k] = take(e * sizeof(int32_t));
        lay->score[k] = take(e * sizeof(float));
        lay->fs[k] = take(e * sizeof(int32_t));
    }
    for (int k = 0; k < 4; ++k) {
        lay->rec_bytes[k] = tkv::record_bytes(c.bits[k], c.codec);
        lay->pool[k] = take(S * (size_t)c.cap[k] * lay->rec_bytes[k]);
    }
    lay->state_bytes = off;
    // logits rows padded to 32 entries so every CTA's slice starts on a 128-byte line
    const int ncap = (c.cap[0] + c.cap[1] + c.cap[2] + c.cap[3] + 31) & ~31;
    const size_t o_rank = take((size_t)c.B * c.max_append * sizeof(int32_t));
    const size_t o_tot = take((size_t)c.B * 4 * sizeof(int32_t));
    const size_t o_lg = take(S * (size_t)ncap * c.G * sizeof(float));
    const size_t o_part = take(tkv::part_bytes(S, c.G));
    const size_t o_seglo = take(S * sizeof(int32_t));
    const size_t o_seghi = take(S * sizeof(int32_t));
    lay->total_bytes = off;
    if (!dev) return;
    dev->B = c.B; dev->Hkv = c.Hkv; dev->G = c.G; dev->S = (int)S;
    dev->n_protect = c.n_protect; dev->max_append = c.max_append;
    dev->dense = c.dense;
    dev->attn_kernel = c.attn_kernel;
    dev->codec = c.codec;
    dev->n = reinterpret_cast<int32_t *>(base + lay->n);
    dev->ft = reinterpret_cast<int32_t *>(base + lay->ft);
    dev->hw = reinterpret_cast<int32_t *>(base + lay->hw);
    dev->err = reinterpret_cast<uint32_t *>(base + lay->err);
    for (int k = 0; k < 4; ++k) {
        dev->cap[k] = c.cap[k];
        dev->rec[k] = lay->rec_bytes[k];
        dev->handle[k] = reinterpret_cast<int32_t *>(base + lay->handle[k]);
        dev->pos[k] = reinterpret_cast<int32_t *>(base + lay->pos[k]);
        dev->score[k] = reinterpret_cast<float *>(base + lay->score[k]);
        dev->fs[k] = reinterpret_cast<int32_t *>(base + lay->fs[k]);
        dev->pool[k] = base + lay->pool[k];
    }
    dev->rank = reinterpret_cast<int32_t *>(base + o_rank);
    dev->totals = reinterpret_cast<int32_t *>(base + o_tot);
    dev->logits = reinterpret_cast<float *>(base + o_lg);
    dev->ncap = ncap;
    dev->part = reinterpret_cast<float *>(base + o_part);
    dev->seg_lo = reinterpret_cast<int32_t *>(base + o_seglo);
    dev->seg_hi = reinterpret_cast<int32_t *>(base + o_seghi);
    dev->ncta_max = tkv::kNctaMax;
}

tkv_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return TKV_OK;
    return fail(TKV_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Hooks for entry points defined in other translation units.
namespace tkv {
const Dev *cache_dev(const tkv_cache *c, int *max_append) {
    *max_append = c->cfg.max_append;
    return &c->dev;
}
void note_append(tkv_cache *c, int64_t launches, int T) {
    c->launches += launches;
    c->live_ub = std::min<long long>(c->dev.ncap, c->live_ub + T);
}
tkv_status api_fail(tkv_status st, const std::string &msg) { return fail(st, msg); }

namespace {
std::atomic<int> g_sm_count[kMaxDevices];
std::mutex g_occ_mu;
}  // namespace

cudaError_t device_sm_count(int *sms) {
    *sms = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        g_sm_count[dev].store(v, std::memory_order_relaxed);
    }
    *sms = v;
    return cudaSuccess;
}

cudaError_t cached_blocks_per_sm(int *slot_per_device, const void *kernel, int threads, size_t smem,
                                 int *blocks) {
    *blocks = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_occ_mu);
    if (slot_per_device[dev] == 0) {
        if (smem > 48 * 1024) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, threads, smem);
        if (e != cudaSuccess) return e;
        slot_per_device[dev] = nb > 0 ? nb : 1;
    }
    *blocks = slot_per_device[dev];
    return cudaSuccess;
}

cudaError_t cached_max_clusters(int *slot_per_device, const void *kernel, int threads, size_t smem, int C,
                                int *clusters) {
    *clusters = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_occ_mu);
    if (slot_per_device[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)C, 1, 1);
        cfg.blockDim = dim3((unsigned)threads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
        if (e != cudaSuccess) return e;
        slot_per_device[dev] = n > 0 ? n : 1;
    }
    *clusters = slot_per_device[dev];
    return cudaSuccess;
}
}  // namespace tkv

extern "C" {

size_t tkv_workspace_bytes(const tkv_config *cfg) {
    std::string why;
    if (!valid_config(cfg, &why)) { g_last_error = why; return 0; }
    tkv_layout lay;
    make_layout(*cfg, &lay, nullptr, nullptr);
    return lay.total_bytes;
}

tkv_status tkv_create(const tkv_config *cfg, void *d_workspace, size_t workspace_bytes,
                      tkv_cache **out) {
    std::string why;
    if (!out) return fail(TKV_ERR_INVALID, "out is NULL");
    *out = nullptr;
    if (!valid_config(cfg, &why)) return fail(TKV_ERR_INVALID, why);
    if (!d_workspace) return fail(TKV_ERR_INVALID, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(d_workspace) % kAlign)
        return fail(TKV_ERR_INVALID, "workspace must be 256-byte aligned");
    tkv_layout lay;
    make_layout(*cfg, &lay, nullptr, nullptr);
    if (workspace_bytes < lay.total_bytes) return fail(TKV_ERR_INVALID, "workspace too small");
    auto *c = new (std::nothrow) tkv_cache();
    if (!c) return fail(TKV_ERR_INVALID, "out of host memory");
    c->cfg = *cfg;
    c->base = static_cast<uint8_t *>(d_workspace);
    make_layout(*cfg, &c->lay, &c->dev, c->base);
    c->live_ub = 0;
    c->launches = 0;
    c->maps_ready = false;
    *out = c;
    return TKV_OK;
}

tkv_status tkv_destroy(tkv_cache *cache) {
    delete cache;
    return TKV_OK;
}

tkv_status tkv_reset(tkv_cache *c, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    auto st = static_cast<cudaStream_t>(stream);
    // n, ft, hw and err are contiguous at the start of the workspace
    cudaError_t e = cudaMemsetAsync(c->base, 0, c->lay.err + 16 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_status(e, "tkv_reset");
    c->live_ub = 0;
    return TKV_OK;
}

tkv_status tkv_get_layout(const tkv_cache *c, tkv_layout *out) {
    if (!c || !out) return fail(TKV_ERR_INVALID, "NULL argument");
    *out = c->lay;
    return TKV_OK;
}

tkv_status tkv_quantize_append(tkv_cache *c, const void *k, const void *v, const uint8_t *cls,
                               const int32_t *pos, int32_t T, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (!k || !v || !cls || !pos) return fail(TKV_ERR_INVALID, "NULL input pointer");
    if (T < 1 || T > c->cfg.max_append) return fail(TKV_ERR_INVALID, "T out of [1, max_append]");
    if (!aligned16(k) || !aligned16(v)) return fail(TKV_ERR_INVALID, "k and v must be 16-byte aligned");
    if (!aligned16(pos)) return fail(TKV_ERR_INVALID, "pos must be 16-byte aligned");
    cudaError_t e = tkv::launch_append(c->dev, k, v, cls, pos, T, static_cast<cudaStream_t>(stream),
                                       &c->launches);
    const long long ncap = c->dev.ncap;
    c->live_ub = std::min(ncap, c->live_ub + T);
    return cuda_status(e, "tkv_quantize_append");
}

namespace {
// The pools' TMA descriptors, encoded once per cache (the pools never move).
tkv_status ensure_maps(tkv_cache *c) {
    if (c->maps_ready) return TKV_OK;
    cudaError_t e = tkv::make_i8_maps(c->dev, &c->maps);
    if (e != cudaSuccess) return cuda_status(e, "encoding the pools' TMA descriptors");
    c->maps_ready = true;
    return TKV_OK;
}
}  // namespace

namespace {
// Decode attention over the cache with `ub` bounding every stream's live entries.
// q_ready: the append was the last launch on `st` (see launch_attention).
tkv_status launch_decode(tkv_cache *c, const void *q, float softmax_scale, float *out, long long ub,
                         cudaStream_t st, const char *what, bool q_ready = false) {
    cudaError_t e;
    if (c->cfg.attn_kernel != 0) {   // the persistent kernels (dense placement)
        const tkv_status ms = ensure_maps(c);
        if (ms != TKV_OK) return ms;
        if (c->cfg.attn_kernel == 1)
            e = tkv::launch_attention_i8(c->dev, c->maps, q, softmax_scale, out, nullptr, nullptr, 0.f, 0.f, ub, st,
                                         &c->launches);
        else
            e = tkv::launch_attention_ws(c->dev, c->maps, q, softmax_scale, out, ub, st, &c->launches);
    } else {
        e = tkv::launch_attention(c->dev, q, softmax_scale, out, ub, st, &c->launches, nullptr, nullptr, 0.f, 0.f,
                                  q_ready);
    }
    return cuda_status(e, what);
}
}  // namespace

tkv_status tkv_decode_attention(tkv_cache *c, const void *q, float softmax_scale, float *out,
                                void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (!q || !out) return fail(TKV_ERR_INVALID, "NULL q or out");
    if (!aligned16(q) || !aligned16(out)) return fail(TKV_ERR_INVALID, "q and out must be 16-byte aligned");
    const long long ub = std::max(1ll, c->live_ub);
    return launch_decode(c, q, softmax_scale, out, ub, static_cast<cudaStream_t>(stream), "tkv_decode_attention");
}

tkv_status tkv_decode_step(tkv_cache *c, const void *k, const void *v, const uint8_t *cls, const int32_t *pos,
                           const void *q, float softmax_scale, float *out, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (!k || !v || !cls || !pos) return fail(TKV_ERR_INVALID, "NULL input pointer");
    if (!q || !out) return fail(TKV_ERR_INVALID, "NULL q or out");
    if (!aligned16(k) || !aligned16(v)) return fail(TKV_ERR_INVALID, "k and v must be 16-byte aligned");
    if (!aligned16(pos)) return fail(TKV_ERR_INVALID, "pos must be 16-byte aligned");
    if (!aligned16(q) || !aligned16(out)) return fail(TKV_ERR_INVALID, "q and out must be 16-byte aligned");
    // the append, then the attention, whose launch overlaps the append's (programmatic
    // dependent launch); one launch with the append inside the attention kernel measured
    // slower in every arrangement tried
    auto st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = tkv::launch_append(c->dev, k, v, cls, pos, 1, st, &c->launches);
    c->live_ub = std::min<long long>(c->dev.ncap, c->live_ub + 1);
    if (e != cudaSuccess) return cuda_status(e, "tkv_decode_step");
    return launch_decode(c, q, softmax_scale, out, std::max(1ll, c->live_ub), st, "tkv_decode_step", true);
}

tkv_status tkv_decode_attention_sparsity(tkv_cache *c, const void *q, float softmax_scale, float *out,
                                         float *sparsity, uint8_t *thought, float th_r, float th_t, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (!q || !out || !sparsity) return fail(TKV_ERR_INVALID, "NULL q, out or sparsity");
    if (!aligned16(q) || !aligned16(out)) return fail(TKV_ERR_INVALID, "q and out must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(sparsity) & 3u) != 0) return fail(TKV_ERR_INVALID, "sparsity must be 4-byte aligned");
    if (!(th_r <= th_t) || !std::isfinite(th_r) || !std::isfinite(th_t))
        return fail(TKV_ERR_INVALID, "thresholds must be finite with th_r <= th_t");
    if (c->cfg.attn_kernel == 2)
        return fail(TKV_ERR_INVALID, "the sparsity statistic needs attn_kernel 0 or 1");
    const long long ub = std::max(1ll, c->live_ub);
    auto st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (c->cfg.attn_kernel == 1) {
        const tkv_status ms = ensure_maps(c);
        if (ms != TKV_OK) return ms;
        e = tkv::launch_attention_i8(c->dev, c->maps, q, softmax_scale, out, sparsity, thought, th_r, th_t, ub, st,
                                     &c->launches);
    } else {
        e = tkv::launch_attention(c->dev, q, softmax_scale, out, ub, st, &c->launches, sparsity, thought, th_r, th_t);
    }
    return cuda_status(e, "tkv_decode_attention_sparsity");
}

tkv_status tkv_evict_compact(tkv_cache *c, int32_t budget, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (budget < 0) return fail(TKV_ERR_INVALID, "budget must be >= 0");
    cudaError_t e = tkv::launch_evict(c->dev, budget, INT32_MAX, static_cast<cudaStream_t>(stream), &c->launches);
    const long long bound = (long long)budget + c->cfg.cap[0];
    c->live_ub = std::min(c->live_ub, bound);
    return cuda_status(e, "tkv_evict_compact");
}

tkv_status tkv_evict_compact_window(tkv_cache *c, int32_t budget, int32_t keep_from, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (budget < 0) return fail(TKV_ERR_INVALID, "budget must be >= 0");
    // the window's size is not known here, so the live-entry bound stays as it is
    cudaError_t e = tkv::launch_evict(c->dev, budget, keep_from, static_cast<cudaStream_t>(stream), &c->launches);
    return cuda_status(e, "tkv_evict_compact_window");
}

tkv_status tkv_evict_segments(tkv_cache *c, const int32_t *seg_start, const uint8_t *seg_label,
                              const int32_t *seg_keep, const int32_t *nseg, int32_t max_seg, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (max_seg < 0 || max_seg > tkv::evict_segments_max())
        return fail(TKV_ERR_INVALID, "max_seg must be in [0, 4096]");
    if (max_seg == 0) return TKV_OK;
    if (!seg_start || !seg_label || !seg_keep || !nseg) return fail(TKV_ERR_INVALID, "NULL segment array");
    auto a4 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
    if (!a4(seg_start) || !a4(seg_keep) || !a4(nseg)) return fail(TKV_ERR_INVALID, "int32 arrays must be 4-byte aligned");
    cudaError_t e = tkv::launch_evict_segments(c->dev, seg_start, seg_label, seg_keep, nseg, max_seg,
                                               static_cast<cudaStream_t>(stream), &c->launches);
    return cuda_status(e, "tkv_evict_segments");
}

tkv_status tkv_evict_tam(tkv_cache *c, const int32_t *seg_start, const uint8_t *seg_label, const int32_t *nseg,
                         int32_t max_seg, int32_t budget, double cpiv, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (max_seg < 0 || max_seg > tkv::evict_segments_max())
        return fail(TKV_ERR_INVALID, "max_seg must be in [0, 4096]");
    if (budget < 0) return fail(TKV_ERR_INVALID, "budget must be >= 0");
    if (!(cpiv >= 0.0) || !std::isfinite(cpiv)) return fail(TKV_ERR_INVALID, "c must be finite and >= 0");
    if (max_seg == 0) return TKV_OK;
    if (!seg_start || !seg_label || !nseg) return fail(TKV_ERR_INVALID, "NULL segment array");
    auto a4 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
    if (!a4(seg_start) || !a4(nseg)) return fail(TKV_ERR_INVALID, "int32 arrays must be 4-byte aligned");
    cudaError_t e = tkv::launch_evict_tam(c->dev, seg_start, seg_label, nseg, max_seg, budget, cpiv,
                                          static_cast<cudaStream_t>(stream), &c->launches);
    return cuda_status(e, "tkv_evict_tam");
}

tkv_status tkv_tbe_schedule(const uint8_t *label, int32_t nseg, int32_t r0, int32_t t_keep, int32_t *keep) {
    if (nseg < 0 || r0 < 0 || t_keep < 0) return fail(TKV_ERR_INVALID, "nseg, r0 and t_keep must be >= 0");
    if (nseg > 0 && (!label || !keep)) return fail(TKV_ERR_INVALID, "NULL array");
    for (int32_t j = 0; j < nseg; ++j)
        if (label[j] > 3) return fail(TKV_ERR_INVALID, "label must be 0..3");
    // one backward sweep: `later` = Transition segments after j
    int32_t later = 0;
    for (int32_t j = nseg - 1; j >= 0; --j) {
        int32_t r = -1;
        if (j != nseg - 1 && later > 0 && label[j] != 0)
            r = label[j] == 3 ? t_keep : (later - 1 < 31 ? (r0 >> (later - 1)) : 0);
        keep[j] = r;
        later += label[j] == 3;
    }
    return TKV_OK;
}

tkv_status tkv_poll_error(tkv_cache *c, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    auto st = static_cast<cudaStream_t>(stream);
    uint32_t w[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(w, c->dev.err, sizeof(w), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(c->dev.err, 0, sizeof(w), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e, "tkv_poll_error");
    if (w[0] == 0) return TKV_OK;
    char msg[160];
    std::snprintf(msg, sizeof(msg), "device error %u (%u occurrences, detail %u)", w[0], w[1], w[2]);
    return fail(static_cast<tkv_status>(w[0]), msg);
}

tkv_status tkv_export_state(tkv_cache *c, void *host_dst, void *stream) {
    if (!c || !host_dst) return fail(TKV_ERR_INVALID, "NULL argument");
    auto st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(host_dst, c->base, c->lay.state_bytes, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e, "tkv_export_state");
}

tkv_status tkv_import_state(tkv_cache *c, const void *host_src, void *stream) {
    if (!c || !host_src) return fail(TKV_ERR_INVALID, "NULL argument");
    auto st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(c->base, host_src, c->lay.state_bytes, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    // the live-entry bound from the imported counters: the largest stream's entry count
    const int32_t *n = reinterpret_cast<const int32_t *>(static_cast<const uint8_t *>(host_src) + c->lay.n);
    long long ub = 0;
    for (int s = 0; s < c->dev.S; ++s) {
        long long tot = 0;
        for (int k = 0; k < 4; ++k) tot += std::max<int32_t>(0, std::min(n[s * 4 + k], c->cfg.cap[k]));
        ub = std::max(ub, tot);
    }
    c->live_ub = ub;
    return cuda_status(e, "tkv_import_state");
}

tkv_status tkv_selftest_wait_timeout(tkv_cache *c, int64_t limit_cycles, void *stream) {
    if (!c) return fail(TKV_ERR_INVALID, "cache is NULL");
    if (limit_cycles < 1 || limit_cycles > (1ll << 31))
        return fail(TKV_ERR_INVALID, "limit_cycles must be in [1, 2^31]");
    cudaError_t e = tkv::launch_wait_timeout(c->dev, (long long)limit_cycles, static_cast<cudaStream_t>(stream),
                                             &c->launches);
    return cuda_status(e, "tkv_selftest_wait_timeout");
}

int64_t tkv_launch_count(const tkv_cache *c) { return c ? c->launches : 0; }

const char *tkv_last_error_string(void) { return g_last_error.c_str(); }

}  // extern "C"
