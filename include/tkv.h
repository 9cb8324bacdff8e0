/*
 * tkv.h -- C ABI of libtkv: one decode step of attention over a thought-adaptive
 * compressed KV cache (ThinKV-style), for NVIDIA B200 (sm_100a).
 *
 * The method (from the ThinKV page, sections "Metodologia" and
 * "Implementacao do Sistema"):
 *   - every token's K/V is group-quantised at a bit-width set by the thought
 *     type of its segment: Reasoning 8-bit, Execution 4-bit, Transition 2-bit
 *     (TBQ, "Think Before you Quantize"); tokens at positions below n_protect
 *     (attention sinks and the question window -- the DYNTS page, section 2.3,
 *     gives the question window infinite importance) stay bf16;
 *   - records live in paged per-precision pools and evicted slots are reused in
 *     place by new tokens of the same type, with no gather-based compaction
 *     (Continuous Thinking block table);
 *   - decode attention dequantises on the fly, and every token accumulates the
 *     attention mass it receives as its importance score (cumulative,
 *     H2O-style -- "Back from the Future", problem statement);
 *   - eviction keeps, per (batch, kv head) stream, the `budget` highest-scoring
 *     unprotected tokens (DYNTS page, section 2.3, selection window: keep the
 *     top-k, evict the rest), then compacts the block table.
 * Two segment-level policies share that compaction: tkv_evict_segments applies
 * per-segment retentions, such as the TBE annealing schedule (ThinKV,
 * "Metodologia", TBE) that tkv_tbe_schedule computes on the host; tkv_evict_tam
 * splits a budget over the segments as the TAM page's allocation rule does and
 * keeps its pivotal tokens.
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses; `stream` is a
 *     cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Calls are asynchronous on `stream` and never synchronise, except
 *     tkv_poll_error, tkv_export_state and tkv_import_state, which do.
 *   - The library never allocates device memory: the caller owns the workspace
 *     and every input/output buffer, and keeps them alive while work that uses
 *     them is in flight.  A tkv_cache is a small host object.
 *   - Argument errors are detected on the host, return TKV_ERR_INVALID and
 *     launch nothing.  Conditions only the device can see (a full pool, an
 *     invalid class id in device memory) skip the offending write, latch a
 *     device error word, and are reported by the next tkv_poll_error.
 *     Launch failures return TKV_ERR_CUDA.  tkv_last_error_string() describes
 *     the last non-OK status of the calling thread.
 *   - One cache may be used from one stream at a time; calls on one cache that
 *     overlap on the GPU race.
 */
#ifndef TKV_H
#define TKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TKV_API __attribute__((visibility("default")))
#else
#define TKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TKV_OK = 0,
    TKV_ERR_INVALID = 1,   /* bad argument (host) or bad class id (device) */
    TKV_ERR_CAPACITY = 2,  /* a pool had no free slot: token dropped       */
    TKV_ERR_CUDA = 3,      /* a CUDA runtime call or launch failed         */
    TKV_ERR_TIMEOUT = 4    /* a bounded device wait gave up                */
} tkv_status;

/* Thought classes.  Class 0 holds bf16 records (protected positions, or tokens
 * the caller labels 0); classes 1..3 hold Reasoning / Execution / Transition
 * tokens at bits[1..3]. */
enum { TKV_CLASS_BF16 = 0, TKV_CLASS_R = 1, TKV_CLASS_E = 2, TKV_CLASS_T = 3 };

typedef struct {
    int32_t B;           /* batch rows                                        */
    int32_t Hkv;         /* kv heads; a stream is s = b * Hkv + kv_head       */
    int32_t G;           /* query heads per kv head (1, 2, 4 or 8)            */
    int32_t D;           /* head dim: must be 128                              */
    int32_t group;       /* quantisation group along head dim: must be 32      */
    int32_t bits[4];     /* must be {16, 8, 4, 2}                              */
    int32_t n_protect;   /* positions [0, n_protect) are bf16, never evicted   */
    int32_t cap[4];      /* slots per stream for each class (>= 0)             */
    int32_t max_append;  /* largest T accepted by tkv_quantize_append (>= 1)   */
    int32_t dense;       /* placement: 0 = evicted slots are reused in place
                            (free stacks, the pages' Continuous Thinking);
                            1 = dense: eviction moves each kept record to the
                            slot equal to its table index and appends always
                            take the next never-used slot, so a class's live
                            records are contiguous in table order (handle[i] ==
                            i) and decode reads them as whole blocks.  Results
                            are identical in both modes.                      */
    int32_t attn_kernel; /* decode-attention kernel: 0 = warp-tile kernel
                            (mma.sync fragments, either placement; a few long
                            streams are each split over more CTAs than a
                            cluster holds and merged by a second pass);
                            1 = tensor-core kernel (tcgen05 MMAs with integer
                            operands: exact code products, accumulators in
                            tensor memory; persistent, one CTA per SM with the
                            step's bytes split evenly; dense placement only);
                            2 = the warp-tile math fed by a persistent TMA
                            pipeline (two CTAs per SM, the step's bytes split
                            evenly; dense placement only).  All compute the
                            same result within the stated tolerances.       */
    int32_t codec;       /* class record formats: 0 = integer codes (classes
                            1/2/3: 8/4/2-bit asymmetric, fp16 scale and zero
                            per group); 1 = floating-point codes (class 1 FP8
                            E4M3, class 2 NVFP4: E2M1 with an E4M3 scale per
                            16 dims, class 3 ternary {0, +1, -1}; FP8 and
                            ternary with an fp16 scale per group).  Codec 1
                            needs attn_kernel 0.                              */
} tkv_config;

typedef struct tkv_cache tkv_cache;

/* Byte offsets of the state arrays inside the workspace (all 256-byte aligned),
 * so a caller can inspect or checkpoint the cache with plain copies.
 * Per stream s and class c:
 *   n[s*4+c], ft[s*4+c], hw[s*4+c]  int32: live entries, free-stack top, next never-used slot
 *   handle_c[s*cap_c + i]           int32: slot of table entry i (i < n), entries in append order
 *   pos_c[s*cap_c + i]              int32: token position of entry i
 *   score_c[s*cap_c + i]            float: accumulated attention mass of entry i
 *   fs_c[s*cap_c + j]               int32: free stack of slots (j < ft; top = j = ft-1)
 *   pool_c[(s*cap_c + slot)*rec_bytes_c]  packed record of a slot:
 *     bf16 class: [K block: D bf16][V block: D bf16]                     (512 bytes)
 *     b-bit class: [K codes D*b/8][V codes D*b/8][K scale x4][K zero x4]
 *                  [V scale x4][V zero x4]  (fp16, little-endian)        (288/160/96 bytes)
 *     Scale and zero of group g (head dims 32g..32g+31) are entry g of their x4.
 *     codec 1 (floating-point codes, same element order as the b-bit classes):
 *       class 1 FP8:    [K E4M3 codes D][V codes D][K scale x4][V scale x4] (fp16)  (272 bytes)
 *       class 2 NVFP4:  [K E2M1 codes D/2][V codes D/2][K scale x8][V scale x8]
 *                       (E4M3; scale j covers head dims 16j..16j+15)       (144 bytes)
 *       class 3 ternary:[K codes D/4][V codes D/4][K scale x4][V scale x4] (fp16; code
 *                       1 = +scale, 3 = -scale, 0 = 0)                     (80 bytes)
 *   Element order inside a K or V block (b = 16 for bf16, else the class's bits):
 *   the block is four quarters of 4*b bytes (quarter q = bytes [4bq, 4b(q+1)));
 *   a quarter is b little-endian 32-bit words; word w of a quarter holds the
 *   16/b head-dim pairs p = w*(16/b) + j, j = 0 .. 16/b - 1, with the pair's first
 *   member in bits [b*j, b*j + b) and its second member 16 bits higher, in bits
 *   [b*j + 16, b*j + 16 + b).  Pair p of quarter q holds head dims
 *     K block: 32*(p/4) + 8*q + 2*(p%4) + {0, 1}
 *     V block: 8*p + 2*q + {0, 1}
 *   (first member = the even dim).  Example (K, b = 8): byte 0 of the block holds
 *   dim 0, byte 1 dim 2, byte 2 dim 1, byte 3 dim 3, byte 4 dim 4, byte 8 dim 32.
 * The state region [0, state_bytes) holds all of the above; the rest of the
 * workspace is scratch. */
typedef struct {
    size_t n, ft, hw, err;
    size_t handle[4], pos[4], score[4], fs[4], pool[4];
    int32_t rec_bytes[4];
    size_t state_bytes;
    size_t total_bytes;
} tkv_layout;

/* Bytes of device workspace a cache with this configuration needs (0 if the
 * configuration is invalid). */
TKV_API size_t tkv_workspace_bytes(const tkv_config *cfg);

/* Create a cache over a caller-owned device workspace of at least
 * tkv_workspace_bytes(cfg) bytes, 256-byte aligned.  The cache starts empty
 * once tkv_reset has run on a stream (tkv_create does not touch the device). */
TKV_API tkv_status tkv_create(const tkv_config *cfg, void *d_workspace, size_t workspace_bytes,
                      tkv_cache **out);

/* Free the host object.  The workspace stays the caller's. */
TKV_API tkv_status tkv_destroy(tkv_cache *cache);

/* Empty the cache: zero every counter (n, ft, hw) and the device error word. */
TKV_API tkv_status tkv_reset(tkv_cache *cache, void *stream);

/* Workspace offsets of the state arrays (see tkv_layout). */
TKV_API tkv_status tkv_get_layout(const tkv_cache *cache, tkv_layout *out);

/*
 * Quantise and append T new tokens per stream (ThinKV, TBQ; Continuous
 * Thinking slot reuse).
 *   k, v   device bf16 [B][Hkv][T][D]  keys / values of the new tokens
 *   cls    device uint8 [B][T]          thought class 1 (R), 2 (E), 3 (T) or 0 (bf16)
 *   pos    device int32 [B][T]          absolute positions
 *   T      1 <= T <= max_append
 * Per stream, tokens are taken in t order.  A token at pos < n_protect is
 * stored in class 0.  For b-bit classes each group of 32 elements gets
 * zero = fp16 round-down(min), scale = fp16 round-up((max - zero)/(2^b-1)),
 * code = round-half-even((x - zero)/scale) in fp32 clamped to [0, 2^b-1]
 * (all codes 0 when scale == 0).  Its slot is popped from the stream's free
 * stack of that class if non-empty, else the next never-used slot; a token that
 * finds neither is dropped (device error TKV_ERR_CAPACITY), and a class id > 3
 * drops the token (device error TKV_ERR_INVALID).  New entries start with
 * score 0.
 */
TKV_API tkv_status tkv_quantize_append(tkv_cache *cache, const void *k, const void *v,
                               const uint8_t *cls, const int32_t *pos, int32_t T, void *stream);

/*
 * tkv_quantize_append without any scratch memory of the caller's (the paper has
 * no counterpart: this is a deployment variant).  Same arguments, semantics and
 * results as tkv_quantize_append, for callers that cannot allocate device memory
 * and so cannot size a workspace scratch for their largest append -- e.g. code
 * running where cudaMalloc is not allowed or an allocator must not grow.  The
 * per-token class ranks of a multi-token append live in a fixed 2 MiB device
 * array inside the library instead (held by every GPU that loads the library
 * until the process exits); it calls no allocating function.
 *   Limit: B * (T + 4) <= 524288 when T > 1 (T == 1 needs no scratch);
 *          larger appends return TKV_ERR_INVALID and launch nothing.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and keeps it for that device's current context; make
 *   that first call before any stream capture, and do not use this entry point
 *   after cudaDeviceReset in the same process.
 *   All calls share the one array and each call rewrites what it uses, so calls
 *   that overlap on the GPU (two streams, or two caches at once) race.
 */
TKV_API tkv_status tkv_quantize_append_noalloc(tkv_cache *cache, const void *k, const void *v,
                                       const uint8_t *cls, const int32_t *pos, int32_t T,
                                       void *stream);

/*
 * One decode step of GQA attention over every live token of every stream
 * (dequantised on the fly), plus score accumulation.
 *   q              device bf16 [B][Hkv*G][D]; query head h reads kv head h / G
 *   softmax_scale  logit = softmax_scale * (q . k_hat)   (typically D^-1/2)
 *   out            device fp32 [B][Hkv*G][D]: sum_t softmax_t(logit) * v_hat_t
 * Every live token t of stream s then gets score_t += sum over the G query
 * heads of s of its softmax weight.  An empty stream yields a zero output.
 */
TKV_API tkv_status tkv_decode_attention(tkv_cache *cache, const void *q, float softmax_scale,
                                float *out, void *stream);

/*
 * One decode step with its new token: exactly tkv_quantize_append with T = 1
 * (k, v, cls, pos as there: k, v device bf16 [B][Hkv][D], cls uint8 [B], pos
 * int32 [B]) followed by tkv_decode_attention (q, softmax_scale, out as there),
 * so the step attends over the new token too, in one call: the two launches go
 * back to back, the attention's launch overlapping the append (programmatic
 * dependent launch; the attention reads q while the append runs, which is safe for
 * any q the caller's earlier work on `stream` produced, since the append starts
 * only after that work).  Results, device errors and the cache state are those of
 * the two calls.  The ThinKV page's decode loop (Implementacao do Sistema) writes each
 * new token into the block table the same step reads.
 * Returns TKV_ERR_INVALID (launching nothing) for a NULL pointer or k, v, pos, q,
 * out not 16-byte aligned.
 */
TKV_API tkv_status tkv_decode_step(tkv_cache *cache, const void *k, const void *v, const uint8_t *cls,
                                   const int32_t *pos, const void *q, float softmax_scale, float *out,
                                   void *stream);

/*
 * tkv_decode_attention plus, per (stream, query head), the attention sparsity of
 * this step and the thought type it indicates (ThinKV page, "Metodologia": the
 * thought types differ in how sparse their attention is -- Transition the most,
 * Execution the least).  The page gives no measure and no thresholds; this library
 * uses the normalised entropy of the step's softmax over the stream's N live tokens:
 *   sparsity = 1 - H(p) / ln N,   H(p) = -sum_t p_t ln p_t   (0 when N < 2),
 * which is 0 for uniform attention and 1 for attention on one token, and the class
 *   3 (Transition) if sparsity >= th_t, else 1 (Reasoning) if sparsity >= th_r,
 *   else 2 (Execution).
 *   sparsity  device fp32 [B][Hkv*G]  (required)
 *   thought   device uint8 [B][Hkv*G] (may be NULL)
 * Requires attn_kernel 0 (either placement; the score pass forms the statistic from the
 * exp2(x - M) it computes anyway) or 1; returns TKV_ERR_INVALID with attn_kernel 2, for
 * NULL q / out / sparsity, unaligned pointers, or thresholds that are not finite with
 * th_r <= th_t.
 */
TKV_API tkv_status tkv_decode_attention_sparsity(tkv_cache *cache, const void *q, float softmax_scale,
                                                 float *out, float *sparsity, uint8_t *thought, float th_r,
                                                 float th_t, void *stream);

/*
 * Budgeted top-k eviction and table compaction, per stream.
 *   budget  >= 0: unprotected tokens kept per stream.
 * Entries with pos < n_protect are always kept.  Among the others the `budget`
 * first under the order (score descending, then position ascending, then
 * class, then table index) are kept; the rest are evicted.  Each class table
 * keeps its survivors in their previous order with their scores; evicted
 * slots are pushed on the class's free stack in reverse table order, so the
 * earliest evicted entry is reused first.  A stream with <= budget
 * unprotected tokens is untouched.  In dense placement (cfg.dense = 1) the kept
 * records are instead moved to the slots equal to their new table indices, the
 * free stack stays empty and the next never-used slot becomes the entry count;
 * dense placement requires handle[i] == i on entry (which it maintains).
 */
TKV_API tkv_status tkv_evict_compact(tkv_cache *cache, int32_t budget, void *stream);

/* tkv_evict_compact with a local window ("DYNTS", section 2.3: the most recently
 * generated tokens are kept for local coherence): entries at positions >= keep_from
 * are kept too and are not candidates, so `budget` applies to positions in
 * [n_protect, keep_from) only.  keep_from = INT32_MAX is tkv_evict_compact.  Returns
 * TKV_ERR_INVALID for a NULL cache or budget < 0. */
TKV_API tkv_status tkv_evict_compact_window(tkv_cache *cache, int32_t budget, int32_t keep_from, void *stream);

/* Segment-level eviction ("ThinKV", section Metodologia, TBE paragraph: when a
 * Transition thought starts, tokens of earlier R/E thought segments are evicted
 * progressively on an annealing schedule, at the granularity of segments).
 *
 * Row b of the segment arrays (row stride max_seg, device memory) describes batch
 * row b: nseg[b] segments (values outside [0, max_seg] are clamped); segment j
 * starts at position seg_start[b*max_seg + j] (strictly increasing) and ends where
 * segment j + 1 starts, the last one is open; its tokens are stored in class
 * seg_label[...] (0 bf16, 1 R, 2 E, 3 T); seg_keep[...] is its retention (-1 keeps
 * the segment whole, r >= 0 keeps r tokens).  For every stream (b, kv head) an
 * entry is kept when its position is below n_protect, lies before the first
 * segment, or its class differs from its segment's label; the other entries of
 * segment j are ranked by (score desc, position asc, table index asc) and the
 * first seg_keep of them are kept.  The tables are then compacted exactly as by
 * tkv_evict_compact.  Class tables must be ordered by position (appends in
 * position order guarantee it).  The call uses the decode step's logits scratch
 * (no other device memory).  Returns TKV_ERR_INVALID for a NULL cache, NULL arrays
 * (when max_seg > 0), unaligned int32 arrays or max_seg outside [0, 4096];
 * max_seg == 0 is a no-op. */
TKV_API tkv_status tkv_evict_segments(tkv_cache *cache, const int32_t *seg_start, const uint8_t *seg_label,
                                      const int32_t *seg_keep, const int32_t *nseg, int32_t max_seg,
                                      void *stream);

/* Thought-aware segment budgets with pivotal-token protection (page "Compactacao de
 * Cache KV Consciente do Pensamento para Raciocinio via Correspondencia de Atencao
 * Adaptativa" (TAM), sections 2.B and 2.C), as a selection policy over the
 * accumulated scores.  Segment arrays as for tkv_evict_segments (no retention
 * array).  For every stream: the candidates of segment j are its unprotected
 * entries in its label's class; w_j is their mean score and n_j their number; a
 * candidate scoring at least c times the mean score of all the stream's candidates
 * is pivotal and kept; the remaining budget T' = max(0, budget - pivotal) gives
 * segment j t_j = min(n_j - pivotal_j, floor(T' * (a_j / D) + 1e-9)) of its other
 * candidates, a_j = sqrt(w_j) * n_j, D = sum a_j (fp64), chosen as in
 * tkv_evict_segments; entries outside every segment's candidates are kept.  The
 * page's attention-matching refit of the kept keys is not performed.  Returns
 * TKV_ERR_INVALID for a NULL cache or array (when max_seg > 0), unaligned int32
 * arrays, max_seg outside [0, 4096], budget < 0, or c negative or not finite. */
TKV_API tkv_status tkv_evict_tam(tkv_cache *cache, const int32_t *seg_start, const uint8_t *seg_label,
                                 const int32_t *nseg, int32_t max_seg, int32_t budget, double c, void *stream);

/* Retention of each of the nseg thought segments of one batch row (labels 0 bf16,
 * 1 R, 2 E, 3 T, host memory; the last segment is the open one) under the TBE
 * annealing schedule, written to keep[0..nseg) (host memory).  Reading of the
 * page: with k the number of Transition segments after segment j, the open
 * segment, a bf16-labelled segment and any segment with k = 0 keep everything
 * (-1); a completed R or E segment keeps r0 >> (k - 1) tokens (64, 32, 16, ...
 * for r0 = 64); a completed T segment with k >= 1 keeps t_keep (the safety net of
 * Transition tokens).  Host only: no GPU, no cache.  Returns TKV_ERR_INVALID for
 * NULL arrays (when nseg > 0), nseg < 0, r0 < 0, t_keep < 0 or a label above 3. */
TKV_API tkv_status tkv_tbe_schedule(const uint8_t *label, int32_t nseg, int32_t r0, int32_t t_keep,
                                    int32_t *keep);

/* Synchronise `stream`, read and clear the device error word; returns the
 * first device-side status latched since the last poll (TKV_OK if none). */
TKV_API tkv_status tkv_poll_error(tkv_cache *cache, void *stream);

/* Copy the state region (see tkv_layout) to / from a host buffer of
 * state_bytes bytes (the buffer is the caller's; the state is the cache's
 * checkpoint: counters, tables, scores, free stacks and records).  Both
 * synchronise `stream`.  Import also derives the host-side launch bound (the
 * largest stream's entry count) from the imported counters, so a cache restored
 * from a checkpoint launches exactly as the cache it was taken from would after
 * the same import.  Returns TKV_ERR_INVALID for NULL arguments. */
TKV_API tkv_status tkv_export_state(tkv_cache *cache, void *host_dst, void *stream);
TKV_API tkv_status tkv_import_state(tkv_cache *cache, const void *host_src, void *stream);

/* Self-test of the bounded device waits; the pages have no counterpart (it checks
 * this library's failure reporting).  Launches, on `stream`, a one-warp kernel that
 * waits on a barrier nothing ever arrives on; after limit_cycles SM cycles (1 ..
 * 2^31) the wait gives up and TKV_ERR_TIMEOUT is latched in the cache's device error
 * word -- the same path a decode kernel takes when a copy never completes -- and the
 * next tkv_poll_error reports it.  The cache's state is not touched; the context stays
 * usable.  Returns TKV_ERR_INVALID for a NULL cache or a limit out of range. */
TKV_API tkv_status tkv_selftest_wait_timeout(tkv_cache *cache, int64_t limit_cycles, void *stream);

/* Launch counters since tkv_create (kernels this cache has launched). */
TKV_API int64_t tkv_launch_count(const tkv_cache *cache);

/* Human-readable description of the calling thread's last non-OK status. */
TKV_API const char *tkv_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* TKV_H */
