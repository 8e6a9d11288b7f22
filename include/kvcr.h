/*
 * kvcr.h -- C ABI of the sink + window chunk-attention library for B200 (sm_100a).
 *
 * The library implements the attention hot path of chunk-wise autoregressive
 * video world models:
 *
 *   - a per-layer KV cache of pinned anchor ("sink") latent frames followed by
 *     a sliding window of recent finalized frames, with eviction of the oldest
 *     non-anchor frame ("LingBot-World-Infinity: The Open-Source World Model
 *     That Refuses to Forget", sections "The trick: treat video like a causal
 *     stream" and "How the cache keeps the world alive"; "Westlake AGI Lab's
 *     'World in World' Steers Frozen Video Models", second paragraph: 6 anchor
 *     + 8 recent + 4 current latent-frame slots);
 *   - 3D (t, h, w) rotary embedding of K applied when a frame is written;
 *   - chunk attention: the current chunk's queries attend the anchors, the
 *     window and the chunk itself;
 *   - attention under the MoBA training mask ("Infinite Worlds with Versatile
 *     Interactions", causal-pretraining paragraph; "Mix Forcing: Causal
 *     Pre-Training via Mixture Attention for Interactive World Models",
 *     "Mix the training modes").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every call returns a kvcr_status.  On a non-OK return nothing was launched
 *    and no state changed; kvcr_last_error() gives a message (thread-local).
 *  - Tensors are dense, row-major, token-major: [tokens][heads][head_dim], in
 *    the cache's dtype (bf16 or fp32).  Device pointers must be 16-byte
 *    aligned.  Tokens of one latent frame are row-major over the (h, w) patch
 *    grid; frames follow each other in ascending frame order.
 *  - "stream" is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Device work is asynchronous on that stream; no call synchronises the host
 *    except kvcr_check_status() and kvcr_trace_read().  Inputs must stay valid
 *    until the stream has consumed them.
 *  - Host-side bookkeeping (slot table, frame order) never reads device memory.
 *  - The library never allocates device memory: the cache lives in one
 *    caller-owned device buffer of kv_cache_storage_bytes() bytes.
 *  - All compute runs in the library's own CUDA kernels; there is no CPU
 *    fallback.
 *  - A failure inside a kernel (a bounded wait that ran out) happens after the
 *    launching call has returned KVCR_OK: poll kvcr_check_status() after the
 *    stream's work to learn of it; until then the outputs of that work are
 *    not to be trusted.  Besides KVCR_ETIMEOUT, the MoBA backward's dQ kernel
 *    records two self-checks there, neither expected on sm_100: KVCR_EUNSUPPORTED
 *    when its shared-memory layout does not fit the block's dynamic shared
 *    memory after alignment, KVCR_ESTATE when its enumeration of key tiles
 *    disagrees with its own count; the kernel then stops without touching dQ.
 */
#ifndef KVCR_H
#define KVCR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVCR_OK = 0,
    KVCR_EINVAL = -1,      /* null pointer, misaligned pointer, bad scalar argument */
    KVCR_ESHAPE = -2,      /* sizes inconsistent with the cache or out of supported range */
    KVCR_ESTATE = -3,      /* call not valid in the cache's state (frame order, no storage) */
    KVCR_ECUDA = -4,       /* a CUDA runtime / driver call failed */
    KVCR_ETIMEOUT = -5,    /* a kernel gave up on a bounded wait (reported by kvcr_check_status) */
    KVCR_ESTORAGE = -6,    /* caller storage too small or misaligned */
    KVCR_EUNSUPPORTED = -7 /* dtype / head_dim combination not built */
} kvcr_status;

typedef enum { KVCR_BF16 = 0, KVCR_F32 = 1 } kvcr_dtype;

/* 3D rotary embedding of a cache.  head_dim is cut into head_dim/2 interleaved
 * pairs (x[2i], x[2i+1]); the first pairs_t pairs rotate with the absolute
 * latent-frame index t, the next pairs_h with the patch row h, the last pairs_w
 * with the patch column w.  In an axis owning P pairs, pair j turns by
 * pos * base^(-2j / (2P)).  pairs_t + pairs_h + pairs_w == head_dim / 2 and
 * grid_h * grid_w == tokens_per_frame.  Angles are computed on the host in
 * double precision.  The 832x464 workload uses 22/21/21 pairs (44/42/42 dims)
 * at head_dim 128, base 10000. */
typedef struct {
    int grid_h, grid_w;
    int pairs_t, pairs_h, pairs_w;
    double base;
} kvcr_rope;

/* MoBA training sequence [C1..Cn | N1..Nn | B], each C/N chunk chunk_tokens long
 * and B n_bidir_chunks * chunk_tokens long.  Mask: a query of C_i reads C_j for
 * j <= i; a query of N_i reads C_j for j < i and N_i; a query of B reads B. */
typedef struct {
    int n_chunks;
    int chunk_tokens;
    int n_bidir_chunks;
} kvcr_moba_layout;

/* Tile classes returned by moba_classify_tiles. */
enum { KVCR_TILE_EMPTY = 0, KVCR_TILE_PARTIAL = 1, KVCR_TILE_FULL = 2 };

typedef struct kvcr_cache kvcr_cache;

/* ---------------------------------------------------------------- cache --- */

/* The cache is the per-layer KV store of a chunk-wise causal video stream:
 * anchor tokens kept at the front plus a sliding window of recent frames
 * ("LingBot-World-Infinity: The Open-Source World Model That Refuses to
 * Forget", "How the cache keeps the world alive"; "Westlake AGI Lab's 'World
 * in World' Steers Frozen Video Models", second paragraph: 6 anchor + 8
 * recent latent-frame slots).
 *
 * Bytes of device storage a cache needs: K and V of sinks+window frame slots,
 * and, when with_rope != 0, scratch for the rotated queries and current-chunk
 * keys of one chunk (chunk_frames frames) plus the (h, w) angle tables.
 * Returns 0 for invalid sizes. */
size_t kv_cache_storage_bytes(int sinks, int window, int tokens_per_frame, int heads,
                              int head_dim, int chunk_frames, int with_rope,
                              kvcr_dtype dtype);

/* Create a cache.  sinks anchor slots + window recent slots; frames of
 * tokens_per_frame tokens; heads x head_dim per token; chunk_frames = most
 * frames in one current chunk.  rope = NULL disables rotary embedding (keys and
 * queries are used as given, e.g. for text cross-attention).  device_storage /
 * storage_bytes: a caller-owned device buffer (>= kv_cache_storage_bytes, 256-
 * byte aligned) that must outlive the cache; the library writes the angle
 * tables into it here (synchronously).  device_storage = NULL with
 * storage_bytes = 0 creates a bookkeeping-only cache: the slot table works,
 * kv_cache_append_rope() must then be given k = v = NULL and launches nothing,
 * and attention calls return KVCR_ESTATE.  Supported: bf16 with head_dim 64 or
 * 128 (tensor-core path), fp32 with head_dim 64 or 128 (fp32 CUDA-core path);
 * sinks + window <= 32.  *out receives the handle. */
int kv_cache_init(kvcr_cache **out, int sinks, int window, int tokens_per_frame, int heads,
                  int head_dim, int chunk_frames, const kvcr_rope *rope, kvcr_dtype dtype,
                  void *device_storage, size_t storage_bytes);

/* Caches with auxiliary slots: temporary attention blocks that carry extra
 * evidence for the current chunk and are removed once it is finalized ("Westlake
 * AGI Lab's 'World in World' Steers Frozen Video Models", second paragraph:
 * source-video observations, target-view projections, rendered geometry,
 * retrieved history, read through the backbone's own attention).  aux_frames
 * more frame slots (sinks + window + aux_frames <= 32) follow the anchor and
 * window slots in the storage; everything else is as for kv_cache_storage_bytes()
 * and kv_cache_init(), which are these with aux_frames = 0. */
size_t kv_cache_storage_bytes_aux(int sinks, int window, int aux_frames, int tokens_per_frame,
                                  int heads, int head_dim, int chunk_frames, int with_rope,
                                  kvcr_dtype dtype);
int kv_cache_init_aux(kvcr_cache **out, int sinks, int window, int aux_frames,
                      int tokens_per_frame, int heads, int head_dim, int chunk_frames,
                      const kvcr_rope *rope, kvcr_dtype dtype, void *device_storage,
                      size_t storage_bytes);

/* Write n_frames auxiliary frames for the current chunk, replacing any set
 * before: k, v device [n_frames * tokens_per_frame][heads][head_dim].  With a
 * RoPE cache and aux_pos != NULL (host, n_frames temporal positions >= 0, e.g. the
 * evidence's event time), K is rotated by RoPE3D at (aux_pos[f], h, w); with
 * aux_pos = NULL (or a cache without RoPE), K is stored as given.  V as is.
 * Every chunk_attention_fwd*() call then reads them after the cached frames,
 * until the next kv_cache_append_rope() (the chunk's finalization) drops them;
 * they never enter the anchor / window slots and are never evicted.  0 <=
 * n_frames <= aux_frames (n_frames = 0 drops them now).  Bookkeeping-only
 * caches take k = v = NULL.  Errors: KVCR_ESHAPE (n_frames), KVCR_EINVAL (NULL or
 * misaligned k / v, negative position), KVCR_ESTATE; nothing changes on error. */
int kv_cache_set_aux(kvcr_cache *c, const void *k, const void *v, const int32_t *aux_pos,
                     int n_frames, void *stream);

/* Cache flags of kv_cache_init_ex(). */
enum {
    /* Keep, beside the bf16 K of every cached and auxiliary frame, an e4m3 copy of
     * it with one fp32 scale per block of 128 tokens and head, written by the same
     * append / set_aux call; chunk_attention_fwd_fp8() reads it.  Needs bf16 and
     * head_dim 128. */
    KVCR_CACHE_FP8_K = 1,
    /* Keep chunk_frames spare frame slots so that chunk_attention_fwd_finalize()
     * can write the chunk's rotated K and its V straight into cache storage while
     * the frames they replace are still read (see there).  bf16 caches. */
    KVCR_CACHE_FUSED_FINALIZE = 2
};

/* kv_cache_storage_bytes_aux() / kv_cache_init_aux() with cache flags (0,
 * KVCR_CACHE_FP8_K or KVCR_CACHE_FUSED_FINALIZE, not both).  With
 * KVCR_CACHE_FP8_K the storage also holds the e4m3 K copies (T * H * D bytes per
 * frame slot), their scales (4 * ceil(T / 128) * H bytes per slot) and the e4m3
 * staging of one chunk's queries and keys; with KVCR_CACHE_FUSED_FINALIZE,
 * chunk_frames more K / V frame slots (sinks + window + aux_frames + chunk_frames
 * <= 32).  kv_cache_init_ex returns KVCR_EUNSUPPORTED for KVCR_CACHE_FP8_K with
 * fp32 or head_dim 64 and for KVCR_CACHE_FUSED_FINALIZE with fp32, KVCR_EINVAL
 * for unknown or combined flags. */
size_t kv_cache_storage_bytes_ex(int sinks, int window, int aux_frames, int tokens_per_frame,
                                 int heads, int head_dim, int chunk_frames, int with_rope,
                                 kvcr_dtype dtype, unsigned flags);
int kv_cache_init_ex(kvcr_cache **out, int sinks, int window, int aux_frames,
                     int tokens_per_frame, int heads, int head_dim, int chunk_frames,
                     const kvcr_rope *rope, kvcr_dtype dtype, unsigned flags,
                     void *device_storage, size_t storage_bytes);

/* Number of auxiliary frames the next attention call reads (0 after the chunk's
 * append; see kv_cache_set_aux).  Host only; KVCR_EINVAL for NULL arguments. */
int kv_cache_num_aux(const kvcr_cache *c, int *n);

/* Append finalized frames (the last denoising step's K and V); this finalizes the
 * chunk, so its auxiliary frames (kv_cache_set_aux) are dropped.  Each generated
 * chunk's state is appended, the oldest non-anchor state evicted and the anchors
 * kept ("LingBot-World-Infinity", "The trick: treat video like a causal stream").
 * k, v: device [n_frames * tokens_per_frame][heads][head_dim].  frame_idx: host,
 * n_frames strictly increasing absolute latent-frame indices, each larger than
 * every frame appended before.  Frame by frame: an unfilled anchor slot is taken
 * first; else, when the window holds `window` frames, the oldest non-anchor
 * frame is evicted and its slot reused; else the lowest free window slot is
 * taken.  K is written rotated (RoPE3D at its absolute (t, h, w)), V as is.
 * A frame evicted by a later frame of the same call is not written.
 * n_frames = 0 is a no-op. */
int kv_cache_append_rope(kvcr_cache *c, const void *k, const void *v,
                         const int32_t *frame_idx, int n_frames, void *stream);

/* kv_cache_append_rope() of the same frames into several caches (e.g. every
 * layer's cache at the end of a chunk) in one launch.  The slot rules are those
 * of kv_cache_append_rope(); batching the layers follows the launch-count
 * reduction of kaarelkaarelson.com/lingbot (step table: ~20 000 -> ~4 800
 * launches per chunk).  caches: host array of
 * n_caches distinct handles with the same tokens_per_frame, heads, head_dim,
 * dtype and RoPE (and all with storage, or all bookkeeping-only); k[i], v[i]:
 * device [n_frames * tokens_per_frame][heads][head_dim] for cache i (host
 * arrays of device pointers; NULL arrays for bookkeeping-only caches).  Each
 * cache's slot table, written K / V and last-append record end up exactly as
 * after kv_cache_append_rope() on it alone.  n_caches * n_frames <= 256.  Errors
 * (checked for every cache before anything changes): KVCR_EINVAL, KVCR_ESHAPE
 * (mismatched caches, sizes), KVCR_ESTATE (frame order). */
int kv_cache_append_rope_batch(kvcr_cache *const *caches, int n_caches, const void *const *k,
                               const void *const *v, const int32_t *frame_idx, int n_frames,
                               void *stream);

/* Dynamic window: evict the oldest non-anchor frames until at most keep_recent
 * remain (0 <= keep_recent <= window).  Host only.  This is the hook of a
 * dynamic KV-cache scheduler that adapts the retained history to the current
 * control signal ("Infinite Worlds with Versatile Interactions", deployment
 * paragraph).  evicted_out (nullable) receives
 * up to evicted_cap evicted frame indices, oldest first; *n_evicted (nullable)
 * the number evicted. */
int kv_cache_evict(kvcr_cache *c, int keep_recent, int32_t *evicted_out, int evicted_cap,
                   int *n_evicted);

/* Slot table: frame_of_slot[s] = frame cached in slot s or -1, s < sinks+window
 * (the anchor and recent slots of "World in World", second paragraph); cap =
 * length of frame_of_slot (>= sinks + window).  Host only. */
int kv_cache_slot_map(const kvcr_cache *c, int32_t *frame_of_slot, int cap);

/* Result of the last append: slot of each appended frame (-1 = not retained)
 * and the frames it evicted (oldest first).  A read-back of the slot rules
 * above; no page has a counterpart (library convention).  Host only. */
int kv_cache_last_append(const kvcr_cache *c, int32_t *slots, int slots_cap,
                         int32_t *evicted, int evicted_cap, int *n_evicted);

/* Number of cached frames (library convention; host only). */
int kv_cache_num_cached(const kvcr_cache *c, int *n);

/* Device addresses of the e4m3 copy of slot `slot`'s K: codes [tokens_per_frame]
 * [heads][head_dim] (one byte each; the block of tokens 128 b .. 128 b + 127 and
 * head h dequantizes to code * scales[b * heads + h]) and scales fp32
 * [ceil(tokens_per_frame / 128)][heads].  Only for caches made with
 * KVCR_CACHE_FP8_K (else KVCR_ESTATE).  For reading back or checking the copy. */
int kv_cache_slot_data_fp8(const kvcr_cache *c, int slot, const void **k_codes,
                           const float **k_scales);

/* Device addresses of slot `slot`'s K and V, each [tokens_per_frame][heads][head_dim]
 * in the cache dtype (K stored rotated).  For reading back or saving a cache.
 * Slots sinks + window .. + aux_frames - 1 are the auxiliary slots. */
int kv_cache_slot_data(const kvcr_cache *c, int slot, const void **k, const void **v);

/* Checkpoint of a cache's host state: the slot table, the anchors filled, the window's
 * recency order, the last frame index, the physical relabelling of a fused-finalize
 * cache, the auxiliary count and the last append's record.  Together with a copy of
 * the caller-owned device storage it restores a cache after a restart without
 * replaying its appends (library convention; the pages describe the state, not a
 * format).  Export: *size receives the byte count; buf = NULL only queries it;
 * KVCR_ESTORAGE when cap < *size.  Import into a cache created with the same
 * configuration (sizes, dtype, RoPE, flags): KVCR_ESHAPE for another configuration,
 * KVCR_EINVAL for a truncated or inconsistent state; nothing changes on error.  The
 * format is little-endian int32 words headed by "KVCR" and a version.  Host only. */
int kv_cache_export_state(const kvcr_cache *c, void *buf, size_t cap, size_t *size);
int kv_cache_import_state(kvcr_cache *c, const void *buf, size_t size);

void kv_cache_destroy(kvcr_cache *c);

/* ------------------------------------------------------------ attention --- */

/* Chunk attention: O = softmax(scale * Q K^T) V where the keys are every cached
 * frame (anchors and window) followed by the current chunk's own n_cur_frames
 * frames; full attention inside the chunk.  The block reads the anchor slots,
 * the recent slots and the current chunk ("Westlake AGI Lab's 'World in World'
 * Steers Frozen Video Models", second paragraph: 6 + 8 + 4 latent-frame slots;
 * "LingBot-World-Infinity", "How the cache keeps the world alive").
 *   q:     device [n_q][heads][head_dim]; with RoPE, n_q must equal
 *          n_cur_frames * tokens_per_frame (the chunk's tokens) and Q is rotated
 *          at the chunk's positions; without RoPE n_q is free (cross-attention).
 *   k_cur, v_cur: device [n_cur_frames * tokens_per_frame][heads][head_dim].
 *   cur_frame_idx: host, strictly increasing, larger than every cached frame.
 *   softmax_scale <= 0 means 1/sqrt(head_dim).
 *   o:     device [n_q][heads][head_dim] in the cache dtype.
 *   lse:   nullable device fp32 [heads][n_q], natural-log sum of exp of scores.
 * The cache is read, not changed. */
int chunk_attention_fwd(kvcr_cache *c, const void *q, int n_q, const void *k_cur,
                        const void *v_cur, const int32_t *cur_frame_idx, int n_cur_frames,
                        float softmax_scale, void *o, float *lse, void *stream);

/* chunk_attention_fwd() for callers that cannot allocate device memory at the
 * time of the call: hosts whose memory pool owns every device allocation and
 * hands the library exactly the cache buffer, and real-time loops that cannot
 * take the implicit device synchronisation of cudaMalloc/cudaFree.  (The
 * papers have no counterpart of this call; it is a property of this library.)
 * Arguments, result and errors are those of
 * chunk_attention_fwd().  The difference: the rotated queries and current-chunk
 * keys are staged in a fixed 36 MiB array that the library holds in device
 * memory on every GPU where it is loaded (until the process exits), not in the
 * cache's scratch region.  A chunk whose staging needs more than that
 * (2 x n_cur_frames * tokens_per_frame * heads * head_dim * sizeof(dtype), each
 * half rounded up to 256 bytes) is rejected with KVCR_ESHAPE before anything is
 * launched; a bf16 chunk of 4 frames x 1508 tokens x 12 heads x 128 fits.  The
 * call allocates nothing.  The first call on a device looks up the array's
 * address once for that device; make that first call before any stream capture.
 * All calls on a device share the array, which keeps the last call's contents
 * (nothing in it needs to start at zero); calls whose GPU work overlaps -- on
 * different streams or from different host threads -- race on it. */
int chunk_attention_fwd_static_scratch(kvcr_cache *c, const void *q, int n_q,
                                       const void *k_cur, const void *v_cur,
                                       const int32_t *cur_frame_idx, int n_cur_frames,
                                       float softmax_scale, void *o, float *lse, void *stream);

/* The last denoising step of a chunk: chunk_attention_fwd() followed by
 * kv_cache_append_rope(k_cur, v_cur, cur_frame_idx), with one pass over the
 * chunk's K and V.  The finalized states enter the retained slots ("Westlake AGI
 * Lab's 'World in World' Steers Frozen Video Models", second paragraph) and the
 * step that finalizes reads the frames they evict: here the chunk's rotated K
 * and its V are written once, into spare frame slots, read from there by this
 * call's attention as the current keys, and then become cached frames by
 * relabelling (the slots of the frames they evict become the spare ones), so
 * the separate append pass over K and V disappears.  Slot maps, eviction and
 * the result of kv_cache_slot_data() are exactly those of the two-call
 * sequence; outputs equal chunk_attention_fwd()'s up to the order of fp32
 * accumulation (the chunk's keys are read frame by frame).  Needs a cache made
 * with KVCR_CACHE_FUSED_FINALIZE (else KVCR_ESTATE).  Arguments and errors are
 * those of chunk_attention_fwd() and kv_cache_append_rope(); on error nothing
 * changes. */
int chunk_attention_fwd_finalize(kvcr_cache *c, const void *q, int n_q, const void *k_cur,
                                 const void *v_cur, const int32_t *cur_frame_idx,
                                 int n_cur_frames, float softmax_scale, void *o, float *lse,
                                 void *stream);

/* chunk_attention_fwd() with the QK^T product in 8 bits: the pages' own speed
 * lever on this path is an 8-bit QK^T (kaarelkaarelson.com/lingbot, kernel table,
 * "SageAttention" row: INT8 QK^T at 65 % of the RTX 5090's INT8 peak); here it is
 * the tensor cores' e4m3 (tcgen05.mma kind::f8f6f4), with P V in bf16.  The
 * rotated queries and current keys (bf16, as chunk_attention_fwd() stages them)
 * and every cached or auxiliary K are block-quantized: per block of 128 tokens
 * and head, amax = max |x|, scale = amax / 448, code = e4m3(x * (448 / amax))
 * rounded to nearest even and saturated (fp32 arithmetic); blocks are 128 tokens
 * of one cached / auxiliary frame, and 128 tokens of the chunk for its own Q and
 * K.  The scores are (Q codes . K codes) * q scale * k scale * softmax_scale;
 * everything after them is as in chunk_attention_fwd() (fp32 softmax, bf16 P,
 * fp32 accumulation of P V).  Arguments, outputs and errors are those of
 * chunk_attention_fwd(); additionally KVCR_ESTATE when the cache was made without
 * KVCR_CACHE_FP8_K, and KVCR_ESHAPE when a cache without RoPE gets n_q >
 * chunk_frames * tokens_per_frame (the size of the query staging). */
int chunk_attention_fwd_fp8(kvcr_cache *c, const void *q, int n_q, const void *k_cur,
                            const void *v_cur, const int32_t *cur_frame_idx, int n_cur_frames,
                            float softmax_scale, void *o, float *lse, void *stream);

/* Attention under the MoBA mask over one sequence of L = layout tokens ("Infinite
 * Worlds with Versatile Interactions", causal-pretraining paragraph: the
 * teacher-forcing mask plus an appended fully bidirectional block; "Mix Forcing",
 * "Mix the training modes").
 * q, k, v, o: device [L][heads][head_dim] bf16 (head_dim 128 or 64); lse nullable
 * fp32 [heads][L].  128 x 128 tiles of the score matrix with no allowed entry
 * are skipped, fully allowed tiles run unmasked, the rest are masked. */
int moba_attention_fwd(const void *q, const void *k, const void *v,
                       const kvcr_moba_layout *layout, int heads, int head_dim,
                       kvcr_dtype dtype, float softmax_scale, void *o, float *lse,
                       void *stream);

/* Backward of moba_attention_fwd(): with P the forward's probabilities
 * (recomputed from its LSE), dV = P^T dO, dP = dO V^T, D = rowsum(dO o O),
 * dS = P o (dP - D), dQ = scale * dS K, dK = scale * dS^T Q, for the model
 * trained under the MoBA mask ("Infinite Worlds with Versatile Interactions",
 * causal-pretraining paragraph; "Mix Forcing", "Mix the training modes"; the
 * pages print no backward pass, this is the chain rule through the forward).
 *   q, k, v, o, d_o: device [L][heads][head_dim] bf16, 16-byte aligned; o and
 *          lse are the forward's outputs for the same q, k, v, layout, scale.
 *   lse:   device fp32 [heads][L] (natural log, as moba_attention_fwd writes).
 *   dq, dk, dv: device [L][heads][head_dim] bf16, written in full (no
 *          accumulation into previous contents).
 *   workspace: caller-owned device buffer of at least
 *          moba_attention_bwd_workspace_bytes() bytes, 16-byte aligned, used
 *          as scratch for the duration of the call's GPU work (no initial
 *          contents needed); calls whose GPU work overlaps need separate ones.
 * Three kernels run on `stream`, no atomics: the result does not depend on
 * scheduling.  Errors: KVCR_EINVAL (NULL / misaligned pointer), KVCR_ESHAPE,
 * KVCR_ESTORAGE (workspace too small), KVCR_EUNSUPPORTED (dtype other than
 * bf16, head_dim other than 64 / 128, GPU other than sm_100); nothing is
 * launched on error. */
int moba_attention_bwd(const void *q, const void *k, const void *v, const void *o,
                       const void *d_o, const float *lse, const kvcr_moba_layout *layout,
                       int heads, int head_dim, kvcr_dtype dtype, float softmax_scale,
                       void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                       void *stream);

/* Bytes of workspace moba_attention_bwd() needs: 8 per (head, row) with the
 * rows rounded up to a multiple of 128; 0 for an invalid layout or heads < 1. */
size_t moba_attention_bwd_workspace_bytes(const kvcr_moba_layout *layout, int heads);

/* Host classification of the tile x tile blocks of the MoBA score matrix into
 * KVCR_TILE_EMPTY / PARTIAL / FULL (only in-range rows and columns count).  The
 * pages give the mask, not a tiling: this is the block-sparse schedule of this
 * library's MoBA kernels (empty tiles skipped, full ones unmasked), exported so
 * it can be checked against a brute-force reduction of the mask.
 * cls: host [nt * nt] row-major, nt = ceil(L / tile); cap = its length. */
int moba_classify_tiles(const kvcr_moba_layout *layout, int tile, uint8_t *cls, size_t cap);

/* ------------------------------------------------------------- status ---- */

/* Synchronise `stream` and return (then clear) the device-side status of the
 * library's kernels on the current device: KVCR_OK or KVCR_ETIMEOUT when a
 * kernel gave up on a bounded wait (its outputs are then invalid; the forward
 * attention kernels write NaN into the rows and LSE of a query tile that gave
 * up, so a missed check still shows in the output).  Library
 * convention (failure detection); no page has a counterpart. */
int kvcr_check_status(void *stream);

/* Message of the last non-OK return on this thread (library convention). */
const char *kvcr_last_error(void);

/* Failure-path test hook (for tests; off by default).  kind = 1 makes every
 * later tensor-core attention launch (forward and backward) withhold one
 * internal "P ready" (or "dS ready") signal, so a wait inside the kernel runs
 * out: the kernel then records KVCR_ETIMEOUT (read
 * with kvcr_check_status), drains its in-flight copies and MMAs, frees its
 * tensor memory and returns with its outputs invalid; the CUDA context stays
 * usable.  kind = 0 turns it off.  wait_ns > 0 replaces the 2 s bound of every
 * device wait of those launches (0 restores it). */
int kvcr_debug_inject(int kind, long long wait_ns);

/* -------------------------------------------------------------- trace ---- */

/* Kernel ids for tracing. */
enum {
    KVCR_K_APPEND_ROPE = 0, /* cache write: RoPE3D(K) + copy V into slots */
    KVCR_K_ROPE_STAGE = 1,  /* RoPE3D of the current chunk's Q and K into scratch */
    KVCR_K_CHUNK_ATTN = 2,  /* tensor-core chunk attention (bf16) */
    KVCR_K_MOBA_ATTN = 3,   /* tensor-core MoBA attention (bf16) */
    KVCR_K_ATTN_F32 = 4,    /* fp32 CUDA-core attention */
    KVCR_K_MOBA_BWD_PREP = 5, /* MoBA backward: per-row LSE and rowsum(dO o O) */
    KVCR_K_MOBA_BWD_DKDV = 6, /* MoBA backward: dK and dV (tensor cores) */
    KVCR_K_MOBA_BWD_DQ = 7,   /* MoBA backward: dQ (tensor cores) */
    KVCR_K_SET_AUX = 8,       /* auxiliary frames written into their slots (RoPE3D of K) */
    KVCR_K_APPEND_BATCH = 9,  /* one cache write for several caches (RoPE3D of K) */
    KVCR_K_QUANT_E4M3 = 10,   /* e4m3 block quantization of K (cache) or Q / current K */
    KVCR_K_CHUNK_ATTN_FP8 = 11, /* tensor-core chunk attention, e4m3 QK^T, bf16 P V */
    KVCR_K_COUNT = 12
};

/* Count of every kernel the library launched in this process (library
 * convention, for launch accounting). */
long long kvcr_launch_count(void);

/* Tracing: when on, each launch is bracketed by two CUDA events recorded on
 * its own stream.  kvcr_trace_reset() clears the records;
 * kvcr_trace_read() waits for the recorded events and returns, for one kernel
 * id, the number of traced launches and their summed device time in ms. */
int kvcr_trace_enable(int on);
int kvcr_trace_reset(void);
int kvcr_trace_read(int kernel_id, long long *launches, double *total_ms);

#ifdef __cplusplus
}
#endif

#endif /* KVCR_H */
