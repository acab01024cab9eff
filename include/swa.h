/*
 * swa.h -- C ABI of the B200 (sm_100a) frame-causal sliding-window attention library.
 *
 * One shared library, libswa_b200.so, exports every function below with C linkage.
 * Signatures carry only plain pointers, integers and sizes.  Tensor pointers are
 * DEVICE pointers owned by the caller unless a comment says otherwise; the library
 * never frees or retains them beyond the call.  ``stream`` is a cudaStream_t passed
 * as void* (NULL = the legacy default stream); every call is asynchronous on it
 * unless documented as synchronous.  Calls validate their arguments on the host and
 * return a negative swa_status before launching anything when they are invalid.
 *
 * Method sources (page title, section):
 *   [AGG] "Sliding Window Attention Mechanism in AggregatorStream: Implementation and
 *         Configuration Guide": "Mask Generation in CausalAttention" (window start
 *         max(0, i - sliding_window_size*num_frame_per_block + 1), ANDed with the
 *         causal mask), "KV Cache Eviction Strategy" (evict before attention; the
 *         first scale frames stay; special tokens can persist), FAQ on
 *         sliding_window_size = -1 (full causal).
 *   [IO]  "Stream.py Aggregator Input and Output Formats": tokens [B*S, P, C],
 *         scalar parameters B, S, P, C, global_idx, num_frame_for_scale,
 *         sliding_window_size.
 *   [BLK] "Method forward" (lingbot_map/layers/block.py FlashInferBlock.forward):
 *         the streaming step append_frame -> evict_frames -> compute_attention on
 *         per-frame q/k/v of shape [tpf, H, D]; global_idx selects the block's cache.
 *   [SWA] sliding-window attention explainer (Mistral 7B): token band i-W+1..i,
 *         rolling KV buffer written at slot i mod W, grouped-query attention.
 *
 * Numerics: bf16 inputs and outputs with float32 accumulation and softmax on the
 * tensor-core path (head_dim 64 or 128); float32 end to end on the SIMT path
 * (head_dim 32, 64 or 128).  The softmax scale is 1/sqrt(head_dim).
 */
#ifndef SWA_B200_H
#define SWA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
typedef enum {
    SWA_OK = 0,
    SWA_ERR_ARG = -1,         /* null pointer, bad enum, negative size            */
    SWA_ERR_SHAPE = -2,       /* inconsistent sizes, e.g. C != heads*head_dim      */
    SWA_ERR_ORDER = -3,       /* streaming frame out of order / attend before append */
    SWA_ERR_CAPACITY = -4,    /* buffer too small, cache full, layer out of range  */
    SWA_ERR_CUDA = -5,        /* a CUDA runtime call failed                        */
    SWA_ERR_TIMEOUT = -6,     /* a bounded device-side wait ran out (latched flag) */
    SWA_ERR_UNSUPPORTED = -7  /* dtype / head_dim combination not built            */
} swa_status;

typedef enum { SWA_F32 = 0, SWA_BF16 = 1 } swa_dtype;

/* Human-readable name of a status code.  Never NULL. */
const char* swa_status_str(int status);

/* Library ABI version (major*100 + minor). */
int swa_version(void);

/* ------------------------------------------------------------ tile scheduler
 * Host-side views of the block-sparse schedule the kernels use (the device code
 * runs the same functions).  Intended for tests and tooling; no GPU needed.
 *
 * swa_sched_frame_intervals: key-frame intervals visible to query frame ``i``
 * ([AGG] "Mask Generation"): [0, min(S, i+1)) for the retained scale frames and
 * [max(S, i - W_f + 1), i + 1) for the window, W_f = sliding_window_size *
 * num_frame_per_block (sliding_window_size <= 0: no window).  Touching intervals
 * are merged.  Writes at most two [lo, hi) pairs into lo[]/hi[] and returns how
 * many (1 or 2), or a negative status.
 */
int swa_sched_frame_intervals(int i, int sliding_window_size, int num_frame_per_block,
                              int num_frame_for_scale, int* lo, int* hi);

/* swa_sched_prefill: the prefill work list in launch (longest-first) order.
 * One item = one batch row b, head h, query frame f and a pair of 128-row query
 * tiles of that frame.  Each item is 8 int32: {b, h, f, q_row0, rows_a, rows_b,
 * n_key_tiles, n_key_tokens}, q_row0 being the first query token of tile a
 * within the frame's sequence (tile b starts 128 rows later; rows_b = 0 when the
 * pair has a single tile).  Key tiles are 128-token runs of the frame's
 * intervals; fully masked tiles never appear.  ``out`` may be NULL to query the
 * count.  Returns the number of items (<= cap written) or a negative status. */
int64_t swa_sched_prefill(int B, int S, int P, int heads, int sliding_window_size,
                          int num_frame_per_block, int num_frame_for_scale,
                          int32_t* out, int64_t cap);

/* swa_sched_decode: the launch swa_decode makes for batch B, Hkv KV heads, a
 * W-slot rolling cache and position ``pos`` on a GPU of ``sms`` SMs
 * (sliding-window explainer, rolling buffer: the valid slots are min(pos+1, W)).
 * Each (batch, KV head) cuts its valid slots into ``pieces`` pieces of
 * ``piece_len`` slots (whole 128-key tiles; the last piece may be shorter or
 * empty), at most ``slots`` = the partial slots the decode workspace holds; the
 * units (batch, KV head, piece) go round-robin to ``grid`` persistent CTAs.
 * out[5] = {pieces, piece_len, grid, slots, n_valid}.  Returns SWA_OK or
 * SWA_ERR_ARG. */
int swa_sched_decode(int B, int Hkv, int W, long long pos, int sms, int32_t* out);

/* swa_sched_stream: the launch swa_stream_attend makes for ``key_tiles`` 128-token
 * key tiles (the key runs of the retained frames and specials, each cut into whole
 * tiles), ``heads`` heads, frames of ``P`` tokens, cfg.max_splits = ``max_splits``
 * and ``sms`` SMs.  The (query-tile pair, head) items are each cut into ``splits``
 * contiguous key-tile ranges, one CTA each; a combine kernel merges the splits when
 * there is more than one.  out[4] = {splits, CTAs, fewest and most key tiles of a
 * split}.  Returns SWA_OK or SWA_ERR_ARG. */
int swa_sched_stream(int key_tiles, int heads, int P, int max_splits, int sms, int32_t* out);

/* ---------------------------------------------------------------- prefill
 * Frame-causal sliding-window attention over a whole clip ([AGG], [IO]).
 *   q, k, v, out: [B, S*P, heads, head_dim] contiguous, i.e. the pages'
 *                 [B*S, P, C] token layout with C = heads*head_dim.
 *   S: number of frames, P: tokens per frame (special + patch tokens).
 *   sliding_window_size <= 0 -> full (frame-)causal attention.
 *   num_frame_for_scale: the first frames every later frame also sees.
 * Query frame i attends to every token of key frame j iff j <= i and
 * (j < num_frame_for_scale or j >= i - sliding_window_size*num_frame_per_block + 1).
 * dtype SWA_BF16 needs head_dim 64 or 128 (tcgen05 path); SWA_F32 accepts
 * 32, 64 or 128 (SIMT path).  Errors: SWA_ERR_ARG, SWA_ERR_SHAPE,
 * SWA_ERR_UNSUPPORTED, SWA_ERR_CUDA. */
swa_status swa_prefill(const void* q, const void* k, const void* v, void* out,
                       int B, int S, int P, int C, int heads, int head_dim,
                       int sliding_window_size, int num_frame_per_block,
                       int num_frame_for_scale, int dtype, void* stream);

/* Head-sliced prefill: the same attention on heads [head0, head0 + heads) of
 * token rows ``row_stride`` elements apart, read and written in place.  q, k, v
 * and out all point at the start of the full tensors [B, S*P, row_stride]; only
 * the slice's elements are read or written.  This is how one GPU of several
 * takes its share of the heads (each head is independent; no exchange inside the
 * attention): rank r attends its heads of the same [B, S*P, C] tensors and an
 * all-gather of the slices rebuilds the output.  Needs row_stride >= (head0 +
 * heads) * head_dim (else SWA_ERR_SHAPE) and row_stride * element size a
 * multiple of 16 bytes (else SWA_ERR_ARG); otherwise as swa_prefill. */
swa_status swa_prefill_heads(const void* q, const void* k, const void* v, void* out,
                             int B, int S, int P, int row_stride, int head0, int heads, int head_dim,
                             int sliding_window_size, int num_frame_per_block,
                             int num_frame_for_scale, int dtype, void* stream);

/* --------------------------------------------------------- streaming cache
 * Per-layer rolling paged KV cache for frame-by-frame streaming ([AGG] "KV Cache
 * Eviction Strategy"; [BLK]).  ``global_idx`` selects the layer's cache.
 *
 * Storage (inside the caller's device buffer): pages of ``page_tokens`` tokens.
 * Slot s holds one frame in pages s*ppf .. s*ppf+ppf-1, ppf = ceil(P/page_tokens).
 * Frame i < scale_frames lives in slot i; a window frame i lives in slot
 * scale_frames + (i mod window_frames) ([SWA] slot i mod W), so the frame that
 * arrives overwrites exactly the frame it evicts.  With cross_frame_special the
 * evicted frame first leaves its first num_special tokens in a packed special
 * region starting at page n_slots*ppf.  Per layer the device keeps the slot map,
 * the page table (retained frames ascending, then special pages), the eviction of
 * the last append and the key segments the attention kernel reads; the host keeps
 * only a frame counter to reject out-of-order calls.
 */
typedef struct swa_stream_cfg {
    int num_layers;          /* caches, indexed by global_idx in [0, num_layers)       */
    int heads;               /* H                                                       */
    int head_dim;            /* D                                                       */
    int P;                   /* tokens per frame                                        */
    int scale_frames;        /* kv_cache_scale_frames: first frames never evicted       */
    int window_frames;       /* kv_cache_sliding_window in frames; <= 0 keeps all frames */
    int page_tokens;         /* tokens per page (16)                                    */
    int cross_frame_special; /* kv_cache_cross_frame_special: keep specials of evicted  */
    int num_special;         /* camera + register tokens at the head of every frame     */
    int max_frames;          /* frames per layer the buffer is sized for               */
    int dtype;               /* swa_dtype of K/V/Q/out                                  */
    int max_splits;          /* split-KV partial buffers for the attend (1..32)         */
} swa_stream_cfg;

typedef struct swa_stream swa_stream;  /* opaque host handle */

/* Device bytes swa_stream_init needs for ``cfg`` (0 if cfg is invalid): every
 * layer's metadata and K/V pages plus the split-KV partials of the attend. */
size_t swa_stream_cache_bytes(const swa_stream_cfg* cfg);

/* Create a handle over ``dev_buf`` (caller-owned device memory of at least
 * swa_stream_cache_bytes(cfg) bytes, 256-byte aligned).  Clears the buffer on
 * ``stream`` and waits for it.  The handle is host memory owned by the library
 * until swa_stream_destroy; the library allocates no device memory.  Errors:
 * SWA_ERR_ARG (invalid cfg, null or misaligned buffer), SWA_ERR_CAPACITY (bytes
 * too small), SWA_ERR_UNSUPPORTED (dtype / head_dim not built). */
swa_status swa_stream_init(swa_stream** out, const swa_stream_cfg* cfg, void* dev_buf,
                           size_t bytes, void* stream);
void swa_stream_destroy(swa_stream* h);

/* Earlier names of swa_stream_cache_bytes and swa_stream_init, kept as aliases
 * (same arguments, same behaviour). */
size_t swa_stream_bytes(const swa_stream_cfg* cfg);
swa_status swa_stream_create(swa_stream** out, const swa_stream_cfg* cfg, void* dev_buf,
                             size_t bytes, void* stream);

/* Empty every layer's cache (the pages' clean_kv_cache). */
swa_status swa_stream_reset(swa_stream* h, void* stream);

/* Append frame ``frame_idx`` (must equal the number of frames this layer has seen)
 * and apply the eviction rule on the device: once more than
 * scale_frames + window_frames full frames are cached, the oldest non-scale frame
 * (frame_idx - window_frames) leaves -- keeping its specials if configured -- and
 * the new frame takes its slot.  k_frame, v_frame: [P, heads, head_dim].
 * Errors: SWA_ERR_ORDER (wrong frame index), SWA_ERR_CAPACITY (beyond max_frames
 * or global_idx out of range). */
swa_status swa_stream_append_evict(swa_stream* h, int global_idx, int frame_idx,
                                   const void* k_frame, const void* v_frame, void* stream);

/* The frame's queries q_frame [P, heads, head_dim] attend to everything the layer's
 * cache holds after the append (retained full frames, the current frame and
 * retained specials); out [P, heads, head_dim].  ``frame_idx`` must be the frame
 * appended last (SWA_ERR_ORDER otherwise).  The keys are split across CTAs (at
 * most cfg.max_splits per query tile); each writes its partial (O, max, sum) into
 * the handle's buffer and a combine kernel, launched behind the attend on the same
 * stream, merges them into ``out`` (two launches; one when a frame needs a single
 * split): calls on one handle must not overlap on the GPU. */
swa_status swa_stream_attend(swa_stream* h, int global_idx, int frame_idx,
                             const void* q_frame, void* out, void* stream);

/* Head-sliced forms of the append and the attend: the cache holds cfg.heads
 * heads, taken from heads [head0, head0 + cfg.heads) of frame tensors whose token
 * rows are ``row_stride`` elements apart (k_frame, v_frame, q_frame and out point
 * at the full [P, row_stride] frames; the attend writes only its heads of out).
 * One GPU of several keeps the cache of its share of the heads this way; the
 * result equals the unsliced call on those heads.  Needs row_stride >= (head0 +
 * cfg.heads) * head_dim (else SWA_ERR_SHAPE) and row_stride * element size a
 * multiple of 16 bytes (else SWA_ERR_ARG); otherwise as the unsliced calls. */
swa_status swa_stream_append_evict_heads(swa_stream* h, int global_idx, int frame_idx, const void* k_frame,
                                         const void* v_frame, int row_stride, int head0, void* stream);
swa_status swa_stream_attend_heads(swa_stream* h, int global_idx, int frame_idx, const void* q_frame,
                                   void* out, int row_stride, int head0, void* stream);

/* Non-keyframe attend ("Non-keyframe path" of the streaming attention block,
 * lingbot-map AggregatorStream guide: append with eviction deferred, attend,
 * roll the append back).  The queries q_frame [P, heads, head_dim] attend to
 * everything the layer's cache holds after its last keyframe (retained full
 * frames and specials, nothing evicted on this frame's account) plus this
 * frame's own k_frame, v_frame [P, heads, head_dim]; out [P, heads, head_dim].
 * Nothing persistent changes: the frame's K/V go to a scratch frame of pages
 * that no page table lists, the frame counter does not advance, no frame or
 * special token moves.  Valid on an empty layer (the frame attends to itself).
 * Shares the split-KV partials and the scratch frame with the handle's other
 * calls: calls on one handle must not overlap on the GPU.  Errors: SWA_ERR_ARG
 * (null or misaligned pointer), SWA_ERR_CAPACITY (global_idx out of range). */
swa_status swa_stream_attend_transient(swa_stream* h, int global_idx, const void* q_frame,
                                       const void* k_frame, const void* v_frame, void* out,
                                       void* stream);

/* Attention prologue of one frame ("Method forward", block forward listing: the
 * compiled attn_pre step "norm1 + qkv linear + reshape + q_norm + k_norm + RoPE +
 * format"; RoPE in the I/O page's complex-valued format).  Readings for the steps
 * the listing names without defining: norm1 = LayerNorm over C with weight ln_w
 * and bias ln_b, qkv = norm1(x) w_qkv^T + b_qkv, q_norm / k_norm = LayerNorm over
 * head_dim of each head with weights qn_w / kn_w and biases qn_b / kn_b, all with
 * epsilon eps (biased variance); RoPE multiplies the (2i, 2i+1) element pairs of
 * every q and k head by the complex number rot[p][i] = (cos, sin) of its token p.
 *   x      [P, C] bf16 (C = heads * head_dim, C a multiple of 256, C <= 2048,
 *          head_dim 64 or 128)          w_qkv [3C, C] bf16 (rows q | k | v)
 *   ln_w, ln_b [C], b_qkv [3C], qn_w, qn_b, kn_w, kn_b [head_dim], rot [P, head_dim/2, 2]: f32
 *   xn_ws  [P, C] bf16 workspace (norm1 output)
 *   q_out, k_out, v_out [P, heads, head_dim] bf16.
 * All device pointers, 16-byte aligned, caller-owned.  Errors: SWA_ERR_ARG (null or
 * misaligned pointer, negative size, eps <= 0), SWA_ERR_UNSUPPORTED (shape). */
swa_status swa_attn_pre(const void* x, const float* ln_w, const float* ln_b, const void* w_qkv,
                        const float* b_qkv, const float* qn_w, const float* qn_b, const float* kn_w,
                        const float* kn_b, const float* rot, int P, int C, int heads, float eps,
                        void* xn_ws, void* q_out, void* k_out, void* v_out, void* stream);

/* Streaming append with the prologue fused in: the eviction and metadata of
 * swa_stream_append_evict for frame ``frame_idx``, then swa_attn_pre on the frame's
 * tokens x [P, C] with K and V written straight into the frame's slot of the
 * layer's page storage (no separate K/V frame), Q to q_out [P, heads, head_dim] for
 * swa_stream_attend.  bf16 caches only; C = heads * head_dim of the cache.  Errors
 * as swa_stream_append_evict and swa_attn_pre. */
swa_status swa_stream_append_evict_pre(swa_stream* h, int global_idx, int frame_idx, const void* x,
                                       const float* ln_w, const float* ln_b, const void* w_qkv,
                                       const float* b_qkv, const float* qn_w, const float* qn_b,
                                       const float* kn_w, const float* kn_b, const float* rot, float eps,
                                       void* xn_ws, void* q_out, void* stream);

/* 3-D RoPE table of one streaming frame, the rotation input of swa_attn_pre (the
 * I/O page's 3-D RoPE: complex-valued positions [.., S_global*P, head_dim/2]
 * from WanRotaryPosEmbed, generated internally when enable_3d_rope is set).
 * Readings: token k of frame ``frame_idx`` sits at (t, h, w) = (frame_idx,
 * (k - num_special) / grid_w, (k - num_special) % grid_w) for patch tokens and
 * (frame_idx, 0, 0) for the num_special special tokens; the head_dim/2 pairs
 * split into bands t | h | w of (head_dim/2 - 2*(head_dim/6), head_dim/6,
 * head_dim/6) pairs; pair j of a band of n pairs turns by pos * theta^(-j/n).
 * rot_out [P, head_dim/2, 2] f32 (cos, sin), device, 16-byte aligned.  Errors:
 * SWA_ERR_ARG (negative index or size, num_special > P, grid_w < 1, odd or
 * small head_dim, theta <= 1, null or misaligned output). */
swa_status swa_rope3d_table(int frame_idx, int P, int num_special, int grid_w, int head_dim, double theta,
                            float* rot_out, void* stream);

/* swa_attn_pre with the 3-D RoPE generated inside the prologue instead of read
 * from a table (the I/O page's enable_3d_rope: positions built internally).  The
 * positions and bands are those of swa_rope3d_table for (frame_idx, num_special,
 * grid_w, theta); the epilogue forms each pair's angle pos * theta^(-j/n), reduces
 * it to [-pi, pi] in double and takes its sine and cosine in float, so no table
 * goes through device memory.  Other arguments, layouts and errors as
 * swa_attn_pre, plus SWA_ERR_ARG for a negative frame_idx, num_special outside
 * [0, P], grid_w < 1 or theta <= 1. */
swa_status swa_attn_pre_rope3d(const void* x, const float* ln_w, const float* ln_b, const void* w_qkv,
                               const float* b_qkv, const float* qn_w, const float* qn_b, const float* kn_w,
                               const float* kn_b, int frame_idx, int num_special, int grid_w, double theta,
                               int P, int C, int heads, float eps, void* xn_ws, void* q_out, void* k_out,
                               void* v_out, void* stream);

/* swa_stream_append_evict_pre with the 3-D RoPE of frame ``frame_idx`` generated
 * inside the prologue (as swa_attn_pre_rope3d; num_special here is the RoPE's
 * count of special tokens at (t, 0, 0), independent of the cache's retention). */
swa_status swa_stream_append_evict_pre_rope3d(swa_stream* h, int global_idx, int frame_idx, const void* x,
                                              const float* ln_w, const float* ln_b, const void* w_qkv,
                                              const float* b_qkv, const float* qn_w, const float* qn_b,
                                              const float* kn_w, const float* kn_b, int num_special, int grid_w,
                                              double theta, float eps, void* xn_ws, void* q_out, void* stream);

/* Layout of one layer's metadata block, in int32 units. */
typedef struct swa_meta_layout {
    int n_ints;          /* size of the block                                  */
    int n_slots;         /* slots (scale + window, or max_frames if no window) */
    int pages_per_frame; /* ppf                                                */
    int max_pages;       /* capacity of the page table                         */
    int max_segs;        /* capacity of the segment list                       */
    int off_slot_frame;  /* int32[n_slots]: frame held by each slot, -1 empty  */
    int off_page_table;  /* int32[max_pages]: physical page ids, logical order */
    int off_seg_row;     /* int32[max_segs]: first storage row of each segment */
    int off_seg_len;     /* int32[max_segs]: tokens in each segment            */
    /* header ints at offsets 0..7: n_frames, n_evicted, n_special_tokens,
       last_evicted (-1 none), n_pages, n_segs, n_slots_used, reserved */
} swa_meta_layout;

swa_status swa_stream_meta_layout(const swa_stream* h, swa_meta_layout* out);

/* Host view of one layer's cache bookkeeping ([AGG] "KV Cache Eviction
 * Strategy": which frames the cache holds, where, and what the last append
 * evicted).  The counts are always filled; each array is the caller's host
 * memory, filled when non-NULL, and must hold its count (else
 * SWA_ERR_CAPACITY). */
typedef struct swa_meta_host {
    int n_frames;          /* frames appended to the layer so far                    */
    int n_evicted;         /* full frames evicted so far                             */
    int n_special_tokens;  /* special tokens retained from evicted frames            */
    int n_pages;           /* entries of the page table                              */
    int n_segs;            /* key segments (contiguous storage runs) the attend reads */
    int n_retained;        /* full frames the cache holds                            */
    int n_slots;           /* slots of the layer (entries of slot_frame)             */
    int n_last_evicted;    /* size of the last append's eviction set: 0 or 1         */
    int last_evicted;      /* the frame it evicted, -1 if none                       */
    int32_t* slot_frame;   /* [n_slots]: frame held by each slot, -1 empty           */
    int slot_cap;
    int32_t* page_table;   /* [n_pages]: physical page ids in logical key order      */
    int page_cap;
    int32_t* seg_row;      /* [n_segs]: first storage row of each key segment        */
    int32_t* seg_len;      /* [n_segs]: tokens in each key segment                   */
    int seg_cap;
} swa_meta_host;

/* Fill ``m`` with layer ``global_idx``'s bookkeeping: a synchronous copy from the
 * device (waits for ``stream``), for tests and inspection.  Errors: SWA_ERR_ARG
 * (null), SWA_ERR_CAPACITY (layer out of range, or an array too small),
 * SWA_ERR_CUDA. */
swa_status swa_stream_get_meta(const swa_stream* h, int global_idx, swa_meta_host* m, void* stream);

/* The same bookkeeping as the raw int32 block of swa_stream_meta_layout (header
 * ints 0..7, then slot map, page table, segment rows and lengths) copied into
 * host ``dst`` (n_ints >= layout.n_ints); synchronous. */
swa_status swa_stream_get_meta_raw(const swa_stream* h, int global_idx, int32_t* dst,
                                   size_t n_ints, void* stream);

/* Device pointers of layer ``global_idx``'s K and V page storage
 * ([n_pages_total * page_tokens, heads, head_dim]); NULL on error. */
void* swa_stream_k_storage(const swa_stream* h, int global_idx);
void* swa_stream_v_storage(const swa_stream* h, int global_idx);

/* ------------------------------------------------- token-band GQA prefill
 * Mistral-style sliding-window attention ([SWA]): token t attends to s iff
 * t - window + 1 <= s <= t; query head h reads KV head h / (Hq / Hkv).
 *   q, out: [B, N, Hq, head_dim]; k, v: [B, N, Hkv, head_dim].
 * bf16: head_dim 64 or 128; f32: 32, 64 or 128. */
swa_status swa_band_prefill(const void* q, const void* k, const void* v, void* out,
                            int B, int N, int Hq, int Hkv, int head_dim, int window,
                            int dtype, void* stream);

/* ------------------------------------------------------ rolling GQA decode
 * One new token per sequence at position ``pos`` ([SWA]): its K/V is written into
 * the rolling cache at slot pos mod W, then q attends over the valid slots (all W
 * once pos >= W-1, else slots 0..pos).
 *   q, out: [B, Hq, head_dim]; k_new, v_new: [B, Hkv, head_dim];
 *   k_cache, v_cache: [B, W, Hkv, head_dim] (updated in place).
 *   workspace: device scratch of at least swa_decode_workspace_bytes(...) bytes
 *   (split-K partials); calls sharing a workspace must not overlap on the GPU.
 * bf16: head_dim 64 or 128 with Hq/Hkv from 1 to 8 (larger groups return
 * SWA_ERR_UNSUPPORTED); f32: head_dim 32, 64 or 128, any Hq/Hkv.  The kernels read
 * only the valid slots' values: slots beyond ``pos`` may hold anything, NaN
 * included. */
size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int head_dim, int W);
swa_status swa_decode(const void* q, const void* k_new, const void* v_new,
                      void* k_cache, void* v_cache, long long pos, int W,
                      int B, int Hq, int Hkv, int head_dim, void* out,
                      void* workspace, size_t workspace_bytes, int dtype, void* stream);

/* ------------------------------------------- decode without any allocation
 * The pages have no counterpart to this entry point; it exists for callers of
 * this library that cannot allocate device memory when they decode: a process
 * whose device memory is fully reserved by another allocator, a host program that
 * forbids allocation calls while it runs (cudaMalloc can synchronize the device and
 * take unbounded time), or a plugin interface that passes inputs and outputs but
 * offers no way to obtain memory.
 *
 * swa_decode_noalloc does what swa_decode does for bf16 (head_dim 64 or 128,
 * Hq/Hkv from 1 to 8) with the same arguments minus the workspace: its split-K
 * scratch is a fixed SWA_DECODE_NOALLOC_SCRATCH_BYTES array inside the library,
 * held on every GPU that loads the library until the process exits.  It calls no
 * allocating routine.  Requests whose scratch would exceed the array return
 * SWA_ERR_CAPACITY (the need is swa_decode_workspace_bytes(B, Hq, Hkv, head_dim, W));
 * f32 or other shapes return SWA_ERR_UNSUPPORTED.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.  All calls share the
 * one array, so calls that overlap on the GPU race and must be serialized by the
 * caller; no state from a previous call is needed or left to clear. */
#define SWA_DECODE_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
swa_status swa_decode_noalloc(const void* q, const void* k_new, const void* v_new,
                              void* k_cache, void* v_cache, long long pos, int W,
                              int B, int Hq, int Hkv, int head_dim, void* out,
                              int dtype, void* stream);

/* Diagnostic: y[i] = 2^x[i] as the attention kernels' FMA-pipe polynomial computes it
 * (Cody-Waite reduction + fitted cubic, relative error <= 8e-5 for x >= -125), for
 * n float32 device values.  Lets tests compare it with the hardware exp2. */
swa_status swa_debug_exp2_poly(const float* x, float* y, int n, void* stream);

/* Kernel launches this library has issued in this process (all devices). */
uint64_t swa_launch_count(void);

/* ------------------------------------------------------- device errors
 * Kernels bound every wait; a wait that runs out latches a per-device flag and
 * the kernel returns early.  The flag is mirrored into pinned, mapped host memory
 * (a static page of the library, registered on first use), so once a kernel has
 * latched an error every later call that would launch work on that device
 * returns SWA_ERR_TIMEOUT at once, without synchronizing and without launching,
 * until the error is cleared.  swa_device_error_check synchronizes ``stream``,
 * reads and clears the flag and returns SWA_ERR_TIMEOUT if it was set (SWA_OK
 * otherwise).  The first call on a device sets the flag up (a symbol lookup and
 * a small synchronous copy): make it before any stream capture.
 * swa_debug_wait_timeout launches one thread that waits on a flag nothing sets for
 * ``timeout_us`` microseconds, so tests can exercise that path. */
swa_status swa_device_error_check(void* stream);
swa_status swa_debug_wait_timeout(int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SWA_B200_H */
