/*
 * lvq.h — C ABI of liblvq: LoopVQ loop-axis vector quantization of a looped
 * transformer's KV cache, and decode attention over the coded cache, for
 * NVIDIA B200 (sm_100a).
 *
 * Method (LoopVQ, "LoopVQ: Sub 1-bit KV Cache Quantization for Looped
 * Transformers"; pages: the onedev.kr LoopVQ summary, sections "how it
 * differs" and "premises and limits"; the rit.work LoopVQ article, sections
 * "one code describes several loop steps" and "when LoopVQ changes the
 * deployment plan"; the weekinpapers.com abstract):
 *   - the T loop steps are cut into blocks of Tc consecutive steps (Tc | T,
 *     Tc | G); one joint G-vector holds c = G/Tc channels of each step of the
 *     block (keys taken before RoPE) and is encoded as the index of its nearest
 *     entry in a 256-entry codebook: 8/G bits per cached element;
 *   - the cache is built from 8-token pages; the first (sink) tokens and the
 *     recent tokens stay bf16, older pages hold one index row per block;
 *     prefill encodes once all Tc steps exist, decode writes new tokens to the
 *     recent window and encodes the oldest page every 8 tokens across all
 *     layers and loop steps;
 *   - attention at loop step t reads only the step-t slice of each codebook,
 *     applies RoPE to the reconstructed keys, splits the coded tokens
 *     Flash-Decoding style and merges the splits with the bf16 tokens by
 *     logsumexp;
 *   - codebooks come from k-means over joint vectors (here the plain,
 *     unweighted form: lvq_encode_prefill assigns, lvq_kmeans_update moves
 *     the entries).
 *
 * Conventions for every entry point:
 *   - The caller owns every buffer (device memory unless stated).  The
 *     library allocates no device memory and keeps no global state, apart from
 *     the fixed workspace of lvq_decode_attention_noalloc and the settings of
 *     the lvq_debug_faults test hook; an lvq_pool is host bookkeeping the
 *     caller creates and destroys.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  Errors the host can see (bad
 *     config, null or misaligned pointer, out-of-range argument) return at
 *     once with nothing launched.  A failed launch returns LVQ_ECUDA.
 *   - Errors only the device can see (a context longer than the layout's
 *     capacity, a recent window overfull) are written to *dev_status, a
 *     caller-owned int32 in device memory, as the first error code seen
 *     (atomic compare-and-swap from LVQ_OK); the affected request is skipped.
 *     Read it after synchronizing.
 *   - Sizes and element strides of every buffer come from lvq_cache_layout.
 *   - Positions are absolute and 0-based: sink token i is at position i,
 *     coded token n at n_sink + n, recent tokens follow the coded ones; the
 *     decode query is the newest token, at position ctx_len - 1.
 *   - Supported shapes: K = 256, page_tokens = 8, head_dim in {64, 128},
 *     c = G/Tc in {4, 8, 16} (64: {4, 8}), G in {16, 32}, n_q_heads a multiple of
 *     n_kv_heads (query head hq reads KV head hq / (n_q_heads / n_kv_heads)).  Anything else returns
 *     LVQ_EUNSUPPORTED: there is no fallback path.
 */
#ifndef LVQ_H
#define LVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LVQ_API __attribute__((visibility("default")))
#else
#define LVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LVQ_OK = 0,
  LVQ_EINVAL = 1,        /* bad argument: null/misaligned pointer, out-of-range value */
  LVQ_EUNSUPPORTED = 2,  /* valid LoopVQ shape that this build has no kernel for */
  LVQ_ECAPACITY = 3,     /* request larger than the layout's capacity (device-side) */
  LVQ_ECUDA = 4,         /* a CUDA call or kernel launch failed */
  LVQ_ETIMEOUT = 5,      /* a bounded device-side wait expired */
  LVQ_EDEVICE = 6        /* no usable sm_100 device */
} lvq_status;

/* Model and cache shape.  Plain data, filled by the caller, validated on
 * every call. */
typedef struct {
  int32_t n_layers;     /* attention layers of the looped block */
  int32_t n_kv_heads;   /* KV heads */
  int32_t n_q_heads;    /* query heads, a multiple of n_kv_heads */
  int32_t head_dim;     /* d: 64 or 128 */
  int32_t T;            /* loop steps */
  int32_t Tc;           /* loop steps per block; Tc | T and Tc | G */
  int32_t G;            /* joint-vector length; c = G/Tc channels per step */
  int32_t K;            /* codebook entries: must be 256 (8-bit codes) */
  int32_t n_sink;       /* bf16 sink tokens at the start of the context */
  int32_t n_recent;     /* bf16 recent-window tokens kept after an encode */
  int32_t page_tokens;  /* must be 8 */
  int32_t max_batch;    /* requests the cache holds */
  int32_t max_ctx;      /* longest context (tokens, including the query) */
  int32_t max_splits;   /* largest num_splits lvq_decode_attention accepts (<= 256) */
  float rope_base;      /* RoPE base (10000 for the Ouro-shaped workloads) */
  /* Code storage.  pool_pages = 0: every (layer, block, request, head, K/V) has its own
   * stream of max_pages pages.  pool_pages > 0: the requests share a pool of pool_pages
   * 8-token pages per (layer, block, head, K/V), and page_table (device int32
   * [max_batch][page_table_stride], see lvq_layout) maps request b's logical page i (its
   * coded tokens 8i .. 8i+7) to a physical page, the same id in every (layer, block, head,
   * K/V) pool; ids come from an lvq_pool.  A page table entry that a call needs but that is
   * out of range (< 0 or >= pool_pages) sets LVQ_ECAPACITY in *dev_status; the decode then
   * reads page 0 in its place (its output for that request is not meaningful) and the
   * encoders skip the page. */
  int32_t pool_pages;
  int32_t reserved_;    /* must be 0 */
  const int32_t* page_table;   /* device pointer; NULL when pool_pages = 0 */
} lvq_config;

/* Derived sizes and layouts.  All byte counts are totals for the whole
 * buffer; strides are in elements of the buffer's own type, outermost
 * dimension first. */
typedef struct {
  int32_t c;            /* channels per group per step, G/Tc */
  int32_t n_groups;     /* n_g = head_dim / c */
  int32_t n_blocks;     /* n_blk = T / Tc: index rows per token, head and K/V */
  int32_t ring_tokens;  /* R = n_recent + page_tokens: recent-window slots */
  int32_t max_pages;    /* coded pages per (layer, block, request, head) */
  int32_t page_bytes;   /* bytes of one coded page of K or of V: n_g * 8 */
  int32_t rope_coarse;  /* rows of the coarse RoPE table (positions 8k) */
  int32_t page_table_stride;   /* int32 entries per request in the page table (pool mode) */
  /* uint8 codes, [layer][n_blk][B][Hkv][kv][page][n_g][8]: byte (g, j) of a
   * page holds group g's code of the page's token j (token n of the coded
   * region sits in page n/8 at j = n%8).  The K pages of a (layer, block,
   * request, head) form one contiguous stream, followed by its V pages.
   * Pool mode: [layer][n_blk][Hkv][kv][pool_pages][n_g][8], request b's logical page i
   * at physical page page_table[b][i] (idx_strides: the 7 dimensions, then 0). */
  size_t idx_bytes;
  int64_t idx_strides[8];
  /* device int32 [max_batch][page_table_stride]; 0 outside pool mode */
  size_t page_table_bytes;
  /* bf16 logical codebooks, [layer][kv][n_blk][Hkv][n_g][256][G]; element
   * s*c + e of an entry is step s of the block, channel g*c + e. */
  size_t cb_bytes;
  int64_t cb_strides[7];
  /* bf16 step-major packed codebooks, [layer][kv][n_blk][Hkv][Tc][256][n_g][c]:
   * the step slice of one (layer, kv, block, head, step) is one contiguous
   * 256*d*2-byte span.  Written by lvq_pack_codebooks. */
  size_t cbp_bytes;
  int64_t cbp_strides[8];
  /* fp32 squared entry norms, [layer][kv][n_blk][Hkv][n_g][256] */
  size_t cb_norm_bytes;
  /* bf16 sink tokens, [layer][kv][T][B][Hkv][n_sink][d] (pre-RoPE keys) */
  size_t sink_bytes;
  int64_t sink_strides[7];
  /* bf16 recent window, [layer][kv][T][B][Hkv][R][d] (pre-RoPE keys); the
   * token at absolute position p >= n_sink lives in slot (p - n_sink) mod R. */
  size_t ring_bytes;
  int64_t ring_strides[7];
  /* fp32 RoPE tables: coarse [rope_coarse][d/2] (cos, sin) of 8k*theta_f,
   * then fine [8][d/2] (cos, sin) of r*theta_f.  Written by lvq_rope_table. */
  size_t rope_bytes;
  /* scratch of lvq_decode_attention: fp32 partials
   * [B][Hq][max_splits][2][d + 2] (per split: its coded tokens, its share of
   * the bf16 tokens), then int32 merge counters [B][Hq].  Zero it once before
   * first use; every call leaves the counters at zero. */
  size_t workspace_bytes;
} lvq_layout;

/* Sizes and strides for cfg.  Host arithmetic only: no CUDA call, usable
 * without a GPU.  Returns LVQ_EINVAL / LVQ_EUNSUPPORTED for a bad shape.  In
 * pool mode cfg->page_table may still be NULL here (the layout gives the page
 * table's size); every other call needs it. */
LVQ_API lvq_status lvq_cache_layout(const lvq_config* cfg, lvq_layout* out);

/* Message for a status code (static string, never NULL). */
LVQ_API const char* lvq_status_string(lvq_status s);

/* Test hook, not for normal use (process-global; not thread-safe).  Every device-side wait
 * of the later calls gives up after `wait_iters` polls (<= 0: the normal bound, about 2^24)
 * and reports LVQ_ETIMEOUT in *dev_status; `fault_mask` makes a copy never happen, so that
 * such a wait runs out: bit 0 -- lvq_decode_attention skips the first code chunk of every
 * CTA; bit 1 -- lvq_kmeans_update skips the first tile of every CTA.  Kernels still wait
 * (bounded) for every copy they did issue before they exit, so the context stays usable.
 * LVQ_EINVAL for unknown bits.  lvq_debug_faults(0, 0) restores normal operation. */
LVQ_API lvq_status lvq_debug_faults(int64_t wait_iters, int32_t fault_mask);

/* Caps the CTAs (one per SM) of the later lvq_decode_attention calls of this process: 0 (the
 * default) launches one CTA per work item (request, query head, split); max_ctas > 0 launches
 * at most that many, each walking a contiguous run of work items ordered by KV head, cost-
 * balanced by coded tokens (the step slices of a KV head are copied once per run, and the next
 * item's code pages stream in while the current item finishes).  Use it to leave SMs to a
 * concurrent kernel.  Both grids compute the same attention (the bf16 share's fp32 summation
 * order differs); on the Ouro-shaped workloads the uncapped grid is as fast or faster.
 * Process-global, not thread-safe.  LVQ_EINVAL if max_ctas < 0. */
LVQ_API lvq_status lvq_decode_max_ctas(int32_t max_ctas);

/* Helper: packs the logical codebooks (cb, see lvq_layout.cb_*) into the
 * step-major layout the decoder reads (cbp) and computes each entry's squared
 * norm in fp64, rounded to fp32 (cb_norm, may be NULL).  All device
 * pointers, 16-byte aligned.  Codebooks are model-specific ("LoopVQ summary",
 * "premises and limits"); this only changes their layout. */
LVQ_API lvq_status lvq_pack_codebooks(const lvq_config* cfg, const lvq_layout* lay, const void* cb,
                              void* cbp, float* cb_norm, void* stream);

/* Helper: writes the RoPE tables (rope, lay->rope_bytes) in fp64 on the
 * device, rounded to fp32.  theta_f = rope_base^(-2f/d), rotate-half pairs
 * (f, f + d/2).  Keys are rotated after dequantisation ("LoopVQ summary",
 * "how it differs"). */
LVQ_API lvq_status lvq_rope_table(const lvq_config* cfg, const lvq_layout* lay, float* rope, void* stream);

/* Prefill encode ("LoopVQ summary", "premises and limits": the keys and values
 * of every loop step are kept until the last step, then each joint vector is
 * encoded against the codebook).
 *   layer: 0..n_layers-1, or -1 for every layer in one call.
 *   req: request 0..max_batch-1.
 *   kv: device bf16 [2][T][n_tok_total][Hkv][d] pre-RoPE keys (kv=0) and values
 *       (kv=1) of one layer and request; kv_tok_stride is the element stride
 *       between consecutive tokens (>= Hkv*d); the step stride is
 *       kv_tok_stride * kv_tokens and the K/V stride T times that.  With
 *       layer = -1 it holds every layer, [n_layers][2][T][...], the layer
 *       stride 2 T times the step stride; the tensor-core encoder then spreads
 *       all layers' work over one persistent launch.
 *   kv_tokens: tokens in kv (its token extent).
 *   tok_begin, n_tok: tokens [tok_begin, tok_begin + n_tok) of kv are encoded
 *       into coded slots [coded_offset, coded_offset + n_tok).
 *   cb: logical codebooks (lay->cb_*); idx: the code buffer (lay->idx_*).
 * Every index is the nearest entry's (squared L2 on the bf16 values, lowest
 * index on exact ties), computed exactly in fp64. */
LVQ_API lvq_status lvq_encode_prefill(const lvq_config* cfg, const lvq_layout* lay, int32_t layer,
                              int32_t req, const void* kv, int64_t kv_tok_stride,
                              int32_t kv_tokens, int32_t tok_begin, int32_t n_tok,
                              int32_t coded_offset, const void* cb, uint8_t* idx,
                              int32_t* dev_status, void* stream);

/* Codebook construction: the update step of one plain k-means (Lloyd)
 * iteration over the joint vectors of one layer ("LoopVQ summary", "how it
 * differs": codebooks are initialised by k-means over joint vectors -- Fisher-
 * weighted there, unweighted here; "premises and limits": k-means over the
 * calibration tokens).  The assignment step is lvq_encode_prefill with the same
 * layer, req, kv, tokens and coded_offset; this call then moves every entry of
 * every (K/V, block, head, group) codebook of `layer` to the mean of the joint
 * vectors coded with it (fp64 sums, the mean rounded once to bf16, to nearest,
 * ties to even) and leaves an entry that no vector chose unchanged.
 *   kv, kv_tok_stride, kv_tokens, tok_begin, n_tok, coded_offset: as for
 *     lvq_encode_prefill (tokens [tok_begin, tok_begin + n_tok) of kv, their
 *     codes in slots [coded_offset, coded_offset + n_tok) of request req).
 *   idx: the code buffer holding those codes (read only).
 *   cb: logical codebooks, updated in place for `layer` (lay->cb_*).
 *   counts: nullable device uint32 [2][n_blk][Hkv][n_g][256]: vectors per entry.
 * The packed codebooks and norms the decoder reads are not touched: call
 * lvq_pack_codebooks after the last iteration.  LVQ_EUNSUPPORTED where
 * (d/c) is not a multiple of 64/G or kv_tok_stride is not a multiple of 8
 * (the values are read by TMA), and in pool mode (codebooks are built before
 * serving, on per-request streams); LVQ_EINVAL for out-of-range arguments, null
 * or misaligned (16-byte) pointers.  Device-side: LVQ_ETIMEOUT in *dev_status
 * if a copy never lands (every wait is bounded). */
LVQ_API lvq_status lvq_kmeans_update(const lvq_config* cfg, const lvq_layout* lay, int32_t layer,
                             int32_t req, const void* kv, int64_t kv_tok_stride, int32_t kv_tokens,
                             int32_t tok_begin, int32_t n_tok, int32_t coded_offset,
                             const uint8_t* idx, void* cb, uint32_t* counts, int32_t* dev_status,
                             void* stream);

/* Decode-time page encode ("LoopVQ summary", "premises and limits": new tokens
 * go to the recent window; every 8 tokens the oldest page is quantized across
 * all layers and loop steps).  For every request b < batch whose recent
 * window holds at least n_recent + 8 tokens (ctx_len[b] - n_sink -
 * coded_len[b] >= R), encodes its 8 oldest recent tokens (every layer, K/V,
 * block, head, group) into coded slots coded_len[b] .. coded_len[b] + 7, then
 * advances coded_len[b] by 8.  Requests with fewer recent tokens are left
 * untouched, so the call can be issued every 8 tokens from a CUDA graph.
 *   ctx_len, coded_len: device int32 [batch] (batch <= 1024, else
 *     LVQ_EUNSUPPORTED).  ring: bf16 recent window.  cb: logical codebooks.
 *   cb_norm: their fp32 squared entry norms as lvq_pack_codebooks writes them
 *     (required).
 * Every codebook is read once per call whatever the number of due requests. */
LVQ_API lvq_status lvq_encode_page(const lvq_config* cfg, const lvq_layout* lay, int32_t batch,
                           const int32_t* ctx_len, int32_t* coded_len, const void* ring,
                           const void* cb, const float* cb_norm, uint8_t* idx, int32_t* dev_status,
                           void* stream);

/* Decode attention of loop step `step` of layer `layer` ("LoopVQ summary",
 * "premises and limits"; "LoopVQ article", "when LoopVQ changes the deployment
 * plan").
 *   q: device bf16 [batch][Hq][d] pre-RoPE queries (rotated here at ctx_len-1).
 *   ctx_len, coded_len: device int32 [batch]; request b attends to sink tokens
 *     [0, n_sink), coded tokens [n_sink, n_sink + coded_len[b]) and recent
 *     tokens [n_sink + coded_len[b], ctx_len[b]).
 *   sink, ring, idx, cbp, rope: cache buffers (lay->*).
 *   num_splits: coded tokens are cut into num_splits ranges, split j covering
 *     [j*chunk, min(L, (j+1)*chunk)), chunk = ceil(L/num_splits) rounded up to
 *     a multiple of 32; the bf16 tokens are one more partial.
 *   workspace: scratch of lay->workspace_bytes, zeroed once before first use
 *     (its merge counters return to zero at the end of every call).  Calls
 *     that share a workspace must not overlap on the GPU.
 *   out: device fp32 [batch][Hq][d]; lse: device fp32 [batch][Hq], natural log
 *     of the softmax denominator (scores scaled by 1/sqrt(d)).
 *   split_lse: NULL, or device fp32 [batch][Hq][num_splits + 1] receiving each
 *     partial's LSE (-inf for an empty one); a test hook. */
LVQ_API lvq_status lvq_decode_attention(const lvq_config* cfg, const lvq_layout* lay, int32_t layer,
                                int32_t step, int32_t batch, const void* q,
                                const int32_t* ctx_len, const int32_t* coded_len,
                                const void* sink, const void* ring, const uint8_t* idx,
                                const void* cbp, const float* rope, int32_t num_splits,
                                float* workspace, float* out, float* lse, float* split_lse,
                                int32_t* dev_status, void* stream);

/* Test hook: step-`step` reconstruction of coded tokens [tok_begin, tok_begin +
 * n_tok) of request req, layer, K (kv=0) or V (kv=1), all heads: device bf16
 * out [n_tok][Hkv][d], pre-RoPE, bit-exact copies of codebook elements
 * ("LoopVQ summary", "how it differs": each step restores only its own share
 * of the entry). */
LVQ_API lvq_status lvq_dequantize(const lvq_config* cfg, const lvq_layout* lay, int32_t layer,
                          int32_t step, int32_t req, int32_t kv, const uint8_t* idx,
                          const void* cbp, int32_t tok_begin, int32_t n_tok, void* out,
                          void* stream);

/* Page pool bookkeeping (host memory only; device buffers stay the caller's).  "LoopVQ
 * summary", "premises and limits": the cache is built from 8-token pages.  An lvq_pool hands
 * out the physical page ids of a pool of n_pages pages (pool mode of lvq_config) to requests
 * of any length and takes them back when a request ends; the caller writes the ids into the
 * device page table.  Ids are handed out lowest first, so a request's pages tend to form
 * runs of consecutive ids (the decode copies a run with one bulk copy).  Not thread-safe:
 * one pool per host thread, or the caller's own lock. */
typedef struct lvq_pool lvq_pool;
/* n_pages >= 1; *out receives the pool (free it with lvq_pool_destroy).  LVQ_EINVAL for a
 * bad argument. */
LVQ_API lvq_status lvq_pool_create(int32_t n_pages, lvq_pool** out);
LVQ_API void lvq_pool_destroy(lvq_pool* pool);
/* n free page ids into ids[0..n), lowest first; LVQ_ECAPACITY (nothing taken) if fewer than
 * n are free. */
LVQ_API lvq_status lvq_pool_alloc(lvq_pool* pool, int32_t n, int32_t* ids);
/* Returns n ids to the pool; LVQ_EINVAL (nothing returned) if an id is out of range, not
 * currently handed out, or repeated. */
LVQ_API lvq_status lvq_pool_free(lvq_pool* pool, const int32_t* ids, int32_t n);
/* Free page ids (-1 for a null pool). */
LVQ_API int32_t lvq_pool_available(const lvq_pool* pool);

/* Decode attention without a caller-supplied workspace.  The pages have no
 * counterpart of this entry point: it exists for callers that cannot allocate
 * device memory for the workspace -- for example a plugin inside a serving
 * engine whose memory pool owns the whole device, or a deployment that forbids
 * allocations once it has reserved its memory budget.
 *
 * Arguments and results are those of lvq_decode_attention without
 * `workspace`.  The workspace is a file-scope device array inside the library
 * (4 MiB, held by every GPU that loads the library until the process exits):
 *   - a layout whose workspace_bytes exceeds 4 MiB is rejected with
 *     LVQ_ECAPACITY before anything is launched;
 *   - the call allocates nothing (no cudaMalloc or allocating library
 *     routine); it zeroes the merge counters with cudaMemsetAsync on `stream`;
 *   - the first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress), and looks it up again only when the
 *     device's current context has changed (e.g. after cudaDeviceReset); make
 *     that first call before any stream capture.  The lookup is guarded by a
 *     lock, so concurrent first calls from several host threads are safe;
 *   - every call shares the one array: calls that overlap on the GPU (other
 *     streams, other host threads, other decode calls in flight) race and must
 *     be serialized by the caller. */
LVQ_API lvq_status lvq_decode_attention_noalloc(const lvq_config* cfg, const lvq_layout* lay, int32_t layer,
                                                int32_t step, int32_t batch, const void* q,
                                                const int32_t* ctx_len, const int32_t* coded_len,
                                                const void* sink, const void* ring, const uint8_t* idx,
                                                const void* cbp, const float* rope, int32_t num_splits,
                                                float* out, float* lse, float* split_lse,
                                                int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LVQ_H */
