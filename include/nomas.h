/*
 * nomas.h -- C ABI of libnomas, segment-over-cache attention for B200 (sm_100a).
 *
 * The operations are those of one attention layer of a segment-autoregressive
 * video world model whose only memory is a per-layer KV cache of past
 * segments:
 *   "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
 *   (ai.thesatyajit.com), sections "How one segment is made", "Writing the
 *   segment into memory", "What 'world memory' stores" and "The 4090 preset".
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned DEVICE memory; the library never allocates,
 *     frees or keeps a pointer after a call returns.
 *   - bf16 values are passed as raw 16-bit patterns (void pointers).  Q, K, V
 *     and O rows have layout [tokens][heads][head_dim], contiguous; a row of
 *     16 x 128 bf16 is 4096 bytes.  Every tensor pointer must be 16-byte
 *     aligned.
 *   - Only heads = 16 and head_dim = 128 are implemented (and 1, 2, 4 or 8
 *     heads for dense bf16 attention -- nomas_segment_attention, _ex, _split
 *     and _split_noalloc -- and for nomas_attention_merge); other values
 *     return NOMAS_ERR_UNSUPPORTED.
 *   - Every call is asynchronous on the caller's stream (`stream` is a
 *     cudaStream_t; NULL is the legacy default stream) and never synchronises.
 *     Argument errors are detected on the host before anything is launched and
 *     leave all memory untouched.
 *   - Errors found on the device (a bad index in a device-resident frame list,
 *     a pipeline wait that exceeded its time limit) never trap: the kernel
 *     ORs a NOMAS_DEVERR_* bit into the caller's optional int32 word
 *     `dev_err` (device memory) and skips the affected work.  The caller
 *     reads the word after synchronising.
 *   - nomas_last_error() returns a per-thread message for the last failing
 *     call made by that thread.
 */
#ifndef NOMAS_H
#define NOMAS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NOMAS_OK = 0,
  NOMAS_ERR_INVALID_ARG = 1, /* NULL / misaligned pointer, bad size or layout */
  NOMAS_ERR_CAPACITY = 2,    /* a write would run past a cache's capacity     */
  NOMAS_ERR_INDEX = 3,       /* a host frame index outside the source cache   */
  NOMAS_ERR_UNSUPPORTED = 4, /* a head count or head_dim not implemented, too many spans */
  NOMAS_ERR_CUDA = 5         /* a CUDA runtime/driver call failed             */
} nomas_status;

/* Bits ORed into *dev_err by kernels. */
#define NOMAS_DEVERR_BAD_FRAME_INDEX 0x1 /* select: device list entry out of range */
#define NOMAS_DEVERR_WAIT_TIMEOUT 0x2    /* attention: a pipeline wait timed out   */
#define NOMAS_DEVERR_BAD_TILE_INDEX 0x4  /* sparse attention: tile id out of range */

#define NOMAS_HEADS 16
#define NOMAS_HEAD_DIM 128
#define NOMAS_MAX_SPANS 4
#define NOMAS_MAX_MERGE_PARTS 32   /* partial results one attention merge combines */
#define NOMAS_MAX_MERGE_OUTPUTS 32 /* outputs one peer merge writes its rows to     */
/* Size of the scratch array built into the library for
 * nomas_segment_attention_split_noalloc: 64 MiB per device that uses it. */
#define NOMAS_NOALLOC_SCRATCH_BYTES (64ll << 20)

/*
 * 3D rotary configuration: the head dimension is split into a temporal chunk
 * of d_t dims, a grid-row chunk of d_h dims and a grid-column chunk of d_w
 * dims (d_t + d_h + d_w = head_dim, each even and > 0); pair j of a chunk of
 * width d turns by pos * theta^(-2j/d) radians.  Pairs are adjacent elements
 * (2j, 2j+1) inside the chunk.  The page's own values are d = 16/56/56 and
 * theta = 256 ("How one segment is made", item "The blocks"); 32/48/48 with
 * theta = 10000 is the default of the measured workloads.
 */
typedef struct {
  int32_t d_t, d_h, d_w;
  float theta;
} nomas_rope3d_cfg;

/*
 * Row layout of one segment: `frames * grid_h * grid_w` video rows first
 * (frame-major, then row-major over the latent grid; one token per grid cell,
 * "How one segment is made", items "Video tokens" and "The blocks"), then
 * `n_text` text rows.  Video row r sits at t = t0 + r / (grid_h*grid_w),
 * h = (r / grid_w) % grid_h, w = r % grid_w; t0 is the number of latent
 * frames already written to the history, so positions continue across
 * segments.  Text rows carry no 3D position and are not rotated.
 */
typedef struct {
  int32_t frames, grid_h, grid_w, t0, n_text;
} nomas_seg_layout;

/*
 * One layer's KV cache ("What 'world memory' stores"): K and V each hold
 * `capacity` rows of [heads][head_dim] bf16; rows [0, len) are valid.  A
 * latent frame is `tokens_per_frame` consecutive rows.  Keys are stored
 * after rotation, so a frame keeps its original position when it is later
 * gathered into a window.  The struct is host memory owned by the caller;
 * k and v point to device memory owned by the caller.
 */
typedef struct {
  void *k, *v;
  int64_t capacity, len;
  int32_t tokens_per_frame, heads, head_dim;
} nomas_kvcache;

/* A contiguous run of `len` key/value rows ([len][heads][head_dim] bf16). */
typedef struct {
  const void *k, *v;
  int64_t len;
} nomas_kv_span;

/* Message describing the last failing call on this host thread ("" if none). */
const char *nomas_last_error(void);

/* Library version string. */
const char *nomas_version(void);

/*
 * 3D RoPE on Q and K ("How one segment is made", item "The blocks": 3D RoPE
 * over (t, h, w)).
 *   q, k       : [n][heads][head_dim] bf16 inputs, n = video rows + n_text.
 *                k may be NULL (then k_out must be NULL): Q only.
 *   q_out,k_out: outputs of the same shape; may equal the inputs (in place),
 *                must not otherwise overlap them.  Text rows are copied.
 *   layout     : row layout (host struct); cfg: rotary configuration (host).
 * Rotation is fp32 arithmetic on the widened bf16 inputs with angles and their
 * cosines/sines evaluated in double, rounded to bf16 to nearest-even.
 * Errors: NOMAS_ERR_INVALID_ARG, NOMAS_ERR_UNSUPPORTED, NOMAS_ERR_CUDA.
 */
nomas_status nomas_rope3d_qk(const void *q, const void *k, void *q_out, void *k_out,
                             const nomas_seg_layout *layout, const nomas_rope3d_cfg *cfg,
                             int32_t heads, int32_t head_dim, void *stream);

/*
 * Segment write-back into the cache, fused with 3D RoPE ("Writing the
 * segment into memory": after a segment is generated its keys and values are
 * stored in the cache; "What 'world memory' stores": the cache grows by one
 * segment per step).
 *   cache   : host struct; rows [len, len + n_tokens) of cache->k receive the
 *             rotated segment keys, the same rows of cache->v the values bit
 *             for bit; every other row is left untouched.  On success
 *             cache->len += n_tokens.
 *   k_seg, v_seg: [n_tokens][heads][head_dim] bf16, the segment's video rows.
 *   q_in, q_out : optional (both NULL, or both set): the segment's Q,
 *             [n_tokens + layout->n_text][heads][head_dim]; video rows are
 *             rotated into q_out, text rows copied (q_out may equal q_in).
 *   layout  : required when cfg != NULL; then n_tokens must equal
 *             frames * grid_h * grid_w.
 *   cfg     : NULL -> plain copy of K and V (and Q), no rotation.
 * Errors: NOMAS_ERR_CAPACITY if len + n_tokens > capacity (nothing written,
 * len unchanged); NOMAS_ERR_INVALID_ARG, NOMAS_ERR_UNSUPPORTED, NOMAS_ERR_CUDA.
 */
nomas_status nomas_kvcache_append(nomas_kvcache *cache, const void *k_seg, const void *v_seg,
                                  int64_t n_tokens, const void *q_in, void *q_out,
                                  const nomas_seg_layout *layout, const nomas_rope3d_cfg *cfg,
                                  void *stream);

/*
 * Bounded active history: gather whole latent frames of `src` into the
 * contiguous `window` ("The 4090 preset": before each segment only a list of
 * past latent frames is restored to the GPU).  Window rows
 * [j*P, (j+1)*P) receive source rows [idx[j]*P, (idx[j]+1)*P), P =
 * src->tokens_per_frame, for K and V, bit for bit.  Repeats are allowed.
 *   frame_idx     : int32[n_frames], host memory if idx_on_device == 0, device
 *                   memory otherwise.
 *   window        : host struct; needs capacity >= n_frames * P and the same
 *                   heads/head_dim; its tokens_per_frame is set to P and, on
 *                   success, its len to n_frames * P.
 *   dev_err       : device int32, required when idx_on_device != 0.
 * A host index outside [0, src->len / P) returns NOMAS_ERR_INDEX before any
 * launch.  A bad device index sets NOMAS_DEVERR_BAD_FRAME_INDEX in *dev_err
 * and its window rows are left untouched; the other frames are copied.
 * Errors: NOMAS_ERR_INDEX, NOMAS_ERR_CAPACITY, NOMAS_ERR_INVALID_ARG,
 * NOMAS_ERR_UNSUPPORTED, NOMAS_ERR_CUDA.
 */
nomas_status nomas_kvcache_select(const nomas_kvcache *src, const int32_t *frame_idx,
                                  int32_t n_frames, int32_t idx_on_device, nomas_kvcache *window,
                                  int32_t *dev_err, void *stream);

/*
 * Segment-over-cache attention ("How one segment is made": joint attention
 * of text and video tokens, causal across segments so the current segment
 * reads earlier ones from the KV cache; "What 'world memory' stores": the
 * queries of segment k attend over the cache).  Every query row attends to
 * every key of every span with no mask:
 *   O[i,h] = sum_j softmax_j(scale * <q[i,h], k[j,h]>) v[j,h]
 *   LSE[h,i] = ln sum_j exp(scale * <q[i,h], k[j,h]>)
 *   q      : [n_q][heads][head_dim] bf16 (already rotated).
 *   spans  : host array of n_spans (1..NOMAS_MAX_SPANS) key/value runs, e.g.
 *            cache (or window), text, segment; len 0 spans are skipped.
 *   o      : [n_q][heads][head_dim] bf16 output, must not overlap inputs.
 *   lse    : optional fp32 [heads][n_q] output (natural log); NULL to skip.
 *   softmax_scale: <= 0 selects 1/sqrt(head_dim).
 *   dev_err: optional device int32 (see the conventions above).
 *   heads  : 16; or 1, 2, 4 or 8 ("What 'world memory' stores": the cache
 *            spread over 8 GPUs; with attention sharded by heads each GPU
 *            holds all rows for its share of the heads), in which case q, the
 *            spans and o hold that many heads per row and lse is
 *            [heads][n_q].  head_dim: 128.
 * With no keys at all, O = 0 and LSE = -inf.  bf16 operands, fp32 scores,
 * softmax and accumulation; O rounded to bf16 to nearest-even.
 * Errors: NOMAS_ERR_INVALID_ARG, NOMAS_ERR_UNSUPPORTED, NOMAS_ERR_CUDA.
 */
nomas_status nomas_segment_attention(const void *q, int64_t n_q, const nomas_kv_span *spans,
                                     int32_t n_spans, void *o, float *lse, float softmax_scale,
                                     int32_t heads, int32_t head_dim, int32_t *dev_err,
                                     void *stream);

/*
 * INT8 layer cache ("The 4090 preset": the cache is quantised once per
 * segment to one byte per value plus an FP32 scale per token and head, 4,224
 * B per token per layer for K and V together).  k and v hold int8 codes
 * [capacity][heads][head_dim]; k_scale and v_scale hold fp32 [capacity][heads].
 * Value = code * scale.  Caller-owned device memory, 16-byte aligned.
 */
typedef struct {
  void *k, *v;
  float *k_scale, *v_scale;
  int64_t capacity, len;
  int32_t tokens_per_frame, heads, head_dim;
} nomas_kvcache_i8;

/*
 * nomas_kvcache_append into an INT8 cache ("The 4090 preset": the finished
 * segment's K/V are quantised to one byte per value once, when they are
 * written to the cache): the rotated segment keys (rounded
 * to bf16, as the bf16 path would store them) and the values are quantised
 * per (token, head): with a = absmax, the stored scale is a / 127 rounded to
 * the nearest fp32, and the code is the integer nearest to the exact
 * quotient 127 x / a, ties to even; an all-zero (token, head) gets scale 0
 * and codes 0.  Q is handled exactly as
 * in nomas_kvcache_append.  Same errors as nomas_kvcache_append.
 */
nomas_status nomas_kvcache_append_i8(nomas_kvcache_i8 *cache, const void *k_seg,
                                     const void *v_seg, int64_t n_tokens, const void *q_in,
                                     void *q_out, const nomas_seg_layout *layout,
                                     const nomas_rope3d_cfg *cfg, void *stream);

/*
 * nomas_kvcache_select from an INT8 cache into a bf16 window ("The 4090
 * preset": the chosen past frames are restored to the GPU before each
 * segment): the listed
 * frames are restored to the GPU-side window as bf16 values: the exact
 * product code * scale rounded once to the nearest bf16, ties to even.  Same
 * arguments, index checks and errors as nomas_kvcache_select.
 */
nomas_status nomas_kvcache_select_i8(const nomas_kvcache_i8 *src, const int32_t *frame_idx,
                                     int32_t n_frames, int32_t idx_on_device,
                                     nomas_kvcache *window, int32_t *dev_err, void *stream);

/*
 * nomas_kvcache_select from an INT8 cache into an INT8 window ("The 4090
 * preset": the chosen past frames are kept on the GPU in INT8, 4,224 B per
 * token per layer): the listed frames' codes and scales are copied bit for
 * bit, nothing is dequantised; the window is then read by
 * nomas_segment_attention_i8.  Window rows [j*P, (j+1)*P) of k, v, k_scale
 * and v_scale receive source rows [idx[j]*P, (idx[j]+1)*P).  The window
 * needs capacity >= n_frames * P; its tokens_per_frame is set to P and, on
 * success, its len to n_frames * P.  Same frame lists, index checks and
 * errors as nomas_kvcache_select.
 */
nomas_status nomas_kvcache_select_i8_codes(const nomas_kvcache_i8 *src, const int32_t *frame_idx,
                                           int32_t n_frames, int32_t idx_on_device,
                                           nomas_kvcache_i8 *window, int32_t *dev_err,
                                           void *stream);

/* A contiguous run of `len` rows of an INT8 cache: codes [len][heads][head_dim]
 * int8 and scales [len][heads] fp32, for K and V; value = code * scale. */
typedef struct {
  const void *k, *v;
  const float *k_scale, *v_scale;
  int64_t len;
} nomas_kv_span_i8;

/*
 * Power-spaced choice of the past latent frames to keep resident ("The 4090
 * preset": N = min(budget, n_past), u_i = i/(N-1), d_i = i + rint((n_past -
 * N) u_i^gamma), kept frames n_past - 1 - d_i; the page's preset uses budget
 * 18 and gamma 2).  Host-only, no CUDA.
 *   out     : host int32[out_capacity]; receives the N kept frames in
 *             ascending order (frame 0, the oldest, is always kept when
 *             n_past > 0).  *n_out = N.
 * Errors: NOMAS_ERR_INVALID_ARG (negative counts, gamma < 0 or not finite,
 * n_out NULL), NOMAS_ERR_CAPACITY (out_capacity < N).
 */
nomas_status nomas_temporal_context_frames(int32_t n_past, int32_t budget, float gamma,
                                           int32_t *out, int32_t out_capacity, int32_t *n_out);

/*
 * Per-call options of nomas_segment_attention_ex.
 *   wait_limit_ns: time limit of every pipeline wait inside the kernel
 *                  (0 selects the default of 2 s).  A wait that runs out sets
 *                  NOMAS_DEVERR_WAIT_TIMEOUT in *dev_err; the affected query
 *                  block then sets its rows of O (and LSE) to NaN, releases
 *                  its resources and exits, and the CUDA context stays
 *                  usable.  The same holds in every attention entry point.
 *   testing_skip_kv_load: -1 in normal use.  For tests of the timeout path
 *                  only: a value k >= 0 makes every block leave out its k-th
 *                  K/V tile load (in the order its schedule loads them: K, V,
 *                  K, V ... for TWO_TILE; K, K, K, then V, K, V, K ... for
 *                  ONE_TILE and PAIR), so a consumer wait cannot complete and
 *                  must time out.
 *   pipeline:      the kernel schedule (NOMAS_ATTN_PIPELINE_*), 0 for the
 *                  library default.
 */
typedef struct {
  uint64_t wait_limit_ns;
  int32_t testing_skip_kv_load;
  int32_t pipeline;  /* NOMAS_ATTN_PIPELINE_*; 0 = the library default */
} nomas_attention_opts;

/*
 * Attention kernel schedules (same operation, arguments and results; they
 * differ in speed only):
 *   NOMAS_ATTN_PIPELINE_TWO_TILE: one CTA per 256 query rows as two 128-row
 *     tiles that share each K/V tile, one score tile per query tile in TMEM.
 *     The only schedule for block-sparse tile lists and INT8 histories.
 *   NOMAS_ATTN_PIPELINE_ONE_TILE: one CTA per 128 query rows, three score
 *     tiles in TMEM so that the scores of the next key tiles are computed
 *     while the softmax works on the current one.
 *   NOMAS_ATTN_PIPELINE_PAIR: as ONE_TILE, run by a cluster of two CTAs on two
 *     SMs with 256-row tensor-core instructions (cta_group::2); each CTA
 *     loads half of every K/V tile.
 * Dense bf16 calls use NOMAS_ATTN_PIPELINE_DEFAULT_DENSE unless told
 * otherwise (by their options or nomas_set_attention_pipeline); sparse and
 * INT8 calls use TWO_TILE whatever the process default, and one that names
 * ONE_TILE or PAIR in its options returns NOMAS_ERR_UNSUPPORTED.
 */
#define NOMAS_ATTN_PIPELINE_TWO_TILE 1
#define NOMAS_ATTN_PIPELINE_ONE_TILE 2
#define NOMAS_ATTN_PIPELINE_PAIR 3
#define NOMAS_ATTN_PIPELINE_DEFAULT_DENSE NOMAS_ATTN_PIPELINE_TWO_TILE

/*
 * A setting of this library, with no counterpart on the pages: sets the
 * schedule every later attention call of this process uses when its options
 * name none (opts NULL or opts->pipeline 0), for dense bf16 calls; 0 restores
 * the built-in choice.  Not synchronised with calls running on other host threads.
 * Errors: NOMAS_ERR_INVALID_ARG for a value outside 0..3.
 */
nomas_status nomas_set_attention_pipeline(int32_t pipeline);

/*
 * nomas_segment_attention ("How one segment is made": the joint attention of
 * the segment and the text over the history and themselves) with per-call
 * options (opts may be NULL for the defaults); identical otherwise.
 */
nomas_status nomas_segment_attention_ex(const void *q, int64_t n_q, const nomas_kv_span *spans,
                                        int32_t n_spans, void *o, float *lse, float softmax_scale,
                                        int32_t heads, int32_t head_dim, int32_t *dev_err,
                                        const nomas_attention_opts *opts, void *stream);

/*
 * nomas_segment_attention over a history held in INT8 ("The 4090 preset":
 * the resident past frames stay on the GPU in INT8; "Hy-Nomas en una RTX
 * 4090", section "El preset de una GPU": stored in INT8, computed in BF16).
 * The keys are `history` (dequantised: value = code * scale) followed by the
 * bf16 `spans` (e.g. text, segment); every query row attends to all of them
 * with no mask, exactly as nomas_segment_attention over the dequantised
 * history.  The kernel converts each 128-key tile of codes to bf16
 * (code * scale rounded to fp32, then to bf16 nearest-even) in shared
 * memory on its way to the tensor cores; the history is never expanded in
 * device memory.
 *   history : host struct; its len may be 0 (then this is
 *             nomas_segment_attention over `spans`).  Codes 16-byte
 *             aligned, scales 16-byte aligned.
 *   spans   : host array of n_spans bf16 runs, 1 + n_spans <=
 *             NOMAS_MAX_SPANS.
 *   opts    : as nomas_segment_attention_ex (may be NULL).
 * Other arguments and errors as nomas_segment_attention_ex; a build whose
 * INT8 kernel did not compile to the register allocation it assumes returns
 * NOMAS_ERR_CUDA before launching anything.
 */
nomas_status nomas_segment_attention_i8(const void *q, int64_t n_q,
                                        const nomas_kv_span_i8 *history,
                                        const nomas_kv_span *spans, int32_t n_spans, void *o,
                                        float *lse, float softmax_scale, int32_t heads,
                                        int32_t head_dim, int32_t *dev_err,
                                        const nomas_attention_opts *opts, void *stream);

/*
 * Block-sparse segment attention.  The single-GPU preset of the pages keeps
 * only a fraction of the candidate video key blocks after the first denoising
 * steps ("Hy-Nomas en una RTX 4090", section "El preset de una GPU": dense on the
 * first two denoising steps, then 25% of the candidate video blocks); the pages do not
 * give the selection rule, so the selection is an input.  Keys are cut into
 * tiles of NOMAS_SPARSE_BLOCK_K keys per span (the last tile of a span is
 * short), numbered consecutively over the spans in order; queries into blocks
 * of NOMAS_SPARSE_BLOCK_Q rows.  Query block b of head h attends to exactly
 * the tiles listed in tile_list[(b * heads + h) * max_tiles + i] for
 * i < tile_count[b * heads + h] (device int32 arrays; a tile listed twice
 * counts twice).  Ids outside the tiles are skipped and set
 * NOMAS_DEVERR_BAD_TILE_INDEX in *dev_err (required).  A block with no valid
 * tile gets O = 0, LSE = -inf.  Otherwise as nomas_segment_attention.
 */
#define NOMAS_SPARSE_BLOCK_Q 256
#define NOMAS_SPARSE_BLOCK_K 128
nomas_status nomas_segment_attention_sparse(const void *q, int64_t n_q,
                                            const nomas_kv_span *spans, int32_t n_spans,
                                            const int32_t *tile_list, const int32_t *tile_count,
                                            int32_t max_tiles, void *o, float *lse,
                                            float softmax_scale, int32_t heads, int32_t head_dim,
                                            int32_t *dev_err, void *stream);

/*
 * Key-split attention: the attention of nomas_segment_attention ("How one
 * segment is made": joint attention of the segment and text over the cached
 * history and themselves), for shapes whose query blocks alone do not fill
 * the GPU.  How the keys are cut is this library's choice, not the page's:
 * the concatenated key tiles (128 keys each, spans in order) are split into
 * kv_splits contiguous ranges; each (256-row query block, head, range) is one
 * CTA that writes a partial O (bf16) and LSE into `scratch`, and one merge
 * (the kernel of nomas_attention_merge) combines them into o and lse.  The
 * result equals nomas_segment_attention's up to the rounding of the partial
 * outputs to bf16.
 *   kv_splits : 1 <= kv_splits <= NOMAS_MAX_MERGE_PARTS; 1 is exactly
 *               nomas_segment_attention (scratch unused, may be NULL).
 *   scratch   : caller-owned device memory of at least
 *               nomas_segment_attention_scratch_bytes(n_q, kv_splits) bytes,
 *               16-byte aligned, overlapping none of q, o, lse and the spans;
 *               its contents are overwritten.
 * Other arguments as nomas_segment_attention.  Errors: as that call, plus
 * NOMAS_ERR_INVALID_ARG (kv_splits out of range, scratch NULL, misaligned or
 * overlapping) and NOMAS_ERR_CAPACITY (scratch_bytes too small).
 */
nomas_status nomas_segment_attention_split(const void *q, int64_t n_q, const nomas_kv_span *spans,
                                           int32_t n_spans, void *o, float *lse,
                                           float softmax_scale, int32_t heads, int32_t head_dim,
                                           int32_t kv_splits, void *scratch,
                                           int64_t scratch_bytes, int32_t *dev_err,
                                           void *stream);

/* Scratch bytes nomas_segment_attention_split needs: kv_splits x n_q x
 * (4096 + 64) for kv_splits > 1 (partial O rows and LSEs), else 0. */
int64_t nomas_segment_attention_scratch_bytes(int64_t n_q, int32_t kv_splits);

/*
 * nomas_segment_attention_split for callers that cannot allocate device
 * memory.  The pages have no counterpart to this call: it exists for this
 * library's users.  A caller whose device memory is claimed up front (a
 * serving process with a fixed budget handed out from its own pools), one
 * inside a framework that owns the device allocator and forbids allocations
 * behind its back, or one on a latency-critical path where cudaMalloc and
 * cudaFree (which can synchronise the device) are not allowed, cannot supply
 * the scratch that nomas_segment_attention_split takes.  This call uses an
 * array of NOMAS_NOALLOC_SCRATCH_BYTES built into the library instead, and
 * allocates nothing.
 *   Arguments as nomas_segment_attention_split, without scratch.
 *   Limit: kv_splits x n_q x (4096 + 64) bytes must fit in the array
 *   (about 8,000 query rows with 2 splits); larger requests return
 *   NOMAS_ERR_CAPACITY with a message giving both sizes, before anything is
 *   launched.
 *   The array is held on every device that uses this call until the process
 *   exits.  Its device address is looked up (with the device current) on
 *   every call made outside stream capture and kept per device; a call made
 *   while its stream is capturing uses the kept address.  So make one call
 *   on a device before any stream capture begins, and one after a reset of
 *   the device's primary context (cudaDeviceReset), which moves the array.
 *   Every call shares the array: calls that can run at the same time on the
 *   GPU (different streams, or different host threads) race on it and must
 *   be ordered by the caller.  Each call writes every byte of scratch it
 *   reads (a block whose pipeline wait ran out writes NaN rows, and its
 *   output rows come out NaN), so a call never sees the previous call's
 *   contents.
 * Errors: as nomas_segment_attention_split, plus NOMAS_ERR_CAPACITY (the
 * request exceeds the array) and NOMAS_ERR_CUDA (the address lookup failed,
 * or no address is known yet and the stream is capturing).
 */
nomas_status nomas_segment_attention_split_noalloc(const void *q, int64_t n_q,
                                                   const nomas_kv_span *spans, int32_t n_spans,
                                                   void *o, float *lse, float softmax_scale,
                                                   int32_t heads, int32_t head_dim,
                                                   int32_t kv_splits, int32_t *dev_err,
                                                   void *stream);

/*
 * Merge of attention results over disjoint key shards ("What 'world memory'
 * stores": the standard preset spreads the cache over eight GPUs, sp_size 8;
 * each GPU attends over its shard and the partial results are combined):
 * LSE = ln sum_r e^{LSE_r}, O = sum_r e^{LSE_r - LSE} O_r, accumulated in fp32.
 *   o_parts  : [n_parts][n_q][heads][head_dim] bf16 partial outputs (device).
 *   lse_parts: [n_parts][heads][n_q] fp32 partial LSEs (natural log, device).
 *   o        : [n_q][heads][head_dim] bf16 output; lse: optional [heads][n_q].
 * Parts with LSE = -inf are empty and contribute nothing; if all are empty the
 * row gets O = 0 and LSE = -inf.  A part with a NaN LSE (a partial whose
 * attention block ran out of time) makes the row's O and LSE NaN.  Outputs
 * must not overlap the inputs.
 * 1 <= n_parts <= NOMAS_MAX_MERGE_PARTS (more returns NOMAS_ERR_UNSUPPORTED).
 * Errors: NOMAS_ERR_INVALID_ARG, NOMAS_ERR_UNSUPPORTED, NOMAS_ERR_CUDA.
 */
nomas_status nomas_attention_merge(const void *o_parts, const float *lse_parts, int32_t n_parts,
                                   int64_t n_q, void *o, float *lse, int32_t heads,
                                   int32_t head_dim, void *stream);

/*
 * Key-sharded attention whose partial results go straight to their owners
 * ("What 'world memory' stores": the cache spread over eight GPUs, sp_size 8;
 * the routing is this library's design).  This GPU attends with every query
 * row over its own key spans, as nomas_segment_attention does, but each query
 * row's partial O and LSE are stored into part `slot` (this GPU's index) of
 * the buffers of the GPU that owns the row, from the epilogue of the
 * attention kernel, so the exchange runs while other tiles still compute.
 * Each owner then merges its rows from its own buffers with
 * nomas_attention_merge_peers (parts = its R slots, outputs = every GPU's O).
 *   n_owners, owner_row0: owner s owns query rows [owner_row0[s],
 *               owner_row0[s + 1]) (host int64[n_owners + 1], from 0 to n_q,
 *               non-decreasing).
 *   owner_o, owner_lse: host arrays of n_owners device pointers to each
 *               owner's stacked buffers, [R][n_q][heads][head_dim] bf16 and
 *               [R][heads][n_q] fp32, R > slot; only rows the owner owns are
 *               written.  They may be other GPUs' memory mapped into this
 *               process (peer access, CUDA IPC or symmetric memory).
 *   slot      : 0 <= slot < NOMAS_MAX_MERGE_PARTS.
 * The caller orders the owners' merges after every GPU's call (a cross-GPU
 * barrier on the streams).  Other arguments as nomas_segment_attention.
 * Errors: as nomas_segment_attention, plus NOMAS_ERR_INVALID_ARG for bad
 * owner tables or buffers that overlap the inputs.
 */
nomas_status nomas_segment_attention_to_owners(const void *q, int64_t n_q,
                                               const nomas_kv_span *spans, int32_t n_spans,
                                               int32_t n_owners, const int64_t *owner_row0,
                                               void *const *owner_o, float *const *owner_lse,
                                               int32_t slot, float softmax_scale, int32_t heads,
                                               int32_t head_dim, int32_t *dev_err, void *stream);

/*
 * The merge of key-shard partials fused with their exchange between GPUs
 * ("What 'world memory' stores": the cache spread over eight GPUs, sp_size 8;
 * how the partial results meet is not on the page).  Each GPU calls it for
 * the query rows it owns: it reads those rows of every GPU's partial result
 * and writes the merged rows into every listed output, so the partials cross
 * NVLink once, only for the rows the caller merges, and the merged rows are
 * distributed in the same kernel.  The pointers may address other GPUs'
 * memory mapped into this process (peer access, CUDA IPC or symmetric
 * memory); the kernel reads and writes them with plain loads and stores.
 *   o_parts, lse_parts: host arrays of n_parts device pointers; part r is a
 *                       [n_q][heads][head_dim] bf16 partial output and its
 *                       [heads][n_q] fp32 LSE (natural log).
 *   row0, n_rows      : the query rows merged by this call.
 *   o_outs, lse_outs  : host arrays of n_outs device pointers to
 *                       [n_q][heads][head_dim] bf16 outputs and [heads][n_q]
 *                       fp32 LSEs; rows [row0, row0 + n_rows) of each are
 *                       written.  lse_outs may be NULL, or hold NULL entries.
 * 1 <= n_parts <= NOMAS_MAX_MERGE_PARTS, 1 <= n_outs <= NOMAS_MAX_MERGE_OUTPUTS.
 * The caller orders the call after every producer of the partials, on every
 * GPU, and every consumer of the outputs after the calls of all GPUs: for
 * example with a one-element NCCL all-reduce on the same streams before and
 * after.  Outputs must not overlap the partials.
 * Errors: NOMAS_ERR_INVALID_ARG, NOMAS_ERR_UNSUPPORTED, NOMAS_ERR_CUDA.
 */
nomas_status nomas_attention_merge_peers(const void *const *o_parts, const float *const *lse_parts,
                                         int32_t n_parts, int64_t n_q, int64_t row0,
                                         int64_t n_rows, void *const *o_outs,
                                         float *const *lse_outs, int32_t n_outs, int32_t heads,
                                         int32_t head_dim, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NOMAS_H */
