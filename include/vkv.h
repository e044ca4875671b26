/*
 * vkv.h -- chunk attention over a segmented KV cache, native on NVIDIA B200 (sm_100a).
 *
 * The queries of the current latent-frame chunk of an autoregressive video
 * diffusion model attend over a KV cache made of sink frames, history and a
 * local window.  Three cache modes are served by one attention entry point:
 *
 *   VKV_MODE_SEGMENTS      the cache is split into a local branch (sink + current
 *                          frames) and a history branch; each branch emits its own
 *                          partial output and log-sum-exp (LSE), and the two are
 *                          merged exactly by online softmax.
 *                          (ISPA summary, gist.science 2607.00712, section 2 step 1
 *                          "Dual-Stream Warmup": decomposable attention tracked by
 *                          LSE; contribution 2: online softmax.)
 *   VKV_MODE_BLOCK_SPARSE  every query attends to a per-head list of persistent
 *                          blocks plus the top-K blocks of the local window picked
 *                          for its 64-query block, in one softmax.
 *                          (Sparse Forcing summary, gist.science 2604.21221,
 *                          section 2 component 3 "PBSA".)
 *   VKV_MODE_RAGGED        each (batch, head) sequence has its own cache length;
 *                          the caches are stored flattened with boundary offsets,
 *                          without padding.
 *                          (Pyramid Forcing summary, gist.science 2605.13111,
 *                          methodology section 3 "Ragged-Cache Attention".)
 *
 * Conventions for every entry point:
 *   - All tensors are device memory allocated and owned by the caller.  The
 *     library allocates no device memory; it keeps no state between calls
 *     except one-time per-device set-up (kernel attributes, driver entry point).
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream);
 *     the library never synchronises.  Host arrays passed in are read during
 *     the call only.
 *   - bf16 tensors are described by vkv_tensor: a pointer to element 0 and the
 *     element strides of the batch, token and head axes; the feature axis (d)
 *     is contiguous.  Pointers must be 16-byte aligned and the three strides
 *     multiples of 8 elements (the tensor-memory-accelerator rule), else
 *     VKV_ERR_ALIGN.
 *   - The return value reports host-side validation and launch errors.  Errors
 *     found on the device (an index outside the cache, non-monotone offsets, a
 *     pipeline wait that exceeded its time limit) are written to the optional
 *     device word `err_word` (first error wins; 0 = no error) and the affected
 *     work is skipped; nothing traps.  Without `err_word` they go unreported.
 *   - Thread-safe; calls on different streams may run concurrently, provided
 *     their output buffers do not overlap.
 */
#ifndef VKV_H_
#define VKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; NULL selects the legacy default stream. */
typedef struct CUstream_st* vkv_stream_t;

typedef enum {
  VKV_OK = 0,
  VKV_ERR_NULL = 1,        /* a required pointer is NULL                                  */
  VKV_ERR_SHAPE = 2,       /* a size is out of range or two sizes disagree                */
  VKV_ERR_ALIGN = 3,       /* a pointer or stride breaks the 16-byte rule                 */
  VKV_ERR_RANGE = 4,       /* a segment or host offset lies outside the cache             */
  VKV_ERR_UNSUPPORTED = 5, /* valid request outside what this build implements            */
  VKV_ERR_CUDA = 6,        /* no usable sm_100 device, or a CUDA call / launch failed     */
  VKV_ERR_WORKSPACE = 7    /* workspace missing or smaller than the reported size         */
} vkv_status;

/* Codes written to *err_word by the device. */
#define VKV_DEVERR_TIMEOUT 1      /* a pipeline wait ran past its limit; outputs incomplete */
#define VKV_DEVERR_BAD_INDEX 2    /* a block index lies outside the cache or the window     */
#define VKV_DEVERR_BAD_OFFSETS 3  /* cu_seqlens decreasing or past the flattened cache      */

typedef enum {
  VKV_MODE_SEGMENTS = 0,
  VKV_MODE_BLOCK_SPARSE = 1,
  VKV_MODE_RAGGED = 2
} vkv_mode;

/* Cache token rows [start, start + len) of one batch/head. */
typedef struct {
  int32_t start;
  int32_t len;
} vkv_segment;

/* A bf16 tensor [B, L, H, d] with element strides sb, st, sh; d contiguous.
 * For the flattened ragged cache [rows, d] only `ptr` and `st` (row stride) are read. */
typedef struct {
  void* ptr;
  int64_t sb;
  int64_t st;
  int64_t sh;
} vkv_tensor;

#define VKV_MAX_BRANCHES 2
#define VKV_MAX_SEGMENTS 8   /* per branch */

typedef struct {
  int32_t mode;  /* vkv_mode */
  int32_t B;     /* batch                                                     */
  int32_t H;     /* heads (queries and keys have the same head count)         */
  int32_t Lq;    /* query rows per batch and head (the current chunk)         */
  int32_t Lkv;   /* cache rows per batch and head; RAGGED: rows of the flat cache */
  int32_t d;     /* head dimension: 64 or 128                                 */
  float scale;   /* softmax scale applied to q.k (usually 1/sqrt(d))          */
  vkv_tensor q;  /* [B, Lq, H, d]                                             */
  vkv_tensor k;  /* SEGMENTS / BLOCK_SPARSE: [B, Lkv, H, d]; RAGGED: [Lkv, d] */
  vkv_tensor v;  /* same layout as k                                          */

  /* VKV_MODE_SEGMENTS: n_branches in {1, 2}; segs[b] is a HOST array of
   * n_segs[b] <= VKV_MAX_SEGMENTS segments; a branch is the union of its
   * segments (which must not overlap).  A branch may be empty (O = 0, LSE = -inf). */
  int32_t n_branches;
  const vkv_segment* segs[VKV_MAX_BRANCHES];
  int32_t n_segs[VKV_MAX_BRANCHES];

  /* VKV_MODE_BLOCK_SPARSE: the cache is cut into blocks of `block` (= 64) rows.
   * persist_idx: DEVICE int32 [B*H][n_persist], absolute block ids attended by every query.
   * sel_idx:     DEVICE int32 [B*H][ceil(Lq/block)][topk], window-relative block ids
   *              (0 <= id < n_win_blk), distinct within a row, ascending, as written by
   *              vkv_block_select; query block j = query rows [j*block, (j+1)*block).
   * The window is blocks [window_blk0, window_blk0 + n_win_blk); persistent blocks
   * must lie outside it.  Requires n_persist + min(n_win_blk, 4*topk) <= 288
   * (one unit holds up to four query blocks; its block list has at most 288 entries). */
  int32_t block;
  const int32_t* persist_idx;
  int32_t n_persist;
  const int32_t* sel_idx;
  int32_t topk;
  int32_t window_blk0;
  int32_t n_win_blk;

  /* VKV_MODE_RAGGED: sequence s = b*H + h reads flat rows [cu[s], cu[s+1]).
   * cu_seqlens: DEVICE int32 [B*H + 1] (authoritative, checked on the device).
   * cu_seqlens_host: optional HOST copy; when given it is validated on the host and
   * used to balance work across SMs (longest sequences first). */
  const int32_t* cu_seqlens;
  const int32_t* cu_seqlens_host;

  /* Outputs.  o[b] bf16 [B, Lq, H, d] and lse[b] fp32 [B, H, Lq] (contiguous) per
   * branch; BLOCK_SPARSE and RAGGED write branch 0 only.  o_merged / lse_merged
   * (SEGMENTS with 2 branches, optional: ptr NULL = skip) receive the exact
   * LSE merge of the two branches, i.e. attention over their union.
   * LSE is the natural log of sum_j exp(scale * q.k_j). */
  vkv_tensor o[VKV_MAX_BRANCHES];
  float* lse[VKV_MAX_BRANCHES];
  vkv_tensor o_merged;
  float* lse_merged;

  int32_t* err_word; /* optional DEVICE int32; see VKV_DEVERR_* */

  /* VKV_MODE_BLOCK_SPARSE, optional (NULL = natural order): DEVICE int32
   * [B*H][ceil(Lq/block)], for each (b, h) a permutation of its query blocks.
   * Work is cut into units of four consecutive entries (two 128-row tiles of
   * two query blocks each) and a unit streams the union of its query blocks'
   * selections, so an order that puts query blocks with similar selections
   * side by side (vkv_block_select's out_order) shrinks the work.  Results do
   * not depend on the order beyond rounding.  An entry outside
   * [0, ceil(Lq/block)) raises VKV_DEVERR_BAD_INDEX; a repeated entry leaves
   * some query block unwritten (not checked). */
  const int32_t* qblk_order;

  /* Optional DEVICE scratch for key-axis splitting (SEGMENTS, BLOCK_SPARSE, and
   * RAGGED with cu_seqlens_host).  NULL: every unit of work is one or two whole query tiles
   * over all of its keys, and the schedule balances whole units over the SMs.
   * Otherwise at least vkv_chunk_attn_workspace_size() bytes, 256-byte aligned,
   * owned by the caller (VKV_ERR_WORKSPACE when smaller): the schedule may then
   * cut some units into pieces over disjoint key ranges that run on different
   * SMs; each piece leaves its partial output and LSE in the workspace, and a
   * small kernel that the call launches behind the attention kernel combines
   * each unit's pieces exactly (the same LSE merge as the two branches) and
   * writes the outputs.  (BLOCK_SPARSE units learn their key count on the
   * device: their pieces are cut as fractions of it.)  Results equal those of an
   * unsplit run up to fp32 rounding.  Its contents need no initialisation (the
   * call marks the partial LSEs on `stream` first) and are dead after the call;
   * calls that overlap on the GPU must not share one. */
  void* workspace;
  size_t workspace_bytes;

  /* VKV_MODE_BLOCK_SPARSE, optional: select the window blocks inside the attention
   * kernel (Sparse Forcing summary, section 2 components 2 and 3: coarse scores
   * of the query-block means against one representative per window block, top-K
   * per query block).  When kbar is not NULL, sel_idx is not read: the kernel
   * pools each unit's query blocks, scores them against kbar and keeps the top
   * `topk` window blocks of each, exactly as vkv_block_select does from the same
   * cached means (the same indices, bit for bit), while the unit's persistent
   * blocks are already being attended.
   * kbar:    DEVICE fp32 [B*H][n_win_blk][d], 16-byte aligned: the window block
   *          means (vkv_block_pool), kept by the caller as blocks enter the cache.
   * sel_out: optional DEVICE int32 [B*H][ceil(Lq/block)][topk]: receives the
   *          selection (ascending ids, as vkv_block_select's out_idx), e.g. to
   *          derive a query-block order for a later call.
   * Requires 1 <= topk <= n_win_blk <= 512 (else VKV_ERR_SHAPE).  Units are not
   * split along the key axis in this form (workspace is ignored); a unit of one
   * 128-row query tile instead splits its key tiles between two accumulators
   * that are merged by their LSEs, so its output rows may differ from those of
   * the attention from sel_idx in the last bits (both are the same softmax
   * attention over the same key set). */
  const float* kbar;
  int32_t* sel_out;
} vkv_attn_args;

/*
 * vkv_chunk_attn -- softmax attention of the chunk's queries over the cache.
 *
 * For each (batch b, head h, query row i) and the key set J selected by the mode:
 *   s_j = scale * <q_i, k_j>,  O_i = sum_j softmax(s)_j v_j,  LSE_i = ln sum_j exp(s_j).
 * Rows of the cache up to 127 past the end of a segment (SEGMENTS, RAGGED) are
 * read but masked; where they lie inside the cache they must hold finite values.
 * Limits: B*H < 2^18 and Lq <= 4096 * 128 (else VKV_ERR_UNSUPPORTED).
 * Sources: ISPA summary section 2 step 1; Sparse Forcing summary section 2
 * component 3; Pyramid Forcing summary methodology section 3.
 */
vkv_status vkv_chunk_attn(const vkv_attn_args* args, vkv_stream_t stream);

/*
 * Bytes of `workspace` that vkv_chunk_attn can use for these arguments (0 when
 * its schedule does not split any unit; always 0 for RAGGED without
 * cu_seqlens_host).  Reads only the host-side fields (mode, shapes, segments,
 * cu_seqlens_host, the block-sparse counts and whether qblk_order is NULL);
 * returns 0 for arguments that
 * vkv_chunk_attn would refuse.  The size depends on the shapes and on the
 * number of SMs of the current device.
 */
size_t vkv_chunk_attn_workspace_size(const vkv_attn_args* args);

/*
 * vkv_debug_schedule -- test aid (host only, no device needed): the work
 * schedule vkv_chunk_attn would run for `args` on a device with `n_sm` SMs
 * (1..160), with key-axis splitting allowed when `split` is non-zero.  Reads
 * the same host-side fields as vkv_chunk_attn_workspace_size.  Output arrays
 * are HOST and caller-owned (NULL = skip): cta_begin / cta_piece0 [n_sm + 1],
 * units [6144], pieces [2 * 384] (uint32 pairs).  Unit code: bits [0, 12)
 * first 128-row query tile, bit 12 piece, bit 13 two tiles, bits [14, 32)
 * sequence b*H + h.  Piece pair: first word = first key step | end step << 16,
 * second = first workspace slot of its unit | piece index << 16 | piece
 * count << 24; the pieces of CTA c start at cta_piece0[c], in unit order.
 */
typedef struct {
  int32_t n_ctas, n_units, n_pieces, n_slots;
  int32_t* cta_begin;
  int32_t* cta_piece0;
  uint32_t* units;
  uint32_t* pieces;
} vkv_schedule;
vkv_status vkv_debug_schedule(const vkv_attn_args* args, int32_t n_sm, int32_t split, vkv_schedule* out);

/*
 * Block selection for VKV_MODE_BLOCK_SPARSE (Sparse Forcing summary, section 2
 * component 2 "Blockified Compression": one representative token per block for
 * coarse scoring; component 3: top-K window blocks).
 *
 * Each query block j (rows [j*block, (j+1)*block) of q, the last one possibly
 * shorter) and each window block w (cache rows [(window_blk0+w)*block, +block))
 * is reduced to the fp32 mean of its rows; score(j, w) = <qbar_j, kbar_w>
 * (no softmax scale: a positive factor does not change the ranking).  For every
 * (batch, head, j) the `topk` highest-scoring window blocks are written to
 * out_idx [B*H][ceil(Lq/block)][topk] in ascending order; equal scores rank
 * the lower block id first.  out_scores [B*H][ceil(Lq/block)][n_win_blk]
 * (optional, fp32) receives every score.
 * `workspace` is DEVICE scratch of at least vkv_block_select_workspace_size()
 * bytes (the window blocks' means: B*H*n_win_blk*d*4, rounded up to 256),
 * 256-byte aligned, owned by the caller; its contents need no initialisation
 * and are dead after the call.  It is not used, and may be NULL, when `kbar`
 * supplies the window means (the query blocks are pooled on chip).
 */
typedef struct {
  int32_t B, H, d, block; /* d in {64, 128}; block = 64                       */
  int32_t Lq;             /* query rows                                        */
  int32_t Lkv;            /* cache rows (window blocks must lie inside)        */
  int32_t window_blk0;    /* first window block                                */
  int32_t n_win_blk;      /* window blocks, 1..1024                            */
  int32_t topk;           /* 1..n_win_blk                                      */
  vkv_tensor q;           /* [B, Lq, H, d]                                     */
  vkv_tensor k;           /* [B, Lkv, H, d]                                    */
  int32_t* out_idx;
  float* out_scores;
  void* workspace;
  size_t workspace_bytes;
  int32_t* err_word;      /* optional DEVICE int32                             */
  /* optional DEVICE int32 [B*H][ceil(Lq/block)] (NULL = skip): for each (b, h)
   * a permutation of its query blocks, sorted by their selections (ascending
   * lexicographic order of the first six selected ids, then by block index),
   * so that query blocks with similar selections are adjacent; pass it to
   * vkv_chunk_attn as qblk_order.  Not part of the pages' method: it only
   * groups work. */
  int32_t* out_order;
  /* optional DEVICE fp32 [B*H][n_win_blk][d] (NULL = pool from k): the window
   * blocks' means as written by vkv_block_pool for blocks [window_blk0,
   * window_blk0 + n_win_blk), kept by the caller as blocks enter the cache
   * (Sparse Forcing summary, section 2 component 2: one representative per
   * block).  Then only the query blocks are pooled and `k` is not read. */
  const float* kbar;
} vkv_select_args;

size_t vkv_block_select_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_win_blk,
                                       int32_t block, int32_t d);
vkv_status vkv_block_select(const vkv_select_args* args, vkv_stream_t stream);

/*
 * vkv_block_order -- the query-block order of vkv_block_select's out_order,
 * from a selection the caller already holds (for instance the sel_out of a
 * vkv_chunk_attn call that selected inside the attention kernel), to pass as
 * a later call's qblk_order.  A work-grouping aid, not part of the pages'
 * method.
 *   sel_idx:   DEVICE int32 [BH][n_qblk][topk], each row's window block ids
 *              ascending, each below 1024 (as the selection writes them);
 *   out_order: DEVICE int32 [BH][n_qblk]: for each of the BH sequences a
 *              permutation of its query blocks, ascending lexicographic order
 *              of the first six selected ids, then by block index.
 * Requires BH >= 1, 1 <= n_qblk <= 4096 and topk >= 1 (VKV_ERR_SHAPE /
 * VKV_ERR_UNSUPPORTED otherwise).  Asynchronous on `stream`, after the work
 * queued before it.
 */
vkv_status vkv_block_order(const int32_t* sel_idx, int32_t* out_order, int32_t BH, int32_t n_qblk,
                           int32_t topk, vkv_stream_t stream);

/*
 * vkv_block_pool -- the representative (fp32 mean of the rows) of each of the
 * 64-row blocks [blk0, blk0 + n_blk) of x [B, L, H, d] (Sparse Forcing summary,
 * section 2 component 2), written to out [B*H][n_blk][d] (DEVICE fp32, caller
 * owned).  The same arithmetic as vkv_block_select's own pooling, so a
 * selection from cached representatives equals one that pools them itself.
 */
vkv_status vkv_block_pool(vkv_tensor x, int32_t B, int32_t L, int32_t H, int32_t d, int32_t blk0,
                          int32_t n_blk, float* out, vkv_stream_t stream);

/*
 * vkv_block_select_noalloc -- vkv_block_select for callers that cannot allocate.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory when they call in (for example a
 * serving loop whose device memory is fully planned at start-up and that
 * gives the library no allocator, or a host program that drives the library
 * through this C interface alone and cannot size and own a workspace).
 *
 * Same arguments, results and errors as vkv_block_select, except that
 * `workspace` / `workspace_bytes` are ignored: the pooled window block vectors
 * go to a fixed scratch array inside the library, VKV_NOALLOC_SCRATCH_BYTES in
 * size, which every GPU that loads the library holds until the process exits.
 * Requests whose vkv_block_select_workspace_size() exceeds that size return
 * VKV_ERR_WORKSPACE; calls that pass cached window means in `kbar` use no
 * scratch and are never refused for size.  The call allocates nothing (no
 * cudaMalloc / cudaFree).  The first call on a device looks up the array's
 * device address on that device (cudaGetSymbolAddress) and keeps it; make that
 * first call before any stream capture, and do not call this entry point again
 * after a cudaDeviceReset of that device in the same process (the kept address
 * belongs to the context that was reset).  All calls on a device share the
 * array and leave the last call's contents in it; calls that overlap on the
 * GPU (e.g. on two streams at once) race on it.  Nothing in it needs clearing
 * between calls.
 */
#define VKV_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)
vkv_status vkv_block_select_noalloc(const vkv_select_args* args, vkv_stream_t stream);

/*
 * vkv_persist_update -- persistent-memory management (Sparse Forcing summary,
 * section 2 component 1 "Structured Memory Decomposition": the blocks evicted
 * from the local window are candidates, and the top C by coarse score are
 * kept in, or replace blocks of, the persistent memory).
 *
 * Per (batch b, head h): the candidates are the current persistent blocks
 * persist_idx[b*H+h][0..C) and the evicted blocks [evict_blk0, evict_blk0 +
 * n_evict); each is scored by <qbar, kbar_c>, where qbar is the mean of the
 * chunk's Lq query rows and kbar_c the mean of block c's rows (no softmax
 * scale: a positive factor does not change the ranking).  The C highest
 * scores are kept (equal scores: the lower block id first) and written to
 * out_idx [B*H][C] in ascending block order.  out_scores (optional, fp32
 * [B*H][C + n_evict]) receives the candidates' scores, persistent ones first.
 * A persistent id outside [0, Lkv/block) or inside the evicted range raises
 * VKV_DEVERR_BAD_INDEX (that candidate is dropped).
 */
typedef struct {
  int32_t B, H, d, block;    /* d in {64, 128}; block = 64                         */
  int32_t Lq, Lkv;           /* query rows; cache rows                             */
  vkv_tensor q;              /* [B, Lq, H, d]                                      */
  vkv_tensor k;              /* [B, Lkv, H, d]                                     */
  const int32_t* persist_idx;/* DEVICE int32 [B*H][n_persist], absolute block ids  */
  int32_t n_persist;         /* C, 1..1024                                         */
  int32_t evict_blk0;        /* first evicted block                                */
  int32_t n_evict;           /* evicted blocks, 0..1024 (C + n_evict <= 2048)      */
  int32_t* out_idx;          /* DEVICE int32 [B*H][n_persist]                      */
  float* out_scores;         /* optional DEVICE fp32 [B*H][n_persist + n_evict]    */
  void* workspace;           /* DEVICE, >= vkv_persist_update_workspace_size(), 256-byte aligned */
  size_t workspace_bytes;
  int32_t* err_word;         /* optional DEVICE int32                              */
} vkv_persist_args;

size_t vkv_persist_update_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_persist,
                                         int32_t n_evict, int32_t block, int32_t d);
vkv_status vkv_persist_update(const vkv_persist_args* args, vkv_stream_t stream);

/*
 * Head-aware cache compaction (Pyramid Forcing summary, methodology section 2
 * "head-aware pyramid KV cache policies" and section 3 "flattened sequences
 * with boundary indices"): every (batch, head) keeps its own subset of the
 * frames of a dense cache, and the kept frames of all heads are packed into
 * one flattened ragged cache with boundary offsets, in one launch.
 *
 * Source frames: 0 .. hist_frames-1 are history (frame 0 is the sink), then
 * cur_frames frames of the current chunk; frame f is cache rows
 * [f*frame_tokens, (f+1)*frame_tokens).  Every head keeps, in this order:
 * the sink, its policy's middle frames (chosen from [1, hist_frames -
 * recent_frames - 1]), the last recent_frames history frames, and the current
 * frames.  Middle frames by policy:
 *   FULL    every middle frame;
 *   ANCHOR  `param` frames evenly spaced over the middle range, both ends
 *           included (frame lo + floor(i * (hi - lo) / (param - 1)));
 *   WAVE    middle frames f with (hist_frames - f) % param == 0 (period
 *           `param`, aligned to the current chunk);
 *   VEIL    the last `param` (even) middle frames, merged in adjacent pairs:
 *           a pair is stored once, as the fp32 mean of its two bf16 frames
 *           rounded to nearest-even bf16.
 */
typedef enum {
  VKV_HEAD_FULL = 0,
  VKV_HEAD_ANCHOR = 1,
  VKV_HEAD_WAVE = 2,
  VKV_HEAD_VEIL = 3
} vkv_head_policy;

typedef struct {
  int32_t policy; /* vkv_head_policy */
  int32_t param;  /* ANCHOR: frames kept (1..middle); WAVE: period >= 1; VEIL: frames merged (even, <= middle) */
} vkv_head_rule;

#define VKV_COMPACT_MAX_SEQS 512      /* B*H */
#define VKV_COMPACT_MAX_PIECES 1024   /* stored frames (or merged pairs) over all sequences */

typedef struct {
  int32_t B, H, d;          /* d in {64, 128}                                        */
  int32_t frame_tokens;     /* rows per frame                                         */
  int32_t hist_frames;      /* history frames (>= 1 + recent_frames)                  */
  int32_t cur_frames;       /* current-chunk frames after the history (>= 0)          */
  int32_t recent_frames;    /* history frames every head keeps before the chunk (>= 0) */
  vkv_tensor k_src;         /* [B, (hist_frames + cur_frames) * frame_tokens, H, d]   */
  vkv_tensor v_src;         /* same layout as k_src                                   */
  const vkv_head_rule* rules; /* HOST [H]: the rule of head h (same for every batch)  */
  void* k_out;              /* DEVICE bf16 [rows, d], rows contiguous, sequence s = b*H + h at rows [cu[s], cu[s+1]) */
  void* v_out;              /* same                                                   */
  int64_t out_rows;         /* capacity of k_out / v_out in rows                      */
  int32_t* cu_seqlens;      /* DEVICE int32 [B*H + 1], written by the launch          */
  int32_t* cu_seqlens_host; /* optional HOST int32 [B*H + 1], filled before the call returns */
} vkv_compact_args;

/* Rows the compacted cache needs (>= 0), or -(vkv_status) for invalid arguments.
 * Reads only the sizes and `rules`; no device work. */
int64_t vkv_compact_rows(const vkv_compact_args* args);

/* Writes k_out, v_out and cu_seqlens on `stream` (one kernel launch).  Returns
 * VKV_ERR_RANGE when out_rows is too small, VKV_ERR_UNSUPPORTED beyond
 * VKV_COMPACT_MAX_SEQS sequences or VKV_COMPACT_MAX_PIECES stored frames. */
vkv_status vkv_compact_cache(const vkv_compact_args* args, vkv_stream_t stream);

/*
 * vkv_lse_merge -- exact recombination of two partial attentions over disjoint
 * key sets (ISPA summary, section 2 step 1 and contribution 2):
 *   M = max(lse_a, lse_b),  w_x = exp(lse_x - M),
 *   O = (w_a O_a + w_b O_b) / (w_a + w_b),  LSE = M + ln(w_a + w_b).
 * Rows where both LSEs are -inf give O = 0 and LSE = -inf.
 * o_a, o_b, o_out: bf16 [B, Lq, H, d] (vkv_tensor strides); lse_*: fp32 [B, H, Lq]
 * contiguous.  o_out may alias o_a or o_b only if it is the same tensor exactly.
 */
vkv_status vkv_lse_merge(vkv_tensor o_a, const float* lse_a, vkv_tensor o_b, const float* lse_b,
                         vkv_tensor o_out, float* lse_out, int32_t B, int32_t H, int32_t Lq,
                         int32_t d, vkv_stream_t stream);

/*
 * vkv_latent_attn -- latent (multi-head latent) attention over a head-shared
 * cache (VideoMLA technical summary, "Methodology": each cached token keeps one
 * content latent c_t of width d_c and one rotary key k^R_t of width d_rope,
 * shared by all heads; each head rebuilds its keys and values from them with
 * its own up-projections).  With the key up-projection absorbed into the query
 * (qa_h = [(W^K_h)^T q^nope_h ; q^R_h]) and the value up-projection left to
 * the output projection, for each (batch b, head h, query row i):
 *   s_t = scale * <qa_{b,i,h}, [c_{b,t} ; k^R_{b,t}]>,
 *   o_{b,i,h} = sum_t softmax(s)_t c_{b,t}     (latent output, width d_c),
 *   LSE_{b,h,i} = ln sum_t exp(s_t).
 * Every head reads the same cache rows.  No position math happens here: q and
 * k^R arrive rotated.  An empty cache (Lkv = 0) gives o = 0 and LSE = -inf.
 */
typedef struct {
  int32_t B, H, Lq, Lkv; /* B, H, Lq >= 1; Lkv >= 0                                 */
  int32_t d_c;     /* latent width: 128 or 192                                     */
  int32_t d_rope;  /* rotary key width: 32                                         */
  float scale;     /* softmax scale, > 0                                           */
  vkv_tensor q;    /* [B, Lq, H, d_c + d_rope]: absorbed, rotated queries          */
  vkv_tensor kv;   /* [B, Lkv, d_c (+ d_rope)]: cached rows [c ; k^R]; sb, st read, sh ignored;
                      may be NULL when Lkv = 0                                     */
  vkv_tensor kr;   /* optional [B, Lkv, d_rope] rotary keys stored apart (sb, st read);
                      ptr NULL = columns [d_c, d_c + d_rope) of kv                */
  vkv_tensor o;    /* [B, Lq, H, d_c] bf16 latent output                           */
  float* lse;      /* optional fp32 [B, H, Lq] contiguous (NULL = skip)            */
  int32_t* err_word; /* optional DEVICE int32; a pipeline timeout sets VKV_DEVERR_TIMEOUT */
} vkv_latent_args;

vkv_status vkv_latent_attn(const vkv_latent_args* args, vkv_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char* vkv_status_string(vkv_status s);

/* Library version as major*10000 + minor*100 + patch. */
int32_t vkv_version(void);

/* sizeof() of the ABI structs, for bindings to check their layout:
 * 0 vkv_attn_args, 1 vkv_select_args, 2 vkv_tensor, 3 vkv_segment,
 * 4 vkv_compact_args, 5 vkv_head_rule, 6 vkv_persist_args, 7 vkv_latent_args,
 * 8 vkv_schedule; -1 otherwise. */
int32_t vkv_abi_sizeof(int32_t which);

#ifdef __cplusplus
}
#endif

#endif /* VKV_H_ */
