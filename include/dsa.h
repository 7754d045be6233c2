/*
 * dsa.h -- C ABI of libdsa: DeepSeek Sparse Attention (DSA) decode on B200.
 *
 * What the library computes (pages cited by title and section):
 *   "大语言模型结构总览" (LLM structure overview), section 2.2 DeepSeek-V3.2:
 *     DSA is a two-stage select-then-attend pipeline.  A lightning indexer
 *     (64 heads, head dim 128, FP8) scores every prior token of a query; a
 *     token selector keeps the k = 2048 best tokens; MLA attention in MQA mode
 *     then runs over those tokens only.  Paged and non-paged forms exist.
 *   Same page, section 2.1 DeepSeek-V3: one cached latent per token, kv rank
 *     512 plus a 64-d RoPE part (576 values), 128 attention heads.
 *   Same page, section 7.2 GLM-5.2 / Figure 7-2: IndexShare -- one indexer per
 *     group of sparse layers; the following layers reuse its top-k indices.
 *     The same section gives GLM-5.2's shapes: 64 MLA heads (qk head dim
 *     192 + 64 RoPE, kv rank 512) and a 32-head FP8 indexer of head dim 128,
 *     top-2048 causal keys.  Absorbed into MQA form its cached latent is the
 *     same 576-value row (512 kv rank + 64 RoPE), so the calls below take
 *     the head counts as arguments: heads = 128 or 64, idx_heads = 64 or 32
 *     (any other value returns DSA_ERR_UNSUPPORTED).
 *   "GLM-5.2 推理部署" (inference deployment), MTP draft + verify flow: top-K
 *     = 2048 indices computed once and reused across the MTP positions.
 *
 * Definitions used throughout (readings where the pages give no formula):
 *   indexer score   I[q,s] = sum_{h<HI} w[q,h] * max(0, sum_{d<128} qi[q,h,d]*K[s,d])
 *                   with HI = idx_heads indexer heads;
 *                   qi and K are FP8 e4m3 bytes at scale 1, w is fp32;
 *   selector        the topk positions s < vis[q] with the largest I[q,s],
 *                   ties to the lower s; if vis[q] < topk every visible s is
 *                   kept and the remaining slots hold -1;
 *   sparse MLA      per head h < heads:  z_j = scale * <q[h,0:576], C[idx_j,0:576]>,
 *                   O[h] = sum_j softmax_j(z) * C[idx_j,0:512],
 *                   LSE[h] = ln sum_j exp(z_j)  (empty set: O = 0, LSE = -inf);
 *   split-K         the selected set is partitioned into num_splits parts, each
 *                   attended separately, then merged exactly by LSE.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or torch-owned)
 *     unless a parameter says "host".  The caller allocates and owns every
 *     buffer, including the workspace; the library allocates nothing and
 *     keeps no per-call state (it caches TMA descriptors and the SM count).
 *   - Calls are asynchronous: work is enqueued on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream) and the caller synchronises.
 *   - Argument checks run on the host before anything is enqueued; a failed
 *     check returns DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED and enqueues
 *     nothing.  Nothing traps and nothing throws across the ABI.
 *   - Values the host cannot check (indices, page ids, lengths living in
 *     device memory) are checked by the kernels: an out-of-range entry is
 *     treated as masked and raises a flag in the workspace that
 *     dsa_check_error() reports as DSA_ERR_DEVICE_BOUNDS.  Device-side waits
 *     are bounded; an expired wait raises DSA_ERR_TIMEOUT the same way.
 *   - Layouts are dense row-major with the shapes given; `e4m3` is one byte
 *     per value (OCP FP8 E4M3), `bf16` two bytes.  Pointers must be 16-byte
 *     aligned.
 *   - Query/sequence bookkeeping: the queries of sequence b are the
 *     contiguous rows q_offsets[b] .. q_offsets[b+1]-1 (at most
 *     DSA_MAX_Q_PER_SEQ of them); the indexer keys of sequence b are rows
 *     seq_offsets[b] .. seq_offsets[b+1]-1 of the packed key array, token
 *     position s of b at row seq_offsets[b] + s.  vis[q] = number of keys
 *     query q may see (positions 0 .. vis[q]-1, causal).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_PAGE_SIZE 64        /* latent-cache page (tokens) of the built-in workloads */
#define DSA_TIER_PAGE 16        /* tokens per slot of the two-tier (HiSparse) cache */
#define DSA_HEADS 128           /* MLA query heads (DeepSeek-V3.2) */
#define DSA_HEADS_GLM 64        /* MLA query heads (GLM-5.2) */
#define DSA_DIM 576             /* latent row: 512 kv-rank + 64 RoPE */
#define DSA_DIM_V 512           /* value dims (first 512 of the row) */
#define DSA_IDX_HEADS 64        /* indexer heads (DeepSeek-V3.2) */
#define DSA_IDX_HEADS_GLM 32    /* indexer heads (GLM-5.2) */
#define DSA_IDX_DIM 128         /* indexer head dim */
#define DSA_MAX_TOPK 2048
#define DSA_MAX_Q_PER_SEQ 8     /* 1 decode token + up to 7 MTP drafts */
#define DSA_MAX_BATCH 2048      /* sequences per call */
#define DSA_MAX_SPLITS 32

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
  DSA_ERR_UNSUPPORTED = 2,   /* shape outside the fixed constants above */
  DSA_ERR_CUDA = 3,          /* a CUDA runtime call failed */
  DSA_ERR_DEVICE_BOUNDS = 4, /* a kernel met an out-of-range index/page/length */
  DSA_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired */
  DSA_ERR_WORKSPACE = 6      /* workspace smaller than dsa_workspace_bytes() */
} dsa_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* dsa_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
int dsa_version(void);

/*
 * Bytes of device workspace the calls below need for Q queries, contexts of at
 * most max_len keys, `topk` selected tokens and `num_splits` split-K parts
 * (0 = let the library choose).  The workspace holds the fp32 score rows
 * [Q, max_len], the split-K partial outputs (sized for 128 heads, so one
 * workspace serves both head counts; Q x splits of them plus one per SM pair,
 * which dsa_decode_step uses to split the last, partial wave of the grouped
 * IndexShare attention), the fused selector's per-query
 * first-digit histograms, counters and threshold-bin candidate lists (which
 * dsa_indexer_topk_fused clears itself) and the device error flag.  The same workspace may be
 * reused by consecutive calls on one stream; it must be zeroed once
 * (cudaMemset) before its first use so the error flag starts clear.
 * Returns 0 for invalid sizes.
 */
size_t dsa_workspace_bytes(int Q, int max_len, int topk, int num_splits);

/*
 * Split-K parts the sparse MLA calls use for Q queries and `topk` selected
 * tokens: num_splits itself when it is 1..DSA_MAX_SPLITS (capped at topk),
 * the library's choice for 0 (the fewest parts whose (query, part) units,
 * each on a pair of SMs, fill the GPU's SM pairs to at least 85% over whole
 * waves, with at least 64 tokens a part).  With more than one part the call
 * also runs the LSE merge.  Returns 0 for invalid sizes.  Host only.
 */
int dsa_choose_splits(int Q, int topk, int num_splits);

/*
 * How dsa_decode_step runs the grouped attention of an IndexShare group of
 * `units` (layer, query) pairs with one split each, every unit on a pair of
 * SMs: when the units leave a last wave that fills at most half of the GPU's
 * 74 SM pairs, those tail units run as a second grid cut into *tail_splits
 * parts (merged by log-sum-exp) and the first *head_units run whole.
 * Without such a tail: *head_units = units, *tail_units = 0, *tail_splits = 1.
 * Returns 1, or 0 (outputs untouched) for invalid sizes or null pointers.
 * Host only; for callers that size or schedule around the step.
 */
int dsa_mla_group_plan(int units, int topk, int* head_units, int* tail_units, int* tail_splits);

/*
 * Lightning indexer, scores only  (section 2.2: the indexer stage).
 *   q_idx  e4m3 [Q,idx_heads,128]   w [Q,idx_heads] fp32   k_idx e4m3 [total_keys,128]
 *   idx_heads  64 (DeepSeek-V3.2) or 32 (GLM-5.2)
 *   seq_offsets int64 [B+1], q_offsets int32 [B+1], q_vis int32 [Q] (device)
 *   scores fp32 [Q, ld_scores]: row q gets I[q,s] for s < q_vis[q]; other
 *          entries are left untouched.  ld_scores >= max_len, multiple of 4.
 *   first_only != 0: only the first query of each sequence is scored.
 * The FP8 products accumulate in fp32 on the tensor cores.
 */
dsa_status dsa_indexer_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                              int64_t total_keys, const int64_t* seq_offsets,
                              const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                              int idx_heads, int max_len, int first_only, float* scores,
                              int ld_scores, void* ws, size_t ws_bytes, void* stream);

/*
 * Token selector on given scores  (section 2.2: the token selector stage).
 *   scores fp32 [Q, ld_scores] (row q, entries s < q_vis[q] are read)
 *   out_idx int32 [Q, topk]: the selected positions of each query in
 *           unspecified order, then -1 padding when q_vis[q] < topk.
 *   out_scores fp32 [Q, topk] or NULL: the score of each selected position
 *           (-inf in padding slots).
 *   first_only != 0: only the first query of each sequence (rows
 *           q_offsets[b]) is selected; other rows are untouched.
 * Exact: the set equals a full sort by (score desc, position asc); -0 == +0.
 * Scores must not be NaN.  ws: at least 256 bytes (only the error flag at its
 * start is used; any workspace from dsa_workspace_bytes qualifies).
 */
dsa_status dsa_topk_select(const float* scores, int ld_scores, const int32_t* q_offsets,
                           const int32_t* q_vis, int B, int Q, int max_len, int topk,
                           int first_only, int32_t* out_idx, float* out_scores,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Indexer + selector in one call  (section 2.2, both stages).  Arguments as
 * above; scores live in the workspace (dsa_workspace_bytes(Q, max_len, topk, 1)
 * bytes at least).  With first_only != 0 (IndexShare on
 * MTP) the first query of each sequence is scored and selected and its index
 * row is copied to every other query of the sequence.
 */
dsa_status dsa_indexer_topk(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                            int64_t total_keys, const int64_t* seq_offsets,
                            const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                            int idx_heads, int max_len, int topk, int first_only,
                            int32_t* out_idx, float* out_scores, void* ws, size_t ws_bytes,
                            void* stream);

/*
 * The same call with the indexer and the selector fused through histograms:
 * the indexer also counts, per query, the first 12-bit radix digit of every
 * score it writes (warp-aggregated atomics), so the selector knows the
 * threshold digit at launch, reads each score row once and resolves the
 * threshold bin from a candidate list.  Same arguments, workspace and result
 * (the same index sets) as dsa_indexer_topk; the call clears its histograms
 * and counters in the workspace before the indexer.  A histogram that
 * disagrees with its row raises DSA_ERR_DEVICE_BOUNDS.  On B200 it measured
 * slower than dsa_indexer_topk for batch-32 decode at 128K (134.8 against
 * 123.6 us: the histogram adds land in the indexer's epilogue, which bounds
 * it) and slightly faster for 4 sequences at 1M (130.9 against 133.6 us), so
 * the decode step uses the two-kernel form.
 */
dsa_status dsa_indexer_topk_fused(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                                  int64_t total_keys, const int64_t* seq_offsets,
                                  const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                                  int idx_heads, int max_len, int topk, int first_only,
                                  int32_t* out_idx, float* out_scores, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * Sparse MLA decode in absorbed-MQA form over the selected tokens
 * (section 2.2: MLA in MQA mode; section 2.1: 576-d latent, 128 heads;
 * section 7.2: GLM-5.2's 64 heads).
 *   q          bf16 [Q,heads,576]  absorbed queries (512 latent + 64 RoPE)
 *   heads      128 (DeepSeek-V3.2) or 64 (GLM-5.2); 64 heads run on the same
 *              128-row tensor-core tiles with the upper rows unused
 *   kv_pool    bf16 [num_pages,page_size,576]  paged latent cache shared by all heads
 *   page_size  tokens per page: a power of two from 1 to 1024 with
 *              num_pages*page_size < 2^31 (64 for the built-in workloads; 16,
 *              DSA_TIER_PAGE, for a device buffer of the two-tier cache below)
 *   page_table int32 [B,max_pages]: page of token s of sequence b is
 *              page_table[b*max_pages + s/page_size], row s%page_size in that
 *              page.  A non-paged cache is the identity table.
 *   idx        int32 [Q,topk]: token positions (any order), -1 = skip.
 *   scale      softmax scale applied to the 576-d dot product.
 *   num_splits split-K parts (1..DSA_MAX_SPLITS, 0 = library's choice); the
 *              idx row is cut into equal-count parts merged exactly by LSE.
 *   out        fp32 [Q,heads,512]    lse fp32 [Q,heads] (natural log)
 * Entries with idx >= q_vis[q], a page id outside [0,num_pages) or a page
 * slot beyond max_pages are skipped and flagged (DSA_ERR_DEVICE_BOUNDS).
 * Precision: bf16 products accumulate in fp32 on the tensor cores.  Each
 * score is the sum of two partial dot products (latent dims split between a
 * pair of SMs); each partial crosses between them as 16-bit integer codes
 * with one fp32 scale per 32 values (error at most 1/65520 of the block's
 * largest magnitude), which moves O by well under 1e-3 of its RMS.  The value
 * product takes P as fp16 (11 significant bits, relative to a running
 * maximum) and the 512 value dims as fp16, rewritten on chip from bf16:
 * exact for magnitudes 2^-14 .. 65504, rounded to fp16's spacing 2^-24 below.
 * Latent values of magnitude 65536 or more do not fit fp16 and are not
 * flagged: the call takes latents inside fp16's range.
 * ws: at least dsa_workspace_bytes(Q, 1, topk, num_splits) bytes.
 */
dsa_status dsa_sparse_mla_decode(const void* q, const void* kv_pool, int num_pages, int page_size,
                                 const int32_t* page_table, int max_pages,
                                 const int32_t* q_offsets, const int32_t* q_vis,
                                 const int32_t* idx, int B, int Q, int heads, int topk,
                                 float scale, int num_splits, float* out, float* lse,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse MLA decode with a sliding window, DeepSeek-V4's CSA  ("大语言模型结构
 * 总览", section 2.3 DeepSeek-V4: the KV cache is compressed 4x along the
 * sequence, DSA keeps the top-1024 (Pro) or top-512 (Flash) compressed
 * entries, and a 128-token sliding window of raw tokens is attended as well).
 * Each query attends, in one softmax, to
 *   the topk selected entries of idx: positions in the compressed cache,
 *     mapped through page_table and checked against q_vis as above, and
 *   the `window` most recent raw tokens: positions win_vis[q]-window ..
 *     win_vis[q]-1 (those below 0 are skipped), mapped through win_page_table
 *     [B,win_max_pages] into the same kv_pool.
 *   win_vis  DEVICE int32 [Q]: raw tokens visible to each query
 *   topk + window <= DSA_MAX_TOPK; window = 0 is dsa_sparse_mla_decode.
 * How the compressed entries are formed is the model's (learned) business;
 * the call takes them as latent rows.  Other arguments, layouts, precision
 * and errors as in dsa_sparse_mla_decode; ws: at least
 * dsa_workspace_bytes(Q, 1, topk + window, num_splits) bytes.
 */
dsa_status dsa_sparse_mla_decode_window(const void* q, const void* kv_pool, int num_pages,
                                        int page_size, const int32_t* page_table, int max_pages,
                                        const int32_t* win_page_table, int win_max_pages,
                                        const int32_t* q_offsets, const int32_t* q_vis,
                                        const int32_t* win_vis, const int32_t* idx, int B, int Q,
                                        int heads, int topk, int window, float scale,
                                        int num_splits, float* out, float* lse, void* ws,
                                        size_t ws_bytes, void* stream);

/*
 * Sparse MLA decode over an FP8 latent cache  ("GLM-5.2 推理部署": MLA plus an
 * FP8 KV cache, --kv-cache-dtype fp8_e4m3, to fit 1M context).
 *   kv_pool   e4m3 [num_pages,page_size,576]: one byte per value; the latent
 *             row is the code's value times kv_scale (one scale for the
 *             whole cache, > 0)
 * Everything else as in dsa_sparse_mla_decode.  The gather widens each e4m3
 * row exactly on chip (every e4m3 value is an fp16 and a bf16 value): the 512
 * latent dims to fp16, the 64 RoPE dims to bf16.  The tensor-core products of
 * the latent dims then take the query's latent dims as fp16, which is exact
 * for every element that is zero or of magnitude 2^-14 .. 65504; smaller ones
 * round to fp16's subnormal spacing 2^-24.  A query element of magnitude
 * 65536 or more (beyond fp16) is flagged as DSA_ERR_DEVICE_BOUNDS through the
 * workspace's error word, and that call's output is not valid.  kv_scale
 * multiplies the scores (with `scale`) and the output.  A row is 576 bytes
 * instead of 1152.
 */
dsa_status dsa_sparse_mla_decode_fp8(const void* q, const void* kv_pool, float kv_scale,
                                     int num_pages, int page_size, const int32_t* page_table,
                                     int max_pages, const int32_t* q_offsets, const int32_t* q_vis,
                                     const int32_t* idx, int B, int Q, int heads, int topk,
                                     float scale, int num_splits, float* out, float* lse, void* ws,
                                     size_t ws_bytes, void* stream);

/*
 * Sparse MLA decode that allocates nothing and takes no workspace.  The
 * pages have no counterpart of this call; it exists for callers that cannot
 * hand the library device memory: a serving engine whose allocator already
 * owns all of HBM (reserved up front for the paged KV cache and weights), or
 * code that must not call cudaMalloc because it synchronises the device.
 *   Arguments, layouts and results are those of dsa_sparse_mla_decode.
 *   The split-K partial outputs live in a fixed 16 MiB array of device memory
 *   owned by the library (every GPU that loads the library holds it until
 *   the process exits), so Q * num_splits (after the library's choice when
 *   num_splits = 0) may not exceed 63 at 128 heads (127 at 64 heads) when it
 *   is above 1; larger requests
 *   return DSA_ERR_UNSUPPORTED and enqueue nothing.  num_splits = 1 uses no
 *   scratch and has no limit on Q.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   All calls share the array and it keeps the last call's contents; calls
 *   whose work overlaps on the GPU (other streams, or several devices'
 *   threads racing on one device) race on it.  Out-of-range indices or pages
 *   are skipped as in dsa_sparse_mla_decode; they, and an expired
 *   device-side wait, raise a flag in an error word at the start of the
 *   array (zero when the library loads), which dsa_noalloc_check_error reads
 *   and clears.  Nothing else in the array needs to start at zero.
 */
dsa_status dsa_sparse_mla_decode_noalloc(const void* q, const void* kv_pool, int num_pages,
                                         int page_size, const int32_t* page_table, int max_pages,
                                         const int32_t* q_offsets, const int32_t* q_vis,
                                         const int32_t* idx, int B, int Q, int heads, int topk,
                                         float scale, int num_splits, float* out, float* lse,
                                         void* stream);

/*
 * The error word of dsa_sparse_mla_decode_noalloc on the current device:
 * synchronises `stream`, reads the word and clears it.  Returns DSA_OK,
 * DSA_ERR_DEVICE_BOUNDS (an index or page outside its range was skipped),
 * DSA_ERR_TIMEOUT (a bounded device-side wait expired; the output of that
 * call is not valid) or DSA_ERR_CUDA.  It allocates nothing either; the pages
 * have no counterpart of it.
 */
dsa_status dsa_noalloc_check_error(void* stream);

/*
 * Merge of split-K partial attentions (exact LSE combine).
 *   o_parts fp32 [Q,S,heads,512], lse_parts fp32 [Q,S,heads] (-inf = empty part)
 *   out fp32 [Q,heads,512], lse fp32 [Q,heads]; heads = 128 or 64.
 */
dsa_status dsa_lse_combine(const float* o_parts, const float* lse_parts, int Q, int S, int heads,
                           float* out, float* lse, void* stream);

/*
 * One DSA decode step over n_layers sparse layers  (section 2.2 pipeline;
 * section 7.2 IndexShare; MTP flow of the inference page for IndexShare on
 * MTP).  Every pointer array below is a HOST array of n_layers device
 * pointers.
 *   index_share      layers per indexer group G >= 1: layer l uses the top-k
 *                    of the indexer of layer G*(l/G); only those layers' entries
 *                    of q_idx_layers / w_layers / k_idx_layers are read.
 *                    G = 4 is GLM-5.2's IndexShare; G = 1 runs every indexer.
 *   mtp_index_share  != 0: the first query of each sequence supplies the
 *                    top-k of all its queries (draft positions reuse step 1).
 *   idx_out          int32 [ceil(n_layers/G), Q, topk]: the index rows used.
 *   out_layers / lse_layers: per layer fp32 [Q,heads,512] / [Q,heads].
 *   heads / idx_heads: 128 / 64 (DeepSeek-V3.2) or 64 / 32 (GLM-5.2).
 * Other arguments as in dsa_indexer_topk and dsa_sparse_mla_decode.
 * The kernels of one call (and of dsa_indexer_topk) are chained with
 * programmatic dependent launch: a kernel may start its set-up while the
 * previous kernel of the same call drains, and waits for it before reading
 * what it wrote.  The first kernel of a call starts only after all earlier
 * work on the stream, as usual.  The call allocates nothing and does not
 * synchronise, so it can be captured into a CUDA graph.
 */
dsa_status dsa_decode_step(int n_layers, int index_share, int mtp_index_share,
                           const uint8_t* const* q_idx_layers, const float* const* w_layers,
                           const uint8_t* const* k_idx_layers, int64_t total_keys,
                           const int64_t* seq_offsets, const int32_t* q_offsets,
                           const int32_t* q_vis, int B, int Q, int heads, int idx_heads,
                           int max_len, int topk,
                           const void* const* q_layers, const void* const* pool_layers,
                           int num_pages, int page_size, const int32_t* const* page_table_layers,
                           int max_pages, float scale, int num_splits,
                           float* const* out_layers, float* const* lse_layers,
                           int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Two-tier latent cache (HiSparse)  ("GLM-5.2 推理部署", section "HiSparse 的
 * 通信路径：GPU↔CPU KV swap": the full cache in pinned host memory, a buffer
 * of hot 16-token slots in HBM; per step, top-K miss detection, LRU
 * eviction, page-table update and an H2D fetch of the missing entries).
 *
 * Layouts.  The host tier of sequence b is pages b*max_pages .. of a pinned
 * host array bf16 [B*max_pages, 16, 576]; its device buffer is slots
 * b*dev_slots .. of a device pool bf16 [B*dev_slots, 16, 576], which
 * dsa_sparse_mla_decode reads with page_size = DSA_TIER_PAGE through the page
 * table the plan produces.  Token s of sequence b is row s%16 of its logical
 * page s/16.
 *
 * Rules (readings of the page): every page a step selects counts as used at
 * that step; the misses of a sequence are placed, in ascending page order,
 * into the slots not selected at this step with the oldest last use (never
 * used first, ties to the lower slot), evicting their pages; a step that
 * selects more distinct pages of one sequence than dev_slots is refused.
 *
 * The state is caller-owned HOST memory of dsa_tier_state_bytes bytes
 * (8-byte aligned); dsa_tier_init resets it (every slot empty).  The plan and
 * the state live on the host: no device work, no synchronisation.
 */
size_t dsa_tier_state_bytes(int B, int dev_slots, int max_pages);   /* 0 = invalid sizes */
dsa_status dsa_tier_init(void* state, size_t state_bytes, int B, int dev_slots, int max_pages);

/*
 * One step's plan, on the host.
 *   idx        HOST int32 [Q,topk]: the step's selected positions (-1 = none),
 *              rows of sequence b at q_offsets[b] .. q_offsets[b+1]-1
 *   q_offsets  HOST int32 [B+1] (q_offsets[B] = Q)
 *   page_table NULL or HOST int32 [B,max_pages] out: device pool page of every
 *              resident logical page, -1 elsewhere (a full table; the fetch
 *              below patches a device table incrementally instead)
 *   copies     HOST int32 [cap_copies,3] out: (host page to fetch, device page
 *              it goes to, host page evicted from that slot or -1)
 *   n_copies   out: copies written;  stats: NULL or int64 [3] out: this
 *              step's hits, misses, evictions (distinct pages)
 * Returns DSA_ERR_UNSUPPORTED if a sequence needs more slots than it has,
 * DSA_ERR_DEVICE_BOUNDS for a position beyond max_pages*16, DSA_ERR_WORKSPACE
 * if the misses exceed cap_copies; a refused step leaves the state unchanged.
 */
dsa_status dsa_tier_plan(void* state, const int32_t* idx, int Q, int topk,
                         const int32_t* q_offsets, int32_t* page_table, int32_t* copies,
                         int cap_copies, int* n_copies, int64_t* stats);

/*
 * Fetch of the planned pages: one kernel reads each planned host page of
 * `copies` (DEVICE int32 [n,3], as the plan wrote them) from the pinned host
 * cache and writes the 18,432-byte page into its device slot, on `stream`.
 *   page_table  NULL or DEVICE int32 [B,max_pages]: patched in the same kernel
 *               (the evicted page's entry becomes -1, the fetched page's
 *               entry its device page), so a table that started as all -1 and
 *               went through every step's fetch equals the plan's table
 *   host_cache  PINNED host memory (cudaHostAlloc / pinned torch tensor) of
 *               host_pages pages; anything else (pageable or device memory)
 *               is refused with DSA_ERR_INVALID_ARG before any launch
 *   dev_pool    device memory of dev_pages pages
 *   ws          workspace (its error word flags copies outside either cache,
 *               which are skipped)
 * Call it once per layer's cache with the same copies.
 */
dsa_status dsa_tier_fetch(const void* host_cache, int64_t host_pages, void* dev_pool,
                          int64_t dev_pages, const int32_t* copies, int n, int32_t* page_table,
                          void* ws, void* stream);

/*
 * The same plan computed on the device, followed by the fetch: one call per
 * step that needs no host round trip (and can be captured in a CUDA graph).
 *   dev_state   DEVICE memory of dsa_tier_dev_state_bytes bytes, reset by
 *               dsa_tier_dev_init (which also sets every page_table entry to
 *               -1); dev_slots <= 8192 (the planner sorts a sequence's slots
 *               in shared memory)
 *   idx         DEVICE int32 [Q,topk]   q_offsets DEVICE int32 [B+1]
 *   page_table  DEVICE int32 [B,max_pages]: the page -> device pool page map,
 *               updated in place (dsa_sparse_mla_decode reads it with
 *               page_size = DSA_TIER_PAGE)
 *   host_cache  PINNED host bf16 [B*max_pages,16,576]   dev_pool DEVICE bf16
 *               [B*dev_slots,16,576]
 *   ws          workspace whose error word takes DSA_ERR_DEVICE_BOUNDS for a
 *               position beyond max_pages*16 (skipped) and DSA_ERR_UNSUPPORTED
 *               (through dsa_check_error) for a sequence that selected more
 *               distinct pages than dev_slots (its step is skipped)
 * The rules are those of dsa_tier_plan; the copy list holds the same triples
 * (sequences may appear in any order).  dsa_tier_dev_stats synchronises the
 * stream and returns the last step's n_copies, hits, misses, evictions and
 * the number of steps so far; dsa_tier_dev_copies is the device address of
 * the copy list (int32 [n_copies,3]) inside dev_state.
 */
size_t dsa_tier_dev_state_bytes(int B, int dev_slots, int max_pages);   /* 0 = invalid sizes */
dsa_status dsa_tier_dev_init(void* dev_state, size_t state_bytes, int B, int dev_slots,
                             int max_pages, int32_t* page_table, void* stream);
dsa_status dsa_tier_swap_in(void* dev_state, size_t state_bytes, int B, int dev_slots,
                            int max_pages, const int32_t* idx, int Q, int topk,
                            const int32_t* q_offsets, int32_t* page_table,
                            const void* host_cache, void* dev_pool, void* ws, void* stream);
dsa_status dsa_tier_dev_stats(const void* dev_state, int64_t* stats /* host int64 [5] */,
                              void* stream);
const int32_t* dsa_tier_dev_copies(const void* dev_state, int B, int dev_slots, int max_pages);

/*
 * Self-test of the device-side failure detection (the pages have no
 * counterpart; it exercises the library's own safety net).  One small kernel
 * waits twice, with the library's bounded waits, on a barrier that never
 * completes, each wait giving up after limit_us microseconds (1 .. 2,000,000;
 * the library's own limit is 2 s), and raises the timeout flag in the error
 * word of `ws` (>= 256 bytes, a workspace from dsa_workspace_bytes
 * qualifies).  The kernel holds no copy, tensor memory or peer CTA, so it
 * simply returns; a following dsa_check_error returns DSA_ERR_TIMEOUT and
 * clears the flag, and the context stays usable.
 */
dsa_status dsa_selftest_bounded_wait(int limit_us, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronises `stream`, reads and clears the workspace's device error flag.
 * Returns DSA_OK, DSA_ERR_DEVICE_BOUNDS, DSA_ERR_TIMEOUT, DSA_ERR_UNSUPPORTED (a device
 * tier step that needed more slots than a sequence has) or DSA_ERR_CUDA.
 */
dsa_status dsa_check_error(void* ws, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
