/*
 * rtp.h — C ABI of librtp.so: headwise hybrid (SWA + sparse retrieval)
 * attention for NVIDIA B200 (sm_100a).
 *
 * The method (RTPurbo / RTPurboV2) routes every (layer, KV head) to one of
 * two head types:
 *   - streaming heads run sliding-window attention (SWA): the pages
 *     "阿里Qwen3 RTPurbo：15%全量Attention长文本5倍压缩方案" (opening section)
 *     and "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳" (window
 *     8192 for the streaming heads) drop the far tokens of these heads;
 *   - retrieval heads (about 15 %) run either dense causal attention (V1) or,
 *     in V2, block-sparse attention: a trained projector maps keys and
 *     queries from D=128 to r=16 dimensions (RTPurboV2 page, "r=16"), keys
 *     are grouped (clustered) and summarised by centroids, the best blocks
 *     for each query block are selected and exact softmax attention runs on
 *     the selected keys only (summary page of "Full Attention Strikes Back":
 *     the 16-dim indexer is a cheap scout; real attention runs on the
 *     selected set).
 *
 * The pages leave the selection policy open; this library fixes it:
 *   - keys are grouped in contiguous blocks of `block` keys; a block's
 *     centroid is the mean of its projected keys;
 *   - one selection per (KV head, query block of `block` rows), shared by the
 *     query heads of the group; the query summary of block t is the sum over
 *     the group's heads of the mean over the block's rows of the projected
 *     queries;
 *   - query block t scores candidate blocks 1..t-n_local by the dot product
 *     of its summary with their centroids, keeps the `topk` best by
 *     (score descending, block index ascending) and adds block 0 (sink) and
 *     the n_local local blocks max(0,t-n_local+1)..t; the list is sorted
 *     ascending; if at most `topk` candidates exist, all blocks 0..t are
 *     kept;
 *   - causal masking j <= i applies inside every selected block;
 *   - SWA: key j is visible to query i iff i-window < j <= i.
 * Three alternatives to this policy are offered beside it, each feeding the
 * same prefill: a per-query-block budget (rtp_block_select_dynamic), the
 * largest logit over a query block's rows as its score
 * (rtp_block_select_rowmax), and one selection per query head
 * (rtp_indexer_project_heads, rtp_block_select_heads,
 * rtp_hybrid_prefill_heads).
 *
 * Conventions
 *   - Every tensor argument is a DEVICE pointer owned by the caller,
 *     contiguous.  Q/K/V/O are bf16 [batch][heads][seq][128]
 *     (`head_dim` must be 128).  All pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = default stream).
 *     Calls are asynchronous on `stream`; none synchronises except the
 *     set-up call rtp_route_heads and rtp_last_device_status.
 *   - Arguments are validated before anything is launched; a bad argument
 *     returns RTP_ERR_INVALID_ARG and launches nothing.  A CUDA launch error
 *     returns RTP_ERR_CUDA.  No C++ exception crosses this boundary.
 *   - Every device-side wait is bounded (about 2 s); a wait that gives up
 *     ends its kernel early and sets a device status word that
 *     rtp_last_device_status reports as RTP_ERR_TIMEOUT.
 *   - A plan is immutable after creation and may be used from several
 *     streams at once.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RTP_OK = 0,
  RTP_ERR_INVALID_ARG = 1,
  RTP_ERR_UNSUPPORTED = 2,
  RTP_ERR_CUDA = 3,
  RTP_ERR_TIMEOUT = 4,
  RTP_ERR_NO_MEMORY = 5
} rtp_status;

/* Head kinds of the routing map (one byte per KV head). */
enum { RTP_HEAD_SWA = 0, RTP_HEAD_FULL = 1, RTP_HEAD_SPARSE = 2 };

typedef struct {
  int batch;       /* sequences                                                  */
  int seq;         /* tokens per sequence (prefill); multiple of `block`.
                      Decode and cache calls: rows allocated per (sequence,
                      KV head) in the cache (its capacity)                      */
  int n_q_heads;   /* query heads                                                */
  int n_kv_heads;  /* KV heads; group = n_q_heads / n_kv_heads must be an even
                      integer <= 16 (prefill processes query heads in pairs)     */
  int head_dim;    /* must be 128                                                */
  int window;      /* SWA keys including self (i-window < j <= i); >= 1          */
  int block;       /* key block = query block for selection: 64 or 128           */
  int rank;        /* projector rank r; must be 16                               */
  int topk;        /* selected candidate blocks per query block                  */
  int n_sink;      /* sink blocks; must be 1 (block 0)                           */
  int n_local;     /* local blocks (diagonal included); >= 1                     */
  float scale;     /* softmax scale; 0 => 1/sqrt(head_dim)                       */
} rtp_attn_cfg;

typedef struct rtp_plan rtp_plan; /* opaque, library-owned */

/* ------------------------------------------------------------------------
 * rtp_route_heads — compile the routing map of one layer into a plan.
 * Pages: RTPurbo page, "RTP-LLM：RTPurbo 在长文上的极致性能优化" (different
 * head types have different costs; schedule heavy tiles first to cut tail
 * latency).
 *   cfg        shapes and selection constants (validated here).
 *   kind_host  HOST array [cfg->n_kv_heads] of RTP_HEAD_* values.
 *   stream     stream for the plan's one-time host-to-device upload.
 *   out        receives the plan; release with rtp_plan_destroy.
 * The plan holds the work list of the prefill kernel: one entry per
 * (sequence, KV head, pair of query heads, 128-row query tile), ordered by
 * descending cost (KV tiles to visit) so that a persistent grid takes the
 * heaviest tiles first.  Retrieval heads of kind RTP_HEAD_SPARSE are
 * numbered 0..n_sparse-1 in KV-head order ("retrieval slots"); the indexer
 * and selection buffers are indexed by slot.
 * This set-up call uploads the work list on `stream` and synchronises it
 * before returning, so the plan may then be used on any stream.
 * Errors: RTP_ERR_INVALID_ARG (bad cfg or kind), RTP_ERR_NO_MEMORY,
 * RTP_ERR_CUDA.
 * ---------------------------------------------------------------------- */
rtp_status rtp_route_heads(const rtp_attn_cfg* cfg, const uint8_t* kind_host, void* stream, rtp_plan** out);

/* ------------------------------------------------------------------------
 * rtp_route_heads_range — a plan for the query rows [q_begin, q_end) of the
 * sequence only: one rank's share under context parallelism (RTPurbo page,
 * "RTP-LLM：RTPurbo 在长文上的极致性能优化": context parallelism instead of
 * tensor parallelism, so that each GPU computes every head's attention for
 * its part of the context).  rtp_route_heads(cfg, ...) is
 * rtp_route_heads_range(cfg, ..., 0, cfg->seq, ...).
 *   q_begin   multiple of 128, 0 <= q_begin < q_end
 *   q_end     multiple of 128, or cfg->seq; q_end <= cfg->seq
 * With a ranged plan the other calls work on that range:
 *   rtp_indexer_project  q and k hold rows [q_begin, q_end) only
 *       ([batch][heads][q_end-q_begin][128]); centroids / qbar keep their
 *       whole-sequence layout and only the blocks q_begin/block ..
 *       q_end/block-1 are written
 *   rtp_block_select(_dynamic)  only the query blocks of the range are
 *       selected (whole-sequence sel/cnt layout); the centroids of every
 *       earlier block must be present (gathered from the other ranks)
 *   rtp_hybrid_prefill  q and o hold rows [q_begin, q_end) only; k and v are
 *       [batch][n_kv_heads][q_end][128] of which only the rows the range's
 *       queries can see are read (the window before q_begin for SWA heads,
 *       every earlier row for full heads, the selected blocks for sparse
 *       heads, and the range itself)
 * ---------------------------------------------------------------------- */
rtp_status rtp_route_heads_range(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int q_begin, int q_end,
                                 void* stream, rtp_plan** out);

/* ------------------------------------------------------------------------
 * rtp_route_heads_split — rtp_route_heads_range with the work list in two
 * parts, so that a context-parallel rank can start attention while the
 * earlier K/V rows it needs are still arriving (RTPurbo page, "RTP-LLM：
 * RTPurbo 在长文上的极致性能优化": context parallelism with communication
 * overlapped by computation).
 *   key_begin  0 <= key_begin <= q_begin: the first K/V row present locally
 *   The first rtp_plan_num_local_items(plan) items are the tiles whose
 *   visible keys all lie at or after key_begin (streaming heads whose window
 *   starts there; a full or sparse head always sees row 0, so its tiles are
 *   local only when key_begin = 0); the other items follow.  Each part is
 *   ordered longest first.  Run the parts with rtp_hybrid_prefill_items;
 *   rtp_hybrid_prefill runs them all.  Every other call works as with
 *   rtp_route_heads_range.
 * Errors: as rtp_route_heads_range, and RTP_ERR_INVALID_ARG for key_begin
 * outside [0, q_begin].
 * ---------------------------------------------------------------------- */
rtp_status rtp_route_heads_split(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int q_begin, int q_end,
                                 int key_begin, void* stream, rtp_plan** out);
/* Items of a split plan that see only local keys (the whole list for a plan
 * made by rtp_route_heads / rtp_route_heads_range); -1 for NULL. */
long rtp_plan_num_local_items(const rtp_plan* plan);
void rtp_plan_destroy(rtp_plan* plan);

/* Number of retrieval slots (KV heads of kind RTP_HEAD_SPARSE). */
int rtp_plan_num_sparse(const rtp_plan* plan);
/* Number of prefill work items (tiles) in the plan. */
long rtp_plan_num_items(const rtp_plan* plan);
/* Copies the KV-head index of each retrieval slot into slots_host
 * [rtp_plan_num_sparse]. */
rtp_status rtp_plan_sparse_heads(const rtp_plan* plan, int32_t* slots_host);
/* Copies the plan's work list (HOST int32 [n_items][4] = {kind | slot<<8,
 * sequence*n_kv_heads + kv_head, query-head pair, query tile}) in the order
 * the prefill kernel consumes it. */
rtp_status rtp_plan_work_items(const rtp_plan* plan, int32_t* items_host);

/* ------------------------------------------------------------------------
 * rtp_indexer_project — low-rank projection, block centroids and query-block
 * summaries for every retrieval slot (RTPurboV2 page: the projector keeps
 * the low-frequency rotary components in r=16 dimensions; clustering of the
 * projected keys; summary page of "Full Attention Strikes Back": the 16-dim
 * indexer).
 *   q          bf16 [batch][n_q_heads][seq][128]
 *   k          bf16 [batch][n_kv_heads][seq][128]
 *   proj       fp32 [128][16], row d = input dimension
 *   centroids  fp32 [batch][n_sparse][seq/block][16] (out):
 *              c_b = (1/block) * sum_{j in block b} proj^T k_j
 *   qbar       fp32 [batch][n_sparse][seq/block][16] (out):
 *              qbar_t = sum_{h in group} (1/block) sum_{i in block t} proj^T q_{h,i}
 * Reductions run in a fixed order (deterministic results).  A plan with no
 * retrieval slot makes this a no-op.
 * ---------------------------------------------------------------------- */
rtp_status rtp_indexer_project(const rtp_plan* plan, const void* q, const void* k, const float* proj,
                               float* centroids, float* qbar, void* stream);

/* ------------------------------------------------------------------------
 * rtp_block_select — per (retrieval slot, query block) selection
 * (RTPurboV2 page: fixed top-k is the classic policy; the rule used is the
 * one stated at the top of this file).
 *   qbar, centroids  as written by rtp_indexer_project
 *   sel      int32 [batch][n_sparse][seq/block][kmax] (out), kmax =
 *            topk + 1 + n_local: selected block indices, ascending; unused
 *            entries are -1
 *   sel_cnt  int32 [batch][n_sparse][seq/block] (out): entries used
 * Scores are fp32 with a fixed summation order; ties in score go to the
 * lower block index.
 * ---------------------------------------------------------------------- */
rtp_status rtp_block_select(const rtp_plan* plan, const float* qbar, const float* centroids, int32_t* sel,
                            int32_t* sel_cnt, void* stream);

/* ------------------------------------------------------------------------
 * rtp_block_select_dynamic — selection with a per-query-block budget instead
 * of a fixed top-k (RTPurboV2 page: the fixed top-k policy is criticised
 * because heads, sequence lengths and queries need very different numbers of
 * context tokens; the page gives no rule, so this is the library's):
 *   candidates j = 1..t-n_local of query block t, scores s_j = qbar_t . c_j
 *   (fp32, fixed order as in rtp_block_select), weights
 *   w_j = exp(beta * (s_j - max s)), Z = sum w_j; keep the shortest prefix of
 *   the candidates in (score desc, index asc) order whose weights sum to
 *   >= mass * Z (all of them if no prefix does), clamped to
 *   [min(min_k, #candidates), min(topk, #candidates)]; add block 0 and the
 *   local blocks max(0,t-n_local+1)..t.
 *   plan      its topk is the cap (<= 1024, else RTP_ERR_UNSUPPORTED)
 *   mass      fraction of the candidates' weight to cover, 0 < mass <= 1
 *   min_k     smallest number of candidates kept, 0 <= min_k <= topk
 *   beta      inverse temperature on the low-rank scores, >= 0 (0: every
 *             candidate weighs the same, so ceil(mass * #candidates) are
 *             kept); the softmax scale divided by the group size weighs a
 *             block like the mean over the group's heads of its logits
 *   qbar, centroids, sel, sel_cnt  as in rtp_block_select (same layout,
 *             kmax = topk + 1 + n_local; rows end with -1 padding), so the
 *             result feeds rtp_hybrid_prefill unchanged
 * Every sum runs in a fixed order: results are bit-reproducible.
 * Errors: RTP_ERR_INVALID_ARG (bad plan, mass, min_k, beta or pointer;
 * nothing launched), RTP_ERR_UNSUPPORTED (topk > 1024), RTP_ERR_CUDA.
 * ---------------------------------------------------------------------- */
rtp_status rtp_block_select_dynamic(const rtp_plan* plan, const float* qbar, const float* centroids, float mass,
                                    int min_k, float beta, int32_t* sel, int32_t* sel_cnt, void* stream);

/* ------------------------------------------------------------------------
 * rtp_block_select_rowmax — the fixed top-k rule with another score: a
 * query block scores a candidate by the largest low-rank logit over its rows
 * instead of the mean (RTPurboV2 page: the query-side aggregate of the
 * indexer is left open; one row pointing at a block is then enough to keep
 * it):
 *   s_j = max_{i in block t} u_i . c_j,  u_i = P^T sum_{h in group} q_{h,i}
 *   (u_i in fp32: the group's bf16 rows summed in head order, projected with
 *   a fixed summation order; each dot product as two fixed-order chains over
 *   ranks 0-7 and 8-15, then their sum); keep the topk best candidates 1..t-n_local by (score
 *   desc, index asc), block 0 and the local blocks, as rtp_block_select.
 *   q          the plan's query rows, as for rtp_hybrid_prefill
 *   proj       fp32 [128][16]
 *   centroids  as written by rtp_indexer_project
 *   sel, sel_cnt  as in rtp_block_select (same layout), so the result feeds
 *             rtp_hybrid_prefill unchanged
 * Work: block x 16 FMA per candidate and query block (6.7 ms on B200 for
 * the 1M-token retrieval head with block 128, against 0.96 ms for the mean
 * scores) on top of one more read of the group's Q rows.
 * Errors: RTP_ERR_INVALID_ARG (bad plan or pointer; nothing launched),
 * RTP_ERR_CUDA.
 * ---------------------------------------------------------------------- */
rtp_status rtp_block_select_rowmax(const rtp_plan* plan, const void* q, const float* proj, const float* centroids,
                                   int32_t* sel, int32_t* sel_cnt, void* stream);

/* ------------------------------------------------------------------------
 * Per-head selection — the other query-side alternative: every query head
 * selects its own blocks instead of its group sharing one list (RTPurboV2
 * page: the indexer scores query against key summaries; which query rows
 * share a selection is left open).  Three calls, for a whole-sequence plan
 * with block 128 and an even group (else RTP_ERR_UNSUPPORTED):
 *
 * rtp_indexer_project_heads — qbar_{h,t} = (1/B) sum_{i in block t} P^T q_{h,i}
 *   for every head h of every retrieval slot's group:
 *   qbar_heads  fp32 [batch][n_sparse][group][seq/block][16] (out); for a
 *               group of one head it is rtp_indexer_project's qbar
 *   (the centroids come from rtp_indexer_project, which is still needed)
 *
 * rtp_block_select_heads — the rule of rtp_block_select for each head's
 *   summary against its slot's centroids:
 *   sel      int32 [batch][n_sparse][group][seq/block][kmax] (out)
 *   sel_cnt  int32 [batch][n_sparse][group][seq/block] (out)
 *
 * rtp_hybrid_prefill_heads — rtp_hybrid_prefill on per-head selections: head
 *   h of a retrieval KV head attends to the blocks of its own list (with the
 *   causal mask).  The two heads of a query-head pair share one stream of
 *   K/V tiles, the union of their lists; a tile outside one head's list is
 *   skipped for that head (no MMAs, no softmax), but the pair's pipeline
 *   still walks the whole union, so the time grows with how much the pair's
 *   lists differ.
 * Errors: RTP_ERR_INVALID_ARG (bad plan or pointer; nothing launched),
 * RTP_ERR_UNSUPPORTED (ranged plan, block 64 or odd group), RTP_ERR_CUDA.
 * ---------------------------------------------------------------------- */
rtp_status rtp_indexer_project_heads(const rtp_plan* plan, const void* q, const float* proj, float* qbar_heads,
                                     void* stream);
rtp_status rtp_block_select_heads(const rtp_plan* plan, const float* qbar_heads, const float* centroids,
                                  int32_t* sel, int32_t* sel_cnt, void* stream);
rtp_status rtp_hybrid_prefill_heads(const rtp_plan* plan, const void* q, const void* k, const void* v,
                                    const int32_t* sel, const int32_t* sel_cnt, void* o, void* stream);

/* ------------------------------------------------------------------------
 * rtp_hybrid_prefill — causal prefill attention over the routing map.
 * RTPurbo page (streaming heads: SWA; full heads: dense causal) and
 * RTPurboV2 page / "Full Attention Strikes Back" summary (sparse heads:
 * exact softmax over the selected blocks).  For query head h (KV head
 * h / group) and query i:  O_i = softmax_j(scale * q_i . k_j) V over the
 * visible keys of the head's kind.
 *   q, k, v  bf16 as in rtp_indexer_project
 *   sel, sel_cnt  from rtp_block_select (may be NULL when the plan has no
 *            retrieval slot)
 *   o        bf16 [batch][n_q_heads][seq][128] (out)
 * bf16 inputs, fp32 accumulation (tensor memory), bf16 output.
 * ---------------------------------------------------------------------- */
rtp_status rtp_hybrid_prefill(const rtp_plan* plan, const void* q, const void* k, const void* v,
                              const int32_t* sel, const int32_t* sel_cnt, void* o, void* stream);

/* ------------------------------------------------------------------------
 * rtp_hybrid_prefill_items — rtp_hybrid_prefill for the work items
 * [item_begin, item_end) of the plan's list only (the order of
 * rtp_plan_work_items), on at most max_ctas persistent CTAs (0 = one per
 * SM).  Tiles are computed exactly as in rtp_hybrid_prefill (same result bit
 * for bit), so launches over disjoint item ranges fill disjoint tiles of o.
 * A cap below the SM count leaves SMs free for kernels that must run
 * alongside, e.g. the collectives of a K/V exchange.
 *   0 <= item_begin <= item_end <= rtp_plan_num_items(plan); max_ctas >= 0
 * Errors: as rtp_hybrid_prefill, and RTP_ERR_INVALID_ARG for a bad range.
 * ---------------------------------------------------------------------- */
rtp_status rtp_hybrid_prefill_items(const rtp_plan* plan, const void* q, const void* k, const void* v,
                                    const int32_t* sel, const int32_t* sel_cnt, void* o, long item_begin,
                                    long item_end, int max_ctas, void* stream);

/* ------------------------------------------------------------------------
 * rtp_hybrid_prefill_host — the prefill of one layer whose Q, K, V and O are
 * in host memory (a serving engine's view of a request).  The layer is cut
 * into n_chunks runs of query rows (whole 128-row tiles; equal runs, except
 * that with four or more the last two are a half and a quarter of the others,
 * since that chunk's kernels and download follow the last upload and overlap
 * nothing; every run has at least one tile); chunk c's Q, K and
 * V rows go to the device on an upload stream, its indexer, selection and
 * attention run on `stream` as soon as they have arrived (the attention of
 * rows [begin, end) only reads K/V rows < end, all of them uploaded by then),
 * and its O rows return on a download stream: uploads, kernels and
 * downloads of different chunks overlap.  The result equals rtp_route_heads
 * + rtp_indexer_project + rtp_block_select + rtp_hybrid_prefill on the same
 * data, bit for bit (each tile is computed the same way).
 *   rtp_pipeline_create  plans the chunks (one ranged plan each; uploads
 *       them on `stream` and synchronises it, like rtp_route_heads)
 *   q_host, k_host, v_host, o_host  HOST bf16 [batch][heads][seq][128];
 *       page-locked memory lets the copies run asynchronously (other host
 *       memory works, with copies that block)
 *   proj       DEVICE fp32 [128][16]
 *   q_dev .. o_dev  DEVICE staging of the same shapes
 *   centroids, qbar, sel, sel_cnt  DEVICE, as for rtp_block_select (may be
 *       NULL without retrieval heads)
 * The call returns once everything is queued; `stream` completes after the
 * last O rows have reached o_host.
 * Errors: RTP_ERR_INVALID_ARG (bad cfg, chunk count, NULL or unaligned
 * pointer), RTP_ERR_NO_MEMORY, RTP_ERR_CUDA.
 * ---------------------------------------------------------------------- */
typedef struct rtp_pipeline rtp_pipeline; /* opaque, library-owned */
rtp_status rtp_pipeline_create(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int n_chunks, void* stream,
                               rtp_pipeline** out);
void rtp_pipeline_destroy(rtp_pipeline* pipeline);
rtp_status rtp_hybrid_prefill_host(rtp_pipeline* pipeline, const void* q_host, const void* k_host, const void* v_host,
                                   const float* proj, void* o_host, void* q_dev, void* k_dev, void* v_dev,
                                   void* o_dev, float* centroids, float* qbar, int32_t* sel, int32_t* sel_cnt,
                                   void* stream);

/* ------------------------------------------------------------------------
 * rtp_sparse_decode — one decode step (one new token per sequence) over a
 * KV cache (RTPurboV2 page: retrieval heads are sparsified in decode; the
 * streaming heads keep a window).  The new token's K/V are already the last
 * cache entry, so the query sits at position cache_len-1.
 *   cfg        batch, n_q_heads, n_kv_heads, head_dim, window, block, rank,
 *              topk, n_sink, n_local, scale are used; seq is the cache
 *              capacity (see below)
 *   kind_host  HOST [n_kv_heads] (n_kv_heads <= 256): RTP_HEAD_SPARSE
 *              (retrieval) or RTP_HEAD_SWA; RTP_HEAD_FULL attends to the
 *              whole cache
 *   q          bf16 [batch][n_q_heads][1][128]
 *   kcache, vcache  bf16 [batch][n_kv_heads][cap][128], of which rows
 *              0..cache_len-1 are read; cap = cfg->seq when cfg->seq >=
 *              cache_len (a cache allocated once and filled by
 *              rtp_cache_append), else cap = cache_len
 *   centroids  fp32 [batch][n_kv_heads][cap/block][16]: centroid of every
 *              complete cache block (entries of non-retrieval heads are not
 *              read; see rtp_cache_centroids / rtp_cache_append)
 *   proj       fp32 [128][16]
 *   o          bf16 [batch][n_q_heads][1][128] (out)
 *   workspace  device scratch of at least rtp_decode_workspace_bytes bytes
 *   sel_out, cnt_out  optional (may be NULL): int32 [batch][n_kv_heads][kmax]
 *              and [batch][n_kv_heads]: the selected blocks of retrieval
 *              heads (rows of other heads are left untouched)
 * Retrieval heads score qbar = sum_{h in group} proj^T q_h against the
 * centroids of blocks 1..t-n_local (t = (cache_len-1)/block) and attend to
 * the selected blocks; split-K over blocks, merged by log-sum-exp.
 * ---------------------------------------------------------------------- */
size_t rtp_decode_workspace_bytes(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len);
rtp_status rtp_sparse_decode(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* q,
                             const void* kcache, const void* vcache, const float* centroids, const float* proj,
                             void* o, void* workspace, size_t ws_bytes, int32_t* sel_out, int32_t* cnt_out,
                             void* stream);

/* ------------------------------------------------------------------------
 * rtp_sparse_decode_noalloc — the decode step of rtp_sparse_decode for
 * callers that cannot allocate device memory at call time: real-time loops
 * that must not enter the allocator (cudaMalloc synchronises the device),
 * or hosts whose memory pools are owned by another runtime.  The method
 * itself has no counterpart to this entry point; it is a variant of
 * rtp_sparse_decode for such callers.
 *   Arguments are those of rtp_sparse_decode without workspace/ws_bytes.
 *   The split-K scratch (selection lists and per-split partial results)
 *   lives in a fixed 16 MiB device array inside the library
 *   (rtp_decode_workspace_bytes tells how much a shape needs); a shape that
 *   needs more returns RTP_ERR_INVALID_ARG.  Nothing is allocated: no
 *   cudaMalloc, cudaFree or allocating library call on this path.
 *   The array's address is looked up once per device, on the first call
 *   made with that device current.
 *   Every call shares the one array and it keeps the last call's contents;
 *   a call writes every word it reads earlier in the same call (selection
 *   lists, then per-split partial results), so nothing needs clearing —
 *   unless one of its bounded waits gives up, in which case that call's
 *   output is undefined and the time-out is reported as below.  Calls that
 *   overlap on the GPU — on different streams, or from several host
 *   threads — race on the array and must be serialised by the caller.
 *   Errors on the device: this path reports in its own status word, a
 *   second fixed device word beside the array (looked up with it), not in
 *   the allocated word of the other entry points.  rtp_last_device_status
 *   reads and clears both and allocates nothing itself, so a caller of this
 *   path reads RTP_ERR_TIMEOUT (a bounded wait gave up) or
 *   RTP_ERR_INVALID_ARG (an out-of-range block index was skipped) there.
 * ---------------------------------------------------------------------- */
rtp_status rtp_sparse_decode_noalloc(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* q,
                                     const void* kcache, const void* vcache, const float* centroids,
                                     const float* proj, void* o, int32_t* sel_out, int32_t* cnt_out, void* stream);

/* ------------------------------------------------------------------------
 * rtp_cache_centroids — block centroids of a KV cache in the layout the
 * decode step reads (RTPurboV2 page: decode scores the centroids of the
 * projected cached keys; the same page describes running full attention in
 * prefill and clustering the K cache afterwards, which is this call after an
 * rtp_hybrid_prefill with RTP_HEAD_FULL heads).
 *   cfg        batch, n_kv_heads, head_dim, block, rank used (validated as
 *              for rtp_sparse_decode); seq = cache capacity as there
 *   kind_host  HOST [n_kv_heads]: only RTP_HEAD_SPARSE heads are written
 *   cache_len  rows held per (sequence, KV head), >= 1; the complete blocks
 *              0 .. cache_len/block - 1 are written
 *   kcache     bf16 [batch][n_kv_heads][cap][128] (device)
 *   proj       fp32 [128][16] (device)
 *   centroids  fp32 [batch][n_kv_heads][cap/block][16] (device, out):
 *              c_b = (1/block) sum_{j in block b} proj^T k_j, summed in the
 *              fixed order of rtp_indexer_project (same fp32 value for the
 *              same keys); other entries are left untouched
 * centroids and proj may be NULL when no head is RTP_HEAD_SPARSE.
 * Errors: RTP_ERR_INVALID_ARG (bad cfg, kind, length, NULL or unaligned
 * pointer; nothing launched), RTP_ERR_CUDA (launch failure).
 * ---------------------------------------------------------------------- */
rtp_status rtp_cache_centroids(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len, const void* kcache,
                               const float* proj, float* centroids, void* stream);

/* ------------------------------------------------------------------------
 * rtp_cache_append — append one token per sequence to a KV cache of fixed
 * capacity and keep the centroids current (RTPurboV2 page: the centroids of
 * the projected keys stand for their cache blocks in decode; a block's
 * centroid is defined once its last row is cached, and the block of the
 * newest token is always one of the local blocks the decode step reads in
 * full).
 *   cfg        as for rtp_cache_centroids; seq = capacity cap (rows
 *              allocated per (sequence, KV head)), required
 *   kind_host  HOST [n_kv_heads]
 *   pos        row of the new token = rows already cached, 0 <= pos < cap
 *   k_new, v_new  bf16 [batch][n_kv_heads][128] (device)
 *   kcache, vcache  bf16 [batch][n_kv_heads][cap][128] (device, in/out):
 *              row pos is written, no other row
 *   proj       fp32 [128][16] (device)
 *   centroids  fp32 [batch][n_kv_heads][cap/block][16] (device, in/out):
 *              when (pos+1) % block == 0, entry (pos+1)/block - 1 of every
 *              RTP_HEAD_SPARSE head is written (as rtp_cache_centroids
 *              would write it); nothing else
 * After the call, rtp_sparse_decode with cache_len = pos + 1 and the same
 * cfg (seq = cap) decodes the new token.
 * Errors: RTP_ERR_INVALID_ARG (bad cfg, kind, pos, NULL or unaligned
 * pointer; nothing launched), RTP_ERR_CUDA (launch failure).
 * ---------------------------------------------------------------------- */
rtp_status rtp_cache_append(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int pos, const void* k_new,
                            const void* v_new, void* kcache, void* vcache, const float* proj, float* centroids,
                            void* stream);

/* ------------------------------------------------------------------------
 * Clustered KV cache (RTPurboV2 page: clustering the projected keys lets
 * decode skip whole groups of unrelated tokens; the page's deployment runs
 * full attention in prefill, clusters the K cache, then decodes sparsely).
 * Rows [block, clu_end) of every retrieval head are grouped by k-means of
 * their projected keys P^T k; each cluster's keys (ascending positions) are
 * cut into chunks of at most 128 keys, the units the decode step selects.
 * All arrays are device memory owned by the caller; n = clu_end - block,
 * max_chunks = n / 128 + n_clusters (an upper bound on the chunks of a head).
 * Entries of non-retrieval heads are not written or read.
 * With k_sorted and v_sorted NULL no cluster-ordered copy of K/V is made
 * (2 x n x 256 bytes per head saved, and its writing): the decode step then
 * gathers each selected chunk's member rows from the cache itself (16-byte
 * asynchronous copies into the same shared-memory layout), with the same
 * result bit for bit.
 * ---------------------------------------------------------------------- */
typedef struct {
  int clu_end;             /* rows [block, clu_end) are clustered: multiple of block, > block */
  int n_clusters;          /* 1 .. 2048, <= n */
  float* centroids;        /* fp32 [batch][n_kv_heads][n_clusters][16] */
  int32_t* members;        /* [batch][n_kv_heads][n]: key rows grouped by cluster, ascending inside */
  int32_t* offsets;        /* [batch][n_kv_heads][n_clusters + 1]: cluster c = members[offsets[c] ..] */
  void* k_sorted;          /* bf16 [batch][n_kv_heads][n][128]: K rows in `members` order, or NULL */
  void* v_sorted;          /* bf16, likewise for V (NULL exactly when k_sorted is) */
  float* chunk_centroids;  /* fp32 [batch][n_kv_heads][max_chunks][16]: the centroid of the chunk's cluster */
  int32_t* chunk_start;    /* [batch][n_kv_heads][max_chunks]: first row of the chunk in `members` order */
  int32_t* chunk_len;      /* [batch][n_kv_heads][max_chunks]: 1..128 */
  int32_t* n_chunks;       /* [batch][n_kv_heads]: chunks in use, cluster-major order */
} rtp_clusters;

/* ------------------------------------------------------------------------
 * rtp_cache_cluster — k-means of the projected cached keys of every
 * retrieval head (the library's reading of the page's clustering):
 * seeds mu_c = X[floor((2c+1) n / (2 n_clusters))] of X_j = P^T k_j
 * (fp32, fixed order); `iters` rounds of: each key to the nearest centroid
 * (squared distance, evaluated as |mu|^2 - 2 x.mu; ties to the lower
 * index), each centroid to the mean of its keys (an empty cluster keeps its
 * centroid).  Then the members, offsets, chunk table and the K/V rows in
 * cluster order are written.  Deterministic (fixed-order sums, a stable
 * counting sort).  The K/V copy is skipped when cl->k_sorted is NULL.
 * The distances are computed on tensor cores in fp16 where that provably
 * decides a key's nearest centroid, and in fp32 otherwise; the result is
 * the fp32 evaluation's for every key.  Setting the environment variable
 * RTP_KMEANS_EXACT_ASSIGN=1 (read once per process) makes every key take
 * the fp32 path (a diagnostic: the results are the same).
 *   cfg        batch, n_kv_heads, head_dim, block, rank used; seq = cache
 *              capacity as for rtp_sparse_decode (must be >= clu_end)
 *   kind_host  HOST [n_kv_heads]; RTP_HEAD_SPARSE heads are clustered
 *   iters      rounds, 1 .. 1000
 *   kcache, vcache, proj  as for rtp_sparse_decode
 *   cl         clu_end, n_clusters and the output arrays
 *   workspace  device scratch of rtp_cache_cluster_workspace_bytes bytes
 * Errors: RTP_ERR_INVALID_ARG (nothing launched), RTP_ERR_CUDA.
 * ---------------------------------------------------------------------- */
size_t rtp_cache_cluster_workspace_bytes(const rtp_attn_cfg* cfg, int clu_end);
rtp_status rtp_cache_cluster(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int iters, const void* kcache,
                             const void* vcache, const float* proj, const rtp_clusters* cl, void* workspace,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * rtp_sparse_decode_clustered — rtp_sparse_decode with clustered retrieval
 * heads: such a head scores the chunks of its clusters by
 * qbar . centroid(cluster) (qbar = sum_{h in group} P^T q_h), keeps the topk
 * best by (score desc, chunk index asc) and attends exactly to their keys,
 * to the sink block [0, block) and to every key of the unclustered tail
 * [clu_end, cache_len) (tokens cached after clustering; clu_end <=
 * cache_len).  Streaming (SWA) and full heads are as in rtp_sparse_decode.
 * Arguments as rtp_sparse_decode (centroids replaced by `cl`); sel_out /
 * cnt_out rows hold, for a retrieval head, entry 0 (the sink) then the
 * selected chunk indices, and cnt = 1 + tail spans + chunks kept.
 * ---------------------------------------------------------------------- */
size_t rtp_decode_clustered_workspace_bytes(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len,
                                            int clu_end);
rtp_status rtp_sparse_decode_clustered(const rtp_attn_cfg* cfg, const uint8_t* kind_host, int cache_len,
                                       const void* q, const void* kcache, const void* vcache, const float* proj,
                                       const rtp_clusters* cl, void* o, void* workspace, size_t ws_bytes,
                                       int32_t* sel_out, int32_t* cnt_out, void* stream);

/* ------------------------------------------------------------------------
 * rtp_last_device_status — synchronise `stream`, then read and clear the
 * device status words of the current device: the word the entry points
 * allocate on first use (if one has) and the fixed word of
 * rtp_sparse_decode_noalloc (if that has run).  Creates neither, so it
 * allocates nothing.  Returns RTP_OK, RTP_ERR_TIMEOUT (a bounded wait gave
 * up), RTP_ERR_INVALID_ARG (a kernel met an out-of-range block index and
 * skipped it) or RTP_ERR_CUDA (the stream reported an error).
 * ---------------------------------------------------------------------- */
rtp_status rtp_last_device_status(void* stream);

/* ------------------------------------------------------------------------
 * rtp_selftest_bounded_wait — diagnostic: launches a one-warp kernel that
 * waits on an mbarrier nothing ever arrives on, using the same bounded wait
 * as every kernel of the library but with a limit of `limit_ms`
 * (1..10000).  The wait must give up, record the time-out in the device
 * status word and let the kernel exit; the call then returns what
 * rtp_last_device_status reports (RTP_ERR_TIMEOUT when the mechanism works)
 * and the context stays usable.  Synchronises `stream`.
 * ---------------------------------------------------------------------- */
rtp_status rtp_selftest_bounded_wait(unsigned limit_ms, void* stream);

/* Human-readable name of a status code (static string). */
const char* rtp_status_str(rtp_status s);

/* Library version, (major << 16) | minor. */
int rtp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H_ */
