// Internal interface between the C ABI layer (rtp_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace rtp {

constexpr int kHeadDim = 128;
constexpr int kRank = 16;

enum : int { KIND_SWA = 0, KIND_FULL = 1, KIND_SPARSE = 2 };

// One prefill work item: {kind | slot << 8, seq * n_kv_heads + kv_head,
// query-head pair, 128-row query tile}.
struct PrefillArgs {
  const int4* items;
  long n_items;
  const int32_t* sel;  // [batch][n_sparse][nqb][kmax]
  const int32_t* cnt;  // [batch][n_sparse][nqb]
  __nv_bfloat16* o;    // [batch][n_q_heads][q_rows][128]
  int batch, seq, n_q_heads, n_kv_heads, group, n_sparse;
  int q_row0, q_rows;  // Q/O arrays hold query rows q_row0 .. q_row0 + q_rows - 1
  int q_slab;          // rows between consecutive (sequence, head) slabs of Q/O (>= q_rows)
  int window, block, kmax, nqb;
  float scale_log2;  // softmax scale * log2(e)
  uint32_t* status;
  // 0: one selection per (retrieval slot, query block), sel [batch][n_sparse][nqb][kmax];
  // 1: one per query head, sel [batch][n_sparse][group][nqb][kmax] (block 128 only)
  int sel_heads;
};

struct IndexerArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const float* proj;
  float* centroids;  // [batch][n_sparse][nb][16]
  float* qbar;       // [batch][n_sparse][nb][16]
  const int32_t* slot_heads;  // device [n_sparse] -> kv head
  int batch, seq, n_q_heads, n_kv_heads, group, n_sparse, block;
  int blk0, rows;  // q/k arrays start at row blk0*block; `rows` = rows between consecutive slabs
                   // (outputs use the whole-sequence block index)
  int n_blocks;    // blocks to process, starting at blk0
};

struct SelectArgs {
  const float* qbar;
  const float* centroids;
  int32_t* sel;
  int32_t* cnt;
  int batch, n_sparse, nb, topk, n_local, kmax;
  int t0, n_rows;  // query blocks t0 .. t0 + n_rows - 1 are selected
  int c_group;     // selection rows per centroid slot: 1, or the group size for per-head selection
  // dynamic selection only: mass fraction, minimum count, beta * log2(e)
  float mass;
  int min_k;
  float beta_log2;
  // row-max scores only: the plan's query rows and the projector
  const __nv_bfloat16* q;  // [batch][n_q_heads][q_slab][128], row 0 = query row q_row0
  const float* proj;       // [128][16]
  const int32_t* slot_heads;
  int n_q_heads, n_kv_heads, group, block, q_row0, q_slab;
};
constexpr int kDynMaxCap = 1024;  // largest top-k cap of the dynamic selection

constexpr int kMaxDecodeKvHeads = 256;

struct DecodeArgs {
  const __nv_bfloat16* q;       // [batch][n_q_heads][128]
  const __nv_bfloat16* kcache;  // [batch][n_kv_heads][cache_cap][128], rows < cache_len used
  const __nv_bfloat16* vcache;
  const float* centroids;       // [batch][n_kv_heads][nbc][16], nbc = cache_cap / block
  const float* proj;
  __nv_bfloat16* o;             // [batch][n_q_heads][128]
  uint8_t kind[kMaxDecodeKvHeads];  // routing map, passed by value
  int32_t* sel;                 // [batch][n_kv_heads][kmax] (workspace or caller)
  int32_t* cnt;                 // [batch][n_kv_heads]
  float* partial;               // [n_spans of both lists][group][kPartStride]
  int batch, n_q_heads, n_kv_heads, group, cache_len, cache_cap, nbc;
  int window, block, topk, n_local, kmax;
  float scale_log2;
  uint32_t* status;
  // Schedule of the attention launch.  The work is cut into spans of at most
  // 128 keys (one block of a retrieval head, or 128 consecutive keys of a
  // window/full head) kept in two lists, each ordered (sequence, head, span):
  // list 0 = what needs no selection (window and full heads, and each
  // retrieval head's sink and local blocks), list 1 = the blocks a retrieval
  // head's top-k picked.  CTA c of n_ctas takes the contiguous range
  // [c*N/n_ctas, (c+1)*N/n_ctas) of each list (N = the list's length).
  int n_ctas;
  int per_b[2];                           // spans per sequence in each list
  int span_off[2][kMaxDecodeKvHeads];     // first span of a head within its sequence's part of each list
  // Clustered retrieval heads (k-means of the cache; 0 = contiguous blocks):
  // a retrieval head attends to the sink block, the unclustered tail
  // [clu_end, cache_len) (both in list 0) and the top-k chunks of its
  // clusters (list 1), streamed from the cluster-ordered copy of K/V or,
  // with `gather`, read in place: the chunk's member rows of the cache.
  int clustered;
  int gather;
  int clu_end, clu_rows, max_chunks;
  const __nv_bfloat16* k_sorted;    // [batch][n_kv_heads][clu_rows][128] (NULL with gather)
  const __nv_bfloat16* v_sorted;
  const int32_t* members;           // [batch][n_kv_heads][clu_rows]: cache rows in cluster order
  const float* chunk_centroids;     // [batch][n_kv_heads][max_chunks][16]
  const int32_t* chunk_start;       // [batch][n_kv_heads][max_chunks]
  const int32_t* chunk_len;
  const int32_t* n_chunks;          // [batch][n_kv_heads]
};
constexpr int kPartStride = 132;  // m, l, pad, pad, o[128]

// KV-cache maintenance: appending one token per sequence, and the block
// centroids of retrieval heads in the layout the decode step reads.
struct CacheArgs {
  const __nv_bfloat16* k_new;  // [batch][n_kv_heads][128] (append only)
  const __nv_bfloat16* v_new;
  __nv_bfloat16* kcache;       // [batch][n_kv_heads][cache_cap][128]
  __nv_bfloat16* vcache;
  const float* proj;           // [128][16]
  float* centroids;            // [batch][n_kv_heads][cache_cap / block][16]
  uint8_t kind[kMaxDecodeKvHeads];
  int batch, n_kv_heads, cache_cap, block;
  int pos;       // append: row of the new token
  int n_blocks;  // centroid build: complete blocks to write
};

// k-means clustering of the projected keys of a KV cache (retrieval heads):
// rows [block, clu_end) of each (sequence, KV head), n = clu_end - block.
struct KmeansArgs {
  const __nv_bfloat16* kcache;  // [batch][n_kv_heads][cache_cap][128]
  const __nv_bfloat16* vcache;
  const float* proj;            // [128][16]
  float* X;                     // workspace [batch][n_kv_heads][n][16]: projected keys
  int32_t* assign;              // workspace [batch][n_kv_heads][n]
  float* centroids;             // [batch][n_kv_heads][nc][16]
  int32_t* members;             // [batch][n_kv_heads][n]: key rows grouped by cluster, ascending inside
  int32_t* offsets;             // [batch][n_kv_heads][nc + 1]
  __nv_bfloat16* k_sorted;      // [batch][n_kv_heads][n][128]: K rows in `members` order
  __nv_bfloat16* v_sorted;
  float* chunk_centroids;       // [batch][n_kv_heads][max_chunks][16]
  int32_t* chunk_start;         // [batch][n_kv_heads][max_chunks]: first row in the sorted K/V
  int32_t* chunk_len;
  int32_t* n_chunks;            // [batch][n_kv_heads]
  int32_t* amb_list;            // workspace [batch][n_kv_heads][n]: keys the tensor-core pass left to the exact one
  int32_t* amb_count;           // workspace [batch][n_kv_heads]
  int32_t* seg;                 // workspace [batch][n_kv_heads][n_seg][nc]: per key segment, counts then starts
  int n_seg;                    // key segments of kKmSegKeys keys
  uint8_t kind[kMaxDecodeKvHeads];
  int batch, n_kv_heads, cache_cap, block, clu_end, n, nc, max_chunks;
};
constexpr int kMaxClusters = 2048;
constexpr int kKmSegKeys = 4096;  // keys per segment of the k-means grouping

// Launchers (return the launch error, never synchronise).
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           int num_ctas, cudaStream_t stream);
cudaError_t launch_indexer(const IndexerArgs& a, cudaStream_t stream);
cudaError_t launch_indexer_heads(const IndexerArgs& a, cudaStream_t stream);
cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream);
cudaError_t launch_select_dynamic(const SelectArgs& a, cudaStream_t stream);
cudaError_t launch_select_rowmax(const SelectArgs& a, cudaStream_t stream);
// mks / mvs: the cluster-ordered K/V of clustered mode (any valid map otherwise).
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mks,
                          const CUtensorMap& mvs, cudaStream_t stream);
cudaError_t launch_cache_append(const CacheArgs& a, cudaStream_t stream);
cudaError_t launch_kmeans(const KmeansArgs& a, int iters, cudaStream_t stream);
cudaError_t launch_cache_centroids(const CacheArgs& a, cudaStream_t stream);

// Fixed-size device scratch used by the allocation-free decode entry point.
constexpr size_t kDecodeStaticScratchBytes = size_t(16) << 20;
// Device addresses of that scratch and of its status word on the current
// device (looked up once per device with cudaGetSymbolAddress; no
// allocation).
cudaError_t decode_static_scratch(void** ptr, uint32_t** status);
// The status word of the allocation-free decode on the current device, or
// NULL if that entry point has not run on it (no lookup, no allocation).
uint32_t* decode_static_status_if_used();

// Shared-memory bytes the prefill kernel needs (host side, for the opt-in).
size_t prefill_smem_bytes();

}  // namespace rtp
