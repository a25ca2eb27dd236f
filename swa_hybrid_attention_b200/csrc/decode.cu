// Sparse decode step: one new token per sequence over a KV cache.
//
// Page "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳": in the
// Qwen3-Coder experiment retrieval heads are sparsified in the decode phase
// while the streaming heads keep a window of 8192; the summary of "Full
// Attention Strikes Back" reports the decode speed-up.  For a retrieval head
// the query summary qbar = sum_{h in group} P^T q_h scores the cached block
// centroids, the sink + top-k + local blocks are selected (the prefill rule
// with t = the block of the new token), and exact softmax attention runs
// over the selected keys; streaming heads attend to the last `window` keys.
//
// Three launches on the caller's stream, chained by programmatic dependent
// launch so each may start while its predecessor finishes:
//  1. decode_select_kernel  (retrieval head, sequence): summary + selection.
//  2. decode_attn_kernel    persistent, one CTA per SM.  The keys to visit are
//     cut into spans of <= 128 (one selected block, or 128 consecutive keys
//     of a window/full head) in two lists, window/full heads first; each CTA
//     takes a contiguous range of each list, so it works through its window
//     spans while the selection is still running and only then waits for it.
//     A producer warp streams the spans' K and V through a 3-stage TMA ring;
//     four consumer warps each take 32 keys of every span and run S^T =
//     K Q^T, their own online softmax and O^T += V^T P^T on tensor cores
//     (mma.sync m16n8k16 with keys, then head dims, as M and the group's
//     query heads as N: each K/V byte is read once per group, no row is
//     padding).  Consecutive spans of one (sequence, head) merge online; the
//     warps merge at the end of a run, which writes one partial (m, l, o).
//  3. decode_combine_kernel (query head, sequence): log-sum-exp merge of the
//     runs of the head.
// The step is bound by HBM reads of the selected K/V and the windows.

#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "internal.cuh"
#include "select_common.cuh"
#include "sm100.cuh"

namespace rtp {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kAttnThreads = 32 * (kConsumerWarps + 1);  // + one producer warp
constexpr int kCombineThreads = 128;
constexpr int kRingStages = 3;
// The producer prefetches the K/V rows of the spans this many steps ahead of
// the ones it loads into the ring into L2 (bulk prefetch): their page walks
// and DRAM latency overlap without shared memory.  148 CTAs x 8 spans x 64 KB
// = 76 MB stays well inside the 126 MB L2.
constexpr int kPrefetchAhead = 8;
constexpr uint32_t kHalfSpanBytes = 128 * 128 * 2;  // K (or V) of one span

// ---------------------------------------------------------------- selection
// One cluster of kSelCluster CTAs per (retrieval head, sequence).  CTA r of
// the cluster scores its slice of the candidate blocks (one or two per
// thread, one round of loads) and keeps its local top-k (radix select +
// ordered compaction); the union of the local top-k lists holds the global
// top-k.  After a cluster barrier CTA 0 gathers the lists from its peers'
// shared memory, in slice order (= block order), and selects the final top-k
// by the same rule, so ties still go to the lower block index.
constexpr int kSelCluster = 8;
constexpr int kDecSelThreads = 128;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// (No memory clobber: the loads of a gather may all be in flight together;
// they are ordered after the cluster barrier, whose asm clobbers memory.)
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// All threads of every CTA in the cluster: prior shared-memory writes become
// visible to the peers (release/acquire).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint64_t ld_cluster_u64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}

// Top-k for k <= 32 on bitonic networks over the lanes of a warp.  A
// candidate is the 64-bit key (order_key(score) << 32) | ~block: keys are
// unique, and a larger key means a larger score or, for equal scores, a
// lower block index -- the selection order.  0 is below every candidate.
__device__ __forceinline__ uint64_t cand_key(float score, int block) {
  return (static_cast<uint64_t>(order_key(score)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(block));
}
__device__ __forceinline__ int cand_block(uint64_t key) { return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key)); }

// Two independent bitonic sorts of 32 keys (one per lane each), descending.
__device__ __forceinline__ void warp_sort2_desc(uint64_t& x, uint64_t& y) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t ox = __shfl_xor_sync(0xffffffffu, x, stride);
      const uint64_t oy = __shfl_xor_sync(0xffffffffu, y, stride);
      const bool take_max = ((lane & stride) == 0) == ((lane & size) == 0);
      x = take_max ? max(x, ox) : min(x, ox);
      y = take_max ? max(y, oy) : min(y, oy);
    }
  }
}

// x and y each sorted descending over the lanes: the 32 largest of the 64,
// sorted descending (bitonic split against the reversed y, then merge).
__device__ __forceinline__ uint64_t warp_merge_top32(uint64_t x, uint64_t y) {
  const int lane = threadIdx.x & 31;
  uint64_t v = max(x, __shfl_sync(0xffffffffu, y, 31 - lane));
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, v, stride);
    v = (lane & stride) == 0 ? max(v, o) : min(v, o);
  }
  return v;
}

// Bitonic sort of 32 values (one per lane), ascending.
__device__ __forceinline__ uint32_t warp_sort_asc(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool take_min = ((lane & stride) == 0) == ((lane & size) == 0);
      v = take_min ? min(v, o) : max(v, o);
    }
  }
  return v;
}

// Block of the new token, and the number of spans every retrieval head
// visits whatever the scores: the sink and the local blocks {0} u {t-L+1..t},
// or, for clustered heads, the sink block and the unclustered tail
// [clu_end, cache_len) in 128-key pieces.
__device__ __forceinline__ int decode_t(const DecodeArgs& a) { return (a.cache_len - 1) / a.block; }
__device__ __forceinline__ int n_fixed(const DecodeArgs& a) {
  return a.clustered ? 1 + (a.cache_len - a.clu_end + 127) / 128 : min(decode_t(a) + 1, a.n_local + 1);
}

// Entries of a full selection row besides the topk picks out[1..topk]: the
// sink marker, then the local blocks (contiguous mode) or nothing (clustered
// mode, whose sink and tail spans need no entry); -1 after; and the count
// the attention launch reads (n_fixed + topk).
__device__ __forceinline__ void finish_selection(const DecodeArgs& a, int32_t* out, int t, size_t bk, int tid) {
  const int n_loc = a.clustered ? 0 : a.n_local;
  if (tid == 0) out[0] = 0;
  for (int m = tid; m < n_loc; m += kDecSelThreads) out[1 + a.topk + m] = t - a.n_local + 1 + m;
  for (int e = 1 + a.topk + n_loc + tid; e < a.kmax; e += kDecSelThreads) out[e] = -1;
  if (tid == 0) a.cnt[bk] = a.clustered ? n_fixed(a) + a.topk : 1 + a.topk + a.n_local;
}

__global__ void __launch_bounds__(kDecSelThreads, 8) __cluster_dims__(kSelCluster, 1, 1)
    decode_select_kernel(const __grid_constant__ DecodeArgs a) {
  // dynamic: keys[chunk] | lkey[topk] | lidx[topk] | ukey[kSelCluster*topk] | uidx[kSelCluster*topk]
  extern __shared__ uint32_t dsel[];
  __shared__ SelectScratchT<kDecSelThreads> sh;
  __shared__ float qpart[kDecSelThreads / 32][kRank];
  __shared__ int n_kept;
  __shared__ uint64_t wlist[kDecSelThreads / 32][32];  // per-warp top-32 lists
  __shared__ uint64_t cta_top[32];                      // this CTA's top-32, read by CTA 0
  const int kvh = blockIdx.x / kSelCluster, b = blockIdx.y;
  // The attention launch that follows may start now: its window-head spans
  // do not need the selection; its retrieval spans wait for this grid.
  griddep_launch_dependents();
  if (a.kind[kvh] != KIND_SPARSE) return;  // the whole cluster leaves
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int t = (a.cache_len - 1) / a.block;
  const size_t bk = static_cast<size_t>(b) * a.n_kv_heads + kvh;
  // Candidates: blocks 1..t-L (candidate x is block x + 1, centroid row
  // x + 1), or the chunks 0..n_chunks-1 of a clustered head (row x).
  const int crow0 = a.clustered ? 0 : 1;
  const int ncand = a.clustered ? min(max(a.n_chunks[bk], 0), a.max_chunks) : max(0, t - a.n_local);
  int32_t* out = a.sel + bk * a.kmax;
  if (a.clustered && (ncand <= a.topk || a.topk == 0)) {  // every chunk (or none)
    if (rank == 0) {
      const int m = min(ncand, a.topk);
      for (int e = tid; e < a.kmax; e += kDecSelThreads) out[e] = e == 0 ? 0 : (e <= m ? e - 1 : -1);
      if (tid == 0) a.cnt[bk] = n_fixed(a) + m;
    }
    return;
  }
  if (ncand <= a.topk) {  // every block 0..t (uniform over the cluster)
    if (rank == 0) {
      for (int e = tid; e < a.kmax; e += kDecSelThreads) out[e] = e <= t ? e : -1;
      if (tid == 0) a.cnt[bk] = t + 1;
    }
    return;
  }
  if (a.topk == 0) {  // sink and local blocks only
    if (rank == 0) {
      for (int e = tid; e < a.kmax; e += kDecSelThreads)
        out[e] = e == 0 ? 0 : (e <= a.n_local ? t - a.n_local + e : -1);
      if (tid == 0) a.cnt[bk] = 1 + a.n_local;
    }
    return;
  }
  const int chunk = (ncand + kSelCluster - 1) / kSelCluster;
  const int lo = static_cast<int>(rank) * chunk;  // candidate x -> block x + 1
  const int nl = max(0, min(ncand, lo + chunk) - lo);
  uint32_t* keys = dsel;
  uint32_t* lkey = keys + chunk;
  uint32_t* lidx = lkey + a.topk;
  uint32_t* ukey = lidx + a.topk;
  uint32_t* uidx = ukey + kSelCluster * a.topk;
  const float* C = a.clustered ? a.chunk_centroids + bk * a.max_chunks * kRank : a.centroids + bk * a.nbc * kRank;

  // Loads first: this thread's first two centroid rows, its query dimension
  // of the group's heads and its row of the projector.
  float4 cv[2][4];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int x = min(lo + min(tid + u * kDecSelThreads, max(nl - 1, 0)), ncand - 1);  // a valid row
    const float4* c4 = reinterpret_cast<const float4*>(C + static_cast<size_t>(x + crow0) * kRank);
#pragma unroll
    for (int w = 0; w < 4; ++w) cv[u][w] = __ldg(c4 + w);
  }
  float4 pr[4];
  {
    const float4* p4 = reinterpret_cast<const float4*>(a.proj + tid * kRank);
#pragma unroll
    for (int w = 0; w < 4; ++w) pr[w] = __ldg(p4 + w);
  }
  // qbar = P^T (sum_h q_h): thread d sums dimension d over the group's heads
  // (fixed order), multiplies by row d of P, and the 128 rows are added by a
  // warp butterfly and then over the four warps (fixed order).
  float q[kRank];
  {
    const __nv_bfloat16* qg = a.q + (static_cast<size_t>(b) * a.n_q_heads + kvh * a.group) * kHeadDim + tid;
    // The group's values of this dimension are loaded eight at a time, all
    // in flight together (one memory round trip per eight heads rather than
    // one per head), then added in head order.
    float qs = 0.f;
    for (int h0 = 0; h0 < a.group; h0 += 8) {
      float qv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) qv[u] = h0 + u < a.group ? __bfloat162float(qg[(h0 + u) * kHeadDim]) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (h0 + u < a.group) qs += qv[u];
    }
    const float prow[kRank] = {pr[0].x, pr[0].y, pr[0].z, pr[0].w, pr[1].x, pr[1].y, pr[1].z, pr[1].w,
                               pr[2].x, pr[2].y, pr[2].z, pr[2].w, pr[3].x, pr[3].y, pr[3].z, pr[3].w};
#pragma unroll
    for (int c = 0; c < kRank; ++c) {
      float v = prow[c] * qs;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) qpart[warp][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kRank; ++c) q[c] = (qpart[0][c] + qpart[1][c]) + (qpart[2][c] + qpart[3][c]);
  }
  if (a.topk <= 32) {
    // Warp w holds candidates x0 + 32w + lane and x0 + 128 + 32w + lane of
    // each round; it keeps a running top-32 (sorted descending) of them.
    uint64_t best = 0;
    for (int x0 = 0; x0 < nl; x0 += 2 * kDecSelThreads) {
      if (x0 > 0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int x = lo + min(x0 + tid + u * kDecSelThreads, nl - 1);
          const float4* c4 = reinterpret_cast<const float4*>(C + static_cast<size_t>(x + crow0) * kRank);
#pragma unroll
          for (int w = 0; w < 4; ++w) cv[u][w] = __ldg(c4 + w);
        }
      }
      const int xa = x0 + tid, xb = x0 + tid + kDecSelThreads;
      uint64_t ka = xa < nl ? cand_key(score16(q, cv[0]), lo + xa + crow0) : 0ull;
      uint64_t kb = xb < nl ? cand_key(score16(q, cv[1]), lo + xb + crow0) : 0ull;
      warp_sort2_desc(ka, kb);
      const uint64_t top = warp_merge_top32(ka, kb);
      best = x0 == 0 ? top : warp_merge_top32(best, top);
    }
    // the four warps' lists -> the CTA's top-32
    wlist[warp][lane] = best;
    __syncthreads();
    uint64_t v = 0;
    if (warp < 2) v = warp_merge_top32(wlist[2 * warp][lane], wlist[2 * warp + 1][lane]);
    __syncthreads();
    if (warp < 2) wlist[warp][lane] = v;
    __syncthreads();
    if (warp == 0) cta_top[lane] = warp_merge_top32(wlist[0][lane], wlist[1][lane]);
    cluster_sync();  // every CTA's top-32 is complete and visible to CTA 0
    if (rank != 0) {
      cluster_sync();  // CTA 0 has read the list
      return;
    }
    // CTA 0: warp w merges the lists of CTAs 2w and 2w+1, then two rounds
    // of merges in shared memory.
    v = warp_merge_top32(ld_cluster_u64(map_to_rank(smem_u32(&cta_top[lane]), 2 * warp)),
                         ld_cluster_u64(map_to_rank(smem_u32(&cta_top[lane]), 2 * warp + 1)));
    wlist[warp][lane] = v;
    __syncthreads();
    cluster_sync();  // the peers may leave: their lists have been read
    if (warp < 2) v = warp_merge_top32(wlist[2 * warp][lane], wlist[2 * warp + 1][lane]);
    __syncthreads();
    if (warp < 2) wlist[warp][lane] = v;
    __syncthreads();
    if (warp == 0) {
      v = warp_merge_top32(wlist[0][lane], wlist[1][lane]);
      // the first topk keys are the selection; put their blocks in order
      const uint32_t blk = lane < a.topk ? static_cast<uint32_t>(cand_block(v)) : 0xFFFFFFFFu;
      const uint32_t sorted = warp_sort_asc(blk);
      if (lane < a.topk) out[1 + lane] = static_cast<int32_t>(sorted);
    }
    finish_selection(a, out, t, bk, tid);
    return;
  }
  // k > 32: radix select.  Scores of this CTA's slice -> order keys.
  for (int x0 = 0; x0 < nl; x0 += 2 * kDecSelThreads) {
    if (x0 > 0) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int x = lo + min(x0 + tid + u * kDecSelThreads, nl - 1);
        const float4* c4 = reinterpret_cast<const float4*>(C + static_cast<size_t>(x + crow0) * kRank);
#pragma unroll
        for (int w = 0; w < 4; ++w) cv[u][w] = __ldg(c4 + w);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int x = x0 + tid + u * kDecSelThreads;
      if (x < nl) keys[x] = order_key(score16(q, cv[u]));
    }
  }
  __syncthreads();
  // Local top-k of the slice (all of it if it is small).
  if (nl <= a.topk) {
    for (int x = tid; x < nl; x += kDecSelThreads) {
      lkey[x] = keys[x];
      lidx[x] = static_cast<uint32_t>(lo + x + crow0);
    }
    if (tid == 0) n_kept = nl;
  } else {
    uint32_t T, need;
    radix_threshold<kDecSelThreads>(keys, nl, a.topk, sh, T, need);
    ordered_select<kDecSelThreads>(keys, nl, T, need, sh, [&](int r, int x) {
      lkey[r] = keys[x];
      lidx[r] = static_cast<uint32_t>(lo + x + crow0);
    });
    if (tid == 0) n_kept = a.topk;
  }
  cluster_sync();  // local lists complete and visible to CTA 0
  if (rank == 0) {
    int off[kSelCluster + 1];
    off[0] = 0;
#pragma unroll
    for (int r = 0; r < kSelCluster; ++r)
      off[r + 1] = off[r] + static_cast<int>(ld_cluster_u32(map_to_rank(smem_u32(&n_kept), r)));
    for (int e0 = 0; e0 < a.topk; e0 += kDecSelThreads) {
      const int e = e0 + tid;
      uint32_t vk[kSelCluster], vi[kSelCluster];
#pragma unroll
      for (int r = 0; r < kSelCluster; ++r) {  // all loads first, then the stores
        const bool in = e < off[r + 1] - off[r];
        vk[r] = in ? ld_cluster_u32(map_to_rank(smem_u32(lkey + e), r)) : 0u;
        vi[r] = in ? ld_cluster_u32(map_to_rank(smem_u32(lidx + e), r)) : 0u;
      }
#pragma unroll
      for (int r = 0; r < kSelCluster; ++r) {
        if (e < off[r + 1] - off[r]) {
          ukey[off[r] + e] = vk[r];
          uidx[off[r] + e] = vi[r];
        }
      }
    }
    __syncthreads();
    cluster_sync();  // the peers may leave: their lists have been read
    const int U = off[kSelCluster];
    uint32_t T, need;
    radix_threshold<kDecSelThreads>(ukey, U, a.topk, sh, T, need);
    ordered_select<kDecSelThreads>(ukey, U, T, need, sh,
                                   [&](int r, int x) { out[1 + r] = static_cast<int32_t>(uidx[x]); });
    finish_selection(a, out, t, bk, tid);
  } else {
    cluster_sync();
  }
}

// Dynamic shared memory of the selection kernel (host side).
size_t decode_select_smem(const DecodeArgs& a) {
  if (a.topk <= 32) return 0;  // static arrays suffice
  const int t = (a.cache_len - 1) / a.block;
  const int ncand = a.clustered ? a.max_chunks : std::max(0, t - a.n_local);
  const int chunk = (ncand + kSelCluster - 1) / kSelCluster;
  return (static_cast<size_t>(chunk) + 2 * static_cast<size_t>(a.topk) * (1 + kSelCluster)) * sizeof(uint32_t);
}

// ---------------------------------------------------------------- schedule

// Spans of one (sequence, head) in a list: list 0 holds a window/full head's
// visible keys in 128-key pieces, or a retrieval head's sink and local
// blocks; list 1 holds the rest of a retrieval head's kmax selected blocks.
__device__ __forceinline__ int n_spans_in(const DecodeArgs& a, int list, int kvh) {
  const int kind = a.kind[kvh];
  if (kind == KIND_SPARSE) return list == 0 ? n_fixed(a) : a.kmax - n_fixed(a);
  if (list == 1) return 0;
  const int len = kind == KIND_SWA ? min(a.cache_len, a.window) : a.cache_len;
  return (len + 127) / 128;
}

// Fixed block s (0 <= s < n_fixed) of a retrieval head in contiguous mode, ascending.
__device__ __forceinline__ int fixed_block(const DecodeArgs& a, int s) {
  const int t = decode_t(a);
  return (t <= a.n_local || s == 0) ? s : t - a.n_local + s;
}

__device__ __forceinline__ long list_len(const DecodeArgs& a, int list) {
  return static_cast<long>(a.batch) * a.per_b[list];
}

// First span of CTA c in a list of length n: floor(c * n / n_ctas).
__device__ __forceinline__ long range_lo(const DecodeArgs& a, long n, int c) {
  return static_cast<long>((static_cast<long long>(c) * n) / a.n_ctas);
}

// The CTA whose range holds span x: the largest c with range_lo(c) <= x.
__device__ __forceinline__ int owner_of(const DecodeArgs& a, long n, long x) {
  return static_cast<int>(((static_cast<long long>(x) + 1) * a.n_ctas - 1) / n);
}

// Span x of a list -> (sequence, head, span index within the head's part).
__device__ __forceinline__ void locate(const DecodeArgs& a, int list, long x, int& b, int& kvh, int& s) {
  b = static_cast<int>(x / a.per_b[list]);
  const int r = static_cast<int>(x - static_cast<long>(b) * a.per_b[list]);
  kvh = 0;
  s = 0;
  for (int h = 0; h < a.n_kv_heads; ++h) {
    const int off = a.span_off[list][h];
    if (r >= off && r < off + n_spans_in(a, list, h)) {
      kvh = h;
      s = r - off;
      return;
    }
  }
}

// Partial-result slot of the run that starts at span x of a list.
__device__ __forceinline__ float* run_partial(const DecodeArgs& a, int list, long x) {
  const long slot = (list == 1 ? list_len(a, 0) : 0) + x;
  return a.partial + slot * a.group * kPartStride;
}

// --------------------------------------------------------------- attention
struct __align__(1024) DecSmem {
  uint8_t k[kRingStages][kHalfSpanBytes];  // 128 keys x 128 dims: two 64-column SW128 chunks
  uint8_t v[kRingStages][kHalfSpanBytes];
  float wo[kConsumerWarps][kHeadDim][8];   // run-end merge: each warp's O^T for 8 heads
  float wm[kConsumerWarps][8], wl[kConsumerWarps][8];
  uint64_t k_full[kRingStages], v_full[kRingStages], empty[kRingStages];
  int nk[kRingStages];                     // valid keys of the span in each stage
  int abort_flag;
};
constexpr size_t kDecSmemBytes = sizeof(DecSmem) + 1024;  // + alignment slack
static_assert(kDecSmemBytes <= 210 * 1024, "leave room for a selection CTA on the same SM");

__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int dim) {
  return base + (dim >> 6) * 16384 + row * 128 + ((((dim & 63) >> 3) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}

// Producer warp: walks the CTA's spans in consumption order and streams K
// and V of each into the ring (four 64x64 boxes each, 128-byte swizzle; rows
// past the cache read as zero).  The spans are taken 32 at a time: lane l
// works out the key range of span l of the chunk (reading the selection for
// retrieval spans), lanes prefetch the rows of the spans kPrefetchAhead ahead
// into L2, and lane 0 waits for free stages and issues the loads.
__device__ __forceinline__ void attn_producer(DecSmem& sm, const CUtensorMap* mk, const CUtensorMap* mv,
                                              const CUtensorMap* mks, const CUtensorMap* mvs, const DecodeArgs& a,
                                              volatile int* abort) {
  const int lane = lane_id();
  const int tq = (a.cache_len - 1) / a.block;  // block of the new token
  uint32_t issued = 0;
  bool ok = true;
  for (int list = 0; list < 2 && ok; ++list) {
    const long n = list_len(a, list);
    if (n == 0) continue;
    if (list == 1) griddep_wait();  // the selection is complete and visible
    const long hi = range_lo(a, n, blockIdx.x + 1);
    long x = range_lo(a, n, blockIdx.x);
    while (x < hi && ok) {
      int b, kvh, s;
      locate(a, list, x, b, kvh, s);
      const int nsp = n_spans_in(a, list, kvh);
      const long run_end = min(hi, x - s + nsp);
      const size_t bk = static_cast<size_t>(b) * a.n_kv_heads + kvh;
      // list 1: the first cnt - n_fixed of the head's spans hold selected blocks
      const int cnt = list == 1 ? max(0, min(a.cnt[bk], a.kmax) - n_fixed(a)) : nsp;
      const int s_end = min(s + static_cast<int>(run_end - x), cnt);
      const bool sparse = a.kind[kvh] == KIND_SPARSE;
      const int start = a.kind[kvh] == KIND_SWA ? max(0, a.cache_len - a.window) : 0;
      // clustered list-1 spans come from the cluster-ordered K/V, or are
      // gathered row by row from the cache (member rows, in place)
      const bool gather_src = a.clustered && a.gather && list == 1;
      const bool sorted_src = a.clustered && !a.gather && list == 1;
      const __nv_bfloat16* kbase = sorted_src ? a.k_sorted + bk * static_cast<size_t>(a.clu_rows) * kHeadDim
                                              : a.kcache + bk * static_cast<size_t>(a.cache_cap) * kHeadDim;
      const __nv_bfloat16* vbase = sorted_src ? a.v_sorted + bk * static_cast<size_t>(a.clu_rows) * kHeadDim
                                              : a.vcache + bk * static_cast<size_t>(a.cache_cap) * kHeadDim;
      // (no L2 prefetch for gathered spans: their rows are not contiguous)
      const int src_rows = gather_src ? 0 : (sorted_src ? a.clu_rows : a.cache_len);
      const CUtensorMap* tk = sorted_src ? mks : mk;
      const CUtensorMap* tv = sorted_src ? mvs : mv;
      for (int s0 = s; s0 < s_end && ok; s0 += 32) {
        const int m = min(32, s_end - s0);
        // lane l: key range of span s0 + l
        int key0_l = 0, nk_l = 0;
        if (lane < m) {
          if (list == 1 && a.clustered) {
            const int ch = a.sel[bk * a.kmax + 1 + s0 + lane];  // a chunk of the head's clusters
            if (ch < 0 || ch >= min(a.n_chunks[bk], a.max_chunks)) {
              flag_error(a.status, RTP_DEVERR_INDEX);
            } else {
              const size_t e = bk * a.max_chunks + ch;
              key0_l = a.chunk_start[e];
              nk_l = min(a.chunk_len[e], a.clu_rows - key0_l);
              if (key0_l < 0 || nk_l < 0) {
                flag_error(a.status, RTP_DEVERR_INDEX);
                key0_l = nk_l = 0;
              }
            }
          } else if (list == 1) {
            const int blk = a.sel[bk * a.kmax + 1 + s0 + lane];  // the sink is entry 0
            if (blk < 0 || blk > tq) {  // not a valid selection: the span contributes nothing
              flag_error(a.status, RTP_DEVERR_INDEX);
            } else {
              key0_l = blk * a.block;
              nk_l = min(a.block, a.cache_len - key0_l);
            }
          } else if (sparse && a.clustered) {  // the sink block, then the unclustered tail
            const int sp = s0 + lane;
            key0_l = sp == 0 ? 0 : a.clu_end + 128 * (sp - 1);
            nk_l = sp == 0 ? min(a.block, a.cache_len) : min(128, a.cache_len - key0_l);
          } else if (sparse) {
            key0_l = fixed_block(a, s0 + lane) * a.block;
            nk_l = min(a.block, a.cache_len - key0_l);
          } else {
            key0_l = start + 128 * (s0 + lane);
            nk_l = min(128, a.cache_len - key0_l);
          }
        }
        // rows the ring load will read: 128 from key0, within the cache
        const uint32_t pf_bytes = static_cast<uint32_t>(max(0, min(128, src_rows - key0_l))) * kHeadDim * 2;
        auto prefetch_span = [&]() {
          if (pf_bytes > 0) {
            prefetch_l2(kbase + static_cast<size_t>(key0_l) * kHeadDim, pf_bytes);
            prefetch_l2(vbase + static_cast<size_t>(key0_l) * kHeadDim, pf_bytes);
          }
        };
        if (lane < min(m, kPrefetchAhead)) prefetch_span();
        for (int i = 0; i < m; ++i) {
          const int key0 = __shfl_sync(0xffffffffu, key0_l, i);
          const int nk = __shfl_sync(0xffffffffu, nk_l, i);
          if (lane == i + kPrefetchAhead && lane < m) prefetch_span();
          const uint32_t st = issued % kRingStages, ph = (issued / kRingStages) & 1u;
          int okl = 1;
          if (gather_src) {
            // The chunk's member rows, gathered from the cache with 16-byte
            // cp.async copies into the consumers' 128-byte-swizzled layout
            // (sw128): lanes 0-15 copy row 2i's sixteen 16-byte pieces, lanes
            // 16-31 row 2i+1's.  Rows past the chunk repeat its first member
            // (masked by nk).  Each lane's copies complete on the stage's
            // barriers (cp.async.mbarrier.arrive raises their pending count
            // when issued); lane 0's plain arrive is the phase's own arrival.
            if (lane == 0) okl = mbar_wait(&sm.empty[st], ph ^ 1u, abort, a.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
            if (!ok) break;
            if (lane == 0) sm.nk[st] = nk;
            // lane l loads the positions of rows 4l .. 4l+3 (all four in flight)
            const int32_t* mem = a.members + bk * static_cast<size_t>(a.clu_rows) + key0;
            int pv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) pv[u] = mem[4 * lane + u < nk ? 4 * lane + u : 0];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (pv[u] < 0 || pv[u] >= a.cache_len) {  // not a cached row: recorded, row 0 read instead
                flag_error(a.status, RTP_DEVERR_INDEX);
                pv[u] = 0;
              }
            const int hi = lane >> 4, piece = lane & 15;
            const uint32_t ks = smem_u32(sm.k[st]), vs = smem_u32(sm.v[st]);
            const __nv_bfloat16* kslab = a.kcache + bk * static_cast<size_t>(a.cache_cap) * kHeadDim + 8 * piece;
            const __nv_bfloat16* vslab = a.vcache + bk * static_cast<size_t>(a.cache_cap) * kHeadDim + 8 * piece;
#pragma unroll 4
            for (int k2 = 0; k2 < 64; ++k2) {
              // rows 2 k2 (lanes 0-15) and 2 k2 + 1 (lanes 16-31): held by
              // lane k2 / 2 in registers 2 (k2 & 1) and 2 (k2 & 1) + 1
              const int e0 = __shfl_sync(0xffffffffu, (k2 & 1) ? pv[2] : pv[0], k2 >> 1);
              const int e1 = __shfl_sync(0xffffffffu, (k2 & 1) ? pv[3] : pv[1], k2 >> 1);
              const int r = 2 * k2 + hi;
              const size_t off = static_cast<size_t>(hi ? e1 : e0) * kHeadDim;
              cp_async16(sw128(ks, r, 8 * piece), kslab + off);
              cp_async16(sw128(vs, r, 8 * piece), vslab + off);
            }
            cp_async_arrive(&sm.k_full[st]);
            cp_async_arrive(&sm.v_full[st]);
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&sm.k_full[st]);
              mbar_arrive(&sm.v_full[st]);
            }
            ++issued;
            continue;
          }
          if (lane == 0) {
            okl = mbar_wait(&sm.empty[st], ph ^ 1u, abort, a.status) ? 1 : 0;
            if (okl) {
              sm.nk[st] = nk;
              mbar_arrive_expect_tx(&sm.k_full[st], kHalfSpanBytes);
              for (int cc = 0; cc < 2; ++cc)
                for (int hh = 0; hh < 2; ++hh)
                  tma_load_3d(sm.k[st] + cc * 16384 + hh * 8192, tk, &sm.k_full[st], 64 * cc, key0 + 64 * hh,
                              static_cast<int>(bk));
              mbar_arrive_expect_tx(&sm.v_full[st], kHalfSpanBytes);
              for (int cc = 0; cc < 2; ++cc)
                for (int hh = 0; hh < 2; ++hh)
                  tma_load_3d(sm.v[st] + cc * 16384 + hh * 8192, tv, &sm.v_full[st], 64 * cc, key0 + 64 * hh,
                              static_cast<int>(bk));
            }
          }
          ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
          if (!ok) break;
          ++issued;
        }
      }
      x = run_end;
    }
  }
  // Wait (bounded) for the copies that may still be in flight so that no TMA
  // write lands in shared memory after the CTA has exited.
  if (lane == 0) {
    for (uint32_t d = 0; d < kRingStages && d < issued; ++d) {
      const uint32_t e = issued - 1 - d;
      mbar_wait(&sm.k_full[e % kRingStages], (e / kRingStages) & 1u, nullptr, a.status);
      mbar_wait(&sm.v_full[e % kRingStages], (e / kRingStages) & 1u, nullptr, a.status);
    }
  }
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// All lanes of the warp wait (bounded) for a phase: lane 0 polls, then every
// lane tests the completed phase once for its own acquire.  Uniform result.
__device__ __forceinline__ bool warp_phase_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                uint32_t* status) {
  int ok = 1;
  if (lane_id() == 0) ok = mbar_wait(bar, parity, abort, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_test(bar, parity);
  return ok != 0;
}

// Named barrier over the 128 consumer threads (the producer warp never
// joins it).
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory");
}

// Consumer warps 0-3, each on its own: warp w takes keys [32w, 32w+32) of
// every span and keeps its own running maximum, row sums and O for them
// (flash-decoding inside the CTA); the four warps merge at the end of a run
// through shared memory and the consumers' named barrier.  A warp whose
// bounded wait gives up does not leave early: it walks the rest of the
// schedule without waiting or computing, so every warp reaches every named
// barrier and none can be left waiting at one.
// The MMAs are transposed so that no row is padding: S^T = K Q^T with the 16
// keys of an m16n8k16 tile as M and 8 query heads as N (NT tiles of 8 heads
// for a group of up to 8 NT), then O^T += V^T P^T with 16 head dims as M,
// where P^T comes straight from the S^T accumulators: each 8x8 block of
// (key, head) values is transposed in registers (movmatrix) into the B
// fragment layout.  Per span and warp: 16 NT MMAs for S^T and 16 NT for O^T.
template <int NT>
__device__ __forceinline__ void attn_consumer(DecSmem& sm, const DecodeArgs& a, volatile int* abort) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = a.group;
  const float sl2 = a.scale_log2;
  const int kbase = 32 * warp;
  uint32_t used = 0;  // spans consumed
  bool dead = false;  // a wait gave up: no more waits or work, barriers only
  for (int list = 0; list < 2; ++list) {
    const long n = list_len(a, list);
    if (n == 0) continue;
    if (list == 1) griddep_wait();
    const long hi = range_lo(a, n, blockIdx.x + 1);
    long x = range_lo(a, n, blockIdx.x);
    while (x < hi) {
      int b, kvh, s;
      locate(a, list, x, b, kvh, s);
      const int nsp = n_spans_in(a, list, kvh);
      const long run_start = x, run_end = min(hi, x - s + nsp);
      const size_t bk = static_cast<size_t>(b) * a.n_kv_heads + kvh;
      const int cnt = list == 1 ? max(0, min(a.cnt[bk], a.kmax) - n_fixed(a)) : nsp;
      const int s_end = min(s + static_cast<int>(run_end - x), cnt);
      // Q^T as B fragments: lane (g, c) holds head 8nt+g, dims 16kk+2c(+1)
      // and 16kk+2c+8(+9); zero for heads beyond the group.
      uint32_t qb[NT][8][2];
      {
        const __nv_bfloat16* qg = a.q + (static_cast<size_t>(b) * a.n_q_heads + kvh * G) * kHeadDim;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int head = 8 * nt + g;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const __nv_bfloat16* qr = qg + head * kHeadDim + 16 * kk + 2 * c;
            qb[nt][kk][0] = head < G ? *reinterpret_cast<const uint32_t*>(qr) : 0u;
            qb[nt][kk][1] = head < G ? *reinterpret_cast<const uint32_t*>(qr + 8) : 0u;
          }
        }
      }
      // running state of heads 8nt+2c and 8nt+2c+1 over this warp's keys
      float m_run[NT][2], l_run[NT][2];
      float oacc[NT][8][4];  // O^T tile dt: dims 16dt+g (+8), heads 8nt+2c (+1)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) oacc[nt][dt][0] = oacc[nt][dt][1] = oacc[nt][dt][2] = oacc[nt][dt][3] = 0.f;
      }
      for (; s < s_end; ++s, ++used) {
        const uint32_t st = used % kRingStages, ph = (used / kRingStages) & 1u;
        if (dead || !warp_phase_wait(&sm.k_full[st], ph, abort, a.status)) {
          dead = true;
          continue;
        }
        const int nk = sm.nk[st];
        const uint32_t ks = smem_u32(sm.k[st]), vs = smem_u32(sm.v[st]);
        // S^T: tile mt holds keys kbase+16mt+g (rows d0,d1) and +8 (d2,d3);
        // even and odd dim steps accumulate separately (chains of 4)
        float sacc[NT][2][4], sac2[NT][2][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[nt][mt][e] = sac2[nt][mt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            uint32_t ra[4];
            const int key = kbase + 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int dim = 16 * kk + (lane >> 4) * 8;
            ldsm_x4(sw128(ks, key, dim), ra);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              float (&acc)[4] = (kk & 1) ? sac2[nt][mt] : sacc[nt][mt];
              mma_bf16(acc, ra, qb[nt][kk][0], qb[nt][kk][1]);
            }
          }
        }
        // scale, mask, per-head maximum over the warp's 32 keys
        float mw[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mw[nt][0] = mw[nt][1] = -INFINITY;
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int key = kbase + 16 * mt + g + 8 * (e >> 1);
              const float v = key < nk ? (sacc[nt][mt][e] + sac2[nt][mt][e]) * sl2 : -INFINITY;
              sacc[nt][mt][e] = v;
              mw[nt][e & 1] = fmaxf(mw[nt][e & 1], v);
            }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            mw[nt][hh] = fmaxf(mw[nt][hh], __shfl_xor_sync(0xffffffffu, mw[nt][hh], 4));
            mw[nt][hh] = fmaxf(mw[nt][hh], __shfl_xor_sync(0xffffffffu, mw[nt][hh], 8));
            mw[nt][hh] = fmaxf(mw[nt][hh], __shfl_xor_sync(0xffffffffu, mw[nt][hh], 16));
          }
        }
        // running maximum, rescale of O and l, P = exp2(S - m) as B fragments
        uint32_t pb[NT][2][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float mref[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float m_new = fmaxf(m_run[nt][hh], mw[nt][hh]);
            mref[hh] = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = exp2f(m_run[nt][hh] - mref[hh]);  // 0 while nothing was visible
            m_run[nt][hh] = m_new;
            l_run[nt][hh] *= alpha;
#pragma unroll
            for (int dt = 0; dt < 8; ++dt) {
              oacc[nt][dt][hh] *= alpha;
              oacc[nt][dt][2 + hh] *= alpha;
            }
          }
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const float p0 = exp2f(sacc[nt][mt][0] - mref[0]), p1 = exp2f(sacc[nt][mt][1] - mref[1]);
            const float p2 = exp2f(sacc[nt][mt][2] - mref[0]), p3 = exp2f(sacc[nt][mt][3] - mref[1]);
            l_run[nt][0] += p0 + p2;
            l_run[nt][1] += p1 + p3;
            // (key g, heads 2c..2c+1) and (key g+8, ...) -> (keys 2c..2c+1, head g), (keys 2c+8.., head g)
            pb[nt][mt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
            pb[nt][mt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
          }
        }
        if (!warp_phase_wait(&sm.v_full[st], ph, abort, a.status)) {
          dead = true;
          continue;
        }
        // O^T += V^T P^T: A = V^T tile (dims 16dt.., keys 16mt..) by ldmatrix.trans
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            uint32_t ra[4];
            const int key = kbase + 16 * mt + (lane & 7) + ((lane >> 4) & 1) * 8;
            const int dim = 16 * dt + ((lane >> 3) & 1) * 8;
            ldsm_x4_t(sw128(vs, key, dim), ra);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(oacc[nt][dt], ra, pb[nt][mt][0], pb[nt][mt][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
      }
      // end of the run: merge the four warps, 8 heads at a time
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float lsum[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v = l_run[nt][hh];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          lsum[hh] = v;
        }
        if (g == 0) {
          sm.wm[warp][2 * c] = m_run[nt][0];
          sm.wm[warp][2 * c + 1] = m_run[nt][1];
          sm.wl[warp][2 * c] = lsum[0];
          sm.wl[warp][2 * c + 1] = lsum[1];
        }
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
          *reinterpret_cast<float2*>(&sm.wo[warp][16 * dt + g][2 * c]) = make_float2(oacc[nt][dt][0], oacc[nt][dt][1]);
          *reinterpret_cast<float2*>(&sm.wo[warp][16 * dt + g + 8][2 * c]) =
              make_float2(oacc[nt][dt][2], oacc[nt][dt][3]);
        }
        consumers_sync();  // every warp's m, l and O^T are posted
        // thread d: output dim d of the 8 heads
        float* part = run_partial(a, list, run_start);
        const int d = tid;
        for (int hh = 0; hh < 8 && 8 * nt + hh < G; ++hh) {
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.wm[w][hh]);
          float L = 0.f, o = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float f = sm.wm[w][hh] == -INFINITY ? 0.f : exp2f(sm.wm[w][hh] - M);
            L = fmaf(f, sm.wl[w][hh], L);
            o = fmaf(f, sm.wo[w][d][hh], o);
          }
          float* pr = part + (8 * nt + hh) * kPartStride;
          pr[4 + d] = o;
          if (d == 0) {
            pr[0] = M;
            pr[1] = L;
          }
        }
        consumers_sync();  // wo, wm and wl are free again
      }
      x = run_end;
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(kAttnThreads, 2) decode_attn_kernel(const __grid_constant__ CUtensorMap mk,
                                                                       const __grid_constant__ CUtensorMap mv,
                                                                       const __grid_constant__ CUtensorMap mks,
                                                                       const __grid_constant__ CUtensorMap mvs,
                                                                       const __grid_constant__ DecodeArgs a) {
  extern __shared__ uint8_t dsmem[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const int warp = warp_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.empty[i], kConsumerWarps);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // The combine launch may be scheduled now; it waits for this grid.
  griddep_launch_dependents();
  volatile int* abort = &sm.abort_flag;
  if (warp == kConsumerWarps) {
    if (lane_id() == 0) {
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      if (a.clustered) {
        tma_prefetch_desc(&mks);
        tma_prefetch_desc(&mvs);
      }
    }
    attn_producer(sm, &mk, &mv, &mks, &mvs, a, abort);
  } else {
    attn_consumer<NT>(sm, a, abort);
  }
}

// Log-sum-exp merge of the runs of one query head.  In each list, the runs
// of (sequence, head) are those of the CTAs whose ranges meet the head's
// spans [x0, x1]:
// the owner of x0 (its run starts at x0) and every later CTA up to the owner
// of x1 that has work (its run starts at its range's first span).  Warp w
// merges runs w, w+4, ... (lane l: dims 4l..4l+3, four runs' loads in
// flight at a time); the four warps' results are merged in shared memory.
__device__ __forceinline__ long run_slot(const DecodeArgs& a, long n, long x0, int c0, int r) {
  if (r == 0) return x0;
  const long lo = range_lo(a, n, c0 + r);
  return lo == range_lo(a, n, c0 + r + 1) ? -1 : lo;  // -1: this CTA has no span
}

__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int kWarps = kCombineThreads / 32;
  __shared__ float wm[kWarps], wl[kWarps];
  __shared__ float4 wo[kWarps][32];
  griddep_wait();  // partials of the preceding attention launch
  const int hq = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = hq / a.group, h = hq % a.group;
  // The head's runs: those of list 0, then those of list 1 (a retrieval head
  // has spans in both; a window/full head only in list 0).
  long n0 = 0, x00 = 0, n1 = 0, x01 = 0;
  int c00 = 0, nr0 = 0, c01 = 0, nr1 = 0;
  if (const int ns = n_spans_in(a, 0, kvh); ns > 0) {
    n0 = list_len(a, 0);
    x00 = static_cast<long>(b) * a.per_b[0] + a.span_off[0][kvh];
    c00 = owner_of(a, n0, x00);
    nr0 = owner_of(a, n0, x00 + ns - 1) - c00 + 1;
  }
  if (const int ns = n_spans_in(a, 1, kvh); ns > 0) {
    n1 = list_len(a, 1);
    x01 = static_cast<long>(b) * a.per_b[1] + a.span_off[1][kvh];
    c01 = owner_of(a, n1, x01);
    nr1 = owner_of(a, n1, x01 + ns - 1) - c01 + 1;
  }
  const int nr = nr0 + nr1;
  float M = -INFINITY, L = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r0 = warp; r0 < nr; r0 += 4 * kWarps) {
    float mr[4], lr[4];
    float4 orr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = r0 + u * kWarps;
      const int list = r < nr0 ? 0 : 1;
      const long slot = r >= nr ? -1
                        : (list == 0 ? run_slot(a, n0, x00, c00, r) : run_slot(a, n1, x01, c01, r - nr0));
      mr[u] = -INFINITY;
      lr[u] = 0.f;
      orr[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (slot >= 0) {
        const float* p = run_partial(a, list, slot) + h * kPartStride;
        mr[u] = p[0];
        lr[u] = p[1];
        orr[u] = *reinterpret_cast<const float4*>(p + 4 + 4 * lane);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (mr[u] == -INFINITY) continue;  // no run, or no visible key in it
      const float mn = fmaxf(M, mr[u]);
      const float fa = exp2f(M - mn), fb = exp2f(mr[u] - mn);
      L = fmaf(L, fa, lr[u] * fb);
      o.x = fmaf(o.x, fa, orr[u].x * fb);
      o.y = fmaf(o.y, fa, orr[u].y * fb);
      o.z = fmaf(o.z, fa, orr[u].z * fb);
      o.w = fmaf(o.w, fa, orr[u].w * fb);
      M = mn;
    }
  }
  if (lane == 0) {
    wm[warp] = M;
    wl[warp] = L;
  }
  wo[warp][lane] = o;
  __syncthreads();
  // thread d: output dimension d
  const int d = tid;
  float Mt = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) Mt = fmaxf(Mt, wm[w]);
  float Lt = 0.f, ot = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float f = wm[w] == -INFINITY ? 0.f : exp2f(wm[w] - Mt);
    Lt = fmaf(f, wl[w], Lt);
    ot = fmaf(f, reinterpret_cast<const float*>(&wo[w][d >> 2])[d & 3], ot);
  }
  const float out = Lt > 0.f ? ot / Lt : 0.f;
  a.o[(static_cast<size_t>(b) * a.n_q_heads + hq) * kHeadDim + d] = __float2bfloat16_rn(out);
}

// Scratch of the allocation-free decode entry point: a file-scope device
// array that every GPU loading this library holds until the process exits,
// and the device status word its kernels report bounded-wait time-outs and
// skipped indices in (the other entry points use an allocated word).
static __device__ __align__(256) unsigned char g_decode_static_scratch[kDecodeStaticScratchBytes];
static __device__ uint32_t g_decode_static_status;

std::mutex g_static_mu;
void* g_static_scratch_addr[64] = {nullptr};
uint32_t* g_static_status_addr[64] = {nullptr};

}  // namespace

cudaError_t decode_static_scratch(void** ptr, uint32_t** status) {
  // Host code may not use the arrays' names as device addresses; look the
  // addresses up once per device, with that device current, and reuse them.
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_scratch_addr[dev]) {
    void* p = nullptr;
    void* w = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_static_scratch);
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress(&w, g_decode_static_status);
    if (e != cudaSuccess) return e;
    g_static_status_addr[dev] = static_cast<uint32_t*>(w);
    g_static_scratch_addr[dev] = p;
  }
  *ptr = g_static_scratch_addr[dev];
  *status = g_static_status_addr[dev];
  return cudaSuccess;
}

uint32_t* decode_static_status_if_used() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_static_mu);
  return g_static_status_addr[dev];
}

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mks,
                          const CUtensorMap& mvs, cudaStream_t stream) {
  // All three kernels prefer the largest shared-memory carveout: an SM that
  // a selection or combine CTA has configured for little shared memory could
  // not take an attention CTA until it drains.
  // The attention kernel is compiled for one or two tiles of 8 query heads.
  const bool two_tiles = a.group > 8;
  const void* attn = two_tiles ? reinterpret_cast<const void*>(decode_attn_kernel<2>)
                               : reinterpret_cast<const void*>(decode_attn_kernel<1>);
  for (const void* fn : {reinterpret_cast<const void*>(decode_select_kernel), attn,
                         reinterpret_cast<const void*>(decode_combine_kernel)}) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
  }
  const size_t sel_smem = decode_select_smem(a);
  if (sel_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
  }
  decode_select_kernel<<<dim3(kSelCluster * a.n_kv_heads, a.batch), kDecSelThreads, sel_smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDecSmemBytes));
  if (e != cudaSuccess) return e;
  // Programmatic dependent launches: each kernel may begin while the
  // previous one finishes; griddepcontrol.wait orders the data it reads.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_ctas);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = kDecSmemBytes;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  e = two_tiles ? cudaLaunchKernelEx(&cfg, decode_attn_kernel<2>, mk, mv, mks, mvs, a)
                : cudaLaunchKernelEx(&cfg, decode_attn_kernel<1>, mk, mv, mks, mvs, a);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(a.n_q_heads, a.batch);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel, a);
}

}  // namespace rtp
