// Fused low-rank indexer: block centroids of the keys and block summaries of
// the queries for every retrieval slot.
//
// Page "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳": a projector
// maps the D=128 features to r=16 (keeping the low-frequency rotary
// components), and clustering the projected keys lets whole groups of
// unrelated tokens be skipped; the summary of "Full Attention Strikes Back"
// calls this 16-dim indexer a cheap scout.  Here:
//   c_b    = (1/B) sum_{j in block b} P^T k_j
//   qbar_t = sum_{h in group} (1/B) sum_{i in block t} P^T q_{h,i}
// By linearity both equal P^T applied to a plain sum, so the kernel sums the
// raw 128-dim rows (fp32) and projects once per block: the work is one pass
// over K and the group's Q, i.e. HBM-bound.
//
// One CTA per (block, retrieval slot, sequence), 256 threads.  Each thread
// reads 16 bytes (8 bf16) per row; 16 threads cover a row, so a warp reads two
// full 256-byte rows per instruction (coalesced).  The 16 row-groups' partial
// sums are reduced through shared memory in a fixed order, so results are
// bit-reproducible (and equal to the KV-cache centroids of cache.cu, which
// use the same order).

#include <cuda_bf16.h>

#include "internal.cuh"
#include "row_sum.cuh"

namespace rtp {
namespace {

constexpr int kThreads = kSumThreads;
constexpr int kRowGroups = kSumRowGroups;  // rows read per pass

__global__ void __launch_bounds__(kThreads) indexer_kernel(const IndexerArgs a) {
  __shared__ float part[2][kRowGroups][kHeadDim];
  __shared__ float total[2][kHeadDim];
  __shared__ float proj[kHeadDim * kRank];

  const int blk = a.blk0 + static_cast<int>(blockIdx.x), slot = blockIdx.y, b = blockIdx.z;
  const int lrow = static_cast<int>(blockIdx.x) * a.block;  // first row of the block in the q/k arrays
  const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
  const int kvh = a.slot_heads[slot];
  const int B = a.block;

  for (int e = tid; e < kHeadDim * kRank; e += kThreads) proj[e] = a.proj[e];

  // keys of this block
  float acck[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const __nv_bfloat16* kbase =
      a.k + ((static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.rows + static_cast<size_t>(lrow)) * kHeadDim;
  sum_rows(acck, kbase, B, rg, cg);

  // queries of this block, every head of the group (heads are consecutive)
  float accq[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int h = 0; h < a.group; ++h) {
    const int hq = kvh * a.group + h;
    const __nv_bfloat16* qbase =
        a.q + ((static_cast<size_t>(b) * a.n_q_heads + hq) * a.rows + static_cast<size_t>(lrow)) * kHeadDim;
    sum_rows(accq, qbase, B, rg, cg);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    part[0][rg][cg * 8 + e] = acck[e];
    part[1][rg][cg * 8 + e] = accq[e];
  }
  __syncthreads();
  {
    const int which = tid >> 7, col = tid & 127;  // 256 threads = 2 x 128 columns
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < kRowGroups; ++g) s += part[which][g][col];
    total[which][col] = s;
  }
  __syncthreads();
  if (tid < 2 * kRank) {
    const int which = tid >> 4, c = tid & 15;
    float s = 0.f;
    for (int d = 0; d < kHeadDim; ++d) s = fmaf(proj[d * kRank + c], total[which][d], s);
    s *= 1.0f / static_cast<float>(B);
    const size_t o = ((static_cast<size_t>(b) * a.n_sparse + slot) * (a.seq / B) + blk) * kRank + c;
    if (which == 0)
      a.centroids[o] = s;
    else
      a.qbar[o] = s;
  }
}

// Per-head query summaries (selection per query head instead of per KV
// head): qbar_{h,t} = (1/B) sum_{i in block t} P^T q_{h,i} for every head h
// of every retrieval slot's group, written to qbar [batch][n_sparse][group]
// [nb][16].  One CTA per (block, slot x head, sequence); the same row order,
// row-group order and projection chain as the indexer, so for a group of one
// head the summary is the indexer's number.
__global__ void __launch_bounds__(kThreads) indexer_heads_kernel(const IndexerArgs a) {
  __shared__ float part[kRowGroups][kHeadDim];
  __shared__ float total[kHeadDim];
  __shared__ float proj[kHeadDim * kRank];
  const int blk = a.blk0 + static_cast<int>(blockIdx.x), b = blockIdx.z;
  const int slot = static_cast<int>(blockIdx.y) / a.group, g = static_cast<int>(blockIdx.y) % a.group;
  const int lrow = static_cast<int>(blockIdx.x) * a.block;
  const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
  const int hq = a.slot_heads[slot] * a.group + g;
  for (int e = tid; e < kHeadDim * kRank; e += kThreads) proj[e] = a.proj[e];
  float accq[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const __nv_bfloat16* qbase =
      a.q + ((static_cast<size_t>(b) * a.n_q_heads + hq) * a.rows + static_cast<size_t>(lrow)) * kHeadDim;
  sum_rows(accq, qbase, a.block, rg, cg);
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][cg * 8 + e] = accq[e];
  __syncthreads();
  if (tid < kHeadDim) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < kRowGroups; ++r) s += part[r][tid];
    total[tid] = s;
  }
  __syncthreads();
  if (tid < kRank) {
    float s = 0.f;
    for (int d = 0; d < kHeadDim; ++d) s = fmaf(proj[d * kRank + tid], total[d], s);
    s *= 1.0f / static_cast<float>(a.block);
    a.qbar[(((static_cast<size_t>(b) * a.n_sparse + slot) * a.group + g) * (a.seq / a.block) + blk) * kRank + tid] = s;
  }
}

}  // namespace

cudaError_t launch_indexer_heads(const IndexerArgs& a, cudaStream_t stream) {
  if (a.n_sparse == 0 || a.n_blocks == 0) return cudaSuccess;
  dim3 grid(a.n_blocks, a.n_sparse * a.group, a.batch);
  indexer_heads_kernel<<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(const IndexerArgs& a, cudaStream_t stream) {
  if (a.n_sparse == 0) return cudaSuccess;
  if (a.n_blocks == 0) return cudaSuccess;
  dim3 grid(a.n_blocks, a.n_sparse, a.batch);
  indexer_kernel<<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
