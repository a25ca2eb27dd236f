// KV-cache maintenance for decode: appending one token per sequence, and the
// block centroids of retrieval heads.
//
// Page "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳": in
// decode the retrieval heads are sparsified by scoring the centroids of the
// projected cached keys; the pages also describe a variant that runs full
// attention in prefill and clusters the K cache afterwards.  The centroid of
// cache block b is c_b = (1/B) sum_{j in block b} P^T k_j, defined once the
// block is complete (its B rows are all cached): the decode step only scores
// complete blocks, and the block of the newest token is always one of the
// local blocks.
//
// cache_centroids_kernel: one CTA per (complete block, KV head, sequence);
//   CTAs of non-retrieval heads leave at once.
// cache_append_kernel: one CTA per (KV head, sequence); writes the new K and V
//   rows, and when that row completes a block of a retrieval head it computes
//   that block's centroid (reading the earlier rows of the block back from the
//   cache and the new row as just written).
// Both use the summation order of the indexer (row_sum.cuh), so a centroid
// is the same fp32 number whichever of the three kernels wrote it.

#include <cuda_bf16.h>

#include "internal.cuh"
#include "row_sum.cuh"

namespace rtp {
namespace {

// Centroid of the block of B rows at `rows` (this CTA's kvh/sequence),
// written to *out (16 floats).  All 256 threads call it.
template <bool kReadOnly>
__device__ __forceinline__ void block_centroid(const __nv_bfloat16* rows, int B, const float* __restrict__ proj_g,
                                               float* out) {
  __shared__ float part[kSumRowGroups][kHeadDim];
  __shared__ float total[kHeadDim];
  __shared__ float proj[kHeadDim * kRank];
  const int tid = threadIdx.x, rg = tid >> 4, cg = tid & 15;
  for (int e = tid; e < kHeadDim * kRank; e += kSumThreads) proj[e] = proj_g[e];
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  sum_rows<kReadOnly>(acc, rows, B, rg, cg);
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][cg * 8 + e] = acc[e];
  __syncthreads();
  if (tid < kHeadDim) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < kSumRowGroups; ++g) s += part[g][tid];
    total[tid] = s;
  }
  __syncthreads();
  if (tid < kRank) {
    float s = 0.f;
    for (int d = 0; d < kHeadDim; ++d) s = fmaf(proj[d * kRank + tid], total[d], s);
    out[tid] = s * (1.0f / static_cast<float>(B));
  }
}

__global__ void __launch_bounds__(kSumThreads) cache_centroids_kernel(const CacheArgs a) {
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (a.kind[h] != KIND_SPARSE) return;
  const size_t bk = static_cast<size_t>(b) * a.n_kv_heads + h;
  const __nv_bfloat16* rows = a.kcache + (bk * a.cache_cap + static_cast<size_t>(blk) * a.block) * kHeadDim;
  const int nbc = a.cache_cap / a.block;
  block_centroid<true>(rows, a.block, a.proj, a.centroids + (bk * nbc + blk) * kRank);
}

__global__ void __launch_bounds__(kSumThreads) cache_append_kernel(const CacheArgs a) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const size_t bk = static_cast<size_t>(b) * a.n_kv_heads + h;
  const size_t row = bk * a.cache_cap + a.pos;
  // 256-byte rows: threads 0..15 copy K, 16..31 copy V, 16 bytes each
  if (tid < 32) {
    const int c = tid & 15;
    const __nv_bfloat16* src = (tid < 16 ? a.k_new : a.v_new) + bk * kHeadDim;
    __nv_bfloat16* dst = (tid < 16 ? a.kcache : a.vcache) + row * kHeadDim;
    reinterpret_cast<uint4*>(dst)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
  }
  if (a.kind[h] != KIND_SPARSE || (a.pos + 1) % a.block != 0) return;  // uniform over the CTA
  __syncthreads();  // the new K row is visible to every thread of the CTA
  const int blk = (a.pos + 1) / a.block - 1;
  const int nbc = a.cache_cap / a.block;
  const __nv_bfloat16* rows = a.kcache + (bk * a.cache_cap + static_cast<size_t>(blk) * a.block) * kHeadDim;
  // plain loads: this kernel has just written one of the rows
  block_centroid<false>(rows, a.block, a.proj, a.centroids + (bk * nbc + blk) * kRank);
}

}  // namespace

cudaError_t launch_cache_append(const CacheArgs& a, cudaStream_t stream) {
  dim3 grid(a.n_kv_heads, a.batch);
  cache_append_kernel<<<grid, kSumThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_cache_centroids(const CacheArgs& a, cudaStream_t stream) {
  if (a.n_blocks == 0) return cudaSuccess;
  dim3 grid(a.n_blocks, a.n_kv_heads, a.batch);
  cache_centroids_kernel<<<grid, kSumThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
