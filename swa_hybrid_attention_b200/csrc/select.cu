// Per-(retrieval slot, query block) block selection.
//
// Page "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳": the classic
// sparse-attention policy keeps a fixed top-k per query; the pages argue for
// a dynamic budget but give no rule, so this library states one: query block
// t scores candidate blocks 1..t-L by s_j = qbar_t . c_j, keeps the k best by
// (score desc, index asc), and adds block 0 (sink) and the L local blocks
// t-L+1..t.  If there are at most k candidates, all blocks 0..t are kept.
//
// Kernel: one CTA (256 threads) per (query block, slot, sequence).
//  1. Scores in fp32 with a fixed summation order, turned into order-
//     preserving 32-bit keys in shared memory.
//  2. Exact radix select (4 passes of 8 bits, histogram in shared memory,
//     digit search with warp shuffles) finds the key value T of the k-th
//     largest score and how many keys equal to T must be taken.
//  3. Ordered compaction: each thread owns a contiguous run of candidates;
//     a block-wide exclusive scan (warp shuffles) gives every kept block its
//     output slot, so the list comes out ascending without a sort, and ties
//     at T go to the lowest indices.
// The centroids of one (slot, sequence) are 16 fp32 per block and stay in L2.

#include "internal.cuh"
#include "select_common.cuh"

namespace rtp {
namespace {

__global__ void __launch_bounds__(kSelThreads) block_select_kernel(const SelectArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectScratch sh;
  const int t = blockIdx.x, slot = blockIdx.y, b = blockIdx.z;
  const size_t row = (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb + t;
  int32_t* out = a.sel + row * a.kmax;
  const float* C = a.centroids + (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb * kRank;
  float q[kRank];
#pragma unroll
  for (int c = 0; c < kRank; ++c) q[c] = a.qbar[row * kRank + c];
  const int n = select_blocks(q, C, t, a.topk, a.n_local, a.kmax, keys, sh, out);
  if (threadIdx.x == 0) a.cnt[row] = n;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  if (a.n_sparse == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(a.nb) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.nb, a.n_sparse, a.batch);
  block_select_kernel<<<grid, kSelThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
