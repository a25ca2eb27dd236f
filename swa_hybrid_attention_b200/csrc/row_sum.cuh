// Column sums of consecutive 128-wide bf16 rows, the first step of a block
// centroid (c_b = (1/B) sum_j P^T k_j = (1/B) P^T sum_j k_j by linearity).
//
// Thread layout shared by every kernel that uses it: 256 threads, thread
// (rg = tid / 16, cg = tid % 16) reads 16 bytes (8 bf16, columns 8cg..8cg+7)
// of rows rg, rg + 16, rg + 32, ... and adds them into its 8 accumulators in
// that row order.  The kernels then add the 16 row groups' partial sums in
// group order 0..15 and project with one fmaf chain over d = 0..127, so every
// centroid they write is the same fp32 number for the same keys.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace rtp {

constexpr int kSumThreads = 256;
constexpr int kSumRowGroups = kSumThreads / 16;

__device__ __forceinline__ void accum_row8(float (&acc)[8], const uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    acc[2 * e] += f.x;
    acc[2 * e + 1] += f.y;
  }
}

// kReadOnly: the rows are not written by the running kernel, so they may be
// read through the non-coherent (read-only) path.
template <bool kReadOnly>
__device__ __forceinline__ uint4 load_row16(const uint4* p) {
  if constexpr (kReadOnly) return __ldg(p);
  return *p;
}

// Sum `rows` consecutive rows starting at `base` into acc (this thread's 8
// columns), 4 loads in flight per thread.
template <bool kReadOnly = true>
__device__ __forceinline__ void sum_rows(float (&acc)[8], const __nv_bfloat16* base, int rows, int rg, int cg) {
  const uint4* p = reinterpret_cast<const uint4*>(base) + cg;
  int r = rg;
  for (; r + 3 * kSumRowGroups < rows; r += 4 * kSumRowGroups) {
    uint4 v0 = load_row16<kReadOnly>(p + static_cast<size_t>(r) * 16);
    uint4 v1 = load_row16<kReadOnly>(p + static_cast<size_t>(r + kSumRowGroups) * 16);
    uint4 v2 = load_row16<kReadOnly>(p + static_cast<size_t>(r + 2 * kSumRowGroups) * 16);
    uint4 v3 = load_row16<kReadOnly>(p + static_cast<size_t>(r + 3 * kSumRowGroups) * 16);
    accum_row8(acc, v0);
    accum_row8(acc, v1);
    accum_row8(acc, v2);
    accum_row8(acc, v3);
  }
  for (; r < rows; r += kSumRowGroups) accum_row8(acc, load_row16<kReadOnly>(p + static_cast<size_t>(r) * 16));
}

}  // namespace rtp
