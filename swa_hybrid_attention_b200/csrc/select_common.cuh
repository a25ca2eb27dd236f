// Block selection shared by the prefill selection kernel and the decode
// step: sink + top-k candidates by (score desc, index asc) + local blocks.
#pragma once
#include <cstdint>

#include "internal.cuh"

namespace rtp {

constexpr int kSelThreads = 256;

template <int NT>
struct SelectScratchT {
  uint32_t hist[256];
  unsigned long long warp_sums[NT / 32];
  uint32_t digit, need;
};
using SelectScratch = SelectScratchT<kSelThreads>;

// Order-preserving map float -> uint32 (larger float, larger key); -0 and +0
// map to the same key.
__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v, SelectScratchT<NT>& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    unsigned long long y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) sh.warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < NT / 32 ? sh.warp_sums[lane] : 0ull;
    unsigned long long wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      unsigned long long y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < NT / 32) sh.warp_sums[lane] = wi - w;  // exclusive
  }
  __syncthreads();
  return sh.warp_sums[warp] + incl - v;
}

// Radix select, most significant byte first, over keys[0, n) in shared
// memory (1 <= k <= n): T = the k-th largest key and `need` = how many keys
// equal to T belong to the k largest.  Called by all NT threads of the CTA.
// With passes < 4 only the top 8 * passes bits are resolved: T is then the
// smallest key of the bin that holds the k-th largest (a lower bound of it)
// and `need` counts within that bin.
template <int NT>
__device__ inline void radix_threshold(const uint32_t* keys, int n, int k, SelectScratchT<NT>& sh, uint32_t& T,
                                       uint32_t& need_out, int passes = 4) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, need = static_cast<uint32_t>(k);
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int e = tid; e < 256; e += NT) sh.hist[e] = 0;
    __syncthreads();
    // Scores cluster in a few bins of the high bytes, so the lanes of a warp
    // that share a bin add their count with one atomic (match + popcount)
    // instead of queueing on the same shared-memory word.  The loop bound is
    // uniform: every lane takes part in every match.
    for (int x0 = 0; x0 < n; x0 += NT) {
      const int x = x0 + tid;
      uint32_t bin = 0xFFFFFFFFu;
      if (x < n) {
        const uint32_t key = keys[x];
        if ((key & hi_mask) == prefix) bin = (key >> shift) & 255u;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xFFFFFFFFu && (tid & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t cnt8[8], own = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cnt8[e] = sh.hist[8 * tid + e];
        own += cnt8[e];
      }
      uint32_t incl = own;  // count in bins of lanes >= this lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
        if (tid + off < 32) incl += y;
      }
      const uint32_t above = incl - own;
      if (above < need && need <= incl) {
        uint32_t acc = above;
        for (int e = 7; e >= 0; --e) {
          if (acc + cnt8[e] >= need) {
            sh.digit = static_cast<uint32_t>(8 * tid + e);
            sh.need = need - acc;
            break;
          }
          acc += cnt8[e];
        }
      }
      __syncwarp();
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    need = sh.need;
    __syncthreads();
  }
  T = prefix;
  need_out = need;
}

// Ordered compaction of the k largest keys found by radix_threshold: every
// key > T, and the first `need` keys equal to T in array order (so ties go
// to the lower position).  emit(r, x) is called for the selected positions x
// in increasing order, r = 0, 1, ... their rank among the selected.
template <int NT, class Emit>
__device__ inline void ordered_select(const uint32_t* keys, int n, uint32_t T, uint32_t need, SelectScratchT<NT>& sh,
                                      Emit emit) {
  const int tid = threadIdx.x;
  const int per = (n + NT - 1) / NT;
  const int x0 = min(n, tid * per), x1 = min(n, x0 + per);
  uint32_t n_gt = 0, n_eq = 0;
  for (int x = x0; x < x1; ++x) {
    const uint32_t key = keys[x];
    n_gt += key > T;
    n_eq += key == T;
  }
  const unsigned long long excl =
      block_exclusive_scan<NT>((static_cast<unsigned long long>(n_gt) << 32) | n_eq, sh);
  uint32_t gt_before = static_cast<uint32_t>(excl >> 32), eq_before = static_cast<uint32_t>(excl & 0xFFFFFFFFu);
  for (int x = x0; x < x1; ++x) {
    const uint32_t key = keys[x];
    if (key > T) {
      emit(static_cast<int>(gt_before + min(eq_before, need)), x);
      ++gt_before;
    } else if (key == T) {
      if (eq_before < need) emit(static_cast<int>(gt_before + eq_before), x);
      ++eq_before;
    }
  }
}

// Score of one centroid row (fixed fma order over the 16 ranks).
__device__ __forceinline__ float score16(const float (&q)[kRank], const float4 (&v)[4]) {
  float s = q[0] * v[0].x;
  s = fmaf(q[1], v[0].y, s);
  s = fmaf(q[2], v[0].z, s);
  s = fmaf(q[3], v[0].w, s);
  s = fmaf(q[4], v[1].x, s);
  s = fmaf(q[5], v[1].y, s);
  s = fmaf(q[6], v[1].z, s);
  s = fmaf(q[7], v[1].w, s);
  s = fmaf(q[8], v[2].x, s);
  s = fmaf(q[9], v[2].y, s);
  s = fmaf(q[10], v[2].z, s);
  s = fmaf(q[11], v[2].w, s);
  s = fmaf(q[12], v[3].x, s);
  s = fmaf(q[13], v[3].y, s);
  s = fmaf(q[14], v[3].z, s);
  s = fmaf(q[15], v[3].w, s);
  return s;
}

// Steps 2 and 3 of a selection once the candidates' order keys are in
// shared memory (ncand > topk >= 1): the topk-th largest key, then the
// ordered compaction into out[1..topk], plus the sink and the local blocks.
// Must be called by all kSelThreads threads of the CTA.
__device__ inline int select_from_keys(const uint32_t* keys, int ncand, int t, int topk, int n_local, int kmax,
                                       SelectScratch& sh, int32_t* out) {
  const int tid = threadIdx.x;
  uint32_t T, need;
  radix_threshold<kSelThreads>(keys, ncand, topk, sh, T, need);
  ordered_select<kSelThreads>(keys, ncand, T, need, sh, [&](int r, int x) { out[1 + r] = x + 1; });
  if (tid == 0) out[0] = 0;
  for (int m = tid; m < n_local; m += kSelThreads) out[1 + topk + m] = t - n_local + 1 + m;
  for (int e = 1 + topk + n_local + tid; e < kmax; e += kSelThreads) out[e] = -1;
  return 1 + topk + n_local;
}

// The selections that need no scores: every block 0..t when there are at
// most topk candidates, or only the sink and local blocks when topk is 0.
// Returns the count, or -1 if scores are needed.
__device__ inline int select_without_scores(int t, int topk, int n_local, int kmax, int32_t* out) {
  const int tid = threadIdx.x;
  const int ncand = t - n_local > 0 ? t - n_local : 0;
  if (ncand <= topk) {
    const int n = t + 1;
    for (int e = tid; e < kmax; e += kSelThreads) out[e] = e < n ? e : -1;
    return n;
  }
  if (topk == 0) {
    for (int e = tid; e < kmax; e += kSelThreads) out[e] = e == 0 ? 0 : (e <= n_local ? t - n_local + e : -1);
    return 1 + n_local;
  }
  return -1;
}

// Selects the blocks of query block t.  Must be called by all kSelThreads
// threads of the CTA.  q: the query summary (16 fp32); C: centroids of this
// (slot, sequence), [>= t-n_local+1][16] fp32; keys: shared scratch of at
// least max(0, t-n_local) words.  Writes out[0..kmax) (ascending, -1 padded)
// and returns the number of entries used.
__device__ inline int select_blocks(const float (&q)[kRank], const float* C, int t, int topk, int n_local, int kmax,
                                    uint32_t* keys, SelectScratch& sh, int32_t* out) {
  const int tid = threadIdx.x;
  const int ncand = t - n_local > 0 ? t - n_local : 0;  // candidates are blocks 1..ncand
  // (top-k 0: sink and local blocks only; the radix select needs k >= 1)
  if (const int n = select_without_scores(t, topk, n_local, kmax, out); n >= 0) return n;
  // 1. scores -> order keys.  Four candidates per round with all their
  // loads issued before any use, so a thread keeps 16 independent 16-byte
  // loads in flight.
  for (int x0 = tid; x0 < ncand; x0 += 4 * kSelThreads) {
    float4 v[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int x = min(x0 + u * kSelThreads, ncand - 1);
      const float4* c4 = reinterpret_cast<const float4*>(C + static_cast<size_t>(x + 1) * kRank);
#pragma unroll
      for (int w = 0; w < 4; ++w) v[u][w] = __ldg(c4 + w);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int x = x0 + u * kSelThreads;
      if (x < ncand) keys[x] = order_key(score16(q, v[u]));
    }
  }
  __syncthreads();
  return select_from_keys(keys, ncand, t, topk, n_local, kmax, sh, out);
}

}  // namespace rtp
