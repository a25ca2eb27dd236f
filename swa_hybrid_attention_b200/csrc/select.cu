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

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.cuh"
#include "select_common.cuh"

namespace rtp {
namespace {

__global__ void __launch_bounds__(kSelThreads) block_select_kernel(const SelectArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectScratch sh;
  const int t = a.t0 + static_cast<int>(blockIdx.x), slot = blockIdx.y, b = blockIdx.z;
  const size_t row = (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb + t;
  int32_t* out = a.sel + row * a.kmax;
  const float* C =
      a.centroids + (static_cast<size_t>(b) * (a.n_sparse / a.c_group) + slot / a.c_group) * a.nb * kRank;
  float q[kRank];
#pragma unroll
  for (int c = 0; c < kRank; ++c) q[c] = a.qbar[row * kRank + c];
  const int n = select_blocks(q, C, t, a.topk, a.n_local, a.kmax, keys, sh, out);
  if (threadIdx.x == 0) a.cnt[row] = n;
}

// ------------------------------------------------------------ dynamic budget
//
// The same page argues that heads, lengths and queries need very different
// numbers of context blocks.  Rule implemented here (the library's reading):
// weights w_j = exp(beta (s_j - max s)) over the candidates, Z = sum w_j; the
// shortest prefix of the candidates in (score desc, index asc) order whose
// weights reach mass * Z, clamped to [min_k, cap]; plus sink and local blocks.
//
// Per CTA (one query block): scores -> keys (as above); max key and Z by
// fixed-order reductions; the cap best candidates (radix select, or all of
// them) are bitonic-sorted in shared memory by (key desc, index asc); a
// fixed-order scan of their weights gives the cut n*; the cut is turned back
// into a (threshold key, ties) pair and the ordered compaction of the fixed
// kernel writes the kept blocks ascending.  Every reduction has a fixed
// order, so results are bit-reproducible.

__device__ __forceinline__ float key_score(uint32_t key) {  // inverse of order_key
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

struct DynScratch {
  unsigned long long srt[kDynMaxCap];  // (key << 32) | ~index, sorted descending
  float red[kSelThreads / 32];
  float warp_excl[kSelThreads / 32];
  uint32_t kred[kSelThreads / 32];
  int cut, first_eq;
};

// Sum over the CTA in a fixed order (butterfly inside each warp, lane 0's
// value per warp, then the warps in index order).  Called by all threads.
__device__ __forceinline__ float cta_sum_fixed(float v, DynScratch& d) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) d.red[warp] = v;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) tot += d.red[w];
  __syncthreads();
  return tot;
}

__device__ __forceinline__ uint32_t cta_max_u32(uint32_t v, DynScratch& d) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
  if (lane == 0) d.kred[warp] = v;
  __syncthreads();
  uint32_t m = 0;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) m = max(m, d.kred[w]);
  __syncthreads();
  return m;
}

// Exclusive prefix sum of one float per thread, in thread order, fixed
// association (shuffle scan inside warps, then over the warp totals).
__device__ __forceinline__ float cta_exclusive_scan_fixed(float v, DynScratch& d) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) d.red[warp] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    float acc = 0.f;
    for (int w = 0; w < kSelThreads / 32; ++w) {
      d.warp_excl[w] = acc;
      acc += d.red[w];
    }
  }
  __syncthreads();
  const float r = d.warp_excl[warp] + (incl - v);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSelThreads) block_select_dynamic_kernel(const SelectArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectScratch sh;
  __shared__ DynScratch d;
  const int tid = threadIdx.x;
  const int t = a.t0 + static_cast<int>(blockIdx.x), slot = blockIdx.y, b = blockIdx.z;
  const size_t row = (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb + t;
  int32_t* out = a.sel + row * a.kmax;
  const float* C = a.centroids + (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb * kRank;
  const int ncand = t - a.n_local > 0 ? t - a.n_local : 0;  // candidates are blocks 1..ncand
  if (ncand == 0) {  // only sink and local blocks exist: blocks 0..t
    for (int e = tid; e < a.kmax; e += kSelThreads) out[e] = e <= t ? e : -1;
    if (tid == 0) a.cnt[row] = t + 1;
    return;
  }
  float q[kRank];
#pragma unroll
  for (int c = 0; c < kRank; ++c) q[c] = a.qbar[row * kRank + c];
  // 1. scores -> order keys
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
  // 2. max score and Z = sum of the weights (each thread a contiguous run)
  const int per = (ncand + kSelThreads - 1) / kSelThreads;
  const int x0 = min(ncand, tid * per), x1 = min(ncand, x0 + per);
  uint32_t kmax_l = 0;
  for (int x = x0; x < x1; ++x) kmax_l = max(kmax_l, keys[x]);
  const float smax = key_score(cta_max_u32(kmax_l, d));
  float zl = 0.f;
  for (int x = x0; x < x1; ++x) zl += exp2f(a.beta_log2 * (key_score(keys[x]) - smax));
  const float Z = cta_sum_fixed(zl, d);
  // 3. the cap best candidates, sorted by (key desc, index asc)
  const int m = min(ncand, a.topk);
  int nstar = 0;
  if (m > 0) {
    int P = 1;
    while (P < m) P <<= 1;
    if (ncand > m) {
      uint32_t T, need;
      radix_threshold<kSelThreads>(keys, ncand, m, sh, T, need);
      ordered_select<kSelThreads>(keys, ncand, T, need, sh, [&](int r, int x) {
        d.srt[r] = (static_cast<unsigned long long>(keys[x]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(x));
      });
    } else {
      for (int x = tid; x < m; x += kSelThreads)
        d.srt[x] = (static_cast<unsigned long long>(keys[x]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(x));
    }
    for (int e = m + tid; e < P; e += kSelThreads) d.srt[e] = 0ull;  // sorts last
    if (tid == 0) {
      d.cut = 0x7FFFFFFF;
      d.first_eq = 0x7FFFFFFF;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < P; i += kSelThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long u = d.srt[i], w = d.srt[ixj];
            if (((i & k) == 0) ? (u < w) : (u > w)) {
              d.srt[i] = w;
              d.srt[ixj] = u;
            }
          }
        }
        __syncthreads();
      }
    }
    // 4. prefix sums of the sorted weights; the first prefix >= mass * Z
    const int rper = (m + kSelThreads - 1) / kSelThreads;  // <= 4
    const int r0 = min(m, tid * rper), r1 = min(m, r0 + rper);
    float wl[4];
    float tot = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      wl[e] = 0.f;
      if (r0 + e < r1) {
        wl[e] = exp2f(a.beta_log2 * (key_score(static_cast<uint32_t>(d.srt[r0 + e] >> 32)) - smax));
        tot += wl[e];
      }
    }
    float acc = cta_exclusive_scan_fixed(tot, d);
    const float thr = a.mass * Z;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (r0 + e < r1) {
        acc += wl[e];
        if (acc >= thr) {
          atomicMin(&d.cut, r0 + e + 1);
          break;
        }
      }
    }
    __syncthreads();
    nstar = d.cut == 0x7FFFFFFF ? m : d.cut;
    nstar = max(nstar, min(a.min_k, m));
    nstar = min(nstar, m);
    // 5. the cut as (threshold key, ties at it), then the ordered compaction
    const uint32_t Tc = static_cast<uint32_t>(d.srt[nstar - 1] >> 32);
    for (int r = tid; r < nstar; r += kSelThreads)
      if (static_cast<uint32_t>(d.srt[r] >> 32) == Tc) atomicMin(&d.first_eq, r);
    __syncthreads();
    const uint32_t need_c = static_cast<uint32_t>(nstar - d.first_eq);
    ordered_select<kSelThreads>(keys, ncand, Tc, need_c, sh, [&](int r, int x) { out[1 + r] = x + 1; });
  }
  if (tid == 0) {
    out[0] = 0;
    a.cnt[row] = 1 + nstar + a.n_local;
  }
  for (int e = tid; e < a.n_local; e += kSelThreads) out[1 + nstar + e] = t - a.n_local + 1 + e;
  for (int e = 1 + nstar + a.n_local + tid; e < a.kmax; e += kSelThreads) out[e] = -1;
}

// ------------------------------------------------------------ row-max scores
//
// The same page's criticism of one fixed policy also leaves open how a query
// block should score a candidate.  Besides the mean (the summary qbar_t), the
// library offers the largest low-rank logit over the block's rows:
//   s_j = max_{i in block t} u_i . c_j,   u_i = P^T sum_{h in group} q_{h,i},
// so that one query row pointing at a block is enough to keep it.  Selection
// rule and output are those of the fixed policy (top-k by score desc, index
// asc; sink and local blocks added).
//
// Per CTA (one query block):
//  1. u_i of the block's rows into shared memory (16 threads per row sum the
//     group's heads over 8 dims each and project; the 16 partial dot
//     products of each rank are added by a fixed reduce-scatter tree, lane
//     c ending with rank c).
//  2. Approximate scores on the tensor cores: the (rows x 16) . (16 x 8
//     candidates) products are mma.sync m16n8k16 on fp16 operands (u scaled
//     by an exact power of two su so that every entry lies below 2^14; c as
//     is), fp32 accumulation, the maximum over rows taken from the
//     accumulator fragments.  Rounding each operand to fp16 costs at most
//     2^-11 of it (plus 2^-25 below fp16's normal range), so an approximate
//     row maximum a_j is within
//       E = 2^-9 max|su u_i| max|c_j| + 2^-22 (max|su u_i| + max|c_j|)
//     (about a 2x margin, the accumulation's rounding included) of su s_j,
//     s_j the exact fp32 score of step 4.  If some |c_j| reaches 2^15 (fp16
//     could overflow) no approximation is used: every candidate goes to step
//     4.
//  3. A lower bound b of the k-th largest approximate score a_(k) (two radix
//     passes: the low edge of its 16-bit key bin).  At least k candidates
//     have su s >= a_(k) - E >= b - E, so a candidate with a_j < b - 2E has
//     su s_j < b - E and is not among the k best: only the others (the k
//     best and those within 2E of the bin, 2^-7 relative wide) need their
//     exact score.
//  4. Those candidates (listed in ascending order) are re-scored exactly
//     (fp32, the 16-term dot product in two fixed-order chains of 8 then
//     their sum, maximum over rows: the score every earlier version of this
//     kernel computed for every candidate).
//  5. The fixed kernel's radix select and ordered compaction over the listed
//     candidates' exact keys: the same selection as exact scores for every
//     candidate.

// u . c with ranks 0-7 and 8-15 in two fma chains (fixed order), added at
// the end: half the dependent latency of one 16-long chain.
__device__ __forceinline__ float score16_two_chains(const float (&u)[kRank], const float4 (&c)[4]) {
  float s0 = u[0] * c[0].x, s1 = u[8] * c[2].x;
  s0 = fmaf(u[1], c[0].y, s0);
  s1 = fmaf(u[9], c[2].y, s1);
  s0 = fmaf(u[2], c[0].z, s0);
  s1 = fmaf(u[10], c[2].z, s1);
  s0 = fmaf(u[3], c[0].w, s0);
  s1 = fmaf(u[11], c[2].w, s1);
  s0 = fmaf(u[4], c[1].x, s0);
  s1 = fmaf(u[12], c[3].x, s1);
  s0 = fmaf(u[5], c[1].y, s0);
  s1 = fmaf(u[13], c[3].y, s1);
  s0 = fmaf(u[6], c[1].z, s0);
  s1 = fmaf(u[14], c[3].z, s1);
  s0 = fmaf(u[7], c[1].w, s0);
  s1 = fmaf(u[15], c[3].w, s1);
  return s0 + s1;
}

struct RowmaxScratch {
  // projector row 8 cg + e at projv[e][cg][0..16), rows padded to 20 words:
  // the 16-byte loads of the 8 lanes of a phase (cg = 0..7 and 8..15) hit
  // distinct banks (a dense [128][16] layout puts all 16 lanes of a row in
  // one bank: a 16-way conflict on every load)
  float projv[8][16][20];
  // block <= 128 rows, padded to 20 words so that the exact re-score's four
  // threads of a candidate (rows 4i .. 4i+3 at a time) read distinct banks
  float u[128][20];
  float red[2][kSelThreads / 32];
  int n_poss;
};

// fp16 pair (x in the low half), round to nearest.
__device__ __forceinline__ uint32_t f16x2_bits(float x, float y) {
  const __half2 v = __floats2half2_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void mma_m16n8k16_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}


__global__ void __launch_bounds__(kSelThreads, 2) block_select_rowmax_kernel(const SelectArgs a) {
  extern __shared__ uint32_t keys[];  // [nb] order keys, then [nb] candidates to re-score
  __shared__ SelectScratch sh;
  __shared__ __align__(16) RowmaxScratch rs;
  const int t = a.t0 + static_cast<int>(blockIdx.x), slot = blockIdx.y, b = blockIdx.z;
  const size_t row = (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb + t;
  int32_t* out = a.sel + row * a.kmax;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (const int n = select_without_scores(t, a.topk, a.n_local, a.kmax, out); n >= 0) {
    if (tid == 0) a.cnt[row] = n;
    return;
  }
  const int ncand = t - a.n_local;
  const int kvh = a.slot_heads[slot];
  for (int e = tid; e < kHeadDim * kRank; e += kSelThreads) {
    const int d = e / kRank, c = e % kRank;
    rs.projv[d & 7][d >> 3][c] = a.proj[e];
  }
  __syncthreads();
  // 1. u_i
  {
    const int rg = tid >> 4, cg = tid & 15;
    for (int i0 = 0; i0 < a.block; i0 += kSelThreads / 16) {
      const int i = i0 + rg;
      const size_t qrow = static_cast<size_t>(t) * a.block + i - a.q_row0;
      float sum[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      // the heads' loads are issued 8 at a time (all in flight), then added
      // in head order
      const __nv_bfloat16* q0 =
          a.q + ((static_cast<size_t>(b) * a.n_q_heads + kvh * a.group) * a.q_slab + qrow) * kHeadDim + 8 * cg;
      const size_t head_stride = static_cast<size_t>(a.q_slab) * kHeadDim;
      for (int h0 = 0; h0 < a.group; h0 += 8) {
        uint4 raw[8];
#pragma unroll
        for (int hh = 0; hh < 8; ++hh)
          if (h0 + hh < a.group) raw[hh] = *reinterpret_cast<const uint4*>(q0 + (h0 + hh) * head_stride);
#pragma unroll
        for (int hh = 0; hh < 8; ++hh) {
          if (h0 + hh < a.group) {
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[hh]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(p2[e]);
              sum[2 * e] += f.x;
              sum[2 * e + 1] += f.y;
            }
          }
        }
      }
      // rank c: sum over e of proj[8 cg + e][c] * sum[e] (fma chain in e order)
      float v[kRank];
#pragma unroll
      for (int c = 0; c < kRank; ++c) v[c] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4* pr = reinterpret_cast<const float4*>(rs.projv[e][cg]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 p4 = pr[w];
          v[4 * w] = fmaf(p4.x, sum[e], v[4 * w]);
          v[4 * w + 1] = fmaf(p4.y, sum[e], v[4 * w + 1]);
          v[4 * w + 2] = fmaf(p4.z, sum[e], v[4 * w + 2]);
          v[4 * w + 3] = fmaf(p4.w, sum[e], v[4 * w + 3]);
        }
      }
      // reduce-scatter over the row's 16 lanes (a fixed tree): at each step a
      // lane keeps the half of its ranks that matches its lane bit and adds
      // the partner's copy of that half, so lane cg ends with rank cg summed
      // over all 16 lanes
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool up = (cg & 8) != 0;
        const float send = up ? v[j] : v[j + 8], keep = up ? v[j + 8] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool up = (cg & 4) != 0;
        const float send = up ? v[j] : v[j + 4], keep = up ? v[j + 4] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool up = (cg & 2) != 0;
        const float send = up ? v[j] : v[j + 2], keep = up ? v[j + 2] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
      {
        const bool up = (cg & 1) != 0;
        const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
        rs.u[i][cg] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      }
    }
  }
  __syncthreads();
  const float* C = a.centroids + (static_cast<size_t>(b) * a.n_sparse + slot) * a.nb * kRank;
  const int mtiles = a.block / 16;  // 16-row tiles of u (4 or 8)
  // the largest |u_i| sets u's scale for the fp16 products: su = 2^(14 - e)
  // with max|u_i| in [2^(e-1), 2^e), so that every su u_i,d lies below 2^14
  // (scaling by a power of two is exact; scores and bounds below are all in
  // this scaled unit, so the comparisons do not change)
  {
    float un2 = 0.f;
    if (tid < a.block) {
#pragma unroll
      for (int c = 0; c < kRank; ++c) un2 = fmaf(rs.u[tid][c], rs.u[tid][c], un2);
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) un2 = fmaxf(un2, __shfl_xor_sync(0xffffffffu, un2, off));
    if (lane == 0) rs.red[0][warp] = un2;
  }
  __syncthreads();
  float u2 = 0.f;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) u2 = fmaxf(u2, rs.red[0][w]);
  const float umax = sqrtf(u2) * 1.001f;
  int ue = 0;
  frexpf(umax, &ue);
  const float su = umax > 0.f ? ldexpf(1.f, 14 - ue) : 1.f;
  // 2. approximate scores, 8 candidates per warp step: the
  // (rows x 16) . (16 x 8 candidates) products as mma.sync m16n8k16 on fp16
  // operands (su u and c), fp32 accumulation.  Fragments (g = lane / 4,
  // q = lane % 4): A rows g and g+8 of the tile, dims 2q, 2q+1 and 2q+8,
  // 2q+9; B column g (candidate 8 gi + g), the same dims; D rows g and g+8,
  // candidates 2q and 2q+1.
  float cn2_max = 0.f;
  {
    const int g = lane >> 2, q = lane & 3;
    uint32_t af[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      if (mt < mtiles) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = 16 * mt + g + 8 * (e & 1), k = 2 * q + 8 * (e >> 1);
          af[mt][e] = f16x2_bits(su * rs.u[r][k], su * rs.u[r][k + 1]);
        }
      }
    }
    const int ngroups = (ncand + 7) / 8;
    for (int gi = warp; gi < ngroups; gi += kSelThreads / 32) {
      const int xg = 8 * gi + g;
      const float* cp = C + static_cast<size_t>(min(xg, ncand - 1) + 1) * kRank;
      const float2 c0 = __ldg(reinterpret_cast<const float2*>(cp + 2 * q));
      const float2 c1 = __ldg(reinterpret_cast<const float2*>(cp + 2 * q + 8));
      const uint32_t b0 = f16x2_bits(c0.x, c0.y), b1 = f16x2_bits(c1.x, c1.y);
      float n2 = c0.x * c0.x + c0.y * c0.y + c1.x * c1.x + c1.y * c1.y;
      n2 += __shfl_xor_sync(0xffffffffu, n2, 1);
      n2 += __shfl_xor_sync(0xffffffffu, n2, 2);
      if (xg < ncand) cn2_max = fmaxf(cn2_max, n2);
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        if (mt < mtiles) {
          float d[4] = {0.f, 0.f, 0.f, 0.f};
          mma_m16n8k16_f16(d, af[mt], b0, b1);
          m0 = fmaxf(m0, fmaxf(d[0], d[2]));
          m1 = fmaxf(m1, fmaxf(d[1], d[3]));
        }
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
      }
      if (g == 0) {
        const int x0 = 8 * gi + 2 * q;
        if (x0 < ncand) keys[x0] = order_key(m0);
        if (x0 + 1 < ncand) keys[x0 + 1] = order_key(m1);
      }
    }
  }
  // the bound E (scaled unit) from the largest |su u_i| and |c_j|
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) cn2_max = fmaxf(cn2_max, __shfl_xor_sync(0xffffffffu, cn2_max, off));
  if (lane == 0) rs.red[1][warp] = cn2_max;
  __syncthreads();
  float c2 = 0.f;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) c2 = fmaxf(c2, rs.red[1][w]);
  const float cmax = sqrtf(c2) * 1.001f, sumax = su * umax;
  // a centroid entry at or above 2^15 could overflow fp16 (65504): then no
  // approximate score is trusted and every candidate is scored exactly
  const bool trusted = cmax < 32768.f;
  const float E = 0x1p-9f * sumax * cmax + 0x1p-22f * (sumax + cmax);
  // 3. a lower bound of the k-th largest approximate score (its 16-bit key
  // bin: within 2^-7 of it), and the candidates within 2E of that bound
  uint32_t T, need;
  radix_threshold<kSelThreads>(keys, ncand, a.topk, sh, T, need, 2);
  const float theta = trusted ? key_score(T) - 2.0f * E : -INFINITY;
  uint32_t* poss = keys + a.nb;
  {
    const int per = (ncand + kSelThreads - 1) / kSelThreads;
    const int x0 = min(ncand, tid * per), x1 = min(ncand, x0 + per);
    uint32_t own = 0;
    for (int x = x0; x < x1; ++x) own += !trusted || key_score(keys[x]) >= theta;
    uint32_t at = static_cast<uint32_t>(block_exclusive_scan<kSelThreads>(own, sh));
    if (tid == kSelThreads - 1) rs.n_poss = static_cast<int>(at + own);
    for (int x = x0; x < x1; ++x)
      if (!trusted || key_score(keys[x]) >= theta) poss[at++] = static_cast<uint32_t>(x);
  }
  __syncthreads();
  // 4. exact scores of those: four threads per candidate, a quarter of the
  // rows each (the maximum does not depend on how the rows are grouped)
  {
    const int n_poss = rs.n_poss, sub = tid & 3, rows_per = a.block / 4;
    for (int p0 = 0; p0 < n_poss; p0 += kSelThreads / 4) {  // sub s takes rows 4i + s
      const int p = p0 + (tid >> 2);
      float best = -INFINITY;
      int x = 0;
      if (p < n_poss) {
        x = static_cast<int>(poss[p]);
        float4 cv[4];
        const float4* c4 = reinterpret_cast<const float4*>(C + static_cast<size_t>(x + 1) * kRank);
#pragma unroll
        for (int w = 0; w < 4; ++w) cv[w] = __ldg(c4 + w);
#pragma unroll 4
        for (int ii = 0; ii < rows_per; ++ii) {
          const float4* u4 = reinterpret_cast<const float4*>(rs.u[4 * ii + sub]);
          const float4 u0 = u4[0], u1 = u4[1], u2v = u4[2], u3 = u4[3];
          const float uq[kRank] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w,
                                   u2v.x, u2v.y, u2v.z, u2v.w, u3.x, u3.y, u3.z, u3.w};
          best = fmaxf(best, score16_two_chains(uq, cv));
        }
      }
      best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 1));
      best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 2));
      if (sub == 0 && p < n_poss) keys[p] = order_key(best);  // keys[p]: candidate poss[p]
    }
  }
  __syncthreads();
  // 5. the k best of the re-scored candidates (the others cannot be): radix
  // select and ordered compaction over their exact keys; poss is ascending,
  // so the output is ascending and ties go to the lower block
  {
    const int n_poss = rs.n_poss;
    uint32_t T2, need2;
    radix_threshold<kSelThreads>(keys, n_poss, a.topk, sh, T2, need2);
    ordered_select<kSelThreads>(keys, n_poss, T2, need2, sh,
                                [&](int r, int p) { out[1 + r] = static_cast<int32_t>(poss[p]) + 1; });
    if (tid == 0) out[0] = 0;
    for (int m = tid; m < a.n_local; m += kSelThreads) out[1 + a.topk + m] = t - a.n_local + 1 + m;
    for (int e = 1 + a.topk + a.n_local + tid; e < a.kmax; e += kSelThreads) out[e] = -1;
    if (tid == 0) a.cnt[row] = 1 + a.topk + a.n_local;
  }
}

}  // namespace

cudaError_t launch_select_dynamic(const SelectArgs& a, cudaStream_t stream) {
  if (a.n_sparse == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(a.nb) * sizeof(uint32_t);
  if (smem + sizeof(DynScratch) + sizeof(SelectScratch) > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(block_select_dynamic_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (a.n_rows == 0) return cudaSuccess;
  dim3 grid(a.n_rows, a.n_sparse, a.batch);
  block_select_dynamic_kernel<<<grid, kSelThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_select_rowmax(const SelectArgs& a, cudaStream_t stream) {
  if (a.n_sparse == 0) return cudaSuccess;
  const size_t smem = 2 * static_cast<size_t>(a.nb) * sizeof(uint32_t);
  if (smem + sizeof(RowmaxScratch) + sizeof(SelectScratch) > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(block_select_rowmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (a.n_rows == 0) return cudaSuccess;
  dim3 grid(a.n_rows, a.n_sparse, a.batch);
  block_select_rowmax_kernel<<<grid, kSelThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  if (a.n_sparse == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(a.nb) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (a.n_rows == 0) return cudaSuccess;
  dim3 grid(a.n_rows, a.n_sparse, a.batch);
  block_select_kernel<<<grid, kSelThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
